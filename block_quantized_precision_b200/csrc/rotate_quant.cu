// rotate_quant.cu -- fused rotation + dynamic block quantization.
//
// Method: "MindIE-SD quantization", FA量化 / 技术特点: Q and K are multiplied
// by an orthogonal rotation, then Q/K/V are quantized per block of tokens
// (Q 128, K/V 256) to float8_e4m3fn; symmetric INT8 per "INT8 量化算子",
// 对称量化 (scale = max|x| / 127, code = round(x / scale)).
//
// Numerics are fixed so that codes and scales are bit-reproducible:
//   y[j]  = float32 FMA chain over k = 0..D-1 ascending, from +0
//   amax  = max |y| over the block (exact)
//   scale = amax / qmax (IEEE float32 division)
//   code  = RNE(y / scale) (IEEE float32 division; INT8 clamped to +-127,
//           e4m3 via the saturating round-to-nearest-even conversion)
//
// Two kernels:
//   rotq_kernel   (R given): FP32-FMA bound. Persistent CTAs keep R (D x D
//                 float32) in shared memory and walk over blocks; each CTA
//                 stages one block of x transposed in shared memory and
//                 computes y with an 8-column register tile per thread.
//   quant_kernel  (no R): HBM bound. One CTA per block; 16-byte loads, the
//                 block max by warp shuffles, 8- or 16-byte code stores.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "qattn_device.cuh"
#include "qattn_internal.h"

namespace qattn {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ void unpack8(uint4 v, bool is_bf16, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (is_bf16) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    } else {
      f[2 * i] = f16_bits_to_f32(w[i] & 0xFFFFu);
      f[2 * i + 1] = f16_bits_to_f32(w[i] >> 16);
    }
  }
}

// Code byte of v = y / scale (scale > 0).
template <bool kInt8>
__device__ __forceinline__ uint32_t code_of(float y, float scale) {
  const float v = __fdiv_rn(y, scale);
  if constexpr (kInt8) {
    int c = __float2int_rn(v);
    c = max(-127, min(127, c));
    return static_cast<uint32_t>(c) & 0xFFu;
  } else {
    return cvt_e4m3x2(v, 0.0f) & 0xFFu;
  }
}

__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < kThreads / 32; ++i) m = fmaxf(m, red[i]);
  __syncthreads();  // red[] may be reused
  return m;
}

// Element offset of token n of head (b, h), channel 0.
__device__ __forceinline__ int64_t row_offset(int layout, int H, int N, int D, int b, int h,
                                              int n) {
  return layout == 0 ? ((static_cast<int64_t>(b) * H + h) * N + n) * D
                     : ((static_cast<int64_t>(b) * N + n) * H + h) * D;
}

// ---------------------------------------------------------------------------
// With rotation
// ---------------------------------------------------------------------------

// Thread tile: kRows rows x 8 columns of y. Column group cg = tid % (D/8),
// row group rg = tid / (D/8); rows rg*kRPT .. rg*kRPT + kRPT - 1.
template <int D, int T, bool kInt8>
__global__ void __launch_bounds__(kThreads, 1)
    rotq_kernel(const uint16_t* __restrict__ x, int is_bf16, int layout, int B, int H, int N,
                const float* __restrict__ rot, uint8_t* __restrict__ codes,
                float* __restrict__ scales) {
  constexpr int kCG = D / 8;               // column groups
  constexpr int kRG = kThreads / kCG;      // row groups
  constexpr int kRPT = T / kRG;            // rows per thread
  constexpr int kXS = T + 4;               // padded row stride of the transposed x tile
  static_assert(kRPT % 4 == 0 && kRPT >= 4, "row tile");
  extern __shared__ __align__(16) float smem[];
  float* sR = smem;                        // [D][D]
  float* sX = smem + D * D;                // [D][kXS]: sX[k * kXS + r] = x[r][k]
  __shared__ float red[kThreads / 32];

  const int tid = threadIdx.x;
  for (int i = tid; i < D * D / 4; i += kThreads)
    reinterpret_cast<float4*>(sR)[i] = reinterpret_cast<const float4*>(rot)[i];

  const int nblk = (N + T - 1) / T;
  const int64_t total = static_cast<int64_t>(B) * H * nblk;
  const int cg = tid % kCG, rg = tid / kCG;
  const float qmax = kInt8 ? 127.0f : 448.0f;

  for (int64_t blk_id = blockIdx.x; blk_id < total; blk_id += gridDim.x) {
    const int blk = static_cast<int>(blk_id % nblk);
    const int bh = static_cast<int>(blk_id / nblk);
    const int b = bh / H, h = bh % H;
    const int n0 = blk * T;
    const int rows = min(T, N - n0);

    __syncthreads();  // sR ready (first pass); previous block's sX reads done
    // Stage x transposed: thread t handles token row (t % T) and a slice of
    // the 16-byte chunks, so consecutive threads write consecutive words.
    for (int idx = tid; idx < T * kCG; idx += kThreads) {
      const int r = idx % T, c = idx / T;
      float f[8];
      if (r < rows) {
        const uint4 v = *reinterpret_cast<const uint4*>(x + row_offset(layout, H, N, D, b, h, n0 + r) + c * 8);
        unpack8(v, is_bf16 != 0, f);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = 0.0f;
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) sX[(c * 8 + e) * kXS + r] = f[e];
    }
    __syncthreads();

    float acc[kRPT][8];
#pragma unroll
    for (int i = 0; i < kRPT; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;

#pragma unroll 2
    for (int k = 0; k < D; ++k) {
      const float4 r0 = *reinterpret_cast<const float4*>(sR + k * D + cg * 8);
      const float4 r1 = *reinterpret_cast<const float4*>(sR + k * D + cg * 8 + 4);
      const float rv[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
#pragma unroll
      for (int i4 = 0; i4 < kRPT / 4; ++i4) {
        const float4 xv = *reinterpret_cast<const float4*>(sX + k * kXS + rg * kRPT + i4 * 4);
        const float xs[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
        for (int ii = 0; ii < 4; ++ii)
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[i4 * 4 + ii][j] = __fmaf_rn(xs[ii], rv[j], acc[i4 * 4 + ii][j]);
      }
    }

    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < kRPT; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(acc[i][j]));  // padded rows are +0
    const float amax = block_max(m, red);
    const float scale = __fdiv_rn(amax, qmax);
    if (tid == 0) scales[static_cast<int64_t>(bh) * nblk + blk] = scale;

#pragma unroll
    for (int i = 0; i < kRPT; ++i) {
      const int r = rg * kRPT + i;
      if (r >= rows) continue;
      uint32_t lo = 0, hi = 0;
      if (scale != 0.0f) {
#pragma unroll
        for (int j = 0; j < 4; ++j) lo |= code_of<kInt8>(acc[i][j], scale) << (8 * j);
#pragma unroll
        for (int j = 0; j < 4; ++j) hi |= code_of<kInt8>(acc[i][j + 4], scale) << (8 * j);
      }
      *reinterpret_cast<uint2*>(codes + row_offset(layout, H, N, D, b, h, n0 + r) + cg * 8) =
          make_uint2(lo, hi);
    }
  }
}

// ---------------------------------------------------------------------------
// Without rotation
// ---------------------------------------------------------------------------

// One CTA per block; each thread owns kV = T*D/8/256 (rounded up) 16-byte
// input vectors, kept in registers between the max and the code pass.
template <int D, int T, bool kInt8>
__global__ void __launch_bounds__(kThreads)
    quant_kernel(const uint16_t* __restrict__ x, int is_bf16, int layout, int B, int H, int N,
                 uint8_t* __restrict__ codes, float* __restrict__ scales) {
  constexpr int kCG = D / 8;
  constexpr int kVec = (T * kCG + kThreads - 1) / kThreads;
  __shared__ float red[kThreads / 32];
  const int nblk = (N + T - 1) / T;
  const int blk = blockIdx.x % nblk;
  const int bh = blockIdx.x / nblk;
  const int b = bh / H, h = bh % H;
  const int n0 = blk * T;
  const int rows = min(T, N - n0);
  const bool bf = is_bf16 != 0;

  uint4 v[kVec];
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < kVec; ++i) {
    const int idx = threadIdx.x + i * kThreads;
    const int r = idx / kCG, c = idx % kCG;
    if (idx < T * kCG && r < rows) {
      v[i] = __ldg(reinterpret_cast<const uint4*>(x + row_offset(layout, H, N, D, b, h, n0 + r) + c * 8));
      float f[8];
      unpack8(v[i], bf, f);
#pragma unroll
      for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(f[e]));
    } else {
      v[i] = make_uint4(0, 0, 0, 0);
    }
  }
  const float amax = block_max(m, red);
  const float scale = __fdiv_rn(amax, kInt8 ? 127.0f : 448.0f);
  if (threadIdx.x == 0) scales[static_cast<int64_t>(bh) * nblk + blk] = scale;
#pragma unroll
  for (int i = 0; i < kVec; ++i) {
    const int idx = threadIdx.x + i * kThreads;
    const int r = idx / kCG, c = idx % kCG;
    if (idx < T * kCG && r < rows) {
      float f[8];
      unpack8(v[i], bf, f);
      uint32_t lo = 0, hi = 0;
      if (scale != 0.0f) {
#pragma unroll
        for (int j = 0; j < 4; ++j) lo |= code_of<kInt8>(f[j], scale) << (8 * j);
#pragma unroll
        for (int j = 0; j < 4; ++j) hi |= code_of<kInt8>(f[j + 4], scale) << (8 * j);
      }
      *reinterpret_cast<uint2*>(codes + row_offset(layout, H, N, D, b, h, n0 + r) + c * 8) =
          make_uint2(lo, hi);
    }
  }
}

template <int D, int T, bool kInt8>
cudaError_t launch_rotq(const RotQuantArgs& a, cudaStream_t st, int num_sms) {
  constexpr size_t smem = sizeof(float) * (D * D + D * (T + 4));
  auto k = rotq_kernel<D, T, kInt8>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t nblocks = static_cast<int64_t>(a.B) * a.H * ((a.N + T - 1) / T);
  const int grid = static_cast<int>(nblocks < num_sms ? nblocks : num_sms);
  k<<<grid, kThreads, smem, st>>>(static_cast<const uint16_t*>(a.x), a.is_bf16, a.layout, a.B, a.H,
                                  a.N, a.rot, static_cast<uint8_t*>(a.codes), a.scales);
  return cudaGetLastError();
}

template <int D, int T, bool kInt8>
cudaError_t launch_quant(const RotQuantArgs& a, cudaStream_t st) {
  const int64_t nblocks = static_cast<int64_t>(a.B) * a.H * ((a.N + T - 1) / T);
  quant_kernel<D, T, kInt8><<<static_cast<unsigned>(nblocks), kThreads, 0, st>>>(
      static_cast<const uint16_t*>(a.x), a.is_bf16, a.layout, a.B, a.H, a.N,
      static_cast<uint8_t*>(a.codes), a.scales);
  return cudaGetLastError();
}

template <int D, int T>
cudaError_t dispatch_t(const RotQuantArgs& a, cudaStream_t st, int num_sms) {
  if (a.rot) return a.int8 ? launch_rotq<D, T, true>(a, st, num_sms) : launch_rotq<D, T, false>(a, st, num_sms);
  return a.int8 ? launch_quant<D, T, true>(a, st) : launch_quant<D, T, false>(a, st);
}

}  // namespace

// Block sizes compiled: 128 and 256 tokens (the method's Q and K/V blocks);
// D in {64, 128}.
cudaError_t launch_rotate_block_quant(const RotQuantArgs& a, cudaStream_t st, int num_sms) {
  if (a.D == 128) {
    if (a.T == 128) return dispatch_t<128, 128>(a, st, num_sms);
    if (a.T == 256) return dispatch_t<128, 256>(a, st, num_sms);
  } else if (a.D == 64) {
    if (a.T == 128) return dispatch_t<64, 128>(a, st, num_sms);
    if (a.T == 256) return dispatch_t<64, 256>(a, st, num_sms);
  }
  return cudaErrorInvalidValue;
}

bool rotate_block_quant_supported(int D, int T) {
  return (D == 64 || D == 128) && (T == 128 || T == 256);
}

}  // namespace qattn
