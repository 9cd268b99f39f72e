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

constexpr int kThreads = 256;                 // quant_kernel
template <int D>
struct RotqThreads {
  static constexpr int value = D == 128 ? 512 : 256;   // 16 warps per SM for D = 128
};

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

// Code byte of RNE(y / scale) with y / scale rounded to float32 first, as
// IEEE division gives it, computed without a division in almost every case.
//
// v0 = y * rcp with rcp = RN(1 / scale) is within 1.5 * 2^-23 |v| of the
// correctly rounded quotient RN(y / scale) (two roundings of 2^-24 relative
// each, plus the half ulp of the quotient itself). The code only depends on
// which side of the nearest rounding boundary that quotient lies (a
// half-integer for INT8, a midpoint between e4m3 values for FP8). When v0 is
// farther than that bound from every boundary both give the same code; in
// the rare remaining cases the IEEE quotient is computed (__fdiv_rn).
//   INT8: |v| <= 127.5, so the bound is below 2.3e-5; v0 is trusted when
//         its distance to the nearest integer is below 0.5 - 1e-4.
//   e4m3: in the normal range the boundary sits where float32 mantissa bits
//         19..0 equal 0x80000, and the bound is 3 units of bit 0; v0 is
//         trusted when those bits are more than 16 units away from 0x80000.
//         Below 2^-6 (e4m3 subnormals) the IEEE quotient is used.
// Saturation needs no care: every value at or beyond +-448 gives +-448.
// A scale below the smallest normal float32 (`slow`, uniform over the block)
// breaks these bounds (the reciprocal loses precision or overflows), so such
// blocks always take the IEEE quotient, clamped for INT8.
__device__ __noinline__ float ieee_div(float y, float scale) { return __fdiv_rn(y, scale); }

template <bool kInt8>
__device__ __forceinline__ uint32_t code_of(float y, float scale, float rcp, bool slow) {
  if (slow) {
    const float v = ieee_div(y, scale);
    if constexpr (kInt8) return static_cast<uint32_t>(max(-127, min(127, __float2int_rn(v)))) & 0xFFu;
    else return cvt_e4m3x2(v, 0.0f) & 0xFFu;
  }
  const float v0 = y * rcp;
  if constexpr (kInt8) {
    const float r = (v0 + 12582912.0f) - 12582912.0f;   // round half to even (|v0| < 2^22)
    const float dist = fabsf(v0 - r);                   // exact
    float v = v0;
    if (dist > 0.4999f) v = ieee_div(y, scale);         // near a half-integer: decide exactly
    const float t = v + 12582912.0f;                    // integer in the low mantissa bits
    return __float_as_uint(t) & 0xFFu;                  // two's complement byte (|v| <= 127.5)
  } else {
    const uint32_t b = __float_as_uint(v0) & 0x7FFFFFFFu;
    const int near_mid = abs(static_cast<int>(b & 0xFFFFFu) - 0x80000) <= 16;
    const float v = (b < 0x3C800000u || near_mid) ? ieee_div(y, scale) : v0;   // 2^-6 = 0x3C800000
    return cvt_e4m3x2(v, 0.0f) & 0xFFu;
  }
}

template <int kNT>
__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < kNT / 32; ++i) m = fmaxf(m, red[i]);
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
// Codes of eight values at a time
// ---------------------------------------------------------------------------

// Codes of 8 values by the fast path of code_of alone (v0 = y * rcp), packed
// little-endian into lo (values 0..3) and hi (4..7). Returns false when any
// value is too close to a rounding boundary (or, for e4m3, in the subnormal
// range) for v0 to be trusted; the caller then takes the exact path.
template <bool kInt8>
__device__ __forceinline__ bool codes8_fast(const float (&f)[8], float rcp, uint32_t& lo, uint32_t& hi) {
  bool ok = true;
  uint32_t t[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float v0 = f[e] * rcp;
    if constexpr (kInt8) {
      const float m = v0 + 12582912.0f;                  // RNE integer in the low mantissa bits
      ok = ok && fabsf(v0 - (m - 12582912.0f)) <= 0.4999f;
      t[e] = __float_as_uint(m);
    } else {
      const uint32_t bb = __float_as_uint(v0) & 0x7FFFFFFFu;
      ok = ok && bb >= 0x3C800000u && abs(static_cast<int>(bb & 0xFFFFFu) - 0x80000) > 16;
      t[e] = __float_as_uint(v0);
    }
  }
  if constexpr (kInt8) {
    lo = __byte_perm(__byte_perm(t[0], t[1], 0x0040), __byte_perm(t[2], t[3], 0x0040), 0x5410);
    hi = __byte_perm(__byte_perm(t[4], t[5], 0x0040), __byte_perm(t[6], t[7], 0x0040), 0x5410);
  } else {
    lo = cvt_e4m3x2(__uint_as_float(t[0]), __uint_as_float(t[1])) |
         (cvt_e4m3x2(__uint_as_float(t[2]), __uint_as_float(t[3])) << 16);
    hi = cvt_e4m3x2(__uint_as_float(t[4]), __uint_as_float(t[5])) |
         (cvt_e4m3x2(__uint_as_float(t[6]), __uint_as_float(t[7])) << 16);
  }
  return ok;
}

// Eight float32 values, passed by value to the rare exact path.
struct F8 {
  float v[8];
};

// Codes of 8 values with the IEEE quotient for every value, packed like
// codes8_fast.
template <bool kInt8>
__device__ __noinline__ uint2 codes8_exact_f(F8 f, float scale) {
  uint32_t lo = 0, hi = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) lo |= code_of<kInt8>(f.v[j], scale, 0.0f, true) << (8 * j);
#pragma unroll
  for (int j = 0; j < 4; ++j) hi |= code_of<kInt8>(f.v[j + 4], scale, 0.0f, true) << (8 * j);
  return make_uint2(lo, hi);
}

// The same for 8 raw 16-bit inputs.
template <bool kInt8>
__device__ __forceinline__ uint2 codes8_exact(uint4 raw, bool is_bf16, float scale) {
  F8 f;
  unpack8(raw, is_bf16, f.v);
  return codes8_exact_f<kInt8>(f, scale);
}

// ---------------------------------------------------------------------------
// With rotation
// ---------------------------------------------------------------------------

// Thread tile: kRPT rows x 8 columns of y. Column group cg = tid % (D/8)
// owns columns 4cg..4cg+3 and D/2+4cg..D/2+4cg+3 (two float4 of each R row,
// consecutive across the warp, so the R reads are free of bank conflicts);
// row group rg = tid / (D/8) owns rows rg*kRPT .. rg*kRPT + kRPT - 1.
template <int D, int T, bool kInt8>
__global__ void __launch_bounds__(RotqThreads<D>::value, 1)
    rotq_kernel(const uint16_t* __restrict__ x, int is_bf16, int layout, int B, int H, int N,
                const float* __restrict__ rot, uint8_t* __restrict__ codes,
                float* __restrict__ scales) {
  constexpr int kNT = RotqThreads<D>::value;
  constexpr int kCG = D / 8;               // column groups
  constexpr int kRG = kNT / kCG;           // row groups
  constexpr int kRPT = T / kRG;            // rows per thread
  constexpr int kXS = T + 4;               // padded row stride of the transposed x tile
  static_assert(kRPT % 4 == 0 && kRPT >= 4, "row tile");
  extern __shared__ __align__(16) float smem[];
  float* sR = smem;                        // [D][D]
  float* sX = smem + D * D;                // [D][kXS]: sX[k * kXS + r] = x[r][k]
  __shared__ float red[kNT / 32];

  const int tid = threadIdx.x;
  for (int i = tid; i < D * D / 4; i += kNT)
    reinterpret_cast<float4*>(sR)[i] = reinterpret_cast<const float4*>(rot)[i];

  const int nblk = (N + T - 1) / T;
  const int64_t total = static_cast<int64_t>(B) * H * nblk;
  const int cg = tid % kCG, rg = tid / kCG;
  const int c0 = 4 * cg, c1 = D / 2 + 4 * cg;   // this thread's two column quads
  const float qmax = kInt8 ? 127.0f : 448.0f;

  // Raw 16-byte input vectors of the next block, loaded into registers while
  // the current block is being computed (thread t: token row idx % T and
  // 8-channel chunk idx / T for idx = t, t + kNT, ...).
  constexpr int kLd = (T * kCG + kNT - 1) / kNT;
  uint4 xr[kLd];
  auto load_block = [&](int64_t id) {
    const int blk_ = static_cast<int>(id % nblk);
    const int bh_ = static_cast<int>(id / nblk);
    const int b_ = bh_ / H, h_ = bh_ % H;
    const int n0_ = blk_ * T;
    const int rows_ = min(T, N - n0_);
#pragma unroll
    for (int i = 0; i < kLd; ++i) {
      const int idx = tid + i * kNT;
      const int r = idx % T, c = idx / T;
      xr[i] = make_uint4(0, 0, 0, 0);
      if (idx < T * kCG && r < rows_)
        xr[i] = __ldcs(reinterpret_cast<const uint4*>(x + row_offset(layout, H, N, D, b_, h_, n0_ + r) + c * 8));
    }
  };
  // Only where the registers allow it (the larger row tiles of 256-token
  // blocks already use them all): otherwise the block is loaded on the spot.
  constexpr bool kPrefetch = kLd <= 4;
  if (kPrefetch && blockIdx.x < total) load_block(blockIdx.x);

  for (int64_t blk_id = blockIdx.x; blk_id < total; blk_id += gridDim.x) {
    const int blk = static_cast<int>(blk_id % nblk);
    const int bh = static_cast<int>(blk_id / nblk);
    const int b = bh / H, h = bh % H;
    const int n0 = blk * T;
    const int rows = min(T, N - n0);

    if (!kPrefetch) load_block(blk_id);
    __syncthreads();  // sR ready (first pass); previous block's sX reads done
    // Stage x transposed: consecutive threads write consecutive words.
#pragma unroll
    for (int i = 0; i < kLd; ++i) {
      const int idx = tid + i * kNT;
      if (idx < T * kCG) {
        const int r = idx % T, c = idx / T;
        float f[8];
        unpack8(xr[i], is_bf16 != 0, f);
#pragma unroll
        for (int e = 0; e < 8; ++e) sX[(c * 8 + e) * kXS + r] = f[e];
      }
    }
    __syncthreads();
    if (kPrefetch && blk_id + gridDim.x < total) load_block(blk_id + gridDim.x);

    // acc[i][j]: row rg*kRPT + i, column (j < 4 ? c0 + j : c1 + j - 4); each
    // is the float32 FMA chain over k ascending, two lanes per f32x2 FMA.
    float2 acc[kRPT][4];
#pragma unroll
    for (int i = 0; i < kRPT; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = make_float2(0.0f, 0.0f);

#pragma unroll 2
    for (int k = 0; k < D; ++k) {
      const float4 r0 = *reinterpret_cast<const float4*>(sR + k * D + c0);
      const float4 r1 = *reinterpret_cast<const float4*>(sR + k * D + c1);
      const float2 rv[4] = {make_float2(r0.x, r0.y), make_float2(r0.z, r0.w), make_float2(r1.x, r1.y),
                            make_float2(r1.z, r1.w)};
#pragma unroll
      for (int i4 = 0; i4 < kRPT / 4; ++i4) {
        const float4 xv = *reinterpret_cast<const float4*>(sX + k * kXS + rg * kRPT + i4 * 4);
        const float xs[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
        for (int ii = 0; ii < 4; ++ii) {
          const float2 x2 = make_float2(xs[ii], xs[ii]);
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i4 * 4 + ii][j] = ffma2(x2, rv[j], acc[i4 * 4 + ii][j]);
        }
      }
    }

    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < kRPT; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) m = fmaxf(m, fmaxf(fabsf(acc[i][j].x), fabsf(acc[i][j].y)));  // padded rows are +0
    const float amax = block_max<kNT>(m, red);
    const float scale = __fdiv_rn(amax, qmax);
    const float rcp = __frcp_rn(scale);
    const bool slow = scale < 1.17549435e-38f;
    if (tid == 0) scales[static_cast<int64_t>(bh) * nblk + blk] = scale;

    // Codes by the division-free fast path, one trust check per row of 8
    // values; the rare rows it cannot decide (and blocks with a subnormal
    // scale) are coded afterwards with IEEE divisions.
    uint32_t fix = 0;
#pragma unroll
    for (int i = 0; i < kRPT; ++i) {
      const int r = rg * kRPT + i;
      if (r >= rows) continue;
      uint32_t w0 = 0, w1 = 0;
      if (scale != 0.0f) {
        const float f[8] = {acc[i][0].x, acc[i][0].y, acc[i][1].x, acc[i][1].y,
                            acc[i][2].x, acc[i][2].y, acc[i][3].x, acc[i][3].y};
        if (!codes8_fast<kInt8>(f, rcp, w0, w1) || slow) {
          fix |= 1u << i;
          continue;
        }
      }
      uint8_t* crow = codes + row_offset(layout, H, N, D, b, h, n0 + r);
      *reinterpret_cast<uint32_t*>(crow + c0) = w0;
      *reinterpret_cast<uint32_t*>(crow + c1) = w1;
    }
    if (fix != 0) {
#pragma unroll
      for (int i = 0; i < kRPT; ++i) {
        if (!((fix >> i) & 1u)) continue;
        const F8 f = {{acc[i][0].x, acc[i][0].y, acc[i][1].x, acc[i][1].y,
                       acc[i][2].x, acc[i][2].y, acc[i][3].x, acc[i][3].y}};
        const uint2 w = codes8_exact_f<kInt8>(f, scale);
        uint8_t* crow = codes + row_offset(layout, H, N, D, b, h, n0 + rg * kRPT + i);
        *reinterpret_cast<uint32_t*>(crow + c0) = w.x;
        *reinterpret_cast<uint32_t*>(crow + c1) = w.y;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Without rotation
// ---------------------------------------------------------------------------

// One CTA per block; each thread owns kVec = T*D/8/256 (rounded up) 16-byte
// input vectors, kept in registers between the max and the code pass. Codes
// are formed by the division-free fast path; the few vectors holding a value
// it cannot decide are reloaded and coded with IEEE divisions afterwards,
// which keeps the unrolled main loop small and branch-free.
template <int D, int T, bool kInt8>
__global__ void __launch_bounds__(kThreads)
    quant_kernel(const uint16_t* __restrict__ x, int is_bf16, int layout, int B, int H, int N,
                 uint8_t* __restrict__ codes, float* __restrict__ scales) {
  constexpr int kCG = D / 8;
  constexpr int kVec = (T * kCG + kThreads - 1) / kThreads;
  static_assert(kVec <= 32, "fix-up mask");
  __shared__ float red[kThreads / 32];
  const int nblk = (N + T - 1) / T;
  const int blk = blockIdx.x % nblk;
  const int bh = blockIdx.x / nblk;
  const int b = bh / H, h = bh % H;
  const int n0 = blk * T;
  const int rows = min(T, N - n0);
  const bool bf = is_bf16 != 0;

  uint4 v[kVec];
  // all loads first (16 bytes each, in flight together), then the max
#pragma unroll
  for (int i = 0; i < kVec; ++i) {
    const int idx = threadIdx.x + i * kThreads;
    const int r = idx / kCG, c = idx % kCG;
    v[i] = make_uint4(0, 0, 0, 0);
    if (idx < T * kCG && r < rows)
      v[i] = __ldcs(reinterpret_cast<const uint4*>(x + row_offset(layout, H, N, D, b, h, n0 + r) + c * 8));
  }
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < kVec; ++i) {
    float f[8];
    unpack8(v[i], bf, f);
#pragma unroll
    for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(f[e]));
  }
  const float amax = block_max<kThreads>(m, red);
  const float scale = __fdiv_rn(amax, kInt8 ? 127.0f : 448.0f);
  const float rcp = __frcp_rn(scale);
  const bool slow = scale < 1.17549435e-38f;          // zero or subnormal scale: exact path
  if (threadIdx.x == 0) scales[static_cast<int64_t>(bh) * nblk + blk] = scale;
  uint32_t fix = 0;
#pragma unroll
  for (int i = 0; i < kVec; ++i) {
    const int idx = threadIdx.x + i * kThreads;
    const int r = idx / kCG, c = idx % kCG;
    if (idx < T * kCG && r < rows) {
      float f[8];
      unpack8(v[i], bf, f);
      uint32_t lo, hi;
      const bool ok = codes8_fast<kInt8>(f, rcp, lo, hi);
      if (ok && !slow) {
        *reinterpret_cast<uint2*>(codes + row_offset(layout, H, N, D, b, h, n0 + r) + c * 8) = make_uint2(lo, hi);
      } else {
        fix |= 1u << i;
      }
    }
  }
  while (fix != 0) {
    const int i = __ffs(fix) - 1;
    fix &= fix - 1;
    const int idx = threadIdx.x + i * kThreads;
    const int r = idx / kCG, c = idx % kCG;
    const int64_t off = row_offset(layout, H, N, D, b, h, n0 + r) + c * 8;
    uint2 w = make_uint2(0, 0);
    if (scale != 0.0f) w = codes8_exact<kInt8>(*reinterpret_cast<const uint4*>(x + off), bf, scale);
    *reinterpret_cast<uint2*>(codes + off) = w;
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
  k<<<grid, RotqThreads<D>::value, smem, st>>>(static_cast<const uint16_t*>(a.x), a.is_bf16, a.layout, a.B,
                                                a.H, a.N, a.rot, static_cast<uint8_t*>(a.codes), a.scales);
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
