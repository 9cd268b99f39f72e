// decode.cu -- one decode step against an INT8 or packed-INT4 KV cache,
// split over the key axis, then a softmax merge of the splits.
//
// Method: "INT8 量化算子", ops-transformer item 3 (KV Cache 也量化): the
// cache stays INT8 and attention is computed on it directly, the query is
// INT8 as well, INT32 accumulation, conversion at the output. Packed INT4
// cache with one fp16 scale per group of elements: "ops-transformer
// INT8/INT4 量化推理", 5.1 (group scales) and 5.2 (two codes per byte, even
// element in the low nibble). The nibbles are widened in registers; nothing
// is written back in fp16.
//
// decode_kernel: grid (splits, H_kv, B), 128 threads. Each CTA owns a
// contiguous range of whole 64-token chunks of one (b, h_kv) and all G =
// H_q / H_kv query heads that share it. One thread streams the chunks into a
// 4-stage shared-memory ring with 1-D bulk copies (no multicast); per chunk:
//   A  scores      thread = (token, half of the heads): full dot product
//                  from shared memory (dp4a for INT8, FMA for INT4)
//   B  softmax     warp per head: chunk max, running max/sum update
//   C  P.V         warp = token subset, lane = 4 channels, all heads
// and writes (O, m, l) of its range to the workspace (log2 domain).
// merge_kernel: grid B*H_q, D threads: out = sum_s w_s O_s / sum_s w_s l_s,
// w_s = 2^(m_s - max m).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math_constants.h>

#include "qattn_device.cuh"
#include "qattn_internal.h"

namespace qattn {

namespace {

constexpr int kThreads = 128;
constexpr int kChunk = 64;   // tokens per pipeline stage
constexpr int kStages = 4;
constexpr int kD = 128;      // head size handled by this kernel
constexpr int kWsStride = kD + 4;  // floats per (b, h_q, split) partial: O[D], m, l, pad

struct DecodeParams {
  const uint16_t* q;
  const uint8_t* k;
  const uint8_t* v;
  const void* ks;
  const void* vs;
  int B, Hq, Hkv, L;
  int kv_block, group;
  int splits, chunks_per_split;
  float scale_log2;  // softmax scale * log2(e)
  float* ws;
  int* err;
};

template <bool kInt4>
struct Layout {
  static constexpr int kRowBytes = kInt4 ? kD / 2 : kD;
  static constexpr int kChunkBytes = kChunk * kRowBytes;
};

__device__ __forceinline__ float bf16f(uint16_t h) { return __uint_as_float(static_cast<uint32_t>(h) << 16); }

// Signed 4-bit code of nibble i (0..7) of a 32-bit word, as float.
__device__ __forceinline__ float nib(uint32_t w, int i) {
  return static_cast<float>(static_cast<int32_t>(w << (28 - 4 * i)) >> 28);
}

template <int G, bool kInt4>
__global__ void __launch_bounds__(kThreads) decode_kernel(const DecodeParams p) {
  using Lay = Layout<kInt4>;
  constexpr int kRowBytes = Lay::kRowBytes;
  constexpr int kChunkBytes = Lay::kChunkBytes;
  constexpr int kHalfHeads = G >= 2 ? G / 2 : 1;
  static_assert(4 * G * kD * sizeof(float) <= 2 * kStages * kChunkBytes, "reduction buffer");

  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* sK = smem;                                   // [stages][chunk bytes]
  uint8_t* sV = sK + kStages * kChunkBytes;
  float (*sRed)[G][kD] = reinterpret_cast<float (*)[G][kD]>(smem);  // after the loop only
  union QBuf {
    float f[G][kD];                                     // INT4: query as float
    uint32_t c[G][kD / 4];                              // INT8: packed query codes
  };
  __shared__ __align__(16) QBuf sQb;
  __shared__ float sQf[G];                              // INT8: sq * scale * log2e
  __shared__ float sS[G][kChunk];                       // scores (log2 domain)
  __shared__ __align__(16) float sP[kChunk][G];         // p * (INT8: v block scale)
  __shared__ float sAlpha[G];
  __shared__ float sM[G], sL[G];
  __shared__ __align__(8) uint64_t full[kStages];
  __shared__ int abort_flag;
  auto& sQ = sQb.f;
  auto& sQc = sQb.c;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int g = p.Hq / p.Hkv;
  const int64_t head = static_cast<int64_t>(b) * p.Hkv + hk;
  const int t_begin = split * p.chunks_per_split * kChunk;
  const int t_end = min(p.L, t_begin + p.chunks_per_split * kChunk);
  const int nchunks = t_end > t_begin ? (t_end - t_begin + kChunk - 1) / kChunk : 0;
  const uint8_t* kbase = p.k + head * static_cast<int64_t>(p.L) * kRowBytes;
  const uint8_t* vbase = p.v + head * static_cast<int64_t>(p.L) * kRowBytes;
  const int ngroups = kD / p.group;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&full[s], 1);
    abort_flag = 0;
    mbar_fence_init();
  }
  // Query of the G heads: warp w handles heads w, w+4, ...; lane = 4 channels.
  for (int hh = warp; hh < G; hh += 4) {
    const uint16_t* qr = p.q + (static_cast<int64_t>(b) * p.Hq + hk * g + hh) * kD + lane * 4;
    const uint2 raw = *reinterpret_cast<const uint2*>(qr);
    float f[4] = {bf16f(raw.x & 0xFFFF), bf16f(raw.x >> 16), bf16f(raw.y & 0xFFFF), bf16f(raw.y >> 16)};
    if constexpr (kInt4) {
#pragma unroll
      for (int e = 0; e < 4; ++e) sQ[hh][lane * 4 + e] = f[e];
    } else {
      float m = fmaxf(fmaxf(fabsf(f[0]), fabsf(f[1])), fmaxf(fabsf(f[2]), fabsf(f[3])));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      const float sq = __fdiv_rn(m, 127.0f);
      uint32_t w = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        int c = 0;
        if (sq != 0.0f) c = max(-127, min(127, __float2int_rn(__fdiv_rn(f[e], sq))));
        w |= (static_cast<uint32_t>(c) & 0xFFu) << (8 * e);
      }
      sQc[hh][lane] = w;
      if (lane == 0) sQf[hh] = sq * p.scale_log2;
    }
    if (lane == 0) {
      sM[hh] = -CUDART_INF_F;
      sL[hh] = 0.0f;
    }
  }
  __syncthreads();

  // Row bytes are multiples of 16 and rows start 16-byte aligned, so every
  // copy meets the bulk-copy alignment rules.
  auto issue = [&](int c) {
    const int s = c % kStages;
    const int t0 = t_begin + c * kChunk;
    const int n = min(kChunk, t_end - t0);
    mbar_arrive_expect_tx(&full[s], 2u * n * kRowBytes);
    bulk_load(sK + s * kChunkBytes, kbase + static_cast<int64_t>(t0) * kRowBytes, n * kRowBytes, &full[s]);
    bulk_load(sV + s * kChunkBytes, vbase + static_cast<int64_t>(t0) * kRowBytes, n * kRowBytes, &full[s]);
  };
  int issued = 0;
  if (tid == 0)
    for (; issued < kStages - 1 && issued < nchunks; ++issued) issue(issued);
  const uint16_t* ks16 = static_cast<const uint16_t*>(p.ks) + head * static_cast<int64_t>(p.L) * ngroups;
  const uint16_t* vs16 = static_cast<const uint16_t*>(p.vs) + head * static_cast<int64_t>(p.L) * ngroups;

  float acc[G][4];
#pragma unroll
  for (int hh = 0; hh < G; ++hh)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[hh][e] = 0.0f;

  const int64_t nkb = (p.L + p.kv_block - 1) / p.kv_block;
  for (int c = 0; c < nchunks; ++c) {
    if (tid == 0 && issued < nchunks) issue(issued++);
    const int s = c % kStages;
    const int t0 = t_begin + c * kChunk;
    const int n = min(kChunk, t_end - t0);
    const bool ok = mbar_wait(&full[s], (c / kStages) & 1, &abort_flag, p.err);
    const uint8_t* cK = sK + s * kChunkBytes;
    const uint8_t* cV = sV + s * kChunkBytes;

    // ---- A: scores ----
    if (ok) {
      const int tt = tid % kChunk, half = tid / kChunk;
      if (G >= 2 || half == 0) {
        float sc[kHalfHeads];
        if (tt < n) {
          if constexpr (!kInt4) {
            int dot[kHalfHeads];
#pragma unroll
            for (int j = 0; j < kHalfHeads; ++j) dot[j] = 0;
#pragma unroll
            for (int i = 0; i < kRowBytes / 16; ++i) {
              const int piece = (i + tt) & (kRowBytes / 16 - 1);   // staggered: no bank conflicts
              const uint4 kv = *reinterpret_cast<const uint4*>(cK + tt * kRowBytes + piece * 16);
#pragma unroll
              for (int j = 0; j < kHalfHeads; ++j) {
                const uint4 qv = *reinterpret_cast<const uint4*>(&sQc[half * kHalfHeads + j][piece * 4]);
                dot[j] = __dp4a(static_cast<int>(kv.x), static_cast<int>(qv.x), dot[j]);
                dot[j] = __dp4a(static_cast<int>(kv.y), static_cast<int>(qv.y), dot[j]);
                dot[j] = __dp4a(static_cast<int>(kv.z), static_cast<int>(qv.z), dot[j]);
                dot[j] = __dp4a(static_cast<int>(kv.w), static_cast<int>(qv.w), dot[j]);
              }
            }
            const float sk = static_cast<const float*>(p.ks)[head * nkb + (t0 + tt) / p.kv_block];
#pragma unroll
            for (int j = 0; j < kHalfHeads; ++j)
              sc[j] = static_cast<float>(dot[j]) * (sQf[half * kHalfHeads + j] * sk);
          } else {
            float part[kHalfHeads][2];          // at most two groups per row
#pragma unroll
            for (int j = 0; j < kHalfHeads; ++j) part[j][0] = part[j][1] = 0.0f;
#pragma unroll
            for (int i = 0; i < kRowBytes / 16; ++i) {
              const int piece = (i + tt) & (kRowBytes / 16 - 1);
              const uint4 kv = *reinterpret_cast<const uint4*>(cK + tt * kRowBytes + piece * 16);
              const uint32_t w4[4] = {kv.x, kv.y, kv.z, kv.w};
              const int gsel = (piece * 32) / p.group;           // group of these 32 channels
#pragma unroll
              for (int j = 0; j < kHalfHeads; ++j) {
                const float* qh = &sQ[half * kHalfHeads + j][piece * 32];
                float a = 0.0f;
#pragma unroll
                for (int wi = 0; wi < 4; ++wi)
#pragma unroll
                  for (int e = 0; e < 8; ++e) a = fmaf(qh[wi * 8 + e], nib(w4[wi], e), a);
                if (gsel == 0) part[j][0] += a; else part[j][1] += a;
              }
            }
            const uint16_t* ksr = ks16 + static_cast<int64_t>(t0 + tt) * ngroups;
            const float sk0 = __half2float(__ushort_as_half(ksr[0]));
            const float sk1 = ngroups > 1 ? __half2float(__ushort_as_half(ksr[1])) : 0.0f;
#pragma unroll
            for (int j = 0; j < kHalfHeads; ++j) {
              float v = part[j][0] * sk0;
              if (ngroups > 1) v += part[j][1] * sk1;
              sc[j] = v * p.scale_log2;
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < kHalfHeads; ++j) sc[j] = -CUDART_INF_F;
        }
#pragma unroll
        for (int j = 0; j < kHalfHeads; ++j)
          if (half * kHalfHeads + j < G) sS[half * kHalfHeads + j][tt] = sc[j];
      }
    }
    if (__syncthreads_or(!ok)) break;   // every thread leaves together on a timeout

    // ---- B: running softmax, one warp per head ----
    for (int hh = warp; hh < G; hh += 4) {
      const float s0 = sS[hh][lane], s1 = sS[hh][lane + 32];
      float m = fmaxf(s0, s1);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      const float m_old = sM[hh];
      const float m_new = fmaxf(m_old, m);
      const float alpha = exp2f(m_old - m_new);        // 0 when m_old = -inf
      const float p0 = exp2f(s0 - m_new), p1 = exp2f(s1 - m_new);
      float sum = p0 + p1;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      float sv = 1.0f;
      if constexpr (!kInt4) sv = static_cast<const float*>(p.vs)[head * nkb + t0 / p.kv_block];
      sP[lane][hh] = p0 * sv;
      sP[lane + 32][hh] = p1 * sv;
      __syncwarp();
      if (lane == 0) {
        sAlpha[hh] = alpha;
        sM[hh] = m_new;
        sL[hh] = sL[hh] * alpha + sum;
      }
    }
    __syncthreads();

    // ---- C: O += P V; warp = tokens warp, warp+4, ...; lane = channels 4*lane.. ----
    {
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        const float a = sAlpha[hh];
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[hh][e] *= a;
      }
      for (int t = warp; t < n; t += 4) {
        float vf[4];
        if constexpr (!kInt4) {
          const uint32_t w = *reinterpret_cast<const uint32_t*>(cV + t * kRowBytes + lane * 4);
#pragma unroll
          for (int e = 0; e < 4; ++e) vf[e] = static_cast<float>(static_cast<int32_t>(w << (24 - 8 * e)) >> 24);
        } else {
          const uint32_t w = *reinterpret_cast<const uint16_t*>(cV + t * kRowBytes + lane * 2);
          const float svs = __half2float(__ushort_as_half(vs16[static_cast<int64_t>(t0 + t) * ngroups + (lane * 4) / p.group]));
#pragma unroll
          for (int e = 0; e < 4; ++e) vf[e] = nib(w, e) * svs;
        }
        float pw[G];
        if constexpr (G % 4 == 0) {
#pragma unroll
          for (int j = 0; j < G; j += 4) {
            const float4 pv = *reinterpret_cast<const float4*>(&sP[t][j]);
            pw[j] = pv.x; pw[j + 1] = pv.y; pw[j + 2] = pv.z; pw[j + 3] = pv.w;
          }
        } else {
#pragma unroll
          for (int j = 0; j < G; ++j) pw[j] = sP[t][j];
        }
#pragma unroll
        for (int hh = 0; hh < G; ++hh)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[hh][e] = fmaf(pw[hh], vf[e], acc[hh][e]);
      }
    }
    __syncthreads();  // stage s and sS/sP are free again
  }

  // On a timeout, let the copies already issued land before the ring is
  // reused as the reduction buffer (bounded as well).
  if (abort_flag && tid == 0) {
    for (int c = 0; c < issued; ++c) mbar_wait(&full[c % kStages], (c / kStages) & 1, nullptr, nullptr, 100000000ull);
  }
  __syncthreads();
  // ---- cross-warp reduction and partial output ----
#pragma unroll
  for (int hh = 0; hh < G; ++hh)
    *reinterpret_cast<float4*>(&sRed[warp][hh][lane * 4]) = make_float4(acc[hh][0], acc[hh][1], acc[hh][2], acc[hh][3]);
  __syncthreads();
  for (int i = tid; i < G * kD; i += kThreads) {
    const int hh = i / kD, d = i % kD;
    const float o = sRed[0][hh][d] + sRed[1][hh][d] + sRed[2][hh][d] + sRed[3][hh][d];
    float* w = p.ws + ((static_cast<int64_t>(b) * p.Hq + hk * g + hh) * p.splits + split) * kWsStride;
    w[d] = o;
    if (d == 0) {
      w[kD] = sM[hh];
      w[kD + 1] = abort_flag ? 0.0f : sL[hh];
    }
  }
}

__global__ void __launch_bounds__(kD) merge_kernel(const float* __restrict__ ws, int splits,
                                                   __nv_bfloat16* __restrict__ out) {
  const int64_t bh = blockIdx.x;
  const float* w = ws + bh * splits * kWsStride;
  const int d = threadIdx.x;
  float M = -CUDART_INF_F;
  for (int s = 0; s < splits; ++s) M = fmaxf(M, w[s * kWsStride + kD]);
  float num = 0.0f, den = 0.0f;
  if (M != -CUDART_INF_F) {
    for (int s = 0; s < splits; ++s) {
      const float l = w[s * kWsStride + kD + 1];
      if (l == 0.0f) continue;
      const float sc = exp2f(w[s * kWsStride + kD] - M);
      num = fmaf(sc, w[s * kWsStride + d], num);
      den = fmaf(sc, l, den);
    }
  }
  out[bh * kD + d] = __float2bfloat16_rn(den > 0.0f ? num / den : 0.0f);
}

template <int G, bool kInt4>
cudaError_t launch_g(const DecodeParams& p, cudaStream_t st) {
  using Lay = Layout<kInt4>;
  const size_t smem = 2 * kStages * Lay::kChunkBytes;
  auto k = decode_kernel<G, kInt4>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(p.splits, p.Hkv, p.B);
  k<<<grid, kThreads, smem, st>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return cudaSuccess;
}

}  // namespace

bool decode_supported(int D, int group_ratio) { return D == kD && (group_ratio == 1 || group_ratio == 2); }

int decode_splits(int B, int Hkv, int L, int num_sms) {
  const int chunks = (L + kChunk - 1) / kChunk;
  if (chunks == 0) return 1;
  const int64_t pairs = static_cast<int64_t>(B) * Hkv;
  const int64_t target = 8LL * num_sms;                 // CTAs to aim for
  int splits = static_cast<int>((target + pairs - 1) / pairs);
  const int min_chunks = 4;                             // keep the ring busy
  splits = max(1, min(splits, (chunks + min_chunks - 1) / min_chunks));
  // Equalise: every split gets the same number of whole chunks.
  const int per = (chunks + splits - 1) / splits;
  return (chunks + per - 1) / per;
}

size_t decode_workspace_bytes(int B, int Hq, int Hkv, int L, int D, int num_sms) {
  (void)D;
  const int splits = decode_splits(B, Hkv, L, num_sms);
  return static_cast<size_t>(B) * Hq * splits * kWsStride * sizeof(float);
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st, int num_sms, int* err) {
  DecodeParams p;
  p.q = static_cast<const uint16_t*>(a.q);
  p.k = static_cast<const uint8_t*>(a.k);
  p.v = static_cast<const uint8_t*>(a.v);
  p.ks = a.ks;
  p.vs = a.vs;
  p.B = a.B; p.Hq = a.Hq; p.Hkv = a.Hkv; p.L = a.L;
  p.kv_block = a.kv_block; p.group = a.group;
  p.splits = decode_splits(a.B, a.Hkv, a.L, num_sms);
  const int chunks = (a.L + kChunk - 1) / kChunk;
  p.chunks_per_split = (chunks + p.splits - 1) / p.splits;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.ws = static_cast<float*>(a.workspace);
  p.err = err;
  const int G = a.Hq / a.Hkv;
  cudaError_t e = cudaErrorInvalidValue;
  if (a.int4) {
    if (G == 1) e = launch_g<1, true>(p, st);
    else if (G == 2) e = launch_g<2, true>(p, st);
    else if (G == 4) e = launch_g<4, true>(p, st);
    else if (G == 8) e = launch_g<8, true>(p, st);
  } else {
    if (G == 1) e = launch_g<1, false>(p, st);
    else if (G == 2) e = launch_g<2, false>(p, st);
    else if (G == 4) e = launch_g<4, false>(p, st);
    else if (G == 8) e = launch_g<8, false>(p, st);
  }
  if (e != cudaSuccess) return e;
  merge_kernel<<<static_cast<unsigned>(static_cast<int64_t>(a.B) * a.Hq), kD, 0, st>>>(
      p.ws, p.splits, static_cast<__nv_bfloat16*>(a.out));
  return cudaGetLastError();
}

}  // namespace qattn
