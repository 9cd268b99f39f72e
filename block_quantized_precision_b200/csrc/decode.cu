// decode.cu -- one decode step against an INT8 or packed-INT4 KV cache,
// split over the key axis, then a softmax merge of the splits.
//
// Method: "INT8 量化算子", ops-transformer item 3 (KV Cache 也量化): the
// cache stays INT8 and attention is computed on it directly, the query is
// INT8 as well, INT32 accumulation, conversion at the output. Packed INT4
// cache with one fp16 scale per group of elements: "ops-transformer
// INT8/INT4 量化推理", 5.1 (group scales) and 5.2 (two codes per byte, even
// element in the low nibble); the nibbles are widened to INT8 in registers
// and meet the INT8 query ("FlashAttention 的 INT8/INT4 量化", 第二层).
// Nothing is ever written back in fp16.
//
// decode_kernel: grid (splits, H_kv, B), 5 warps. Each CTA owns a contiguous
// range of whole chunks of one (b, h_kv) and all G = H_q / H_kv query heads
// that share it.
//   warp 4      producer: K and V chunks (64 tokens INT8 / 128 tokens INT4)
//               by TMA tensor loads with hardware swizzle into a 4-stage
//               ring (no multicast).
//   warps 0-3   consumers, each on its own quarter of every chunk with its
//               own running softmax (no block barrier per chunk), 16 tokens
//               per step:
//                 scores   lane pair per token, each lane half a row: dp4a on
//                          the INT8 query codes held in registers (INT4
//                          nibbles widened to bytes first), pair sum by shuffle
//                 softmax  warp max by redux on order-preserving integer keys,
//                          exp2, per-lane partial sums
//                 P.V      lane = 4 channels x all heads; bytes/nibbles turned
//                          into floats with byte-permute/magic-number tricks
//                          on the ALU/FMA pipes, packed f32x2 FMAs
//               then the four warps merge their states and write (O, m, l)
//               of the range to the workspace (log2 domain).
// merge_kernel: grid B*H_q, D threads: out = sum_s w_s O_s / sum_s w_s l_s,
// w_s = 2^(m_s - max m).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math_constants.h>

#include <cmath>

#include "qattn_device.cuh"
#include "qattn_internal.h"

namespace qattn {

namespace {

constexpr int kD = 128;               // head size handled by this kernel
constexpr int kConsumers = 4;         // consumer warps
constexpr int kThreads = 32 * (kConsumers + 1);
constexpr int kStages = 4;
constexpr int kStep = 16;             // tokens per consumer step
constexpr int kWsStride = kD + 4;     // floats per (b, h_q, split) partial: O[D], m, l, pad

template <bool kInt4>
struct Cfg {
  static constexpr int kRowBytes = kInt4 ? kD / 2 : kD;
  static constexpr int kChunk = kInt4 ? 128 : 64;             // tokens per stage
  static constexpr int kTileBytes = kChunk * kRowBytes;       // one tensor, one stage (8 KB)
  static constexpr int kPerWarp = kChunk / kConsumers;        // tokens per warp per chunk
  static constexpr int kSmemBytes = 2 * kStages * kTileBytes + 1024;
};

struct DecodeParams {
  const uint16_t* q;
  const void* ks;
  const void* vs;
  int B, Hq, Hkv, L;
  int kv_block, group;
  int splits, chunks_per_split;
  float scale_log2;  // softmax scale * log2(e)
  float* ws;
  int* err;
};

__device__ __forceinline__ float bf16f(uint32_t h) { return __uint_as_float(h << 16); }

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Four signed bytes of w -> floats: byte b becomes the mantissa of
// 2^23 + (b + 128), then 2^23 + 128 is subtracted (exact).
__device__ __forceinline__ void s8x4_to_f32(uint32_t w, float2& lo, float2& hi) {
  const uint32_t u = w ^ 0x80808080u;
  const float2 off = make_float2(-8388736.0f, -8388736.0f);
  lo = fadd2(make_float2(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7540)),
                         __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7541))), off);
  hi = fadd2(make_float2(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7542)),
                         __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7543))), off);
}

// Four signed nibbles (bits 0..15 of w, element i in bits 4i..4i+3) ->
// floats: 2^23 + (c + 8) built by one LOP3 each, then 2^23 + 8 subtracted.
__device__ __forceinline__ void s4x4_to_f32(uint32_t w, float2& lo, float2& hi) {
  const float2 off = make_float2(-8388616.0f, -8388616.0f);
  lo = fadd2(make_float2(__uint_as_float((w & 0xFu) ^ 0x4B000008u), __uint_as_float(((w >> 4) & 0xFu) ^ 0x4B000008u)),
             off);
  hi = fadd2(make_float2(__uint_as_float(((w >> 8) & 0xFu) ^ 0x4B000008u),
                         __uint_as_float(((w >> 12) & 0xFu) ^ 0x4B000008u)),
             off);
}

template <int G, bool kInt4, int kGroups>
__global__ void __launch_bounds__(kThreads, kInt4 ? 2 : 3)
    decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const DecodeParams p) {
  using C = Cfg<kInt4>;
  constexpr int kRowBytes = C::kRowBytes;
  constexpr int kTile = C::kTileBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem;                          // [stages][chunk rows], swizzled
  uint8_t* sV = smem + kStages * kTile;
  float* sRed = reinterpret_cast<float*>(smem);   // after the loop: [warps][G][D]

  __shared__ __align__(16) uint32_t sQw[G][kD / 4];    // query codes, 4 per word (natural order)
  __shared__ int sQsum[G][2];                          // INT4: sum of query codes per half row
  __shared__ float sQf[G];                             // sq * softmax scale * log2(e)
  __shared__ __align__(16) float2 sP[kConsumers][kStep][G];  // (p, p) * v scale, per warp
  __shared__ float sSV[kConsumers][kStep][2];          // INT4 with two groups: v scales
  // Scales of each staged chunk, written by the producer warp: INT8 one K and
  // one V block scale per chunk; INT4 one fp16 per token and group.
  __shared__ float sKsc[kStages], sVsc[kStages];
  __shared__ uint16_t sKs16[kInt4 ? kStages : 1][kInt4 ? C::kChunk * kGroups : 1];
  __shared__ uint16_t sVs16[kInt4 ? kStages : 1][kInt4 ? C::kChunk * kGroups : 1];
  __shared__ float sWm[kConsumers][G], sWl[kConsumers][G];
  __shared__ __align__(8) uint64_t full[kStages], empty[kStages];
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int g = p.Hq / p.Hkv;
  const int64_t head = static_cast<int64_t>(b) * p.Hkv + hk;
  const int t_begin = split * p.chunks_per_split * C::kChunk;
  const int t_end = min(p.L, t_begin + p.chunks_per_split * C::kChunk);
  const int nchunks = t_end > t_begin ? (t_end - t_begin + C::kChunk - 1) / C::kChunk : 0;
  const int64_t nkb = (p.L + p.kv_block - 1) / p.kv_block;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 2);          // TMA transaction arrive + scales arrive
      mbar_init(&empty[s], kConsumers);
    }
    abort_flag = 0;
    mbar_fence_init();
  }
  // Query codes of the G heads (consumer warps; warp w: heads w, w+4, ...).
  if (warp < kConsumers) {
    for (int hh = warp; hh < G; hh += kConsumers) {
      const uint2 raw = *reinterpret_cast<const uint2*>(p.q + (static_cast<int64_t>(b) * p.Hq + hk * g + hh) * kD + lane * 4);
      const float f[4] = {bf16f(raw.x & 0xFFFF), bf16f(raw.x >> 16), bf16f(raw.y & 0xFFFF), bf16f(raw.y >> 16)};
      float m = fmaxf(fmaxf(fabsf(f[0]), fabsf(f[1])), fmaxf(fabsf(f[2]), fabsf(f[3])));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      const float sq = __fdiv_rn(m, 127.0f);
      uint32_t w = 0;
      int csum = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        int c = 0;
        if (sq != 0.0f) c = max(-127, min(127, __float2int_rn(__fdiv_rn(f[e], sq))));
        csum += c;
        w |= (static_cast<uint32_t>(c) & 0xFFu) << (8 * e);
      }
      sQw[hh][lane] = w;
      // lanes 0..15 hold channels 0..63 (first half row), 16..31 the second
      const int half_sum0 = __reduce_add_sync(0xffffffffu, lane < 16 ? csum : 0);
      const int half_sum1 = __reduce_add_sync(0xffffffffu, lane >= 16 ? csum : 0);
      if (lane == 0) {
        sQf[hh] = sq * p.scale_log2;
        sQsum[hh][0] = half_sum0;
        sQsum[hh][1] = half_sum1;
      }
    }
  }
  __syncthreads();

  if (warp == kConsumers) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
    }
    // The scales of chunk c + 1 are loaded into registers while chunk c is
    // being staged, so their global-load latency overlaps the ring waits.
    constexpr int kScalePerLane = kInt4 ? (C::kChunk * kGroups) / 32 : 1;
    uint16_t ksv[kScalePerLane], vsv[kScalePerLane];
    float ksc = 0.0f, vsc = 0.0f;
    auto load_scales = [&](int cc) {
      const int t0 = t_begin + cc * C::kChunk;
      if constexpr (!kInt4) {
        ksc = static_cast<const float*>(p.ks)[head * nkb + t0 / p.kv_block];
        vsc = static_cast<const float*>(p.vs)[head * nkb + t0 / p.kv_block];
      } else {
        const uint16_t* kss = static_cast<const uint16_t*>(p.ks) + (head * p.L + t0) * kGroups;
        const uint16_t* vss = static_cast<const uint16_t*>(p.vs) + (head * p.L + t0) * kGroups;
        const int nvals = min(C::kChunk, t_end - t0) * kGroups;
#pragma unroll
        for (int j = 0; j < kScalePerLane; ++j) {
          const int i = lane + 32 * j;
          ksv[j] = i < nvals ? kss[i] : static_cast<uint16_t>(0);
          vsv[j] = i < nvals ? vss[i] : static_cast<uint16_t>(0);
        }
      }
    };
    if (nchunks > 0) load_scales(0);
    int c = 0;
    for (; c < nchunks; ++c) {
      const int s = c % kStages;
      if (c >= kStages) {
        const bool ok = mbar_wait(&empty[s], ((c / kStages) - 1) & 1, &abort_flag, p.err);
        if (!__all_sync(0xffffffffu, ok)) break;
      }
      const int t0 = t_begin + c * C::kChunk;
      if (lane == 0) {
        mbar_arrive_expect_tx(&full[s], 2 * kTile);
        tma_load_3d(sK + s * kTile, &tmK, &full[s], 0, t0, static_cast<int>(head));
        tma_load_3d(sV + s * kTile, &tmV, &full[s], 0, t0, static_cast<int>(head));
      }
      if constexpr (!kInt4) {
        if (lane == 0) {
          sKsc[s] = ksc;
          sVsc[s] = vsc;
        }
      } else {
#pragma unroll
        for (int j = 0; j < kScalePerLane; ++j) {
          sKs16[s][lane + 32 * j] = ksv[j];
          sVs16[s][lane + 32 * j] = vsv[j];
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&full[s]);
      if (c + 1 < nchunks) load_scales(c + 1);
    }
    if (abort_flag && lane == 0) {
      for (int i = max(0, c - kStages); i < c; ++i)
        mbar_wait(&full[i % kStages], (i / kStages) & 1, nullptr, nullptr, 100000000ull);
    }
    __syncwarp();
    return;   // the producer takes no part in the final merge
  }

  // ---------------------------------------------------------------- consumers
  const int tp = lane >> 1;          // token of this lane within a step
  const int half = lane & 1;         // which half row this lane scores
  // Query words for this lane's half row, in the order the key words are read.
  int qreg[G][16];
  int qsum_half[G];
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    qsum_half[hh] = sQsum[hh][half];
    if constexpr (!kInt4) {
#pragma unroll
      for (int j = 0; j < 16; ++j) qreg[hh][j] = static_cast<int>(sQw[hh][half * 16 + j]);
    } else {
      // 8 key words (64 nibbles) per half row; word j holds channels
      // half*64 + 8j + {0..7}: even channels (low nibbles) and odd channels
      // (high nibbles) are widened into separate byte vectors.
      const uint8_t* qb = reinterpret_cast<const uint8_t*>(&sQw[hh][0]);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int d0 = half * 64 + 8 * j;
        qreg[hh][2 * j] = static_cast<int>(qb[d0] | (qb[d0 + 2] << 8) | (qb[d0 + 4] << 16) | (static_cast<uint32_t>(qb[d0 + 6]) << 24));
        qreg[hh][2 * j + 1] = static_cast<int>(qb[d0 + 1] | (qb[d0 + 3] << 8) | (qb[d0 + 5] << 16) | (static_cast<uint32_t>(qb[d0 + 7]) << 24));
      }
    }
  }
  float qf[G];
#pragma unroll
  for (int hh = 0; hh < G; ++hh) qf[hh] = sQf[hh];
  const int my_group = kGroups == 2 ? (lane >> 4) : 0;   // group of this lane's 4 P.V channels
  // Byte offset of this lane's 4 P.V channels inside a swizzled V row: the
  // unswizzled offset is 4*lane (INT8) or 2*lane (INT4); the swizzle XORs
  // the 16-byte chunk index with row % 8 (INT8) or (row / 2) % 4 (INT4).
  // Steps start at multiples of 16 rows, so the XOR term is a compile-time
  // function of the row within the step.
  const int lane_off = kInt4 ? 2 * lane : 4 * lane;

  float m_run[G], l_run[G];
  float2 acc[G][2];
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    m_run[hh] = -CUDART_INF_F;
    l_run[hh] = 0.0f;
    acc[hh][0] = acc[hh][1] = make_float2(0.0f, 0.0f);
  }

  for (int c = 0; c < nchunks; ++c) {
    const int s = c % kStages;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&full[s], (c / kStages) & 1, &abort_flag, p.err));
    if (!ok) break;
    const uint8_t* cK = sK + s * kTile;
    const uint8_t* cV = sV + s * kTile;
    const int chunk_t0 = t_begin + c * C::kChunk;
#pragma unroll 1
    for (int sub = 0; sub < C::kPerWarp / kStep; ++sub) {
      const int r0 = warp * C::kPerWarp + sub * kStep;      // first row (token) of this step in the chunk
      const int tok = chunk_t0 + r0 + tp;                   // this lane's token
      const bool valid = tok < t_end;
      const int row = r0 + tp;
      // ---------------- scores ----------------
      float sc[G];
      if constexpr (!kInt4) {
        int dot[G];
#pragma unroll
        for (int hh = 0; hh < G; ++hh) dot[hh] = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int ch = half * 4 + i;                       // 16-byte chunk of the 128-byte row
          const uint4 kv = *reinterpret_cast<const uint4*>(cK + row * 128 + ((ch ^ (row & 7)) << 4));
#pragma unroll
          for (int hh = 0; hh < G; ++hh) {
            dot[hh] = __dp4a(static_cast<int>(kv.x), qreg[hh][4 * i + 0], dot[hh]);
            dot[hh] = __dp4a(static_cast<int>(kv.y), qreg[hh][4 * i + 1], dot[hh]);
            dot[hh] = __dp4a(static_cast<int>(kv.z), qreg[hh][4 * i + 2], dot[hh]);
            dot[hh] = __dp4a(static_cast<int>(kv.w), qreg[hh][4 * i + 3], dot[hh]);
          }
        }
        const float sk = sKsc[s];
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
          const int full_dot = dot[hh] + __shfl_xor_sync(0xffffffffu, dot[hh], 1);
          sc[hh] = valid ? static_cast<float>(full_dot) * (qf[hh] * sk) : -CUDART_INF_F;
        }
      } else {
        int dot[G];
#pragma unroll
        for (int hh = 0; hh < G; ++hh) dot[hh] = 0;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int ch = half * 2 + i;                       // 16-byte chunk of the 64-byte row
          const uint4 kv = *reinterpret_cast<const uint4*>(cK + row * 64 + ((ch ^ ((row >> 1) & 3)) << 4));
          const uint32_t w4[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
          for (int wi = 0; wi < 4; ++wi) {
            const int ev = static_cast<int>((w4[wi] & 0x0F0F0F0Fu) ^ 0x08080808u);        // code + 8, even channels
            const int od = static_cast<int>(((w4[wi] >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u); // code + 8, odd channels
            const int j = i * 4 + wi;
#pragma unroll
            for (int hh = 0; hh < G; ++hh) {
              dot[hh] = __dp4a(ev, qreg[hh][2 * j], dot[hh]);
              dot[hh] = __dp4a(od, qreg[hh][2 * j + 1], dot[hh]);
            }
          }
        }
        const float skg = __half2float(__ushort_as_half(sKs16[s][row * kGroups + (kGroups == 2 ? half : 0)]));
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
          const float part = static_cast<float>(dot[hh] - 8 * qsum_half[hh]) * skg;
          const float tot = part + __shfl_xor_sync(0xffffffffu, part, 1);
          sc[hh] = valid ? tot * qf[hh] : -CUDART_INF_F;
        }
      }
      // ---------------- running softmax ----------------
      float alpha[G];
      bool any = false;
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        const float step_max = key_float(__reduce_max_sync(0xffffffffu, float_key(sc[hh])));
        const float m_new = fmaxf(m_run[hh], step_max);
        any = step_max != -CUDART_INF_F;
        alpha[hh] = any ? ex2(m_run[hh] - m_new) : 1.0f;
        const float pr = valid ? ex2(sc[hh] - m_new) : 0.0f;
        l_run[hh] = l_run[hh] * alpha[hh] + (half == 0 ? pr : 0.0f);
        if (any) m_run[hh] = m_new;
        float pw = pr;
        if constexpr (!kInt4) {
          pw *= sVsc[s];
        } else if constexpr (kGroups == 1) {
          pw *= __half2float(__ushort_as_half(sVs16[s][row]));
        }
        if (half == 0) sP[warp][tp][hh] = make_float2(pw, pw);
      }
      if constexpr (kInt4 && kGroups == 2) {
        sSV[warp][tp][half] = __half2float(__ushort_as_half(sVs16[s][row * 2 + half]));
      }
      __syncwarp();
      if (!any) continue;            // no valid token in this step (warp-uniform)
      // ---------------- P.V ----------------
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        const float2 a2 = make_float2(alpha[hh], alpha[hh]);
        acc[hh][0] = fmul2(acc[hh][0], a2);
        acc[hh][1] = fmul2(acc[hh][1], a2);
      }
      const uint8_t* vbase = cV + r0 * kRowBytes;
#pragma unroll 4
      for (int t = 0; t < kStep; ++t) {
        float2 v01, v23;
        if constexpr (!kInt4) {
          const uint32_t w = *reinterpret_cast<const uint32_t*>(vbase + t * 128 + (lane_off ^ ((t & 7) << 4)));
          s8x4_to_f32(w, v01, v23);
        } else {
          const uint32_t w = *reinterpret_cast<const uint16_t*>(vbase + t * 64 + (lane_off ^ (((t >> 1) & 3) << 4)));
          s4x4_to_f32(w, v01, v23);
          if constexpr (kGroups == 2) {
            const float sv = sSV[warp][t][my_group];
            v01 = fmul2(v01, make_float2(sv, sv));
            v23 = fmul2(v23, make_float2(sv, sv));
          }
        }
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
          const float2 p2 = sP[warp][t][hh];
          acc[hh][0] = ffma2(p2, v01, acc[hh][0]);
          acc[hh][1] = ffma2(p2, v23, acc[hh][1]);
        }
      }
      __syncwarp();                  // sP / sSV reused by the next step
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }

  // ---------------- merge the four consumer warps ----------------
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    float l = l_run[hh];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    l_run[hh] = l;
  }
  // every issued copy was consumed (or waited for on a timeout): the ring can
  // be reused for the reduction once all consumer warps are past their loops
  named_bar_sync(1, 32 * kConsumers);
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    *reinterpret_cast<float4*>(&sRed[(warp * G + hh) * kD + lane * 4]) =
        make_float4(acc[hh][0].x, acc[hh][0].y, acc[hh][1].x, acc[hh][1].y);
    if (lane == 0) {
      sWm[warp][hh] = m_run[hh];
      sWl[warp][hh] = l_run[hh];
    }
  }
  named_bar_sync(1, 32 * kConsumers);
  for (int i = tid; i < G * kD; i += 32 * kConsumers) {
    const int hh = i / kD, d = i % kD;
    float M = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < kConsumers; ++w) M = fmaxf(M, sWm[w][hh]);
    float o = 0.0f, l = 0.0f;
    if (M != -CUDART_INF_F) {
#pragma unroll
      for (int w = 0; w < kConsumers; ++w) {
        if (sWm[w][hh] == -CUDART_INF_F) continue;
        const float sc = ex2(sWm[w][hh] - M);
        o = fmaf(sc, sRed[(w * G + hh) * kD + d], o);
        l = fmaf(sc, sWl[w][hh], l);
      }
    }
    float* wsp = p.ws + ((static_cast<int64_t>(b) * p.Hq + hk * g + hh) * p.splits + split) * kWsStride;
    wsp[d] = o;
    if (d == 0) {
      wsp[kD] = M;
      wsp[kD + 1] = abort_flag ? 0.0f : l;
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
      const float sc = ex2(w[s * kWsStride + kD] - M);
      num = fmaf(sc, w[s * kWsStride + d], num);
      den = fmaf(sc, l, den);
    }
  }
  out[bh * kD + d] = __float2bfloat16_rn(den > 0.0f ? num / den : 0.0f);
}

// 3-D map {row bytes, L, B*H_kv} over the cache; box {row bytes, chunk, 1}
// with the swizzle the consumers' address arithmetic expects.
template <bool kInt4>
bool make_cache_map(CUtensorMap* m, const void* base, int B, int Hkv, int L) {
  using C = Cfg<kInt4>;
  const uint64_t dims[3] = {static_cast<uint64_t>(C::kRowBytes), static_cast<uint64_t>(L),
                            static_cast<uint64_t>(B) * Hkv};
  const uint64_t strides[2] = {static_cast<uint64_t>(C::kRowBytes), static_cast<uint64_t>(L) * C::kRowBytes};
  const uint32_t box[3] = {static_cast<uint32_t>(C::kRowBytes), static_cast<uint32_t>(C::kChunk), 1};
  return encode_map_u8(m, 3, base, dims, strides, box,
                       kInt4 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B);
}

template <int G, bool kInt4, int kGroups>
cudaError_t launch_g(const DecodeArgs& a, const DecodeParams& p, cudaStream_t st) {
  CUtensorMap mk, mv;
  if (!make_cache_map<kInt4>(&mk, a.k, a.B, a.Hkv, a.L) || !make_cache_map<kInt4>(&mv, a.v, a.B, a.Hkv, a.L))
    return cudaErrorInvalidValue;
  auto k = decode_kernel<G, kInt4, kGroups>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<kInt4>::kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(p.splits, p.Hkv, p.B);
  k<<<grid, kThreads, Cfg<kInt4>::kSmemBytes, st>>>(mk, mv, p);
  return cudaGetLastError();
}

template <bool kInt4, int kGroups>
cudaError_t dispatch_g(const DecodeArgs& a, const DecodeParams& p, cudaStream_t st) {
  switch (a.Hq / a.Hkv) {
    case 1: return launch_g<1, kInt4, kGroups>(a, p, st);
    case 2: return launch_g<2, kInt4, kGroups>(a, p, st);
    case 4: return launch_g<4, kInt4, kGroups>(a, p, st);
    case 8: return launch_g<8, kInt4, kGroups>(a, p, st);
  }
  return cudaErrorInvalidValue;
}

int chunk_tokens(bool int4) { return int4 ? Cfg<true>::kChunk : Cfg<false>::kChunk; }

}  // namespace

bool decode_supported(int D, int group_ratio) { return D == kD && (group_ratio == 1 || group_ratio == 2); }

// Split count: each split is a whole number of chunks (at least 4, to keep
// the ring busy); among the counts that give at least two waves of resident
// CTAs, take the smallest whose last wave is at least 90% full (else the
// fullest). Resident CTAs per SM: 3 (INT8) / 2 (INT4), set by registers and
// shared memory.
static int splits_for(int B, int Hkv, int L, int num_sms, bool int4) {
  const int ck = chunk_tokens(int4);
  const int chunks = (L + ck - 1) / ck;
  if (chunks == 0) return 1;
  const int64_t pairs = static_cast<int64_t>(B) * Hkv;
  const int64_t slots = static_cast<int64_t>(num_sms) * (int4 ? 2 : 3);
  const int max_splits = max(1, min(64, chunks / 4));
  int best = 1;
  double best_fill = -1.0;
  for (int sp = 1; sp <= max_splits; ++sp) {
    const int per = (chunks + sp - 1) / sp;
    const int real = (chunks + per - 1) / per;
    const int64_t total = pairs * real;
    const double waves = static_cast<double>(total) / slots;
    const double fill = waves / std::ceil(waves);
    if (waves >= 2.0 && fill >= 0.9) return real;
    if (fill > best_fill + 1e-9) {
      best_fill = fill;
      best = real;
    }
  }
  return best;
}

int decode_splits(int B, int Hkv, int L, int num_sms) {
  // The workspace is sized for the larger of the two chunkings.
  return max(splits_for(B, Hkv, L, num_sms, false), splits_for(B, Hkv, L, num_sms, true));
}

size_t decode_workspace_bytes(int B, int Hq, int Hkv, int L, int D, int num_sms) {
  (void)D;
  const int splits = decode_splits(B, Hkv, L, num_sms);
  return static_cast<size_t>(B) * Hq * splits * kWsStride * sizeof(float);
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st, int num_sms, int* err) {
  if (a.L == 0) {
    // No keys: the output is defined as zeros.
    return cudaMemsetAsync(a.out, 0, static_cast<size_t>(a.B) * a.Hq * kD * sizeof(__nv_bfloat16), st);
  }
  DecodeParams p;
  p.q = static_cast<const uint16_t*>(a.q);
  p.ks = a.ks;
  p.vs = a.vs;
  p.B = a.B; p.Hq = a.Hq; p.Hkv = a.Hkv; p.L = a.L;
  p.kv_block = a.kv_block; p.group = a.group;
  p.splits = splits_for(a.B, a.Hkv, a.L, num_sms, a.int4 != 0);
  const int ck = chunk_tokens(a.int4 != 0);
  const int chunks = (a.L + ck - 1) / ck;
  p.chunks_per_split = (chunks + p.splits - 1) / p.splits;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.ws = static_cast<float*>(a.workspace);
  p.err = err;
  cudaError_t e;
  if (a.int4) e = (kD / a.group == 2) ? dispatch_g<true, 2>(a, p, st) : dispatch_g<true, 1>(a, p, st);
  else e = dispatch_g<false, 1>(a, p, st);
  if (e != cudaSuccess) return e;
  merge_kernel<<<static_cast<unsigned>(static_cast<int64_t>(a.B) * a.Hq), kD, 0, st>>>(
      p.ws, p.splits, static_cast<__nv_bfloat16*>(a.out));
  return cudaGetLastError();
}

}  // namespace qattn
