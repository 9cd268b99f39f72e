// prefill_bf16.cu -- the dequantize-first path that the pages contrast with
// quantized attention, for measuring that contrast on B200:
//   dequant_bf16_kernel   codes x block scale -> bfloat16 in HBM (the
//                         "INT8 -> FP16" pass)
//   attn_bf16_kernel      softmax(Q K^T * scale) V on bfloat16 Q/K/V with
//                         the 16-bit tensor-core path (tcgen05 kind::f16,
//                         float32 accumulation), probabilities unquantized
//                         (rounded to bfloat16 only as the MMA operand).
//
// Method: "INT8 量化算子", ops-transformer items 1-2: the standard INT8
// path converts INT8 back to FP16 and multiplies in FP16; the optimised one
// feeds INT8 codes to the matrix unit directly. This file is the former, so
// that its cost can be measured beside the latter (prefill.cu).
//
// attn_bf16_kernel: one CTA = two consecutive tiles of 128 query rows (A, B)
// of one (b, h), 12 warps, the roles of prefill.cu:
//   warp 0      TMA producer: both Q tiles once, then K/V tiles of 64 keys
//               (bfloat16 rows are 2D bytes: for D = 128 each tile arrives as
//               two 64-channel boxes, one 128-byte swizzle atom wide each)
//               into a three-stage ring (no multicast).
//   warps 1, 2  MMA issuers of tile A / tile B:
//                 S  = Q K^T  M=128, N=64, K=D  -> TMEM [256x, 256x+64)
//                 PV = P V    M=128, N=D,  K=64 -> TMEM [256x+128, +D)
//               P from shared memory (K-major), V MN-major from its tile.
//   warp 3      idle (completes warpgroup 0 for the register split).
//   warps 4-11  one query row per thread (tile A: 4-7, B: 8-11). Per key
//               tile: row max, probabilities (float32, summed unrounded),
//               P as bfloat16 to shared memory, then PV of the previous tile
//               folded into the float32 output row in registers.
// Every wait is bounded.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math_constants.h>

#include <atomic>

#include "prefill_common.cuh"
#include "qattn_device.cuh"
#include "qattn_internal.h"

namespace qattn {

namespace {

constexpr int kThreadsB = 384;
constexpr int kRegsLowB = 40;
constexpr int kRegsHighB = 232;
constexpr int kRegsNeededB = (128 * kRegsLowB + 256 * kRegsHighB + kThreadsB - 1) / kThreadsB;
constexpr int kTileNB = 64;          // keys per tile (bfloat16: 128 bytes of P per row)

// D bf16 channels per row; tiles are stored as D/64 column blocks of 128-byte
// swizzled rows (one TMA box each).
template <int D>
struct SmemB {
  static constexpr int kCols = D / 64;                 // 128-byte column blocks per row
  static constexpr int kQTile = kTileM * D * 2;
  static constexpr int kKVTile = kTileNB * D * 2;
  static constexpr int kQ = 0;
  static constexpr int kP = kQ + 2 * kQTile;           // two P tiles: 128 rows x 64 bf16
  static constexpr int kK = kP + 2 * kTileM * 128;
  static constexpr int kV = kK + kStagesKV * kKVTile;
  static constexpr int kEnd = kV + kStagesKV * kKVTile;
  static constexpr int kBytes = kEnd + 1024;
};

struct BarsB {
  uint64_t s_full, p_full, pv_full, pv_free;
};

struct AttnBf16Params {
  __nv_bfloat16* out;
  float* lse;
  int B, H, Nq, Nkv;
  int nqt, npairs;
  int causal, layout;
  float scale_log2;
  int* err;
};

// D[tmem] (+)= A[smem] * B[smem]^T, 16-bit operands (kind::f16), one MMA of
// K = 16 elements. Issued by one thread.
__device__ __forceinline__ void mma_f16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

template <int D, bool kPartial>
__device__ __forceinline__ float tile_max_bf(uint32_t tS, int kmax) {
  float f0 = -CUDART_INF_F, f1 = -CUDART_INF_F, f2 = -CUDART_INF_F, f3 = -CUDART_INF_F;
  tmem_chunks<kTileNB / 16, 16>(tS, [&](int c, uint32_t(&v)[16]) {
    if constexpr (kPartial) {
#pragma unroll
      for (int e = 0; e < 16; ++e)
        if (c * 16 + e >= kmax) v[e] = 0xFF800000u;
    }
#pragma unroll
    for (int e = 0; e < 16; e += 8) {
      f0 = fmax3(f0, __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
      f1 = fmax3(f1, __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
      f2 = fmax3(f2, __uint_as_float(v[e + 4]), __uint_as_float(v[e + 5]));
      f3 = fmax3(f3, __uint_as_float(v[e + 6]), __uint_as_float(v[e + 7]));
    }
  });
  return fmaxf(fmaxf(f0, f1), fmaxf(f2, f3));
}

// p = 2^(S * sl2 - m2) for the 64 keys of a tile: bfloat16 pairs to this
// row of P (128 bytes, 16-byte chunk c at c ^ (row % 8)); returns the sum of
// the float32 values.
template <bool kPartial>
__device__ __forceinline__ float tile_probs_bf(uint32_t tS, uint8_t* prow, int rsw, float sl2, float m2, int kmax) {
  const float2 k2 = make_float2(sl2, sl2);
  const float2 t2 = make_float2(-m2, -m2);
  float s0 = 0.0f, s1 = 0.0f;
  tmem_chunks<kTileNB / 16, 16>(tS, [&](int c, uint32_t(&v)[16]) {
    uint32_t w[8];
#pragma unroll
    for (int e = 0; e < 16; e += 2) {
      const float2 t = ffma2(make_float2(__uint_as_float(v[e]), __uint_as_float(v[e + 1])), k2, t2);
      float p0 = ex2(t.x), p1 = ex2(t.y);
      if constexpr (kPartial) {
        p0 = c * 16 + e < kmax ? p0 : 0.0f;
        p1 = c * 16 + e + 1 < kmax ? p1 : 0.0f;
      }
      s0 += p0;
      s1 += p1;
      const __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
      w[e >> 1] = *reinterpret_cast<const uint32_t*>(&b2);
    }
    // keys 16c .. 16c + 15 = 16-byte chunks 2c, 2c + 1 of this row
    *reinterpret_cast<uint4*>(prow + (((2 * c) ^ rsw) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
    *reinterpret_cast<uint4*>(prow + (((2 * c + 1) ^ rsw) << 4)) = make_uint4(w[4], w[5], w[6], w[7]);
  });
  return s0 + s1;
}

// O <- alpha (O + PV) (kScaleO) or O + PV, over the D columns of PV.
template <int D, bool kScaleO>
__device__ __forceinline__ void fold_bf(float (&O)[D], uint32_t tPV, float alpha) {
  const float2 a2 = make_float2(alpha, alpha);
  tmem_chunks<D / 16, 16>(tPV, [&](int i, uint32_t(&pv)[16]) {
#pragma unroll
    for (int e = 0; e < 16; e += 2) {
      const float2 x = make_float2(__uint_as_float(pv[e]), __uint_as_float(pv[e + 1]));
      float2 o = make_float2(O[i * 16 + e], O[i * 16 + e + 1]);
      if constexpr (kScaleO) o = ffma2(x, a2, fmul2(o, a2));
      else o = fadd2(o, x);
      O[i * 16 + e] = o.x;
      O[i * 16 + e + 1] = o.y;
    }
  });
}

// The rows of one query tile (4 warps, one row per thread).
template <int D>
__device__ __forceinline__ void rows_bf(const AttnBf16Params& p, BarsB& bars, uint32_t tS, uint32_t tPV, uint8_t* sP,
                                        int qt, int ntiles, int b, int h, int quarter, int lane,
                                        volatile int* abort_flag) {
  const int r = quarter * 32 + lane;            // row within the tile (= TMEM lane)
  const int q0 = qt * kTileM;
  const int qrow = q0 + r;
  tS += static_cast<uint32_t>(quarter * 32) << 16;
  tPV += static_cast<uint32_t>(quarter * 32) << 16;
  uint8_t* prow = sP + r * 128;
  const int rsw = r & 7;
  float O[D];
#pragma unroll
  for (int d = 0; d < D; ++d) O[d] = 0.0f;
  float m_run = -CUDART_INF_F, l_run = 0.0f;
  bool ok = true;
  for (int j = 0; j < ntiles; ++j) {
    ok = __all_sync(0xffffffffu, mbar_wait(&bars.s_full, j & 1, abort_flag, p.err));
    if (!ok) break;
    tc_fence_after();
    const int key0 = j * kTileNB;
    // masked keys only on the last tile (ragged N_kv) and the causal diagonal
    const bool partial = (key0 + kTileNB > p.Nkv) || (p.causal && key0 + kTileNB - 1 > q0);
    int kmax = p.Nkv - key0;                    // keys valid for this row: [0, kmax)
    if (p.causal) kmax = min(kmax, qrow - key0 + 1);

    // ---- (1) row max, log2 domain ----
    const float smax = partial ? tile_max_bf<D, true>(tS, kmax) : tile_max_bf<D, false>(tS, kmax);
    const float tmax = smax == -CUDART_INF_F ? -CUDART_INF_F : smax * p.scale_log2;
    const float m_new = fmaxf(m_run, tmax);
    const float m_use = m_new == -CUDART_INF_F ? 0.0f : m_new;
    const float alpha = ex2(m_run - m_use);     // 0 on the first tile

    // P_{j-1} must have been consumed (PV_{j-1} complete) before P_j is written.
    if (j > 0) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars.pv_full, (j - 1) & 1, abort_flag, p.err));
      if (!ok) break;
      tc_fence_after();
    }
    // ---- (2) probabilities -> P_j (bfloat16) ----
    const float rowsum = partial ? tile_probs_bf<true>(tS, prow, rsw, p.scale_log2, m_use, kmax)
                                 : tile_probs_bf<false>(tS, prow, rsw, p.scale_log2, m_use, kmax);
    fence_proxy_async_smem();
    tc_fence_before();
    mbar_arrive(&bars.p_full);
    l_run = l_run * alpha + rowsum;
    m_run = m_new;

    // ---- (3) fold PV_{j-1}: O <- alpha_j (O + PV_{j-1}) ----
    if (j > 0) {
      if (__all_sync(0xffffffffu, alpha == 1.0f)) fold_bf<D, false>(O, tPV, alpha);
      else fold_bf<D, true>(O, tPV, alpha);
      tc_fence_before();
      mbar_arrive(&bars.pv_free);
    }
  }
  if (!ok || ntiles == 0) return;
  ok = __all_sync(0xffffffffu, mbar_wait(&bars.pv_full, (ntiles - 1) & 1, abort_flag, p.err));
  if (!ok) return;
  tc_fence_after();
  fold_bf<D, false>(O, tPV, 1.0f);

  if (qrow < p.Nq) {
    const float inv_l = l_run > 0.0f ? 1.0f / l_run : 0.0f;
    __nv_bfloat16* orow = p.out + row_offset(p.layout, p.H, p.Nq, D, b, h, qrow);
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
      uint32_t w4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const __nv_bfloat162 t = __floats2bfloat162_rn(O[c * 8 + 2 * e] * inv_l, O[c * 8 + 2 * e + 1] * inv_l);
        w4[e] = *reinterpret_cast<const uint32_t*>(&t);
      }
      *reinterpret_cast<uint4*>(orow + c * 8) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
    }
    if (p.lse) p.lse[(static_cast<int64_t>(b) * p.H + h) * p.Nq + qrow] = m_run * 0.6931471805599453f + logf(l_run);
  }
}

// Grid: one CTA per pair of consecutive query tiles of one (b, h): the pairs
// with the most key tiles first (causal), else head-major.
template <int D>
__global__ void __launch_bounds__(kThreadsB, 1)
    attn_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const AttnBf16Params p) {
  using L = SmemB<D>;
  constexpr int kColBytesQ = kTileM * 128;          // one 128-byte column block of a Q tile
  constexpr int kColBytesKV = kTileNB * 128;        // ... of a K/V tile
  // S = Q K^T: A = Q (K-major), B = K (K-major); BF16 x BF16 -> F32.
  constexpr uint32_t kIdescQK = instr_desc(1u, 1u, 1u, 0u, 0u, kTileNB, kTileM);
  // PV = P V: A = P (K-major over keys), B = V (MN-major), N = D.
  constexpr uint32_t kIdescPV = instr_desc(1u, 1u, 1u, 0u, 1u, D, kTileM);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + L::kQ;
  uint8_t* sP = smem + L::kP;
  uint8_t* sK = smem + L::kK;
  uint8_t* sV = smem + L::kV;

  __shared__ __align__(8) uint64_t bar_q_full;
  __shared__ __align__(8) uint64_t bar_kv_full[kStagesKV];
  __shared__ __align__(8) uint64_t bar_kv_empty[kStagesKV];
  __shared__ __align__(8) BarsB bars[2];
  __shared__ __align__(8) uint64_t bar_drain[2];
  __shared__ uint32_t tmem_base_slot;
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int BH = p.B * p.H;
  const int pair = p.causal ? p.npairs - 1 - static_cast<int>(blockIdx.x) / BH
                            : static_cast<int>(blockIdx.x) % p.npairs;
  const int bh = p.causal ? static_cast<int>(blockIdx.x) % BH : static_cast<int>(blockIdx.x) / p.npairs;
  const int b = bh / p.H, h = bh % p.H;
  const int qt2[2] = {2 * pair, 2 * pair + 1 < p.nqt ? 2 * pair + 1 : -1};
  const int nkt_all = (p.Nkv + kTileNB - 1) / kTileNB;
  int nt2[2];
#pragma unroll
  for (int x = 0; x < 2; ++x)
    nt2[x] = qt2[x] < 0 ? 0 : (p.causal ? min(nkt_all, (qt2[x] * kTileM + kTileM - 1) / kTileNB + 1) : nkt_all);
  const int nt_max = max(nt2[0], nt2[1]);

  if (threadIdx.x == 0) {
    mbar_init(&bar_q_full, 1);
    for (int s = 0; s < kStagesKV; ++s) {
      mbar_init(&bar_kv_full[s], 1);
      mbar_init(&bar_kv_empty[s], 2);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars[x].s_full, 1);
      mbar_init(&bars[x].p_full, 128);
      mbar_init(&bars[x].pv_full, 1);
      mbar_init(&bars[x].pv_free, 128);
    }
    mbar_init(&bar_drain[0], 1);
    mbar_init(&bar_drain[1], 1);
    abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    regs_dec<kRegsLowB>();
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(&bar_q_full, (qt2[1] >= 0 ? 2 : 1) * L::kQTile);
      for (int x = 0; x < 2; ++x)
        if (qt2[x] >= 0)
          for (int cb = 0; cb < L::kCols; ++cb)
            tma_load_4d(sQ + x * L::kQTile + cb * kColBytesQ, &tmQ, &bar_q_full, cb * 64, qt2[x] * kTileM, h, b);
    }
    int j = 0;
    for (; j < nt_max; ++j) {
      const int st = j % kStagesKV;
      if (j >= kStagesKV) {
        const bool ok = mbar_wait(&bar_kv_empty[st], ((j / kStagesKV) - 1) & 1, &abort_flag, p.err);
        if (!__all_sync(0xffffffffu, ok)) break;
      }
      if (lane == 0) {
        mbar_arrive_expect_tx(&bar_kv_full[st], 2 * L::kKVTile);
        for (int cb = 0; cb < L::kCols; ++cb) {
          tma_load_4d(sK + st * L::kKVTile + cb * kColBytesKV, &tmK, &bar_kv_full[st], cb * 64, j * kTileNB, h, b);
          tma_load_4d(sV + st * L::kKVTile + cb * kColBytesKV, &tmV, &bar_kv_full[st], cb * 64, j * kTileNB, h, b);
        }
      }
      __syncwarp();
    }
    if (abort_flag && lane == 0) {
      mbar_wait(&bar_q_full, 0, nullptr, nullptr, 100000000ull);
      for (int i = max(0, j - kStagesKV); i < j; ++i)
        mbar_wait(&bar_kv_full[i % kStagesKV], (i / kStagesKV) & 1, nullptr, nullptr, 100000000ull);
    }
    __syncwarp();
  } else if (warp == 1 || warp == 2) {
    // ------------------------------------------------------------ MMA issuers
    // Per key tile j: S(j+1) once P(j) is written (S free) and K/V(j+1) has
    // landed; PV(j) once PV(j-1) has been read; then K/V stage j is released.
    regs_dec<kRegsLowB>();
    const int x = warp - 1;
    const int nt = nt2[x];
    const uint32_t aQ = smem_u32(sQ) + x * L::kQTile, aP = smem_u32(sP) + x * kTileM * 128;
    const uint32_t aK = smem_u32(sK), aV = smem_u32(sV);
    const uint32_t tS = tmem + x * 256, tPV = tmem + x * 256 + 128;
    BarsB& tb = bars[x];
    auto issue_s = [&](int jj) {
      if (lane == 0) {
        const uint32_t kbase = aK + (jj % kStagesKV) * L::kKVTile;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          // 16 channels = 32 bytes of 128-byte column block kk / 4
          const uint32_t off = (kk & 3) * 32;
          const uint64_t da = smem_desc(aQ + (kk >> 2) * kColBytesQ + off, 16, 1024, 2u);
          const uint64_t db = smem_desc(kbase + (kk >> 2) * kColBytesKV + off, 16, 1024, 2u);
          mma_f16_ss(tS, da, db, kIdescQK, kk > 0 ? 1u : 0u);
        }
        mma_commit(&tb.s_full);
      }
      __syncwarp();
    };
    bool ok = nt == 0 || __all_sync(0xffffffffu, mbar_wait(&bar_q_full, 0, &abort_flag, p.err));
    for (int j = 0; ok && j < nt_max; ++j) {
      const int st = j % kStagesKV;
      ok = __all_sync(0xffffffffu, mbar_wait(&bar_kv_full[st], (j / kStagesKV) & 1, &abort_flag, p.err));
      if (!ok) break;
      if (j >= nt) {
        if (lane == 0) mbar_arrive(&bar_kv_empty[st]);
        __syncwarp();
        continue;
      }
      if (j == 0) {
        tc_fence_after();
        issue_s(0);
      }
      ok = __all_sync(0xffffffffu, mbar_wait(&tb.p_full, j & 1, &abort_flag, p.err));
      if (!ok) break;
      if (j + 1 < nt) {
        const int j1 = j + 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&bar_kv_full[j1 % kStagesKV], (j1 / kStagesKV) & 1, &abort_flag, p.err));
        if (!ok) break;
        tc_fence_after();
        issue_s(j1);
      }
      if (j > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(&tb.pv_free, (j - 1) & 1, &abort_flag, p.err));
        if (!ok) break;
      }
      tc_fence_after();
      if (lane == 0) {
        const uint32_t vbase = aV + st * L::kKVTile;
#pragma unroll
        for (int kk = 0; kk < kTileNB / 16; ++kk) {
          const uint64_t da = smem_desc(aP + kk * 32, 16, 1024, 2u);
          // MN-major V: 16 keys per MMA = 2 groups of 8 key rows (SBO apart);
          // the channel column blocks of the tile are kColBytesKV apart (LBO)
          const uint64_t db = smem_desc(vbase + kk * 16 * 128, kColBytesKV, 1024, 2u);
          mma_f16_ss(tPV, da, db, kIdescPV, kk > 0 ? 1u : 0u);
        }
        mma_commit(&tb.pv_full);
        mma_commit(&bar_kv_empty[st]);
      }
      __syncwarp();
    }
    if (abort_flag && lane == 0) {
      mma_commit(&bar_drain[x]);
      mbar_wait(&bar_drain[x], 0, nullptr, nullptr, 100000000ull);
    }
    __syncwarp();
  } else if (warp == 3) {
    regs_dec<kRegsLowB>();
  } else {
    // ------------------------------------------------------------ softmax rows
    regs_inc<kRegsHighB>();
    const int x = (warp - 4) >> 2;
    if (qt2[x] >= 0)
      rows_bf<D>(p, bars[x], tmem + x * 256, tmem + x * 256 + 128, sP + x * kTileM * 128, qt2[x], nt2[x], b, h,
                 warp & 3, lane, &abort_flag);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// out[i] = bf16(RN(code[i] * scale[b, h, token / block])), 16 codes per
// thread (16-byte load, two 16-byte stores).
template <bool kInt8>
__global__ void __launch_bounds__(256)
    dequant_bf16_kernel(const uint8_t* __restrict__ codes, const float* __restrict__ scales, int layout, int H,
                        int N, int D, int block, int nblk, int64_t n16, __nv_bfloat16* __restrict__ out) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n16;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t e0 = i * 16;
    const int64_t row = e0 / D;                       // token row of the layout
    int64_t bb, hh, t;
    if (layout == 0) {                                 // BNSD: row = (b * H + h) * N + t
      t = row % N;
      hh = (row / N) % H;
      bb = row / (static_cast<int64_t>(N) * H);
    } else {                                           // BSND: row = (b * N + t) * H + h
      hh = row % H;
      t = (row / H) % N;
      bb = row / (static_cast<int64_t>(N) * H);
    }
    const float s = scales[(bb * H + hh) * nblk + t / block];
    const uint4 c = *reinterpret_cast<const uint4*>(codes + e0);
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
    uint32_t o[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float f[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t byte = (w[k] >> (8 * e)) & 0xFFu;
        if constexpr (kInt8) {
          f[e] = static_cast<float>(static_cast<int8_t>(byte));
        } else {
          const uint32_t h2 = cvt_e4m3x2_to_f16x2(static_cast<uint16_t>(byte));
          f[e] = __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
        }
      }
      const __nv_bfloat162 a = __floats2bfloat162_rn(f[0] * s, f[1] * s);
      const __nv_bfloat162 bq = __floats2bfloat162_rn(f[2] * s, f[3] * s);
      o[2 * k] = *reinterpret_cast<const uint32_t*>(&a);
      o[2 * k + 1] = *reinterpret_cast<const uint32_t*>(&bq);
    }
    uint4* dst = reinterpret_cast<uint4*>(out + e0);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

// 4-D map {D, N, H, B} over bfloat16; box {64, rows, 1, 1} with the 128-byte
// swizzle (one 128-byte column block of a tile per load).
bool make_map_bf16(CUtensorMap* m, const void* base, int layout, int B, int H, int N, int D, int rows) {
  const uint64_t dims[4] = {static_cast<uint64_t>(D), static_cast<uint64_t>(N), static_cast<uint64_t>(H),
                            static_cast<uint64_t>(B)};
  uint64_t strides[3];
  if (layout == 0) {
    strides[0] = static_cast<uint64_t>(D) * 2;
    strides[1] = static_cast<uint64_t>(N) * D * 2;
    strides[2] = static_cast<uint64_t>(H) * N * D * 2;
  } else {
    strides[0] = static_cast<uint64_t>(H) * D * 2;
    strides[1] = static_cast<uint64_t>(D) * 2;
    strides[2] = static_cast<uint64_t>(N) * H * D * 2;
  }
  const uint32_t box[4] = {64u, static_cast<uint32_t>(rows), 1, 1};
  return encode_map_u16(m, 4, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

template <int D>
cudaError_t launch_attn_bf16_d(const AttnBf16Args& a, cudaStream_t st, int* err) {
  CUtensorMap mq, mk, mv;
  if (!make_map_bf16(&mq, a.q, a.layout, a.B, a.H, a.Nq, D, kTileM) ||
      !make_map_bf16(&mk, a.k, a.layout, a.B, a.H, a.Nkv, D, kTileNB) ||
      !make_map_bf16(&mv, a.v, a.layout, a.B, a.H, a.Nkv, D, kTileNB))
    return cudaErrorInvalidValue;
  AttnBf16Params p;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.lse = a.lse;
  p.B = a.B; p.H = a.H; p.Nq = a.Nq; p.Nkv = a.Nkv;
  p.nqt = (a.Nq + kTileM - 1) / kTileM;
  p.npairs = (p.nqt + 1) / 2;
  p.causal = a.causal;
  p.layout = a.layout;
  p.scale_log2 = a.scale_log2;
  p.err = err;
  auto k = attn_bf16_kernel<D>;
  constexpr int kSmem = SmemB<D>::kBytes;
  cudaError_t e = set_max_dyn_smem(reinterpret_cast<const void*>(k), kSmem);
  if (e != cudaSuccess) return e;
  static std::atomic<int> regs{-1};
  if (regs.load() < 0) {
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, k);
    if (e != cudaSuccess) return e;
    regs.store(fa.numRegs);
  }
  if (regs.load() < kRegsNeededB) return cudaErrorInvalidConfiguration;
  const int64_t grid = static_cast<int64_t>(p.npairs) * a.B * a.H;
  k<<<static_cast<unsigned>(grid), kThreadsB, kSmem, st>>>(mq, mk, mv, p);
  return cudaGetLastError();
}

}  // namespace

bool attn_bf16_supported(int D) { return D == 64 || D == 128; }

cudaError_t launch_attn_bf16(const AttnBf16Args& a, cudaStream_t st, int* err) {
  if (a.D == 128) return launch_attn_bf16_d<128>(a, st, err);
  if (a.D == 64) return launch_attn_bf16_d<64>(a, st, err);
  return cudaErrorInvalidValue;
}

cudaError_t launch_dequant_bf16(const DequantArgs& a, cudaStream_t st, int num_sms) {
  const int64_t n16 = static_cast<int64_t>(a.B) * a.H * a.N * a.D / 16;
  if (n16 == 0) return cudaSuccess;
  const int nblk = (a.N + a.block - 1) / a.block;
  const int64_t want = (n16 + 255) / 256;
  const unsigned grid = static_cast<unsigned>(want < 8LL * num_sms ? want : 8LL * num_sms);
  if (a.int8)
    dequant_bf16_kernel<true><<<grid, 256, 0, st>>>(static_cast<const uint8_t*>(a.codes), a.scales, a.layout, a.H,
                                                     a.N, a.D, a.block, nblk, n16, static_cast<__nv_bfloat16*>(a.out));
  else
    dequant_bf16_kernel<false><<<grid, 256, 0, st>>>(static_cast<const uint8_t*>(a.codes), a.scales, a.layout, a.H,
                                                      a.N, a.D, a.block, nblk, n16, static_cast<__nv_bfloat16*>(a.out));
  return cudaGetLastError();
}

}  // namespace qattn
