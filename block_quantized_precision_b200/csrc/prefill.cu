// prefill.cu -- quantized attention on 5th-generation tensor cores (tcgen05).
//
// Method: "MindIE-SD quantization", FA量化 / FP8 Attention (attention in the
// FP8 domain, output dequantized to the original precision); "INT8 量化算子",
// ops-transformer items 1-2 (INT8 x INT8 -> INT32 on the matrix unit with no
// input dequantization, one conversion at the output, scales kept on chip);
// "FlashAttention 的 INT8/INT4 量化", 三层实现详解 (outer loop over query
// tiles, inner loop over key/value tiles with a running softmax; the page's
// normalisation is replaced by the standard running-max form).
//
// One CTA = two consecutive tiles of 128 query rows (A, B) of one (b, h);
// one CTA per SM (all 512 TMEM columns, ~161 KB of shared memory at D = 128),
// 12 warps.
//   warp 0      TMA producer: both Q tiles once, then K/V tiles of 128 keys
//               into a three-stage ring (128B / 64B swizzle, no multicast).
//   warps 1, 2  MMA issuers of tile A and tile B (warp 1 also allocates
//               TMEM); one lane each, so neither tile waits for the other:
//                 S_x  = Q_x K_j^T   M=128, N=128, K=D   -> TMEM [256x, 256x+128)
//                 PV_x = P_x V_j     M=128, N=D,   K=128 -> TMEM [256x+128, +D)
//               kind::i8 (s32 accumulate) or kind::f8f6f4 (e4m3, f32). P is
//               read from shared memory (K-major); V is used MN-major straight
//               from its token-major tile.
//   warp 3      idle (it completes warpgroup 0 for the register split).
//   warps 4-7   tile A, warps 8-11 tile B: one query row per thread. Per key
//               tile j: (1) row max of S_j, (2) probabilities in the log2
//               domain, rounded to 8 bits (e4m3, or RNE(127 p) for INT8),
//               written to shared memory in the swizzled K-major layout --
//               from here the tensor core may compute S_{j+1}; (3) PV_{j-1}
//               folded into the float32 output held in registers -- from
//               here it may compute PV_j. Finally O / l as bfloat16 (and the
//               LSE).
// With two tiles per CTA the tensor core works on one tile's products while
// the other tile's rows are in their softmax. With FP8 codes the two tiles
// also take turns in step (2), so one tile's row max and fold overlap the
// other's exponentials. Every wait is bounded.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math_constants.h>

#include <atomic>
#include <climits>

#include "prefill_common.cuh"
#include "qattn_device.cuh"
#include "qattn_internal.h"

namespace qattn {

namespace {

constexpr int kThreads = 384;   // 12 warps = 3 warpgroups
// Register split (setmaxnreg): the launch gives every thread the kernel's register count (168);
// warpgroup 0 (TMA, two MMA issuers, one idle warp) drops to kRegsLow so that the two
// row warpgroups can rise to kRegsHigh (each row thread keeps its 128-float
// output row in registers). 128 * kRegsLow + 256 * kRegsHigh must not exceed
// 384 * (registers per thread at launch); the host checks this before every
// launch.
constexpr int kRegsLow = 40;
constexpr int kRegsHigh = 232;
constexpr int kRegsNeeded = (128 * kRegsLow + 256 * kRegsHigh + kThreads - 1) / kThreads;
// Of the 8 pairs of scores in a 16-key chunk, those whose bit is set here
// get their exponentials from a polynomial on the FMA pipe instead of MUFU.
// Measured: one pair in eight shortens the FP8 probability pass (MUFU is
// its busiest unit); the INT8 pass, with its integer-to-float conversions
// and rounding on the FMA pipe, is fastest with none.
template <bool kPInt8>
constexpr uint32_t kPolyPairs = kPInt8 ? 0x00u : 0x02u;
// Whether the two tiles of a CTA take turns in the probability pass.
// Measured: FP8, whose pass is MUFU-heavy (exponentials and e4m3
// conversions), gains from it; INT8 loses, its pass being bound by integer
// and float32 issue that the other tile's row max and fold compete for.
template <bool kPInt8>
constexpr bool kPingPong = !kPInt8;

// kQKCode / kVCode: code type of Q and K / of V (0 e4m3, 1 INT8, 2 packed
// INT4 widened to INT8 on chip).
template <int D, int kQKCode, int kVCode>
struct Smem {
  static constexpr bool kK4 = kQKCode == 2, kV4 = kVCode == 2;
  static constexpr int kTileBytes = kTileM * D;       // one 128-row tile of 8-bit codes
  static constexpr int kQTileBytes = kK4 ? kTileM * D / 2 : kTileBytes;    // one Q tile as loaded
  static constexpr int kKTileBytes = kK4 ? kTileN * D / 2 : kTileBytes;    // one K tile as loaded
  static constexpr int kVTileBytes = kV4 ? kTileN * D / 2 : kTileBytes;    // one V tile as loaded
  static constexpr int kQ = 0;                        // two Q tiles (8-bit codes)
  static constexpr int kP = kQ + 2 * kTileBytes;      // two P tiles: 128 rows x 128 keys
  static constexpr int kK = kP + 2 * kTileM * kTileN; // K stages as loaded
  static constexpr int kV = kK + kStagesKV * kKTileBytes;
  static constexpr int kW = kV + kStagesKV * kVTileBytes;        // INT4 V: two widened tiles
  static constexpr int kKw = kW + (kV4 ? 2 * kTileBytes : 0);    // INT4 K: two widened tiles
  static constexpr int kQp = kKw + (kK4 ? 2 * kTileBytes : 0);   // INT4 Q: the two packed tiles
  static constexpr int kEnd = kQp + (kK4 ? 2 * kQTileBytes : 0);
  static constexpr int kBytes = kEnd + 1024;          // slack for 1024-byte alignment
};

struct TileBars {
  uint64_t s_full;    // S_j in TMEM               (MMA commit)
  uint64_t p_full;    // P_j in shared memory      (128 row threads)
  uint64_t pv_full;   // PV_j in TMEM              (MMA commit)
  uint64_t pv_free;   // PV_j read by the rows     (128 row threads)
  uint64_t turn;      // the other tile's probability pass is done (its 128 row threads)
};

// Columns per TMEM load in the fold and in the row max (double-buffered).
constexpr int kFoldW = 16;
constexpr int kMaxW = 16;

template <int D, bool kPInt8, bool kScaleO>
__device__ __forceinline__ void fold_pv(float (&O)[D], uint32_t tPV, float alpha, float g) {
  const float2 a2 = make_float2(alpha, alpha);
  const float2 g2 = make_float2(g, g);
  tmem_chunks<D / kFoldW, kFoldW>(tPV, [&](int i, uint32_t(&pv)[kFoldW]) {
#pragma unroll
    for (int e = 0; e < kFoldW; e += 2) {
      const float2 x = kPInt8 ? s32x2_to_f32x2(pv[e], pv[e + 1])
                             : make_float2(__uint_as_float(pv[e]), __uint_as_float(pv[e + 1]));
      float2 o = make_float2(O[i * kFoldW + e], O[i * kFoldW + e + 1]);
      if constexpr (kScaleO) o = fmul2(o, a2);
      o = ffma2(x, g2, o);
      O[i * kFoldW + e] = o.x;
      O[i * kFoldW + e + 1] = o.y;
    }
  });
}

// Row max of one 128-key tile of S, scaled: INT8 the integer max of the
// INT32 scores, FP8 the float max; keys >= kmax are masked when kPartial.
// Returns -inf if every key is masked.
template <bool kInt8, bool kPartial>
__device__ __forceinline__ float tile_row_max(uint32_t tS, int kmax, float ksc, int sub) {
  if constexpr (kInt8) {
    int i0 = INT_MIN, i1 = INT_MIN, i2 = INT_MIN, i3 = INT_MIN;
    tmem_chunks<kTileN / kMaxW, kMaxW>(tS, [&](int c, uint32_t(&v)[kMaxW]) {
      if constexpr (kPartial) {
#pragma unroll
        for (int e = 0; e < kMaxW; ++e)
          if (c * kMaxW + e >= kmax) v[e] = 0x80000000u;
      }
#pragma unroll
      for (int e = 0; e < kMaxW; e += 4) {
        i0 = max(i0, static_cast<int>(v[e]));
        i1 = max(i1, static_cast<int>(v[e + 1]));
        i2 = max(i2, static_cast<int>(v[e + 2]));
        i3 = max(i3, static_cast<int>(v[e + 3]));
      }
    });
    const int im = max(max(i0, i1), max(i2, i3));
    return im == INT_MIN ? -CUDART_INF_F : static_cast<float>(im - sub) * ksc;
  } else {
    float f0 = -CUDART_INF_F, f1 = -CUDART_INF_F, f2 = -CUDART_INF_F, f3 = -CUDART_INF_F;
    tmem_chunks<kTileN / kMaxW, kMaxW>(tS, [&](int c, uint32_t(&v)[kMaxW]) {
      if constexpr (kPartial) {
#pragma unroll
        for (int e = 0; e < kMaxW; ++e)
          if (c * kMaxW + e >= kmax) v[e] = 0xFF800000u;        // -inf
      }
#pragma unroll
      for (int e = 0; e < kMaxW; e += 8) {
        f0 = fmax3(f0, __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
        f1 = fmax3(f1, __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
        f2 = fmax3(f2, __uint_as_float(v[e + 4]), __uint_as_float(v[e + 5]));
        f3 = fmax3(f3, __uint_as_float(v[e + 6]), __uint_as_float(v[e + 7]));
      }
    });
    const float fm = fmaxf(fmaxf(f0, f1), fmaxf(f2, f3));
    return fm == -CUDART_INF_F ? -CUDART_INF_F : fm * ksc;
  }
}

// Probabilities of one 128-key tile, rounded to 8 bits and written to this
// row of P in shared memory (128-byte swizzled K-major rows); returns the row
// sum of the rounded values. t = S * ksc + toff; INT8: code = RNE(2^t) with
// toff = log2(127) - m (so 2^t = 127 p); FP8: e4m3(2^t) with toff = -m.
template <bool kSInt8, bool kPInt8, bool kPartial>
__device__ __forceinline__ float tile_probs(uint32_t tS, uint8_t* prow, int rsw, float ksc, float toff, int kmax) {
  const float2 k2 = make_float2(ksc, ksc);
  const float2 t2 = make_float2(toff, toff);
  int ri0 = 0, ri1 = 0;
  float rf0 = 0.0f, rf1 = 0.0f, rf2 = 0.0f, rf3 = 0.0f;
  tmem_chunks<kTileN / 16, 16>(tS, [&](int c, uint32_t(&v)[16]) {
    uint32_t packed[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      float2 t01, t23;
      if constexpr (kSInt8) {
        t01 = ffma2(s32x2_to_f32x2(v[4 * w], v[4 * w + 1]), k2, t2);
        t23 = ffma2(s32x2_to_f32x2(v[4 * w + 2], v[4 * w + 3]), k2, t2);
      } else {
        t01 = ffma2(make_float2(__uint_as_float(v[4 * w]), __uint_as_float(v[4 * w + 1])), k2, t2);
        t23 = ffma2(make_float2(__uint_as_float(v[4 * w + 2]), __uint_as_float(v[4 * w + 3])), k2, t2);
      }
      // the pairs marked in kPolyPairs go to the FMA pipe, the rest to MUFU
      float pr[4];
      if ((kPolyPairs<kPInt8> >> (2 * w)) & 1) {
        const float2 e = exp2_poly2(t01);
        pr[0] = e.x;
        pr[1] = e.y;
      } else {
        pr[0] = ex2(t01.x);
        pr[1] = ex2(t01.y);
      }
      if ((kPolyPairs<kPInt8> >> (2 * w + 1)) & 1) {
        const float2 e = exp2_poly2(t23);
        pr[2] = e.x;
        pr[3] = e.y;
      } else {
        pr[2] = ex2(t23.x);
        pr[3] = ex2(t23.y);
      }
      if constexpr (kPartial) {
#pragma unroll
        for (int e = 0; e < 4; ++e) pr[e] = c * 16 + w * 4 + e < kmax ? pr[e] : 0.0f;
      }
      if constexpr (kPInt8) {
        // adding 1.5 * 2^23 rounds to an integer (half to even) and leaves it
        // in the low mantissa byte
        const float2 q01 = fadd2(make_float2(pr[0], pr[1]), make_float2(12582912.0f, 12582912.0f));
        const float2 q23 = fadd2(make_float2(pr[2], pr[3]), make_float2(12582912.0f, 12582912.0f));
        const uint32_t b01 = __byte_perm(__float_as_uint(q01.x), __float_as_uint(q01.y), 0x0040);
        const uint32_t b23 = __byte_perm(__float_as_uint(q23.x), __float_as_uint(q23.y), 0x0040);
        const uint32_t word = __byte_perm(b01, b23, 0x5410);
        if (w & 1) ri1 = __dp4a(static_cast<int>(word), 0x01010101, ri1);
        else ri0 = __dp4a(static_cast<int>(word), 0x01010101, ri0);
        packed[w] = word;
      } else {
        const uint32_t lo = cvt_e4m3x2(pr[0], pr[1]);
        const uint32_t hi = cvt_e4m3x2(pr[2], pr[3]);
        packed[w] = lo | (hi << 16);
        // row sum of the rounded probabilities (exact values via fp16)
        if (w & 1) {
          rf2 = add_f32_f16x2(cvt_e4m3x2_to_f16x2(static_cast<uint16_t>(lo)), rf2);
          rf3 = add_f32_f16x2(cvt_e4m3x2_to_f16x2(static_cast<uint16_t>(hi)), rf3);
        } else {
          rf0 = add_f32_f16x2(cvt_e4m3x2_to_f16x2(static_cast<uint16_t>(lo)), rf0);
          rf1 = add_f32_f16x2(cvt_e4m3x2_to_f16x2(static_cast<uint16_t>(hi)), rf1);
        }
      }
    }
    // keys 16c .. 16c+15 = 16-byte chunk c of this row
    *reinterpret_cast<uint4*>(prow + ((c ^ rsw) << 4)) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
  });
  return kPInt8 ? static_cast<float>(ri0 + ri1) * (1.0f / 127.0f) : (rf0 + rf1) + (rf2 + rf3);
}

// The rows of one query tile (4 warps, one row per thread).
//
// The two tiles of a CTA take turns in pass (2), which keeps the MUFU unit
// busiest: A(0), B(0), A(1), B(1), ... Each tile's row max and fold run while
// the other tile computes its probabilities. Tile A waits before pass (2) of
// tile j for B's pass of tile j - 1, tile B for A's pass of tile j; a tile
// arrives only where its partner will wait (the causal tile B has one key
// tile more than A, and a pair may lack B).
// kVBias: V arrives as code + 8 (INT4 widened to unsigned bytes); the
// output then carries 8 * g * (sum of the row's P codes) per tile in every
// channel, which the scalar C accumulates with the same rescaling as O and
// removes at the end (O_true = O + C).
// kKBias: K arrives as code + 8 (INT4 widened to unsigned bytes); every
// score of row i then carries 8 * sum_d Q[i][d], subtracted with the scale
// (q_wide: completes when the widened Q tile qrows is in shared memory).
template <int D, bool kSInt8, bool kPInt8, bool kVBias, bool kKBias>
__device__ __forceinline__ void tile_rows(const PrefillParams& p, TileBars& bars, TileBars& partner, uint32_t tS,
                                          uint32_t tPV, uint8_t* sP, const float* sKsc, const float* sVsc, int qt,
                                          int ntiles, int x, int nt_partner, int bh, int b, int h, int quarter,
                                          int lane, volatile int* abort_flag, uint64_t* q_wide,
                                          const uint8_t* qrows) {
  const int r = quarter * 32 + lane;            // row within the tile (= TMEM lane)
  const int q0 = qt * kTileM;
  const int qrow = q0 + r;
  tS += static_cast<uint32_t>(quarter * 32) << 16;
  tPV += static_cast<uint32_t>(quarter * 32) << 16;
  const float sq = p.qs[static_cast<int64_t>(bh) * p.nqb + qt];
  uint8_t* prow = sP + r * 128;
  const int rsw = r & 7;

  float O[D];
#pragma unroll
  for (int d = 0; d < D; ++d) O[d] = 0.0f;
  float m_run = -CUDART_INF_F, l_run = 0.0f;
  float g_prev = 0.0f;                          // V dequantization factor of the previous tile
  float r_prev = 0.0f;                          // kVBias: sum of the previous tile's P codes
  float C = 0.0f;                               // kVBias: -8 * accumulated g * P-code sums
  bool ok = true;
  int sub = 0;                                  // kKBias: 8 * sum of this row's Q codes
  if constexpr (kKBias) {
    ok = __all_sync(0xffffffffu, mbar_wait(q_wide, 0, abort_flag, p.err));
    if (!ok) return;
    const int* qr = reinterpret_cast<const int*>(qrows + r * D);   // (chunk order does not matter)
#pragma unroll
    for (int w = 0; w < D / 4; ++w) sub = __dp4a(qr[w], 0x01010101, sub);
    sub *= 8;
  }
  for (int j = 0; j < ntiles; ++j) {
    ok = __all_sync(0xffffffffu, mbar_wait(&bars.s_full, j & 1, abort_flag, p.err));
    if (!ok) break;
    tc_fence_after();
    const int blk = j >> 1;
    const float kscale = blk < kMaxBlk ? sKsc[blk] : p.ks[static_cast<int64_t>(bh) * p.nkb + blk];
    const float vscale = blk < kMaxBlk ? sVsc[blk] : p.vs[static_cast<int64_t>(bh) * p.nkb + blk];
    const float ksc = sq * kscale * p.scale_log2;
    const int key0 = j * kTileN;
    // Only the last tile (ragged N_kv) and the causal diagonal tiles have
    // masked keys; the mask is applied on those tiles only (warp-uniform).
    const bool partial = (key0 + kTileN > p.Nkv) || (p.causal && key0 + kTileN - 1 > q0);
    int kmax = p.Nkv - key0;                    // keys valid for this row: [0, kmax)
    if (p.causal) kmax = min(kmax, qrow - key0 + 1);

    // ---- (1) row max ----
    const float tmax = partial ? tile_row_max<kSInt8, true>(tS, kmax, ksc, sub)
                               : tile_row_max<kSInt8, false>(tS, kmax, ksc, sub);
    const float m_new = fmaxf(m_run, tmax);
    const float m_use = m_new == -CUDART_INF_F ? 0.0f : m_new;
    const float alpha = ex2(m_run - m_use);     // 0 on the first tile

    // P_{j-1} must have been consumed (PV_{j-1} complete) before P_j is written.
    if (j > 0) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars.pv_full, (j - 1) & 1, abort_flag, p.err));
      if (!ok) break;
      tc_fence_after();
    }

    // ---- (2) probabilities, 8-bit rounding, P to shared memory ----
    const bool my_turn_waits = kPingPong<kPInt8> && (x == 0 ? (j >= 1 && j - 1 < nt_partner) : (j < nt_partner));
    if (my_turn_waits) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars.turn, (x == 0 ? j - 1 : j) & 1, abort_flag, p.err));
      if (!ok) break;
    }
    // (kKBias: the scores' offset 8 * sum(Q codes) leaves with the scale)
    const float toff = (kPInt8 ? kLog2_127 : 0.0f) - m_use - (kKBias ? static_cast<float>(sub) * ksc : 0.0f);
    const float rowsum = partial ? tile_probs<kSInt8, kPInt8, true>(tS, prow, rsw, ksc, toff, kmax)
                                 : tile_probs<kSInt8, kPInt8, false>(tS, prow, rsw, ksc, toff, kmax);
    fence_proxy_async_smem();
    tc_fence_before();
    mbar_arrive(&bars.p_full);
    if (kPingPong<kPInt8> && (x == 0 ? j < nt_partner : j + 1 < nt_partner)) mbar_arrive(&partner.turn);
    l_run = l_run * alpha + rowsum;
    m_run = m_new;

    // ---- (3) fold PV_{j-1}: O <- alpha_j (O + g_{j-1} PV_{j-1}) ----
    // (O is kept relative to the newest running max.)
    if (j > 0) {
      if (__all_sync(0xffffffffu, alpha == 1.0f)) fold_pv<D, kPInt8, false>(O, tPV, alpha, alpha * g_prev);
      else fold_pv<D, kPInt8, true>(O, tPV, alpha, alpha * g_prev);
      tc_fence_before();
      mbar_arrive(&bars.pv_free);
      if constexpr (kVBias) C = alpha * (C - 8.0f * g_prev * r_prev);
    }
    g_prev = vscale * (kPInt8 ? (1.0f / 127.0f) : 1.0f);
    if constexpr (kVBias) r_prev = rintf(rowsum * 127.0f);    // the integer sum of the P codes
  }
  if (!ok || ntiles == 0) return;
  // last product: O += g_{n-1} PV_{n-1}
  ok = __all_sync(0xffffffffu, mbar_wait(&bars.pv_full, (ntiles - 1) & 1, abort_flag, p.err));
  if (!ok) return;
  tc_fence_after();
  fold_pv<D, kPInt8, false>(O, tPV, 1.0f, g_prev);
  if constexpr (kVBias) {
    C -= 8.0f * g_prev * r_prev;
#pragma unroll
    for (int d = 0; d < D; ++d) O[d] += C;
  }

  // epilogue: out = O / l (bf16), lse
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
    if (p.lse) p.lse[static_cast<int64_t>(bh) * p.Nq + qrow] = m_run * 0.6931471805599453f + logf(l_run);
  }
}

// 32 packed INT4 codes (16 bytes; element 2i in the low nibble of byte i,
// two's complement) -> the 32 values code + 8 (0..15) as unsigned bytes in
// element order (two 16-byte chunks). Flipping bit 3 of every nibble adds 8
// to it modulo 16, which maps -8..7 onto 0..15.
__device__ __forceinline__ void widen_int4x32_biased(uint4 w, uint4& lo16, uint4& hi16) {
  const uint32_t in[4] = {w.x, w.y, w.z, w.w};
  uint32_t o[8];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t u = in[k] ^ 0x88888888u;
    const uint32_t lo = u & 0x0F0F0F0Fu;                // elements 8k, 8k+2, 8k+4, 8k+6
    const uint32_t hi = (u >> 4) & 0x0F0F0F0Fu;         // elements 8k+1, 8k+3, ...
    o[2 * k] = __byte_perm(lo, hi, 0x5140);
    o[2 * k + 1] = __byte_perm(lo, hi, 0x7362);
  }
  lo16 = make_uint4(o[0], o[1], o[2], o[3]);
  hi16 = make_uint4(o[4], o[5], o[6], o[7]);
}

// The same, as signed bytes (INT4 Q, widened once per CTA): bit 3 of each
// nibble times 0x1E spreads to 0xF0 within its byte.
__device__ __forceinline__ void widen_int4x32_signed(uint4 w, uint4& lo16, uint4& hi16) {
  const uint32_t in[4] = {w.x, w.y, w.z, w.w};
  uint32_t o[8];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    uint32_t lo = in[k] & 0x0F0F0F0Fu;
    uint32_t hi = (in[k] >> 4) & 0x0F0F0F0Fu;
    lo |= (lo & 0x08080808u) * 0x1Eu;
    hi |= (hi & 0x08080808u) * 0x1Eu;
    o[2 * k] = __byte_perm(lo, hi, 0x5140);
    o[2 * k + 1] = __byte_perm(lo, hi, 0x7362);
  }
  lo16 = make_uint4(o[0], o[1], o[2], o[3]);
  hi16 = make_uint4(o[4], o[5], o[6], o[7]);
}

// Widens one 128-row tile of packed INT4 codes (D/2 bytes per row, linear)
// into 8-bit codes laid out as a TMA load of 8-bit codes with the tile's
// swizzle would leave them (16-byte chunk c of row t at chunk c ^ swz(t)).
// One warp; kBiased: code + 8 as unsigned bytes, else signed codes.
template <int D, bool kBiased>
__device__ __forceinline__ void widen_tile(const uint8_t* packed, uint8_t* dst, int lane) {
  constexpr int kPC = D / 32;                          // packed 16-byte chunks per row
  const uint4* src = reinterpret_cast<const uint4*>(packed);
#pragma unroll 4
  for (int q = lane; q < kTileN * kPC; q += 32) {
    const int t = q / kPC, c = q % kPC;
    uint4 lo16, hi16;
    if constexpr (kBiased) widen_int4x32_biased(src[q], lo16, hi16);
    else widen_int4x32_signed(src[q], lo16, hi16);
    const int swz = D == 128 ? (t & 7) : ((t >> 1) & 3);
    *reinterpret_cast<uint4*>(dst + t * D + (((2 * c) ^ swz) << 4)) = lo16;
    *reinterpret_cast<uint4*>(dst + t * D + (((2 * c + 1) ^ swz) << 4)) = hi16;
  }
}

// Grid: one CTA per pair of consecutive query tiles (2i, 2i+1) of one (b, h):
// the pairs with the most key tiles first (causal), else head-major. kQKCode: Q/K codes e4m3
// (0), INT8 (1) or packed INT4 (2: Q widened once to INT8 by warp 3, each K
// tile widened to code + 8 in unsigned bytes, and the 8 * sum(Q codes) this
// adds to every score of a row subtracted with the scale); kVCode: V codes
// e4m3 (0), INT8 (1) or packed INT4 (2, widened in shared memory by warp 3 before the P.V products, as code + 8 in unsigned
// bytes; the 8 * sum(P codes) this adds to every output channel of a row is
// removed by a per-row scalar). P is rounded to INT8 codes for integer V and
// to e4m3 for e4m3 V.
template <int D, int kQKCode, int kVCode>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
  constexpr bool kSInt8 = kQKCode != 0;
  constexpr bool kK4 = kQKCode == 2;
  constexpr bool kPInt8 = kVCode != 0;
  constexpr bool kV4 = kVCode == 2;
  using L = Smem<D, kQKCode, kVCode>;
  constexpr uint32_t kSwz = D == 128 ? 2u : 4u;       // descriptor swizzle: 128B / 64B
  constexpr uint32_t kRowB = D;                        // bytes per code row
  constexpr uint32_t kSBO = 8 * kRowB;                 // 8-row core-matrix group stride
  // S = Q K^T: A = Q (K-major), B = K (K-major), M = N = 128.
  // (INT4 K is widened to unsigned bytes: B format u8.)
  constexpr uint32_t kIdescQK =
      instr_desc(kSInt8 ? 2u : 1u, kSInt8 ? 1u : 0u, kSInt8 && !kK4 ? 1u : 0u, 0u, 0u, kTileN, kTileM);
  // PV = P V: A = P (K-major over keys), B = V (MN-major: channels contiguous), N = D.
  // (INT4 V is widened to unsigned bytes: B format u8.)
  constexpr uint32_t kIdescPV =
      instr_desc(kPInt8 ? 2u : 1u, kPInt8 ? 1u : 0u, kPInt8 && !kV4 ? 1u : 0u, 0u, 1u, D, kTileM);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + L::kQ;                          // [2][128 x D]
  uint8_t* sP = smem + L::kP;                          // [2][128 x 128]
  uint8_t* sK = smem + L::kK;                          // [stages][128 x D]
  uint8_t* sV = smem + L::kV;                          // [stages][128 x D] (INT4: 128 x D/2)
  uint8_t* sW = smem + L::kW;                          // INT4: [2][128 x D] widened V
  uint8_t* sKw = smem + L::kKw;                        // INT4: [2][128 x D] widened K
  uint8_t* sQp = smem + L::kQp;                        // INT4: [2][128 x D/2] packed Q

  __shared__ __align__(8) uint64_t bar_q_full;
  __shared__ __align__(8) uint64_t bar_kv_full[kStagesKV];
  __shared__ __align__(8) uint64_t bar_kv_empty[kStagesKV];
  __shared__ __align__(8) TileBars bars[2];
  __shared__ __align__(8) uint64_t bar_drain[2];
  __shared__ __align__(8) uint64_t bar_wv_full[2];     // INT4: widened V(j) in sW[j & 1] (warp 3)
  __shared__ __align__(8) uint64_t bar_wv_empty[2];    // INT4: sW[j & 1] read by both tiles' P.V
  __shared__ __align__(8) uint64_t bar_wk_full[2];     // INT4: widened K(j) in sKw[j & 1]
  __shared__ __align__(8) uint64_t bar_wk_empty[2];    // INT4: sKw[j & 1] read by both tiles' S
  __shared__ __align__(8) uint64_t bar_q_wide;         // INT4: both Q tiles widened into sQ
  __shared__ uint32_t tmem_base_slot;
  __shared__ int abort_flag;
  __shared__ float sKsc[kMaxBlk], sVsc[kMaxBlk];

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Causal: the pairs with the most key tiles first (all heads of a pair
  // together). Non-causal: head-major, so that the CTAs resident at one time
  // cover few heads and share their K/V tiles in L2.
  const int BH = p.B * p.H;
  const int pair = p.causal ? p.npairs - 1 - static_cast<int>(blockIdx.x) / BH
                            : static_cast<int>(blockIdx.x) % p.npairs;
  const int bh = p.causal ? static_cast<int>(blockIdx.x) % BH : static_cast<int>(blockIdx.x) / p.npairs;
  const int b = bh / p.H, h = bh % p.H;
  const int qt2[2] = {2 * pair, 2 * pair + 1 < p.nqt ? 2 * pair + 1 : -1};
  const int nkt_all = (p.Nkv + kTileN - 1) / kTileN;
  int nt2[2];
#pragma unroll
  for (int x = 0; x < 2; ++x)
    nt2[x] = qt2[x] < 0 ? 0 : (p.causal ? min(nkt_all, (qt2[x] * kTileM + kTileM - 1) / kTileN + 1) : nkt_all);
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
      mbar_init(&bars[x].turn, 128);
    }
    mbar_init(&bar_drain[0], 1);
    mbar_init(&bar_drain[1], 1);
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bar_wv_full[x], 1);
      mbar_init(&bar_wv_empty[x], 2);
      mbar_init(&bar_wk_full[x], 1);
      mbar_init(&bar_wk_empty[x], 2);
    }
    mbar_init(&bar_q_wide, 1);
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
    regs_dec<kRegsLow>();
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(&bar_q_full, (qt2[1] >= 0 ? 2 : 1) * L::kQTileBytes);
      uint8_t* qdst = kK4 ? sQp : sQ;                  // INT4: packed, widened by warp 3
      for (int x = 0; x < 2; ++x)
        if (qt2[x] >= 0) tma_load_4d(qdst + x * L::kQTileBytes, &tmQ, &bar_q_full, 0, qt2[x] * kTileM, h, b);
    }
    // K/V tile j into stage j % 3 (after both tiles' P.V(j - 3) released it).
    auto load = [&](int jj) -> bool {
      const int st = jj % kStagesKV;
      if (jj >= kStagesKV) {
        const bool ok = mbar_wait(&bar_kv_empty[st], ((jj / kStagesKV) - 1) & 1, &abort_flag, p.err);
        if (!__all_sync(0xffffffffu, ok)) return false;
      }
      if (lane == 0) {
        mbar_arrive_expect_tx(&bar_kv_full[st], L::kKTileBytes + L::kVTileBytes);
        tma_load_4d(sK + st * L::kKTileBytes, &tmK, &bar_kv_full[st], 0, jj * kTileN, h, b);
        tma_load_4d(sV + st * L::kVTileBytes, &tmV, &bar_kv_full[st], 0, jj * kTileN, h, b);
      }
      __syncwarp();
      return true;
    };
    // INT4 K: this warp also widens each K tile (warp 3 has Q and V), K(jj)
    // into sKw[jj & 1] once it has landed and both tiles' S(jj - 2) read the
    // buffer. K(j + 1) is widened before the wait that frees stage j, so the
    // scores never wait on a P.V product.
    auto widen_k = [&](int jj) -> bool {
      bool ok = mbar_wait(&bar_kv_full[jj % kStagesKV], (jj / kStagesKV) & 1, &abort_flag, p.err);
      if (ok && jj >= 2) ok = mbar_wait(&bar_wk_empty[jj & 1], ((jj >> 1) - 1) & 1, &abort_flag, p.err);
      if (!__all_sync(0xffffffffu, ok)) return false;
      widen_tile<D, true>(sK + (jj % kStagesKV) * L::kKTileBytes, sKw + (jj & 1) * L::kTileBytes, lane);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_wk_full[jj & 1]);
      return true;
    };
    int j = 0;                                         // K/V tiles loaded so far
    if constexpr (kK4) {
      bool ok = true;
      for (; ok && j < min(nt_max, kStagesKV); ++j) ok = load(j);
      if (ok && nt_max > 0) ok = widen_k(0);
      for (int jw = 0; ok && jw < nt_max; ++jw) {
        if (jw + 1 < nt_max) ok = widen_k(jw + 1);
        if (ok && j < nt_max) {
          ok = load(j);
          if (ok) ++j;
        }
      }
    } else {
      // (this form of the loop measured faster than calling load())
      for (; j < nt_max; ++j) {
        const int st = j % kStagesKV;
        if (j >= kStagesKV) {
          const bool ok = mbar_wait(&bar_kv_empty[st], ((j / kStagesKV) - 1) & 1, &abort_flag, p.err);
          if (!__all_sync(0xffffffffu, ok)) break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(&bar_kv_full[st], L::kKTileBytes + L::kVTileBytes);
          tma_load_4d(sK + st * L::kKTileBytes, &tmK, &bar_kv_full[st], 0, j * kTileN, h, b);
          tma_load_4d(sV + st * L::kVTileBytes, &tmV, &bar_kv_full[st], 0, j * kTileN, h, b);
        }
        __syncwarp();
      }
    }
    if (abort_flag && lane == 0) {
      // Let issued copies land before the CTA can exit (bounded).
      mbar_wait(&bar_q_full, 0, nullptr, nullptr, 100000000ull);
      for (int i = max(0, j - kStagesKV); i < j; ++i)
        mbar_wait(&bar_kv_full[i % kStagesKV], (i / kStagesKV) & 1, nullptr, nullptr, 100000000ull);
    }
    __syncwarp();
  } else if (warp == 1 || warp == 2) {
    // ------------------------------------------------------------ MMA issuers
    // Warp 1 issues tile A's products, warp 2 tile B's (one elected lane
    // each), so neither tile waits for the other. Per key tile j:
    //   S(j+1)  once P(j) has been written (S free) and K/V(j+1) has landed,
    //   PV(j)   once PV(j-1) has been read,
    // then a commit releases K/V stage j (two arrivals: one per tile; a tile
    // with fewer key tiles arrives at once for the stages it does not read).
    regs_dec<kRegsLow>();
    const int x = warp - 1;
    const int nt = nt2[x];
    const uint32_t aQ = smem_u32(sQ) + x * L::kTileBytes, aP = smem_u32(sP) + x * kTileM * kTileN;
    const uint32_t aK = smem_u32(sK), aV = smem_u32(sV), aW = smem_u32(sW), aKw = smem_u32(sKw);
    const uint32_t tS = tmem + x * 256, tPV = tmem + x * 256 + 128;
    TileBars& tb = bars[x];
    // (INT4 K: the caller has waited for the widened tile.)
    auto issue_s = [&](int j) {
      if (lane == 0) {
        const uint32_t kbase = kK4 ? aKw + (j & 1) * L::kTileBytes : aK + (j % kStagesKV) * L::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk) {
          const uint64_t da = smem_desc(aQ + kk * 32, 16, kSBO, kSwz);
          const uint64_t db = smem_desc(kbase + kk * 32, 16, kSBO, kSwz);
          mma_ss<kSInt8>(tS, da, db, kIdescQK, kk > 0 ? 1u : 0u);
        }
        mma_commit(&tb.s_full);
        if constexpr (kK4) mma_commit(&bar_wk_empty[j & 1]);
      }
      __syncwarp();
    };
    bool ok = nt == 0 || __all_sync(0xffffffffu, mbar_wait(kK4 ? &bar_q_wide : &bar_q_full, 0, &abort_flag, p.err));
    for (int j = 0; ok && j < nt_max; ++j) {
      const int st = j % kStagesKV;
      ok = __all_sync(0xffffffffu, mbar_wait(&bar_kv_full[st], (j / kStagesKV) & 1, &abort_flag, p.err));
      if (!ok) break;
      if (j >= nt) {
        // (INT4: arrive only once the widened tiles are there, so that these
        // early arrivals cannot count toward a buffer's previous use.)
        if constexpr (kK4) {
          ok = __all_sync(0xffffffffu, mbar_wait(&bar_wk_full[j & 1], (j >> 1) & 1, &abort_flag, p.err));
          if (!ok) break;
        }
        if constexpr (kV4) {
          ok = __all_sync(0xffffffffu, mbar_wait(&bar_wv_full[j & 1], (j >> 1) & 1, &abort_flag, p.err));
          if (!ok) break;
        }
        if (lane == 0) {
          mbar_arrive(&bar_kv_empty[st]);
          if constexpr (kK4) mbar_arrive(&bar_wk_empty[j & 1]);
          if constexpr (kV4) mbar_arrive(&bar_wv_empty[j & 1]);
        }
        __syncwarp();
        continue;
      }
      if (j == 0) {
        if constexpr (kK4) {
          ok = __all_sync(0xffffffffu, mbar_wait(&bar_wk_full[0], 0, &abort_flag, p.err));
          if (!ok) break;
        }
        tc_fence_after();
        issue_s(0);
      }
      // S(j) consumed: P(j) is in shared memory
      ok = __all_sync(0xffffffffu, mbar_wait(&tb.p_full, j & 1, &abort_flag, p.err));
      if (!ok) break;
      if (j + 1 < nt) {
        const int j1 = j + 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&bar_kv_full[j1 % kStagesKV], (j1 / kStagesKV) & 1, &abort_flag, p.err));
        if (!ok) break;
        if constexpr (kK4) {
          ok = __all_sync(0xffffffffu, mbar_wait(&bar_wk_full[j1 & 1], (j1 >> 1) & 1, &abort_flag, p.err));
          if (!ok) break;
        }
        tc_fence_after();
        issue_s(j1);
      }
      if (j > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(&tb.pv_free, (j - 1) & 1, &abort_flag, p.err));
        if (!ok) break;
      }
      if constexpr (kV4) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bar_wv_full[j & 1], (j >> 1) & 1, &abort_flag, p.err));
        if (!ok) break;
      }
      tc_fence_after();
      if (lane == 0) {
        const uint32_t vbase = kV4 ? aW + (j & 1) * L::kTileBytes : aV + st * L::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kTileN / 32; ++kk) {
          const uint64_t da = smem_desc(aP + kk * 32, 16, 1024, 2u);
          // MN-major V: 32 keys per MMA = 4 groups of 8 key rows, SBO apart.
          const uint64_t db = smem_desc(vbase + kk * 32 * kRowB, kTileN * kRowB, kSBO, kSwz);
          mma_ss<kPInt8>(tPV, da, db, kIdescPV, kk > 0 ? 1u : 0u);
        }
        mma_commit(&tb.pv_full);
        mma_commit(&bar_kv_empty[st]);
        if constexpr (kV4) mma_commit(&bar_wv_empty[j & 1]);
      }
      __syncwarp();
    }
    if (abort_flag && lane == 0) {
      // Wait (bounded) until every MMA this thread issued has completed.
      mma_commit(&bar_drain[x]);
      mbar_wait(&bar_drain[x], 0, nullptr, nullptr, 100000000ull);
    }
    __syncwarp();
  } else if (warp == 3) {
    regs_dec<kRegsLow>();
    if constexpr (kK4 || kV4) {
      // ------------------------------------------------------------ INT4 widening
      // Packed tiles -> 8-bit codes laid out as TMA loads of 8-bit codes
      // would leave them: the two Q tiles once (signed), then per key tile j
      // V(j) into sW[j & 1] (code + 8, unsigned). (Warp 0 widens K.)
      bool ok = true;
      if constexpr (kK4) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bar_q_full, 0, &abort_flag, p.err));
        if (ok) {
          for (int x = 0; x < 2; ++x)
            if (qt2[x] >= 0) widen_tile<D, false>(sQp + x * L::kQTileBytes, sQ + x * L::kTileBytes, lane);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar_q_wide);
        }
      }
      for (int j = 0; ok && j < nt_max; ++j) {
        const int st = j % kStagesKV;
        ok = __all_sync(0xffffffffu, mbar_wait(&bar_kv_full[st], (j / kStagesKV) & 1, &abort_flag, p.err));
        if (!ok) break;
        if constexpr (kV4) {
          if (j >= 2)
            ok = __all_sync(0xffffffffu, mbar_wait(&bar_wv_empty[j & 1], ((j >> 1) - 1) & 1, &abort_flag, p.err));
          if (!ok) break;
          widen_tile<D, true>(sV + st * L::kVTileBytes, sW + (j & 1) * L::kTileBytes, lane);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar_wv_full[j & 1]);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ softmax rows
    regs_inc<kRegsHigh>();
    const int x = (warp - 4) >> 2;                // which query tile
    // K/V block scales of this head, staged once by tile A's warps (beyond
    // kMaxBlk blocks they are read from global memory).
    if (x == 0) {
      for (int i = threadIdx.x - 128; i < min(p.nkb, kMaxBlk); i += 128) {
        sKsc[i] = p.ks[static_cast<int64_t>(bh) * p.nkb + i];
        sVsc[i] = p.vs[static_cast<int64_t>(bh) * p.nkb + i];
      }
    }
    named_bar_sync(1, 256);
    if (qt2[x] >= 0)
      tile_rows<D, kSInt8, kPInt8, kV4, kK4>(p, bars[x], bars[1 - x], tmem + x * 256, tmem + x * 256 + 128, sP + x * kTileM * kTileN,
                          sKsc, sVsc, qt2[x], nt2[x], x, nt2[1 - x], bh, b, h, warp & 3, lane, &abort_flag,
                          &bar_q_wide, sQ + x * L::kTileBytes);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

template <int D, int kQKCode, int kVCode>
cudaError_t launch_t(const PrefillArgs& a, cudaStream_t st, int* err) {
  CUtensorMap mq, mk, mv;
  const bool v_ok = kVCode == 2 ? make_map_v4(&mv, a.v, a.layout, a.B, a.H, a.Nkv, D)
                                : make_map(&mv, a.v, a.layout, a.B, a.H, a.Nkv, D);
  const bool qk_ok = kQKCode == 2 ? make_map_v4(&mq, a.q, a.layout, a.B, a.H, a.Nq, D) &&
                                        make_map_v4(&mk, a.k, a.layout, a.B, a.H, a.Nkv, D)
                                  : make_map(&mq, a.q, a.layout, a.B, a.H, a.Nq, D) &&
                                        make_map(&mk, a.k, a.layout, a.B, a.H, a.Nkv, D);
  if (!qk_ok || !v_ok) return cudaErrorInvalidValue;
  PrefillParams p;
  p.qs = a.qs; p.ks = a.ks; p.vs = a.vs;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.lse = a.lse;
  p.B = a.B; p.H = a.H; p.Nq = a.Nq; p.Nkv = a.Nkv;
  p.nqt = (a.Nq + kTileM - 1) / kTileM;
  p.npairs = (p.nqt + 1) / 2;
  p.nqb = (a.Nq + 127) / 128;
  p.nkb = (a.Nkv + 255) / 256;
  p.causal = a.causal;
  p.layout = a.layout;
  p.scale_log2 = a.scale_log2;
  p.err = err;
  auto k = prefill_kernel<D, kQKCode, kVCode>;
  constexpr int kSmem = Smem<D, kQKCode, kVCode>::kBytes;
  cudaError_t e = set_max_dyn_smem(reinterpret_cast<const void*>(k), kSmem);
  if (e != cudaSuccess) return e;
  // The register split inside the kernel needs at least kRegsNeeded
  // registers per thread at launch; never launch with fewer. (The count is
  // a property of the compiled kernel: looked up once.)
  static std::atomic<int> regs{-1};
  if (regs.load() < 0) {
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, k);
    if (e != cudaSuccess) return e;
    regs.store(fa.numRegs);
  }
  if (regs.load() < kRegsNeeded) return cudaErrorInvalidConfiguration;
  const int64_t grid = static_cast<int64_t>(p.npairs) * a.B * a.H;
  k<<<static_cast<unsigned>(grid), kThreads, kSmem, st>>>(mq, mk, mv, p);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_d(const PrefillArgs& a, cudaStream_t st, int* err) {
  if (a.qk_code == 1) {
    if (a.v_code == 1) return launch_t<D, 1, 1>(a, st, err);
    if (a.v_code == 0) return launch_t<D, 1, 0>(a, st, err);
    if (a.v_code == 2) return launch_t<D, 1, 2>(a, st, err);
  } else if (a.qk_code == 0 && a.v_code == 0) {
    return launch_t<D, 0, 0>(a, st, err);
  } else if (a.qk_code == 2 && a.v_code == 2) {
    return launch_t<D, 2, 2>(a, st, err);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

bool prefill_supported(int D) { return D == 64 || D == 128; }

// Q/K INT8 with V e4m3, INT8 or packed INT4; Q/K e4m3 with V e4m3; Q/K/V
// packed INT4.
bool prefill_codes_supported(int qk_code, int v_code) {
  if (qk_code == 1) return v_code >= 0 && v_code <= 2;
  return qk_code == v_code && (qk_code == 0 || qk_code == 2);
}

cudaError_t launch_prefill(const PrefillArgs& a, cudaStream_t st, int num_sms, int* err) {
  (void)num_sms;
  if (!prefill_codes_supported(a.qk_code, a.v_code)) return cudaErrorInvalidValue;
  if (a.D == 128) return launch_d<128>(a, st, err);
  if (a.D == 64) return launch_d<64>(a, st, err);
  return cudaErrorInvalidValue;
}


}  // namespace qattn
