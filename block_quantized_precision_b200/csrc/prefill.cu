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
// One CTA = one tile of 128 query rows of one (b, h); two CTAs share an SM
// (each allocates 256 TMEM columns and ~97 KB of shared memory).
//   warp 0      TMA producer: Q once, then K/V tiles of 128 keys into a
//               two-stage ring (128B / 64B swizzle, no multicast).
//   warp 1      TMEM allocation; lane 0 issues the MMAs:
//                 S  = Q K^T        M=128, N=128, K=D      -> TMEM cols [0,128)
//                 PV = P V          M=128, N=D,   K=128    -> TMEM cols [0,D)
//               kind::i8 (s32 accumulate) or kind::f8f6f4 (e4m3, f32).
//               P is read from shared memory (K-major), V is used MN-major
//               straight from its token-major tile.
//   warps 2-5   one thread per query row: reads S from TMEM, applies the
//               block scales and the mask, running max / sum in the log2
//               domain, rounds P to 8 bits (e4m3, or round(127 p) for INT8)
//               and writes it to shared memory in the swizzled K-major
//               layout; then folds PV into the float32 output kept in TMEM
//               cols [128, 128+D): O = O * alpha + PV * c_j; finally writes
//               O / l as bfloat16 (and the LSE).
// Per key tile: QK^T -> softmax -> PV -> fold, handed over with mbarriers
// (all waits bounded).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math_constants.h>

#include <climits>

#include "qattn_device.cuh"
#include "qattn_internal.h"

namespace qattn {

namespace {

constexpr int kThreads = 192;
constexpr int kTileM = 128;   // query rows per CTA
constexpr int kTileN = 128;   // keys per tile
constexpr int kStagesKV = 2;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColO = 128;
constexpr int kMaxBlk = 512;  // K/V block scales staged in shared memory (keys up to 131072)

struct PrefillParams {
  const float* qs;
  const float* ks;
  const float* vs;
  __nv_bfloat16* out;
  float* lse;
  int B, H, Nq, Nkv;
  int nqt, nqb, nkb;
  int causal;
  int layout;
  float scale_log2;
  int* err;
};

template <int D>
struct Smem {
  static constexpr int kTileBytes = kTileM * D;       // one 128-row code tile
  static constexpr int kQ = 0;
  static constexpr int kP = kQ + kTileBytes;
  static constexpr int kK = kP + kTileM * kTileN;     // P tile: 128 rows x 128 keys
  static constexpr int kV = kK + kStagesKV * kTileBytes;
  static constexpr int kEnd = kV + kStagesKV * kTileBytes;
  static constexpr int kBytes = kEnd + 1024;          // slack for 1024-byte alignment
};

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// acc + lo + hi of a half2 (bits of `h2`), float32 accumulation.
__device__ __forceinline__ float add_f32_f16x2(uint32_t h2, float acc) {
  float r;
  asm("{\n\t.reg .f16 lo, hi;\n\t.reg .f32 t;\n\tmov.b32 {lo, hi}, %1;\n\t"
      "add.rn.f32.f16 t, lo, %2;\n\tadd.rn.f32.f16 %0, hi, t;\n\t}"
      : "=f"(r) : "r"(h2), "f"(acc));
  return r;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Element offset of token n of head (b, h), channel 0.
__device__ __forceinline__ int64_t row_offset(int layout, int H, int N, int D, int b, int h, int n) {
  return layout == 0 ? ((static_cast<int64_t>(b) * H + h) * N + n) * D
                     : ((static_cast<int64_t>(b) * N + n) * H + h) * D;
}

template <int D, bool kInt8>
__global__ void __launch_bounds__(kThreads, 2)
    prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
  using L = Smem<D>;
  constexpr uint32_t kSwz = D == 128 ? 2u : 4u;       // descriptor swizzle: 128B / 64B
  constexpr uint32_t kRowB = D;                        // bytes per code row
  constexpr uint32_t kSBO = 8 * kRowB;                 // 8-row core-matrix group stride
  // S = Q K^T: A = Q (K-major), B = K (K-major), M = N = 128.
  constexpr uint32_t kIdescQK = instr_desc(kInt8 ? 2u : 1u, kInt8 ? 1u : 0u, kInt8 ? 1u : 0u, 0u, 0u, kTileN, kTileM);
  // PV = P V: A = P (K-major over keys), B = V (MN-major: channels contiguous), N = D.
  constexpr uint32_t kIdescPV = instr_desc(kInt8 ? 2u : 1u, kInt8 ? 1u : 0u, kInt8 ? 1u : 0u, 0u, 1u, D, kTileM);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + L::kQ;
  uint8_t* sP = smem + L::kP;
  uint8_t* sK = smem + L::kK;
  uint8_t* sV = smem + L::kV;

  __shared__ __align__(8) uint64_t bar_q_full;
  __shared__ __align__(8) uint64_t bar_kv_full[kStagesKV];
  __shared__ __align__(8) uint64_t bar_kv_empty[kStagesKV];
  __shared__ __align__(8) uint64_t bar_s_full, bar_p_full, bar_pv_full, bar_free, bar_drain;
  __shared__ uint32_t tmem_base_slot;
  __shared__ int abort_flag;
  __shared__ float sKsc[kMaxBlk], sVsc[kMaxBlk];

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int BH = p.B * p.H;
  const int qt = p.nqt - 1 - static_cast<int>(blockIdx.x) / BH;   // longest (causal) tiles first
  const int bh = static_cast<int>(blockIdx.x) % BH;
  const int b = bh / p.H, h = bh % p.H;
  const int q0 = qt * kTileM;
  const int nkt_all = (p.Nkv + kTileN - 1) / kTileN;
  const int ntiles = p.causal ? min(nkt_all, (q0 + kTileM - 1) / kTileN + 1) : nkt_all;

  if (threadIdx.x == 0) {
    mbar_init(&bar_q_full, 1);
    for (int s = 0; s < kStagesKV; ++s) {
      mbar_init(&bar_kv_full[s], 1);
      mbar_init(&bar_kv_empty[s], 1);
    }
    mbar_init(&bar_s_full, 1);
    mbar_init(&bar_p_full, 128);
    mbar_init(&bar_pv_full, 1);
    mbar_init(&bar_free, 128);
    mbar_init(&bar_drain, 1);
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

  // Waits below are made warp-uniform (__all_sync): a whole warp leaves its
  // loop together, so every .sync.aligned instruction stays convergent.
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(&bar_q_full, L::kTileBytes);
      tma_load_4d(sQ, &tmQ, &bar_q_full, 0, q0, h, b);
    }
    int j = 0;
    for (; j < ntiles; ++j) {
      const int st = j % kStagesKV;
      if (j >= kStagesKV) {
        const bool ok = mbar_wait(&bar_kv_empty[st], ((j / kStagesKV) - 1) & 1, &abort_flag, p.err);
        if (!__all_sync(0xffffffffu, ok)) break;
      }
      if (lane == 0) {
        mbar_arrive_expect_tx(&bar_kv_full[st], 2 * L::kTileBytes);
        tma_load_4d(sK + st * L::kTileBytes, &tmK, &bar_kv_full[st], 0, j * kTileN, h, b);
        tma_load_4d(sV + st * L::kTileBytes, &tmV, &bar_kv_full[st], 0, j * kTileN, h, b);
      }
      __syncwarp();
    }
    if (abort_flag && lane == 0) {
      // Let issued copies land before the CTA can exit (bounded).
      mbar_wait(&bar_q_full, 0, nullptr, nullptr, 100000000ull);
      for (int i = max(0, j - kStagesKV); i < j; ++i)
        mbar_wait(&bar_kv_full[i % kStagesKV], (i / kStagesKV) & 1, nullptr, nullptr, 100000000ull);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t aQ = smem_u32(sQ), aP = smem_u32(sP);
    const uint32_t aK = smem_u32(sK), aV = smem_u32(sV);
    bool ok = __all_sync(0xffffffffu, mbar_wait(&bar_q_full, 0, &abort_flag, p.err));
    for (int j = 0; ok && j < ntiles; ++j) {
      const int st = j % kStagesKV;
      ok = __all_sync(0xffffffffu, mbar_wait(&bar_kv_full[st], (j / kStagesKV) & 1, &abort_flag, p.err));
      if (ok && j > 0) ok = __all_sync(0xffffffffu, mbar_wait(&bar_free, (j - 1) & 1, &abort_flag, p.err));
      if (!ok) break;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t kbase = aK + st * L::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk) {
          const uint64_t da = smem_desc(aQ + kk * 32, 16, kSBO, kSwz);
          const uint64_t db = smem_desc(kbase + kk * 32, 16, kSBO, kSwz);
          mma_ss<kInt8>(tmem, da, db, kIdescQK, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bar_s_full);
      }
      __syncwarp();
      ok = __all_sync(0xffffffffu, mbar_wait(&bar_p_full, j & 1, &abort_flag, p.err));
      if (!ok) break;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t vbase = aV + st * L::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kTileN / 32; ++kk) {
          const uint64_t da = smem_desc(aP + kk * 32, 16, 1024, 2u);
          // MN-major V: 32 keys per MMA = 4 groups of 8 key rows, SBO apart.
          const uint64_t db = smem_desc(vbase + kk * 32 * kRowB, kTileN * kRowB, kSBO, kSwz);
          mma_ss<kInt8>(tmem, da, db, kIdescPV, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bar_pv_full);
        mma_commit(&bar_kv_empty[st]);
      }
      __syncwarp();
    }
    if (abort_flag && lane == 0) {
      // Wait (bounded) until every MMA issued so far has completed.
      mma_commit(&bar_drain);
      mbar_wait(&bar_drain, 0, nullptr, nullptr, 100000000ull);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax rows
    const int quarter = warp & 3;                 // TMEM lane quarter of this warp
    const int r = quarter * 32 + lane;            // query row within the tile
    const int qrow = q0 + r;
    const uint32_t trow = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const float sq = p.qs[static_cast<int64_t>(bh) * p.nqb + qt];
    // K/V block scales of this head, staged once (beyond kMaxBlk blocks they
    // are read from global memory).
    for (int i = threadIdx.x - 64; i < min(p.nkb, kMaxBlk); i += 128) {
      sKsc[i] = p.ks[static_cast<int64_t>(bh) * p.nkb + i];
      sVsc[i] = p.vs[static_cast<int64_t>(bh) * p.nkb + i];
    }
    named_bar_sync(1, 128);
    float m_run = -CUDART_INF_F, l_run = 0.0f;
    uint8_t* prow = sP + r * 128;
    const int rsw = r & 7;
    bool ok = true;
    for (int j = 0; j < ntiles; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bar_s_full, j & 1, &abort_flag, p.err));
      if (!ok) break;
      tc_fence_after();
      const int blk = j >> 1;
      const float kscale = blk < kMaxBlk ? sKsc[blk] : p.ks[static_cast<int64_t>(bh) * p.nkb + blk];
      const float vscale = blk < kMaxBlk ? sVsc[blk] : p.vs[static_cast<int64_t>(bh) * p.nkb + blk];
      const float ksc = sq * kscale * p.scale_log2;
      const int key0 = j * kTileN;
      // Only the last tile (ragged N_kv) and the causal diagonal tile have
      // masked keys; the mask is applied on those tiles only (warp-uniform).
      const bool partial = (key0 + kTileN > p.Nkv) || (p.causal && key0 + kTileN - 1 > q0);
      int kmax = p.Nkv - key0;                    // keys valid for this row: [0, kmax)
      if (p.causal) kmax = min(kmax, qrow - key0 + 1);

      // ---- pass 1: row max (integer max of the INT32 scores, or float max) ----
      float tmax;
      if constexpr (kInt8) {
        int im = INT_MIN;
#pragma unroll 1
        for (int c = 0; c < kTileN / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(trow + c * 32, v);
          tmem_wait_ld();
          if (partial) {
#pragma unroll
            for (int e = 0; e < 32; ++e) im = max(im, c * 32 + e < kmax ? static_cast<int>(v[e]) : INT_MIN);
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) im = max(im, static_cast<int>(v[e]));
          }
        }
        tmax = im == INT_MIN ? -CUDART_INF_F : static_cast<float>(im) * ksc;
      } else {
        float fm = -CUDART_INF_F;
#pragma unroll 1
        for (int c = 0; c < kTileN / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(trow + c * 32, v);
          tmem_wait_ld();
          if (partial) {
#pragma unroll
            for (int e = 0; e < 32; e += 2)
              fm = fmax3(fm, c * 32 + e < kmax ? __uint_as_float(v[e]) : -CUDART_INF_F,
                         c * 32 + e + 1 < kmax ? __uint_as_float(v[e + 1]) : -CUDART_INF_F);
          } else {
#pragma unroll
            for (int e = 0; e < 32; e += 2) fm = fmax3(fm, __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
          }
        }
        tmax = fm * ksc;
      }
      const float m_new = fmaxf(m_run, tmax);
      const float alpha = ex2(m_run - m_new);     // 0 on the first tile
      const float2 k2 = make_float2(ksc, ksc);
      const float2 nm2 = make_float2(-m_new, -m_new);

      // ---- pass 2: probabilities, 8-bit rounding, P to shared memory ----
      float rs0 = 0.0f, rs1 = 0.0f;
      int rsum_i = 0;
#pragma unroll 1
      for (int c = 0; c < kTileN / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(trow + c * 32, v);
        tmem_wait_ld();
        uint32_t packed[8];
#pragma unroll
        for (int w = 0; w < 8; ++w) {
          float2 t01, t23;
          if constexpr (kInt8) {
            // exact INT32 -> float32: 1.5 * 2^23 + S has S in its low mantissa bits
            const float2 f01 = fadd2(make_float2(__int_as_float(static_cast<int>(v[4 * w]) + 0x4B400000),
                                                 __int_as_float(static_cast<int>(v[4 * w + 1]) + 0x4B400000)),
                                     make_float2(-12582912.0f, -12582912.0f));
            const float2 f23 = fadd2(make_float2(__int_as_float(static_cast<int>(v[4 * w + 2]) + 0x4B400000),
                                                 __int_as_float(static_cast<int>(v[4 * w + 3]) + 0x4B400000)),
                                     make_float2(-12582912.0f, -12582912.0f));
            t01 = ffma2(f01, k2, nm2);
            t23 = ffma2(f23, k2, nm2);
          } else {
            t01 = ffma2(make_float2(__uint_as_float(v[4 * w]), __uint_as_float(v[4 * w + 1])), k2, nm2);
            t23 = ffma2(make_float2(__uint_as_float(v[4 * w + 2]), __uint_as_float(v[4 * w + 3])), k2, nm2);
          }
          float pr[4] = {ex2(t01.x), ex2(t01.y), ex2(t23.x), ex2(t23.y)};
          if (partial) {
#pragma unroll
            for (int e = 0; e < 4; ++e) pr[e] = c * 32 + w * 4 + e < kmax ? pr[e] : 0.0f;
          }
          if constexpr (kInt8) {
            // code = RNE(p * 127): product rounded to float32, then the
            // 1.5 * 2^23 addend rounds it to an integer (half to even)
            const float2 q01 = fadd2(fmul2(make_float2(pr[0], pr[1]), make_float2(127.0f, 127.0f)),
                                     make_float2(12582912.0f, 12582912.0f));
            const float2 q23 = fadd2(fmul2(make_float2(pr[2], pr[3]), make_float2(127.0f, 127.0f)),
                                     make_float2(12582912.0f, 12582912.0f));
            const uint32_t b01 = __byte_perm(__float_as_uint(q01.x), __float_as_uint(q01.y), 0x0040);
            const uint32_t b23 = __byte_perm(__float_as_uint(q23.x), __float_as_uint(q23.y), 0x0040);
            const uint32_t word = __byte_perm(b01, b23, 0x5410);
            rsum_i = __dp4a(static_cast<int>(word), 0x01010101, rsum_i);
            packed[w] = word;
          } else {
            const uint32_t lo = cvt_e4m3x2(pr[0], pr[1]);
            const uint32_t hi = cvt_e4m3x2(pr[2], pr[3]);
            packed[w] = lo | (hi << 16);
            // row sum of the rounded probabilities (exact values via fp16)
            rs0 = add_f32_f16x2(cvt_e4m3x2_to_f16x2(static_cast<uint16_t>(lo)), rs0);
            rs1 = add_f32_f16x2(cvt_e4m3x2_to_f16x2(static_cast<uint16_t>(hi)), rs1);
          }
        }
        // keys c*32 .. c*32+31 = 16-byte chunks 2c and 2c+1 of this row
#pragma unroll
        for (int hchunk = 0; hchunk < 2; ++hchunk) {
          const int chunk = 2 * c + hchunk;
          *reinterpret_cast<uint4*>(prow + ((chunk ^ rsw) << 4)) =
              make_uint4(packed[4 * hchunk], packed[4 * hchunk + 1], packed[4 * hchunk + 2], packed[4 * hchunk + 3]);
        }
      }
      const float rowsum = kInt8 ? static_cast<float>(rsum_i) * (1.0f / 127.0f) : rs0 + rs1;
      tc_fence_before();
      fence_proxy_async_smem();
      mbar_arrive(&bar_p_full);
      l_run = l_run * alpha + rowsum;
      m_run = m_new;

      // ---- fold PV into O: O = O * alpha + PV * c_j ----
      ok = __all_sync(0xffffffffu, mbar_wait(&bar_pv_full, j & 1, &abort_flag, p.err));
      if (!ok) break;
      tc_fence_after();
      const float cj = vscale * (kInt8 ? (1.0f / 127.0f) : 1.0f);
      const float2 c2 = make_float2(cj, cj);
      const float2 a2 = make_float2(alpha, alpha);
      const bool unit_alpha = __all_sync(0xffffffffu, alpha == 1.0f);
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t pv[32], o[32];
        tmem_ld32(trow + c * 32, pv);
        if (j > 0) tmem_ld32(trow + kColO + c * 32, o);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float2 x;
          if constexpr (kInt8) {
            x = fadd2(make_float2(__int_as_float(static_cast<int>(pv[e]) + 0x4B400000),
                                  __int_as_float(static_cast<int>(pv[e + 1]) + 0x4B400000)),
                      make_float2(-12582912.0f, -12582912.0f));
          } else {
            x = make_float2(__uint_as_float(pv[e]), __uint_as_float(pv[e + 1]));
          }
          float2 y;
          if (j == 0) {
            y = fmul2(x, c2);
          } else {
            const float2 prev = make_float2(__uint_as_float(o[e]), __uint_as_float(o[e + 1]));
            y = ffma2(x, c2, unit_alpha ? prev : fmul2(prev, a2));
          }
          o[e] = __float_as_uint(y.x);
          o[e + 1] = __float_as_uint(y.y);
        }
        tmem_st32(trow + kColO + c * 32, o);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar_free);
    }
    // epilogue: out = O / l (bf16), lse. TMEM reads are done by the whole
    // warp; only the stores depend on the row.
    if (ok && ntiles > 0) {
      const bool store = qrow < p.Nq;
      const float inv_l = l_run > 0.0f ? 1.0f / l_run : 0.0f;
      __nv_bfloat16* orow = p.out + row_offset(p.layout, p.H, p.Nq, D, b, h, store ? qrow : 0);
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(trow + kColO + c * 32, o);
        tmem_wait_ld();
        uint32_t wds[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const __nv_bfloat162 t2 = __floats2bfloat162_rn(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
          wds[e] = *reinterpret_cast<const uint32_t*>(&t2);
        }
        if (store) {
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            *reinterpret_cast<uint4*>(orow + c * 32 + q4 * 8) = make_uint4(wds[4 * q4], wds[4 * q4 + 1], wds[4 * q4 + 2], wds[4 * q4 + 3]);
        }
      }
      if (store && p.lse) p.lse[static_cast<int64_t>(bh) * p.Nq + qrow] = m_run * 0.6931471805599453f + logf(l_run);
    }
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

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 4-D map {D, N, H, B} over 8-bit codes; box {D, 128, 1, 1}: one tile of 128
// token rows of one head lands as 128 rows of D bytes (swizzled).
bool make_map(CUtensorMap* m, const void* base, int layout, int B, int H, int N, int D) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3];
  if (layout == 0) {
    strides[0] = static_cast<cuuint64_t>(D);
    strides[1] = static_cast<cuuint64_t>(N) * D;
    strides[2] = static_cast<cuuint64_t>(H) * N * D;
  } else {
    strides[0] = static_cast<cuuint64_t>(H) * D;
    strides[1] = static_cast<cuuint64_t>(D);
    strides[2] = static_cast<cuuint64_t>(N) * H * D;
  }
  cuuint32_t box[4] = {static_cast<cuuint32_t>(D), static_cast<cuuint32_t>(kTileM), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, bool kInt8>
cudaError_t launch_t(const PrefillArgs& a, cudaStream_t st, int* err) {
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, a.q, a.layout, a.B, a.H, a.Nq, D) || !make_map(&mk, a.k, a.layout, a.B, a.H, a.Nkv, D) ||
      !make_map(&mv, a.v, a.layout, a.B, a.H, a.Nkv, D))
    return cudaErrorInvalidValue;
  PrefillParams p;
  p.qs = a.qs; p.ks = a.ks; p.vs = a.vs;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.lse = a.lse;
  p.B = a.B; p.H = a.H; p.Nq = a.Nq; p.Nkv = a.Nkv;
  p.nqt = (a.Nq + kTileM - 1) / kTileM;
  p.nqb = (a.Nq + 127) / 128;
  p.nkb = (a.Nkv + 255) / 256;
  p.causal = a.causal;
  p.layout = a.layout;
  p.scale_log2 = a.scale_log2;
  p.err = err;
  auto k = prefill_kernel<D, kInt8>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, Smem<D>::kBytes);
  if (e != cudaSuccess) return e;
  const int64_t grid = static_cast<int64_t>(p.nqt) * a.B * a.H;
  k<<<static_cast<unsigned>(grid), kThreads, Smem<D>::kBytes, st>>>(mq, mk, mv, p);
  return cudaGetLastError();
}

}  // namespace

bool prefill_supported(int D) { return D == 64 || D == 128; }

cudaError_t launch_prefill(const PrefillArgs& a, cudaStream_t st, int num_sms, int* err) {
  (void)num_sms;
  if (a.D == 128) return a.int8 ? launch_t<128, true>(a, st, err) : launch_t<128, false>(a, st, err);
  if (a.D == 64) return a.int8 ? launch_t<64, true>(a, st, err) : launch_t<64, false>(a, st, err);
  return cudaErrorInvalidValue;
}

}  // namespace qattn
