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
    float m_run = -CUDART_INF_F, l_run = 0.0f;
    uint8_t* prow = sP + r * 128;
    const int rsw = r & 7;
    bool ok = true;
    for (int j = 0; j < ntiles; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bar_s_full, j & 1, &abort_flag, p.err));
      if (!ok) break;
      tc_fence_after();
      const float ksc = sq * p.ks[static_cast<int64_t>(bh) * p.nkb + (j >> 1)] * p.scale_log2;
      const int key0 = j * kTileN;
      int kmax = p.Nkv - key0;                    // keys valid for this row: [0, kmax)
      if (p.causal) kmax = min(kmax, qrow - key0 + 1);
      // pass 1: row max of the scaled scores
      float tmax = -CUDART_INF_F;
#pragma unroll 1
      for (int c = 0; c < kTileN / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(trow + c * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float sv = kInt8 ? static_cast<float>(static_cast<int>(v[e])) : __uint_as_float(v[e]);
          if (c * 32 + e < kmax) tmax = fmaxf(tmax, sv * ksc);
        }
      }
      const float m_new = fmaxf(m_run, tmax);
      const float alpha = ex2(m_run - m_new);     // 0 on the first tile
      // pass 2: probabilities, 8-bit rounding, P to shared memory
      float rowsum = 0.0f;
      int rowsum_i = 0;
#pragma unroll 1
      for (int c = 0; c < kTileN / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(trow + c * 32, v);
        tmem_wait_ld();
        uint32_t packed[8];
#pragma unroll
        for (int w = 0; w < 8; ++w) {
          float pr[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int col = c * 32 + w * 4 + e;
            const float sv = kInt8 ? static_cast<float>(static_cast<int>(v[w * 4 + e])) : __uint_as_float(v[w * 4 + e]);
            pr[e] = col < kmax ? ex2(sv * ksc - m_new) : 0.0f;
          }
          if constexpr (kInt8) {
            uint32_t word = 0;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int code = __float2int_rn(pr[e] * 127.0f);
              rowsum_i += code;
              word |= static_cast<uint32_t>(code) << (8 * e);
            }
            packed[w] = word;
          } else {
            const uint32_t lo = cvt_e4m3x2(pr[0], pr[1]);
            const uint32_t hi = cvt_e4m3x2(pr[2], pr[3]);
            packed[w] = lo | (hi << 16);
            uint32_t h0 = cvt_e4m3x2_to_f16x2(static_cast<uint16_t>(lo));
            uint32_t h1 = cvt_e4m3x2_to_f16x2(static_cast<uint16_t>(hi));
            const float2 f0 = __half22float2(*reinterpret_cast<const __half2*>(&h0));
            const float2 f1 = __half22float2(*reinterpret_cast<const __half2*>(&h1));
            rowsum += (f0.x + f0.y) + (f1.x + f1.y);
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
      if constexpr (kInt8) rowsum = static_cast<float>(rowsum_i) * (1.0f / 127.0f);
      tc_fence_before();
      fence_proxy_async_smem();
      mbar_arrive(&bar_p_full);
      l_run = l_run * alpha + rowsum;
      m_run = m_new;

      // fold PV into O
      ok = __all_sync(0xffffffffu, mbar_wait(&bar_pv_full, j & 1, &abort_flag, p.err));
      if (!ok) break;
      tc_fence_after();
      const float cj = p.vs[static_cast<int64_t>(bh) * p.nkb + (j >> 1)] * (kInt8 ? (1.0f / 127.0f) : 1.0f);
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t pv[32], o[32];
        tmem_ld32(trow + c * 32, pv);
        if (j > 0) tmem_ld32(trow + kColO + c * 32, o);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float x = kInt8 ? static_cast<float>(static_cast<int>(pv[e])) : __uint_as_float(pv[e]);
          const float prev = j > 0 ? __uint_as_float(o[e]) * alpha : 0.0f;
          o[e] = __float_as_uint(fmaf(x, cj, prev));
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
