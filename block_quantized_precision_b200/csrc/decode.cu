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
// Nothing is ever written back in fp16 to global memory.
//
// decode_kernel: grid (splits, H_kv, B), 5 warps. Each CTA owns a contiguous
// range of whole chunks of one (b, h_kv) and all G = H_q / H_kv query heads
// that share it.
//   warp 4      producer: K and V chunks (64 tokens INT8 / 128 tokens INT4)
//               by TMA tensor loads with hardware swizzle into a ring (no
//               multicast); it also stages each chunk's scales and the
//               largest V scale of the chunk.
//   warps 0-3   consumers, each on its own quarter of every chunk with its
//               own running softmax, one step per chunk (16 tokens INT8, 32
//               INT4: two 16-token halves whose score MMAs are independent
//               and which share one max reduction), on the warp-level
//               tensor-core instructions:
//                 scores  S^T[16 tokens x 8 heads] = K Q^T by
//                         mma.m16n8k32 s8 x s8 -> s32: key rows straight from
//                         the swizzled tile (INT4 nibbles read as signed
//                         bytes times 16 by one mask each, the 16 folded
//                         into the group scales); the query codes live in 8
//                         registers
//                 softmax per head over the 16 tokens (shuffles), running
//                         max / sum in the log2 domain
//                 P.V     O^T[128 x heads] += V'^T P'^T by mma.m16n8k16
//                         f16 x f16 -> f32 (channels fill the 16-row side,
//                         heads the 8-column side). P' = p * (v scale /
//                         running max v scale)
//                         in [0, 1], split into an fp16 high part and an fp16
//                         remainder (two MMAs, ~22 significant bits). V' is
//                         the code plus a constant offset, exact in fp16 and
//                         built with byte permutes only (odd INT4 channels
//                         also carry a factor 16); the offsets are removed at
//                         the end with sum(P'), which two more MMAs against a
//                         tile of ones provide. V' goes through a per-warp
//                         fp16 tile and ldmatrix.trans.
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
constexpr int kStep = 16;             // tokens per consumer step
constexpr int kWsStride = kD + 4;     // floats per (b, h_q, split) partial: O[D], m, l, pad
constexpr uint32_t kOnesF16x2 = 0x3C003C00u;

template <bool kInt4>
struct Cfg {
  static constexpr int kRowBytes = kInt4 ? kD / 2 : kD;
  static constexpr int kChunk = kInt4 ? 128 : 64;             // tokens per stage
  static constexpr int kStages = 3;
  // resident CTAs per SM: 4 (<= 96 registers) for INT8; the 32-token steps
  // of INT4 need more registers: 3 (<= 136)
  static constexpr int kCtasPerSm = kInt4 ? 3 : 4;
  static constexpr int kTileBytes = kChunk * kRowBytes;       // one tensor, one stage (8 KB)
  static constexpr int kPerWarp = kChunk / kConsumers;        // tokens per warp per chunk
  static constexpr int kHalves = kInt4 ? 2 : 1;               // 16-token halves per consumer step
  // floats per head row of the per-warp P' buffer (the step's tokens + pad:
  // the rows' float2 reads of one warp fall on distinct banks)
  static constexpr int kPStride = kInt4 ? 40 : 20;
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

// D[16x8] (+)= A[16x32] B[32x8]; signed 8-bit inputs, 32-bit accumulation.
__device__ __forceinline__ void mma_s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                       uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D[16x8] += A[16x16] B[16x8], fp16 inputs, fp32 accumulation (all four
// accumulator registers used).
__device__ __forceinline__ void mma_f16x4(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                          uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// Two fp16 parts of (x, y): high = RN_f16(x, y), low = RN_f16((x, y) - high).
// Exact int -> float for |x| < 2^22 on the integer pipe: the float with
// bits 0x4B400000 + x is 1.5 * 2^23 + x, and the subtraction is exact.
__device__ __forceinline__ float i2f_exact(int x) { return __int_as_float(x + 0x4B400000) - 12582912.0f; }

__device__ __forceinline__ void split_f16x2(float x, float y, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(x, y);
  const float2 f = __half22float2(h);
  const __half2 l = __floats2half2_rn(x - f.x, y - f.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

template <int G, bool kInt4, int kGroups>
__global__ void __launch_bounds__(kThreads, Cfg<kInt4>::kCtasPerSm)
    decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const DecodeParams p) {
  static_assert(G >= 1 && G <= 8, "query heads per kv head");
  using C = Cfg<kInt4>;
  constexpr int kStages = C::kStages;
  constexpr int kTile = C::kTileBytes;
  constexpr int kNAcc = (kInt4 && kGroups == 2) ? 2 : 1;      // score accumulators (one per INT4 group)
  // V' = code + kOff (INT8, INT4 even channels) or 16 * (code + 8) + 1024
  // (INT4 odd channels, kept in stored columns 4i+2, 4i+3).
  constexpr float kOffA = kInt4 ? 1032.0f : 1152.0f;
  constexpr float kOffB = 1152.0f;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem;                          // [stages][chunk rows], swizzled
  uint8_t* sV = smem + kStages * kTile;
  float* sRed = reinterpret_cast<float*>(smem);   // after the loop: [warps][G][D]

  __shared__ __align__(16) uint32_t sQw[G][kD / 4];    // query codes, 4 per word (natural order)
  __shared__ float sQf[G];                             // sq * softmax scale * log2(e)
  // P'[head][token] per warp; rows of kPStride floats keep the stores of a
  // warp on distinct banks
  __shared__ __align__(16) float sPw[kConsumers][kGroups][8][C::kPStride];
  __shared__ float sKsc[kStages], sVsc[kStages], sVmax[kStages];
  // INT4 group scales of the chunk as float [token][group]: K as stored, V
  // already divided by the running max V scale (sVmax)
  __shared__ __align__(8) float sKsf[kInt4 ? kStages : 1][kInt4 ? C::kChunk * kGroups : 1];
  __shared__ __align__(8) float sVsf[kInt4 ? kStages : 1][kInt4 ? C::kChunk * kGroups : 1];
  __shared__ float sWm[kConsumers][8], sWl[kConsumers][8];
  __shared__ __align__(8) uint64_t full[kStages], empty[kStages];
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int g_all = p.Hq / p.Hkv;
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
  // Query codes of the G heads (consumer warps; warp w: heads w, w+4).
  if (warp < kConsumers) {
    for (int hh = warp; hh < G; hh += kConsumers) {
      const uint2 raw = *reinterpret_cast<const uint2*>(p.q + (static_cast<int64_t>(b) * p.Hq + hk * g_all + hh) * kD + lane * 4);
      const float f[4] = {bf16f(raw.x & 0xFFFF), bf16f(raw.x >> 16), bf16f(raw.y & 0xFFFF), bf16f(raw.y >> 16)};
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
      sQw[hh][lane] = w;
      if (lane == 0) sQf[hh] = sq * p.scale_log2;
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
    float vrun = 0.0f;                 // running max V scale over the chunks staged so far
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
      // The consumers weight P by v scale / running max v scale; the running
      // max (sVmax) and the weights are formed here, once per chunk.
      if constexpr (!kInt4) {
        vrun = fmaxf(vrun, fabsf(vsc));
        const float inv = vrun > 0.0f ? 1.0f / vrun : 0.0f;
        if (lane == 0) {
          sKsc[s] = ksc;
          sVsc[s] = vsc * inv;
          sVmax[s] = vrun;
        }
      } else {
        // largest V scale of the chunk (non-negative fp16 values order as
        // their bit patterns; the sign bit is cleared)
        uint32_t vm = 0;
#pragma unroll
        for (int j = 0; j < kScalePerLane; ++j) vm = max(vm, static_cast<uint32_t>(vsv[j] & 0x7FFFu));
        vm = __reduce_max_sync(0xffffffffu, vm);
        vrun = fmaxf(vrun, __half2float(__ushort_as_half(static_cast<unsigned short>(vm))));
        const float inv = vrun > 0.0f ? 1.0f / vrun : 0.0f;
#pragma unroll
        for (int j = 0; j < kScalePerLane; ++j) {
          sKsf[s][lane + 32 * j] = __half2float(__ushort_as_half(ksv[j])) * 0.0625f;   // keys arrive x16
          sVsf[s][lane + 32 * j] = __half2float(__ushort_as_half(vsv[j])) * inv;
        }
        if (lane == 0) sVmax[s] = vrun;
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
  const int gq = lane >> 2;          // mma group: token row (scores) / head row (P.V)
  const int cq = lane & 3;           // mma thread in group
  // Query fragments (B of the score MMA): for 32-channel block kb this lane
  // supplies head gq, channels kb*32 + 8*cq + {0..3} (b0) and {4..7} (b1);
  // INT4: the even channels of those 8 (b0) and the odd ones (b1). Any
  // channel order works as long as the key fragments use the same one.
  // With G <= 4 the 8 MMA columns hold each head twice (column n: head
  // n % 4): the score columns 4-7 repeat 0-3, and in P.V columns 0-3 take
  // the fp16 high part of P', columns 4-7 its remainder, so that one MMA
  // does both (the two halves are added at the end).
  constexpr bool kHiLo = G <= 4;
  const int qh = kHiLo ? (gq & 3) : gq;     // head of MMA column gq
  const bool qok = qh < G;
  uint32_t qb0[4], qb1[4];
  {
    const uint8_t* qbytes = reinterpret_cast<const uint8_t*>(&sQw[qok ? qh : 0][0]);
#pragma unroll
    for (int kb = 0; kb < 4; ++kb) {
      const int d0 = kb * 32 + 8 * cq;
      uint32_t x0, x1;
      if constexpr (!kInt4) {
        x0 = *reinterpret_cast<const uint32_t*>(qbytes + d0);
        x1 = *reinterpret_cast<const uint32_t*>(qbytes + d0 + 4);
      } else {
        const uint32_t w0 = *reinterpret_cast<const uint32_t*>(qbytes + d0);
        const uint32_t w1 = *reinterpret_cast<const uint32_t*>(qbytes + d0 + 4);
        x0 = __byte_perm(w0, w1, 0x6420);
        x1 = __byte_perm(w0, w1, 0x7531);
      }
      qb0[kb] = qok ? x0 : 0u;
      qb1[kb] = qok ? x1 : 0u;
    }
  }
  // Heads of this lane's score columns 2*cq and 2*cq + 1.
  // (with kHiLo, lanes cq >= 2 hold copies of heads 2(cq-2), 2(cq-2) + 1)
  const int h0 = kHiLo ? (2 * cq) & 3 : 2 * cq, h1 = h0 + 1;
  const bool h0ok = h0 < G, h1ok = h1 < G;
  const bool own = !kHiLo || cq < 2;        // this lane writes its heads' P' and state
  const float qf0 = h0ok ? sQf[h0] : 0.0f, qf1 = h1ok ? sQf[h1] : 0.0f;
  float (*myP)[8][C::kPStride] = sPw[warp];
  constexpr int kH = C::kHalves;
  // P.V is computed transposed, O^T[channels x heads] += V'^T P'^T, with
  // A = V'^T taken straight from the swizzled V tile: ldmatrix.trans on
  // 2-byte elements gives each lane, for tokens (2cq, 2cq+1) of a 16-token
  // step, the bytes of one 2-byte element (2 INT8 channels / 4 INT4
  // channels) of both tokens; byte permutes turn them into fp16 pairs
  // (V' = code + offset, exact). Rows of each 16-channel MMA tile are
  // therefore a permutation of the channels, undone at the output.
  // ldmatrix row of this lane: matrix lane/8 = (token half = (lane/8)%2,
  // 16-byte chunk offset = lane/16), row lane%8 = token.
  const int ldsm_tok = ((lane >> 3) & 1) * 8 + (lane & 7);
  const int ldsm_chunk = lane >> 4;
  float m_run0 = -CUDART_INF_F, m_run1 = -CUDART_INF_F;   // heads h0, h1
  float l_run0 = 0.0f, l_run1 = 0.0f;                      // over this lane's tokens
  float vref = 0.0f;                                       // running max V scale
  // acc[mt]: stored channels 16mt + gq ([0] head h0, [1] head h1) and
  // 16mt + gq + 8 ([2] h0, [3] h1); sacc[gg]: sum of P' of group gg for
  // heads h0 ([0]) and h1 ([1]).
  float acc[8][4];
  float sacc[kGroups][4];
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.0f;
#pragma unroll
  for (int gg = 0; gg < kGroups; ++gg) sacc[gg][0] = sacc[gg][1] = sacc[gg][2] = sacc[gg][3] = 0.0f;

  for (int c = 0; c < nchunks; ++c) {
    const int s = c % kStages;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&full[s], (c / kStages) & 1, &abort_flag, p.err));
    if (!ok) break;
    const uint8_t* cK = sK + s * kTile;
    const uint8_t* cV = sV + s * kTile;
    const int chunk_t0 = t_begin + c * C::kChunk;
    // running V-scale reference: P' = p * vscale / vref stays in [0, 1]
    const float vref_new = fmaxf(vref, sVmax[s]);
    const float vratio = vref_new > 0.0f ? vref / vref_new : 1.0f;
    vref = vref_new;
    if (vratio != 1.0f) {                     // the same on every lane
#pragma unroll
      for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[mt][e] *= vratio;
#pragma unroll
      for (int gg = 0; gg < kGroups; ++gg)
#pragma unroll
        for (int e = 0; e < 4; ++e) sacc[gg][e] *= vratio;
    }
#pragma unroll 1
    for (int sub = 0; sub < C::kPerWarp / (kStep * kH); ++sub) {
      const int r0 = warp * C::kPerWarp + sub * kStep * kH;  // first row of this step in the chunk
      // ---------------- scores: S^T = K Q^T, per 16-token half ----------------
      // sv[hf]: (row ra, head h0), (ra, h1), (rb, h0), (rb, h1) with ra =
      // r0 + 16 hf + gq, rb = ra + 8 (the accumulator layout)
      float sv[kH][4];
#pragma unroll
      for (int hf = 0; hf < kH; ++hf) {
        const int ra = r0 + kStep * hf + gq, rb = ra + 8;   // this lane's score rows (tokens)
        const bool va = chunk_t0 + ra < t_end, vb = chunk_t0 + rb < t_end;
        // INT8: one accumulator per 32-channel slice so that the four MMAs do
        // not wait on one another; INT4: one per 64-channel half (the two
        // 16-token halves of a step supply the independent chains); the
        // accumulators are then added (exact in INT32)
        constexpr int kAcc = kInt4 ? 2 : 4;
        int sck[kAcc][4];
#pragma unroll
        for (int a = 0; a < kAcc; ++a) sck[a][0] = sck[a][1] = sck[a][2] = sck[a][3] = 0;
#pragma unroll
        for (int kb = 0; kb < 4; ++kb) {
          if constexpr (!kInt4) {
            // 8 bytes of rows ra / rb at channel kb*32 + 8*cq: 16-byte chunk
            // 2kb + cq/2, stored at chunk ^ (row % 8)
            const int ch = 2 * kb + (cq >> 1);
            const int off = ((ch ^ gq) << 4) + (cq & 1) * 8;
            const uint2 xa = *reinterpret_cast<const uint2*>(cK + ra * 128 + off);
            const uint2 xb = *reinterpret_cast<const uint2*>(cK + rb * 128 + off);
            mma_s8(sck[kb], xa.x, xb.x, xa.y, xb.y, qb0[kb], qb1[kb]);
          } else {
            // 4 bytes (8 nibbles) of rows ra / rb at channel kb*32 + 8*cq:
            // 16-byte chunk kb, stored at kb ^ ((row / 2) % 4)
            const int off = ((kb ^ ((gq >> 1) & 3)) << 4) + 4 * cq;
            const uint32_t wa = *reinterpret_cast<const uint32_t*>(cK + ra * 64 + off);
            const uint32_t wb = *reinterpret_cast<const uint32_t*>(cK + rb * 64 + off);
            // the nibbles as signed bytes times 16 (exact two's complement):
            // high nibble w & 0xF0 (odd channels), low nibble (w << 4) & 0xF0
            // (even channels); the factor 16 is in the group scales
            const uint32_t ea = (wa << 4) & 0xF0F0F0F0u, oa = wa & 0xF0F0F0F0u;
            const uint32_t eb = (wb << 4) & 0xF0F0F0F0u, ob = wb & 0xF0F0F0F0u;
            mma_s8(sck[kb >> 1], ea, eb, oa, ob, qb0[kb], qb1[kb]);
          }
        }
        int sc[kNAcc][4];                                  // per INT4 group (else all 128 channels)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if constexpr (kNAcc == 2) {
            sc[0][e] = sck[0][e];
            sc[kNAcc - 1][e] = sck[kAcc - 1][e];
          } else if constexpr (kInt4) {
            sc[0][e] = sck[0][e] + sck[kAcc - 1][e];
          } else {
            sc[0][e] = (sck[0][e] + sck[1][e]) + (sck[kAcc - 2][e] + sck[kAcc - 1][e]);
          }
        }
        if constexpr (!kInt4) {
          const float kq0 = qf0 * sKsc[s], kq1 = qf1 * sKsc[s];
          sv[hf][0] = i2f_exact(sc[0][0]) * kq0;
          sv[hf][1] = i2f_exact(sc[0][1]) * kq1;
          sv[hf][2] = i2f_exact(sc[0][2]) * kq0;
          sv[hf][3] = i2f_exact(sc[0][3]) * kq1;
        } else {
          float t0 = 0.0f, t1 = 0.0f, t2 = 0.0f, t3 = 0.0f;
#pragma unroll
          for (int gg = 0; gg < kNAcc; ++gg) {
            const float ka = sKsf[s][ra * kGroups + gg];
            const float kb2 = sKsf[s][rb * kGroups + gg];
            t0 = fmaf(i2f_exact(sc[gg][0]), ka, t0);
            t1 = fmaf(i2f_exact(sc[gg][1]), ka, t1);
            t2 = fmaf(i2f_exact(sc[gg][2]), kb2, t2);
            t3 = fmaf(i2f_exact(sc[gg][3]), kb2, t3);
          }
          sv[hf][0] = t0 * qf0; sv[hf][1] = t1 * qf1; sv[hf][2] = t2 * qf0; sv[hf][3] = t3 * qf1;
        }
        if (!va) { sv[hf][0] = -CUDART_INF_F; sv[hf][1] = -CUDART_INF_F; }
        if (!vb) { sv[hf][2] = -CUDART_INF_F; sv[hf][3] = -CUDART_INF_F; }
      }
      // ---------------- running softmax per head over the step's tokens ----------------
      float mx0 = fmaxf(sv[0][0], sv[0][2]), mx1 = fmaxf(sv[0][1], sv[0][3]);
#pragma unroll
      for (int hf = 1; hf < kH; ++hf) {
        mx0 = fmaxf(mx0, fmaxf(sv[hf][0], sv[hf][2]));
        mx1 = fmaxf(mx1, fmaxf(sv[hf][1], sv[hf][3]));
      }
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
      }
      if (mx0 == -CUDART_INF_F) continue;     // no valid token in this step (the same on every lane)
      const float mn0 = fmaxf(m_run0, mx0), mn1 = fmaxf(m_run1, mx1);
      const float al0 = ex2(m_run0 - mn0), al1 = ex2(m_run1 - mn1);
      m_run0 = mn0;
      m_run1 = mn1;
      float pr[kH][4];
      float ls0 = 0.0f, ls1 = 0.0f;
#pragma unroll
      for (int hf = 0; hf < kH; ++hf) {
        pr[hf][0] = ex2(sv[hf][0] - mn0);
        pr[hf][1] = ex2(sv[hf][1] - mn1);
        pr[hf][2] = ex2(sv[hf][2] - mn0);
        pr[hf][3] = ex2(sv[hf][3] - mn1);
        ls0 += pr[hf][0] + pr[hf][2];
        ls1 += pr[hf][1] + pr[hf][3];
      }
      l_run0 = l_run0 * al0 + ls0;
      l_run1 = l_run1 * al1 + ls1;
      // P' = p * vscale / vref -> per-warp buffer [group][head][token of the step]
#pragma unroll
      for (int hf = 0; hf < kH; ++hf) {
        const int ta = kStep * hf + gq;                    // token of row ra within the step
        if constexpr (!kInt4) {
          const float f = sVsc[s];
          if (own && h0ok) { myP[0][h0][ta] = pr[hf][0] * f; myP[0][h0][ta + 8] = pr[hf][2] * f; }
          if (own && h1ok) { myP[0][h1][ta] = pr[hf][1] * f; myP[0][h1][ta + 8] = pr[hf][3] * f; }
        } else {
          const int ra = r0 + ta, rb = ra + 8;
#pragma unroll
          for (int gg = 0; gg < kGroups; ++gg) {
            const float fa = sVsf[s][ra * kGroups + gg];
            const float fb = sVsf[s][rb * kGroups + gg];
            if (own && h0ok) { myP[gg][h0][ta] = pr[hf][0] * fa; myP[gg][h0][ta + 8] = pr[hf][2] * fb; }
            if (own && h1ok) { myP[gg][h1][ta] = pr[hf][1] * fa; myP[gg][h1][ta + 8] = pr[hf][3] * fb; }
          }
        }
      }
      __syncwarp();
      // ---------------- rescale O^T and sum(P') by alpha (heads h0, h1 of this lane) ----------------
      if (!__all_sync(0xffffffffu, al0 == 1.0f && al1 == 1.0f)) {
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          acc[mt][0] *= al0; acc[mt][1] *= al1; acc[mt][2] *= al0; acc[mt][3] *= al1;
        }
#pragma unroll
        for (int gg = 0; gg < kGroups; ++gg) {
          sacc[gg][0] *= al0; sacc[gg][1] *= al1; sacc[gg][2] *= al0; sacc[gg][3] *= al1;
        }
      }
#pragma unroll
      for (int hf = 0; hf < kH; ++hf) {
        // P'^T fragments (B): column gq = head qh, tokens 2cq, 2cq+1 (b0) and
        // 2cq+8, 2cq+9 (b1) of this half, as fp16 high and low parts; with
        // kHiLo column gq carries the high part (gq < 4) or the remainder
        // (gq >= 4) alone, in the *_hi registers
        uint32_t p0_hi[kGroups], p0_lo[kGroups], p1_hi[kGroups], p1_lo[kGroups];
#pragma unroll
        for (int gg = 0; gg < kGroups; ++gg) {
          float2 x01 = make_float2(0.0f, 0.0f), x89 = make_float2(0.0f, 0.0f);
          if (qok) {
            x01 = *reinterpret_cast<const float2*>(&myP[gg][qh][kStep * hf + 2 * cq]);
            x89 = *reinterpret_cast<const float2*>(&myP[gg][qh][kStep * hf + 2 * cq + 8]);
          }
          split_f16x2(x01.x, x01.y, p0_hi[gg], p0_lo[gg]);
          split_f16x2(x89.x, x89.y, p1_hi[gg], p1_lo[gg]);
          if constexpr (kHiLo) {
            if (gq >= 4) { p0_hi[gg] = p0_lo[gg]; p1_hi[gg] = p1_lo[gg]; }
          }
        }
        // ---------------- O^T += V'^T P'^T, sum(P') against a tile of ones ----------------
        const int vt = r0 + kStep * hf + ldsm_tok;            // this lane's ldmatrix row (token)
        const uint32_t vrow = smem_u32(cV + vt * C::kRowBytes);
#pragma unroll
        for (int cp = 0; cp < (kInt4 ? 2 : 4); ++cp) {        // pairs of 16-byte chunks
          const int chunk = 2 * cp + ldsm_chunk;
          const int pos = kInt4 ? (chunk ^ ((vt >> 1) & 3)) : (chunk ^ (vt & 7));
          uint32_t r[4];                                     // (tokens 0-7 | 8-15) x (chunk 2cp | 2cp+1)
          ldsm_x4_trans(vrow + (pos << 4), r[0], r[1], r[2], r[3]);
          if constexpr (!kInt4) {
            // chunk 2cp + h -> m-tile 2cp + h: row g = channel 2g, row g+8 =
            // channel 2g+1 of the chunk; byte b -> fp16 bits 0x64 | (b ^ 0x80)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint32_t xl = r[2 * h] ^ 0x80808080u, xh = r[2 * h + 1] ^ 0x80808080u;
              const uint32_t a0 = __byte_perm(xl, 0x64646464u, 0x4240), a1 = __byte_perm(xl, 0x64646464u, 0x4341);
              const uint32_t a2 = __byte_perm(xh, 0x64646464u, 0x4240), a3 = __byte_perm(xh, 0x64646464u, 0x4341);
              const int mt = 2 * cp + h;
              mma_f16x4(acc[mt], a0, a1, a2, a3, p0_hi[0], p1_hi[0]);
              if constexpr (!kHiLo) mma_f16x4(acc[mt], a0, a1, a2, a3, p0_lo[0], p1_lo[0]);
            }
          } else {
            // chunk 2cp + h (32 channels) -> m-tiles 4cp + 2h + u: row g =
            // channel 4g + 2u (low nibble, 1032 + code), row g+8 = channel
            // 4g + 2u + 1 (high nibble, 1152 + 16 code); byte 0 of each
            // 16-bit half is already in place (u = 0), byte 1 is moved down
#pragma unroll
            for (int h = 0; h < 2; ++h) {
#pragma unroll
              for (int u = 0; u < 2; ++u) {
                const uint32_t yl = u ? __byte_perm(r[2 * h], 0u, 0x4341) : r[2 * h];
                const uint32_t yh = u ? __byte_perm(r[2 * h + 1], 0u, 0x4341) : r[2 * h + 1];
                const uint32_t a0 = (yl & 0x000F000Fu) ^ 0x64086408u, a1 = (yl & 0x00F000F0u) ^ 0x64806480u;
                const uint32_t a2 = (yh & 0x000F000Fu) ^ 0x64086408u, a3 = (yh & 0x00F000F0u) ^ 0x64806480u;
                const int mt = 4 * cp + 2 * h + u;
                const int gg = (kGroups == 2 && mt >= 4) ? 1 : 0;
                mma_f16x4(acc[mt], a0, a1, a2, a3, p0_hi[gg], p1_hi[gg]);
                if constexpr (!kHiLo) mma_f16x4(acc[mt], a0, a1, a2, a3, p0_lo[gg], p1_lo[gg]);
              }
            }
          }
        }
#pragma unroll
        for (int gg = 0; gg < kGroups; ++gg) {
          mma_f16x4(sacc[gg], kOnesF16x2, kOnesF16x2, kOnesF16x2, kOnesF16x2, p0_hi[gg], p1_hi[gg]);
          if constexpr (!kHiLo)
            mma_f16x4(sacc[gg], kOnesF16x2, kOnesF16x2, kOnesF16x2, kOnesF16x2, p0_lo[gg], p1_lo[gg]);
        }
      }
      __syncwarp();                  // buffers reused by the next step
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }

  // ---------------- merge the four consumer warps ----------------
  // l: sum over the 8 token rows (lanes with the same cq)
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    l_run0 += __shfl_xor_sync(0xffffffffu, l_run0, o);
    l_run1 += __shfl_xor_sync(0xffffffffu, l_run1, o);
  }
  // every issued copy was consumed (or waited for on a timeout): the ring can
  // be reused for the reduction once all consumer warps are past their loops
  named_bar_sync(1, 32 * kConsumers);
  if (gq == 0 && own) {
    if (h0ok) { sWm[warp][h0] = m_run0; sWl[warp][h0] = l_run0; }
    if (h1ok) { sWm[warp][h1] = m_run1; sWl[warp][h1] = l_run1; }
  }
  if constexpr (kHiLo) {
    // columns 2cq, 2cq+1 (cq < 2) gathered the high parts of P', columns
    // 2cq+4, 2cq+5 (lane ^ 2) the remainders of the same heads
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][e] += __shfl_xor_sync(0xffffffffu, acc[mt][e], 2);
#pragma unroll
    for (int gg = 0; gg < kGroups; ++gg)
#pragma unroll
      for (int e = 0; e < 4; ++e) sacc[gg][e] += __shfl_xor_sync(0xffffffffu, sacc[gg][e], 2);
  }
  // O = (acc - offset * sum(P')) * vref; INT4 odd channels also / 16.
  // Row g of m-tile mt holds channel 16mt + 2g (INT8) or 32(mt/4)... see the
  // P.V comment: INT8 rows g / g+8 = channels 16mt + 2g / +1; INT4 rows
  // g / g+8 = channels 32(mt/2) + 4g + 2(mt%2) / +1.
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) {
    const int gg = (kGroups == 2 && mt >= 4) ? 1 : 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int hh = 2 * cq + (e & 1);
      if (hh >= G || !own) continue;
      const bool odd = (e >> 1) != 0;                        // row g+8
      const float sp = sacc[gg][e & 1];
      float o;
      int ch;
      if constexpr (kInt4) {
        ch = 32 * (mt >> 1) + 4 * gq + 2 * (mt & 1) + (odd ? 1 : 0);
        o = (acc[mt][e] - (odd ? kOffB : kOffA) * sp) * (odd ? vref * 0.0625f : vref);
      } else {
        ch = 16 * mt + 2 * gq + (odd ? 1 : 0);
        o = (acc[mt][e] - kOffA * sp) * vref;
      }
      sRed[(warp * G + hh) * kD + ch] = o;
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
    float* wsp = p.ws + ((static_cast<int64_t>(b) * p.Hq + hk * g_all + hh) * p.splits + split) * kWsStride;
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
  cudaError_t e = set_max_dyn_smem(reinterpret_cast<const void*>(k), Cfg<kInt4>::kSmemBytes);
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
// fullest). Cfg::kCtasPerSm CTAs per SM are resident.
static int splits_for(int B, int Hkv, int L, int num_sms, bool int4) {
  const int ck = chunk_tokens(int4);
  const int chunks = (L + ck - 1) / ck;
  if (chunks == 0) return 1;
  const int64_t pairs = static_cast<int64_t>(B) * Hkv;
  const int64_t slots = static_cast<int64_t>(num_sms) * (int4 ? Cfg<true>::kCtasPerSm : Cfg<false>::kCtasPerSm);
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

size_t decode_workspace_bytes_for(int B, int Hq, int Hkv, int L, bool int4, int num_sms) {
  const int splits = splits_for(B, Hkv, L, num_sms, int4);
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
