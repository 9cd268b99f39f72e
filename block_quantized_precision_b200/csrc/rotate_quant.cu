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
//   quant_kernel  (no R): HBM bound. Persistent CTAs stream whole blocks
//                 through a three-stage shared-memory ring by TMA (two blocks
//                 ahead); block max on the raw 16-bit lanes, codes by the
//                 division-free path, the rare undecided values redone one by
//                 one from the IEEE quotient.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "qattn_device.cuh"
#include "qattn_internal.h"

namespace qattn {

namespace {

// Threads per team (one team computes one block at a time): at D = 128,
// 8 x 8 thread tiles, 256 threads for 128-token blocks (two teams per CTA
// share R, so one team's staging and coding overlap the other's FMA loop;
// 256 threads keep the FMA pipe near 88 % busy while a team computes alone)
// and 512 for 256-token blocks (one team); at D = 64, 4 x 8 tiles (256
// threads).
template <int D, int T>
struct RotqThreads {
  static constexpr int value = D == 128 ? (T == 256 ? 512 : 256) : 256;
};
template <int D, int T>
struct RotqTeams {
  static constexpr int value = D == 128 && T == 128 ? 2 : 1;
};

// Barrier of one team: the whole CTA when it is the only team, else the
// team's named barrier (1 + team).
template <int kNT, int kTeams>
__device__ __forceinline__ void team_sync(int team) {
  if constexpr (kTeams == 1) __syncthreads();
  else named_bar_sync(1 + team, kNT);
}

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

// True on every thread of the team iff v is true on every thread of it
// (a barrier with an AND reduction: the whole CTA for one team, else the
// team's named barrier 1 + team).
template <int kNT, int kTeams>
__device__ __forceinline__ bool team_all(bool v, int team) {
  if constexpr (kTeams == 1) return __syncthreads_and(v) != 0;
  int r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.b32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\tselp.b32 %0, 1, 0, q;\n\t}\n"
      : "=r"(r)
      : "r"(static_cast<int>(v)), "r"(1 + team), "r"(kNT)
      : "memory");
  return r != 0;
}

// Maximum of v over the kNT threads of a team (ttid: thread within the team;
// red: kNT / 32 floats of the team).
template <int kNT, int kTeams = 1>
__device__ __forceinline__ float block_max(float v, float* red, int ttid = threadIdx.x, int team = 0) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = ttid >> 5;
  if ((ttid & 31) == 0) red[w] = v;
  team_sync<kNT, kTeams>(team);
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < kNT / 32; ++i) m = fmaxf(m, red[i]);
  team_sync<kNT, kTeams>(team);  // red[] may be reused
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

// Eight integer codes held in the low bits of t[e] (two's complement, |c| <= 7)
// -> one word of nibbles, element e in bits 4e .. 4e+3.
__device__ __forceinline__ uint32_t pack_nibbles8(const uint32_t (&t)[8]) {
  uint32_t w = 0;
#pragma unroll
  for (int e = 0; e < 8; ++e) w |= (t[e] & 0xFu) << (4 * e);
  return w;
}

// Codes of 8 values by the division-free path, packed little-endian into lo
// (values 0..3) and hi (4..7). Returns false when any value is too close to a
// rounding boundary (or, for e4m3, in the subnormal range) for the product
// with rcp to be trusted; the caller then takes the exact path.
//   INT8 (pairs of values per f32x2 FMA): m = RN(y * rcp + 1.5 * 2^23) holds
//   RNE(y * rcp) in its low mantissa bits; d = y * rcp - that integer
//   (the exact product, one rounding). y * rcp is within 1.5e-5 of the IEEE
//   quotient (|quotient| <= 127.5), so every code agrees with it when
//   max |d| <= 0.4999.
//   e4m3: as code_of.
// kPacked false: the same INT8 decision one value at a time (d from
// y * rcp rounded first; the bound holds as well). The rotation kernel uses
// it: the packed form measured slower there, its FMA loop being compiled
// differently next to it.
template <bool kInt8, bool kPacked = true, bool kInt4 = false>
__device__ __forceinline__ bool codes8_fast(const float (&f)[8], float rcp, uint32_t& lo, uint32_t& hi) {
  uint32_t t[8];
  if constexpr (kInt8 && !kPacked) {
    bool ok = true;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float v0 = f[e] * rcp;
      const float m = v0 + 12582912.0f;                  // RNE integer in the low mantissa bits
      ok = ok && fabsf(v0 - (m - 12582912.0f)) <= 0.4999f;
      t[e] = __float_as_uint(m);
    }
    if constexpr (kInt4) {
      lo = pack_nibbles8(t);
      hi = 0;
    } else {
      lo = __byte_perm(__byte_perm(t[0], t[1], 0x0040), __byte_perm(t[2], t[3], 0x0040), 0x5410);
      hi = __byte_perm(__byte_perm(t[4], t[5], 0x0040), __byte_perm(t[6], t[7], 0x0040), 0x5410);
    }
    return ok;
  } else if constexpr (kInt8) {
    const float2 rc = make_float2(rcp, rcp);
    const float2 mg = make_float2(12582912.0f, 12582912.0f);
    float dmax = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 y = make_float2(f[2 * i], f[2 * i + 1]);
      const float2 m = ffma2(y, rc, mg);
      const float2 nr = ffma2(m, make_float2(-1.0f, -1.0f), mg);     // -RNE(y * rcp), exact
      const float2 d = ffma2(y, rc, nr);
      dmax = fmaxf(dmax, fmaxf(fabsf(d.x), fabsf(d.y)));
      t[2 * i] = __float_as_uint(m.x);
      t[2 * i + 1] = __float_as_uint(m.y);
    }
    if constexpr (kInt4) {
      lo = pack_nibbles8(t);
      hi = 0;
    } else {
      lo = __byte_perm(__byte_perm(t[0], t[1], 0x0040), __byte_perm(t[2], t[3], 0x0040), 0x5410);
      hi = __byte_perm(__byte_perm(t[4], t[5], 0x0040), __byte_perm(t[6], t[7], 0x0040), 0x5410);
    }
    return dmax <= 0.4999f;
  } else {
    bool ok = true;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float v0 = f[e] * rcp;
      const uint32_t bb = __float_as_uint(v0) & 0x7FFFFFFFu;
      ok = ok && bb >= 0x3C800000u && abs(static_cast<int>(bb & 0xFFFFFu) - 0x80000) > 16;
      t[e] = __float_as_uint(v0);
    }
    lo = cvt_e4m3x2(__uint_as_float(t[0]), __uint_as_float(t[1])) |
         (cvt_e4m3x2(__uint_as_float(t[2]), __uint_as_float(t[3])) << 16);
    hi = cvt_e4m3x2(__uint_as_float(t[4]), __uint_as_float(t[5])) |
         (cvt_e4m3x2(__uint_as_float(t[6]), __uint_as_float(t[7])) << 16);
    return ok;
  }
}

// The packed INT8 / e4m3 fast path with one flag per value: bit e of the
// result is set when value e's code must come from the IEEE quotient (same
// bounds as codes8_fast). The codes of unflagged values are final.
// kInt4 (with kInt8): the same integer codes (|quotient| <= 7.5), packed two
// per byte into lo (element 2i in the low nibble of byte i); hi is unused.
template <bool kInt8, bool kInt4 = false>
__device__ __forceinline__ uint32_t codes8_flags(const float (&f)[8], float rcp, uint32_t& lo, uint32_t& hi) {
  uint32_t t[8];
  uint32_t flags = 0;
  if constexpr (kInt8) {
    const float2 rc = make_float2(rcp, rcp);
    const float2 mg = make_float2(12582912.0f, 12582912.0f);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 y = make_float2(f[2 * i], f[2 * i + 1]);
      const float2 m = ffma2(y, rc, mg);
      const float2 nr = ffma2(m, make_float2(-1.0f, -1.0f), mg);     // -RNE(y * rcp), exact
      const float2 d = ffma2(y, rc, nr);
      flags |= (fabsf(d.x) > 0.4999f ? 1u : 0u) << (2 * i);
      flags |= (fabsf(d.y) > 0.4999f ? 1u : 0u) << (2 * i + 1);
      t[2 * i] = __float_as_uint(m.x);
      t[2 * i + 1] = __float_as_uint(m.y);
    }
    if constexpr (kInt4) {
      lo = pack_nibbles8(t);
      hi = 0;
    } else {
      lo = __byte_perm(__byte_perm(t[0], t[1], 0x0040), __byte_perm(t[2], t[3], 0x0040), 0x5410);
      hi = __byte_perm(__byte_perm(t[4], t[5], 0x0040), __byte_perm(t[6], t[7], 0x0040), 0x5410);
    }
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float v0 = f[e] * rcp;
      const uint32_t bb = __float_as_uint(v0) & 0x7FFFFFFFu;
      flags |= (bb < 0x3C800000u || abs(static_cast<int>(bb & 0xFFFFFu) - 0x80000) <= 16 ? 1u : 0u) << e;
      t[e] = __float_as_uint(v0);
    }
    lo = cvt_e4m3x2(__uint_as_float(t[0]), __uint_as_float(t[1])) |
         (cvt_e4m3x2(__uint_as_float(t[2]), __uint_as_float(t[3])) << 16);
    hi = cvt_e4m3x2(__uint_as_float(t[4]), __uint_as_float(t[5])) |
         (cvt_e4m3x2(__uint_as_float(t[6]), __uint_as_float(t[7])) << 16);
  }
  return flags;
}

// Code byte of one value from the IEEE quotient (the rare path; inline, as a
// call per value measured far slower).
template <bool kInt8, bool kInt4 = false>
__device__ __forceinline__ uint32_t code_exact(float y, float scale) {
  const float v = __fdiv_rn(y, scale);
  if constexpr (kInt4) return static_cast<uint32_t>(max(-7, min(7, __float2int_rn(v)))) & 0xFu;
  else if constexpr (kInt8) return static_cast<uint32_t>(max(-127, min(127, __float2int_rn(v)))) & 0xFFu;
  else return cvt_e4m3x2(v, 0.0f) & 0xFFu;
}

// Eight float32 values, passed by value to the rare exact path.
struct F8 {
  float v[8];
};

// Codes of 8 values with the IEEE quotient for every value, packed like
// codes8_fast.
template <bool kInt8, bool kInt4 = false>
__device__ __noinline__ uint2 codes8_exact_f(F8 f, float scale) {
  if constexpr (kInt4) {
    uint32_t w = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) w |= code_exact<true, true>(f.v[e], scale) << (4 * e);
    return make_uint2(w, 0);
  }
  uint32_t lo = 0, hi = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) lo |= code_of<kInt8>(f.v[j], scale, 0.0f, true) << (8 * j);
#pragma unroll
  for (int j = 0; j < 4; ++j) hi |= code_of<kInt8>(f.v[j + 4], scale, 0.0f, true) << (8 * j);
  return make_uint2(lo, hi);
}

// ---------------------------------------------------------------------------
// With rotation
// ---------------------------------------------------------------------------

// Thread tile: kRPT rows x 8 columns of y. Column group cg = tid % (D/8)
// owns columns 4cg..4cg+3 and D/2+4cg..D/2+4cg+3 (two float4 of each R row,
// consecutive across the warp, so the R reads are free of bank conflicts);
// row group rg = tid / (D/8) owns rows rg*kRPT .. rg*kRPT + kRPT - 1.
// kInt4 (with kInt8): INT4 codes (scale absmax / 7), two per byte.
template <int D, int T, bool kInt8, bool kInt4>
__global__ void __launch_bounds__(RotqThreads<D, T>::value * RotqTeams<D, T>::value, 1)
    rotq_kernel(const uint16_t* __restrict__ x, int is_bf16, int layout, int B, int H, int N,
                const float* __restrict__ rot, uint8_t* __restrict__ codes,
                float* __restrict__ scales, int* err) {
  constexpr int kNT = RotqThreads<D, T>::value;
  constexpr int kTeams = RotqTeams<D, T>::value;
  constexpr int kCG = D / 8;               // column groups
  constexpr int kRG = kNT / kCG;           // row groups
  constexpr int kRPT = T / kRG;            // rows per thread
  constexpr int kXS = T + 4;               // padded row stride of the transposed x tile
  static_assert(kRPT % 4 == 0 && kRPT >= 4, "row tile");
  extern __shared__ __align__(16) float smem[];
  const int team = threadIdx.x / kNT;
  const int tid = threadIdx.x % kNT;       // thread within the team
  float* sR = smem;                        // [D][D]
  float* sX = smem + D * D + team * D * kXS;   // this team's [D][kXS]: sX[k * kXS + r] = x[r][k]
  __shared__ float red_all[kTeams][kNT / 32];
  float* red = red_all[team];
  // start1: completes when team 0 has finished its first FMA loop (two teams)
  __shared__ __align__(8) uint64_t start1;
  if (kTeams > 1 && threadIdx.x == 0) {
    mbar_init(&start1, kNT);
    mbar_fence_init();
  }

  for (int i = threadIdx.x; i < D * D / 4; i += kNT * kTeams)
    reinterpret_cast<float4*>(sR)[i] = reinterpret_cast<const float4*>(rot)[i];
  if constexpr (kTeams > 1) __syncthreads();   // sR ready

  const int nblk = (N + T - 1) / T;
  const int64_t total = static_cast<int64_t>(B) * H * nblk;
  const int cg = tid % kCG, rg = tid / kCG;
  const int c0 = 4 * cg, c1 = D / 2 + 4 * cg;   // this thread's two column quads
  const float qmax = kInt4 ? 7.0f : kInt8 ? 127.0f : 448.0f;

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
  // Team t of CTA c takes the blocks c + (t + kTeams i) * gridDim.x.
  const int64_t first = blockIdx.x + static_cast<int64_t>(team) * gridDim.x;
  const int64_t step = static_cast<int64_t>(kTeams) * gridDim.x;
  if (kPrefetch && first < total) load_block(first);
  // With two teams, team 1 starts its first FMA loop once team 0 has
  // finished its own, so that the teams' loops run out of phase and one
  // team's loading, staging and coding overlap the other's loop. (Strict
  // turn-taking of every loop measured slower.) Team 0 arrives only if team
  // 1 has a block; the wait is bounded (QATTN_ERR_TIMEOUT, and the team
  // stops).
  const bool team1_has_work = blockIdx.x + static_cast<int64_t>(gridDim.x) < total;
  int64_t it = 0;

  for (int64_t blk_id = first; blk_id < total; blk_id += step, ++it) {
    const int blk = static_cast<int>(blk_id % nblk);
    const int bh = static_cast<int>(blk_id / nblk);
    const int b = bh / H, h = bh % H;
    const int n0 = blk * T;
    const int rows = min(T, N - n0);

    if (!kPrefetch) load_block(blk_id);
    team_sync<kNT, kTeams>(team);  // sR ready (first pass); previous block's sX reads done
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
    team_sync<kNT, kTeams>(team);
    if (kPrefetch && blk_id + step < total) load_block(blk_id + step);
    if constexpr (kTeams > 1) {
      if (team == 1 && it == 0) {
        const bool ok = mbar_wait(&start1, 0, nullptr, err);
        if (!team_all<kNT, kTeams>(ok, team)) break;
      }
    }

    // acc[p][j]: rows rg*kRPT + 2p (.x) and + 2p + 1 (.y), column (j < 4 ?
    // c0 + j : c1 + j - 4); each is the float32 FMA chain over k ascending,
    // two rows per f32x2 FMA (x pairs straight from the transposed tile, the
    // R value duplicated).
    float2 acc[kRPT / 2][8];
#pragma unroll
    for (int i = 0; i < kRPT / 2; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = make_float2(0.0f, 0.0f);

#pragma unroll 2
    for (int k = 0; k < D; ++k) {
      const float4 r0 = *reinterpret_cast<const float4*>(sR + k * D + c0);
      const float4 r1 = *reinterpret_cast<const float4*>(sR + k * D + c1);
      const float rs[8] = {r0.x, r0.y, r0.z, r0.w, r1.x, r1.y, r1.z, r1.w};
      float2 r2[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) r2[j] = make_float2(rs[j], rs[j]);
#pragma unroll
      for (int i4 = 0; i4 < kRPT / 4; ++i4) {
        const float4 xv = *reinterpret_cast<const float4*>(sX + k * kXS + rg * kRPT + i4 * 4);
        const float2 xa = make_float2(xv.x, xv.y), xb = make_float2(xv.z, xv.w);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          acc[2 * i4][j] = ffma2(xa, r2[j], acc[2 * i4][j]);
          acc[2 * i4 + 1][j] = ffma2(xb, r2[j], acc[2 * i4 + 1][j]);
        }
      }
    }
    if constexpr (kTeams > 1) {
      if (team == 0 && it == 0 && team1_has_work) mbar_arrive(&start1);
    }
    // the 8 values of row i (columns c0..c0+3, c1..c1+3)
    auto row8 = [&](int i, float (&f)[8]) {
#pragma unroll
      for (int j = 0; j < 8; ++j) f[j] = (i & 1) ? acc[i >> 1][j].y : acc[i >> 1][j].x;
    };

    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < kRPT / 2; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) m = fmaxf(m, fmaxf(fabsf(acc[i][j].x), fabsf(acc[i][j].y)));  // padded rows are +0
    const float amax = block_max<kNT, kTeams>(m, red, tid, team);
    const float scale = __fdiv_rn(amax, qmax);
    const float rcp = __frcp_rn(scale);
    const bool slow = scale < 1.17549435e-38f;
    if (tid == 0) scales[static_cast<int64_t>(bh) * nblk + blk] = scale;

    // Codes by the division-free fast path, one trust check per row of 8
    // values; the rare rows it cannot decide (and blocks with a subnormal
    // scale) are coded afterwards with IEEE divisions.
    // All codes first, with no branch between the rows, then the stores.
    uint2 w[kRPT];
    uint32_t fix = 0;
#pragma unroll
    for (int i = 0; i < kRPT; ++i) {
      float f[8];
      row8(i, f);
      fix |= codes8_fast<kInt8, false, kInt4>(f, rcp, w[i].x, w[i].y) ? 0u : 1u << i;
    }
    if (scale == 0.0f) {                              // all-zero block: zero codes
      fix = 0;
#pragma unroll
      for (int i = 0; i < kRPT; ++i) w[i] = make_uint2(0, 0);
    } else if (slow) {
      fix = (1u << kRPT) - 1;
    }
    // (INT4: byte offsets halved; columns c0.. and c1.. are 2 bytes each)
    constexpr int kDiv = kInt4 ? 2 : 1;
    uint8_t* crow0 = codes + row_offset(layout, H, N, D, b, h, n0 + rg * kRPT) / kDiv;
    const int64_t rstride = (layout == 0 ? D : static_cast<int64_t>(H) * D) / kDiv;   // between token rows
    auto store = [&](int i, uint2 w2) {
      if constexpr (kInt4) {
        *reinterpret_cast<uint16_t*>(crow0 + i * rstride + c0 / 2) = static_cast<uint16_t>(w2.x & 0xFFFFu);
        *reinterpret_cast<uint16_t*>(crow0 + i * rstride + c1 / 2) = static_cast<uint16_t>(w2.x >> 16);
      } else {
        *reinterpret_cast<uint32_t*>(crow0 + i * rstride + c0) = w2.x;
        *reinterpret_cast<uint32_t*>(crow0 + i * rstride + c1) = w2.y;
      }
    };
#pragma unroll
    for (int i = 0; i < kRPT; ++i) {
      if (((fix >> i) & 1u) || rg * kRPT + i >= rows) continue;
      store(i, w[i]);
    }
    if (fix != 0) {
#pragma unroll
      for (int i = 0; i < kRPT; ++i) {
        if (!((fix >> i) & 1u) || rg * kRPT + i >= rows) continue;
        F8 f;
        row8(i, f.v);
        store(i, codes8_exact_f<kInt8, kInt4>(f, scale));
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Without rotation
// ---------------------------------------------------------------------------

// Persistent, one CTA per SM: whole blocks stream through a three-stage
// shared-memory ring by TMA, issued two blocks ahead, so the HBM reads of
// later blocks overlap the coding of the current one. Each of the 512
// threads keeps its kVec 16-byte input vectors of the current block in
// registers between the max and the code pass. The block max is taken on
// the raw 16-bit lanes (|x| of bf16 and fp16 values orders like the bits
// with the sign cleared); codes come from the division-free path, the rare
// vectors it cannot decide from IEEE divisions. Every wait is bounded: a
// timeout is decided for the whole CTA at the next barrier.
constexpr int kQThreads = 512;
constexpr int kQStages = 3;

// Lane-wise max of two pairs of unsigned 16-bit integers.
__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

template <int D, int T>
struct QuantSmem {
  static constexpr int kStage = T * D * 2;             // one block of 16-bit inputs
  static constexpr int kBytes = kQStages * kStage + 128;
};

// kInt4 (with kInt8): INT4 codes, scale absmax / 7, two per byte.
template <int D, int T, bool kInt8, bool kBf16, bool kInt4>
__global__ void __launch_bounds__(kQThreads, 1)
    quant_kernel(const __grid_constant__ CUtensorMap tmX, int layout, int B, int H, int N,
                 uint8_t* __restrict__ codes, float* __restrict__ scales, int* err) {
  constexpr int kCG = D / 8;                           // 16-byte vectors per row
  constexpr int kVec = T * kCG / kQThreads;            // per thread
  static_assert(kVec * kQThreads == T * kCG && kVec <= 32, "vectors per thread");
  using L = QuantSmem<D, T>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  __shared__ __align__(8) uint64_t full[kQStages];
  __shared__ float red[2][kQThreads / 32];
  __shared__ int abort_flag;

  const int tid = threadIdx.x;
  const int nblk = (N + T - 1) / T;
  const int64_t total = static_cast<int64_t>(B) * H * nblk;
  constexpr bool bf = kBf16;
  if (tid == 0) {
    for (int st = 0; st < kQStages; ++st) mbar_init(&full[st], 1);
    abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();
  auto issue = [&](int64_t id, int slot) {
    const int blk_ = static_cast<int>(id % nblk);
    const int bh_ = static_cast<int>(id / nblk);
    mbar_arrive_expect_tx(&full[slot], L::kStage);
    tma_load_4d(smem + slot * L::kStage, &tmX, &full[slot], 0, blk_ * T, bh_ % H, bh_ / H);
  };
  int64_t issued = blockIdx.x;                         // next block to load
  if (tid == 0) {
    tma_prefetch_desc(&tmX);
    for (int st = 0; st < kQStages - 1 && issued < total; ++st, issued += gridDim.x) issue(issued, st);
  }

  int it = 0;
  for (int64_t id = blockIdx.x; id < total; id += gridDim.x, ++it) {
    const int slot = it % kQStages;
    const uint32_t parity = (it / kQStages) & 1;
    // Every thread waits for the copy itself (bounded); the CTA decides on a
    // timeout together at the barrier of the block maximum below.
    const bool ok = mbar_wait(&full[slot], parity, &abort_flag, err);
    const int blk = static_cast<int>(id % nblk);
    const int bh = static_cast<int>(id / nblk);
    const int b = bh / H, h = bh % H;
    const int n0 = blk * T;
    const int rows = min(T, N - n0);                   // rows beyond N were zero-filled

    const uint4* src = reinterpret_cast<const uint4*>(smem + slot * L::kStage);
    uint4 v[kVec];
    uint32_t mb0 = 0, mb1 = 0;
#pragma unroll
    for (int i = 0; i < kVec; ++i) {
      v[i] = ok ? src[tid + i * kQThreads] : make_uint4(0, 0, 0, 0);
      mb0 = max_u16x2(mb0, max_u16x2(v[i].x & 0x7FFF7FFFu, v[i].y & 0x7FFF7FFFu));
      mb1 = max_u16x2(mb1, max_u16x2(v[i].z & 0x7FFF7FFFu, v[i].w & 0x7FFF7FFFu));
    }
    const uint32_t mb = max_u16x2(mb0, mb1);
    const uint32_t m16 = max(mb & 0xFFFFu, mb >> 16);
    float m = bf ? bf16_bits_to_f32(m16) : f16_bits_to_f32(m16);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((tid & 31) == 0) red[it & 1][tid >> 5] = m;
    if (!__syncthreads_and(ok)) break;  // also: every thread is done with the slot of block it - 1
    float amax = 0.0f;
#pragma unroll
    for (int w = 0; w < kQThreads / 32; ++w) amax = fmaxf(amax, red[it & 1][w]);
    if (tid == 0) {
      if (issued < total) issue(issued, (it + kQStages - 1) % kQStages);
      issued += gridDim.x;
    }
    const float scale = __fdiv_rn(amax, kInt4 ? 7.0f : kInt8 ? 127.0f : 448.0f);
    const float rcp = __frcp_rn(scale);
    const bool slow = scale < 1.17549435e-38f;        // zero or subnormal scale: exact path
    if (tid == 0) scales[static_cast<int64_t>(bh) * nblk + blk] = scale;

    // Vector i of this thread: row r0 + i * kRowStep, channels 8c .. 8c + 7
    // (code bytes 8c .. 8c + 7; INT4: bytes 4c .. 4c + 3).
    constexpr int kRowStep = kQThreads / kCG;
    constexpr int kCB = kInt4 ? 4 : 8;                 // code bytes per vector
    const int r0 = tid / kCG, c = tid % kCG;
    const int64_t rstride = (layout == 0 ? D : static_cast<int64_t>(H) * D) / (kInt4 ? 2 : 1);
    uint8_t* out = codes + row_offset(layout, H, N, D, b, h, n0 + r0) / (kInt4 ? 2 : 1) + c * kCB;
    auto store = [&](int i, uint2 w) {
      if constexpr (kInt4) *reinterpret_cast<uint32_t*>(out + i * kRowStep * rstride) = w.x;
      else *reinterpret_cast<uint2*>(out + i * kRowStep * rstride) = w;
    };
    // All codes first, with no branch between the vectors (so their
    // dependent arithmetic interleaves), stored at once; then the vectors
    // holding a value too close to a rounding boundary for the fast path are
    // recomputed (re-read from the stage, which stays until the next
    // barrier), the flagged values taken from the IEEE quotient, and stored
    // again. A zero scale gives zero codes; a subnormal one sends every value
    // to the exact path.
    uint32_t flagged = 0;                                  // vectors with a value to redo
#pragma unroll
    for (int i = 0; i < kVec; ++i) {
      float f[8];
      unpack8(v[i], bf, f);
      uint2 w;
      const bool ok = codes8_fast<kInt8, true, kInt4>(f, rcp, w.x, w.y);
      if (scale == 0.0f) w = make_uint2(0, 0);
      else flagged |= (ok && !slow ? 0u : 1u) << i;
      if (r0 + i * kRowStep < rows) store(i, w);
    }
#pragma unroll 1
    while (flagged != 0) {
      const int i = __ffs(flagged) - 1;
      flagged &= flagged - 1;
      if (r0 + i * kRowStep >= rows) continue;
      float f[8];
      unpack8(src[tid + i * kQThreads], bf, f);
      uint2 w;
      uint32_t fl = codes8_flags<kInt8, kInt4>(f, rcp, w.x, w.y);
      if (slow) fl = 0xFFu;
#pragma unroll 1
      while (fl != 0) {
        const int e = __ffs(fl) - 1;
        fl &= fl - 1;
        float y = f[0];
#pragma unroll
        for (int k = 1; k < 8; ++k) y = e == k ? f[k] : y;
        const uint32_t cd = code_exact<kInt8, kInt4>(y, scale);
        if constexpr (kInt4) {
          w.x = (w.x & ~(0xFu << (4 * e))) | (cd << (4 * e));
        } else {
          const int sh = 8 * (e & 3);
          if (e < 4) w.x = (w.x & ~(0xFFu << sh)) | (cd << sh);
          else w.y = (w.y & ~(0xFFu << sh)) | (cd << sh);
        }
      }
      store(i, w);
    }
  }
  if (abort_flag && tid == 0) {
    // Let the copies already issued land before the CTA exits (bounded).
    for (int k = 0; k < kQStages; ++k) {
      const int i2 = it + k;
      if (blockIdx.x + static_cast<int64_t>(i2) * gridDim.x >= issued) break;
      mbar_wait(&full[i2 % kQStages], (i2 / kQStages) & 1, nullptr, nullptr, 100000000ull);
    }
  }
}

template <int D, int T, bool kInt8, bool kInt4 = false>
cudaError_t launch_rotq(const RotQuantArgs& a, cudaStream_t st, int num_sms, int* err) {
  constexpr int kTeams = RotqTeams<D, T>::value;
  constexpr size_t smem = sizeof(float) * (D * D + kTeams * D * (T + 4));
  auto k = rotq_kernel<D, T, kInt8, kInt4>;
  cudaError_t e = set_max_dyn_smem(reinterpret_cast<const void*>(k), static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int64_t nblocks = static_cast<int64_t>(a.B) * a.H * ((a.N + T - 1) / T);
  const int grid = static_cast<int>(nblocks < num_sms ? nblocks : num_sms);
  k<<<grid, RotqThreads<D, T>::value * kTeams, smem, st>>>(static_cast<const uint16_t*>(a.x), a.is_bf16, a.layout, a.B,
                                                a.H, a.N, a.rot, static_cast<uint8_t*>(a.codes), a.scales, err);
  return cudaGetLastError();
}

// 4-D map {D, N, H, B} over the 16-bit inputs; box {D, T, 1, 1}: one block of
// T token rows of one head, unswizzled (rows beyond N read as zeros).
bool make_map_x(CUtensorMap* m, const void* base, int layout, int B, int H, int N, int D, int T) {
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
  const uint32_t box[4] = {static_cast<uint32_t>(D), static_cast<uint32_t>(T), 1, 1};
  return encode_map_u16(m, 4, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}

template <int D, int T, bool kInt8>
cudaError_t launch_quant(const RotQuantArgs& a, cudaStream_t st, int num_sms, int* err) {
  CUtensorMap tm;
  if (!make_map_x(&tm, a.x, a.layout, a.B, a.H, a.N, D, T)) return cudaErrorInvalidValue;
  using L = QuantSmem<D, T>;
  auto k = a.int4 ? (a.is_bf16 ? quant_kernel<D, T, true, true, true> : quant_kernel<D, T, true, false, true>)
                  : (a.is_bf16 ? quant_kernel<D, T, kInt8, true, false> : quant_kernel<D, T, kInt8, false, false>);
  cudaError_t e = set_max_dyn_smem(reinterpret_cast<const void*>(k), L::kBytes);
  if (e != cudaSuccess) return e;
  const int64_t nblocks = static_cast<int64_t>(a.B) * a.H * ((a.N + T - 1) / T);
  const int grid = static_cast<int>(nblocks < num_sms ? nblocks : num_sms);
  k<<<grid, kQThreads, L::kBytes, st>>>(tm, a.layout, a.B, a.H, a.N, static_cast<uint8_t*>(a.codes), a.scales,
                                         err);
  return cudaGetLastError();
}

template <int D, int T>
cudaError_t dispatch_t(const RotQuantArgs& a, cudaStream_t st, int num_sms, int* err) {
  if (a.rot) {
    if (a.int4) return launch_rotq<D, T, true, true>(a, st, num_sms, err);
    return a.int8 ? launch_rotq<D, T, true>(a, st, num_sms, err) : launch_rotq<D, T, false>(a, st, num_sms, err);
  }
  return a.int8 ? launch_quant<D, T, true>(a, st, num_sms, err) : launch_quant<D, T, false>(a, st, num_sms, err);
}

}  // namespace

// Block sizes compiled: 128 and 256 tokens (the method's Q and K/V blocks);
// D in {64, 128}.
cudaError_t launch_rotate_block_quant(const RotQuantArgs& a, cudaStream_t st, int num_sms, int* err) {
  if (a.D == 128) {
    if (a.T == 128) return dispatch_t<128, 128>(a, st, num_sms, err);
    if (a.T == 256) return dispatch_t<128, 256>(a, st, num_sms, err);
  } else if (a.D == 64) {
    if (a.T == 128) return dispatch_t<64, 128>(a, st, num_sms, err);
    if (a.T == 256) return dispatch_t<64, 256>(a, st, num_sms, err);
  }
  return cudaErrorInvalidValue;
}

bool rotate_block_quant_supported(int D, int T) {
  return (D == 64 || D == 128) && (T == 128 || T == 256);
}

}  // namespace qattn
