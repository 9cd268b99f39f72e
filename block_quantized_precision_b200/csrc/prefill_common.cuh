// prefill_common.cuh -- pieces of the prefill kernel (prefill.cu) kept
// apart from its control flow: tile sizes, the kernel parameters,
// arithmetic helpers (exponentials, exact INT32 -> float32), the chunked
// tensor-memory reader and the TMA maps.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math_constants.h>

#include "qattn_device.cuh"
#include "qattn_internal.h"

namespace qattn {

namespace {

constexpr int kTileM = 128;     // query rows per tile
constexpr int kTileN = 128;     // keys per tile
constexpr int kStagesKV = 3;
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxBlk = 512;    // K/V block scales staged in shared memory (keys up to 131072)
constexpr float kLog2_127 = 6.988684686772166f;
struct PrefillParams {
  const float* qs;
  const float* ks;
  const float* vs;
  __nv_bfloat16* out;
  float* lse;
  int B, H, Nq, Nkv;
  int nqt, npairs, nqb, nkb;
  int causal;
  int layout;
  float scale_log2;
  int* err;
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

// 2^x for a pair on the FMA pipe, to take part of the exponentials off the
// MUFU unit: x = n + f with n = RN(x) (the 1.5 * 2^23 rounding addend) and
// f in [-1/2, 1/2]; 2^f by a degree-5 polynomial (Remez fit of the minimax
// relative error on [-1/2, 1/2], exp2_poly_fit.py: 7.5e-8 levelled, 2.1e-7
// in float32 Horner/FMA arithmetic, like ex2.approx); 2^n added to the
// exponent field. x is
// clamped at -120 (2^-120 rounds to a zero code in every 8-bit format used
// here) and is at most log2(127) on this path.
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  x.x = fmaxf(x.x, -120.0f);
  x.y = fmaxf(x.y, -120.0f);
  const float2 r = fadd2(x, make_float2(12582912.0f, 12582912.0f));
  const float2 n = fadd2(r, make_float2(-12582912.0f, -12582912.0f));
  const float2 f = ffma2(n, make_float2(-1.0f, -1.0f), x);
  float2 q = ffma2(make_float2(1.32764725e-3f, 1.32764725e-3f), f, make_float2(9.67554096e-3f, 9.67554096e-3f));
  q = ffma2(q, f, make_float2(5.55071309e-2f, 5.55071309e-2f));
  q = ffma2(q, f, make_float2(2.40221202e-1f, 2.40221202e-1f));
  q = ffma2(q, f, make_float2(6.93146944e-1f, 6.93146944e-1f));
  q = ffma2(q, f, make_float2(1.00000012f, 1.00000012f));
  return make_float2(__int_as_float(__float_as_int(q.x) + (__float_as_int(r.x) << 23)),
                     __int_as_float(__float_as_int(q.y) + (__float_as_int(r.y) << 23)));
}

// Exact INT32 -> float32 of two accumulator words (|S| < 2^22): the bits of
// 1.5 * 2^23 + S are formed by an integer add, then 1.5 * 2^23 is removed.
__device__ __forceinline__ float2 s32x2_to_f32x2(uint32_t a, uint32_t b) {
  return fadd2(make_float2(__int_as_float(static_cast<int>(a) + 0x4B400000),
                           __int_as_float(static_cast<int>(b) + 0x4B400000)),
               make_float2(-12582912.0f, -12582912.0f));
}

template <int N>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

template <int N>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

// Element offset of token n of head (b, h), channel 0.
__device__ __forceinline__ int64_t row_offset(int layout, int H, int N, int D, int b, int h, int n) {
  return layout == 0 ? ((static_cast<int64_t>(b) * H + h) * N + n) * D
                     : ((static_cast<int64_t>(b) * N + n) * H + h) * D;
}

// Calls body(c, v) for the W-column chunks c = 0..N-1 of this thread's TMEM
// lane starting at taddr (W = 16 or 32); chunk c + 1 is loaded while chunk c
// is processed.
template <int W>
__device__ __forceinline__ void tmem_ld_w(uint32_t taddr, uint32_t (&r)[W]) {
  if constexpr (W == 16) tmem_ld16(taddr, r);
  else tmem_ld32(taddr, r);
}

template <int N, int W, typename F>
__device__ __forceinline__ void tmem_chunks(uint32_t taddr, F&& body) {
  uint32_t a[W], b[W];
  tmem_ld_w<W>(taddr, a);
  tmem_wait_ld();
  reg_fence(a);
#pragma unroll
  for (int c = 0; c < N; ++c) {
    uint32_t(&cur)[W] = (c & 1) ? b : a;
    uint32_t(&nxt)[W] = (c & 1) ? a : b;
    if (c + 1 < N) tmem_ld_w<W>(taddr + (c + 1) * W, nxt);
    body(c, cur);
    if (c + 1 < N) {
      tmem_wait_ld();
      reg_fence(nxt);
    }
  }
}

// 4-D map {D, N, H, B} over 8-bit codes; box {D, 128, 1, 1}: one tile of 128
// token rows of one head lands as 128 rows of D bytes (swizzled).
bool make_map(CUtensorMap* m, const void* base, int layout, int B, int H, int N, int D) {
  const uint64_t dims[4] = {static_cast<uint64_t>(D), static_cast<uint64_t>(N), static_cast<uint64_t>(H),
                            static_cast<uint64_t>(B)};
  uint64_t strides[3];
  if (layout == 0) {
    strides[0] = static_cast<uint64_t>(D);
    strides[1] = static_cast<uint64_t>(N) * D;
    strides[2] = static_cast<uint64_t>(H) * N * D;
  } else {
    strides[0] = static_cast<uint64_t>(H) * D;
    strides[1] = static_cast<uint64_t>(D);
    strides[2] = static_cast<uint64_t>(N) * H * D;
  }
  const uint32_t box[4] = {static_cast<uint32_t>(D), static_cast<uint32_t>(kTileM), 1, 1};
  return encode_map_u8(m, 4, base, dims, strides, box,
                       D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B);
}

// Packed INT4 V: {D/2, N, H, B} bytes, box {D/2, 128, 1, 1}, unswizzled (the
// widening warp reads it linearly).
bool make_map_v4(CUtensorMap* m, const void* base, int layout, int B, int H, int N, int D) {
  const uint64_t Db = static_cast<uint64_t>(D / 2);
  const uint64_t dims[4] = {Db, static_cast<uint64_t>(N), static_cast<uint64_t>(H), static_cast<uint64_t>(B)};
  uint64_t strides[3];
  if (layout == 0) {
    strides[0] = Db;
    strides[1] = static_cast<uint64_t>(N) * Db;
    strides[2] = static_cast<uint64_t>(H) * N * Db;
  } else {
    strides[0] = static_cast<uint64_t>(H) * Db;
    strides[1] = Db;
    strides[2] = static_cast<uint64_t>(N) * H * Db;
  }
  const uint32_t box[4] = {static_cast<uint32_t>(Db), static_cast<uint32_t>(kTileN), 1, 1};
  return encode_map_u8(m, 4, base, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_NONE);
}

}  // namespace

}  // namespace qattn
