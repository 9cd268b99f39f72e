// kv_append.cu -- quantize new K or V rows into the decode cache.
//
// Method: "INT8 量化算子", ops-transformer item 3 (KV Cache 也量化): in the
// decode phase new K/V rows are written into the cache as INT8 codes; packed
// INT4 with one fp16 scale per group of channels: "ops-transformer INT8/INT4
// 量化推理", 5.1 (group scales) and 5.2 (two codes per byte, element 2i in
// the low nibble).
//
// INT8 cache, one float32 scale per 256-token block of each (b, h_kv): the
// block scale stays absmax / 127 of every token written to the block so far.
//   kv_append_int8_kernel: one CTA per (touched block, h_kv, b).
//     a = max |x| over the block's new tokens; s = max(s_old, a / 127);
//     if s grew and the block already held tokens, each of their codes c is
//     replaced by RNE(f32(c * s_old) / s); new codes RNE(x / s); float32,
//     each code as the IEEE quotient decides it (code_fast), clamped to
//     [-127, 127].
// Packed INT4 cache, one fp16 scale per token per group:
//   kv_append_int4_kernel: eight lanes per new token of one (b, h_kv), 16
//     channels each; s16 = fp16(absmax_group / 7) (the quotient IEEE-
//     rounded to float32 first), codes RNE(x / s16) clamped to [-7, 7] (the
//     product with 1/s16 unless it is within 1e-4 of a half-integer),
//     packed two per byte.
// Both are small, memory-bound kernels (the new rows are read once, the
// codes written once; a growing INT8 block also rewrites its earlier codes).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "qattn_device.cuh"
#include "qattn_internal.h"

namespace qattn {

namespace {

constexpr int kAppendThreads = 256;

__device__ __forceinline__ int rne_clamp(float v, int lim) {
  return max(-lim, min(lim, __float2int_rn(v)));
}

// RNE(y / s) as the IEEE quotient decides it, mostly without dividing: the
// product y * RN(1/s) is within 1.5 ulp of the rounded quotient, so its
// integer rounding agrees unless it lies within 1e-4 of a half-integer (for
// |y/s| <= 128); those, and scales below the smallest normal float32
// (`slow`), use the IEEE division.
__device__ __forceinline__ int code_fast(float y, float s, float rcp, bool slow, int lim) {
  float v = y * rcp;
  const float r = (v + 12582912.0f) - 12582912.0f;
  if (slow || fabsf(v - r) > 0.4999f) v = __fdiv_rn(y, s);
  return rne_clamp(v, lim);
}

// INT8 codes of the 8 bf16 values of v (two's complement bytes, value e in
// byte e): the magic-number rounding of y * rcp in f32x2 pairs, the integer
// landing in the low mantissa byte (|y / s| <= 127 here), with d = y * rcp -
// RNE(y * rcp) from the exact product; when any |d| comes within 1e-4 of
// 0.5, or the scale is below the smallest normal float32, all 8 are decided
// by code_fast (the IEEE quotient where the product cannot decide).
__device__ __forceinline__ uint2 codes8_i8(uint4 v, float s, float rcp, bool slow) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float f[8];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    f[2 * k] = __uint_as_float(w[k] << 16);
    f[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
  }
  const float2 rc = make_float2(rcp, rcp);
  const float2 mg = make_float2(12582912.0f, 12582912.0f);
  uint32_t t[8];
  float dmax = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 y = make_float2(f[2 * i], f[2 * i + 1]);
    const float2 m = ffma2(y, rc, mg);                                        // RNE(y * rcp) in the low bits
    const float2 d = ffma2(y, rc, ffma2(m, make_float2(-1.0f, -1.0f), mg));   // y * rcp - that integer
    dmax = fmaxf(dmax, fmaxf(fabsf(d.x), fabsf(d.y)));
    t[2 * i] = __float_as_uint(m.x);
    t[2 * i + 1] = __float_as_uint(m.y);
  }
  if (slow || dmax > 0.4999f) {                                               // rare: value by value
#pragma unroll
    for (int e = 0; e < 8; ++e) t[e] = static_cast<uint32_t>(code_fast(f[e], s, rcp, slow, 127));
  }
  return make_uint2(__byte_perm(__byte_perm(t[0], t[1], 0x0040), __byte_perm(t[2], t[3], 0x0040), 0x5410),
                    __byte_perm(__byte_perm(t[4], t[5], 0x0040), __byte_perm(t[6], t[7], 0x0040), 0x5410));
}

// x: bf16 [B, H_kv, n, D]; cache int8 [B, H_kv, L_max, D]; scales float32
// [B, H_kv, nblk]. D is a multiple of 8 (16-byte vectors of x, 8-byte code
// stores).
__global__ void __launch_bounds__(kAppendThreads)
    kv_append_int8_kernel(const uint16_t* __restrict__ x, int Hkv, int n, int D, int L, int Lmax, int kv_block,
                          int8_t* __restrict__ cache, float* __restrict__ scales) {
  __shared__ float red[kAppendThreads / 32];
  const int blk = L / kv_block + static_cast<int>(blockIdx.x);
  const int h = blockIdx.y, b = blockIdx.z;
  const int64_t head = static_cast<int64_t>(b) * Hkv + h;
  const int nblk = (Lmax + kv_block - 1) / kv_block;
  const int b0 = blk * kv_block;
  const int t0 = max(L, b0), t1 = min(L + n, b0 + kv_block);
  if (t0 >= t1) return;                                 // (uniform per CTA)
  const int vecs = D / 8;
  const int64_t total = static_cast<int64_t>(t1 - t0) * vecs;
  const uint16_t* xb = x + (head * n + (t0 - L)) * D;

  // Four vectors per thread in flight at a time; |x| of bf16 values orders
  // like the bits with the sign cleared.
  uint32_t mb = 0;
  for (int64_t i0 = threadIdx.x; i0 < total; i0 += 4 * kAppendThreads) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t i = i0 + u * kAppendThreads;
      v[u] = i < total ? *reinterpret_cast<const uint4*>(xb + i * 8) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      mb = __vmaxu2(mb, __vmaxu2(v[u].x & 0x7FFF7FFFu, v[u].y & 0x7FFF7FFFu));
      mb = __vmaxu2(mb, __vmaxu2(v[u].z & 0x7FFF7FFFu, v[u].w & 0x7FFF7FFFu));
    }
  }
  float m = bf16_bits_to_f32(max(mb & 0xFFFFu, mb >> 16));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < kAppendThreads / 32; ++i) a = fmaxf(a, red[i]);

  const float s_old = t0 > b0 ? scales[head * nblk + blk] : 0.0f;
  const float s1 = __fdiv_rn(a, 127.0f);
  const float s = s1 > s_old ? s1 : s_old;
  const float rcp = __frcp_rn(s);
  const bool slow = s < 1.17549435e-38f;

  // earlier tokens of a block whose scale grew
  if (s > s_old && t0 > b0) {
    int8_t* cb = cache + (head * Lmax + b0) * D;
    const int64_t old_total = static_cast<int64_t>(t0 - b0) * vecs;
    for (int64_t i = threadIdx.x; i < old_total; i += kAppendThreads) {
      const uint2 c = *reinterpret_cast<const uint2*>(cb + i * 8);
      const uint32_t w[2] = {c.x, c.y};
      uint32_t o[2] = {0, 0};
#pragma unroll
      for (int k = 0; k < 2; ++k)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float y = __fmul_rn(static_cast<float>(static_cast<int8_t>((w[k] >> (8 * e)) & 0xFFu)), s_old);
          o[k] |= (static_cast<uint32_t>(code_fast(y, s, rcp, slow, 127)) & 0xFFu) << (8 * e);
        }
      *reinterpret_cast<uint2*>(cb + i * 8) = make_uint2(o[0], o[1]);
    }
  }
  // new tokens (four vectors in flight at a time)
  int8_t* cn = cache + (head * Lmax + t0) * D;
  for (int64_t i0 = threadIdx.x; i0 < total; i0 += 4 * kAppendThreads) {
    uint4 vv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t i = i0 + u * kAppendThreads;
      vv[u] = i < total ? *reinterpret_cast<const uint4*>(xb + i * 8) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t i = i0 + u * kAppendThreads;
      if (i >= total) break;
      const uint2 o = s != 0.0f ? codes8_i8(vv[u], s, rcp, slow) : make_uint2(0, 0);
      *reinterpret_cast<uint2*>(cn + i * 8) = o;
    }
  }
  if (threadIdx.x == 0) scales[head * nblk + blk] = s;
}

// x: bf16 [B, H_kv, n, D], D = 128; cache bytes [B, H_kv, L_max, D/2]; scales
// fp16 [B, H_kv, L_max, D/group], group 128 or 64. Eight lanes per row (lane
// q of the row's octet owns channels 16q .. 16q + 15: two 16-byte loads, one
// 8-byte store), so one warp instruction serves four rows and the per-row
// work (group maximum, scale, reciprocal) is shared by them.
constexpr int kInt4RowsPerCta = 64;                 // 32 rows per pass of 256 threads, two passes

__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// Codes RNE(y / s) of 16 values, packed two per byte (element 2i in the low
// nibble of byte i) into 8 bytes: the product with rcp (1/s within 2^-22)
// rounded by the 1.5 * 2^23 addend. That decides the code unless the product
// lies within 1e-4 of a half-integer; `redo` is then set (it may already be
// set when a product can exceed 7.5, see the caller) and the caller
// completes the codes with int4_codes16_exact.
__device__ __forceinline__ uint2 int4_codes16(const float (&f)[16], float rcp, bool& redo) {
  const float2 rc = make_float2(rcp, rcp);
  const float2 mg = make_float2(12582912.0f, 12582912.0f);
  uint32_t b[8];                                  // byte i: codes 2i (low nibble) and 2i + 1
  float dmax = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float2 y = make_float2(f[2 * i], f[2 * i + 1]);
    const float2 m = ffma2(y, rc, mg);                               // RNE(y * rcp) in the low bits
    const float2 d = ffma2(y, rc, ffma2(m, make_float2(-1.0f, -1.0f), mg));   // y * rcp - that integer
    dmax = fmaxf(dmax, fmaxf(fabsf(d.x), fabsf(d.y)));
    b[i] = (__float_as_uint(m.x) & 0xFu) | ((__float_as_uint(m.y) & 0xFu) << 4);
  }
  redo = redo || dmax > 0.4999f;
  return make_uint2(__byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410),
                    __byte_perm(__byte_perm(b[4], b[5], 0x0040), __byte_perm(b[6], b[7], 0x0040), 0x5410));
}

// Completes the codes of int4_codes16 where it could not decide them all
// (the values come as their bf16 bits, two per word, element 2k in the low
// half): each value's product is formed and checked again, and only the
// values within 1e-4 of a half-integer (every value when `wide`) take the
// IEEE quotient, clamped to [-7, 7], one division per such value; with bf16
// inputs that is about one value in a thousand. Out of line, so that the
// common path carries none of this.
__device__ __noinline__ uint2 int4_codes16_exact(uint4 lo, uint4 hi, float s, float rcp, bool wide, uint2 codes) {
  const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
  const float mg = 12582912.0f;
  uint32_t redo = 0;                                  // bit e: value e takes the quotient
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const float y = __uint_as_float((e & 1) ? (w[e >> 1] & 0xFFFF0000u) : (w[e >> 1] << 16));
    const float m = __fmaf_rn(y, rcp, mg);                           // as in int4_codes16
    const float d = __fmaf_rn(y, rcp, mg - m);
    if (wide || fabsf(d) > 0.4999f) redo |= 1u << e;
  }
#pragma unroll 1
  while (redo != 0) {
    const int e = __ffs(static_cast<int>(redo)) - 1;
    redo &= redo - 1;
    const int k = e >> 1;
    const uint4 v = k < 4 ? lo : hi;
    const uint32_t wd = (k & 3) == 0 ? v.x : (k & 3) == 1 ? v.y : (k & 3) == 2 ? v.z : v.w;
    const float y = __uint_as_float((e & 1) ? (wd & 0xFFFF0000u) : (wd << 16));
    const uint32_t c = static_cast<uint32_t>(max(-7, min(7, __float2int_rn(__fdiv_rn(y, s))))) & 0xFu;
    const int sh = 4 * (e & 7);
    if (e < 8) codes.x = (codes.x & ~(0xFu << sh)) | (c << sh);
    else codes.y = (codes.y & ~(0xFu << sh)) | (c << sh);
  }
  return codes;
}

// RN(m / 7) for the rare group maxima whose fp16 rounding the product with
// RN(1/7) cannot decide; out of line for the same reason.
__device__ __noinline__ float div7_exact(float m) { return __fdiv_rn(m, 7.0f); }

// Grid (ceil(n / kInt4RowsPerCta), B * H_kv): blockIdx.y is the (b, h_kv) head.
__global__ void __launch_bounds__(kAppendThreads)
    kv_append_int4_kernel(const uint16_t* __restrict__ x, int n, int L, int Lmax, int group,
                          uint8_t* __restrict__ cache, uint16_t* __restrict__ scales) {
  constexpr int D = 128;
  constexpr int kPasses = kInt4RowsPerCta / (kAppendThreads / 8);
  const int q = threadIdx.x & 7;                      // lane within the row's octet
  const int64_t head = blockIdx.y;
  const uint16_t* xh = x + head * n * D;
  const int ng = D / group;
  const int width = group / 16;                       // lanes per group: 8 (group 128) or 4 (64)
  // both passes' rows are loaded first (four 16-byte loads in flight)
  uint4 raw[kPasses][2];
  int row[kPasses];
#pragma unroll
  for (int ps = 0; ps < kPasses; ++ps) {
    row[ps] = static_cast<int>(blockIdx.x) * kInt4RowsPerCta + ps * (kAppendThreads / 8) + (threadIdx.x >> 3);
    const bool in = row[ps] < n;
    const uint4* src = reinterpret_cast<const uint4*>(xh + static_cast<int64_t>(row[ps]) * D + q * 16);
    raw[ps][0] = in ? __ldcs(src) : make_uint4(0, 0, 0, 0);
    raw[ps][1] = in ? __ldcs(src + 1) : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int ps = 0; ps < kPasses; ++ps) {
    const uint32_t w[8] = {raw[ps][0].x, raw[ps][0].y, raw[ps][0].z, raw[ps][0].w,
                           raw[ps][1].x, raw[ps][1].y, raw[ps][1].z, raw[ps][1].w};
    float f[16];
    uint32_t mb = 0;                                  // max |x| on the bf16 bits (sign cleared)
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      f[2 * k] = bf16_bits_to_f32(w[k] & 0xFFFFu);
      f[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
      mb = __vmaxu2(mb, w[k] & 0x7FFF7FFFu);
    }
    float m = bf16_bits_to_f32(max(mb & 0xFFFFu, mb >> 16));
    // maximum over the lanes of this lane's group (within the octet)
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) {
      const float other = __shfl_xor_sync(0xffffffffu, m, o);
      if (o < width) m = fmaxf(m, other);
    }
    // s16 = fp16(m / 7), the quotient IEEE-rounded to float32 first. m *
    // RN(1/7) is within 1.75 float32 units of that quotient, so its fp16
    // rounding is the same unless it lies within 3 units of an fp16 rounding
    // midpoint (float32 mantissa bits 12..0 = 0x1000) or in the fp16
    // subnormal range; those take the IEEE division.
    float q7 = m * 0.142857149f;
    if (q7 < 6.103515625e-05f || abs(static_cast<int>(__float_as_uint(q7) & 0x1FFFu) - 0x1000) <= 3)
      q7 = div7_exact(m);
    const __half s16 = __float2half_rn(q7);
    const float s = __half2float(s16);
    uint2 codes = make_uint2(0, 0);
    if (s != 0.0f) {                                  // (fp16 scales are never subnormal in float32)
      // the approximate reciprocal (relative error below 2^-22) keeps every
      // product within 2e-6 of the quotient (|y / s| <= 7.5), far inside the
      // codes' 1e-4 margin; `wide` is decided with room for it
      const float rcp = rcp_approx(s);
      const bool wide = m * rcp >= 7.4999f;
      bool redo = wide;
      codes = int4_codes16(f, rcp, redo);
      if (redo) codes = int4_codes16_exact(raw[ps][0], raw[ps][1], s, rcp, wide, codes);
    }
    if (row[ps] < n) {
      const int t = L + row[ps];
      *reinterpret_cast<uint2*>(cache + (head * Lmax + t) * (D / 2) + q * 8) = codes;
      if ((q % width) == 0) scales[(head * Lmax + t) * ng + q / width] = __half_as_ushort(s16);
    }
  }
}

}  // namespace

bool kv_append_supported(int D, bool int4, int kv_block, int group) {
  if (int4) return D == 128 && (group == 128 || group == 64);
  return D % 8 == 0 && D <= 1024 && kv_block == 256;
}

cudaError_t launch_kv_append(const KvAppendArgs& a, cudaStream_t st) {
  if (!a.int4) {
    const int first = a.L / a.kv_block, last = (a.L + a.n - 1) / a.kv_block;
    dim3 grid(static_cast<unsigned>(last - first + 1), a.Hkv, a.B);
    kv_append_int8_kernel<<<grid, kAppendThreads, 0, st>>>(static_cast<const uint16_t*>(a.x), a.Hkv, a.n, a.D, a.L,
                                                            a.Lmax, a.kv_block, static_cast<int8_t*>(a.cache),
                                                            static_cast<float*>(a.scales));
  } else {
    const dim3 grid(static_cast<unsigned>((a.n + kInt4RowsPerCta - 1) / kInt4RowsPerCta),
                    static_cast<unsigned>(a.B * a.Hkv));
    kv_append_int4_kernel<<<grid, kAppendThreads, 0, st>>>(static_cast<const uint16_t*>(a.x), a.n, a.L, a.Lmax,
                                                           a.group, static_cast<uint8_t*>(a.cache),
                                                           static_cast<uint16_t*>(a.scales));
  }
  return cudaGetLastError();
}

}  // namespace qattn
