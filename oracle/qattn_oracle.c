/*
 * qattn_oracle.c -- plain, slow CPU oracle for block-quantized attention.
 *
 * TEST INFRASTRUCTURE ONLY. Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this file's library. It shares no
 * code, header, table or constant with the CUDA library.
 *
 * What it computes, and where each step is stated:
 *
 *  - Rotation of Q and K by an orthogonal matrix before quantization:
 *    "MindIE-SD quantization" page, section "FA量化 / 技术特点 / 旋转(Rotate)".
 *  - Dynamic block quantization to float8_e4m3fn with one scale per block,
 *    Q blocks of 128 tokens and K/V blocks of 256 tokens:
 *    same page, "块量化(Block Quant)".
 *  - Symmetric absmax INT8 quantization, value = round(x / scale),
 *    scale = max|x| / 127, zero point 0:
 *    "INT8 量化算子" page, section "1. 对称量化 vs 非对称量化".
 *  - INT8 x INT8 -> INT32 products with the conversion only at the output:
 *    same page, "ops-transformer 里的 INT8 量化算子优化", items 1 and 3.
 *  - Block-tiled attention with a running softmax (outer loop over query
 *    blocks, inner loop over key/value blocks): "FlashAttention 的 INT8/INT4
 *    量化" page, section "三层实现详解 / 第一层". The page's normalisation is
 *    wrong (the accumulator is never rescaled and it divides by a sum of
 *    logs); this file uses the standard running-max softmax instead.
 *  - INT4 codes, two per byte, element 2i in the low nibble and 2i+1 in the
 *    high nibble; one fp16 scale per group of 128 elements:
 *    "ops-transformer INT8/INT4 量化推理" page, sections 5.1 and 5.2.
 *  - float8_e4m3fn: OCP 8-bit floating point specification (E4M3: bias 7,
 *    no infinities, one NaN pattern per sign, largest finite 448).
 *  - INT4 block codes for attention inputs (round(x / scale) clamped to the
 *    INT4 range, scale per group) and INT4 widened to INT8 for the matmul:
 *    "FlashAttention 的 INT8/INT4 量化" page, 第二层 (INT4); Q/K in INT8 with
 *    V in INT4: same page, 第三层 (混合精度). Here the INT4 scale is dynamic
 *    per block of tokens like the INT8/e4m3 ones (absmax / 7, codes in
 *    [-7, 7], packed as above).
 *
 * Precision: every step whose result decides an integer code (rotation,
 * block absmax, scale, code rounding, the probabilities that are rounded to
 * 8-bit codes) is carried out in IEEE float32, one rounding per operation, in
 * the order written here; everything else (dot products of codes, the
 * softmax sums, the output accumulation) is exact or float64.
 *
 * Built with: gcc -O2 -ffp-contract=off -fno-fast-math -shared -fPIC.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_BNSD 0
#define ORC_BSND 1

#define ORC_F16 0
#define ORC_BF16 1
#define ORC_INT8 2
#define ORC_FP8_E4M3 3
#define ORC_INT4_PACKED 4
#define ORC_F32 100 /* oracle-only: float32 "codes" (no quantization), for pins */

/* ------------------------------------------------------------------------ */
/* Scalar codecs                                                            */
/* ------------------------------------------------------------------------ */

float orc_bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

float orc_f16_to_f32(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1F;
  int m = h & 0x3FF;
  double v;
  if (e == 0)
    v = ldexp((double)m, -24);               /* subnormal: m * 2^-24 */
  else if (e == 31)
    v = m ? NAN : INFINITY;
  else
    v = ldexp(1.0 + m / 1024.0, e - 15);
  return (float)(sign ? -v : v);             /* exact: fits in float32 */
}

/* float64 -> bfloat16, round to nearest even, straight from the float64
 * value (no intermediate float32 rounding). Values below the smallest
 * normal bfloat16 go through float32 first (they never occur in outputs of
 * interest). */
uint16_t orc_f64_to_bf16(double x) {
  if (isnan(x)) return 0x7FC0;
  double a = fabs(x);
  if (a < ldexp(1.0, -126)) {
    float f = (float)x;
    uint32_t u;
    memcpy(&u, &f, 4);
    u = u + 0x7FFF + ((u >> 16) & 1);
    return (uint16_t)(u >> 16);
  }
  uint64_t u;
  memcpy(&u, &x, 8);
  uint64_t lsb = (u >> 45) & 1;              /* bf16 keeps 7 of 52 mantissa bits */
  u = u + ((1ull << 44) - 1) + lsb;          /* round half to even at bit 45 */
  uint64_t sign = u >> 63;
  int64_t e = (int64_t)((u >> 52) & 0x7FF) - 1023;   /* after rounding */
  uint64_t mant7 = (u >> 45) & 0x7F;
  if (e > 127) return (uint16_t)((sign << 15) | 0x7F80); /* overflow -> inf */
  return (uint16_t)((sign << 15) | ((uint64_t)(e + 127) << 7) | mant7);
}

uint16_t orc_f32_to_bf16(float x) { return orc_f64_to_bf16((double)x); }

/* float32 -> e4m3fn, round to nearest even, saturating to +-448 (the value
 * nearest to the input among the finite codes when the input is beyond the
 * range, as the SATFINITE conversion does). NaN -> 0x7F with the sign. */
uint8_t orc_e4m3_from_f32(float x) {
  uint32_t bits;
  memcpy(&bits, &x, 4);
  uint8_t sign = (uint8_t)((bits >> 31) << 7);
  if (isnan(x)) return sign | 0x7F;
  double a = fabs((double)x);
  if (a >= 448.0) return sign | 0x7E;        /* 448 = 1.75 * 2^8, largest finite */
  int e;
  frexp(a, &e);                              /* a = f * 2^e, f in [0.5, 1) */
  int E = e - 1;                             /* floor(log2 a) for a > 0 */
  if (a == 0.0 || E < -6) E = -6;            /* subnormal range shares 2^-9 steps */
  double quantum = ldexp(1.0, E - 3);        /* 3 explicit mantissa bits */
  double q = nearbyint(a / quantum);         /* exact quotient; ties to even */
  double v = q * quantum;                    /* nearest representable value */
  if (v == 0.0) return sign;
  if (v < ldexp(1.0, -6)) {                  /* subnormal: v = m * 2^-9 */
    int m = (int)(v / ldexp(1.0, -9));
    return sign | (uint8_t)m;
  }
  frexp(v, &e);
  E = e - 1;
  int m = (int)((v / ldexp(1.0, E) - 1.0) * 8.0);
  return sign | (uint8_t)(((E + 7) << 3) | m);
}

float orc_e4m3_to_f32(uint8_t c) {
  int sign = c >> 7;
  int e = (c >> 3) & 0xF;
  int m = c & 7;
  double v;
  if (e == 15 && m == 7)
    v = NAN;
  else if (e == 0)
    v = m * ldexp(1.0, -9);
  else
    v = (1.0 + m / 8.0) * ldexp(1.0, e - 7);
  return (float)(sign ? -v : v);
}

void orc_e4m3_encode_n(const float* x, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_from_f32(x[i]);
}

void orc_e4m3_decode_n(const uint8_t* c, int64_t n, float* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_to_f32(c[i]);
}

/* INT4: two's-complement 4-bit codes; element 2i in bits 0..3, 2i+1 in bits
 * 4..7 ("ops-transformer INT8/INT4 量化推理", 5.2 INT4 打包格式). */
uint8_t orc_int4_pack(int w0, int w1) {
  return (uint8_t)((((unsigned)w1 & 0xF) << 4) | ((unsigned)w0 & 0xF));
}

int orc_int4_lo(uint8_t b) { int v = b & 0xF; return v >= 8 ? v - 16 : v; }
int orc_int4_hi(uint8_t b) { int v = (b >> 4) & 0xF; return v >= 8 ? v - 16 : v; }

/* ------------------------------------------------------------------------ */
/* Layout helpers                                                           */
/* ------------------------------------------------------------------------ */

/* Element offset of (b, h, n, 0) for a [B,H,N,D] (BNSD) or [B,N,H,D] (BSND)
 * tensor. */
static int64_t row_off(int layout, int B, int H, int N, int D, int b, int h, int n) {
  (void)B;
  if (layout == ORC_BNSD) return (((int64_t)b * H + h) * N + n) * D;
  return (((int64_t)b * N + n) * H + h) * D;
}

static float in_to_f32(const uint16_t* x, int dtype, int64_t i) {
  return dtype == ORC_BF16 ? orc_bf16_to_f32(x[i]) : orc_f16_to_f32(x[i]);
}

/* ------------------------------------------------------------------------ */
/* Rotation + dynamic block quantization                                    */
/* ------------------------------------------------------------------------ */

/*
 * Rotation of one row: y[j] = sum_k x[k] R[k][j] (R row-major D x D), as a
 * chain of float32 fused multiply-adds in ascending k starting from +0, one
 * rounding per step. R == NULL: y = x.
 */
void orc_rotate_row(const float* x, const float* R, int D, float* y) {
  for (int j = 0; j < D; ++j) {
    if (!R) { y[j] = x[j]; continue; }
    float acc = 0.0f;
    for (int k = 0; k < D; ++k) acc = fmaf(x[k], R[(int64_t)k * D + j], acc);
    y[j] = acc;
  }
}

/*
 * One block of one (b, h): rows n in [blk*T, min(N, (blk+1)*T)).
 *   y = x R           (y[j] = sum_k x[k] R[k][j], float32 fused multiply-adds
 *                      in ascending k starting from +0; R == NULL: y = x)
 *   amax = max |y|    over the block's valid rows and all D columns
 *   s = amax / qmax   (one float32 division; qmax 127 for INT8, 448 for e4m3)
 *   code = RNE(y / s) (float32 division, then round half to even; INT8
 *                      clamped to [-127, 127]; e4m3 saturating); s == 0 gives
 *                      all-zero codes.
 * Writes the block's codes into `codes` (same layout as x, 1 byte per
 * element) and scales[(b*H + h)*nblk + blk].
 */
int orc_quant_block(const uint16_t* x, int x_dtype, int layout, int B, int H, int N, int D,
                    const float* R, int T, int code_dtype, int b, int h, int blk,
                    uint8_t* codes, float* scales) {
  if (T <= 0 || D <= 0 || D > 1024) return 1;
  int n0 = blk * T, n1 = n0 + T < N ? n0 + T : N;
  int rows = n1 - n0;
  if (rows <= 0) return 1;
  float* y = (float*)malloc(sizeof(float) * (size_t)rows * D);
  float* xr = (float*)malloc(sizeof(float) * (size_t)D);
  if (!y || !xr) { free(y); free(xr); return 2; }
  float amax = 0.0f;
  for (int r = 0; r < rows; ++r) {
    int64_t off = row_off(layout, B, H, N, D, b, h, n0 + r);
    for (int k = 0; k < D; ++k) xr[k] = in_to_f32(x, x_dtype, off + k);   /* exact */
    orc_rotate_row(xr, R, D, y + (int64_t)r * D);
    for (int j = 0; j < D; ++j) {
      float a = fabsf(y[(int64_t)r * D + j]);
      if (a > amax) amax = a;
    }
  }
  float qmax = code_dtype == ORC_INT8 ? 127.0f : code_dtype == ORC_INT4_PACKED ? 7.0f : 448.0f;
  float s = amax / qmax;
  int nblk = (N + T - 1) / T;
  scales[((int64_t)b * H + h) * nblk + blk] = s;
  for (int r = 0; r < rows; ++r) {
    int64_t off = row_off(layout, B, H, N, D, b, h, n0 + r);
    for (int j = 0; j < D; ++j) {
      uint8_t c = 0;
      if (s != 0.0f) {
        float v = y[(int64_t)r * D + j] / s;
        if (code_dtype == ORC_INT8) {
          float q = rintf(v);                  /* default rounding: half to even */
          if (q > 127.0f) q = 127.0f;
          if (q < -127.0f) q = -127.0f;
          c = (uint8_t)(int8_t)q;
        } else if (code_dtype == ORC_INT4_PACKED) {
          float q = rintf(v);                  /* one signed code per byte here; */
          if (q > 7.0f) q = 7.0f;              /* the caller packs two per byte  */
          if (q < -7.0f) q = -7.0f;
          c = (uint8_t)(int8_t)q;
        } else {
          c = orc_e4m3_from_f32(v);
        }
      }
      codes[off + j] = c;
    }
  }
  free(y);
  free(xr);
  return 0;
}

/* All blocks of one (b, h). */
int orc_quant_head(const uint16_t* x, int x_dtype, int layout, int B, int H, int N, int D,
                   const float* R, int T, int code_dtype, int b, int h,
                   uint8_t* codes, float* scales) {
  int nblk = (N + T - 1) / T;
  for (int blk = 0; blk < nblk; ++blk) {
    int rc = orc_quant_block(x, x_dtype, layout, B, H, N, D, R, T, code_dtype, b, h, blk, codes, scales);
    if (rc) return rc;
  }
  return 0;
}

/* ------------------------------------------------------------------------ */
/* Quantized prefill attention                                              */
/* ------------------------------------------------------------------------ */

static double code_value(const void* c, int dtype, int64_t i) {
  if (dtype == ORC_INT8) return (double)((const int8_t*)c)[i];
  if (dtype == ORC_INT4_PACKED) {              /* element i of a packed array */
    uint8_t b = ((const uint8_t*)c)[i >> 1];
    return (double)((i & 1) ? orc_int4_hi(b) : orc_int4_lo(b));
  }
  if (dtype == ORC_FP8_E4M3) return (double)orc_e4m3_to_f32(((const uint8_t*)c)[i]);
  return (double)((const float*)c)[i];       /* ORC_F32 */
}

/*
 * Output rows of quantized attention for one (b, h).
 *
 * Inputs are the codes and per-block scales of Q (blocks of q_block tokens),
 * K and V (blocks of kv_block tokens), laid out as the quantizer writes them;
 * Q and K have code_dtype, V has v_dtype (INT4_PACKED: two codes per byte).
 * For each requested query row i:
 *
 *   for each key tile t of kv_tile keys, ascending (tiles whose keys are all
 *   masked for this row are skipped):
 *     dot_j  = sum_d qcode[i][d] * kcode[j][d]             (exact)
 *     s_j    = (float)dot_j * sQ * sK[j / kv_block] * scale (float32, in
 *                                                          this order)
 *     keys j > i are masked when causal; keys j >= N_kv do not exist
 *     m_new  = max(m, max_j s_j)                           (float32)
 *     alpha  = expf(m - m_new)                             (float32; 0 at start)
 *     p_j    = expf(s_j - m_new)                           (float32)
 *     P_j    = Q(p_j): e4m3(p_j) when V has e4m3 codes, RNE(p_j * 127) / 127
 *              when V has INT8 or INT4 codes (computed as rintf(p_j *
 *              127.0f)), p_j itself when p_quant == 0
 *     l      = l * alpha + sum_j P_j                       (float64)
 *     O      = O * alpha + sum_j P_j * vcode[j] * sV[j / kv_block] (float64)
 *   out = O / l, rounded to bfloat16 (RNE); lse = m + ln(l).
 *
 * rows: query row indices (0..N_q-1); out_bf16: [nrows, D]; out_f64,
 * lse: optional [nrows, D] / [nrows].
 */
int orc_prefill_rows(const void* qc, const float* qs, const void* kc, const float* ks,
                     const void* vc, const float* vs, int code_dtype, int v_dtype, int layout,
                     int B, int H, int Nq, int Nkv, int D, int q_block, int kv_block,
                     int kv_tile, int causal, float softmax_scale, int p_quant,
                     int b, int h, const int* rows, int nrows,
                     uint16_t* out_bf16, double* out_f64, double* lse) {
  if (kv_tile <= 0 || q_block <= 0 || kv_block <= 0) return 1;
  if (softmax_scale <= 0.0f) softmax_scale = 1.0f / sqrtf((float)D);
  int nqb = (Nq + q_block - 1) / q_block;
  int nkb = (Nkv + kv_block - 1) / kv_block;
  double* qv = (double*)malloc(sizeof(double) * D);
  double* O = (double*)malloc(sizeof(double) * D);
  float* s = (float*)malloc(sizeof(float) * kv_tile);
  if (!qv || !O || !s) { free(qv); free(O); free(s); return 2; }
  for (int r = 0; r < nrows; ++r) {
    int i = rows[r];
    int64_t qoff = row_off(layout, B, H, Nq, D, b, h, i);
    for (int d = 0; d < D; ++d) qv[d] = code_value(qc, code_dtype, qoff + d);
    float sq = qs[((int64_t)b * H + h) * nqb + i / q_block];
    float m = -INFINITY;
    double l = 0.0;
    for (int d = 0; d < D; ++d) O[d] = 0.0;
    int last_key = causal ? (i < Nkv - 1 ? i : Nkv - 1) : Nkv - 1;
    for (int t0 = 0; t0 <= last_key; t0 += kv_tile) {
      int t1 = t0 + kv_tile - 1;
      if (t1 > last_key) t1 = last_key;
      float tile_max = -INFINITY;
      for (int j = t0; j <= t1; ++j) {
        int64_t koff = row_off(layout, B, H, Nkv, D, b, h, j);
        double dot = 0.0;                    /* exact: see header note */
        for (int d = 0; d < D; ++d) dot += qv[d] * code_value(kc, code_dtype, koff + d);
        float sk = ks[((int64_t)b * H + h) * nkb + j / kv_block];
        float sj = (float)dot * sq * sk * softmax_scale;
        s[j - t0] = sj;
        if (sj > tile_max) tile_max = sj;
      }
      float m_new = m > tile_max ? m : tile_max;
      float alpha = expf(m - m_new);         /* expf(-inf) = 0 on the first tile */
      double tile_l = 0.0;
      for (int d = 0; d < D; ++d) O[d] *= (double)alpha;
      for (int j = t0; j <= t1; ++j) {
        float p = expf(s[j - t0] - m_new);
        double pq;
        if (!p_quant)
          pq = (double)p;
        else if (v_dtype == ORC_INT8 || v_dtype == ORC_INT4_PACKED)
          pq = (double)rintf(p * 127.0f) / 127.0;
        else
          pq = (double)orc_e4m3_to_f32(orc_e4m3_from_f32(p));
        tile_l += pq;
        if (pq != 0.0) {
          int64_t voff = row_off(layout, B, H, Nkv, D, b, h, j);
          double sv = (double)vs[((int64_t)b * H + h) * nkb + j / kv_block];
          for (int d = 0; d < D; ++d) O[d] += pq * code_value(vc, v_dtype, voff + d) * sv;
        }
      }
      l = l * (double)alpha + tile_l;
      m = m_new;
    }
    for (int d = 0; d < D; ++d) {
      double o = O[d] / l;
      out_bf16[(int64_t)r * D + d] = orc_f64_to_bf16(o);
      if (out_f64) out_f64[(int64_t)r * D + d] = o;
    }
    if (lse) lse[r] = (double)m + log(l);
  }
  free(qv);
  free(O);
  free(s);
  return 0;
}

/*
 * Exact attention in float64 on the unquantized, unrotated inputs
 * (bfloat16/float16 bit patterns): softmax(q K^T * scale) V for the
 * requested rows of one (b, h). For error reporting only.
 */
int orc_exact_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v, int in_dtype,
                   int layout, int B, int H, int Nq, int Nkv, int D, int causal,
                   double softmax_scale, int b, int h, const int* rows, int nrows, double* out) {
  if (softmax_scale <= 0.0) softmax_scale = 1.0 / sqrt((double)D);
  double* s = (double*)malloc(sizeof(double) * (Nkv > 0 ? Nkv : 1));
  if (!s) return 2;
  for (int r = 0; r < nrows; ++r) {
    int i = rows[r];
    int64_t qoff = row_off(layout, B, H, Nq, D, b, h, i);
    int last = causal ? (i < Nkv - 1 ? i : Nkv - 1) : Nkv - 1;
    double m = -INFINITY;
    for (int j = 0; j <= last; ++j) {
      int64_t koff = row_off(layout, B, H, Nkv, D, b, h, j);
      double dot = 0.0;
      for (int d = 0; d < D; ++d)
        dot += (double)in_to_f32(q, in_dtype, qoff + d) * (double)in_to_f32(k, in_dtype, koff + d);
      s[j] = dot * softmax_scale;
      if (s[j] > m) m = s[j];
    }
    double l = 0.0;
    for (int d = 0; d < D; ++d) out[(int64_t)r * D + d] = 0.0;
    for (int j = 0; j <= last; ++j) {
      double p = exp(s[j] - m);
      l += p;
      int64_t voff = row_off(layout, B, H, Nkv, D, b, h, j);
      for (int d = 0; d < D; ++d) out[(int64_t)r * D + d] += p * (double)in_to_f32(v, in_dtype, voff + d);
    }
    for (int d = 0; d < D; ++d) out[(int64_t)r * D + d] /= l;
  }
  free(s);
  return 0;
}

/* ------------------------------------------------------------------------ */
/* Decode against a quantized KV cache                                      */
/* ------------------------------------------------------------------------ */

/*
 * One query token of one (b, h_q) against the KV cache of kv head
 * h_kv = h_q / (H_q / H_kv).
 *
 * The query is quantized per (b, h_q) for both cache types:
 *   sq     = max_d |q[d]| / 127 (float32), qcode[d] = RNE(q[d] / sq) (float32
 *            division), clamped to [-127, 127]; sq == 0 gives zero codes
 * INT8 cache ("INT8 量化算子", item 3 of the ops-transformer section: K/V
 * stored as INT8 and read without converting back to fp16; Q is INT8 too):
 *   s_t    = (sum_d qcode[d] kcode[t][d]) * sq * sK[t / kv_block] * scale
 *   v_t[d] = vcode[t][d] * sV[t / kv_block]
 * Packed INT4 cache (two codes per byte, element 2i low nibble; one fp16
 * scale per token per group of `group` elements along D): the nibbles are
 * widened to INT8 and multiplied with the same INT8 query codes ("FlashAttention
 * 的 INT8/INT4 量化", 第二层: INT4 is converted to INT8 before the matrix
 * multiply; "INT8 量化算子": the query is INT8 too):
 *   s_t    = sum_g sK[t][g] * (sum_{d in g} qcode[d] kcode[t][d]) * sq * scale
 *   v_t[d] = vcode[t][d] * sV[t][d / group]
 * Softmax over all L keys (probabilities are not quantized), float64:
 *   out = sum_t p_t v_t / sum_t p_t with p_t = exp(s_t - max s), rounded to
 *   bfloat16.
 * With splits > 1 the L keys are cut into `splits` contiguous ranges of
 * ceil(L / splits) keys; each range keeps its own (max, sum, accumulator) and
 * the ranges are merged at the end: M = max m_r, w_r = exp(m_r - M),
 * out = sum_r w_r O_r / sum_r w_r l_r. The result equals splits == 1 up to
 * float64 rounding.
 *
 * q: bfloat16 bits [B, H_q, D]. k/v: INT8 [B,H_kv,L,D] or bytes
 * [B,H_kv,L,D/2]. k_scales/v_scales: float32 [B,H_kv,ceil(L/kv_block)] (INT8)
 * or float16 bits [B,H_kv,L,D/group] (INT4).
 */
int orc_decode_one(const uint16_t* q, const void* kc, const void* vc, const void* ksc,
                   const void* vsc, int kv_dtype, int B, int Hq, int Hkv, int L, int D,
                   int kv_block, int group, float softmax_scale, int splits, int b, int hq,
                   uint16_t* out_bf16, double* out_f64) {
  (void)B;
  if (Hkv <= 0 || Hq % Hkv || splits <= 0 || D <= 0) return 1;
  if (softmax_scale <= 0.0f) softmax_scale = 1.0f / sqrtf((float)D);
  int hk = hq / (Hq / Hkv);
  const uint16_t* qrow = q + ((int64_t)b * Hq + hq) * D;
  double* qf = (double*)malloc(sizeof(double) * D);
  double* O = (double*)malloc(sizeof(double) * D * (size_t)splits);
  double* ms = (double*)malloc(sizeof(double) * splits);
  double* ls = (double*)malloc(sizeof(double) * splits);
  if (!qf || !O || !ms || !ls) { free(qf); free(O); free(ms); free(ls); return 2; }
  float sq = 0.0f;
  {
    float amax = 0.0f;
    for (int d = 0; d < D; ++d) {
      float a = fabsf(orc_bf16_to_f32(qrow[d]));
      if (a > amax) amax = a;
    }
    sq = amax / 127.0f;
    for (int d = 0; d < D; ++d) {
      float c = 0.0f;
      if (sq != 0.0f) {
        c = rintf(orc_bf16_to_f32(qrow[d]) / sq);
        if (c > 127.0f) c = 127.0f;
        if (c < -127.0f) c = -127.0f;
      }
      qf[d] = (double)c;
    }
  }
  int nkb = (L + kv_block - 1) / kv_block;
  int ngroups = D / group;
  int per = (L + splits - 1) / splits;
  int64_t head = (int64_t)b * Hkv + hk;
  for (int sp = 0; sp < splits; ++sp) {
    int t0 = sp * per, t1 = t0 + per < L ? t0 + per : L;
    double m = -INFINITY, l = 0.0;
    double* Os = O + (int64_t)sp * D;
    for (int d = 0; d < D; ++d) Os[d] = 0.0;
    for (int t = t0; t < t1; ++t) {
      double s;
      if (kv_dtype == ORC_INT8) {
        const int8_t* kr = (const int8_t*)kc + (head * L + t) * D;
        int64_t dot = 0;
        for (int d = 0; d < D; ++d) dot += (int64_t)qf[d] * kr[d];
        double sk = ((const float*)ksc)[head * nkb + t / kv_block];
        s = (double)dot * (double)sq * sk * (double)softmax_scale;
      } else {
        const uint8_t* kr = (const uint8_t*)kc + (head * L + t) * (D / 2);
        const uint16_t* skr = (const uint16_t*)ksc + (head * L + t) * ngroups;
        s = 0.0;
        for (int g = 0; g < ngroups; ++g) {
          int64_t part = 0;
          for (int d = g * group; d < (g + 1) * group; ++d) {
            int c = (d & 1) ? orc_int4_hi(kr[d / 2]) : orc_int4_lo(kr[d / 2]);
            part += (int64_t)qf[d] * c;
          }
          s += (double)part * (double)orc_f16_to_f32(skr[g]);
        }
        s *= (double)sq * (double)softmax_scale;
      }
      double m_new = s > m ? s : m;
      double alpha = exp(m - m_new);
      double p = exp(s - m_new);
      l = l * alpha + p;
      for (int d = 0; d < D; ++d) Os[d] *= alpha;
      if (kv_dtype == ORC_INT8) {
        const int8_t* vr = (const int8_t*)vc + (head * L + t) * D;
        double sv = ((const float*)vsc)[head * nkb + t / kv_block];
        for (int d = 0; d < D; ++d) Os[d] += p * vr[d] * sv;
      } else {
        const uint8_t* vr = (const uint8_t*)vc + (head * L + t) * (D / 2);
        const uint16_t* svr = (const uint16_t*)vsc + (head * L + t) * ngroups;
        for (int d = 0; d < D; ++d) {
          int c = (d & 1) ? orc_int4_hi(vr[d / 2]) : orc_int4_lo(vr[d / 2]);
          Os[d] += p * c * (double)orc_f16_to_f32(svr[d / group]);
        }
      }
      m = m_new;
    }
    ms[sp] = m;
    ls[sp] = l;
  }
  double M = -INFINITY;
  for (int sp = 0; sp < splits; ++sp)
    if (ms[sp] > M) M = ms[sp];
  double lt = 0.0;
  for (int d = 0; d < D; ++d) qf[d] = 0.0;   /* reuse as the merged accumulator */
  for (int sp = 0; sp < splits; ++sp) {
    if (ls[sp] == 0.0) continue;             /* empty range */
    double w = exp(ms[sp] - M);
    lt += w * ls[sp];
    for (int d = 0; d < D; ++d) qf[d] += w * O[(int64_t)sp * D + d];
  }
  for (int d = 0; d < D; ++d) {
    double o = lt > 0.0 ? qf[d] / lt : 0.0;
    out_bf16[d] = orc_f64_to_bf16(o);
    if (out_f64) out_f64[d] = o;
  }
  free(qf);
  free(O);
  free(ms);
  free(ls);
  return 0;
}

/* ------------------------------------------------------------------------ */
/* KV-cache quantize-on-append                                              */
/* ------------------------------------------------------------------------ */

/* float32 -> fp16 bits, round to nearest even (overflow -> inf; subnormal
 * results rounded at their own spacing of 2^-24). Worked from the binary16
 * format: 1 sign, 5 exponent (bias 15), 10 mantissa bits. */
uint16_t orc_f32_to_f16(float x) {
  uint16_t sign = signbit(x) ? 0x8000 : 0;
  double a = fabs((double)x);
  if (isnan(x)) return sign | 0x7E00;
  if (a >= 65520.0) return sign | 0x7C00;     /* rounds beyond the largest finite 65504 */
  int e;
  frexp(a, &e);                               /* a = f * 2^e, f in [0.5, 1) */
  int ulp_e = (e - 1) - 10;                   /* spacing 2^(e-1-10) for normals */
  if (ulp_e < -24) ulp_e = -24;               /* subnormal spacing */
  double q = a / ldexp(1.0, ulp_e);           /* exact: a power-of-two scaling */
  double r = nearbyint(q);                    /* default rounding mode: half to even */
  double v = r * ldexp(1.0, ulp_e);
  if (v == 0.0) return sign;
  int ev;
  frexp(v, &ev);
  if (ev - 1 < -14) return sign | (uint16_t)(v / ldexp(1.0, -24));      /* subnormal */
  uint16_t bits = (uint16_t)(((ev - 1 + 15) << 10) | ((uint32_t)(ldexp(v, -(ev - 1)) * 1024.0) - 1024));
  return sign | bits;
}

/*
 * INT8 cache, one float32 scale per block of kv_block tokens per (b, h_kv):
 * "INT8 量化算子", ops-transformer item 3 (KV Cache 也量化: in the decode phase
 * the new K/V rows are written into the cache as INT8 codes). How a block's
 * scale evolves while tokens are appended to it is not on the pages; the
 * reading taken here keeps it at absmax / 127 of every token written to the
 * block so far. For each block touched by the n new tokens at [L, L + n):
 *   a     = max |x| over the block's new tokens and all D channels
 *   s_new = max(s_old, a / 127)        (float32 division; s_old = 0 when the
 *                                       block holds no token before L)
 *   if s_new > s_old and the block holds tokens before L, each of their codes
 *   is requantized:  c' = clamp(RNE(f32(c * s_old) / s_new), -127, 127)
 *   new tokens:      c  = clamp(RNE(x / s_new), -127, 127)   (float32 division)
 *   s_new == 0 gives zero codes.
 * x: bf16 [B, H_kv, n, D]; cache: int8 [B, H_kv, L_max, D]; scales: float32
 * [B, H_kv, ceil(L_max / kv_block)]. Updates (b, h) in place.
 */
int orc_kv_append_int8(const uint16_t* x, int B, int Hkv, int n, int D, int L, int Lmax, int kv_block,
                       int8_t* cache, float* scales, int b, int h) {
  if (n <= 0 || L < 0 || L + n > Lmax || kv_block <= 0 || b >= B || h >= Hkv) return 1;
  int64_t head = (int64_t)b * Hkv + h;
  int nblk = (Lmax + kv_block - 1) / kv_block;
  for (int blk = L / kv_block; blk * kv_block < L + n; ++blk) {
    int b0 = blk * kv_block;
    int t0 = L > b0 ? L : b0;                               /* first new token of the block */
    int t1 = L + n < b0 + kv_block ? L + n : b0 + kv_block; /* one past the last */
    float a = 0.0f;
    for (int t = t0; t < t1; ++t)
      for (int d = 0; d < D; ++d) {
        float v = fabsf(orc_bf16_to_f32(x[(head * n + (t - L)) * D + d]));
        if (v > a) a = v;
      }
    float s_old = t0 > b0 ? scales[head * nblk + blk] : 0.0f;
    float s1 = a / 127.0f;
    float s = s1 > s_old ? s1 : s_old;
    if (s > s_old && t0 > b0) {
      for (int t = b0; t < t0; ++t)
        for (int d = 0; d < D; ++d) {
          int8_t* c = &cache[(head * Lmax + t) * D + d];
          float y = (float)(*c) * s_old;                    /* one float32 rounding */
          float q = rintf(y / s);
          if (q > 127.0f) q = 127.0f;
          if (q < -127.0f) q = -127.0f;
          *c = (int8_t)q;
        }
    }
    for (int t = t0; t < t1; ++t)
      for (int d = 0; d < D; ++d) {
        float q = 0.0f;
        if (s != 0.0f) {
          q = rintf(orc_bf16_to_f32(x[(head * n + (t - L)) * D + d]) / s);
          if (q > 127.0f) q = 127.0f;
          if (q < -127.0f) q = -127.0f;
        }
        cache[(head * Lmax + t) * D + d] = (int8_t)q;
      }
    scales[head * nblk + blk] = s;
  }
  return 0;
}

/*
 * Packed INT4 cache ("ops-transformer INT8/INT4 量化推理", 5.1: one fp16 scale
 * per group of `group` elements; 5.2: two codes per byte, element 2i in the
 * low nibble): each new token gets its own scales, one per group along D.
 *   a = max |x| over the group;  s16 = fp16(a / 7) (float32 division, then
 *   RNE to fp16);  s = (float) s16
 *   c = clamp(RNE(x / s), -7, 7) (float32 division); s == 0 gives zero codes
 * x: bf16 [B, H_kv, n, D]; cache: bytes [B, H_kv, L_max, D/2]; scales: fp16
 * bits [B, H_kv, L_max, D/group]. Updates (b, h) in place.
 */
int orc_kv_append_int4(const uint16_t* x, int B, int Hkv, int n, int D, int L, int Lmax, int group,
                       uint8_t* cache, uint16_t* scales, int b, int h) {
  if (n <= 0 || L < 0 || L + n > Lmax || group <= 0 || D % group || D % 2 || b >= B || h >= Hkv) return 1;
  int64_t head = (int64_t)b * Hkv + h;
  int ng = D / group;
  int codes[1024];
  if (D > 1024) return 1;
  for (int t = L; t < L + n; ++t) {
    const uint16_t* xr = x + (head * n + (t - L)) * D;
    for (int g = 0; g < ng; ++g) {
      float a = 0.0f;
      for (int d = g * group; d < (g + 1) * group; ++d) {
        float v = fabsf(orc_bf16_to_f32(xr[d]));
        if (v > a) a = v;
      }
      uint16_t s16 = orc_f32_to_f16(a / 7.0f);
      float s = orc_f16_to_f32(s16);
      scales[(head * Lmax + t) * ng + g] = s16;
      for (int d = g * group; d < (g + 1) * group; ++d) {
        float q = 0.0f;
        if (s != 0.0f) {
          q = rintf(orc_bf16_to_f32(xr[d]) / s);
          if (q > 7.0f) q = 7.0f;
          if (q < -7.0f) q = -7.0f;
        }
        codes[d] = (int)q;
      }
    }
    uint8_t* row = cache + (head * Lmax + t) * (D / 2);
    for (int i = 0; i < D / 2; ++i) row[i] = orc_int4_pack(codes[2 * i], codes[2 * i + 1]);
  }
  return 0;
}

int orc_abi_version(void) { return 1; }
