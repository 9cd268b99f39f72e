/*
 * qattn.h -- C ABI of libqattn: block-quantized attention on NVIDIA B200
 * (sm_100a).
 *
 * The method (as stated on the pages this library implements):
 *   1. Q and K are multiplied by one shared orthogonal matrix R before
 *      quantization, to spread outlier channels ("MindIE-SD quantization",
 *      section FA量化 / 技术特点 / 旋转(Rotate)). V is not rotated.
 *   2. Q, K, V are quantized dynamically per block of tokens, one scale per
 *      (batch, head, block): Q blocks of 128 tokens, K/V blocks of 256, to
 *      float8_e4m3fn (same page, 块量化) or to symmetric INT8 with
 *      scale = max|x| / 127, code = round(x / scale), zero point 0
 *      ("INT8 量化算子", 对称量化).
 *   3. Attention runs on the codes: INT8 x INT8 -> INT32 (or e4m3 x e4m3 ->
 *      FP32) for Q K^T, a running softmax over key tiles, P quantized to the
 *      same 8-bit type, P V with the per-block V scale, output in bfloat16
 *      ("MindIE-SD quantization", FP8 Attention; "INT8 量化算子",
 *      ops-transformer items 1-3; "FlashAttention 的 INT8/INT4 量化",
 *      三层实现详解).
 *   4. Decode reads an INT8 or packed INT4 KV cache directly, with no
 *      dequantize-to-fp16 pass ("INT8 量化算子", item 3 KV Cache 也量化;
 *      "ops-transformer INT8/INT4 量化推理", 5.1 and 5.2 for INT4 groups and
 *      packing).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller (except
 *     the host inputs and output of qattn_attention_path_host); the
 *     library never frees or keeps them. The library allocates no device
 *     memory per call (scratch for decode is passed in as `workspace`).
 *   - Work is enqueued asynchronously on `stream` (NULL = legacy default
 *     stream). The call returns once the launch is enqueued.
 *   - Arguments are validated before anything is launched; on any error
 *     nothing is launched and a status other than QATTN_OK is returned.
 *     A failed launch returns QATTN_ERR_CUDA.
 *   - Kernels that wait on on-chip barriers give up after about one second,
 *     record QATTN_ERR_TIMEOUT in a per-device error word and exit cleanly;
 *     qattn_device_error() reads and clears that word.
 *   - Layouts: QATTN_BNSD = [B, H, N, D] (head-major), QATTN_BSND =
 *     [B, N, H, D] (token-major); N is the number of tokens, H the number
 *     of heads. Both are dense and row-major.
 *   - Pointers must be 16-byte aligned (QATTN_ERR_ALIGNMENT otherwise).
 *   - Supported head sizes: D in {64, 128} (D = 128 for decode).
 */
#ifndef QATTN_H_
#define QATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define QATTN_ABI_VERSION 1

typedef enum qattn_status {
  QATTN_OK = 0,
  QATTN_ERR_INVALID_ARG = 1, /* null pointer, negative size, inconsistent shapes */
  QATTN_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. D = 96) */
  QATTN_ERR_ALIGNMENT = 3,   /* a pointer is not 16-byte aligned */
  QATTN_ERR_WORKSPACE = 4,   /* decode workspace missing or too small */
  QATTN_ERR_CUDA = 5,        /* a CUDA runtime call or launch failed */
  QATTN_ERR_TIMEOUT = 6      /* a kernel's bounded barrier wait ran out */
} qattn_status_t;

typedef enum qattn_layout { QATTN_BNSD = 0, QATTN_BSND = 1 } qattn_layout_t;

typedef enum qattn_dtype {
  QATTN_F16 = 0,
  QATTN_BF16 = 1,
  QATTN_INT8 = 2,        /* signed 8-bit codes */
  QATTN_FP8_E4M3 = 3,    /* float8_e4m3fn codes (OCP E4M3, finite) */
  QATTN_INT4_PACKED = 4  /* two signed 4-bit codes per byte, element 2i in bits 0..3 */
} qattn_dtype_t;

/* Same type as cudaStream_t. */
typedef struct CUstream_st* qattn_stream_t;

/* Returns QATTN_ABI_VERSION of the built library. */
int qattn_abi_version(void);

/* Static, human-readable name of a status code. */
const char* qattn_status_string(qattn_status_t status);

/*
 * Fused rotation + dynamic block quantization (one launch per tensor).
 *
 * Defined by: "MindIE-SD quantization", FA量化 / 技术特点 (旋转, 块量化);
 * "INT8 量化算子", 1. 对称量化.
 *
 * For every (b, h) and every block of `block_tokens` consecutive tokens
 * (the last block may be shorter when N is not a multiple):
 *   y      = x R                  rotation; R == NULL means y = x. Each
 *                                 y[j] is the float32 fused multiply-add
 *                                 chain over k = 0..D-1 in ascending order
 *                                 starting from +0 (bit-reproducible).
 *   amax   = max |y| over the block's tokens and all D channels
 *   scale  = amax / qmax          float32 IEEE division; qmax = 127 (INT8)
 *                                 or 448 (e4m3)
 *   code   = RNE(y / scale)       float32 IEEE division, then round half to
 *                                 even; INT8 saturates to [-127, 127], e4m3
 *                                 saturates to +-448. scale == 0 gives all
 *                                 codes 0.
 *
 * x:            x_dtype (QATTN_F16 or QATTN_BF16) values, `layout`,
 *               [B,H,N,D] or [B,N,H,D].
 * rot:          D x D float32 row-major (rot[k*D + j] = R[k][j]), or NULL.
 * block_tokens: tokens per block: 128 (Q) or 256 (K/V).
 * code_dtype:   QATTN_INT8, QATTN_FP8_E4M3, or QATTN_INT4_PACKED:
 *               scale = max|x| / 7, codes RNE(x / scale) clamped to [-7, 7]
 *               ("FlashAttention 的 INT8/INT4 量化", 第二层, with the block
 *               scales above), two per byte, element 2i in the low nibble
 *               ("ops-transformer INT8/INT4 量化推理", 5.2).
 * codes:        output, 1 byte per element (INT4: per 2 elements), same
 *               layout as x ([..., D/2] for INT4).
 * scales:       output, float32 [B, H, ceil(N / block_tokens)].
 */
qattn_status_t qattn_rotate_block_quant(const void* x, qattn_dtype_t x_dtype,
                                        qattn_layout_t layout, int B, int H, int N, int D,
                                        const float* rot, int block_tokens,
                                        qattn_dtype_t code_dtype, void* codes, float* scales,
                                        qattn_stream_t stream);

/*
 * The three quantizations of one prefill at once: Q (blocks of 128 tokens)
 * and K (blocks of 256) rotated by the same R, V (blocks of 256) not rotated,
 * all to code_dtype -- the same codes and scales, bit for bit, as three
 * qattn_rotate_block_quant calls ("MindIE-SD quantization", FA量化 / 技术特点:
 * rotation of Q and K, then block quantization of Q/K/V).
 *
 * With rot != NULL the two rotations (bound by float32 FMA throughput, one
 * persistent CTA per SM) run concurrently, each on half of the SMs, on two
 * streams internal to the library (created on first use per device and
 * kept); the quantization of V is enqueued on `stream` and takes SMs as they
 * free up; `stream` then waits for both rotations, so the call behaves as an
 * ordinary stream-ordered operation. Concurrent calls on one device
 * serialise their enqueueing. The call can be captured in a CUDA graph (the
 * internal streams join the capture through events recorded on `stream`);
 * the first call on a device creates those streams and events and should
 * come before any capture. With rot == NULL the three passes run one after
 * the other on `stream`.
 *
 * Arguments as qattn_rotate_block_quant, for three tensors of one shape:
 *   q, k, v:            F16/BF16 [B,H,N,D] (BNSD) or [B,N,H,D] (BSND).
 *   q_codes, q_scales:  codes like q (D/2 bytes per row for INT4), float32
 *                       [B,H,ceil(N/128)].
 *   k_codes/v_codes, k_scales/v_scales: likewise with [B,H,ceil(N/256)].
 * Errors: those of qattn_rotate_block_quant for any of the three; nothing is
 * launched on an argument error.
 */
qattn_status_t qattn_rotate_block_quant_qkv(const void* q, const void* k, const void* v,
                                            qattn_dtype_t x_dtype, qattn_layout_t layout, int B,
                                            int H, int N, int D, const float* rot,
                                            qattn_dtype_t code_dtype, void* q_codes,
                                            float* q_scales, void* k_codes, float* k_scales,
                                            void* v_codes, float* v_scales, qattn_stream_t stream);

/*
 * Quantized attention over block-quantized codes (prefill).
 *
 * Defined by: "MindIE-SD quantization", FA量化 / FP8 Attention (attention in
 * the FP8 domain, output returned in the original precision); "INT8 量化算子",
 * ops-transformer items 1-2 (INT8 x INT8 -> INT32, convert at the output,
 * scales kept on chip); "FlashAttention 的 INT8/INT4 量化", 三层实现详解
 * (outer loop over query tiles, inner loop over key/value tiles).
 *
 * For query row i of head (b, h), key tiles of 128 keys in ascending order:
 *   S[i,j] = sum_d qcode[i,d] kcode[j,d]   exact INT32 (INT8 codes) or
 *                                          FP32-accumulated (e4m3 codes)
 *   s[i,j] = S[i,j] * q_scales[b,h,i/q_block] * k_scales[b,h,j/kv_block]
 *            * softmax_scale              (masked: j > i when causal)
 *   running max m, alpha = exp(m_old - m_new), p = exp(s - m_new)
 *   P = e4m3(p) for e4m3 codes; round(127 p) / 127 for INT8 codes
 *   l = l * alpha + sum_j P;  O = O * alpha + sum_j P vcode[j] v_scales[b,h,j/kv_block]
 *   out = bf16(O / l);  lse = m + ln(l) (natural log)
 *
 * q_codes/k_codes/v_codes: code_dtype bytes in `layout`; Q is [B,H,N_q,D]
 *               (or [B,N_q,H,D]), K and V use N_kv tokens.
 * q_scales:     float32 [B, H, ceil(N_q / q_block)];
 * k_scales, v_scales: float32 [B, H, ceil(N_kv / kv_block)].
 * q_block:      must be 128; kv_block: must be 256 (the method's sizes).
 * causal:       0 or 1; causal requires N_q == N_kv (top-left aligned).
 * softmax_scale: <= 0 selects 1/sqrt(D) (computed in float32).
 * out:          bfloat16, same layout as Q.
 * lse:          optional (NULL) float32 [B, H, N_q].
 * code_dtype:   QATTN_INT8 or QATTN_FP8_E4M3 (Q, K and V alike; see
 *               qattn_prefill_mixed for V in another type).
 */
qattn_status_t qattn_prefill(const void* q_codes, const float* q_scales, const void* k_codes,
                             const float* k_scales, const void* v_codes, const float* v_scales,
                             qattn_dtype_t code_dtype, qattn_layout_t layout, int B, int H,
                             int N_q, int N_kv, int D, int q_block, int kv_block, int causal,
                             float softmax_scale, void* out, float* lse, qattn_stream_t stream);

/*
 * Quantized prefill attention with V in its own code type (mixed precision).
 *
 * Defined by: "FlashAttention 的 INT8/INT4 量化", 第三层 (混合精度: Q/K in
 * INT8 for the scores, V in a narrower format for the weighted sum) and
 * 第二层 (INT4 codes widened to INT8 for the matmul).
 *
 * Same computation and arguments as qattn_prefill, with:
 *   qk_dtype: QATTN_INT8, QATTN_FP8_E4M3 or QATTN_INT4_PACKED (Q and K);
 *   v_dtype:  QATTN_INT8, QATTN_FP8_E4M3 or QATTN_INT4_PACKED (V codes;
 *             packed INT4 tensors are [B,H,N,D/2] or [B,N,H,D/2] bytes, as
 *             written by qattn_rotate_block_quant). Supported pairs: INT8 Q/K
 *             with any V; e4m3 Q/K with e4m3 V; INT4 Q/K with INT4 V
 *             ("FlashAttention 的 INT8/INT4 量化", 第二层: every INT4 operand
 *             widened to INT8 for the matmul; the scores are exact integers).
 *             Other pairs: QATTN_ERR_UNSUPPORTED.
 *   P is rounded to INT8 codes (round(127 p) / 127) when V is INT8 or INT4
 *   (INT4 V is widened to INT8 on chip) and to e4m3 when V is e4m3.
 * v_scales: float32 [B, H, ceil(N_kv / kv_block)] for every V type.
 */
qattn_status_t qattn_prefill_mixed(const void* q_codes, const float* q_scales, const void* k_codes,
                                   const float* k_scales, const void* v_codes, const float* v_scales,
                                   qattn_dtype_t qk_dtype, qattn_dtype_t v_dtype, qattn_layout_t layout,
                                   int B, int H, int N_q, int N_kv, int D, int q_block, int kv_block,
                                   int causal, float softmax_scale, void* out, float* lse,
                                   qattn_stream_t stream);

/*
 * Packed INT4 codes widened to INT8 codes of the same values.
 *
 * Defined by: "FlashAttention 的 INT8/INT4 量化", 第二层 (INT4 codes are
 * widened to INT8 before the integer matmul); packing as in
 * "ops-transformer INT8/INT4 量化推理", 5.2.
 *
 * out[2i] = the low nibble of packed[i], out[2i + 1] = its high nibble, each
 * as a signed 4-bit value (-8..7) stored in one INT8 byte. A packed code
 * tensor [B,H,N,D/2] or [B,N,H,D/2] thus becomes the INT8 code tensor
 * [B,H,N,D] or [B,N,H,D] with the same block scales, and
 *   qattn_widen_int4(q), (k), (v) then qattn_prefill(..., QATTN_INT8, ...)
 * computes what qattn_prefill_mixed(..., QATTN_INT4_PACKED,
 * QATTN_INT4_PACKED, ...) computes: the same integer scores and P.V sums
 * (qattn_prefill_mixed widens each nibble on chip as code + 8 and removes
 * the offset in float32, so the two outputs can differ in the last bits;
 * both stay within the prefill's tolerance). Widening V alone does the same
 * for INT8 Q/K with INT4 V. On B200 this order is the faster one: this pass
 * is bound by HBM (n_packed bytes read, 2 n_packed written, the output left
 * in L2), the prefill by instruction issue, where qattn_prefill_mixed
 * widens inside the pipeline that feeds the softmax warps and needs no
 * extra memory.
 *
 *   packed:   n_packed bytes, device memory, 16-byte aligned.
 *   out:      2 * n_packed bytes, device memory, 16-byte aligned,
 *             caller-owned; must not overlap packed.
 * Errors: QATTN_ERR_INVALID_ARG (n_packed < 0, null pointer with
 * n_packed > 0, overlapping ranges), QATTN_ERR_ALIGNMENT, QATTN_ERR_CUDA.
 * n_packed == 0 does nothing. Asynchronous on `stream`; allocates nothing.
 */
qattn_status_t qattn_widen_int4(const void* packed, int64_t n_packed, void* out, qattn_stream_t stream);

/*
 * The dequantize-first comparison path: the standard INT8 path that the
 * pages contrast with quantized attention ("INT8 量化算子", ops-transformer
 * items 1-2: INT8 is converted back to FP16 and multiplied in FP16, where the
 * optimised path feeds INT8 to the matrix unit directly). Built to measure
 * that contrast on B200 beside qattn_prefill; not a step of the method.
 *
 * qattn_dequant_bf16: out[...] = bf16(code * scale[b, h, token / block_tokens])
 * for every element (the float32 product rounded to nearest even).
 *   codes:  INT8 or e4m3 codes (code_dtype), [B,H,N,D] (BNSD) or [B,N,H,D]
 *           (BSND), 16-byte aligned; scales float32 [B,H,ceil(N/block_tokens)].
 *   out:    bfloat16, same layout and shape, 16-byte aligned, caller-owned.
 *   D must be a multiple of 16.
 *
 * qattn_attention_bf16: softmax(Q K^T * softmax_scale) V over bfloat16 Q/K/V
 * with float32 accumulation on the 16-bit tensor-core path; probabilities
 * are not quantized (they are rounded to bfloat16 only as the operand of the
 * P.V product; the row sums use their float32 values). Running softmax over
 * tiles of 64 keys.
 *   q/k/v:  bfloat16 [B,H,N,D] or [B,N,H,D], 16-byte aligned; N_q rows of Q,
 *           N_kv of K and V; D in {64, 128}.
 *   causal: 0/1 (1 needs N_q == N_kv; key j visible to query i iff j <= i).
 *   softmax_scale: <= 0 selects 1/sqrt(D).
 *   out:    bfloat16, layout of Q; lse: nullable float32 [B,H,N_q], natural log.
 * Errors as qattn_prefill.
 */
qattn_status_t qattn_dequant_bf16(const void* codes, const float* scales, qattn_dtype_t code_dtype,
                                  qattn_layout_t layout, int B, int H, int N, int D, int block_tokens,
                                  void* out, qattn_stream_t stream);

qattn_status_t qattn_attention_bf16(const void* q, const void* k, const void* v, qattn_layout_t layout,
                                    int B, int H, int N_q, int N_kv, int D, int causal,
                                    float softmax_scale, void* out, float* lse, qattn_stream_t stream);

/*
 * Bytes of device workspace qattn_decode_kvq needs for these sizes on the
 * current device (0 when no scratch is needed). The value depends on the
 * device's SM count.
 */
size_t qattn_decode_workspace_size(int B, int H_q, int H_kv, int L, int D);

/*
 * One decode step against a quantized KV cache, split over the key axis,
 * with a final softmax merge of the splits.
 *
 * Defined by: "INT8 量化算子", ops-transformer item 3 (KV Cache 也量化: K/V
 * stored as INT8 and attended without converting back to fp16; the query is
 * INT8 too) and its Int8Attention listing; "ops-transformer INT8/INT4
 * 量化推理", 5.1 (one fp16 scale per group of G elements) and 5.2 (two INT4
 * per byte, element 2i in the low nibble).
 *
 * Query head h uses KV head h / (H_q / H_kv). The query is quantized per
 * head: sq = max|q| / 127, qcode = RNE(q / sq) (float32, clamped to
 * [-127, 127]).
 *   INT8 cache:  s_t = (qcode . kcode_t) * sq * k_scales[b,hk,t/kv_block]
 *                * softmax_scale; v_t = vcode_t * v_scales[b,hk,t/kv_block].
 *   INT4 cache:  the nibbles are widened to INT8 ("FlashAttention 的
 *                INT8/INT4 量化", 第二层) and s_t = sum_g k_scales[b,hk,t,g] *
 *                (qcode . kcode_t over group g) * sq * softmax_scale;
 *                v_t[d] = vcode_t[d] * v_scales[b,hk,t,d/group].
 *   out = bf16(sum_t p_t v_t / sum_t p_t), p_t = exp(s_t - max s) in float32.
 *
 * q:        bfloat16 [B, H_q, 1, D].
 * k_cache, v_cache: QATTN_INT8: int8 [B, H_kv, L, D];
 *           QATTN_INT4_PACKED: bytes [B, H_kv, L, D/2].
 * k_scales, v_scales: QATTN_INT8: float32 [B, H_kv, ceil(L/kv_block)];
 *           QATTN_INT4_PACKED: float16 [B, H_kv, L, D/group].
 * kv_block: 256 (INT8); group: 128 or 64 (INT4, must divide D).
 * softmax_scale: <= 0 selects 1/sqrt(D) (float32).
 * out:      bfloat16 [B, H_q, 1, D].
 * workspace / workspace_bytes: device scratch of at least
 *           qattn_decode_workspace_size(B, H_q, H_kv, L, D) bytes (enough
 *           for either cache type; a smaller workspace that holds this
 *           call's own partials is accepted too), 16-byte aligned; its contents need no initialisation and are
 *           overwritten. Calls that share a workspace must not overlap.
 * L == 0 writes zeros to out.
 */
qattn_status_t qattn_decode_kvq(const void* q, const void* k_cache, const void* v_cache,
                                const void* k_scales, const void* v_scales,
                                qattn_dtype_t kv_dtype, int B, int H_q, int H_kv, int L, int D,
                                int kv_block, int group, float softmax_scale, void* out,
                                void* workspace, size_t workspace_bytes, qattn_stream_t stream);

/*
 * qattn_decode_kvq without a workspace argument: the split partials go to a
 * fixed 16 MiB device array inside the library (16777216 bytes, held on every
 * GPU that loads the library until the process exits). No counterpart on
 * the pages; it exists for callers that cannot allocate device memory on
 * their decode path -- their memory is reserved up front by an allocator
 * they do not own, or a cudaMalloc/cudaFree there could synchronise the
 * device and stall other streams. The caller still passes inputs and output.
 *
 * Arguments and results are those of qattn_decode_kvq, bit for bit. A call
 * whose partials (B * H_q * splits * 528 bytes, with the split count of its
 * own cache type) exceed 16 MiB is rejected with QATTN_ERR_WORKSPACE before
 * anything is launched; both stated decode problems fit (B=64 H_q=32 L=8192
 * INT8: 8.25 MiB; B=16 H_q=32 L=32768 INT4: 3.4 MiB). The first call on a
 * device looks up the array's device address (cudaGetSymbolAddress, with
 * that device current) and keeps it for the life of the process; make that
 * first call before any stream capture, and do not call this entry point
 * again on a device after cudaDeviceReset() (the kept address would be
 * stale). Nothing is allocated or freed, ever. Every call shares the one
 * array and it keeps the last call's contents; nothing in it needs to start
 * at zero (each call writes every partial before reading it). Calls that
 * overlap on the GPU (different streams, or host threads without ordering)
 * race on the array: serialise them.
 */
qattn_status_t qattn_decode_kvq_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                        const void* k_scales, const void* v_scales,
                                        qattn_dtype_t kv_dtype, int B, int H_q, int H_kv, int L,
                                        int D, int kv_block, int group, float softmax_scale,
                                        void* out, qattn_stream_t stream);

/*
 * Quantize-on-append: writes n new K (or V) rows into a quantized decode
 * cache at token positions [L, L + n) of every (b, h_kv).
 * "INT8 量化算子", ops-transformer item 3 (KV Cache 也量化: in the decode phase
 * the new K/V rows are stored as INT8); packed INT4 with fp16 group scales:
 * "ops-transformer INT8/INT4 量化推理", 5.1 and 5.2.
 *
 * x_new:   bfloat16 [B, H_kv, n, D], 16-byte aligned.
 * kv_dtype QATTN_INT8:
 *   cache  int8 [B, H_kv, L_max, D] (16-byte aligned); scales float32
 *          [B, H_kv, ceil(L_max / kv_block)]; kv_block must be 256; D a
 *          multiple of 8 up to 1024. A block's scale is absmax / 127 of
 *          every token written to it so far: for each block touched,
 *          s = max(s_old, a / 127) with a the largest |x| of its new rows
 *          (s_old ignored for a block that held no token before L); if s
 *          grew and the block held tokens, their codes become
 *          RNE(f32(c * s_old) / s); new codes RNE(x / s). float32, IEEE
 *          division, codes clamped to [-127, 127]; s == 0 gives zero codes.
 * kv_dtype QATTN_INT4_PACKED:
 *   cache  bytes [B, H_kv, L_max, D/2] (two codes per byte, element 2i in
 *          the low nibble); scales fp16 [B, H_kv, L_max, D/group]; D = 128,
 *          group 128 or 64. Per new token and group: s = fp16(absmax / 7)
 *          (float32 division, RNE to fp16), codes RNE(x / s) clamped to
 *          [-7, 7]; s == 0 gives zero codes.
 * Requires L >= 0, n >= 0 and L + n <= L_max. The caller owns all memory;
 * cache and scales are updated in place on `stream`; rows outside
 * [L, L + n) are not written except the earlier rows of a growing INT8
 * block. Errors: QATTN_ERR_INVALID_ARG (ranges, null pointers),
 * QATTN_ERR_UNSUPPORTED (D, kv_block, group; B or H_kv above 65535, or
 * B * H_kv above 65535 for INT4), QATTN_ERR_ALIGNMENT; nothing
 * is launched on error. n == 0 returns QATTN_OK without a launch.
 */
qattn_status_t qattn_kv_append(const void* x_new, int B, int H_kv, int n, int D,
                               qattn_dtype_t kv_dtype, int L, int L_max, void* cache,
                               void* scales, int kv_block, int group, qattn_stream_t stream);

/*
 * The whole prefill path from HOST buffers: rotation and block quantization
 * of Q and K (qattn_rotate_block_quant with R, blocks of 128 and 256
 * tokens), quantization of V (no rotation, 256-token blocks) and
 * qattn_prefill on the codes -- the path of "MindIE-SD quantization", FA量化
 * (rotate, quantize per block, attention in the low-precision domain,
 * output in the original precision). The results are those of the four
 * device calls made one after another on the same inputs, bit for bit.
 *
 * No counterpart on the pages: it moves the inputs to the GPU and the
 * output back with the copies overlapped with the compute. The (b, h) heads
 * are split into `groups` consecutive groups; group g is copied in on one
 * internal stream, computed on `stream`, and copied out on another, so the
 * copy-in of group g + 1 and the copy-out of group g - 1 run while group g
 * is computed. Two workspace slots alternate between the groups.
 *
 * q, k, v: HOST pointers, x_dtype (QATTN_BF16 or QATTN_F16) [B, H, N, D] or
 *          [B, N, H, D] (layout). Page-locked memory (cudaHostAlloc or
 *          cudaHostRegister) is needed for the copies to overlap; pageable
 *          memory gives the same results, slower.
 * rot:     DEVICE pointer, float32 [D, D] row-major (y = x R), 16-byte
 *          aligned; NULL quantizes Q and K without rotation.
 * code_dtype: QATTN_INT8 or QATTN_FP8_E4M3 (Q, K and V alike).
 * causal, softmax_scale: as for qattn_prefill (N_q = N_kv = N).
 * out:     HOST pointer, bfloat16, same layout as q.
 * groups:  number of head groups, 1..64; 0 selects 8. With layout BSND and
 *          groups > B every group lies within one b (ceil(groups / B) head
 *          ranges per b).
 * workspace: DEVICE memory of at least
 *          qattn_attention_path_host_workspace_size(B, H, N, D, layout,
 *          groups) bytes, 256-byte aligned; contents need no initialisation.
 *          Calls that share a workspace must not overlap.
 * stream:  the compute stream; the call returns once everything is
 *          enqueued, and `out` is complete when `stream` reaches the end of
 *          this call's work. The library keeps two copy streams per device
 *          (created on first use, never destroyed) and serialises the
 *          enqueueing of concurrent calls.
 * Errors: as the device calls (checked for the whole problem before
 * anything is enqueued), QATTN_ERR_WORKSPACE for a missing or small
 * workspace; QATTN_ERR_CUDA if a copy or launch fails to enqueue, in which
 * case `out` is unspecified and the copies already enqueued have finished
 * when the call returns (none still reads or writes the caller's buffers).
 */
size_t qattn_attention_path_host_workspace_size(int B, int H, int N, int D, qattn_layout_t layout,
                                                int groups);
qattn_status_t qattn_attention_path_host(const void* q, const void* k, const void* v,
                                         qattn_dtype_t x_dtype, qattn_layout_t layout, int B, int H,
                                         int N, int D, const float* rot, qattn_dtype_t code_dtype,
                                         int causal, float softmax_scale, void* out, int groups,
                                         void* workspace, size_t workspace_bytes,
                                         qattn_stream_t stream);

/*
 * Waits for `stream`, then reads and clears the per-device error word that
 * kernels set when a bounded barrier wait runs out. Returns QATTN_OK,
 * QATTN_ERR_TIMEOUT, or QATTN_ERR_CUDA if the synchronisation itself failed.
 */
qattn_status_t qattn_device_error(qattn_stream_t stream);

/*
 * Self-test of the bounded-wait path: launches one block that waits on an
 * on-chip barrier that nothing completes, with a limit of `timeout_ms`
 * milliseconds (1..2000). The kernel records QATTN_ERR_TIMEOUT and returns;
 * nothing faults or hangs. Follow with qattn_device_error() to observe it.
 * No counterpart on the pages: it exists to test failure reporting.
 */
qattn_status_t qattn_selftest_wait_timeout(int timeout_ms, qattn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* QATTN_H_ */
