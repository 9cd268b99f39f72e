// qattn_abi.cu -- the extern "C" entry points declared in include/qattn.h:
// argument validation, per-device state (SM count, error word), dispatch to
// the kernel launchers.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <mutex>
#include <unordered_map>

#include "../../include/qattn.h"
#include "qattn_device.cuh"
#include "qattn_internal.h"

namespace qattn {

// Per-device error word written by kernels whose bounded waits run out.
__device__ int g_error_word;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceState {
  bool ready = false;
  int num_sms = 0;
  int* err = nullptr;  // device address of g_error_word on this device
};

DeviceState g_dev[kMaxDevices];
std::mutex g_mu;

// Per-device set-up, done once per device with that device current: SM
// count and the device address of the error word.
qattn_status_t device_state(DeviceState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState& s = g_dev[dev];
  if (!s.ready) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return QATTN_ERR_CUDA;
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return QATTN_ERR_CUDA;
    if (major != 10) return QATTN_ERR_UNSUPPORTED;  // built for sm_100a only
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return QATTN_ERR_CUDA;
    s.num_sms = sms;
    s.err = static_cast<int*>(p);
    s.ready = true;
  }
  *out = &s;
  return QATTN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

qattn_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? QATTN_OK : QATTN_ERR_CUDA; }

__global__ void wait_selftest_kernel(int* err, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();
  // Nothing ever arrives on `bar`: the bounded wait must run out, record
  // QATTN_ERR_TIMEOUT and return.
  mbar_wait(&bar, 0, &abort_flag, err, limit_ns);
}

}  // namespace

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

}  // namespace

namespace {

bool encode_map(CUtensorMap* map, CUtensorMapDataType type, int rank, const void* base, const uint64_t* dims,
                const uint64_t* strides, const uint32_t* box, CUtensorMapSwizzle swizzle) {
  EncodeTiledFn enc = encode_fn();
  if (!enc || rank < 1 || rank > 5) return false;
  cuuint64_t d[5], s[4];
  cuuint32_t b[5], e[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    e[i] = 1;
    if (i + 1 < rank) s[i] = strides[i];
  }
  return enc(map, type, rank, const_cast<void*>(base), d, s, b, e, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool encode_map_u8(CUtensorMap* map, int rank, const void* base, const uint64_t* dims, const uint64_t* strides,
                   const uint32_t* box, CUtensorMapSwizzle swizzle) {
  return encode_map(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, rank, base, dims, strides, box, swizzle);
}

bool encode_map_u16(CUtensorMap* map, int rank, const void* base, const uint64_t* dims, const uint64_t* strides,
                    const uint32_t* box, CUtensorMapSwizzle swizzle) {
  return encode_map(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, rank, base, dims, strides, box, swizzle);
}

cudaError_t set_max_dyn_smem(const void* func, int bytes) {
  static std::mutex mu;
  static std::unordered_map<const void*, uint64_t> done;   // kernel -> devices (bit per id < 64) already set
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0;
  std::lock_guard<std::mutex> lock(mu);
  uint64_t& mask = done[func];
  if (bit != 0 && (mask & bit) != 0) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) mask |= bit;
  return e;
}

cudaError_t launch_wait_selftest(int timeout_ms, cudaStream_t st, int* err) {
  wait_selftest_kernel<<<1, 32, 0, st>>>(err, static_cast<uint64_t>(timeout_ms) * 1000000ull);
  return cudaGetLastError();
}

}  // namespace qattn

using namespace qattn;

namespace {

// Argument checks of one rotate/quantize call; QATTN_OK also for an empty
// problem (nothing to launch: *empty is set).
qattn_status_t check_rotq(const void* x, qattn_dtype_t x_dtype, qattn_layout_t layout, int B, int H, int N, int D,
                          const float* rot, int block_tokens, qattn_dtype_t code_dtype, const void* codes,
                          const float* scales, bool* empty) {
  *empty = false;
  if (B < 0 || H < 0 || N < 0 || D <= 0 || block_tokens <= 0) return QATTN_ERR_INVALID_ARG;
  if (x_dtype != QATTN_F16 && x_dtype != QATTN_BF16) return QATTN_ERR_INVALID_ARG;
  if (code_dtype != QATTN_INT8 && code_dtype != QATTN_FP8_E4M3 && code_dtype != QATTN_INT4_PACKED)
    return QATTN_ERR_INVALID_ARG;
  if (layout != QATTN_BNSD && layout != QATTN_BSND) return QATTN_ERR_INVALID_ARG;
  if (!rotate_block_quant_supported(D, block_tokens)) return QATTN_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(B) * H * N == 0) {
    *empty = true;
    return QATTN_OK;
  }
  if (!x || !codes || !scales) return QATTN_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(codes) || (rot && !aligned16(rot))) return QATTN_ERR_ALIGNMENT;
  return QATTN_OK;
}

RotQuantArgs rotq_args(const void* x, qattn_dtype_t x_dtype, qattn_layout_t layout, int B, int H, int N, int D,
                       const float* rot, int block_tokens, qattn_dtype_t code_dtype, void* codes, float* scales) {
  RotQuantArgs a;
  a.x = x;
  a.is_bf16 = x_dtype == QATTN_BF16;
  a.layout = layout;
  a.B = B; a.H = H; a.N = N; a.D = D; a.T = block_tokens;
  a.rot = rot;
  a.int8 = code_dtype == QATTN_INT8 || code_dtype == QATTN_INT4_PACKED;
  a.int4 = code_dtype == QATTN_INT4_PACKED;
  a.codes = codes;
  a.scales = scales;
  return a;
}

// Two internal streams and three events per device for
// qattn_rotate_block_quant_qkv, created on first use and kept; `enqueue`
// serialises the calls' enqueueing (they share the streams).
struct QkvStreams {
  bool ready = false;
  cudaStream_t sq = nullptr, sk = nullptr;
  cudaEvent_t fork = nullptr, done_q = nullptr, done_k = nullptr;
  std::mutex enqueue;
};
QkvStreams g_qkv[kMaxDevices];
std::mutex g_qkv_mu;

qattn_status_t qkv_streams(QkvStreams** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_qkv_mu);
  QkvStreams& S = g_qkv[dev];
  if (!S.ready) {
    if (cudaStreamCreateWithFlags(&S.sq, cudaStreamNonBlocking) != cudaSuccess ||
        cudaStreamCreateWithFlags(&S.sk, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&S.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&S.done_q, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&S.done_k, cudaEventDisableTiming) != cudaSuccess)
      return QATTN_ERR_CUDA;
    S.ready = true;
  }
  *out = &S;
  return QATTN_OK;
}

}  // namespace

extern "C" {

int qattn_abi_version(void) { return QATTN_ABI_VERSION; }

const char* qattn_status_string(qattn_status_t s) {
  switch (s) {
    case QATTN_OK: return "ok";
    case QATTN_ERR_INVALID_ARG: return "invalid argument";
    case QATTN_ERR_UNSUPPORTED: return "unsupported configuration";
    case QATTN_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case QATTN_ERR_WORKSPACE: return "workspace missing or too small";
    case QATTN_ERR_CUDA: return "CUDA error";
    case QATTN_ERR_TIMEOUT: return "kernel barrier wait timed out";
  }
  return "unknown status";
}

qattn_status_t qattn_rotate_block_quant(const void* x, qattn_dtype_t x_dtype, qattn_layout_t layout, int B,
                                        int H, int N, int D, const float* rot, int block_tokens,
                                        qattn_dtype_t code_dtype, void* codes, float* scales,
                                        qattn_stream_t stream) {
  bool empty = false;
  const qattn_status_t c = check_rotq(x, x_dtype, layout, B, H, N, D, rot, block_tokens, code_dtype, codes, scales,
                                      &empty);
  if (c != QATTN_OK || empty) return c;
  DeviceState* ds = nullptr;
  qattn_status_t s = device_state(&ds);
  if (s != QATTN_OK) return s;
  const RotQuantArgs a = rotq_args(x, x_dtype, layout, B, H, N, D, rot, block_tokens, code_dtype, codes, scales);
  return from_cuda(launch_rotate_block_quant(a, reinterpret_cast<cudaStream_t>(stream), ds->num_sms, ds->err));
}

qattn_status_t qattn_rotate_block_quant_qkv(const void* q, const void* k, const void* v, qattn_dtype_t x_dtype,
                                            qattn_layout_t layout, int B, int H, int N, int D, const float* rot,
                                            qattn_dtype_t code_dtype, void* q_codes, float* q_scales, void* k_codes,
                                            float* k_scales, void* v_codes, float* v_scales,
                                            qattn_stream_t stream) {
  bool empty = false;
  qattn_status_t c = check_rotq(q, x_dtype, layout, B, H, N, D, rot, 128, code_dtype, q_codes, q_scales, &empty);
  if (c == QATTN_OK) c = check_rotq(k, x_dtype, layout, B, H, N, D, rot, 256, code_dtype, k_codes, k_scales, &empty);
  if (c == QATTN_OK) c = check_rotq(v, x_dtype, layout, B, H, N, D, nullptr, 256, code_dtype, v_codes, v_scales, &empty);
  if (c != QATTN_OK || empty) return c;
  DeviceState* ds = nullptr;
  qattn_status_t s = device_state(&ds);
  if (s != QATTN_OK) return s;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const RotQuantArgs aq = rotq_args(q, x_dtype, layout, B, H, N, D, rot, 128, code_dtype, q_codes, q_scales);
  const RotQuantArgs ak = rotq_args(k, x_dtype, layout, B, H, N, D, rot, 256, code_dtype, k_codes, k_scales);
  const RotQuantArgs av = rotq_args(v, x_dtype, layout, B, H, N, D, nullptr, 256, code_dtype, v_codes, v_scales);
  if (rot == nullptr) {
    // three memory-bound passes: one after the other on the whole GPU
    cudaError_t e = launch_rotate_block_quant(aq, st, ds->num_sms, ds->err);
    if (e == cudaSuccess) e = launch_rotate_block_quant(ak, st, ds->num_sms, ds->err);
    if (e == cudaSuccess) e = launch_rotate_block_quant(av, st, ds->num_sms, ds->err);
    return from_cuda(e);
  }
  QkvStreams* S = nullptr;
  s = qkv_streams(&S);
  if (s != QATTN_OK) return s;
  // The rotations of Q and K (FMA-bound, one persistent CTA per SM) run at
  // the same time on two internal streams, each on half of the SMs; V's
  // memory-bound quantization is enqueued on the caller's stream and takes
  // SMs as they free up. The caller's stream waits for both rotations.
  const int half = ds->num_sms / 2 > 0 ? ds->num_sms / 2 : 1;
  std::lock_guard<std::mutex> lock(S->enqueue);
  cudaError_t e = cudaEventRecord(S->fork, st);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(S->sq, S->fork, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(S->sk, S->fork, 0);
  if (e == cudaSuccess) e = launch_rotate_block_quant(aq, S->sq, half, ds->err);
  if (e == cudaSuccess) e = launch_rotate_block_quant(ak, S->sk, ds->num_sms - half, ds->err);
  if (e == cudaSuccess) e = launch_rotate_block_quant(av, st, ds->num_sms, ds->err);
  if (e == cudaSuccess) e = cudaEventRecord(S->done_q, S->sq);
  if (e == cudaSuccess) e = cudaEventRecord(S->done_k, S->sk);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(st, S->done_q, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(st, S->done_k, 0);
  return from_cuda(e);
}

qattn_status_t qattn_prefill_mixed(const void* q_codes, const float* q_scales, const void* k_codes,
                                   const float* k_scales, const void* v_codes, const float* v_scales,
                                   qattn_dtype_t qk_dtype, qattn_dtype_t v_dtype, qattn_layout_t layout, int B,
                                   int H, int N_q, int N_kv, int D, int q_block, int kv_block, int causal,
                                   float softmax_scale, void* out, float* lse, qattn_stream_t stream) {
  if (B < 0 || H < 0 || N_q < 0 || N_kv < 0 || D <= 0) return QATTN_ERR_INVALID_ARG;
  if (qk_dtype != QATTN_INT8 && qk_dtype != QATTN_FP8_E4M3 && qk_dtype != QATTN_INT4_PACKED)
    return QATTN_ERR_INVALID_ARG;
  if (v_dtype != QATTN_INT8 && v_dtype != QATTN_FP8_E4M3 && v_dtype != QATTN_INT4_PACKED)
    return QATTN_ERR_INVALID_ARG;
  if (layout != QATTN_BNSD && layout != QATTN_BSND) return QATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return QATTN_ERR_INVALID_ARG;
  const int v_code = v_dtype == QATTN_FP8_E4M3 ? 0 : v_dtype == QATTN_INT8 ? 1 : 2;
  const int qk_code = qk_dtype == QATTN_FP8_E4M3 ? 0 : qk_dtype == QATTN_INT8 ? 1 : 2;
  if (!prefill_codes_supported(qk_code, v_code)) return QATTN_ERR_UNSUPPORTED;
  if (causal && N_q != N_kv) return QATTN_ERR_UNSUPPORTED;
  if (q_block != 128 || kv_block != 256) return QATTN_ERR_UNSUPPORTED;
  if (!prefill_supported(D)) return QATTN_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(B) * H * N_q == 0) return QATTN_OK;
  if (N_kv == 0) return QATTN_ERR_UNSUPPORTED;  // softmax over no keys is undefined
  if (!q_codes || !q_scales || !k_codes || !k_scales || !v_codes || !v_scales || !out) return QATTN_ERR_INVALID_ARG;
  if (!aligned16(q_codes) || !aligned16(k_codes) || !aligned16(v_codes) || !aligned16(out))
    return QATTN_ERR_ALIGNMENT;
  if (static_cast<int64_t>(B) * H * ((N_q + 127) / 128) >= (1LL << 31)) return QATTN_ERR_UNSUPPORTED;
  DeviceState* ds = nullptr;
  qattn_status_t s = device_state(&ds);
  if (s != QATTN_OK) return s;
  if (!(softmax_scale > 0.0f)) softmax_scale = 1.0f / sqrtf(static_cast<float>(D));
  PrefillArgs a;
  a.q = q_codes; a.qs = q_scales;
  a.k = k_codes; a.ks = k_scales;
  a.v = v_codes; a.vs = v_scales;
  a.qk_code = qk_code;
  a.v_code = v_code;
  a.layout = layout;
  a.B = B; a.H = H; a.Nq = N_q; a.Nkv = N_kv; a.D = D;
  a.causal = causal;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  a.out = out;
  a.lse = lse;
  return from_cuda(launch_prefill(a, reinterpret_cast<cudaStream_t>(stream), ds->num_sms, ds->err));
}

qattn_status_t qattn_prefill(const void* q_codes, const float* q_scales, const void* k_codes, const float* k_scales,
                             const void* v_codes, const float* v_scales, qattn_dtype_t code_dtype,
                             qattn_layout_t layout, int B, int H, int N_q, int N_kv, int D, int q_block,
                             int kv_block, int causal, float softmax_scale, void* out, float* lse,
                             qattn_stream_t stream) {
  if (code_dtype != QATTN_INT8 && code_dtype != QATTN_FP8_E4M3) return QATTN_ERR_INVALID_ARG;
  return qattn_prefill_mixed(q_codes, q_scales, k_codes, k_scales, v_codes, v_scales, code_dtype, code_dtype,
                             layout, B, H, N_q, N_kv, D, q_block, kv_block, causal, softmax_scale, out, lse,
                             stream);
}

qattn_status_t qattn_widen_int4(const void* packed, int64_t n_packed, void* out, qattn_stream_t stream) {
  if (n_packed < 0) return QATTN_ERR_INVALID_ARG;
  if (n_packed == 0) return QATTN_OK;
  if (!packed || !out) return QATTN_ERR_INVALID_ARG;
  if (!aligned16(packed) || !aligned16(out)) return QATTN_ERR_ALIGNMENT;
  const uintptr_t p0 = reinterpret_cast<uintptr_t>(packed), o0 = reinterpret_cast<uintptr_t>(out);
  const uintptr_t n = static_cast<uintptr_t>(n_packed);
  if (p0 < o0 + 2 * n && o0 < p0 + n) return QATTN_ERR_INVALID_ARG;   // overlapping ranges
  DeviceState* ds = nullptr;
  qattn_status_t s = device_state(&ds);
  if (s != QATTN_OK) return s;
  return from_cuda(launch_widen_int4(packed, n_packed, out, reinterpret_cast<cudaStream_t>(stream), ds->num_sms));
}

qattn_status_t qattn_dequant_bf16(const void* codes, const float* scales, qattn_dtype_t code_dtype,
                                  qattn_layout_t layout, int B, int H, int N, int D, int block_tokens, void* out,
                                  qattn_stream_t stream) {
  if (B < 0 || H < 0 || N < 0 || D <= 0 || block_tokens <= 0) return QATTN_ERR_INVALID_ARG;
  if (code_dtype != QATTN_INT8 && code_dtype != QATTN_FP8_E4M3) return QATTN_ERR_INVALID_ARG;
  if (layout != QATTN_BNSD && layout != QATTN_BSND) return QATTN_ERR_INVALID_ARG;
  if (D % 16) return QATTN_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(B) * H * N == 0) return QATTN_OK;
  if (!codes || !scales || !out) return QATTN_ERR_INVALID_ARG;
  if (!aligned16(codes) || !aligned16(out)) return QATTN_ERR_ALIGNMENT;
  DeviceState* ds = nullptr;
  qattn_status_t s = device_state(&ds);
  if (s != QATTN_OK) return s;
  DequantArgs a;
  a.codes = codes;
  a.scales = scales;
  a.int8 = code_dtype == QATTN_INT8;
  a.layout = layout;
  a.B = B; a.H = H; a.N = N; a.D = D; a.block = block_tokens;
  a.out = out;
  return from_cuda(launch_dequant_bf16(a, reinterpret_cast<cudaStream_t>(stream), ds->num_sms));
}

qattn_status_t qattn_attention_bf16(const void* q, const void* k, const void* v, qattn_layout_t layout, int B, int H,
                                    int N_q, int N_kv, int D, int causal, float softmax_scale, void* out, float* lse,
                                    qattn_stream_t stream) {
  if (B < 0 || H < 0 || N_q < 0 || N_kv < 0 || D <= 0) return QATTN_ERR_INVALID_ARG;
  if (layout != QATTN_BNSD && layout != QATTN_BSND) return QATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return QATTN_ERR_INVALID_ARG;
  if (causal && N_q != N_kv) return QATTN_ERR_UNSUPPORTED;
  if (!attn_bf16_supported(D)) return QATTN_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(B) * H * N_q == 0) return QATTN_OK;
  if (N_kv == 0) return QATTN_ERR_UNSUPPORTED;
  if (!q || !k || !v || !out) return QATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return QATTN_ERR_ALIGNMENT;
  if (static_cast<int64_t>(B) * H * ((N_q + 127) / 128) >= (1LL << 31)) return QATTN_ERR_UNSUPPORTED;
  DeviceState* ds = nullptr;
  qattn_status_t s = device_state(&ds);
  if (s != QATTN_OK) return s;
  if (!(softmax_scale > 0.0f)) softmax_scale = 1.0f / sqrtf(static_cast<float>(D));
  AttnBf16Args a;
  a.q = q; a.k = k; a.v = v;
  a.layout = layout;
  a.B = B; a.H = H; a.Nq = N_q; a.Nkv = N_kv; a.D = D;
  a.causal = causal;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  a.out = out;
  a.lse = lse;
  return from_cuda(launch_attn_bf16(a, reinterpret_cast<cudaStream_t>(stream), ds->err));
}

size_t qattn_decode_workspace_size(int B, int H_q, int H_kv, int L, int D) {
  if (B <= 0 || H_q <= 0 || H_kv <= 0 || L < 0 || D <= 0 || H_q % H_kv) return 0;
  DeviceState* ds = nullptr;
  if (device_state(&ds) != QATTN_OK) return 0;
  return decode_workspace_bytes(B, H_q, H_kv, L, D, ds->num_sms);
}

qattn_status_t qattn_decode_kvq(const void* q, const void* k_cache, const void* v_cache, const void* k_scales,
                                const void* v_scales, qattn_dtype_t kv_dtype, int B, int H_q, int H_kv, int L,
                                int D, int kv_block, int group, float softmax_scale, void* out, void* workspace,
                                size_t workspace_bytes, qattn_stream_t stream) {
  if (B < 0 || H_q <= 0 || H_kv <= 0 || L < 0 || D <= 0) return QATTN_ERR_INVALID_ARG;
  if (H_q % H_kv) return QATTN_ERR_INVALID_ARG;
  if (kv_dtype != QATTN_INT8 && kv_dtype != QATTN_INT4_PACKED) return QATTN_ERR_INVALID_ARG;
  const int G = H_q / H_kv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return QATTN_ERR_UNSUPPORTED;
  int group_ratio = 1;
  if (kv_dtype == QATTN_INT8) {
    if (kv_block != 256) return QATTN_ERR_UNSUPPORTED;
  } else {
    if (group <= 0 || D % group) return QATTN_ERR_INVALID_ARG;
    group_ratio = D / group;
  }
  if (!decode_supported(D, group_ratio)) return QATTN_ERR_UNSUPPORTED;
  if (B == 0) return QATTN_OK;
  if (!q || !out || !workspace) return QATTN_ERR_INVALID_ARG;
  if (L > 0 && (!k_cache || !v_cache || !k_scales || !v_scales)) return QATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(out) || !aligned16(workspace) || (L > 0 && (!aligned16(k_cache) || !aligned16(v_cache))))
    return QATTN_ERR_ALIGNMENT;
  DeviceState* ds = nullptr;
  qattn_status_t s = device_state(&ds);
  if (s != QATTN_OK) return s;
  // (the call's own split count: qattn_decode_workspace_size() is at least this)
  if (workspace_bytes < decode_workspace_bytes_for(B, H_q, H_kv, L, kv_dtype == QATTN_INT4_PACKED, ds->num_sms))
    return QATTN_ERR_WORKSPACE;
  if (!(softmax_scale > 0.0f)) softmax_scale = 1.0f / sqrtf(static_cast<float>(D));
  DecodeArgs a;
  a.q = q; a.k = k_cache; a.v = v_cache; a.ks = k_scales; a.vs = v_scales;
  a.int4 = kv_dtype == QATTN_INT4_PACKED;
  a.B = B; a.Hq = H_q; a.Hkv = H_kv; a.L = L; a.D = D;
  a.kv_block = kv_dtype == QATTN_INT8 ? kv_block : 256;
  a.group = kv_dtype == QATTN_INT4_PACKED ? group : D;
  a.scale = softmax_scale;
  a.out = out;
  a.workspace = workspace;
  return from_cuda(launch_decode(a, reinterpret_cast<cudaStream_t>(stream), ds->num_sms, ds->err));
}

qattn_status_t qattn_kv_append(const void* x_new, int B, int H_kv, int n, int D, qattn_dtype_t kv_dtype, int L,
                               int L_max, void* cache, void* scales, int kv_block, int group,
                               qattn_stream_t stream) {
  if (B < 0 || H_kv < 0 || n < 0 || D <= 0 || L < 0 || L_max < 0) return QATTN_ERR_INVALID_ARG;
  if (kv_dtype != QATTN_INT8 && kv_dtype != QATTN_INT4_PACKED) return QATTN_ERR_INVALID_ARG;
  if (static_cast<int64_t>(L) + n > L_max) return QATTN_ERR_INVALID_ARG;
  const bool int4 = kv_dtype == QATTN_INT4_PACKED;
  if (int4 && (group <= 0 || D % group)) return QATTN_ERR_INVALID_ARG;
  if (!int4 && kv_block <= 0) return QATTN_ERR_INVALID_ARG;
  if (!kv_append_supported(D, int4, kv_block, group)) return QATTN_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(B) * H_kv * n == 0) return QATTN_OK;
  if (!x_new || !cache || !scales) return QATTN_ERR_INVALID_ARG;
  if (!aligned16(x_new) || !aligned16(cache)) return QATTN_ERR_ALIGNMENT;
  if (static_cast<int64_t>(B) * H_kv * n >= (1LL << 31) * 8) return QATTN_ERR_UNSUPPORTED;
  if (B > 65535 || H_kv > 65535 || (int4 && static_cast<int64_t>(B) * H_kv > 65535)) return QATTN_ERR_UNSUPPORTED;
  DeviceState* ds = nullptr;
  qattn_status_t s = device_state(&ds);
  if (s != QATTN_OK) return s;
  KvAppendArgs a;
  a.x = x_new;
  a.int4 = int4;
  a.B = B; a.Hkv = H_kv; a.n = n; a.D = D; a.L = L; a.Lmax = L_max;
  a.kv_block = int4 ? 256 : kv_block;
  a.group = int4 ? group : D;
  a.cache = cache;
  a.scales = scales;
  return from_cuda(launch_kv_append(a, reinterpret_cast<cudaStream_t>(stream)));
}

qattn_status_t qattn_device_error(qattn_stream_t stream) {
  DeviceState* ds = nullptr;
  qattn_status_t s = device_state(&ds);
  if (s != QATTN_OK) return s;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return QATTN_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, ds->err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return QATTN_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpy(ds->err, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return QATTN_ERR_CUDA;
  }
  return static_cast<qattn_status_t>(v);
}

qattn_status_t qattn_selftest_wait_timeout(int timeout_ms, qattn_stream_t stream) {
  if (timeout_ms < 1 || timeout_ms > 2000) return QATTN_ERR_INVALID_ARG;
  DeviceState* ds = nullptr;
  qattn_status_t s = device_state(&ds);
  if (s != QATTN_OK) return s;
  return from_cuda(launch_wait_selftest(timeout_ms, reinterpret_cast<cudaStream_t>(stream), ds->err));
}

}  // extern "C"
