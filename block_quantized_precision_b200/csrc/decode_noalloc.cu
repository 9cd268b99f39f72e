// decode_noalloc.cu -- qattn_decode_kvq_noalloc: the split-KV decode step
// with its scratch in a fixed device array owned by this library, for
// callers that cannot hand over a workspace.
//
// Who needs it: a caller whose device memory is entirely reserved up front
// (for example for the KV cache) by an allocator it does not control, a
// caller that must not call cudaMalloc/cudaFree on its decode loop because
// those calls can synchronise the whole device and stall other streams, or a
// host program that embeds this library without any device allocator of its
// own. Such a caller still owns the inputs and the output; only the split
// partials live here.
//
// The scratch is a file-scope __device__ array of kNoAllocScratchBytes
// bytes; every GPU that loads the library keeps it until the process exits.
// In host code the array's name only stands for it, so its device address is
// looked up once per device (with that device current) and passed to the
// kernels as an ordinary pointer. The address is kept for the life of the
// process: a cudaDeviceReset() on that device would leave it stale.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/qattn.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

void* g_scratch_ptr[kMaxDevices];
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device, looked up on
// the first call for that device. Returns QATTN_ERR_CUDA if the lookup fails.
qattn_status_t scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return QATTN_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return QATTN_OK;
}

}  // namespace

extern "C" {

qattn_status_t qattn_decode_kvq_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                        const void* k_scales, const void* v_scales, qattn_dtype_t kv_dtype, int B,
                                        int H_q, int H_kv, int L, int D, int kv_block, int group,
                                        float softmax_scale, void* out, qattn_stream_t stream) {
  void* scratch = nullptr;
  const qattn_status_t s = scratch_address(&scratch);
  if (s != QATTN_OK) return s;
  // Same validation and kernels as qattn_decode_kvq; a call whose own
  // partials do not fit the fixed array is refused there with
  // QATTN_ERR_WORKSPACE before anything is launched. The partials of every
  // split are written before they are read, so nothing needs clearing.
  return qattn_decode_kvq(q, k_cache, v_cache, k_scales, v_scales, kv_dtype, B, H_q, H_kv, L, D, kv_block, group,
                          softmax_scale, out, scratch, kNoAllocScratchBytes, stream);
}

}  // extern "C"
