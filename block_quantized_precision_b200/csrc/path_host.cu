// path_host.cu -- qattn_attention_path_host: the prefill path (rotate and
// quantize Q/K, quantize V, attention on the codes) from host buffers, with
// the host<->device copies of one group of heads overlapped with the
// compute of another.
//
// Path: "MindIE-SD quantization", FA量化 (rotation of Q and K, dynamic block
// quantization, attention in the low-precision domain, output returned in
// the original precision). The compute of every group is the four public
// device calls on a sub-problem of whole (b, h) heads, so the results are
// those of the device calls on the whole problem: the method works head by
// head (every block, scale and softmax row lies within one head).
//
// Schedule (groups g = 0, 1, ...; slot = g % 2 of the workspace):
//   copy-in stream:  [wait compute(g-2)] copy q, k, v of g -> slot   (ev_in[g])
//   compute stream:  [wait ev_in[g], copy-out(g-2)] rotate/quantize Q, K,
//                    quantize V, prefill                             (ev_comp[g])
//   copy-out stream: [wait ev_comp[g]] copy out of g -> host         (ev_out[g])
// and the compute stream finally waits for the last copy-out (the copy-out
// stream runs in order).
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "../../include/qattn.h"
#include "qattn_internal.h"

namespace qattn {
namespace {

constexpr int kMaxGroups = 64;
constexpr int kDefaultGroups = 8;
constexpr int kMaxDev = 64;
constexpr size_t kAlign = 256;

// One group: the sub-problem [Bp, Hp, N, D] (or [Bp, N, Hp, D]) whose first
// element is `off` elements into the full tensors. Strided groups (BSND,
// part of the heads of one b) are N rows of Hp * D elements, H * D apart.
struct Group {
  int64_t off;
  int Bp, Hp;
  bool strided;
};

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

int clamp_groups(int groups) { return groups <= 0 ? kDefaultGroups : std::min(groups, kMaxGroups); }

std::vector<Group> plan(int B, int H, int N, int D, qattn_layout_t layout, int groups) {
  std::vector<Group> out;
  const int G = clamp_groups(groups);
  const int64_t units = static_cast<int64_t>(B) * H;
  if (units == 0) return out;
  if (layout == QATTN_BNSD) {
    // consecutive (b, h) heads are consecutive [N, D] slabs
    const int64_t per = cdiv(units, std::min<int64_t>(G, units));
    for (int64_t u0 = 0; u0 < units; u0 += per) {
      const int64_t n = std::min(per, units - u0);
      out.push_back({u0 * N * D, 1, static_cast<int>(n), false});
    }
  } else if (G <= B) {
    // whole b's: consecutive [N, H, D] slabs
    const int per = static_cast<int>(cdiv(B, G));
    for (int b0 = 0; b0 < B; b0 += per)
      out.push_back({static_cast<int64_t>(b0) * N * H * D, std::min(per, B - b0), H, false});
  } else {
    // ranges of heads within each b
    const int hg = static_cast<int>(std::min<int64_t>(cdiv(G, B), H));
    const int per = static_cast<int>(cdiv(H, hg));
    for (int b = 0; b < B; ++b)
      for (int h0 = 0; h0 < H; h0 += per)
        out.push_back({(static_cast<int64_t>(b) * N * H + h0) * D, 1, std::min(per, H - h0), per < H});
  }
  return out;
}

// Byte offsets of the buffers of one workspace slot.
struct Slot {
  size_t xq, xk, xv, qc, kc, vc, qs, ks, vs, out, bytes;
};

size_t up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

Slot slot_layout(const std::vector<Group>& gs, int N, int D) {
  int64_t heads = 0;
  for (const Group& g : gs) heads = std::max<int64_t>(heads, static_cast<int64_t>(g.Bp) * g.Hp);
  const size_t e = static_cast<size_t>(heads) * N * D;      // elements of one tensor of the largest group
  const size_t nqb = static_cast<size_t>(cdiv(N, 128)), nkb = static_cast<size_t>(cdiv(N, 256));
  Slot s;
  size_t o = 0;
  s.xq = o; o += up(2 * e);
  s.xk = o; o += up(2 * e);
  s.xv = o; o += up(2 * e);
  s.qc = o; o += up(e);
  s.kc = o; o += up(e);
  s.vc = o; o += up(e);
  s.qs = o; o += up(sizeof(float) * heads * nqb);
  s.ks = o; o += up(sizeof(float) * heads * nkb);
  s.vs = o; o += up(sizeof(float) * heads * nkb);
  s.out = o; o += up(2 * e);
  s.bytes = o;
  return s;
}

// Per-device copy streams and events, created on first use and kept for
// the life of the process.
struct Pool {
  bool ready = false;
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr;
  cudaEvent_t ev_in[kMaxGroups], ev_comp[kMaxGroups], ev_out[kMaxGroups];
  std::mutex enqueue;
};

Pool g_pool[kMaxDev];
std::mutex g_pool_mu;

qattn_status_t pool(Pool** p) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return QATTN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_pool_mu);
  Pool& P = g_pool[dev];
  if (!P.ready) {
    if (cudaStreamCreateWithFlags(&P.in, cudaStreamNonBlocking) != cudaSuccess) return QATTN_ERR_CUDA;
    if (cudaStreamCreateWithFlags(&P.out, cudaStreamNonBlocking) != cudaSuccess) return QATTN_ERR_CUDA;
    if (cudaEventCreateWithFlags(&P.start, cudaEventDisableTiming) != cudaSuccess) return QATTN_ERR_CUDA;
    for (int i = 0; i < kMaxGroups; ++i) {
      if (cudaEventCreateWithFlags(&P.ev_in[i], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&P.ev_comp[i], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&P.ev_out[i], cudaEventDisableTiming) != cudaSuccess)
        return QATTN_ERR_CUDA;
    }
    P.ready = true;
  }
  *p = &P;
  return QATTN_OK;
}

// Copies one group of one tensor (elements of `esize` bytes) between the
// full host tensor and a dense device buffer.
cudaError_t copy_group(const Group& g, int N, int H, int D, size_t esize, void* dst, const void* src, bool to_device,
                       cudaStream_t st) {
  const cudaMemcpyKind kind = to_device ? cudaMemcpyHostToDevice : cudaMemcpyDeviceToHost;
  const size_t bytes = static_cast<size_t>(g.Bp) * g.Hp * N * D * esize;
  const size_t host_off = static_cast<size_t>(g.off) * esize;
  if (!g.strided) {
    return to_device ? cudaMemcpyAsync(dst, static_cast<const char*>(src) + host_off, bytes, kind, st)
                     : cudaMemcpyAsync(static_cast<char*>(dst) + host_off, src, bytes, kind, st);
  }
  const size_t width = static_cast<size_t>(g.Hp) * D * esize;      // one token row of the group
  const size_t host_pitch = static_cast<size_t>(H) * D * esize;
  return to_device ? cudaMemcpy2DAsync(dst, width, static_cast<const char*>(src) + host_off, host_pitch, width, N,
                                       kind, st)
                   : cudaMemcpy2DAsync(static_cast<char*>(dst) + host_off, host_pitch, src, width, width, N, kind,
                                       st);
}

}  // namespace
}  // namespace qattn

using namespace qattn;

extern "C" {

size_t qattn_attention_path_host_workspace_size(int B, int H, int N, int D, qattn_layout_t layout, int groups) {
  if (B <= 0 || H <= 0 || N <= 0 || D <= 0 || (layout != QATTN_BNSD && layout != QATTN_BSND)) return 0;
  const std::vector<Group> gs = plan(B, H, N, D, layout, groups);
  return 2 * slot_layout(gs, N, D).bytes;
}

qattn_status_t qattn_attention_path_host(const void* q, const void* k, const void* v, qattn_dtype_t x_dtype,
                                         qattn_layout_t layout, int B, int H, int N, int D, const float* rot,
                                         qattn_dtype_t code_dtype, int causal, float softmax_scale, void* out,
                                         int groups, void* workspace, size_t workspace_bytes,
                                         qattn_stream_t stream) {
  // the checks of the device calls, for the whole problem, before anything is enqueued
  if (B < 0 || H < 0 || N < 0 || D <= 0 || groups < 0) return QATTN_ERR_INVALID_ARG;
  if (x_dtype != QATTN_F16 && x_dtype != QATTN_BF16) return QATTN_ERR_INVALID_ARG;
  if (code_dtype != QATTN_INT8 && code_dtype != QATTN_FP8_E4M3) return QATTN_ERR_INVALID_ARG;
  if (layout != QATTN_BNSD && layout != QATTN_BSND) return QATTN_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return QATTN_ERR_INVALID_ARG;
  if (!rotate_block_quant_supported(D, 128) || !rotate_block_quant_supported(D, 256) || !prefill_supported(D))
    return QATTN_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(B) * H * N == 0) return QATTN_OK;
  if (!q || !k || !v || !out) return QATTN_ERR_INVALID_ARG;
  if (rot && (reinterpret_cast<uintptr_t>(rot) & 15u) != 0) return QATTN_ERR_ALIGNMENT;
  if (static_cast<int64_t>(B) * H * ((N + 127) / 128) >= (1LL << 31)) return QATTN_ERR_UNSUPPORTED;
  const std::vector<Group> gs = plan(B, H, N, D, layout, groups);
  const Slot sl = slot_layout(gs, N, D);
  if (!workspace || workspace_bytes < 2 * sl.bytes) return QATTN_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0) return QATTN_ERR_ALIGNMENT;
  Pool* P = nullptr;
  qattn_status_t s = pool(&P);
  if (s != QATTN_OK) return s;

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lock(P->enqueue);
  auto ok = [](cudaError_t e) { return e == cudaSuccess; };
  // On a failure after the first copy was enqueued, the copies already on
  // the internal streams finish before the error is returned, so none of
  // them touches the caller's buffers afterwards.
  auto fail = [&](qattn_status_t status) {
    cudaStreamSynchronize(P->in);
    cudaStreamSynchronize(P->out);
    return status;
  };
  // the copies start after the work already on `stream` (earlier users of
  // the workspace and of the host buffers)
  if (!ok(cudaEventRecord(P->start, st)) || !ok(cudaStreamWaitEvent(P->in, P->start, 0)) ||
      !ok(cudaStreamWaitEvent(P->out, P->start, 0)))
    return QATTN_ERR_CUDA;
  const size_t es = 2;   // bytes per input / output element
  for (size_t gi = 0; gi < gs.size(); ++gi) {
    const Group& g = gs[gi];
    const int e = static_cast<int>(gi % kMaxGroups);
    char* base = static_cast<char*>(workspace) + (gi % 2) * sl.bytes;
    if (gi >= 2) {
      const int e2 = static_cast<int>((gi - 2) % kMaxGroups);
      if (!ok(cudaStreamWaitEvent(P->in, P->ev_comp[e2], 0))) return fail(QATTN_ERR_CUDA);   // slot inputs consumed
    }
    if (!ok(copy_group(g, N, H, D, es, base + sl.xq, q, true, P->in)) ||
        !ok(copy_group(g, N, H, D, es, base + sl.xk, k, true, P->in)) ||
        !ok(copy_group(g, N, H, D, es, base + sl.xv, v, true, P->in)) ||
        !ok(cudaEventRecord(P->ev_in[e], P->in)) || !ok(cudaStreamWaitEvent(st, P->ev_in[e], 0)))
      return fail(QATTN_ERR_CUDA);
    if (gi >= 2) {
      const int e2 = static_cast<int>((gi - 2) % kMaxGroups);
      if (!ok(cudaStreamWaitEvent(st, P->ev_out[e2], 0))) return fail(QATTN_ERR_CUDA);       // slot output copied out
    }
    float* qs = reinterpret_cast<float*>(base + sl.qs);
    float* ks = reinterpret_cast<float*>(base + sl.ks);
    float* vs = reinterpret_cast<float*>(base + sl.vs);
    s = qattn_rotate_block_quant(base + sl.xq, x_dtype, layout, g.Bp, g.Hp, N, D, rot, 128, code_dtype,
                                 base + sl.qc, qs, stream);
    if (s == QATTN_OK)
      s = qattn_rotate_block_quant(base + sl.xk, x_dtype, layout, g.Bp, g.Hp, N, D, rot, 256, code_dtype,
                                   base + sl.kc, ks, stream);
    if (s == QATTN_OK)
      s = qattn_rotate_block_quant(base + sl.xv, x_dtype, layout, g.Bp, g.Hp, N, D, nullptr, 256, code_dtype,
                                   base + sl.vc, vs, stream);
    if (s == QATTN_OK)
      s = qattn_prefill(base + sl.qc, qs, base + sl.kc, ks, base + sl.vc, vs, code_dtype, layout, g.Bp, g.Hp, N, N,
                        D, 128, 256, causal, softmax_scale, base + sl.out, nullptr, stream);
    if (s != QATTN_OK) return fail(s);
    if (!ok(cudaEventRecord(P->ev_comp[e], st)) || !ok(cudaStreamWaitEvent(P->out, P->ev_comp[e], 0)) ||
        !ok(copy_group(g, N, H, D, es, out, base + sl.out, false, P->out)) ||
        !ok(cudaEventRecord(P->ev_out[e], P->out)))
      return fail(QATTN_ERR_CUDA);
  }
  const int last = static_cast<int>((gs.size() - 1) % kMaxGroups);
  return ok(cudaStreamWaitEvent(st, P->ev_out[last], 0)) ? QATTN_OK : fail(QATTN_ERR_CUDA);
}

}  // extern "C"
