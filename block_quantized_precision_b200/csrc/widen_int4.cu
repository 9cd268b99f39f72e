// widen_int4.cu -- packed INT4 codes to INT8 codes of the same values.
//
// Method: "FlashAttention 的 INT8/INT4 量化", 第二层 (INT4 codes are widened
// to INT8 before the integer matmul); the packing is that of
// "ops-transformer INT8/INT4 量化推理", 5.2 (two signed 4-bit codes per byte,
// element 2i in the low nibble, 2i+1 in the high one).
//
// The code tensors keep their channels consecutive in both layouts, so byte
// i of a packed tensor becomes bytes 2i and 2i+1 of the widened one and the
// whole tensor widens as one flat byte array; the block scales stay as they
// are. On B200 the prefill is bound by instruction issue and this pass by
// HBM (n bytes read, 2n written, the output left in L2 for the kernel that
// follows), so widening here instead of inside the prefill's pipeline takes
// its integer work off the softmax warps' sub-partitions.
#include <cstdint>

#include "qattn_internal.h"

namespace qattn {

namespace {

constexpr int kWidenThreads = 256;

// Four packed bytes -> eight INT8 codes, as two words in element order.
// A nibble n in a byte becomes the byte n | 0xF0 when its sign bit (8) is
// set: (n & 8) * 30 = 0xF0 for each byte, no carry into its neighbour.
__device__ __forceinline__ uint2 widen4(uint32_t w) {
  uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
  lo |= (lo & 0x08080808u) * 30u;
  hi |= (hi & 0x08080808u) * 30u;
  // bytes (lo0 hi0 lo1 hi1) and (lo2 hi2 lo3 hi3)
  return make_uint2(__byte_perm(lo, hi, 0x5140), __byte_perm(lo, hi, 0x7362));
}

__device__ __forceinline__ uint32_t widen1(uint8_t b) {
  const uint32_t lo = b & 0xFu, hi = b >> 4;
  return (lo | ((lo & 8u) * 30u)) | ((hi | ((hi & 8u) * 30u)) << 8);
}

// Two 16-byte packed vectors per thread and iteration (32 bytes in flight),
// four 16-byte stores; a byte tail (n not a multiple of 16) one per thread.
__global__ void __launch_bounds__(kWidenThreads)
    widen_int4_kernel(const uint8_t* __restrict__ in, int64_t n, uint8_t* __restrict__ out) {
  const int64_t n16 = n / 16;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kWidenThreads;
  const uint4* src = reinterpret_cast<const uint4*>(in);
  uint4* dst = reinterpret_cast<uint4*>(out);
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kWidenThreads + threadIdx.x; i < n16; i += 2 * stride) {
    const bool two = i + stride < n16;
    const uint4 a = __ldcs(src + i);
    const uint4 b = two ? __ldcs(src + i + stride) : make_uint4(0, 0, 0, 0);
    uint2 w0 = widen4(a.x), w1 = widen4(a.y), w2 = widen4(a.z), w3 = widen4(a.w);
    dst[2 * i] = make_uint4(w0.x, w0.y, w1.x, w1.y);
    dst[2 * i + 1] = make_uint4(w2.x, w2.y, w3.x, w3.y);
    if (two) {
      w0 = widen4(b.x); w1 = widen4(b.y); w2 = widen4(b.z); w3 = widen4(b.w);
      dst[2 * (i + stride)] = make_uint4(w0.x, w0.y, w1.x, w1.y);
      dst[2 * (i + stride) + 1] = make_uint4(w2.x, w2.y, w3.x, w3.y);
    }
  }
  if (blockIdx.x == 0) {
    for (int64_t j = n16 * 16 + threadIdx.x; j < n; j += kWidenThreads) {
      const uint32_t v = widen1(in[j]);
      out[2 * j] = static_cast<uint8_t>(v & 0xFFu);
      out[2 * j + 1] = static_cast<uint8_t>(v >> 8);
    }
  }
}

}  // namespace

cudaError_t launch_widen_int4(const void* packed, int64_t n, void* out, cudaStream_t st, int num_sms) {
  if (n <= 0) return cudaSuccess;
  const int64_t n16 = n / 16;
  // grid: 8 CTAs of 256 threads per SM at most, each thread two vectors per pass
  const int64_t want = (n16 + 2 * kWidenThreads - 1) / (2 * kWidenThreads);
  const int64_t cap = 8LL * num_sms;
  const unsigned grid = static_cast<unsigned>(want < 1 ? 1 : (want < cap ? want : cap));
  widen_int4_kernel<<<grid, kWidenThreads, 0, st>>>(static_cast<const uint8_t*>(packed), n,
                                                     static_cast<uint8_t*>(out));
  return cudaGetLastError();
}

}  // namespace qattn
