// qattn_internal.h -- launcher interfaces between the C ABI (qattn_abi.cu)
// and the kernel files. Arguments arrive here already validated.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace qattn {

// Encodes a TMA tensor map over 8-bit data (no interleave, zero fill out of
// bounds) through the driver entry point; false if that fails. dims[0] is the
// contiguous dimension; strides (bytes) are given for dims 1..rank-1.
bool encode_map_u8(CUtensorMap* map, int rank, const void* base, const uint64_t* dims,
                   const uint64_t* strides, const uint32_t* box, CUtensorMapSwizzle swizzle);
// The same over 16-bit data.
bool encode_map_u16(CUtensorMap* map, int rank, const void* base, const uint64_t* dims,
                    const uint64_t* strides, const uint32_t* box, CUtensorMapSwizzle swizzle);

struct RotQuantArgs {
  const void* x;      // F16/BF16 bits
  int is_bf16;
  int layout;         // 0 = BNSD, 1 = BSND
  int B, H, N, D, T;  // T = block tokens
  const float* rot;   // D x D or nullptr
  int int8;           // 1: INT8 codes, 0: e4m3
  int int4;           // 1: packed INT4 codes (with int8 = 1)
  void* codes;
  float* scales;
};

bool rotate_block_quant_supported(int D, int T);
// err: the library's device error word (timeouts of the pipelined quantizer).
cudaError_t launch_rotate_block_quant(const RotQuantArgs& a, cudaStream_t st, int num_sms, int* err);

struct PrefillArgs {
  const void* q;
  const float* qs;
  const void* k;
  const float* ks;
  const void* v;
  const float* vs;
  int qk_code;        // Q/K codes: 0 e4m3, 1 INT8, 2 packed INT4 (two per byte)
  int v_code;         // V codes: 0 e4m3, 1 INT8, 2 packed INT4
  int layout;
  int B, H, Nq, Nkv, D;
  int causal;
  float scale_log2;   // softmax_scale * log2(e)
  void* out;          // bf16
  float* lse;         // nullable
};

bool prefill_supported(int D);
bool prefill_codes_supported(int qk_code, int v_code);
cudaError_t launch_prefill(const PrefillArgs& a, cudaStream_t st, int num_sms, int* err);

// Packed INT4 codes (n bytes) to INT8 codes (2n bytes), element order kept
// (widen_int4.cu).
cudaError_t launch_widen_int4(const void* packed, int64_t n, void* out, cudaStream_t st, int num_sms);

// The dequantize-first comparison path (prefill_bf16.cu).
struct DequantArgs {
  const void* codes;  // INT8 or e4m3, 1 byte per element, layout as the input
  const float* scales;
  int int8;           // 1: INT8 codes, 0: e4m3
  int layout;
  int B, H, N, D, block;
  void* out;          // bf16, same layout
};

struct AttnBf16Args {
  const void* q;      // bf16
  const void* k;
  const void* v;
  int layout;
  int B, H, Nq, Nkv, D;
  int causal;
  float scale_log2;
  void* out;          // bf16
  float* lse;         // nullable
};

bool attn_bf16_supported(int D);
cudaError_t launch_attn_bf16(const AttnBf16Args& a, cudaStream_t st, int* err);
cudaError_t launch_dequant_bf16(const DequantArgs& a, cudaStream_t st, int num_sms);

struct DecodeArgs {
  const void* q;      // bf16 [B, Hq, 1, D]
  const void* k;
  const void* v;
  const void* ks;
  const void* vs;
  int int4;           // 1: packed INT4 cache, 0: INT8 cache
  int B, Hq, Hkv, L, D;
  int kv_block, group;
  float scale;        // softmax scale
  void* out;          // bf16 [B, Hq, 1, D]
  void* workspace;
};

bool decode_supported(int D, int group_size_ratio);
int decode_splits(int B, int Hkv, int L, int num_sms);
size_t decode_workspace_bytes(int B, int Hq, int Hkv, int L, int D, int num_sms);
// The bytes one call of the given cache type writes (its own split count);
// at most decode_workspace_bytes().
size_t decode_workspace_bytes_for(int B, int Hq, int Hkv, int L, bool int4, int num_sms);
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t st, int num_sms, int* err);

struct KvAppendArgs {
  const void* x;      // bf16 [B, H_kv, n, D]
  int int4;           // 1: packed INT4 cache, 0: INT8 cache
  int B, Hkv, n, D, L, Lmax;
  int kv_block, group;
  void* cache;
  void* scales;
};

bool kv_append_supported(int D, bool int4, int kv_block, int group);
cudaError_t launch_kv_append(const KvAppendArgs& a, cudaStream_t st);

cudaError_t launch_wait_selftest(int timeout_ms, cudaStream_t st, int* err);

// Sets kernel `func`'s dynamic shared-memory limit on the current device the
// first time it is asked for there (the attribute stays set for the life of
// the context), so that launches do not repeat the runtime call.
cudaError_t set_max_dyn_smem(const void* func, int bytes);

}  // namespace qattn
