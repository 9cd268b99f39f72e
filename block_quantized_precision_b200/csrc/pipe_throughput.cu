// pipe_throughput.cu -- issue throughput of the instructions the kernels of
// this library lean on, per SM and clock, on the GPU it runs on. The FP32
// FMA figure is the peak of the rotation's roofline ("alu" in bench.py);
// the others explain where the softmax of the prefill spends its issue slots
// (exponentials and e4m3 conversions on the transcendental unit, integer
// maxima and byte permutes on the integer pipe).
//
// Each kernel runs independent chains (8 or 16 per thread, no dependence
// between them within an iteration) on 8 CTAs of 256 threads per SM, so the
// figure is the unit's throughput, not its latency. Warp instructions per
// clock per SM use the SM clock given on the command line (MHz, default
// 1965) -- compare runs at the same clock.
#include <cuda_runtime.h>

#include <cstdio>
#include <cstdlib>

namespace {

constexpr int kChains = 8;

__global__ void k_ffma(float* out, int iters, float a) {
  float x[16];
  for (int i = 0; i < 16; ++i) x[i] = threadIdx.x * 0.001f + i;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < 16; ++i) x[i] = fmaf(x[i], a, 0.5f);
  }
  float s = 0.0f;
  for (int i = 0; i < 16; ++i) s += x[i];
  out[blockIdx.x * blockDim.x + threadIdx.x] = s;
}

__global__ void k_ffma2(float* out, int iters, float a) {
  float2 x[kChains];
  for (int i = 0; i < kChains; ++i) x[i] = make_float2(threadIdx.x * 0.001f + i, i + 0.5f);
  const float2 a2 = make_float2(a, a), h = make_float2(0.5f, 0.5f);
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < kChains; ++i) x[i] = __ffma2_rn(x[i], a2, h);
  }
  float s = 0.0f;
  for (int i = 0; i < kChains; ++i) s += x[i].x + x[i].y;
  out[blockIdx.x * blockDim.x + threadIdx.x] = s;
}

__global__ void k_ex2(float* out, int iters, float a) {
  float x[kChains];
  for (int i = 0; i < kChains; ++i) x[i] = threadIdx.x * 1e-6f - i * 0.01f;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < kChains; ++i) {
      float y;
      asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x[i]));
      x[i] = y * a - 1.0f;
    }
  }
  float s = 0.0f;
  for (int i = 0; i < kChains; ++i) s += x[i];
  out[blockIdx.x * blockDim.x + threadIdx.x] = s;
}

__global__ void k_e4m3(float* out, int iters, float a) {
  float x[kChains];
  unsigned acc = 0;
  for (int i = 0; i < kChains; ++i) x[i] = threadIdx.x * 1e-3f + i * 0.1f;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < kChains; ++i) {
      unsigned short r;
      asm volatile("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(x[i]), "f"(x[(i + 1) % kChains]));
      acc += r;
    }
  }
  out[blockIdx.x * blockDim.x + threadIdx.x] = static_cast<float>(acc) * a;
}

__global__ void k_i2f(float* out, int iters, float) {
  int x[kChains];
  for (int i = 0; i < kChains; ++i) x[i] = threadIdx.x * 7 + i;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < kChains; ++i) {
      float f;
      asm volatile("cvt.rn.f32.s32 %0, %1;" : "=f"(f) : "r"(x[i]));
      x[i] ^= __float_as_int(f);
    }
  }
  int s = 0;
  for (int i = 0; i < kChains; ++i) s += x[i];
  out[blockIdx.x * blockDim.x + threadIdx.x] = static_cast<float>(s);
}

__global__ void k_imnmx(float* out, int iters, float) {
  int x[kChains];
  const int y = threadIdx.x;
  for (int i = 0; i < kChains; ++i) x[i] = threadIdx.x * 7 + i;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < kChains; ++i) asm volatile("max.s32 %0, %0, %1;" : "+r"(x[i]) : "r"(y + it));
  }
  int s = 0;
  for (int i = 0; i < kChains; ++i) s += x[i];
  out[blockIdx.x * blockDim.x + threadIdx.x] = static_cast<float>(s);
}

__global__ void k_prmt(float* out, int iters, float) {
  unsigned x[kChains];
  const unsigned y = threadIdx.x * 0x01010101u;
  for (int i = 0; i < kChains; ++i) x[i] = threadIdx.x * 7 + i;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < kChains; ++i) asm volatile("prmt.b32 %0, %0, %1, 0x5140;" : "+r"(x[i]) : "r"(y));
  }
  unsigned s = 0;
  for (int i = 0; i < kChains; ++i) s += x[i];
  out[blockIdx.x * blockDim.x + threadIdx.x] = static_cast<float>(s);
}

__global__ void k_fadd(float* out, int iters, float) {
  float x[kChains];
  for (int i = 0; i < kChains; ++i) x[i] = threadIdx.x * 0.5f + i;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < kChains; ++i) asm volatile("add.rn.f32 %0, %0, 0f3F000000;" : "+f"(x[i]));
  }
  float s = 0.0f;
  for (int i = 0; i < kChains; ++i) s += x[i];
  out[blockIdx.x * blockDim.x + threadIdx.x] = s;
}

typedef void (*Kernel)(float*, int, float);

}  // namespace

int main(int argc, char** argv) {
  const double mhz = argc > 1 ? atof(argv[1]) : 1965.0;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0) != cudaSuccess) return 1;
  float* out = nullptr;
  if (cudaMalloc(&out, static_cast<size_t>(sms) * 8 * 256 * sizeof(float)) != cudaSuccess) return 1;
  cudaEvent_t e0, e1;
  cudaEventCreate(&e0);
  cudaEventCreate(&e1);
  const int iters = 4096, blocks = sms * 8, threads = 256;
  struct Case {
    const char* name;
    Kernel k;
    int per_iter;      // warp instructions per thread per iteration
    int lanes_ops;     // operations per lane per instruction
  } cases[] = {
      {"FFMA (fma.rn.f32)", k_ffma, 16, 1},      {"FFMA2 (fma.rn.f32x2)", k_ffma2, kChains, 2},
      {"MUFU ex2.approx.f32 (+1 FFMA each)", k_ex2, kChains, 1},
      {"cvt.rn.satfinite.e4m3x2.f32", k_e4m3, kChains, 2},
      {"cvt.rn.f32.s32", k_i2f, kChains, 1},     {"max.s32", k_imnmx, kChains, 1},
      {"prmt.b32", k_prmt, kChains, 1},          {"add.rn.f32", k_fadd, kChains, 1},
  };
  printf("%-38s %10s %22s %18s\n", "instruction", "ms", "warp-instr/clk/SM", "ops/clk/SM");
  for (int rep = 0; rep < 2; ++rep) {
    for (const Case& c : cases) {
      float ms = 0.0f;
      cudaEventRecord(e0);
      c.k<<<blocks, threads>>>(out, iters, 0.999f);
      cudaEventRecord(e1);
      cudaEventSynchronize(e1);
      cudaEventElapsedTime(&ms, e0, e1);
      const double warp_instr = 1.0 * blocks * threads / 32 * iters * c.per_iter;
      const double per_clk = warp_instr / (ms * 1e-3) / sms / (mhz * 1e6);
      if (rep == 1) printf("%-38s %10.3f %22.2f %18.1f\n", c.name, ms, per_clk, per_clk * 32 * c.lanes_ops);
    }
  }
  const cudaError_t err = cudaGetLastError();
  printf("status: %s\n", cudaGetErrorString(err));
  cudaFree(out);
  return err != cudaSuccess;
}
