// throughput.cu -- instruction-throughput microbenchmark for sm_100a
// (libmambamicro.so).  It measures how many FP32 fused multiply-adds (scalar
// fma.rn.f32 and packed fma.rn.f32x2) and special-function operations
// (ex2.approx, lg2.approx, rcp.approx) one B200 retires per second, the rates
// that bound the selective-scan kernels' arithmetic.  Every thread runs eight
// independent dependency chains so that each pipe stays busy; the grid fills
// every SM to its thread limit.  Not part of the scan library.
#include <cuda_runtime.h>
#include <stdint.h>

#define MICRO_API extern "C" __attribute__((visibility("default")))

namespace {

constexpr int kChains = 8;
constexpr int kThreads = 256;

enum Kind { FFMA = 0, FMA_F32X2 = 1, EX2 = 2, LG2 = 3, RCP = 4, NKINDS = 5 };

__device__ __forceinline__ float op_ex2(float x) {
  float y;
  asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(-x));
  return y;
}
__device__ __forceinline__ float op_lg2(float x) {
  float y;
  asm volatile("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(fabsf(x)));
  return -y;
}
__device__ __forceinline__ float op_rcp(float x) {
  // 1 / (1 + |x|) stays in (0, 1]: the chain cannot fold two reciprocals
  // into the identity (the add runs on the FMA pipe beside the MUFU one)
  float y;
  asm volatile("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(1.f + fabsf(x)));
  return y;
}

template <int KIND>
__global__ void __launch_bounds__(kThreads) micro_kernel(float *out, int iters, float seed) {
  float v[kChains];
  const float a = seed * 0.999f, b = seed * 1e-3f;
#pragma unroll
  for (int c = 0; c < kChains; ++c) v[c] = seed + 0.01f * float(threadIdx.x + c);
  if constexpr (KIND == FMA_F32X2) {
    unsigned long long p[kChains], pa, pb;
    asm("mov.b64 %0, {%1, %2};" : "=l"(pa) : "f"(a), "f"(a));
    asm("mov.b64 %0, {%1, %2};" : "=l"(pb) : "f"(b), "f"(b));
#pragma unroll
    for (int c = 0; c < kChains; ++c) asm("mov.b64 %0, {%1, %2};" : "=l"(p[c]) : "f"(v[c]), "f"(-v[c]));
    for (int i = 0; i < iters; ++i) {
#pragma unroll
      for (int c = 0; c < kChains; ++c)
        asm volatile("fma.rn.f32x2 %0, %0, %1, %2;" : "+l"(p[c]) : "l"(pa), "l"(pb));
    }
#pragma unroll
    for (int c = 0; c < kChains; ++c) {
      float lo, hi;
      asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(p[c]));
      v[c] = lo + hi;
    }
  } else {
    for (int i = 0; i < iters; ++i) {
#pragma unroll
      for (int c = 0; c < kChains; ++c) {
        if constexpr (KIND == FFMA) {
          asm volatile("fma.rn.f32 %0, %0, %1, %2;" : "+f"(v[c]) : "f"(a), "f"(b));
        } else if constexpr (KIND == EX2) {
          v[c] = op_ex2(v[c]);
        } else if constexpr (KIND == LG2) {
          v[c] = op_lg2(v[c]);
        } else {
          v[c] = op_rcp(v[c]);
        }
      }
    }
  }
  float s = 0.f;
#pragma unroll
  for (int c = 0; c < kChains; ++c) s += v[c];
  // Written only for an impossible value, so the chains cannot be removed.
  if (s == 1234.5678f) out[blockIdx.x * kThreads + threadIdx.x] = s;
}

template <int KIND>
cudaError_t launch(int grid, float *out, int iters, float seed, cudaStream_t st) {
  micro_kernel<KIND><<<grid, kThreads, 0, st>>>(out, iters, seed);
  return cudaGetLastError();
}

cudaError_t launch_kind(int kind, int grid, float *out, int iters, float seed, cudaStream_t st) {
  switch (kind) {
    case FFMA: return launch<FFMA>(grid, out, iters, seed, st);
    case FMA_F32X2: return launch<FMA_F32X2>(grid, out, iters, seed, st);
    case EX2: return launch<EX2>(grid, out, iters, seed, st);
    case LG2: return launch<LG2>(grid, out, iters, seed, st);
    case RCP: return launch<RCP>(grid, out, iters, seed, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

// Runs operation `kind` (0 fma.rn.f32, 1 fma.rn.f32x2, 2 ex2.approx, 3
// lg2.approx, 4 rcp.approx) with `iters` iterations of 8 chains per thread on
// blocks_per_sm x SMs blocks of 256 threads, on the current device.  Writes
// the timed launch's duration (CUDA events, after one untimed launch) to
// *ms and the operations it retired to *ops (a packed f32x2 FMA counts as
// two FMAs).  Returns 0, or a CUDA error code.
MICRO_API int mamba_micro_run(int kind, int iters, int blocks_per_sm, double *ms, double *ops) {
  if (kind < 0 || kind >= NKINDS || iters < 1 || blocks_per_sm < 1 || !ms || !ops)
    return int(cudaErrorInvalidValue);
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return int(e);
  const int grid = sms * blocks_per_sm;
  float *out = nullptr;
  cudaEvent_t t0 = nullptr, t1 = nullptr;
  if ((e = cudaMalloc(&out, size_t(grid) * kThreads * sizeof(float))) != cudaSuccess) return int(e);
  e = cudaEventCreate(&t0);
  if (e == cudaSuccess) e = cudaEventCreate(&t1);
  if (e == cudaSuccess) e = launch_kind(kind, grid, out, iters, 0.5f, nullptr);
  if (e == cudaSuccess) e = cudaEventRecord(t0, nullptr);
  if (e == cudaSuccess) e = launch_kind(kind, grid, out, iters, 0.25f, nullptr);
  if (e == cudaSuccess) e = cudaEventRecord(t1, nullptr);
  if (e == cudaSuccess) e = cudaEventSynchronize(t1);
  float el = 0.f;
  if (e == cudaSuccess) e = cudaEventElapsedTime(&el, t0, t1);
  if (t0) cudaEventDestroy(t0);
  if (t1) cudaEventDestroy(t1);
  cudaFree(out);
  if (e != cudaSuccess) return int(e);
  *ms = el;
  *ops = double(grid) * kThreads * kChains * double(iters) * (kind == FMA_F32X2 ? 2.0 : 1.0);
  return 0;
}
