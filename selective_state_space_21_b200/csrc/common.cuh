// common.cuh -- shared device helpers of libmambascan (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

namespace mscan {

constexpr int kMaxN = 16;

// Sticky per-device error word (bit 0: a bounded wait expired).  Each .cu file
// of the library is a whole program (no relocatable device code), so every
// translation unit that includes this header has its own copy.
__device__ unsigned int g_error_word = 0;
constexpr unsigned int kErrTimeout = 1u;

struct FwdArgs {
  const void *u, *delta, *z, *B, *C;
  const float *bias, *A, *D;
  void *y;
  float *last_state;
  int64_t batch, dim, L;
  int N;
};

struct BwdArgs {
  const void *u, *delta, *z, *B, *C, *dy;
  const float *bias, *A, *D;
  void *du, *ddelta, *dz, *dB, *dC;
  float *dA, *dD, *dbias;
  int64_t batch, dim, L;
  int N;
};

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// softplus(v) = log(1 + e^v) in the stable form, with the CUDA math library's
// accurate log1pf / expf.
__device__ __forceinline__ float softplus_acc(float v) {
  return v > 0.f ? v + log1pf(expf(-v)) : log1pf(expf(v));
}

__device__ __forceinline__ float sigmoid_acc(float v) { return 1.f / (1.f + expf(-v)); }

// (x e^x - expm1(x)) / x^2, the derivative of expm1(x)/x.  Taylor series
// sum_k (k+1)/(k+2)! x^k near zero, where the closed form cancels.
__device__ __forceinline__ float dpsi_acc(float x) {
  if (fabsf(x) < 0.1f) {
    return 0.5f + x * (1.f / 3.f + x * (0.125f + x * (1.f / 30.f + x * (1.f / 144.f +
           x * (1.f / 840.f)))));
  }
  return (x * expf(x) - expm1f(x)) / (x * x);
}

// ----------------------------------------------------------- host: workspace

// Workspace comes stream-ordered from one library-owned memory pool per device
// that keeps up to kPoolKeepBytes reserved between calls, so that repeated
// calls do not map and unmap hundreds of megabytes each time (the default
// pool gives memory back to the system at every synchronization).
constexpr uint64_t kPoolKeepBytes = uint64_t(4) << 30;

inline cudaMemPool_t library_pool() {
  static std::mutex mu;
  static cudaMemPool_t pools[64] = {};
  static bool tried[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!tried[dev]) {
    tried[dev] = true;
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool = nullptr;
    if (cudaMemPoolCreate(&pool, &props) == cudaSuccess) {
      uint64_t keep = kPoolKeepBytes;
      cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
      pools[dev] = pool;
    } else {
      cudaGetLastError();
    }
  }
  return pools[dev];
}

inline cudaError_t ws_alloc(void **ptr, size_t bytes, cudaStream_t s) {
  cudaMemPool_t pool = library_pool();
  if (pool) return cudaMallocFromPoolAsync(ptr, bytes, pool, s);
  return cudaMallocAsync(ptr, bytes, s);
}

inline cudaError_t ws_free(void *ptr, cudaStream_t s) { return cudaFreeAsync(ptr, s); }

}  // namespace mscan
