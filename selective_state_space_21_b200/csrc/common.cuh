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
constexpr unsigned int kErrBounds = 2u;

// Index check of the bounds-checking build (MAMBA_DEBUG_BOUNDS): an index
// outside [0, n) sets the sticky error word's bounds bit and the access that
// it guards is skipped, so that a wrong index shows up as a status instead of
// a fault.  In the normal build it is always true and costs nothing.
#if defined(MAMBA_DEBUG_BOUNDS)
__device__ __forceinline__ bool in_bounds(int64_t i, int64_t n) {
  if (i >= 0 && i < n) return true;
  atomicOr(&g_error_word, kErrBounds);
  return false;
}
#else
__device__ __forceinline__ constexpr bool in_bounds(int64_t, int64_t) { return true; }
#endif

// With conv_w set, `u` points at the input x of the Mamba block's causal
// depthwise convolution, and the scan runs on u = SiLU(conv(x)) computed on
// the fly (see ConvFilter); conv_w is (dim, conv_width), conv_b (dim) or null.
struct FwdArgs {
  const void *u, *delta, *z, *B, *C;
  const float *bias, *A, *D;
  void *y;
  float *last_state;
  int64_t batch, dim, L;
  int N;
  const float *conv_w = nullptr, *conv_b = nullptr;
  int conv_width = 0;
  // With W_dt set (the fused low-rank Delta projection), delta is not read:
  // delta[b,d,t] = sum_r W_dt[d,r] dt_low[b,r,t] is formed on the tensor cores.
  const void *dt_low = nullptr, *W_dt = nullptr;
  int R = 0;
};

// With conv_w set, `u` is x as in FwdArgs and `du` receives the gradient with
// respect to u = SiLU(conv(x)); the convolution's own backward runs after.
struct BwdArgs {
  const void *u, *delta, *z, *B, *C, *dy;
  const float *bias, *A, *D;
  void *du, *ddelta, *dz, *dB, *dC;
  float *dA, *dD, *dbias;
  int64_t batch, dim, L;
  int N;
  const float *conv_w = nullptr, *conv_b = nullptr;
  int conv_width = 0;
  // fused low-rank Delta projection, as in FwdArgs (delta is not read)
  const void *dt_low = nullptr, *W_dt = nullptr;
  int R = 0;
};

// The short causal depthwise convolution in front of the S6 layer (Knowl 3
// "Mamba Block Architecture", step 3, chapterpal.com page: width d_conv = 4,
// then SiLU), for widths W <= 4: the filter is held right-aligned, w3 on the
// current step and w0 on the step three back, so that
//     pre_t = b + w0 x_{t-3} + w1 x_{t-2} + w2 x_{t-1} + w3 x_t
// with x = 0 before the first step, and u_t = pre_t sigmoid(pre_t).
constexpr int kMaxConvWidth = 4;
struct ConvFilter {
  float w0, w1, w2, w3, b;
};

__device__ __forceinline__ ConvFilter load_conv_filter(const float *conv_w, const float *conv_b,
                                                       int W, int64_t d) {
  const float *r = conv_w + d * W;
  ConvFilter c;
  c.w3 = r[W - 1];
  c.w2 = W >= 2 ? r[W - 2] : 0.f;
  c.w1 = W >= 3 ? r[W - 3] : 0.f;
  c.w0 = W >= 4 ? r[W - 4] : 0.f;
  c.b = conv_b ? conv_b[d] : 0.f;
  return c;
}

__device__ __forceinline__ float conv_pre(const ConvFilter &c, float xm3, float xm2, float xm1,
                                          float x0) {
  return fmaf(c.w0, xm3, fmaf(c.w1, xm2, fmaf(c.w2, xm1, fmaf(c.w3, x0, c.b))));
}

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

// u_t of the convolution prologue at step t of the row x (I/O type), with
// CUDA's accurate expf: the plain form used by the one-thread-per-channel
// kernels.
template <typename T>
__device__ __forceinline__ float conv_u_acc(const ConvFilter &c, const T *x, int64_t t) {
  const float xm3 = t >= 3 ? to_f(x[t - 3]) : 0.f;
  const float xm2 = t >= 2 ? to_f(x[t - 2]) : 0.f;
  const float xm1 = t >= 1 ? to_f(x[t - 1]) : 0.f;
  const float p = conv_pre(c, xm3, xm2, xm1, to_f(x[t]));
  return p * sigmoid_acc(p);
}

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
// that keeps up to a reserve (kPoolKeepBytes unless the caller sets another)
// between calls, so that repeated calls do not map and unmap hundreds of
// megabytes each time (the default pool gives memory back to the system at
// every synchronization).
constexpr uint64_t kPoolKeepBytes = uint64_t(4) << 30;
constexpr int kMaxDevices = 64;

struct PoolRegistry {
  std::mutex mu;
  cudaMemPool_t pools[kMaxDevices] = {};
  bool tried[kMaxDevices] = {};
  uint64_t keep[kMaxDevices];
  PoolRegistry() {
    for (int i = 0; i < kMaxDevices; ++i) keep[i] = kPoolKeepBytes;
  }
};

inline PoolRegistry &pool_registry() {
  static PoolRegistry r;
  return r;
}

inline int current_device_or(int fallback) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return fallback;
  }
  return dev;
}

// The pool of the current device (created on first use), or null.
inline cudaMemPool_t library_pool() {
  const int dev = current_device_or(-1);
  if (dev < 0) return nullptr;
  PoolRegistry &r = pool_registry();
  std::lock_guard<std::mutex> lock(r.mu);
  if (!r.tried[dev]) {
    r.tried[dev] = true;
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool = nullptr;
    if (cudaMemPoolCreate(&pool, &props) == cudaSuccess) {
      uint64_t keep = r.keep[dev];
      cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
      r.pools[dev] = pool;
    } else {
      cudaGetLastError();
    }
  }
  return r.pools[dev];
}

// Test hook: the number of workspace allocations of the calling thread that
// still succeed before one fails (negative: none fails).
inline int &alloc_failure_countdown() {
  static thread_local int n = -1;
  return n;
}

inline cudaError_t ws_alloc(void **ptr, size_t bytes, cudaStream_t s) {
  int &countdown = alloc_failure_countdown();
  if (countdown == 0) {
    countdown = -1;
    *ptr = nullptr;
    return cudaErrorMemoryAllocation;
  }
  if (countdown > 0) --countdown;
  cudaMemPool_t pool = library_pool();
  if (pool) return cudaMallocFromPoolAsync(ptr, bytes, pool, s);
  return cudaMallocAsync(ptr, bytes, s);
}

inline cudaError_t ws_free(void *ptr, cudaStream_t s) { return cudaFreeAsync(ptr, s); }

}  // namespace mscan
