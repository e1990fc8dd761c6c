// dtproj.h -- the low-rank Delta projection in front of the scan (host side).
//
// "Mamba: Linear-Time Sequence Modeling with Selective State Spaces",
// paper-graph-ui summary, section 3.6 "Parameterization of Delta's input
// projection": s_Delta(x) = Linear_D(Linear_R(x)) with a small rank R.  Given
// the rank-R projection dt_low (batch, R, L) and the weight W_dt (dim, R) of
// Linear_D (its bias is the scan's delta_bias),
//     delta[b,d,t] = sum_r W_dt[d,r] dt_low[b,r,t],
// a dense contraction of K = R per token-channel.  On B200 it runs as a
// tensor-core GEMM (cuBLAS, fp32 accumulation) into a stream-ordered
// workspace that the scan then reads: the scan kernels are bound by FP32
// issue with two CTAs per SM, and holding a 128 x R weight tile in shared
// memory inside them would leave room for one.
//
// cuBLAS is opened with dlopen on first use, so the library links no cuBLAS
// and the other entry points work without it; a process without
// libcublas.so.12 gets MAMBA_ERR_UNSUPPORTED from the projection calls.
#pragma once

#include <cublas_v2.h>
#include <cuda_runtime.h>
#include <dlfcn.h>

namespace mscan {

struct CublasApi {
  using CreateFn = cublasStatus_t (*)(cublasHandle_t *);
  using SetStreamFn = cublasStatus_t (*)(cublasHandle_t, cudaStream_t);
  using GemmExFn = cublasStatus_t (*)(cublasHandle_t, cublasOperation_t, cublasOperation_t, int,
                                      int, int, const void *, const void *, cudaDataType, int,
                                      const void *, cudaDataType, int, const void *, void *,
                                      cudaDataType, int, cublasComputeType_t, cublasGemmAlgo_t);
  using GemmStridedBatchedExFn = cublasStatus_t (*)(
      cublasHandle_t, cublasOperation_t, cublasOperation_t, int, int, int, const void *,
      const void *, cudaDataType, int, long long, const void *, cudaDataType, int, long long,
      const void *, void *, cudaDataType, int, long long, int, cublasComputeType_t,
      cublasGemmAlgo_t);
  CreateFn create = nullptr;
  SetStreamFn set_stream = nullptr;
  GemmExFn gemm = nullptr;
  GemmStridedBatchedExFn gemm_sb = nullptr;
  bool ok = false;
};

inline const CublasApi &cublas_api() {
  static const CublasApi api = [] {
    CublasApi a;
    void *h = dlopen("libcublas.so.12", RTLD_NOW | RTLD_GLOBAL);
    if (!h) h = dlopen("/usr/local/cuda/lib64/libcublas.so.12", RTLD_NOW | RTLD_GLOBAL);
    if (!h) return a;
    a.create = reinterpret_cast<CublasApi::CreateFn>(dlsym(h, "cublasCreate_v2"));
    a.set_stream = reinterpret_cast<CublasApi::SetStreamFn>(dlsym(h, "cublasSetStream_v2"));
    a.gemm = reinterpret_cast<CublasApi::GemmExFn>(dlsym(h, "cublasGemmEx"));
    a.gemm_sb = reinterpret_cast<CublasApi::GemmStridedBatchedExFn>(
        dlsym(h, "cublasGemmStridedBatchedEx"));
    a.ok = a.create && a.set_stream && a.gemm && a.gemm_sb;
    return a;
  }();
  return api;
}

// One handle per (host thread, device): a cuBLAS handle must not be used by
// two threads at once, and it belongs to the device current at creation.
inline cublasHandle_t cublas_handle(int dev) {
  constexpr int kMaxDev = 64;
  thread_local cublasHandle_t handles[kMaxDev] = {};
  if (dev < 0 || dev >= kMaxDev) return nullptr;
  const CublasApi &api = cublas_api();
  if (!api.ok) return nullptr;
  if (!handles[dev] && api.create(&handles[dev]) != CUBLAS_STATUS_SUCCESS) handles[dev] = nullptr;
  return handles[dev];
}

// The three products of the projection, for row-major tensors with L
// contiguous (cuBLAS sees each as its column-major transpose).  `io` is the
// I/O type (CUDA_R_32F or CUDA_R_16BF); every product accumulates in fp32.
struct DtProj {
  cublasHandle_t h;
  cudaDataType io;
  int64_t batch, dim, L, R;

  // delta_b (dim, L) = W_dt (dim, R) . dt_low_b (R, L), every batch row.
  bool forward(const void *dt_low, const void *W_dt, void *delta) const {
    const float one = 1.f, zero = 0.f;
    return cublas_api().gemm_sb(h, CUBLAS_OP_N, CUBLAS_OP_N, int(L), int(dim), int(R), &one,
                                dt_low, io, int(L), R * L, W_dt, io, int(R), 0, &zero, delta, io,
                                int(L), dim * L, int(batch), CUBLAS_COMPUTE_32F,
                                CUBLAS_GEMM_DEFAULT) == CUBLAS_STATUS_SUCCESS;
  }

  // d_dt_low_b (R, L) = W_dt^T (R, dim) . ddelta_b (dim, L), every batch row.
  bool grad_input(const void *ddelta, const void *W_dt, void *d_dt_low) const {
    const float one = 1.f, zero = 0.f;
    return cublas_api().gemm_sb(h, CUBLAS_OP_N, CUBLAS_OP_T, int(L), int(R), int(dim), &one,
                                ddelta, io, int(L), dim * L, W_dt, io, int(R), 0, &zero, d_dt_low,
                                io, int(L), R * L, int(batch), CUBLAS_COMPUTE_32F,
                                CUBLAS_GEMM_DEFAULT) == CUBLAS_STATUS_SUCCESS;
  }

  // dW_dt (dim, R) fp32 = sum_b ddelta_b (dim, L) . dt_low_b^T (L, R): one
  // product per batch row accumulated in a fixed order.
  bool grad_weight(const void *ddelta, const void *dt_low, float *dW, size_t es) const {
    const float one = 1.f, zero = 0.f;
    for (int64_t b = 0; b < batch; ++b) {
      const char *dl = static_cast<const char *>(dt_low) + size_t(b * R * L) * es;
      const char *dd = static_cast<const char *>(ddelta) + size_t(b * dim * L) * es;
      if (cublas_api().gemm(h, CUBLAS_OP_T, CUBLAS_OP_N, int(R), int(dim), int(L), &one, dl, io,
                            int(L), dd, io, int(L), b == 0 ? &zero : &one, dW, CUDA_R_32F, int(R),
                            CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT) != CUBLAS_STATUS_SUCCESS)
        return false;
    }
    return true;
  }
};

}  // namespace mscan
