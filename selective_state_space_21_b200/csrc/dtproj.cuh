// dtproj.cuh -- the contractions of the low-rank Delta projection
// ("Mamba: Linear-Time Sequence Modeling with Selective State Spaces",
// paper-graph-ui summary, section 3.6 "Parameterization of Delta's input
// projection": s_Delta(x) = Linear_D(Linear_R(x)), R small), on CUDA cores:
//     delta[b,d,t]    = sum_r W[d,r] dt_low[b,r,t]
//     d_dt_low[b,r,t] = sum_d W[d,r] ddelta[b,d,t]
//     dW[d,r]         = sum_b sum_t ddelta[b,d,t] dt_low[b,r,t]
// as one strided, tiled FP32 contraction kernel (exact fp32 products and
// sums, inputs widened exactly, outputs rounded once).  It serves fp32 I/O
// (whose tensor-core form would round the operands to tf32), the shapes the
// fused kernels do not take, and the reference path; the bf16 hot path
// computes delta inside the scan kernels on the tensor cores and the two
// gradient products with the tcgen05 GEMM of dtproj_gemm.cuh.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "common.cuh"

namespace mscan {

// C[m][n] (+ over batch rows if reduce) = sum_k A[m][k] B[k][n], every
// operand addressed through element strides; batch index z = blockIdx.z.
struct Contraction {
  const void *A, *B;
  void *C;
  int64_t M, N, K, batch;
  int64_t a_m, a_k, a_b;  // strides of A
  int64_t b_k, b_n, b_b;  // strides of B
  int64_t c_m, c_n, c_b;  // strides of C
  bool reduce_batch;      // C = sum over batch rows (one C), in batch order
};

constexpr int kCT = 64;   // output tile
constexpr int kCK = 16;   // k step

template <typename TI, typename TO>
__global__ void __launch_bounds__(256) contraction_kernel(const Contraction c) {
  __shared__ float As[kCK][kCT + 1];
  __shared__ float Bs[kCK][kCT + 1];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int64_t m0 = int64_t(blockIdx.y) * kCT, n0 = int64_t(blockIdx.x) * kCT;
  const TI *A = static_cast<const TI *>(c.A);
  const TI *B = static_cast<const TI *>(c.B);
  float acc[4][4] = {};
  const int64_t b_lo = c.reduce_batch ? 0 : blockIdx.z;
  const int64_t b_hi = c.reduce_batch ? c.batch : blockIdx.z + 1;
  for (int64_t bb = b_lo; bb < b_hi; ++bb) {
    const TI *Ab = A + bb * c.a_b;
    const TI *Bb = B + bb * c.b_b;
    for (int64_t k0 = 0; k0 < c.K; k0 += kCK) {
      for (int i = threadIdx.x; i < kCK * kCT; i += 256) {
        const int kk = i % kCK, mm = i / kCK;  // A: consecutive threads walk k
        const int64_t m = m0 + mm, k = k0 + kk;
        As[kk][mm] = (m < c.M && k < c.K) ? to_f(Ab[m * c.a_m + k * c.a_k]) : 0.f;
        const int nn = i % kCT, kb = i / kCT;  // B: consecutive threads walk n
        const int64_t n = n0 + nn, k2 = k0 + kb;
        Bs[kb][nn] = (n < c.N && k2 < c.K) ? to_f(Bb[k2 * c.b_k + n * c.b_n]) : 0.f;
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < kCK; ++kk) {
        float a[4], b[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          a[i] = As[kk][ty + 16 * i];
          b[i] = Bs[kk][tx + 16 * i];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
      }
      __syncthreads();
    }
  }
  TO *C = static_cast<TO *>(c.C) + (c.reduce_batch ? 0 : int64_t(blockIdx.z) * c.c_b);
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t m = m0 + ty + 16 * i, n = n0 + tx + 16 * j;
      if (m < c.M && n < c.N) C[m * c.c_m + n * c.c_n] = from_f<TO>(acc[i][j]);
    }
}

template <typename TI, typename TO>
inline cudaError_t launch_contraction(const Contraction &c, cudaStream_t s) {
  const int64_t gx = (c.N + kCT - 1) / kCT, gy = (c.M + kCT - 1) / kCT;
  const int64_t gz = c.reduce_batch ? 1 : c.batch;
  if (gx > 0x7fffffff || gy > 65535 || gz > 65535) return cudaErrorInvalidConfiguration;
  contraction_kernel<TI, TO><<<dim3(unsigned(gx), unsigned(gy), unsigned(gz)), 256, 0, s>>>(c);
  return cudaGetLastError();
}

// delta_b = W . dt_low_b  (W: (dim, R), dt_low: (batch, R, L), delta: (batch, dim, L))
inline Contraction proj_delta(const void *W, const void *dt_low, void *delta, int64_t batch,
                              int64_t dim, int64_t L, int64_t R) {
  Contraction c;
  c.A = W; c.B = dt_low; c.C = delta;
  c.M = dim; c.N = L; c.K = R; c.batch = batch;
  c.a_m = R; c.a_k = 1; c.a_b = 0;
  c.b_k = L; c.b_n = 1; c.b_b = R * L;
  c.c_m = L; c.c_n = 1; c.c_b = dim * L;
  c.reduce_batch = false;
  return c;
}

// d_dt_low_b = W^T . ddelta_b
inline Contraction proj_grad_input(const void *W, const void *ddelta, void *d_dt_low, int64_t batch,
                                   int64_t dim, int64_t L, int64_t R) {
  Contraction c;
  c.A = W; c.B = ddelta; c.C = d_dt_low;
  c.M = R; c.N = L; c.K = dim; c.batch = batch;
  c.a_m = 1; c.a_k = R; c.a_b = 0;
  c.b_k = L; c.b_n = 1; c.b_b = dim * L;
  c.c_m = L; c.c_n = 1; c.c_b = R * L;
  c.reduce_batch = false;
  return c;
}

// dW = sum_b ddelta_b . dt_low_b^T
inline Contraction proj_grad_weight(const void *ddelta, const void *dt_low, float *dW, int64_t batch,
                                    int64_t dim, int64_t L, int64_t R) {
  Contraction c;
  c.A = ddelta; c.B = dt_low; c.C = dW;
  c.M = dim; c.N = R; c.K = L; c.batch = batch;
  c.a_m = L; c.a_k = 1; c.a_b = dim * L;
  c.b_k = 1; c.b_n = L; c.b_b = R * L;
  c.c_m = R; c.c_n = 1; c.c_b = 0;
  c.reduce_batch = true;
  return c;
}

}  // namespace mscan
