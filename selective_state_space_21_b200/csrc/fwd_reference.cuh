// fwd_reference.cuh -- the plain forward: one thread per (batch, channel),
// sequential over time, any diagonal A, loads straight from global memory.
//
// It follows the per-element loop of Knowl 1 "Selective State Space Layer
// (S6)" ("Mamba: Linear-Time Sequence Modeling with Selective State Spaces",
// chapterpal.com): discretize with zero-order hold, update the state, read it
// out with C_t; plus softplus on Delta, the D skip and the SiLU gate.  It is
// the path for shapes the staged kernels do not take (rows that are not
// 16-byte multiples) and the slow-but-simple GPU comparison point.  With a
// convolution filter in the arguments, u is computed from x at every step.
#pragma once
#include "common.cuh"

namespace mscan {

constexpr int kRefThreads = 128;

template <typename T, int NM>
__global__ void __launch_bounds__(kRefThreads) fwd_reference_kernel(FwdArgs a) {
  const int64_t ch = (int64_t)blockIdx.x * kRefThreads + threadIdx.x;
  if (ch >= a.batch * a.dim) return;
  const int64_t b = ch / a.dim, d = ch % a.dim;
  const int64_t L = a.L;
  const int N = a.N;
  const T *u = static_cast<const T *>(a.u) + ch * L;
  const T *dl = static_cast<const T *>(a.delta) + ch * L;
  const T *z = a.z ? static_cast<const T *>(a.z) + ch * L : nullptr;
  const T *Bp = static_cast<const T *>(a.B) + b * N * L;
  const T *Cp = static_cast<const T *>(a.C) + b * N * L;
  T *y = static_cast<T *>(a.y) + ch * L;
  const float bias = a.bias ? a.bias[d] : 0.f;
  const float Dd = a.D ? a.D[d] : 0.f;
  const bool conv = a.conv_w != nullptr;  // u is x; the scan input is SiLU(conv(x))
  ConvFilter cf = {0.f, 0.f, 0.f, 1.f, 0.f};
  if (conv) cf = load_conv_filter(a.conv_w, a.conv_b, a.conv_width, d);

  float Av[NM], invA[NM], h[NM];
#pragma unroll
  for (int n = 0; n < NM; ++n) {
    Av[n] = n < N ? a.A[d * N + n] : -1.f;
    invA[n] = Av[n] != 0.f ? 1.f / Av[n] : 0.f;
    h[n] = 0.f;
  }
  for (int64_t t = 0; t < L; ++t) {
    const float Delta = softplus_acc(to_f(dl[t]) + bias);
    const float ut = conv ? conv_u_acc(cf, u, t) : to_f(u[t]);
    float y0 = 0.f;
#pragma unroll
    for (int n = 0; n < NM; ++n) {
      if (n < N) {
        const float x = Delta * Av[n];
        const float Abar = expf(x);
        // Bbar / B = (exp(x) - 1) / A, written without cancellation.
        const float E = Av[n] != 0.f ? expm1f(x) * invA[n] : Delta;
        h[n] = Abar * h[n] + E * to_f(Bp[n * L + t]) * ut;
        y0 += to_f(Cp[n * L + t]) * h[n];
      }
    }
    if (a.D) y0 += Dd * ut;
    if (z) {
      const float zt = to_f(z[t]);
      y0 *= zt * sigmoid_acc(zt);
    }
    y[t] = from_f<T>(y0);
  }
  if (a.last_state) {
#pragma unroll
    for (int n = 0; n < NM; ++n)
      if (n < N) a.last_state[ch * N + n] = h[n];
  }
}

}  // namespace mscan
