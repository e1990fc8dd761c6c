// decode.cuh -- one step of the selective SSM per (batch, channel): the
// recurrent mode used for autoregressive inference, constant work per token
// and no cache of earlier tokens ("Mamba: Linear-Time Sequence Modeling with
// Selective State Spaces", trishampatil.com walk-through, Part II section 4,
// and the paper-graph-ui summary's "What the recurrence computes").
//
// Given the state h (batch, dim, N) -- e.g. the last_state of a forward over
// the prompt -- one token (u, delta, z of shape (batch, dim), B and C of shape
// (batch, N)) updates it in place and produces y (batch, dim):
//     Delta = softplus(delta + bias)
//     h_n  <- exp(Delta A_n) h_n + (exp(Delta A_n) - 1)/A_n B_n u
//     y     = (sum_n C_n h_n + D u) silu(z)
// The step moves the state twice (read and write, 8N bytes per channel) and
// does O(N) arithmetic per channel, so it is bound by memory traffic and
// launch latency, not by the ALUs; it uses the generic arithmetic (one exp per
// state, Delta psi(Delta A) with a series near 0) for any A.
#pragma once

#include "common.cuh"
#include "fwd_staged.cuh"

namespace mscan {

struct DecodeArgs {
  float *state;
  const void *u, *delta, *z, *B, *C;
  const float *bias, *A, *D;
  void *y;
  int64_t batch, dim;
  int N;
};

constexpr int kDecodeThreads = 128;

template <typename T, int NM>
__global__ void __launch_bounds__(kDecodeThreads) decode_step_kernel(const DecodeArgs a) {
  const int64_t ch = int64_t(blockIdx.x) * kDecodeThreads + threadIdx.x;
  if (ch >= a.batch * a.dim) return;
  const int64_t b = ch / a.dim, d = ch % a.dim;
  const int N = a.N;
  const T *Bp = static_cast<const T *>(a.B) + b * N;
  const T *Cp = static_cast<const T *>(a.C) + b * N;
  float *st = a.state + ch * N;
  const float uv = to_f(static_cast<const T *>(a.u)[ch]);
  const float v = to_f(static_cast<const T *>(a.delta)[ch]) + (a.bias ? a.bias[d] : 0.f);
  const float Delta = softplus_fast(v);
  float y0 = a.D ? a.D[d] * uv : 0.f;
#pragma unroll
  for (int n = 0; n < NM; ++n) {
    if (n < N) {
      const float An = a.A[d * N + n];
      const float x = Delta * An;
      const float e = ex2f(x * kLog2e);
      float p = fmaf(x, 1.f / 720.f, 1.f / 120.f);
      p = fmaf(x, p, 1.f / 24.f);
      p = fmaf(x, p, 1.f / 6.f);
      p = fmaf(x, p, 0.5f);
      p = fmaf(x, p, 1.f);
      // Bbar / B = Delta psi(x): the series near 0, (e^x - 1)/A away from it
      const float Eb = fabsf(x) < 0.25f ? Delta * p : (e - 1.f) / An;
      const float h = fmaf(e, st[n], Eb * to_f(Bp[n]) * uv);
      st[n] = h;
      y0 = fmaf(to_f(Cp[n]), h, y0);
    }
  }
  if (a.z) {
    const float zv = to_f(static_cast<const T *>(a.z)[ch]);
    y0 *= zv * rcpf(1.f + ex2f(-zv * kLog2e));
  }
  static_cast<T *>(a.y)[ch] = from_f<T>(y0);
}

}  // namespace mscan
