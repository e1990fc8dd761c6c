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
  // convolution prologue (CONV kernels): u is the block input x of this token;
  // conv_state (batch, dim, W - 1) fp32 holds the previous W - 1 inputs,
  // oldest first, and is shifted in place.
  float *conv_state = nullptr;
  const float *conv_w = nullptr, *conv_b = nullptr;
  int conv_width = 0;
};

// u of this token from x and the channel's convolution state (see ConvFilter
// for the right-aligned filter), and the state shifted by one input.
__device__ __forceinline__ float decode_conv_u(const DecodeArgs &a, int64_t ch, int64_t d, float x,
                                               bool write_state) {
  const int W = a.conv_width;
  const ConvFilter c = load_conv_filter(a.conv_w, a.conv_b, W, d);
  float *cs = a.conv_state + ch * (W - 1);
  const float xm1 = W >= 2 ? cs[W - 2] : 0.f;
  const float xm2 = W >= 3 ? cs[W - 3] : 0.f;
  const float xm3 = W >= 4 ? cs[W - 4] : 0.f;
  const float pre = conv_pre(c, xm3, xm2, xm1, x);
  if (write_state && W >= 2) {
    if (W >= 4) cs[W - 4] = xm2;
    if (W >= 3) cs[W - 3] = xm1;
    cs[W - 2] = x;
  }
  return pre * rcpf(1.f + ex2f(-pre * kLog2e));
}

constexpr int kDecodeThreads = 128;

template <typename T, int NM, bool CONV = false>
__global__ void __launch_bounds__(kDecodeThreads) decode_step_kernel(const DecodeArgs a) {
  const int64_t ch = int64_t(blockIdx.x) * kDecodeThreads + threadIdx.x;
  if (ch >= a.batch * a.dim) return;
  const int64_t b = ch / a.dim, d = ch % a.dim;
  const int N = a.N;
  const T *Bp = static_cast<const T *>(a.B) + b * N;
  const T *Cp = static_cast<const T *>(a.C) + b * N;
  float *st = a.state + ch * N;
  float uv = to_f(static_cast<const T *>(a.u)[ch]);
  if constexpr (CONV) uv = decode_conv_u(a, ch, d, uv, true);
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

// The same step with four states per thread (N a multiple of 4, 16-byte
// aligned state and A): a warp's state and A accesses are then contiguous
// 16-byte vectors, and the NM/4 threads of a channel join their partial
// readouts with shuffles.
template <typename T> struct Quad;
template <> struct Quad<float> {
  __device__ static float4 load(const float *p) { return *reinterpret_cast<const float4 *>(p); }
};
template <> struct Quad<__nv_bfloat16> {
  __device__ static float4 load(const __nv_bfloat16 *p) {
    const uint2 v = *reinterpret_cast<const uint2 *>(p);
    return make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u),
                       __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u));
  }
};

template <typename T, int NM, bool CONV = false>
__global__ void __launch_bounds__(kDecodeThreads) decode_step_vec4_kernel(const DecodeArgs a) {
  constexpr int TPC = NM / 4;  // threads per channel
  const int64_t gid = int64_t(blockIdx.x) * kDecodeThreads + threadIdx.x;
  const int64_t ch = gid / TPC;
  const int g = int(gid % TPC);
  const bool live = ch < a.batch * a.dim;  // dead threads still join the shuffles
  const int64_t chs = live ? ch : 0;
  const int64_t b = chs / a.dim, d = chs % a.dim;
  const float4 h = *reinterpret_cast<const float4 *>(a.state + chs * NM + 4 * g);
  const float4 Av = *reinterpret_cast<const float4 *>(a.A + d * NM + 4 * g);
  const float4 Bv = Quad<T>::load(static_cast<const T *>(a.B) + b * NM + 4 * g);
  const float4 Cv = Quad<T>::load(static_cast<const T *>(a.C) + b * NM + 4 * g);
  float uv = to_f(static_cast<const T *>(a.u)[chs]);
  // every thread of the channel forms u; the first one shifts the state (after
  // all of them have read it: the shuffles below order the warp)
  if constexpr (CONV) uv = decode_conv_u(a, chs, d, uv, false);
  const float v = to_f(static_cast<const T *>(a.delta)[chs]) + (a.bias ? a.bias[d] : 0.f);
  const float Delta = softplus_fast(v);
  const float hs[4] = {h.x, h.y, h.z, h.w}, As[4] = {Av.x, Av.y, Av.z, Av.w};
  const float Bs_[4] = {Bv.x, Bv.y, Bv.z, Bv.w}, Cs_[4] = {Cv.x, Cv.y, Cv.z, Cv.w};
  float hn[4], yp = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float x = Delta * As[i];
    const float e = ex2f(x * kLog2e);
    float p = fmaf(x, 1.f / 720.f, 1.f / 120.f);
    p = fmaf(x, p, 1.f / 24.f);
    p = fmaf(x, p, 1.f / 6.f);
    p = fmaf(x, p, 0.5f);
    p = fmaf(x, p, 1.f);
    const float Eb = fabsf(x) < 0.25f ? Delta * p : (e - 1.f) / As[i];
    hn[i] = fmaf(e, hs[i], Eb * Bs_[i] * uv);
    yp = fmaf(Cs_[i], hn[i], yp);
  }
#pragma unroll
  for (int o = 1; o < TPC; o <<= 1) yp += __shfl_xor_sync(0xffffffffu, yp, o);
  if (!live) return;
  *reinterpret_cast<float4 *>(a.state + ch * NM + 4 * g) = make_float4(hn[0], hn[1], hn[2], hn[3]);
  if (g == 0) {
    if constexpr (CONV) {
      const int W = a.conv_width;
      float *cs = a.conv_state + ch * (W - 1);
      if (W >= 2) {
        if (W >= 4) cs[W - 4] = cs[W - 3];
        if (W >= 3) cs[W - 3] = cs[W - 2];
        cs[W - 2] = to_f(static_cast<const T *>(a.u)[ch]);
      }
    }
    float y0 = yp + (a.D ? a.D[d] * uv : 0.f);
    if (a.z) {
      const float zv = to_f(static_cast<const T *>(a.z)[ch]);
      y0 *= zv * rcpf(1.f + ex2f(-zv * kLog2e));
    }
    static_cast<T *>(a.y)[ch] = from_f<T>(y0);
  }
}

}  // namespace mscan
