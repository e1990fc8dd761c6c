// conv_bwd.cuh -- backward of the convolution prologue of the Mamba block.
//
// The main branch of the block runs a short causal depthwise convolution and
// SiLU before the S6 layer (Knowl 3 "Mamba Block Architecture", step 3, of
// the chapterpal.com page of "Mamba: Linear-Time Sequence Modeling with
// Selective State Spaces"; "The Mamba Architecture (Section 3.4)" of the
// paper-graph-ui summary).  With the filter right-aligned as in ConvFilter,
//     pre_t = b + w0 x_{t-3} + w1 x_{t-2} + w2 x_{t-1} + w3 x_t,
//     u_t   = pre_t sigmoid(pre_t).
// Given du (the scan backward's gradient with respect to u), the chain rule
// gives
//     dpre_t = du_t sigmoid(pre_t) (1 + pre_t (1 - sigmoid(pre_t)))
//     dx_t   = w3 dpre_t + w2 dpre_{t+1} + w1 dpre_{t+2} + w0 dpre_{t+3}
//     dw_j   = sum_t dpre_t x_{t-3+j},  db = sum_t dpre_t.
//
// The kernel works in place: the gradient buffer holds du on entry and dx on
// exit.  One warp owns one (batch, channel) row and walks it from the end in
// passes of 32 lanes x V steps: each lane loads its V steps of x and du,
// takes the three x before them from the lane below (lane 0 reads them from
// memory) and the three dpre after them from the lane above (lane 31 keeps
// them from the previous pass), then overwrites its own V steps.  A pass only
// writes steps it has already read, and the steps it reads beyond its own
// were read by an earlier pass, so the in-place update is safe.  The memory
// traffic is one read of x and du and one write of dx.
#pragma once

#include "common.cuh"
#include "fwd_staged.cuh"

namespace mscan {

constexpr int kConvWarps = 8;

template <typename T> struct Row16;  // 16-byte vectors of a row
template <> struct Row16<float> {
  static constexpr int V = 4;
  __device__ static void load(const float *p, float (&o)[4]) {
    const float4 v = *reinterpret_cast<const float4 *>(p);
    o[0] = v.x;
    o[1] = v.y;
    o[2] = v.z;
    o[3] = v.w;
  }
  __device__ static void store(float *p, const float (&o)[4]) {
    *reinterpret_cast<float4 *>(p) = make_float4(o[0], o[1], o[2], o[3]);
  }
};
template <> struct Row16<__nv_bfloat16> {
  static constexpr int V = 8;
  __device__ static void load(const __nv_bfloat16 *p, float (&o)[8]) {
    Vec<__nv_bfloat16>::unpack(*reinterpret_cast<const uint4 *>(p), o);
  }
  __device__ static void store(__nv_bfloat16 *p, const float (&o)[8]) {
    *reinterpret_cast<uint4 *>(p) = Vec<__nv_bfloat16>::pack(o);
  }
};

// VEC: rows are 16-byte aligned multiples of 16 bytes, so whole passes use
// 16-byte loads and stores; otherwise every access is a bounds-checked
// scalar one (V = 4 steps per lane).
template <typename T, bool VEC>
__global__ void __launch_bounds__(32 * kConvWarps)
    conv_bwd_kernel(const T *__restrict__ x, T *g, const float *__restrict__ conv_w,
                    const float *__restrict__ conv_b, int W, int64_t rows, int64_t dim, int64_t L,
                    float *__restrict__ part) {
  constexpr int V = VEC ? Row16<T>::V : 4;
  constexpr int CH = 32 * V;
  const int lane = threadIdx.x & 31;
  const int64_t row = int64_t(blockIdx.x) * kConvWarps + (threadIdx.x >> 5);
  if (row >= rows) return;  // the whole warp leaves together
  const ConvFilter c = load_conv_filter(conv_w, conv_b, W, row % dim);
  const T *xr = x + row * L;
  T *gr = g + row * L;
  const unsigned full = 0xffffffffu;

  float r0 = 0.f, r1 = 0.f, r2 = 0.f;  // dpre at the three steps after this pass
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f, ab = 0.f;
  for (int64_t pass = (L + CH - 1) / CH - 1; pass >= 0; --pass) {
    const int64_t p0 = pass * CH + int64_t(lane) * V;
    float xv[V], dv[V];
    if (VEC && p0 + V <= L) {
      if constexpr (VEC) {
        Row16<T>::load(xr + p0, xv);
        Row16<T>::load(gr + p0, dv);
      }
    } else {
#pragma unroll
      for (int i = 0; i < V; ++i) {
        xv[i] = p0 + i < L ? to_f(xr[p0 + i]) : 0.f;
        dv[i] = p0 + i < L ? to_f(gr[p0 + i]) : 0.f;
      }
    }
    // x at p0-3 .. p0-1
    float xm3 = __shfl_up_sync(full, xv[V - 3], 1);
    float xm2 = __shfl_up_sync(full, xv[V - 2], 1);
    float xm1 = __shfl_up_sync(full, xv[V - 1], 1);
    if (lane == 0) {
      xm3 = p0 >= 3 ? to_f(xr[p0 - 3]) : 0.f;
      xm2 = p0 >= 2 ? to_f(xr[p0 - 2]) : 0.f;
      xm1 = p0 >= 1 ? to_f(xr[p0 - 1]) : 0.f;
    }
    float win[V + 3];
    win[0] = xm3;
    win[1] = xm2;
    win[2] = xm1;
#pragma unroll
    for (int i = 0; i < V; ++i) win[3 + i] = xv[i];
    float dp[V + 3];
#pragma unroll
    for (int i = 0; i < V; ++i) {
      const float pre = conv_pre(c, win[i], win[i + 1], win[i + 2], win[i + 3]);
      const float s = rcpf(1.f + ex2f(-pre * kLog2e));
      dp[i] = dv[i] * s * fmaf(pre, 1.f - s, 1.f);  // 0 past the end, where du reads as 0
      a0 = fmaf(dp[i], win[i], a0);
      a1 = fmaf(dp[i], win[i + 1], a1);
      a2 = fmaf(dp[i], win[i + 2], a2);
      a3 = fmaf(dp[i], win[i + 3], a3);
      ab += dp[i];
    }
    // dpre at p0+V .. p0+V+2
    dp[V] = __shfl_down_sync(full, dp[0], 1);
    dp[V + 1] = __shfl_down_sync(full, dp[1], 1);
    dp[V + 2] = __shfl_down_sync(full, dp[2], 1);
    if (lane == 31) {
      dp[V] = r0;
      dp[V + 1] = r1;
      dp[V + 2] = r2;
    }
    r0 = __shfl_sync(full, dp[0], 0);
    r1 = __shfl_sync(full, dp[1], 0);
    r2 = __shfl_sync(full, dp[2], 0);
    float dx[V];
#pragma unroll
    for (int i = 0; i < V; ++i)
      dx[i] = fmaf(c.w3, dp[i], fmaf(c.w2, dp[i + 1], fmaf(c.w1, dp[i + 2], c.w0 * dp[i + 3])));
    if (VEC && p0 + V <= L) {
      if constexpr (VEC) Row16<T>::store(gr + p0, dx);
    } else {
#pragma unroll
      for (int i = 0; i < V; ++i)
        if (p0 + i < L) gr[p0 + i] = from_f<T>(dx[i]);
    }
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    a0 += __shfl_xor_sync(full, a0, o);
    a1 += __shfl_xor_sync(full, a1, o);
    a2 += __shfl_xor_sync(full, a2, o);
    a3 += __shfl_xor_sync(full, a3, o);
    ab += __shfl_xor_sync(full, ab, o);
  }
  if (lane == 0) {
    float *pr = part + row * 5;
    pr[0] = a0;
    pr[1] = a1;
    pr[2] = a2;
    pr[3] = a3;
    pr[4] = ab;
  }
}

// dconv_w[d, k] and dconv_b[d]: the per-row partials summed over the batch in
// a fixed order.  Partial slot j is the right-aligned tap, k = j - (4 - W).
__global__ void conv_bwd_finalize(const float *__restrict__ part, int64_t batch, int64_t dim, int W,
                                  float *dconv_w, float *dconv_b) {
  for (int64_t d = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; d < dim;
       d += int64_t(gridDim.x) * blockDim.x) {
    float s[5] = {0.f, 0.f, 0.f, 0.f, 0.f};
    for (int64_t b = 0; b < batch; ++b) {
      const float *pr = part + (b * dim + d) * 5;
#pragma unroll
      for (int j = 0; j < 5; ++j) s[j] += pr[j];
    }
    for (int k = 0; k < W; ++k) dconv_w[d * W + k] = s[k + kMaxConvWidth - W];
    if (dconv_b) dconv_b[d] = s[4];
  }
}

}  // namespace mscan
