// cplx.cuh -- the selective scan with a complex-valued diagonal A.
//
// "Mamba: Linear-Time Sequence Modeling with Selective State Spaces",
// paper-graph-ui summary, section 3.6 "Real vs. Complex parameters" (prior
// SSMs such as S4D-Lin keep complex states and parameters; the paper keeps
// the option for continuous signals such as audio) and the Table 8 ablation
// (S4D-Lin, A_n = -1/2 + n i).  A, B, C and the state are complex; u, delta,
// z and y are real:
//     Abar = exp(Delta A_n),  Bbar = (exp(Delta A_n) - 1) / A_n B_n,
//     h_n  = Abar h_n + Bbar u,   y = (Re(sum_n C_n h_n) + D u) silu(z).
// A complex vector of N entries is stored planar, real parts first: A
// (dim, 2N), B and C (batch, 2N, L), states (batch, dim, 2N); gradients of
// complex inputs are the pairs (d/d re, d/d im) in the same layout.
//
// One thread owns one (batch, channel) and its N complex states, sequential
// over time; a CTA holds channels of one batch row, so the B and C rows of a
// step are shared: they are staged per tile of steps in shared memory as
// fp32 tables.  In general each state costs three special-function
// operations per step (exp of the real part, sine and cosine of the
// range-reduced half of the imaginary part) and about 35 FP32 operations,
// without branches.  A thread whose states have the S4D-Lin structure shares
// one exp and two sine/cosine pairs per step over them; where also |A| >= 1/8
// the update takes the form h += (Abar - 1)(h + (B/A) u), 10 FP32 operations
// per state on top of the 7 of its decay.
//
// The backward follows the real one-thread-per-channel kernel: a forward
// sweep keeps the state at the start of every block of steps, the reverse
// sweep recomputes a block into shared memory and walks it backwards with the
// adjoint (the gradient g = dl/d re + i dl/d im of a complex quantity passes a
// product by the conjugate of the other factor):
//     G_t = conj(C_t) dy0_t + conj(Abar_{t+1}) G_{t+1},
//     du += Re(conj(G) Bbar),  dDelta += Re(conj(G) (A h_t + B u))
//        (A h_t + B u = Abar (A h_{t-1} + B u)),
//     gA += conj(Delta Abar h_{t-1} + Delta^2 phi(Delta A) B u) G
//        (= conj(1/A) conj(Delta dh/dDelta - Bbar u) G, used where |A| >= 1/8),
//     gB += conj(Delta psi(Delta A)) u G,  gC += conj(h_t) dy0,
// with deterministic reductions as in the real kernels.
#pragma once

#include "common.cuh"
#include "fwd_staged.cuh"

namespace mscan {

struct CplxArgs {
  const void *u, *delta, *z, *B, *C, *dy;  // B, C: (batch, 2N, L) planar
  const float *bias, *A, *D;               // A: (dim, 2N) planar
  void *y, *du, *ddelta, *dz, *dB, *dC;
  float *last_state, *dA, *dD, *dbias;  // last_state (batch, dim, 2N), dA (dim, 2N)
  int64_t batch, dim, L;
  int N;
  // (the saving forward) the state at the start of every kCplxBwdTC-step
  // block, laid out as the backward's block checkpoints: (batch*dim,
  // n_blocks, 2 NM), real parts first; null: not stored
  float *save_ckpt = nullptr;
  int64_t save_blocks = 0;
  // (the backward from saved states) those checkpoints, written by the
  // saving forward of the same inputs: the forward sweep does not run
  const float *saved_ckpt = nullptr;
};

constexpr int kCplxThreads = 128;
constexpr int kCplxTT = 32;         // steps per staged B / C tile (forward)
constexpr int kCplxBwdThreads = 64;
constexpr int kCplxBwdTC = 8;       // steps per recomputed block (backward)

// exp(Delta a) and E = (exp(Delta a) - 1)/a = Delta psi(Delta a) for complex
// a = ar + i ai (ira + i iai = 1/a), without branches.  With x = Delta a,
//     exp(x) - 1 = (expm1(Re x) - 2 e^{Re x} sin^2(Im x / 2))
//                  + i 2 e^{Re x} sin(Im x / 2) cos(Im x / 2),
// which has no cancellation anywhere: expm1 takes its Taylor series below
// |Re x| = 1/4 and the sine of the half angle (reduced to [-pi, pi]) its
// series below 1/2, so that small arguments keep their relative accuracy.
// a = 0 gives E = Delta (the limit).
__device__ __forceinline__ void cplx_decay(float Delta, float ar, float ai, float ira, float iai,
                                           float &abr, float &abi, float &Er, float &Ei) {
  const float xr = Delta * ar, xi = Delta * ai;
  const float e = ex2f(xr * kLog2e);
  const float pm = xr * (1.f + xr * (0.5f + xr * (1.f / 6.f + xr * (1.f / 24.f + xr * (1.f / 120.f +
                   xr * (1.f / 720.f))))));
  const float em1 = fabsf(xr) < 0.25f ? pm : e - 1.f;
  const float hh = 0.5f * xi;
  const float k = rintf(hh * 0.15915494309189535f);
  float r = fmaf(-k, 6.28318548202514648f, hh);
  r = fmaf(-k, -1.7484556e-7f, r);  // 2 pi = 6.28318548 - 1.7484556e-7
  float s2, c2;
  __sincosf(r, &s2, &c2);
  const float r2 = r * r;
  const float ps = r * (1.f - r2 * (1.f / 6.f - r2 * (1.f / 120.f - r2 * (1.f / 5040.f))));
  s2 = fabsf(r) < 0.5f ? ps : s2;
  const float es = 2.f * e * s2;
  const float mr = fmaf(-es, s2, em1), mi = es * c2;
  abr = 1.f + mr;
  abi = mi;
  const bool zero = ira == 0.f && iai == 0.f;
  Er = zero ? Delta : fmaf(mr, ira, -mi * iai);
  Ei = zero ? 0.f : fmaf(mr, iai, mi * ira);
}

// cos and sin of phi, phi reduced to [-pi, pi] first; the sine takes its
// series below 1/2 so that small angles keep their relative accuracy.
__device__ __forceinline__ void cis_reduced(float phi, float &c, float &s) {
  const float k = rintf(phi * 0.15915494309189535f);
  float r = fmaf(-k, 6.28318548202514648f, phi);
  r = fmaf(-k, -1.7484556e-7f, r);  // 2 pi = 6.28318548 - 1.7484556e-7
  __sincosf(r, &s, &c);
  const float r2 = r * r;
  const float ps = r * (1.f - r2 * (1.f / 6.f - r2 * (1.f / 120.f - r2 * (1.f / 5040.f))));
  s = fabsf(r) < 0.5f ? ps : s;
}

// Whether a thread's NS states have the S4D-Lin form A_j = a + i (b + j c)
// with a < 0 and no sign change of the imaginary part across them (then the
// half-angle recurrence below has no cancellation).
template <int NS>
__device__ __forceinline__ bool cplx_lin_structure(const float (&ar)[NS], const float (&ai)[NS]) {
  bool lin = ar[0] < 0.f && isfinite(ar[0]) && isfinite(ai[0]);
  const float c = NS > 1 ? ai[NS > 1 ? 1 : 0] - ai[0] : 0.f;
#pragma unroll
  for (int j = 1; j < NS; ++j) lin = lin && ar[j] == ar[0] && ai[j] == ai[0] + float(j) * c;
  return lin && (ai[0] == 0.f || ai[0] * c >= 0.f);
}

// M_j = Abar_j - 1 = exp(Delta A_j) - 1 for a thread's NS states with the
// S4D-Lin structure A_j = a + i (b + j c): M_j = expm1(Delta a) + e^{Delta a}
// (e^{i th_j} - 1) with th_j = Delta (b + j c) and e^{i th} - 1 =
// 2i sin(th/2) e^{i th/2}; the half angles e^{i th_j/2} follow from
// e^{i th_0/2} by repeated multiplication with e^{i Delta c/2}.  One exp and
// two sine/cosine pairs per step, 7 FP32 operations per state, all free of
// cancellation.
template <int NS>
__device__ __forceinline__ void cplx_lin_m(float Delta, float a, float b, float c, float (&Mr)[NS],
                                           float (&Mi)[NS]) {
  const float xr = Delta * a;
  const float ea = ex2f(xr * kLog2e);
  const float pm = xr * (1.f + xr * (0.5f + xr * (1.f / 6.f + xr * (1.f / 24.f + xr * (1.f / 120.f +
                   xr * (1.f / 720.f))))));
  const float em = fabsf(xr) < 0.25f ? pm : ea - 1.f;
  const float ea2 = 2.f * ea;
  float qr, qi, zr, zi;
  cis_reduced(0.5f * Delta * b, qr, qi);
  cis_reduced(0.5f * Delta * c, zr, zi);
#pragma unroll
  for (int j = 0; j < NS; ++j) {
    const float t = ea2 * qi;
    Mr[j] = fmaf(-t, qi, em);  // expm1(Delta a) - 2 e^{Delta a} sin^2(th/2)
    Mi[j] = t * qr;            // 2 e^{Delta a} sin(th/2) cos(th/2)
    if (j + 1 < NS) {
      const float nr = fmaf(qr, zr, -qi * zi);
      qi = fmaf(qr, zi, qi * zr);
      qr = nr;
    }
  }
}

// The spacing c of a thread's imaginary parts (0 with one state).
template <int NS>
__device__ __forceinline__ float cplx_lin_step(const float (&ai)[NS]) {
  return NS > 1 ? ai[NS > 1 ? 1 : 0] - ai[0] : 0.f;
}

// Whether every state of the thread has |A| >= 1/8, so that forms divided by
// A lose no more than a few ulp against the other terms.
template <int NS>
__device__ __forceinline__ bool cplx_not_small(const float (&ar)[NS], const float (&ai)[NS]) {
  bool ok = true;
#pragma unroll
  for (int j = 0; j < NS; ++j) ok = ok && ar[j] * ar[j] + ai[j] * ai[j] >= 1.f / 64.f;
  return ok;
}

// One step of a thread's states in the form h += M (h + (B/A) u), M = Abar - 1
// (S4D-Lin structure and |A| >= 1/8): E B u = M (B/A) u without forming E.
// bre / bim point at the staged Re B and Im B of this thread's states.
template <int NS>
__device__ __forceinline__ void cplx_update_m(const float (&Mr)[NS], const float (&Mi)[NS],
                                              const float (&ira)[NS], const float (&iai)[NS],
                                              float ut, const float *bre, const float *bim,
                                              float (&hr)[NS], float (&hi)[NS]) {
#pragma unroll
  for (int j = 0; j < NS; ++j) {
    const float br = bre[j], bi = bim[j];
    const float wr = fmaf(br, ira[j], -bi * iai[j]), wi = fmaf(br, iai[j], bi * ira[j]);  // B/A
    const float sr = fmaf(wr, ut, hr[j]), si = fmaf(wi, ut, hi[j]);
    hr[j] = fmaf(Mr[j], sr, fmaf(-Mi[j], si, hr[j]));
    hi[j] = fmaf(Mr[j], si, fmaf(Mi[j], sr, hi[j]));
  }
}

// Decays of a thread's NS states at one step: Abar_j = exp(Delta A_j) and
// E_j = (Abar_j - 1)/A_j, from cplx_lin_m with the S4D-Lin structure, else
// per state from cplx_decay.
template <int NS>
__device__ __forceinline__ void cplx_decays(float Delta, bool lin, const float (&ar)[NS],
                                            const float (&ai)[NS], const float (&ira)[NS],
                                            const float (&iai)[NS], float (&abr)[NS],
                                            float (&abi)[NS], float (&Er)[NS], float (&Ei)[NS]) {
  if (lin) {
    float Mr[NS], Mi[NS];
    cplx_lin_m<NS>(Delta, ar[0], ai[0], cplx_lin_step<NS>(ai), Mr, Mi);
#pragma unroll
    for (int j = 0; j < NS; ++j) {
      abr[j] = 1.f + Mr[j];
      abi[j] = Mi[j];
      Er[j] = fmaf(Mr[j], ira[j], -Mi[j] * iai[j]);
      Ei[j] = fmaf(Mr[j], iai[j], Mi[j] * ira[j]);
    }
  } else {
#pragma unroll
    for (int j = 0; j < NS; ++j) cplx_decay(Delta, ar[j], ai[j], ira[j], iai[j], abr[j], abi[j], Er[j], Ei[j]);
  }
}

// phi(x) = (x e^x - (e^x - 1)) / x^2 for complex x, from e^x = (er, ei);
// its Taylor series where |x| < 1/4.
__device__ __forceinline__ void cplx_phi(float xr, float xi, float er, float ei, float &pr,
                                         float &pi) {
  // both forms, then a select: no divergence between the channels of a warp
  // sum_k (k+1)/(k+2)! x^k, k = 0..5
  float ar = 1.f / 840.f, ai = 0.f;
  const float cs[5] = {1.f / 144.f, 1.f / 30.f, 0.125f, 1.f / 3.f, 0.5f};
#pragma unroll
  for (int j = 0; j < 5; ++j) {
    const float tr = fmaf(ar, xr, fmaf(-ai, xi, cs[j]));
    const float ti = fmaf(ar, xi, ai * xr);
    ar = tr;
    ai = ti;
  }
  // numerator x e^x - e^x + 1, divided by x^2
  const float nr = fmaf(xr, er, -xi * ei) - er + 1.f;
  const float ni = fmaf(xr, ei, xi * er) - ei;
  const float x2r = fmaf(xr, xr, -xi * xi), x2i = 2.f * xr * xi;
  const float den = rcpf(fmaf(x2r, x2r, x2i * x2i));
  const bool small = xr * xr + xi * xi < 0.0625f;
  pr = small ? ar : fmaf(nr, x2r, ni * x2i) * den;
  pi = small ? ai : fmaf(ni, x2r, -nr * x2i) * den;
}

// Row stride of the staged tables, padded so that the staging writes fall in
// distinct banks: a warp writes 32 / TT slots of TT consecutive steps, which
// wants a stride of 1 modulo 32 for TT = 32 and of 4 modulo 32 for TT = 8.
template <int NM, int TT> constexpr int cplx_tab_stride() { return 4 * NM + (TT >= 32 ? 1 : 4); }

// Stages the B and C columns of steps [t0, t0 + TT) of batch row b into
// tab[t][4 NM] = (Re B, Im B, Re C, Im C) as fp32 (rows cplx_tab_stride apart),
// zero past N and past L.
template <typename T, int NM, int TT>
__device__ __forceinline__ void cplx_stage_bc(const CplxArgs &a, int64_t b, int64_t t0, float *tab,
                                              bool with_c, int nthreads) {
  const int N = a.N;
  const T *Bp = static_cast<const T *>(a.B) + b * 2 * N * a.L;
  const T *Cp = static_cast<const T *>(a.C) + b * 2 * N * a.L;
  for (int w = threadIdx.x; w < TT * 4 * NM; w += nthreads) {
    const int t = w % TT, slot = w / TT;  // consecutive threads read consecutive steps
    const int part = slot / NM, n = slot % NM;  // 0 Re B, 1 Im B, 2 Re C, 3 Im C
    const int64_t tt = t0 + t;
    float v = 0.f;
    if (n < N && tt < a.L && (with_c || part < 2)) {
      const T *src = part < 2 ? Bp : Cp;
      v = to_f(src[(int64_t(part & 1) * N + n) * a.L + tt]);
    }
    tab[t * cplx_tab_stride<NM, TT>() + slot] = v;
  }
}

// TPC threads share one channel, NM / TPC states each (adjacent lanes; their
// partial readouts are joined by shuffles): with few channels per SM, more
// threads per channel hide more of the recurrence's latency.
template <typename T, int NM, int TPC>
__global__ void __launch_bounds__(kCplxThreads) cplx_fwd_kernel(const CplxArgs a) {
  constexpr int NS = NM / TPC;  // states per thread
  __shared__ __align__(16) float tab[kCplxTT * cplx_tab_stride<NM, kCplxTT>()];
  const int tid = threadIdx.x;
  const int part = tid % TPC;
  const int64_t b = blockIdx.y;
  const int64_t d_raw = int64_t(blockIdx.x) * (kCplxThreads / TPC) + tid / TPC;
  const bool valid = d_raw < a.dim;
  const int64_t d = valid ? d_raw : a.dim - 1;
  const int64_t row = (b * a.dim + d) * a.L;
  const int N = a.N;
  const T *u = static_cast<const T *>(a.u) + row;
  const T *dl = static_cast<const T *>(a.delta) + row;
  const T *z = a.z ? static_cast<const T *>(a.z) + row : nullptr;
  T *y = static_cast<T *>(a.y) + row;
  const float bias = a.bias ? a.bias[d] : 0.f;
  const float Dd = (a.D && part == 0) ? a.D[d] : 0.f;
  float ar[NS], ai[NS], ira[NS], iai[NS], hr[NS], hi[NS];
#pragma unroll
  for (int j = 0; j < NS; ++j) {
    const int n = part * NS + j;
    ar[j] = n < N ? a.A[d * 2 * N + n] : -1.f;
    ai[j] = n < N ? a.A[d * 2 * N + N + n] : 0.f;
    const float m = ar[j] * ar[j] + ai[j] * ai[j];
    ira[j] = m > 0.f ? ar[j] / m : 0.f;
    iai[j] = m > 0.f ? -ai[j] / m : 0.f;
    hr[j] = hi[j] = 0.f;
  }
  const bool lin = cplx_lin_structure<NS>(ar, ai);
  const bool mform = lin && cplx_not_small<NS>(ar, ai);
  const float clin = cplx_lin_step<NS>(ai);
  for (int64_t t0 = 0; t0 < a.L; t0 += kCplxTT) {
    __syncthreads();
    cplx_stage_bc<T, NM, kCplxTT>(a, b, t0, tab, true, kCplxThreads);
    __syncthreads();
    const int steps = int(a.L - t0 < kCplxTT ? a.L - t0 : kCplxTT);
    for (int i = 0; i < steps; ++i) {
      const int64_t t = t0 + i;
      if (a.save_ckpt && valid && t % kCplxBwdTC == 0) {  // the state at a block start
        float *ck = a.save_ckpt + ((b * a.dim + d) * a.save_blocks + t / kCplxBwdTC) * 2 * NM + part * NS;
        if constexpr (NS == 4) {  // 16-byte stores (the row is 128-byte aligned)
          *reinterpret_cast<float4 *>(ck) = make_float4(hr[0], hr[1], hr[2], hr[3]);
          *reinterpret_cast<float4 *>(ck + NM) = make_float4(hi[0], hi[1], hi[2], hi[3]);
        } else {
#pragma unroll
          for (int j = 0; j < NS; ++j) {
            ck[j] = hr[j];
            ck[NM + j] = hi[j];
          }
        }
      }
      const float Delta = softplus_fast(to_f(dl[t]) + bias);
      const float ut = to_f(u[t]);
      const float *tr = tab + i * cplx_tab_stride<NM, kCplxTT>() + part * NS;
      float y0 = Dd * ut;
      if (mform) {
        float Mr[NS], Mi[NS];
        cplx_lin_m<NS>(Delta, ar[0], ai[0], clin, Mr, Mi);
        cplx_update_m<NS>(Mr, Mi, ira, iai, ut, tr, tr + NM, hr, hi);
      } else {
        float Abr[NS], Abi[NS], Ebr[NS], Ebi[NS];
        cplx_decays<NS>(Delta, lin, ar, ai, ira, iai, Abr, Abi, Ebr, Ebi);
#pragma unroll
        for (int j = 0; j < NS; ++j) {
          const float abr = Abr[j], abi = Abi[j], Er = Ebr[j], Ei = Ebi[j];
          const float br = tr[j], bi = tr[NM + j];
          // Bbar u = E B u
          const float bbr = fmaf(Er, br, -Ei * bi) * ut, bbi = fmaf(Er, bi, Ei * br) * ut;
          const float nr = fmaf(abr, hr[j], fmaf(-abi, hi[j], bbr));
          const float ni = fmaf(abr, hi[j], fmaf(abi, hr[j], bbi));
          hr[j] = nr;
          hi[j] = ni;
        }
      }
#pragma unroll
      for (int j = 0; j < NS; ++j) y0 = fmaf(tr[2 * NM + j], hr[j], fmaf(-tr[3 * NM + j], hi[j], y0));
#pragma unroll
      for (int o = 1; o < TPC; o <<= 1) y0 += __shfl_xor_sync(0xffffffffu, y0, o);
      if (z) {
        const float zt = to_f(z[t]);
        y0 *= zt * rcpf(1.f + ex2f(-zt * kLog2e));
      }
      if (valid && part == 0) y[t] = from_f<T>(y0);
    }
  }
  if (valid && a.last_state) {
    float *ls = a.last_state + (b * a.dim + d) * 2 * N;
#pragma unroll
    for (int j = 0; j < NS; ++j) {
      const int n = part * NS + j;
      if (n < N) {
        ls[n] = hr[j];
        ls[N + n] = hi[j];
      }
    }
  }
}

struct CplxWork {
  float *ckpt;       // (batch*dim, n_blocks, 2 NM) block-start states
  float *part_bc;    // (n_dblk, batch, 4 kMaxN, L): Re dB, Im dB, Re dC, Im dC
  float *part_A;     // (K, batch*dim, 2N): per chunk
  float *part_D;     // (K, batch*dim)
  float *part_bias;  // (K, batch*dim)
  int64_t n_blocks, n_dblk;
  // The sequence of every channel block splits into K chunks of `bpc` blocks
  // (the last may be shorter).  The forward sweep hands each chunk's end
  // state on to the next chunk, the reverse sweep each chunk's entering
  // adjoint back to the previous one, through `carry` (per channel block
  // and thread: the state, or G and Abar) and the flags (per channel block:
  // how many chunks have handed on, in the sweep's order).
  int K;
  int64_t bpc;
  int *counter;      // ticket counters of the two launches, zero before the first
  int *flags;        // (n_dblk * batch): the forward sweep counts chunks 1..K, the reverse K+1..2K
  int flag_base;     // the reverse sweep's count starts here: K, or 0 without a forward sweep
                     // (block checkpoints saved by the forward)
  float *carry;      // (n_dblk * batch, kCplxBwdThreads, 4 NS)
  uint64_t timeout_ns;
};

// Sums S values over the lanes of a warp that share lane % TPC (the channels
// of one state range), leaving S * TPC / 32 of the sums on each lane: a
// butterfly reduce-scatter over lane bits 4 down to log2(TPC).  Lane l keeps
// the sums of value indices base(l) + r, r < S * TPC / 32, where base(l) is
// the sum of the upper half sizes of the stages whose lane bit is set.
template <int S, int TPC>
__device__ __forceinline__ void lane_reduce_scatter(float (&v)[S], int lane) {
  int h = S / 2;
#pragma unroll
  for (int o = 16; o >= TPC; o >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < S / 2; ++i) {
      if (i < h) {
        const float send = up ? v[i] : v[i + h];
        const float keep = up ? v[i + h] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
      }
    }
    h /= 2;
  }
}

template <int S, int TPC>
__device__ __forceinline__ int lane_scatter_base(int lane) {
  int base = 0, h = S / 2;
  for (int o = 16; o >= TPC; o >>= 1) {
    if (lane & o) base += h;
    h /= 2;
  }
  return base;
}

// Row stride of the per-block rows of u, delta, z, dy and of du, ddelta, dz
// staged in shared memory (one float of padding: distinct banks for the
// channels of a warp).
constexpr int kCplxRow = kCplxBwdTC + 1;

// Shared memory of cplx_bwd_kernel: block states, B / C table, dB / dC warp
// sums, then the staged rows (4 inputs, 3 outputs) of the CTA's channels.
template <int NM, int TPC>
constexpr size_t cplx_bwd_smem() {
  return 4 * (size_t(kCplxBwdTC) * 2 * (NM / TPC) * kCplxBwdThreads +
              size_t(kCplxBwdTC) * cplx_tab_stride<NM, kCplxBwdTC>() + 2 * 4 * kMaxN * kCplxRow +
              7 * size_t(kCplxBwdThreads / TPC) * kCplxRow);
}

// Steps [t0, t0 + steps) of one (batch row, channel) row of a (batch, dim, L)
// tensor to dst[0 .. kCplxBwdTC) as fp32, zero past `steps` (and for d past
// dim): 16-byte loads where the rows are 16-byte aligned and the block whole.
template <typename T>
__device__ __forceinline__ void cplx_load_block(const void *src, const CplxArgs &a, int64_t b,
                                                int64_t d, int64_t t0, int steps, bool vec,
                                                float *dst) {
  float v[kCplxBwdTC];
#pragma unroll
  for (int i = 0; i < kCplxBwdTC; ++i) v[i] = 0.f;
  if (d < a.dim) {
    const T *p = static_cast<const T *>(src) + (b * a.dim + d) * a.L + t0;
    if (vec && steps == kCplxBwdTC) {
      constexpr int V = Vec<T>::kN;
#pragma unroll
      for (int k = 0; k < kCplxBwdTC / V; ++k) {
        float o[V];
        Vec<T>::unpack(*reinterpret_cast<const uint4 *>(p + k * V), o);
#pragma unroll
        for (int i = 0; i < V; ++i) v[k * V + i] = o[i];
      }
    } else {
#pragma unroll
      for (int i = 0; i < kCplxBwdTC; ++i)
        if (i < steps) v[i] = to_f(p[i]);
    }
  }
#pragma unroll
  for (int i = 0; i < kCplxBwdTC; ++i) dst[i] = v[i];
}

// The inverse of cplx_load_block for an output row (nothing for d past dim).
template <typename T>
__device__ __forceinline__ void cplx_store_block(void *dst, const CplxArgs &a, int64_t b, int64_t d,
                                                 int64_t t0, int steps, bool vec, const float *src) {
  if (d >= a.dim) return;
  T *p = static_cast<T *>(dst) + (b * a.dim + d) * a.L + t0;
  if (vec && steps == kCplxBwdTC) {
    constexpr int V = Vec<T>::kN;
#pragma unroll
    for (int k = 0; k < kCplxBwdTC / V; ++k) {
      float o[V];
#pragma unroll
      for (int i = 0; i < V; ++i) o[i] = src[k * V + i];
      *reinterpret_cast<uint4 *>(p + k * V) = Vec<T>::pack(o);
    }
  } else {
    for (int i = 0; i < steps; ++i) p[i] = from_f<T>(src[i]);
  }
}

// TPC threads share one channel, NM / TPC states each (adjacent lanes), as in
// the forward: more threads per channel, fewer registers per thread.  Per
// block of steps the CTA stages B and C and the u, delta, z, dy rows of its
// channels in shared memory (one 16-byte load per row where aligned), and
// writes its du, ddelta, dz rows back from there.
//
// Two launches: REVERSE = false, the forward sweep storing the block-start
// states; REVERSE = true, the reverse sweep.  The work units are (chunk,
// channel block) pairs that persistent CTAs claim from a ticket counter,
// chunk by chunk (the reverse sweep from the last chunk): a unit that waits
// for its neighbour chunk's hand-off (bounded) waits only on a unit claimed
// before it.  Splitting the sequences into chunks lets the units of the last
// round fill the GPU instead of leaving most SMs idle for a whole sequence.
template <typename T, int NM, int TPC, bool REVERSE>
__global__ void __launch_bounds__(kCplxBwdThreads, 8) cplx_bwd_kernel(const CplxArgs a, const CplxWork w) {
  constexpr int NS = NM / TPC;                 // states per thread
  constexpr int NV = 4 * NS < 32 / TPC ? 32 / TPC : 4 * NS;  // dB / dC values (padded)
  constexpr int NKEEP = NV * TPC / 32;         // sums left on each lane
  extern __shared__ __align__(16) float smem[];
  float *hs = smem;                                          // [TC][2 NS][threads]
  float *tab = hs + kCplxBwdTC * 2 * NS * kCplxBwdThreads;  // [TC][stride]
  float *wsum = tab + kCplxBwdTC * cplx_tab_stride<NM, kCplxBwdTC>();  // [2 warps][4 kMaxN][kCplxRow]
  constexpr int CPB = kCplxBwdThreads / TPC;                 // channels per CTA
  float *xs = wsum + 2 * 4 * kMaxN * kCplxRow;               // [u, delta, z, dy][CPB][kCplxRow]
  float *os = xs + 4 * CPB * kCplxRow;                       // [du, ddelta, dz][CPB][kCplxRow]
  __shared__ int s_ticket, s_abort;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int part = tid % TPC, lc = tid / TPC;
  for (int i = tid; i < 2 * 4 * kMaxN * kCplxRow; i += kCplxBwdThreads) wsum[i] = 0.f;
  const int64_t n_cb = w.n_dblk * a.batch;  // channel blocks
  for (;;) {  // one (chunk, channel block) unit per pass
  __syncthreads();
  if (tid == 0) {
    s_ticket = atomicAdd(w.counter + (REVERSE ? 1 : 0), 1);
    s_abort = 0;
  }
  __syncthreads();
  if (int64_t(s_ticket) >= n_cb * w.K) break;
  const int64_t cb = s_ticket % n_cb;
  const int k = REVERSE ? w.K - 1 - int(s_ticket / n_cb) : int(s_ticket / n_cb);
  const int64_t c_beg = int64_t(k) * w.bpc;
  const int64_t c_end = std::min<int64_t>(w.n_blocks, c_beg + w.bpc);
  const int64_t dblk = cb % w.n_dblk;
  const int64_t b = cb / w.n_dblk;
  const int64_t d0 = dblk * CPB;
  const int64_t d_raw = d0 + lc;
  const bool valid = d_raw < a.dim;
  const int64_t d = valid ? d_raw : a.dim - 1;
  const int64_t ch = b * a.dim + d;
  const int N = a.N;
  const bool has_z = a.z != nullptr;
  // 16-byte rows: every row start and block start is 16-byte aligned
  const bool vec = (a.L * int64_t(sizeof(T))) % 16 == 0 &&
                   ((reinterpret_cast<uintptr_t>(a.u) | reinterpret_cast<uintptr_t>(a.delta) |
                     reinterpret_cast<uintptr_t>(a.z) | reinterpret_cast<uintptr_t>(a.dy) |
                     reinterpret_cast<uintptr_t>(a.du) | reinterpret_cast<uintptr_t>(a.ddelta) |
                     reinterpret_cast<uintptr_t>(a.dz)) & 15) == 0;
  const float *xu = xs + lc * kCplxRow, *xd = xs + (CPB + lc) * kCplxRow;
  const float *xz = xs + (2 * CPB + lc) * kCplxRow, *xdy = xs + (3 * CPB + lc) * kCplxRow;
  const float bias = a.bias ? a.bias[d] : 0.f;
  const float Dd = a.D ? a.D[d] : 0.f;
  float *ckpt = w.ckpt + ch * w.n_blocks * 2 * NM;
  float *carry = w.carry + (cb * kCplxBwdThreads + tid) * 4 * NS;

  float ar[NS], ai[NS], ira[NS], iai[NS], hr[NS], hi[NS];
#pragma unroll
  for (int j = 0; j < NS; ++j) {
    const int n = part * NS + j;
    ar[j] = n < N ? a.A[d * 2 * N + n] : -1.f;
    ai[j] = n < N ? a.A[d * 2 * N + N + n] : 0.f;
    const float m = ar[j] * ar[j] + ai[j] * ai[j];
    ira[j] = m > 0.f ? ar[j] / m : 0.f;
    iai[j] = m > 0.f ? -ai[j] / m : 0.f;
    hr[j] = hi[j] = 0.f;
  }

  const bool lin = cplx_lin_structure<NS>(ar, ai);
  // dA through A dh/dA = Delta dh/dDelta - E B u (no phi) where every state of
  // the thread has |A| >= 1/8; the fp32 error of that difference, relative to
  // the other terms of dA, is then about 8 eps.  Smaller |A| take phi.
  const bool ident = cplx_not_small<NS>(ar, ai);
  const bool mform = lin && ident;
  const float clin = cplx_lin_step<NS>(ai);

  // one forward step of this thread's states (B from the staged table row)
  auto step = [&](float Delta, float ut, const float *trow) {
    if (mform) {
      float Mr[NS], Mi[NS];
      cplx_lin_m<NS>(Delta, ar[0], ai[0], clin, Mr, Mi);
      cplx_update_m<NS>(Mr, Mi, ira, iai, ut, trow + part * NS, trow + NM + part * NS, hr, hi);
      return;
    }
    float Abr[NS], Abi[NS], Ebr[NS], Ebi[NS];
    cplx_decays<NS>(Delta, lin, ar, ai, ira, iai, Abr, Abi, Ebr, Ebi);
#pragma unroll
    for (int j = 0; j < NS; ++j) {
      const float abr = Abr[j], abi = Abi[j], Er = Ebr[j], Ei = Ebi[j];
      const float br = trow[part * NS + j], bi = trow[NM + part * NS + j];
      const float bbr = fmaf(Er, br, -Ei * bi) * ut, bbi = fmaf(Er, bi, Ei * br) * ut;
      const float nr = fmaf(abr, hr[j], fmaf(-abi, hi[j], bbr));
      const float ni = fmaf(abr, hi[j], fmaf(abi, hr[j], bbi));
      hr[j] = nr;
      hi[j] = ni;
    }
  };

  if constexpr (!REVERSE) {
  // Forward sweep over the chunk: the state at the start of every block,
  // from the state the previous chunk handed on.
  if (k > 0) {
    if (tid == 0 && !wait_flag_geq(w.flags + cb, k, w.timeout_ns)) {  // chunks 0..k-1 done
      record_timeout();
      s_abort = 1;
    }
    __syncthreads();
    if (s_abort) return;
#pragma unroll
    for (int j = 0; j < NS; ++j) {
      hr[j] = __ldcg(carry + j);
      hi[j] = __ldcg(carry + NS + j);
    }
  }
  for (int64_t c = c_beg; c < c_end; ++c) {
    const int64_t t0 = c * kCplxBwdTC;
    // (padding channels run on zero rows and share the last channel's slots:
    // they must not write them)
    if (valid) {
#pragma unroll
      for (int j = 0; j < NS; ++j) {
        ckpt[c * 2 * NM + part * NS + j] = hr[j];
        ckpt[c * 2 * NM + NM + part * NS + j] = hi[j];
      }
    }
    const int steps = int(a.L - t0 < kCplxBwdTC ? a.L - t0 : kCplxBwdTC);
    __syncthreads();
    cplx_stage_bc<T, NM, kCplxBwdTC>(a, b, t0, tab, false, kCplxBwdThreads);
    for (int r = tid; r < 2 * CPB; r += kCplxBwdThreads)
      cplx_load_block<T>(r < CPB ? a.u : a.delta, a, b, d0 + r % CPB, t0, steps, vec, xs + r * kCplxRow);
    __syncthreads();
    for (int i = 0; i < steps; ++i)
      step(softplus_fast(xd[i] + bias), xu[i], tab + i * cplx_tab_stride<NM, kCplxBwdTC>());
  }
  if (k + 1 < w.K) {  // the state at the chunk's end, for the next chunk
#pragma unroll
    for (int j = 0; j < NS; ++j) {
      carry[j] = hr[j];
      carry[NS + j] = hi[j];
    }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) st_release_gpu(w.flags + cb, k + 1);
  continue;
  } else {

  float Gr[NS], Gi[NS], Anr[NS], Ani[NS], gAr[NS], gAi[NS];
#pragma unroll
  for (int j = 0; j < NS; ++j) Gr[j] = Gi[j] = Anr[j] = Ani[j] = gAr[j] = gAi[j] = 0.f;
  float dDacc = 0.f, dbacc = 0.f;
  const int kbase = lane_scatter_base<NV, TPC>(lane);
  if (k + 1 < w.K) {  // the adjoint entering from the later chunk (and its Abar)
    // (the reverse sweep counts on from the forward sweep's K)
    if (tid == 0 && !wait_flag_geq(w.flags + cb, w.flag_base + (w.K - 1 - k), w.timeout_ns)) {
      record_timeout();
      s_abort = 1;
    }
    __syncthreads();
    if (s_abort) return;
#pragma unroll
    for (int j = 0; j < NS; ++j) {
      Gr[j] = __ldcg(carry + j);
      Gi[j] = __ldcg(carry + NS + j);
      Anr[j] = __ldcg(carry + 2 * NS + j);
      Ani[j] = __ldcg(carry + 3 * NS + j);
    }
  }

  for (int64_t c = c_end - 1; c >= c_beg; --c) {
    const int64_t t0 = c * kCplxBwdTC;
    const int steps = int(a.L - t0 < kCplxBwdTC ? a.L - t0 : kCplxBwdTC);
    __syncthreads();
    cplx_stage_bc<T, NM, kCplxBwdTC>(a, b, t0, tab, true, kCplxBwdThreads);
    for (int r = tid; r < 4 * CPB; r += kCplxBwdThreads) {
      const int q = r / CPB;  // u, delta, z, dy
      const void *src = q == 0 ? a.u : q == 1 ? a.delta : q == 2 ? a.z : a.dy;
      if (src) cplx_load_block<T>(src, a, b, d0 + r % CPB, t0, steps, vec, xs + r * kCplxRow);
    }
    __syncthreads();
    // recompute the block; hs[s] holds the state before step t0 + s
#pragma unroll
    for (int j = 0; j < NS; ++j) {
      hr[j] = ckpt[c * 2 * NM + part * NS + j];
      hi[j] = ckpt[c * 2 * NM + NM + part * NS + j];
    }
    for (int s = 0; s < steps; ++s) {
#pragma unroll
      for (int j = 0; j < NS; ++j) {
        hs[(s * 2 * NS + j) * kCplxBwdThreads + tid] = hr[j];
        hs[(s * 2 * NS + NS + j) * kCplxBwdThreads + tid] = hi[j];
      }
      step(softplus_fast(xd[s] + bias), xu[s], tab + s * cplx_tab_stride<NM, kCplxBwdTC>());
    }
    // reverse sweep over the block
    for (int s = steps - 1; s >= 0; --s) {
      const float v = xd[s] + bias;
      const float Delta = softplus_fast(v);
      const float sv = rcpf(1.f + ex2f(-v * kLog2e));
      const float ut = xu[s];
      const float dyt = xdy[s];
      float dy0 = dyt, zt = 0.f, sz = 0.f;
      if (has_z) {
        zt = xz[s];
        sz = rcpf(1.f + ex2f(-zt * kLog2e));
        dy0 = dyt * zt * sz;
      }
      const float *trow = tab + s * cplx_tab_stride<NM, kCplxBwdTC>() + part * NS;
      float y0 = 0.f, du = 0.f, dDelta = 0.f;
      float vals[NV];  // per state j: Re dB, Im dB, Re dC, Im dC at j, NS + j, 2 NS + j, 3 NS + j
#pragma unroll
      for (int i = 0; i < NV; ++i) vals[i] = 0.f;
      const float um = valid ? ut : 0.f, dym = valid ? dy0 : 0.f;  // padding channels add 0
      float Abr[NS], Abi[NS], Ebr[NS], Ebi[NS];
      cplx_decays<NS>(Delta, lin, ar, ai, ira, iai, Abr, Abi, Ebr, Ebi);
#pragma unroll
      for (int j = 0; j < NS; ++j) {
        const float hpr = hs[(s * 2 * NS + j) * kCplxBwdThreads + tid];
        const float hpi = hs[(s * 2 * NS + NS + j) * kCplxBwdThreads + tid];
        const float abr = Abr[j], abi = Abi[j], Er = Ebr[j], Ei = Ebi[j];
        const float br = trow[j], bi = trow[NM + j], cr = trow[2 * NM + j], ci = trow[3 * NM + j];
        // h_t = Abar h_{t-1} + E B u
        const float bur = br * ut, bui = bi * ut;
        const float ebr = fmaf(Er, br, -Ei * bi), ebi = fmaf(Er, bi, Ei * br);  // E B
        const float ebur = ebr * ut, ebui = ebi * ut;
        const float hcr = fmaf(abr, hpr, fmaf(-abi, hpi, ebur));
        const float hci = fmaf(abr, hpi, fmaf(abi, hpr, ebui));
        y0 = fmaf(cr, hcr, fmaf(-ci, hci, y0));
        // G_t = conj(C) dy0 + conj(Abar_{t+1}) G_{t+1}
        const float gr = fmaf(cr, dy0, fmaf(Anr[j], Gr[j], Ani[j] * Gi[j]));
        const float gi = fmaf(-ci, dy0, fmaf(Anr[j], Gi[j], -Ani[j] * Gr[j]));
        Gr[j] = gr;
        Gi[j] = gi;
        Anr[j] = abr;
        Ani[j] = abi;
        // du += Re(conj(G) E B); dDelta += Re(conj(G) p) with
        // p = dh_t/dDelta = Abar (A h_{t-1} + B u) = A h_t + B u
        du = fmaf(gr, ebr, fmaf(gi, ebi, du));
        const float pr_ = fmaf(ar[j], hcr, fmaf(-ai[j], hci, bur));
        const float pi_ = fmaf(ar[j], hci, fmaf(ai[j], hcr, bui));
        dDelta = fmaf(gr, pr_, fmaf(gi, pi_, dDelta));
        // gA += conj(k) G with k = dh_t/dA = Delta Abar h_{t-1} + Delta^2 phi(x) B u;
        // with `ident` the sum runs over k A = Delta p - E B u and is divided
        // by A at the end
        float kr, ki;
        if (ident) {
          kr = fmaf(Delta, pr_, -ebur);
          ki = fmaf(Delta, pi_, -ebui);
        } else {
          float phr, phi_;
          cplx_phi(Delta * ar[j], Delta * ai[j], abr, abi, phr, phi_);
          const float D2 = Delta * Delta;
          kr = fmaf(Delta, fmaf(abr, hpr, -abi * hpi), D2 * fmaf(phr, bur, -phi_ * bui));
          ki = fmaf(Delta, fmaf(abr, hpi, abi * hpr), D2 * fmaf(phr, bui, phi_ * bur));
        }
        gAr[j] = fmaf(kr, gr, fmaf(ki, gi, gAr[j]));
        gAi[j] = fmaf(kr, gi, fmaf(-ki, gr, gAi[j]));
        // gB = conj(E) u G, gC = conj(h_t) dy0
        vals[j] = fmaf(Er, gr, Ei * gi) * um;
        vals[NS + j] = fmaf(Er, gi, -Ei * gr) * um;
        vals[2 * NS + j] = hcr * dym;
        vals[3 * NS + j] = -hci * dym;
      }
      // join the partial sums of the TPC threads of this channel
#pragma unroll
      for (int o = 1; o < TPC; o <<= 1) {
        y0 += __shfl_xor_sync(0xffffffffu, y0, o);
        du += __shfl_xor_sync(0xffffffffu, du, o);
        dDelta += __shfl_xor_sync(0xffffffffu, dDelta, o);
      }
      y0 = fmaf(Dd, ut, y0);
      du = fmaf(Dd, dy0, du);
      const float ddl = dDelta * sv;
      // du, ddelta, dz to the staged output rows, one per thread of the channel
      const float dzv = dyt * y0 * sz * (1.f + zt * (1.f - sz));
      for (int k = part; k < 3; k += TPC) os[(k * CPB + lc) * kCplxRow + s] = k == 0 ? du : k == 1 ? ddl : dzv;
      if (valid && part == 0) {
        dDacc = fmaf(dy0, ut, dDacc);
        dbacc += ddl;
      }
      lane_reduce_scatter<NV, TPC>(vals, lane);
#pragma unroll
      for (int r = 0; r < NKEEP; ++r) {
        const int idx = kbase + r;  // value index of this lane's sum
        if (idx < 4 * NS) {
          const int q = idx / NS, n = part * NS + idx % NS;
          wsum[(warp * 4 * kMaxN + q * kMaxN + n) * kCplxRow + s] = vals[r];
        }
      }
    }
    __syncthreads();
    for (int idx = tid; idx < 4 * kMaxN * kCplxBwdTC; idx += kCplxBwdThreads) {
      const int slot = idx / kCplxBwdTC, s = idx % kCplxBwdTC;
      if (s < steps) {
        const float sum = wsum[(0 * 4 * kMaxN + slot) * kCplxRow + s] +
                          wsum[(1 * 4 * kMaxN + slot) * kCplxRow + s];
        w.part_bc[((dblk * a.batch + b) * 4 * kMaxN + slot) * a.L + t0 + s] = sum;
      }
    }
    for (int r = tid; r < 3 * CPB; r += kCplxBwdThreads) {
      const int q = r / CPB;  // du, ddelta, dz
      void *dst = q == 0 ? a.du : q == 1 ? a.ddelta : a.dz;
      if (dst) cplx_store_block<T>(dst, a, b, d0 + r % CPB, t0, steps, vec, os + r * kCplxRow);
    }
  }
  if (k > 0) {  // the adjoint entering this chunk, for the previous one
#pragma unroll
    for (int j = 0; j < NS; ++j) {
      carry[j] = Gr[j];
      carry[NS + j] = Gi[j];
      carry[2 * NS + j] = Anr[j];
      carry[3 * NS + j] = Ani[j];
    }
  }
  if (ident) {  // conj(1/A) times the sums of conj(k A) G
#pragma unroll
    for (int j = 0; j < NS; ++j) {
      const float sr = gAr[j], si = gAi[j];
      gAr[j] = fmaf(ira[j], sr, iai[j] * si);
      gAi[j] = fmaf(ira[j], si, -iai[j] * sr);
    }
  }
  if (valid) {  // this chunk's parts of dA, dD, dbias
    const int64_t bd = a.batch * a.dim;
#pragma unroll
    for (int j = 0; j < NS; ++j) {
      const int n = part * NS + j;
      if (n < N) {
        w.part_A[(k * bd + ch) * 2 * N + n] = gAr[j];
        w.part_A[(k * bd + ch) * 2 * N + N + n] = gAi[j];
      }
    }
    if (part == 0) {
      w.part_D[k * bd + ch] = dDacc;
      w.part_bias[k * bd + ch] = dbacc;
    }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) st_release_gpu(w.flags + cb, w.flag_base + (w.K - k));
  }
  }
}

// dB, dC (batch, 2N, L): the per-CTA partials summed over channel blocks.
template <typename T>
__global__ void cplx_finalize_bc(const CplxArgs a, const CplxWork w) {
  const int64_t total = a.batch * 2 * a.N * a.L;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t t = i % a.L, j = (i / a.L) % (2 * a.N), b = i / (a.L * 2 * a.N);
    const int64_t n = j % a.N, im = j / a.N;
    float sb = 0.f, sc = 0.f;
    for (int64_t k = 0; k < w.n_dblk; ++k) {
      const float *p = w.part_bc + ((k * a.batch + b) * 4 * kMaxN) * a.L + t;
      sb += p[(im * 16 + n) * a.L];
      sc += p[(32 + im * 16 + n) * a.L];
    }
    static_cast<T *>(a.dB)[i] = from_f<T>(sb);
    static_cast<T *>(a.dC)[i] = from_f<T>(sc);
  }
}

// dA (dim, 2N), dD, dbias: the per-channel partials summed over the batch.
__global__ void cplx_finalize_params(const CplxArgs a, const CplxWork w) {
  const int64_t total = a.dim * 2 * a.N;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t d = i / (2 * a.N), j = i % (2 * a.N);
    const int64_t bd = a.batch * a.dim;
    float s = 0.f;
    for (int64_t b = 0; b < a.batch; ++b)
      for (int k = 0; k < w.K; ++k) s += w.part_A[(k * bd + b * a.dim + d) * 2 * a.N + j];
    a.dA[i] = s;
    if (j == 0) {
      float sd = 0.f, sb = 0.f;
      for (int64_t b = 0; b < a.batch; ++b)
        for (int k = 0; k < w.K; ++k) {
          sd += w.part_D[k * bd + b * a.dim + d];
          sb += w.part_bias[k * bd + b * a.dim + d];
        }
      if (a.dD) a.dD[d] = sd;
      if (a.dbias) a.dbias[d] = sb;
    }
  }
}

}  // namespace mscan
