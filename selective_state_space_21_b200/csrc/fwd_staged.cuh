// fwd_staged.cuh -- the staged, chunked forward of the selective scan for
// sm_100a.
//
// What it computes is the forward of Knowl 1 "Selective State Space Layer
// (S6)" ("Mamba: Linear-Time Sequence Modeling with Selective State Spaces",
// chapterpal.com) plus softplus on Delta, the D skip and the SiLU gate.  How it
// is organised for B200:
//
//  * One thread owns one (batch, channel) and keeps its N <= 16 fp32 states in
//    registers for the whole chunk; the expanded (B, L, D, N) tensors never
//    exist anywhere (the fusion of section 3.3 of the paper-graph-ui page).
//  * A CTA is 128 channels of one batch row.  TMA streams 64-byte-per-channel
//    time tiles of u, delta and z (swizzled so that each thread reads its own
//    row without bank conflicts) and the matching B and C rows through a
//    3-stage mbarrier pipeline; y leaves through a TMA store.  Only u, delta,
//    z, B, C, the parameters, y and the final state touch HBM.
//  * Work is split into units = (channel group, time chunk) handed out by a
//    ticket counter to persistent CTAs.  The state crosses chunk boundaries in
//    one of two ways (the chunking of section 3.3, "Handling long sequences
//    with chunking"):
//      - SEQ: chunk k of a group waits (bounded) for chunk k-1 to publish its
//        end state; tickets are issued chunk-major, so the predecessor was
//        claimed earlier by a running CTA and the wait always ends.  Used when
//        there are enough channel groups to fill the GPU.
//      - PAR: an aggregate pass computes, for every chunk but the last, the
//        state it produces from zero and the sum of its Delta; a small kernel
//        scans those across chunks (the associative combine of affine maps,
//        the total decay of a chunk being exp(A * sum Delta)); the main pass
//        then runs every chunk from its true initial state.  Used for few
//        channels and long sequences.
//  * Arithmetic.  For channels whose A has the S4D-Real structure
//    A[d,n] = (n+1) A[d,0] < 0, the decays of all states follow from one
//    expm1 per (t, channel): with E(j) = expm1(j x), x = Delta A[d,0], the
//    doubling relation E(m+k) = E(m) + exp(m x) E(k) gives E(1..16) in 15
//    FMAs.  The zero-order-hold update is then
//        h_n <- h_n + E(n+1) (h_n + B_n/(n+1) * u/A[d,0]),
//    which equals Abar h + Bbar u with Abar = 1 + E(n+1) and
//    Bbar = E(n+1)/A_n B.  When A[d,0] = -1, exp(-softplus(v)) = sigma(-v)
//    (the identity in the proof of Theorem 1, Knowl 4 of the same page), so
//    no log or expm1 is needed at all.  Other channels take the generic
//    arithmetic: one exp per state element and Bbar/B = Delta psi(Delta A)
//    with a series for small arguments.  Both use packed fma.rn.f32x2 where
//    the work pairs up.
#pragma once

#include <algorithm>
#include <type_traits>

#include "../../include/mamba_scan.h"
#include "common.cuh"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace mscan {

constexpr int kSThreads = 128;
constexpr int kStages = 3;
constexpr int kRowBytes = 64;
constexpr int kTileBytes = kSThreads * kRowBytes;     // 8 KB per (u | delta | z | y) tile
constexpr int kRawBytes = kMaxN * kRowBytes;          // 1 KB per B / C tile
constexpr int kStageBytes = 3 * kTileBytes + 2 * kRawBytes;
constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;

// SEQ / PAR: the forward with y.  AGG: chunk aggregates for PAR.  CKPT_SEQ /
// CKPT_PAR: the forward without y that stores the state every kCkptEvery
// steps (the checkpoints the backward recomputes from).
// LOC: the forward with y of every chunk from a zero entering state, which
// also stores each chunk's end state and sum of Delta; the closed-form
// correction (fwd_correct_kernel) then adds the entering state's
// contribution once the scan over chunks has produced it.  CKPT_LOC: the same
// without y, storing the checkpoints of every chunk from zero with the sum of
// Delta up to each; the reader of a checkpoint adds exp(A_n cum) h_in,n.
// SEQ_SAVE, LOC_SAVE and PAR_SAVE: SEQ, LOC and PAR that also store the
// checkpoints (and, for LOC, the sums of Delta up to them) and the
// Delta-range flags, for a backward that reads them instead of re-running the
// forward.
enum StagedKind { KIND_SEQ = 0, KIND_PAR = 1, KIND_AGG = 2, KIND_CKPT_SEQ = 3, KIND_CKPT_PAR = 4,
                  KIND_LOC = 5, KIND_CKPT_LOC = 6, KIND_SEQ_SAVE = 7, KIND_LOC_SAVE = 8,
                  KIND_PAR_SAVE = 9 };
constexpr int kCkptEvery = 16;
enum UnitMode { MODE_SIG = 0, MODE_STRUCT = 1, MODE_GEN = 2 };

struct StagedArgs {
  FwdArgs f;
  int G;           // channel groups (batch rows x groups per row)
  int gpb;         // groups per batch row
  int K;           // chunks per group
  int chunk_len;   // time steps per chunk (a multiple of the tile length)
  int n_units;     // units handled by this launch
  int *counter;    // ticket counter, zero before the launch
  int *flags;      // SEQ: per group, number of chunks whose end state is published
  float *carry;    // SEQ: [G][NM][128] state handed to the next chunk
  float *agg_h;    // PAR: [G][K][NM][128] state each chunk produces from zero
  double *agg_S;   // PAR: [G][K][128] sum of Delta over each chunk
  float *hin;      // PAR: [G][K][NM][128] state entering each chunk
  float *ckpt;     // CKPT: [G][ceil(L/16)][NM][128] state before every 16th step
  uint64_t timeout_ns;
  int test_hook;   // 1: unit (group 0, chunk 0) never publishes (tests the bounded wait)
  int force_generic;  // 1: generic arithmetic for every channel
  // fused Delta projection (PROJ kernels): R padded to a multiple of 16, the
  // bytes of one pipeline stage and the number of stages; delta_out, when
  // set, receives delta in fp32 (batch, dim, L) for kernels that read it later
  int Rp = 0;
  uint32_t stage_bytes = 0;
  int nst = 0;
  float *delta_out = nullptr;
  // CKPT kinds, when set: [G][ceil(L/64)] flags, 1 where no step of any
  // channel of the group has its delta in structured_delta_range (the
  // backward's choice of arithmetic)
  unsigned char *range_flags = nullptr;
  int64_t n_flags = 0;
  // CKPT_LOC: [G][ceil(L/16)][128] sum of Delta from the chunk's start to each
  // checkpoint
  float *ckpt_cum = nullptr;
  int64_t n_ckpt_cum = 0;
  // element counts of the workspace buffers as allocated (the bounds-checking
  // build checks every index against them)
  int64_t n_carry = 0, n_agg = 0, n_aggS = 0, n_ckpt = 0, n_blk = 0;
  // LOC: [G][ceil(L/64)][128] sum of Delta from the start of the chunk to the
  // end of each 64-step block (where the correction of a block starts)
  float *blk_cum = nullptr;
};
constexpr int kCorrBlock = 64;  // steps per CTA of the closed-form correction

// Fused Delta projection: TMEM columns of one CTA (W rows in [0, Rp/2), two
// fp32 accumulators of one tile each after kProjAcc).
constexpr int kProjMaxRp = 256;
constexpr uint32_t kProjAcc = kProjMaxRp / 2;
constexpr uint32_t kProjTmemCols = 256;
// The thread that issues the projection MMAs: lane 0 of the last warp, so that
// it is not one of the threads that store y and issue the TMA loads.
constexpr int kMmaThread = 96;
// The forward's TMA producer (tile loads, unit tickets): a thread of warp 1,
// so that its work after each tile's barrier runs beside warp 0's store of
// the y tile instead of after it.
constexpr int kProdThread = 32;

// Thread's row d of W_dt (bf16, R per row) into its TMEM lane from column
// `taddr`'s on: Rp/2 columns of bf16 pairs (even k in the low half), zero
// beyond R (and for a channel past dim).  With R a multiple of 8 and the row
// 16-byte aligned, 16-byte loads, up to sixteen issued before the first use;
// else 2-byte loads.
__device__ __forceinline__ void proj_load_w(const __nv_bfloat16 *W, int64_t d, bool valid, int R, int Rp,
                                            uint32_t taddr) {
  const __nv_bfloat16 *wrow = W + (valid ? d * R : 0);
  if (R % 8 == 0 && (reinterpret_cast<uintptr_t>(wrow) & 15) == 0) {
    for (int c0 = 0; c0 < Rp / 16; c0 += 8) {  // eight 16-column groups per round of loads
      uint4 v[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int k = 16 * c0 + 8 * i;
        v[i] = (valid && k < R) ? __ldg(reinterpret_cast<const uint4 *>(wrow + k)) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        if (c0 + c < Rp / 16) {
          const uint32_t r[8] = {v[2 * c].x,     v[2 * c].y,     v[2 * c].z,     v[2 * c].w,
                                 v[2 * c + 1].x, v[2 * c + 1].y, v[2 * c + 1].z, v[2 * c + 1].w};
          tmem_st8(taddr + uint32_t(c0 + c) * 8u, r);
        }
      }
    }
    return;
  }
  for (int c8 = 0; c8 < Rp / 16; ++c8) {
    uint32_t r[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int k = 16 * c8 + 2 * i;
      const uint32_t lo = (valid && k < R) ? __bfloat16_as_ushort(wrow[k]) : 0u;
      const uint32_t hi = (valid && k + 1 < R) ? __bfloat16_as_ushort(wrow[k + 1]) : 0u;
      r[i] = lo | (hi << 16);
    }
    tmem_st8(taddr + uint32_t(c8) * 8u, r);
  }
}

// Shared-memory offsets of the fused-projection forward: a stage holds u,
// the dt_low tile (Rp rows), z, B and C.
struct ProjStage {
  uint32_t dt, z, B, C, bytes;
  __host__ __device__ ProjStage(int Rp) {
    dt = kTileBytes;
    z = dt + uint32_t(Rp) * kRowBytes;
    B = z + kTileBytes;
    C = B + kRawBytes;
    bytes = (C + kRawBytes + 1023u) & ~1023u;
  }
};

// ------------------------------------------------------------------ math

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2f(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcpf(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

using f2 = unsigned long long;  // two packed fp32 lanes for fma.rn.f32x2

__device__ __forceinline__ f2 pk(float lo, float hi) {
  f2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float lo_of(f2 v) { return __uint_as_float(unsigned(v)); }
__device__ __forceinline__ float hi_of(f2 v) { return __uint_as_float(unsigned(v >> 32)); }
__device__ __forceinline__ f2 fma2(f2 a, f2 b, f2 c) {
  f2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

// log(1 + e^v): a 5-term series of log1p(w) for w = e^v < 1/16 (relative
// error below 2e-7), log2(1 + w) ln 2 above, and v + e^-v for v > 15.
__device__ __forceinline__ float softplus_fast(float v) {
  const float w = ex2f(v * kLog2e);
  const float s = w * (1.f - w * (0.5f - w * (1.f / 3.f - w * (0.25f - w * 0.2f))));
  const float l = lg2f(1.f + w) * kLn2;
  const float r = w < 0.0625f ? s : l;
  return v > 15.f ? v + ex2f(-v * kLog2e) : r;
}

// Where the backward's structured forms keep their relative accuracy:
// Delta |A_0| in [1e-5, 6].  Above, the decay chain keeps the small decays'
// absolute but not their relative accuracy, which ddelta needs; below, the dA
// identity A dh/dA = Delta dh/dDelta - Bbar u cancels.  Either way the error
// is at fp32 resolution of the terms of a step in the range, so it matters
// only where no step is: a unit (or, with the fused projection, a tile) in
// which every step of every channel lies outside takes the generic
// arithmetic.  In terms of v = delta (before the bias): [lo, hi] with
// softplus(lo + bias) = 1e-5 / |A_0| and softplus(hi + bias) = 6 / |A_0|.
__device__ __forceinline__ void structured_delta_range(float A0, float bias, float &lo, float &hi) {
  const float ylo = 1e-5f / fabsf(A0), yhi = 6.f / fabsf(A0);
  lo = logf(expm1f(ylo)) - bias;
  hi = yhi + logf(-expm1f(-yhi)) - bias;
}
constexpr int kRangeBlock = 64;  // steps per range flag

// softplus(v) from e^-v and s = sigma(v), which the sigma form of the update
// already has: softplus(v) = -ln(1 - s) with 1 - s = e^-v s.  Below s = 1/16
// the series s + s^2/2 + ... + s^6/6 (relative error below 1e-8); above
// v = 15, v + e^-v (e^-v s would leave fp32's range).
__device__ __forceinline__ float softplus_from_sigmoid(float v, float ev, float s) {
  const float ser = s * (1.f + s * (0.5f + s * (1.f / 3.f + s * (0.25f + s * (0.2f + s * (1.f / 6.f))))));
  const float l = -lg2f(ev * s) * kLn2;
  const float r = s < 0.0625f ? ser : l;
  return v > 15.f ? v + ev : r;
}

// expm1(x) for x <= 0: a degree-6 Taylor polynomial for x > -1/4 (relative
// error below 6e-8), exp(x) - 1 below (no cancellation there).
__device__ __forceinline__ float expm1_neg(float x) {
  const float p = x * (1.f + x * (0.5f + x * (1.f / 6.f + x * (1.f / 24.f + x * (1.f / 120.f +
                  x * (1.f / 720.f))))));
  const float q = ex2f(x * kLog2e) - 1.f;
  return x > -0.25f ? p : q;
}

// Decays E(j) = expm1(j x), j = 1..NM, as pairs (E(2i+1), E(2i+2)), from
// E(1) and exp(x) = a1 by E(m+k) = E(m) + exp(m x) E(k).
template <int NM>
__device__ __forceinline__ void decay_pairs(float E1, float a1, f2 (&P)[NM / 2]) {
  const float E2 = fmaf(a1, E1, E1);
  P[0] = pk(E1, E2);
  if constexpr (NM >= 4) {
    const float a2 = 1.f + E2;
    P[1] = fma2(pk(a2, a2), P[0], pk(E2, E2));
  }
  if constexpr (NM >= 8) {
    const float E4 = hi_of(P[1]);
    const float a4 = 1.f + E4;
    const f2 A4 = pk(a4, a4), E4p = pk(E4, E4);
    P[2] = fma2(A4, P[0], E4p);
    P[3] = fma2(A4, P[1], E4p);
  }
  if constexpr (NM >= 16) {
    const float E8 = hi_of(P[3]);
    const float a8 = 1.f + E8;
    const f2 A8 = pk(a8, a8), E8p = pk(E8, E8);
#pragma unroll
    for (int i = 0; i < 4; ++i) P[4 + i] = fma2(A8, P[i], E8p);
  }
}

// One structured step for one channel: h_n += E(n+1) (h_n + B'_n u'),
// returns yinit + sum_n C_n h_n.  Brow / Crow are 16-byte aligned fp32 rows
// of B' = B/(n+1) and C for this time step.
template <int NM>
__device__ __forceinline__ float struct_update(f2 (&H)[NM / 2], const f2 (&P)[NM / 2], float up,
                                               float yinit, const float *Brow, const float *Crow) {
  const f2 U = pk(up, up);
  f2 Y0 = pk(yinit, 0.f), Y1 = pk(0.f, 0.f);  // two accumulators halve the chain
  if constexpr (NM == 2) {
    const f2 b = *reinterpret_cast<const f2 *>(Brow);
    const f2 c = *reinterpret_cast<const f2 *>(Crow);
    H[0] = fma2(P[0], fma2(b, U, H[0]), H[0]);
    Y0 = fma2(c, H[0], Y0);
  } else {
#pragma unroll
    for (int i = 0; i < NM / 2; i += 2) {
      const ulonglong2 b = *reinterpret_cast<const ulonglong2 *>(Brow + 2 * i);
      const ulonglong2 c = *reinterpret_cast<const ulonglong2 *>(Crow + 2 * i);
      H[i] = fma2(P[i], fma2(b.x, U, H[i]), H[i]);
      H[i + 1] = fma2(P[i + 1], fma2(b.y, U, H[i + 1]), H[i + 1]);
      Y0 = fma2(c.x, H[i], Y0);
      Y1 = fma2(c.y, H[i + 1], Y1);
    }
  }
  return (lo_of(Y0) + hi_of(Y0)) + (lo_of(Y1) + hi_of(Y1));
}

// One generic step for one channel (any A): per state, Abar = exp(Delta A_n)
// and Bbar/B = Delta psi(Delta A_n) with psi(x) = expm1(x)/x.  SCALED_B: the
// B row holds B_n / (n + 1) (the structured arithmetic's table).
template <int NM, bool SCALED_B = false>
__device__ __forceinline__ float generic_update(float (&h)[NM], float Delta, float uv, float yinit,
                                                const float (&A)[NM], const float (&A2)[NM],
                                                const float (&invA)[NM], const float *Brow,
                                                const float *Crow) {
  float y = yinit;
#pragma unroll
  for (int n = 0; n < NM; ++n) {
    const float x = Delta * A[n];
    const float a = ex2f(Delta * A2[n]);
    float p = fmaf(x, 1.f / 720.f, 1.f / 120.f);
    p = fmaf(x, p, 1.f / 24.f);
    p = fmaf(x, p, 1.f / 6.f);
    p = fmaf(x, p, 0.5f);
    p = fmaf(x, p, 1.f);
    const float E = fabsf(x) < 0.25f ? Delta * p : (a - 1.f) * invA[n];
    const float Bn = SCALED_B ? Brow[n] * float(n + 1) : Brow[n];
    h[n] = fmaf(a, h[n], E * (Bn * uv));
    y = fmaf(Crow[n], h[n], y);
  }
  return y;
}

// ------------------------------------------------------------ tile access

template <typename T> struct Vec;
template <> struct Vec<__nv_bfloat16> {
  static constexpr int kN = 8;
  __device__ static void unpack(const uint4 &v, float (&o)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      o[2 * i] = __uint_as_float(w[i] << 16);
      o[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  __device__ static uint4 pack(const float (&o)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 p = __floats2bfloat162_rn(o[2 * i], o[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t *>(&p);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
  }
};
template <> struct Vec<float> {
  static constexpr int kN = 4;
  __device__ static void unpack(const uint4 &v, float (&o)[4]) {
    o[0] = __uint_as_float(v.x);
    o[1] = __uint_as_float(v.y);
    o[2] = __uint_as_float(v.z);
    o[3] = __uint_as_float(v.w);
  }
  __device__ static uint4 pack(const float (&o)[4]) {
    return make_uint4(__float_as_uint(o[0]), __float_as_uint(o[1]), __float_as_uint(o[2]),
                      __float_as_uint(o[3]));
  }
};

// Byte offset of 16-byte chunk j of row r in a 64-byte-row tile written by
// TMA with 64-byte swizzling (chunk index XOR bits 8:7 of the address).
__device__ __forceinline__ int swz64(int r, int j) { return r * kRowBytes + ((j ^ ((r >> 1) & 3)) << 4); }

__device__ __forceinline__ float raw_to_f(const __nv_bfloat16 *p, int i) { return __bfloat162float(p[i]); }
__device__ __forceinline__ float raw_to_f(const float *p, int i) { return p[i]; }

// --------------------------------------------------------------- the kernel

template <typename T, int NM>
struct StagedLayout {
  static constexpr int TT = kRowBytes / (int)sizeof(T);  // time steps per tile
  static constexpr int VEC = 16 / (int)sizeof(T);        // time steps per 16-byte chunk
  static constexpr int NV = TT / VEC;                    // chunks per row
  static constexpr int BSTR = (NM < 4 ? 4 : NM) + 4;     // fp32 row stride of B' / C
  static constexpr int OFF_Y = kStages * kStageBytes;
  static constexpr int OFF_BS = OFF_Y + 2 * kTileBytes;
  static constexpr int OFF_CS = OFF_BS + 2 * TT * BSTR * 4;   // B' and C: two buffers each
  static constexpr int OFF_BAR = OFF_CS + 2 * TT * BSTR * 4;
  static constexpr int OFF_Q = OFF_BAR + 8 * 5;  // stage barriers (3) + MMA barriers (2)
  static constexpr int BYTES = OFF_Q + 16 * 4;
  static constexpr int ALLOC = BYTES + 1024;  // slack to align the base to 1 KB
};

// CONV: the u tiles hold the input x of the block's causal depthwise
// convolution, and each thread turns its row into u = SiLU(conv(x)) as it
// reads it (the three inputs before the unit's first step come from global
// memory; after that the last three stay in registers).
//
// PROJ: delta is not read.  The tiles of the low-rank projection's input
// dt_low (Rp x TT, bf16) come through the pipeline instead, the CTA's 128 rows
// of W_dt sit in tensor memory, and one elected thread issues per tile the
// tcgen05 MMA delta_tile (128 channels x TT steps, fp32 in TMEM) = W_g (128 x
// Rp) . dt_low_tile (Rp x TT); each thread then reads its own channel's TT
// values of delta with tcgen05.ld.  The MMA of the next tile is issued while
// the current one is scanned, into the other of two accumulators.
template <typename T, int NM, int KIND, bool CONV = false, bool PROJ = false>
__global__ void __launch_bounds__(kSThreads, 2)
    fwd_staged_kernel(const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_d,
                      const __grid_constant__ CUtensorMap tm_z, const __grid_constant__ CUtensorMap tm_y,
                      const __grid_constant__ CUtensorMap tm_B, const __grid_constant__ CUtensorMap tm_C,
                      const StagedArgs p) {
  using Lay = StagedLayout<T, NM>;
  constexpr int TT = Lay::TT, VEC = Lay::VEC, NV = Lay::NV, BSTR = Lay::BSTR;
  static_assert(!PROJ || (std::is_same<T, __nv_bfloat16>::value && !CONV),
                "the fused projection takes bf16 operands and no convolution prologue");
  constexpr bool kLoc = KIND == KIND_LOC || KIND == KIND_LOC_SAVE;  // y from zero chunk starts
  constexpr bool kOut = KIND == KIND_SEQ || KIND == KIND_PAR || kLoc || KIND == KIND_SEQ_SAVE ||
                        KIND == KIND_PAR_SAVE;  // stores y
  constexpr bool kAgg = KIND == KIND_AGG || kLoc || KIND == KIND_CKPT_LOC;  // chunk aggregates
  constexpr bool kSeq = KIND == KIND_SEQ || KIND == KIND_CKPT_SEQ || KIND == KIND_SEQ_SAVE;
  constexpr bool kPar = KIND == KIND_PAR || KIND == KIND_CKPT_PAR || KIND == KIND_PAR_SAVE;
  constexpr bool kCkpt = KIND == KIND_CKPT_SEQ || KIND == KIND_CKPT_PAR || KIND == KIND_CKPT_LOC ||
                         KIND == KIND_SEQ_SAVE || KIND == KIND_LOC_SAVE || KIND == KIND_PAR_SAVE;
  // checkpoints of chunks run from zero: stored with the sums of Delta up to them
  constexpr bool kCkptCum = KIND == KIND_CKPT_LOC || KIND == KIND_LOC_SAVE;

  // Offsetting the __shared__ array itself (not a cast integer) keeps every
  // derived pointer in the shared address space, so the compiler emits
  // shared-memory loads and stores instead of generic ones.
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  // stage geometry: fixed, or (PROJ) set by the dt_low tile's rows
  const ProjStage ps(PROJ ? p.Rp : 0);
  const uint32_t SST = PROJ ? ps.bytes : uint32_t(kStageBytes);
  const int NST = PROJ ? p.nst : kStages;
  const uint32_t OFF_Z = PROJ ? ps.z : 2u * kTileBytes;
  const uint32_t OFF_B = PROJ ? ps.B : 3u * kTileBytes;
  const uint32_t OFF_C = PROJ ? ps.C : 3u * kTileBytes + kRawBytes;
  const uint32_t OFF_Y = uint32_t(NST) * SST;
  const uint32_t OFF_BS = OFF_Y + 2 * kTileBytes;
  const uint32_t OFF_CS = OFF_BS + 2 * TT * BSTR * 4;
  const uint32_t OFF_BAR = OFF_CS + 2 * TT * BSTR * 4;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_BAR);  // [stages], then 2 MMA barriers
  uint64_t *mma_bar = bars + 3;
  int *q = reinterpret_cast<int *>(sm + OFF_BAR + 8 * 5);  // [0..7] ticket ring, [8] abort, [12] TMEM
  float *Bs = reinterpret_cast<float *>(sm + OFF_BS);
  float *Cs = reinterpret_cast<float *>(sm + OFF_CS);

  const int tid = threadIdx.x;
  const FwdArgs &f = p.f;
  const int N = f.N;
  const bool has_z = kOut && f.z != nullptr;
  const uint32_t tile_bytes = (kOut ? (has_z ? 2u : 1u) : 1u) * kTileBytes +
                              (PROJ ? uint32_t(p.Rp) * kRowBytes : kTileBytes) +
                              (kOut ? 2u : 1u) * uint32_t(N) * kRowBytes;
  // fused projection: the MMA's instruction descriptor (M = 128 channels,
  // N = TT steps; A = W from TMEM, K-major; B = dt_low, MN-major) and TMEM
  [[maybe_unused]] constexpr uint32_t kIdesc = mma_idesc_bf16(128, TT, false, true);
  [[maybe_unused]] uint32_t tbase = 0;
  [[maybe_unused]] int mma_issued = -1;  // kMmaThread: last tile whose MMA it issued

  if (tid == 0) {
#pragma unroll
    for (int s = 0; s < kStages; ++s) mbar_init(&bars[s], 1);
    if (PROJ) {
      mbar_init(&mma_bar[0], 1);
      mbar_init(&mma_bar[1], 1);
    }
    fence_barrier_init();
    prefetch_tensormap(&tm_u);
    prefetch_tensormap(&tm_d);
    prefetch_tensormap(&tm_B);
    if (kOut) {
      prefetch_tensormap(&tm_C);
      prefetch_tensormap(&tm_y);
      if (has_z) prefetch_tensormap(&tm_z);
    }
    q[8] = 0;
  }
  if constexpr (PROJ) {
    if (tid < 32) {
      tmem_alloc(reinterpret_cast<uint32_t *>(&q[12]), kProjTmemCols);
      tmem_relinquish();
    }
  }
  __syncthreads();
  if constexpr (PROJ) {
    tc_fence_after_sync();
    tbase = uint32_t(q[12]);
  }

  // Issues (kMmaThread) the projection MMAs of consumed-tile index `ct` into
  // accumulator ct & 1, once the tile's dt_low rows have landed.
  [[maybe_unused]] auto issue_mma = [&](int ct) {
    const int stg = ct % NST;
    if (!mbar_wait_bounded(&bars[stg], uint32_t(ct / NST) & 1u, p.timeout_ns)) {
      record_timeout();
      q[8] = 1;
      return;
    }
    tc_fence_after_sync();
    const uint32_t acc = tbase + kProjAcc + uint32_t(ct & 1) * TT;
    // 16 rows of dt_low (two 8-row swizzle atoms of 512 bytes) per MMA: the
    // descriptor's start address (in 16-byte units) advances by 1024 bytes
    const uint64_t bdesc0 = smem_desc(smem_u32(sm + stg * SST + ps.dt), 16u, 512u, 4u);
    for (int kk = 0; kk < p.Rp / 16; ++kk)
      mma_ts(acc, tbase + uint32_t(kk) * 8u, bdesc0 + uint64_t(kk) * 64u, kIdesc, kk > 0);
    mma_commit(&mma_bar[ct & 1]);
    mma_issued = ct;
  };

  // ---- producer state (meaningful in thread 0 only)
  int p_ticket = 0, p_tile = 0, p_ntiles = 0, p_tail = 0, p_issued = 0;
  bool p_done = false;

  auto unit_tiles = [&](int ticket) {
    const int k = ticket / p.G;
    const int64_t t0 = int64_t(k) * p.chunk_len;
    const int64_t t1 = std::min<int64_t>(f.L, t0 + p.chunk_len);
    return int((t1 - t0 + TT - 1) / TT);
  };

  // Issues the next tile of this CTA's stream into stage p_issued % kStages.
  // In the sequential hand-off the next unit is claimed only once the current
  // one is finished (claiming early would let a unit be claimed while its
  // predecessor is still queued behind another unit, and waits would pile up).
  auto produce = [&](bool may_claim) {
    if (p_done) return;
    if (p_tile == p_ntiles) {
      if (!may_claim) return;
      p_ticket = atomicAdd(p.counter, 1);
      q[p_tail & 7] = p_ticket;
      ++p_tail;
      if (p_ticket >= p.n_units) {
        p_done = true;
        return;
      }
      p_ntiles = unit_tiles(p_ticket);
      p_tile = 0;
    }
    const int g = p_ticket % p.G, k = p_ticket / p.G;
    const int b = g / p.gpb, d0 = (g % p.gpb) * kSThreads;
    const int t0 = k * p.chunk_len + p_tile * TT;
    const int stage = p_issued % NST;
    unsigned char *st = sm + stage * SST;
    uint64_t *bar = &bars[stage];
    mbar_arrive_expect_tx(bar, tile_bytes);
    tma_load_3d(st, &tm_u, bar, t0, d0, b);
    if (PROJ) tma_load_3d(st + kTileBytes, &tm_d, bar, t0, 0, b);  // dt_low rows 0..Rp-1
    else tma_load_3d(st + kTileBytes, &tm_d, bar, t0, d0, b);
    if (has_z) tma_load_3d(st + OFF_Z, &tm_z, bar, t0, d0, b);
    tma_load_3d(st + OFF_B, &tm_B, bar, t0, 0, b);
    if (kOut) tma_load_3d(st + OFF_C, &tm_C, bar, t0, 0, b);
    ++p_tile;
    ++p_issued;
  };

  constexpr bool kLookahead = !kSeq;
  if (tid == kProdThread) {
    produce(true);
    for (int s = 1; s < NST; ++s) produce(kLookahead);
  }

  int head = 0;   // consumer position in the ticket ring
  int ctile = 0;  // tiles consumed by this CTA
  bool aborted = false;

  while (true) {
    __syncthreads();
    const int ticket = q[head & 7];
    ++head;
    if (ticket >= p.n_units) break;
    const int g = ticket % p.G, k = ticket / p.G;
    const int b = g / p.gpb, d0 = (g % p.gpb) * kSThreads;
    const int d = d0 + tid;
    const bool valid = d < f.dim;
    const int64_t tbeg = int64_t(k) * p.chunk_len;
    const int64_t tend = std::min<int64_t>(f.L, tbeg + p.chunk_len);
    const int ntiles = int((tend - tbeg + TT - 1) / TT);

    // per-channel parameters and the arithmetic this unit can use
    float Arow[NM];
#pragma unroll
    for (int n = 0; n < NM; ++n) Arow[n] = (valid && n < N) ? f.A[int64_t(d) * N + n] : -float(n + 1);
    if (valid) {  // padding states (n >= N) carry B = C = 0; give them a finite A of the same form
      const float pad0 = (Arow[0] < 0.f && isfinite(Arow[0])) ? Arow[0] : -1.f;
#pragma unroll
      for (int n = 1; n < NM; ++n)
        if (n >= N) Arow[n] = float(n + 1) * pad0;
    }
    const float bias = (valid && f.bias) ? f.bias[d] : 0.f;
    const float Dd = (valid && f.D && kOut) ? f.D[d] : 0.f;
    bool structured = Arow[0] < 0.f && isfinite(Arow[0]);
#pragma unroll
    for (int n = 1; n < NM; ++n) structured = structured && (Arow[n] == float(n + 1) * Arow[0]);
    const bool sig = structured && Arow[0] == -1.f;
    // (CKPT with range flags) the structured range of delta + bias, empty
    // for channels that are not checked
    [[maybe_unused]] float rlo = 3.4e38f, rhi = -3.4e38f;
    [[maybe_unused]] bool rin = false;  // a step of the current 64-step block in range
    if constexpr (kCkpt) {
      if (p.range_flags && valid && Arow[0] < 0.f && isfinite(Arow[0])) {
        structured_delta_range(Arow[0], 0.f, rlo, rhi);
      }
    }
    if constexpr (PROJ) {
      // This group's rows of W_dt into TMEM columns [0, Rp/2), bf16 pairs
      // (even k in the low half).  The previous unit's MMAs have completed:
      // its threads waited for every one of them.
      proj_load_w(static_cast<const __nv_bfloat16 *>(f.W_dt), d, valid, f.R, p.Rp,
                  tmem_at(tbase, uint32_t(tid >> 5) * 32u, 0));
      tmem_st_wait();
      tc_fence_before_sync();
      __syncthreads();
      if (tid == kMmaThread) issue_mma(ctile);
    }
    int mode = MODE_GEN;
    if (!p.force_generic) {
      if (__syncthreads_and(sig)) mode = MODE_SIG;
      else if (__syncthreads_and(structured)) mode = MODE_STRUCT;
    }

    // state entering the chunk
    float hs[NM];
#pragma unroll
    for (int n = 0; n < NM; ++n) hs[n] = 0.f;
    if (kSeq && k > 0) {
      if (tid == 0 && !wait_flag_geq(p.flags + g, k, p.timeout_ns)) {
        record_timeout();
        q[8] = 1;
      }
      __syncthreads();
      if (q[8]) {
        aborted = true;
        break;
      }
#pragma unroll
      for (int n = 0; n < NM; ++n) {
        const int64_t i = (int64_t(g) * NM + n) * kSThreads + tid;
        hs[n] = in_bounds(i, p.n_carry) ? __ldcg(p.carry + i) : 0.f;
      }
    } else if (kPar && k > 0) {
#pragma unroll
      for (int n = 0; n < NM; ++n)
      {
        const int64_t i = ((int64_t(g) * p.K + k) * NM + n) * kSThreads + tid;
        hs[n] = in_bounds(i, p.n_agg) ? __ldcg(p.hin + i) : 0.f;
      }
    }

    double Ssum = 0.0;  // sum of Delta over the chunk (aggregate pass)

    // convolution prologue: the filter and x at the three steps before the chunk
    ConvFilter cf = {0.f, 0.f, 0.f, 1.f, 0.f};
    float xm1 = 0.f, xm2 = 0.f, xm3 = 0.f;
    if constexpr (CONV) {
      if (valid) {
        cf = load_conv_filter(f.conv_w, f.conv_b, f.conv_width, d);
        if (tbeg > 0) {  // chunks start at multiples of 64 steps
          const T *xr = static_cast<const T *>(f.u) + (int64_t(b) * f.dim + d) * f.L + tbeg;
          if (in_bounds((int64_t(b) * f.dim + d) * f.L + tbeg - 3, f.batch * f.dim * f.L)) {
            xm3 = to_f(xr[-3]);
            xm2 = to_f(xr[-2]);
            xm1 = to_f(xr[-1]);
          }
        }
      }
    }

    // Runs every tile of this unit with the arithmetic of mode M.
    auto run = [&](auto mode_tag) {
      constexpr int M = decltype(mode_tag)::value;
      f2 H[NM / 2];
      float h[NM];
      float A2[NM], invA[NM];
      if constexpr (M == MODE_GEN) {
#pragma unroll
        for (int n = 0; n < NM; ++n) {
          h[n] = hs[n];
          A2[n] = Arow[n] * kLog2e;
          invA[n] = Arow[n] != 0.f ? 1.f / Arow[n] : 0.f;
        }
      } else {
#pragma unroll
        for (int i = 0; i < NM / 2; ++i) H[i] = pk(hs[2 * i], hs[2 * i + 1]);
      }
      const float A0 = Arow[0];
      const float invA0 = 1.f / A0;

      // Waits for the tile in stage slot `ct % kStages` and writes its B and C
      // rows as fp32, time-major, into buffer ct & 1 (B scaled by 1/(n+1) for
      // the structured arithmetic).  The tables are double-buffered so that
      // the next tile's are written at the end of the current one, under the
      // same barrier as the y tile.
      auto stage_tables = [&](int ct) {
        const int stg = ct % NST;
        if (!mbar_wait_bounded(&bars[stg], uint32_t(ct / NST) & 1u, p.timeout_ns)) {
          record_timeout();
          q[8] = 1;
        }
        const unsigned char *sst = sm + stg * SST;
        const T *Braw = reinterpret_cast<const T *>(sst + OFF_B);
        const T *Craw = reinterpret_cast<const T *>(sst + OFF_C);
        float *Bd = Bs + (ct & 1) * TT * BSTR;
        float *Cd = Cs + (ct & 1) * TT * BSTR;
        constexpr int ITEMS = NM * (TT / 4);
        for (int w = tid; w < (kOut ? 2 : 1) * ITEMS; w += kSThreads) {
          const bool isC = w >= ITEMS;
          const int r = isC ? w - ITEMS : w;
          const int n = r % NM, tg = r / NM;
          const T *src = (isC ? Craw : Braw) + n * TT + 4 * tg;
          float *dst = (isC ? Cd : Bd) + 4 * tg * BSTR + n;
          const float scale = (!isC && M != MODE_GEN) ? 1.f / float(n + 1) : 1.f;
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i * BSTR] = n < N ? raw_to_f(src, i) * scale : 0.f;
        }
      };
      stage_tables(ctile);
      __syncthreads();
      if (q[8]) return;

      for (int it = 0; it < ntiles; ++it, ++ctile) {
        [[maybe_unused]] float Stile = 0.f;  // Delta summed over the tile (fp32; fp64 across tiles)
        const int stage = ctile % NST;
        unsigned char *st = sm + stage * SST;
        const float *Bt = Bs + (ctile & 1) * TT * BSTR;
        const float *Ct = Cs + (ctile & 1) * TT * BSTR;
        const int64_t t0 = tbeg + int64_t(it) * TT;
        const unsigned char *su = st;
        [[maybe_unused]] const unsigned char *sd = st + kTileBytes;
        const unsigned char *sz = st + OFF_Z;
        unsigned char *sy = sm + OFF_Y + (ctile & 1) * kTileBytes;
        [[maybe_unused]] uint32_t dacc = 0;
        [[maybe_unused]] bool mma_next = false;  // (kMmaThread) the next tile's MMA is issued
        if constexpr (PROJ) {  // this tile's delta: wait for its MMA
          if (!mbar_wait_bounded(&mma_bar[ctile & 1], uint32_t(ctile >> 1) & 1u, p.timeout_ns)) {
            record_timeout();
            q[8] = 1;
          }
          tc_fence_after_sync();
          dacc = tmem_at(tbase + kProjAcc + uint32_t(ctile & 1) * TT, uint32_t(tid >> 5) * 32u, 0);
        }
        for (int j = 0; j < NV; ++j) {
          if (t0 + int64_t(j) * VEC >= tend) break;  // past the end of the sequence
          if constexpr (kCkpt) {
            const int64_t tj = t0 + int64_t(j) * VEC;
            if (tj % kCkptEvery == 0) {
              const int64_t ci = ((int64_t(g) * ((f.L + kCkptEvery - 1) / kCkptEvery) +
                                   tj / kCkptEvery) * NM) * kSThreads + tid;
              float *dst = p.ckpt + (in_bounds(ci + (NM - 1) * kSThreads, p.n_ckpt) ? ci : 0);
              if constexpr (kCkptCum) {  // Delta summed from the chunk's start
                const int64_t cc = (int64_t(g) * ((f.L + kCkptEvery - 1) / kCkptEvery) + tj / kCkptEvery) *
                                       kSThreads + tid;
                if (in_bounds(cc, p.n_ckpt_cum)) p.ckpt_cum[cc] = float(Ssum + double(Stile));
              }
              if constexpr (M == MODE_GEN) {
#pragma unroll
                for (int n = 0; n < NM; ++n) dst[n * kSThreads] = h[n];
              } else {
#pragma unroll
                for (int i = 0; i < NM / 2; ++i) {
                  dst[(2 * i) * kSThreads] = lo_of(H[i]);
                  dst[(2 * i + 1) * kSThreads] = hi_of(H[i]);
                }
              }
            }
          }
          const int off = swz64(tid, j);
          float uv[VEC], dv[VEC], zv[VEC], yv[VEC];
          Vec<T>::unpack(*reinterpret_cast<const uint4 *>(su + off), uv);
          if constexpr (CONV) {  // x -> u = SiLU(conv(x)), in time order
#pragma unroll
            for (int i = 0; i < VEC; ++i) {
              const float xv = uv[i];
              const float pre = conv_pre(cf, xm3, xm2, xm1, xv);
              uv[i] = pre * rcpf(1.f + ex2f(-pre * kLog2e));
              xm3 = xm2;
              xm2 = xm1;
              xm1 = xv;
            }
          }
          if constexpr (PROJ) {
            static_assert(VEC == 8, "eight steps per 16-byte chunk");
            tmem_ld8(dacc + uint32_t(j) * 8u, dv);
            tmem_ld_wait();
            if (p.delta_out && valid &&
                in_bounds((int64_t(b) * f.dim + d) * f.L + t0 + int64_t(j) * VEC + 7, f.batch * f.dim * f.L)) {
              float *o = p.delta_out + (int64_t(b) * f.dim + d) * f.L + t0 + int64_t(j) * VEC;
              *reinterpret_cast<float4 *>(o) = make_float4(dv[0], dv[1], dv[2], dv[3]);
              *reinterpret_cast<float4 *>(o + 4) = make_float4(dv[4], dv[5], dv[6], dv[7]);
            }
            // the next tile's MMA, into the other accumulator: as soon as its
            // dt_low tile has landed, at this tile's last chunk at the latest
            if (tid == kMmaThread && !mma_next && it + 1 < ntiles && j >= 1 &&
                (j == NV - 1 || mbar_test_wait(&bars[(ctile + 1) % NST], uint32_t((ctile + 1) / NST) & 1u))) {
              issue_mma(ctile + 1);
              mma_next = true;
            }
            __syncwarp();
          } else {
            Vec<T>::unpack(*reinterpret_cast<const uint4 *>(sd + off), dv);
          }
          if (has_z) Vec<T>::unpack(*reinterpret_cast<const uint4 *>(sz + off), zv);
#pragma unroll
          for (int i = 0; i < VEC; ++i) {
            const int tl = j * VEC + i;
            const float *Brow = Bt + tl * BSTR;
            const float *Crow = Ct + tl * BSTR;
            const float v = dv[i] + bias;
            if constexpr (kCkpt) rin = rin || (v >= rlo && v <= rhi);
            float y0;
            if constexpr (M == MODE_SIG) {
              // e^-v overflows below v = -88; above +88 it flushes to 0 and
              // the decays are exactly 0 (sigma = 1), as they should be
              const float vc = fmaxf(v, -87.f);
              const float ev = ex2f(-vc * kLog2e);  // e^-v
              const float s = rcpf(1.f + ev);      // sigma(v) = 1 - exp(-Delta)
              f2 P[NM / 2];
              decay_pairs<NM>(-s, ev * s, P);
              if (kOut) {
                y0 = struct_update<NM>(H, P, -uv[i], Dd * uv[i], Brow, Crow);
              } else {
                struct_update<NM>(H, P, -uv[i], 0.f, Brow, Brow);
              }
              if constexpr (kAgg) Stile += softplus_from_sigmoid(v, ev, s);
            } else if constexpr (M == MODE_STRUCT) {
              const float Delta = softplus_fast(v);
              const float E1 = expm1_neg(Delta * A0);
              f2 P[NM / 2];
              decay_pairs<NM>(E1, 1.f + E1, P);
              if (kOut) {
                y0 = struct_update<NM>(H, P, uv[i] * invA0, Dd * uv[i], Brow, Crow);
              } else {
                struct_update<NM>(H, P, uv[i] * invA0, 0.f, Brow, Brow);
              }
              if constexpr (kAgg) Stile += Delta;
            } else {
              const float Delta = softplus_fast(v);
              y0 = generic_update<NM>(h, Delta, uv[i], Dd * uv[i], Arow, A2, invA, Brow,
                                      kOut ? Crow : Brow);
              if constexpr (kAgg) Stile += Delta;
            }
            if (kOut) {
              if (has_z) {
                const float ez = ex2f(-zv[i] * kLog2e);
                y0 *= zv[i] * rcpf(1.f + ez);
              }
              yv[i] = y0;
            }
          }
          if (kOut) *reinterpret_cast<uint4 *>(sy + off) = Vec<T>::pack(yv);
        }
        if constexpr (kAgg) Ssum += double(Stile);
        if constexpr (kLoc) {  // the block's running sum, where a block ends
          if ((t0 + TT) % kCorrBlock == 0 || it + 1 == ntiles) {
            const int64_t bi = (int64_t(g) * ((f.L + kCorrBlock - 1) / kCorrBlock) + t0 / kCorrBlock) *
                               kSThreads + tid;
            if (in_bounds(bi, p.n_blk)) p.blk_cum[bi] = float(Ssum);
          }
        }
        if (it + 1 < ntiles) stage_tables(ctile + 1);
        if (kOut) fence_proxy_async_smem();
        if (PROJ) tc_fence_before_sync();
        if (kCkpt && p.range_flags && ((t0 + TT) % kRangeBlock == 0 || it + 1 == ntiles)) {
          // (uniform over the CTA) the flag of the 64-step block this tile ends
          const bool any_in = __syncthreads_or(rin);
          rin = false;
          const int64_t fi = int64_t(g) * ((f.L + kRangeBlock - 1) / kRangeBlock) + t0 / kRangeBlock;
          if (tid == 0 && in_bounds(fi, p.n_flags)) p.range_flags[fi] = any_in ? 0 : 1;
        } else {
          __syncthreads();
        }
        if (q[8]) return;
        // the y tile's store (warp 0) and the next loads (warp 1) in parallel
        if (kOut && tid == 0) {
          tma_store_3d(&tm_y, sy, int(t0), d0, b);
          bulk_commit();
          bulk_wait_read<1>();
        }
        if (tid == kProdThread) produce(kLookahead);
      }
      if constexpr (M == MODE_GEN) {
#pragma unroll
        for (int n = 0; n < NM; ++n) hs[n] = h[n];
      } else {
#pragma unroll
        for (int i = 0; i < NM / 2; ++i) {
          hs[2 * i] = lo_of(H[i]);
          hs[2 * i + 1] = hi_of(H[i]);
        }
      }
    };

    if (mode == MODE_SIG) run(std::integral_constant<int, MODE_SIG>{});
    else if (mode == MODE_STRUCT) run(std::integral_constant<int, MODE_STRUCT>{});
    else run(std::integral_constant<int, MODE_GEN>{});
    if (q[8]) {
      aborted = true;
      break;
    }

    // hand the end state on
    if (kAgg) {
#pragma unroll
      for (int n = 0; n < NM; ++n)
        if (in_bounds(((int64_t(g) * p.K + k) * NM + n) * kSThreads + tid, p.n_agg))
          p.agg_h[((int64_t(g) * p.K + k) * NM + n) * kSThreads + tid] = hs[n];
      if (in_bounds((int64_t(g) * p.K + k) * kSThreads + tid, p.n_aggS))
        p.agg_S[(int64_t(g) * p.K + k) * kSThreads + tid] = Ssum;
    } else if (k == p.K - 1) {
      if (kOut && valid && f.last_state) {
#pragma unroll
        for (int n = 0; n < NM; ++n)
          if (n < N && in_bounds((int64_t(b) * f.dim + d) * N + n, f.batch * f.dim * N))
            f.last_state[(int64_t(b) * f.dim + d) * N + n] = hs[n];
      }
    } else if (kSeq) {
#pragma unroll
      for (int n = 0; n < NM; ++n)
        if (in_bounds((int64_t(g) * NM + n) * kSThreads + tid, p.n_carry))
          p.carry[(int64_t(g) * NM + n) * kSThreads + tid] = hs[n];
      __threadfence();
      __syncthreads();
      if (tid == 0 && !(p.test_hook == 1 && g == 0 && k == 0)) st_release_gpu(p.flags + g, k + 1);
    }
    if (!kLookahead && tid == kProdThread) {  // claim the next unit and fill the free stages
      produce(true);
      while (!p_done && p_issued < ctile + NST && p_tile < p_ntiles) produce(false);
    }
  }

  // Drain: every TMA load this CTA issued must land before it exits, and
  // (PROJ) every MMA it issued must complete before TMEM is freed.
  __syncthreads();
  if (tid == kProdThread && aborted) {
    for (int t = ctile; t < p_issued; ++t)
      mbar_wait_bounded(&bars[t % NST], uint32_t(t / NST) & 1u, p.timeout_ns);
  }
  if (tid == 0) bulk_wait<0>();
  if (PROJ && tid == kMmaThread && mma_issued >= 0)
    mbar_wait_bounded(&mma_bar[mma_issued & 1], uint32_t(mma_issued >> 1) & 1u, p.timeout_ns);
  if constexpr (PROJ) {
    tc_fence_before_sync();
    __syncthreads();
    if (tid < 32) {
      tc_fence_after_sync();
      tmem_dealloc(tbase, kProjTmemCols);
    }
  }
}

// The scan over chunks of the three-phase carry, as a parallel scan of the
// associative operator of affine maps ("Mamba: Linear-Time Sequence Modeling
// with Selective State Spaces", trishampatil.com walk-through, Part III
// section 2, "Parallel scan: why a recurrence isn't as sequential as it
// looks"; the chunking of section 3.3 of the paper-graph-ui summary).  Chunk
// k maps an entering state h to exp(A_n S_k) h + hl_k (S_k its sum of Delta,
// hl_k the state it produces from zero); two chunks compose as
//     (S_a, hl_a) then (S_b, hl_b)  =  (S_a + S_b, exp(A_n S_b) hl_a + hl_b).
// With few chunks (K <= kChunkScanSerialK) one thread takes a sequence -- one
// (channel group, state, channel) -- in order, its loads issued eight chunks
// at a time.  With more, a sequence is scanned by the CTA's four warps in
// blocks of 128 chunks: a Kogge-Stone scan within each warp by shuffles, the
// warp totals combined through shared memory, the state carried from block to
// block.  The chunk-entering values go back to HBM.  Element e of a scan is
// chunk e (forward) or chunk K-1-e (REVERSE: the adjoint of the backward runs
// from the end).  fp32 with the hardware exp2.
struct ChunkScanIO {
  const double *S;   // [G][K][128] sum of Delta per chunk
  const float *hl;   // [G][K][NM][128] value each chunk produces from zero
  float *hin;        // [G][K][NM][128] value entering each chunk
  const float *A;    // (dim, N)
  int G, K, gpb, N;
  int64_t dim;
};
// (its buffers hold G * K * 128 and G * K * NM * 128 elements)

constexpr int kChunkScanSerialK = 32;

// CTAs of 128 threads for the scan of `nseq` sequences of K chunks.
inline int64_t chunk_scan_grid(int64_t nseq, int K) {
  return K <= kChunkScanSerialK ? (nseq + 127) / 128 : nseq;
}

template <int NM, bool REVERSE>
__global__ void __launch_bounds__(128) chunk_scan_kernel(const ChunkScanIO io) {
  __shared__ float wS[4], wh[4];
  __shared__ float carry;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const bool serial = io.K <= kChunkScanSerialK;
  const int64_t seq = serial ? int64_t(blockIdx.x) * 128 + threadIdx.x : int64_t(blockIdx.x);
  const int64_t nseq = int64_t(io.G) * NM * kSThreads;
  if (seq >= nseq) return;  // (uniform per CTA when not serial)
  const int c = int(seq % kSThreads), n = int((seq / kSThreads) % NM), g = int(seq / (kSThreads * NM));
  const int d = (g % io.gpb) * kSThreads + c;
  const float A2 = (d < io.dim && n < io.N) ? io.A[int64_t(d) * io.N + n] * kLog2e : 0.f;
  const int64_t nk = int64_t(io.G) * io.K;
  if (serial) {
    float h = 0.f;  // the value entering element e
    for (int e0 = 0; e0 < io.K; e0 += 8) {
      float S[8], hl[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = e0 + i, k = REVERSE ? io.K - 1 - e : e;
        const bool live = e < io.K - 1 && in_bounds(int64_t(g) * io.K + k, nk);  // the last map is never applied
        const int64_t base = int64_t(g) * io.K + (live ? k : 0);
        S[i] = live ? float(io.S[base * kSThreads + c]) : 0.f;
        hl[i] = live ? io.hl[(base * NM + n) * kSThreads + c] : 0.f;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = e0 + i, k = REVERSE ? io.K - 1 - e : e;
        if (e < io.K && in_bounds(int64_t(g) * io.K + k, nk))
          io.hin[((int64_t(g) * io.K + k) * NM + n) * kSThreads + c] = h;
        h = fmaf(ex2f(A2 * S[i]), h, hl[i]);
      }
    }
    return;
  }
  if (threadIdx.x == 0) carry = 0.f;
  __syncthreads();
  for (int k0 = 0; k0 < io.K; k0 += 128) {
    const int e = k0 + int(threadIdx.x);  // element of the scan
    const int k = REVERSE ? io.K - 1 - e : e;
    const bool live = e < io.K - 1 && in_bounds(int64_t(g) * io.K + k, nk);
    const int64_t base = int64_t(g) * io.K + (live ? k : 0);
    float S = live ? float(io.S[base * kSThreads + c]) : 0.f;
    float h = live ? io.hl[(base * NM + n) * kSThreads + c] : 0.f;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {  // inclusive scan within the warp
      const float So = __shfl_up_sync(0xffffffffu, S, o);
      const float ho = __shfl_up_sync(0xffffffffu, h, o);
      if (lane >= o) {
        h = fmaf(ex2f(A2 * S), ho, h);
        S = So + S;
      }
    }
    if (lane == 31) {
      wS[warp] = S;
      wh[warp] = h;
    }
    __syncthreads();
    float cin = carry;  // through the earlier blocks, then the earlier warps
    for (int w = 0; w < warp; ++w) cin = fmaf(ex2f(A2 * wS[w]), cin, wh[w]);
    float Se = __shfl_up_sync(0xffffffffu, S, 1);  // exclusive prefix within the warp
    float he = __shfl_up_sync(0xffffffffu, h, 1);
    if (lane == 0) {
      Se = 0.f;
      he = 0.f;
    }
    if (e < io.K && in_bounds(int64_t(g) * io.K + k, nk))
      io.hin[((int64_t(g) * io.K + k) * NM + n) * kSThreads + c] = fmaf(ex2f(A2 * Se), cin, he);
    __syncthreads();
    if (threadIdx.x == 127) carry = fmaf(ex2f(A2 * S), cin, h);  // through the whole block
    __syncthreads();
  }
}

// Closed-form correction after the LOC pass (one CTA per channel group and
// 64-step block of the chunks k >= 1, one thread per channel).  A chunk run
// from a zero entering state misses the contribution of its true entering
// state h_in: with cumDelta_t the sum of Delta over the chunk up to step t,
// the state the chunk really has is h_t + exp(A_n cumDelta_t) h_in,n (the
// homogeneous solution of the recurrence, Abar multiplying it step by step),
// so
//     y_t += silu(z_t) sum_n C_tn exp(A_n cumDelta_t) h_in,n
// and the last chunk's final state gains exp(A_n S) h_in,n.  For the
// structured A (A_n = (n+1) A_0 < 0) the sum is a polynomial in
// q_t = exp(A_0 cumDelta_t), evaluated by Horner's rule; otherwise one exp per
// state.  A block starts from the LOC pass's running sum at its start, and a
// CTA has nothing to add once every decay of its channels has fallen below
// 2^-32 (the terms left are below fp32 resolution of the state they correct).
template <typename T, int NM>
__global__ void __launch_bounds__(kSThreads) fwd_correct_kernel(const StagedArgs p) {
  constexpr int V = 16 / int(sizeof(T));  // steps per 16-byte vector
  constexpr int BLK = kCorrBlock;
  __shared__ __align__(16) float Cs[BLK][NM + 2];  // this block's C rows, fp32, time-major (even rows)
  const FwdArgs &f = p.f;
  const int64_t nblk = (f.L + BLK - 1) / BLK;
  const int64_t first = p.chunk_len / BLK;  // the first block of chunk 1
  const int g = int(blockIdx.x % unsigned(p.G));
  const int64_t jb = first + blockIdx.x / unsigned(p.G);
  const int64_t t0 = jb * BLK;
  const int k = int(t0 / p.chunk_len);
  const int b = g / p.gpb, c = threadIdx.x;
  const int d = (g % p.gpb) * kSThreads + c;
  const bool valid = d < f.dim;
  const int N = f.N;
  float hin[NM], An[NM];
  bool any = false;
#pragma unroll
  for (int n = 0; n < NM; ++n) {
    const int64_t hi = ((int64_t(g) * p.K + k) * NM + n) * kSThreads + c;
    hin[n] = in_bounds(hi, p.n_agg) ? __ldcg(p.hin + hi) : 0.f;
    An[n] = (valid && n < N) ? f.A[int64_t(d) * N + n] : -float(n + 1);
    any = any || (valid && n < N && hin[n] != 0.f);
  }
  if (valid && k == p.K - 1 && t0 == int64_t(k) * p.chunk_len && f.last_state) {  // the true final state
    const int64_t si = (int64_t(g) * p.K + k) * kSThreads + c;
    const double S = in_bounds(si, p.n_aggS) ? p.agg_S[si] : 0.0;
#pragma unroll
    for (int n = 0; n < NM; ++n)
      if (n < N && in_bounds(((int64_t(g) * p.K + k) * NM + n) * kSThreads + c, p.n_agg) &&
          in_bounds((int64_t(b) * f.dim + d) * N + n, f.batch * f.dim * N)) {
        const float hl = __ldcg(p.agg_h + ((int64_t(g) * p.K + k) * NM + n) * kSThreads + c);
        f.last_state[(int64_t(b) * f.dim + d) * N + n] = hl + float(exp(double(An[n]) * S)) * hin[n];
      }
  }
  float cum = 0.f;  // Delta summed from the chunk's start to step t0 - 1
  if (t0 > int64_t(k) * p.chunk_len) {
    const int64_t bi = (int64_t(g) * nblk + jb - 1) * kSThreads + c;
    cum = in_bounds(bi, p.n_blk) ? __ldcg(p.blk_cum + bi) : 0.f;
  }
  float amax = An[0];  // slowest decay
#pragma unroll
  for (int n = 1; n < NM; ++n) amax = fmaxf(amax, An[n]);
  const bool active = any && amax * cum >= -22.2f;  // exp(amax cumDelta) >= 2^-32
  if (!__syncthreads_or(active)) return;
  const int steps = int(std::min<int64_t>(BLK, f.L - t0));
  const T *Cb = static_cast<const T *>(f.C) + int64_t(b) * N * f.L;
  for (int i = threadIdx.x; i < BLK * NM; i += kSThreads) {
    const int n = i / BLK, tl = i % BLK;  // consecutive threads read consecutive steps
    Cs[tl][n] = (n < N && tl < steps && in_bounds(int64_t(b) * N * f.L + int64_t(n) * f.L + t0 + tl,
                                                   f.batch * N * f.L))
                    ? to_f(Cb[int64_t(n) * f.L + t0 + tl])
                    : 0.f;
  }
  __syncthreads();
  if (!active) return;
  bool structured = An[0] < 0.f && isfinite(An[0]);
#pragma unroll
  for (int n = 1; n < NM; ++n) structured = structured && (An[n] == float(n + 1) * An[0]);
  f2 H2[NM / 2];  // h_in in pairs (even, odd state)
#pragma unroll
  for (int i = 0; i < NM / 2; ++i) H2[i] = pk(hin[2 * i], hin[2 * i + 1]);
  const float bias = f.bias ? f.bias[d] : 0.f;
  const int64_t row = (int64_t(b) * f.dim + d) * f.L;
  const T *dl = static_cast<const T *>(f.delta) + row;
  const T *zr = f.z ? static_cast<const T *>(f.z) + row : nullptr;
  T *yr = static_cast<T *>(f.y) + row;
  for (int j = 0; j < steps; j += V) {  // rows are 16-byte multiples
    if (!in_bounds(row + t0 + j + V - 1, f.batch * f.dim * f.L)) break;
    float dv[V], zv[V], yv[V];
    Vec<T>::unpack(*reinterpret_cast<const uint4 *>(dl + t0 + j), dv);
    Vec<T>::unpack(*reinterpret_cast<const uint4 *>(yr + t0 + j), yv);
    if (zr) Vec<T>::unpack(*reinterpret_cast<const uint4 *>(zr + t0 + j), zv);
#pragma unroll
    for (int i = 0; i < V; ++i) {
      cum += softplus_fast(dv[i] + bias);
      const float *crow = Cs[j + i];
      float corr;
      if (structured) {
        // sum_n c_n q^(n+1) with c_n = C_n hin_n and q = exp(A_0 cumDelta):
        // the even and the odd states as two polynomials in q^2, evaluated
        // together by Horner's rule in packed pairs, then
        // q (sum_k c_2k q^2k + q sum_k c_2k+1 q^2k)
        const float q = ex2f(An[0] * cum * kLog2e);
        const f2 X = pk(q * q, q * q), Z = pk(0.f, 0.f);
        const f2 *c2 = reinterpret_cast<const f2 *>(crow);
        f2 r = fma2(c2[NM / 2 - 1], H2[NM / 2 - 1], Z);
#pragma unroll
        for (int k = NM / 2 - 2; k >= 0; --k) r = fma2(r, X, fma2(c2[k], H2[k], Z));
        corr = q * fmaf(q, hi_of(r), lo_of(r));
      } else {
        corr = 0.f;
#pragma unroll
        for (int n = 0; n < NM; ++n) corr = fmaf(crow[n] * hin[n], ex2f(An[n] * cum * kLog2e), corr);
      }
      if (zr) corr *= zv[i] * rcpf(1.f + ex2f(-zv[i] * kLog2e));
      yv[i] += corr;
    }
    *reinterpret_cast<uint4 *>(yr + t0 + j) = Vec<T>::pack(yv);
  }
}

// ------------------------------------------------------------------ host

struct StagedPlan {
  int kind;       // KIND_SEQ or KIND_PAR
  int chunk_len;
  int K;
};

inline int device_sm_count() {
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms > 0 ? sms : 148;
}

// Whether the staged kernels can take a problem of this shape: rows of
// 16-byte multiples, N >= 3, L and dim within the index limits.
inline bool staged_shape_ok(int64_t L, int64_t dim, int64_t N, size_t es) {
  if (N < 3) return false;
  if ((L * int64_t(es)) % 16 != 0) return false;
  return L <= (int64_t(1) << 31) - 1024 && dim <= (int64_t(1) << 31) - 1;
}

// ... and this problem: also 16-byte aligned bases.
inline bool staged_supported(const FwdArgs &a, size_t es) {
  auto al = [](const void *ptr) { return ptr == nullptr || (reinterpret_cast<uintptr_t>(ptr) & 15) == 0; };
  if (!staged_shape_ok(a.L, a.dim, a.N, es)) return false;
  return al(a.u) && al(a.delta) && al(a.z) && al(a.y) && al(a.B) && al(a.C);
}

// Dynamic shared memory of the fused-projection forward with `nst` stages.
template <typename T, int NM>
inline int proj_smem_bytes(int Rp, int nst) {
  using Lay = StagedLayout<T, NM>;
  return int(uint32_t(nst) * ProjStage(Rp).bytes) + 2 * kTileBytes + 4 * Lay::TT * Lay::BSTR * 4 +
         8 * 5 + 16 * 4 + 1024;
}

// Largest dynamic shared memory per CTA that still lets two CTAs share an SM
// (228 KB per SM, 1 KB of it reserved per CTA).
constexpr int kTwoPerSmBytes = (233472 - 2 * 1024) / 2;

// CTAs of `kern` resident per SM with `smem` bytes of dynamic shared memory.
// The occupancy query answers one for any kernel that allocates tensor memory,
// whatever its registers and shared memory; a CTA that holds `tmem_cols` of
// the SM's 512 TMEM columns (0: none) has its count taken from registers and
// shared memory, capped at 512 / tmem_cols.  (Should more CTAs than that land
// on one SM, the extra one waits in its TMEM allocation, which comes before
// it claims any work, until one exits.)
template <typename K>
inline cudaError_t resident_ctas(K kern, int smem, int tmem_cols, int *bps) {
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(bps, kern, kSThreads, smem);
  if (e != cudaSuccess || tmem_cols <= 0) return e;
  cudaFuncAttributes at;
  if ((e = cudaFuncGetAttributes(&at, kern)) != cudaSuccess) return e;
  int dev = 0, sm_smem = 0, reserved = 0, sm_regs = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&sm_smem, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&sm_regs, cudaDevAttrMaxRegistersPerMultiprocessor, dev)) != cudaSuccess)
    return e;
  const int warp_regs = (at.numRegs * 32 + 255) / 256 * 256;  // allocated per warp in units of 256
  const int by_regs = sm_regs / std::max(1, warp_regs * (kSThreads / 32));
  const int by_smem = sm_smem / std::max(1, smem + int(at.sharedSizeBytes) + reserved);
  *bps = std::max(*bps, std::min(std::min(by_regs, by_smem), 512 / tmem_cols));
  return cudaSuccess;
}

template <typename T, int NM, int KIND, bool CONV = false, bool PROJ = false>
inline cudaError_t prepare_kernel(int *blocks_per_sm, int bytes = StagedLayout<T, NM>::ALLOC) {
  auto kern = fwd_staged_kernel<T, NM, KIND, CONV, PROJ>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  return resident_ctas(kern, bytes, PROJ ? int(kProjTmemCols) : 0, blocks_per_sm);
}

template <typename T, int NM, int KIND, bool CONV = false, bool PROJ = false>
inline void launch_staged(const CUtensorMap (&maps)[6], const StagedArgs &sa, int grid, cudaStream_t s,
                          int bytes = StagedLayout<T, NM>::ALLOC) {
  fwd_staged_kernel<T, NM, KIND, CONV, PROJ><<<grid, kSThreads, bytes, s>>>(
      maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], sa);
}

struct StagedOptions {
  int path, chunk_len, carry, timeout_us, test_hook;
};

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Picks the chunking: the sequential hand-off when the channel groups alone
// fill the resident CTAs (about eight chunks per group keeps the tail short),
// else the three-phase scheme with about four units per resident CTA.
inline StagedPlan plan_staged(int64_t G, int64_t L, int slots, const StagedOptions &o,
                              int64_t min_par_chunk = 512) {
  StagedPlan pl;
  int carry = o.carry;
  if (carry == 0) carry = G >= slots ? 1 : 2;
  int64_t chunk = o.chunk_len;
  if (chunk <= 0) {
    if (carry == 1) {
      const int64_t kt = std::max<int64_t>(1, (8 * int64_t(slots) + G / 2) / G);
      chunk = std::max<int64_t>(256, ceil_div(ceil_div(L, kt), 64) * 64);
    } else {
      const int64_t kt = std::max<int64_t>(1, ceil_div(4 * int64_t(slots), G));
      chunk = std::max<int64_t>(min_par_chunk, ceil_div(ceil_div(L, kt), 64) * 64);
    }
  }
  chunk = std::min<int64_t>(chunk, ceil_div(L, 64) * 64);
  pl.chunk_len = int(chunk);
  pl.K = int(ceil_div(L, chunk));
  pl.kind = (pl.K == 1) ? KIND_SEQ : (carry == 1 ? KIND_SEQ : KIND_PAR);
  return pl;
}

// The forward's chunking for a problem of this size on the current device
// (what StagedForward::prepare decides, without tensor maps): G channel
// groups, the plan, and the CTA slots of the main kernel.
template <typename T, int NM, bool CONV = false, bool PROJ = false>
inline mamba_status_t staged_forward_plan(int64_t batch, int64_t dim, int64_t L, const StagedOptions &o,
                                          int smem, StagedPlan *pl, int64_t *G, int *sms, int *slots) {
  int bps_main = 0;
  if (prepare_kernel<T, NM, KIND_SEQ, CONV, PROJ>(&bps_main, smem) != cudaSuccess) return MAMBA_ERR_CUDA;
  *sms = device_sm_count();
  *slots = *sms * std::max(1, bps_main);
  *G = batch * ceil_div(dim, kSThreads);
  if (*G > (int64_t(1) << 30)) return MAMBA_ERR_UNSUPPORTED;
  *pl = plan_staged(*G, L, *slots, o);
  if (*G * pl->K > (int64_t(1) << 30)) return MAMBA_ERR_UNSUPPORTED;
  return MAMBA_OK;
}

// What a saving forward stores for the backward (byte offsets into the
// caller's buffer, each 256-byte aligned, and element counts):
//   ckpt  [G][ceil(L/16)][NM][128] fp32  the state before every 16th step
//   flags [G][ceil(L/64)] bytes         the Delta-range flags of the backward
// and with the three-phase carry for 16-bit I/O, whose chunks run from zero
// (LOC_SAVE; fp32 takes the aggregate pass and PAR_SAVE, whose checkpoints
// are the true states),
//   cum   [G][ceil(L/16)][128] fp32     Delta summed from the chunk's start
//   hin   [G][K][NM][128] fp32          the state entering each chunk
// (the backward adds exp(A_n cum) h_in,n to a checkpoint of chunk k >= 1).
struct SavedLayout {
  StagedPlan pl;
  int64_t G = 0;
  size_t ckpt = 0, flags = 0, cum = 0, hin = 0, bytes = 0;
  int64_t n_ckpt = 0, n_flags = 0, n_cum = 0, n_hin = 0;
};

template <typename T, int NM, bool CONV = false, bool PROJ = false>
inline mamba_status_t saved_layout(int64_t batch, int64_t dim, int64_t L, const StagedOptions &o,
                                   SavedLayout *out, int R = 0) {
  SavedLayout sl;
  int sms = 0, slots = 0;
  int smem = StagedLayout<T, NM>::ALLOC;
  if constexpr (PROJ) {  // the fused projection's stages (as StagedForward::prepare sizes them)
    const int Rp = (R + 15) / 16 * 16;
    if (R < 1 || Rp > kProjMaxRp) return MAMBA_ERR_UNSUPPORTED;
    smem = proj_smem_bytes<T, NM>(Rp, proj_smem_bytes<T, NM>(Rp, 3) <= kTwoPerSmBytes ? 3 : 2);
  }
  const mamba_status_t st =
      staged_forward_plan<T, NM, CONV, PROJ>(batch, dim, L, o, smem, &sl.pl, &sl.G, &sms, &slots);
  if (st != MAMBA_OK) return st;
  auto up = [](size_t b) { return (b + 255) / 256 * 256; };
  const int64_t n16 = ceil_div(L, kCkptEvery);
  sl.n_ckpt = sl.G * n16 * NM * kSThreads;
  sl.n_flags = sl.G * ceil_div(L, kRangeBlock);
  sl.ckpt = 0;
  sl.flags = up(size_t(sl.n_ckpt) * 4);
  sl.bytes = sl.flags + up(size_t(sl.n_flags));
  if (sl.pl.kind != KIND_SEQ && sizeof(T) == 2 && !PROJ) {
    sl.n_cum = sl.G * n16 * kSThreads;
    sl.n_hin = sl.G * sl.pl.K * NM * kSThreads;
    sl.cum = sl.bytes;
    sl.hin = sl.cum + up(size_t(sl.n_cum) * 4);
    sl.bytes = sl.hin + up(size_t(sl.n_hin) * 4);
  }
  *out = sl;
  return MAMBA_OK;
}

// The staged forward, split into a preparation (tensor maps, plan, the
// workspace size; nothing enqueued) and the launches on a given workspace, so
// that a caller can take one workspace for several steps and fail before
// enqueuing anything when it cannot be had.
template <typename T, int NM, bool CONV = false, bool PROJ = false>
struct StagedForward {
  using Lay = StagedLayout<T, NM>;
  // The three-phase forward with y runs the chunks from zero and corrects
  // them in closed form (LOC + scan + fwd_correct_kernel) for 16-bit I/O; the
  // correction is a pass over delta, z, C and y, which in fp32 moves twice
  // the bytes and costs more than the aggregate pass it replaces (measured on
  // fp32 8 x 1536 x 2048: 0.304 against 0.256 ms).  The checkpoint pass needs
  // the true states at every 16th step, and the fused projection does not
  // store delta for the correction: those, and fp32, take the aggregate pass
  // and a second full pass.
  static constexpr bool kLocCarry = sizeof(T) == 2 && !PROJ;
  // (a caller with a bounded workspace may turn the closed-form carry off:
  // its running sums of Delta take L / 64 floats per channel whatever the
  // chunking, where the aggregate pass needs none)
  bool use_loc = true;
  // The three-phase checkpoint pass runs the chunks from zero (CKPT_LOC +
  // scan) in place of the aggregate pass and a second pass; its checkpoints
  // in chunks k >= 1 then lack exp(A_n cum) h_in,n, which the backward adds
  // as it reads them (cum in sa.ckpt_cum, h_in in sa.hin).
  bool ckpt_loc = true;
  bool for_ckpt = false;  // prepared for a checkpoint pass
  // A saving forward (set before prepare): y as usual, and the layout of
  // what it stores for the backward into save_buf (set before run).
  const SavedLayout *save = nullptr;
  unsigned char *save_buf = nullptr;
  CUtensorMap maps[6];
  StagedArgs sa;
  StagedPlan pl;
  int sms = 0, slots = 0;
  size_t int_bytes = 0, bytes = 0;
  int smem = Lay::ALLOC;  // dynamic shared memory per CTA

  // Builds the tensor maps and the plan; with `ckpt` the forward runs without
  // y and stores the state before every kCkptEvery-th step into ckpt
  // ([G][ceil(L/16)][NM][128] floats; `ckpt_mode` sizes the workspace for a
  // checkpoint pass whose buffer is set later).  Returns
  // MAMBA_ERR_UNSUPPORTED if the driver rejects a tensor map.
  mamba_status_t prepare(const FwdArgs &a, const StagedOptions &o, float *ckpt, bool ckpt_mode = false) {
    for_ckpt = ckpt_mode || ckpt != nullptr;
    constexpr bool bf16 = std::is_same<T, __nv_bfloat16>::value;
    const uint64_t L = a.L, dim = a.dim, batch = a.batch, N = a.N;
    const CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_64B, none = CU_TENSOR_MAP_SWIZZLE_NONE;
    int Rp = 0, nst = kStages;
    if (PROJ) {  // the dt_low tiles: Rp rows (R rounded up to 16, zero-filled) of TT steps
      Rp = (a.R + 15) / 16 * 16;
      if (a.R < 1 || Rp > kProjMaxRp) return MAMBA_ERR_UNSUPPORTED;
      nst = proj_smem_bytes<T, NM>(Rp, 3) <= kTwoPerSmBytes ? 3 : 2;
      smem = proj_smem_bytes<T, NM>(Rp, nst);
    }
    const bool dmap = PROJ ? make_map_3d(&maps[1], a.dt_low, bf16, L, uint64_t(a.R), batch, Lay::TT,
                                         uint32_t(Rp), sw)
                           : make_map_3d(&maps[1], a.delta, bf16, L, dim, batch, Lay::TT, kSThreads, sw);
    if (!make_map_3d(&maps[0], a.u, bf16, L, dim, batch, Lay::TT, kSThreads, sw) || !dmap ||
        !make_map_3d(&maps[2], a.z ? a.z : a.u, bf16, L, dim, batch, Lay::TT, kSThreads, sw) ||
        !make_map_3d(&maps[3], a.y ? a.y : a.u, bf16, L, dim, batch, Lay::TT, kSThreads, sw) ||
        !make_map_3d(&maps[4], a.B, bf16, L, N, batch, Lay::TT, uint32_t(N), none) ||
        !make_map_3d(&maps[5], a.C, bf16, L, N, batch, Lay::TT, uint32_t(N), none)) {
      return MAMBA_ERR_UNSUPPORTED;
    }
    const int64_t gpb = ceil_div(a.dim, kSThreads);
    int64_t G = 0;
    {
      const mamba_status_t st =
          staged_forward_plan<T, NM, CONV, PROJ>(a.batch, a.dim, a.L, o, smem, &pl, &G, &sms, &slots);
      if (st != MAMBA_OK) return st;
    }

    sa.f = a;
    sa.G = int(G);
    sa.gpb = int(gpb);
    sa.K = pl.K;
    sa.chunk_len = pl.chunk_len;
    sa.timeout_ns = o.timeout_us > 0 ? uint64_t(o.timeout_us) * 1000ull : kDefaultTimeoutNs;
    sa.test_hook = o.test_hook;
    sa.force_generic = o.path == MAMBA_PATH_GENERIC ? 1 : 0;
    sa.flags = nullptr;
    sa.counter = nullptr;
    sa.carry = sa.agg_h = sa.hin = nullptr;
    sa.agg_S = nullptr;
    sa.ckpt = ckpt;
    sa.Rp = Rp;
    sa.nst = nst;
    sa.stage_bytes = PROJ ? ProjStage(Rp).bytes : 0;
    sa.delta_out = nullptr;

    // workspace: [ints: 2 counters + G flags][carry | agg_S, agg_h, hin]
    const size_t n_int = 2 + size_t(G);
    int_bytes = ceil_div(n_int * 4, 256) * 256;
    bytes = int_bytes;
    const size_t gk = size_t(G) * size_t(pl.K);
    if (pl.kind == KIND_SEQ) {
      bytes += size_t(G) * NM * kSThreads * 4;
    } else if (save && sizeof(T) == 2 && !PROJ) {  // agg_S, agg_h and the running sums (h_in is saved)
      bytes += gk * kSThreads * 8 + gk * NM * kSThreads * 4 +
               size_t(G) * size_t(ceil_div(a.L, kCorrBlock)) * kSThreads * 4;
    } else {
      bytes += gk * kSThreads * 8 + 2 * gk * NM * kSThreads * 4;
      if (for_ckpt && ckpt_loc)  // the CKPT_LOC pass's sums of Delta at the checkpoints
        bytes += size_t(G) * size_t(ceil_div(a.L, kCkptEvery)) * kSThreads * 4;
      else if (kLocCarry && use_loc && !for_ckpt)  // the LOC pass's running sums of Delta
        bytes += size_t(G) * size_t(ceil_div(a.L, kCorrBlock)) * kSThreads * 4;
    }
    bytes = ceil_div(bytes, 256) * 256;
    return MAMBA_OK;
  }

  // The scan over chunks (three-phase carry): h_in of every chunk.
  mamba_status_t launch_chunk_scan(cudaStream_t s, mamba_status_t (*launched)()) {
    ChunkScanIO io;
    io.S = sa.agg_S;
    io.hl = sa.agg_h;
    io.hin = sa.hin;
    io.A = sa.f.A;
    io.G = sa.G;
    io.K = sa.K;
    io.gpb = sa.gpb;
    io.N = sa.f.N;
    io.dim = sa.f.dim;
    const int64_t nseq = int64_t(sa.G) * NM * kSThreads;
    chunk_scan_kernel<NM, false><<<unsigned(chunk_scan_grid(nseq, sa.K)), 128, 0, s>>>(io);
    return launched();
  }

  // The saving forward: SEQ_SAVE; for 16-bit I/O LOC_SAVE + scan +
  // fwd_correct_kernel (with h_in and the checkpoints' sums of Delta in the
  // saved buffer); for fp32 and the fused projection AGG + scan + PAR_SAVE.
  mamba_status_t run_save(unsigned char *ws, cudaStream_t s, mamba_status_t (*launched)()) {
    int *counters = reinterpret_cast<int *>(ws);
    const size_t gk = size_t(sa.G) * size_t(pl.K);
    sa.ckpt = reinterpret_cast<float *>(save_buf + save->ckpt);
    sa.range_flags = sa.force_generic ? nullptr : save_buf + save->flags;
    sa.n_flags = save->n_flags;
    int bps = 0;
    if (pl.kind == KIND_SEQ) {
      if (prepare_kernel<T, NM, KIND_SEQ_SAVE, CONV, PROJ>(&bps, smem) != cudaSuccess) return MAMBA_ERR_CUDA;
      sa.carry = reinterpret_cast<float *>(ws + int_bytes);
      sa.counter = counters;
      sa.n_units = int(gk);
      launch_staged<T, NM, KIND_SEQ_SAVE, CONV, PROJ>(maps, sa, int(std::min<int64_t>(gk, sms * std::max(1, bps))),
                                                      s, smem);
      return launched();
    }
    if constexpr (sizeof(T) != 2 || PROJ) {
      int bps_agg = 0;
      if (prepare_kernel<T, NM, KIND_AGG, CONV, PROJ>(&bps_agg, smem) != cudaSuccess ||
          prepare_kernel<T, NM, KIND_PAR_SAVE, CONV, PROJ>(&bps, smem) != cudaSuccess)
        return MAMBA_ERR_CUDA;
      sa.agg_S = reinterpret_cast<double *>(ws + int_bytes);
      sa.agg_h = reinterpret_cast<float *>(ws + int_bytes + gk * kSThreads * 8);
      sa.hin = sa.agg_h + gk * NM * kSThreads;
      StagedArgs sg = sa;
      sg.counter = counters;
      sg.n_units = int(size_t(sa.G) * size_t(pl.K - 1));
      launch_staged<T, NM, KIND_AGG, CONV, PROJ>(
          maps, sg, int(std::min<int64_t>(sg.n_units, sms * std::max(1, bps_agg))), s, smem);
      mamba_status_t st = launched();
      if (st == MAMBA_OK) st = launch_chunk_scan(s, launched);
      if (st == MAMBA_OK) {
        StagedArgs sp = sa;
        sp.counter = counters + 1;
        sp.n_units = int(gk);
        launch_staged<T, NM, KIND_PAR_SAVE, CONV, PROJ>(
            maps, sp, int(std::min<int64_t>(gk, sms * std::max(1, bps))), s, smem);
        st = launched();
      }
      return st;
    }
    if (prepare_kernel<T, NM, KIND_LOC_SAVE, CONV, PROJ>(&bps, smem) != cudaSuccess) return MAMBA_ERR_CUDA;
    sa.agg_S = reinterpret_cast<double *>(ws + int_bytes);
    sa.agg_h = reinterpret_cast<float *>(ws + int_bytes + gk * kSThreads * 8);
    sa.blk_cum = sa.agg_h + gk * NM * kSThreads;
    sa.n_blk = int64_t(sa.G) * ceil_div(sa.f.L, kCorrBlock) * kSThreads;
    sa.hin = reinterpret_cast<float *>(save_buf + save->hin);
    sa.ckpt_cum = reinterpret_cast<float *>(save_buf + save->cum);
    sa.n_ckpt_cum = save->n_cum;
    StagedArgs sl = sa;
    sl.counter = counters;
    sl.n_units = int(gk);
    launch_staged<T, NM, KIND_LOC_SAVE, CONV, PROJ>(maps, sl, int(std::min<int64_t>(gk, sms * std::max(1, bps))),
                                                    s, smem);
    mamba_status_t st = launched();
    if (st == MAMBA_OK) st = launch_chunk_scan(s, launched);
    if (st == MAMBA_OK) {
      const int64_t nb = ceil_div(sa.f.L, kCorrBlock) - pl.chunk_len / kCorrBlock;  // blocks of chunks 1..K-1
      fwd_correct_kernel<T, NM><<<unsigned(int64_t(sa.G) * nb), kSThreads, 0, s>>>(sa);
      st = launched();
    }
    return st;
  }

  // Enqueues the launches on `ws` (at least `bytes`, 256-byte aligned).
  mamba_status_t run(unsigned char *ws, cudaStream_t s, mamba_status_t (*launched)()) {
    mamba_status_t st = MAMBA_OK;
    if (cudaMemsetAsync(ws, 0, int_bytes, s) != cudaSuccess) return MAMBA_ERR_CUDA;
    int *counters = reinterpret_cast<int *>(ws);
    sa.flags = counters + 2;
    const size_t gk = size_t(sa.G) * size_t(pl.K);
    sa.n_carry = int64_t(sa.G) * NM * kSThreads;
    sa.n_agg = int64_t(gk) * NM * kSThreads;
    sa.n_aggS = int64_t(gk) * kSThreads;
    sa.n_ckpt = int64_t(sa.G) * ((sa.f.L + kCkptEvery - 1) / kCkptEvery) * NM * kSThreads;
    if (save) return run_save(ws, s, launched);
    if (pl.kind == KIND_SEQ) {
      sa.carry = reinterpret_cast<float *>(ws + int_bytes);
      sa.counter = counters;
      sa.n_units = int(gk);
      const int grid = int(std::min<int64_t>(gk, slots));
      if (sa.ckpt) {
        int bps = 0;
        if (prepare_kernel<T, NM, KIND_CKPT_SEQ, CONV, PROJ>(&bps, smem) != cudaSuccess)
          return MAMBA_ERR_CUDA;
        launch_staged<T, NM, KIND_CKPT_SEQ, CONV, PROJ>(
            maps, sa, int(std::min<int64_t>(gk, sms * std::max(1, bps))), s, smem);
      } else {
        launch_staged<T, NM, KIND_SEQ, CONV, PROJ>(maps, sa, grid, s, smem);
      }
      return launched();
    }
    sa.agg_S = reinterpret_cast<double *>(ws + int_bytes);
    sa.agg_h = reinterpret_cast<float *>(ws + int_bytes + gk * kSThreads * 8);
    sa.hin = sa.agg_h + gk * NM * kSThreads;
    [[maybe_unused]] const int64_t nblk = ceil_div(sa.f.L, kCorrBlock);
    if constexpr (kLocCarry) {
      if (!sa.ckpt && use_loc) {
        // Every chunk from zero, with y and its aggregates; the scan over
        // chunks; the closed-form correction of chunks 1..K-1 (and of the
        // final state).
        int bps_loc = 0;
        if (prepare_kernel<T, NM, KIND_LOC, CONV, PROJ>(&bps_loc, smem) != cudaSuccess) return MAMBA_ERR_CUDA;
        sa.blk_cum = sa.hin + gk * NM * kSThreads;
        sa.n_blk = int64_t(sa.G) * nblk * kSThreads;
        StagedArgs sl = sa;
        sl.counter = counters;
        sl.n_units = int(gk);
        launch_staged<T, NM, KIND_LOC, CONV, PROJ>(
            maps, sl, int(std::min<int64_t>(gk, sms * std::max(1, bps_loc))), s, smem);
        st = launched();
        if (st == MAMBA_OK) st = launch_chunk_scan(s, launched);
        if (st == MAMBA_OK) {
          const int64_t nb = nblk - pl.chunk_len / kCorrBlock;  // the blocks of chunks 1..K-1
          fwd_correct_kernel<T, NM><<<unsigned(int64_t(sa.G) * nb), kSThreads, 0, s>>>(sa);
          st = launched();
        }
        return st;
      }
    }
    if (sa.ckpt && ckpt_loc) {
      // Every chunk from zero, storing its checkpoints with the sums of Delta
      // up to them and its aggregates; the scan over chunks (h_in).
      int bps_loc = 0;
      if (prepare_kernel<T, NM, KIND_CKPT_LOC, CONV, PROJ>(&bps_loc, smem) != cudaSuccess)
        return MAMBA_ERR_CUDA;
      const int64_t n16 = ceil_div(sa.f.L, kCkptEvery);
      sa.ckpt_cum = sa.hin + gk * NM * kSThreads;
      sa.n_ckpt_cum = int64_t(sa.G) * n16 * kSThreads;
      StagedArgs sl = sa;
      sl.counter = counters;
      sl.n_units = int(gk);
      launch_staged<T, NM, KIND_CKPT_LOC, CONV, PROJ>(
          maps, sl, int(std::min<int64_t>(gk, sms * std::max(1, bps_loc))), s, smem);
      st = launched();
      if (st == MAMBA_OK) st = launch_chunk_scan(s, launched);
      return st;
    }
    int bps_agg = 0, bps_par = 0;
    if (prepare_kernel<T, NM, KIND_AGG, CONV, PROJ>(&bps_agg, smem) != cudaSuccess ||
        (sa.ckpt ? prepare_kernel<T, NM, KIND_CKPT_PAR, CONV, PROJ>(&bps_par, smem)
                 : prepare_kernel<T, NM, KIND_PAR, CONV, PROJ>(&bps_par, smem)) != cudaSuccess) {
      return MAMBA_ERR_CUDA;
    }
    {
      StagedArgs sg = sa;
      sg.counter = counters;
      sg.n_units = int(size_t(sa.G) * size_t(pl.K - 1));
      launch_staged<T, NM, KIND_AGG, CONV, PROJ>(
          maps, sg, int(std::min<int64_t>(sg.n_units, sms * std::max(1, bps_agg))), s, smem);
      st = launched();
    }
    if (st == MAMBA_OK) st = launch_chunk_scan(s, launched);
    if (st == MAMBA_OK) {
      StagedArgs sm = sa;
      sm.counter = counters + 1;
      sm.n_units = int(gk);
      const int grid = int(std::min<int64_t>(gk, sms * std::max(1, bps_par)));
      if (sa.ckpt) launch_staged<T, NM, KIND_CKPT_PAR, CONV, PROJ>(maps, sm, grid, s, smem);
      else launch_staged<T, NM, KIND_PAR, CONV, PROJ>(maps, sm, grid, s, smem);
      st = launched();
    }
    return st;
  }
};

// The staged forward with its own stream-ordered workspace.  Returns
// MAMBA_ERR_UNSUPPORTED (nothing enqueued) if the driver rejects a tensor map,
// MAMBA_ERR_OUT_OF_MEMORY (nothing enqueued) if the workspace cannot be had.
// CONV selects the kernels with the convolution prologue (a.conv_w set).
// With `save`, the forward also stores what the backward would recompute,
// laid out as saved_layout gives it.
template <typename T, int NM, bool CONV = false, bool PROJ = false>
mamba_status_t staged_forward(const FwdArgs &a, const StagedOptions &o, cudaStream_t s,
                              mamba_status_t (*launched)(), float *ckpt = nullptr,
                              unsigned char *save = nullptr) {
  StagedForward<T, NM, CONV, PROJ> sf;
  SavedLayout lay;
  if (save) {
    const mamba_status_t ls = saved_layout<T, NM, CONV, PROJ>(a.batch, a.dim, a.L, o, &lay, a.R);
    if (ls != MAMBA_OK) return ls;
    sf.save = &lay;
    sf.save_buf = save;
  }
  mamba_status_t st = sf.prepare(a, o, ckpt);
  if (st != MAMBA_OK) return st;
  unsigned char *ws = nullptr;
  if (ws_alloc(reinterpret_cast<void **>(&ws), sf.bytes, s) != cudaSuccess) {
    cudaGetLastError();
    return MAMBA_ERR_OUT_OF_MEMORY;
  }
  st = sf.run(ws, s, launched);
  if (ws_free(ws, s) != cudaSuccess && st == MAMBA_OK) st = MAMBA_ERR_CUDA;
  return st;
}

}  // namespace mscan
