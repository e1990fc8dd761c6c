// bwd_staged.cuh -- the staged backward of the selective scan for sm_100a.
//
// Gradients of the scalar sum(dy * y) with respect to every input, with the
// states recomputed instead of stored (the recomputation of section 3.3 of
// "Mamba: Linear-Time Sequence Modeling with Selective State Spaces",
// paper-graph-ui summary, and of Part III section 4 of the trishampatil.com
// walk-through).  The pages give no gradient formulas; the adjoint below is
// derived from the forward of Knowl 1 (chapterpal.com page).
//
// Organisation:
//  * The forward runs first in checkpoint mode (fwd_staged.cuh, no y): it
//    stores the state before every 16th step, (batch, dim, L/16, N) fp32.
//  * This kernel then walks every (channel group, chunk) unit from the last
//    chunk to the first.  One thread owns one channel and its N states.  Per
//    16-step tile (TMA-staged u, delta, z, dy, B, C, read in reverse order) it
//    re-runs the tile forward from its checkpoint, keeping the state before
//    every segment of 2 (bf16) or 4 (fp32) steps in shared memory, then for
//    each segment from the last re-runs it into registers and walks it
//    backwards.
//  * The adjoint of h_t is G_t = C_t dy0_t + Abar_{t+1} G_{t+1} with
//    dy0 = dy silu(z); the thread carries Ga = Abar_t G_t, which is also the
//    factor of dDelta.  With the structured A of the forward (decays E(n+1)
//    from one expm1, Bbar = E(n+1) B/(n+1) / A[d,0]) the local gradients are
//        du     = D dy0 + (1/A0) sum_n (G E) B'
//        dDelta = A0 sum_n (n+1) Ga (h_{t-1} + B' u')        (Ga = (1+E) G)
//        dB_n   = sum_d (G E) u' / (n+1),   dC_n = sum_d dy0 h_t
//        dA_n   = (1/A_n) sum_t [A_n Delta (G dh/dDelta)_n - (G Bbar u)_n]
//    the last from A_n dh/dA_n = Delta dh/dDelta - Bbar u, which needs no
//    second derivative of psi.  Channels without that structure take the
//    generic arithmetic (dA through psi'(x) = (x e^x - expm1 x)/x^2).
//  * The adjoint crosses chunk boundaries backwards by the same bounded-wait
//    hand-off as the forward (unit tickets are issued chunk-major from the
//    end).  dB and dC (sums over channels) are reduced per warp by a
//    butterfly, per CTA in shared memory, then across CTAs by a finalize
//    kernel in a fixed order, as are dA, dD and the bias gradient: results
//    are bitwise reproducible.
#pragma once

#include "bwd_reference.cuh"
#include "fwd_staged.cuh"

namespace mscan {

constexpr int kBTT = kCkptEvery;  // time steps per backward tile
constexpr int kBStages = 2;
// Tensor memory of the fused projection's backward (kProjTmemCols columns
// per CTA): W_dt's rows in [0, Rp/2), the two 16-step delta accumulators in
// [kProjBwdAcc, kProjBwdAcc + 32), the segment states from kProjBwdSub.
constexpr uint32_t kProjBwdAcc = 96;
constexpr uint32_t kProjBwdSub = 128;
constexpr int kProjBwdMaxRp = 2 * int(kProjBwdAcc);

// TSUB: the state before every segment lives in tensor memory (each thread's
// own lane, NSEG x NM columns): one tcgen05.st / tcgen05.ld of the NM states
// in place of NM / 2 shared-memory stores / loads.  The kernels take TSUB;
// the layout without it sizes the rank limit of the fused projection.
template <typename T, int NM, bool TSUB = false>
struct BwdLayout {
  static constexpr int RB = kBTT * (int)sizeof(T);  // bytes of one channel row in a tile
  static constexpr int TILE = kSThreads * RB;
  static constexpr int RAW = kMaxN * RB;
  static constexpr int STAGE = 4 * TILE + 2 * RAW;  // u, delta, z, dy, B, C
  // Steps per recompute segment: the states of one segment live in
  // registers, the state before every segment in shared or tensor memory.
  // Two-step segments keep the register footprint down; fp32 tiles are twice
  // as large, which leaves room for four-step segments only.
  static constexpr int SEG = sizeof(T) == 2 ? 2 : 4;
  static constexpr int NSEG = kBTT / SEG;
  static constexpr int BSTR = NM;  // rows of B / C are read as broadcasts; no padding
  static constexpr int OFF_SUB = kBStages * STAGE;
  static constexpr int SUB_BYTES = TSUB ? 0 : NSEG * NM * kSThreads * 4;
  static constexpr int TMEM_COLS = !TSUB ? 0 : (NSEG * NM < 32 ? 32 : NSEG * NM);
  static constexpr int OFF_BS = OFF_SUB + SUB_BYTES;
  static constexpr int OFF_CS = OFF_BS + kBTT * BSTR * 4;
  static constexpr int OFF_RED = OFF_CS + kBTT * BSTR * 4;
  static constexpr int RED_BYTES = (kSThreads / 32) * kBTT * 33 * 4;
  static constexpr int OFF_BAR = OFF_RED + RED_BYTES;
  static constexpr int OFF_Q = OFF_BAR + 8 * 4;  // stage barriers (2) + MMA barriers (2)
  static constexpr int BYTES = OFF_Q + 16 * 4;
  static constexpr int ALLOC = BYTES + 512;
};

// Stage geometry of the backward: u, then delta (or, with the fused
// projection, the Rp x 16 dt_low tile), z, dy, B and C.
template <typename T, int NM>
struct BwdStage {
  uint32_t z, dy, B, C, bytes;
  __host__ __device__ BwdStage(int Rp) {
    using Lay = BwdLayout<T, NM>;
    const uint32_t dsz = Rp > 0 ? uint32_t(Rp) * Lay::RB : uint32_t(Lay::TILE);
    z = Lay::TILE + dsz;
    dy = z + Lay::TILE;
    B = dy + Lay::TILE;
    C = B + Lay::RAW;
    bytes = (C + Lay::RAW + 511u) & ~511u;
  }
};

struct BwdStagedArgs {
  BwdArgs w;
  int G, gpb, K, chunk_len, n_units;
  int *counter;
  int *flags;          // per group: number of later chunks whose adjoint is published
  float *carry;        // [G][NM][128] Abar G handed to the previous chunk
  const float *ckpt;   // [G][ceil(L/16)][NM][128] state before every 16th step
  float *part_bc;      // [gpb][batch][32][L] per-CTA sums: dB in slots 0..15, dC in 16..31
  float *part_A;       // [G][K][NM][128]
  float *part_D;       // [G][K][128]
  float *part_bias;    // [G][K][128]
  uint64_t timeout_ns;
  int force_generic;
  int test_hook;  // 1: the last chunk of group 0 never publishes its adjoint (tests the bounded wait)
  // three-phase carry of the adjoint (null in the sequential hand-off):
  float *gin;        // [G][K][NM][128] Abar G entering each chunk from the later one
  float *agg_G;      // [G][K][NM][128] the same produced by each chunk from zero
  double *agg_S;     // [G][K][128] sum of Delta over each chunk
  // fused Delta projection (PROJ kernels): R padded to 16; bytes of a stage
  int Rp = 0;
  uint32_t stage_bytes = 0;
  // element counts of the workspace buffers as allocated (the bounds-checking
  // build checks every index against them)
  int64_t n_ckpt = 0, n_carry = 0, n_bc = 0, n_unit = 0, n_gin = 0;
  // [G][ceil(L/64)]: 1 where no step of any channel has its delta in the
  // range the structured forms take (written by the checkpoint pass; null: no
  // check, and the fused projection checks per tile)
  const unsigned char *range_flags = nullptr;
  int64_t n_flags = 0;
  // checkpoints of a three-phase checkpoint pass, stored from a zero state at
  // the start of each of its chunks (ckpt_chunk steps long, ckpt_K of them):
  // the state at a checkpoint of chunk k >= 1 is the stored one plus
  // exp(A_n cum) h_in,n, cum the sum of Delta from the chunk's start
  // ([G][ceil(L/16)][128]) and h_in the state entering the chunk
  // ([G][ckpt_K][NM][128]).  Null: the checkpoints are the states.
  const float *ckpt_hin = nullptr;
  const float *ckpt_cum = nullptr;
  int ckpt_chunk = 0, ckpt_K = 0;
  int64_t n_ckpt_hin = 0, n_ckpt_cum = 0;
};

// Byte offset of 16-byte chunk c of row r in a tile with RB-byte rows written
// by TMA with RB-byte swizzling (chunk index XOR address bits from bit 7 up).
template <int RB>
__device__ __forceinline__ int swz_rows(int r, int c) {
  return r * RB + ((c ^ ((r * RB >> 7) & (RB / 16 - 1))) << 4);
}

// The SEG consecutive values of row r that make segment `seg` of a tile.
template <typename T, int SEG> struct SegIO;
template <> struct SegIO<__nv_bfloat16, 2> {  // 32-byte rows: 2 chunks of 8 steps
  __device__ static void load(const unsigned char *tile, int r, int seg, float (&o)[2]) {
    const uint32_t v = *reinterpret_cast<const uint32_t *>(tile + swz_rows<32>(r, seg >> 2) + (seg & 3) * 4);
    o[0] = __uint_as_float(v << 16);
    o[1] = __uint_as_float(v & 0xffff0000u);
  }
  __device__ static void store(__nv_bfloat16 *dst, const float (&o)[2]) {
    __nv_bfloat162 a = __floats2bfloat162_rn(o[0], o[1]);
    *reinterpret_cast<uint32_t *>(dst) = *reinterpret_cast<uint32_t *>(&a);
  }
};
template <> struct SegIO<float, 4> {  // 64-byte rows: 4 chunks of 4 steps
  __device__ static void load(const unsigned char *tile, int r, int seg, float (&o)[4]) {
    const float4 v = *reinterpret_cast<const float4 *>(tile + swz_rows<64>(r, seg));
    o[0] = v.x;
    o[1] = v.y;
    o[2] = v.z;
    o[3] = v.w;
  }
  __device__ static void store(float *dst, const float (&o)[4]) {
    *reinterpret_cast<float4 *>(dst) = make_float4(o[0], o[1], o[2], o[3]);
  }
};

// psi'(x) = (x e^x - expm1(x)) / x^2 = sum_k (k+1)/(k+2)! x^k; the series
// below |x| = 1/4 (truncation below 5e-8 relative), the closed form above.
__device__ __forceinline__ float dpsi_fast(float x, float ex) {
  const float p = 0.5f + x * (1.f / 3.f + x * (0.125f + x * (1.f / 30.f + x * (1.f / 144.f +
                  x * (1.f / 840.f)))));
  const float q = (x * ex - (ex - 1.f)) / (x * x);
  return fabsf(x) < 0.25f ? p : q;
}

// First butterfly stage for one state: lanes with bit 4 set keep the dC value
// and receive their partner's dC; the others keep dB.  Folding this stage
// into the per-state loop halves the values live at once.
__device__ __forceinline__ float bfly_first(float db, float dc, bool up) {
  const float send = up ? db : dc;
  const float keep = up ? dc : db;
  return keep + __shfl_xor_sync(0xffffffffu, send, 16);
}

// Remaining stages (lane bits 3..0) of the reduce-scatter over 16 values:
// lane l returns the warp sum of value l (dB of state l for l < 16, dC of
// state l - 16 otherwise).
__device__ __forceinline__ float bfly_rest(float (&v)[16], int lane) {
#pragma unroll
  for (int o = 8; o >= 1; o >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < o; ++i) {
      const float send = up ? v[i] : v[i + o];
      const float keep = up ? v[i + o] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  return v[0];
}

// The same two steps for values kept in packed pairs (v2[i] = values 2i, 2i+1):
// the adds of a pair are one fma.rn.f32x2, the shuffles and selects as before.
__device__ __forceinline__ f2 bfly_first2(f2 db, f2 dc, bool up) {
  const f2 send = up ? db : dc;
  const f2 keep = up ? dc : db;
  const float rl = __shfl_xor_sync(0xffffffffu, lo_of(send), 16);
  const float rh = __shfl_xor_sync(0xffffffffu, hi_of(send), 16);
  return fma2(pk(rl, rh), pk(1.f, 1.f), keep);
}
__device__ __forceinline__ float bfly_rest2(f2 (&v2)[8], int lane) {
#pragma unroll
  for (int o = 4; o >= 1; o >>= 1) {  // lane bits 3, 2, 1: pairs o apart
    const bool up = (lane & (2 * o)) != 0;
#pragma unroll
    for (int i = 0; i < o; ++i) {
      const f2 send = up ? v2[i] : v2[i + o];
      const f2 keep = up ? v2[i + o] : v2[i];
      const float rl = __shfl_xor_sync(0xffffffffu, lo_of(send), 2 * o);
      const float rh = __shfl_xor_sync(0xffffffffu, hi_of(send), 2 * o);
      v2[i] = fma2(pk(rl, rh), pk(1.f, 1.f), keep);
    }
  }
  const bool up = (lane & 1) != 0;  // lane bit 0: the two halves of the last pair
  const float send = up ? lo_of(v2[0]) : hi_of(v2[0]);
  const float keep = up ? hi_of(v2[0]) : lo_of(v2[0]);
  return keep + __shfl_xor_sync(0xffffffffu, send, 1);
}

// Four consecutive x values of a row (16-byte aligned for float, 8-byte for
// bf16), widened to float.
__device__ __forceinline__ void load_x4(const float *p, float (&o)[4]) {
  const float4 v = __ldg(reinterpret_cast<const float4 *>(p));
  o[0] = v.x;
  o[1] = v.y;
  o[2] = v.z;
  o[3] = v.w;
}
__device__ __forceinline__ void load_x4(const __nv_bfloat16 *p, float (&o)[4]) {
  const uint2 v = __ldg(reinterpret_cast<const uint2 *>(p));
  o[0] = __uint_as_float(v.x << 16);
  o[1] = __uint_as_float(v.x & 0xffff0000u);
  o[2] = __uint_as_float(v.y << 16);
  o[3] = __uint_as_float(v.y & 0xffff0000u);
}

// CONV: the u tiles hold the input x of the block's causal depthwise
// convolution; every read of a segment's u computes SiLU(conv(x)) from the
// segment's x, the x just before it in the tile, and for the first steps of
// a tile the four x values before the tile (read from global memory).  du is
// the gradient with respect to u; the convolution's backward runs after.
//
// PROJ: delta is formed on the tensor cores as in the forward's fused
// projection (fwd_staged.cuh): the Rp x 16 dt_low tiles come through the
// pipeline, W_dt's rows for the CTA's channels sit in TMEM, and each thread
// reads its channel's 16 values of the tile with one tcgen05.ld into its own
// slots of shared memory, where both passes over the tile read them.
template <typename T, int NM, bool CONV = false, bool PROJ = false>
__global__ void __launch_bounds__(kSThreads, 2)
    bwd_staged_kernel(const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_d,
                      const __grid_constant__ CUtensorMap tm_z, const __grid_constant__ CUtensorMap tm_dy,
                      const __grid_constant__ CUtensorMap tm_B, const __grid_constant__ CUtensorMap tm_C,
                      const BwdStagedArgs p) {
  using Lay = BwdLayout<T, NM, true>;  // segment states in tensor memory
  constexpr int RB = Lay::RB, BSTR = Lay::BSTR;
  constexpr int NP = NM / 2;
  constexpr int SEG = Lay::SEG;
  using IO = SegIO<T, SEG>;
  static_assert(!PROJ || (std::is_same<T, __nv_bfloat16>::value && !CONV),
                "the fused projection takes bf16 operands and no convolution prologue");
  static_assert(!PROJ || Lay::NSEG * NM <= int(kProjTmemCols - kProjBwdSub),
                "the segment states must fit after the projection's columns");

  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *sm = smem_raw + ((512u - (smem_u32(smem_raw) & 511u)) & 511u);
  const BwdStage<T, NM> bst(PROJ ? p.Rp : 0);
  const uint32_t SST = PROJ ? bst.bytes : uint32_t(Lay::STAGE);
  const uint32_t OFF_Z = PROJ ? bst.z : 2u * Lay::TILE;
  const uint32_t OFF_DY = PROJ ? bst.dy : 3u * Lay::TILE;
  const uint32_t OFF_B = PROJ ? bst.B : 4u * Lay::TILE;
  const uint32_t OFF_C = PROJ ? bst.C : 4u * Lay::TILE + Lay::RAW;
  const uint32_t OFF_SUB = kBStages * SST;
  const uint32_t OFF_BS = OFF_SUB + uint32_t(Lay::OFF_BS - Lay::OFF_SUB);
  const uint32_t OFF_CS = OFF_SUB + uint32_t(Lay::OFF_CS - Lay::OFF_SUB);
  const uint32_t OFF_RED = OFF_SUB + uint32_t(Lay::OFF_RED - Lay::OFF_SUB);
  const uint32_t OFF_BAR = OFF_SUB + uint32_t(Lay::OFF_BAR - Lay::OFF_SUB);
  // (PROJ) the tile's delta, fp32 pairs [segment][thread], each thread's own
  const uint32_t OFF_DS = (OFF_SUB + uint32_t(Lay::BYTES - Lay::OFF_SUB) + 15u) & ~15u;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_BAR);  // [2 stages], then 2 MMA barriers
  uint64_t *mma_bar = bars + 2;
  int *q = reinterpret_cast<int *>(sm + OFF_BAR + 8 * 4);  // [0..7] tickets, [8] abort, [12] TMEM
  float *Bs = reinterpret_cast<float *>(sm + OFF_BS);
  float *Cs = reinterpret_cast<float *>(sm + OFF_CS);
  float *red = reinterpret_cast<float *>(sm + OFF_RED);  // [4 warps][kBTT][33] (padded rows)

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const BwdArgs &f = p.w;
  const int N = f.N;
  const bool has_z = f.z != nullptr;
  const int64_t n16 = (f.L + kBTT - 1) / kBTT;
  const uint32_t tile_bytes = (has_z ? 3u : 2u) * Lay::TILE +
                              (PROJ ? uint32_t(p.Rp) * RB : uint32_t(Lay::TILE)) + 2u * uint32_t(N) * RB;
  [[maybe_unused]] constexpr uint32_t kIdesc = mma_idesc_bf16(128, kBTT, false, true);
  [[maybe_unused]] uint32_t tbase = 0;
  [[maybe_unused]] int mma_issued = -1;

  if (tid == 0) {
#pragma unroll
    for (int s = 0; s < kBStages; ++s) mbar_init(&bars[s], 1);
    if (PROJ) {
      mbar_init(&mma_bar[0], 1);
      mbar_init(&mma_bar[1], 1);
    }
    fence_barrier_init();
    prefetch_tensormap(&tm_u);
    prefetch_tensormap(&tm_d);
    prefetch_tensormap(&tm_dy);
    prefetch_tensormap(&tm_B);
    prefetch_tensormap(&tm_C);
    if (has_z) prefetch_tensormap(&tm_z);
    q[8] = 0;
  }
  constexpr uint32_t kTmemCols = PROJ ? kProjTmemCols : uint32_t(Lay::TMEM_COLS);
  if (tid < 32) {
    tmem_alloc(reinterpret_cast<uint32_t *>(&q[12]), kTmemCols);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after_sync();
  tbase = uint32_t(q[12]);
  // this thread's lane: the state before segment s in columns s*NM .. (after
  // the projection's columns with PROJ)
  const uint32_t tsub = tmem_at(tbase, uint32_t(warp) * 32u, PROJ ? kProjBwdSub : 0u);

  // Issues (kMmaThread) the projection MMAs of consumed-tile index `ct` into
  // accumulator ct & 1 once the tile's dt_low rows have landed: 16 rows of
  // 32 bytes (two 256-byte swizzle atoms) per MMA.
  [[maybe_unused]] auto issue_mma = [&](int ct) {
    const int stg = ct % kBStages;
    if (!mbar_wait_bounded(&bars[stg], uint32_t(ct / kBStages) & 1u, p.timeout_ns)) {
      record_timeout();
      q[8] = 1;
      return;
    }
    tc_fence_after_sync();
    const uint32_t dt_addr = smem_u32(sm + stg * SST + Lay::TILE);
    const uint32_t acc = tbase + kProjBwdAcc + uint32_t(ct & 1) * kBTT;
    for (int kk = 0; kk < p.Rp / 16; ++kk) {
      const uint64_t bdesc = smem_desc(dt_addr + uint32_t(kk) * 512u, 16u, 256u, 6u);
      mma_ts(acc, tbase + uint32_t(kk) * 8u, bdesc, kIdesc, kk > 0);
    }
    mma_commit(&mma_bar[ct & 1]);
    mma_issued = ct;
  };

  // ---- producer (thread 0): tiles of the current unit, last tile first
  int p_ticket = 0, p_tile = 0, p_ntiles = 0, p_tail = 0, p_issued = 0;
  bool p_done = false;
  auto unit_tiles = [&](int ticket) {
    const int k = p.K - 1 - ticket / p.G;
    const int64_t t0 = int64_t(k) * p.chunk_len;
    const int64_t t1 = std::min<int64_t>(f.L, t0 + p.chunk_len);
    return int((t1 - t0 + kBTT - 1) / kBTT);
  };
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
    const int g = p_ticket % p.G, k = p.K - 1 - p_ticket / p.G;
    const int b = g / p.gpb, d0 = (g % p.gpb) * kSThreads;
    const int t0 = k * p.chunk_len + (p_ntiles - 1 - p_tile) * kBTT;
    const int stage = p_issued % kBStages;
    unsigned char *st = sm + stage * SST;
    uint64_t *bar = &bars[stage];
    mbar_arrive_expect_tx(bar, tile_bytes);
    tma_load_3d(st, &tm_u, bar, t0, d0, b);
    if (PROJ) tma_load_3d(st + Lay::TILE, &tm_d, bar, t0, 0, b);  // dt_low rows 0..Rp-1
    else tma_load_3d(st + Lay::TILE, &tm_d, bar, t0, d0, b);
    if (has_z) tma_load_3d(st + OFF_Z, &tm_z, bar, t0, d0, b);
    tma_load_3d(st + OFF_DY, &tm_dy, bar, t0, d0, b);
    tma_load_3d(st + OFF_B, &tm_B, bar, t0, 0, b);
    tma_load_3d(st + OFF_C, &tm_C, bar, t0, 0, b);
    ++p_tile;
    ++p_issued;
  };
  if (tid == 0) {
    produce(true);
    for (int s = 1; s < kBStages; ++s) produce(false);
  }

  int head = 0, ctile = 0;
  bool aborted = false;

  while (true) {
    __syncthreads();
    const int ticket = q[head & 7];
    ++head;
    if (ticket >= p.n_units) break;
    const int r = ticket / p.G;
    const int g = ticket % p.G, k = p.K - 1 - r;
    const int b = g / p.gpb, d0 = (g % p.gpb) * kSThreads;
    const int d = d0 + tid;
    const bool valid = d < f.dim;
    const int64_t tbeg = int64_t(k) * p.chunk_len;
    const int64_t tend = std::min<int64_t>(f.L, tbeg + p.chunk_len);
    const int ntiles = int((tend - tbeg + kBTT - 1) / kBTT);
    const int64_t row = (int64_t(b) * f.dim + (valid ? d : 0)) * f.L;  // row offset in (batch, dim, L)

    float Arow[NM];
#pragma unroll
    for (int n = 0; n < NM; ++n) Arow[n] = (valid && n < N) ? f.A[int64_t(d) * N + n] : -float(n + 1);
    if (valid) {
      const float pad0 = (Arow[0] < 0.f && isfinite(Arow[0])) ? Arow[0] : -1.f;
#pragma unroll
      for (int n = 1; n < NM; ++n)
        if (n >= N) Arow[n] = float(n + 1) * pad0;
    }
    const float bias = (valid && f.bias) ? f.bias[d] : 0.f;
    const float Dd = (valid && f.D) ? f.D[d] : 0.f;
    bool structured = Arow[0] < 0.f && isfinite(Arow[0]);
#pragma unroll
    for (int n = 1; n < NM; ++n) structured = structured && (Arow[n] == float(n + 1) * Arow[0]);
    const bool sig = structured && Arow[0] == -1.f;
    if constexpr (PROJ) {
      // this group's rows of W_dt into TMEM (as in the forward's fused projection)
      proj_load_w(static_cast<const __nv_bfloat16 *>(f.W_dt), d, valid, f.R, p.Rp,
                  tmem_at(tbase, uint32_t(warp) * 32u, 0));
      tmem_st_wait();
      tc_fence_before_sync();
      __syncthreads();
      if (tid == kMmaThread) issue_mma(ctile);
    }
    // The structured arithmetic keeps its relative accuracy for Delta |A0| in
    // 1e-5 .. 6: below, its dA cancels (Delta Abar B u against Bbar u); above,
    // its Abar = 1 + expm1 has only absolute accuracy, and ddelta (~Abar) loses
    // it.  A unit none of whose steps is in that range takes the generic
    // arithmetic (one exp per state, dA through psi'), which has neither
    // problem.  (The fused projection's kernels, whose delta is formed tile by
    // tile, decide per tile.)
    bool unit_extreme = false;
    if constexpr (!PROJ) {  // the unit's range flags (from the checkpoint pass): all set?
      if (p.range_flags) {
        const int64_t nblk = (f.L + kRangeBlock - 1) / kRangeBlock;
        const int64_t ub = int64_t(k) * p.chunk_len;
        const int64_t ue = std::min<int64_t>(f.L, ub + p.chunk_len);
        unit_extreme = true;
        for (int64_t i = ub / kRangeBlock + tid; i < (ue + kRangeBlock - 1) / kRangeBlock; i += kSThreads) {
          const int64_t fi = int64_t(g) * nblk + i;
          if (in_bounds(fi, p.n_flags) && !p.range_flags[fi]) unit_extreme = false;
        }
      }
    }
    int mode = MODE_GEN;
    if (!p.force_generic) {
      const bool ext = __syncthreads_and(unit_extreme);
      if (!ext && __syncthreads_and(sig)) mode = MODE_SIG;
      else if (!ext && __syncthreads_and(structured)) mode = MODE_STRUCT;
    }

    // adjoint entering from the later chunk
    float gt[NM];
#pragma unroll
    for (int n = 0; n < NM; ++n) gt[n] = 0.f;
    if (p.gin) {  // three-phase carry: the entering adjoint is known
#pragma unroll
      for (int n = 0; n < NM; ++n)
      {
        const int64_t i = ((int64_t(g) * p.K + k) * NM + n) * kSThreads + tid;
        gt[n] = in_bounds(i, p.n_gin) ? __ldcg(p.gin + i) : 0.f;
      }
    } else if (r > 0) {
      if (tid == 0 && !wait_flag_geq(p.flags + g, r, p.timeout_ns)) {
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
        gt[n] = in_bounds(i, p.n_carry) ? __ldcg(p.carry + i) : 0.f;
      }
    }
    float dA[NM];
    float dDsum = 0.f, dbsum = 0.f;
    ConvFilter cf = {0.f, 0.f, 0.f, 1.f, 0.f};
    if constexpr (CONV) {
      if (valid) cf = load_conv_filter(f.conv_w, f.conv_b, f.conv_width, d);
    }

    auto run = [&](auto mode_tag) {
      constexpr int M = decltype(mode_tag)::value;
      constexpr bool kS = M != MODE_GEN;
      const float A0 = Arow[0];
      const float invA0 = 1.f / A0;
      [[maybe_unused]] float d_lo = 0.f, d_hi = 0.f;  // the structured forms' range of delta
      if constexpr (kS && PROJ) structured_delta_range(A0, bias, d_lo, d_hi);
      // per-mode state: pairs for the structured arithmetic, scalars otherwise
      f2 Gt[NP], Acc[NP];
      float gs[NM], accs[NM], A2[NM], invA[NM];
      if constexpr (kS) {
#pragma unroll
        for (int i = 0; i < NP; ++i) {
          Gt[i] = pk(gt[2 * i], gt[2 * i + 1]);
          Acc[i] = pk(0.f, 0.f);
        }
      } else {
#pragma unroll
        for (int n = 0; n < NM; ++n) {
          gs[n] = gt[n];
          accs[n] = 0.f;
          A2[n] = Arow[n] * kLog2e;
          invA[n] = Arow[n] != 0.f ? 1.f / Arow[n] : 0.f;
        }
      }

      // Decays of one step: pairs (E(2i+1), E(2i+2)) for the structured
      // arithmetic; also returns Delta and sigma(v).
      auto step_decay = [&](float v, f2 (&P)[NP], float &Delta, float &sv) {
        if constexpr (M == MODE_SIG) {
          const float vc = fmaxf(v, -87.f);  // e^-v overflows below -88
          const float ev = ex2f(-vc * kLog2e);
          const float s = rcpf(1.f + ev);
          decay_pairs<NM>(-s, ev * s, P);
          sv = s;
          Delta = softplus_fast(v);
        } else {
          Delta = softplus_fast(v);
          const float E1 = expm1_neg(Delta * A0);
          decay_pairs<NM>(E1, 1.f + E1, P);
          sv = rcpf(1.f + ex2f(-v * kLog2e));
        }
      };

      for (int it = 0; it < ntiles; ++it, ++ctile) {
        const int tile = ntiles - 1 - it;  // tiles run from the end of the chunk
        const int64_t t0 = tbeg + int64_t(tile) * kBTT;
        const int steps = int(std::min<int64_t>(kBTT, tend - t0));
        const int nseg = steps / SEG;
        const int stage = ctile % kBStages;
        const uint32_t parity = uint32_t(ctile / kBStages) & 1u;
        unsigned char *st = sm + stage * SST;
        // checkpoint of the tile start (issued before the wait to overlap)
        float h0[NM];
        {
          const int64_t ci = ((int64_t(g) * n16 + t0 / kBTT) * NM) * kSThreads + tid;
          const float *ck = p.ckpt + (in_bounds(ci + (NM - 1) * kSThreads, p.n_ckpt) ? ci : 0);
#pragma unroll
          for (int n = 0; n < NM; ++n) h0[n] = __ldcg(ck + n * kSThreads);
        }
        if (p.ckpt_hin && t0 >= p.ckpt_chunk) {  // a checkpoint stored from a zero chunk start
          const int64_t kf = t0 / p.ckpt_chunk;
          const int64_t cc = (int64_t(g) * n16 + t0 / kBTT) * kSThreads + tid;
          const float cum = in_bounds(cc, p.n_ckpt_cum) ? __ldcg(p.ckpt_cum + cc) : 0.f;
          const int64_t hb = ((int64_t(g) * p.ckpt_K + kf) * NM) * kSThreads + tid;
          const float *hin = p.ckpt_hin + (in_bounds(hb + (NM - 1) * kSThreads, p.n_ckpt_hin) ? hb : 0);
          if constexpr (kS) {  // A_n = (n+1) A0: the decays are powers of the first
            const float e1 = ex2f(A0 * cum * kLog2e);
            float e = e1;
#pragma unroll
            for (int n = 0; n < NM; ++n) {
              h0[n] = fmaf(e, __ldcg(hin + n * kSThreads), h0[n]);
              e *= e1;
            }
          } else {
#pragma unroll
            for (int n = 0; n < NM; ++n) h0[n] = fmaf(ex2f(A2[n] * cum), __ldcg(hin + n * kSThreads), h0[n]);
          }
        }
        // convolution prologue: x at the four steps before the tile (0 before
        // the sequence start and on padding channels)
        [[maybe_unused]] float hx[4] = {0.f, 0.f, 0.f, 0.f};
        if constexpr (CONV) {
          if (valid && t0 > 0 && in_bounds(row + t0 - 4, f.batch * f.dim * f.L))
            load_x4(static_cast<const T *>(f.u) + row + t0 - 4, hx);
        }
        if (!mbar_wait_bounded(&bars[stage], parity, p.timeout_ns)) {
          record_timeout();
          q[8] = 1;
        }
        [[maybe_unused]] bool d_in = false;  // (PROJ) a step of the tile in [d_lo, d_hi]
        if constexpr (PROJ) {  // this tile's delta: wait for its MMA, then one TMEM load
          if (!mbar_wait_bounded(&mma_bar[ctile & 1], uint32_t(ctile >> 1) & 1u, p.timeout_ns)) {
            record_timeout();
            q[8] = 1;
          }
          tc_fence_after_sync();
          float dt16[kBTT];  // warp-collective load: every lane takes part
          tmem_ld16(tmem_at(tbase + kProjBwdAcc + uint32_t(ctile & 1) * kBTT, uint32_t(warp) * 32u, 0), dt16);
          tmem_ld_wait();
          float2 *ds = reinterpret_cast<float2 *>(sm + OFF_DS);
#pragma unroll
          for (int sg = 0; sg < kBTT / 2; ++sg) ds[sg * kSThreads + tid] = make_float2(dt16[2 * sg], dt16[2 * sg + 1]);
          if constexpr (kS) {
#pragma unroll
            for (int i = 0; i < kBTT; ++i) d_in = d_in || (dt16[i] >= d_lo && dt16[i] <= d_hi);
          }
        }
        {
          const T *Braw = reinterpret_cast<const T *>(st + OFF_B);
          const T *Craw = reinterpret_cast<const T *>(st + OFF_C);
          constexpr int ITEMS = NM * (kBTT / 4);
          for (int w = tid; w < 2 * ITEMS; w += kSThreads) {
            const bool isC = w >= ITEMS;
            const int rr = isC ? w - ITEMS : w;
            const int n = rr % NM, tg = rr / NM;
            const T *src = (isC ? Craw : Braw) + n * kBTT + 4 * tg;
            float *dst = (isC ? Cs : Bs) + 4 * tg * BSTR + n;
            const float scale = (!isC && kS) ? 1.f / float(n + 1) : 1.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i * BSTR] = n < N ? raw_to_f(src, i) * scale : 0.f;
          }
        }
        bool tile_gen = false;
        if constexpr (kS && PROJ) {  // no step of the tile in the structured range?
          tile_gen = !__syncthreads_or(valid && d_in);
        } else {
          __syncthreads();
        }
        if (q[8]) return;

        const unsigned char *su = st;
        [[maybe_unused]] const unsigned char *sd = st + Lay::TILE;
        const unsigned char *sz = st + OFF_Z;
        const unsigned char *sdy = st + OFF_DY;

        // delta of one segment: from the tile, or (PROJ) from TMEM
        auto load_d = [&](int seg, float (&dv)[SEG]) {
          if constexpr (PROJ) {  // this thread's pair, stored at the tile's start
            static_assert(SEG == 2, "two-step segments in bf16");
            const float2 v = reinterpret_cast<const float2 *>(sm + OFF_DS)[seg * kSThreads + tid];
            dv[0] = v.x;
            dv[1] = v.y;
          } else {
            IO::load(sd, tid, seg, dv);
          }
        };

        // u of one segment of the tile
        auto load_u = [&](int seg, float (&uv)[SEG]) {
          IO::load(su, tid, seg, uv);
          if constexpr (CONV) {
            float win[SEG + 3];  // x at the steps seg*SEG-3 .. seg*SEG+SEG-1 of the tile
            if constexpr (SEG == 2) {
              float p1[2], p2[2];
              if (seg >= 1) {
                IO::load(su, tid, seg - 1, p1);
              } else {
                p1[0] = hx[2];
                p1[1] = hx[3];
              }
              if (seg >= 2) {
                IO::load(su, tid, seg - 2, p2);
              } else {
                p2[0] = seg == 1 ? hx[2] : hx[0];
                p2[1] = seg == 1 ? hx[3] : hx[1];
              }
              win[0] = p2[1];
              win[1] = p1[0];
              win[2] = p1[1];
            } else {
              static_assert(SEG == 4, "segments of 2 or 4 steps");
              float p1[4];
              if (seg >= 1) {
                IO::load(su, tid, seg - 1, p1);
              } else {
#pragma unroll
                for (int i = 0; i < 4; ++i) p1[i] = hx[i];
              }
              win[0] = p1[1];
              win[1] = p1[2];
              win[2] = p1[3];
            }
#pragma unroll
            for (int i = 0; i < SEG; ++i) win[3 + i] = uv[i];
#pragma unroll
            for (int i = 0; i < SEG; ++i) {
              const float pre = conv_pre(cf, win[i], win[i + 1], win[i + 2], win[i + 3]);
              uv[i] = pre * rcpf(1.f + ex2f(-pre * kLog2e));
            }
          }
        };

        // One tile with the structured (S) or the generic arithmetic.
        auto tile_body = [&](auto stag) {
          constexpr bool S = decltype(stag)::value;
          // forward over the tile: the state before every segment -> tensor memory
          {
            f2 H[NP];
            float h[NM];
            if constexpr (S) {
  #pragma unroll
              for (int i = 0; i < NP; ++i) H[i] = pk(h0[2 * i], h0[2 * i + 1]);
            } else {
  #pragma unroll
              for (int n = 0; n < NM; ++n) h[n] = h0[n];
            }
            for (int seg = 0; seg < nseg; ++seg) {
              {  // one tensor-memory store of the NM states
                float hv[NM];
                if constexpr (S) {
  #pragma unroll
                  for (int i = 0; i < NP; ++i) {
                    hv[2 * i] = lo_of(H[i]);
                    hv[2 * i + 1] = hi_of(H[i]);
                  }
                } else {
  #pragma unroll
                  for (int n = 0; n < NM; ++n) hv[n] = h[n];
                }
                tmem_st_row<NM>(tsub + uint32_t(seg * NM), hv);
              }
              if (seg == nseg - 1) break;  // the last segment is re-run below anyway
              float uv[SEG], dv[SEG];
              load_u(seg, uv);
              load_d(seg, dv);
  #pragma unroll
              for (int i = 0; i < SEG; ++i) {
                const float *Brow = Bs + (seg * SEG + i) * BSTR;
                if constexpr (S) {
                  f2 P[NP];
                  float Delta, sv;
                  step_decay(dv[i] + bias, P, Delta, sv);
                  struct_update<NM>(H, P, uv[i] * invA0, 0.f, Brow, Brow);
                } else {
                  const float Delta = softplus_fast(dv[i] + bias);
                  generic_update<NM, kS>(h, Delta, uv[i], 0.f, Arow, A2, invA, Brow, Brow);
                }
              }
            }
          }

          tmem_st_wait();  // the segment states, before they are read back

          // the next tile's projection MMA, into the other accumulator
          if constexpr (PROJ) {
            if (tid == kMmaThread && it + 1 < ntiles) issue_mma(ctile + 1);
            __syncwarp();
          }

          // segments from the last: re-run into registers, then walk backwards
          for (int seg = nseg - 1; seg >= 0; --seg) {
            float uv[SEG], dv[SEG], zv[SEG], dyv[SEG];
            load_u(seg, uv);
            load_d(seg, dv);
            IO::load(sdy, tid, seg, dyv);
            if (has_z) IO::load(sz, tid, seg, zv);
            float du_o[SEG], dd_o[SEG], dz_o[SEG];

            if constexpr (S) {
              // states before each step of the segment (the state after a step
              // is recomputed in the reverse step from h_{t-1} and t1)
              f2 Hs[SEG][NP];
              {
                float hv[NM];
                tmem_ld_row<NM>(tsub + uint32_t(seg * NM), hv);
                tmem_ld_wait();
  #pragma unroll
                for (int i = 0; i < NP; ++i) Hs[0][i] = pk(hv[2 * i], hv[2 * i + 1]);
              }
  #pragma unroll
              for (int i = 0; i + 1 < SEG; ++i) {
                const float *Brow = Bs + (seg * SEG + i) * BSTR;
                f2 P[NP];
                float Delta, sv;
                step_decay(dv[i] + bias, P, Delta, sv);
  #pragma unroll
                for (int j = 0; j < NP; ++j) Hs[i + 1][j] = Hs[i][j];
                struct_update<NM>(Hs[i + 1], P, uv[i] * invA0, 0.f, Brow, Brow);
              }
  #pragma unroll
              for (int i = SEG - 1; i >= 0; --i) {
                const int tl = seg * SEG + i;
                const float *Brow = Bs + tl * BSTR;
                const float *Crow = Cs + tl * BSTR;
                f2 P[NP];
                float Delta, sv;
                step_decay(dv[i] + bias, P, Delta, sv);
                float dy0 = dyv[i], sz = 0.f;
                if (has_z) {
                  sz = rcpf(1.f + ex2f(-zv[i] * kLog2e));
                  dy0 *= zv[i] * sz;
                }
                const float up = uv[i] * invA0;
                const float x1 = Delta * A0;
                const f2 U = pk(up, up), DY = pk(dy0, dy0), X1n = pk(-x1, -x1), Z = pk(0.f, 0.f);
                f2 DU = Z, DD = Z, Y0 = Z;
                const bool up16 = (lane & 16) != 0;
                f2 v2[8];
  #pragma unroll
                for (int j = 0; j < NP; j += 2) {
                  const ulonglong2 bq = *reinterpret_cast<const ulonglong2 *>(Brow + 2 * j);
                  const ulonglong2 cq2 = *reinterpret_cast<const ulonglong2 *>(Crow + 2 * j);
  #pragma unroll
                  for (int e = 0; e < 2; ++e) {
                    const int jj = j + e;
                    const f2 Bp = e ? bq.y : bq.x;
                    const f2 Cp = e ? cq2.y : cq2.x;
                    const f2 CN = pk(float(2 * jj + 1), float(2 * jj + 2));
                    const f2 Gv = fma2(Cp, DY, Gt[jj]);
                    const f2 Ga = fma2(Gv, P[jj], Gv);
                    const f2 w = fma2(Gv, P[jj], Z);
                    const f2 t1 = fma2(Bp, U, Hs[i][jj]);
                    const f2 hcur = fma2(P[jj], t1, Hs[i][jj]);  // h_t
                    const f2 cq = fma2(fma2(Ga, t1, Z), CN, Z);
                    DD = fma2(cq, pk(1.f, 1.f), DD);
                    Acc[jj] = fma2(X1n, cq, Acc[jj]);
                    const f2 dBc = fma2(w, U, Z);
                    Acc[jj] = fma2(dBc, Bp, Acc[jj]);
                    DU = fma2(w, Bp, DU);
                    Y0 = fma2(Cp, hcur, Y0);
                    const f2 dCc = fma2(DY, hcur, Z);
                    Gt[jj] = Ga;
                    // Channels past `dim` contribute exact zeros: TMA fills their
                    // rows with 0, so dy0 = 0 and their adjoint stays 0.
                    v2[jj] = bfly_first2(dBc, dCc, up16);
                  }
                }
  #pragma unroll
                for (int jj = NM / 2; jj < kMaxN / 2; ++jj) v2[jj] = pk(0.f, 0.f);
                const float du = fmaf(lo_of(DU) + hi_of(DU), invA0, Dd * dy0);
                const float dd = A0 * (lo_of(DD) + hi_of(DD)) * sv;
                const float y0 = (lo_of(Y0) + hi_of(Y0)) + Dd * uv[i];
                du_o[i] = du;
                dd_o[i] = dd;
                dz_o[i] = has_z ? dyv[i] * y0 * sz * (1.f + zv[i] * (1.f - sz)) : 0.f;
                dDsum = fmaf(dy0, uv[i], dDsum);
                dbsum += dd;
                const float rsum = bfly_rest2(v2, lane);
                // lane l holds dB (l < 16, to be divided by l+1) or dC of state l-16
                red[(warp * kBTT + tl) * 33 + lane] = (lane < kMaxN) ? rsum * (1.f / float(lane + 1)) : rsum;
              }
            } else {
              float Hs[SEG][NM];
              tmem_ld_row<NM>(tsub + uint32_t(seg * NM), Hs[0]);
              tmem_ld_wait();
  #pragma unroll
              for (int i = 0; i + 1 < SEG; ++i) {
                const float *Brow = Bs + (seg * SEG + i) * BSTR;
                const float Delta = softplus_fast(dv[i] + bias);
  #pragma unroll
                for (int n = 0; n < NM; ++n) Hs[i + 1][n] = Hs[i][n];
                generic_update<NM, kS>(Hs[i + 1], Delta, uv[i], 0.f, Arow, A2, invA, Brow, Brow);
              }
  #pragma unroll
              for (int i = SEG - 1; i >= 0; --i) {
                const int tl = seg * SEG + i;
                const float *Brow = Bs + tl * BSTR;
                const float *Crow = Cs + tl * BSTR;
                const float v = dv[i] + bias;
                const float Delta = softplus_fast(v);
                const float sv = rcpf(1.f + ex2f(-v * kLog2e));
                float dy0 = dyv[i], sz = 0.f;
                if (has_z) {
                  sz = rcpf(1.f + ex2f(-zv[i] * kLog2e));
                  dy0 *= zv[i] * sz;
                }
                float du_acc = 0.f, dD_acc = 0.f, y0 = Dd * uv[i];
                const bool up16 = (lane & 16) != 0;
                float v16[16];
  #pragma unroll
                for (int n = 0; n < NM; ++n) {
                  const float x = Delta * Arow[n];
                  const float a = ex2f(Delta * A2[n]);
                  float pp = fmaf(x, 1.f / 720.f, 1.f / 120.f);
                  pp = fmaf(x, pp, 1.f / 24.f);
                  pp = fmaf(x, pp, 1.f / 6.f);
                  pp = fmaf(x, pp, 0.5f);
                  pp = fmaf(x, pp, 1.f);
                  const float Eb = fabsf(x) < 0.25f ? Delta * pp : (a - 1.f) * invA[n];  // Bbar / B
                  const float Bn = kS ? Brow[n] * float(n + 1) : Brow[n], Cn = Crow[n];
                  const float hprev = Hs[i][n];
                  const float hcur = fmaf(a, hprev, Eb * (Bn * uv[i]));  // h_t, as in the forward
                  const float Gv = fmaf(Cn, dy0, gs[n]);
                  const float Ga = a * Gv;
                  const float wv = Gv * Eb;
                  du_acc = fmaf(wv, Bn, du_acc);
                  dD_acc = fmaf(Ga, fmaf(Bn, uv[i], Arow[n] * hprev), dD_acc);
                  accs[n] = fmaf(Gv, Delta * a * hprev + Bn * uv[i] * Delta * Delta * dpsi_fast(x, a), accs[n]);
                  y0 = fmaf(Cn, hcur, y0);
                  v16[n] = bfly_first(wv * uv[i], dy0 * hcur, up16);  // zero past `dim`
                  gs[n] = Ga;
                }
  #pragma unroll
                for (int n = NM; n < kMaxN; ++n) v16[n] = 0.f;
                const float dd = dD_acc * sv;
                du_o[i] = fmaf(Dd, dy0, du_acc);
                dd_o[i] = dd;
                dz_o[i] = has_z ? dyv[i] * y0 * sz * (1.f + zv[i] * (1.f - sz)) : 0.f;
                dDsum = fmaf(dy0, uv[i], dDsum);
                dbsum += dd;
                red[(warp * kBTT + tl) * 33 + lane] = bfly_rest(v16, lane);
              }
            }
            if (valid) {
              const int64_t o = row + t0 + seg * SEG;
              if (in_bounds(o + SEG - 1, f.batch * f.dim * f.L)) {
                IO::store(static_cast<T *>(f.du) + o, du_o);
                IO::store(static_cast<T *>(f.ddelta) + o, dd_o);
                if (has_z) IO::store(static_cast<T *>(f.dz) + o, dz_o);
              }
            }
          }
        };
        if constexpr (kS && PROJ) {
          if (tile_gen) {
            // No step of this tile has Delta |A0| in the range where the
            // structured arithmetic keeps its relative accuracy (1e-5 .. 6):
            // the tile runs the generic arithmetic (one exp per state, dA
            // through psi'), whose dA has no cancellation at small Delta and
            // whose Abar keeps its relative accuracy at large Delta.
#pragma unroll
            for (int n = 0; n < NM; ++n) {
              gs[n] = (n & 1) ? hi_of(Gt[n >> 1]) : lo_of(Gt[n >> 1]);
              accs[n] = 0.f;
              A2[n] = Arow[n] * kLog2e;
              invA[n] = Arow[n] != 0.f ? 1.f / Arow[n] : 0.f;
            }
            tile_body(std::false_type{});
#pragma unroll
            for (int i = 0; i < NP; ++i) {  // back to the structured units (Acc = -A_n dA_n)
              Gt[i] = pk(gs[2 * i], gs[2 * i + 1]);
              Acc[i] = fma2(pk(-Arow[2 * i], -Arow[2 * i + 1]), pk(accs[2 * i], accs[2 * i + 1]), Acc[i]);
            }
          } else {
            tile_body(std::true_type{});
          }
        } else {
          tile_body(std::integral_constant<bool, kS>{});
        }
        if (PROJ) tc_fence_before_sync();
        __syncthreads();
        // CTA sums of dB / dC for this tile -> partials
        for (int idx = tid; idx < 32 * kBTT; idx += kSThreads) {
          const int slot = idx / kBTT, tl = idx % kBTT;
          if (tl < steps) {
            float sum = 0.f;
#pragma unroll
            for (int wv = 0; wv < kSThreads / 32; ++wv) sum += red[(wv * kBTT + tl) * 33 + slot];
            const int64_t bi = ((int64_t(g % p.gpb) * f.batch + b) * 32 + slot) * f.L + t0 + tl;
            if (in_bounds(bi, p.n_bc)) p.part_bc[bi] = sum;
          }
        }
        if (tid == 0) produce(false);
      }
      // unit results
      if constexpr (kS) {
#pragma unroll
        for (int i = 0; i < NP; ++i) {
          gt[2 * i] = lo_of(Gt[i]);
          gt[2 * i + 1] = hi_of(Gt[i]);
          // Acc holds -A_n dA_n
          dA[2 * i] = -lo_of(Acc[i]) / (float(2 * i + 1) * A0);
          dA[2 * i + 1] = -hi_of(Acc[i]) / (float(2 * i + 2) * A0);
        }
      } else {
#pragma unroll
        for (int n = 0; n < NM; ++n) {
          gt[n] = gs[n];
          dA[n] = accs[n];
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

    const int64_t pu = int64_t(g) * p.K + k;
#pragma unroll
    for (int n = 0; n < NM; ++n)
      if (in_bounds((pu * NM + n) * kSThreads + tid, p.n_unit * NM))
        p.part_A[(pu * NM + n) * kSThreads + tid] = valid ? dA[n] : 0.f;
    if (in_bounds(pu * kSThreads + tid, p.n_unit)) {
      p.part_D[pu * kSThreads + tid] = valid ? dDsum : 0.f;
      p.part_bias[pu * kSThreads + tid] = valid ? dbsum : 0.f;
    }
    if (k > 0 && !p.gin) {
#pragma unroll
      for (int n = 0; n < NM; ++n)
        if (in_bounds((int64_t(g) * NM + n) * kSThreads + tid, p.n_carry))
          p.carry[(int64_t(g) * NM + n) * kSThreads + tid] = gt[n];
      __threadfence();
      __syncthreads();
      if (tid == 0 && !(p.test_hook == 1 && g == 0 && r == 0)) st_release_gpu(p.flags + g, r + 1);
    }
    if (tid == 0) {  // claim the next unit and fill the free stages
      produce(true);
      while (!p_done && p_issued < ctile + kBStages && p_tile < p_ntiles) produce(false);
    }
  }

  __syncthreads();
  if (tid == 0 && aborted) {
    for (int t = ctile; t < p_issued; ++t)
      mbar_wait_bounded(&bars[t % kBStages], uint32_t(t / kBStages) & 1u, p.timeout_ns);
  }
  if constexpr (PROJ) {  // every MMA issued must complete before TMEM is freed
    if (tid == kMmaThread && mma_issued >= 0)
      mbar_wait_bounded(&mma_bar[mma_issued & 1], uint32_t(mma_issued >> 1) & 1u, p.timeout_ns);
  } else {
    tmem_st_wait();
  }
  tc_fence_before_sync();
  __syncthreads();
  if (tid < 32) {
    tc_fence_after_sync();
    tmem_dealloc(tbase, kTmemCols);
  }
}

// Three-phase carry of the adjoint, used when there are too few channel groups
// to fill the GPU with whole-sequence units.  The adjoint recurrence
//     Ga_t = Abar_t (C_t dy0_t + Ga_{t+1})
// does not involve the states, and it is linear: a chunk that starts from the
// carried Ga_in produces  Ga_local + exp(A_n sum_chunk Delta) Ga_in,  where
// Ga_local is what it produces from zero (the associative combine of affine
// maps of the trishampatil.com walk-through, Part III section 2, run
// backwards).  This kernel computes Ga_local and sum Delta of every chunk but
// the first, one thread per (channel, chunk) walking the chunk from its end;
// the parallel scan over chunks (chunk_scan_kernel, from the last chunk)
// combines them, and the main reverse kernel then runs every chunk from its
// true entering adjoint.
template <typename T, int NM, typename TD = T>
__global__ void __launch_bounds__(kSThreads) bwd_adjoint_agg_kernel(const BwdStagedArgs p) {
  constexpr int V = Vec<T>::kN;  // steps per 16-byte vector
  __shared__ float cs[NM * V];   // the C rows of the current V steps
  const BwdArgs &f = p.w;
  const int unit = blockIdx.x;  // < G * (K - 1)
  const int g = unit % p.G, k = p.K - 1 - unit / p.G;
  const int b = g / p.gpb, d_raw = (g % p.gpb) * kSThreads + threadIdx.x;
  const bool valid = d_raw < f.dim;
  const int64_t d = valid ? d_raw : f.dim - 1;  // loads stay in bounds
  const int N = f.N;
  const int64_t row = (int64_t(b) * f.dim + d) * f.L;
  const TD *dl = static_cast<const TD *>(f.delta) + row;
  const T *dy = static_cast<const T *>(f.dy) + row;
  const T *z = f.z ? static_cast<const T *>(f.z) + row : nullptr;
  const T *Cp = static_cast<const T *>(f.C) + int64_t(b) * N * f.L;
  const float bias = f.bias ? f.bias[d] : 0.f;
  float Arow[NM], Ga[NM];
#pragma unroll
  for (int n = 0; n < NM; ++n) {
    Arow[n] = n < N ? f.A[d * N + n] : float(n + 1) * f.A[d * N];
    Ga[n] = 0.f;
  }
  // S4D-Real structure (as in the forward): all decays from one expm1
  bool structured = Arow[0] < 0.f && isfinite(Arow[0]) && !p.force_generic;
#pragma unroll
  for (int n = 1; n < NM; ++n) structured = structured && (Arow[n] == float(n + 1) * Arow[0]);
  const int64_t tbeg = int64_t(k) * p.chunk_len;
  const int64_t tend = std::min<int64_t>(f.L, tbeg + p.chunk_len);
  double S = 0.0;
  // V steps at a time from the chunk's end (rows are 16-byte aligned multiples
  // of 16 bytes and chunks start at multiples of 64 steps): every load of the V
  // steps is issued before it is used
  for (int64_t tb = tend - V; tb >= tbeg; tb -= V) {
    if (!in_bounds(row + tb + V - 1, f.batch * f.dim * f.L)) break;
    float dv[V], dyv[V], zv[V];
    if constexpr (std::is_same<TD, T>::value) {
      Vec<T>::unpack(*reinterpret_cast<const uint4 *>(dl + tb), dv);
    } else {  // fp32 delta beside bf16 tiles: V / 4 vectors of four
#pragma unroll
      for (int v4 = 0; v4 < V / 4; ++v4) {
        float tmp[4];
        Vec<float>::unpack(*reinterpret_cast<const uint4 *>(dl + tb + 4 * v4), tmp);
#pragma unroll
        for (int i = 0; i < 4; ++i) dv[4 * v4 + i] = tmp[i];
      }
    }
    Vec<T>::unpack(*reinterpret_cast<const uint4 *>(dy + tb), dyv);
    if (z) Vec<T>::unpack(*reinterpret_cast<const uint4 *>(z + tb), zv);
    __syncthreads();  // the previous steps' C rows are no longer read
    if (threadIdx.x < NM * V) {
      const int n = threadIdx.x / V, i = threadIdx.x % V;
      cs[threadIdx.x] = n < N ? to_f(Cp[int64_t(n) * f.L + tb + i]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int i = V - 1; i >= 0; --i) {
      const float Delta = softplus_fast(dv[i] + bias);
      S += double(Delta);
      float dy0 = dyv[i];
      if (z) dy0 *= zv[i] * rcpf(1.f + ex2f(-zv[i] * kLog2e));
      if (structured) {
        const float E1 = expm1_neg(Delta * Arow[0]);
        f2 P[NM / 2];
        decay_pairs<NM>(E1, 1.f + E1, P);
        const f2 DY = pk(dy0, dy0);
#pragma unroll
        for (int j = 0; j < NM / 2; ++j) {
          const f2 c = pk(cs[(2 * j) * V + i], cs[(2 * j + 1) * V + i]);
          const f2 v = fma2(c, DY, pk(Ga[2 * j], Ga[2 * j + 1]));
          const f2 w = fma2(P[j], v, v);  // Abar v = v + E v
          Ga[2 * j] = lo_of(w);
          Ga[2 * j + 1] = hi_of(w);
        }
      } else {
#pragma unroll
        for (int n = 0; n < NM; ++n)
          if (n < N) Ga[n] = ex2f(Delta * Arow[n] * kLog2e) * fmaf(cs[n * V + i], dy0, Ga[n]);
      }
    }
  }
#pragma unroll
  for (int n = 0; n < NM; ++n)
    if (in_bounds(((int64_t(g) * p.K + k) * NM + n) * kSThreads + threadIdx.x, p.n_gin))
      p.agg_G[((int64_t(g) * p.K + k) * NM + n) * kSThreads + threadIdx.x] = valid ? Ga[n] : 0.f;
  if (in_bounds((int64_t(g) * p.K + k) * kSThreads + threadIdx.x, p.n_unit))
    p.agg_S[(int64_t(g) * p.K + k) * kSThreads + threadIdx.x] = valid ? S : 0.0;
}

// Four consecutive outputs in one store (8 bytes of bf16, 16 of fp32).
template <typename T> struct Vec4Out;
template <> struct Vec4Out<float> {
  __device__ static void store(float *dst, const float (&v)[4]) {
    *reinterpret_cast<float4 *>(dst) = make_float4(v[0], v[1], v[2], v[3]);
  }
};
template <> struct Vec4Out<__nv_bfloat16> {
  __device__ static void store(__nv_bfloat16 *dst, const float (&v)[4]) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]), c = __floats2bfloat162_rn(v[2], v[3]);
    uint2 w;
    w.x = *reinterpret_cast<const uint32_t *>(&a);
    w.y = *reinterpret_cast<const uint32_t *>(&c);
    *reinterpret_cast<uint2 *>(dst) = w;
  }
};

// dB / dC: sum of the per-CTA partials over the channel groups of a batch row,
// four consecutive steps per thread (16-byte loads; L is a multiple of 4 on
// this path), each element summed over the groups in order.
template <typename T>
__global__ void bwd_staged_finalize_bc(const BwdStagedArgs p) {
  const BwdArgs &f = p.w;
  const int64_t L4 = f.L / 4;
  const int64_t total = f.batch * f.N * L4;
  const bool vec_out = ((reinterpret_cast<uintptr_t>(f.dB) | reinterpret_cast<uintptr_t>(f.dC)) %
                        (4 * sizeof(T))) == 0;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t t = (i % L4) * 4, n = (i / L4) % f.N, b = i / (L4 * f.N);
    float4 sb = make_float4(0.f, 0.f, 0.f, 0.f), sc = sb;
#pragma unroll 8
    for (int j = 0; j < p.gpb; ++j) {
      const int64_t o = ((int64_t(j) * f.batch + b) * 32) * f.L + t;
      if (!in_bounds(o + (kMaxN + n) * f.L + 3, p.n_bc)) break;
      const float4 xb = __ldcs(reinterpret_cast<const float4 *>(p.part_bc + o + n * f.L));
      const float4 xc = __ldcs(reinterpret_cast<const float4 *>(p.part_bc + o + (kMaxN + n) * f.L));
      sb.x += xb.x; sb.y += xb.y; sb.z += xb.z; sb.w += xb.w;
      sc.x += xc.x; sc.y += xc.y; sc.z += xc.z; sc.w += xc.w;
    }
    const int64_t e = (b * f.N + n) * f.L + t;  // first of the four outputs
    T *dB = static_cast<T *>(f.dB) + e;
    T *dC = static_cast<T *>(f.dC) + e;
    if (vec_out) {
      const float vb[4] = {sb.x, sb.y, sb.z, sb.w}, vc[4] = {sc.x, sc.y, sc.z, sc.w};
      Vec4Out<T>::store(dB, vb);
      Vec4Out<T>::store(dC, vc);
    } else {
      dB[0] = from_f<T>(sb.x); dB[1] = from_f<T>(sb.y); dB[2] = from_f<T>(sb.z); dB[3] = from_f<T>(sb.w);
      dC[0] = from_f<T>(sc.x); dC[1] = from_f<T>(sc.y); dC[2] = from_f<T>(sc.z); dC[3] = from_f<T>(sc.w);
    }
  }
}

// dA, dD, dbias: sums over batch rows and chunks of the per-unit partials.
template <int NM>
__global__ void bwd_staged_finalize_params(const BwdStagedArgs p) {
  const BwdArgs &f = p.w;
  const int64_t total = f.dim * f.N;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t d = i / f.N, n = i % f.N;
    const int64_t gi = d / kSThreads, c = d % kSThreads;
    float s = 0.f, sd = 0.f, sb = 0.f;
    for (int64_t b = 0; b < f.batch; ++b) {
      const int64_t g = b * p.gpb + gi;
      for (int k = 0; k < p.K; ++k) {
        const int64_t pu = g * p.K + k;
        s += p.part_A[(pu * NM + n) * kSThreads + c];
        if (n == 0) {
          sd += p.part_D[pu * kSThreads + c];
          sb += p.part_bias[pu * kSThreads + c];
        }
      }
    }
    f.dA[i] = s;
    if (n == 0) {
      if (f.dD) f.dD[d] = sd;
      if (f.dbias) f.dbias[d] = sb;
    }
  }
}

// Whether the staged backward takes this problem (as the staged forward).
inline bool staged_bwd_supported(const BwdArgs &a, size_t es) {
  auto al = [](const void *ptr) { return ptr == nullptr || (reinterpret_cast<uintptr_t>(ptr) & 15) == 0; };
  if (a.N < 3) return false;
  if ((a.L * int64_t(es)) % 16 != 0 || a.L % 4 != 0) return false;
  if (a.L > (int64_t(1) << 31) - 1024 || a.dim > (int64_t(1) << 31) - 1) return false;
  return al(a.u) && al(a.delta) && al(a.z) && al(a.dy) && al(a.B) && al(a.C) && al(a.du) &&
         al(a.ddelta) && al(a.dz);
}

// Dynamic shared memory of the fused-projection backward (its stages hold the
// Rp x 16 dt_low tile in place of delta's; the tile's fp32 delta follows).
template <typename T, int NM>
inline int proj_bwd_smem_bytes(int Rp) {
  using Lay = BwdLayout<T, NM, true>;
  constexpr int kDeltaBytes = kBTT * kSThreads * 4 + 16;  // the tile's delta (and its alignment)
  return int(kBStages * BwdStage<T, NM>(Rp).bytes) + (Lay::BYTES - Lay::OFF_SUB) + kDeltaBytes + 512;
}

// Largest R the fused projection takes: its tiles must leave room for two
// CTAs per SM in both the forward and the backward, and W_dt's columns must
// end before the backward's delta accumulators in tensor memory.
template <typename T, int NM>
inline int proj_max_rank() {
  int r = 16;
  while (r + 16 <= kProjBwdMaxRp && proj_bwd_smem_bytes<T, NM>(r + 16) <= kTwoPerSmBytes) r += 16;
  return r;
}

// The backward's chunking of its adjoint carry, as staged_backward decides it
// (for a caller that must know it without launching anything).
template <typename T, int NM, bool CONV = false, bool PROJ = false>
inline mamba_status_t staged_backward_plan(int64_t batch, int64_t dim, int64_t L, const StagedOptions &o,
                                           int R, StagedPlan *pl) {
  using Lay = BwdLayout<T, NM, true>;
  int smem = Lay::ALLOC;
  if (PROJ) {
    const int Rp = (R + 15) / 16 * 16;
    if (R < 1 || Rp > proj_max_rank<T, NM>()) return MAMBA_ERR_UNSUPPORTED;
    smem = proj_bwd_smem_bytes<T, NM>(Rp);
  }
  auto kern = bwd_staged_kernel<T, NM, CONV, PROJ>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return MAMBA_ERR_CUDA;
  int bps = 0;
  if (resident_ctas(kern, smem, PROJ ? int(kProjTmemCols) : Lay::TMEM_COLS, &bps) != cudaSuccess)
    return MAMBA_ERR_CUDA;
  const int slots = device_sm_count() * std::max(1, bps);
  const int64_t G = batch * ceil_div(dim, kSThreads);
  *pl = plan_staged(G, L, slots, o, 256);
  return MAMBA_OK;
}

// With `saved`, the checkpoints, range flags and (three-phase) h_in and sums
// of Delta come from
// a saving forward of the same inputs and options, laid out as saved_layout
// gives it, and the checkpoint pass does not run.
template <typename T, int NM, bool CONV = false, bool PROJ = false>
mamba_status_t staged_backward(const BwdArgs &a, const StagedOptions &o, cudaStream_t s,
                               mamba_status_t (*launched)(), const unsigned char *saved = nullptr) {
  SavedLayout sl;
  if (saved) {
    const mamba_status_t ls = saved_layout<T, NM, CONV, PROJ>(a.batch, a.dim, a.L, o, &sl, a.R);
    if (ls != MAMBA_OK) return ls;
  }
  using Lay = BwdLayout<T, NM, true>;
  constexpr bool bf16 = std::is_same<T, __nv_bfloat16>::value;
  const uint64_t L = a.L, dim = a.dim, batch = a.batch, N = a.N;
  const CUtensorMapSwizzle sw = bf16 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_64B;
  const CUtensorMapSwizzle none = CU_TENSOR_MAP_SWIZZLE_NONE;
  CUtensorMap maps[6];
  int Rp = 0, smem = Lay::ALLOC;
  if (PROJ) {
    Rp = (a.R + 15) / 16 * 16;
    if (a.R < 1 || Rp > proj_max_rank<T, NM>()) return MAMBA_ERR_UNSUPPORTED;
    smem = proj_bwd_smem_bytes<T, NM>(Rp);
  }
  const bool dmap = PROJ ? make_map_3d(&maps[1], a.dt_low, bf16, L, uint64_t(a.R), batch, kBTT,
                                       uint32_t(Rp), sw)
                         : make_map_3d(&maps[1], a.delta, bf16, L, dim, batch, kBTT, kSThreads, sw);
  if (!make_map_3d(&maps[0], a.u, bf16, L, dim, batch, kBTT, kSThreads, sw) || !dmap ||
      !make_map_3d(&maps[2], a.z ? a.z : a.u, bf16, L, dim, batch, kBTT, kSThreads, sw) ||
      !make_map_3d(&maps[3], a.dy, bf16, L, dim, batch, kBTT, kSThreads, sw) ||
      !make_map_3d(&maps[4], a.B, bf16, L, N, batch, kBTT, uint32_t(N), none) ||
      !make_map_3d(&maps[5], a.C, bf16, L, N, batch, kBTT, uint32_t(N), none)) {
    return MAMBA_ERR_UNSUPPORTED;
  }
  auto kern = bwd_staged_kernel<T, NM, CONV, PROJ>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return MAMBA_ERR_CUDA;
  int bps = 0;
  if (resident_ctas(kern, smem, PROJ ? int(kProjTmemCols) : Lay::TMEM_COLS, &bps) != cudaSuccess)
    return MAMBA_ERR_CUDA;
  const int sms = device_sm_count();
  const int slots = sms * std::max(1, bps);
  const int64_t gpb = ceil_div(a.dim, kSThreads);
  const int64_t G = int64_t(a.batch) * gpb;
  if (G > (int64_t(1) << 30)) return MAMBA_ERR_UNSUPPORTED;
  // The adjoint crosses chunks by the sequential hand-off when the channel
  // groups fill the GPU, else by the three-phase carry (whose aggregate pass is
  // cheap here -- no states -- so it takes shorter chunks than the forward's).
  StagedPlan pl = plan_staged(G, a.L, slots, o, 256);
  const bool par = pl.kind == KIND_PAR;
  if (G * pl.K > (int64_t(1) << 30)) return MAMBA_ERR_UNSUPPORTED;
  // (the fused projection's three-phase adjoint carry reads delta from the
  // checkpoint pass, which saved states replace: not taken from saved states)
  if (PROJ && saved && par) return MAMBA_ERR_UNSUPPORTED;
  const int64_t n16 = ceil_div(a.L, kBTT);

  // workspace: [ints][ckpt][carry][part_bc][part_A][part_D][part_bias]
  //            (three-phase: + [agg_S][agg_G][gin])
  const size_t int_bytes = ceil_div((1 + size_t(G)) * 4, 256) * 256;
  const size_t n_ckpt = size_t(G) * size_t(n16) * NM * kSThreads;
  const size_t n_ckpt_ws = saved ? 0 : n_ckpt;  // checkpoints in the workspace
  const size_t n_carry = size_t(G) * NM * kSThreads;
  const size_t n_bc = size_t(gpb) * size_t(a.batch) * 32 * size_t(a.L);
  const size_t gk = size_t(G) * size_t(pl.K);
  const size_t n_A = gk * NM * kSThreads, n_D = gk * kSThreads;
  const size_t n_par = par ? gk * NM * kSThreads : 0;  // agg_G and gin each
  // the fused projection's three-phase carry: delta in fp32 for the aggregate pass
  const size_t n_delta = (PROJ && par) ? size_t(a.batch) * size_t(a.dim) * size_t(a.L) : 0;
  const size_t bytes_f = ceil_div(int_bytes + 4 * (n_ckpt_ws + n_carry + n_bc + n_A + 2 * n_D + n_delta) +
                                      (par ? 8 * n_D + 8 * n_par : 0), 256) * 256;
  // the range flags of delta, written by the checkpoint pass (not with the
  // fused projection, which checks per tile, nor with the generic arithmetic
  // forced)
  const bool range = !PROJ && o.path != MAMBA_PATH_GENERIC;
  const size_t n_flags = range ? size_t(G) * size_t(ceil_div(a.L, kRangeBlock)) : 0;
  const size_t bytes = bytes_f + (saved ? 0 : ceil_div(n_flags, 256) * 256);
  // The checkpoint pass (the forward without y) is prepared first so that one
  // workspace holds both: a failed allocation then leaves nothing enqueued.
  FwdArgs fa;
  fa.u = a.u; fa.delta = a.delta; fa.z = nullptr; fa.B = a.B; fa.C = a.C;
  fa.bias = a.bias; fa.A = a.A; fa.D = nullptr; fa.y = nullptr; fa.last_state = nullptr;
  fa.batch = a.batch; fa.dim = a.dim; fa.L = a.L; fa.N = a.N;
  fa.conv_w = a.conv_w; fa.conv_b = a.conv_b; fa.conv_width = a.conv_width;
  fa.dt_low = a.dt_low; fa.W_dt = a.W_dt; fa.R = a.R;
  StagedOptions fo = o;
  fo.chunk_len = 0;
  fo.carry = 0;
  fo.test_hook = 0;  // the hook targets the reverse hand-off
  StagedForward<T, NM, CONV, PROJ> ckpt_pass;
  unsigned char *ws = nullptr;
  if (!saved) {
    // the checkpoint buffer is set once the workspace exists (before run)
    const mamba_status_t pst = ckpt_pass.prepare(fa, fo, nullptr, true);
    if (pst != MAMBA_OK) return pst;
  }
  if (ws_alloc(reinterpret_cast<void **>(&ws), bytes + (saved ? 0 : ckpt_pass.bytes), s) != cudaSuccess) {
    cudaGetLastError();
    return MAMBA_ERR_OUT_OF_MEMORY;
  }
  BwdStagedArgs bp;
  bp.w = a;
  bp.G = int(G);
  bp.gpb = int(gpb);
  bp.K = pl.K;
  bp.chunk_len = pl.chunk_len;
  bp.n_units = int(gk);
  bp.counter = reinterpret_cast<int *>(ws);
  bp.flags = bp.counter + 1;
  float *fws = reinterpret_cast<float *>(ws + int_bytes);
  float *ckpt = fws;
  bp.ckpt = saved ? reinterpret_cast<const float *>(saved + sl.ckpt) : ckpt;
  bp.carry = ckpt + n_ckpt_ws;
  bp.part_bc = bp.carry + n_carry;
  bp.part_A = bp.part_bc + n_bc;
  bp.part_D = bp.part_A + n_A;
  bp.part_bias = bp.part_D + n_D;
  bp.gin = nullptr;
  bp.agg_G = nullptr;
  bp.agg_S = nullptr;
  float *delta_f32 = nullptr;
  if (par) {
    bp.agg_S = reinterpret_cast<double *>(bp.part_bias + n_D);  // 8-byte aligned: offsets are
    bp.agg_G = reinterpret_cast<float *>(bp.agg_S + n_D);       // multiples of 128 floats
    bp.gin = bp.agg_G + n_par;
    if (n_delta) delta_f32 = bp.gin + n_par;  // 16-byte aligned (multiples of 128 floats)
  }
  bp.Rp = Rp;
  bp.stage_bytes = PROJ ? BwdStage<T, NM>(Rp).bytes : 0;
  bp.n_ckpt = int64_t(n_ckpt);
  bp.n_carry = int64_t(n_carry);
  bp.n_bc = int64_t(n_bc);
  bp.n_unit = int64_t(n_D);
  bp.n_gin = int64_t(n_par);
  bp.range_flags = !range ? nullptr : saved ? saved + sl.flags : ws + bytes_f;
  bp.n_flags = int64_t(n_flags);
  bp.timeout_ns = o.timeout_us > 0 ? uint64_t(o.timeout_us) * 1000ull : kDefaultTimeoutNs;
  bp.force_generic = o.path == MAMBA_PATH_GENERIC ? 1 : 0;
  bp.test_hook = o.test_hook;

  mamba_status_t st = MAMBA_OK;
  if (cudaMemsetAsync(ws, 0, int_bytes, s) != cudaSuccess) st = MAMBA_ERR_CUDA;
  if (saved && sl.n_hin > 0) {  // the forward's chunks ran from zero
    bp.ckpt_hin = reinterpret_cast<const float *>(saved + sl.hin);
    bp.ckpt_cum = reinterpret_cast<const float *>(saved + sl.cum);
    bp.ckpt_chunk = sl.pl.chunk_len;
    bp.ckpt_K = sl.pl.K;
    bp.n_ckpt_hin = sl.n_hin;
    bp.n_ckpt_cum = sl.n_cum;
  }
  if (st == MAMBA_OK && !saved) {
    ckpt_pass.sa.ckpt = ckpt;
    ckpt_pass.sa.delta_out = delta_f32;
    ckpt_pass.sa.range_flags = range ? ws + bytes_f : nullptr;
    ckpt_pass.sa.n_flags = int64_t(n_flags);
    st = ckpt_pass.run(ws + bytes, s, launched);
    if (ckpt_pass.sa.ckpt_cum) {  // checkpoints from zero chunk starts: corrected as they are read
      bp.ckpt_hin = ckpt_pass.sa.hin;
      bp.ckpt_cum = ckpt_pass.sa.ckpt_cum;
      bp.ckpt_chunk = ckpt_pass.pl.chunk_len;
      bp.ckpt_K = ckpt_pass.pl.K;
      bp.n_ckpt_hin = ckpt_pass.sa.n_agg;
      bp.n_ckpt_cum = ckpt_pass.sa.n_ckpt_cum;
    }
  }
  if (st == MAMBA_OK && par) {
    if (delta_f32) {  // the aggregate pass reads the fp32 delta the checkpoint pass formed
      BwdStagedArgs bq = bp;
      bq.w.delta = delta_f32;
      bwd_adjoint_agg_kernel<T, NM, float><<<unsigned(size_t(G) * size_t(pl.K - 1)), kSThreads, 0, s>>>(bq);
    } else {
      bwd_adjoint_agg_kernel<T, NM, T><<<unsigned(size_t(G) * size_t(pl.K - 1)), kSThreads, 0, s>>>(bp);
    }
    st = launched();
    if (st == MAMBA_OK) {  // Ga_in(K-1) = 0, Ga_in(k-1) = exp(A_n S_k) Ga_in(k) + Ga_local(k)
      ChunkScanIO io;
      io.S = bp.agg_S;
      io.hl = bp.agg_G;
      io.hin = bp.gin;
      io.A = a.A;
      io.G = int(G);
      io.K = pl.K;
      io.gpb = int(gpb);
      io.N = a.N;
      io.dim = a.dim;
      const int64_t nseq = G * NM * kSThreads;
      chunk_scan_kernel<NM, true><<<unsigned(chunk_scan_grid(nseq, pl.K)), 128, 0, s>>>(io);
      st = launched();
    }
  }
  if (st == MAMBA_OK) {
    kern<<<unsigned(std::min<int64_t>(gk, slots)), kSThreads, smem, s>>>(
        maps[0], maps[1], maps[2], maps[3], maps[4], maps[5], bp);
    st = launched();
  }
  if (st == MAMBA_OK) {
    const int64_t nbc = a.batch * a.N * (a.L / 4);
    bwd_staged_finalize_bc<T><<<unsigned(std::min<int64_t>(ceil_div(nbc, 256), sms * 8)), 256, 0, s>>>(bp);
    st = launched();
  }
  if (st == MAMBA_OK) {
    const int64_t np = a.dim * a.N;
    bwd_staged_finalize_params<NM><<<unsigned(std::min<int64_t>(ceil_div(np, 256), sms * 8)), 256, 0, s>>>(bp);
    st = launched();
  }
  if (ws_free(ws, s) != cudaSuccess && st == MAMBA_OK) st = MAMBA_ERR_CUDA;
  return st;
}

}  // namespace mscan
