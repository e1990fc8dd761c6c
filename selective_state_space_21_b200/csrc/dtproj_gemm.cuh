// dtproj_gemm.cuh -- the two gradient products of the low-rank Delta
// projection ("Mamba: Linear-Time Sequence Modeling with Selective State
// Spaces", paper-graph-ui summary, section 3.6, s_Delta = Linear_D(Linear_R))
// for bf16 I/O, as tcgen05 GEMMs with fp32 accumulators in tensor memory:
//     d_dt_low[b,r,t] = sum_d W[d,r] ddelta[b,d,t]            (per batch row)
//     dW[d,r]         = sum_b sum_t ddelta[b,d,t] dt_low[b,r,t]
// One kernel computes D (M x N, fp32, TMEM) = sum_k A[m,k] B[n,k] over its
// k tiles:
//  * a producer thread streams 64-deep k tiles of A (128 rows) and B (BN
//    rows) by TMA with 128-byte swizzling into a 4-stage mbarrier ring;
//  * one thread issues four 128 x BN x 16 MMAs per stage and releases the
//    stage with tcgen05.commit;
//  * the 128 threads read the accumulator back (each its own row) and store
//    it.
// GRAD_INPUT: M = 128 steps t of one batch row, N = Rp (rank, padded to 64),
// K = the channels d; both operands are MN-major (t and r contiguous).
// Output transposed into d_dt_low (bf16).
// GRAD_WEIGHT: M = 128 channels d, N = Rp, K = (batch row, step) pairs split
// over the grid's y dimension; both operands K-major (t contiguous).  Each
// split writes fp32 partial sums that a finalize kernel adds in a fixed order.
#pragma once

#include "common.cuh"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace mscan {

// TMA ring stages: four for d_dt_low (its B tile is up to 256 rows of dt_low);
// three for dW, so that two CTAs share an SM (108 KB each at R = 160).
template <bool GRAD_INPUT>
__host__ __device__ constexpr int proj_gemm_stages() {
  return GRAD_INPUT ? 4 : 3;
}
constexpr int kGBK = 64;  // k per stage (128 bytes of bf16)
constexpr uint32_t kGTileA = 128 * kGBK * 2;  // 16 KB

struct ProjGemmArgs {
  int64_t batch, dim, L;
  int R, Rp;            // rank, rank padded (GRAD_INPUT: to 64; GRAD_WEIGHT: to 16)
  int k_tiles;          // k tiles of the whole contraction
  int k_per_split;      // GRAD_WEIGHT: k tiles per split
  void *out;            // GRAD_INPUT: d_dt_low (bf16); GRAD_WEIGHT: partials [split][dim][R] fp32
  uint64_t timeout_ns;
};

template <bool GRAD_INPUT>
__host__ __device__ constexpr uint32_t proj_gemm_btile(int Rp) {
  return uint32_t(Rp) * kGBK * 2;
}

template <bool GRAD_INPUT>
__global__ void __launch_bounds__(128, 1)
    proj_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const ProjGemmArgs p) {
  constexpr int kGStages = proj_gemm_stages<GRAD_INPUT>();
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t btile = proj_gemm_btile<GRAD_INPUT>(p.Rp);
  const uint32_t stage_bytes = kGTileA + btile;
  uint64_t *full = reinterpret_cast<uint64_t *>(sm + kGStages * stage_bytes);
  uint64_t *empty = full + kGStages;
  uint64_t *done = empty + kGStages;
  uint32_t *tslot = reinterpret_cast<uint32_t *>(done + 1);
  int *abort_flag = reinterpret_cast<int *>(tslot + 1);
  int *issued = abort_flag + 1;  // loads the producer issued
  const int tid = threadIdx.x, warp = tid >> 5;

  // this CTA's tile and k range
  int64_t m0, b = 0;
  int k0, k1;
  if constexpr (GRAD_INPUT) {
    m0 = int64_t(blockIdx.x) * 128;  // steps
    b = blockIdx.y;
    k0 = 0;
    k1 = p.k_tiles;
  } else {
    m0 = int64_t(blockIdx.x) * 128;  // channels
    k0 = blockIdx.y * p.k_per_split;
    k1 = min(p.k_tiles, k0 + p.k_per_split);
  }
  const int nk = k1 - k0;

  if (tid == 0) {
    for (int s = 0; s < kGStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    fence_barrier_init();
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    *abort_flag = 0;
    *issued = 0;
  }
  if (warp == 0) {
    tmem_alloc(tslot, 256);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tacc = *tslot;

  // Loads k tile `kt` (global index) into stage s.
  auto load = [&](int kt, int s) {
    unsigned char *a = sm + s * stage_bytes;
    unsigned char *bt = a + kGTileA;
    mbar_arrive_expect_tx(&full[s], stage_bytes);
    if constexpr (GRAD_INPUT) {
      const int d0 = kt * kGBK;
      // A: ddelta rows d0.. (k) x 128 steps (m), two 64-step boxes
      tma_load_3d(a, &tmA, &full[s], int(m0), d0, int(b));
      tma_load_3d(a + kGTileA / 2, &tmA, &full[s], int(m0) + 64, d0, int(b));
      // B: W rows d0.. (k) x Rp ranks (n), 64-rank boxes
      for (int j = 0; j < p.Rp / 64; ++j) tma_load_3d(bt + j * (kGBK * 128), &tmB, &full[s], 64 * j, d0, 0);
    } else {
      const int tiles_per_row = int((p.L + kGBK - 1) / kGBK);
      const int bb = kt / tiles_per_row, t0 = (kt % tiles_per_row) * kGBK;
      tma_load_3d(a, &tmA, &full[s], t0, int(m0), bb);   // ddelta: 128 channels x 64 steps
      tma_load_3d(bt, &tmB, &full[s], t0, 0, bb);        // dt_low: Rp ranks x 64 steps
    }
  };

  const uint32_t idesc = mma_idesc_bf16(128, p.Rp, GRAD_INPUT, GRAD_INPUT);

  if (tid == 0) {  // producer
    for (int i = 0; i < nk; ++i) {
      const int s = i % kGStages;
      if (i >= kGStages &&
          !mbar_wait_bounded(&empty[s], uint32_t((i / kGStages) - 1) & 1u, p.timeout_ns)) {
        record_timeout();
        *abort_flag = 1;
        break;
      }
      load(k0 + i, s);
      *issued = i + 1;
    }
  } else if (tid == 32) {  // MMA issuer
    for (int i = 0; i < nk; ++i) {
      const int s = i % kGStages;
      if (!mbar_wait_bounded(&full[s], uint32_t(i / kGStages) & 1u, p.timeout_ns)) {
        record_timeout();
        *abort_flag = 1;
        break;
      }
      tc_fence_after_sync();
      const uint32_t a = smem_u32(sm + s * stage_bytes);
      const uint32_t bt = a + kGTileA;
      for (int kk = 0; kk < kGBK / 16; ++kk) {
        uint64_t ad, bd;
        if constexpr (GRAD_INPUT) {  // MN-major: 16 k rows = two 1 KB atoms; 64-wide MN blocks 8 KB apart
          ad = smem_desc(a + uint32_t(kk) * 2048u, 8192u, 1024u, 2u);
          bd = smem_desc(bt + uint32_t(kk) * 2048u, 8192u, 1024u, 2u);
        } else {  // K-major: 16 k = 32 bytes along the 128-byte row; 8-row atoms 1 KB apart
          ad = smem_desc(a + uint32_t(kk) * 32u, 16u, 1024u, 2u);
          bd = smem_desc(bt + uint32_t(kk) * 32u, 16u, 1024u, 2u);
        }
        mma_ss(tacc, ad, bd, idesc, (i > 0) || (kk > 0));
      }
      mma_commit(&empty[s]);  // the stage is free once these MMAs have read it
    }
    mma_commit(done);
  }
  __syncwarp();
  // epilogue: wait for the last MMA, then each thread reads its row
  if (!mbar_wait_bounded(done, 0u, p.timeout_ns)) {
    record_timeout();
    *abort_flag = 1;
  }
  tc_fence_after_sync();
  const int row = tid;  // accumulator lane = M row
  if (nk > 0 && !*abort_flag) {
    for (int c0 = 0; c0 < p.Rp; c0 += 8) {
      float v[8];
      tmem_ld8(tmem_at(tacc, uint32_t(warp) * 32u, uint32_t(c0)), v);
      tmem_ld_wait();
      if constexpr (GRAD_INPUT) {
        const int64_t t = m0 + row;
        if (t < p.L) {
          __nv_bfloat16 *o = static_cast<__nv_bfloat16 *>(p.out) + (b * p.R) * p.L + t;
#pragma unroll
          for (int i = 0; i < 8; ++i)
            if (c0 + i < p.R) o[int64_t(c0 + i) * p.L] = __float2bfloat16_rn(v[i]);
        }
      } else {
        const int64_t d = m0 + row;
        if (d < p.dim) {
          float *o = static_cast<float *>(p.out) + (int64_t(blockIdx.y) * p.dim + d) * p.R;
#pragma unroll
          for (int i = 0; i < 8; ++i)
            if (c0 + i < p.R) o[c0 + i] = v[i];
        }
      }
    }
  }
  // drain after an expired wait: every load issued must land before the CTA
  // exits (at most the last kGStages can still be in flight)
  if (tid == 0 && *abort_flag) {
    const int n = *issued;
    for (int i = n > kGStages ? n - kGStages : 0; i < n; ++i)
      mbar_wait_bounded(&full[i % kGStages], uint32_t(i / kGStages) & 1u, p.timeout_ns);
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tacc, 256);
  }
}

// dW = sum over the splits of the partials, in split order.
__global__ void proj_grad_weight_finalize(const float *part, float *dW, int64_t n, int splits) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
    float s = 0.f;
    for (int j = 0; j < splits; ++j) s += part[int64_t(j) * n + i];
    dW[i] = s;
  }
}

template <bool GRAD_INPUT>
inline int proj_gemm_smem(int Rp) {
  constexpr int kGStages = proj_gemm_stages<GRAD_INPUT>();
  return int(kGStages * (kGTileA + proj_gemm_btile<GRAD_INPUT>(Rp))) + 8 * (2 * kGStages + 1) + 16 +
         1024;
}

}  // namespace mscan
