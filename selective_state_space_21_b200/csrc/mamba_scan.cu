// mamba_scan.cu -- the C ABI of libmambascan: argument validation, workspace,
// kernel selection and launch.  The operation is documented in
// include/mamba_scan.h.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>

#include "../../include/mamba_scan.h"
#include "bwd_reference.cuh"
#include "bwd_staged.cuh"
#include "common.cuh"
#include "conv_bwd.cuh"
#include "cplx.cuh"
#include "dtproj.cuh"
#include "dtproj_gemm.cuh"
#include "decode.cuh"
#include "fwd_reference.cuh"
#include "fwd_staged.cuh"

namespace mscan {

EncodeTiledFn get_encode_tiled() {
  static const EncodeTiledFn fn = []() -> EncodeTiledFn {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    return reinterpret_cast<EncodeTiledFn>(ptr);
  }();
  return fn;
}

}  // namespace mscan

using namespace mscan;

namespace {

constexpr int kAbiVersion = 1;

std::atomic<uint64_t> g_launches{0};

struct Range {
  uintptr_t lo, hi;
};

size_t dtype_size(mamba_dtype_t dt) { return dt == MAMBA_BF16 ? 2 : 4; }

// A pointer the kernels may dereference: device (or managed) memory visible
// from the current device.
bool is_device_ptr(const void *p, int dev) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  if (at.type == cudaMemoryTypeManaged) return true;
  return at.type == cudaMemoryTypeDevice && at.device == dev;
}

struct Checker {
  int dev = 0;
  mamba_status_t st = MAMBA_OK;
  Range ranges[24];
  bool is_out[24];
  int n = 0;

  // Records a buffer of `bytes` bytes; `required` buffers may not be NULL.
  void buf(const void *p, size_t bytes, size_t align, bool required, bool output) {
    if (st != MAMBA_OK) return;
    if (!p) {
      if (required && bytes > 0) st = MAMBA_ERR_INVALID_ARG;
      return;
    }
    if (bytes == 0) return;
    if (reinterpret_cast<uintptr_t>(p) % align != 0 || !is_device_ptr(p, dev)) {
      st = MAMBA_ERR_INVALID_ARG;
      return;
    }
    const uintptr_t lo = reinterpret_cast<uintptr_t>(p);
    for (int i = 0; i < n; ++i) {
      const bool overlap = lo < ranges[i].hi && ranges[i].lo < lo + bytes;
      if (overlap && (output || is_out[i])) {
        st = MAMBA_ERR_INVALID_ARG;
        return;
      }
    }
    ranges[n] = {lo, lo + bytes};
    is_out[n] = output;
    ++n;
  }
};

mamba_status_t check_shape(int64_t batch, int64_t dim, int64_t L, int64_t N, mamba_dtype_t dt) {
  if (dt != MAMBA_F32 && dt != MAMBA_BF16) return MAMBA_ERR_INVALID_ARG;
  if (batch < 0 || dim < 0 || L < 0) return MAMBA_ERR_INVALID_ARG;
  if (N < 1 || N > kMaxN) return MAMBA_ERR_UNSUPPORTED;
  // Keep every flattened index inside int64 with room to spare, and the batch
  // inside a grid dimension.
  if (batch > 65535 || dim > (int64_t(1) << 31) || L > (int64_t(1) << 40)) return MAMBA_ERR_UNSUPPORTED;
  const double elems = double(batch) * double(dim) * double(L);
  if (elems > 9.0e15) return MAMBA_ERR_UNSUPPORTED;
  return MAMBA_OK;
}

mamba_status_t check_options(const mamba_scan_options_t *o) {
  if (!o) return MAMBA_OK;
  if (o->path < MAMBA_PATH_AUTO || o->path > MAMBA_PATH_STRUCTURED) return MAMBA_ERR_INVALID_ARG;
  if (o->chunk_len < 0 || (o->chunk_len > 0 && o->chunk_len % 64 != 0)) return MAMBA_ERR_INVALID_ARG;
  if (o->carry < 0 || o->carry > 2 || o->wait_timeout_us < 0 || o->test_hook < 0 || o->test_hook > 1)
    return MAMBA_ERR_INVALID_ARG;
  for (int i = 0; i < 3; ++i)
    if (o->reserved[i] != 0) return MAMBA_ERR_INVALID_ARG;
  return MAMBA_OK;
}

mamba_status_t cuda_status() {
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) return MAMBA_OK;
  return e == cudaErrorMemoryAllocation ? MAMBA_ERR_OUT_OF_MEMORY : MAMBA_ERR_CUDA;
}

// Status of the kernel launch just made (counted for mamba_scan_launch_count).
mamba_status_t launch_status() {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cuda_status();
}

// Dispatch on N (rounded up to 1, 2, 4, 8 or 16; the padding states carry
// B = C = 0 and so stay 0) and on the I/O type.
template <template <typename, int> class Launcher, typename... Args>
mamba_status_t dispatch(mamba_dtype_t dt, int N, Args &&...args) {
#define MSCAN_CASE(NMV)                                                            \
  if (N <= NMV) {                                                                  \
    return dt == MAMBA_BF16 ? Launcher<__nv_bfloat16, NMV>::run(args...)          \
                            : Launcher<float, NMV>::run(args...);                  \
  }
  MSCAN_CASE(1)
  MSCAN_CASE(2)
  MSCAN_CASE(4)
  MSCAN_CASE(8)
  MSCAN_CASE(16)
#undef MSCAN_CASE
  return MAMBA_ERR_UNSUPPORTED;
}

template <typename T, int NM>
struct FwdReferenceLauncher {
  static mamba_status_t run(const FwdArgs &a, cudaStream_t s) {
    const int64_t ch = a.batch * a.dim;
    const int64_t grid = (ch + kRefThreads - 1) / kRefThreads;
    fwd_reference_kernel<T, NM><<<(unsigned)grid, kRefThreads, 0, s>>>(a);
    return launch_status();
  }
};

template <typename T, bool CONV>
mamba_status_t staged_bwd_dispatch(const BwdArgs &a, const StagedOptions &o, cudaStream_t s,
                                   const unsigned char *saved = nullptr) {
  if (a.N <= 4) return staged_backward<T, 4, CONV>(a, o, s, &launch_status, saved);
  if (a.N <= 8) return staged_backward<T, 8, CONV>(a, o, s, &launch_status, saved);
  return staged_backward<T, 16, CONV>(a, o, s, &launch_status, saved);
}

template <typename T, bool CONV>
mamba_status_t staged_dispatch(const FwdArgs &a, const StagedOptions &o, cudaStream_t s,
                               unsigned char *save = nullptr) {
  if (a.N <= 4) return staged_forward<T, 4, CONV>(a, o, s, &launch_status, nullptr, save);
  if (a.N <= 8) return staged_forward<T, 8, CONV>(a, o, s, &launch_status, nullptr, save);
  return staged_forward<T, 16, CONV>(a, o, s, &launch_status, nullptr, save);
}

// Bytes a saving forward stores for its backward: 0 where the problem takes
// the one-thread-per-channel kernels (then the saving calls are the plain
// ones), else the layout of saved_layout on the current device.
template <typename T, bool CONV>
mamba_status_t saved_bytes_t(int64_t batch, int64_t dim, int64_t L, int64_t N, const StagedOptions &so,
                             uint64_t *bytes) {
  SavedLayout sl;
  mamba_status_t st;
  if (N <= 4) st = saved_layout<T, 4, CONV>(batch, dim, L, so, &sl);
  else if (N <= 8) st = saved_layout<T, 8, CONV>(batch, dim, L, so, &sl);
  else st = saved_layout<T, 16, CONV>(batch, dim, L, so, &sl);
  *bytes = st == MAMBA_OK ? uint64_t(sl.bytes) : 0;
  return st;
}

// (conv: the forward with the convolution prologue, whose kernels the chunking
// is planned for)
mamba_status_t saved_bytes_for(int64_t batch, int64_t dim, int64_t L, int64_t N, mamba_dtype_t dtype,
                               const StagedOptions &so, uint64_t *bytes, bool conv = false) {
  *bytes = 0;
  if (batch == 0 || dim == 0 || L == 0 || so.path == MAMBA_PATH_REFERENCE ||
      !staged_shape_ok(L, dim, N, dtype_size(dtype)))
    return MAMBA_OK;
  if (conv)
    return dtype == MAMBA_BF16 ? saved_bytes_t<__nv_bfloat16, true>(batch, dim, L, N, so, bytes)
                               : saved_bytes_t<float, true>(batch, dim, L, N, so, bytes);
  return dtype == MAMBA_BF16 ? saved_bytes_t<__nv_bfloat16, false>(batch, dim, L, N, so, bytes)
                             : saved_bytes_t<float, false>(batch, dim, L, N, so, bytes);
}

template <typename T, int NM>
struct BwdReferenceLauncher {
  static mamba_status_t run(const BwdArgs &a, cudaStream_t s) {
    BwdWork w;
    w.n_chunks = (a.L + kBwdTC - 1) / kBwdTC;
    w.n_dblk = (a.dim + kBwdThreads - 1) / kBwdThreads;
    const size_t bd = size_t(a.batch * a.dim);
    const size_t n_ckpt = bd * size_t(w.n_chunks) * NM;
    const size_t n_bc = size_t(w.n_dblk) * size_t(a.batch) * kBwdSlots * size_t(a.L);
    const size_t n_A = bd * size_t(a.N);
    const size_t total = n_ckpt + n_bc + n_A + 2 * bd;
    float *ws = nullptr;
    if (ws_alloc(reinterpret_cast<void **>(&ws), total * sizeof(float), s) != cudaSuccess) {
      cudaGetLastError();
      return MAMBA_ERR_OUT_OF_MEMORY;
    }
    w.ckpt = ws;
    w.part_bc = w.ckpt + n_ckpt;
    w.part_A = w.part_bc + n_bc;
    w.part_D = w.part_A + n_A;
    w.part_bias = w.part_D + bd;
    const size_t smem = sizeof(float) * (kBwdTC * NM * kBwdThreads + 2 * kBwdSlots * kBwdTC);
    mamba_status_t st = MAMBA_OK;
    if (cudaFuncSetAttribute(bwd_reference_kernel<T, NM>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) {
      st = MAMBA_ERR_CUDA;
    }
    if (st == MAMBA_OK) {
      dim3 grid((unsigned)w.n_dblk, (unsigned)a.batch);
      bwd_reference_kernel<T, NM><<<grid, kBwdThreads, smem, s>>>(a, w);
      st = launch_status();
    }
    if (st == MAMBA_OK) {
      const int64_t nbc = a.batch * a.N * a.L;
      const int64_t g = std::min<int64_t>((nbc + 255) / 256, 148 * 16);
      bwd_finalize_bc_kernel<T><<<(unsigned)g, 256, 0, s>>>(a, w);
      st = launch_status();
    }
    if (st == MAMBA_OK) {
      const int64_t np = a.dim * a.N;
      const int64_t g = std::min<int64_t>((np + 255) / 256, 148 * 16);
      bwd_finalize_params_kernel<<<(unsigned)g, 256, 0, s>>>(a, w);
      st = launch_status();
    }
    if (ws_free(ws, s) != cudaSuccess && st == MAMBA_OK) st = MAMBA_ERR_CUDA;
    return st;
  }
};

template <typename T, int NM>
struct CplxFwdLauncher {
  // four threads per channel for 16 states, two for 8
  static constexpr int TPC = NM >= 16 ? 4 : (NM >= 8 ? 2 : 1);
  static mamba_status_t run(const CplxArgs &a, cudaStream_t s) {
    constexpr int per_block = kCplxThreads / TPC;
    const dim3 grid(unsigned((a.dim + per_block - 1) / per_block), unsigned(a.batch));
    cplx_fwd_kernel<T, NM, TPC><<<grid, kCplxThreads, 0, s>>>(a);
    return launch_status();
  }
};

template <typename T, int NM>
struct CplxBwdLauncher {
  // four threads per channel for 16 states, two for 8; one state per thread
  // when the channels fill at most half of the GPU's CTA slots
  static constexpr int TPC = NM >= 16 ? 4 : (NM >= 8 ? 2 : 1);
  static constexpr int TPC_SMALL = NM;

  template <int P>
  static mamba_status_t launch(const CplxArgs &a, cudaStream_t s) {
    constexpr int per_block = kCplxBwdThreads / P;
    constexpr size_t smem = cplx_bwd_smem<NM, P>();
    auto kf = cplx_bwd_kernel<T, NM, P, false>;
    auto kr = cplx_bwd_kernel<T, NM, P, true>;
    int occ = 0;
    if (cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess ||
        cudaFuncSetAttribute(kr, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kr, kCplxBwdThreads, smem) != cudaSuccess) {
      cudaGetLastError();
      return MAMBA_ERR_CUDA;
    }
    const int64_t slots = int64_t(device_sm_count()) * std::max(occ, 1);
    CplxWork w;
    w.n_blocks = (a.L + kCplxBwdTC - 1) / kCplxBwdTC;
    w.n_dblk = (a.dim + per_block - 1) / per_block;
    const int64_t n_cb = w.n_dblk * a.batch;
    // More channel blocks than CTA slots: four chunks per sequence, so that
    // the last round of units is a quarter of a sequence long.  Otherwise one
    // (the units all run at once, and chunks would only wait on each other).
    const int64_t K0 = n_cb > slots ? 4 : 1;
    w.bpc = (w.n_blocks + K0 - 1) / K0;
    w.K = int((w.n_blocks + w.bpc - 1) / w.bpc);
    if (n_cb * w.K > (int64_t(1) << 30)) return MAMBA_ERR_UNSUPPORTED;
    w.timeout_ns = kDefaultTimeoutNs;
    const size_t bd = size_t(a.batch * a.dim);
    const bool saved = a.saved_ckpt != nullptr;  // block checkpoints from the saving forward
    const size_t n_ckpt = saved ? 0 : bd * size_t(w.n_blocks) * 2 * NM;
    const size_t n_bc = size_t(w.n_dblk) * size_t(a.batch) * 4 * kMaxN * size_t(a.L);
    const size_t n_A = size_t(w.K) * bd * 2 * size_t(a.N);
    const size_t n_par = size_t(w.K) * bd;
    const size_t n_carry = size_t(n_cb) * kCplxBwdThreads * 4 * (NM / P);
    const size_t int_bytes = (size_t(2 + n_cb) * 4 + 255) / 256 * 256;
    unsigned char *ws = nullptr;
    if (ws_alloc(reinterpret_cast<void **>(&ws),
                 int_bytes + (n_ckpt + n_bc + n_A + 2 * n_par + n_carry) * 4, s) != cudaSuccess) {
      cudaGetLastError();
      return MAMBA_ERR_OUT_OF_MEMORY;
    }
    w.counter = reinterpret_cast<int *>(ws);
    w.flags = w.counter + 2;
    w.flag_base = saved ? 0 : w.K;
    w.ckpt = saved ? const_cast<float *>(a.saved_ckpt) : reinterpret_cast<float *>(ws + int_bytes);
    w.part_bc = reinterpret_cast<float *>(ws + int_bytes) + n_ckpt;
    w.part_A = w.part_bc + n_bc;
    w.part_D = w.part_A + n_A;
    w.part_bias = w.part_D + n_par;
    w.carry = w.part_bias + n_par;
    mamba_status_t st = MAMBA_OK;
    if (cudaMemsetAsync(ws, 0, int_bytes, s) != cudaSuccess) st = MAMBA_ERR_CUDA;
    const unsigned grid = unsigned(std::min<int64_t>(n_cb * w.K, slots));
    if (st == MAMBA_OK && !saved) {  // the forward sweep (block-start states), then the reverse sweep
      kf<<<grid, kCplxBwdThreads, smem, s>>>(a, w);
      st = launch_status();
    }
    if (st == MAMBA_OK) {
      kr<<<grid, kCplxBwdThreads, smem, s>>>(a, w);
      st = launch_status();
    }
    if (st == MAMBA_OK) {
      const int64_t nbc = a.batch * 2 * a.N * a.L;
      cplx_finalize_bc<T><<<unsigned(std::min<int64_t>((nbc + 255) / 256, 148 * 16)), 256, 0, s>>>(a, w);
      st = launch_status();
    }
    if (st == MAMBA_OK) {
      const int64_t np = a.dim * 2 * a.N;
      cplx_finalize_params<<<unsigned(std::min<int64_t>((np + 255) / 256, 148 * 16)), 256, 0, s>>>(a, w);
      st = launch_status();
    }
    if (ws_free(ws, s) != cudaSuccess && st == MAMBA_OK) st = MAMBA_ERR_CUDA;
    return st;
  }

  static mamba_status_t run(const CplxArgs &a, cudaStream_t s) {
    // When the channel blocks fill at most half of one round of CTA slots,
    // every CTA is latency-bound, and one state per thread (more threads per
    // channel, shorter per-step chains) finishes sooner: 3.66 against 4.02 ms
    // at batch 1 x 5120 channels, L 2048.
    constexpr size_t smem = cplx_bwd_smem<NM, TPC>();
    if (cudaFuncSetAttribute(cplx_bwd_kernel<T, NM, TPC, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(smem)) != cudaSuccess) {
      cudaGetLastError();
      return MAMBA_ERR_CUDA;
    }
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, cplx_bwd_kernel<T, NM, TPC, true>,
                                                      kCplxBwdThreads, smem) != cudaSuccess) {
      cudaGetLastError();
      return MAMBA_ERR_CUDA;
    }
    constexpr int per_block = kCplxBwdThreads / TPC;
    const int64_t units = (a.dim + per_block - 1) / per_block * a.batch;
    const int64_t slots = int64_t(device_sm_count()) * std::max(occ, 1);
    if (TPC_SMALL > TPC && 2 * units <= slots) return launch<TPC_SMALL>(a, s);
    return launch<TPC>(a, s);
  }
};

StagedOptions staged_options(const mamba_scan_options_t *options) {
  StagedOptions so;
  so.path = options ? options->path : MAMBA_PATH_AUTO;
  so.chunk_len = options ? options->chunk_len : 0;
  so.carry = options ? options->carry : 0;
  so.timeout_us = options ? options->wait_timeout_us : 0;
  so.test_hook = options ? options->test_hook : 0;
  return so;
}

// Kernel choice of the forward: the staged kernels where they apply (CONV:
// their convolution-prologue instances), else the one-thread-per-channel
// kernel (which handles the prologue at run time).
template <bool CONV>
mamba_status_t forward_paths(const FwdArgs &a, size_t es, mamba_dtype_t dtype,
                             const StagedOptions &so, cudaStream_t s, unsigned char *save = nullptr) {
  const bool stageable = staged_supported(a, es);
  if (save) {  // a saving forward: the staged kernels, no other path
    if (!stageable) return MAMBA_ERR_INVALID_ARG;
    return dtype == MAMBA_BF16 ? staged_dispatch<__nv_bfloat16, CONV>(a, so, s, save)
                               : staged_dispatch<float, CONV>(a, so, s, save);
  }
  if (so.path == MAMBA_PATH_REFERENCE || (!stageable && so.path == MAMBA_PATH_AUTO))
    return dispatch<FwdReferenceLauncher>(dtype, a.N, a, s);
  if (!stageable) return MAMBA_ERR_UNSUPPORTED;
  const mamba_status_t st = dtype == MAMBA_BF16 ? staged_dispatch<__nv_bfloat16, CONV>(a, so, s)
                                                : staged_dispatch<float, CONV>(a, so, s);
  if (st == MAMBA_ERR_UNSUPPORTED && so.path == MAMBA_PATH_AUTO)
    return dispatch<FwdReferenceLauncher>(dtype, a.N, a, s);
  return st;
}

template <bool CONV>
mamba_status_t backward_paths(const BwdArgs &a, size_t es, mamba_dtype_t dtype,
                              const StagedOptions &so, cudaStream_t s,
                              const unsigned char *saved = nullptr) {
  const bool stageable = staged_bwd_supported(a, es);
  if (saved) {  // from a saving forward: the staged kernels, no other path
    if (!stageable) return MAMBA_ERR_INVALID_ARG;
    return dtype == MAMBA_BF16 ? staged_bwd_dispatch<__nv_bfloat16, CONV>(a, so, s, saved)
                               : staged_bwd_dispatch<float, CONV>(a, so, s, saved);
  }
  if (so.path == MAMBA_PATH_REFERENCE || (!stageable && so.path == MAMBA_PATH_AUTO))
    return dispatch<BwdReferenceLauncher>(dtype, a.N, a, s);
  if (!stageable) return MAMBA_ERR_UNSUPPORTED;
  const mamba_status_t st = dtype == MAMBA_BF16 ? staged_bwd_dispatch<__nv_bfloat16, CONV>(a, so, s)
                                                : staged_bwd_dispatch<float, CONV>(a, so, s);
  if (st == MAMBA_ERR_UNSUPPORTED && so.path == MAMBA_PATH_AUTO)
    return dispatch<BwdReferenceLauncher>(dtype, a.N, a, s);
  return st;
}

// Whether the fused projection (delta formed on the tensor cores inside the
// staged kernels) takes this forward: bf16, a shape the staged kernels take,
// a rank its tiles fit, and no explicit path other than automatic/structured.
bool proj_fused_ok(const FwdArgs &a, mamba_dtype_t dtype, const StagedOptions &so) {
  if (dtype != MAMBA_BF16 || so.path == MAMBA_PATH_REFERENCE) return false;
  if (!staged_supported(a, 2) || !a.dt_low || !a.W_dt) return false;
  auto al = [](const void *ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15) == 0; };
  if (!al(a.dt_low) || (int64_t(a.L) * 2) % 16 != 0) return false;
  const int Rp = (a.R + 15) / 16 * 16;
  return a.R >= 1 && Rp <= proj_max_rank<__nv_bfloat16, 16>();
}

mamba_status_t proj_fused_dispatch(const FwdArgs &a, const StagedOptions &o, cudaStream_t s,
                                   unsigned char *save = nullptr) {
  if (a.N <= 4) return staged_forward<__nv_bfloat16, 4, false, true>(a, o, s, &launch_status, nullptr, save);
  if (a.N <= 8) return staged_forward<__nv_bfloat16, 8, false, true>(a, o, s, &launch_status, nullptr, save);
  return staged_forward<__nv_bfloat16, 16, false, true>(a, o, s, &launch_status, nullptr, save);
}

mamba_status_t proj_fused_bwd_dispatch(const BwdArgs &a, const StagedOptions &o, cudaStream_t s,
                                       const unsigned char *saved = nullptr) {
  if (a.N <= 4) return staged_backward<__nv_bfloat16, 4, false, true>(a, o, s, &launch_status, saved);
  if (a.N <= 8) return staged_backward<__nv_bfloat16, 8, false, true>(a, o, s, &launch_status, saved);
  return staged_backward<__nv_bfloat16, 16, false, true>(a, o, s, &launch_status, saved);
}

// Bytes the fused projection's saving forward stores: 0 unless the fused
// kernels take the shape and the backward hands its adjoint on in sequence
// (its three-phase carry reads delta from the checkpoint pass).
template <int NM>
mamba_status_t dtproj_saved_nm(int64_t batch, int64_t dim, int64_t L, int64_t R, const StagedOptions &so,
                               uint64_t *bytes) {
  StagedPlan bpl;
  mamba_status_t st = staged_backward_plan<__nv_bfloat16, NM, false, true>(batch, dim, L, so, int(R), &bpl);
  if (st == MAMBA_ERR_UNSUPPORTED) return MAMBA_OK;
  if (st != MAMBA_OK) return st;
  if (bpl.kind != KIND_SEQ) return MAMBA_OK;
  SavedLayout sl;
  st = saved_layout<__nv_bfloat16, NM, false, true>(batch, dim, L, so, &sl, int(R));
  if (st == MAMBA_ERR_UNSUPPORTED) return MAMBA_OK;
  if (st != MAMBA_OK) return st;
  *bytes = sl.bytes;
  return MAMBA_OK;
}

mamba_status_t dtproj_saved_bytes_for(int64_t batch, int64_t dim, int64_t L, int64_t N, int64_t R,
                                      mamba_dtype_t dtype, const StagedOptions &so, uint64_t *bytes) {
  *bytes = 0;
  if (batch == 0 || dim == 0 || L == 0 || dtype != MAMBA_BF16 || so.path == MAMBA_PATH_REFERENCE ||
      !staged_shape_ok(L, dim, N, 2) || L % 8 != 0)
    return MAMBA_OK;
  if (R < 1 || (R + 15) / 16 * 16 > proj_max_rank<__nv_bfloat16, 16>()) return MAMBA_OK;
  if (N <= 4) return dtproj_saved_nm<4>(batch, dim, L, R, so, bytes);
  if (N <= 8) return dtproj_saved_nm<8>(batch, dim, L, R, so, bytes);
  return dtproj_saved_nm<16>(batch, dim, L, R, so, bytes);
}

// How the projection's gradient products split dW's contraction over the
// grid (tensor-core path); 0 splits when the shapes or alignments do not suit
// its TMA tiles (the CUDA-core contraction is used instead).
struct ProjGradPlan {
  int splits = 0, k_per_split = 0, k_tiles = 0;
  size_t part_bytes = 0;  // fp32 partial sums of dW, one set per split
};

ProjGradPlan proj_grads_plan(const void *W, const void *dt_low, int64_t batch, int64_t dim,
                             int64_t L, int64_t R, mamba_dtype_t dtype) {
  ProjGradPlan pl;
  auto al = [](const void *ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15) == 0; };
  if (dtype != MAMBA_BF16 || R % 8 != 0 || L % 8 != 0 || !al(W) || !al(dt_low)) return pl;
  const int Rp_in = int((R + 63) / 64 * 64), Rp_w = int((R + 15) / 16 * 16);
  if (Rp_in > 256 || Rp_w > 256 || L > (int64_t(1) << 30) || dim > (int64_t(1) << 30) ||
      batch > 65535)
    return pl;
  const int mt = int((dim + 127) / 128);
  pl.k_tiles = int(batch * ((L + 63) / 64));
  // one wave of two CTAs per SM
  int splits = std::max(1, std::min(pl.k_tiles, (2 * device_sm_count()) / mt));
  pl.k_per_split = (pl.k_tiles + splits - 1) / splits;
  pl.splits = (pl.k_tiles + pl.k_per_split - 1) / pl.k_per_split;
  pl.part_bytes = (size_t(pl.splits) * size_t(dim) * size_t(R) * 4 + 255) / 256 * 256;
  return pl;
}

// The projection's gradient products on the tensor cores (bf16, tcgen05),
// with the plan's partial sums in `part`: false (nothing enqueued) if a
// tensor map is refused, so that the caller takes the CUDA-core contraction.
bool proj_grads_tc(const ProjGradPlan &pl, float *part, const void *W, const void *dt_low,
                   const void *ddelta, void *d_dt_low, float *dW, int64_t batch, int64_t dim,
                   int64_t L, int64_t R, cudaStream_t s, mamba_status_t *st) {
  auto al = [](const void *ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15) == 0; };
  if (pl.splits == 0 || !part || !al(ddelta)) return false;
  const int Rp_in = int((R + 63) / 64 * 64), Rp_w = int((R + 15) / 16 * 16);
  const CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;
  CUtensorMap a_in, b_in, a_w, b_w;
  if (!make_map_3d(&a_in, ddelta, true, uint64_t(L), uint64_t(dim), uint64_t(batch), 64, 64, sw) ||
      !make_map_3d(&b_in, W, true, uint64_t(R), uint64_t(dim), 1, 64, 64, sw) ||
      !make_map_3d(&a_w, ddelta, true, uint64_t(L), uint64_t(dim), uint64_t(batch), 64, 128, sw) ||
      !make_map_3d(&b_w, dt_low, true, uint64_t(L), uint64_t(R), uint64_t(batch), 64, uint32_t(Rp_w), sw))
    return false;
  const int smem_in = proj_gemm_smem<true>(Rp_in), smem_w = proj_gemm_smem<false>(Rp_w);
  if (cudaFuncSetAttribute(proj_gemm_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem_in) != cudaSuccess ||
      cudaFuncSetAttribute(proj_gemm_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem_w) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  const int mt = int((dim + 127) / 128);
  ProjGemmArgs gi;
  gi.batch = batch; gi.dim = dim; gi.L = L; gi.R = int(R); gi.Rp = Rp_in;
  gi.k_tiles = int((dim + 63) / 64); gi.k_per_split = gi.k_tiles;
  gi.out = d_dt_low; gi.timeout_ns = kDefaultTimeoutNs;
  proj_gemm_kernel<true><<<dim3(unsigned((L + 127) / 128), unsigned(batch)), 128, smem_in, s>>>(a_in, b_in, gi);
  *st = launch_status();
  if (*st == MAMBA_OK) {
    ProjGemmArgs gw = gi;
    gw.Rp = Rp_w;
    gw.k_tiles = pl.k_tiles;
    gw.k_per_split = pl.k_per_split;
    gw.out = part;
    proj_gemm_kernel<false><<<dim3(unsigned(mt), unsigned(pl.splits)), 128, smem_w, s>>>(a_w, b_w, gw);
    *st = launch_status();
  }
  if (*st == MAMBA_OK) {
    const int64_t n = dim * R;
    proj_grad_weight_finalize<<<unsigned(std::min<int64_t>((n + 255) / 256, 1184)), 256, 0, s>>>(
        part, dW, n, pl.splits);
    *st = launch_status();
  }
  return true;
}

// d_dt_low = W^T ddelta per batch row and dW = sum_b ddelta_b dt_low_b^T.
mamba_status_t proj_grads(const ProjGradPlan &pl, float *part, const void *W, const void *dt_low,
                          const void *ddelta, void *d_dt_low, float *dW, int64_t batch, int64_t dim,
                          int64_t L, int64_t R, mamba_dtype_t dtype, cudaStream_t s) {
  {
    mamba_status_t st = MAMBA_OK;
    if (proj_grads_tc(pl, part, W, dt_low, ddelta, d_dt_low, dW, batch, dim, L, R, s, &st)) return st;
  }
  const Contraction gi = proj_grad_input(W, ddelta, d_dt_low, batch, dim, L, R);
  const Contraction gw = proj_grad_weight(ddelta, dt_low, dW, batch, dim, L, R);
  cudaError_t e;
  if (dtype == MAMBA_BF16) {
    e = launch_contraction<__nv_bfloat16, __nv_bfloat16>(gi, s);
    if (e == cudaSuccess && launch_status() == MAMBA_OK) e = launch_contraction<__nv_bfloat16, float>(gw, s);
  } else {
    e = launch_contraction<float, float>(gi, s);
    if (e == cudaSuccess && launch_status() == MAMBA_OK) e = launch_contraction<float, float>(gw, s);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return MAMBA_ERR_CUDA;
  }
  return launch_status();
}

// The forward and backward entry points with and without a saved buffer
// (`saving`: the calls of the saving pair, whose buffer holds
// mamba_scan_saved_bytes bytes or more).
mamba_status_t fwd_entry(const void *u, const void *delta, const float *delta_bias,
                                 const float *A, const void *B, const void *C, const float *D,
                                 const void *z, void *y, float *last_state, int64_t batch,
                                 int64_t dim, int64_t L, int64_t N, mamba_dtype_t dtype,
                                 const mamba_scan_options_t *options, mamba_stream_t stream,
                                 bool saving, void *saved, uint64_t saved_bytes) {
  mamba_status_t st = check_shape(batch, dim, L, N, dtype);
  if (st != MAMBA_OK) return st;
  if ((st = check_options(options)) != MAMBA_OK) return st;
  Checker ck;
  if (cudaGetDevice(&ck.dev) != cudaSuccess) {
    cudaGetLastError();
    return MAMBA_ERR_CUDA;
  }
  const size_t es = dtype_size(dtype);
  const size_t nbdl = size_t(batch) * size_t(dim) * size_t(L);
  const size_t nbnl = size_t(batch) * size_t(N) * size_t(L);
  ck.buf(u, nbdl * es, es, true, false);
  ck.buf(delta, nbdl * es, es, true, false);
  ck.buf(z, nbdl * es, es, false, false);
  ck.buf(B, nbnl * es, es, true, false);
  ck.buf(C, nbnl * es, es, true, false);
  ck.buf(A, size_t(dim) * N * 4, 4, true, false);
  ck.buf(D, size_t(dim) * 4, 4, false, false);
  ck.buf(delta_bias, size_t(dim) * 4, 4, false, false);
  ck.buf(y, nbdl * es, es, true, true);
  ck.buf(last_state, size_t(batch) * dim * N * 4, 4, false, true);
  const StagedOptions so = staged_options(options);
  uint64_t need = 0;
  if (saving) {  // what this forward stores for its backward (0: nothing)
    if ((st = saved_bytes_for(batch, dim, L, N, dtype, so, &need)) != MAMBA_OK) return st;
    if (need > saved_bytes) return MAMBA_ERR_INVALID_ARG;
    ck.buf(saved, need, 16, true, true);
  }
  if (ck.st != MAMBA_OK) return ck.st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (batch == 0 || dim == 0) return MAMBA_OK;
  if (L == 0) {
    if (last_state && cudaMemsetAsync(last_state, 0, size_t(batch) * dim * N * 4, s) != cudaSuccess)
      return cuda_status();
    return MAMBA_OK;
  }
  FwdArgs a;
  a.u = u; a.delta = delta; a.z = z; a.B = B; a.C = C;
  a.bias = delta_bias; a.A = A; a.D = D; a.y = y; a.last_state = last_state;
  a.batch = batch; a.dim = dim; a.L = L; a.N = (int)N;
  return forward_paths<false>(a, es, dtype, so, s, need ? static_cast<unsigned char *>(saved) : nullptr);
}


mamba_status_t bwd_entry(const void *u, const void *delta, const float *delta_bias,
                                 const float *A, const void *B, const void *C, const float *D,
                                 const void *z, const void *dy, void *du, void *ddelta,
                                 float *dA, void *dB, void *dC, float *dD, void *dz,
                                 float *ddelta_bias, int64_t batch, int64_t dim, int64_t L,
                                 int64_t N, mamba_dtype_t dtype,
                                 const mamba_scan_options_t *options, mamba_stream_t stream,
                                 bool saving, const void *saved, uint64_t saved_bytes) {
  mamba_status_t st = check_shape(batch, dim, L, N, dtype);
  if (st != MAMBA_OK) return st;
  if ((st = check_options(options)) != MAMBA_OK) return st;
  if ((z == nullptr) != (dz == nullptr) || (D == nullptr) != (dD == nullptr))
    return MAMBA_ERR_INVALID_ARG;
  Checker ck;
  if (cudaGetDevice(&ck.dev) != cudaSuccess) {
    cudaGetLastError();
    return MAMBA_ERR_CUDA;
  }
  const size_t es = dtype_size(dtype);
  const size_t nbdl = size_t(batch) * size_t(dim) * size_t(L);
  const size_t nbnl = size_t(batch) * size_t(N) * size_t(L);
  ck.buf(u, nbdl * es, es, true, false);
  ck.buf(delta, nbdl * es, es, true, false);
  ck.buf(z, nbdl * es, es, false, false);
  ck.buf(dy, nbdl * es, es, true, false);
  ck.buf(B, nbnl * es, es, true, false);
  ck.buf(C, nbnl * es, es, true, false);
  ck.buf(A, size_t(dim) * N * 4, 4, true, false);
  ck.buf(D, size_t(dim) * 4, 4, false, false);
  ck.buf(delta_bias, size_t(dim) * 4, 4, false, false);
  ck.buf(du, nbdl * es, es, true, true);
  ck.buf(ddelta, nbdl * es, es, true, true);
  ck.buf(dz, nbdl * es, es, false, true);
  ck.buf(dB, nbnl * es, es, true, true);
  ck.buf(dC, nbnl * es, es, true, true);
  ck.buf(dA, size_t(dim) * N * 4, 4, true, true);
  ck.buf(dD, size_t(dim) * 4, 4, false, true);
  ck.buf(ddelta_bias, size_t(dim) * 4, 4, false, true);
  const StagedOptions so = staged_options(options);
  uint64_t need = 0;
  if (saving) {  // what the saving forward stored (0: nothing; recompute)
    if ((st = saved_bytes_for(batch, dim, L, N, dtype, so, &need)) != MAMBA_OK) return st;
    if (need > saved_bytes) return MAMBA_ERR_INVALID_ARG;
    ck.buf(saved, need, 16, true, false);
  }
  if (ck.st != MAMBA_OK) return ck.st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (dim == 0) return MAMBA_OK;
  if (batch == 0 || L == 0) {
    // Empty sum: parameter gradients are zero, and dB / dC have no elements
    // unless batch > 0 and L > 0.
    if (cudaMemsetAsync(dA, 0, size_t(dim) * N * 4, s) != cudaSuccess) return cuda_status();
    if (dD && cudaMemsetAsync(dD, 0, size_t(dim) * 4, s) != cudaSuccess) return cuda_status();
    if (ddelta_bias && cudaMemsetAsync(ddelta_bias, 0, size_t(dim) * 4, s) != cudaSuccess)
      return cuda_status();
    return MAMBA_OK;
  }
  BwdArgs a;
  a.u = u; a.delta = delta; a.z = z; a.B = B; a.C = C; a.dy = dy;
  a.bias = delta_bias; a.A = A; a.D = D;
  a.du = du; a.ddelta = ddelta; a.dz = dz; a.dB = dB; a.dC = dC;
  a.dA = dA; a.dD = dD; a.dbias = ddelta_bias;
  a.batch = batch; a.dim = dim; a.L = L; a.N = (int)N;
  return backward_paths<false>(a, es, dtype, so, s,
                               need ? static_cast<const unsigned char *>(saved) : nullptr);
}

}  // namespace

extern "C" {

int mamba_scan_abi_version(void) { return kAbiVersion; }

uint64_t mamba_scan_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char *mamba_scan_status_string(mamba_status_t s) {
  switch (s) {
    case MAMBA_OK: return "MAMBA_OK";
    case MAMBA_ERR_INVALID_ARG: return "MAMBA_ERR_INVALID_ARG";
    case MAMBA_ERR_UNSUPPORTED: return "MAMBA_ERR_UNSUPPORTED";
    case MAMBA_ERR_CUDA: return "MAMBA_ERR_CUDA";
    case MAMBA_ERR_OUT_OF_MEMORY: return "MAMBA_ERR_OUT_OF_MEMORY";
    case MAMBA_ERR_DEVICE_TIMEOUT: return "MAMBA_ERR_DEVICE_TIMEOUT";
    case MAMBA_ERR_OUT_OF_BOUNDS: return "MAMBA_ERR_OUT_OF_BOUNDS";
  }
  return "MAMBA_ERR_UNKNOWN";
}

mamba_status_t mamba_scan_stream_status(mamba_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return MAMBA_ERR_CUDA;
  }
  unsigned int word = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word)) != cudaSuccess ||
      cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)) != cudaSuccess) {
    cudaGetLastError();
    return MAMBA_ERR_CUDA;
  }
  if (word & kErrTimeout) return MAMBA_ERR_DEVICE_TIMEOUT;
  return (word & kErrBounds) ? MAMBA_ERR_OUT_OF_BOUNDS : MAMBA_OK;
}

mamba_status_t mamba_scan_fwd_ex(const void *u, const void *delta, const float *delta_bias,
                                 const float *A, const void *B, const void *C, const float *D,
                                 const void *z, void *y, float *last_state, int64_t batch,
                                 int64_t dim, int64_t L, int64_t N, mamba_dtype_t dtype,
                                 const mamba_scan_options_t *options, mamba_stream_t stream) {
  return fwd_entry(u, delta, delta_bias, A, B, C, D, z, y, last_state, batch, dim, L, N, dtype, options,
                   stream, false, nullptr, 0);
}

mamba_status_t mamba_scan_saved_bytes(int64_t batch, int64_t dim, int64_t L, int64_t N,
                                      mamba_dtype_t dtype, const mamba_scan_options_t *options,
                                      uint64_t *bytes) {
  if (!bytes) return MAMBA_ERR_INVALID_ARG;
  *bytes = 0;
  mamba_status_t st = check_shape(batch, dim, L, N, dtype);
  if (st != MAMBA_OK) return st;
  if ((st = check_options(options)) != MAMBA_OK) return st;
  return saved_bytes_for(batch, dim, L, N, dtype, staged_options(options), bytes);
}

mamba_status_t mamba_scan_fwd_save(const void *u, const void *delta, const float *delta_bias,
                                   const float *A, const void *B, const void *C, const float *D,
                                   const void *z, void *y, float *last_state, int64_t batch,
                                   int64_t dim, int64_t L, int64_t N, mamba_dtype_t dtype,
                                   const mamba_scan_options_t *options, void *saved,
                                   uint64_t saved_bytes, mamba_stream_t stream) {
  return fwd_entry(u, delta, delta_bias, A, B, C, D, z, y, last_state, batch, dim, L, N, dtype, options,
                   stream, true, saved, saved_bytes);
}

mamba_status_t mamba_scan_fwd(const void *u, const void *delta, const float *delta_bias,
                              const float *A, const void *B, const void *C, const float *D,
                              const void *z, void *y, float *last_state, int64_t batch,
                              int64_t dim, int64_t L, int64_t N, mamba_dtype_t dtype,
                              mamba_stream_t stream) {
  return mamba_scan_fwd_ex(u, delta, delta_bias, A, B, C, D, z, y, last_state, batch, dim, L, N,
                           dtype, nullptr, stream);
}

mamba_status_t mamba_scan_bwd_ex(const void *u, const void *delta, const float *delta_bias,
                                 const float *A, const void *B, const void *C, const float *D,
                                 const void *z, const void *dy, void *du, void *ddelta,
                                 float *dA, void *dB, void *dC, float *dD, void *dz,
                                 float *ddelta_bias, int64_t batch, int64_t dim, int64_t L,
                                 int64_t N, mamba_dtype_t dtype,
                                 const mamba_scan_options_t *options, mamba_stream_t stream) {
  return bwd_entry(u, delta, delta_bias, A, B, C, D, z, dy, du, ddelta, dA, dB, dC, dD, dz, ddelta_bias,
                   batch, dim, L, N, dtype, options, stream, false, nullptr, 0);
}

mamba_status_t mamba_scan_bwd_saved(const void *u, const void *delta, const float *delta_bias,
                                    const float *A, const void *B, const void *C, const float *D,
                                    const void *z, const void *dy, void *du, void *ddelta,
                                    float *dA, void *dB, void *dC, float *dD, void *dz,
                                    float *ddelta_bias, int64_t batch, int64_t dim, int64_t L,
                                    int64_t N, mamba_dtype_t dtype,
                                    const mamba_scan_options_t *options, const void *saved,
                                    uint64_t saved_bytes, mamba_stream_t stream) {
  return bwd_entry(u, delta, delta_bias, A, B, C, D, z, dy, du, ddelta, dA, dB, dC, dD, dz, ddelta_bias,
                   batch, dim, L, N, dtype, options, stream, true, saved, saved_bytes);
}

}  // extern "C"

namespace {

// One decoding token, validated once: the kernel arguments and the launch
// shape.  A plan (mamba_scan_step_plan_create) keeps one of these so that a
// decoding loop pays the pointer checks once instead of every token.
struct StepPlan {
  DecodeArgs a;
  bool conv = false;
  bool vec4 = false;
  mamba_dtype_t dtype = MAMBA_F32;
  int64_t grid = 0;
  int dev = 0;
};

// Validates one decoding token's arguments (CONV: with the convolution
// prologue) and fills `p`; enqueues nothing.
template <bool CONV>
mamba_status_t decode_prepare(StepPlan *p, float *state, float *conv_state, const void *u,
                              const float *conv_w, const float *conv_b, int64_t conv_width,
                              const void *delta, const float *delta_bias, const float *A,
                              const void *B, const void *C, const float *D, const void *z, void *y,
                              int64_t batch, int64_t dim, int64_t N, mamba_dtype_t dtype) {
  mamba_status_t st = check_shape(batch, dim, 1, N, dtype);
  if (st != MAMBA_OK) return st;
  if (CONV && (conv_width < 1 || conv_width > kMaxConvWidth)) return MAMBA_ERR_UNSUPPORTED;
  Checker ck;
  if (cudaGetDevice(&ck.dev) != cudaSuccess) {
    cudaGetLastError();
    return MAMBA_ERR_CUDA;
  }
  const size_t es = dtype_size(dtype);
  const size_t nbd = size_t(batch) * size_t(dim);
  ck.buf(u, nbd * es, es, true, false);
  ck.buf(delta, nbd * es, es, true, false);
  ck.buf(z, nbd * es, es, false, false);
  ck.buf(B, size_t(batch) * N * es, es, true, false);
  ck.buf(C, size_t(batch) * N * es, es, true, false);
  ck.buf(A, size_t(dim) * N * 4, 4, true, false);
  ck.buf(D, size_t(dim) * 4, 4, false, false);
  ck.buf(delta_bias, size_t(dim) * 4, 4, false, false);
  ck.buf(state, nbd * N * 4, 4, true, true);
  ck.buf(y, nbd * es, es, true, true);
  if (CONV) {
    ck.buf(conv_w, size_t(dim) * size_t(conv_width) * 4, 4, true, false);
    ck.buf(conv_b, size_t(dim) * 4, 4, false, false);
    ck.buf(conv_state, nbd * size_t(conv_width - 1) * 4, 4, conv_width > 1, true);
  }
  if (ck.st != MAMBA_OK) return ck.st;
  DecodeArgs &a = p->a;
  a.state = state; a.u = u; a.delta = delta; a.z = z; a.B = B; a.C = C;
  a.bias = delta_bias; a.A = A; a.D = D; a.y = y;
  a.batch = batch; a.dim = dim; a.N = (int)N;
  if (CONV) {
    a.conv_state = conv_state; a.conv_w = conv_w; a.conv_b = conv_b; a.conv_width = (int)conv_width;
  }
  p->conv = CONV;
  p->dtype = dtype;
  p->dev = ck.dev;
  // four states per thread when N is 4, 8 or 16 and the state, A, B and C
  // rows are 16- (B, C: 8-) byte aligned
  const bool al16 = ((reinterpret_cast<uintptr_t>(state) | reinterpret_cast<uintptr_t>(A)) & 15) == 0;
  const bool alBC = ((reinterpret_cast<uintptr_t>(B) | reinterpret_cast<uintptr_t>(C)) & (4 * es - 1)) == 0;
  p->vec4 = (N == 4 || N == 8 || N == 16) && al16 && alBC;
  const int64_t threads = p->vec4 ? int64_t(nbd) * (N / 4) : int64_t(nbd);
  p->grid = (threads + kDecodeThreads - 1) / kDecodeThreads;
  if (p->grid > (int64_t(1) << 31) - 1) return MAMBA_ERR_UNSUPPORTED;
  return MAMBA_OK;
}

// Enqueues the one launch of a validated decoding token (nothing for an
// empty problem).
template <bool CONV>
mamba_status_t decode_launch_t(const StepPlan &p, cudaStream_t s) {
  const DecodeArgs &a = p.a;
  const int N = a.N;
  const unsigned g = unsigned(p.grid);
  if (p.vec4) {
#define MSCAN_VEC4(TT, NN) decode_step_vec4_kernel<TT, NN, CONV><<<g, kDecodeThreads, 0, s>>>(a)
    if (p.dtype == MAMBA_BF16) {
      if (N == 4) MSCAN_VEC4(__nv_bfloat16, 4);
      else if (N == 8) MSCAN_VEC4(__nv_bfloat16, 8);
      else MSCAN_VEC4(__nv_bfloat16, 16);
    } else {
      if (N == 4) MSCAN_VEC4(float, 4);
      else if (N == 8) MSCAN_VEC4(float, 8);
      else MSCAN_VEC4(float, 16);
    }
#undef MSCAN_VEC4
    return launch_status();
  }
  auto launch = [&](auto tag, auto nm) {
    using T = typename decltype(tag)::type;
    decode_step_kernel<T, decltype(nm)::value, CONV><<<g, kDecodeThreads, 0, s>>>(a);
  };
  struct TF { using type = float; };
  struct TB { using type = __nv_bfloat16; };
  if (p.dtype == MAMBA_BF16) {
    if (N <= 4) launch(TB{}, std::integral_constant<int, 4>{});
    else if (N <= 8) launch(TB{}, std::integral_constant<int, 8>{});
    else launch(TB{}, std::integral_constant<int, 16>{});
  } else {
    if (N <= 4) launch(TF{}, std::integral_constant<int, 4>{});
    else if (N <= 8) launch(TF{}, std::integral_constant<int, 8>{});
    else launch(TF{}, std::integral_constant<int, 16>{});
  }
  return launch_status();
}

mamba_status_t decode_launch(const StepPlan &p, cudaStream_t s) {
  if (p.a.batch == 0 || p.a.dim == 0) return MAMBA_OK;
  return p.conv ? decode_launch_t<true>(p, s) : decode_launch_t<false>(p, s);
}

// One decoding token, with (CONV) or without the convolution prologue.
template <bool CONV>
mamba_status_t decode_step(float *state, float *conv_state, const void *u, const float *conv_w,
                           const float *conv_b, int64_t conv_width, const void *delta,
                           const float *delta_bias, const float *A, const void *B, const void *C,
                           const float *D, const void *z, void *y, int64_t batch, int64_t dim,
                           int64_t N, mamba_dtype_t dtype, mamba_stream_t stream) {
  StepPlan p;
  const mamba_status_t st = decode_prepare<CONV>(&p, state, conv_state, u, conv_w, conv_b,
                                                 conv_width, delta, delta_bias, A, B, C, D, z, y,
                                                 batch, dim, N, dtype);
  if (st != MAMBA_OK) return st;
  return decode_launch(p, reinterpret_cast<cudaStream_t>(stream));
}

}  // namespace

extern "C" {

mamba_status_t mamba_scan_step(float *state, const void *u, const void *delta,
                               const float *delta_bias, const float *A, const void *B, const void *C,
                               const float *D, const void *z, void *y, int64_t batch, int64_t dim,
                               int64_t N, mamba_dtype_t dtype, mamba_stream_t stream) {
  return decode_step<false>(state, nullptr, u, nullptr, nullptr, 0, delta, delta_bias, A, B, C, D,
                            z, y, batch, dim, N, dtype, stream);
}

mamba_status_t mamba_conv_scan_step(float *state, float *conv_state, const void *x,
                                    const float *conv_w, const float *conv_b, int64_t conv_width,
                                    const void *delta, const float *delta_bias, const float *A,
                                    const void *B, const void *C, const float *D, const void *z,
                                    void *y, int64_t batch, int64_t dim, int64_t N,
                                    mamba_dtype_t dtype, mamba_stream_t stream) {
  return decode_step<true>(state, conv_state, x, conv_w, conv_b, conv_width, delta, delta_bias, A,
                           B, C, D, z, y, batch, dim, N, dtype, stream);
}

mamba_status_t mamba_scan_bwd(const void *u, const void *delta, const float *delta_bias,
                              const float *A, const void *B, const void *C, const float *D,
                              const void *z, const void *dy, void *du, void *ddelta, float *dA,
                              void *dB, void *dC, float *dD, void *dz, float *ddelta_bias,
                              int64_t batch, int64_t dim, int64_t L, int64_t N,
                              mamba_dtype_t dtype, mamba_stream_t stream) {
  return mamba_scan_bwd_ex(u, delta, delta_bias, A, B, C, D, z, dy, du, ddelta, dA, dB, dC, dD,
                           dz, ddelta_bias, batch, dim, L, N, dtype, nullptr, stream);
}

// ------------------------------------------------ convolution prologue

static mamba_status_t conv_fwd_entry(const void *x, const float *conv_w, const float *conv_b,
                                     int64_t conv_width, const void *delta,
                                     const float *delta_bias, const float *A, const void *B,
                                     const void *C, const float *D, const void *z, void *y,
                                     float *last_state, int64_t batch, int64_t dim, int64_t L,
                                     int64_t N, mamba_dtype_t dtype,
                                     const mamba_scan_options_t *options, mamba_stream_t stream,
                                     bool saving, void *saved, uint64_t saved_bytes) {
  mamba_status_t st = check_shape(batch, dim, L, N, dtype);
  if (st != MAMBA_OK) return st;
  if ((st = check_options(options)) != MAMBA_OK) return st;
  if (conv_width < 1 || conv_width > kMaxConvWidth) return MAMBA_ERR_UNSUPPORTED;
  Checker ck;
  if (cudaGetDevice(&ck.dev) != cudaSuccess) {
    cudaGetLastError();
    return MAMBA_ERR_CUDA;
  }
  const size_t es = dtype_size(dtype);
  const size_t nbdl = size_t(batch) * size_t(dim) * size_t(L);
  const size_t nbnl = size_t(batch) * size_t(N) * size_t(L);
  ck.buf(x, nbdl * es, es, true, false);
  ck.buf(conv_w, size_t(dim) * size_t(conv_width) * 4, 4, true, false);
  ck.buf(conv_b, size_t(dim) * 4, 4, false, false);
  ck.buf(delta, nbdl * es, es, true, false);
  ck.buf(z, nbdl * es, es, false, false);
  ck.buf(B, nbnl * es, es, true, false);
  ck.buf(C, nbnl * es, es, true, false);
  ck.buf(A, size_t(dim) * N * 4, 4, true, false);
  ck.buf(D, size_t(dim) * 4, 4, false, false);
  ck.buf(delta_bias, size_t(dim) * 4, 4, false, false);
  ck.buf(y, nbdl * es, es, true, true);
  ck.buf(last_state, size_t(batch) * dim * N * 4, 4, false, true);
  const StagedOptions so = staged_options(options);
  uint64_t need = 0;
  if (saving) {  // what this forward stores for its backward (0: nothing)
    if ((st = saved_bytes_for(batch, dim, L, N, dtype, so, &need, true)) != MAMBA_OK) return st;
    if (need > saved_bytes) return MAMBA_ERR_INVALID_ARG;
    ck.buf(saved, need, 16, true, true);
  }
  if (ck.st != MAMBA_OK) return ck.st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (batch == 0 || dim == 0) return MAMBA_OK;
  if (L == 0) {
    if (last_state && cudaMemsetAsync(last_state, 0, size_t(batch) * dim * N * 4, s) != cudaSuccess)
      return cuda_status();
    return MAMBA_OK;
  }
  FwdArgs a;
  a.u = x; a.delta = delta; a.z = z; a.B = B; a.C = C;
  a.bias = delta_bias; a.A = A; a.D = D; a.y = y; a.last_state = last_state;
  a.batch = batch; a.dim = dim; a.L = L; a.N = (int)N;
  a.conv_w = conv_w; a.conv_b = conv_b; a.conv_width = (int)conv_width;
  return forward_paths<true>(a, es, dtype, so, s, need ? static_cast<unsigned char *>(saved) : nullptr);
}

mamba_status_t mamba_conv_scan_fwd(const void *x, const float *conv_w, const float *conv_b,
                                   int64_t conv_width, const void *delta,
                                   const float *delta_bias, const float *A, const void *B,
                                   const void *C, const float *D, const void *z, void *y,
                                   float *last_state, int64_t batch, int64_t dim, int64_t L,
                                   int64_t N, mamba_dtype_t dtype,
                                   const mamba_scan_options_t *options, mamba_stream_t stream) {
  return conv_fwd_entry(x, conv_w, conv_b, conv_width, delta, delta_bias, A, B, C, D, z, y, last_state,
                        batch, dim, L, N, dtype, options, stream, false, nullptr, 0);
}

mamba_status_t mamba_conv_scan_saved_bytes(int64_t batch, int64_t dim, int64_t L, int64_t N,
                                           int64_t conv_width, mamba_dtype_t dtype,
                                           const mamba_scan_options_t *options, uint64_t *bytes) {
  if (!bytes) return MAMBA_ERR_INVALID_ARG;
  *bytes = 0;
  mamba_status_t st = check_shape(batch, dim, L, N, dtype);
  if (st != MAMBA_OK) return st;
  if ((st = check_options(options)) != MAMBA_OK) return st;
  if (conv_width < 1 || conv_width > kMaxConvWidth) return MAMBA_ERR_UNSUPPORTED;
  return saved_bytes_for(batch, dim, L, N, dtype, staged_options(options), bytes, true);
}

mamba_status_t mamba_conv_scan_fwd_save(const void *x, const float *conv_w, const float *conv_b,
                                        int64_t conv_width, const void *delta,
                                        const float *delta_bias, const float *A, const void *B,
                                        const void *C, const float *D, const void *z, void *y,
                                        float *last_state, int64_t batch, int64_t dim, int64_t L,
                                        int64_t N, mamba_dtype_t dtype,
                                        const mamba_scan_options_t *options, void *saved,
                                        uint64_t saved_bytes, mamba_stream_t stream) {
  return conv_fwd_entry(x, conv_w, conv_b, conv_width, delta, delta_bias, A, B, C, D, z, y, last_state,
                        batch, dim, L, N, dtype, options, stream, true, saved, saved_bytes);
}

static mamba_status_t conv_bwd_entry(const void *x, const float *conv_w, const float *conv_b,
                                     int64_t conv_width, const void *delta,
                                     const float *delta_bias, const float *A, const void *B,
                                     const void *C, const float *D, const void *z, const void *dy,
                                     void *dx, float *dconv_w, float *dconv_b, void *ddelta,
                                     float *dA, void *dB, void *dC, float *dD, void *dz,
                                     float *ddelta_bias, int64_t batch, int64_t dim, int64_t L,
                                     int64_t N, mamba_dtype_t dtype,
                                     const mamba_scan_options_t *options, mamba_stream_t stream,
                                     bool saving, const void *saved, uint64_t saved_bytes) {
  mamba_status_t st = check_shape(batch, dim, L, N, dtype);
  if (st != MAMBA_OK) return st;
  if ((st = check_options(options)) != MAMBA_OK) return st;
  if (conv_width < 1 || conv_width > kMaxConvWidth) return MAMBA_ERR_UNSUPPORTED;
  if ((z == nullptr) != (dz == nullptr) || (D == nullptr) != (dD == nullptr))
    return MAMBA_ERR_INVALID_ARG;
  Checker ck;
  if (cudaGetDevice(&ck.dev) != cudaSuccess) {
    cudaGetLastError();
    return MAMBA_ERR_CUDA;
  }
  const size_t es = dtype_size(dtype);
  const size_t nbdl = size_t(batch) * size_t(dim) * size_t(L);
  const size_t nbnl = size_t(batch) * size_t(N) * size_t(L);
  const size_t nw = size_t(dim) * size_t(conv_width) * 4;
  ck.buf(x, nbdl * es, es, true, false);
  ck.buf(conv_w, nw, 4, true, false);
  ck.buf(conv_b, size_t(dim) * 4, 4, false, false);
  ck.buf(delta, nbdl * es, es, true, false);
  ck.buf(z, nbdl * es, es, false, false);
  ck.buf(dy, nbdl * es, es, true, false);
  ck.buf(B, nbnl * es, es, true, false);
  ck.buf(C, nbnl * es, es, true, false);
  ck.buf(A, size_t(dim) * N * 4, 4, true, false);
  ck.buf(D, size_t(dim) * 4, 4, false, false);
  ck.buf(delta_bias, size_t(dim) * 4, 4, false, false);
  ck.buf(dx, nbdl * es, es, true, true);
  ck.buf(dconv_w, nw, 4, true, true);
  ck.buf(dconv_b, size_t(dim) * 4, 4, false, true);
  ck.buf(ddelta, nbdl * es, es, true, true);
  ck.buf(dz, nbdl * es, es, false, true);
  ck.buf(dB, nbnl * es, es, true, true);
  ck.buf(dC, nbnl * es, es, true, true);
  ck.buf(dA, size_t(dim) * N * 4, 4, true, true);
  ck.buf(dD, size_t(dim) * 4, 4, false, true);
  ck.buf(ddelta_bias, size_t(dim) * 4, 4, false, true);
  const StagedOptions so = staged_options(options);
  uint64_t need = 0;
  if (saving) {  // what the saving forward stored (0: nothing; recompute)
    if ((st = saved_bytes_for(batch, dim, L, N, dtype, so, &need, true)) != MAMBA_OK) return st;
    if (need > saved_bytes) return MAMBA_ERR_INVALID_ARG;
    ck.buf(saved, need, 16, true, false);
  }
  if (ck.st != MAMBA_OK) return ck.st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (dim == 0) return MAMBA_OK;
  if (batch == 0 || L == 0) {  // empty sums
    if (cudaMemsetAsync(dA, 0, size_t(dim) * N * 4, s) != cudaSuccess ||
        cudaMemsetAsync(dconv_w, 0, nw, s) != cudaSuccess ||
        (dconv_b && cudaMemsetAsync(dconv_b, 0, size_t(dim) * 4, s) != cudaSuccess) ||
        (dD && cudaMemsetAsync(dD, 0, size_t(dim) * 4, s) != cudaSuccess) ||
        (ddelta_bias && cudaMemsetAsync(ddelta_bias, 0, size_t(dim) * 4, s) != cudaSuccess))
      return cuda_status();
    return MAMBA_OK;
  }
  const int64_t rows = batch * dim;
  const int64_t conv_grid = (rows + kConvWarps - 1) / kConvWarps;
  if (conv_grid > (int64_t(1) << 31) - 1) return MAMBA_ERR_UNSUPPORTED;
  // 1. the scan backward with the prologue recomputed; the gradient with
  //    respect to u lands in dx
  BwdArgs a;
  a.u = x; a.delta = delta; a.z = z; a.B = B; a.C = C; a.dy = dy;
  a.bias = delta_bias; a.A = A; a.D = D;
  a.du = dx; a.ddelta = ddelta; a.dz = dz; a.dB = dB; a.dC = dC;
  a.dA = dA; a.dD = dD; a.dbias = ddelta_bias;
  a.batch = batch; a.dim = dim; a.L = L; a.N = (int)N;
  a.conv_w = conv_w; a.conv_b = conv_b; a.conv_width = (int)conv_width;
  // the per-row filter sums of step 2 are allocated first, so that a failed
  // allocation leaves nothing enqueued
  float *part = nullptr;
  if (ws_alloc(reinterpret_cast<void **>(&part), size_t(rows) * 5 * 4, s) != cudaSuccess) {
    cudaGetLastError();
    return MAMBA_ERR_OUT_OF_MEMORY;
  }
  if ((st = backward_paths<true>(a, es, dtype, so, s,
                                need ? static_cast<const unsigned char *>(saved) : nullptr)) !=
      MAMBA_OK) {
    ws_free(part, s);
    return st;
  }
  // 2. through SiLU and the convolution, in place on dx, then the filter sums
  const bool vec = (size_t(L) * es) % 16 == 0 &&
                   ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(dx)) & 15) == 0;
  const int W = (int)conv_width;
#define MSCAN_CONV_BWD(TT, VV)                                                               \
  conv_bwd_kernel<TT, VV><<<unsigned(conv_grid), 32 * kConvWarps, 0, s>>>(                    \
      static_cast<const TT *>(x), static_cast<TT *>(dx), conv_w, conv_b, W, rows, dim, L, part)
  if (dtype == MAMBA_BF16) {
    if (vec) MSCAN_CONV_BWD(__nv_bfloat16, true);
    else MSCAN_CONV_BWD(__nv_bfloat16, false);
  } else {
    if (vec) MSCAN_CONV_BWD(float, true);
    else MSCAN_CONV_BWD(float, false);
  }
#undef MSCAN_CONV_BWD
  st = launch_status();
  if (st == MAMBA_OK) {
    const int64_t g = std::min<int64_t>((dim + 255) / 256, 148 * 8);
    conv_bwd_finalize<<<unsigned(g), 256, 0, s>>>(part, batch, dim, W, dconv_w, dconv_b);
    st = launch_status();
  }
  if (ws_free(part, s) != cudaSuccess && st == MAMBA_OK) st = MAMBA_ERR_CUDA;
  return st;
}

mamba_status_t mamba_conv_scan_bwd(const void *x, const float *conv_w, const float *conv_b,
                                   int64_t conv_width, const void *delta,
                                   const float *delta_bias, const float *A, const void *B,
                                   const void *C, const float *D, const void *z, const void *dy,
                                   void *dx, float *dconv_w, float *dconv_b, void *ddelta,
                                   float *dA, void *dB, void *dC, float *dD, void *dz,
                                   float *ddelta_bias, int64_t batch, int64_t dim, int64_t L,
                                   int64_t N, mamba_dtype_t dtype,
                                   const mamba_scan_options_t *options, mamba_stream_t stream) {
  return conv_bwd_entry(x, conv_w, conv_b, conv_width, delta, delta_bias, A, B, C, D, z, dy, dx, dconv_w,
                        dconv_b, ddelta, dA, dB, dC, dD, dz, ddelta_bias, batch, dim, L, N, dtype, options,
                        stream, false, nullptr, 0);
}

mamba_status_t mamba_conv_scan_bwd_saved(const void *x, const float *conv_w, const float *conv_b,
                                         int64_t conv_width, const void *delta,
                                         const float *delta_bias, const float *A, const void *B,
                                         const void *C, const float *D, const void *z, const void *dy,
                                         void *dx, float *dconv_w, float *dconv_b, void *ddelta,
                                         float *dA, void *dB, void *dC, float *dD, void *dz,
                                         float *ddelta_bias, int64_t batch, int64_t dim, int64_t L,
                                         int64_t N, mamba_dtype_t dtype,
                                         const mamba_scan_options_t *options, const void *saved,
                                         uint64_t saved_bytes, mamba_stream_t stream) {
  return conv_bwd_entry(x, conv_w, conv_b, conv_width, delta, delta_bias, A, B, C, D, z, dy, dx, dconv_w,
                        dconv_b, ddelta, dA, dB, dC, dD, dz, ddelta_bias, batch, dim, L, N, dtype, options,
                        stream, true, saved, saved_bytes);
}

// ------------------------------------------- low-rank Delta projection

static mamba_status_t dtproj_fwd_entry(const void *u, const void *dt_low, const void *W_dt,
                                       int64_t R, const float *delta_bias, const float *A,
                                       const void *B, const void *C, const float *D, const void *z,
                                       void *y, float *last_state, int64_t batch, int64_t dim,
                                       int64_t L, int64_t N, mamba_dtype_t dtype,
                                       const mamba_scan_options_t *options, mamba_stream_t stream,
                                       bool saving, void *saved, uint64_t saved_bytes) {
  mamba_status_t st = check_shape(batch, dim, L, N, dtype);
  if (st != MAMBA_OK) return st;
  if ((st = check_options(options)) != MAMBA_OK) return st;
  if (R < 1 || R > (int64_t(1) << 20)) return MAMBA_ERR_INVALID_ARG;
  if (dim >= (int64_t(1) << 31) || L >= (int64_t(1) << 31)) return MAMBA_ERR_UNSUPPORTED;
  Checker ck;
  if (cudaGetDevice(&ck.dev) != cudaSuccess) {
    cudaGetLastError();
    return MAMBA_ERR_CUDA;
  }
  const size_t es = dtype_size(dtype);
  const size_t nbdl = size_t(batch) * size_t(dim) * size_t(L);
  const size_t nbnl = size_t(batch) * size_t(N) * size_t(L);
  ck.buf(u, nbdl * es, es, true, false);
  ck.buf(dt_low, size_t(batch) * size_t(R) * size_t(L) * es, es, true, false);
  ck.buf(W_dt, size_t(dim) * size_t(R) * es, es, true, false);
  ck.buf(z, nbdl * es, es, false, false);
  ck.buf(B, nbnl * es, es, true, false);
  ck.buf(C, nbnl * es, es, true, false);
  ck.buf(A, size_t(dim) * N * 4, 4, true, false);
  ck.buf(D, size_t(dim) * 4, 4, false, false);
  ck.buf(delta_bias, size_t(dim) * 4, 4, false, false);
  ck.buf(y, nbdl * es, es, true, true);
  ck.buf(last_state, size_t(batch) * dim * N * 4, 4, false, true);
  uint64_t need = 0;
  if (saving) {  // what this forward stores for its backward (0: nothing)
    if ((st = dtproj_saved_bytes_for(batch, dim, L, N, R, dtype, staged_options(options), &need)) != MAMBA_OK)
      return st;
    if (need > saved_bytes) return MAMBA_ERR_INVALID_ARG;
    ck.buf(saved, need, 16, true, true);
  }
  if (ck.st != MAMBA_OK) return ck.st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (batch == 0 || dim == 0) return MAMBA_OK;
  if (L == 0) {
    if (last_state && cudaMemsetAsync(last_state, 0, size_t(batch) * dim * N * 4, s) != cudaSuccess)
      return cuda_status();
    return MAMBA_OK;
  }
  FwdArgs a;
  a.u = u; a.delta = nullptr; a.z = z; a.B = B; a.C = C;
  a.bias = delta_bias; a.A = A; a.D = D; a.y = y; a.last_state = last_state;
  a.batch = batch; a.dim = dim; a.L = L; a.N = (int)N;
  a.dt_low = dt_low; a.W_dt = W_dt; a.R = (int)R;
  const StagedOptions so = staged_options(options);
  if (need) {  // a saving forward: the fused kernels, no other path
    if (!proj_fused_ok(a, dtype, so)) return MAMBA_ERR_INVALID_ARG;
    return proj_fused_dispatch(a, so, s, static_cast<unsigned char *>(saved));
  }
  // bf16 on the staged kernels: delta formed on the tensor cores inside the scan
  if (proj_fused_ok(a, dtype, so)) {
    st = proj_fused_dispatch(a, so, s);
    if (st != MAMBA_ERR_UNSUPPORTED) return st;
  }
  // otherwise delta is formed first, in the I/O type, by the FP32 contraction
  void *delta = nullptr;
  if (ws_alloc(&delta, nbdl * es, s) != cudaSuccess) {
    cudaGetLastError();
    return MAMBA_ERR_OUT_OF_MEMORY;
  }
  const Contraction cd = proj_delta(W_dt, dt_low, delta, batch, dim, L, R);
  st = (dtype == MAMBA_BF16 ? launch_contraction<__nv_bfloat16, __nv_bfloat16>(cd, s)
                            : launch_contraction<float, float>(cd, s)) == cudaSuccess
           ? launch_status()
           : MAMBA_ERR_CUDA;
  if (st == MAMBA_OK) {
    a.delta = delta;
    a.dt_low = a.W_dt = nullptr;
    a.R = 0;
    st = forward_paths<false>(a, es, dtype, so, s);
  }
  if (ws_free(delta, s) != cudaSuccess && st == MAMBA_OK) st = MAMBA_ERR_CUDA;
  return st;
}

mamba_status_t mamba_dtproj_scan_fwd(const void *u, const void *dt_low, const void *W_dt,
                                     int64_t R, const float *delta_bias, const float *A,
                                     const void *B, const void *C, const float *D, const void *z,
                                     void *y, float *last_state, int64_t batch, int64_t dim,
                                     int64_t L, int64_t N, mamba_dtype_t dtype,
                                     const mamba_scan_options_t *options, mamba_stream_t stream) {
  return dtproj_fwd_entry(u, dt_low, W_dt, R, delta_bias, A, B, C, D, z, y, last_state, batch, dim, L,
                          N, dtype, options, stream, false, nullptr, 0);
}

mamba_status_t mamba_dtproj_scan_saved_bytes(int64_t batch, int64_t dim, int64_t L, int64_t N,
                                             int64_t R, mamba_dtype_t dtype,
                                             const mamba_scan_options_t *options, uint64_t *bytes) {
  if (!bytes) return MAMBA_ERR_INVALID_ARG;
  *bytes = 0;
  mamba_status_t st = check_shape(batch, dim, L, N, dtype);
  if (st != MAMBA_OK) return st;
  if ((st = check_options(options)) != MAMBA_OK) return st;
  if (R < 1 || R > (int64_t(1) << 20)) return MAMBA_ERR_INVALID_ARG;
  return dtproj_saved_bytes_for(batch, dim, L, N, R, dtype, staged_options(options), bytes);
}

mamba_status_t mamba_dtproj_scan_fwd_save(const void *u, const void *dt_low, const void *W_dt,
                                          int64_t R, const float *delta_bias, const float *A,
                                          const void *B, const void *C, const float *D,
                                          const void *z, void *y, float *last_state, int64_t batch,
                                          int64_t dim, int64_t L, int64_t N, mamba_dtype_t dtype,
                                          const mamba_scan_options_t *options, void *saved,
                                          uint64_t saved_bytes, mamba_stream_t stream) {
  return dtproj_fwd_entry(u, dt_low, W_dt, R, delta_bias, A, B, C, D, z, y, last_state, batch, dim, L,
                          N, dtype, options, stream, true, saved, saved_bytes);
}

static mamba_status_t dtproj_bwd_entry(const void *u, const void *dt_low, const void *W_dt,
                                       int64_t R, const float *delta_bias, const float *A,
                                       const void *B, const void *C, const float *D, const void *z,
                                       const void *dy, void *du, void *d_dt_low, float *dW_dt,
                                       float *dA, void *dB, void *dC, float *dD, void *dz,
                                       float *ddelta_bias, int64_t batch, int64_t dim, int64_t L,
                                       int64_t N, mamba_dtype_t dtype,
                                       const mamba_scan_options_t *options, mamba_stream_t stream,
                                       bool saving, const void *saved, uint64_t saved_bytes) {
  mamba_status_t st = check_shape(batch, dim, L, N, dtype);
  if (st != MAMBA_OK) return st;
  if ((st = check_options(options)) != MAMBA_OK) return st;
  if (R < 1 || R > (int64_t(1) << 20)) return MAMBA_ERR_INVALID_ARG;
  if (dim >= (int64_t(1) << 31) || L >= (int64_t(1) << 31)) return MAMBA_ERR_UNSUPPORTED;
  if ((z == nullptr) != (dz == nullptr) || (D == nullptr) != (dD == nullptr))
    return MAMBA_ERR_INVALID_ARG;
  Checker ck;
  if (cudaGetDevice(&ck.dev) != cudaSuccess) {
    cudaGetLastError();
    return MAMBA_ERR_CUDA;
  }
  const size_t es = dtype_size(dtype);
  const size_t nbdl = size_t(batch) * size_t(dim) * size_t(L);
  const size_t nbnl = size_t(batch) * size_t(N) * size_t(L);
  const size_t nbrl = size_t(batch) * size_t(R) * size_t(L);
  ck.buf(u, nbdl * es, es, true, false);
  ck.buf(dt_low, nbrl * es, es, true, false);
  ck.buf(W_dt, size_t(dim) * size_t(R) * es, es, true, false);
  ck.buf(z, nbdl * es, es, false, false);
  ck.buf(dy, nbdl * es, es, true, false);
  ck.buf(B, nbnl * es, es, true, false);
  ck.buf(C, nbnl * es, es, true, false);
  ck.buf(A, size_t(dim) * N * 4, 4, true, false);
  ck.buf(D, size_t(dim) * 4, 4, false, false);
  ck.buf(delta_bias, size_t(dim) * 4, 4, false, false);
  ck.buf(du, nbdl * es, es, true, true);
  ck.buf(d_dt_low, nbrl * es, es, true, true);
  ck.buf(dW_dt, size_t(dim) * size_t(R) * 4, 4, true, true);
  ck.buf(dz, nbdl * es, es, false, true);
  ck.buf(dB, nbnl * es, es, true, true);
  ck.buf(dC, nbnl * es, es, true, true);
  ck.buf(dA, size_t(dim) * N * 4, 4, true, true);
  ck.buf(dD, size_t(dim) * 4, 4, false, true);
  ck.buf(ddelta_bias, size_t(dim) * 4, 4, false, true);
  uint64_t need = 0;
  if (saving) {  // what the saving forward stored (0: nothing; recompute)
    if ((st = dtproj_saved_bytes_for(batch, dim, L, N, R, dtype, staged_options(options), &need)) != MAMBA_OK)
      return st;
    if (need > saved_bytes) return MAMBA_ERR_INVALID_ARG;
    ck.buf(saved, need, 16, true, false);
  }
  if (ck.st != MAMBA_OK) return ck.st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (dim == 0) return MAMBA_OK;
  if (batch == 0 || L == 0) {  // empty sums
    if (cudaMemsetAsync(dA, 0, size_t(dim) * N * 4, s) != cudaSuccess ||
        cudaMemsetAsync(dW_dt, 0, size_t(dim) * size_t(R) * 4, s) != cudaSuccess ||
        (dD && cudaMemsetAsync(dD, 0, size_t(dim) * 4, s) != cudaSuccess) ||
        (ddelta_bias && cudaMemsetAsync(ddelta_bias, 0, size_t(dim) * 4, s) != cudaSuccess))
      return cuda_status();
    return MAMBA_OK;
  }
  BwdArgs a;
  a.u = u; a.delta = nullptr; a.z = z; a.B = B; a.C = C; a.dy = dy;
  a.bias = delta_bias; a.A = A; a.D = D;
  a.du = du; a.ddelta = nullptr; a.dz = dz; a.dB = dB; a.dC = dC;
  a.dA = dA; a.dD = dD; a.dbias = ddelta_bias;
  a.batch = batch; a.dim = dim; a.L = L; a.N = (int)N;
  a.dt_low = dt_low; a.W_dt = W_dt; a.R = (int)R;
  const StagedOptions so = staged_options(options);
  FwdArgs fa;
  fa.u = u; fa.delta = nullptr; fa.z = z; fa.B = B; fa.C = C; fa.bias = delta_bias; fa.A = A;
  fa.D = D; fa.y = nullptr; fa.last_state = nullptr; fa.batch = batch; fa.dim = dim; fa.L = L;
  fa.N = (int)N; fa.dt_low = dt_low; fa.W_dt = W_dt; fa.R = (int)R;
  const bool fused = proj_fused_ok(fa, dtype, so) && staged_bwd_supported(a, es);
  if (need && !fused) return MAMBA_ERR_INVALID_ARG;  // saved states: the fused kernels only
  const ProjGradPlan gp = proj_grads_plan(W_dt, dt_low, batch, dim, L, R, dtype);
  // workspace: the gradient products' partial sums, ddelta (the scan
  // backward's gradient of delta, in the I/O type), then (unfused) delta
  const size_t half = (nbdl * es + 255) / 256 * 256;
  unsigned char *ws = nullptr;
  if (ws_alloc(reinterpret_cast<void **>(&ws), gp.part_bytes + (fused ? half : 2 * half), s) !=
      cudaSuccess) {
    cudaGetLastError();
    return MAMBA_ERR_OUT_OF_MEMORY;
  }
  float *part = gp.part_bytes ? reinterpret_cast<float *>(ws) : nullptr;
  void *ddelta = ws + gp.part_bytes, *delta = fused ? nullptr : ws + gp.part_bytes + half;
  a.ddelta = ddelta;
  st = MAMBA_ERR_UNSUPPORTED;
  if (fused) st = proj_fused_bwd_dispatch(a, so, s, need ? static_cast<const unsigned char *>(saved) : nullptr);
  if (need && st != MAMBA_OK) {  // no other path reads saved states
    ws_free(ws, s);
    return st;
  }
  if (st == MAMBA_ERR_UNSUPPORTED && delta == nullptr) {  // the fused kernels declined
    ws_free(ws, s);
    ws = nullptr;
    if (ws_alloc(reinterpret_cast<void **>(&ws), gp.part_bytes + 2 * half, s) != cudaSuccess) {
      cudaGetLastError();
      return MAMBA_ERR_OUT_OF_MEMORY;
    }
    part = gp.part_bytes ? reinterpret_cast<float *>(ws) : nullptr;
    ddelta = ws + gp.part_bytes;
    delta = ws + gp.part_bytes + half;
    a.ddelta = ddelta;
  }
  if (st == MAMBA_ERR_UNSUPPORTED) {
    const Contraction cd = proj_delta(W_dt, dt_low, delta, batch, dim, L, R);
    st = (dtype == MAMBA_BF16 ? launch_contraction<__nv_bfloat16, __nv_bfloat16>(cd, s)
                              : launch_contraction<float, float>(cd, s)) == cudaSuccess
             ? launch_status()
             : MAMBA_ERR_CUDA;
    if (st == MAMBA_OK) {
      a.delta = delta;
      a.dt_low = a.W_dt = nullptr;
      a.R = 0;
      st = backward_paths<false>(a, es, dtype, so, s);
    }
  }
  // the two gradient products of the projection, from ddelta
  if (st == MAMBA_OK)
    st = proj_grads(gp, part, W_dt, dt_low, ddelta, d_dt_low, dW_dt, batch, dim, L, R, dtype, s);
  if (ws_free(ws, s) != cudaSuccess && st == MAMBA_OK) st = MAMBA_ERR_CUDA;
  return st;
}

mamba_status_t mamba_dtproj_scan_bwd(const void *u, const void *dt_low, const void *W_dt,
                                     int64_t R, const float *delta_bias, const float *A,
                                     const void *B, const void *C, const float *D, const void *z,
                                     const void *dy, void *du, void *d_dt_low, float *dW_dt,
                                     float *dA, void *dB, void *dC, float *dD, void *dz,
                                     float *ddelta_bias, int64_t batch, int64_t dim, int64_t L,
                                     int64_t N, mamba_dtype_t dtype,
                                     const mamba_scan_options_t *options, mamba_stream_t stream) {
  return dtproj_bwd_entry(u, dt_low, W_dt, R, delta_bias, A, B, C, D, z, dy, du, d_dt_low, dW_dt, dA, dB,
                          dC, dD, dz, ddelta_bias, batch, dim, L, N, dtype, options, stream, false, nullptr,
                          0);
}

mamba_status_t mamba_dtproj_scan_bwd_saved(const void *u, const void *dt_low, const void *W_dt,
                                           int64_t R, const float *delta_bias, const float *A,
                                           const void *B, const void *C, const float *D,
                                           const void *z, const void *dy, void *du, void *d_dt_low,
                                           float *dW_dt, float *dA, void *dB, void *dC, float *dD,
                                           void *dz, float *ddelta_bias, int64_t batch, int64_t dim,
                                           int64_t L, int64_t N, mamba_dtype_t dtype,
                                           const mamba_scan_options_t *options, const void *saved,
                                           uint64_t saved_bytes, mamba_stream_t stream) {
  return dtproj_bwd_entry(u, dt_low, W_dt, R, delta_bias, A, B, C, D, z, dy, du, d_dt_low, dW_dt, dA, dB,
                          dC, dD, dz, ddelta_bias, batch, dim, L, N, dtype, options, stream, true, saved,
                          saved_bytes);
}

// ------------------------------------------------ complex diagonal A

// Bytes of the complex forward's saved block checkpoints: (batch*dim,
// ceil(L/8), 2 NM) fp32, NM the state count the kernels are instantiated for.
static uint64_t cplx_saved_bytes_for(int64_t batch, int64_t dim, int64_t L, int64_t N) {
  const int64_t nm = N <= 1 ? 1 : N <= 2 ? 2 : N <= 4 ? 4 : N <= 8 ? 8 : 16;
  return uint64_t(batch) * uint64_t(dim) * uint64_t((L + kCplxBwdTC - 1) / kCplxBwdTC) * 2 * nm * 4;
}

static mamba_status_t cplx_fwd_entry(const void *u, const void *delta, const float *delta_bias,
                                     const float *A, const void *B, const void *C, const float *D,
                                     const void *z, void *y, float *last_state, int64_t batch,
                                     int64_t dim, int64_t L, int64_t N, mamba_dtype_t dtype,
                                     mamba_stream_t stream, void *saved, uint64_t saved_bytes) {
  mamba_status_t st = check_shape(batch, dim, L, N, dtype);
  if (st != MAMBA_OK) return st;
  Checker ck;
  if (cudaGetDevice(&ck.dev) != cudaSuccess) {
    cudaGetLastError();
    return MAMBA_ERR_CUDA;
  }
  const size_t es = dtype_size(dtype);
  const size_t nbdl = size_t(batch) * size_t(dim) * size_t(L);
  const size_t nbnl = size_t(batch) * 2 * size_t(N) * size_t(L);
  ck.buf(u, nbdl * es, es, true, false);
  ck.buf(delta, nbdl * es, es, true, false);
  ck.buf(z, nbdl * es, es, false, false);
  ck.buf(B, nbnl * es, es, true, false);
  ck.buf(C, nbnl * es, es, true, false);
  ck.buf(A, size_t(dim) * 2 * N * 4, 4, true, false);
  ck.buf(D, size_t(dim) * 4, 4, false, false);
  ck.buf(delta_bias, size_t(dim) * 4, 4, false, false);
  ck.buf(y, nbdl * es, es, true, true);
  ck.buf(last_state, size_t(batch) * dim * 2 * N * 4, 4, false, true);
  const uint64_t need = saved ? cplx_saved_bytes_for(batch, dim, L, N) : 0;
  if (saved) {
    if (need > saved_bytes) return MAMBA_ERR_INVALID_ARG;
    ck.buf(saved, need, 16, true, true);
  }
  if (ck.st != MAMBA_OK) return ck.st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (batch == 0 || dim == 0) return MAMBA_OK;
  if (L == 0) {
    if (last_state && cudaMemsetAsync(last_state, 0, size_t(batch) * dim * 2 * N * 4, s) != cudaSuccess)
      return cuda_status();
    return MAMBA_OK;
  }
  if ((dim + kCplxThreads / 4 - 1) / (kCplxThreads / 4) > (int64_t(1) << 31) - 1)
    return MAMBA_ERR_UNSUPPORTED;
  CplxArgs a = {};
  a.u = u; a.delta = delta; a.z = z; a.B = B; a.C = C;
  a.bias = delta_bias; a.A = A; a.D = D; a.y = y; a.last_state = last_state;
  a.batch = batch; a.dim = dim; a.L = L; a.N = (int)N;
  if (need) {
    a.save_ckpt = static_cast<float *>(saved);
    a.save_blocks = (L + kCplxBwdTC - 1) / kCplxBwdTC;
  }
  return dispatch<CplxFwdLauncher>(dtype, (int)N, a, s);
}

mamba_status_t mamba_cplx_scan_fwd(const void *u, const void *delta, const float *delta_bias,
                                   const float *A, const void *B, const void *C, const float *D,
                                   const void *z, void *y, float *last_state, int64_t batch,
                                   int64_t dim, int64_t L, int64_t N, mamba_dtype_t dtype,
                                   mamba_stream_t stream) {
  return cplx_fwd_entry(u, delta, delta_bias, A, B, C, D, z, y, last_state, batch, dim, L, N, dtype,
                        stream, nullptr, 0);
}

mamba_status_t mamba_cplx_scan_saved_bytes(int64_t batch, int64_t dim, int64_t L, int64_t N,
                                           mamba_dtype_t dtype, uint64_t *bytes) {
  if (!bytes) return MAMBA_ERR_INVALID_ARG;
  *bytes = 0;
  const mamba_status_t st = check_shape(batch, dim, L, N, dtype);
  if (st != MAMBA_OK) return st;
  *bytes = cplx_saved_bytes_for(batch, dim, L, N);
  return MAMBA_OK;
}

mamba_status_t mamba_cplx_scan_fwd_save(const void *u, const void *delta, const float *delta_bias,
                                        const float *A, const void *B, const void *C, const float *D,
                                        const void *z, void *y, float *last_state, int64_t batch,
                                        int64_t dim, int64_t L, int64_t N, mamba_dtype_t dtype,
                                        void *saved, uint64_t saved_bytes, mamba_stream_t stream) {
  if (!saved && cplx_saved_bytes_for(batch, dim, L, N) > 0) return MAMBA_ERR_INVALID_ARG;
  return cplx_fwd_entry(u, delta, delta_bias, A, B, C, D, z, y, last_state, batch, dim, L, N, dtype,
                        stream, saved, saved_bytes);
}

static mamba_status_t cplx_bwd_entry(const void *u, const void *delta, const float *delta_bias,
                                     const float *A, const void *B, const void *C, const float *D,
                                     const void *z, const void *dy, void *du, void *ddelta,
                                     float *dA, void *dB, void *dC, float *dD, void *dz,
                                     float *ddelta_bias, int64_t batch, int64_t dim, int64_t L,
                                     int64_t N, mamba_dtype_t dtype, mamba_stream_t stream,
                                     const void *saved, uint64_t saved_bytes) {
  mamba_status_t st = check_shape(batch, dim, L, N, dtype);
  if (st != MAMBA_OK) return st;
  if ((z == nullptr) != (dz == nullptr) || (D == nullptr) != (dD == nullptr))
    return MAMBA_ERR_INVALID_ARG;
  Checker ck;
  if (cudaGetDevice(&ck.dev) != cudaSuccess) {
    cudaGetLastError();
    return MAMBA_ERR_CUDA;
  }
  const size_t es = dtype_size(dtype);
  const size_t nbdl = size_t(batch) * size_t(dim) * size_t(L);
  const size_t nbnl = size_t(batch) * 2 * size_t(N) * size_t(L);
  ck.buf(u, nbdl * es, es, true, false);
  ck.buf(delta, nbdl * es, es, true, false);
  ck.buf(z, nbdl * es, es, false, false);
  ck.buf(dy, nbdl * es, es, true, false);
  ck.buf(B, nbnl * es, es, true, false);
  ck.buf(C, nbnl * es, es, true, false);
  ck.buf(A, size_t(dim) * 2 * N * 4, 4, true, false);
  ck.buf(D, size_t(dim) * 4, 4, false, false);
  ck.buf(delta_bias, size_t(dim) * 4, 4, false, false);
  ck.buf(du, nbdl * es, es, true, true);
  ck.buf(ddelta, nbdl * es, es, true, true);
  ck.buf(dz, nbdl * es, es, false, true);
  ck.buf(dB, nbnl * es, es, true, true);
  ck.buf(dC, nbnl * es, es, true, true);
  ck.buf(dA, size_t(dim) * 2 * N * 4, 4, true, true);
  ck.buf(dD, size_t(dim) * 4, 4, false, true);
  ck.buf(ddelta_bias, size_t(dim) * 4, 4, false, true);
  if (saved) {
    const uint64_t need = cplx_saved_bytes_for(batch, dim, L, N);
    if (need > saved_bytes) return MAMBA_ERR_INVALID_ARG;
    ck.buf(saved, need, 16, true, false);
  }
  if (ck.st != MAMBA_OK) return ck.st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (dim == 0) return MAMBA_OK;
  if (batch == 0 || L == 0) {
    if (cudaMemsetAsync(dA, 0, size_t(dim) * 2 * N * 4, s) != cudaSuccess ||
        (dD && cudaMemsetAsync(dD, 0, size_t(dim) * 4, s) != cudaSuccess) ||
        (ddelta_bias && cudaMemsetAsync(ddelta_bias, 0, size_t(dim) * 4, s) != cudaSuccess))
      return cuda_status();
    return MAMBA_OK;
  }
  if ((dim + kCplxBwdThreads - 1) / kCplxBwdThreads > (int64_t(1) << 31) - 1)
    return MAMBA_ERR_UNSUPPORTED;
  CplxArgs a = {};
  a.u = u; a.delta = delta; a.z = z; a.B = B; a.C = C; a.dy = dy;
  a.bias = delta_bias; a.A = A; a.D = D;
  a.du = du; a.ddelta = ddelta; a.dz = dz; a.dB = dB; a.dC = dC;
  a.dA = dA; a.dD = dD; a.dbias = ddelta_bias;
  a.batch = batch; a.dim = dim; a.L = L; a.N = (int)N;
  a.saved_ckpt = static_cast<const float *>(saved);
  return dispatch<CplxBwdLauncher>(dtype, (int)N, a, s);
}

mamba_status_t mamba_cplx_scan_bwd(const void *u, const void *delta, const float *delta_bias,
                                   const float *A, const void *B, const void *C, const float *D,
                                   const void *z, const void *dy, void *du, void *ddelta,
                                   float *dA, void *dB, void *dC, float *dD, void *dz,
                                   float *ddelta_bias, int64_t batch, int64_t dim, int64_t L,
                                   int64_t N, mamba_dtype_t dtype, mamba_stream_t stream) {
  return cplx_bwd_entry(u, delta, delta_bias, A, B, C, D, z, dy, du, ddelta, dA, dB, dC, dD, dz,
                        ddelta_bias, batch, dim, L, N, dtype, stream, nullptr, 0);
}

mamba_status_t mamba_cplx_scan_bwd_saved(const void *u, const void *delta, const float *delta_bias,
                                         const float *A, const void *B, const void *C, const float *D,
                                         const void *z, const void *dy, void *du, void *ddelta,
                                         float *dA, void *dB, void *dC, float *dD, void *dz,
                                         float *ddelta_bias, int64_t batch, int64_t dim, int64_t L,
                                         int64_t N, mamba_dtype_t dtype, const void *saved,
                                         uint64_t saved_bytes, mamba_stream_t stream) {
  if (!saved && cplx_saved_bytes_for(batch, dim, L, N) > 0) return MAMBA_ERR_INVALID_ARG;
  return cplx_bwd_entry(u, delta, delta_bias, A, B, C, D, z, dy, du, ddelta, dA, dB, dC, dD, dz,
                        ddelta_bias, batch, dim, L, N, dtype, stream, saved, saved_bytes);
}

}  // extern "C"

// ------------------------------------------------ decoding plans, pool, hooks

struct mamba_step_plan_st {
  StepPlan p;
};

extern "C" {

mamba_status_t mamba_scan_step_plan_create(mamba_step_plan_t *plan, float *state,
                                           float *conv_state, const void *x, const float *conv_w,
                                           const float *conv_b, int64_t conv_width,
                                           const void *delta, const float *delta_bias,
                                           const float *A, const void *B, const void *C,
                                           const float *D, const void *z, void *y, int64_t batch,
                                           int64_t dim, int64_t N, mamba_dtype_t dtype) {
  if (!plan) return MAMBA_ERR_INVALID_ARG;
  *plan = nullptr;
  if (conv_width < 0) return MAMBA_ERR_INVALID_ARG;
  if (conv_width == 0 && (conv_state || conv_w || conv_b)) return MAMBA_ERR_INVALID_ARG;
  mamba_step_plan_st *h = new (std::nothrow) mamba_step_plan_st;
  if (!h) return MAMBA_ERR_OUT_OF_MEMORY;
  const mamba_status_t st =
      conv_width == 0
          ? decode_prepare<false>(&h->p, state, nullptr, x, nullptr, nullptr, 0, delta,
                                  delta_bias, A, B, C, D, z, y, batch, dim, N, dtype)
          : decode_prepare<true>(&h->p, state, conv_state, x, conv_w, conv_b, conv_width, delta,
                                 delta_bias, A, B, C, D, z, y, batch, dim, N, dtype);
  if (st != MAMBA_OK) {
    delete h;
    return st;
  }
  *plan = h;
  return MAMBA_OK;
}

mamba_status_t mamba_scan_step_plan_run(mamba_step_plan_t plan, mamba_stream_t stream) {
  if (!plan) return MAMBA_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return MAMBA_ERR_CUDA;
  }
  if (dev != plan->p.dev) return MAMBA_ERR_INVALID_ARG;
  return decode_launch(plan->p, reinterpret_cast<cudaStream_t>(stream));
}

void mamba_scan_step_plan_destroy(mamba_step_plan_t plan) { delete plan; }

mamba_status_t mamba_scan_pool_set_reserve(uint64_t bytes) {
  const int dev = current_device_or(-1);
  if (dev < 0) return MAMBA_ERR_CUDA;
  PoolRegistry &r = pool_registry();
  cudaMemPool_t pool = nullptr;
  {
    std::lock_guard<std::mutex> lock(r.mu);
    r.keep[dev] = bytes;
    pool = r.pools[dev];
  }
  if (pool && cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &bytes) != cudaSuccess) {
    cudaGetLastError();
    return MAMBA_ERR_CUDA;
  }
  return MAMBA_OK;
}

mamba_status_t mamba_scan_pool_trim(uint64_t keep_bytes) {
  const int dev = current_device_or(-1);
  if (dev < 0) return MAMBA_ERR_CUDA;
  PoolRegistry &r = pool_registry();
  cudaMemPool_t pool = nullptr;
  {
    std::lock_guard<std::mutex> lock(r.mu);
    pool = r.pools[dev];
  }
  if (pool && cudaMemPoolTrimTo(pool, size_t(keep_bytes)) != cudaSuccess) {
    cudaGetLastError();
    return MAMBA_ERR_CUDA;
  }
  return MAMBA_OK;
}

mamba_status_t mamba_scan_pool_reserved(uint64_t *bytes) {
  if (!bytes) return MAMBA_ERR_INVALID_ARG;
  *bytes = 0;
  const int dev = current_device_or(-1);
  if (dev < 0) return MAMBA_ERR_CUDA;
  PoolRegistry &r = pool_registry();
  cudaMemPool_t pool = nullptr;
  {
    std::lock_guard<std::mutex> lock(r.mu);
    pool = r.pools[dev];
  }
  if (!pool) return MAMBA_OK;
  cuuint64_t v = 0;
  if (cudaMemPoolGetAttribute(pool, cudaMemPoolAttrReservedMemCurrent, &v) != cudaSuccess) {
    cudaGetLastError();
    return MAMBA_ERR_CUDA;
  }
  *bytes = uint64_t(v);
  return MAMBA_OK;
}

void mamba_scan_test_fail_alloc(int32_t after) { alloc_failure_countdown() = after < 0 ? -1 : after; }

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free forward (mamba_scan_fwd_noalloc).
//
// Some callers cannot let a library allocate device memory: programs that
// hand all device memory to their own allocator at start-up (so an
// allocation by the library fails, or breaks their budget), latency-critical
// loops whose owners forbid any call into the CUDA allocator, and hosts that
// call the scan from code that must not enter the allocator at all.  For
// them the chunked forward keeps its scratch -- the unit ticket counter, the
// per-group hand-off flags and the carried chunk-end states -- in the fixed
// array below instead of taking a workspace per call.  The array is part of
// the library's device code, so every GPU that loads the library holds it
// (8 MiB) until the process exits.

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // per device
constexpr int kNoAllocMaxDevices = 64;

}  // namespace

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

std::mutex g_noalloc_mutex;
unsigned char *g_noalloc_ptr[kNoAllocMaxDevices] = {};

// Device address of g_noalloc_scratch on device `dev` (the current device).
// In host code the array's name only stands for the symbol, so the address
// is looked up with cudaGetSymbolAddress, once per device.
mamba_status_t noalloc_scratch(int dev, unsigned char **out) {
  if (dev < 0 || dev >= kNoAllocMaxDevices) return MAMBA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_ptr[dev] == nullptr) {
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) {
      cudaGetLastError();
      return MAMBA_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = static_cast<unsigned char *>(ptr);
  }
  *out = g_noalloc_ptr[dev];
  return MAMBA_OK;
}

// The staged forward with its workspace carved out of the fixed array: the
// plan the regular call would take (the sequential hand-off when the channel
// groups fill the GPU, else chunks from zero with the parallel scan over
// chunks and the closed-form correction) when its workspace fits; for the
// latter, fewer and longer chunks until it does; else the sequential
// hand-off.  Enqueues a memset of the counters and flags and the kernels.
template <typename T, int NM>
mamba_status_t noalloc_forward(const FwdArgs &a, unsigned char *scratch, cudaStream_t s) {
  StagedOptions o;
  o.path = MAMBA_PATH_AUTO;
  o.chunk_len = 0;
  o.carry = 0;
  o.timeout_us = 0;
  o.test_hook = 0;
  StagedForward<T, NM> sf;
  mamba_status_t st = sf.prepare(a, o, nullptr);
  if (st != MAMBA_OK) return st;
  if (sf.pl.kind == KIND_PAR && sf.bytes > kNoAllocScratchBytes) {
    // the aggregate pass (no running sums of Delta), then fewer, longer chunks
    sf.use_loc = false;
    if ((st = sf.prepare(a, o, nullptr)) != MAMBA_OK) return st;
  }
  if (sf.pl.kind == KIND_PAR && sf.bytes > kNoAllocScratchBytes) {
    for (int64_t chunk = int64_t(sf.pl.chunk_len) * 2; chunk < a.L && chunk < (int64_t(1) << 30);
         chunk *= 2) {
      o.carry = 2;
      o.chunk_len = int(chunk);
      if ((st = sf.prepare(a, o, nullptr)) != MAMBA_OK) return st;
      if (sf.bytes <= kNoAllocScratchBytes) break;
    }
  }
  if (sf.bytes > kNoAllocScratchBytes || sf.pl.K < 2) {
    o.carry = 1;
    o.chunk_len = 0;
    if ((st = sf.prepare(a, o, nullptr)) != MAMBA_OK) return st;
  }
  // the limit: what the sequential hand-off needs (counters, one flag and one
  // carried state per channel group) must fit the array
  if (sf.bytes > kNoAllocScratchBytes) return MAMBA_ERR_UNSUPPORTED;
  // The array keeps whatever the previous call left: run() clears the
  // counters and flags first; every other word is written before it is read.
  return sf.run(scratch, s, &launch_status);
}

}  // namespace

extern "C" mamba_status_t mamba_scan_fwd_noalloc(const void *u, const void *delta,
                                                 const float *delta_bias, const float *A,
                                                 const void *B, const void *C, const float *D,
                                                 const void *z, void *y, float *last_state,
                                                 int64_t batch, int64_t dim, int64_t L, int64_t N,
                                                 mamba_dtype_t dtype, mamba_stream_t stream) {
  mamba_status_t st = check_shape(batch, dim, L, N, dtype);
  if (st != MAMBA_OK) return st;
  Checker ck;
  if (cudaGetDevice(&ck.dev) != cudaSuccess) {
    cudaGetLastError();
    return MAMBA_ERR_CUDA;
  }
  const size_t es = dtype_size(dtype);
  const size_t nbdl = size_t(batch) * size_t(dim) * size_t(L);
  const size_t nbnl = size_t(batch) * size_t(N) * size_t(L);
  ck.buf(u, nbdl * es, es, true, false);
  ck.buf(delta, nbdl * es, es, true, false);
  ck.buf(z, nbdl * es, es, false, false);
  ck.buf(B, nbnl * es, es, true, false);
  ck.buf(C, nbnl * es, es, true, false);
  ck.buf(A, size_t(dim) * N * 4, 4, true, false);
  ck.buf(D, size_t(dim) * 4, 4, false, false);
  ck.buf(delta_bias, size_t(dim) * 4, 4, false, false);
  ck.buf(y, nbdl * es, es, true, true);
  ck.buf(last_state, size_t(batch) * dim * N * 4, 4, false, true);
  if (ck.st != MAMBA_OK) return ck.st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (batch == 0 || dim == 0) return MAMBA_OK;
  if (L == 0) {
    if (last_state && cudaMemsetAsync(last_state, 0, size_t(batch) * dim * N * 4, s) != cudaSuccess)
      return cuda_status();
    return MAMBA_OK;
  }
  FwdArgs a;
  a.u = u; a.delta = delta; a.z = z; a.B = B; a.C = C;
  a.bias = delta_bias; a.A = A; a.D = D; a.y = y; a.last_state = last_state;
  a.batch = batch; a.dim = dim; a.L = L; a.N = (int)N;
  // Shapes the staged kernels do not take use the one-thread-per-channel
  // kernel, which needs no scratch at all.
  if (!staged_supported(a, es)) return dispatch<FwdReferenceLauncher>(dtype, (int)N, a, s);
  unsigned char *scratch = nullptr;
  if ((st = noalloc_scratch(ck.dev, &scratch)) != MAMBA_OK) return st;
  if (dtype == MAMBA_BF16) {
    if (N <= 4) return noalloc_forward<__nv_bfloat16, 4>(a, scratch, s);
    if (N <= 8) return noalloc_forward<__nv_bfloat16, 8>(a, scratch, s);
    return noalloc_forward<__nv_bfloat16, 16>(a, scratch, s);
  }
  if (N <= 4) return noalloc_forward<float, 4>(a, scratch, s);
  if (N <= 8) return noalloc_forward<float, 8>(a, scratch, s);
  return noalloc_forward<float, 16>(a, scratch, s);
}
