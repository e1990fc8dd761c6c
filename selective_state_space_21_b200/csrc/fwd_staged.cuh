// fwd_staged.cuh -- staged, chunked forward kernels (sm_100a).
#pragma once
#include "../../include/mamba_scan.h"
#include "common.cuh"

namespace mscan {

inline bool staged_supported(const FwdArgs &a, size_t es) { return false; }

template <typename T, int NM>
mamba_status_t staged_forward(const FwdArgs &a, int path, int chunk_len, cudaStream_t s) {
  return MAMBA_ERR_UNSUPPORTED;
}

}  // namespace mscan
