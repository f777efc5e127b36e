// Backward attention kernels for sm_100a (placeholder: filled in below the
// forward once it is verified).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include "attn.h"
#include "ptx.cuh"

namespace eta {

// Rows of the per-row statistics are padded to a multiple of this.
constexpr int kBwdRowPad = 128;

inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline size_t bwd_workspace_bytes(int B, int Hq, int N, int D) {
  const size_t rows = static_cast<size_t>(B) * Hq;
  const size_t npad = round_up(static_cast<size_t>(N), kBwdRowPad);
  return round_up(rows * N * D * 4, 256) + 2 * round_up(rows * npad * 4, 256);
}

inline attn_status_t launch_bwd(const attn_tensor_t&, const attn_tensor_t&, const attn_tensor_t&,
                                const attn_tensor_t&, const float*, const attn_tensor_t&,
                                const attn_tensor_t&, const attn_tensor_t&, const attn_tensor_t&,
                                int, int, int, int, int, bool, float, void*, int*,
                                unsigned long long, cudaStream_t) {
  return ATTN_ERR_UNSUPPORTED;
}

}  // namespace eta
