// Small HBM-bound kernels shared by the entry points.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/kvb.h"

namespace kvb {

// out[h][ldOut*h + off + r] = ||X[h][xoff + r]||^2 * inv_h + add, r < n (uniform or per-head n_dev),
// X [H][ldX][d] of `dtype`.  One warp per row.
cudaError_t launch_row_terms(const void* X, kvb_dtype dtype, int H, long long ldX, int d, int n_uni,
                             const int* n_dev, int max_n, float inv_h, float add, float* out, long long ldOut,
                             cudaStream_t st);

}  // namespace kvb
