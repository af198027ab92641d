// The augmented-row kernel shared by the entry points (HBM-bound).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "kvb.h"

namespace kvb {

// Augmented rows for the density MMA: for x = X[h][r] (r < n), with
// nrm = -||x||^2 / 2 split exactly into three bf16 parts (hi, mid, lo) and the
// constant `reg` split into two (rhi, rlo):
//   out[h][r][0..15]  = [hi, mid, lo, 1, 1, 1, rhi, rlo, 0 ...]   (row form, A operand)
//   out[h][r][16..31] = [1, 1, 1, hi, mid, lo, 1, 1, 0 ...]       (column form, B operand)
// so that an extra K=16 MMA step adds -(||a||^2 + ||b||^2)/2 + reg to a.b.  The
// density passes take reg = -eps h / 2, so the accumulator holds
// -(h/2) (||a - b||^2 / h + eps) for every pair.  If norm_max is not null it is
// raised to the largest ||x||^2 seen (atomic max, >= 0).
cudaError_t launch_aug_rows(const void* X, kvb_dtype dtype, int H, long long ldX, int d, int n_uni, const int* n_dev,
                            int max_n, uint16_t* out, long long ldOut, float* norm_max, float reg, cudaStream_t st);

}  // namespace kvb
