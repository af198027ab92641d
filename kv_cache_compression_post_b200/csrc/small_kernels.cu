#include <cuda_bf16.h>

#include "host_util.h"
#include "kvb_device.cuh"
#include "small_kernels.cuh"

namespace kvb {
namespace {

template <typename T>
__global__ void row_terms_kernel(const T* __restrict__ X, long long ldX, int d, int n_uni, const int* n_dev,
                                 float inv_h, float add, float* __restrict__ out, long long ldOut) {
  const int h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * (blockDim.x >> 5) + warp;
  const int n = n_dev ? n_dev[h] : n_uni;
  if (r >= n) return;
  const T* x = X + (static_cast<long long>(h) * ldX + r) * d;
  float acc = 0.f;
  for (int k = lane; k < d; k += 32) {
    const float v = load_elem(x, k);
    acc = fmaf(v, v, acc);
  }
  acc = warp_sum(acc);
  if (lane == 0) out[static_cast<long long>(h) * ldOut + r] = fmaf(acc, inv_h, add);
}

}  // namespace

cudaError_t launch_row_terms(const void* X, kvb_dtype dtype, int H, long long ldX, int d, int n_uni,
                             const int* n_dev, int max_n, float inv_h, float add, float* out, long long ldOut,
                             cudaStream_t st) {
  if (max_n <= 0 || H <= 0) return cudaSuccess;
  dim3 grid((max_n + 7) / 8, H);
  note_launch();
  if (dtype == KVB_BF16)
    row_terms_kernel<<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(X), ldX, d, n_uni, n_dev, inv_h, add,
                                           out, ldOut);
  else
    row_terms_kernel<<<grid, 256, 0, st>>>(static_cast<const float*>(X), ldX, d, n_uni, n_dev, inv_h, add, out,
                                           ldOut);
  return cudaGetLastError();
}

}  // namespace kvb
