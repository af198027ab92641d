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

template <typename T>
__global__ void aug_rows_kernel(const T* __restrict__ X, long long ldX, int d, int n_uni, const int* n_dev,
                                uint16_t* __restrict__ out, long long ldOut, float* norm_max) {
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
  if (norm_max && lane == 0) atomicMax(reinterpret_cast<int*>(norm_max), __float_as_int(acc));
  const float nrm = -0.5f * acc;
  const __nv_bfloat16 hi = __float2bfloat16_rn(nrm);
  const __nv_bfloat16 mid = __float2bfloat16_rn(nrm - __bfloat162float(hi));
  const __nv_bfloat16 lo = __float2bfloat16_rn(nrm - __bfloat162float(hi) - __bfloat162float(mid));
  const __nv_bfloat16 one = __float2bfloat16_rn(1.f), zero = __float2bfloat16_rn(0.f);
  __nv_bfloat16 v = zero;
  const int c = lane & 15;
  const bool colform = lane >= 16;
  if (c < 3) v = colform ? one : (c == 0 ? hi : (c == 1 ? mid : lo));
  else if (c < 6) v = colform ? (c == 3 ? hi : (c == 4 ? mid : lo)) : one;
  out[(static_cast<long long>(h) * ldOut + r) * 32 + lane] = *reinterpret_cast<uint16_t*>(&v);
}

}  // namespace

cudaError_t launch_aug_rows(const void* X, kvb_dtype dtype, int H, long long ldX, int d, int n_uni, const int* n_dev,
                            int max_n, uint16_t* out, long long ldOut, float* norm_max, cudaStream_t st) {
  if (max_n <= 0 || H <= 0) return cudaSuccess;
  dim3 grid((max_n + 7) / 8, H);
  LaunchTrace trace("aug_rows_kernel", st);
  if (dtype == KVB_BF16)
    aug_rows_kernel<<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(X), ldX, d, n_uni, n_dev, out, ldOut,
                                          norm_max);
  else
    aug_rows_kernel<<<grid, 256, 0, st>>>(static_cast<const float*>(X), ldX, d, n_uni, n_dev, out, ldOut, norm_max);
  return cudaGetLastError();
}

cudaError_t launch_row_terms(const void* X, kvb_dtype dtype, int H, long long ldX, int d, int n_uni,
                             const int* n_dev, int max_n, float inv_h, float add, float* out, long long ldOut,
                             cudaStream_t st) {
  if (max_n <= 0 || H <= 0) return cudaSuccess;
  dim3 grid((max_n + 7) / 8, H);
  LaunchTrace trace("row_terms_kernel", st);
  if (dtype == KVB_BF16)
    row_terms_kernel<<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(X), ldX, d, n_uni, n_dev, inv_h, add,
                                           out, ldOut);
  else
    row_terms_kernel<<<grid, 256, 0, st>>>(static_cast<const float*>(X), ldX, d, n_uni, n_dev, inv_h, add, out,
                                           ldOut);
  return cudaGetLastError();
}

}  // namespace kvb
