#include <cuda_bf16.h>

#include "host_util.h"
#include "kvb_device.cuh"
#include "small_kernels.cuh"

namespace kvb {
namespace {

// Rows are read by lane groups (row_group: 16-byte words, several rows per warp,
// rows strided over the grid); the largest ||x||^2 seen by the CTA goes to
// norm_max with a single atomic (per-row atomics on one word serialise).
template <typename T>
__global__ void aug_rows_kernel(const T* __restrict__ X, long long ldX, int d, int n_uni, const int* n_dev,
                                uint16_t* __restrict__ out, long long ldOut, float* norm_max) {
  pdl_wait();
  pdl_trigger();
  __shared__ float s_max[32];
  const int h = blockIdx.y;
  const int n = n_dev ? n_dev[h] : n_uni;
  const int row_bytes = d * static_cast<int>(sizeof(T));
  const RowGroup g = row_group(row_bytes);
  const __nv_bfloat16 one = __float2bfloat16_rn(1.f), zero = __float2bfloat16_rn(0.f);
  float gmax = 0.f;
  // the loop runs warp-uniformly (every lane reaches the shuffles); a group whose
  // row is past the end only skips its loads and stores
  const int lane_group = (threadIdx.x & 31) / g.L;
  for (int r0 = g.first - lane_group; r0 < n; r0 += g.stride) {
    const int r = r0 + lane_group;
    const bool live = r < n;
    float acc = 0.f;
    if (live) {
      const uint4* x = reinterpret_cast<const uint4*>(X + (static_cast<long long>(h) * ldX + r) * d);
      for (int w = g.sub; w < row_bytes / 16; w += g.L) {
        const uint4 u = __ldg(x + w);
        const uint32_t q[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          if (sizeof(T) == 2) {
            const float lo = __uint_as_float(q[k] << 16), hi = __uint_as_float(q[k] & 0xFFFF0000u);
            acc = fmaf(lo, lo, fmaf(hi, hi, acc));
          } else {
            const float v = __uint_as_float(q[k]);
            acc = fmaf(v, v, acc);
          }
        }
      }
    }
    for (int o = g.L >> 1; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (!live) continue;
    gmax = fmaxf(gmax, acc);
    // 32 entries: row form [hi, mid, lo, 1, 1, 1, 0...], column form [1, 1, 1, hi, mid, lo, 0...]
    const float nrm = -0.5f * acc;
    const __nv_bfloat16 hi = __float2bfloat16_rn(nrm);
    const __nv_bfloat16 mid = __float2bfloat16_rn(nrm - __bfloat162float(hi));
    const __nv_bfloat16 lo = __float2bfloat16_rn(nrm - __bfloat162float(hi) - __bfloat162float(mid));
    for (int e = g.sub; e < 32; e += g.L) {
      const int c = e & 15;
      const bool colform = e >= 16;
      __nv_bfloat16 v = zero;
      if (c < 3) v = colform ? one : (c == 0 ? hi : (c == 1 ? mid : lo));
      else if (c < 6) v = colform ? (c == 3 ? hi : (c == 4 ? mid : lo)) : one;
      out[(static_cast<long long>(h) * ldOut + r) * 32 + e] = *reinterpret_cast<uint16_t*>(&v);
    }
  }
  if (!norm_max) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int o = 16; o > 0; o >>= 1) gmax = fmaxf(gmax, __shfl_xor_sync(0xffffffffu, gmax, o));
  if (lane == 0) s_max[warp] = gmax;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = 0.f;
    for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) m = fmaxf(m, s_max[i]);
    if (m > 0.f) atomicMax(reinterpret_cast<int*>(norm_max), __float_as_int(m));
  }
}

}  // namespace

cudaError_t launch_aug_rows(const void* X, kvb_dtype dtype, int H, long long ldX, int d, int n_uni, const int* n_dev,
                            int max_n, uint16_t* out, long long ldOut, float* norm_max, cudaStream_t st) {
  if (max_n <= 0 || H <= 0) return cudaSuccess;
  dim3 grid(mover_blocks(max_n, d * (dtype == KVB_BF16 ? 2 : 4), H), H);
  LaunchTrace trace("aug_rows_kernel", st);
  if (dtype == KVB_BF16)
    return launch_pdl(aug_rows_kernel<__nv_bfloat16>, grid, dim3(256), 0, st, static_cast<const __nv_bfloat16*>(X),
                      ldX, d, n_uni, n_dev, out, ldOut, norm_max);
  return launch_pdl(aug_rows_kernel<float>, grid, dim3(256), 0, st, static_cast<const float*>(X), ldX, d, n_uni,
                    n_dev, out, ldOut, norm_max);
}


}  // namespace kvb
