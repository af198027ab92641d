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
                                uint16_t* __restrict__ out, long long ldOut, float* norm_max, float reg) {
  pdl_wait();
  pdl_trigger();
  __shared__ float s_max[32];
  const int h = blockIdx.y;
  const int n = n_dev ? n_dev[h] : n_uni;
  const int row_bytes = d * static_cast<int>(sizeof(T));
  const RowGroup g = row_group(row_bytes);
  float gmax = 0.f;
  // rows of at most 32 words of 16 bytes: one word per lane of a group (g.L = words).
  // Two rows per group in flight; the loop runs warp-uniformly (every lane
  // reaches the shuffles), a group whose row is past the end only skips its load
  // and store
  const int lane_group = (threadIdx.x & 31) / g.L;
  for (int r0 = g.first - lane_group; r0 < n; r0 += 2 * g.stride) {
    float acc[2] = {0.f, 0.f};
    uint4 u[2];
    bool live[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int r = r0 + lane_group + k * g.stride;
      live[k] = r < n;
      if (live[k] && g.sub < row_bytes / 16)
        u[k] = __ldg(reinterpret_cast<const uint4*>(X + (static_cast<long long>(h) * ldX + r) * d) + g.sub);
      else
        u[k] = make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const uint32_t q[4] = {u[k].x, u[k].y, u[k].z, u[k].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (sizeof(T) == 2) {
          const float lo = __uint_as_float(q[j] << 16), hi = __uint_as_float(q[j] & 0xFFFF0000u);
          acc[k] = fmaf(lo, lo, fmaf(hi, hi, acc[k]));
        } else {
          const float v = __uint_as_float(q[j]);
          acc[k] = fmaf(v, v, acc[k]);
        }
      }
      for (int o = g.L >> 1; o > 0; o >>= 1) acc[k] += __shfl_xor_sync(0xffffffffu, acc[k], o);
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      if (!live[k]) continue;
      gmax = fmaxf(gmax, acc[k]);
      // 32 entries: row form [hi, mid, lo, 1, 1, 1, rhi, rlo, 0...], column form
      // [1, 1, 1, hi, mid, lo, 1, 1, 0...];
      // lanes 0..3 of the group write one 16-byte word each
      if (g.sub >= 4) continue;
      const float nrm = -0.5f * acc[k];
      const __nv_bfloat16 bhi = __float2bfloat16_rn(nrm);
      const __nv_bfloat16 bmid = __float2bfloat16_rn(nrm - __bfloat162float(bhi));
      const __nv_bfloat16 blo = __float2bfloat16_rn(nrm - __bfloat162float(bhi) - __bfloat162float(bmid));
      const __nv_bfloat16 brh = __float2bfloat16_rn(reg);
      const __nv_bfloat16 brl = __float2bfloat16_rn(reg - __bfloat162float(brh));
      const uint32_t one = 0x3F80u;  // bf16 1.0
      const uint32_t hi = *reinterpret_cast<const uint16_t*>(&bhi), mid = *reinterpret_cast<const uint16_t*>(&bmid),
                     lo = *reinterpret_cast<const uint16_t*>(&blo);
      const uint32_t rh = *reinterpret_cast<const uint16_t*>(&brh), rl = *reinterpret_cast<const uint16_t*>(&brl);
      uint4 w = make_uint4(0u, 0u, 0u, 0u);
      if (g.sub == 0) w = make_uint4(hi | (mid << 16), lo | (one << 16), one | (one << 16), rh | (rl << 16));
      else if (g.sub == 2) w = make_uint4(one | (one << 16), one | (hi << 16), mid | (lo << 16), one | (one << 16));
      const int r = r0 + lane_group + k * g.stride;
      reinterpret_cast<uint4*>(out + (static_cast<long long>(h) * ldOut + r) * 32)[g.sub] = w;
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
                            int max_n, uint16_t* out, long long ldOut, float* norm_max, float reg, cudaStream_t st) {
  if (max_n <= 0 || H <= 0) return cudaSuccess;
  dim3 grid(mover_blocks(max_n, d * (dtype == KVB_BF16 ? 2 : 4), H), H);
  LaunchTrace trace("aug_rows_kernel", st);
  if (dtype == KVB_BF16)
    return launch_pdl(aug_rows_kernel<__nv_bfloat16>, grid, dim3(256), 0, st, static_cast<const __nv_bfloat16*>(X),
                      ldX, d, n_uni, n_dev, out, ldOut, norm_max, reg);
  return launch_pdl(aug_rows_kernel<float>, grid, dim3(256), 0, st, static_cast<const float*>(X), ldX, d, n_uni,
                    n_dev, out, ldOut, norm_max, reg);
}


}  // namespace kvb
