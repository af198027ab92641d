// Device-side helpers shared by every kernel of the library.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace kvb {

// Record the first device error in the status word (0 = none).  Never traps.
__device__ __forceinline__ void latch_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// Programmatic dependent launch (kernels launched with launch_pdl): wait until
// the previous kernel on the stream has completed and its writes are visible;
// allow the next kernel to be scheduled.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Element access for the two storage types.
__device__ __forceinline__ float load_elem(const __nv_bfloat16* p, size_t i) { return __bfloat162float(p[i]); }
__device__ __forceinline__ float load_elem(const float* p, size_t i) { return p[i]; }

// Monotone map of a non-negative-or-any float to uint32 (ascending order kept).
__device__ __forceinline__ uint32_t float_key(float f) {
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Inverse of float_key.
__device__ __forceinline__ float key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ int warp_sum_int(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Rows are moved by groups of L = min(32, row_bytes / 16) lanes, one 16-byte
// word per lane per step: a warp moves 32/L rows at once, and each group strides
// over the rows of its head (row_bytes a multiple of 16 and L a power of two:
// 128, 256 or 512-byte rows).
struct RowGroup {
  int L, sub, first, stride;
};
__device__ __forceinline__ RowGroup row_group(int row_bytes) {
  RowGroup g;
  const int words = row_bytes / 16;
  g.L = words < 32 ? words : 32;
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  g.sub = t % g.L;
  g.first = t / g.L;
  g.stride = gridDim.x * blockDim.x / g.L;
  return g;
}
__device__ __forceinline__ void copy_row(void* dst, const void* src, int row_bytes, const RowGroup& g) {
  const uint4* s = static_cast<const uint4*>(src);
  uint4* d = static_cast<uint4*>(dst);
  for (int o = g.sub; o < row_bytes / 16; o += g.L) d[o] = s[o];
}

// K and V rows (and, for the group's lanes 0..3, a 64-byte augmented row) moved
// together: every load is issued before the first store, so a lane has all its
// words in flight at once (rows of at most 32 words of 16 bytes per lane group:
// 512 bytes).  Null pointers skip that row.
struct RowWords {
  uint4 k[2], v[2], a;
};
__device__ __forceinline__ void load_rows(RowWords& w, const void* k, const void* v, const void* aug, int row_bytes,
                                          const RowGroup& g) {
  const int words = row_bytes / 16;
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int o = g.sub + u * g.L;
    if (o < words) {
      if (k) w.k[u] = __ldg(static_cast<const uint4*>(k) + o);
      if (v) w.v[u] = __ldg(static_cast<const uint4*>(v) + o);
    }
  }
  if (aug && g.sub < 4) w.a = __ldg(static_cast<const uint4*>(aug) + g.sub);
}
__device__ __forceinline__ void store_rows(const RowWords& w, void* k, void* v, void* aug, int row_bytes,
                                           const RowGroup& g) {
  const int words = row_bytes / 16;
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int o = g.sub + u * g.L;
    if (o < words) {
      if (k) static_cast<uint4*>(k)[o] = w.k[u];
      if (v) static_cast<uint4*>(v)[o] = w.v[u];
    }
  }
  if (aug && g.sub < 4) static_cast<uint4*>(aug)[g.sub] = w.a;
}

}  // namespace kvb
