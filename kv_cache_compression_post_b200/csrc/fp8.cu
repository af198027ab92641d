// FP8 E4M3 conversions for an E4M3 K/V store (see fp8.cuh).  Every kernel moves
// 16-byte words with a grid-stride loop over about one wave of CTAs.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "fp8.cuh"
#include "host_util.h"
#include "kvb_device.cuh"

namespace kvb {
namespace {

constexpr int kThreads = 256;

// two bf16 (one 32-bit word) -> two E4M3 codes (16 bits)
__device__ __forceinline__ uint32_t to_e4m3x2(uint32_t w) {
  __nv_bfloat162_raw r;
  r.x = static_cast<unsigned short>(w & 0xFFFFu);
  r.y = static_cast<unsigned short>(w >> 16);
  return static_cast<uint32_t>(__nv_cvt_bfloat16raw2_to_fp8x2(r, __NV_SATFINITE, __NV_E4M3));
}

// two E4M3 codes -> two bf16 (exact: every E4M3 value is a half and a bf16)
__device__ __forceinline__ uint32_t from_e4m3x2(uint32_t c) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(c & 0xFFFFu), __NV_E4M3);
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
  const __nv_bfloat162 b = __floats2bfloat162_rn(f.x, f.y);
  return *reinterpret_cast<const uint32_t*>(&b);
}

__global__ void round_e4m3_kernel(const uint4* __restrict__ in, uint4* __restrict__ out, size_t nvec) {
  pdl_wait();
  pdl_trigger();
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < nvec;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const uint4 v = in[i];
    out[i] = make_uint4(from_e4m3x2(to_e4m3x2(v.x)), from_e4m3x2(to_e4m3x2(v.y)), from_e4m3x2(to_e4m3x2(v.z)),
                        from_e4m3x2(to_e4m3x2(v.w)));
  }
}

// one thread per 16 elements (32 bytes of bf16 in, 16 bytes of codes out)
__global__ void quant_rows_kernel(const uint4* __restrict__ in, uint4* __restrict__ out, int M, int words_per_row,
                                  const int* __restrict__ size) {
  pdl_wait();
  pdl_trigger();
  const int h = blockIdx.y;
  const int n = min(max(size[h], 0), M);
  const size_t per_head = static_cast<size_t>(M) * words_per_row;
  const size_t nw = static_cast<size_t>(n) * words_per_row;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < nw;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t k = h * per_head + i;
    const uint4 a = in[2 * k], b = in[2 * k + 1];
    out[k] = make_uint4(to_e4m3x2(a.x) | (to_e4m3x2(a.y) << 16), to_e4m3x2(a.z) | (to_e4m3x2(a.w) << 16),
                        to_e4m3x2(b.x) | (to_e4m3x2(b.y) << 16), to_e4m3x2(b.z) | (to_e4m3x2(b.w) << 16));
  }
}

__global__ void dequant_kernel(const uint4* __restrict__ in, uint4* __restrict__ out, size_t nvec) {
  pdl_wait();
  pdl_trigger();
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < nvec;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const uint4 c = in[i];
    out[2 * i] = make_uint4(from_e4m3x2(c.x), from_e4m3x2(c.x >> 16), from_e4m3x2(c.y), from_e4m3x2(c.y >> 16));
    out[2 * i + 1] = make_uint4(from_e4m3x2(c.z), from_e4m3x2(c.z >> 16), from_e4m3x2(c.w), from_e4m3x2(c.w >> 16));
  }
}

int wave_blocks(size_t items) {
  DeviceInfo dev;
  const int sms = current_device(&dev) ? dev.n_sm : 148;
  const size_t need = (items + kThreads - 1) / kThreads;
  const size_t cap = static_cast<size_t>(sms) * 8;
  return static_cast<int>(need < 1 ? 1 : (need < cap ? need : cap));
}

}  // namespace

cudaError_t launch_round_e4m3(const void* in, void* out, size_t n, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  if (n % 8 != 0) return cudaErrorInvalidValue;
  LaunchTrace trace("round_e4m3_kernel", st);
  return launch_pdl(round_e4m3_kernel, dim3(wave_blocks(n / 8)), dim3(kThreads), 0, st, static_cast<const uint4*>(in),
                    static_cast<uint4*>(out), n / 8);
}

cudaError_t launch_quant_rows(const void* in, void* out, int H, int M, int d, const int* size, cudaStream_t st) {
  if (H <= 0 || M <= 0) return cudaSuccess;
  if (d % 16 != 0) return cudaErrorInvalidValue;
  const int wpr = d / 16;
  const int bx = (wave_blocks(static_cast<size_t>(M) * wpr * H) + H - 1) / H;
  LaunchTrace trace("quant_rows_kernel", st);
  return launch_pdl(quant_rows_kernel, dim3(bx < 1 ? 1 : bx, H), dim3(kThreads), 0, st,
                    static_cast<const uint4*>(in), static_cast<uint4*>(out), M, wpr, size);
}

cudaError_t launch_dequant(const void* in, void* out, size_t n, cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  if (n % 16 != 0) return cudaErrorInvalidValue;
  LaunchTrace trace("dequant_kernel", st);
  return launch_pdl(dequant_kernel, dim3(wave_blocks(n / 16)), dim3(kThreads), 0, st, static_cast<const uint4*>(in),
                    static_cast<uint4*>(out), n / 16);
}

}  // namespace kvb
