// FP8 E4M3 storage of the retained K/V (the Forcing-KV reading notes' FP8
// combination, read as the history held in E4M3): elementwise rounding and the
// conversions between the bf16 working copy and the E4M3 store (HBM-bound).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace kvb {

// out[i] = bf16(E4M3(in[i])) for n bf16 elements (round to nearest even,
// saturating at +-448; exact in bf16).  n a multiple of 8, both 16-byte aligned.
cudaError_t launch_round_e4m3(const void* in, void* out, size_t n, cudaStream_t st);

// E4M3 codes of the bf16 rows [0, size[h]) of every head: in [H][M][d] bf16,
// out [H][M][d] bytes.  d * 2 a multiple of 32.
cudaError_t launch_quant_rows(const void* in, void* out, int H, int M, int d, const int* size, cudaStream_t st);

// bf16 values of n E4M3 codes (n a multiple of 16, both 16-byte aligned).
cudaError_t launch_dequant(const void* in, void* out, size_t n, cudaStream_t st);

}  // namespace kvb
