// Attention of the current chunk's queries over a ragged per-head list of K/V
// segments [sink | history | window] (DensityKV Fig. 2: retained states are read
// by native attention together with the local window; Forcing-KV §3.3/§3.5).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace kvb {

constexpr int kAttnMaxSeg = 5;
// Persistent grid cap of the bf16 kernel (>= the SM count of a B200); the scratch
// below is sized for it.
constexpr int kAttnMaxCtas = 160;

// Scratch of the bf16 kernel: partial results of query tiles whose key range is
// split between CTAs, and one arrival counter per (query-tile pair, tile).
inline size_t attend_partial_floats(int d) { return static_cast<size_t>(4) * kAttnMaxCtas * (128 * d + 256); }
inline size_t attend_counter_count(int heads, int max_queries) {
  const int nqt = (max_queries + 127) / 128;
  return static_cast<size_t>(heads) * ((nqt + 1) / 2) * 2;
}

// One K/V source: [H][ld][d] buffers; per head a start row and a length, each
// uniform or from a device array indexed by head.
struct AttnSeg {
  const void* K = nullptr;
  const void* V = nullptr;
  long long ld = 0;
  int len_uni = 0;
  const int* len_dev = nullptr;
  int off_uni = 0;
  const int* off_dev = nullptr;
};

struct AttnArgs {
  int H = 0, d = 0, Nq = 0;
  float scale = 0.f;            // 1/sqrt(d)
  int nseg = 0;
  AttnSeg seg[kAttnMaxSeg];
  const void* Q = nullptr;      // [H][Nq][d]
  void* O = nullptr;            // [H][Nq][d]
  float* lse = nullptr;         // [H][Nq] or null
  int* status = nullptr;
  // bf16 path scratch (attend_partial_floats / attend_counter_count entries)
  float* part = nullptr;
  unsigned long long* cnt = nullptr;
  unsigned int epoch = 1;       // nonzero, different on consecutive launches
};

struct AttnMaps {
  CUtensorMap q;
  CUtensorMap k[kAttnMaxSeg];
  CUtensorMap v[kAttnMaxSeg];
};

// bf16 tcgen05 path (d = 64 or 128); builds the tensor maps itself.
cudaError_t launch_attend_bf16(const AttnArgs& a, cudaStream_t st);
// f32 CUDA-core path (small problems).
cudaError_t launch_attend_f32(const AttnArgs& a, cudaStream_t st);

size_t attend_smem_bytes(int d);

}  // namespace kvb
