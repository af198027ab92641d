// Host-side helpers: status mapping, device properties, TMA descriptors and a
// bump carver for caller workspaces.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "kvb.h"

namespace kvb {

struct DeviceInfo {
  int device = -1;
  int n_sm = 0;
  int cc_major = 0;
  int cc_minor = 0;
};

// Properties of the current device (cached per device).  false if unavailable.
bool current_device(DeviceInfo* out);

// 3D tiled tensor map over a bf16 [heads][rows][d] buffer, box 64 x box_rows x 1,
// 128-byte swizzle, zero fill out of bounds.
bool make_tmap_bf16(CUtensorMap* m, const void* base, int d, long long rows, int heads, int box_rows);
// Tensor map over the augmented rows [heads][rows][32] bf16 (64 bytes per row),
// box 16 x box_rows x 1, 32-byte swizzle (one K=16 slice of an MMA operand).
bool make_tmap_aug(CUtensorMap* m, const void* base, long long rows, int heads, int box_rows);

// Every kernel launch of the library goes through one of these, constructed just
// before the launch in the same scope: it counts the launch and, while tracing is
// on, records a CUDA event pair around it on the launch stream (the destructor,
// run after the launch statement, records the second event).
class LaunchTrace {
 public:
  LaunchTrace(const char* kernel, cudaStream_t st);
  ~LaunchTrace();
  LaunchTrace(const LaunchTrace&) = delete;
  LaunchTrace& operator=(const LaunchTrace&) = delete;

 private:
  const char* kernel_;
  cudaStream_t st_;
  int slot_ = -1;
};

// Launch with programmatic dependent launch: the kernel's CTAs may be scheduled,
// and run their prologue, while the previous kernel on the stream is finishing.
// Every kernel launched this way executes pdl_wait() (kvb_device.cuh) before it
// touches global memory that earlier work on the stream writes or reads, so the
// stream's ordering is kept; it also calls pdl_trigger() to let its own
// successor be scheduled early.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

// CTAs per head of a row-moving kernel (256 threads, row_group lanes per row):
// enough for `rows` rows, capped so that the grid stays near one wave (about
// 1024 CTAs over all heads).
inline int mover_blocks(int rows, int row_bytes, int H) {
  const int words = row_bytes / 16;
  const int per_cta = 256 / (words < 32 ? words : 32);
  const int need = (rows + per_cta - 1) / per_cta;
  const int cap = 1024 / (H > 0 ? H : 1);
  return need < 1 ? 1 : (need < cap ? need : (cap < 1 ? 1 : cap));
}

inline kvb_status cuda_status(cudaError_t e) { return e == cudaSuccess ? KVB_OK : KVB_E_CUDA; }

// Bump allocation inside a caller workspace, 256-byte aligned pieces.
struct Carver {
  uintptr_t base = 0;
  size_t used = 0;
  explicit Carver(void* p = nullptr) : base(reinterpret_cast<uintptr_t>(p)) {}
  template <typename T>
  T* take(size_t count) {
    used = (used + 255) & ~size_t(255);
    T* p = reinterpret_cast<T*>(base + used);
    used += count * sizeof(T);
    return base ? p : nullptr;
  }
  size_t bytes() const { return (used + 255) & ~size_t(255); }
};

}  // namespace kvb
