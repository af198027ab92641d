// kvb_density_noalloc: kvb_density for callers that cannot allocate device memory.
//
// Some callers cannot hand the library a workspace: a plugin inside a host
// application whose allocator owns all device memory and forbids allocations
// outside it, or a latency-critical loop that must never pay for an allocation
// (cudaMalloc may synchronise the device).  For them this entry point keeps its
// scratch (the device status word, per-row norm terms and the per-CTA partial
// sums of the density Gram) in one fixed, file-scope device array instead of a
// caller workspace.  It runs exactly the kernels of kvb_density.
//
// Properties a caller must know:
//  * The array is kNoAllocScratchBytes (4 MiB) and is part of the library image:
//    every GPU that loads the library holds it until the process exits.
//  * Sizes whose scratch does not fit are rejected with KVB_E_WORKSPACE before
//    anything is launched (see kvb_density_noalloc in kvb.h for the formula).
//  * The first call on a device looks up the array's device address with that
//    device current; make that first call before any stream capture begins.  The
//    address is cached for the life of the process: a cudaDeviceReset of that
//    device makes it stale, and the entry point must not be used there again.
//  * Every call on a device shares the one array, which keeps the last call's
//    contents.  Calls whose kernels overlap on the GPU (different streams without
//    ordering between them) race on it; serialise them.
//  * Device-side failures (a bounded wait that gave up) are latched into the
//    caller's `status_out` word when one is passed (zeroed by the call); without
//    one they land in a status word inside the array that nothing reads back.
#include <cmath>
#include <mutex>

#include "gram.cuh"
#include "host_util.h"
#include "small_kernels.cuh"

using namespace kvb;

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of g_noalloc_scratch on the current device (looked up once per
// device, with that device current).  In host code the symbol's name is only a
// host-side handle; kernels must be given this address instead.
void* scratch_address(int dev) {
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return nullptr;
    g_scratch_ptr[dev] = p;
  }
  return g_scratch_ptr[dev];
}

struct NoAllocLayout {
  size_t status = 0, rowAug = 0, colAug = 0, partial = 0, bytes = 0;
};

NoAllocLayout noalloc_layout(int H, int nR, int nC) {
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  NoAllocLayout L;
  L.status = 0;
  L.rowAug = up(L.status + 256);
  L.colAug = up(L.rowAug + 64 * static_cast<size_t>(H) * nR);
  L.partial = up(L.colAug + 64 * static_cast<size_t>(H) * nC);
  L.bytes = up(L.partial + sizeof(float) * static_cast<size_t>(16) * H * nR);
  return L;
}

}  // namespace

extern "C" kvb_status kvb_density_noalloc(const void* rows, int32_t n_rows, const void* cols, int32_t n_cols,
                                          int32_t heads, int32_t head_dim, kvb_dtype dtype, float dist_scale,
                                          float eps, float s, int32_t exclude_diagonal, float* out,
                                          int32_t* status_out, void* stream) {
  if (heads < 1 || heads > 64 || n_rows < 0 || n_cols < 0) return KVB_E_INVAL;
  if (dtype != KVB_BF16) return KVB_E_UNSUPPORTED;
  if (head_dim != 64 && head_dim != 128) return KVB_E_UNSUPPORTED;
  if (!(eps > 0.f) || !std::isfinite(eps) || !std::isfinite(s) || s < 0.f || !(dist_scale >= 0.f))
    return KVB_E_INVAL;
  if (exclude_diagonal && n_rows != n_cols) return KVB_E_INVAL;
  const NoAllocLayout L = noalloc_layout(heads, n_rows, n_cols);
  if (L.bytes > kNoAllocScratchBytes) return KVB_E_WORKSPACE;
  if (n_rows == 0) return KVB_OK;
  if (!rows || !out || (n_cols > 0 && !cols)) return KVB_E_INVAL;
  DeviceInfo dev;
  if (!current_device(&dev) || dev.device >= kMaxDevices) return KVB_E_CUDA;
  char* base = static_cast<char*>(scratch_address(dev.device));
  if (!base) return KVB_E_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int* status = status_out ? status_out : reinterpret_cast<int*>(base + L.status);
  uint16_t* rowAug = reinterpret_cast<uint16_t*>(base + L.rowAug);
  uint16_t* colAug = reinterpret_cast<uint16_t*>(base + L.colAug);
  // the status word is the only piece that must start at zero on every call (the
  // augmented rows and the partials are written in full before they are read)
  if (cudaMemsetAsync(status, 0, sizeof(int), st) != cudaSuccess) return KVB_E_CUDA;
  // the largest key norm of this call (decides whether t >= eps must be clamped)
  float* norm_max = reinterpret_cast<float*>(base + L.status + 4);
  if (cudaMemsetAsync(norm_max, 0, sizeof(float), st) != cudaSuccess) return KVB_E_CUDA;
  if (n_cols == 0) return cuda_status(cudaMemsetAsync(out, 0, sizeof(float) * heads * n_rows, st));

  const float h = dist_scale > 0.f ? dist_scale : static_cast<float>(head_dim);
  cudaError_t e =
      launch_aug_rows(rows, dtype, heads, n_rows, head_dim, n_rows, nullptr, n_rows, rowAug, n_rows, norm_max, -0.5f * eps * h, st);
  if (e == cudaSuccess)
    e = launch_aug_rows(cols, dtype, heads, n_cols, head_dim, n_cols, nullptr, n_cols, colAug, n_cols, norm_max, -0.5f * eps * h, st);
  if (e != cudaSuccess) return KVB_E_CUDA;
  GramMaps m;
  if (!make_tmap_bf16(&m.R, rows, head_dim, n_rows, heads, 128) ||
      !make_tmap_bf16(&m.C, cols, head_dim, n_cols, heads, kGramColTile) || !make_tmap_aug(&m.Ra, rowAug, n_rows, heads, 128) ||
      !make_tmap_aug(&m.Ca, colAug, n_cols, heads, kGramColTile))
    return KVB_E_INVAL;
  GramArgs a;
  a.H = heads;
  a.d = head_dim;
  a.rows.n_uni = n_rows;
  a.cols.n_uni = n_cols;
  a.use_diag = exclude_diagonal ? 1 : 0;
  a.diag_uni = 0;
  a.kscale = -2.f / h;
  a.eps = eps;
  a.s = s;
  a.max_rows = n_rows;
  a.status = status;
  a.norm_max = norm_max;
  a.partial = reinterpret_cast<float*>(base + L.partial);
  a.ldOut = n_rows;
  gram_plan(a, (n_cols + kGramColTile - 1) / kGramColTile, dev.n_sm);
  m.R2 = m.R;  // no alternate operands
  m.C2 = m.C;
  m.Ra2 = m.Ra;
  m.Ca2 = m.Ca;
  e = launch_gram_bf16(a, m, st);
  if (e == cudaSuccess) e = launch_gram_reduce(a, out, n_rows, st);
  return cuda_status(e);
}
