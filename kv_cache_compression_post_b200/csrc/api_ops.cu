// Operation-level C entry points (kvb_density, kvb_segment_cosine) and the
// status strings.
#include <cmath>
#include <cstring>

#include "gram.cuh"
#include "host_util.h"
#include "small_kernels.cuh"

using namespace kvb;

namespace {

struct DensityLayout {
  int* status = nullptr;
  uint16_t* rowAug = nullptr;
  uint16_t* colAug = nullptr;
  float* partial = nullptr;
  size_t bytes = 0;
};

DensityLayout density_layout(void* ws, int H, int nR, int nC, kvb_dtype dtype) {
  Carver c(ws);
  DensityLayout L;
  L.status = c.take<int>(64);
  if (dtype == KVB_BF16) {
    L.rowAug = c.take<uint16_t>(static_cast<size_t>(H) * nR * 32);
    L.colAug = c.take<uint16_t>(static_cast<size_t>(H) * nC * 32);
    L.partial = c.take<float>(static_cast<size_t>(16) * H * nR);
  }
  L.bytes = c.bytes();
  return L;
}

bool density_args_ok(int32_t heads, int32_t n_rows, int32_t n_cols, int32_t head_dim, kvb_dtype dtype) {
  if (heads < 1 || heads > 64 || n_rows < 0 || n_cols < 0) return false;
  if (dtype != KVB_BF16 && dtype != KVB_F32) return false;
  if (head_dim < 1 || head_dim > 256) return false;
  return true;
}

}  // namespace

extern "C" {

const char* kvb_status_string(kvb_status st) {
  switch (st) {
    case KVB_OK: return "ok";
    case KVB_E_INVAL: return "invalid argument";
    case KVB_E_WORKSPACE: return "workspace missing, too small or misaligned";
    case KVB_E_CUDA: return "CUDA runtime error";
    case KVB_E_DEVICE_TIMEOUT: return "device-side wait timed out";
    case KVB_E_DEVICE_BOUNDS: return "device-side bounds check refused an access";
    case KVB_E_STATE: return "call not valid for this bank";
    case KVB_E_UNSUPPORTED: return "configuration not supported";
  }
  return "unknown status";
}

size_t kvb_density_workspace_size(int32_t heads, int32_t n_rows, int32_t n_cols, int32_t head_dim,
                                  kvb_dtype dtype) {
  if (!density_args_ok(heads, n_rows, n_cols, head_dim, dtype)) return 0;
  return density_layout(nullptr, heads, n_rows, n_cols, dtype).bytes;
}

kvb_status kvb_density(const void* rows, int32_t n_rows, const void* cols, int32_t n_cols, int32_t heads,
                       int32_t head_dim, kvb_dtype dtype, float dist_scale, float eps, float s,
                       int32_t exclude_diagonal, float* out, void* workspace, size_t workspace_bytes,
                       void* stream) {
  if (!density_args_ok(heads, n_rows, n_cols, head_dim, dtype)) return KVB_E_INVAL;
  if (dtype == KVB_BF16 && head_dim != 64 && head_dim != 128) return KVB_E_UNSUPPORTED;
  if (!(eps > 0.f) || !std::isfinite(eps) || !std::isfinite(s) || s < 0.f || !(dist_scale >= 0.f))
    return KVB_E_INVAL;
  if (exclude_diagonal && n_rows != n_cols) return KVB_E_INVAL;
  if (n_rows == 0) return KVB_OK;
  if (!rows || !out || (n_cols > 0 && !cols)) return KVB_E_INVAL;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return KVB_E_WORKSPACE;
  const DensityLayout L = density_layout(workspace, heads, n_rows, n_cols, dtype);
  if (workspace_bytes < L.bytes) return KVB_E_WORKSPACE;
  DeviceInfo dev;
  if (!current_device(&dev)) return KVB_E_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const float h = dist_scale > 0.f ? dist_scale : static_cast<float>(head_dim);
  // status word and the largest key norm seen (status[1]) start at zero
  if (cudaMemsetAsync(L.status, 0, 2 * sizeof(int), st) != cudaSuccess) return KVB_E_CUDA;
  float* norm_max = reinterpret_cast<float*>(L.status + 1);

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
  a.status = L.status;

  if (dtype == KVB_F32) {
    a.R32 = static_cast<const float*>(rows);
    a.C32 = static_cast<const float*>(cols);
    a.ldR = n_rows;
    a.ldC = n_cols;
    a.partial = out;
    a.ldOut = n_rows;
    return cuda_status(launch_gram_f32(a, st));
  }
  if (n_cols == 0) return cuda_status(cudaMemsetAsync(out, 0, sizeof(float) * heads * n_rows, st));
  cudaError_t e =
      launch_aug_rows(rows, dtype, heads, n_rows, head_dim, n_rows, nullptr, n_rows, L.rowAug, n_rows, norm_max, -0.5f * eps * h, st);
  if (e == cudaSuccess)
    e = launch_aug_rows(cols, dtype, heads, n_cols, head_dim, n_cols, nullptr, n_cols, L.colAug, n_cols, norm_max, -0.5f * eps * h, st);
  a.norm_max = norm_max;
  if (e != cudaSuccess) return KVB_E_CUDA;
  GramMaps m;
  if (!make_tmap_bf16(&m.R, rows, head_dim, n_rows, heads, 128) ||
      !make_tmap_bf16(&m.C, cols, head_dim, n_cols, heads, kGramColTile) || !make_tmap_aug(&m.Ra, L.rowAug, n_rows, heads, 128) ||
      !make_tmap_aug(&m.Ca, L.colAug, n_cols, heads, kGramColTile))
    return KVB_E_INVAL;
  a.partial = L.partial;
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

}  // extern "C"
