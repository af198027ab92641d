// DensityKV admit step: selection, eviction and compaction kernels
// (DensityKV App. B.1 "Online Bank Update", App. E default policy).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "kvb.h"

namespace kvb {

// One layer's bank arrays (slot-indexed, [H][M] or [H][M][d]) and the step's
// scratch.  Every pointer is device memory inside the bank workspace.
struct AdmitPlan {
  int H = 0, M = 0, N = 0, d = 0;
  kvb_dtype dtype = KVB_BF16;
  int row_bytes = 0;        // d * element size
  float tau = 2.f;
  int sync_heads = 1;
  int cand_order = KVB_ORDER_DISTURBANCE;
  int baselines = KVB_BASELINES_FIXED;
  int evict_order = KVB_EVICT_THRESHOLD_RATIO;
  const int* p_bound = nullptr;  // device: an outside bound on P (the other ranks' prefixes), or null
  // bank (this layer)
  void* K = nullptr;
  void* V = nullptr;
  int* ids = nullptr;
  float* rho = nullptr;
  float* rho0 = nullptr;
  uint16_t* aug = nullptr;  // [H][M][32] augmented rows of the keys (norm terms for the MMA)
  int* size = nullptr;      // [H]
  kvb_admit_stats* stats = nullptr;  // [H]
  // candidates (caller)
  const void* candK = nullptr;
  const void* candV = nullptr;
  const int* cand_ids = nullptr;
  // scratch
  const uint16_t* caug = nullptr;  // [H][Nmax][32] augmented candidate rows
  float* rhoB = nullptr;         // [H][Nmax]  density against the bank
  float* mean0 = nullptr;        // [H]
  int* feasible = nullptr;       // [H]
  int* P = nullptr;              // [H] admitted count
  int* adm_idx = nullptr;        // [H][Nmax] admitted candidate indices (ascending)
  void* EA = nullptr;            // [H][M + Nmax][d] evicted keys at [M - E, M), admitted at [M, M + P)
  uint16_t* EAaug = nullptr;     // [H][M + Nmax][32]
  int ldEA = 0;                  // M + Nmax
  int* EAoff = nullptr;          // [H] M - E_h
  int* EAcnt = nullptr;          // [H] E_h (pass 3a column count)
  float* proj = nullptr;         // [H][M]  sum over admitted of phi(c, i)
  int* ev_slot = nullptr;        // [H][M]  evicted slots (ascending)
  int* E = nullptr;              // [H] evicted count
  int* n_old = nullptr;          // [H] size before the update
  int* hole = nullptr;           // [H][M] evicted slots below the new size
  int* nhole = nullptr;          // [H]
  int* tail = nullptr;           // [H][M] surviving slots at or above the new size
  int* ntail = nullptr;          // [H]
  int* newp = nullptr;           // [H][M] admitted index living in a slot, -1 for old entries
  float* sub = nullptr;          // [H][M]  -sum over evicted of phi(i, e)
  float* coadm = nullptr;        // [H][Nmax] sum over co-admitted (c' != c) of phi(c, c')
  int ldN = 0;                   // Nmax
  int* status = nullptr;
};

cudaError_t launch_admit_count(const AdmitPlan& p, cudaStream_t st);
// out[0] = min(min_h feasible_h, M, N): the prefix this bank's heads allow
cudaError_t launch_feasible_min(const AdmitPlan& p, int* out, cudaStream_t st);
cudaError_t launch_admit_select(const AdmitPlan& p, cudaStream_t st);
cudaError_t launch_gather_admitted(const AdmitPlan& p, int maxP, cudaStream_t st);
cudaError_t launch_evict_select(const AdmitPlan& p, cudaStream_t st);
cudaError_t launch_gather_evicted(const AdmitPlan& p, cudaStream_t st);
cudaError_t launch_compact(const AdmitPlan& p, cudaStream_t st);
cudaError_t launch_finalize(const AdmitPlan& p, cudaStream_t st);

}  // namespace kvb
