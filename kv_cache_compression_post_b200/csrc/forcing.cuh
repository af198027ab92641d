// Forcing-KV hybrid prune kernels (Forcing-KV reading notes §3.3, §3.4, §3.5).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "kvb.h"

namespace kvb {

struct SegGeom {
  int frame_h = 0, frame_w = 0, seg_h = 0, seg_w = 0;
  int F = 0, seg_rows = 0, seg_cols = 0, n_seg = 0;
};

// sim[h][t][j] = mean over tokens p of segment j of cos(K[h][t*F + p], succ[h][t][p]),
// succ = frame t+1 of K, or nextK for t = n_frames-1.  Heads with bit h of
// skip_mask set are not computed.
cudaError_t launch_seg_cosine(const void* K, const void* nextK, kvb_dtype dtype, int H, int n_frames, int d,
                              const SegGeom& g, unsigned long long skip_mask, float* sim, cudaStream_t st);
// same, with head stride ld_sim in the output (sim[h*ld_sim + t*n_seg + j])
cudaError_t launch_seg_cosine_ld(const void* K, const void* nextK, kvb_dtype dtype, int H, int n_frames, int d,
                                 const SegGeom& g, unsigned long long skip_mask, float* sim, int ld_sim,
                                 cudaStream_t st);

// Most (frame, segment) pairs one call may rank together (KVB_BOTTOMK_CALL).
constexpr int kPruneMaxPairs = 4096;

// One layer's Forcing-KV state and the prune step's scratch.
struct PrunePlan {
  int H = 0, d = 0, n_frames = 0, hist_frames = 0, ring_cap = 0, keep = 0, row_bytes = 0;
  int scope = KVB_BOTTOMK_FRAME;  // kvb_bottomk_scope; `keep` counts segments per frame or pairs per call
  SegGeom g;
  unsigned long long static_mask = 0;
  const void* newK = nullptr;
  const void* newV = nullptr;
  const int* new_ids = nullptr;
  const float* sims = nullptr;     // [H][max_new_frames][n_seg]
  const int* seg_tok = nullptr;    // [n_seg + 1]
  int* plan = nullptr;             // [H][max_new_frames * F][2] (source row, ring position)
  int* plan_n = nullptr;           // [H]
  int* keep_list = nullptr;        // [H][max_new_frames][n_seg]
  int ld_plan = 0;                 // max_new_frames * F
  int ld_sims = 0;                 // max_new_frames * n_seg
  // state (this layer)
  void* tK = nullptr;
  void* tV = nullptr;
  int* tids = nullptr;
  int* tlen = nullptr;
  void* rK = nullptr;
  void* rV = nullptr;
  int* rids = nullptr;
  int* fstart = nullptr;
  int* fcount = nullptr;
  int* rstate = nullptr;
  int* aseg = nullptr;             // [4][H]
  kvb_admit_stats* stats = nullptr;
  int* status = nullptr;
};

cudaError_t launch_prune_plan(const PrunePlan& p, cudaStream_t st);
cudaError_t launch_prune_gather(const PrunePlan& p, cudaStream_t st);

}  // namespace kvb
