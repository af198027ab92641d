// Host-side bank object: where every array of the bank lives in the caller's
// workspace.
#pragma once

#include <cstddef>
#include <cstdint>

#include "kvb.h"
#include "host_util.h"

struct kvb_bank {
  kvb_config cfg;
  void* ws = nullptr;
  size_t ws_bytes = 0;
  int elem = 2;             // bytes per K/V element
  int row_bytes = 0;        // d * elem
  float h = 0.f;            // distance scale
  int F = 0;                // tokens per frame (Forcing-KV)
  int n_seg = 0;            // segments per frame (Forcing-KV)
  int ring_cap = 0;         // tokens a dynamic head's FIFO can hold
  int* status = nullptr;
  // attention scratch (bf16 path): split-unit partials and arrival counters
  float* attn_part = nullptr;
  unsigned long long* attn_cnt = nullptr;
  unsigned int attn_epoch = 0;  // launches so far (the kernel's epoch tag, never 0)

  // ---- DensityKV, per layer: base pointers of layer 0 and strides
  char* K = nullptr;        // [L][H][M][d]; E4M3 storage: the bf16 working copy of one layer, [H][M][d]
  char* V = nullptr;
  uint8_t* K8 = nullptr;    // E4M3 storage: [L][H][M][d] codes (null otherwise)
  uint8_t* V8 = nullptr;
  char* candQ = nullptr;    // E4M3 storage: the step's candidates rounded to E4M3, [2][H][Nmax][d] bf16 (K, V)
  int work_layer = -1;      // E4M3 storage: the layer the working copy holds (-1: none)
  int* ids = nullptr;       // [L][H][M]
  float* rho = nullptr;
  float* rho0 = nullptr;
  uint16_t* aug = nullptr;  // [L][H][M][32] augmented rows of the bank keys
  int* size = nullptr;      // [L][H]
  kvb_admit_stats* stats = nullptr;  // [L][H]

  // ---- DensityKV scratch (shared by layers)
  int ldN = 0, ldEA = 0, ldPart = 0;
  uint16_t* caug = nullptr; // [H][Nmax][32] augmented candidate rows
  float* rhoB = nullptr;
  float* mean0 = nullptr;
  int* feasible = nullptr;
  int* P = nullptr;
  int* E = nullptr;
  int* n_old = nullptr;
  int* nhole = nullptr;
  int* ntail = nullptr;
  int* EAoff = nullptr;
  int* EAcnt = nullptr;
  int* adm_idx = nullptr;
  char* EA = nullptr;
  uint16_t* EAaug = nullptr; // [H][M + Nmax][32]
  float* proj = nullptr;
  int* ev_slot = nullptr;
  int* tail = nullptr;
  int* newp = nullptr;
  float* sub = nullptr;
  float* coadm = nullptr;
  float* partial = nullptr;
  // a kvb_admit_begin whose kvb_admit_finish is still due (host-side)
  struct PendingAdmit {
    int layer = -1;
    const void* candK = nullptr;
    const void* candV = nullptr;
    const int32_t* cand_ids = nullptr;
    int N = 0;
  } pending;

  // ---- Forcing-KV, per layer
  char* tK = nullptr;       // [L][H][F][d] transition frame (static heads)
  char* tV = nullptr;
  int* tids = nullptr;      // [L][H][F]
  int* tlen = nullptr;      // [L][H] transition length (0 before the first prune)
  char* rK = nullptr;       // [L][H][ring_cap][d] FIFO of pruned frames (dynamic heads)
  char* rV = nullptr;
  int* rids = nullptr;      // [L][H][ring_cap]
  int* fstart = nullptr;    // [L][H][hist_frames] ring position of each stored frame
  int* fcount = nullptr;    // [L][H][hist_frames]
  int* rstate = nullptr;    // [L][H][4]: first frame slot, frames held, token start, tokens held
  uint8_t* is_static = nullptr;  // [L][H] labels of the last prune
  int* aseg = nullptr;      // [L][4][H]: transition length, ring part-1 start, part-1 length, part-2 length
  // ---- Forcing-KV scratch
  float* sims = nullptr;    // [H][max_new_frames][n_seg]
  int* keep = nullptr;      // [H][max_new_frames][n_seg] kept segment ids, ascending
  int* seg_tok = nullptr;   // [n_seg + 1] token offsets of each segment in segment-major order
  int* plan = nullptr;      // [H][max_new_frames*F][2] (source row, ring position) pairs
  int* plan_n = nullptr;    // [H]
  // KVB_SIM_FIRST_LAYER: frames of layer 0's last prune, whose similarities (left
  // in `sims`) the later layers reuse; -1 before the first one
  int proxy_frames = -1;

  size_t layout(void* base);  // carve (base may be null to measure); returns bytes
};

// E4M3 storage: make the bank's bf16 working copy hold `layer` (api_bank.cu).
cudaError_t kvb_work_layer(kvb_bank* b, int layer, cudaStream_t st);
