// Bank-level C entry points: create/destroy, kvb_admit (DensityKV), export /
// import, counters and the device status word.  Forcing-KV's prune and the
// attention entry point live in api_forcing.cu and api_attend.cu.
#include <climits>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <new>

#include "admit.cuh"
#include "attend.cuh"
#include "bank.h"
#include "forcing.cuh"
#include "fp8.cuh"
#include "gram.cuh"
#include "small_kernels.cuh"

using namespace kvb;

namespace {

bool config_ok(const kvb_config* c) {
  if (!c) return false;
  if (c->method != KVB_DENSITYKV && c->method != KVB_FORCINGKV) return false;
  if (c->dtype != KVB_BF16 && c->dtype != KVB_F32) return false;
  if (c->layers < 1 || c->heads < 1 || c->heads > 64) return false;
  if (c->head_dim != 64 && c->head_dim != 128) return false;
  if (c->max_queries < 1) return false;
  if (c->storage != KVB_STORE_NATIVE && c->storage != KVB_STORE_FP8_E4M3) return false;
  // E4M3 storage: DensityKV banks of bf16 keys and values
  if (c->storage == KVB_STORE_FP8_E4M3 && (c->method != KVB_DENSITYKV || c->dtype != KVB_BF16)) return false;
  if (c->method == KVB_DENSITYKV) {
    if (c->capacity < 1 || c->max_candidates < 1) return false;
    if (!(c->eps > 0.f) || !std::isfinite(c->eps) || !(c->s >= 0.f) || !std::isfinite(c->s)) return false;
    if (!(c->tau > 0.f) || !(c->dist_scale >= 0.f)) return false;
    if (c->cand_order != KVB_ORDER_DISTURBANCE && c->cand_order != KVB_ORDER_SOURCE) return false;
    if (c->baselines != KVB_BASELINES_FIXED && c->baselines != KVB_BASELINES_REFRESH) return false;
    if (c->evict_order != KVB_EVICT_THRESHOLD_RATIO && c->evict_order != KVB_EVICT_DENSEST &&
        c->evict_order != KVB_EVICT_THRESHOLD_SOURCE)
      return false;
  } else {
    if (c->frame_h < 1 || c->frame_w < 1 || c->seg_h < 1 || c->seg_w < 1) return false;
    if (c->hist_frames < 1 || c->max_new_frames < 1) return false;
    if (!(c->retention >= 0.f && c->retention <= 1.f)) return false;
    if (c->bottomk_scope != KVB_BOTTOMK_FRAME && c->bottomk_scope != KVB_BOTTOMK_CALL) return false;
    if (c->sim_source != KVB_SIM_PER_LAYER && c->sim_source != KVB_SIM_FIRST_LAYER) return false;
    const long long n_seg = static_cast<long long>((c->frame_h + c->seg_h - 1) / c->seg_h) *
                            ((c->frame_w + c->seg_w - 1) / c->seg_w);
    if (c->bottomk_scope == KVB_BOTTOMK_CALL && n_seg * c->max_new_frames > kPruneMaxPairs) return false;
  }
  return true;
}

}  // namespace

size_t kvb_bank::layout(void* base) {
  Carver c(base);
  const kvb_config& g = cfg;
  const size_t L = g.layers, H = g.heads, d = g.head_dim;
  status = c.take<int>(64);
  attn_cnt = c.take<unsigned long long>(attend_counter_count(g.heads, g.max_queries));
  attn_part = g.dtype == KVB_BF16 ? c.take<float>(attend_partial_floats(g.head_dim)) : nullptr;
  if (g.method == KVB_DENSITYKV) {
    const size_t M = g.capacity, N = g.max_candidates;
    ldN = static_cast<int>(N);
    ldEA = static_cast<int>(M + N);
    ldPart = static_cast<int>(M > N ? M : N);
    if (g.storage == KVB_STORE_FP8_E4M3) {
      // one layer's bf16 working copy, every layer's E4M3 codes, the rounded candidates
      K = c.take<char>(H * M * d * elem);
      V = c.take<char>(H * M * d * elem);
      K8 = c.take<uint8_t>(L * H * M * d);
      V8 = c.take<uint8_t>(L * H * M * d);
      candQ = c.take<char>(2 * H * N * d * elem);
    } else {
      K = c.take<char>(L * H * M * d * elem);
      V = c.take<char>(L * H * M * d * elem);
    }
    ids = c.take<int>(L * H * M);
    rho = c.take<float>(L * H * M);
    rho0 = c.take<float>(L * H * M);
    aug = c.take<uint16_t>(L * H * M * 32);
    size = c.take<int>(L * H);
    stats = c.take<kvb_admit_stats>(L * H);
    caug = c.take<uint16_t>(H * N * 32);
    rhoB = c.take<float>(H * N);
    mean0 = c.take<float>(H);
    feasible = c.take<int>(H);
    P = c.take<int>(H);
    E = c.take<int>(H);
    n_old = c.take<int>(H);
    nhole = c.take<int>(H);
    ntail = c.take<int>(H);
    EAoff = c.take<int>(H);
    EAcnt = c.take<int>(H);
    adm_idx = c.take<int>(H * N);
    EA = c.take<char>(H * (M + N) * d * elem);
    EAaug = c.take<uint16_t>(H * (M + N) * 32);
    proj = c.take<float>(H * M);
    ev_slot = c.take<int>(H * M);
    tail = c.take<int>(H * M);
    newp = c.take<int>(H * M);
    sub = c.take<float>(H * M);
    coadm = c.take<float>(H * N);
    partial = c.take<float>(16 * H * static_cast<size_t>(ldPart));
  } else {
    F = g.frame_h * g.frame_w;
    n_seg = ((g.frame_h + g.seg_h - 1) / g.seg_h) * ((g.frame_w + g.seg_w - 1) / g.seg_w);
    ring_cap = g.hist_frames * F;
    const size_t nf = g.max_new_frames;
    tK = c.take<char>(L * H * F * d * elem);
    tV = c.take<char>(L * H * F * d * elem);
    tids = c.take<int>(L * H * F);
    tlen = c.take<int>(L * H);
    rK = c.take<char>(L * H * static_cast<size_t>(ring_cap) * d * elem);
    rV = c.take<char>(L * H * static_cast<size_t>(ring_cap) * d * elem);
    rids = c.take<int>(L * H * static_cast<size_t>(ring_cap));
    fstart = c.take<int>(L * H * g.hist_frames);
    fcount = c.take<int>(L * H * g.hist_frames);
    rstate = c.take<int>(L * H * 4);
    is_static = c.take<uint8_t>(L * H);
    aseg = c.take<int>(L * 4 * H);
    stats = c.take<kvb_admit_stats>(L * H);
    sims = c.take<float>(H * nf * n_seg);
    keep = c.take<int>(H * nf * n_seg);
    seg_tok = c.take<int>(n_seg + 1);
    plan = c.take<int>(2 * H * nf * F);  // (source row, ring slot) pairs
    plan_n = c.take<int>(H);
  }
  return c.bytes();
}

extern "C" {

size_t kvb_workspace_size(const kvb_config* cfg) {
  if (!config_ok(cfg)) return 0;
  kvb_bank b;
  b.cfg = *cfg;
  b.elem = cfg->dtype == KVB_BF16 ? 2 : 4;
  return b.layout(nullptr);
}

// implemented in api_forcing.cu
kvb_status kvb_forcing_init(kvb_bank* b, cudaStream_t st);

kvb_status kvb_bank_create(const kvb_config* cfg, void* workspace, size_t workspace_bytes, void* stream,
                           kvb_bank** out) {
  if (!out || !config_ok(cfg)) return KVB_E_INVAL;
  *out = nullptr;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return KVB_E_WORKSPACE;
  DeviceInfo dev;
  if (!current_device(&dev)) return KVB_E_CUDA;
  if (dev.cc_major != 10) return KVB_E_UNSUPPORTED;
  kvb_bank* b = new (std::nothrow) kvb_bank();
  if (!b) return KVB_E_INVAL;
  b->cfg = *cfg;
  b->elem = cfg->dtype == KVB_BF16 ? 2 : 4;
  b->row_bytes = cfg->head_dim * b->elem;
  b->h = cfg->dist_scale > 0.f ? cfg->dist_scale : static_cast<float>(cfg->head_dim);
  const size_t need = b->layout(nullptr);
  if (workspace_bytes < need) {
    delete b;
    return KVB_E_WORKSPACE;
  }
  b->ws = workspace;
  b->ws_bytes = workspace_bytes;
  b->layout(workspace);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t LH = static_cast<size_t>(cfg->layers) * cfg->heads;
  // status word, and status[1] = the largest ||k||^2 ever stored (density clamp guard)
  cudaError_t e = cudaMemsetAsync(b->status, 0, 2 * sizeof(int), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(b->stats, 0, LH * sizeof(kvb_admit_stats), st);
  if (e == cudaSuccess)
    e = cudaMemsetAsync(b->attn_cnt, 0, attend_counter_count(cfg->heads, cfg->max_queries) * sizeof(unsigned long long),
                        st);
  if (cfg->method == KVB_DENSITYKV) {
    // rows past a bank's size are read by full attention tiles (and masked): keep
    // them finite by starting from zeros
    const bool fp8 = cfg->storage == KVB_STORE_FP8_E4M3;
    const size_t kv = (fp8 ? static_cast<size_t>(cfg->heads) : LH) * cfg->capacity * static_cast<size_t>(b->row_bytes);
    if (e == cudaSuccess) e = cudaMemsetAsync(b->size, 0, LH * sizeof(int), st);
    if (e == cudaSuccess) e = cudaMemsetAsync(b->K, 0, kv, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(b->V, 0, kv, st);
    if (fp8) {
      const size_t codes = LH * cfg->capacity * static_cast<size_t>(cfg->head_dim);
      if (e == cudaSuccess) e = cudaMemsetAsync(b->K8, 0, codes, st);
      if (e == cudaSuccess) e = cudaMemsetAsync(b->V8, 0, codes, st);
      b->work_layer = -1;
    }
  } else if (e == cudaSuccess) {
    const kvb_status fs = kvb_forcing_init(b, st);
    if (fs != KVB_OK) {
      delete b;
      return fs;
    }
  }
  if (e != cudaSuccess) {
    delete b;
    return KVB_E_CUDA;
  }
  *out = b;
  return KVB_OK;
}

kvb_status kvb_bank_destroy(kvb_bank* bank) {
  if (!bank) return KVB_E_INVAL;
  delete bank;
  return KVB_OK;
}

}  // extern "C"

// E4M3 storage: make the bf16 working copy hold `layer` (decompressing its codes
// if it holds another layer or none).  Nothing to do for native storage.
cudaError_t kvb_work_layer(kvb_bank* b, int layer, cudaStream_t st) {
  if (b->cfg.method != KVB_DENSITYKV || b->cfg.storage != KVB_STORE_FP8_E4M3 || b->work_layer == layer)
    return cudaSuccess;
  const size_t n = static_cast<size_t>(b->cfg.heads) * b->cfg.capacity * b->cfg.head_dim;
  b->work_layer = -1;
  cudaError_t e = launch_dequant(b->K8 + static_cast<size_t>(layer) * n, b->K, n, st);
  if (e == cudaSuccess) e = launch_dequant(b->V8 + static_cast<size_t>(layer) * n, b->V, n, st);
  if (e == cudaSuccess) b->work_layer = layer;
  return e;
}

namespace {

// E4M3 storage: write the working copy's rows [0, size) back into `layer`'s codes
// (its values are E4M3 values already, so the rounding is exact).
cudaError_t store_work_layer(kvb_bank* b, int layer, cudaStream_t st) {
  if (b->cfg.storage != KVB_STORE_FP8_E4M3) return cudaSuccess;
  const kvb_config& g = b->cfg;
  const size_t n = static_cast<size_t>(g.heads) * g.capacity * g.head_dim;
  const int* size = b->size + static_cast<size_t>(layer) * g.heads;
  cudaError_t e = launch_quant_rows(b->K, b->K8 + static_cast<size_t>(layer) * n, g.heads, g.capacity, g.head_dim, size, st);
  if (e == cudaSuccess)
    e = launch_quant_rows(b->V, b->V8 + static_cast<size_t>(layer) * n, g.heads, g.capacity, g.head_dim, size, st);
  return e;
}

// E4M3 storage: the step's candidates rounded to E4M3 (once per step, `round`)
// replace the caller's in the plan.
cudaError_t use_rounded_candidates(kvb_bank* b, AdmitPlan& p, bool round, cudaStream_t st) {
  if (b->cfg.storage != KVB_STORE_FP8_E4M3) return cudaSuccess;
  const size_t n = static_cast<size_t>(p.H) * p.N * p.d;
  char* qK = b->candQ;
  char* qV = b->candQ + static_cast<size_t>(p.H) * b->cfg.max_candidates * p.d * b->elem;
  cudaError_t e = cudaSuccess;
  if (round) {
    e = launch_round_e4m3(p.candK, qK, n, st);
    if (e == cudaSuccess) e = launch_round_e4m3(p.candV, qV, n, st);
  }
  p.candK = qK;
  p.candV = qV;
  return e;
}

// One density pass: out[h][r] = sum over the column set of sign * phi, through the
// tcgen05 kernel (bf16) or the CUDA-core kernel (f32).
struct Pass {
  const void* R;       // rows buffer [H][ldR][d]
  long long ldR;
  GramSet rows;
  const uint16_t* Raug;  // [H][ldR][32] augmented rows of R
  const void* C;
  long long ldC;
  GramSet cols;
  const uint16_t* Caug;  // [H][ldC][32]
  int max_rows;
  int max_cols;
  int use_diag = 0;
  int nneg = 0;
  float* out;
  int ldOut;
  // rows per head of Raug / Caug when they differ from ldR / ldC (0: the same)
  long long ldRaug = 0, ldCaug = 0;
  // bf16: alternate operands for heads whose row (column) count is alt_rows_n
  // (alt_cols_n): read from row 0 of R2 / C2 instead (null: none)
  const void* R2 = nullptr;
  long long ldR2 = 0;
  const uint16_t* Raug2 = nullptr;
  long long ldRaug2 = 0;
  int alt_rows_n = -1;
  const void* C2 = nullptr;
  long long ldC2 = 0;
  const uint16_t* Caug2 = nullptr;
  long long ldCaug2 = 0;
  int alt_cols_n = -1;
};

cudaError_t run_pass(kvb_bank* b, const Pass& ps, const DeviceInfo& dev, cudaStream_t st) {
  const kvb_config& g = b->cfg;
  GramArgs a;
  a.H = g.heads;
  a.d = g.head_dim;
  a.rows = ps.rows;
  a.cols = ps.cols;
  a.use_diag = ps.use_diag;
  a.diag_uni = 0;
  a.nneg_uni = ps.nneg;
  a.kscale = -2.f / b->h;
  a.eps = g.eps;
  a.s = g.s;
  a.max_rows = ps.max_rows;
  a.status = b->status;
  if (g.dtype == KVB_F32) {
    a.R32 = static_cast<const float*>(ps.R);
    a.C32 = static_cast<const float*>(ps.C);
    a.ldR = static_cast<int>(ps.ldR);
    a.ldC = static_cast<int>(ps.ldC);
    a.partial = ps.out;
    a.ldOut = ps.ldOut;
    return launch_gram_f32(a, st);
  }
  GramMaps m;
  if (!make_tmap_bf16(&m.R, ps.R, g.head_dim, ps.ldR, g.heads, 128) ||
      !make_tmap_bf16(&m.C, ps.C, g.head_dim, ps.ldC, g.heads, kGramColTile) ||
      !make_tmap_aug(&m.Ra, ps.Raug, ps.ldRaug ? ps.ldRaug : ps.ldR, g.heads, 128) ||
      !make_tmap_aug(&m.Ca, ps.Caug, ps.ldCaug ? ps.ldCaug : ps.ldC, g.heads, kGramColTile))
    return cudaErrorInvalidValue;
  m.R2 = m.R;
  m.Ra2 = m.Ra;
  m.C2 = m.C;
  m.Ca2 = m.Ca;
  if (ps.R2) {
    if (!make_tmap_bf16(&m.R2, ps.R2, g.head_dim, ps.ldR2, g.heads, 128) ||
        !make_tmap_aug(&m.Ra2, ps.Raug2, ps.ldRaug2 ? ps.ldRaug2 : ps.ldR2, g.heads, 128))
      return cudaErrorInvalidValue;
    a.alt_rows_n = ps.alt_rows_n;
  }
  if (ps.C2) {
    if (!make_tmap_bf16(&m.C2, ps.C2, g.head_dim, ps.ldC2, g.heads, kGramColTile) ||
        !make_tmap_aug(&m.Ca2, ps.Caug2, ps.ldCaug2 ? ps.ldCaug2 : ps.ldC2, g.heads, kGramColTile))
      return cudaErrorInvalidValue;
    a.alt_cols_n = ps.alt_cols_n;
  }
  a.partial = b->partial;
  a.ldOut = b->ldPart;
  a.norm_max = reinterpret_cast<const float*>(b->status + 1);
  gram_plan(a, (ps.max_cols + kGramColTile - 1) / kGramColTile, dev.n_sm);
  cudaError_t e = launch_gram_bf16(a, m, st);
  if (e == cudaSuccess) e = launch_gram_reduce(a, ps.out, ps.ldOut, st);
  return e;
}

// Checks the arguments of an admit step and fills its plan (no launch).
kvb_status admit_plan(kvb_bank* b, int32_t layer, const void* candK, const void* candV, const int32_t* cand_ids,
                      int32_t N, AdmitPlan* out) {
  if (!b) return KVB_E_INVAL;
  const kvb_config& g = b->cfg;
  if (g.method != KVB_DENSITYKV) return KVB_E_STATE;
  if (layer < 0 || layer >= g.layers || N < 1 || N > g.max_candidates) return KVB_E_INVAL;
  if (!candK || !candV || !cand_ids) return KVB_E_INVAL;
  // the rounding kernels move 16-byte words
  if (g.storage == KVB_STORE_FP8_E4M3 &&
      ((reinterpret_cast<uintptr_t>(candK) | reinterpret_cast<uintptr_t>(candV)) & 15) != 0)
    return KVB_E_INVAL;
  const int H = g.heads, M = g.capacity, d = g.head_dim;
  const size_t lo = static_cast<size_t>(layer) * H * M;  // slot offset of this layer

  AdmitPlan& p = *out;
  p = AdmitPlan();
  p.H = H;
  p.M = M;
  p.N = N;
  p.d = d;
  p.dtype = g.dtype;
  p.row_bytes = b->row_bytes;
  p.tau = g.tau;
  p.sync_heads = g.sync_heads;
  p.cand_order = g.cand_order;
  p.baselines = g.baselines;
  p.evict_order = g.evict_order;
  // E4M3 storage: the kernels work on the bf16 working copy of the layer
  const size_t klo = g.storage == KVB_STORE_FP8_E4M3 ? 0 : lo;
  p.K = b->K + klo * b->row_bytes;
  p.V = b->V + klo * b->row_bytes;
  p.ids = b->ids + lo;
  p.rho = b->rho + lo;
  p.rho0 = b->rho0 + lo;
  p.aug = b->aug + lo * 32;
  p.size = b->size + static_cast<size_t>(layer) * H;
  p.stats = b->stats + static_cast<size_t>(layer) * H;
  p.candK = candK;
  p.candV = candV;
  p.cand_ids = cand_ids;
  p.caug = b->caug;
  p.rhoB = b->rhoB;
  p.mean0 = b->mean0;
  p.feasible = b->feasible;
  p.P = b->P;
  p.adm_idx = b->adm_idx;
  p.EA = b->EA;
  p.EAaug = b->EAaug;
  p.ldEA = b->ldEA;
  p.EAoff = b->EAoff;
  p.EAcnt = b->EAcnt;
  p.proj = b->proj;
  p.ev_slot = b->ev_slot;
  p.E = b->E;
  p.n_old = b->n_old;
  p.hole = b->ev_slot;
  p.nhole = b->nhole;
  p.tail = b->tail;
  p.ntail = b->ntail;
  p.newp = b->newp;
  p.sub = b->sub;
  p.coadm = b->coadm;
  p.ldN = b->ldN;
  p.status = b->status;

  return KVB_OK;
}

// Pass 1 and the feasible counts: everything before the prefix is fixed.
cudaError_t admit_phase1(kvb_bank* b, const AdmitPlan& p, const DeviceInfo& dev, cudaStream_t st) {
  const kvb_config& g = b->cfg;
  const int H = p.H, M = p.M, N = p.N, d = p.d;
  const void* candK = p.candK;
  cudaError_t e = cudaSuccess;
  if (g.dtype == KVB_BF16)
    e = launch_aug_rows(candK, g.dtype, H, N, d, N, nullptr, N, b->caug, b->ldN, reinterpret_cast<float*>(b->status + 1),
                        -0.5f * g.eps * b->h, st);

  // pass 1: candidate density against the bank, rho_B(c)
  if (e == cudaSuccess) {
    Pass ps{candK, N, GramSet{N, nullptr, 0, nullptr}, b->caug, p.K, M, GramSet{0, p.size, 0, nullptr}, p.aug, N, M};
    ps.ldRaug = b->ldN;  // the candidates' augmented rows are laid out for max_candidates
    ps.out = b->rhoB;
    ps.ldOut = b->ldN;
    e = run_pass(b, ps, dev, st);
  }
  if (e == cudaSuccess) e = launch_admit_count(p, st);
  return e;
}

// Selection under the prefix, projected growth, eviction, compaction and the
// incremental density update.
cudaError_t admit_phase2(kvb_bank* b, const AdmitPlan& p, const DeviceInfo& dev, cudaStream_t st) {
  const int M = p.M, N = p.N;
  cudaError_t e = launch_admit_select(p, st);
  if (e == cudaSuccess) e = launch_gather_admitted(p, N < M ? N : M, st);
  // pass 2: projected growth of every bank entry from the admitted block
  if (e == cudaSuccess) {
    Pass ps{p.K, M, GramSet{0, p.size, 0, nullptr}, p.aug, b->EA, b->ldEA, GramSet{0, b->P, M, nullptr}, b->EAaug, M, N};
    ps.out = b->proj;
    ps.ldOut = M;
    if (b->cfg.dtype == KVB_BF16) {
      // a head that admits every candidate (P = N, in candidate order) reads them in place
      ps.C2 = p.candK;
      ps.ldC2 = N;
      ps.Caug2 = b->caug;
      ps.ldCaug2 = b->ldN;
      ps.alt_cols_n = N;
    }
    e = run_pass(b, ps, dev, st);
  }
  if (e == cudaSuccess) e = launch_evict_select(p, st);
  if (e == cudaSuccess) e = launch_gather_evicted(p, st);
  if (e == cudaSuccess) e = launch_compact(p, st);
  // pass 3a: every entry of the new bank loses its evicted neighbours
  if (e == cudaSuccess) {
    Pass ps{p.K, M, GramSet{0, p.size, 0, nullptr}, p.aug, b->EA, b->ldEA, GramSet{0, b->EAcnt, 0, b->EAoff}, b->EAaug,
            M, M};
    ps.nneg = INT_MAX;
    ps.out = b->sub;
    ps.ldOut = M;
    e = run_pass(b, ps, dev, st);
  }
  // pass 3b: co-admitted entries see one another (self excluded)
  if (e == cudaSuccess) {
    Pass ps{b->EA, b->ldEA, GramSet{0, b->P, M, nullptr}, b->EAaug, b->EA, b->ldEA, GramSet{0, b->P, M, nullptr}, b->EAaug,
            N, N};
    ps.use_diag = 1;
    ps.out = b->coadm;
    ps.ldOut = b->ldN;
    if (b->cfg.dtype == KVB_BF16) {
      ps.R2 = ps.C2 = p.candK;
      ps.ldR2 = ps.ldC2 = N;
      ps.Raug2 = ps.Caug2 = b->caug;
      ps.ldRaug2 = ps.ldCaug2 = b->ldN;
      ps.alt_rows_n = ps.alt_cols_n = N;
    }
    e = run_pass(b, ps, dev, st);
  }
  if (e == cudaSuccess) e = launch_finalize(p, st);
  return e;
}

}  // namespace

extern "C" kvb_status kvb_admit(kvb_bank* b, int32_t layer, const void* candK, const void* candV,
                                const int32_t* cand_ids, int32_t N, void* stream) {
  AdmitPlan p;
  const kvb_status s = admit_plan(b, layer, candK, candV, cand_ids, N, &p);
  if (s != KVB_OK) return s;
  DeviceInfo dev;
  if (!current_device(&dev)) return KVB_E_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  b->pending.layer = -1;  // the scratch of a begun step is overwritten
  cudaError_t e = kvb_work_layer(b, layer, st);
  if (e == cudaSuccess) e = use_rounded_candidates(b, p, true, st);
  if (e == cudaSuccess) e = admit_phase1(b, p, dev, st);
  if (e == cudaSuccess) e = admit_phase2(b, p, dev, st);
  if (e == cudaSuccess) e = store_work_layer(b, layer, st);
  return cuda_status(e);
}

extern "C" kvb_status kvb_admit_begin(kvb_bank* b, int32_t layer, const void* candK, const void* candV,
                                      const int32_t* cand_ids, int32_t N, int32_t* prefix_out, void* stream) {
  if (!prefix_out) return KVB_E_INVAL;
  AdmitPlan p;
  const kvb_status s = admit_plan(b, layer, candK, candV, cand_ids, N, &p);
  if (s != KVB_OK) return s;
  DeviceInfo dev;
  if (!current_device(&dev)) return KVB_E_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  b->pending.layer = -1;
  cudaError_t e = kvb_work_layer(b, layer, st);
  if (e == cudaSuccess) e = use_rounded_candidates(b, p, true, st);
  if (e == cudaSuccess) e = admit_phase1(b, p, dev, st);
  if (e == cudaSuccess) e = launch_feasible_min(p, prefix_out, st);
  if (e != cudaSuccess) return cuda_status(e);
  b->pending.layer = layer;
  b->pending.candK = candK;
  b->pending.candV = candV;
  b->pending.cand_ids = cand_ids;
  b->pending.N = N;
  return KVB_OK;
}

extern "C" kvb_status kvb_admit_finish(kvb_bank* b, int32_t layer, const int32_t* prefix_bound, void* stream) {
  if (!b) return KVB_E_INVAL;
  if (b->cfg.method != KVB_DENSITYKV || b->pending.layer < 0 || b->pending.layer != layer) return KVB_E_STATE;
  if (prefix_bound && !b->cfg.sync_heads) return KVB_E_INVAL;
  AdmitPlan p;
  const kvb_status s = admit_plan(b, layer, b->pending.candK, b->pending.candV, b->pending.cand_ids, b->pending.N, &p);
  if (s != KVB_OK) return s;
  DeviceInfo dev;
  if (!current_device(&dev)) return KVB_E_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  p.p_bound = prefix_bound;
  b->pending.layer = -1;
  // the working copy and the rounded candidates of the begun step are still in place
  cudaError_t e = use_rounded_candidates(b, p, false, st);
  if (e == cudaSuccess) e = admit_phase2(b, p, dev, st);
  if (e == cudaSuccess) e = store_work_layer(b, layer, st);
  return cuda_status(e);
}

extern "C" {

kvb_status kvb_read_stats(kvb_bank* b, int32_t layer, kvb_admit_stats* host_out, void* stream) {
  if (!b || !host_out || layer < 0 || layer >= b->cfg.layers) return KVB_E_INVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int H = b->cfg.heads;
  cudaError_t e = cudaMemcpyAsync(host_out, b->stats + static_cast<size_t>(layer) * H,
                                  sizeof(kvb_admit_stats) * H, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  return cuda_status(e);
}

kvb_status kvb_device_status(kvb_bank* b, void* stream) {
  if (!b) return KVB_E_INVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, b->status, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return KVB_E_CUDA;
  return static_cast<kvb_status>(v);
}

// implemented in api_forcing.cu
kvb_status kvb_forcing_export(kvb_bank* b, int32_t layer, int32_t head, int32_t* ids, void* K, void* V,
                              int32_t* size, cudaStream_t st);

kvb_status kvb_bank_export(kvb_bank* b, int32_t layer, int32_t head, int32_t* ids, float* rho, float* rho0,
                           void* K, void* V, int32_t* size, void* stream) {
  if (!b || !size || layer < 0 || layer >= b->cfg.layers || head < 0 || head >= b->cfg.heads)
    return KVB_E_INVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (b->cfg.method == KVB_FORCINGKV) return kvb_forcing_export(b, layer, head, ids, K, V, size, st);
  const int M = b->cfg.capacity;
  const size_t slot0 = (static_cast<size_t>(layer) * b->cfg.heads + head) * M;
  // K/V rows: the layer's own (native storage) or the working copy, made to hold it (E4M3)
  const bool fp8 = b->cfg.storage == KVB_STORE_FP8_E4M3;
  const size_t kslot0 = fp8 ? static_cast<size_t>(head) * M : slot0;
  if (fp8 && kvb_work_layer(b, layer, st) != cudaSuccess) return KVB_E_CUDA;
  int n = 0;
  cudaError_t e = cudaMemcpyAsync(&n, b->size + static_cast<size_t>(layer) * b->cfg.heads + head, sizeof(int),
                                  cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return KVB_E_CUDA;
  if (n < 0 || n > M) return KVB_E_DEVICE_BOUNDS;
  *size = n;
  if (n == 0) return KVB_OK;
  if (ids && e == cudaSuccess)
    e = cudaMemcpyAsync(ids, b->ids + slot0, sizeof(int) * n, cudaMemcpyDeviceToDevice, st);
  if (rho && e == cudaSuccess)
    e = cudaMemcpyAsync(rho, b->rho + slot0, sizeof(float) * n, cudaMemcpyDeviceToDevice, st);
  if (rho0 && e == cudaSuccess)
    e = cudaMemcpyAsync(rho0, b->rho0 + slot0, sizeof(float) * n, cudaMemcpyDeviceToDevice, st);
  if (K && e == cudaSuccess)
    e = cudaMemcpyAsync(K, b->K + kslot0 * b->row_bytes, static_cast<size_t>(n) * b->row_bytes,
                        cudaMemcpyDeviceToDevice, st);
  if (V && e == cudaSuccess)
    e = cudaMemcpyAsync(V, b->V + kslot0 * b->row_bytes, static_cast<size_t>(n) * b->row_bytes,
                        cudaMemcpyDeviceToDevice, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  return cuda_status(e);
}

kvb_status kvb_bank_import(kvb_bank* b, int32_t layer, int32_t head, const int32_t* ids, const float* rho,
                           const float* rho0, const void* K, const void* V, int32_t size, void* stream) {
  if (!b || layer < 0 || layer >= b->cfg.layers || head < 0 || head >= b->cfg.heads) return KVB_E_INVAL;
  if (b->cfg.method != KVB_DENSITYKV) return KVB_E_STATE;
  b->pending.layer = -1;  // a begun admit step was computed against the old bank
  const int M = b->cfg.capacity;
  if (size < 0 || size > M) return KVB_E_INVAL;
  if (size > 0 && (!ids || !rho || !rho0 || !K || !V)) return KVB_E_INVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t slot0 = (static_cast<size_t>(layer) * b->cfg.heads + head) * M;
  // E4M3 storage: K/V go into the working copy of the layer, rounded to E4M3, and
  // from there into the layer's codes
  const bool fp8 = b->cfg.storage == KVB_STORE_FP8_E4M3;
  const size_t kslot0 = fp8 ? static_cast<size_t>(head) * M : slot0;
  if (fp8 && size > 0 && ((reinterpret_cast<uintptr_t>(K) | reinterpret_cast<uintptr_t>(V)) & 15) != 0)
    return KVB_E_INVAL;
  cudaError_t e = fp8 ? kvb_work_layer(b, layer, st) : cudaSuccess;
  if (size > 0 && e == cudaSuccess) {
    e = cudaMemcpyAsync(b->ids + slot0, ids, sizeof(int) * size, cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess) e = cudaMemcpyAsync(b->rho + slot0, rho, sizeof(float) * size, cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(b->rho0 + slot0, rho0, sizeof(float) * size, cudaMemcpyDeviceToDevice, st);
    const size_t elems = static_cast<size_t>(size) * b->cfg.head_dim;
    if (e == cudaSuccess)
      e = fp8 ? launch_round_e4m3(K, b->K + kslot0 * b->row_bytes, elems, st)
              : cudaMemcpyAsync(b->K + kslot0 * b->row_bytes, K, static_cast<size_t>(size) * b->row_bytes,
                                cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess)
      e = fp8 ? launch_round_e4m3(V, b->V + kslot0 * b->row_bytes, elems, st)
              : cudaMemcpyAsync(b->V + kslot0 * b->row_bytes, V, static_cast<size_t>(size) * b->row_bytes,
                                cudaMemcpyDeviceToDevice, st);
    if (e == cudaSuccess && b->cfg.dtype == KVB_BF16)
      e = launch_aug_rows(b->K + kslot0 * b->row_bytes, b->cfg.dtype, 1, size, b->cfg.head_dim, size, nullptr, size,
                          b->aug + slot0 * 32, size, reinterpret_cast<float*>(b->status + 1),
                          -0.5f * b->cfg.eps * b->h, st);
  }
  // the size word comes from host memory; the call synchronises before returning
  int host_size = size;
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(b->size + static_cast<size_t>(layer) * b->cfg.heads + head, &host_size, sizeof(int),
                        cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess && fp8) e = store_work_layer(b, layer, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  return cuda_status(e);
}

}  // extern "C"
