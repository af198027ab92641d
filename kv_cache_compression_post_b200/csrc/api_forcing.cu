// Forcing-KV entry points: bank initialisation, kvb_prune_hybrid, history export
// and the operation-level kvb_segment_cosine.
#include <cstring>
#include <vector>

#include "bank.h"
#include "forcing.cuh"

using namespace kvb;

namespace {

SegGeom geom(int frame_h, int frame_w, int seg_h, int seg_w) {
  SegGeom g;
  g.frame_h = frame_h;
  g.frame_w = frame_w;
  g.seg_h = seg_h;
  g.seg_w = seg_w;
  g.F = frame_h * frame_w;
  g.seg_rows = (frame_h + seg_h - 1) / seg_h;
  g.seg_cols = (frame_w + seg_w - 1) / seg_w;
  g.n_seg = g.seg_rows * g.seg_cols;
  return g;
}

int keep_count(int n_seg, float r) {
  // floor(r * n) in double, with a little slack so that e.g. 0.3 * 10 is 3
  const double v = static_cast<double>(r) * n_seg + 1e-6;
  int k = static_cast<int>(v);
  return k < 0 ? 0 : (k > n_seg ? n_seg : k);
}

}  // namespace

extern "C" kvb_status kvb_forcing_init(kvb_bank* b, cudaStream_t st) {
  const kvb_config& g = b->cfg;
  const SegGeom sg = geom(g.frame_h, g.frame_w, g.seg_h, g.seg_w);
  if (sg.n_seg > 1024) return KVB_E_UNSUPPORTED;
  // segment-major token order: segment j (row-major over segments) lists its
  // tokens row-major; seg_tok[j] is its first position in that order
  std::vector<int> tok(sg.n_seg + 1);
  int pos = 0;
  for (int sr = 0; sr < sg.seg_rows; ++sr)
    for (int sc = 0; sc < sg.seg_cols; ++sc) {
      tok[sr * sg.seg_cols + sc] = pos;
      const int rows = std::min((sr + 1) * sg.seg_h, sg.frame_h) - sr * sg.seg_h;
      const int cols = std::min((sc + 1) * sg.seg_w, sg.frame_w) - sc * sg.seg_w;
      pos += rows * cols;
    }
  tok[sg.n_seg] = pos;
  const size_t LH = static_cast<size_t>(g.layers) * g.heads;
  cudaError_t e = cudaMemcpyAsync(b->seg_tok, tok.data(), sizeof(int) * tok.size(), cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);  // the host vector goes out of scope
  // rows past a history's length are read by full attention tiles (and masked):
  // keep them finite by starting from zeros
  if (e == cudaSuccess) e = cudaMemsetAsync(b->tK, 0, LH * b->F * static_cast<size_t>(b->row_bytes), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(b->tV, 0, LH * b->F * static_cast<size_t>(b->row_bytes), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(b->rK, 0, LH * b->ring_cap * static_cast<size_t>(b->row_bytes), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(b->rV, 0, LH * b->ring_cap * static_cast<size_t>(b->row_bytes), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(b->tlen, 0, LH * sizeof(int), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(b->rstate, 0, LH * 4 * sizeof(int), st);
  if (e == cudaSuccess) e = cudaMemsetAsync(b->aseg, 0, LH * 4 * sizeof(int), st);
  return cuda_status(e);
}

extern "C" kvb_status kvb_prune_hybrid(kvb_bank* b, int32_t layer, const uint8_t* head_is_static, const void* newK,
                                       const void* newV, const void* nextK, const int32_t* new_ids,
                                       int32_t n_frames, void* stream) {
  if (!b) return KVB_E_INVAL;
  const kvb_config& g = b->cfg;
  if (g.method != KVB_FORCINGKV) return KVB_E_STATE;
  if (layer < 0 || layer >= g.layers || n_frames < 1 || n_frames > g.max_new_frames) return KVB_E_INVAL;
  if (!head_is_static || !newK || !newV || !nextK || !new_ids) return KVB_E_INVAL;
  // rows are moved and read in 16-byte chunks
  if (((reinterpret_cast<uintptr_t>(newK) | reinterpret_cast<uintptr_t>(newV) | reinterpret_cast<uintptr_t>(nextK)) &
       15) != 0)
    return KVB_E_INVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int H = g.heads;
  unsigned long long mask = 0;
  for (int h = 0; h < H; ++h)
    if (head_is_static[h]) mask |= 1ull << h;
  const SegGeom sg = geom(g.frame_h, g.frame_w, g.seg_h, g.seg_w);
  const size_t lh = static_cast<size_t>(layer) * H;

  // first-block proxy: layer 0 computes every head's similarities, later layers
  // reuse them (they must follow a layer-0 prune of the same chunk)
  const bool proxy = g.sim_source == KVB_SIM_FIRST_LAYER;
  if (proxy && layer > 0 && b->proxy_frames != n_frames) return KVB_E_STATE;

  PrunePlan p;
  p.H = H;
  p.d = g.head_dim;
  p.n_frames = n_frames;
  p.hist_frames = g.hist_frames;
  p.ring_cap = b->ring_cap;
  p.scope = g.bottomk_scope;
  p.keep = g.bottomk_scope == KVB_BOTTOMK_CALL ? keep_count(sg.n_seg * n_frames, g.retention)
                                               : keep_count(sg.n_seg, g.retention);
  p.row_bytes = b->row_bytes;
  p.g = sg;
  p.static_mask = mask;
  p.newK = newK;
  p.newV = newV;
  p.new_ids = new_ids;
  p.sims = b->sims;
  p.seg_tok = b->seg_tok;
  p.plan = b->plan;
  p.plan_n = b->plan_n;
  p.keep_list = b->keep;
  p.ld_plan = g.max_new_frames * b->F;
  p.ld_sims = g.max_new_frames * sg.n_seg;
  p.tK = b->tK + lh * b->F * b->row_bytes;
  p.tV = b->tV + lh * b->F * b->row_bytes;
  p.tids = b->tids + lh * b->F;
  p.tlen = b->tlen + lh;
  p.rK = b->rK + lh * b->ring_cap * b->row_bytes;
  p.rV = b->rV + lh * b->ring_cap * b->row_bytes;
  p.rids = b->rids + lh * b->ring_cap;
  p.fstart = b->fstart + lh * g.hist_frames;
  p.fcount = b->fcount + lh * g.hist_frames;
  p.rstate = b->rstate + lh * 4;
  p.aseg = b->aseg + lh * 4;
  p.stats = b->stats + lh;
  p.status = b->status;

  cudaError_t e = cudaSuccess;
  const unsigned long long all = (H >= 64) ? ~0ull : ((1ull << H) - 1);
  if (proxy && layer == 0)
    e = launch_seg_cosine_ld(newK, nextK, g.dtype, H, n_frames, g.head_dim, sg, 0ull, b->sims, p.ld_sims, st);
  else if (!proxy && (mask & all) != all)
    e = launch_seg_cosine_ld(newK, nextK, g.dtype, H, n_frames, g.head_dim, sg, mask, b->sims, p.ld_sims, st);
  if (proxy && layer == 0) b->proxy_frames = e == cudaSuccess ? n_frames : -1;
  if (e == cudaSuccess) e = launch_prune_plan(p, st);
  if (e == cudaSuccess) e = launch_prune_gather(p, st);  // static heads' transition frames too
  return cuda_status(e);
}

extern "C" kvb_status kvb_forcing_export(kvb_bank* b, int32_t layer, int32_t head, int32_t* ids, void* K, void* V,
                                         int32_t* size, cudaStream_t st) {
  const int H = b->cfg.heads;
  int as[4];
  for (int k = 0; k < 4; ++k) {
    cudaError_t e = cudaMemcpyAsync(&as[k], b->aseg + static_cast<size_t>(layer) * 4 * H + k * H + head,
                                    sizeof(int), cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess) return KVB_E_CUDA;
  }
  if (cudaStreamSynchronize(st) != cudaSuccess) return KVB_E_CUDA;
  const size_t lh = static_cast<size_t>(layer) * H + head;
  cudaError_t e = cudaSuccess;
  if (as[0] > 0) {  // static head: its transition frame
    if (as[0] > b->F) return KVB_E_DEVICE_BOUNDS;
    *size = as[0];
    const size_t r0 = lh * b->F;
    if (ids) e = cudaMemcpyAsync(ids, b->tids + r0, sizeof(int) * as[0], cudaMemcpyDeviceToDevice, st);
    if (K && e == cudaSuccess)
      e = cudaMemcpyAsync(K, b->tK + r0 * b->row_bytes, static_cast<size_t>(as[0]) * b->row_bytes,
                          cudaMemcpyDeviceToDevice, st);
    if (V && e == cudaSuccess)
      e = cudaMemcpyAsync(V, b->tV + r0 * b->row_bytes, static_cast<size_t>(as[0]) * b->row_bytes,
                          cudaMemcpyDeviceToDevice, st);
  } else {          // dynamic head: the ring, oldest frame first
    const int start = as[1], p1 = as[2], p2 = as[3];
    if (start < 0 || p1 < 0 || p2 < 0 || start + p1 > b->ring_cap || p1 + p2 > b->ring_cap)
      return KVB_E_DEVICE_BOUNDS;
    *size = p1 + p2;
    const size_t r0 = lh * b->ring_cap;
    const size_t rb = b->row_bytes;
    if (ids && p1) e = cudaMemcpyAsync(ids, b->rids + r0 + start, sizeof(int) * p1, cudaMemcpyDeviceToDevice, st);
    if (ids && p2 && e == cudaSuccess)
      e = cudaMemcpyAsync(ids + p1, b->rids + r0, sizeof(int) * p2, cudaMemcpyDeviceToDevice, st);
    for (int which = 0; which < 2 && e == cudaSuccess; ++which) {
      char* dst = static_cast<char*>(which == 0 ? K : V);
      const char* src = (which == 0 ? b->rK : b->rV) + r0 * rb;
      if (!dst) continue;
      if (p1) e = cudaMemcpyAsync(dst, src + start * rb, p1 * rb, cudaMemcpyDeviceToDevice, st);
      if (p2 && e == cudaSuccess) e = cudaMemcpyAsync(dst + p1 * rb, src, p2 * rb, cudaMemcpyDeviceToDevice, st);
    }
  }
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  return cuda_status(e);
}

extern "C" kvb_status kvb_segment_cosine(const void* K, const void* nextK, int32_t heads, int32_t n_frames,
                                         int32_t frame_h, int32_t frame_w, int32_t seg_h, int32_t seg_w,
                                         int32_t head_dim, kvb_dtype dtype, float* sim, void* stream) {
  if (!K || !nextK || !sim || heads < 1 || heads > 64 || n_frames < 1) return KVB_E_INVAL;
  if (frame_h < 1 || frame_w < 1 || seg_h < 1 || seg_w < 1 || head_dim < 1 || head_dim > 1024) return KVB_E_INVAL;
  if (dtype != KVB_BF16 && dtype != KVB_F32) return KVB_E_INVAL;
  if (static_cast<size_t>(seg_h) * frame_w * sizeof(float) > 48 * 1024) return KVB_E_UNSUPPORTED;
  const int esize = dtype == KVB_BF16 ? 2 : 4;
  if ((head_dim * esize) % 16 != 0) return KVB_E_UNSUPPORTED;  // rows are read in 16-byte chunks
  if (((reinterpret_cast<uintptr_t>(K) | reinterpret_cast<uintptr_t>(nextK)) & 15) != 0) return KVB_E_INVAL;
  const SegGeom sg = geom(frame_h, frame_w, seg_h, seg_w);
  return cuda_status(launch_seg_cosine(K, nextK, dtype, heads, n_frames, head_dim, sg, 0ull, sim,
                                       static_cast<cudaStream_t>(stream)));
}
