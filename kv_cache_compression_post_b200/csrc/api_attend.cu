// kvb_attend: attention of the current chunk over [sink | history | window].
//   DensityKV:  history = the layer's bank, [0, size_h) per head.
//   Forcing-KV: history = transition frame (static heads) or the pruned FIFO of
//               the dynamic heads, stored as a ring: two contiguous parts.
#include "attend.cuh"
#include "bank.h"

using namespace kvb;

extern "C" kvb_status kvb_attend(kvb_bank* b, int32_t layer, const void* Q, int32_t Nq, const void* sinkK,
                                 const void* sinkV, int32_t Ls, const void* winK, const void* winV, int32_t Lw,
                                 void* O, float* lse, void* stream) {
  if (!b) return KVB_E_INVAL;
  const kvb_config& g = b->cfg;
  if (layer < 0 || layer >= g.layers || Nq < 1 || Nq > g.max_queries || Ls < 0 || Lw < 0) return KVB_E_INVAL;
  if (!Q || !O || (Ls > 0 && (!sinkK || !sinkV)) || (Lw > 0 && (!winK || !winV))) return KVB_E_INVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int H = g.heads;
  AttnArgs a;
  a.H = H;
  a.d = g.head_dim;
  a.Nq = Nq;
  a.scale = 1.f / sqrtf(static_cast<float>(g.head_dim));
  a.Q = Q;
  a.O = O;
  a.lse = lse;
  a.status = b->status;
  a.part = b->attn_part;
  a.cnt = b->attn_cnt;
  if (++b->attn_epoch == 0) ++b->attn_epoch;
  a.epoch = b->attn_epoch;
  int n = 0;
  if (Ls > 0) {
    a.seg[n].K = sinkK;
    a.seg[n].V = sinkV;
    a.seg[n].ld = Ls;
    a.seg[n].len_uni = Ls;
    ++n;
  }
  if (g.method == KVB_DENSITYKV) {
    // E4M3 storage: attention reads the bf16 working copy, made to hold the layer
    const bool fp8 = g.storage == KVB_STORE_FP8_E4M3;
    if (fp8 && kvb_work_layer(b, layer, st) != cudaSuccess) return KVB_E_CUDA;
    const size_t lo = fp8 ? 0 : static_cast<size_t>(layer) * H * g.capacity;
    a.seg[n].K = b->K + lo * b->row_bytes;
    a.seg[n].V = b->V + lo * b->row_bytes;
    a.seg[n].ld = g.capacity;
    a.seg[n].len_dev = b->size + static_cast<size_t>(layer) * H;
    ++n;
  } else {
    const int* as = b->aseg + static_cast<size_t>(layer) * 4 * H;
    const size_t tlo = static_cast<size_t>(layer) * H * b->F;
    a.seg[n].K = b->tK + tlo * b->row_bytes;
    a.seg[n].V = b->tV + tlo * b->row_bytes;
    a.seg[n].ld = b->F;
    a.seg[n].len_dev = as;  // transition length (F for static heads after a prune, else 0)
    ++n;
    const size_t rlo = static_cast<size_t>(layer) * H * b->ring_cap;
    for (int part = 0; part < 2; ++part) {
      a.seg[n].K = b->rK + rlo * b->row_bytes;
      a.seg[n].V = b->rV + rlo * b->row_bytes;
      a.seg[n].ld = b->ring_cap;
      a.seg[n].off_dev = part == 0 ? as + H : nullptr;
      a.seg[n].off_uni = 0;
      a.seg[n].len_dev = part == 0 ? as + 2 * H : as + 3 * H;
      ++n;
    }
  }
  if (Lw > 0) {
    a.seg[n].K = winK;
    a.seg[n].V = winV;
    a.seg[n].ld = Lw;
    a.seg[n].len_uni = Lw;
    ++n;
  }
  a.nseg = n;
  cudaError_t e = g.dtype == KVB_BF16 ? launch_attend_bf16(a, st) : launch_attend_f32(a, st);
  if (e == cudaErrorInvalidValue) return KVB_E_INVAL;
  return cuda_status(e);
}
