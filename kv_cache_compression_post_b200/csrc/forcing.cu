// Forcing-KV hybrid prune (Forcing-KV reading notes §3.3 static structural
// pruning, §3.4 dynamic similarity pruning, §3.5 code map).
//
//   seg_cosine   per dynamic head and new frame t: token-wise cosine between frame
//                t and its successor at the same spatial position, averaged over
//                each seg_h x seg_w segment (one CTA per row of segments, one
//                warp per token, fixed-order segment sums)
//   prune_plan   per dynamic head: per frame the BottomK(floor(r n)) least
//                similar segments (ties: lower index), kept segments ascending,
//                tokens row-major inside each; the frame is pushed into a FIFO of
//                hist_frames frames stored as a token ring (the oldest frame is
//                dropped when the FIFO is full); emits (source row, ring slot)
//   prune_gather one warp per kept token: K, V rows and the id into the ring
//   static_copy  static heads: the last new frame becomes the transition frame
#include <cuda_bf16.h>

#include "forcing.cuh"
#include "host_util.h"
#include "kvb_device.cuh"

namespace kvb {
namespace {

template <typename T>
__global__ void seg_cosine_kernel(const T* __restrict__ K, const T* __restrict__ nextK, int n_frames, int d,
                                  SegGeom g, unsigned long long skip_mask, float* __restrict__ sim, int ld_sim) {
  extern __shared__ float cosv[];  // [seg_h * frame_w]
  const int sr = blockIdx.x, t = blockIdx.y, h = blockIdx.z;
  if ((skip_mask >> h) & 1ull) return;
  const int r0 = sr * g.seg_h;
  const int nrows = min(g.seg_h, g.frame_h - r0);
  const int ntok = nrows * g.frame_w;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const size_t Fd = static_cast<size_t>(g.F) * d;
  const T* base = K + static_cast<size_t>(h) * n_frames * Fd + static_cast<size_t>(t) * Fd;
  const T* succ = (t + 1 < n_frames) ? base + Fd : nextK + static_cast<size_t>(h) * Fd;
  for (int i = warp; i < ntok; i += nw) {
    const size_t p = static_cast<size_t>(r0 + i / g.frame_w) * g.frame_w + (i % g.frame_w);
    const T* a = base + p * d;
    const T* b = succ + p * d;
    float dot = 0.f, na = 0.f, nb = 0.f;
    for (int k = lane; k < d; k += 32) {
      const float x = load_elem(a, k), y = load_elem(b, k);
      dot = fmaf(x, y, dot);
      na = fmaf(x, x, na);
      nb = fmaf(y, y, nb);
    }
    dot = warp_sum(dot);
    na = warp_sum(na);
    nb = warp_sum(nb);
    if (lane == 0) cosv[i] = dot / fmaxf(sqrtf(na) * sqrtf(nb), 1e-8f);
  }
  __syncthreads();
  for (int sc = threadIdx.x; sc < g.seg_cols; sc += blockDim.x) {
    const int c0 = sc * g.seg_w, c1 = min(c0 + g.seg_w, g.frame_w);
    float s = 0.f;
    for (int r = 0; r < nrows; ++r)
      for (int c = c0; c < c1; ++c) s += cosv[r * g.frame_w + c];
    sim[static_cast<size_t>(h) * ld_sim + static_cast<size_t>(t) * g.n_seg + sr * g.seg_cols + sc] =
        s / static_cast<float>(nrows * (c1 - c0));
  }
}

constexpr int kPlanThreads = 256;

__global__ void __launch_bounds__(kPlanThreads) prune_plan_kernel(const PrunePlan p) {
  __shared__ int s_kept[1024];   // kept segments of the current frame, ascending
  __shared__ int s_off[1025];    // token offset of each kept segment
  __shared__ int s_flag[1024];
  __shared__ int s_state[4];
  __shared__ int s_fs, s_cnt, s_total;
  const int h = blockIdx.x;
  const bool is_static = (p.static_mask >> h) & 1ull;
  const int n_seg = p.g.n_seg;
  int* rs = p.rstate + 4 * h;
  if (is_static) {
    if (threadIdx.x == 0) {
      p.aseg[h] = p.g.F;
      p.aseg[p.H + h] = 0;
      p.aseg[2 * p.H + h] = 0;
      p.aseg[3 * p.H + h] = 0;
      p.plan_n[h] = 0;
      p.stats[h].admitted = p.g.F;
      p.stats[h].size = p.g.F;
    }
    return;
  }
  if (n_seg > 1024) {
    if (threadIdx.x == 0) latch_status(p.status, KVB_E_DEVICE_BOUNDS);
    return;
  }
  if (threadIdx.x < 4) s_state[threadIdx.x] = rs[threadIdx.x];
  if (threadIdx.x == 0) s_total = 0;
  __syncthreads();
  int* plan = p.plan + static_cast<size_t>(h) * p.ld_plan * 2;
  for (int t = 0; t < p.n_frames; ++t) {
    const float* s = p.sims + static_cast<size_t>(h) * p.ld_sims + static_cast<size_t>(t) * n_seg;
    // BottomK: segment j is kept iff fewer than `keep` segments precede it in
    // (similarity ascending, index ascending) order
    for (int j = threadIdx.x; j < n_seg; j += blockDim.x) {
      const float sj = s[j];
      int rank = 0;
      for (int i = 0; i < n_seg; ++i) {
        const float si = s[i];
        rank += (si < sj) || (si == sj && i < j);
      }
      s_flag[j] = rank < p.keep ? 1 : 0;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int q = 0, off = 0;
      for (int j = 0; j < n_seg; ++j) {
        if (!s_flag[j]) continue;
        s_kept[q] = j;
        s_off[q] = off;
        off += p.seg_tok[j + 1] - p.seg_tok[j];
        ++q;
      }
      s_off[q] = off;
      s_cnt = off;
      // FIFO: drop the oldest frame when full, then append this one
      int first = s_state[0], held = s_state[1], tstart = s_state[2], theld = s_state[3];
      if (held == p.hist_frames) {
        const int c = p.fcount[h * p.hist_frames + first];
        tstart = (tstart + c) % p.ring_cap;
        theld -= c;
        first = (first + 1) % p.hist_frames;
        --held;
      }
      const int slot = (first + held) % p.hist_frames;
      s_fs = (tstart + theld) % p.ring_cap;
      p.fstart[h * p.hist_frames + slot] = s_fs;
      p.fcount[h * p.hist_frames + slot] = off;
      s_state[0] = first;
      s_state[1] = held + 1;
      s_state[2] = tstart;
      s_state[3] = theld + off;
      for (int k = 0; k < q; ++k) p.keep_list[static_cast<size_t>(h) * p.ld_sims + t * n_seg + k] = s_kept[k];
    }
    __syncthreads();
    // plan entries of this frame: kept segment q, token m of it
    const int nk = p.keep;
    const int base = s_total;
    for (int q = 0; q < nk; ++q) {
      const int j = s_kept[q];
      const int t0 = p.seg_tok[j], t1 = p.seg_tok[j + 1];
      for (int m = threadIdx.x; m < t1 - t0; m += blockDim.x) {
        const int e = base + s_off[q] + m;
        if (e < p.ld_plan) {
          plan[2 * e] = t * p.g.F + p.seg_list[t0 + m];
          plan[2 * e + 1] = (s_fs + s_off[q] + m) % p.ring_cap;
        }
      }
    }
    __syncthreads();
    if (threadIdx.x == 0) s_total += s_cnt;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    for (int k = 0; k < 4; ++k) rs[k] = s_state[k];
    const int start = s_state[2], held = s_state[3];
    const int part1 = min(held, p.ring_cap - start);
    p.aseg[h] = 0;
    p.aseg[p.H + h] = start;
    p.aseg[2 * p.H + h] = part1;
    p.aseg[3 * p.H + h] = held - part1;
    p.plan_n[h] = s_total;
    p.stats[h].admitted = s_total;
    p.stats[h].feasible = p.keep;
    p.stats[h].size = held;
    if (s_total > p.ld_plan) latch_status(p.status, KVB_E_DEVICE_BOUNDS);
  }
}

__device__ __forceinline__ void copy_row16(void* dst, const void* src, int row_bytes, int lane) {
  const uint4* s = static_cast<const uint4*>(src);
  uint4* d = static_cast<uint4*>(dst);
  for (int o = lane; o < row_bytes / 16; o += 32) d[o] = s[o];
}

__global__ void prune_gather_kernel(const PrunePlan p) {
  const int h = blockIdx.y;
  const int e = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if ((p.static_mask >> h) & 1ull) return;
  if (e >= min(p.plan_n[h], p.ld_plan)) return;
  const int* plan = p.plan + static_cast<size_t>(h) * p.ld_plan * 2;
  const int src = plan[2 * e], dst = plan[2 * e + 1];
  if (src < 0 || src >= p.n_frames * p.g.F || dst < 0 || dst >= p.ring_cap) {
    if (lane == 0) latch_status(p.status, KVB_E_DEVICE_BOUNDS);
    return;
  }
  const size_t s = static_cast<size_t>(h) * p.n_frames * p.g.F + src;
  const size_t t = static_cast<size_t>(h) * p.ring_cap + dst;
  copy_row16(static_cast<char*>(p.rK) + t * p.row_bytes, static_cast<const char*>(p.newK) + s * p.row_bytes,
             p.row_bytes, lane);
  copy_row16(static_cast<char*>(p.rV) + t * p.row_bytes, static_cast<const char*>(p.newV) + s * p.row_bytes,
             p.row_bytes, lane);
  if (lane == 0) p.rids[t] = p.new_ids[src];
}

__global__ void static_copy_kernel(const PrunePlan p) {
  const int h = blockIdx.y;
  const int i = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (!((p.static_mask >> h) & 1ull) || i >= p.g.F) return;
  const int src = (p.n_frames - 1) * p.g.F + i;
  const size_t s = static_cast<size_t>(h) * p.n_frames * p.g.F + src;
  const size_t t = static_cast<size_t>(h) * p.g.F + i;
  copy_row16(static_cast<char*>(p.tK) + t * p.row_bytes, static_cast<const char*>(p.newK) + s * p.row_bytes,
             p.row_bytes, lane);
  copy_row16(static_cast<char*>(p.tV) + t * p.row_bytes, static_cast<const char*>(p.newV) + s * p.row_bytes,
             p.row_bytes, lane);
  if (lane == 0) {
    p.tids[t] = p.new_ids[src];
    if (i == 0) p.tlen[h] = p.g.F;
  }
}

}  // namespace

cudaError_t launch_seg_cosine(const void* K, const void* nextK, kvb_dtype dtype, int H, int n_frames, int d,
                              const SegGeom& g, unsigned long long skip_mask, float* sim, cudaStream_t st) {
  return launch_seg_cosine_ld(K, nextK, dtype, H, n_frames, d, g, skip_mask, sim, n_frames * g.n_seg, st);
}

cudaError_t launch_seg_cosine_ld(const void* K, const void* nextK, kvb_dtype dtype, int H, int n_frames, int d,
                                 const SegGeom& g, unsigned long long skip_mask, float* sim, int ld_sim,
                                 cudaStream_t st) {
  if (H <= 0 || n_frames <= 0) return cudaSuccess;
  dim3 grid(g.seg_rows, n_frames, H);
  const size_t smem = sizeof(float) * g.seg_h * g.frame_w;
  LaunchTrace trace("seg_cosine_kernel", st);
  if (dtype == KVB_BF16)
    seg_cosine_kernel<<<grid, 256, smem, st>>>(static_cast<const __nv_bfloat16*>(K),
                                               static_cast<const __nv_bfloat16*>(nextK), n_frames, d, g, skip_mask,
                                               sim, ld_sim);
  else
    seg_cosine_kernel<<<grid, 256, smem, st>>>(static_cast<const float*>(K), static_cast<const float*>(nextK),
                                               n_frames, d, g, skip_mask, sim, ld_sim);
  return cudaGetLastError();
}

cudaError_t launch_prune_plan(const PrunePlan& p, cudaStream_t st) {
  LaunchTrace trace("prune_plan_kernel", st);
  prune_plan_kernel<<<p.H, kPlanThreads, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_prune_gather(const PrunePlan& p, cudaStream_t st) {
  LaunchTrace trace("prune_gather_kernel", st);
  prune_gather_kernel<<<dim3((p.ld_plan + 7) / 8, p.H), 256, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_static_copy(const PrunePlan& p, cudaStream_t st) {
  LaunchTrace trace("static_copy_kernel", st);
  static_copy_kernel<<<dim3((p.g.F + 7) / 8, p.H), 256, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace kvb
