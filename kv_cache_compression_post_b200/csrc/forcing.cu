// Forcing-KV hybrid prune (Forcing-KV reading notes §3.3 static structural
// pruning, §3.4 dynamic similarity pruning, §3.5 code map).
//
//   seg_cosine   per dynamic head and new frame t: token-wise cosine between frame
//                t and its successor at the same spatial position, averaged over
//                each seg_h x seg_w segment (one CTA per row of segments, a
//                lane group of 16-byte loads per token, fixed-order segment sums)
//   prune_plan   per dynamic head: per frame the BottomK(floor(r n)) least
//                similar segments (ties: lower index) -- or, in the call scope,
//                the floor(r n n_frames) least similar (frame, segment) pairs of
//                all the call's frames ranked together -- kept segments ascending,
//                tokens row-major inside each; the frame is pushed into a FIFO of
//                hist_frames frames stored as a token ring (the oldest frame is
//                dropped when the FIFO is full); emits (source row, ring slot)
//   prune_gather dynamic heads: kept tokens' K, V rows and ids into the ring;
//                static heads: the last new frame becomes the transition frame
//                (lane groups of 16 bytes per lane, grid-strided)
#include <cuda_bf16.h>

#include "forcing.cuh"
#include "host_util.h"
#include "kvb_device.cuh"

namespace kvb {
namespace {

// Sum over the `width` lanes of an aligned lane group (width a power of two <= 32).
__device__ __forceinline__ float group_sum(float v, int width) {
  for (int o = width >> 1; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ void acc_words(uint4 a, uint4 b, float& dot, float& na, float& nb, __nv_bfloat16) {
  const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float xl = __uint_as_float(wa[k] << 16), xh = __uint_as_float(wa[k] & 0xFFFF0000u);
    const float yl = __uint_as_float(wb[k] << 16), yh = __uint_as_float(wb[k] & 0xFFFF0000u);
    dot = fmaf(xl, yl, fmaf(xh, yh, dot));
    na = fmaf(xl, xl, fmaf(xh, xh, na));
    nb = fmaf(yl, yl, fmaf(yh, yh, nb));
  }
}
__device__ __forceinline__ void acc_words(uint4 a, uint4 b, float& dot, float& na, float& nb, float) {
  const float xa[4] = {__uint_as_float(a.x), __uint_as_float(a.y), __uint_as_float(a.z), __uint_as_float(a.w)};
  const float xb[4] = {__uint_as_float(b.x), __uint_as_float(b.y), __uint_as_float(b.z), __uint_as_float(b.w)};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    dot = fmaf(xa[k], xb[k], dot);
    na = fmaf(xa[k], xa[k], na);
    nb = fmaf(xb[k], xb[k], nb);
  }
}

constexpr int kSegThreads = 512;

// One CTA per (row of segments, frame, head).  A token's two rows are read by a
// group of L lanes with 16-byte loads.  With CPL > 0 each lane holds CPL words of
// each row (L = words / CPL, a power of two, 4 for the rows of up to 64 words the
// banks use), and a round issues every load of its U tokens per group before the
// first product; the three sums per token then need log2(L) shuffle steps.
// CPL = 0 takes any row: L = the largest power of two up to min(words, 32) and a
// loop over each lane's words.
template <typename T, int CPL>
__global__ void __launch_bounds__(kSegThreads)
    seg_cosine_kernel(const T* __restrict__ K, const T* __restrict__ nextK, int n_frames, int d, SegGeom g,
                      unsigned long long skip_mask, float* __restrict__ sim, int ld_sim) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ float cosv[];  // [seg_h * frame_w]
  constexpr int U = CPL > 0 ? (CPL >= 8 ? 1 : 8 / CPL) : 2;  // tokens per lane group and round
  const int sr = blockIdx.x, t = blockIdx.y, h = blockIdx.z;
  if ((skip_mask >> h) & 1ull) return;
  const int r0 = sr * g.seg_h;
  const int nrows = min(g.seg_h, g.frame_h - r0);
  const int ntok = nrows * g.frame_w;
  const int chunks = d * static_cast<int>(sizeof(T)) / 16;  // 16-byte words per row
  int L = 1;                                                 // lanes per token
  if constexpr (CPL > 0) {
    L = chunks / CPL;
  } else {
    while (2 * L <= chunks && L < 32) L *= 2;
  }
  const int per_pass = blockDim.x / L;                       // tokens per pass of the CTA
  const int slot = threadIdx.x / L, sub = threadIdx.x % L;
  const size_t Fd = static_cast<size_t>(g.F) * d;
  const T* base = K + static_cast<size_t>(h) * n_frames * Fd + static_cast<size_t>(t) * Fd;
  const T* succ = (t + 1 < n_frames) ? base + Fd : nextK + static_cast<size_t>(h) * Fd;
  const size_t first = static_cast<size_t>(r0) * g.frame_w;  // segment rows are contiguous tokens
  for (int i0 = 0; i0 < ntok; i0 += U * per_pass) {
    float dot[U], na[U], nb[U];
#pragma unroll
    for (int u = 0; u < U; ++u) dot[u] = na[u] = nb[u] = 0.f;
    if constexpr (CPL > 0) {
      uint4 wa[U][CPL], wb[U][CPL];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = i0 + u * per_pass + slot;
        const uint4* a = reinterpret_cast<const uint4*>(base + (first + i) * d);
        const uint4* b = reinterpret_cast<const uint4*>(succ + (first + i) * d);
#pragma unroll
        for (int k = 0; k < CPL; ++k) {
          wa[u][k] = wb[u][k] = make_uint4(0u, 0u, 0u, 0u);
          if (i < ntok) {
            wa[u][k] = __ldg(a + sub + k * L);
            wb[u][k] = __ldg(b + sub + k * L);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int k = 0; k < CPL; ++k) acc_words(wa[u][k], wb[u][k], dot[u], na[u], nb[u], T());
    } else {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = i0 + u * per_pass + slot;
        if (i < ntok) {
          const uint4* a = reinterpret_cast<const uint4*>(base + (first + i) * d);
          const uint4* b = reinterpret_cast<const uint4*>(succ + (first + i) * d);
          for (int c = sub; c < chunks; c += L) acc_words(__ldg(a + c), __ldg(b + c), dot[u], na[u], nb[u], T());
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const float dd = group_sum(dot[u], L), aa = group_sum(na[u], L), bb = group_sum(nb[u], L);
      const int i = i0 + u * per_pass + slot;
      if (sub == 0 && i < ntok) cosv[i] = dd / fmaxf(sqrtf(aa) * sqrtf(bb), 1e-8f);
    }
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
constexpr int kPlanMaxSeg = 1024;

// Token (row-major position in the frame) of the m-th token of segment j, tokens
// numbered row-major inside the segment; segments are seg_h x seg_w tiles
// numbered row-major, partial at the right and bottom edges.
__device__ __forceinline__ int seg_token(const SegGeom& g, int j, int m) {
  const int sr = j / g.seg_cols, sc = j - sr * g.seg_cols;
  const int c0 = sc * g.seg_w;
  const int w = min(c0 + g.seg_w, g.frame_w) - c0;
  const int r = sr * g.seg_h + m / w;
  return r * g.frame_w + c0 + (m - (m / w) * w);
}
constexpr int kPlanMaxHist = 256;

// Exclusive scan of two ints over the CTA (kPlanThreads threads); returns the
// totals through *ta / *tb.
__device__ __forceinline__ int2 plan_scan2(int a, int b, int2* warp_tot, int* ta, int* tb) {
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  int ia = a, ib = b;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int xa = __shfl_up_sync(0xffffffffu, ia, o), xb = __shfl_up_sync(0xffffffffu, ib, o);
    if (l >= o) {
      ia += xa;
      ib += xb;
    }
  }
  if (l == 31) warp_tot[w] = make_int2(ia, ib);
  __syncthreads();
  int oa = 0, ob = 0, sa = 0, sb = 0;
  for (int k = 0; k < kPlanThreads / 32; ++k) {
    const int2 v = warp_tot[k];
    if (k < w) {
      oa += v.x;
      ob += v.y;
    }
    sa += v.x;
    sb += v.y;
  }
  *ta = sa;
  *tb = sb;
  __syncthreads();  // warp_tot may be reused right after
  return make_int2(oa + ia - a, ob + ib - b);
}

__global__ void __launch_bounds__(kPlanThreads) prune_plan_kernel(const PrunePlan p) {
  pdl_wait();
  pdl_trigger();
  // similarities: one frame's (per-frame scope) or every frame's of the call
  __shared__ float s_sim[kPruneMaxPairs];
  __shared__ int s_tok[kPlanMaxSeg + 1];  // token offset of each segment (segment-major list)
  __shared__ int s_kept[kPlanMaxSeg];     // kept segments of the current frame, ascending
  __shared__ int s_off[kPlanMaxSeg + 1];  // token offset of each kept segment in the frame
  __shared__ int2 s_wtot[kPlanThreads / 32];
  __shared__ int s_fc[kPlanMaxHist];      // the FIFO's frame token counts (histories up to kPlanMaxHist)
  __shared__ uint8_t s_kflag[kPruneMaxPairs];  // kept flag of every (frame, segment) pair
  __shared__ int s_state[4];
  __shared__ int s_fs, s_total;
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
  const bool call = p.scope == KVB_BOTTOMK_CALL;
  const int n_pairs = p.n_frames * n_seg;
  if (n_seg > kPlanMaxSeg || (call && n_pairs > kPruneMaxPairs)) {
    if (threadIdx.x == 0) latch_status(p.status, KVB_E_DEVICE_BOUNDS);
    return;
  }
  // every frame's similarities at hand from the start when they fit (always in the
  // call scope, whose pairs are ranked together), and the FIFO's frame counts:
  // no global load on the per-frame path
  const bool sims_at_hand = n_pairs <= kPruneMaxPairs;
  const bool fc_at_hand = p.hist_frames <= kPlanMaxHist;
  if (sims_at_hand)
    for (int q = threadIdx.x; q < n_pairs; q += blockDim.x)
      s_sim[q] = p.sims[static_cast<size_t>(h) * p.ld_sims + q];
  if (fc_at_hand)
    for (int k = threadIdx.x; k < p.hist_frames; k += blockDim.x) s_fc[k] = p.fcount[h * p.hist_frames + k];
  if (threadIdx.x < 4) s_state[threadIdx.x] = rs[threadIdx.x];
  if (threadIdx.x == 0) s_total = 0;
  for (int j = threadIdx.x; j <= n_seg; j += blockDim.x) s_tok[j] = p.seg_tok[j];
  int* plan = p.plan + static_cast<size_t>(h) * p.ld_plan * 2;
  // BottomK: a pair is kept iff fewer than `keep` entries precede it in
  // (similarity ascending, position ascending) order, among its frame's segments
  // (per-frame scope) or among the call's (frame, segment) pairs, position
  // t * n_seg + j (call scope).  With every similarity at hand all pairs are
  // ranked at once, before the frames are placed one after another.
  if (sims_at_hand) {
    __syncthreads();
    for (int q = threadIdx.x; q < n_pairs; q += blockDim.x) {
      const int lo = call ? 0 : (q / n_seg) * n_seg, hi = call ? n_pairs : lo + n_seg;
      const float sq = s_sim[q];
      int rank = 0;
      for (int i = lo; i < hi; ++i) {
        const float si = s_sim[i];
        rank += (si < sq) || (si == sq && i < q);
      }
      s_kflag[q] = rank < p.keep ? 1 : 0;
    }
  }
  // each thread owns a run of consecutive segments (for the ordered scans)
  const int per = (n_seg + kPlanThreads - 1) / kPlanThreads;
  const int j0 = threadIdx.x * per, j1 = min(n_seg, j0 + per);
  for (int t = 0; t < p.n_frames; ++t) {
    if (!sims_at_hand) {  // per-frame scope: this frame's similarities only
      const float* sg = p.sims + static_cast<size_t>(h) * p.ld_sims + static_cast<size_t>(t) * n_seg;
      for (int j = threadIdx.x; j < n_seg; j += blockDim.x) s_sim[j] = sg[j];
    }
    __syncthreads();
    int nk = 0, ntok = 0;
    unsigned int kept_bits = 0;  // per <= 32 segments per thread
    for (int j = j0; j < j1; ++j) {
      bool kept;
      if (sims_at_hand) {
        kept = s_kflag[t * n_seg + j] != 0;
      } else {
        const float sj = s_sim[j];
        int rank = 0;
        for (int i = 0; i < n_seg; ++i) {
          const float si = s_sim[i];
          rank += (si < sj) || (si == sj && i < j);
        }
        kept = rank < p.keep;
      }
      if (kept) {
        kept_bits |= 1u << (j - j0);
        ++nk;
        ntok += s_tok[j + 1] - s_tok[j];
      }
    }
    int tot_k, tot_tok;
    const int2 pos = plan_scan2(nk, ntok, s_wtot, &tot_k, &tot_tok);
    {
      int q = pos.x, off = pos.y;
      for (int j = j0; j < j1; ++j) {
        if (!((kept_bits >> (j - j0)) & 1u)) continue;
        s_kept[q] = j;
        s_off[q] = off;
        off += s_tok[j + 1] - s_tok[j];
        ++q;
      }
    }
    if (threadIdx.x == 0) {
      s_off[tot_k] = tot_tok;
      // FIFO: drop the oldest frame when full, then append this one
      int first = s_state[0], held = s_state[1], tstart = s_state[2], theld = s_state[3];
      if (held == p.hist_frames) {
        const int c = fc_at_hand ? s_fc[first] : p.fcount[h * p.hist_frames + first];
        tstart = (tstart + c) % p.ring_cap;
        theld -= c;
        first = (first + 1) % p.hist_frames;
        --held;
      }
      const int slot = (first + held) % p.hist_frames;
      s_fs = (tstart + theld) % p.ring_cap;
      p.fstart[h * p.hist_frames + slot] = s_fs;
      p.fcount[h * p.hist_frames + slot] = tot_tok;
      if (fc_at_hand) s_fc[slot] = tot_tok;
      s_state[0] = first;
      s_state[1] = held + 1;
      s_state[2] = tstart;
      s_state[3] = theld + tot_tok;
    }
    __syncthreads();
    for (int k = threadIdx.x; k < tot_k; k += blockDim.x)
      p.keep_list[static_cast<size_t>(h) * p.ld_sims + t * n_seg + k] = s_kept[k];
    // plan entries of this frame: entry e lies in kept segment q with
    // s_off[q] <= e < s_off[q + 1] (binary search)
    const int base = s_total;
    for (int e = threadIdx.x; e < tot_tok; e += blockDim.x) {
      int lo = 0, hi = tot_k - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_off[mid] <= e) lo = mid;
        else hi = mid - 1;
      }
      const int j = s_kept[lo];
      const int m = e - s_off[lo];
      const int g = base + e;
      if (g < p.ld_plan) {
        plan[2 * g] = t * p.g.F + seg_token(p.g, j, m);
        plan[2 * g + 1] = (s_fs + e) % p.ring_cap;
      }
    }
    __syncthreads();
    if (threadIdx.x == 0) s_total += tot_tok;
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

// Static heads: the last new frame becomes the transition frame.
__device__ __forceinline__ void static_copy(const PrunePlan& p, int h, const RowGroup& g) {
  const char* nK = static_cast<const char*>(p.newK);
  const char* nV = static_cast<const char*>(p.newV);
  for (int i0 = g.first; i0 < p.g.F; i0 += 2 * g.stride) {
    RowWords rw[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int i = i0 + u * g.stride;
      if (i >= p.g.F) continue;
      const size_t s = static_cast<size_t>(h) * p.n_frames * p.g.F + (p.n_frames - 1) * p.g.F + i;
      load_rows(rw[u], nK + s * p.row_bytes, nV + s * p.row_bytes, nullptr, p.row_bytes, g);
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int i = i0 + u * g.stride;
      if (i >= p.g.F) continue;
      const size_t t = static_cast<size_t>(h) * p.g.F + i;
      store_rows(rw[u], static_cast<char*>(p.tK) + t * p.row_bytes, static_cast<char*>(p.tV) + t * p.row_bytes,
                 nullptr, p.row_bytes, g);
      if (g.sub == 0) {
        p.tids[t] = p.new_ids[(p.n_frames - 1) * p.g.F + i];
        if (i == 0) p.tlen[h] = p.g.F;
      }
    }
  }
}

// Row moves of a prune: dynamic heads' kept tokens into their rings (two per
// lane group and iteration, every load before the first store), static heads'
// transition frame; one grid row per head.
__global__ void prune_gather_kernel(const PrunePlan p) {
  pdl_wait();
  pdl_trigger();
  const int h = blockIdx.y;
  const RowGroup g = row_group(p.row_bytes);
  if ((p.static_mask >> h) & 1ull) {
    static_copy(p, h, g);
    return;
  }
  const int n = min(p.plan_n[h], p.ld_plan);
  const int* plan = p.plan + static_cast<size_t>(h) * p.ld_plan * 2;
  const char* nK = static_cast<const char*>(p.newK);
  const char* nV = static_cast<const char*>(p.newV);
  for (int e0 = g.first; e0 < n; e0 += 2 * g.stride) {
    int src[2], dst[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int e = e0 + u * g.stride;
      src[u] = dst[u] = -1;
      if (e < n) {
        src[u] = plan[2 * e];
        dst[u] = plan[2 * e + 1];
        if (src[u] < 0 || src[u] >= p.n_frames * p.g.F || dst[u] < 0 || dst[u] >= p.ring_cap) {
          if (g.sub == 0) latch_status(p.status, KVB_E_DEVICE_BOUNDS);
          src[u] = -1;
        }
      }
    }
    RowWords rw[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (src[u] < 0) continue;
      const size_t s = static_cast<size_t>(h) * p.n_frames * p.g.F + src[u];
      load_rows(rw[u], nK + s * p.row_bytes, nV + s * p.row_bytes, nullptr, p.row_bytes, g);
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (src[u] < 0) continue;
      const size_t t = static_cast<size_t>(h) * p.ring_cap + dst[u];
      store_rows(rw[u], static_cast<char*>(p.rK) + t * p.row_bytes, static_cast<char*>(p.rV) + t * p.row_bytes,
                 nullptr, p.row_bytes, g);
      if (g.sub == 0) p.rids[t] = p.new_ids[src[u]];
    }
  }
}

}  // namespace

cudaError_t launch_seg_cosine(const void* K, const void* nextK, kvb_dtype dtype, int H, int n_frames, int d,
                              const SegGeom& g, unsigned long long skip_mask, float* sim, cudaStream_t st) {
  return launch_seg_cosine_ld(K, nextK, dtype, H, n_frames, d, g, skip_mask, sim, n_frames * g.n_seg, st);
}

template <typename T>
cudaError_t launch_seg_typed(const void* K, const void* nextK, int n_frames, int d, const SegGeom& g,
                             unsigned long long skip_mask, float* sim, int ld_sim, dim3 grid, size_t smem,
                             cudaStream_t st) {
  // four lanes per token when a row is 4, 8, 16 or 32 words long (each lane holds a
  // fixed number of words); any other row takes the looping form
  const int words = d * static_cast<int>(sizeof(T)) / 16;
  const T* k = static_cast<const T*>(K);
  const T* n = static_cast<const T*>(nextK);
  switch (words) {
    case 4:
      return launch_pdl(seg_cosine_kernel<T, 1>, grid, dim3(kSegThreads), smem, st, k, n, n_frames, d, g, skip_mask,
                        sim, ld_sim);
    case 8:
      return launch_pdl(seg_cosine_kernel<T, 2>, grid, dim3(kSegThreads), smem, st, k, n, n_frames, d, g, skip_mask,
                        sim, ld_sim);
    case 16:
      return launch_pdl(seg_cosine_kernel<T, 4>, grid, dim3(kSegThreads), smem, st, k, n, n_frames, d, g, skip_mask,
                        sim, ld_sim);
    case 32:
      return launch_pdl(seg_cosine_kernel<T, 8>, grid, dim3(kSegThreads), smem, st, k, n, n_frames, d, g, skip_mask,
                        sim, ld_sim);
    default:
      return launch_pdl(seg_cosine_kernel<T, 0>, grid, dim3(kSegThreads), smem, st, k, n, n_frames, d, g, skip_mask,
                        sim, ld_sim);
  }
}

cudaError_t launch_seg_cosine_ld(const void* K, const void* nextK, kvb_dtype dtype, int H, int n_frames, int d,
                                 const SegGeom& g, unsigned long long skip_mask, float* sim, int ld_sim,
                                 cudaStream_t st) {
  if (H <= 0 || n_frames <= 0) return cudaSuccess;
  dim3 grid(g.seg_rows, n_frames, H);
  const size_t smem = sizeof(float) * g.seg_h * g.frame_w;
  LaunchTrace trace("seg_cosine_kernel", st);
  if (dtype == KVB_BF16)
    return launch_seg_typed<__nv_bfloat16>(K, nextK, n_frames, d, g, skip_mask, sim, ld_sim, grid, smem, st);
  return launch_seg_typed<float>(K, nextK, n_frames, d, g, skip_mask, sim, ld_sim, grid, smem, st);
}

cudaError_t launch_prune_plan(const PrunePlan& p, cudaStream_t st) {
  LaunchTrace trace("prune_plan_kernel", st);
  return launch_pdl(prune_plan_kernel, dim3(p.H), dim3(kPlanThreads), 0, st, p);
}

cudaError_t launch_prune_gather(const PrunePlan& p, cudaStream_t st) {
  LaunchTrace trace("prune_gather_kernel", st);
  return launch_pdl(prune_gather_kernel, dim3(mover_blocks(p.ld_plan, p.row_bytes, p.H), p.H), dim3(256), 0, st, p);
}


}  // namespace kvb
