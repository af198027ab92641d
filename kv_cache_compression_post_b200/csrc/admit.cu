// DensityKV admit step, the parts that are not a density contraction
// (DensityKV App. B.1 "Online Bank Update", §3, App. E default policy):
//
//   count     per head: mean frozen baseline of the bank, number of candidates
//             whose disturbance score rho_B(c) / mean rho0 is <= tau
//   select    P = min over heads (synchronised prefix) of the feasible counts,
//             capped by M and N (and by an outside bound when the layer's heads
//             are split across banks); each head keeps its P lowest (score, id)
//             keys (radix select over 64-bit composite keys: exact, tie-free)
//   evict     projected ratio (rho_i + sum_A phi) / rho0_i; every entry above tau
//             is evicted, then max(0, |B| - mandatory + P - M) more by (ratio
//             descending, id ascending) -- another radix select
//
// App. E's ablation switches change only keys and flags of these kernels: source
// candidate order (the feasible prefix is the leading run in id order, admitted
// by id), densest-only eviction (no threshold step, capacity cut by projected
// density), source-order completion (capacity cut by id), refreshed baselines
// (finalize writes rho0 = rho for every entry).
//   compact   admitted entries fill the evicted slots below the new size, then
//             append; surviving entries beyond the new size move into the
//             remaining holes, so every bank stays dense in [0, size)
//   finalize  incremental densities: survivors rho + sum_A phi - sum_E phi,
//             new entries rho_B(c) - sum_E phi + sum_{A, c' != c} phi, and new
//             baselines rho0 = rho (co-admitted entries set them together)
//
// The selection kernels run one 1024-thread CTA per head (latency-bound, a few
// microseconds); the row movers move each K/V row with a group of lanes, one
// 16-byte word per lane, over a grid of about one wave.
#include <climits>

#include "admit.cuh"
#include "host_util.h"
#include "kvb_device.cuh"

namespace kvb {
namespace {

constexpr int kSelThreads = 1024;
// banks whose 64-bit keys and flag bytes fit in this many bytes keep them in shared memory
constexpr size_t kEvictKeyBytes = 216 * 1024;

// the radix histogram is split in kHistCopies copies (warp w counts into copy
// w % kHistCopies): keys that share a digit then contend on an address only
// within their group of warps
constexpr int kHistCopies = 8;

struct SelShared {
  unsigned int hist[kHistCopies][256];
  unsigned long long kmin[32], kmax[32];
  unsigned long long prefix, mask;
  int kRem;
  int done;
  int warp_tot[32];
  float fred[32];
};

__device__ __forceinline__ float block_sum(float v, SelShared* S) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) S->fred[w] = v;
  __syncthreads();
  float t = 0.f;
  if (w == 0) {
    t = (l < static_cast<int>(blockDim.x >> 5)) ? S->fred[l] : 0.f;
    t = warp_sum(t);
    if (l == 0) S->fred[0] = t;
  }
  __syncthreads();
  t = S->fred[0];
  __syncthreads();
  return t;
}

// block-wide max (min via negation); every thread receives the result
__device__ __forceinline__ float block_max(float v, SelShared* S) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) S->fred[w] = v;
  __syncthreads();
  float t = -INFINITY;
  if (w == 0) {
    t = (l < static_cast<int>(blockDim.x >> 5)) ? S->fred[l] : -INFINITY;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t = fmaxf(t, __shfl_xor_sync(0xffffffffu, t, o));
    if (l == 0) S->fred[0] = t;
  }
  __syncthreads();
  t = S->fred[0];
  __syncthreads();
  return t;
}

// Near-tie accounting (the decisions another rounding could take the other way):
// a value within kTieMargin, relative, of its threshold, or a cut whose two sides
// (last value taken, first value left) are that close.  Counted per head into
// kvb_admit_stats.near_ties from the kernels' own fp32 values.
constexpr float kTieMargin = 1e-4f;
__device__ __forceinline__ bool near_tau(float v, float tau) { return fabsf(v - tau) < kTieMargin * tau; }
__device__ __forceinline__ bool near_cut(float taken, float left) {
  return taken != 0.f && fabsf(left - taken) < kTieMargin * fabsf(taken);
}

// exclusive scan over the block; *total receives the sum
__device__ __forceinline__ int block_excl_scan(int v, SelShared* S, int* total) {
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (l >= o) incl += t;
  }
  __syncthreads();
  if (l == 31) S->warp_tot[w] = incl;
  __syncthreads();
  if (w == 0) {
    const int nw = blockDim.x >> 5;
    int x = (l < nw) ? S->warp_tot[l] : 0;
    int xi = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, xi, o);
      if (l >= o) xi += t;
    }
    if (l < nw) S->warp_tot[l] = xi - x;  // exclusive warp offsets
    if (l == nw - 1) S->kRem = xi;        // reuse as total holder
  }
  __syncthreads();
  const int res = S->warp_tot[w] + incl - v;
  *total = S->kRem;
  __syncthreads();
  return res;
}

// Write, in ascending order, every i in [lo, hi) with pred(i) to out; returns count.
template <class Pred>
__device__ int block_compact(int lo, int hi, Pred pred, int* out, SelShared* S) {
  const int n = hi > lo ? hi - lo : 0;
  const int chunk = (n + blockDim.x - 1) / blockDim.x;
  const int b = lo + threadIdx.x * chunk, e = min(hi, b + chunk);
  int cnt = 0;
  for (int i = b; i < e; ++i) cnt += pred(i) ? 1 : 0;
  int total;
  int pos = block_excl_scan(cnt, S, &total);
  if (out)
    for (int i = b; i < e; ++i)
      if (pred(i)) out[pos++] = i;
  __syncthreads();
  return total;
}

// Radix select of the k smallest 64-bit keys among {i < n : keep(i)} (1 <= k <
// count).  On return S->prefix / S->mask define the selection:
// keep(i) && (key(i) & mask) <= prefix.  Keys are unique (they carry the id).
// A key of all ones is a sentinel for entries that are never among the k
// smallest (they are larger than every other key).
//
// The bits every candidate key shares (the common prefix of the smallest and the
// largest non-sentinel key) are skipped: at these sizes the keys of one call often
// agree on their top byte (ratios in [1, 2), say), and a pass over it would send
// every key to one histogram bin.  Each warp counts into one of kHistCopies
// copies of the histogram, so a crowded bin is contended only within a group of
// warps; the copies are summed when the digit is chosen.
template <class KeyFn, class KeepFn>
__device__ void block_radix_select(int n, int k, KeyFn key, KeepFn keep, SelShared* S) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = static_cast<int>(blockDim.x >> 5);
  unsigned long long lo = ~0ull, hi = 0ull;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    if (!keep(i)) continue;
    const unsigned long long kk = key(i);
    if (kk == ~0ull) continue;
    lo = kk < lo ? kk : lo;
    hi = kk > hi ? kk : hi;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long a = __shfl_xor_sync(0xffffffffu, lo, o), b = __shfl_xor_sync(0xffffffffu, hi, o);
    lo = a < lo ? a : lo;
    hi = b > hi ? b : hi;
  }
  if (lane == 0) {
    S->kmin[warp] = lo;
    S->kmax[warp] = hi;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long mn = ~0ull, mx = 0ull;
    for (int w = 0; w < nwarps; ++w) {
      mn = S->kmin[w] < mn ? S->kmin[w] : mn;
      mx = S->kmax[w] > mx ? S->kmax[w] : mx;
    }
    S->kRem = k;
    S->done = 0;
    if (mn >= mx) {  // one candidate key: it is the selection
      S->prefix = mn;
      S->mask = ~0ull;
      S->done = 1;
    } else {
      // digits start at the byte holding the highest bit where min and max differ
      const int top = 63 - __clzll(static_cast<long long>(mn ^ mx));
      const int shift0 = (top / 8) * 8;
      const unsigned long long above = shift0 >= 56 ? 0ull : ~((1ull << (shift0 + 8)) - 1ull);
      S->prefix = mn & above;
      S->mask = above;
      S->kmin[0] = static_cast<unsigned long long>(shift0);
    }
  }
  __syncthreads();
  if (S->done) return;
  const int shift0 = static_cast<int>(S->kmin[0]);
  for (int shift = shift0; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < kHistCopies * 256; i += blockDim.x) (&S->hist[0][0])[i] = 0u;
    __syncthreads();
    const unsigned long long prefix = S->prefix, mask = S->mask;
    for (int i0 = warp * 32; i0 < n; i0 += blockDim.x) {
      const int i = i0 + lane;
      unsigned int bin = 256u;
      if (i < n && keep(i)) {
        const unsigned long long kk = key(i);
        if ((kk & mask) == prefix) bin = static_cast<unsigned int>((kk >> shift) & 0xFFull);
      }
      // one shared-memory atomic per key: with the histogram copies this measured
      // faster than aggregating equal digits per warp with __match_any_sync
      if (bin < 256u) atomicAdd(&S->hist[warp % kHistCopies][bin], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      unsigned int loc[8];
      unsigned int s = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        unsigned int b = 0u;
#pragma unroll
        for (int c = 0; c < kHistCopies; ++c) b += S->hist[c][lane * 8 + j];
        loc[j] = b;
        s += loc[j];
      }
      unsigned int incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      const unsigned int excl = incl - s;
      const unsigned int kr = static_cast<unsigned int>(S->kRem);
      __syncwarp();
      if (excl < kr && kr <= incl) {
        unsigned int c = excl;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (c + loc[j] >= kr) {
            S->prefix = prefix | (static_cast<unsigned long long>(lane * 8 + j) << shift);
            S->mask = mask | (0xFFull << shift);
            S->kRem = static_cast<int>(kr - c);
            if (loc[j] == kr - c) S->done = 1;
            break;
          }
          c += loc[j];
        }
      }
    }
    __syncthreads();
    if (S->done) break;
  }
}

__device__ __forceinline__ float score_of(float rhoB, float mean0) {
  return mean0 > 0.f ? __fdiv_rn(rhoB, mean0) : 0.f;
}
__device__ __forceinline__ float ratio_of(float rho, float proj, float rho0) {
  return rho0 > 0.f ? __fdiv_rn(rho + proj, rho0) : 0.f;
}

// -------------------------------------------------------------------- kernels
__global__ void __launch_bounds__(kSelThreads) admit_count_kernel(const AdmitPlan p) {
  pdl_wait();
  pdl_trigger();
  __shared__ SelShared S;
  const int h = blockIdx.x;
  const int n = p.size[h];
  // each thread adds its baselines in index order; four loads in flight per round
  constexpr int kU = 4;
  const float* r0h = p.rho0 + static_cast<size_t>(h) * p.M;
  float s = 0.f;
  for (int i0 = threadIdx.x; i0 < n; i0 += kU * static_cast<int>(blockDim.x)) {
    float v[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int i = i0 + u * static_cast<int>(blockDim.x);
      v[u] = i < n ? __ldg(r0h + i) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kU; ++u)
      if (i0 + u * static_cast<int>(blockDim.x) < n) s += v[u];
  }
  const float sum = block_sum(s, &S);
  const float mean0 = n > 0 ? sum / static_cast<float>(n) : 0.f;
  const float* rb = p.rhoB + static_cast<size_t>(h) * p.ldN;
  int cnt = 0;
  if (p.cand_order == KVB_ORDER_SOURCE) {
    // the leading run in id order: every candidate below the lowest infeasible id
    __shared__ unsigned int s_first_bad;
    if (threadIdx.x == 0) s_first_bad = UINT_MAX;
    __syncthreads();
    for (int c = threadIdx.x; c < p.N; c += blockDim.x)
      if (!(score_of(rb[c], mean0) <= p.tau)) atomicMin(&s_first_bad, static_cast<unsigned int>(p.cand_ids[c]));
    __syncthreads();
    const unsigned int bad = s_first_bad;
    for (int c = threadIdx.x; c < p.N; c += blockDim.x) cnt += (static_cast<unsigned int>(p.cand_ids[c]) < bad) ? 1 : 0;
  }
  // admission-threshold near ties (scores exist only against a bank with a mean baseline)
  const bool scored = n > 0 && mean0 > 0.f;
  int nt = 0;
  for (int c0 = threadIdx.x; c0 < p.N; c0 += kU * static_cast<int>(blockDim.x)) {
    float v[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int c = c0 + u * static_cast<int>(blockDim.x);
      v[u] = c < p.N ? rb[c] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      if (c0 + u * static_cast<int>(blockDim.x) >= p.N) break;
      const float sc = score_of(v[u], mean0);
      if (p.cand_order != KVB_ORDER_SOURCE) cnt += (sc <= p.tau) ? 1 : 0;
      nt += (scored && near_tau(sc, p.tau)) ? 1 : 0;
    }
  }
  int total, ties;
  block_excl_scan(cnt, &S, &total);
  block_excl_scan(nt, &S, &ties);
  if (threadIdx.x == 0) {
    p.mean0[h] = mean0;
    p.feasible[h] = total;
    p.n_old[h] = n;
    p.stats[h].near_ties = ties;
  }
}

__global__ void __launch_bounds__(kSelThreads) admit_select_kernel(const AdmitPlan p) {
  pdl_wait();
  pdl_trigger();
  __shared__ SelShared S;
  __shared__ int sPt;
  const int h = blockIdx.x;
  if (threadIdx.x < 32) {
    // the shared prefix: one warp loads the heads' feasible counts side by side
    int v = p.feasible[h];
    if (p.sync_heads)
      for (int g = threadIdx.x; g < p.H; g += 32) v = min(v, p.feasible[g]);
    for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (threadIdx.x == 0) sPt = v;
  }
  __syncthreads();
  int Pt = sPt;
  if (p.p_bound) Pt = min(Pt, max(0, *p.p_bound));
  const int P = min(Pt, min(p.M, p.N));
  const float mean0 = p.mean0[h];
  const float* rb = p.rhoB + static_cast<size_t>(h) * p.ldN;
  int* out = p.adm_idx + static_cast<size_t>(h) * p.ldN;
  const bool by_source = p.cand_order == KVB_ORDER_SOURCE;
  auto key = [&](int c) -> unsigned long long {
    const unsigned long long hi = by_source ? 0ull : static_cast<unsigned long long>(float_key(score_of(rb[c], mean0)));
    return (hi << 32) | static_cast<unsigned int>(p.cand_ids[c]);
  };
  auto all = [](int) { return true; };
  if (P >= p.N) {
    for (int c = threadIdx.x; c < p.N; c += blockDim.x) out[c] = c;
  } else if (P > 0) {
    block_radix_select(p.N, P, key, all, &S);
    const unsigned long long prefix = S.prefix, mask = S.mask;
    const int got = block_compact(0, p.N, [&](int c) { return (key(c) & mask) <= prefix; }, out, &S);
    if (threadIdx.x == 0 && got != P) latch_status(p.status, KVB_E_DEVICE_BOUNDS);
    if (!by_source && P < p.feasible[h]) {
      // the cut inside the feasible set: last admitted score vs first rejected one
      float lo = -INFINITY, nhi = -INFINITY;
      for (int c = threadIdx.x; c < p.N; c += blockDim.x) {
        const float sc = score_of(rb[c], mean0);
        if ((key(c) & mask) <= prefix) lo = fmaxf(lo, sc);
        else nhi = fmaxf(nhi, -sc);
      }
      lo = block_max(lo, &S);
      nhi = block_max(nhi, &S);
      if (threadIdx.x == 0 && near_cut(lo, -nhi)) p.stats[h].near_ties += 1;
    }
  }
  if (threadIdx.x == 0) {
    p.P[h] = P;
    p.stats[h].admitted = P;
    p.stats[h].feasible = p.feasible[h];
  }
}

__global__ void feasible_min_kernel(const AdmitPlan p, int* out) {
  pdl_wait();
  pdl_trigger();
  int v = min(p.M, p.N);
  for (int h = threadIdx.x; h < p.H; h += 32) v = min(v, p.feasible[h]);
  for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
  if (threadIdx.x == 0) out[0] = v;
}

// Two rows per lane group and iteration, every load before the first store.
__global__ void gather_admitted_kernel(const AdmitPlan p) {
  pdl_wait();
  pdl_trigger();
  const int h = blockIdx.y;
  const RowGroup g = row_group(p.row_bytes);
  const int P = p.P[h];
  // bf16: a head that admits every candidate has its admitted block read in place
  // by the density passes (the admitted indices are then 0..N-1)
  if (p.dtype == KVB_BF16 && P >= p.N) return;
  const char* cK = static_cast<const char*>(p.candK);
  char* EA = static_cast<char*>(p.EA);
  for (int w0 = g.first; w0 < P; w0 += 2 * g.stride) {
    RowWords rw[2];
    int c[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int w = w0 + u * g.stride;
      c[u] = w < P ? p.adm_idx[static_cast<size_t>(h) * p.ldN + w] : -1;
    }
#pragma unroll
    for (int u = 0; u < 2; ++u)
      if (c[u] >= 0)
        load_rows(rw[u], cK + (static_cast<size_t>(h) * p.N + c[u]) * p.row_bytes, nullptr,
                  p.caug + (static_cast<size_t>(h) * p.ldN + c[u]) * 32, p.row_bytes, g);
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (c[u] < 0) continue;
      const size_t dst = static_cast<size_t>(h) * p.ldEA + p.M + w0 + u * g.stride;
      store_rows(rw[u], EA + dst * p.row_bytes, nullptr, p.EAaug + dst * 32, p.row_bytes, g);
    }
  }
}

// Exclusive scan of three counts packed in one 64-bit word (21 bits each: counts
// below 2^21) over the block; returns this thread's offsets, *total the totals.
__device__ __forceinline__ unsigned long long block_excl_scan3(unsigned long long v, SelShared* S,
                                                               unsigned long long* total) {
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  unsigned long long incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long t = __shfl_up_sync(0xffffffffu, incl, o);
    if (l >= o) incl += t;
  }
  __syncthreads();
  if (l == 31) S->kmin[w] = incl;
  __syncthreads();
  if (w == 0) {
    const int nw = blockDim.x >> 5;
    const unsigned long long x = (l < nw) ? S->kmin[l] : 0ull;
    unsigned long long xi = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long t = __shfl_up_sync(0xffffffffu, xi, o);
      if (l >= o) xi += t;
    }
    if (l < nw) S->kmin[l] = xi - x;   // exclusive warp offsets
    if (l == nw - 1) S->kmax[0] = xi;  // totals
  }
  __syncthreads();
  const unsigned long long res = S->kmin[w] + incl - v;
  *total = S->kmax[0];
  __syncthreads();
  return res;
}

// SKEYS: every entry's 64-bit key is computed once into shared memory (the radix
// passes then read 8 bytes of shared memory instead of recomputing the ratio), and
// its eviction flag (0 survivor, 1 above tau, 2 capacity) sits beside it, so the
// lists built at the end (evicted slots, holes, tail survivors) come from one pass
// over shared memory; mandatory evictions get the largest key, so the selection
// needs no flags.  Without SKEYS (banks too large for shared memory) keys are
// recomputed and flags live in global memory.
template <bool SKEYS>
__global__ void __launch_bounds__(kSelThreads) evict_select_kernel(const AdmitPlan p) {
  pdl_wait();
  pdl_trigger();
  __shared__ SelShared S;
  extern __shared__ unsigned long long s_key[];  // [M] keys, then [M] flag bytes (SKEYS)
  uint8_t* s_flag = reinterpret_cast<uint8_t*>(s_key + p.M);
  const int h = blockIdx.x;
  const int n = p.n_old[h];
  const int Ph = p.P[h];
  const size_t base = static_cast<size_t>(h) * p.M;
  const float* rho = p.rho + base;
  const float* rho0 = p.rho0 + base;
  const float* proj = p.proj + base;
  const int* ids = p.ids + base;
  int* evflag = p.tail + base;  // global flags (no SKEYS) live in the tail array until the tail list is built
  auto getf = [&](int i) -> int { return SKEYS ? static_cast<int>(s_flag[i]) : evflag[i]; };
  auto setf = [&](int i, int v) {
    if (SKEYS) s_flag[i] = static_cast<uint8_t>(v);
    else evflag[i] = v;
  };
  auto ratio = [&](int i) { return ratio_of(rho[i], proj[i], rho0[i]); };
  const int mode = p.evict_order;
  // the capacity-cut key of a non-mandatory entry (ascending = evicted first):
  // ratio descending (default), projected density descending (densest-only), or
  // nothing (source order); id ascending breaks ties.  Ratios and densities are
  // >= 0, so no such key has the top byte 0xFF of the mandatory entries' key.
  auto cut_key_of = [&](float r, float dens, int id) -> unsigned long long {
    unsigned long long hi = 0ull;
    if (mode == KVB_EVICT_THRESHOLD_RATIO) hi = ~float_key(r);
    else if (mode == KVB_EVICT_DENSEST) hi = ~float_key(dens);
    return (hi << 32) | static_cast<unsigned int>(id);
  };
  auto cut_key = [&](int i, float r) { return cut_key_of(r, rho[i] + proj[i], ids[i]); };
  // mandatory evictions: projected growth above tau (none when densest-only);
  // near ties at the threshold are counted on the way.  Each thread takes four
  // entries per round and issues all their loads before using any (one memory
  // latency per round instead of one per entry)
  int cnt = 0, nt = 0;
  constexpr int kU = 4;
  for (int i0 = threadIdx.x; i0 < n; i0 += kU * static_cast<int>(blockDim.x)) {
    float rv[kU], pv[kU], r0v[kU];
    int idv[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int i = i0 + u * static_cast<int>(blockDim.x);
      const bool in = i < n;
      rv[u] = in ? __ldg(rho + i) : 0.f;
      pv[u] = in ? __ldg(proj + i) : 0.f;
      r0v[u] = in ? __ldg(rho0 + i) : 0.f;
      idv[u] = in ? __ldg(ids + i) : 0;
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int i = i0 + u * static_cast<int>(blockDim.x);
      if (i >= n) break;
      const float r = ratio_of(rv[u], pv[u], r0v[u]);
      const bool m = mode != KVB_EVICT_DENSEST && r > p.tau;
      setf(i, m ? 1 : 0);
      cnt += m ? 1 : 0;
      nt += (mode != KVB_EVICT_DENSEST && near_tau(r, p.tau)) ? 1 : 0;
      if (SKEYS) s_key[i] = m ? ~0ull : cut_key_of(r, rv[u] + pv[u], idv[u]);
    }
  }
  int n_mand, ties;
  block_excl_scan(cnt, &S, &n_mand);
  block_excl_scan(nt, &S, &ties);
  const int ecap = max(0, n - n_mand + Ph - p.M);
  const int n_free = n - n_mand;
  if (ecap > 0) {
    auto key = [&](int i) -> unsigned long long {
      if (SKEYS) return s_key[i];
      return cut_key(i, ratio(i));
    };
    auto keep = [&](int i) { return SKEYS || evflag[i] == 0; };
    if (ecap >= n_free) {
      for (int i = threadIdx.x; i < n; i += blockDim.x) setf(i, 1);
    } else {
      block_radix_select(n, ecap, key, keep, &S);
      const unsigned long long prefix = S.prefix, mask = S.mask;
      for (int i = threadIdx.x; i < n; i += blockDim.x)
        if (getf(i) == 0 && (key(i) & mask) <= prefix) setf(i, 2);
    }
  }
  __syncthreads();
  // near ties: projected ratios within the margin of tau, and the capacity cut
  // (last capacity eviction vs first non-mandatory survivor by the cut value)
  {
    if (ecap > 0 && ecap < n_free && mode != KVB_EVICT_THRESHOLD_SOURCE) {
      float lo = -INFINITY, hi = -INFINITY;  // lo holds -min over the evicted
      for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int f = getf(i);
        if (f == 1) continue;
        // the cut value: read back from the key when the keys are in shared memory
        const float v = SKEYS ? key_float(~static_cast<uint32_t>(s_key[i] >> 32))
                              : ((mode == KVB_EVICT_DENSEST) ? rho[i] + proj[i] : ratio(i));
        if (f == 2) lo = fmaxf(lo, -v);
        else hi = fmaxf(hi, v);
      }
      lo = block_max(lo, &S);
      hi = block_max(hi, &S);
      if (near_cut(-lo, hi)) ties += 1;
    }
    if (threadIdx.x == 0) p.stats[h].near_ties += ties;
  }
  const int E = n_mand + min(ecap, n_free);
  const int n_new = n - E + Ph;
  int* ev = p.ev_slot + base;
  int* tmp = p.newp + base;
  __shared__ int s_ntail, s_gotE, s_nh;
  if (SKEYS) {
    // one ordered pass over contiguous chunks: the evicted slots (ascending), the
    // number of them below the new size (holes), and the survivors at or above
    // the new size (they move into holes), listed ascending into the tail array
    const int chunk = (n + blockDim.x - 1) / blockDim.x;
    const int b0 = threadIdx.x * chunk, b1 = min(n, b0 + chunk);
    unsigned long long c3 = 0ull;
    for (int i = b0; i < b1; ++i) {
      const int f = s_flag[i];
      c3 += (f != 0) ? 1ull : 0ull;
      c3 += (f != 0 && i < n_new) ? (1ull << 21) : 0ull;
      c3 += (f == 0 && i >= n_new) ? (1ull << 42) : 0ull;
    }
    unsigned long long tot;
    const unsigned long long off = block_excl_scan3(c3, &S, &tot);
    int pe = static_cast<int>(off & 0x1FFFFFull), pt = static_cast<int>((off >> 42) & 0x1FFFFFull);
    for (int i = b0; i < b1; ++i) {
      const int f = s_flag[i];
      if (f != 0) ev[pe++] = i;
      else if (i >= n_new) evflag[pt++] = i;
    }
    if (threadIdx.x == 0) {
      s_gotE = static_cast<int>(tot & 0x1FFFFFull);
      s_nh = static_cast<int>((tot >> 21) & 0x1FFFFFull);
      s_ntail = static_cast<int>((tot >> 42) & 0x1FFFFFull);
    }
    __syncthreads();
  } else {
    const int gotE = block_compact(0, n, [&](int i) { return evflag[i] != 0; }, ev, &S);
    const int nh = block_compact(0, n, [&](int i) { return evflag[i] != 0 && i < n_new; }, nullptr, &S);
    // survivors at or above the new size move into holes; list them (ascending):
    // count first (flags are still needed), then write the list over the flag array
    const int ntl = block_compact(n_new < n ? n_new : n, n, [&](int i) { return evflag[i] == 0; }, nullptr, &S);
    if (threadIdx.x == 0) {
      s_ntail = ntl;
      s_gotE = gotE;
      s_nh = nh;
    }
    __syncthreads();
    // the tail list is short; build it in the newp scratch and copy it over the flags
    block_compact(n_new < n ? n_new : n, n, [&](int i) { return evflag[i] == 0; }, tmp, &S);
    for (int k = threadIdx.x; k < s_ntail; k += blockDim.x) evflag[k] = tmp[k];
    __syncthreads();
  }
  // every slot of the new bank starts as an old, unmoved entry
  const int top = max(n, n_new);
  for (int i = threadIdx.x; i < top; i += blockDim.x) tmp[i] = -1;
  if (threadIdx.x == 0) {
    if (s_gotE != E) latch_status(p.status, KVB_E_DEVICE_BOUNDS);
    p.E[h] = E;
    p.nhole[h] = s_nh;
    p.ntail[h] = s_ntail;
    p.EAoff[h] = p.M - E;
    p.EAcnt[h] = E;
    p.size[h] = n_new;
    p.stats[h].mandatory = n_mand;
    p.stats[h].capacity_evicted = E - n_mand;
    p.stats[h].size = n_new;
    p.stats[h].moved = s_ntail;
  }
}

__global__ void gather_evicted_kernel(const AdmitPlan p) {
  pdl_wait();
  pdl_trigger();
  const int h = blockIdx.y;
  const RowGroup g = row_group(p.row_bytes);
  const int E = p.E[h];
  const char* K = static_cast<const char*>(p.K);
  char* EA = static_cast<char*>(p.EA);
  for (int w0 = g.first; w0 < E; w0 += 2 * g.stride) {
    RowWords rw[2];
    int slot[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int w = w0 + u * g.stride;
      slot[u] = w < E ? p.ev_slot[static_cast<size_t>(h) * p.M + w] : -1;
    }
#pragma unroll
    for (int u = 0; u < 2; ++u)
      if (slot[u] >= 0) {
        const size_t src = static_cast<size_t>(h) * p.M + slot[u];
        load_rows(rw[u], K + src * p.row_bytes, nullptr, p.aug + src * 32, p.row_bytes, g);
      }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (slot[u] < 0) continue;
      const size_t dst = static_cast<size_t>(h) * p.ldEA + (p.M - E) + w0 + u * g.stride;
      store_rows(rw[u], EA + dst * p.row_bytes, nullptr, p.EAaug + dst * 32, p.row_bytes, g);
    }
  }
}

// moves: [0, P) admitted candidates, [P, P + ntail) surviving tail entries.  Two
// moves per lane group and iteration, every load before the first store (sources
// and destinations are disjoint: destinations are evicted slots or slots past the
// old size, sources candidates or survivors at or past the new size).
__global__ void compact_kernel(const AdmitPlan p) {
  pdl_wait();
  pdl_trigger();
  const int h = blockIdx.y;
  const RowGroup g = row_group(p.row_bytes);
  const int P = p.P[h], nt = p.ntail[h], nh = p.nhole[h], n_old = p.n_old[h];
  const size_t base = static_cast<size_t>(h) * p.M;
  const int* hole = p.ev_slot + base;  // evicted slots ascending: the first nh are holes
  char* K = static_cast<char*>(p.K);
  char* V = static_cast<char*>(p.V);
  const char* cK = static_cast<const char*>(p.candK);
  const char* cV = static_cast<const char*>(p.candV);
  for (int w0 = g.first; w0 < P + nt; w0 += 2 * g.stride) {
    int src[2], dst[2];  // src: candidate index (admitted) or bank slot (tail); -1: nothing to move
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int w = w0 + u * g.stride;
      src[u] = dst[u] = -1;
      if (w < P) {
        dst[u] = (w < nh) ? hole[w] : n_old + (w - nh);
        src[u] = p.adm_idx[static_cast<size_t>(h) * p.ldN + w];
      } else if (w < P + nt) {
        src[u] = p.tail[base + (w - P)];
        dst[u] = hole[w];
        if (src[u] < 0 || src[u] >= p.M) dst[u] = -1;
      }
      if (dst[u] < 0 || dst[u] >= p.M) {
        if (w < P + nt && g.sub == 0) latch_status(p.status, KVB_E_DEVICE_BOUNDS);
        src[u] = dst[u] = -1;
      }
    }
    RowWords rw[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (src[u] < 0) continue;
      if (w0 + u * g.stride < P) {
        const size_t srow = static_cast<size_t>(h) * p.N + src[u];
        load_rows(rw[u], cK + srow * p.row_bytes, cV + srow * p.row_bytes,
                  p.caug + (static_cast<size_t>(h) * p.ldN + src[u]) * 32, p.row_bytes, g);
      } else {
        const size_t sb = base + src[u];
        load_rows(rw[u], K + sb * p.row_bytes, V + sb * p.row_bytes, p.aug + sb * 32, p.row_bytes, g);
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (src[u] < 0) continue;
      const int w = w0 + u * g.stride;
      const size_t db = base + dst[u];
      store_rows(rw[u], K + db * p.row_bytes, V + db * p.row_bytes, p.aug + db * 32, p.row_bytes, g);
      if (g.sub != 0) continue;
      if (w < P) {
        const int c = src[u];
        p.ids[db] = p.cand_ids[c];
        p.rho[db] = p.rhoB[static_cast<size_t>(h) * p.ldN + c];
        p.newp[db] = w;
      } else {
        const size_t sb = base + src[u];
        p.ids[db] = p.ids[sb];
        p.rho0[db] = p.rho0[sb];
        p.rho[db] = p.rho[sb] + p.proj[sb];
        p.newp[db] = -2;
      }
    }
  }
}

__global__ void finalize_kernel(const AdmitPlan p) {
  pdl_wait();
  pdl_trigger();
  const int h = blockIdx.y;
  const int s = blockIdx.x * blockDim.x + threadIdx.x;
  const int n_new = p.size[h];
  if (s >= n_new) return;
  const size_t i = static_cast<size_t>(h) * p.M + s;
  const int tag = p.newp[i];
  float v = p.rho[i] + p.sub[i];
  if (tag == -1) {
    v += p.proj[i];
  } else if (tag >= 0) {
    v += p.coadm[static_cast<size_t>(h) * p.ldN + tag];
  }
  // new entries set their baselines after the update; refreshed baselines follow
  // every entry's density in the updated bank
  if (tag >= 0 || p.baselines == KVB_BASELINES_REFRESH) p.rho0[i] = v;
  p.rho[i] = v;
}

}  // namespace

cudaError_t launch_admit_count(const AdmitPlan& p, cudaStream_t st) {
  LaunchTrace trace("admit_count_kernel", st);
  return launch_pdl(admit_count_kernel, dim3(p.H), dim3(kSelThreads), 0, st, p);
}
cudaError_t launch_feasible_min(const AdmitPlan& p, int* out, cudaStream_t st) {
  LaunchTrace trace("feasible_min_kernel", st);
  return launch_pdl(feasible_min_kernel, dim3(1), dim3(32), 0, st, p, out);
}
cudaError_t launch_admit_select(const AdmitPlan& p, cudaStream_t st) {
  LaunchTrace trace("admit_select_kernel", st);
  return launch_pdl(admit_select_kernel, dim3(p.H), dim3(kSelThreads), 0, st, p);
}
cudaError_t launch_gather_admitted(const AdmitPlan& p, int maxP, cudaStream_t st) {
  if (maxP <= 0) return cudaSuccess;
  LaunchTrace trace("gather_admitted_kernel", st);
  return launch_pdl(gather_admitted_kernel, dim3(mover_blocks(maxP, p.row_bytes, p.H), p.H), dim3(256), 0, st, p);
}
cudaError_t launch_evict_select(const AdmitPlan& p, cudaStream_t st) {
  // keys (8 bytes) and flags (1 byte) of every entry in shared memory
  const size_t keys = (sizeof(unsigned long long) + 1) * static_cast<size_t>(p.M);
  if (keys <= kEvictKeyBytes) {
    cudaError_t e = cudaFuncSetAttribute(evict_select_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(keys));
    if (e != cudaSuccess) return e;
    LaunchTrace trace("evict_select_kernel", st);
    return launch_pdl(evict_select_kernel<true>, dim3(p.H), dim3(kSelThreads), keys, st, p);
  } else {
    LaunchTrace trace("evict_select_kernel", st);
    return launch_pdl(evict_select_kernel<false>, dim3(p.H), dim3(kSelThreads), 0, st, p);
  }
}
cudaError_t launch_gather_evicted(const AdmitPlan& p, cudaStream_t st) {
  LaunchTrace trace("gather_evicted_kernel", st);
  return launch_pdl(gather_evicted_kernel, dim3(mover_blocks(p.M, p.row_bytes, p.H), p.H), dim3(256), 0, st, p);
}
cudaError_t launch_compact(const AdmitPlan& p, cudaStream_t st) {
  LaunchTrace trace("compact_kernel", st);
  return launch_pdl(compact_kernel, dim3(mover_blocks(p.N + p.M, p.row_bytes, p.H), p.H), dim3(256), 0, st, p);
}
cudaError_t launch_finalize(const AdmitPlan& p, cudaStream_t st) {
  LaunchTrace trace("finalize_kernel", st);
  return launch_pdl(finalize_kernel, dim3((p.M + 255) / 256, p.H), dim3(256), 0, st, p);
}

}  // namespace kvb
