// Attention over ragged per-head segment lists on the 5th-generation tensor cores.
//
// Work is a set of units, one per (head, pair of 128-query tiles A and B); a unit
// walks its head's 128-key tiles.  The kernel is persistent: every CTA takes an
// equal share of the total (unit, key tile) work as one contiguous range (a
// stream-K split), so heads of very different history length (DensityKV bank
// sizes, Forcing-KV static vs dynamic heads) and unit counts that are not a
// multiple of the SM count still keep every SM busy to the end.  A unit cut by a
// range boundary is finished by whichever of its pieces arrives last: every piece
// stores its unnormalised partial (O, running max, running sum) and bumps an
// arrival counter; the last one merges them, so no CTA ever waits for another.
//
// Per key tile j and query tile t of a unit:
//     S_t = Q_t K_j^T          tcgen05.mma, Q and K in shared memory, fp32 in TMEM
//     P_t = exp2(S_t*c - m)    4 softmax warps per query tile, one thread per row;
//                              P (bf16) is written back into S_t's own columns
//     O_t += P_t V_j           tcgen05.mma with A read from TMEM, V read MN-major
//                              straight from its TMA tile
// TMEM holds S_A, S_B, O_A, O_B (4 x 128 columns).  The MMA warp issues
// PV_A(j-1), S_A(j), PV_B(j-1), S_B(j): while one query tile's softmax runs, the
// tensor core works through the other tile's pair of MMAs.  Tensor-core
// instructions of one thread execute in issue order, so S_t(j) overwriting P_t
// once PV_t(j-1) has been issued is safe.  The running max only moves when it
// grows by more than 8 (log2 units); the O rescale (a TMEM read-modify-write) is
// then rare and P stays below 2^8.  K and V stream through separate TMA
// rings (2 stages each), each fed by its own producer thread.
//
// Warp roles: 0 Q/K producer, 1 MMA issuer, 2 TMEM owner, 3 V producer,
// 4-7 softmax/epilogue of query tile A, 8-11 of query tile B.
#include <cuda_bf16.h>

#include <cfloat>
#include <cmath>

#include "attend.cuh"
#include "host_util.h"
#include "kvb_device.cuh"
#include "sm100.cuh"

namespace kvb {
using namespace sm100;

namespace {

constexpr int kThreads = 384;
constexpr int kTile = 128;  // queries per query tile and keys per key tile
constexpr int kBarBytes = 256;
constexpr float kRescaleThreshold = 8.f;
// scheduling cost of one key tile: for a unit of two query tiles / a lone tile
constexpr int kW2 = 8;
constexpr int kW1 = 7;
// a CTA's share is at least this many key tiles of a two-tile unit
constexpr int kMinTilesPerCta = 8;
// K and V ring depths (a third K stage measured no faster: the loop is bound by
// the tensor-core issue of its 128x128x16 MMAs, not by key-tile arrival)
constexpr int kKStages = 2;
constexpr int kVStages = 2;

struct alignas(8) AttnBars {
  uint64_t q_full, q_empty;
  uint64_t k_full[kKStages], k_empty[kKStages], v_full[kVStages], v_empty[kVStages];
  uint64_t s_full[2], p_full[2], o_full[2];  // per query tile
  uint64_t mma_done;
  uint32_t tmem_base;
  uint64_t grp[2];  // per query tile: its four softmax warps meet here (bounded waits)
  int abort;
  int last[2];  // per query tile: this piece merges its unit
};
static_assert(sizeof(AttnBars) <= kBarBytes, "barrier block overflows its reservation");

__device__ __forceinline__ int seg_len(const AttnSeg& s, int h) {
  const int v = s.len_dev ? s.len_dev[h] : s.len_uni;
  return v > 0 ? v : 0;
}
__device__ __forceinline__ int seg_off(const AttnSeg& s, int h) { return s.off_dev ? s.off_dev[h] : s.off_uni; }

__device__ __forceinline__ int head_tiles(const AttnArgs& a, int h) {
  int t = 0;
  for (int s = 0; s < a.nseg; ++s) t += (seg_len(a.seg[s], h) + kTile - 1) / kTile;
  return t;
}

// tile j of head h: its segment, first buffer row and number of valid keys
__device__ __forceinline__ void tile_info(const AttnArgs& a, int h, int j, int& s, int& row, int& nvalid) {
  for (s = 0; s < a.nseg; ++s) {
    const int len = seg_len(a.seg[s], h);
    const int nt = (len + kTile - 1) / kTile;
    if (j < nt) {
      row = seg_off(a.seg[s], h) + j * kTile;
      nvalid = min(kTile, len - j * kTile);
      return;
    }
    j -= nt;
  }
  s = 0;
  row = 0;
  nvalid = 0;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// ------------------------------------------------------------------ schedule
// Unit (h, p) covers query tiles 2p and 2p+1 of head h; units are ordered head by
// head.  Key tile j of unit u starts at cost C_u + w_u * j, where w_u is kW2 (kW1
// for the lone last tile of an odd tile count); it belongs to CTA
// floor(start * G / total), so CTA c takes the starts in [ceil(c*total/G),
// ceil((c+1)*total/G)).
struct SchedShared {
  long long C[65];  // cost prefix over heads
  int T[64];        // key tiles per head
  long long total;
  int G;            // CTAs with a share
};

struct Sched {
  const SchedShared* s;
  int H, npair;
  bool single;
  __device__ int w(int p) const { return (single && p == npair - 1) ? kW1 : kW2; }
  __device__ int ntq(int p) const { return (single && p == npair - 1) ? 1 : 2; }
  __device__ long long start(int h, int p) const { return s->C[h] + static_cast<long long>(p) * kW2 * s->T[h]; }
  __device__ int cta_of(long long x) const { return static_cast<int>((x * s->G) / s->total); }
  __device__ long long lo(int c) const { return (static_cast<long long>(c) * s->total + s->G - 1) / s->G; }
};

struct Piece {
  int h, p, j0, j1, ntq;
  int npieces;  // pieces the unit is cut into (1: this CTA runs it whole)
  int which;    // partial slot of this piece within its CTA (0: its first piece, 1: its last)
  int cfirst;   // CTA holding the unit's first piece
  int wfirst;   // slot of the unit's first piece within that CTA
};

// The pieces of one CTA, in order; every role walks the same sequence.
struct PieceIter {
  int h = 0, p = 0, j = 0, c = 0;
  long long hi = 0;
  bool first = true;

  __device__ void skip_done(const Sched& S) {
    while (h < S.H && (S.s->T[h] == 0 || j >= S.s->T[h])) {
      j = 0;
      if (S.s->T[h] != 0 && ++p < S.npair) continue;
      ++h;
      p = 0;
    }
  }
  __device__ void init(const Sched& S, int cta) {
    c = cta;
    first = true;
    h = S.H;
    if (S.s->total <= 0) return;
    const long long x = S.lo(cta);
    hi = S.lo(cta + 1);
    h = 0;
    while (h < S.H && S.s->C[h + 1] <= x) ++h;
    if (h >= S.H) return;
    p = min(static_cast<int>((x - S.s->C[h]) / (static_cast<long long>(kW2) * S.s->T[h])), S.npair - 1);
    const long long cu = S.start(h, p);
    const int w = S.w(p);
    j = static_cast<int>((x - cu + w - 1) / w);
    skip_done(S);
  }
  __device__ bool next(const Sched& S, Piece& pc) {
    if (h >= S.H) return false;
    const long long cu = S.start(h, p);
    const int w = S.w(p);
    const int T = S.s->T[h];
    if (cu + static_cast<long long>(w) * j >= hi) return false;
    pc.h = h;
    pc.p = p;
    pc.j0 = j;
    pc.j1 = static_cast<int>(min(static_cast<long long>(T), (hi - cu + w - 1) / w));
    pc.ntq = S.ntq(p);
    const int cf = S.cta_of(cu), cl = S.cta_of(cu + static_cast<long long>(w) * (T - 1));
    pc.npieces = cl - cf + 1;
    pc.cfirst = cf;
    pc.which = first ? 0 : 1;
    // the tile just before this unit (in the global order) starts wprev earlier
    const int wprev = (p > 0) ? kW2 : (S.single ? kW1 : kW2);
    pc.wfirst = (cu == 0 || S.cta_of(cu - wprev) < cf) ? 0 : 1;
    first = false;
    j = pc.j1;
    skip_done(S);
    return true;
  }
};

__global__ void __launch_bounds__(kThreads, 1)
    attend_bf16_kernel(const __grid_constant__ AttnMaps maps, const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ SchedShared sch;
  // softmax warps keep their piece walk here, out of the registers of the hot loop
  __shared__ PieceIter s_it[8];
  __shared__ Piece s_pc[8];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int d = a.d;
  const int nbox = d / 64;
  const uint32_t tileBytes = static_cast<uint32_t>(kTile) * d * 2;  // Q, K or V tile
  uint8_t* sQ = smem;                        // Q_A, Q_B
  uint8_t* sK = sQ + 2 * tileBytes;          // kKStages stages
  uint8_t* sV = sK + kKStages * tileBytes;   // kVStages stages
  AttnBars* bars = reinterpret_cast<AttnBars*>(sV + kVStages * tileBytes);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int H = a.H;
  const int nqt = (a.Nq + kTile - 1) / kTile;

  // the segment lengths (bank sizes) come from the previous kernels
  pdl_wait();
  pdl_trigger();

  // ---------------------------------------------------------------- schedule
  if (tid < H) sch.T[tid] = head_tiles(a, tid);
  __syncthreads();
  if (tid == 0) {
    const long long wh = static_cast<long long>(kW2) * (nqt / 2) + ((nqt & 1) ? kW1 : 0);
    long long acc = 0;
    for (int h = 0; h < H; ++h) {
      sch.C[h] = acc;
      acc += wh * sch.T[h];
    }
    sch.C[H] = acc;
    sch.total = acc;
    const long long g = acc / (static_cast<long long>(kW2) * kMinTilesPerCta);
    sch.G = static_cast<int>(max(1ll, min(static_cast<long long>(gridDim.x), g)));
  }
  __syncthreads();
  if (static_cast<int>(blockIdx.x) >= sch.G) return;  // no share of the work
  Sched S;
  S.s = &sch;
  S.H = H;
  S.npair = (nqt + 1) / 2;
  S.single = (nqt & 1) != 0;

  if (tid == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(&bars->k_full[i], 1);
      mbar_init(&bars->k_empty[i], 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(&bars->v_full[i], 1);
      mbar_init(&bars->v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->p_full[i], 4);
      mbar_init(&bars->o_full[i], 1);
      mbar_init(&bars->grp[i], 4);
    }
    mbar_init(&bars->mma_done, 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (warp == 2) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort = &bars->abort;

  if (warp == 0) {
    // ------------------------------------------------------------ Q and K producer
    if (lane == 0) {
      prefetch_tmap(&maps.q);
      bool ok = true;
      int g = 0, np = 0;
      PieceIter it;
      it.init(S, blockIdx.x);
      Piece pc;
      while (ok && it.next(S, pc)) {
        for (int j = pc.j0; j < pc.j1; ++j) {
          int s, row, nv;
          tile_info(a, pc.h, j, s, row, nv);
          const int st = g % kKStages;
          if (!(ok = mbar_wait(&bars->k_empty[st], ((g / kKStages) & 1) ^ 1, abort, a.status))) break;
          mbar_arrive_expect_tx(&bars->k_full[st], tileBytes);
          for (int b = 0; b < nbox; ++b)
            tma_load_3d(sK + st * tileBytes + b * 16384, &maps.k[s], &bars->k_full[st], b * 64, row, pc.h);
          ++g;
          if (j == pc.j0) {
            // this piece's Q, once the previous piece's S MMAs are done
            if (np > 0 && !(ok = mbar_wait(&bars->q_empty, (np - 1) & 1, abort, a.status))) break;
            mbar_arrive_expect_tx(&bars->q_full, pc.ntq * tileBytes);
            for (int t = 0; t < pc.ntq; ++t)
              for (int b = 0; b < nbox; ++b)
                tma_load_3d(sQ + t * tileBytes + b * 16384, &maps.q, &bars->q_full, b * 64,
                            pc.p * 2 * kTile + t * kTile, pc.h);
            ++np;
          }
        }
      }
      if (!ok) {
        // let loads in flight land before the CTA exits
        if (np > 0) mbar_wait_drain(&bars->q_full, (np - 1) & 1, 200000000ull);
        for (int i = max(0, g - kKStages); i < g; ++i)
          mbar_wait_drain(&bars->k_full[i % kKStages], (i / kKStages) & 1, 200000000ull);
      }
    }
  } else if (warp == 3) {
    // ------------------------------------------------------------ V producer
    if (lane == 0) {
      bool ok = true;
      int g = 0;
      PieceIter it;
      it.init(S, blockIdx.x);
      Piece pc;
      while (ok && it.next(S, pc)) {
        for (int j = pc.j0; j < pc.j1; ++j) {
          int s, row, nv;
          tile_info(a, pc.h, j, s, row, nv);
          const int st = g % kVStages;
          if (!(ok = mbar_wait(&bars->v_empty[st], ((g / kVStages) & 1) ^ 1, abort, a.status))) break;
          mbar_arrive_expect_tx(&bars->v_full[st], tileBytes);
          for (int b = 0; b < nbox; ++b)
            tma_load_3d(sV + st * tileBytes + b * 16384, &maps.v[s], &bars->v_full[st], b * 64, row, pc.h);
          ++g;
        }
      }
      if (!ok)
        for (int i = max(0, g - kVStages); i < g; ++i)
          mbar_wait_drain(&bars->v_full[i % kVStages], (i / kVStages) & 1, 200000000ull);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idS = idesc_bf16_f32(128, kTile, 0, 0);
      const uint32_t idO = idesc_bf16_f32(128, d, 0, 1);
      const uint32_t qB = smem_u32(sQ), kB = smem_u32(sK), vB = smem_u32(sV);
      bool ok = true;
      bool issued = false;
      int g = 0, np = 0;
      int ns[2] = {0, 0};  // S tiles issued per query tile (= P tiles to wait for)
      PieceIter it;
      it.init(S, blockIdx.x);
      Piece pc;
      // O_t (+)= P_t V: P_t from S_t's first 64 TMEM columns, 8 columns per 16 keys;
      // V tile: keys are the K dimension (rows of 128 B), d the N dimension
      // (64-column halves 16 KB apart)
      auto pv = [&](int t, int vst, bool first_pv) {
        for (int kk = 0; kk < kTile / 16; ++kk)
          mma_f16_ts(tmem + 256 + t * kTile, tmem + t * kTile + kk * 8,
                     sdesc_sw128(vB + vst * tileBytes + kk * 2048, 16384, 1024), idO,
                     (!first_pv || kk > 0) ? 1u : 0u);
      };
      while (ok && it.next(S, pc)) {
        if (!(ok = mbar_wait(&bars->q_full, np & 1, abort, a.status))) break;
        tc_fence_after();
        for (int j = pc.j0; j < pc.j1 && ok; ++j) {
          const int kst = g % kKStages;
          const int vprev = (g + kVStages - 1) % kVStages;  // V stage of tile g-1
          if (!(ok = mbar_wait(&bars->k_full[kst], (g / kKStages) & 1, abort, a.status))) break;
          if (j > pc.j0 && !(ok = mbar_wait(&bars->v_full[vprev], ((g - 1) / kVStages) & 1, abort, a.status)))
            break;
          tc_fence_after();
          for (int t = 0; t < pc.ntq; ++t) {
            if (j > pc.j0) {
              if (!(ok = mbar_wait(&bars->p_full[t], (ns[t] - 1) & 1, abort, a.status))) break;
              tc_fence_after();
              pv(t, vprev, j - 1 == pc.j0);
            }
            for (int kk = 0; kk < d / 16; ++kk) {
              const uint32_t koff = static_cast<uint32_t>((kk >> 2) * 16384 + (kk & 3) * 32);
              mma_f16_ss(tmem + t * kTile, sdesc_sw128(qB + t * tileBytes + koff, 16, 1024),
                         sdesc_sw128(kB + kst * tileBytes + koff, 16, 1024), idS, kk > 0 ? 1u : 0u);
            }
            issued = true;
            mma_commit(&bars->s_full[t]);
            ++ns[t];
          }
          if (!ok) break;
          mma_commit(&bars->k_empty[kst]);
          if (j > pc.j0) mma_commit(&bars->v_empty[vprev]);
          if (j == pc.j1 - 1) mma_commit(&bars->q_empty);
          ++g;
        }
        if (!ok) break;
        // the last key tile's PV; then O of the piece is complete
        const int vst = (g - 1) % kVStages;
        if (!(ok = mbar_wait(&bars->v_full[vst], ((g - 1) / kVStages) & 1, abort, a.status))) break;
        for (int t = 0; t < pc.ntq && ok; ++t) {
          if (!(ok = mbar_wait(&bars->p_full[t], (ns[t] - 1) & 1, abort, a.status))) break;
          tc_fence_after();
          pv(t, vst, pc.j1 - 1 == pc.j0);
          mma_commit(&bars->o_full[t]);
        }
        if (!ok) break;
        mma_commit(&bars->v_empty[vst]);
        ++np;
      }
      if (!ok && issued) {
        // no MMA may still write TMEM when it is freed: the commit below arrives
        // once every MMA issued by this thread has completed
        mma_commit(&bars->mma_done);
        mbar_wait_drain(&bars->mma_done, 0, 200000000ull);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax / epilogue
    const int t = (warp - 4) >> 2;  // query tile of the unit
    const int q = warp & 3;         // TMEM lane quarter
    const int r = q * 32 + lane;    // row inside the query tile
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const uint32_t tS = tmem + t * kTile;        // S_t, and P_t in its first 64 columns
    const uint32_t tO = tmem + 256 + t * kTile;  // O_t
    const float sl2 = a.scale * 1.4426950408889634f;  // scale * log2(e)
    const float thr_raw = kRescaleThreshold / sl2;     // rescale threshold in raw score units
    const size_t slot_floats = static_cast<size_t>(kTile) * d + 2 * kTile;
    const size_t ml_off = static_cast<size_t>(kTile) * d;  // m, then l, after O in a slot
    bool ok = true;
    int ns = 0, npt = 0, ngs = 0;
    // every lane of the warp takes the same branch after a wait
    auto wait_warp = [&](uint64_t* bar, uint32_t parity) -> bool {
      const bool w = mbar_wait(bar, parity, abort, a.status);
      return __all_sync(0xffffffffu, w);
    };
    auto group_sync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->grp[t]);
      return wait_warp(&bars->grp[t], (ngs++) & 1);
    };
    PieceIter& it = s_it[warp - 4];
    Piece& pc = s_pc[warp - 4];
    if (lane == 0) it.init(S, blockIdx.x);
    __syncwarp();
    for (;;) {
      int more = 0;
      __syncwarp();  // every lane is done with the previous piece before lane 0 moves on
      if (lane == 0) more = it.next(S, pc) ? 1 : 0;
      more = __shfl_sync(0xffffffffu, more, 0);
      __syncwarp();  // lane 0's writes of the piece are visible to the warp
      if (!more || !ok) break;
      if (t >= pc.ntq) continue;
      float m = -INFINITY, l = 0.f;  // m: running max of the raw scores
      for (int j = pc.j0; j < pc.j1; ++j) {
        int s, row, nv;
        tile_info(a, pc.h, j, s, row, nv);
        if (!(ok = wait_warp(&bars->s_full[t], ns & 1))) break;
        ++ns;
        tc_fence_after();
        // all four 32-column loads in flight before one wait
        uint32_t v0[32], v1[32], v2[32], v3[32];
        tmem_ld32(tS + lane_off + 0, v0);
        tmem_ld32(tS + lane_off + 32, v1);
        tmem_ld32(tS + lane_off + 64, v2);
        tmem_ld32(tS + lane_off + 96, v3);
        tmem_wait_ld_reg(v0);  // the first wait covers all four loads; the others
        tmem_wait_ld_reg(v1);  // only tie the registers to it
        tmem_wait_ld_reg(v2);
        tmem_wait_ld_reg(v3);
        auto X = [&](int k) -> uint32_t& {
          return k < 32 ? v0[k] : (k < 64 ? v1[k - 32] : (k < 96 ? v2[k - 64] : v3[k - 96]));
        };
        if (nv < kTile) {  // the last tile of a segment: keys past its end do not exist
#pragma unroll
          for (int k = 0; k < kTile; ++k)
            if (k >= nv) X(k) = __float_as_uint(-INFINITY);
        }
        // row max of the raw scores: three-input max, four independent chains
        float mx[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) mx[i] = fmax3(__uint_as_float(X(i)), __uint_as_float(X(i + 4)), __uint_as_float(X(i + 8)));
#pragma unroll
        for (int k = 12; k < kTile - 4; k += 8)
#pragma unroll
          for (int i = 0; i < 4; ++i) mx[i] = fmax3(mx[i], __uint_as_float(X(k + i)), __uint_as_float(X(k + 4 + i)));
#pragma unroll
        for (int i = 0; i < 4; ++i) mx[i] = fmaxf(mx[i], __uint_as_float(X(kTile - 4 + i)));
        const float mt = fmaxf(fmax3(mx[0], mx[1], mx[2]), mx[3]);
        float alpha = 1.f;
        bool resc = false;
        if (j == pc.j0) {
          m = mt;
        } else if (mt > m + thr_raw) {
          alpha = ex2_approx((m - mt) * sl2);
          m = mt;
          resc = true;
        }
        // p = 2^((s - m) * scale * log2 e): one FFMA and one ex2 per score; the bf16
        // row goes into S_t's first 64 columns (two keys per column, even key low),
        // eight columns per store to keep register pressure below the 168 limit
        const float nb = -m * sl2;
        float rsa = 0.f, rsb = 0.f;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          uint32_t pk[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int k = ch * 16 + 2 * i;
            const float px = ex2_approx(fmaf(__uint_as_float(X(k)), sl2, nb));
            const float py = ex2_approx(fmaf(__uint_as_float(X(k + 1)), sl2, nb));
            rsa += px;
            rsb += py;
            pk[i] = pack_bf16(px, py);
          }
          tmem_st8(tS + lane_off + ch * 8, pk);
        }
        // rare: the running max moved.  O_t is stable here (PV_t(j-1) completed
        // before S_t(j) did) and PV_t(j) waits for this tile's P.
        if (__any_sync(0xffffffffu, resc)) {
          for (int c = 0; c < d / 32; ++c) {
            uint32_t v[32];
            tmem_ld32(tO + lane_off + c * 32, v);
            tmem_wait_ld_reg(v);
#pragma unroll
            for (int k = 0; k < 32; ++k) v[k] = __float_as_uint(__uint_as_float(v[k]) * alpha);
            tmem_st32(tO + lane_off + c * 32, v);
          }
        }
        l = l * alpha + (rsa + rsb);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_full[t]);
      }
      if (!ok) break;
      if (!(ok = wait_warp(&bars->o_full[t], npt & 1))) break;
      ++npt;
      tc_fence_after();
      const int qrow = pc.p * 2 * kTile + t * kTile + r;
      const size_t obase = static_cast<size_t>(pc.h) * a.Nq;
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(a.O) + (obase + qrow) * d;
      if (pc.npieces == 1) {
        // the whole unit ran here: normalise and store
        const float inv_l = l > 0.f ? 1.f / l : 0.f;
        for (int c = 0; c < d / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tO + lane_off + c * 32, v);
          tmem_wait_ld_reg(v);
          if (qrow < a.Nq) {
#pragma unroll
            for (int k = 0; k < 32; k += 8) {
              uint4 o;
              o.x = pack_bf16(__uint_as_float(v[k + 0]) * inv_l, __uint_as_float(v[k + 1]) * inv_l);
              o.y = pack_bf16(__uint_as_float(v[k + 2]) * inv_l, __uint_as_float(v[k + 3]) * inv_l);
              o.z = pack_bf16(__uint_as_float(v[k + 4]) * inv_l, __uint_as_float(v[k + 5]) * inv_l);
              o.w = pack_bf16(__uint_as_float(v[k + 6]) * inv_l, __uint_as_float(v[k + 7]) * inv_l);
              *reinterpret_cast<uint4*>(orow + c * 32 + k) = o;
            }
          }
        }
        if (a.lse && qrow < a.Nq) a.lse[obase + qrow] = (m * sl2 + __log2f(l)) * 0.6931471805599453f;
        continue;
      }
      // a piece of a split unit: store the partial (O as [d/4][128] float4, so that
      // consecutive rows are consecutive 16-byte words, then m and l per row)
      float* slot = a.part + static_cast<size_t>((blockIdx.x * 2 + pc.which) * 2 + t) * slot_floats;
      for (int c = 0; c < d / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tO + lane_off + c * 32, v);
        tmem_wait_ld_reg(v);
#pragma unroll
        for (int k = 0; k < 32; k += 4)
          reinterpret_cast<float4*>(slot)[static_cast<size_t>(c * 8 + k / 4) * kTile + r] =
              make_float4(__uint_as_float(v[k]), __uint_as_float(v[k + 1]), __uint_as_float(v[k + 2]),
                          __uint_as_float(v[k + 3]));
      }
      slot[ml_off + r] = m;
      slot[ml_off + kTile + r] = l;
      __threadfence();
      if (!(ok = group_sync())) break;
      if (r == 0) {
        // arrival count tagged with this launch's epoch; the last arrival resets it
        unsigned long long* cp = a.cnt + (static_cast<size_t>(pc.h) * S.npair + pc.p) * 2 + t;
        unsigned long long cur = *reinterpret_cast<volatile unsigned long long*>(cp);
        int last = -1;
        for (int n = 0; n < (1 << 16); ++n) {
          const unsigned int have =
              (static_cast<unsigned int>(cur >> 32) == a.epoch) ? static_cast<unsigned int>(cur) : 0u;
          const bool fin = have + 1 >= static_cast<unsigned int>(pc.npieces);
          const unsigned long long want =
              fin ? 0ull : ((static_cast<unsigned long long>(a.epoch) << 32) | (have + 1));
          const unsigned long long prev = atomicCAS(cp, cur, want);
          if (prev == cur) {
            last = fin ? 1 : 0;
            break;
          }
          cur = prev;
        }
        if (last < 0) latch_status(a.status, KVB_E_DEVICE_TIMEOUT);
        bars->last[t] = last > 0 ? 1 : 0;
      }
      if (!(ok = group_sync())) break;
      if (!bars->last[t]) continue;
      __threadfence();
      // the last piece merges every piece of the unit (itself included), row by row
      auto slot_of = [&](int k) -> const float* {
        const int wk = (k == 0) ? pc.wfirst : 0;  // later pieces open their CTA's range
        return a.part + static_cast<size_t>(((pc.cfirst + k) * 2 + wk) * 2 + t) * slot_floats;
      };
      float M = -INFINITY;
      for (int k = 0; k < pc.npieces; ++k) M = fmaxf(M, __ldcg(slot_of(k) + ml_off + r));
      float L = 0.f;
      for (int k = 0; k < pc.npieces; ++k)
        L += __ldcg(slot_of(k) + ml_off + kTile + r) * ex2_approx((__ldcg(slot_of(k) + ml_off + r) - M) * sl2);
      const float inv_L = L > 0.f ? 1.f / L : 0.f;
      for (int c4 = 0; c4 < d / 4; c4 += 2) {
        float4 acc0 = make_float4(0.f, 0.f, 0.f, 0.f), acc1 = acc0;
        for (int k = 0; k < pc.npieces; ++k) {
          const float* sk = slot_of(k);
          const float wk = ex2_approx((__ldcg(sk + ml_off + r) - M) * sl2) * inv_L;
          const float4 x0 = __ldcg(reinterpret_cast<const float4*>(sk) + static_cast<size_t>(c4) * kTile + r);
          const float4 x1 = __ldcg(reinterpret_cast<const float4*>(sk) + static_cast<size_t>(c4 + 1) * kTile + r);
          acc0.x += wk * x0.x;
          acc0.y += wk * x0.y;
          acc0.z += wk * x0.z;
          acc0.w += wk * x0.w;
          acc1.x += wk * x1.x;
          acc1.y += wk * x1.y;
          acc1.z += wk * x1.z;
          acc1.w += wk * x1.w;
        }
        if (qrow < a.Nq)
          *reinterpret_cast<uint4*>(orow + c4 * 4) = make_uint4(pack_bf16(acc0.x, acc0.y), pack_bf16(acc0.z, acc0.w),
                                                                pack_bf16(acc1.x, acc1.y), pack_bf16(acc1.z, acc1.w));
      }
      if (a.lse && qrow < a.Nq) a.lse[obase + qrow] = (M * sl2 + __log2f(L)) * 0.6931471805599453f;
    }
    // query tiles of heads without a single key: zeros (lse -inf), spread over CTAs
    if (ok) {
      for (int h = 0; h < H; ++h) {
        if (sch.T[h] != 0) continue;
        for (int p = 0; p < S.npair; ++p) {
          if ((h * S.npair + p) % sch.G != static_cast<int>(blockIdx.x) || t >= S.ntq(p)) continue;
          const int qrow = p * 2 * kTile + t * kTile + r;
          if (qrow >= a.Nq) continue;
          __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(a.O) + (static_cast<size_t>(h) * a.Nq + qrow) * d;
          for (int c = 0; c < d; c += 8) *reinterpret_cast<uint4*>(orow + c) = make_uint4(0u, 0u, 0u, 0u);
          if (a.lse) a.lse[static_cast<size_t>(h) * a.Nq + qrow] = -INFINITY;
        }
      }
    }
  }

  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// -------------------------------------------------------------------- f32 path
// One warp per query; lanes stride over keys with a per-lane online softmax,
// then merge.  For the small fp32 workload only.
constexpr int kF32MaxD = 128;

__global__ void attend_f32_kernel(const AttnArgs a) {
  pdl_wait();
  pdl_trigger();
  const int h = blockIdx.y;
  const int qi = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (qi >= a.Nq) return;
  const int d = a.d;
  const float* qv = static_cast<const float*>(a.Q) + (static_cast<size_t>(h) * a.Nq + qi) * d;
  float qr[kF32MaxD];
  for (int k = 0; k < d; ++k) qr[k] = qv[k] * a.scale;
  float m = -INFINITY, l = 0.f;
  float acc[kF32MaxD];
  for (int k = 0; k < d; ++k) acc[k] = 0.f;
  for (int s = 0; s < a.nseg; ++s) {
    const AttnSeg& sg = a.seg[s];
    const int len = seg_len(sg, h), off = seg_off(sg, h);
    const float* Kb = static_cast<const float*>(sg.K) + (static_cast<size_t>(h) * sg.ld + off) * d;
    const float* Vb = static_cast<const float*>(sg.V) + (static_cast<size_t>(h) * sg.ld + off) * d;
    for (int j = lane; j < len; j += 32) {
      float dot = 0.f;
      for (int k = 0; k < d; ++k) dot = fmaf(qr[k], Kb[static_cast<size_t>(j) * d + k], dot);
      const float mn = fmaxf(m, dot);
      const float sc = expf(m - mn), p = expf(dot - mn);
      l = l * sc + p;
      for (int k = 0; k < d; ++k) acc[k] = acc[k] * sc + p * Vb[static_cast<size_t>(j) * d + k];
      m = mn;
    }
  }
  // merge lanes
  float M = m;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  const float sc = (m == -INFINITY) ? 0.f : expf(m - M);
  float L = warp_sum(l * sc);
  float* orow = static_cast<float*>(a.O) + (static_cast<size_t>(h) * a.Nq + qi) * d;
  for (int k = 0; k < d; ++k) {
    const float v = warp_sum(acc[k] * sc);
    if (lane == 0) orow[k] = v / L;
  }
  if (lane == 0 && a.lse) a.lse[static_cast<size_t>(h) * a.Nq + qi] = M + logf(L);
}

}  // namespace

size_t attend_smem_bytes(int d) {
  const size_t tile = static_cast<size_t>(kTile) * d * 2;
  return 1024 + (2 + kKStages + kVStages) * tile + kBarBytes;  // Q_A, Q_B, K and V rings, barriers
}

cudaError_t launch_attend_bf16(const AttnArgs& a, cudaStream_t st) {
  if (a.Nq <= 0) return cudaSuccess;
  if (!a.part || !a.cnt || a.epoch == 0 || a.H > 64) return cudaErrorInvalidValue;
  DeviceInfo dev;
  if (!current_device(&dev)) return cudaErrorInvalidDevice;
  AttnMaps maps;
  if (!make_tmap_bf16(&maps.q, a.Q, a.d, a.Nq, a.H, kTile)) return cudaErrorInvalidValue;
  for (int s = 0; s < kAttnMaxSeg; ++s) {
    // unused slots reuse the query map (never read: their length is 0)
    const AttnSeg& g = a.seg[s];
    if (s < a.nseg && g.K && g.ld > 0) {
      if (!make_tmap_bf16(&maps.k[s], g.K, a.d, g.ld, a.H, kTile) ||
          !make_tmap_bf16(&maps.v[s], g.V, a.d, g.ld, a.H, kTile))
        return cudaErrorInvalidValue;
    } else {
      maps.k[s] = maps.q;
      maps.v[s] = maps.q;
    }
  }
  const size_t smem = attend_smem_bytes(a.d);
  cudaError_t e = cudaFuncSetAttribute(attend_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // persistent: one CTA per SM; the kernel itself uses fewer when the work is small
  const int grid = dev.n_sm < kAttnMaxCtas ? dev.n_sm : kAttnMaxCtas;
  LaunchTrace trace("attend_bf16_kernel", st);
  return launch_pdl(attend_bf16_kernel, dim3(grid), dim3(kThreads), smem, st, maps, a);
}

cudaError_t launch_attend_f32(const AttnArgs& a, cudaStream_t st) {
  if (a.Nq <= 0) return cudaSuccess;
  if (a.d > kF32MaxD) return cudaErrorInvalidValue;
  dim3 grid((a.Nq + 3) / 4, a.H);
  LaunchTrace trace("attend_f32_kernel", st);
  return launch_pdl(attend_f32_kernel, grid, dim3(128), 0, st, a);
}

}  // namespace kvb
