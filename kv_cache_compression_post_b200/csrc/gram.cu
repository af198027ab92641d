// Soft-Riesz density Gram on the 5th-generation tensor cores.
//
// DensityKV §3 "Soft-Riesz Density" / App. B.1: every admit step needs, per head,
// sums of phi(||a - b||^2 / h) over candidate x bank (and bank x admitted, bank x
// evicted, admitted x admitted) pairs: O(N M d_k).  With the norm expansion
//     -||a - b||^2 / 2 = a.b - ||a||^2/2 - ||b||^2/2
// the whole right-hand side is one bf16 contraction: each key carries 32 extra
// bf16 values ("augmented row": -||k||^2/2 split exactly into three bf16 parts,
// the constant -eps h/2 split into two, and ones), and one extra K=16 MMA step adds
// the norm terms and the regulariser, so the fp32 TMEM accumulator holds
//     D = -||a - b||^2 / 2 - eps h / 2 = -(h/2) t,   t = ||a - b||^2 / h + eps,
// for every pair.  The epilogue on CUDA cores sums 1/D directly (phi = 1/t =
// -(h/2)/D for the default s = 2): four reciprocals share one MUFU op,
//     1/D0 + 1/D1 + 1/D2 + 1/D3 = ((D0+D1) D2 D3 + (D2+D3) D0 D1) / (D0 D1 D2 D3),
// the arithmetic runs two pairs per instruction (packed f32x2 ADD/MUL/FMA), and the
// tile's sum is scaled by -h/2 once.  Other exponents take t = D (-2/h) per pair.
// The clamp t >= eps (D <= -eps h/2) is applied only when the largest key norm
// makes the fp32 rounding of x comparable to eps (a per-launch flag).
//
// Work = the sequence of (head, 256-row block, 256-column tile) steps, split evenly
// over a persistent grid (one CTA per SM).  A CTA keeps its 256 rows (two 128-row
// MMA tiles) in shared memory and streams 256-column tiles through a 2-stage TMA
// ring.  Each row tile has one 128 x 256 fp32 accumulator in TMEM (N = 256 MMAs run
// at full tensor rate); the two row tiles ping-pong: while the tensor core fills
// one, the 8 epilogue warps of the other drain it.
// Warp roles: 0 = TMA producer, 1 = MMA issuer, 2 = TMEM owner, 4..11 epilogue of
// row tile 0, 12..19 of row tile 1 (4 TMEM lane quarters x 2 column halves; one
// thread per row and half, so row sums need no cross-thread reduction).
#include <climits>

#include "gram.cuh"
#include "host_util.h"
#include "kvb_device.cuh"
#include "sm100.cuh"

namespace kvb {
using namespace sm100;

namespace {

constexpr int kStages = 2;
constexpr int kColTile = 256;   // columns per MMA (N) and per step
constexpr int kEpiWarpsPerTile = 8;
constexpr uint32_t kAugRowBytes = 32;  // 16 bf16 of the augmented row per operand row

struct alignas(8) GramBars {
  uint64_t a_full, a_empty;
  uint64_t full[kStages], empty[kStages];
  uint64_t acc_full[2], acc_empty[2];   // per row tile
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
};
constexpr int kBarBytes = 256;
static_assert(sizeof(GramBars) <= kBarBytes, "barrier block overflows its reservation");

__device__ __forceinline__ int set_n(const GramSet& s, int h) { return s.n_dev ? s.n_dev[h] : s.n_uni; }
__device__ __forceinline__ int set_off(const GramSet& s, int h) { return s.off_dev ? s.off_dev[h] : s.off_uni; }

// Per-head sizes of a launch, read once per CTA into shared memory: the counts
// can live in device memory (bank sizes, admitted counts), and a walk over the
// heads that loads them one after another costs a memory round trip per head.
struct HeadDims {
  int nR, nC, rOff, cOff;
  int RB, CT;            // row blocks / column tiles
  int nneg, diag;        // signed-column count, self-pair offset
  int altR, altC;        // rows / columns through the alternate maps (offset 0)
  long long L0;          // first step of the head; entry H holds the total
};
constexpr int kTabBytes = (kGramMaxHeads + 1) * static_cast<int>(sizeof(HeadDims));

// Filled by one warp: each lane loads one head's sizes, a warp scan places the
// heads' step ranges one after another.
__device__ __forceinline__ void build_head_table(const GramArgs& a, HeadDims* tab, int lane) {
  long long carry = 0;
  for (int base = 0; base < a.H; base += 32) {
    const int h = base + lane;
    HeadDims t{};
    long long n = 0;
    if (h < a.H) {
      t.nR = set_n(a.rows, h);
      t.nC = set_n(a.cols, h);
      t.altR = (a.alt_rows_n >= 0 && t.nR == a.alt_rows_n) ? 1 : 0;
      t.altC = (a.alt_cols_n >= 0 && t.nC == a.alt_cols_n) ? 1 : 0;
      t.rOff = t.altR ? 0 : set_off(a.rows, h);
      t.cOff = t.altC ? 0 : set_off(a.cols, h);
      t.RB = t.nC > 0 ? (t.nR + kGramRowBlock - 1) / kGramRowBlock : 0;
      t.CT = t.nR > 0 ? (t.nC + kColTile - 1) / kColTile : 0;
      t.nneg = a.nneg_dev ? a.nneg_dev[h] : a.nneg_uni;
      t.diag = a.use_diag ? (a.diag_dev ? a.diag_dev[h] : a.diag_uni) : INT_MIN / 2;
      n = static_cast<long long>(t.RB) * t.CT;
    }
    long long x = n;  // inclusive scan of the step counts over the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (h < a.H) {
      t.L0 = carry + x - n;
      tab[h] = t;
    }
    carry += __shfl_sync(0xffffffffu, x, 31);
  }
  if (lane == 0) tab[a.H].L0 = carry;
}

// Position in the (head, row block, column tile) step sequence.
struct Cursor {
  int h, rb, j;          // current step
  int RB, CT;            // row blocks / column tiles of head h
  int nR, nC, rOff, cOff;
};

__device__ __forceinline__ int active_grid(const GramArgs& a, long long T) {
  long long g = T / a.min_steps;
  if (g > a.grid) g = a.grid;
  if (g < 1) g = 1;
  return static_cast<int>(g);
}

__device__ __forceinline__ void cursor_load_head(const HeadDims* tab, Cursor& c) {
  const HeadDims& t = tab[c.h];
  c.RB = t.RB;
  c.CT = t.CT;
  c.nR = t.nR;
  c.nC = t.nC;
  c.rOff = t.rOff;
  c.cOff = t.cOff;
}

// position the cursor at step L (0 <= L < total)
__device__ __forceinline__ void cursor_seek(const GramArgs& a, const HeadDims* tab, long long L, Cursor& c) {
  c.h = 0;
  while (c.h + 1 < a.H && L >= tab[c.h + 1].L0) ++c.h;
  cursor_load_head(tab, c);
  L -= tab[c.h].L0;
  c.rb = static_cast<int>(L / c.CT);
  c.j = static_cast<int>(L % c.CT);
}

__device__ __forceinline__ void cursor_next(const GramArgs& a, const HeadDims* tab, Cursor& c) {
  if (++c.j < c.CT) return;
  c.j = 0;
  if (++c.rb < c.RB) return;
  c.rb = 0;
  do {
    ++c.h;
    if (c.h >= a.H) return;
  } while (tab[c.h].RB * tab[c.h].CT == 0);
  cursor_load_head(tab, c);
}

// the CTA (of G_eff) whose range contains step L
__device__ __forceinline__ int cta_of(long long L, long long T, int G) {
  return static_cast<int>(((L + 1) * G - 1) / T);
}

__device__ __forceinline__ int nact_of(const Cursor& c) {
  return (c.nR - c.rb * kGramRowBlock > kGramRowTile) ? 2 : 1;
}

// phi for one pair given t = x + eps
template <int SMODE>
__device__ __forceinline__ float phi_t(float t, float nhs) {
  if constexpr (SMODE == 2) return rcp_approx(t);
  else if constexpr (SMODE == 1) return rsqrt_approx(t);
  else return ex2_approx(nhs * lg2_approx(t));
}

__device__ __forceinline__ float2 f2(uint32_t x, uint32_t y) { return make_float2(__uint_as_float(x), __uint_as_float(y)); }

// Sum of 1/D over 16 accumulator columns (s = 2, packed f32x2, 4 MUFU ops): pairs
// (D_{2i}, D_{2i+1}) travel together, and each lane of a float2 folds four
// reciprocals into one.  dmax = -eps h/2 is the clamp (D <= dmax).
template <bool CLAMP>
__device__ __forceinline__ float2 sum_recip16(const uint32_t (&v)[16], float dmax, float2 acc) {
#pragma unroll
  for (int k = 0; k < 16; k += 8) {
    float2 A = f2(v[k + 0], v[k + 1]);
    float2 B = f2(v[k + 2], v[k + 3]);
    float2 C = f2(v[k + 4], v[k + 5]);
    float2 D = f2(v[k + 6], v[k + 7]);
    if constexpr (CLAMP) {
      A = make_float2(fminf(A.x, dmax), fminf(A.y, dmax));
      B = make_float2(fminf(B.x, dmax), fminf(B.y, dmax));
      C = make_float2(fminf(C.x, dmax), fminf(C.y, dmax));
      D = make_float2(fminf(D.x, dmax), fminf(D.y, dmax));
    }
    const float2 s = __fadd2_rn(A, B), p = __fmul2_rn(A, B);     // lane x: D0+D2, D0 D2; lane y: D1+D3, D1 D3
    const float2 s2 = __fadd2_rn(C, D), p2 = __fmul2_rn(C, D);
    const float2 num = __ffma2_rn(s, p2, __fmul2_rn(s2, p));      // (Da+Db) Dc Dd + (Dc+Dd) Da Db
    const float2 den = __fmul2_rn(p, p2);
    acc = __ffma2_rn(num, make_float2(rcp_approx(den.x), rcp_approx(den.y)), acc);
  }
  return acc;
}

// Sum of 1/D over a thread's 128 accumulator columns (8 chunks of 16, s = 2, no
// masked pair), releasing the accumulator (one arrival per warp on acc_empty) as
// soon as the last chunk is in registers.  tcgen05.wait::ld waits for every load
// of the thread, so four 16-column buffers work in pairs: two loads in flight
// over two chunks' arithmetic (a TMEM load takes ~200 clk while the other row
// tile's MMAs run).
template <bool CLAMP>
__device__ __forceinline__ float2 drain_recip128(uint32_t taddr, float dmax, uint64_t* acc_empty, int lane) {
  float2 acc = make_float2(0.f, 0.f);
  uint32_t va[16], vb[16], vc[16], vd[16];
  tmem_ld16(taddr + 0, va);
  tmem_ld16(taddr + 16, vb);
  tmem_wait_ld_reg16(va);
  reg_fence16(vb);
  tmem_ld16(taddr + 32, vc);
  tmem_ld16(taddr + 48, vd);
  acc = sum_recip16<CLAMP>(va, dmax, acc);
  acc = sum_recip16<CLAMP>(vb, dmax, acc);
  tmem_wait_ld_reg16(vc);
  reg_fence16(vd);
  tmem_ld16(taddr + 64, va);
  tmem_ld16(taddr + 80, vb);
  acc = sum_recip16<CLAMP>(vc, dmax, acc);
  acc = sum_recip16<CLAMP>(vd, dmax, acc);
  tmem_wait_ld_reg16(va);
  reg_fence16(vb);
  tmem_ld16(taddr + 96, vc);
  tmem_ld16(taddr + 112, vd);
  acc = sum_recip16<CLAMP>(va, dmax, acc);
  acc = sum_recip16<CLAMP>(vb, dmax, acc);
  tmem_wait_ld_reg16(vc);
  reg_fence16(vd);
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(acc_empty);
  acc = sum_recip16<CLAMP>(vc, dmax, acc);
  return sum_recip16<CLAMP>(vd, dmax, acc);
}

template <int SMODE>
__global__ void __launch_bounds__(kGramThreads, 1)
    gram_bf16_kernel(const __grid_constant__ GramMaps maps, const GramArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int nbox = a.d / 64;
  const uint32_t aBytes = static_cast<uint32_t>(kGramRowTile) * a.d * 2;   // one 128-row tile
  const uint32_t bBytes = static_cast<uint32_t>(kColTile) * a.d * 2;       // one 256-row column tile
  const uint32_t aAug = kGramRowTile * kAugRowBytes, bAug = kColTile * kAugRowBytes;
  uint8_t* sA = smem;                          // 2 row tiles
  uint8_t* sB = sA + 2 * aBytes;               // kStages column tiles
  uint8_t* sAa = sB + kStages * bBytes;        // 2 augmented row tiles
  uint8_t* sBa = sAa + 2 * aAug;               // kStages augmented column tiles
  GramBars* bars = reinterpret_cast<GramBars*>(sBa + kStages * bAug);
  HeadDims* tab = reinterpret_cast<HeadDims*>(reinterpret_cast<uint8_t*>(bars) + kBarBytes);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&bars->a_full, 1);
    mbar_init(&bars->a_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int r = 0; r < 2; ++r) {
      mbar_init(&bars->acc_full[r], 1);
      mbar_init(&bars->acc_empty[r], kEpiWarpsPerTile);
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
  // everything above touched only shared memory and TMEM: from here on the
  // previous kernel's results are read
  pdl_wait();
  pdl_trigger();
  if (warp == 3) build_head_table(a, tab, lane);
  __syncthreads();

  const long long T = tab[a.H].L0;
  const int G = active_grid(a, T);
  const int cta = blockIdx.x;
  const long long L0 = (cta < G) ? (T * cta) / G : 0;
  const long long L1 = (cta < G) ? (T * (cta + 1)) / G : 0;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&maps.R);
      prefetch_tmap(&maps.C);
      prefetch_tmap(&maps.Ra);
      prefetch_tmap(&maps.Ca);
      prefetch_tmap(&maps.R2);
      prefetch_tmap(&maps.C2);
      prefetch_tmap(&maps.Ra2);
      prefetch_tmap(&maps.Ca2);
      int it = 0, aload = 0;
      bool ok = true;
      Cursor c;
      if (L0 < L1) cursor_seek(a, tab, L0, c);
      for (long long L = L0; L < L1; ++L, cursor_next(a, tab, c)) {
        if (L == L0 || c.j == 0) {
          if (aload > 0 && !(ok = mbar_wait(&bars->a_empty, (aload - 1) & 1, abort, a.status))) break;
          const int nact = nact_of(c);
          const bool alt = tab[c.h].altR != 0;
          const CUtensorMap* mR = alt ? &maps.R2 : &maps.R;
          const CUtensorMap* mRa = alt ? &maps.Ra2 : &maps.Ra;
          mbar_arrive_expect_tx(&bars->a_full, nact * (aBytes + aAug));
          for (int r = 0; r < nact; ++r) {
            const int y = c.rOff + c.rb * kGramRowBlock + r * kGramRowTile;
            for (int k = 0; k < nbox; ++k)
              tma_load_3d(sA + r * aBytes + k * (kGramRowTile * 128), mR, &bars->a_full, k * 64, y, c.h);
            tma_load_3d(sAa + r * aAug, mRa, &bars->a_full, 0, y, c.h);  // row form
          }
          ++aload;
        }
        const int s = it % kStages;
        if (!(ok = mbar_wait(&bars->empty[s], ((it / kStages) & 1) ^ 1, abort, a.status))) break;
        mbar_arrive_expect_tx(&bars->full[s], bBytes + bAug);
        const int y = c.cOff + c.j * kColTile;
        const bool alt = tab[c.h].altC != 0;
        const CUtensorMap* mC = alt ? &maps.C2 : &maps.C;
        const CUtensorMap* mCa = alt ? &maps.Ca2 : &maps.Ca;
        for (int k = 0; k < nbox; ++k)
          tma_load_3d(sB + s * bBytes + k * (kColTile * 128), mC, &bars->full[s], k * 64, y, c.h);
        tma_load_3d(sBa + s * bAug, mCa, &bars->full[s], 16, y, c.h);  // column form
        ++it;
      }
      if (!ok) {
        // abort path: let the copies already issued land before the CTA exits
        for (int k = max(0, it - kStages); k < it; ++k)
          mbar_wait_drain(&bars->full[k % kStages], (k / kStages) & 1, 200000000ull);
        if (aload > 0) mbar_wait_drain(&bars->a_full, (aload - 1) & 1, 200000000ull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, kColTile, 0, 0);
      const uint32_t aBase = smem_u32(sA), bBase = smem_u32(sB);
      const uint32_t aaBase = smem_u32(sAa), baBase = smem_u32(sBa);
      int it = 0, aload = 0;
      int tr[2] = {0, 0};  // tiles issued into each row tile's accumulator
      bool ok = true;
      Cursor c;
      if (L0 < L1) cursor_seek(a, tab, L0, c);
      for (long long L = L0; L < L1 && ok; ++L) {
        const int nact = nact_of(c);
        if (L == L0 || c.j == 0) {
          if (!(ok = mbar_wait(&bars->a_full, aload & 1, abort, a.status))) break;
          tc_fence_after();
          ++aload;
        }
        const int s = it % kStages;
        if (!(ok = mbar_wait(&bars->full[s], (it / kStages) & 1, abort, a.status))) break;
        for (int r = 0; r < nact && ok; ++r) {
          // the row tile's accumulator is free once its 8 epilogue warps hold it in registers
          if (!(ok = mbar_wait(&bars->acc_empty[r], (tr[r] & 1) ^ 1, abort, a.status))) break;
          tc_fence_after();
          const uint32_t dcol = tmem + static_cast<uint32_t>(r * kColTile);
          for (int kk = 0; kk < a.d / 16; ++kk) {
            const uint32_t ka = static_cast<uint32_t>((kk >> 2) * (kGramRowTile * 128) + (kk & 3) * 32);
            const uint32_t kb = static_cast<uint32_t>((kk >> 2) * (kColTile * 128) + (kk & 3) * 32);
            mma_f16_ss(dcol, sdesc_sw128(aBase + r * aBytes + ka, 16, 1024), sdesc_sw128(bBase + s * bBytes + kb, 16, 1024),
                       idesc, kk > 0 ? 1u : 0u);
          }
          // the norm terms: one more K=16 step over the augmented rows
          mma_f16_ss(dcol, sdesc_sw32(aaBase + r * aAug, 256), sdesc_sw32(baBase + s * bAug, 256), idesc, 1u);
          mma_commit(&bars->acc_full[r]);
          ++tr[r];
        }
        if (!ok) break;
        mma_commit(&bars->empty[s]);
        ++it;
        const bool last_of_block = (L + 1 == L1) || (c.j + 1 == c.CT);
        if (last_of_block) mma_commit(&bars->a_empty);
        cursor_next(a, tab, c);
      }
      if (!ok && (tr[0] + tr[1]) > 0) {
        // abort path: no MMA may still write TMEM when it is freed (the commit
        // arrives once every MMA issued by this thread has completed)
        mma_commit(&bars->mma_done);
        mbar_wait_drain(&bars->mma_done, 0, 200000000ull);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int e = warp - 4;
    const int r = e >> 3;            // row tile
    const int q = warp & 3;          // TMEM lane quarter (warp_id % 4)
    const int hf = (e >> 2) & 1;     // column half of the 256-column tile
    const int row_in_tile = q * 32 + lane;
    const float ks = a.kscale, eps = a.eps, nhs = -0.5f * a.s;
    const float kinv = 1.f / ks;     // -h/2: sum of 1/D -> sum of phi (s = 2)
    const float dmax = eps * kinv;   // -eps h/2: D <= dmax <=> t >= eps
    // clamp t >= eps only when fp32 rounding of x could reach eps / 2 (see header)
    const bool clamp = a.norm_max ? (*a.norm_max) * 1e-4f >= eps * (-2.f / ks) : true;
    int t = 0;                       // tiles seen by this row tile (phase of its barriers)
    bool ok = true;
    Cursor c;
    if (L0 < L1) cursor_seek(a, tab, L0, c);
    float acc_pos = 0.f, acc_neg = 0.f;
    int row = 0, nneg = 0, diag = 0, rt0 = 0;
    bool active = false, valid_row = false;
    long long Lblock = L0;  // first step of the current row block
    for (long long L = L0; L < L1; ++L) {
      if (L == L0 || c.j == 0) {
        Lblock = L - c.j;
        rt0 = c.rb * kGramRowBlock + r * kGramRowTile;
        row = rt0 + row_in_tile;
        active = r < nact_of(c);
        valid_row = active && row < c.nR;
        nneg = tab[c.h].nneg;
        diag = tab[c.h].diag;
        acc_pos = 0.f;
        acc_neg = 0.f;
      }
      if (active) {
        if (!(ok = mbar_wait(&bars->acc_full[r], t & 1, abort, a.status))) break;
        tc_fence_after();
        const int c0 = c.j * kColTile + hf * 128;  // first column of this thread's half
        const bool tail = c0 + 128 > c.nC;
        const bool allneg = c0 + 128 <= nneg;
        const bool mixed = (c0 < nneg) && !allneg;
        const bool diag_hit = a.use_diag && (rt0 + diag < c0 + 128) && (rt0 + diag + kGramRowTile > c0);
        const bool masked = tail || mixed || diag_hit;
        const uint32_t taddr =
            tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(r * kColTile + hf * 128);
        float2 acc2 = make_float2(0.f, 0.f);
        float accs = 0.f;
        // masked tiles (ragged end, self pair, sign change) take an exact scalar path
        auto chunk = [&](const uint32_t (&v)[16], int cc) {
          const int cb = c0 + cc * 16;
          if (SMODE == 2 && !masked) {
            acc2 = clamp ? sum_recip16<true>(v, dmax, acc2) : sum_recip16<false>(v, dmax, acc2);
          } else {
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              const int col = cb + k;
              const float tv = fmaxf(__uint_as_float(v[k]) * ks, eps);
              const bool valid = (col < c.nC) && (col != row + diag);
              const float ph = valid ? phi_t<SMODE>(tv, nhs) : 0.f;
              if (masked && col < nneg) acc_neg += ph;
              else accs += ph;
            }
          }
        };
        if (SMODE == 2 && !masked) {
          acc2 = clamp ? drain_recip128<true>(taddr, dmax, &bars->acc_empty[r], lane)
                       : drain_recip128<false>(taddr, dmax, &bars->acc_empty[r], lane);
        } else {
        // 8 chunks of 16 columns; chunk c+1 is in flight while chunk c is processed
        uint32_t va[16], vb[16];
        tmem_ld16(taddr + 0, va);
        tmem_wait_ld_reg16(va);
#pragma unroll 1
        for (int cc = 0; cc < 8; cc += 2) {
          tmem_ld16(taddr + (cc + 1) * 16, vb);
          chunk(va, cc);
          tmem_wait_ld_reg16(vb);
          if (cc + 2 < 8) {
            tmem_ld16(taddr + (cc + 2) * 16, va);
          } else {
            // every column this warp needs is in registers: hand the accumulator back
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->acc_empty[r]);
          }
          chunk(vb, cc + 1);
          if (cc + 2 < 8) tmem_wait_ld_reg16(va);
        }
        }
        if (!masked) {
          const float tile = (acc2.x + acc2.y) * kinv + accs;
          if (allneg) acc_neg += tile;
          else acc_pos += tile;
        } else {
          acc_pos += accs;
        }
        ++t;
      }
      const bool last_of_block = (L + 1 == L1) || (c.j + 1 == c.CT);
      if (last_of_block && valid_row) {
        const int slot = 2 * (cta - cta_of(Lblock, T, G)) + hf;
        if (slot >= 0 && slot < a.slots)
          a.partial[(static_cast<size_t>(slot) * a.H + c.h) * a.ldOut + row] = acc_pos - acc_neg;
        else
          latch_status(a.status, 5 /* KVB_E_DEVICE_BOUNDS */);
      }
      cursor_next(a, tab, c);
    }
  }

  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// -------------------------------------------------------------------- f32 path
// One warp per row, 32 columns per step staged in shared memory, direct
// differences in fp32 (no norm expansion), same masks and phi as above.
constexpr int kF32Warps = 8;
constexpr int kF32Cols = 32;

__global__ void __launch_bounds__(kF32Warps * 32) gram_f32_kernel(const GramArgs a) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ float sh[];  // [kF32Warps][d] rows + [kF32Cols][d + 1] cols
  const int d = a.d;
  float* sRow = sh;
  float* sCol = sh + kF32Warps * d;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y;
  const int nR = set_n(a.rows, h), nC = set_n(a.cols, h);
  const int rOff = set_off(a.rows, h), cOff = set_off(a.cols, h);
  const int row = blockIdx.x * kF32Warps + warp;
  if (blockIdx.x * kF32Warps >= nR) return;
  const float inv_h = -0.5f * a.kscale;
  const float nhs = -0.5f * a.s;
  const int nneg = a.nneg_dev ? a.nneg_dev[h] : a.nneg_uni;
  const int diag = a.use_diag ? (a.diag_dev ? a.diag_dev[h] : a.diag_uni) : INT_MIN / 2;
  for (int k = lane; k < d; k += 32)
    sRow[warp * d + k] = (row < nR) ? a.R32[(static_cast<size_t>(h) * a.ldR + rOff + row) * d + k] : 0.f;
  float acc = 0.f;
  for (int c0 = 0; c0 < nC; c0 += kF32Cols) {
    __syncthreads();
    for (int i = threadIdx.x; i < kF32Cols * d; i += blockDim.x) {
      const int cc = i / d, k = i % d;
      const int col = c0 + cc;
      sCol[cc * (d + 1) + k] = (col < nC) ? a.C32[(static_cast<size_t>(h) * a.ldC + cOff + col) * d + k] : 0.f;
    }
    __syncthreads();
    const int col = c0 + lane;
    float dist = 0.f;
    for (int k = 0; k < d; ++k) {
      const float df = sRow[warp * d + k] - sCol[lane * (d + 1) + k];
      dist = fmaf(df, df, dist);
    }
    const float tv = fmaf(dist, inv_h, a.eps);
    float ph = 0.f;
    if (col < nC && col != row + diag) {
      ph = (a.s == 2.f) ? 1.f / tv : powf(tv, nhs);
      if (col < nneg) ph = -ph;
    }
    acc += ph;
  }
  acc = warp_sum(acc);
  if (lane == 0 && row < nR) a.partial[static_cast<size_t>(h) * a.ldOut + row] = acc;
}

// One CTA per (256-row block, head): the block's partials were written by the
// CTAs whose step ranges covered it, two column halves each, in slot order.
__global__ void __launch_bounds__(kGramRowBlock) gram_reduce_kernel(const GramArgs a, float* out, int ldOut) {
  __shared__ HeadDims tab[kGramMaxHeads + 1];
  __shared__ int nslots;
  pdl_wait();
  pdl_trigger();
  const int h = blockIdx.y, rb = blockIdx.x;
  if (threadIdx.x < 32) build_head_table(a, tab, threadIdx.x);
  __syncthreads();
  if (threadIdx.x == 0) {
    const HeadDims& t = tab[h];
    int n = 0;
    if (t.CT > 0 && rb < t.RB) {
      const long long T = tab[a.H].L0;
      const int G = active_grid(a, T);
      const long long Lb = t.L0 + static_cast<long long>(rb) * t.CT;
      n = 2 * (cta_of(Lb + t.CT - 1, T, G) - cta_of(Lb, T, G) + 1);
    }
    nslots = n < a.slots ? n : a.slots;
  }
  __syncthreads();
  const int r = rb * kGramRowBlock + threadIdx.x;
  if (r >= tab[h].nR) return;
  const int n = nslots;
  float acc = 0.f;
  for (int sl = 0; sl < n; ++sl) acc += a.partial[(static_cast<size_t>(sl) * a.H + h) * a.ldOut + r];
  out[static_cast<size_t>(h) * ldOut + r] = acc;
}

}  // namespace

size_t gram_smem_bytes(int d) {
  const size_t a = static_cast<size_t>(kGramRowTile) * (d * 2 + kAugRowBytes);
  const size_t b = static_cast<size_t>(kColTile) * (d * 2 + kAugRowBytes);
  return 1024 + 2 * a + kStages * b + kBarBytes + kTabBytes;
}

void gram_plan(GramArgs& a, int max_col_tiles, int n_sm) {
  // at most 8 CTAs cover a row block (every active CTA takes >= min_steps steps);
  // each CTA writes one partial per column half
  a.grid = n_sm;
  a.slots = 16;
  const int m = (max_col_tiles + 6) / 7;
  a.min_steps = m < 1 ? 1 : m;
}

cudaError_t launch_gram_bf16(const GramArgs& a, const GramMaps& m, cudaStream_t st) {
  if (a.H < 1 || a.H > kGramMaxHeads) return cudaErrorInvalidValue;
  const size_t smem = gram_smem_bytes(a.d);
  const int grid = a.grid;
  if (grid <= 0) return cudaSuccess;
  cudaError_t e;
  if (a.s == 2.f) {
    e = cudaFuncSetAttribute(gram_bf16_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    LaunchTrace trace("gram_bf16_kernel", st);
    e = launch_pdl(gram_bf16_kernel<2>, dim3(grid), dim3(kGramThreads), smem, st, m, a);
  } else if (a.s == 1.f) {
    e = cudaFuncSetAttribute(gram_bf16_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    LaunchTrace trace("gram_bf16_kernel", st);
    e = launch_pdl(gram_bf16_kernel<1>, dim3(grid), dim3(kGramThreads), smem, st, m, a);
  } else {
    e = cudaFuncSetAttribute(gram_bf16_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    LaunchTrace trace("gram_bf16_kernel", st);
    e = launch_pdl(gram_bf16_kernel<0>, dim3(grid), dim3(kGramThreads), smem, st, m, a);
  }
  return e;
}

cudaError_t launch_gram_f32(const GramArgs& a, cudaStream_t st) {
  const int maxR = a.max_rows;
  dim3 grid((maxR + kF32Warps - 1) / kF32Warps, a.H);
  const size_t smem = sizeof(float) * (kF32Warps * a.d + kF32Cols * (a.d + 1));
  LaunchTrace trace("gram_f32_kernel", st);
  return launch_pdl(gram_f32_kernel, grid, dim3(kF32Warps * 32), smem, st, a);
}

cudaError_t launch_gram_reduce(const GramArgs& a, float* out, int ldOut, cudaStream_t st) {
  if (a.H < 1 || a.H > kGramMaxHeads) return cudaErrorInvalidValue;
  const int maxR = a.max_rows;
  dim3 grid((maxR + kGramRowBlock - 1) / kGramRowBlock, a.H);
  LaunchTrace trace("gram_reduce_kernel", st);
  return launch_pdl(gram_reduce_kernel, grid, dim3(kGramRowBlock), 0, st, a, out, ldOut);
}

}  // namespace kvb
