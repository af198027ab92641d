// Attention over ragged per-head segment lists on the 5th-generation tensor cores.
//
// One CTA per (head, 128-query tile); CTAs are ordered longest head first (LPT),
// since the history length differs per head (DensityKV bank sizes, Forcing-KV
// static vs dynamic heads).  Per 128-key tile j:
//     S_j = Q K_j^T            tcgen05.mma, bf16 in shared memory, fp32 in TMEM
//     P_j = exp2(S_j*c - m)    4 softmax warps, one thread per query row
//     O  += P_j V_j            tcgen05.mma, P from swizzled shared memory,
//                              V read MN-major straight from its TMA tile
// S is double-buffered in TMEM (2 x 128 columns) so S_{j+1} runs on the tensor
// core while the softmax of tile j runs; O (128 x d fp32) stays in TMEM for the
// whole loop.  The running max is only moved when it grows by more than 8 (log2
// units), so the O rescale (a TMEM read-modify-write) is rare; P values are then
// bounded by 2^8, harmless in bf16 and fp32.  K and V stream through separate
// 2-stage TMA rings so K_{j+2} can land as soon as S_j is done.
//
// Warp roles: 0 TMA producer, 1 MMA issuer, 2 TMEM owner, 4-7 softmax/epilogue.
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

constexpr int kThreads = 256;
constexpr int kTile = 128;  // queries per CTA and keys per KV tile
constexpr int kBarBytes = 256;
constexpr float kRescaleThreshold = 8.f;

struct alignas(8) AttnBars {
  uint64_t q_full;
  uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full, o_ready, mma_done;
  uint32_t tmem_base;
  int abort;
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

__global__ void __launch_bounds__(kThreads, 1)
    attend_bf16_kernel(const __grid_constant__ AttnMaps maps, const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ int s_tiles[64];
  __shared__ int s_order[64];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int d = a.d;
  const int nbox = d / 64;
  const uint32_t tileBytes = static_cast<uint32_t>(kTile) * d * 2;  // Q, K or V tile
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + tileBytes;
  uint8_t* sV = sK + 2 * tileBytes;
  uint8_t* sP = sV + 2 * tileBytes;  // 128 x 128 bf16
  AttnBars* bars = reinterpret_cast<AttnBars*>(sP + kTile * kTile * 2);

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    mbar_init(&bars->q_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->k_full[i], 1);
      mbar_init(&bars->k_empty[i], 1);
      mbar_init(&bars->v_full[i], 1);
      mbar_init(&bars->v_empty[i], 1);
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->s_empty[i], 4);
    }
    mbar_init(&bars->p_full, 4);
    mbar_init(&bars->o_ready, 1);
    mbar_init(&bars->mma_done, 1);
    bars->abort = 0;
    fence_barrier_init();
  }
  if (tid < a.H) s_tiles[tid] = head_tiles(a, tid);
  if (warp == 2) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  __syncthreads();
  if (tid < a.H) {
    // longest head first; ties keep head order
    const int mine = s_tiles[tid];
    int rank = 0;
    for (int g = 0; g < a.H; ++g) rank += (s_tiles[g] > mine) || (s_tiles[g] == mine && g < tid);
    s_order[rank] = tid;
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort = &bars->abort;

  const int nqt = (a.Nq + kTile - 1) / kTile;
  const int h = s_order[blockIdx.x / nqt];
  const int q0 = (blockIdx.x % nqt) * kTile;
  const int T = s_tiles[h];
  const uint32_t tS = tmem;            // S buffers at columns [0, 256)
  const uint32_t tO = tmem + 256;      // O at columns [256, 256 + d)

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&maps.q);
      bool ok = true;
      int kissued = 0, vissued = 0;
      mbar_arrive_expect_tx(&bars->q_full, tileBytes);
      for (int b = 0; b < nbox; ++b) tma_load_3d(sQ + b * 16384, &maps.q, &bars->q_full, b * 64, q0, h);
      for (int j = 0; j < T && ok; ++j) {
        int s, row, nv;
        tile_info(a, h, j, s, row, nv);
        const int st = j & 1;
        if (!(ok = mbar_wait(&bars->k_empty[st], ((j >> 1) & 1) ^ 1, abort, a.status))) break;
        mbar_arrive_expect_tx(&bars->k_full[st], tileBytes);
        for (int b = 0; b < nbox; ++b)
          tma_load_3d(sK + st * tileBytes + b * 16384, &maps.k[s], &bars->k_full[st], b * 64, row, h);
        ++kissued;
        if (!(ok = mbar_wait(&bars->v_empty[st], ((j >> 1) & 1) ^ 1, abort, a.status))) break;
        mbar_arrive_expect_tx(&bars->v_full[st], tileBytes);
        for (int b = 0; b < nbox; ++b)
          tma_load_3d(sV + st * tileBytes + b * 16384, &maps.v[s], &bars->v_full[st], b * 64, row, h);
        ++vissued;
      }
      if (!ok) {
        mbar_wait_drain(&bars->q_full, 0, 200000000ull);
        for (int j = max(0, kissued - 2); j < kissued; ++j)
          mbar_wait_drain(&bars->k_full[j & 1], (j >> 1) & 1, 200000000ull);
        for (int j = max(0, vissued - 2); j < vissued; ++j)
          mbar_wait_drain(&bars->v_full[j & 1], (j >> 1) & 1, 200000000ull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idS = idesc_bf16_f32(128, kTile, 0, 0);
      const uint32_t idO = idesc_bf16_f32(128, d, 0, 1);
      const uint32_t qB = smem_u32(sQ), kB = smem_u32(sK), vB = smem_u32(sV), pB = smem_u32(sP);
      bool ok = mbar_wait(&bars->q_full, 0, abort, a.status);
      int committed = 0;
      for (int j = 0; j <= T && ok; ++j) {
        if (j < T) {
          const int sb = j & 1;
          if (!(ok = mbar_wait(&bars->k_full[sb], (j >> 1) & 1, abort, a.status))) break;
          if (!(ok = mbar_wait(&bars->s_empty[sb], ((j >> 1) & 1) ^ 1, abort, a.status))) break;
          tc_fence_after();
          for (int kk = 0; kk < d / 16; ++kk) {
            const uint32_t koff = static_cast<uint32_t>((kk >> 2) * 16384 + (kk & 3) * 32);
            mma_f16_ss(tS + sb * kTile, sdesc_sw128(qB + koff, 16, 1024),
                       sdesc_sw128(kB + sb * tileBytes + koff, 16, 1024), idS, kk > 0 ? 1u : 0u);
          }
          mma_commit(&bars->s_full[sb]);
          mma_commit(&bars->k_empty[sb]);
          ++committed;
        }
        if (j >= 1) {
          const int jj = j - 1, vb = jj & 1;
          if (!(ok = mbar_wait(&bars->v_full[vb], (jj >> 1) & 1, abort, a.status))) break;
          if (!(ok = mbar_wait(&bars->p_full, jj & 1, abort, a.status))) break;
          tc_fence_after();
          for (int kk = 0; kk < kTile / 16; ++kk) {
            const uint32_t poff = static_cast<uint32_t>((kk >> 2) * 16384 + (kk & 3) * 32);
            // V tile: keys are the K dimension (rows of 128 B), d the N dimension
            // (64-column halves 16 KB apart)
            mma_f16_ss(tO, sdesc_sw128(pB + poff, 16, 1024),
                       sdesc_sw128(vB + vb * tileBytes + kk * 2048, 16384, 1024), idO,
                       (jj > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&bars->v_empty[vb]);
          mma_commit(&bars->o_ready);
          ++committed;
        }
      }
      if (!ok && committed > 0) {
        // no MMA may still write TMEM when it is freed: the commit below arrives
        // once every MMA issued by this thread has completed
        mma_commit(&bars->mma_done);
        mbar_wait_drain(&bars->mma_done, 0, 200000000ull);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax / epilogue
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const float sl2 = a.scale * 1.4426950408889634f;  // scale * log2(e)
    const float thr_raw = kRescaleThreshold / sl2;     // rescale threshold in raw score units
    float m = -INFINITY, l = 0.f;                      // m: running max of the raw scores
    bool ok = true;
    for (int j = 0; j < T; ++j) {
      int s, row, nv;
      tile_info(a, h, j, s, row, nv);
      const int sb = j & 1;
      if (!(ok = mbar_wait(&bars->s_full[sb], (j >> 1) & 1, abort, a.status))) break;
      tc_fence_after();
      // all four 32-column loads in flight before one wait
      uint32_t v0[32], v1[32], v2[32], v3[32];
      tmem_ld32(tS + sb * kTile + lane_off + 0, v0);
      tmem_ld32(tS + sb * kTile + lane_off + 32, v1);
      tmem_ld32(tS + sb * kTile + lane_off + 64, v2);
      tmem_ld32(tS + sb * kTile + lane_off + 96, v3);
      tmem_wait_ld_reg(v0);  // the first wait covers all four loads; the others
      tmem_wait_ld_reg(v1);  // only tie the registers to it
      tmem_wait_ld_reg(v2);
      tmem_wait_ld_reg(v3);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->s_empty[sb]);
      float x[kTile];
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        x[k] = __uint_as_float(v0[k]);
        x[32 + k] = __uint_as_float(v1[k]);
        x[64 + k] = __uint_as_float(v2[k]);
        x[96 + k] = __uint_as_float(v3[k]);
      }
      if (nv < kTile) {  // the last tile of a segment: keys past its end do not exist
#pragma unroll
        for (int k = 0; k < kTile; ++k)
          if (k >= nv) x[k] = -INFINITY;
      }
      // row max of the raw scores, eight independent chains
      float mx[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx[i] = x[i];
#pragma unroll
      for (int k = 8; k < kTile; ++k) mx[k & 7] = fmaxf(mx[k & 7], x[k]);
      const float mt = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
      float alpha = 1.f;
      bool resc = false;
      if (j == 0) {
        m = mt;
      } else if (mt > m + thr_raw) {
        alpha = ex2_approx((m - mt) * sl2);
        m = mt;
        resc = true;
      }
      // p = 2^((s - m) * scale * log2 e): one FFMA and one ex2 per score
      const float nb = -m * sl2;
      float rs4[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t pk[kTile / 2];
#pragma unroll
      for (int k = 0; k < kTile; k += 2) {
        const float p0 = ex2_approx(fmaf(x[k], sl2, nb)), p1 = ex2_approx(fmaf(x[k + 1], sl2, nb));
        rs4[(k >> 1) & 3] += p0 + p1;
        pk[k >> 1] = pack_bf16(p0, p1);
      }
      const float rs = (rs4[0] + rs4[1]) + (rs4[2] + rs4[3]);
      if (j >= 1) {
        // P buffer free and O final for tile j-1
        if (!(ok = mbar_wait(&bars->o_ready, (j - 1) & 1, abort, a.status))) break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, resc)) {
          for (int c = 0; c < d / 32; ++c) {
            uint32_t v[32];
            tmem_ld32(tO + lane_off + c * 32, v);
            tmem_wait_ld_reg(v);
#pragma unroll
            for (int k = 0; k < 32; ++k) v[k] = __float_as_uint(__uint_as_float(v[k]) * alpha);
            tmem_st32(tO + lane_off + c * 32, v);
          }
          tmem_wait_st();
        }
      }
      l = l * alpha + rs;
      // P row -> shared memory, 128-byte swizzled K-major (16-byte chunk c of row r
      // sits at chunk position c ^ (r & 7) of its 128-byte line)
#pragma unroll
      for (int c = 0; c < kTile / 8; ++c) {
        const int box = c >> 3, cc = c & 7;
        uint4 val = make_uint4(pk[c * 4 + 0], pk[c * 4 + 1], pk[c * 4 + 2], pk[c * 4 + 3]);
        *reinterpret_cast<uint4*>(sP + box * 16384 + r * 128 + ((cc ^ (r & 7)) << 4)) = val;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full);
    }
    if (ok && T > 0) ok = mbar_wait(&bars->o_ready, (T - 1) & 1, abort, a.status);
    if (ok) {
      tc_fence_after();
      const int qrow = q0 + r;
      const float inv_l = (T > 0 && l > 0.f) ? 1.f / l : 0.f;
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(a.O) + (static_cast<size_t>(h) * a.Nq + qrow) * d;
      for (int c = 0; c < d / 32; ++c) {
        uint32_t v[32];
        if (T > 0) {
          tmem_ld32(tO + lane_off + c * 32, v);
          tmem_wait_ld_reg(v);
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) v[k] = 0u;
        }
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
      if (a.lse && qrow < a.Nq)
        a.lse[static_cast<size_t>(h) * a.Nq + qrow] =
            (T > 0) ? (m * sl2 + __log2f(l)) * 0.6931471805599453f : -INFINITY;
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
  return 1024 + 5 * tile + static_cast<size_t>(kTile) * kTile * 2 + kBarBytes;
}

cudaError_t launch_attend_bf16(const AttnArgs& a, cudaStream_t st) {
  if (a.Nq <= 0) return cudaSuccess;
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
  const int grid = a.H * ((a.Nq + kTile - 1) / kTile);
  LaunchTrace trace("attend_bf16_kernel", st);
  attend_bf16_kernel<<<grid, kThreads, smem, st>>>(maps, a);
  return cudaGetLastError();
}

cudaError_t launch_attend_f32(const AttnArgs& a, cudaStream_t st) {
  if (a.Nq <= 0) return cudaSuccess;
  if (a.d > kF32MaxD) return cudaErrorInvalidValue;
  dim3 grid((a.Nq + 3) / 4, a.H);
  LaunchTrace trace("attend_f32_kernel", st);
  attend_f32_kernel<<<grid, 128, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace kvb
