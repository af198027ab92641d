// Soft-Riesz density Gram: out[h][r] = sum_c sign(c) * phi(||R_r - C_c||^2 / h)
// (DensityKV §3 "Soft-Riesz Density", App. B.1 incremental update).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace kvb {

constexpr int kGramRowTile = 128;      // rows per TMEM accumulator (M of the MMA)
constexpr int kGramRowBlock = 256;     // rows per work unit (two accumulators)
constexpr int kGramColTile = 256;      // columns per MMA (N) and per work step
constexpr int kGramThreads = 640;      // 4 control warps + 16 epilogue warps
constexpr int kGramMaxHeads = 64;      // heads of one launch

// A set of rows/cols: per head a count and a start row inside its buffer.  Each
// field is either a uniform value or (if the pointer is non-null) a device array
// indexed by head.
struct GramSet {
  int n_uni = 0;
  const int* n_dev = nullptr;
  int off_uni = 0;
  const int* off_dev = nullptr;
};

struct GramArgs {
  int H = 0;
  int d = 0;
  GramSet rows, cols;
  int use_diag = 0;                // exclude pair (r, c) with c == r + diag
  int diag_uni = 0;
  const int* diag_dev = nullptr;
  int nneg_uni = 0;                // columns c < nneg enter with sign -1
  const int* nneg_dev = nullptr;
  float kscale = 0.f;              // -2/h
  float eps = 0.f;
  float s = 2.f;
  int max_rows = 0;                // upper bound of the row count of any head
  int grid = 0;                    // CTAs launched
  int slots = 0;                   // partial slots per row block (two column halves per CTA)
  int min_steps = 1;               // every active CTA takes at least this many steps
  float* partial = nullptr;        // [slots][H][ldOut]
  int ldOut = 0;
  int* status = nullptr;
  // largest ||k||^2 among the rows and columns (null: unknown, always clamp t >= eps)
  const float* norm_max = nullptr;
  // a head whose row (column) count equals alt_rows_n (alt_cols_n) reads its rows
  // (columns) through the alternate tensor maps, from row 0; -1: never
  int alt_rows_n = -1, alt_cols_n = -1;
  // f32 SIMT path only
  const float* R32 = nullptr;      // [H][ldR][d]
  const float* C32 = nullptr;      // [H][ldC][d]
  int ldR = 0, ldC = 0;
};

// bf16 operands through TMA: tensor maps over [H][rows][d] and over the augmented
// rows [H][rows][32] (see launch_aug_rows); row maps use 128-row boxes, column maps
// 256-row boxes (kGramColTile).  The MMA accumulates a.b - (||a||^2 + ||b||^2)/2 =
// -||a - b||^2 / 2 directly.  R2 .. Ca2 are the alternate maps (GramArgs
// alt_rows_n / alt_cols_n); callers without alternates repeat R .. Ca.
struct GramMaps {
  CUtensorMap R, C, Ra, Ca;
  CUtensorMap R2, C2, Ra2, Ca2;
};
cudaError_t launch_gram_bf16(const GramArgs& a, const GramMaps& m, cudaStream_t st);
// f32 operands, CUDA-core direct differences (small problems).
cudaError_t launch_gram_f32(const GramArgs& a, cudaStream_t st);

// Sum the per-CTA partials of every row: out[h][r] = sum over the CTAs whose
// tile range covered the row's block (fixed order: deterministic).
cudaError_t launch_gram_reduce(const GramArgs& a, float* out, int ldOut, cudaStream_t st);

// Work of a launch is the sequence of (head, 256-row block, 256-column tile)
// steps, T in total (known only on the device).  Only G_eff = clamp(T / min_steps,
// 1, grid) CTAs work; CTA b takes steps [T b / G_eff, T (b+1) / G_eff), so a row
// block is covered by at most `slots` CTAs.  Fills grid/slots/min_steps.
void gram_plan(GramArgs& a, int max_col_tiles, int n_sm);

size_t gram_smem_bytes(int d);

}  // namespace kvb
