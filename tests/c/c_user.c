/* A plain C caller of the whole DensityKV path through include/kvb.h: one
 * workspace from cudaMalloc, one admit of a block of candidates, one attention
 * of the chunk's queries over [sink | bank | window], the per-head counters and
 * the device status.  Inputs are zero-filled (the point is the calling
 * sequence, argument layout and error handling, not the numbers).  Built by
 * tests/test_abi.py as a compile-and-link check and run on the GPU by
 * tests/test_gpu_c_user.py; it needs a GPU with
 * sm_100a: ./c_user */
#include <stdio.h>
#include <stdlib.h>

#include <cuda_runtime.h>

#include "kvb.h"

#define CHECK(call)                                                          \
  do {                                                                       \
    kvb_status s_ = (call);                                                  \
    if (s_ != KVB_OK) {                                                      \
      fprintf(stderr, "%s: %s\n", #call, kvb_status_string(s_));            \
      return 1;                                                              \
    }                                                                        \
  } while (0)

int main(void) {
  enum { H = 2, D = 128, M = 512, N = 256, NQ = 256, LS = 64 };
  kvb_config c = {0};
  c.method = KVB_DENSITYKV;
  c.dtype = KVB_BF16;
  c.layers = 1;
  c.heads = H;
  c.head_dim = D;
  c.capacity = M;
  c.max_candidates = N;
  c.tau = 2.0f;
  c.eps = 1e-3f;
  c.s = 2.0f;
  c.sync_heads = 1;
  c.max_queries = NQ;

  const size_t ws_bytes = kvb_workspace_size(&c);
  if (ws_bytes == 0) return 1;
  void *ws = NULL, *cand = NULL, *q = NULL, *o = NULL, *sink = NULL;
  int32_t* ids = NULL;
  const size_t row = (size_t)D * 2; /* bf16 */
  if (cudaMalloc(&ws, ws_bytes) != cudaSuccess || cudaMalloc(&cand, (size_t)H * N * row) != cudaSuccess ||
      cudaMalloc((void**)&ids, N * sizeof(int32_t)) != cudaSuccess ||
      cudaMalloc(&q, (size_t)H * NQ * row) != cudaSuccess || cudaMalloc(&o, (size_t)H * NQ * row) != cudaSuccess ||
      cudaMalloc(&sink, (size_t)H * LS * row) != cudaSuccess)
    return 1;
  cudaMemset(cand, 0, (size_t)H * N * row);
  cudaMemset(q, 0, (size_t)H * NQ * row);
  cudaMemset(sink, 0, (size_t)H * LS * row);
  int32_t host_ids[N];
  for (int i = 0; i < N; ++i) host_ids[i] = 1000 + i;
  cudaMemcpy(ids, host_ids, sizeof(host_ids), cudaMemcpyHostToDevice);

  cudaStream_t st;
  cudaStreamCreate(&st);
  kvb_bank* bank = NULL;
  CHECK(kvb_bank_create(&c, ws, ws_bytes, st, &bank));
  /* candidates double as keys and values here */
  CHECK(kvb_admit(bank, 0, cand, cand, ids, N, st));
  /* the chunk's own tokens are the window: reuse the candidate buffer */
  CHECK(kvb_attend(bank, 0, q, NQ, sink, sink, LS, cand, cand, N, o, NULL, st));
  kvb_admit_stats stats[H];
  CHECK(kvb_read_stats(bank, 0, stats, st));
  CHECK(kvb_device_status(bank, st));
  for (int h = 0; h < H; ++h)
    printf("head %d: admitted %d, bank size %d\n", h, stats[h].admitted, stats[h].size);
  CHECK(kvb_bank_destroy(bank));
  cudaStreamDestroy(st);
  cudaFree(ws);
  cudaFree(cand);
  cudaFree(ids);
  cudaFree(q);
  cudaFree(o);
  cudaFree(sink);
  return 0;
}
