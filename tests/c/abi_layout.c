/* Plain C99 user of the kvb C ABI: prints the layout of the public structs and
 * the results of the host-only entry points, one "key value" pair per line, so
 * that tests/test_abi.py can check the ctypes mirror against the C compiler's
 * view of include/kvb.h.  Calls nothing that needs a GPU. */
#include <stddef.h>
#include <stdio.h>

#include "kvb.h"

#define FIELD(T, f) printf(#T "." #f " %zu\n", offsetof(T, f))

int main(void) {
  printf("sizeof.kvb_config %zu\n", sizeof(kvb_config));
  FIELD(kvb_config, method);
  FIELD(kvb_config, dtype);
  FIELD(kvb_config, layers);
  FIELD(kvb_config, heads);
  FIELD(kvb_config, head_dim);
  FIELD(kvb_config, capacity);
  FIELD(kvb_config, max_candidates);
  FIELD(kvb_config, tau);
  FIELD(kvb_config, eps);
  FIELD(kvb_config, s);
  FIELD(kvb_config, dist_scale);
  FIELD(kvb_config, sync_heads);
  FIELD(kvb_config, frame_h);
  FIELD(kvb_config, frame_w);
  FIELD(kvb_config, seg_h);
  FIELD(kvb_config, seg_w);
  FIELD(kvb_config, hist_frames);
  FIELD(kvb_config, max_new_frames);
  FIELD(kvb_config, retention);
  FIELD(kvb_config, max_queries);
  FIELD(kvb_config, cand_order);
  FIELD(kvb_config, baselines);
  FIELD(kvb_config, evict_order);
  FIELD(kvb_config, bottomk_scope);
  FIELD(kvb_config, sim_source);
  FIELD(kvb_config, storage);
  printf("sizeof.kvb_admit_stats %zu\n", sizeof(kvb_admit_stats));
  FIELD(kvb_admit_stats, admitted);
  FIELD(kvb_admit_stats, feasible);
  FIELD(kvb_admit_stats, mandatory);
  FIELD(kvb_admit_stats, capacity_evicted);
  FIELD(kvb_admit_stats, size);
  FIELD(kvb_admit_stats, moved);
  FIELD(kvb_admit_stats, near_ties);
  FIELD(kvb_admit_stats, reserved);
  printf("sizeof.kvb_trace_record %zu\n", sizeof(kvb_trace_record));
  FIELD(kvb_trace_record, kernel);
  FIELD(kvb_trace_record, ms);
  FIELD(kvb_trace_record, device);

  /* the 480P DensityKV layer: 12 heads, d 128, M 9360, N 4680 */
  kvb_config c = {0};
  c.method = KVB_DENSITYKV;
  c.dtype = KVB_BF16;
  c.layers = 1;
  c.heads = 12;
  c.head_dim = 128;
  c.capacity = 9360;
  c.max_candidates = 4680;
  c.tau = 2.0f;
  c.eps = 1e-3f;
  c.s = 2.0f;
  c.sync_heads = 1;
  c.seg_h = 4;
  c.seg_w = 4;
  c.hist_frames = 21;
  c.max_new_frames = 3;
  c.retention = 0.7f;
  c.max_queries = 4680;
  printf("workspace.wan480 %zu\n", kvb_workspace_size(&c));
  c.evict_order = 3; /* not a kvb_evict_order */
  printf("workspace.invalid %zu\n", kvb_workspace_size(&c));
  printf("status.0 %s\n", kvb_status_string(KVB_OK));
  return 0;
}
