/*
 * kvb -- historical KV-bank management for chunk-by-chunk autoregressive video
 * diffusion, and attention of the current chunk over the retained history.
 * Hand-written sm_100a (B200) kernels behind a plain C ABI.
 *
 * Two cache policies are implemented:
 *
 *  - DensityKV ("DensityKV: Density-Guided KV Cache Compression for Long Video
 *    Generation"): per-(layer, head) banks of exact K/V pairs, at most M per
 *    head (App. B.1 "Online Bank Update"), updated after every finalised block by
 *    Soft-Riesz density over post-RoPE keys (§3 "Soft-Riesz Density"): candidates
 *    are ordered by mean-normalised disturbance, the largest prefix feasible for
 *    every head is admitted (synchronised admission, App. E), bank entries whose
 *    projected growth ratio crosses tau are evicted first, then the highest-ratio
 *    entries until the bank fits M (§3), co-admitted entries set their insertion
 *    baselines together (App. B.1).
 *  - Forcing-KV ("Forcing-KV: Hybrid KV Cache Compression for Efficient
 *    Autoregressive Video Diffusion Models"): static heads attend [sink,
 *    transition frame, current chunk] (§3.3); dynamic heads keep, per history
 *    frame, the BottomK(floor(r n)) segments least similar (mean token cosine) to
 *    the same segment of the next frame (§3.4, §3.5).
 *
 * Formulas where the pages give none (the readings this library implements):
 *   phi(x) = (x + eps)^(-s/2),  x = ||a - b||^2 / h   (h = dist_scale, 0 => d)
 *   rho_B(c) = sum_{i in B} phi(x(c, k_i))
 *   score(c) = rho_B(c) / mean_{i in B} rho0_i        (feasible iff <= tau;
 *              an empty bank or a zero mean baseline makes every candidate
 *              feasible with score 0)
 *   P = min(min_h #feasible_h, M, N) (sync_heads=1); each head admits its P
 *       lowest (score, id)
 *   ratio_i = (rho_i + sum_{c in A_h} phi(c, i)) / rho0_i  (0 if rho0_i = 0);
 *       evicted: every ratio_i > tau, then max(0, |B|-|mandatory|+P-M) more by
 *       (ratio descending, id ascending)
 *   new entries: rho0 = rho = density within the updated bank.
 *   (The App. E ablation switches of kvb_config -- cand_order, baselines,
 *   evict_order -- each replace one of these rules; see their enums.)
 *
 * Conventions
 *  - All device pointers are caller-owned device memory, head-major and
 *    contiguous: a [H][L][d] tensor is H*L*d elements, row d contiguous.  Key
 *    and value element type is the bank's dtype (bf16 or f32); ids are int32.
 *  - `stream` is a cudaStream_t (passed as void*).  Every call is asynchronous on
 *    that stream unless its comment says it synchronises.
 *  - The library never allocates device memory.  The caller provides one device
 *    workspace (size from kvb_workspace_size, 256-byte aligned) that holds every
 *    bank, the scratch of every step and a device status word.  Host-side state
 *    (the opaque kvb_bank) is malloc'd by kvb_bank_create and freed by destroy.
 *  - Argument errors return before anything is launched.  Device-side failures
 *    (a bounded wait that gave up, an index a kernel refused) are latched into
 *    the status word and reported by kvb_device_status; kernels never trap.
 *  - Token ids must be unique across a layer's bank and the candidate block, and
 *    non-negative: every ordering by id (tie-breaks, source order) compares them
 *    as unsigned 32-bit values.
 */
#ifndef KVB_H
#define KVB_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KVB_API __attribute__((visibility("default")))
#else
#define KVB_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KVB_OK = 0,
  KVB_E_INVAL = 1,          /* bad argument (null, size out of range, ...); nothing launched */
  KVB_E_WORKSPACE = 2,      /* workspace null, too small or not 256-byte aligned */
  KVB_E_CUDA = 3,           /* a CUDA runtime call (launch, memcpy, attribute) failed */
  KVB_E_DEVICE_TIMEOUT = 4, /* a kernel's bounded wait gave up (latched on device) */
  KVB_E_DEVICE_BOUNDS = 5,  /* a kernel refused an out-of-range index (latched on device) */
  KVB_E_STATE = 6,          /* call not valid for this bank (wrong method, layer, ...) */
  KVB_E_UNSUPPORTED = 7     /* valid but not implemented here (e.g. head_dim not 64/128) */
} kvb_status;

typedef enum { KVB_BF16 = 0, KVB_F32 = 1 } kvb_dtype;

typedef enum { KVB_DENSITYKV = 0, KVB_FORCINGKV = 1 } kvb_method;

typedef struct {
  kvb_method method;
  kvb_dtype dtype;        /* storage/compute input type of K, V, Q, O */
  int32_t layers;         /* number of independent layers held by the bank */
  int32_t heads;          /* H, 1..64 */
  int32_t head_dim;       /* d: 64 or 128 */
  /* DensityKV */
  int32_t capacity;       /* M per (layer, head), >= 1 */
  int32_t max_candidates; /* upper bound on N of kvb_admit */
  float tau;              /* growth bound (DensityKV App. D default 2.0) */
  float eps;              /* Soft-Riesz regulariser */
  float s;                /* Soft-Riesz decay exponent */
  float dist_scale;       /* h; 0 => head_dim */
  int32_t sync_heads;     /* 1: shared admitted count across heads (App. E default) */
  /* Forcing-KV */
  int32_t frame_h, frame_w; /* token grid of one latent frame; F = frame_h*frame_w */
  int32_t seg_h, seg_w;     /* segment tile (edge segments are partial) */
  int32_t hist_frames;      /* frames of pruned history kept by dynamic heads */
  int32_t max_new_frames;   /* upper bound on the frames pushed per kvb_prune_hybrid */
  float retention;          /* r: each frame keeps floor(r * n_segments) segments */
  /* attention */
  int32_t max_queries;      /* upper bound on Nq of kvb_attend */
  /* DensityKV ablation switches (DensityKV App. E "Ablation Details"); 0 is the
   * default policy everywhere, so a zero-filled tail keeps it. */
  int32_t cand_order;       /* kvb_cand_order */
  int32_t baselines;        /* kvb_baselines */
  int32_t evict_order;      /* kvb_evict_order */
  /* Forcing-KV variants (reading notes §3.4, §3.5); 0 is the per-frame, per-layer
   * rule, so a zero-filled tail keeps it. */
  int32_t bottomk_scope;    /* kvb_bottomk_scope */
  int32_t sim_source;       /* kvb_sim_source */
  /* storage of the retained K/V (0: the bank's dtype) */
  int32_t storage;          /* kvb_storage */
} kvb_config;

/* Candidate ordering (App. E, candidate ordering).
 *  KVB_ORDER_DISTURBANCE: candidates by (score ascending, id ascending); the
 *    feasible prefix is every candidate with score <= tau.
 *  KVB_ORDER_SOURCE: candidates in spatiotemporal source order, i.e. by id
 *    ascending; a head's feasible prefix is the run of candidates, from the
 *    lowest id, that ends before its lowest-id infeasible candidate. */
typedef enum { KVB_ORDER_DISTURBANCE = 0, KVB_ORDER_SOURCE = 1 } kvb_cand_order;

/* Density baselines (App. E, baselines).
 *  KVB_BASELINES_FIXED: rho0 is frozen at insertion (co-admitted entries set it
 *    together, after the update).
 *  KVB_BASELINES_REFRESH: after every update every entry's rho0 becomes its
 *    density within the updated bank. */
typedef enum { KVB_BASELINES_FIXED = 0, KVB_BASELINES_REFRESH = 1 } kvb_baselines;

/* Eviction set (App. E, eviction).
 *  KVB_EVICT_THRESHOLD_RATIO: every ratio_i > tau, then the capacity evictions by
 *    (ratio descending, id ascending).
 *  KVB_EVICT_DENSEST: no threshold step; max(0, |B| + P - M) entries by
 *    (projected density rho_i + sum_A phi descending, id ascending).
 *  KVB_EVICT_THRESHOLD_SOURCE: every ratio_i > tau, then the capacity evictions
 *    by id ascending (oldest source position first). */
typedef enum { KVB_EVICT_THRESHOLD_RATIO = 0, KVB_EVICT_DENSEST = 1, KVB_EVICT_THRESHOLD_SOURCE = 2 } kvb_evict_order;

/* Scope of Forcing-KV's BottomK (reading notes §3.4 formula vs the §3.5 listing).
 *  KVB_BOTTOMK_FRAME: each frame keeps its floor(r n) least similar segments.
 *  KVB_BOTTOMK_CALL: the (frame, segment) pairs of all frames one
 *    kvb_prune_hybrid call pushes are ranked together and the
 *    floor(r n n_frames) least similar are kept (ties: the lower frame, then the
 *    lower segment), so a frame may keep more or fewer than floor(r n).
 *    Requires max_new_frames * n_segments <= 4096. */
typedef enum { KVB_BOTTOMK_FRAME = 0, KVB_BOTTOMK_CALL = 1 } kvb_bottomk_scope;

/* Where Forcing-KV's segment similarities come from (reading notes §3.4
 * implementation notes: a first-block proxy with shared indices).
 *  KVB_SIM_PER_LAYER: every layer's dynamic heads rank their own keys.
 *  KVB_SIM_FIRST_LAYER: layer 0's call computes the similarities of every head
 *    (static ones too) from its own keys; a later layer's call reuses them, so
 *    head h of every layer keeps the segments head h of layer 0 selects, filled
 *    with that layer's own K and V.  Layer 0 must be pruned first with each new
 *    chunk: a call for layer > 0 returns KVB_E_STATE before layer 0 has been
 *    pruned, or when its n_frames differs from layer 0's last call. */
typedef enum { KVB_SIM_PER_LAYER = 0, KVB_SIM_FIRST_LAYER = 1 } kvb_sim_source;

/* Storage of a DensityKV bank's K and V (bf16 banks).  The Forcing-KV reading
 * notes report the method combined with FP8 (results); this library's reading is
 * the retained history held in FP8 E4M3.
 *  KVB_STORE_NATIVE: K and V in the bank's dtype.
 *  KVB_STORE_FP8_E4M3: every layer's bank K and V are held in FP8 E4M3 (1 sign,
 *    4 exponent bits with bias 7, 3 mantissa bits; one byte per element).
 *    kvb_admit first rounds the candidates' K and V to E4M3 (to nearest, ties
 *    to even, saturating at +-448), so every density, score, ratio and baseline
 *    of the step and of later steps is computed from the values the bank stores;
 *    kvb_bank_import rounds what it is given the same way and kvb_bank_export
 *    returns the stored values as bf16.  The layer being updated or attended is
 *    decompressed into one bf16 working copy (one layer's K and V, shared by the
 *    layers) that the density and attention kernels read; the persistent
 *    per-layer storage is half that of bf16.  An f32 bank returns KVB_E_INVAL
 *    from kvb_workspace_size / kvb_bank_create with this storage. */
typedef enum { KVB_STORE_NATIVE = 0, KVB_STORE_FP8_E4M3 = 1 } kvb_storage;

/* Per-(layer, head) counters of the last kvb_admit / kvb_prune_hybrid. */
typedef struct {
  int32_t admitted;      /* P (DensityKV) or kept tokens pushed (Forcing-KV) */
  int32_t feasible;      /* DensityKV: length of the head's feasible prefix (the
                            candidates with score <= tau; KVB_ORDER_SOURCE: the
                            leading run of them in id order) */
  int32_t mandatory;     /* evictions with ratio > tau */
  int32_t capacity_evicted;
  int32_t size;          /* bank size after the update (ring size for Forcing-KV) */
  int32_t moved;         /* DensityKV: surviving entries moved from the tail into holes */
  int32_t near_ties;     /* DensityKV: decisions of this step whose deciding value, as the
                            kernels compute it in fp32, lies within 1e-4 (relative) of its
                            threshold (a score or projected ratio vs tau) or of the value
                            across its cut (the shared-prefix cut, the capacity cut):
                            the decisions another rounding could take the other way */
  int32_t reserved;
} kvb_admit_stats;

typedef struct kvb_bank kvb_bank; /* opaque, host-side */

/* Bytes of device workspace kvb_bank_create needs for `cfg`; 0 if cfg is invalid. */
KVB_API size_t kvb_workspace_size(const kvb_config* cfg);

/* A bank holds the retained history of every (layer, head): for DensityKV an
 * independent bank of at most M exact (id, K, V) entries per layer and head with
 * their densities and insertion baselines (DensityKV App. B.1 "Online Bank
 * Update", App. D); for Forcing-KV each static head's transition frame and each
 * dynamic head's FIFO of pruned frames (Forcing-KV reading notes §3.3, §3.4).
 * Bind a bank to a caller-owned workspace (>= kvb_workspace_size bytes, 256-B
 * aligned).  Clears the status word and every bank to empty with async memsets
 * on `stream`.  *out receives a host handle.  KVB_E_INVAL / KVB_E_WORKSPACE /
 * KVB_E_UNSUPPORTED on bad config or workspace; KVB_E_CUDA if the device is not
 * an sm_100 part. */
KVB_API kvb_status kvb_bank_create(const kvb_config* cfg, void* workspace, size_t workspace_bytes,
                           void* stream, kvb_bank** out);

/* Free the host handle (the workspace stays the caller's). */
KVB_API kvb_status kvb_bank_destroy(kvb_bank* bank);

/* DensityKV admit of one finalised block into layer `layer` (App. B.1):
 * candK, candV: device [H][N][d]; cand_ids: device [N] int32 (new ids);
 * 1 <= N <= max_candidates.  Launches the density Gram passes, selection,
 * eviction and compaction on `stream`; no host synchronisation. */
KVB_API kvb_status kvb_admit(kvb_bank* bank, int32_t layer, const void* candK, const void* candV,
                     const int32_t* cand_ids, int32_t N, void* stream);

/* kvb_admit in two halves, for banks whose heads are split across processes or
 * GPUs (each holding some heads of a layer) under synchronised admission: the
 * shared prefix P = min over ALL heads of the layer is the one value they must
 * exchange (DensityKV App. E cross-head synchronisation).
 *   kvb_admit_begin: the arguments of kvb_admit plus prefix_out (device int32):
 *     launches the candidate densities and feasible counts, then writes
 *     min(min_h #feasible_h over this bank's heads, M, N) to *prefix_out.
 *   kvb_admit_finish: completes the begun step of `layer` with
 *     P = min(this bank's prefix, max(0, *prefix_bound)); prefix_bound is a
 *     device int32 (typically the MIN over every process's prefix_out) or NULL
 *     (then the result equals kvb_admit's).  Requires sync_heads = 1 when
 *     prefix_bound is not NULL (KVB_E_INVAL otherwise).
 * Between the two calls the caller's candidate buffers must stay valid and
 * nothing else may run on this bank; kvb_admit, kvb_admit_begin and
 * kvb_bank_import cancel a begun step.  kvb_admit_finish without a begun step
 * of that layer returns KVB_E_STATE.  Both are asynchronous on `stream`. */
KVB_API kvb_status kvb_admit_begin(kvb_bank* bank, int32_t layer, const void* candK, const void* candV,
                                   const int32_t* cand_ids, int32_t N, int32_t* prefix_out, void* stream);
KVB_API kvb_status kvb_admit_finish(kvb_bank* bank, int32_t layer, const int32_t* prefix_bound, void* stream);

/* Forcing-KV history update with the frames of a finalised chunk (§3.3-§3.5):
 * head_is_static: host [H] (1 static, 0 dynamic); newK/newV: device
 * [H][n_frames*F][d] (frames oldest first; the sink frame is never passed);
 * nextK: device [H][F][d], the first frame of the next chunk (successor of the
 * last new frame); new_ids: device [n_frames*F] int32.  Static heads take the
 * last new frame as their transition frame; dynamic heads push each new frame's
 * BottomK segments into their FIFO of hist_frames frames.  newK, newV and nextK
 * must be 16-byte aligned (KVB_E_INVAL otherwise). */
KVB_API kvb_status kvb_prune_hybrid(kvb_bank* bank, int32_t layer, const uint8_t* head_is_static,
                            const void* newK, const void* newV, const void* nextK,
                            const int32_t* new_ids, int32_t n_frames, void* stream);

/* Attention of the current chunk's queries over [sink | history(layer) | window]
 * -- the retained states read directly by the model's native attention (DensityKV
 * Fig. 2 and §5; Forcing-KV reading notes §3.3 and the §3.5 listing: static heads
 * over [sink, transition frame, current chunk], dynamic heads over [sink, retained
 * history, current chunk]):
 * Q, O: device [H][Nq][d]; sinkK/V [H][Ls][d]; winK/V [H][Lw][d]; lse: device
 * [H][Nq] f32 (natural log) or NULL.  O = softmax(Q K^T / sqrt(d)) V, no mask.
 * History is the DensityKV bank, or for Forcing-KV the transition frame (static
 * heads) / the pruned FIFO (dynamic heads).  1 <= Nq <= max_queries. */
KVB_API kvb_status kvb_attend(kvb_bank* bank, int32_t layer, const void* Q, int32_t Nq,
                      const void* sinkK, const void* sinkV, int32_t Ls,
                      const void* winK, const void* winV, int32_t Lw,
                      void* O, float* lse, void* stream);

/* Copy the counters of `layer` (H entries) to host memory.  Synchronises `stream`. */
KVB_API kvb_status kvb_read_stats(kvb_bank* bank, int32_t layer, kvb_admit_stats* host_out, void* stream);

/* Export one (layer, head) DensityKV bank, or Forcing-KV history, into caller
 * device buffers of capacity rows (M for DensityKV, hist_frames*F for
 * Forcing-KV): ids [cap] int32, rho/rho0 [cap] f32 (may be NULL; zero for
 * Forcing-KV), K/V [cap][d].  *size (host) receives the entry count.  Rows are in
 * the bank's slot order (Forcing-KV: oldest frame first).  Synchronises `stream`. */
KVB_API kvb_status kvb_bank_export(kvb_bank* bank, int32_t layer, int32_t head, int32_t* ids, float* rho,
                           float* rho0, void* K, void* V, int32_t* size, void* stream);

/* Load one (layer, head) DensityKV bank from caller device buffers (size <= M):
 * ids, rho (current density within the bank), rho0 (frozen baselines), K, V.
 * Replaces the bank's contents; used for checkpoint/resume and stepwise tests.
 * A Forcing-KV bank returns KVB_E_STATE: its history is exported, not restored. */
KVB_API kvb_status kvb_bank_import(kvb_bank* bank, int32_t layer, int32_t head, const int32_t* ids,
                           const float* rho, const float* rho0, const void* K, const void* V,
                           int32_t size, void* stream);

/* Synchronise `stream` and return the first latched device error (KVB_OK if none). */
KVB_API kvb_status kvb_device_status(kvb_bank* bank, void* stream);

/* Number of kernels the library has launched in this process (all entry points,
 * all devices); a diagnostic for callers that account launches. */
KVB_API unsigned long long kvb_launch_count(void);

/* Launch tracing, a per-kernel timing aid.  While enabled, every kernel launch of
 * the library is bracketed by a pair of CUDA events recorded on the stream the
 * kernel is launched on, and the pair is kept with the kernel's name.  Meant for a
 * single host thread driving the library.  Off by default.
 *   kvb_trace_enable: switch tracing on (nonzero) or off; either way, drop the
 *     records held so far.  Never fails.
 *   kvb_trace_read: wait for the recorded events, write up to `max_records`
 *     records in launch order into caller host memory `out`, set *n_out to the
 *     number of records held (which may exceed max_records), then drop them all.
 *     kernel: static name string owned by the library; ms: the launch's device
 *     time in milliseconds, or -1 when its events could not be read (the call then
 *     returns KVB_E_CUDA after filling the rest); device: CUDA ordinal.
 *     KVB_E_INVAL if n_out is NULL or max_records < 0 or out is NULL with
 *     max_records > 0.  At most 65536 launches are held; later ones are counted
 *     by kvb_launch_count but not traced. */
typedef struct {
  const char* kernel;
  float ms;
  int32_t device;
} kvb_trace_record;
KVB_API kvb_status kvb_trace_enable(int32_t enable);
KVB_API kvb_status kvb_trace_read(kvb_trace_record* out, int32_t max_records, int32_t* n_out);

/* Static string for a status code. */
KVB_API const char* kvb_status_string(kvb_status st);

/* Self-test of the device-side failure detection (no counterpart on the pages).
 * Every mbarrier wait of the tensor-core kernels is bounded; on expiry it
 * latches KVB_E_DEVICE_TIMEOUT into the status word and raises its CTA's abort
 * flag, on which every other role of the CTA gives up its own wait.  This call
 * runs that wait, asynchronously on `stream`, in one CTA with two roles, each on
 * an mbarrier that nothing ever arrives on: role 0 with the limit `timeout_ns`,
 * role 1 with 50 x `timeout_ns`, so that role 1 returns early only through the
 * abort flag.  No fault, trap or unbounded wait is involved.
 *   status: device int32, the word the timeout is latched into (the first
 *           nonzero code stays; clear it to 0 before the call to observe it).
 *   out:    device int64[4]: out[0] = 1 if role 0's wait completed (never),
 *           out[1] = role 0's wait in ns, out[2], out[3] the same for role 1.
 *   timeout_ns: 1e3 .. 1e8 (1 us .. 100 ms; the kernels' own limit is 2 s).
 * KVB_E_INVAL on a NULL pointer or a limit out of range (nothing launched);
 * KVB_E_CUDA if the launch fails. */
KVB_API kvb_status kvb_selftest_timeout(int32_t* status, int64_t* out, int64_t timeout_ns, void* stream);

/* ------------------------------------------------------------------------------
 * Operation-level entry points: the same kernels on caller buffers, for callers
 * that manage their own caches.  They use the scratch of a caller workspace.
 * ---------------------------------------------------------------------------- */

/* Bytes of scratch kvb_density needs for these sizes (0 on invalid sizes). */
KVB_API size_t kvb_density_workspace_size(int32_t heads, int32_t n_rows, int32_t n_cols, int32_t head_dim,
                                  kvb_dtype dtype);

/* Soft-Riesz density of every row against every column, per head (DensityKV §3):
 *   out[h][r] = sum_{c < n_cols} phi(||rows[h][r] - cols[h][c]||^2 / h_scale)
 * rows [H][n_rows][d], cols [H][n_cols][d] device; out [H][n_rows] f32 device.
 * If `exclude_diagonal` is nonzero, rows and cols must be the same set in the same
 * order (n_rows == n_cols) and the pair c == r is skipped (a key's density within
 * its own bank).  dist_scale 0 => head_dim.  workspace: device scratch of
 * kvb_density_workspace_size bytes, 256-B aligned.  The first 4 bytes of the
 * workspace are this call's device status word (zeroed by the call, then set to a
 * kvb_status code by a kernel that gives up; read it with a copy after a sync). */
KVB_API kvb_status kvb_density(const void* rows, int32_t n_rows, const void* cols, int32_t n_cols,
                       int32_t heads, int32_t head_dim, kvb_dtype dtype, float dist_scale,
                       float eps, float s, int32_t exclude_diagonal, float* out,
                       void* workspace, size_t workspace_bytes, void* stream);

/* kvb_density for callers that cannot allocate device memory.  (The pages have
 * no counterpart: this is an interface for a host application whose allocator
 * owns all device memory and forbids allocations outside it, or for a
 * latency-critical loop that must not pay for an allocation, and which therefore
 * cannot hand the library a scratch workspace.)
 * Same inputs, outputs and results as kvb_density with dtype KVB_BF16; the
 * scratch lives in one 4 MiB array inside the library's device image, held by
 * every GPU that loads the library until the process exits.  Sizes are rejected
 * with KVB_E_WORKSPACE (nothing launched) unless
 *   256 + 64*H*n_rows + 64*H*n_cols + 64*H*n_rows  (each term rounded up to
 *   256 bytes)  <=  4 MiB.
 * The first call on a device looks up the array's address with that device
 * current: make it before any stream capture.  The address is kept for the life
 * of the process; after a cudaDeviceReset of that device it is stale, so do not
 * call this entry point on a device that has been reset.  All calls on a device
 * share the array (it keeps the last call's contents); calls that overlap on the
 * GPU race, so order them on one stream.  status_out: device int32 that receives
 * this call's device status (zeroed by the call).  It may be NULL: a device-side
 * failure (a bounded wait that gave up) is then written to a word inside the
 * shared array that no call reads back, so it goes unreported and `out` may hold
 * partial sums; pass status_out to learn of it. */
KVB_API kvb_status kvb_density_noalloc(const void* rows, int32_t n_rows, const void* cols, int32_t n_cols,
                                       int32_t heads, int32_t head_dim, kvb_dtype dtype, float dist_scale,
                                       float eps, float s, int32_t exclude_diagonal, float* out,
                                       int32_t* status_out, void* stream);

/* Segment-wise cosine similarity of Forcing-KV (§3.4): for every head and every
 * frame t < n_frames, sim[h][t][j] = mean over the tokens p of segment j of
 * cos(K[h][t][p], succ[h][t][p]) with succ = frame t+1 of K, or `nextK` for the
 * last frame.  K [H][n_frames*F][d], nextK [H][F][d]; sim [H][n_frames][n_seg]
 * f32 with n_seg = ceil(frame_h/seg_h)*ceil(frame_w/seg_w), segments row-major.
 * cos(a, b) = a.b / max(|a| |b|, 1e-8).  K and nextK must be 16-byte aligned
 * (KVB_E_INVAL) and head_dim * element size a multiple of 16 bytes
 * (KVB_E_UNSUPPORTED). */
KVB_API kvb_status kvb_segment_cosine(const void* K, const void* nextK, int32_t heads, int32_t n_frames,
                              int32_t frame_h, int32_t frame_w, int32_t seg_h, int32_t seg_w,
                              int32_t head_dim, kvb_dtype dtype, float* sim, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* KVB_H */
