/*
 * isa.h -- C ABI of libisa.so: importance-sampled block-sparse attention on
 * NVIDIA B200 (sm_100a).
 *
 * The method (pages cited by title and section):
 *   "AB-Attention: Accurate Block Attention for Accelerating Video Diffusion
 *   Transformers" -- abstract, and the discussion of the Intra-Block Clustering
 *   Selector (IBCS), Sampling with Inclusion-Probability weighting (SIP), the
 *   logit-shift form of the weights, and fine-grained selection with tiled
 *   execution;
 *   "InstaGen: Group-Shared Importance Sampling for Fast Video Generation" --
 *   abstract: block selection as importance sampling (exact set + a sample
 *   reweighted by inverse probability), one sample shared per query cluster.
 *
 * Pipeline: isa_score (estimated attention mass per query group and key
 * block) -> isa_select (plan: exact top blocks + a capped systematic PPS
 * sample with log(1/pi) weights) -> isa_attention (one sparse flash-attention
 * pass over the plan).  isa_dense_attention is the 100%-density limit.
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers owned by the caller, unless a
 *     parameter says "host".  The library never allocates or frees memory in a
 *     call; isa_create allocates the context's 4-byte device status word.
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL is the legacy default stream) and returns after enqueueing.
 *   - Host-side checks (shapes, null pointers, 16-byte alignment, budgets) are
 *     made before anything is enqueued; a failing call returns
 *     ISA_ERR_INVALID_ARG / ISA_ERR_UNSUPPORTED, enqueues nothing, and
 *     isa_last_error() says why.
 *   - Problems only the device can see (a block index out of range,
 *     non-finite mass, malformed group offsets, a pipeline wait that ran out)
 *     set the context's device status word; the kernel finishes without a
 *     fault.  isa_sync_status() synchronises the stream and returns (and
 *     clears) that word.
 *   - Layouts are contiguous row-major:
 *       Q, K, V, O   [B, H, N, d]  bf16
 *       mass         [B, H, G, nK] fp32       nK = ceil(N / k_block)
 *       idx, log_w   [B, H, G, S]  int32, fp32 S = n_exact + n_sample
 *       lse          [B, H, N]     fp32 (natural log)
 *   - A context serves one device; calls on one context are not thread-safe
 *     with respect to each other's status word.
 */
#ifndef ISA_H_
#define ISA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ISA_API __attribute__((visibility("default")))
#else
#define ISA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum isa_status {
  ISA_OK = 0,
  ISA_ERR_INVALID_ARG = 1,  /* bad shape, pointer, alignment or budget      */
  ISA_ERR_UNSUPPORTED = 2,  /* valid but not built (e.g. head_dim 96)        */
  ISA_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed             */
  ISA_ERR_TIMEOUT = 4,      /* device: a pipeline wait ran out (no fault)    */
  ISA_ERR_DEVICE_CHECK = 5  /* device: bad index / offsets / non-finite mass */
} isa_status;

typedef struct isa_context isa_context;

/* Problem shape shared by all calls.
 * Query groups: when q_offsets == NULL the groups are uniform blocks of
 * q_block rows, group g = rows [g*q_block, min((g+1)*q_block, N)) and
 * num_groups must equal ceil(N / q_block).  Otherwise group g is the cluster
 * of rows [q_offsets[g], q_offsets[g+1]) of a permuted layout ("each query
 * cluster draws one sample shared by all its queries", InstaGen abstract);
 * q_offsets is a DEVICE int32 array of num_groups+1 entries with
 * q_offsets[0] = 0, q_offsets[G] = N, strictly increasing (checked on the
 * device).  The same groups apply to every batch entry and head.
 * Key blocks: block b = rows [b*k_block, min((b+1)*k_block, N)); the last
 * block may be partial.  Small key blocks are gathered into 128-row tiles by
 * the attention kernel ("fine-grained selection with tiled execution"). */
typedef struct isa_shape {
  int32_t batch;             /* B >= 1                                   */
  int32_t heads;             /* H >= 1                                   */
  int32_t seq_len;           /* N >= 1                                   */
  int32_t head_dim;          /* d: 64 or 128                             */
  int32_t q_block;           /* uniform group rows, >= 1 (ignored if q_offsets) */
  int32_t k_block;           /* 16, 32, 64 or 128                        */
  int32_t num_groups;        /* G                                        */
  const int32_t* q_offsets;  /* device [G+1] or NULL                     */
  float scale;               /* logit scale > 0, normally 1/sqrt(d)      */
} isa_shape;

/* Sampling parameters of the fused pipeline calls. */
typedef struct isa_params {
  int32_t n_clusters;  /* C: k-means clusters per query group, 1..16     */
  int32_t n_iters;     /* I: k-means iterations, 1..16                   */
  int32_t n_exact;     /* k_e: exact top blocks per group                */
  int32_t n_sample;    /* n_s: sampled blocks per group                  */
  uint64_t seed;       /* Philox key of the per-group uniforms           */
} isa_params;

/* Create a context on CUDA device `device` (allocates its 4-byte device
 * status word).  *out receives the context.  Returns ISA_ERR_CUDA if the
 * device cannot be used, ISA_ERR_UNSUPPORTED if it is not sm_100. */
ISA_API isa_status isa_create(int device, isa_context** out);

/* Destroy a context (frees its status word).  NULL is allowed. */
ISA_API void isa_destroy(isa_context* ctx);

/* Static string for a status code. */
ISA_API const char* isa_status_string(isa_status status);

/* Message of the last host-side failure on this context ("" if none). */
ISA_API const char* isa_last_error(const isa_context* ctx);

/* Synchronise `stream`, then return and clear the device status word
 * (ISA_OK, ISA_ERR_TIMEOUT or ISA_ERR_DEVICE_CHECK), or ISA_ERR_CUDA if the
 * stream reported an error. */
ISA_API isa_status isa_sync_status(isa_context* ctx, void* stream);

/* ---------------------------------------------------------------------------
 * isa_score -- IBCS block scorer ("AB-Attention", Intra-Block Clustering
 * Selector: queries are clustered only within each query block; each cluster
 * gets a representative and a weight equal to its size; the representatives
 * score small key blocks without permuting tokens).
 *   kbar_b   = mean of the valid rows of key block b, L_b = their count;
 *   mu_c,n_c = Lloyd's k-means in each query group: init mu_c = row
 *              floor(c*n_g/C) of the group, n_iters rounds of (assign to the
 *              nearest centroid, ties to the lower c; move non-empty centroids
 *              to the mean of their rows); n_c = sizes of the last assignment;
 *   mass     = sum_c n_c * softmax_b(scale * mu_c . kbar_b + ln L_b),
 *              so every mass row sums to the group's row count.
 * q, k: [B,H,N,d] bf16.  mass: [B,H,G,nK] fp32 (written).
 * centroids: optional [B,H,G,C,d] fp32 output, counts: optional [B,H,G,C]
 * int32 output (NULL to skip).  workspace: device scratch of at least
 * isa_score_workspace_bytes(shape, n_clusters) bytes, 256-byte aligned.
 * 1 <= n_clusters <= 16, 1 <= n_iters <= 16.  A group with fewer rows than
 * clusters is allowed (duplicate initial centroids stay empty).
 * ------------------------------------------------------------------------- */
ISA_API size_t isa_score_workspace_bytes(const isa_shape* shape, int32_t n_clusters);
ISA_API isa_status isa_score(isa_context* ctx, const isa_shape* shape, const void* q, const void* k,
                     int32_t n_clusters, int32_t n_iters, float* mass, float* centroids,
                     int32_t* counts, void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * isa_select -- exact set + SIP sample, one plan row per (batch, head, group)
 * ("AB-Attention", Sampling with Inclusion-Probability weighting; "InstaGen"
 * abstract).
 *   exact set E = the n_exact largest mass values, ties to the lower block;
 *   rest R: integer weights w_b = floor(m_b / max_R m * 2^31) + 1 (all 1 if
 *   max_R m = 0), inclusion probabilities n' w_b / T capped at 1 by the
 *   fixed-point iteration (capped blocks always enter, log_w = 0);
 *   systematic PPS over the uncapped rest in ascending block order with one
 *   Philox4x64-10 uniform per group (key (seed, 0), counter (g, h, b, 0),
 *   U = high 32 bits of word 0), in exact 128-bit integer arithmetic;
 *   drawn blocks carry log_w = ln T - ln(n' w_b) = ln(1/pi) (fp64, stored fp32).
 *   Row layout: E ascending, then the capped and drawn blocks ascending.
 *   If n_sample >= nK - n_exact every remaining block enters with log_w 0.
 * mass: [B,H,G,nK] fp32 (non-finite values count as 0 and set
 * ISA_ERR_DEVICE_CHECK).  idx: [B,H,G,S] int32, log_w: [B,H,G,S] fp32
 * (written).  n_exact, n_sample >= 0, 1 <= n_exact + n_sample <= nK.
 * The result is bit-identical to the CPU oracle for identical mass.
 * ------------------------------------------------------------------------- */
ISA_API isa_status isa_select(isa_context* ctx, const isa_shape* shape, const float* mass,
                      int32_t n_exact, int32_t n_sample, uint64_t seed, int32_t* idx,
                      float* log_w, void* stream);

/* ---------------------------------------------------------------------------
 * isa_select_top_p -- a plan of n_select blocks per row whose exact part is
 * set by a share of the mass instead of a fixed count ("iCATS", top-p
 * sparsity: keep the blocks that carry a share p of the attention mass).
 * Per row, in exact integers:
 *   q_b = floor(m_b / max m * 2^31) (fp64; 0 where m_b <= 0),
 *   target = ceil(top_p * sum_b q_b) (fp64),
 *   k_e = min(n_select, the fewest blocks, taken by descending mass with
 *         ties to the lower block, whose q sum reaches target; 0 if target 0);
 * then the row is planned as isa_select with n_exact = k_e and
 * n_sample = n_select - k_e (same uniform, weights and row layout), so every
 * row holds n_select entries and the rest of the budget is sampled.
 * mass: [B,H,G,nK] fp32.  idx, log_w: [B,H,G,n_select] (written).
 * n_exact_rows: [B,H,G] int32 (written: k_e per row).  0 < top_p <= 1,
 * 1 <= n_select <= nK.  Bit-identical to the CPU oracle for identical mass.
 * ------------------------------------------------------------------------- */
ISA_API isa_status isa_select_top_p(isa_context* ctx, const isa_shape* shape, const float* mass,
                            double top_p, int32_t n_select, uint64_t seed, int32_t* idx,
                            float* log_w, int32_t* n_exact_rows, void* stream);

/* ---------------------------------------------------------------------------
 * Token clustering: the permuted layout of permuted block-sparse attention
 * ("InstaGen", abstract: PBSA computes blocks of a semantically permuted
 * attention matrix, and InstaGen is parameterised by SVG2, whose
 * semantic-aware permutation clusters the tokens of the whole sequence;
 * "AB-Attention" names that sequence-wide clustering and permutation as the
 * cost its in-block clustering avoids).  Per (batch, head), Lloyd's k-means
 * over all N rows of x with C clusters:
 *   init    mu_c = row floor(c N / C);
 *   assign  label_r = argmin_c ||x_r - mu_c||^2, ties to the lower c;
 *   sort    perm = the rows in (label, row) order (a stable counting sort);
 *           offsets[c] .. offsets[c+1] are cluster c's positions in perm;
 *   update  mu_c = mean of cluster c's rows (an empty cluster keeps mu_c);
 * n_iters rounds of (assign, sort, update); the labels, perm and offsets of
 * the last round are returned with the centroids after its update.  A query
 * cluster is one query group of the attention calls (q permuted by perm,
 * q_offsets = that head's groups, out un-permuted by isa_permute_rows with
 * inverse = 1); keys permuted by their own clustering form the key blocks.
 * Only batch, heads, seq_len and head_dim of `shape` are read; x is
 * [B,H,N,d] bf16.  The distances use x exact in bf16 and mu split into bf16
 * hi + lo parts (relative error at most 2^-18).  Relative to ||x||^2 + ||mu||^2,
 * the split moves a distance by at most 2^-18 (4e-6), and the fp32
 * accumulation of the d-term dot product and of ||mu||^2 by at most about
 * 2 d 2^-24 (1.5e-5 at d = 128): below 2e-5 together.  An assignment decided
 * by a margin below 3e-5 of that scale may therefore differ from an exact
 * computation (the bound is deliberately loose).
 * ------------------------------------------------------------------------- */
/* Scratch for isa_cluster / isa_cluster_assign / isa_cluster_update: the
 * centroids' bf16 hi / lo parts and squared norms (C rounded up to 64).
 * 0 for an invalid shape. */
ISA_API size_t isa_cluster_workspace_bytes(const isa_shape* shape, int32_t n_clusters);

/* The whole clustering.  1 <= n_clusters <= min(N, 8192), 1 <= n_iters <=
 * 1000.  centroids: [B,H,C,d] fp32 (written).  labels, perm: [B,H,N] int32
 * (written).  offsets: [B,H,C+1] int32 (written).  groups: optional
 * [B,H,C+1] int32, the offsets of the non-empty clusters only, and
 * n_groups: [B,H] int32 their count (both NULL, or both given).  workspace:
 * isa_cluster_workspace_bytes bytes, 16-byte aligned. */
ISA_API isa_status isa_cluster(isa_context* ctx, const isa_shape* shape, const void* x, int32_t n_clusters,
                       int32_t n_iters, float* centroids, int32_t* labels, int32_t* perm,
                       int32_t* offsets, int32_t* groups, int32_t* n_groups, void* workspace,
                       size_t workspace_bytes, void* stream);

/* One assignment round against given centroids ([B,H,C,d] fp32, read). */
ISA_API isa_status isa_cluster_assign(isa_context* ctx, const isa_shape* shape, const void* x,
                              const float* centroids, int32_t n_clusters, int32_t* labels,
                              void* workspace, size_t workspace_bytes, void* stream);

/* The stable counting sort of given labels ([B,H,N] int32 in [0, C); a
 * label outside it is skipped and sets ISA_ERR_DEVICE_CHECK). */
ISA_API isa_status isa_cluster_sort(isa_context* ctx, const isa_shape* shape, const int32_t* labels,
                            int32_t n_clusters, int32_t* perm, int32_t* offsets, int32_t* groups,
                            int32_t* n_groups, void* stream);

/* The mean update from a sorted layout (perm, offsets as isa_cluster_sort
 * writes them); centroids are read (the empty clusters' rows) and written. */
ISA_API isa_status isa_cluster_update(isa_context* ctx, const isa_shape* shape, const void* x,
                              const int32_t* perm, const int32_t* offsets, int32_t n_clusters,
                              float* centroids, void* workspace, size_t workspace_bytes,
                              void* stream);

/* Rows of d bf16 values, per (batch, head): out[i] = x[perm[i]] (inverse =
 * 0, gather) or out[perm[i]] = x[i] (inverse = 1, scatter).  x, out:
 * [B,H,N,d], distinct buffers, 16-byte aligned; perm: [B,H,N], a
 * permutation of 0..N-1 (an index outside it is skipped and sets
 * ISA_ERR_DEVICE_CHECK). */
ISA_API isa_status isa_permute_rows(isa_context* ctx, const isa_shape* shape, const void* x,
                            const int32_t* perm, int32_t inverse, void* out, void* stream);

/* ---------------------------------------------------------------------------
 * isa_attention -- one sparse flash-attention pass over a plan
 * ("AB-Attention": the weights become shifts of the sampled blocks' scores
 * before the softmax, and only selected blocks receive exact attention; small
 * key/value blocks are gathered into full tensor-core tiles).  For every
 * query row r of group g:
 *   z_k = scale * q_r . k_k + log_w[g][s]  for every valid row k of every
 *         plan block idx[g][s], s < n_sel;
 *   out_r = sum_k e^{z_k} v_k / sum_k e^{z_k};  lse_r = ln sum_k e^{z_k}.
 * q, k, v: [B,H,N,d] bf16.  idx, log_w: [B,H,G,n_sel] (n_sel >= 1; a plan may
 * be reused across calls).  out: [B,H,N,d] bf16 (written; every row of N is
 * written exactly once).  lse: optional [B,H,N] fp32 (NULL to skip).
 * workspace: device scratch of isa_attention_workspace_bytes(shape) bytes
 * (0 when q_offsets == NULL; then workspace may be NULL).
 * An idx entry outside [0, nK) is replaced by an empty block and sets
 * ISA_ERR_DEVICE_CHECK.  All device pointers must be 16-byte aligned.
 * ------------------------------------------------------------------------- */
ISA_API size_t isa_attention_workspace_bytes(const isa_shape* shape);
ISA_API isa_status isa_attention(isa_context* ctx, const isa_shape* shape, const void* q, const void* k,
                         const void* v, const int32_t* idx, const float* log_w, int32_t n_sel,
                         void* out, float* lse, void* workspace, size_t workspace_bytes,
                         void* stream);

/* ---------------------------------------------------------------------------
 * isa_tail_merge -- tail merging for the permuted layout ("iCATS: Fast Video
 * Generation via Interaction-Aware Sparse Attention and Timestep-Adaptive
 * Sparsity", AI summary, "Approach": the tail blocks of query clusters are
 * merged with Hamming-nearest compatible clusters, to cut the padding of their
 * last tiles).  shape->q_offsets must be set.  From the plan idx, log_w
 * ([B,H,G,n_sel], the blocks of a row distinct, as isa_select writes them) it
 * builds per (b, h) the schedule isa_attention_merged runs:
 *   - the tail of cluster g is its last t = n_g mod 128 rows (none when 0); it
 *     takes a slot of ceil(t / 32) * 32 rows of a 128-row tile (whole
 *     quarters: each softmax warp's 32 rows share one plan);
 *   - tails are taken by decreasing t (ties: lower g).  A tail joins an open
 *     tile when its slot fits, the tile has fewer than 4 members, and the
 *     union U of the members' plans with the tail's plan P added needs fewer
 *     KV tiles of 128 / k_block blocks than U and P apart; of those tiles it
 *     joins the one whose U is nearest to P in Hamming distance (ties: the
 *     tile opened first); otherwise it opens a tile;
 *   - a merged tile runs the blocks of U in ascending order, and every row
 *     keeps its own cluster's plan and log-weights (a block outside it is
 *     masked for that row), so each output row equals isa_attention's up to
 *     rounding.
 * schedule: device buffer of isa_tail_merge_workspace_bytes(shape, n_sel)
 * bytes, 256-byte aligned, owned by the caller.  It holds the schedule until
 * it is overwritten: a plan reused across calls reuses its schedule.  An idx
 * entry outside [0, nK) sets ISA_ERR_DEVICE_CHECK.
 * ------------------------------------------------------------------------- */
ISA_API size_t isa_tail_merge_workspace_bytes(const isa_shape* shape, int32_t n_sel);
ISA_API isa_status isa_tail_merge(isa_context* ctx, const isa_shape* shape, const int32_t* idx, const float* log_w,
                                  int32_t n_sel, void* schedule, size_t schedule_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * isa_attention_merged -- isa_attention over the schedule isa_tail_merge
 * built from the same plan and shape: the full 128-row tiles of every cluster
 * on the cluster's plan, then the tail tiles, a merged one on the union of its
 * members' plans with per-row log-weights.  q, k, v, idx, log_w, n_sel, out and
 * lse as in isa_attention (every row of N written once); schedule read only.
 * ------------------------------------------------------------------------- */
ISA_API isa_status isa_attention_merged(isa_context* ctx, const isa_shape* shape, const void* q, const void* k,
                                        const void* v, const int32_t* idx, const float* log_w, int32_t n_sel,
                                        const void* schedule, size_t schedule_bytes, void* out, float* lse,
                                        void* stream);

/* ---------------------------------------------------------------------------
 * isa_dense_attention -- the 100%-density limit: softmax(scale Q K^T) V over
 * all keys ("AB-Attention", problem statement: full attention weighs every
 * query against every key, which the sparse pass estimates; with every block
 * in the exact set the sparse pass reduces to this).  The same tensor-core
 * kernel runs with the whole sequence as plan and zero log-weights.  Groups
 * are ignored.  q, k, v, out as in isa_attention; lse optional.
 * ------------------------------------------------------------------------- */
ISA_API isa_status isa_dense_attention(isa_context* ctx, const isa_shape* shape, const void* q,
                               const void* k, const void* v, void* out, float* lse, void* stream);

/* ---------------------------------------------------------------------------
 * isa_plan -- score -> select in one call: the plan of every query group
 * straight from q and k ("AB-Attention": the selector's estimates feed the
 * sampler directly; plans are made from the current activations and may then
 * serve several attention calls).  The result equals isa_select(isa_score(.))
 * bit for bit, but the estimated mass never reaches HBM: the layer is
 * scored and selected in chunks of heads whose mass (at most 88 MiB, at
 * least one head) stays in L2 between the two steps, and the selector drops
 * every mass line it has read from L2 without writing it back.  The
 * workspace (isa_plan_workspace_bytes, 256-byte aligned) holds one chunk's
 * scorer scratch and mass, so it is also much smaller than the whole mass
 * tensor.  idx, log_w: [B,H,G,S] as isa_select writes them.
 * ------------------------------------------------------------------------- */
ISA_API size_t isa_plan_workspace_bytes(const isa_shape* shape, const isa_params* params);
ISA_API isa_status isa_plan(isa_context* ctx, const isa_shape* shape, const isa_params* params,
                    const void* q, const void* k, int32_t* idx, float* log_w, void* workspace,
                    size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * isa_pipeline -- score -> select -> attention in one call on device
 * buffers (the whole hot path of one attention layer).  The mass tensor,
 * the plan and the scorer's scratch are carved from `workspace`
 * (isa_pipeline_workspace_bytes bytes).  plan_idx / plan_log_w: optional
 * device outputs [B,H,G,S] receiving the plan (NULL: kept in the workspace).
 * ------------------------------------------------------------------------- */
ISA_API size_t isa_pipeline_workspace_bytes(const isa_shape* shape, const isa_params* params);
ISA_API isa_status isa_pipeline(isa_context* ctx, const isa_shape* shape, const isa_params* params,
                        const void* q, const void* k, const void* v, void* out, float* lse,
                        int32_t* plan_idx, float* plan_log_w, void* workspace,
                        size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * isa_pipeline_host -- the same from HOST buffers: copies q, k, v (host,
 * [B,H,N,d] bf16; page-locked memory makes the copies asynchronous) into the
 * device arena, runs the pipeline, and copies the output back to out_host
 * ([B,H,N,d] bf16).  The arena holds Q, K, V, O and the pipeline workspace:
 * isa_pipeline_host_workspace_bytes bytes.  shape->q_offsets stays a device
 * pointer.  The layer runs in chunks of heads (up to 16 per batch entry) so
 * that the copies overlap the compute: the inputs go up and the outputs come
 * down on two copy streams the context owns, the compute runs on `stream`,
 * and events order them.  The result equals isa_pipeline on the whole layer
 * (the selector's uniform is keyed by the global head and batch index).
 * Returns after enqueueing; `stream` completes only after the last output
 * copy, so out_host is valid once `stream` is synchronised.  Work already on
 * `stream` is finished before the arena is overwritten.  Calls that share a
 * context share its copy streams.  Unlike the other calls this one creates
 * CUDA objects: its first call on a context creates the two copy streams
 * (kept until isa_destroy), and every call creates and releases a few
 * events.  It is therefore not meant for stream capture into a CUDA graph.
 * ------------------------------------------------------------------------- */
ISA_API size_t isa_pipeline_host_workspace_bytes(const isa_shape* shape, const isa_params* params);
ISA_API isa_status isa_pipeline_host(isa_context* ctx, const isa_shape* shape, const isa_params* params,
                             const void* q_host, const void* k_host, const void* v_host,
                             void* out_host, void* workspace, size_t workspace_bytes,
                             void* stream);

/* ---------------------------------------------------------------------------
 * isa_debug_set -- test hooks for failure detection (not for production use).
 *   ISA_DEBUG_WAIT_TIMEOUT_NS: per-wait time limit, in ns, of every bounded
 *     pipeline wait in kernels launched on this context (default 2e9; 0
 *     restores the default).
 *   ISA_DEBUG_STALL_ATTENTION: when non-zero, attention launches on this
 *     context make their MMA warp wait on a barrier that nothing arrives at;
 *     the wait runs out after the per-wait limit, every CTA takes its abort
 *     path (drains in-flight copies, frees tensor memory) and the status word
 *     reads ISA_ERR_TIMEOUT.  The outputs of such a launch are undefined.
 * Returns ISA_ERR_INVALID_ARG for an unknown knob.
 * ------------------------------------------------------------------------- */
enum { ISA_DEBUG_WAIT_TIMEOUT_NS = 1, ISA_DEBUG_STALL_ATTENTION = 2 };
ISA_API isa_status isa_debug_set(isa_context* ctx, int32_t knob, uint64_t value);

/* ---------------------------------------------------------------------------
 * isa_attention_noalloc -- isa_attention for callers that cannot allocate.
 * No counterpart in the pages: it is an interface convenience of this library.
 * Some callers cannot give the library device memory: a framework custom-op
 * or plugin interface that hands a kernel only its inputs and outputs, or
 * latency-critical code that must not call cudaMalloc (which may synchronise
 * the device).  This call computes exactly what isa_attention computes, with
 * the same arguments minus the workspace; the tile list that variable
 * clusters and groups of more than 128 rows need lives in a 1 MiB array
 * inside the library, so num_groups + seq_len / 128 must stay below 65535
 * (larger shapes return ISA_ERR_INVALID_ARG).  Every GPU that loads the
 * library holds that 1 MiB until the process exits.  The first call on each
 * device looks up the array's device address (make that first call before
 * any stream capture) and keeps it for the life of the process; a device
 * reset (cudaDeviceReset, or a reset of the primary context) may move the
 * array, so do not call this entry point after one.  All calls share the one
 * array: calls whose kernels overlap on the GPU race on it, so order them
 * (one stream, or events).  The call allocates nothing.
 * ------------------------------------------------------------------------- */
ISA_API isa_status isa_attention_noalloc(isa_context* ctx, const isa_shape* shape, const void* q,
                                         const void* k, const void* v, const int32_t* idx,
                                         const float* log_w, int32_t n_sel, void* out, float* lse,
                                         void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ISA_H_ */
