/*
 * libssa: forward pass of one content-routed block-sparse attention (SSA)
 * layer on NVIDIA B200 (sm_100a).
 *
 * The layer, as stated on "Subquadratic Sparse Attention (SSA)" (opening
 * section and "The idea in one screen"):
 *   (i)   summarise every block of B consecutive keys by its mean mu_c and
 *         covariance Sigma_c (full, or its diagonal sigma_c^2), and route each
 *         query with the second-cumulant score
 *             r_c(q) = <q, mu_c> + (beta/2) q^T Sigma_c q ,
 *         keeping a fixed budget of the top-k blocks;
 *   (ii)  add a causal local window of W keys;
 *   (iii) compute exact softmax attention over the selected keys.
 *
 * Conventions shared by every call
 * --------------------------------
 *  * All tensors are dense, row-major, caller-owned DEVICE buffers unless a
 *    call says otherwise, and must be 16-byte aligned.  No call allocates
 *    memory and none keeps per-call state; scratch comes from the caller's
 *    workspace.  The library's own device footprint is fixed: a 4-byte
 *    failure word and the 16 MiB scratch array of ssa_route_topk_static
 *    (below), both module globals that exist on a device once the module
 *    holding them is loaded there.
 *  * Per device the library caches the addresses of those globals and the
 *    SM count the first time a call runs on it.  A cudaDeviceReset destroys
 *    the globals, so the library must not be used on a device after it has
 *    been reset in the same process.
 *  * Layouts (b = batch, nb = n_kv / block, G = h_q / h_kv):
 *      Q, O        [b, n_q,  h_q,  d]   elements of `dtype`
 *      K, V        [b, n_kv, h_kv, d]   elements of `dtype`
 *      mu          [b, h_kv, nb, d]     float32
 *      sigma       [b, h_kv, nb, d]     float32   (SSA_SIGMA_DIAG: sigma_c^2)
 *                  [b, h_kv, nb, d, d]  float32   (SSA_SIGMA_FULL: Sigma_c)
 *      route_table [b, h_kv, nb, 2d]    bfloat16  row c = [mu_c ; sigma_c^2]
 *                                       (bf16 problems only)
 *      block_idx   [b, n_q, h_kv, topk] int32, ascending, padded with -1
 *      top_scores  [b, n_q, h_kv, topk] float32 score of each block_idx entry
 *      lse         [b, n_q, h_q]        float32, log sum_j exp(scale q.k_j)
 *  * Query row i sits at key position pos = q_offset + i (prefill: 0;
 *    one decode token: n_kv - 1).  Block c is a routing candidate only when
 *    fully visible, (c+1)*block - 1 <= pos.  The window is the keys
 *    pos-W+1 .. pos.  The attended set is the union of the selected blocks'
 *    keys and the window keys.  Ties in the routing score go to the lower
 *    block index.  With grouped-query attention the G query heads of a
 *    kv-head share one selection, ranked by the sum of their scores.
 *  * bf16 problems route on bf16 features f = [bf16(sum_h q_h),
 *    bf16((beta/2) sum_h q_h*q_h)] (float32 sums in head order) against the
 *    bf16 route table; float32 problems route in float32 on mu / sigma.
 *  * Every call validates its arguments before launching anything and
 *    returns SSA_ERR_INVALID_ARG / SSA_ERR_UNSUPPORTED / SSA_ERR_WORKSPACE
 *    without side effects.  Work is enqueued asynchronously on `stream`
 *    (a cudaStream_t; NULL = legacy default stream).  A failed launch returns
 *    SSA_ERR_CUDA.  A kernel whose internal wait exceeds its time limit stops
 *    early and records a code read by ssa_device_error().  No C++ exception
 *    crosses this interface.  Calls are reentrant.
 *  * Supported: d in {64, 128}; block in {64, 128}; G in {1, 2, 4, 8};
 *    1 <= topk <= 32; 1 <= window <= 4032; n_kv % block == 0;
 *    0 <= q_offset and q_offset + n_q <= n_kv; bf16 requires SSA_SIGMA_DIAG.
 *    batch == 0 or n_q == 0 is a valid empty problem (nothing is launched).
 */
#ifndef SSA_H_
#define SSA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SSA_API __attribute__((visibility("default")))
#else
#define SSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SSA_OK = 0,
  SSA_ERR_INVALID_ARG = 1,   /* null / misaligned pointer, inconsistent shape  */
  SSA_ERR_UNSUPPORTED = 2,   /* valid problem outside the supported set         */
  SSA_ERR_WORKSPACE = 3,     /* workspace pointer or size too small             */
  SSA_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed     */
  SSA_ERR_DEVICE = 5         /* a kernel recorded a device-side failure          */
} ssa_status;

typedef enum { SSA_F32 = 0, SSA_BF16 = 1 } ssa_dtype;
typedef enum { SSA_SIGMA_DIAG = 0, SSA_SIGMA_FULL = 1 } ssa_sigma;

/* Routing kernel choice for bf16 problems (ssa_params.route_impl). */
typedef enum {
  SSA_ROUTE_AUTO = 0,   /* tensor-core tiles when n_q >= 128, else per row    */
  SSA_ROUTE_TILED = 1,  /* tcgen05 128-row tiles with fused streaming top-k    */
  SSA_ROUTE_ROWWISE = 2 /* one CTA per query row (decode-shaped work)          */
} ssa_route_impl;

/* 72 bytes, no padding: twelve int32, one int64, two float32, two int32. */
typedef struct {
  int32_t batch;      /* b                                               */
  int32_t n_q;        /* query rows per sequence                         */
  int32_t n_kv;       /* keys per sequence (multiple of block)           */
  int32_t h_q;        /* query heads                                     */
  int32_t h_kv;       /* key/value heads (h_q % h_kv == 0)               */
  int32_t d;          /* head dimension                                  */
  int32_t block;      /* B, keys per routing block                       */
  int32_t topk;       /* k, routed blocks per (query row, kv-head)       */
  int32_t window;     /* W, causal local window in keys                  */
  int32_t dtype;      /* ssa_dtype of Q, K, V, O                          */
  int32_t sigma;      /* ssa_sigma                                        */
  int32_t route_impl; /* ssa_route_impl                                   */
  int64_t q_offset;   /* key position of query row 0                      */
  float beta;         /* routing inverse temperature                      */
  float scale;        /* attention logit scale (normally 1/sqrt(d))        */
  int32_t subblocks;  /* S in {1, 2, 4}: summaries per block (see below)  */
  int32_t outlier;    /* 1: outlier-channel row per block (see below); 0  */
} ssa_params;

/*
 * Sub-block summaries (subblocks = S > 1): every block of B keys is
 * summarised as S sub-blocks of B/S consecutive keys (B/S >= 32), and a
 * block's routing score is the largest of its sub-blocks' scores, each the
 * second-cumulant score of those keys (summed over the kv-head's query
 * heads).  The finer summaries keep a single strongly matching key from
 * being averaged away over the whole block — the sub-block part of the
 * selector named "Certified Causal Cascade" ("Subquadratic Sparse Attention
 * (SSA)", artifact list: sub-block max-pool).  Selection, the window and the
 * attention still work on whole blocks.  Summary outputs then have nb * S
 * rows per (batch, kv-head), sub-block s of block c at row c * S + s.
 *
 * Outlier channel (outlier = 1, with subblocks = 1): the same page names an
 * outlier channel beside the sub-block max-pool, without a rule.  Here every
 * block gets a second summary row: its key of largest 2-norm k*_c (squared
 * norms in float64, equal norms to the earlier key) with a zero covariance,
 * so the row's score is the exact group logit sum_h <q_h, k*_c>; a block
 * scores the larger of its two rows.  Summary outputs then have 2 nb rows
 * per (batch, kv-head): row 2c the block's (mu, Sigma), row 2c + 1 the
 * outlier key (sigma rows zero; route_table row [k*_c ; 0]).  outlier = 1
 * with subblocks > 1 is SSA_ERR_UNSUPPORTED; any value other than 0 or 1 is
 * SSA_ERR_INVALID_ARG.
 */

/* Human-readable name of a status code (static string, never NULL). */
SSA_API const char* ssa_status_string(int32_t status);

/* Library ABI version (major*1000 + minor). */
SSA_API int32_t ssa_version(void);

/* Number of kernels this process has launched through libssa so far. */
SSA_API uint64_t ssa_launch_count(void);

/*
 * Reads and clears the device-side failure word of the current device
 * (synchronises the device).  *code is 0 when no kernel recorded a failure,
 * else an identifier of the wait that timed out.  Returns SSA_ERR_DEVICE when
 * *code != 0.
 */
SSA_API ssa_status ssa_device_error(uint32_t* code);

/*
 * Step (i), summaries: "routes ... using only per-block summary statistics"
 * [Subquadratic Sparse Attention (SSA), opening section] with
 * mu_c = (1/B) sum_{j in c} k_j and the population covariance
 * Sigma_c = (1/B) sum_{j in c} (k_j - mu_c)(k_j - mu_c)^T (or its diagonal).
 * Sums are accumulated in float64; mu / sigma are the float32 roundings and
 * route_table holds their bfloat16 roundings.
 *   K            device, [b, n_kv, h_kv, d] of dtype (read)
 *   mu, sigma    device float32 outputs, may each be NULL (not written)
 *   route_table  device bf16 output [b, h_kv, nb, 2d]; bf16 problems only,
 *                may be NULL; must be NULL for float32 problems
 */
SSA_API ssa_status ssa_block_summary(const ssa_params* p, const void* K, float* mu, float* sigma,
                             void* route_table, void* stream);

/* Bytes of device workspace ssa_route_topk needs (0 when none). */
SSA_API size_t ssa_route_workspace_size(const ssa_params* p);

/*
 * Step (i), routing and selection: r_c(q) = <q, mu_c> + (beta/2) q^T Sigma_c q
 * ["The idea in one screen", routing-score equation] for every fully visible
 * block, then the top-k blocks under (higher score, lower index) with a fixed
 * budget k ["fixed budget kappa << n", opening section].  The score matrix is
 * never written to memory: selection runs in the scoring kernel's epilogue.
 *   Q            device [b, n_q, h_q, d] of dtype
 *   mu, sigma    device float32 summaries (float32 problems; else ignored)
 *   route_table  device bf16 table (bf16 problems; else ignored)
 *   block_idx    device int32 output
 *   top_scores   device float32 output, may be NULL
 *   ws, ws_bytes device workspace of at least ssa_route_workspace_size(p)
 */
SSA_API ssa_status ssa_route_topk(const ssa_params* p, const void* Q, const float* mu,
                          const float* sigma, const void* route_table, int32_t* block_idx,
                          float* top_scores, void* ws, size_t ws_bytes, void* stream);

/* Bytes of device workspace that lets ssa_sparse_attn run block-major (0 when
 * the problem always runs the per-query gather). */
SSA_API size_t ssa_attn_workspace_size(const ssa_params* p);

/*
 * Steps (ii)+(iii): exact softmax attention of every query head over the
 * union of its kv-head's selected blocks and the causal window
 * [opening section, (ii) and (iii)].  block_idx entries that are not -1 are
 * used when they are fully visible and larger than every earlier in-range
 * entry of their row (ascending, distinct); any other entry is skipped and,
 * when bad_index_count is not NULL, counted into that device int32
 * (atomically added, not reset).
 * Two evaluations give the same result up to rounding.  With a workspace
 * of ssa_attn_workspace_size(p) bytes (bf16 problems with n_q >= 1024,
 * d = 128, G in {1, 2, 4, 8}, topk * G <= 128, at most 32 key blocks per
 * window and 16384 key blocks) the evaluation is block-major: every
 * (query, kv-head) row is split into slots — its used selected blocks of
 * the (batch, kv-head)'s hot set (its at most 128 most selected blocks)
 * taken two at a time in block order, one slot per pair; every other used
 * block a slot of its own; and the chunks of the window outside them — the
 * slots are inverted into per-key lists, each block or pair of blocks is
 * multiplied once against all its slots' queries on the tensor cores, the
 * window chunks run as dense sliding-window tiles, and the slot partials are
 * merged per row.  With ws NULL (or too small) every (query, kv-head)
 * gathers its own keys.
 *   O            device output [b, n_q, h_q, d] of dtype
 *   lse          device float32 output, may be NULL
 *   ws, ws_bytes device workspace, may be NULL / 0
 */
SSA_API ssa_status ssa_sparse_attn(const ssa_params* p, const void* Q, const void* K, const void* V,
                                   const int32_t* block_idx, void* O, float* lse,
                                   int32_t* bad_index_count, void* ws, size_t ws_bytes, void* stream);

/*
 * The block-major evaluation of ssa_sparse_attn as four calls, for callers
 * that schedule or time the stages themselves.  Made in this order on one
 * stream with one workspace (ssa_attn_workspace_size(p) bytes, 16-byte
 * aligned; its contents are private to the library and live from the plan
 * call to the merge call), they give exactly the bytes ssa_sparse_attn gives
 * with that workspace.  A row's keys fall in "slots": each pair of used
 * selected hot blocks (or used selected block outside the pairs), and each
 * 256-key chunk of the window (pos-W+1 .. pos; 128 keys when G = 1) minus
 * the keys of its used selected blocks.
 *   ssa_attn_plan    inverts block_idx: the selected slots of every row as
 *                    per-(batch, kv-head, block or pair) lists, in tiles of
 *                    128 / G queries, and each row's window blocks that no
 *                    used entry selects;
 *   ssa_attn_blocks  per tile, S = Q_tile K^T and O = P V over the block's
 *                    or pair's keys on the tensor cores; writes each selected
 *                    slot's normalised partial output and base-2 log-sum-exp
 *                    into the workspace;
 *   ssa_attn_window  per run of 128 / G consecutive queries and window
 *                    chunk, the same over the chunk's keys (dense tensor-core
 *                    tiles masked per row); writes the window slots' partials;
 *   ssa_attn_merge   per (query, kv-head): the softmax merge of the row's
 *                    slot partials into O and lse; counts skipped block_idx
 *                    entries as ssa_sparse_attn does.  It reads each row's
 *                    slots as the plan call recorded them, so block_idx
 *                    must be the array that call was given.
 * ssa_attn_blocks and ssa_attn_window write disjoint parts of the workspace
 * and may run in either order (or on two streams ordered after the plan and
 * before the merge).
 * Problems that do not qualify return SSA_ERR_UNSUPPORTED, a missing or
 * short workspace SSA_ERR_WORKSPACE; both before any launch.
 */
SSA_API ssa_status ssa_attn_plan(const ssa_params* p, const int32_t* block_idx, void* ws, size_t ws_bytes,
                                 void* stream);
SSA_API ssa_status ssa_attn_blocks(const ssa_params* p, const void* Q, const void* K, const void* V,
                                   void* ws, size_t ws_bytes, void* stream);
SSA_API ssa_status ssa_attn_window(const ssa_params* p, const void* Q, const void* K, const void* V,
                                   void* ws, size_t ws_bytes, void* stream);
SSA_API ssa_status ssa_attn_merge(const ssa_params* p, const int32_t* block_idx, void* O, float* lse,
                                  int32_t* bad_index_count, const void* ws, size_t ws_bytes, void* stream);

/*
 * ssa_route_topk without a caller workspace.  No counterpart in the paper:
 * this is an interface convenience for callers that cannot allocate device
 * memory when they route (a host framework whose allocator owns the whole
 * device pool, or a loop that cannot afford cudaMalloc's implicit device
 * synchronisation).  The routing-feature scratch lives in a fixed array of
 * SSA_ROUTE_STATIC_SCRATCH_BYTES inside the library.  The array occupies
 * device memory on every device where the module that holds it has been
 * loaded, until the process exits: with CUDA's lazy module loading (the
 * default) that is the first call of this function on the device, with
 * eager loading (CUDA_MODULE_LOADING=EAGER) the first CUDA call of the
 * process.  Problems that need more than the array return
 * SSA_ERR_WORKSPACE before any launch: the routing features take
 * batch * h_kv * n_q * 2d bf16 values (rounded up to 256 bytes), so at
 * d = 128 at most 32768 (query row, kv-head) pairs fit.  The first call on
 * a device looks up the array's address with that device current; make it
 * before any stream capture.  All calls share the array, so calls whose kernels overlap on the
 * GPU race on it and must be serialised.  Arguments and results are those of
 * ssa_route_topk.  Allocates nothing.
 */
#define SSA_ROUTE_STATIC_SCRATCH_BYTES (16u << 20)
SSA_API ssa_status ssa_route_topk_static(const ssa_params* p, const void* Q, const float* mu,
                                         const float* sigma, const void* route_table,
                                         int32_t* block_idx, float* top_scores, void* stream);

/* Bytes of device workspace ssa_forward needs. */
SSA_API size_t ssa_workspace_size(const ssa_params* p);

/*
 * The whole layer: ssa_block_summary, ssa_route_topk and ssa_sparse_attn on
 * `stream`, with the summaries, routing features, block indices and the
 * attention workspace carved from the caller's workspace (at least
 * ssa_workspace_size(p) bytes).
 */
SSA_API ssa_status ssa_forward(const ssa_params* p, const void* Q, const void* K, const void* V,
                       void* O, float* lse, void* ws, size_t ws_bytes, void* stream);

/* Bytes of device buffer ssa_forward_hostio needs. */
SSA_API size_t ssa_hostio_buffer_size(const ssa_params* p);

/*
 * ssa_forward on HOST inputs and outputs: copies hQ, hK, hV into dev_buf,
 * runs the layer and copies O (and lse when hlse is not NULL) back, all
 * enqueued on `stream`; the caller synchronises.  Host buffers should be
 * page-locked for the copies to be asynchronous.  dev_buf must hold
 * ssa_hostio_buffer_size(p) bytes of device memory.
 */
SSA_API ssa_status ssa_forward_hostio(const ssa_params* p, const void* hQ, const void* hK,
                              const void* hV, void* hO, float* hlse, void* dev_buf,
                              size_t dev_bytes, void* stream);

/*
 * Hierarchical routing with per-row certificates.  "Subquadratic Sparse
 * Attention (SSA)" names a tree router with a recursive radius (artifact
 * list, Barnes-Hut style), exact branch-and-bound selection under an
 * admissible bound (same list) and sound per-query certificates with
 * escalation ("Certified Causal Cascade" entry); it does not fix their rules.
 * The rules here:
 *
 *   node N = the M consecutive blocks N*M .. N*M+M-1 (nn = nb / M complete
 *   nodes per (batch, kv-head); trailing blocks form no node).  From the
 *   blocks' bf16 routing rows T_c = [mu_c ; s_c]:
 *     centre m_N = bf16(f32(mean of mu_c)), cap v_N = max of s_c (per dim),
 *     radius R_N = max_c ||mu_c - m_N||_2 (float64, rounded up to float32).
 *   For routing features f = [f_s ; f_q] (f_q >= 0) every block c of N has
 *     f . T_c <= f . [m_N ; v_N] + ||f_s|| R_N.
 *
 *   A query row ranks its complete visible nodes by w_N = f . [m_N ; v_N]
 *   (higher first, then lower index), scores exactly the blocks of its best
 *   `probe` nodes and every visible block outside a complete visible node,
 *   and keeps the top-k of those.  The row is certified when no complete
 *   visible node is left unexpanded, or when its k-th kept score exceeds
 *   w_(probe+1) + ||f_s|| R* + 2^-12 ||f|| T*, where R* is the largest node
 *   radius and T* the largest 2-norm of any block or node row of its
 *   (batch, kv-head) (the last term absorbs float32 rounding).  A certified
 *   row's kept set is the top-k of all its visible blocks, as
 *   ssa_route_topk selects it (up to the order of near-equal scores).
 *   With escalate = 1 every uncertified row is routed again over all its
 *   visible blocks (by ssa_route_topk's kernels), so block_idx is
 *   ssa_route_topk's selection for every row.
 *
 *   levels = 2 adds a tree level: super-node S = nodes S*M .. S*M+M-1
 *   (complete super-nodes only) with centre bf16(f32(mean of m_N)), cap the
 *   per-dimension max of v_N and the recursive radius
 *   R_S = max_N (||m_N - m_S||_2 + R_N) (float64, rounded up to float32),
 *   so every block of S has f . T_c <= f . [m_S ; v_S] + ||f_s|| R_S.  A row
 *   ranks its complete visible super-nodes, scores exactly the nodes of its
 *   best `probe` and the complete visible nodes outside complete super-
 *   nodes, and probes the best `probe` of those nodes as above; certified
 *   when the k-th kept score also exceeds the best unexpanded super-node's
 *   w_S + ||f_s|| R2* + 2^-12 ||f|| T* (R2*: largest super-node radius;
 *   T* then also covers the super-node rows), or no complete visible
 *   super-node is left unexpanded.
 *
 * bf16 problems with a diagonal Sigma, subblocks = 1, outlier = 0 and d in {64, 128}
 * (else SSA_ERR_UNSUPPORTED).
 */
typedef struct {
  int32_t fanout;    /* M, blocks per node: a power of two, 1..64                 */
  int32_t probe;     /* nodes expanded per row before the certificate, 1..31      */
  int32_t escalate;  /* 1: uncertified rows are re-routed over all blocks; or 0   */
  int32_t levels;    /* tree levels: 2, or 1 (0 reads as 1)                       */
} ssa_hier_params;

/*
 * Errors of the hierarchical calls, checked before any launch: the
 * ssa_params checks of the other calls; hp NULL, levels outside 0..2, fanout not a
 * power of two in 1..64, probe outside 1..31 or escalate not 0/1 ->
 * SSA_ERR_INVALID_ARG; (probe + 1) * fanout > 512 (the probe's candidate
 * capacity), a float32 problem, subblocks != 1 or outlier != 0 -> SSA_ERR_UNSUPPORTED;
 * NULL or misaligned (not 16-byte) pointers -> SSA_ERR_INVALID_ARG; a
 * workspace smaller than ssa_route_hier_workspace_size ->
 * SSA_ERR_WORKSPACE.  ssa_route_hier returns SSA_OK without a launch when
 * batch or n_q is 0, ssa_hier_nodes when batch is 0.  The size calls return
 * 0 on any of these errors.
 */

/*
 * Bytes of the node store of (p, hp): the node rows (bf16 [b, h_kv, nn, 2d],
 * at offset 0), the radii (float32 [b, h_kv, nn], at offset
 * round_up(node row bytes, 256)) and two floats per (batch, kv-head) (largest
 * radius, largest row norm; after the radii, also 256-byte aligned); with
 * levels = 2 then the super-node rows (bf16 [b, h_kv, nn / M, 2d]), their
 * radii and one float per (batch, kv-head) (largest super-node radius), each
 * part 256-byte aligned.  0 on invalid arguments.
 */
SSA_API size_t ssa_hier_nodes_size(const ssa_params* p, const ssa_hier_params* hp);

/*
 * Builds the node store from a bf16 routing table (ssa_block_summary's
 * route_table output, device [b, h_kv, nb, 2d]) into the device buffer
 * `nodes` of ssa_hier_nodes_size bytes (16-byte aligned, caller-owned).
 */
SSA_API ssa_status ssa_hier_nodes(const ssa_params* p, const ssa_hier_params* hp, const void* route_table,
                                  void* nodes, void* stream);

/* Bytes of device workspace ssa_route_hier needs. */
SSA_API size_t ssa_route_hier_workspace_size(const ssa_params* p, const ssa_hier_params* hp);

/*
 * Routes every query row through the node store (see above).
 *   Q            device [b, n_q, h_q, d] bf16
 *   route_table  device bf16 [b, h_kv, nb, 2d] (the table the nodes were built from)
 *   nodes        device node store from ssa_hier_nodes
 *   block_idx    device int32 output [b, n_q, h_kv, k], ascending, -1 padded
 *   certified    device uint8 output [b, n_q, h_kv]: 1 certified, 0 not
 *                (rows re-routed by escalation stay 0); may be NULL
 *   ws, ws_bytes device workspace of at least ssa_route_hier_workspace_size
 */
SSA_API ssa_status ssa_route_hier(const ssa_params* p, const ssa_hier_params* hp, const void* Q,
                                  const void* route_table, const void* nodes, int32_t* block_idx,
                                  uint8_t* certified, void* ws, size_t ws_bytes, void* stream);

/*
 * Self-test of the failure path (not part of the layer).  Launches on
 * `stream` one kernel that waits on an mbarrier nothing arrives at, through
 * the bounded wait every kernel of the library uses: after the wait limit
 * (1 s) it records SSA_SITE_SELFTEST in the device failure word and returns.
 * After synchronising, ssa_device_error reports SSA_ERR_DEVICE with that
 * code (and clears it); the context stays usable.  Returns SSA_OK once the
 * kernel is launched.
 */
#define SSA_SITE_SELFTEST 0x7F1u
SSA_API ssa_status ssa_selftest_wait_timeout(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SSA_H_ */
