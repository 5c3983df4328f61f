/*
 * glga.h -- C ABI of libglga: the forward pass of a gated local-global graph-attention
 * layer over a fixed sparse adjacency, on NVIDIA B200 (sm_100a).
 *
 * What the layer computes (method page "Gated Local-Global Graph Attention", section
 * "Key formulas"; heads of width r as in the tinymesh page "Sparse attention
 * experiment", section "Multiple heads are composition"):
 *
 *   per head h (columns h*r .. h*r+r-1):
 *     q_i = x_i W_Q,  k_j = x_j W_K,  v_j = x_j W_V
 *     L_i = sum over in-neighbours j of i of softmax_j(q_i . k_j / sqrt(r)) v_j
 *     G_i = phi(q_i)^T S / (phi(q_i)^T z + eps),  S = sum_j phi(k_j) v_j^T,
 *           z = sum_j phi(k_j),  phi(x) = elu(x) + 1,  j over all N nodes
 *   g_i = sigmoid(x_i . w_g + b_g),  Y_i = g_i L_i + (1 - g_i) G_i   (heads concatenated)
 *
 * Conventions for every entry point:
 *  - Pointers marked (device) are CUDA device pointers on the current device; pointers
 *    marked (host) are ordinary host memory.  All matrices are dense, row-major and
 *    contiguous.  The caller owns every buffer it passes; the library never frees them.
 *  - `io` is the element type of X, W_Q, W_K, W_V, w_g and Y: GLGA_F32 (float) or
 *    GLGA_BF16 (bfloat16 bits).  Internal accumulation is float32.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *  - No entry point aborts, throws or prints; failures return a glga_status and leave a
 *    one-line reason retrievable with glga_last_error_message() (per calling thread).
 *  - The graph is a target-grouped CSR: row i lists the sources j of the edges j -> i
 *    (A_ij = 1), so a row's entries are i's in-neighbours.  Self-loops are whatever the
 *    CSR holds; the library never adds or removes edges.  A duplicated entry is one more
 *    softmax term.  A row without entries has L_i = 0 (an empty weighted sum).
 */
#ifndef GLGA_H_
#define GLGA_H_

#include <stdint.h>

#if defined(__GNUC__)
#define GLGA_API __attribute__((visibility("default")))
#else
#define GLGA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct glga_ctx glga_ctx;

typedef enum {
    GLGA_OK = 0,
    GLGA_ERR_INVALID_ARG = 1,   /* null pointer, negative size, misaligned buffer       */
    GLGA_ERR_BAD_GRAPH = 2,     /* CSR/COO violates its invariants (see glga_create)    */
    GLGA_ERR_UNSUPPORTED = 3,   /* shape outside the supported set (see glga_create)    */
    GLGA_ERR_OOM = 4,           /* a device allocation failed                           */
    GLGA_ERR_CUDA = 5,          /* a CUDA runtime/driver call failed                    */
    GLGA_ERR_TIMEOUT = 6,       /* a bounded device-side wait gave up (reported late)   */
    GLGA_ERR_DEVICE = 7         /* a device-side check failed (reported late)           */
} glga_status;

typedef enum { GLGA_F32 = 0, GLGA_BF16 = 1 } glga_dtype;

/* Scheduling of target rows by in-degree (deg = row_ptr[i+1] - row_ptr[i]):
 *   deg <= warp_max_degree                 -> bucket 0: warp tasks; each edge slot of a
 *        warp takes one row (rows ordered by descending degree, ties by ascending row,
 *        and packed up to 32 rows / about 256 edges per task)
 *   warp_max_degree < deg <= chunk_edges   -> bucket 1: one thread block per row
 *   deg > chunk_edges                      -> bucket 2: the row is cut into chunks of
 *        chunk_edges edges, one thread block per chunk, chunks merged in order.
 * Buckets 1 and 2 keep rows in ascending order.  Requires
 * 0 <= warp_max_degree <= chunk_edges and chunk_edges >= 1.
 *
 * debug_checks != 0 selects kernel builds that check every column index read from the
 * CSR against [0, N) and every scheduled row; a failed check is skipped (the edge is
 * masked) and reported as GLGA_ERR_DEVICE by glga_last_device_error.  Slower; for
 * debugging only.
 * debug_fail_alloc = n > 0 makes the n-th device allocation of glga_create fail with
 * GLGA_ERR_OOM (a test hook for the clean-up path); 0 disables it.
 * backward != 0 allocates the workspaces of glga_backward at create (a transposed CSR,
 * chunk lists of the rows with more than 64 entries, a second stream and fp32 buffers of
 * about N*(6*H*r + 4*H + 1) floats; for bf16 layers with d a multiple of 8 also the
 * range partials of the tensor-core weight-gradient GEMM, about num_SMs*d*3*H*r floats);
 * glga_forward on such a context also stores each row's softmax log-sum-exp per head for
 * the backward.  Whole-graph, one-segment contexts
 * with at most 32 heads (GLGA_ERR_UNSUPPORTED otherwise).
 * fuse_stats != 0 asks for the global statistics inside the projection GEMM: a
 * one-segment bf16 context with H*r = 128 and r dividing 64 then accumulates
 * phi(K)^T [V | 1] in the GEMM's epilogue (per-CTA partial sums, then the same
 * fixed-order reduction) instead of launching the statistics kernel; other contexts
 * ignore it.  Off by default: on the arxiv-shaped graph the fused GEMM plus reduction
 * take longer than the GEMM and the statistics kernel, and the statistics kernel's pass
 * over K and V also leaves them in L2 for the local kernel that follows.               */
typedef struct {
    int32_t warp_max_degree;
    int32_t chunk_edges;
    int32_t debug_checks;
    int32_t debug_fail_alloc;
    int32_t backward;
    int32_t fuse_stats;
} glga_options;

/* Fills *opts with the defaults used when glga_create gets opts == NULL:
 * warp_max_degree 256, chunk_edges 2048, no debug checks, no backward workspaces.     */
GLGA_API glga_status glga_default_options(glga_options *opts);

/* glga_create -- bind a fixed graph and the layer shape; allocate all workspaces.
 *   N        number of nodes (>= 0, < 2^31)
 *   d        input width (>= 1)
 *   H, r     heads and per-head width; r in {8, 16, 32, 64, 128}, H >= 1, and the row
 *            width D = H*r must satisfy D*sizeof(io) <= 2048 bytes
 *   row_ptr  (device) int32 [N+1], row_ptr[0] = 0, non-decreasing, row_ptr[N] = E
 *   col_idx  (device) int32 [E], every entry in [0, N)
 *   E        number of CSR entries (>= 0, < 2^31)
 *   opts     (host, nullable) bucket thresholds; NULL selects the defaults
 * The CSR is copied into the context and validated on the device (GLGA_ERR_BAD_GRAPH if
 * it violates the invariants above), then bucketed by degree.  This call synchronises
 * `stream` (validation result and bucket sizes are read back).  The caller may free its
 * CSR afterwards.  Workspaces are O(N*(3*H*r + d) + E); nothing is O(N^2) or O(E*r).
 * On success *out owns device memory until glga_destroy.                              */
GLGA_API glga_status glga_create(glga_ctx **out, int64_t N, int32_t d, int32_t H, int32_t r,
                        glga_dtype io, const int32_t *row_ptr, const int32_t *col_idx,
                        int64_t E, const glga_options *opts, void *stream);

/* glga_create_segmented -- as glga_create, for a batch of graphs laid out as contiguous
 * node ranges (segments).  Method page "Gated Local-Global Graph Attention",
 * "Implementation notes" (the layer takes X [batch, N, d]) and "Key formulas" (S and z
 * sum over the nodes of one graph): the global statistics are summed per segment, and
 * row i's readout uses the S, z of its own segment.  The local branch follows the CSR
 * as always (edges may cross segments; a batch of separate graphs has none that do).
 *   seg_ptr  (host) int64 [n_seg + 1]: segment k holds nodes [seg_ptr[k], seg_ptr[k+1]);
 *            seg_ptr[0] = 0, non-decreasing, seg_ptr[n_seg] = N.  Empty segments are
 *            allowed.  Copied; the caller keeps ownership.
 *   n_seg    >= 1; n_seg = 1 with {0, N} is glga_create.
 * GLGA_ERR_INVALID_ARG for a malformed seg_ptr.  The statistics workspace holds one
 * H*r*(r+1)*4-byte partial per row range, and every non-empty segment takes at least
 * one range; GLGA_ERR_UNSUPPORTED if that workspace would exceed 4 GiB.             */
GLGA_API glga_status glga_create_segmented(glga_ctx **out, int64_t N, int32_t d, int32_t H,
                        int32_t r, glga_dtype io, const int32_t *row_ptr,
                        const int32_t *col_idx, int64_t E, const int64_t *seg_ptr,
                        int64_t n_seg, const glga_options *opts, void *stream);

/* glga_forward -- Y = layer(X) for the graph bound at create.
 *   X    (device) io [N, d]          W_Q, W_K, W_V (device) io [d, H*r]
 *   w_g  (device) io [d]             b_g, eps (host) gate bias and readout epsilon
 *   Y    (device) io [N, H*r], written entirely
 * Enqueued on `stream` with no host synchronisation; the context's workspaces are
 * reused, so calls on one context must be ordered (same stream, or synchronised).
 * Device-side failures (bounded waits, debug checks) surface through
 * glga_last_device_error().  eps must be > 0 and finite.                              */
GLGA_API glga_status glga_forward(glga_ctx *ctx, const void *X, const void *W_Q, const void *W_K,
                         const void *W_V, const void *w_g, float b_g, float eps, void *Y,
                         void *stream);

/* Frees every device buffer of the context (synchronises the device first).  NULL is a
 * no-op.                                                                              */
GLGA_API glga_status glga_destroy(glga_ctx *ctx);

/* glga_csr_from_coo -- target-grouped CSR from an edge list (tinymesh page, "Target
 * softmax": segment reductions traverse destination CSR).
 *   src, dst  (device) int32 [E]: edge e is src[e] -> dst[e]
 *   row_ptr   (device) int32 [N+1] out;  col_idx (device) int32 [E] out
 * Rows are targets; inside a row the sources are sorted ascending; duplicates are kept.
 * The result depends only on the multiset of edges, not on their order.  Returns
 * GLGA_ERR_BAD_GRAPH if an endpoint is outside [0, N).  Allocates temporary device
 * memory and synchronises `stream` once.                                              */
GLGA_API glga_status glga_csr_from_coo(int64_t N, int64_t E, const int32_t *src, const int32_t *dst,
                              int32_t *row_ptr, int32_t *col_idx, void *stream);

/* Bucket sizes chosen at create: counts (host) int64 [4] = rows in buckets 0, 1, 2 and
 * the number of bucket-2 chunks.                                                      */
GLGA_API glga_status glga_bucket_counts(const glga_ctx *ctx, int64_t *counts);

/* Row-sharded forward (one context per rank; one process per GPU).  Target rows are cut
 * into contiguous blocks; rank p owns rows [row_begin, row_end) of the n_nodes nodes.
 * The one exchange step of the method, moved by the caller (NCCL over NVLink, e.g.
 * torch.distributed): every rank's K/V rows to every rank, and the per-rank partial
 * statistics (method page "Gated Local-Global Graph Attention", "Key formulas": S and z
 * are sums over all nodes, so they split into per-rank partial sums).
 *
 * glga_create_sharded -- row_ptr (device) int32 [n_own + 1] and col_idx (device) int32
 *   [E] are the CSR of the owned rows only (row_ptr[0] = 0, local row numbering), with
 *   column indices in [0, n_nodes) (global node ids).  kv (device, caller-owned, 16-byte
 *   aligned, io [n_nodes, 2*H*r], row j = k_j | v_j) is the K/V buffer the rank's
 *   projection writes its rows into (rows row_begin .. row_end-1) and that the exchange
 *   fills with the other ranks' rows; it must outlive the context.  Other arguments and
 *   errors as glga_create.
 * glga_forward_begin -- X (device) io [n_own, d]: the owned rows' inputs.  Projects them
 *   (Q, t into the context; k, v into kv) and writes the rank's partial statistics to
 *   own_partial (device) float [H][r][r+1] (per head, row a: S_h[a][0..r-1] then z_h[a]).
 * glga_forward_end -- after the exchange: partials (device) float [P][H][r][r+1] holds the
 *   P ranks' partials in rank order and kv holds every node's k/v.  Sums the partials in
 *   a fixed order (the same on every rank), then computes the owned rows' Y (device, io
 *   [n_own, H*r]).
 * Both are stream-ordered with no host synchronisation.  glga_forward refuses a sharded
 * context; glga_get_intermediates returns the owned rows.                             */
GLGA_API glga_status glga_create_sharded(glga_ctx **out, int64_t n_nodes, int64_t row_begin,
                        int64_t row_end, int32_t d, int32_t H, int32_t r, glga_dtype io,
                        const int32_t *row_ptr, const int32_t *col_idx, int64_t E, void *kv,
                        const glga_options *opts, void *stream);
GLGA_API glga_status glga_forward_begin(glga_ctx *ctx, const void *X, const void *W_Q,
                        const void *W_K, const void *W_V, const void *w_g, float *own_partial,
                        void *stream);
GLGA_API glga_status glga_forward_end(glga_ctx *ctx, const float *partials, int32_t P, float b_g,
                        float eps, void *Y, void *stream);

/* glga_backward -- gradients of sum(Y * dY) for the Y of the last glga_forward on this
 * context, which must have been called with the same X, W_Q, W_K, W_V, w_g, b_g, eps
 * (the forward's Q, K, V, gate logits, S, z and L are reused).  Method page "Gated
 * Local-Global Graph Attention", "Key formulas", differentiated (the softmax maximum is
 * held constant, tinymesh "Target softmax").
 *   dY (device) io [N, H*r]
 *   dX (device) float [N, d]; dW_Q, dW_K, dW_V (device) float [d, H*r]; dw_g (device)
 *   float [d]; db_g (device) float [1] -- all written.
 * Needs glga_options.backward at create.  Every sum runs in a fixed order (the source
 * side walks a transposed CSR, rows with more than 64 entries are cut into 32-entry
 * chunks summed in chunk order; no atomics), so repeated calls give identical bits.
 * Stream-ordered, no host synchronisation: the source-side kernels run on a stream of the
 * context forked from and joined back into `stream` by events (capture-safe).          */
GLGA_API glga_status glga_backward(glga_ctx *ctx, const void *X, const void *W_Q, const void *W_K,
                        const void *W_V, const void *w_g, float b_g, float eps, const void *dY,
                        float *dX, float *dW_Q, float *dW_K, float *dW_V, float *dw_g, float *db_g,
                        void *stream);

/* glga_block_output -- the block around the layer, Z = LayerNorm(X + Y Wo): the output
 * projection, the residual and a LayerNorm over the d features.  Method page "Gated
 * Local-Global Graph Attention", "Implementation notes", item 2 ("return
 * LayerNorm(X + Wo(g*L+(1-g)*G))"); Wo has no bias, the LayerNorm uses the population
 * variance and a per-feature gain and bias.
 *   Y      (device) io [n, H*r]: a glga_forward output of this context (n = its rows)
 *   X      (device) io [n, d]: the layer's input rows (the residual)
 *   Wo     (device) io [H*r, d]      gamma, beta (device) io [d]
 *   ln_eps (host) >= 0, added to the variance        Z (device) io [n, d], written
 * Requires d to be a multiple of 32 and at most 512 (GLGA_ERR_UNSUPPORTED otherwise).
 * Y, X and Z 16-byte aligned.  Stream-ordered, no host synchronisation; uses only
 * workspaces allocated at create.                                                     */
GLGA_API glga_status glga_block_output(glga_ctx *ctx, const void *Y, const void *X, const void *Wo,
                        const void *gamma, const void *beta, float ln_eps, void *Z,
                        void *stream);

/* Copies the bucket lists (device -> device, on `stream`) into caller buffers sized by
 * glga_bucket_counts: warp_rows [counts[0]], cta_rows [counts[1]], split_rows [counts[2]],
 * chunk_row [counts[3]], chunk_begin [counts[3]] (the CSR offset of the chunk's first
 * edge).  Any pointer may be NULL to skip that list.                                  */
GLGA_API glga_status glga_get_buckets(const glga_ctx *ctx, int32_t *warp_rows, int32_t *cta_rows,
                             int32_t *split_rows, int32_t *chunk_row, int32_t *chunk_begin,
                             void *stream);

/* Copies the intermediates of the last glga_forward (device -> device, on `stream`):
 *   Q (io [N, H*r]), K and V (io [N, H*r] each), t (float [N], gate logit x_i . w_g),
 *   S (float [n_seg, H, r, r]), z (float [n_seg, H, r]) with n_seg = 1 for glga_create,
 *   L (io [N, H*r], the local branch).  Any pointer may be NULL.                        */
GLGA_API glga_status glga_get_intermediates(const glga_ctx *ctx, void *Q, void *K, void *V, float *t,
                                   float *S, float *z, void *L, void *stream);

/* Per-stage timing.  When enabled, glga_forward records CUDA events on its stream around
 * every stage.  glga_stage_times synchronises on the last forward's final event and
 * writes up to n_max durations in milliseconds (host) in this order:
 *   0 weight packing and input preparation, 1 projection GEMM, 2 global statistics
 *   (tensor-core partials + ordered reduction), 3 local branch (per-target softmax
 *   kernel), 4 readout GEMM with the fused gate blend, 5 whole forward.  Row-sharded
 *   contexts record them in glga_forward_begin and glga_forward_end: stage 2 then also
 *   spans the caller's exchange between the two calls.  A forward recorded into a CUDA
 *   graph with timing on records the events as event record nodes: glga_stage_times
 *   after a replay reports that replay's stages.
 * Returns the number of values written through *n_written.                            */
GLGA_API glga_status glga_set_timing(glga_ctx *ctx, int enable);
GLGA_API glga_status glga_stage_times(glga_ctx *ctx, float *ms, int32_t n_max, int32_t *n_written);

/* Number of kernel launches glga_forward has issued on this context so far (host-side
 * count, incremented at every launch).                                                */
GLGA_API glga_status glga_kernel_launches(const glga_ctx *ctx, int64_t *n);

/* Bytes of device memory the context holds (workspaces + CSR copy + buckets).         */
GLGA_API glga_status glga_workspace_bytes(const glga_ctx *ctx, int64_t *bytes);

/* Synchronises `stream` and reports (then clears) the device-side error flag of the
 * context: GLGA_OK, GLGA_ERR_TIMEOUT or GLGA_ERR_DEVICE.                              */
GLGA_API glga_status glga_last_device_error(glga_ctx *ctx, void *stream);

/* glga_global_stats_static -- the global statistics S and z of glga_forward, computed
 * without allocating any device memory.  The paper has no counterpart to this entry
 * point.  It is for callers that must not allocate on their enqueue path: plugin
 * interfaces whose enqueue callback may not allocate, services that reserve all device
 * memory up front through their own pool, and latency-critical code that cannot afford
 * cudaMalloc's possible implicit device synchronisation.
 *   KV  (device) io [N, 2*H*r]: row j holds k_j (H*r values) followed by v_j (H*r values)
 *   Sz  (device) float [H*r*r + H*r], written: S [H][r][r] followed by z [H][r]
 * r must be one of 8, 16, 32, 64, 128; N >= 0; H >= 1.
 * Partial sums go to one fixed 2 MiB array inside the library's device image; every GPU
 * that loads the library holds it until the process exits.  Limit: one row range needs
 * H*r*(r+1)*4 bytes, which must fit in those 2 MiB; larger shapes return
 * GLGA_ERR_UNSUPPORTED before any device work.  The first call on a device looks up the
 * array's device address and caches it (again when the device's CUDA context has changed,
 * e.g. after cudaDeviceReset); make that first call before any stream capture.
 * All calls share the array and it keeps the last call's contents: each call writes every
 * partial sum it later reads, so nothing needs clearing, but calls that overlap on the
 * GPU (other streams or threads) race on it; the caller must order them.  No cudaMalloc,
 * cudaFree or allocating library routine is called.  The call is asynchronous: a bounded
 * wait inside its kernel that gave up (the S and z of that call are then incomplete) is
 * reported by glga_global_stats_static_error.                                           */
GLGA_API glga_status glga_global_stats_static(const void *KV, int64_t N, int32_t H, int32_t r,
                                              glga_dtype io, float *Sz, void *stream);

/* glga_global_stats_static_error -- synchronises `stream`, then reports and clears the
 * device-side flag that the glga_global_stats_static calls on the current device raise:
 * GLGA_OK, GLGA_ERR_TIMEOUT (a bounded wait of one of the calls since the last report gave
 * up, so its S and z are incomplete) or GLGA_ERR_DEVICE.  One flag per device, shared by
 * all those calls; it stays raised until this call clears it.  Allocates nothing.  The
 * paper has no counterpart (it is the error path of the entry point above).           */
GLGA_API glga_status glga_global_stats_static_error(void *stream);

/* Static strings; never NULL. */
/* Test entry points of the failure paths (the pages have no counterpart).
 *
 * glga_debug_bounded_wait -- enqueues on `stream` one thread that waits on a
 * shared-memory mbarrier nothing arrives on, with the same bounded wait the tensor-core
 * kernels use, given up after `limit_ns` nanoseconds (1e3 <= limit_ns <= 1e10).  The
 * thread then sets the context's device flag and returns, so the next
 * glga_last_device_error reports GLGA_ERR_TIMEOUT and the context stays usable.
 *
 * glga_debug_static_bounded_wait -- the same probe for the flag of the
 * glga_global_stats_static calls on the current device (reported by
 * glga_global_stats_static_error).
 *
 * glga_debug_set_col_idx -- overwrites entry e of the context's CSR copy with `value`,
 * skipping glga_create's validation, so that the device-side checks of a context made
 * with debug_checks != 0 can be exercised.  Refused (GLGA_ERR_INVALID_ARG) when the
 * context was made without debug_checks or e is outside [0, E).  Stream-ordered.      */
GLGA_API glga_status glga_debug_bounded_wait(glga_ctx *ctx, int64_t limit_ns, void *stream);
GLGA_API glga_status glga_debug_static_bounded_wait(int64_t limit_ns, void *stream);
GLGA_API glga_status glga_debug_set_col_idx(glga_ctx *ctx, int64_t e, int32_t value, void *stream);

GLGA_API const char *glga_status_string(glga_status s);
GLGA_API const char *glga_last_error_message(void);

#ifdef __cplusplus
}
#endif

#endif /* GLGA_H_ */
