/*
 * indexcache.h - C ABI of the B200 (sm_100a) DeepSeek-Sparse-Attention hot
 * path with IndexCache cross-layer index reuse.
 *
 * The path (IndexCache paper, "IndexCache: Accelerating Sparse Attention via
 * Cross-Layer Index Reuse", Abstract and Figure 2 caption):
 *   1. lightning indexer  I[t,s] = sum_j w[t,j] * ReLU(q_I[t,j,:] . k_I[s,:])
 *      over causal keys s <= t (the DSA indexer of DeepSeek-V3.2, which the
 *      paper builds on; the paper names it but prints no formula);
 *   2. per-query top-k over those scores (higher score first, equal scores
 *      to the lower key index), streamed so no L x L matrix exists;
 *   3. sparse attention over the k selected rows of a latent KV;
 *   4. a per-layer F/S pattern: Full layers run 1-2 and overwrite one index
 *      buffer, Shared layers reuse it (IndexCache repository README, "Launch
 *      with IndexCache": index_topk_freq / index_topk_pattern; neither set =
 *      standard DSA).
 *
 * Conventions for every entry point:
 *  - Tensor arguments are DEVICE pointers to row-major contiguous arrays,
 *    owned by the caller (ic_layer_stack_host also takes host pointers). The
 *    library never allocates device memory; calls
 *    that need scratch take a caller-provided workspace whose size the
 *    matching *_workspace_size function reports. A workspace pointer, when
 *    not NULL, must be 256-byte aligned (IC_ERR_WORKSPACE otherwise).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream). Work is enqueued asynchronously; no call synchronises, so the
 *    launching calls may be captured into a CUDA graph.
 *  - Arguments are validated on the host before anything is enqueued; an
 *    invalid call returns an error status and enqueues nothing. A launch
 *    failure returns IC_ERR_CUDA. Device-side bounded waits that expire set a
 *    sticky device status read by ic_get_device_status. No C++ exception
 *    crosses the ABI.
 *  - Element formats: IC_BF16 (bfloat16 bits), IC_FP8_E4M3 (OCP E4M3 codes,
 *    one byte), IC_F32.
 *  - Positions: query row t of batch element b sits at absolute position
 *    q_pos0 + t; it sees keys s with s <= q_pos0 + t and s < n_k. Prefill
 *    uses q_pos0 = 0 and n_q = n_k; a decode step with one new token per
 *    request uses n_q = 1, q_pos0 = n_k - 1.
 */
#ifndef INDEXCACHE_H
#define INDEXCACHE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    IC_OK = 0,
    IC_ERR_INVALID_ARG = 1,  /* null pointer, negative or inconsistent size      */
    IC_ERR_BAD_PATTERN = 2,  /* F/S pattern string malformed                      */
    IC_ERR_UNSUPPORTED = 3,  /* valid request outside the compiled kernel shapes  */
    IC_ERR_CUDA = 4,         /* a CUDA runtime/driver call or launch failed       */
    IC_ERR_TIMEOUT = 5,      /* a device-side bounded wait expired (sticky)       */
    IC_ERR_WORKSPACE = 6,    /* workspace pointer null or smaller than required   */
    IC_ERR_INTERNAL = 7      /* a device-side consistency check failed; the access
                                was skipped and the results are invalid (sticky)  */
} ic_status;

typedef enum { IC_BF16 = 0, IC_FP8_E4M3 = 1, IC_F32 = 2 } ic_dtype;

/* Human-readable name of a status code (static string, never NULL). */
const char* ic_status_string(ic_status status);

/* ABI version of this library: (major << 16) | minor. */
int ic_version(void);

/*
 * Resolve the per-layer F/S assignment (host only, no device work).
 * Source: IndexCache README, "Launch with IndexCache" - Option A uniform
 * interleaving ("every N-th layer keeps its indexer"), Option B custom
 * pattern (one character per DSA layer, 'F' = Full, 'S' = Shared), and the
 * default (neither set: all layers Full).
 *   n_layers              number of layers, >= 1
 *   index_topk_freq       0 = unset; N >= 1: layer l is Full iff l % N == 0
 *   index_topk_pattern    NULL = unset; else exactly n_layers chars of F/S,
 *                         first char 'F'
 *   is_full_out[n_layers] host array: 1 for Full layers
 *   src_layer_out[n_layers] host array: the Full layer whose indices layer l
 *                         uses (the nearest preceding Full layer, l itself
 *                         for a Full layer)
 * Errors: IC_ERR_INVALID_ARG (n_layers < 1, freq < 0, both options set, null
 * outputs), IC_ERR_BAD_PATTERN (wrong length, other characters, leading 'S').
 */
ic_status ic_resolve_pattern(int n_layers, int index_topk_freq, const char* index_topk_pattern,
                             uint8_t* is_full_out, int32_t* src_layer_out);

/*
 * Fused lightning indexer + streaming top-k (one Full layer).
 * Source: IndexCache paper, Abstract ("a lightweight lightning indexer
 * selects the top-k most relevant tokens per query"); score definition of
 * the DSA lightning indexer (see file header).
 *   q_I     [batch, n_q, H_I, d_I]  qk_dtype (IC_BF16 or IC_FP8_E4M3)
 *   q_scale [batch, n_q]  fp32, per-token scale of q_I (NULL for bf16;
 *           required and > 0 for FP8)
 *   w       [batch, n_q, H_I]  w_dtype (IC_BF16 or IC_F32)
 *   k_I     [batch, n_k, d_I]  qk_dtype
 *   k_scale [batch, n_k]  fp32 per-token scale of k_I (NULL for bf16;
 *           required and > 0 for FP8)
 *           The scales live in device memory and are NOT checked: the host
 *           never reads them (that would need a copy and a synchronisation).
 *           A scale that is zero, negative or not finite breaks the
 *           factoring of the scales out of the ReLU, and the selected keys
 *           are then unspecified (no fault, no error status).
 *   idx_out [batch, n_q, topk] int32: for each query the indices of its top-k
 *           keys, each once, followed by -1 entries when fewer than topk keys
 *           are visible. Which keys are selected is exact: score descending,
 *           equal scores broken toward the lower key index (and -0.0 ==
 *           +0.0). Scores are computed in fp32 from fp32 tensor-core
 *           accumulators. The order of a row's entries is deterministic (the
 *           same inputs give the same bytes) but otherwise unspecified: a
 *           query that sees at most topk keys lists 0..t; H_I = 4 shapes and
 *           decode score rows list ascending indices; the other 64-head
 *           paths list the keys grouped by (index mod 128) / 32, ascending
 *           within a group. Consumers treat a row as a set.
 * Supported shapes: H_I in {4, 64} (d_I = 64 for H_I = 4, 128 for H_I = 64),
 * FP8 only with d_I = 128, 1 <= topk <= 2048. Others: IC_ERR_UNSUPPORTED.
 * Workspace: ic_indexer_workspace_size (0 bytes for prefill; decode-style
 * calls with n_q == 1 split the key range and need scratch).
 */
ic_status ic_indexer_workspace_size(int batch, int n_q, int n_k, int H_I, int d_I, int topk,
                                    ic_dtype qk_dtype, size_t* bytes_out);
ic_status ic_indexer_topk(const void* q_I, const float* q_scale, const void* w, ic_dtype w_dtype,
                          const void* k_I, const float* k_scale, ic_dtype qk_dtype,
                          int batch, int n_q, int n_k, int q_pos0, int H_I, int d_I, int topk,
                          int32_t* idx_out, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Sparse attention over selected latent-KV rows (one layer).
 * Source: IndexCache paper, Abstract (core attention over the k selected
 * tokens, O(Lk)). All H query heads share one latent KV row per key; the
 * score uses the first d_qk columns, the value the first d_v columns:
 *   out[b,t,h,:] = sum_{s in idx[b,t]} softmax_s(sm_scale * q[b,t,h,:d_qk].kv[b,s,:d_qk])
 *                  * kv[b,s,:d_v]
 *   q   [batch, n_q, H, d_qk] bf16
 *   kv  [batch, n_k, d_qk] bf16
 *   idx [batch, n_q, topk] int32; entries outside [0, n_k) (e.g. -1 padding)
 *       are skipped; order is irrelevant. A row with no valid entry yields 0.
 *   out [batch, n_q, H, d_v] bf16 (fp32 accumulation, online softmax)
 * Supported: H <= 64, d_qk a multiple of 64 up to 576, d_v a multiple of 64
 * with d_v <= d_qk and d_v <= 512. Decode-style calls (n_q == 1) split the
 * key list across CTAs and need workspace (ic_sparse_attn_workspace_size).
 */
ic_status ic_sparse_attn_workspace_size(int batch, int n_q, int H, int d_v, int topk,
                                        size_t* bytes_out);
ic_status ic_sparse_attn(const void* q, const void* kv, const int32_t* idx,
                         int batch, int n_q, int n_k, int H, int d_qk, int d_v, int topk,
                         float sm_scale, void* out, void* workspace, size_t workspace_bytes,
                         void* stream);

/*
 * Allocation-free variant of ic_indexer_topk (the IndexCache paper has no
 * counterpart; this is a library facility). Same arguments and results as
 * ic_indexer_topk, without the workspace: calls that need scratch (the
 * decode-style split of the key range) use a fixed array that the library
 * owns in device memory, so nothing is allocated per call. It is meant for
 * callers that cannot call cudaMalloc: code whose device memory belongs to
 * another allocator or a fixed arena (a framework's caching allocator, an
 * embedding application with a hard memory budget), and code paths that
 * must not risk the implicit device-wide synchronisation an allocation can
 * cause.
 *   - The array holds ic_indexer_noalloc_max_scratch() bytes (8 MiB) on
 *     every device that loads the library, until the process exits. A call
 *     that needs more returns IC_ERR_WORKSPACE (text in
 *     ic_last_error_string) and enqueues nothing; prefill-style calls need
 *     no scratch at all.
 *   - The first call on a device that needs scratch resolves the array's
 *     device address (cudaGetSymbolAddress, with that device current); make
 *     that first call before any stream capture.
 *   - All calls share the one array and it keeps the last call's contents.
 *     Calls whose kernels overlap on the GPU (different streams, no ordering
 *     between them) race on it; order them on one stream or with events.
 */
ic_status ic_indexer_topk_noalloc(const void* q_I, const float* q_scale, const void* w,
                                  ic_dtype w_dtype, const void* k_I, const float* k_scale,
                                  ic_dtype qk_dtype, int batch, int n_q, int n_k, int q_pos0,
                                  int H_I, int d_I, int topk, int32_t* idx_out, void* stream);
size_t ic_indexer_noalloc_max_scratch(void);
/* Scratch bytes ic_indexer_topk_noalloc would use for this shape (the split
 * candidate lists of a decode-style call; 0 for prefill-style calls). Unlike
 * ic_indexer_topk, the allocation-free call never uses the decode score rows,
 * whose size grows with batch x n_k. */
ic_status ic_indexer_noalloc_scratch_size(int batch, int n_q, int n_k, int H_I, int d_I, int topk,
                                          ic_dtype qk_dtype, size_t* bytes_out);

/* Per-layer device pointers for ic_layer_stack. Shared layers may leave the
 * indexer fields NULL (they are never read). */
typedef struct {
    const void* q_I;
    const float* q_scale;
    const void* w;
    const void* k_I;
    const float* k_scale;
    const void* q;
    const void* kv;
    void* out;
} ic_layer_io;

/* Shape shared by every layer of the stack. */
typedef struct {
    int batch, n_q, n_k, q_pos0;
    int H_I, d_I, topk;
    ic_dtype qk_dtype, w_dtype;
    int H, d_qk, d_v;
    float sm_scale;
} ic_stack_shape;

/*
 * The IndexCache layer loop (paper, Figure 2 caption): for l = 0..n-1,
 * if layer l is Full, run ic_indexer_topk into `idx_buffer` (overwriting it);
 * then run ic_sparse_attn with whatever idx_buffer holds. Shared layers thus
 * reuse the nearest preceding Full layer's indices with no extra memory:
 * idx_buffer [batch, n_q, topk] int32 is the single cached index tensor.
 *   layers  HOST array of n_layers ic_layer_io (device pointers inside)
 *   index_topk_freq / index_topk_pattern as in ic_resolve_pattern
 * All kernels are enqueued on `stream` in layer order; the call does not
 * synchronise. Workspace: ic_layer_stack_workspace_size.
 */
ic_status ic_layer_stack_workspace_size(const ic_stack_shape* shape, size_t* bytes_out);
ic_status ic_layer_stack(const ic_layer_io* layers, int n_layers, int index_topk_freq,
                         const char* index_topk_pattern, const ic_stack_shape* shape,
                         int32_t* idx_buffer, void* workspace, size_t workspace_bytes,
                         void* stream);

/*
 * The same layer loop with tensors that may live in HOST memory (the loop is
 * the paper's Figure 2 caption, as for ic_layer_stack).
 *   layers       HOST array of n_layers ic_layer_io. Each pointer inside may be
 *                host memory (page-locked or pageable) or device memory: the
 *                library asks CUDA which (cudaPointerGetAttributes). Device
 *                tensors are used in place (a resident KV cache, say). Host
 *                inputs are copied into a device slot before the layer runs,
 *                and a host `out` receives the layer's output once it is done.
 *   idx_host_out the final index buffer [batch, n_q, topk] int32 (the last
 *                Full layer's indices), host or device memory, or NULL
 *   staging      device memory, 256-byte aligned, of the size that
 *                ic_layer_stack_host_staging_size reports for the same layers
 *                and shape: two layer slots, the index buffer, the workspace
 *   h2d_bytes_out, d2h_bytes_out  optional (NULL): bytes the call copies in
 *                and out. Layer l uses slot l % 2; a host input buffer that
 *                the slot already holds (staged there by an earlier layer of
 *                the same call and not overwritten since) is not copied again.
 * Layer l+1's input copies and layer l-1's output copy run on two internal
 * streams of the library while layer l's kernels run on `stream`; events
 * order each slot's reuse. The internal streams fork from `stream` at the
 * start and join it at the end, so the call's work is complete when `stream`
 * drains, and the call can be captured in a CUDA graph with `stream` (with
 * page-locked host buffers). Overlap needs page-locked host buffers; pageable
 * ones work, with serialised copies. The host buffers must stay valid and
 * unchanged until then. A host `out` that overlaps a host input of the same
 * call returns IC_ERR_INVALID_ARG (a layer's inputs may be copied in before
 * an earlier layer's output has been copied out). Validation as ic_layer_stack, before anything is
 * enqueued; a staging area that is NULL, unaligned or smaller than required
 * returns IC_ERR_WORKSPACE.
 */
ic_status ic_layer_stack_host_staging_size(const ic_layer_io* layers, int n_layers,
                                           const ic_stack_shape* shape, size_t* bytes_out);
ic_status ic_layer_stack_host(const ic_layer_io* layers, int n_layers, int index_topk_freq,
                              const char* index_topk_pattern, const ic_stack_shape* shape,
                              int32_t* idx_host_out, void* staging, size_t staging_bytes,
                              void* stream, size_t* h2d_bytes_out, size_t* d2h_bytes_out);

/*
 * Multi-layer distillation target (IndexCache paper, Abstract: each retained
 * indexer is trained against the averaged attention distributions of all
 * the layers it serves; Table 3, "w/o cross-layer loss": one served layer,
 * the Full layer itself). Forward quantities only. For query row r and the
 * positions j of idx[r] whose key s_j lies in [0, n_k):
 *   P[j]  = (1 / (n_served * H)) * sum over served layers l and heads h of
 *           softmax_j(sm_scale * q_l[r,h,:d_qk] . kv_l[s_j,:d_qk])
 *   Q[j]  = softmax_j(I[r, s_j]), I the Full layer's indexer score (as in
 *           ic_indexer_topk, without the causal mask: the keys are given)
 *   kl[r] = sum_j P[j] * (log P[j] - log Q[j])
 *   q_layers, kv_layers  HOST arrays of n_served DEVICE pointers: the served
 *           layers' q [batch, n_q, H, d_qk] and kv [batch, n_k, d_qk], bf16
 *   q_I, q_scale, w, k_I, k_scale  the Full layer's indexer tensors, as for
 *           ic_indexer_topk (H_I heads of d_I)
 *   idx     [batch, n_q, topk] int32, the Full layer's index rows
 *   target_out [batch, n_q, topk] fp32 P aligned with idx (0 at invalid
 *           positions), or NULL; kl_out [batch, n_q] fp32 (0 for a row with
 *           no valid position)
 * fp32 arithmetic. Supported: 1 <= n_served <= 64, d_qk in {64, 576},
 * 1 <= H <= 64, H_I in {4, 64}, d_I a multiple of 8 (<= 128), topk <= 2048;
 * others IC_ERR_UNSUPPORTED. The model's shapes (H = 64, d_qk = 576,
 * H_I = 64, d_I = 128) run on the tensor cores and, for topk > 1024, need
 * workspace (ic_distill_target_workspace_size bytes, 256-byte aligned; else
 * IC_ERR_WORKSPACE): logits of up to 8 tiles of 128 keys per CTA wait there
 * between a statistics pass and a probability pass. Other shapes need none
 * (workspace may be NULL). q_I, k_I and the q/kv pointers 16-byte aligned.
 * Asynchronous on `stream`.
 */
ic_status ic_distill_target_workspace_size(int batch, int n_q, int topk, int H, int d_qk, int H_I, int d_I,
                                           size_t* bytes_out);
ic_status ic_distill_target(const void* const* q_layers, const void* const* kv_layers, int n_served,
                            const void* q_I, const float* q_scale, const void* w, ic_dtype w_dtype,
                            const void* k_I, const float* k_scale, ic_dtype qk_dtype,
                            const int32_t* idx, int batch, int n_q, int n_k, int H_I, int d_I,
                            int topk, int H, int d_qk, float sm_scale, float* target_out,
                            float* kl_out, void* workspace,
                            size_t workspace_bytes, void* stream);

/*
 * Pattern tools (IndexCache paper, Appendix Figure 4: the pairwise top-k
 * index overlap ratio between layer pairs; Table 5: a pattern searched from
 * that similarity; Abstract: the training-free greedy search that removes
 * indexers one at a time by a loss on calibration data).
 *
 * ic_topk_overlap: counts_out[r] = |valid(idx_a[r]) intersect valid(idx_b[r])|
 * for `rows` index rows of `topk` entries each (device pointers; an entry is
 * valid when it lies in [0, n_k); a row holds no index twice, as
 * ic_indexer_topk writes them). Order of entries within a row does not
 * matter. n_k <= 1,800,000 (the per-row key set lives in shared memory),
 * else IC_ERR_UNSUPPORTED. Asynchronous on `stream`.
 */
ic_status ic_topk_overlap(const int32_t* idx_a, const int32_t* idx_b, int rows, int topk, int n_k,
                          int32_t* counts_out, void* stream);

/*
 * ic_overlap_matrix: the layer x layer overlap-ratio matrix of n_layers index
 * buffers (each layer run with its own indexer), written to the host array
 * ratio_out (row-major n_layers x n_layers, doubles):
 *     ratio_out[a][b] = sum_r |valid(T_a[r]) & valid(T_b[r])| / sum_r |valid(T_a[r])|
 * (the share of layer a's selections that layer b also selects; 1 on the
 * diagonal, 0 rows when layer a selects nothing). idx_layers is a HOST array
 * of n_layers device pointers, each [rows, topk] int32 as ic_indexer_topk
 * writes it. Validity and the n_k limit as for ic_topk_overlap; n_layers <=
 * 128, else IC_ERR_UNSUPPORTED. The counts accumulate in the caller's device
 * workspace (ic_overlap_matrix_workspace_size bytes, else
 * IC_ERR_WORKSPACE). Enqueued on `stream`, then the call synchronises that
 * stream to read the counts back and returns with ratio_out filled.
 */
ic_status ic_overlap_matrix_workspace_size(int n_layers, size_t* bytes_out);
ic_status ic_overlap_matrix(const int32_t* const* idx_layers, int n_layers, int rows, int topk, int n_k,
                            void* workspace, size_t workspace_bytes, double* ratio_out, void* stream);

/*
 * ic_pattern_score (host only): the objective ic_search_pattern maximises,
 * for one pattern: sum over layers l of overlap[l * n_layers + src(l)], with
 * src(l) the nearest Full layer at or before l. `pattern` is n_layers
 * characters 'F'/'S' starting with 'F' (else IC_ERR_BAD_PATTERN).
 */
ic_status ic_pattern_score(const double* overlap, int n_layers, const char* pattern, double* score_out);

/*
 * ic_search_pattern (host only): the F/S pattern with exactly n_full Full
 * layers, layer 0 Full, that maximises
 *     sum over layers l of overlap[l * n_layers + src(l)],
 * src(l) = the nearest Full layer at or before l, i.e. the share of each
 * layer's own top-k that the indices it reuses recover. `overlap` is a host
 * row-major n_layers x n_layers matrix of finite values (overlap[l][f]: the
 * fraction of layer l's selections that layer f also selects). Exact, by
 * dynamic programming over the segments between Full layers; among equal
 * scores the earliest last segment wins. Writes n_layers characters 'F'/'S'
 * plus a terminating 0 to pattern_out and the score to score_out (may be
 * NULL).
 */
ic_status ic_search_pattern(const double* overlap, int n_layers, int n_full, char* pattern_out,
                            double* score_out);

/*
 * ic_greedy_pattern (host only): the greedy search that starts with every
 * layer Full and, until n_full Full layers remain, turns into Shared the one
 * Full layer (never layer 0) whose removal gives the smallest
 * objective(pattern, ctx) (lower is better; among equal values the lowest
 * layer). `objective` is called with a 0-terminated F/S string of n_layers
 * characters and returns a finite value; a non-finite value stops the search
 * with IC_ERR_INVALID_ARG. Writes the final pattern (n_layers + 1 bytes) to
 * pattern_out and its objective to value_out (may be NULL).
 */
typedef double (*ic_pattern_objective)(const char* pattern, void* ctx);
ic_status ic_greedy_pattern(int n_layers, int n_full, ic_pattern_objective objective, void* ctx,
                            char* pattern_out, double* value_out);

/*
 * Sticky device status of the current device: IC_OK, IC_ERR_TIMEOUT when a
 * kernel's bounded wait expired, or IC_ERR_INTERNAL when a kernel's
 * consistency check failed (a split candidate list whose stored length is
 * out of range), since the last reset. The first error recorded
 * is kept. Synchronises the device. reset != 0 clears it.
 */
ic_status ic_get_device_status(int reset);

/*
 * Text of the last CUDA failure seen by this thread's calls (the call site and
 * cudaGetErrorString), "" if none. Static per-thread storage, never NULL.
 */
const char* ic_last_error_string(void);

/*
 * Test hook for the failure path: launches one CTA that waits on a barrier
 * nothing ever completes, giving up after `timeout_ns` nanoseconds; the
 * expired wait sets the sticky device status to IC_ERR_TIMEOUT. No fault,
 * trap or hang is involved.
 */
ic_status ic_debug_expire_wait(long long timeout_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* INDEXCACHE_H */
