/*
 * recsa.h — C ABI of librecsa.so, RecSA (Recursive Sparse Attention) tree
 * sparse attention for one attention layer on an NVIDIA B200 (sm_100a).
 *
 * The method ("Recursive Sparse Attention: Million-Token Length
 * Extrapolation at Logarithmic Cost", arXiv 2611.07232, abstract; the
 * kongchang.com RecSA article, "Core Idea" and "Position Encoding"):
 *   - a tree is kept over each (sequence, KV head) slice of the KV cache; the
 *     bottom level is the exact tokens, node m of level j covers children
 *     [m b, (m+1) b) of level j-1 and tokens [m b^j, (m+1) b^j);
 *   - a node's value is the exact mean of its subtree's token values; its key
 *     is one per-layer pooler W (d x d, y = W x) applied to the mean of its
 *     children's stored keys;
 *   - the top level J is the first level with at most b nodes; a query scores
 *     every top-level node, keeps the k best (ranked by the sum of its G query
 *     heads' logits, ties to the smaller node id), scores the children of the
 *     kept nodes, and so on down to the tokens;
 *   - every scored-but-not-kept node enters one shared softmax as a summary
 *     (its key's logit, its mean value); the tokens under the kept level-1
 *     nodes enter exactly;
 *   - each entry is RoPE-rotated (rotate-half, theta_i = base^(-2i/d)) at its
 *     index among its level's candidates (ascending node order), and the query
 *     of a level with n candidates sits at index n-1; logits are scaled by
 *     1/sqrt(d).
 *
 * Memory. The caller owns all device memory: the KV cache, the workspace
 * (tree levels, running sums, RoPE table, pooler copy, lengths) and every
 * input and output buffer. The library makes no allocation call and never
 * synchronises the device except in recsa_check_device. The one piece of
 * device memory it owns is a fixed 8 MiB array used only by
 * recsa_dense_decode_static (see there).
 *
 * Layouts (row-major, element type = config.dtype unless stated):
 *   cache      K, V [B][H_kv][capacity][d]   keys stored before RoPE
 *   decode     q, out [B][H_q][d]            query head h reads KV head h / G
 *   append     k_new, v_new [B][n][H_kv][d]
 *   prefill    q, out [B][C][H_q][d]; k, v [B][C][H_kv][d]
 *
 * Pointers documented as "device" may also be pinned host memory that is
 * mapped into the device's address space (cudaHostAlloc memory under unified
 * addressing): the kernels then read or write it over the bus.
 *
 * Streams. Every call that launches work is asynchronous on the given
 * stream (a cudaStream_t; NULL = legacy default stream). Argument errors are
 * detected on the host, return a status and launch nothing;
 * recsa_last_error() then describes the error (thread-local string).
 */
#ifndef RECSA_H
#define RECSA_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* recsa_stream_t; /* same type as cudaStream_t */
typedef struct recsa_ctx recsa_ctx;

typedef enum {
    RECSA_OK = 0,
    RECSA_ERR_INVALID_ARG = 1, /* bad pointer, size, alignment or config   */
    RECSA_ERR_CAPACITY = 2,    /* would exceed capacity or the workspace    */
    RECSA_ERR_UNSUPPORTED = 3, /* valid but not built (e.g. head_dim 96)   */
    RECSA_ERR_CUDA = 4,        /* a CUDA runtime call failed                */
    RECSA_ERR_DEVICE = 5       /* a kernel reported an inconsistent state   */
} recsa_status;

typedef enum { RECSA_F32 = 0, RECSA_BF16 = 1 } recsa_dtype;

typedef struct {
    int batch;          /* B independent sequences, >= 1                      */
    int n_kv_heads;     /* H_kv >= 1                                          */
    int n_q_heads;      /* H_q = G * H_kv, G in {1, 2, 4, 8}                  */
    int head_dim;       /* d in {64, 128}                                     */
    int branching;      /* b in [2, 256]                                      */
    int k;              /* kept nodes per level, 1 <= k <= 64, k * b <= 4096  */
    long long capacity; /* maximum tokens per sequence, >= 1                  */
    int max_chunk;      /* largest prefill chunk C (0: prefill not used)      */
    double rope_base;   /* RoPE base, > 1                                     */
    recsa_dtype dtype;  /* storage and I/O type of cache, nodes, q, out       */
} recsa_config;

/* Bytes of device workspace recsa_init needs for this configuration (0 if
 * the configuration is invalid; recsa_last_error says why). */
size_t recsa_workspace_bytes(const recsa_config* cfg);

/* Creates a context. k_cache / v_cache: the caller's cache buffers (layout
 * above), borrowed for the context's lifetime. workspace: >=
 * recsa_workspace_bytes(cfg) bytes of device memory, 256-byte aligned, owned
 * by the context until recsa_destroy. pooler_w: device pointer to W [d][d]
 * (row-major, y = W x) in cfg->dtype; copied into the workspace on `stream`,
 * so it may be freed once that stream has passed this call. All sequence
 * lengths start at 0. On error *out is left NULL. */
recsa_status recsa_init(recsa_ctx** out, const recsa_config* cfg, void* k_cache, void* v_cache, void* workspace,
                        size_t workspace_bytes, const void* pooler_w, recsa_stream_t stream);

/* recsa_init with a paged token cache: instead of K, V [B][H_kv][capacity]
 * [d], the tokens live in a pool of pages shared by the sequences, K, V
 * [num_pages][H_kv][page_size][d] (the caller's, borrowed). Token t of
 * sequence b is row t % page_size of pool page page_table[b * max_pages +
 * t / page_size]; page_table (device int32 [B][max_pages], borrowed) is
 * read by the kernels at every call, so the caller assigns a page before the
 * tokens that land in it are appended (for example a serving engine handing
 * out pages on demand), and may change entries of pages not yet used.
 * page_size must be a multiple of the branching factor (the children of a
 * level-1 node, b consecutive tokens, then lie in one page) and max_pages *
 * page_size must cover cfg->capacity. The tree levels stay in the workspace.
 * A page id outside [0, num_pages) is reported by recsa_check_device (shape
 * bit) and page 0 is read instead. Every other call is unchanged. This is
 * the paged, variable-length cache of a serving engine; the pages (RecSA
 * abstract: a tree over the KV cache) do not change what is computed. */
recsa_status recsa_init_paged(recsa_ctx** out, const recsa_config* cfg, void* k_pool, void* v_pool,
                              long long num_pages, int page_size, const int* page_table, int max_pages,
                              void* workspace, size_t workspace_bytes, const void* pooler_w, recsa_stream_t stream);

/* Sets sequence b's length to lengths[b] (host array of B entries, each in
 * [0, capacity]) and builds every tree level from the tokens already in the
 * cache. The tree is the one the RecSA abstract keeps over the KV cache: node
 * values are subtree means of the token values, node keys the layer's pooler
 * applied to the mean of the children's keys (kongchang.com article, "Core
 * Idea": mean pooling of values, learned pooling of keys). */
recsa_status recsa_build_tree(recsa_ctx* ctx, const long long* lengths, recsa_stream_t stream);

/* Appends n >= 1 tokens to every sequence: copies k_new / v_new
 * ([B][n][H_kv][d], device) into the cache after each sequence's current
 * tokens, then brings every node whose subtree gained tokens up to date, so
 * that the tree stays the one over the whole cache (RecSA abstract: the tree
 * lives over the KV cache and grows with it; kongchang.com "Core Idea": node
 * value = mean of its tokens, node key = pooler of its children's keys).
 * Right-edge nodes stay exact means; their keys are recomputed by the pooler.
 * A prefill chunk is appended with this call after recsa_prefill (the tree is
 * updated after each chunk). RECSA_ERR_CAPACITY (nothing launched) if any
 * sequence would exceed the capacity. */
recsa_status recsa_append(recsa_ctx* ctx, const void* k_new, const void* v_new, int n, recsa_stream_t stream);

/* One decode query per sequence (per-level top-k descent, shared softmax and
 * candidate-index RoPE: abstract; "Core Idea"; "Position Encoding").
 * q [B][H_q][d] (device) is the query of the last cached position: append
 * the current token first; the query descends the tree over every cached
 * token. out [B][H_q][d] (device). sel_out (nullable, device int32 [B][H_kv][J_cap][k]): the kept
 * node ids of level j in row j-1, ascending, -1 padded (levels above the
 * current top level are all -1). rows_out (nullable, device int64
 * [B][H_kv][2]): K rows and V rows (= softmax entries) read per KV head.
 * Every sequence must hold at least one token. */
recsa_status recsa_decode(recsa_ctx* ctx, const void* q, void* out, int* sel_out, long long* rows_out,
                          recsa_stream_t stream);

/* One decode step in a single launch: appends one token per sequence (as
 * recsa_append with n = 1, same node arithmetic) and decodes q against the
 * grown tree (as recsa_decode). k_new, v_new [B][1][H_kv][d], q, out
 * [B][H_q][d] (device, 16-byte aligned); sel_out and rows_out as in
 * recsa_decode. RECSA_ERR_CAPACITY (nothing launched) if a sequence is full.
 * The appended token is the one q belongs to: the query attends it. */
recsa_status recsa_append_decode(recsa_ctx* ctx, const void* k_new, const void* v_new, const void* q, void* out,
                                 int* sel_out, long long* rows_out, recsa_stream_t stream);

/* Chunked causal prefill of C tokens per sequence (1 <= C <= max_chunk):
 * token t of the chunk runs the same descent as a decode query (RecSA
 * abstract: top-down selection of at most k nodes per level, one softmax over
 * the unselected summaries and the exact tokens, RoPE at candidate indices;
 * kongchang.com "Core Idea" and "Position Encoding") over the tree of the
 * sequence's cached tokens [0, s), and also attends the chunk's own tokens
 * s..t exactly, which follow the level-0 candidates in the RoPE index order
 * (causality inside the chunk is this library's reading: the pages do not
 * spell out chunked prefill). q [B][C][H_q][d], k, v
 * [B][C][H_kv][d], out [B][C][H_q][d] (device). sel_out (nullable, device
 * int32 [B][C][H_kv][J_cap][k]) as in recsa_decode. rows_out (nullable,
 * device int64 [B][C][H_kv][2]): key rows scored and value rows (softmax
 * entries, the chunk's own tokens included) per token and KV head. scratch: device memory
 * of recsa_prefill_scratch_bytes(cfg, C) bytes, 256-byte aligned. The chunk
 * is not appended: call recsa_append(k, v, C) afterwards. Built for bf16
 * storage only (RECSA_ERR_UNSUPPORTED for fp32, or when k * b candidates
 * per level exceed the kernel's shared memory). */
size_t recsa_prefill_scratch_bytes(const recsa_config* cfg, int C);
recsa_status recsa_prefill(recsa_ctx* ctx, const void* q, const void* k, const void* v, int C, void* out,
                           int* sel_out, long long* rows_out, void* scratch, size_t scratch_bytes,
                           recsa_stream_t stream);

/* Host-side view of the state, for tests and tools. */
recsa_status recsa_get_lengths(const recsa_ctx* ctx, long long* lengths /* host [B] */);
/* J_cap (levels kept) and, for j = 1..J_cap, rows[j] = node rows per unit. */
recsa_status recsa_tree_shape(const recsa_ctx* ctx, int* j_cap, long long* rows /* host [J_cap + 1] */);
/* Device pointers of level j (1..J_cap): keys and values [B][H_kv][rows[j]][d]
 * in cfg->dtype, and the fp32 value sums [B][H_kv][rows[j]][d]. */
recsa_status recsa_level_arrays(const recsa_ctx* ctx, int level, void** keys, void** values, float** value_sums);

/* Per-unit statistics of the most recent recsa_decode or
 * recsa_append_decode on this context, for checking the logarithmic read
 * cost the RecSA abstract claims (a query reads O(log L) entries). Waits for
 * `stream`, then fills, for every (sequence, KV head) unit u = b * H_kv + h:
 *   depth[u]  levels the query descended, the tokens included (J + 1);
 *   k_rows[u] key rows read (node keys and token keys; levels that keep all
 *             of their at most k candidates are not read);
 *   v_rows[u] value rows read, which is the number of softmax entries.
 * Host arrays of B * H_kv entries each; any may be NULL. All zero before the
 * first decode. RECSA_ERR_CUDA if the stream reports an error. */
recsa_status recsa_query_stats(recsa_ctx* ctx, int* depth, long long* k_rows, long long* v_rows,
                               recsa_stream_t stream);

/* ---------------------------------------------------------------------
 * Gradients of decode queries (the training side of the method). The RecSA
 * abstract's output is one softmax over the summaries of the candidates not
 * kept and the exact tokens under the kept level-1 nodes; a summary's value
 * is the mean of its subtree's token values and its key the pooler W applied
 * to the mean of its children's keys (kongchang.com article, "Core Idea"),
 * so the gradient of a query's output reaches q, every cached token's key
 * and value, and W. The top-k choice is discrete and held fixed: the caller
 * passes the selections its recsa_decode returned. Rounding of stored node
 * keys and values to the storage type is taken as the identity.
 *
 * Two stages, so that any number of queries can be summed before the part
 * whose cost grows with the cache:
 *   recsa_decode_backward  per query: dq, and the gradients of the softmax
 *                          entries (tokens: added into dk, dv; summaries:
 *                          added into node accumulators held in `scratch`);
 *   recsa_tree_backward    once: carries the node accumulators down the
 *                          tree into every token's dk, dv and into dw, then
 *                          clears them.
 * `scratch`: device memory of recsa_backward_scratch_bytes(cfg) bytes,
 * 256-byte aligned, ZEROED by the caller before its first use; every
 * recsa_tree_backward leaves it zeroed again. Gradient arrays are fp32:
 *   dk, dv  one row of d per cache row, in the cache's own layout (contiguous
 *           [B][H_kv][capacity][d]; paged [num_pages][H_kv][page_size][d]);
 *           both calls ADD into them;
 *   dw      [d][d], dw[r][c] = dLoss/dW[r][c] (W row-major as given to
 *           recsa_init); recsa_tree_backward ADDS into it.
 * Asynchronous on `stream`; the context's tree and lengths must be the ones
 * the forward used (no append in between). */
size_t recsa_backward_scratch_bytes(const recsa_config* cfg);

/* q [B][H_q][d] (the forward's query) and dout [B][H_q][d] (dLoss/dout),
 * both in cfg->dtype, device, 16-byte aligned; sel [B][H_kv][J_cap][k]
 * int32 device, as recsa_decode's sel_out wrote it. dq [B][H_q][d] fp32 is
 * overwritten. A unit whose selections are not a valid descent over its
 * tree is skipped (its dq is zero) and flagged in the device error word
 * (bit 2, read by recsa_check_device). RECSA_ERR_INVALID_ARG (nothing
 * launched) for NULL or misaligned pointers, a short scratch or an empty
 * sequence. */
recsa_status recsa_decode_backward(recsa_ctx* ctx, const void* q, const void* dout, const int* sel, float* dq,
                                   float* dk, float* dv, void* scratch, size_t scratch_bytes, recsa_stream_t stream);

/* Carries the node accumulators in `scratch` into dk, dv and dw (see
 * above), level by level from the top, and clears them. dk, dv, dw: device,
 * 16-byte aligned (RECSA_ERR_INVALID_ARG otherwise); when dk, dv are 32-byte
 * aligned (and the key cache aligned to eight elements) every token row is
 * updated with 256-bit accesses, else with 128-bit ones: the same dk, dv, and
 * dw up to the order of its fp32 sums. */
recsa_status recsa_tree_backward(recsa_ctx* ctx, float* dk, float* dv, float* dw, void* scratch,
                                 size_t scratch_bytes, recsa_stream_t stream);

/* ---------------------------------------------------------------------
 * One distillation step of the pooler. The RecSA abstract trains the
 * pooler so that tree attention reproduces dense attention; this is the
 * plainest reading of that step for decode queries: the loss is the mean
 * squared difference between the layer's outputs and the caller's dense
 * attention outputs for the same queries over the same cache,
 *   loss = sum over (sequence, query head, coordinate) of (out - target)^2 / n,
 *   n = B * H_q * d,
 * with the selections of this forward held fixed; W moves by plain gradient
 * descent, w_master <- w_master - lr * dLoss/dW, the context's pooler takes
 * the new values (rounded to cfg->dtype) and every node key is rebuilt
 * under it (as recsa_build_tree over the current lengths).
 * q [B][H_q][d] in cfg->dtype and target [B][H_q][d] fp32 (device, 16-byte
 * aligned); w_master [d][d] fp32 device, row-major like the pooler given
 * to recsa_init (the caller keeps this master copy; updated in place); loss
 * (nullable) device fp32 scalar, the step's loss before the update; dw_out
 * (nullable) device [d][d] fp32, the step's gradient. scratch: device
 * memory of recsa_distill_scratch_bytes(cfg) bytes, 256-byte aligned (no
 * clearing needed). Asynchronous on `stream`. */
size_t recsa_distill_scratch_bytes(const recsa_config* cfg);
recsa_status recsa_distill_step(recsa_ctx* ctx, const void* q, const float* target, float lr, float* w_master,
                                float* loss, float* dw_out, void* scratch, size_t scratch_bytes,
                                recsa_stream_t stream);

/* Waits for `stream`, then reads and clears the device error word:
 * RECSA_ERR_DEVICE if a kernel flagged an inconsistent state (bits: 1 a
 * length out of range, 2 a tree shape inconsistent with the lengths, 4 a
 * bounded wait for an asynchronous copy ran out, about a second). */
recsa_status recsa_check_device(recsa_ctx* ctx, recsa_stream_t stream);

const char* recsa_last_error(void);
void recsa_destroy(recsa_ctx* ctx);

/* ---------------------------------------------------------------------
 * LSA-style variant: the tree over a clustered token order. The "Latent
 * Sparse Attention" abstract clusters the keys hierarchically in a learned
 * latent space and lets the queries score the hierarchy of clusters. Read
 * with this tree's fan-out b: level j has one learned direction Z_j and the
 * latent coordinate z_j(t) = <Z_j, k_t> (fp64, summed in index order); from
 * the top level down, the tokens of every block of b^(j+1) consecutive
 * positions of the current order are sorted by (z_j, token index). The
 * level-j nodes of the tree over the reordered tokens are then blocks of b^j
 * positions whose z_j ranges follow one another inside their parent; the
 * descent and the attention over that tree are the method's own (a RoPE
 * index is a position among candidates, so the original order does not
 * enter). Contiguous caches only.
 *
 * recsa_cluster_load: for every sequence b and KV head h, orders the source
 * tokens [0, lengths[b]) as above (the level count J of that length), writes
 * the order to perm and the reordered key and value rows into the cache
 * (positions [0, lengths[b])), then builds the tree as recsa_build_tree
 * does. Afterwards recsa_decode runs over the clustered tree; an append adds
 * its token at the right edge, outside the clustered order.
 *   k_src, v_src  device [B][H_kv][src_len][d] in cfg->dtype, 16-byte aligned,
 *                 read only;
 *   lengths       host [B], 0 <= lengths[b] <= min(capacity, src_len);
 *   Z             device fp32 [J_cap][d] (recsa_tree_shape gives J_cap), row
 *                 j - 1 the direction of level j, 16-byte aligned;
 *   perm          device int32 [B][H_kv][capacity]: perm[b][h][p] = the source
 *                 token index placed at cache position p (p < lengths[b]; the
 *                 rest untouched);
 *   scratch       device, recsa_cluster_scratch_bytes(cfg) bytes, 256-byte
 *                 aligned, no contents needed.
 * RECSA_ERR_INVALID_ARG / RECSA_ERR_CAPACITY (nothing launched) for NULL or
 * misaligned pointers, a short scratch, src_len outside [1, 2^31) or a length
 * out of range; RECSA_ERR_UNSUPPORTED for a paged context. */
size_t recsa_cluster_scratch_bytes(const recsa_config* cfg);
recsa_status recsa_cluster_load(recsa_ctx* ctx, const void* k_src, const void* v_src, long long src_len,
                                const long long* lengths, const float* Z, int* perm, void* scratch,
                                size_t scratch_bytes, recsa_stream_t stream);

/* Comparator, not part of the method: dense GQA flash-decode of one query
 * per sequence over every cached token, keys used as stored (no RoPE).
 * k_cache, v_cache [B][H_kv][L_stride][d], q, out [B][H_q][d], bf16 or fp32.
 * scratch: recsa_dense_decode_scratch_bytes(...) bytes of device memory. */
size_t recsa_dense_decode_scratch_bytes(int batch, int n_q_heads, int head_dim);
recsa_status recsa_dense_decode(const void* k_cache, const void* v_cache, const void* q, void* out, int batch,
                                int n_kv_heads, int n_q_heads, int head_dim, long long length, long long l_stride,
                                recsa_dtype dtype, void* scratch, size_t scratch_bytes, recsa_stream_t stream);

/* The dense comparator above, for callers that cannot allocate device
 * memory: they hold only their input and output buffers (for example a
 * plugin whose host application owns all device memory, or a path where
 * allocation is forbidden after start-up), so they cannot provide `scratch`.
 * The paper has no counterpart; this is a property of the library.
 * Instead of a caller buffer, the partial results go to a fixed 8 MiB array
 * in device memory that every GPU which loads the library holds until the
 * process exits. Same arguments and results as recsa_dense_decode, minus the
 * scratch; nothing is allocated and nothing needs clearing (every partial is
 * written before it is read). Limit: batch * n_q_heads * (head_dim + 2) * 4
 * bytes must fit in 8 MiB (batch * n_q_heads <= 16131 at head_dim 128);
 * larger calls return RECSA_ERR_CAPACITY and launch nothing; the split count
 * shrinks to fit. The first call on each device looks up the array's device
 * address (with that device current), so make it before any stream capture.
 * All calls share the one array: calls whose kernels overlap on a device
 * (for example on two streams) race and corrupt each other's results. The
 * looked-up address is kept for the life of the process: after
 * cudaDeviceReset on a device (which unloads the library's device code
 * there) do not call this entry point on that device again. */
recsa_status recsa_dense_decode_static(const void* k_cache, const void* v_cache, const void* q, void* out, int batch,
                                       int n_kv_heads, int n_q_heads, int head_dim, long long length,
                                       long long l_stride, recsa_dtype dtype, recsa_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif
