// Host side of the C ABI declared in include/recsa.h: argument checks,
// workspace layout, RoPE table, kernel dispatch. Every launch goes on the
// caller's stream; nothing here allocates device memory.
#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "../../include/recsa.h"
#include "backward.cuh"
#include "common.cuh"

namespace recsa {
template <typename T, int D>
cudaError_t launch_build_level(const TreeParams&, int, long long, int, long long, cudaStream_t);
template <typename T, int D>
cudaError_t launch_append_one(const TreeParams&, const void*, const void*, cudaStream_t);
template <typename T, int D>
cudaError_t launch_copy_tokens(const TreeParams&, const void*, const void*, int, cudaStream_t);
cudaError_t launch_set_lengths(const TreeParams&, const long long*, cudaStream_t);
cudaError_t launch_bump_lengths(const TreeParams&, long long, cudaStream_t);
template <typename T, int D, int G>
cudaError_t launch_decode(const TreeParams&, const void*, const void*, const void*, void*, int*, long long*,
                          float*, cudaStream_t);
template <typename T, int D, int G>
cudaError_t launch_dense(const void*, const void*, const void*, void*, int, long long, long long, float*, int,
                         cudaStream_t);
int dense_splits(long long units, long long L);
template <int D>
cudaError_t launch_prefill_attn(const TreeParams&, const void*, const void*, const void*, float*, void*, void*, int,
                                int, int, int, cudaStream_t);
template <int D, int G>
cudaError_t launch_prefill_tree_tc(const TreeParams&, const void*, void*, const float*, int*, long long*, int, int,
                                   const long long*, void*, cudaStream_t);
size_t prefill_tree_scratch_bytes(const TreeParams& p, int C, int Hq);
bool prefill_tree_supported(int D, int b);
size_t decode_smem_bytes(int D, int G, int elem, int k, int b, int J_cap, bool fused);
cudaError_t launch_distill_loss(const float*, const float*, float*, float*, long long, cudaStream_t);
long long cluster_records(long long units, long long cap);
size_t cluster_rec_bytes(long long units, long long cap);
template <typename T, int D>
cudaError_t launch_cluster(const TreeParams&, const void*, const void*, long long, const float*, const long long*,
                           long long, int, int*, void*, cudaStream_t);
template <typename T>
cudaError_t launch_pooler_update(float*, const float*, float, void*, float*, int, cudaStream_t);
size_t dense_static_scratch_bytes();
cudaError_t dense_static_scratch(float** out);
}  // namespace recsa

using namespace recsa;

struct recsa_ctx {
    recsa_config cfg;
    TreeParams p;
    std::vector<long long> len;  // host mirror of every sequence's length
    long long* len_stage;        // device [B] staging for recsa_build_tree
    int G;
};

namespace {

thread_local std::string g_err;

recsa_status fail(recsa_status s, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return s;
}

recsa_status cuda_fail(cudaError_t e, const char* what) {
    return fail(RECSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

long long span_sat(int b, int j) {
    long long s = 1;
    for (int i = 0; i < j; i++) {
        if (s > (1LL << 61) / b) return 1LL << 61;
        s *= b;
    }
    return s;
}

// Top level over L >= 1 tokens (first level with at most b nodes).
int levels_for(long long L, int b) {
    long long n = L;
    int j = 0;
    do {
        n = (n + b - 1) / b;
        j++;
    } while (n > b);
    return j;
}

recsa_status check_config(const recsa_config* c) {
    if (!c) return fail(RECSA_ERR_INVALID_ARG, "config is NULL");
    if (c->batch < 1 || c->n_kv_heads < 1) return fail(RECSA_ERR_INVALID_ARG, "batch and n_kv_heads must be >= 1");
    if (c->n_q_heads < c->n_kv_heads || c->n_q_heads % c->n_kv_heads)
        return fail(RECSA_ERR_INVALID_ARG, "n_q_heads must be a multiple of n_kv_heads");
    int G = c->n_q_heads / c->n_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return fail(RECSA_ERR_UNSUPPORTED, "group size %d not in {1,2,4,8}", G);
    if (c->head_dim != 64 && c->head_dim != 128) return fail(RECSA_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
    if (c->branching < 2 || c->branching > 256) return fail(RECSA_ERR_INVALID_ARG, "branching must be in [2, 256]");
    if (c->k < 1 || c->k > 64) return fail(RECSA_ERR_INVALID_ARG, "k must be in [1, 64]");
    if ((long long)c->k * c->branching > 4096) return fail(RECSA_ERR_INVALID_ARG, "k * branching must be <= 4096");
    if (c->capacity < 1 || c->capacity >= (1LL << 31)) return fail(RECSA_ERR_INVALID_ARG, "capacity out of range");
    if (c->max_chunk < 0 || c->max_chunk > 65536) return fail(RECSA_ERR_INVALID_ARG, "max_chunk out of range");
    if (!(c->rope_base > 1.0)) return fail(RECSA_ERR_INVALID_ARG, "rope_base must be > 1");
    if (c->dtype != RECSA_F32 && c->dtype != RECSA_BF16) return fail(RECSA_ERR_INVALID_ARG, "unknown dtype");
    return RECSA_OK;
}

struct Layout {
    int J_cap, npos;
    long long rows[MAXJ + 1];
    size_t off_K[MAXJ + 1], off_V[MAXJ + 1], off_VS[MAXJ + 1], off_PK[MAXJ + 1], off_PV[MAXJ + 1];
    size_t off_Wt, off_rope, off_len, off_stats, off_err, off_stage, total;
};

Layout layout_for(const recsa_config* c) {
    Layout l{};
    const size_t es = c->dtype == RECSA_BF16 ? 2 : 4;
    const size_t units = (size_t)c->batch * c->n_kv_heads, D = c->head_dim;
    l.J_cap = levels_for(c->capacity, c->branching);
    long long maxc = (long long)c->k * c->branching;
    if (maxc < c->branching) maxc = c->branching;
    l.npos = (int)(maxc + c->max_chunk);
    size_t o = 0;
    l.rows[0] = c->capacity;
    for (int j = 1; j <= l.J_cap; j++) {
        l.rows[j] = (c->capacity + span_sat(c->branching, j) - 1) / span_sat(c->branching, j);
        size_t n = units * (size_t)l.rows[j] * D;
        l.off_K[j] = o; o = align256(o + n * es);
        l.off_V[j] = o; o = align256(o + n * es);
        l.off_VS[j] = o; o = align256(o + n * 4);
        l.off_PK[j] = o; o = align256(o + units * D * 4);
        l.off_PV[j] = o; o = align256(o + units * D * 4);
    }
    l.off_Wt = o; o = align256(o + D * D * es);
    l.off_rope = o; o = align256(o + (size_t)l.npos * 3 * (D / 2) * 4);
    l.off_len = o; o = align256(o + units * 8);
    l.off_stats = o; o = align256(o + units * 3 * 8);
    l.off_err = o; o = align256(o + 4);
    l.off_stage = o; o = align256(o + (size_t)c->batch * 8);
    l.total = o;
    return l;
}

// Wt[c][r] = W[r][c], same element type (a copy, no rounding).
__global__ void pooler_transpose_kernel(const void* w, int bf16, int D, void* wt) {
    int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= D * D) return;
    int r = i / D, c = i % D;
    if (bf16)
        reinterpret_cast<__nv_bfloat16*>(wt)[c * D + r] = reinterpret_cast<const __nv_bfloat16*>(w)[i];
    else
        reinterpret_cast<float*>(wt)[c * D + r] = reinterpret_cast<const float*>(w)[i];
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

}  // namespace

#define DISPATCH_TD(dtype, D, ...)                                                        \
    do {                                                                                  \
        if ((dtype) == RECSA_BF16) {                                                      \
            using T = __nv_bfloat16;                                                      \
            if ((D) == 64) { constexpr int DD = 64; __VA_ARGS__; }                        \
            else { constexpr int DD = 128; __VA_ARGS__; }                                 \
        } else {                                                                          \
            using T = float;                                                              \
            if ((D) == 64) { constexpr int DD = 64; __VA_ARGS__; }                        \
            else { constexpr int DD = 128; __VA_ARGS__; }                                 \
        }                                                                                 \
    } while (0)

#define DISPATCH_G(G, ...)                                                                \
    do {                                                                                  \
        switch (G) {                                                                      \
            case 1: { constexpr int GG = 1; __VA_ARGS__; } break;                         \
            case 2: { constexpr int GG = 2; __VA_ARGS__; } break;                         \
            case 4: { constexpr int GG = 4; __VA_ARGS__; } break;                         \
            default: { constexpr int GG = 8; __VA_ARGS__; } break;                        \
        }                                                                                 \
    } while (0)

extern "C" {

const char* recsa_last_error(void) { return g_err.c_str(); }

size_t recsa_workspace_bytes(const recsa_config* cfg) {
    if (check_config(cfg) != RECSA_OK) return 0;
    return layout_for(cfg).total;
}

}  // extern "C"

namespace {
struct PageArgs {
    const int* table;
    int page_size, max_pages;
    long long num_pages;
};

recsa_status init_ctx(recsa_ctx** out, const recsa_config* cfg, void* k_cache, void* v_cache, void* workspace,
                      size_t workspace_bytes, const void* pooler_w, recsa_stream_t stream, const PageArgs* pg) {
    if (!out) return fail(RECSA_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    recsa_status st = check_config(cfg);
    if (st != RECSA_OK) return st;
    if (!k_cache || !v_cache || !workspace || !pooler_w) return fail(RECSA_ERR_INVALID_ARG, "NULL buffer");
    if (pg) {
        if (!pg->table) return fail(RECSA_ERR_INVALID_ARG, "NULL page table");
        if (pg->page_size < cfg->branching || pg->page_size % cfg->branching)
            return fail(RECSA_ERR_INVALID_ARG, "page_size %d must be a multiple of branching %d", pg->page_size,
                        cfg->branching);
        if (pg->max_pages < 1 || (long long)pg->max_pages * pg->page_size < cfg->capacity)
            return fail(RECSA_ERR_INVALID_ARG, "max_pages * page_size must cover the capacity");
        if (pg->num_pages < 1 || pg->num_pages >= (1LL << 31))
            return fail(RECSA_ERR_INVALID_ARG, "num_pages out of range");
    }
    if (!aligned(k_cache, 16) || !aligned(v_cache, 16)) return fail(RECSA_ERR_INVALID_ARG, "cache not 16-byte aligned");
    if (!aligned(workspace, 256)) return fail(RECSA_ERR_INVALID_ARG, "workspace not 256-byte aligned");
    Layout l = layout_for(cfg);
    {
        const int G = cfg->n_q_heads / cfg->n_kv_heads, elem = cfg->dtype == RECSA_BF16 ? 2 : 4;
        const size_t need = decode_smem_bytes(cfg->head_dim, G, elem, cfg->k, cfg->branching, l.J_cap, true);
        if (need > 227 * 1024)
            return fail(RECSA_ERR_UNSUPPORTED,
                        "k * branching = %d candidates per level need %zu bytes of decode shared memory (> 227 KB)",
                        cfg->k * cfg->branching, need);
    }
    if (workspace_bytes < l.total)
        return fail(RECSA_ERR_CAPACITY, "workspace has %zu bytes, needs %zu", workspace_bytes, l.total);

    recsa_ctx* c = new recsa_ctx();
    c->cfg = *cfg;
    c->G = cfg->n_q_heads / cfg->n_kv_heads;
    c->len.assign(cfg->batch, 0);
    TreeParams& p = c->p;
    memset(&p, 0, sizeof p);
    const int D = cfg->head_dim;
    char* ws = static_cast<char*>(workspace);
    p.B = cfg->batch; p.H = cfg->n_kv_heads; p.G = c->G; p.D = D; p.b = cfg->branching; p.k = cfg->k;
    p.J_cap = l.J_cap; p.npos = l.npos; p.cap = cfg->capacity;
    p.K[0] = k_cache; p.V[0] = v_cache;
    if (pg) {
        p.pages = pg->table;
        p.page_size = pg->page_size;
        p.max_pages = pg->max_pages;
        p.num_pages = pg->num_pages;
    }
    for (int j = 0; j <= MAXJ; j++) p.span[j] = span_sat(cfg->branching, j);
    p.rows[0] = cfg->capacity;
    for (int j = 1; j <= l.J_cap; j++) {
        p.rows[j] = l.rows[j];
        p.K[j] = ws + l.off_K[j];
        p.V[j] = ws + l.off_V[j];
        p.VS[j] = reinterpret_cast<float*>(ws + l.off_VS[j]);
        p.PK[j] = reinterpret_cast<float*>(ws + l.off_PK[j]);
        p.PV[j] = reinterpret_cast<float*>(ws + l.off_PV[j]);
    }
    p.Wt = ws + l.off_Wt;
    p.rope = reinterpret_cast<float*>(ws + l.off_rope);
    p.len = reinterpret_cast<long long*>(ws + l.off_len);
    p.stats = reinterpret_cast<long long*>(ws + l.off_stats);
    p.err = reinterpret_cast<int*>(ws + l.off_err);
    p.scale = (float)(1.0 / std::sqrt((double)D));
    c->len_stage = reinterpret_cast<long long*>(ws + l.off_stage);

    // RoPE table, fp64 on the host: row pos = [cos | sin | -sin](pos * base^(-2i/d)), i < d/2
    const int HD = D / 2;
    std::vector<float> tab((size_t)l.npos * 3 * HD);
    for (int pos = 0; pos < l.npos; pos++)
        for (int i = 0; i < HD; i++) {
            const double th = std::pow(cfg->rope_base, -2.0 * i / D);
            const float c = (float)std::cos(pos * th), sn = (float)std::sin(pos * th);
            float* row = tab.data() + (size_t)pos * 3 * HD;
            row[i] = c;
            row[HD + i] = sn;
            row[2 * HD + i] = -sn;
        }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync((void*)p.rope, tab.data(), tab.size() * sizeof(float), cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(p.len, 0, (size_t)p.B * p.H * 8, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(p.stats, 0, (size_t)p.B * p.H * 3 * 8, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(p.err, 0, 4, s);
    if (e == cudaSuccess) {
        pooler_transpose_kernel<<<(D * D + 255) / 256, 256, 0, s>>>(pooler_w, cfg->dtype == RECSA_BF16, D,
                                                                     const_cast<void*>(p.Wt));
        e = cudaGetLastError();
    }
    if (e != cudaSuccess) {
        delete c;
        return cuda_fail(e, "recsa_init");
    }
    *out = c;
    return RECSA_OK;
}
}  // namespace

extern "C" {

recsa_status recsa_init(recsa_ctx** out, const recsa_config* cfg, void* k_cache, void* v_cache, void* workspace,
                        size_t workspace_bytes, const void* pooler_w, recsa_stream_t stream) {
    return init_ctx(out, cfg, k_cache, v_cache, workspace, workspace_bytes, pooler_w, stream, nullptr);
}

recsa_status recsa_init_paged(recsa_ctx** out, const recsa_config* cfg, void* k_pool, void* v_pool,
                              long long num_pages, int page_size, const int* page_table, int max_pages,
                              void* workspace, size_t workspace_bytes, const void* pooler_w, recsa_stream_t stream) {
    const PageArgs pg{page_table, page_size, max_pages, num_pages};
    return init_ctx(out, cfg, k_pool, v_pool, workspace, workspace_bytes, pooler_w, stream, &pg);
}

void recsa_destroy(recsa_ctx* ctx) { delete ctx; }

recsa_status recsa_build_tree(recsa_ctx* ctx, const long long* lengths, recsa_stream_t stream) {
    if (!ctx || !lengths) return fail(RECSA_ERR_INVALID_ARG, "NULL argument");
    const recsa_config& c = ctx->cfg;
    long long maxL = 0;
    for (int b = 0; b < c.batch; b++) {
        if (lengths[b] < 0 || lengths[b] > c.capacity)
            return fail(RECSA_ERR_CAPACITY, "length %lld of sequence %d outside [0, %lld]", lengths[b], b, c.capacity);
        maxL = lengths[b] > maxL ? lengths[b] : maxL;
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(ctx->len_stage, lengths, (size_t)c.batch * 8, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = launch_set_lengths(ctx->p, ctx->len_stage, s);
    for (int j = 1; j <= ctx->p.J_cap && e == cudaSuccess; j++) {
        long long nodes = (maxL + ctx->p.span[j] - 1) / ctx->p.span[j];
        if (nodes == 0) continue;
        DISPATCH_TD(c.dtype, c.head_dim, e = launch_build_level<T, DD>(ctx->p, j, 0, 0, nodes, s));
    }
    if (e != cudaSuccess) return cuda_fail(e, "recsa_build_tree");
    for (int b = 0; b < c.batch; b++) ctx->len[b] = lengths[b];
    return RECSA_OK;
}

recsa_status recsa_append(recsa_ctx* ctx, const void* k_new, const void* v_new, int n, recsa_stream_t stream) {
    if (!ctx || !k_new || !v_new) return fail(RECSA_ERR_INVALID_ARG, "NULL argument");
    if (n < 1) return fail(RECSA_ERR_INVALID_ARG, "n must be >= 1");
    if (!aligned(k_new, 16) || !aligned(v_new, 16)) return fail(RECSA_ERR_INVALID_ARG, "k_new/v_new not 16-byte aligned");
    const recsa_config& c = ctx->cfg;
    long long maxL = 0, minL = c.capacity;
    for (int b = 0; b < c.batch; b++) {
        if (ctx->len[b] + n > c.capacity)
            return fail(RECSA_ERR_CAPACITY, "sequence %d: %lld + %d tokens exceed capacity %lld", b, ctx->len[b], n,
                        c.capacity);
        maxL = ctx->len[b] > maxL ? ctx->len[b] : maxL;
        minL = ctx->len[b] < minL ? ctx->len[b] : minL;
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaSuccess;
    if (n == 1) {
        DISPATCH_TD(c.dtype, c.head_dim, e = launch_append_one<T, DD>(ctx->p, k_new, v_new, s));
    } else {
        DISPATCH_TD(c.dtype, c.head_dim, e = launch_copy_tokens<T, DD>(ctx->p, k_new, v_new, n, s));
        for (int j = 1; j <= ctx->p.J_cap && e == cudaSuccess; j++) {
            const long long sp = ctx->p.span[j];
            long long nodes = (maxL + n + sp - 1) / sp - minL / sp;
            if (nodes < 1) nodes = 1;
            DISPATCH_TD(c.dtype, c.head_dim, e = launch_build_level<T, DD>(ctx->p, j, n, 1, nodes, s));
        }
        if (e == cudaSuccess) e = launch_bump_lengths(ctx->p, n, s);
    }
    if (e != cudaSuccess) return cuda_fail(e, "recsa_append");
    for (int b = 0; b < c.batch; b++) ctx->len[b] += n;
    return RECSA_OK;
}

recsa_status recsa_decode(recsa_ctx* ctx, const void* q, void* out, int* sel_out, long long* rows_out,
                          recsa_stream_t stream) {
    if (!ctx || !q || !out) return fail(RECSA_ERR_INVALID_ARG, "NULL argument");
    const recsa_config& c = ctx->cfg;
    for (int b = 0; b < c.batch; b++)
        if (ctx->len[b] < 1) return fail(RECSA_ERR_INVALID_ARG, "sequence %d holds no tokens", b);
    if (!aligned(q, 16) || !aligned(out, 16)) return fail(RECSA_ERR_INVALID_ARG, "q/out not 16-byte aligned");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaSuccess;
    DISPATCH_TD(c.dtype, c.head_dim,
                DISPATCH_G(ctx->G, e = launch_decode<T, DD, GG>(ctx->p, nullptr, nullptr, q, out, sel_out, rows_out, nullptr, s)));
    if (e != cudaSuccess) return cuda_fail(e, "recsa_decode");
    return RECSA_OK;
}

recsa_status recsa_append_decode(recsa_ctx* ctx, const void* k_new, const void* v_new, const void* q, void* out,
                                 int* sel_out, long long* rows_out, recsa_stream_t stream) {
    if (!ctx || !k_new || !v_new || !q || !out) return fail(RECSA_ERR_INVALID_ARG, "NULL argument");
    if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(q, 16) || !aligned(out, 16))
        return fail(RECSA_ERR_INVALID_ARG, "k_new/v_new/q/out not 16-byte aligned");
    const recsa_config& c = ctx->cfg;
    for (int b = 0; b < c.batch; b++)
        if (ctx->len[b] + 1 > c.capacity)
            return fail(RECSA_ERR_CAPACITY, "sequence %d: %lld + 1 tokens exceed capacity %lld", b, ctx->len[b],
                        c.capacity);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaSuccess;
    DISPATCH_TD(c.dtype, c.head_dim,
                DISPATCH_G(ctx->G, e = launch_decode<T, DD, GG>(ctx->p, k_new, v_new, q, out, sel_out, rows_out, nullptr, s)));
    if (e != cudaSuccess) return cuda_fail(e, "recsa_append_decode");
    for (int b = 0; b < c.batch; b++) ctx->len[b] += 1;
    return RECSA_OK;
}

namespace {
// Prefill scratch: [local softmax state: B C Hq (d + 2) fp32][rotated queries:
// B C Hq d bf16][rotated keys: B C H d bf16][the tree part's arrays], each
// 256-byte aligned.
struct PrefillScratch {
    size_t state, qr, kr, tree, total;
};
PrefillScratch prefill_scratch(const recsa_config* c, int C) {
    PrefillScratch s{};
    const size_t rows_q = (size_t)c->batch * C * c->n_q_heads, rows_k = (size_t)c->batch * C * c->n_kv_heads;
    s.state = 0;
    s.qr = align256(rows_q * (c->head_dim + 2) * sizeof(float));
    s.kr = s.qr + align256(rows_q * c->head_dim * 2);
    s.tree = s.kr + align256(rows_k * c->head_dim * 2);
    const Layout l = layout_for(c);
    TreeParams tp{};
    tp.B = c->batch;
    tp.H = c->n_kv_heads;
    tp.D = c->head_dim;
    tp.b = c->branching;
    tp.k = c->k;
    tp.J_cap = l.J_cap;
    for (int j = 0; j <= l.J_cap; j++) tp.rows[j] = l.rows[j];
    s.total = s.tree + align256(prefill_tree_scratch_bytes(tp, C, c->n_q_heads));
    return s;
}
}  // namespace

size_t recsa_prefill_scratch_bytes(const recsa_config* cfg, int C) {
    if (check_config(cfg) != RECSA_OK || C < 1) return 0;
    return prefill_scratch(cfg, C).total;
}

recsa_status recsa_prefill(recsa_ctx* ctx, const void* q, const void* k, const void* v, int C, void* out,
                           int* sel_out, long long* rows_out, void* scratch, size_t scratch_bytes,
                           recsa_stream_t stream) {
    if (!ctx || !q || !k || !v || !out || !scratch) return fail(RECSA_ERR_INVALID_ARG, "NULL argument");
    const recsa_config& c = ctx->cfg;
    if (c.dtype != RECSA_BF16) return fail(RECSA_ERR_UNSUPPORTED, "prefill is built for bf16 storage only");
    if (C < 1 || C > c.max_chunk) return fail(RECSA_ERR_INVALID_ARG, "chunk %d outside [1, max_chunk=%d]", C, c.max_chunk);
    for (int b = 0; b < c.batch; b++)
        if (ctx->len[b] + C > c.capacity)
            return fail(RECSA_ERR_CAPACITY, "sequence %d: %lld + %d tokens exceed capacity %lld", b, ctx->len[b], C,
                        c.capacity);
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16))
        return fail(RECSA_ERR_INVALID_ARG, "q/k/v/out not 16-byte aligned");
    if (!aligned(scratch, 256)) return fail(RECSA_ERR_INVALID_ARG, "scratch not 256-byte aligned");
    const size_t need = recsa_prefill_scratch_bytes(&c, C);
    if (scratch_bytes < need) return fail(RECSA_ERR_CAPACITY, "scratch has %zu bytes, needs %zu", scratch_bytes, need);
    if (!prefill_tree_supported(c.head_dim, c.branching))
        return fail(RECSA_ERR_UNSUPPORTED, "prefill needs branching rounded up to 32 <= min(head_dim, 128)");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const PrefillScratch ps = prefill_scratch(&c, C);
    char* sc = static_cast<char*>(scratch);
    float* state = reinterpret_cast<float*>(sc + ps.state);
    cudaError_t e;
    if (c.head_dim == 64)
        e = launch_prefill_attn<64>(ctx->p, q, k, v, state, sc + ps.qr, sc + ps.kr, c.batch, C, c.n_q_heads,
                                    c.n_kv_heads, s);
    else
        e = launch_prefill_attn<128>(ctx->p, q, k, v, state, sc + ps.qr, sc + ps.kr, c.batch, C, c.n_q_heads,
                                     c.n_kv_heads, s);
    if (e == cudaSuccess) {
        void* tree = sc + ps.tree;
        const long long* lens = ctx->len.data();
        if (c.head_dim == 64) {
            constexpr int DD = 64;
            DISPATCH_G(ctx->G, e = launch_prefill_tree_tc<DD, GG>(ctx->p, q, out, state, sel_out, rows_out, C,
                                                                  c.n_q_heads, lens, tree, s));
        } else {
            constexpr int DD = 128;
            DISPATCH_G(ctx->G, e = launch_prefill_tree_tc<DD, GG>(ctx->p, q, out, state, sel_out, rows_out, C,
                                                                  c.n_q_heads, lens, tree, s));
        }
    }
    if (e != cudaSuccess) return cuda_fail(e, "recsa_prefill");
    return RECSA_OK;
}

recsa_status recsa_get_lengths(const recsa_ctx* ctx, long long* lengths) {
    if (!ctx || !lengths) return fail(RECSA_ERR_INVALID_ARG, "NULL argument");
    for (int b = 0; b < ctx->cfg.batch; b++) lengths[b] = ctx->len[b];
    return RECSA_OK;
}

recsa_status recsa_tree_shape(const recsa_ctx* ctx, int* j_cap, long long* rows) {
    if (!ctx || !j_cap) return fail(RECSA_ERR_INVALID_ARG, "NULL argument");
    *j_cap = ctx->p.J_cap;
    if (rows)
        for (int j = 0; j <= ctx->p.J_cap; j++) rows[j] = ctx->p.rows[j];
    return RECSA_OK;
}

recsa_status recsa_level_arrays(const recsa_ctx* ctx, int level, void** keys, void** values, float** value_sums) {
    if (!ctx) return fail(RECSA_ERR_INVALID_ARG, "NULL context");
    if (level < 1 || level > ctx->p.J_cap) return fail(RECSA_ERR_INVALID_ARG, "level %d outside [1, %d]", level,
                                                       ctx->p.J_cap);
    if (keys) *keys = ctx->p.K[level];
    if (values) *values = ctx->p.V[level];
    if (value_sums) *value_sums = ctx->p.VS[level];
    return RECSA_OK;
}

recsa_status recsa_query_stats(recsa_ctx* ctx, int* depth, long long* k_rows, long long* v_rows,
                               recsa_stream_t stream) {
    if (!ctx) return fail(RECSA_ERR_INVALID_ARG, "NULL context");
    const size_t units = (size_t)ctx->p.B * ctx->p.H;
    std::vector<long long> st(units * 3);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(s);
    if (e == cudaSuccess) e = cudaMemcpy(st.data(), ctx->p.stats, units * 3 * 8, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "recsa_query_stats");
    for (size_t u = 0; u < units; u++) {
        if (depth) depth[u] = (int)st[u * 3];
        if (k_rows) k_rows[u] = st[u * 3 + 1];
        if (v_rows) v_rows[u] = st[u * 3 + 2];
    }
    return RECSA_OK;
}

recsa_status recsa_check_device(recsa_ctx* ctx, recsa_stream_t stream) {
    if (!ctx) return fail(RECSA_ERR_INVALID_ARG, "NULL context");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "recsa_check_device");
    int word = 0;
    e = cudaMemcpy(&word, ctx->p.err, 4, cudaMemcpyDeviceToHost);
    if (e == cudaSuccess) e = cudaMemset(ctx->p.err, 0, 4);
    if (e != cudaSuccess) return cuda_fail(e, "recsa_check_device");
    if (word) return fail(RECSA_ERR_DEVICE, "device error word 0x%x (1: length, 2: shape, 4: timeout)", word);
    return RECSA_OK;
}

size_t recsa_dense_decode_scratch_bytes(int batch, int n_q_heads, int head_dim) {
    if (batch < 1 || n_q_heads < 1 || head_dim < 1) return 0;
    return (size_t)batch * n_q_heads * 256 * (head_dim + 2) * sizeof(float);
}

recsa_status recsa_dense_decode(const void* k_cache, const void* v_cache, const void* q, void* out, int batch,
                                int n_kv_heads, int n_q_heads, int head_dim, long long length, long long l_stride,
                                recsa_dtype dtype, void* scratch, size_t scratch_bytes, recsa_stream_t stream) {
    if (!k_cache || !v_cache || !q || !out || !scratch) return fail(RECSA_ERR_INVALID_ARG, "NULL argument");
    if (batch < 1 || n_kv_heads < 1 || n_q_heads % n_kv_heads) return fail(RECSA_ERR_INVALID_ARG, "bad head counts");
    int G = n_q_heads / n_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return fail(RECSA_ERR_UNSUPPORTED, "group size %d", G);
    if (head_dim != 64 && head_dim != 128) return fail(RECSA_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
    if (length < 1 || l_stride < length) return fail(RECSA_ERR_INVALID_ARG, "bad length / stride");
    if (scratch_bytes < recsa_dense_decode_scratch_bytes(batch, n_q_heads, head_dim))
        return fail(RECSA_ERR_CAPACITY, "scratch too small");
    if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(q, 16))
        return fail(RECSA_ERR_INVALID_ARG, "buffers not 16-byte aligned");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaSuccess;
    const int units = batch * n_kv_heads;
    DISPATCH_TD(dtype, head_dim,
                DISPATCH_G(G, e = launch_dense<T, DD, GG>(k_cache, v_cache, q, out, units, length, l_stride,
                                                         static_cast<float*>(scratch), 256, s)));
    if (e != cudaSuccess) return cuda_fail(e, "recsa_dense_decode");
    return RECSA_OK;
}

recsa_status recsa_dense_decode_static(const void* k_cache, const void* v_cache, const void* q, void* out, int batch,
                                       int n_kv_heads, int n_q_heads, int head_dim, long long length,
                                       long long l_stride, recsa_dtype dtype, recsa_stream_t stream) {
    if (!k_cache || !v_cache || !q || !out) return fail(RECSA_ERR_INVALID_ARG, "NULL argument");
    if (batch < 1 || n_kv_heads < 1 || n_q_heads % n_kv_heads) return fail(RECSA_ERR_INVALID_ARG, "bad head counts");
    int G = n_q_heads / n_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return fail(RECSA_ERR_UNSUPPORTED, "group size %d", G);
    if (head_dim != 64 && head_dim != 128) return fail(RECSA_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
    if (dtype != RECSA_F32 && dtype != RECSA_BF16) return fail(RECSA_ERR_INVALID_ARG, "unknown dtype");
    if (length < 1 || l_stride < length) return fail(RECSA_ERR_INVALID_ARG, "bad length / stride");
    if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(q, 16))
        return fail(RECSA_ERR_INVALID_ARG, "buffers not 16-byte aligned");
    const int units = batch * n_kv_heads;
    const size_t per_split = (size_t)units * G * (head_dim + 2) * sizeof(float);
    const size_t limit = dense_static_scratch_bytes();
    if (per_split > limit)
        return fail(RECSA_ERR_CAPACITY,
                    "batch * n_q_heads = %d needs %zu bytes of scratch per split; the fixed scratch holds %zu bytes",
                    batch * n_q_heads, per_split, limit);
    const int max_splits = (int)(limit / per_split);
    float* scratch = nullptr;
    cudaError_t e = dense_static_scratch(&scratch);
    if (e != cudaSuccess) return cuda_fail(e, "recsa_dense_decode_static: scratch address");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    DISPATCH_TD(dtype, head_dim,
                DISPATCH_G(G, e = launch_dense<T, DD, GG>(k_cache, v_cache, q, out, units, length, l_stride, scratch,
                                                         max_splits < 256 ? max_splits : 256, s)));
    if (e != cudaSuccess) return cuda_fail(e, "recsa_dense_decode_static");
    return RECSA_OK;
}

}  // extern "C"

// ------------------------------------------------------------ backward

namespace {
// Backward scratch: [node-key accumulators, levels 1..J_cap][node-value
// accumulators, levels 1..J_cap] (fp32, [B*H][rows[j]][d] each; the prefix
// the tree pass clears) then W^T h per node of levels 2..J_cap (written
// before it is read), the per-call plan, logits, <dout, v> and softmax
// statistics.
struct BwdLayout {
    size_t gK[MAXJ + 1], gV[MAXJ + 1], gW[MAXJ + 1], nodes_end, plan, ubase, lg, ag, st, total;
    int E_cap;
};
BwdLayout bwd_layout(const recsa_config* c) {
    BwdLayout b{};
    const Layout l = layout_for(c);
    const size_t units = (size_t)c->batch * c->n_kv_heads, D = c->head_dim;
    const size_t G = (size_t)(c->n_q_heads / c->n_kv_heads);
    size_t o = 0;
    for (int j = 1; j <= l.J_cap; j++) { b.gK[j] = o; o = align256(o + units * (size_t)l.rows[j] * D * 4); }
    for (int j = 1; j <= l.J_cap; j++) { b.gV[j] = o; o = align256(o + units * (size_t)l.rows[j] * D * 4); }
    b.nodes_end = o;
    for (int j = 2; j <= l.J_cap; j++) { b.gW[j] = o; o = align256(o + units * (size_t)l.rows[j] * D * 4); }
    long long maxc = (long long)c->k * c->branching;
    if (maxc < c->branching) maxc = c->branching;
    b.E_cap = (int)((l.J_cap + 1) * maxc);
    b.plan = o; o = align256(o + units * PLAN_INTS * 4);
    b.ubase = o; o = align256(o + (units + 1) * 4);
    b.lg = o; o = align256(o + units * (size_t)b.E_cap * G * 4);
    b.ag = o; o = align256(o + units * (size_t)b.E_cap * G * 4);
    b.st = o; o = align256(o + units * G * 3 * 4);
    b.total = o;
    return b;
}
BwdArgs bwd_args(const recsa_ctx* ctx, void* scratch) {
    const BwdLayout l = bwd_layout(&ctx->cfg);
    char* base = static_cast<char*>(scratch);
    BwdArgs a{};
    for (int j = 1; j <= ctx->p.J_cap; j++) {
        a.gK[j] = reinterpret_cast<float*>(base + l.gK[j]);
        a.gV[j] = reinterpret_cast<float*>(base + l.gV[j]);
        if (j >= 2) a.gW[j] = reinterpret_cast<float*>(base + l.gW[j]);
    }
    a.plan = reinterpret_cast<int*>(base + l.plan);
    a.ubase = reinterpret_cast<int*>(base + l.ubase);
    a.lg = reinterpret_cast<float*>(base + l.lg);
    a.ag = reinterpret_cast<float*>(base + l.ag);
    a.st = reinterpret_cast<float*>(base + l.st);
    a.E_cap = l.E_cap;
    return a;
}
}  // namespace

extern "C" {

size_t recsa_backward_scratch_bytes(const recsa_config* cfg) {
    if (check_config(cfg) != RECSA_OK) return 0;
    return bwd_layout(cfg).total;
}

recsa_status recsa_decode_backward(recsa_ctx* ctx, const void* q, const void* dout, const int* sel, float* dq,
                                   float* dk, float* dv, void* scratch, size_t scratch_bytes, recsa_stream_t stream) {
    if (!ctx || !q || !dout || !sel || !dq || !dk || !dv || !scratch) return fail(RECSA_ERR_INVALID_ARG, "NULL argument");
    if (!aligned(q, 16) || !aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16))
        return fail(RECSA_ERR_INVALID_ARG, "q/dout/dq/dk/dv not 16-byte aligned");
    if (!aligned(scratch, 256)) return fail(RECSA_ERR_INVALID_ARG, "scratch not 256-byte aligned");
    const recsa_config& c = ctx->cfg;
    if (scratch_bytes < bwd_layout(&c).total)
        return fail(RECSA_ERR_INVALID_ARG, "scratch of %zu bytes, %zu needed", scratch_bytes, bwd_layout(&c).total);
    for (int b = 0; b < c.batch; b++)
        if (ctx->len[b] < 1) return fail(RECSA_ERR_INVALID_ARG, "sequence %d holds no tokens", b);
    BwdArgs a = bwd_args(ctx, scratch);
    a.q = q;
    a.dout = dout;
    a.sel = sel;
    a.dq = dq;
    a.dk = dk;
    a.dv = dv;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaSuccess;
    DISPATCH_TD(c.dtype, c.head_dim, DISPATCH_G(ctx->G, e = launch_decode_backward<T, DD, GG>(ctx->p, a, s)));
    if (e != cudaSuccess) return cuda_fail(e, "recsa_decode_backward");
    return RECSA_OK;
}

recsa_status recsa_tree_backward(recsa_ctx* ctx, float* dk, float* dv, float* dw, void* scratch,
                                 size_t scratch_bytes, recsa_stream_t stream) {
    if (!ctx || !dk || !dv || !dw || !scratch) return fail(RECSA_ERR_INVALID_ARG, "NULL argument");
    if (!aligned(dk, 16) || !aligned(dv, 16) || !aligned(dw, 16))
        return fail(RECSA_ERR_INVALID_ARG, "dk/dv/dw not 16-byte aligned");
    if (!aligned(scratch, 256)) return fail(RECSA_ERR_INVALID_ARG, "scratch not 256-byte aligned");
    const recsa_config& c = ctx->cfg;
    const BwdLayout l = bwd_layout(&c);
    if (scratch_bytes < l.total) return fail(RECSA_ERR_INVALID_ARG, "scratch of %zu bytes, %zu needed", scratch_bytes, l.total);
    BwdArgs a = bwd_args(ctx, scratch);
    a.dk = dk;
    a.dv = dv;
    a.dw = dw;
    long long maxL = 0;
    for (int b = 0; b < c.batch; b++) maxL = ctx->len[b] > maxL ? ctx->len[b] : maxL;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaSuccess;
    if (maxL > 0) DISPATCH_TD(c.dtype, c.head_dim, e = launch_tree_backward<T, DD>(ctx->p, a, maxL, s));
    if (e == cudaSuccess) e = cudaMemsetAsync(scratch, 0, l.nodes_end, s);
    if (e != cudaSuccess) return cuda_fail(e, "recsa_tree_backward");
    return RECSA_OK;
}

}  // extern "C"

// ------------------------------------------------------------ distillation

namespace {
// Distillation scratch: [the backward scratch][fp32 output B Hq d][its
// gradient B Hq d][dq B Hq d][selections B H J_cap k int32][dW d d][loss].
struct DistillLayout {
    BwdLayout bwd;
    size_t out, dout, dq, sel, dw, loss, total;
};
DistillLayout distill_layout(const recsa_config* c) {
    DistillLayout d{};
    d.bwd = bwd_layout(c);
    const size_t n = (size_t)c->batch * c->n_q_heads * c->head_dim;
    const Layout l = layout_for(c);
    size_t o = d.bwd.total;
    d.out = o; o = align256(o + n * 4);
    d.dout = o; o = align256(o + n * 4);
    d.dq = o; o = align256(o + n * 4);
    d.sel = o; o = align256(o + (size_t)c->batch * c->n_kv_heads * l.J_cap * c->k * 4);
    d.dw = o; o = align256(o + (size_t)c->head_dim * c->head_dim * 4);
    d.loss = o; o = align256(o + 4);
    d.total = o;
    return d;
}
}  // namespace

extern "C" {

size_t recsa_distill_scratch_bytes(const recsa_config* cfg) {
    if (check_config(cfg) != RECSA_OK) return 0;
    return distill_layout(cfg).total;
}

recsa_status recsa_distill_step(recsa_ctx* ctx, const void* q, const float* target, float lr, float* w_master,
                                float* loss, float* dw_out, void* scratch, size_t scratch_bytes,
                                recsa_stream_t stream) {
    if (!ctx || !q || !target || !w_master || !scratch) return fail(RECSA_ERR_INVALID_ARG, "NULL argument");
    if (!aligned(q, 16) || !aligned(target, 16)) return fail(RECSA_ERR_INVALID_ARG, "q/target not 16-byte aligned");
    if (!aligned(scratch, 256)) return fail(RECSA_ERR_INVALID_ARG, "scratch not 256-byte aligned");
    if (!(lr >= 0.f)) return fail(RECSA_ERR_INVALID_ARG, "lr must be >= 0");
    const recsa_config& c = ctx->cfg;
    const DistillLayout l = distill_layout(&c);
    if (scratch_bytes < l.total) return fail(RECSA_ERR_INVALID_ARG, "scratch of %zu bytes, %zu needed", scratch_bytes, l.total);
    long long maxL = 0;
    for (int b = 0; b < c.batch; b++) {
        if (ctx->len[b] < 1) return fail(RECSA_ERR_INVALID_ARG, "sequence %d holds no tokens", b);
        maxL = ctx->len[b] > maxL ? ctx->len[b] : maxL;
    }
    char* base = static_cast<char*>(scratch);
    float* out = reinterpret_cast<float*>(base + l.out);
    float* dout = reinterpret_cast<float*>(base + l.dout);
    int* sel = reinterpret_cast<int*>(base + l.sel);
    float* dw = reinterpret_cast<float*>(base + l.dw);
    float* lossd = reinterpret_cast<float*>(base + l.loss);
    const long long n = (long long)c.batch * c.n_q_heads * c.head_dim;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // node accumulators, dW and the loss start at zero
    cudaError_t e = cudaMemsetAsync(scratch, 0, l.bwd.nodes_end, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(dw, 0, (size_t)c.head_dim * c.head_dim * 4, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(lossd, 0, 4, s);
    // forward (fp32 output, selections kept), loss and its gradient
    if (e == cudaSuccess)
        DISPATCH_TD(c.dtype, c.head_dim,
                    DISPATCH_G(ctx->G, e = launch_decode<T, DD, GG>(ctx->p, nullptr, nullptr, q, nullptr, sel,
                                                                    nullptr, out, s)));
    if (e == cudaSuccess) e = launch_distill_loss(out, target, dout, lossd, n, s);
    // the pooler's gradient only: no token gradients
    BwdArgs a = bwd_args(ctx, scratch);
    a.q = q;
    a.dout = dout;
    a.dout_f32 = 1;
    a.sel = sel;
    a.dq = reinterpret_cast<float*>(base + l.dq);
    a.dk = nullptr;
    a.dv = nullptr;
    a.dw = dw;
    if (e == cudaSuccess)
        DISPATCH_TD(c.dtype, c.head_dim, DISPATCH_G(ctx->G, e = launch_decode_backward<T, DD, GG>(ctx->p, a, s)));
    if (e == cudaSuccess) DISPATCH_TD(c.dtype, c.head_dim, e = launch_tree_backward<T, DD>(ctx->p, a, maxL, s));
    // update, then every node key again under the new pooler
    if (e == cudaSuccess) {
        if (c.dtype == RECSA_BF16)
            e = launch_pooler_update<__nv_bfloat16>(w_master, dw, lr, const_cast<void*>(ctx->p.Wt), dw_out,
                                                    c.head_dim, s);
        else
            e = launch_pooler_update<float>(w_master, dw, lr, const_cast<void*>(ctx->p.Wt), dw_out, c.head_dim, s);
    }
    for (int j = 1; j <= ctx->p.J_cap && e == cudaSuccess; j++) {
        const long long nodes = (maxL + ctx->p.span[j] - 1) / ctx->p.span[j];
        if (nodes == 0) continue;
        DISPATCH_TD(c.dtype, c.head_dim, e = launch_build_level<T, DD>(ctx->p, j, 0, 0, nodes, s));
    }
    if (e == cudaSuccess && loss) e = cudaMemcpyAsync(loss, lossd, 4, cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, "recsa_distill_step");
    return RECSA_OK;
}

}  // extern "C"

// ------------------------------------------------------------ clustered order

namespace {
// Levels of the tree over L >= 1 tokens (the first j >= 1 with ceil(L / b^j) <= b).
int levels_of(long long L, int b) {
    int j = 1;
    long long s = b;
    while (j < MAXJ && (L + s - 1) / s > b) {
        s = s > LLONG_MAX / b ? LLONG_MAX : s * b;
        j++;
    }
    return j;
}
}  // namespace

extern "C" {

size_t recsa_cluster_scratch_bytes(const recsa_config* cfg) {
    if (check_config(cfg) != RECSA_OK) return 0;
    const long long units = (long long)cfg->batch * cfg->n_kv_heads;
    return align256(cluster_rec_bytes(units, cfg->capacity)) + align256((size_t)(cfg->batch + 1) * 8);
}

recsa_status recsa_cluster_load(recsa_ctx* ctx, const void* k_src, const void* v_src, long long src_len,
                                const long long* lengths, const float* Z, int* perm, void* scratch,
                                size_t scratch_bytes, recsa_stream_t stream) {
    if (!ctx || !k_src || !v_src || !lengths || !Z || !perm || !scratch)
        return fail(RECSA_ERR_INVALID_ARG, "NULL argument");
    if (!aligned(k_src, 16) || !aligned(v_src, 16) || !aligned(Z, 16) || !aligned(perm, 4))
        return fail(RECSA_ERR_INVALID_ARG, "k_src/v_src/Z not 16-byte or perm not 4-byte aligned");
    if (!aligned(scratch, 256)) return fail(RECSA_ERR_INVALID_ARG, "scratch not 256-byte aligned");
    if (ctx->p.pages) return fail(RECSA_ERR_UNSUPPORTED, "the clustered order needs a contiguous cache");
    const recsa_config& c = ctx->cfg;
    if (scratch_bytes < recsa_cluster_scratch_bytes(&c))
        return fail(RECSA_ERR_INVALID_ARG, "scratch of %zu bytes, %zu needed", scratch_bytes,
                    recsa_cluster_scratch_bytes(&c));
    if (src_len < 1 || src_len > INT_MAX) return fail(RECSA_ERR_INVALID_ARG, "src_len %lld outside [1, 2^31)", src_len);
    std::vector<long long> sstart((size_t)c.batch + 1, 0);
    int J_max = 0;
    for (int b = 0; b < c.batch; b++) {
        if (lengths[b] < 0 || lengths[b] > c.capacity || lengths[b] > src_len)
            return fail(RECSA_ERR_CAPACITY, "length %lld of sequence %d outside [0, min(capacity, src_len)]",
                        lengths[b], b);
        sstart[b + 1] = sstart[b] + lengths[b];
        if (lengths[b] > 0) J_max = std::max(J_max, levels_of(lengths[b], c.branching));
    }
    const long long n = (long long)c.n_kv_heads * sstart[c.batch];
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaSuccess;
    if (n > 0) {
        char* base = static_cast<char*>(scratch);
        long long* sstart_dev =
            reinterpret_cast<long long*>(base + align256(cluster_rec_bytes((long long)c.batch * c.n_kv_heads, c.capacity)));
        e = cudaMemcpyAsync(sstart_dev, sstart.data(), sstart.size() * 8, cudaMemcpyHostToDevice, s);
        if (e == cudaSuccess)
            DISPATCH_TD(c.dtype, c.head_dim,
                        e = launch_cluster<T, DD>(ctx->p, k_src, v_src, src_len, Z, sstart_dev, n, J_max, perm, base, s));
        if (e != cudaSuccess) return cuda_fail(e, "recsa_cluster_load");
    }
    return recsa_build_tree(ctx, lengths, stream);
}

}  // extern "C"
