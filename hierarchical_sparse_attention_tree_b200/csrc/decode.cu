// Fused decode: per-level scoring + top-k descent + shared-softmax gather
// attention, one thread-block cluster per (sequence, KV head) unit.
//
// Method (RecSA abstract; kongchang.com article "Core Idea", "Position
// Encoding"): each level above the tokens keeps at most k candidates; the
// query filters at the top level and drills down through the children of the
// kept nodes; summaries of the candidates that were not kept share one
// softmax with the exact tokens under the kept level-1 nodes; every entry is
// RoPE-rotated at its index among its level's candidates and the query at the
// last index of that level. GQA: the G query heads of a KV head share one
// selection ranked by the sum of their logits.
//
// Work split and data movement. A level's candidates are the children of the
// kept parents, in ascending node order; each parent's children are one
// contiguous block of rows. The CS CTAs of the cluster take contiguous rank
// ranges of that list and bring their key and value rows into shared memory
// with 1D bulk async copies (one per contiguous piece, completion counted on
// an mbarrier), so all of a CTA's rows are in flight at once. Each CTA scores
// its range, ranks its keys to get a local top-k, and the CTAs exchange those
// lists through distributed shared memory; every CTA then derives the same
// global top-k (keys are unique: score, then node id), so one cluster barrier
// per level is the only wait on another CTA. The next level's key rows are
// requested as soon as the selection is known, while this level's summaries
// are accumulated. A level with at most k candidates keeps them all: it is
// neither read nor scored (same result, fewer bytes). RoPE at index r*b + o:
// the key is rotated by o and the query by P - r*b (only the angle difference
// enters a logit), so the keys use b table rows however long the lists are.
#include <cooperative_groups.h>

#include "append.cuh"
#include "common.cuh"
#include "score.cuh"

namespace cg = cooperative_groups;

namespace recsa {

constexpr int DEC_THREADS = 256;
constexpr int DEC_WARPS = DEC_THREADS / 32;
constexpr int DEC_CLUSTER = 8;
constexpr int KMAX = 64;

struct DecodeArgs {
    const void* k_new;    // nullable [B][H][D]: append this token first (fused step)
    const void* v_new;
    const void* q;
    void* out;
    float* out_f32;       // nullable [B][Hq][D]: the output in fp32 instead of `out`
    int* sel_out;         // nullable [B*H][J_cap][k]
    long long* rows_out;  // nullable [B*H][2]
    int my_max;           // candidates per CTA, upper bound
    int region0;          // bytes of the K/V tile region (reused for the warp merge)
};

// Where a paged cache keeps this unit's tokens (set up once per CTA).
struct DecPages {
    const int* row;  // the sequence's page table row
    int psize, nheads, head, npages;
};

struct DecSmem {
    uint64_t bar[3];                     // [0]: key tile, [1]: value tile, [2]: pooler (append)
    DecPages pg;                         // paged cache (row null: contiguous)
    TokenMap tok;                        // where the token rows live (for the append)
    unsigned long long wl[DEC_WARPS][KMAX];  // per-warp top-k lists, sorted, zero padded
    unsigned long long picked[KMAX];     // global top-k keys, best first
    unsigned long long thresh;           // the k-th best key
    int par[KMAX];                       // kept parents of the current level, ascending
    int chosen[KMAX];                    // kept nodes of the current level, ascending
    int nlev[MAXJ + 1];                  // nodes per level over L tokens
    LevelRef lv[MAXJ + 1];               // the levels' addresses
    float red[DEC_WARPS][8];             // per-warp partial maxima / sums (G <= 8)
    float M[8];                          // running softmax maximum per head (this CTA)
};

// Softmax-value accumulation layout: thread t owns CPT output columns
// (chunk t % NCC) of one entry group (t / NCC) for every head.
constexpr int CPT = 4;

template <int D>
__host__ __device__ constexpr int dec_ncc() { return D / CPT; }
template <int D>
__host__ __device__ constexpr int dec_neg() { return DEC_THREADS / (D / CPT); }

// Shared memory: [region0: K tile | V tile; at the end: entry-group partials]
// [DecSmem][key: u64 MY][gkeys: u64 2*CS*KMAX][qf G*D][lg MY*G (logits, then
// softmax weights)][cacc G*D][cml 2G][gat: (rank 0) the CTAs' states CS*(G*D + 2G)]
__host__ __device__ inline size_t decode_smem_tail(int D, int G, int MY) {
    return sizeof(DecSmem) + (size_t)MY * 8 + (size_t)2 * DEC_CLUSTER * KMAX * 8 +
           (size_t)(G * D + MY * G + G * D + 2 * G) * 4 + (size_t)DEC_CLUSTER * (G * D + 2 * G) * 4;
}
__host__ __device__ inline size_t decode_region0(int D, int G, int MY, int elem, int J_cap, bool fused) {
    // the appending CTA of a fused step first holds the pooler and the
    // append scratch here
    const size_t app = fused ? (((size_t)D * D * elem + append_scratch_floats(D, J_cap) * 4 + 127) & ~(size_t)127) +
                                   128 + 4 * (size_t)D * elem + 128
                             : 0;
    const size_t tiles0 = 2 * (size_t)MY * D * elem;
    const size_t tiles = tiles0 > app ? tiles0 : app;
    const size_t eg = (size_t)(DEC_THREADS / (D / CPT)) * G * D * 4;
    const size_t eg_al = (eg + 127) & ~(size_t)127;
    const size_t need = eg_al;
    const size_t r0 = tiles > need ? tiles : need;
    return (r0 + 127) & ~(size_t)127;
}

// Number of keys in key[0..n) greater than kt (keys in shared memory).
__device__ __forceinline__ int rank_among(const unsigned long long* key, int n, unsigned long long kt) {
    int r0 = 0, r1 = 0, r2 = 0, r3 = 0;
    int x = 0;
    for (; x + 4 <= n; x += 4) {
        r0 += key[x] > kt;
        r1 += key[x + 1] > kt;
        r2 += key[x + 2] > kt;
        r3 += key[x + 3] > kt;
    }
    for (; x < n; x++) r0 += key[x] > kt;
    return (r0 + r1) + (r2 + r3);
}

// Sorts one key per lane in descending order across the warp (bitonic network).
__device__ __forceinline__ unsigned long long warp_sort_desc(unsigned long long x, int lane) {
#pragma unroll 1
    for (int k2 = 2; k2 <= 32; k2 <<= 1)
#pragma unroll 1
        for (int j2 = k2 >> 1; j2 > 0; j2 >>= 1) {
            const unsigned long long y = __shfl_xor_sync(0xffffffffu, x, j2);
            const bool desc = (lane & k2) == 0, lower = (lane & j2) == 0;
            x = (lower == desc) ? (x > y ? x : y) : (x < y ? x : y);
        }
    return x;
}

// Rank of key x among NL lists (list l at lists + l*stride, n keys each,
// sorted descending, zero padded): the number of keys greater than x, by one
// binary search per list, all lists advancing together. Keys are distinct.
template <int NL>
__device__ __forceinline__ int rank_in_lists(const unsigned long long* lists, int stride, int n,
                                             unsigned long long x) {
    int cnt[NL];
#pragma unroll
    for (int l = 0; l < NL; l++) cnt[l] = 0;
#pragma unroll 1
    for (int st = KMAX; st >= 1; st >>= 1) {
        if (st > n) continue;  // uniform: n is the same in every thread
        // every probe is a load at a valid index (clamped), so the NL loads of
        // a round are independent of each other
#pragma unroll
        for (int l = 0; l < NL; l++) {
            const int pos = cnt[l] + st;
            const unsigned long long y = lists[l * stride + min(pos, n) - 1];
            cnt[l] = (pos <= n && y > x) ? pos : cnt[l];
        }
    }
    int r = 0;
#pragma unroll
    for (int l = 0; l < NL; l++) r += cnt[l];
    return r;
}

// Thread 0: request rows [r0, r1) of a level's candidate list (the children
// of the kept parents par[], b per parent, n_j nodes in the level) from the
// node rows at `base` into dst, one 1D bulk copy per contiguous piece, all
// counted on one mbarrier. Out-of-range pieces are flagged, not copied.
// (Inline: as an out-of-line call it cost a register spill around every call
// site and about a microsecond per step.)
template <typename T, int D>
__device__ __forceinline__ void issue_rows(T* dst, const T* base, const int* par, int n_j, int b, int r0, int r1,
                                        uint64_t* bar, int* err, const DecPages* pg) {
    // pg set (level 0 of a paged cache): base is the pool and each piece
    // (part of one parent's children, which lie in one page) is translated;
    // else base is the unit's first row
    auto src = [&](int id0) {
        if (!pg) return base + (size_t)id0 * D;
        int page = pg->row[id0 / pg->psize];
        if (page < 0 || page >= pg->npages) {
            flag_error(err, ERR_SHAPE);
            page = 0;
        }
        return base + (((size_t)page * pg->nheads + pg->head) * pg->psize + id0 % pg->psize) * D;
    };
    const int pr = r0 / b, o0 = r0 - pr * b;
    uint32_t total = 0;
    for (int r = r0, q = pr, o = o0; r < r1; q++, o = 0) {
        const int n = min(b - o, r1 - r);
        const int id0 = par[q] * b + o;
        if (id0 >= 0 && id0 + n <= n_j) total += (uint32_t)(n * D * sizeof(T));
        r += n;
    }
    if (r1 > r0) {  // (an empty request only completes the barrier's phase: nothing to order)
        fence_proxy_async_shared();
        fence_proxy_async_global();  // global writes of a fused append seen by the bulk reads
    }
    mbar_arrive_expect_tx(bar, total);
    for (int r = r0, q = pr, o = o0; r < r1; q++, o = 0) {
        const int n = min(b - o, r1 - r);
        const int id0 = par[q] * b + o;
        if (id0 >= 0 && id0 + n <= n_j)
            bulk_g2s(dst + (size_t)(r - r0) * D, src(id0), (uint32_t)(n * D * sizeof(T)), bar);
        else
            flag_error(err, ERR_SHAPE);
        r += n;
    }
}

// The fused step's append (inline: out of line, its call cost the step about
// a microsecond of register spills and an instruction fetch): appends the
// token of unit u at position P, leaves the refreshed node of level jf (the
// first scored level; jf = 0: the token itself) in patch[0..D) (key) and
// patch[D..2D) (value), and makes its global writes visible to later bulk
// reads (fence = false: the caller fences later, before this CTA's next
// bulk read and before other CTAs may read the appended rows). Every thread
// of the block calls it. False if the pooler copy (on wbar, into the start
// of smem) did not arrive.
template <typename T, int D>
__device__ __forceinline__ bool fused_append(AppendDims dims, const LevelRef* lv, long long u, long long P, const T* kn,
                                          const T* vn, unsigned char* smem, T* patch, int jf, uint64_t* wbar,
                                          int* err, bool fence) {
    const int tid = threadIdx.x;
    const bool ok = append_token<T, D>(
        dims, lv, u, P, kn, vn, reinterpret_cast<const T*>(smem), reinterpret_cast<float*>(smem + D * D * sizeof(T)),
        [&]() {
            const int timed_out = !mbar_wait(wbar, 0);
            if (__syncthreads_or(timed_out)) {
                if (tid == 0) flag_error(err, ERR_TIMEOUT);
                return false;
            }
            return true;
        },
        [&](int jj, T ky, T vy) {
            if (jj == jf) {
                patch[tid] = ky;
                patch[D + tid] = vy;
            }
        });
    if (jf == 0 && tid < D) {
        patch[tid] = kn[tid];
        patch[D + tid] = vn[tid];
    }
    if (fence) fence_proxy_async_global();  // this CTA's writes, before its later bulk reads
    __syncthreads();
    return ok;
}

__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <typename T, int D, int G>
__global__ void __launch_bounds__(DEC_THREADS, 2) decode_kernel(TreeParams p, DecodeArgs a) {
    constexpr int NCC = dec_ncc<D>();     // column chunks in accumulation
    constexpr int NEG = dec_neg<D>();     // entry groups in accumulation
    constexpr int W = DEC_WARPS;
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int CS = (int)cluster.num_blocks();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long long u = blockIdx.y;
    const int MY = a.my_max;
    const int b = p.b;

    extern __shared__ __align__(128) unsigned char smem_raw[];
    T* Kt = reinterpret_cast<T*>(smem_raw);
    T* Vt = Kt + (size_t)MY * D;
    float* egacc = reinterpret_cast<float*>(smem_raw);  // [NEG][G][D], after the last tile
    DecSmem* sm = reinterpret_cast<DecSmem*>(smem_raw + a.region0);
    unsigned long long* key = reinterpret_cast<unsigned long long*>(sm + 1);
    unsigned long long* gkeys = key + MY;  // [2][CS][KMAX]: the CTAs' top-k lists, by level parity
    float* qf = reinterpret_cast<float*>(gkeys + 2 * DEC_CLUSTER * KMAX);
    float* lg = qf + G * D;    // [MY][G] logits, then softmax weights
    float* cacc = lg + MY * G;
    float* cml = cacc + G * D;  // [G] max, [G] sum
    float* gat = cml + 2 * G;   // [CS][G*D + 2G] (rank 0: every CTA's state)

    // set-up that does not read the tree (overlaps the previous kernel under
    // programmatic dependent launch)
    // fused step: the last CTA of the cluster appends the token (its rows
    // of the first scored level are the last ones, which the append changes)
    const bool app = a.k_new != nullptr;
    const bool appender = app && rank == CS - 1;
    if (tid == 0) {
        sm->pg = DecPages{p.pages ? p.pages + (u / p.H) * p.max_pages : nullptr, p.page_size, p.H, (int)(u % p.H),
                          (int)p.num_pages};
        sm->tok = token_map(p);
        mbar_init(&sm->bar[0], 1);
        mbar_init(&sm->bar[1], 1);
        mbar_init(&sm->bar[2], 1);
        fence_mbar_init();
        if (appender) {  // the pooler is constant: fetch it before the dependency wait
            mbar_arrive_expect_tx(&sm->bar[2], (uint32_t)(D * D * sizeof(T)));
            bulk_g2s(smem_raw, p.Wt, (uint32_t)(D * D * sizeof(T)), &sm->bar[2]);
        }
    }
    asm volatile("griddepcontrol.launch_dependents;");
    {  // the RoPE table is constant: every CTA brings its share of it into L2
       // now, so that no scoring step waits for it in DRAM
        const long long lines = ((long long)p.npos * 3 * (D / 2) * 4 + 127) / 128;
        const long long nct = (long long)gridDim.y * CS, ci = (long long)blockIdx.y * CS + rank;
        const long long per = (lines + nct - 1) / nct;
        const long long l0 = ci * per + tid;
        if (tid < per && l0 < lines) asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<const char*>(p.rope) + l0 * 128));
    }
    load_levels(p, sm->lv, tid);  // visible after the set-up barrier below
    if (tid < 8) sm->M[tid] = -INFINITY;
    grid_dependency_wait();  // from here on, every earlier kernel's writes are visible
    if (appender) {
        // the append reads every level's right-edge prefix sums and the new
        // token's rows; their addresses do not depend on the length, so they
        // are brought into L1 now, together with the length and the query
        constexpr int LPR = D * 4 / 128;  // 128-byte lines of one fp32 row
        const int nl = 2 * p.J_cap * LPR;
        if (tid < nl) {
            const int jj = tid / (2 * LPR) + 1, x = tid % (2 * LPR);
            const float* row = (x < LPR ? p.PK[jj] : p.PV[jj]) + u * D;
            asm volatile("prefetch.global.L1 [%0];" ::"l"(reinterpret_cast<const char*>(row) + (x % LPR) * 128));
        } else if (tid < nl + 2 * (int)((D * sizeof(T) + 127) / 128)) {
            const int x = tid - nl, per = (int)((D * sizeof(T) + 127) / 128);
            const T* row = reinterpret_cast<const T*>(x < per ? a.k_new : a.v_new) + u * D;
            asm volatile("prefetch.global.L1 [%0];" ::"l"(reinterpret_cast<const char*>(row) + (x % per) * 128));
        }
    }
    const long long Lraw = p.len[u];  // both loads in flight together
    {
        const T* qg = reinterpret_cast<const T*>(a.q) + (u * G) * D;
        constexpr int QV = (G * D) / DEC_THREADS >= 4 ? 4 : 2;  // elements per thread and load
        float f[QV];
        for (int i = tid * QV; i < G * D; i += DEC_THREADS * QV) {
            load_vec<T, QV>(qg + i, f);
#pragma unroll
            for (int x = 0; x < QV; x++) qf[i + x] = f[x];
        }
    }
    // after a fused append the tree holds one more token
    const bool bad_len = app ? (Lraw < 0 || Lraw >= p.cap) : (Lraw <= 0 || Lraw > p.cap);
    const int L = bad_len ? 0 : (int)Lraw + (app ? 1 : 0);
    bool bad = bad_len;
    bool appended = false;
    if (tid == 0 && bad_len && rank == 0) flag_error(p.err, ERR_LENGTH);
    if (tid <= p.J_cap) {  // n_j = ceil(L / b^j), the same as j nested ceilings
        long long pw = 1;
        for (int x = 0; x < tid && pw <= L; x++) pw *= b;
        sm->nlev[tid] = (int)((L + pw - 1) / pw);
    }
    __syncthreads();

    // this thread's share of the softmax: columns [cc*CPT, cc*CPT + CPT) of
    // entry group eg, every head
    const int cc = tid % NCC, eg = tid / NCC;
    float2 acc[G][CPT / 2];
    float lpart[G];
#pragma unroll
    for (int g = 0; g < G; g++) {
        lpart[g] = 0.f;
#pragma unroll
        for (int c = 0; c < CPT / 2; c++) acc[g][c] = make_float2(0.f, 0.f);
    }
    uint32_t phase[2] = {0u, 0u};
    long long krows = 0, vrows = 0;

    // Thread 0: request rows [r0, r1) of level j's candidate list (children of
    // sm->par) into the key (which = 0) or value (which = 1) tile.
    auto issue = [&](int which, int j, int r0, int r1) {
        const bool paged = j == 0 && p.pages;
        const T* lb = reinterpret_cast<const T*>(which == 0 ? sm->lv[j].K : sm->lv[j].V);
        issue_rows<T, D>(which == 0 ? Kt : Vt, paged ? lb : lb + (u * sm->lv[j].rows) * D, sm->par, sm->nlev[j], b, r0,
                         r1, &sm->bar[which], p.err, paged ? &sm->pg : nullptr);
    };
    auto wait_tile = [&](int which) {
        if (!mbar_wait(&sm->bar[which], phase[which])) {
            if (lane == 0) flag_error(p.err, ERR_TIMEOUT);
            bad = true;
        }
        phase[which] ^= 1u;
    };
    // candidates at level j: children of the npar kept parents in sm->par
    auto ncand_of = [&](int j, int npar) -> int {
        const int n_j = sm->nlev[j];
        const int last = sm->par[npar - 1];
        if (last < 0 || last * b >= n_j) return 0;
        return (npar - 1) * b + min(b, n_j - last * b);
    };

    // One shared softmax over every level's entries: entries [0, nmy) of this
    // CTA join with weights exp(logit - running max); `tokens` = every entry
    // counts, otherwise only candidates that were not kept. The scoring pass
    // has left each warp's largest logit per head in sm->red (over all rows,
    // kept ones included: a bound on the entries that join, which is all the
    // running maximum needs).
    const int gt = tid % G;  // the head of this thread's weights (DEC_THREADS % G == 0)
    auto accumulate = [&](int nmy, bool tokens) {
        float Mt = 0.f, Mown = 0.f, alpha[G];
#pragma unroll
        for (int g = 0; g < G; g++) {
            float m = sm->M[g];
            const float mold = m;
#pragma unroll
            for (int w = 0; w < W; w++) m = fmaxf(m, sm->red[w][g]);
            alpha[g] = (m == -INFINITY) ? 1.f : (mold == -INFINITY ? 0.f : expf(mold - m));
            lpart[g] *= alpha[g];
            if (g == gt) Mt = m;
            if (g == tid) Mown = m;
        }
        float lsum = 0.f;
        for (int x = tid; x < nmy * G; x += DEC_THREADS) {
            const int e = x / G;
            const bool valid = tokens || key[e] < sm->thresh;
            const float pe = valid ? expf(lg[x] - Mt) : 0.f;
            lg[x] = pe;
            lsum += pe;
        }
#pragma unroll
        for (int g = 0; g < G; g++)
            if (g == gt) lpart[g] += lsum;
        __syncthreads();  // weights in place; every thread has read sm->M
        if (tid < G) sm->M[tid] = Mown;
#pragma unroll
        for (int g = 0; g < G; g++)
#pragma unroll
            for (int c = 0; c < CPT / 2; c++) acc[g][c] = fmul2(acc[g][c], make_float2(alpha[g], alpha[g]));
#pragma unroll 2
        for (int e = eg; e < nmy; e += NEG) {
            float2 v[CPT / 2];
            load_row2<T, CPT>(Vt + (size_t)e * D + cc * CPT, v);
#pragma unroll
            for (int g = 0; g < G; g++) {
                const float pe = lg[e * G + g];
                const float2 pp = make_float2(pe, pe);
#pragma unroll
                for (int c = 0; c < CPT / 2; c++) acc[g][c] = ffma2(pp, v[c], acc[g][c]);
            }
        }
    };

    if (appender && bad_len) {  // no append; the pooler copy must land before the area is reused
        if (!mbar_wait(&sm->bar[2], 0) && tid == 0) flag_error(p.err, ERR_TIMEOUT);
        __syncthreads();
    }
    // [pooler | append scratch | patch rows: key, value | the appender's first tiles]
    auto patch_rows = [&]() {
        return reinterpret_cast<T*>(
            smem_raw + ((D * D * sizeof(T) + append_scratch_floats(D, p.J_cap) * 4 + 127) & ~(size_t)127));
    };
    // Fused step, usual case: the appending CTA holds only the right-edge row
    // of the first scored level (the only row the append changes), so it
    // appends at once and needs no copy of that row. The first scored level
    // is the highest level with more than k nodes (every level above keeps
    // all of its candidates), else the tokens.
    bool chained = false, fenced = false;
    if (appender && !bad_len) {
        int jt = 1;
        while (jt < p.J_cap && sm->nlev[jt] > b) jt++;
        int jf = 0;
        for (int x = jt; x >= 1 && jf == 0; x--)
            if (sm->nlev[x] > p.k) jf = x;
        if (sm->nlev[jf] - 1 <= (CS - 1) * MY) {
            const bool ok = fused_append<T, D>(AppendDims{p.cap, p.J_cap, p.b, &sm->tok}, sm->lv, u, Lraw,
                                               reinterpret_cast<const T*>(a.k_new) + u * D,
                                               reinterpret_cast<const T*>(a.v_new) + u * D, smem_raw, patch_rows(), jf,
                                               &sm->bar[2], p.err, false);
            appended = ok;
            if (!ok) bad = true;
            chained = true;
        }
    }
    if (!bad_len) {
        int j = 1;
        while (j < p.J_cap && sm->nlev[j] > b) j++;  // top level
        int npar = 1;
        if (tid == 0) sm->par[0] = 0;  // the top level = children of one virtual root
        __syncthreads();
        // levels that keep every candidate: nothing to read or score
        while (j >= 1) {
            const int nc = ncand_of(j, npar);
            if (nc > p.k || nc < 1) break;
            if (tid < nc) sm->chosen[tid] = sm->par[tid / b] * b + tid % b;
            __syncthreads();
            if (rank == 0 && a.sel_out)  // not thread 0: it issues the copies
                for (int x = tid - 32; x >= 0 && x < p.k; x += DEC_THREADS - 32)
                    a.sel_out[(u * p.J_cap + (j - 1)) * p.k + x] = x < nc ? sm->chosen[x] : -1;
            if (tid < nc) sm->par[tid] = sm->chosen[tid];
            npar = nc;
            j--;
            __syncthreads();
        }

        int ncand = ncand_of(j, npar);
        if (ncand < 1) {
            bad = true;
            if (tid == 0) flag_error(p.err, ERR_SHAPE);
        }
        // contiguous row ranges counted from the end: the last CTA holds the
        // last rows of every level
        int per = (ncand + CS - 1) / CS;
        int r0 = max(0, ncand - (CS - rank) * per), r1 = max(0, ncand - (CS - 1 - rank) * per);
        if (app && ncand >= 1 && ncand - 1 <= (CS - 1) * MY) {  // same test as the appender's early append
            // fused step: the appending CTA takes only the right-edge row (it
            // appends first), the others share the rest
            const int per1 = (ncand - 1 + CS - 2) / (CS - 1);
            r0 = rank == CS - 1 ? ncand - 1 : min(ncand - 1, rank * per1);
            r1 = rank == CS - 1 ? ncand : min(ncand - 1, r0 + per1);
        }
        // Fused step, other case (a first level too large for the one-row
        // split): the appending CTA holds the last rows of this level; its
        // tiles are requested now into a place after the pooler and the append
        // scratch (when they fit), it appends, and the refreshed right-edge
        // row is written over the copied one once the tile has landed. The
        // other CTAs read the right edge only after the first selection
        // barrier, which this CTA reaches after the append.
        const size_t tiles_off = ((reinterpret_cast<unsigned char*>(patch_rows() + 2 * D) - smem_raw) + 127) & ~(size_t)127;
        const bool early = appender && tiles_off + 2 * (size_t)(r1 - r0) * D * sizeof(T) <= (size_t)a.region0;
        if (early) {
            Kt = reinterpret_cast<T*>(smem_raw + tiles_off);
            Vt = Kt + (size_t)(r1 - r0) * D;
        }
        int patch_row = -1;  // row of this CTA's first tiles to overwrite
        if (chained) {
            // the one row is the refreshed right edge: written here, not copied
            // (empty requests complete the tile barriers' phases)
            if (tid < D) {
                Kt[(size_t)(ncand - 1 - r0) * D + tid] = patch_rows()[tid];
                Vt[(size_t)(ncand - 1 - r0) * D + tid] = patch_rows()[D + tid];
            }
            if (tid == 0) {
                issue(0, j, r0, r0);
                issue(1, j, r0, r0);
            }
            __syncthreads();
        } else {
            if (tid == 0 && (!appender || early)) {
                issue(0, j, r0, r1);
                issue(1, j, r0, r1);
            }
            if (appender) {
                const bool ok = fused_append<T, D>(AppendDims{p.cap, p.J_cap, p.b, &sm->tok}, sm->lv, u, Lraw,
                                                   reinterpret_cast<const T*>(a.k_new) + u * D,
                                                   reinterpret_cast<const T*>(a.v_new) + u * D, smem_raw, patch_rows(),
                                                   j, &sm->bar[2], p.err, true);
                appended = ok;
                if (!ok) bad = true;
                if (early)
                    patch_row = ncand - 1 - r0;
                else if (tid == 0) {
                    issue(0, j, r0, r1);
                    issue(1, j, r0, r1);
                }
            }
        }
        for (;;) {
            const int nmy = r1 - r0;
            const int P = ncand > 0 ? ncand - 1 : 0;  // query position at this level
            wait_tile(0);
            if (patch_row >= 0) {
                if (tid < D) Kt[(size_t)patch_row * D + tid] = patch_rows()[tid];
                __syncthreads();
            }
            krows += ncand;
            // logits of this CTA's rows, each warp's largest logit per head,
            // selection keys (score, node id)
            score_rows<T, D, G, W>(p.rope, p.scale, b, Kt, qf, r0, nmy, P, warp, lane, sm->red[warp],
                                   [&](int i, int h, float logit, float S, int r, int o) {
                                       lg[i * G + h] = logit;
                                       if (h == 0 && j > 0) key[i] = sel_key(S, sm->par[r] * b + o);
                                   });
            const int kk = max(1, min(p.k, ncand));
            const int chunk = (nmy + W - 1) / W;  // rows per warp, as in the scoring
            if (j > 0 && nmy > 1) {  // each warp's top keys, sorted (its own rows: a warp barrier suffices)
                __syncwarp();
                const int w_lo = warp * chunk, nw = max(0, min(nmy, w_lo + chunk) - w_lo);
                unsigned long long* wl = sm->wl[warp];
                if (chunk <= 32) {
                    unsigned long long x = lane < nw ? key[w_lo + lane] : 0ull;
                    x = warp_sort_desc(x, lane);
                    if (lane < kk) wl[lane] = x;
                    for (int y = 32 + lane; y < kk; y += 32) wl[y] = 0ull;
                } else {
                    for (int e = lane; e < nw; e += 32) {
                        const unsigned long long kt = key[w_lo + e];
                        const int c = rank_among(key + w_lo, nw, kt);
                        if (c < kk) wl[c] = kt;
                    }
                    for (int x = nw + lane; x < kk; x += 32) wl[x] = 0ull;
                }
            }
            __syncthreads();  // logits, keys and warp lists in place; key tile free

            int nc_next = 0, per_n = 0, r0n = 0, r1n = 0;
            if (j > 0) {
                // this CTA's top keys, written to slot `rank` of every CTA's
                // list area for this level
                unsigned long long* gk = gkeys + (j & 1) * (DEC_CLUSTER * KMAX);
                if (nmy <= 1) {  // the list is this CTA's one key (or nothing): no sort, no merge
                    for (int t = tid; t < CS * kk; t += DEC_THREADS) {
                        const int r = t / kk, c = t - r * kk;
                        cluster.map_shared_rank(gk, r)[rank * KMAX + c] = (c == 0 && nmy == 1) ? key[0] : 0ull;
                    }
                } else {
                    for (int t = tid; t < W * kk; t += DEC_THREADS) {
                        const unsigned long long x = sm->wl[t / kk][t % kk];
                        if (x == 0ull) continue;
                        const int c = rank_in_lists<W>(&sm->wl[0][0], KMAX, kk, x);
                        if (c < kk)
                            for (int r = 0; r < CS; r++) cluster.map_shared_rank(gk, r)[rank * KMAX + c] = x;
                    }
                    for (int t = nmy + tid; t < kk; t += DEC_THREADS)  // fewer rows than kk
                        for (int r = 0; r < CS; r++) cluster.map_shared_rank(gk, r)[rank * KMAX + t] = 0ull;
                }
                if (chained && !fenced) {  // the append's global writes, before anyone's bulk reads of them
                    fence_proxy_async_global();
                    fenced = true;
                }
                cluster.sync();
                // global top-kk (the same in every CTA) and the kept ids in
                // ascending order (ids are distinct)
                for (int t = tid; t < CS * kk; t += DEC_THREADS) {
                    const unsigned long long x = gk[(t / kk) * KMAX + t % kk];
                    if (x == 0ull) continue;
                    const int c = rank_in_lists<DEC_CLUSTER>(gk, KMAX, kk, x);
                    if (c < kk) sm->picked[c] = x;
                }
                __syncthreads();
                // the kept ids in ascending order: the next level's parents
                if (tid < kk) {
                    const int id = (int)key_id(sm->picked[tid]);
                    int pos = 0;
                    for (int r = 0; r < kk; r++) pos += (int)key_id(sm->picked[r]) < id;
                    sm->chosen[pos] = id;
                    sm->par[pos] = id;  // no one reads this level's parents any more
                    if (rank == 0 && a.sel_out) a.sel_out[(u * p.J_cap + (j - 1)) * p.k + pos] = id;
                }
                if (rank == 0 && a.sel_out)
                    for (int x = kk + tid; x < p.k; x += DEC_THREADS) a.sel_out[(u * p.J_cap + (j - 1)) * p.k + x] = -1;
                if (tid == 0) sm->thresh = sm->picked[kk - 1];
                __syncthreads();
                // the next level's candidates are the children of the kept nodes
                nc_next = ncand_of(j - 1, kk);
                if (nc_next < 1) {
                    bad = true;
                    if (tid == 0) flag_error(p.err, ERR_SHAPE);
                }
                per_n = (nc_next + CS - 1) / CS;
                r0n = max(0, nc_next - (CS - rank) * per_n);
                r1n = max(0, nc_next - (CS - 1 - rank) * per_n);
                Kt = reinterpret_cast<T*>(smem_raw);
                if (tid == 0) issue(0, j - 1, r0n, r1n);  // key tile is free since the barriers above
            }
            wait_tile(1);
            if (patch_row >= 0) {
                if (tid < D) Vt[(size_t)patch_row * D + tid] = patch_rows()[D + tid];
                __syncthreads();
                patch_row = -1;
            }
            // level 0: every token; above: the summaries of the candidates not kept
            accumulate(nmy, j == 0);
            vrows += j == 0 ? ncand : ncand - kk;
            if (j == 0) break;
            __syncthreads();  // value tile and weights consumed
            Vt = reinterpret_cast<T*>(smem_raw) + (size_t)MY * D;
            if (tid == 0) issue(1, j - 1, r0n, r1n);
            npar = kk;
            j--;
            ncand = nc_next;
            per = per_n;
            r0 = r0n;
            r1 = r1n;
        }
    }

    // CTA state: sum the entry groups (egacc overlays the tiles, consumed by now)
    __syncthreads();
#pragma unroll
    for (int g = 0; g < G; g++) {
#pragma unroll
        for (int c = 0; c < CPT / 2; c++) {
            egacc[(eg * G + g) * D + cc * CPT + 2 * c] = acc[g][c].x;
            egacc[(eg * G + g) * D + cc * CPT + 2 * c + 1] = acc[g][c].y;
        }
        float s = lpart[g];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) sm->red[warp][g] = s;
    }
    __syncthreads();
    // Every CTA merges one slice of the output columns: each CTA sends slice r
    // of its (unnormalised) output, with its maxima and sums, to CTA r (the
    // gather area has a place of its own: no barrier is needed before it).
    // Each column's sum over the entry groups goes straight to its CTA.
    constexpr int SL = G * D / DEC_CLUSTER;  // output columns per CTA
    constexpr int GST = SL + 2 * G;          // one source's record in the gather area
    static_assert((G * D) % DEC_CLUSTER == 0, "output slices");
    for (int idx = tid; idx < G * D; idx += DEC_THREADS) {
        float s = 0.f;
#pragma unroll
        for (int x = 0; x < NEG; x++) s += egacc[x * G * D + idx];
        const int r = idx / SL;
        cluster.map_shared_rank(gat, r)[rank * GST + (idx - r * SL)] = s;
    }
    if (tid < G) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < W; w++) s += sm->red[w][tid];
        const float mx = sm->M[tid];
        for (int r = 0; r < CS; r++) {
            float* g_r = cluster.map_shared_rank(gat, r) + rank * GST + SL;
            g_r[tid] = mx;
            g_r[G + tid] = s;
        }
    }
    if (chained && !fenced) fence_proxy_async_global();
    cluster.sync();  // every CTA's gather area is complete
    if (appended && tid == 0) p.len[u] = Lraw + 1;  // every CTA has read the old length
    {
        // per head: the common maximum, each source's factor, the denominator
        float* fac = cacc;  // [CS][G] factors, then [G] reciprocal denominators (cacc is free now)
        if (tid < G) {
            float M = -INFINITY;
            for (int r = 0; r < CS; r++) M = fmaxf(M, gat[r * GST + SL + tid]);
            float den = 0.f;
            for (int r = 0; r < CS; r++) {
                const float mr = gat[r * GST + SL + tid];
                const float f = (mr == -INFINITY) ? 0.f : expf(mr - M);
                fac[r * G + tid] = f;
                den += gat[r * GST + SL + G + tid] * f;
            }
            fac[CS * G + tid] = 1.f / den;
        }
        __syncthreads();
        T* outp = reinterpret_cast<T*>(a.out) + (u * G) * D + rank * SL;
        for (int i = tid; i < SL; i += DEC_THREADS) {
            const int g = (rank * SL + i) / D;
            float s = 0.f;
            for (int r = 0; r < CS; r++) s += gat[r * GST + i] * fac[r * G + g];
            const float o = bad ? 0.f : s * fac[CS * G + g];
            if (a.out_f32)
                a.out_f32[(u * G) * D + rank * SL + i] = o;
            else
                outp[i] = from_f<T>(o);
        }
    }
    if (rank == 0) {
        int J = 0;
        if (!bad_len) {
            J = 1;
            while (J < p.J_cap && sm->nlev[J] > b) J++;
        }
        if (tid == 0) {
            if (a.rows_out) {
                a.rows_out[u * 2] = krows;
                a.rows_out[u * 2 + 1] = vrows;
            }
            p.stats[u * 3] = bad_len ? 0 : J + 1;
            p.stats[u * 3 + 1] = krows;
            p.stats[u * 3 + 2] = vrows;
        }
        if (a.sel_out)
            for (int i = tid; i < (p.J_cap - J) * p.k; i += DEC_THREADS)
                a.sel_out[(u * p.J_cap + J) * p.k + i] = -1;
    }
}

// Dynamic shared memory of one decode CTA (fused: the appending CTA's
// pooler and scratch included).
size_t decode_smem_bytes(int D, int G, int elem, int k, int b, int J_cap, bool fused) {
    const long long maxc = (long long)k * b > b ? (long long)k * b : b;
    const int my = (int)((maxc + DEC_CLUSTER - 1) / DEC_CLUSTER);
    return decode_region0(D, G, my, elem, J_cap, fused) + decode_smem_tail(D, G, my);
}

// k_new, v_new: null for a decode alone; else the fused step (append the
// token of every unit, then decode against the grown tree).
template <typename T, int D, int G>
cudaError_t launch_decode(const TreeParams& p, const void* k_new, const void* v_new, const void* q, void* out,
                          int* sel_out, long long* rows_out, float* out_f32, cudaStream_t s) {
    const int CS = DEC_CLUSTER;
    const long long maxc = (long long)p.k * p.b > p.b ? (long long)p.k * p.b : p.b;
    const bool fused = k_new != nullptr;
    DecodeArgs a{k_new, v_new, q, out, out_f32, sel_out, rows_out, (int)((maxc + CS - 1) / CS), 0};
    a.region0 = (int)decode_region0(D, G, a.my_max, (int)sizeof(T), p.J_cap, fused);
    const size_t smem = a.region0 + decode_smem_tail(D, G, a.my_max);
    auto kern = decode_kernel<T, D, G>;
    if (smem > 227 * 1024) return cudaErrorInvalidValue;
    static std::atomic<unsigned long long> attr_done{0};  // per instantiation, per device
    cudaError_t e = set_smem_limit(kern, 227 * 1024, attr_done);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(CS, p.B * p.H, 1);
    cfg.blockDim = dim3(DEC_THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // may start while the previous kernel on the stream finishes; the kernel
    // waits for it before reading the tree
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, p, a);
}

#define RECSA_INST_DEC(T, D, G) \
    template cudaError_t launch_decode<T, D, G>(const TreeParams&, const void*, const void*, const void*, void*, \
                                                int*, long long*, float*, cudaStream_t);
#define RECSA_INST_DEC_G(T, D) RECSA_INST_DEC(T, D, 1) RECSA_INST_DEC(T, D, 2) RECSA_INST_DEC(T, D, 4) RECSA_INST_DEC(T, D, 8)
RECSA_INST_DEC_G(float, 64)
RECSA_INST_DEC_G(float, 128)
RECSA_INST_DEC_G(__nv_bfloat16, 64)
RECSA_INST_DEC_G(__nv_bfloat16, 128)

}  // namespace recsa
