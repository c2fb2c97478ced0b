// Prefill, tree part: one CTA per (chunk token, KV head).
//
// Token t of a chunk [s, s+C) attends the tree over the s tokens cached
// before the chunk (RecSA abstract: per-level selection of at most k
// candidates, summaries of the unselected candidates in one softmax with the
// exact tokens, candidate-index RoPE), then the chunk's own tokens s..t,
// which follow the level-0 candidates: the query sits at index n0 + (t - s)
// among n0 kept tokens plus the chunk prefix. The chunk-local part (causal
// attention inside the chunk) has already been computed as a softmax state
// per (token, query head); this kernel runs the descent, accumulates the
// tree's entries into a second state and merges the two.
//
// Per level, the candidates (children of the kept parents, ascending) are
// brought into shared memory TILE rows at a time with bulk async copies and
// scored in fp32 on CUDA cores (the selection must match the fp64 reference
// exactly); the top k come from a bitonic sort of the packed (score, id)
// keys; the value rows of the candidates not kept are then streamed for the
// softmax. Level-0 candidates are scored and accumulated tile by tile.
#include "common.cuh"
#include "score.cuh"

namespace recsa {

constexpr int PT_THREADS = 256;
constexpr int PT_WARPS = PT_THREADS / 32;
constexpr int PT_TILE = 128;
constexpr int PT_KMAX = 64;
constexpr int PT_CPT = 4;  // output columns per thread in the softmax-value product

struct PrefillTreeArgs {
    const void* q;       // [B][C][Hq][D]
    void* out;           // [B][C][Hq][D]
    const float* state;  // [B][C][Hq][D + 2] local part: unnormalised acc, max, sum
    int* sel_out;        // nullable [B][C][H][J_cap][k]
    long long* rows_out;  // nullable [B][C][H][2]: key rows scored, value rows (softmax entries)
    int C, Hq;
    int maxc;            // most candidates a level can have
    int sortn;           // power of two >= maxc
};

struct PtSmem {
    uint64_t bar[2];
    unsigned long long thresh;
    int par[PT_KMAX], chosen[PT_KMAX];
    unsigned long long picked[PT_KMAX];  // the level's top keys, best first
    int nlev[MAXJ + 1];
    LevelRef lv[MAXJ + 1];  // the levels' addresses
    float red[PT_WARPS][8];
    float M[8];
};

// [tiles: K | V (2 * TILE * D * elem), later the entry-group partials][PtSmem]
// [key u64 maxc][skey u64 sortn][qf G*D][lg G*maxc][pbuf TILE*G][cacc G*D][cl G]
__host__ __device__ inline size_t prefill_tree_smem(int D, int G, int elem, int maxc, int sortn) {
    size_t tiles = 2 * (size_t)PT_TILE * D * elem;
    const size_t eg = (size_t)(PT_THREADS / (D / PT_CPT)) * G * D * 4;
    if (eg > tiles) tiles = eg;
    tiles = (tiles + 127) & ~(size_t)127;
    return tiles + sizeof(PtSmem) + (size_t)maxc * 8 + (size_t)sortn * 8 +
           (size_t)(G * D + G * maxc + PT_TILE * G + G * D + G) * 4;
}
__host__ __device__ inline size_t prefill_tree_tiles(int D, int G, int elem) {
    size_t tiles = 2 * (size_t)PT_TILE * D * elem;
    const size_t eg = (size_t)(PT_THREADS / (D / PT_CPT)) * G * D * 4;
    if (eg > tiles) tiles = eg;
    return (tiles + 127) & ~(size_t)127;
}

// Four independent runs of one key per lane, each sorted descending across
// the warp (bitonic network; the four advance together).
__device__ __forceinline__ void warp_sort4_desc32(unsigned long long (&x)[4], int lane) {
#pragma unroll 1
    for (int k2 = 2; k2 <= 32; k2 <<= 1)
#pragma unroll 1
        for (int j2 = k2 >> 1; j2 > 0; j2 >>= 1) {
            const bool desc = (lane & k2) == 0, lower = (lane & j2) == 0;
#pragma unroll
            for (int r = 0; r < 4; r++) {
                const unsigned long long y = __shfl_xor_sync(0xffffffffu, x[r], j2);
                x[r] = (lower == desc) ? (x[r] > y ? x[r] : y) : (x[r] < y ? x[r] : y);
            }
        }
}

// The lanes hold a bitonic sequence (largest first run, then smallest);
// returns it sorted descending.
__device__ __forceinline__ unsigned long long warp_merge_desc32(unsigned long long x, int lane) {
#pragma unroll
    for (int j2 = 16; j2 > 0; j2 >>= 1) {
        const unsigned long long y = __shfl_xor_sync(0xffffffffu, x, j2);
        x = (lane & j2) == 0 ? (x > y ? x : y) : (x < y ? x : y);
    }
    return x;
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(PT_THREADS, 2) prefill_tree_kernel(TreeParams p, PrefillTreeArgs a) {
    constexpr int NCC = D / PT_CPT, NEG = PT_THREADS / NCC;
    constexpr int W = PT_WARPS;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t = blockIdx.x;            // token of the chunk
    const long long u = blockIdx.y;      // (sequence, KV head)
    const int bseq = (int)(u / p.H), h = (int)(u % p.H);
    const int b = p.b, MC = a.maxc;

    extern __shared__ __align__(128) unsigned char smem_pt[];
    const size_t tiles_bytes = prefill_tree_tiles(D, G, (int)sizeof(T));
    float* egacc = reinterpret_cast<float*>(smem_pt);
    PtSmem* sm = reinterpret_cast<PtSmem*>(smem_pt + tiles_bytes);
    unsigned long long* key = reinterpret_cast<unsigned long long*>(sm + 1);
    unsigned long long* skey = key + MC;
    float* qf = reinterpret_cast<float*>(skey + a.sortn);
    float* lg = qf + G * D;           // [MC][G] logits of a level's candidates
    float* pbuf = lg + G * MC;        // [TILE][G]
    float* cacc = pbuf + PT_TILE * G;
    float* cl = cacc + G * D;

    if (tid == 0) {
        mbar_init(&sm->bar[0], 1);
        mbar_init(&sm->bar[1], 1);
        fence_mbar_init();
    }
    if (tid < 8) sm->M[tid] = -INFINITY;
    load_levels(p, sm->lv, tid);  // visible after the set-up barrier below
    {
        const T* qg = reinterpret_cast<const T*>(a.q) + (((size_t)bseq * a.C + t) * a.Hq + h * G) * D;
        for (int i = tid; i < G * D; i += PT_THREADS) qf[i] = to_f(qg[i]);
    }
    const long long Sraw = p.len[u];  // tokens in the tree (the chunk starts here)
    const bool bad_len = (Sraw < 0 || Sraw + a.C > p.cap);
    const int S = bad_len ? 0 : (int)Sraw;
    bool bad = bad_len;
    if (tid == 0) {
        if (bad_len) flag_error(p.err, ERR_LENGTH);
        int n = S;
        sm->nlev[0] = n;
        for (int j = 1; j <= p.J_cap; j++) {
            n = (n + b - 1) / b;
            sm->nlev[j] = n;
        }
    }
    __syncthreads();

    const int cc = tid % NCC, eg = tid / NCC;
    float2 acc[G][PT_CPT / 2];
    float lpart[G];
#pragma unroll
    for (int g = 0; g < G; g++) {
        lpart[g] = 0.f;
#pragma unroll
        for (int c = 0; c < PT_CPT / 2; c++) acc[g][c] = make_float2(0.f, 0.f);
    }
    uint32_t phase[2] = {0u, 0u};

    // Thread 0: rows [r0, r1) of level j's candidate list (children of
    // sm->par) into tile buffer buf (two buffers of PT_TILE rows, one
    // mbarrier each): what = 0 keys, 1 values, 2 both (keys in the first half
    // of the buffer, values in the second; at most PT_TILE / 2 rows).
    auto issue = [&](int buf, int what, int j, int r0, int r1) {
        T* dst = reinterpret_cast<T*>(smem_pt) + (size_t)buf * PT_TILE * D;
        T* dstv = what == 2 ? dst + (size_t)(PT_TILE / 2) * D : dst;
        const T* kb = reinterpret_cast<const T*>(sm->lv[j].K) + (u * sm->lv[j].rows) * D;
        const T* vb = reinterpret_cast<const T*>(sm->lv[j].V) + (u * sm->lv[j].rows) * D;
        const int n_j = sm->nlev[j];
        const int pr = r0 / b, o0 = r0 - pr * b;
        uint32_t total = 0;
        for (int r = r0, q = pr, o = o0; r < r1; q++, o = 0) {
            const int n = min(b - o, r1 - r);
            const int id0 = sm->par[q] * b + o;
            if (id0 >= 0 && id0 + n <= n_j) total += (uint32_t)(n * D * sizeof(T));
            r += n;
        }
        fence_proxy_async_shared();
        mbar_arrive_expect_tx(&sm->bar[buf], what == 2 ? 2 * total : total);
        for (int r = r0, q = pr, o = o0; r < r1; q++, o = 0) {
            const int n = min(b - o, r1 - r);
            const int id0 = sm->par[q] * b + o;
            const uint32_t bytes = (uint32_t)(n * D * sizeof(T));
            if (id0 >= 0 && id0 + n <= n_j) {
                if (what != 1) bulk_g2s(dst + (size_t)(r - r0) * D, kb + (size_t)id0 * D, bytes, &sm->bar[buf]);
                if (what != 0) bulk_g2s(dstv + (size_t)(r - r0) * D, vb + (size_t)id0 * D, bytes, &sm->bar[buf]);
            } else {
                flag_error(p.err, ERR_SHAPE);
            }
            r += n;
        }
    };
    auto tile = [&](int buf) { return reinterpret_cast<T*>(smem_pt) + (size_t)buf * PT_TILE * D; };
    auto wait_tile = [&](int which) {
        if (!mbar_wait(&sm->bar[which], phase[which])) {
            if (lane == 0) flag_error(p.err, ERR_TIMEOUT);
            bad = true;
        }
        phase[which] ^= 1u;
    };
    auto ncand_of = [&](int j, int npar) -> int {
        const int n_j = sm->nlev[j];
        const int last = sm->par[npar - 1];
        if (last < 0 || last * b >= n_j) return 0;
        return (npar - 1) * b + min(b, n_j - last * b);
    };

    // Scores of tile rows [0, nmy) = candidate ranks [r0, r0 + nmy) with the
    // query at index P (logits, and the selection keys when want_keys).
    // Each warp's largest logit per head is folded into sm->red[warp]
    // (reset by reset_max).
    auto score_tile = [&](const T* Kt, int r0, int nmy, int P, bool want_keys) {
        score_rows<T, D, G, W>(
            p.rope, p.scale, b, Kt, qf, r0, nmy, P, warp, lane, sm->red[warp],
            [&](int i, int hh, float logit, float Ssum, int r, int o) {
                lg[(r0 + i) * G + hh] = logit;
                if (hh == 0 && want_keys) key[r0 + i] = sel_key(Ssum, sm->par[r] * b + o);
            },
            true);
    };
    auto reset_max = [&]() {  // each warp its own slots
        if (lane < G) sm->red[warp][lane] = -INFINITY;
        __syncwarp();
    };

    // Entries of tile rows [0, nmy) (ranks r0..) join the CTA's softmax:
    // all of them (tokens) or the candidates not kept (key < threshold). The
    // running maximum takes the scoring pass's per-warp maxima (over every
    // scored row, kept ones included: a bound on the entries that join).
    const int gt = tid % G;  // the head of this thread's weights (PT_THREADS % G == 0)
    auto accumulate = [&](const T* Vt, int r0, int nmy, bool tokens) {
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
        for (int x = tid; x < nmy * G; x += PT_THREADS) {
            const int e = x / G;
            const bool valid = tokens || key[r0 + e] < sm->thresh;
            const float pe = valid ? expf(lg[r0 * G + x] - Mt) : 0.f;
            pbuf[x] = pe;
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
            for (int c = 0; c < PT_CPT / 2; c++) acc[g][c] = fmul2(acc[g][c], make_float2(alpha[g], alpha[g]));
#pragma unroll 2
        for (int e = eg; e < nmy; e += NEG) {
            float2 vv[PT_CPT / 2];
            load_row2<T, PT_CPT>(Vt + (size_t)e * D + cc * PT_CPT, vv);
#pragma unroll
            for (int g = 0; g < G; g++) {
                const float pe = pbuf[e * G + g];
                const float2 pp = make_float2(pe, pe);
#pragma unroll
                for (int c = 0; c < PT_CPT / 2; c++) acc[g][c] = ffma2(pp, vv[c], acc[g][c]);
            }
        }
    };

    int J = 0;
    long long krows = 0, vrows = 0;
    if (!bad_len && S > 0) {
        J = 1;
        while (J < p.J_cap && sm->nlev[J] > b) J++;  // top level of the tree over S tokens
        int j = J, npar = 1;
        if (tid == 0) sm->par[0] = 0;
        __syncthreads();
        int* selrow = a.sel_out ? a.sel_out + (((size_t)bseq * a.C + t) * p.H + h) * p.J_cap * p.k : nullptr;
        for (; j >= 1; j--) {
            const int ncand = ncand_of(j, npar);
            if (ncand < 1) {
                if (tid == 0) flag_error(p.err, ERR_SHAPE);
                bad = true;
                break;
            }
            const int kk = min(p.k, ncand);
            if (ncand > p.k) {
                krows += ncand;
                vrows += ncand - kk;
                // score every candidate, tile by tile; the next tile is in
                // flight while one is scored
                const int nt = (ncand + PT_TILE - 1) / PT_TILE;
                if (tid == 0) issue(0, 0, j, 0, min(PT_TILE, ncand));
                reset_max();
                for (int ti = 0; ti < nt; ti++) {
                    const int bi = ti & 1, r0 = ti * PT_TILE, nmy = min(PT_TILE, ncand - r0);
                    if (tid == 0 && ti + 1 < nt) issue(bi ^ 1, 0, j, r0 + PT_TILE, min(r0 + 2 * PT_TILE, ncand));
                    wait_tile(bi);
                    score_tile(tile(bi), r0, nmy, ncand - 1, true);
                    __syncthreads();
                }
                // the values of the first tile are requested before the sort
                if (tid == 0) issue(0, 1, j, 0, min(PT_TILE, ncand));
                if (kk <= 32 && ncand <= W * 128 && a.sortn >= W * 32) {
                    // each warp: the top 32 of its 128 keys (four sorted runs
                    // of 32, merged pairwise); then the CTA's top kk by rank
                    // among the eight warp lists
                    unsigned long long R[4];
#pragma unroll
                    for (int r = 0; r < 4; r++) {
                        const int i = warp * 128 + r * 32 + lane;
                        R[r] = i < ncand ? key[i] : 0ull;
                    }
                    warp_sort4_desc32(R, lane);
#pragma unroll
                    for (int m = 0; m < 2; m++) {
                        const unsigned long long y = __shfl_sync(0xffffffffu, R[2 * m + 1], 31 - lane);
                        R[m] = warp_merge_desc32(R[2 * m] > y ? R[2 * m] : y, lane);
                    }
                    const unsigned long long y = __shfl_sync(0xffffffffu, R[1], 31 - lane);
                    skey[warp * 32 + lane] = warp_merge_desc32(R[0] > y ? R[0] : y, lane);
                    __syncthreads();
                    for (int x = tid; x < W * kk; x += PT_THREADS) {
                        const unsigned long long kx = skey[(x / kk) * 32 + x % kk];
                        if (kx == 0ull) continue;
                        // keys of each list greater than kx (descending, distinct):
                        // one binary search per list, the lists advancing together
                        int lo[W];
#pragma unroll
                        for (int l = 0; l < W; l++) lo[l] = 0;
#pragma unroll 1
                        for (int st = 32; st >= 1; st >>= 1) {
                            if (st > kk) continue;
#pragma unroll
                            for (int l = 0; l < W; l++) {
                                const int pos = lo[l] + st;
                                const unsigned long long yk = skey[l * 32 + min(pos, kk) - 1];
                                lo[l] = (pos <= kk && yk > kx) ? pos : lo[l];
                            }
                        }
                        int c = 0;
#pragma unroll
                        for (int l = 0; l < W; l++) c += lo[l];
                        if (c < kk) sm->picked[c] = kx;
                    }
                    __syncthreads();
                    if (tid < kk) {
                        const int id = (int)key_id(sm->picked[tid]);
                        int pos = 0;
                        for (int r = 0; r < kk; r++) pos += (int)key_id(sm->picked[r]) < id;
                        sm->chosen[pos] = id;
                    }
                    if (tid == 0) sm->thresh = sm->picked[kk - 1];
                    __syncthreads();
                } else {
                    // top kk by a descending bitonic sort of the packed keys
                    int sn = 2;
                    while (sn < ncand) sn <<= 1;
                    for (int i = tid; i < sn; i += PT_THREADS) skey[i] = i < ncand ? key[i] : 0ull;
                    __syncthreads();
                    for (int k2 = 2; k2 <= sn; k2 <<= 1)
                        for (int j2 = k2 >> 1; j2 > 0; j2 >>= 1) {
                            for (int i = tid; i < sn; i += PT_THREADS) {
                                const int ixj = i ^ j2;
                                if (ixj > i) {
                                    const unsigned long long x = skey[i], y = skey[ixj];
                                    const bool desc = (i & k2) == 0;
                                    if (desc ? (x < y) : (x > y)) {
                                        skey[i] = y;
                                        skey[ixj] = x;
                                    }
                                }
                            }
                            __syncthreads();
                        }
                    if (tid < kk) {
                        const int id = (int)key_id(skey[tid]);
                        int pos = 0;
                        for (int r = 0; r < kk; r++) pos += (int)key_id(skey[r]) < id;
                        sm->chosen[pos] = id;
                    }
                    if (tid == 0) sm->thresh = skey[kk - 1];
                    __syncthreads();
                }
                // summaries of the candidates not kept, tile by tile
                for (int ti = 0; ti < nt; ti++) {
                    const int bi = ti & 1, r0 = ti * PT_TILE, nmy = min(PT_TILE, ncand - r0);
                    if (tid == 0 && ti + 1 < nt) issue(bi ^ 1, 1, j, r0 + PT_TILE, min(r0 + 2 * PT_TILE, ncand));
                    wait_tile(bi);
                    accumulate(tile(bi), r0, nmy, false);
                    __syncthreads();
                }
            } else {  // keeps every candidate: nothing to read or score
                if (tid < ncand) sm->chosen[tid] = sm->par[tid / b] * b + tid % b;
                __syncthreads();
            }
            if (selrow)
                for (int x = tid; x < p.k; x += PT_THREADS) selrow[(j - 1) * p.k + x] = x < kk ? sm->chosen[x] : -1;
            if (tid < kk) sm->par[tid] = sm->chosen[tid];
            npar = kk;
            __syncthreads();
        }
        // level 0: the tokens under the kept level-1 nodes, then (in index
        // order) the chunk's own tokens, already in the local state
        const int n0 = bad ? 0 : ncand_of(0, npar);
        const int P0 = n0 + t;
        krows += n0;
        vrows += n0;
        // keys and values of half-size tiles together, the next tile in flight
        constexpr int T0 = PT_TILE / 2;
        const int nt0 = (n0 + T0 - 1) / T0;
        if (tid == 0 && nt0 > 0) issue(0, 2, 0, 0, min(T0, n0));
        for (int ti = 0; ti < nt0; ti++) {
            const int bi = ti & 1, r0 = ti * T0, nmy = min(T0, n0 - r0);
            if (tid == 0 && ti + 1 < nt0) issue(bi ^ 1, 2, 0, r0 + T0, min(r0 + 2 * T0, n0));
            wait_tile(bi);
            reset_max();
            score_tile(tile(bi), r0, nmy, P0, false);
            __syncthreads();
            accumulate(tile(bi) + (size_t)T0 * D, r0, nmy, true);
            __syncthreads();
        }
    }
    if (a.rows_out && tid == 0) {  // the chunk's own tokens s..t are entries too
        long long* r = a.rows_out + (((size_t)bseq * a.C + t) * p.H + h) * 2;
        r[0] = krows;
        r[1] = vrows + t + 1;
    }
    if (a.sel_out) {
        int* selrow = a.sel_out + (((size_t)bseq * a.C + t) * p.H + h) * p.J_cap * p.k;
        for (int i = tid; i < (p.J_cap - J) * p.k; i += PT_THREADS) selrow[J * p.k + i] = -1;
    }

    // CTA state of the tree entries (egacc overlays the tiles)
    __syncthreads();
#pragma unroll
    for (int g = 0; g < G; g++) {
#pragma unroll
        for (int c = 0; c < PT_CPT / 2; c++) {
            egacc[(eg * G + g) * D + cc * PT_CPT + 2 * c] = acc[g][c].x;
            egacc[(eg * G + g) * D + cc * PT_CPT + 2 * c + 1] = acc[g][c].y;
        }
        float s = lpart[g];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) sm->red[warp][g] = s;
    }
    __syncthreads();
    for (int idx = tid; idx < G * D; idx += PT_THREADS) {
        float s = 0.f;
#pragma unroll
        for (int x = 0; x < NEG; x++) s += egacc[x * G * D + idx];
        cacc[idx] = s;
    }
    if (tid < G) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < W; w++) s += sm->red[w][tid];
        cl[tid] = s;
    }
    __syncthreads();
    // merge with the chunk-local state and write the output
    for (int idx = tid; idx < G * D; idx += PT_THREADS) {
        const int g = idx / D, e = idx % D;
        const float* st = a.state + (((size_t)bseq * a.C + t) * a.Hq + h * G + g) * (D + 2);
        const float ml = st[D], ll = st[D + 1], mt = sm->M[g];
        const float M = fmaxf(ml, mt);
        const float ft = (mt == -INFINITY) ? 0.f : expf(mt - M);
        const float fl = (ml == -INFINITY) ? 0.f : expf(ml - M);
        const float num = cacc[idx] * ft + st[e] * fl;
        const float den = cl[g] * ft + ll * fl;
        T* outp = reinterpret_cast<T*>(a.out) + (((size_t)bseq * a.C + t) * a.Hq + h * G + g) * D;
        outp[e] = from_f<T>(bad ? 0.f : num / den);
    }
}

template <typename T, int D, int G>
cudaError_t launch_prefill_tree(const TreeParams& p, const void* q, void* out, const float* state, int* sel_out,
                                long long* rows_out, int B, int C, int Hq, cudaStream_t s) {
    PrefillTreeArgs a{q, out, state, sel_out, rows_out, C, Hq, 0, 1};
    a.maxc = p.k * p.b > p.b ? p.k * p.b : p.b;
    while (a.sortn < a.maxc) a.sortn <<= 1;
    const size_t smem = prefill_tree_smem(D, G, (int)sizeof(T), a.maxc, a.sortn);
    if (smem > 227 * 1024) return cudaErrorInvalidValue;
    auto kern = prefill_tree_kernel<T, D, G>;
    static std::atomic<unsigned long long> attr_done{0};
    cudaError_t e = set_smem_limit(kern, 227 * 1024, attr_done);
    if (e != cudaSuccess) return e;
    dim3 grid(C, B * p.H);
    kern<<<grid, PT_THREADS, smem, s>>>(p, a);
    return cudaGetLastError();
}

size_t prefill_tree_smem_bytes(int D, int G, int elem, int k, int b) {
    int maxc = k * b > b ? k * b : b, sortn = 1;
    while (sortn < maxc) sortn <<= 1;
    return prefill_tree_smem(D, G, elem, maxc, sortn);
}

#define RECSA_INST_PT(T, D, G)                                                                                   \
    template cudaError_t launch_prefill_tree<T, D, G>(const TreeParams&, const void*, void*, const float*, int*, \
                                                      long long*, int, int, int, cudaStream_t);
#define RECSA_INST_PT_G(T, D) RECSA_INST_PT(T, D, 1) RECSA_INST_PT(T, D, 2) RECSA_INST_PT(T, D, 4) RECSA_INST_PT(T, D, 8)
RECSA_INST_PT_G(__nv_bfloat16, 64)
RECSA_INST_PT_G(__nv_bfloat16, 128)

}  // namespace recsa
