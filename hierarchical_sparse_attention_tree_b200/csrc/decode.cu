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

#include "common.cuh"

namespace cg = cooperative_groups;

namespace recsa {

constexpr int DEC_THREADS = 256;
constexpr int DEC_WARPS = DEC_THREADS / 32;
constexpr int DEC_CLUSTER = 8;
constexpr int KMAX = 64;

struct DecodeArgs {
    const void* q;
    void* out;
    int* sel_out;         // nullable [B*H][J_cap][k]
    long long* rows_out;  // nullable [B*H][2]
    int my_max;           // candidates per CTA, upper bound
    int region0;          // bytes of the K/V tile region (reused for the warp merge)
};

struct DecSmem {
    uint64_t bar[2];                     // [0]: key tile, [1]: value tile
    unsigned long long topbuf[2][KMAX];  // local top-k lists (sorted), double-buffered by level parity
    unsigned long long picked[KMAX];     // global top-k keys, best first
    unsigned long long thresh;           // the k-th best key
    int par[KMAX];                       // kept parents of the current level, ascending
    int chosen[KMAX];                    // kept nodes of the current level, ascending
    int nlev[MAXJ + 1];                  // nodes per level over L tokens
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

// Shared memory: [region0: K tile | V tile; at the end: entry-group partials,
// then (rank 0) the cluster gather area][DecSmem][key: u64 MY][gkeys: u64
// CS*KMAX][qf G*D][lg G*MY][pbuf MY*G][cacc G*D][cml 2G]
__host__ __device__ inline size_t decode_smem_tail(int D, int G, int MY) {
    return sizeof(DecSmem) + (size_t)MY * 8 + (size_t)DEC_CLUSTER * KMAX * 8 +
           (size_t)(G * D + G * MY + MY * G + G * D + 2 * G) * 4;
}
__host__ __device__ inline size_t decode_region0(int D, int G, int MY, int elem) {
    const size_t tiles = 2 * (size_t)MY * D * elem;
    const size_t eg = (size_t)(DEC_THREADS / (D / CPT)) * G * D * 4;
    const size_t eg_al = (eg + 127) & ~(size_t)127;
    const size_t gat = (size_t)DEC_CLUSTER * (G * D + 2 * G) * 4;
    const size_t need = eg_al + gat;
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

__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <typename T, int D, int G>
__global__ void __launch_bounds__(DEC_THREADS, 2) decode_kernel(TreeParams p, DecodeArgs a) {
    constexpr int HD = D / 2;
    constexpr int PL = 4;                 // rotation pairs per lane in scoring
    constexpr int LPC = HD / PL;          // lanes per candidate in scoring
    constexpr int CPW = 32 / LPC;         // candidates per warp step in scoring
    static_assert(G <= LPC && 32 % LPC == 0 && G <= 8, "scoring layout");
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
    float* gat = reinterpret_cast<float*>(smem_raw + ((NEG * G * D * 4 + 127) & ~127));  // [CS][G*D + 2G]
    DecSmem* sm = reinterpret_cast<DecSmem*>(smem_raw + a.region0);
    unsigned long long* key = reinterpret_cast<unsigned long long*>(sm + 1);
    unsigned long long* gkeys = key + MY;
    float* qf = reinterpret_cast<float*>(gkeys + DEC_CLUSTER * KMAX);
    float* lg = qf + G * D;    // [G][MY] logits
    float* pbuf = lg + G * MY; // [MY][G] softmax weights
    float* cacc = pbuf + MY * G;
    float* cml = cacc + G * D;  // [G] max, [G] sum

    // set-up that does not read the tree (overlaps the previous kernel under
    // programmatic dependent launch)
    if (tid == 0) {
        mbar_init(&sm->bar[0], 1);
        mbar_init(&sm->bar[1], 1);
        fence_mbar_init();
    }
    if (tid < 8) sm->M[tid] = -INFINITY;
    grid_dependency_wait();  // from here on, every earlier kernel's writes are visible
    {
        const T* qg = reinterpret_cast<const T*>(a.q) + (u * G) * D;
        for (int i = tid; i < G * D; i += DEC_THREADS) qf[i] = to_f(qg[i]);
    }

    const long long Lraw = p.len[u];
    const bool bad_len = (Lraw <= 0 || Lraw > p.cap);
    const int L = bad_len ? 0 : (int)Lraw;
    bool bad = bad_len;
    if (tid == 0) {
        if (bad_len && rank == 0) flag_error(p.err, ERR_LENGTH);
        int n = L;
        sm->nlev[0] = n;
        for (int j = 1; j <= p.J_cap; j++) {
            n = (n + b - 1) / b;
            sm->nlev[j] = n;
        }
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
        T* dst = which == 0 ? Kt : Vt;
        const T* base = reinterpret_cast<const T*>(which == 0 ? p.K[j] : p.V[j]) + (u * p.rows[j]) * D;
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
        mbar_arrive_expect_tx(&sm->bar[which], total);
        for (int r = r0, q = pr, o = o0; r < r1; q++, o = 0) {
            const int n = min(b - o, r1 - r);
            const int id0 = sm->par[q] * b + o;
            if (id0 >= 0 && id0 + n <= n_j)
                bulk_g2s(dst + (size_t)(r - r0) * D, base + (size_t)id0 * D, (uint32_t)(n * D * sizeof(T)),
                         &sm->bar[which]);
            else
                flag_error(p.err, ERR_SHAPE);
            r += n;
        }
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
    // counts, otherwise only candidates that were not kept.
    auto accumulate = [&](int nmy, bool tokens) {
        float mx[G];
#pragma unroll
        for (int g = 0; g < G; g++) mx[g] = -INFINITY;
        for (int e = tid; e < nmy; e += DEC_THREADS) {
            if (tokens || key[e] < sm->thresh)
#pragma unroll
                for (int g = 0; g < G; g++) mx[g] = fmaxf(mx[g], lg[g * MY + e]);
        }
#pragma unroll
        for (int g = 0; g < G; g++) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx[g] = fmaxf(mx[g], __shfl_xor_sync(0xffffffffu, mx[g], o));
            if (lane == 0) sm->red[warp][g] = mx[g];
        }
        __syncthreads();
        float Mn[G], alpha[G];
#pragma unroll
        for (int g = 0; g < G; g++) {
            float m = sm->M[g];
            const float mold = m;
#pragma unroll
            for (int w = 0; w < W; w++) m = fmaxf(m, sm->red[w][g]);
            Mn[g] = m;
            alpha[g] = (m == -INFINITY) ? 1.f : (mold == -INFINITY ? 0.f : expf(mold - m));
            lpart[g] *= alpha[g];
        }
        for (int e = tid; e < nmy; e += DEC_THREADS) {
            const bool valid = tokens || key[e] < sm->thresh;
#pragma unroll
            for (int g = 0; g < G; g++) {
                const float pe = valid ? expf(lg[g * MY + e] - Mn[g]) : 0.f;
                pbuf[e * G + g] = pe;
                lpart[g] += pe;
            }
        }
        __syncthreads();
        if (tid < G) sm->M[tid] = Mn[tid];
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
                const float pe = pbuf[e * G + g];
                const float2 pp = make_float2(pe, pe);
#pragma unroll
                for (int c = 0; c < CPT / 2; c++) acc[g][c] = ffma2(pp, v[c], acc[g][c]);
            }
        }
    };

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
            if (rank == 0 && a.sel_out)
                for (int x = tid; x < p.k; x += DEC_THREADS)
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
        int per = (ncand + CS - 1) / CS;
        int r0 = min(ncand, rank * per), r1 = min(ncand, r0 + per);
        if (tid == 0) {
            issue(0, j, r0, r1);
            issue(1, j, r0, r1);
        }
        for (;;) {
            const int nmy = r1 - r0;
            const int P = ncand > 0 ? ncand - 1 : 0;  // query position at this level
            wait_tile(0);
            krows += ncand;
            // Scoring. A group of LPC lanes takes one candidate, PL rotation
            // pairs per lane. Index r*b + o: the key is rotated by o, the query
            // by P - r*b (angle difference), so the key needs one small table
            // row and the query is re-rotated only when the block r changes.
            {
                const int grp = lane / LPC, gl = lane % LPC;
                const int chunk = (nmy + W - 1) / W;
                const int w_lo = warp * chunk, w_hi = min(nmy, w_lo + chunk);
                constexpr int P2 = PL / 2;
                float2 qa2[G][P2], qb2[G][P2];
                int rcur = -1;
                for (int base = w_lo; base < w_hi; base += CPW) {
                    const int i = base + grp;
                    float v[G];
#pragma unroll
                    for (int g = 0; g < G; g++) v[g] = 0.f;
                    if (i < w_hi) {
                        const int rnk = r0 + i, r = rnk / b, o = rnk - r * b;
                        if (r != rcur) {  // query rotated by P - r*b
                            const float* row = p.rope + (size_t)(P - r * b) * 3 * HD + gl * PL;
                            float2 c2[P2], s2[P2], n2[P2];
                            load_tab2<PL>(row, c2);
                            load_tab2<PL>(row + HD, s2);
                            load_tab2<PL>(row + 2 * HD, n2);
#pragma unroll
                            for (int g = 0; g < G; g++)
#pragma unroll
                                for (int x = 0; x < P2; x++) {
                                    const float2 xa = make_float2(qf[g * D + gl * PL + 2 * x], qf[g * D + gl * PL + 2 * x + 1]);
                                    const float2 xb = make_float2(qf[g * D + HD + gl * PL + 2 * x],
                                                                  qf[g * D + HD + gl * PL + 2 * x + 1]);
                                    qa2[g][x] = ffma2(xa, c2[x], fmul2(xb, n2[x]));
                                    qb2[g][x] = ffma2(xb, c2[x], fmul2(xa, s2[x]));
                                }
                            rcur = r;
                        }
                        // key rotated by o
                        const float* row = p.rope + (size_t)o * 3 * HD + gl * PL;
                        float2 c2[P2], s2[P2], n2[P2], ka[P2], kb[P2];
                        load_tab2<PL>(row, c2);
                        load_tab2<PL>(row + HD, s2);
                        load_tab2<PL>(row + 2 * HD, n2);
                        load_row2<T, PL>(Kt + (size_t)i * D + gl * PL, ka);
                        load_row2<T, PL>(Kt + (size_t)i * D + HD + gl * PL, kb);
                        float2 v2[G];
#pragma unroll
                        for (int g = 0; g < G; g++) v2[g] = make_float2(0.f, 0.f);
#pragma unroll
                        for (int x = 0; x < P2; x++) {
                            const float2 ra = ffma2(ka[x], c2[x], fmul2(kb[x], n2[x]));
                            const float2 rb = ffma2(kb[x], c2[x], fmul2(ka[x], s2[x]));
#pragma unroll
                            for (int g = 0; g < G; g++) v2[g] = ffma2(qa2[g][x], ra, ffma2(qb2[g][x], rb, v2[g]));
                        }
#pragma unroll
                        for (int g = 0; g < G; g++) v[g] = v2[g].x + v2[g].y;
                    }
                    // reduce over the group's lanes; transposing while G > 1 value
                    int cnt = G, h = 0, tbits = 0;
#pragma unroll
                    for (int sft = LPC / 2; sft >= 1; sft >>= 1) {
                        if (cnt > 1) {
                            const int half = cnt / 2;
                            const bool hi = (gl & sft) != 0;
#pragma unroll
                            for (int x = 0; x < G / 2; x++) {
                                if (x < half) {
                                    const float send = hi ? v[x] : v[x + half];
                                    const float keep = hi ? v[x + half] : v[x];
                                    v[x] = keep + __shfl_xor_sync(0xffffffffu, send, sft);
                                }
                            }
                            h += hi ? half : 0;
                            tbits |= sft;
                            cnt = half;
                        } else {
                            v[0] += __shfl_xor_sync(0xffffffffu, v[0], sft);
                        }
                    }
                    const float logit = v[0] * p.scale;
                    float S = logit;
#pragma unroll
                    for (int sft = LPC / 2; sft >= 1; sft >>= 1)
                        if (tbits & sft) S += __shfl_xor_sync(0xffffffffu, S, sft);
                    if (i < w_hi && (gl & ~tbits) == 0) {
                        lg[h * MY + i] = logit;
                        if (h == 0 && j > 0) {
                            const int rnk = r0 + i, q = rnk / b;
                            key[i] = sel_key(S, sm->par[q] * b + (rnk - q * b));
                        }
                    }
                }
            }
            __syncthreads();  // logits and keys of every warp in place; key tile free

            if (j == 0) {
                wait_tile(1);
                accumulate(nmy, true);
                vrows += ncand;
                break;
            }
            const int kk = max(1, min(p.k, ncand));
            unsigned long long* mybuf = sm->topbuf[j & 1];
            // local top-kk: each key's rank among this CTA's keys (two threads per key)
            for (int base2 = warp * 32; base2 < 2 * nmy; base2 += DEC_THREADS) {
                const int x = base2 + lane, e = x >> 1, half = x & 1;
                const bool act = x < 2 * nmy;
                const unsigned long long kt = act ? key[e] : 0ull;
                const int lo = half ? nmy / 2 : 0, hi = half ? nmy : nmy / 2;
                int c = act ? rank_among(key + lo, hi - lo, kt) : 0;
                c += __shfl_xor_sync(0xffffffffu, c, 1);
                if (act && half == 0 && c < kk) mybuf[c] = kt;
            }
            if (tid >= nmy && tid < kk) mybuf[tid] = 0ull;
            cluster.sync();
            // global top-kk: merge the CTAs' sorted lists (same result in every CTA)
            const int total = CS * kk;
            for (int t = tid; t < total; t += DEC_THREADS)
                gkeys[t] = cluster.map_shared_rank(mybuf, t / kk)[t % kk];
            __syncthreads();
            for (int base2 = warp * 32; base2 < 2 * total; base2 += DEC_THREADS) {
                const int x = base2 + lane, t = x >> 1, half = x & 1;
                const bool act = x < 2 * total;
                const unsigned long long kt = act ? gkeys[t] : 0ull;
                const int lo = half ? total / 2 : 0, hi = half ? total : total / 2;
                int c = (act && kt != 0ull) ? rank_among(gkeys + lo, hi - lo, kt) : 0;
                c += __shfl_xor_sync(0xffffffffu, c, 1);
                if (act && half == 0 && kt != 0ull && c < kk) sm->picked[c] = kt;
            }
            __syncthreads();
            if (tid < kk) {  // kept ids in ascending order (ids are distinct)
                const int id = (int)key_id(sm->picked[tid]);
                int pos = 0;
                for (int r = 0; r < kk; r++) pos += (int)key_id(sm->picked[r]) < id;
                sm->chosen[pos] = id;
            }
            if (tid == 0) sm->thresh = sm->picked[kk - 1];
            __syncthreads();
            if (rank == 0 && a.sel_out)
                for (int x = tid; x < p.k; x += DEC_THREADS)
                    a.sel_out[(u * p.J_cap + (j - 1)) * p.k + x] = x < kk ? sm->chosen[x] : -1;
            if (tid < kk) sm->par[tid] = sm->chosen[tid];
            __syncthreads();
            // the next level's candidates are the children of the kept nodes
            const int nc_next = ncand_of(j - 1, kk);
            if (nc_next < 1) {
                bad = true;
                if (tid == 0) flag_error(p.err, ERR_SHAPE);
            }
            const int per_n = (nc_next + CS - 1) / CS;
            const int r0n = min(nc_next, rank * per_n), r1n = min(nc_next, r0n + per_n);
            if (tid == 0) issue(0, j - 1, r0n, r1n);  // key tile is free since the barriers above
            wait_tile(1);
            accumulate(nmy, false);  // summaries of the candidates not kept
            vrows += ncand - kk;
            __syncthreads();         // value tile and weights consumed
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
    for (int idx = tid; idx < G * D; idx += DEC_THREADS) {
        float s = 0.f;
#pragma unroll
        for (int x = 0; x < NEG; x++) s += egacc[x * G * D + idx];
        cacc[idx] = s;
    }
    if (tid < G) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < W; w++) s += sm->red[w][tid];
        cml[tid] = sm->M[tid];
        cml[G + tid] = s;
    }
    cluster.sync();  // every CTA is done with its tiles: rank 0's gather area is free
    {
        float* dst = cluster.map_shared_rank(gat, 0) + rank * (G * D + 2 * G);
        for (int idx = tid; idx < G * D + 2 * G; idx += DEC_THREADS) dst[idx] = idx < G * D ? cacc[idx] : cml[idx - G * D];
    }
    cluster.sync();  // the gather area of rank 0 is complete
    if (rank == 0) {
        T* outp = reinterpret_cast<T*>(a.out) + (u * G) * D;
        const int stride = G * D + 2 * G;
        for (int idx = tid; idx < G * D; idx += DEC_THREADS) {
            const int g = idx / D;
            float M = -INFINITY;
            for (int r = 0; r < CS; r++) M = fmaxf(M, gat[r * stride + G * D + g]);
            float s = 0.f, lsum = 0.f;
            for (int r = 0; r < CS; r++) {
                const float mr = gat[r * stride + G * D + g];
                const float f = (mr == -INFINITY) ? 0.f : expf(mr - M);
                s += gat[r * stride + idx] * f;
                lsum += gat[r * stride + G * D + G + g] * f;
            }
            outp[idx] = from_f<T>(bad ? 0.f : s / lsum);
        }
        if (tid == 0 && a.rows_out) {
            a.rows_out[u * 2] = krows;
            a.rows_out[u * 2 + 1] = vrows;
        }
        if (a.sel_out) {
            int J = 0;
            if (!bad_len) {
                J = 1;
                while (J < p.J_cap && sm->nlev[J] > b) J++;
            }
            for (int i = tid; i < (p.J_cap - J) * p.k; i += DEC_THREADS)
                a.sel_out[(u * p.J_cap + J) * p.k + i] = -1;
        }
    }
}

template <typename T, int D, int G>
cudaError_t launch_decode(const TreeParams& p, const void* q, void* out, int* sel_out, long long* rows_out,
                          cudaStream_t s) {
    const int CS = DEC_CLUSTER;
    const long long maxc = (long long)p.k * p.b > p.b ? (long long)p.k * p.b : p.b;
    DecodeArgs a{q, out, sel_out, rows_out, (int)((maxc + CS - 1) / CS), 0};
    a.region0 = (int)decode_region0(D, G, a.my_max, (int)sizeof(T));
    const size_t smem = a.region0 + decode_smem_tail(D, G, a.my_max);
    auto kern = decode_kernel<T, D, G>;
    static bool attr_set = false;  // per instantiation
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    if (smem > 227 * 1024) return cudaErrorInvalidValue;
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
    // may start while the previous kernel on the stream (the append) finishes;
    // the kernel waits for it before reading the tree
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, p, a);
}

#define RECSA_INST_DEC(T, D, G) \
    template cudaError_t launch_decode<T, D, G>(const TreeParams&, const void*, void*, int*, long long*, cudaStream_t);
#define RECSA_INST_DEC_G(T, D) RECSA_INST_DEC(T, D, 1) RECSA_INST_DEC(T, D, 2) RECSA_INST_DEC(T, D, 4) RECSA_INST_DEC(T, D, 8)
RECSA_INST_DEC_G(float, 64)
RECSA_INST_DEC_G(float, 128)
RECSA_INST_DEC_G(__nv_bfloat16, 64)
RECSA_INST_DEC_G(__nv_bfloat16, 128)

}  // namespace recsa
