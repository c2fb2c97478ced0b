// Gradients of a decode query's output, with the selections held fixed.
//
// Method (RecSA abstract; kongchang.com article "Core Idea", "Position
// Encoding"): the output of a query head is one softmax over the summaries of
// the candidates that were not kept (node key and value at level j >= 1) and
// the exact tokens under the kept level-1 nodes, each RoPE-rotated at its
// index among its level's candidates, the query at the last index. A node's
// value is the mean of its subtree's token values and its key the pooler W
// applied to the mean of its children's keys, so the gradient reaches every
// token and W through the summaries. The top-k choice is discrete: it is
// held fixed (the caller passes the selections the forward made).
//
// Two stages:
//  1. Entry gradients (recsa_decode_backward): per (sequence, KV head) unit,
//     a plan of the candidate lists (from the selections), one warp per
//     entry for the logits and <dout, v>, a per-unit softmax reduction, one
//     warp per entry again for
//       dl = p (<dout, v> - sum_f p_f <dout, v_f>),
//       dv_e += sum_g p dout_g,   dk_e += sum_g dl R(P - i) q_g / sqrt(d),
//       dq_g  = sum_e dl R(i - P) k_e / sqrt(d).
//     Token entries add into the caller's token gradients; node entries into
//     per-node accumulators (fp32, one row per tree node), so that any number
//     of queries can be summed before stage 2.
//  2. Propagation (recsa_tree_backward), level by level from the top:
//       g_m = acc_K[m] + h[parent],          h[m] = W^T g_m / children(m),
//       s_m = acc_V[m] / tokens(m) + s[parent],
//       dW += g_m mean_m^T  (mean_m = mean of m's stored child keys),
//     and for every token t under level-1 node m: dK_t += h[m], dV_t += s[m].
//     h and s overwrite the accumulators in place; the caller's call clears
//     them afterwards. Storage rounding of node keys and values is taken as
//     the identity.
//
// Lanes hold rotate-half pairs: lane l keeps elements l*NP .. l*NP+NP-1 of
// each half (NP = D / 64), so every rotation is lane-local and a warp reads
// each half of a row as one contiguous piece.
#include "backward.cuh"

namespace recsa {

constexpr int BWD_THREADS = 256;
constexpr int BWD_WARPS = BWD_THREADS / 32;
constexpr int BWD_ITEMS_PER_CTA = 64;  // entry kernels: candidates per CTA
constexpr int BWD_NODES_PER_PASS = BWD_WARPS;
__device__ __forceinline__ int* plan_off(int* pl) { return pl + 4; }
__device__ __forceinline__ int* plan_nc(int* pl) { return pl + 4 + (MAXJ + 1); }

// Children of node m of level j (j >= 1) over L tokens.
__device__ __forceinline__ long long n_children(const TreeParams& p, int j, long long m, long long L) {
    const long long nlow = level_rows(p, j - 1, L);
    const long long c = nlow - m * p.b;
    return c < p.b ? c : p.b;
}

// Tokens under node m of level j over L tokens.
__device__ __forceinline__ long long n_tokens(const TreeParams& p, int j, long long m, long long L) {
    const long long c = L - m * p.span[j];
    return c < p.span[j] ? c : p.span[j];
}

// This lane's pair elements of a row: lo[i] = x[l*NP + i], hi[i] = x[D/2 + l*NP + i].
template <typename T, int D>
__device__ __forceinline__ void load_pairs(const T* row, int lane, float* lo, float* hi) {
    constexpr int NP = D / 64;
    if constexpr (NP == 1) {
        lo[0] = to_f(row[lane]);
        hi[0] = to_f(row[D / 2 + lane]);
    } else {
        load_vec<T, NP>(row + lane * NP, lo);
        load_vec<T, NP>(row + D / 2 + lane * NP, hi);
    }
}
template <int D>
__device__ __forceinline__ void store_pairs(float* row, int lane, const float* lo, const float* hi) {
    constexpr int NP = D / 64;
    if constexpr (NP == 1) {
        row[lane] = lo[0];
        row[D / 2 + lane] = hi[0];
    } else {
        *reinterpret_cast<float2*>(row + lane * NP) = make_float2(lo[0], lo[1]);
        *reinterpret_cast<float2*>(row + D / 2 + lane * NP) = make_float2(hi[0], hi[1]);
    }
}
template <int D>
__device__ __forceinline__ void add_pairs(float* row, int lane, const float* lo, const float* hi) {
    constexpr int NP = D / 64;
#pragma unroll
    for (int i = 0; i < NP; i++) {
        row[lane * NP + i] += lo[i];
        row[D / 2 + lane * NP + i] += hi[i];
    }
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// ------------------------------------------------------------------ plan

// One warp per unit: J, the candidate count of every level and where each
// level's candidates start in the unit's item list (top level first), after
// checking that the selections are a valid descent: at level j, min(k, nc_j)
// strictly ascending ids, each a candidate (top level: < n_J; below: a child
// of a node kept one level up). An invalid unit is flagged (shape bit) and
// skipped by every later kernel.
__global__ void __launch_bounds__(128) bwd_plan_kernel(TreeParams p, BwdArgs a) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long u = (long long)blockIdx.x * 4 + warp;
    if (u >= (long long)p.B * p.H) return;
    int* pl = a.plan + u * PLAN_INTS;
    const long long L = p.len[u];
    int J = 0;
    if (L >= 1) {
        for (int j = 1; j <= p.J_cap; j++)
            if (level_rows(p, j, L) <= p.b) { J = j; break; }
    }
    bool ok = L >= 1 && L <= p.cap && J >= 1;
    const int* sel = a.sel + u * p.J_cap * p.k;
    long long nc = ok ? level_rows(p, J, L) : 0, off = 0;
    int kk_up = 0;  // nodes kept one level up
    for (int j = J; j >= 1 && ok; j--) {
        if (lane == 0) {
            plan_off(pl)[j] = (int)off;
            plan_nc(pl)[j] = (int)nc;
        }
        off += nc;
        const int kk = (int)(nc < p.k ? nc : p.k);
        const long long nj = level_rows(p, j, L);
        long long kids = 0;
        bool good = true;
        for (int x = lane; x < kk; x += 32) {
            const long long m = sel[(j - 1) * p.k + x];
            bool v = m >= 0 && m < nj && (x == 0 || sel[(j - 1) * p.k + x - 1] < m);
            if (v && j < J) {  // the parent must have been kept one level up
                const long long par = m / p.b;
                bool found = false;
                for (int y = 0; y < kk_up; y++) found |= sel[j * p.k + y] == par;
                v = found;
            }
            good &= v;
            if (v) kids += n_children(p, j, m, L);
        }
        ok = __all_sync(0xffffffffu, good);
        for (int o = 16; o > 0; o >>= 1) kids += __shfl_xor_sync(0xffffffffu, kids, o);
        nc = kids;
        kk_up = kk;
    }
    if (ok && lane == 0) {
        plan_off(pl)[0] = (int)off;
        plan_nc(pl)[0] = (int)nc;
        off += nc;
    }
    if (lane == 0) {
        ok = ok && off <= a.E_cap;
        pl[0] = ok ? 1 : 0;
        pl[1] = J;
        pl[2] = ok ? (int)off : 0;
        if (!ok) flag_error(p.err, ERR_SHAPE);
    }
}

// Level, rank and node of item x of a unit's plan (levels J..0 in order).
struct Item {
    int j;
    long long i, m, P;
};
__device__ __forceinline__ Item plan_item(const TreeParams& p, const int* sel, const int* off, const int* nc, int J,
                                          int x) {
    int j = J;
    while (j > 0 && x >= off[j] + nc[j]) j--;
    Item it;
    it.j = j;
    it.i = x - off[j];
    it.P = nc[j] - 1;
    if (j == J)
        it.m = it.i;
    else
        it.m = (long long)sel[j * p.k + it.i / p.b] * p.b + it.i % p.b;  // children of the kept nodes of level j + 1
    return it;
}

// Whether node m of level j >= 1 was kept (then it is not an entry).
__device__ __forceinline__ bool kept(const TreeParams& p, const int* sel, int j, long long m, long long nc) {
    const int kk = (int)(nc < p.k ? nc : p.k);
    bool f = false;
    for (int y = 0; y < kk; y++) f |= sel[(j - 1) * p.k + y] == m;
    return f;
}

// Shared by the two entry kernels: the unit's plan and this warp's view of
// the query heads and output gradients.
struct BwdUnit {
    int off[MAXJ + 1], nc[MAXJ + 1];
    int J, items, valid;
};

template <typename T, int D>
__device__ __forceinline__ const T* entry_row(const TreeParams& p, const TokenMap& tok, int j, long long u,
                                              long long m, bool value) {
    if (j >= 1) {
        const T* base = reinterpret_cast<const T*>(value ? p.V[j] : p.K[j]);
        return base + (u * p.rows[j] + m) * D;
    }
    const T* base = reinterpret_cast<const T*>(value ? p.V[0] : p.K[0]);
    return base + token_row(tok, u, m) * D;
}

// R(delta) x on this lane's pairs: table row delta = [cos | sin | -sin].
template <int D>
__device__ __forceinline__ void rot_pairs(const float* tab, int lane, const float* lo, const float* hi, bool inverse,
                                          float* ylo, float* yhi) {
    constexpr int NP = D / 64;
#pragma unroll
    for (int i = 0; i < NP; i++) {
        const int c = lane * NP + i;
        const float cs = __ldg(tab + c), sn = inverse ? __ldg(tab + D + c) : __ldg(tab + D / 2 + c);
        ylo[i] = lo[i] * cs - hi[i] * sn;
        yhi[i] = hi[i] * cs + lo[i] * sn;
    }
}

template <int D, int G>
__device__ __forceinline__ void load_unit(const TreeParams& p, const BwdArgs& a, long long u, int lane,
                                          BwdUnit* su, float (*ql)[D / 64], float (*qh)[D / 64], float (*dl)[D / 64],
                                          float (*dh)[D / 64], bool is_bf16) {
    constexpr int NP = D / 64;
#pragma unroll
    for (int g = 0; g < G; g++) {
        const long long row = (u * G + g) * D;
        if (is_bf16) {
            load_pairs<__nv_bfloat16, D>(reinterpret_cast<const __nv_bfloat16*>(a.q) + row, lane, ql[g], qh[g]);
            load_pairs<__nv_bfloat16, D>(reinterpret_cast<const __nv_bfloat16*>(a.dout) + row, lane, dl[g], dh[g]);
        } else {
            load_pairs<float, D>(reinterpret_cast<const float*>(a.q) + row, lane, ql[g], qh[g]);
            load_pairs<float, D>(reinterpret_cast<const float*>(a.dout) + row, lane, dl[g], dh[g]);
        }
    }
    (void)NP;
    (void)su;
}

__device__ __forceinline__ void read_plan(const BwdArgs& a, long long u, BwdUnit* su, int tid) {
    const int* pl = a.plan + u * PLAN_INTS;
    if (tid <= MAXJ) {
        su->off[tid] = pl[4 + tid];
        su->nc[tid] = pl[4 + MAXJ + 1 + tid];
    }
    if (tid == 0) {
        su->valid = pl[0];
        su->J = pl[1];
        su->items = pl[2];
    }
}

// --------------------------------------------------- entry logits, <dout, v>

template <typename T, int D, int G>
__global__ void __launch_bounds__(BWD_THREADS) bwd_score_kernel(TreeParams p, BwdArgs a) {
    constexpr int NP = D / 64;
    __shared__ BwdUnit su;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long u = blockIdx.y;
    read_plan(a, u, &su, tid);
    __syncthreads();
    const int x0 = blockIdx.x * BWD_ITEMS_PER_CTA;
    if (!su.valid || x0 >= su.items) return;
    float ql[G][NP], qh[G][NP], dl[G][NP], dh[G][NP];
    load_unit<D, G>(p, a, u, lane, &su, ql, qh, dl, dh, sizeof(T) == 2);
    const TokenMap tok = token_map(p);
    const int* sel = a.sel + u * p.J_cap * p.k;
    const int x1 = min(x0 + BWD_ITEMS_PER_CTA, su.items);
    for (int x = x0 + warp; x < x1; x += BWD_WARPS) {
        const Item it = plan_item(p, sel, su.off, su.nc, su.J, x);
        float* lgx = a.lg + (u * a.E_cap + x) * G;
        float* agx = a.ag + (u * a.E_cap + x) * G;
        if (it.j >= 1 && kept(p, sel, it.j, it.m, su.nc[it.j])) {
            if (lane < G) {
                lgx[lane] = -INFINITY;
                agx[lane] = 0.f;
            }
            continue;
        }
        float klo[NP], khi[NP], vlo[NP], vhi[NP];
        load_pairs<T, D>(entry_row<T, D>(p, tok, it.j, u, it.m, false), lane, klo, khi);
        load_pairs<T, D>(entry_row<T, D>(p, tok, it.j, u, it.m, true), lane, vlo, vhi);
        const float* tab = p.rope + (it.P - it.i) * 3 * (D / 2);
        float lgv[G], agv[G];
#pragma unroll
        for (int g = 0; g < G; g++) {
            float rl[NP], rh[NP];
            rot_pairs<D>(tab, lane, ql[g], qh[g], false, rl, rh);
            float s = 0.f, t = 0.f;
#pragma unroll
            for (int i = 0; i < NP; i++) {
                s += rl[i] * klo[i] + rh[i] * khi[i];
                t += dl[g][i] * vlo[i] + dh[g][i] * vhi[i];
            }
            lgv[g] = warp_sum(s) * p.scale;
            agv[g] = warp_sum(t);
        }
        if (lane == 0) {
#pragma unroll
            for (int g = 0; g < G; g++) {
                lgx[g] = lgv[g];
                agx[g] = agv[g];
            }
        }
    }
}

// One CTA per unit: per query head the softmax maximum M, denominator S and
// D = sum_e p_e <dout, v_e>; clears the unit's dq rows.
template <int D, int G>
__global__ void __launch_bounds__(BWD_THREADS) bwd_stats_kernel(TreeParams p, BwdArgs a) {
    __shared__ float red[BWD_WARPS][G];
    __shared__ float Ms[G];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long u = blockIdx.x;
    for (int i = tid; i < G * D; i += BWD_THREADS) a.dq[u * G * D + i] = 0.f;
    const int* pl = a.plan + u * PLAN_INTS;
    const int items = pl[0] ? pl[2] : 0;
    const float* lg = a.lg + u * a.E_cap * G;
    const float* ag = a.ag + u * a.E_cap * G;
    float m[G];
#pragma unroll
    for (int g = 0; g < G; g++) m[g] = -INFINITY;
    for (int x = tid; x < items; x += BWD_THREADS)
#pragma unroll
        for (int g = 0; g < G; g++) m[g] = fmaxf(m[g], lg[x * G + g]);
#pragma unroll
    for (int g = 0; g < G; g++) {
        float v = m[g];
        for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (lane == 0) red[warp][g] = v;
    }
    __syncthreads();
    if (tid < G) {
        float v = -INFINITY;
        for (int w = 0; w < BWD_WARPS; w++) v = fmaxf(v, red[w][tid]);
        Ms[tid] = v;
    }
    __syncthreads();
    float s[G], t[G];
#pragma unroll
    for (int g = 0; g < G; g++) s[g] = t[g] = 0.f;
    for (int x = tid; x < items; x += BWD_THREADS)
#pragma unroll
        for (int g = 0; g < G; g++) {
            const float e = expf(lg[x * G + g] - Ms[g]);  // -inf entries give 0
            s[g] += e;
            t[g] += e * ag[x * G + g];
        }
    __shared__ float rs[BWD_WARPS][G], rt[BWD_WARPS][G];
#pragma unroll
    for (int g = 0; g < G; g++) {
        const float vs = warp_sum(s[g]), vt = warp_sum(t[g]);
        if (lane == 0) {
            rs[warp][g] = vs;
            rt[warp][g] = vt;
        }
    }
    __syncthreads();
    if (tid < G) {
        float S = 0.f, Tt = 0.f;
        for (int w = 0; w < BWD_WARPS; w++) {
            S += rs[w][tid];
            Tt += rt[w][tid];
        }
        float* st = a.st + (u * G + tid) * 3;
        st[0] = Ms[tid];
        st[1] = S;
        st[2] = S > 0.f ? Tt / S : 0.f;
    }
}

// --------------------------------------------------- entry gradients

template <typename T, int D, int G>
__global__ void __launch_bounds__(BWD_THREADS) bwd_entry_kernel(TreeParams p, BwdArgs a) {
    constexpr int NP = D / 64;
    __shared__ BwdUnit su;
    __shared__ float dqs[BWD_WARPS][G][D];
    __shared__ float sts[G][3];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long u = blockIdx.y;
    read_plan(a, u, &su, tid);
    if (tid < G * 3) sts[tid / 3][tid % 3] = a.st[u * G * 3 + tid];
    __syncthreads();
    const int x0 = blockIdx.x * BWD_ITEMS_PER_CTA;
    if (!su.valid || x0 >= su.items) return;
    float ql[G][NP], qh[G][NP], dl[G][NP], dh[G][NP];
    load_unit<D, G>(p, a, u, lane, &su, ql, qh, dl, dh, sizeof(T) == 2);
    float aql[G][NP], aqh[G][NP];  // this warp's dq partial
#pragma unroll
    for (int g = 0; g < G; g++)
#pragma unroll
        for (int i = 0; i < NP; i++) aql[g][i] = aqh[g][i] = 0.f;
    const TokenMap tok = token_map(p);
    const int* sel = a.sel + u * p.J_cap * p.k;
    const int x1 = min(x0 + BWD_ITEMS_PER_CTA, su.items);
    for (int x = x0 + warp; x < x1; x += BWD_WARPS) {
        const float* lgx = a.lg + (u * a.E_cap + x) * G;
        const float* agx = a.ag + (u * a.E_cap + x) * G;
        float pg[G], dlg[G];
        bool any = false;
#pragma unroll
        for (int g = 0; g < G; g++) {
            const float l = lgx[g];
            pg[g] = l == -INFINITY ? 0.f : expf(l - sts[g][0]) / sts[g][1];
            dlg[g] = pg[g] * (agx[g] - sts[g][2]);
            any |= l != -INFINITY;
        }
        if (!any) continue;  // a kept node: not an entry
        const Item it = plan_item(p, sel, su.off, su.nc, su.J, x);
        float klo[NP], khi[NP];
        load_pairs<T, D>(entry_row<T, D>(p, tok, it.j, u, it.m, false), lane, klo, khi);
        const float* tab = p.rope + (it.P - it.i) * 3 * (D / 2);
        float gkl[NP], gkh[NP], gvl[NP], gvh[NP], rkl[NP], rkh[NP];
#pragma unroll
        for (int i = 0; i < NP; i++) gkl[i] = gkh[i] = gvl[i] = gvh[i] = 0.f;
        rot_pairs<D>(tab, lane, klo, khi, true, rkl, rkh);  // R(i - P) k
#pragma unroll
        for (int g = 0; g < G; g++) {
            float rl[NP], rh[NP];
            rot_pairs<D>(tab, lane, ql[g], qh[g], false, rl, rh);  // R(P - i) q
            const float c = dlg[g] * p.scale;
#pragma unroll
            for (int i = 0; i < NP; i++) {
                gkl[i] += c * rl[i];
                gkh[i] += c * rh[i];
                gvl[i] += pg[g] * dl[g][i];
                gvh[i] += pg[g] * dh[g][i];
                aql[g][i] += c * rkl[i];
                aqh[g][i] += c * rkh[i];
            }
        }
        float* rk;
        float* rv;
        if (it.j >= 1) {
            rk = a.gK[it.j] + (u * p.rows[it.j] + it.m) * D;
            rv = a.gV[it.j] + (u * p.rows[it.j] + it.m) * D;
        } else {
            const long long row = token_row(tok, u, it.m);
            rk = a.dk + row * D;
            rv = a.dv + row * D;
        }
        add_pairs<D>(rk, lane, gkl, gkh);
        add_pairs<D>(rv, lane, gvl, gvh);
    }
    // dq: this CTA's partial, summed over its warps, added once per element
#pragma unroll
    for (int g = 0; g < G; g++)
#pragma unroll
        for (int i = 0; i < NP; i++) {
            dqs[warp][g][lane * NP + i] = aql[g][i];
            dqs[warp][g][D / 2 + lane * NP + i] = aqh[g][i];
        }
    __syncthreads();
    for (int e = tid; e < G * D; e += BWD_THREADS) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < BWD_WARPS; w++) s += dqs[w][e / D][e % D];
        atomicAdd(a.dq + u * G * D + e, s);
    }
}

// ------------------------------------------------------- propagation

// Shared memory of the propagation kernels: W (fp32, W[r][c] at r * D + c)
// and the staged (g, mean) pairs of one pass of nodes.
template <int D>
struct PropSmem {
    float W[D * D];
    float g[BWD_NODES_PER_PASS][D];
    float mean[BWD_NODES_PER_PASS][D];
};

// Each thread owns D*D/256 consecutive elements of one row of dW:
// row r = tid % D, columns [cb * CW, (cb + 1) * CW) with cb = tid / D.
template <int D>
__device__ __forceinline__ void accumulate_dw(const PropSmem<D>& sm, int tid, float* acc) {
    constexpr int CW = D * D / BWD_THREADS;
    const int r = tid % D, cb = tid / D;
#pragma unroll 1
    for (int w = 0; w < BWD_NODES_PER_PASS; w++) {
        const float gr = sm.g[w][r];
        if (gr == 0.f) continue;
        const float4* mrow = reinterpret_cast<const float4*>(&sm.mean[w][cb * CW]);
#pragma unroll
        for (int c = 0; c < CW / 4; c++) {
            const float4 mv = mrow[c];
            acc[4 * c] += gr * mv.x;
            acc[4 * c + 1] += gr * mv.y;
            acc[4 * c + 2] += gr * mv.z;
            acc[4 * c + 3] += gr * mv.w;
        }
    }
}

template <int D>
__device__ __forceinline__ void flush_dw(float* dw, int tid, const float* acc) {
    constexpr int CW = D * D / BWD_THREADS;
    const int r = tid % D, cb = tid / D;
#pragma unroll
    for (int c = 0; c < CW; c++)
        if (acc[c] != 0.f) atomicAdd(dw + r * D + cb * CW + c, acc[c]);
}

template <typename T, int D>
__device__ __forceinline__ void load_w(const TreeParams& p, PropSmem<D>& sm, int tid) {
    const T* wt = reinterpret_cast<const T*>(p.Wt);  // Wt[c * D + r] = W[r][c]
    for (int i = tid; i < D * D; i += BWD_THREADS) {
        const int c = i / D, r = i % D;
        sm.W[r * D + c] = to_f(wt[i]);
    }
}

// h = W^T g / n on this lane's pairs; g is the warp's staged row.
template <int D>
__device__ __forceinline__ void wt_times(const PropSmem<D>& sm, const float* g, int lane, float inv_n, float* hlo,
                                         float* hhi) {
    constexpr int NP = D / 64;
#pragma unroll
    for (int i = 0; i < NP; i++) hlo[i] = hhi[i] = 0.f;
#pragma unroll 4
    for (int r = 0; r < D; r++) {
        const float gr = g[r];
#pragma unroll
        for (int i = 0; i < NP; i++) {
            hlo[i] += sm.W[r * D + lane * NP + i] * gr;
            hhi[i] += sm.W[r * D + D / 2 + lane * NP + i] * gr;
        }
    }
#pragma unroll
    for (int i = 0; i < NP; i++) {
        hlo[i] *= inv_n;
        hhi[i] *= inv_n;
    }
}

// Level j (1..J_cap): one warp per node, BWD_NODES_PER_PASS nodes per pass,
// `passes` passes per CTA. At level 1 the warp also adds h and s into the
// gradients of the node's tokens.
template <typename T, int D>
__global__ void __launch_bounds__(BWD_THREADS) bwd_prop_kernel(TreeParams p, BwdArgs a, int j, int passes) {
    constexpr int NP = D / 64;
    constexpr int CW = D * D / BWD_THREADS;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    PropSmem<D>& sm = *reinterpret_cast<PropSmem<D>*>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long u = blockIdx.y;
    const long long L = p.len[u];
    const long long nj = L >= 1 ? level_rows(p, j, L) : 0;
    const long long m_first = (long long)blockIdx.x * passes * BWD_NODES_PER_PASS;
    if (m_first >= nj) return;
    load_w<T, D>(p, sm, tid);
    float acc[CW];
#pragma unroll
    for (int c = 0; c < CW; c++) acc[c] = 0.f;
    const TokenMap tok = token_map(p);
    const bool top = j == p.J_cap;
    for (int pass = 0; pass < passes; pass++) {
        const long long m = m_first + (long long)pass * BWD_NODES_PER_PASS + warp;
        __syncthreads();  // W loaded / the previous pass's rows consumed
        float glo[NP], ghi[NP], slo[NP], shi[NP], mlo[NP], mhi[NP];
#pragma unroll
        for (int i = 0; i < NP; i++) glo[i] = ghi[i] = slo[i] = shi[i] = mlo[i] = mhi[i] = 0.f;
        long long nch = 0;
        const bool live = m < nj;
        if (live) {
            float* gk = a.gK[j] + (u * p.rows[j] + m) * D;
            float* gv = a.gV[j] + (u * p.rows[j] + m) * D;
            load_pairs<float, D>(gk, lane, glo, ghi);
            load_pairs<float, D>(gv, lane, slo, shi);
            const float inv_t = 1.f / (float)n_tokens(p, j, m, L);
#pragma unroll
            for (int i = 0; i < NP; i++) {
                slo[i] *= inv_t;
                shi[i] *= inv_t;
            }
            if (!top) {  // the parent's h and s (already propagated)
                const long long par = u * p.rows[j + 1] + m / p.b;
                float hl[NP], hh[NP], sl[NP], sh[NP];
                load_pairs<float, D>(a.gK[j + 1] + par * D, lane, hl, hh);
                load_pairs<float, D>(a.gV[j + 1] + par * D, lane, sl, sh);
#pragma unroll
                for (int i = 0; i < NP; i++) {
                    glo[i] += hl[i];
                    ghi[i] += hh[i];
                    slo[i] += sl[i];
                    shi[i] += sh[i];
                }
            }
            nch = n_children(p, j, m, L);
            // mean of the stored child keys
#pragma unroll 8
            for (long long c = 0; c < nch; c++) {
                float kl[NP], kh[NP];
                const T* row = j == 1 ? reinterpret_cast<const T*>(p.K[0]) + token_row(tok, u, m * p.b + c) * D
                                      : reinterpret_cast<const T*>(p.K[j - 1]) + (u * p.rows[j - 1] + m * p.b + c) * D;
                load_pairs<T, D>(row, lane, kl, kh);
#pragma unroll
                for (int i = 0; i < NP; i++) {
                    mlo[i] += kl[i];
                    mhi[i] += kh[i];
                }
            }
            const float inv_c = 1.f / (float)nch;
#pragma unroll
            for (int i = 0; i < NP; i++) {
                mlo[i] *= inv_c;
                mhi[i] *= inv_c;
            }
        }
#pragma unroll
        for (int i = 0; i < NP; i++) {
            sm.g[warp][lane * NP + i] = glo[i];
            sm.g[warp][D / 2 + lane * NP + i] = ghi[i];
            sm.mean[warp][lane * NP + i] = mlo[i];
            sm.mean[warp][D / 2 + lane * NP + i] = mhi[i];
        }
        __syncwarp();
        if (live) {
            float hlo[NP], hhi[NP];
            wt_times<D>(sm, sm.g[warp], lane, 1.f / (float)nch, hlo, hhi);
            if (j > 1) {  // in place: the children read h and s
                float* gk = a.gK[j] + (u * p.rows[j] + m) * D;
                float* gv = a.gV[j] + (u * p.rows[j] + m) * D;
                store_pairs<D>(gk, lane, hlo, hhi);
                store_pairs<D>(gv, lane, slo, shi);
            } else {  // the node's tokens (contiguous rows: a node never straddles a page)
                const long long row0 = token_row(tok, u, m * p.b);
                constexpr int U = 4;  // rows in flight per lane and array
                long long c = 0;
                for (; c + U <= nch; c += U) {
                    float kl[U][NP], kh[U][NP], vl[U][NP], vh[U][NP];
#pragma unroll
                    for (int x = 0; x < U; x++) {
                        load_pairs<float, D>(a.dk + (row0 + c + x) * D, lane, kl[x], kh[x]);
                        load_pairs<float, D>(a.dv + (row0 + c + x) * D, lane, vl[x], vh[x]);
                    }
#pragma unroll
                    for (int x = 0; x < U; x++) {
#pragma unroll
                        for (int i = 0; i < NP; i++) {
                            kl[x][i] += hlo[i];
                            kh[x][i] += hhi[i];
                            vl[x][i] += slo[i];
                            vh[x][i] += shi[i];
                        }
                        store_pairs<D>(a.dk + (row0 + c + x) * D, lane, kl[x], kh[x]);
                        store_pairs<D>(a.dv + (row0 + c + x) * D, lane, vl[x], vh[x]);
                    }
                }
                for (; c < nch; c++) {
                    add_pairs<D>(a.dk + (row0 + c) * D, lane, hlo, hhi);
                    add_pairs<D>(a.dv + (row0 + c) * D, lane, slo, shi);
                }
            }
        }
        __syncthreads();
        accumulate_dw<D>(sm, tid, acc);
    }
    flush_dw<D>(a.dw, tid, acc);
}

// ---------------------------------------------------------------- host

size_t bwd_prop_smem(int D) { return D == 64 ? sizeof(PropSmem<64>) : sizeof(PropSmem<128>); }

template <typename T, int D, int G>
cudaError_t launch_decode_backward(const TreeParams& p, const BwdArgs& a, cudaStream_t s) {
    const long long units = (long long)p.B * p.H;
    bwd_plan_kernel<<<(unsigned)((units + 3) / 4), 128, 0, s>>>(p, a);
    const dim3 grid((unsigned)((a.E_cap + BWD_ITEMS_PER_CTA - 1) / BWD_ITEMS_PER_CTA), (unsigned)units);
    bwd_score_kernel<T, D, G><<<grid, BWD_THREADS, 0, s>>>(p, a);
    bwd_stats_kernel<D, G><<<(unsigned)units, BWD_THREADS, 0, s>>>(p, a);
    bwd_entry_kernel<T, D, G><<<grid, BWD_THREADS, 0, s>>>(p, a);
    return cudaGetLastError();
}

// Levels J_cap .. 1 (one launch each; a level reads its parents' h and s).
template <typename T, int D>
cudaError_t launch_tree_backward(const TreeParams& p, const BwdArgs& a, long long max_len, cudaStream_t s) {
    const long long units = (long long)p.B * p.H;
    const size_t smem = sizeof(PropSmem<D>);
    static std::atomic<unsigned long long> attr_done{0};
    cudaError_t e = set_smem_limit(bwd_prop_kernel<T, D>, (int)smem, attr_done);
    if (e != cudaSuccess) return e;
    int sms = 148;
    {
        int dev = 0;
        if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    }
    const long long target = (long long)sms * 6;  // about two waves of three resident CTAs per SM
    for (int j = p.J_cap; j >= 1; j--) {
        const long long nodes = (max_len + p.span[j] - 1) / p.span[j];
        // enough nodes per CTA that the dW partials are flushed by about `target` CTAs
        long long passes = (nodes * units + target * BWD_NODES_PER_PASS - 1) / (target * BWD_NODES_PER_PASS);
        const long long most = (nodes + BWD_NODES_PER_PASS - 1) / BWD_NODES_PER_PASS;
        if (passes > most) passes = most;
        if (passes < 1) passes = 1;
        const long long per = passes * BWD_NODES_PER_PASS;
        const dim3 grid((unsigned)((nodes + per - 1) / per), (unsigned)units);
        bwd_prop_kernel<T, D><<<grid, BWD_THREADS, smem, s>>>(p, a, j, (int)passes);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

#define RECSA_INST_BWD(T, D, G) \
    template cudaError_t launch_decode_backward<T, D, G>(const TreeParams&, const BwdArgs&, cudaStream_t);
#define RECSA_INST_BWD_G(T, D) RECSA_INST_BWD(T, D, 1) RECSA_INST_BWD(T, D, 2) RECSA_INST_BWD(T, D, 4) RECSA_INST_BWD(T, D, 8)
RECSA_INST_BWD_G(float, 64)
RECSA_INST_BWD_G(float, 128)
RECSA_INST_BWD_G(__nv_bfloat16, 64)
RECSA_INST_BWD_G(__nv_bfloat16, 128)
template cudaError_t launch_tree_backward<float, 64>(const TreeParams&, const BwdArgs&, long long, cudaStream_t);
template cudaError_t launch_tree_backward<float, 128>(const TreeParams&, const BwdArgs&, long long, cudaStream_t);
template cudaError_t launch_tree_backward<__nv_bfloat16, 64>(const TreeParams&, const BwdArgs&, long long,
                                                             cudaStream_t);
template cudaError_t launch_tree_backward<__nv_bfloat16, 128>(const TreeParams&, const BwdArgs&, long long,
                                                              cudaStream_t);

}  // namespace recsa
