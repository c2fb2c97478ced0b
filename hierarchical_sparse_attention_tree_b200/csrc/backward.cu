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
#include <algorithm>

#include "backward.cuh"

namespace recsa {

constexpr int BWD_THREADS = 256;
constexpr int BWD_WARPS = BWD_THREADS / 32;
constexpr int BWD_ITEMS_PER_CTA = 64;  // entry kernels: candidates per CTA
constexpr int BWD_NODES_PER_PASS = BWD_WARPS;
constexpr int BWD_BATCH = 4;           // entries a warp has in flight at once
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
// E consecutive floats (E = 2 or 4, naturally aligned) stored at once.
template <int E>
__device__ __forceinline__ void store_vecf(float* p, const float* v) {
    if constexpr (E == 4)
        *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
    else
        *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
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

// Eight consecutive floats in one 256-bit access (sm_100); the address must
// be 32-byte aligned.
__device__ __forceinline__ void ld8f(const float* p, float* r) {
    asm volatile("ld.global.v8.f32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=f"(r[0]), "=f"(r[1]), "=f"(r[2]), "=f"(r[3]), "=f"(r[4]), "=f"(r[5]), "=f"(r[6]), "=f"(r[7])
                 : "l"(p));
}
__device__ __forceinline__ void st8f(float* p, const float* v) {
    asm volatile("st.global.v8.f32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "f"(v[0]), "f"(v[1]),
                 "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7])
                 : "memory");
}

// The level-1 sweep over one node's nch tokens (rows row0 .. row0 + nch - 1,
// contiguous): dk += h, dv += s for every token, and the sum of the tokens'
// keys returned in mc (this lane's eight columns). Each lane takes eight
// consecutive columns of a row, so a warp covers 32 / (D / 8) rows per
// access, with 256-bit loads and stores of dk and dv (32-byte aligned rows;
// the key rows aligned to eight elements). bf16 keys stay packed until they
// are added. hc, sc: h and s at this lane's columns.
template <typename T, int D>
__device__ __forceinline__ void sweep_tokens_v8(const T* K0, float* dk, float* dv, long long row0, long long nch,
                                                int lane, const float* hc, const float* sc, float* mc) {
    constexpr bool PACKED = sizeof(T) == 2;
    constexpr int LPR = D / 8, RPI = 32 / LPR;    // lanes per row, rows per access
    constexpr int UR = PACKED ? 4 : 3;            // accesses in flight per lane and array
    constexpr int KW = PACKED ? 4 : 8;            // 32-bit words of one lane's key piece
    const int rsub = lane / LPR, col = (lane % LPR) * 8;
    const T* kp = K0 + (row0 + rsub) * D + col;
    float* dkp = dk + (row0 + rsub) * D + col;
    float* dvp = dv + (row0 + rsub) * D + col;
#pragma unroll
    for (int e = 0; e < 8; e++) mc[e] = 0.f;
    auto add_row = [&](const uint32_t* kw, float* xx, float* yy) {
#pragma unroll
        for (int e = 0; e < 8; e++) {
            mc[e] += PACKED ? __uint_as_float(e & 1 ? kw[e / 2] & 0xFFFF0000u : kw[e / 2] << 16)
                            : __uint_as_float(kw[e]);
            xx[e] += hc[e];
            yy[e] += sc[e];
        }
    };
    auto load_key = [&](const T* src, uint32_t* kw) {
        if constexpr (PACKED) {
            const uint4 v = *reinterpret_cast<const uint4*>(src);
            kw[0] = v.x;
            kw[1] = v.y;
            kw[2] = v.z;
            kw[3] = v.w;
        } else {
            float t8[8];
            ld8f(reinterpret_cast<const float*>(src), t8);
#pragma unroll
            for (int e = 0; e < 8; e++) kw[e] = __float_as_uint(t8[e]);
        }
    };
    constexpr int STEP = RPI * UR;
    long long c = rsub;
    // whole groups: every row of the UR accesses exists
    for (; c + (UR - 1) * RPI < nch; c += STEP, kp += STEP * D, dkp += STEP * D, dvp += STEP * D) {
        uint32_t kw[UR][KW];
        float xx[UR][8], yy[UR][8];
#pragma unroll
        for (int x = 0; x < UR; x++) {
            load_key(kp + x * RPI * D, kw[x]);
            ld8f(dkp + x * RPI * D, xx[x]);
            ld8f(dvp + x * RPI * D, yy[x]);
        }
#pragma unroll
        for (int x = 0; x < UR; x++) {
            add_row(kw[x], xx[x], yy[x]);
            st8f(dkp + x * RPI * D, xx[x]);
            st8f(dvp + x * RPI * D, yy[x]);
        }
    }
    // the rest, one access at a time
    for (; c < nch; c += RPI, kp += RPI * D, dkp += RPI * D, dvp += RPI * D) {
        uint32_t kw[KW];
        float xx[8], yy[8];
        load_key(kp, kw);
        ld8f(dkp, xx);
        ld8f(dvp, yy);
        add_row(kw, xx, yy);
        st8f(dkp, xx);
        st8f(dvp, yy);
    }
    // the lanes that share columns (one per row of an access) add up
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1)
#pragma unroll
        for (int e = 0; e < 8; e++) mc[e] += __shfl_xor_sync(0xffffffffu, mc[e], off);
}

// Sums each of V values (V a power of two, at most 32) over the warp with
// V - 1 + 5 - log2(V) shuffles: each halving step sends half of the values
// still held and keeps the other half. Returns the sum of value `which`;
// the lanes whose lowest 5 - log2(V) bits are zero hold distinct values.
template <int V>
__device__ __forceinline__ float warp_transpose_sum(float (&v)[V], int lane, int& which) {
    int cnt = V;
    which = 0;
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) {
        if (cnt > 1) {
            const int half = cnt / 2;
            const bool hi = (lane & s) != 0;
#pragma unroll
            for (int x = 0; x < V / 2; x++)
                if (x < half) {
                    const float send = hi ? v[x] : v[x + half];
                    const float keep = hi ? v[x + half] : v[x];
                    v[x] = keep + __shfl_xor_sync(0xffffffffu, send, s);
                }
            which += hi ? half : 0;
            cnt = half;
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], s);
        }
    }
    return v[0];
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

// The unit a warp is working on: its plan (level offsets and candidate
// counts copied to the warp's slot of shared memory), its selections and
// this lane's pairs of its query heads and output gradients; reloaded
// whenever the warp's item range crosses into another unit.
template <int D, int G>
struct UnitView {
    long long u;
    int ubeg, uend, J;
    int* off;  // shared memory, MAXJ + 1 each
    int* nc;
    const int* sel;
    float ql[G][D / 64], qh[G][D / 64], dl[G][D / 64], dh[G][D / 64];
};

template <typename T, int D, int G>
__device__ __forceinline__ void load_unit(const TreeParams& p, const BwdArgs& a, long long u, int lane,
                                          UnitView<D, G>& v) {
    const int* pl = a.plan + u * PLAN_INTS;
    v.u = u;
    v.ubeg = a.ubase[u];
    v.uend = a.ubase[u + 1];
    v.J = pl[1];
    v.sel = a.sel + u * p.J_cap * p.k;
    __syncwarp();
    for (int y = lane; y <= MAXJ; y += 32) {
        v.off[y] = pl[4 + y];
        v.nc[y] = pl[4 + MAXJ + 1 + y];
    }
#pragma unroll
    for (int g = 0; g < G; g++) {
        const long long row = (u * G + g) * D;
        load_pairs<T, D>(reinterpret_cast<const T*>(a.q) + row, lane, v.ql[g], v.qh[g]);
        if (a.dout_f32)
            load_pairs<float, D>(reinterpret_cast<const float*>(a.dout) + row, lane, v.dl[g], v.dh[g]);
        else
            load_pairs<T, D>(reinterpret_cast<const T*>(a.dout) + row, lane, v.dl[g], v.dh[g]);
    }
    __syncwarp();
}

// Items xg .. xg + nb - 1 of the current unit (nb <= NI): lane t < nb works
// out item t (level, rank, node, query position, kept or not) and the warp
// receives all of them, so the item's row loads can all be in flight at once.
template <int NI>
struct Batch {
    int j[NI], i[NI], m[NI], P[NI];  // node ids fit in int: capacity < 2^31
    bool skip[NI];  // a kept node (not an entry), or past the batch
};
template <int NI, int D, int G>
__device__ __forceinline__ void batch_items(const TreeParams& p, const UnitView<D, G>& v, int xg, int nb, int lane,
                                            Batch<NI>& bt) {
    int mj = 0, mi = 0, mm = 0, mP = 0, mk = 1;
    if (lane < nb) {
        const Item it = plan_item(p, v.sel, v.off, v.nc, v.J, xg + lane - v.ubeg);
        mj = it.j;
        mi = (int)it.i;
        mm = (int)it.m;
        mP = (int)it.P;
        mk = it.j >= 1 && kept(p, v.sel, it.j, it.m, v.nc[it.j]);
    }
#pragma unroll
    for (int t = 0; t < NI; t++) {
        bt.j[t] = __shfl_sync(0xffffffffu, mj, t);
        bt.i[t] = __shfl_sync(0xffffffffu, mi, t);
        bt.m[t] = __shfl_sync(0xffffffffu, mm, t);
        bt.P[t] = __shfl_sync(0xffffffffu, mP, t);
        bt.skip[t] = __shfl_sync(0xffffffffu, mk, t) != 0;
    }
}

// The items of all units form one list (unit u's items at ubase[u] ..
// ubase[u + 1]); every warp of the grid takes one contiguous slice of it,
// so the work is balanced whatever the units' sizes.
struct Slice {
    int x0, x1;
};
__device__ __forceinline__ Slice warp_slice(const BwdArgs& a, long long units) {
    const int total = a.ubase[units];
    const long long warps = (long long)gridDim.x * BWD_WARPS;
    const long long gw = (long long)blockIdx.x * BWD_WARPS + (threadIdx.x >> 5);
    const long long per = (total + warps - 1) / warps;
    Slice sl;
    sl.x0 = (int)min((long long)total, gw * per);
    sl.x1 = (int)min((long long)total, sl.x0 + per);
    return sl;
}
// The unit holding global item x (binary search over ubase).
__device__ __forceinline__ long long unit_of(const BwdArgs& a, long long units, int x) {
    long long lo = 0, hi = units - 1;
    while (lo < hi) {
        const long long mid = (lo + hi + 1) >> 1;
        if (a.ubase[mid] <= x) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Prefix sums of the units' item counts (one CTA).
__global__ void __launch_bounds__(1024) bwd_scan_kernel(TreeParams p, BwdArgs a) {
    __shared__ int part[1024];
    const long long units = (long long)p.B * p.H;
    const int tid = threadIdx.x;
    const long long per = (units + 1023) / 1024;
    const long long u0 = tid * per, u1 = min(units, u0 + per);
    int s = 0;
    for (long long u = u0; u < u1; u++) s += a.plan[u * PLAN_INTS + 2];
    part[tid] = s;
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {  // inclusive scan
        const int v = tid >= o ? part[tid - o] : 0;
        __syncthreads();
        part[tid] += v;
        __syncthreads();
    }
    int base = tid ? part[tid - 1] : 0;
    for (long long u = u0; u < u1; u++) {
        a.ubase[u] = base;
        base += a.plan[u * PLAN_INTS + 2];
    }
    if (tid == 1023) a.ubase[units] = part[1023];
}

// --------------------------------------------------- entry logits, <dout, v>

template <typename T, int D, int G>
__global__ void __launch_bounds__(BWD_THREADS, 2) bwd_score_kernel(TreeParams p, BwdArgs a) {
    constexpr int NP = D / 64, NI = G >= 8 ? 2 : BWD_BATCH;
    __shared__ int s_plan[BWD_WARPS][2][MAXJ + 1];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long units = (long long)p.B * p.H;
    const Slice sl = warp_slice(a, units);
    if (sl.x0 >= sl.x1) return;
    const TokenMap tok = token_map(p);
    UnitView<D, G> v;
    v.off = s_plan[warp][0];
    v.nc = s_plan[warp][1];
    v.uend = 0;
    for (int xg = sl.x0; xg < sl.x1;) {
        if (xg >= v.uend) load_unit<T, D, G>(p, a, unit_of(a, units, xg), lane, v);
        const long long u = v.u;
        const int nb = min(NI, min(sl.x1, v.uend) - xg);
        Batch<NI> bt;
        batch_items<NI>(p, v, xg, nb, lane, bt);
        float klo[NI][NP], khi[NI][NP], vlo[NI][NP], vhi[NI][NP];
#pragma unroll
        for (int t = 0; t < NI; t++)
            if (!bt.skip[t]) {
                load_pairs<T, D>(entry_row<T, D>(p, tok, bt.j[t], u, bt.m[t], false), lane, klo[t], khi[t]);
                load_pairs<T, D>(entry_row<T, D>(p, tok, bt.j[t], u, bt.m[t], true), lane, vlo[t], vhi[t]);
            }
#pragma unroll
        for (int t = 0; t < NI; t++) {
            if (t >= nb) break;
            const int x = xg + t - v.ubeg;
            float* lgx = a.lg + (u * a.E_cap + x) * G;
            float* agx = a.ag + (u * a.E_cap + x) * G;
            if (bt.skip[t]) {
                if (lane < G) {
                    lgx[lane] = -INFINITY;
                    agx[lane] = 0.f;
                }
                continue;
            }
            // <R(P - i) q_g, k> = <q_g, R(i - P) k>: the key is rotated once
            const float* tab = p.rope + (bt.P[t] - bt.i[t]) * 3 * (D / 2);
            float rkl[NP], rkh[NP];
            rot_pairs<D>(tab, lane, klo[t], khi[t], true, rkl, rkh);
            float part[2 * G];  // this lane's share of the G logits, then of the G <dout_g, v>
#pragma unroll
            for (int g = 0; g < G; g++) {
                float s = 0.f, w = 0.f;
#pragma unroll
                for (int i = 0; i < NP; i++) {
                    s += v.ql[g][i] * rkl[i] + v.qh[g][i] * rkh[i];
                    w += v.dl[g][i] * vlo[t][i] + v.dh[g][i] * vhi[t][i];
                }
                part[g] = s;
                part[G + g] = w;
            }
            int which;
            const float tot = warp_transpose_sum<2 * G>(part, lane, which);
            if ((lane & (32 / (2 * G) - 1)) == 0) {  // one lane per value
                if (which < G)
                    lgx[which] = tot * p.scale;
                else
                    agx[which - G] = tot;
            }
        }
        xg += nb;
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

// Adds a warp's dq partial of unit u into dq and clears it.
template <int D, int G>
__device__ __forceinline__ void flush_dq(float* dq, long long u, int lane, float (*aql)[D / 64],
                                         float (*aqh)[D / 64]) {
    constexpr int NP = D / 64;
#pragma unroll
    for (int g = 0; g < G; g++) {
        float* row = dq + (u * G + g) * D;
#pragma unroll
        for (int i = 0; i < NP; i++) {
            if (aql[g][i] != 0.f) atomicAdd(row + lane * NP + i, aql[g][i]);
            if (aqh[g][i] != 0.f) atomicAdd(row + D / 2 + lane * NP + i, aqh[g][i]);
            aql[g][i] = aqh[g][i] = 0.f;
        }
    }
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(BWD_THREADS, 2) bwd_entry_kernel(TreeParams p, BwdArgs a) {
    constexpr int NP = D / 64, NI = G >= 8 ? 1 : BWD_BATCH;
    __shared__ int s_plan[BWD_WARPS][2][MAXJ + 1];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long units = (long long)p.B * p.H;
    const Slice sl = warp_slice(a, units);
    if (sl.x0 >= sl.x1) return;
    const TokenMap tok = token_map(p);
    UnitView<D, G> v;
    v.off = s_plan[warp][0];
    v.nc = s_plan[warp][1];
    v.uend = 0;
    v.u = -1;
    float st[G][3];
    float aql[G][NP], aqh[G][NP];  // this warp's dq partial of unit v.u
#pragma unroll
    for (int g = 0; g < G; g++)
#pragma unroll
        for (int i = 0; i < NP; i++) aql[g][i] = aqh[g][i] = 0.f;
    for (int xg = sl.x0; xg < sl.x1;) {
        if (xg >= v.uend) {
            if (v.u >= 0) flush_dq<D, G>(a.dq, v.u, lane, aql, aqh);
            load_unit<T, D, G>(p, a, unit_of(a, units, xg), lane, v);
#pragma unroll
            for (int g = 0; g < G; g++)
#pragma unroll
                for (int c = 0; c < 3; c++) st[g][c] = a.st[(v.u * G + g) * 3 + c];
        }
        const long long u = v.u;
        const int nb = min(NI, min(sl.x1, v.uend) - xg);
        Batch<NI> bt;
        batch_items<NI>(p, v, xg, nb, lane, bt);
        float klo[NI][NP], khi[NI][NP], lgt[NI][G], agt[NI][G];
#pragma unroll
        for (int t = 0; t < NI; t++)
            if (!bt.skip[t]) {
                const int x = xg + t - v.ubeg;
                load_pairs<T, D>(entry_row<T, D>(p, tok, bt.j[t], u, bt.m[t], false), lane, klo[t], khi[t]);
#pragma unroll
                for (int g = 0; g < G; g++) {
                    lgt[t][g] = a.lg[(u * a.E_cap + x) * G + g];
                    agt[t][g] = a.ag[(u * a.E_cap + x) * G + g];
                }
            }
#pragma unroll
        for (int t = 0; t < NI; t++) {
            if (bt.skip[t]) continue;
            float pg[G], dlg[G];
#pragma unroll
            for (int g = 0; g < G; g++) {
                pg[g] = expf(lgt[t][g] - st[g][0]) / st[g][1];
                dlg[g] = pg[g] * (agt[t][g] - st[g][2]);
            }
            const float* tab = p.rope + (bt.P[t] - bt.i[t]) * 3 * (D / 2);
            float gkl[NP], gkh[NP], gvl[NP], gvh[NP], rkl[NP], rkh[NP], sql[NP], sqh[NP];
#pragma unroll
            for (int i = 0; i < NP; i++) sql[i] = sqh[i] = gvl[i] = gvh[i] = 0.f;
            rot_pairs<D>(tab, lane, klo[t], khi[t], true, rkl, rkh);  // R(i - P) k
#pragma unroll
            for (int g = 0; g < G; g++) {
                const float c = dlg[g] * p.scale;
#pragma unroll
                for (int i = 0; i < NP; i++) {
                    sql[i] += c * v.ql[g][i];  // sum_g c_g q_g, rotated once below
                    sqh[i] += c * v.qh[g][i];
                    gvl[i] += pg[g] * v.dl[g][i];
                    gvh[i] += pg[g] * v.dh[g][i];
                    aql[g][i] += c * rkl[i];
                    aqh[g][i] += c * rkh[i];
                }
            }
            rot_pairs<D>(tab, lane, sql, sqh, false, gkl, gkh);  // R(P - i) sum_g c_g q_g
            float* rk = nullptr;
            float* rv = nullptr;
            if (bt.j[t] >= 1) {
                rk = a.gK[bt.j[t]] + (u * p.rows[bt.j[t]] + bt.m[t]) * D;
                rv = a.gV[bt.j[t]] + (u * p.rows[bt.j[t]] + bt.m[t]) * D;
            } else if (a.dk) {
                const long long row = token_row(tok, u, bt.m[t]);
                rk = a.dk + row * D;
                rv = a.dv + row * D;
            }
            if (rk) {
                add_pairs<D>(rk, lane, gkl, gkh);
                add_pairs<D>(rv, lane, gvl, gvh);
            }
        }
        xg += nb;
    }
    if (v.u >= 0) flush_dq<D, G>(a.dq, v.u, lane, aql, aqh);
}

// ------------------------------------------------------- propagation

// Shared memory of the propagation kernel: W in the storage type (W[r][c]
// at r * D + c), this CTA's dW partial (fp32, [D][D]) and the staged
// (g, mean) rows of one pass of nodes.
template <typename T, int D>
struct PropSmem {
    float dw[D * D];
    float g[BWD_NODES_PER_PASS][D];
    float mean[BWD_NODES_PER_PASS][D];
    float hp[D];    // a shared parent's h (pairs layout), for dW
    float msum[D];  // the pass's means summed
    T W[D * D];
};

// Each thread owns D*D/256 consecutive elements of one row of dW: row
// r = tid % D, columns [cb * CW, (cb + 1) * CW) with cb = tid / D. The
// partial stays in shared memory between passes; a pass adds the outer
// products of its staged rows.
template <typename T, int D>
__device__ __forceinline__ void accumulate_dw(PropSmem<T, D>& sm, int tid) {
    constexpr int CW = D * D / BWD_THREADS;
    const int r = tid % D, cb = tid / D;
    float gr[BWD_NODES_PER_PASS];
    bool any = false;
#pragma unroll
    for (int w = 0; w < BWD_NODES_PER_PASS; w++) {
        gr[w] = sm.g[w][r];
        any |= gr[w] != 0.f;
    }
    if (!any) return;
    float4* dst = reinterpret_cast<float4*>(&sm.dw[r * D + cb * CW]);
#pragma unroll 4
    for (int c = 0; c < CW / 4; c++) {
        float4 acc = dst[c];
#pragma unroll
        for (int w = 0; w < BWD_NODES_PER_PASS; w++) {
            const float4 mv = reinterpret_cast<const float4*>(&sm.mean[w][cb * CW])[c];
            acc.x += gr[w] * mv.x;
            acc.y += gr[w] * mv.y;
            acc.z += gr[w] * mv.z;
            acc.w += gr[w] * mv.w;
        }
        dst[c] = acc;
    }
}

// The same when the pass's nodes share one parent: g_m = own_m + hp for
// every node, so sum_m g_m mean_m^T = hp msum^T + sum_m own_m mean_m^T, and
// the own rows (sm.g) are zero but for the nodes that were entries.
template <typename T, int D>
__device__ __forceinline__ void accumulate_dw_shared(PropSmem<T, D>& sm, int tid) {
    constexpr int CW = D * D / BWD_THREADS;
    const int r = tid % D, cb = tid / D;
    const float hr = sm.hp[r];
    float gr[BWD_NODES_PER_PASS];
    bool any = false;
#pragma unroll
    for (int w = 0; w < BWD_NODES_PER_PASS; w++) {
        gr[w] = sm.g[w][r];
        any |= gr[w] != 0.f;
    }
    if (!any && hr == 0.f) return;
    float4* dst = reinterpret_cast<float4*>(&sm.dw[r * D + cb * CW]);
#pragma unroll 4
    for (int c = 0; c < CW / 4; c++) {
        float4 acc = dst[c];
        const float4 ms = reinterpret_cast<const float4*>(&sm.msum[cb * CW])[c];
        acc.x += hr * ms.x;
        acc.y += hr * ms.y;
        acc.z += hr * ms.z;
        acc.w += hr * ms.w;
        if (any) {
#pragma unroll
            for (int w = 0; w < BWD_NODES_PER_PASS; w++) {
                if (gr[w] == 0.f) continue;
                const float4 mv = reinterpret_cast<const float4*>(&sm.mean[w][cb * CW])[c];
                acc.x += gr[w] * mv.x;
                acc.y += gr[w] * mv.y;
                acc.z += gr[w] * mv.z;
                acc.w += gr[w] * mv.w;
            }
        }
        dst[c] = acc;
    }
}

// h = W^T g / n on this lane's pairs; g is the warp's staged row.
template <typename T, int D>
__device__ __forceinline__ void wt_times(const PropSmem<T, D>& sm, const float* g, int lane, float inv_n, float* hlo,
                                         float* hhi) {
    constexpr int NP = D / 64;
#pragma unroll
    for (int i = 0; i < NP; i++) hlo[i] = hhi[i] = 0.f;
#pragma unroll 4
    for (int r = 0; r < D; r++) {
        const float gr = g[r];
        float wl[NP], wh[NP];
        load_pairs<T, D>(sm.W + r * D, lane, wl, wh);
#pragma unroll
        for (int i = 0; i < NP; i++) {
            hlo[i] += wl[i] * gr;
            hhi[i] += wh[i] * gr;
        }
    }
#pragma unroll
    for (int i = 0; i < NP; i++) {
        hlo[i] *= inv_n;
        hhi[i] *= inv_n;
    }
}

// Level j (1..J_cap), persistent: the grid walks chunks of
// BWD_NODES_PER_PASS consecutive nodes of one unit (one node per warp) with
// a grid stride. Per node: g = acc_K + parent h, s = acc_V / tokens + parent
// s, h = W^T g / children, and the mean of the stored child keys (for dW).
// Level j > 1 writes h and s in place for the level below; level 1 adds them
// into the node's tokens' dk and dv in the same pass that reads the tokens'
// keys for the mean.
template <typename T, int D>
__global__ void __launch_bounds__(BWD_THREADS, 2)
    bwd_prop_kernel(TreeParams p, BwdArgs a, int j, long long chunks_per_unit) {
    constexpr int NP = D / 64;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    PropSmem<T, D>& sm = *reinterpret_cast<PropSmem<T, D>*>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    {
        const T* wt = reinterpret_cast<const T*>(p.Wt);  // Wt[c * D + r] = W[r][c]
        for (int i = tid; i < D * D; i += BWD_THREADS) {
            sm.W[(i % D) * D + i / D] = wt[i];
            sm.dw[i] = 0.f;
        }
    }
    const TokenMap tok = token_map(p);
    const bool top = j == p.J_cap;
    const long long total = (long long)p.B * p.H * chunks_per_unit;
    // 256-bit token sweep when every row of the key cache, dk and dv starts
    // where such an access may (else 64/128-bit accesses)
    const bool wide = a.dk && (reinterpret_cast<uintptr_t>(p.K[0]) % (8 * sizeof(T))) == 0 &&
                      ((reinterpret_cast<uintptr_t>(a.dk) | reinterpret_cast<uintptr_t>(a.dv)) % 32) == 0;
    for (long long ch = blockIdx.x; ch < total; ch += gridDim.x) {
        const long long u = ch / chunks_per_unit;
        const long long m0 = (ch % chunks_per_unit) * BWD_NODES_PER_PASS;
        const long long m = m0 + warp;
        const long long L = p.len[u];
        const bool live = L >= 1 && m < level_rows(p, j, L);
        // every node of the pass under one parent (or none, at the top): its
        // W^T h comes precomputed, and dW takes one outer product for it
        const bool shared = top || (m0 / p.b == (m0 + BWD_NODES_PER_PASS - 1) / p.b);
        __syncthreads();  // W loaded / the previous pass's staged rows consumed
        float glo[NP], ghi[NP], slo[NP], shi[NP], plo[NP], phi[NP], wlo[NP], whi[NP];
#pragma unroll
        for (int i = 0; i < NP; i++) glo[i] = ghi[i] = slo[i] = shi[i] = plo[i] = phi[i] = wlo[i] = whi[i] = 0.f;
        long long nch = 1;
        if (live) {
            load_pairs<float, D>(a.gK[j] + (u * p.rows[j] + m) * D, lane, glo, ghi);
            load_pairs<float, D>(a.gV[j] + (u * p.rows[j] + m) * D, lane, slo, shi);
            const float inv_t = 1.f / (float)n_tokens(p, j, m, L);
#pragma unroll
            for (int i = 0; i < NP; i++) {
                slo[i] *= inv_t;
                shi[i] *= inv_t;
            }
            if (!top) {  // the parent's h and s (already propagated), and W^T h
                const long long par = (u * p.rows[j + 1] + m / p.b) * D;
                float sl[NP], sh[NP];
                load_pairs<float, D>(a.gK[j + 1] + par, lane, plo, phi);
                load_pairs<float, D>(a.gV[j + 1] + par, lane, sl, sh);
                if (shared) load_pairs<float, D>(a.gW[j + 1] + par, lane, wlo, whi);
#pragma unroll
                for (int i = 0; i < NP; i++) {
                    slo[i] += sl[i];
                    shi[i] += sh[i];
                }
            }
            nch = n_children(p, j, m, L);
        }
        if (!shared) {  // g = own + parent h, staged whole
#pragma unroll
            for (int i = 0; i < NP; i++) {
                glo[i] += plo[i];
                ghi[i] += phi[i];
            }
        }
        store_pairs<D>(sm.g[warp], lane, glo, ghi);  // shared: the own part only (zero unless an entry)
        if (shared && warp == 0) store_pairs<D>(sm.hp, lane, plo, phi);
        __syncwarp();
        float mlo[NP], mhi[NP];
#pragma unroll
        for (int i = 0; i < NP; i++) mlo[i] = mhi[i] = 0.f;
        bool mean_staged = false;  // the token branch writes the mean row itself
        if (live) {
            const float inv_c = 1.f / (float)nch;
            float hlo[NP], hhi[NP];
            bool own = true;
            if (shared) {
                bool nz = false;
#pragma unroll
                for (int i = 0; i < NP; i++) nz |= glo[i] != 0.f || ghi[i] != 0.f;
                own = __any_sync(0xffffffffu, nz);
            }
            if (own) {
                wt_times<T, D>(sm, sm.g[warp], lane, 1.f, hlo, hhi);
            } else {
#pragma unroll
                for (int i = 0; i < NP; i++) hlo[i] = hhi[i] = 0.f;
            }
#pragma unroll
            for (int i = 0; i < NP; i++) {  // h = (W^T g) / children, W^T g = W^T own + W^T h_parent
                hlo[i] = (hlo[i] + wlo[i]) * inv_c;
                hhi[i] = (hhi[i] + whi[i]) * inv_c;
            }
            if (j > 1) {
                // W^T h for this node's children (their shared-parent passes),
                // through the warp's mean row, which is free until the mean
                float* stage = sm.mean[warp];
                store_pairs<D>(stage, lane, hlo, hhi);
                __syncwarp();
                float xlo[NP], xhi[NP];
                wt_times<T, D>(sm, stage, lane, 1.f, xlo, xhi);
                __syncwarp();
                store_pairs<D>(a.gW[j] + (u * p.rows[j] + m) * D, lane, xlo, xhi);
                // mean of the stored child keys, then h and s in place for the children
                const T* kb = reinterpret_cast<const T*>(p.K[j - 1]) + (u * p.rows[j - 1] + m * p.b) * D;
#pragma unroll 8
                for (long long c = 0; c < nch; c++) {
                    float kl[NP], kh[NP];
                    load_pairs<T, D>(kb + c * D, lane, kl, kh);
#pragma unroll
                    for (int i = 0; i < NP; i++) {
                        mlo[i] += kl[i];
                        mhi[i] += kh[i];
                    }
                }
                store_pairs<D>(a.gK[j] + (u * p.rows[j] + m) * D, lane, hlo, hhi);
                store_pairs<D>(a.gV[j] + (u * p.rows[j] + m) * D, lane, slo, shi);
            } else if (!a.dk) {
                // pooler gradient only: the tokens' keys for the mean
                const T* kb = reinterpret_cast<const T*>(p.K[0]) + token_row(tok, u, m * p.b) * D;
#pragma unroll 8
                for (long long c = 0; c < nch; c++) {
                    float kl[NP], kh[NP];
                    load_pairs<T, D>(kb + c * D, lane, kl, kh);
#pragma unroll
                    for (int i = 0; i < NP; i++) {
                        mlo[i] += kl[i];
                        mhi[i] += kh[i];
                    }
                }
            } else if (wide) {
                // the node's tokens (contiguous rows: a node never straddles
                // a page), 256-bit accesses: h and s at this lane's eight
                // columns (the lanes of the other rows of an access hold the
                // same ones) through the warp's mean row
                float* stage = sm.mean[warp];
                const int col = (lane % (D / 8)) * 8;
                float hc[8], sc[8], mc[8];
                store_pairs<D>(stage, lane, hlo, hhi);
                __syncwarp();
                load_vec<float, 8>(stage + col, hc);
                __syncwarp();
                store_pairs<D>(stage, lane, slo, shi);
                __syncwarp();
                load_vec<float, 8>(stage + col, sc);
                sweep_tokens_v8<T, D>(reinterpret_cast<const T*>(p.K[0]), a.dk, a.dv, token_row(tok, u, m * p.b), nch,
                                      lane, hc, sc, mc);
                const float inv_n = 1.f / (float)nch;
                __syncwarp();
                if (lane < D / 8)
#pragma unroll
                    for (int e = 0; e < 8; e++) stage[col + e] = mc[e] * inv_n;
                mean_staged = true;
            } else {
                // the node's tokens (contiguous rows: a node never straddles
                // a page): their keys for the mean, dk += h, dv += s. Here no
                // rotation pairs are needed, so the rows are read and written
                // contiguously (E elements per lane, one access per row and
                // array); h and s change layout through the warp's mean row.
                constexpr int E = D / 32;
                float* stage = sm.mean[warp];
                float hc[E], sc[E], mc[E];
                const long long row0 = token_row(tok, u, m * p.b);
                store_pairs<D>(stage, lane, hlo, hhi);
                __syncwarp();
                load_vec<float, E>(stage + lane * E, hc);
                __syncwarp();
                store_pairs<D>(stage, lane, slo, shi);
                __syncwarp();
                load_vec<float, E>(stage + lane * E, sc);
#pragma unroll
                for (int e = 0; e < E; e++) mc[e] = 0.f;
                const T* kb = reinterpret_cast<const T*>(p.K[0]) + row0 * D + lane * E;
                float* dkb = a.dk + row0 * D + lane * E;
                float* dvb = a.dv + row0 * D + lane * E;
                constexpr int U = 8;  // rows in flight per lane and array
                long long c = 0;
                for (; c + U <= nch; c += U) {
                    float kx[U][E], xx[U][E], yy[U][E];
#pragma unroll
                    for (int x = 0; x < U; x++) {
                        load_vec<T, E>(kb + (c + x) * D, kx[x]);
                        load_vec<float, E>(dkb + (c + x) * D, xx[x]);
                        load_vec<float, E>(dvb + (c + x) * D, yy[x]);
                    }
#pragma unroll
                    for (int x = 0; x < U; x++) {
#pragma unroll
                        for (int e = 0; e < E; e++) {
                            mc[e] += kx[x][e];
                            xx[x][e] += hc[e];
                            yy[x][e] += sc[e];
                        }
                        store_vecf<E>(dkb + (c + x) * D, xx[x]);
                        store_vecf<E>(dvb + (c + x) * D, yy[x]);
                    }
                }
                for (; c < nch; c++) {
                    float kx[E], xx[E], yy[E];
                    load_vec<T, E>(kb + c * D, kx);
                    load_vec<float, E>(dkb + c * D, xx);
                    load_vec<float, E>(dvb + c * D, yy);
#pragma unroll
                    for (int e = 0; e < E; e++) {
                        mc[e] += kx[e];
                        xx[e] += hc[e];
                        yy[e] += sc[e];
                    }
                    store_vecf<E>(dkb + c * D, xx);
                    store_vecf<E>(dvb + c * D, yy);
                }
                const float inv_n = 1.f / (float)nch;
                __syncwarp();
#pragma unroll
                for (int e = 0; e < E; e++) stage[lane * E + e] = mc[e] * inv_n;
                mean_staged = true;
            }
#pragma unroll
            for (int i = 0; i < NP; i++) {
                mlo[i] *= inv_c;
                mhi[i] *= inv_c;
            }
        }
        if (!mean_staged) store_pairs<D>(sm.mean[warp], lane, mlo, mhi);
        __syncthreads();
        if (shared) {
            for (int c = tid; c < D; c += BWD_THREADS) {
                float t = 0.f;
#pragma unroll
                for (int w = 0; w < BWD_NODES_PER_PASS; w++) t += sm.mean[w][c];
                sm.msum[c] = t;
            }
            __syncthreads();
            accumulate_dw_shared<T, D>(sm, tid);
        } else {
            accumulate_dw<T, D>(sm, tid);
        }
    }
    __syncthreads();
    for (int i = tid; i < D * D; i += BWD_THREADS)
        if (sm.dw[i] != 0.f) atomicAdd(a.dw + i, sm.dw[i]);
}

// ---------------------------------------------------------------- host

template <typename T, int D, int G>
cudaError_t launch_decode_backward(const TreeParams& p, const BwdArgs& a, cudaStream_t s) {
    const long long units = (long long)p.B * p.H;
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    bwd_plan_kernel<<<(unsigned)((units + 3) / 4), 128, 0, s>>>(p, a);
    bwd_scan_kernel<<<1, 1024, 0, s>>>(p, a);
    // one wave of resident CTAs (no more warps than items at the cap)
    auto grid_for = [&](auto kern) {
        int per_sm = 1;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, BWD_THREADS, 0) != cudaSuccess || per_sm < 1)
            per_sm = 1;
        const long long need = (units * a.E_cap + BWD_WARPS - 1) / BWD_WARPS;
        return (unsigned)std::max(1LL, std::min(need, (long long)sms * per_sm));
    };
    bwd_score_kernel<T, D, G><<<grid_for(bwd_score_kernel<T, D, G>), BWD_THREADS, 0, s>>>(p, a);
    bwd_stats_kernel<D, G><<<(unsigned)units, BWD_THREADS, 0, s>>>(p, a);
    bwd_entry_kernel<T, D, G><<<grid_for(bwd_entry_kernel<T, D, G>), BWD_THREADS, 0, s>>>(p, a);
    return cudaGetLastError();
}

// Levels J_cap .. 1 (one launch each; a level reads its parents' h and s).
template <typename T, int D>
cudaError_t launch_tree_backward(const TreeParams& p, const BwdArgs& a, long long max_len, cudaStream_t s) {
    const long long units = (long long)p.B * p.H;
    const size_t smem = sizeof(PropSmem<T, D>);
    auto kern = bwd_prop_kernel<T, D>;
    static std::atomic<unsigned long long> attr_done{0};
    cudaError_t e = set_smem_limit(kern, (int)smem, attr_done);
    if (e != cudaSuccess) return e;
    int sms = 148, dev = 0, per_sm = 1;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, BWD_THREADS, smem);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    for (int j = p.J_cap; j >= 1; j--) {
        const long long nodes = (max_len + p.span[j] - 1) / p.span[j];
        const long long chunks = (nodes + BWD_NODES_PER_PASS - 1) / BWD_NODES_PER_PASS;
        const long long grid = std::max(1LL, std::min(chunks * units, (long long)sms * per_sm));
        kern<<<(unsigned)grid, BWD_THREADS, smem, s>>>(p, a, j, chunks);
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
