// One appended token per unit: the right edge of every level is refreshed
// (RecSA abstract: a node's value is the mean of the token values under it;
// its key is the layer's pooler applied to the mean of its children's keys).
//
// The arithmetic is the one the level builder uses, so a tree grown token by
// token is bit-identical to one built at once: fp32 child sums accumulated in
// child order (kept as right-edge prefix sums PK, PV), value = sum / count
// rounded once to storage, key = W . (key sum / child count) rounded once,
// the product taken as pool_product below defines it.
//
// Used by the standalone append kernel and by the decode kernel that appends
// before it descends. Every thread of the block calls it (it contains block
// barriers); thread t < D owns coordinate t, the others only take part in
// the barriers.
#pragma once

#include "common.cuh"

namespace recsa {

// P / s and P % s for 0 <= P < 2^31 and s >= 1 (s may be larger than 2^31:
// the node spans saturate), in 32-bit arithmetic.
__device__ __forceinline__ void divmod_pos(long long P, long long s, long long& q, long long& r) {
    if (s > P) {
        q = 0;
        r = P;
    } else {
        const unsigned up = (unsigned)P, us = (unsigned)s;
        const unsigned uq = up / us;
        q = uq;
        r = up - uq * us;
    }
}

// The pooler product of one output coordinate o: four fmaf chains, one per
// quarter of the input coordinate c (ascending c, starting from 0), summed as
// (y0 + y1) + (y2 + y3). Wt is the pooler transposed ([c][o]), x the input.
// Quarters [q0, q0 + 2) of the four (q0 = 0 or 2), summed: the two halves of
// the final sum can come from two threads.
template <typename T, int D>
__device__ __forceinline__ float pool_product_half(const T* Wt, const float* x, int o, int q0) {
    constexpr int Q = D / 4;
    float ya = 0.f, yb = 0.f;
    const int ca = q0 * Q, cb = (q0 + 1) * Q;
#pragma unroll 8
    for (int c = 0; c < Q; c++) {
        ya = fmaf(to_f(Wt[(ca + c) * D + o]), x[ca + c], ya);
        yb = fmaf(to_f(Wt[(cb + c) * D + o]), x[cb + c], yb);
    }
    return ya + yb;
}

// The tree sizes the append needs (a few scalars, so that the routine can be
// called out of line without the whole parameter block).
struct AppendDims {
    long long cap;
    int J_cap, b;
    const TokenMap* tok;  // where the token rows live (in shared memory)
};

// Shared memory it needs besides the pooler: km [D], part [2][D] and pre
// [J_cap][4][D] floats.
__host__ __device__ inline size_t append_scratch_floats(int D, int J_cap) { return (size_t)3 * D + 4 * (size_t)J_cap * D; }

// Appends the token at position P of unit u (k_row, v_row: its key and value,
// D elements each) to the tree. Wsm: the pooler, transposed ([c][out]), in
// shared memory once wait_w() has returned true (wait_w runs in every thread
// and must return the same answer in all of them). scratch: shared memory of
// append_scratch_floats(D, J_cap) floats. on_node(j, key, value) runs in
// thread t < D with coordinate t of the refreshed right-edge node of level j.
// lv: the levels' addresses (load_levels), in shared memory. Returns false
// (nothing of the tree written) if the pooler did not arrive.
// With at least 2D threads the pooler product is split over two threads per
// output coordinate (same arithmetic).
template <typename T, int D, typename WaitW, typename OnNode>
__device__ __forceinline__ bool append_token(const AppendDims& p, const LevelRef* lv, long long u, long long P,
                                             const T* k_row,
                                             const T* v_row, const T* Wsm, float* scratch, WaitW wait_w,
                                             OnNode on_node) {
    const int t = threadIdx.x;
    const bool own = t < D;
    const bool split = blockDim.x >= 2 * D;
    float* km = scratch;
    float* part = scratch + D;
    float* pre = scratch + 3 * D;
    T kn = from_f<T>(0.f), vn = from_f<T>(0.f);
    T* K0 = reinterpret_cast<T*>(lv[0].K);
    T* V0 = reinterpret_cast<T*>(lv[0].V);
    // per level j: prefix sums of the right edge and, if a child of level
    // j-1 completed at this token, that child's stored key and value sum
    auto load_level = [&](int j, float& pk, float& pv, float& ko, float& vo) {
        pk = pv = ko = vo = 0.f;
        if (j > p.J_cap) return;
        long long qj, rj, qm, rm;
        divmod_pos(P, lv[j].span, qj, rj);
        divmod_pos(P, lv[j - 1].span, qm, rm);
        if (rj == 0) return;  // a new node starts at this token
        pk = lv[j].PK[u * D + t];
        pv = lv[j].PV[u * D + t];
        if (rm == 0) {
            const long long c = qm - 1;  // completed child of level j-1
            if (j == 1) {
                const long long rc = token_row(*p.tok, u, c);
                ko = to_f(K0[rc * D + t]);
                vo = to_f(V0[rc * D + t]);
            } else {
                const long long row = u * lv[j - 1].rows + c;
                ko = to_f(reinterpret_cast<const T*>(lv[j - 1].K)[row * D + t]);
                vo = lv[j - 1].VS[row * D + t];
            }
        }
    };
    if (own) {
        kn = k_row[t];
        vn = v_row[t];
        // every load that does not depend on this call's results is issued
        // before the chain: the chain itself touches shared memory only
        constexpr int JU = 6;
        float r[JU][4];
#pragma unroll
        for (int jj = 0; jj < JU; jj++) load_level(jj + 1, r[jj][0], r[jj][1], r[jj][2], r[jj][3]);
#pragma unroll
        for (int jj = 0; jj < JU; jj++)
            if (jj + 1 <= p.J_cap)
#pragma unroll
                for (int x = 0; x < 4; x++) pre[((size_t)jj * 4 + x) * D + t] = r[jj][x];
        for (int j = JU + 1; j <= p.J_cap; j++) {
            float r4[4];
            load_level(j, r4[0], r4[1], r4[2], r4[3]);
            for (int x = 0; x < 4; x++) pre[((size_t)(j - 1) * 4 + x) * D + t] = r4[x];
        }
        const long long rp = token_row(*p.tok, u, P);
        K0[rp * D + t] = kn;
        V0[rp * D + t] = vn;
    }
    if (!wait_w()) return false;  // no node has been written

    float kcur = to_f(kn), vcur = to_f(vn);  // new last child of level j-1
    for (int j = 1; j <= p.J_cap; j++) {
        const long long sj = lv[j].span;
        long long m, rj, qm, rm;
        divmod_pos(P, sj, m, rj);
        divmod_pos(P, lv[j - 1].span, qm, rm);
        const bool new_node = rj == 0;
        const bool child_done = rm == 0;
        const long long row = u * lv[j].rows + m;
        T vy = from_f<T>(0.f);
        if (own) {
            const float* q4 = pre + (size_t)(j - 1) * 4 * D;
            float pk = q4[t], pv = q4[D + t];
            if (!new_node && child_done) {
                pk = pk + q4[2 * D + t];
                pv = pv + q4[3 * D + t];
            }
            if (new_node || child_done) {
                lv[j].PK[u * D + t] = pk;
                lv[j].PV[u * D + t] = pv;
            }
            const float ks = pk + kcur, vsum = pv + vcur;
            const long long cnt = rj + 1;
            const long long nc = qm - m * p.b + 1;
            lv[j].VS[row * D + t] = vsum;
            vy = from_f<T>(__fdiv_rn(vsum, (float)cnt));
            reinterpret_cast<T*>(lv[j].V)[row * D + t] = vy;
            km[t] = __fdiv_rn(ks, (float)nc);
            vcur = vsum;
        }
        __syncthreads();
        float y = 0.f;
        if (split) {
            if (t < 2 * D) part[t] = pool_product_half<T, D>(Wsm, km, t % D, 2 * (t / D));
            __syncthreads();
            if (own) y = part[t] + part[D + t];
        } else if (own) {
            y = pool_product_half<T, D>(Wsm, km, t, 0) + pool_product_half<T, D>(Wsm, km, t, 2);
        }
        if (own) {
            const T ky = from_f<T>(y);
            reinterpret_cast<T*>(lv[j].K)[row * D + t] = ky;
            kcur = to_f(ky);
            on_node(j, ky, vy);
        }
        __syncthreads();
    }
    return true;
}

}  // namespace recsa
