// Candidate scoring of the decode kernel (the prefill scores on tensor cores).
//
// Logit of a candidate at index i among its level's candidates, for query
// head g with the query at index P (RecSA abstract: every entry is RoPE-rotated
// at its index among the candidates of its level, the query at the last one):
//     l_g = <rope(q_g, P), rope(k, i)> / sqrt(d),
// and its selection score S = sum_g l_g (one selection per KV head). With
// i = r*b + o (o < b), only the angle difference enters the product, so the
// key is rotated by o and the query by P - r*b: the keys need only the first
// b rows of the RoPE table, and a query is re-rotated when the block r
// changes. All arithmetic is fp32 (packed f32x2 where possible).
//
// Layout: a group of LPC lanes takes one candidate, PL rotation pairs
// (x_i, x_{i + D/2}) per lane. A group scores NC candidates per step, all of
// whose loads are issued before any arithmetic (independent chains), and the
// NC x G partial dots are summed over the group's lanes by a transposing
// butterfly that ends with one value per lane.
#pragma once

#include "common.cuh"

namespace recsa {

template <int D, int G>
struct ScoreLayout {
    static constexpr int HD = D / 2;
    static constexpr int PL = G >= 8 ? 2 : 4;  // rotation pairs per lane (register budget)
    static constexpr int P2 = PL / 2;
    static constexpr int LPC = HD / PL;
    static constexpr int CPW = 32 / LPC;
    static constexpr int NC = 2;  // candidates per group and step (more made the step slower: code size, spills)
    static_assert(G <= LPC && 32 % LPC == 0 && G <= 8, "scoring layout");
};

// Rotated query (all G heads, this lane's PL pairs) at angle `angle`.
template <int D, int G>
__device__ __forceinline__ void rotate_query(const float* rope, const float* qf, int angle, int gl,
                                             float2 (*qa2)[ScoreLayout<D, G>::P2],
                                             float2 (*qb2)[ScoreLayout<D, G>::P2]) {
    using SL = ScoreLayout<D, G>;
    constexpr int HD = SL::HD, PL = SL::PL, P2 = SL::P2;
    const float* row = rope + (size_t)angle * 3 * HD + gl * PL;
    float2 c2[P2], s2[P2], n2[P2];
    load_tab2<PL>(row, c2);
    load_tab2<PL>(row + HD, s2);
    load_tab2<PL>(row + 2 * HD, n2);
#pragma unroll
    for (int g = 0; g < G; g++)
#pragma unroll
        for (int x = 0; x < P2; x++) {
            const float2 xa = make_float2(qf[g * D + gl * PL + 2 * x], qf[g * D + gl * PL + 2 * x + 1]);
            const float2 xb = make_float2(qf[g * D + HD + gl * PL + 2 * x], qf[g * D + HD + gl * PL + 2 * x + 1]);
            qa2[g][x] = ffma2(xa, c2[x], fmul2(xb, n2[x]));
            qb2[g][x] = ffma2(xb, c2[x], fmul2(xa, s2[x]));
        }
}

// Scores rows [0, nmy) of the key tile Kt (row i = candidate index r0 + i)
// for the query at index P (fp32 query heads qf[G][D] in shared memory); each
// of the W warps takes a contiguous slice of the rows. For every row and
// head, emit(i, h, logit, S, r, o) runs on exactly one lane, where r*b + o is
// the candidate index. If wmax is given, lane 0 stores there the warp's
// largest logit per head (-inf for heads without rows), or, with
// wmax_fold, the larger of that and the value already there.
template <typename T, int D, int G, int W, typename Emit>
__device__ __forceinline__ void score_rows(const float* rope, float scale, int b, const T* Kt, const float* qf,
                                           int r0, int nmy, int P, int warp, int lane, float* wmax, Emit emit,
                                           bool wmax_fold = false) {
    using SL = ScoreLayout<D, G>;
    constexpr int HD = SL::HD, PL = SL::PL, P2 = SL::P2, LPC = SL::LPC, CPW = SL::CPW, NC = SL::NC;
    constexpr int STEP = CPW * NC;
    const int grp = lane / LPC, gl = lane % LPC;
    const int chunk = (nmy + W - 1) / W;
    const int w_lo = warp * chunk, w_hi = min(nmy, w_lo + chunk);
    float2 qa2[G][P2], qb2[G][P2];
#pragma unroll
    for (int g = 0; g < G; g++)
#pragma unroll
        for (int x = 0; x < P2; x++) qa2[g][x] = qb2[g][x] = make_float2(0.f, 0.f);
    int rcur = -1;
    // candidate index of this lane's c-th row as block r and offset o, advanced
    // by STEP rows per iteration
    int rc[NC], oc[NC];
#pragma unroll
    for (int c = 0; c < NC; c++) {
        const int rnk = r0 + w_lo + c * CPW + grp;
        rc[c] = rnk / b;
        oc[c] = rnk - rc[c] * b;
    }
    float lmax = -INFINITY;
    int myh = 0;
    for (int base = w_lo; base < w_hi; base += STEP) {
        // candidate by candidate (rows past the slice repeat its last row and
        // are discarded); the loads do not depend on earlier candidates
        float v[NC * G];
#pragma unroll
        for (int c = 0; c < NC; c++) {
            const int i = min(base + c * CPW + grp, w_hi - 1);
            float2 c2[P2], s2[P2], ka[P2], kb[P2];
            const float* row = rope + (size_t)oc[c] * 3 * HD + gl * PL;
            load_tab2<PL>(row, c2);
            load_tab2<PL>(row + HD, s2);
            load_row2<T, PL>(Kt + (size_t)i * D + gl * PL, ka);
            load_row2<T, PL>(Kt + (size_t)i * D + HD + gl * PL, kb);
            if (base + c * CPW + grp < w_hi && rc[c] != rcur) {
                rotate_query<D, G>(rope, qf, P - rc[c] * b, gl, qa2, qb2);
                rcur = rc[c];
            }
            float2 v2[G];
#pragma unroll
            for (int g = 0; g < G; g++) v2[g] = make_float2(0.f, 0.f);
#pragma unroll
            for (int x = 0; x < P2; x++) {
                const float2 ns = make_float2(-s2[x].x, -s2[x].y);
                const float2 ra = ffma2(ka[x], c2[x], fmul2(kb[x], ns));
                const float2 rb = ffma2(kb[x], c2[x], fmul2(ka[x], s2[x]));
#pragma unroll
                for (int g = 0; g < G; g++) v2[g] = ffma2(qa2[g][x], ra, ffma2(qb2[g][x], rb, v2[g]));
            }
#pragma unroll
            for (int g = 0; g < G; g++) v[c * G + g] = v2[g].x + v2[g].y;
        }
        // transposing reduction over the group's LPC lanes: each halving step
        // sends one half of the values still held and keeps the other
        int cnt = NC * G, idx = 0, tbits = 0;
#pragma unroll
        for (int sft = LPC / 2; sft >= 1; sft >>= 1) {
            if (cnt > 1) {
                const int half = cnt / 2;
                const bool hi = (gl & sft) != 0;
#pragma unroll
                for (int x = 0; x < NC * G / 2; x++) {
                    if (x < half) {
                        const float send = hi ? v[x] : v[x + half];
                        const float keep = hi ? v[x + half] : v[x];
                        v[x] = keep + __shfl_xor_sync(0xffffffffu, send, sft);
                    }
                }
                idx += hi ? half : 0;
                tbits |= sft;
                cnt = half;
            } else {
                v[0] += __shfl_xor_sync(0xffffffffu, v[0], sft);
            }
        }
        // the lane holds value idx = c*G + h; the G heads of candidate c sit
        // on lanes that differ in the lowest log2(G) transposed lane bits
        const float logit = v[0] * scale;
        float S = logit;
        int hb = 0;
#pragma unroll
        for (int sft = 1; sft < LPC; sft <<= 1) {
            if ((tbits & sft) && hb < G - 1) {
                S += __shfl_xor_sync(0xffffffffu, S, sft);
                hb = hb * 2 + 1;
            }
        }
        const int c = idx / G, h = idx - c * G;
        const int i = base + c * CPW + grp;
        myh = h;
        int r = rc[0], o = oc[0];
#pragma unroll
        for (int x = 1; x < NC; x++)
            if (c == x) r = rc[x], o = oc[x];
        if (i < w_hi) {
            lmax = fmaxf(lmax, logit);
            if ((gl & ~tbits) == 0) emit(i, h, logit, S, r, o);
        }
#pragma unroll
        for (int x = 0; x < NC; x++) {
            oc[x] += STEP;
            if (oc[x] >= b) {
                const int q = oc[x] / b;
                rc[x] += q;
                oc[x] -= q * b;
            }
        }
    }
    if (wmax != nullptr) {
#pragma unroll
        for (int g = 0; g < G; g++) {
            float m = myh == g ? lmax : -INFINITY;
#pragma unroll
            for (int sft = 16; sft > 0; sft >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, sft));
            if (lane == 0) wmax[g] = wmax_fold ? fmaxf(wmax[g], m) : m;
        }
    }
}

}  // namespace recsa
