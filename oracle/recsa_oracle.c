/*
 * fp64 CPU oracle for RecSA tree sparse attention — TEST INFRASTRUCTURE.
 *
 * Plain, slow and meant to be checked by eye against the method's pages:
 * "Recursive Sparse Attention: Million-Token Length Extrapolation at
 * Logarithmic Cost" (arXiv 2611.07232, abstract) and the kongchang.com
 * article on RecSA ("Core Idea", "Position Encoding"). No blocking, no
 * fusion, no reordering: every quantity is formed from its definition.
 * Only the tests, the smoke check and the benchmark's CPU-baseline leg may
 * call it. It shares no code with the CUDA path.
 *
 * What the pages fix:
 *   - a tree over the KV cache; the bottom level is the exact tokens and each
 *     node summarises its subtree with one key and one value (abstract;
 *     "Core Idea");
 *   - a node's value is the mean of all token values in its subtree
 *     ("Core Idea", mean pooling paragraph);
 *   - node keys come from one pooler per layer, shared by all levels
 *     (abstract);
 *   - each level above the tokens keeps at most k candidates; queries filter
 *     at the top and drill down level by level (abstract; "Core Idea");
 *   - summaries of unselected candidates share one softmax with the exact
 *     tokens (abstract);
 *   - each entry's RoPE position is its index among the candidates of its
 *     level (abstract; "Position Encoding").
 *
 * Readings where the pages are silent (each one is a choice of this oracle):
 *   R1 pooler: a d x d linear map W (no bias) applied to the arithmetic mean
 *      of the node's children's stored keys; one W for all levels and heads.
 *   R2 top level J: the first level with at most b nodes (J >= 1).
 *   R3 the last node of each level may be partial; its value is the mean of
 *      the tokens it has, its key uses the mean of the children it has.
 *   R4 "at most k" means exactly min(k, |candidates|).
 *   R5 candidates are ordered by ascending node id; the top-k ranks by the
 *      selection score, ties going to the smaller node id.
 *   R6 at a level with n candidates the query sits at RoPE position n - 1.
 *   R7 logits are scaled by 1/sqrt(d), with no size bias; a selected node
 *      contributes no summary (its children replace it); tokens are never
 *      top-k'd.
 *   R8 decode: the query at position T-1 descends the tree over all T tokens.
 *   R9 prefill: a chunk [s, s+C) sees the tree over [0, s) plus its own
 *      causal tokens, which follow the level-0 candidates in the index order.
 *   R10 GQA: one selection per KV head, ranked by the sum of the G query
 *      heads' logits.
 *   R11 RoPE: rotate-half pairs (i, i + d/2), theta_i = base^(-2i/d).
 *   R12 node keys and values are rounded to the storage type once, when
 *      formed; child keys are read as stored.
 *   R20 LSA-style variant ("Latent Sparse Attention" abstract: keys are
 *      clustered hierarchically in a learned latent space and queries score
 *      the hierarchy of clusters; nothing more is given): a balanced
 *      hierarchical partition with the tree's own fan-out. Level j has one
 *      learned direction Z_j and the latent coordinate z_j(t) = <Z_j, k_t>
 *      (fp64, summed in index order). From the top level J down to level 1,
 *      the tokens of every block of b^(j+1) consecutive positions of the
 *      current order are sorted by (z_j, token index); the level-j nodes of
 *      the tree over the reordered tokens are then blocks of b^j positions
 *      whose z_j ranges follow one another inside their parent. The tree,
 *      the descent and the attention are the method's own over the
 *      reordered cache (a RoPE index is a position among candidates, so the
 *      tokens' original order does not enter).
 *
 * Parity unpinned: R6 at levels >= 1 (the query position there; level 0 is
 * pinned by the dense equivalence), R7's absence of a subtree-size bias, and
 * R8 are fixed only by these readings. Every other step is pinned by the
 * tests against the dense closed form, exact subtree means, the read bound,
 * an independent brute force and hand-derived examples.
 */
#include "recsa_oracle.h"

#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------ helpers */

static double tok_at(const void* p, int tok_dtype, long long idx) {
    if (tok_dtype == ORC_TOK_BF16) {
        uint32_t u = (uint32_t)((const uint16_t*)p)[idx] << 16;
        float f;
        memcpy(&f, &u, 4);
        return (double)f;
    }
    return (double)((const float*)p)[idx];
}

/* bf16 keeps 8 significant bits; nearest-even via nearbyint in the default
 * rounding mode. Subnormals keep a fixed quantum of 2^-133. */
static double round_bf16(double x) {
    if (x == 0.0 || !isfinite(x)) return x;
    int e;
    double m = frexp(x, &e); /* x = m 2^e, 0.5 <= |m| < 1 */
    int bits = 8;
    if (e + 133 < bits) bits = e + 133;
    if (bits < 0) return copysign(0.0, x);
    double y = ldexp(nearbyint(ldexp(m, bits)), e - bits);
    if (fabs(y) > 3.38953138925153547590470800371487866880e38) return copysign(INFINITY, x);
    return y;
}

double orc_round(double x, int storage) {
    if (storage == ORC_STORE_F32) return (double)(float)x;
    if (storage == ORC_STORE_BF16) return round_bf16(x);
    return x;
}

int orc_levels(long long T, int b, long long* n) {
    for (int j = 0; j <= ORC_MAXLEV; j++) n[j] = T > 0 ? 1 : 0;
    n[0] = T;
    if (T <= 0 || b < 2) return 0;
    int J = 0;
    for (int j = 1; j <= ORC_MAXLEV; j++) {
        n[j] = (n[j - 1] + b - 1) / b;
        if (J == 0 && n[j] <= b) J = j;
        if (n[j] == 1 && J != 0) break;
    }
    return J;
}

/* b^j, saturating */
static long long ipow_sat(int b, int j) {
    long long p = 1;
    for (int i = 0; i < j; i++) {
        if (p > (1LL << 61) / b) return 1LL << 61;
        p *= b;
    }
    return p;
}

/* --------------------------------------------------------------- tree */

/* The pooler (R1): y = W x for the mean x of a node's children's keys,
 * rounded to the storage type. */
static void pool_mean(const double* mean, int d, const float* W, int storage, double* out) {
    for (int r = 0; r < d; r++) {
        double y = 0.0;
        for (int c = 0; c < d; c++) y += (double)W[r * d + c] * mean[c];
        out[r] = orc_round(y, storage);
    }
}

int orc_build(const void* Ktok, const void* Vtok, int tok_dtype, long long T, int d, int b, const float* W,
              int storage, long long t_from, int J_keep, double* const* Knode, double* const* Vnode) {
    long long n[ORC_MAXLEV + 1];
    int J = orc_levels(T, b, n);
    if (J == 0) return 0;
    int Jb = J > J_keep ? J : J_keep;
    if (Jb > ORC_MAXLEV) Jb = ORC_MAXLEV;
    double* mean = (double*)malloc(sizeof(double) * (size_t)d);
    if (!mean) return -1;
    for (int j = 1; j <= Jb; j++) {
        long long span = ipow_sat(b, j); /* tokens under one node of level j */
        long long m0 = t_from / span;
        for (long long m = m0; m < n[j]; m++) {
            /* value: mean of the subtree's token values ("Core Idea") */
            long long t_lo = m * span, t_hi = (m + 1) * span < T ? (m + 1) * span : T;
            for (int i = 0; i < d; i++) {
                double s = 0.0;
                for (long long t = t_lo; t < t_hi; t++) s += tok_at(Vtok, tok_dtype, t * d + i);
                Vnode[j][m * d + i] = orc_round(s / (double)(t_hi - t_lo), storage);
            }
            /* key: pooler applied to the mean of the children's stored keys (R1) */
            long long c_lo = m * b, c_hi = (m + 1) * b < n[j - 1] ? (m + 1) * b : n[j - 1];
            for (int i = 0; i < d; i++) {
                double s = 0.0;
                for (long long c = c_lo; c < c_hi; c++)
                    s += (j == 1) ? tok_at(Ktok, tok_dtype, c * d + i) : Knode[j - 1][c * d + i];
                mean[i] = s / (double)(c_hi - c_lo);
            }
            pool_mean(mean, d, W, storage, Knode[j] + m * d);
        }
    }
    free(mean);
    return Jb;
}

int orc_pool_level(const double* child_keys, long long n_children, int d, int b, const float* W, int storage,
                   double* out) {
    if (n_children < 1 || d < 1 || b < 2) return -1;
    double* mean = (double*)malloc(sizeof(double) * (size_t)d);
    if (!mean) return -1;
    long long n = (n_children + b - 1) / b;
    for (long long m = 0; m < n; m++) {
        long long c_lo = m * b, c_hi = (m + 1) * b < n_children ? (m + 1) * b : n_children;
        for (int i = 0; i < d; i++) {
            double s = 0.0;
            for (long long c = c_lo; c < c_hi; c++) s += child_keys[c * d + i];
            mean[i] = s / (double)(c_hi - c_lo);
        }
        pool_mean(mean, d, W, storage, out + m * d);
    }
    free(mean);
    return 0;
}

/* --------------------------------------------------------------- RoPE */

/* rope(x, p): rotate-half pairs (i, i + d/2) by p * theta_i (R11). */
static void rope(const double* x, long long p, int d, double base, double* y) {
    int h = d / 2;
    for (int i = 0; i < h; i++) {
        double th = pow(base, -2.0 * (double)i / (double)d);
        double c = cos((double)p * th), s = sin((double)p * th);
        y[i] = x[i] * c - x[i + h] * s;
        y[i + h] = x[i + h] * c + x[i] * s;
    }
}

/* -------------------------------------------------------------- query */

typedef struct {
    double S;
    long long m;
} scored;

/* descending score, ascending node id on ties (R5) */
static int by_score(const void* a, const void* b) {
    const scored* x = (const scored*)a;
    const scored* y = (const scored*)b;
    if (x->S > y->S) return -1;
    if (x->S < y->S) return 1;
    return (x->m > y->m) - (x->m < y->m);
}

static int by_id(const void* a, const void* b) {
    long long x = *(const long long*)a, y = *(const long long*)b;
    return (x > y) - (x < y);
}

typedef struct {
    int level;      /* 0 = token, -1 = local token, j >= 1 = node summary */
    long long id;
} entry;

int orc_query(int d, int b, int k, int G, double rope_base, long long T, const double* const* Knode,
              const double* const* Vnode, const void* Ktok, const void* Vtok, int tok_dtype, const void* Kloc,
              const void* Vloc, long long nloc, const float* q, double* out, int* sel, double* margin,
              long long* rows) {
    if (d <= 0 || d % 2 || b < 2 || k < 1 || G < 1 || T < 0 || nloc < 0 || (T == 0 && nloc == 0)) return -1;
    long long n[ORC_MAXLEV + 1];
    int J = orc_levels(T, b, n);
    double scale = 1.0 / sqrt((double)d);

    long long max_cand = (long long)k * b > b ? (long long)k * b : b;
    long long max_entries = (long long)J * max_cand + max_cand + nloc + 1;
    long long* cand = (long long*)malloc(sizeof(long long) * (size_t)max_cand);
    long long* next = (long long*)malloc(sizeof(long long) * (size_t)max_cand);
    scored* sc = (scored*)malloc(sizeof(scored) * (size_t)max_cand);
    double* lg = (double*)malloc(sizeof(double) * (size_t)(max_cand * G));
    entry* ent = (entry*)malloc(sizeof(entry) * (size_t)max_entries);
    double* elog = (double*)malloc(sizeof(double) * (size_t)(max_entries * G));
    double* qd = (double*)malloc(sizeof(double) * (size_t)d);
    double* qr = (double*)malloc(sizeof(double) * (size_t)(G * d));
    double* kv = (double*)malloc(sizeof(double) * (size_t)d);
    double* kr = (double*)malloc(sizeof(double) * (size_t)d);
    long long* sl = (long long*)malloc(sizeof(long long) * (size_t)(k + 1));
    if (!cand || !next || !sc || !lg || !ent || !elog || !qd || !qr || !kv || !kr || !sl) {
        free(cand); free(next); free(sc); free(lg); free(ent); free(elog); free(qd); free(qr); free(kv); free(kr);
        free(sl);
        return -1;
    }
    if (sel)
        for (long long i = 0; i < (long long)J * k; i++) sel[i] = -1;
    long long n_ent = 0, k_rows = 0;

    /* the top level's candidates are all its nodes */
    long long nc = (J > 0) ? n[J] : 0;
    for (long long i = 0; i < nc; i++) cand[i] = i;

    for (int j = J; j >= 1; j--) {
        long long P = nc - 1; /* query position at this level (R6) */
        for (int g = 0; g < G; g++) {
            for (int i = 0; i < d; i++) qd[i] = (double)q[g * d + i];
            rope(qd, P, d, rope_base, qr + g * d);
        }
        for (long long i = 0; i < nc; i++) {
            const double* krow = Knode[j] + cand[i] * d;
            rope(krow, i, d, rope_base, kr); /* RoPE at the candidate's index (abstract) */
            double S = 0.0;
            for (int g = 0; g < G; g++) {
                double dot = 0.0;
                for (int e = 0; e < d; e++) dot += qr[g * d + e] * kr[e];
                lg[i * G + g] = dot * scale;
                S += lg[i * G + g];
            }
            sc[i].S = S;
            sc[i].m = cand[i];
        }
        k_rows += nc;
        qsort(sc, (size_t)nc, sizeof(scored), by_score);
        long long kk = nc < k ? nc : k; /* R4 */
        if (margin) margin[j - 1] = (nc > kk) ? sc[kk - 1].S - sc[kk].S : HUGE_VAL;
        for (long long r = 0; r < kk; r++) sl[r] = sc[r].m;
        qsort(sl, (size_t)kk, sizeof(long long), by_id);
        if (sel)
            for (long long r = 0; r < kk; r++) sel[(long long)(j - 1) * k + r] = (int)sl[r];
        /* unselected candidates enter the softmax as summaries (abstract) */
        for (long long i = 0; i < nc; i++) {
            int chosen = 0;
            for (long long r = 0; r < kk; r++) chosen |= (sl[r] == cand[i]);
            if (chosen) continue;
            ent[n_ent].level = j;
            ent[n_ent].id = cand[i];
            for (int g = 0; g < G; g++) elog[n_ent * G + g] = lg[i * G + g];
            n_ent++;
        }
        /* next candidates: children of the selected nodes, ascending (R5) */
        long long nn = 0;
        for (long long r = 0; r < kk; r++) {
            long long c_lo = sl[r] * b, c_hi = (sl[r] + 1) * b < n[j - 1] ? (sl[r] + 1) * b : n[j - 1];
            for (long long c = c_lo; c < c_hi; c++) next[nn++] = c;
        }
        memcpy(cand, next, sizeof(long long) * (size_t)nn);
        nc = nn;
    }

    /* level 0: the exact tokens under the selected leaf-parents, then the
     * local causal tokens (R9); RoPE index = rank in this list */
    long long P0 = nc + nloc - 1;
    for (int g = 0; g < G; g++) {
        for (int i = 0; i < d; i++) qd[i] = (double)q[g * d + i];
        rope(qd, P0, d, rope_base, qr + g * d);
    }
    for (long long i = 0; i < nc + nloc; i++) {
        int local = i >= nc;
        for (int e = 0; e < d; e++)
            kv[e] = local ? tok_at(Kloc, tok_dtype, (i - nc) * d + e) : tok_at(Ktok, tok_dtype, cand[i] * d + e);
        rope(kv, i, d, rope_base, kr);
        ent[n_ent].level = local ? -1 : 0;
        ent[n_ent].id = local ? i - nc : cand[i];
        for (int g = 0; g < G; g++) {
            double dot = 0.0;
            for (int e = 0; e < d; e++) dot += qr[g * d + e] * kr[e];
            elog[n_ent * G + g] = dot * scale;
        }
        n_ent++;
    }
    k_rows += nc + nloc;

    /* one softmax per query head over every entry */
    for (int g = 0; g < G; g++) {
        double mx = -HUGE_VAL;
        for (long long e = 0; e < n_ent; e++) mx = elog[e * G + g] > mx ? elog[e * G + g] : mx;
        double den = 0.0;
        for (int i = 0; i < d; i++) out[g * d + i] = 0.0;
        for (long long e = 0; e < n_ent; e++) {
            double w = exp(elog[e * G + g] - mx);
            den += w;
            for (int i = 0; i < d; i++) {
                double v;
                if (ent[e].level >= 1)
                    v = Vnode[ent[e].level][ent[e].id * d + i];
                else if (ent[e].level == 0)
                    v = tok_at(Vtok, tok_dtype, ent[e].id * d + i);
                else
                    v = tok_at(Vloc, tok_dtype, ent[e].id * d + i);
                out[g * d + i] += w * v;
            }
        }
        for (int i = 0; i < d; i++) out[g * d + i] /= den;
    }
    if (rows) {
        rows[0] = k_rows;
        rows[1] = n_ent;
    }
    free(cand); free(next); free(sc); free(lg); free(ent); free(elog); free(qd); free(qr); free(kv); free(kr);
    free(sl);
    return J;
}

/* ----------------------------------------------------------- gradients */

/* Coordinate i of entry (level, id): a node row (level >= 1), a token row
 * (level 0) or a row of the chunk's own tokens (level -1). */
static double entry_at(const double* const* node, const void* tok, const void* loc, int tok_dtype, int level,
                       long long id, int d, int i) {
    if (level > 0) return node[level][id * d + i];
    return tok_at(level == 0 ? tok : loc, tok_dtype, id * d + i);
}

/* Gradient of one query's output (orc_query; a decode query, or a prefill
 * query with its chunk's own causal tokens Kloc, Vloc [nloc][d], whose
 * gradients go to dKloc, dVloc) with the selections held fixed (they are not
 * differentiable): given dout [G][d], returns dq [G][d] (overwritten) and adds
 * into dKtok, dVtok [T][d] and dW [d][d] the gradients with respect to the token keys and
 * values and the pooler, through the direct token entries and through the
 * summaries (a node value is the mean of its subtree's token values, a node
 * key is W times the mean of its children's stored keys; storage rounding is
 * taken as the identity). Written from the definitions, step by step:
 *   logit l_e,g = <rope(q_g, P), rope(k_e, i)> / sqrt(d), p = softmax_e(l),
 *   out_g = sum_e p_e,g v_e;
 *   dv_e = sum_g p_e,g dout_g;  dl_e,g = p_e,g (<dout_g, v_e> - sum_f p_f,g <dout_g, v_f>);
 *   dq_g = sum_e dl_e,g rope(k_e, i - P) / sqrt(d);  dk_e = sum_g dl_e,g rope(q_g, P - i) / sqrt(d);
 * then, level by level from the top, the key gradient g_m of node m (its own
 * entry gradient plus W^T g_parent / children(parent)) adds g_m mean_m^T to
 * dW, and each token gets W^T g_parent / children(parent) for its level-1
 * parent plus, for every ancestor a, dv_a / tokens(a).
 * Returns J, or -1 on bad arguments / allocation failure. */
static int query_grad_impl(int d, int b, int k, int G, double rope_base, long long T, const double* const* Knode,
                           const double* const* Vnode, const void* Ktok, const void* Vtok, int tok_dtype,
                           const void* Kloc, const void* Vloc, long long nloc, const float* W, const float* q,
                           const double* dout, double* dq, double* dKtok, double* dVtok, double* dKloc, double* dVloc,
                           double* dW) {
    if (d <= 0 || d % 2 || b < 2 || k < 1 || G < 1 || T < 0 || nloc < 0 || T + nloc < 1) return -1;
    if (nloc > 0 && (!Kloc || !Vloc || !dKloc || !dVloc)) return -1;
    long long n[ORC_MAXLEV + 1];
    int J = orc_levels(T, b, n);
    int* sel = (int*)malloc(sizeof(int) * (size_t)(J * k + 1));
    double* out = (double*)malloc(sizeof(double) * (size_t)(G * d));
    if (!sel || !out) {
        free(sel);
        free(out);
        return -1;
    }
    /* the forward's selections */
    if (orc_query(d, b, k, G, rope_base, T, Knode, Vnode, Ktok, Vtok, tok_dtype, Kloc, Vloc, nloc, q, out, sel, NULL,
                  NULL) != J) {
        free(sel);
        free(out);
        return -1;
    }
    double scale = 1.0 / sqrt((double)d);
    long long max_cand = (long long)k * b > b ? (long long)k * b : b;
    long long max_ent = (long long)(J + 1) * max_cand + nloc + 1;
    long long* cand = (long long*)malloc(sizeof(long long) * (size_t)max_cand);
    long long* next = (long long*)malloc(sizeof(long long) * (size_t)max_cand);
    int* e_lev = (int*)malloc(sizeof(int) * (size_t)max_ent);
    long long* e_id = (long long*)malloc(sizeof(long long) * (size_t)max_ent);
    long long* e_rank = (long long*)malloc(sizeof(long long) * (size_t)max_ent);
    long long* e_pos = (long long*)malloc(sizeof(long long) * (size_t)max_ent);
    double* lg = (double*)malloc(sizeof(double) * (size_t)(max_ent * G));
    double* kv = (double*)malloc(sizeof(double) * (size_t)d);
    double* vv = (double*)malloc(sizeof(double) * (size_t)d);
    double* qd = (double*)malloc(sizeof(double) * (size_t)d);
    double* r1 = (double*)malloc(sizeof(double) * (size_t)d);
    double* r2 = (double*)malloc(sizeof(double) * (size_t)d);
    /* per-level node gradients (entries) and the top-down sums */
    double** dKn = (double**)calloc((size_t)J + 2, sizeof(double*));
    double** dVn = (double**)calloc((size_t)J + 2, sizeof(double*));
    int ok = cand && next && e_lev && e_id && e_rank && e_pos && lg && kv && vv && qd && r1 && r2 && dKn && dVn;
    for (int j = 1; ok && j <= J; j++) {
        dKn[j] = (double*)calloc((size_t)(n[j] * d), sizeof(double));
        dVn[j] = (double*)calloc((size_t)(n[j] * d), sizeof(double));
        ok = dKn[j] && dVn[j];
    }
    long long n_ent = 0;
    if (ok) {
        /* the entries: unselected candidates of every level, then the tokens
         * under the selected level-1 nodes (as the forward) */
        long long nc = n[J];
        for (long long i = 0; i < nc; i++) cand[i] = i;
        for (int j = J; j >= 1; j--) {
            long long kk = nc < k ? nc : k;
            for (long long i = 0; i < nc; i++) {
                int chosen = 0;
                for (long long r = 0; r < kk; r++) chosen |= (sel[(j - 1) * k + r] == cand[i]);
                if (chosen) continue;
                e_lev[n_ent] = j;
                e_id[n_ent] = cand[i];
                e_rank[n_ent] = i;
                e_pos[n_ent] = nc - 1;
                n_ent++;
            }
            long long nn = 0;
            for (long long r = 0; r < kk; r++) {
                long long m = sel[(j - 1) * k + r];
                long long c_lo = m * b, c_hi = (m + 1) * b < n[j - 1] ? (m + 1) * b : n[j - 1];
                for (long long c = c_lo; c < c_hi; c++) next[nn++] = c;
            }
            memcpy(cand, next, sizeof(long long) * (size_t)nn);
            nc = nn;
        }
        /* level 0: the tokens, then the chunk's own causal tokens (level -1);
         * the query sits at the last index of that list (R6, R9) */
        for (long long i = 0; i < nc; i++) {
            e_lev[n_ent] = 0;
            e_id[n_ent] = cand[i];
            e_rank[n_ent] = i;
            e_pos[n_ent] = nc + nloc - 1;
            n_ent++;
        }
        for (long long i = 0; i < nloc; i++) {
            e_lev[n_ent] = -1;
            e_id[n_ent] = i;
            e_rank[n_ent] = nc + i;
            e_pos[n_ent] = nc + nloc - 1;
            n_ent++;
        }
        /* logits and softmax per head */
        for (long long e = 0; e < n_ent; e++) {
            for (int i = 0; i < d; i++)
                kv[i] = entry_at(Knode, Ktok, Kloc, tok_dtype, e_lev[e], e_id[e], d, i);
            rope(kv, e_rank[e], d, rope_base, r1);
            for (int g = 0; g < G; g++) {
                for (int i = 0; i < d; i++) qd[i] = (double)q[g * d + i];
                rope(qd, e_pos[e], d, rope_base, r2);
                double dot = 0.0;
                for (int i = 0; i < d; i++) dot += r2[i] * r1[i];
                lg[e * G + g] = dot * scale;
            }
        }
        for (int g = 0; g < G; g++) {
            double mx = -HUGE_VAL, den = 0.0, Dg = 0.0;
            for (long long e = 0; e < n_ent; e++) mx = lg[e * G + g] > mx ? lg[e * G + g] : mx;
            for (long long e = 0; e < n_ent; e++) den += exp(lg[e * G + g] - mx);
            /* p_e, <dout, v_e> and their weighted sum D */
            for (long long e = 0; e < n_ent; e++) {
                double p = exp(lg[e * G + g] - mx) / den, a = 0.0;
                for (int i = 0; i < d; i++) {
                    vv[i] = entry_at(Vnode, Vtok, Vloc, tok_dtype, e_lev[e], e_id[e], d, i);
                    a += dout[g * d + i] * vv[i];
                }
                Dg += p * a;
            }
            for (int i = 0; i < d; i++) dq[g * d + i] = 0.0;
            for (long long e = 0; e < n_ent; e++) {
                double p = exp(lg[e * G + g] - mx) / den, a = 0.0;
                for (int i = 0; i < d; i++) {
                    vv[i] = entry_at(Vnode, Vtok, Vloc, tok_dtype, e_lev[e], e_id[e], d, i);
                    a += dout[g * d + i] * vv[i];
                }
                double dl = p * (a - Dg);
                /* dq: the key rotated by i - P; dk: the query rotated by P - i */
                for (int i = 0; i < d; i++)
                    kv[i] = entry_at(Knode, Ktok, Kloc, tok_dtype, e_lev[e], e_id[e], d, i);
                rope(kv, e_rank[e] - e_pos[e], d, rope_base, r1);
                for (int i = 0; i < d; i++) qd[i] = (double)q[g * d + i];
                rope(qd, e_pos[e] - e_rank[e], d, rope_base, r2);
                double* dk = e_lev[e] > 0 ? dKn[e_lev[e]] + e_id[e] * d
                                          : (e_lev[e] == 0 ? dKtok : dKloc) + e_id[e] * d;
                double* dv = e_lev[e] > 0 ? dVn[e_lev[e]] + e_id[e] * d
                                          : (e_lev[e] == 0 ? dVtok : dVloc) + e_id[e] * d;
                for (int i = 0; i < d; i++) {
                    dq[g * d + i] += dl * scale * r1[i];
                    dk[i] += dl * scale * r2[i];
                    dv[i] += p * dout[g * d + i];
                }
            }
        }
        /* top-down through the tree: hk = W^T g / children (to the children's
         * keys), hv = dv / tokens accumulated over the ancestors (to every
         * token of the subtree); dW += g mean^T */
        double* hk_up = NULL;
        double* hv_up = NULL;
        for (int j = J; j >= 1 && ok; j--) {
            double* hk = (double*)calloc((size_t)(n[j] * d), sizeof(double));
            double* hv = (double*)calloc((size_t)(n[j] * d), sizeof(double));
            if (!hk || !hv) {
                free(hk);
                free(hv);
                ok = 0;
                break;
            }
            long long span = ipow_sat(b, j);
            for (long long m = 0; m < n[j]; m++) {
                long long c_lo = m * b, c_hi = (m + 1) * b < n[j - 1] ? (m + 1) * b : n[j - 1];
                long long t_lo = m * span, t_hi = (m + 1) * span < T ? (m + 1) * span : T;
                for (int i = 0; i < d; i++) {
                    qd[i] = dKn[j][m * d + i] + (hk_up ? hk_up[(m / b) * d + i] : 0.0); /* g_m */
                    hv[m * d + i] = dVn[j][m * d + i] / (double)(t_hi - t_lo) + (hv_up ? hv_up[(m / b) * d + i] : 0.0);
                    double s = 0.0;
                    for (long long c = c_lo; c < c_hi; c++)
                        s += (j == 1) ? tok_at(Ktok, tok_dtype, c * d + i) : Knode[j - 1][c * d + i];
                    kv[i] = s / (double)(c_hi - c_lo); /* mean of the children's keys */
                }
                for (int r = 0; r < d; r++)
                    for (int c = 0; c < d; c++) dW[r * d + c] += qd[r] * kv[c];
                for (int c = 0; c < d; c++) {
                    double s = 0.0;
                    for (int r = 0; r < d; r++) s += (double)W[r * d + c] * qd[r];
                    hk[m * d + c] = s / (double)(c_hi - c_lo);
                }
            }
            free(hk_up);
            free(hv_up);
            hk_up = hk;
            hv_up = hv;
        }
        if (ok && hk_up)
            for (long long t = 0; t < T; t++)
                for (int i = 0; i < d; i++) {
                    dKtok[t * d + i] += hk_up[(t / b) * d + i];
                    dVtok[t * d + i] += hv_up[(t / b) * d + i];
                }
        free(hk_up);
        free(hv_up);
    }
    for (int j = 1; j <= J; j++) {
        if (dKn) free(dKn[j]);
        if (dVn) free(dVn[j]);
    }
    free(dKn); free(dVn); free(sel); free(out); free(cand); free(next); free(e_lev); free(e_id); free(e_rank);
    free(e_pos); free(lg); free(kv); free(vv); free(qd); free(r1); free(r2);
    return ok ? J : -1;
}

int orc_query_grad(int d, int b, int k, int G, double rope_base, long long T, const double* const* Knode,
                   const double* const* Vnode, const void* Ktok, const void* Vtok, int tok_dtype, const float* W,
                   const float* q, const double* dout, double* dq, double* dKtok, double* dVtok, double* dW) {
    if (T < 1) return -1;
    return query_grad_impl(d, b, k, G, rope_base, T, Knode, Vnode, Ktok, Vtok, tok_dtype, NULL, NULL, 0, W, q, dout,
                           dq, dKtok, dVtok, NULL, NULL, dW);
}

int orc_query_grad_local(int d, int b, int k, int G, double rope_base, long long T, const double* const* Knode,
                         const double* const* Vnode, const void* Ktok, const void* Vtok, int tok_dtype,
                         const void* Kloc, const void* Vloc, long long nloc, const float* W, const float* q,
                         const double* dout, double* dq, double* dKtok, double* dVtok, double* dKloc, double* dVloc,
                         double* dW) {
    return query_grad_impl(d, b, k, G, rope_base, T, Knode, Vnode, Ktok, Vtok, tok_dtype, Kloc, Vloc, nloc, W, q,
                           dout, dq, dKtok, dVtok, dKloc, dVloc, dW);
}

/* ---------------------------------------------- clustered order (R20) */

typedef struct {
    double z;
    long long id;
} latent;

static int by_latent(const void* a, const void* b) {
    const latent* x = (const latent*)a;
    const latent* y = (const latent*)b;
    if (x->z < y->z) return -1;
    if (x->z > y->z) return 1;
    return (x->id > y->id) - (x->id < y->id);
}

int orc_cluster_order(const void* Ktok, int tok_dtype, long long T, int d, int b, const float* Z, int* perm) {
    if (T < 1 || d < 1 || b < 2 || !Ktok || !Z || !perm) return -1;
    long long n[ORC_MAXLEV + 1];
    const int J = orc_levels(T, b, n);
    long long* ord = (long long*)malloc(sizeof(long long) * (size_t)T);
    latent* seg = (latent*)malloc(sizeof(latent) * (size_t)T);
    if (!ord || !seg) {
        free(ord);
        free(seg);
        return -1;
    }
    for (long long p = 0; p < T; p++) ord[p] = p;
    for (int j = J; j >= 1; j--) {
        const long long S = ipow_sat(b, j + 1); /* the parent blocks (one block at the top) */
        const float* Zj = Z + (size_t)(j - 1) * d;
        for (long long s0 = 0; s0 < T; s0 += S) {
            const long long s1 = s0 + S < T ? s0 + S : T;
            for (long long p = s0; p < s1; p++) {
                const long long t = ord[p];
                double z = 0.0;
                for (int e = 0; e < d; e++) z = z + (double)Zj[e] * tok_at(Ktok, tok_dtype, t * d + e);
                seg[p - s0].z = z + 0.0; /* -0 and +0 are one value */
                seg[p - s0].id = t;
            }
            qsort(seg, (size_t)(s1 - s0), sizeof(latent), by_latent);
            for (long long p = s0; p < s1; p++) ord[p] = seg[p - s0].id;
        }
    }
    for (long long p = 0; p < T; p++) perm[p] = (int)ord[p];
    free(ord);
    free(seg);
    return J;
}
