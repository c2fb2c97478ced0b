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
// Work split. The CS CTAs of a cluster divide each level's candidate list
// (ascending node order) into contiguous rank ranges. Each CTA scores its
// range, keeps its local top-k, and the CTAs merge their local lists through
// distributed shared memory; every CTA then derives the same global top-k,
// so no CTA waits for another's decision. The softmax runs online per warp;
// warps merge per CTA, CTAs merge through DSMEM at the end.
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
};

// A lane owns PPL = D/64 rotation pairs (x_i, x_{i+D/2}), i = lane*PPL + e.
template <typename T, int PPL>
__device__ __forceinline__ void load_pairs(const T* row, int lane, float* a, float* b) {
    constexpr int H = PPL * 32;  // D / 2
#pragma unroll
    for (int e = 0; e < PPL; e++) {
        a[e] = to_f(row[lane * PPL + e]);
        b[e] = to_f(row[H + lane * PPL + e]);
    }
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(DEC_THREADS) decode_kernel(TreeParams p, DecodeArgs a) {
    constexpr int PPL = D / 64;
    constexpr int HD = D / 2;
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int CS = (int)cluster.num_blocks();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long long u = blockIdx.y;

    extern __shared__ __align__(16) unsigned char smem_raw[];
    unsigned long long* topbuf = reinterpret_cast<unsigned long long*>(smem_raw);  // [2][KMAX]
    unsigned long long* skey = topbuf + 2 * KMAX;                                  // [my_max]
    long long* par = reinterpret_cast<long long*>(skey + a.my_max);                // [KMAX]
    long long* chosen = par + KMAX;                                                // [KMAX]
    long long* picked = chosen + KMAX;                                             // [KMAX]
    float* cm = reinterpret_cast<float*>(picked + KMAX);                           // [G]
    float* cl = cm + G;                                                            // [G]
    float* cacc = cl + G;                                                          // [G][D]
    float* wm = cacc + G * D;                                                      // [W][G]
    float* wl = wm + DEC_WARPS * G;                                                // [W][G]
    float* wacc = wl + DEC_WARPS * G;                                              // [W][G][D]
    float* slg = wacc + DEC_WARPS * G * D;                                         // [G][my_max]

    const long long L = p.len[u];
    const bool bad = (L <= 0 || L > p.cap);
    if (bad) {
        if (tid == 0 && rank == 0) flag_error(p.err, ERR_LENGTH);
    }

    // raw query, this lane's pairs
    const T* qg = reinterpret_cast<const T*>(a.q) + (u * G) * D;
    float qa[G][PPL], qb[G][PPL];
#pragma unroll
    for (int g = 0; g < G; g++) load_pairs<T, PPL>(qg + g * D, lane, qa[g], qb[g]);

    // online-softmax state of this warp
    float m_[G], l_[G], acc_a[G][PPL], acc_b[G][PPL];
#pragma unroll
    for (int g = 0; g < G; g++) {
        m_[g] = -INFINITY; l_[g] = 0.f;
#pragma unroll
        for (int e = 0; e < PPL; e++) { acc_a[g][e] = 0.f; acc_b[g][e] = 0.f; }
    }

    auto accumulate = [&](const float* lg, const float* va, const float* vb) {
#pragma unroll
        for (int g = 0; g < G; g++) {
            const float mn = fmaxf(m_[g], lg[g]);
            const float sa = expf(m_[g] - mn);
            const float w = expf(lg[g] - mn);
            l_[g] = l_[g] * sa + w;
#pragma unroll
            for (int e = 0; e < PPL; e++) {
                acc_a[g][e] = acc_a[g][e] * sa + w * va[e];
                acc_b[g][e] = acc_b[g][e] * sa + w * vb[e];
            }
            m_[g] = mn;
        }
    };

    // scores of one key row at candidate index `idx` against the query
    // rotated at P (qra/qrb); returns the G logits in lg (all lanes)
    auto score = [&](const T* krow, int idx, const float (*qra)[PPL], const float (*qrb)[PPL], float* lg) {
        float ka[PPL], kb[PPL];
        load_pairs<T, PPL>(krow, lane, ka, kb);
        const float2* cs = p.rope + (long long)idx * HD + lane * PPL;
        float ra[PPL], rb[PPL];
#pragma unroll
        for (int e = 0; e < PPL; e++) {
            const float2 c = cs[e];
            ra[e] = ka[e] * c.x - kb[e] * c.y;
            rb[e] = kb[e] * c.x + ka[e] * c.y;
        }
#pragma unroll
        for (int g = 0; g < G; g++) {
            float s = 0.f;
#pragma unroll
            for (int e = 0; e < PPL; e++) s = fmaf(qra[g][e], ra[e], fmaf(qrb[g][e], rb[e], s));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
            lg[g] = s * p.scale;
        }
    };

    long long krows = 0, vrows = 0;
    if (!bad) {
        const int J = top_level(p, L);
        if (tid == 0) par[0] = 0;  // the top level = children of one virtual root
        int npar = 1;
        __syncthreads();

        for (int j = J; j >= 0; j--) {
            const long long n_j = level_rows(p, j, L);
            const long long last = par[npar - 1];
            const long long ncand = (long long)(npar - 1) * p.b + min((long long)p.b, n_j - last * p.b);
            const long long P = ncand - 1;
            const long long per = (ncand + CS - 1) / CS;
            const long long r0 = min(ncand, rank * per), r1 = min(ncand, r0 + per);

            // query rotated at this level's position P
            float qra[G][PPL], qrb[G][PPL];
            {
                const float2* cs = p.rope + P * HD + lane * PPL;
#pragma unroll
                for (int e = 0; e < PPL; e++) {
                    const float2 c = cs[e];
#pragma unroll
                    for (int g = 0; g < G; g++) {
                        qra[g][e] = qa[g][e] * c.x - qb[g][e] * c.y;
                        qrb[g][e] = qb[g][e] * c.x + qa[g][e] * c.y;
                    }
                }
            }
            const T* Kj = reinterpret_cast<const T*>(p.K[j]) + (u * p.rows[j]) * D;
            const T* Vj = reinterpret_cast<const T*>(p.V[j]) + (u * p.rows[j]) * D;
            krows += ncand;

            if (j == 0) {
                // exact tokens under the kept level-1 nodes
                for (long long i = r0 + warp; i < r1; i += DEC_WARPS) {
                    const long long id = par[i / p.b] * p.b + i % p.b;
                    if (id < 0 || id >= n_j) {
                        if (lane == 0) flag_error(p.err, ERR_SHAPE);
                        continue;
                    }
                    float lg[G], va[PPL], vb[PPL];
                    score(Kj + id * D, (int)i, qra, qrb, lg);
                    load_pairs<T, PPL>(Vj + id * D, lane, va, vb);
                    accumulate(lg, va, vb);
                }
                vrows += ncand;
                break;
            }

            // score this CTA's candidates
            for (long long i = r0 + warp; i < r1; i += DEC_WARPS) {
                const long long id = par[i / p.b] * p.b + i % p.b;
                if (id < 0 || id >= n_j) {
                    if (lane == 0) {
                        flag_error(p.err, ERR_SHAPE);
                        skey[i - r0] = 0;
                    }
                    continue;
                }
                float lg[G];
                score(Kj + id * D, (int)i, qra, qrb, lg);
                if (lane == 0) {
                    float S = 0.f;
#pragma unroll
                    for (int g = 0; g < G; g++) {
                        slg[g * a.my_max + (i - r0)] = lg[g];
                        S += lg[g];
                    }
                    skey[i - r0] = sel_key(S, id);
                }
            }
            __syncthreads();

            const int kk = (int)min((long long)p.k, ncand);
            unsigned long long* mybuf = topbuf + (j & 1) * KMAX;
            if (warp == 0) {
                // local top-kk by repeated warp arg-max (keys are unique, 0 = empty)
                const int nmy = (int)(r1 - r0);
                for (int r = 0; r < kk; r++) {
                    unsigned long long best = 0;
                    for (int i = lane; i < nmy; i += 32) best = skey[i] > best ? skey[i] : best;
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) {
                        unsigned long long other = shfl_xor_u64(best, o);
                        best = other > best ? other : best;
                    }
                    if (best != 0) {
                        for (int i = lane; i < nmy; i += 32)
                            if (skey[i] == best) skey[i] = 0;
                    }
                    if (lane == 0) mybuf[r] = best;
                    __syncwarp();
                }
            }
            cluster.sync();
            if (warp == 0) {
                // global top-kk over every CTA's local list; identical in every CTA
                const int total = CS * kk;
                unsigned long long mine[(DEC_CLUSTER * KMAX + 31) / 32];
                int nm = 0;
                for (int i = lane; i < total; i += 32) {
                    const unsigned long long* rb = cluster.map_shared_rank(mybuf, i / kk);
                    mine[nm++] = rb[i % kk];
                }
                for (int r = 0; r < kk; r++) {
                    unsigned long long best = 0;
                    for (int x = 0; x < nm; x++) best = mine[x] > best ? mine[x] : best;
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) {
                        unsigned long long other = shfl_xor_u64(best, o);
                        best = other > best ? other : best;
                    }
                    for (int x = 0; x < nm; x++)
                        if (mine[x] == best) mine[x] = 0;
                    if (lane == 0) picked[r] = key_id(best);
                    __syncwarp();
                }
                // ascending node order (ids are distinct: rank = number of smaller ids)
                for (int x = lane; x < kk; x += 32) {
                    const long long id = picked[x];
                    int pos = 0;
                    for (int r = 0; r < kk; r++) pos += (picked[r] < id);
                    chosen[pos] = id;
                }
                __syncwarp();
                if (rank == 0 && a.sel_out) {
                    for (int x = lane; x < p.k; x += 32)
                        a.sel_out[(u * p.J_cap + (j - 1)) * p.k + x] = x < kk ? (int)chosen[x] : -1;
                }
            }
            __syncthreads();

            // candidates that were not kept enter the softmax as summaries
            for (long long i = r0 + warp; i < r1; i += DEC_WARPS) {
                const long long id = par[i / p.b] * p.b + i % p.b;
                if (id < 0 || id >= n_j) continue;
                bool kept = false;
                for (int r = 0; r < kk; r++) kept |= (chosen[r] == id);
                if (kept) continue;
                float lg[G], va[PPL], vb[PPL];
#pragma unroll
                for (int g = 0; g < G; g++) lg[g] = slg[g * a.my_max + (i - r0)];
                load_pairs<T, PPL>(Vj + id * D, lane, va, vb);
                accumulate(lg, va, vb);
            }
            vrows += ncand - kk;
            __syncthreads();
            if (tid < kk) par[tid] = chosen[tid];
            npar = kk;
            __syncthreads();
        }
    }

    // merge warp states -> CTA state
    if (lane == 0) {
#pragma unroll
        for (int g = 0; g < G; g++) { wm[warp * G + g] = m_[g]; wl[warp * G + g] = l_[g]; }
    }
#pragma unroll
    for (int g = 0; g < G; g++)
#pragma unroll
        for (int e = 0; e < PPL; e++) {
            wacc[(warp * G + g) * D + lane * PPL + e] = acc_a[g][e];
            wacc[(warp * G + g) * D + HD + lane * PPL + e] = acc_b[g][e];
        }
    __syncthreads();
    for (int idx = tid; idx < G * D; idx += DEC_THREADS) {
        const int g = idx / D, e = idx % D;
        float M = -INFINITY;
        for (int w = 0; w < DEC_WARPS; w++) M = fmaxf(M, wm[w * G + g]);
        float s = 0.f, lsum = 0.f;
        for (int w = 0; w < DEC_WARPS; w++) {
            const float f = (wm[w * G + g] == -INFINITY) ? 0.f : expf(wm[w * G + g] - M);
            s += wacc[(w * G + g) * D + e] * f;
            lsum += wl[w * G + g] * f;
        }
        cacc[g * D + e] = s;
        if (e == 0) { cm[g] = M; cl[g] = lsum; }
    }
    cluster.sync();

    // merge CTA states across the cluster and write the output
    T* outp = reinterpret_cast<T*>(a.out) + (u * G) * D;
    for (int idx = rank * DEC_THREADS + tid; idx < G * D; idx += CS * DEC_THREADS) {
        const int g = idx / D, e = idx % D;
        float M = -INFINITY;
        for (int r = 0; r < CS; r++) M = fmaxf(M, cluster.map_shared_rank(cm, r)[g]);
        float s = 0.f, lsum = 0.f;
        for (int r = 0; r < CS; r++) {
            const float mr = cluster.map_shared_rank(cm, r)[g];
            const float f = (mr == -INFINITY) ? 0.f : expf(mr - M);
            s += cluster.map_shared_rank(cacc, r)[g * D + e] * f;
            lsum += cluster.map_shared_rank(cl, r)[g] * f;
        }
        outp[g * D + e] = from_f<T>(bad ? 0.f : s / lsum);
    }
    if (rank == 0 && tid == 0 && a.rows_out) {
        a.rows_out[u * 2] = krows;
        a.rows_out[u * 2 + 1] = vrows;
    }
    if (rank == 0 && a.sel_out) {
        // levels above the current top level, or everything for a bad unit
        const int J = bad ? 0 : top_level(p, L);
        for (int i = tid; i < (p.J_cap - J) * p.k; i += DEC_THREADS)
            a.sel_out[(u * p.J_cap + J) * p.k + i] = -1;
    }
    cluster.sync();  // keep this CTA's shared memory alive for remote readers
}

size_t decode_smem_bytes(int D, int G, int my_max) {
    size_t s = 2 * KMAX * 8 + (size_t)my_max * 8 + 3 * KMAX * 8;
    s += (size_t)(2 * G + G * D + 2 * DEC_WARPS * G + DEC_WARPS * G * D + G * my_max) * 4;
    return s;
}

template <typename T, int D, int G>
cudaError_t launch_decode(const TreeParams& p, const void* q, void* out, int* sel_out, long long* rows_out,
                          cudaStream_t s) {
    const int CS = DEC_CLUSTER;
    long long maxc = (long long)p.k * p.b > p.b ? (long long)p.k * p.b : p.b;
    DecodeArgs a{q, out, sel_out, rows_out, (int)((maxc + CS - 1) / CS)};
    size_t smem = decode_smem_bytes(D, G, a.my_max);
    auto kern = decode_kernel<T, D, G>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(CS, p.B * p.H, 1);
    cfg.blockDim = dim3(DEC_THREADS, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
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
