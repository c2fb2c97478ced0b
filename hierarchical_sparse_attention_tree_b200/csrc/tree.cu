// Tree build and append kernels.
//
// The tree over the KV cache (RecSA abstract): every node stands for its
// subtree through a single key and a single value; the value is the average
// of the subtree's token values (kongchang.com article, "Core Idea"), the key
// comes from the layer's one pooler, which every level uses (abstract).
//
// Arithmetic contract, shared by every path that writes a node so that a tree
// grown token by token is bit-identical to one built at once:
//   value sum  VS_j[m] = (((0 + s_0) + s_1) + ...) over the children in order,
//              s_c = token value (j = 1) or VS_{j-1}[c] (j >= 2), fp32;
//   value      V_j[m]  = round(VS_j[m] / tokens(m));
//   key        K_j[m]  = round(W * (((0 + k_0) + k_1) + ... ) / children(m)),
//              k_c = stored child key; the product is an fmaf chain over the
//              input coordinate c = 0..d-1 starting from 0;
//   right edge PK_j, PV_j = the same running sums over every child of the
//              last node but its last child, so an append only adds the
//              completed child and the new last child.
#include "common.cuh"
#include "append.cuh"

namespace recsa {

// ------------------------------------------------------------- lengths

__global__ void set_lengths_kernel(long long* len, const long long* src, int B, int H) {
    int u = blockIdx.x * blockDim.x + threadIdx.x;
    if (u < B * H) len[u] = src[u / H];
}

__global__ void bump_lengths_kernel(long long* len, int n_units, long long n) {
    int u = blockIdx.x * blockDim.x + threadIdx.x;
    if (u < n_units) len[u] += n;
}

// ------------------------------------------------------------ copy rows

// Copies n new tokens [B][n][H][D] into the cache after each unit's tokens.
template <typename T, int D>
__global__ void copy_tokens_kernel(TreeParams p, const T* __restrict__ k_new, const T* __restrict__ v_new, int n) {
    constexpr int VEC = 16 / sizeof(T);
    constexpr int PER_ROW = D / VEC;
    long long units = (long long)p.B * p.H;
    long long total = units * n * PER_ROW;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        int piece = (int)(i % PER_ROW);
        long long r = i / PER_ROW;      // (b, t, h)
        int h = (int)(r % p.H);
        long long t = (r / p.H) % n;
        int b = (int)(r / ((long long)p.H * n));
        long long u = (long long)b * p.H + h;
        long long L = p.len[u];
        if (L + t >= p.cap) { flag_error(p.err, ERR_LENGTH); continue; }
        const uint4* ks = reinterpret_cast<const uint4*>(k_new + (r * D)) + piece;
        const uint4* vs = reinterpret_cast<const uint4*>(v_new + (r * D)) + piece;
        const long long row = token_row(token_map(p), u, L + t);
        T* kd = reinterpret_cast<T*>(p.K[0]) + row * D;
        T* vd = reinterpret_cast<T*>(p.V[0]) + row * D;
        reinterpret_cast<uint4*>(kd)[piece] = *ks;
        reinterpret_cast<uint4*>(vd)[piece] = *vs;
    }
}

// ---------------------------------------------------------- build level

// One node m of level j of unit u (one warp; kmw: the warp's row of shared
// memory for the key mean).
template <typename T, int D>
__device__ __forceinline__ void build_node(const TreeParams& p, int j, long long u, long long m, long long L,
                                           long long n_j, long long n_prev, const T* Wt, float* kmw, int lane) {
    constexpr int DPL = D / 32;  // columns per lane, contiguous
    const bool right_edge = (m == n_j - 1);
    const long long c_lo = m * p.b;
    const long long c_hi = min(c_lo + (long long)p.b, n_prev);
    // child rows c_lo .. c_hi - 1, indexed from c_lo (one page of tokens at j = 1)
    const long long crow = j == 1 ? token_row(token_map(p), u, c_lo) : u * p.rows[j - 1] + c_lo;
    const T* Kc = reinterpret_cast<const T*>(p.K[j - 1]) + (crow - c_lo) * D + lane * DPL;
    const T* Vc = reinterpret_cast<const T*>(p.V[0]) + (crow - c_lo) * D + lane * DPL;  // j == 1
    const float* Sc = (j >= 2) ? p.VS[j - 1] + (crow - c_lo) * D + lane * DPL : nullptr;

    float ks[DPL], vs[DPL];
#pragma unroll
    for (int e = 0; e < DPL; e++) { ks[e] = 0.f; vs[e] = 0.f; }

    // Right-edge prefix sums: the running sums before the last child.
    auto keep_edge = [&](long long c) {
        if (right_edge && c == c_hi - 1) {
            float* pk = p.PK[j] + u * D + lane * DPL;
            float* pv = p.PV[j] + u * D + lane * DPL;
#pragma unroll
            for (int e = 0; e < DPL; e++) { pk[e] = ks[e]; pv[e] = vs[e]; }
        }
    };
    if constexpr (sizeof(T) == 2 && DPL == 4) {
        if (j == 1) {
            // tokens (bf16): the rows stay packed (8 bytes a lane, no
            // conversion registers) until they are added
            constexpr int UB = 8;
            auto add_row = [&](uint2 kr, uint2 vr) {
                const __nv_bfloat162 k01 = *reinterpret_cast<const __nv_bfloat162*>(&kr.x);
                const __nv_bfloat162 k23 = *reinterpret_cast<const __nv_bfloat162*>(&kr.y);
                const __nv_bfloat162 v01 = *reinterpret_cast<const __nv_bfloat162*>(&vr.x);
                const __nv_bfloat162 v23 = *reinterpret_cast<const __nv_bfloat162*>(&vr.y);
                ks[0] = ks[0] + __low2float(k01);
                ks[1] = ks[1] + __high2float(k01);
                ks[2] = ks[2] + __low2float(k23);
                ks[3] = ks[3] + __high2float(k23);
                vs[0] = vs[0] + __low2float(v01);
                vs[1] = vs[1] + __high2float(v01);
                vs[2] = vs[2] + __low2float(v23);
                vs[3] = vs[3] + __high2float(v23);
            };
            long long c0 = c_lo;
            for (; c0 + UB <= c_hi; c0 += UB) {
                const T* kb0 = Kc + c0 * D;
                const T* vb0 = Vc + c0 * D;
                uint2 kr[UB], vr[UB];
#pragma unroll
                for (int i = 0; i < UB; i++) {
                    kr[i] = *reinterpret_cast<const uint2*>(kb0 + i * D);
                    vr[i] = *reinterpret_cast<const uint2*>(vb0 + i * D);
                }
#pragma unroll
                for (int i = 0; i < UB; i++) {
                    keep_edge(c0 + i);
                    add_row(kr[i], vr[i]);
                }
            }
            for (; c0 < c_hi; c0++) {
                const uint2 kr = *reinterpret_cast<const uint2*>(Kc + c0 * D);
                const uint2 vr = *reinterpret_cast<const uint2*>(Vc + c0 * D);
                keep_edge(c0);
                add_row(kr, vr);
            }
        }
    }
    constexpr int U = (sizeof(T) == 2 && DPL == 4) ? 4 : 8;  // (bf16, d = 128: only the small levels j >= 2 come here)
    const bool packed = sizeof(T) == 2 && DPL == 4 && j == 1;
    for (long long c0 = c_lo; c0 < c_hi && !packed; c0 += U) {
        float kb[U][DPL], vb[U][DPL];
#pragma unroll
        for (int i = 0; i < U; i++) {
            long long c = c0 + i;
            if (c < c_hi) {
                load_vec<T, DPL>(Kc + c * D, kb[i]);
                if (j == 1)
                    load_vec<T, DPL>(Vc + c * D, vb[i]);
                else
                    load_vec<float, DPL>(Sc + c * D, vb[i]);
            }
        }
#pragma unroll
        for (int i = 0; i < U; i++) {
            long long c = c0 + i;
            if (c < c_hi) {
                keep_edge(c);
#pragma unroll
                for (int e = 0; e < DPL; e++) { ks[e] = ks[e] + kb[i][e]; vs[e] = vs[e] + vb[i][e]; }
            }
        }
    }

    const long long t_lo = m * p.span[j];
    const long long cnt = min(t_lo + p.span[j], L) - t_lo;
    const float fcnt = (float)cnt, fnc = (float)(c_hi - c_lo);
    float* vs_out = p.VS[j] + (u * p.rows[j] + m) * D + lane * DPL;
    T* v_out = reinterpret_cast<T*>(p.V[j]) + (u * p.rows[j] + m) * D + lane * DPL;
    float vm[DPL];
#pragma unroll
    for (int e = 0; e < DPL; e++) { vs_out[e] = vs[e]; vm[e] = __fdiv_rn(vs[e], fcnt); }
    store_vec<T, DPL>(v_out, vm);

#pragma unroll
    for (int e = 0; e < DPL; e++) kmw[lane * DPL + e] = __fdiv_rn(ks[e], fnc);
    __syncwarp();
    // the pooler product as the append computes it: one fmaf chain per
    // quarter of the input coordinate, then (y0 + y1) + (y2 + y3)
    constexpr int Q = D / 4;
    float y4[4][DPL];
#pragma unroll
    for (int q = 0; q < 4; q++)
#pragma unroll
        for (int e = 0; e < DPL; e++) y4[q][e] = 0.f;
#pragma unroll 4
    for (int c = 0; c < Q; c++) {
#pragma unroll
        for (int q = 0; q < 4; q++) {
            const float x = kmw[q * Q + c];
            float w[DPL];
            load_vec<T, DPL>(Wt + (q * Q + c) * D + lane * DPL, w);
#pragma unroll
            for (int e = 0; e < DPL; e++) y4[q][e] = fmaf(w[e], x, y4[q][e]);
        }
    }
    float y[DPL];
#pragma unroll
    for (int e = 0; e < DPL; e++) y[e] = (y4[0][e] + y4[1][e]) + (y4[2][e] + y4[3][e]);
    T* k_out = reinterpret_cast<T*>(p.K[j]) + (u * p.rows[j] + m) * D + lane * DPL;
    store_vec<T, DPL>(k_out, y);
    __syncwarp();  // kmw is read by every lane before the warp's next node writes it
}

// One warp per node of level j; persistent: the grid walks blocks of
// `nwarps` consecutive nodes of one unit with a grid stride, so each CTA
// brings the pooler into shared memory once. Recomputes nodes m >= m0 of
// the tree over L' = len[u] + add tokens, where m0 = 0 for a full build and
// len[u] / b^j when `add` new tokens were just copied in.
template <typename T, int D>
__global__ void __launch_bounds__(256, 2) build_level_kernel(TreeParams p, int j, long long add, int from_len,
                                                          long long blocks_per_unit) {
    extern __shared__ __align__(16) unsigned char smem_b[];
    T* Wt = reinterpret_cast<T*>(smem_b);                          // [D][D], storage type
    float* km = reinterpret_cast<float*>(smem_b + D * D * sizeof(T));  // [warps][D]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    for (int i = threadIdx.x; i < (int)(D * D * sizeof(T) / 16); i += blockDim.x)
        reinterpret_cast<uint4*>(Wt)[i] = reinterpret_cast<const uint4*>(p.Wt)[i];
    __syncthreads();

    const long long total = (long long)p.B * p.H * blocks_per_unit;
    for (long long blk = blockIdx.x; blk < total; blk += gridDim.x) {
        const long long u = blk / blocks_per_unit;
        const long long L = p.len[u] + add;
        const long long n_j = level_rows(p, j, L);
        const long long n_prev = level_rows(p, j - 1, L);
        const long long m0 = from_len ? p.len[u] / p.span[j] : 0;
        const long long m = m0 + (blk % blocks_per_unit) * nwarps + warp;
        if (m >= n_j) continue;
        if (n_j > p.rows[j] || L > p.cap) {
            if (lane == 0) flag_error(p.err, ERR_SHAPE);
            continue;
        }
        build_node<T, D>(p, j, u, m, L, n_j, n_prev, Wt, km + warp * D, lane);
    }
}

// ----------------------------------------------------------- append one

// Appends one token per unit and refreshes the right edge of every level.
// One CTA of D threads per unit; the pooler comes into shared memory by one
// bulk async copy while the per-level loads are in flight.
template <typename T, int D>
__global__ void __launch_bounds__(D) append_one_kernel(TreeParams p, const T* __restrict__ k_new,
                                                       const T* __restrict__ v_new) {
    extern __shared__ __align__(128) unsigned char smem_a[];
    T* Wt = reinterpret_cast<T*>(smem_a);                                   // [D][D]
    float* scratch = reinterpret_cast<float*>(smem_a + D * D * sizeof(T));  // append_scratch_floats
    __shared__ uint64_t wbar;
    __shared__ LevelRef lv[MAXJ + 1];
    __shared__ TokenMap tok;
    const long long u = blockIdx.x;
    // the next kernel on the stream (a decode) may start its own set-up now
    asm volatile("griddepcontrol.launch_dependents;");
    const long long P = p.len[u];  // position of the new token
    if (P >= p.cap) {
        if (threadIdx.x == 0) flag_error(p.err, ERR_LENGTH);
        return;
    }
    if (threadIdx.x == 0) {
        tok = token_map(p);
        mbar_init(&wbar, 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(&wbar, (uint32_t)(D * D * sizeof(T)));
        bulk_g2s(Wt, p.Wt, (uint32_t)(D * D * sizeof(T)), &wbar);
    }
    load_levels(p, lv, threadIdx.x);
    __syncthreads();
    const bool ok = append_token<T, D>(
        AppendDims{p.cap, p.J_cap, p.b, &tok}, lv, u, P, k_new + u * D, v_new + u * D, Wt, scratch,
        [&]() {
            const int timed_out = !mbar_wait(&wbar, 0);
            if (__syncthreads_or(timed_out)) {  // same decision in every thread
                if (threadIdx.x == 0) flag_error(p.err, ERR_TIMEOUT);
                return false;
            }
            return true;
        },
        [](int, T, T) {});
    if (ok && threadIdx.x == 0) p.len[u] = P + 1;
}

// --------------------------------------------------------------- launch

template <typename T, int D>
cudaError_t launch_build_level(const TreeParams& p, int j, long long add, int from_len, long long max_nodes,
                               cudaStream_t s) {
    const int threads = 256, wpb = threads / 32;
    size_t smem = (size_t)D * D * sizeof(T) + (size_t)wpb * D * sizeof(float);
    auto kern = build_level_kernel<T, D>;
    static std::atomic<unsigned long long> attr_done{0};
    cudaError_t e = set_smem_limit(kern, (int)smem, attr_done);
    if (e != cudaSuccess) return e;
    long long per_unit = (max_nodes + wpb - 1) / wpb;
    if (per_unit < 1) per_unit = 1;
    // resident CTAs per SM and SMs, looked up once per device
    static std::atomic<int> cached[64];
    int dev = 0;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int slots = dev < 64 ? cached[dev].load(std::memory_order_relaxed) : 0;
    if (slots <= 0) {
        int sms = 148, per_sm = 1;
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem);
        if (e != cudaSuccess) return e;
        slots = sms * (per_sm < 1 ? 1 : per_sm);
        if (dev < 64) cached[dev].store(slots, std::memory_order_relaxed);
    }
    const long long total = per_unit * p.B * p.H;
    const long long grid = total < slots ? total : slots;
    kern<<<(unsigned)grid, threads, smem, s>>>(p, j, add, from_len, per_unit);
    return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_append_one(const TreeParams& p, const void* k_new, const void* v_new, cudaStream_t s) {
    size_t smem = (size_t)D * D * sizeof(T) + append_scratch_floats(D, p.J_cap) * sizeof(float);
    auto kern = append_one_kernel<T, D>;
    static std::atomic<unsigned long long> attr_done{0};
    cudaError_t e = set_smem_limit(kern, (int)smem, attr_done);
    if (e != cudaSuccess) return e;
    kern<<<p.B * p.H, D, smem, s>>>(p, reinterpret_cast<const T*>(k_new), reinterpret_cast<const T*>(v_new));
    return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_copy_tokens(const TreeParams& p, const void* k_new, const void* v_new, int n, cudaStream_t s) {
    long long total = (long long)p.B * p.H * n * (D * sizeof(T) / 16);
    long long blocks = (total + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (blocks < 1) blocks = 1;
    copy_tokens_kernel<T, D><<<(unsigned)blocks, 256, 0, s>>>(p, reinterpret_cast<const T*>(k_new),
                                                               reinterpret_cast<const T*>(v_new), n);
    return cudaGetLastError();
}

cudaError_t launch_set_lengths(const TreeParams& p, const long long* dev_src, cudaStream_t s) {
    int n = p.B * p.H;
    set_lengths_kernel<<<(n + 255) / 256, 256, 0, s>>>(p.len, dev_src, p.B, p.H);
    return cudaGetLastError();
}

cudaError_t launch_bump_lengths(const TreeParams& p, long long n, cudaStream_t s) {
    int units = p.B * p.H;
    bump_lengths_kernel<<<(units + 255) / 256, 256, 0, s>>>(p.len, units, n);
    return cudaGetLastError();
}

#define RECSA_INST_TREE(T, D)                                                                                   \
    template cudaError_t launch_build_level<T, D>(const TreeParams&, int, long long, int, long long,           \
                                                  cudaStream_t);                                               \
    template cudaError_t launch_append_one<T, D>(const TreeParams&, const void*, const void*, cudaStream_t);   \
    template cudaError_t launch_copy_tokens<T, D>(const TreeParams&, const void*, const void*, int, cudaStream_t);
RECSA_INST_TREE(float, 64)
RECSA_INST_TREE(float, 128)
RECSA_INST_TREE(__nv_bfloat16, 64)
RECSA_INST_TREE(__nv_bfloat16, 128)

}  // namespace recsa
