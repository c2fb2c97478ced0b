// Prefill, chunk-local part: causal RoPE attention among the chunk's own
// tokens, on tensor cores.
//
// In a prefill chunk [s, s+C) the query of token t sees, after the tree's
// entries, the chunk's tokens s..t exactly; those follow the level-0
// candidates in the RoPE index order (kongchang.com article, "Position
// Encoding": positions are ranks within a level's candidate list). Only index
// differences enter a logit, so this part is ordinary causal attention with
// the query at t - s and the keys at u - s, whatever the tree selected; its
// softmax state (running max, sum, unnormalised output) is merged with the
// tree part's state afterwards.
//
// Layout: one CTA per (64-query tile, query head), 4 warps of 16 query rows
// (flash-attention-2 order). Q and K are rotated in fp32 (host fp64 table),
// rounded to bf16 into shared memory; S = Q K^T and O += P V run on
// mma.sync m16n8k16 (bf16 in, fp32 accumulate); V fragments come from
// ldmatrix.trans. Rows are padded by 8 elements so the fragment loads hit
// distinct banks.
#include "common.cuh"

namespace recsa {

constexpr int PL_TILE = 64;          // queries per CTA and keys per tile
constexpr int PL_THREADS = 128;      // 4 warps x 16 query rows

struct PrefillLocalArgs {
    const __nv_bfloat16* q;  // [B][C][Hq][D]
    const __nv_bfloat16* k;  // [B][C][H][D]
    const __nv_bfloat16* v;  // [B][C][H][D]
    float* state;            // [B][C][Hq][D + 2]: unnormalised acc, max, sum
    int C, Hq, H, G;
    float scale;
};

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void mma_bf16_16816(float* c, const uint32_t* a, const uint32_t* b) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t* r, const void* smem_row) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_addr(smem_row)));
}

// Rows [row0, row0 + PL_TILE) of x ([C][heads][D], head `hd`), rotated by
// their offset in the chunk and rounded to bf16, into dst [PL_TILE][D + 8].
// Rows past C are zero.
template <int D>
__device__ __forceinline__ void load_rotated_tile(const TreeParams& p, const __nv_bfloat16* x, int heads, int hd,
                                                  int row0, int C, __nv_bfloat16* dst) {
    constexpr int HD = D / 2, LD = D + 8;
    for (int idx = threadIdx.x; idx < PL_TILE * HD / 2; idx += PL_THREADS) {
        const int r = idx / (HD / 2), i = (idx % (HD / 2)) * 2;  // pairs (i, i+HD) and (i+1, i+1+HD)
        const int t = row0 + r;
        float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
        if (t < C) {
            const __nv_bfloat16* src = x + ((size_t)t * heads + hd) * D;
            const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(src + i);
            const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(src + HD + i);
            const float* row = p.rope + (size_t)t * 3 * HD;
            const float c0 = row[i], c1 = row[i + 1], s0 = row[HD + i], s1 = row[HD + i + 1];
            const float xa0 = __low2float(lo), xa1 = __high2float(lo), xb0 = __low2float(hi), xb1 = __high2float(hi);
            a0 = xa0 * c0 - xb0 * s0;
            a1 = xa1 * c1 - xb1 * s1;
            b0 = xb0 * c0 + xa0 * s0;
            b1 = xb1 * c1 + xa1 * s1;
        }
        *reinterpret_cast<uint32_t*>(dst + r * LD + i) = pack_bf16(a0, a1);
        *reinterpret_cast<uint32_t*>(dst + r * LD + HD + i) = pack_bf16(b0, b1);
    }
}

template <int D>
__global__ void __launch_bounds__(PL_THREADS) prefill_local_kernel(TreeParams p, PrefillLocalArgs a) {
    constexpr int LD = D + 8;   // padded row (elements)
    constexpr int KS = D / 16;  // k-steps over d in Q K^T
    constexpr int NT = D / 8;   // n-tiles over d in P V
    extern __shared__ __align__(16) unsigned char smem_pl[];
    __nv_bfloat16* Qs = reinterpret_cast<__nv_bfloat16*>(smem_pl);
    __nv_bfloat16* Ks = Qs + PL_TILE * LD;
    __nv_bfloat16* Vs = Ks + PL_TILE * LD;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, tig = lane & 3;
    const int qt = blockIdx.x, hq = blockIdx.y % a.Hq, bseq = blockIdx.y / a.Hq, h = hq / a.G;
    const __nv_bfloat16* qb = a.q + (size_t)bseq * a.C * a.Hq * D;
    const __nv_bfloat16* kb = a.k + (size_t)bseq * a.C * a.H * D;
    const __nv_bfloat16* vb = a.v + (size_t)bseq * a.C * a.H * D;

    load_rotated_tile<D>(p, qb, a.Hq, hq, qt * PL_TILE, a.C, Qs);
    __syncthreads();
    const int r0 = warp * 16;
    uint32_t qa[KS][4];
#pragma unroll
    for (int ks = 0; ks < KS; ks++) {
        qa[ks][0] = *reinterpret_cast<const uint32_t*>(Qs + (r0 + g) * LD + ks * 16 + 2 * tig);
        qa[ks][1] = *reinterpret_cast<const uint32_t*>(Qs + (r0 + g + 8) * LD + ks * 16 + 2 * tig);
        qa[ks][2] = *reinterpret_cast<const uint32_t*>(Qs + (r0 + g) * LD + ks * 16 + 8 + 2 * tig);
        qa[ks][3] = *reinterpret_cast<const uint32_t*>(Qs + (r0 + g + 8) * LD + ks * 16 + 8 + 2 * tig);
    }
    const int row_a = qt * PL_TILE + r0 + g, row_b = row_a + 8;  // query rows (in-chunk index)
    float o[NT][4];
#pragma unroll
    for (int n = 0; n < NT; n++) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;

    for (int kt = 0; kt <= qt; kt++) {
        __syncthreads();  // previous tiles consumed
        load_rotated_tile<D>(p, kb, a.H, h, kt * PL_TILE, a.C, Ks);
        for (int idx = tid; idx < PL_TILE * D / 8; idx += PL_THREADS) {
            const int r = idx / (D / 8), c = (idx % (D / 8)) * 8, t = kt * PL_TILE + r;
            uint4 val = make_uint4(0, 0, 0, 0);
            if (t < a.C) val = *reinterpret_cast<const uint4*>(vb + ((size_t)t * a.H + h) * D + c);
            *reinterpret_cast<uint4*>(Vs + r * LD + c) = val;
        }
        __syncthreads();
        float s[8][4];
#pragma unroll
        for (int n = 0; n < 8; n++) {
            s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
            for (int ks = 0; ks < KS; ks++) {
                uint32_t bf[2];
                bf[0] = *reinterpret_cast<const uint32_t*>(Ks + (n * 8 + g) * LD + ks * 16 + 2 * tig);
                bf[1] = *reinterpret_cast<const uint32_t*>(Ks + (n * 8 + g) * LD + ks * 16 + 8 + 2 * tig);
                mma_bf16_16816(s[n], qa[ks], bf);
            }
        }
        // scale, causal mask, online softmax (rows row_a / row_b; a quad shares a row)
        float mx_a = -INFINITY, mx_b = -INFINITY;
#pragma unroll
        for (int n = 0; n < 8; n++)
#pragma unroll
            for (int c = 0; c < 4; c++) {
                const int key = kt * PL_TILE + n * 8 + 2 * tig + (c & 1);
                const int row = c < 2 ? row_a : row_b;
                float x = s[n][c] * a.scale;
                if (key > row || key >= a.C) x = -INFINITY;
                s[n][c] = x;
                if (c < 2) mx_a = fmaxf(mx_a, x); else mx_b = fmaxf(mx_b, x);
            }
#pragma unroll
        for (int off = 1; off <= 2; off <<= 1) {
            mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, off));
            mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, off));
        }
        const float mn_a = fmaxf(m_a, mx_a), mn_b = fmaxf(m_b, mx_b);
        const float al_a = (mn_a == -INFINITY) ? 1.f : (m_a == -INFINITY ? 0.f : expf(m_a - mn_a));
        const float al_b = (mn_b == -INFINITY) ? 1.f : (m_b == -INFINITY ? 0.f : expf(m_b - mn_b));
        m_a = mn_a;
        m_b = mn_b;
        float sum_a = 0.f, sum_b = 0.f;
#pragma unroll
        for (int n = 0; n < 8; n++)
#pragma unroll
            for (int c = 0; c < 4; c++) {
                const float mref = c < 2 ? mn_a : mn_b;
                const float e = (s[n][c] == -INFINITY) ? 0.f : expf(s[n][c] - mref);
                s[n][c] = e;
                if (c < 2) sum_a += e; else sum_b += e;
            }
        l_a = l_a * al_a + sum_a;
        l_b = l_b * al_b + sum_b;
#pragma unroll
        for (int n = 0; n < NT; n++) {
            o[n][0] *= al_a; o[n][1] *= al_a;
            o[n][2] *= al_b; o[n][3] *= al_b;
        }
        // O += P V, 16 keys per k-step
#pragma unroll
        for (int kk = 0; kk < 4; kk++) {
            uint32_t pa[4];
            pa[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
            pa[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
            pa[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
            pa[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
            for (int np = 0; np < NT / 2; np++) {
                uint32_t bv[4];
                ldmatrix_x4_trans(bv, Vs + (kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8) * LD + np * 16 +
                                          ((lane >> 4) & 1) * 8);
                mma_bf16_16816(o[2 * np], pa, bv);
                mma_bf16_16816(o[2 * np + 1], pa, bv + 2);
            }
        }
    }
    // per-row sums over the quad, then the row's state
#pragma unroll
    for (int off = 1; off <= 2; off <<= 1) {
        l_a += __shfl_xor_sync(0xffffffffu, l_a, off);
        l_b += __shfl_xor_sync(0xffffffffu, l_b, off);
    }
    const size_t SW = D + 2;
    if (row_a < a.C) {
        float* st = a.state + (((size_t)bseq * a.C + row_a) * a.Hq + hq) * SW;
#pragma unroll
        for (int n = 0; n < NT; n++) *reinterpret_cast<float2*>(st + n * 8 + 2 * tig) = make_float2(o[n][0], o[n][1]);
        if (tig == 0) { st[D] = m_a; st[D + 1] = l_a; }
    }
    if (row_b < a.C) {
        float* st = a.state + (((size_t)bseq * a.C + row_b) * a.Hq + hq) * SW;
#pragma unroll
        for (int n = 0; n < NT; n++) *reinterpret_cast<float2*>(st + n * 8 + 2 * tig) = make_float2(o[n][2], o[n][3]);
        if (tig == 0) { st[D] = m_b; st[D + 1] = l_b; }
    }
}

template <int D>
cudaError_t launch_prefill_local(const TreeParams& p, const void* q, const void* k, const void* v, float* state,
                                 int B, int C, int Hq, int H, cudaStream_t s) {
    PrefillLocalArgs a{reinterpret_cast<const __nv_bfloat16*>(q), reinterpret_cast<const __nv_bfloat16*>(k),
                       reinterpret_cast<const __nv_bfloat16*>(v), state, C, Hq, H, Hq / H,
                       (float)(1.0 / sqrt((double)D))};
    const size_t smem = (size_t)3 * PL_TILE * (D + 8) * sizeof(__nv_bfloat16);
    auto kern = prefill_local_kernel<D>;
    static std::atomic<unsigned long long> attr_done{0};
    cudaError_t e = set_smem_limit(kern, (int)smem, attr_done);
    if (e != cudaSuccess) return e;
    dim3 grid((C + PL_TILE - 1) / PL_TILE, B * Hq);
    kern<<<grid, PL_THREADS, smem, s>>>(p, a);
    return cudaGetLastError();
}

template cudaError_t launch_prefill_local<64>(const TreeParams&, const void*, const void*, const void*, float*, int,
                                              int, int, int, cudaStream_t);
template cudaError_t launch_prefill_local<128>(const TreeParams&, const void*, const void*, const void*, float*, int,
                                               int, int, int, cudaStream_t);

}  // namespace recsa
