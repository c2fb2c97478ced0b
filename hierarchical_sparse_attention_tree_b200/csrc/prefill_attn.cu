// Prefill, chunk-local part: causal RoPE attention among the chunk's own
// tokens, on the 5th-generation tensor cores (tcgen05, accumulators in TMEM)
// with tiles brought in by TMA.
//
// In a prefill chunk [s, s+C) the query of token t sees, after the tree's
// entries, the chunk's tokens s..t exactly; those follow the level-0
// candidates in the RoPE index order (kongchang.com article, "Position
// Encoding": positions are ranks within a level's candidate list). Only index
// differences enter a logit, so this part is ordinary causal attention with
// the query at t - s and the keys at u - s, whatever the tree selected; its
// softmax state (reference maximum, sum, unnormalised output) is merged with
// the tree part's state afterwards.
//
// Two launches. (1) rope_chunk_kernel rotates the chunk's queries and keys by
// their offset in the chunk (fp32, the host fp64 table) and rounds them to
// bf16 into scratch. (2) prefill_attn_kernel: one CTA of 256 threads per
// (128-query tile, query head); threads t and t + 128 share query row t, each
// owning half of the key columns of S and half of the output columns. Per
// 128-key tile: one thread issues S = Q K^T (tcgen05.mma kind::f16,
// M = N = 128, fp32 in TMEM columns [0, 128)); every thread reads its half
// row of S from TMEM, scales it (log2 units) and masks it on the diagonal
// tile, the two halves exchange their maxima, and each writes its
// probabilities as bf16 into a 128-byte-swizzled shared tile; then O += P V
// (M = 128, N = d, V read as an MN-major operand) accumulates in TMEM
// columns [128, 128 + d). K and V tiles are double-buffered; each tile's key
// load is issued as soon as its buffer's S product has completed, its value
// load once the P V product that used the buffer has, and the next S product
// right after this tile's P V product. The softmax keeps a reference maximum
// that moves only when a row's maximum exceeds it by more than 2^8; then the
// row of O in TMEM is rescaled. Exact either way: numerator and denominator
// share the reference.
#include "tc.cuh"

#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

namespace recsa {

constexpr int PA_T = 128;        // queries per CTA = keys per tile
constexpr int PA_THREADS = 256;  // two threads per query row (halves of the key and output columns)
constexpr float PA_RESCALE = 8.f;  // log2 units: the reference moves when a row's maximum exceeds it by 2^8

struct PrefillAttnArgs {
    float* state;  // [B][C][Hq][D + 2]: unnormalised acc, reference max, sum
    int C, Hq, G, n_tiles;
    float scale;
    int* err;
};

// Rotates rows of x [B][C][heads][D] (bf16) by their chunk offset into y.
template <int D>
__global__ void rope_chunk_kernel(const __nv_bfloat16* __restrict__ x, __nv_bfloat16* __restrict__ y,
                                  const float* __restrict__ rope, long long rows, int C, int heads) {
    constexpr int HD = D / 2;
    const long long total = rows * (HD / 2);
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const long long r = i / (HD / 2);
        const int c = (int)(i % (HD / 2)) * 2;  // pairs (c, c + HD) and (c + 1, c + 1 + HD)
        const int t = (int)((r / heads) % C);
        const __nv_bfloat16* src = x + r * D;
        const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(src + c);
        const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(src + HD + c);
        const float* tab = rope + (size_t)t * 3 * HD;
        const float2 cs = *reinterpret_cast<const float2*>(tab + c);
        const float2 sn = *reinterpret_cast<const float2*>(tab + HD + c);
        const float xa0 = __low2float(lo), xa1 = __high2float(lo), xb0 = __low2float(hi), xb1 = __high2float(hi);
        __nv_bfloat16* dst = y + r * D;
        *reinterpret_cast<__nv_bfloat162*>(dst + c) =
            __floats2bfloat162_rn(xa0 * cs.x - xb0 * sn.x, xa1 * cs.y - xb1 * sn.y);
        *reinterpret_cast<__nv_bfloat162*>(dst + HD + c) =
            __floats2bfloat162_rn(xb0 * cs.x + xa0 * sn.x, xb1 * cs.y + xa1 * sn.y);
    }
}

template <int D>
struct PaLayout {
    static constexpr int DT = D / 64;                      // 64-wide operand tiles along d
    static constexpr uint32_t TILE = PA_T * 128;           // one 64-wide tile of 128 rows
    static constexpr uint32_t QB = DT * TILE, KB = DT * TILE, PB = 2 * TILE;
    static constexpr uint32_t OFF_K = QB, OFF_V = OFF_K + 2 * KB, OFF_P = OFF_V + 2 * KB, OFF_BAR = OFF_P + PB;
    static constexpr uint32_t BYTES = OFF_BAR + 128 + 4 * PA_T * 4 + 1024;  // barriers, TMEM address, row
                                                                              // maxima and sums, alignment slack
};

template <int D>
__global__ void __launch_bounds__(PA_THREADS, 1)
    prefill_attn_kernel(const __grid_constant__ CUtensorMap mq, const __grid_constant__ CUtensorMap mk,
                        const __grid_constant__ CUtensorMap mv, PrefillAttnArgs a) {
    using LY = PaLayout<D>;
    constexpr int DT = LY::DT;
    constexpr int HK = PA_T / 2, HDC = D / 2;  // this thread's keys of a tile / output columns
    extern __shared__ unsigned char smem_pa[];
    const uint32_t raw = smem_addr(smem_pa);
    unsigned char* sm = smem_pa + (((raw + 1023u) & ~1023u) - raw);  // 1024-byte aligned tiles
    unsigned char* sQ = sm;
    auto sK = [&](int bf) { return sm + LY::OFF_K + bf * LY::KB; };  // double-buffered key tiles
    auto sV = [&](int bf) { return sm + LY::OFF_V + bf * LY::KB; };  // and value tiles
    unsigned char* sP = sm + LY::OFF_P;
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + LY::OFF_BAR);  // 0 q, 1-2 k, 3-4 v, 5-6 s, 7 o, 8 drain
    uint32_t* tbase = reinterpret_cast<uint32_t*>(bar + 10);         // TMEM base address
    float* xmax = reinterpret_cast<float*>(tbase + 4);               // [2][128] row maxima of the two halves
    float* xsum = xmax + 2 * PA_T;                                   // [2][128] row sums

    const int tid = threadIdx.x, warp = tid >> 5;
    const int rr = tid & (PA_T - 1), half = tid >> 7;  // query row, half of the columns
    const int qt = a.n_tiles - 1 - (int)blockIdx.x;  // longest rows first
    const int hq = blockIdx.y % a.Hq, bseq = blockIdx.y / a.Hq, h = hq / a.G;
    const int nkt = qt + 1;
    const int row = qt * PA_T + rr;  // this thread's query, offset in the chunk

    if (tid == 0) {
        for (int i = 0; i < 9; i++) mbar_init(&bar[i], 1);
        fence_mbar_init();
        tma_prefetch_map(&mq);
        tma_prefetch_map(&mk);
        tma_prefetch_map(&mv);
    }
    if (warp == 0) {
        tmem_alloc(tbase, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tbase;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;  // warps w and w + 4 share TMEM lanes
    // two S buffers (columns [0, 128) and [128, 256)): the product of the
    // next key tile runs while this tile's softmax does; O in [256, 256 + d)
    auto tS = [&](int bf) { return tmem + lane_off + bf * PA_T + half * HK; };
    const uint32_t tO = tmem + lane_off + 2 * PA_T + half * HDC;
    constexpr uint32_t ID_S = idesc_bf16(PA_T, PA_T, 0, 0), ID_O = idesc_bf16(PA_T, D, 0, 1);
    constexpr float LOG2E = 1.4426950408889634f;
    const float sc2 = a.scale * LOG2E;  // logits in log2 units

    // thread 0's bookkeeping of loads issued / waited per K and V buffer
    uint32_t k_iss0 = 0, k_iss1 = 0, k_wt0 = 0, k_wt1 = 0, v_iss0 = 0, v_iss1 = 0, v_wt0 = 0, v_wt1 = 0;
    auto load_tile = [&](const CUtensorMap* m, unsigned char* dst, int head, int row0, uint64_t* b) {
        mbar_arrive_expect_tx(b, DT * LY::TILE);
        for (int x = 0; x < DT; x++) tma_load_4d(dst + x * LY::TILE, m, x * 64, head, row0, bseq, b);
    };
    auto load_k = [&](int kt) {
        const int bf = kt & 1;
        load_tile(&mk, sK(bf), h, kt * PA_T, &bar[1 + bf]);
        (bf ? k_iss1 : k_iss0)++;
    };
    auto load_v = [&](int kt) {
        const int bf = kt & 1;
        load_tile(&mv, sV(bf), h, kt * PA_T, &bar[3 + bf]);
        (bf ? v_iss1 : v_iss0)++;
    };
    bool timeout = false;
    auto wait1 = [&](uint64_t* b, uint32_t& waited) {  // thread 0 only
        if (!mbar_wait(b, waited & 1u)) timeout = true;
        waited++;
    };
    auto issue_s = [&](int bf) {  // key buffer bf into S buffer bf (tile kt uses buffers kt & 1)
#pragma unroll
        for (int ks = 0; ks < D / 16; ks++) {
            const uint32_t off = (uint32_t)((ks >> 2) * LY::TILE + (ks & 3) * 32);
            mma_bf16_ss(tmem + bf * PA_T, kmajor_desc(smem_addr(sQ) + off), kmajor_desc(smem_addr(sK(bf)) + off),
                        ID_S, ks > 0);
        }
    };
    auto issue_pv = [&](int bf, bool acc) {
#pragma unroll
        for (int ks = 0; ks < PA_T / 16; ks++) {
            const uint32_t aoff = (uint32_t)((ks >> 2) * LY::TILE + (ks & 3) * 32);
            mma_bf16_ss(tmem + 2 * PA_T, kmajor_desc(smem_addr(sP) + aoff),
                        mnmajor_desc(smem_addr(sV(bf)) + (uint32_t)ks * 16 * 128, PA_T), ID_O, acc || ks > 0);
        }
    };

    uint32_t q_wt = 0;
    if (tid == 0) {
        mbar_arrive_expect_tx(&bar[0], DT * LY::TILE);
        for (int x = 0; x < DT; x++) tma_load_4d(sQ + x * LY::TILE, &mq, x * 64, hq, qt * PA_T, bseq, &bar[0]);
        load_k(0);
        load_v(0);
        if (nkt > 1) {
            load_k(1);
            load_v(1);
        }
        wait1(&bar[0], q_wt);
        wait1(&bar[1], k_wt0);
        tc_fence_after();
        if (!timeout) issue_s(0);
        mma_commit(&bar[5]);
        if (nkt > 1) {
            wait1(&bar[2], k_wt1);
            tc_fence_after();
            if (!timeout) issue_s(1);
            mma_commit(&bar[6]);
        }
    }

    float m_ref = -INFINITY, l = 0.f;  // log2 units
    bool ok = true;
    for (int kt = 0; kt < nkt; kt++) {
        const int bf = kt & 1;
        // S of this tile is in TMEM (S buffer bf, its (kt / 2)-th use)
        int bad = !mbar_wait(&bar[5 + bf], (uint32_t)(kt >> 1) & 1u);
        if (__syncthreads_or(bad || timeout)) {
            ok = false;
            break;
        }
        tc_fence_after();
        // S(kt) has completed: its key buffer takes tile kt + 2
        if (tid == 0 && kt + 2 < nkt) load_k(kt + 2);
        float s[HK];
#pragma unroll
        for (int c = 0; c < HK / 32; c++) tmem_ld32(tS(bf) + c * 32, s + c * 32);
        tmem_wait_ld();
        float mx = -INFINITY;
        if (kt == qt) {  // the diagonal tile: causal mask (and the chunk's end)
            const int key0 = kt * PA_T + half * HK;
#pragma unroll
            for (int j = 0; j < HK; j++) {
                const int key = key0 + j;
                s[j] = (key > row || key >= a.C) ? -INFINITY : s[j] * sc2;
                mx = fmaxf(mx, s[j]);
            }
        } else {
#pragma unroll
            for (int j = 0; j < HK; j++) {
                s[j] *= sc2;
                mx = fmaxf(mx, s[j]);
            }
        }
        xmax[half * PA_T + rr] = mx;
        // the previous tile's P V product is done: P and O are free, and so
        // is the value buffer of tile kt - 1, which takes tile kt + 1
        if (kt > 0) bad = !mbar_wait(&bar[7], (uint32_t)(kt - 1) & 1u);
        if (__syncthreads_or(bad)) {  // also publishes xmax
            ok = false;
            break;
        }
        tc_fence_after();
        if (tid == 0 && kt >= 1 && kt + 1 < nkt) load_v(kt + 1);
        mx = fmaxf(xmax[rr], xmax[PA_T + rr]);
        const float m_new = (mx > m_ref + PA_RESCALE) ? mx : m_ref;
        const bool move = kt > 0 && m_new != m_ref;
        const float alpha = move ? exp2f(m_ref - m_new) : 1.f;
        if (__any_sync(0xffffffffu, move)) {  // TMEM accesses are warp-wide
#pragma unroll 1
            for (int c = 0; c < HDC / 32; c++) {
                float o[32];
                tmem_ld32(tO + c * 32, o);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; i++) o[i] *= alpha;
                tmem_st32(tO + c * 32, o);
            }
            tmem_wait_st();
        }
        l *= alpha;
        m_ref = m_new;
        float ls = 0.f;
#pragma unroll
        for (int j = 0; j < HK; j += 8) {
            float p[8];
#pragma unroll
            for (int i = 0; i < 8; i++) {
                p[i] = exp2f(s[j + i] - m_ref);  // 0 for masked keys
                ls += p[i];
            }
            uint4 pk;
            __nv_bfloat162 h0 = __floats2bfloat162_rn(p[0], p[1]), h1 = __floats2bfloat162_rn(p[2], p[3]);
            __nv_bfloat162 h2 = __floats2bfloat162_rn(p[4], p[5]), h3 = __floats2bfloat162_rn(p[6], p[7]);
            pk.x = *reinterpret_cast<uint32_t*>(&h0);
            pk.y = *reinterpret_cast<uint32_t*>(&h1);
            pk.z = *reinterpret_cast<uint32_t*>(&h2);
            pk.w = *reinterpret_cast<uint32_t*>(&h3);
            *reinterpret_cast<uint4*>(sP + sw128_offset(rr, half * HK + j, PA_T)) = pk;
        }
        l += ls;
        fence_proxy_async_shared();  // P (generic writes) before the tensor core reads it
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            wait1(&bar[3 + bf], bf ? v_wt1 : v_wt0);
            if (!timeout) issue_pv(bf, kt > 0);
            mma_commit(&bar[7]);
            if (kt + 2 < nkt) {  // every thread has read S(kt): its buffer takes S(kt + 2)
                wait1(&bar[1 + bf], bf ? k_wt1 : k_wt0);
                if (!timeout) issue_s(bf);
                mma_commit(&bar[5 + bf]);
            }
        }
    }
    if (ok) {
        const int bad = !mbar_wait(&bar[7], (uint32_t)(nkt - 1) & 1u);
        ok = !__syncthreads_or(bad);
    }
    if (ok) {  // every thread loads (TMEM loads are warp-wide); rows past the chunk store nothing
        xsum[half * PA_T + rr] = l;
        tc_fence_after();
        float* st = a.state + (((size_t)bseq * a.C + row) * a.Hq + hq) * (D + 2);
#pragma unroll 1
        for (int c = 0; c < HDC / 32; c++) {
            float o[32];
            tmem_ld32(tO + c * 32, o);
            tmem_wait_ld();
            if (row < a.C)  // state rows are d + 2 floats: 8-byte aligned
#pragma unroll
                for (int i = 0; i < 32; i += 2)
                    *reinterpret_cast<float2*>(st + half * HDC + c * 32 + i) = make_float2(o[i], o[i + 1]);
        }
        __syncthreads();
        if (row < a.C && half == 0) {  // natural-log units for the merge
            st[D] = m_ref / LOG2E;
            st[D + 1] = xsum[rr] + xsum[PA_T + rr];
        }
    }
    if (!ok && tid == 0) {
        flag_error(a.err, ERR_TIMEOUT);
        // let every product and copy still in flight finish before the CTA
        // frees its tensor memory and leaves (each wait bounded)
        mma_commit(&bar[8]);
        mbar_wait(&bar[8], 0);
        while (k_wt0 < k_iss0) wait1(&bar[1], k_wt0);
        while (k_wt1 < k_iss1) wait1(&bar[2], k_wt1);
        while (v_wt0 < v_iss0) wait1(&bar[3], v_wt0);
        while (v_wt1 < v_iss1) wait1(&bar[4], v_wt1);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------ tensor maps

namespace {
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;
}  // namespace

bool encode_bf16_map(CUtensorMap* map, int rank, void* base, const unsigned long long* dims,
                     const unsigned long long* strides, const unsigned* box) {
    std::call_once(g_encode_once, []() {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    if (!g_encode || rank < 2 || rank > 5) return false;
    cuuint64_t gd[5], gs[4];
    cuuint32_t bx[5], es[5];
    for (int i = 0; i < rank; i++) {
        gd[i] = dims[i];
        bx[i] = box[i];
        es[i] = 1;
    }
    for (int i = 0; i < rank - 1; i++) gs[i] = strides[i];
    CUtensorMap m;
    const CUresult r = g_encode(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, base, gd, gs, bx, es,
                                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return false;
    *map = m;
    return true;
}

// q [B][C][Hq][D], k, v [B][C][H][D] (bf16); qr, kr: scratch of the same
// shapes as q and k (256-byte aligned) for the rotated copies.
template <int D>
cudaError_t launch_prefill_attn(const TreeParams& p, const void* q, const void* k, const void* v, float* state,
                                void* qr, void* kr, int B, int C, int Hq, int H, cudaStream_t s) {
    const __nv_bfloat16* qb = reinterpret_cast<const __nv_bfloat16*>(q);
    const __nv_bfloat16* kb = reinterpret_cast<const __nv_bfloat16*>(k);
    __nv_bfloat16* qrb = reinterpret_cast<__nv_bfloat16*>(qr);
    __nv_bfloat16* krb = reinterpret_cast<__nv_bfloat16*>(kr);
    {
        const long long rq = (long long)B * C * Hq, rk = (long long)B * C * H;
        const int blocks_q = (int)std::min<long long>((rq * (D / 4) + 255) / 256, 148 * 16);
        const int blocks_k = (int)std::min<long long>((rk * (D / 4) + 255) / 256, 148 * 16);
        rope_chunk_kernel<D><<<blocks_q, 256, 0, s>>>(qb, qrb, p.rope, rq, C, Hq);
        rope_chunk_kernel<D><<<blocks_k, 256, 0, s>>>(kb, krb, p.rope, rk, C, H);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    CUtensorMap mq, mk, mv;
    const unsigned box[4] = {64, 1, PA_T, 1};
    const unsigned long long dq[4] = {(unsigned long long)D, (unsigned long long)Hq, (unsigned long long)C,
                                      (unsigned long long)B};
    const unsigned long long sq[3] = {(unsigned long long)D * 2, (unsigned long long)Hq * D * 2,
                                      (unsigned long long)C * Hq * D * 2};
    const unsigned long long dk[4] = {(unsigned long long)D, (unsigned long long)H, (unsigned long long)C,
                                      (unsigned long long)B};
    const unsigned long long sk[3] = {(unsigned long long)D * 2, (unsigned long long)H * D * 2,
                                      (unsigned long long)C * H * D * 2};
    if (!encode_bf16_map(&mq, 4, qr, dq, sq, box) || !encode_bf16_map(&mk, 4, kr, dk, sk, box) ||
        !encode_bf16_map(&mv, 4, const_cast<void*>(v), dk, sk, box))
        return cudaErrorInvalidValue;
    PrefillAttnArgs a{state, C, Hq, Hq / H, (C + PA_T - 1) / PA_T, (float)(1.0 / sqrt((double)D)), p.err};
    const int smem = (int)PaLayout<D>::BYTES;
    auto kern = prefill_attn_kernel<D>;
    static std::atomic<unsigned long long> attr_done{0};
    cudaError_t e = set_smem_limit(kern, smem, attr_done);
    if (e != cudaSuccess) return e;
    dim3 grid(a.n_tiles, B * Hq);
    kern<<<grid, PA_THREADS, smem, s>>>(mq, mk, mv, a);
    return cudaGetLastError();
}

template cudaError_t launch_prefill_attn<64>(const TreeParams&, const void*, const void*, const void*, float*, void*,
                                             void*, int, int, int, int, cudaStream_t);
template cudaError_t launch_prefill_attn<128>(const TreeParams&, const void*, const void*, const void*, float*,
                                              void*, void*, int, int, int, int, cudaStream_t);

}  // namespace recsa
