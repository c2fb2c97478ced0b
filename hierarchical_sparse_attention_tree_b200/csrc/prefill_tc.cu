// Prefill, tree part, on the tensor cores: the chunk's tokens descend the
// tree together, level by level, with the candidate scoring and the value
// products as tcgen05 matrix products over parent buckets.
//
// Method (RecSA abstract; kongchang.com article "Core Idea", "Position
// Encoding"): each chunk token t runs the decode descent over the tree of
// the s cached tokens: at each level the candidates are the children of its
// kept parents (ascending), each scored at its index among them (RoPE), the
// best k kept (GQA: ranked by the sum of the G heads' logits), the others
// entering one softmax as summaries; the tokens under the kept level-1 nodes
// enter exactly, followed by the chunk's own tokens s..t (the chunk-local
// part, computed separately and merged here).
//
// Work split. The children of one parent node are one contiguous block of b
// rows, and in token t's candidate list the block of its r-th kept parent
// starts at index r*b. So a (token, rank, parent) pair needs the logits of
// the query, rotated to P_t - r*b, against the parent's b child keys,
// rotated by their offset o < b (only the angle difference enters a logit).
// Per level the pairs are grouped by parent (a counting sort); one tile is a
// parent and up to 128 / G of its pairs, i.e. the product
//     [128 rows (pair, head) x d] x [d x b]
// on tcgen05 (M = 128, N = b rounded up to 32, fp32 accumulator in TMEM).
// The operands are fp32 after rotation; each is split into bf16 hi + lo
// parts and the product taken as hi*hi + hi*lo + lo*hi, which leaves an
// error of about 2^-16 of each term: far below the 1e-4 margin under which
// two selection scores count as a near tie. One kernel writes the selection
// scores (the G logits summed), one warp per token then takes the exact top
// k of its packed (score, node id) keys. After the descent the same tiles
// are run again for the value products: the logits are recomputed, turned
// into weights exp(logit - M) with one reference M per (token, head) (the
// largest tree logit of any level, so no rescaling is needed), kept children
// masked out, and [128 x b] x [b x d] (weights split hi + lo, values bf16)
// accumulated in TMEM, then added into per-(token, head) fp32 sums.
#include "tc.cuh"

#include <algorithm>

namespace recsa {

constexpr int TP_THREADS = 128;
constexpr int TP_KMAX = 64;
constexpr int MODE_SCORE = 0, MODE_MAX = 1, MODE_VALUE = 2;

// Per-level arrays in the prefill scratch. Level j's pairs are grouped by
// their parent, a node of level j + 1 (R rows per unit).
struct PfLevel {
    int* kept;    // [U][C][k] kept node ids of level j, ascending (j >= 1)
    int* nkept;   // [U][C]
    int* nc;      // [U][C] candidates at level j (0: no tree or above the unit's top)
    int* cnt;     // [U * R] pairs per parent
    int* off;     // [U * R] first pair of each parent's bucket
    int* toff;    // [U * R] first tile of each parent's bucket
    int* cursor;  // [U * R]
    int* pairs;   // [U * C * k] t * 64 + r, grouped by parent
    int4* tiles;  // [max_tiles] (unit, parent, first pair, pairs)
    int* ntiles;  // [1]
    int R, max_tiles;
};

struct PfArgs {
    const __nv_bfloat16* q;  // [B][C][Hq][D]
    int C, Hq, TP;           // TP: pairs per tile (128 / G)
    float* S;                // [U][C][maxc] selection scores of the level being descended
    int maxc;
    unsigned* mkey;          // [B][C][Hq] ordered key of the largest tree logit (0: none)
    float* oacc;             // [B][C][Hq][D]
    float* lacc;             // [B][C][Hq]
    long long* rows;         // [U][C][2] key rows scored, value rows (tree entries)
    int* sel_out;            // nullable [B][C][H][J_cap][k]
};

// Top level of the tree over S >= 1 tokens: the first level with at most b nodes.
__device__ __forceinline__ int pf_top(const TreeParams& p, long long S) {
    int J = 1;
    while (J < p.J_cap && ceil_div_ll(S, p.span[J]) > p.b) J++;
    return J;
}

// Parents of token t of unit u at level j (nodes of level j + 1): the kept
// list of level j + 1, or the single top node above the unit's top level.
__device__ __forceinline__ const int* pf_parents(const PfLevel& up, int j, int J, long long ut, int k, int* npar,
                                                 const int* zero) {
    if (j == J) {
        *npar = 1;
        return zero;
    }
    *npar = up.nkept[ut];
    return up.kept + ut * k;
}

__device__ __forceinline__ float key_float(unsigned key) {
    const unsigned u = (key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key;
    return __uint_as_float(u);
}

// ---------------------------------------------------------- candidates

// Per (unit, token): the candidate count at level j and, for a level that
// is scored (more than k candidates) or the tokens (j = 0), one pair per
// kept parent counted into its parent's bucket.
__global__ void pf_cand_kernel(TreeParams p, PfArgs a, PfLevel L, PfLevel up, int j) {
    const long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    const long long U = (long long)p.B * p.H;
    const bool act = idx < U * a.C;
    const long long u = act ? idx / a.C : 0;
    const long long S = act ? p.len[u] : 0;
    int nc = 0, npar = 0;
    const int zero = 0;
    const int* par = &zero;
    if (S > 0) {
        const int J = pf_top(p, S);
        if (j <= J) {
            par = pf_parents(up, j, J, idx, p.k, &npar, &zero);
            const long long n_j = j == 0 ? S : ceil_div_ll(S, p.span[j]);
            const int last = par[npar - 1];
            nc = (npar - 1) * p.b + (int)min((long long)p.b, n_j - (long long)last * p.b);
            if (j == 0) {  // every token under the kept level-1 nodes is read and enters the softmax
                a.rows[idx * 2] += nc;
                a.rows[idx * 2 + 1] += nc;
            }
        }
    }
    if (act) L.nc[idx] = nc;
    // one pair per kept parent into its bucket's count; lanes adding to the
    // same bucket are combined into one atomic (tokens of a warp tend to keep
    // the same parents)
    const int np = (j == 0 || nc > p.k) ? npar : 0;
    int maxnp = np;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) maxnp = max(maxnp, __shfl_xor_sync(0xffffffffu, maxnp, o));
    const int lane = threadIdx.x & 31;
    for (int r = 0; r < maxnp; r++) {
        const bool mine = r < np;
        const unsigned am = __ballot_sync(0xffffffffu, mine);
        if (mine) {
            const long long slot = u * L.R + par[r];
            const unsigned m = __match_any_sync(am, slot);
            if (lane == __ffs(m) - 1) atomicAdd(&L.cnt[slot], __popc(m));
        }
    }
}

// Exclusive scans of the bucket sizes (pairs) and of the tiles per bucket,
// one CTA of 1024 threads, each scanning a contiguous range (a multiple of 4
// buckets, read and written as int4 with every load of the range in flight
// at once); also clears the scatter cursors and stores the tile count.
__global__ void __launch_bounds__(1024) pf_scan_kernel(PfLevel L, int n, int TP, int* err) {
    __shared__ int sp[1024], st[1024];
    const int tid = threadIdx.x;
    const int per = (((n + 1023) / 1024) + 3) & ~3;
    const int lo = min(n, tid * per), hi = min(n, lo + per);
    const int nv = (hi - lo) / 4;  // whole int4 groups (lo is a multiple of 4)
    int cp = 0, ct = 0;
    {
        const int4* c4 = reinterpret_cast<const int4*>(L.cnt + lo);
#pragma unroll 8
        for (int v = 0; v < nv; v++) {
            const int4 c = c4[v];
            cp += (c.x + c.y) + (c.z + c.w);
            ct += (c.x + TP - 1) / TP + (c.y + TP - 1) / TP + (c.z + TP - 1) / TP + (c.w + TP - 1) / TP;
        }
        for (int i = lo + 4 * nv; i < hi; i++) {
            const int c = L.cnt[i];
            cp += c;
            ct += (c + TP - 1) / TP;
        }
    }
    sp[tid] = cp;
    st[tid] = ct;
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {  // inclusive Hillis-Steele scan
        const int vp = tid >= o ? sp[tid - o] : 0, vt = tid >= o ? st[tid - o] : 0;
        __syncthreads();
        sp[tid] += vp;
        st[tid] += vt;
        __syncthreads();
    }
    int rp = sp[tid] - cp, rt = st[tid] - ct;
    {
        const int4* c4 = reinterpret_cast<const int4*>(L.cnt + lo);
        int4* o4 = reinterpret_cast<int4*>(L.off + lo);
        int4* t4 = reinterpret_cast<int4*>(L.toff + lo);
        int4* z4 = reinterpret_cast<int4*>(L.cursor + lo);
#pragma unroll 4
        for (int v = 0; v < nv; v++) {
            const int4 c = c4[v];
            int4 o, t;
            o.x = rp; t.x = rt; rp += c.x; rt += (c.x + TP - 1) / TP;
            o.y = rp; t.y = rt; rp += c.y; rt += (c.y + TP - 1) / TP;
            o.z = rp; t.z = rt; rp += c.z; rt += (c.z + TP - 1) / TP;
            o.w = rp; t.w = rt; rp += c.w; rt += (c.w + TP - 1) / TP;
            o4[v] = o;
            t4[v] = t;
            z4[v] = make_int4(0, 0, 0, 0);
        }
        for (int i = lo + 4 * nv; i < hi; i++) {
            const int c = L.cnt[i];
            L.off[i] = rp;
            L.toff[i] = rt;
            L.cursor[i] = 0;
            rp += c;
            rt += (c + TP - 1) / TP;
        }
    }
    if (tid == 1023) {
        const int total = st[1023];
        if (total > L.max_tiles) flag_error(err, ERR_SHAPE);
        *L.ntiles = min(total, L.max_tiles);
    }
}

// Writes each pair (t, r) into its parent's bucket (positions taken per
// group of lanes with the same bucket, one atomic per group).
__global__ void pf_scatter_kernel(TreeParams p, PfArgs a, PfLevel L, PfLevel up, int j) {
    const long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    const long long U = (long long)p.B * p.H;
    const bool act = idx < U * a.C;
    const int nc = act ? L.nc[idx] : 0;
    const bool scored = nc > 0 && (j == 0 || nc > p.k);
    const long long u = act ? idx / a.C : 0;
    const int t = act ? (int)(idx % a.C) : 0;
    const int zero = 0;
    int npar = 0;
    const int* par = &zero;
    if (scored) par = pf_parents(up, j, pf_top(p, p.len[u]), idx, p.k, &npar, &zero);
    int maxnp = npar;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) maxnp = max(maxnp, __shfl_xor_sync(0xffffffffu, maxnp, o));
    const int lane = threadIdx.x & 31;
    for (int r = 0; r < maxnp; r++) {
        const bool mine = r < npar;
        const unsigned am = __ballot_sync(0xffffffffu, mine);
        if (mine) {
            const long long slot = u * L.R + par[r];
            const unsigned m = __match_any_sync(am, slot);
            const int leader = __ffs(m) - 1;
            int base = 0;
            if (lane == leader) base = atomicAdd(&L.cursor[slot], __popc(m));
            base = __shfl_sync(m, base, leader);
            const int pos = L.off[slot] + base + __popc(m & ((1u << lane) - 1u));
            L.pairs[pos] = t * 64 + r;
        }
    }
}

// The tile list: bucket of (unit, parent) cut into pieces of TP pairs.
__global__ void pf_tiles_kernel(PfLevel L, int n, int TP) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const int c = L.cnt[i];
    for (int x = 0, t0 = L.toff[i]; x * TP < c; x++) {
        if (t0 + x >= L.max_tiles) return;
        L.tiles[t0 + x] = make_int4(i / L.R, i % L.R, L.off[i] + x * TP, min(TP, c - x * TP));
    }
}

// ------------------------------------------------------------ the tiles

template <int D>
struct TpLayout {
    static constexpr int DT = D / 64;
    static constexpr uint32_t A = DT * 128 * 128;  // one of A_hi / A_lo (128 rows)
    __host__ __device__ static uint32_t B(int NB) { return (uint32_t)DT * NB * 128; }
    // alignment slack for a dynamic shared memory start that is 128-byte
    // aligned (checked at run time): small enough that two CTAs fit an SM
    static constexpr uint32_t SLACK = 896;
    __host__ __device__ static uint32_t bytes(int NB) { return 2 * A + 3 * B(NB) + 16 + SLACK; }
};

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

// Rotation of one pair (xa, xb) by the table row (c, s), the same fp32
// arithmetic as the decode path's scoring.
__device__ __forceinline__ void rot_pair(float xa, float xb, float c, float s, float& ra, float& rb) {
    ra = fmaf(xa, c, xb * -s);
    rb = fmaf(xb, c, xa * s);
}

__device__ __forceinline__ uint4 pack8(const float* v) {
    uint4 r;
    __nv_bfloat162 h0 = __floats2bfloat162_rn(v[0], v[1]), h1 = __floats2bfloat162_rn(v[2], v[3]);
    __nv_bfloat162 h2 = __floats2bfloat162_rn(v[4], v[5]), h3 = __floats2bfloat162_rn(v[6], v[7]);
    r.x = *reinterpret_cast<uint32_t*>(&h0);
    r.y = *reinterpret_cast<uint32_t*>(&h1);
    r.z = *reinterpret_cast<uint32_t*>(&h2);
    r.w = *reinterpret_cast<uint32_t*>(&h3);
    return r;
}
// Splits 8 floats into bf16 hi (round to nearest) and lo = x - hi (rounded).
__device__ __forceinline__ void split8(const float* x, uint4& hi, uint4& lo) {
    float h[8], l[8];
#pragma unroll
    for (int i = 0; i < 8; i++) {
        h[i] = __bfloat162float(__float2bfloat16_rn(x[i]));
        l[i] = x[i] - h[i];
    }
    hi = pack8(h);
    lo = pack8(l);
}

// bf16 pair (packed in 32 bits) <-> two floats.
__device__ __forceinline__ float2 bf2_f2(uint32_t v) {
    return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xFFFF0000u));
}
__device__ __forceinline__ uint32_t f2_bf2(float2 x) {
    __nv_bfloat162 h = __floats2bfloat162_rn(x.x, x.y);
    return *reinterpret_cast<uint32_t*>(&h);
}

// One 8-frequency chunk: rotates (xa, xb) = dims [f, f + 8) and [HD + f,
// HD + f + 8) by the table's (cos, sin), in packed fp32 (the same arithmetic
// as the decode path's scoring), and stores both halves at `row` of two
// K-major swizzled operands of `rows` rows: hi = bf16(x) and, if LO,
// lo = bf16(x - hi). cs: cos [2], sin [2] as float4 (x b (-s) is the exact
// negation of b s, so -sin is not loaded).
template <int D, bool LO>
__device__ __forceinline__ void put_chunk(uint4 xa_raw, uint4 xb_raw, const float4* cs, int f,
                                          unsigned char* hi_base, unsigned char* lo_base, int row, int rows) {
    constexpr int HD = D / 2;
    const uint32_t xa[4] = {xa_raw.x, xa_raw.y, xa_raw.z, xa_raw.w};
    const uint32_t xb[4] = {xb_raw.x, xb_raw.y, xb_raw.z, xb_raw.w};
    const float2 c2[4] = {make_float2(cs[0].x, cs[0].y), make_float2(cs[0].z, cs[0].w), make_float2(cs[1].x, cs[1].y),
                          make_float2(cs[1].z, cs[1].w)};
    const float2 s2[4] = {make_float2(cs[2].x, cs[2].y), make_float2(cs[2].z, cs[2].w), make_float2(cs[3].x, cs[3].y),
                          make_float2(cs[3].z, cs[3].w)};
    const float2 n2[4] = {make_float2(-cs[2].x, -cs[2].y), make_float2(-cs[2].z, -cs[2].w),
                          make_float2(-cs[3].x, -cs[3].y), make_float2(-cs[3].z, -cs[3].w)};
    uint32_t ha[4], la[4], hb[4], lb[4];
    const float2 m1 = make_float2(-1.f, -1.f);
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const float2 a = bf2_f2(xa[i]), b = bf2_f2(xb[i]);
        const float2 ra = ffma2(a, c2[i], fmul2(b, n2[i]));
        const float2 rb = ffma2(b, c2[i], fmul2(a, s2[i]));
        ha[i] = f2_bf2(ra);
        hb[i] = f2_bf2(rb);
        if (LO) {
            la[i] = f2_bf2(ffma2(bf2_f2(ha[i]), m1, ra));
            lb[i] = f2_bf2(ffma2(bf2_f2(hb[i]), m1, rb));
        }
    }
    const uint32_t oa = sw128_offset(row, f, rows), ob = sw128_offset(row, HD + f, rows);
    *reinterpret_cast<uint4*>(hi_base + oa) = make_uint4(ha[0], ha[1], ha[2], ha[3]);
    *reinterpret_cast<uint4*>(hi_base + ob) = make_uint4(hb[0], hb[1], hb[2], hb[3]);
    if (LO) {
        *reinterpret_cast<uint4*>(lo_base + oa) = make_uint4(la[0], la[1], la[2], la[3]);
        *reinterpret_cast<uint4*>(lo_base + ob) = make_uint4(lb[0], lb[1], lb[2], lb[3]);
    }
}
// The table's cos and sin of frequencies [f, f + 8) of row `tab`.
template <int D>
__device__ __forceinline__ void load_cs(const float* tab, int f, float4* cs) {
    constexpr int HD = D / 2;
#pragma unroll
    for (int x = 0; x < 2; x++) {
        cs[2 * x] = __ldg(reinterpret_cast<const float4*>(tab + x * HD + f));
        cs[2 * x + 1] = __ldg(reinterpret_cast<const float4*>(tab + x * HD + f + 4));
    }
}

__device__ __forceinline__ void cp_async16(void* dst_smem, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst_smem)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
__device__ __forceinline__ void prefetch_l2(const void* p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// One persistent CTA loops over the level's tiles. MODE_SCORE: selection
// scores and the largest logit; MODE_MAX (tokens): the largest logit;
// MODE_VALUE: the weighted values of the entries. NB = b rounded up to 32.
template <int D, int NB, int MODE>
__global__ void __launch_bounds__(TP_THREADS, 2) pf_tile_kernel(TreeParams p, PfArgs a, PfLevel L, int j, int G) {
    using LY = TpLayout<D>;
    constexpr int HD = D / 2, NCH = HD / 8;           // 8-frequency chunks per row
    constexpr int BU = NB * NCH / TP_THREADS;         // (key row, chunk) units per thread
    constexpr int VU = NB * (D / 8) / TP_THREADS;     // 16-byte value pieces per thread
    extern __shared__ unsigned char smem_tp[];
    const uint32_t raw = smem_addr(smem_tp);
    const uint32_t pad = ((raw + 1023u) & ~1023u) - raw;
    unsigned char* sm = smem_tp + pad;
    unsigned char* sAh = sm;
    unsigned char* sAl = sm + LY::A;
    unsigned char* sBh = sm + 2 * LY::A;
    unsigned char* sBl = sBh + LY::B(NB);
    unsigned char* sV = sBl + LY::B(NB);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sV + LY::B(NB));
    uint32_t* tbase = reinterpret_cast<uint32_t*>(bar + 1);
    if (pad > LY::SLACK) {  // the dynamic shared memory start was not aligned as assumed
        if (threadIdx.x == 0) flag_error(p.err, ERR_SHAPE);
        return;
    }

    const int tid = threadIdx.x, warp = tid >> 5;
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tbase, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tbase;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    constexpr uint32_t ID_L = idesc_bf16(128, NB, 0, 0), ID_O = idesc_bf16(128, D, 0, 1);
    uint32_t phase = 0;
    bool ok = true;

    const int ntiles = *L.ntiles;
    const int b = p.b, k = p.k;
    const __nv_bfloat16* kb = reinterpret_cast<const __nv_bfloat16*>(p.K[j]);
    const __nv_bfloat16* vb = reinterpret_cast<const __nv_bfloat16*>(p.V[j]);
    const long long ustride = j == 0 ? p.cap : p.rows[j];
    const int pr = tid / G, g = tid % G;  // this thread's row: pair pr, head g
    // Each tile's descriptor, its unit's length, this thread's pair and the
    // pair's candidate count are loaded one tile ahead (a chain of dependent
    // loads that then overlaps the previous tile's products).
    int4 tile_n = make_int4(0, 0, 0, 0);
    long long S_n = 0;
    int pk_n = 0, nc_n = 0;
    if ((int)blockIdx.x < ntiles) {
        tile_n = L.tiles[blockIdx.x];
        S_n = p.len[tile_n.x];
        if (pr < tile_n.w) {
            pk_n = L.pairs[tile_n.z + pr];
            nc_n = L.nc[tile_n.x * a.C + (pk_n >> 6)];
        }
    }
    for (int ti = blockIdx.x; ti < ntiles && ok; ti += gridDim.x) {
        const int4 tile = tile_n;
        const long long u = tile.x;
        const int par = tile.y, first = tile.z, npairs = tile.w;
        const int bseq = (int)(u / p.H), h = (int)(u % p.H);
        const long long S = S_n;
        const int pk_cur = pk_n, nc_cur = nc_n;
        const bool has_next = ti + (int)gridDim.x < ntiles;
        if (has_next) tile_n = L.tiles[ti + gridDim.x];
        const long long n_j = j == 0 ? S : ceil_div_ll(S, p.span[j]);
        const int nchild = (int)min((long long)b, n_j - (long long)par * b);
        // first child row (a page of tokens at level 0 of a paged cache)
        const long long crow = j == 0 ? token_row(token_map(p), u, (long long)par * b) : u * ustride + (long long)par * b;
        const bool valid = pr < npairs;
        int t = 0, r = 0, P = -1;
        if (valid) {
            t = pk_cur >> 6;
            r = pk_cur & 63;
            P = (j == 0 ? nc_cur + t : nc_cur - 1) - r * b;  // the query's angle for this parent's block
        }
        (void)first;
        const int hq = h * G + g;
        const long long orow = ((long long)bseq * a.C + t) * a.Hq + hq;  // (sequence, token, head)
        const bool qok = valid && P >= 0 && P < p.npos;
        // ---- every load of this tile issued before any arithmetic
        uint4 qa[NCH], qb[NCH];
        if (qok) {
            const __nv_bfloat16* src = a.q + orow * D;
#pragma unroll
            for (int c = 0; c < NCH; c++) {
                qa[c] = __ldg(reinterpret_cast<const uint4*>(src + c * 8));
                qb[c] = __ldg(reinterpret_cast<const uint4*>(src + HD + c * 8));
            }
        }
        uint4 ka[BU], kbv[BU];
#pragma unroll
        for (int x = 0; x < BU; x++) {
            const int unit = tid + x * TP_THREADS, o = unit / NCH, c = unit % NCH;
            if (o < nchild) {
                const __nv_bfloat16* src = kb + (crow + o) * D;
                ka[x] = __ldg(reinterpret_cast<const uint4*>(src + c * 8));
                kbv[x] = __ldg(reinterpret_cast<const uint4*>(src + HD + c * 8));
            }
        }
        if (MODE == MODE_VALUE) {
#pragma unroll
            for (int x = 0; x < VU; x++) {
                const int unit = tid + x * TP_THREADS, o = unit / (D / 8), c = (unit % (D / 8)) * 8;
                unsigned char* dst = sV + sw128_offset(o, c, NB);
                if (o < nchild)
                    cp_async16(dst, vb + (crow + o) * D + c);
                else
                    *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
            }
        }
        // the next tile's child rows into L2 while this one is computed, and
        // the next links of its metadata chain
        if (has_next) {
            const int4 nt = tile_n;
            const long long nrow = j == 0 ? token_row(token_map(p), nt.x, (long long)nt.y * b)
                                          : (long long)nt.x * ustride + (long long)nt.y * b;
            if (tid * 64 < b * D) prefetch_l2(kb + nrow * D + tid * 64);
            if (MODE == MODE_VALUE && tid * 64 < b * D) prefetch_l2(vb + nrow * D + tid * 64);
            S_n = p.len[nt.x];
            pk_n = pr < nt.w ? L.pairs[nt.z + pr] : 0;
        }
        // ---- operands: the rotated query and keys, split hi / lo
        // (the largest-logit pass of the tokens needs only an approximate
        // reference maximum: hi parts and one product)
        constexpr bool LO = MODE != MODE_MAX;
        {
            const float* tab = p.rope + (size_t)(qok ? P : 0) * 3 * HD;
            float4 cs[4], cn[4];
            load_cs<D>(tab, 0, cs);
            const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int c = 0; c < NCH; c++) {
                if (c + 1 < NCH) load_cs<D>(tab, (c + 1) * 8, cn);
                put_chunk<D, LO>(qok ? qa[c] : z, qok ? qb[c] : z, cs, c * 8, sAh, sAl, tid, 128);
#pragma unroll
                for (int i = 0; i < 4; i++) cs[i] = cn[i];
            }
        }
#pragma unroll
        for (int x = 0; x < BU; x++) {
            const int unit = tid + x * TP_THREADS, o = unit / NCH, c = unit % NCH;
            float4 cs[4];
            load_cs<D>(p.rope + (size_t)o * 3 * HD, c * 8, cs);
            const uint4 z = make_uint4(0, 0, 0, 0);
            put_chunk<D, LO>(o < nchild ? ka[x] : z, o < nchild ? kbv[x] : z, cs, c * 8, sBh, sBl, o, NB);
        }
        if (has_next && pr < tile_n.w) nc_n = L.nc[tile_n.x * a.C + (pk_n >> 6)];
        // value pass: the children this token kept (not entries) and its
        // reference maximum, loaded before the products so that their
        // latency overlaps them
        unsigned long long keep[(NB + 63) / 64];
#pragma unroll
        for (int x = 0; x < (NB + 63) / 64; x++) keep[x] = 0ull;
        unsigned mk = 0u;
        if (MODE == MODE_VALUE) {
            if (valid && j > 0) {
                const int* kl = L.kept + (u * a.C + t) * k;
                const int nk = L.nkept[u * a.C + t];
                for (int x = 0; x < nk; x++) {
                    const int o = kl[x] - par * b;
                    if (o >= 0 && o < NB) keep[o >> 6] |= 1ull << (o & 63);
                }
            }
            mk = valid ? a.mkey[orow] : 0u;
            cp_async_wait_all();
        }
        fence_proxy_async_shared();
        tc_fence_before();
        __syncthreads();
        // ---- logits: hi*hi + hi*lo + lo*hi
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int pass = 0; pass < (MODE == MODE_MAX ? 1 : 3); pass++) {
                const uint32_t ab = smem_addr(pass == 2 ? sAl : sAh), bb = smem_addr(pass == 1 ? sBl : sBh);
#pragma unroll
                for (int ks = 0; ks < D / 16; ks++) {
                    const uint32_t ao = (uint32_t)((ks >> 2) * 128 * 128 + (ks & 3) * 32);
                    const uint32_t bo = (uint32_t)((ks >> 2) * NB * 128 + (ks & 3) * 32);
                    mma_bf16_ss(tmem, kmajor_desc(ab + ao), kmajor_desc(bb + bo), ID_L, pass > 0 || ks > 0);
                }
            }
            mma_commit(bar);
        }
        {
            const int bad = !mbar_wait(bar, phase);
            phase ^= 1u;
            if (__syncthreads_or(bad)) {
                ok = false;
                break;
            }
        }
        tc_fence_after();
        float lg[NB];
#pragma unroll
        for (int c = 0; c < NB / 32; c++) tmem_ld32(tmem + lane_off + c * 32, lg + c * 32);
        tmem_wait_ld();
        float mx = -INFINITY;
#pragma unroll
        for (int o = 0; o < NB; o++) {
            lg[o] = o < nchild ? lg[o] * p.scale : -INFINITY;
            mx = fmaxf(mx, lg[o]);
        }
        if (MODE != MODE_VALUE) {
            if (valid && mx > -INFINITY) atomicMax(&a.mkey[orow], float_key(mx));
        }
        if (MODE == MODE_SCORE) {
            // S = sum over the G heads (G consecutive lanes), written by the
            // G lanes in turn
            // (each lane then writes a contiguous 1/G of the row, 16 bytes at a time)
            float* srow = a.S + (u * a.C + t) * (long long)a.maxc + (long long)r * b;
#pragma unroll
            for (int o = 0; o < NB; o++)
                for (int m = 1; m < G; m <<= 1) lg[o] += __shfl_xor_sync(0xffffffffu, lg[o], m);
            const int per = NB / G;
            if (valid) {
#pragma unroll
                for (int o0 = 0; o0 < NB; o0 += 4) {
                    if (o0 >= g * per && o0 < (g + 1) * per) {
                        if (o0 + 4 <= nchild)
                            *reinterpret_cast<float4*>(srow + o0) = make_float4(lg[o0], lg[o0 + 1], lg[o0 + 2], lg[o0 + 3]);
                        else
                            for (int i = o0; i < nchild; i++) srow[i] = lg[i];
                    }
                }
            }
        }
        if (MODE == MODE_VALUE) {
            // weights of the entries: every token; above, the children this
            // token did not keep
            const float mref = mk ? key_float(mk) : 0.f;
            constexpr float LOG2E = 1.4426950408889634f;
            const float mref2 = mref * LOG2E;
            float lsum = 0.f;
#pragma unroll
            for (int o0 = 0; o0 < NB; o0 += 8) {
                float w[8];
#pragma unroll
                for (int i = 0; i < 8; i++) {
                    const int o = o0 + i;
                    const bool kept = (keep[o >> 6] >> (o & 63)) & 1ull;
                    w[i] = (mk != 0u && o < nchild && !kept) ? exp2f(fmaf(lg[o], LOG2E, -mref2)) : 0.f;
                    lsum += w[i];
                }
                uint4 hi, lo;
                split8(w, hi, lo);
                *reinterpret_cast<uint4*>(sAh + sw128_offset(tid, o0, 128)) = hi;
                *reinterpret_cast<uint4*>(sAl + sw128_offset(tid, o0, 128)) = lo;
            }
            if (lsum > 0.f) atomicAdd(&a.lacc[orow], lsum);
            fence_proxy_async_shared();
            tc_fence_before();
            __syncthreads();
            if (tid == 0) {
                tc_fence_after();
#pragma unroll
                for (int pass = 0; pass < 2; pass++) {
                    const uint32_t ab = smem_addr(pass == 0 ? sAh : sAl), vbs = smem_addr(sV);
#pragma unroll
                    for (int ks = 0; ks < NB / 16; ks++) {
                        const uint32_t ao = (uint32_t)((ks >> 2) * 128 * 128 + (ks & 3) * 32);
                        mma_bf16_ss(tmem + 128, kmajor_desc(ab + ao), mnmajor_desc(vbs + (uint32_t)ks * 16 * 128, NB),
                                    ID_O, pass > 0 || ks > 0);
                    }
                }
                mma_commit(bar);
            }
            {
                const int bad = !mbar_wait(bar, phase);
                phase ^= 1u;
                if (__syncthreads_or(bad)) {
                    ok = false;
                    break;
                }
            }
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < D / 32; c++) {
                float o[32];
                tmem_ld32(tmem + lane_off + 128 + c * 32, o);
                tmem_wait_ld();
                if (lsum > 0.f) {
                    float* dst = a.oacc + orow * D + c * 32;
#pragma unroll
                    for (int i = 0; i < 32; i += 4) red_add_v4(dst + i, o[i], o[i + 1], o[i + 2], o[i + 3]);
                }
            }
        }
        tc_fence_before();
        __syncthreads();  // smem and TMEM free for the next tile
    }
    if (!ok && tid == 0) {
        flag_error(p.err, ERR_TIMEOUT);
        mma_commit(bar);  // let every product in flight finish (bounded)
        mbar_wait(bar, phase);
    }
    if (MODE == MODE_VALUE) cp_async_wait_all();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

// ----------------------------------------------------------- selection

// One warp per (unit, token) at level j >= 1: keeps every candidate when
// there are at most k, else the k best by (score, smaller node id). The
// candidates are in ascending node order, so the smaller id is the smaller
// index. Up to 32 * KPL candidates: the scores sit in registers, the k-th
// largest score is found bit by bit on its order-preserving 32-bit key, and
// the keys equal to it are taken in index order until k are kept. Larger
// lists: packed 64-bit (score, id) keys in shared memory, same search on 64
// bits.
constexpr int SEL_WARPS = 4;
constexpr int SEL_KPL = 32;  // candidates per lane held in registers (1024 per warp)

__device__ __forceinline__ int warp_sum(int n) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
    return n;
}

// The register path of pf_select_kernel for lists of at most 32 * KPL
// candidates: KPL scores per lane; the k-th largest found bit by bit on the
// order-preserving 32-bit keys; keys equal to it taken in index order until
// k are kept. Returns the number kept (k).
template <int KPL>
__device__ __forceinline__ int select_regs(const float* srow, int nc, int k, int lane, const int* par, int b,
                                           int* kept, int* selrow) {
    auto cand_id = [&](int i) { return par[i / b] * b + i % b; };
    int nk = 0;
    unsigned fk[KPL];
#pragma unroll
    for (int x = 0; x < KPL; x++) {
        const int i = x * 32 + lane;
        fk[x] = i < nc ? float_key(srow[i]) : 0u;  // 0: below every real key
    }
    unsigned thr = 0u;
    for (int bit = 31; bit >= 0; bit--) {
        const unsigned c = thr | (1u << bit);
        int n = 0;
#pragma unroll
        for (int x = 0; x < KPL; x++) n += fk[x] >= c;
        if (warp_sum(n) >= k) thr = c;
    }
    int gt = 0;
#pragma unroll
    for (int x = 0; x < KPL; x++) gt += fk[x] > thr;
    int need_eq = k - warp_sum(gt);  // keys equal to the k-th score, smallest indices first
#pragma unroll
    for (int x = 0; x < KPL; x++) {
        const int i = x * 32 + lane;
        const unsigned meq = __ballot_sync(0xffffffffu, i < nc && fk[x] == thr);
        const unsigned take = need_eq <= 0 ? 0u : (__popc(meq) <= need_eq ? meq : [&]() {
            unsigned m = meq, r = 0u;
            for (int c = 0; c < need_eq; c++) {
                const unsigned low = m & (~m + 1u);
                r |= low;
                m ^= low;
            }
            return r;
        }());
        need_eq -= __popc(take);
        const bool in = i < nc && (fk[x] > thr || ((take >> lane) & 1u));
        const unsigned m = __ballot_sync(0xffffffffu, in);
        if (in) {
            const int pos = nk + __popc(m & ((1u << lane) - 1u));
            const int id = cand_id(i);
            kept[pos] = id;
            if (selrow) selrow[pos] = id;
        }
        nk += __popc(m);
    }
    return nk;
}

// Larger lists (more than 128 candidates, k <= 32): a threshold T0 = the
// k-th largest of the 32 lane maxima bounds the k-th largest key from below
// (at least k keys, those maxima, are >= T0), so every key of the result,
// ties included, is >= T0. Those keys are packed in index order into the
// warp's shared buffers (usually a few dozen), and the same bitwise search
// and tie rule as select_regs run over them only. The result is exactly
// select_regs's.
template <int KPL>
__device__ __forceinline__ int select_compact(const float* srow, int nc, int k, int lane, const int* par, int b,
                                              int* kept, int* selrow, unsigned* ckey, int* cidx) {
    auto cand_id = [&](int i) { return par[i / b] * b + i % b; };
    unsigned fk[KPL];
    unsigned lm = 0u;
#pragma unroll
    for (int x = 0; x < KPL; x++) {
        const int i = x * 32 + lane;
        fk[x] = i < nc ? float_key(srow[i]) : 0u;
        lm = fk[x] > lm ? fk[x] : lm;
    }
    // T0: the k-th largest lane maximum (bit by bit over one value per lane)
    unsigned t0 = 0u;
    for (int bit = 31; bit >= 0; bit--) {
        const unsigned c = t0 | (1u << bit);
        if (__popc(__ballot_sync(0xffffffffu, lm >= c)) >= k) t0 = c;
    }
    // the keys >= T0, in index order
    int m = 0;
#pragma unroll
    for (int x = 0; x < KPL; x++) {
        const int i = x * 32 + lane;
        const bool in = i < nc && fk[x] >= t0;
        const unsigned bm = __ballot_sync(0xffffffffu, in);
        if (in) {
            const int pos = m + __popc(bm & ((1u << lane) - 1u));
            ckey[pos] = fk[x];
            cidx[pos] = i;
        }
        m += __popc(bm);
    }
    __syncwarp();
    unsigned thr = 0u;
    for (int bit = 31; bit >= 0; bit--) {
        const unsigned c = thr | (1u << bit);
        int n = 0;
        for (int y = lane; y < m; y += 32) n += ckey[y] >= c;
        if (warp_sum(n) >= k) thr = c;
    }
    int gt = 0;
    for (int y = lane; y < m; y += 32) gt += ckey[y] > thr;
    int need_eq = k - warp_sum(gt);
    int nk = 0;
    for (int y0 = 0; y0 < m; y0 += 32) {
        const int y = y0 + lane;
        const unsigned key = y < m ? ckey[y] : 0u;
        const unsigned meq = __ballot_sync(0xffffffffu, y < m && key == thr);
        const unsigned take = need_eq <= 0 ? 0u : (__popc(meq) <= need_eq ? meq : [&]() {
            unsigned mm = meq, r = 0u;
            for (int c = 0; c < need_eq; c++) {
                const unsigned low = mm & (~mm + 1u);
                r |= low;
                mm ^= low;
            }
            return r;
        }());
        need_eq -= __popc(take);
        const bool in = y < m && (key > thr || ((take >> lane) & 1u));
        const unsigned bm = __ballot_sync(0xffffffffu, in);
        if (in) {
            const int pos = nk + __popc(bm & ((1u << lane) - 1u));
            const int id = cand_id(cidx[y]);
            kept[pos] = id;
            if (selrow) selrow[pos] = id;
        }
        nk += __popc(bm);
    }
    __syncwarp();  // the buffers are free for the warp's next list
    return nk;
}

__global__ void __launch_bounds__(SEL_WARPS * 32) pf_select_kernel(TreeParams p, PfArgs a, PfLevel L, PfLevel up,
                                                                   int j) {
    extern __shared__ unsigned long long skeys[];  // [SEL_WARPS][maxc] when maxc > 32 * SEL_KPL
    __shared__ int sids[SEL_WARPS][TP_KMAX];
    __shared__ unsigned ckey[SEL_WARPS][32 * SEL_KPL];  // select_compact's packed keys and indices
    __shared__ int cidx[SEL_WARPS][32 * SEL_KPL];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long idx = blockIdx.x * (long long)SEL_WARPS + warp;
    const long long U = (long long)p.B * p.H;
    if (idx >= U * a.C) return;
    const long long u = idx / a.C;
    const int t = (int)(idx % a.C);
    const int bseq = (int)(u / p.H), h = (int)(u % p.H);
    const int k = p.k, b = p.b;
    int* selrow = a.sel_out ? a.sel_out + ((((long long)bseq * a.C + t) * p.H + h) * p.J_cap + (j - 1)) * k : nullptr;
    const int nc = L.nc[idx];
    int* kept = L.kept + idx * k;
    if (nc == 0) {
        if (selrow)
            for (int x = lane; x < k; x += 32) selrow[x] = -1;
        if (lane == 0) L.nkept[idx] = 0;
        return;
    }
    const int J = pf_top(p, p.len[u]);
    const int zero = 0;
    int npar;
    const int* par = pf_parents(up, j, J, idx, k, &npar, &zero);
    auto cand_id = [&](int i) { return par[i / b] * b + i % b; };
    if (nc <= k) {
        for (int x = lane; x < k; x += 32) {
            const int id = x < nc ? cand_id(x) : -1;
            if (x < nc) kept[x] = id;
            if (selrow) selrow[x] = id;
        }
        if (lane == 0) L.nkept[idx] = nc;
        return;
    }
    const float* srow = a.S + idx * (long long)a.maxc;
    int nk = 0;  // kept so far (uniform)
    if (nc <= 32 * SEL_KPL) {  // as many registers per lane as the list needs
        const int kpl = (nc + 31) / 32;
        if (kpl <= 4)
            nk = select_regs<4>(srow, nc, k, lane, par, b, kept, selrow);
        else if (k > 32)
            nk = select_regs<SEL_KPL>(srow, nc, k, lane, par, b, kept, selrow);
        else if (kpl <= 8)
            nk = select_compact<8>(srow, nc, k, lane, par, b, kept, selrow, ckey[warp], cidx[warp]);
        else if (kpl <= 16)
            nk = select_compact<16>(srow, nc, k, lane, par, b, kept, selrow, ckey[warp], cidx[warp]);
        else
            nk = select_compact<SEL_KPL>(srow, nc, k, lane, par, b, kept, selrow, ckey[warp], cidx[warp]);
    } else {
        unsigned long long* key = skeys + (long long)warp * a.maxc;
        for (int i = lane; i < nc; i += 32)
            key[i] = ((unsigned long long)float_key(srow[i]) << 32) |
                     (unsigned long long)(0xFFFFFFFFu - (uint32_t)cand_id(i));
        __syncwarp();
        unsigned long long thr = 0ull;
        for (int bit = 63; bit >= 0; bit--) {
            const unsigned long long c = thr | (1ull << bit);
            int n = 0;
            for (int i = lane; i < nc; i += 32) n += key[i] >= c;
            if (warp_sum(n) >= k) thr = c;
        }
        // the k keys >= thr in index order, which is ascending id order
        for (int i0 = 0; i0 < nc; i0 += 32) {
            const int i = i0 + lane;
            const bool in = i < nc && key[i] >= thr;
            const unsigned m = __ballot_sync(0xffffffffu, in);
            if (in) {
                const int pos = nk + __popc(m & ((1u << lane) - 1u));
                if (pos < TP_KMAX) sids[warp][pos] = cand_id(i);
            }
            nk += __popc(m);
        }
        __syncwarp();
        for (int x = lane; x < k; x += 32) {
            kept[x] = sids[warp][x];
            if (selrow) selrow[x] = sids[warp][x];
        }
    }
    if (lane == 0) {
        L.nkept[idx] = k;
        a.rows[idx * 2] += nc;
        a.rows[idx * 2 + 1] += nc - k;
    }
}

// ----------------------------------------------------------------- merge

// out = (tree sums + chunk-local sums), each scaled to the common maximum;
// also the row counts (the chunk's own t + 1 tokens are entries too) and
// the selection rows of levels above every unit's top.
template <int D>
__global__ void pf_final_kernel(TreeParams p, PfArgs a, const float* state, __nv_bfloat16* out, long long* rows_out,
                                int J_top) {
    const long long n = (long long)p.B * a.C * a.Hq * (D / 4);
    const int G = a.Hq / p.H;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
        const long long row = i / (D / 4);  // (sequence, token, query head)
        const int c = (int)(i % (D / 4)) * 4;
        const float* st = state + row * (D + 2);
        const float ml = st[D], ll = st[D + 1];
        const unsigned key = a.mkey[row];
        const float mt = key ? key_float(key) : -INFINITY;
        const float M = fmaxf(ml, mt);
        const float ft = mt == -INFINITY ? 0.f : expf(mt - M);
        const float fl = ml == -INFINITY ? 0.f : expf(ml - M);
        const float den = a.lacc[row] * ft + ll * fl;
        const float4 oa = *reinterpret_cast<const float4*>(a.oacc + row * D + c);
        const float2 ol01 = *reinterpret_cast<const float2*>(st + c);  // state rows: d + 2 floats, 8-byte aligned
        const float2 ol23 = *reinterpret_cast<const float2*>(st + c + 2);
        const float4 ol = make_float4(ol01.x, ol01.y, ol23.x, ol23.y);
        const float inv = 1.f / den;
        __nv_bfloat162 lo = __floats2bfloat162_rn((oa.x * ft + ol.x * fl) * inv, (oa.y * ft + ol.y * fl) * inv);
        __nv_bfloat162 hi = __floats2bfloat162_rn((oa.z * ft + ol.z * fl) * inv, (oa.w * ft + ol.w * fl) * inv);
        __nv_bfloat16* o = out + row * D + c;
        *reinterpret_cast<__nv_bfloat162*>(o) = lo;
        *reinterpret_cast<__nv_bfloat162*>(o + 2) = hi;
        const int hq = (int)(row % a.Hq);
        if (c == 0 && hq % G == 0) {  // once per (sequence, token, KV head)
            const long long bt = row / a.Hq;  // sequence * C + token
            const int bseq = (int)(bt / a.C), t = (int)(bt % a.C), h = hq / G;
            const long long ut = ((long long)bseq * p.H + h) * a.C + t;
            if (rows_out) {
                rows_out[(bt * p.H + h) * 2] = a.rows[ut * 2];
                rows_out[(bt * p.H + h) * 2 + 1] = a.rows[ut * 2 + 1] + t + 1;
            }
            if (a.sel_out)
                for (int x = J_top * p.k; x < p.J_cap * p.k; x++) a.sel_out[(bt * p.H + h) * p.J_cap * p.k + x] = -1;
        }
    }
}

// ------------------------------------------------------------------ host

// Scratch of the tree part for chunks of C tokens (bytes; layout computed
// the same way by pf_layout).
struct PfScratch {
    size_t S, mkey, oacc, lacc, rows;
    size_t kept[MAXJ + 1], nkept[MAXJ + 1], nc[MAXJ + 1], cnt[MAXJ + 1], off[MAXJ + 1], toff[MAXJ + 1],
        cursor[MAXJ + 1], pairs[MAXJ + 1], tiles[MAXJ + 1], ntiles[MAXJ + 1];
    int R[MAXJ + 1], max_tiles[MAXJ + 1];
    size_t total;
};

static size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

PfScratch pf_layout(const TreeParams& p, int C, int Hq) {
    // uses p.B, p.H, p.D, p.b, p.k, p.J_cap and p.rows only
    PfScratch s{};
    const size_t U = (size_t)p.B * p.H, UC = U * C;
    const int G = Hq / p.H, TP = 128 / G;
    const int maxc = p.k * p.b > p.b ? p.k * p.b : p.b;
    size_t o = 0;
    s.S = o;
    o = al256(o + UC * maxc * 4);
    s.mkey = o;
    o = al256(o + (size_t)p.B * C * Hq * 4);
    s.oacc = o;
    o = al256(o + (size_t)p.B * C * Hq * p.D * 4);
    s.lacc = o;
    o = al256(o + (size_t)p.B * C * Hq * 4);
    s.rows = o;
    o = al256(o + UC * 16);
    for (int j = 0; j <= p.J_cap; j++) {
        const long long R = j + 1 <= p.J_cap ? p.rows[j + 1] : 1;
        s.R[j] = (int)R;
        const long long pairs = (long long)UC * p.k;
        const long long nonempty = std::min<long long>(R, (long long)C * p.k);
        s.max_tiles[j] = (int)((long long)U * (((long long)C * p.k + TP - 1) / TP + nonempty));
        s.kept[j] = o;
        o = al256(o + UC * p.k * 4);
        s.nkept[j] = o;
        o = al256(o + UC * 4);
        s.nc[j] = o;
        o = al256(o + UC * 4);
        s.cnt[j] = o;
        o = al256(o + U * R * 4);
        s.off[j] = o;
        o = al256(o + U * R * 4);
        s.toff[j] = o;
        o = al256(o + U * R * 4);
        s.cursor[j] = o;
        o = al256(o + U * R * 4);
        s.pairs[j] = o;
        o = al256(o + (size_t)pairs * 4);
        s.tiles[j] = o;
        o = al256(o + (size_t)s.max_tiles[j] * 16);
        s.ntiles[j] = o;
        o = al256(o + 4);
    }
    s.total = o;
    return s;
}

size_t prefill_tree_scratch_bytes(const TreeParams& p, int C, int Hq) { return pf_layout(p, C, Hq).total; }

// The tile kernel's limits: b rounded up to 32, 64 or 128 must fit the
// weights tile (at most d columns) and 128 TMEM columns.
bool prefill_tree_supported(int D, int b) { return b <= 64 || (D >= 128 && b <= 128); }

static PfLevel pf_level(const PfScratch& s, char* base, int j) {
    PfLevel L{};
    L.kept = reinterpret_cast<int*>(base + s.kept[j]);
    L.nkept = reinterpret_cast<int*>(base + s.nkept[j]);
    L.nc = reinterpret_cast<int*>(base + s.nc[j]);
    L.cnt = reinterpret_cast<int*>(base + s.cnt[j]);
    L.off = reinterpret_cast<int*>(base + s.off[j]);
    L.toff = reinterpret_cast<int*>(base + s.toff[j]);
    L.cursor = reinterpret_cast<int*>(base + s.cursor[j]);
    L.pairs = reinterpret_cast<int*>(base + s.pairs[j]);
    L.tiles = reinterpret_cast<int4*>(base + s.tiles[j]);
    L.ntiles = reinterpret_cast<int*>(base + s.ntiles[j]);
    L.R = s.R[j];
    L.max_tiles = s.max_tiles[j];
    return L;
}

template <int D, int NB, int MODE>
static cudaError_t launch_tiles_nb(const TreeParams& p, const PfArgs& a, const PfLevel& L, int j, int G,
                                   cudaStream_t s) {
    auto kern = pf_tile_kernel<D, NB, MODE>;
    const int smem = (int)TpLayout<D>::bytes(NB);
    static std::atomic<unsigned long long> attr_done{0};
    cudaError_t e = set_smem_limit(kern, smem, attr_done);
    if (e != cudaSuccess) return e;
    const int grid = std::min(2 * 148, std::max(1, L.max_tiles));  // two CTAs per SM (2 x 256 TMEM columns)
    kern<<<grid, TP_THREADS, smem, s>>>(p, a, L, j, G);
    return cudaGetLastError();
}
template <int D, int MODE>
static cudaError_t launch_tiles(const TreeParams& p, const PfArgs& a, const PfLevel& L, int j, int G, cudaStream_t s) {
    if (p.b <= 32) return launch_tiles_nb<D, 32, MODE>(p, a, L, j, G, s);
    if (p.b <= 64) return launch_tiles_nb<D, 64, MODE>(p, a, L, j, G, s);
    if (D >= 128 && p.b <= 128) return launch_tiles_nb<D, (D >= 128 ? 128 : 64), MODE>(p, a, L, j, G, s);
    return cudaErrorInvalidValue;
}

// The tree part of a prefill chunk: q [B][C][Hq][D] (bf16), the chunk-local
// state [B][C][Hq][D + 2], out [B][C][Hq][D]. lengths: the host's copy of
// every sequence's cached length (the tree each chunk descends).
template <int D, int G>
cudaError_t launch_prefill_tree_tc(const TreeParams& p, const void* q, void* out, const float* state, int* sel_out,
                                   long long* rows_out, int C, int Hq, const long long* lengths, void* scratch,
                                   cudaStream_t s) {
    const PfScratch sc = pf_layout(p, C, Hq);
    char* base = static_cast<char*>(scratch);
    const long long U = (long long)p.B * p.H;
    PfArgs a{};
    a.q = reinterpret_cast<const __nv_bfloat16*>(q);
    a.C = C;
    a.Hq = Hq;
    a.TP = 128 / G;
    a.S = reinterpret_cast<float*>(base + sc.S);
    a.maxc = p.k * p.b > p.b ? p.k * p.b : p.b;
    a.mkey = reinterpret_cast<unsigned*>(base + sc.mkey);
    a.oacc = reinterpret_cast<float*>(base + sc.oacc);
    a.lacc = reinterpret_cast<float*>(base + sc.lacc);
    a.rows = reinterpret_cast<long long*>(base + sc.rows);
    a.sel_out = sel_out;
    cudaError_t e = cudaMemsetAsync(a.mkey, 0, (size_t)p.B * C * Hq * 4, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(a.oacc, 0, (size_t)p.B * C * Hq * D * 4, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(a.lacc, 0, (size_t)p.B * C * Hq * 4, s);
    if (e == cudaSuccess) e = cudaMemsetAsync(a.rows, 0, (size_t)U * C * 16, s);
    if (e != cudaSuccess) return e;
    // the highest top level over the sequences that hold a tree
    int J_top = 0;
    for (int bq = 0; bq < p.B; bq++) {
        if (lengths[bq] <= 0) continue;
        int J = 1;
        while (J < p.J_cap && (lengths[bq] + p.span[J] - 1) / p.span[J] > p.b) J++;
        J_top = std::max(J_top, J);
    }
    const int thr = 256;
    const unsigned gUC = (unsigned)((U * C + thr - 1) / thr);
    if (J_top > 0) {
        for (int j = J_top; j >= 0; j--) {
            PfLevel L = pf_level(sc, base, j);
            PfLevel up = pf_level(sc, base, j + 1 <= p.J_cap ? j + 1 : j);
            const int nR = (int)(U * L.R);
            e = cudaMemsetAsync(L.cnt, 0, (size_t)nR * 4, s);
            if (e != cudaSuccess) return e;
            pf_cand_kernel<<<gUC, thr, 0, s>>>(p, a, L, up, j);
            pf_scan_kernel<<<1, 1024, 0, s>>>(L, nR, a.TP, p.err);
            pf_scatter_kernel<<<gUC, thr, 0, s>>>(p, a, L, up, j);
            pf_tiles_kernel<<<(nR + thr - 1) / thr, thr, 0, s>>>(L, nR, a.TP);
            e = cudaGetLastError();
            if (e != cudaSuccess) return e;
            if (j > 0) {
                e = launch_tiles<D, MODE_SCORE>(p, a, L, j, G, s);
                if (e != cudaSuccess) return e;
                const size_t smem = a.maxc > 32 * SEL_KPL ? (size_t)SEL_WARPS * a.maxc * 8 : 0;
                static std::atomic<unsigned long long> sel_attr{0};
                // room for k * b <= 4096 keys per warp; the kernel also has
                // static shared memory, and both together must fit 227 KB
                e = set_smem_limit(pf_select_kernel, SEL_WARPS * 4096 * 8, sel_attr);
                if (e != cudaSuccess) return e;
                pf_select_kernel<<<(unsigned)((U * C + SEL_WARPS - 1) / SEL_WARPS), SEL_WARPS * 32, smem, s>>>(
                    p, a, L, up, j);
            } else {
                e = launch_tiles<D, MODE_MAX>(p, a, L, j, G, s);
            }
            if (e == cudaSuccess) e = cudaGetLastError();
            if (e != cudaSuccess) return e;
        }
        for (int j = J_top; j >= 0; j--) {
            e = launch_tiles<D, MODE_VALUE>(p, a, pf_level(sc, base, j), j, G, s);
            if (e != cudaSuccess) return e;
        }
    }
    const long long n = (long long)p.B * C * Hq * (D / 4);
    pf_final_kernel<D><<<(unsigned)std::min<long long>((n + 255) / 256, 148 * 16), 256, 0, s>>>(
        p, a, state, reinterpret_cast<__nv_bfloat16*>(out), rows_out, J_top);
    return cudaGetLastError();
}

#define RECSA_INST_PTC(D, G)                                                                                    \
    template cudaError_t launch_prefill_tree_tc<D, G>(const TreeParams&, const void*, void*, const float*, int*, \
                                                      long long*, int, int, const long long*, void*, cudaStream_t);
RECSA_INST_PTC(64, 1)
RECSA_INST_PTC(64, 2)
RECSA_INST_PTC(64, 4)
RECSA_INST_PTC(64, 8)
RECSA_INST_PTC(128, 1)
RECSA_INST_PTC(128, 2)
RECSA_INST_PTC(128, 4)
RECSA_INST_PTC(128, 8)

}  // namespace recsa
