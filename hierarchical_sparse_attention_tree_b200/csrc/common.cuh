// Device-side types and helpers shared by the RecSA kernels (sm_100a).
//
// Method: "Recursive Sparse Attention: Million-Token Length Extrapolation at
// Logarithmic Cost" (arXiv 2611.07232), abstract; kongchang.com RecSA
// article, "Core Idea" and "Position Encoding".
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace recsa {

constexpr int MAXJ = 32;  // levels kept above the tokens (b >= 2, capacity < 2^32)

// Device error word bits.
enum : int { ERR_LENGTH = 1, ERR_SHAPE = 2, ERR_TIMEOUT = 4 };

// Everything a kernel needs to address the tree of every (sequence, KV head)
// unit. Level 0 is the caller's cache; levels 1..J_cap live in the workspace.
// Unit u = b * H + h owns rows [u * rows[j], (u + 1) * rows[j]) of level j.
struct TreeParams {
    int B, H, G, D, b, k, J_cap, npos;
    long long cap;
    long long rows[MAXJ + 1];  // node rows per unit at each level (rows[0] = cap)
    long long span[MAXJ + 1];  // tokens under one node: b^j (saturating)
    void* K[MAXJ + 1];         // keys   [B*H][rows[j]][D], storage type
    void* V[MAXJ + 1];         // values [B*H][rows[j]][D], storage type
    float* VS[MAXJ + 1];       // fp32 value sums [B*H][rows[j]][D] (j >= 1)
    float* PK[MAXJ + 1];       // right-edge key prefix sums [B*H][D] (j >= 1)
    float* PV[MAXJ + 1];       // right-edge value prefix sums [B*H][D] (j >= 1)
    const void* Wt;            // pooler, transposed, storage type: Wt[c * D + r] = W[r][c]
    const float* rope;         // [npos][3][D/2]: cos, sin, -sin of (p * theta_i), theta_i = base^(-2i/d)
    const int* pages;          // paged token cache: [B][max_pages] pool page of each page of tokens (null: contiguous)
    int page_size, max_pages;  // tokens per page (a multiple of b), pages per sequence
    long long num_pages;       // pages in the pool
    long long* len;            // [B*H] tokens held by each unit
    long long* stats;          // [B*H][3] last decode: depth, K rows read, V rows read
    int* err;                  // device error word
    float scale;               // 1 / sqrt(D)
};

// Where the token rows live. Contiguous: unit u's rows at base + (u * cap + t) * D.
// Paged: a pool [pages][H][page_size][D]; token t of unit u = (sequence
// u / H, KV head u % H) is row t % page_size of page pages[seq * max_pages +
// t / page_size]. Rows t .. t + n - 1 are contiguous while they stay in one
// page (a node's children always do: the page size is a multiple of b).
struct TokenMap {
    const int* pages;
    int page_size, max_pages, H;
    long long cap, num_pages;
    int* err;
};
// A page id outside the pool is reported in the error word (shape bit) and
// replaced by page 0, so that no access leaves the pool.
__device__ __forceinline__ long long token_row(const TokenMap& m, long long u, long long t) {
    if (!m.pages) return u * m.cap + t;
    long long pg = m.pages[(u / m.H) * m.max_pages + t / m.page_size];
    if (pg < 0 || pg >= m.num_pages) {
        atomicOr(m.err, 2);
        pg = 0;
    }
    return (pg * m.H + u % m.H) * m.page_size + t % m.page_size;
}
__device__ __forceinline__ TokenMap token_map(const TreeParams& p) {
    return TokenMap{p.pages, p.page_size, p.max_pages, p.H, p.cap, p.num_pages, p.err};
}

// One level's addresses and sizes together. Kernels that index the levels
// with a runtime j copy these into shared memory once: kernel parameters
// indexed at run time are constant-cache reads, one line per array, each a
// miss the first time it is touched.
struct LevelRef {
    void* K;
    void* V;
    float* VS;
    float* PK;
    float* PV;
    long long rows;
    long long span;
};

// Threads 0..J_cap each copy one level.
__device__ __forceinline__ void load_levels(const TreeParams& p, LevelRef* lv, int tid) {
    if (tid <= p.J_cap) {
        LevelRef r;
        r.K = p.K[tid];
        r.V = p.V[tid];
        r.VS = p.VS[tid];
        r.PK = p.PK[tid];
        r.PV = p.PV[tid];
        r.rows = p.rows[tid];
        r.span = p.span[tid];
        lv[tid] = r;
    }
}

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Loads N consecutive elements (N * sizeof(T) bytes, naturally aligned) as floats.
template <typename T, int N>
__device__ __forceinline__ void load_vec(const T* p, float* out);

template <>
__device__ __forceinline__ void load_vec<float, 2>(const float* p, float* o) {
    float2 v = *reinterpret_cast<const float2*>(p);
    o[0] = v.x; o[1] = v.y;
}
template <>
__device__ __forceinline__ void load_vec<float, 4>(const float* p, float* o) {
    float4 v = *reinterpret_cast<const float4*>(p);
    o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
}
template <>
__device__ __forceinline__ void load_vec<__nv_bfloat16, 2>(const __nv_bfloat16* p, float* o) {
    __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(p);
    o[0] = __low2float(v); o[1] = __high2float(v);
}
template <>
__device__ __forceinline__ void load_vec<__nv_bfloat16, 4>(const __nv_bfloat16* p, float* o) {
    uint2 u = *reinterpret_cast<const uint2*>(p);
    __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&u.x);
    __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&u.y);
    o[0] = __low2float(a); o[1] = __high2float(a); o[2] = __low2float(b); o[3] = __high2float(b);
}
template <>
__device__ __forceinline__ void load_vec<__nv_bfloat16, 8>(const __nv_bfloat16* p, float* o) {
    uint4 u = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; i++) { o[2 * i] = __low2float(h[i]); o[2 * i + 1] = __high2float(h[i]); }
}
template <>
__device__ __forceinline__ void load_vec<float, 8>(const float* p, float* o) {
    load_vec<float, 4>(p, o);
    load_vec<float, 4>(p + 4, o + 4);
}

template <typename T, int N>
__device__ __forceinline__ void store_vec(T* p, const float* v) {
#pragma unroll
    for (int i = 0; i < N; i++) p[i] = from_f<T>(v[i]);
}

// Order-preserving map of a float to uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t float_key(float f) {
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
// Selection key: higher score first, then the smaller node id.
__device__ __forceinline__ unsigned long long sel_key(float S, long long id) {
    return ((unsigned long long)float_key(S) << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)id);
}
__device__ __forceinline__ long long key_id(unsigned long long key) {
    return (long long)(0xFFFFFFFFu - (uint32_t)(key & 0xFFFFFFFFull));
}

__device__ __forceinline__ long long ceil_div_ll(long long a, long long b) { return (a + b - 1) / b; }

// Number of nodes of level j over L tokens.
__device__ __forceinline__ long long level_rows(const TreeParams& p, int j, long long L) {
    return j == 0 ? L : ceil_div_ll(L, p.span[j]);
}

__device__ __forceinline__ void flag_error(int* err, int bits) { atomicOr(err, bits); }

// Raises a kernel's dynamic shared memory limit on the current device, once
// per device and kernel (the attribute is per device; `done` is a bit mask
// of devices 0..63, higher devices set it on every call).
template <typename F>
inline cudaError_t set_smem_limit(F kern, int bytes, std::atomic<unsigned long long>& done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = dev < 64 ? (1ull << dev) : 0ull;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
    return e;
}

}  // namespace recsa

// ---------------------------------------------------------------------
// mbarrier + 1D bulk async copy (global -> this CTA's shared memory).
// PTX ISA: mbarrier.*, cp.async.bulk.shared::cluster.global.mbarrier::
// complete_tx::bytes. Addresses 16-byte aligned, sizes multiples of 16.

namespace recsa {

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Arrive once and add `bytes` to the transaction count of the current phase.
// Relaxed: the barrier only counts the copy's bytes; it orders none of this
// thread's earlier memory operations (so it does not wait for them).
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.relaxed.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Waits for phase `parity` of `bar` to complete, for at most ~2^31 clock
// cycles (about a second). Returns false on timeout (the caller flags an
// error and carries on without using the data; it never exits early, so
// cluster barriers stay balanced).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > (1LL << 31)) return false;
    }
    return true;
}

__device__ __forceinline__ void bulk_g2s(void* dst_smem, const void* src_gmem, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst_smem)),
        "l"(src_gmem), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

}  // namespace recsa

namespace recsa {

// Orders this thread's earlier generic-proxy accesses to shared memory before
// later async-proxy (bulk copy) writes to it.
__device__ __forceinline__ void fence_proxy_async_shared() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// Orders this thread's generic-proxy global accesses with async-proxy ones.
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

}  // namespace recsa

namespace recsa {

// Packed fp32 arithmetic (two independent IEEE fp32 operations per
// instruction, round to nearest even): same results as two fmaf / fmul.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;"
        : "=l"(*reinterpret_cast<unsigned long long*>(&d))
        : "l"(*reinterpret_cast<unsigned long long*>(&a)), "l"(*reinterpret_cast<unsigned long long*>(&b)),
          "l"(*reinterpret_cast<unsigned long long*>(&c)));
    return d;
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
    float2 d;
    asm("mul.rn.f32x2 %0, %1, %2;"
        : "=l"(*reinterpret_cast<unsigned long long*>(&d))
        : "l"(*reinterpret_cast<unsigned long long*>(&a)), "l"(*reinterpret_cast<unsigned long long*>(&b)));
    return d;
}

// N consecutive floats of a RoPE table block (N = 2: one 8-byte load; N a
// multiple of 4: 16-byte loads), as float2 pairs.
template <int N>
__device__ __forceinline__ void load_tab2(const float* p, float2* out) {
    static_assert(N == 2 || N % 4 == 0, "table load width");
    if constexpr (N == 2) {
        out[0] = __ldg(reinterpret_cast<const float2*>(p));
    } else {
#pragma unroll
        for (int x = 0; x < N / 4; x++) {
            const float4 v = __ldg(reinterpret_cast<const float4*>(p) + x);
            out[2 * x] = make_float2(v.x, v.y);
            out[2 * x + 1] = make_float2(v.z, v.w);
        }
    }
}

// N consecutive elements of a row as float2 pairs (N = 2, 4 or 8).
template <typename T, int N>
__device__ __forceinline__ void load_row2(const T* row, float2* out) {
    float f[N];
    load_vec<T, N>(row, f);
#pragma unroll
    for (int x = 0; x < N / 2; x++) out[x] = make_float2(f[2 * x], f[2 * x + 1]);
}

}  // namespace recsa
