// Device-side types and helpers shared by the RecSA kernels (sm_100a).
//
// Method: "Recursive Sparse Attention: Million-Token Length Extrapolation at
// Logarithmic Cost" (arXiv 2611.07232), abstract; kongchang.com RecSA
// article, "Core Idea" and "Position Encoding".
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

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
    const float* Wt;           // pooler, transposed: Wt[c * D + r] = W[r][c]
    const float2* rope;        // [npos][D/2] = (cos, sin)(p * theta_i)
    long long* len;            // [B*H] tokens held by each unit
    int* err;                  // device error word
    float scale;               // 1 / sqrt(D)
};

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

__device__ __forceinline__ unsigned long long shfl_xor_u64(unsigned long long v, int m) {
    return __shfl_xor_sync(0xffffffffu, v, m);
}

__device__ __forceinline__ long long ceil_div_ll(long long a, long long b) { return (a + b - 1) / b; }

// Number of nodes of level j over L tokens.
__device__ __forceinline__ long long level_rows(const TreeParams& p, int j, long long L) {
    return j == 0 ? L : ceil_div_ll(L, p.span[j]);
}

// Top level J over L >= 1 tokens: the first level with at most b nodes.
__device__ __forceinline__ int top_level(const TreeParams& p, long long L) {
    int j = 1;
    while (j < p.J_cap && level_rows(p, j, L) > p.b) j++;
    return j;
}

__device__ __forceinline__ void flag_error(int* err, int bits) { atomicOr(err, bits); }

}  // namespace recsa
