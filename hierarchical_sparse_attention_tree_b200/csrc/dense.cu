// Dense GQA flash-decode: the comparator for RecSA's speed claim (the RecSA
// abstract reports end-to-end speedups over dense attention at 524K tokens).
// Not part of the method. One query per sequence attends every cached token;
// keys are used as stored (a dense cache holds keys already rotated).
//
// Split-KV: CTA (s, u) streams tokens [s*chunk, (s+1)*chunk) of unit u with
// 16-byte loads, keeps an online softmax per row group, and writes a partial
// (max, sum, acc) that a second kernel merges.
#include <mutex>

#include "common.cuh"

namespace recsa {

constexpr int DN_THREADS = 256;

template <typename T, int D, int G>
__global__ void __launch_bounds__(DN_THREADS) dense_partial_kernel(const T* __restrict__ K, const T* __restrict__ V,
                                                                   const T* __restrict__ q, float* __restrict__ part,
                                                                   long long L, long long ld, int splits,
                                                                   float scale) {
    constexpr int EPL = 16 / sizeof(T);       // elements per lane per row
    constexpr int LPR = D / EPL;              // lanes per row
    constexpr int RPW = 32 / LPR;             // rows per warp step
    constexpr int NG = DN_THREADS / LPR;      // row groups per CTA
    constexpr int U = 4;
    const int tid = threadIdx.x;
    const int grp = tid / LPR, gl = tid % LPR;
    const long long u = blockIdx.y;
    const int s = blockIdx.x;
    const long long chunk = (L + splits - 1) / splits;
    const long long t0 = s * chunk, t1 = min(L, t0 + chunk);

    float qv[G][EPL];
#pragma unroll
    for (int g = 0; g < G; g++) load_vec<T, EPL>(q + (u * G + g) * D + gl * EPL, qv[g]);
    float m_[G], l_[G], acc[G][EPL];
#pragma unroll
    for (int g = 0; g < G; g++) {
        m_[g] = -INFINITY; l_[g] = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; e++) acc[g][e] = 0.f;
    }
    const T* Ku = K + u * ld * D + gl * EPL;
    const T* Vu = V + u * ld * D + gl * EPL;
    // Warp-uniform loop: every lane of a warp runs the same iterations (the
    // shuffles below need all 32 lanes); rows past t1 are masked, not skipped.
    constexpr int NW = DN_THREADS / 32;
    const int warp = tid >> 5, gi = (tid & 31) / LPR;
    for (long long base = t0 + (long long)warp * RPW; base < t1; base += (long long)NW * RPW * U) {
        float kr[U][EPL] = {}, vr[U][EPL] = {};
#pragma unroll
        for (int i = 0; i < U; i++) {
            const long long t = base + gi + (long long)i * NW * RPW;
            if (t < t1) {
                load_vec<T, EPL>(Ku + t * D, kr[i]);
                load_vec<T, EPL>(Vu + t * D, vr[i]);
            }
        }
#pragma unroll
        for (int i = 0; i < U; i++) {
            const long long t = base + gi + (long long)i * NW * RPW;
            float lg[G];
#pragma unroll
            for (int g = 0; g < G; g++) {
                float d = 0.f;
#pragma unroll
                for (int e = 0; e < EPL; e++) d = fmaf(qv[g][e], kr[i][e], d);
#pragma unroll
                for (int o = LPR / 2; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
                lg[g] = d * scale;
            }
            if (t < t1) {
#pragma unroll
                for (int g = 0; g < G; g++) {
                    const float mn = fmaxf(m_[g], lg[g]);
                    const float sa = expf(m_[g] - mn), w = expf(lg[g] - mn);
                    l_[g] = l_[g] * sa + w;
#pragma unroll
                    for (int e = 0; e < EPL; e++) acc[g][e] = acc[g][e] * sa + w * vr[i][e];
                    m_[g] = mn;
                }
            }
        }
    }
    // merge the NG row groups of this CTA, one head at a time
    __shared__ float sm[NG][G], sl[NG][G];
    __shared__ float sacc[NG][D];
    if (gl == 0)
#pragma unroll
        for (int g = 0; g < G; g++) { sm[grp][g] = m_[g]; sl[grp][g] = l_[g]; }
    float* out = part + ((u * splits + s) * G) * (D + 2);
#pragma unroll
    for (int g = 0; g < G; g++) {
#pragma unroll
        for (int e = 0; e < EPL; e++) sacc[grp][gl * EPL + e] = acc[g][e];
        __syncthreads();
        for (int e = tid; e < D; e += DN_THREADS) {
            float M = -INFINITY;
            for (int r = 0; r < NG; r++) M = fmaxf(M, sm[r][g]);
            float a = 0.f, lsum = 0.f;
            for (int r = 0; r < NG; r++) {
                const float f = sm[r][g] == -INFINITY ? 0.f : expf(sm[r][g] - M);
                a += sacc[r][e] * f;
                lsum += sl[r][g] * f;
            }
            out[g * (D + 2) + e] = a;
            if (e == 0) { out[g * (D + 2) + D] = M; out[g * (D + 2) + D + 1] = lsum; }
        }
        __syncthreads();
    }
}

template <typename T, int D, int G>
__global__ void dense_combine_kernel(const float* __restrict__ part, T* __restrict__ out, int splits) {
    const long long u = blockIdx.x;
    for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
        const int g = idx / D, e = idx % D;
        float M = -INFINITY;
        for (int s = 0; s < splits; s++) M = fmaxf(M, part[((u * splits + s) * G + g) * (D + 2) + D]);
        float a = 0.f, lsum = 0.f;
        for (int s = 0; s < splits; s++) {
            const float* ps = part + ((u * splits + s) * G + g) * (D + 2);
            const float f = ps[D] == -INFINITY ? 0.f : expf(ps[D] - M);
            a += ps[e] * f;
            lsum += ps[D + 1] * f;
        }
        out[(u * G + g) * D + e] = from_f<T>(a / lsum);
    }
}

constexpr int DN_MAX_SPLITS = 256;

int dense_splits(long long units, long long L) {
    long long s = (4LL * 148 + units - 1) / units;
    if (s > DN_MAX_SPLITS) s = DN_MAX_SPLITS;
    long long by_len = (L + 255) / 256;
    if (s > by_len) s = by_len;
    return (int)(s < 1 ? 1 : s);
}

// Fixed-size device scratch for recsa_dense_decode_static: 8 MiB, held by
// every device that loads the library until the process exits. Host code
// must not pass the symbol itself to a kernel (on the host it names a
// stand-in, not device memory); dense_static_scratch() looks up its device
// address once per device.
constexpr size_t DN_STATIC_BYTES = size_t(8) << 20;
static __device__ __align__(256) float g_dense_static_scratch[DN_STATIC_BYTES / sizeof(float)];

size_t dense_static_scratch_bytes() { return DN_STATIC_BYTES; }

cudaError_t dense_static_scratch(float** out) {
    static std::mutex mu;
    static void* addr[256] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 256) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_dense_static_scratch);  // with `dev` current
        if (e != cudaSuccess) return e;
        addr[dev] = p;
    }
    *out = static_cast<float*>(addr[dev]);
    return cudaSuccess;
}

// max_splits bounds the split count so the partials fit the scratch given.
template <typename T, int D, int G>
cudaError_t launch_dense(const void* K, const void* V, const void* q, void* out, int units, long long L, long long ld,
                         float* scratch, int max_splits, cudaStream_t st) {
    int splits = dense_splits(units, L);
    if (splits > max_splits) splits = max_splits;
    if (splits < 1) return cudaErrorInvalidValue;
    dim3 grid(splits, units);
    dense_partial_kernel<T, D, G><<<grid, DN_THREADS, 0, st>>>(
        reinterpret_cast<const T*>(K), reinterpret_cast<const T*>(V), reinterpret_cast<const T*>(q), scratch, L, ld,
        splits, 1.0f / sqrtf((float)D));
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    dense_combine_kernel<T, D, G><<<units, 256, 0, st>>>(scratch, reinterpret_cast<T*>(out), splits);
    return cudaGetLastError();
}

#define RECSA_INST_DN(T, D, G)                                                                                   \
    template cudaError_t launch_dense<T, D, G>(const void*, const void*, const void*, void*, int, long long,     \
                                               long long, float*, int, cudaStream_t);
#define RECSA_INST_DN_G(T, D) RECSA_INST_DN(T, D, 1) RECSA_INST_DN(T, D, 2) RECSA_INST_DN(T, D, 4) RECSA_INST_DN(T, D, 8)
RECSA_INST_DN_G(float, 64)
RECSA_INST_DN_G(float, 128)
RECSA_INST_DN_G(__nv_bfloat16, 64)
RECSA_INST_DN_G(__nv_bfloat16, 128)

}  // namespace recsa
