// The pieces of one distillation step of the pooler that are not the
// forward, the gradient or the tree build: the squared-error loss against
// dense-attention outputs with its gradient, and the plain gradient-descent
// update of the pooler (RecSA abstract: the pooler is trained so that the
// tree's attention follows dense attention).
#include <algorithm>

#include "common.cuh"

namespace recsa {

constexpr int DS_THREADS = 256;

// loss += sum_i (out_i - target_i)^2 / n;  dout_i = 2 (out_i - target_i) / n.
__global__ void __launch_bounds__(DS_THREADS) distill_loss_kernel(const float* __restrict__ out,
                                                                  const float* __restrict__ target,
                                                                  float* __restrict__ dout, float* loss, long long n) {
    __shared__ float red[DS_THREADS / 32];
    const float inv = 1.f / (float)n;
    float s = 0.f;
    for (long long i = (long long)blockIdx.x * DS_THREADS + threadIdx.x; i < n; i += (long long)gridDim.x * DS_THREADS) {
        const float d = out[i] - target[i];
        dout[i] = 2.f * d * inv;
        s += d * d;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        float t = 0.f;
        for (int w = 0; w < DS_THREADS / 32; w++) t += red[w];
        atomicAdd(loss, t * inv);
    }
}

// w <- w - lr dw (fp32 master copy, row-major [D][D]); the context's pooler
// (transposed, storage type) refreshed from it; dw copied out if asked.
template <typename T>
__global__ void __launch_bounds__(DS_THREADS) pooler_update_kernel(float* w, const float* __restrict__ dw, float lr,
                                                                   T* wt, float* dw_out, int D) {
    const int i = blockIdx.x * DS_THREADS + threadIdx.x;
    if (i >= D * D) return;
    const int r = i / D, c = i % D;
    const float g = dw[i];
    const float x = w[i] - lr * g;
    w[i] = x;
    wt[c * D + r] = from_f<T>(x);
    if (dw_out) dw_out[i] = g;
}

cudaError_t launch_distill_loss(const float* out, const float* target, float* dout, float* loss, long long n,
                                cudaStream_t s) {
    const long long blocks = std::min<long long>((n + DS_THREADS - 1) / DS_THREADS, 4 * 148);
    distill_loss_kernel<<<(unsigned)std::max<long long>(1, blocks), DS_THREADS, 0, s>>>(out, target, dout, loss, n);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_pooler_update(float* w, const float* dw, float lr, void* wt, float* dw_out, int D,
                                 cudaStream_t s) {
    pooler_update_kernel<T><<<(D * D + DS_THREADS - 1) / DS_THREADS, DS_THREADS, 0, s>>>(
        w, dw, lr, reinterpret_cast<T*>(wt), dw_out, D);
    return cudaGetLastError();
}

template cudaError_t launch_pooler_update<float>(float*, const float*, float, void*, float*, int, cudaStream_t);
template cudaError_t launch_pooler_update<__nv_bfloat16>(float*, const float*, float, void*, float*, int,
                                                         cudaStream_t);

}  // namespace recsa
