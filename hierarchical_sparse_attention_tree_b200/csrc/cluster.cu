// LSA-style clustered token order: the "Latent Sparse Attention" abstract
// clusters the keys hierarchically in a learned latent space and lets the
// queries score the hierarchy of clusters. Read with the tree's own fan-out
// b: level j has one learned direction Z_j and the latent coordinate
// z_j(t) = <Z_j, k_t>; from the top level down, the tokens of every block of
// b^(j+1) consecutive positions of the current order are sorted by
// (z_j, token index), so that the level-j nodes of the tree over the
// reordered tokens are blocks of b^j positions whose z_j ranges follow one
// another inside their parent. The tree, the descent and the attention over
// the reordered cache are the method's own kernels (a RoPE index is a
// position among candidates: the tokens' original order does not enter).
//
// The order is one bitonic sort per level over every unit's tokens at once:
// records (unit | block, order key of z, token) in one array padded to a
// power of two; stages with partner distance below CL_TILE run in shared
// memory, the longer distances two per global pass. z is summed in fp64 in
// index order with separately rounded products (the decision of an integer
// order taken in one stated precision).
#include <climits>

#include "common.cuh"

namespace recsa {

struct ClRec {
    unsigned long long hi;  // unit << 32 | block (padding: all ones)
    unsigned long long lo;  // order key of z (or the position, to keep the order)
    int id;                 // token index in the unit's source rows
    int pad;
};

constexpr int CL_TILE = 1024;  // records sorted in shared memory by one block
constexpr int CL_THREADS = CL_TILE / 2;

__device__ __forceinline__ bool cl_less(const ClRec& a, const ClRec& b) {
    if (a.hi != b.hi) return a.hi < b.hi;
    if (a.lo != b.lo) return a.lo < b.lo;
    return a.id < b.id;
}

// Order-preserving 64-bit key of a double (no NaN; -0 was made +0).
__device__ __forceinline__ unsigned long long order_key(double z) {
    const unsigned long long b = (unsigned long long)__double_as_longlong(z);
    return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}

struct ClArgs {
    const void* ksrc;        // [B][H][src_len][D], storage type
    const void* vsrc;
    long long src_len;
    const float* Z;          // [J_cap][D] learned directions, row j - 1 for level j
    const long long* sstart; // [B + 1] prefix sums of the sequences' lengths
    int* perm;               // [B][H][cap]
    ClRec* rec;              // [n_pad]
    long long n, n_pad;      // records in use (every unit's tokens), padded count
};

// The unit of sequence b = u / H, KV head h = u % H, and its first record.
__device__ __forceinline__ long long unit_start(const ClArgs& a, int H, long long u, long long& L) {
    const long long b = u / H;
    L = a.sstart[b + 1] - a.sstart[b];
    return H * a.sstart[b] + (u % H) * L;
}

// Levels of the tree over L tokens: the first j >= 1 with ceil(L / b^j) <= b.
__device__ __forceinline__ int unit_levels(long long L, int b) {
    int j = 1;
    long long s = b;
    while (j < MAXJ && (L + s - 1) / s > b) {
        s = s > LLONG_MAX / b ? LLONG_MAX : s * b;
        j++;
    }
    return j;
}

__device__ __forceinline__ long long pow_sat(int b, int e) {
    long long s = 1;
    for (int i = 0; i < e; i++) s = s > LLONG_MAX / b ? LLONG_MAX : s * b;
    return s;
}

// Keys of level j for every record. first: the records are laid out from
// their index (unit by unit, identity order); else they hold the order the
// previous level's sort left. Units with fewer than j levels keep their order.
template <typename T, int D>
__global__ void __launch_bounds__(256) cl_keys_kernel(TreeParams p, ClArgs a, int j, int first) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= a.n_pad) return;
    if (i >= a.n) {
        a.rec[i] = ClRec{~0ull, ~0ull, INT_MAX, 0};
        return;
    }
    long long u, id;
    if (first) {
        int b = 0;  // the sequence holding record i (a few sequences: a linear scan)
        while (b + 1 < p.B && p.H * a.sstart[b + 1] <= i) b++;
        const long long L = a.sstart[b + 1] - a.sstart[b];
        const long long off = i - p.H * a.sstart[b];
        u = (long long)b * p.H + off / L;
        id = off % L;
    } else {
        u = (long long)(a.rec[i].hi >> 32);
        id = a.rec[i].id;
    }
    long long L;
    const long long pos = i - unit_start(a, p.H, u, L);
    ClRec r;
    r.id = (int)id;
    r.pad = 0;
    if (j <= unit_levels(L, p.b)) {
        const T* k = reinterpret_cast<const T*>(a.ksrc) + (u * a.src_len + id) * D;
        const float* zd = a.Z + (size_t)(j - 1) * D;
        double z = 0.0;
#pragma unroll 8
        for (int e = 0; e < D; e++) z = __dadd_rn(z, __dmul_rn((double)zd[e], (double)to_f(k[e])));
        z = __dadd_rn(z, 0.0);
        r.hi = ((unsigned long long)u << 32) | (unsigned long long)(pos / pow_sat(p.b, j + 1));
        r.lo = order_key(z);
    } else {
        r.hi = (unsigned long long)u << 32;
        r.lo = (unsigned long long)pos;
    }
    a.rec[i] = r;
}

// Compare-exchange of records i < l in the network's direction for stage k.
__device__ __forceinline__ void cl_cmpx(ClRec& x, ClRec& y, bool asc) {
    if (cl_less(y, x) == asc) {
        const ClRec t = x;
        x = y;
        y = t;
    }
}

// Stages k = 2 .. CL_TILE in shared memory (first = true), or the distances
// CL_TILE / 2 .. 1 of stage k (first = false), for one tile of CL_TILE records.
__global__ void __launch_bounds__(CL_THREADS) cl_tile_kernel(ClRec* rec, long long k, int first) {
    __shared__ ClRec s[CL_TILE];
    const long long base = (long long)blockIdx.x * CL_TILE;
    const int t = threadIdx.x;
    s[t] = rec[base + t];
    s[t + CL_THREADS] = rec[base + t + CL_THREADS];
    __syncthreads();
    const long long k_lo = first ? 2 : k, k_hi = first ? CL_TILE : k;
    for (long long kk = k_lo; kk <= k_hi; kk <<= 1) {
        for (int jj = (int)min(kk >> 1, (long long)(CL_TILE / 2)); jj > 0; jj >>= 1) {
            const int lo = 2 * t - (t & (jj - 1));  // the pair (lo, lo + jj) of this thread
            const bool asc = ((base + lo) & kk) == 0;
            cl_cmpx(s[lo], s[lo + jj], asc);
            __syncthreads();
        }
    }
    rec[base + t] = s[t];
    rec[base + t + CL_THREADS] = s[t + CL_THREADS];
}

// One distance j >= CL_TILE of stage k over the whole array.
__global__ void __launch_bounds__(256) cl_pass_kernel(ClRec* rec, long long n_pad, long long k, long long j) {
    const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= n_pad / 2) return;
    const long long lo = 2 * t - (t & (j - 1));
    const bool asc = (lo & k) == 0;
    ClRec x = rec[lo], y = rec[lo + j];
    if (cl_less(y, x) == asc) {
        rec[lo] = y;
        rec[lo + j] = x;
    }
}

// Two distances j and j / 2 of stage k in one pass (j / 2 >= CL_TILE): each
// thread holds the four records i0, i0 + j/2, i0 + j, i0 + 3j/2 (bits j and
// j/2 of i0 clear), which the two steps only exchange among themselves, and
// applies the distance-j then the distance-j/2 compare-exchanges.
__global__ void __launch_bounds__(256) cl_pass2_kernel(ClRec* rec, long long n_pad, long long k, long long j) {
    const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= n_pad / 4) return;
    const long long h = j >> 1;
    const long long i0 = (t & (h - 1)) | ((t & ~(h - 1)) << 2);
    const bool asc = (i0 & k) == 0;
    ClRec a = rec[i0], b = rec[i0 + h], c = rec[i0 + j], d = rec[i0 + j + h];
    cl_cmpx(a, c, asc);
    cl_cmpx(b, d, asc);
    cl_cmpx(a, b, asc);
    cl_cmpx(c, d, asc);
    rec[i0] = a;
    rec[i0 + h] = b;
    rec[i0 + j] = c;
    rec[i0 + j + h] = d;
}

// The order after the last level: perm[u][pos] = the token placed at pos, and
// the token's key and value rows copied there (one warp per record).
template <typename T, int D>
__global__ void __launch_bounds__(256) cl_place_kernel(TreeParams p, ClArgs a) {
    const long long i = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (i >= a.n) return;
    const long long u = (long long)(a.rec[i].hi >> 32);
    const long long id = a.rec[i].id;
    long long L;
    const long long pos = i - unit_start(a, p.H, u, L);
    if (lane == 0) a.perm[u * p.cap + pos] = (int)id;
    constexpr int V = 16 / sizeof(T);  // elements per 16-byte piece
    const uint4* ks = reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(a.ksrc) + (u * a.src_len + id) * D);
    const uint4* vs = reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(a.vsrc) + (u * a.src_len + id) * D);
    uint4* kd = reinterpret_cast<uint4*>(reinterpret_cast<T*>(p.K[0]) + (u * p.cap + pos) * D);
    uint4* vd = reinterpret_cast<uint4*>(reinterpret_cast<T*>(p.V[0]) + (u * p.cap + pos) * D);
    for (int c = lane; c < D / V; c += 32) {
        kd[c] = ks[c];
        vd[c] = vs[c];
    }
}

// Records needed for every unit at capacity, as a power of two.
long long cluster_records(long long units, long long cap) {
    long long n = 1;
    while (n < units * cap) n <<= 1;
    return n < CL_TILE ? CL_TILE : n;
}
size_t cluster_rec_bytes(long long units, long long cap) { return (size_t)cluster_records(units, cap) * sizeof(ClRec); }

template <typename T, int D>
cudaError_t launch_cluster(const TreeParams& p, const void* ksrc, const void* vsrc, long long src_len, const float* Z,
                           const long long* sstart_dev, long long n, int J_max, int* perm, void* rec_mem,
                           cudaStream_t s) {
    ClArgs a;
    a.ksrc = ksrc;
    a.vsrc = vsrc;
    a.src_len = src_len;
    a.Z = Z;
    a.sstart = sstart_dev;
    a.perm = perm;
    a.rec = static_cast<ClRec*>(rec_mem);
    a.n = n;
    a.n_pad = CL_TILE;
    while (a.n_pad < n) a.n_pad <<= 1;
    const unsigned gk = (unsigned)((a.n_pad + 255) / 256), gp = (unsigned)((a.n_pad / 2 + 255) / 256);
    const unsigned gp2 = (unsigned)((a.n_pad / 4 + 255) / 256);
    const unsigned gt = (unsigned)(a.n_pad / CL_TILE);
    for (int j = J_max; j >= 1; j--) {
        cl_keys_kernel<T, D><<<gk, 256, 0, s>>>(p, a, j, j == J_max);
        cl_tile_kernel<<<gt, CL_THREADS, 0, s>>>(a.rec, 0, 1);
        for (long long k = 2 * CL_TILE; k <= a.n_pad; k <<= 1) {
            long long jj = k >> 1;
            for (; (jj >> 1) >= CL_TILE; jj >>= 2) cl_pass2_kernel<<<gp2, 256, 0, s>>>(a.rec, a.n_pad, k, jj);
            if (jj >= CL_TILE) cl_pass_kernel<<<gp, 256, 0, s>>>(a.rec, a.n_pad, k, jj);
            cl_tile_kernel<<<gt, CL_THREADS, 0, s>>>(a.rec, k, 0);
        }
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    cl_place_kernel<T, D><<<(unsigned)((n * 32 + 255) / 256), 256, 0, s>>>(p, a);
    return cudaGetLastError();
}

template cudaError_t launch_cluster<float, 64>(const TreeParams&, const void*, const void*, long long, const float*,
                                               const long long*, long long, int, int*, void*, cudaStream_t);
template cudaError_t launch_cluster<float, 128>(const TreeParams&, const void*, const void*, long long, const float*,
                                                const long long*, long long, int, int*, void*, cudaStream_t);
template cudaError_t launch_cluster<__nv_bfloat16, 64>(const TreeParams&, const void*, const void*, long long,
                                                       const float*, const long long*, long long, int, int*, void*,
                                                       cudaStream_t);
template cudaError_t launch_cluster<__nv_bfloat16, 128>(const TreeParams&, const void*, const void*, long long,
                                                        const float*, const long long*, long long, int, int*, void*,
                                                        cudaStream_t);

}  // namespace recsa
