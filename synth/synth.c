/*
 * Seeded synthetic inputs for the RecSA tree-attention workloads.
 *
 * This file generates data only: it holds none of the attention method's
 * arithmetic. Both the CUDA path and the CPU oracle consume the arrays it
 * writes, so they always see the same bits.
 *
 * Generator: a counter-based use of splitmix64 (Steele, Lea and Flood,
 * "Fast splittable pseudorandom number generators", OOPSLA 2014; the
 * finaliser constants are Vigna's published splitmix64). The i-th draw of a
 * stream whose state starts at `base` is mix64(base + (i+1)*GOLDEN), so any
 * element can be produced independently of the others and the work splits
 * across threads with no shared state. Uniforms in (0,1) take the top 53
 * bits; standard normals come from the Box-Muller transform applied to the
 * uniform pair (2p, 2p+1), element 2p taking the cosine branch and 2p+1 the
 * sine branch.
 *
 * Workload recipe (keys from a Gaussian mixture laid out in contiguous runs,
 * values N(0,1), queries aimed at one planted run, a random linear pooler):
 *   - runs: consecutive token runs per sequence, lengths uniform in
 *     [run_min, run_max]; the layout is shared by every KV head;
 *   - centroids: M per KV head, each coordinate N(0, 1), shared by all
 *     sequences;
 *   - run r of sequence s uses centroid floor(U * M) for head h;
 *   - key k[h][t] = centroid + sigma * N(0, I);  value v[h][t] = N(0, I);
 *   - decode query for step n: a run chosen uniformly among the runs that
 *     start before the current length; q[g] = that run's centroid for KV head
 *     g / G plus sigma * N(0, I);
 *   - prefill query for token t: the centroid of t's own run plus noise;
 *   - pooler W[i][j] = N(0, 1) / sqrt(d).
 * Results are rounded once, double -> float (round to nearest even), and for
 * bf16 outputs float -> bf16 (round to nearest even).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define GOLDEN 0x9E3779B97F4A7C15ULL

enum {
    TAG_RUN_LEN = 1,
    TAG_RUN_CENT = 2,
    TAG_CENTROID = 3,
    TAG_KEY_NOISE = 4,
    TAG_VALUE = 5,
    TAG_DQ_RUN = 6,
    TAG_DQ_NOISE = 7,
    TAG_PQ_NOISE = 8,
    TAG_POOLER = 9,
    TAG_PLAIN = 10,
};

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

uint64_t synth_splitmix64_at(uint64_t base, uint64_t i) { return mix64(base + (i + 1) * GOLDEN); }

static inline double u01_at(uint64_t base, uint64_t i) {
    return ((double)(synth_splitmix64_at(base, i) >> 11) + 0.5) * 0x1.0p-53;
}

double synth_uniform_at(uint64_t base, uint64_t i) { return u01_at(base, i); }

static inline void normal_pair(uint64_t base, uint64_t p, double* c, double* s) {
    double u1 = u01_at(base, 2 * p), u2 = u01_at(base, 2 * p + 1);
    double r = sqrt(-2.0 * log(u1));
    double th = 6.283185307179586476925286766559 * u2;
    *c = r * cos(th);
    *s = r * sin(th);
}

double synth_normal_at(uint64_t base, uint64_t i) {
    double c, s;
    normal_pair(base, i >> 1, &c, &s);
    return (i & 1) ? s : c;
}

/* Stream base for (seed, tag, a): a fixed hash of the three. */
uint64_t synth_stream(uint64_t seed, uint64_t tag, uint64_t a) {
    return mix64(mix64(mix64(seed ^ 0x5EEDF00DULL) ^ (tag * GOLDEN)) ^ (a * 0xD1B54A32D192ED03ULL + 1));
}

static inline uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

static inline void store(void* out, int out_bf16, int64_t idx, double x) {
    float f = (float)x;
    if (out_bf16)
        ((uint16_t*)out)[idx] = f32_to_bf16_rne(f);
    else
        ((float*)out)[idx] = f;
}

/* ---------------------------------------------------------------- runs */

/* Fills run_start[0..n] with the starts of the runs covering [0, L) and
 * run_start[n] = L; returns n (or -1 if max_runs is too small). */
long long synth_runs(uint64_t seed, int seq, long long L, int run_min, int run_max, long long* run_start,
                     long long max_runs) {
    uint64_t base = synth_stream(seed, TAG_RUN_LEN, (uint64_t)seq);
    long long t = 0, n = 0;
    while (t < L) {
        if (n >= max_runs) return -1;
        run_start[n] = t;
        long long len = run_min + (long long)(u01_at(base, (uint64_t)n) * (double)(run_max - run_min + 1));
        if (len > run_max) len = run_max;
        t += len;
        n++;
    }
    run_start[n] = L;
    return n;
}

static inline long long run_centroid(uint64_t seed, int seq, long long run, int H, int h, int M) {
    uint64_t base = synth_stream(seed, TAG_RUN_CENT, (uint64_t)seq);
    long long m = (long long)(u01_at(base, (uint64_t)run * (uint64_t)H + (uint64_t)h) * (double)M);
    return m >= M ? M - 1 : m;
}

static inline double centroid_coord(uint64_t seed, int H, int h, long long m, int M, int d, int i) {
    (void)H;
    uint64_t base = synth_stream(seed, TAG_CENTROID, 0);
    return synth_normal_at(base, ((uint64_t)h * (uint64_t)M + (uint64_t)m) * (uint64_t)d + (uint64_t)i);
}

/* ------------------------------------------------------------- threads */

typedef struct {
    void (*fn)(void* arg, long long lo, long long hi);
    void* arg;
    long long lo, hi;
} job_t;

static void* job_main(void* p) {
    job_t* j = (job_t*)p;
    j->fn(j->arg, j->lo, j->hi);
    return NULL;
}

static void parallel_for(long long n, int nthreads, void (*fn)(void*, long long, long long), void* arg) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (n < 4096 || nthreads == 1) {
        fn(arg, 0, n);
        return;
    }
    pthread_t th[256];
    job_t jobs[256];
    long long chunk = (n + nthreads - 1) / nthreads;
    int started = 0;
    for (int t = 0; t < nthreads; t++) {
        long long lo = t * chunk, hi = lo + chunk < n ? lo + chunk : n;
        if (lo >= hi) break;
        jobs[t].fn = fn;
        jobs[t].arg = arg;
        jobs[t].lo = lo;
        jobs[t].hi = hi;
        if (pthread_create(&th[t], NULL, job_main, &jobs[t]) != 0) {
            fn(arg, lo, hi);
            jobs[t].fn = NULL;
        }
        started = t + 1;
    }
    for (int t = 0; t < started; t++)
        if (jobs[t].fn) pthread_join(th[t], NULL);
}

/* ------------------------------------------------------- keys, values */

typedef struct {
    uint64_t seed;
    int seq, H, d, M, out_bf16, is_key;
    double sigma;
    const long long* run_start;
    long long n_runs, t0, t1, head_stride;
    void* out;
} kv_args;

static void kv_rows(void* p, long long lo, long long hi) {
    kv_args* a = (kv_args*)p;
    long long T = a->t1 - a->t0;
    uint64_t bn = synth_stream(a->seed, a->is_key ? TAG_KEY_NOISE : TAG_VALUE, (uint64_t)a->seq);
    long long run = -1;
    double* cent = (double*)malloc(sizeof(double) * (size_t)a->H * (size_t)a->d);
    long long cent_run = -2;
    for (long long r = lo; r < hi; r++) { /* r indexes (h, t) rows, head-major */
        int h = (int)(r / T);
        long long t = a->t0 + r % T;
        if (a->is_key) {
            /* locate the run of token t (runs are sorted) */
            if (run < 0 || !(a->run_start[run] <= t && t < a->run_start[run + 1])) {
                long long L0 = 0, H0 = a->n_runs - 1;
                while (L0 < H0) {
                    long long mid = (L0 + H0 + 1) / 2;
                    if (a->run_start[mid] <= t)
                        L0 = mid;
                    else
                        H0 = mid - 1;
                }
                run = L0;
            }
            if (cent_run != run * a->H + h) {
                long long m = run_centroid(a->seed, a->seq, run, a->H, h, a->M);
                for (int i = 0; i < a->d; i++) cent[i] = centroid_coord(a->seed, a->H, h, m, a->M, a->d, i);
                cent_run = run * a->H + h;
            }
        }
        uint64_t ctr = ((uint64_t)h << 40) + (uint64_t)t * (uint64_t)a->d;
        int64_t obase = (int64_t)h * a->head_stride + (int64_t)(t - a->t0) * a->d;
        for (int i = 0; i < a->d; i += 2) {
            double c, s;
            normal_pair(bn, (ctr + (uint64_t)i) >> 1, &c, &s);
            double x0 = a->is_key ? cent[i] + a->sigma * c : c;
            double x1 = a->is_key ? cent[i + 1] + a->sigma * s : s;
            store(a->out, a->out_bf16, obase + i, x0);
            store(a->out, a->out_bf16, obase + i + 1, x1);
        }
    }
    free(cent);
}

/* Keys of sequence `seq`, tokens [t0, t1), every KV head: element (h, t, i)
 * goes to out[h*head_stride + (t-t0)*d + i]. d must be even. */
void synth_keys(uint64_t seed, int seq, int H, int d, int M, double sigma, const long long* run_start,
                long long n_runs, long long t0, long long t1, long long head_stride, int out_bf16, void* out,
                int nthreads) {
    kv_args a = {seed, seq, H, d, M, out_bf16, 1, sigma, run_start, n_runs, t0, t1, head_stride, out};
    parallel_for((long long)H * (t1 - t0), nthreads, kv_rows, &a);
}

/* Values of sequence `seq`, same addressing as synth_keys. */
void synth_values(uint64_t seed, int seq, int H, int d, long long t0, long long t1, long long head_stride,
                  int out_bf16, void* out, int nthreads) {
    kv_args a = {seed, seq, H, d, 1, out_bf16, 0, 0.0, NULL, 0, t0, t1, head_stride, out};
    parallel_for((long long)H * (t1 - t0), nthreads, kv_rows, &a);
}

/* ------------------------------------------------------------ queries */

/* Decode query of sequence `seq` at step `step`, when the cache holds
 * `length` tokens: out[g*d + i] for the Hq = G*H query heads. Returns the
 * planted run. */
long long synth_decode_query(uint64_t seed, int seq, long long step, long long length, int H, int G, int d, int M,
                             double sigma, const long long* run_start, long long n_runs, int out_bf16, void* out) {
    long long n_cached = 0;
    while (n_cached < n_runs && run_start[n_cached] < length) n_cached++;
    if (n_cached == 0) n_cached = 1;
    uint64_t br = synth_stream(seed, TAG_DQ_RUN, (uint64_t)seq);
    long long run = (long long)(u01_at(br, (uint64_t)step) * (double)n_cached);
    if (run >= n_cached) run = n_cached - 1;
    uint64_t bn = synth_stream(seed, TAG_DQ_NOISE, (uint64_t)seq);
    for (int g = 0; g < H * G; g++) {
        int h = g / G;
        long long m = run_centroid(seed, seq, run, H, h, M);
        for (int i = 0; i < d; i++) {
            double x = centroid_coord(seed, H, h, m, M, d, i) +
                       sigma * synth_normal_at(bn, ((uint64_t)step << 24) + (uint64_t)g * (uint64_t)d + (uint64_t)i);
            store(out, out_bf16, (int64_t)g * d + i, x);
        }
    }
    return run;
}

typedef struct {
    uint64_t seed;
    int seq, H, G, d, M, out_bf16;
    double sigma;
    const long long* run_start;
    long long n_runs, t0;
    void* out;
} pq_args;

static void pq_rows(void* p, long long lo, long long hi) {
    pq_args* a = (pq_args*)p;
    uint64_t bn = synth_stream(a->seed, TAG_PQ_NOISE, (uint64_t)a->seq);
    int Hq = a->H * a->G;
    double* cent = (double*)malloc(sizeof(double) * (size_t)a->H * (size_t)a->d);
    long long cent_run = -1;
    for (long long r = lo; r < hi; r++) { /* r indexes (t - t0) */
        long long t = a->t0 + r;
        long long L0 = 0, H0 = a->n_runs - 1;
        while (L0 < H0) {
            long long mid = (L0 + H0 + 1) / 2;
            if (a->run_start[mid] <= t)
                L0 = mid;
            else
                H0 = mid - 1;
        }
        if (L0 != cent_run) { /* centroids of this run, every KV head */
            for (int h = 0; h < a->H; h++) {
                long long m = run_centroid(a->seed, a->seq, L0, a->H, h, a->M);
                for (int i = 0; i < a->d; i++) cent[h * a->d + i] = centroid_coord(a->seed, a->H, h, m, a->M, a->d, i);
            }
            cent_run = L0;
        }
        for (int g = 0; g < Hq; g++) {
            int h = g / a->G;
            uint64_t ctr = ((uint64_t)t << 24) + (uint64_t)g * (uint64_t)a->d;
            for (int i = 0; i < a->d; i += 2) {
                double c, sn;
                normal_pair(bn, (ctr + (uint64_t)i) >> 1, &c, &sn);
                store(a->out, a->out_bf16, (r * Hq + g) * (int64_t)a->d + i, cent[h * a->d + i] + a->sigma * c);
                store(a->out, a->out_bf16, (r * Hq + g) * (int64_t)a->d + i + 1,
                      cent[h * a->d + i + 1] + a->sigma * sn);
            }
        }
    }
    free(cent);
}

/* Prefill queries for tokens [t0, t1) of sequence `seq`: out[(t-t0)][g][i]. */
void synth_prefill_queries(uint64_t seed, int seq, long long t0, long long t1, int H, int G, int d, int M,
                           double sigma, const long long* run_start, long long n_runs, int out_bf16, void* out,
                           int nthreads) {
    pq_args a = {seed, seq, H, G, d, M, out_bf16, sigma, run_start, n_runs, t0, out};
    parallel_for(t1 - t0, nthreads, pq_rows, &a);
}

/* Pooler W[i][j] = N(0,1)/sqrt(d), row-major d x d. */
void synth_pooler(uint64_t seed, int d, int out_bf16, void* out) {
    uint64_t b = synth_stream(seed, TAG_POOLER, (uint64_t)d);
    double s = 1.0 / sqrt((double)d);
    for (int i = 0; i < d * d; i++) store(out, out_bf16, i, s * synth_normal_at(b, (uint64_t)i));
}

/* Plain N(mean, scale^2) fill of n elements of stream `a`: for tests that
 * need unstructured data. */
void synth_plain(uint64_t seed, uint64_t a, long long n, double mean, double scale, int out_bf16, void* out) {
    uint64_t b = synth_stream(seed, TAG_PLAIN, a);
    for (long long i = 0; i < n; i++) store(out, out_bf16, i, mean + scale * synth_normal_at(b, (uint64_t)i));
}
