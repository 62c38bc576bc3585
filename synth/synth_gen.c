/*
 * Seeded synthetic input generator (host C).
 *
 * Counter-based: the i-th number of stream (seed, stream) depends only on
 * (seed, stream, i), so any slice of a tensor can be regenerated on its own.
 *
 *   key      = splitmix64_mix(seed * 0x100000001B3 + stream + 1)
 *   bits(i)  = splitmix64_mix(key + (i + 1) * 0x9E3779B97F4A7C15)
 *   u(i)     = ((bits(i) >> 11) + 0.5) * 2^-53          in (0, 1)
 *   normal(j) = sqrt(-2 ln u(2j)) * cos(2 pi u(2j+1))    (Box-Muller, cosine branch)
 *
 * splitmix64_mix is the finaliser of Steele, Lea and Flood's SplitMix64
 * ("Fast splittable pseudorandom number generators", OOPSLA 2014), with the
 * shift/multiply constants published there.
 *
 * This file holds no arithmetic of the recurrence itself: it draws numbers
 * and shapes them into the workloads' value distributions (normalisation,
 * softplus, sigmoid, rounding to the storage dtype).
 */
#include <math.h>
#include <pthread.h>
#include <stddef.h>
#include <stdint.h>

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

static inline uint64_t stream_key(uint64_t seed, uint64_t stream) {
    return mix64(seed * 0x100000001B3ULL + stream + 1ULL);
}

static inline double unit_open(uint64_t key, uint64_t i) {
    uint64_t z = mix64(key + (i + 1ULL) * 0x9E3779B97F4A7C15ULL);
    return ((double)(z >> 11) + 0.5) * (1.0 / 9007199254740992.0);
}

/* out[j] = j-th uniform in (0,1) of the stream, j = offset .. offset+n-1 */
void synth_uniform(uint64_t seed, uint64_t stream, uint64_t offset, size_t n, double *out) {
    uint64_t key = stream_key(seed, stream);
    for (size_t j = 0; j < n; ++j) out[j] = unit_open(key, offset + j);
}

/* out[j] = j-th standard normal of the stream, j = offset .. offset+n-1 */
void synth_normal(uint64_t seed, uint64_t stream, uint64_t offset, size_t n, double *out) {
    const double two_pi = 6.283185307179586476925286766559;
    uint64_t key = stream_key(seed, stream);
    for (size_t j = 0; j < n; ++j) {
        uint64_t idx = 2ULL * (offset + j);
        double u1 = unit_open(key, idx);
        double u2 = unit_open(key, idx + 1ULL);
        out[j] = sqrt(-2.0 * log(u1)) * cos(two_pi * u2);
    }
}

/* Row gather: out[r*rowlen + j] = normal number (offsets[r] + j) of the stream. */
void synth_normal_rows(uint64_t seed, uint64_t stream, const uint64_t *offsets, size_t nrows,
                       size_t rowlen, double *out) {
    for (size_t r = 0; r < nrows; ++r) synth_normal(seed, stream, offsets[r], rowlen, out + r * rowlen);
}

typedef struct {
    uint64_t seed, stream, offset;
    size_t n;
    double *out;
} span_job;

static void *span_worker(void *p) {
    span_job *j = (span_job *)p;
    synth_normal(j->seed, j->stream, j->offset, j->n, j->out);
    return NULL;
}

/* Same numbers as synth_normal, drawn by up to `nthreads` host threads. */
void synth_normal_mt(uint64_t seed, uint64_t stream, uint64_t offset, size_t n, double *out, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 64) nthreads = 64;
    if (n < (size_t)nthreads * 65536 || nthreads == 1) {
        synth_normal(seed, stream, offset, n, out);
        return;
    }
    pthread_t tid[64];
    span_job jobs[64];
    size_t per = (n + (size_t)nthreads - 1) / (size_t)nthreads;
    int started = 0;
    for (int t = 0; t < nthreads; ++t) {
        size_t lo = (size_t)t * per;
        if (lo >= n) break;
        size_t cnt = (lo + per > n) ? n - lo : per;
        jobs[t].seed = seed; jobs[t].stream = stream; jobs[t].offset = offset + lo;
        jobs[t].n = cnt; jobs[t].out = out + lo;
        if (pthread_create(&tid[t], NULL, span_worker, &jobs[t]) != 0) {
            span_worker(&jobs[t]);
            tid[t] = 0;
        }
        started = t + 1;
    }
    for (int t = 0; t < started; ++t)
        if (tid[t]) pthread_join(tid[t], NULL);
}

/* ------------------------------------------------------------------ shaped rows
 * kind 0: x = scale * N(0,1)                          (v, S0)
 * kind 1: x = N(0,1) row, L2-normalised over the row  (q, k)
 * kind 2: x = sigmoid(N(0,1))                         (b, w, beta)
 * kind 3: x = exp(-scale * softplus(N(0,1) + mu))     (alpha)
 * Row r of the output is row index rows[r] (or row0 + r when rows == NULL) of the
 * full tensor; its element j has counter rows[r]*d + j, or rows[r] alone when
 * per_token != 0 (one draw broadcast over the row).  Values are computed in fp64,
 * rounded to fp32 (round-to-nearest-even), and, with bf16 != 0, further rounded to
 * bfloat16 precision (round-to-nearest-even on the fp32 bit pattern).  Output is fp32.
 */
typedef struct {
    uint64_t seed, stream;
    int kind;
    double mu, scale;
    const uint64_t *rows;
    uint64_t row0;
    size_t r_lo, r_hi, d;
    int per_token, bf16;
    float *out;
} rows_job;

static inline float round_bf16(float f) {
    union { float f; uint32_t u; } x;
    x.f = f;
    uint32_t lsb = (x.u >> 16) & 1u;
    x.u = (x.u + 0x7FFFu + lsb) & 0xFFFF0000u;
    return x.f;
}

static inline double shape_value(int kind, double z, double mu, double scale) {
    switch (kind) {
        case 2: return 1.0 / (1.0 + exp(-z));
        case 3: {
            double t = z + mu;
            double sp = t > 0 ? t + log1p(exp(-t)) : log1p(exp(t));
            return exp(-scale * sp);
        }
        default: return scale * z;
    }
}

static void *rows_worker(void *p) {
    rows_job *J = (rows_job *)p;
    const double two_pi = 6.283185307179586476925286766559;
    uint64_t key = stream_key(J->seed, J->stream);
    double buf[1024];
    for (size_t r = J->r_lo; r < J->r_hi; ++r) {
        uint64_t row = J->rows ? J->rows[r] : J->row0 + r;
        float *o = J->out + r * J->d;
        if (J->per_token) {
            uint64_t idx = 2ULL * row;
            double z = sqrt(-2.0 * log(unit_open(key, idx))) * cos(two_pi * unit_open(key, idx + 1ULL));
            float f = (float)shape_value(J->kind, z, J->mu, J->scale);
            if (J->bf16) f = round_bf16(f);
            for (size_t j = 0; j < J->d; ++j) o[j] = f;
            continue;
        }
        for (size_t j0 = 0; j0 < J->d; j0 += 1024) {
            size_t n = J->d - j0 < 1024 ? J->d - j0 : 1024;
            double ss = 0.0;
            for (size_t j = 0; j < n; ++j) {
                uint64_t idx = 2ULL * (row * J->d + j0 + j);
                double z = sqrt(-2.0 * log(unit_open(key, idx))) * cos(two_pi * unit_open(key, idx + 1ULL));
                buf[j] = z;
                ss += z * z;
            }
            double inv = 1.0;
            if (J->kind == 1) inv = 1.0 / sqrt(ss > 0 ? ss : 1e-300);  /* d <= 1024 for kind 1 */
            for (size_t j = 0; j < n; ++j) {
                double x = J->kind == 1 ? buf[j] * inv : shape_value(J->kind, buf[j], J->mu, J->scale);
                float f = (float)x;
                if (J->bf16) f = round_bf16(f);
                o[j0 + j] = f;
            }
        }
    }
    return NULL;
}

int synth_rows(uint64_t seed, uint64_t stream, int kind, double mu, double scale, const uint64_t *rows,
               uint64_t row0, size_t nrows, size_t d, int per_token, int bf16, float *out, int nthreads) {
    if (kind == 1 && d > 1024) return -1;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 64) nthreads = 64;
    if ((size_t)nthreads > nrows) nthreads = nrows ? (int)nrows : 1;
    pthread_t tid[64];
    rows_job jobs[64];
    size_t per = (nrows + (size_t)nthreads - 1) / (size_t)nthreads;
    int started = 0;
    for (int t = 0; t < nthreads; ++t) {
        size_t lo = (size_t)t * per;
        if (lo >= nrows) break;
        size_t hi = lo + per > nrows ? nrows : lo + per;
        rows_job J = {seed, stream, kind, mu, scale, rows, row0, lo, hi, d, per_token, bf16, out};
        jobs[t] = J;
        started = t + 1;
    }
    if (started <= 1) {
        if (started == 1) rows_worker(&jobs[0]);
        return 0;
    }
    for (int t = 0; t < started; ++t)
        if (pthread_create(&tid[t], NULL, rows_worker, &jobs[t]) != 0) {
            rows_worker(&jobs[t]);
            tid[t] = 0;
        }
    for (int t = 0; t < started; ++t)
        if (tid[t]) pthread_join(tid[t], NULL);
    return 0;
}
