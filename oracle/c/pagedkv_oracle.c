/*
 * Plain C oracle of the paged KV-cache decode step — TEST INFRASTRUCTURE ONLY
 * (used by tests and by the CPU-baseline leg of the benchmark; never by the
 * library). Shares no code with the CUDA path.
 *
 * Definition followed ("vLLM / PagedAttention — 分页 KV Cache 分析", §2.2 and
 * §3.1, with the per-page loop read as one softmax per (sequence, query head)
 * over all of the sequence's tokens): gather the sequence's pages into a
 * contiguous K and V (exact fp32 copies of the fp16/bf16 values), then
 *   x_t = scale * sum_i q_i K_t,i ;  out = sum_t softmax(x)_t V_t
 * with fp64 accumulation. Query head h reads KV head h / (Hq / Hkv).
 * Zero-length contexts give 0.
 *
 * The cache write follows §3.2 of the same page: token t's K/V row goes to row
 * slot % bs of page slot / bs; slot < 0 is padding.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static float half_to_float(uint16_t h) {
    int sign = (h >> 15) & 1, e = (h >> 10) & 31, m = h & 1023;
    float v;
    if (e == 0)
        v = ldexpf((float)m, -24);
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexpf((float)(1024 + m), e - 25);
    return sign ? -v : v;
}

static float bf16_to_float(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

static float to_float(uint16_t x, int dtype) {
    return dtype == 0 ? half_to_float(x) : bf16_to_float(x);
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* out: double [B, Hq, d]; q [B, Hq, d]; caches [NB, Hkv, bs, d] (uint16 bits). */
int oracle_paged_decode(double *out, const uint16_t *q, const uint16_t *k_cache,
                        const uint16_t *v_cache, const int32_t *block_tables,
                        const int32_t *context_lens, int B, int Hq, int Hkv, int d, int bs,
                        int max_blocks_per_seq, double scale, int dtype, int nthreads) {
    if (Hkv <= 0 || Hq % Hkv != 0) return -1;
    const int G = Hq / Hkv;
    const long pairs = (long)B * Hkv;
    int bad = 0;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads) reduction(| : bad)
#endif
    for (long w = 0; w < pairs; ++w) {
        const int s = (int)(w / Hkv), hk = (int)(w % Hkv);
        const int n = context_lens[s];
        double *o = out + ((size_t)s * Hq + (size_t)hk * G) * d;
        if (n <= 0) {
            memset(o, 0, sizeof(double) * G * d);
            continue;
        }
        float *K = (float *)malloc(sizeof(float) * (size_t)n * d);
        float *V = (float *)malloc(sizeof(float) * (size_t)n * d);
        double *x = (double *)malloc(sizeof(double) * (size_t)n);
        if (!K || !V || !x) {
            free(K); free(V); free(x);
            bad = 1;
            continue;
        }
        /* gather: logical token t -> page block_tables[s][t / bs], row t % bs */
        for (int t = 0; t < n; ++t) {
            const int page = block_tables[(size_t)s * max_blocks_per_seq + t / bs];
            const size_t base = (((size_t)page * Hkv + hk) * bs + (t % bs)) * d;
            for (int i = 0; i < d; ++i) {
                K[(size_t)t * d + i] = to_float(k_cache[base + i], dtype);
                V[(size_t)t * d + i] = to_float(v_cache[base + i], dtype);
            }
        }
        for (int g = 0; g < G; ++g) {
            const uint16_t *qh = q + ((size_t)s * Hq + (size_t)hk * G + g) * d;
            double mx = -INFINITY;
            for (int t = 0; t < n; ++t) {
                double acc = 0.0;
                for (int i = 0; i < d; ++i) acc += (double)to_float(qh[i], dtype) * K[(size_t)t * d + i];
                x[t] = scale * acc;
                if (x[t] > mx) mx = x[t];
            }
            double sum = 0.0;
            for (int t = 0; t < n; ++t) {
                x[t] = exp(x[t] - mx);
                sum += x[t];
            }
            double *oh = o + (size_t)g * d;
            for (int i = 0; i < d; ++i) oh[i] = 0.0;
            for (int t = 0; t < n; ++t) {
                const double p = x[t] / sum;
                for (int i = 0; i < d; ++i) oh[i] += p * V[(size_t)t * d + i];
            }
        }
        free(K); free(V); free(x);
    }
    return bad ? -2 : 0;
}

/* In-place cache write: k_new/v_new [T, Hkv, d]; caches [NB, Hkv, bs, d]. */
int oracle_reshape_and_cache(const uint16_t *k_new, const uint16_t *v_new, uint16_t *k_cache,
                             uint16_t *v_cache, const int64_t *slot_mapping, int T, int Hkv,
                             int d, int bs) {
    for (int t = 0; t < T; ++t) {
        const int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        const int64_t page = slot / bs, row = slot % bs;
        for (int h = 0; h < Hkv; ++h) {
            const size_t dst = (((size_t)page * Hkv + h) * bs + row) * d;
            const size_t src = ((size_t)t * Hkv + h) * d;
            memcpy(k_cache + dst, k_new + src, sizeof(uint16_t) * d);
            memcpy(v_cache + dst, v_new + src, sizeof(uint16_t) * d);
        }
    }
    return 0;
}
