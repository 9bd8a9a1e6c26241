/*
 * synth.c - seeded synthetic inputs for the MoE layer forward.
 *
 * This is the one module that both the CPU oracle's tests and the CUDA path's
 * tests/bench draw their inputs from.  It holds none of the MoE arithmetic:
 * it only turns (seed, tensor id, element index) into numbers.
 *
 *   - Philox4x32-10, the counter-based generator of Salmon, Moraes, Dror and
 *     Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3" (SC'11): key =
 *     (seed, tensor id), counter = (block index lo, block index hi, 0, 0).
 *     Any slice of any tensor can be generated on its own.
 *   - Box-Muller (Box & Muller 1958) in double: one Philox block gives the two
 *     normals of elements 2b and 2b+1.
 *   - Storage rounding: value -> fp32 (round to nearest even) -> bf16 (round
 *     to nearest even), the same as torch's float->bfloat16 conversion.
 *
 * The skewed-routing workload (a Zipf(s) popularity over experts) is built by
 * shifting router rows and hidden states along one random unit vector u; the
 * per-expert shifts are calibrated here on a Gaussian model of the router
 * scores (synth_zipf_shift), never on the layer itself.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define PHILOX_M0 0xD2511F53u
#define PHILOX_M1 0xCD9E8D57u
#define PHILOX_W0 0x9E3779B9u
#define PHILOX_W1 0xBB67AE85u

void synth_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4]) {
    uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int r = 0; r < 10; ++r) {
        uint64_t p0 = (uint64_t)PHILOX_M0 * c0;
        uint64_t p1 = (uint64_t)PHILOX_M1 * c2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c1 ^ k0;
        uint32_t n1 = lo1;
        uint32_t n2 = hi0 ^ c3 ^ k1;
        uint32_t n3 = lo0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
        k0 += PHILOX_W0;
        k1 += PHILOX_W1;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* Two standard normals for Philox block `blk` of stream (seed, tid). */
static inline void normal_pair(uint32_t seed, uint32_t tid, uint64_t blk, double* z0, double* z1) {
    uint32_t ctr[4] = {(uint32_t)blk, (uint32_t)(blk >> 32), 0u, 0u};
    uint32_t key[2] = {seed, tid};
    uint32_t r[4];
    synth_philox4x32_10(ctr, key, r);
    uint64_t a = (((uint64_t)r[0] << 32) | r[1]) >> 11;     /* 53 bits */
    uint64_t b = (((uint64_t)r[2] << 32) | r[3]) >> 11;
    double u1 = ((double)a + 0.5) * 0x1.0p-53;                 /* (0,1) */
    double u2 = (double)b * 0x1.0p-53;                         /* [0,1) */
    double rad = sqrt(-2.0 * log(u1));
    double th = 6.283185307179586476925286766559 * u2;
    *z0 = rad * cos(th);
    *z1 = rad * sin(th);
}

/* One uniform in [0,1) for element i of stream (seed, tid): 53 bits of word pair i%2. */
static inline double uniform01(uint32_t seed, uint32_t tid, uint64_t i) {
    uint64_t blk = i >> 1;
    uint32_t ctr[4] = {(uint32_t)blk, (uint32_t)(blk >> 32), 0u, 0u};
    uint32_t key[2] = {seed, tid};
    uint32_t r[4];
    synth_philox4x32_10(ctr, key, r);
    uint64_t a = (i & 1) ? ((((uint64_t)r[2] << 32) | r[3]) >> 11) : ((((uint64_t)r[0] << 32) | r[1]) >> 11);
    return (double)a * 0x1.0p-53;
}

static inline uint16_t f32_to_bf16_rne(float f) {
    uint32_t bits;
    memcpy(&bits, &f, 4);
    uint32_t lsb = (bits >> 16) & 1u;
    bits += 0x7FFFu + lsb;
    return (uint16_t)(bits >> 16);
}

static inline double normal_at(uint32_t seed, uint32_t tid, uint64_t i) {
    double z0, z1;
    normal_pair(seed, tid, i >> 1, &z0, &z1);
    return (i & 1) ? z1 : z0;
}

/* out[i] = bf16(fp32(std * N_i)), i in [offset, offset+count) of stream (seed, tid). */
void synth_normal_bf16(uint32_t seed, uint32_t tid, uint64_t offset, uint64_t count, double stdv, uint16_t* out) {
    if (count == 0) return;
    uint64_t first_blk = offset >> 1, last_blk = (offset + count - 1) >> 1;
    int64_t nblk = (int64_t)(last_blk - first_blk + 1);
#pragma omp parallel for schedule(static)
    for (int64_t bb = 0; bb < nblk; ++bb) {
        uint64_t blk = first_blk + (uint64_t)bb;
        double z0, z1;
        normal_pair(seed, tid, blk, &z0, &z1);
        uint64_t i0 = blk * 2, i1 = i0 + 1;
        if (i0 >= offset && i0 < offset + count) out[i0 - offset] = f32_to_bf16_rne((float)(stdv * z0));
        if (i1 >= offset && i1 < offset + count) out[i1 - offset] = f32_to_bf16_rne((float)(stdv * z1));
    }
}

/* out[i] = N_i (double), the unrounded draws. */
void synth_normal_f64(uint32_t seed, uint32_t tid, uint64_t offset, uint64_t count, double* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)count; ++i) out[i] = normal_at(seed, tid, offset + (uint64_t)i);
}

/* out[i] = fp32(lo + (hi-lo) * U_i). */
void synth_uniform_f32(uint32_t seed, uint32_t tid, uint64_t offset, uint64_t count, double lo, double hi, float* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < (int64_t)count; ++i)
        out[i] = (float)(lo + (hi - lo) * uniform01(seed, tid, offset + (uint64_t)i));
}

/*
 * Shifted normal matrix, rows [row0, row0+nrows) of a [*, ncols] tensor:
 *   out[r, c] = bf16(fp32(std * N[r*ncols + c] + shift[r] * u[c]))
 * shift is indexed by absolute row (shift[row0 + r]); u has ncols entries.
 */
void synth_shifted_bf16(uint32_t seed, uint32_t tid, uint64_t row0, uint64_t nrows, uint64_t ncols, double stdv,
                        const double* shift, const double* u, uint16_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < (int64_t)nrows; ++r) {
        uint64_t row = row0 + (uint64_t)r;
        double sh = shift[row];
        for (uint64_t c = 0; c < ncols; ++c) {
            double v = stdv * normal_at(seed, tid, row * ncols + c) + sh * u[c];
            out[(uint64_t)r * ncols + c] = f32_to_bf16_rne((float)v);
        }
    }
}

/*
 * Per-expert shifts b_e that make the top-k popularity of a Gaussian model of
 * the router scores follow p*_e ~ (e+1)^(-s):
 *   score_e = nrm_e * g_e + off_e + b_e * (mu + s_t),  g ~ N(0, I), s_t ~ N(0,1)
 * where nrm_e is the norm of the unshifted router row e and off_e = mu * <row_e, u>
 * (both passed in).  Fixed point: b_e += 0.7 (ln p*_e - ln phat_e) / mu, `iters` times,
 * over `samples` model tokens drawn from streams tid_g / tid_s.
 */
void synth_zipf_shift(uint32_t seed, uint32_t tid_g, uint32_t tid_s, int E, int k, double s_exp, double mu,
                      const double* nrm, const double* off, int iters, int samples, double* b_out) {
    double* target = (double*)malloc(sizeof(double) * E);
    double* g = (double*)malloc(sizeof(double) * (size_t)samples * E);
    double* sv = (double*)malloc(sizeof(double) * samples);
    double tot = 0.0;
    for (int e = 0; e < E; ++e) { target[e] = pow((double)(e + 1), -s_exp); tot += target[e]; }
    for (int e = 0; e < E; ++e) { target[e] /= tot; b_out[e] = 0.0; }
    synth_normal_f64(seed, tid_g, 0, (uint64_t)samples * E, g);
    synth_normal_f64(seed, tid_s, 0, (uint64_t)samples, sv);
    long* cnt = (long*)malloc(sizeof(long) * E);
    for (int it = 0; it < iters; ++it) {
        memset(cnt, 0, sizeof(long) * E);
#pragma omp parallel
        {
            long* lc = (long*)calloc(E, sizeof(long));
            double* sc = (double*)malloc(sizeof(double) * E);
            unsigned char* used = (unsigned char*)malloc(E);
#pragma omp for schedule(static)
            for (int m = 0; m < samples; ++m) {
                for (int e = 0; e < E; ++e) sc[e] = nrm[e] * g[(size_t)m * E + e] + off[e] + b_out[e] * (mu + sv[m]);
                memset(used, 0, E);
                for (int j = 0; j < k; ++j) {
                    int best = -1;
                    for (int e = 0; e < E; ++e)
                        if (!used[e] && (best < 0 || sc[e] > sc[best])) best = e;
                    used[best] = 1;
                    lc[best]++;
                }
            }
#pragma omp critical
            for (int e = 0; e < E; ++e) cnt[e] += lc[e];
            free(lc); free(sc); free(used);
        }
        double denom = (double)samples * k;
        for (int e = 0; e < E; ++e) {
            double ph = (double)cnt[e] / denom;
            if (ph < 0.5 / denom) ph = 0.5 / denom;
            b_out[e] += 0.7 * (log(target[e]) - log(ph)) / mu;
        }
    }
    free(cnt); free(target); free(g); free(sv);
}

/*
 * fp8 e4m3 ("fn" variant: no infinities, max 448) quantisation of bf16 weight rows, one fp32
 * scale per row: s_r = max_i |w_ri| / 448 (1 for an all-zero row), q_ri = e4m3(w_ri / s_r)
 * rounded to nearest even.  This turns the synthetic bf16 checkpoint into the low-bit one;
 * the layer's arithmetic (dequantised weight = e4m3(q) * s) is defined elsewhere.
 */
static uint8_t f32_to_e4m3_rne(float v) {
    uint32_t bits;
    memcpy(&bits, &v, 4);
    uint8_t sign = (uint8_t)((bits >> 24) & 0x80u);
    float a = fabsf(v);
    if (a != a) return 0x7F;                        /* NaN */
    if (a >= 464.0f) return sign | 0x7E;            /* saturate to 448 */
    if (a < 0x1p-10f) return sign;                  /* below half the smallest subnormal (2^-9) */
    int ex;
    frexpf(a, &ex);                                 /* a = m * 2^ex, 0.5 <= m < 1 */
    int e = ex - 1;                                 /* a = 1.f * 2^e */
    if (e < -6) e = -6;                             /* subnormal range: quantum 2^-9 */
    float quantum = ldexpf(1.0f, e - 3);            /* 3 mantissa bits */
    float r = nearbyintf(a / quantum) * quantum;    /* ties to even (exact division by 2^k) */
    if (r >= 464.0f) return sign | 0x7E;
    if (r == 0.0f) return sign;
    int er;
    float mr = frexpf(r, &er);
    int E = er - 1;
    if (E < -6) {                                   /* subnormal: r = m * 2^-9, m in 1..7 */
        int m = (int)(r / 0x1p-9f);
        return sign | (uint8_t)m;
    }
    int mant = (int)((mr * 2.0f - 1.0f) * 8.0f + 0.5f);
    return sign | (uint8_t)(((E + 7) << 3) | mant);
}

void synth_quantize_e4m3_rows(const uint16_t* w, uint64_t rows, uint64_t K, uint8_t* q, float* scale) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < (int64_t)rows; ++r) {
        const uint16_t* wr = w + (uint64_t)r * K;
        float amax = 0.0f;
        for (uint64_t i = 0; i < K; ++i) {
            uint32_t b = (uint32_t)wr[i] << 16;
            float f;
            memcpy(&f, &b, 4);
            if (fabsf(f) > amax) amax = fabsf(f);
        }
        float s = amax > 0.0f ? amax / 448.0f : 1.0f;
        scale[r] = s;
        for (uint64_t i = 0; i < K; ++i) {
            uint32_t b = (uint32_t)wr[i] << 16;
            float f;
            memcpy(&f, &b, 4);
            q[(uint64_t)r * K + i] = f32_to_e4m3_rne(f / s);
        }
    }
}
