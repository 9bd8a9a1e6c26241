/*
 * moe_oracle.c - plain CPU oracle for the MoE layer forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
 * CPU-baseline leg load this library.  It shares no code, header, helper or
 * constant with the CUDA path; the product never calls it.
 *
 * What it computes, and where the pages define it (page titles abbreviated:
 *   [EP-KV]  "MoE 推理中的 Expert Parallel、KV Cache 与大规模专家并行架构解析"
 *   [EP-Ops] "MoE Expert Parallelism 实战：稀疏大模型推理的通信与负载均衡治理"
 *   [EP-DS3] "MoE 推理架构深度实战：从 Expert Parallelism 到 DeepSeek-V3 的工程落地"):
 *
 *   router logits   [EP-DS3] §2.1 code block (ProductionMoeRouter: gate = Linear(hidden, E, bias=False))
 *   softmax, top-k, renormalise  [EP-DS3] §2.1 code block, steps 1-3
 *   selection bias  [EP-DS3] §2.1 code block, step 4 comment ("add bias on logits"), used for selection only
 *   counts, capacity int(T/E*cf)  [EP-DS3] §2.1 code block (bincount, capacity) and get_expert_capacity
 *   token dropping  [EP-KV] §9 (capacity control), [EP-Ops] "常见误区" (token dropping)
 *   count/sort/pack by expert  [EP-KV] §8; [EP-DS3] §3.1 (sort by expert id)
 *   expert = FFN with SwiGLU gate  [EP-KV] §1 (FFN(x)=W2 σ(W1 x), SwiGLU adds a gate projection)
 *   weighted combine y = Σ g_i E_i(x)  [EP-KV] §2 (Top-2 example) and §7 (restore order + aggregate)
 *   shared expert   [EP-KV] §3 (routed + shared experts)
 *
 * Readings where the pages are silent (each stated in full here):
 *   - SwiGLU: E(x) = W2 (silu(W1 x) * (W3 x)), W1 = gate, W3 = up, silu(a) = a / (1 + e^-a).
 *   - Selection key = fp32(logit + bias); k largest keys, equal keys -> lower expert index,
 *     slots in descending key order.  Weights come from the unbiased softmax.
 *   - Capacity: per expert, the first C assignments in token order are kept; dropped
 *     slots contribute 0 and the kept weights are not renormalised again.
 *   - Shared expert output is added with weight 1 after the routed sum.
 *   - Rounding: products and sums in double; the stored tensors are rounded once
 *     where the layer stores them: logits -> fp32, routing weights -> fp32,
 *     H, Y_perm, Y_shared and out -> bf16 (round to nearest even).
 *
 * bf16 values are passed as uint16 bit patterns.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---- bf16 <-> double (oracle's own) ------------------------------------------------- */

static double bf(uint16_t h) {
    uint32_t bits = (uint32_t)h << 16;
    float f;
    memcpy(&f, &bits, 4);
    return (double)f;
}

/* Round a double to the nearest bf16 (8 significant bits), ties to even. */
static uint16_t bf16_round(double v) {
    if (v == 0.0 || !isfinite(v)) {
        float f = (float)v;
        uint32_t bits;
        memcpy(&bits, &f, 4);
        return (uint16_t)(bits >> 16);
    }
    int ex;
    double m = frexp(v, &ex);              /* v = m * 2^ex, 0.5 <= |m| < 1 */
    double r = nearbyint(ldexp(m, 8));     /* 8 significant bits, ties to even */
    float q = (float)ldexp(r, ex - 8);     /* exactly representable */
    uint32_t bits;
    memcpy(&bits, &q, 4);
    return (uint16_t)(bits >> 16);
}

uint16_t oracle_bf16_round(double v) { return bf16_round(v); }

/* ---- router ------------------------------------------------------------------------- */

/* logits[t,e] = fp32( sum_i x[t,i] * wg[e,i] ), summed in double. */
void oracle_router_logits(const uint16_t* x, const uint16_t* wg, int T, int d, int E, float* logits) {
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t)
        for (int e = 0; e < E; ++e) {
            double s = 0.0;
            for (int i = 0; i < d; ++i) s += bf(x[(size_t)t * d + i]) * bf(wg[(size_t)e * d + i]);
            logits[(size_t)t * E + e] = (float)s;
        }
}

typedef struct { float key; int e; } keyed_t;

/* key descending, then expert index ascending */
static int key_order(const void* a, const void* b) {
    const keyed_t* p = (const keyed_t*)a;
    const keyed_t* q = (const keyed_t*)b;
    if (p->key > q->key) return -1;
    if (p->key < q->key) return 1;
    return (p->e < q->e) ? -1 : (p->e > q->e);
}

/*
 * Softmax over all E logits, top-k on (logit + bias), renormalise the k weights.
 * idx[t, j] in descending key order; w[t, j] = p_idx / sum_sel p.
 * Returns 0, or -1 if a logit or key is not finite.
 */
int oracle_route(const float* logits, const float* bias, int T, int E, int k, int32_t* idx, float* w) {
    int bad = 0;
#pragma omp parallel
    {
        keyed_t* kv = (keyed_t*)malloc(sizeof(keyed_t) * E);
        double* p = (double*)malloc(sizeof(double) * E);
#pragma omp for schedule(static)
        for (int t = 0; t < T; ++t) {
            const float* L = logits + (size_t)t * E;
            double m = -INFINITY;
            for (int e = 0; e < E; ++e) {
                float key = L[e] + (bias ? bias[e] : 0.0f);   /* fp32 add */
                if (!isfinite(L[e]) || !isfinite(key)) bad = 1;
                kv[e].key = key;
                kv[e].e = e;
                if ((double)L[e] > m) m = (double)L[e];
            }
            /* softmax in double over all E (step 1) */
            double z = 0.0;
            for (int e = 0; e < E; ++e) { p[e] = exp((double)L[e] - m); z += p[e]; }
            for (int e = 0; e < E; ++e) p[e] /= z;
            /* top-k selection (step 2) */
            qsort(kv, E, sizeof(keyed_t), key_order);
            /* renormalise the k selected probabilities (step 3) */
            double s = 0.0;
            for (int j = 0; j < k; ++j) s += p[kv[j].e];
            for (int j = 0; j < k; ++j) {
                idx[(size_t)t * k + j] = kv[j].e;
                w[(size_t)t * k + j] = (float)(p[kv[j].e] / s);
            }
        }
        free(kv);
        free(p);
    }
    return bad ? -1 : 0;
}

/* ---- dispatch ----------------------------------------------------------------------- */

/* Capacity per expert; -1 = unlimited.  mode 1: int(T/E*cf) (the router's formula);
 * mode 2: int(T*k/E*cf) (per assignment).  Python's int() truncates toward zero. */
int64_t oracle_capacity(int T, int E, int k, double cf, int mode) {
    if (mode == 0) return -1;
    double tokens = (mode == 1) ? (double)T : (double)T * (double)k;
    double c = tokens / (double)E * cf;
    return (int64_t)c;
}

/*
 * Histogram, capacity in token order, offsets, stable permutation.
 *   counts_raw[e] = #{(t,j): idx[t,j] = e}
 *   kept in token order: walking t = 0..T-1, j = 0..k-1, an assignment to e is kept
 *   while fewer than C assignments to e have been kept.
 *   counts[e] = kept count, offsets = exclusive scan of counts (E+1 entries),
 *   dest[t,j] = offsets[e] + (position among e's kept assignments) or -1,
 *   src_token[dest] = t.
 * Returns N = offsets[E].
 */
int oracle_dispatch(const int32_t* idx, int T, int E, int k, int64_t C, int32_t* counts_raw, int32_t* counts,
                    int32_t* offsets, int32_t* dest, int32_t* src_token) {
    int64_t* fill = (int64_t*)calloc(E, sizeof(int64_t));
    for (int e = 0; e < E; ++e) { counts_raw[e] = 0; counts[e] = 0; }
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int e = idx[(size_t)t * k + j];
            counts_raw[e]++;
            if (C < 0 || fill[e] < C) { fill[e]++; counts[e]++; }
        }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    memset(fill, 0, sizeof(int64_t) * E);
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int e = idx[(size_t)t * k + j];
            if (fill[e] < counts[e]) {
                int r = offsets[e] + (int)fill[e];
                fill[e]++;
                dest[(size_t)t * k + j] = r;
                src_token[r] = t;
            } else {
                dest[(size_t)t * k + j] = -1;
            }
        }
    free(fill);
    return offsets[E];
}

/* x_perm[dest[t,j]] = x[t] for every kept assignment. */
void oracle_gather(const uint16_t* x, const int32_t* dest, int T, int d, int k, uint16_t* x_perm) {
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int r = dest[(size_t)t * k + j];
            if (r >= 0) memcpy(x_perm + (size_t)r * d, x + (size_t)t * d, sizeof(uint16_t) * d);
        }
}

/*
 * Overflow-driven selection bias ([EP-DS3] §2.1, the expert_bias update of the router code):
 *   overflow_e = counts_raw_e - C,  bias_e = -clamp(overflow_e / C, -1, 1)
 * computed in fp32 like the page's float tensors (the difference is exact; one division).
 * Sign: the page's comment says an overloaded expert's bias is set negative so that later
 * tokens avoid it; the formula it prints is positive for an overloaded expert.  The
 * stated intent is taken: the bias is the negated clamped overflow ratio.
 * Returns -1 for C <= 0 (no capacity: the update is undefined).
 */
int oracle_update_bias(const int32_t* counts_raw, int E, int64_t C, float* bias) {
    if (C <= 0) return -1;
    for (int e = 0; e < E; ++e) {
        float over = (float)((int64_t)counts_raw[e] - C);
        float r = over / (float)C;
        if (r > 1.0f) r = 1.0f;
        if (r < -1.0f) r = -1.0f;
        bias[e] = -r;
    }
    return 0;
}

/* ---- experts ------------------------------------------------------------------------ */

/*
 * One expert on `rows` rows: h = bf16( silu(x W1^T) * (x W3^T) ),  y = bf16( h W2^T ).
 * W1, W3: [f, d]; W2: [d, f]; x: [rows, d]; h: [rows, f]; y: [rows, d].
 */
void oracle_expert_ffn(const uint16_t* x, int rows, const uint16_t* W1, const uint16_t* W3, const uint16_t* W2,
                       int d, int f, uint16_t* h, uint16_t* y) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < rows; ++r) {
        const uint16_t* xr = x + (size_t)r * d;
        uint16_t* hr = h + (size_t)r * f;
        for (int n = 0; n < f; ++n) {
            double g = 0.0, u = 0.0;
            for (int i = 0; i < d; ++i) {
                double xi = bf(xr[i]);
                g += xi * bf(W1[(size_t)n * d + i]);
                u += xi * bf(W3[(size_t)n * d + i]);
            }
            double silu = g / (1.0 + exp(-g));
            hr[n] = bf16_round(silu * u);
        }
        for (int m = 0; m < d; ++m) {
            double s = 0.0;
            for (int n = 0; n < f; ++n) s += bf(hr[n]) * bf(W2[(size_t)m * f + n]);
            y[(size_t)r * d + m] = bf16_round(s);
        }
    }
}

/*
 * Low-bit expert weights (the "low-bit expert weights for decode" extension of the
 * deployment page's quantization option): each weight is one fp8 e4m3 byte q and each
 * output row n one fp32 scale s_n; the weight is e4m3(q) * s_n.
 *   e4m3 ("fn"): sign | 4 exponent bits (bias 7) | 3 mantissa bits; exponent 0 is subnormal
 *   (m * 2^-9); exponent 15 with mantissa 7 is NaN; no infinities.
 */
double oracle_e4m3(uint8_t b) {
    int sgn = b >> 7, e = (b >> 3) & 15, m = b & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return sgn ? -v : v;
}

/* oracle_expert_ffn with W1 = e4m3(W1q) * s1 (row scales [f]), W3 likewise, W2 = e4m3(W2q) * s2 ([d]). */
void oracle_expert_ffn_q8(const uint16_t* x, int rows, const uint8_t* W1q, const float* s1, const uint8_t* W3q,
                          const float* s3, const uint8_t* W2q, const float* s2, int d, int f, uint16_t* h, uint16_t* y) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < rows; ++r) {
        const uint16_t* xr = x + (size_t)r * d;
        uint16_t* hr = h + (size_t)r * f;
        for (int n = 0; n < f; ++n) {
            double g = 0.0, u = 0.0;
            for (int i = 0; i < d; ++i) {
                double xi = bf(xr[i]);
                g += xi * (oracle_e4m3(W1q[(size_t)n * d + i]) * (double)s1[n]);
                u += xi * (oracle_e4m3(W3q[(size_t)n * d + i]) * (double)s3[n]);
            }
            double silu = g / (1.0 + exp(-g));
            hr[n] = bf16_round(silu * u);
        }
        for (int m = 0; m < d; ++m) {
            double acc = 0.0;
            for (int n = 0; n < f; ++n) acc += bf(hr[n]) * (oracle_e4m3(W2q[(size_t)m * f + n]) * (double)s2[m]);
            y[(size_t)r * d + m] = bf16_round(acc);
        }
    }
}

/*
 * fp8 activations ("w4afp8" on the deployment page: low-bit weights with fp8 activations; here
 * fp8 weights and fp8 activations).  Every activation row (a token's hidden state before the
 * first expert GEMM, its h before the second) is quantised on its own:
 *   s = amax(|x|) / 448 in fp32 (1 for an all-zero row), q_i = e4m3(fp32(x_i) / s) rounded to
 *   nearest, ties to even, saturating at 448;
 * the expert GEMMs then multiply fp8 by fp8 and scale the sum by s_row * s_col.
 */

/* fp32 -> e4m3 ("fn") code by the format's definition: sign | 4 exponent bits (bias 7) | 3
 * mantissa bits, subnormals m * 2^-9, round to nearest even, values beyond 448 saturate to 448. */
uint8_t oracle_e4m3_encode(float v) {
    if (v != v) return 0x7F;
    uint8_t sgn = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    if (a >= 448.0) return sgn | 0x7E;
    /* candidates are multiples of the code spacing at a's binade: 2^-9 below 2^-6 */
    int e;
    frexp(a, &e);              /* a = f * 2^e, f in [0.5, 1) -> binade exponent e - 1 */
    int be = e - 1;
    if (be < -6) be = -6;      /* subnormal range shares the spacing of [2^-6, 2^-5) */
    double step = ldexp(1.0, be - 3);
    double k = a / step;       /* exact: a is an fp32 value, step a power of two */
    double kf = floor(k);
    double rem = k - kf;
    if (rem > 0.5 || (rem == 0.5 && fmod(kf, 2.0) != 0.0)) kf += 1.0;
    double r = kf * step;      /* the rounded magnitude */
    if (r >= 448.0) return sgn | 0x7E;
    if (r == 0.0) return sgn;
    /* encode r */
    if (r < ldexp(1.0, -6)) return sgn | (uint8_t)(int)(r / ldexp(1.0, -9));        /* subnormal */
    int re;
    double rf = frexp(r, &re);                 /* r = rf * 2^re, rf in [0.5, 1) */
    int ex = re - 1 + 7;
    int m = (int)((rf * 2.0 - 1.0) * 8.0);
    return sgn | (uint8_t)((ex << 3) | m);
}

/* bf16 rows [rows, K] -> e4m3 codes [rows, K] and one fp32 scale per row (see above). */
void oracle_quantize_rows_e4m3(const uint16_t* x, int rows, int K, uint8_t* q, float* scale) {
#pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; ++r) {
        const uint16_t* xr = x + (size_t)r * K;
        float amax = 0.0f;
        for (int i = 0; i < K; ++i) {
            float a = fabsf((float)bf(xr[i]));
            if (a > amax) amax = a;
        }
        float s = amax > 0.0f ? amax / 448.0f : 1.0f;
        scale[r] = s;
        for (int i = 0; i < K; ++i) q[(size_t)r * K + i] = oracle_e4m3_encode((float)bf(xr[i]) / s);
    }
}

/* First GEMM of an expert with fp8 weights and fp8 activations: x rows quantised,
 * G = s_x s1 (xq . W1q), U likewise, h = bf16(silu(G) U). */
void oracle_expert_gate_up_w8a8(const uint16_t* x, int rows, const uint8_t* W1q, const float* s1,
                                const uint8_t* W3q, const float* s3, int d, int f, uint16_t* h) {
    uint8_t* xq = (uint8_t*)malloc((size_t)(rows > 0 ? rows : 1) * d);
    float* sx = (float*)malloc(sizeof(float) * (size_t)(rows > 0 ? rows : 1));
    oracle_quantize_rows_e4m3(x, rows, d, xq, sx);
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < rows; ++r) {
        const uint8_t* xr = xq + (size_t)r * d;
        uint16_t* hr = h + (size_t)r * f;
        for (int n = 0; n < f; ++n) {
            double g = 0.0, u = 0.0;
            for (int i = 0; i < d; ++i) {
                double xi = oracle_e4m3(xr[i]);
                g += xi * oracle_e4m3(W1q[(size_t)n * d + i]);
                u += xi * oracle_e4m3(W3q[(size_t)n * d + i]);
            }
            g *= (double)sx[r] * (double)s1[n];
            u *= (double)sx[r] * (double)s3[n];
            hr[n] = bf16_round(g / (1.0 + exp(-g)) * u);
        }
    }
    free(xq); free(sx);
}

/* Second GEMM: h rows quantised, y = bf16(s_h s2 (hq . W2q)). */
void oracle_expert_down_w8a8(const uint16_t* h, int rows, const uint8_t* W2q, const float* s2, int d, int f,
                             uint16_t* y) {
    uint8_t* hq = (uint8_t*)malloc((size_t)(rows > 0 ? rows : 1) * f);
    float* sh = (float*)malloc(sizeof(float) * (size_t)(rows > 0 ? rows : 1));
    oracle_quantize_rows_e4m3(h, rows, f, hq, sh);
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < rows; ++r) {
        const uint8_t* hr = hq + (size_t)r * f;
        for (int m = 0; m < d; ++m) {
            double acc = 0.0;
            for (int n = 0; n < f; ++n) acc += oracle_e4m3(hr[n]) * oracle_e4m3(W2q[(size_t)m * f + n]);
            y[(size_t)r * d + m] = bf16_round(acc * (double)sh[r] * (double)s2[m]);
        }
    }
    free(hq); free(sh);
}

/* One expert with fp8 weights (row scales s1, s3, s2) and fp8 activations: the two GEMMs above. */
void oracle_expert_ffn_w8a8(const uint16_t* x, int rows, const uint8_t* W1q, const float* s1, const uint8_t* W3q,
                            const float* s3, const uint8_t* W2q, const float* s2, int d, int f, uint16_t* h,
                            uint16_t* y) {
    oracle_expert_gate_up_w8a8(x, rows, W1q, s1, W3q, s3, d, f, h);
    oracle_expert_down_w8a8(h, rows, W2q, s2, d, f, y);
}

/* ---- combine ------------------------------------------------------------------------ */

/*
 * out[t] = bf16( sum_{j: dest>=0} w[t,j] * y_perm[dest[t,j]]  (+ y_shared[t]) ),
 * j in order 0..k-1, the shared expert added last with weight 1.
 */
void oracle_combine(const uint16_t* y_perm, const int32_t* dest, const float* w, const uint16_t* y_shared,
                    int T, int d, int k, uint16_t* out) {
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t)
        for (int m = 0; m < d; ++m) {
            double acc = 0.0;
            for (int j = 0; j < k; ++j) {
                int r = dest[(size_t)t * k + j];
                if (r >= 0) acc += (double)w[(size_t)t * k + j] * bf(y_perm[(size_t)r * d + m]);
            }
            if (y_shared) acc += bf(y_shared[(size_t)t * d + m]);
            out[(size_t)t * d + m] = bf16_round(acc);
        }
}

/* ---- whole layer -------------------------------------------------------------------- */

/*
 * Router -> dispatch -> experts (+ shared) -> combine.
 * logits_in (nullable): route these instead of computing the router GEMM.
 * Every output pointer except `out` may be NULL.  Scratch is allocated here.
 * Returns N (kept assignments) or -1 on non-finite routing input.
 */
int oracle_layer_forward(const uint16_t* x, const uint16_t* wg, const float* bias, const float* logits_in,
                         const uint16_t* W1, const uint16_t* W3, const uint16_t* W2,
                         const uint16_t* W1s, const uint16_t* W3s, const uint16_t* W2s, int f_shared,
                         int T, int d, int E, int k, int f, int64_t C,
                         uint16_t* out, float* logits_out, int32_t* idx_out, float* w_out,
                         int32_t* counts_raw_out, int32_t* counts_out, int32_t* offsets_out,
                         int32_t* dest_out, int32_t* src_out, uint16_t* y_shared_out) {
    size_t Tk = (size_t)T * k;
    float* logits = (float*)malloc(sizeof(float) * (size_t)T * E);
    int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * Tk);
    float* w = (float*)malloc(sizeof(float) * Tk);
    int32_t* craw = (int32_t*)malloc(sizeof(int32_t) * E);
    int32_t* cnt = (int32_t*)malloc(sizeof(int32_t) * E);
    int32_t* off = (int32_t*)malloc(sizeof(int32_t) * (E + 1));
    int32_t* dest = (int32_t*)malloc(sizeof(int32_t) * Tk);
    int32_t* src = (int32_t*)malloc(sizeof(int32_t) * (Tk ? Tk : 1));
    if (logits_in) memcpy(logits, logits_in, sizeof(float) * (size_t)T * E);
    else oracle_router_logits(x, wg, T, d, E, logits);
    int rc = oracle_route(logits, bias, T, E, k, idx, w);
    int N = oracle_dispatch(idx, T, E, k, C, craw, cnt, off, dest, src);
    uint16_t* xp = (uint16_t*)malloc(sizeof(uint16_t) * ((size_t)N * d + 1));
    uint16_t* hp = (uint16_t*)malloc(sizeof(uint16_t) * ((size_t)N * f + 1));
    uint16_t* yp = (uint16_t*)malloc(sizeof(uint16_t) * ((size_t)N * d + 1));
    oracle_gather(x, dest, T, d, k, xp);
    for (int e = 0; e < E; ++e) {
        int r0 = off[e], n = cnt[e];
        if (n == 0) continue;
        oracle_expert_ffn(xp + (size_t)r0 * d, n, W1 + (size_t)e * f * d, W3 + (size_t)e * f * d,
                          W2 + (size_t)e * d * f, d, f, hp + (size_t)r0 * f, yp + (size_t)r0 * d);
    }
    uint16_t* ysh = NULL;
    if (W1s && W3s && W2s && f_shared > 0) {
        ysh = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)T * d);
        uint16_t* hs = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)T * f_shared);
        oracle_expert_ffn(x, T, W1s, W3s, W2s, d, f_shared, hs, ysh);
        free(hs);
    }
    oracle_combine(yp, dest, w, ysh, T, d, k, out);
    if (logits_out) memcpy(logits_out, logits, sizeof(float) * (size_t)T * E);
    if (idx_out) memcpy(idx_out, idx, sizeof(int32_t) * Tk);
    if (w_out) memcpy(w_out, w, sizeof(float) * Tk);
    if (counts_raw_out) memcpy(counts_raw_out, craw, sizeof(int32_t) * E);
    if (counts_out) memcpy(counts_out, cnt, sizeof(int32_t) * E);
    if (offsets_out) memcpy(offsets_out, off, sizeof(int32_t) * (E + 1));
    if (dest_out) memcpy(dest_out, dest, sizeof(int32_t) * Tk);
    if (src_out) memcpy(src_out, src, sizeof(int32_t) * (size_t)N);
    if (y_shared_out && ysh) memcpy(y_shared_out, ysh, sizeof(uint16_t) * (size_t)T * d);
    free(logits); free(idx); free(w); free(craw); free(cnt); free(off); free(dest); free(src);
    free(xp); free(hp); free(yp); free(ysh);
    return rc < 0 ? -1 : N;
}
