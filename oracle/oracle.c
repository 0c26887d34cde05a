/*
 * CPU oracle for the ExpertsInt8 mixture-of-experts layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, plain, obviously correct
 * statement of what the layer computes.  Only the tests, the smoke check and
 * the benchmark's CPU-baseline leg may load it; the product (the C-ABI
 * library and its Python binding) never calls it, and it shares no code,
 * header, table or helper with the CUDA path.
 *
 * Sources (web pages on the method; cited by page title and section):
 *  [J15]  "Jamba-1.5: Hybrid Transformer-Mamba Models at Scale" (paper summary,
 *         arXiv 2408.12570), section "ExpertsInt8 Quantization (Section 3.1)",
 *         steps 1-4, and section "The Jamba Hybrid Block Structure" (the MoE
 *         equation MoE(x) = sum over TopK(x,2) of g_i(x) * Expert_i(x)).
 *  [J1]   "Jamba: A Hybrid Transformer-Mamba Language Model" (paper summary,
 *         arXiv 2403.19887), section "Mixture-of-Experts (MoE) in Jamba:
 *         Router, Top-K, and Load Balancing": g = softmax(W_r h), top-K
 *         selection, y = sum over the selected set of g_i * Expert_i(h) with
 *         g renormalised over the selected set; and the layer list (experts
 *         are MLPs with SwiGLU activation).
 *
 * Readings where the pages leave a step open:
 *  - quantisation is symmetric, per output row (output channel), with
 *    scale s = absmax/127 computed as one fp32 division, q = round-half-even
 *    of the fp32 quotient w/s, clamped to [-127, 127]; an all-zero row gets
 *    s = 0 and q = 0.  [J15 step 1 says only "calibration-free"; the section's
 *    "presumably symmetric ... absolute maximum" remark.]
 *  - the dequantised weight is the exact product q*s (fp64 here); the
 *    pages' "scaling and casting" to BF16 is a storage detail of the kernel.
 *  - router logits are fp64 dot products summed in one canonical order
 *    (32 interleaved partial sums, then a halving tree), rounded once to
 *    fp32 after adding an optional per-expert bias; top-k is chosen on those
 *    fp32 logits, ties to the lower expert index.
 *  - gates: fp64 softmax over all experts, renormalised over the selected set.
 *  - SwiGLU: the first d_ff rows of the gate/up matrix are the gate (silu
 *    applied), the next d_ff rows the up projection; silu(z) = z/(1+e^-z).
 *
 * Everything else is fp64 with no intermediate rounding, so the oracle sits
 * within rounding of the real-number definition.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static float bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Round an fp64 value once, to nearest with ties to even, to the nearest     */
/* bfloat16 (8 significant bits; fp32's exponent range, subnormals down to    */
/* 2^-133); returns the bf16 bit pattern.  Scaling by powers of two and rint  */
/* (ties to even in the default mode) are exact, so there is one rounding.    */
static uint16_t f64_to_bf16_bits(double v) {
    if (v != v) return 0x7fc0u;
    const uint16_t sign = signbit(v) ? 0x8000u : 0u;
    double a = fabs(v);
    double r;
    if (a < ldexp(1.0, -126)) {
        r = rint(a * ldexp(1.0, 133)) * ldexp(1.0, -133);
    } else {
        int e;
        frexp(a, &e); /* a = m * 2^e, m in [0.5, 1) */
        const double q = ldexp(1.0, e - 8);
        r = rint(a / q) * q;
    }
    if (r >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7f80u);
    float f = (float)r; /* exact: r has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, 4);
    return (uint16_t)(sign | (uint16_t)((u >> 16) & 0x7fffu));
}

/* ------------------------------------------------------------------------ */
/* RMSNorm ahead of the router (the pages: RMSNorm precedes the modules of   */
/* a Jamba block).  Plain reading, with every rounding fixed so the routing   */
/* that follows is reproducible bit for bit:                                  */
/*   ss = sum of x_k^2 in fp64 in the canonical order of the router (lane j   */
/*        of 32 sums k = j mod 32 ascending, then the halving tree; squares   */
/*        of bf16 values are exact in fp64),                                  */
/*   r  = 1 / sqrt(ss / d + eps)  (fp64, correctly rounded sqrt and divides), */
/*   y_k = bf16( (x_k * r) * gamma_k )  (fp64 products, one rounding).        */
void oracle_rmsnorm(const uint16_t* x_bf16, int64_t T, int64_t d, const uint16_t* gamma_bf16,
                    float eps, uint16_t* y_bf16) {
    for (int64_t t = 0; t < T; ++t) {
        const uint16_t* x = x_bf16 + t * d;
        double p[32];
        for (int j = 0; j < 32; ++j) {
            p[j] = 0.0;
            for (int64_t k = j; k < d; k += 32) {
                const double v = (double)bf16_to_f32(x[k]);
                p[j] += v * v;
            }
        }
        for (int o = 16; o >= 1; o /= 2)
            for (int j = 0; j < o; ++j) p[j] = p[j] + p[j + o];
        const double r = 1.0 / sqrt(p[0] / (double)d + (double)eps);
        for (int64_t k = 0; k < d; ++k)
            y_bf16[t * d + k] = f64_to_bf16_bits(((double)bf16_to_f32(x[k]) * r) *
                                                 (double)bf16_to_f32(gamma_bf16[k]));
    }
}

/* ------------------------------------------------------------------------ */
/* Step 1 of [J15]: BF16 weights -> INT8 + one fp32 scale per output row.    */
/* w_bf16 is row-major [rows][cols]; a row is one output channel.           */
void oracle_quantize(const uint16_t* w_bf16, int64_t rows, int64_t cols, int8_t* q,
                     float* scales) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const uint16_t* w = w_bf16 + r * cols;
        float amax = 0.0f;
        for (int64_t k = 0; k < cols; ++k) {
            float a = fabsf(bf16_to_f32(w[k]));
            if (a > amax) amax = a;
        }
        if (amax == 0.0f) {
            scales[r] = 0.0f;
            memset(q + r * cols, 0, (size_t)cols);
            continue;
        }
        float s = amax / 127.0f; /* one IEEE fp32 division */
        scales[r] = s;
        for (int64_t k = 0; k < cols; ++k) {
            float v = rintf(bf16_to_f32(w[k]) / s); /* half-to-even in the default mode */
            if (v > 127.0f) v = 127.0f;
            if (v < -127.0f) v = -127.0f;
            q[r * cols + k] = (int8_t)v;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Router logits l = W_r h of [J1] (plus an optional bias per expert).      */
/* Canonical fp64 order: p_j = sum over k = j, j+32, j+64, ... ascending of  */
/* x_k * w_ek (j = 0..31); then p_j += p_{j+o} for o = 16, 8, 4, 2, 1 and    */
/* j < o; the logit is fp32(p_0 + bias_e).  Every product x_k * w_ek is      */
/* exact in fp64 (8-bit by 24-bit significands).                            */
void oracle_router_logits(const uint16_t* x_bf16, int64_t T, int64_t d, const float* w_router,
                          int E, const float* bias_or_null, float* logits) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const uint16_t* x = x_bf16 + t * d;
        for (int e = 0; e < E; ++e) {
            const float* w = w_router + (int64_t)e * d;
            double p[32];
            for (int j = 0; j < 32; ++j) {
                p[j] = 0.0;
                for (int64_t k = j; k < d; k += 32) p[j] += (double)bf16_to_f32(x[k]) * (double)w[k];
            }
            for (int o = 16; o >= 1; o /= 2)
                for (int j = 0; j < o; ++j) p[j] = p[j] + p[j + o];
            double b = bias_or_null ? (double)bias_or_null[e] : 0.0;
            logits[t * E + e] = (float)(p[0] + b);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Top-k selection of [J1] and its gates.                                   */
/* ids[t][j] is the j-th selected expert (largest logit first; among equal  */
/* logits the smaller index first).  With renorm != 0 ([J1]: renormalised   */
/* over the selected set) gates[t][j] = p_{ids[t][j]} / sum over the        */
/* selected set of p; with renorm == 0 (the plain reading of [J15]'s        */
/* "softmax-normalized" gates) gates[t][j] = p_{ids[t][j]}; p = softmax over */
/* all E logits (fp64).                                                      */
int oracle_topk_gates_mode(const float* logits, int64_t T, int E, int top_k, int renorm,
                           int32_t* ids, double* gates) {
    if (E < 1 || E > 64 || top_k < 1 || top_k > E) return 1;
    for (int64_t t = 0; t < T; ++t) {
        const float* l = logits + t * E;
        int chosen[64];
        for (int j = 0; j < top_k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                int taken = 0;
                for (int i = 0; i < j; ++i)
                    if (chosen[i] == e) taken = 1;
                if (taken) continue;
                if (best < 0 || l[e] > l[best]) best = e; /* strict: ties keep the lower index */
            }
            chosen[j] = best;
            ids[t * top_k + j] = best;
        }
        double m = -INFINITY;
        for (int e = 0; e < E; ++e)
            if ((double)l[e] > m) m = (double)l[e];
        double z = 0.0;
        double p[64];
        for (int e = 0; e < E; ++e) {
            p[e] = exp((double)l[e] - m);
            z += p[e];
        }
        for (int e = 0; e < E; ++e) p[e] /= z;
        double sel = 0.0;
        for (int j = 0; j < top_k; ++j) sel += p[chosen[j]];
        for (int j = 0; j < top_k; ++j)
            gates[t * top_k + j] = renorm ? p[chosen[j]] / sel : p[chosen[j]];
    }
    return 0;
}

int oracle_topk_gates(const float* logits, int64_t T, int E, int top_k, int32_t* ids,
                      double* gates) {
    return oracle_topk_gates_mode(logits, T, E, top_k, 1, ids, gates);
}

/* ------------------------------------------------------------------------ */
/* Grouping of token assignments by expert (the dispatch that the fused MoE  */
/* kernel of [J15] performs).  Assignment a = t*top_k + j goes to expert     */
/* ids[a].  Stable counting sort: perm lists the assignments of expert 0 in  */
/* ascending a, then expert 1, ...; offsets[e] is the start of expert e's    */
/* run (offsets[E] = T*top_k); inv[perm[i]] = i.                            */
void oracle_permute(const int32_t* ids, int64_t T, int top_k, int E, int32_t* offsets,
                    int32_t* perm, int32_t* inv) {
    int64_t A = T * top_k;
    for (int e = 0; e <= E; ++e) offsets[e] = 0;
    for (int64_t a = 0; a < A; ++a) offsets[ids[a] + 1] += 1;
    for (int e = 0; e < E; ++e) offsets[e + 1] += offsets[e];
    int32_t* next = (int32_t*)malloc(sizeof(int32_t) * (size_t)(E > 0 ? E : 1));
    for (int e = 0; e < E; ++e) next[e] = offsets[e];
    for (int64_t a = 0; a < A; ++a) {
        int32_t pos = next[ids[a]]++;
        perm[pos] = (int32_t)a;
        inv[a] = pos;
    }
    free(next);
}

/* ------------------------------------------------------------------------ */
/* One expert (a SwiGLU MLP, [J1]) on one token, with the INT8 weights       */
/* dequantised as w = q * s (step 3 of [J15]) and BF16 activations (step 4). */
/*   u_n = sum_k x_k * (q_gu[n][k] * s_gu[n])         n < 2 d_ff             */
/*   h_n = silu(u_n) * u_{d_ff + n}                    n < d_ff               */
/*   y_m = sum_n h_n * (q_d[m][n] * s_d[m])           m < d_model            */
static void expert_ffn(const uint16_t* x, int64_t d, int64_t f, const int8_t* q_gu,
                       const float* s_gu, const int8_t* q_d, const float* s_d, double* u,
                       double* h, double* y) {
    double* xd = (double*)malloc(sizeof(double) * (size_t)d);
    for (int64_t k = 0; k < d; ++k) xd[k] = (double)bf16_to_f32(x[k]);
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < 2 * f; ++n) {
        const int8_t* qr = q_gu + n * d;
        double acc = 0.0;
        for (int64_t k = 0; k < d; ++k) acc += xd[k] * ((double)qr[k] * (double)s_gu[n]);
        u[n] = acc;
    }
    for (int64_t n = 0; n < f; ++n) {
        double g = u[n];
        double silu = g / (1.0 + exp(-g));
        h[n] = silu * u[f + n];
    }
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < d; ++m) {
        const int8_t* qr = q_d + m * f;
        double acc = 0.0;
        for (int64_t n = 0; n < f; ++n) acc += h[n] * ((double)qr[n] * (double)s_d[m]);
        y[m] = acc;
    }
    free(xd);
}

/* ------------------------------------------------------------------------ */
/* The MoE layer output of [J15]/[J1]:  out_t = sum_j gates[t][j] *          */
/* Expert_{ids[t][j]}(x_t).  Per-expert weights are passed as pointer tables */
/* (an entry may be NULL for an expert no token selects).                   */
int oracle_moe_forward(const uint16_t* x_bf16, int64_t T, int64_t d, int64_t f, int E,
                       int top_k, const int32_t* ids, const double* gates,
                       const int8_t* const* q_gu, const float* const* s_gu,
                       const int8_t* const* q_d, const float* const* s_d, double* out) {
    double* u = (double*)malloc(sizeof(double) * (size_t)(2 * f));
    double* h = (double*)malloc(sizeof(double) * (size_t)f);
    double* y = (double*)malloc(sizeof(double) * (size_t)d);
    int rc = 0;
    for (int64_t t = 0; t < T && rc == 0; ++t) {
        for (int64_t m = 0; m < d; ++m) out[t * d + m] = 0.0;
        for (int j = 0; j < top_k; ++j) {
            int e = ids[t * top_k + j];
            if (e < 0 || e >= E || !q_gu[e] || !s_gu[e] || !q_d[e] || !s_d[e]) {
                rc = 1;
                break;
            }
            expert_ffn(x_bf16 + t * d, d, f, q_gu[e], s_gu[e], q_d[e], s_d[e], u, h, y);
            double g = gates[t * top_k + j];
            for (int64_t m = 0; m < d; ++m) out[t * d + m] += g * y[m];
        }
    }
    free(u);
    free(h);
    free(y);
    return rc;
}

/* The dense MLP of [J15] step 1 ("MoE and MLP weights" are quantised): one  */
/* SwiGLU MLP applied to every token, out_t = Expert(x_t).                  */
void oracle_mlp_forward(const uint16_t* x_bf16, int64_t T, int64_t d, int64_t f,
                        const int8_t* q_gu, const float* s_gu, const int8_t* q_d, const float* s_d,
                        double* out) {
    double* u = (double*)malloc(sizeof(double) * (size_t)(2 * f));
    double* h = (double*)malloc(sizeof(double) * (size_t)f);
    for (int64_t t = 0; t < T; ++t)
        expert_ffn(x_bf16 + t * d, d, f, q_gu, s_gu, q_d, s_d, u, h, out + t * d);
    free(u);
    free(h);
}
