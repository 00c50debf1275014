/*
 * FP64 CPU oracle for the Gated DeltaNet (GDN) decode step.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check in __graft_entry__
 * and bench.py's CPU-baseline leg load this library. The CUDA product path never
 * does, and this file shares no code, header or constant table with it.
 *
 * Source of the method: the page "spark_model/forward/qwen3_5/linear_attention.rs"
 * (Atlas, single-token GDN decode layer), steps 3 to 8 and the SiLU(z) gate of the
 * fused steps 9+10+11, together with the gated delta rule it launches in step 7:
 *
 *   g = -exp(A_log) * softplus(a + dt_bias),  beta = sigmoid(b)
 *   S <- exp(g) * S;   S <- S + beta * k (v - S^T k)^T;   o = S^T q
 *
 * Every intermediate is a double. Inputs arrive as the exact bit patterns the GPU
 * receives (bf16 as uint16, fp32 as float) and are widened exactly. Each function
 * takes the steps in the order the method states them; nothing is fused, blocked
 * or reordered.
 *
 * Layouts (row-major, innermost last):
 *   qkv        [B][T][C] bf16, C = 2*Hk*dk + Hv*dv, channels Q | K | V, head-major
 *   conv_w     [C][W]    bf16, tap W-1 multiplies the current token
 *   conv_pool  [P][W-1][C] bf16, row 0 the oldest raw input
 *   state_pool [P][Hv][dk][dv] double
 *   a, b       [B][T][Hv] bf16;  A_log, dt_bias [Hv] fp32
 *   z          [B][T][Hv][dv] bf16;  norm_w [dv] bf16
 *   q, k       [B][T][Hk][dk];  v, o, out [B][T][Hv][dv];  alpha, beta [B][T][Hv]
 * v-head h reads k-head h / (Hv/Hk).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int num_k_heads, num_v_heads, head_k_dim, head_v_dim, conv_width;
    double l2_eps;   /* inside the root of the q/k L2 norm */
    double rms_eps;  /* inside the root of the output RMSNorm */
    double q_scale;  /* factor on the normalised q; 0 selects 1/sqrt(head_k_dim) */
} oracle_cfg;

static double from_bf16(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double silu(double x) { return x / (1.0 + exp(-x)); }
static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }
/* log(1 + e^x), written so that it neither overflows nor loses the small tail. */
static double softplus(double x) { return (x > 0.0 ? x : 0.0) + log1p(exp(-fabs(x))); }

static int channels(const oracle_cfg* c) {
    return 2 * c->num_k_heads * c->head_k_dim + c->num_v_heads * c->head_v_dim;
}

/*
 * Step 3, "fused causal_conv1d_update_l2norm" (+ the 1/sqrt(d_k) q scale noted
 * after it): per channel, a depthwise causal convolution of width W over the
 * W-1 stored raw inputs followed by this launch's T raw inputs, no bias; SiLU on
 * every channel; then an L2 norm over each Q head and each K head (eps inside
 * the root); V keeps the SiLU output. Step 6 splits the result Q | K | V.
 * Afterwards the slot's history holds the last W-1 raw inputs (a bit copy).
 */
void oracle_conv_update(const oracle_cfg* c, int B, int T, const uint16_t* qkv,
                        const uint16_t* conv_w, uint16_t* conv_pool, int pool_slots,
                        const int32_t* slots, double* q, double* k, double* v) {
    const int Hk = c->num_k_heads, Hv = c->num_v_heads, dk = c->head_k_dim, dv = c->head_v_dim;
    const int W = c->conv_width, C = channels(c);
    const double qs = c->q_scale != 0.0 ? c->q_scale : 1.0 / sqrt((double)dk);
    double* s = (double*)malloc(sizeof(double) * (size_t)T * C);
    uint16_t* hist = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(W - 1 + T));
    (void)pool_slots;
    for (int b = 0; b < B; ++b) {
        uint16_t* st = conv_pool + (size_t)slots[b] * (W - 1) * C;
        for (int ch = 0; ch < C; ++ch) {
            /* the raw sequence for this channel: W-1 history rows, then the T new inputs */
            for (int r = 0; r < W - 1; ++r) hist[r] = st[(size_t)r * C + ch];
            for (int t = 0; t < T; ++t) hist[W - 1 + t] = qkv[((size_t)b * T + t) * C + ch];
            for (int t = 0; t < T; ++t) {
                double u = 0.0;
                for (int j = 0; j < W; ++j)
                    u += from_bf16(conv_w[(size_t)ch * W + j]) * from_bf16(hist[t + j]);
                s[(size_t)t * C + ch] = silu(u);
            }
            for (int r = 0; r < W - 1; ++r) st[(size_t)r * C + ch] = hist[T + r];
        }
        for (int t = 0; t < T; ++t) {
            const double* st_q = s + (size_t)t * C;
            const double* st_k = st_q + Hk * dk;
            const double* st_v = st_q + 2 * Hk * dk;
            for (int h = 0; h < Hk; ++h) {
                double sq = 0.0, sk = 0.0;
                for (int i = 0; i < dk; ++i) {
                    sq += st_q[h * dk + i] * st_q[h * dk + i];
                    sk += st_k[h * dk + i] * st_k[h * dk + i];
                }
                const double nq = 1.0 / sqrt(sq + c->l2_eps), nk = 1.0 / sqrt(sk + c->l2_eps);
                for (int i = 0; i < dk; ++i) {
                    q[(((size_t)b * T + t) * Hk + h) * dk + i] = st_q[h * dk + i] * nq * qs;
                    k[(((size_t)b * T + t) * Hk + h) * dk + i] = st_k[h * dk + i] * nk;
                }
            }
            for (int h = 0; h < Hv; ++h)
                for (int j = 0; j < dv; ++j)
                    v[(((size_t)b * T + t) * Hv + h) * dv + j] = st_v[h * dv + j];
        }
    }
    free(hist);
    free(s);
}

/*
 * Steps 4 and 5: gate = exp(softplus(a + dt_bias) * -exp(A_log)) and
 * beta = sigmoid(b), per (row, v-head); rows = B*T.
 */
void oracle_gate(const oracle_cfg* c, int rows, const uint16_t* a, const uint16_t* b,
                 const float* A_log, const float* dt_bias, double* alpha, double* beta) {
    const int Hv = c->num_v_heads;
    for (int r = 0; r < rows; ++r)
        for (int h = 0; h < Hv; ++h) {
            const size_t i = (size_t)r * Hv + h;
            const double g = -exp((double)A_log[h]) * softplus(from_bf16(a[i]) + (double)dt_bias[h]);
            alpha[i] = exp(g);
            beta[i] = sigmoid(from_bf16(b[i]));
        }
}

/*
 * Step 7, "gated_delta_rule_decode": for each sequence, token (in order) and
 * v-head h, with k-head h / (Hv/Hk):
 *   S <- alpha S;  m = S^T k;  delta = beta (v - m);  S <- S + k delta^T;  o = S^T q.
 * S is [dk][dv]; S^T k has length dv.
 */
void oracle_delta_rule(const oracle_cfg* c, int B, int T, const double* q, const double* k,
                       const double* v, const double* alpha, const double* beta,
                       double* state_pool, int pool_slots, const int32_t* slots, double* o) {
    const int Hk = c->num_k_heads, Hv = c->num_v_heads, dk = c->head_k_dim, dv = c->head_v_dim;
    const int G = Hv / Hk;
    double* m = (double*)malloc(sizeof(double) * dv);
    double* d = (double*)malloc(sizeof(double) * dv);
    (void)pool_slots;
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t)
            for (int h = 0; h < Hv; ++h) {
                const size_t row = (size_t)b * T + t;
                const double* kk = k + (row * Hk + h / G) * dk;
                const double* qq = q + (row * Hk + h / G) * dk;
                const double* vv = v + (row * Hv + h) * dv;
                const double al = alpha[row * Hv + h], be = beta[row * Hv + h];
                double* S = state_pool + ((size_t)slots[b] * Hv + h) * dk * dv;
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) S[i * dv + j] *= al;
                for (int j = 0; j < dv; ++j) {
                    m[j] = 0.0;
                    for (int i = 0; i < dk; ++i) m[j] += S[i * dv + j] * kk[i];
                }
                for (int j = 0; j < dv; ++j) d[j] = be * (vv[j] - m[j]);
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) S[i * dv + j] += kk[i] * d[j];
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < dk; ++i) acc += S[i * dv + j] * qq[i];
                    o[(row * Hv + h) * dv + j] = acc;
                }
            }
    free(d);
    free(m);
}

/*
 * The same step written as one matrix map, S' = alpha (I - beta k k^T) S + beta k v^T,
 * o = S'^T q: an independent second form kept only to cross-check the first.
 */
void oracle_delta_rule_matrix_form(const oracle_cfg* c, int B, int T, const double* q,
                                   const double* k, const double* v, const double* alpha,
                                   const double* beta, double* state_pool, int pool_slots,
                                   const int32_t* slots, double* o) {
    const int Hk = c->num_k_heads, Hv = c->num_v_heads, dk = c->head_k_dim, dv = c->head_v_dim;
    const int G = Hv / Hk;
    double* M = (double*)malloc(sizeof(double) * dk * dk);
    double* Sn = (double*)malloc(sizeof(double) * dk * dv);
    (void)pool_slots;
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t)
            for (int h = 0; h < Hv; ++h) {
                const size_t row = (size_t)b * T + t;
                const double* kk = k + (row * Hk + h / G) * dk;
                const double* qq = q + (row * Hk + h / G) * dk;
                const double* vv = v + (row * Hv + h) * dv;
                const double al = alpha[row * Hv + h], be = beta[row * Hv + h];
                double* S = state_pool + ((size_t)slots[b] * Hv + h) * dk * dv;
                for (int i = 0; i < dk; ++i)
                    for (int l = 0; l < dk; ++l) M[i * dk + l] = (i == l ? 1.0 : 0.0) - be * kk[i] * kk[l];
                for (int i = 0; i < dk; ++i)
                    for (int j = 0; j < dv; ++j) {
                        double acc = 0.0;
                        for (int l = 0; l < dk; ++l) acc += M[i * dk + l] * S[l * dv + j];
                        Sn[i * dv + j] = al * acc + be * kk[i] * vv[j];
                    }
                memcpy(S, Sn, sizeof(double) * dk * dv);
                for (int j = 0; j < dv; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < dk; ++i) acc += S[i * dv + j] * qq[i];
                    o[(row * Hv + h) * dv + j] = acc;
                }
            }
    free(Sn);
    free(M);
}

/*
 * Step 8 and the gate of steps 9+10+11: per v-head row of dv values,
 * y = o / sqrt(mean(o^2) + eps) * norm_w, then out = y * silu(z).
 */
void oracle_gated_rmsnorm(const oracle_cfg* c, int rows, const double* o, const uint16_t* z,
                          const uint16_t* norm_w, double* out) {
    const int dv = c->head_v_dim;
    for (int r = 0; r < rows; ++r) {
        double ss = 0.0;
        for (int j = 0; j < dv; ++j) ss += o[(size_t)r * dv + j] * o[(size_t)r * dv + j];
        const double inv = 1.0 / sqrt(ss / dv + c->rms_eps);
        for (int j = 0; j < dv; ++j) {
            const size_t i = (size_t)r * dv + j;
            out[i] = o[i] * inv * from_bf16(norm_w[j]) * silu(from_bf16(z[i]));
        }
    }
}

/*
 * One decode launch: the stages above in the page's order. The optional
 * intermediates (q, k, v, alpha, beta, o) are written when non-null.
 */
void oracle_decode_step(const oracle_cfg* c, int B, int T, const uint16_t* qkv, const uint16_t* a,
                        const uint16_t* b, const uint16_t* z, const uint16_t* conv_w,
                        const float* A_log, const float* dt_bias, const uint16_t* norm_w,
                        uint16_t* conv_pool, double* state_pool, int pool_slots,
                        const int32_t* slots, double* out, double* q_opt, double* k_opt,
                        double* v_opt, double* alpha_opt, double* beta_opt, double* o_opt) {
    const size_t nq = (size_t)B * T * c->num_k_heads * c->head_k_dim;
    const size_t nv = (size_t)B * T * c->num_v_heads * c->head_v_dim;
    const size_t nh = (size_t)B * T * c->num_v_heads;
    double* q = q_opt ? q_opt : (double*)malloc(sizeof(double) * nq);
    double* k = k_opt ? k_opt : (double*)malloc(sizeof(double) * nq);
    double* v = v_opt ? v_opt : (double*)malloc(sizeof(double) * nv);
    double* al = alpha_opt ? alpha_opt : (double*)malloc(sizeof(double) * nh);
    double* be = beta_opt ? beta_opt : (double*)malloc(sizeof(double) * nh);
    double* o = o_opt ? o_opt : (double*)malloc(sizeof(double) * nv);
    oracle_conv_update(c, B, T, qkv, conv_w, conv_pool, pool_slots, slots, q, k, v);
    oracle_gate(c, B * T, a, b, A_log, dt_bias, al, be);
    oracle_delta_rule(c, B, T, q, k, v, al, be, state_pool, pool_slots, slots, o);
    oracle_gated_rmsnorm(c, B * T * c->num_v_heads, o, z, norm_w, out);
    if (!o_opt) free(o);
    if (!beta_opt) free(be);
    if (!alpha_opt) free(al);
    if (!v_opt) free(v);
    if (!k_opt) free(k);
    if (!q_opt) free(q);
}

/*
 * bf16 round-to-nearest-even of a double, done directly (no float detour, so no
 * double rounding): keep 8 significant bits. Used to compare the GPU's bf16
 * outputs with the correctly rounded oracle value.
 */
void oracle_round_bf16(const double* x, uint16_t* out, size_t n) {
    for (size_t i = 0; i < n; ++i) {
        double a = x[i], r;
        if (a == 0.0 || !isfinite(a)) {
            r = a;
        } else {
            int e;
            frexp(a, &e);                 /* |a| = m * 2^e, m in [0.5, 1) */
            if (e - 1 < -126) e = -125;   /* bf16 subnormals share the ulp 2^-133 */
            r = ldexp(nearbyint(ldexp(a, 8 - e)), e - 8);
        }
        float f = (float)r; /* exact: r has at most 8 significant bits */
        uint32_t u;
        memcpy(&u, &f, sizeof u);
        out[i] = (uint16_t)(u >> 16);
    }
}
