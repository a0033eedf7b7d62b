/*
 * moe_oracle.c -- plain CPU oracle for the Mixtral sparse-MoE feed-forward layer.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test suite, the smoke check
 * and the CPU-baseline leg of the benchmark may load this library.  The CUDA
 * path shares no code, header, table or helper with it.
 *
 * What it computes, and where the pages state it:
 *   "Mixtral" (llm-arch-research textbook), section "Прямой проход в формулах"
 *   (forward pass in formulas), MoE equation:
 *       g = u W_r,  S = TopK(g, k),  w_i = exp(g_i) / sum_{j in S} exp(g_j),
 *       MoE(u) = sum_{i in S} w_i (SiLU(u W_gate^i) * (u W_up^i)) W_down^i
 *   and section "Алгоритм" (algorithm): a loop over experts; expert e gets the
 *   tokens whose top-k list holds e (in token order), and each token receives
 *   exactly k gate-weighted terms.  No capacity, no dropped tokens.
 *
 * Arithmetic: every input is a bf16 value; products of two bf16 values are exact
 * in double, and every dot product is accumulated in double in ascending index
 * order.  The router logits are rounded once to float (the router softmax runs in
 * float32 per section "MoE изнутри"), the top-k choice is taken on those float
 * logits, lower expert index first on equal logits.  When `round_h` is set the
 * expert intermediate h = SiLU(u W_gate) * (u W_up) is rounded to bf16 (round to
 * nearest, ties to even): it is the bf16 input of the down projection in a bf16
 * model.  The expert outputs o and the layer output y are returned unrounded
 * (double); a bf16 implementation is expected to round y once, at the end.
 * With `round_h` clear everything after the inputs stays in double.
 *
 * Build: gcc -O3 -fopenmp -ffp-contract=off -fPIC -shared (no fast-math: the
 * compiler may not reorder any sum).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---- bf16 encoding --------------------------------------------------------
 * A bf16 value is the upper 16 bits of an IEEE binary32: 1 sign bit, 8 exponent
 * bits, 7 stored mantissa bits (8 significant bits). */

double orc_bf16_value(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a double to the nearest bf16 value, ties to even, straight from the
 * binary expansion: the spacing of bf16 values in the binade [2^(e-1), 2^e) is
 * 2^(e-8); below 2^-126 the spacing is the subnormal step 2^-133.  Values whose
 * rounded magnitude exceeds the largest finite bf16 (255 * 2^120) become inf. */
double orc_round_bf16(double v) {
    if (isnan(v) || isinf(v) || v == 0.0) return v;
    int e;
    (void)frexp(v, &e);               /* |v| in [2^(e-1), 2^e) */
    int q = e - 8;
    if (q < -133) q = -133;
    double r = nearbyint(ldexp(v, -q)); /* default rounding mode: nearest, ties to even */
    double out = ldexp(r, q);
    if (fabs(out) > ldexp(255.0, 120)) out = copysign(INFINITY, v);
    return out;
}

uint16_t orc_bf16_bits(double v) {
    if (isnan(v)) return 0x7FC0;
    float f = (float)orc_round_bf16(v); /* exact: a bf16 value is a float value */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(u >> 16);
}

void orc_round_bf16_array(int64_t n, const double* in, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_bf16_bits(in[i]);
}

/* SiLU(a) = a * sigmoid(a) = a / (1 + exp(-a))  (SwiGLU expert, section
 * "Прямой проход в формулах"). */
double orc_silu(double a) { return a / (1.0 + exp(-a)); }

/* ---- router: logits, top-k, softmax over the selected k ------------------
 * Section "Прямой проход в формулах" (g = u W_r, S = TopK(g,k), w_i) and
 * section "Алгоритм" (topk of X W_r, softmax over the k selected logits in
 * float32).  `bias` (nullable, [E] float) is added to the logits when given
 * (the library's `bias: true` router; Mixtral 8x7B itself has none).
 *   x  [T, d] bf16, wg [d, E] bf16 (row-major, E fastest)
 *   idx [T, k] int32: slot 0 holds the largest logit
 *   gate [T, k] float, logits [T, E] float (nullable). */
static void route_one(int d, int E, int k, const uint16_t* xrow, const uint16_t* wg,
                      const float* bias, int32_t* idx, float* gate, float* logits) {
    float g[64];
    for (int e = 0; e < E; ++e) {
        double acc = 0.0;
        for (int j = 0; j < d; ++j)
            acc += orc_bf16_value(xrow[j]) * orc_bf16_value(wg[(int64_t)j * E + e]);
        if (bias) acc += (double)bias[e];
        g[e] = (float)acc;
        if (logits) logits[e] = g[e];
    }
    /* TopK: k rounds of "largest logit not yet taken"; scanning e upwards with a
     * strict '>' keeps the lower index among equal logits. */
    int taken[64] = {0};
    for (int s = 0; s < k; ++s) {
        int best = -1;
        for (int e = 0; e < E; ++e)
            if (!taken[e] && (best < 0 || g[e] > g[best])) best = e;
        taken[best] = 1;
        idx[s] = best;
    }
    /* w_s = exp(g_s) / sum_j exp(g_j) over the selected k; the largest selected
     * logit is subtracted first, which leaves the ratio unchanged. */
    double m = (double)g[idx[0]];
    double den = 0.0;
    for (int s = 0; s < k; ++s) den += exp((double)g[idx[s]] - m);
    for (int s = 0; s < k; ++s) gate[s] = (float)(exp((double)g[idx[s]] - m) / den);
}

int orc_route(int T, int d, int E, int k, const uint16_t* x, const uint16_t* wg,
              const float* bias, int32_t* idx, float* gate, float* logits) {
    if (T < 0 || d < 1 || E < 1 || E > 64 || k < 1 || k > E) return 1;
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t)
        route_one(d, E, k, x + (int64_t)t * d, wg, bias, idx + (int64_t)t * k,
                  gate + (int64_t)t * k, logits ? logits + (int64_t)t * E : NULL);
    return 0;
}

/* ---- dispatch ---------------------------------------------------------------
 * Section "Алгоритм": for expert e, the (token, slot) pairs whose top-k list
 * names e, read in row-major order, i.e. by ascending token.  The per-expert lists are laid end
 * to end: offsets[e] = number of (token, slot) entries routed to experts < e.
 *   offsets [E+1], perm_tok [T*k] (token of each sorted row),
 *   inv [T, k] (sorted row of each (token, slot)). */
int orc_dispatch(int T, int E, int k, const int32_t* idx, int32_t* offsets,
                 int32_t* perm_tok, int32_t* inv) {
    if (T < 0 || E < 1 || k < 1 || k > E) return 1;
    for (int64_t i = 0; i < (int64_t)T * k; ++i)
        if (idx[i] < 0 || idx[i] >= E) return 1;
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) {
        int32_t pos = offsets[e];
        for (int t = 0; t < T; ++t)
            for (int s = 0; s < k; ++s)
                if (idx[(int64_t)t * k + s] == e) {
                    perm_tok[pos] = t;
                    inv[(int64_t)t * k + s] = pos;
                    ++pos;
                }
        offsets[e + 1] = pos;
    }
    return 0;
}

/* X[tok] of section "Алгоритм": the rows of x in expert-sorted order. */
void orc_gather(int R, int d, const int32_t* perm_tok, const uint16_t* x, uint16_t* x_sorted) {
    for (int r = 0; r < R; ++r)
        memcpy(x_sorted + (int64_t)r * d, x + (int64_t)perm_tok[r] * d, (size_t)d * sizeof(uint16_t));
}

/* ---- one SwiGLU expert on one row -----------------------------------------
 * Section "Прямой проход в формулах": (SiLU(u W_gate) * (u W_up)) W_down with
 * W_gate = W1[e], W_up = W3[e] of shape [d, d_ff] and W_down = W2[e] of shape
 * [d_ff, d], all row-major.  h [d_ff] holds the bf16-rounded value (round_h) or
 * the unrounded one; o [d] is unrounded.  b1e/b3e [d_ff] and b2e [d] are the
 * float biases of the three Linear layers when the layer is built with bias
 * (section "Подсчёт параметров", teaching configuration: bias on every Linear),
 * else NULL.
 * acc_a / acc_b are caller scratch of d_ff doubles. */
static void expert_row(int d, int d_ff, const uint16_t* u, const uint16_t* W1e,
                       const uint16_t* W3e, const uint16_t* W2e, const float* b1e,
                       const float* b3e, const float* b2e, int round_h,
                       double* acc_a, double* acc_b, double* h, double* o) {
    for (int n = 0; n < d_ff; ++n) { acc_a[n] = 0.0; acc_b[n] = 0.0; }
    /* a_n = sum_j u_j W1[j][n], b_n = sum_j u_j W3[j][n]; each sum runs over j
     * in ascending order. */
    for (int j = 0; j < d; ++j) {
        double uj = orc_bf16_value(u[j]);
        const uint16_t* w1 = W1e + (int64_t)j * d_ff;
        const uint16_t* w3 = W3e + (int64_t)j * d_ff;
        for (int n = 0; n < d_ff; ++n) {
            acc_a[n] += uj * orc_bf16_value(w1[n]);
            acc_b[n] += uj * orc_bf16_value(w3[n]);
        }
    }
    /* Linear layers with bias (the teaching configuration) add b after the sum. */
    if (b1e) for (int n = 0; n < d_ff; ++n) acc_a[n] += (double)b1e[n];
    if (b3e) for (int n = 0; n < d_ff; ++n) acc_b[n] += (double)b3e[n];
    for (int n = 0; n < d_ff; ++n) {
        double hv = orc_silu(acc_a[n]) * acc_b[n];
        h[n] = round_h ? orc_round_bf16(hv) : hv;
    }
    /* o_c = sum_n h_n W2[n][c], n ascending (+ b2_c). */
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    for (int n = 0; n < d_ff; ++n) {
        double hn = h[n];
        const uint16_t* w2 = W2e + (int64_t)n * d;
        for (int c = 0; c < d; ++c) o[c] += hn * orc_bf16_value(w2[c]);
    }
    if (b2e) for (int c = 0; c < d; ++c) o[c] += (double)b2e[c];
}

/* Expert_e(X[tok]) for every expert over its sorted rows (section "Алгоритм";
 * an expert with no rows is not called).
 *   x_sorted [R, d] bf16, offsets [E+1], W1/W3 [E, d, d_ff], W2 [E, d_ff, d]
 *   h [R, d_ff] double, o [R, d] double. */
int orc_expert_bias(int R, int d, int d_ff, int E, const int32_t* offsets,
                    const uint16_t* x_sorted, const uint16_t* W1, const uint16_t* W3,
                    const uint16_t* W2, const float* b1, const float* b3, const float* b2,
                    int round_h, double* h, double* o) {
    if (offsets[0] != 0 || offsets[E] != R) return 1;
    for (int e = 0; e < E; ++e)
        if (offsets[e + 1] < offsets[e]) return 1;
    int ok = 1;
#pragma omp parallel
    {
        double* acc_a = (double*)malloc(sizeof(double) * (size_t)d_ff);
        double* acc_b = (double*)malloc(sizeof(double) * (size_t)d_ff);
        if (!acc_a || !acc_b) {
#pragma omp atomic write
            ok = 0;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int r = 0; r < R; ++r) {
                int e = 0;
                while (offsets[e + 1] <= r) ++e;
                const int64_t wsz = (int64_t)d * d_ff;
                expert_row(d, d_ff, x_sorted + (int64_t)r * d, W1 + e * wsz, W3 + e * wsz,
                           W2 + e * wsz, b1 ? b1 + (int64_t)e * d_ff : NULL,
                           b3 ? b3 + (int64_t)e * d_ff : NULL, b2 ? b2 + (int64_t)e * d : NULL,
                           round_h, acc_a, acc_b, h + (int64_t)r * d_ff, o + (int64_t)r * d);
            }
        }
        free(acc_a);
        free(acc_b);
    }
    return ok ? 0 : 2;
}

int orc_expert(int R, int d, int d_ff, int E, const int32_t* offsets, const uint16_t* x_sorted,
               const uint16_t* W1, const uint16_t* W3, const uint16_t* W2, int round_h,
               double* h, double* o) {
    return orc_expert_bias(R, d, d_ff, E, offsets, x_sorted, W1, W3, W2, NULL, NULL, NULL,
                           round_h, h, o);
}

/* ---- combine ------------------------------------------------------------------
 * Section "Алгоритм": Y[tok] += W[tok, slot] * Expert_e(X[tok]); every token gets
 * exactly k terms.  Here the k terms of a token are summed in slot order.
 *   o [R, d] double, inv [T, k], gate [T, k] float -> y [T, d] double. */
void orc_combine(int T, int d, int k, const double* o, const int32_t* inv, const float* gate,
                 double* y) {
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t)
        for (int c = 0; c < d; ++c) {
            double acc = 0.0;
            for (int s = 0; s < k; ++s)
                acc += (double)gate[(int64_t)t * k + s] * o[(int64_t)inv[(int64_t)t * k + s] * d + c];
            y[(int64_t)t * d + c] = acc;
        }
}

/* ---- whole layer, expert-major (the loop of section "Алгоритм") ------------
 * Scratch is allocated here; outputs idx/gate/offsets/perm_tok/inv are
 * nullable. */
int orc_forward_bias(int T, int d, int d_ff, int E, int k, const uint16_t* x, const uint16_t* wg,
                     const float* bias, const uint16_t* W1, const uint16_t* W3,
                     const uint16_t* W2, const float* b1, const float* b3, const float* b2,
                     int round_h, double* y, int32_t* idx_out, float* gate_out) {
    const int R = T * k;
    int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * (size_t)(R > 0 ? R : 1));
    float* gate = (float*)malloc(sizeof(float) * (size_t)(R > 0 ? R : 1));
    int32_t* offsets = (int32_t*)malloc(sizeof(int32_t) * (size_t)(E + 1));
    int32_t* perm = (int32_t*)malloc(sizeof(int32_t) * (size_t)(R > 0 ? R : 1));
    int32_t* inv = (int32_t*)malloc(sizeof(int32_t) * (size_t)(R > 0 ? R : 1));
    uint16_t* xs = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(R > 0 ? R : 1) * d);
    double* h = (double*)malloc(sizeof(double) * (size_t)(R > 0 ? R : 1) * d_ff);
    double* o = (double*)malloc(sizeof(double) * (size_t)(R > 0 ? R : 1) * d);
    int rc = 0;
    if (!idx || !gate || !offsets || !perm || !inv || !xs || !h || !o) { rc = 2; goto done; }
    if ((rc = orc_route(T, d, E, k, x, wg, bias, idx, gate, NULL))) goto done;
    if ((rc = orc_dispatch(T, E, k, idx, offsets, perm, inv))) goto done;
    orc_gather(R, d, perm, x, xs);
    if ((rc = orc_expert_bias(R, d, d_ff, E, offsets, xs, W1, W3, W2, b1, b3, b2, round_h, h, o)))
        goto done;
    orc_combine(T, d, k, o, inv, gate, y);
    if (idx_out) memcpy(idx_out, idx, sizeof(int32_t) * (size_t)R);
    if (gate_out) memcpy(gate_out, gate, sizeof(float) * (size_t)R);
done:
    free(idx); free(gate); free(offsets); free(perm); free(inv); free(xs); free(h); free(o);
    return rc;
}

int orc_forward(int T, int d, int d_ff, int E, int k, const uint16_t* x, const uint16_t* wg,
                const float* bias, const uint16_t* W1, const uint16_t* W3, const uint16_t* W2,
                int round_h, double* y, int32_t* idx_out, float* gate_out) {
    return orc_forward_bias(T, d, d_ff, E, k, x, wg, bias, W1, W3, W2, NULL, NULL, NULL, round_h,
                            y, idx_out, gate_out);
}

/* ---- naive per-token loop ------------------------------------------------------
 * The same layer computed token by token, straight from the formula of section
 * "Прямой проход в формулах" (the reference's own test compares MoE against such
 * a loop, section "Алгоритм").  Computes y only for the n listed tokens:
 *   toks [n] token ids; y [n, d] double; idx_out [n, k], gate_out [n, k]
 * (nullable).  Used for sampled checks at sizes where the full layer is too slow. */
int orc_forward_tokens_bias(int n, const int32_t* toks, int T, int d, int d_ff, int E, int k,
                            const uint16_t* x, const uint16_t* wg, const float* bias,
                            const uint16_t* W1, const uint16_t* W3, const uint16_t* W2,
                            const float* b1, const float* b3, const float* b2, int round_h,
                            double* y, int32_t* idx_out, float* gate_out) {
    if (E < 1 || E > 64 || k < 1 || k > E) return 1;
    for (int i = 0; i < n; ++i)
        if (toks[i] < 0 || toks[i] >= T) return 1;
    int ok = 1;
#pragma omp parallel
    {
        double* acc_a = (double*)malloc(sizeof(double) * (size_t)d_ff);
        double* acc_b = (double*)malloc(sizeof(double) * (size_t)d_ff);
        double* h = (double*)malloc(sizeof(double) * (size_t)d_ff);
        double* o = (double*)malloc(sizeof(double) * (size_t)d * (size_t)k);
        if (!acc_a || !acc_b || !h || !o) {
#pragma omp atomic write
            ok = 0;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int i = 0; i < n; ++i) {
                const uint16_t* u = x + (int64_t)toks[i] * d;
                int32_t sel[64];
                float w[64];
                route_one(d, E, k, u, wg, bias, sel, w, NULL);
                const int64_t wsz = (int64_t)d * d_ff;
                for (int s = 0; s < k; ++s) {
                    const int e = sel[s];
                    expert_row(d, d_ff, u, W1 + e * wsz, W3 + e * wsz, W2 + e * wsz,
                               b1 ? b1 + (int64_t)e * d_ff : NULL,
                               b3 ? b3 + (int64_t)e * d_ff : NULL, b2 ? b2 + (int64_t)e * d : NULL,
                               round_h, acc_a, acc_b, h, o + (int64_t)s * d);
                }
                for (int c = 0; c < d; ++c) {
                    double acc = 0.0;
                    for (int s = 0; s < k; ++s) acc += (double)w[s] * o[(int64_t)s * d + c];
                    y[(int64_t)i * d + c] = acc;
                }
                if (idx_out) for (int s = 0; s < k; ++s) idx_out[(int64_t)i * k + s] = sel[s];
                if (gate_out) for (int s = 0; s < k; ++s) gate_out[(int64_t)i * k + s] = w[s];
            }
        }
        free(acc_a); free(acc_b); free(h); free(o);
    }
    return ok ? 0 : 2;
}

int orc_forward_tokens(int n, const int32_t* toks, int T, int d, int d_ff, int E, int k,
                       const uint16_t* x, const uint16_t* wg, const float* bias,
                       const uint16_t* W1, const uint16_t* W3, const uint16_t* W2, int round_h,
                       double* y, int32_t* idx_out, float* gate_out) {
    return orc_forward_tokens_bias(n, toks, T, d, d_ff, E, k, x, wg, bias, W1, W3, W2, NULL, NULL,
                                   NULL, round_h, y, idx_out, gate_out);
}

/* ---- parameter count ------------------------------------------------------------
 * Section "Подсчёт параметров" (parameter count) of the Mixtral page:
 *   N_attn  = d*H*dh + 2*d*G*dh + H*dh*d        (Q, K, V, O projections)
 *   N_exp   = 3*d*d_ff                          (W_gate, W_up [d, d_ff]; W_down [d_ff, d])
 *   total   = V*d + L*(N_attn + d*E + E*N_exp + 2d) + d + d*V
 *   active  = same with k experts in place of E
 * With bias every Linear also holds d_out parameters (the teaching config of the
 * same section): router + E, expert + 2*d_ff + d, attention + H*dh + 2*G*dh + d,
 * output head + V.  The expert term uses the same three weight shapes the
 * expert routine above reads. */
void orc_param_count(int64_t V, int64_t d, int64_t L, int64_t H, int64_t G, int64_t dh,
                     int64_t d_ff, int64_t E, int64_t k, int bias, int64_t* total, int64_t* active) {
    int64_t attn = d * H * dh + 2 * d * G * dh + H * dh * d;
    int64_t router = d * E;
    int64_t expert = d * d_ff + d * d_ff + d_ff * d; /* W1, W3, W2 */
    int64_t head = d * V;
    if (bias) {
        attn += H * dh + 2 * G * dh + d;
        router += E;
        expert += d_ff + d_ff + d;
        head += V;
    }
    int64_t norms = 2 * d;
    int64_t embed = V * d;
    *total = embed + L * (attn + router + E * expert + norms) + d + head;
    *active = embed + L * (attn + router + k * expert + norms) + d + head;
}

/* ---- load-balancing auxiliary loss -------------------------------------------
 * Mixtral page, section "Load-balancing loss":
 *     aux = E * sum_{s<k} sum_{i<E} f_{s,i} * P_i
 * f_{s,i}: fraction of the counted tokens whose top-k slot s holds expert i;
 * P_i:     mean over the counted tokens of the softmax over all E router
 *          logits, entry i.
 * (the training loss adds alpha * aux; under uniform load aux = k.)
 * Counted tokens are all T, or those with mask[t] != 0 when mask is given
 * (padding excluded).  f [k*E] and P [E] are written when non-null.  Returns
 * aux (0 when no token is counted). */
double orc_aux_loss(int T, int E, int k, const float* logits, const int32_t* idx,
                    const uint8_t* mask, double* f_out, double* P_out) {
    double* f = (double*)calloc((size_t)k * E, sizeof(double));
    double* P = (double*)calloc((size_t)E, sizeof(double));
    double* p = (double*)malloc(sizeof(double) * (size_t)E);
    double n = 0.0;
    for (int t = 0; t < T; ++t) {
        if (mask && !mask[t]) continue;
        n += 1.0;
        const float* g = logits + (int64_t)t * E;
        double m = (double)g[0];
        for (int e = 1; e < E; ++e)
            if ((double)g[e] > m) m = (double)g[e];
        double den = 0.0;
        for (int e = 0; e < E; ++e) {
            p[e] = exp((double)g[e] - m);
            den += p[e];
        }
        for (int e = 0; e < E; ++e) P[e] += p[e] / den;
        for (int s = 0; s < k; ++s) {
            const int e = idx[(int64_t)t * k + s];
            if (e >= 0 && e < E) f[(int64_t)s * E + e] += 1.0;
        }
    }
    double aux = 0.0;
    if (n > 0) {
        for (int i = 0; i < k * E; ++i) f[i] /= n;
        for (int e = 0; e < E; ++e) P[e] /= n;
        for (int s = 0; s < k; ++s)
            for (int e = 0; e < E; ++e) aux += f[(int64_t)s * E + e] * P[e];
        aux *= (double)E;
    }
    if (f_out) memcpy(f_out, f, sizeof(double) * (size_t)k * E);
    if (P_out) memcpy(P_out, P, sizeof(double) * (size_t)E);
    free(f); free(P); free(p);
    return aux;
}

/* ---- block edges: RMSNorm before the layer, residual after it ------------------
 * Mixtral page, section "Прямой проход в формулах":
 *     H = U + MoE(RMSNorm_2(U)),   RMSNorm(z) = z / sqrt(mean_j z_j^2 + eps) (.) gamma
 * (eps = rms_norm_eps, 1e-5 for Mixtral 8x7B).  The normalised rows are the
 * bf16 input of the layer, so they are rounded to bf16 (nearest even).
 *   U [T,d] bf16, gamma [d] bf16 -> u [T,d] bf16 bits. */
void orc_rmsnorm(int T, int d, const uint16_t* U, const uint16_t* gamma, double eps, uint16_t* u) {
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        const uint16_t* z = U + (int64_t)t * d;
        double ss = 0.0;
        for (int j = 0; j < d; ++j) {
            const double v = orc_bf16_value(z[j]);
            ss += v * v;
        }
        const double r = sqrt(ss / d + eps);
        for (int j = 0; j < d; ++j)
            u[(int64_t)t * d + j] = orc_bf16_bits(orc_bf16_value(z[j]) / r * orc_bf16_value(gamma[j]));
    }
}

/* H = U + MoE(RMSNorm(U)) with the layer of orc_forward (H unrounded, double). */
int orc_block_forward(int T, int d, int d_ff, int E, int k, const uint16_t* U, const uint16_t* gamma,
                      double eps, const uint16_t* wg, const float* bias, const uint16_t* W1,
                      const uint16_t* W3, const uint16_t* W2, int round_h, double* H,
                      int32_t* idx_out, float* gate_out) {
    uint16_t* u = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(T > 0 ? T : 1) * d);
    if (!u) return 2;
    orc_rmsnorm(T, d, U, gamma, eps, u);
    const int rc = orc_forward(T, d, d_ff, E, k, u, wg, bias, W1, W3, W2, round_h, H, idx_out,
                               gate_out);
    if (!rc)
        for (int64_t i = 0; i < (int64_t)T * d; ++i) H[i] += orc_bf16_value(U[i]);
    free(u);
    return rc;
}
