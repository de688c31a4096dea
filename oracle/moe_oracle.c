/*
 * CPU oracle for the dropless sparse-MoE expert-MLP forward.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the package entry's smoke check and the bench's CPU
 * baseline leg may load this library. It shares no code, header, table or helper with the CUDA
 * library; neither includes or loads the other.
 *
 * Every function is the plain definition of one step, in fp64, with inputs given as float32
 * arrays (bf16 inputs are exactly representable in float32). Loops are written in the order of
 * the definitions; the only liberties are the loop nesting of the dot products (a d-outer /
 * f-inner order that walks the [D,F] weights contiguously; each output is still summed over
 * d = 0..D-1 in ascending order) and OpenMP parallelism over independent tokens or slots.
 *
 * Sources (page title, then section / equation):
 *  - "ScatterMoE Guide: Fast Fused Kernels for Sparse MoE LLMs"
 *      "1. The Dynamic Routing Imbalance Dilemma", router equation H(X) = Softmax(TopK(X W_gate, k))
 *      "1. The Anatomy of ParallelLinear", ParallelLinear(X, W, I, G) with W in R^{E x Din x Dout}
 *      "2. Grouped Coordinate Indexing Without Padding", Histogram(e) and Offsets(e) equations
 *      "The ParallelLinear Core Abstraction" figure, Steps 1-3 (gather, tile GEMM, gate + scatter)
 *      "3. Assembling the ScatterMoE FFN Block" (SwiGLU: silu(gate) * up, gate half first)
 *  - "Add scalable sparse map kernel for large MoE models (128+ experts)"
 *      "Pass 1: Histogram with Atomics", "Pass 2: Two Assignment Variants",
 *      "4. Correctness Validation" (unique rows, rows inside their expert's range, counts,
 *      non-overlapping ranges, determinism)
 *
 * Readings taken where the pages are silent or inconsistent (all listed in the design notes):
 *  - softmax over the k selected logits (weights sum to 1); the guide's code takes the full
 *    softmax, then top-k, then renormalises, which is the same in exact arithmetic;
 *  - top-k order: logits descending, equal logits -> smaller expert id first;
 *  - slot order inside an expert follows the flat route index i = s*k + j (a stable sort), which is
 *    the one deterministic result the map tests demand;
 *  - the optional logit bias is added to the logits before selection and softmax;
 *  - weights are used as x * W[e] with W[e] of shape [Din, Dout].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Router logits l[s,e] = sum_d x[s,d] * W_gate[d,e] (+ bias[e]), and the magnitude sum
 * a[s,e] = sum_d |x[s,d] * W_gate[d,e]| that bounds the rounding error of any float evaluation of
 * the same dot product. W_gate is [D,E]. Computed for the listed tokens only. */
static void logits_one(const float *xs, const float *w_gate, const float *bias, int64_t D,
                       int32_t E, double *l, double *a) {
    for (int32_t e = 0; e < E; ++e) {
        l[e] = 0.0;
        if (a) a[e] = 0.0;
    }
    for (int64_t d = 0; d < D; ++d) {
        const double xv = (double)xs[d];
        const float *wrow = w_gate + d * E;
        for (int32_t e = 0; e < E; ++e) {
            const double p = xv * (double)wrow[e];
            l[e] += p;
            if (a) a[e] += fabs(p);
        }
    }
    if (bias)
        for (int32_t e = 0; e < E; ++e) l[e] += (double)bias[e];
}

void oracle_router_logits(const float *x, const float *w_gate, const float *bias, int64_t D,
                          int32_t E, const int32_t *tokens, int64_t n_tokens, double *logits,
                          double *absdot) {
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < n_tokens; ++t)
        logits_one(x + (int64_t)tokens[t] * D, w_gate, bias, D, E, logits + t * E,
                   absdot ? absdot + t * E : NULL);
}

/* Top-k selection and softmax over the selected logits for one token.
 * J_0..J_{k-1}: the k largest logits, in descending order; on equal logits the smaller expert id
 * ranks first. Selection is k passes of "best not yet taken"; the strict '>' keeps the smaller id
 * on ties. Weights w_j = exp(l_{J_j} - l_{J_0}) / sum_j' exp(l_{J_j'} - l_{J_0}). */
static void topk_one(const double *l, int32_t E, int32_t k, int32_t *J, double *w) {
    for (int32_t j = 0; j < k; ++j) {
        int32_t best = -1;
        for (int32_t e = 0; e < E; ++e) {
            int taken = 0;
            for (int32_t q = 0; q < j; ++q)
                if (J[q] == e) taken = 1;
            if (taken) continue;
            if (best < 0 || l[e] > l[best]) best = e;
        }
        J[j] = best;
    }
    const double m = l[J[0]];
    double den = 0.0;
    for (int32_t j = 0; j < k; ++j) den += exp(l[J[j]] - m);
    for (int32_t j = 0; j < k; ++j) w[j] = exp(l[J[j]] - m) / den;
}

void oracle_topk_softmax(const double *logits, int64_t n_tokens, int32_t E, int32_t k,
                         int32_t *top_experts, double *top_weights) {
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < n_tokens; ++t)
        topk_one(logits + t * E, E, k, top_experts + t * k, top_weights + t * k);
}

/* Softmax weights for a given (externally chosen) expert list J of each token, in J's order. */
void oracle_weights_for(const double *logits, const int32_t *top_experts, int64_t n_tokens,
                        int32_t E, int32_t k, double *top_weights) {
    for (int64_t t = 0; t < n_tokens; ++t) {
        const double *l = logits + t * E;
        const int32_t *J = top_experts + t * k;
        double m = l[J[0]];
        for (int32_t j = 1; j < k; ++j)
            if (l[J[j]] > m) m = l[J[j]];
        double den = 0.0;
        for (int32_t j = 0; j < k; ++j) den += exp(l[J[j]] - m);
        for (int32_t j = 0; j < k; ++j) top_weights[t * k + j] = exp(l[J[j]] - m) / den;
    }
}

/* Sparse map over the flat route list i = 0..R-1 (i = s*k + j), expert(i) = top_experts[i]:
 *   counts[e]       = #{i : expert(i) = e}                             (Histogram(e))
 *   offsets[e]      = sum_{e' < e} counts[e'],  offsets[E] = R          (Offsets(e))
 *   sparse_rows[i]  = offsets[expert(i)] + #{i' < i : expert(i') = expert(i)}   (stable slot)
 *   sorted_rows[p]  = the i with sparse_rows[i] = p                    (expert-sorted route list)
 * A sequential counting sort. Returns 0, or -1 (and writes nothing) if an id is outside [0, E). */
int oracle_sparse_map(const int32_t *top_experts, int64_t R, int32_t E, int32_t *counts,
                      int32_t *offsets, int32_t *sparse_rows, int32_t *sorted_rows) {
    for (int64_t i = 0; i < R; ++i)
        if (top_experts[i] < 0 || top_experts[i] >= E) return -1;
    for (int32_t e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t i = 0; i < R; ++i) counts[top_experts[i]] += 1;
    offsets[0] = 0;
    for (int32_t e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int32_t *next = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E > 0 ? E : 1));
    for (int32_t e = 0; e < E; ++e) next[e] = offsets[e];
    for (int64_t i = 0; i < R; ++i) {
        const int32_t e = top_experts[i];
        sparse_rows[i] = next[e];
        sorted_rows[next[e]] = (int32_t)i;
        next[e] += 1;
    }
    free(next);
    return 0;
}

static double silu(double z) { return z / (1.0 + exp(-z)); }

/* Expert hidden row h = silu(v . W_gate_e[e]) * (v . W_up[e]), W_gate_e[e], W_up[e] of shape [D,F]
 * (the gate half is the one passed through SiLU). */
static void expert_hidden(const float *v, const float *wge, const float *wu, int64_t D, int64_t F,
                          double *g, double *u, double *h) {
    for (int64_t f = 0; f < F; ++f) {
        g[f] = 0.0;
        u[f] = 0.0;
    }
    for (int64_t d = 0; d < D; ++d) {
        const double vd = (double)v[d];
        const float *gr = wge + d * F;
        const float *ur = wu + d * F;
        for (int64_t f = 0; f < F; ++f) {
            g[f] += vd * (double)gr[f];
            u[f] += vd * (double)ur[f];
        }
    }
    for (int64_t f = 0; f < F; ++f) h[f] = silu(g[f]) * u[f];
}

void oracle_expert_hidden(const float *x, const float *w_gate_e, const float *w_up, int64_t D,
                          int64_t F, int32_t token, int32_t expert, double *h) {
    double *g = (double *)malloc(sizeof(double) * (size_t)F);
    double *u = (double *)malloc(sizeof(double) * (size_t)F);
    expert_hidden(x + (int64_t)token * D, w_gate_e + (int64_t)expert * D * F,
                  w_up + (int64_t)expert * D * F, D, F, g, u, h);
    free(g);
    free(u);
}

/* The same hidden row for n (token, expert) pairs, h [n, F]; the rows are independent. */
void oracle_expert_hidden_rows(const float *x, const float *w_gate_e, const float *w_up,
                               int64_t D, int64_t F, const int32_t *tokens,
                               const int32_t *experts, int64_t n, double *h) {
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < n; ++i)
        oracle_expert_hidden(x, w_gate_e, w_up, D, F, tokens[i], experts[i], h + i * F);
}

/* Forward for the listed tokens: y[s] = sum_j w_j * FFN_{J_j}(x[s]) with
 * FFN_e(v) = (silu(v W_gate_e[e]) * (v W_up[e])) W_down[e], W_down[e] of shape [F,D].
 * If given_top_experts ([S,k], indexed by token) is non-null, its experts replace the oracle's
 * own selection and the weights are the softmax of the fp64 logits over that list.
 * Outputs: out [n_tokens, D]; top_experts_out / top_weights_out [n_tokens, k] (nullable). */
void oracle_mlp_forward(const float *x, const float *w_gate, const float *bias,
                        const float *w_gate_e, const float *w_up, const float *w_down, int64_t D,
                        int64_t F, int32_t E, int32_t k, const int32_t *tokens, int64_t n_tokens,
                        const int32_t *given_top_experts, double *out, int32_t *top_experts_out,
                        double *top_weights_out) {
    #pragma omp parallel
    {
        double *l = (double *)malloc(sizeof(double) * (size_t)E);
        double *g = (double *)malloc(sizeof(double) * (size_t)F);
        double *u = (double *)malloc(sizeof(double) * (size_t)F);
        double *h = (double *)malloc(sizeof(double) * (size_t)F);
        int32_t J[64];
        double w[64];
        #pragma omp for schedule(dynamic, 1)
        for (int64_t t = 0; t < n_tokens; ++t) {
            const int32_t s = tokens[t];
            logits_one(x + (int64_t)s * D, w_gate, bias, D, E, l, NULL);
            if (given_top_experts) {
                for (int32_t j = 0; j < k; ++j) J[j] = given_top_experts[(int64_t)s * k + j];
                oracle_weights_for(l, J, 1, E, k, w);
            } else {
                topk_one(l, E, k, J, w);
            }
            double *y = out + t * D;
            for (int64_t d = 0; d < D; ++d) y[d] = 0.0;
            const float *v = x + (int64_t)s * D;
            for (int32_t j = 0; j < k; ++j) {
                const int64_t e = J[j];
                expert_hidden(v, w_gate_e + e * D * F, w_up + e * D * F, D, F, g, u, h);
                const float *wd = w_down + e * F * D;
                for (int64_t f = 0; f < F; ++f) {
                    const double c = w[j] * h[f];
                    const float *row = wd + f * D;
                    for (int64_t d = 0; d < D; ++d) y[d] += c * (double)row[d];
                }
            }
            if (top_experts_out)
                for (int32_t j = 0; j < k; ++j) top_experts_out[t * k + j] = J[j];
            if (top_weights_out)
                for (int32_t j = 0; j < k; ++j) top_weights_out[t * k + j] = w[j];
        }
        free(l);
        free(g);
        free(u);
        free(h);
    }
}

/* ParallelLinear(X, W, I, G): for every slot p of expert e (offsets[e] <= p < offsets[e+1]) with
 * route i = sorted_rows[p] and token s = i / k:
 *   v_p = src_p . W[e],  src_p = X[s] if gather_in else X[p],  W of shape [E, Din, Dout];
 *   c_p = gates[i] * v_p if gates is non-null, else v_p;
 *   scatter_out: Y[s] += c_p  (Y [S, Dout], zeroed here; slot contributions added in slot order)
 *   else:        Y[p]  = c_p  (Y [R, Dout], expert-grouped rows).   */
void oracle_scatter_linear(const float *X, const float *W, int64_t S, int64_t Din, int64_t Dout,
                           int32_t E, int32_t k, const int32_t *sorted_rows,
                           const int32_t *offsets, const float *gates, int gather_in,
                           int scatter_out, double *Y) {
    const int64_t P = offsets[E];
    double *grouped = (double *)calloc((size_t)(P > 0 ? P : 1) * (size_t)Dout, sizeof(double));
    #pragma omp parallel for schedule(dynamic, 4)
    for (int64_t p = 0; p < P; ++p) {
        int32_t e = 0;
        while (e < E && !(offsets[e] <= p && p < offsets[e + 1])) ++e;
        const int64_t i = sorted_rows[p];
        const int64_t s = i / k;
        const float *src = X + (gather_in ? s : p) * Din;
        const float *We = W + (int64_t)e * Din * Dout;
        double *v = grouped + p * Dout;
        for (int64_t d = 0; d < Din; ++d) {
            const double xv = (double)src[d];
            const float *wr = We + d * Dout;
            for (int64_t n = 0; n < Dout; ++n) v[n] += xv * (double)wr[n];
        }
        if (gates) {
            const double g = (double)gates[i];
            for (int64_t n = 0; n < Dout; ++n) v[n] *= g;
        }
    }
    if (scatter_out) {
        memset(Y, 0, sizeof(double) * (size_t)S * (size_t)Dout);
        for (int64_t p = 0; p < P; ++p) {
            const int64_t s = sorted_rows[p] / k;
            for (int64_t n = 0; n < Dout; ++n) Y[s * Dout + n] += grouped[p * Dout + n];
        }
    } else {
        memcpy(Y, grouped, sizeof(double) * (size_t)P * (size_t)Dout);
    }
    free(grouped);
}

/* Backward of ParallelLinear, the ScatterMoE guide's "3. Fused Backward Pass Dynamics": the input
 * gradient gathers the output gradient of each slot, multiplies by the transposed expert weight and
 * the gate, and sums back into the token (the guide's grad-X sum over TopK); the weight gradient of
 * expert e sums the outer products of its slots' inputs and gated output gradients (the guide's
 * grad-W_e sum over Tokens(e)); the gate gradient is the derivative of Y in g. With dY shaped like
 * Y ([S, Dout] if scatter_out, else [R, Dout]), for every slot p of expert e, route i, token s:
 *   dc_p = dY[s] if scatter_out else dY[p];   dv_p = g_i * dc_p  (g_i = 1 without gates)
 *   dsrc_p = dv_p . W[e]^T          -> dX[s] += dsrc_p (gather_in, dX [S, Din]) or dX[p] = dsrc_p
 *   dW[e] += src_p^T dv_p           -> dW [E, Din, Dout]
 *   dgates[i] = dc_p . (src_p . W[e])  (only with gates)
 * fp64 throughout; dX, dW and dgates may each be null (not computed); outputs are overwritten. */
void oracle_scatter_linear_backward(const float *X, const float *W, const float *dY, int64_t S,
                                    int64_t Din, int64_t Dout, int32_t E, int32_t k,
                                    const int32_t *sorted_rows, const int32_t *offsets,
                                    const float *gates, int gather_in, int scatter_out, double *dX,
                                    double *dW, double *dgates) {
    const int64_t P = offsets[E];
    int32_t *slot_e = (int32_t *)malloc(sizeof(int32_t) * (size_t)(P > 0 ? P : 1));
    for (int32_t e = 0; e < E; ++e)
        for (int64_t p = offsets[e]; p < offsets[e + 1]; ++p) slot_e[p] = e;
    if (dX) {
        const int64_t rows = gather_in ? S : P;
        double *dsrc = (double *)calloc((size_t)(P > 0 ? P : 1) * (size_t)Din, sizeof(double));
        #pragma omp parallel for schedule(dynamic, 4)
        for (int64_t p = 0; p < P; ++p) {
            const int32_t e = slot_e[p];
            const int64_t i = sorted_rows[p];
            const int64_t s = i / k;
            const float *dc = dY + (scatter_out ? s : p) * Dout;
            const double g = gates ? (double)gates[i] : 1.0;
            const float *We = W + (int64_t)e * Din * Dout;
            for (int64_t d = 0; d < Din; ++d) {
                double acc = 0.0;
                for (int64_t n = 0; n < Dout; ++n) acc += (double)dc[n] * (double)We[d * Dout + n];
                dsrc[p * Din + d] = g * acc;
            }
        }
        memset(dX, 0, sizeof(double) * (size_t)rows * (size_t)Din);
        for (int64_t p = 0; p < P; ++p) {
            const int64_t r = gather_in ? (int64_t)sorted_rows[p] / k : p;
            for (int64_t d = 0; d < Din; ++d) dX[r * Din + d] += dsrc[p * Din + d];
        }
        free(dsrc);
    }
    if (dW) {
        #pragma omp parallel for schedule(dynamic, 1) collapse(2)
        for (int32_t e = 0; e < E; ++e) {
            for (int64_t d = 0; d < Din; ++d) {
                double *row = dW + ((int64_t)e * Din + d) * Dout;
                for (int64_t n = 0; n < Dout; ++n) row[n] = 0.0;
                for (int64_t p = offsets[e]; p < offsets[e + 1]; ++p) {
                    const int64_t i = sorted_rows[p];
                    const int64_t s = i / k;
                    const double xv = (double)X[(gather_in ? s : p) * Din + d];
                    const double g = gates ? (double)gates[i] : 1.0;
                    const float *dc = dY + (scatter_out ? s : p) * Dout;
                    for (int64_t n = 0; n < Dout; ++n) row[n] += xv * g * (double)dc[n];
                }
            }
        }
    }
    if (dgates && gates) {
        const int64_t R = (int64_t)S * k;
        for (int64_t i = 0; i < R; ++i) dgates[i] = 0.0;
        #pragma omp parallel for schedule(dynamic, 4)
        for (int64_t p = 0; p < P; ++p) {
            const int32_t e = slot_e[p];
            const int64_t i = sorted_rows[p];
            const int64_t s = i / k;
            const float *src = X + (gather_in ? s : p) * Din;
            const float *dc = dY + (scatter_out ? s : p) * Dout;
            const float *We = W + (int64_t)e * Din * Dout;
            double acc = 0.0;
            for (int64_t n = 0; n < Dout; ++n) {
                double v = 0.0;
                for (int64_t d = 0; d < Din; ++d) v += (double)src[d] * (double)We[d * Dout + n];
                acc += (double)dc[n] * v;
            }
            dgates[i] = acc;
        }
    }
    free(slot_e);
}

/* Backward of the expert MLP forward (oracle_mlp_forward) for all S tokens, given the gradient of
 * the output dout [S, D]. The routing is the oracle's own top-k, or given_top_experts ([S, k]) if
 * non-null; the selection itself has no derivative. Per token s and selected expert e = J_j,
 * with a = x W_gate_e[e], b = x W_up[e], h = silu(a) * b, v = h W_down[e], w = softmax(l_J):
 *   dw_j = dout . v;  dv = w_j dout;  dh = dv W_down[e]^T;  dW_down[e] += h^T dv
 *   da = dh * b * silu'(a), silu'(z) = sig(z) (1 + z (1 - sig(z)));  db = dh * silu(a)
 *   dW_gate_e[e] += x^T da;  dW_up[e] += x^T db;  dx += da W_gate_e[e]^T + db W_up[e]^T
 *   softmax over the selected logits: dl_j = w_j (dw_j - sum_j' w_j' dw_j')
 *   dW_gate[:, e] += x dl_j;  dx += dl_j W_gate[:, e]
 * (the ScatterMoE guide's backward of each ParallelLinear, "3. Fused Backward Pass Dynamics",
 * chained through SwiGLU and the router softmax). fp64; every output is overwritten:
 * dx [S, D], dw_gate [D, E], dw_gate_e and dw_up [E, D, F], dw_down [E, F, D]. The weight
 * gradients are nullable (not computed); dx of a token depends on that token alone. */
void oracle_mlp_backward(const float *x, const float *w_gate, const float *bias,
                         const float *w_gate_e, const float *w_up, const float *w_down,
                         const float *dout, int64_t S, int64_t D, int64_t F, int32_t E, int32_t k,
                         const int32_t *given_top_experts, double *dx, double *dw_gate,
                         double *dw_gate_e, double *dw_up, double *dw_down) {
    memset(dx, 0, sizeof(double) * (size_t)S * (size_t)D);
    if (dw_gate) memset(dw_gate, 0, sizeof(double) * (size_t)D * (size_t)E);
    if (dw_gate_e) memset(dw_gate_e, 0, sizeof(double) * (size_t)E * (size_t)D * (size_t)F);
    if (dw_up) memset(dw_up, 0, sizeof(double) * (size_t)E * (size_t)D * (size_t)F);
    if (dw_down) memset(dw_down, 0, sizeof(double) * (size_t)E * (size_t)F * (size_t)D);
    /* Tokens run in parallel only when no weight gradient (a sum over tokens) is requested:
     * dx rows are per token. */
    const int tokens_independent = !dw_gate && !dw_gate_e && !dw_up && !dw_down;
    #pragma omp parallel if (tokens_independent)
    {
    double *l = (double *)malloc(sizeof(double) * (size_t)E);
    double *a = (double *)malloc(sizeof(double) * (size_t)F);
    double *b = (double *)malloc(sizeof(double) * (size_t)F);
    double *h = (double *)malloc(sizeof(double) * (size_t)F);
    double *dh = (double *)malloc(sizeof(double) * (size_t)F);
    double *da = (double *)malloc(sizeof(double) * (size_t)F);
    double *db = (double *)malloc(sizeof(double) * (size_t)F);
    double *dv = (double *)malloc(sizeof(double) * (size_t)D);
    int32_t J[64];
    double w[64], dwj[64];
    #pragma omp for schedule(dynamic, 1)
    for (int64_t s = 0; s < S; ++s) {
        const float *xs = x + s * D;
        const float *ds = dout + s * D;
        double *dxs = dx + s * D;
        logits_one(xs, w_gate, bias, D, E, l, NULL);
        if (given_top_experts) {
            for (int32_t j = 0; j < k; ++j) J[j] = given_top_experts[s * k + j];
            oracle_weights_for(l, J, 1, E, k, w);
        } else {
            topk_one(l, E, k, J, w);
        }
        for (int32_t j = 0; j < k; ++j) {
            const int64_t e = J[j];
            const float *wge = w_gate_e + e * D * F, *wu = w_up + e * D * F;
            const float *wd = w_down + e * F * D;
            expert_hidden(xs, wge, wu, D, F, a, b, h);
            double dwv = 0.0;
            for (int64_t f = 0; f < F; ++f) {
                double vd_dot = 0.0;  /* (W_down[e] row f) . dout */
                for (int64_t d = 0; d < D; ++d) vd_dot += (double)wd[f * D + d] * (double)ds[d];
                dwv += h[f] * vd_dot;
                dh[f] = w[j] * vd_dot;
            }
            dwj[j] = dwv;
            for (int64_t d = 0; d < D; ++d) dv[d] = w[j] * (double)ds[d];
            if (dw_down) {
                double *dwd = dw_down + e * F * D;
                for (int64_t f = 0; f < F; ++f)
                    for (int64_t d = 0; d < D; ++d) dwd[f * D + d] += h[f] * dv[d];
            }
            for (int64_t f = 0; f < F; ++f) {
                const double sg = 1.0 / (1.0 + exp(-a[f]));
                da[f] = dh[f] * b[f] * sg * (1.0 + a[f] * (1.0 - sg));
                db[f] = dh[f] * a[f] * sg;
            }
            double *dge = dw_gate_e ? dw_gate_e + e * D * F : NULL;
            double *dup = dw_up ? dw_up + e * D * F : NULL;
            for (int64_t d = 0; d < D; ++d) {
                const double xd = (double)xs[d];
                double acc = 0.0;
                if (dge)
                    for (int64_t f = 0; f < F; ++f) dge[d * F + f] += xd * da[f];
                if (dup)
                    for (int64_t f = 0; f < F; ++f) dup[d * F + f] += xd * db[f];
                for (int64_t f = 0; f < F; ++f)
                    acc += da[f] * (double)wge[d * F + f] + db[f] * (double)wu[d * F + f];
                dxs[d] += acc;
            }
        }
        double mean = 0.0;
        for (int32_t j = 0; j < k; ++j) mean += w[j] * dwj[j];
        for (int32_t j = 0; j < k; ++j) {
            const double dl = w[j] * (dwj[j] - mean);
            const int64_t e = J[j];
            for (int64_t d = 0; d < D; ++d) {
                if (dw_gate) dw_gate[d * E + e] += (double)xs[d] * dl;
                dxs[d] += dl * (double)w_gate[d * E + e];
            }
        }
    }
    free(l); free(a); free(b); free(h); free(dh); free(da); free(db); free(dv);
    }
}

/* Mixture of Attention through ParallelLinear (ScatterMoE guide, "2. Generalization to Mixture of
 * Attention (MoA)"; the ScatterMoE abstract's MoA demonstration): the router and top-k softmax
 * of the expert MLP select k of E attention experts per token; expert e owns a query projection
 * W_q[e] [D, H*dh] and an output projection W_o[e] [H*dh, D]; keys and values are shared,
 * K = x W_k, V = x W_v ([S, H*dh]). For token s and selected expert e = J_j, per head h:
 *   q = x_s W_q[e];  o_h = sum_{t <= s} softmax_t(q_h . K[t,h] / sqrt(dh)) V[t,h]  (causal)
 *   y_s += w_j * (o W_o[e]).
 * fp64; routing given ([S, k]) or the oracle's own. Outputs out [S, D] and, nullable, the
 * routing top_experts_out [S, k] / top_weights_out [S, k]. */
/* Mixture of Attention for the query tokens `tokens` (n of them; every token 0..S-1 when tokens
 * is NULL). Keys and values are computed for every token up to the largest query token, so a
 * query's output is the same whichever other tokens are listed. out, top_experts_out and
 * top_weights_out are indexed by list position; given_top_experts by token. */
static void moa_forward_tokens(const float *x, const float *w_gate, const float *bias,
                               const float *w_q, const float *w_k, const float *w_v,
                               const float *w_o, int64_t S, int64_t D, int32_t H, int32_t dh,
                               int32_t E, int32_t k, const int32_t *given_top_experts,
                               const int32_t *tokens, int64_t n, double *out,
                               int32_t *top_experts_out, double *top_weights_out) {
    const int64_t HD = (int64_t)H * dh;
    int64_t S_kv = tokens ? 0 : S;
    for (int64_t i = 0; tokens && i < n; ++i)
        if ((int64_t)tokens[i] + 1 > S_kv) S_kv = (int64_t)tokens[i] + 1;
    double *K = (double *)calloc((size_t)(S_kv > 0 ? S_kv : 1) * (size_t)HD, sizeof(double));
    double *V = (double *)calloc((size_t)(S_kv > 0 ? S_kv : 1) * (size_t)HD, sizeof(double));
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < S_kv; ++t) {
        for (int64_t d = 0; d < D; ++d) {
            const double xv = (double)x[t * D + d];
            for (int64_t c = 0; c < HD; ++c) {
                K[t * HD + c] += xv * (double)w_k[d * HD + c];
                V[t * HD + c] += xv * (double)w_v[d * HD + c];
            }
        }
    }
    const double scale = 1.0 / sqrt((double)dh);
    #pragma omp parallel
    {
        double *l = (double *)malloc(sizeof(double) * (size_t)E);
        double *q = (double *)malloc(sizeof(double) * (size_t)HD);
        double *o = (double *)malloc(sizeof(double) * (size_t)HD);
        double *sc = (double *)malloc(sizeof(double) * (size_t)(S > 0 ? S : 1));
        int32_t J[64];
        double w[64];
        #pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < n; ++i) {
            const int64_t s = tokens ? (int64_t)tokens[i] : i;
            const float *xs = x + s * D;
            logits_one(xs, w_gate, bias, D, E, l, NULL);
            if (given_top_experts) {
                for (int32_t j = 0; j < k; ++j) J[j] = given_top_experts[s * k + j];
                oracle_weights_for(l, J, 1, E, k, w);
            } else {
                topk_one(l, E, k, J, w);
            }
            double *y = out + i * D;
            for (int64_t d = 0; d < D; ++d) y[d] = 0.0;
            for (int32_t j = 0; j < k; ++j) {
                const int64_t e = J[j];
                const float *wq = w_q + e * D * HD, *wo = w_o + e * HD * D;
                for (int64_t c = 0; c < HD; ++c) q[c] = 0.0;
                for (int64_t d = 0; d < D; ++d) {
                    const double xv = (double)xs[d];
                    for (int64_t c = 0; c < HD; ++c) q[c] += xv * (double)wq[d * HD + c];
                }
                for (int32_t h = 0; h < H; ++h) {
                    const double *qh = q + (int64_t)h * dh;
                    double mx = -INFINITY;
                    for (int64_t t = 0; t <= s; ++t) {
                        double acc = 0.0;
                        for (int32_t c = 0; c < dh; ++c) acc += qh[c] * K[t * HD + (int64_t)h * dh + c];
                        sc[t] = acc * scale;
                        if (sc[t] > mx) mx = sc[t];
                    }
                    double den = 0.0;
                    for (int64_t t = 0; t <= s; ++t) {
                        sc[t] = exp(sc[t] - mx);
                        den += sc[t];
                    }
                    double *oh = o + (int64_t)h * dh;
                    for (int32_t c = 0; c < dh; ++c) oh[c] = 0.0;
                    for (int64_t t = 0; t <= s; ++t) {
                        const double pt = sc[t] / den;
                        for (int32_t c = 0; c < dh; ++c) oh[c] += pt * V[t * HD + (int64_t)h * dh + c];
                    }
                }
                for (int64_t c = 0; c < HD; ++c) {
                    const double cw = w[j] * o[c];
                    for (int64_t d = 0; d < D; ++d) y[d] += cw * (double)wo[c * D + d];
                }
            }
            if (top_experts_out)
                for (int32_t j = 0; j < k; ++j) top_experts_out[i * k + j] = J[j];
            if (top_weights_out)
                for (int32_t j = 0; j < k; ++j) top_weights_out[i * k + j] = w[j];
        }
        free(l); free(q); free(o); free(sc);
    }
    free(K);
    free(V);
}

void oracle_moa_forward(const float *x, const float *w_gate, const float *bias, const float *w_q,
                        const float *w_k, const float *w_v, const float *w_o, int64_t S, int64_t D,
                        int32_t H, int32_t dh, int32_t E, int32_t k,
                        const int32_t *given_top_experts, double *out, int32_t *top_experts_out,
                        double *top_weights_out) {
    moa_forward_tokens(x, w_gate, bias, w_q, w_k, w_v, w_o, S, D, H, dh, E, k, given_top_experts,
                       NULL, S, out, top_experts_out, top_weights_out);
}

/* The same for a list of query tokens (outputs [n, D], [n, k] by list position). */
void oracle_moa_forward_tokens(const float *x, const float *w_gate, const float *bias,
                               const float *w_q, const float *w_k, const float *w_v,
                               const float *w_o, int64_t S, int64_t D, int32_t H, int32_t dh,
                               int32_t E, int32_t k, const int32_t *given_top_experts,
                               const int32_t *tokens, int64_t n, double *out,
                               int32_t *top_experts_out, double *top_weights_out) {
    moa_forward_tokens(x, w_gate, bias, w_q, w_k, w_v, w_o, S, D, H, dh, E, k, given_top_experts,
                       tokens, n, out, top_experts_out, top_weights_out);
}
