/*
 * moe_oracle.c -- plain, slow, fp64 CPU oracle for the capacity-limited top-k
 * sparse mixture-of-experts layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link or
 * call this file: only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark load it (through oracle/oracle.py).  It shares no code, header,
 * table or helper with the CUDA library.
 *
 * Every routine is a direct loop transcription of the definition it cites:
 *   [P1] "Sparse MoE Layer in NumPy -- Token Drop, Exact Dispatch/Combine,
 *        Aux Loss & Backward" (ob1.it.com), sections 1-4.
 *   [P2] "Top-k MoE Router with Load Statistics" (tensortonic), problem
 *        statement, Examples, Requirements, Constraints.
 *   [P3] "Module 7. Mixture of Experts" (vladkulikov notebook): functions
 *        stable_softmax, stable_sigmoid, _deterministic_top_k, route_logits,
 *        expert_capacity, dispatch_with_capacity, switch_auxiliary_loss,
 *        router_z_loss, swiglu_expert, EducationalMoE.
 *   [P4] "32. Sparse MoE Token Dispatch & Combine (Capacity-Limited)",
 *        Step-by-Step Approach and Reference solution.
 *   [P5] "mixture-of-experts/3" (llm-atlas): Expert, TopKMoE,
 *        _load_balancing_loss.
 *
 * All arithmetic is double precision.  Matrices are dense row-major.  Expert
 * weights follow the pages' x@W convention: W has shape (E, K_in, N_out) and
 * the expert output row is out[n] = sum_k x[k] * W[e][k][n].
 *
 * OpenMP (when compiled with -fopenmp) only splits the outermost independent
 * loop over tokens or experts; it does not change any summation order.
 *
 * Parity status: every function here is pinned by tests/test_oracle_pins.py
 * (worked examples, closed forms, invariants, brute force, finite
 * differences).  No function is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OMP_FOR _Pragma("omp parallel for schedule(static)")

/* ------------------------------------------------------------------------ */
/* Capacity.  [P3] expert_capacity: ceil(capacity_factor * T * k / E) with a  */
/* floor of 1; [P1] section 1 item 2 states the same ceil.  Evaluated in fp64 */
/* in [P3]'s operand order.  A non-positive factor is rejected (returns -1),  */
/* matching [P3]'s negative test on capacity_factor=0.                        */
/* ------------------------------------------------------------------------ */
int64_t oracle_capacity(int64_t T, int32_t k, int32_t E, double capacity_factor) {
    if (T < 1 || k < 1 || E < 1 || k > E) return -1;
    if (!(capacity_factor > 0.0) || !isfinite(capacity_factor)) return -1;
    double v = capacity_factor * (double)T * (double)k / (double)E;
    int64_t c = (int64_t)ceil(v);
    return c < 1 ? 1 : c;
}

/* ------------------------------------------------------------------------ */
/* Router scores.  [P2] s_{t,e} = x_t^T w_e with w_e column e of w_router     */
/* (D,E); an optional per-expert logit bias b_e is added (the skewed-logit    */
/* workload of the full layer).  [P5] router = Linear(d_model, E, no bias).   */
/* ------------------------------------------------------------------------ */
void oracle_router_logits(const double* x, const double* w_router, const double* bias,
                          int64_t T, int64_t D, int32_t E, double* s) {
    /* Each s[t,e] accumulates its D products in ascending d; the loop nest
     * only walks w_router row by row. */
    OMP_FOR
    for (int64_t t = 0; t < T; ++t) {
        double* acc = s + t * E;
        for (int32_t e = 0; e < E; ++e) acc[e] = 0.0;
        for (int64_t d = 0; d < D; ++d) {
            const double xv = x[t * D + d];
            const double* wr = w_router + d * E;
            for (int32_t e = 0; e < E; ++e) acc[e] += xv * wr[e];
        }
        for (int32_t e = 0; e < E; ++e) acc[e] += bias ? bias[e] : 0.0;
    }
}

/* Router backward: s = x w_router + b is linear in x, w_router and b, so for
 * the gradient g = dL/ds (T, E):
 *   dx[t,d] = sum_e g[t,e] w_router[d,e],  dw[d,e] = sum_t x[t,d] g[t,e],
 *   db[e] = sum_t g[t,e].                                                     */
void oracle_router_backward(const double* x, const double* w_router, const double* g, int64_t T,
                            int64_t D, int32_t E, double* dx, double* dw, double* db) {
    OMP_FOR
    for (int64_t t = 0; t < T; ++t)
        for (int64_t d = 0; d < D; ++d) {
            double acc = 0.0;
            for (int32_t e = 0; e < E; ++e) acc += g[t * E + e] * w_router[d * E + e];
            dx[t * D + d] = acc;
        }
    OMP_FOR
    for (int64_t d = 0; d < D; ++d)
        for (int32_t e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int64_t t = 0; t < T; ++t) acc += x[t * D + d] * g[t * E + e];
            dw[d * E + e] = acc;
        }
    for (int32_t e = 0; e < E; ++e) {
        double acc = 0.0;
        for (int64_t t = 0; t < T; ++t) acc += g[t * E + e];
        db[e] = acc;
    }
}

/* ------------------------------------------------------------------------ */
/* Routing.  For each token:                                                  */
/*  - softmax over all E experts with the maximum subtracted first           */
/*    ([P3] stable_softmax; [P1] section 2 top_k_gating; [P2] m_e uses it);  */
/*  - top-k by descending score, exact ties to the lower expert index         */
/*    ([P2] problem statement and Requirements; [P3] _deterministic_top_k     */
/*    ranks raw logits with a lexicographic (score desc, index asc) key).     */
/*    Done here as k selection passes: each pass scans experts in ascending   */
/*    order and takes a strictly larger score, so the lowest index wins ties; */
/*  - gates alpha_{t,j} = exp(s_j) / sum_r exp(s_r) over the selected experts */
/*    ([P2] alpha formula; [P3] route_logits: renormalising the softmax over  */
/*    the top-k equals a softmax of the selected logits);                     */
/*  - counts count_e = #{(t,j): e_{t,j} = e} taken before any capacity drop */
/*    ([P1] section 1 item 6; [P3] route_logits expert_counts)               */
/*  - prob_sum_e = sum_t softmax(s_t)_e  ([P2] m_e before the 1/T).           */
/* ------------------------------------------------------------------------ */
void oracle_route(const double* s, int64_t T, int32_t E, int32_t k,
                  double* probs, int64_t* selected, double* gates,
                  int64_t* counts, double* prob_sum) {
    OMP_FOR
    for (int64_t t = 0; t < T; ++t) {
        const double* st = s + t * E;
        double mx = st[0];
        for (int32_t e = 1; e < E; ++e) if (st[e] > mx) mx = st[e];
        double den = 0.0;
        for (int32_t e = 0; e < E; ++e) den += exp(st[e] - mx);
        for (int32_t e = 0; e < E; ++e) probs[t * E + e] = exp(st[e] - mx) / den;

        char* taken = (char*)calloc((size_t)E, 1);
        for (int32_t j = 0; j < k; ++j) {
            int32_t best = -1;
            for (int32_t e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || st[e] > st[best]) best = e;
            }
            taken[best] = 1;
            selected[t * k + j] = best;
        }
        free(taken);

        double smax = st[selected[t * k + 0]];
        for (int32_t j = 1; j < k; ++j) if (st[selected[t * k + j]] > smax) smax = st[selected[t * k + j]];
        double gden = 0.0;
        for (int32_t j = 0; j < k; ++j) gden += exp(st[selected[t * k + j]] - smax);
        for (int32_t j = 0; j < k; ++j) gates[t * k + j] = exp(st[selected[t * k + j]] - smax) / gden;
    }
    for (int32_t e = 0; e < E; ++e) { counts[e] = 0; prob_sum[e] = 0.0; }
    for (int64_t t = 0; t < T; ++t) {
        for (int32_t j = 0; j < k; ++j) counts[selected[t * k + j]] += 1;
        for (int32_t e = 0; e < E; ++e) prob_sum[e] += probs[t * E + e];
    }
}

/* ------------------------------------------------------------------------ */
/* Greedy position-priority slot assignment ([P1] section 2                   */
/* position_priority_dispatch; [P3] dispatch_with_capacity, FIFO policy;      */
/* [P4] Problem: earlier tokens claim an expert's buffer first).  Tokens in   */
/* order, route slots j in selection (descending gate) order; an assignment   */
/* is kept iff its expert has fewer than C accepted rows so far.              */
/*   slot[t,j]   = rank among the expert's accepted rows, -1 when dropped     */
/*   kept[t,j]   = 1 / 0                                                       */
/*   used[e]     = accepted rows of e (= min(count_e, C))                      */
/*   overflow[e] = attempts - used  ([P1] section 1 item 3: one overflow per   */
/*                 rejected assignment)                                        */
/*   drops[t]    = number of dropped assignments of token t                    */
/*   token_of_slot[e,c] = token placed in (e,c), -1 when the slot is empty.    */
/* An index outside [0,E) is reported (return value -1) and not placed; the   */
/* pages reject such inputs ([P3] dispatch_with_capacity index check).        */
/* ------------------------------------------------------------------------ */
int oracle_dispatch(const int64_t* selected, int64_t T, int32_t k, int32_t E, int64_t C,
                    int64_t* slot, uint8_t* kept, int64_t* used, int64_t* overflow,
                    int64_t* drops, int64_t* token_of_slot) {
    int bad = 0;
    int64_t* attempts = (int64_t*)calloc((size_t)E, sizeof(int64_t));
    for (int32_t e = 0; e < E; ++e) used[e] = 0;
    for (int64_t i = 0; i < (int64_t)E * C; ++i) token_of_slot[i] = -1;
    for (int64_t t = 0; t < T; ++t) {
        drops[t] = 0;
        for (int32_t j = 0; j < k; ++j) {
            int64_t e = selected[t * k + j];
            slot[t * k + j] = -1;
            kept[t * k + j] = 0;
            if (e < 0 || e >= E) { bad = 1; drops[t] += 1; continue; }
            attempts[e] += 1;
            if (used[e] < C) {
                slot[t * k + j] = used[e];
                kept[t * k + j] = 1;
                token_of_slot[e * C + used[e]] = t;
                used[e] += 1;
            } else {
                drops[t] += 1;
            }
        }
    }
    for (int32_t e = 0; e < E; ++e) overflow[e] = attempts[e] - used[e];
    free(attempts);
    return bad ? -1 : 0;
}

/* ------------------------------------------------------------------------ */
/* Expert functions, one token row at a time.                                 */
/* ------------------------------------------------------------------------ */

/* Logistic sigmoid in the overflow-free two-branch form of [P3] stable_sigmoid. */
static double sigmoid_stable(double z) {
    if (z >= 0.0) return 1.0 / (1.0 + exp(-z));
    double ez = exp(z);
    return ez / (1.0 + ez);
}

/* Exact (erf) GELU, as torch.nn.functional.gelu defaults to in [P5] Expert. */
static double gelu_erf(double z) { return 0.5 * z * (1.0 + erf(z / sqrt(2.0))); }

/* Linear expert out = x @ W[e]  ([P1] section 2 expert einsum; [P4] bmm).
 * W: (E, D, N). */
void oracle_expert_linear_row(const double* xrow, const double* W, int32_t e,
                              int64_t D, int64_t N, double* out) {
    const double* We = W + (int64_t)e * D * N;
    for (int64_t n = 0; n < N; ++n) out[n] = 0.0;
    for (int64_t d = 0; d < D; ++d)        /* out[n] sums over d ascending */
        for (int64_t n = 0; n < N; ++n) out[n] += xrow[d] * We[d * N + n];
}

/* Two-layer GELU MLP with biases ([P5] Expert: fc2(gelu(fc1(x)))).
 * W1: (E, D, F), b1: (E, F), W2: (E, F, N), b2: (E, N). */
void oracle_expert_gelu_row(const double* xrow, const double* W1, const double* b1,
                            const double* W2, const double* b2, int32_t e,
                            int64_t D, int64_t F, int64_t N, double* out) {
    double* h = (double*)malloc((size_t)F * sizeof(double));
    const double* W1e = W1 + (int64_t)e * D * F;
    const double* W2e = W2 + (int64_t)e * F * N;
    for (int64_t f = 0; f < F; ++f) h[f] = 0.0;
    for (int64_t d = 0; d < D; ++d)
        for (int64_t f = 0; f < F; ++f) h[f] += xrow[d] * W1e[d * F + f];
    for (int64_t f = 0; f < F; ++f) h[f] = gelu_erf(h[f] + b1[(int64_t)e * F + f]);
    for (int64_t n = 0; n < N; ++n) out[n] = 0.0;
    for (int64_t f = 0; f < F; ++f)
        for (int64_t n = 0; n < N; ++n) out[n] += h[f] * W2e[f * N + n];
    for (int64_t n = 0; n < N; ++n) out[n] += b2[(int64_t)e * N + n];
    free(h);
}

/* SwiGLU expert ([P3] swiglu_expert: (g * sigmoid(g) * u) @ down with
 * g = x @ gate, u = x @ up).  Wg, Wu: (E, D, F); Wd: (E, F, N). */
void oracle_expert_swiglu_row(const double* xrow, const double* Wg, const double* Wu,
                              const double* Wd, int32_t e, int64_t D, int64_t F, int64_t N,
                              double* out) {
    double* h = (double*)malloc((size_t)F * sizeof(double));
    const double* Wge = Wg + (int64_t)e * D * F;
    const double* Wue = Wu + (int64_t)e * D * F;
    const double* Wde = Wd + (int64_t)e * F * N;
    double* u = (double*)malloc((size_t)F * sizeof(double));
    for (int64_t f = 0; f < F; ++f) { h[f] = 0.0; u[f] = 0.0; }
    for (int64_t d = 0; d < D; ++d)
        for (int64_t f = 0; f < F; ++f) { h[f] += xrow[d] * Wge[d * F + f]; u[f] += xrow[d] * Wue[d * F + f]; }
    for (int64_t f = 0; f < F; ++f) h[f] = h[f] * sigmoid_stable(h[f]) * u[f];
    for (int64_t n = 0; n < N; ++n) out[n] = 0.0;
    for (int64_t f = 0; f < F; ++f)
        for (int64_t n = 0; n < N; ++n) out[n] += h[f] * Wde[f * N + n];
    free(u);
    free(h);
}

/* kind: 0 linear, 1 GELU MLP, 2 SwiGLU.  Weight arguments as above; unused
 * ones may be NULL. */
static void expert_row(int kind, const double* xrow, const double* w1, const double* b1,
                       const double* w2, const double* b2, const double* w3, int32_t e,
                       int64_t D, int64_t F, int64_t N, double* out) {
    if (kind == 0) oracle_expert_linear_row(xrow, w1, e, D, N, out);
    else if (kind == 1) oracle_expert_gelu_row(xrow, w1, b1, w2, b2, e, D, F, N, out);
    else oracle_expert_swiglu_row(xrow, w1, w3, w2, e, D, F, N, out);
}

/* ------------------------------------------------------------------------ */
/* Sparse layer output for a list of tokens.                                   */
/*   y_t = base_t + sum_{j kept} gate[t,j] * Expert_{e_{t,j}}(x_t)             */
/* ([P1] section 1 item 4: y = x + sum_kept gate * Expert(x); [P2] y_t =        */
/* u_shared + sum_j alpha_j u_{t,e_j}; [P4]/[P5] base 0: a dropped token row    */
/* is all zero).  base_kind: 0 zero, 1 the input row x_t (residual; needs       */
/* N == D), 2 the given base row (e.g. a shared-expert output).                */
/* Only the tokens listed in `tokens` (n_tokens of them) are computed; row i   */
/* of y belongs to tokens[i].                                                   */
/* ------------------------------------------------------------------------ */
void oracle_layer_rows(int kind, const double* x, int64_t T, int64_t D,
                       const int64_t* selected, const uint8_t* kept, const double* gates,
                       int32_t k, const double* w1, const double* b1, const double* w2,
                       const double* b2, const double* w3, int64_t F, int64_t N,
                       int base_kind, const double* base, const int64_t* tokens,
                       int64_t n_tokens, double* y) {
    (void)T;
    OMP_FOR
    for (int64_t i = 0; i < n_tokens; ++i) {
        int64_t t = tokens[i];
        const double* xrow = x + t * D;
        double* yrow = y + i * N;
        double* out = (double*)malloc((size_t)N * sizeof(double));
        for (int64_t n = 0; n < N; ++n)
            yrow[n] = base_kind == 1 ? xrow[n] : (base_kind == 2 ? base[t * N + n] : 0.0);
        for (int32_t j = 0; j < k; ++j) {
            if (!kept[t * k + j]) continue;
            expert_row(kind, xrow, w1, b1, w2, b2, w3, (int32_t)selected[t * k + j], D, F, N, out);
            for (int64_t n = 0; n < N; ++n) yrow[n] += gates[t * k + j] * out[n];
        }
        free(out);
    }
}

/* Expert outputs (no gate) for a list of kept (token, expert) pairs: the
 * content of the expert-major output buffer at (e, slot). */
void oracle_expert_rows(int kind, const double* x, int64_t D, const int64_t* tokens,
                        const int64_t* experts, int64_t n_rows, const double* w1,
                        const double* b1, const double* w2, const double* b2,
                        const double* w3, int64_t F, int64_t N, double* out) {
    OMP_FOR
    for (int64_t i = 0; i < n_rows; ++i)
        expert_row(kind, x + tokens[i] * D, w1, b1, w2, b2, w3, (int32_t)experts[i], D, F, N,
                   out + i * N);
}

/* ------------------------------------------------------------------------ */
/* Load statistics and the Switch auxiliary loss.                              */
/*   f_e = count_e / T            ([P2] token_fraction; [P5] f)                */
/*   P_e = prob_sum_e / T         ([P2] probability_mass m_e; [P5] P)          */
/*   aux = E * sum_e (count_e / (T * kn)) * P_e                                */
/* with kn = k when normalize_by_k ([P1] section 1 item 6 and [P3]             */
/* switch_auxiliary_loss: f = count/(T*k), aux = 1 at uniform routing) and     */
/* kn = 1 otherwise ([P5] _load_balancing_loss).                               */
/* ------------------------------------------------------------------------ */
void oracle_aux(const int64_t* counts, const double* prob_sum, int64_t T, int32_t E, int32_t k,
                int normalize_by_k, double* f, double* P, double* aux) {
    double kn = normalize_by_k ? (double)k : 1.0;
    double acc = 0.0;
    for (int32_t e = 0; e < E; ++e) {
        f[e] = (double)counts[e] / (double)T;
        P[e] = prob_sum[e] / (double)T;
        acc += ((double)counts[e] / ((double)T * kn)) * P[e];
    }
    *aux = (double)E * acc;
}

/* Router z-loss mean_t(logsumexp(s_t)^2)  ([P3] router_z_loss). */
double oracle_z_loss(const double* s, int64_t T, int32_t E) {
    double acc = 0.0;
    for (int64_t t = 0; t < T; ++t) {
        double mx = s[t * E];
        for (int32_t e = 1; e < E; ++e) if (s[t * E + e] > mx) mx = s[t * E + e];
        double den = 0.0;
        for (int32_t e = 0; e < E; ++e) den += exp(s[t * E + e] - mx);
        double lse = mx + log(den);
        acc += lse * lse;
    }
    return acc / (double)T;
}

/* ------------------------------------------------------------------------ */
/* Backward of the linear-expert layer with the kept mask held constant        */
/* ([P1] section 1 item 7: quotient rule + softmax Jacobian, discrete drops    */
/* are constants; section 2 moe_backward: dM, dW, dx, dcombine).               */
/*                                                                              */
/* Loss L = sum_t dy_t . y_t + aux_coef * aux with                             */
/*   y_t = [x_t] + sum_{j kept} gate_{t,j} * (x_t @ W[e_{t,j}]).               */
/*   dgate[t,j]  = kept ? dy_t . (x_t @ W[e]) : 0                              */
/*   dlogits[t,e_i] = gate_i * (dgate_i - sum_j gate_j dgate_j), 0 elsewhere   */
/*     (gate = softmax of the selected logits, so its Jacobian is              */
/*      gate_j (delta_ij - gate_i)).                                          */
/*   + aux term: aux = E sum_e c_e/(T kn) * (1/T) sum_t p[t,e] with counts c   */
/*     constant, and dp[t,e']/ds[t,e] = p[t,e'](delta - p[t,e]), giving        */
/*     aux_coef * E/(T*T*kn) * p[t,e] * (c_e - sum_e' c_e' p[t,e']).           */
/*   dW[e][a][b] = sum_{kept (t,j): e_{t,j}=e} gate * x[t][a] * dy[t][b]       */
/*   dx[t][a]    = [dy[t][a]] + sum_{kept j} gate_j * sum_b dy[t][b] W[e][a][b] */
/* W: (E, D, N); residual requires N == D.                                     */
/* ------------------------------------------------------------------------ */
void oracle_backward_linear(const double* dy, const double* x, const double* s,
                            const int64_t* selected, const uint8_t* kept, const double* gates,
                            const double* W, int64_t T, int32_t k, int32_t E, int64_t D,
                            int64_t N, int use_residual, double aux_coef, int normalize_by_k,
                            const int64_t* counts, double* dx, double* dW, double* dlogits,
                            double* dgate) {
    /* dgate and dlogits */
    OMP_FOR
    for (int64_t t = 0; t < T; ++t) {
        double* out = (double*)malloc((size_t)N * sizeof(double));
        for (int32_t j = 0; j < k; ++j) {
            dgate[t * k + j] = 0.0;
            if (!kept[t * k + j]) continue;
            oracle_expert_linear_row(x + t * D, W, (int32_t)selected[t * k + j], D, N, out);
            double acc = 0.0;
            for (int64_t n = 0; n < N; ++n) acc += dy[t * N + n] * out[n];
            dgate[t * k + j] = acc;
        }
        free(out);
        for (int32_t e = 0; e < E; ++e) dlogits[t * E + e] = 0.0;
        double gdot = 0.0;
        for (int32_t j = 0; j < k; ++j) gdot += gates[t * k + j] * dgate[t * k + j];
        for (int32_t i = 0; i < k; ++i)
            dlogits[t * E + selected[t * k + i]] += gates[t * k + i] * (dgate[t * k + i] - gdot);
        if (aux_coef != 0.0) {
            double kn = normalize_by_k ? (double)k : 1.0;
            const double* st = s + t * E;
            double mx = st[0];
            for (int32_t e = 1; e < E; ++e) if (st[e] > mx) mx = st[e];
            double den = 0.0;
            for (int32_t e = 0; e < E; ++e) den += exp(st[e] - mx);
            double cp = 0.0;
            for (int32_t e = 0; e < E; ++e) cp += (double)counts[e] * (exp(st[e] - mx) / den);
            double scale = aux_coef * (double)E / ((double)T * (double)T * kn);
            for (int32_t e = 0; e < E; ++e) {
                double p = exp(st[e] - mx) / den;
                dlogits[t * E + e] += scale * p * ((double)counts[e] - cp);
            }
        }
    }
    /* dW, one expert per iteration */
    OMP_FOR
    for (int32_t e = 0; e < E; ++e) {
        double* dWe = dW + (int64_t)e * D * N;
        for (int64_t i = 0; i < D * N; ++i) dWe[i] = 0.0;
        for (int64_t t = 0; t < T; ++t) {
            for (int32_t j = 0; j < k; ++j) {
                if (!kept[t * k + j] || selected[t * k + j] != e) continue;
                double g = gates[t * k + j];
                for (int64_t a = 0; a < D; ++a) {
                    double gx = g * x[t * D + a];
                    for (int64_t b = 0; b < N; ++b) dWe[a * N + b] += gx * dy[t * N + b];
                }
            }
        }
    }
    /* dx */
    OMP_FOR
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t a = 0; a < D; ++a) dx[t * D + a] = use_residual ? dy[t * N + a] : 0.0;
        for (int32_t j = 0; j < k; ++j) {
            if (!kept[t * k + j]) continue;
            const double* We = W + selected[t * k + j] * D * N;
            double g = gates[t * k + j];
            for (int64_t a = 0; a < D; ++a) {
                double acc = 0.0;
                for (int64_t b = 0; b < N; ++b) acc += dy[t * N + b] * We[a * N + b];
                dx[t * D + a] += g * acc;
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Backward of the SwiGLU-expert layer with the kept mask constant (the        */
/* [P1] section 1 item 7 backward carried over to [P3] swiglu_expert).  For a   */
/* kept assignment of token t to expert e with gate g:                          */
/*   a = x Wg_e, b = x Wu_e, h = silu(a) * b, o = h Wd_e,  y_t += g o           */
/* and for the upstream gradient dy_t:                                          */
/*   dgate = dy_t . o,  do = g dy_t,  dh = do Wd_e^T,                           */
/*   da = dh * b * silu'(a),  db = dh * silu(a),  silu'(a) = s (1 + a (1 - s)), */
/*   s = sigmoid(a);  dWd_e += h^T do,  dWg_e += x^T da,  dWu_e += x^T db,      */
/*   dx_t += da Wg_e^T + db Wu_e^T  (+ dy_t with the residual base).           */
/* dlogits follows from dgate exactly as in the linear case.  Weights in the    */
/* x@W layout: Wg, Wu (E, D, F); Wd (E, F, N).                                  */
/* ------------------------------------------------------------------------ */

/* One kept assignment: recompute the forward quantities and the gradients of
 * the expert's hidden layer.  a, b, h, da, db: (F); o: (N). */
static void swiglu_assignment(const double* xrow, const double* dyrow, double g, const double* Wge,
                              const double* Wue, const double* Wde, int64_t D, int64_t F, int64_t N,
                              double* a, double* b, double* h, double* o, double* da, double* db,
                              double* dgate_out) {
    for (int64_t f = 0; f < F; ++f) { a[f] = 0.0; b[f] = 0.0; }
    for (int64_t d = 0; d < D; ++d)
        for (int64_t f = 0; f < F; ++f) {
            a[f] += xrow[d] * Wge[d * F + f];
            b[f] += xrow[d] * Wue[d * F + f];
        }
    for (int64_t f = 0; f < F; ++f) h[f] = a[f] * sigmoid_stable(a[f]) * b[f];
    for (int64_t n = 0; n < N; ++n) o[n] = 0.0;
    for (int64_t f = 0; f < F; ++f)
        for (int64_t n = 0; n < N; ++n) o[n] += h[f] * Wde[f * N + n];
    double dg = 0.0;
    for (int64_t n = 0; n < N; ++n) dg += dyrow[n] * o[n];
    *dgate_out = dg;
    for (int64_t f = 0; f < F; ++f) {
        double dh = 0.0;
        for (int64_t n = 0; n < N; ++n) dh += g * dyrow[n] * Wde[f * N + n];
        const double sg = sigmoid_stable(a[f]);
        da[f] = dh * b[f] * sg * (1.0 + a[f] * (1.0 - sg));
        db[f] = dh * a[f] * sg;
    }
}

void oracle_backward_swiglu(const double* dy, const double* x, const double* s,
                            const int64_t* selected, const uint8_t* kept, const double* gates,
                            const double* Wg, const double* Wu, const double* Wd, int64_t T,
                            int32_t k, int32_t E, int64_t D, int64_t F, int64_t N,
                            int use_residual, double aux_coef, int normalize_by_k,
                            const int64_t* counts, double* dx, double* dWg, double* dWu,
                            double* dWd, double* dlogits, double* dgate) {
    /* per token: dgate, dlogits, dx */
    OMP_FOR
    for (int64_t t = 0; t < T; ++t) {
        double* a = (double*)malloc((size_t)(5 * F + N) * sizeof(double));
        double *b = a + F, *h = b + F, *da = h + F, *db = da + F, *o = db + F;
        for (int64_t d = 0; d < D; ++d) dx[t * D + d] = use_residual ? dy[t * N + d] : 0.0;
        for (int32_t j = 0; j < k; ++j) {
            dgate[t * k + j] = 0.0;
            if (!kept[t * k + j]) continue;
            const int64_t e = selected[t * k + j];
            const double* Wge = Wg + e * D * F;
            const double* Wue = Wu + e * D * F;
            swiglu_assignment(x + t * D, dy + t * N, gates[t * k + j], Wge, Wue, Wd + e * F * N, D, F, N,
                              a, b, h, o, da, db, &dgate[t * k + j]);
            for (int64_t d = 0; d < D; ++d) {
                double acc = 0.0;
                for (int64_t f = 0; f < F; ++f) acc += da[f] * Wge[d * F + f] + db[f] * Wue[d * F + f];
                dx[t * D + d] += acc;
            }
        }
        free(a);
        for (int32_t e = 0; e < E; ++e) dlogits[t * E + e] = 0.0;
        double gdot = 0.0;
        for (int32_t j = 0; j < k; ++j) gdot += gates[t * k + j] * dgate[t * k + j];
        for (int32_t i = 0; i < k; ++i)
            dlogits[t * E + selected[t * k + i]] += gates[t * k + i] * (dgate[t * k + i] - gdot);
        if (aux_coef != 0.0) {
            double kn = normalize_by_k ? (double)k : 1.0;
            const double* st = s + t * E;
            double mx = st[0];
            for (int32_t e = 1; e < E; ++e) if (st[e] > mx) mx = st[e];
            double den = 0.0;
            for (int32_t e = 0; e < E; ++e) den += exp(st[e] - mx);
            double cp = 0.0;
            for (int32_t e = 0; e < E; ++e) cp += (double)counts[e] * (exp(st[e] - mx) / den);
            double scale = aux_coef * (double)E / ((double)T * (double)T * kn);
            for (int32_t e = 0; e < E; ++e) {
                double p = exp(st[e] - mx) / den;
                dlogits[t * E + e] += scale * p * ((double)counts[e] - cp);
            }
        }
    }
    /* weight gradients, one expert per iteration */
    OMP_FOR
    for (int32_t e = 0; e < E; ++e) {
        double* a = (double*)malloc((size_t)(5 * F + N) * sizeof(double));
        double *b = a + F, *h = b + F, *da = h + F, *db = da + F, *o = db + F;
        double* dWge = dWg + (int64_t)e * D * F;
        double* dWue = dWu + (int64_t)e * D * F;
        double* dWde = dWd + (int64_t)e * F * N;
        for (int64_t i = 0; i < D * F; ++i) { dWge[i] = 0.0; dWue[i] = 0.0; }
        for (int64_t i = 0; i < F * N; ++i) dWde[i] = 0.0;
        for (int64_t t = 0; t < T; ++t) {
            for (int32_t j = 0; j < k; ++j) {
                if (!kept[t * k + j] || selected[t * k + j] != e) continue;
                const double g = gates[t * k + j];
                double unused;
                swiglu_assignment(x + t * D, dy + t * N, g, Wg + (int64_t)e * D * F, Wu + (int64_t)e * D * F,
                                  Wd + (int64_t)e * F * N, D, F, N, a, b, h, o, da, db, &unused);
                for (int64_t f = 0; f < F; ++f)
                    for (int64_t n = 0; n < N; ++n) dWde[f * N + n] += h[f] * g * dy[t * N + n];
                for (int64_t d = 0; d < D; ++d)
                    for (int64_t f = 0; f < F; ++f) {
                        dWge[d * F + f] += x[t * D + d] * da[f];
                        dWue[d * F + f] += x[t * D + d] * db[f];
                    }
            }
        }
        free(a);
    }
}

/* ------------------------------------------------------------------------ */
/* Backward of the GELU-MLP-expert layer ([P5] Expert, fc2(gelu(fc1(x)))),     */
/* the kept mask constant as in [P1] section 1 item 7.  For a kept assignment   */
/* of token t to expert e with gate g:                                          */
/*   z = x W1_e + b1_e,  h = gelu(z),  o = h W2_e + b2_e,  y_t += g o           */
/* and for the upstream gradient dy_t:                                          */
/*   dgate = dy_t . o,  do = g dy_t,  dh = do W2_e^T,                           */
/*   dz = dh * gelu'(z),  gelu'(z) = Phi(z) + z phi(z)  (the derivative of     */
/*   z Phi(z), Phi the standard normal CDF, phi its density),                   */
/*   dW2_e += h^T do,  db2_e += do,  dW1_e += x^T dz,  db1_e += dz,             */
/*   dx_t += dz W1_e^T  (+ dy_t with the residual base).                        */
/* dlogits follows from dgate as in the linear case.  Weights in the x@W        */
/* layout: W1 (E, D, F), b1 (E, F), W2 (E, F, N), b2 (E, N).                    */
/* ------------------------------------------------------------------------ */

static double gelu_erf_grad(double z) {
    const double cdf = 0.5 * (1.0 + erf(z / sqrt(2.0)));
    const double pdf = exp(-0.5 * z * z) / sqrt(2.0 * acos(-1.0));
    return cdf + z * pdf;
}

/* One kept assignment: z, h (F), o (N), dz (F) and dgate. */
static void gelu_assignment(const double* xrow, const double* dyrow, double g, const double* W1e,
                            const double* b1e, const double* W2e, const double* b2e, int64_t D, int64_t F,
                            int64_t N, double* z, double* h, double* o, double* dz, double* dgate_out) {
    for (int64_t f = 0; f < F; ++f) z[f] = 0.0;
    for (int64_t d = 0; d < D; ++d)
        for (int64_t f = 0; f < F; ++f) z[f] += xrow[d] * W1e[d * F + f];
    for (int64_t f = 0; f < F; ++f) {
        z[f] += b1e[f];
        h[f] = gelu_erf(z[f]);
    }
    for (int64_t n = 0; n < N; ++n) o[n] = b2e[n];
    for (int64_t f = 0; f < F; ++f)
        for (int64_t n = 0; n < N; ++n) o[n] += h[f] * W2e[f * N + n];
    double dg = 0.0;
    for (int64_t n = 0; n < N; ++n) dg += dyrow[n] * o[n];
    *dgate_out = dg;
    for (int64_t f = 0; f < F; ++f) {
        double dh = 0.0;
        for (int64_t n = 0; n < N; ++n) dh += g * dyrow[n] * W2e[f * N + n];
        dz[f] = dh * gelu_erf_grad(z[f]);
    }
}

void oracle_backward_gelu(const double* dy, const double* x, const double* s, const int64_t* selected,
                          const uint8_t* kept, const double* gates, const double* W1, const double* b1,
                          const double* W2, const double* b2, int64_t T, int32_t k, int32_t E, int64_t D,
                          int64_t F, int64_t N, int use_residual, double aux_coef, int normalize_by_k,
                          const int64_t* counts, double* dx, double* dW1, double* db1, double* dW2, double* db2,
                          double* dlogits, double* dgate) {
    /* per token: dgate, dlogits, dx */
    OMP_FOR
    for (int64_t t = 0; t < T; ++t) {
        double* z = (double*)malloc((size_t)(3 * F + N) * sizeof(double));
        double *h = z + F, *dz = h + F, *o = dz + F;
        for (int64_t d = 0; d < D; ++d) dx[t * D + d] = use_residual ? dy[t * N + d] : 0.0;
        for (int32_t j = 0; j < k; ++j) {
            dgate[t * k + j] = 0.0;
            if (!kept[t * k + j]) continue;
            const int64_t e = selected[t * k + j];
            const double* W1e = W1 + e * D * F;
            gelu_assignment(x + t * D, dy + t * N, gates[t * k + j], W1e, b1 + e * F, W2 + e * F * N, b2 + e * N,
                            D, F, N, z, h, o, dz, &dgate[t * k + j]);
            for (int64_t d = 0; d < D; ++d) {
                double acc = 0.0;
                for (int64_t f = 0; f < F; ++f) acc += dz[f] * W1e[d * F + f];
                dx[t * D + d] += acc;
            }
        }
        free(z);
        for (int32_t e = 0; e < E; ++e) dlogits[t * E + e] = 0.0;
        double gdot = 0.0;
        for (int32_t j = 0; j < k; ++j) gdot += gates[t * k + j] * dgate[t * k + j];
        for (int32_t i = 0; i < k; ++i)
            dlogits[t * E + selected[t * k + i]] += gates[t * k + i] * (dgate[t * k + i] - gdot);
        if (aux_coef != 0.0) {
            double kn = normalize_by_k ? (double)k : 1.0;
            const double* st = s + t * E;
            double mx = st[0];
            for (int32_t e = 1; e < E; ++e) if (st[e] > mx) mx = st[e];
            double den = 0.0;
            for (int32_t e = 0; e < E; ++e) den += exp(st[e] - mx);
            double cp = 0.0;
            for (int32_t e = 0; e < E; ++e) cp += (double)counts[e] * (exp(st[e] - mx) / den);
            double scale = aux_coef * (double)E / ((double)T * (double)T * kn);
            for (int32_t e = 0; e < E; ++e) {
                double p = exp(st[e] - mx) / den;
                dlogits[t * E + e] += scale * p * ((double)counts[e] - cp);
            }
        }
    }
    /* weight and bias gradients, one expert per iteration */
    OMP_FOR
    for (int32_t e = 0; e < E; ++e) {
        double* z = (double*)malloc((size_t)(3 * F + N) * sizeof(double));
        double *h = z + F, *dz = h + F, *o = dz + F;
        double* dW1e = dW1 + (int64_t)e * D * F;
        double* dW2e = dW2 + (int64_t)e * F * N;
        double* db1e = db1 + (int64_t)e * F;
        double* db2e = db2 + (int64_t)e * N;
        for (int64_t i = 0; i < D * F; ++i) dW1e[i] = 0.0;
        for (int64_t i = 0; i < F * N; ++i) dW2e[i] = 0.0;
        for (int64_t f = 0; f < F; ++f) db1e[f] = 0.0;
        for (int64_t n = 0; n < N; ++n) db2e[n] = 0.0;
        for (int64_t t = 0; t < T; ++t) {
            for (int32_t j = 0; j < k; ++j) {
                if (!kept[t * k + j] || selected[t * k + j] != e) continue;
                const double g = gates[t * k + j];
                double unused;
                gelu_assignment(x + t * D, dy + t * N, g, W1 + (int64_t)e * D * F, b1 + (int64_t)e * F,
                                W2 + (int64_t)e * F * N, b2 + (int64_t)e * N, D, F, N, z, h, o, dz, &unused);
                for (int64_t f = 0; f < F; ++f)
                    for (int64_t n = 0; n < N; ++n) dW2e[f * N + n] += h[f] * g * dy[t * N + n];
                for (int64_t n = 0; n < N; ++n) db2e[n] += g * dy[t * N + n];
                for (int64_t d = 0; d < D; ++d)
                    for (int64_t f = 0; f < F; ++f) dW1e[d * F + f] += x[t * D + d] * dz[f];
                for (int64_t f = 0; f < F; ++f) db1e[f] += dz[f];
            }
        }
        free(z);
    }
}

/* ------------------------------------------------------------------------ */
/* Dense reference with the explicit (T,E,C) tensors ([P1] section 1 item 5:   */
/* dispatch_mask (T,E,C) bool and combine_weights (T,E,C), zero on dropped     */
/* slots; section 2: M = combine.sum(axis=2), xe = x @ W for every (t,e),      */
/* out = sum_e M[t,e] xe[t,e]; section 3: "an independent dense reference      */
/* loops over all experts").  Linear experts only.  For tiny cases.            */
/* ------------------------------------------------------------------------ */
void oracle_dense_linear(const double* x, const int64_t* selected, const int64_t* slot,
                         const uint8_t* kept, const double* gates, const double* W,
                         int64_t T, int32_t k, int32_t E, int64_t C, int64_t D, int64_t N,
                         int use_residual, uint8_t* dispatch_mask, double* combine_weights,
                         double* y) {
    memset(dispatch_mask, 0, (size_t)(T * E * C));
    for (int64_t i = 0; i < T * E * C; ++i) combine_weights[i] = 0.0;
    for (int64_t t = 0; t < T; ++t)
        for (int32_t j = 0; j < k; ++j)
            if (kept[t * k + j]) {
                int64_t idx = (t * E + selected[t * k + j]) * C + slot[t * k + j];
                dispatch_mask[idx] = 1;
                combine_weights[idx] = gates[t * k + j];
            }
    double* xe = (double*)malloc((size_t)N * sizeof(double));
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t n = 0; n < N; ++n) y[t * N + n] = use_residual ? x[t * D + n] : 0.0;
        for (int32_t e = 0; e < E; ++e) {
            double M = 0.0;
            for (int64_t c = 0; c < C; ++c) M += combine_weights[(t * E + e) * C + c];
            oracle_expert_linear_row(x + t * D, W, e, D, N, xe);
            for (int64_t n = 0; n < N; ++n) y[t * N + n] += M * xe[n];
        }
    }
    free(xe);
}

/* ------------------------------------------------------------------------ */
/* Combine from given expert outputs.                                          */
/*  (a) [P2] form: u is (T, E, N), the output of every expert for every        */
/*      token; y_t = base_t + sum_j alpha_{t,j} u_{t,e_{t,j}} over kept j.     */
/*  (b) expert-major form ([P4] combine einsum "tec,ecd->td"): ybuf is         */
/*      (E, C, N); the kept assignment (t,j) reads row ybuf[e_{t,j}, slot].    */
/* base_kind as in oracle_layer_rows (1 = residual reads x with row width N). */
/* ------------------------------------------------------------------------ */
void oracle_combine_precomputed(const double* u, int64_t T, int32_t E, int64_t N,
                                const int64_t* selected, const uint8_t* kept,
                                const double* gates, int32_t k, int base_kind,
                                const double* base, double* y) {
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t n = 0; n < N; ++n) y[t * N + n] = base_kind ? base[t * N + n] : 0.0;
        for (int32_t j = 0; j < k; ++j) {
            if (!kept[t * k + j]) continue;
            const double* ut = u + (t * E + selected[t * k + j]) * N;
            for (int64_t n = 0; n < N; ++n) y[t * N + n] += gates[t * k + j] * ut[n];
        }
    }
}

void oracle_combine_slots(const double* ybuf, int64_t T, int32_t E, int64_t C, int64_t N,
                          const int64_t* selected, const int64_t* slot, const uint8_t* kept,
                          const double* gates, int32_t k, int base_kind, const double* base,
                          double* y) {
    (void)E;
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t n = 0; n < N; ++n) y[t * N + n] = base_kind ? base[t * N + n] : 0.0;
        for (int32_t j = 0; j < k; ++j) {
            if (!kept[t * k + j]) continue;
            const double* row = ybuf + (selected[t * k + j] * C + slot[t * k + j]) * N;
            for (int64_t n = 0; n < N; ++n) y[t * N + n] += gates[t * k + j] * row[n];
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Router variants of [P3] route_logits.                                       */
/*   scoring 0: softmax clean scores; 1: logistic sigmoid clean scores         */
/*   ([P3] stable_softmax / stable_sigmoid, element-wise for the sigmoid).     */
/*   Selection key: the raw logits when no selection bias is given, else the   */
/*   clean score plus the per-expert selection bias ([P3]: the bias moves the  */
/*   selection only).  Ties go to the lower expert index.                      */
/*   Gates: softmax of the selected logits (softmax scoring), or the selected  */
/*   sigmoids normalised to sum one, computed as a softmax of log-sigmoids so  */
/*   that it stays finite when every sigmoid underflows ([P3] sigmoid branch). */
/*   clean (T,E) receives the clean scores.                                    */
/* ------------------------------------------------------------------------ */
static double log_sigmoid(double z) {
    /* log(sigmoid(z)) = -log(1 + exp(-z)), split by sign to avoid overflow */
    if (z >= 0.0) return -log1p(exp(-z));
    return z - log1p(exp(z));
}

void oracle_route_variant(const double* s, int64_t T, int32_t E, int32_t k, int scoring,
                          const double* selection_bias, double* clean, int64_t* selected,
                          double* gates, int64_t* counts) {
    OMP_FOR
    for (int64_t t = 0; t < T; ++t) {
        const double* st = s + t * E;
        double* ct = clean + t * E;
        if (scoring == 0) {
            double mx = st[0];
            for (int32_t e = 1; e < E; ++e) if (st[e] > mx) mx = st[e];
            double den = 0.0;
            for (int32_t e = 0; e < E; ++e) den += exp(st[e] - mx);
            for (int32_t e = 0; e < E; ++e) ct[e] = exp(st[e] - mx) / den;
        } else {
            for (int32_t e = 0; e < E; ++e) ct[e] = sigmoid_stable(st[e]);
        }
        double* key = (double*)malloc((size_t)E * sizeof(double));
        for (int32_t e = 0; e < E; ++e) key[e] = selection_bias ? ct[e] + selection_bias[e] : st[e];
        char* taken = (char*)calloc((size_t)E, 1);
        for (int32_t j = 0; j < k; ++j) {
            int32_t best = -1;
            for (int32_t e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || key[e] > key[best]) best = e;
            }
            taken[best] = 1;
            selected[t * k + j] = best;
        }
        free(taken);
        free(key);
        /* gates: softmax over the selected logits, or over their log-sigmoids */
        double* w = (double*)malloc((size_t)k * sizeof(double));
        for (int32_t j = 0; j < k; ++j) {
            double z = st[selected[t * k + j]];
            w[j] = scoring == 0 ? z : log_sigmoid(z);
        }
        double wmax = w[0];
        for (int32_t j = 1; j < k; ++j) if (w[j] > wmax) wmax = w[j];
        double den = 0.0;
        for (int32_t j = 0; j < k; ++j) den += exp(w[j] - wmax);
        for (int32_t j = 0; j < k; ++j) gates[t * k + j] = exp(w[j] - wmax) / den;
        free(w);
    }
    for (int32_t e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t i = 0; i < T * k; ++i) counts[selected[i]] += 1;
}

/* Survivor renormalisation ([P3] dispatch_with_capacity with                  */
/* renormalize_kept_gates): dropped assignments get weight 0 and the kept      */
/* weights of a token are divided by their sum; a token with nothing kept      */
/* keeps all-zero weights.                                                     */
void oracle_renormalize_kept(const double* gates, const uint8_t* kept, int64_t T, int32_t k,
                             double* out) {
    for (int64_t t = 0; t < T; ++t) {
        double mass = 0.0;
        for (int32_t j = 0; j < k; ++j) mass += kept[t * k + j] ? gates[t * k + j] : 0.0;
        for (int32_t j = 0; j < k; ++j) {
            double g = kept[t * k + j] ? gates[t * k + j] : 0.0;
            out[t * k + j] = mass > 0.0 ? g / mass : 0.0;
        }
    }
}
