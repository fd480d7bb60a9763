/*
 * moe_oracle.c -- the CPU oracle of the MoE layer. TEST INFRASTRUCTURE ONLY.
 *
 * This file is a plain, slow, explicitly looped restatement of what the MoE
 * layer computes. Only the test suite, the package's smoke check and the
 * benchmark's CPU-baseline leg load it. The product path never calls it, and
 * it shares no code, header, table or helper with the CUDA library.
 *
 * Sources, cited by page title and section:
 *  [TE]  Transformer Engine docs, "Mixture of Experts": sections Router, Token
 *        dispatch, Token combine, Token probabilities, Grouped GEMM (the
 *        equation Y_i = X_i W_i^T), Grouped MLP, and "Example: MoE layer on a
 *        single device".
 *  [MIX] Transformer Engine example te_mixtral.py: TEMixtralSparseMoeBlock.forward
 *        (softmax in fp32, top-k, renormalise) and _expert_ffn (loop mode:
 *        gate, up = linear(x, W_gate_up).chunk(2); silu(gate) * up; down).
 *  [TT]  torchtitan pull request 1269 (tp2ep): GroupedExperts.forward
 *        (h = silu(x w1) * (x w3); out = h w2) and MoE.forward (shared expert
 *        output plus the scatter-added routed output).
 *
 * Precision:
 *  - Router: fp32 throughout. [TE] Router says all internal math runs in FP32.
 *  - Expert MLP, combine and backward: fp64 accumulation. The pages do not fix
 *    it. The bf16 inputs are exact in fp64.
 *  - With round_bf16 != 0, the two tensors that the pages' bf16 pipeline
 *    stores are rounded to bf16: the SwiGLU intermediate h, because FC2 reads
 *    it from memory ([TE] Grouped MLP), and the expert output y, because FC2
 *    is a bf16 grouped linear whose output token combine merges with fp32
 *    weights ([TE] Grouped GEMM and Token combine; [TT] _grouped_mm returns
 *    bf16; [MIX] the loop's F.linear output). round_bf16 = 0 keeps both exact;
 *    the finite-difference checks use that.
 *
 * Pins. Each function is checked in tests/ against something other than
 * itself: brute-force sorts, invariants, closed forms, a special case that
 * reduces to a dense SwiGLU MLP computed by torch, fp64 central finite
 * differences and torch autograd (tests/test_oracle_*.py, one file per part).
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>

/* ---------------------------------------------------------------- bf16 --- */

static double bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Round a double to the nearest bf16, ties to even, directly (no
 * intermediate float rounding). bf16 has 8 significant bits, and its smallest
 * exponent is -126. Subnormals are kept. */
static uint16_t double_to_bf16(double d)
{
    if (isnan(d)) return 0x7FC0;
    double a = fabs(d);
    uint16_t sign = signbit(d) ? 0x8000 : 0;
    if (isinf(d)) return sign | 0x7F80;
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e);                   /* a = m * 2^e, m in [0.5, 1) */
    int qexp = e - 8;               /* quantum of an 8-significant-bit number */
    if (qexp < -133) qexp = -133;   /* subnormal quantum 2^-133 */
    double q = rint(ldexp(a, -qexp)) ; /* exact scaling; rint rounds half to even */
    double r = ldexp(q, qexp);
    if (r >= 0x1p128) return sign | 0x7F80;
    float f = (float)r;             /* exact: r has <= 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, 4);
    return sign | (uint16_t)((u >> 16) & 0x7FFF);
}

uint16_t oracle_round_bf16(double d) { return double_to_bf16(d); }

void oracle_round_bf16_array(const double* v, int64_t n, uint16_t* out)
{
    for (int64_t i = 0; i < n; i++) out[i] = double_to_bf16(v[i]);
}

/* ------------------------------------------------------------- router --- */

/* Selection key order: larger score first; among equal scores the lower
 * expert index first. NaN ranks below every number, -inf included. */
static int key_better(float a, int ia, float b, int ib)
{
    int na = isnan(a), nb = isnan(b);
    if (na || nb) {
        if (na && nb) return ia < ib;
        return nb;                      /* a is a number and b is NaN */
    }
    if (a != b) return a > b;
    return ia < ib;
}

/*
 * oracle_router_topk -- [TE] Router; [MIX] TEMixtralSparseMoeBlock.forward.
 *
 * For each token t, the score of expert e is s_e = logit (softmax score
 * function) or sigmoid(logit) (sigmoid score function), in fp32. The selection
 * key is s_e + expert_bias[e] when a bias is given ([TE] Load balancing: the
 * bias only changes which experts are picked). Otherwise it is the logit
 * itself (a bias is accepted with the sigmoid score only, as on the page).
 * Softmax and sigmoid are strictly increasing, so ranking logits ranks
 * scores without rounding ties. The k best keys are chosen one after the
 * other, in (key descending, index ascending) order.
 *
 * Routing weights of the chosen experts, in fp32:
 *   softmax, renormalize=1 (softmax after top-k):
 *       p_j = exp(l_j - l_max) / sum_i exp(l_i - l_max) over the k chosen,
 *       summed in selection order. This equals softmax over all experts
 *       followed by p / sum(p) ([MIX]).
 *   softmax, renormalize=0 (softmax before top-k, use_pre_softmax):
 *       p_j = exp(l_j - m) / sum over all E experts of exp(l_e - m),
 *       where m is the row maximum.
 *   sigmoid: p_j = 1 / (1 + exp(-l_j)); with renormalize=1, also divided by
 *       their sum.
 * Each weight is then multiplied by `scaling` ([TE] Router: scaling_factor).
 *
 * Outputs: topk_idx[T,k], topk_prob[T,k], routing_map[T,E] (1 at the chosen
 * experts; may be NULL), counts[E] (column sums of the routing map) and
 * offsets[E+1] (offsets[0] = 0, offsets[e+1] = offsets[e] + counts[e]).
 */
int oracle_router_topk(const float* logits, int64_t T, int E, int k, int score_fn,
                       int renormalize, float scaling, const float* expert_bias,
                       int32_t* topk_idx, float* topk_prob, uint8_t* routing_map,
                       int32_t* counts, int32_t* offsets)
{
    if (E < 1 || k < 1 || k > E) return 1;
    if (expert_bias && score_fn != 1) return 1;   /* bias is defined for sigmoid scores */
    float* key = (float*)malloc(sizeof(float) * (size_t)E);
    char* taken = (char*)malloc((size_t)E);
    for (int e = 0; e < E; e++) counts[e] = 0;
    for (int64_t t = 0; t < T; t++) {
        const float* l = logits + t * E;
        for (int e = 0; e < E; e++) {
            float s = l[e];
            if (expert_bias) {
                float sc = (score_fn == 1) ? 1.0f / (1.0f + expf(-l[e])) : l[e];
                s = sc + expert_bias[e];
            }
            key[e] = s;
            taken[e] = 0;
        }
        for (int j = 0; j < k; j++) {
            int best = -1;
            for (int e = 0; e < E; e++) {
                if (taken[e]) continue;
                if (best < 0 || key_better(key[e], e, key[best], best)) best = e;
            }
            taken[best] = 1;
            topk_idx[t * k + j] = best;
        }
        /* routing weights */
        float* p = topk_prob + t * k;
        const int32_t* sel = topk_idx + t * k;
        if (score_fn == 0) {
            if (renormalize) {
                float m = l[sel[0]];
                for (int j = 1; j < k; j++) if (l[sel[j]] > m) m = l[sel[j]];
                float sum = 0.0f;
                for (int j = 0; j < k; j++) { p[j] = expf(l[sel[j]] - m); sum += p[j]; }
                for (int j = 0; j < k; j++) p[j] = p[j] / sum;
            } else {
                float m = l[0];
                for (int e = 1; e < E; e++) if (l[e] > m) m = l[e];
                float sum = 0.0f;
                for (int e = 0; e < E; e++) sum += expf(l[e] - m);
                for (int j = 0; j < k; j++) p[j] = expf(l[sel[j]] - m) / sum;
            }
        } else {
            float sum = 0.0f;
            for (int j = 0; j < k; j++) { p[j] = 1.0f / (1.0f + expf(-l[sel[j]])); sum += p[j]; }
            if (renormalize) for (int j = 0; j < k; j++) p[j] = p[j] / sum;
        }
        for (int j = 0; j < k; j++) p[j] = p[j] * scaling;
        for (int j = 0; j < k; j++) counts[sel[j]] += 1;
        if (routing_map) {
            for (int e = 0; e < E; e++) routing_map[t * E + e] = 0;
            for (int j = 0; j < k; j++) routing_map[t * E + sel[j]] = 1;
        }
    }
    offsets[0] = 0;
    for (int e = 0; e < E; e++) offsets[e + 1] = offsets[e] + counts[e];
    free(key);
    free(taken);
    return 0;
}

/*
 * oracle_router_backward -- [TE] Router: the gradient of the loss with
 * respect to the logits, given dprob = dL/dp for the routing weights p[t,j]
 * of the experts that oracle_router_topk chose (topk_idx). The selection is
 * piecewise constant in the logits, so it contributes no gradient. With
 * g_j = scaling * dprob[t,j] (p = scaling * q), in fp64:
 *   softmax, renormalize=1: q_j = exp(l_j) / sum_{i in sel} exp(l_i);
 *       dl[sel_j] = q_j (g_j - sum_i q_i g_i), 0 for experts not chosen.
 *   softmax, renormalize=0: q_e = exp(l_e) / sum_{all e'} exp(l_e');
 *       dl[e] = q_e (G_e - sum_j q_{sel_j} g_j), G_e = g_j if e = sel_j else 0.
 *   sigmoid, renormalize=0: dl[sel_j] = g_j s_j (1 - s_j), s = sigmoid(l).
 *   sigmoid, renormalize=1: r_j = s_j / S, S = sum_j s_j;
 *       dl[sel_j] = ((g_j - sum_i r_i g_i) / S) s_j (1 - s_j).
 * An expert bias only moves the selection, so it does not appear here.
 * Writes dlogits[T,E]. Returns nonzero on an invalid index.
 */
int oracle_router_backward(const float* logits, int64_t T, int E, int k, int score_fn,
                           int renormalize, float scaling, const int32_t* topk_idx,
                           const float* dprob, float* dlogits)
{
    double* q = (double*)malloc(sizeof(double) * (size_t)(E > k ? E : k));
    double* g = (double*)malloc(sizeof(double) * (size_t)k);
    for (int64_t t = 0; t < T; t++) {
        const float* l = logits + t * E;
        const int32_t* sel = topk_idx + t * k;
        float* dl = dlogits + t * E;
        for (int e = 0; e < E; e++) dl[e] = 0.0f;
        for (int j = 0; j < k; j++) {
            if (sel[j] < 0 || sel[j] >= E) { free(q); free(g); return 1; }
            g[j] = (double)scaling * (double)dprob[t * k + j];
        }
        if (score_fn == 0 && renormalize) {
            double m = l[sel[0]], sum = 0.0, c = 0.0;
            for (int j = 1; j < k; j++) if (l[sel[j]] > m) m = l[sel[j]];
            for (int j = 0; j < k; j++) { q[j] = exp((double)l[sel[j]] - m); sum += q[j]; }
            for (int j = 0; j < k; j++) { q[j] /= sum; c += q[j] * g[j]; }
            for (int j = 0; j < k; j++) dl[sel[j]] = (float)(q[j] * (g[j] - c));
        } else if (score_fn == 0) {
            double m = l[0], sum = 0.0, c = 0.0;
            for (int e = 1; e < E; e++) if (l[e] > m) m = l[e];
            for (int e = 0; e < E; e++) { q[e] = exp((double)l[e] - m); sum += q[e]; }
            for (int e = 0; e < E; e++) q[e] /= sum;
            for (int j = 0; j < k; j++) c += q[sel[j]] * g[j];
            for (int e = 0; e < E; e++) dl[e] = (float)(q[e] * (0.0 - c));
            for (int j = 0; j < k; j++) dl[sel[j]] = (float)(q[sel[j]] * (g[j] - c));
        } else {
            double S = 0.0, c = 0.0;
            for (int j = 0; j < k; j++) { q[j] = 1.0 / (1.0 + exp(-(double)l[sel[j]])); S += q[j]; }
            for (int j = 0; j < k; j++) {
                double ds = g[j];   /* dL/ds_j without renormalisation */
                if (renormalize) {
                    if (j == 0) for (int i = 0; i < k; i++) c += (q[i] / S) * g[i];
                    ds = (g[j] - c) / S;
                }
                dl[sel[j]] = (float)(ds * q[j] * (1.0 - q[j]));
            }
        }
    }
    free(q);
    free(g);
    return 0;
}

/*
 * oracle_expert_bias_update -- torchtitan pull request 1269, llama4 moe.py,
 * MoE._update_expert_bias (auxiliary-loss-free load balancing): with the
 * per-expert token counts c[E] of the last step,
 *   delta_e = coeff * sign(mean(c) - c_e),  delta_e -= mean(delta),
 *   bias_e += delta_e.
 * sign(mean(c) - c_e) is decided exactly, as sign(sum(c) - E * c_e), and the
 * mean of delta in double precision. bias is updated in place (fp32).
 */
void oracle_expert_bias_update(const int32_t* counts, int E, float coeff, float* bias)
{
    int64_t sum = 0;
    for (int e = 0; e < E; e++) sum += counts[e];
    double mean_delta = 0.0;
    double* delta = (double*)malloc(sizeof(double) * (size_t)E);
    for (int e = 0; e < E; e++) {
        const int64_t d = sum - (int64_t)E * counts[e];
        delta[e] = (double)coeff * (double)((d > 0) - (d < 0));
        mean_delta += delta[e];
    }
    mean_delta /= E;
    for (int e = 0; e < E; e++) bias[e] = (float)((double)bias[e] + (delta[e] - mean_delta));
    free(delta);
}

/* ---------------------------------------------------------- aux loss --- */

/*
 * oracle_aux_scores -- [TE] Mixture of Experts, Load balancing: the dense
 * routing scores that the auxiliary loss takes, one per expert rather than
 * only for the chosen k: the softmax over all E experts (score_fn 0) or the
 * sigmoid of each logit (score_fn 1), in fp64. The page's score helper
 * ignores an expert bias, so none is applied. Writes scores[T,E].
 */
void oracle_aux_scores(const float* logits, int64_t T, int E, int score_fn, double* scores)
{
    for (int64_t t = 0; t < T; t++) {
        const float* l = logits + t * E;
        double* s = scores + t * E;
        if (score_fn == 0) {
            double m = l[0], sum = 0.0;
            for (int e = 1; e < E; e++) if (l[e] > m) m = l[e];
            for (int e = 0; e < E; e++) { s[e] = exp((double)l[e] - m); sum += s[e]; }
            for (int e = 0; e < E; e++) s[e] /= sum;
        } else {
            for (int e = 0; e < E; e++) s[e] = 1.0 / (1.0 + exp(-(double)l[e]));
        }
    }
}

/*
 * oracle_aux_loss -- [TE] Mixture of Experts, Load balancing
 * (fused_moe_aux_loss). The page names the inputs -- the dense scores, the
 * per-expert token counts c[E] taken from the router's routing map, the
 * number of tokens T and of experts E, the top-k and a coefficient -- but
 * prints no formula. Reading: the switch-style load-balancing loss
 *   loss = coeff * E / (k * T^2) * sum_e (sum_t s[t,e]) * c_e
 *        = coeff * E * sum_e f_e * P_e,
 *   f_e = c_e / (k T) (share of assignments), P_e = (1/T) sum_t s[t,e].
 * With every expert at T k / E assignments and a mean score of 1/E it is
 * exactly coeff, and it grows as the counts gather where the scores are
 * high. Sums run in fp64, t then e in order.
 */
double oracle_aux_loss(const double* scores, const int32_t* counts, int64_t T, int E, int k, double coeff)
{
    double total = 0.0;
    for (int e = 0; e < E; e++) {
        double P = 0.0;
        for (int64_t t = 0; t < T; t++) P += scores[t * E + e];
        total += P * (double)counts[e];
    }
    return coeff * (double)E / ((double)k * (double)T * (double)T) * total;
}

/*
 * oracle_aux_loss_backward -- the gradient of grad_loss * loss with respect
 * to the logits, the counts held fixed (they come from the discrete
 * selection). dloss/ds[t,e] is the same for every token,
 *   G_e = grad_loss * coeff * E * c_e / (k T^2),
 * and the chain rule through the score function gives
 *   softmax: dl[t,i] = s[t,i] * (G_i - sum_e s[t,e] G_e);
 *   sigmoid: dl[t,i] = G_i * s[t,i] * (1 - s[t,i]).
 * Writes dlogits[T,E] in fp64.
 */
void oracle_aux_loss_backward(const float* logits, const int32_t* counts, int64_t T, int E, int k,
                              int score_fn, double coeff, double grad_loss, double* dlogits)
{
    double* s = (double*)malloc(sizeof(double) * (size_t)E);
    double* G = (double*)malloc(sizeof(double) * (size_t)E);
    for (int e = 0; e < E; e++)
        G[e] = grad_loss * coeff * (double)E * (double)counts[e] / ((double)k * (double)T * (double)T);
    for (int64_t t = 0; t < T; t++) {
        oracle_aux_scores(logits + t * E, 1, E, score_fn, s);
        double* dl = dlogits + t * E;
        if (score_fn == 0) {
            double c = 0.0;
            for (int e = 0; e < E; e++) c += s[e] * G[e];
            for (int e = 0; e < E; e++) dl[e] = s[e] * (G[e] - c);
        } else {
            for (int e = 0; e < E; e++) dl[e] = G[e] * s[e] * (1.0 - s[e]);
        }
    }
    free(s);
    free(G);
}

/* ----------------------------------------------------------- dispatch --- */

/*
 * oracle_dispatch -- [TE] Token dispatch: rows routed to the same expert are
 * stored contiguously, expert blocks in expert order, starting at offsets[e]
 * (the cumulative per-expert counts). Inside a block, rows are in ascending
 * token order: this layer's reading of the opaque row_id_map. The assignment
 * (t, j) with e = topk_idx[t,j] lands in row
 *     offsets[e] + #{ t' < t : e is among the experts of t' }.
 * Outputs sorted_token[A] (the token of each permuted row) and row_of[T,k]
 * (the permuted row of each assignment, the inverse map used by combine).
 * Returns nonzero if an expert index is out of range or a block overflows.
 */
int oracle_dispatch(const int32_t* topk_idx, int64_t T, int k, int E,
                    const int32_t* offsets, int32_t* sorted_token, int32_t* row_of)
{
    int64_t* fill = (int64_t*)calloc((size_t)E, sizeof(int64_t));
    int rc = 0;
    for (int64_t t = 0; t < T && !rc; t++) {        /* token order */
        for (int j = 0; j < k; j++) {
            int e = topk_idx[t * k + j];
            if (e < 0 || e >= E) { rc = 2; break; }
            int64_t row = offsets[e] + fill[e];
            if (row >= offsets[e + 1]) { rc = 3; break; }
            fill[e] += 1;
            sorted_token[row] = (int32_t)t;
            row_of[t * k + j] = (int32_t)row;
        }
    }
    free(fill);
    return rc;
}

/*
 * oracle_dispatch_padded -- [TE] Mixture of Experts, Token permutation,
 * Padding and alignment: each expert's block is rounded up to a multiple of
 * align rows (an empty block stays empty), the blocks follow one another in
 * expert order, and the rows past an expert's tokens are padding.
 *   padded_offsets[0] = 0,
 *   padded_offsets[e+1] = padded_offsets[e] + align * ceil(counts[e] / align),
 * with counts[e] = offsets[e+1] - offsets[e]. Inside a block the tokens keep
 * the unpadded order, so the assignment (t, j) lands in row
 *   padded_offsets[e] + #{ t' < t : e is among the experts of t' },
 * which is oracle_dispatch on the padded offsets. Writes padded_offsets[E+1],
 * row_of[T,k] and sorted_token[padded_offsets[E]] (the token of each row; the
 * caller fills the pad rows' entries with -1 beforehand). Returns nonzero on
 * an invalid routing or align < 1.
 */
int oracle_dispatch_padded(const int32_t* topk_idx, int64_t T, int k, int E, const int32_t* offsets,
                           int align, int32_t* padded_offsets, int32_t* sorted_token, int32_t* row_of)
{
    if (align < 1) return 4;
    padded_offsets[0] = 0;
    for (int e = 0; e < E; e++) {
        const int64_t c = (int64_t)offsets[e + 1] - offsets[e];
        if (c < 0) return 5;
        padded_offsets[e + 1] = padded_offsets[e] + (int32_t)(((c + align - 1) / align) * align);
    }
    return oracle_dispatch(topk_idx, T, k, E, padded_offsets, sorted_token, row_of);
}

/* x_perm[row] = x[sorted_token[row]]: a plain copy of bf16 rows; a row whose
 * sorted_token is negative (a pad row of the padded dispatch) is zeros. */
void oracle_gather_rows(const uint16_t* x, int H, const int32_t* sorted_token,
                        int64_t A, uint16_t* x_perm)
{
    for (int64_t r = 0; r < A; r++) {
        if (sorted_token[r] < 0)
            memset(x_perm + r * H, 0, sizeof(uint16_t) * (size_t)H);
        else
            memcpy(x_perm + r * H, x + (int64_t)sorted_token[r] * H, sizeof(uint16_t) * (size_t)H);
    }
}

/* ---------------------------------------------------------- expert MLP -- */

static double silu(double g) { return g / (1.0 + exp(-g)); }

/*
 * oracle_expert_mlp -- one SwiGLU expert on n token rows.
 * [TE] Grouped MLP: FC1, GLU activation, FC2. [MIX] _expert_ffn: gate and up
 * are the first and second halves of the FC1 output. [TT] GroupedExperts:
 * silu(x w1) * (x w3), times w2.
 *   g = x . Wgu[:, 0:I]    u = x . Wgu[:, I:2I]    (Wgu is [H, 2I], row-major)
 *   h = silu(g) * u        (rounded to bf16 when round_bf16)
 *   y = h . Wd             (Wd is [I, H], row-major; rounded to bf16 when round_bf16)
 * Accumulation is fp64, in ascending index order. g, u, h are optional
 * outputs.
 */
void oracle_expert_mlp(const uint16_t* x, int64_t n, int H, int I,
                       const uint16_t* w_gate_up, const uint16_t* w_down, int round_bf16,
                       double* y, double* g_out, double* u_out, double* h_out)
{
    double* g = (double*)malloc(sizeof(double) * (size_t)I);
    double* u = (double*)malloc(sizeof(double) * (size_t)I);
    double* h = (double*)malloc(sizeof(double) * (size_t)I);
    for (int64_t r = 0; r < n; r++) {
        const uint16_t* xr = x + r * H;
        for (int i = 0; i < I; i++) { g[i] = 0.0; u[i] = 0.0; }
        for (int hh = 0; hh < H; hh++) {
            double xv = bf16_to_double(xr[hh]);
            const uint16_t* wrow = w_gate_up + (int64_t)hh * 2 * I;
            for (int i = 0; i < I; i++) {
                g[i] += xv * bf16_to_double(wrow[i]);
                u[i] += xv * bf16_to_double(wrow[I + i]);
            }
        }
        for (int i = 0; i < I; i++) {
            double v = silu(g[i]) * u[i];
            h[i] = round_bf16 ? bf16_to_double(double_to_bf16(v)) : v;
        }
        double* yr = y + r * H;
        for (int c = 0; c < H; c++) yr[c] = 0.0;
        for (int i = 0; i < I; i++) {
            const uint16_t* wrow = w_down + (int64_t)i * H;
            for (int c = 0; c < H; c++) yr[c] += h[i] * bf16_to_double(wrow[c]);
        }
        if (round_bf16)
            for (int c = 0; c < H; c++) yr[c] = bf16_to_double(double_to_bf16(yr[c]));
        if (g_out) memcpy(g_out + r * I, g, sizeof(double) * (size_t)I);
        if (u_out) memcpy(u_out + r * I, u, sizeof(double) * (size_t)I);
        if (h_out) memcpy(h_out + r * I, h, sizeof(double) * (size_t)I);
    }
    free(g); free(u); free(h);
}

/*
 * oracle_grouped_mlp -- [TE] Grouped GEMM: Y_i = X_i W_i^T for each expert
 * block i, and Y = concat(Y_0 ... Y_{G-1}). Like the page's baseline, it runs a
 * loop with one call per expert over the expert-contiguous rows
 * [offsets[e], offsets[e+1]), each with the SwiGLU expert above. An empty
 * block is skipped.
 */
void oracle_grouped_mlp(const uint16_t* x_perm, const int32_t* offsets, int E, int H, int I,
                        const uint16_t* w_gate_up, const uint16_t* w_down, int round_bf16,
                        double* y_perm)
{
    for (int e = 0; e < E; e++) {
        int64_t r0 = offsets[e], n = (int64_t)offsets[e + 1] - offsets[e];
        if (n <= 0) continue;
        oracle_expert_mlp(x_perm + r0 * H, n, H, I,
                          w_gate_up + (int64_t)e * H * 2 * I, w_down + (int64_t)e * I * H,
                          round_bf16, y_perm + r0 * H, NULL, NULL, NULL);
    }
}

/*
 * oracle_combine -- [TE] Token combine with merging_probs:
 *   out[t] = shared[t] + sum_j p[t,j] * y[row_of[t,j]]
 * j ascending, in fp64. With probs == NULL the contributions are summed
 * unweighted, as the page says for a combine without merging_probs. `shared`
 * may be NULL ([TT] MoE.forward: the shared expert output is the base that
 * the routed outputs are added to).
 */
void oracle_combine(const double* y_perm, const int32_t* row_of, const float* probs,
                    int64_t T, int k, int H, const double* shared, double* out)
{
    for (int64_t t = 0; t < T; t++) {
        double* o = out + t * H;
        for (int c = 0; c < H; c++) o[c] = shared ? shared[t * H + c] : 0.0;
        for (int j = 0; j < k; j++) {
            double p = probs ? (double)probs[t * k + j] : 1.0;
            const double* yr = y_perm + (int64_t)row_of[t * k + j] * H;
            for (int c = 0; c < H; c++) o[c] += p * yr[c];
        }
    }
}

/*
 * oracle_moe_forward_tokens -- the layer by its plain definition, one token at
 * a time, with no permutation:
 *   out[t] = shared_mlp(x_t) + sum_j p_j * MLP_{e_j}(x_t)
 * where (e_j, p_j) come from oracle_router_topk on that token's logits row.
 * This is the four stages of [TE] Introduction: route, dispatch, experts,
 * combine. Dispatch and combine are a pure reordering, so they drop out.
 * The per-expert loop is the page's "same outputs" baseline (Grouped GEMM).
 * Only the tokens in token_list are computed, and their rows are written to
 * out in list order.
 */
int oracle_moe_forward_tokens(const uint16_t* x, const float* logits, int H, int I, int E, int k,
                              int score_fn, int renormalize, float scaling, const float* expert_bias,
                              const uint16_t* w_gate_up, const uint16_t* w_down,
                              const uint16_t* shared_gate_up, const uint16_t* shared_down,
                              int round_bf16, const int64_t* token_list, int64_t n_tokens, double* out)
{
    int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * (size_t)k);
    float* p = (float*)malloc(sizeof(float) * (size_t)k);
    int32_t* cnt = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
    int32_t* off = (int32_t*)malloc(sizeof(int32_t) * (size_t)(E + 1));
    double* y = (double*)malloc(sizeof(double) * (size_t)H);
    int rc = 0;
    for (int64_t n = 0; n < n_tokens && !rc; n++) {
        int64_t t = token_list[n];
        rc = oracle_router_topk(logits + t * E, 1, E, k, score_fn, renormalize, scaling,
                                expert_bias, idx, p, NULL, cnt, off);
        double* o = out + n * H;
        if (shared_gate_up) {
            oracle_expert_mlp(x + t * H, 1, H, I, shared_gate_up, shared_down, round_bf16, o,
                              NULL, NULL, NULL);
        } else {
            for (int c = 0; c < H; c++) o[c] = 0.0;
        }
        for (int j = 0; j < k; j++) {
            int e = idx[j];
            oracle_expert_mlp(x + t * H, 1, H, I, w_gate_up + (int64_t)e * H * 2 * I,
                              w_down + (int64_t)e * I * H, round_bf16, y, NULL, NULL, NULL);
            for (int c = 0; c < H; c++) o[c] += (double)p[j] * y[c];
        }
    }
    free(idx); free(p); free(cnt); free(off); free(y);
    return rc;
}

/* ------------------------------------------------------------ backward --- */

/*
 * oracle_moe_backward -- the gradients of out = sum_j p_j MLP_{e_j}(x) with
 * respect to x, W_gate_up, W_down and the routing weights p, for a given
 * routing (topk_idx, topk_prob) and upstream gradient dout. It is the chain
 * rule applied to the forward above. [TE] Example: every stage is
 * differentiable. The routing weights are an input here, so nothing flows into
 * the logits.
 * Per assignment (t, j) with e = topk_idx[t,j] and p = topk_prob[t,j]:
 *   y = MLP_e(x_t);           dprob[t,j] = <dout_t, y>
 *   dy = p * dout_t;          dWd[e]   += h^T dy
 *   dh = dy . Wd[e]^T;        du = dh * silu(g);  dg = dh * u * silu'(g)
 *   silu'(g) = s + g s (1 - s),  s = 1 / (1 + e^-g)
 *   dWgu[e][:, 0:I] += x_t^T dg;   dWgu[e][:, I:2I] += x_t^T du
 *   dxp = dg . Wgu[e][:, 0:I]^T + du . Wgu[e][:, I:2I]^T;   dx_t += dxp
 * All in fp64. With round_bf16, every tensor that a bf16 pipeline stores
 * between its stages is rounded to bf16, as in the forward: the saved FC1
 * outputs g and u that the SwiGLU backward reads; the gradient dy of the
 * bf16 expert output, which is the fp32 product p * dout rounded to bf16
 * ([TT] MoE.forward, patch "multiply scores in FP32 datatype": the bf16 expert
 * output is cast to fp32, multiplied by the fp32 scores and cast back to
 * bf16, so the chain rule through that product gives the bf16 rounding of the
 * fp32 product of the score and the bf16 upstream gradient); the gradients
 * dg, du of the bf16 FC1 output; and the gradient dxp of each bf16 permuted
 * token row, which the unpermute then sums.
 * The rounding functions themselves pass gradients through unchanged.
 * With round_bf16 = 0, nothing is rounded, and the result is the exact
 * derivative that the finite-difference pin checks.
 * only_expert >= 0 restricts the sums to that expert's
 * assignments. token_list (NULL = all T tokens) restricts t, and dx / dprob
 * rows are then written in list order. With only_expert >= 0 the dw_* outputs
 * hold that one expert ([H,2I] and [I,H]), else all E. Output pointers may be
 * NULL. Every non-NULL output is zeroed first, so an expert that gets no
 * assignment has a zero weight gradient.
 */
int oracle_moe_backward_state(const uint16_t* x, int64_t T, int H, int I, int E, int k,
                              const int32_t* topk_idx, const float* topk_prob,
                              const uint16_t* w_gate_up, const uint16_t* w_down, const uint16_t* dout,
                              int round_bf16, int only_expert, const int64_t* token_list,
                              int64_t n_tokens, const int32_t* row_of, const uint16_t* st_gu,
                              const uint16_t* st_h, const uint16_t* st_y,
                              double* dx, double* dw_gate_up, double* dw_down, double* dprob);

int oracle_moe_backward(const uint16_t* x, int64_t T, int H, int I, int E, int k,
                        const int32_t* topk_idx, const float* topk_prob,
                        const uint16_t* w_gate_up, const uint16_t* w_down, const uint16_t* dout,
                        int round_bf16, int only_expert, const int64_t* token_list, int64_t n_tokens,
                        double* dx, double* dw_gate_up, double* dw_down, double* dprob)
{
    return oracle_moe_backward_state(x, T, H, I, E, k, topk_idx, topk_prob, w_gate_up, w_down, dout,
                                     round_bf16, only_expert, token_list, n_tokens, NULL, NULL, NULL,
                                     NULL, dx, dw_gate_up, dw_down, dprob);
}

/*
 * oracle_moe_backward_state -- oracle_moe_backward on a given saved forward
 * state. [TE] Grouped MLP: the pipeline stores the FC1 output and the
 * activation between its stages, and the backward of each stage reads what
 * the forward stored; the combine's backward reads the stored expert outputs.
 * With row_of != NULL, the forward values of assignment (t, j) are read from
 * row r = row_of[t * k + j] of the stored bf16 tensors instead of being
 * recomputed: g = st_gu[r][0:I], u = st_gu[r][I:2I], h = st_h[r], y = st_y[r]
 * (st_gu [rows][2I], st_h [rows][I], st_y [rows][H]). Everything after that is
 * the chain rule of oracle_moe_backward, unchanged. Given the oracle's own
 * rounded forward values, it returns what oracle_moe_backward returns.
 */
int oracle_moe_backward_state(const uint16_t* x, int64_t T, int H, int I, int E, int k,
                              const int32_t* topk_idx, const float* topk_prob,
                              const uint16_t* w_gate_up, const uint16_t* w_down, const uint16_t* dout,
                              int round_bf16, int only_expert, const int64_t* token_list,
                              int64_t n_tokens, const int32_t* row_of, const uint16_t* st_gu,
                              const uint16_t* st_h, const uint16_t* st_y,
                              double* dx, double* dw_gate_up, double* dw_down, double* dprob)
{
    if (row_of && (!st_gu || !st_h || !st_y)) return 3;
    int64_t nt = token_list ? n_tokens : T;
    if (dx) memset(dx, 0, sizeof(double) * (size_t)(nt * H));
    if (dprob) memset(dprob, 0, sizeof(double) * (size_t)(nt * k));
    int64_t n_dw = only_expert >= 0 ? 1 : E;     /* experts held by dw_* */
    if (dw_gate_up) memset(dw_gate_up, 0, sizeof(double) * (size_t)(n_dw * H * 2 * I));
    if (dw_down) memset(dw_down, 0, sizeof(double) * (size_t)(n_dw * I * H));
    double* g = (double*)malloc(sizeof(double) * (size_t)I);
    double* u = (double*)malloc(sizeof(double) * (size_t)I);
    double* h = (double*)malloc(sizeof(double) * (size_t)I);
    double* y = (double*)malloc(sizeof(double) * (size_t)H);
    double* dy = (double*)malloc(sizeof(double) * (size_t)H);
    double* dh = (double*)malloc(sizeof(double) * (size_t)I);
    double* dg = (double*)malloc(sizeof(double) * (size_t)I);
    double* du = (double*)malloc(sizeof(double) * (size_t)I);
    for (int64_t n = 0; n < nt; n++) {
        int64_t t = token_list ? token_list[n] : n;
        const uint16_t* xt = x + t * H;
        const uint16_t* dot = dout + t * H;
        for (int j = 0; j < k; j++) {
            int e = topk_idx[t * k + j];
            if (e < 0 || e >= E) return 2;
            if (only_expert >= 0 && e != only_expert) continue;
            double p = (double)topk_prob[t * k + j];
            const uint16_t* wgu = w_gate_up + (int64_t)e * H * 2 * I;
            const uint16_t* wd = w_down + (int64_t)e * I * H;
            if (row_of) {
                int64_t r = row_of[t * k + j];
                if (r < 0) return 2;
                for (int i = 0; i < I; i++) {
                    g[i] = bf16_to_double(st_gu[r * 2 * I + i]);
                    u[i] = bf16_to_double(st_gu[r * 2 * I + I + i]);
                    h[i] = bf16_to_double(st_h[r * I + i]);
                }
                for (int c = 0; c < H; c++) y[c] = bf16_to_double(st_y[r * H + c]);
            } else {
                oracle_expert_mlp(xt, 1, H, I, wgu, wd, round_bf16, y, g, u, h);
            }
            if (dprob) {
                double s = 0.0;
                for (int c = 0; c < H; c++) s += bf16_to_double(dot[c]) * y[c];
                dprob[n * k + j] = s;
            }
            if (round_bf16)
                for (int i = 0; i < I; i++) {
                    g[i] = bf16_to_double(double_to_bf16(g[i]));
                    u[i] = bf16_to_double(double_to_bf16(u[i]));
                }
            for (int c = 0; c < H; c++) {
                if (round_bf16) {
                    /* the stored dy is the bf16 rounding of the fp32 product
                     * p * dout ([TT] MoE.forward multiplies the expert output by
                     * the scores in fp32 before the bf16 cast; its backward
                     * takes the same product in fp32) */
                    const float pf = topk_prob[t * k + j];
                    const float v = pf * (float)bf16_to_double(dot[c]);
                    dy[c] = bf16_to_double(double_to_bf16((double)v));
                } else {
                    dy[c] = p * bf16_to_double(dot[c]);
                }
            }
            if (dw_down) {
                double* dwd = dw_down + (only_expert >= 0 ? 0 : (int64_t)e * I * H);
                for (int i = 0; i < I; i++)
                    for (int c = 0; c < H; c++) dwd[(int64_t)i * H + c] += h[i] * dy[c];
            }
            for (int i = 0; i < I; i++) {
                double s = 0.0;
                for (int c = 0; c < H; c++) s += bf16_to_double(wd[(int64_t)i * H + c]) * dy[c];
                dh[i] = s;
            }
            for (int i = 0; i < I; i++) {
                double sg = 1.0 / (1.0 + exp(-g[i]));
                double a = g[i] * sg;                      /* silu(g) */
                du[i] = dh[i] * a;
                dg[i] = dh[i] * u[i] * (sg + g[i] * sg * (1.0 - sg));
                if (round_bf16) {
                    du[i] = bf16_to_double(double_to_bf16(du[i]));
                    dg[i] = bf16_to_double(double_to_bf16(dg[i]));
                }
            }
            if (dw_gate_up) {
                double* dw = dw_gate_up + (only_expert >= 0 ? 0 : (int64_t)e * H * 2 * I);
                for (int hh = 0; hh < H; hh++) {
                    double xv = bf16_to_double(xt[hh]);
                    double* row = dw + (int64_t)hh * 2 * I;
                    for (int i = 0; i < I; i++) { row[i] += xv * dg[i]; row[I + i] += xv * du[i]; }
                }
            }
            if (dx) {
                double* dxr = dx + n * H;
                for (int hh = 0; hh < H; hh++) {
                    const uint16_t* row = wgu + (int64_t)hh * 2 * I;
                    double s = 0.0;
                    for (int i = 0; i < I; i++)
                        s += dg[i] * bf16_to_double(row[i]) + du[i] * bf16_to_double(row[I + i]);
                    if (round_bf16) s = bf16_to_double(double_to_bf16(s));
                    dxr[hh] += s;
                }
            }
        }
    }
    free(g); free(u); free(h); free(y); free(dy); free(dh); free(dg); free(du);
    return 0;
}

/*
 * oracle_moe_backward_scaled -- the gradients of the ScaledSwiGLU layer
 * ([TE] Grouped MLP, scale_bias: the routing weight p multiplies the SwiGLU
 * output before FC2, and the combine adds the expert outputs unweighted):
 *   out_t = sum_j MLP'_{e_j}(x_t; p_j),  MLP'(x; p) = (p * silu(g) * u) . Wd.
 * Per assignment (t, j), with s = silu(g) * u:
 *   dy = dout_t;                dWd[e] += h^T dy   (h = p * s, as stored)
 *   dh = dy . Wd[e]^T;          dprob[t,j] = <dh, s>
 *   ds = p * dh;                dg = ds * u * silu'(g);  du = ds * silu(g)
 *   dWgu[e][:, 0:I] += x_t^T dg;  dWgu[e][:, I:2I] += x_t^T du
 *   dxp = dg . Wgu[e][:, 0:I]^T + du . Wgu[e][:, I:2I]^T;   dx_t += dxp
 * All in fp64. With round_bf16, the stored tensors are bf16 as in
 * oracle_moe_backward: h = bf16(p * s) from the forward's exact g and u; the
 * backward reads g and u rounded to bf16 (so s in dprob and ds is formed from
 * them); dg, du and each permuted row's dxp are rounded; dy = dout is bf16
 * already. Unrounded, the layer equals the one with the weight applied in the
 * combine (p (s . Wd) = (p s) . Wd), and so do all four gradients. A saved
 * state (row_of != NULL) gives g, u and the stored h of each assignment's row,
 * as in oracle_moe_backward_state. Other arguments as there.
 */
int oracle_moe_backward_scaled(const uint16_t* x, int64_t T, int H, int I, int E, int k,
                               const int32_t* topk_idx, const float* topk_prob,
                               const uint16_t* w_gate_up, const uint16_t* w_down, const uint16_t* dout,
                               int round_bf16, int only_expert, const int64_t* token_list,
                               int64_t n_tokens, const int32_t* row_of, const uint16_t* st_gu,
                               const uint16_t* st_h,
                               double* dx, double* dw_gate_up, double* dw_down, double* dprob)
{
    if (row_of && (!st_gu || !st_h)) return 3;
    int64_t nt = token_list ? n_tokens : T;
    if (dx) memset(dx, 0, sizeof(double) * (size_t)(nt * H));
    if (dprob) memset(dprob, 0, sizeof(double) * (size_t)(nt * k));
    int64_t n_dw = only_expert >= 0 ? 1 : E;
    if (dw_gate_up) memset(dw_gate_up, 0, sizeof(double) * (size_t)(n_dw * H * 2 * I));
    if (dw_down) memset(dw_down, 0, sizeof(double) * (size_t)(n_dw * I * H));
    double* g = (double*)malloc(sizeof(double) * (size_t)I);
    double* u = (double*)malloc(sizeof(double) * (size_t)I);
    double* h = (double*)malloc(sizeof(double) * (size_t)I);
    double* y = (double*)malloc(sizeof(double) * (size_t)H);
    double* dy = (double*)malloc(sizeof(double) * (size_t)H);
    double* dh = (double*)malloc(sizeof(double) * (size_t)I);
    double* dg = (double*)malloc(sizeof(double) * (size_t)I);
    double* du = (double*)malloc(sizeof(double) * (size_t)I);
    int rc = 0;
    for (int64_t n = 0; n < nt && rc == 0; n++) {
        int64_t t = token_list ? token_list[n] : n;
        const uint16_t* xt = x + t * H;
        const uint16_t* dot = dout + t * H;
        for (int j = 0; j < k; j++) {
            int e = topk_idx[t * k + j];
            if (e < 0 || e >= E) { rc = 2; break; }
            if (only_expert >= 0 && e != only_expert) continue;
            double p = (double)topk_prob[t * k + j];
            const uint16_t* wgu = w_gate_up + (int64_t)e * H * 2 * I;
            const uint16_t* wd = w_down + (int64_t)e * I * H;
            if (row_of) {
                int64_t r = row_of[t * k + j];
                if (r < 0) { rc = 2; break; }
                for (int i = 0; i < I; i++) {
                    g[i] = bf16_to_double(st_gu[r * 2 * I + i]);
                    u[i] = bf16_to_double(st_gu[r * 2 * I + I + i]);
                    h[i] = bf16_to_double(st_h[r * I + i]);
                }
            } else {
                /* the forward's exact g and u; the stored h is p * silu(g) * u */
                oracle_expert_mlp(xt, 1, H, I, wgu, wd, 0, y, g, u, NULL);
                for (int i = 0; i < I; i++) {
                    double v = p * silu(g[i]) * u[i];
                    h[i] = round_bf16 ? bf16_to_double(double_to_bf16(v)) : v;
                }
                if (round_bf16)
                    for (int i = 0; i < I; i++) {
                        g[i] = bf16_to_double(double_to_bf16(g[i]));
                        u[i] = bf16_to_double(double_to_bf16(u[i]));
                    }
            }
            for (int c = 0; c < H; c++) dy[c] = bf16_to_double(dot[c]);
            if (dw_down) {
                double* dwd = dw_down + (only_expert >= 0 ? 0 : (int64_t)e * I * H);
                for (int i = 0; i < I; i++)
                    for (int c = 0; c < H; c++) dwd[(int64_t)i * H + c] += h[i] * dy[c];
            }
            for (int i = 0; i < I; i++) {
                double sum = 0.0;
                for (int c = 0; c < H; c++) sum += bf16_to_double(wd[(int64_t)i * H + c]) * dy[c];
                dh[i] = sum;
            }
            double dp = 0.0;
            for (int i = 0; i < I; i++) {
                double sg = 1.0 / (1.0 + exp(-g[i]));
                double a = g[i] * sg;                      /* silu(g) */
                dp += dh[i] * a * u[i];
                double ds = p * dh[i];
                du[i] = ds * a;
                dg[i] = ds * u[i] * (sg + g[i] * sg * (1.0 - sg));
                if (round_bf16) {
                    du[i] = bf16_to_double(double_to_bf16(du[i]));
                    dg[i] = bf16_to_double(double_to_bf16(dg[i]));
                }
            }
            if (dprob) dprob[n * k + j] = dp;
            if (dw_gate_up) {
                double* dw = dw_gate_up + (only_expert >= 0 ? 0 : (int64_t)e * H * 2 * I);
                for (int hh = 0; hh < H; hh++) {
                    double xv = bf16_to_double(xt[hh]);
                    double* row = dw + (int64_t)hh * 2 * I;
                    for (int i = 0; i < I; i++) { row[i] += xv * dg[i]; row[I + i] += xv * du[i]; }
                }
            }
            if (dx) {
                double* dxr = dx + n * H;
                for (int hh = 0; hh < H; hh++) {
                    const uint16_t* row = wgu + (int64_t)hh * 2 * I;
                    double sum = 0.0;
                    for (int i = 0; i < I; i++)
                        sum += dg[i] * bf16_to_double(row[i]) + du[i] * bf16_to_double(row[I + i]);
                    if (round_bf16) sum = bf16_to_double(double_to_bf16(sum));
                    dxr[hh] += sum;
                }
            }
        }
    }
    free(g); free(u); free(h); free(y); free(dy); free(dh); free(dg); free(du);
    return rc;
}

