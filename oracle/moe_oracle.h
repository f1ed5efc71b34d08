/*
 * CPU oracle for the MoE routing-and-dispatch layer.
 *
 * TEST INFRASTRUCTURE ONLY. Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load or call this library.
 * It shares no code, header, table or helper with the CUDA library and never
 * includes anything from it.
 *
 * Plain, slow, single-threaded definitions written from these pages:
 *   [TC-vs-EC]  "Token choice vs expert choice routing in MoE" (fanout.sh)
 *   [EC-math]   "Expert choice routing" (aicassindra.com, transformer math)
 *   [TC-card]   "MoE token-choice routing" (zenaique.com flashcard)
 *   [Strat]     "How MoE routing strategies make large language models
 *                efficient" (ehga.org)
 *   [Guide]     "MoE routing strategies explained: top-k, expert choice,
 *                sigmoid gating and dynamic routing (2026 guide)"
 *                (ncijnetwork.com)
 * Every sum is accumulated in double; values the GPU stores in fp32 or bf16
 * are rounded to that type at the same storage point.
 *
 * Parity status of each function is stated beside it; all are pinned by the
 * `-m "not gpu"` tests except where marked otherwise.
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* score functions, activations, weight modes and storage types */
enum { ORC_SOFTMAX = 0, ORC_SIGMOID = 1, ORC_SQRTSOFTPLUS = 2 };
enum { ORC_RELU = 0, ORC_GELU = 1, ORC_SWIGLU = 2 };
enum { ORC_W_RAW = 0, ORC_W_NORMALIZED = 1 };
enum { ORC_STORE_F32 = 0, ORC_STORE_BF16 = 1 };

/* Round a double to the nearest bf16 value (ties to even); result as float. */
float orc_round_bf16(double v);
void orc_round_bf16_n(long long count, const double* in, float* out);

/* Router: logits L = X.W_g (+ per-expert logit bias), S = softmax or sigmoid
 * of L, lse = logsumexp of each row of L.
 * X [n,d], Wg [d,E], logit_bias [E] or NULL; outputs logits/S [n,E], lse [n]. */
void orc_router(int n, int d, int E, const float* X, const float* Wg,
                const float* logit_bias, int score, float* logits, float* S,
                double* lse);

/* Expert choice: per expert e, the k tokens with the largest S[:,e], ordered
 * by (score desc, token asc). I, G: [E,k]. */
void orc_select_ec(int n, int E, int k, const float* S, int32_t* I, float* G);

/* Token choice: per token, the K experts with the largest key, key = S
 * (+ sel_bias[e] in fp32 when sel_bias != NULL), ordered by (key desc,
 * expert asc); optionally group-limited (n_groups > 1): group score = fp32
 * sum of its group_topn largest keys, largest first; keep topk_groups groups
 * by (group score desc, group asc). Mixing weight per weights mode, always
 * from the raw S. idx, w: [n,K]. */
void orc_select_tc(int n, int E, int K, const float* S, const float* sel_bias,
                   int n_groups, int topk_groups, int group_topn, int weights,
                   int32_t* idx, float* w);

/* The mixing weights of a given selection idx [n,K] (raw, or normalised over
 * the K selected raw scores in idx order): orc_select_tc's weights for its
 * own selection. */
void orc_weights_tc(int n, int E, int K, const float* S, const int32_t* idx, int weights,
                    float* w);

/* Capacity in arrival (token) order. cap < 0 means dropless.
 * load[E] = selections per expert, kept[E] = rows kept per expert,
 * drop[n,K] = 1 where the assignment overflowed, pos[n,K] = queue position
 * of each kept assignment (-1 if dropped). */
void orc_capacity(int n, int E, int K, const int32_t* idx, int cap,
                  uint8_t* drop, int32_t* load, int32_t* kept, int32_t* pos);

/* One expert FFN on m rows: Y = act(X W1^T) W2^T, or for SwiGLU
 * Y = (silu(X W1^T) * (X W3^T)) W2^T. W1, W3 [h,d], W2 [d,h], X [m,d].
 * The hidden activations and Y are rounded to `store` (fp32 or bf16). */
void orc_expert_ffn(int m, int d, int h, int act, int store, const float* X,
                    const float* W1, const float* W3, const float* W2,
                    float* Y);

/* Combine: out[t] += gate[p] * Y[p] for each pair p with pair_token[p] = t,
 * summed in double over the pairs in the order given, then rounded to
 * `store`. Tokens with no pair get 0. out [n,d], Y [P,d]. */
void orc_combine(int n, int d, int P, const int32_t* pair_token,
                 const float* pair_gate, const float* Y, int store, float* out);

/* Aux values. lb = coef * E * sum_e f_e P_e with f_e = load_e / (n K) and
 * P_e = mean_t S[t,e]; z = coef * mean_t lse_t^2; maxvio = max_e load_e /
 * (n K / E) - 1. */
void orc_aux(int n, int E, int K, const int32_t* load, const float* S,
             const double* lse, double lb_coef, double z_coef, double* lb,
             double* z, double* maxvio);

/* Selection-only bias update after one step: b_e <- b_e - rate *
 * sign(load_e - n K / E), in fp32. */
void orc_bias_update(int n, int E, int K, const int32_t* load, float rate,
                     float* bias);

/* Expert-choice experts-per-token histogram: hist[j] = number of tokens
 * picked by exactly j experts, j = 0..E. */
void orc_ec_histogram(int n, int E, int k, const int32_t* I, int32_t* hist);

/* ---- backward pass: the chain rule through the forward above ----------
 * The loss is <dout, out> + lb_coef L_lb + z_coef L_z (token choice; expert
 * choice has no aux loss). Counts, selections and drops are piecewise
 * constant and pass no gradient. Values the GPU stores are rounded to
 * `store` at the same points: dY, the pre-activations U (= X W1^T) and
 * V (= X W3^T), dU, dV, the per-row dX of an expert and the weight
 * gradients. */

/* Combine backward, for each pair p = (token t, gate g): dY[p] = g dout[t]
 * (rounded to store) and dgate[p] = <dout[t], Y[p]> (double sum, fp32). */
void orc_combine_backward(int n, int d, int P, const int32_t* pair_token,
                          const float* pair_gate, const float* Y,
                          const float* dout, int store, float* dY,
                          float* dgate);

/* One expert's backward over its m rows X [m,d] with the stored output
 * gradient dY [m,d]: dH = dY W2; dU = dH * act'(U) (SwiGLU: dU = dH V
 * silu'(U), dV = dH silu(U), from the stored U, V); dX = dU W1 (+ dV W3)
 * [m,d]; dW1 = dU^T X, dW3 = dV^T X [h,d]; dW2 = dY^T H [d,h], H as the
 * forward stores it. dW3 only for SwiGLU (else may be NULL). absW1 / absW3
 * / absW2, when absW1 is not NULL, receive the same sums taken over the
 * absolute values of their terms (sum_r |dU_rj| |x_ri| and so on): not part
 * of the method, a bound for comparing a computed gradient whose factors
 * were stored at lower precision (a factor's rounding moves an element by at
 * most its relative spacing times that term). */
void orc_expert_ffn_backward(int m, int d, int h, int act, int store,
                             const float* X, const float* W1, const float* W3,
                             const float* W2, const float* dY, float* dX,
                             float* dW1, float* dW3, float* dW2, float* absW1,
                             float* absW3, float* absW2);

/* Token-choice mixing weights backward: dS [n,E] (double, accumulated into)
 * from the weight gradients dw [n,K] of the selected experts idx [n,K]:
 * raw weights pass dw through; normalised weights w_k = s_k / sum_j s_j give
 * dS_k = (dw_k - sum_j w_j dw_j) / sum_j s_j. */
void orc_gate_backward_tc(int n, int E, int K, const float* S,
                          const int32_t* idx, int weights, const double* dw,
                          double* dS);

/* Score backward: dL [n,E] from dS [n,E] plus the balance-loss term
 * lb_coef E f_e / n (f_e = load_e / (n K)), through softmax (dL = S (dS -
 * <S, dS>)), sigmoid (dS s (1 - s)) or sqrt(softplus) (dS sigma(l) / (2 s)),
 * plus the z-loss term z_coef 2 lse_t / n softmax(l_t). lb_coef = 0 and
 * z_coef = 0 switch the aux terms off (load may then be NULL). */
void orc_score_backward(int n, int E, int K, int score, const float* logits,
                        const float* S, const double* lse, const int32_t* load,
                        double lb_coef, double z_coef, const double* dS,
                        double* dL);

/* Router backward: dWg = X^T dL [d,E] (fp32), dXr = dL Wg^T [n,d] (double,
 * the router's share of dX). */
void orc_router_backward(int n, int d, int E, const float* X, const float* Wg,
                         const double* dL, float* dWg, double* dXr);

#ifdef __cplusplus
}
#endif
#endif
