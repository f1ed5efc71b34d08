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

#ifdef __cplusplus
}
#endif
#endif
