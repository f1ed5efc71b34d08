/*
 * CPU oracle for the MoE routing-and-dispatch layer. TEST INFRASTRUCTURE
 * ONLY: see moe_oracle.h for who may call it and the page key used in the
 * citations below. Single-threaded, double accumulation, no blocking or
 * reordering beyond what each definition states.
 */
#include "moe_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ */
/* storage rounding                                                     */
/* ------------------------------------------------------------------ */

/* bf16: 8 exponent bits, 7 stored mantissa bits. Round v itself (not an
 * intermediate float) to the nearest representable value, ties to even. */
float orc_round_bf16(double v) {
  if (v != v) return (float)v;
  if (v == 0.0) return (float)v;
  if (isinf(v)) return (float)v;
  int ex;
  frexp(v, &ex);            /* |v| = m * 2^ex, m in [0.5, 1) */
  int e = ex - 1;           /* |v| in [2^e, 2^(e+1)) */
  if (e < -126) e = -126;   /* subnormal range keeps the smallest spacing */
  int ulp_exp = e - 7;      /* spacing of bf16 values in that binade */
  double q = ldexp(v, -ulp_exp);
  double r = nearbyint(q);  /* default rounding mode: ties to even */
  double out = ldexp(r, ulp_exp);
  /* largest finite bf16 = (2 - 2^-7) * 2^127 */
  double maxv = ldexp(255.0, 120);
  if (out > maxv) return INFINITY;
  if (out < -maxv) return -INFINITY;
  return (float)out; /* exactly representable: 8 significant bits */
}

void orc_round_bf16_n(long long count, const double* in, float* out) {
  for (long long i = 0; i < count; ++i) out[i] = orc_round_bf16(in[i]);
}

static float round_store(double v, int store) {
  return store == ORC_STORE_BF16 ? orc_round_bf16(v) : (float)v;
}

/* ------------------------------------------------------------------ */
/* router: [EC-math] "Token-choice and its load-balance headache" and    */
/* "The transposed selection" (S = softmax(X W_g), W_g: [d,E]);          */
/* [TC-card] "Token-choice: the token picks experts" (z_t = W h_t);      */
/* [Guide] "4. Sigmoid gating with aux-loss-free bias" (sigmoid score).  */
/* ------------------------------------------------------------------ */
void orc_router(int n, int d, int E, const float* X, const float* Wg,
                const float* logit_bias, int score, float* logits, float* S,
                double* lse) {
  double* acc = (double*)malloc(sizeof(double) * (size_t)E);
  for (int t = 0; t < n; ++t) {
    /* each logit is the plain sum over i = 0..d-1 in increasing order; the
     * expert index runs innermost only so that W_g is read row by row */
    for (int e = 0; e < E; ++e) acc[e] = 0.0;
    for (int i = 0; i < d; ++i) {
      const double x = (double)X[(size_t)t * d + i];
      const float* w = Wg + (size_t)i * E;
      for (int e = 0; e < E; ++e) acc[e] += x * (double)w[e];
    }
    for (int e = 0; e < E; ++e) {
      double v = acc[e];
      if (logit_bias) v += (double)logit_bias[e];
      logits[(size_t)t * E + e] = (float)v;
    }
    const float* L = logits + (size_t)t * E;
    double m = L[0];
    for (int e = 1; e < E; ++e)
      if (L[e] > m) m = L[e];
    double z = 0.0;
    for (int e = 0; e < E; ++e) z += exp((double)L[e] - m);
    lse[t] = m + log(z);
    for (int e = 0; e < E; ++e) {
      double s;
      if (score == ORC_SIGMOID) {
        s = 1.0 / (1.0 + exp(-(double)L[e]));
      } else if (score == ORC_SQRTSOFTPLUS) {
        /* [Guide] "4. Sigmoid gating with aux-loss-free bias" names the
         * score only; read as sqrt(softplus(l)), softplus(l) = ln(1 + e^l),
         * evaluated as l + ln(1 + e^-l) for l > 0 so that e^l cannot
         * overflow */
        const double l = (double)L[e];
        const double sp = l > 0.0 ? l + log1p(exp(-l)) : log1p(exp(l));
        s = sqrt(sp);
      } else {
        s = exp((double)L[e] - m) / z;
      }
      S[(size_t)t * E + e] = (float)s;
    }
  }
  free(acc);
}

/* ------------------------------------------------------------------ */
/* top-k with a strict total order: larger key first, lower index first  */
/* among equal keys. IEEE comparison, so -0 == +0.                       */
/* ------------------------------------------------------------------ */
typedef struct {
  float key;
  int idx;
} keyed;

static int cmp_keyed(const void* pa, const void* pb) {
  const keyed* a = (const keyed*)pa;
  const keyed* b = (const keyed*)pb;
  if (a->key > b->key) return -1;
  if (a->key < b->key) return 1;
  return (a->idx < b->idx) ? -1 : (a->idx > b->idx);
}

/* [EC-math] "The math: a gating matrix and top-k over tokens": G, I = TopK
 * over the token axis of S^T, one (index, gate) pair per kept token, so
 * I, G are [E,k]. [TC-vs-EC] "Who picks whom": k = n c / e per expert. */
void orc_select_ec(int n, int E, int k, const float* S, int32_t* I, float* G) {
  keyed* col = (keyed*)malloc(sizeof(keyed) * (size_t)n);
  for (int e = 0; e < E; ++e) {
    for (int t = 0; t < n; ++t) {
      col[t].key = S[(size_t)t * E + e];
      col[t].idx = t;
    }
    qsort(col, (size_t)n, sizeof(keyed), cmp_keyed);
    for (int j = 0; j < k; ++j) {
      I[(size_t)e * k + j] = col[j].idx;
      G[(size_t)e * k + j] = S[(size_t)col[j].idx * E + e];
    }
  }
  free(col);
}

/* [EC-math] "Token-choice ..." (each token to its top-k experts);
 * [Guide] "1. Softmax top-k token choice" (softmax over the kept scores
 * sets the mixing weights), "4. Sigmoid gating with aux-loss-free bias"
 * (bias only when choosing; weights from raw scores), "5. Group-limited and
 * node-limited routing" (8 groups, keep 4, then the final top-8). */
void orc_select_tc(int n, int E, int K, const float* S, const float* sel_bias,
                   int n_groups, int topk_groups, int group_topn, int weights,
                   int32_t* idx, float* w) {
  keyed* all = (keyed*)malloc(sizeof(keyed) * (size_t)E);
  keyed* cand = (keyed*)malloc(sizeof(keyed) * (size_t)E);
  keyed* grp = (keyed*)malloc(sizeof(keyed) * (size_t)(n_groups > 0 ? n_groups : 1));
  char* allowed = (char*)malloc((size_t)E);
  keyed* tmp = (keyed*)malloc(sizeof(keyed) * (size_t)E); /* one group's keys */
  for (int t = 0; t < n; ++t) {
    const float* s = S + (size_t)t * E;
    for (int e = 0; e < E; ++e) {
      all[e].key = sel_bias ? s[e] + sel_bias[e] : s[e]; /* fp32 add */
      all[e].idx = e;
      allowed[e] = 1;
    }
    if (n_groups > 1) {
      int gsize = E / n_groups;
      for (int g = 0; g < n_groups; ++g) {
        for (int j = 0; j < gsize; ++j) tmp[j] = all[g * gsize + j];
        qsort(tmp, (size_t)gsize, sizeof(keyed), cmp_keyed);
        float sum = 0.0f; /* fp32, largest key first */
        for (int j = 0; j < group_topn; ++j) sum = sum + tmp[j].key;
        grp[g].key = sum;
        grp[g].idx = g;
      }
      qsort(grp, (size_t)n_groups, sizeof(keyed), cmp_keyed);
      for (int e = 0; e < E; ++e) allowed[e] = 0;
      for (int j = 0; j < topk_groups; ++j) {
        int g = grp[j].idx;
        for (int e = g * gsize; e < (g + 1) * gsize; ++e) allowed[e] = 1;
      }
    }
    int nc = 0;
    for (int e = 0; e < E; ++e)
      if (allowed[e]) cand[nc++] = all[e];
    qsort(cand, (size_t)nc, sizeof(keyed), cmp_keyed);
    double denom = 0.0;
    for (int j = 0; j < K; ++j) denom += (double)s[cand[j].idx];
    for (int j = 0; j < K; ++j) {
      int e = cand[j].idx;
      idx[(size_t)t * K + j] = e;
      w[(size_t)t * K + j] =
          (weights == ORC_W_NORMALIZED) ? (float)((double)s[e] / denom) : s[e];
    }
  }
  free(all);
  free(cand);
  free(grp);
  free(allowed);
  free(tmp);
}

/* Mixing weights of a given token-choice selection idx [n,K]: the raw score
 * of each selected expert, or ([Guide] "1." softmax over the kept scores,
 * "4." weights from the raw sigmoid scores) each selected raw score divided
 * by their sum, taken in the order idx lists them. For the selection
 * orc_select_tc makes, this is the weight it returns. */
void orc_weights_tc(int n, int E, int K, const float* S, const int32_t* idx, int weights,
                    float* w) {
  for (int t = 0; t < n; ++t) {
    const float* s = S + (size_t)t * E;
    const int32_t* sel = idx + (size_t)t * K;
    double denom = 0.0;
    for (int j = 0; j < K; ++j) denom += (double)s[sel[j]];
    for (int j = 0; j < K; ++j)
      w[(size_t)t * K + j] =
          (weights == ORC_W_NORMALIZED) ? (float)((double)s[sel[j]] / denom) : s[sel[j]];
  }
}

/* [TC-vs-EC] "Dropped tokens flow in opposite directions": tokens that arrive
 * after an expert's buffer fills skip it and pass on the residual.
 * [Guide] "2. Top-1 switch routing with a capacity factor": buffer = tokens
 * per batch / experts x capacity factor. Arrival order = token order. */
void orc_capacity(int n, int E, int K, const int32_t* idx, int cap,
                  uint8_t* drop, int32_t* load, int32_t* kept, int32_t* pos) {
  int32_t* used = (int32_t*)calloc((size_t)E, sizeof(int32_t));
  for (int e = 0; e < E; ++e) load[e] = 0;
  for (int t = 0; t < n; ++t) {
    for (int j = 0; j < K; ++j) {
      size_t a = (size_t)t * K + j;
      int e = idx[a];
      load[e] += 1;
      if (cap < 0 || used[e] < cap) {
        pos[a] = used[e];
        used[e] += 1;
        drop[a] = 0;
      } else {
        pos[a] = -1;
        drop[a] = 1;
      }
    }
  }
  for (int e = 0; e < E; ++e) kept[e] = used[e];
  free(used);
}

/* ------------------------------------------------------------------ */
/* expert FFN: [EC-math] "The math": Y[e] = G[e] * Expert_e(X_in[e]) on  */
/* dense per-expert batches (the gate is applied in orc_combine). The    */
/* expert is the block's MLP ([Strat] "The Core Mechanism").             */
/* ------------------------------------------------------------------ */
static double act_fn(int act, double u) {
  if (act == ORC_RELU) return u > 0.0 ? u : 0.0;
  /* GELU, exact erf form */
  return 0.5 * u * (1.0 + erf(u / sqrt(2.0)));
}

void orc_expert_ffn(int m, int d, int h, int act, int store, const float* X,
                    const float* W1, const float* W3, const float* W2,
                    float* Y) {
  float* H = (float*)malloc(sizeof(float) * (size_t)h);
  for (int r = 0; r < m; ++r) {
    const float* x = X + (size_t)r * d;
    for (int j = 0; j < h; ++j) {
      double a = 0.0;
      for (int i = 0; i < d; ++i) a += (double)x[i] * (double)W1[(size_t)j * d + i];
      double hv;
      if (act == ORC_SWIGLU) {
        double b = 0.0;
        for (int i = 0; i < d; ++i) b += (double)x[i] * (double)W3[(size_t)j * d + i];
        hv = (a / (1.0 + exp(-a))) * b; /* silu(a) * b */
      } else {
        hv = act_fn(act, a);
      }
      H[j] = round_store(hv, store);
    }
    for (int i = 0; i < d; ++i) {
      double y = 0.0;
      for (int j = 0; j < h; ++j) y += (double)W2[(size_t)i * h + j] * (double)H[j];
      Y[(size_t)r * d + i] = round_store(y, store);
    }
  }
  free(H);
}

/* [EC-math] "The math": out = scatter_add(Y, I) back to [n, d]: each token's
 * gate-scaled expert outputs summed into its slot; a token no expert picked
 * gets nothing ("Variable tokens-per-token"). */
void orc_combine(int n, int d, int P, const int32_t* pair_token,
                 const float* pair_gate, const float* Y, int store, float* out) {
  double* acc = (double*)calloc((size_t)n * d, sizeof(double));
  for (int p = 0; p < P; ++p) {
    int t = pair_token[p];
    double g = pair_gate[p];
    for (int i = 0; i < d; ++i) acc[(size_t)t * d + i] += g * (double)Y[(size_t)p * d + i];
  }
  for (size_t q = 0; q < (size_t)n * d; ++q) out[q] = round_store(acc[q], store);
  free(acc);
}

/* [TC-vs-EC] "What each direction guarantees": load-balancing loss at
 * coefficient 0.01 against a target of n K / E tokens per expert, router
 * z-loss at 0.001. The pages name the losses, not their formulas; these are
 * the readings stated in moe_oracle.h. MaxVio: [Guide] TL;DR. */
void orc_aux(int n, int E, int K, const int32_t* load, const float* S,
             const double* lse, double lb_coef, double z_coef, double* lb,
             double* z, double* maxvio) {
  double sum = 0.0;
  for (int e = 0; e < E; ++e) {
    double col = 0.0;
    for (int t = 0; t < n; ++t) col += (double)S[(size_t)t * E + e];
    double f = (double)load[e] / ((double)n * K);
    double p = col / n;
    sum += f * p;
  }
  *lb = lb_coef * E * sum;
  double zz = 0.0;
  for (int t = 0; t < n; ++t) zz += lse[t] * lse[t];
  *z = z_coef * zz / n;
  double mean = (double)n * K / E;
  int mx = 0;
  for (int e = 0; e < E; ++e)
    if (load[e] > mx) mx = load[e];
  *maxvio = (double)mx / mean - 1.0;
}

/* [Guide] "4. Sigmoid gating with aux-loss-free bias": after each step the
 * bias drops for overloaded experts and rises for idle ones. */
void orc_bias_update(int n, int E, int K, const int32_t* load, float rate,
                     float* bias) {
  for (int e = 0; e < E; ++e) {
    long long diff = (long long)load[e] * E - (long long)n * K; /* sign only */
    if (diff > 0)
      bias[e] = bias[e] - rate;
    else if (diff < 0)
      bias[e] = bias[e] + rate;
  }
}

/* [TC-vs-EC] "Who picks whom" / [EC-math] "Variable tokens-per-token":
 * under expert choice a token gets 0..E experts. */
void orc_ec_histogram(int n, int E, int k, const int32_t* I, int32_t* hist) {
  int32_t* cnt = (int32_t*)calloc((size_t)n, sizeof(int32_t));
  for (size_t a = 0; a < (size_t)E * k; ++a) cnt[I[a]] += 1;
  for (int j = 0; j <= E; ++j) hist[j] = 0;
  for (int t = 0; t < n; ++t) hist[cnt[t]] += 1;
  free(cnt);
}

/* ------------------------------------------------------------------ */
/* backward pass: the gradient of the forward above by the chain rule.   */
/* [TC-vs-EC] "What each direction guarantees" names the training-time  */
/* losses (load balance 0.01, router z-loss 0.001) whose gradients join  */
/* the gradient of <dout, out> here. Storage points mirror the forward:  */
/* values the GPU stores are rounded to `store` where it stores them.    */
/* ------------------------------------------------------------------ */
static double sigm(double u) { return 1.0 / (1.0 + exp(-u)); }

/* d act / du; SwiGLU's gate part is handled by the caller */
static double act_grad(int act, double u) {
  if (act == ORC_RELU) return u > 0.0 ? 1.0 : 0.0;
  /* d/du [u Phi(u)] = Phi(u) + u phi(u) */
  const double pi = 3.14159265358979323846;
  return 0.5 * (1.0 + erf(u / sqrt(2.0))) + u * exp(-0.5 * u * u) / sqrt(2.0 * pi);
}

void orc_combine_backward(int n, int d, int P, const int32_t* pair_token,
                          const float* pair_gate, const float* Y,
                          const float* dout, int store, float* dY,
                          float* dgate) {
  (void)n;
  for (int p = 0; p < P; ++p) {
    const int t = pair_token[p];
    const double gate = pair_gate[p];
    double s = 0.0;
    for (int i = 0; i < d; ++i) {
      const double go = dout[(size_t)t * d + i];
      dY[(size_t)p * d + i] = round_store(gate * go, store);
      s += go * (double)Y[(size_t)p * d + i];
    }
    dgate[p] = (float)s;
  }
}

void orc_expert_ffn_backward(int m, int d, int h, int act, int store,
                             const float* X, const float* W1, const float* W3,
                             const float* W2, const float* dY, float* dX,
                             float* dW1, float* dW3, float* dW2, float* absW1,
                             float* absW3, float* absW2) {
  const int swiglu = act == ORC_SWIGLU;
  const int want_abs = absW1 != NULL;
  double* aW1 = (double*)calloc((size_t)h * d, sizeof(double));
  double* aW3 = swiglu ? (double*)calloc((size_t)h * d, sizeof(double)) : NULL;
  double* aW2 = (double*)calloc((size_t)d * h, sizeof(double));
  /* the same sums over |terms| (a bound helper for comparing stored values) */
  double* bW1 = want_abs ? (double*)calloc((size_t)h * d, sizeof(double)) : NULL;
  double* bW3 = want_abs && swiglu ? (double*)calloc((size_t)h * d, sizeof(double)) : NULL;
  double* bW2 = want_abs ? (double*)calloc((size_t)d * h, sizeof(double)) : NULL;
  float* Hs = (float*)malloc(sizeof(float) * (size_t)h);
  float* dUs = (float*)malloc(sizeof(float) * (size_t)h);
  float* dVs = (float*)malloc(sizeof(float) * (size_t)h);
  for (int r = 0; r < m; ++r) {
    const float* x = X + (size_t)r * d;
    const float* dy = dY + (size_t)r * d;
    for (int j = 0; j < h; ++j) {
      /* pre-activations, as the forward computes them */
      double u = 0.0, v = 0.0;
      for (int i = 0; i < d; ++i) u += (double)x[i] * (double)W1[(size_t)j * d + i];
      if (swiglu)
        for (int i = 0; i < d; ++i) v += (double)x[i] * (double)W3[(size_t)j * d + i];
      Hs[j] = round_store(swiglu ? (u / (1.0 + exp(-u))) * v : act_fn(act, u), store);
      /* the stored pre-activations the backward works from */
      const double us = round_store(u, store);
      const double vs = swiglu ? (double)round_store(v, store) : 0.0;
      /* dH = dY W2 (column j of W2), not stored */
      double dh = 0.0;
      for (int i = 0; i < d; ++i) dh += (double)dy[i] * (double)W2[(size_t)i * h + j];
      if (swiglu) {
        const double sg = sigm(us);
        /* silu(u) = u sigma(u); silu'(u) = sigma(u) (1 + u (1 - sigma(u))) */
        dUs[j] = round_store(dh * vs * sg * (1.0 + us * (1.0 - sg)), store);
        dVs[j] = round_store(dh * us * sg, store);
      } else {
        dUs[j] = round_store(dh * act_grad(act, us), store);
      }
    }
    /* dX = dU W1 (+ dV W3) */
    for (int i = 0; i < d; ++i) {
      double a = 0.0;
      for (int j = 0; j < h; ++j) a += (double)dUs[j] * (double)W1[(size_t)j * d + i];
      if (swiglu)
        for (int j = 0; j < h; ++j) a += (double)dVs[j] * (double)W3[(size_t)j * d + i];
      dX[(size_t)r * d + i] = round_store(a, store);
    }
    /* weight gradients: outer products summed over the rows */
    for (int j = 0; j < h; ++j)
      for (int i = 0; i < d; ++i) {
        aW1[(size_t)j * d + i] += (double)dUs[j] * (double)x[i];
        if (swiglu) aW3[(size_t)j * d + i] += (double)dVs[j] * (double)x[i];
      }
    for (int i = 0; i < d; ++i)
      for (int j = 0; j < h; ++j) aW2[(size_t)i * h + j] += (double)dy[i] * (double)Hs[j];
    if (want_abs) {
      for (int j = 0; j < h; ++j)
        for (int i = 0; i < d; ++i) {
          bW1[(size_t)j * d + i] += fabs((double)dUs[j]) * fabs((double)x[i]);
          if (swiglu) bW3[(size_t)j * d + i] += fabs((double)dVs[j]) * fabs((double)x[i]);
        }
      for (int i = 0; i < d; ++i)
        for (int j = 0; j < h; ++j)
          bW2[(size_t)i * h + j] += fabs((double)dy[i]) * fabs((double)Hs[j]);
    }
  }
  for (size_t q = 0; q < (size_t)h * d; ++q) {
    dW1[q] = round_store(aW1[q], store);
    if (swiglu) dW3[q] = round_store(aW3[q], store);
    dW2[q] = round_store(aW2[q], store);
  }
  if (want_abs)
    for (size_t q = 0; q < (size_t)h * d; ++q) {
      absW1[q] = (float)bW1[q];
      if (swiglu && absW3) absW3[q] = (float)bW3[q];
      if (absW2) absW2[q] = (float)bW2[q];
    }
  free(aW1);
  free(aW3);
  free(aW2);
  free(bW1);
  free(bW3);
  free(bW2);
  free(Hs);
  free(dUs);
  free(dVs);
}

void orc_gate_backward_tc(int n, int E, int K, const float* S,
                          const int32_t* idx, int weights, const double* dw,
                          double* dS) {
  for (int t = 0; t < n; ++t) {
    const int32_t* it = idx + (size_t)t * K;
    const double* g = dw + (size_t)t * K;
    double* ds = dS + (size_t)t * E;
    if (weights == ORC_W_NORMALIZED) {
      /* w_k = s_k / sum_j s_j over the K selected experts */
      double sum = 0.0, dot = 0.0;
      for (int j = 0; j < K; ++j) sum += (double)S[(size_t)t * E + it[j]];
      for (int j = 0; j < K; ++j) dot += ((double)S[(size_t)t * E + it[j]] / sum) * g[j];
      for (int j = 0; j < K; ++j) ds[it[j]] += (g[j] - dot) / sum;
    } else {
      for (int j = 0; j < K; ++j) ds[it[j]] += g[j];
    }
  }
}

void orc_score_backward(int n, int E, int K, int score, const float* logits,
                        const float* S, const double* lse, const int32_t* load,
                        double lb_coef, double z_coef, const double* dS,
                        double* dL) {
  double* g = (double*)malloc(sizeof(double) * (size_t)E);
  for (int t = 0; t < n; ++t) {
    const float* L = logits + (size_t)t * E;
    const float* s = S + (size_t)t * E;
    double* out = dL + (size_t)t * E;
    /* dS plus the balance loss: d/dS[t,e] of lb E sum_e f_e mean_t S[t,e],
     * with f_e = load_e / (n K) held fixed (it counts choices) */
    for (int e = 0; e < E; ++e) {
      g[e] = dS[(size_t)t * E + e];
      if (lb_coef != 0.0)
        g[e] += lb_coef * E * ((double)load[e] / ((double)n * K)) / n;
    }
    if (score == ORC_SIGMOID) {
      for (int e = 0; e < E; ++e) out[e] = g[e] * (double)s[e] * (1.0 - (double)s[e]);
    } else if (score == ORC_SQRTSOFTPLUS) {
      /* s = sqrt(softplus(l)): ds/dl = sigma(l) / (2 s) */
      for (int e = 0; e < E; ++e) out[e] = g[e] * sigm((double)L[e]) / (2.0 * (double)s[e]);
    } else {
      double dot = 0.0;
      for (int e = 0; e < E; ++e) dot += (double)s[e] * g[e];
      for (int e = 0; e < E; ++e) out[e] = (double)s[e] * (g[e] - dot);
    }
    /* z-loss: z mean_t lse_t^2; d lse_t / d l_e = softmax(l)_e */
    if (z_coef != 0.0)
      for (int e = 0; e < E; ++e)
        out[e] += z_coef * 2.0 * lse[t] / n * exp((double)L[e] - lse[t]);
  }
  free(g);
}

void orc_router_backward(int n, int d, int E, const float* X, const float* Wg,
                         const double* dL, float* dWg, double* dXr) {
  double* acc = (double*)calloc((size_t)d * E, sizeof(double));
  for (int t = 0; t < n; ++t) {
    const double* g = dL + (size_t)t * E;
    for (int i = 0; i < d; ++i) {
      const double x = X[(size_t)t * d + i];
      double a = 0.0;
      for (int e = 0; e < E; ++e) {
        acc[(size_t)i * E + e] += x * g[e];
        a += g[e] * (double)Wg[(size_t)i * E + e];
      }
      dXr[(size_t)t * d + i] = a;
    }
  }
  for (size_t q = 0; q < (size_t)d * E; ++q) dWg[q] = (float)acc[q];
  free(acc);
}
