/*
 * libmoe: the forward hot path of a mixture-of-experts layer on one B200
 * (sm_100a): route -> dispatch -> grouped expert FFN -> gate-scaled combine.
 *
 * Source pages of the operations (cited by title and section):
 *   [TC-vs-EC]  "Token choice vs expert choice routing in MoE" (fanout.sh)
 *   [EC-math]   "Expert choice routing" (aicassindra.com, transformer math)
 *   [TC-card]   "MoE token-choice routing" (zenaique.com flashcard)
 *   [Strat]     "How MoE routing strategies make large language models
 *                efficient" (ehga.org)
 *   [Guide]     "MoE routing strategies explained: top-k, expert choice,
 *                sigmoid gating and dynamic routing (2026 guide)"
 *                (ncijnetwork.com)
 *
 * Conventions shared by every entry point
 *   - Every tensor argument is a DEVICE pointer to contiguous row-major
 *     memory owned by the caller. The library never allocates or frees
 *     memory, never synchronises the stream (except moe_read_error), and
 *     never keeps a pointer after a call returns.
 *   - All work is enqueued on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) in launch order; outputs are valid once the stream
 *     reaches them.
 *   - Arguments are validated on the host before any launch; on a non-OK
 *     status nothing was enqueued. MOE_ERR_CUDA means a launch failed (the
 *     stream may hold the launches enqueued before it).
 *   - Device-side waits are bounded (2 s each); a wait that gives up writes
 *     an error code into the first 256 bytes of the workspace (moe_dispatch,
 *     which takes no workspace: into a per-device word), and the kernel
 *     returns. moe_read_error() reports it as MOE_ERR_TIMEOUT.
 *   - Indices are int32, gates fp32. Activations X, expert weights, the
 *     dispatched rows, the hidden activations and the expert outputs are
 *     all of the config's dtype (fp32 or bf16); the router weight W_g, the
 *     logits and the scores are always fp32.
 *
 * Dispatched-row layout ("dense per-expert batches", [EC-math] "The math:
 * a gating matrix and top-k over tokens")
 *   Expert e's rows form one contiguous segment of X_perm / H / Y_perm
 *   starting at offsets[e]; every segment starts on a multiple of
 *   MOE_ROW_ALIGN rows, so one 128-row GEMM tile never spans two experts.
 *   The padding rows between segments are never read for results and are
 *   left unwritten. Within a segment the rows are in token order (token
 *   choice) or in the expert's selection order (expert choice). Shared
 *   experts, when present, own n_pad = roundup(n, 128) rows each after the
 *   routed rows, starting at row moe_shared_row_base().
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(MOE_BUILD)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_ROW_ALIGN 128
#define MOE_AUX_LEN 8
#define MOE_MAX_EXPERTS 256
#define MOE_MAX_TOPK 32
#define MOE_MAX_SHARED 4
#define MOE_EC_MAX_TOKENS 16384
#define MOE_WS_ERROR_BYTES 256

/* a cudaStream_t */
typedef struct CUstream_st* moe_stream_t;

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* a null required pointer, a bad size or mode */
  MOE_ERR_UNSUPPORTED = 2, /* a valid shape the library has no kernel for */
  MOE_ERR_WORKSPACE = 3,   /* workspace null or smaller than required */
  MOE_ERR_CUDA = 4,        /* a CUDA call or launch failed */
  MOE_ERR_TIMEOUT = 5      /* a bounded device-side wait gave up */
} moe_status;

/* [EC-math] "The routing problem: who picks whom": the same score matrix,
 * top-k along the expert axis (token choice) or the token axis (expert
 * choice). */
typedef enum { MOE_EXPERT_CHOICE = 0, MOE_TOKEN_CHOICE = 1 } moe_mode;

/* softmax over experts ([EC-math] "The transposed selection"), an
 * element-wise sigmoid ([Guide] "4. Sigmoid gating with aux-loss-free
 * bias"), or the element-wise sqrt(softplus(l)) = sqrt(ln(1 + e^l)) that the
 * same section names for DeepSeek-V4 (the pages give only the name; this is
 * the plain reading). Selection bias and weight modes apply to every score. */
typedef enum {
  MOE_SCORE_SOFTMAX = 0,
  MOE_SCORE_SIGMOID = 1,
  MOE_SCORE_SQRTSOFTPLUS = 2
} moe_score;

/* Token-choice mixing weights: RAW = the score of the selected expert;
 * NORMALIZED = the selected raw scores divided by their sum. For softmax
 * scores NORMALIZED equals a softmax over the kept logits ([Guide] "1.
 * Softmax top-k token choice"); for sigmoid scores it is [Guide] "4." */
typedef enum { MOE_W_RAW = 0, MOE_W_NORMALIZED = 1 } moe_weights;

/* expert FFN: Y = act(X W1^T) W2^T, or SwiGLU Y = (silu(X W1^T) * X W3^T) W2^T;
 * GELU is the exact erf form. */
typedef enum { MOE_ACT_RELU = 0, MOE_ACT_GELU = 1, MOE_ACT_SWIGLU = 2 } moe_act;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

typedef struct {
  int n;  /* tokens in the routing group (the whole batch) */
  int d;  /* model dim; multiple of 64 (bf16) or of 8 (fp32) */
  int E;  /* routed experts, 1..MOE_MAX_EXPERTS */
  int h;  /* expert hidden dim; multiple of 64 (bf16) or of 8 (fp32) */
  moe_mode mode;
  moe_score score;
  /* token choice: experts per token (1..min(E, MOE_MAX_TOPK)).
   * expert choice: tokens per expert; 0 derives k = floor(n c / E) with
   * c = capacity_factor ([TC-vs-EC] "Who picks whom"). */
  int k;
  float capacity_factor;
  /* token choice only: -1 = dropless; 0 = floor(n / E * capacity_factor)
   * ([Guide] "2. Top-1 switch routing with a capacity factor"); > 0 =
   * explicit rows per expert. Assignments past the buffer are dropped in
   * token order ([TC-vs-EC] "Dropped tokens flow in opposite directions"). */
  int capacity;
  /* group-limited token choice ([Guide] "5. Group-limited and node-limited
   * routing"): n_groups contiguous expert groups; a group's score is the
   * fp32 sum of its group_topn largest selection keys; the topk_groups best
   * groups are kept. n_groups <= 1 disables it. */
  int n_groups, topk_groups, group_topn;
  moe_weights weights;
  moe_act act;
  moe_dtype dtype;
  /* always-on shared experts added with weight 1 ([Guide] "3. Shared plus
   * routed experts"); 0..MOE_MAX_SHARED, same hidden size h. */
  int n_shared;
  /* aux-loss coefficients ([TC-vs-EC] "What each direction guarantees") */
  float lb_coef, z_coef;
} moe_config;

/* aux[] slots (fp32) */
enum {
  MOE_AUX_LB = 0,          /* lb_coef * E * sum_e (load_e / (n K)) * mean_t S[t,e] (token choice) */
  MOE_AUX_Z = 1,           /* z_coef * mean_t logsumexp(logits_t)^2 (moe_route only) */
  MOE_AUX_MAXVIO = 2,      /* max_e load_e / (n K / E) - 1 (token choice) */
  MOE_AUX_DROPPED = 3,     /* assignments dropped by the capacity */
  MOE_AUX_TOKENS_SOME_DROPPED = 4,
  MOE_AUX_TOKENS_ALL_DROPPED = 5,
  MOE_AUX_TOKENS_NO_EXPERT = 6, /* expert choice: tokens no expert picked */
  MOE_AUX_RESERVED = 7
};

/* Routing results. Every pointer is a caller-owned device buffer.
 * slots = K (token choice) or E (expert choice); rows = moe_rows(). */
typedef struct {
  int32_t* idx;       /* required. TC: [n,K] expert ids in (key desc, id asc)
                         order; EC: [E,k] token ids in (score desc, token asc)
                         order ([EC-math] "The math": I = TopK(S^T, k)) */
  float* gate;        /* required. same shape as idx: mixing weight (TC) or
                         gate G = S[token, e] (EC) */
  int32_t* load;      /* required. [E] selections per expert before capacity */
  int32_t* counts;    /* required. [E] rows kept per expert */
  int32_t* offsets;   /* required. [E+1] first dispatched row of each expert;
                         offsets[E] = routed rows in use (padded) */
  int32_t* row_token; /* required. [rows] source token of each dispatched row,
                         -1 on padding rows (entries past offsets[E] unused) */
  int32_t* tok_row;   /* required. [n, slots] dispatched rows feeding each
                         token: the kept ones first (TC: selection order; EC:
                         expert order), then -1 */
  float* tok_gate;    /* required. [n, slots] the matching gates, 0 past the end */
  uint8_t* drop;      /* TC required, EC ignored. [n,K] 1 = dropped by capacity */
  float* scores;      /* required. [n,E] S = softmax or sigmoid of the logits */
  float* logits;      /* optional. [n,E] logits (moe_route only) */
  float* lse;         /* optional. [n] logsumexp of each logits row (moe_route only) */
  float* aux;         /* required. [MOE_AUX_LEN], see the enum above */
  int32_t* ec_hist;   /* optional (EC). [E+1] tokens picked by exactly j experts */
} moe_route_out;

/* Human-readable name of a status. Never NULL. */
MOE_API const char* moe_status_string(moe_status s);

/* Checks a config; MOE_OK if every entry point accepts it. */
MOE_API moe_status moe_validate(const moe_config* cfg);

/* Kernels each call enqueues for `cfg` on the current device (for graph
 * capture and accounting): moe_route (router, one more for the split-k
 * reduce that small batches use, then EC select + finish or TC histogram +
 * scan + scatter), moe_dispatch, moe_expert_ffn, moe_combine. Any output
 * pointer may be NULL. No counterpart on the pages. */
MOE_API moe_status moe_launch_counts(const moe_config* cfg, int* route, int* dispatch,
                                     int* ffn, int* combine);

/* Derived sizes: k_eff (EC tokens per expert or TC experts per token),
 * capacity_eff (TC rows per expert, -1 dropless), slots (columns of
 * tok_row), rows (rows of X_perm / H / Y_perm, shared rows included),
 * shared_row_base (first shared-expert row). Any output pointer may be NULL. */
MOE_API moe_status moe_sizes(const moe_config* cfg, int* k_eff, int* capacity_eff, int* slots,
                     int* rows, int* shared_row_base);

/* Workspace bytes for moe_route / moe_route_from_scores / moe_expert_ffn
 * (route_bytes) and for moe_layer_forward (layer_bytes, which also holds
 * X_perm, H and Y_perm). Any output pointer may be NULL. The workspace needs
 * 256-byte alignment; only its first MOE_WS_ERROR_BYTES (the error word)
 * must be zeroed once, by moe_workspace_init, before the first call. */
MOE_API moe_status moe_workspace_size(const moe_config* cfg, size_t* route_bytes,
                              size_t* layer_bytes);

/* Router + selection + capacity + aux.
 * X [n,d] (cfg dtype), Wg [d,E] fp32, logit_bias [E] fp32 or NULL (added to
 * the logits: it moves both selection and weights), sel_bias [E] fp32 or
 * NULL (token choice only: added to the scores for selection only, [Guide]
 * "4. Sigmoid gating with aux-loss-free bias").
 * [EC-math] "The transposed selection": S = softmax(X W_g); [TC-card]
 * "Token-choice: the token picks experts": z_t = W h_t. */
MOE_API moe_status moe_route(const moe_config* cfg, const void* X, const float* Wg,
                     const float* logit_bias, const float* sel_bias, moe_route_out* out,
                     void* ws, size_t ws_bytes, moe_stream_t stream);

/* Selection + capacity + aux from a caller-supplied score matrix S [n,E]
 * fp32 (scores written to out->scores are copied from S). Given identical S,
 * idx, load, counts, offsets, row_token, tok_row and drop are bit-identical
 * to moe_route's. aux Z is 0 (no logits). */
MOE_API moe_status moe_route_from_scores(const moe_config* cfg, const float* S,
                                 const float* sel_bias, moe_route_out* out, void* ws,
                                 size_t ws_bytes, moe_stream_t stream);

/* Gather ([EC-math] "The math": X_in[e] = P[e] X with P = onehot(I), done as
 * an index gather): X_perm[r] = X[t] for every token t and every row r >= 0
 * of its list route->tok_row[t, :] (the same rows as those with
 * row_token[r] == t). X [n,d], X_perm [rows,d], both 16-byte aligned (else
 * MOE_ERR_INVALID_ARG). Rows not in any list are left untouched. Uses
 * route->tok_row, row_token and offsets. When a token feeds 4 or more rows
 * (token choice with K >= 4), each token's row is read once and written to
 * all of its rows by TMA bulk copies staged in shared memory; the staging
 * wait is bounded, and a timeout is reported by the next moe_read_error on
 * this device. Otherwise each row is copied by one warp with 16-byte loads. */
MOE_API moe_status moe_dispatch(const moe_config* cfg, const void* X, const moe_route_out* route,
                        void* X_perm, moe_stream_t stream);

/* Grouped expert FFN over the dispatched layout ([EC-math] "The math":
 * Expert_e(X_in[e]) on dense per-expert batches). Routed expert e reads rows
 * [offsets[e], offsets[e+1]) of X_perm; shared expert s reads all n rows of
 * X. W1, W3 [E,h,d]; W2 [E,d,h]; sW1, sW3 [n_shared,h,d]; sW2
 * [n_shared,d,h]; W3 / sW3 only for SwiGLU (else NULL); shared pointers only
 * when n_shared > 0. H [rows,h] receives the hidden activations, Y_perm
 * [rows,d] the expert outputs (gate not applied). counts [E] (moe_route's
 * out->counts: the real rows at the start of each segment) may be NULL; with
 * it, token choice with 128 to 512 rows per expert on average computes the
 * down projection for those rows only (16-row granularity, weights as the
 * MMA's M side) instead of whole 128-row blocks, and rows past counts[e] of
 * Y_perm are then left unwritten. bf16 runs on the tcgen05 tensor cores with
 * fp32 accumulation; fp32 runs on FFMA. */
MOE_API moe_status moe_expert_ffn(const moe_config* cfg, const void* X, const void* X_perm,
                          const int32_t* offsets, const int32_t* counts, const void* W1,
                          const void* W3, const void* W2, const void* sW1, const void* sW3,
                          const void* sW2, void* H, void* Y_perm, void* ws,
                          size_t ws_bytes, moe_stream_t stream);

/* moe_dispatch + moe_expert_ffn without X_perm: the first projection reads
 * each routed row of X directly (row r of expert e's segment is
 * X[route->row_token[r]]; padding rows read token 0 and are never used), so
 * the gathered copy never goes through HBM ([EC-math] "The math": X_in[e] =
 * P[e] X feeds Expert_e). Same weights, H, Y_perm and workspace as
 * moe_expert_ffn; results are identical to dispatch followed by
 * moe_expert_ffn. bf16 gathers with TMA tile::gather4 loads, 32 per 64-deep
 * k-block of a 128-row tile: it saves X_perm's memory and HBM round trip but
 * runs the first projection about 2x slower than the unfused pair on B200,
 * so moe_layer_forward does not use it. */
MOE_API moe_status moe_expert_ffn_gathered(const moe_config* cfg, const void* X,
                                           const moe_route_out* route, const void* W1,
                                           const void* W3, const void* W2, const void* sW1,
                                           const void* sW3, const void* sW2, void* H,
                                           void* Y_perm, void* ws, size_t ws_bytes,
                                           moe_stream_t stream);

/* Gate-scaled combine ([EC-math] "The math": Y[e] = G[e] * Expert_e(.),
 * out = scatter_add(Y, I)), computed owner-side: out[t] = sum over t's
 * tok_row entries of tok_gate * Y_perm[row] (+ each shared expert's row with
 * weight 1), accumulated in fp32 in list order, stored in the cfg dtype. A
 * token with no entry gets 0 (it passes on the residual, which the caller
 * adds). out [n,d]. */
MOE_API moe_status moe_combine(const moe_config* cfg, const void* Y_perm, const moe_route_out* route,
                       void* out, moe_stream_t stream);

/* The whole layer on one stream: moe_route, moe_dispatch, moe_expert_ffn,
 * moe_combine, with X_perm, H and Y_perm inside the workspace (layer_bytes). */
MOE_API moe_status moe_layer_forward(const moe_config* cfg, const void* X, const float* Wg,
                             const float* logit_bias, const float* sel_bias,
                             const void* W1, const void* W3, const void* W2,
                             const void* sW1, const void* sW3, const void* sW2, void* out,
                             moe_route_out* route, void* ws, size_t ws_bytes,
                             moe_stream_t stream);

/* moe_layer_forward for a caller whose activations live in host memory:
 * enqueues on `stream` one cudaMemcpyAsync of X_host [n,d] into X_dev, the
 * whole layer on X_dev (as moe_layer_forward, writing out_dev), and one
 * cudaMemcpyAsync of out_dev [n,d] back into out_host, all of the config's
 * dtype. X_host and out_host should be page-locked (cudaHostAlloc or
 * cudaHostRegister) so that the copies run asynchronously; pageable memory
 * still gives correct results, with the copies synchronous to the host.
 * X_dev and out_dev are caller-owned device buffers of n*d elements (16-byte
 * aligned); nothing is allocated. out_host holds the result once the stream
 * reaches the end of the call (the call itself does not synchronise). Every
 * check of moe_layer_forward runs before the first copy is enqueued; a
 * failed copy returns MOE_ERR_CUDA. The pages' problem statement ([EC-math]
 * "The math") starts and ends on the device; the copies are the only
 * addition. */
MOE_API moe_status moe_layer_forward_host(const moe_config* cfg, const void* X_host,
                                          const float* Wg, const float* logit_bias,
                                          const float* sel_bias, const void* W1,
                                          const void* W3, const void* W2, const void* sW1,
                                          const void* sW3, const void* sW2, void* out_host,
                                          void* X_dev, void* out_dev, moe_route_out* route,
                                          void* ws, size_t ws_bytes, moe_stream_t stream);

/* Selection-bias update after a step ([Guide] "4. Sigmoid gating with
 * aux-loss-free bias"): bias[e] -= rate * sign(load[e] - n K / E), in fp32;
 * load [E] int32 (from moe_route_out.load), bias [E] fp32 updated in place. */
MOE_API moe_status moe_bias_update(const moe_config* cfg, const int32_t* load, float rate,
                           float* bias, moe_stream_t stream);

/* moe_route without a workspace, for callers that cannot allocate device
 * memory when they route (an application whose device memory budget is fixed
 * at start-up, or a plugin inside a framework that owns all device
 * allocations). The pages have no counterpart: this is a memory-management
 * variant of moe_route, with identical arguments minus the workspace and
 * identical results. Its scratch is a library-owned static device array of
 * MOE_ROUTE_NOALLOC_SCRATCH_BYTES, held on every GPU that loads the library
 * until the process exits; configs needing more routing scratch than that
 * (moe_workspace_size's route_bytes) return MOE_ERR_WORKSPACE before
 * anything is enqueued. It calls no cudaMalloc, cudaFree or other allocating
 * routine. The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress); make that first call before any stream capture.
 * Every call first zeroes the array's error word with a cudaMemsetAsync on
 * `stream`, so the word reports that call's routing only; read it with
 * moe_read_error(NULL, stream, &detail) after the call and before the next
 * one. Every call shares the one array, so calls that overlap on the GPU (on
 * different streams or threads) race. */
#define MOE_ROUTE_NOALLOC_SCRATCH_BYTES (4u << 20)
MOE_API moe_status moe_route_noalloc(const moe_config* cfg, const void* X, const float* Wg,
                                     const float* logit_bias, const float* sel_bias,
                                     moe_route_out* out, moe_stream_t stream);

/* moe_expert_ffn + moe_combine with the combine fused into the down
 * projection's epilogue ([EC-math] "The math": out = scatter_add(G * Y)):
 * each row's output is scaled by its gate and added, in fp32, into acc
 * [n,d] at its token (vector reductions, so the summation order is not
 * fixed), and acc is then rounded into out [n,d]. Y_perm is never written,
 * and Y rows are not rounded to bf16 before the gate multiplies them. X_perm
 * may be NULL: the first projection then gathers its rows from X as in
 * moe_expert_ffn_gathered. acc (16-byte aligned) and row_gate [rows] are
 * caller-owned scratch. bf16 configs only. Measured slower than the separate
 * combine on every workload; the layer does not use it. */
MOE_API moe_status moe_expert_ffn_combined(const moe_config* cfg, const void* X,
                                           const void* X_perm, const moe_route_out* route,
                                           const void* W1, const void* W3, const void* W2,
                                           const void* sW1, const void* sW3, const void* sW2,
                                           void* H, float* acc, float* row_gate, void* out,
                                           void* ws, size_t ws_bytes, moe_stream_t stream);

/* ---- backward pass of moe_layer_forward -------------------------------
 * The gradient, by the chain rule, of
 *     loss = <dout, out> + L_lb + L_z
 * where out is moe_layer_forward's output and L_lb, L_z are the aux losses
 * of [TC-vs-EC] "What each direction guarantees" (token choice; coefficients
 * lb_coef, z_coef as in aux[]). Selections, capacity drops and counts are
 * piecewise constant and carry no gradient; the selection bias and the logit
 * bias get none. Steps, in order ([EC-math] "The math": out =
 * scatter_add(G * Expert(X_in))):
 *   combine:  dY[r] = g dout[t] for each kept row r of token t with gate g
 *             (stored bf16); dgate = <dout[t], Y_perm[r]> (fp32);
 *   weights:  raw: dS = dgate; normalised w = s / sum s over the K selected:
 *             dS_k = (dw_k - sum_j w_j dw_j) / sum_j s_j; expert choice:
 *             dS[t, e] = dgate; plus lb_coef E f_e / n (f_e = load_e / (n K));
 *   scores:   softmax dL = S (dS - <S, dS>); sigmoid dL = dS s (1 - s);
 *             sqrt(softplus) dL = dS sigmoid(l) / (2 s); plus the z-loss
 *             term z_coef 2 lse_t / n softmax(l_t);
 *   experts:  U = X W1^T, V = X W3^T recomputed and stored bf16, H as the
 *             forward computes it; dH = dY W2; dU = dH act'(U) (SwiGLU:
 *             dU = dH V silu'(U), dV = dH silu(U)), stored bf16;
 *             dX_perm = dU W1 + dV W3 (bf16); dW1 = dU^T X_perm,
 *             dW3 = dV^T X_perm, dW2 = dY^T H over each expert's kept rows
 *             (fp32 accumulation, stored bf16); shared experts take dout
 *             itself as dY over all n tokens;
 *   router:   dWg = X^T dL (fp32); dX = dL Wg^T + the sum of dX_perm over
 *             the token's kept rows and shared rows (fp32, stored bf16).
 * bf16 configs run the grouped GEMMs on the tcgen05 tensor cores (d and h
 * multiples of 64); fp32 configs run them on FFMA and store every value in
 * fp32 (no rounding to bf16 anywhere). */

/* Backward workspace bytes and the kernels moe_layer_backward enqueues
 * (moe_layer_backward_train enqueues one fewer for bf16 configs: it skips
 * the recompute of the up projection). */
MOE_API moe_status moe_backward_workspace_size(const moe_config* cfg, size_t* bytes,
                                               int* launches);

/* Kernels the training pair enqueues for `cfg`: forward =
 * moe_layer_forward_train's (moe_layer_forward's plus, for bf16, the clear of
 * the dispatched rows' padding), backward = moe_layer_backward_train's.
 * Either output may be NULL. No counterpart on the pages. */
MOE_API moe_status moe_train_launch_counts(const moe_config* cfg, int* forward, int* backward);

/* Arguments: the forward's inputs X, Wg, W1, W3, W2 (sW* for shared
 * experts, else NULL); `route`, the routing moe_layer_forward wrote (with
 * logits, and lse, filled when the score is sqrt(softplus) or token choice
 * has z_coef != 0); fwd_ws, the workspace of that moe_layer_forward call,
 * untouched since: its dispatched rows and expert outputs are read, and the
 * padding rows of its dispatched rows are overwritten with zeros; dout [n,d]
 * (the config's dtype). Outputs (device, caller-owned, every element
 * written): dX [n,d] of the config's dtype, dWg [d,E] fp32, dW1, dW3 [E,h,d]
 * and dW2 [E,d,h] of the config's dtype (dW3 only for SwiGLU), dsW1, dsW3,
 * dsW2 likewise for shared experts; dL [n,E] fp32, the
 * logits' gradient, may be NULL. ws: moe_backward_workspace_size bytes,
 * 256-byte aligned, error word zeroed once by moe_workspace_init; bounded
 * waits report through it (moe_read_error). X, dout, dX, the weights and
 * their gradients must be 16-byte aligned. */
MOE_API moe_status moe_layer_backward(const moe_config* cfg, const void* X, const float* Wg,
                                      const void* W1, const void* W3, const void* W2,
                                      const void* sW1, const void* sW3, const void* sW2,
                                      const moe_route_out* route, void* fwd_ws,
                                      size_t fwd_ws_bytes, const void* dout, void* dX,
                                      float* dWg, void* dW1, void* dW3, void* dW2,
                                      void* dsW1, void* dsW3, void* dsW2, float* dL,
                                      void* ws, size_t ws_bytes, moe_stream_t stream);

/* The training pair. moe_layer_forward_train is moe_layer_forward that also
 * keeps, in `bwd_ws` (moe_backward_workspace_size bytes), what the backward
 * would otherwise recompute: the up projection's pre-activations U = X W1^T
 * (and V = X W3^T for SwiGLU) and H, all bf16, with the dispatched rows'
 * padding rows cleared first so that they are zero there. out, route and
 * ws are as for moe_layer_forward (H is kept in bwd_ws instead of ws).
 * moe_layer_backward_train takes moe_layer_backward's arguments, with ws the
 * same bwd_ws, and skips the recompute. fp32 configs keep nothing: the pair
 * then behaves as moe_layer_forward / moe_layer_backward. */
MOE_API moe_status moe_layer_forward_train(const moe_config* cfg, const void* X,
                                           const float* Wg, const float* logit_bias,
                                           const float* sel_bias, const void* W1,
                                           const void* W3, const void* W2, const void* sW1,
                                           const void* sW3, const void* sW2, void* out,
                                           moe_route_out* route, void* ws, size_t ws_bytes,
                                           void* bwd_ws, size_t bwd_ws_bytes,
                                           moe_stream_t stream);
MOE_API moe_status moe_layer_backward_train(const moe_config* cfg, const void* X,
                                            const float* Wg, const void* W1, const void* W3,
                                            const void* W2, const void* sW1, const void* sW3,
                                            const void* sW2, const moe_route_out* route,
                                            void* fwd_ws, size_t fwd_ws_bytes, const void* dout,
                                            void* dX, float* dWg, void* dW1, void* dW3,
                                            void* dW2, void* dsW1, void* dsW3, void* dsW2,
                                            float* dL, void* ws, size_t ws_bytes,
                                            moe_stream_t stream);

/* Failure-path test hooks (no counterpart on the pages). Arms one fault,
 * taken by the next grouped-FFN up projection that can honour it, in any
 * thread of the process; MOE_FAULT_NONE disarms.
 *   MOE_FAULT_GEMM_NO_LOADS: the next up projection that runs on the
 *     single-CTA kernel (bf16, fewer than 256 rows per expert on average)
 *     issues no operand loads; its MMA warp's bounded wait runs out after
 *     the 2 s limit, every warp of the kernel returns, and the workspace's
 *     error word then reads MOE_ERR_TIMEOUT. That call's outputs are
 *     undefined; the GPU context stays usable.
 *   MOE_FAULT_LAUNCH: the next up projection is not launched and the call
 *     returns MOE_ERR_CUDA, as for a failed launch (the kernels enqueued
 *     before it stay enqueued).
 * Nothing here faults the device. Returns MOE_ERR_INVALID_ARG for an
 * unknown fault. */
typedef enum {
  MOE_FAULT_NONE = 0,
  MOE_FAULT_GEMM_NO_LOADS = 1,
  MOE_FAULT_LAUNCH = 2
} moe_fault;
MOE_API moe_status moe_debug_inject_fault(moe_fault fault);

/* Zeroes the error word at the start of `ws` (enqueued on `stream`). */
MOE_API moe_status moe_workspace_init(void* ws, moe_stream_t stream);

/* Synchronises `stream`, then reads and clears the error word at the start
 * of `ws` and, when that is clear, the current device's word for moe_dispatch
 * calls (which take no workspace): MOE_OK, MOE_ERR_TIMEOUT (a bounded wait
 * gave up) or MOE_ERR_CUDA. With ws == NULL it reads and clears instead the
 * error word of moe_route_noalloc's scratch array on the current device (a
 * clear word if that device has made no such call), then the moe_dispatch
 * word. If detail != NULL it receives the raw device code (0 = none). */
MOE_API moe_status moe_read_error(void* ws, moe_stream_t stream, int* detail);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H */
