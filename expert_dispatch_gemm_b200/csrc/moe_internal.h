// Internal host-side declarations shared by the libmoe translation units.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

constexpr int kTokBlock = 256;    // tokens per block in the capacity scan
constexpr int kRowAlign = MOE_ROW_ALIGN;

inline int ceil_div(long long a, long long b) { return (int)((a + b - 1) / b); }
inline long long round_up(long long a, long long b) { return (a + b - 1) / b * b; }

// Router tile: padded expert count; rows per CTA of the pass that writes the
// per-CTA column sums (>= 16); k slices (1, or a split-k first pass plus a
// reduce pass over [ksplit][n][E] partial logits).
int router_tile_et(int E);
int router_block_rows(int E, int n, int d, bool x_bf16);
int router_ksplit(int E, int n, int d, bool x_bf16);
constexpr int kRouterMinBlockRows = 4;  // also the rows per CTA of the split-k reduce

struct Derived {
  int k;            // EC tokens per expert / TC experts per token
  int cap;          // TC rows per expert, -1 dropless (EC: k)
  int slots;        // columns of tok_row
  int kpad;         // EC: k rounded up to the row alignment
  long long rows_routed;  // upper bound on offsets[E]
  long long rows;         // rows of X_perm / H / Y_perm
  long long shared_base;  // first shared-expert row
  int n_pad;              // roundup(n, 128)
  int router_blocks;      // CTAs of the router / score-selection pass
  int tok_blocks;         // token blocks of the capacity scan
};

// Workspace regions (byte offsets from the workspace base).
struct WsLayout {
  size_t err;        // 256 B error words
  size_t colsum;     // [router_blocks, E] f32 partial column sums of S
  size_t lse2;       // [router_blocks] f64 partial sums of lse^2
  size_t blk_hist;   // [tok_blocks, E] i32
  size_t blk_base;   // [tok_blocks, E] i32
  size_t ec_row;     // [n, E] i32 (expert choice, dense)
  size_t ec_gate;    // [n, E] f32 (expert choice, dense)
  size_t rpart;      // [ksplit, n, E] f32 split-k router partials (small batches)
  size_t route_end;
  size_t xperm, hbuf, yperm;  // layer only
  size_t layer_end;
};

// 2-D bf16 row-major [rows, cols] TMA map, box 64 columns x box_rows rows,
// 128-byte swizzle; out-of-range elements load as zero. False when the shape
// or alignment cannot be encoded.
bool make_bf16_sw128_map(CUtensorMap* m, const void* ptr, long long rows, long long cols,
                         int box_rows);

moe_status derive(const moe_config* c, Derived* d);
WsLayout ws_layout(const moe_config* c, const Derived& d);

// ----- launchers (return the launch error; nothing is synchronised) -----
struct RouterArgs {
  const void* X;
  const float* Wg;
  const float* logit_bias;
  const float* sel_bias;
  int n, d, E, x_bf16, score;
  // token choice selection (fused), or K = 0 for expert choice
  int K, n_groups, topk_groups, group_topn, weights;
  int32_t* idx;
  float* gate;
  float* logits;     // optional
  float* scores;
  float* lse;        // optional
  float* colsum;     // [blocks, E]
  double* lse2;      // [blocks]
  float* partial;    // [ksplit, n, E] split-k partial logits (workspace)
  int ksplit, chunks_per_split;  // set by launch_router
};
cudaError_t launch_router(const RouterArgs& a, cudaStream_t s);

struct SelectTcArgs {
  const float* S;
  const float* sel_bias;
  int n, E, K, n_groups, topk_groups, group_topn, weights;
  int32_t* idx;
  float* gate;
  float* scores_copy;  // optional copy of S
  float* colsum;       // [blocks, E]
};
cudaError_t launch_select_tc(const SelectTcArgs& a, cudaStream_t s);
int select_tc_block_rows();

struct SelectEcArgs {
  const float* S;
  int n, E, k, kpad;
  int32_t* idx;
  float* gate;
  int32_t* ec_row;    // [n, E] dense: dispatched row or -1
  float* ec_gate;     // [n, E]
  int32_t* row_token; // [E * kpad]
  int32_t* load;
  int32_t* counts;
  int32_t* offsets;
  int* err;
  // block 0 also resets the accumulators the finish kernel adds into
  int32_t* hist;        // optional [E+1]
  float* aux;
  const double* lse2;   // [lse_blocks] or NULL
  int lse_blocks;
  float z_coef;
};
cudaError_t launch_select_ec(const SelectEcArgs& a, cudaStream_t s);

struct EcFinishArgs {
  const int32_t* ec_row;
  const float* ec_gate;
  int n, E;
  int32_t* tok_row;
  float* tok_gate;
  int32_t* hist;        // optional [E+1]
  float* aux;
  const double* lse2;   // [lse_blocks] or NULL
  int lse_blocks;
  float z_coef;
};
cudaError_t launch_ec_finish(const EcFinishArgs& a, cudaStream_t s);

struct TcAssignArgs {
  const int32_t* idx;
  const float* gate;
  int n, E, K, cap, tok_blocks;
  int32_t* blk_hist;
  int32_t* blk_base;
  int32_t* load;
  int32_t* counts;
  int32_t* offsets;
  int32_t* row_token;
  int32_t* tok_row;
  float* tok_gate;
  uint8_t* drop;
  float* aux;
  const float* colsum;
  int colsum_blocks;
  const double* lse2;   // or NULL
  int lse_blocks;
  float lb_coef, z_coef;
  int* err;             // device error word
};
cudaError_t launch_tc_assign(const TcAssignArgs& a, cudaStream_t s);

struct GatherArgs {
  const void* X;
  const int32_t* tok_row;    // [n, slots]: the token's dispatched rows, then -1
  const int32_t* row_token;  // [rows]: source token of each row, -1 padding
  const int32_t* offsets;    // [E+1]: offsets[E] = rows in use
  int E, n, slots;
  int fanout;                // expected rows per token (K, or EC capacity factor)
  int row_bytes;           // d * element size (a multiple of 16)
  long long max_rows;
  void* X_perm;
  int* err;                // device error word, or NULL for the module's own
};
cudaError_t launch_gather(const GatherArgs& a, cudaStream_t s);
// Reads and clears the error word of dispatch calls made without a workspace.
int take_dispatch_error();
// Reads and clears the error word of moe_route_noalloc's static scratch on the
// current device (0 when that device has made no such call).
int take_noalloc_error();
// Arms a one-shot failure-path test fault (moe_debug_inject_fault).
moe_status set_fault(int fault);
// moe_route's host-side checks of the config, X, W_g and the route outputs
// (those that need no workspace).
moe_status route_call_check(const moe_config* c, const void* X, const float* Wg,
                            const moe_route_out* o);

struct CombineArgs {
  const void* Y;
  const int32_t* tok_row;
  const float* tok_gate;
  int n, d, slots, bf16, n_shared, n_pad;
  long long shared_base;
  long long max_rows;   // routed rows bound; larger slot entries are ignored
  void* out;
  int* err;             // device error word, or NULL for the module's own
};
cudaError_t launch_combine(const CombineArgs& a, cudaStream_t s);

struct FfnArgs {
  const void* X;        // [n, d] (shared experts read it)
  const void* X_perm;   // [rows, d], or NULL: routed rows are read from X via row_token
  const int32_t* row_token;  // [rows] (needed when X_perm is NULL)
  const int32_t* offsets;
  const int32_t* counts;  // [E] real rows of each segment, or NULL (unknown)
  const void *W1, *W3, *W2, *sW1, *sW3, *sW2;
  void* H;              // [rows, h]
  void* Y;              // [rows, d]
  int n, d, h, E, act, n_shared, n_pad;
  long long rows_routed, shared_base, rows;
  int* err;
  bool pair;  // bf16: CTA-pair (cta_group::2) kernel instead of the single-CTA one
  bool skip_down;  // run the up projection only
  // combine fused into the down projection: out32[token] += gate * row
  // (fp32 reductions), row_gate [rows]; Y is then not written
  const float* row_gate;
  float* out32;
  // training: the up projection also stores U (and V) [rows, h] (bf16)
  void* save_u;
  void* save_v;
};
// GEMM kernel choice for a config
bool ffn_uses_pair(const moe_config* c, const Derived& d);
moe_status run_ffn_bf16(const FfnArgs& a, cudaStream_t s);
// the weights-as-M down projection for fine-grained experts (needs the counts)
bool swap_up_supported(const FfnArgs& a);
moe_status run_ffn_up_swap(const FfnArgs& a, cudaStream_t s);
bool swap_down_supported(const FfnArgs& a);
// the backward's dX_perm = dU W1 (+ dV W3) with the weights as the M side
struct SwapDxArgs {
  const void* duv;          // [rows, kcols]: dU, then dV (SwiGLU) in columns h..2h
  long long rows;           // rows of duv and dxp (routed, padding, shared)
  long long rows_routed;
  int kcols, E, h, d, n_shared, n;
  long long shared_base, n_pad;
  const void *W1, *W3, *sW1, *sW3;  // W3 / sW3 NULL without SwiGLU
  const int32_t* offsets;
  const int32_t* counts;
  void* dxp;                // [rows, d]
  int* err;
};
bool swap_dx_supported(const SwapDxArgs& a);
moe_status run_bwd_dx_swap(const SwapDxArgs& a, cudaStream_t s);
moe_status run_ffn_down_swap(const FfnArgs& a, cudaStream_t s);
moe_status run_ffn_f32(const FfnArgs& a, cudaStream_t s);

// ----- backward pass -----
// grouped GEMMs of the expert FFN's backward (gemm_bwd.cu)
enum { BW_SAVE = 0, BW_DACT = 1, BW_DX = 2, BW_WG2 = 3, BW_WG13 = 4 };
struct BwdParams {
  const int32_t* offsets;
  const int32_t* counts;   // [E] rows kept per expert (weight gradients reduce over these)
  int E, n_shared, n;
  int swiglu, act;
  // row modes (SAVE, DACT, DX): 128-row blocks of the dispatched rows
  int K;                   // reduction length, multiple of 64
  int k_split;             // DX: K rows below come from the W1 map, above from W3
  int n_total;             // output columns
  int n_block;             // output columns per tile (SAVE with SwiGLU: 128)
  int nt_tiles;            // column blocks (weight gradients: 256-column blocks)
  int b_rows_per_expert;   // weight rows per expert in the B map
  int shared_blocks;       // 128-row blocks per shared expert
  int max_routed_blocks;   // bound on offsets[E] / 128
  long long a1_row_base, a1_row_stride;  // shared experts' A rows
  long long out_shared_base, n_pad;
  __nv_bfloat16 *out0, *out1, *out2;
  long long ld_out;
  const __nv_bfloat16 *in0, *in1;
  long long ld_in;
  // weight-gradient modes (WG2, WG13): the expert's [m_total, ld_w] output
  int m_total, m_split, mt_tiles, ld_w;
  long long b1_row_base, b1_row_stride;  // shared experts' B rows
  long long w_expert_stride;             // elements between experts' outputs
  __nv_bfloat16 *w_out0, *w_out1, *sw_out0, *sw_out1;  // rows < m_split / >= m_split
  int* err;
};
struct BwdMaps {
  CUtensorMap a0, a1, b0, b0g, b1, b1g;
  CUtensorMap o0, o1, o2, o3;  // weight-gradient outputs (TMA stores), boxes 64 x 32
};
// pair: CTA pairs (cta_group::2, 256-row tiles); weight modes then take
// mt_tiles in 256-row blocks
cudaError_t run_bwd_gemm(int mode, bool pair, const BwdMaps& m, const BwdParams& p,
                         cudaStream_t s);

// fp32 grouped GEMMs of the backward on FFMA (bwd_f32.cu), same modes
struct BwdF32Args {
  const int32_t* offsets;
  const int32_t* counts;
  int E, n_shared, n, n_pad;
  long long rows_routed, shared_base;
  int act, swiglu;
  // row modes: C[rows, N] over K
  int N, K, k_split;
  const float* A;                     // routed A rows, row pitch lda
  long long lda;
  const float* A_sh;                  // shared A rows: A_sh + (a_sh_base + s * a_sh_stride + i) * lda
  long long a_sh_base, a_sh_stride;
  const float *B, *B3, *sB, *sB3;     // weights; SAVE: [.., N, K]; DACT/DX: [.., K, N]
  long long b_expert_stride;
  float *out0, *out1, *out2;
  long long ld_out;
  const float *in0, *in1;
  long long ld_in;
  // weight modes: per expert C[M, N] = sum over its rows k of A(m, k) B(n, k),
  // A(m, k) = WA[(row0 + k) * ld_wa + m], B(n, k) = WB[(row0 + k) * ld_wb + n]
  int M, m_split;
  const float *WA, *WA_sh, *WB, *WB_sh;
  long long ld_wa, ld_wb, wa_sh_base, wa_sh_stride, wb_sh_base, wb_sh_stride;
  float *w_out0, *w_out1, *sw_out0, *sw_out1;
  long long w_expert_stride;
};
cudaError_t run_bwd_f32(int mode, const BwdF32Args& a, cudaStream_t s);

// element-wise and FFMA kernels of the backward (bwd.cu); activations,
// expert outputs and their gradients are bf16 or fp32 (bf16 = 1)
struct CombineBwdArgs {
  int bf16;
  const void* Y_perm;            // [rows, d] the forward's expert outputs
  const void* dout;              // [n, d]
  const int32_t* tok_row;        // [n, slots]
  const float* tok_gate;         // [n, slots]
  const int32_t* idx;            // TC [n, K]
  const uint8_t* drop;           // TC [n, K]
  const int32_t* offsets;        // [E+1]
  const int32_t* load;           // [E]
  const float* scores;           // [n, E]
  const float* logits;           // [n, E] (z-loss, sqrt(softplus)) or NULL
  const float* lse;              // [n] or NULL
  int n, d, E, slots, tc, K, score, weights;
  float lb_coef, z_coef;
  void* dY_perm;                 // [rows, d]: kept rows written
  float* dL;                     // [n, E]
  long long max_rows;            // routed rows bound; larger tok_row entries are skipped
  int* err;                      // device error word
};
cudaError_t launch_combine_backward(const CombineBwdArgs& a, cudaStream_t s);
// zero rows [offsets[e] + counts[e], offsets[e+1]) of two [rows, row_bytes] buffers
cudaError_t launch_pad_zero(const int32_t* offsets, const int32_t* counts, int E, int row_bytes,
                            void* a, void* b, cudaStream_t s);
struct RouterBwdArgs {
  int bf16;
  const void* X;                 // [n, d]
  const float* Wg;               // [d, E]
  float* WgT;                    // [E, d] workspace: W_g transposed
  const float* dL;               // [n, E]
  const void* dX_perm;           // [rows, d]
  const int32_t* tok_row;        // [n, slots]
  int n, d, E, slots, n_shared;
  long long shared_base, n_pad;
  void* dX;                      // [n, d]
  float* dWg;                    // [d, E]
  float* partial;                // [splits, d, E]
  int splits;
  long long max_rows;            // routed rows bound; larger tok_row entries are skipped
  int* err;                      // device error word
};
int router_bwd_splits(int n, int d, int E);
cudaError_t launch_router_backward(const RouterBwdArgs& a, cudaStream_t s);

// the fused combine's bookkeeping: zero out32 [n, d] and write each
// dispatched row's gate; then round out32 into the output
cudaError_t launch_combine_prep(const int32_t* tok_row, const float* tok_gate, int n, int slots,
                                int d, long long max_rows, float* row_gate, float* out32,
                                int* err, cudaStream_t s);
cudaError_t launch_combine_finish(const float* out32, int n, int d, void* out, cudaStream_t s);

cudaError_t launch_bias_update(int n, int E, int K, const int32_t* load, float rate,
                               float* bias, cudaStream_t s);

}  // namespace moe
