// C-ABI entry points of libmoe: host-side validation, derived sizes,
// workspace layout and the launch sequence of each call. Nothing here
// allocates, frees or synchronises (except moe_read_error).
#include <math.h>
#include <string.h>

#include "device_common.cuh"
#include "moe_internal.h"

namespace moe {

static bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

moe_status derive(const moe_config* c, Derived* d) {
  if (!c || !d) return MOE_ERR_INVALID_ARG;
  if (c->n < 1 || c->d < 1 || c->h < 1 || c->E < 1) return MOE_ERR_INVALID_ARG;
  if (c->E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED;
  if (c->dtype != MOE_F32 && c->dtype != MOE_BF16) return MOE_ERR_INVALID_ARG;
  if (c->mode != MOE_EXPERT_CHOICE && c->mode != MOE_TOKEN_CHOICE) return MOE_ERR_INVALID_ARG;
  if (c->score != MOE_SCORE_SOFTMAX && c->score != MOE_SCORE_SIGMOID &&
      c->score != MOE_SCORE_SQRTSOFTPLUS)
    return MOE_ERR_INVALID_ARG;
  if (c->act != MOE_ACT_RELU && c->act != MOE_ACT_GELU && c->act != MOE_ACT_SWIGLU)
    return MOE_ERR_INVALID_ARG;
  if (c->weights != MOE_W_RAW && c->weights != MOE_W_NORMALIZED) return MOE_ERR_INVALID_ARG;
  if (c->n_shared < 0 || c->n_shared > MOE_MAX_SHARED) return MOE_ERR_INVALID_ARG;
  if (c->dtype == MOE_BF16) {
    if (c->d % 64 || c->h % 64) return MOE_ERR_UNSUPPORTED;
  } else {
    if (c->d % 8 || c->h % 8) return MOE_ERR_UNSUPPORTED;
  }
  const int E = c->E, n = c->n;
  d->n_pad = (int)round_up(n, kRowAlign);
  if (c->mode == MOE_EXPERT_CHOICE) {
    int k = c->k;
    if (k == 0) {
      if (!(c->capacity_factor > 0.0f)) return MOE_ERR_INVALID_ARG;
      k = (int)floor((double)n * (double)c->capacity_factor / (double)E + 1e-9);
    }
    if (k < 1 || k > n) return MOE_ERR_INVALID_ARG;
    if (n > MOE_EC_MAX_TOKENS) return MOE_ERR_UNSUPPORTED;
    d->k = k;
    d->cap = k;
    d->slots = E;
    d->kpad = (int)round_up(k, kRowAlign);
    d->rows_routed = (long long)E * d->kpad;
  } else {
    const int K = c->k;
    if (K < 1 || K > E || K > MOE_MAX_TOPK) return MOE_ERR_INVALID_ARG;
    int cap;
    if (c->capacity < 0) {
      cap = -1;
    } else if (c->capacity == 0) {
      if (!(c->capacity_factor > 0.0f)) return MOE_ERR_INVALID_ARG;
      cap = (int)floor((double)n / (double)E * (double)c->capacity_factor + 1e-9);
      if (cap < 1) return MOE_ERR_INVALID_ARG;
    } else {
      cap = c->capacity;
    }
    if (c->n_groups > 1) {
      const int G = c->n_groups;
      if (E % G) return MOE_ERR_INVALID_ARG;
      const int gs = E / G;
      const int et = router_tile_et(E);
      const int V = et >= 32 ? et / 32 : 1;
      if (gs % V || !is_pow2(gs / V) || gs / V > 32) return MOE_ERR_UNSUPPORTED;
      if (c->topk_groups < 1 || c->topk_groups > G) return MOE_ERR_INVALID_ARG;
      if (c->group_topn < 1 || c->group_topn > gs) return MOE_ERR_INVALID_ARG;
      if (K > c->topk_groups * gs) return MOE_ERR_INVALID_ARG;
    }
    d->k = K;
    d->cap = cap;
    d->slots = K;
    d->kpad = 0;
    long long a = (long long)n * K;
    long long bound = round_up(a + (long long)E * (kRowAlign - 1), kRowAlign);
    bound = bound / kRowAlign * kRowAlign;
    if (cap >= 0) {
      long long capb = (long long)E * round_up(cap, kRowAlign);
      if (capb < bound) bound = capb;
    }
    // floor to a multiple of 128 of (a + 127 E) is also a valid bound
    long long fl = (a + (long long)E * (kRowAlign - 1)) / kRowAlign * kRowAlign;
    if (fl < bound) bound = fl;
    if (bound < kRowAlign) bound = kRowAlign;
    d->rows_routed = bound;
  }
  d->shared_base = d->rows_routed;
  d->rows = d->rows_routed + (long long)c->n_shared * d->n_pad;
  if (d->rows > (1LL << 30)) return MOE_ERR_UNSUPPORTED;
  // covers every router tile height and the score-only selection blocks
  d->router_blocks = ceil_div(n, kRouterMinBlockRows);
  d->tok_blocks = ceil_div(n, kTokBlock);
  return MOE_OK;
}

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

WsLayout ws_layout(const moe_config* c, const Derived& d) {
  WsLayout w{};
  size_t off = 0;
  w.err = off;
  off += MOE_WS_ERROR_BYTES;
  w.colsum = off;
  off = align_up(off + (size_t)d.router_blocks * c->E * 4, 256);
  w.lse2 = off;
  off = align_up(off + (size_t)d.router_blocks * 8, 256);
  w.blk_hist = off;
  off = align_up(off + (size_t)d.tok_blocks * c->E * 4, 256);
  w.blk_base = off;
  off = align_up(off + (size_t)d.tok_blocks * c->E * 4, 256);
  w.ec_row = off;
  if (c->mode == MOE_EXPERT_CHOICE) off = align_up(off + (size_t)c->n * c->E * 4, 256);
  w.ec_gate = off;
  if (c->mode == MOE_EXPERT_CHOICE) off = align_up(off + (size_t)c->n * c->E * 4, 256);
  w.rpart = off;
  {
    const int ks = router_ksplit(c->E, c->n, c->d, c->dtype == MOE_BF16);
    if (ks > 1) off = align_up(off + (size_t)ks * c->n * c->E * 4, 256);
  }
  w.route_end = align_up(off, 1024);
  const size_t elt = c->dtype == MOE_BF16 ? 2 : 4;
  off = w.route_end;
  w.xperm = off;
  off = align_up(off + (size_t)d.rows * c->d * elt, 1024);
  w.hbuf = off;
  off = align_up(off + (size_t)d.rows * c->h * elt, 1024);
  w.yperm = off;
  off = align_up(off + (size_t)d.rows * c->d * elt, 1024);
  w.layer_end = off;
  return w;
}

static moe_status check_route_out(const moe_config* c, const moe_route_out* o) {
  if (!o) return MOE_ERR_INVALID_ARG;
  if (!o->idx || !o->gate || !o->load || !o->counts || !o->offsets || !o->row_token ||
      !o->tok_row || !o->tok_gate || !o->scores || !o->aux)
    return MOE_ERR_INVALID_ARG;
  if (c->mode == MOE_TOKEN_CHOICE && !o->drop) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

moe_status route_call_check(const moe_config* c, const void* X, const float* Wg,
                            const moe_route_out* o) {
  Derived d;
  moe_status st = derive(c, &d);
  if (st != MOE_OK) return st;
  if (!X || !Wg) return MOE_ERR_INVALID_ARG;
  return check_route_out(c, o);
}

static moe_status check_ws(void* ws, size_t have, size_t need) {
  if (!ws) return MOE_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) & 255) return MOE_ERR_WORKSPACE;
  if (have < need) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

template <typename T>
static T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

#define MOE_CU(x)                          \
  do {                                     \
    if ((x) != cudaSuccess) return MOE_ERR_CUDA; \
  } while (0)

// selection bookkeeping after the scores (and, for TC, idx/gate) exist
static moe_status finish_route(const moe_config* c, const Derived& dv, const WsLayout& w,
                               moe_route_out* o, void* ws, const float* S, int colsum_blocks,
                               bool have_lse, cudaStream_t s) {
  int* err = at<int>(ws, w.err);
  if (c->mode == MOE_EXPERT_CHOICE) {
    SelectEcArgs a{};
    a.S = S;
    a.n = c->n;
    a.E = c->E;
    a.k = dv.k;
    a.kpad = dv.kpad;
    a.idx = o->idx;
    a.gate = o->gate;
    a.ec_row = at<int32_t>(ws, w.ec_row);
    a.ec_gate = at<float>(ws, w.ec_gate);
    a.row_token = o->row_token;
    a.load = o->load;
    a.counts = o->counts;
    a.offsets = o->offsets;
    a.err = err;
    a.hist = o->ec_hist;
    a.aux = o->aux;
    a.lse2 = have_lse ? at<double>(ws, w.lse2) : nullptr;
    a.lse_blocks = colsum_blocks;
    a.z_coef = c->z_coef;
    MOE_CU(launch_select_ec(a, s));
    EcFinishArgs f{};
    f.ec_row = a.ec_row;
    f.ec_gate = a.ec_gate;
    f.n = c->n;
    f.E = c->E;
    f.tok_row = o->tok_row;
    f.tok_gate = o->tok_gate;
    f.hist = o->ec_hist;
    f.aux = o->aux;
    f.lse2 = have_lse ? at<double>(ws, w.lse2) : nullptr;
    f.lse_blocks = colsum_blocks;
    f.z_coef = c->z_coef;
    MOE_CU(launch_ec_finish(f, s));
    return MOE_OK;
  }
  TcAssignArgs a{};
  a.idx = o->idx;
  a.gate = o->gate;
  a.n = c->n;
  a.E = c->E;
  a.K = dv.k;
  a.cap = dv.cap;
  a.tok_blocks = dv.tok_blocks;
  a.blk_hist = at<int32_t>(ws, w.blk_hist);
  a.blk_base = at<int32_t>(ws, w.blk_base);
  a.load = o->load;
  a.counts = o->counts;
  a.offsets = o->offsets;
  a.row_token = o->row_token;
  a.tok_row = o->tok_row;
  a.tok_gate = o->tok_gate;
  a.drop = o->drop;
  a.aux = o->aux;
  a.colsum = at<float>(ws, w.colsum);
  a.colsum_blocks = colsum_blocks;
  a.lse2 = have_lse ? at<double>(ws, w.lse2) : nullptr;
  a.lse_blocks = colsum_blocks;
  a.lb_coef = c->lb_coef;
  a.z_coef = c->z_coef;
  a.err = err;
  MOE_CU(launch_tc_assign(a, s));
  return MOE_OK;
}

static moe_status route_impl(const moe_config* c, const Derived& dv, const WsLayout& w,
                             const void* X, const float* Wg, const float* logit_bias,
                             const float* sel_bias, moe_route_out* o, void* ws,
                             cudaStream_t s) {
  RouterArgs r{};
  r.X = X;
  r.Wg = Wg;
  r.logit_bias = logit_bias;
  r.sel_bias = c->mode == MOE_TOKEN_CHOICE ? sel_bias : nullptr;
  r.n = c->n;
  r.d = c->d;
  r.E = c->E;
  r.x_bf16 = c->dtype == MOE_BF16;
  r.score = c->score;
  r.K = c->mode == MOE_TOKEN_CHOICE ? dv.k : 0;
  r.n_groups = c->n_groups > 1 ? c->n_groups : 1;
  r.topk_groups = c->topk_groups;
  r.group_topn = c->group_topn;
  r.weights = c->weights;
  r.idx = o->idx;
  r.gate = o->gate;
  r.logits = o->logits;
  r.scores = o->scores;
  r.lse = o->lse;
  r.colsum = at<float>(ws, w.colsum);
  r.lse2 = at<double>(ws, w.lse2);
  r.partial = at<float>(ws, w.rpart);
  MOE_CU(launch_router(r, s));
  return finish_route(
      c, dv, w, o, ws, o->scores,
      ceil_div(c->n, router_block_rows(c->E, c->n, c->d, c->dtype == MOE_BF16)), true, s);
}

// X_perm == NULL: the routed rows are read from X through row_token (the
// dispatch gather fused into the first projection's A loads)
// rows per expert on average (token choice: min(nK/E, capacity); expert
// choice: the padded quota)
static long long avg_expert_rows(const moe_config* c, const Derived& dv) {
  if (c->mode != MOE_TOKEN_CHOICE) return dv.kpad;
  long long avg = ((long long)c->n * dv.k + c->E - 1) / c->E;
  if (dv.cap > 0 && avg > dv.cap) avg = dv.cap;
  return avg;
}

// CTA pairs compute two 128-row blocks of one expert per tile: worth it when
// experts own at least two blocks on average. With fewer rows per expert
// (small batches, decoding) half of a pair's MMA work would be padding, and
// the 128-row tiles of the single-CTA kernel waste half as much.
bool ffn_uses_pair(const moe_config* c, const Derived& dv) {
  return c->dtype == MOE_BF16 && avg_expert_rows(c, dv) >= 2 * kRowAlign;
}

// Fine-grained token choice (128 to 512 rows per expert on average): the
// weights-as-M projections compute each expert's exact token count (16-row
// granularity) where the 128-row tiles would round ~256 rows up to 384 or
// 512. They need the counts, which the caller passes. The SwiGLU up
// projection takes W1 and W3 as two A operands into two accumulators; other
// activations, the fused gather and the training forward's kept U and V
// keep the up projection on the token-side kernels.
static bool ffn_uses_swap(const moe_config* c, const Derived& dv) {
  if (c->dtype != MOE_BF16 || c->mode != MOE_TOKEN_CHOICE) return false;
  const long long avg = avg_expert_rows(c, dv);
  return avg >= kRowAlign && avg <= 4 * kRowAlign;
}

// row_gate / out32: the combine fused into the down projection (then Y is
// not written and may be NULL)
static moe_status ffn_impl(const moe_config* c, const Derived& dv, const void* X,
                           const void* X_perm, const int32_t* row_token, const int32_t* offsets,
                           const int32_t* counts, const void* W1, const void* W3,
                           const void* W2, const void* sW1,
                           const void* sW3, const void* sW2, void* H, void* Y, int* err,
                           cudaStream_t s, const float* row_gate = nullptr,
                           float* out32 = nullptr, void* save_u = nullptr,
                           void* save_v = nullptr) {
  if (!offsets || !W1 || !W2 || !H || (!Y && !out32)) return MOE_ERR_INVALID_ARG;
  if (!X_perm && (!X || !row_token)) return MOE_ERR_INVALID_ARG;
  if (c->act == MOE_ACT_SWIGLU && !W3) return MOE_ERR_INVALID_ARG;
  if (c->n_shared > 0) {
    if (!X || !sW1 || !sW2) return MOE_ERR_INVALID_ARG;
    if (c->act == MOE_ACT_SWIGLU && !sW3) return MOE_ERR_INVALID_ARG;
  }
  FfnArgs f{};
  f.X = X;
  f.X_perm = X_perm;
  f.row_token = row_token;
  f.offsets = offsets;
  f.counts = counts;
  f.W1 = W1;
  f.W3 = W3;
  f.W2 = W2;
  f.sW1 = sW1;
  f.sW3 = sW3;
  f.sW2 = sW2;
  f.H = H;
  f.Y = Y;
  f.n = c->n;
  f.d = c->d;
  f.h = c->h;
  f.E = c->E;
  f.act = c->act;
  f.n_shared = c->n_shared;
  f.n_pad = dv.n_pad;
  f.rows_routed = dv.rows_routed;
  f.shared_base = dv.shared_base;
  f.rows = dv.rows;
  f.err = err;
  f.pair = ffn_uses_pair(c, dv);
  f.row_gate = row_gate;
  f.out32 = out32;
  f.save_u = save_u;
  f.save_v = save_v;
  if (c->dtype != MOE_BF16) return out32 ? MOE_ERR_UNSUPPORTED : run_ffn_f32(f, s);
  if (!out32 && ffn_uses_swap(c, dv) && swap_down_supported(f)) {
    moe_status st;
    if (swap_up_supported(f)) {
      st = run_ffn_up_swap(f, s);
    } else {
      f.skip_down = true;
      st = run_ffn_bf16(f, s);
    }
    if (st != MOE_OK) return st;
    return run_ffn_down_swap(f, s);
  }
  return run_ffn_bf16(f, s);
}

// err: the workspace error word, or NULL (standalone moe_dispatch)
static moe_status dispatch_impl(const moe_config* c, const Derived& dv, const void* X,
                                const moe_route_out* o, void* X_perm, int* err,
                                cudaStream_t s) {
  if ((reinterpret_cast<uintptr_t>(X) | reinterpret_cast<uintptr_t>(X_perm)) & 15)
    return MOE_ERR_INVALID_ARG;
  GatherArgs g{};
  g.X = X;
  g.tok_row = o->tok_row;
  g.row_token = o->row_token;
  g.offsets = o->offsets;
  g.E = c->E;
  g.n = c->n;
  g.fanout = c->mode == MOE_TOKEN_CHOICE
                 ? dv.k
                 : (int)(((long long)dv.k * c->E + c->n - 1) / c->n);
  g.slots = dv.slots;
  g.row_bytes = c->d * (c->dtype == MOE_BF16 ? 2 : 4);
  g.max_rows = dv.rows_routed;
  g.X_perm = X_perm;
  g.err = err;
  MOE_CU(launch_gather(g, s));
  return MOE_OK;
}

// err: the workspace error word, or NULL (standalone moe_combine)
static moe_status combine_impl(const moe_config* c, const Derived& dv, const void* Y,
                               const moe_route_out* o, void* out, cudaStream_t s,
                               int* err = nullptr) {
  CombineArgs a{};
  a.Y = Y;
  a.tok_row = o->tok_row;
  a.tok_gate = o->tok_gate;
  a.n = c->n;
  a.d = c->d;
  a.slots = dv.slots;
  a.bf16 = c->dtype == MOE_BF16;
  a.n_shared = c->n_shared;
  a.n_pad = dv.n_pad;
  a.shared_base = dv.shared_base;
  a.max_rows = dv.rows_routed;
  a.out = out;
  a.err = err;
  MOE_CU(launch_combine(a, s));
  return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" {

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape or option";
    case MOE_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_TIMEOUT: return "a bounded device wait gave up";
  }
  return "unknown status";
}

moe_status moe_validate(const moe_config* cfg) {
  Derived d;
  return derive(cfg, &d);
}

moe_status moe_sizes(const moe_config* cfg, int* k_eff, int* capacity_eff, int* slots,
                     int* rows, int* shared_row_base) {
  Derived d;
  moe_status st = derive(cfg, &d);
  if (st != MOE_OK) return st;
  if (k_eff) *k_eff = d.k;
  if (capacity_eff) *capacity_eff = cfg->mode == MOE_TOKEN_CHOICE ? d.cap : d.k;
  if (slots) *slots = d.slots;
  if (rows) *rows = (int)d.rows;
  if (shared_row_base) *shared_row_base = (int)d.shared_base;
  return MOE_OK;
}

moe_status moe_launch_counts(const moe_config* cfg, int* route, int* dispatch, int* ffn,
                             int* combine) {
  Derived d;
  moe_status st = derive(cfg, &d);
  if (st != MOE_OK) return st;
  const int split = router_ksplit(cfg->E, cfg->n, cfg->d, cfg->dtype == MOE_BF16) > 1;
  if (route) *route = 1 + split + (cfg->mode == MOE_EXPERT_CHOICE ? 2 : 3);
  if (dispatch) *dispatch = 1;
  if (ffn) *ffn = 2;
  if (combine) *combine = 1;
  return MOE_OK;
}

moe_status moe_workspace_size(const moe_config* cfg, size_t* route_bytes,
                              size_t* layer_bytes) {
  Derived d;
  moe_status st = derive(cfg, &d);
  if (st != MOE_OK) return st;
  const WsLayout w = ws_layout(cfg, d);
  if (route_bytes) *route_bytes = w.route_end;
  if (layer_bytes) *layer_bytes = w.layer_end;
  return MOE_OK;
}

moe_status moe_route(const moe_config* cfg, const void* X, const float* Wg,
                     const float* logit_bias, const float* sel_bias, moe_route_out* out,
                     void* ws, size_t ws_bytes, moe_stream_t stream) {
  Derived d;
  moe_status st = derive(cfg, &d);
  if (st != MOE_OK) return st;
  if (!X || !Wg) return MOE_ERR_INVALID_ARG;
  if ((st = check_route_out(cfg, out)) != MOE_OK) return st;
  const WsLayout w = ws_layout(cfg, d);
  if ((st = check_ws(ws, ws_bytes, w.route_end)) != MOE_OK) return st;
  return route_impl(cfg, d, w, X, Wg, logit_bias, sel_bias, out, ws, (cudaStream_t)stream);
}

moe_status moe_route_from_scores(const moe_config* cfg, const float* S, const float* sel_bias,
                                 moe_route_out* out, void* ws, size_t ws_bytes,
                                 moe_stream_t stream) {
  Derived d;
  moe_status st = derive(cfg, &d);
  if (st != MOE_OK) return st;
  if (!S) return MOE_ERR_INVALID_ARG;
  if ((st = check_route_out(cfg, out)) != MOE_OK) return st;
  const WsLayout w = ws_layout(cfg, d);
  if ((st = check_ws(ws, ws_bytes, w.route_end)) != MOE_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  if (cfg->mode == MOE_TOKEN_CHOICE) {
    SelectTcArgs a{};
    a.S = S;
    a.sel_bias = sel_bias;
    a.n = cfg->n;
    a.E = cfg->E;
    a.K = d.k;
    a.n_groups = cfg->n_groups > 1 ? cfg->n_groups : 1;
    a.topk_groups = cfg->topk_groups;
    a.group_topn = cfg->group_topn;
    a.weights = cfg->weights;
    a.idx = out->idx;
    a.gate = out->gate;
    a.scores_copy = out->scores != S ? out->scores : nullptr;
    a.colsum = at<float>(ws, w.colsum);
    MOE_CU(launch_select_tc(a, s));
    return finish_route(cfg, d, w, out, ws, S, ceil_div(cfg->n, select_tc_block_rows()), false,
                        s);
  }
  if (out->scores != S)
    MOE_CU(cudaMemcpyAsync(out->scores, S, (size_t)cfg->n * cfg->E * sizeof(float),
                           cudaMemcpyDeviceToDevice, s));
  return finish_route(cfg, d, w, out, ws, S, 0, false, s);
}

moe_status moe_dispatch(const moe_config* cfg, const void* X, const moe_route_out* route,
                        void* X_perm, moe_stream_t stream) {
  Derived d;
  moe_status st = derive(cfg, &d);
  if (st != MOE_OK) return st;
  if (!X || !X_perm || !route || !route->tok_row || !route->row_token || !route->offsets)
    return MOE_ERR_INVALID_ARG;
  return dispatch_impl(cfg, d, X, route, X_perm, nullptr, (cudaStream_t)stream);
}

moe_status moe_expert_ffn(const moe_config* cfg, const void* X, const void* X_perm,
                          const int32_t* offsets, const int32_t* counts, const void* W1,
                          const void* W3, const void* W2, const void* sW1, const void* sW3,
                          const void* sW2, void* H, void* Y_perm, void* ws, size_t ws_bytes,
                          moe_stream_t stream) {
  Derived d;
  moe_status st = derive(cfg, &d);
  if (st != MOE_OK) return st;
  if ((st = check_ws(ws, ws_bytes, MOE_WS_ERROR_BYTES)) != MOE_OK) return st;
  if (!X_perm) return MOE_ERR_INVALID_ARG;
  return ffn_impl(cfg, d, X, X_perm, nullptr, offsets, counts, W1, W3, W2, sW1, sW3, sW2, H,
                  Y_perm, at<int>(ws, 0), (cudaStream_t)stream);
}

moe_status moe_combine(const moe_config* cfg, const void* Y_perm, const moe_route_out* route,
                       void* out, moe_stream_t stream) {
  Derived d;
  moe_status st = derive(cfg, &d);
  if (st != MOE_OK) return st;
  if (!Y_perm || !out || !route || !route->tok_row || !route->tok_gate)
    return MOE_ERR_INVALID_ARG;
  return combine_impl(cfg, d, Y_perm, route, out, (cudaStream_t)stream);
}

// the layer's host-side checks: on a non-OK status nothing may be enqueued
static moe_status layer_forward_check(const moe_config* cfg, Derived* d, WsLayout* w,
                                      const void* X, const float* Wg, const void* out,
                                      const void* W1, const void* W2,
                                      const moe_route_out* route, void* ws, size_t ws_bytes) {
  moe_status st = derive(cfg, d);
  if (st != MOE_OK) return st;
  if (!X || !Wg || !out || !W1 || !W2) return MOE_ERR_INVALID_ARG;
  if ((st = check_route_out(cfg, route)) != MOE_OK) return st;
  *w = ws_layout(cfg, *d);
  return check_ws(ws, ws_bytes, w->layer_end);
}

static moe_status layer_forward_impl(const moe_config* cfg, const Derived& d, const WsLayout& w,
                                     const void* X, const float* Wg, const float* logit_bias,
                                     const float* sel_bias, const void* W1, const void* W3,
                                     const void* W2, const void* sW1, const void* sW3,
                                     const void* sW2, void* out, moe_route_out* route, void* ws,
                                     cudaStream_t s) {
  moe_status st;
  void* xp = at<void>(ws, w.xperm);
  void* hb = at<void>(ws, w.hbuf);
  void* yp = at<void>(ws, w.yperm);
  if ((st = route_impl(cfg, d, w, X, Wg, logit_bias, sel_bias, route, ws, s)) != MOE_OK)
    return st;
  // the gather stays a separate pass: fused into the GEMM's A loads it costs
  // 32 four-row TMA gathers per 64-deep k-block, which the TMA unit issues
  // far slower than the two box loads the unfused GEMM needs
  if ((st = dispatch_impl(cfg, d, X, route, xp, at<int>(ws, w.err), s)) != MOE_OK) return st;
  if ((st = ffn_impl(cfg, d, X, xp, nullptr, route->offsets, route->counts, W1, W3, W2, sW1,
                     sW3, sW2, hb, yp,
                     at<int>(ws, w.err), s)) != MOE_OK)
    return st;
  return combine_impl(cfg, d, yp, route, out, s, at<int>(ws, w.err));
}

moe_status moe_layer_forward(const moe_config* cfg, const void* X, const float* Wg,
                             const float* logit_bias, const float* sel_bias, const void* W1,
                             const void* W3, const void* W2, const void* sW1, const void* sW3,
                             const void* sW2, void* out, moe_route_out* route, void* ws,
                             size_t ws_bytes, moe_stream_t stream) {
  Derived d;
  WsLayout w;
  moe_status st = layer_forward_check(cfg, &d, &w, X, Wg, out, W1, W2, route, ws, ws_bytes);
  if (st != MOE_OK) return st;
  return layer_forward_impl(cfg, d, w, X, Wg, logit_bias, sel_bias, W1, W3, W2, sW1, sW3, sW2,
                            out, route, ws, (cudaStream_t)stream);
}

moe_status moe_layer_forward_host(const moe_config* cfg, const void* X_host, const float* Wg,
                                  const float* logit_bias, const float* sel_bias,
                                  const void* W1, const void* W3, const void* W2,
                                  const void* sW1, const void* sW3, const void* sW2,
                                  void* out_host, void* X_dev, void* out_dev,
                                  moe_route_out* route, void* ws, size_t ws_bytes,
                                  moe_stream_t stream) {
  Derived d;
  WsLayout w;
  if (!X_host || !out_host) return MOE_ERR_INVALID_ARG;
  moe_status st = layer_forward_check(cfg, &d, &w, X_dev, Wg, out_dev, W1, W2, route, ws,
                                      ws_bytes);
  if (st != MOE_OK) return st;
  const size_t bytes = (size_t)cfg->n * cfg->d * (cfg->dtype == MOE_BF16 ? 2 : 4);
  cudaStream_t s = (cudaStream_t)stream;
  MOE_CU(cudaMemcpyAsync(X_dev, X_host, bytes, cudaMemcpyHostToDevice, s));
  if ((st = layer_forward_impl(cfg, d, w, X_dev, Wg, logit_bias, sel_bias, W1, W3, W2, sW1, sW3,
                               sW2, out_dev, route, ws, s)) != MOE_OK)
    return st;
  MOE_CU(cudaMemcpyAsync(out_host, out_dev, bytes, cudaMemcpyDeviceToHost, s));
  return MOE_OK;
}

moe_status moe_expert_ffn_gathered(const moe_config* cfg, const void* X,
                                   const moe_route_out* route, const void* W1, const void* W3,
                                   const void* W2, const void* sW1, const void* sW3,
                                   const void* sW2, void* H, void* Y_perm, void* ws,
                                   size_t ws_bytes, moe_stream_t stream) {
  Derived d;
  moe_status st = derive(cfg, &d);
  if (st != MOE_OK) return st;
  if (!X || !route || !route->row_token || !route->offsets) return MOE_ERR_INVALID_ARG;
  if ((st = check_ws(ws, ws_bytes, MOE_WS_ERROR_BYTES)) != MOE_OK) return st;
  return ffn_impl(cfg, d, X, nullptr, route->row_token, route->offsets, nullptr, W1, W3, W2,
                  sW1, sW3,
                  sW2, H, Y_perm, at<int>(ws, 0), (cudaStream_t)stream);
}

moe_status moe_expert_ffn_combined(const moe_config* cfg, const void* X, const void* X_perm,
                                   const moe_route_out* route, const void* W1, const void* W3,
                                   const void* W2, const void* sW1, const void* sW3,
                                   const void* sW2, void* H, float* acc, float* row_gate,
                                   void* out, void* ws, size_t ws_bytes, moe_stream_t stream) {
  Derived d;
  moe_status st = derive(cfg, &d);
  if (st != MOE_OK) return st;
  if (cfg->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if (!X || !route || !route->row_token || !route->offsets || !route->tok_row ||
      !route->tok_gate || !acc || !row_gate || !out)
    return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(acc) | reinterpret_cast<uintptr_t>(out)) & 15)
    return MOE_ERR_INVALID_ARG;
  if ((st = check_ws(ws, ws_bytes, MOE_WS_ERROR_BYTES)) != MOE_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  MOE_CU(launch_combine_prep(route->tok_row, route->tok_gate, cfg->n, d.slots, cfg->d,
                             d.rows_routed, row_gate, acc, at<int>(ws, 0), s));
  if ((st = ffn_impl(cfg, d, X, X_perm, route->row_token, route->offsets, nullptr, W1, W3, W2,
                     sW1, sW3, sW2, H, nullptr, at<int>(ws, 0), s, row_gate, acc)) != MOE_OK)
    return st;
  MOE_CU(launch_combine_finish(acc, cfg->n, cfg->d, out, s));
  return MOE_OK;
}

moe_status moe_bias_update(const moe_config* cfg, const int32_t* load, float rate, float* bias,
                           moe_stream_t stream) {
  Derived d;
  moe_status st = derive(cfg, &d);
  if (st != MOE_OK) return st;
  if (cfg->mode != MOE_TOKEN_CHOICE) return MOE_ERR_INVALID_ARG;
  if (!load || !bias) return MOE_ERR_INVALID_ARG;
  MOE_CU(launch_bias_update(cfg->n, cfg->E, d.k, load, rate, bias, (cudaStream_t)stream));
  return MOE_OK;
}

// ---------------------------------------------------------------------------
// backward pass
// ---------------------------------------------------------------------------
struct BwdLayout {
  size_t err, dy, u, v, hh, duv, dxp, dl, wgt, part, end;
  int splits, launches;
};

static BwdLayout bwd_layout(const moe_config* c, const Derived& d) {
  BwdLayout b{};
  const bool swiglu = c->act == MOE_ACT_SWIGLU;
  const size_t elt = c->dtype == MOE_BF16 ? 2 : 4;
  size_t off = 0;
  b.err = off;
  off += MOE_WS_ERROR_BYTES;
  off = align_up(off, 1024);
  b.dy = off;
  off = align_up(off + (size_t)d.rows_routed * c->d * elt, 1024);
  b.u = off;
  off = align_up(off + (size_t)d.rows * c->h * elt, 1024);
  b.v = off;
  if (swiglu) off = align_up(off + (size_t)d.rows * c->h * elt, 1024);
  b.hh = off;
  off = align_up(off + (size_t)d.rows * c->h * elt, 1024);
  b.duv = off;
  off = align_up(off + (size_t)d.rows * c->h * elt * (swiglu ? 2 : 1), 1024);
  b.dxp = off;
  off = align_up(off + (size_t)d.rows * c->d * elt, 1024);
  b.dl = off;
  off = align_up(off + (size_t)c->n * c->E * 4, 1024);
  b.wgt = off;
  off = align_up(off + (size_t)c->d * c->E * 4, 1024);
  b.splits = router_bwd_splits(c->n, c->d, c->E);
  b.part = off;
  if (b.splits > 1) off = align_up(off + (size_t)b.splits * c->d * c->E * 4, 1024);
  b.end = off;
  // pad clear, combine backward, five grouped GEMMs, W_g transpose, router
  // dX, router dWg (+ its ordered reduce)
  b.launches = 10 + (b.splits > 1 ? 1 : 0);
  return b;
}

// The buffers of one backward call (device, the config's dtype).
struct BwdBufs {
  void *xp, *dy, *U, *V, *H, *duv, *dxp;
  bool saved;  // U, V and H were kept by moe_layer_forward_train (bf16)
};

// The five grouped GEMMs of an fp32 layer, on FFMA.
// (err: the FFMA kernels wait on nothing, so they report no error)
static moe_status bwd_gemms_f32(const moe_config* cfg, const Derived& d, const BwdBufs& B,
                                const void* X, const void* W1, const void* W3, const void* W2,
                                const void* sW1, const void* sW3, const void* sW2,
                                const moe_route_out* route, const void* dout, void* dW1,
                                void* dW3, void* dW2, void* dsW1, void* dsW3, void* dsW2,
                                int* /*err*/, cudaStream_t s) {
  const bool swiglu = cfg->act == MOE_ACT_SWIGLU;
  const int n = cfg->n, D = cfg->d, h = cfg->h, E = cfg->E, ns = cfg->n_shared;
  void* xp = B.xp;
  void* dy = B.dy;
  void* U = B.U;
  void* V = B.V;
  void* H = B.H;
  void* duv = B.duv;
  void* dxp = B.dxp;
  auto fp = [](const void* p) { return static_cast<const float*>(p); };
  auto fm = [](void* p) { return static_cast<float*>(p); };
  BwdF32Args f{};
  f.offsets = route->offsets;
  f.counts = route->counts;
  f.E = E;
  f.n_shared = ns;
  f.n = n;
  f.n_pad = d.n_pad;
  f.rows_routed = d.rows_routed;
  f.shared_base = d.shared_base;
  f.act = cfg->act;
  f.swiglu = swiglu;
  const long long hcols = swiglu ? 2LL * h : h;
  float* Uf = static_cast<float*>(U);
  float* Vf = static_cast<float*>(V);
  float* Hf = static_cast<float*>(H);
  float* duvf = static_cast<float*>(duv);
  float* dyf = static_cast<float*>(dy);
  float* dxpf = static_cast<float*>(dxp);
  float* xpf = static_cast<float*>(xp);
  // SAVE: U (V), H
  BwdF32Args q = f;
  q.N = h;
  q.K = D;
  q.A = xpf;
  q.lda = D;
  q.A_sh = fp(X);
  q.B = fp(W1);
  q.B3 = fp(W3);
  q.sB = fp(sW1);
  q.sB3 = fp(sW3);
  q.b_expert_stride = (long long)h * D;
  q.out0 = Uf;
  q.out1 = Vf;
  q.out2 = Hf;
  q.ld_out = h;
  MOE_CU(run_bwd_f32(BW_SAVE, q, s));
  // DACT: dU (dV) = (dY W2) * act'
  q = f;
  q.N = h;
  q.K = D;
  q.A = dyf;
  q.lda = D;
  q.A_sh = fp(dout);
  q.B = fp(W2);
  q.sB = fp(sW2);
  q.b_expert_stride = (long long)D * h;
  q.in0 = Uf;
  q.in1 = Vf;
  q.ld_in = h;
  q.out0 = duvf;
  q.ld_out = hcols;
  MOE_CU(run_bwd_f32(BW_DACT, q, s));
  // DX: dX_perm = dU W1 (+ dV W3)
  q = f;
  q.N = D;
  q.K = (int)hcols;
  q.k_split = h;
  q.A = duvf;
  q.lda = hcols;
  q.A_sh = duvf;
  q.a_sh_base = d.shared_base;
  q.a_sh_stride = d.n_pad;
  q.B = fp(W1);
  q.B3 = fp(W3);
  q.sB = fp(sW1);
  q.sB3 = fp(sW3);
  q.b_expert_stride = (long long)h * D;
  q.out0 = dxpf;
  q.ld_out = D;
  MOE_CU(run_bwd_f32(BW_DX, q, s));
  // WG2: dW2_e = dY_e^T H_e
  q = f;
  q.M = D;
  q.m_split = D;
  q.N = h;
  q.WA = dyf;
  q.ld_wa = D;
  q.WA_sh = fp(dout);
  q.WB = Hf;
  q.ld_wb = h;
  q.WB_sh = Hf;
  q.wb_sh_base = d.shared_base;
  q.wb_sh_stride = d.n_pad;
  q.w_out0 = q.w_out1 = fm(dW2);
  q.sw_out0 = q.sw_out1 = ns > 0 ? fm(dsW2) : fm(dW2);
  q.w_expert_stride = (long long)D * h;
  MOE_CU(run_bwd_f32(BW_WG2, q, s));
  // WG13: [dW1_e; dW3_e] = [dU_e | dV_e]^T X_e
  q = f;
  q.M = (int)hcols;
  q.m_split = h;
  q.N = D;
  q.WA = duvf;
  q.ld_wa = hcols;
  q.WA_sh = duvf;
  q.wa_sh_base = d.shared_base;
  q.wa_sh_stride = d.n_pad;
  q.WB = xpf;
  q.ld_wb = D;
  q.WB_sh = fp(X);
  q.w_out0 = fm(dW1);
  q.w_out1 = swiglu ? fm(dW3) : fm(dW1);
  q.sw_out0 = ns > 0 ? fm(dsW1) : fm(dW1);
  q.sw_out1 = ns > 0 && swiglu ? fm(dsW3) : q.sw_out0;
  q.w_expert_stride = (long long)h * D;
  MOE_CU(run_bwd_f32(BW_WG13, q, s));
  return MOE_OK;
}

// The five grouped GEMMs of a bf16 layer, on the tcgen05 tensor cores.
static moe_status bwd_gemms_bf16(const moe_config* cfg, const Derived& d, const BwdBufs& B,
                                 const void* X, const void* W1, const void* W3, const void* W2,
                                 const void* sW1, const void* sW3, const void* sW2,
                                 const moe_route_out* route, const void* dout, void* dW1,
                                 void* dW3, void* dW2, void* dsW1, void* dsW3, void* dsW2,
                                 int* err, cudaStream_t s) {
  const bool swiglu = cfg->act == MOE_ACT_SWIGLU;
  const int n = cfg->n, D = cfg->d, h = cfg->h, E = cfg->E, ns = cfg->n_shared;
  const long long rows = d.rows;
  __nv_bfloat16* xp = static_cast<__nv_bfloat16*>(B.xp);
  __nv_bfloat16* dy = static_cast<__nv_bfloat16*>(B.dy);
  __nv_bfloat16* U = static_cast<__nv_bfloat16*>(B.U);
  __nv_bfloat16* V = static_cast<__nv_bfloat16*>(B.V);
  __nv_bfloat16* H = static_cast<__nv_bfloat16*>(B.H);
  __nv_bfloat16* duv = static_cast<__nv_bfloat16*>(B.duv);
  __nv_bfloat16* dxp = static_cast<__nv_bfloat16*>(B.dxp);
  auto bf = [](const void* p) { return static_cast<__nv_bfloat16*>(const_cast<void*>(p)); };
  BwdParams base{};
  base.offsets = route->offsets;
  base.counts = route->counts;
  base.E = E;
  base.n_shared = ns;
  base.n = n;
  base.swiglu = swiglu;
  base.act = cfg->act;
  base.shared_blocks = d.n_pad / kRowAlign;
  base.max_routed_blocks = (int)(d.rows_routed / kRowAlign);
  base.out_shared_base = d.shared_base;
  base.n_pad = d.n_pad;
  base.err = err;
  const int rbox = kRowAlign;
  auto map = [](CUtensorMap* m, const void* p, long long r, long long c, int box) {
    return make_bf16_sw128_map(m, p, r, c, box);
  };
  // row GEMMs on CTA pairs when experts average two 128-row blocks, as the
  // forward does; the weight gradients too. A single CTA's 128 x 256 tile
  // over an expert's few k-blocks waits on its operands (c5: the MMA thread
  // idles 46% of the time for loads); a pair's 256 x 256 tile loads half of
  // B per CTA (16% waiting for loads, 27% for the epilogue), 8-9% fewer
  // cycles per launch
  const bool rpair = ffn_uses_pair(cfg, d);
  const bool wpair = rpair;
  // 3. SAVE: U (and V), H of every dispatched row again (unless the
  //    training forward kept them)
  if (!B.saved) {
    BwdMaps m{};
    BwdParams p = base;
    if (!map(&m.a0, xp, rows, D, rbox)) return MOE_ERR_UNSUPPORTED;
    m.a1 = m.a0;
    if (ns > 0 && !map(&m.a1, X, n, D, rbox)) return MOE_ERR_UNSUPPORTED;
    const int bbox = swiglu || rpair ? 128 : 256;
    if (!map(&m.b0, W1, (long long)E * h, D, bbox)) return MOE_ERR_UNSUPPORTED;
    m.b0g = m.b0;
    if (swiglu && !map(&m.b0g, W3, (long long)E * h, D, bbox)) return MOE_ERR_UNSUPPORTED;
    m.b1 = m.b0;
    m.b1g = m.b0g;
    if (ns > 0) {
      if (!map(&m.b1, sW1, (long long)ns * h, D, bbox)) return MOE_ERR_UNSUPPORTED;
      if (swiglu && !map(&m.b1g, sW3, (long long)ns * h, D, bbox)) return MOE_ERR_UNSUPPORTED;
    }
    p.K = D;
    p.n_total = h;
    p.n_block = swiglu ? 128 : 256;
    p.nt_tiles = ceil_div(h, p.n_block);
    p.b_rows_per_expert = h;
    p.out0 = U;
    p.out1 = V;
    p.out2 = H;
    p.ld_out = h;
    MOE_CU(run_bwd_gemm(BW_SAVE, rpair, m, p, s));
  }
  // 4. DACT: dU (and dV) = (dY W2) * act'
  {
    BwdMaps m{};
    BwdParams p = base;
    if (!map(&m.a0, dy, d.rows_routed, D, rbox)) return MOE_ERR_UNSUPPORTED;
    m.a1 = m.a0;
    if (ns > 0 && !map(&m.a1, dout, n, D, rbox)) return MOE_ERR_UNSUPPORTED;
    if (!map(&m.b0, W2, (long long)E * D, h, 64)) return MOE_ERR_UNSUPPORTED;
    m.b0g = m.b1 = m.b1g = m.b0;
    if (ns > 0 && !map(&m.b1, sW2, (long long)ns * D, h, 64)) return MOE_ERR_UNSUPPORTED;
    p.K = D;
    p.n_total = h;
    p.n_block = 256;
    p.nt_tiles = ceil_div(h, 256);
    p.b_rows_per_expert = D;
    p.in0 = U;
    p.in1 = V;
    p.ld_in = h;
    p.out0 = duv;
    p.ld_out = swiglu ? 2LL * h : h;
    MOE_CU(run_bwd_gemm(BW_DACT, rpair, m, p, s));
  }
  // 5. DX: dX_perm = dU W1 (+ dV W3). Fine-grained token choice (128 to 512
  //    rows per expert on average) puts the weights on the M side, as the
  //    forward's down projection does: each expert's exact token count instead
  //    of whole 256-row pair tiles
  SwapDxArgs sx{};
  sx.duv = duv;
  sx.rows = rows;
  sx.rows_routed = d.rows_routed;
  sx.kcols = swiglu ? 2 * h : h;
  sx.E = E;
  sx.h = h;
  sx.d = D;
  sx.n_shared = ns;
  sx.n = n;
  sx.shared_base = d.shared_base;
  sx.n_pad = d.n_pad;
  sx.W1 = W1;
  sx.W3 = swiglu ? W3 : nullptr;
  sx.sW1 = sW1;
  sx.sW3 = swiglu ? sW3 : nullptr;
  sx.offsets = route->offsets;
  sx.counts = route->counts;
  sx.dxp = dxp;
  sx.err = err;
  if (ffn_uses_swap(cfg, d) && swap_dx_supported(sx)) {
    const moe_status st = run_bwd_dx_swap(sx, s);
    if (st != MOE_OK) return st;
  } else {
    BwdMaps m{};
    BwdParams p = base;
    const long long kcols = swiglu ? 2LL * h : h;
    if (!map(&m.a0, duv, rows, kcols, rbox)) return MOE_ERR_UNSUPPORTED;
    m.a1 = m.a0;
    p.a1_row_base = d.shared_base;
    p.a1_row_stride = d.n_pad;
    if (!map(&m.b0, W1, (long long)E * h, D, 64)) return MOE_ERR_UNSUPPORTED;
    m.b0g = m.b0;
    if (swiglu && !map(&m.b0g, W3, (long long)E * h, D, 64)) return MOE_ERR_UNSUPPORTED;
    m.b1 = m.b0;
    m.b1g = m.b0g;
    if (ns > 0) {
      if (!map(&m.b1, sW1, (long long)ns * h, D, 64)) return MOE_ERR_UNSUPPORTED;
      if (swiglu && !map(&m.b1g, sW3, (long long)ns * h, D, 64)) return MOE_ERR_UNSUPPORTED;
    }
    p.K = (int)kcols;
    p.k_split = h;
    p.n_total = D;
    p.n_block = 256;
    p.nt_tiles = ceil_div(D, 256);
    p.b_rows_per_expert = h;
    p.out0 = dxp;
    p.ld_out = D;
    MOE_CU(run_bwd_gemm(BW_DX, rpair, m, p, s));
  }
  // 6. WG2: dW2_e = dY_e^T H_e
  {
    BwdMaps m{};
    BwdParams p = base;
    if (!map(&m.a0, dy, d.rows_routed, D, 64)) return MOE_ERR_UNSUPPORTED;
    m.a1 = m.a0;
    if (ns > 0 && !map(&m.a1, dout, n, D, 64)) return MOE_ERR_UNSUPPORTED;
    if (!map(&m.b0, H, rows, h, 64)) return MOE_ERR_UNSUPPORTED;
    m.b0g = m.b1 = m.b1g = m.b0;
    p.b1_row_base = d.shared_base;
    p.b1_row_stride = d.n_pad;
    p.m_total = D;
    p.m_split = D;
    p.mt_tiles = ceil_div(D, wpair ? 256 : 128);
    p.ld_w = h;
    p.nt_tiles = ceil_div(h, 256);
    p.w_expert_stride = (long long)D * h;
    p.w_out0 = bf(dW2);
    p.w_out1 = bf(dW2);
    p.sw_out0 = p.sw_out1 = ns > 0 ? bf(dsW2) : bf(dW2);
    if (!map(&m.o0, dW2, (long long)E * D, h, 32)) return MOE_ERR_UNSUPPORTED;
    m.o1 = m.o2 = m.o3 = m.o0;
    if (ns > 0 && !map(&m.o2, dsW2, (long long)ns * D, h, 32)) return MOE_ERR_UNSUPPORTED;
    m.o3 = m.o2;
    MOE_CU(run_bwd_gemm(BW_WG2, wpair, m, p, s));
  }
  // 7. WG13: [dW1_e; dW3_e] = [dU_e | dV_e]^T X_e
  {
    BwdMaps m{};
    BwdParams p = base;
    const long long mcols = swiglu ? 2LL * h : h;
    if (!map(&m.a0, duv, rows, mcols, 64)) return MOE_ERR_UNSUPPORTED;
    m.a1 = m.a0;
    p.a1_row_base = d.shared_base;
    p.a1_row_stride = d.n_pad;
    if (!map(&m.b0, xp, rows, D, 64)) return MOE_ERR_UNSUPPORTED;
    m.b0g = m.b1 = m.b1g = m.b0;
    if (ns > 0 && !map(&m.b1, X, n, D, 64)) return MOE_ERR_UNSUPPORTED;
    p.m_total = (int)mcols;
    p.m_split = h;
    p.mt_tiles = ceil_div(mcols, wpair ? 256 : 128);
    p.ld_w = D;
    p.nt_tiles = ceil_div(D, 256);
    p.w_expert_stride = (long long)h * D;
    p.w_out0 = bf(dW1);
    p.w_out1 = swiglu ? bf(dW3) : bf(dW1);
    p.sw_out0 = ns > 0 ? bf(dsW1) : bf(dW1);
    p.sw_out1 = ns > 0 && swiglu ? bf(dsW3) : p.sw_out0;
    if (!map(&m.o0, dW1, (long long)E * h, D, 32)) return MOE_ERR_UNSUPPORTED;
    m.o1 = m.o2 = m.o3 = m.o0;
    if (swiglu && !map(&m.o1, dW3, (long long)E * h, D, 32)) return MOE_ERR_UNSUPPORTED;
    if (ns > 0) {
      if (!map(&m.o2, dsW1, (long long)ns * h, D, 32)) return MOE_ERR_UNSUPPORTED;
      m.o3 = m.o2;
      if (swiglu && !map(&m.o3, dsW3, (long long)ns * h, D, 32)) return MOE_ERR_UNSUPPORTED;
    }
    MOE_CU(run_bwd_gemm(BW_WG13, wpair, m, p, s));
  }
  return MOE_OK;
}

moe_status moe_backward_workspace_size(const moe_config* cfg, size_t* bytes, int* launches) {
  Derived d;
  moe_status st = derive(cfg, &d);
  if (st != MOE_OK) return st;
  const BwdLayout b = bwd_layout(cfg, d);
  if (bytes) *bytes = b.end;
  if (launches) *launches = b.launches;
  return MOE_OK;
}

moe_status moe_train_launch_counts(const moe_config* cfg, int* forward, int* backward) {
  int r = 0, g = 0, f = 0, c = 0, b = 0;
  moe_status st = moe_launch_counts(cfg, &r, &g, &f, &c);
  if (st != MOE_OK) return st;
  if ((st = moe_backward_workspace_size(cfg, nullptr, &b)) != MOE_OK) return st;
  // bf16: the training forward also clears the dispatched rows' padding
  // before its up projection, and the training backward skips the recompute
  const int bf16 = cfg->dtype == MOE_BF16;
  if (forward) *forward = r + g + f + c + bf16;
  if (backward) *backward = b - bf16;
  return MOE_OK;
}

static moe_status layer_backward_impl(const moe_config* cfg, const void* X, const float* Wg,
                                      const void* W1, const void* W3, const void* W2,
                                      const void* sW1, const void* sW3, const void* sW2,
                                      const moe_route_out* route, void* fwd_ws,
                                      size_t fwd_ws_bytes, const void* dout, void* dX,
                                      float* dWg, void* dW1, void* dW3, void* dW2, void* dsW1,
                                      void* dsW3, void* dsW2, float* dL, void* ws,
                                      size_t ws_bytes, moe_stream_t stream, bool saved) {
  Derived d;
  moe_status st = derive(cfg, &d);
  if (st != MOE_OK) return st;
  const bool bf16 = cfg->dtype == MOE_BF16;
  // the bf16 weight-gradient epilogue writes 32-row groups that never
  // straddle the W1 / W3 boundary (h) or the end of the output (d, h or 2h)
  if (bf16 && (cfg->d % 64 != 0 || cfg->h % 64 != 0)) return MOE_ERR_UNSUPPORTED;
  const bool swiglu = cfg->act == MOE_ACT_SWIGLU;
  const bool tc = cfg->mode == MOE_TOKEN_CHOICE;
  if (!X || !Wg || !W1 || !W2 || !dout || !dX || !dWg || !dW1 || !dW2) return MOE_ERR_INVALID_ARG;
  if (swiglu && (!W3 || !dW3)) return MOE_ERR_INVALID_ARG;
  if (cfg->n_shared > 0 && (!sW1 || !sW2 || !dsW1 || !dsW2 || (swiglu && (!sW3 || !dsW3))))
    return MOE_ERR_INVALID_ARG;
  if ((st = check_route_out(cfg, route)) != MOE_OK) return st;
  const bool need_logits = (tc && cfg->z_coef != 0.0f) || cfg->score == MOE_SCORE_SQRTSOFTPLUS;
  if (need_logits && (!route->logits || (tc && cfg->z_coef != 0.0f && !route->lse)))
    return MOE_ERR_INVALID_ARG;
  const WsLayout fw = ws_layout(cfg, d);
  if ((st = check_ws(fwd_ws, fwd_ws_bytes, fw.layer_end)) != MOE_OK) return st;
  const BwdLayout b = bwd_layout(cfg, d);
  if ((st = check_ws(ws, ws_bytes, b.end)) != MOE_OK) return st;
  const void* aligned[] = {X, dout, dX, fwd_ws, W1, W2, dW1, dW2, W3, dW3,
                           sW1, sW2, sW3, dsW1, dsW2, dsW3};
  for (const void* ptr : aligned)
    if (reinterpret_cast<uintptr_t>(ptr) & 15) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  __nv_bfloat16* xp = at<__nv_bfloat16>(fwd_ws, fw.xperm);
  const __nv_bfloat16* yp = at<__nv_bfloat16>(fwd_ws, fw.yperm);
  __nv_bfloat16* dy = at<__nv_bfloat16>(ws, b.dy);
  __nv_bfloat16* U = at<__nv_bfloat16>(ws, b.u);
  __nv_bfloat16* V = swiglu ? at<__nv_bfloat16>(ws, b.v) : nullptr;
  __nv_bfloat16* H = at<__nv_bfloat16>(ws, b.hh);
  __nv_bfloat16* duv = at<__nv_bfloat16>(ws, b.duv);
  __nv_bfloat16* dxp = at<__nv_bfloat16>(ws, b.dxp);
  float* dl = dL ? dL : at<float>(ws, b.dl);
  int* err = at<int>(ws, b.err);
  const int n = cfg->n, D = cfg->d, E = cfg->E, ns = cfg->n_shared;

  // 1. padding rows of the dispatched inputs and output gradients read as
  //    zeros by the weight-gradient reductions
  const int elt = bf16 ? 2 : 4;
  MOE_CU(launch_pad_zero(route->offsets, route->counts, E, D * elt, xp, dy, s));
  // 2. output gradient per kept row, gate gradients, logit gradients
  CombineBwdArgs cb{};
  cb.bf16 = bf16;
  cb.Y_perm = yp;
  cb.dout = dout;
  cb.tok_row = route->tok_row;
  cb.tok_gate = route->tok_gate;
  cb.idx = route->idx;
  cb.drop = route->drop;
  cb.offsets = route->offsets;
  cb.load = route->load;
  cb.scores = route->scores;
  cb.logits = route->logits;
  cb.lse = route->lse;
  cb.n = n;
  cb.d = D;
  cb.E = E;
  cb.slots = d.slots;
  cb.tc = tc;
  cb.K = tc ? d.k : 0;
  cb.score = cfg->score;
  cb.weights = cfg->weights;
  cb.lb_coef = tc ? cfg->lb_coef : 0.0f;
  cb.z_coef = tc ? cfg->z_coef : 0.0f;
  cb.dY_perm = dy;
  cb.dL = dl;
  cb.max_rows = d.rows_routed;
  cb.err = err;
  MOE_CU(launch_combine_backward(cb, s));

  const BwdBufs bufs{xp, dy, U, V, H, duv, dxp, saved && bf16};
  if ((st = (bf16 ? bwd_gemms_bf16 : bwd_gemms_f32)(cfg, d, bufs, X, W1, W3, W2, sW1, sW3, sW2,
                                                     route, dout, dW1, dW3, dW2, dsW1, dsW3,
                                                     dsW2, err, s)) != MOE_OK)
    return st;
  // 8, 9. router: dX = dL Wg^T + the token's dispatched rows; dWg = X^T dL
  RouterBwdArgs rb{};
  rb.bf16 = bf16;
  rb.X = X;
  rb.Wg = Wg;
  rb.WgT = at<float>(ws, b.wgt);
  rb.dL = dl;
  rb.dX_perm = dxp;
  rb.tok_row = route->tok_row;
  rb.n = n;
  rb.d = D;
  rb.E = E;
  rb.slots = d.slots;
  rb.n_shared = ns;
  rb.shared_base = d.shared_base;
  rb.n_pad = d.n_pad;
  rb.dX = dX;
  rb.dWg = dWg;
  rb.max_rows = d.rows_routed;
  rb.err = err;
  rb.partial = at<float>(ws, b.part);
  rb.splits = b.splits;
  MOE_CU(launch_router_backward(rb, s));
  return MOE_OK;
}

moe_status moe_layer_backward(const moe_config* cfg, const void* X, const float* Wg,
                              const void* W1, const void* W3, const void* W2, const void* sW1,
                              const void* sW3, const void* sW2, const moe_route_out* route,
                              void* fwd_ws, size_t fwd_ws_bytes, const void* dout, void* dX,
                              float* dWg, void* dW1, void* dW3, void* dW2, void* dsW1,
                              void* dsW3, void* dsW2, float* dL, void* ws, size_t ws_bytes,
                              moe_stream_t stream) {
  return layer_backward_impl(cfg, X, Wg, W1, W3, W2, sW1, sW3, sW2, route, fwd_ws, fwd_ws_bytes,
                             dout, dX, dWg, dW1, dW3, dW2, dsW1, dsW3, dsW2, dL, ws, ws_bytes,
                             stream, false);
}

moe_status moe_layer_backward_train(const moe_config* cfg, const void* X, const float* Wg,
                                    const void* W1, const void* W3, const void* W2,
                                    const void* sW1, const void* sW3, const void* sW2,
                                    const moe_route_out* route, void* fwd_ws,
                                    size_t fwd_ws_bytes, const void* dout, void* dX,
                                    float* dWg, void* dW1, void* dW3, void* dW2, void* dsW1,
                                    void* dsW3, void* dsW2, float* dL, void* ws, size_t ws_bytes,
                                    moe_stream_t stream) {
  return layer_backward_impl(cfg, X, Wg, W1, W3, W2, sW1, sW3, sW2, route, fwd_ws, fwd_ws_bytes,
                             dout, dX, dWg, dW1, dW3, dW2, dsW1, dsW3, dsW2, dL, ws, ws_bytes,
                             stream, true);
}

moe_status moe_layer_forward_train(const moe_config* cfg, const void* X, const float* Wg,
                                   const float* logit_bias, const float* sel_bias,
                                   const void* W1, const void* W3, const void* W2,
                                   const void* sW1, const void* sW3, const void* sW2, void* out,
                                   moe_route_out* route, void* ws, size_t ws_bytes,
                                   void* bwd_ws, size_t bwd_ws_bytes, moe_stream_t stream) {
  if (!cfg || cfg->dtype != MOE_BF16)  // fp32 layers keep nothing: their backward recomputes
    return moe_layer_forward(cfg, X, Wg, logit_bias, sel_bias, W1, W3, W2, sW1, sW3, sW2, out,
                             route, ws, ws_bytes, stream);
  Derived d;
  moe_status st = derive(cfg, &d);
  if (st != MOE_OK) return st;
  if (!X || !Wg || !out || !W1 || !W2) return MOE_ERR_INVALID_ARG;
  if ((st = check_route_out(cfg, route)) != MOE_OK) return st;
  const WsLayout w = ws_layout(cfg, d);
  if ((st = check_ws(ws, ws_bytes, w.layer_end)) != MOE_OK) return st;
  const BwdLayout b = bwd_layout(cfg, d);
  if ((st = check_ws(bwd_ws, bwd_ws_bytes, b.end)) != MOE_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  void* xp = at<void>(ws, w.xperm);
  void* yp = at<void>(ws, w.yperm);
  void* U = at<void>(bwd_ws, b.u);
  void* V = cfg->act == MOE_ACT_SWIGLU ? at<void>(bwd_ws, b.v) : nullptr;
  void* H = at<void>(bwd_ws, b.hh);
  if ((st = route_impl(cfg, d, w, X, Wg, logit_bias, sel_bias, route, ws, s)) != MOE_OK)
    return st;
  if ((st = dispatch_impl(cfg, d, X, route, xp, at<int>(ws, w.err), s)) != MOE_OK) return st;
  // padding rows of X_perm as zeros, so that the kept U, V and H are zero
  // there and the weight-gradient reductions may read them
  MOE_CU(launch_pad_zero(route->offsets, route->counts, cfg->E, cfg->d * 2, xp, nullptr, s));
  if ((st = ffn_impl(cfg, d, X, xp, nullptr, route->offsets, route->counts, W1, W3, W2, sW1,
                     sW3, sW2, H, yp, at<int>(ws, w.err), s, nullptr, nullptr, U, V)) != MOE_OK)
    return st;
  return combine_impl(cfg, d, yp, route, out, s, at<int>(ws, w.err));
}

moe_status moe_debug_inject_fault(moe_fault fault) { return set_fault((int)fault); }

moe_status moe_workspace_init(void* ws, moe_stream_t stream) {
  if (!ws) return MOE_ERR_WORKSPACE;
  MOE_CU(cudaMemsetAsync(ws, 0, MOE_WS_ERROR_BYTES, (cudaStream_t)stream));
  return MOE_OK;
}

moe_status moe_read_error(void* ws, moe_stream_t stream, int* detail) {
  cudaStream_t s = (cudaStream_t)stream;
  int code = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  if (ws == nullptr) {
    // no workspace: the word of moe_route_noalloc's static scratch
    code = take_noalloc_error();
  } else {
    if (cudaMemcpy(&code, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
      return MOE_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpy(ws, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  if (code == 0) code = take_dispatch_error();
  if (detail) *detail = code;
  if (code == 0) return MOE_OK;
  return (code & 0xF00) == kErrGemmTimeout ? MOE_ERR_TIMEOUT : MOE_ERR_CUDA;
}

}  // extern "C"
