// Router: logits = X W_g (+ logit bias) on FP32 FFMA, with the score
// function, logsumexp, partial column sums of S and (token choice) the
// per-token top-k fused into the epilogue.
//
// "Expert choice routing" (aicassindra.com), "The transposed selection":
// S = softmax(X W_g), X [n,d], W_g [d,E]; "MoE token-choice routing"
// (zenaique.com), "Token-choice: the token picks experts": z_t = W h_t
// depends only on h_t; "MoE routing strategies explained" (ncijnetwork.com),
// "4. Sigmoid gating with aux-loss-free bias" and "5. Group-limited and
// node-limited routing".
//
// The router contraction stays on CUDA cores in fp32: its scores decide
// integer selections, and the expert FFN is the only step that runs on the
// tensor cores.
//
// Main loop: one CTA owns BM rows and all E columns (so the epilogue sees
// whole rows). X and W_g chunks of BK along d stream through a 3- or 4-deep
// cp.async ring; each X chunk is transposed once into one of two A tiles
// (bf16 X stays bf16 there and is widened per fragment). One barrier per
// chunk: the next chunk's transposition and copies are spread over the
// current chunk's FMA steps. Each thread holds TM x TN accumulators, updated
// with packed fp32x2 FMAs; a lane's TN columns are groups of 4 that sit 4*LY
// columns apart, so every 8-lane phase of a 128-bit shared load reads one
// contiguous 128 bytes (no bank conflicts). WK > 1 splits each chunk's k
// range across warp groups, summed in a fixed order.
#include <math.h>

#include "device_common.cuh"
#include "moe_internal.h"

namespace moe {

template <int ET_, int TM_, int TN_, int LX_, int WX_, int WY_, int WK_, int BK_, int ST_>
struct RCfg {
  static constexpr int ET = ET_, TM = TM_, TN = TN_, LX = LX_, LY = 32 / LX_, WX = WX_,
                       WY = WY_, WK = WK_, BK = BK_, ST = ST_, BM = WX_ * LX_ * TM_;
  static constexpr int NW = WX * WY * WK, NT = 32 * NW;  // warps, threads
  static_assert(WY * LY * TN == ET, "columns");
  static_assert(NW == 8 || NW == 12, "8 or 12 warps");
  static_assert(TN == 4 || TN == 8 || TN == 16, "TN");
  static_assert(TM >= 1 && TM <= 8, "TM");
  static_assert(BK % WK == 0 && ST >= 3, "pipeline");
};
// 4 x 8 (E = 64, 128) or 8 x 8 (E = 256) register tiles: the larger the tile
// the fewer shared-memory fragment loads per FMA. The "s" variants trade rows
// per CTA for an in-CTA K split when the batch is too small to give every SM
// a CTA. E = 8 is bound by reading X, so its chunks are long (BK 96, twelve
// warps of eight steps each: the capacity layer's route stage 72.7-73.7 us
// against 77.8-81.9 with eight warps and BK 128).
//                   ET   TM TN LX WX WY WK  BK  ST
using R8 = RCfg<8, 1, 8, 32, 1, 1, 12, 96, 4>;
using R32 = RCfg<32, 2, 4, 4, 4, 1, 2, 64, 4>;
using R64 = RCfg<64, 4, 8, 4, 4, 1, 2, 32, 4>;
using R64s = RCfg<64, 4, 8, 4, 1, 1, 8, 64, 4>;
using R128 = RCfg<128, 4, 8, 4, 2, 2, 2, 32, 4>;
using R256 = RCfg<256, 8, 8, 4, 1, 4, 2, 32, 3>;
using R256s = RCfg<256, 2, 8, 4, 2, 4, 1, 32, 3>;
// bf16 X, E > 32: a family over TM (rows per thread), so that the batch
// splits into about one CTA's worth of rows per SM (the contraction is bound
// by the FFMA pipe, so an SM holding two CTAs' rows while another holds one
// sets the time). "A" splits each chunk's k range over 8 warps (few rows per
// CTA), "C" over 3 warp groups of 4 (many rows per CTA): 12 warps, 48-deep
// chunks, so that one CTA per SM of 112 rows hides its loads (n 16384, d 2048:
// route stage 147.4 us, against 174.1 with 8 warps and two CTAs of 64 rows)
template <int TM> using R64A = RCfg<64, TM, 8, 4, 1, 1, 8, 64, 4>;   // BM = 4 TM
template <int TM> using R64C = RCfg<64, TM, 8, 4, 4, 1, 3, 48, 3>;   // BM = 16 TM
// R64A's tiles on 12 warps (a twelve-way k split of 96-deep chunks): in a
// single wave of one CTA per SM, 50% more warps to hide the chunks' loads.
// 96-deep chunks (eight steps per warp between barriers) measured 46.0 us
// for the expert-choice route stage at n 4096, d 1024 against 48.1 with 48
// (longer chunks or deeper rings gave no more)
template <int TM> using R64D = RCfg<64, TM, 8, 4, 1, 1, 12, 96, 4>;  // BM = 4 TM
template <int TM> using R128A = RCfg<128, TM, 8, 4, 2, 2, 2, 32, 4>; // BM = 8 TM
template <int TM> using R256A = RCfg<256, TM, 8, 4, 1, 4, 2, 32, 3>; // BM = 4 TM
// E = 256 with 16 columns per thread: per 16-deep step a warp issues TM*16
// FFMAs for TM + 16 shared-memory wavefronts (TM x 8 tiles: TM*8 for TM + 8),
// so the FMA pipe, not shared-memory bandwidth, sets the pace; one CTA per
// SM (about 160 registers a thread)
template <int TM> using R256B = RCfg<256, TM, 16, 4, 2, 2, 2, 32, 3>; // BM = 8 TM
// the same tiles with a three-way k split over 12 warps (three per SM
// sub-partition instead of two, so one warp's shared-memory and dependency
// waits hide behind two others'), 48-deep chunks; one CTA per SM, at most
// 168 registers a thread
template <int TM> using R256C = RCfg<256, TM, 16, 4, 2, 2, 3, 48, 3>; // BM = 8 TM

constexpr int kSelectRowsPerWarp = 4;

int router_tile_et(int E) {
  return E <= 8 ? 8 : E <= 32 ? 32 : E <= 64 ? 64 : E <= 128 ? 128 : 256;
}

static int num_sms_cached() {
  static int sms = 0;
  if (!sms) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      sms = 148;
  }
  return sms;
}

// Which tile variant a (E, n, X dtype) uses. fp32 X: fixed tiles, the
// small-row one when the big tile would leave SMs without a CTA. bf16 X with
// E > 32: the (family, TM) whose rows per SM, BM * ceil(CTAs / SMs), is
// smallest (ties to the larger BM). Codes: kFamilyCode + fam * 16 + TM with
// fam 1 = R64A, 2 = R64C, 3 = R128A, 4 = R256A, 5 = R256B, 6 = R256C,
// 7 = R64D; otherwise the fixed tile's ET (257: R256s, 65: R64s).
constexpr int kFamilyCode = 1000;
struct RouterFamily {
  int code, unit, tm_lo;
};
static int router_variant(int E, int n, bool x_bf16) {
  const int et = router_tile_et(E);
  const int sms = num_sms_cached();
  if (x_bf16 && et >= 64) {
    static const RouterFamily fams64[] = {{7, 4, 4}, {1, 4, 4}, {2, 16, 4}};
    static const RouterFamily fams128[] = {{3, 8, 2}};
    static const RouterFamily fams256[] = {{6, 8, 4}, {5, 8, 4}, {4, 4, 4}};
    const RouterFamily* fams = et == 64 ? fams64 : et == 128 ? fams128 : fams256;
    const int nf = et == 128 ? 1 : 3;
    long long best_cost = -1;
    int best = 0, best_bm = 0;
    for (int f = 0; f < nf; ++f)
      for (int tm = fams[f].tm_lo; tm <= 8; ++tm) {
        const int bm = fams[f].unit * tm;
        const long long ctas = (n + bm - 1) / bm;
        long long cost = (long long)bm * ((ctas + sms - 1) / sms);
        // measured on B200: R64A (eight-way k split, few rows) pays off only
        // in a single wave (c2: 28 rows per SM 26.9 us); with more CTAs than
        // SMs its per-CTA reduction costs more than R64C's (n = 16384: 195 us
        // vs 174, when R64C had 8 warps).
        if ((fams[f].code == 1 || fams[f].code == 7) && ctas > sms) continue;
        // TM x 8 tiles at E = 256 are bound by shared-memory wavefronts
        // (TM + 8 per TM*8 FFMAs per step), the 16-column tiles by the FMA
        // pipe: charge the narrower tile a quarter more per row
        if (fams[f].code == 4) cost = cost * 5 / 4;
        // 12 warps where their registers fit (TM <= 7); listed first, so an
        // equal cost keeps them
        if (fams[f].code == 6 && tm > 7) continue;
        if (best_cost < 0 || cost < best_cost || (cost == best_cost && bm > best_bm)) {
          best_cost = cost;
          best = kFamilyCode + fams[f].code * 16 + tm;
          best_bm = bm;
        }
      }
    return best;
  }
  if (et == 64) return (n + R64::BM - 1) / R64::BM >= sms ? 64 : 65;
  if (et == 256) return (n + R256::BM - 1) / R256::BM >= sms ? 256 : 257;
  return et;
}

// rows (BM) and chunk length (BK) of a variant
static void variant_tile(int v, int* bm, int* bk) {
  switch (v) {
    case 8: *bm = R8::BM; *bk = R8::BK; return;
    case 32: *bm = R32::BM; *bk = R32::BK; return;
    case 64: *bm = R64::BM; *bk = R64::BK; return;
    case 65: *bm = R64s::BM; *bk = R64s::BK; return;
    case 128: *bm = R128::BM; *bk = R128::BK; return;
    case 256: *bm = R256::BM; *bk = R256::BK; return;
    case 257: *bm = R256s::BM; *bk = R256s::BK; return;
    default: {
      const int code = v - kFamilyCode, fam = code / 16, tm = code % 16;
      *bm = (fam == 2 ? 16 : fam == 3 || fam == 5 || fam == 6 ? 8 : 4) * tm;
      *bk = fam == 1 ? 64 : fam == 7 ? 96 : fam == 6 || fam == 2 ? 48 : 32;
    }
  }
}

static int split_of(int ctas, int nchunks);

// k slices the router uses for (E, n, d, X dtype): 1, or >= 2 with a reduce
// pass whose CTAs own 16 rows each
int router_ksplit(int E, int n, int d, bool x_bf16) {
  int bm, bk;
  variant_tile(router_variant(E, n, x_bf16), &bm, &bk);
  const int nchunks = ceil_div(d, bk);
  const int ks = split_of(ceil_div(n, bm), nchunks);
  if (ks == 1) return 1;
  return ceil_div(nchunks, ceil_div(nchunks, ks));
}

int router_block_rows(int E, int n, int d, bool x_bf16) {
  if (router_ksplit(E, n, d, x_bf16) > 1) return kRouterMinBlockRows;
  int bm, bk;
  variant_tile(router_variant(E, n, x_bf16), &bm, &bk);
  return bm;
}

int select_tc_block_rows() { return 8 * kSelectRowsPerWarp; }

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
  const int n = valid ? 16 : 0;  // 0 source bytes = zero fill
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(n)
               : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src, bool valid) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
  const int n = valid ? 4 : 0;
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(d), "l"(src), "r"(n)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ---------------------------------------------------------------------------
// Token-choice selection of one row by one warp. Lane l holds experts
// l*V .. l*V+V-1 (contiguous, so a group of gs experts is gs/V lanes).
// Order: key desc, expert asc. Group score: fp32 sum of the group_topn
// largest keys, largest first; groups ranked by (score desc, group asc).
// Weights always come from the raw scores.
//
// Each key becomes a 32-bit code that orders like the IEEE comparison
// (-0 folded into +0; code 0 means "no candidate"), so one round of a
// top-k is a lane-local max, one warp max-reduction (redux.sync) and a
// ballot: the winner is the lowest lane holding the maximum code, and
// within it the lowest slot, i.e. the lowest expert index among equal keys.
// NaN keys are outside the contract.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t select_code(float k) {
  const uint32_t u = __float_as_uint(k + 0.0f);  // -0 + 0 = +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float select_key(uint32_t c) {
  return __uint_as_float((c & 0x80000000u) ? (c & 0x7fffffffu) : ~c);
}
template <int V>
__device__ __forceinline__ uint32_t lane_max_code(const uint32_t (&c)[V]) {
  uint32_t m[V];
#pragma unroll
  for (int v = 0; v < V; ++v) m[v] = c[v];
#pragma unroll
  for (int w = 1; w < V; w <<= 1)
#pragma unroll
    for (int v = 0; v + w < V; v += 2 * w) m[v] = max(m[v], m[v + w]);
  return m[0];
}
// Clears the lowest slot holding code M (the caller knows there is one) and
// returns that slot.
template <int V>
__device__ __forceinline__ int take_code(uint32_t (&c)[V], uint32_t M) {
  int pos = 0;
#pragma unroll
  for (int v = V - 1; v >= 0; --v)
    if (c[v] == M) pos = v;
#pragma unroll
  for (int v = 0; v < V; ++v)
    if (v == pos) c[v] = 0u;
  return pos;
}

template <int V>
__device__ __forceinline__ void tc_select_row(const float (&key)[V], const float (&raw)[V],
                                              const bool (&ok)[V], int lane, int E, int K,
                                              int n_groups, int topk_groups, int group_topn,
                                              int weights, int32_t* idx_out,
                                              float* gate_out) {
  uint32_t code[V];
#pragma unroll
  for (int v = 0; v < V; ++v) code[v] = ok[v] ? select_code(key[v]) : 0u;
  if (n_groups > 1) {
    const int gs = E / n_groups;
    const int lpg = gs / V;             // lanes per group, a power of two <= 16
    const int g = lane / lpg;           // this lane's group
    const unsigned gmask = lpg >= 32 ? 0xffffffffu : ((1u << lpg) - 1u) << (g * lpg);
    uint32_t gc[V];
#pragma unroll
    for (int v = 0; v < V; ++v) gc[v] = code[v];
    float gsum = 0.0f;
    for (int r = 0; r < group_topn; ++r) {
      const uint32_t best = lane_max_code<V>(gc);
      uint32_t M = best;
      for (int m = 1; m < lpg; m <<= 1) M = max(M, __shfl_xor_sync(0xffffffffu, M, m));
      const unsigned hold = __ballot_sync(0xffffffffu, M != 0u && best == M) & gmask;
      if (M == 0u) continue;            // the group has no candidate left
      gsum = gsum + select_key(M);
      if (lane == __ffs(hold) - 1) take_code<V>(gc, M);
    }
    // rank of this lane's group: groups ahead of it by (score desc, group asc)
    int rank = 0;
    for (int h = 0; h < n_groups; ++h) {
      const float o = __shfl_sync(0xffffffffu, gsum, h * lpg);
      rank += (o > gsum || (o == gsum && h < g)) ? 1 : 0;
    }
    const bool gsel = g < n_groups && rank < topk_groups;
#pragma unroll
    for (int v = 0; v < V; ++v) code[v] = gsel ? code[v] : 0u;
  }
  int my_e = -1;
  float my_raw = 0.0f;
  for (int j = 0; j < K; ++j) {
    const uint32_t best = lane_max_code<V>(code);
    const uint32_t M = __reduce_max_sync(0xffffffffu, best);
    const unsigned hold = __ballot_sync(0xffffffffu, M != 0u && best == M);
    const int win = hold ? __ffs(hold) - 1 : 0;
    int e = -1;
    float rv = 0.0f;
    if (hold && lane == win) {
      const int pos = take_code<V>(code, M);
      e = lane * V + pos;
#pragma unroll
      for (int v = 0; v < V; ++v)
        if (v == pos) rv = raw[v];
    }
    e = __shfl_sync(0xffffffffu, e, win);
    rv = __shfl_sync(0xffffffffu, rv, win);
    if (lane == j) {
      my_e = e;
      my_raw = rv;
    }
  }
  float w = my_raw;
  if (weights == MOE_W_NORMALIZED) {
    float denom = 0.0f;
    for (int j = 0; j < K; ++j) denom = denom + __shfl_sync(0xffffffffu, my_raw, j);
    w = my_raw / denom;
  }
  if (lane < K) {
    idx_out[lane] = my_e;
    gate_out[lane] = w;
  }
}

// ---------------------------------------------------------------------------
// Row epilogue shared by both router main loops. Ls holds the CTA's logits
// tile [BM][ET + 1] without the logit bias; 8 warps take one row at a time.
// Adds the bias, applies the score function, writes logits / scores / lse,
// selects the token-choice experts, and leaves this CTA's partial column sums
// of S and its sum of lse^2 in colsum / lse2 at index blockIdx.x.
// colsum_w [NW][ET] floats and lse2_w [NW] doubles are shared-memory scratch
// (NW warps).
// ---------------------------------------------------------------------------
template <int ET, int NW>
__device__ __forceinline__ void router_rows_epilogue(const RouterArgs& a, const float* Ls,
                                                     float* colsum_w, double* lse2_w, int BM,
                                                     int m0) {
  constexpr int LST = ET + 1;
  constexpr int V = ET >= 32 ? ET / 32 : 1;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = a.n, E = a.E;
  float csum[V];
#pragma unroll
  for (int v = 0; v < V; ++v) csum[v] = 0.0f;
  double my_lse2 = 0.0;

  for (int r = warp; r < BM; r += NW) {
    const int t = m0 + r;
    if (t >= n) break;
    float l[V], s[V], key[V];
    bool ok[V];
#pragma unroll
    for (int v = 0; v < V; ++v) {
      const int cc = lane * V + v;
      ok[v] = cc < E;
      l[v] = ok[v] ? Ls[r * LST + cc] + (a.logit_bias ? a.logit_bias[cc] : 0.0f) : -INFINITY;
    }
    float m = -INFINITY;
#pragma unroll
    for (int v = 0; v < V; ++v) m = fmaxf(m, l[v]);
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float ex[V], z = 0.0f;
#pragma unroll
    for (int v = 0; v < V; ++v) {
      ex[v] = ok[v] ? expf(l[v] - m) : 0.0f;
      z += ex[v];
    }
    for (int o = 16; o; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    const float lse = m + logf(z);
#pragma unroll
    for (int v = 0; v < V; ++v) {
      if (a.score == MOE_SCORE_SIGMOID) {
        s[v] = ok[v] ? 1.0f / (1.0f + expf(-l[v])) : 0.0f;
      } else if (a.score == MOE_SCORE_SQRTSOFTPLUS) {
        // sqrt(ln(1 + e^l)), as l + ln(1 + e^-l) for l > 0 (no overflow)
        const float sp = l[v] > 0.0f ? l[v] + log1pf(expf(-l[v])) : log1pf(expf(l[v]));
        s[v] = ok[v] ? sqrtf(sp) : 0.0f;
      } else {
        s[v] = ex[v] / z;
      }
      csum[v] += ok[v] ? s[v] : 0.0f;
      const int cc = lane * V + v;
      if (ok[v]) {
        a.scores[(size_t)t * E + cc] = s[v];
        if (a.logits) a.logits[(size_t)t * E + cc] = l[v];
      }
      key[v] = ok[v] ? (a.sel_bias ? s[v] + a.sel_bias[cc] : s[v]) : 0.0f;
    }
    if (lane == 0) {
      if (a.lse) a.lse[t] = lse;
      my_lse2 += (double)lse * (double)lse;
    }
    if (a.K > 0)
      tc_select_row<V>(key, s, ok, lane, E, a.K, a.n_groups, a.topk_groups, a.group_topn,
                       a.weights, a.idx + (size_t)t * a.K, a.gate + (size_t)t * a.K);
  }
#pragma unroll
  for (int v = 0; v < V; ++v) {
    const int cc = lane * V + v;
    if (cc < ET) colsum_w[warp * ET + cc] = csum[v];
  }
  if (lane == 0) lse2_w[warp] = my_lse2;
  __syncthreads();
  for (int cc = tid; cc < E; cc += 32 * NW) {
    float sum = 0.0f;
    for (int w = 0; w < NW; ++w) sum += colsum_w[w * ET + cc];
    a.colsum[(size_t)blockIdx.x * E + cc] = sum;
  }
  if (tid == 0) {
    double sum = 0.0;
    for (int w = 0; w < NW; ++w) sum += lse2_w[w];
    a.lse2[blockIdx.x] = sum;
  }
}

// ---------------------------------------------------------------------------
// Router GEMM + epilogue
// ---------------------------------------------------------------------------
template <class C, bool XBF16>
struct RouterSmem {
  static constexpr int XB = XBF16 ? 2 : 4;
  // The transposed A tile As[kk][row] keeps X's own type: bf16 X stays bf16
  // (each value widens exactly to fp32 when loaded), so a thread's rows come
  // in one vector load of half the bytes. A thread's TM rows sit together;
  // with bf16 an odd TM gets one padding slot (TMP = TM + 1) so the group
  // starts on an even element.
  static constexpr int TMP = (XBF16 && (C::TM % 2)) ? C::TM + 1 : C::TM;
  static constexpr int BMP = C::BM / C::TM * TMP;          // padded rows
  static constexpr int AST = BMP + (XBF16 ? 8 : 4);        // row stride, elements
  static constexpr size_t xs_bytes = (size_t)C::ST * C::BM * C::BK * XB;
  static constexpr size_t ws_bytes = (size_t)C::ST * C::BK * C::ET * 4;
  static constexpr size_t as_bytes = (size_t)C::BK * AST * XB;
  static constexpr size_t main_bytes = xs_bytes + ws_bytes + 2 * as_bytes;  // two A tiles
  static constexpr size_t epi_bytes =
      ((size_t)C::WK * C::BM * (C::ET + 1) + C::NW * C::ET) * 4 + C::NW * 8;
  static constexpr size_t bytes = (main_bytes > epi_bytes ? main_bytes : epi_bytes) + 128;
};

template <class C, bool XBF16>
__global__ void __launch_bounds__(C::NT) router_kernel(RouterArgs a) {
  pdl_wait();
  using SM = RouterSmem<C, XBF16>;
  constexpr int ET = C::ET, BM = C::BM, BK = C::BK, TM = C::TM, TN = C::TN;
  constexpr int XB = SM::XB, AST = SM::AST, TMP = SM::TMP;
  extern __shared__ __align__(16) unsigned char rsm[];
  unsigned char* Xs = rsm;                                        // [S][BM][BK] raw
  float* Ws = reinterpret_cast<float*>(rsm + SM::xs_bytes);       // [S][BK][ET]
  float* As = reinterpret_cast<float*>(rsm + SM::xs_bytes + SM::ws_bytes);  // [2][BK][AST] fp32
  uint16_t* As16 = reinterpret_cast<uint16_t*>(As);                         // [2][BK][AST] bf16

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int lx = lane / C::LY, ly = lane % C::LY;
  const int wk = warp / (C::WX * C::WY);
  const int wrem = warp % (C::WX * C::WY);
  const int wx = wrem / C::WY, wy = wrem % C::WY;
  const int row0 = (wx * C::LX + lx) * TM;
  const int arow0 = (wx * C::LX + lx) * TMP;  // the same rows in the (padded) A tile
  const int colb = wy * C::LY * TN + ly * 4;  // first column of group 0; group g adds g*4*LY
  const int m0 = blockIdx.x * BM;
  const int n = a.n, d = a.d, E = a.E;
  const bool w_vec = (E % 4 == 0);

  // accumulators in column pairs: one packed fp32x2 FMA (__ffma2_rn: a
  // single-rounding fma per element, so each logit is the same chain of
  // fmaf as one at a time) updates two of them per issue slot
  float2 acc[TM][TN / 2];
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < TN / 2; ++j) acc[i][j] = make_float2(0.0f, 0.0f);

  // Chunk c's loads, as parts that can be spread over the previous chunk's
  // FMA steps: part i < XIT copies 16-byte piece tid + i*NT of the X chunk
  // [BM][BK], the rest pieces of the W_g chunk [BK][ET] (4-float pieces when
  // E % 4 == 0, else single floats, all in part XIT).
  constexpr int XCH = BM * BK * XB / 16;          // 16-byte pieces of the X chunk
  constexpr int XPR = BK * XB / 16;               // pieces per row
  constexpr int XIT = (XCH + C::NT - 1) / C::NT;
  constexpr int WCH = BK * ET / 4;
  constexpr int WIT = (WCH + C::NT - 1) / C::NT;
  auto issue_part = [&](int c, int i) {
    const int st = c % C::ST;
    const int k0 = c * BK;
    if (i < XIT) {
      const int q = tid + i * C::NT;
      if (XCH % C::NT == 0 || q < XCH) {
        unsigned char* xs = Xs + (size_t)st * BM * BK * XB;
        const int r = q / XPR, p = q % XPR;
        const int row = m0 + r, k = k0 + p * (16 / XB);
        const bool ok = row < n && k < d;
        const char* src = static_cast<const char*>(a.X) +
                          ((size_t)(ok ? row : 0) * d + (ok ? k : 0)) * XB;
        cp_async16(xs + (size_t)r * BK * XB + p * 16, src, ok);
      }
      return;
    }
    float* ws = Ws + (size_t)st * BK * ET;
    if (w_vec) {
      const int q = tid + (i - XIT) * C::NT;
      if (WCH % C::NT == 0 || q < WCH) {
        const int kk = q / (ET / 4), c4 = (q % (ET / 4)) * 4;
        const int k = k0 + kk;
        const bool ok = k < d && c4 < E;
        cp_async16(ws + kk * ET + c4, a.Wg + (ok ? (size_t)k * E + c4 : 0), ok);
      }
    } else if (i == XIT) {
      for (int q = tid; q < BK * ET; q += C::NT) {
        const int kk = q / ET, cc = q % ET;
        const int k = k0 + kk;
        const bool ok = k < d && cc < E;
        cp_async4(ws + kk * ET + cc, a.Wg + (ok ? (size_t)k * E + cc : 0), ok);
      }
    }
  };
  // Part i of chunk c's transposition into its A tile (As buffer c % 2):
  // 16-byte piece tid + i*NT of the X chunk, written column-wise, As[kk][r]
  // (bf16 X stays bf16; fp32 X stays fp32).
  constexpr int EPP = 16 / XB;                     // elements per 16-byte piece
  constexpr int PCS = BM * BK / EPP;
  constexpr int TIT = (PCS + C::NT - 1) / C::NT;
  auto transpose_part = [&](int c, int i) {
    const int q = tid + i * C::NT;
    if (PCS % C::NT != 0 && q >= PCS) return;
    const unsigned char* xs = Xs + (size_t)(c % C::ST) * BM * BK * XB;
    const int r = q % BM, p = q / BM;
    const uint4 v = *reinterpret_cast<const uint4*>(xs + (size_t)r * BK * XB + p * 16);
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
    if (XBF16) {
      uint16_t* as16 = As16 + (size_t)(c & 1) * BK * AST;
      const int rr = r / TM * TMP + r % TM;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        as16[(p * 8 + 2 * j) * AST + rr] = (uint16_t)(w4[j] & 0xffffu);
        as16[(p * 8 + 2 * j + 1) * AST + rr] = (uint16_t)(w4[j] >> 16);
      }
    } else {
      float* as = As + (size_t)(c & 1) * BK * AST;
#pragma unroll
      for (int j = 0; j < 4; ++j) as[(p * 4 + j) * AST + r] = __uint_as_float(w4[j]);
    }
  };

  // this CTA's k range: all of d, or one of a.ksplit slices of it
  const int nchunks = (d + BK - 1) / BK;
  const int cb = (int)blockIdx.y * a.chunks_per_split;
  const int ce = min(nchunks, cb + a.chunks_per_split);
#pragma unroll 1
  for (int c = cb; c < cb + C::ST - 1; ++c) {
    if (c < ce)
      for (int i = 0; i < XIT + WIT; ++i) issue_part(c, i);
    cp_async_commit();
  }
  cp_async_wait<C::ST - 2>();
  __syncthreads();
  if (cb < ce)
    for (int i = 0; i < TIT; ++i) transpose_part(cb, i);
  // One barrier per chunk. At the top of chunk c: chunk c + 1 has landed,
  // chunk c's A tile is written, and every warp is done with chunk c - 1, so
  // its ring stage and A buffer are free. During chunk c's FMA steps each
  // thread transposes its pieces of chunk c + 1 and issues its copies of
  // chunk c + ST - 1 (into chunk c - 1's stage), a few per step, so that no
  // phase of the loop leaves the FMA pipe to itself.
  constexpr int QS = BK / C::WK;                  // FMA steps per warp per chunk
  constexpr int NPART = TIT + XIT + WIT;
#pragma unroll 1
  for (int c = cb; c < ce; ++c) {
    cp_async_wait<C::ST - 3>();
    __syncthreads();
    const bool do_t = c + 1 < ce, do_i = c + C::ST - 1 < ce;
    const float* ws = Ws + (size_t)(c % C::ST) * BK * ET;
    const uint16_t* as16 = As16 + (size_t)(c & 1) * BK * AST;
    const float* as = As + (size_t)(c & 1) * BK * AST;
#pragma unroll
    for (int q = 0; q < QS; ++q) {
#pragma unroll
      for (int i = (q * NPART + QS - 1) / QS; i < ((q + 1) * NPART + QS - 1) / QS; ++i) {
        if (i < TIT) {
          if (do_t) transpose_part(c + 1, i);
        } else if (do_i) {
          issue_part(c + C::ST - 1, i - TIT);
        }
      }
      const int kk = wk * QS + q;
      float av[TM], bv[TN];
      if constexpr (XBF16) {
        // the thread's TMP bf16 values: one 16- or 8-byte load, else 4-byte loads
        const uint16_t* ap = as16 + kk * AST + arow0;
        uint32_t w[TMP / 2];
        if constexpr (TMP == 8) {
          const uint4 t = *reinterpret_cast<const uint4*>(ap);
          w[0] = t.x;
          w[1] = t.y;
          w[2] = t.z;
          w[3] = t.w;
        } else if constexpr (TMP == 4) {
          const uint2 t = *reinterpret_cast<const uint2*>(ap);
          w[0] = t.x;
          w[1] = t.y;
        } else {
#pragma unroll
          for (int i = 0; i < TMP / 2; ++i) w[i] = reinterpret_cast<const uint32_t*>(ap)[i];
        }
#pragma unroll
        for (int i = 0; i < TM; ++i)
          av[i] = __uint_as_float(i % 2 ? (w[i / 2] & 0xffff0000u) : (w[i / 2] << 16));
      } else if (TM % 4 == 0) {
#pragma unroll
        for (int i4 = 0; i4 < TM / 4; ++i4) {
          const float4 t = *reinterpret_cast<const float4*>(as + kk * AST + row0 + 4 * i4);
          av[(4 * i4 + 0) % TM] = t.x;
          av[(4 * i4 + 1) % TM] = t.y;
          av[(4 * i4 + 2) % TM] = t.z;
          av[(4 * i4 + 3) % TM] = t.w;
        }
      } else if (TM % 2 == 0) {
#pragma unroll
        for (int i2 = 0; i2 < TM / 2; ++i2) {
          const float2 t = *reinterpret_cast<const float2*>(as + kk * AST + row0 + 2 * i2);
          av[(2 * i2) % TM] = t.x;
          av[(2 * i2 + 1) % TM] = t.y;
        }
      } else {
#pragma unroll
        for (int i = 0; i < TM; ++i) av[i] = as[kk * AST + row0 + i];
      }
#pragma unroll
      for (int g = 0; g < TN / 4; ++g) {
        const float4 t = *reinterpret_cast<const float4*>(ws + kk * ET + colb + g * 4 * C::LY);
        bv[4 * g + 0] = t.x;
        bv[4 * g + 1] = t.y;
        bv[4 * g + 2] = t.z;
        bv[4 * g + 3] = t.w;
      }
#pragma unroll
      for (int i = 0; i < TM; ++i) {
        const float2 a2 = make_float2(av[i], av[i]);
#pragma unroll
        for (int j = 0; j < TN / 2; ++j)
          acc[i][j] = __ffma2_rn(a2, make_float2(bv[2 * j], bv[2 * j + 1]), acc[i][j]);
      }
    }
    cp_async_commit();
  }
  cp_async_wait<0>();
  __syncthreads();

  // ---- epilogue: logits tile in shared memory ----
  constexpr int LST = ET + 1;
  float* Ls = reinterpret_cast<float*>(rsm);  // [WK][BM][LST]
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < TN; ++j)
      Ls[(wk * BM + row0 + i) * LST + colb + (j / 4) * 4 * C::LY + (j % 4)] =
          (j % 2) ? acc[i][j / 2].y : acc[i][j / 2].x;
  __syncthreads();
  if (C::WK > 1) {
    for (int q = tid; q < BM * ET; q += C::NT) {
      const int r = q / ET, cc = q % ET;
      float s = Ls[r * LST + cc];
#pragma unroll
      for (int w = 1; w < C::WK; ++w) s += Ls[(w * BM + r) * LST + cc];
      Ls[r * LST + cc] = s;
    }
    __syncthreads();
  }

  if (a.ksplit > 1) {
    // a k slice: its partial logits go to a.partial[slice][n][E]; the
    // reduce kernel sums the slices in order and runs the epilogue
    float* part = a.partial + (size_t)blockIdx.y * n * E;
    for (int q = tid; q < BM * E; q += C::NT) {
      const int r = q / E, cc = q % E;
      if (m0 + r < n) part[(size_t)(m0 + r) * E + cc] = Ls[r * LST + cc];
    }
    return;
  }
  float* colsum_w = Ls + C::WK * BM * LST;                          // [NW][ET]
  double* lse2_w = reinterpret_cast<double*>(colsum_w + C::NW * ET);  // [NW]
  router_rows_epilogue<ET, C::NW>(a, Ls, colsum_w, lse2_w, BM, m0);
}

// Split-k router, second pass: kRouterMinBlockRows (4) rows per CTA, so that
// the partials are read by many CTAs at once; each logit is the sum of the k
// slices' partials in slice order (fixed, so results are reproducible), then
// the common row epilogue.
template <int ET>
__global__ void __launch_bounds__(256) router_reduce_kernel(RouterArgs a) {
  pdl_wait();
  constexpr int LST = ET + 1, BMR = kRouterMinBlockRows;
  __shared__ float Ls[BMR * LST];
  __shared__ float colsum_w[8 * ET];
  __shared__ double lse2_w[8];
  const int n = a.n, E = a.E, m0 = blockIdx.x * BMR;
  if (E % 4 == 0) {
    const int E4 = E / 4;
    for (int q = threadIdx.x; q < BMR * E4; q += 256) {
      const int r = q / E4, c4 = (q % E4) * 4, t = m0 + r;
      float4 sum = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      if (t < n) {
#pragma unroll 8
        for (int k = 0; k < a.ksplit; ++k) {
          const float4 v = __ldcg(
              reinterpret_cast<const float4*>(a.partial + ((size_t)k * n + t) * E + c4));
          sum.x += v.x;
          sum.y += v.y;
          sum.z += v.z;
          sum.w += v.w;
        }
      }
      float* dst = Ls + r * LST + c4;
      dst[0] = sum.x;
      dst[1] = sum.y;
      dst[2] = sum.z;
      dst[3] = sum.w;
    }
  } else {
    for (int q = threadIdx.x; q < BMR * E; q += 256) {
      const int r = q / E, cc = q % E, t = m0 + r;
      float sum = 0.0f;
      if (t < n)
#pragma unroll 8
        for (int k = 0; k < a.ksplit; ++k) sum += __ldcg(a.partial + ((size_t)k * n + t) * E + cc);
      Ls[r * LST + cc] = sum;
    }
  }
  __syncthreads();
  router_rows_epilogue<ET, 8>(a, Ls, colsum_w, lse2_w, BMR, m0);
}

// k slices for a batch whose row tiles would fill fewer than half the SMs
// (small batches, decoding): enough slices to give every SM a CTA, each at
// least two chunks long, at most 32.
static int split_of(int ctas, int nchunks) {
  const int sms = num_sms_cached();
  if (ctas * 2 > sms) return 1;
  int ks = sms / ctas;
  if (ks > nchunks / 2) ks = nchunks / 2;
  if (ks > 32) ks = 32;
  return ks < 2 ? 1 : ks;
}

template <class C, bool XBF16>
static cudaError_t launch_router_t(const RouterArgs& a0, cudaStream_t s) {
  const size_t bytes = RouterSmem<C, XBF16>::bytes;
  auto kern = router_kernel<C, XBF16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)bytes);
  if (e != cudaSuccess) return e;
  const int grid = ceil_div(a0.n, C::BM);
  const int nchunks = ceil_div(a0.d, C::BK);
  RouterArgs a = a0;
  a.ksplit = router_ksplit(a.E, a.n, a.d, XBF16);
  a.chunks_per_split = ceil_div(nchunks, a.ksplit);
  if (a.ksplit > 1 && !a.partial) return cudaErrorInvalidValue;
  if (a.ksplit == 1) return launch_pdl(kern, grid, C::NT, bytes, s, a);
  e = launch_pdl(kern, dim3(grid, a.ksplit), C::NT, bytes, s, a);
  if (e != cudaSuccess) return e;
  return launch_pdl(router_reduce_kernel<C::ET>, ceil_div(a.n, kRouterMinBlockRows), 256, 0,
                    s, a);
}

template <template <int> class F>
static cudaError_t launch_family(int tm, const RouterArgs& a, cudaStream_t s) {
  switch (tm) {
    case 2: return launch_router_t<F<2>, true>(a, s);
    case 3: return launch_router_t<F<3>, true>(a, s);
    case 4: return launch_router_t<F<4>, true>(a, s);
    case 5: return launch_router_t<F<5>, true>(a, s);
    case 6: return launch_router_t<F<6>, true>(a, s);
    case 7: return launch_router_t<F<7>, true>(a, s);
    default: return launch_router_t<F<8>, true>(a, s);
  }
}

// families whose register budget stops at TM = 7 (12 warps)
template <template <int> class F>
static cudaError_t launch_family_upto7(int tm, const RouterArgs& a, cudaStream_t s) {
  switch (tm) {
    case 4: return launch_router_t<F<4>, true>(a, s);
    case 5: return launch_router_t<F<5>, true>(a, s);
    case 6: return launch_router_t<F<6>, true>(a, s);
    default: return launch_router_t<F<7>, true>(a, s);
  }
}

static cudaError_t launch_router_bf16_family(int code, const RouterArgs& a, cudaStream_t s) {
  const int fam = code / 16, tm = code % 16;
  switch (fam) {
    case 1: return launch_family<R64A>(tm, a, s);
    case 2: return launch_family<R64C>(tm, a, s);
    case 3: return launch_family<R128A>(tm, a, s);
    case 4: return launch_family<R256A>(tm, a, s);
    case 5: return launch_family<R256B>(tm, a, s);
    case 6: return launch_family_upto7<R256C>(tm, a, s);
    default: return launch_family<R64D>(tm, a, s);
  }
}

template <bool XBF16>
static cudaError_t launch_router_dt(const RouterArgs& a, cudaStream_t s) {
  const int v = router_variant(a.E, a.n, XBF16);
  if constexpr (XBF16) {
    if (v >= kFamilyCode) return launch_router_bf16_family(v - kFamilyCode, a, s);
    return v == 8 ? launch_router_t<R8, true>(a, s) : launch_router_t<R32, true>(a, s);
  } else {
    switch (v) {
      case 8: return launch_router_t<R8, false>(a, s);
      case 32: return launch_router_t<R32, false>(a, s);
      case 64: return launch_router_t<R64, false>(a, s);
      case 65: return launch_router_t<R64s, false>(a, s);
      case 128: return launch_router_t<R128, false>(a, s);
      case 256: return launch_router_t<R256, false>(a, s);
      default: return launch_router_t<R256s, false>(a, s);
    }
  }
}

cudaError_t launch_router(const RouterArgs& a, cudaStream_t s) {
  return a.x_bf16 ? launch_router_dt<true>(a, s) : launch_router_dt<false>(a, s);
}


// ---------------------------------------------------------------------------
// Token-choice selection from a given score matrix (one warp per row).
// Uses the same tc_select_row as the fused router epilogue, so identical S
// gives identical selections.
// ---------------------------------------------------------------------------
template <int V>
__global__ void __launch_bounds__(256) select_tc_kernel(SelectTcArgs a) {
  pdl_wait();
  __shared__ float colsum_w[8][V * 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int rows_per_block = 8 * kSelectRowsPerWarp;
  const int E = a.E;
  float csum[V];
#pragma unroll
  for (int v = 0; v < V; ++v) csum[v] = 0.0f;
  for (int q = 0; q < kSelectRowsPerWarp; ++q) {
    const int t = blockIdx.x * rows_per_block + warp * kSelectRowsPerWarp + q;
    if (t >= a.n) break;
    float s[V], key[V];
    bool ok[V];
#pragma unroll
    for (int v = 0; v < V; ++v) {
      const int cc = lane * V + v;
      ok[v] = cc < E;
      s[v] = ok[v] ? a.S[(size_t)t * E + cc] : 0.0f;
      if (ok[v] && a.scores_copy) a.scores_copy[(size_t)t * E + cc] = s[v];
      key[v] = ok[v] ? (a.sel_bias ? s[v] + a.sel_bias[cc] : s[v]) : 0.0f;
      csum[v] += s[v];
    }
    tc_select_row<V>(key, s, ok, lane, E, a.K, a.n_groups, a.topk_groups, a.group_topn,
                     a.weights, a.idx + (size_t)t * a.K, a.gate + (size_t)t * a.K);
  }
#pragma unroll
  for (int v = 0; v < V; ++v) colsum_w[warp][lane * V + v] = csum[v];
  __syncthreads();
  for (int cc = threadIdx.x; cc < E; cc += 256) {
    float sum = 0.0f;
    for (int w = 0; w < 8; ++w) sum += colsum_w[w][cc];
    a.colsum[(size_t)blockIdx.x * E + cc] = sum;
  }
}

cudaError_t launch_select_tc(const SelectTcArgs& a, cudaStream_t s) {
  const int grid = ceil_div(a.n, select_tc_block_rows());
  const int et = router_tile_et(a.E);
  switch (et) {
    case 8:
    case 32: return launch_pdl(select_tc_kernel<1>, grid, 256, 0, s, a);
    case 64: return launch_pdl(select_tc_kernel<2>, grid, 256, 0, s, a);
    case 128: return launch_pdl(select_tc_kernel<4>, grid, 256, 0, s, a);
    default: return launch_pdl(select_tc_kernel<8>, grid, 256, 0, s, a);
  }
}

}  // namespace moe
