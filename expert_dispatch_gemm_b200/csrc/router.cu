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
#include <math.h>

#include "device_common.cuh"
#include "moe_internal.h"

namespace moe {

// Per-thread TM x TN outputs; LX x LY lanes per warp; WX x WY x WK warps
// (WK splits each K chunk; partial sums are reduced in a fixed order).
template <int ET>
struct RouterTile;
template <>
struct RouterTile<8> {
  static constexpr int TM = 1, TN = 8, LX = 32, LY = 1, WX = 1, WY = 1, WK = 8;
};
template <>
struct RouterTile<32> {
  static constexpr int TM = 2, TN = 4, LX = 4, LY = 8, WX = 4, WY = 1, WK = 2;
};
template <>
struct RouterTile<64> {
  static constexpr int TM = 2, TN = 8, LX = 4, LY = 8, WX = 8, WY = 1, WK = 1;
};
template <>
struct RouterTile<128> {
  static constexpr int TM = 2, TN = 8, LX = 4, LY = 8, WX = 4, WY = 2, WK = 1;
};
template <>
struct RouterTile<256> {
  static constexpr int TM = 4, TN = 8, LX = 4, LY = 8, WX = 2, WY = 4, WK = 1;
};

constexpr int kRouterBK = 32;
constexpr int kSelectRowsPerWarp = 4;

int router_tile_et(int E) {
  return E <= 8 ? 8 : E <= 32 ? 32 : E <= 64 ? 64 : E <= 128 ? 128 : 256;
}

template <int ET>
constexpr int router_bm() {
  return RouterTile<ET>::WX * RouterTile<ET>::LX * RouterTile<ET>::TM;
}

int router_block_rows(int E) {
  switch (router_tile_et(E)) {
    case 8: return router_bm<8>();
    case 32: return router_bm<32>();
    case 64: return router_bm<64>();
    case 128: return router_bm<128>();
    default: return router_bm<256>();
  }
}

int select_tc_block_rows() { return 8 * kSelectRowsPerWarp; }

// ---------------------------------------------------------------------------
// Token-choice selection of one row by one warp. Lane l holds experts
// l*V .. l*V+V-1 (contiguous, so a group of gs experts is gs/V lanes).
// Order: key desc, expert asc. Group score: fp32 sum of the group_topn
// largest keys, largest first; groups ranked by (score desc, group asc).
// Weights always come from the raw scores.
// ---------------------------------------------------------------------------
template <int V>
__device__ __forceinline__ void tc_select_row(const float (&key)[V], const float (&raw)[V],
                                              const bool (&ok)[V], int lane, int E, int K,
                                              int n_groups, int topk_groups, int group_topn,
                                              int weights, int32_t* idx_out,
                                              float* gate_out) {
  bool allowed[V];
#pragma unroll
  for (int v = 0; v < V; ++v) allowed[v] = ok[v];
  if (n_groups > 1) {
    const int gs = E / n_groups;
    const int lpg = gs / V;
    const int g = (lane * V) / gs;
    bool taken[V];
#pragma unroll
    for (int v = 0; v < V; ++v) taken[v] = false;
    float gsum = 0.0f;
    for (int r = 0; r < group_topn; ++r) {
      Cand c{0.0f, 0, false};
#pragma unroll
      for (int v = 0; v < V; ++v) {
        Cand x{key[v], lane * V + v, allowed[v] && !taken[v]};
        if (cand_better(x, c)) c = x;
      }
      c = group_best(c, lpg);
      if (c.valid) gsum = gsum + c.key;
#pragma unroll
      for (int v = 0; v < V; ++v)
        if (c.valid && c.idx == lane * V + v) taken[v] = true;
    }
    bool gsel = false;
    const bool gvalid = g < n_groups;
    for (int r = 0; r < topk_groups; ++r) {
      Cand c{gsum, g, gvalid && !gsel};
      c = group_best(c, 32);
      if (c.valid && c.idx == g) gsel = true;
    }
#pragma unroll
    for (int v = 0; v < V; ++v) allowed[v] = allowed[v] && gsel;
  }
  bool picked[V];
#pragma unroll
  for (int v = 0; v < V; ++v) picked[v] = false;
  int my_e = -1;
  float my_raw = 0.0f;
  for (int j = 0; j < K; ++j) {
    Cand c{0.0f, 0, false};
#pragma unroll
    for (int v = 0; v < V; ++v) {
      Cand x{key[v], lane * V + v, allowed[v] && !picked[v]};
      if (cand_better(x, c)) c = x;
    }
    c = group_best(c, 32);
    float rv = 0.0f;
#pragma unroll
    for (int v = 0; v < V; ++v)
      if (c.valid && c.idx == lane * V + v) {
        picked[v] = true;
        rv = raw[v];
      }
    const int owner = c.valid ? c.idx / V : 0;
    rv = __shfl_sync(0xffffffffu, rv, owner);
    if (lane == j) {
      my_e = c.valid ? c.idx : -1;
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
// Router GEMM + epilogue
// ---------------------------------------------------------------------------
template <int ET, bool XBF16>
__global__ void __launch_bounds__(256) router_kernel(RouterArgs a) {
  using T = RouterTile<ET>;
  constexpr int BM = router_bm<ET>();
  constexpr int BK = kRouterBK;
  constexpr int AST = BM + 4;  // As row stride (floats)
  constexpr int V = ET >= 32 ? ET / 32 : 1;
  extern __shared__ __align__(16) float smem[];
  float* As = smem;                 // [2][BK][AST]
  float* Bs = As + 2 * BK * AST;    // [2][BK][ET]

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int lx = lane / T::LY, ly = lane % T::LY;
  const int wk = warp / (T::WX * T::WY);
  const int wrem = warp % (T::WX * T::WY);
  const int wx = wrem / T::WY, wy = wrem % T::WY;
  const int row0 = (wx * T::LX + lx) * T::TM;
  const int col0 = (wy * T::LY + ly) * T::TN;
  const int m0 = blockIdx.x * BM;
  const int n = a.n, d = a.d, E = a.E;

  constexpr int XV = XBF16 ? 8 : 4;             // elements per 16-byte vector
  constexpr int XVEC = BM * BK / XV;
  constexpr int XPT = (XVEC + 255) / 256;
  constexpr int WPT = (BK * ET + 255) / 256;        // scalar Wg loads per thread
  constexpr int WV4 = (BK * ET / 4 + 255) / 256;    // float4 Wg loads per thread
  constexpr int WREG = WPT > 4 * WV4 ? WPT : 4 * WV4;
  const bool w_vec = (E % 4 == 0);

  float acc[T::TM][T::TN];
#pragma unroll
  for (int i = 0; i < T::TM; ++i)
#pragma unroll
    for (int j = 0; j < T::TN; ++j) acc[i][j] = 0.0f;

  uint4 xr[XPT];
  float wr[WREG];

  auto load_regs = [&](int kb) {
#pragma unroll
    for (int i = 0; i < XPT; ++i) {
      const int v = tid + i * 256;
      xr[i] = make_uint4(0, 0, 0, 0);
      if (v < XVEC) {
        const int r = v / (BK / XV), kv = v % (BK / XV);
        const int row = m0 + r, k = kb + kv * XV;
        if (row < n && k < d) {
          const char* base = reinterpret_cast<const char*>(a.X);
          const size_t off = ((size_t)row * d + k) * (XBF16 ? 2 : 4);
          xr[i] = __ldg(reinterpret_cast<const uint4*>(base + off));
        }
      }
    }
    if (w_vec) {
#pragma unroll
      for (int i = 0; i < WV4; ++i) {
        const int v = tid + i * 256;  // float4 index in the [BK][ET] tile
        if (v < BK * ET / 4) {
          const int kk = v / (ET / 4), c = (v % (ET / 4)) * 4;
          const int k = kb + kk;
          float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
          if (k < d && c < E) f = __ldg(reinterpret_cast<const float4*>(a.Wg + (size_t)k * E + c));
          wr[4 * i + 0] = f.x;
          wr[4 * i + 1] = f.y;
          wr[4 * i + 2] = f.z;
          wr[4 * i + 3] = f.w;
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < WPT; ++i) {
        const int v = tid + i * 256;
        wr[i] = 0.0f;
        if (v < BK * ET) {
          const int kk = v / ET, c = v % ET;
          const int k = kb + kk;
          if (k < d && c < E) wr[i] = __ldg(a.Wg + (size_t)k * E + c);
        }
      }
    }
  };

  auto store_smem = [&](int buf) {
    float* as = As + buf * BK * AST;
    float* bs = Bs + buf * BK * ET;
#pragma unroll
    for (int i = 0; i < XPT; ++i) {
      const int v = tid + i * 256;
      if (v < XVEC) {
        const int r = v / (BK / XV), kv = v % (BK / XV);
        if (XBF16) {
          const uint32_t w4[4] = {xr[i].x, xr[i].y, xr[i].z, xr[i].w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            as[(kv * XV + 2 * j) * AST + r] = __uint_as_float(w4[j] << 16);
            as[(kv * XV + 2 * j + 1) * AST + r] = __uint_as_float(w4[j] & 0xffff0000u);
          }
        } else {
          as[(kv * XV + 0) * AST + r] = __uint_as_float(xr[i].x);
          as[(kv * XV + 1) * AST + r] = __uint_as_float(xr[i].y);
          as[(kv * XV + 2) * AST + r] = __uint_as_float(xr[i].z);
          as[(kv * XV + 3) * AST + r] = __uint_as_float(xr[i].w);
        }
      }
    }
    if (w_vec) {
#pragma unroll
      for (int i = 0; i < WV4; ++i) {
        const int v = tid + i * 256;
        if (v < BK * ET / 4) {
          *reinterpret_cast<float4*>(bs + v * 4) =
              make_float4(wr[4 * i], wr[4 * i + 1], wr[4 * i + 2], wr[4 * i + 3]);
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < WPT; ++i) {
        const int v = tid + i * 256;
        if (v < BK * ET) bs[v] = wr[i];
      }
    }
  };

  const int nchunks = (d + BK - 1) / BK;
  load_regs(0);
  store_smem(0);
  __syncthreads();
  for (int c = 0; c < nchunks; ++c) {
    if (c + 1 < nchunks) load_regs((c + 1) * BK);
    const float* as = As + (c & 1) * BK * AST;
    const float* bs = Bs + (c & 1) * BK * ET;
#pragma unroll
    for (int q = 0; q < BK / T::WK; ++q) {
      const int kk = wk * (BK / T::WK) + q;
      float av[T::TM], bv[T::TN];
#pragma unroll
      for (int i = 0; i < T::TM; ++i) av[i] = as[kk * AST + row0 + i];
#pragma unroll
      for (int j = 0; j < T::TN; ++j) bv[j] = bs[kk * ET + col0 + j];
#pragma unroll
      for (int i = 0; i < T::TM; ++i)
#pragma unroll
        for (int j = 0; j < T::TN; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    if (c + 1 < nchunks) store_smem((c + 1) & 1);
    __syncthreads();
  }

  // ---- epilogue: logits tile in shared memory ----
  constexpr int LST = ET + 1;
  float* Ls = smem;  // [WK][BM][LST]
#pragma unroll
  for (int i = 0; i < T::TM; ++i)
#pragma unroll
    for (int j = 0; j < T::TN; ++j) Ls[(wk * BM + row0 + i) * LST + col0 + j] = acc[i][j];
  __syncthreads();
  if (T::WK > 1) {
    for (int q = tid; q < BM * ET; q += 256) {
      const int r = q / ET, cc = q % ET;
      float s = Ls[r * LST + cc];
#pragma unroll
      for (int w = 1; w < T::WK; ++w) s += Ls[(w * BM + r) * LST + cc];
      Ls[r * LST + cc] = s;
    }
    __syncthreads();
  }

  float* colsum_w = smem + T::WK * BM * LST;              // [8][ET]
  double* lse2_w = reinterpret_cast<double*>(colsum_w + 8 * ET);  // [8]
  float csum[V];
#pragma unroll
  for (int v = 0; v < V; ++v) csum[v] = 0.0f;
  double my_lse2 = 0.0;

  for (int r = warp; r < BM; r += 8) {
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
      if (a.score == MOE_SCORE_SIGMOID)
        s[v] = ok[v] ? 1.0f / (1.0f + expf(-l[v])) : 0.0f;
      else
        s[v] = ex[v] / z;
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
  for (int cc = tid; cc < E; cc += 256) {
    float s = 0.0f;
    for (int w = 0; w < 8; ++w) s += colsum_w[w * ET + cc];
    a.colsum[(size_t)blockIdx.x * E + cc] = s;
  }
  if (tid == 0) {
    double s = 0.0;
    for (int w = 0; w < 8; ++w) s += lse2_w[w];
    a.lse2[blockIdx.x] = s;
  }
}

template <int ET, bool XBF16>
static cudaError_t launch_router_t(const RouterArgs& a, cudaStream_t s) {
  using T = RouterTile<ET>;
  constexpr int BM = router_bm<ET>();
  const size_t main_f = 2 * kRouterBK * (BM + 4) + 2 * kRouterBK * ET;
  const size_t epi_f = (size_t)T::WK * BM * (ET + 1) + 8 * ET + 2 * 8;
  const size_t bytes = (main_f > epi_f ? main_f : epi_f) * sizeof(float) + 64;
  auto kern = router_kernel<ET, XBF16>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)bytes);
  if (e != cudaSuccess) return e;
  const int grid = ceil_div(a.n, BM);
  kern<<<grid, 256, bytes, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_router(const RouterArgs& a, cudaStream_t s) {
  const int et = router_tile_et(a.E);
  if (a.x_bf16) {
    switch (et) {
      case 8: return launch_router_t<8, true>(a, s);
      case 32: return launch_router_t<32, true>(a, s);
      case 64: return launch_router_t<64, true>(a, s);
      case 128: return launch_router_t<128, true>(a, s);
      default: return launch_router_t<256, true>(a, s);
    }
  }
  switch (et) {
    case 8: return launch_router_t<8, false>(a, s);
    case 32: return launch_router_t<32, false>(a, s);
    case 64: return launch_router_t<64, false>(a, s);
    case 128: return launch_router_t<128, false>(a, s);
    default: return launch_router_t<256, false>(a, s);
  }
}

// ---------------------------------------------------------------------------
// Token-choice selection from a given score matrix (one warp per row).
// Uses the same tc_select_row as the fused router epilogue, so identical S
// gives identical selections.
// ---------------------------------------------------------------------------
template <int V>
__global__ void __launch_bounds__(256) select_tc_kernel(SelectTcArgs a) {
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
    case 32: select_tc_kernel<1><<<grid, 256, 0, s>>>(a); break;
    case 64: select_tc_kernel<2><<<grid, 256, 0, s>>>(a); break;
    case 128: select_tc_kernel<4><<<grid, 256, 0, s>>>(a); break;
    default: select_tc_kernel<8><<<grid, 256, 0, s>>>(a); break;
  }
  return cudaGetLastError();
}

}  // namespace moe
