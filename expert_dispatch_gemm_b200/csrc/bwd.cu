// Element-wise and FFMA kernels of the layer's backward pass: the combine's
// backward with the mixing-weight, score and aux-loss gradients fused in, the
// padding-row clear that the weight gradients rely on, and the router's
// backward (input gradient fused with the sum over each token's dispatched
// rows; router-weight gradient with an ordered split over the tokens).
//
// "Expert choice routing" (aicassindra.com), "The math: a gating matrix and
// top-k over tokens": out = scatter_add(G * Expert(X_in)), so for each pair
// (token t, gate g) the output gradient reaches the expert as g * dout[t]
// and the gate's gradient is <dout[t], Y_pair>. "Token choice vs expert
// choice routing in MoE", "What each direction guarantees": the balance loss
// and the router z-loss add their gradients at the scores and the logits.
#include <math.h>

#include "device_common.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// 16 bytes of T as floats (bf16: 8, fp32: 4)
template <typename T>
struct V16;
template <>
struct V16<__nv_bfloat16> {
  static constexpr int W = 8;
  __device__ static void unpack(const uint4 x, float* f) {
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = bf_lo(w[i]);
      f[2 * i + 1] = bf_hi(w[i]);
    }
  }
  __device__ static uint4 pack(const float* f) {
    return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                      pack_bf16x2(f[6], f[7]));
  }
};
template <>
struct V16<float> {
  static constexpr int W = 4;
  __device__ static void unpack(const uint4 x, float* f) {
    f[0] = __uint_as_float(x.x);
    f[1] = __uint_as_float(x.y);
    f[2] = __uint_as_float(x.z);
    f[3] = __uint_as_float(x.w);
  }
  __device__ static uint4 pack(const float* f) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
  }
};

// four consecutive elements (8 bytes of bf16, 16 of fp32)
__device__ __forceinline__ void load4(const __nv_bfloat16* p, float* f) {
  const uint2 x = *reinterpret_cast<const uint2*>(p);
  f[0] = bf_lo(x.x);
  f[1] = bf_hi(x.x);
  f[2] = bf_lo(x.y);
  f[3] = bf_hi(x.y);
}
__device__ __forceinline__ void load4(const float* p, float* f) {
  const float4 x = *reinterpret_cast<const float4*>(p);
  f[0] = x.x;
  f[1] = x.y;
  f[2] = x.z;
  f[3] = x.w;
}
__device__ __forceinline__ void store4(__nv_bfloat16* p, const float* f) {
  *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]));
}
__device__ __forceinline__ void store4(float* p, const float* f) {
  *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
}
__device__ __forceinline__ void load2(const __nv_bfloat16* p, float& lo, float& hi) {
  const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
  lo = bf_lo(w);
  hi = bf_hi(w);
}
__device__ __forceinline__ void load2(const float* p, float& lo, float& hi) {
  const float2 w = *reinterpret_cast<const float2*>(p);
  lo = w.x;
  hi = w.y;
}

// sum over the block (256 threads); every thread gets the total
__device__ __forceinline__ float block_sum256(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();  // red[] free from any previous use
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = 0.0f;
#pragma unroll
  for (int w = 0; w < 8; ++w) t += red[w];  // fixed order: the same on every thread
  return t;
}

// One CTA per token. For each kept slot (row r, gate g): dY_perm[r] =
// bf16(g * dout[t]) and dgate = <dout[t], Y_perm[r]> (fp32). Then the
// token's logit gradient: the mixing weights' backward (raw: dS = dgate;
// normalised w = s / sum s: dS_k = (dw_k - sum_j w_j dw_j) / sum s; expert
// choice: dS[t, e] = dgate), the balance-loss term lb E f_e / n
// (f_e = load_e / (n K)), the score's backward and the z-loss term
// 2 z lse_t / n softmax(l_t).
template <typename T>
__global__ void __launch_bounds__(256) combine_backward_kernel(CombineBwdArgs a) {
  pdl_wait();
  __shared__ int rows_s[MOE_MAX_EXPERTS];
  __shared__ float gates_s[MOE_MAX_EXPERTS];
  __shared__ float dots_s[MOE_MAX_EXPERTS];
  __shared__ float dS_s[MOE_MAX_EXPERTS];
  __shared__ float red[8];
  __shared__ int cnt_s;
  const int t = blockIdx.x, tid = threadIdx.x;
  const int slots = a.slots;
  if (tid == 0) cnt_s = slots;
  for (int e = tid; e < a.E; e += 256) dS_s[e] = 0.0f;
  __syncthreads();
  for (int j = tid; j < slots; j += 256) {
    int r = a.tok_row[(size_t)t * slots + j];
    if (r < -1 || r >= a.max_rows) {
      bad_index(a.err, kSiteBwdTokRow);
      r = -1;
    }
    rows_s[j] = r;
    gates_s[j] = a.tok_gate[(size_t)t * slots + j];
    if (r < 0) atomicMin(&cnt_s, j);
  }
  __syncthreads();
  const int cnt = cnt_s;
  constexpr int W = V16<T>::W;
  const int nvec = a.d / W;
  const uint4* go = reinterpret_cast<const uint4*>(a.dout) + (size_t)t * nvec;
  for (int j = 0; j < cnt; ++j) {
    const long long r = rows_s[j];
    const float g = gates_s[j];
    const uint4* y = reinterpret_cast<const uint4*>(a.Y_perm) + (size_t)r * nvec;
    uint4* dy = reinterpret_cast<uint4*>(a.dY_perm) + (size_t)r * nvec;
    float part = 0.0f;
    for (int v = tid; v < nvec; v += 256) {
      float o[W], yy[W], res[W];
      V16<T>::unpack(__ldg(go + v), o);
      V16<T>::unpack(__ldg(y + v), yy);
#pragma unroll
      for (int i = 0; i < W; ++i) {
        part = fmaf(o[i], yy[i], part);
        res[i] = g * o[i];
      }
      dy[v] = V16<T>::pack(res);
    }
    const float dot = block_sum256(part, red);
    if (tid == 0) dots_s[j] = dot;
  }
  __syncthreads();
  // scatter the gate gradients onto the score row
  if (tid == 0) {
    if (a.tc) {
      const int32_t* it = a.idx + (size_t)t * a.K;
      const uint8_t* dr = a.drop + (size_t)t * a.K;
      const float* s = a.scores + (size_t)t * a.E;
      float dw[MOE_MAX_TOPK];
      int kept = 0;
      for (int j = 0; j < a.K; ++j) dw[j] = dr[j] ? 0.0f : dots_s[kept++];
      if (a.weights == MOE_W_NORMALIZED) {
        float sum = 0.0f, dot = 0.0f;
        for (int j = 0; j < a.K; ++j) sum += s[it[j]];
        for (int j = 0; j < a.K; ++j) dot = fmaf(s[it[j]] / sum, dw[j], dot);
        for (int j = 0; j < a.K; ++j) dS_s[it[j]] += (dw[j] - dot) / sum;
      } else {
        for (int j = 0; j < a.K; ++j) dS_s[it[j]] += dw[j];
      }
    } else {
      for (int j = 0; j < cnt; ++j) {
        const int r = rows_s[j];
        int lo = 0, hi = a.E - 1;  // the expert whose segment holds row r
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (a.offsets[mid] <= r) lo = mid; else hi = mid - 1;
        }
        dS_s[lo] += dots_s[j];
      }
    }
  }
  __syncthreads();
  const int e = tid;
  float ds = 0.0f, s = 0.0f;
  if (e < a.E) {
    ds = dS_s[e];
    if (a.tc && a.lb_coef != 0.0f)
      ds += a.lb_coef * (float)a.E * ((float)a.load[e] / ((float)a.n * (float)a.K)) / (float)a.n;
    s = a.scores[(size_t)t * a.E + e];
  }
  float dl;
  if (a.score == MOE_SCORE_SOFTMAX) {
    const float dot = block_sum256(e < a.E ? s * ds : 0.0f, red);
    dl = s * (ds - dot);
  } else if (a.score == MOE_SCORE_SIGMOID) {
    dl = ds * s * (1.0f - s);
  } else {
    // s = sqrt(softplus(l)): ds/dl = sigmoid(l) / (2 s)
    const float l = e < a.E ? a.logits[(size_t)t * a.E + e] : 0.0f;
    dl = e < a.E ? ds * (1.0f / (1.0f + __expf(-l))) / (2.0f * s) : 0.0f;
  }
  if (e < a.E) {
    if (a.tc && a.z_coef != 0.0f) {
      const float lse = a.lse[t];
      const float l = a.logits[(size_t)t * a.E + e];
      dl += a.z_coef * 2.0f * lse / (float)a.n * __expf(l - lse);
    }
    a.dL[(size_t)t * a.E + e] = dl;
  }
}

// zero rows [offsets[e] + counts[e], offsets[e+1]) of two [rows, row_bytes] buffers
__global__ void __launch_bounds__(256) pad_zero_kernel(const int32_t* offsets,
                                                       const int32_t* counts, int row_bytes,
                                                       void* a, void* b) {
  pdl_wait();
  const int e = blockIdx.x;
  const int beg = offsets[e], end = offsets[e + 1];
  const int first = beg + max(0, min(counts[e], end - beg));
  const int nvec = row_bytes / 16;
  const long long total = (long long)(end - first) * nvec;
  const uint4 z = make_uint4(0, 0, 0, 0);
  for (long long q = threadIdx.x; q < total; q += 256) {
    const size_t off = (size_t)first * nvec + q;
    reinterpret_cast<uint4*>(a)[off] = z;
    if (b) reinterpret_cast<uint4*>(b)[off] = z;
  }
}

// WgT[e, i] = Wg[i, e], through 32 x 32 shared-memory tiles, so that the
// input-gradient tiles below read rows of W_g^T with consecutive threads on
// consecutive addresses
__global__ void __launch_bounds__(256) transpose_wg_kernel(const float* Wg, int d, int E,
                                                           float* WgT) {
  pdl_wait();
  __shared__ float tile[32][33];
  const int i0 = blockIdx.x * 32, e0 = blockIdx.y * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int r = ty; r < 32; r += 8) {
    const int i = i0 + r, e = e0 + tx;
    tile[r][tx] = (i < d && e < E) ? Wg[(size_t)i * E + e] : 0.0f;
  }
  __syncthreads();
  for (int r = ty; r < 32; r += 8) {
    const int e = e0 + r, i = i0 + tx;
    if (e < E && i < d) WgT[(size_t)e * d + i] = tile[tx][r];
  }
}

// dX[t, i] = sum_e dL[t, e] Wg[i, e] + sum over the token's dispatched rows
// of dX_perm[row, i] (+ the shared experts' rows), fp32, stored bf16.
// Tile: 64 tokens x 128 columns, experts in chunks of 32; thread (ty, tx)
// holds tokens 8ty..8ty+7 and columns 4tx..4tx+3, so each expert step takes
// three 16-byte shared-memory loads for 32 FMAs, issued as 16 packed fp32x2
// FMAs (__ffma2_rn: each element rounds once, as fmaf would).
constexpr int kRxBM = 64, kRxBN = 128, kRxEC = 32;
template <typename T>
__global__ void __launch_bounds__(256) router_dx_kernel(RouterBwdArgs a) {
  pdl_wait();
  __shared__ __align__(16) float dls[kRxEC][kRxBM + 4];  // transposed: [expert][token]
  __shared__ __align__(16) float wts[kRxEC][kRxBN];      // [expert][column]
  const int tid = threadIdx.x, tx = tid & 31, ty = tid >> 5;
  const int t0 = blockIdx.x * kRxBM, i0 = blockIdx.y * kRxBN;
  float2 acc[8][2];
#pragma unroll
  for (int k = 0; k < 8; ++k)
#pragma unroll
    for (int c = 0; c < 2; ++c) acc[k][c] = make_float2(0.0f, 0.0f);
  for (int e0 = 0; e0 < a.E; e0 += kRxEC) {
    __syncthreads();
    for (int q = tid; q < kRxBM * kRxEC; q += 256) {
      const int r = q / kRxEC, c = q % kRxEC;  // consecutive threads: consecutive experts
      const int t = t0 + r, e = e0 + c;
      dls[c][r] = (t < a.n && e < a.E) ? a.dL[(size_t)t * a.E + e] : 0.0f;
    }
    for (int q = tid; q < kRxBN * kRxEC; q += 256) {
      const int i = q % kRxBN, c = q / kRxBN;  // consecutive threads: consecutive columns
      const int gi = i0 + i, e = e0 + c;
      wts[c][i] = (gi < a.d && e < a.E) ? a.WgT[(size_t)e * a.d + gi] : 0.0f;
    }
    __syncthreads();
#pragma unroll 8
    for (int c = 0; c < kRxEC; ++c) {
      const float4 w = *reinterpret_cast<const float4*>(&wts[c][4 * tx]);
      const float4 g0 = *reinterpret_cast<const float4*>(&dls[c][8 * ty]);
      const float4 g1 = *reinterpret_cast<const float4*>(&dls[c][8 * ty + 4]);
      const float g[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
      const float2 w01 = make_float2(w.x, w.y), w23 = make_float2(w.z, w.w);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float2 gg = make_float2(g[k], g[k]);
        acc[k][0] = __ffma2_rn(gg, w01, acc[k][0]);
        acc[k][1] = __ffma2_rn(gg, w23, acc[k][1]);
      }
    }
  }
  const int col = i0 + 4 * tx;
  if (col >= a.d) return;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int t = t0 + 8 * ty + k;
    if (t >= a.n) continue;
    float v[4] = {acc[k][0].x, acc[k][0].y, acc[k][1].x, acc[k][1].y};
    const T* xp = static_cast<const T*>(a.dX_perm);
    auto add = [&](const float* x) {
      v[0] += x[0];
      v[1] += x[1];
      v[2] += x[2];
      v[3] += x[3];
    };
    // the token's rows four at a time, so that four independent loads are in
    // flight (sums stay in slot order)
    const int32_t* tr = a.tok_row + (size_t)t * a.slots;
    for (int j = 0; j < a.slots; j += 4) {
      int r[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        r[u] = j + u < a.slots ? tr[j + u] : -1;
        if (r[u] < -1 || r[u] >= a.max_rows) {
          bad_index(a.err, kSiteBwdTokRow);
          r[u] = -1;
        }
      }
      float x[4][4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (r[u] >= 0) load4(xp + (size_t)r[u] * a.d + col, x[u]);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (r[u] >= 0) add(x[u]);
      if (r[3] < 0) break;
    }
    for (int sidx = 0; sidx < a.n_shared; ++sidx) {
      float x[4];
      load4(xp + (size_t)(a.shared_base + sidx * a.n_pad + t) * a.d + col, x);
      add(x);
    }
    store4(static_cast<T*>(a.dX) + (size_t)t * a.d + col, v);
  }
}

// dWg[i, e] = sum_t X[t, i] dL[t, e]. Tile 128 (i) x 64 (e), tokens in
// chunks of 32; thread (ti, te) holds rows 8ti..8ti+7 and experts
// 4te..4te+3 (packed fp32x2 FMAs over expert pairs). blockIdx.z = a
// contiguous slice of the tokens; slices are added in slice order by
// router_dwg_reduce_kernel.
constexpr int kRwBM = 128, kRwBN = 64, kRwBT = 32;
template <typename T>
__global__ void __launch_bounds__(256) router_dwg_kernel(RouterBwdArgs a, int per_split) {
  pdl_wait();
  __shared__ __align__(16) float xs[kRwBT][kRwBM];
  __shared__ __align__(16) float ls[kRwBT][kRwBN];
  const int tid = threadIdx.x, te = tid & 15, ti = tid >> 4;
  const int i0 = blockIdx.x * kRwBM, e0 = blockIdx.y * kRwBN;
  const int tb = blockIdx.z * per_split, tend = min(a.n, tb + per_split);
  float2 acc[8][2];
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int c = 0; c < 2; ++c) acc[r][c] = make_float2(0.0f, 0.0f);
  for (int c0 = tb; c0 < tend; c0 += kRwBT) {
    __syncthreads();
    // X chunk: 32 tokens x 128 columns as pairs of bf16
    for (int q = tid; q < kRwBT * kRwBM / 2; q += 256) {
      const int r = q / (kRwBM / 2), c = 2 * (q % (kRwBM / 2));
      const int t = c0 + r, i = i0 + c;
      float lo = 0.0f, hi = 0.0f;
      if (t < tend && i < a.d) load2(static_cast<const T*>(a.X) + (size_t)t * a.d + i, lo, hi);
      xs[r][c] = lo;
      xs[r][c + 1] = hi;
    }
    for (int q = tid; q < kRwBT * kRwBN; q += 256) {
      const int r = q / kRwBN, c = q % kRwBN;
      const int t = c0 + r, e = e0 + c;
      ls[r][c] = (t < tend && e < a.E) ? a.dL[(size_t)t * a.E + e] : 0.0f;
    }
    __syncthreads();
#pragma unroll 4
    for (int r = 0; r < kRwBT; ++r) {
      const float4 x0 = *reinterpret_cast<const float4*>(&xs[r][8 * ti]);
      const float4 x1 = *reinterpret_cast<const float4*>(&xs[r][8 * ti + 4]);
      const float4 l = *reinterpret_cast<const float4*>(&ls[r][4 * te]);
      const float xv[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
      const float2 l01 = make_float2(l.x, l.y), l23 = make_float2(l.z, l.w);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float2 xx = make_float2(xv[u], xv[u]);
        acc[u][0] = __ffma2_rn(xx, l01, acc[u][0]);
        acc[u][1] = __ffma2_rn(xx, l23, acc[u][1]);
      }
    }
  }
  float* dst = a.splits > 1 ? a.partial + (size_t)blockIdx.z * a.d * a.E : a.dWg;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int i = i0 + 8 * ti + u;
    if (i >= a.d) continue;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int e = e0 + 4 * te + c;
      if (e < a.E) dst[(size_t)i * a.E + e] = c & 1 ? acc[u][c >> 1].y : acc[u][c >> 1].x;
    }
  }
}

__global__ void __launch_bounds__(256) router_dwg_reduce_kernel(const float* partial, int splits,
                                                                long long count, float* out) {
  pdl_wait();
  const long long q = (long long)blockIdx.x * 256 + threadIdx.x;
  if (q >= count) return;
  float s = 0.0f;
  for (int z = 0; z < splits; ++z) s += __ldcg(partial + (size_t)z * count + q);
  out[q] = s;
}

}  // namespace

cudaError_t launch_combine_backward(const CombineBwdArgs& a, cudaStream_t s) {
  if (a.bf16) return launch_pdl(combine_backward_kernel<__nv_bfloat16>, a.n, 256, 0, s, a);
  return launch_pdl(combine_backward_kernel<float>, a.n, 256, 0, s, a);
}

cudaError_t launch_pad_zero(const int32_t* offsets, const int32_t* counts, int E, int row_bytes,
                            void* a, void* b, cudaStream_t s) {
  return launch_pdl(pad_zero_kernel, E, 256, 0, s, offsets, counts, row_bytes, a, b);
}

// token slices of the router-weight gradient: enough CTAs for two waves,
// at least 256 tokens per slice
int router_bwd_splits(int n, int d, int E) {
  const int tiles = ceil_div(d, kRwBM) * ceil_div(E, kRwBN);
  int sp = ceil_div(2 * 148, tiles);
  const int most = n / 256 > 1 ? n / 256 : 1;
  if (sp > most) sp = most;
  return sp < 1 ? 1 : sp;
}

cudaError_t launch_router_backward(const RouterBwdArgs& a, cudaStream_t s) {
  const dim3 gt(ceil_div(a.d, 32), ceil_div(a.E, 32));
  cudaError_t e = launch_pdl(transpose_wg_kernel, gt, 256, 0, s, a.Wg, a.d, a.E, a.WgT);
  if (e != cudaSuccess) return e;
  const dim3 gx(ceil_div(a.n, kRxBM), ceil_div(a.d, kRxBN));
  e = a.bf16 ? launch_pdl(router_dx_kernel<__nv_bfloat16>, gx, 256, 0, s, a)
             : launch_pdl(router_dx_kernel<float>, gx, 256, 0, s, a);
  if (e != cudaSuccess) return e;
  const int per = ceil_div(ceil_div(a.n, a.splits), kRwBT) * kRwBT;
  const dim3 gw(ceil_div(a.d, kRwBM), ceil_div(a.E, kRwBN), a.splits);
  e = a.bf16 ? launch_pdl(router_dwg_kernel<__nv_bfloat16>, gw, 256, 0, s, a, per)
             : launch_pdl(router_dwg_kernel<float>, gw, 256, 0, s, a, per);
  if (e != cudaSuccess || a.splits <= 1) return e;
  const long long count = (long long)a.d * a.E;
  return launch_pdl(router_dwg_reduce_kernel, ceil_div(count, 256), 256, 0, s,
                    (const float*)a.partial, a.splits, count, a.dWg);
}

}  // namespace moe
