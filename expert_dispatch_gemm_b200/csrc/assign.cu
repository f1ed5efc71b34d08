// Selection bookkeeping: expert-choice top-k over the token axis, token-choice
// capacity (arrival positions, drop mask, counts, offsets), the per-token
// slot lists used by the combine, and the aux values.
//
// "Expert choice routing" (aicassindra.com), "The math: a gating matrix and
// top-k over tokens": G, I = TopK(S^T, k), I and G are [E,k]; "Token choice
// vs expert choice routing in MoE" (fanout.sh), "Dropped tokens flow in
// opposite directions": assignments that arrive after an expert's buffer is
// full skip it; "MoE routing strategies explained" (ncijnetwork.com), "2.
// Top-1 switch routing with a capacity factor".
#include "device_common.cuh"
#include "moe_internal.h"

namespace moe {

// fp32 -> uint32 whose unsigned order is the float order (-0 folded to +0).
__device__ __forceinline__ uint32_t ordered_key(float f) {
  f = f + 0.0f;  // -0 + 0 = +0 under round-to-nearest
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// ---------------------------------------------------------------------------
// Expert choice: one CTA per expert. Radix-select the k-th largest key of the
// column (one block histogram per 8-bit pass, warp-aggregated shared-memory
// atomics), take every key above it plus the lowest-index ties (ordered block
// scans, no atomics), then order the k picks by (score desc, token asc): by
// counting ranks for k <= kEcRankMax, by a bitonic sort of 64-bit composite
// keys beyond that. The dense slot map is [E, n] so each CTA clears and
// fills its own contiguous row.
// ---------------------------------------------------------------------------
constexpr int kEcRankMax = 1024;
constexpr int kEcMaxPerThread = 16;  // keys per thread, in registers
static_assert(MOE_EC_MAX_TOKENS <= 1024 * kEcMaxPerThread, "EC keys must fit in registers");

// exclusive prefix sum over the CTA (threads in order); returns the total.
// The 32 warp totals are scanned with shuffles by every warp.
__device__ __forceinline__ int block_exclusive_scan(int v, int* excl, int* warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  __syncthreads();  // warp_tot may still be read from a previous scan
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  const int nw = blockDim.x >> 5;
  const int wt = lane < nw ? warp_tot[lane] : 0;
  int winc = wt;
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, winc, o);
    if (lane >= o) winc += y;
  }
  const int wbase = __shfl_sync(0xffffffffu, winc - wt, warp);
  const int total = __shfl_sync(0xffffffffu, winc, 31);
  *excl = wbase + incl - v;
  return total;
}

template <int NT>
__global__ void __launch_bounds__(NT) select_ec_kernel(SelectEcArgs a) {
  pdl_wait();
  extern __shared__ __align__(16) unsigned char ec_smem[];
  const int n = a.n, E = a.E, k = a.k, e = blockIdx.x;
  const bool by_rank = k <= kEcRankMax;
  int kp = 1;
  while (kp < k) kp <<= 1;
  uint64_t* sbuf = reinterpret_cast<uint64_t*>(ec_smem);    // [k] picks, or [kp] to sort
  uint64_t* sorted = by_rank ? sbuf + k : sbuf;              // [k]
  __shared__ int hist[256];
  __shared__ int warp_tot[32];
  __shared__ uint32_t s_prefix, s_mask;
  __shared__ int s_need, s_done;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int32_t* my_rows = a.ec_row + (size_t)e * n;

  // thread tid owns tokens [tid*C, tid*C + C), keys kept in registers
  const int C = (n + NT - 1) / NT;
  const int t0 = tid * C;
  uint32_t kreg[kEcMaxPerThread];
#pragma unroll
  for (int i = 0; i < kEcMaxPerThread; ++i) {
    const int t = t0 + i;
    kreg[i] = (i < C && t < n) ? ordered_key(a.S[(size_t)t * E + e]) : 0u;
  }
  for (int t = tid; t < n; t += NT) my_rows[t] = -1;
  if (tid == 0) {
    s_prefix = 0u;
    s_mask = 0u;
    s_need = k;
    s_done = 0;
  }
  __syncthreads();

  for (int b = tid; b < 256; b += NT) hist[b] = 0;
  __syncthreads();
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    const uint32_t prefix = s_prefix, mask = s_mask;
    // one block histogram; warp-aggregated: the lanes that share a digit add
    // once, through their lowest lane (integer counts: exact in any order)
#pragma unroll
    for (int i = 0; i < kEcMaxPerThread; ++i) {
      if (i >= C) break;
      const int t = t0 + i;
      const bool ok = t < n && (kreg[i] & mask) == prefix;
      const unsigned act = __ballot_sync(0xffffffffu, ok);
      if (ok) {
        const unsigned dig = (kreg[i] >> shift) & 255u;
        const unsigned peers = __match_any_sync(act, dig);
        if (lane == __ffs(peers) - 1) atomicAdd(&hist[dig], (int)__popc(peers));
      }
    }
    __syncthreads();
    if (warp == 0) {
      // lane l holds digits 255-8l down to 248-8l (descending); it clears
      // them for the next pass as it reads them
      int cnt[8], local = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        cnt[i] = hist[255 - 8 * lane - i];
        hist[255 - 8 * lane - i] = 0;
        local += cnt[i];
      }
      int incl = local;
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const int excl = incl - local;
      const int need = s_need;
      const bool here = excl < need && need <= incl;
      const unsigned who = __ballot_sync(0xffffffffu, here);
      if (here && lane == __ffs(who) - 1) {
        int above = excl;
        int digit = 0, dcount = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (above + cnt[i] >= need) {
            digit = 255 - 8 * lane - i;
            dcount = cnt[i];
            break;
          }
          above += cnt[i];
        }
        s_need = need - above;
        s_prefix = prefix | ((uint32_t)digit << shift);
        s_mask = mask | (255u << shift);
        // every key in the chosen bucket is a pick: no later digit matters
        if (above + dcount == need) s_done = 1;
      }
    }
    __syncthreads();
    if (s_done) break;
  }
  // picks: keys whose masked bits exceed T, plus the lowest-token need_eq of
  // those equal to T (all of them when the passes stopped early)
  const uint32_t T = s_prefix, M = s_mask;
  const int need_eq = s_need;

  // the ties' ranks in token order, then every pick's slot in token order
  int my_eq = 0;
#pragma unroll
  for (int i = 0; i < kEcMaxPerThread; ++i)
    my_eq += (i < C && t0 + i < n && (kreg[i] & M) == T);
  int eq_base;
  block_exclusive_scan(my_eq, &eq_base, warp_tot);
  int my_sel = 0;
  {
    int rank = eq_base;
#pragma unroll
    for (int i = 0; i < kEcMaxPerThread; ++i) {
      if (!(i < C && t0 + i < n)) continue;
      const uint32_t u = kreg[i] & M;
      if (u > T) ++my_sel;
      else if (u == T) my_sel += (rank++ < need_eq);
    }
  }
  int slot;
  const int total = block_exclusive_scan(my_sel, &slot, warp_tot);
  {
    int rank = eq_base;
#pragma unroll
    for (int i = 0; i < kEcMaxPerThread; ++i) {
      if (!(i < C && t0 + i < n)) continue;
      const uint32_t u = kreg[i];
      bool sel = (u & M) > T;
      if ((u & M) == T) sel = rank++ < need_eq;
      if (sel)
        sbuf[slot++] = ((uint64_t)u << 32) | (uint64_t)(0xffffffffu - (uint32_t)(t0 + i));
    }
  }
  if (total != k && tid == 0) report_error(a.err, kErrBadIndex | 1);
  __syncthreads();
  if (by_rank) {
    // composite keys are distinct: a pick's place is how many picks beat it
    for (int j = tid; j < k; j += NT) {
      const uint64_t c = sbuf[j];
      int r = 0;
#pragma unroll 8
      for (int i = 0; i < k; ++i) r += sbuf[i] > c;
      sorted[r] = c;
    }
  } else {
    for (int i = k + tid; i < kp; i += NT) sbuf[i] = 0ull;
    __syncthreads();
    for (int size = 2; size <= kp; size <<= 1) {
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        for (int i = tid; i < kp / 2; i += NT) {
          const int lo = 2 * i - (i & (stride - 1));
          const int hi = lo + stride;
          const bool desc = ((lo & size) == 0);
          const uint64_t x = sbuf[lo], y = sbuf[hi];
          if ((x < y) == desc) {
            sbuf[lo] = y;
            sbuf[hi] = x;
          }
        }
        __syncthreads();
      }
    }
  }
  __syncthreads();
  for (int j = tid; j < a.kpad; j += NT) {
    const size_t row = (size_t)e * a.kpad + j;
    if (j < k) {
      const int t = (int)(0xffffffffu - (uint32_t)(sorted[j] & 0xffffffffull));
      const float g = a.S[(size_t)t * E + e];
      a.idx[(size_t)e * k + j] = t;
      a.gate[(size_t)e * k + j] = g;
      a.row_token[row] = t;
      my_rows[t] = (int)row;
      a.ec_gate[(size_t)e * n + t] = g;
    } else {
      a.row_token[row] = -1;
    }
  }
  if (tid == 0) {
    a.load[e] = k;
    a.counts[e] = k;
    a.offsets[e] = e * a.kpad;
    if (e == E - 1) a.offsets[E] = E * a.kpad;
  }
  if (e == 0) {
    // zero what the finish kernel accumulates into, and the fixed aux slots
    if (a.hist)
      for (int i = tid; i <= E; i += NT) a.hist[i] = 0;
    if (tid < MOE_AUX_LEN && tid != MOE_AUX_Z) a.aux[tid] = 0.0f;
    if (warp == 1) {
      double s = 0.0;
      if (a.lse2)
        for (int b = lane; b < a.lse_blocks; b += 32) s += a.lse2[b];
      for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) a.aux[MOE_AUX_Z] = (float)((double)a.z_coef * s / (double)n);
    }
  }
}

static size_t select_ec_smem(int /*nt*/, int k) {
  int kp = 1;
  while (kp < k) kp <<= 1;
  return k <= kEcRankMax ? (size_t)2 * k * 8 : (size_t)kp * 8;
}

template <int NT>
static cudaError_t launch_select_ec_t(const SelectEcArgs& a, cudaStream_t s) {
  const size_t bytes = select_ec_smem(NT, a.k);
  cudaError_t err = cudaFuncSetAttribute(select_ec_kernel<NT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)bytes);
  if (err != cudaSuccess) return err;
  return launch_pdl(select_ec_kernel<NT>, a.E, NT, bytes, s, a);
}

// One thread count for every batch: 256-thread CTAs (cheaper barriers, more
// keys per thread) measured slower on B200 at n = 4096 (17.7 vs 16.6 us).
cudaError_t launch_select_ec(const SelectEcArgs& a, cudaStream_t s) {
  return launch_select_ec_t<1024>(a, s);
}

// Expert choice: each token's picks (expert order) compacted into its slot
// list, the experts-per-token histogram and the aux count of tokens no expert
// picked. A CTA transposes a [E, 32-token] tile of the slot map through
// shared memory (coalesced reads), then one warp per token compacts it.
__global__ void __launch_bounds__(256) ec_finish_kernel(EcFinishArgs a) {
  pdl_wait();
  extern __shared__ __align__(16) unsigned char fin_smem[];
  int* rows_s = reinterpret_cast<int*>(fin_smem);              // [E][33]
  float* gates_s = reinterpret_cast<float*>(rows_s + a.E * 33);  // [E][33]
  __shared__ int hist_s[MOE_MAX_EXPERTS + 1];
  __shared__ int none_s;
  const int E = a.E, n = a.n, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t0 = blockIdx.x * 32;
  for (int i = threadIdx.x; i <= E; i += blockDim.x) hist_s[i] = 0;
  if (threadIdx.x == 0) none_s = 0;
  // a warp's experts e = warp, warp + 8, ...: all their loads are issued
  // before any is used (the gate is read whether or not the expert picked
  // the token, and kept only when it did), so one round trip covers them
  {
    constexpr int U = MOE_MAX_EXPERTS / 8;
    const bool in = t0 + lane < n;
    int r[U];
    float g[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int e = warp + 8 * u;
      const bool ok = in && e < E;
      r[u] = ok ? a.ec_row[(size_t)e * n + t0 + lane] : -1;
      g[u] = ok ? a.ec_gate[(size_t)e * n + t0 + lane] : 0.0f;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int e = warp + 8 * u;
      if (e < E) {
        rows_s[e * 33 + lane] = r[u];
        gates_s[e * 33 + lane] = r[u] >= 0 ? g[u] : 0.0f;
      }
    }
  }
  __syncthreads();
  for (int tt = warp; tt < 32; tt += 8) {
    const int t = t0 + tt;
    if (t >= n) break;
    int base = 0;
    for (int c = 0; c < E; c += 32) {
      const int e = c + lane;
      const int r = e < E ? rows_s[e * 33 + tt] : -1;
      const unsigned m = __ballot_sync(0xffffffffu, r >= 0);
      if (r >= 0) {
        const int p = base + __popc(m & ((1u << lane) - 1u));
        a.tok_row[(size_t)t * E + p] = r;
        a.tok_gate[(size_t)t * E + p] = gates_s[e * 33 + tt];
      }
      base += __popc(m);
    }
    for (int p = base + lane; p < E; p += 32) {
      a.tok_row[(size_t)t * E + p] = -1;
      a.tok_gate[(size_t)t * E + p] = 0.0f;
    }
    if (lane == 0) {
      atomicAdd(&hist_s[base], 1);
      if (base == 0) atomicAdd(&none_s, 1);
    }
  }
  __syncthreads();
  if (a.hist)
    for (int i = threadIdx.x; i <= E; i += blockDim.x)
      if (hist_s[i]) atomicAdd(&a.hist[i], hist_s[i]);
  if (threadIdx.x == 0 && none_s) atomicAdd(&a.aux[MOE_AUX_TOKENS_NO_EXPERT], (float)none_s);
}

// (select_ec_kernel's block 0 has zeroed hist and the aux slots)
cudaError_t launch_ec_finish(const EcFinishArgs& a, cudaStream_t s) {
  const size_t bytes = (size_t)a.E * 33 * 8;
  cudaError_t e = cudaFuncSetAttribute(ec_finish_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  return launch_pdl(ec_finish_kernel, ceil_div(a.n, 32), 256, bytes, s, a);
}

// ---------------------------------------------------------------------------
// Token choice: per-block expert histograms, a scan over blocks (counts,
// offsets, aux), then arrival positions, drops and slot lists.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kTokBlock) tc_hist_kernel(TcAssignArgs a) {
  pdl_wait();
  __shared__ int hist[MOE_MAX_EXPERTS];
  for (int i = threadIdx.x; i < a.E; i += kTokBlock) hist[i] = 0;
  __syncthreads();
  const int t = blockIdx.x * kTokBlock + threadIdx.x;
  if (t < a.n)
    for (int j = 0; j < a.K; ++j) {
      const int e = a.idx[(size_t)t * a.K + j];
      if ((unsigned)e < (unsigned)a.E)
        atomicAdd(&hist[e], 1);
      else
        bad_index(a.err, kSiteScatterIdx);
    }
  __syncthreads();
  for (int i = threadIdx.x; i < a.E; i += kTokBlock)
    a.blk_hist[(size_t)blockIdx.x * a.E + i] = hist[i];
}

constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads) tc_scan_kernel(TcAssignArgs a) {
  pdl_wait();
  __shared__ int seg[MOE_MAX_EXPERTS];
  __shared__ int off[MOE_MAX_EXPERTS + 1];
  __shared__ int load_s[MOE_MAX_EXPERTS], kept_s[MOE_MAX_EXPERTS];
  __shared__ double fp[MOE_MAX_EXPERTS];
  __shared__ double part[1024];  // [slice][expert] partial column sums of S
  __shared__ double z_s;
  const int E = a.E, tid = threadIdx.x;
  // column sums of S for the balance loss: thread (slice, e) adds the router
  // blocks b = slice, slice + S, ... in order; the slices are then added in
  // order, so the result does not depend on scheduling
  const int S = max(1, (int)blockDim.x / E);
  if (tid < S * E) {
    const int e = tid % E, slice = tid / E;
    double col = 0.0;
    // eight loads in flight, added in the same block order as one at a time
    constexpr int U = 8;
    int b = slice;
    for (; b + (U - 1) * S < a.colsum_blocks; b += U * S) {
      float v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) v[u] = a.colsum[(size_t)(b + u * S) * E + e];
#pragma unroll
      for (int u = 0; u < U; ++u) col += (double)v[u];
    }
    for (; b < a.colsum_blocks; b += S) col += (double)a.colsum[(size_t)b * E + e];
    part[tid] = col;
  }
  __syncthreads();
  // per expert: exclusive prefix of the token blocks' counts, one warp per
  // expert, 32 blocks per step (a shuffle scan), so the block count adds
  // steps of one load each, not a chain of dependent loads; a warp loads the
  // first 32 blocks of all its experts before scanning any of them
  const int lane = tid & 31, warp = tid >> 5;
  constexpr int nwarps = kScanThreads / 32;
  constexpr int kExpertsPerWarp = (MOE_MAX_EXPERTS + nwarps - 1) / nwarps;
  int first[kExpertsPerWarp];
#pragma unroll
  for (int j = 0; j < kExpertsPerWarp; ++j) {
    const int e = warp + j * nwarps;
    first[j] = (e < E && lane < a.tok_blocks) ? a.blk_hist[(size_t)lane * E + e] : 0;
  }
#pragma unroll
  for (int j = 0; j < kExpertsPerWarp; ++j) {
    const int e = warp + j * nwarps;
    if (e >= E) break;
    int run = 0;
    for (int b0 = 0; b0 < a.tok_blocks; b0 += 32) {
      const int b = b0 + lane;
      const int v = b0 == 0 ? first[j] : (b < a.tok_blocks ? a.blk_hist[(size_t)b * E + e] : 0);
      int incl = v;
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (b < a.tok_blocks) a.blk_base[(size_t)b * E + e] = run + incl - v;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) load_s[e] = run;
  }
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) {
    const int run = load_s[e];
    const int kept = a.cap < 0 ? run : min(run, a.cap);
    a.load[e] = run;
    a.counts[e] = kept;
    kept_s[e] = kept;
    seg[e] = (kept + kRowAlign - 1) / kRowAlign * kRowAlign;
    double col = 0.0;
    for (int sl = 0; sl < S; ++sl) col += part[sl * E + e];
    fp[e] = ((double)run / ((double)a.n * a.K)) * (col / (double)a.n);
  }
  if (tid < 32) {
    // sum of lse^2 over the router blocks: lane-strided, then a fixed
    // shuffle tree, so the order never depends on scheduling
    double z = 0.0;
    if (a.lse2)
      for (int b = tid; b < a.lse_blocks; b += 32) z += a.lse2[b];
    for (int o = 16; o; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    if (tid == 0) z_s = z;
  }
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    double lbs = 0.0;
    int mx = 0;
    long long dropped = 0;
    for (int e = 0; e < E; ++e) {
      off[e] = run;
      run += seg[e];
      lbs += fp[e];
      mx = max(mx, load_s[e]);
      dropped += load_s[e] - kept_s[e];
    }
    off[E] = run;
    a.aux[MOE_AUX_LB] = (float)((double)a.lb_coef * E * lbs);
    a.aux[MOE_AUX_Z] = a.lse2 ? (float)((double)a.z_coef * z_s / (double)a.n) : 0.0f;
    a.aux[MOE_AUX_MAXVIO] = (float)((double)mx / ((double)a.n * a.K / E) - 1.0);
    a.aux[MOE_AUX_DROPPED] = (float)dropped;
    a.aux[MOE_AUX_TOKENS_SOME_DROPPED] = 0.0f;
    a.aux[MOE_AUX_TOKENS_ALL_DROPPED] = 0.0f;
    a.aux[MOE_AUX_TOKENS_NO_EXPERT] = 0.0f;
    a.aux[MOE_AUX_RESERVED] = 0.0f;
  }
  __syncthreads();
  for (int e = tid; e <= E; e += blockDim.x) a.offsets[e] = off[e];
  // padding rows of each segment (fewer than kRowAlign per expert)
  for (int i = tid; i < E * kRowAlign; i += blockDim.x) {
    const int e = i / kRowAlign, r = off[e] + kept_s[e] + i % kRowAlign;
    if (r < off[e + 1]) a.row_token[r] = -1;
  }
}

__global__ void __launch_bounds__(kTokBlock) tc_scatter_kernel(TcAssignArgs a) {
  pdl_wait();
  extern __shared__ __align__(16) unsigned char sc_smem[];
  constexpr int W = kTokBlock / 32;
  const int E = a.E, K = a.K;
  uint32_t* mask = reinterpret_cast<uint32_t*>(sc_smem);      // [W][E]
  int* wbase = reinterpret_cast<int*>(mask + W * E);          // [W][E]
  int* base_s = wbase + W * E;                                // [E] block base + offset
  __shared__ int some_s, all_s;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int i = tid; i < W * E; i += kTokBlock) mask[i] = 0u;
  for (int e = tid; e < E; e += kTokBlock)
    base_s[e] = a.offsets[e] + a.blk_base[(size_t)blockIdx.x * E + e];
  if (tid == 0) {
    some_s = 0;
    all_s = 0;
  }
  __syncthreads();
  const int t = blockIdx.x * kTokBlock + tid;
  const bool live = t < a.n;
  if (live)
    for (int j = 0; j < K; ++j) {
      const int e = a.idx[(size_t)t * K + j];
      if ((unsigned)e < (unsigned)E) atomicOr(&mask[warp * E + e], 1u << lane);
    }
  __syncthreads();
  for (int e = tid; e < E; e += kTokBlock) {
    int run = 0;
    for (int w = 0; w < W; ++w) {
      wbase[w * E + e] = run;
      run += __popc(mask[w * E + e]);
    }
  }
  __syncthreads();
  if (live) {
    int kept = 0;
    for (int j = 0; j < K; ++j) {
      const size_t aj = (size_t)t * K + j;
      const int e = a.idx[aj];
      bool keep = false;
      int row = -1;
      if ((unsigned)e < (unsigned)E) {
        // arrival position: earlier blocks, earlier warps, earlier lanes
        const int in_blk = wbase[warp * E + e] + __popc(mask[warp * E + e] & ((1u << lane) - 1u));
        const int pos = base_s[e] - a.offsets[e] + in_blk;
        keep = a.cap < 0 || pos < a.cap;
        if (keep) {
          row = base_s[e] + in_blk;
          a.row_token[row] = t;
          a.tok_row[(size_t)t * K + kept] = row;
          a.tok_gate[(size_t)t * K + kept] = a.gate[aj];
          ++kept;
        }
      }
      a.drop[aj] = keep ? 0 : 1;
    }
    for (int j = kept; j < K; ++j) {
      a.tok_row[(size_t)t * K + j] = -1;
      a.tok_gate[(size_t)t * K + j] = 0.0f;
    }
    if (kept < K) atomicAdd(&some_s, 1);
    if (kept == 0) atomicAdd(&all_s, 1);
  }
  __syncthreads();
  if (tid == 0) {
    if (some_s) atomicAdd(&a.aux[MOE_AUX_TOKENS_SOME_DROPPED], (float)some_s);
    if (all_s) atomicAdd(&a.aux[MOE_AUX_TOKENS_ALL_DROPPED], (float)all_s);
  }
}

cudaError_t launch_tc_assign(const TcAssignArgs& a, cudaStream_t s) {
  cudaError_t e = launch_pdl(tc_hist_kernel, a.tok_blocks, kTokBlock, 0, s, a);
  if (e != cudaSuccess) return e;
  e = launch_pdl(tc_scan_kernel, 1, kScanThreads, 0, s, a);
  if (e != cudaSuccess) return e;
  const size_t bytes = (size_t)(2 * (kTokBlock / 32) + 1) * a.E * 4;
  e = cudaFuncSetAttribute(tc_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)bytes);
  if (e != cudaSuccess) return e;
  return launch_pdl(tc_scatter_kernel, a.tok_blocks, kTokBlock, bytes, s, a);
}

}  // namespace moe
