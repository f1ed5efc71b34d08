// Grouped expert GEMMs of the layer's backward pass on the tcgen05 tensor
// cores.
//
// The backward of "Expert choice routing" (aicassindra.com), "The math: a
// gating matrix and top-k over tokens": the per-expert FFN Y = act(X W1^T
// [, X W3^T]) W2^T is differentiated by the chain rule, one grouped GEMM per
// step:
//   SAVE   [U | V], H = X W1^T, X W3^T, act      (the forward's up projection
//                                                 again, keeping U and V)
//   DACT   dU, dV = (dY W2) * act'(U, V)          (W2 read MN-major)
//   DX     dX_perm = dU W1 + dV W3                (W1, W3 read MN-major)
//   WG2    dW2_e = dY_e^T H_e                     (both operands MN-major,
//   WG13   [dW1_e; dW3_e] = [dU_e | dV_e]^T X_e    K = the expert's rows)
// The first three tile the dispatched rows like the forward kernels (128-row
// blocks of one expert x 256 output columns, shared experts after the routed
// ones); the weight gradients tile each expert's output matrix (128 x 256)
// and reduce over its rows.
//
// Persistent kernels, one CTA per SM or one CTA pair (cta_group::2) per two
// SMs: warp 0 issues the TMA loads into the shared-memory ring (a single CTA:
// stages of A 128x64 + B 256x64; a pair: stages of A 128x64 + half of B,
// 128x64, per CTA), warp 1 issues tcgen05.mma (M128 or, from the pair
// leader, M256; N256 K16) into one of two TMEM accumulators, and warps 2-9
// run the epilogue, two per TMEM lane quadrant with half of the columns
// each. The row modes take pairs when experts average at least two 128-row
// blocks (a pair tile is two blocks of one expert; with an odd count the
// second CTA repeats the first block and stores nothing), the weight
// gradients whenever the output has more than one 128-row block. The weight
// gradients reduce over a few k-blocks per tile, so their epilogue sets the
// pace: it stages 32 x 64 blocks in shared memory and writes whole 128-byte
// rows. An operand that is K-major in memory comes in as one
// 128-byte-swizzled box;
// an MN-major one (a weight matrix read along its input dimension, or a row
// block read across its columns) as boxes of 64 MN-elements x 64 K-rows,
// described to the MMA as the canonical MN-major 128-byte-swizzle layout:
// 64 contiguous MN-elements per 128-byte row, eight K-rows per 1024-byte
// swizzle atom (the stride between atoms along K), and 8 KB between
// consecutive 64-element MN chunks.
// Every mbarrier wait is bounded (2 s): on a timeout the CTA records an
// error, stops issuing, waits (bounded) for its own copies and MMAs, frees
// TMEM and returns.
#include <cuda.h>
#include <math.h>

#include "device_common.cuh"
#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {

namespace {

constexpr int kWBM = 128, kWBN = 256, kWBK = 64;
constexpr int kWABytes = kWBM * kWBK * 2;          // 16 KB: this CTA's 128 rows of A
constexpr int kWThreads = 320;  // producer, MMA, eight epilogue warps
constexpr int kEpiThreads = 256;
constexpr uint64_t kWWaitNs = 2000000000ull;       // 2 s
constexpr uint32_t kMnChunkBytes = sm100::kMnChunkBytes;  // one 64 x 64 MN-major box: 8 KB
constexpr int kWStagesMax = 6;

// shared-memory ring: a single CTA holds all 256 rows of B (48 KB stages);
// a CTA pair splits B, 128 rows each (32 KB stages). The weight gradients
// reduce over a few k-blocks per tile and give two stages to the epilogue's
// staging blocks.
template <bool PAIR, bool WG>
struct Ring {
  static constexpr int stages = PAIR ? (WG ? 4 : 6) : (WG ? 3 : 4);
  static constexpr int b_bytes = (PAIR ? kWBN / 2 : kWBN) * kWBK * 2;
  static constexpr int stage_bytes = kWABytes + b_bytes;
};

struct BwdState {
  uint64_t full[kWStagesMax];
  uint64_t empty[kWStagesMax];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  volatile int abort_flag;
  int offs[MOE_MAX_EXPERTS + 1];
  int cnt[MOE_MAX_EXPERTS];
  int tprefix[MOE_MAX_EXPERTS + 1];
};

constexpr int kStateBytes = (sizeof(BwdState) + 127) / 128 * 128;
// weight-gradient epilogue staging: per warp two 32 x 128-byte blocks
constexpr int kWStageOut = 8 * 2 * 32 * 128;

template <bool CLUSTER_ACQUIRE>
__device__ __forceinline__ bool bwait(uint64_t* bar, uint32_t parity, BwdState* st, int* err,
                                      int code) {
  auto probe = [&]() {
    return CLUSTER_ACQUIRE ? sm100::mbar_try_wait_cluster(bar, parity)
                           : sm100::mbar_try_wait(bar, parity);
  };
  if (probe()) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (probe()) return true;
    if ((it & 63u) == 0) {
      if (st->abort_flag) return false;
      if (global_timer_ns() - t0 > kWWaitNs) {
        st->abort_flag = 1;
        report_error(err, code);
        return false;
      }
    }
  }
}

// kind::f16 instruction descriptor with the operands' majorness: bit 15 = A
// MN-major, bit 16 = B MN-major
__host__ __device__ constexpr uint32_t idesc_major(int M, bool a_mn, bool b_mn) {
  return sm100::idesc_bf16_f32(M, kWBN) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16);
}

template <int MODE>
struct ModeTraits {
  static constexpr bool A_MN = MODE == BW_WG2 || MODE == BW_WG13;
  static constexpr bool B_MN = MODE != BW_SAVE;
  static constexpr bool WGRAD = A_MN;
};

struct BTile {
  bool skip;           // a weight-gradient tile of an expert with no rows: write zeros
  bool valid;          // this CTA's rows are real (a pair's second block may repeat the first)
  bool shared;
  int expert;          // routed expert or shared index
  int a_row;           // K-major A: first row; MN-major A: first K row
  int b_row;           // K-major B: this CTA's first row; MN-major B: first K row
  int m0, n0;          // weight gradients: this CTA's output rows; first column
  int b_n0;            // MN-major B: this CTA's first column of B
  int kb;              // k-blocks of this tile
  long long out_row;   // row modes: this CTA's first output row
};

// Row modes: tiles expert by expert, 256-column block by block, the expert's
// 128-row blocks (CTA pairs: pairs of blocks) innermost; shared experts after
// the routed ones. Weight-gradient modes: expert by expert, 128-row (pairs:
// 256-row) output block, 256-column output block innermost.
template <int MODE, bool PAIR>
__device__ __forceinline__ BTile decode(int tile, const BwdParams& p, const BwdState* st,
                                        int routed, uint32_t rank) {
  BTile t{};
  t.valid = true;
  if (!ModeTraits<MODE>::WGRAD) {
    int nt;
    if (tile < routed) {
      int lo = 0, hi = p.E - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (st->tprefix[mid] <= tile) lo = mid; else hi = mid - 1;
      }
      const int local = tile - st->tprefix[lo];
      const int blocks = (st->offs[lo + 1] - st->offs[lo]) / kWBM;
      int mloc;
      if (PAIR) {
        const int pairs = max((blocks + 1) / 2, 1);
        nt = local / pairs;
        mloc = 2 * (local % pairs) + (int)rank;
        t.valid = mloc < blocks;
        if (!t.valid) mloc -= 1;
      } else {
        const int nb = max(blocks, 1);
        nt = local / nb;
        mloc = local % nb;
      }
      t.a_row = st->offs[lo] + mloc * kWBM;
      t.out_row = t.a_row;
      t.expert = lo;
      t.shared = false;
    } else {
      const int spb = PAIR ? (p.shared_blocks + 1) / 2 : p.shared_blocks;
      const int per = spb * p.nt_tiles;
      const int q = tile - routed;
      const int s = q / per, local = q % per;
      nt = local / spb;
      int lm = local % spb;
      if (PAIR) {
        lm = 2 * lm + (int)rank;
        t.valid = lm < p.shared_blocks;
        if (!t.valid) lm -= 1;
      }
      t.a_row = (int)(p.a1_row_base + s * p.a1_row_stride + (long long)lm * kWBM);
      t.out_row = p.out_shared_base + s * p.n_pad + (long long)lm * kWBM;
      t.expert = s;
      t.shared = true;
    }
    t.n0 = nt * p.n_block;
    t.kb = p.K / kWBK;
    if (MODE == BW_SAVE) {
      // K-major B: the expert's weight rows of this column block (a pair:
      // SwiGLU W1 on the leader, W3 on the peer; otherwise 128 rows each)
      t.b_row = t.expert * p.b_rows_per_expert + t.n0 +
                (PAIR && !p.swiglu ? (int)rank * (kWBN / 2) : 0);
    } else {
      t.b_row = t.expert * p.b_rows_per_expert;
      t.b_n0 = t.n0 + (PAIR ? (int)rank * (kWBN / 2) : 0);
    }
  } else {
    const int mblk = PAIR ? 2 * kWBM : kWBM;
    const int per = p.mt_tiles * p.nt_tiles;
    const int q = tile / per, local = tile % per;
    t.m0 = (local / p.nt_tiles) * mblk + (PAIR ? (int)rank * kWBM : 0);
    t.n0 = (local % p.nt_tiles) * kWBN;
    t.b_n0 = t.n0 + (PAIR ? (int)rank * (kWBN / 2) : 0);
    if (q < p.E) {
      t.kb = (st->cnt[q] + kWBK - 1) / kWBK;
      t.a_row = st->offs[q];
      t.b_row = st->offs[q];
      t.expert = q;
      t.shared = false;
    } else {
      const int s = q - p.E;
      t.kb = (p.n + kWBK - 1) / kWBK;
      t.a_row = (int)(p.a1_row_base + s * p.a1_row_stride);
      t.b_row = (int)(p.b1_row_base + s * p.b1_row_stride);
      t.expert = s;
      t.shared = true;
    }
    t.skip = t.kb == 0;
  }
  return t;
}

// epilogue of the row modes: one thread per row, 32 columns at a time
template <int MODE>
__device__ __forceinline__ void row_epilogue(const BwdParams& p, const BTile& t, uint32_t tbase,
                                             int row_in_tile, int half) {
  const long long row = t.out_row + row_in_tile;
  const int ncols = MODE == BW_SAVE && p.swiglu ? kWBN / 2 : kWBN;
#pragma unroll 1
  for (int cc = half * (ncols / 2); cc < (half + 1) * (ncols / 2); cc += 32) {
    const int col = t.n0 + cc;
    if (col >= p.n_total) break;
    // DACT: the stored U (and V) of this row's 32 columns, loaded before the
    // accumulator so the two latencies overlap
    uint4 ur[4], vr[4];
    if (MODE == BW_DACT) {
      const uint4* pu = reinterpret_cast<const uint4*>(p.in0 + row * p.ld_in + col);
#pragma unroll
      for (int j = 0; j < 4; ++j) ur[j] = pu[j];
      if (p.swiglu) {
        const uint4* pv = reinterpret_cast<const uint4*>(p.in1 + row * p.ld_in + col);
#pragma unroll
        for (int j = 0; j < 4; ++j) vr[j] = pv[j];
      }
    }
    uint32_t v[32];
    sm100::tmem_ld_32x32b_x32(tbase + cc, v);
    float f[32], g[32];
    if (MODE == BW_SAVE && p.swiglu) {
      uint32_t w[32];
      sm100::tmem_ld_32x32b_x32(tbase + kWBN / 2 + cc, w);
      sm100::tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        f[i] = __uint_as_float(v[i]);
        g[i] = __uint_as_float(w[i]);
      }
    } else {
      sm100::tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(v[i]);
    }
    if (MODE == BW_SAVE) {
      // U (and V) as stored pre-activations, H as the forward computes it
      uint4* du = reinterpret_cast<uint4*>(p.out0 + row * p.ld_out + col);
      uint4* dh = reinterpret_cast<uint4*>(p.out2 + row * p.ld_out + col);
      float hv[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        if (p.swiglu) hv[i] = f[i] * __frcp_rn(1.0f + __expf(-f[i])) * g[i];
        else if (p.act == MOE_ACT_RELU) hv[i] = fmaxf(f[i], 0.0f);
        else hv[i] = 0.5f * f[i] * (1.0f + erff(f[i] * 0.70710678118654752f));
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        du[j] = make_uint4(pack_bf16x2(f[8 * j], f[8 * j + 1]), pack_bf16x2(f[8 * j + 2], f[8 * j + 3]),
                           pack_bf16x2(f[8 * j + 4], f[8 * j + 5]), pack_bf16x2(f[8 * j + 6], f[8 * j + 7]));
        dh[j] = make_uint4(pack_bf16x2(hv[8 * j], hv[8 * j + 1]), pack_bf16x2(hv[8 * j + 2], hv[8 * j + 3]),
                           pack_bf16x2(hv[8 * j + 4], hv[8 * j + 5]), pack_bf16x2(hv[8 * j + 6], hv[8 * j + 7]));
      }
      if (p.swiglu) {
        uint4* dv = reinterpret_cast<uint4*>(p.out1 + row * p.ld_out + col);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          dv[j] = make_uint4(pack_bf16x2(g[8 * j], g[8 * j + 1]), pack_bf16x2(g[8 * j + 2], g[8 * j + 3]),
                             pack_bf16x2(g[8 * j + 4], g[8 * j + 5]), pack_bf16x2(g[8 * j + 6], g[8 * j + 7]));
      }
    } else if (MODE == BW_DACT) {
      // f = dH; the stored U (and V) of the same row and columns
      float u[32], vv[32];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint4 x = ur[j];
        const uint32_t w4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          u[8 * j + 2 * k] = __uint_as_float(w4[k] << 16);
          u[8 * j + 2 * k + 1] = __uint_as_float(w4[k] & 0xFFFF0000u);
        }
      }
      if (p.swiglu) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint4 x = vr[j];
          const uint32_t w4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            vv[8 * j + 2 * k] = __uint_as_float(w4[k] << 16);
            vv[8 * j + 2 * k + 1] = __uint_as_float(w4[k] & 0xFFFF0000u);
          }
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float sg = __frcp_rn(1.0f + __expf(-u[i]));
          g[i] = f[i] * u[i] * sg;                                   // dV = dH silu(U)
          f[i] = f[i] * vv[i] * sg * (1.0f + u[i] * (1.0f - sg));    // dU = dH V silu'(U)
        }
      } else if (p.act == MOE_ACT_RELU) {
#pragma unroll
        for (int i = 0; i < 32; ++i) f[i] = u[i] > 0.0f ? f[i] : 0.0f;
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float cdf = 0.5f * (1.0f + erff(u[i] * 0.70710678118654752f));
          const float pdf = 0.3989422804014327f * __expf(-0.5f * u[i] * u[i]);
          f[i] = f[i] * (cdf + u[i] * pdf);
        }
      }
      uint4* du = reinterpret_cast<uint4*>(p.out0 + row * p.ld_out + col);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        du[j] = make_uint4(pack_bf16x2(f[8 * j], f[8 * j + 1]), pack_bf16x2(f[8 * j + 2], f[8 * j + 3]),
                           pack_bf16x2(f[8 * j + 4], f[8 * j + 5]), pack_bf16x2(f[8 * j + 6], f[8 * j + 7]));
      if (p.swiglu) {
        uint4* dv = reinterpret_cast<uint4*>(p.out0 + row * p.ld_out + p.n_total + col);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          dv[j] = make_uint4(pack_bf16x2(g[8 * j], g[8 * j + 1]), pack_bf16x2(g[8 * j + 2], g[8 * j + 3]),
                             pack_bf16x2(g[8 * j + 4], g[8 * j + 5]), pack_bf16x2(g[8 * j + 6], g[8 * j + 7]));
      }
    } else {  // BW_DX
      uint4* o = reinterpret_cast<uint4*>(p.out0 + row * p.ld_out + col);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        o[j] = make_uint4(pack_bf16x2(f[8 * j], f[8 * j + 1]), pack_bf16x2(f[8 * j + 2], f[8 * j + 3]),
                          pack_bf16x2(f[8 * j + 4], f[8 * j + 5]), pack_bf16x2(f[8 * j + 6], f[8 * j + 7]));
    }
  }
}

// this thread's output row of a weight gradient, or nullptr past the end
__device__ __forceinline__ __nv_bfloat16* wgrad_row(const BwdParams& p, const BTile& t, int m) {
  if (m >= p.m_total) return nullptr;
  const bool hi = m >= p.m_split;
  __nv_bfloat16* dst = t.shared ? (hi ? p.sw_out1 : p.sw_out0) : (hi ? p.w_out1 : p.w_out0);
  return dst + (size_t)t.expert * p.w_expert_stride + (size_t)(hi ? m - p.m_split : m) * p.ld_w;
}

template <int MODE, bool PAIR>
// tmO0..tmO3: weight-gradient outputs for TMA stores (routed rows below /
// above m_split, shared rows below / above), boxes of 64 columns x 32 rows
__device__ __forceinline__ void bwd_body(const CUtensorMap* tmA0, const CUtensorMap* tmA1,
                                         const CUtensorMap* tmB0, const CUtensorMap* tmB0g,
                                         const CUtensorMap* tmB1, const CUtensorMap* tmB1g,
                                         const CUtensorMap* tmO0, const CUtensorMap* tmO1,
                                         const CUtensorMap* tmO2, const CUtensorMap* tmO3,
                                         const BwdParams& p, unsigned char* base) {
  using Tr = ModeTraits<MODE>;
  using R = Ring<PAIR, Tr::WGRAD>;
  unsigned char* sA = base;
  unsigned char* sB = base + R::stages * kWABytes;
  BwdState* st = reinterpret_cast<BwdState*>(base + R::stages * R::stage_bytes);
  // weight-gradient epilogue staging: [8 warps][2][32 rows][128 bytes],
  // 1024-byte aligned like a 128-byte-swizzled TMA box
  unsigned char* wstage = base + R::stages * R::stage_bytes + (kStateBytes + 1023) / 1024 * 1024;
  const uint32_t rank = PAIR ? sm100::cluster_ctarank() : 0u;
  const bool leader = rank == 0;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < R::stages; ++s) {
      sm100::mbar_init(&st->full[s], 1);
      sm100::mbar_init(&st->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      sm100::mbar_init(&st->tfull[a], 1);
      sm100::mbar_init(&st->tempty[a], PAIR ? 2 * kEpiThreads : kEpiThreads);
    }
    sm100::mbar_init(&st->drain, 1);
    st->abort_flag = 0;
    sm100::fence_mbar_init();
  }
  if (warp == 1) {
    if (PAIR) {
      sm100::tmem_alloc_pair(&st->tmem_base, 512);
      sm100::tmem_relinquish_pair();
    } else {
      sm100::tmem_alloc(&st->tmem_base, 512);
      sm100::tmem_relinquish();
    }
  }
  pdl_wait();
  for (int i = tid; i <= p.E; i += kWThreads) st->offs[i] = p.offsets[i];
  for (int i = tid; i < p.E; i += kWThreads) {
    const int seg = p.offsets[i + 1] - p.offsets[i];
    const int c = p.counts ? p.counts[i] : seg;
    st->cnt[i] = max(0, min(c, seg));
  }
  __syncthreads();
  if (tid == 0 && !Tr::WGRAD) {
    int run = 0;
    for (int e = 0; e < p.E; ++e) {
      st->tprefix[e] = run;
      const int blocks = max(st->offs[e + 1] - st->offs[e], 0) / kWBM;
      run += (PAIR ? (blocks + 1) / 2 : blocks) * p.nt_tiles;
    }
    st->tprefix[p.E] = run;
  }
  sm100::tc_fence_before();
  __syncthreads();
  if (PAIR) sm100::cluster_sync();  // both CTAs' barriers exist before any remote arrive
  sm100::tc_fence_after();
  const uint32_t tmem = st->tmem_base;

  int routed, total;
  if (Tr::WGRAD) {
    routed = p.E * p.mt_tiles * p.nt_tiles;
    total = (p.E + p.n_shared) * p.mt_tiles * p.nt_tiles;
  } else {
    const int cap = PAIR ? (p.max_routed_blocks + p.E) : p.max_routed_blocks;
    routed = min(st->tprefix[p.E], cap * p.nt_tiles);
    const int sb = PAIR ? (p.shared_blocks + 1) / 2 : p.shared_blocks;
    total = routed + p.n_shared * sb * p.nt_tiles;
  }
  const int first = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int stride = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = first; ok && tile < total; tile += stride) {
        const BTile t = decode<MODE, PAIR>(tile, p, st, routed, rank);
        if (t.skip) continue;
        const CUtensorMap* ma = t.shared ? tmA1 : tmA0;
        for (int kb = 0; kb < t.kb; ++kb) {
          if (!bwait<false>(&st->empty[stage], phase ^ 1u, st, p.err, kErrGemmTimeout | 0x51)) {
            ok = false;
            break;
          }
          unsigned char* a_dst = sA + stage * kWABytes;
          unsigned char* b_dst = sB + stage * R::b_bytes;
          const int k0 = kb * kWBK;
          // every copy of the stage completes on the leader's barrier
          uint32_t fl = 0;
          uint64_t* fb = &st->full[stage];
          if (PAIR) {
            fl = sm100::mapa_shared(sm100::smem_addr(fb), 0);
            if (leader) sm100::mbar_arrive_expect_tx(fb, 2 * R::stage_bytes);
          } else {
            sm100::mbar_arrive_expect_tx(fb, R::stage_bytes);
          }
          auto load = [&](void* dst, const CUtensorMap* m, int x, int y) {
            if (PAIR) sm100::tma_load_2d_pair(dst, m, fl, x, y);
            else sm100::tma_load_2d(dst, m, fb, x, y);
          };
          if (Tr::A_MN) {
#pragma unroll
            for (int c = 0; c < kWBM / 64; ++c)
              load(a_dst + c * kMnChunkBytes, ma, t.m0 + 64 * c, t.a_row + k0);
          } else {
            load(a_dst, ma, k0, t.a_row);
          }
          if (MODE == BW_SAVE) {
            const CUtensorMap* mb = t.shared ? tmB1 : tmB0;
            const CUtensorMap* mbg = t.shared ? tmB1g : tmB0g;
            if (PAIR) {
              load(b_dst, p.swiglu && !leader ? mbg : mb, k0, t.b_row);
            } else if (p.swiglu) {
              load(b_dst, mb, k0, t.b_row);
              load(b_dst + R::b_bytes / 2, mbg, k0, t.b_row);
            } else {
              load(b_dst, mb, k0, t.b_row);
            }
          } else {
            // MN-major B: this CTA's 64-column chunks of K rows k0..k0+63
            const CUtensorMap* mb;
            int krow;
            if (MODE == BW_DX && k0 >= p.k_split) {
              mb = t.shared ? tmB1g : tmB0g;
              krow = t.b_row + k0 - p.k_split;
            } else {
              mb = t.shared ? tmB1 : tmB0;
              krow = t.b_row + k0;
            }
#pragma unroll
            for (int c = 0; c < R::b_bytes / (int)kMnChunkBytes; ++c)
              load(b_dst + c * kMnChunkBytes, mb, t.b_n0 + 64 * c, krow);
          }
          ++issued;
          if (++stage == R::stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok && leader) {
        // wait (bounded) until the copies of the outstanding stages have landed
        int s = stage;
        uint32_t ph = phase;
        const int pending = issued < R::stages ? issued : R::stages;
        for (int i = 0; i < pending; ++i) {
          if (--s < 0) {
            s = R::stages - 1;
            ph ^= 1u;
          }
          const uint64_t t0 = global_timer_ns();
          while (!sm100::mbar_try_wait(&st->full[s], ph) && global_timer_ns() - t0 < kWWaitNs) {
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      constexpr uint32_t idesc = idesc_major(PAIR ? 2 * kWBM : kWBM, Tr::A_MN, Tr::B_MN);
      int stage = 0, used = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = first; ok && tile < total; tile += stride) {
        const BTile t = decode<MODE, PAIR>(tile, p, st, routed, rank);
        if (t.skip) continue;
        const int acc = used & 1;
        const uint32_t acc_phase = (uint32_t)(used >> 1) & 1u;
        ++used;
        if (!bwait<PAIR>(&st->tempty[acc], acc_phase ^ 1u, st, p.err, kErrGemmTimeout | 0x52)) {
          ok = false;
          break;
        }
        sm100::tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(acc * kWBN);
        for (int kb = 0; kb < t.kb; ++kb) {
          if (!bwait<false>(&st->full[stage], phase, st, p.err, kErrGemmTimeout | 0x53)) {
            ok = false;
            break;
          }
          sm100::tc_fence_after();
          const uint32_t a_addr = sm100::smem_addr(sA + stage * kWABytes);
          const uint32_t b_addr = sm100::smem_addr(sB + stage * R::b_bytes);
          const uint64_t adesc =
              Tr::A_MN ? sm100::sw128_mnmajor_desc(a_addr) : sm100::sw128_kmajor_desc(a_addr);
          const uint64_t bdesc =
              Tr::B_MN ? sm100::sw128_mnmajor_desc(b_addr) : sm100::sw128_kmajor_desc(b_addr);
          // one K16 step: +32 bytes inside a K-major row (+2 in the address
          // field); +16 rows of 128 bytes in an MN-major tile (+128)
          constexpr uint64_t a_step = Tr::A_MN ? 128 : 2;
          constexpr uint64_t b_step = Tr::B_MN ? 128 : 2;
#pragma unroll
          for (int k = 0; k < kWBK / 16; ++k) {
            if (PAIR)
              sm100::umma_f16_pair(d_tmem, adesc + a_step * k, bdesc + b_step * k, idesc,
                                   (kb | k) != 0);
            else
              sm100::umma_f16(d_tmem, adesc + a_step * k, bdesc + b_step * k, idesc,
                              (kb | k) != 0);
          }
          if (PAIR) sm100::umma_commit_pair_mc(&st->empty[stage], 0x3);
          else sm100::umma_commit(&st->empty[stage]);
          if (++stage == R::stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (PAIR) sm100::umma_commit_pair_mc(&st->tfull[acc], 0x3);
        else sm100::umma_commit(&st->tfull[acc]);
      }
      if (PAIR) sm100::umma_commit_pair_mc(&st->drain, 0x1);
      else sm100::umma_commit(&st->drain);
      const uint64_t t0 = global_timer_ns();
      while (!sm100::mbar_try_wait(&st->drain, 0) && global_timer_ns() - t0 < kWWaitNs) {
      }
    }
  } else {
    // two epilogue warps per TMEM lane quadrant (a warp reaches lanes
    // 32 * (warp % 4) and up), each taking half of the tile's columns
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row_in_tile = q * 32 + lane;
    int used = 0;
    int sbuf = 0;  // weight gradients: the staging block to fill next
    for (int tile = first; tile < total; tile += stride) {
      const BTile t = decode<MODE, PAIR>(tile, p, st, routed, rank);
      if (Tr::WGRAD && t.skip) {
        __nv_bfloat16* orow = wgrad_row(p, t, t.m0 + row_in_tile);
        if (orow) {
          const uint4 z = make_uint4(0, 0, 0, 0);
          for (int cc = half * (kWBN / 2); cc < (half + 1) * (kWBN / 2) && t.n0 + cc < p.ld_w;
               cc += 8)
            *reinterpret_cast<uint4*>(orow + t.n0 + cc) = z;
        }
        continue;
      }
      const int acc = used & 1;
      const uint32_t acc_phase = (uint32_t)(used >> 1) & 1u;
      ++used;
      if (!bwait<PAIR>(&st->tfull[acc], acc_phase, st, p.err, kErrGemmTimeout | 0x54)) break;
      sm100::tc_fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * kWBN);
      if (Tr::WGRAD) {
        // 64 columns at a time: each thread packs its row's 128 bytes into
        // one of the warp's two staging blocks in the 128-byte-swizzled
        // layout (16-byte piece j of row r at piece j ^ (r % 8)), and lane 0
        // stores the block with one TMA copy; the block is rewritten only
        // once that copy has finished reading it
        const int grp = t.m0 + q * 32;  // the warp's 32 rows never straddle m_split or m_total
        const bool hi = grp >= p.m_split;
        const CUtensorMap* om = t.shared ? (hi ? tmO3 : tmO2) : (hi ? tmO1 : tmO0);
        const int orow = t.expert * (hi ? p.m_total - p.m_split : p.m_split) +
                         (hi ? grp - p.m_split : grp);
        // rows past the end (an output of fewer rows than the tile) store
        // nothing, so every staging block that is written is also stored
        // and the two blocks strictly alternate between committed copies
#pragma unroll 1
        for (int cc = half * (kWBN / 2); cc < (half + 1) * (kWBN / 2) && grp < p.m_total;
             cc += 64) {
          if (t.n0 + cc >= p.ld_w) break;
          uint32_t v[32], w[32];
          sm100::tmem_ld_32x32b_x32(tbase + cc, v);
          sm100::tmem_ld_32x32b_x32(tbase + cc + 32, w);
          sm100::tmem_ld_wait();
          unsigned char* stg = wstage + ((warp - 2) * 2 + sbuf) * (32 * 128);
          if (lane == 0) sm100::bulk_wait_read_1();
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint32_t* src = j < 4 ? v + 8 * j : w + 8 * (j - 4);
            const uint4 pk = make_uint4(
                pack_bf16x2(__uint_as_float(src[0]), __uint_as_float(src[1])),
                pack_bf16x2(__uint_as_float(src[2]), __uint_as_float(src[3])),
                pack_bf16x2(__uint_as_float(src[4]), __uint_as_float(src[5])),
                pack_bf16x2(__uint_as_float(src[6]), __uint_as_float(src[7])));
            *reinterpret_cast<uint4*>(stg + lane * 128 + ((j ^ (lane & 7)) * 16)) = pk;
          }
          sm100::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            sm100::tma_store_2d(om, t.n0 + cc, orow, stg);
            sm100::bulk_commit_group();
          }
          sbuf ^= 1;
        }
      } else if (t.valid) {
        row_epilogue<MODE>(p, t, tbase, row_in_tile, half);
      }
      sm100::tc_fence_before();
      if (PAIR) sm100::mbar_arrive_cluster(sm100::mapa_shared(sm100::smem_addr(&st->tempty[acc]), 0));
      else sm100::mbar_arrive(&st->tempty[acc]);
    }
    // the weight gradients' TMA stores complete before the CTA exits
    if (Tr::WGRAD && lane == 0) sm100::bulk_wait_all();
  }
  sm100::tc_fence_before();
  __syncthreads();
  if (PAIR) sm100::cluster_sync();  // no CTA leaves while its peer may still signal it
  if (warp == 1) {
    sm100::tc_fence_after();
    if (PAIR) sm100::tmem_dealloc_pair(tmem, 512);
    else sm100::tmem_dealloc(tmem, 512);
  }
}

__device__ __forceinline__ unsigned char* aligned_smem(unsigned char* p) {
  return reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(p) + 1023) &
                                          ~uintptr_t(1023));
}

template <int MODE>
__global__ void __launch_bounds__(kWThreads, 1)
    tc_bwd_gemm_kernel(const __grid_constant__ CUtensorMap tmA0,
                       const __grid_constant__ CUtensorMap tmA1,
                       const __grid_constant__ CUtensorMap tmB0,
                       const __grid_constant__ CUtensorMap tmB0g,
                       const __grid_constant__ CUtensorMap tmB1,
                       const __grid_constant__ CUtensorMap tmB1g,
                       const __grid_constant__ CUtensorMap tmO0,
                       const __grid_constant__ CUtensorMap tmO1,
                       const __grid_constant__ CUtensorMap tmO2,
                       const __grid_constant__ CUtensorMap tmO3, const BwdParams p) {
  extern __shared__ __align__(1024) unsigned char bsm[];
  bwd_body<MODE, false>(&tmA0, &tmA1, &tmB0, &tmB0g, &tmB1, &tmB1g, &tmO0, &tmO1, &tmO2, &tmO3,
                        p, aligned_smem(bsm));
}

// CTA pairs (cta_group::2): each CTA loads its 128 rows of A and one half
// (128 columns) of B; the leader issues M=256 MMAs; both CTAs' copies
// complete on the leader's stage barrier, commits arrive on both CTAs'
// barriers, both epilogues release the accumulator on the leader's.
template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kWThreads, 1)
    tc_bwd_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA0,
                            const __grid_constant__ CUtensorMap tmA1,
                            const __grid_constant__ CUtensorMap tmB0,
                            const __grid_constant__ CUtensorMap tmB0g,
                            const __grid_constant__ CUtensorMap tmB1,
                            const __grid_constant__ CUtensorMap tmB1g,
                            const __grid_constant__ CUtensorMap tmO0,
                            const __grid_constant__ CUtensorMap tmO1,
                            const __grid_constant__ CUtensorMap tmO2,
                            const __grid_constant__ CUtensorMap tmO3, const BwdParams p) {
  extern __shared__ __align__(1024) unsigned char bsm[];
  bwd_body<MODE, true>(&tmA0, &tmA1, &tmB0, &tmB0g, &tmB1, &tmB1g, &tmO0, &tmO1, &tmO2, &tmO3,
                       p, aligned_smem(bsm));
}

}  // namespace

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
template <int MODE, bool PAIR>
static cudaError_t launch_bwd(const BwdMaps& m, const BwdParams& p, cudaStream_t s) {
  using R = Ring<PAIR, ModeTraits<MODE>::WGRAD>;
  const size_t bytes = (size_t)R::stages * R::stage_bytes + (kStateBytes + 1023) / 1024 * 1024 +
                       (ModeTraits<MODE>::WGRAD ? kWStageOut : 0) + 1024;
  auto kern = PAIR ? tc_bwd_gemm_pair_kernel<MODE> : tc_bwd_gemm_kernel<MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  long long tiles;
  if (ModeTraits<MODE>::WGRAD) {
    tiles = (long long)(p.E + p.n_shared) * p.mt_tiles * p.nt_tiles;
  } else {
    const long long blocks = PAIR ? p.max_routed_blocks + p.E : p.max_routed_blocks;
    const long long sb = PAIR ? (p.shared_blocks + 1) / 2 : p.shared_blocks;
    tiles = blocks * p.nt_tiles + (long long)p.n_shared * sb * p.nt_tiles;
  }
  const long long slots = PAIR ? sms / 2 : sms;
  const long long units = tiles < slots ? (tiles < 1 ? 1 : tiles) : slots;
  const int grid = (int)(PAIR ? 2 * units : units);
  return launch_pdl(kern, grid, kWThreads, bytes, s, m.a0, m.a1, m.b0, m.b0g, m.b1, m.b1g, m.o0,
                    m.o1, m.o2, m.o3, p);
}

template <bool PAIR>
static cudaError_t run_bwd_gemm_t(int mode, const BwdMaps& m, const BwdParams& p,
                                  cudaStream_t s) {
  switch (mode) {
    case BW_SAVE: return launch_bwd<BW_SAVE, PAIR>(m, p, s);
    case BW_DACT: return launch_bwd<BW_DACT, PAIR>(m, p, s);
    case BW_DX: return launch_bwd<BW_DX, PAIR>(m, p, s);
    case BW_WG2: return launch_bwd<BW_WG2, PAIR>(m, p, s);
    default: return launch_bwd<BW_WG13, PAIR>(m, p, s);
  }
}

cudaError_t run_bwd_gemm(int mode, bool pair, const BwdMaps& m, const BwdParams& p,
                         cudaStream_t s) {
  return pair ? run_bwd_gemm_t<true>(mode, m, p, s) : run_bwd_gemm_t<false>(mode, m, p, s);
}

}  // namespace moe
