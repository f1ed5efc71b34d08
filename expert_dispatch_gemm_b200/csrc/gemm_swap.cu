// Grouped expert GEMMs for fine-grained experts with the weights as the M
// side: the SwiGLU up projection, the down projection, and the backward's
// dX_perm.
//
// "Expert choice routing" (aicassindra.com), "The math: a gating matrix and
// top-k over tokens": each expert's gathered rows form a dense batch; here
// each product is taken transposed (Y_e^T = W2_e H_e^T, H_e^T = silu(W1_e
// X_e^T) * (W3_e X_e^T), dX_e^T = W1_e^T dU_e^T + W3_e^T dV_e^T), so that an
// expert's tokens are the N side of the MMA and need only 16-row granularity,
// where the 128-row M tiles of the token-side kernels round an expert of ~256
// rows up to 384 or 512.
//
// CTA pairs (cta_group::2). A tile is (expert, 256 weight rows, up to 256 of
// the expert's tokens): each CTA loads its 128 weight rows as A and half of
// the tile's tokens as B (exactly its N/2 rows), and the MMA is M=256 with
// N = tokens (a multiple of 16).
//
// On B200 one thread issues at most one tcgen05.mma about every 95 cycles,
// whatever N is, while an M=256 pair MMA needs N/2 cycles of the tensor
// pipe: below N = 192 a single issuer leaves the pipe idle, and the token
// chunks of experts with more than 256 rows are 128-160 wide. Two issuers
// on independent accumulators keep it busy down to N = 128. So:
// - tc_swap_pair_kernel (down projection; backward dX with the weights read
//   MN-major) runs two tile streams, each with its own producer,
//   shared-memory ring and 256-column TMEM accumulator; stream s takes every
//   other tile of the pair.
//     warps 0 / 2   TMA producers of streams 0 / 1 (3-stage rings of 32 KB:
//                   A 16 KB + B up to 16 KB);
//     warps 1 / 3   the leader's lane 0 issues the MMAs of stream 0 / 1
//                   (warp 1 also holds the TMEM allocation);
//     warps 4-11    epilogue, four per stream (one per TMEM lane quadrant):
//                   tcgen05.ld 32 tokens at a time, a transpose through
//                   shared memory, and 16-byte stores of each token's 32
//                   consecutive output columns.
//   While one stream's epilogue drains its accumulator the other stream
//   keeps the tensor pipe busy.
// - tc_swap_up_pair_kernel (SwiGLU up projection) loads W1 and W3 rows as
//   two A operands of one stage and issues their MMAs from two threads into
//   two accumulators (U, V), which meet in one epilogue thread.
// Every mbarrier wait is bounded, as in the other GEMM kernels.
#include <cuda.h>
#include <math.h>

#include "device_common.cuh"
#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {

namespace {

// warps: 0/2 producers, 1/3 MMA issuers, 4-11 epilogue (streams 0 and 1)
constexpr int kSBK = 64, kSStages = 3, kSStreams = 2, kSEpiWarps = 8;
constexpr int kSThreads = 32 * (4 + kSEpiWarps);
constexpr int kSABytes = 128 * kSBK * 2;         // this CTA's 128 weight rows
constexpr int kSBBytes = 128 * kSBK * 2;         // up to 128 token rows
constexpr int kSStageBytes = kSABytes + kSBBytes;
constexpr int kSTmemCols = 512;                  // one 256-column accumulator per stream
constexpr int kSMaxTokens = 256;                 // tokens per tile (MMA N <= 256)
constexpr uint64_t kSWaitNs = 2000000000ull;     // 2 s

struct SwapParams {
  const int32_t* offsets;   // [E+1] segment starts
  const int32_t* counts;    // [E] tokens of each expert (kept rows)
  int E, K;                 // reduction length (multiple of 64)
  int m_per_expert;         // weight rows (outputs) per expert: d
  int mt_tiles;             // 256-row weight tiles per expert
  int n_shared, n;          // shared experts run over all n tokens
  long long shared_in_row;  // shared experts' token rows: base + s * stride
  long long shared_in_stride;
  long long shared_out_row; // shared experts' output rows: base + s * n_pad
  long long n_pad;
  int n_out;                // output row pitch (d)
  __nv_bfloat16* out;
  int* err;
  // MN-major weights (the backward's dX = dU W1 + dV W3): K index where the
  // second weight matrix takes over, and K rows per expert in the maps
  int k_split;
  int w_k_rows;
};

struct SwapState {
  uint64_t full[kSStreams][kSStages];
  uint64_t empty[kSStreams][kSStages];
  uint64_t tfull[kSStreams];
  uint64_t tempty[kSStreams];
  uint64_t drain[kSStreams];
  uint32_t tmem_base;
  volatile int abort_flag;
  int offs[MOE_MAX_EXPERTS + 1];
  int cnt[MOE_MAX_EXPERTS];
  int tprefix[MOE_MAX_EXPERTS + 1];  // tiles of the experts before e
};

template <bool CLUSTER_ACQUIRE, class State>
__device__ __forceinline__ bool swap_wait(uint64_t* bar, uint32_t parity, State* st, int* err,
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
      if (global_timer_ns() - t0 > kSWaitNs) {
        st->abort_flag = 1;
        report_error(err, code);
        return false;
      }
    }
  }
}

struct SwapTile {
  bool shared;
  int expert;          // routed expert, or shared expert index
  int m0;              // first weight row of the pair (within the expert)
  long long tok_row;   // first token row of the tile in the B source
  long long out_row;   // output row of the tile's first token
  int valid;           // tokens of the tile that are real
  int n;               // MMA N: valid rounded up to 16
};

// Tile order: expert by expert, weight tile by weight tile, token chunks
// innermost; shared experts last. An expert's tokens split into
// ceil(count / 256) chunks of equal size (rounded up to 16), so that 272
// tokens become 144 + 128 rather than 256 + 16.
template <class State>
__device__ __forceinline__ SwapTile decode_swap(int tile, const SwapParams& p, const State* st,
                                               int routed) {
  SwapTile t;
  int chunk, chunks, count;
  if (tile < routed) {
    int lo = 0, hi = p.E - 1;  // largest e with tprefix[e] <= tile
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (st->tprefix[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    count = st->cnt[lo];
    chunks = max((count + kSMaxTokens - 1) / kSMaxTokens, 1);
    const int local = tile - st->tprefix[lo];
    t.shared = false;
    t.expert = lo;
    t.m0 = (local / chunks) * (2 * 128);
    chunk = local % chunks;
    t.tok_row = st->offs[lo];
    t.out_row = t.tok_row;
  } else {
    count = p.n;
    chunks = (count + kSMaxTokens - 1) / kSMaxTokens;
    const int per = p.mt_tiles * chunks;
    const int q = tile - routed;
    const int s = q / per, local = q % per;
    t.shared = true;
    t.expert = s;
    t.m0 = (local / chunks) * (2 * 128);
    chunk = local % chunks;
    t.tok_row = p.shared_in_row + s * p.shared_in_stride;
    t.out_row = p.shared_out_row + s * p.n_pad;
  }
  const int size = (((count + chunks - 1) / chunks) + 15) & ~15;  // <= 256
  const int first = chunk * size;
  t.tok_row += first;
  t.out_row += first;
  t.valid = min(size, count - first);
  t.n = (t.valid + 15) & ~15;
  return t;
}

// The token operand: a CTA loads exactly its N/2 rows (a multiple of 8, at
// most 128) as boxes of 128, 64, 32, 16 and 8 rows, each at a 1 KB-aligned
// shared-memory offset (whole 8-row atoms of the 128-byte swizzle, so the
// tile is laid out as one box would lay it out), all completing on the
// leader's barrier `fl`.
constexpr int kTokBoxes = 5;
struct TokenMaps {
  CUtensorMap m[kTokBoxes];  // box of 8 << b rows
};

__device__ __forceinline__ void load_token_rows(unsigned char* dst, const TokenMaps& tk,
                                                uint32_t fl, int x, long long row0, int rows) {
  int off = 0;
#pragma unroll
  for (int b = kTokBoxes - 1; b >= 0; --b) {
    const int r = 8 << b;
    if (rows & r) {
      sm100::tma_load_2d_pair(dst + off * 128, &tk.m[b], fl, x, (int)(row0 + off));
      off += r;
    }
  }
}

// token maps: tk / tks = routed / shared token rows of the B source; weights:
// tmW (routed) / tmWs (shared), K-major boxes of 128 rows. A_MN: the weights
// are read MN-major (the backward's dX^T = W1^T dU^T + W3^T dV^T: W1 and W3
// stored [h, d], the output index d contiguous) as two 64 x 64 boxes per
// stage, from tmW / tmWs below K = k_split and tmW3 / tmW3s above it.
template <bool A_MN>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kSThreads, 1)
    tc_swap_pair_kernel(const __grid_constant__ TokenMaps tk,
                        const __grid_constant__ TokenMaps tks,
                        const __grid_constant__ CUtensorMap tmW,
                        const __grid_constant__ CUtensorMap tmW3,
                        const __grid_constant__ CUtensorMap tmWs,
                        const __grid_constant__ CUtensorMap tmW3s, const SwapParams p) {
  extern __shared__ __align__(1024) unsigned char ssm[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(ssm) + 1023) & ~uintptr_t(1023));
  constexpr int kRingBytes = kSStreams * kSStages * kSStageBytes;
  SwapState* st = reinterpret_cast<SwapState*>(base + kRingBytes);
  // epilogue staging, [8 warps][32 tokens][32 columns] bf16
  __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(
      base + kRingBytes + ((sizeof(SwapState) + 127) & ~size_t(127)));
  auto sA = [&](int sx, int j) { return base + (sx * kSStages + j) * kSStageBytes; };
  auto sB = [&](int sx, int j) { return sA(sx, j) + kSABytes; };

  const uint32_t rank = sm100::cluster_ctarank();
  const bool leader = rank == 0;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int sx = 0; sx < kSStreams; ++sx) {
      for (int j = 0; j < kSStages; ++j) {
        sm100::mbar_init(&st->full[sx][j], 1);
        sm100::mbar_init(&st->empty[sx][j], 1);
      }
      sm100::mbar_init(&st->tfull[sx], 1);
      // every thread of the stream's epilogue warps, in both CTAs
      sm100::mbar_init(&st->tempty[sx], 2 * 32 * (kSEpiWarps / kSStreams));
      sm100::mbar_init(&st->drain[sx], 1);
    }
    st->abort_flag = 0;
    sm100::fence_mbar_init();
  }
  if (warp == 1) {
    sm100::tmem_alloc_pair(&st->tmem_base, kSTmemCols);
    sm100::tmem_relinquish_pair();
  }
  // the set-up above needs nothing from the previous kernel; the segment
  // starts, the counts and the token rows are read from here on
  pdl_wait();
  for (int i = tid; i <= p.E; i += kSThreads) st->offs[i] = p.offsets[i];
  for (int i = tid; i < p.E; i += kSThreads) {
    const int seg = p.offsets[i + 1] - p.offsets[i];
    const int c = p.counts ? p.counts[i] : seg;
    if (seg < 0 || c < 0 || c > seg) bad_index(p.err, kSiteSwapOffsets);
    st->cnt[i] = max(0, min(c, seg));  // never past the expert's own segment
  }
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int e = 0; e < p.E; ++e) {
      st->tprefix[e] = run;
      run += (st->cnt[e] + kSMaxTokens - 1) / kSMaxTokens * p.mt_tiles;
    }
    st->tprefix[p.E] = run;
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::cluster_sync();  // both CTAs' barriers exist before any remote arrive
  sm100::tc_fence_after();
  const uint32_t tmem = st->tmem_base;

  const int routed = st->tprefix[p.E];
  const int shared_chunks = (p.n + kSMaxTokens - 1) / kSMaxTokens;
  const int total = routed + p.n_shared * p.mt_tiles * shared_chunks;
  const int KB = p.K / kSBK;
  const int pair_id = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;
  // the pair's tiles are pair_id + i * num_pairs; stream sx takes i = sx, sx + 2, ...
  const int sx = warp < 4 ? (warp >> 1) : (warp - 4) / (kSEpiWarps / kSStreams);
  const int first = pair_id + sx * num_pairs, step = kSStreams * num_pairs;

  if (warp < 4 && (warp & 1) == 0) {
    // producer of stream sx
    if (lane == 0) {
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = first; ok && tile < total; tile += step) {
        const SwapTile t = decode_swap(tile, p, st, routed);
        const TokenMaps& tmk = t.shared ? tks : tk;
        const int half_rows = t.n / 2;  // this CTA's token rows
        const uint32_t bytes = kSABytes + (uint32_t)half_rows * kSBK * 2;
        const CUtensorMap* mw = t.shared ? &tmWs : &tmW;
        const int wrow = t.expert * p.m_per_expert + t.m0 + (int)rank * 128;  // this CTA's 128
        // this CTA's half of the tile's tokens
        const long long trow1 = t.tok_row + (long long)rank * (t.n / 2);
        for (int kb = 0; kb < KB; ++kb) {
          if (!swap_wait<false>(&st->empty[sx][stage], phase ^ 1u, st, p.err,
                                kErrGemmTimeout | 0xA1)) {
            ok = false;
            break;
          }
          const uint32_t fl = sm100::mapa_shared(sm100::smem_addr(&st->full[sx][stage]), 0);
          if (leader) sm100::mbar_arrive_expect_tx(&st->full[sx][stage], 2 * bytes);
          if (A_MN) {
            const int k0 = kb * kSBK;
            const bool second = k0 >= p.k_split;
            const CUtensorMap* mk = t.shared ? (second ? &tmW3s : &tmWs) : (second ? &tmW3 : &tmW);
            const int ky = t.expert * p.w_k_rows + (second ? k0 - p.k_split : k0);
            const int mx = t.m0 + (int)rank * 128;  // this CTA's 128 outputs, two 64-wide boxes
            sm100::tma_load_2d_pair(sA(sx, stage), mk, fl, mx, ky);
            sm100::tma_load_2d_pair(sA(sx, stage) + sm100::kMnChunkBytes, mk, fl, mx + 64, ky);
          } else {
            sm100::tma_load_2d_pair(sA(sx, stage), mw, fl, kb * kSBK, wrow);
          }
          load_token_rows(sB(sx, stage), tmk, fl, kb * kSBK, trow1, half_rows);
          ++issued;
          if (++stage == kSStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok && leader) {
        // wait (bounded) until the copies of the outstanding stages have landed
        int j = stage;
        uint32_t ph = phase;
        const int pending = issued < kSStages ? issued : kSStages;
        for (int i = 0; i < pending; ++i) {
          if (--j < 0) {
            j = kSStages - 1;
            ph ^= 1u;
          }
          const uint64_t t0 = global_timer_ns();
          while (!sm100::mbar_try_wait(&st->full[sx][j], ph) && global_timer_ns() - t0 < kSWaitNs) {
          }
        }
      }
    }
  } else if (warp < 4) {
    // MMA issuer of stream sx: the leader's lane 0
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      const uint32_t d_tmem = tmem + (uint32_t)(sx * 256);
      for (int tile = first; ok && tile < total; tile += step, ++local) {
        const SwapTile t = decode_swap(tile, p, st, routed);
        // the accumulator is free once both CTAs' epilogues drained the last tile
        if (!swap_wait<true>(&st->tempty[sx], ((uint32_t)local & 1u) ^ 1u, st, p.err,
                             kErrGemmTimeout | 0xB2)) {
          ok = false;
          break;
        }
        sm100::tc_fence_after();
        // bit 15: A MN-major
        const uint32_t idesc = sm100::idesc_bf16_f32(256, t.n) | (A_MN ? (1u << 15) : 0u);
        for (int kb = 0; kb < KB; ++kb) {
          if (!swap_wait<false>(&st->full[sx][stage], phase, st, p.err, kErrGemmTimeout | 0xB3)) {
            ok = false;
            break;
          }
          sm100::tc_fence_after();
          const uint32_t a_addr = sm100::smem_addr(sA(sx, stage));
          const uint64_t adesc =
              A_MN ? sm100::sw128_mnmajor_desc(a_addr) : sm100::sw128_kmajor_desc(a_addr);
          const uint64_t bdesc = sm100::sw128_kmajor_desc(sm100::smem_addr(sB(sx, stage)));
          // one K16 step: +32 bytes in a K-major row, +16 rows in an MN-major tile
          constexpr uint64_t a_step = A_MN ? 128 : 2;
#pragma unroll
          for (int k = 0; k < kSBK / 16; ++k)
            sm100::umma_f16_pair(d_tmem, adesc + a_step * k, bdesc + 2 * k, idesc, (kb | k) != 0);
          sm100::umma_commit_pair_mc(&st->empty[sx][stage], 0x3);
          if (++stage == kSStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        sm100::umma_commit_pair_mc(&st->tfull[sx], 0x3);
      }
      sm100::umma_commit_pair_mc(&st->drain[sx], 0x1);
      const uint64_t t0 = global_timer_ns();
      while (!sm100::mbar_try_wait(&st->drain[sx], 0) && global_timer_ns() - t0 < kSWaitNs) {
      }
    }
  } else {
    // epilogue of stream sx: TMEM lanes = this CTA's 128 weight rows (output
    // columns), TMEM columns = tokens; warp q = warp % 4 owns lanes
    // 32q..32q+31 and walks all the tile's tokens, 32 at a time
    const int q = warp & 3;
    constexpr int CW = 32;  // output columns per warp
    constexpr int VPR = CW * 2 / 16;  // 16-byte pieces of a token's CW columns
    __nv_bfloat16* stg = stage + (warp - 4) * (32 * CW);  // [32 tokens][CW] bf16
    int local = 0;
    for (int tile = first; tile < total; tile += step, ++local) {
      const SwapTile t = decode_swap(tile, p, st, routed);
      const int col0 = t.m0 + (int)rank * 128 + 32 * q;
      __nv_bfloat16* outt = p.out + (size_t)t.out_row * p.n_out + col0;
      if (!swap_wait<true>(&st->tfull[sx], (uint32_t)local & 1u, st, p.err, kErrGemmTimeout | 0xC4))
        break;
      sm100::tc_fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(sx * 256);
#pragma unroll 1
      for (int cc = 0; cc < t.n; cc += 32) {
        uint32_t v[32];
        sm100::tmem_ld_32x32b_x32(tbase + cc, v);
        sm100::tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) stg[i * CW + lane] = __float2bfloat16_rn(__uint_as_float(v[i]));
        __syncwarp();
        // each token's CW columns leave as 16-byte stores
#pragma unroll
        for (int idx = lane; idx < 32 * VPR; idx += 32) {
          const int i = idx / VPR, vv = idx % VPR;
          const int j = cc + i;  // token within the tile
          if (j < t.valid)
            *reinterpret_cast<uint4*>(outt + (size_t)j * p.n_out + vv * 8) =
                *reinterpret_cast<const uint4*>(stg + i * CW + vv * 8);
        }
        __syncwarp();
      }
      sm100::tc_fence_before();
      sm100::mbar_arrive_cluster(sm100::mapa_shared(sm100::smem_addr(&st->tempty[sx]), 0));
    }
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::cluster_sync();  // no CTA leaves while its peer may still signal it
  if (warp == 1) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc_pair(tmem, kSTmemCols);
  }
}

// ---------------------------------------------------------------------------
// SwiGLU up projection with the weights as the M side: H_e^T = silu(W1_e
// X_e^T) * (W3_e X_e^T). A tile is (expert, 256 hidden units, up to 256 of
// the expert's tokens). Each CTA loads its 128 rows of W1 and the same 128
// rows of W3 as two A operands and half of the tile's tokens as B. Two
// threads of the leader issue the MMAs: one the W1 products into TMEM
// columns [0, 256) (the gate pre-activation U), the other the W3 products
// into [256, 512) (V), both from the same stage, so a hidden unit's U and V
// sit in one TMEM lane and meet in one epilogue thread, and the tensor pipe
// sees two issuers (a single one cannot feed it below N = 192). The 512
// columns hold one tile; the producer runs ahead into the next tile's stages
// while the epilogue drains.
//   warp 0     TMA producer (4-stage ring: W1 16 KB + W3 16 KB + tokens <= 16 KB);
//   warp 1     TMEM allocation; the leader's lane 0 issues the W1 MMAs;
//   warp 2     the leader's lane 0 issues the W3 MMAs;
//   warp 3     idle;
//   warps 4-11 epilogue, two per TMEM lane quadrant on alternate 32-token
//              groups: U and V 32 tokens at a time, silu(U) V in fp32, bf16,
//              a transpose through shared memory, and 16-byte stores of each
//              token's 32 consecutive hidden units.
// ---------------------------------------------------------------------------
constexpr int kUStages = 4, kUEpiWarps = 8, kUThreads = 32 * (4 + kUEpiWarps);
constexpr int kUWBytes = 128 * kSBK * 2;                       // 128 rows of W1 or W3
constexpr int kUStageBytes = 2 * kUWBytes + kSBBytes;          // 48 KB

struct UpState {
  uint64_t full[kUStages];
  uint64_t empty[kUStages];   // released by both issuers' commits
  uint64_t tfull;             // both issuers' last commits of a tile
  uint64_t tempty;            // both CTAs' epilogues
  uint64_t drain[2];
  uint32_t tmem_base;
  volatile int abort_flag;
  int offs[MOE_MAX_EXPERTS + 1];
  int cnt[MOE_MAX_EXPERTS];
  int tprefix[MOE_MAX_EXPERTS + 1];
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kUThreads, 1)
    tc_swap_up_pair_kernel(const __grid_constant__ TokenMaps tk,
                           const __grid_constant__ TokenMaps tks,
                           const __grid_constant__ CUtensorMap tmW1,
                           const __grid_constant__ CUtensorMap tmW3,
                           const __grid_constant__ CUtensorMap tmW1s,
                           const __grid_constant__ CUtensorMap tmW3s, const SwapParams p) {
  extern __shared__ __align__(1024) unsigned char usm[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(usm) + 1023) & ~uintptr_t(1023));
  UpState* st = reinterpret_cast<UpState*>(base + kUStages * kUStageBytes);
  // epilogue staging, [8 warps][32 tokens][32 hidden units] bf16
  __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(
      base + kUStages * kUStageBytes + ((sizeof(UpState) + 127) & ~size_t(127)));
  auto sW = [&](int j, int which) { return base + j * kUStageBytes + which * kUWBytes; };
  auto sB = [&](int j) { return base + j * kUStageBytes + 2 * kUWBytes; };

  const uint32_t rank = sm100::cluster_ctarank();
  const bool leader = rank == 0;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int j = 0; j < kUStages; ++j) {
      sm100::mbar_init(&st->full[j], 1);
      sm100::mbar_init(&st->empty[j], 2);
    }
    sm100::mbar_init(&st->tfull, 2);
    sm100::mbar_init(&st->tempty, 2 * 32 * kUEpiWarps);  // both CTAs' epilogues
    sm100::mbar_init(&st->drain[0], 1);
    sm100::mbar_init(&st->drain[1], 1);
    st->abort_flag = 0;
    sm100::fence_mbar_init();
  }
  if (warp == 1) {
    sm100::tmem_alloc_pair(&st->tmem_base, kSTmemCols);
    sm100::tmem_relinquish_pair();
  }
  // the set-up above needs nothing from the previous kernel; the segment
  // starts, the counts and the dispatched rows are read from here on
  pdl_wait();
  for (int i = tid; i <= p.E; i += kUThreads) st->offs[i] = p.offsets[i];
  for (int i = tid; i < p.E; i += kUThreads) {
    const int seg = p.offsets[i + 1] - p.offsets[i];
    const int c = p.counts ? p.counts[i] : seg;
    if (seg < 0 || c < 0 || c > seg) bad_index(p.err, kSiteSwapOffsets);
    st->cnt[i] = max(0, min(c, seg));  // never past the expert's own segment
  }
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int e = 0; e < p.E; ++e) {
      st->tprefix[e] = run;
      run += (st->cnt[e] + kSMaxTokens - 1) / kSMaxTokens * p.mt_tiles;
    }
    st->tprefix[p.E] = run;
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::cluster_sync();  // both CTAs' barriers exist before any remote arrive
  sm100::tc_fence_after();
  const uint32_t tmem = st->tmem_base;

  const int routed = st->tprefix[p.E];
  const int shared_chunks = (p.n + kSMaxTokens - 1) / kSMaxTokens;
  const int total = routed + p.n_shared * p.mt_tiles * shared_chunks;
  const int KB = p.K / kSBK;
  const int pair_id = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = pair_id; ok && tile < total; tile += num_pairs) {
        const SwapTile t = decode_swap(tile, p, st, routed);
        const TokenMaps& tmk = t.shared ? tks : tk;
        const int half_rows = t.n / 2;  // this CTA's token rows
        const uint32_t bytes = 2 * kUWBytes + (uint32_t)half_rows * kSBK * 2;
        const CUtensorMap* mw1 = t.shared ? &tmW1s : &tmW1;
        const CUtensorMap* mw3 = t.shared ? &tmW3s : &tmW3;
        const int wrow = t.expert * p.m_per_expert + t.m0 + (int)rank * 128;  // this CTA's 128
        // this CTA's half of the tile's tokens
        const long long trow1 = t.tok_row + (long long)rank * (t.n / 2);
        for (int kb = 0; kb < KB; ++kb) {
          if (!swap_wait<false>(&st->empty[stage], phase ^ 1u, st, p.err, kErrGemmTimeout | 0xD1)) {
            ok = false;
            break;
          }
          const uint32_t fl = sm100::mapa_shared(sm100::smem_addr(&st->full[stage]), 0);
          if (leader) sm100::mbar_arrive_expect_tx(&st->full[stage], 2 * bytes);
          sm100::tma_load_2d_pair(sW(stage, 0), mw1, fl, kb * kSBK, wrow);
          sm100::tma_load_2d_pair(sW(stage, 1), mw3, fl, kb * kSBK, wrow);
          load_token_rows(sB(stage), tmk, fl, kb * kSBK, trow1, half_rows);
          ++issued;
          if (++stage == kUStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok && leader) {
        // wait (bounded) until the copies of the outstanding stages have landed
        int j = stage;
        uint32_t ph = phase;
        const int pending = issued < kUStages ? issued : kUStages;
        for (int i = 0; i < pending; ++i) {
          if (--j < 0) {
            j = kUStages - 1;
            ph ^= 1u;
          }
          const uint64_t t0 = global_timer_ns();
          while (!sm100::mbar_try_wait(&st->full[j], ph) && global_timer_ns() - t0 < kSWaitNs) {
          }
        }
      }
    }
  } else if (warp == 1 || warp == 2) {
    // issuer `which`: W1 products into columns [0, 256), W3 into [256, 512)
    if (lane == 0 && leader) {
      const int which = warp - 1;
      const uint32_t d_tmem = tmem + (uint32_t)(which * 256);
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int tile = pair_id; ok && tile < total; tile += num_pairs, ++local) {
        const SwapTile t = decode_swap(tile, p, st, routed);
        if (!swap_wait<true>(&st->tempty, ((uint32_t)local & 1u) ^ 1u, st, p.err,
                             kErrGemmTimeout | 0xE2)) {
          ok = false;
          break;
        }
        sm100::tc_fence_after();
        const uint32_t idesc = sm100::idesc_bf16_f32(256, t.n);
        for (int kb = 0; kb < KB; ++kb) {
          if (!swap_wait<false>(&st->full[stage], phase, st, p.err, kErrGemmTimeout | 0xE3)) {
            ok = false;
            break;
          }
          sm100::tc_fence_after();
          const uint64_t da = sm100::sw128_kmajor_desc(sm100::smem_addr(sW(stage, which)));
          const uint64_t db = sm100::sw128_kmajor_desc(sm100::smem_addr(sB(stage)));
#pragma unroll
          for (int k = 0; k < kSBK / 16; ++k)
            sm100::umma_f16_pair(d_tmem, da + 2 * k, db + 2 * k, idesc, (kb | k) != 0);
          sm100::umma_commit_pair_mc(&st->empty[stage], 0x3);
          if (++stage == kUStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        sm100::umma_commit_pair_mc(&st->tfull, 0x3);
      }
      sm100::umma_commit_pair_mc(&st->drain[which], 0x1);
      const uint64_t t0 = global_timer_ns();
      while (!sm100::mbar_try_wait(&st->drain[which], 0) && global_timer_ns() - t0 < kSWaitNs) {
      }
    }
  } else if (warp >= 4) {
    // epilogue: TMEM lanes = this CTA's 128 hidden units, columns = tokens
    // (U in [0, 256), V in [256, 512)); warps q and q + 4 own lanes
    // 32q..32q+31 (q = warp % 4) and take alternate 32-token groups
    const int q = warp & 3;
    const int half = (warp - 4) >> 2;
    constexpr int CW = 32;            // hidden units per warp
    constexpr int VPR = CW * 2 / 16;  // 16-byte pieces of a token's CW units
    __nv_bfloat16* stg = stage + (warp - 4) * (32 * CW);  // [32 tokens][CW] bf16
    int local = 0;
    for (int tile = pair_id; tile < total; tile += num_pairs, ++local) {
      const SwapTile t = decode_swap(tile, p, st, routed);
      const int col0 = t.m0 + (int)rank * 128 + 32 * q;
      __nv_bfloat16* outt = p.out + (size_t)t.out_row * p.n_out + col0;
      if (!swap_wait<true>(&st->tfull, (uint32_t)local & 1u, st, p.err, kErrGemmTimeout | 0xF4))
        break;
      sm100::tc_fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16);
#pragma unroll 1
      for (int cc = 32 * half; cc < t.n; cc += 64) {
        uint32_t u[32], v[32];
        sm100::tmem_ld_32x32b_x32(tbase + cc, u);
        sm100::tmem_ld_32x32b_x32(tbase + 256u + cc, v);
        sm100::tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float a = __uint_as_float(u[i]);
          const float b = __uint_as_float(v[i]);
          stg[i * CW + lane] = __float2bfloat16_rn(a * __frcp_rn(1.0f + __expf(-a)) * b);
        }
        __syncwarp();
        // each token's CW hidden units leave as 16-byte stores
#pragma unroll
        for (int idx = lane; idx < 32 * VPR; idx += 32) {
          const int i = idx / VPR, vv = idx % VPR;
          const int j = cc + i;  // token within the tile
          if (j < t.valid)
            *reinterpret_cast<uint4*>(outt + (size_t)j * p.n_out + vv * 8) =
                *reinterpret_cast<const uint4*>(stg + i * CW + vv * 8);
        }
        __syncwarp();
      }
      sm100::tc_fence_before();
      sm100::mbar_arrive_cluster(sm100::mapa_shared(sm100::smem_addr(&st->tempty), 0));
    }
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::cluster_sync();  // no CTA leaves while its peer may still signal it
  if (warp == 1) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc_pair(tmem, kSTmemCols);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
struct SwapMaps {
  TokenMaps t, ts;
  CUtensorMap w, ws;
};

template <bool A_MN>
static cudaError_t launch_swap(const SwapMaps& m, const CUtensorMap& w3, const CUtensorMap& w3s,
                               const SwapParams& p, int pairs, cudaStream_t s) {
  const size_t bytes = (size_t)kSStreams * kSStages * kSStageBytes +
                       ((sizeof(SwapState) + 127) & ~size_t(127)) +
                       kSEpiWarps * 32 * 32 * sizeof(__nv_bfloat16) + 1024;
  auto kern = tc_swap_pair_kernel<A_MN>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, 2 * pairs, kSThreads, bytes, s, m.t, m.ts, m.w, w3, m.ws, w3s, p);
}

static bool token_maps(TokenMaps& t, const void* ptr, long long rows, long long cols) {
  for (int b = 0; b < kTokBoxes; ++b)
    if (!make_bf16_sw128_map(&t.m[b], ptr, rows, cols, 8 << b)) return false;
  return true;
}

static int swap_pairs(const SwapParams& p, long long max_routed_rows) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // an upper bound on the tiles: every expert's tokens plus one partial chunk
  const long long chunks = (max_routed_rows + kSMaxTokens - 1) / kSMaxTokens + p.E +
                           (long long)p.n_shared * ((p.n + kSMaxTokens - 1) / kSMaxTokens);
  const long long tiles = chunks * p.mt_tiles;
  const long long g = tiles < sms / 2 ? tiles : sms / 2;
  return g < 1 ? 1 : (int)g;
}


static cudaError_t launch_swap_up(const SwapMaps& m, const CUtensorMap& w3,
                                  const CUtensorMap& w3s, const SwapParams& p, int pairs,
                                  cudaStream_t s) {
  const size_t bytes = (size_t)kUStages * kUStageBytes +
                       ((sizeof(UpState) + 127) & ~size_t(127)) +
                       kUEpiWarps * 32 * 32 * sizeof(__nv_bfloat16) + 1024;
  auto kern = tc_swap_up_pair_kernel;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, 2 * pairs, kUThreads, bytes, s, m.t, m.ts, m.w, w3, m.ws, w3s, p);
}

}  // namespace

bool swap_up_supported(const FfnArgs& f) {
  return f.act == MOE_ACT_SWIGLU && f.X_perm != nullptr && f.save_u == nullptr &&
         f.counts != nullptr && f.E <= MOE_MAX_EXPERTS && f.h % 256 == 0 && f.d % kSBK == 0;
}

// H = silu(X_perm W1^T) * (X_perm W3^T) per expert over each expert's real
// tokens (and per shared expert over the n rows of X), weights as the M side;
// padding rows of H are not written
moe_status run_ffn_up_swap(const FfnArgs& f, cudaStream_t s) {
  SwapMaps m;
  if (!token_maps(m.t, f.X_perm, f.rows, f.d)) return MOE_ERR_UNSUPPORTED;
  CUtensorMap w3, w3s;
  if (!make_bf16_sw128_map(&m.w, f.W1, (long long)f.E * f.h, f.d, 128)) return MOE_ERR_UNSUPPORTED;
  if (!make_bf16_sw128_map(&w3, f.W3, (long long)f.E * f.h, f.d, 128)) return MOE_ERR_UNSUPPORTED;
  if (f.n_shared > 0) {
    // shared experts read the tokens of X itself
    if (!token_maps(m.ts, f.X, f.n, f.d)) return MOE_ERR_UNSUPPORTED;
    if (!make_bf16_sw128_map(&m.ws, f.sW1, (long long)f.n_shared * f.h, f.d, 128) ||
        !make_bf16_sw128_map(&w3s, f.sW3, (long long)f.n_shared * f.h, f.d, 128))
      return MOE_ERR_UNSUPPORTED;
  } else {
    m.ts = m.t;
    m.ws = m.w;
    w3s = w3;
  }
  SwapParams q{};
  q.offsets = f.offsets;
  q.counts = f.counts;
  q.E = f.E;
  q.K = f.d;
  q.m_per_expert = f.h;
  q.mt_tiles = f.h / 256;
  q.n_shared = f.n_shared;
  q.n = f.n;
  q.shared_in_row = 0;
  q.shared_in_stride = 0;
  q.shared_out_row = f.shared_base;
  q.n_pad = f.n_pad;
  q.n_out = f.h;
  q.out = static_cast<__nv_bfloat16*>(f.H);
  q.err = f.err;
  if (launch_swap_up(m, w3, w3s, q, swap_pairs(q, f.rows_routed), s) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

bool swap_down_supported(const FfnArgs& f) {
  return f.counts != nullptr && f.E <= MOE_MAX_EXPERTS && f.d % 256 == 0 && f.h % kSBK == 0;
}

// Y^T = W2 H^T per expert (and per shared expert), over each expert's real
// tokens only; padding rows of Y are not written
moe_status run_ffn_down_swap(const FfnArgs& f, cudaStream_t s) {
  SwapMaps m;
  if (!token_maps(m.t, f.H, f.rows, f.h)) return MOE_ERR_UNSUPPORTED;
  m.ts = m.t;  // shared rows are rows of H too
  if (!make_bf16_sw128_map(&m.w, f.W2, (long long)f.E * f.d, f.h, 128)) return MOE_ERR_UNSUPPORTED;
  if (f.n_shared > 0) {
    if (!make_bf16_sw128_map(&m.ws, f.sW2, (long long)f.n_shared * f.d, f.h, 128))
      return MOE_ERR_UNSUPPORTED;
  } else {
    m.ws = m.w;
  }
  SwapParams q{};
  q.offsets = f.offsets;
  q.counts = f.counts;
  q.E = f.E;
  q.K = f.h;
  q.m_per_expert = f.d;
  q.mt_tiles = f.d / 256;
  q.n_shared = f.n_shared;
  q.n = f.n;
  q.shared_in_row = f.shared_base;
  q.shared_in_stride = f.n_pad;
  q.shared_out_row = f.shared_base;
  q.n_pad = f.n_pad;
  q.n_out = f.d;
  q.out = static_cast<__nv_bfloat16*>(f.Y);
  q.err = f.err;
  q.k_split = q.K;
  q.w_k_rows = 0;
  if (launch_swap<false>(m, m.w, m.ws, q, swap_pairs(q, f.rows_routed), s) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

bool swap_dx_supported(const SwapDxArgs& a) {
  return a.counts != nullptr && a.E <= MOE_MAX_EXPERTS && a.d % 256 == 0 && a.h % kSBK == 0 &&
         a.kcols % kSBK == 0;
}

// dX_perm^T = W1^T dU^T (+ W3^T dV^T) per expert (and per shared expert), over
// each expert's real tokens only; padding rows of dX_perm are not written
moe_status run_bwd_dx_swap(const SwapDxArgs& a, cudaStream_t s) {
  SwapMaps m;
  if (!token_maps(m.t, a.duv, a.rows, a.kcols)) return MOE_ERR_UNSUPPORTED;
  m.ts = m.t;  // shared rows are rows of dU (dV) too
  CUtensorMap w3, w3s;
  // MN-major weights: [experts * h, d] with 64 x 64 boxes
  if (!make_bf16_sw128_map(&m.w, a.W1, (long long)a.E * a.h, a.d, 64)) return MOE_ERR_UNSUPPORTED;
  w3 = m.w;
  if (a.W3 && !make_bf16_sw128_map(&w3, a.W3, (long long)a.E * a.h, a.d, 64))
    return MOE_ERR_UNSUPPORTED;
  m.ws = m.w;
  w3s = w3;
  if (a.n_shared > 0) {
    if (!make_bf16_sw128_map(&m.ws, a.sW1, (long long)a.n_shared * a.h, a.d, 64))
      return MOE_ERR_UNSUPPORTED;
    w3s = m.ws;
    if (a.sW3 && !make_bf16_sw128_map(&w3s, a.sW3, (long long)a.n_shared * a.h, a.d, 64))
      return MOE_ERR_UNSUPPORTED;
  }
  SwapParams q{};
  q.offsets = a.offsets;
  q.counts = a.counts;
  q.E = a.E;
  q.K = a.kcols;
  q.m_per_expert = a.d;
  q.mt_tiles = a.d / 256;
  q.n_shared = a.n_shared;
  q.n = a.n;
  q.shared_in_row = a.shared_base;
  q.shared_in_stride = a.n_pad;
  q.shared_out_row = a.shared_base;
  q.n_pad = a.n_pad;
  q.n_out = a.d;
  q.out = static_cast<__nv_bfloat16*>(a.dxp);
  q.err = a.err;
  q.k_split = a.W3 ? a.h : a.kcols;
  q.w_k_rows = a.h;
  if (launch_swap<true>(m, w3, w3s, q, swap_pairs(q, a.rows_routed), s) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // namespace moe
