// Down projection of the grouped expert FFN for fine-grained experts, with
// the weights as the M side.
//
// "Expert choice routing" (aicassindra.com), "The math: a gating matrix and
// top-k over tokens": each expert's gathered rows form a dense batch; here the
// product Y_e = H_e W2_e^T is taken transposed, Y_e^T = W2_e H_e^T, so that an
// expert's tokens are the N side of the MMA and need only 16-row granularity,
// where the 128-row M tiles of the other kernels round an expert of ~256 rows
// up to 384 or 512.
//
// CTA pairs (cta_group::2). A tile is (expert, 256 rows of W2, up to 256 of
// the expert's tokens): each CTA loads its 128 weight rows as A and half of
// the tile's tokens as B, and the leader issues M=256 MMAs with N = tokens (a
// multiple of 16) into one of two 256-column TMEM accumulators, so one tile's
// epilogue overlaps the next tile's main loop.
//   warp 0     TMA producer (6-stage ring: A 16 KB + B up to 16 KB);
//   warp 1     TMEM allocation; the leader's lane 0 issues the MMAs;
//   warps 2-9  epilogue, two per TMEM lane quadrant on alternate 32-token
//              groups: tcgen05.ld 32 tokens at a time, a transpose through
//              shared memory, and 16-byte stores of each token's 32
//              consecutive output columns.
// Every mbarrier wait is bounded, as in the other GEMM kernels.
//
// Only the down projection runs here. The same scheme for the SwiGLU up
// projection (64 W1 and 64 W3 rows per CTA, gate and up values meeting
// through shared memory) was slower on B200 than the token-side CTA pairs.
#include <cuda.h>
#include <math.h>

#include "device_common.cuh"
#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {

namespace {

// warps: 0 producer, 1 MMA, 2-9 epilogue (two per TMEM lane quadrant)
constexpr int kSBK = 64, kSStages = 6, kSEpiWarps = 8, kSThreads = 32 * (2 + kSEpiWarps);
constexpr int kSABytes = 128 * kSBK * 2;         // this CTA's 128 weight rows
constexpr int kSBBytes = 128 * kSBK * 2;         // up to 128 token rows
constexpr int kSStageBytes = kSABytes + kSBBytes;
constexpr int kSTmemCols = 512;                  // two 256-column accumulators
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
};

struct SwapState {
  uint64_t full[kSStages];
  uint64_t empty[kSStages];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  volatile int abort_flag;
  int offs[MOE_MAX_EXPERTS + 1];
  int cnt[MOE_MAX_EXPERTS];
  int tprefix[MOE_MAX_EXPERTS + 1];  // tiles of the experts before e
};

template <bool CLUSTER_ACQUIRE>
__device__ __forceinline__ bool swap_wait(uint64_t* bar, uint32_t parity, SwapState* st, int* err,
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
__device__ __forceinline__ SwapTile decode_swap(int tile, const SwapParams& p, const SwapState* st,
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

// token rows one CTA loads for an N-column slot: N/2, as a TMA box of 32, 64 or 128
__device__ __forceinline__ int box_rows(int n) {
  const int half = n / 2;
  return half <= 32 ? 32 : half <= 64 ? 64 : 128;
}

// token maps: tmT[b] / tmTs[b] = routed / shared token rows of H with a box
// of 32 << b rows; weights: tmW (routed) / tmWs (shared), boxes of 128 rows
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kSThreads, 1)
    tc_swap_pair_kernel(const __grid_constant__ CUtensorMap tmT0,
                        const __grid_constant__ CUtensorMap tmT1,
                        const __grid_constant__ CUtensorMap tmT2,
                        const __grid_constant__ CUtensorMap tmTs0,
                        const __grid_constant__ CUtensorMap tmTs1,
                        const __grid_constant__ CUtensorMap tmTs2,
                        const __grid_constant__ CUtensorMap tmW,
                        const __grid_constant__ CUtensorMap tmWs, const SwapParams p) {
  extern __shared__ __align__(1024) unsigned char ssm[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(ssm) + 1023) & ~uintptr_t(1023));
  SwapState* st = reinterpret_cast<SwapState*>(base + kSStages * kSStageBytes);
  // epilogue staging, [8 warps][32 tokens][32 columns] bf16
  __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(
      base + kSStages * kSStageBytes + ((sizeof(SwapState) + 127) & ~size_t(127)));
  auto sA = [&](int s) { return base + s * kSStageBytes; };
  auto sB = [&](int s) { return base + s * kSStageBytes + kSABytes; };

  const uint32_t rank = sm100::cluster_ctarank();
  const bool leader = rank == 0;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < kSStages; ++s) {
      sm100::mbar_init(&st->full[s], 1);
      sm100::mbar_init(&st->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      sm100::mbar_init(&st->tfull[a], 1);
      sm100::mbar_init(&st->tempty[a], 2 * 32 * kSEpiWarps);  // both CTAs' epilogues
    }
    sm100::mbar_init(&st->drain, 1);
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

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = pair_id; ok && tile < total; tile += num_pairs) {
        const SwapTile t = decode_swap(tile, p, st, routed);
        const CUtensorMap* tm[3];
        if (t.shared) {
          tm[0] = &tmTs0; tm[1] = &tmTs1; tm[2] = &tmTs2;
        } else {
          tm[0] = &tmT0; tm[1] = &tmT1; tm[2] = &tmT2;
        }
        const int b1 = box_rows(t.n);
        const CUtensorMap* m1 = tm[b1 == 32 ? 0 : b1 == 64 ? 1 : 2];
        const uint32_t bytes = kSABytes + (uint32_t)b1 * kSBK * 2;
        const CUtensorMap* mw = t.shared ? &tmWs : &tmW;
        const int wrow = t.expert * p.m_per_expert + t.m0 + (int)rank * 128;  // this CTA's 128
        // this CTA's half of the tile's tokens
        const long long trow1 = t.tok_row + (long long)rank * (t.n / 2);
        for (int kb = 0; kb < KB; ++kb) {
          if (!swap_wait<false>(&st->empty[stage], phase ^ 1u, st, p.err, kErrGemmTimeout | 0xA1)) {
            ok = false;
            break;
          }
          const uint32_t fl = sm100::mapa_shared(sm100::smem_addr(&st->full[stage]), 0);
          if (leader) sm100::mbar_arrive_expect_tx(&st->full[stage], 2 * bytes);
          sm100::tma_load_2d_pair(sA(stage), mw, fl, kb * kSBK, wrow);
          sm100::tma_load_2d_pair(sB(stage), m1, fl, kb * kSBK, (int)trow1);
          ++issued;
          if (++stage == kSStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok && leader) {
        // wait (bounded) until the copies of the outstanding stages have landed
        int s = stage;
        uint32_t ph = phase;
        const int pending = issued < kSStages ? issued : kSStages;
        for (int i = 0; i < pending; ++i) {
          if (--s < 0) {
            s = kSStages - 1;
            ph ^= 1u;
          }
          const uint64_t t0 = global_timer_ns();
          while (!sm100::mbar_try_wait(&st->full[s], ph) && global_timer_ns() - t0 < kSWaitNs) {
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int tile = pair_id; ok && tile < total; tile += num_pairs, ++local) {
        const SwapTile t = decode_swap(tile, p, st, routed);
        const int acc = local & 1;
        const uint32_t acc_phase = (uint32_t)(local >> 1) & 1u;
        if (!swap_wait<true>(&st->tempty[acc], acc_phase ^ 1u, st, p.err, kErrGemmTimeout | 0xB2)) {
          ok = false;
          break;
        }
        sm100::tc_fence_after();
        const uint32_t idesc = sm100::idesc_bf16_f32(256, t.n);
        const uint32_t d_tmem = tmem + (uint32_t)(acc * 256);
        for (int kb = 0; kb < KB; ++kb) {
          if (!swap_wait<false>(&st->full[stage], phase, st, p.err, kErrGemmTimeout | 0xB3)) {
            ok = false;
            break;
          }
          sm100::tc_fence_after();
          const uint64_t adesc = sm100::sw128_kmajor_desc(sm100::smem_addr(sA(stage)));
          const uint64_t bdesc = sm100::sw128_kmajor_desc(sm100::smem_addr(sB(stage)));
#pragma unroll
          for (int k = 0; k < kSBK / 16; ++k)
            sm100::umma_f16_pair(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, (kb | k) != 0);
          sm100::umma_commit_pair_mc(&st->empty[stage], 0x3);
          if (++stage == kSStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        sm100::umma_commit_pair_mc(&st->tfull[acc], 0x3);
      }
      sm100::umma_commit_pair_mc(&st->drain, 0x1);
      const uint64_t t0 = global_timer_ns();
      while (!sm100::mbar_try_wait(&st->drain, 0) && global_timer_ns() - t0 < kSWaitNs) {
      }
    }
  } else {
    // epilogue: TMEM lanes = this CTA's 128 weight rows (output columns),
    // TMEM columns = tokens; warps q and q + 4 own lanes 32q..32q+31 (q =
    // warp % 4) and take alternate 32-token column groups
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    constexpr int CW = 32;  // output columns per warp
    constexpr int VPR = CW * 2 / 16;  // 16-byte pieces of a token's CW columns
    __nv_bfloat16* stg = stage + (warp - 2) * (32 * CW);  // [32 tokens][CW] bf16
    int local = 0;
    for (int tile = pair_id; tile < total; tile += num_pairs, ++local) {
      const SwapTile t = decode_swap(tile, p, st, routed);
      const int acc = local & 1;
      const uint32_t acc_phase = (uint32_t)(local >> 1) & 1u;
      const int col0 = t.m0 + (int)rank * 128 + 32 * q;
      __nv_bfloat16* outt = p.out + (size_t)t.out_row * p.n_out + col0;
      {
        if (!swap_wait<true>(&st->tfull[acc], acc_phase, st, p.err, kErrGemmTimeout | 0xC4))
          break;
        sm100::tc_fence_after();
        const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * 256);
#pragma unroll 1
        for (int cc = 32 * half; cc < t.n; cc += 64) {
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
        sm100::mbar_arrive_cluster(sm100::mapa_shared(sm100::smem_addr(&st->tempty[acc]), 0));
      }
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
  CUtensorMap t[3], ts[3], w, ws;
};

static cudaError_t launch_swap(const SwapMaps& m, const SwapParams& p, int pairs, cudaStream_t s) {
  const size_t bytes = (size_t)kSStages * kSStageBytes + ((sizeof(SwapState) + 127) & ~size_t(127)) +
                       kSEpiWarps * 32 * 32 * sizeof(__nv_bfloat16) + 1024;
  auto kern = tc_swap_pair_kernel;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, 2 * pairs, kSThreads, bytes, s, m.t[0], m.t[1], m.t[2], m.ts[0],
                    m.ts[1], m.ts[2], m.w, m.ws, p);
}

static bool token_maps(CUtensorMap (&t)[3], const void* ptr, long long rows, long long cols) {
  for (int b = 0; b < 3; ++b)
    if (!make_bf16_sw128_map(&t[b], ptr, rows, cols, 32 << b)) return false;
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

}  // namespace

bool swap_down_supported(const FfnArgs& f) {
  return f.counts != nullptr && f.E <= MOE_MAX_EXPERTS && f.d % 256 == 0 && f.h % kSBK == 0;
}

// Y^T = W2 H^T per expert (and per shared expert), over each expert's real
// tokens only; padding rows of Y are not written
moe_status run_ffn_down_swap(const FfnArgs& f, cudaStream_t s) {
  SwapMaps m;
  if (!token_maps(m.t, f.H, f.rows, f.h)) return MOE_ERR_UNSUPPORTED;
  for (int b = 0; b < 3; ++b) m.ts[b] = m.t[b];  // shared rows are rows of H too
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
  if (launch_swap(m, q, swap_pairs(q, f.rows_routed), s) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // namespace moe
