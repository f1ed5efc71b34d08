// Grouped expert FFN on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// "Expert choice routing" (aicassindra.com), "The math: a gating matrix and
// top-k over tokens": the gathered per-expert batches are dense matrices
// "ideal for batched matmuls"; each expert's FFN is one up projection (with
// the activation, or SwiGLU's two projections fused) and one down projection.
//
// One persistent CTA per SM, warp-specialised:
//   warp 0      TMA producer: A tile 128x64 and B tile 256x64 (bf16, 128-byte
//               swizzle) per stage into a 4-deep shared-memory ring;
//   warp 1      allocates 512 TMEM columns and issues tcgen05.mma
//               (M=128, N=256, K=16) from one thread; commits free the smem
//               stage and, per tile, hand the accumulator to the epilogue;
//   warps 2..5  epilogue: tcgen05.ld 32 columns at a time, activation, bf16,
//               16-byte stores of each thread's row.
// Two TMEM accumulators (2 x 256 columns) let the epilogue of one tile
// overlap the main loop of the next. Tiles are (128-row block of one
// expert's segment, 256-column block); rows of a block never straddle two
// experts because segments start on 128-row boundaries. The B tile of a
// SwiGLU up projection holds 128 rows of W1 followed by the same 128 rows of
// W3, so one N=256 MMA produces both halves of the gate.
// Every mbarrier wait is bounded; on a timeout the CTA records an error,
// stops issuing, waits (bounded) for its own copies and MMAs, frees TMEM and
// returns.
#include <cuda.h>
#include <math.h>

#include <atomic>
#include <mutex>

#include "device_common.cuh"
#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {

constexpr int kBM = 128, kBN = 256, kBK = 64, kStages = 4;
constexpr int kABytes = kBM * kBK * 2;       // 16 KB
constexpr int kBBytes = kBN * kBK * 2;       // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kTmemCols = 512;
constexpr int kGemmThreads = 192;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

enum { ACT_NONE = 0, ACT_RELU = 1, ACT_GELU = 2, ACT_SWIGLU = 3 };
// what a projection fuses: nothing; the dispatch gather into its A loads (up
// projection); the gate-scaled scatter-add of the combine into its epilogue
// (down projection); or, for training, the up projection also stores its
// pre-activations U (and V) beside H for the backward pass
enum { FUSE_NONE = 0, FUSE_GATHER = 1, FUSE_SCATTER = 2, FUSE_SAVE = 3 };

struct TcGemmParams {
  const int32_t* offsets;
  int E;
  int K;                    // reduction length (multiple of 64)
  int n_out;                // output columns
  int nt_tiles;             // column blocks
  int b_rows_per_expert;    // rows of B per expert
  int shared_tiles_per;     // 128-row blocks per shared expert
  int n_shared;
  int max_routed_tiles;     // host bound on offsets[E] / 128
  long long a1_row_base;    // shared experts' A rows: base + s*stride + block*128
  long long a1_row_stride;
  long long out_shared_base;
  long long n_pad;
  __nv_bfloat16* out;       // [rows, n_out]
  int* err;
  const int32_t* row_token;  // source token of each dispatched row (gathered A, scatter)
  const float* row_gate;     // scatter: gate of each dispatched row
  float* out32;              // scatter: [n_tok, n_out] fp32 sums
  int n_tok;                 // tokens (rows of X and out32)
  __nv_bfloat16* save_u;     // save: [rows, n_out] pre-activations U = X W1^T
  __nv_bfloat16* save_v;     // save (SwiGLU): [rows, n_out] V = X W3^T
  int inject_no_loads;       // failure-path test: the producer issues no loads
};

struct SharedState {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  volatile int abort_flag;
  int offs[MOE_MAX_EXPERTS + 1];
  int tprefix[MOE_MAX_EXPERTS + 1];  // tiles of the experts before e
};

__device__ __forceinline__ bool bounded_wait(uint64_t* bar, uint32_t parity, SharedState* st,
                                             int* err, int code) {
  if (sm100::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (sm100::mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (st->abort_flag) return false;
      if (global_timer_ns() - t0 > kWaitLimitNs) {
        st->abort_flag = 1;
        report_error(err, code);
        return false;
      }
    }
  }
}

struct TileCoord {
  int a_sel, a_row, b_sel, b_row;
  long long out_row;
  int col0;
};

// Tile schedule: expert by expert; inside an expert column block by column
// block, and the expert's 128-row blocks innermost, so CTAs that run at the
// same time share one weight tile (read from HBM once) instead of each
// streaming a different one. Shared experts follow the routed ones.
template <int ACT>
__device__ __forceinline__ TileCoord decode_tile(int tile, const TcGemmParams& p,
                                                 const int* offs, const int* tprefix,
                                                 int routed_tiles) {
  constexpr int BNO = ACT == ACT_SWIGLU ? kBN / 2 : kBN;
  TileCoord c;
  int nt;
  if (tile < routed_tiles) {
    int lo = 0, hi = p.E - 1;  // largest e with tprefix[e] <= tile
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (tprefix[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    const int local = tile - tprefix[lo];
    const int blocks = max((offs[lo + 1] - offs[lo]) / kBM, 1);
    nt = local / blocks;
    const int row = offs[lo] + (local % blocks) * kBM;
    c.a_sel = 0;
    c.a_row = row;
    c.b_sel = 0;
    c.b_row = lo * p.b_rows_per_expert;
    c.out_row = row;
  } else {
    const int per = p.shared_tiles_per * p.nt_tiles;
    const int q = tile - routed_tiles;
    const int s = q / per, local = q % per;
    nt = local / p.shared_tiles_per;
    const int lm = local % p.shared_tiles_per;
    c.a_sel = 1;
    c.a_row = (int)(p.a1_row_base + s * p.a1_row_stride + (long long)lm * kBM);
    c.b_sel = 1;
    c.b_row = s * p.b_rows_per_expert;
    c.out_row = p.out_shared_base + s * p.n_pad + (long long)lm * kBM;
  }
  c.col0 = nt * BNO;
  c.b_row += c.col0;
  return c;
}

// 32 fp32 accumulator values (as bits) rounded to bf16 into 64 bytes
__device__ __forceinline__ void store_row32(__nv_bfloat16* dst, const uint32_t* v) {
  uint4* o = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int j = 0; j < 4; ++j)
    o[j] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * j]), __uint_as_float(v[8 * j + 1])),
                      pack_bf16x2(__uint_as_float(v[8 * j + 2]), __uint_as_float(v[8 * j + 3])),
                      pack_bf16x2(__uint_as_float(v[8 * j + 4]), __uint_as_float(v[8 * j + 5])),
                      pack_bf16x2(__uint_as_float(v[8 * j + 6]), __uint_as_float(v[8 * j + 7])));
}

// fp32 vector reduction into global memory (sm_90+), 16-byte aligned
__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}

template <int ACT>
__device__ __forceinline__ float act_fn(float v) {
  if (ACT == ACT_RELU) return fmaxf(v, 0.0f);
  if (ACT == ACT_GELU) return 0.5f * v * (1.0f + erff(v * 0.70710678118654752f));
  return v;
}

template <int ACT, int FUSE>
__global__ void __launch_bounds__(kGemmThreads, 1)
    tc_grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA0,
                           const __grid_constant__ CUtensorMap tmA1,
                           const __grid_constant__ CUtensorMap tmB0,
                           const __grid_constant__ CUtensorMap tmB0g,
                           const __grid_constant__ CUtensorMap tmB1,
                           const __grid_constant__ CUtensorMap tmB1g,
                           const __grid_constant__ CUtensorMap tmXg, const TcGemmParams p) {
  constexpr bool SWIGLU = ACT == ACT_SWIGLU;
  extern __shared__ __align__(1024) unsigned char gsm[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(gsm) + 1023) & ~uintptr_t(1023));
  unsigned char* sA = base;                            // [kStages][16 KB]
  unsigned char* sB = base + kStages * kABytes;        // [kStages][32 KB]
  SharedState* st = reinterpret_cast<SharedState*>(base + kStages * kStageBytes);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      sm100::mbar_init(&st->full[s], 1);
      sm100::mbar_init(&st->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      sm100::mbar_init(&st->tfull[a], 1);
      sm100::mbar_init(&st->tempty[a], 128);
    }
    sm100::mbar_init(&st->drain, 1);
    st->abort_flag = 0;
    sm100::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    sm100::tma_prefetch_desc(&tmA0);
    sm100::tma_prefetch_desc(&tmB0);
    if (SWIGLU) sm100::tma_prefetch_desc(&tmB0g);
  }
  if (warp == 1) {
    sm100::tmem_alloc(&st->tmem_base, kTmemCols);
    sm100::tmem_relinquish();
  }
  // the set-up above needs nothing from the previous kernel; from here on
  // the routing offsets (and, for the second projection, H) are read
  pdl_wait();
  for (int i = tid; i <= p.E; i += kGemmThreads) st->offs[i] = p.offsets[i];
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int e = 0; e < p.E; ++e) {
      st->tprefix[e] = run;
      const int seg = st->offs[e + 1] - st->offs[e];
      if (seg < 0 || (st->offs[e] % kBM) != 0) bad_index(p.err, kSiteGemmOffsets);
      run += max(seg, 0) / kBM * p.nt_tiles;
    }
    st->tprefix[p.E] = run;
    if (st->offs[p.E] > p.max_routed_tiles * kBM) bad_index(p.err, kSiteGemmOffsets);
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = st->tmem_base;

  const int routed = min(st->tprefix[p.E], p.max_routed_tiles * p.nt_tiles);
  const int total = routed + p.n_shared * p.shared_tiles_per * p.nt_tiles;
  const int KB = p.K / kBK;

  if (warp == 0) {
    // the whole warp walks the schedule; lane 0 waits and issues the 2-D
    // loads, and with FUSE_GATHER every lane issues one 4-row gather of A
    int stage = 0;
    uint32_t phase = 0;
    int issued = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
      const TileCoord c = decode_tile<ACT>(tile, p, st->offs, st->tprefix, routed);
      const CUtensorMap* ma = c.a_sel ? &tmA1 : &tmA0;
      const CUtensorMap* mb = c.b_sel ? &tmB1 : &tmB0;
      const CUtensorMap* mbg = c.b_sel ? &tmB1g : &tmB0g;
      // routed rows straight from X: lane l brings rows 4l..4l+3 of the block;
      // padding rows read token 0 and their outputs are never used
      const bool gather = FUSE == FUSE_GATHER && c.a_sel == 0;
      int tok[4] = {0, 0, 0, 0};
      if (gather) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int t = p.row_token[c.a_row + 4 * lane + j];
          if (t < -1 || t >= p.n_tok) bad_index(p.err, kSiteGemmGatherToken);
          tok[j] = (t >= 0 && t < p.n_tok) ? t : 0;
        }
      }
      for (int kb = 0; kb < KB; ++kb) {
        int okw = 1;
        if (lane == 0)
          okw = bounded_wait(&st->empty[stage], phase ^ 1u, st, p.err, kErrGemmTimeout | 0x01);
        if (!__shfl_sync(0xffffffffu, okw, 0)) {
          ok = false;
          break;
        }
        unsigned char* a_dst = sA + stage * kABytes;
        unsigned char* b_dst = sB + stage * kBBytes;
        // (a failure-path test withholds every load: the MMA warp's bounded
        // wait on this stage then runs out)
        if (!p.inject_no_loads) {
          if (lane == 0) {
            sm100::mbar_arrive_expect_tx(&st->full[stage], kStageBytes);
            if (!gather) sm100::tma_load_2d(a_dst, ma, &st->full[stage], kb * kBK, c.a_row);
            if (SWIGLU) {
              sm100::tma_load_2d(b_dst, mb, &st->full[stage], kb * kBK, c.b_row);
              sm100::tma_load_2d(b_dst + kBBytes / 2, mbg, &st->full[stage], kb * kBK, c.b_row);
            } else {
              sm100::tma_load_2d(b_dst, mb, &st->full[stage], kb * kBK, c.b_row);
            }
          }
          if (gather)
            sm100::tma_gather4(a_dst + lane * 4 * (kBK * 2), &tmXg, &st->full[stage], kb * kBK,
                               tok[0], tok[1], tok[2], tok[3]);
          ++issued;
        }
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (lane == 0) {
      if (!ok) {
        // wait (bounded) for the copies still in flight into our stages
        int s = stage;
        uint32_t ph = phase;
        const int pending = issued < kStages ? issued : kStages;
        for (int i = 0; i < pending; ++i) {
          if (--s < 0) {
            s = kStages - 1;
            ph ^= 1u;
          }
          const uint64_t t0 = global_timer_ns();
          while (!sm100::mbar_try_wait(&st->full[s], ph) &&
                 global_timer_ns() - t0 < kWaitLimitNs) {
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = sm100::idesc_bf16_f32(kBM, kBN);
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x, ++local) {
        const int acc = local & 1;
        const uint32_t acc_phase = (uint32_t)(local >> 1) & 1u;
        if (!bounded_wait(&st->tempty[acc], acc_phase ^ 1u, st, p.err, kErrGemmTimeout | 0x12)) {
          ok = false;
          break;
        }
        sm100::tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(acc * kBN);
        for (int kb = 0; kb < KB; ++kb) {
          if (!bounded_wait(&st->full[stage], phase, st, p.err, kErrGemmTimeout | 0x13)) {
            ok = false;
            break;
          }
          sm100::tc_fence_after();
          const uint64_t adesc = sm100::sw128_kmajor_desc(sm100::smem_addr(sA + stage * kABytes));
          const uint64_t bdesc = sm100::sw128_kmajor_desc(sm100::smem_addr(sB + stage * kBBytes));
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            // +32 bytes along K inside the swizzled 128-byte row = +2 in the
            // address field
            sm100::umma_f16(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, (kb | k) != 0);
          }
          sm100::umma_commit(&st->empty[stage]);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        sm100::umma_commit(&st->tfull[acc]);
      }
      // wait (bounded) until every MMA this thread issued has completed
      sm100::umma_commit(&st->drain);
      const uint64_t t0 = global_timer_ns();
      while (!sm100::mbar_try_wait(&st->drain, 0) && global_timer_ns() - t0 < kWaitLimitNs) {
      }
    }
  } else {
    // epilogue warps 2..5: TMEM lane quadrant = warp % 4
    const int q = warp & 3;
    const int row_in_tile = q * 32 + lane;
    constexpr int BNO = SWIGLU ? kBN / 2 : kBN;
    int local = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++local) {
      const int acc = local & 1;
      const uint32_t acc_phase = (uint32_t)(local >> 1) & 1u;
      if (!bounded_wait(&st->tfull[acc], acc_phase, st, p.err, kErrGemmTimeout | 0x24)) break;
      sm100::tc_fence_after();
      const TileCoord c = decode_tile<ACT>(tile, p, st->offs, st->tprefix, routed);
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * kBN);
      __nv_bfloat16* orow = p.out + (size_t)(c.out_row + row_in_tile) * p.n_out;
      // scatter: the row's token and gate (shared experts: weight 1, the
      // token is the row within the expert's block of n_pad rows)
      int tok = -1;
      float gate = 0.0f;
      if (FUSE == FUSE_SCATTER) {
        const long long r = c.out_row + row_in_tile;
        if (c.a_sel == 0) {
          tok = p.row_token[r];
          if (tok < -1 || tok >= p.n_tok) {
            bad_index(p.err, kSiteGemmScatterToken);
            tok = -1;
          }
          gate = tok >= 0 ? p.row_gate[r] : 0.0f;
        } else {
          const long long q2 = (r - p.out_shared_base) % p.n_pad;
          tok = q2 < p.n_tok ? (int)q2 : -1;
          gate = 1.0f;
        }
      }
#pragma unroll 1
      for (int cc = 0; cc < BNO; cc += 32) {
        if (c.col0 + cc >= p.n_out) break;
        uint32_t v[32];
        sm100::tmem_ld_32x32b_x32(tbase + cc, v);
        float f[32];
        if (SWIGLU) {
          uint32_t g[32];
          sm100::tmem_ld_32x32b_x32(tbase + BNO + cc, g);
          sm100::tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float a = __uint_as_float(v[i]);
            const float b = __uint_as_float(g[i]);
            f[i] = a * __frcp_rn(1.0f + __expf(-a)) * b;
          }
          if (FUSE == FUSE_SAVE) store_row32(p.save_v + (orow - p.out) + c.col0 + cc, g);
        } else {
          sm100::tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) f[i] = act_fn<ACT>(__uint_as_float(v[i]));
        }
        if (FUSE == FUSE_SAVE) store_row32(p.save_u + (orow - p.out) + c.col0 + cc, v);
        if (FUSE == FUSE_SCATTER) {
          if (tok >= 0) {
            float* dst = p.out32 + (size_t)tok * p.n_out + c.col0 + cc;
#pragma unroll
            for (int j = 0; j < 8; ++j)
              red_add_v4(dst + 4 * j, gate * f[4 * j], gate * f[4 * j + 1], gate * f[4 * j + 2],
                         gate * f[4 * j + 3]);
          }
        } else {
          uint4* dst = reinterpret_cast<uint4*>(orow + c.col0 + cc);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint4 o;
            o.x = pack_bf16x2(f[8 * j + 0], f[8 * j + 1]);
            o.y = pack_bf16x2(f[8 * j + 2], f[8 * j + 3]);
            o.z = pack_bf16x2(f[8 * j + 4], f[8 * j + 5]);
            o.w = pack_bf16x2(f[8 * j + 6], f[8 * j + 7]);
            dst[j] = o;
          }
        }
      }
      sm100::tc_fence_before();
      sm100::mbar_arrive(&st->tempty[acc]);
    }
  }
  sm100::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// CTA-pair variant (cta_group::2). A cluster of two CTAs on one TPC computes a
// 256 x 256 tile: each CTA loads 128 rows of A and one half (128 rows) of the
// 256-row B tile into its own shared memory, the pair leader issues
// tcgen05.mma.cta_group::2 (M=256, N=256, K=16), and each CTA's TMEM receives
// its own 128 rows. Per CTA that is 32 KB of operands per 64-deep k-block
// instead of 48 KB, and the ring holds six stages instead of four. Both CTAs'
// TMA loads complete on the leader's stage barrier; MMA commits arrive on
// both CTAs' barriers (multicast commit); both epilogues release the
// accumulator on the leader's barrier. A pair tile takes two consecutive
// 128-row blocks of one expert's segment; when the expert has an odd number
// of blocks the second CTA recomputes the first block and stores nothing.
// For SwiGLU the leader's B half is 128 rows of W1 and the peer's the same
// rows of W3, so TMEM columns 0..127 / 128..255 hold the two projections.
// ---------------------------------------------------------------------------
constexpr int kPStages = 6;
constexpr int kPABytes = kBM * kBK * 2;           // 16 KB: this CTA's 128 rows of A
constexpr int kPBBytes = (kBN / 2) * kBK * 2;     // 16 KB: this CTA's half of B
constexpr int kPStageBytes = kPABytes + kPBBytes; // 32 KB

struct PairState {
  uint64_t full[kPStages];   // leader: both CTAs' bytes of a stage have landed
  uint64_t empty[kPStages];  // each CTA: its copy of a stage may be refilled
  uint64_t tfull[2];         // each CTA: accumulator ready to read
  uint64_t tempty[2];        // leader: both epilogues are done with an accumulator
  uint64_t drain;
  uint32_t tmem_base;
  volatile int abort_flag;
  int offs[MOE_MAX_EXPERTS + 1];
  int tprefix[MOE_MAX_EXPERTS + 1];  // pair tiles of the experts before e
};

template <bool CLUSTER_ACQUIRE>
__device__ __forceinline__ bool bounded_wait_pair(uint64_t* bar, uint32_t parity, PairState* st,
                                                  int* err, int code) {
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
      if (global_timer_ns() - t0 > kWaitLimitNs) {
        st->abort_flag = 1;
        report_error(err, code);
        return false;
      }
    }
  }
}

struct PairCoord {
  int a_sel, a_row, b_sel, b_row;
  long long out_row;
  int col0;
  bool valid;
};

// Same schedule as decode_tile, over pairs of 128-row blocks.
template <int ACT>
__device__ __forceinline__ PairCoord decode_pair(int tile, const TcGemmParams& p,
                                                 const int* offs, const int* tprefix,
                                                 int routed_tiles, uint32_t rank) {
  constexpr int BNO = ACT == ACT_SWIGLU ? kBN / 2 : kBN;
  PairCoord c;
  int b_base, nt;
  if (tile < routed_tiles) {
    int lo = 0, hi = p.E - 1;  // largest e with tprefix[e] <= tile
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (tprefix[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    const int cnt = (offs[lo + 1] - offs[lo]) / kBM;
    const int pairs = max((cnt + 1) / 2, 1);
    const int local = tile - tprefix[lo];
    nt = local / pairs;
    const int j = local % pairs;
    int mloc = 2 * j + (int)rank;
    c.valid = mloc < cnt;
    if (!c.valid) mloc = 2 * j;
    const int row = offs[lo] + mloc * kBM;
    c.a_sel = 0;
    c.a_row = row;
    c.out_row = row;
    c.b_sel = 0;
    b_base = lo * p.b_rows_per_expert;
  } else {
    const int spp = (p.shared_tiles_per + 1) / 2;
    const int per = spp * p.nt_tiles;
    const int q = tile - routed_tiles;
    const int s = q / per, local = q % per;
    nt = local / spp;
    const int jj = local % spp;
    int lm = 2 * jj + (int)rank;
    c.valid = lm < p.shared_tiles_per;
    if (!c.valid) lm = 2 * jj;
    c.a_sel = 1;
    c.a_row = (int)(p.a1_row_base + s * p.a1_row_stride + (long long)lm * kBM);
    c.out_row = p.out_shared_base + s * p.n_pad + (long long)lm * kBM;
    c.b_sel = 1;
    b_base = s * p.b_rows_per_expert;
  }
  c.col0 = nt * BNO;
  c.b_row = b_base + c.col0 + (ACT == ACT_SWIGLU ? 0 : (int)rank * (kBN / 2));
  return c;
}

template <int ACT, int FUSE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    tc_grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA0,
                                const __grid_constant__ CUtensorMap tmA1,
                                const __grid_constant__ CUtensorMap tmB0,
                                const __grid_constant__ CUtensorMap tmB0g,
                                const __grid_constant__ CUtensorMap tmB1,
                                const __grid_constant__ CUtensorMap tmB1g,
                                const __grid_constant__ CUtensorMap tmXg,
                                const TcGemmParams p) {
  constexpr bool SWIGLU = ACT == ACT_SWIGLU;
  extern __shared__ __align__(1024) unsigned char gsm[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(gsm) + 1023) & ~uintptr_t(1023));
  PairState* st = reinterpret_cast<PairState*>(base + kPStages * kPStageBytes);
  auto sA = [&](int s) { return base + s * kPStageBytes; };
  auto sB = [&](int s) { return base + s * kPStageBytes + kPABytes; };

  const uint32_t rank = sm100::cluster_ctarank();
  const bool leader = rank == 0;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < kPStages; ++s) {
      sm100::mbar_init(&st->full[s], 1);
      sm100::mbar_init(&st->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      sm100::mbar_init(&st->tfull[a], 1);
      sm100::mbar_init(&st->tempty[a], 256);
    }
    sm100::mbar_init(&st->drain, 1);
    st->abort_flag = 0;
    sm100::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    sm100::tma_prefetch_desc(&tmA0);
    sm100::tma_prefetch_desc(&tmB0);
    if (SWIGLU) sm100::tma_prefetch_desc(&tmB0g);
  }
  if (warp == 1) {
    sm100::tmem_alloc_pair(&st->tmem_base, kTmemCols);
    sm100::tmem_relinquish_pair();
  }
  // the set-up above needs nothing from the previous kernel; from here on
  // the routing offsets (and, for the second projection, H) are read
  pdl_wait();
  for (int i = tid; i <= p.E; i += kGemmThreads) st->offs[i] = p.offsets[i];
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int e = 0; e < p.E; ++e) {
      st->tprefix[e] = run;
      const int seg = st->offs[e + 1] - st->offs[e];
      if (seg < 0 || (st->offs[e] % kBM) != 0) bad_index(p.err, kSiteGemmPairOffsets);
      const int cnt = max(seg, 0) / kBM;
      run += (cnt + 1) / 2 * p.nt_tiles;
    }
    st->tprefix[p.E] = run;
    if (st->offs[p.E] > p.max_routed_tiles * kBM) bad_index(p.err, kSiteGemmPairOffsets);
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::cluster_sync();  // both CTAs' barriers exist before any remote arrive
  sm100::tc_fence_after();
  const uint32_t tmem = st->tmem_base;

  const int routed = min(st->tprefix[p.E], p.max_routed_tiles * p.nt_tiles);
  const int spp = (p.shared_tiles_per + 1) / 2;
  const int total = routed + p.n_shared * spp * p.nt_tiles;
  const int KB = p.K / kBK;
  const int pair_id = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;

  if (warp == 0) {
    // the whole warp walks the schedule; lane 0 waits and issues the 2-D
    // loads, and with FUSE_GATHER every lane issues one 4-row gather of A
    int stage = 0;
    uint32_t phase = 0;
    int issued = 0;
    bool ok = true;
    for (int tile = pair_id; ok && tile < total; tile += num_pairs) {
      const PairCoord c = decode_pair<ACT>(tile, p, st->offs, st->tprefix, routed, rank);
      const CUtensorMap* ma = c.a_sel ? &tmA1 : &tmA0;
      const CUtensorMap* mb;
      if (SWIGLU)
        mb = leader ? (c.b_sel ? &tmB1 : &tmB0) : (c.b_sel ? &tmB1g : &tmB0g);
      else
        mb = c.b_sel ? &tmB1 : &tmB0;
      // routed rows straight from X: lane l brings rows 4l..4l+3 of the block;
      // padding rows read token 0 and their outputs are never used
      const bool gather = FUSE == FUSE_GATHER && c.a_sel == 0;
      int tok[4] = {0, 0, 0, 0};
      if (gather) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int t = p.row_token[c.a_row + 4 * lane + j];
          if (t < -1 || t >= p.n_tok) bad_index(p.err, kSiteGemmGatherToken);
          tok[j] = (t >= 0 && t < p.n_tok) ? t : 0;
        }
      }
      for (int kb = 0; kb < KB; ++kb) {
        int okw = 1;
        if (lane == 0)
          okw = bounded_wait_pair<false>(&st->empty[stage], phase ^ 1u, st, p.err,
                                         kErrGemmTimeout | 0x41);
        if (!__shfl_sync(0xffffffffu, okw, 0)) {
          ok = false;
          break;
        }
        const uint32_t full_leader = sm100::mapa_shared(sm100::smem_addr(&st->full[stage]), 0);
        if (lane == 0) {
          if (leader) sm100::mbar_arrive_expect_tx(&st->full[stage], 2 * kPStageBytes);
          if (!gather) sm100::tma_load_2d_pair(sA(stage), ma, full_leader, kb * kBK, c.a_row);
          sm100::tma_load_2d_pair(sB(stage), mb, full_leader, kb * kBK, c.b_row);
        }
        if (gather)
          sm100::tma_gather4_pair(sA(stage) + lane * 4 * (kBK * 2), &tmXg, full_leader,
                                  kb * kBK, tok[0], tok[1], tok[2], tok[3]);
        ++issued;
        if (++stage == kPStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (lane == 0) {
      if (!ok && leader) {
        // wait (bounded) until the copies of the outstanding stages have landed
        int s = stage;
        uint32_t ph = phase;
        const int pending = issued < kPStages ? issued : kPStages;
        for (int i = 0; i < pending; ++i) {
          if (--s < 0) {
            s = kPStages - 1;
            ph ^= 1u;
          }
          const uint64_t t0 = global_timer_ns();
          while (!sm100::mbar_try_wait(&st->full[s], ph) &&
                 global_timer_ns() - t0 < kWaitLimitNs) {
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      constexpr uint32_t idesc = sm100::idesc_bf16_f32(2 * kBM, kBN);
      int stage = 0;
      uint32_t phase = 0;
      int local = 0;
      bool ok = true;
      for (int tile = pair_id; ok && tile < total; tile += num_pairs, ++local) {
        const int acc = local & 1;
        const uint32_t acc_phase = (uint32_t)(local >> 1) & 1u;
        if (!bounded_wait_pair<true>(&st->tempty[acc], acc_phase ^ 1u, st, p.err,
                                     kErrGemmTimeout | 0x52)) {
          ok = false;
          break;
        }
        sm100::tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(acc * kBN);
        for (int kb = 0; kb < KB; ++kb) {
          if (!bounded_wait_pair<false>(&st->full[stage], phase, st, p.err,
                                        kErrGemmTimeout | 0x53)) {
            ok = false;
            break;
          }
          sm100::tc_fence_after();
          const uint64_t adesc = sm100::sw128_kmajor_desc(sm100::smem_addr(sA(stage)));
          const uint64_t bdesc = sm100::sw128_kmajor_desc(sm100::smem_addr(sB(stage)));
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)
            sm100::umma_f16_pair(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, (kb | k) != 0);
          sm100::umma_commit_pair_mc(&st->empty[stage], 0x3);
          if (++stage == kPStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        sm100::umma_commit_pair_mc(&st->tfull[acc], 0x3);
      }
      sm100::umma_commit_pair_mc(&st->drain, 0x1);
      const uint64_t t0 = global_timer_ns();
      while (!sm100::mbar_try_wait(&st->drain, 0) && global_timer_ns() - t0 < kWaitLimitNs) {
      }
    }
  } else {
    const int q = warp & 3;
    const int row_in_tile = q * 32 + lane;
    constexpr int BNO = SWIGLU ? kBN / 2 : kBN;
    int local = 0;
    for (int tile = pair_id; tile < total; tile += num_pairs, ++local) {
      const int acc = local & 1;
      const uint32_t acc_phase = (uint32_t)(local >> 1) & 1u;
      if (!bounded_wait_pair<true>(&st->tfull[acc], acc_phase, st, p.err,
                                   kErrGemmTimeout | 0x64))
        break;
      sm100::tc_fence_after();
      const PairCoord c = decode_pair<ACT>(tile, p, st->offs, st->tprefix, routed, rank);
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * kBN);
      __nv_bfloat16* orow = p.out + (size_t)(c.out_row + row_in_tile) * p.n_out;
      // scatter: the row's token and gate (shared experts: weight 1, the
      // token is the row within the expert's block of n_pad rows)
      int tok = -1;
      float gate = 0.0f;
      if (FUSE == FUSE_SCATTER) {
        const long long r = c.out_row + row_in_tile;
        if (c.a_sel == 0) {
          tok = p.row_token[r];
          if (tok < -1 || tok >= p.n_tok) {
            bad_index(p.err, kSiteGemmScatterToken);
            tok = -1;
          }
          gate = tok >= 0 ? p.row_gate[r] : 0.0f;
        } else {
          const long long q2 = (r - p.out_shared_base) % p.n_pad;
          tok = q2 < p.n_tok ? (int)q2 : -1;
          gate = 1.0f;
        }
      }
      if (c.valid) {
#pragma unroll 1
        for (int cc = 0; cc < BNO; cc += 32) {
          if (c.col0 + cc >= p.n_out) break;
          uint32_t v[32];
          sm100::tmem_ld_32x32b_x32(tbase + cc, v);
          float f[32];
          if (SWIGLU) {
            uint32_t g[32];
            sm100::tmem_ld_32x32b_x32(tbase + BNO + cc, g);
            sm100::tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float a = __uint_as_float(v[i]);
              const float b = __uint_as_float(g[i]);
              f[i] = a * __frcp_rn(1.0f + __expf(-a)) * b;
            }
            if (FUSE == FUSE_SAVE) store_row32(p.save_v + (orow - p.out) + c.col0 + cc, g);
          } else {
            sm100::tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) f[i] = act_fn<ACT>(__uint_as_float(v[i]));
          }
          if (FUSE == FUSE_SAVE) store_row32(p.save_u + (orow - p.out) + c.col0 + cc, v);
          if (FUSE == FUSE_SCATTER) {
            if (tok >= 0) {
              float* dst = p.out32 + (size_t)tok * p.n_out + c.col0 + cc;
#pragma unroll
              for (int j = 0; j < 8; ++j)
                red_add_v4(dst + 4 * j, gate * f[4 * j], gate * f[4 * j + 1], gate * f[4 * j + 2],
                           gate * f[4 * j + 3]);
            }
          } else {
            uint4* dst = reinterpret_cast<uint4*>(orow + c.col0 + cc);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              uint4 o;
              o.x = pack_bf16x2(f[8 * j + 0], f[8 * j + 1]);
              o.y = pack_bf16x2(f[8 * j + 2], f[8 * j + 3]);
              o.z = pack_bf16x2(f[8 * j + 4], f[8 * j + 5]);
              o.w = pack_bf16x2(f[8 * j + 6], f[8 * j + 7]);
              dst[j] = o;
            }
          }
        }
      }
      sm100::tc_fence_before();
      sm100::mbar_arrive_cluster(sm100::mapa_shared(sm100::smem_addr(&st->tempty[acc]), 0));
    }
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::cluster_sync();  // no CTA leaves while its peer may still signal it
  if (warp == 1) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc_pair(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D bf16 row-major [rows, cols] map with a box of 64 columns x box_rows rows
// and 128-byte swizzle. Out-of-range elements (including a box taller than
// the whole tensor) load as zero.
bool make_bf16_sw128_map(CUtensorMap* m, const void* ptr, long long rows, long long cols,
                         int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows < 1 || cols < kBK) return false;
  if ((reinterpret_cast<uintptr_t>(ptr) & 15) || ((cols * 2) & 15)) return false;
  const cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t gstride[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)box_rows};
  const cuuint32_t estride[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), gdim, gstride,
            box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static size_t gemm_smem_bytes(bool pair) {
  return pair ? (size_t)kPStages * kPStageBytes + sizeof(PairState) + 1024
              : (size_t)kStages * kStageBytes + sizeof(SharedState) + 1024;
}

struct Maps {
  CUtensorMap a0, a1, b0, b0g, b1, b1g, xg;  // xg: X with a one-row box (gathered A)
};

template <class K>
static cudaError_t launch_one(K kern, const Maps& m, const TcGemmParams& p, int ctas,
                             size_t bytes, cudaStream_t s) {
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, ctas, kGemmThreads, bytes, s, m.a0, m.a1, m.b0, m.b0g, m.b1, m.b1g, m.xg, p);
}

// grid: CTAs for the single-CTA kernel, CTA pairs for the pair kernel
template <int ACT, int FUSE>
static cudaError_t launch_gemm_t(const Maps& m, const TcGemmParams& p, bool pair, int grid,
                                 cudaStream_t s) {
  const size_t bytes = gemm_smem_bytes(pair);
  if (pair) return launch_one(tc_grouped_gemm_pair_kernel<ACT, FUSE>, m, p, 2 * grid, bytes, s);
  return launch_one(tc_grouped_gemm_kernel<ACT, FUSE>, m, p, grid, bytes, s);
}

// up projections fuse nothing, the gather, or the saving of U (and V)
template <int ACT>
static cudaError_t launch_gemm(const Maps& m, const TcGemmParams& p, bool pair, bool gather,
                               int grid, cudaStream_t s) {
  if (p.save_u) return launch_gemm_t<ACT, FUSE_SAVE>(m, p, pair, grid, s);
  return gather ? launch_gemm_t<ACT, FUSE_GATHER>(m, p, pair, grid, s)
                : launch_gemm_t<ACT, FUSE_NONE>(m, p, pair, grid, s);
}

static int num_sms() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

// Persistent grid: one CTA (or CTA pair) per SM (pair of SMs), never more
// than there are tiles.
static int persistent_grid(const TcGemmParams& p, bool pair) {
  const int sms = num_sms();
  long long units;
  int slots;
  if (pair) {
    const long long spp = (p.shared_tiles_per + 1) / 2;
    units = ((long long)p.max_routed_tiles + p.n_shared * spp) * p.nt_tiles;
    slots = sms / 2;
  } else {
    units = ((long long)p.max_routed_tiles + (long long)p.n_shared * p.shared_tiles_per) *
            p.nt_tiles;
    slots = sms;
  }
  long long g = units < slots ? units : slots;
  return g < 1 ? 1 : (int)g;
}

// One-shot failure-path test hooks (moe_debug_inject_fault): armed on the
// host, taken by the next up projection that can honour them.
static std::atomic<int> g_fault{0};

moe_status set_fault(int fault) {
  if (fault < MOE_FAULT_NONE || fault > MOE_FAULT_LAUNCH) return MOE_ERR_INVALID_ARG;
  g_fault.store(fault);
  return MOE_OK;
}

// the armed fault if it is `kind` (then disarmed), else MOE_FAULT_NONE
static int take_fault(int kind) {
  int want = kind;
  return g_fault.compare_exchange_strong(want, MOE_FAULT_NONE) ? kind : MOE_FAULT_NONE;
}

moe_status run_ffn_bf16(const FfnArgs& f, cudaStream_t s) {
  const bool swiglu = f.act == MOE_ACT_SWIGLU;
  const bool pair = f.pair;
  const long long rows = f.rows;
  const int sh_tiles = f.n_pad / kBM;
  // ---- up projection: H = act(X_perm W1^T) or silu(X_perm W1^T) * (X_perm W3^T)
  // B box rows: a pair CTA loads half of the 256-row B tile; a single CTA
  // loads all of it (SwiGLU: 128 rows of W1 plus 128 of W3)
  const int b_box_up = (pair || swiglu) ? kBN / 2 : kBN;
  const int b_box_dn = pair ? kBN / 2 : kBN;
  const int out_cols_up = swiglu ? kBN / 2 : kBN;
  Maps m;
  const bool gather = f.X_perm == nullptr;  // A rows read from X through row_token
  if (gather) {
    // a box one row high: what a 4-row gather needs
    if (!make_bf16_sw128_map(&m.xg, f.X, f.n, f.d, 1)) return MOE_ERR_UNSUPPORTED;
    m.a0 = m.xg;  // unused for routed tiles when gathering
  } else {
    if (!make_bf16_sw128_map(&m.a0, f.X_perm, rows, f.d, kBM)) return MOE_ERR_UNSUPPORTED;
    m.xg = m.a0;
  }
  if (f.n_shared > 0) {
    if (!make_bf16_sw128_map(&m.a1, f.X, f.n, f.d, kBM)) return MOE_ERR_UNSUPPORTED;
  } else {
    m.a1 = m.a0;
  }
  if (!make_bf16_sw128_map(&m.b0, f.W1, (long long)f.E * f.h, f.d, b_box_up)) return MOE_ERR_UNSUPPORTED;
  if (swiglu) {
    if (!make_bf16_sw128_map(&m.b0g, f.W3, (long long)f.E * f.h, f.d, b_box_up))
      return MOE_ERR_UNSUPPORTED;
  } else {
    m.b0g = m.b0;
  }
  if (f.n_shared > 0) {
    if (!make_bf16_sw128_map(&m.b1, f.sW1, (long long)f.n_shared * f.h, f.d, b_box_up))
      return MOE_ERR_UNSUPPORTED;
    if (swiglu) {
      if (!make_bf16_sw128_map(&m.b1g, f.sW3, (long long)f.n_shared * f.h, f.d, b_box_up))
        return MOE_ERR_UNSUPPORTED;
    } else {
      m.b1g = m.b1;
    }
  } else {
    m.b1 = m.b0;
    m.b1g = m.b0g;
  }
  TcGemmParams p{};
  p.offsets = f.offsets;
  p.E = f.E;
  p.K = f.d;
  p.n_out = f.h;
  p.nt_tiles = ceil_div(f.h, out_cols_up);
  p.b_rows_per_expert = f.h;
  p.shared_tiles_per = sh_tiles;
  p.n_shared = f.n_shared;
  p.max_routed_tiles = (int)(f.rows_routed / kBM);
  p.a1_row_base = 0;
  p.a1_row_stride = 0;
  p.out_shared_base = f.shared_base;
  p.n_pad = f.n_pad;
  p.out = static_cast<__nv_bfloat16*>(f.H);
  p.err = f.err;
  p.row_token = f.row_token;
  p.n_tok = f.n;
  p.save_u = static_cast<__nv_bfloat16*>(f.save_u);
  p.save_v = static_cast<__nv_bfloat16*>(f.save_v);
  // failure-path tests: a launch that fails on the host, or (single-CTA
  // kernel) a producer that issues no loads
  if (take_fault(MOE_FAULT_LAUNCH) == MOE_FAULT_LAUNCH) return MOE_ERR_CUDA;
  if (!pair) p.inject_no_loads = take_fault(MOE_FAULT_GEMM_NO_LOADS) == MOE_FAULT_GEMM_NO_LOADS;
  cudaError_t e = cudaSuccess;
  const int grid_up = persistent_grid(p, pair);
  switch (f.act) {
    case MOE_ACT_RELU: e = launch_gemm<ACT_RELU>(m, p, pair, gather, grid_up, s); break;
    case MOE_ACT_GELU: e = launch_gemm<ACT_GELU>(m, p, pair, gather, grid_up, s); break;
    default: e = launch_gemm<ACT_SWIGLU>(m, p, pair, gather, grid_up, s); break;
  }
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  if (f.skip_down) return MOE_OK;

  // ---- down projection: Y = H W2^T
  Maps dm;
  if (!make_bf16_sw128_map(&dm.a0, f.H, rows, f.h, kBM)) return MOE_ERR_UNSUPPORTED;
  dm.a1 = dm.a0;
  if (!make_bf16_sw128_map(&dm.b0, f.W2, (long long)f.E * f.d, f.h, b_box_dn)) return MOE_ERR_UNSUPPORTED;
  dm.b0g = dm.b0;
  if (f.n_shared > 0) {
    if (!make_bf16_sw128_map(&dm.b1, f.sW2, (long long)f.n_shared * f.d, f.h, b_box_dn))
      return MOE_ERR_UNSUPPORTED;
  } else {
    dm.b1 = dm.b0;
  }
  dm.b1g = dm.b1;
  dm.xg = dm.a0;
  TcGemmParams q = p;
  q.save_u = q.save_v = nullptr;
  q.inject_no_loads = 0;
  q.K = f.h;
  q.n_out = f.d;
  q.nt_tiles = ceil_div(f.d, kBN);
  q.b_rows_per_expert = f.d;
  q.a1_row_base = f.shared_base;
  q.a1_row_stride = f.n_pad;
  q.out = static_cast<__nv_bfloat16*>(f.Y);
  if (f.out32) {
    // the combine fused into the epilogue: out32[token] += gate * Y row
    q.row_gate = f.row_gate;
    q.out32 = f.out32;
    q.n_tok = f.n;
    e = launch_gemm_t<ACT_NONE, FUSE_SCATTER>(dm, q, pair, persistent_grid(q, pair), s);
  } else {
    e = launch_gemm_t<ACT_NONE, FUSE_NONE>(dm, q, pair, persistent_grid(q, pair), s);
  }
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // namespace moe
