// Dispatch gather, gate-scaled combine and the selection-bias update.
//
// "Expert choice routing" (aicassindra.com), "The math: a gating matrix and
// top-k over tokens": X_in[e] = P[e] X with P = onehot(I) is done here as an
// index gather (never a one-hot matmul); Y[e] = G[e] * Expert_e(X_in[e]) and
// out = scatter_add(Y, I) are done owner-side: each output row sums its own
// gate-scaled expert rows, so no two threads ever add into the same output
// and the result does not depend on scheduling.
#include "device_common.cuh"
#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {

// ---------------------------------------------------------------------------
// Dispatch gather, token by token, with TMA row staging. Each warp runs its
// own ring of row buffers in shared memory. Lane 0 brings a token's row (or
// one segment of a long row) in with one bulk copy that completes on the
// slot's mbarrier; then each lane that holds one of the token's dispatched
// rows (tok_row: kept entries first, then -1) writes the staged bytes there
// with a bulk copy out of shared memory. X is read from HBM once, every
// dispatched row is written once, and the copy engine moves all the bytes.
// Loads run ring - 1 units ahead of the stores. The slot wait is bounded: on
// a timeout the warp records an error, waits (bounded) for its own loads
// still in flight, and stops.
// ---------------------------------------------------------------------------
constexpr int kGatherSeg = 16384;   // largest staged unit, bytes
constexpr int kGatherMaxRing = 8;
constexpr int kGatherMaxWarps = 8;
constexpr size_t kGatherSmemBudget = 200 * 1024;
constexpr uint64_t kGatherWaitNs = 2000000000ull;  // 2 s
constexpr int kGatherRowRegs = MOE_MAX_EXPERTS / 32;
// average rows per token from which the staged kernel is used (measured on
// B200: it wins at 8 rows per token, loses at 2)
constexpr int kGatherStagedFanout = 4;

__device__ int g_dispatch_error;  // timeouts of standalone dispatch calls

__global__ void gather_kernel(GatherArgs a, int seg, int nseg, int ring, int slot_stride) {
  pdl_wait();
  extern __shared__ __align__(128) unsigned char gsm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  unsigned char* buf = gsm + (size_t)warp * ring * slot_stride;
  uint64_t* bar = reinterpret_cast<uint64_t*>(gsm + (size_t)warps * ring * slot_stride) +
                  warp * kGatherMaxRing;
  int* err = a.err ? a.err : &g_dispatch_error;
  if (lane == 0) {
    for (int i = 0; i < ring; ++i) sm100::mbar_init(&bar[i], 1);
    sm100::fence_mbar_init();
  }
  __syncwarp();
  const int row_bytes = a.row_bytes;
  const long long units = (long long)a.n * nseg;
  const long long first = (long long)blockIdx.x * warps + warp;
  const long long stride = (long long)gridDim.x * warps;
  const unsigned char* X = static_cast<const unsigned char*>(a.X);
  unsigned char* XP = static_cast<unsigned char*>(a.X_perm);
  auto unit_bytes = [&](int sg) { return (uint32_t)min(seg, row_bytes - sg * seg); };
  auto issue = [&](long long i) {  // lane 0: stage unit i of this warp
    const long long u = first + i * stride;
    if (u >= units) return;
    const int t = (int)(u / nseg), sg = (int)(u % nseg);
    const int slot = (int)(i % ring);
    const uint32_t b = unit_bytes(sg);
    sm100::mbar_arrive_expect_tx(&bar[slot], b);
    sm100::bulk_load_smem(buf + (size_t)slot * slot_stride,
                          X + (size_t)t * row_bytes + (size_t)sg * seg, b, &bar[slot]);
  };
  if (lane == 0)
    for (int i = 0; i < ring - 1; ++i) issue(i);
  long long i = 0;
  bool ok = true;
  for (; first + i * stride < units; ++i) {
    const long long u = first + i * stride;
    const int t = (int)(u / nseg), sg = (int)(u % nseg);
    const int slot = (int)(i % ring);
    const uint32_t parity = (uint32_t)((i / ring) & 1);
    int rr[kGatherRowRegs];
#pragma unroll
    for (int c = 0; c < kGatherRowRegs; ++c) {
      const int j = c * 32 + lane;
      rr[c] = j < a.slots ? a.tok_row[(size_t)t * a.slots + j] : -1;
    }
    // refill the slot unit i - 1 used: its stores finished reading it
    if (lane == 0) issue(i + ring - 1);
    int okw = 1;
    if (lane == 0) {
      if (!sm100::mbar_try_wait(&bar[slot], parity)) {
        const uint64_t t0 = global_timer_ns();
        while (!sm100::mbar_try_wait(&bar[slot], parity)) {
          if (global_timer_ns() - t0 > kGatherWaitNs) {
            report_error(err, kErrGemmTimeout | 0x50);
            okw = 0;
            break;
          }
        }
      }
    }
    if (!__shfl_sync(0xffffffffu, okw, 0)) {
      ok = false;
      break;
    }
    sm100::fence_proxy_async_smem();
    const unsigned char* src = buf + (size_t)slot * slot_stride;
    const uint32_t b = unit_bytes(sg);
#pragma unroll
    for (int c = 0; c < kGatherRowRegs; ++c) {
      const int r = rr[c];
      if (r >= 0 && r < a.max_rows)
        sm100::bulk_store_global(XP + (size_t)r * row_bytes + (size_t)sg * seg, src, b);
      else if (r < -1 || r >= a.max_rows)
        bad_index(err, kSiteGatherTokRow);
    }
    sm100::bulk_commit_group();
    sm100::bulk_wait_read_all();
    __syncwarp();
  }
  if (!ok && lane == 0) {
    // wait (bounded) for the loads this warp still has in flight
    for (long long q = i; q < i + ring - 1 + 1 && first + q * stride < units; ++q) {
      const uint64_t t0 = global_timer_ns();
      while (!sm100::mbar_try_wait(&bar[q % ring], (uint32_t)((q / ring) & 1)) &&
             global_timer_ns() - t0 < kGatherWaitNs) {
      }
    }
  }
  sm100::bulk_wait_all();
}

// Low fan-out (a token feeds one or two rows on average): each warp copies
// kRowsPerWarp consecutive dispatched rows with 16-byte vectors. The row
// indices are loaded together, then every row's vectors, so a warp keeps
// kRowsPerWarp rows' worth of loads in flight instead of one. A token's row
// is read about once anyway, and the warps cover all rows at once, where the
// staged kernel would serialise a few round trips per warp.
constexpr int kRowsPerWarp = 4;

__global__ void __launch_bounds__(256) gather_rows_kernel(GatherArgs a) {
  pdl_wait();
  int* err = a.err ? a.err : &g_dispatch_error;
  const long long used = a.offsets[a.E];
  const long long rows = min(used, a.max_rows);
  if (blockIdx.x == 0 && threadIdx.x == 0 && (used < 0 || used > a.max_rows))
    bad_index(err, kSiteGatherOffsets);
  const int lane = threadIdx.x & 31;
  const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long nw = ((long long)gridDim.x * blockDim.x) >> 5;
  const int nvec = a.row_bytes / 16;
  const uint4* src = reinterpret_cast<const uint4*>(a.X);
  uint4* dst = reinterpret_cast<uint4*>(a.X_perm);
  for (long long r0 = gw * kRowsPerWarp; r0 < rows; r0 += nw * kRowsPerWarp) {
    int tok[kRowsPerWarp];
#pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i) {
      const long long r = r0 + i;
      const int t = r < rows ? a.row_token[r] : -1;
      tok[i] = (t >= 0 && t < a.n) ? t : -1;
      if (t < -1 || t >= a.n) bad_index(err, kSiteGatherRowToken);
    }
    for (int v0 = 0; v0 < nvec; v0 += 128) {
      uint4 x[kRowsPerWarp][4];
#pragma unroll
      for (int i = 0; i < kRowsPerWarp; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int v = v0 + j * 32 + lane;
          if (tok[i] >= 0 && v < nvec) x[i][j] = __ldg(src + (size_t)tok[i] * nvec + v);
        }
#pragma unroll
      for (int i = 0; i < kRowsPerWarp; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int v = v0 + j * 32 + lane;
          if (tok[i] >= 0 && v < nvec) dst[(size_t)(r0 + i) * nvec + v] = x[i][j];
        }
    }
  }
}

int take_dispatch_error() {
  int code = 0;
  if (cudaMemcpyFromSymbol(&code, g_dispatch_error, sizeof(int)) != cudaSuccess) return 0;
  if (code) {
    const int zero = 0;
    cudaMemcpyToSymbol(g_dispatch_error, &zero, sizeof(int));
  }
  return code;
}

cudaError_t launch_gather(const GatherArgs& a, cudaStream_t s) {
  if (a.row_bytes <= 0 || a.row_bytes % 16 || a.n < 1) return cudaErrorInvalidValue;
  if (a.fanout < kGatherStagedFanout) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long warps = (a.max_rows + kRowsPerWarp - 1) / kRowsPerWarp;
    long long ctas = (warps + 7) / 8;
    if (ctas > (long long)sms * 8) ctas = (long long)sms * 8;
    if (ctas < 1) ctas = 1;
    return launch_pdl(gather_rows_kernel, (int)ctas, 256, 0, s, a);
  }
  const int nseg = (a.row_bytes + kGatherSeg - 1) / kGatherSeg;
  const int seg = ((a.row_bytes + nseg - 1) / nseg + 15) / 16 * 16;
  if ((long long)(nseg - 1) * seg >= a.row_bytes) return cudaErrorInvalidValue;
  const int slot_stride = (seg + 127) / 128 * 128;
  int ring = (int)(kGatherSmemBudget / ((size_t)kGatherMaxWarps * slot_stride));
  ring = ring < 2 ? 2 : ring > kGatherMaxRing ? kGatherMaxRing : ring;
  int warps = (int)(kGatherSmemBudget / ((size_t)ring * slot_stride));
  warps = warps < 1 ? 1 : warps > kGatherMaxWarps ? kGatherMaxWarps : warps;
  const size_t smem = (size_t)warps * ring * slot_stride + (size_t)warps * kGatherMaxRing * 8;
  int dev = 0, sms = 148, max_smem = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
  cudaError_t e = cudaFuncSetAttribute(gather_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = (int)(max_smem / (smem + 1024));
  per_sm = per_sm < 1 ? 1 : per_sm > 4 ? 4 : per_sm;
  return launch_pdl(gather_kernel, sms * per_sm, warps * 32, smem, s, a, seg, nseg, ring, slot_stride);
}

// One CTA per token; each thread owns 16-byte chunks of the output row and
// sums the gate-scaled expert rows in list order (fp32), then the shared
// experts with weight 1.
template <bool BF16>
__global__ void __launch_bounds__(128) combine_kernel(CombineArgs a) {
  pdl_wait();
  __shared__ int rows_s[MOE_MAX_EXPERTS];
  __shared__ float gates_s[MOE_MAX_EXPERTS];
  __shared__ int cnt_s;
  const int t = blockIdx.x;
  const int slots = a.slots;
  if (threadIdx.x == 0) cnt_s = slots;
  __syncthreads();
  for (int j = threadIdx.x; j < slots; j += blockDim.x) {
    int r = a.tok_row[(size_t)t * slots + j];
    if (r < -1 || r >= a.max_rows) {
      bad_index(a.err ? a.err : &g_dispatch_error, kSiteCombineTokRow);
      r = -1;
    }
    rows_s[j] = r;
    gates_s[j] = a.tok_gate[(size_t)t * slots + j];
    if (r < 0) atomicMin(&cnt_s, j);
  }
  __syncthreads();
  const int cnt = cnt_s;
  constexpr int EPV = BF16 ? 8 : 4;  // elements per 16-byte vector
  const int nvec = a.d / EPV;
  const uint4* Y = reinterpret_cast<const uint4*>(a.Y);
  uint4* out = reinterpret_cast<uint4*>(a.out);
  for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
    float acc[EPV];
#pragma unroll
    for (int i = 0; i < EPV; ++i) acc[i] = 0.0f;
    auto add = [&](long long row, float g) {
      const uint4 y = __ldg(Y + (size_t)row * nvec + v);
      const uint32_t w[4] = {y.x, y.y, y.z, y.w};
      if (BF16) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[2 * i] = fmaf(g, __uint_as_float(w[i] << 16), acc[2 * i]);
          acc[2 * i + 1] = fmaf(g, __uint_as_float(w[i] & 0xffff0000u), acc[2 * i + 1]);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[i] = fmaf(g, __uint_as_float(w[i]), acc[i]);
      }
    };
    for (int j = 0; j < cnt; ++j) add(rows_s[j], gates_s[j]);
    for (int sidx = 0; sidx < a.n_shared; ++sidx)
      add(a.shared_base + (long long)sidx * a.n_pad + t, 1.0f);
    uint4 o;
    if (BF16) {
      o.x = pack_bf16x2(acc[0], acc[1]);
      o.y = pack_bf16x2(acc[2], acc[3]);
      o.z = pack_bf16x2(acc[4], acc[5]);
      o.w = pack_bf16x2(acc[6], acc[7]);
    } else {
      o.x = __float_as_uint(acc[0]);
      o.y = __float_as_uint(acc[1]);
      o.z = __float_as_uint(acc[2]);
      o.w = __float_as_uint(acc[3]);
    }
    out[(size_t)t * nvec + v] = o;
  }
}

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t s) {
  if (a.bf16)
    return launch_pdl(combine_kernel<true>, a.n, 128, 0, s, a);
  return launch_pdl(combine_kernel<false>, a.n, 128, 0, s, a);
}

// The combine fused into the down projection ("Expert choice routing",
// "The math": out = scatter_add(G * Y)): the epilogue adds gate * Y rows into
// an fp32 [n, d] buffer with vector reductions. Before it, this kernel zeroes
// the buffer and writes each dispatched row's gate; after it, the buffer is
// rounded into the output.
__global__ void __launch_bounds__(256) combine_prep_kernel(const int32_t* tok_row,
                                                           const float* tok_gate, int n,
                                                           int slots, int d, long long max_rows,
                                                           float* row_gate, float* out32,
                                                           int* err) {
  pdl_wait();
  const long long tid = (long long)blockIdx.x * 256 + threadIdx.x;
  const long long nthreads = (long long)gridDim.x * 256;
  for (long long q = tid; q < (long long)n * slots; q += nthreads) {
    const int r = tok_row[q];
    if (r >= 0 && r < max_rows)
      row_gate[r] = tok_gate[q];
    else if (r < -1 || r >= max_rows)
      bad_index(err ? err : &g_dispatch_error, kSiteCombinePrepTokRow);
  }
  const long long nvec = (long long)n * d / 4;
  const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
  for (long long q = tid; q < nvec; q += nthreads) reinterpret_cast<float4*>(out32)[q] = z;
}

__global__ void __launch_bounds__(256) combine_finish_kernel(const float* out32, long long count,
                                                             __nv_bfloat16* out) {
  pdl_wait();
  const long long nvec = count / 8;
  for (long long q = (long long)blockIdx.x * 256 + threadIdx.x; q < nvec;
       q += (long long)gridDim.x * 256) {
    const float4 a = reinterpret_cast<const float4*>(out32)[2 * q];
    const float4 b = reinterpret_cast<const float4*>(out32)[2 * q + 1];
    reinterpret_cast<uint4*>(out)[q] = make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w),
                                                  pack_bf16x2(b.x, b.y), pack_bf16x2(b.z, b.w));
  }
}

static int fill_grid() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return 4 * sms;
}

cudaError_t launch_combine_prep(const int32_t* tok_row, const float* tok_gate, int n, int slots,
                                int d, long long max_rows, float* row_gate, float* out32,
                                int* err, cudaStream_t s) {
  return launch_pdl(combine_prep_kernel, fill_grid(), 256, 0, s, tok_row, tok_gate, n, slots, d,
                    max_rows, row_gate, out32, err);
}

cudaError_t launch_combine_finish(const float* out32, int n, int d, void* out, cudaStream_t s) {
  return launch_pdl(combine_finish_kernel, fill_grid(), 256, 0, s, out32, (long long)n * d,
                    static_cast<__nv_bfloat16*>(out));
}

// "MoE routing strategies explained", "4. Sigmoid gating with aux-loss-free
// bias": after each step the bias drops for overloaded experts and rises for
// idle ones. The sign is taken exactly in integers: load*E vs n*K.
__global__ void bias_update_kernel(int n, int E, int K, const int32_t* load, float rate,
                                   float* bias) {
  pdl_wait();
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= E) return;
  const long long diff = (long long)load[e] * E - (long long)n * K;
  if (diff > 0)
    bias[e] = bias[e] - rate;
  else if (diff < 0)
    bias[e] = bias[e] + rate;
}

cudaError_t launch_bias_update(int n, int E, int K, const int32_t* load, float rate,
                               float* bias, cudaStream_t s) {
  return launch_pdl(bias_update_kernel, ceil_div(E, 256), 256, 0, s, n, E, K, load, rate, bias);
}

}  // namespace moe
