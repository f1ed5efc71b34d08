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

namespace moe {

// One warp per dispatched row, 16-byte vectors, four in flight per lane.
__global__ void __launch_bounds__(256) gather_kernel(GatherArgs a) {
  const int rows = min((long long)a.offsets[a.E], a.max_rows);
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  const int nvec = a.d * a.elt_bytes / 16;
  const uint4* src = reinterpret_cast<const uint4*>(a.X);
  uint4* dst = reinterpret_cast<uint4*>(a.X_perm);
  for (int r = gw; r < rows; r += nw) {
    const int t = a.row_token[r];
    if (t < 0) continue;
    const uint4* s = src + (size_t)t * nvec;
    uint4* o = dst + (size_t)r * nvec;
    int v = lane;
    for (; v + 96 < nvec; v += 128) {
      const uint4 x0 = __ldg(s + v), x1 = __ldg(s + v + 32), x2 = __ldg(s + v + 64),
                  x3 = __ldg(s + v + 96);
      o[v] = x0;
      o[v + 32] = x1;
      o[v + 64] = x2;
      o[v + 96] = x3;
    }
    for (; v < nvec; v += 32) o[v] = __ldg(s + v);
  }
}

cudaError_t launch_gather(const GatherArgs& a, cudaStream_t s) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  gather_kernel<<<sms * 8, 256, 0, s>>>(a);
  return cudaGetLastError();
}

// One CTA per token; each thread owns 16-byte chunks of the output row and
// sums the gate-scaled expert rows in list order (fp32), then the shared
// experts with weight 1.
template <bool BF16>
__global__ void __launch_bounds__(128) combine_kernel(CombineArgs a) {
  __shared__ int rows_s[MOE_MAX_EXPERTS];
  __shared__ float gates_s[MOE_MAX_EXPERTS];
  __shared__ int cnt_s;
  const int t = blockIdx.x;
  const int slots = a.slots;
  if (threadIdx.x == 0) cnt_s = slots;
  __syncthreads();
  for (int j = threadIdx.x; j < slots; j += blockDim.x) {
    int r = a.tok_row[(size_t)t * slots + j];
    if (r >= a.max_rows) r = -1;
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
    combine_kernel<true><<<a.n, 128, 0, s>>>(a);
  else
    combine_kernel<false><<<a.n, 128, 0, s>>>(a);
  return cudaGetLastError();
}

// "MoE routing strategies explained", "4. Sigmoid gating with aux-loss-free
// bias": after each step the bias drops for overloaded experts and rises for
// idle ones. The sign is taken exactly in integers: load*E vs n*K.
__global__ void bias_update_kernel(int n, int E, int K, const int32_t* load, float rate,
                                   float* bias) {
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
  bias_update_kernel<<<ceil_div(E, 256), 256, 0, s>>>(n, E, K, load, rate, bias);
  return cudaGetLastError();
}

}  // namespace moe
