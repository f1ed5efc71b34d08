// fp32 grouped expert FFN on FFMA (no TF32: the fp32 workload keeps full
// single precision end to end). Same dispatched-row layout as the tensor-core
// path: a 64-row tile always lies inside one expert's 128-aligned segment.
//
// "Expert choice routing" (aicassindra.com), "The math": Expert_e(X_in[e])
// on dense per-expert batches.
#include <math.h>

#include "device_common.cuh"
#include "moe_internal.h"

namespace moe {

constexpr int kFBM = 64, kFBN = 64, kFBK = 16;

struct F32GemmArgs {
  const float* A;        // routed A rows [rows, K], or NULL: gather X rows via row_token
  const float* Xg;       // X [n, K] for the gathered routed rows
  const int32_t* row_token;
  const float* A_shared; // shared A rows [n, K] (X for the up projection, else A)
  long long a_shared_base;  // row of shared expert 0 in A_shared, stride a_shared_stride
  long long a_shared_stride;
  const int32_t* offsets;
  const float* B;        // [E, N, K]
  const float* B3;       // [E, N, K] (SwiGLU)
  const float* sB;       // [n_shared, N, K]
  const float* sB3;
  float* C;              // [rows, N]
  int N, K, E, n, n_pad, n_shared, act;  // act: 0 none, 1 relu, 2 gelu, 3 swiglu
  long long rows_routed;
  long long shared_base;
};

__device__ __forceinline__ int find_expert(const int32_t* offsets, int E, int row) {
  int lo = 0, hi = E - 1;  // largest e with offsets[e] <= row
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (offsets[mid] <= row) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <bool SWIGLU>
__global__ void __launch_bounds__(256) ffn_f32_kernel(F32GemmArgs a) {
  pdl_wait();
  __shared__ float As[kFBK][kFBM + 4];
  __shared__ float Bs[kFBK][kFBN + 4];
  __shared__ float B3s[SWIGLU ? kFBK : 1][kFBN + 4];
  const long long m0 = (long long)blockIdx.y * kFBM;
  const int n0 = blockIdx.x * kFBN;
  const float* A;
  const float* B;
  const float* B3 = nullptr;
  long long out_row0;
  int a_rows_valid;  // rows of this tile backed by real A rows
  bool gathered = false;
  if (m0 < a.rows_routed) {
    const int used = a.offsets[a.E];
    if (m0 >= used) return;
    const int e = find_expert(a.offsets, a.E, (int)m0);
    gathered = a.A == nullptr;
    A = gathered ? a.Xg : a.A + m0 * a.K;
    B = a.B + (size_t)e * a.N * a.K;
    if (SWIGLU) B3 = a.B3 + (size_t)e * a.N * a.K;
    out_row0 = m0;
    a_rows_valid = kFBM;
  } else {
    const long long q = m0 - a.rows_routed;
    const int s = (int)(q / a.n_pad);
    const long long local = q % a.n_pad;
    A = a.A_shared + (a.a_shared_base + s * a.a_shared_stride + local) * a.K;
    B = a.sB + (size_t)s * a.N * a.K;
    if (SWIGLU) B3 = a.sB3 + (size_t)s * a.N * a.K;
    out_row0 = a.shared_base + (long long)s * a.n_pad + local;
    a_rows_valid = (int)min((long long)kFBM, (long long)a.n - local);
  }
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  float acc[4][4] = {}, acc3[4][4] = {};
  for (int k0 = 0; k0 < a.K; k0 += kFBK) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int q = tid + i * 256;  // 0..1023 over a 64 x 16 tile
      const int r = q / kFBK, kk = q % kFBK;
      const int k = k0 + kk;
      float av = 0.0f;
      if (r < a_rows_valid && k < a.K) {
        if (gathered) {
          const int t = a.row_token[m0 + r];
          if (t >= 0) av = A[(size_t)t * a.K + k];
        } else {
          av = A[(size_t)r * a.K + k];
        }
      }
      As[kk][r] = av;
      const int c = n0 + r;
      Bs[kk][r] = (c < a.N && k < a.K) ? B[(size_t)c * a.K + k] : 0.0f;
      if (SWIGLU) B3s[kk][r] = (c < a.N && k < a.K) ? B3[(size_t)c * a.K + k] : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kFBK; ++kk) {
      float av[4], bv[4], b3v[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        bv[j] = Bs[kk][tx * 4 + j];
        if (SWIGLU) b3v[j] = B3s[kk][tx * 4 + j];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
          if (SWIGLU) acc3[i][j] = fmaf(av[i], b3v[j], acc3[i][j]);
        }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const long long row = out_row0 + ty * 4 + i;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = n0 + tx * 4 + j;
      if (c >= a.N) continue;
      float v = acc[i][j];
      if (SWIGLU) {
        v = v / (1.0f + expf(-v)) * acc3[i][j];
      } else if (a.act == 1) {
        v = fmaxf(v, 0.0f);
      } else if (a.act == 2) {
        v = 0.5f * v * (1.0f + erff(v * 0.70710678118654752f));
      }
      a.C[(size_t)row * a.N + c] = v;
    }
  }
}

static cudaError_t launch_f32_gemm(const F32GemmArgs& a, long long total_rows,
                                   cudaStream_t s) {
  dim3 grid(ceil_div(a.N, kFBN), (unsigned)(total_rows / kFBM));
  if (a.act == 3)
    return launch_pdl(ffn_f32_kernel<true>, grid, 256, 0, s, a);
  return launch_pdl(ffn_f32_kernel<false>, grid, 256, 0, s, a);
}

moe_status run_ffn_f32(const FfnArgs& f, cudaStream_t s) {
  const long long total_rows = f.rows_routed + (long long)f.n_shared * f.n_pad;
  F32GemmArgs up{};
  up.A = static_cast<const float*>(f.X_perm);
  up.Xg = static_cast<const float*>(f.X);
  up.row_token = f.row_token;
  up.A_shared = static_cast<const float*>(f.X);
  up.a_shared_base = 0;
  up.a_shared_stride = 0;
  up.offsets = f.offsets;
  up.B = static_cast<const float*>(f.W1);
  up.B3 = static_cast<const float*>(f.W3);
  up.sB = static_cast<const float*>(f.sW1);
  up.sB3 = static_cast<const float*>(f.sW3);
  up.C = static_cast<float*>(f.H);
  up.N = f.h;
  up.K = f.d;
  up.E = f.E;
  up.n = f.n;
  up.n_pad = f.n_pad;
  up.n_shared = f.n_shared;
  up.act = f.act == MOE_ACT_SWIGLU ? 3 : f.act == MOE_ACT_GELU ? 2 : 1;
  up.rows_routed = f.rows_routed;
  up.shared_base = f.shared_base;
  if (launch_f32_gemm(up, total_rows, s) != cudaSuccess) return MOE_ERR_CUDA;

  F32GemmArgs dn = up;
  dn.A = static_cast<const float*>(f.H);
  dn.A_shared = static_cast<const float*>(f.H);
  dn.a_shared_base = f.shared_base;
  dn.a_shared_stride = f.n_pad;
  dn.B = static_cast<const float*>(f.W2);
  dn.B3 = nullptr;
  dn.sB = static_cast<const float*>(f.sW2);
  dn.sB3 = nullptr;
  dn.C = static_cast<float*>(f.Y);
  dn.N = f.d;
  dn.K = f.h;
  dn.act = 0;
  if (launch_f32_gemm(dn, total_rows, s) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // namespace moe
