// fp32 grouped GEMMs of the layer's backward pass on FFMA (no TF32: the fp32
// workload keeps full single precision end to end, as its forward does).
// The same five steps as the tensor-core backward (gemm_bwd.cu), by the chain
// rule through "Expert choice routing" (aicassindra.com), "The math": the
// recompute of U, V, H; dU, dV = (dY W2) * act'; dX_perm = dU W1 + dV W3;
// dW2 = dY^T H and [dW1; dW3] = [dU | dV]^T X per expert.
// 64 x 64 output tiles, 256 threads with 4 x 4 outputs each, 16-deep K chunks
// through shared memory. Row modes tile the dispatched rows (a 64-row tile
// lies inside one expert's 128-aligned segment); weight modes tile each
// expert's output and reduce over its rows.
#include <math.h>

#include "device_common.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

constexpr int kGM = 64, kGN = 64, kGK = 16;

__device__ __forceinline__ int expert_of_row(const int32_t* offsets, int E, int row) {
  int lo = 0, hi = E - 1;  // largest e with offsets[e] <= row
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (offsets[mid] <= row) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <int MODE>
__global__ void __launch_bounds__(256) bwd_f32_kernel(BwdF32Args a) {
  pdl_wait();
  constexpr bool WG = MODE == BW_WG2 || MODE == BW_WG13;
  __shared__ float As[kGK][kGM + 4];
  __shared__ float Bs[kGK][kGN + 4];
  __shared__ float B3s[kGK][kGN + 4];  // SAVE with SwiGLU: the W3 tile beside W1
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  const int n0 = blockIdx.x * kGN;
  const bool swg = MODE == BW_SAVE && a.swiglu;

  // ---- the tile: A and B sources, the reduction length, the output rows
  const float* A;          // row modes: this tile's first A row; weight modes: A(m, k) rows
  const float* B;
  const float* B3 = nullptr;
  int K, rows_valid = kGM, m0 = 0, expert = 0;
  bool shared = false;
  long long out_row0 = 0;
  if (!WG) {
    const long long mrow = (long long)blockIdx.y * kGM;
    K = a.K;
    if (mrow < a.rows_routed) {
      if (mrow >= a.offsets[a.E]) return;
      expert = expert_of_row(a.offsets, a.E, (int)mrow);
      A = a.A + mrow * a.lda;
      out_row0 = mrow;
    } else {
      const long long q = mrow - a.rows_routed;
      const int s = (int)(q / a.n_pad);
      const long long local = q % a.n_pad;
      A = a.A_sh + (a.a_sh_base + s * a.a_sh_stride + local) * a.lda;
      out_row0 = a.shared_base + (long long)s * a.n_pad + local;
      rows_valid = (int)min((long long)kGM, (long long)a.n - local);
      expert = s;
      shared = true;
    }
    const size_t eoff = (size_t)expert * a.b_expert_stride;
    B = (shared ? a.sB : a.B) + eoff;
    const float* b3 = shared ? a.sB3 : a.B3;
    if ((swg || MODE == BW_DX) && b3) B3 = b3 + eoff;
  } else {
    m0 = blockIdx.y * kGM;
    const int q = blockIdx.z;
    shared = q >= a.E;
    expert = shared ? q - a.E : q;
    long long ar, br;
    if (!shared) {
      const int seg = a.offsets[q + 1] - a.offsets[q];
      K = max(0, min(a.counts[q], seg));
      ar = a.offsets[q];
      br = a.offsets[q];
    } else {
      K = a.n;
      ar = a.wa_sh_base + (long long)expert * a.wa_sh_stride;
      br = a.wb_sh_base + (long long)expert * a.wb_sh_stride;
    }
    A = (shared ? a.WA_sh : a.WA) + ar * a.ld_wa;
    B = (shared ? a.WB_sh : a.WB) + br * a.ld_wb;
  }

  float acc[4][4] = {}, acc3[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += kGK) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int q = tid + i * 256;  // 0..1023 over a 64 x 16 tile
      const int r = q / kGK, kk = q % kGK;
      const int k = k0 + kk;
      float av = 0.0f, bv = 0.0f, b3v = 0.0f;
      if (k < K) {
        if (!WG) {
          if (r < rows_valid) av = A[(size_t)r * a.lda + k];
          const int c = n0 + r;
          if (c < a.N) {
            if (MODE == BW_SAVE) {
              bv = B[(size_t)c * a.K + k];
              if (swg) b3v = B3[(size_t)c * a.K + k];
            } else if (MODE == BW_DX && k >= a.k_split) {
              bv = B3[(size_t)(k - a.k_split) * a.N + c];
            } else {
              bv = B[(size_t)k * a.N + c];
            }
          }
        } else {
          if (m0 + r < a.M) av = A[(size_t)k * a.ld_wa + m0 + r];
          if (n0 + r < a.N) bv = B[(size_t)k * a.ld_wb + n0 + r];
        }
      }
      As[kk][r] = av;
      Bs[kk][r] = bv;
      if (swg) B3s[kk][r] = b3v;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kGK; ++kk) {
      float av[4], bv[4], b3v[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        bv[j] = Bs[kk][tx * 4 + j];
        if (swg) b3v[j] = B3s[kk][tx * 4 + j];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
          if (swg) acc3[i][j] = fmaf(av[i], b3v[j], acc3[i][j]);
        }
    }
    __syncthreads();
  }

  // ---- epilogue
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = n0 + tx * 4 + j;
      if (c >= a.N) continue;
      const float v = acc[i][j];
      if (WG) {
        const int m = m0 + ty * 4 + i;
        if (m >= a.M) continue;
        const bool hi = m >= a.m_split;
        float* dst = shared ? (hi ? a.sw_out1 : a.sw_out0) : (hi ? a.w_out1 : a.w_out0);
        dst[(size_t)expert * a.w_expert_stride + (size_t)(hi ? m - a.m_split : m) * a.N + c] = v;
        continue;
      }
      const long long row = out_row0 + ty * 4 + i;
      if (MODE == BW_SAVE) {
        // U (and V), and H as the fp32 forward computes it
        a.out0[row * a.ld_out + c] = v;
        float h;
        if (swg) {
          const float g = acc3[i][j];
          a.out1[row * a.ld_out + c] = g;
          h = v / (1.0f + expf(-v)) * g;
        } else if (a.act == MOE_ACT_RELU) {
          h = fmaxf(v, 0.0f);
        } else {
          h = 0.5f * v * (1.0f + erff(v * 0.70710678118654752f));
        }
        a.out2[row * a.ld_out + c] = h;
      } else if (MODE == BW_DACT) {
        // v = dH; the stored U (and V) of the same element
        const float u = a.in0[row * a.ld_in + c];
        if (a.swiglu) {
          const float vv = a.in1[row * a.ld_in + c];
          const float sg = 1.0f / (1.0f + expf(-u));
          a.out0[row * a.ld_out + c] = v * vv * sg * (1.0f + u * (1.0f - sg));
          a.out0[row * a.ld_out + a.N + c] = v * u * sg;
        } else if (a.act == MOE_ACT_RELU) {
          a.out0[row * a.ld_out + c] = u > 0.0f ? v : 0.0f;
        } else {
          const float cdf = 0.5f * (1.0f + erff(u * 0.70710678118654752f));
          const float pdf = 0.3989422804014327f * expf(-0.5f * u * u);
          a.out0[row * a.ld_out + c] = v * (cdf + u * pdf);
        }
      } else {  // BW_DX
        a.out0[row * a.ld_out + c] = v;
      }
    }
  }
}

}  // namespace

cudaError_t run_bwd_f32(int mode, const BwdF32Args& a, cudaStream_t s) {
  const bool wg = mode == BW_WG2 || mode == BW_WG13;
  const long long total_rows = a.rows_routed + (long long)a.n_shared * a.n_pad;
  dim3 grid(ceil_div(a.N, kGN), wg ? ceil_div(a.M, kGM) : (unsigned)(total_rows / kGM),
            wg ? a.E + a.n_shared : 1);
  switch (mode) {
    case BW_SAVE: return launch_pdl(bwd_f32_kernel<BW_SAVE>, grid, 256, 0, s, a);
    case BW_DACT: return launch_pdl(bwd_f32_kernel<BW_DACT>, grid, 256, 0, s, a);
    case BW_DX: return launch_pdl(bwd_f32_kernel<BW_DX>, grid, 256, 0, s, a);
    case BW_WG2: return launch_pdl(bwd_f32_kernel<BW_WG2>, grid, 256, 0, s, a);
    default: return launch_pdl(bwd_f32_kernel<BW_WG13>, grid, 256, 0, s, a);
  }
}

}  // namespace moe
