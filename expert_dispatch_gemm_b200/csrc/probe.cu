// Throughput probe for the router's roof: the router contraction runs on
// FP32 FFMA, whose peak is not among the measured HBM / tensor figures, so
// the benchmark measures it on the device it runs on. Every thread runs 16
// independent fmaf chains (enough to cover the FMA latency at any
// occupancy), as single FFMAs or (packed = 1) as 8 packed fp32x2 FMAs; the
// launch does blocks * threads * iters * 16 FMAs either way.
// Built into its own library: it is measurement, not part of the layer.
#include <cuda_runtime.h>

#define PROBE_API extern "C" __attribute__((visibility("default")))

namespace {

__global__ void __launch_bounds__(256) ffma_probe_kernel(float* out, int iters, float a, float b) {
  float x[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) x[i] = (float)threadIdx.x * 1e-3f + (float)i;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < 16; ++i) x[i] = fmaf(x[i], a, b);
  }
  float s = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) s += x[i];
  if (s == -1.0f) out[blockIdx.x] = s;  // never true; keeps the chains live
}

__global__ void __launch_bounds__(256) ffma2_probe_kernel(float* out, int iters, float a,
                                                          float b) {
  float2 x[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    x[i] = make_float2((float)threadIdx.x * 1e-3f + (float)(2 * i),
                       (float)threadIdx.x * 1e-3f + (float)(2 * i + 1));
  const float2 a2 = make_float2(a, a), b2 = make_float2(b, b);
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] = __ffma2_rn(x[i], a2, b2);
  }
  float s = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) s += x[i].x + x[i].y;
  if (s == -1.0f) out[blockIdx.x] = s;  // never true; keeps the chains live
}

}  // namespace

// Launches blocks x 256 threads, iters rounds of 16 FMAs per thread, on
// `stream`: single FFMAs (packed = 0) or packed fp32x2 FMAs (packed = 1).
// `out` needs `blocks` floats (written only in a case that does not occur).
// Returns the cudaError_t of the launch.
PROBE_API int moe_probe_ffma(int blocks, int iters, float* out, void* stream) {
  if (blocks < 1 || iters < 1 || !out) return (int)cudaErrorInvalidValue;
  ffma_probe_kernel<<<blocks, 256, 0, (cudaStream_t)stream>>>(out, iters, 0.999999f, 1e-6f);
  return (int)cudaGetLastError();
}

PROBE_API int moe_probe_ffma2(int blocks, int iters, float* out, void* stream) {
  if (blocks < 1 || iters < 1 || !out) return (int)cudaErrorInvalidValue;
  ffma2_probe_kernel<<<blocks, 256, 0, (cudaStream_t)stream>>>(out, iters, 0.999999f, 1e-6f);
  return (int)cudaGetLastError();
}
