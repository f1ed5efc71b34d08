// Device helpers shared by the libmoe kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

namespace moe {

// Device error codes written to the workspace error word.
enum : int {
  kErrNone = 0,
  kErrGemmTimeout = 0x100,   // | role << 4 | which barrier
  kErrBadIndex = 0x200,
};

// Programmatic dependent launch. Every kernel of the library is launched
// with programmatic stream serialisation (launch_pdl), so its launch is
// processed while the previous kernel in the stream drains, and it calls
// pdl_wait() before it touches anything that kernel wrote (the wait returns
// once the previous grid has completed and its writes are visible; every
// kernel waits, so the order is transitive). No kernel triggers its
// dependents early: CTAs of the next kernel parked on SMs beside this one's
// measured slower on B200 than letting them start as this one's CTAs exit.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

__device__ __forceinline__ void report_error(int* err, int code) {
  if (err) atomicCAS(err, 0, code);
}

// Index checks. Every build skips an index read from the routing outputs
// (row_token, tok_row, offsets, counts, idx) that lies outside its range
// instead of reading or writing through it. The checked build
// (-DMOE_DEBUG_CHECKS, libmoe_checked.so) also reports each such index as
// kErrBadIndex | site in the error word, where moe_read_error finds it; the
// default build compiles the report away.
#ifdef MOE_DEBUG_CHECKS
constexpr bool kDebugChecks = true;
#else
constexpr bool kDebugChecks = false;
#endif

enum : int {
  kSiteGatherTokRow = 0x01,
  kSiteGatherRowToken = 0x02,
  kSiteGatherOffsets = 0x03,
  kSiteCombineTokRow = 0x04,
  kSiteCombinePrepTokRow = 0x05,
  kSiteGemmOffsets = 0x10,
  kSiteGemmPairOffsets = 0x11,
  kSiteGemmGatherToken = 0x12,
  kSiteGemmScatterToken = 0x13,
  kSiteSwapOffsets = 0x20,
  kSiteScatterIdx = 0x30,
  kSiteEcFinishIdx = 0x31,
  kSiteBwdTokRow = 0x40,
  kSiteBwdOffsets = 0x41,
};

__device__ __forceinline__ void bad_index(int* err, int site) {
  if (kDebugChecks) report_error(err, kErrBadIndex | site);
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ float bf16_to_f32(uint16_t b) {
  return __uint_as_float(((uint32_t)b) << 16);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

}  // namespace moe
