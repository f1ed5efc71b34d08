// moe_route_noalloc: moe_route for callers that cannot allocate device memory.
//
// Some callers of this library cannot allocate device memory when they route
// a batch: a host application whose device memory budget is fixed when it
// starts, or a plugin running inside a framework that owns every device
// allocation. Such callers cannot hand moe_route a workspace. This entry
// point runs the same routing kernels with their scratch in a fixed,
// library-owned device array instead:
//   - the array is MOE_ROUTE_NOALLOC_SCRATCH_BYTES (4 MiB) of static device
//     memory, held on every GPU that loads the library until the process
//     exits;
//   - configs whose routing scratch is larger are rejected with
//     MOE_ERR_WORKSPACE before anything is enqueued;
//   - nothing here calls cudaMalloc, cudaFree or any allocating routine.
//
// Host code cannot use the array's name as a device address: it stands for a
// host-side shadow of the symbol. The first call on each device therefore
// looks up the array's device address with cudaGetSymbolAddress (with that
// device current); make that first call before any stream capture. Every call
// then zeroes the array's error word with a cudaMemsetAsync on the caller's
// stream before its kernels, so the word holds that call's routing errors
// only (a stale code from an earlier call never survives into a later one);
// moe_read_error(NULL, ...) reads and clears it. All calls share the one
// array and it keeps the last call's contents, so calls that overlap on the
// GPU (on different streams, or from different threads) race with each other.
#include <mutex>

#include "moe_internal.h"

namespace {

constexpr size_t kScratchBytes = MOE_ROUTE_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_route_scratch[kScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices];  // device address of g_route_scratch, per device

// Device address of the scratch array on the current device, looked up on the
// first call for that device.
moe_status scratch_on_current_device(void** addr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || p == nullptr)
      return MOE_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *addr = g_scratch_addr[dev];
  return MOE_OK;
}

}  // namespace

namespace moe {

// The scratch array's error word on the current device, read and cleared
// (synchronous copies; the caller has synchronised its stream). 0 when this
// device has made no moe_route_noalloc call.
int take_noalloc_error() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  void* p = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    p = g_scratch_addr[dev];
  }
  if (p == nullptr) return 0;
  int code = 0;
  if (cudaMemcpy(&code, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return 0;
  if (code != 0) {
    const int zero = 0;
    cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice);
  }
  return code;
}

}  // namespace moe

extern "C" MOE_API moe_status moe_route_noalloc(const moe_config* cfg, const void* X,
                                                const float* Wg, const float* logit_bias,
                                                const float* sel_bias, moe_route_out* out,
                                                moe_stream_t stream) {
  size_t need = 0;
  moe_status st = moe_workspace_size(cfg, &need, nullptr);
  if (st != MOE_OK) return st;
  if (need > kScratchBytes) return MOE_ERR_WORKSPACE;
  // every check moe_route makes comes first: on an error nothing is enqueued
  if ((st = moe::route_call_check(cfg, X, Wg, out)) != MOE_OK) return st;
  void* scratch = nullptr;
  if ((st = scratch_on_current_device(&scratch)) != MOE_OK) return st;
  // re-arm the error word on the caller's stream, ordered before the kernels
  if (cudaMemsetAsync(scratch, 0, MOE_WS_ERROR_BYTES, (cudaStream_t)stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  return moe_route(cfg, X, Wg, logit_bias, sel_bias, out, scratch, kScratchBytes, stream);
}
