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
// device current) and zeroes its error word with a synchronous cudaMemset;
// make that first call before any stream capture. All calls share the one
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

// Device address of the scratch array on the current device; looked up (and
// its error word zeroed) on the first call for that device.
moe_status scratch_on_current_device(void** addr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || p == nullptr)
      return MOE_ERR_CUDA;
    if (cudaMemset(p, 0, MOE_WS_ERROR_BYTES) != cudaSuccess) return MOE_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *addr = g_scratch_addr[dev];
  return MOE_OK;
}

}  // namespace

extern "C" MOE_API moe_status moe_route_noalloc(const moe_config* cfg, const void* X,
                                                const float* Wg, const float* logit_bias,
                                                const float* sel_bias, moe_route_out* out,
                                                moe_stream_t stream) {
  size_t need = 0;
  moe_status st = moe_workspace_size(cfg, &need, nullptr);
  if (st != MOE_OK) return st;
  if (need > kScratchBytes) return MOE_ERR_WORKSPACE;
  void* scratch = nullptr;
  if ((st = scratch_on_current_device(&scratch)) != MOE_OK) return st;
  return moe_route(cfg, X, Wg, logit_bias, sel_bias, out, scratch, kScratchBytes, stream);
}
