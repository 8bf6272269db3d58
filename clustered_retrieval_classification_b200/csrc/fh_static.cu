// fh_static.cu — the batch-1 greedy head for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc or hand the library a workspace: code embedded in a host
// framework that owns the whole device heap and allows no raw allocations, or a latency-critical
// decode loop where cudaMalloc's implicit device-wide synchronisation is not acceptable and no spare
// buffer of the right size exists.  For them this file keeps the scratch of one call in a file-scope
// device array (FH_STATIC_SCRATCH_BYTES, declared in include/flashhead.h), which every GPU that loads
// the library holds until the process exits.
//
// Host code cannot use the array's name as a device address (in host code it is only a host-side
// stand-in), so the address is looked up with cudaGetSymbolAddress, once per device with that device
// current, and passed to the kernels as an ordinary workspace pointer.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "../../include/flashhead.h"

static __device__ __align__(256) unsigned char g_static_scratch[FH_STATIC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 256;
std::mutex g_mutex;
void* g_scratch_addr[kMaxDevices] = {};

}  // namespace

// Defined in fh_api.cu: records the message returned by fh_last_error().
fh_status fh_internal_set_error(fh_status st, const char* msg);

extern "C" fh_status fh_head_greedy_static(const fh_index* idx, const void* H, int p,
                                           int32_t* out_tok, fh_stream stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fh_internal_set_error(FH_ERR_CUDA, cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fh_internal_set_error(FH_ERR_UNSUPPORTED, "device ordinal too large");
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_addr[dev]) {
      void* addr = nullptr;
      e = cudaGetSymbolAddress(&addr, g_static_scratch);
      if (e != cudaSuccess || !addr) {
        char msg[160];
        snprintf(msg, sizeof msg, "cudaGetSymbolAddress of the static scratch failed: %s",
                 cudaGetErrorString(e));
        return fh_internal_set_error(FH_ERR_CUDA, msg);
      }
      g_scratch_addr[dev] = addr;
    }
    scratch = g_scratch_addr[dev];
  }
  const size_t need = fh_workspace_bytes(idx, FH_OP_GREEDY, 1, p, 0, 0);
  if (need == 0) return fh_internal_set_error(FH_ERR_ARG, "invalid index handle or p");
  if (need > (size_t)FH_STATIC_SCRATCH_BYTES) {
    char msg[160];
    snprintf(msg, sizeof msg, "this index needs %zu bytes of scratch at p=%d; the static scratch "
             "holds %d bytes", need, p, (int)FH_STATIC_SCRATCH_BYTES);
    return fh_internal_set_error(FH_ERR_WORKSPACE, msg);
  }
  // Every call shares the array and it keeps the previous call's contents: clear the part this call
  // uses (its counters and histogram must start at zero).
  e = cudaMemsetAsync(scratch, 0, need, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fh_internal_set_error(FH_ERR_CUDA, cudaGetErrorString(e));
  return fh_head_greedy(idx, H, 1, p, out_tok, scratch, (size_t)FH_STATIC_SCRATCH_BYTES, stream,
                        nullptr);
}
