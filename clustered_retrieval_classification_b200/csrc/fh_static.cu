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
//
// The array is used exactly like a workspace: it starts zeroed (a static device array is
// zero-initialised when the module loads), every call returns the words that must start at zero
// (histogram, arg-max, tickets) to zero before it ends and tags everything else with its call
// generation, and a device-side error stays in the array's status word until fh_static_status reads
// it and zeroes the control block again.  A call writes -1 to out_tok before it launches, so a call
// that fails on the device leaves -1 there instead of a plausible token.
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

// Defined in fh_api.cu: records the message returned by fh_last_error(), and the host-side argument
// checks of a head call.
fh_status fh_internal_set_error(fh_status st, const char* msg);
fh_status fh_internal_check_head(const fh_index* idx, const void* H, int B, int p, const int32_t* out_tok);

// The array's device address on the current device (looked up on first use there).
static fh_status static_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fh_internal_set_error(FH_ERR_CUDA, cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fh_internal_set_error(FH_ERR_UNSUPPORTED, "device ordinal too large");
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
  *out = g_scratch_addr[dev];
  return FH_OK;
}

extern "C" fh_status fh_head_greedy_static(const fh_index* idx, const void* H, int p,
                                           int32_t* out_tok, fh_stream stream) {
  // argument errors are found before anything is queued on the stream
  fh_status r = fh_internal_check_head(idx, H, 1, p, out_tok);
  if (r != FH_OK) return r;
  const size_t need = fh_workspace_bytes(idx, FH_OP_GREEDY, 1, p, 0, 0);
  if (need == 0) return fh_internal_set_error(FH_ERR_ARG, "invalid index handle or p");
  if (need > (size_t)FH_STATIC_SCRATCH_BYTES) {
    char msg[160];
    snprintf(msg, sizeof msg, "this index needs %zu bytes of scratch at p=%d; the static scratch "
             "holds %d bytes", need, p, (int)FH_STATIC_SCRATCH_BYTES);
    return fh_internal_set_error(FH_ERR_WORKSPACE, msg);
  }
  void* scratch = nullptr;
  if ((r = static_scratch(&scratch)) != FH_OK) return r;
  // A call that fails on the device (a bounded wait that gave up) never writes its token: it leaves
  // this -1, and the error waits in the status word for fh_static_status.
  cudaError_t e = cudaMemsetAsync(out_tok, 0xFF, sizeof(int32_t), static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fh_internal_set_error(FH_ERR_CUDA, cudaGetErrorString(e));
  return fh_head_greedy(idx, H, 1, p, out_tok, scratch, (size_t)FH_STATIC_SCRATCH_BYTES, stream,
                        nullptr);
}

extern "C" fh_status fh_static_status(fh_stream stream) {
  void* scratch = nullptr;
  const fh_status r = static_scratch(&scratch);
  if (r != FH_OK) return r;
  return fh_ws_status(scratch, stream);
}

extern "C" fh_status fh_static_scratch(void** dev_ptr, size_t* bytes) {
  if (!dev_ptr || !bytes) return fh_internal_set_error(FH_ERR_ARG, "dev_ptr or bytes is NULL");
  const fh_status r = static_scratch(dev_ptr);
  if (r == FH_OK) *bytes = (size_t)FH_STATIC_SCRATCH_BYTES;
  return r;
}
