// stem_noalloc.cu — stem_prefill for callers that cannot allocate device memory.
//
// stem_prefill needs a caller-provided workspace (status word, value bonus,
// block scores and the CSR lists).  Some callers cannot provide one: code that
// runs where cudaMalloc is not allowed or not wanted (inside a host callback
// or a custom allocator hook, a plugin whose host owns all device memory, or a
// deployment whose memory pool is fixed up front).  For them this file keeps a
// built-in workspace in a file-scope device array and runs the same pipeline
// on it.  No device memory is allocated or freed here.
//
// Limits and rules, stated for the user:
//  * The built-in workspace holds kStaticWorkspaceBytes (32 MiB).  A problem
//    whose stem_plan().ws_prefill_bytes exceeds it is rejected with
//    STEM_ERR_WORKSPACE_TOO_SMALL before anything is enqueued (with 32 query
//    heads the largest single sequence that fits is about 61K tokens).
//  * Every GPU that loads the library holds the 32 MiB until the process exits.
//  * All calls on one device share the one array and it keeps the last call's
//    contents: calls that can overlap on the GPU (different streams without
//    ordering between them) race and corrupt each other.  Serialise them.
//  * The first call on each device looks up the array's device address (with
//    that device current); make that first call before any stream capture.
//    The address is cached per device for the life of the process; it does
//    not survive cudaDeviceReset.
//  * `stream` must belong to the current device (STEM_ERR_INVALID_ARG
//    otherwise), so the kernels never get another device's array.
//  * Device-side errors (a bounded wait that ran out, a malformed list entry)
//    are recorded in the built-in workspace's status word: read it with
//    stem_noalloc_read_device_status after the call.
#include <cuda_runtime.h>

#include <mutex>

#include "stem.h"

namespace {

constexpr size_t kStaticWorkspaceBytes = size_t(32) << 20;
constexpr int kMaxDevices = 64;

// The built-in workspace.  In host code `g_static_ws` names a host-side
// stand-in, not device memory: only the address returned by
// cudaGetSymbolAddress may be passed to kernels.
static __device__ __align__(256) unsigned char g_static_ws[kStaticWorkspaceBytes];

std::mutex g_mu;
void* g_ws_addr[kMaxDevices] = {};

// Device address of the built-in workspace on the current device (looked up
// once per device).  Returns nullptr on failure.
void* static_ws_address() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_ws_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_ws) != cudaSuccess || p == nullptr) return nullptr;
    g_ws_addr[dev] = p;
  }
  return g_ws_addr[dev];
}

// STEM_OK when `stream` runs on the current device (the legacy and per-thread
// default streams always do).
stem_status_t check_stream_device(cudaStream_t stream) {
  int cur = -1, sdev = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) return STEM_ERR_CUDA;
  if (stream == nullptr || stream == cudaStreamLegacy || stream == cudaStreamPerThread) return STEM_OK;
  if (cudaStreamGetDevice(stream, &sdev) != cudaSuccess) return STEM_ERR_INVALID_ARG;
  return sdev == cur ? STEM_OK : STEM_ERR_INVALID_ARG;
}

}  // namespace

extern "C" stem_status_t stem_noalloc_read_device_status(stem_stream_t stream, stem_status_t* out) {
  if (!out) return STEM_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  stem_status_t st = check_stream_device(s);
  if (st != STEM_OK) return st;
  void* ws = static_ws_address();
  if (ws == nullptr) return STEM_ERR_CUDA;
  return stem_read_device_status(ws, stream, out);
}

extern "C" stem_status_t stem_prefill_noalloc(const stem_qkv_t* qkv, const stem_params_t* params, void* out,
                                              float* lse, int32_t* row_ptr_out, int32_t* col_idx_out,
                                              stem_stream_t stream) {
  stem_plan_t pl;
  stem_status_t st = stem_plan(qkv, params, &pl);
  if (st != STEM_OK) return st;
  if (pl.ws_prefill_bytes > kStaticWorkspaceBytes) return STEM_ERR_WORKSPACE_TOO_SMALL;
  if ((st = check_stream_device(reinterpret_cast<cudaStream_t>(stream))) != STEM_OK) return st;
  void* ws = static_ws_address();
  if (ws == nullptr) return STEM_ERR_CUDA;
  return stem_prefill(qkv, params, out, lse, row_ptr_out, col_idx_out, ws, kStaticWorkspaceBytes, stream);
}
