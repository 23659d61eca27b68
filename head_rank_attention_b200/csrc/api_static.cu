// api_static.cu -- mlra_decode_static: the decode without a caller-provided workspace.
//
// Some callers cannot allocate device memory when they run the decode: code that runs
// inside another framework's memory pool or a serving runtime that forbids allocation on
// its hot path (no cudaMalloc, no allocator round trip), and plain C callers that have
// no allocator of their own.  For them this entry point takes its scratch (absorbed
// queries, split-KV partial states, device status word) from one file-scope device array
// of fixed size instead of the `workspace` pointer, and allocates nothing itself.
//
// Rules that follow from sharing one array:
//   * Every GPU that loads this library holds the array (kStaticScratchBytes) until the
//     process exits.
//   * All calls on a device share it and it keeps the previous call's contents.  What
//     must start at zero -- the status word -- is cleared at the start of every call (a
//     memset on the stream, which allocates nothing); everything else is written before
//     it is read.
//   * Calls that overlap on the GPU (concurrent streams, or host threads launching on
//     different streams) race on the array and give wrong results; serialize them.
//   * The first call on a device looks the array's device address up
//     (cudaGetSymbolAddress) with that device current; make that first call before any
//     stream capture.  The address is kept for the life of the process, so the library
//     must not be used across a device reset (cudaDeviceReset or a primary-context
//     teardown), after which the array is mapped anew.
//   * Expired device waits are recorded in the array's status word, which
//     hra_check_device_status cannot reach; launch and argument errors are returned.
#include <cuda_runtime.h>

#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "hra.h"

namespace hra {
void set_last_error(const char* msg);                           // api.cu
hra_status workspace_bytes(const hra_decode_params* p, size_t* bytes);  // api.cu
}  // namespace hra

namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;  // 32 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

hra_status static_fail(hra_status st, const std::string& msg) {
  hra::set_last_error(msg.c_str());
  return st;
}

}  // namespace

extern "C" HRA_API hra_status mlra_decode_static(const hra_decode_params* p, void* stream) {
  if (p == nullptr) return static_fail(HRA_ERR_INVALID_ARG, "params is NULL");
  // Size check first.  It validates the parameters and, unless num_splits > 0, queries the
  // current device's SM count (the default split count depends on it).
  size_t need = 0;
  const hra_status st = hra::workspace_bytes(p, &need);
  if (st != HRA_OK) return st;  // the reason is recorded for hra_last_error
  if (need > kStaticScratchBytes) {
    char buf[256];
    snprintf(buf, sizeof(buf),
             "mlra_decode_static: this call needs %zu bytes of scratch, more than the %zu-byte static array; "
             "use mlra_decode with a caller workspace",
             need, kStaticScratchBytes);
    return static_fail(HRA_ERR_WORKSPACE, buf);
  }
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return static_fail(HRA_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return static_fail(HRA_ERR_UNSUPPORTED, "device ordinal out of range");
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
      // Host code only holds a stand-in for the array; its device address for the
      // current device comes from the runtime.
      void* ptr = nullptr;
      e = cudaGetSymbolAddress(&ptr, g_static_scratch);
      if (e != cudaSuccess || ptr == nullptr)
        return static_fail(HRA_ERR_CUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
      g_scratch_ptr[dev] = ptr;
    }
    scratch = g_scratch_ptr[dev];
  }
  hra_decode_params q = *p;
  q.workspace = scratch;
  q.workspace_bytes = kStaticScratchBytes;
  return mlra_decode(&q, stream);  // records its own errors
}
