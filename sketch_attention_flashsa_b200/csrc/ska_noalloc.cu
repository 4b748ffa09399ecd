// sa_forward_noalloc: the SA forward for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc or hand over a workspace: code that runs inside a memory
// pool it does not own, plugins that receive only input and output pointers from a host
// framework, and service paths that must not allocate after start-up. For them this entry point
// runs the same kernels as sa_forward, with the scratch memory (tile schedule, per-cluster
// partial sketches, status word) in a file-scope device array of fixed size instead of a
// caller-provided workspace.
//
// Costs and limits:
// * Every GPU that loads this library holds kNoAllocScratchBytes of device memory for the
//   array until the process exits.
// * Problems whose scratch need exceeds the array are rejected with
//   SKA_ERR_WORKSPACE_TOO_SMALL before anything is launched.
// * All calls on one device share the array and it keeps the last call's contents; the kernels
//   rewrite every scratch word they read (the schedule kernel clears the status word), so
//   nothing carries over between calls. Calls that overlap on the GPU (on different streams,
//   or from several host threads) race on the array: serialise them.
// * The first call on each device looks up the array's device address with
//   cudaGetSymbolAddress; make that first call before any stream capture.
// * Device-side errors (a bounded wait that ran out, an fp16 overflow) land in the array's
//   status word; sa_forward_noalloc_read_status reads and clears it.
#include <mutex>

#include "ska_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(40) << 20;  // 40 MiB per device

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;

// Device address of g_noalloc_scratch for the current device (looked up once per device).
void* scratch_address(cudaError_t* err) {
  static void* addr[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= kMaxDevices) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    *err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (*err != cudaSuccess) return nullptr;
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace

extern "C" size_t sa_forward_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

extern "C" ska_status sa_forward_noalloc(const ska_sa_desc* desc, const void* q, const void* k, const void* v,
                                         const int32_t* cu_seqlens, const int32_t* seqused, float* sketch,
                                         float* lse, float* mass, void* stream) {
  if (!desc) return SKA_ERR_INVALID_VALUE;
  const size_t need = sa_forward_workspace_size(desc);
  if (need > kNoAllocScratchBytes) return SKA_ERR_WORKSPACE_TOO_SMALL;
  cudaError_t err = cudaSuccess;
  void* scratch = scratch_address(&err);
  if (!scratch || err != cudaSuccess) return SKA_ERR_CUDA;
  return sa_forward(desc, q, k, v, cu_seqlens, seqused, sketch, lse, mass, scratch, kNoAllocScratchBytes, stream);
}

extern "C" ska_status sa_forward_noalloc_read_status(void* stream) {
  cudaError_t err = cudaSuccess;
  void* scratch = scratch_address(&err);
  if (!scratch || err != cudaSuccess) return SKA_ERR_CUDA;
  return ska_read_device_status(scratch, stream);
}
