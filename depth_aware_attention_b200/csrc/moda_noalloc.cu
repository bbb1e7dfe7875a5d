// moda_noalloc.cu -- moda_backward_noalloc: the MoDA backward for callers that cannot
// allocate device memory.
//
// moda_backward needs a caller-provided workspace (an fp32 dq accumulator and the fp32
// row terms D).  Some callers have no way to provide one: their device memory is owned
// by another allocator or by a fixed memory plan that hands out only the tensors it
// planned, or they reach this library through a plain C binding with no device
// allocation API at all.  This entry point gives them the same backward with the
// workspace taken from a statically sized array that the library itself declares, so
// neither the caller nor the library allocates anything.
//
// The array is a file-scope __device__ variable: every GPU that loads the library holds
// it, kNoAllocScratchBytes in size, until the process exits.  In host code its name is
// only a host-side stand-in for the symbol, not a device address, so the host looks up
// the device address with cudaGetSymbolAddress, once per device, with that device
// current, and passes that address on as the workspace.
#include <cuda_runtime.h>
#include <stdio.h>

#include <mutex>

#include "../../include/moda.h"
#include "moda_internal.h"

namespace moda {

// Maximum workspace this entry point can serve: 64 MiB.
constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

// Device address of g_noalloc_scratch on the calling thread's current device, looked up
// on the first call for that device and cached for the life of the process.  The cache
// is not invalidated: a cudaDeviceReset() (which unloads the module, so the array may come
// back elsewhere) between calls is not supported.  NULL (with *err set) on failure.
void* noalloc_scratch(int dev, cudaError_t* err) {
  static std::mutex mu;
  static void* addr[64] = {nullptr};
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) {
      *err = e;
      return nullptr;
    }
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace
}  // namespace moda

extern "C" moda_status_t moda_backward_noalloc(
    const void* q, const void* k, const void* v, const void* kd, const void* vd,
    const void* out, const float* lse, const void* dout, void* dq, void* dk, void* dv,
    void* dkd, void* dvd, int B, int Hq, int Hkv, int T, int L, int d, float scale,
    int causal, moda_stream_t stream) {
  // Every argument check that needs neither the workspace nor the device runs first, so
  // a bad call is refused before anything touches the GPU.
  moda_status_t s = backward_entry(q, k, v, kd, vd, out, lse, dout, dq, dk, dv, dkd, dvd,
                                   nullptr, 0, B, Hq, Hkv, T, L, d, scale, causal,
                                   moda::kStagesAll, 0, stream, /*validate_only=*/true);
  if (s != MODA_OK) return s;
  const size_t need = moda_backward_workspace_size(B, Hq, Hkv, T, L, d);
  if (need > moda::kNoAllocScratchBytes) {
    snprintf(g_msg, sizeof(g_msg),
             "moda_backward_noalloc needs %zu bytes of workspace for these sizes but its static "
             "scratch holds %zu; call moda_backward with a caller workspace instead",
             need, moda::kNoAllocScratchBytes);
    return MODA_ERR_UNSUPPORTED;
  }
  s = injected_at_launch();
  if (s != MODA_OK) return s;
  s = check_device();
  if (s != MODA_OK) return s;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    snprintf(g_msg, sizeof(g_msg), "moda_backward_noalloc: no usable current CUDA device");
    return MODA_ERR_CUDA;
  }
  cudaError_t e = cudaSuccess;
  void* scratch = moda::noalloc_scratch(dev, &e);
  if (scratch == nullptr) {
    snprintf(g_msg, sizeof(g_msg), "moda_backward_noalloc: cudaGetSymbolAddress failed: %s",
             cudaGetErrorString(e));
    return MODA_ERR_CUDA;
  }
  return moda_backward(q, k, v, kd, vd, out, lse, dout, dq, dk, dv, dkd, dvd, scratch,
                       moda::kNoAllocScratchBytes, B, Hq, Hkv, T, L, d, scale, causal, stream);
}
