// specopd_e2e_tv_noalloc: the E2E-TV entry point for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc: code that runs inside another
// framework's memory pool (which owns the device memory and forbids
// allocations outside it), or code on a path where cudaMalloc's implicit
// device-wide synchronisation is not allowed.  This entry point needs no
// workspace argument: its scratch is a fixed array in the library's own
// device image (below), which every GPU that loads the library holds until
// the process exits.  The caller still passes every input and output.
//
// The array is shared by every call on a device and keeps the last call's
// contents; specopd_e2e_tv clears the counters it needs at the start of each
// call.  Calls that overlap on the GPU (other streams, other host threads)
// race on the array and must be serialised by the caller.
#include <mutex>

#include "common.cuh"

namespace specopd {

constexpr size_t kTVStaticScratchBytes = SPECOPD_E2E_TV_STATIC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_tv_static_scratch[kTVStaticScratchBytes];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_tv_static_mu;
void* g_tv_static_ptr[kMaxDevices] = {};

// Device address of g_tv_static_scratch on the current device.  In host code
// the array's name is only a host-side stand-in, so the address is resolved
// with cudaGetSymbolAddress, once per device, with that device current.
cudaError_t tv_static_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_tv_static_mu);
  if (!g_tv_static_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_tv_static_scratch);
    if (e != cudaSuccess) return e;
    if (!p) return cudaErrorInvalidSymbol;
    g_tv_static_ptr[dev] = p;
  }
  *out = g_tv_static_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace specopd

extern "C" specopd_status specopd_e2e_tv_noalloc(const specopd_tv_desc* desc,
                                                  const void* z_target,
                                                  const int32_t* target_row,
                                                  const void* z_draft, float* a, float* prefix,
                                                  float* loss, double* numer, void* grad_draft,
                                                  void* stream) {
  if (!desc) return SPECOPD_ERR_INVALID_ARG;
  if (specopd_e2e_tv_workspace_size(desc) == 0) return SPECOPD_ERR_INVALID_ARG;  // invalid descriptor
  void* scratch = nullptr;
  const cudaError_t e = specopd::tv_static_scratch(&scratch);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return SPECOPD_ERR_CUDA;
  }
  // The size limit applies to the scratch of the schedule this call runs:
  // the whole-row schedule needs a few bytes per position, the slice
  // fallback a few hundred.  Beyond the array: SPECOPD_ERR_WORKSPACE, before
  // anything is launched.
  return e2e_tv_checked(desc, z_target, target_row, z_draft, a, prefix, loss, numer, grad_draft,
                        scratch, specopd::kTVStaticScratchBytes, stream, true);
}
