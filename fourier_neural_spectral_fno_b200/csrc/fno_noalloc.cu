// fno_spectral_conv_fwd_noalloc: the spectral-convolution forward with its
// scratch in a fixed device array compiled into the library, for callers that
// cannot allocate device memory themselves (see include/fno.h).
//
// The array below exists once per GPU that loads the library and stays
// allocated until the process exits.  In host code its name is only a
// host-side stand-in, never a device address: the device address is looked
// up here with cudaGetSymbolAddress, once per device (with that device
// current), and handed to the ordinary entry point as its workspace.
#include <stdio.h>

#include <mutex>

#include "fno.h"
#include "fno_kernels.cuh"

namespace {

constexpr size_t kScratchBytes = FNO_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_fno_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device (set up on the
// first call per device); nullptr on failure, with the error message set.
void *scratch_for_current_device() {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    fno::set_last_error("no usable current CUDA device (%s)", cudaGetErrorString(e));
    cudaGetLastError();
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_addr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_fno_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      fno::set_last_error("cudaGetSymbolAddress of the built-in scratch failed: %s",
                          cudaGetErrorString(e));
      cudaGetLastError();
      return nullptr;
    }
    g_scratch_addr[dev] = p;
  }
  return g_scratch_addr[dev];
}

}  // namespace

extern "C" {

int fno_spectral_conv_fwd_noalloc(const fno_block_desc *desc, const void *x, const void *R,
                                  void *y, float *xhat_save, fno_stream_t stream) {
  const size_t need = fno_workspace_size(desc, FNO_OP_SPECTRAL_FWD);
  if (need == 0) return FNO_ERR_INVALID_ARG;   // message left by fno_workspace_size
  if (need > kScratchBytes) {
    fno::set_last_error(
        "this problem needs %zu bytes of scratch but the built-in scratch holds %zu bytes; "
        "use fno_spectral_conv_fwd with a caller workspace",
        need, kScratchBytes);
    return FNO_ERR_WORKSPACE;
  }
  void *ws = scratch_for_current_device();
  if (!ws) return FNO_ERR_CUDA;
  return fno_spectral_conv_fwd(desc, x, R, y, xhat_save, ws, kScratchBytes, stream);
}

}  // extern "C"
