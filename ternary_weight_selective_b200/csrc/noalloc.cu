// bitlinear_forward_noalloc: the standalone BitLinear for callers that may
// not allocate device memory, running on a fixed scratch array that lives in
// the library itself.  The contract is in include/bitssm.h.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "bitssm.h"

namespace bitssm {
void set_last_error_message(const char* msg);
}

namespace {

// The scratch of bitlinear_forward_noalloc.  One copy exists on every device
// that loads this library, for as long as the process runs.  Host code never
// uses this name as an address: the device address is looked up with
// cudaGetSymbolAddress, once per device, with that device current.
static __device__ __align__(256) unsigned char g_noalloc_scratch[BITSSM_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up on the
// first call for that device).
int scratch_on_current_device(void** ptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    bitssm::set_last_error_message("bitlinear_forward_noalloc: no usable current CUDA device");
    return BITSSM_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      char msg[256];
      std::snprintf(msg, sizeof(msg), "bitlinear_forward_noalloc: cudaGetSymbolAddress failed: %s",
                    cudaGetErrorString(e));
      bitssm::set_last_error_message(msg);
      return BITSSM_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *ptr = g_scratch_ptr[dev];
  return BITSSM_OK;
}

}  // namespace

extern "C" int bitlinear_forward_noalloc(const bitssm_tw* w, const void* x, int M, int x_dtype,
                                         void* y, int y_dtype, int act_mode, void* stream) {
  size_t need = 0;
  int rc = bitlinear_workspace_size(w, M, act_mode, &need);
  if (rc != BITSSM_OK) return rc;
  if (need > (size_t)BITSSM_NOALLOC_SCRATCH_BYTES) {
    char msg[256];
    std::snprintf(msg, sizeof(msg),
                  "bitlinear_forward_noalloc: this shape needs %zu bytes of scratch; the built-in "
                  "array holds %zu (use bitlinear_forward with a caller workspace)",
                  need, (size_t)BITSSM_NOALLOC_SCRATCH_BYTES);
    bitssm::set_last_error_message(msg);
    return BITSSM_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  rc = scratch_on_current_device(&scratch);
  if (rc != BITSSM_OK) return rc;
  return bitlinear_forward(w, x, M, x_dtype, y, y_dtype, act_mode, scratch,
                           (size_t)BITSSM_NOALLOC_SCRATCH_BYTES, stream);
}
