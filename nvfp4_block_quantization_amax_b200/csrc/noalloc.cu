// noalloc.cu -- nvfp4_quantize without a caller-supplied workspace.
//
// Who needs this: code that must not allocate device memory when it
// quantizes -- a plugin hosted inside another runtime that owns all device
// memory, or a program that fixes its memory plan at start-up and may not
// call cudaMalloc afterwards.  Such a caller still owns x and every output
// buffer; only the scratch comes from a fixed array compiled into this
// library: the per-CTA amax partials of the amax pass and, with
// NVFP4_SINGLE_PASS, the grid barrier's arrival counter after them.
//
// The array is a file-scope __device__ symbol, so every GPU that loads the
// library holds it (kNoAllocScratchBytes bytes) until the process exits.
// Host code cannot use the symbol's name as a device address: the first call
// on each device, with that device current, looks the address up with
// cudaGetSymbolAddress and keeps it for later calls.  Make that first call on
// a device before any stream capture starts, and do not reset the device
// (cudaDeviceReset) between calls: a reset reloads the module, the array may
// move, and the kept address would then be stale.  Arguments are checked
// before the lookup, so a call the library rejects never performs it.
//
// All calls on a device share the one array and it keeps whatever the last
// call wrote.  The amax partials need no clearing (the amax pass writes every
// partial that the quantize kernel then reads); the barrier counter must
// start at zero and each single-pass call clears it with a stream-ordered
// memset.  Two calls whose kernels may run at the same time on the GPU (for
// example on two unordered streams) race on the partials and on the counter
// and can produce wrong results or a barrier that gives up (NVFP4_ERR_TIMEOUT
// in the status word); order such calls on one stream.
#include <cuda_runtime.h>
#include <cstdint>
#include <mutex>

#include "nvfp4.h"
#include "nvfp4_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 8192;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device (looked up once
// per device).  nullptr if the lookup failed.
void* scratch_on_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    g_scratch_ptr[dev] = p;
  }
  return g_scratch_ptr[dev];
}

}  // namespace

extern "C" {

nvfp4_status_t nvfp4_quantize_noalloc(const void* x, int64_t R, int64_t C, int64_t ld, nvfp4_mode_t mode,
                                      uint32_t flags, uint64_t seed, uint32_t stream_id,
                                      const float* alpha_in, const nvfp4_qtensor_t* out, void* stream) {
  bool empty = false;
  const nvfp4_status_t chk =
      nvfp4::check_quantize_args(x, R, C, ld, mode, flags, stream_id, alpha_in, out, &empty);
  if (chk != NVFP4_OK || empty) return chk;
  const size_t need = nvfp4_workspace_size(R, C, flags);
  if (need > kNoAllocScratchBytes) return NVFP4_ERR_WORKSPACE;  // more scratch than the fixed array holds
  void* scratch = nullptr;
  if (need > 0) {
    scratch = scratch_on_current_device();
    if (!scratch) return NVFP4_ERR_CUDA;
  }
  return nvfp4_quantize(x, R, C, ld, mode, flags, seed, stream_id, alpha_in, out, scratch,
                        need > 0 ? kNoAllocScratchBytes : 0, stream);
}

}  // extern "C"
