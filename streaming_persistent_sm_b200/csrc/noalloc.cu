// wpk_step_noalloc: one decode step whose activation scratch lives in a
// statically allocated device array instead of a caller-allocated buffer.
//
// Who needs it: callers that cannot allocate device memory when they step the
// model - for example a host application that reserves the whole device pool
// up front and hands plugins no allocator, or a real-time loop that must never
// enter an allocator (allocation can block on locks and synchronize the
// device).  Such a caller still passes its inputs and outputs; only the
// scratch moves into the library.
//
// The array below is part of the library image: every GPU that loads the
// library holds its kStaticScratchBytes until the process exits, whether or
// not this entry point is used.
#include <cuda_runtime.h>

#include <atomic>

#include "wpk_internal.h"

extern "C" int wpk_internal_step_scratch(wpk_handle* h, void* scratch, size_t scratch_bytes,
                                         const int32_t* in_tok_dev, int32_t* out_tok_dev, float* logits_dev,
                                         void* stream);

// 8 MiB: a GEMV decode step of the 1B shape at batch 48 with a 624-token
// context needs ~6.9 MiB (only the decode step's scratch moves here; the
// prefill program's buffers stay in the caller's scratch).
static constexpr size_t kStaticScratchBytes = 8u << 20;
static constexpr int kMaxDevices = 64;

// Device storage for the step scratch.  In host code this name is only a
// host-side stand-in for the symbol: its device address comes from
// cudaGetSymbolAddress below and is what the kernels receive.
static __device__ __align__(256) uint8_t g_step_scratch[kStaticScratchBytes];

// Device address of g_step_scratch, per device, looked up by the first call
// on that device.  A device reset (cudaDeviceReset) or a new primary context
// may move the array: this entry point is not meant to be used across one.
static std::atomic<void*> g_scratch_addr[kMaxDevices];

extern "C" int wpk_step_noalloc(wpk_handle* h, const int32_t* in_tok_dev, int32_t* out_tok_dev, float* logits_dev,
                                void* stream) {
  if (!h) return WPK_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return WPK_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return WPK_ERR_UNSUPPORTED;
  void* addr = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (!addr) {
    // One-time set-up on this device (the device must be current).  Racing
    // first callers on different host threads look up the same address.
    if (cudaGetSymbolAddress(&addr, g_step_scratch) != cudaSuccess || !addr) return WPK_ERR_CUDA;
    g_scratch_addr[dev].store(addr, std::memory_order_release);
  }
  return wpk_internal_step_scratch(h, addr, kStaticScratchBytes, in_tok_dev, out_tok_dev, logits_dev, stream);
}
