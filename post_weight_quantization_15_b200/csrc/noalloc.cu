// gptq_quantize_layer_noalloc: gptq_quantize_layer with its scratch in a
// file-scope __device__ array instead of a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they quantize:
// a plugin whose host application owns every device allocation and forbids
// cudaMalloc inside its execute callback, code that runs while another thread
// may be capturing a stream (cudaMalloc is not allowed during a global-mode
// capture), or a service that must not grow its footprint after start-up.  They
// still pass their own inputs and outputs; only the scratch comes from here.
//
// The array is GPTQ_NOALLOC_SCRATCH_BYTES (32 MiB).  Every GPU that loads this
// library holds one copy of it until the process exits.  All calls on a device
// share it and it keeps the last call's contents; every byte a call reads from it
// is written by that same call first, so nothing needs clearing between calls.
// Calls whose kernels overlap on the GPU (different streams, or different host
// threads without ordering) race on the array.
#include <cuda_runtime.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace {

constexpr size_t kScratchBytes = GPTQ_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the array on the current device.  Host code cannot use
// g_noalloc_scratch itself: on the host that name is a stand-in, not a device
// address.  Looked up once per device, with that device current, and kept for the
// life of the process: after cudaDeviceReset the cached address belongs to a
// context that no longer exists, so this entry point must not be used across a
// device reset.
int scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return GPTQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return GPTQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) return GPTQ_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return GPTQ_OK;
}

}  // namespace

using namespace gptq;

extern "C" int gptq_quantize_layer_noalloc(const void* W, int w_dtype, int out, int n, const float* U,
                                           const int32_t* perm, const uint8_t* dead, int bits, int group_size,
                                           int sym, int block, int32_t* qweight, uint16_t* scales,
                                           uint16_t* zeros, int32_t* g_idx, uint8_t* codes, float* err_sq,
                                           int32_t* d_status, void* stream) {
  // the arguments are checked exactly as gptq_quantize_layer checks them, before the size
  const int arc = check_quantize_args(W, w_dtype, out, n, n, U, bits, group_size, block, qweight, scales, zeros,
                                      g_idx, d_status);
  if (arc != GPTQ_OK) return arc;
  if (quantize_ws_bytes(out, n, block) > kScratchBytes) return GPTQ_ERR_WORKSPACE;
  void* ws = nullptr;
  const int rc = scratch_address(&ws);
  if (rc != GPTQ_OK) return rc;
  return gptq_quantize_layer(W, w_dtype, out, n, U, perm, dead, bits, group_size, sym, block, qweight, scales,
                             zeros, g_idx, codes, err_sq, ws, kScratchBytes, d_status, stream);
}
