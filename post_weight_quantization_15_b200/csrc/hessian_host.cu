// H += 2 . X . X^T from X in host memory ("polydesk.ai/glossaire/gptq", "Etape 2"),
// with the transfer hidden behind the tile products: X crosses PCIe in chunks of
// tokens (one 2-D copy per chunk: n rows of a token slab) on a copy stream, into a
// caller-provided device staging area split in two halves; chunk i's tile product
// runs on the caller's stream while chunk i + 1 is copied into the other half.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace gptq {

namespace {

// One copy stream and four events per host thread and device, created on first use
// and kept for the life of the process.
struct CopyStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr;
  cudaEvent_t copied[2] = {nullptr, nullptr};
  cudaEvent_t consumed[2] = {nullptr, nullptr};
};

int copy_stream(CopyStream** out) {
  thread_local CopyStream per_dev[64];
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return GPTQ_ERR_CUDA;
  CopyStream& c = per_dev[dev];
  if (c.s == nullptr) {
    if (cudaStreamCreateWithFlags(&c.s, cudaStreamNonBlocking) != cudaSuccess) return GPTQ_ERR_CUDA;
    const unsigned f = cudaEventDisableTiming;
    cudaEvent_t* evs[] = {&c.fork, &c.copied[0], &c.copied[1], &c.consumed[0], &c.consumed[1]};
    for (cudaEvent_t* e : evs)
      if (cudaEventCreateWithFlags(e, f) != cudaSuccess) return GPTQ_ERR_CUDA;
  }
  *out = &c;
  return GPTQ_OK;
}

}  // namespace

int64_t hessian_host_chunk(int n, size_t staging_bytes) {
  // tokens per staging half, a multiple of the tile product's 64-token stage
  const int64_t per_half = (int64_t)(staging_bytes / 2 / ((size_t)n * 2));
  return per_half / 64 * 64;
}

int launch_hessian_host(float* H, double* hdiag, int n, const void* X_host, int x_rows, int64_t ld_x_host,
                        int64_t tokens, void* staging, size_t staging_bytes, int32_t* st, cudaStream_t s) {
  // only X's x_rows rows cross; the rest of H's n rows are zero padding
  const int64_t chunk = std::min(hessian_host_chunk(x_rows, staging_bytes), (int64_t)align_up((size_t)tokens, 64));
  if (chunk < 64) return GPTQ_ERR_WORKSPACE;
  CopyStream* cs = nullptr;
  int rc = copy_stream(&cs);
  if (rc != GPTQ_OK) return rc;
  // the copies follow whatever the caller's stream has queued (the staging area may still be read)
  GPTQ_CUDA_TRY(cudaEventRecord(cs->fork, s));
  GPTQ_CUDA_TRY(cudaStreamWaitEvent(cs->s, cs->fork, 0));
  const char* src = static_cast<const char*>(X_host);
  int i = 0;
  for (int64_t t0 = 0; t0 < tokens; t0 += chunk, ++i) {
    const int b = i & 1;
    const int64_t cw = std::min(chunk, tokens - t0);
    char* dst = static_cast<char*>(staging) + (size_t)b * (size_t)x_rows * (size_t)chunk * 2;
    if (i >= 2) GPTQ_CUDA_TRY(cudaStreamWaitEvent(cs->s, cs->consumed[b], 0));   // that half is free again
    GPTQ_CUDA_TRY(cudaMemcpy2DAsync(dst, (size_t)chunk * 2, src + t0 * 2, (size_t)ld_x_host * 2, (size_t)cw * 2,
                                    (size_t)x_rows, cudaMemcpyHostToDevice, cs->s));
    GPTQ_CUDA_TRY(cudaEventRecord(cs->copied[b], cs->s));
    GPTQ_CUDA_TRY(cudaStreamWaitEvent(s, cs->copied[b], 0));
    rc = launch_hessian(H, n, dst, x_rows, chunk, cw, st, s);
    if (rc == GPTQ_OK && hdiag != nullptr) rc = launch_hessian_diag64(hdiag, x_rows, dst, chunk, cw, st, s);
    if (rc != GPTQ_OK) return rc;
    GPTQ_CUDA_TRY(cudaEventRecord(cs->consumed[b], s));
  }
  return GPTQ_OK;
}

}  // namespace gptq
