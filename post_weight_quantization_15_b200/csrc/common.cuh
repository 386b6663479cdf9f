// Shared device-side helpers of the GPTQ library (status block, loads, launch checks).
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/gptq.h"

namespace gptq {

// Index of the fields of the caller's device status block.
enum { ST_CODE = 0, ST_INFO = 1, ST_STAGE = 2 };

// Stage ids recorded in d_status[ST_STAGE] next to an error.
enum {
  STAGE_HESSIAN = 1, STAGE_PREP_DIAG = 2, STAGE_POTRF = 3, STAGE_TRINV = 4,
  STAGE_INGEST = 5, STAGE_SWEEP = 6, STAGE_TRAILING = 7, STAGE_PACK = 8, STAGE_DEQUANT = 9,
  STAGE_LINEAR = 10
};

// First error wins; later kernels see a non-zero code and skip their work.
__device__ __forceinline__ void set_error(int32_t* st, int code, int info, int stage) {
  if (st == nullptr) return;
  if (atomicCAS(reinterpret_cast<int*>(st + ST_CODE), 0, code) == 0) {
    st[ST_INFO] = info;
    st[ST_STAGE] = stage;
    __threadfence();
  }
}

__device__ __forceinline__ bool has_error(const int32_t* st) {
  if (st == nullptr) return false;
  return *reinterpret_cast<const volatile int32_t*>(st + ST_CODE) != 0;
}

template <typename T> __device__ __forceinline__ float load_as_float(const T* p);
template <> __device__ __forceinline__ float load_as_float<float>(const float* p) { return *p; }
template <> __device__ __forceinline__ float load_as_float<__half>(const __half* p) { return __half2float(*p); }
template <> __device__ __forceinline__ float load_as_float<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}

__host__ __device__ constexpr int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
__host__ __device__ constexpr size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

}  // namespace gptq

namespace gptq {
// Host-side count of enqueued kernels (see gptq_kernel_launches).
void count_launch();
void count_launches(int64_t delta);   // a replayed graph's kernels (or, negative, a captured graph's)
}  // namespace gptq

// Host-side: turn a CUDA launch/runtime failure into GPTQ_ERR_CUDA.
#define GPTQ_CUDA_TRY(expr)                        \
  do {                                             \
    cudaError_t _e = (expr);                       \
    if (_e != cudaSuccess) return GPTQ_ERR_CUDA;   \
  } while (0)

#define GPTQ_LAUNCH_CHECK()                                   \
  do {                                                        \
    ::gptq::count_launch();                                   \
    cudaError_t _e = cudaGetLastError();                      \
    if (_e != cudaSuccess) return GPTQ_ERR_CUDA;              \
  } while (0)
