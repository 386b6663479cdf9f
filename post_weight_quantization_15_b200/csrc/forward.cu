// The elementwise steps of a quantized block's forward pass, for the sequential
// pipeline in which each layer is calibrated on the outputs of the layers already
// quantized before it ("polydesk.ai/glossaire/gptq": GPTQ works layer by layer;
// "wikiprompt.org", "GPTQ").  Activations keep the calibration layout of the Hessian,
// [features, tokens] bf16 with tokens contiguous; the products run on the tensor
// cores (linear_kernel in linear.cu); these kernels are HBM-bound and move 16 bytes
// per thread where the layout allows.
//   transpose_bf16_kernel   X [rows, cols] -> Xt [cols, rows] (the K-major operand of
//                           the product), 64 x 64 tiles through shared memory
//   silu_mul_kernel         h = bf16(silu(g) . u), g and u fp32 (the gated MLP)
//   residual_add_kernel     Xn = bf16(x + y), x bf16, y fp32
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace gptq {

namespace {

constexpr int TT = 64;

__global__ void __launch_bounds__(256) transpose_bf16_kernel(const __nv_bfloat16* X, int rows, int cols, int64_t ldx,
                                                             __nv_bfloat16* Xt, int64_t ldt, const int32_t* st) {
  if (has_error(st)) return;
  __shared__ __nv_bfloat16 t[TT][TT + 2];
  const int r0 = blockIdx.y * TT, c0 = blockIdx.x * TT;
  for (int i = threadIdx.x; i < TT * TT; i += blockDim.x) {
    const int r = i / TT, c = i % TT;
    t[r][c] = (r0 + r < rows && c0 + c < cols) ? X[(int64_t)(r0 + r) * ldx + c0 + c] : __float2bfloat16(0.f);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < TT * TT; i += blockDim.x) {
    const int c = i / TT, r = i % TT;
    if (c0 + c < cols && r0 + r < rows) Xt[(int64_t)(c0 + c) * ldt + r0 + r] = t[r][c];
  }
}

__device__ __forceinline__ float silu(float g) { return g / (1.f + expf(-g)); }

__global__ void silu_mul_kernel(const float* G, const float* U, int64_t count, __nv_bfloat16* h, const int32_t* st) {
  if (has_error(st)) return;
  const int64_t i = 4 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 3 < count) {
    const float4 g = *reinterpret_cast<const float4*>(G + i);
    const float4 u = *reinterpret_cast<const float4*>(U + i);
    const __nv_bfloat162 a = __floats2bfloat162_rn(silu(g.x) * u.x, silu(g.y) * u.y);
    const __nv_bfloat162 b = __floats2bfloat162_rn(silu(g.z) * u.z, silu(g.w) * u.w);
    reinterpret_cast<__nv_bfloat162*>(h + i)[0] = a;
    reinterpret_cast<__nv_bfloat162*>(h + i)[1] = b;
  } else {
    for (int64_t j = i; j < count; ++j) h[j] = __float2bfloat16_rn(silu(G[j]) * U[j]);
  }
}

__global__ void residual_add_kernel(const __nv_bfloat16* X, const float* Y, int64_t count, __nv_bfloat16* Xn,
                                    const int32_t* st) {
  if (has_error(st)) return;
  const int64_t i = 4 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 3 < count) {
    const float4 y = *reinterpret_cast<const float4*>(Y + i);
    const __nv_bfloat162 x0 = reinterpret_cast<const __nv_bfloat162*>(X + i)[0];
    const __nv_bfloat162 x1 = reinterpret_cast<const __nv_bfloat162*>(X + i)[1];
    reinterpret_cast<__nv_bfloat162*>(Xn + i)[0] =
        __floats2bfloat162_rn(__low2float(x0) + y.x, __high2float(x0) + y.y);
    reinterpret_cast<__nv_bfloat162*>(Xn + i)[1] =
        __floats2bfloat162_rn(__low2float(x1) + y.z, __high2float(x1) + y.w);
  } else {
    for (int64_t j = i; j < count; ++j) Xn[j] = __float2bfloat16_rn(__bfloat162float(X[j]) + Y[j]);
  }
}

}  // namespace

int launch_transpose_bf16(const void* X, int rows, int cols, int64_t ldx, void* Xt, int64_t ldt, const int32_t* st,
                          cudaStream_t s) {
  TraceScope ts("transpose_bf16", "byte", 4.0 * rows * (double)cols, s);
  dim3 grd((unsigned)cdiv(cols, TT), (unsigned)cdiv(rows, TT));
  transpose_bf16_kernel<<<grd, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(X), rows, cols, ldx,
                                            static_cast<__nv_bfloat16*>(Xt), ldt, st);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

int launch_silu_mul(const float* G, const float* U, int64_t count, void* h, const int32_t* st, cudaStream_t s) {
  TraceScope ts("silu_mul", "byte", 10.0 * (double)count, s);
  silu_mul_kernel<<<(unsigned)cdiv(cdiv(count, 4), 256), 256, 0, s>>>(G, U, count,
                                                                      static_cast<__nv_bfloat16*>(h), st);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

int launch_residual_add(const void* X, const float* Y, int64_t count, void* Xn, const int32_t* st, cudaStream_t s) {
  TraceScope ts("residual_add", "byte", 8.0 * (double)count, s);
  residual_add_kernel<<<(unsigned)cdiv(cdiv(count, 4), 256), 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(X), Y, count, static_cast<__nv_bfloat16*>(Xn), st);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

}  // namespace gptq
