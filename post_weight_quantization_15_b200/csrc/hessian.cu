// K1: H += 2 . X . X^T  ("polydesk.ai/glossaire/gptq", "Etape 2": H = 2.X.X^T).
//
// hessian_diag64_kernel: the act-order key, 2 . sum_t x_it^2 in fp64 (every bf16
// square is exact in fp64).
#include "common.cuh"
#include "internal.h"

namespace gptq {

namespace {

constexpr int DIAG_THREADS = 256;

__global__ void __launch_bounds__(DIAG_THREADS)
hessian_diag64_kernel(double* hdiag, int n, const __nv_bfloat16* X, int64_t ld_x, int64_t tokens,
                      const int32_t* st) {
  const int i = blockIdx.x;
  if (i >= n || has_error(st)) return;
  const __nv_bfloat16* row = X + (int64_t)i * ld_x;
  double acc = 0.0;
  for (int64_t t = threadIdx.x; t < tokens; t += DIAG_THREADS) {
    const double v = (double)__bfloat162float(row[t]);
    acc = fma(v, v, acc);
  }
  __shared__ double red[DIAG_THREADS / 32];
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < DIAG_THREADS / 32; ++w) t += red[w];
    hdiag[i] += 2.0 * t;
  }
}

// Plain CUDA-core version of the Hessian tile product: one 64x64 upper tile per
// CTA, 4x4 outputs per thread, tokens staged through shared memory.
constexpr int HT = 64;
constexpr int HK = 32;

__global__ void __launch_bounds__(256)
hessian_simple_kernel(float* H, int n, const __nv_bfloat16* X, int64_t ld_x, int64_t tokens,
                      const int32_t* st) {
  if (has_error(st)) return;
  const int T = (int)cdiv(n, HT);
  int t = blockIdx.x, bi = 0;
  while (t >= T - bi) { t -= T - bi; ++bi; }
  const int bj = bi + t;
  __shared__ float As[HK][HT + 4];
  __shared__ float Bs[HK][HT + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int64_t k0 = 0; k0 < tokens; k0 += HK) {
    for (int idx = threadIdx.x; idx < HT * HK; idx += 256) {
      const int r = idx / HK, k = idx % HK;
      const int64_t gk = k0 + k;
      const int gi = bi * HT + r, gj = bj * HT + r;
      As[k][r] = (gi < n && gk < tokens) ? __bfloat162float(X[(int64_t)gi * ld_x + gk]) : 0.f;
      Bs[k][r] = (gj < n && gk < tokens) ? __bfloat162float(X[(int64_t)gj * ld_x + gk]) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < HK; ++k) {
      float a[4], b[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) { a[u] = As[k][ty * 4 + u]; b[u] = Bs[k][tx * 4 + u]; }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(a[u], b[v], acc[u][v]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int gi = bi * HT + ty * 4 + u;
    if (gi >= n) continue;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int gj = bj * HT + tx * 4 + v;
      if (gj < n) H[(int64_t)gi * n + gj] += 2.f * acc[u][v];
    }
  }
}

}  // namespace

int launch_hessian_diag64(double* hdiag, int n, const void* X, int64_t ld_x, int64_t tokens,
                          int32_t* st, cudaStream_t s) {
  hessian_diag64_kernel<<<n, DIAG_THREADS, 0, s>>>(hdiag, n, static_cast<const __nv_bfloat16*>(X), ld_x,
                                                   tokens, st);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

int launch_hessian(float* H, int n, const void* X, int64_t ld_x, int64_t tokens, int32_t* st,
                   cudaStream_t s) {
  const int T = (int)cdiv(n, HT);
  const int tiles = T * (T + 1) / 2;
  hessian_simple_kernel<<<tiles, 256, 0, s>>>(H, n, static_cast<const __nv_bfloat16*>(X), ld_x, tokens, st);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

}  // namespace gptq
