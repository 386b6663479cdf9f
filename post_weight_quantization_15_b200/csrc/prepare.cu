// K2: dead inputs, act-order, damping and U, the upper Cholesky factor of the
// damped inverse Hessian ("polydesk.ai/glossaire/gptq", "Etape 2": the inverse
// Hessian through a Cholesky decomposition; desc_act; "skillmd.com/skills/
// artubss/gptq": damp_percent).
//
// U is obtained with one Cholesky factorization and one triangular inverse:
// with J the exchange matrix and A = J.Hd.J = L'.L'^T, Hd = R.R^T for the upper
// triangular R = J.L'.J, so Hd^-1 = R^-T.R^-1 and U = R^-1 = J.L'^-1.J is the
// upper factor with Hd^-1 = U^T.U (positive diagonal, hence the unique one).
// The permutation and the reversal are folded into one gather:
// A[i][j] = H[q(i)][q(j)] + lambda.delta_ij with q(i) = perm[n-1-i].
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace gptq {

namespace {

constexpr int NB = 64;  // panel width of the blocked factorization and inverse

struct PrepWs {
  float* A;        // [n, n] lower triangle: the reversed, permuted, damped H, then L'
  float* Xi;       // [n, n] lower triangle: L'^-1
  double* key;     // [n] act-order key
  float* dfix;     // [n] diag(H) with dead inputs set to 1
  double* scal;    // [0] sum of dfix, [1] lambda
};

PrepWs carve(void* ws, int n) {
  char* p = static_cast<char*>(ws);
  PrepWs w;
  const size_t nn = (size_t)n * n * sizeof(float);
  w.A = reinterpret_cast<float*>(p);   p += align_up(nn, 256);
  w.Xi = reinterpret_cast<float*>(p);  p += align_up(nn, 256);
  w.key = reinterpret_cast<double*>(p); p += align_up((size_t)n * 8, 256);
  w.dfix = reinterpret_cast<float*>(p); p += align_up((size_t)n * 4, 256);
  w.scal = reinterpret_cast<double*>(p);
  return w;
}

// (1) dead inputs, the fixed diagonal, the act-order key.
__global__ void prep_diag_kernel(const float* H, const double* hdiag, int n, int desc_act, uint8_t* dead,
                                 double* key, float* dfix, int32_t* st) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n || has_error(st)) return;
  const float d = H[(int64_t)i * n + i];
  if (!isfinite(d)) { set_error(st, GPTQ_ERR_NONFINITE, i, STAGE_PREP_DIAG); return; }
  const bool isdead = d == 0.f;
  dead[i] = isdead ? 1 : 0;
  const float df = isdead ? 1.f : d;
  dfix[i] = df;
  if (desc_act) key[i] = isdead ? 1.0 : (hdiag != nullptr ? hdiag[i] : (double)df);
}

// (2) lambda = damp . mean(dfix): a fixed-order fp64 sum in one block.
__global__ void __launch_bounds__(1024) prep_lambda_kernel(const float* dfix, int n, float damp, double* scal,
                                                           const int32_t* st) {
  if (has_error(st)) return;
  double acc = 0.0;
  for (int i = threadIdx.x; i < n; i += 1024) acc += (double)dfix[i];
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  __shared__ double red[32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < 32; ++w) t += red[w];
    scal[0] = t;
    scal[1] = (double)damp * (t / (double)n);
  }
}

// (3) perm: position of i = #{j : key_j > key_i} + #{j < i : key_j == key_i}
// (a stable descending order, ties by lower index).
constexpr int RANK_TILE = 2048;
__global__ void __launch_bounds__(256) prep_rank_kernel(const double* key, int n, int32_t* perm,
                                                        const int32_t* st) {
  if (has_error(st)) return;
  __shared__ double tile[RANK_TILE];
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const double ki = i < n ? key[i] : 0.0;
  int rank = 0;
  for (int j0 = 0; j0 < n; j0 += RANK_TILE) {
    const int m = min(RANK_TILE, n - j0);
    __syncthreads();
    for (int t = threadIdx.x; t < m; t += blockDim.x) tile[t] = key[j0 + t];
    __syncthreads();
    if (i < n) {
      for (int t = 0; t < m; ++t) {
        const double kj = tile[t];
        rank += (kj > ki) || (kj == ki && j0 + t < i);
      }
    }
  }
  if (i < n) perm[rank] = i;
}

__global__ void prep_identity_kernel(int32_t* perm, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) perm[i] = i;
}

// (4) A[i][j] (i >= j) = H[q(i)][q(j)] + lambda.delta_ij, q(i) = perm[n-1-i];
// H is read from its upper triangle, the diagonal from dfix.
__global__ void prep_gather_kernel(const float* H, const float* dfix, const int32_t* perm, int n,
                                   const double* scal, float* A, int32_t* st) {
  if (has_error(st)) return;
  const int j = blockIdx.x * 32 + threadIdx.x;
  const int i = blockIdx.y * 8 + threadIdx.y;
  if (i >= n || j > i) return;
  const int a = perm[n - 1 - i], b = perm[n - 1 - j];
  float v;
  if (i == j) {
    v = (float)((double)dfix[a] + scal[1]);
  } else {
    const int lo = min(a, b), hi = max(a, b);
    v = H[(int64_t)lo * n + hi];
    if (!isfinite(v)) set_error(st, GPTQ_ERR_NONFINITE, i, STAGE_PREP_DIAG);
  }
  A[(int64_t)i * n + j] = v;
}

// (5a) Cholesky of the NB x NB diagonal block at k0 (all earlier updates applied).
__global__ void __launch_bounds__(256) potrf_kernel(float* A, int n, int k0, int32_t* st) {
  if (has_error(st)) return;
  const int nb = min(NB, n - k0);
  __shared__ float S[NB][NB + 1];
  __shared__ int bad;
  if (threadIdx.x == 0) bad = 0;
  for (int idx = threadIdx.x; idx < NB * NB; idx += blockDim.x) {
    const int r = idx / NB, c = idx % NB;
    S[r][c] = (r < nb && c <= r) ? A[(int64_t)(k0 + r) * n + k0 + c] : 0.f;
  }
  __syncthreads();
  for (int c = 0; c < nb; ++c) {
    if (threadIdx.x == 0) {
      const float d = S[c][c];
      if (!(d > 0.f) || !isfinite(d)) {
        set_error(st, isfinite(d) ? GPTQ_ERR_NOT_SPD : GPTQ_ERR_NONFINITE, n - 1 - (k0 + c), STAGE_POTRF);
        bad = 1;
      } else {
        S[c][c] = sqrtf(d);
      }
    }
    __syncthreads();
    if (bad) return;
    const float dc = S[c][c];
    for (int r = c + 1 + threadIdx.x; r < nb; r += blockDim.x) S[r][c] /= dc;
    __syncthreads();
    const int m = nb - c - 1;
    for (int idx = threadIdx.x; idx < m * m; idx += blockDim.x) {
      const int r = c + 1 + idx / m, cc = c + 1 + idx % m;
      if (cc <= r) S[r][cc] = fmaf(-S[r][c], S[cc][c], S[r][cc]);
    }
    __syncthreads();
  }
  for (int idx = threadIdx.x; idx < NB * NB; idx += blockDim.x) {
    const int r = idx / NB, c = idx % NB;
    if (r < nb && c <= r) A[(int64_t)(k0 + r) * n + k0 + c] = S[r][c];
  }
}

// (5b) Rows below the diagonal block: x . L_kk^T = a  (one thread per row).
__global__ void __launch_bounds__(64) trsm_kernel(float* A, int n, int k0, const int32_t* st) {
  if (has_error(st)) return;
  __shared__ float L[NB][NB + 1];
  const int nb = min(NB, n - k0);
  for (int idx = threadIdx.x; idx < NB * NB; idx += blockDim.x) {
    const int r = idx / NB, c = idx % NB;
    L[r][c] = (r < nb && c <= r) ? A[(int64_t)(k0 + r) * n + k0 + c] : 0.f;
  }
  __syncthreads();
  const int row = k0 + nb + blockIdx.x * 64 + threadIdx.x;
  if (row >= n) return;
  float* a = A + (int64_t)row * n + k0;
  float x[NB];
#pragma unroll
  for (int c = 0; c < NB; ++c) x[c] = c < nb ? a[c] : 0.f;
#pragma unroll
  for (int c = 0; c < NB; ++c) {
    if (c < nb) {
      float v = x[c];
#pragma unroll
      for (int m = 0; m < c; ++m) v = fmaf(-x[m], L[c][m], v);
      x[c] = v / L[c][c];
    }
  }
#pragma unroll
  for (int c = 0; c < NB; ++c)
    if (c < nb) a[c] = x[c];
}

// C[r][c] -= sum_m P[r][m] . Q(m, c) on 64x64 tiles (CUDA-core fp32); used for the
// trailing update of the factorization (Q(m, c) = Qp[c][m], lower tiles only)
// and of the inverse (Q(m, c) = Qp[m][c]).  All pointers are pre-offset to the
// first row / column of the update.
constexpr int TT = 64;
constexpr int TK = 16;

template <bool LOWER_ONLY, bool Q_ROWS_ARE_K>
__global__ void __launch_bounds__(256)
tile_update_kernel(float* C, int ldc, int M, int N, int K, const float* P, int ldp, const float* Q, int ldq,
                   const int32_t* st) {
  if (has_error(st)) return;
  const int ti = blockIdx.y, tj = blockIdx.x;
  if (LOWER_ONLY && tj > ti) return;
  __shared__ float Ps[TK][TT + 4];
  __shared__ float Qs[TK][TT + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int rbase = ti * TT, cbase = tj * TT;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += TK) {
    for (int idx = threadIdx.x; idx < TT * TK; idx += 256) {
      {  // P tile: rows rbase.., k0..  (k fastest across threads)
        const int r = idx / TK, k = idx % TK;
        const int gr = rbase + r, gk = k0 + k;
        Ps[k][r] = (gr < M && gk < K) ? P[(int64_t)gr * ldp + gk] : 0.f;
      }
      if (Q_ROWS_ARE_K) {  // Q(m, c) = Q[m][c]: columns fastest
        const int k = idx / TT, c = idx % TT;
        const int gc = cbase + c, gk = k0 + k;
        Qs[k][c] = (gc < N && gk < K) ? Q[(int64_t)gk * ldq + gc] : 0.f;
      } else {             // Q(m, c) = Q[c][m]: k fastest
        const int c = idx / TK, k = idx % TK;
        const int gc = cbase + c, gk = k0 + k;
        Qs[k][c] = (gc < N && gk < K) ? Q[(int64_t)gc * ldq + gk] : 0.f;
      }
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < TK; ++k) {
      float a[4], b[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) { a[u] = Ps[k][ty * 4 + u]; b[u] = Qs[k][tx * 4 + u]; }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(a[u], b[v], acc[u][v]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int gr = rbase + ty * 4 + u;
    if (gr >= M) continue;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int gc = cbase + tx * 4 + v;
      if (gc < N && (!LOWER_ONLY || gc <= gr)) C[(int64_t)gr * ldc + gc] -= acc[u][v];
    }
  }
}

// (6) L'^-1: start from the identity.
__global__ void trinv_init_kernel(float* Xi, int n, const int32_t* st) {
  if (has_error(st)) return;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)n * n) return;
  const int64_t i = idx / n, j = idx % n;
  Xi[idx] = (i == j) ? 1.f : 0.f;
}

// (6a) Rows k0.. of the inverse: solve L_kk . Y = B for columns [0, k0 + nb), one
// thread per column (forward substitution).
__global__ void __launch_bounds__(128) trinv_diag_kernel(const float* A, float* Xi, int n, int k0,
                                                         const int32_t* st) {
  if (has_error(st)) return;
  __shared__ float L[NB][NB + 1];
  const int nb = min(NB, n - k0);
  for (int idx = threadIdx.x; idx < NB * NB; idx += blockDim.x) {
    const int r = idx / NB, c = idx % NB;
    L[r][c] = (r < nb && c <= r) ? A[(int64_t)(k0 + r) * n + k0 + c] : 0.f;
  }
  __syncthreads();
  const int col = blockIdx.x * blockDim.x + threadIdx.x;
  if (col >= k0 + nb) return;
  float y[NB];
#pragma unroll
  for (int r = 0; r < NB; ++r) y[r] = r < nb ? Xi[(int64_t)(k0 + r) * n + col] : 0.f;
#pragma unroll
  for (int r = 0; r < NB; ++r) {
    if (r < nb) {
      float v = y[r];
#pragma unroll
      for (int m = 0; m < r; ++m) v = fmaf(-L[r][m], y[m], v);
      y[r] = v / L[r][r];
    }
  }
#pragma unroll
  for (int r = 0; r < NB; ++r)
    if (r < nb) Xi[(int64_t)(k0 + r) * n + col] = y[r];
}

// (7) U[i][j] = L'^-1[n-1-i][n-1-j] for j >= i, 0 below the diagonal.
__global__ void write_u_kernel(const float* Xi, int n, float* U, const int32_t* st) {
  if (has_error(st)) return;
  const int j = blockIdx.x * 32 + threadIdx.x;
  const int i = blockIdx.y * 8 + threadIdx.y;
  if (i >= n || j >= n) return;
  U[(int64_t)i * n + j] = (j >= i) ? Xi[(int64_t)(n - 1 - i) * n + (n - 1 - j)] : 0.f;
}

}  // namespace

size_t prepare_ws_bytes(int n) {
  const size_t nn = (size_t)n * n * sizeof(float);
  return 2 * align_up(nn, 256) + align_up((size_t)n * 8, 256) + align_up((size_t)n * 4, 256) + 256;
}

int launch_prepare(const float* H, const double* hdiag, int n, float damp, int desc_act, float* U,
                   int32_t* perm, uint8_t* dead, void* ws, int32_t* st, cudaStream_t s) {
  PrepWs w = carve(ws, n);
  const int nthr = 256;
  prep_diag_kernel<<<(int)cdiv(n, nthr), nthr, 0, s>>>(H, hdiag, n, desc_act, dead, w.key, w.dfix, st);
  GPTQ_LAUNCH_CHECK();
  prep_lambda_kernel<<<1, 1024, 0, s>>>(w.dfix, n, damp, w.scal, st);
  GPTQ_LAUNCH_CHECK();
  if (desc_act) prep_rank_kernel<<<(int)cdiv(n, 256), 256, 0, s>>>(w.key, n, perm, st);
  else prep_identity_kernel<<<(int)cdiv(n, 256), 256, 0, s>>>(perm, n);
  GPTQ_LAUNCH_CHECK();
  {
    dim3 blk(32, 8), grd((unsigned)cdiv(n, 32), (unsigned)cdiv(n, 8));
    prep_gather_kernel<<<grd, blk, 0, s>>>(H, w.dfix, perm, n, w.scal, w.A, st);
    GPTQ_LAUNCH_CHECK();
  }
  // Blocked right-looking Cholesky A = L'.L'^T (lower, in place).
  for (int k0 = 0; k0 < n; k0 += NB) {
    const int nb = std::min(NB, n - k0);
    potrf_kernel<<<1, 256, 0, s>>>(w.A, n, k0, st);
    GPTQ_LAUNCH_CHECK();
    const int rest = n - k0 - nb;
    if (rest > 0) {
      trsm_kernel<<<(int)cdiv(rest, 64), 64, 0, s>>>(w.A, n, k0, st);
      GPTQ_LAUNCH_CHECK();
      float* P = w.A + (int64_t)(k0 + nb) * n + k0;
      float* C = w.A + (int64_t)(k0 + nb) * n + (k0 + nb);
      dim3 grd((unsigned)cdiv(rest, TT), (unsigned)cdiv(rest, TT));
      tile_update_kernel<true, false><<<grd, 256, 0, s>>>(C, n, rest, rest, nb, P, n, P, n, st);
      GPTQ_LAUNCH_CHECK();
    }
  }
  // Blocked forward substitution L'.Xi = I.
  trinv_init_kernel<<<(unsigned)cdiv((int64_t)n * n, 256), 256, 0, s>>>(w.Xi, n, st);
  GPTQ_LAUNCH_CHECK();
  for (int k0 = 0; k0 < n; k0 += NB) {
    const int nb = std::min(NB, n - k0);
    trinv_diag_kernel<<<(int)cdiv(k0 + nb, 128), 128, 0, s>>>(w.A, w.Xi, n, k0, st);
    GPTQ_LAUNCH_CHECK();
    const int rest = n - k0 - nb;
    if (rest > 0) {
      const float* P = w.A + (int64_t)(k0 + nb) * n + k0;   // L'[k0+nb.., k0..k0+nb)
      const float* Q = w.Xi + (int64_t)k0 * n;              // Xi[k0..k0+nb, 0..)
      float* C = w.Xi + (int64_t)(k0 + nb) * n;             // Xi[k0+nb.., 0..k0+nb)
      dim3 grd((unsigned)cdiv(k0 + nb, TT), (unsigned)cdiv(rest, TT));
      tile_update_kernel<false, true><<<grd, 256, 0, s>>>(C, n, rest, k0 + nb, nb, P, n, Q, n, st);
      GPTQ_LAUNCH_CHECK();
    }
  }
  {
    dim3 blk(32, 8), grd((unsigned)cdiv(n, 32), (unsigned)cdiv(n, 8));
    write_u_kernel<<<grd, blk, 0, s>>>(w.Xi, n, U, st);
    GPTQ_LAUNCH_CHECK();
  }
  return GPTQ_OK;
}

}  // namespace gptq
