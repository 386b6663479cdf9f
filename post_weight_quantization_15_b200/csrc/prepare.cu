// K2: dead inputs, act-order, damping and U, the upper Cholesky factor of the
// damped inverse Hessian ("polydesk.ai/glossaire/gptq", "Etape 2": the inverse
// Hessian through a Cholesky decomposition; desc_act; "skillmd.com/skills/
// artubss/gptq": damp_percent).
//
// U is obtained with one Cholesky factorization and one triangular inverse:
// with J the exchange matrix and A = J.Hd.J = L.L^T, Hd = R.R^T for the upper
// triangular R = J.L.J, so Hd^-1 = R^-T.R^-1 and U = R^-1 = J.L^-1.J is the
// upper factor with Hd^-1 = U^T.U (positive diagonal, hence the unique one).
// The permutation and the reversal are folded into one gather:
// A[i][j] = H[q(i)][q(j)] + lambda.delta_ij with q(i) = perm[n-1-i].
//
// Both factorizations are blocked by 128-wide panels.  For panel k:
//   1. one CTA factors the diagonal block L_kk and inverts it in shared memory,
//      writing L_kk, the split of L_kk^-1 and the diagonal block of the inverse;
//   2. L21 = A21 . L_kk^-T        (tensor-core GEMM, store, split output)
//   3. A22 -= L21 . L21^T         (tensor-core GEMM, lower tiles)
//   4. the block column k of the inverse, kept transposed as Xt = (L^-1)^T:
//      Xt[:k0, k] = Xt[:k0, k] . L_kk^-T, then Xt[:k0+nb, later] -= Xt[:, k] . L21^T.
// The GEMMs run in 3 x TF32 (fp32-level accuracy) on tcgen05.
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

// Phase marks of the diagonal-block kernel; empty in the library build.
#ifndef GPTQ_PHASE_MARK
#define GPTQ_PHASE_MARK(i)
#endif

namespace gptq {

namespace {

constexpr int PB = 128;          // panel width

int ld_of(int n) { return (int)align_up((size_t)n, 32); }

struct PrepWs {
  float* A;        // [n, ldn] lower triangle: the reversed, permuted, damped H, then L
  float* Xt;       // [n, ldn] upper triangle: (L^-1)^T
  float* Phi; float* Plo;     // [n, PB] split of the panel A21 before the solve
  float* Lhi; float* Llo;     // [n, PB] split of L21
  float* XPhi; float* XPlo;   // [n, PB] split of Xt[:k0, k] before the solve
  float* XQhi; float* XQlo;   // [n, PB] split of the finished Xt[:, k]
  float* LIhi; float* LIlo;   // [PB, PB] split of L_kk^-1
  double* key;     // [n] act-order key
  float* dfix;     // [n] diag(H) with dead inputs set to 1
  double* scal;    // [0] sum of dfix, [1] lambda
};

PrepWs carve(void* ws, int n) {
  const int ldn = ld_of(n);
  char* p = static_cast<char*>(ws);
  auto take = [&](size_t bytes) { char* q = p; p += align_up(bytes, 256); return q; };
  PrepWs w;
  const size_t nn = (size_t)n * ldn * sizeof(float);
  const size_t panel = (size_t)n * PB * sizeof(float);
  w.A = reinterpret_cast<float*>(take(nn));
  w.Xt = reinterpret_cast<float*>(take(nn));
  w.Phi = reinterpret_cast<float*>(take(panel));  w.Plo = reinterpret_cast<float*>(take(panel));
  w.Lhi = reinterpret_cast<float*>(take(panel));  w.Llo = reinterpret_cast<float*>(take(panel));
  w.XPhi = reinterpret_cast<float*>(take(panel)); w.XPlo = reinterpret_cast<float*>(take(panel));
  w.XQhi = reinterpret_cast<float*>(take(panel)); w.XQlo = reinterpret_cast<float*>(take(panel));
  w.LIhi = reinterpret_cast<float*>(take((size_t)PB * PB * 4));
  w.LIlo = reinterpret_cast<float*>(take((size_t)PB * PB * 4));
  w.key = reinterpret_cast<double*>(take((size_t)n * 8));
  w.dfix = reinterpret_cast<float*>(take((size_t)n * 4));
  w.scal = reinterpret_cast<double*>(take(256));
  return w;
}

__device__ __forceinline__ float tf32_hi(float x) { return __uint_as_float(__float_as_uint(x) & 0xFFFFE000u); }

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
__global__ void prep_gather_kernel(const float* H, const float* dfix, const int32_t* perm, int n, int ldn,
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
    if (!isfinite(v)) set_error(st, GPTQ_ERR_NONFINITE, n - 1 - i, STAGE_PREP_DIAG);
  }
  A[(int64_t)i * ldn + j] = v;
}

// ---------------------------------------------------------------------------
// (5) The diagonal block of panel k: Cholesky L_kk and its inverse T = L_kk^-1
// (rows/columns past nb padded with the identity), in one pass over the 128
// pivots.  256 threads form a 16 x 16 grid; thread (ty, tx) keeps the entries
// (ty + 16a, tx + 16b), a, b < 8, of L and of T in registers.  Pivot j:
//   1. the owners of column j scale it by 1 / L_jj (published to shared memory),
//      and the owners of row j of T scale it by the same factor (row j of T is
//      final: T = L^-1 is the forward elimination of the identity);
//   2. every thread applies the rank-1 updates L[i][k] -= L_ij L_kj (j < k <= i)
//      and T[i][c] -= L_ij T_jc (i > j, c <= j), and the owner of the next
//      pivot computes its square root and reciprocal.
// The pivot loop is unrolled over its eight 16-pivot slot blocks, so every
// register index is a compile-time constant and finished slots are skipped at
// compile time.
// ---------------------------------------------------------------------------
constexpr int POTRF_THREADS = 256;
constexpr size_t POTRF_SMEM = 0;

__device__ __forceinline__ void pivot_publish(float d, int j, float* piv, int* bad, int k0, int n, int32_t* st) {
  if (!(d > 0.f) || !isfinite(d)) {
    if (!*bad) {
      *bad = 1;
      set_error(st, isfinite(d) ? GPTQ_ERR_NOT_SPD : GPTQ_ERR_NONFINITE, n - 1 - (k0 + j), STAGE_POTRF);
    }
    d = 1.f;   // keep the arithmetic finite; every later stage sees the error and skips
  }
  const float sq = sqrtf(d);
  piv[0] = sq;
  piv[1] = __frcp_rn(sq);
}

__global__ void __launch_bounds__(POTRF_THREADS)
potrf_inv_kernel(float* A, int lda, int k0, int nb, int n, float* LIhi, float* LIlo, float* Xt, int ldx,
                 float* XQhi, float* XQlo, int32_t* st) {
  __shared__ float colL[PB];
  __shared__ float rowT[PB];
  __shared__ float piv[2];
  __shared__ int bad;
  if (has_error(st)) return;
  const int tid = threadIdx.x;
  const int ty = tid >> 4, tx = tid & 15;
  if (tid == 0) bad = 0;
  if (tid < PB) { colL[tid] = 0.f; rowT[tid] = 0.f; }

  float l[8][8], t[8][8];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      const int i = ty + 16 * a, k = tx + 16 * b;
      float v = 0.f;
      if (b <= a) v = (i < nb && k <= i) ? A[(int64_t)(k0 + i) * lda + k0 + k] : (i == k ? 1.f : 0.f);
      l[a][b] = v;
      t[a][b] = (i == k) ? 1.f : 0.f;
    }
  __syncthreads();
  GPTQ_PHASE_MARK(0);
  if (tid == 0) pivot_publish(l[0][0], 0, piv, &bad, k0, n, st);   // thread (0, 0) owns (0, 0)
  __syncthreads();

#pragma unroll
  for (int J = 0; J < 8; ++J) {
#pragma unroll 1
    for (int jj = 0; jj < 16; ++jj) {
      const int j = 16 * J + jj;
      const float sq = piv[0], rinv = piv[1];
      // 1. column j of L (owners: tx == jj, slot b = J) and row j of T (owners: ty == jj, slot a = J).
      //    colL[i] is 0 for every row i <= j (a row's entry is zeroed when it is the
      //    pivot and never rewritten), and rowT[c] is 0 for every c > j (never
      //    written yet), so the updates below need no masks.
      if (tx == jj) {
#pragma unroll
        for (int a = J; a < 8; ++a) {
          const int i = ty + 16 * a;
          if (i > j) { l[a][J] *= rinv; colL[i] = l[a][J]; }
          else if (i == j) { l[a][J] = sq; colL[j] = 0.f; }
        }
      }
      if (ty == jj) {
#pragma unroll
        for (int b = 0; b <= J; ++b) {
          const int c = tx + 16 * b;
          if (c <= j) { t[J][b] *= rinv; rowT[c] = t[J][b]; }
        }
      }
      __syncthreads();
      // 2. rank-1 updates (branch-free): L[i][k] -= L_ij L_kj and T[i][c] -= L_ij T_jc.
      //    Entries above the diagonal of the diagonal slots also change; they are
      //    never read.
      float lk[8];
#pragma unroll
      for (int b = J; b < 8; ++b) lk[b] = colL[tx + 16 * b];
      float tr[8];
#pragma unroll
      for (int b = 0; b <= J; ++b) tr[b] = rowT[tx + 16 * b];
#pragma unroll
      for (int a = J; a < 8; ++a) {
        const float li = colL[ty + 16 * a];
#pragma unroll
        for (int b = J; b <= a; ++b) l[a][b] = fmaf(-li, lk[b], l[a][b]);
#pragma unroll
        for (int b = 0; b <= J; ++b) t[a][b] = fmaf(-li, tr[b], t[a][b]);
      }
      // the owner of pivot j + 1 publishes it
      if (jj < 15) {
        if (ty == jj + 1 && tx == jj + 1) pivot_publish(l[J][J], j + 1, piv, &bad, k0, n, st);
      } else if (J < 7) {
        if (ty == 0 && tx == 0) pivot_publish(l[J + 1][J + 1], j + 1, piv, &bad, k0, n, st);
      }
      __syncthreads();
    }
  }
  GPTQ_PHASE_MARK(13);
  if (bad) return;

  // outputs
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      const int i = ty + 16 * a, k = tx + 16 * b;
      if (b <= a && i < nb && k <= i) A[(int64_t)(k0 + i) * lda + k0 + k] = l[a][b];
      // split of L_kk^-1 (B operand rows i, K index k), zero outside nb
      const float tv = (i < nb && k < nb) ? t[a][b] : 0.f;
      const float th = tf32_hi(tv);
      LIhi[i * PB + k] = th;
      LIlo[i * PB + k] = tv - th;
      // transposed: Xt[k0 + k][k0 + i] = T[i][k] and its split XQ[k0 + k][i]
      if (i < nb && k < nb) {
        Xt[(int64_t)(k0 + k) * ldx + k0 + i] = tv;
        XQhi[(int64_t)(k0 + k) * PB + i] = th;
        XQlo[(int64_t)(k0 + k) * PB + i] = tv - th;
      }
    }
}

// (6) U[i][j] = (L^-1)[n-1-i][n-1-j] = Xt[n-1-j][n-1-i] for j >= i, 0 below the diagonal.
__global__ void write_u_kernel(const float* Xt, int n, int ldx, float* U, const int32_t* st) {
  if (has_error(st)) return;
  __shared__ float t[32][33];
  const int i0 = blockIdx.y * 32, j0 = blockIdx.x * 32;
  for (int yy = threadIdx.y; yy < 32; yy += 8) {
    const int j = j0 + yy, i = i0 + threadIdx.x;
    t[yy][threadIdx.x] = (i < n && j < n && j >= i) ? Xt[(int64_t)(n - 1 - j) * ldx + (n - 1 - i)] : 0.f;
  }
  __syncthreads();
  for (int yy = threadIdx.y; yy < 32; yy += 8) {
    const int i = i0 + yy, j = j0 + threadIdx.x;
    if (i < n && j < n) U[(int64_t)i * n + j] = t[threadIdx.x][yy];
  }
}

}  // namespace

size_t prepare_ws_bytes(int n) {
  const int ldn = ld_of(n);
  const size_t nn = align_up((size_t)n * ldn * sizeof(float), 256);
  const size_t panel = align_up((size_t)n * PB * sizeof(float), 256);
  return 2 * nn + 8 * panel + 2 * align_up((size_t)PB * PB * 4, 256) + align_up((size_t)n * 8, 256) +
         align_up((size_t)n * 4, 256) + 256;
}

int launch_prepare(const float* H, const double* hdiag, int n, float damp, int desc_act, float* U,
                   int32_t* perm, uint8_t* dead, void* ws, int32_t* st, cudaStream_t s) {
  PrepWs w = carve(ws, n);
  const int ldn = ld_of(n);
  prep_diag_kernel<<<(int)cdiv(n, 256), 256, 0, s>>>(H, hdiag, n, desc_act, dead, w.key, w.dfix, st);
  GPTQ_LAUNCH_CHECK();
  prep_lambda_kernel<<<1, 1024, 0, s>>>(w.dfix, n, damp, w.scal, st);
  GPTQ_LAUNCH_CHECK();
  if (desc_act) prep_rank_kernel<<<(int)cdiv(n, 256), 256, 0, s>>>(w.key, n, perm, st);
  else prep_identity_kernel<<<(int)cdiv(n, 256), 256, 0, s>>>(perm, n);
  GPTQ_LAUNCH_CHECK();
  {
    dim3 blk(32, 8), grd((unsigned)cdiv(n, 32), (unsigned)cdiv(n, 8));
    prep_gather_kernel<<<grd, blk, 0, s>>>(H, w.dfix, perm, n, ldn, w.scal, w.A, st);
    GPTQ_LAUNCH_CHECK();
  }
  GPTQ_CUDA_TRY(cudaMemsetAsync(w.Xt, 0, (size_t)n * ldn * sizeof(float), s));

  for (int k0 = 0; k0 < n; k0 += PB) {
    const int nb = std::min(PB, n - k0);
    const int rest = n - k0 - nb;
    potrf_inv_kernel<<<1, POTRF_THREADS, 0, s>>>(w.A, ldn, k0, nb, n, w.LIhi, w.LIlo, w.Xt, ldn, w.XQhi,
                                                          w.XQlo, st);
    GPTQ_LAUNCH_CHECK();
    int rc = GPTQ_OK;
    if (rest > 0) {
      float* A21 = w.A + (int64_t)(k0 + nb) * ldn + k0;
      // L21 = A21 . L_kk^-T (stored in place of A21), with its split
      rc = launch_split_tf32(A21, rest, nb, ldn, w.Phi, w.Plo, PB, st, s);
      if (rc == GPTQ_OK)
        rc = launch_gemm3(A21, ldn, rest, nb, nb, w.Phi, w.Plo, PB, w.LIhi, w.LIlo, PB, false, st, s, true, w.Lhi,
                          w.Llo, PB);
      // A22 -= L21 . L21^T (lower tiles)
      if (rc == GPTQ_OK)
        rc = launch_gemm3(w.A + (int64_t)(k0 + nb) * ldn + (k0 + nb), ldn, rest, rest, nb, w.Lhi, w.Llo, PB, w.Lhi,
                          w.Llo, PB, true, st, s);
    }
    if (rc != GPTQ_OK) return rc;
    if (k0 > 0) {
      // Xt[:k0, k] = Xt[:k0, k] . L_kk^-T, with its split (rows 0..k0 of XQ)
      float* Xk = w.Xt + k0;
      rc = launch_split_tf32(Xk, k0, nb, ldn, w.XPhi, w.XPlo, PB, st, s);
      if (rc == GPTQ_OK)
        rc = launch_gemm3(Xk, ldn, k0, nb, nb, w.XPhi, w.XPlo, PB, w.LIhi, w.LIlo, PB, false, st, s, true, w.XQhi,
                          w.XQlo, PB);
      if (rc != GPTQ_OK) return rc;
    }
    if (rest > 0) {
      // Xt[:k0+nb, later] -= Xt[:k0+nb, k] . L21^T
      rc = launch_gemm3(w.Xt + (k0 + nb), ldn, k0 + nb, rest, nb, w.XQhi, w.XQlo, PB, w.Lhi, w.Llo, PB, false, st, s);
      if (rc != GPTQ_OK) return rc;
    }
  }
  {
    dim3 blk(32, 8), grd((unsigned)cdiv(n, 32), (unsigned)cdiv(n, 32));
    write_u_kernel<<<grd, blk, 0, s>>>(w.Xt, n, ldn, U, st);
    GPTQ_LAUNCH_CHECK();
  }
  return GPTQ_OK;
}

}  // namespace gptq
