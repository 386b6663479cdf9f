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
  float* Lhi[2]; float* Llo[2];   // [n, PB] split of L21 (two panels in flight)
  float* XPhi; float* XPlo;   // [n, PB] split of Xt[:k0, k] before the solve
  float* XQhi; float* XQlo;   // [n, PB] split of the finished Xt[:, k]
  float* LIhi[2]; float* LIlo[2]; // [PB, PB] split of L_kk^-1 (two panels in flight)
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
  for (int b = 0; b < 2; ++b) {
    w.Lhi[b] = reinterpret_cast<float*>(take(panel));
    w.Llo[b] = reinterpret_cast<float*>(take(panel));
  }
  w.XPhi = reinterpret_cast<float*>(take(panel)); w.XPlo = reinterpret_cast<float*>(take(panel));
  w.XQhi = reinterpret_cast<float*>(take(panel)); w.XQlo = reinterpret_cast<float*>(take(panel));
  for (int b = 0; b < 2; ++b) {
    w.LIhi[b] = reinterpret_cast<float*>(take((size_t)PB * PB * 4));
    w.LIlo[b] = reinterpret_cast<float*>(take((size_t)PB * PB * 4));
  }
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
// pivots with one CTA barrier per pivot.
//   Layout: warp w owns the columns k = w + 8c (c < 16), lane l the rows
//   i = l + 32r (r < 4); every thread keeps those 64 entries of L and of T in
//   registers.
//   Pivot s, phase A (the warp owning column s only): the pivot comes from the
//   owning lane by a shuffle; the warp scales its column and publishes it
//   (zero for rows <= s) together with 1 / L_ss.
//   Barrier.
//   Phase B (every warp): L[i][k] -= L_is L_ks; T absorbs the previous pivot,
//   T[i][c] -= L_i,s-1 T_s-1,c; then the lanes holding row s of T scale it by
//   1 / L_ss (row s is final: T = L^-1 is the forward elimination of the
//   identity) and publish it for the next pivot.
//   The published vectors rotate through three buffers, so no second barrier
//   is needed.  The pivot loop is unrolled over its 16 column-slot blocks, so
//   every register index is a compile-time constant.
// ---------------------------------------------------------------------------
constexpr int POTRF_THREADS = 256;
constexpr int SLD = PB + 1;
constexpr size_t POTRF_SMEM = (size_t)PB * SLD * sizeof(float);

__global__ void __launch_bounds__(POTRF_THREADS)
potrf_inv_kernel(float* A, int lda, int k0, int nb, int n, float* LIhi, float* LIlo, float* Xt, int ldx,
                 float* XQhi, float* XQlo, int32_t* st) {
  extern __shared__ float stage[];          // [PB][SLD] input / output staging
  __shared__ float colL[3][PB];
  __shared__ float rowT[3][PB];
  __shared__ float piv[3];
  __shared__ int bad;
  if (has_error(st)) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) bad = 0;

  // coalesced load of the lower triangle (identity past nb)
  for (int idx = tid; idx < PB * PB; idx += POTRF_THREADS * 8) {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = idx + u * POTRF_THREADS;
      const int r = e / PB, c = e % PB;
      v[u] = (e < PB * PB && r < nb && c <= r) ? A[(int64_t)(k0 + r) * lda + k0 + c] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = idx + u * POTRF_THREADS;
      const int r = e / PB, c = e % PB;
      if (e < PB * PB) stage[r * SLD + c] = (r >= nb && r == c) ? 1.f : v[u];
    }
  }
  __syncthreads();
  float l[4][16], t[4][16];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const int i = lane + 32 * r, k = warp + 8 * c;
      l[r][c] = k <= i ? stage[i * SLD + k] : 0.f;
      t[r][c] = i == k ? 1.f : 0.f;
    }
  __syncthreads();
  GPTQ_PHASE_MARK(0);

#pragma unroll
  for (int C = 0; C < 16; ++C) {
    const int R = C / 4;                       // row slot of the pivots of this block
#pragma unroll 1
    for (int ws = 0; ws < 8; ++ws) {
      const int s = 8 * C + ws;
      const int buf = s % 3, prev = (s + 2) % 3;
      // ---- phase A: the warp owning column s ----
      if (warp == ws) {
        float d = __shfl_sync(0xffffffffu, l[R][C], 8 * (C % 4) + ws);
        const bool badp = !(d > 0.f) || !isfinite(d);
        if (badp) {
          if (lane == 0 && !bad) {
            bad = 1;
            set_error(st, isfinite(d) ? GPTQ_ERR_NOT_SPD : GPTQ_ERR_NONFINITE, n - 1 - (k0 + s), STAGE_POTRF);
          }
          d = 1.f;   // keep the arithmetic finite; every later stage sees the error and skips
        }
        const float sq = sqrtf(d);
        const float rinv = __frcp_rn(sq);
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int i = lane + 32 * r;
          float v = l[r][C];
          if (i > s) v *= rinv;
          else if (i == s) v = sq;
          if (i >= s) l[r][C] = v;
          colL[buf][i] = i > s ? v : 0.f;
        }
        if (lane == 0) piv[buf] = rinv;
      }
      __syncthreads();
      // ---- phase B: every warp ----
      {
        float li[4];
#pragma unroll
        for (int r = R; r < 4; ++r) li[r] = colL[buf][lane + 32 * r];
#pragma unroll
        for (int c = C; c < 16; ++c) {
          const float lk = colL[buf][warp + 8 * c];
#pragma unroll
          for (int r = R; r < 4; ++r) l[r][c] = fmaf(-li[r], lk, l[r][c]);
        }
        if (s > 0) {
          // T absorbs pivot s - 1 (rows <= s - 1 have a zero multiplier, columns > s - 1 a zero row entry)
          float lp[4];
#pragma unroll
          for (int r = R; r < 4; ++r) lp[r] = colL[prev][lane + 32 * r];
#pragma unroll
          for (int c = 0; c <= C; ++c) {
            const float tk = rowT[prev][warp + 8 * c];
#pragma unroll
            for (int r = R; r < 4; ++r) t[r][c] = fmaf(-lp[r], tk, t[r][c]);
          }
        }
        if (lane == 8 * (C % 4) + ws) {
          // row s of T is final after scaling
          const float rinv = piv[buf];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            if (c <= C) t[R][c] *= rinv;
            rowT[buf][warp + 8 * c] = t[R][c];
          }
        }
      }
    }
  }
  __syncthreads();
  GPTQ_PHASE_MARK(13);
  if (bad) return;

  // outputs, staged through shared memory for coalesced global access
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 16; ++c) stage[(lane + 32 * r) * SLD + warp + 8 * c] = l[r][c];
  __syncthreads();
  for (int idx = tid; idx < PB * PB; idx += POTRF_THREADS) {
    const int i = idx / PB, k = idx % PB;
    if (i < nb && k <= i) A[(int64_t)(k0 + i) * lda + k0 + k] = stage[i * SLD + k];
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 16; ++c) stage[(lane + 32 * r) * SLD + warp + 8 * c] = t[r][c];
  __syncthreads();
  for (int idx = tid; idx < PB * PB; idx += POTRF_THREADS) {
    {
      // split of L_kk^-1 (B operand rows i, K index k), zero outside nb
      const int i = idx / PB, k = idx % PB;
      const float tv = (i < nb && k < nb) ? stage[i * SLD + k] : 0.f;
      const float th = tf32_hi(tv);
      LIhi[i * PB + k] = th;
      LIlo[i * PB + k] = tv - th;
    }
    {
      // transposed: Xt[k0 + k][k0 + i] = T[i][k] and its split XQ[k0 + k][i]
      const int k = idx / PB, i = idx % PB;
      if (i < nb && k < nb) {
        const float tv = stage[i * SLD + k];
        const float th = tf32_hi(tv);
        Xt[(int64_t)(k0 + k) * ldx + k0 + i] = tv;
        XQhi[(int64_t)(k0 + k) * PB + i] = th;
        XQlo[(int64_t)(k0 + k) * PB + i] = tv - th;
      }
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

// The blocked inverse's updates and the trailing updates beyond the next panel run
// on two auxiliary streams next to the factorization: two non-blocking streams and
// a few events per host thread and device, created on first use and kept for the
// life of the process.
struct AuxStream {
  cudaStream_t s = nullptr;    // the inverse's chain
  cudaStream_t t = nullptr;    // the trailing updates beyond the next panel
  cudaEvent_t fork = nullptr, panel = nullptr, join = nullptr, done[2] = {nullptr, nullptr};
  cudaEvent_t rest = nullptr, tjoin = nullptr;
};

int aux_stream(AuxStream** out) {
  // one set per host thread and device, so concurrent callers never share it
  thread_local AuxStream per_dev[64];
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return GPTQ_ERR_CUDA;
  AuxStream& a = per_dev[dev];
  if (a.s == nullptr) {
    if (cudaStreamCreateWithFlags(&a.s, cudaStreamNonBlocking) != cudaSuccess) return GPTQ_ERR_CUDA;
    if (cudaStreamCreateWithFlags(&a.t, cudaStreamNonBlocking) != cudaSuccess) return GPTQ_ERR_CUDA;
    const unsigned f = cudaEventDisableTiming;
    if (cudaEventCreateWithFlags(&a.fork, f) != cudaSuccess || cudaEventCreateWithFlags(&a.panel, f) != cudaSuccess ||
        cudaEventCreateWithFlags(&a.join, f) != cudaSuccess || cudaEventCreateWithFlags(&a.done[0], f) != cudaSuccess ||
        cudaEventCreateWithFlags(&a.done[1], f) != cudaSuccess || cudaEventCreateWithFlags(&a.rest, f) != cudaSuccess ||
        cudaEventCreateWithFlags(&a.tjoin, f) != cudaSuccess)
      return GPTQ_ERR_CUDA;
  }
  *out = &a;
  return GPTQ_OK;
}

}  // namespace

size_t prepare_ws_bytes(int n) {
  const int ldn = ld_of(n);
  const size_t nn = align_up((size_t)n * ldn * sizeof(float), 256);
  const size_t panel = align_up((size_t)n * PB * sizeof(float), 256);
  return 2 * nn + 10 * panel + 4 * align_up((size_t)PB * PB * 4, 256) + align_up((size_t)n * 8, 256) +
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

  GPTQ_CUDA_TRY(cudaFuncSetAttribute(potrf_inv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)POTRF_SMEM));
  AuxStream* aux = nullptr;
  int rc = aux_stream(&aux);
  if (rc != GPTQ_OK) return rc;
  cudaStream_t s2 = aux->s;
  cudaStream_t s3 = aux->t;
  GPTQ_CUDA_TRY(cudaEventRecord(aux->fork, s));
  GPTQ_CUDA_TRY(cudaStreamWaitEvent(s2, aux->fork, 0));
  GPTQ_CUDA_TRY(cudaStreamWaitEvent(s3, aux->fork, 0));
  bool rest_pending = false;

  int panel = 0;
  for (int k0 = 0; k0 < n; k0 += PB, ++panel) {
    const int nb = std::min(PB, n - k0);
    const int rest = n - k0 - nb;
    const int b = panel & 1;
    // the inverse's chain must be done with this buffer's previous use (panel - 2)
    if (panel >= 2) GPTQ_CUDA_TRY(cudaStreamWaitEvent(s, aux->done[b], 0));
    potrf_inv_kernel<<<1, POTRF_THREADS, POTRF_SMEM, s>>>(w.A, ldn, k0, nb, n, w.LIhi[b], w.LIlo[b], w.Xt, ldn,
                                                           w.XQhi, w.XQlo, st);
    GPTQ_LAUNCH_CHECK();
    if (rest > 0) {
      float* A21 = w.A + (int64_t)(k0 + nb) * ldn + k0;
      // L21 = A21 . L_kk^-T (stored in place of A21), with its split
      rc = launch_split_tf32(A21, rest, nb, ldn, w.Phi, w.Plo, PB, st, s);
      if (rc == GPTQ_OK)
        rc = launch_gemm3(A21, ldn, rest, nb, nb, w.Phi, w.Plo, PB, w.LIhi[b], w.LIlo[b], PB, false, st, s, true,
                          w.Lhi[b], w.Llo[b], PB);
      if (rc != GPTQ_OK) return rc;
    }
    GPTQ_CUDA_TRY(cudaEventRecord(aux->panel, s));
    if (rest > 0) {
      // A22 -= L21 . L21^T.  Look-ahead: the next panel's column block on this
      // stream (the next diagonal factorization needs only it); the lower tiles
      // beyond it on the trailing stream, overlapping the next panel's work.
      const int nb2 = std::min(PB, rest);
      float* A22 = w.A + (int64_t)(k0 + nb) * ldn + (k0 + nb);
      // the trailing stream's previous update overlaps this column block
      if (rest_pending) GPTQ_CUDA_TRY(cudaStreamWaitEvent(s, aux->rest, 0));
      rc = launch_gemm3(A22, ldn, rest, nb2, nb, w.Lhi[b], w.Llo[b], PB, w.Lhi[b], w.Llo[b], PB, false, st, s);
      if (rc != GPTQ_OK) return rc;
      if (rest > nb2) {
        GPTQ_CUDA_TRY(cudaStreamWaitEvent(s3, aux->panel, 0));
        rc = launch_gemm3(A22 + (int64_t)nb2 * ldn + nb2, ldn, rest - nb2, rest - nb2, nb, w.Lhi[b] + (int64_t)nb2 * PB,
                          w.Llo[b] + (int64_t)nb2 * PB, PB, w.Lhi[b] + (int64_t)nb2 * PB, w.Llo[b] + (int64_t)nb2 * PB,
                          PB, true, st, s3);
        if (rc != GPTQ_OK) return rc;
        GPTQ_CUDA_TRY(cudaEventRecord(aux->rest, s3));
        rest_pending = true;
      } else {
        rest_pending = false;
      }
    }
    // ---- the inverse's block column k, on the auxiliary stream ----
    GPTQ_CUDA_TRY(cudaStreamWaitEvent(s2, aux->panel, 0));
    if (k0 > 0) {
      // Xt[:k0, k] = Xt[:k0, k] . L_kk^-T, with its split (rows 0..k0 of XQ)
      float* Xk = w.Xt + k0;
      rc = launch_split_tf32(Xk, k0, nb, ldn, w.XPhi, w.XPlo, PB, st, s2);
      if (rc == GPTQ_OK)
        rc = launch_gemm3(Xk, ldn, k0, nb, nb, w.XPhi, w.XPlo, PB, w.LIhi[b], w.LIlo[b], PB, false, st, s2, true,
                          w.XQhi, w.XQlo, PB);
      if (rc != GPTQ_OK) return rc;
    }
    if (rest > 0) {
      // Xt[:k0+nb, later] -= Xt[:k0+nb, k] . L21^T
      rc = launch_gemm3(w.Xt + (k0 + nb), ldn, k0 + nb, rest, nb, w.XQhi, w.XQlo, PB, w.Lhi[b], w.Llo[b], PB, false,
                        st, s2);
      if (rc != GPTQ_OK) return rc;
    }
    GPTQ_CUDA_TRY(cudaEventRecord(aux->done[b], s2));
  }
  GPTQ_CUDA_TRY(cudaEventRecord(aux->join, s2));
  GPTQ_CUDA_TRY(cudaStreamWaitEvent(s, aux->join, 0));
  GPTQ_CUDA_TRY(cudaEventRecord(aux->tjoin, s3));
  GPTQ_CUDA_TRY(cudaStreamWaitEvent(s, aux->tjoin, 0));
  {
    dim3 blk(32, 8), grd((unsigned)cdiv(n, 32), (unsigned)cdiv(n, 32));
    write_u_kernel<<<grd, blk, 0, s>>>(w.Xt, n, ldn, U, st);
    GPTQ_LAUNCH_CHECK();
  }
  return GPTQ_OK;
}

}  // namespace gptq
