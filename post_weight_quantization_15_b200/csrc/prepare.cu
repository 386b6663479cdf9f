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
#include <atomic>
#include <cstring>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

// Phase marks of the diagonal-block kernel; empty in the library build.
#ifndef GPTQ_PHASE_MARK
#define GPTQ_PHASE_MARK(i)
#endif

namespace gptq {

namespace {

constexpr int PB = 128;          // panel width
constexpr int NBUF = 3;          // panels in flight (per-panel loop): per-panel buffers form a ring
constexpr int SPB = 4 * PB;      // super-panel width (deferred loop)
constexpr int NSUP = 3;          // super-panels in flight (deferred loop)
constexpr int NLI = 3 * (SPB / PB);   // ring of L_kk^-1 splits and per-panel events

int ld_of(int n) { return (int)align_up((size_t)n, 32); }

struct PrepWs {
  float* A;        // [n, ldn] lower triangle: the reversed, permuted, damped H, then L
  float* Xt;       // [n, ldn] upper triangle: (L^-1)^T
  float* Phi; float* Plo;     // [n, PB] split of the panel A21 before the solve
  float* XPhi; float* XPlo;   // [n, PB] split of Xt[:k0, k] before the solve
  // per-panel loop: a ring of L21 splits and the finished Xt[:, k]
  float* Lhi[NBUF]; float* Llo[NBUF];     // [n, PB]
  float* XQhi; float* XQlo;               // [n, PB]
  // deferred loop (the same memory): a super-panel's L21 and finished Xt columns
  float* Shi[NSUP]; float* Slo[NSUP];     // [n, SPB], row r holds L(r, super-panel columns)
  float* SXhi; float* SXlo;               // [n, SPB], row r holds Xt(r, super-panel columns)
  float* LIhi[NLI]; float* LIlo[NLI];     // [PB, PB] split of L_kk^-1 (a ring)
  double* key;     // [n] act-order key
  float* dfix;     // [n] diag(H) with dead inputs set to 1
  double* scal;    // [0] sum of dfix, [1] lambda
};

PrepWs carve(void* ws, int n) {
  const int ldn = ld_of(n);
  char* p = static_cast<char*>(ws);
  auto take = [&](size_t bytes) { char* q = p; p += align_up(bytes, 256); return q; };
  auto f = [](char* q) { return reinterpret_cast<float*>(q); };
  PrepWs w;
  const size_t nn = (size_t)n * ldn * sizeof(float);
  const size_t panel = (size_t)n * PB * sizeof(float);
  const size_t sup = (size_t)n * SPB * sizeof(float);
  w.A = f(take(nn));
  w.Xt = f(take(nn));
  w.Phi = f(take(panel));  w.Plo = f(take(panel));
  w.XPhi = f(take(panel)); w.XPlo = f(take(panel));
  // the two loops' buffers share one region
  static_assert((2 * NBUF + 2) * PB <= (2 * NSUP + 2) * SPB, "the per-panel buffers fit in the shared region");
  char* shared = take((2 * NSUP + 2) * align_up(sup, 256));
  char* q = shared;
  for (int b = 0; b < NSUP; ++b) {
    w.Shi[b] = f(q); q += align_up(sup, 256);
    w.Slo[b] = f(q); q += align_up(sup, 256);
  }
  w.SXhi = f(q); q += align_up(sup, 256);
  w.SXlo = f(q);
  q = shared;
  for (int b = 0; b < NBUF; ++b) {
    w.Lhi[b] = f(q); q += align_up(panel, 256);
    w.Llo[b] = f(q); q += align_up(panel, 256);
  }
  w.XQhi = f(q); q += align_up(panel, 256);
  w.XQlo = f(q);
  for (int b = 0; b < NLI; ++b) {
    w.LIhi[b] = f(take((size_t)PB * PB * 4));
    w.LIlo[b] = f(take((size_t)PB * PB * 4));
  }
  w.key = reinterpret_cast<double*>(take((size_t)n * 8));
  w.dfix = f(take((size_t)n * 4));
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

// (4') The same with the identity order, q(i) = n-1-i: row i of A is row n-1-i of
// H read backwards, so reads and writes are both contiguous.  One block per row.
// The act-order gather in two coalesced passes (for n up to kGatherRowMax): the full
// symmetric H is written out from its upper triangle (32 x 32 tiles through shared
// memory) into a scratch matrix S, then each row i of A takes row q(i) of S staged in
// shared memory, A[i][j] = S[q(i)][q(j)] for j < i.  (prep_gather_kernel reads H
// element by element at permuted positions instead.)
constexpr int kGatherRowMax = 48 * 1024;   // floats of one staged row (192 KB of shared memory)

__global__ void prep_symmetrize_kernel(const float* H, int n, float* Sm, int lds, const int32_t* st) {
  if (has_error(st)) return;
  __shared__ float t[32][33];
  const int bi = blockIdx.y, bj = blockIdx.x;                 // output tile (bi, bj) of S
  const int ti = min(bi, bj), tj = max(bi, bj);               // the upper tile of H it comes from
  for (int yy = threadIdx.y; yy < 32; yy += 8) {
    const int r = ti * 32 + yy, c = tj * 32 + threadIdx.x;
    t[yy][threadIdx.x] = (r < n && c < n) ? H[(int64_t)r * n + c] : 0.f;
  }
  __syncthreads();
  for (int yy = threadIdx.y; yy < 32; yy += 8) {
    const int r = bi * 32 + yy, c = bj * 32 + threadIdx.x;
    if (r >= n || c >= n) continue;
    float v;
    if (bi < bj) v = t[yy][threadIdx.x];
    else if (bi > bj) v = t[threadIdx.x][yy];
    else v = yy <= (int)threadIdx.x ? t[yy][threadIdx.x] : t[threadIdx.x][yy];   // the diagonal tile
    Sm[(int64_t)r * lds + c] = v;
  }
}

__global__ void __launch_bounds__(256) prep_gather_rows_kernel(const float* Sm, int lds, const float* dfix,
                                                              const int32_t* perm, int n, int ldn,
                                                              const double* scal, float* A, int32_t* st) {
  if (has_error(st)) return;
  extern __shared__ float srow[];
  const int i = blockIdx.x;
  const int a = perm[n - 1 - i];
  const float* src = Sm + (int64_t)a * lds;
  for (int c = threadIdx.x; c < n; c += blockDim.x) srow[c] = src[c];
  __syncthreads();
  float* dst = A + (int64_t)i * ldn;
  bool bad = false;
  for (int j = threadIdx.x; j <= i; j += blockDim.x) {
    float v;
    if (j == i) {
      v = (float)((double)dfix[a] + scal[1]);
    } else {
      v = srow[perm[n - 1 - j]];
      bad = bad || !isfinite(v);
    }
    dst[j] = v;
  }
  if (bad) set_error(st, GPTQ_ERR_NONFINITE, n - 1 - i, STAGE_PREP_DIAG);
}

__global__ void __launch_bounds__(256) prep_reverse_kernel(const float* H, const float* dfix, int n, int ldn,
                                                           const double* scal, float* A, int32_t* st) {
  if (has_error(st)) return;
  const int i = blockIdx.x;
  const float* h = H + (int64_t)(n - 1 - i) * n + (n - 1);   // h[-j] = H[n-1-i][n-1-j]
  float* a = A + (int64_t)i * ldn;
  const float diag = (float)((double)dfix[n - 1 - i] + scal[1]);
  bool bad = false;
  for (int j = 4 * threadIdx.x; j <= i; j += 4 * 256) {
    float v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int jj = j + u;
      v[u] = jj < i ? h[-jj] : (jj == i ? diag : 0.f);
      bad = bad || (jj < i && !isfinite(v[u]));
    }
    *reinterpret_cast<float4*>(a + j) = make_float4(v[0], v[1], v[2], v[3]);
  }
  if (bad) set_error(st, GPTQ_ERR_NONFINITE, n - 1 - i, STAGE_PREP_DIAG);
}

// (4'') Xt starts at zero right of its 128-wide block diagonal, where the blocked
// inverse accumulates; its diagonal blocks are written whole and nothing reads
// below them.
__global__ void zero_upper_blocks_kernel(float* Xt, int n, int ldn) {
  const int r = blockIdx.x;
  const int c0 = (r / PB + 1) * PB;
  float* row = Xt + (int64_t)r * ldn;
  for (int c = c0 + 4 * (int)threadIdx.x; c < n; c += 4 * (int)blockDim.x)
    *reinterpret_cast<float4*>(row + c) = make_float4(0.f, 0.f, 0.f, 0.f);
}

// ---------------------------------------------------------------------------
// (5) The diagonal block of panel k: Cholesky L_kk and its inverse T = L_kk^-1
// (rows/columns past nb padded with the identity), blocked by 32-wide
// sub-blocks q = 32p, p = 0..3, with the block and its inverse in shared memory:
//   A  one warp factors the 32 x 32 diagonal sub-block (lane i keeps row i).  At
//      pivot j the column j of L goes through a shared buffer (kept: it is also
//      the operand of the triangular solves) and updates the later columns; the
//      next pivot is derived by its own lane and broadcast before that update, so
//      its reciprocal square root overlaps it.
//   B  forward substitution with L_pp, one right-hand side per lane: the rows of
//      L21 = A21 . L_pp^-T (in place, and into a scratch panel) and the columns
//      of T_pp = L_pp^-1; next to it Y = L[p, 0:q] . T[0:q, 0:q].
//   C  A22 -= L21 . L21^T (lower block triangle) and T[p, 0:q] = -T_pp . Y
//      (L T = I gives L_pp T_pr = -sum_{r<=m<p} L_pm T_mr).
// The products of B and C run on mma.sync (m16n8k8, TF32) with every operand
// split into hi + lo and three products (hi.hi + hi.lo + lo.hi), fp32-level
// accuracy; one warp computes one 16 x 32 tile.
// ---------------------------------------------------------------------------
constexpr int DT = 384;            // threads (12 warps)
constexpr int NWARP = DT / 32;
constexpr int LDL = 132;           // row stride (floats) of the L and T stages
constexpr int LDY = 104;           // row stride of Y
constexpr int LDP = 36;            // row stride of the scratch panel
constexpr int OPND_BYTES = 131072;  // the prologue's tensor-core operand tiles (then the T stage)
constexpr int OFF_T = 0;
constexpr int OFF_L = OPND_BYTES / 4;
constexpr int OFF_Y = OFF_L + PB * LDL;
constexpr int OFF_P = OFF_Y + 32 * LDY;
constexpr int OFF_C = OFF_P + (PB - 32) * LDP;
constexpr int OFF_R = OFF_C + 32 * 32;
static_assert(PB * LDL <= OFF_L, "the T stage fits in the operand area");
// + 1024: the base is rounded up to the 1024-byte alignment of the swizzled tiles
constexpr size_t POTRF_SMEM = (size_t)(OFF_R + PB) * sizeof(float) + 1024;

__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
  hi = __float_as_uint(x) & 0xFFFFE000u;
  lo = __float_as_uint(x - __uint_as_float(hi));
}

__device__ __forceinline__ void mma_m16n8k8_tf32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// acc (16 x 32, fragment layout) += A (16 x K) . B (K x 32):
//   A(r, k) = A[r * lda + k];  B(k, n) = B[k * ldb + n] (NN) or B[n * ldb + k] (NT).
// acc[s][e] holds the element (g + 8 (e >> 1), 8 s + 2 t + (e & 1)), g = lane / 4, t = lane % 4.
template <bool NN>
__device__ __forceinline__ void mma_tile_16x32(const float* A, int lda, const float* B, int ldb, int K, int lane,
                                               float (&acc)[4][4]) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll 1
  for (int k0 = 0; k0 < K; k0 += 8) {
    uint32_t ah[4], al[4];
    split_tf32(A[g * lda + k0 + t], ah[0], al[0]);
    split_tf32(A[(g + 8) * lda + k0 + t], ah[1], al[1]);
    split_tf32(A[g * lda + k0 + t + 4], ah[2], al[2]);
    split_tf32(A[(g + 8) * lda + k0 + t + 4], ah[3], al[3]);
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const float x0 = NN ? B[(k0 + t) * ldb + 8 * s + g] : B[(8 * s + g) * ldb + k0 + t];
      const float x1 = NN ? B[(k0 + t + 4) * ldb + 8 * s + g] : B[(8 * s + g) * ldb + k0 + t + 4];
      uint32_t bh0, bl0, bh1, bl1;
      split_tf32(x0, bh0, bl0);
      split_tf32(x1, bh1, bl1);
      mma_m16n8k8_tf32(acc[s], al, bh0, bh1);
      mma_m16n8k8_tf32(acc[s], ah, bl0, bl1);
      mma_m16n8k8_tf32(acc[s], ah, bh0, bh1);
    }
  }
}

// Phase A: Cholesky of the 32 x 32 sub-block at (q, q).  One warp.  The factor
// is kept as Cs[j][k] = L_kj (k > j, else 0) and Rv[j] = 1 / L_jj, the operands
// of phase B; L_jj itself is never needed.  1 / L_jj is the hardware reciprocal
// square root of the pivot (a few ulp); every later use takes that same value,
// so the factor stays consistent and the backward error stays at the fp32
// rounding level.
// *bad receives the first failing pivot (or -1), *bad_nan its kind.
__device__ __forceinline__ void chol32(const float* Ls, float* Cs, float* Rv, int q, int lane, int* bad, int* bad_nan) {
  float a[32];
  const float* row = Ls + (q + lane) * LDL + q;
#pragma unroll
  for (int k = 0; k < 32; k += 4) {
    const float4 v = *reinterpret_cast<const float4*>(row + k);
    a[k] = k <= lane ? v.x : 0.f;
    a[k + 1] = k + 1 <= lane ? v.y : 0.f;
    a[k + 2] = k + 2 <= lane ? v.z : 0.f;
    a[k + 3] = k + 3 <= lane ? v.w : 0.f;
  }
  // A failing pivot gets 1 / L_jj = 1, which keeps the arithmetic finite (every
  // later stage sees the error and skips); lane j keeps pivot j as it came.
  float mine = 1.f;
  auto inv_root = [&](float d, int j) {
    if (lane == j) mine = d;
    const float y = rsqrtf(d);
    return (d > 0.f && isfinite(d)) ? y : 1.f;
  };
  float y = inv_root(__shfl_sync(0xffffffffu, a[0], 0), 0);
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const float lij = lane > j ? a[j] * y : 0.f;
    a[j] = lij;
    Cs[j * 32 + lane] = lane > j ? lij : 0.f;
    if (lane == j) Rv[j] = y;
    // lane j + 1 holds the next pivot once this column's term is removed
    float dn = j + 1 < 32 ? __shfl_sync(0xffffffffu, fmaf(-lij, lij, a[(j + 1) & 31]), (j + 1) & 31) : 1.f;
    __syncwarp();
    float4 c4[8];
#pragma unroll
    for (int k4 = (j + 1) & ~3; k4 < 32; k4 += 4) c4[k4 / 4] = *reinterpret_cast<const float4*>(Cs + j * 32 + k4);
    const float yn = j + 1 < 32 ? inv_root(dn, j + 1) : 1.f;
#pragma unroll
    for (int k4 = (j + 1) & ~3; k4 < 32; k4 += 4) {
      const float cc[4] = {c4[k4 / 4].x, c4[k4 / 4].y, c4[k4 / 4].z, c4[k4 / 4].w};
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (k4 + u > j) a[k4 + u] = fmaf(-lij, cc[u], a[k4 + u]);
    }
    y = yn;
  }
  const uint32_t badm = __ballot_sync(0xffffffffu, !(mine > 0.f && isfinite(mine)));
  const uint32_t nanm = __ballot_sync(0xffffffffu, !isfinite(mine));
  *bad = badm ? __ffs(badm) - 1 : -1;
  *bad_nan = badm ? (int)((nanm >> (__ffs(badm) - 1)) & 1u) : 0;
}

// x = L_pp^-1 b for one right-hand side per lane: x_j = b_j / L_jj, then
// b_k -= L_kj x_j for k > j (column j of L_pp from Cs).  b is overwritten by x.
__device__ __forceinline__ void fwd_subst32(const float* Cs, const float* Rv, float (&b)[32]) {
  float4 cur[8], nxt[8];
  float rcur = Rv[0], rnxt = 1.f;
#pragma unroll
  for (int k4 = 0; k4 < 32; k4 += 4) cur[k4 / 4] = *reinterpret_cast<const float4*>(Cs + k4);
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    if (j + 1 < 32) {   // the next column, one step ahead
      rnxt = Rv[(j + 1) & 31];
#pragma unroll
      for (int k4 = (j + 2) & ~3; k4 < 32; k4 += 4)
        nxt[k4 / 4] = *reinterpret_cast<const float4*>(Cs + ((j + 1) & 31) * 32 + k4);
    }
    b[j] *= rcur;
#pragma unroll
    for (int k4 = (j + 1) & ~3; k4 < 32; k4 += 4) {
      const float cc[4] = {cur[k4 / 4].x, cur[k4 / 4].y, cur[k4 / 4].z, cur[k4 / 4].w};
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (k4 + u > j) b[k4 + u] = fmaf(-cc[u], b[j], b[k4 + u]);
    }
#pragma unroll
    for (int k4 = 0; k4 < 32; k4 += 4) cur[k4 / 4] = nxt[k4 / 4];
    rcur = rnxt;
  }
}

// Tensor-core operand tiles: 128 rows x 32 fp32 (128-byte rows) in the
// 128-byte-swizzled K-major layout, 16-byte piece j of row r at r * 128 + ((j ^ (r & 7)) << 4).
__device__ __forceinline__ void sw_store4(uint8_t* tile, int r, int j, float4 v) {
  *reinterpret_cast<float4*>(tile + r * 128 + ((j ^ (r & 7)) << 4)) = v;
}

__device__ __forceinline__ void split4(float4 x, float4& h, float4& l) {
  h = make_float4(tf32_hi(x.x), tf32_hi(x.y), tf32_hi(x.z), tf32_hi(x.w));
  l = make_float4(x.x - h.x, x.y - h.y, x.z - h.z, x.w - h.w);
}

// D[tmem] (+)= A . B^T over one 32-wide K chunk in 3 x TF32 (128 x 128, K = 8 steps).
__device__ __forceinline__ void mma_chunk_3x(uint32_t d, uint32_t ah, uint32_t al, uint32_t bh, uint32_t bl,
                                             bool accumulate) {
  constexpr uint32_t IDESC = tc::idesc_f32acc(2, 128, 128);
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    const uint32_t o = kk * 32;
    tc::mma_tf32(d, tc::sdesc_k_sw128(al + o), tc::sdesc_k_sw128(bh + o), IDESC, accumulate || kk > 0);
    tc::mma_tf32(d, tc::sdesc_k_sw128(ah + o), tc::sdesc_k_sw128(bl + o), IDESC, true);
    tc::mma_tf32(d, tc::sdesc_k_sw128(ah + o), tc::sdesc_k_sw128(bh + o), IDESC, true);
  }
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Lower-triangular 16 x 32 tiles of a 128 x 128 result: row tile rt (16 rows),
// column chunk ch <= rt / 2 (32 columns); 20 tiles in all.
__device__ __forceinline__ void lower_tile(int task, int& rt, int& ch) {
  rt = 0;
  while (task >= rt / 2 + 1) { task -= rt / 2 + 1; ++rt; }
  ch = task;
}

// D (lower triangle of block (k, k), identity past nb) into a stage.
__device__ __forceinline__ void load_diag_block(const float* A, int lda, int k0, int nb, float* D, int tid) {
  for (int idx = tid; idx < PB * PB / 4; idx += DT) {
    const int r = idx / (PB / 4), c = 4 * (idx % (PB / 4));
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r < nb && c <= r) v = *reinterpret_cast<const float4*>(A + (int64_t)(k0 + r) * lda + k0 + c);
    float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (c + u > r) e[u] = 0.f;
      if (r >= nb && r == c + u) e[u] = 1.f;
    }
    *reinterpret_cast<float4*>(D + r * LDL + c) = make_float4(e[0], e[1], e[2], e[3]);
  }
}

// kp < 0: the first panel; D = A[k0.., k0..] is final.
// kp >= 0: the previous panel (columns kp .. kp + PB) has its inverse T' = Tphi + Tplo,
// and A[k0.., k0..] lacks only that panel's term.  The kernel first forms
// L(k, k-1) = A(k, k-1) . T'^T and D -= L(k, k-1) . L(k, k-1)^T itself, on the
// tensor cores (tcgen05, 3 x TF32, accumulators in TMEM), so that the chain of
// diagonal blocks is one launch per panel; the other rows of L21 and their
// updates run off this chain.
__global__ void __launch_bounds__(DT, 1)
potrf_inv_kernel(const float* A, int lda, int k0, int nb, int n, const float* Tphi, const float* Tplo, int kp,
                 float* LIhi, float* LIlo, int32_t* st) {
  extern __shared__ __align__(1024) uint8_t sm_raw[];
  // offset arithmetic on the shared array keeps every access a shared-memory one
  uint8_t* base = sm_raw + ((1024u - (tc::smem_u32(sm_raw) & 1023u)) & 1023u);
  float* sm = reinterpret_cast<float*>(base);
  float* Ls = sm + OFF_L;
  float* Ts = sm + OFF_T;
  float* Ys = sm + OFF_Y;
  float* Ps = sm + OFF_P;
  float* Cs = sm + OFF_C;
  float* Rv = sm + OFF_R;
  __shared__ int bad;
  __shared__ uint64_t pbar[6];   // operand buffers of the two products (2 + 2), accumulator complete, drain
  __shared__ uint32_t tmem_base;
  __shared__ int pfail;
  if (has_error(st)) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t4 = lane & 3;
  if (tid == 0) bad = 0;

  // The prologue's operands move in chunks of 32 columns; each thread moves (up to)
  // PF pieces of each operand per chunk, and the next chunk's loads are in flight
  // while a chunk is stored and multiplied.  The first chunk's loads go out before
  // the diagonal block's, so that the two latencies overlap.
  constexpr int PF = (PB * 8 + DT - 1) / DT;
  float4 pa[PF], ph[PF], pl[PF];
  auto fetch_a = [&](int kc) {
#pragma unroll
    for (int u = 0; u < PF; ++u) {
      const int idx = tid + u * DT;
      const int r = idx >> 3, c = kc * 32 + 4 * (idx & 7);
      pa[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (idx < PB * 8 && r < nb) pa[u] = *reinterpret_cast<const float4*>(A + (int64_t)(k0 + r) * lda + kp + c);
    }
  };
  auto fetch_t = [&](int kc) {
#pragma unroll
    for (int u = 0; u < PF; ++u) {
      const int idx = tid + u * DT;
      const int r = idx >> 3, c = kc * 32 + 4 * (idx & 7);
      ph[u] = pl[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (idx < PB * 8) {
        ph[u] = *reinterpret_cast<const float4*>(Tphi + r * PB + c);
        pl[u] = *reinterpret_cast<const float4*>(Tplo + r * PB + c);
      }
    }
  };
  // Consecutive launches of the chain are programmatic dependents (launch_potrf_inv): the
  // next panel's kernel may start once this one has begun and issue what the other streams'
  // kernels produced (its diagonal block, A(k, k-1)), which are complete when it starts.
  // T' = L_{k-1,k-1}^-1, the previous launch's output, is read only after
  // griddepcontrol.wait, which returns once the previous launch has completed and its
  // writes are visible.  (Launched without the attribute, both instructions do nothing.)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (kp >= 0) fetch_a(0);
  // The diagonal block: for a full panel, 16-byte asynchronous copies that land while the
  // prologue's products run (the block is first read after them).  Its upper triangle is
  // copied as it lies in A (never written there): every reader of the block masks or
  // skips it (the Cholesky keeps k <= row; the solves and products read the lower part).
  // A partial last panel takes the masked load with the identity past nb.
  const bool async_diag = nb == PB && (lda & 3) == 0;
  if (async_diag) {
    for (int idx = tid; idx < PB * PB / 4; idx += DT) {
      const int r = idx / (PB / 4), c = 4 * (idx % (PB / 4));
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(tc::smem_u32(Ls + r * LDL + c)),
                   "l"(A + (int64_t)(k0 + r) * lda + k0 + c)
                   : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  } else {
    load_diag_block(A, lda, k0, nb, Ls, tid);
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (kp >= 0) fetch_t(0);
  if (kp >= 0) {
    if (tid == 0) {
      for (int i = 0; i < 6; ++i) tc::mbar_init(&pbar[i], 1);
      tc::fence_barrier_init();
      pfail = 0;
    }
    if (warp == 0) tc::tmem_alloc<256>(&tmem_base);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tm = tmem_base;
    volatile int* fail = &pfail;
    uint32_t done_parity = 0;
    auto wait_bar = [&](uint64_t* bar, uint32_t parity) {   // thread 0 only
      if (!*fail && !tc::mbar_wait(bar, parity, fail)) *fail = 1;
    };
    // ---- L(k, k-1) = A(k, k-1) . T'^T into TMEM columns [0, 128), by 32-wide K chunks
    // through two 64 KB operand buffers (A hi, A lo, T' hi, T' lo) ----
    for (int kc = 0; kc < 4; ++kc) {
      const int bf = kc & 1;
      uint8_t* ob = base + bf * 65536;
      if (kc >= 2) {                         // chunk kc - 2's products read this buffer
        if (tid == 0) wait_bar(&pbar[bf], 0);
        __syncthreads();
      }
#pragma unroll
      for (int u = 0; u < PF; ++u) {
        const int idx = tid + u * DT;
        if (idx < PB * 8) {
          const int r = idx >> 3, j = idx & 7;
          float4 ah, al;
          split4(pa[u], ah, al);
          sw_store4(ob, r, j, ah);
          sw_store4(ob + 16384, r, j, al);
          sw_store4(ob + 32768, r, j, ph[u]);
          sw_store4(ob + 49152, r, j, pl[u]);
        }
      }
      if (kc + 1 < 4) {
        fetch_a(kc + 1);
        fetch_t(kc + 1);
      }
      fence_proxy_async();
      __syncthreads();
      if (tid == 0 && !*fail) {
        tc::tc_fence_after();
        const uint32_t o = tc::smem_u32(ob);
        mma_chunk_3x(tm, o, o + 16384, o + 32768, o + 49152, kc > 0);
        tc::mma_commit(&pbar[bf]);
      }
    }
    if (tid == 0) {
      if (!*fail) tc::mma_commit(&pbar[4]);
      wait_bar(&pbar[4], done_parity);
      done_parity ^= 1;
    }
    __syncthreads();
    tc::tc_fence_after();
    // ---- D -= L . L^T into TMEM columns [128, 256): L leaves TMEM by 32-column chunks,
    // split into one tile pair (hi, lo) that is both operands ----
    for (int kc = 0; kc < 4; ++kc) {
      const int bf = kc & 1;
      uint8_t* lb = base + bf * 32768;
      if (kc >= 2) {
        if (tid == 0) wait_bar(&pbar[2 + bf], 0);
        __syncthreads();
      }
      if (warp < 4 && !*fail) {
        float v[32];
        tc::tmem_ld_32x32b_x32(tm + ((uint32_t)(warp * 32) << 16) + kc * 32, v);
        const int r = warp * 32 + lane;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          float4 h, l;
          split4(make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]), h, l);
          sw_store4(lb, r, j, h);
          sw_store4(lb + 16384, r, j, l);
        }
      }
      fence_proxy_async();
      tc::tc_fence_before();
      __syncthreads();
      if (tid == 0 && !*fail) {
        tc::tc_fence_after();
        const uint32_t o = tc::smem_u32(lb);
        mma_chunk_3x(tm + 128, o, o + 16384, o, o + 16384, kc > 0);
        tc::mma_commit(&pbar[2 + bf]);
      }
    }
    if (tid == 0) {
      if (!*fail) tc::mma_commit(&pbar[4]);
      wait_bar(&pbar[4], done_parity);
    }
    asm volatile("cp.async.wait_all;" ::: "memory");   // this thread's copies of the diagonal block
    __syncthreads();
    tc::tc_fence_after();
    if (warp < 4 && !*fail) {
      const int r = warp * 32 + lane;
#pragma unroll 1
      for (int c0 = 0; c0 < PB; c0 += 32) {
        float v[32];
        tc::tmem_ld_32x32b_x32(tm + ((uint32_t)(warp * 32) << 16) + 128 + c0, v);
        float* d = Ls + r * LDL + c0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          float4 x = *reinterpret_cast<float4*>(d + 4 * j);
          x.x -= v[4 * j]; x.y -= v[4 * j + 1]; x.z -= v[4 * j + 2]; x.w -= v[4 * j + 3];
          *reinterpret_cast<float4*>(d + 4 * j) = x;
        }
      }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (*fail && tid == 0) {
      // a wait gave up: let whatever was issued finish (bounded) before TMEM goes back
      tc::mma_commit(&pbar[5]);
      const uint64_t t0 = tc::globaltimer();
      while (!tc::mbar_try_wait(&pbar[5], 0) && tc::globaltimer() - t0 < 1000000000ull) {
      }
      set_error(st, GPTQ_ERR_TIMEOUT, n - 1 - k0, STAGE_POTRF);
    }
    __syncthreads();
    if (warp == 0) {
      __syncwarp();
      tc::tmem_dealloc<256>(tm);
    }
    if (*fail) return;
  }
  asm volatile("cp.async.wait_all;" ::: "memory");     // (the first panel's block: no prologue)
  // T starts at zero
  for (int idx = tid; idx < PB * PB / 4; idx += DT) {
    const int r = idx / (PB / 4), c = 4 * (idx % (PB / 4));
    *reinterpret_cast<float4*>(Ts + r * LDL + c) = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  __syncthreads();
  GPTQ_PHASE_MARK(0);

  // The factor-and-invert loop over the four 32-column sub-blocks (q = 32 p):
  //   A  warp 0 factors the diagonal tile (the one-warp Cholesky).  Meanwhile the other
  //      warps finish sub-block p - 1: its trailing tiles below the next diagonal tile,
  //      its rows of T (T[q - 32 + a][c] = -T_pp Y), and they write out the split of
  //      sub-block p - 2's rows of T, final since.
  //   B  the rows below by forward substitution (into L and the scratch panel), T_pp,
  //      and Y = L(p, :q) T(:q, :q).
  //   C  the next diagonal tile's update (two 16 x 32 tiles), all that A of the next
  //      sub-block reads.
  // Lower 16 x 32 tiles of the trailing block of the sub-block at q: row tile rt
  // (16 rows), column chunk ch <= rt / 2; tasks 0 and 1 are the next diagonal tile.
  auto trail_task = [&](int q, int task) {
    int rt = 0, rem = task;
    while (rem >= rt / 2 + 1) { rem -= rt / 2 + 1; ++rt; }
    const int ch = rem;
    float acc[4][4] = {};
    mma_tile_16x32<false>(Ps + 16 * rt * LDP, LDP, Ps + 32 * ch * LDP, LDP, 32, lane, acc);
    const int i0 = q + 32 + 16 * rt, c0 = q + 32 + 32 * ch;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      float2* e0 = reinterpret_cast<float2*>(Ls + (i0 + g) * LDL + c0 + 8 * s + 2 * t4);
      float2* e1 = reinterpret_cast<float2*>(Ls + (i0 + g + 8) * LDL + c0 + 8 * s + 2 * t4);
      float2 v0 = *e0, v1 = *e1;
      v0.x -= acc[s][0]; v0.y -= acc[s][1]; v1.x -= acc[s][2]; v1.y -= acc[s][3];
      *e0 = v0; *e1 = v1;
    }
  };
  auto trail_tasks = [](int q) {
    const int rt_n = (PB - q - 32) / 16;
    int ntc = 0;
    for (int rt = 0; rt < rt_n; ++rt) ntc += rt / 2 + 1;
    return ntc;
  };
  // T[q + a][c] = -sum_b T_pp[a][b] Y[b][c] (T_pp[a][b] = 0 for b > a), rows a0 .. a0 + 16,
  // columns 32 ch ..
  auto t_task = [&](int q, int u) {
    const int a0 = 16 * (u & 1), ch = u >> 1;
    float acc[4][4] = {};
    mma_tile_16x32<true>(Ts + (q + a0) * LDL + q, LDL, Ys + 32 * ch, LDY, a0 + 16, lane, acc);
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      float* t0 = Ts + (q + a0 + g) * LDL + 32 * ch + 8 * s + 2 * t4;
      *reinterpret_cast<float2*>(t0) = make_float2(-acc[s][0], -acc[s][1]);
      *reinterpret_cast<float2*>(t0 + 8 * LDL) = make_float2(-acc[s][2], -acc[s][3]);
    }
  };
  // the TF32 split of T's rows r0 .. r0 + 32 (L_kk itself is not needed later: the
  // trailing steps use L21 and T; the block of Xt comes from this split, off this chain)
  auto write_rows = [&](int r0, int first, int stride) {
#pragma unroll 4
    for (int idx = first; idx < 32 * PB / 4; idx += stride) {
      const int i = r0 + idx / (PB / 4), k = 4 * (idx % (PB / 4));
      const float4 v = *reinterpret_cast<const float4*>(Ts + i * LDL + k);
      float e[4] = {v.x, v.y, v.z, v.w}, h[4], l[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (i >= nb || k + u >= nb) e[u] = 0.f;
        h[u] = tf32_hi(e[u]);
        l[u] = e[u] - h[u];
      }
      *reinterpret_cast<float4*>(LIhi + i * PB + k) = make_float4(h[0], h[1], h[2], h[3]);
      *reinterpret_cast<float4*>(LIlo + i * PB + k) = make_float4(l[0], l[1], l[2], l[3]);
    }
  };

#pragma unroll 1
  for (int p = 0; p < 4; ++p) {
    const int q = 32 * p;
    const int R = PB - q - 32;          // rows below the sub-block
    // ---- A (and the rest of sub-block p - 1) ----
    if (warp == 0) {
      int bj, bn;
      chol32(Ls, Cs, Rv + q, q, lane, &bj, &bn);
      if (bj >= 0 && lane == 0 && !bad) {
        bad = 1;
        set_error(st, bn ? GPTQ_ERR_NONFINITE : GPTQ_ERR_NOT_SPD, n - 1 - (k0 + q + bj), STAGE_POTRF);
      }
    } else if (p > 0) {
      const int qp = q - 32;
      const int nrest = trail_tasks(qp) - 2;
#pragma unroll 1
      for (int task = warp - 1; task < nrest + 2 * (p - 1); task += NWARP - 1) {
        if (task < nrest) trail_task(qp, task + 2);
        else t_task(qp, task - nrest);
      }
      if (p > 1) write_rows(q - 64, tid - 32, DT - 32);
    }
    __syncthreads();
    GPTQ_PHASE_MARK(1 + 3 * p);
    // ---- B ----
    const int wl = R / 32;              // warps on the rows of L21
    if (warp < wl) {
      const int i = q + 32 + 32 * warp + lane;
      float* row = Ls + i * LDL + q;
      float b[32];
#pragma unroll
      for (int k = 0; k < 32; k += 4) {
        const float4 v = *reinterpret_cast<const float4*>(row + k);
        b[k] = v.x; b[k + 1] = v.y; b[k + 2] = v.z; b[k + 3] = v.w;
      }
      fwd_subst32(Cs, Rv + q, b);
      float* prow = Ps + (i - q - 32) * LDP;
#pragma unroll
      for (int k = 0; k < 32; k += 4) {
        const float4 v = make_float4(b[k], b[k + 1], b[k + 2], b[k + 3]);
        *reinterpret_cast<float4*>(row + k) = v;
        *reinterpret_cast<float4*>(prow + k) = v;
      }
    } else if (warp == wl) {
      float b[32];
#pragma unroll
      for (int k = 0; k < 32; ++k) b[k] = k == lane ? 1.f : 0.f;
      fwd_subst32(Cs, Rv + q, b);
#pragma unroll
      for (int k = 0; k < 32; ++k) Ts[(q + k) * LDL + q + lane] = b[k];
    } else if (warp - wl - 1 < 2 * p) {
      // Y rows a0..a0+15, columns 32 ch..: T[m][c] = 0 for m < 32 ch
      const int u = warp - wl - 1;
      const int a0 = 16 * (u & 1), ch = u >> 1;
      float acc[4][4] = {};
      mma_tile_16x32<true>(Ls + (q + a0) * LDL + 32 * ch, LDL, Ts + 32 * ch * LDL + 32 * ch, LDL, q - 32 * ch, lane,
                           acc);
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        float* y0 = Ys + (a0 + g) * LDY + 32 * ch + 8 * s + 2 * t4;
        *reinterpret_cast<float2*>(y0) = make_float2(acc[s][0], acc[s][1]);
        *reinterpret_cast<float2*>(y0 + 8 * LDY) = make_float2(acc[s][2], acc[s][3]);
      }
    }
    __syncthreads();
    GPTQ_PHASE_MARK(2 + 3 * p);
    // ---- C: the next diagonal tile ----
    if (R > 0 && warp < 2) trail_task(q, warp);
    __syncthreads();
    GPTQ_PHASE_MARK(3 + 3 * p);
  }
  // the last sub-block's rows of T, sub-block 2's rows written out meanwhile
  if (warp < 6) t_task(96, warp);
  else write_rows(64, tid - 192, DT - 192);
  __syncthreads();
  if (bad) return;
  write_rows(96, tid, DT);
  GPTQ_PHASE_MARK(13);
}

// (5b) The diagonal block of Xt = (L^-1)^T and the last nb rows of its split XQ,
// from the split of T = L_kk^-1: Xt[k0 + k][k0 + i] = T[i][k] (hi + lo is exact),
// XQ[k0 + k][i] = (hi, lo)(T[i][k]) (row stride ldq).  32 x 32 tiles through shared memory.
__global__ void xt_diag_kernel(const float* LIhi, const float* LIlo, int k0, int nb, float* Xt, int ldx, float* XQhi,
                               float* XQlo, int ldq, const int32_t* st) {
  if (has_error(st)) return;
  __shared__ float th[32][33], tl[32][33];
  const int i0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
  for (int yy = threadIdx.y; yy < 32; yy += 8) {
    th[yy][threadIdx.x] = LIhi[(i0 + yy) * PB + c0 + threadIdx.x];
    tl[yy][threadIdx.x] = LIlo[(i0 + yy) * PB + c0 + threadIdx.x];
  }
  __syncthreads();
  for (int yy = threadIdx.y; yy < 32; yy += 8) {
    const int k = c0 + yy, i = i0 + threadIdx.x;
    if (k >= nb) continue;
    const float h = th[threadIdx.x][yy], l = tl[threadIdx.x][yy];
    if (i < nb) Xt[(int64_t)(k0 + k) * ldx + k0 + i] = h + l;
    XQhi[(int64_t)(k0 + k) * ldq + i] = h;
    XQlo[(int64_t)(k0 + k) * ldq + i] = l;
  }
}

// (6) U[i][j] = (L^-1)[n-1-i][n-1-j] = Xt[n-1-j][n-1-i] for j >= i, 0 below the diagonal.
// 64 x 64 tiles through shared memory (64 x 4 threads, 16 entries each); tiles
// wholly below the diagonal only write zeros.
__global__ void __launch_bounds__(256) write_u_kernel(const float* Xt, int n, int ldx, float* U,
                                                      const int32_t* st) {
  if (has_error(st)) return;
  __shared__ float t[64][65];
  const int i0 = blockIdx.y * 64, j0 = blockIdx.x * 64;
  const int tx = threadIdx.x, ty = threadIdx.y;
  if (j0 + 63 < i0) {
#pragma unroll 4
    for (int yy = ty; yy < 64; yy += 4) {
      const int i = i0 + yy, j = j0 + tx;
      if (i < n && j < n) U[(int64_t)i * n + j] = 0.f;
    }
    return;
  }
#pragma unroll 4
  for (int yy = ty; yy < 64; yy += 4) {
    const int j = j0 + yy, i = i0 + tx;
    t[yy][tx] = (i < n && j < n && j >= i) ? Xt[(int64_t)(n - 1 - j) * ldx + (n - 1 - i)] : 0.f;
  }
  __syncthreads();
#pragma unroll 4
  for (int yy = ty; yy < 64; yy += 4) {
    const int i = i0 + yy, j = j0 + tx;
    if (i < n && j < n) U[(int64_t)i * n + j] = t[tx][yy];
  }
}

// One launch of the diagonal-block chain, as a programmatic dependent of the previous
// launch on its stream (the kernel orders its reads of the previous launch's output).
int launch_potrf_inv(const PrepWs& w, int ldn, int k0, int nb, int n, int b1, int kp, int b, int32_t* st,
                     cudaStream_t c) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(DT);
  cfg.dynamicSmemBytes = POTRF_SMEM;
  cfg.stream = c;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  GPTQ_CUDA_TRY(cudaLaunchKernelEx(&cfg, potrf_inv_kernel, (const float*)w.A, ldn, k0, nb, n,
                                   (const float*)w.LIhi[b1], (const float*)w.LIlo[b1], kp, w.LIhi[b], w.LIlo[b], st));
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

// The panel loop runs on four streams.// The panel loop runs on four streams.  High priority, so that their small
// launches get SMs ahead of the bulk work: the chain of diagonal blocks (one
// launch per panel), and the rest of each panel's factorization (all rows of
// L21, and the update of the next block column below its diagonal block).  Low
// priority: the trailing updates beyond the next block column, and the blocked
// inverse.  Streams and events exist once per host thread and device, created
// on first use and kept for the life of the process.
struct AuxStream {
  cudaStream_t c = nullptr;    // diagonal blocks
  cudaStream_t o = nullptr;    // L21 and the next block column
  cudaStream_t t = nullptr;    // trailing updates
  cudaStream_t s = nullptr;    // the inverse
  cudaEvent_t fork = nullptr, join[4] = {};
  // per panel (ring slot): diagonal block done, L21 split ready, next block column
  // updated, trailing update done, inverse done with the panel's buffers
  cudaEvent_t diag[NLI] = {}, l21[NLI] = {}, next[NLI] = {}, trail[NLI] = {}, done[NLI] = {};
  // per super-panel (deferred loop): its L21 complete, the next super-panel's block
  // column updated, the bulk trailing update done, the bulk inverse update done
  cudaEvent_t lsup[NSUP] = {}, col[NSUP] = {}, bulk[NSUP] = {}, inv[NSUP] = {};
};

int aux_stream(AuxStream** out) {
  // one set per host thread and device, so concurrent callers never share it
  thread_local AuxStream per_dev[64];
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return GPTQ_ERR_CUDA;
  AuxStream& a = per_dev[dev];
  if (a.s == nullptr) {
    int least = 0, greatest = 0;
    if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess) return GPTQ_ERR_CUDA;
    if (cudaStreamCreateWithPriority(&a.c, cudaStreamNonBlocking, greatest) != cudaSuccess ||
        cudaStreamCreateWithPriority(&a.o, cudaStreamNonBlocking, greatest) != cudaSuccess ||
        cudaStreamCreateWithPriority(&a.t, cudaStreamNonBlocking, least) != cudaSuccess ||
        cudaStreamCreateWithPriority(&a.s, cudaStreamNonBlocking, least) != cudaSuccess)
      return GPTQ_ERR_CUDA;
    const unsigned f = cudaEventDisableTiming;
    if (cudaEventCreateWithFlags(&a.fork, f) != cudaSuccess) return GPTQ_ERR_CUDA;
    for (cudaEvent_t& e : a.join)
      if (cudaEventCreateWithFlags(&e, f) != cudaSuccess) return GPTQ_ERR_CUDA;
    for (int b = 0; b < NLI; ++b) {
      cudaEvent_t* evs[] = {&a.diag[b], &a.l21[b], &a.next[b], &a.trail[b], &a.done[b]};
      for (cudaEvent_t* e : evs)
        if (cudaEventCreateWithFlags(e, f) != cudaSuccess) return GPTQ_ERR_CUDA;
    }
    for (int b = 0; b < NSUP; ++b) {
      cudaEvent_t* evs[] = {&a.lsup[b], &a.col[b], &a.bulk[b], &a.inv[b]};
      for (cudaEvent_t* e : evs)
        if (cudaEventCreateWithFlags(e, f) != cudaSuccess) return GPTQ_ERR_CUDA;
    }
  }
  *out = &a;
  return GPTQ_OK;
}

// The blocked factorization and inverse, panel by panel.  Panel k (columns k0 ..
// k0 + nb, buffers of parity b = k & 1):
//   c  the diagonal block: its last update (the previous panel's term, formed in
//      the kernel) and its factorization and inverse T_k -> LI[b].
//      Waits for panel k - 2's next-block-column update and trailing update
//      (the inputs of block k) and for the inverse's use of LI[b].
//   o  L21 = A21 . T_k^T for all rows below (split only: Lhi/Llo[b]); then the
//      next block column below its diagonal block, A(i, k+1) -= L(i, k) L(k+1, k)^T
//      for i >= k + 2, whose split is the next panel's A21 (Phi/Plo).
//   t  the trailing update of blocks >= k + 2 (lower triangle).
//   s  the inverse's block column k (Xt = (L^-1)^T): its diagonal block from T_k,
//      Xt[:k0, k] = Xt[:k0, k] . T_k^T, then Xt[:k0+nb, later] -= Xt[:, k] . L21^T.
// Block (k+1, k+1) gets panel k's term in the next diagonal launch, not on o.
int panel_loop(const PrepWs& w, int n, int ldn, AuxStream* aux, int32_t* st) {
  cudaStream_t c = aux->c, o = aux->o, t = aux->t, s2 = aux->s;
  int rc = GPTQ_OK;
  int panel = 0;
  for (int k0 = 0; k0 < n; k0 += PB, ++panel) {
    const int nb = std::min(PB, n - k0);
    const int rest = n - k0 - nb;
    const int b = panel % NBUF;                       // this panel's ring slot
    const int b1 = (panel + NBUF - 1) % NBUF;         // panel k - 1's
    const int b2 = (panel + NBUF - 2) % NBUF;         // panel k - 2's
    // ---- the diagonal block ----
    if (panel >= 2) {   // its inputs: panel k - 2's next-column and trailing updates
      GPTQ_CUDA_TRY(cudaStreamWaitEvent(c, aux->next[b2], 0));
      GPTQ_CUDA_TRY(cudaStreamWaitEvent(c, aux->trail[b2], 0));
    }
    if (panel >= NBUF) GPTQ_CUDA_TRY(cudaStreamWaitEvent(c, aux->done[b], 0));   // LI[b] is free again
    // useful flops: the previous panel's two 128-deep products (when there is one), the
    // block's Cholesky factorization and its triangular inverse
    TraceScope ts_d("potrf_inv", "flop", (panel > 0 ? 4.0 * nb * nb * PB : 0.0) + 2.0 / 3.0 * nb * nb * nb, c);
    rc = launch_potrf_inv(w, ldn, k0, nb, n, b1, panel > 0 ? k0 - PB : -1, b, st, c);
    if (rc != GPTQ_OK) return rc;
    GPTQ_CUDA_TRY(cudaEventRecord(aux->diag[b], c));
    if (rest > 0) {
      // ---- L21 and the next block column ----
      GPTQ_CUDA_TRY(cudaStreamWaitEvent(o, aux->diag[b], 0));
      if (panel >= NBUF) {   // Lhi/Llo[b]: the slot's previous trailing update and inverse are done
        GPTQ_CUDA_TRY(cudaStreamWaitEvent(o, aux->trail[b], 0));
        GPTQ_CUDA_TRY(cudaStreamWaitEvent(o, aux->done[b], 0));
      }
      // the split of A21 comes from the previous panel's update of this block column;
      // the first panel has none
      if (panel == 0) rc = launch_split_tf32(w.A + (int64_t)nb * ldn, rest, nb, ldn, w.Phi, w.Plo, PB, st, o);
      if (rc == GPTQ_OK)
        rc = launch_gemm3(nullptr, 0, rest, nb, nb, w.Phi, w.Plo, PB, w.LIhi[b], w.LIlo[b], PB, false, st, o, true,
                          w.Lhi[b], w.Llo[b], PB, "prepare_gemm3");
      if (rc != GPTQ_OK) return rc;
      GPTQ_CUDA_TRY(cudaEventRecord(aux->l21[b], o));
      const int nb2 = std::min(PB, rest);
      if (rest > nb2) {
        // A(i, k+1) for i >= k + 2; panel k - 1's trailing update reached it first
        if (panel >= 1) GPTQ_CUDA_TRY(cudaStreamWaitEvent(o, aux->trail[b1], 0));
        float* Anext = w.A + (int64_t)(k0 + nb + nb2) * ldn + (k0 + nb);
        rc = launch_gemm3(Anext, ldn, rest - nb2, nb2, nb, w.Lhi[b] + (int64_t)nb2 * PB, w.Llo[b] + (int64_t)nb2 * PB,
                          PB, w.Lhi[b], w.Llo[b], PB, false, st, o, false, w.Phi, w.Plo, PB, "prepare_gemm3");
        if (rc != GPTQ_OK) return rc;
        GPTQ_CUDA_TRY(cudaEventRecord(aux->next[b], o));
        // ---- the trailing update of blocks >= k + 2 ----
        GPTQ_CUDA_TRY(cudaStreamWaitEvent(t, aux->l21[b], 0));
        const float* Lh2 = w.Lhi[b] + (int64_t)nb2 * PB;
        const float* Ll2 = w.Llo[b] + (int64_t)nb2 * PB;
        rc = launch_gemm3(Anext + nb2, ldn, rest - nb2, rest - nb2, nb, Lh2, Ll2, PB, Lh2, Ll2, PB, true, st, t, false, nullptr, nullptr, 0,
                          "prepare_gemm3");
        if (rc != GPTQ_OK) return rc;
        GPTQ_CUDA_TRY(cudaEventRecord(aux->trail[b], t));
      }
    }
    // ---- the inverse's block column k ----
    GPTQ_CUDA_TRY(cudaStreamWaitEvent(s2, aux->diag[b], 0));
    {
      dim3 blk(32, 8), grd(PB / 32, PB / 32);
      xt_diag_kernel<<<grd, blk, 0, s2>>>(w.LIhi[b], w.LIlo[b], k0, nb, w.Xt, ldn, w.XQhi, w.XQlo, PB, st);
      GPTQ_LAUNCH_CHECK();
    }
    if (k0 > 0) {
      // Xt[:k0, k] = Xt[:k0, k] . T_k^T, with its split (rows 0..k0 of XQ)
      float* Xk = w.Xt + k0;
      rc = launch_split_tf32(Xk, k0, nb, ldn, w.XPhi, w.XPlo, PB, st, s2);
      if (rc == GPTQ_OK)
        rc = launch_gemm3(Xk, ldn, k0, nb, nb, w.XPhi, w.XPlo, PB, w.LIhi[b], w.LIlo[b], PB, false, st, s2, true,
                          w.XQhi, w.XQlo, PB, "prepare_gemm3");
      if (rc != GPTQ_OK) return rc;
    }
    if (rest > 0) {
      // Xt[:k0+nb, later] -= Xt[:k0+nb, k] . L21^T
      GPTQ_CUDA_TRY(cudaStreamWaitEvent(s2, aux->l21[b], 0));
      rc = launch_gemm3(w.Xt + (k0 + nb), ldn, k0 + nb, rest, nb, w.XQhi, w.XQlo, PB, w.Lhi[b], w.Llo[b], PB, false,
                        st, s2, false, nullptr, nullptr, 0, "prepare_gemm3");
      if (rc != GPTQ_OK) return rc;
    }
    GPTQ_CUDA_TRY(cudaEventRecord(aux->done[b], s2));
  }
  return GPTQ_OK;
}

// The same factorization and inverse with their bulk updates deferred to
// super-panels of SPB = 4 panels (for large n, where the per-panel loop is set by
// the bulk: each K = 128 rank update reads and writes its whole trailing matrix).
// Super-panel S (columns s0 .. se), buffers of parity sb = S % NSUP:
//   per panel p = s0 / PB + j, j = 0 .. 3, as in the per-panel loop but confined
//   to the super-panel's columns:
//     c  the diagonal block (panel p - 1's term formed in the kernel when p - 1
//        lies in the super-panel; earlier panels' terms are already in A);
//     o  L21 of all rows below into the super-panel's L (columns PB j), then the
//        next block column when it lies in the super-panel (its split: Phi/Plo);
//     t  the super-panel's columns beyond the next block column, all rows below
//        (lower, K = PB);
//     s  the inverse's block column p (Xt[:k0, p] and its split into the
//        super-panel's Xt split), then Xt[:k0+nb, later columns of the
//        super-panel] -= Xt[:, p] . L(later, p)^T.
//   then, once for the super-panel (K = se - s0):
//     o  the next super-panel's block column: A[se:, se:se2] -= L(se:, S) L(se:se2, S)^T
//        (lower), and the split of its first panel's A21;
//     t  the rest of the trailing matrix: A[se2:, se2:] -= L(se2:, S) L(se2:, S)^T;
//     s  the inverse beyond: Xt[:se, se:] -= Xt[:se, S] . L(se:, S)^T.
// Every product is the same 3 x TF32 tensor-core GEMM; only the grouping of the
// rank updates changes (four K = 128 updates of the trailing matrix become one
// K = 512 update), which is the blocked algorithm with 512-wide outer panels.
int panel_loop_deferred(const PrepWs& w, int n, int ldn, AuxStream* aux, int32_t* st) {
  cudaStream_t c = aux->c, o = aux->o, t = aux->t, s2 = aux->s;
  auto wait = [](cudaStream_t strm, cudaEvent_t ev) { return cudaStreamWaitEvent(strm, ev, 0); };
  int rc = GPTQ_OK;
  for (int s0 = 0, S = 0; s0 < n; s0 += SPB, ++S) {
    const int se = std::min(n, s0 + SPB);
    const int sb = S % NSUP;
    float* const Lh = w.Shi[sb];
    float* const Ll = w.Slo[sb];
    for (int k0 = s0; k0 < se; k0 += PB) {
      const int panel = k0 / PB, j = (k0 - s0) / PB;
      const int nb = std::min(PB, n - k0);
      const int rest = n - k0 - nb;
      const int b = panel % NLI, b1 = (panel + NLI - 1) % NLI, b2 = (panel + NLI - 2) % NLI;
      const int64_t cj = (int64_t)PB * j;   // the panel's columns in the super-panel buffers
      // ---- the diagonal block ----
      if (j == 0 && S > 0) GPTQ_CUDA_TRY(wait(c, aux->col[sb]));   // the super-panel's block column
      if (j >= 2) {   // panel p - 2's next-column and in-super-panel trailing updates
        GPTQ_CUDA_TRY(wait(c, aux->next[b2]));
        GPTQ_CUDA_TRY(wait(c, aux->trail[b2]));
      }
      if (panel >= NLI) GPTQ_CUDA_TRY(wait(c, aux->done[b]));   // LI[b] is free again
      TraceScope ts_d("potrf_inv", "flop", (j > 0 ? 4.0 * nb * nb * PB : 0.0) + 2.0 / 3.0 * nb * nb * nb, c);
      rc = launch_potrf_inv(w, ldn, k0, nb, n, b1, j > 0 ? k0 - PB : -1, b, st, c);
      if (rc != GPTQ_OK) return rc;
      GPTQ_CUDA_TRY(cudaEventRecord(aux->diag[b], c));
      if (rest > 0) {
        // ---- L21 and the next block column ----
        GPTQ_CUDA_TRY(wait(o, aux->diag[b]));
        if (j == 0 && S >= NSUP) {   // the super-panel buffers' previous readers are done
          GPTQ_CUDA_TRY(wait(o, aux->bulk[sb]));
          GPTQ_CUDA_TRY(wait(o, aux->inv[sb]));
        }
        if (panel == 0) rc = launch_split_tf32(w.A + (int64_t)nb * ldn, rest, nb, ldn, w.Phi, w.Plo, PB, st, o);
        if (rc == GPTQ_OK)
          rc = launch_gemm3(nullptr, 0, rest, nb, nb, w.Phi, w.Plo, PB, w.LIhi[b], w.LIlo[b], PB, false, st, o, true,
                            Lh + (int64_t)(k0 + nb) * SPB + cj, Ll + (int64_t)(k0 + nb) * SPB + cj, SPB,
                            "prepare_gemm3");
        if (rc != GPTQ_OK) return rc;
        GPTQ_CUDA_TRY(cudaEventRecord(aux->l21[b], o));
        const int nb2 = std::min(PB, rest);
        if (k0 + nb < se && rest > nb2) {
          // A(i, p+1) for i >= p + 2; panel p - 1's in-super-panel update reached it first
          if (j >= 1) GPTQ_CUDA_TRY(wait(o, aux->trail[b1]));
          const int r2 = k0 + nb + nb2;
          rc = launch_gemm3(w.A + (int64_t)r2 * ldn + (k0 + nb), ldn, n - r2, nb2, nb, Lh + (int64_t)r2 * SPB + cj,
                            Ll + (int64_t)r2 * SPB + cj, SPB, Lh + (int64_t)(k0 + nb) * SPB + cj,
                            Ll + (int64_t)(k0 + nb) * SPB + cj, SPB, false, st, o, false, w.Phi, w.Plo, PB,
                            "prepare_gemm3");
          if (rc != GPTQ_OK) return rc;
        }
        GPTQ_CUDA_TRY(cudaEventRecord(aux->next[b], o));
        // ---- the super-panel's columns beyond the next block column ----
        const int c0 = k0 + 2 * PB;
        if (c0 < se) {
          GPTQ_CUDA_TRY(wait(t, aux->l21[b]));
          rc = launch_gemm3(w.A + (int64_t)c0 * ldn + c0, ldn, n - c0, se - c0, nb, Lh + (int64_t)c0 * SPB + cj,
                            Ll + (int64_t)c0 * SPB + cj, SPB, Lh + (int64_t)c0 * SPB + cj, Ll + (int64_t)c0 * SPB + cj,
                            SPB, true, st, t, false, nullptr, nullptr, 0, "prepare_gemm3");
          if (rc != GPTQ_OK) return rc;
        }
        GPTQ_CUDA_TRY(cudaEventRecord(aux->trail[b], t));
      }
      // ---- the inverse's block column p ----
      GPTQ_CUDA_TRY(wait(s2, aux->diag[b]));
      {
        dim3 blk(32, 8), grd(PB / 32, PB / 32);
        xt_diag_kernel<<<grd, blk, 0, s2>>>(w.LIhi[b], w.LIlo[b], k0, nb, w.Xt, ldn, w.SXhi + cj, w.SXlo + cj, SPB,
                                            st);
        GPTQ_LAUNCH_CHECK();
      }
      if (k0 > 0) {
        float* Xk = w.Xt + k0;
        rc = launch_split_tf32(Xk, k0, nb, ldn, w.XPhi, w.XPlo, PB, st, s2);
        if (rc == GPTQ_OK)
          rc = launch_gemm3(Xk, ldn, k0, nb, nb, w.XPhi, w.XPlo, PB, w.LIhi[b], w.LIlo[b], PB, false, st, s2, true,
                            w.SXhi + cj, w.SXlo + cj, SPB, "prepare_gemm3");
        if (rc != GPTQ_OK) return rc;
      }
      if (se > k0 + nb) {
        // rows of the split below this panel's diagonal block inside the super-panel: Xt
        // is upper triangular there, and the bulk inverse update reads them
        GPTQ_CUDA_TRY(cudaMemset2DAsync(w.SXhi + (int64_t)(k0 + nb) * SPB + cj, SPB * sizeof(float), 0,
                                        PB * sizeof(float), se - k0 - nb, s2));
        GPTQ_CUDA_TRY(cudaMemset2DAsync(w.SXlo + (int64_t)(k0 + nb) * SPB + cj, SPB * sizeof(float), 0,
                                        PB * sizeof(float), se - k0 - nb, s2));
      }
      if (rest > 0) {
        GPTQ_CUDA_TRY(wait(s2, aux->l21[b]));
        const int c1 = k0 + nb;
        if (c1 < se) {   // Xt[:k0+nb, later columns of the super-panel] -= Xt[:, p] . L(later, p)^T
          rc = launch_gemm3(w.Xt + c1, ldn, k0 + nb, se - c1, nb, w.SXhi + cj, w.SXlo + cj, SPB,
                            Lh + (int64_t)c1 * SPB + cj, Ll + (int64_t)c1 * SPB + cj, SPB, false, st, s2, false,
                            nullptr, nullptr, 0, "prepare_gemm3");
          if (rc != GPTQ_OK) return rc;
        }
      }
      GPTQ_CUDA_TRY(cudaEventRecord(aux->done[b], s2));
    }
    if (se >= n) break;
    // ---- the super-panel's bulk updates (K = se - s0) ----
    const int se2 = std::min(n, se + SPB);
    const int K = se - s0;
    const int sn = (S + 1) % NSUP;
    GPTQ_CUDA_TRY(cudaEventRecord(aux->lsup[sb], o));
    // the next super-panel's block column; the previous super-panel's bulk update reached it first
    if (S >= 1) GPTQ_CUDA_TRY(wait(o, aux->bulk[(S + NSUP - 1) % NSUP]));
    const float* Lse_h = Lh + (int64_t)se * SPB;
    const float* Lse_l = Ll + (int64_t)se * SPB;
    rc = launch_gemm3(w.A + (int64_t)se * ldn + se, ldn, n - se, se2 - se, K, Lse_h, Lse_l, SPB, Lse_h, Lse_l, SPB,
                      true, st, o, false, nullptr, nullptr, 0, "prepare_gemm3");
    if (rc != GPTQ_OK) return rc;
    {
      const int nbn = std::min(PB, n - se);
      if (n - se - nbn > 0)
        rc = launch_split_tf32(w.A + (int64_t)(se + nbn) * ldn + se, n - se - nbn, nbn, ldn, w.Phi, w.Plo, PB, st, o);
      if (rc != GPTQ_OK) return rc;
    }
    GPTQ_CUDA_TRY(cudaEventRecord(aux->col[sn], o));
    // the rest of the trailing matrix
    GPTQ_CUDA_TRY(wait(t, aux->lsup[sb]));
    if (se2 < n) {
      const float* L2h = Lh + (int64_t)se2 * SPB;
      const float* L2l = Ll + (int64_t)se2 * SPB;
      rc = launch_gemm3(w.A + (int64_t)se2 * ldn + se2, ldn, n - se2, n - se2, K, L2h, L2l, SPB, L2h, L2l, SPB, true,
                        st, t, false, nullptr, nullptr, 0, "prepare_gemm3");
      if (rc != GPTQ_OK) return rc;
    }
    GPTQ_CUDA_TRY(cudaEventRecord(aux->bulk[sb], t));
    // the inverse beyond the super-panel
    GPTQ_CUDA_TRY(wait(s2, aux->lsup[sb]));
    rc = launch_gemm3(w.Xt + se, ldn, se, n - se, K, w.SXhi, w.SXlo, SPB, Lse_h, Lse_l, SPB, false, st, s2, false,
                      nullptr, nullptr, 0, "prepare_gemm3");
    if (rc != GPTQ_OK) return rc;
    GPTQ_CUDA_TRY(cudaEventRecord(aux->inv[sb], s2));
  }
  return GPTQ_OK;
}

}  // namespace

namespace {
std::atomic<int> g_deferred_min_n{8192};
}  // namespace

int prepare_set_deferred_min_n(int min_n) {
  return min_n > 0 ? g_deferred_min_n.exchange(min_n) : g_deferred_min_n.load();
}

size_t prepare_ws_bytes(int n) {
  const int ldn = ld_of(n);
  const size_t nn = align_up((size_t)n * ldn * sizeof(float), 256);
  const size_t panel = align_up((size_t)n * PB * sizeof(float), 256);
  const size_t sup = align_up((size_t)n * SPB * sizeof(float), 256);
  return 2 * nn + 4 * panel + (2 * NSUP + 2) * sup + 2 * NLI * align_up((size_t)PB * PB * 4, 256) +
         align_up((size_t)n * 8, 256) + align_up((size_t)n * 4, 256) + 256;
}

namespace {

// The whole stage enqueued on stream s (and the library's streams, joined back to s).
int enqueue_prepare(const float* H, const double* hdiag, int n, float damp, int desc_act, float* U, int32_t* perm,
                    uint8_t* dead, void* ws, int32_t* st, bool deferred, cudaStream_t s) {
  PrepWs w = carve(ws, n);
  const int ldn = ld_of(n);
  prep_diag_kernel<<<(int)cdiv(n, 256), 256, 0, s>>>(H, hdiag, n, desc_act, dead, w.key, w.dfix, st);
  GPTQ_LAUNCH_CHECK();
  prep_lambda_kernel<<<1, 1024, 0, s>>>(w.dfix, n, damp, w.scal, st);
  GPTQ_LAUNCH_CHECK();
  if (desc_act) prep_rank_kernel<<<(int)cdiv(n, 256), 256, 0, s>>>(w.key, n, perm, st);
  else prep_identity_kernel<<<(int)cdiv(n, 256), 256, 0, s>>>(perm, n);
  GPTQ_LAUNCH_CHECK();
  if (desc_act && n <= kGatherRowMax) {
    // Xt is scratch until the factorization starts (it is written before it is read)
    dim3 blk(32, 8), grd((unsigned)cdiv(n, 32), (unsigned)cdiv(n, 32));
    prep_symmetrize_kernel<<<grd, blk, 0, s>>>(H, n, w.Xt, ldn, st);
    GPTQ_LAUNCH_CHECK();
    const size_t smem = (size_t)n * sizeof(float);
    GPTQ_CUDA_TRY(cudaFuncSetAttribute(prep_gather_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    prep_gather_rows_kernel<<<n, 256, smem, s>>>(w.Xt, ldn, w.dfix, perm, n, ldn, w.scal, w.A, st);
  } else if (desc_act) {
    dim3 blk(32, 8), grd((unsigned)cdiv(n, 32), (unsigned)cdiv(n, 8));
    prep_gather_kernel<<<grd, blk, 0, s>>>(H, w.dfix, perm, n, ldn, w.scal, w.A, st);
  } else {
    prep_reverse_kernel<<<n, 256, 0, s>>>(H, w.dfix, n, ldn, w.scal, w.A, st);
  }
  GPTQ_LAUNCH_CHECK();
  if (n > PB) {
    // rows above the last block row (which starts at the last multiple of PB below n)
    zero_upper_blocks_kernel<<<(unsigned)((n - 1) / PB * PB), 256, 0, s>>>(w.Xt, n, ldn);
    GPTQ_LAUNCH_CHECK();
  }

  GPTQ_CUDA_TRY(cudaFuncSetAttribute(potrf_inv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)POTRF_SMEM));
  AuxStream* aux = nullptr;
  int rc = aux_stream(&aux);
  if (rc != GPTQ_OK) return rc;
  cudaStream_t loop_streams[4] = {aux->c, aux->o, aux->t, aux->s};
  GPTQ_CUDA_TRY(cudaEventRecord(aux->fork, s));
  for (cudaStream_t ls : loop_streams) GPTQ_CUDA_TRY(cudaStreamWaitEvent(ls, aux->fork, 0));
  rc = deferred ? panel_loop_deferred(w, n, ldn, aux, st) : panel_loop(w, n, ldn, aux, st);
  // the loop's streams join the caller's stream, after an error too
  for (int i = 0; i < 4; ++i) {
    GPTQ_CUDA_TRY(cudaEventRecord(aux->join[i], loop_streams[i]));
    GPTQ_CUDA_TRY(cudaStreamWaitEvent(s, aux->join[i], 0));
  }
  if (rc != GPTQ_OK) return rc;
  {
    dim3 blk(64, 4), grd((unsigned)cdiv(n, 64), (unsigned)cdiv(n, 64));
    write_u_kernel<<<grd, blk, 0, s>>>(w.Xt, n, ldn, U, st);
    GPTQ_LAUNCH_CHECK();
  }
  return GPTQ_OK;
}

}  // namespace

// The stage is a chain of small dependent launches on four streams: replayed as one
// CUDA graph (run_graph_cached), its dependencies are graph edges instead of
// cross-stream event waits, which shortens every link of the chain (n = 4096: 1.70 ->
// 1.52 ms).  The key is every argument the graph holds by value.
int launch_prepare(const float* H, const double* hdiag, int n, float damp, int desc_act, float* U,
                   int32_t* perm, uint8_t* dead, void* ws, int32_t* st, cudaStream_t s) {
  const bool deferred = n >= g_deferred_min_n.load();
  uint32_t db;
  memcpy(&db, &damp, sizeof(db));
  GraphKey key;
  key.add(1).add(H).add(hdiag).add(n).add(db).add(desc_act).add(U).add(perm).add(dead).add(ws).add(st).add(deferred);
  return run_graph_cached(key, s, [&](cudaStream_t strm) {
    return enqueue_prepare(H, hdiag, n, damp, desc_act, U, perm, dead, ws, st, deferred, strm);
  });
}

}  // namespace gptq
