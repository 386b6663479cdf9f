// K0 ingest, K3 column sweep, K4 lazy trailing update, K5 packing; the zero points
// packed into words; W read as the first columns of a zero-padded layer
// ("polydesk.ai/glossaire/gptq", "Limites de GPTQ": weights padded with zeros).
//
// "polydesk.ai/glossaire/gptq":
//   "Etape 2" - per column: quantize (rounding + scale), take the error, push it
//               onto the remaining columns through the inverse Hessian's
//               Cholesky factor;
//   "Etape 3" - the updates are batched per block of 128 columns;
//   "sym"     - symmetric grid [-2^(b-1)+1, 2^(b-1)-1] with an exact zero, or an
//               asymmetric zero point;
//   group_size - groups sharing one scale (-1: one per row).
// "dev.ayinedjimi-consultants.fr ... ia-quantization-gptq-gguf-awq",
// "Calibration et dataset": scale and zero point are stored in FP16.
#include <math.h>

#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "internal.h"

// Timeline marks for probes; empty in the library build.
#ifndef GPTQ_SWEEP_MARK
#define GPTQ_SWEEP_MARK(i)
#endif

namespace gptq {

namespace {

constexpr int BLK = 128;           // columns per lazy batch
constexpr int SUPER = 4;           // lazy batches per super-block
constexpr int SBK = SUPER * BLK;   // columns per super-block

// Super-block s uses the error and operand buffers of parity s & 1: the trailing
// update of super-block s still reads them while super-block s + 1 is swept.
struct QuantWs {
  float* Wf;          // [out, n] working weights, processing order
  float* Ehi[2];      // [out, SBK] scaled errors of a super-block, TF32-exact high part
  float* Elo[2];      // [out, SBK] and the remainder
  float* Bhi[2];      // [n, SBK] U[super-block rows, later columns]^T, high part (K-major operand)
  float* Blo[2];      // [n, SBK] and the remainder
  uint8_t* codes_p;   // [out, n] codes, processing order
  int32_t* invperm;   // [n] processing position of every input column
  float* rows;        // [out] row-wide scale, [out] row-wide zero (group_size = -1)
};

QuantWs carve(void* ws, int out, int n) {
  char* p = static_cast<char*>(ws);
  QuantWs w;
  w.Wf = reinterpret_cast<float*>(p);        p += align_up((size_t)out * n * 4, 256);
  for (int b = 0; b < 2; ++b) {
    w.Ehi[b] = reinterpret_cast<float*>(p);  p += align_up((size_t)out * SBK * 4, 256);
    w.Elo[b] = reinterpret_cast<float*>(p);  p += align_up((size_t)out * SBK * 4, 256);
    w.Bhi[b] = reinterpret_cast<float*>(p);  p += align_up((size_t)n * SBK * 4, 256);
    w.Blo[b] = reinterpret_cast<float*>(p);  p += align_up((size_t)n * SBK * 4, 256);
  }
  w.codes_p = reinterpret_cast<uint8_t*>(p); p += align_up((size_t)out * n, 256);
  w.invperm = reinterpret_cast<int32_t*>(p); p += align_up((size_t)n * 4, 256);
  w.rows = reinterpret_cast<float*>(p);
  return w;
}

__device__ __forceinline__ float tf32_hi(float x) { return __uint_as_float(__float_as_uint(x) & 0xFFFFE000u); }

// ---------------------------------------------------------------------------
// The quantizer.  Every operation is one IEEE fp32 operation (round to nearest
// even), so identical inputs give identical decisions on any IEEE machine.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float to_f16_scale(float s) {
  // Round to FP16 (the stored precision) before use; keep within fp16's positive range.
  const float kMin = 5.9604644775390625e-08f;  // 2^-24, the smallest fp16 subnormal
  s = fminf(fmaxf(s, kMin), 65504.f);
  return fmaxf(__half2float(__float2half_rn(s)), kMin);
}

struct QParams { float s, z, rs, s24; };   // scale, zero point, fp32 reciprocal of the scale, s . 2^-24

__device__ __forceinline__ QParams params_asym(float lo, float hi, float maxq) {
  lo = fminf(lo, 0.f);
  hi = fmaxf(hi, 0.f);
  if (hi == lo) { lo = -1.f; hi = 1.f; }
  QParams p;
  p.s = to_f16_scale(__fdiv_rn(__fsub_rn(hi, lo), maxq));
  p.z = fminf(fmaxf(rintf(__fdiv_rn(-lo, p.s)), 0.f), maxq);
  p.rs = __frcp_rn(p.s);
  p.s24 = p.s * 5.9604644775390625e-08f;
  return p;
}

__device__ __forceinline__ QParams params_sym(float amax, int bits) {
  if (amax == 0.f) amax = 1.f;
  QParams p;
  p.s = to_f16_scale(__fdiv_rn(amax, (float)((1 << (bits - 1)) - 1)));
  p.z = (float)(1 << (bits - 1));
  p.rs = __frcp_rn(p.s);
  p.s24 = p.s * 5.9604644775390625e-08f;
  return p;
}

// rint(fl(w / s)), fl = IEEE round-to-nearest division, without dividing and
// without branches (the column loop stays one basic block).  With t = w . fl(1/s)
// and a lower candidate k, the answer is k or k + 1; round_up tells which.
//   t is within |w/s| . 2^-22 of w/s, so for |t| < 1024 the answer is floor(t) or
//   floor(t) + 1, i.e. it is decided by the side of h = floor(t) + 1/2 on which the
//   rounded quotient lies.  d = fma(-h, s, w) = RN(w - h.s): h.s is exact (h has at
//   most 13 significant bits, s is an fp16 value), so the sign of d is the sign of
//   w/s - h, and d itself is exact whenever w/s is within 1/4 of h (Sterbenz).  The
//   rounded quotient equals h exactly iff |w/s - h| <= ulp(h)/2, i.e.
//   |d| <= s . ulp(h)/2 (h's last mantissa bit is 0 for |h| < 2^22, so a tie rounds
//   to h); then rint picks the even one of k, k + 1.
//   The candidate is k = rint(t - 1/2), formed by adding and subtracting 1.5 . 2^23
//   (no conversion instruction): it is floor(t), except that for an integer t it may
//   be t - 1; then w/s lies half a unit above h = t - 1/2 and d > 0 picks k + 1 = t,
//   the right answer again.  The sum's last mantissa bit is the parity of k.
//   s . ulp(h)/2 = (s . 2^-24) . 2^e(h), 2^e(h) being the exponent bits of h alone.
//   For |t| >= 1024 both candidates saturate to the same code (codes have at most 8
//   bits), so the answer does not matter there.
struct Cand { float k; bool odd; };

__device__ __forceinline__ Cand lower_candidate(float t) {
  const float y = (t - 0.5f) + 12582912.f;   // rint(t - 1/2) + 1.5 . 2^23
  return {y - 12582912.f, (__float_as_uint(y) & 1u) != 0u};
}

__device__ __forceinline__ bool round_up(float w, Cand c, QParams p) {
  const float h = c.k + 0.5f;
  const float d = fmaf(-h, p.s, w);
  const float thr = p.s24 * __uint_as_float(__float_as_uint(h) & 0x7F800000u);
  return fabsf(d) <= thr ? c.odd : d > 0.f;
}

__device__ __forceinline__ float code_from_q(float q, QParams p, int bits, bool sym) {
  if (sym) {
    const float h = (float)((1 << (bits - 1)) - 1);
    return fminf(fmaxf(q, -h), h) + p.z;
  }
  return fminf(fmaxf(q + p.z, 0.f), (float)((1 << bits) - 1));
}

// ---------------------------------------------------------------------------
// K0: Wf[r][k] = W[r][perm[k]] (0 for dead inputs), invperm, g_idx.
// ---------------------------------------------------------------------------
// Four consecutive columns per thread (n % 4 == 0): 16-byte stores, and the loads of a
// warp cover 128 consecutive columns of a row for the identity order.  W has w_cols
// columns (its row stride); columns w_cols .. n-1 are the zero padding of a layer
// whose width the group size or the packing does not divide.
// Rows may come from several layers of one input (WRows: row r belongs to the layer
// whose range holds it).
template <typename T>
__global__ void ingest_kernel(const __grid_constant__ WRows W, int out, int w_cols, int n, const int32_t* perm,
                              const uint8_t* dead, int gs, float* Wf, int32_t* invperm, int32_t* g_idx, int32_t* st) {
  if (has_error(st)) return;
  const int k0 = 4 * (blockIdx.x * 32 + threadIdx.x);
  const int r = blockIdx.y * 8 + threadIdx.y;
  if (k0 >= n) return;
  int src[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) src[u] = perm ? perm[k0 + u] : k0 + u;
  if (r == 0) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      invperm[src[u]] = k0 + u;
      g_idx[src[u]] = gs > 0 ? (k0 + u) / gs : 0;
    }
  }
  if (r >= out) return;
  int li = 0;
  while (li + 1 < W.count && r >= W.row0[li + 1]) ++li;
  const T* row = static_cast<const T*>(W.W[li]) + (int64_t)(r - W.row0[li]) * w_cols;
  float v[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    v[u] = src[u] < w_cols ? load_as_float<T>(row + src[u]) : 0.f;
    if (!isfinite(v[u])) set_error(st, GPTQ_ERR_NONFINITE, src[u], STAGE_INGEST);
    if (dead && dead[src[u]]) v[u] = 0.f;
  }
  *reinterpret_cast<float4*>(Wf + (int64_t)r * n + k0) = make_float4(v[0], v[1], v[2], v[3]);
}

// group_size = -1: one scale / zero per row, from the whole (uncompensated) row.
__global__ void __launch_bounds__(256) row_params_kernel(const float* Wf, int out, int n, int bits, int sym,
                                                         float* rows, uint16_t* scales, uint16_t* zeros,
                                                         const int32_t* st) {
  if (has_error(st)) return;
  const int r = blockIdx.x;
  if (r >= out) return;
  float lo = INFINITY, hi = -INFINITY, amax = 0.f;
  for (int k = threadIdx.x; k < n; k += blockDim.x) {
    const float v = Wf[(int64_t)r * n + k];
    lo = fminf(lo, v); hi = fmaxf(hi, v); amax = fmaxf(amax, fabsf(v));
  }
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  }
  __shared__ float red[3][8];
  if ((threadIdx.x & 31) == 0) { red[0][threadIdx.x >> 5] = lo; red[1][threadIdx.x >> 5] = hi; red[2][threadIdx.x >> 5] = amax; }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < 8; ++w) { lo = fminf(lo, red[0][w]); hi = fmaxf(hi, red[1][w]); amax = fmaxf(amax, red[2][w]); }
    lo = fminf(lo, red[0][0]); hi = fmaxf(hi, red[1][0]); amax = fmaxf(amax, red[2][0]);
    const QParams p = sym ? params_sym(amax, bits) : params_asym(lo, hi, (float)((1 << bits) - 1));
    rows[r] = p.s;
    rows[out + r] = p.z;
    scales[r] = __half_as_ushort(__float2half_rn(p.s));
    zeros[r] = __half_as_ushort(__float2half_rn(p.z));
  }
}

// ---------------------------------------------------------------------------
// K3: the sweep of one block [b0, b0 + bw) of columns.
//
// TPR lanes of one warp own one row; lane `seg` of the row holds the block's
// columns [seg.SEG, seg.SEG + SEG) in registers.  For column j the owning lane's
// error e is broadcast with a shuffle and every lane applies e . U[j, :] to its own
// columns.  The U block sits in shared memory with its strictly-lower part
// zeroed, so the update needs no masking: columns before j see U = 0, and the
// owner overwrites column j with e afterwards.  Rows are independent given U
// ("polydesk.ai/glossaire/gptq", "Etape 1": the inverse-Hessian work is shared by
// all rows), so rows never synchronize.
// GS = group size (32/64/128), or 0 for row-wide parameters given in `rows`.
// ---------------------------------------------------------------------------
template <int TPR>
struct SweepShape {
  static constexpr int SEG = BLK / TPR;          // columns per lane
  // padded segment stride in shared memory (4-column segments are conflict-free as they are)
  static constexpr int SEGP = SEG >= 8 ? SEG + 4 : SEG;
  static constexpr int LDU = TPR * SEGP;         // padded U row stride
  static constexpr int THREADS = TPR == 32 ? 256 : 128;
  static constexpr int ROWS = THREADS / TPR;     // rows per CTA
  static constexpr int LDE = BLK + 4;            // error row stride (16-byte aligned rows)
  // two U stages (the block's U, then the near passes alternating), 1/U_jj, errors, and
  // the block's codes of the CTA's rows (the fused packing)
  static constexpr size_t SMEM = 2 * (size_t)BLK * LDU * sizeof(float) + BLK * sizeof(float) +
                                 (size_t)ROWS * LDE * sizeof(float) + (size_t)ROWS * BLK;
};

template <int GS, int TPR, bool SYM>
__global__ void __launch_bounds__(SweepShape<TPR>::THREADS)
sweep_kernel(float* Wf, int out, int n, int s0, int se, const float* U, float* Ehi, float* Elo,
             uint8_t* codes_p, int32_t* qweight,
             uint16_t* scales, uint16_t* zeros, const float* rows, float* err_sq, int bits, int sym,
             const int32_t* st) {
  using SS = SweepShape<TPR>;
  constexpr int SEG = SS::SEG;
  if (has_error(st)) return;
  GPTQ_SWEEP_MARK(0);
  extern __shared__ float smem[];
  // two U stages of [BLK][LDU], at smem and smem + BLK * LDU
  float* dinv = smem + 2 * BLK * SS::LDU; // [BLK] 1 / U_jj
  // U[r0 + j][c0 + c] (j < rows_n, c < cols_n, zero elsewhere) into a stage, in
  // 16-byte asynchronous copies, all in flight together.
  auto stage = [&](float* buf, int r0, int c0, int rows_n, int cols_n) {
    for (int idx = threadIdx.x; idx < BLK * (BLK / 4); idx += blockDim.x) {
      const int j = idx / (BLK / 4), c = (idx % (BLK / 4)) * 4;
      float* dst = buf + j * SS::LDU + (c / SEG) * SS::SEGP + (c % SEG);
      if (j < rows_n && c < cols_n) {
        const float* src = U + (int64_t)(r0 + j) * n + c0 + c;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
                     "l"(src)
                     : "memory");
      } else {
        *reinterpret_cast<float4*>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  const int lane = threadIdx.x & 31;
  const int seg = lane % TPR;
  const int r = blockIdx.x * SS::ROWS + threadIdx.x / TPR;
  const bool live = r < out;
  const int rr = live ? r : 0;
  constexpr bool symq = SYM;   // a compile-time choice: the column loop has no branch on it
  const float maxq = (float)((1 << bits) - 1);
  QParams p;
  if (GS == 0) { p.s = rows[rr]; p.z = rows[out + rr]; p.rs = __frcp_rn(p.s); p.s24 = p.s * 5.9604644775390625e-08f; }
  else { p.s = 1.f; p.z = 0.f; p.rs = 1.f; p.s24 = 5.9604644775390625e-08f; }
  float esq = 0.f;
  const int group_lane0 = lane & ~(TPR - 1);

  // The blocks of the super-block [s0, se) one after the other.  A block's U is
  // staged during the previous block's last near pass (the first block's here); the
  // block's first near pass is fetched behind it and lands during the sweep.
  int d = 0;                                        // the stage holding this block's U
  stage(smem, s0, s0, min(BLK, se - s0), min(BLK, se - s0));
#pragma unroll 1
  for (int b0 = s0; b0 < se; b0 += BLK) {
  const int bw = min(BLK, se - b0);
  const int eoff = b0 - s0;
  const bool has_near = b0 + bw < se;
  float* Us = smem + d * (BLK * SS::LDU);           // the block's U; then near passes 1, 3
  float* Uo = smem + (d ^ 1) * (BLK * SS::LDU);     // near passes 0, 2
  __syncthreads();                                  // the previous block is done with Uo
  if (has_near) stage(Uo, b0, b0 + bw, bw, min(BLK, se - b0 - bw));
  if (has_near) asm volatile("cp.async.wait_group 1;" ::: "memory");
  else asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();
  for (int j = threadIdx.x; j < BLK; j += blockDim.x) {
    float* dj = Us + j * SS::LDU + (j / SEG) * SS::SEGP + (j % SEG);
    dinv[j] = (j < bw) ? 1.f / *dj : 0.f;
    *dj = 0.f;   // the update by column j then leaves columns <= j alone
  }
  __syncthreads();
  GPTQ_SWEEP_MARK(1);

  float w[SEG];
  {
    const float* src = Wf + (int64_t)rr * n + b0 + seg * SEG;
    const bool inb = live && seg * SEG < bw;
#pragma unroll
    for (int k = 0; k < SEG; k += 4) {
      float4 v = inb ? *reinterpret_cast<const float4*>(src + k) : make_float4(0.f, 0.f, 0.f, 0.f);
      w[k] = v.x; w[k + 1] = v.y; w[k + 2] = v.z; w[k + 3] = v.w;
    }
  }
  GPTQ_SWEEP_MARK(6);
  uint32_t cw[SEG / 4];
#pragma unroll
  for (int k = 0; k < SEG / 4; ++k) cw[k] = 0u;

  // Column j's error reaches the lanes' registers one column late: the update by
  // column j - 1 is applied in step j, after column j's decision, so the broadcast of
  // that error overlaps the decision instead of preceding it.  The owner of column j
  // folds the pending term into its value itself (wq), from its own previous error
  // inside its segment and from the broadcast one at a segment's first column.
  // Group parameters read every lane's columns, so a group start applies the
  // pending update first.
  auto apply = [&](float e, const float* urow) {
#pragma unroll
    for (int k = 0; k < SEG; k += 4) {
      const float4 u = *reinterpret_cast<const float4*>(urow + k);
      w[k] = fmaf(-e, u.x, w[k]);
      w[k + 1] = fmaf(-e, u.y, w[k + 1]);
      w[k + 2] = fmaf(-e, u.z, w[k + 2]);
      w[k + 3] = fmaf(-e, u.w, w[k + 3]);
    }
  };
  float e_prev = 0.f;   // the pending (broadcast) error of column j - 1
  float e_mine = 0.f;   // this lane's error of column j - 1 when it owned it
  for (int jb = 0; jb < TPR; ++jb) {
    if (jb * SEG >= bw) break;
    const bool owner = seg == jb;
#pragma unroll
    for (int jj = 0; jj < SEG; ++jj) {
      const int j = jb * SEG + jj;
      const float* urow_p = Us + (j > 0 ? j - 1 : 0) * SS::LDU + seg * SS::SEGP;   // U row j - 1
      if (GS > 0 && jj == 0 && ((b0 + j) % (GS > 0 ? GS : 1)) == 0) {
        apply(e_prev, urow_p);
        e_prev = 0.f;
        // group [j, j + GS): lanes whose segment lies inside it contribute
        const int g_lo = j, g_hi = j + GS;
        const bool in = seg * SEG >= g_lo && seg * SEG + SEG <= g_hi;
        float lo = INFINITY, hi = -INFINITY, amax = 0.f;
        if (in) {
#pragma unroll
          for (int k = 0; k < SEG; ++k) { lo = fminf(lo, w[k]); hi = fmaxf(hi, w[k]); amax = fmaxf(amax, fabsf(w[k])); }
        }
#pragma unroll
        for (int o = 1; o < TPR; o <<= 1) {
          lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
          hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
          amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        }
        p = symq ? params_sym(amax, bits) : params_asym(lo, hi, maxq);
        if (owner && live) {
          const int g = (b0 + j) / (GS > 0 ? GS : 1);
          scales[(int64_t)g * out + r] = __half_as_ushort(__float2half_rn(p.s));
          zeros[(int64_t)g * out + r] = __half_as_ushort(__float2half_rn(p.z));
        }
      }
      // the owner's column j with every update up to column j - 1 (U[j-1][j] is read by
      // every lane at the owner's address: one broadcast)
      const float ep = jj == 0 ? e_prev : e_mine;
      const float u_pj = Us[(j > 0 ? j - 1 : 0) * SS::LDU + jb * SS::SEGP + jj];
      const float wq = fmaf(-ep, u_pj, w[jj]);
      // rint(fl(wq / s)) is k or k + 1 (round_up); both candidates' codes and errors
      // are formed beside the decision, which then only selects
      const float t = wq * p.rs;
      const Cand kc = lower_candidate(t);
      const float k = kc.k;
      const float c_lo = code_from_q(k, p, bits, symq), c_hi = code_from_q(k + 1.f, p, bits, symq);
      const float dj = dinv[j];
      const float e_lo = (wq - p.s * (c_lo - p.z)) * dj;
      const float e_hi = (wq - p.s * (c_hi - p.z)) * dj;
      const bool up = round_up(wq, kc, p);
      const float c = up ? c_hi : c_lo;
      const float e_own = up ? e_hi : e_lo;
      const float e_cur = __shfl_sync(0xffffffffu, e_own, group_lane0 | jb);
      apply(e_prev, urow_p);            // the lagged update by column j - 1
      if (owner) {
        w[jj] = e_own;
        esq = fmaf(e_own, e_own, esq);
        cw[jj / 4] |= ((uint32_t)c) << (8 * (jj % 4));
      }
      e_mine = e_own;
      e_prev = e_cur;
    }
  }
  // (the update by the block's last column reaches no column of the block)
  GPTQ_SWEEP_MARK(2);
  if (!live || seg * SEG >= bw) {
    // nothing to store for this lane
  } else {
    float* ehi = Ehi + (int64_t)r * SBK + eoff + seg * SEG;
    float* elo = Elo + (int64_t)r * SBK + eoff + seg * SEG;
#pragma unroll
    for (int k = 0; k < SEG; k += 4) {
      const float4 h = make_float4(tf32_hi(w[k]), tf32_hi(w[k + 1]), tf32_hi(w[k + 2]), tf32_hi(w[k + 3]));
      *reinterpret_cast<float4*>(ehi + k) = h;
      *reinterpret_cast<float4*>(elo + k) = make_float4(w[k] - h.x, w[k + 1] - h.y, w[k + 2] - h.z, w[k + 3] - h.w);
    }
    // this lane's SEG codes (n % 32 == 0 keeps every width aligned)
    uint8_t* crow = codes_p + (int64_t)r * n + b0 + seg * SEG;
    if constexpr (SEG % 16 == 0) {
#pragma unroll
      for (int k = 0; k < SEG; k += 16)
        *reinterpret_cast<uint4*>(crow + k) = make_uint4(cw[k / 4], cw[k / 4 + 1], cw[k / 4 + 2], cw[k / 4 + 3]);
    } else if constexpr (SEG == 8) {
      *reinterpret_cast<uint2*>(crow) = make_uint2(cw[0], cw[1]);
    } else {
      *reinterpret_cast<uint32_t*>(crow) = cw[0];
    }
    if (qweight != nullptr) {   // the codes of the CTA's rows for the fused packing below
      uint32_t* cs = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(dinv + BLK + SS::ROWS * SS::LDE) +
                                                 (threadIdx.x / TPR) * BLK + seg * SEG);
#pragma unroll
      for (int k = 0; k < SEG / 4; ++k) cs[k] = cw[k];
    }
  }
  // Packing fused into the sweep (identity column order, qweight given): the block's words
  // of the bit stream (column k at bits k.bits; a 128-column block holds whole words for
  // every width) straight from the staged codes; word wi of row r goes to
  // qweight[b0 . bits / 32 + wi][r], consecutive threads on consecutive rows.
  if (qweight != nullptr) {
    __syncthreads();
    const uint8_t* cs = reinterpret_cast<const uint8_t*>(dinv + BLK + SS::ROWS * SS::LDE);
    const int wpr = bw * bits / 32;
    const int64_t wbase = (int64_t)b0 * bits / 32;
    const uint32_t mask = (1u << bits) - 1u;
    for (int idx = threadIdx.x; idx < SS::ROWS * wpr; idx += blockDim.x) {
      const int rl = idx % SS::ROWS, wi = idx / SS::ROWS;
      const int row = blockIdx.x * SS::ROWS + rl;
      if (row >= out) continue;
      const int pos0 = wi * 32;
      const int k_lo = pos0 / bits, k_hi = min((pos0 + 31) / bits, bw - 1);
      uint64_t acc = 0;
      for (int k = k_lo; k <= k_hi; ++k) {
        const uint64_t c = cs[rl * BLK + k] & mask;
        const int sh = k * bits - pos0;   // negative for a code straddling in from the left
        acc |= sh >= 0 ? c << sh : c >> -sh;
      }
      qweight[(wbase + wi) * out + row] = (int32_t)(uint32_t)acc;
    }
  }
  GPTQ_SWEEP_MARK(3);

  // Near update: the rest of this super-block, columns [b0 + bw, se), absorbs this
  // block's errors, W[r][c] -= sum_j e_j U[b0 + j][c], in fp32 on the CUDA cores,
  // 128 columns at a time with the U rows staged in shared memory.  The columns past
  // the super-block are updated once per super-block by the tensor-core GEMM.
  if (has_near) {
    float* Es = dinv + BLK;                        // [ROWS][LDE] this block's errors per row
    const int rloc = threadIdx.x / TPR;
#pragma unroll
    for (int k = 0; k < SEG; ++k) Es[rloc * SS::LDE + seg * SEG + k] = (seg * SEG < bw) ? w[k] : 0.f;
    int pass = 0;
    for (int c0n = b0 + bw; c0n < se; c0n += BLK, ++pass) {
      const int cwid = min(BLK, se - c0n);
      float* cur = (pass & 1) ? Us : Uo;
      float* nxt = (pass & 1) ? Uo : Us;
      asm volatile("cp.async.wait_group 0;" ::: "memory");
      __syncthreads();                             // cur has landed; Es is complete; nxt is free
      if (c0n + BLK < se) {
        stage(nxt, b0, c0n + BLK, bw, min(BLK, se - c0n - BLK));   // the next pass's rows
      } else {
        // the last pass: the next block's own U goes to the other stage
        const int bn = b0 + BLK, bwn = min(BLK, se - bn);
        stage(nxt, bn, bn, bwn, bwn);
        d = (pass & 1) ? d ^ 1 : d;
      }
      GPTQ_SWEEP_MARK(4);
      // two accumulators (even and odd groups of four rows) halve the dependent
      // chains; the errors past bw are zero
      float acc[SEG], acc2[SEG];
#pragma unroll
      for (int k = 0; k < SEG; ++k) { acc[k] = 0.f; acc2[k] = 0.f; }
      const float* erow = Es + rloc * SS::LDE;
#pragma unroll 2
      for (int j = 0; j < bw; j += 8) {
        const float4 e4a = *reinterpret_cast<const float4*>(erow + j);
        const float4 e4b = *reinterpret_cast<const float4*>(erow + j + 4);
        const float ea[4] = {e4a.x, e4a.y, e4a.z, e4a.w};
        const float eb[4] = {e4b.x, e4b.y, e4b.z, e4b.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float* ua = cur + (j + q) * SS::LDU + seg * SS::SEGP;
          const float* ub = cur + (j + 4 + q) * SS::LDU + seg * SS::SEGP;
#pragma unroll
          for (int k = 0; k < SEG; k += 4) {
            const float4 u = *reinterpret_cast<const float4*>(ua + k);
            const float4 v = *reinterpret_cast<const float4*>(ub + k);
            acc[k] = fmaf(ea[q], u.x, acc[k]);
            acc[k + 1] = fmaf(ea[q], u.y, acc[k + 1]);
            acc[k + 2] = fmaf(ea[q], u.z, acc[k + 2]);
            acc[k + 3] = fmaf(ea[q], u.w, acc[k + 3]);
            acc2[k] = fmaf(eb[q], v.x, acc2[k]);
            acc2[k + 1] = fmaf(eb[q], v.y, acc2[k + 1]);
            acc2[k + 2] = fmaf(eb[q], v.z, acc2[k + 2]);
            acc2[k + 3] = fmaf(eb[q], v.w, acc2[k + 3]);
          }
        }
      }
#pragma unroll
      for (int k = 0; k < SEG; ++k) acc[k] += acc2[k];
      if (live && seg * SEG < cwid) {
        float* dst = Wf + (int64_t)r * n + c0n + seg * SEG;
#pragma unroll
        for (int k = 0; k < SEG; k += 4) {
          float4 o = *reinterpret_cast<float4*>(dst + k);
          o.x -= acc[k]; o.y -= acc[k + 1]; o.z -= acc[k + 2]; o.w -= acc[k + 3];
          *reinterpret_cast<float4*>(dst + k) = o;
        }
      }
      GPTQ_SWEEP_MARK(5);
    }
  }
  }   // the blocks of the super-block
#pragma unroll
  for (int o = 1; o < TPR; o <<= 1) esq += __shfl_xor_sync(0xffffffffu, esq, o);
  if (err_sq && live && seg == 0) err_sq[r] += esq;
}

// ---------------------------------------------------------------------------
// K4 operand: B[c - e][k] = U[b0 + k][c] for c in [e, n), k < kw, split into its
// TF32 high part and remainder (rows of ldk, K-major for the tensor cores).
// 32 x 32 tiles through shared memory keep both the read and the write coalesced.
// ---------------------------------------------------------------------------
__global__ void u_block_transpose_split_kernel(const float* U, int n, int b0, int kw, int e, float* Bhi, float* Blo,
                                               int ldk, const int32_t* st) {
  if (has_error(st)) return;
  __shared__ float t[32][33];
  const int c0 = e + blockIdx.x * 32;      // U column tile
  const int k0 = blockIdx.y * 32;          // U row tile within the super-block
  for (int yy = threadIdx.y; yy < 32; yy += 8) {
    const int k = k0 + yy, c = c0 + threadIdx.x;
    t[yy][threadIdx.x] = (k < kw && c < n) ? U[(int64_t)(b0 + k) * n + c] : 0.f;
  }
  __syncthreads();
  for (int yy = threadIdx.y; yy < 32; yy += 8) {
    const int c = c0 + yy, k = k0 + threadIdx.x;
    if (c < n && k < ldk) {
      const float x = t[threadIdx.x][yy];
      const float h = tf32_hi(x);
      Bhi[(int64_t)(c - e) * ldk + k] = h;
      Blo[(int64_t)(c - e) * ldk + k] = x - h;
    }
  }
}

// ---------------------------------------------------------------------------
// K5: qweight[w][o] = bits of the codes of input columns k with k.bits in
// [32w, 32w + 32), original order; code of column k = codes[o][invperm[k]].
// A 32 x 32 tile of (rows o, words w) per block: a warp packs consecutive words of one
// row (reading the row's codes in order), the tile turns through shared memory, and
// a warp writes 32 consecutive o of one word.
// ---------------------------------------------------------------------------
__global__ void pack_kernel(const uint8_t* codes, const int32_t* invperm, int out, int n, int ld_codes,
                            int bits, int32_t* qweight, const int32_t* st) {
  if (has_error(st)) return;
  __shared__ uint32_t tile[32][33];
  const int words = n * bits / 32;
  const int o0 = blockIdx.x * 32, w0 = blockIdx.y * 32;
  const int tx = threadIdx.x, ty = threadIdx.y;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int o = o0 + ty + 8 * r, wi = w0 + tx;
    uint64_t acc = 0;
    if (o < out && wi < words) {
      const int pos0 = wi * 32;
      const int k_lo = pos0 / bits, k_hi = (pos0 + 31) / bits;
      const uint8_t* crow = codes + (int64_t)o * ld_codes;
      for (int k = k_lo; k <= k_hi && k < n; ++k) {
        const int src = invperm ? invperm[k] : k;
        const uint64_t c = crow[src] & ((1u << bits) - 1u);
        const int sh = k * bits - pos0;  // may be negative for a code straddling in from the left
        if (sh >= 0) acc |= c << sh; else acc |= c >> (-sh);
      }
    }
    tile[ty + 8 * r][tx] = (uint32_t)(acc & 0xFFFFFFFFull);
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int wi = w0 + ty + 8 * r, o = o0 + tx;
    if (wi < words && o < out) qweight[(int64_t)wi * out + o] = (int32_t)tile[tx][ty + 8 * r];
  }
}

// Zero points packed along the output dimension: qzeros[g][w] holds the bit stream of
// (zeros[g][o] - zero_offset) mod 2^bits for o = 0 .. out-1 (column o at stream bits
// o*bits .., codes straddling words as in qweight).  One thread per output word.  A zero
// that is not an integer in [0, 2^bits - 1] is reported (GPTQ_ERR_INVALID_ARG, info =
// group * out + column) and packed masked like the others.
__global__ void pack_zeros_kernel(const uint16_t* zeros, int groups, int out, int bits, int zero_offset,
                                  int32_t* qzeros, int32_t* st) {
  if (has_error(st)) return;
  const int words = out * bits / 32;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)groups * words) return;
  const int g = (int)(i / words), wi = (int)(i % words);
  const int pos0 = wi * 32;
  const int o_lo = pos0 / bits, o_hi = min((pos0 + 31) / bits, out - 1);
  const uint32_t mask = (1u << bits) - 1u;
  const uint16_t* zrow = zeros + (int64_t)g * out;
  uint64_t acc = 0;
  for (int o = o_lo; o <= o_hi; ++o) {
    const float z = __half2float(__ushort_as_half(zrow[o]));
    if (!(z >= 0.f && z <= (float)mask && z == rintf(z)))
      set_error(st, GPTQ_ERR_INVALID_ARG, (int)((int64_t)g * out + o), STAGE_PACK);
    const uint64_t v = (uint32_t)((int)z - zero_offset) & mask;
    const int sh = o * bits - pos0;  // negative for a code straddling in from the previous word
    if (sh >= 0) acc |= v << sh; else acc |= v >> (-sh);
  }
  qzeros[i] = (int32_t)(uint32_t)(acc & 0xFFFFFFFFull);
}

// Optional output: codes in the original column order.
__global__ void codes_out_kernel(const uint8_t* codes_p, const int32_t* invperm, int out, int n, uint8_t* codes,
                                 const int32_t* st) {
  if (has_error(st)) return;
  const int k = blockIdx.x * 32 + threadIdx.x;
  const int r = blockIdx.y * 8 + threadIdx.y;
  if (k >= n || r >= out) return;
  codes[(int64_t)r * n + k] = codes_p[(int64_t)r * n + invperm[k]];
}

}  // namespace

size_t quantize_ws_bytes(int out, int n, int block) {
  (void)block;
  return align_up((size_t)out * n * 4, 256) + 4 * align_up((size_t)out * SBK * 4, 256) +
         4 * align_up((size_t)n * SBK * 4, 256) + align_up((size_t)out * n, 256) + align_up((size_t)n * 4, 256) +
         align_up((size_t)out * 8, 256);
}

namespace {

// Two library streams per host thread and device: the sweeps and the update of the
// next super-block on a high-priority stream (the critical chain), the rest of each
// trailing update and the U operands of later super-blocks on a low-priority one.
// Created on first use, kept for the life of the process.
struct QuantStreams {
  cudaStream_t hi = nullptr, lo = nullptr;
  cudaEvent_t fork = nullptr, join_hi = nullptr, join_lo = nullptr;
  cudaEvent_t swept = nullptr;   // the latest sweep is done: its errors are complete
  cudaEvent_t near = nullptr;    // the latest next-super-block update is done with its operand buffers
  cudaEvent_t far = nullptr;     // the latest far update is done with its columns and error buffers
  cudaEvent_t opnd[2] = {};      // the U operand in buffer b is written
};

int quant_streams(QuantStreams** out) {
  thread_local QuantStreams per_dev[64];
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return GPTQ_ERR_CUDA;
  QuantStreams& q = per_dev[dev];
  if (q.hi == nullptr) {
    int least = 0, greatest = 0;
    if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess) return GPTQ_ERR_CUDA;
    if (cudaStreamCreateWithPriority(&q.hi, cudaStreamNonBlocking, greatest) != cudaSuccess ||
        cudaStreamCreateWithPriority(&q.lo, cudaStreamNonBlocking, least) != cudaSuccess)
      return GPTQ_ERR_CUDA;
    cudaEvent_t* evs[] = {&q.fork, &q.join_hi, &q.join_lo, &q.swept, &q.near, &q.far, &q.opnd[0], &q.opnd[1]};
    for (cudaEvent_t* e : evs)
      if (cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess) return GPTQ_ERR_CUDA;
  }
  *out = &q;
  return GPTQ_OK;
}

}  // namespace

int launch_pack(const uint8_t* codes, const int32_t* invperm, int out, int n, int ld_codes, int bits,
                int32_t* qweight, const int32_t* st, cudaStream_t s) {
  const int words = n * bits / 32;
  dim3 blk(32, 8), grd((unsigned)cdiv(out, 32), (unsigned)cdiv(words, 32));
  TraceScope ts("pack", "byte", (double)out * n * (1.0 + bits / 8.0) + 4.0 * n, s);
  pack_kernel<<<grd, blk, 0, s>>>(codes, invperm, out, n, ld_codes, bits, qweight, st);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

int launch_pack_zeros(const uint16_t* zeros, int groups, int out, int bits, int zero_offset, int32_t* qzeros,
                      int32_t* st, cudaStream_t s) {
  const int64_t total = (int64_t)groups * (out * bits / 32);
  pack_zeros_kernel<<<(unsigned)cdiv(total, 256), 256, 0, s>>>(zeros, groups, out, bits, zero_offset, qzeros, st);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

// The super-blocks of one layer on the two library streams (ordering: see launch_quantize).
template <typename SweepFn>
int super_block_loop(QuantStreams* q, const QuantWs& w, int out, int n, const float* U, int bits, int sym,
                     int32_t* qweight_fused, uint16_t* scales, uint16_t* zeros, float* err_sq, int32_t* st,
                     SweepFn sweep, size_t smem, int rows_per_cta, int threads) {
  int rc = GPTQ_OK;
  const int S = (int)cdiv(n, SBK);
  // U[super-block sb rows, the columns after it]^T, split, into B[sb & 1] (on lo)
  auto operand = [&](int sb) -> int {
    const int b0 = sb * SBK, be = b0 + SBK;   // sb < S - 1: a whole super-block with columns after it
    dim3 blk(32, 8), grd((unsigned)cdiv(n - be, 32), (unsigned)(SBK / 32));
    TraceScope ts_t("u_operand", "byte", 12.0 * SBK * (double)(n - be), q->lo);
    u_block_transpose_split_kernel<<<grd, blk, 0, q->lo>>>(U, n, b0, SBK, be, w.Bhi[sb & 1], w.Blo[sb & 1], SBK, st);
    GPTQ_LAUNCH_CHECK();
    GPTQ_CUDA_TRY(cudaEventRecord(q->opnd[sb & 1], q->lo));
    return GPTQ_OK;
  };
  for (int sb = 0; sb < std::min(2, S - 1); ++sb)
    if ((rc = operand(sb)) != GPTQ_OK) return rc;
  for (int sb = 0; sb < S; ++sb) {
    const int b = sb & 1;
    const int s0 = sb * SBK, se = std::min(n, s0 + SBK);
    // bytes of the section's work: W in, both error halves and the codes out, U's block
    TraceScope ts_s("sweep", "byte", (double)out * (se - s0) * 13.0 + 4.0 * (se - s0) * (se - s0), q->hi);
    sweep<<<(unsigned)cdiv(out, rows_per_cta), threads, smem, q->hi>>>(w.Wf, out, n, s0, se, U, w.Ehi[b], w.Elo[b],
                                                                    w.codes_p, qweight_fused, scales, zeros, w.rows,
                                                                    err_sq, bits, sym, st);
    GPTQ_LAUNCH_CHECK();
    if (se >= n) break;
    const int kn = std::min(SBK, n - se);   // the next super-block's width
    GPTQ_CUDA_TRY(cudaEventRecord(q->swept, q->hi));
    GPTQ_CUDA_TRY(cudaStreamWaitEvent(q->hi, q->opnd[b], 0));
    if (sb > 0) GPTQ_CUDA_TRY(cudaStreamWaitEvent(q->hi, q->far, 0));
    rc = launch_gemm3(w.Wf + se, n, out, kn, SBK, w.Ehi[b], w.Elo[b], SBK, w.Bhi[b], w.Blo[b], SBK, false, st, q->hi,
                      false, nullptr, nullptr, 0, "trailing_update");
    if (rc != GPTQ_OK) return rc;
    GPTQ_CUDA_TRY(cudaEventRecord(q->near, q->hi));
    if (n - se > kn) {
      GPTQ_CUDA_TRY(cudaStreamWaitEvent(q->lo, q->swept, 0));
      rc = launch_gemm3(w.Wf + se + kn, n, out, n - se - kn, SBK, w.Ehi[b], w.Elo[b], SBK,
                        w.Bhi[b] + (size_t)kn * SBK, w.Blo[b] + (size_t)kn * SBK, SBK, false, st, q->lo,
                        false, nullptr, nullptr, 0, "trailing_update");
      if (rc != GPTQ_OK) return rc;
    }
    GPTQ_CUDA_TRY(cudaEventRecord(q->far, q->lo));
    if (sb + 2 < S - 1) {
      GPTQ_CUDA_TRY(cudaStreamWaitEvent(q->lo, q->near, 0));
      if ((rc = operand(sb + 2)) != GPTQ_OK) return rc;
    }
  }
  return GPTQ_OK;
}

int join_streams(QuantStreams* q, cudaStream_t s) {
  GPTQ_CUDA_TRY(cudaEventRecord(q->join_hi, q->hi));
  GPTQ_CUDA_TRY(cudaEventRecord(q->join_lo, q->lo));
  GPTQ_CUDA_TRY(cudaStreamWaitEvent(s, q->join_hi, 0));
  GPTQ_CUDA_TRY(cudaStreamWaitEvent(s, q->join_lo, 0));
  return GPTQ_OK;
}

namespace {

// The whole stage enqueued on stream s (and the library's streams, joined back to s).
int enqueue_quantize(const WRows& W, int w_dtype, int out, int w_cols, int n, const float* U, const int32_t* perm,
                     const uint8_t* dead, int bits, int gs, int sym, int32_t* qweight, uint16_t* scales,
                     uint16_t* zeros, int32_t* g_idx, uint8_t* codes, float* err_sq, void* ws, int32_t* st,
                     cudaStream_t s) {
  QuantWs w = carve(ws, out, n);
  {
    dim3 blk(32, 8), grd((unsigned)cdiv(n, 128), (unsigned)cdiv(std::max(out, 1), 8));
    const double esz = w_dtype == GPTQ_F32 ? 4.0 : 2.0;
    TraceScope ts("ingest", "byte", (double)out * w_cols * esz + (double)out * n * 4.0, s);
    if (w_dtype == GPTQ_F32)
      ingest_kernel<float><<<grd, blk, 0, s>>>(W, out, w_cols, n, perm, dead, gs, w.Wf, w.invperm, g_idx, st);
    else if (w_dtype == GPTQ_F16)
      ingest_kernel<__half><<<grd, blk, 0, s>>>(W, out, w_cols, n, perm, dead, gs, w.Wf, w.invperm, g_idx, st);
    else
      ingest_kernel<__nv_bfloat16><<<grd, blk, 0, s>>>(W, out, w_cols, n, perm, dead, gs, w.Wf, w.invperm, g_idx, st);
    GPTQ_LAUNCH_CHECK();
  }
  if (err_sq) GPTQ_CUDA_TRY(cudaMemsetAsync(err_sq, 0, (size_t)out * 4, s));
  if (gs <= 0) {
    row_params_kernel<<<out, 256, 0, s>>>(w.Wf, out, n, bits, sym, w.rows, scales, zeros, st);
    GPTQ_LAUNCH_CHECK();
  }
  // Lanes per row: the sweep is a chain of dependent column steps per row, so with few
  // rows a whole warp per row (more warps per SM to hide the chain's latency), with
  // many rows 4 (less redundant work per row).
  const int tpr = out <= 2048 ? 32 : (out < 4096 ? 16 : 4);
  auto pick_gs = [&](auto tpr_tag, auto sym_tag) {
    constexpr int T = decltype(tpr_tag)::value;
    constexpr bool Y = decltype(sym_tag)::value;
    return gs == 32 ? sweep_kernel<32, T, Y> : gs == 64 ? sweep_kernel<64, T, Y>
                                             : gs == 128 ? sweep_kernel<128, T, Y> : sweep_kernel<0, T, Y>;
  };
  auto pick = [&](auto tpr_tag) {
    return sym ? pick_gs(tpr_tag, std::true_type{}) : pick_gs(tpr_tag, std::false_type{});
  };
  auto sweep = tpr == 32 ? pick(std::integral_constant<int, 32>{})
                         : tpr == 16 ? pick(std::integral_constant<int, 16>{}) : pick(std::integral_constant<int, 4>{});
  const size_t smem = tpr == 32 ? SweepShape<32>::SMEM : tpr == 16 ? SweepShape<16>::SMEM : SweepShape<4>::SMEM;
  const int rows_per_cta = tpr == 32 ? SweepShape<32>::ROWS : tpr == 16 ? SweepShape<16>::ROWS : SweepShape<4>::ROWS;
  const int threads = tpr == 32 ? SweepShape<32>::THREADS : tpr == 16 ? SweepShape<16>::THREADS
                                                                      : SweepShape<4>::THREADS;
  GPTQ_CUDA_TRY(cudaFuncSetAttribute(sweep, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  // Two-level lazy batches: blocks of 128 columns inside super-blocks of 512.  A
  // block's sweep also updates the rest of its super-block; the columns after a
  // super-block absorb its 512 errors at once on the tensor cores, as
  // Wf[:, se:] -= Err[:, super-block] . U[super-block, se:] (K = 512, accumulated by
  // the GEMM in 128-deep chunks summed in fp32 registers: one long tensor-core
  // accumulation let the codes of a 28,672-column layer drift past 0.5 %).
  // That update is split in two: the next super-block's columns on the critical
  // chain (hi), the columns after them (and the U operand of super-block s + 2) on
  // the low-priority stream, beside the next sweep.  Ordering, for super-block s
  // with buffers b = s & 1:
  //   near(s)   waits far(s - 1), which updated the same columns, and operand(s);
  //   far(s)    waits sweep(s); far(s - 1) precedes it on lo;
  //   sweep(s + 1) follows near(s) on hi, so it sees both updates of its columns;
  //   sweep(s + 2) rewrites the errors E[b]: near(s + 1) waited far(s) before it;
  //   operand(s + 2) rewrites B[b]: it waits near(s) and follows far(s) on lo.
  QuantStreams* q = nullptr;
  int rc = quant_streams(&q);
  if (rc != GPTQ_OK) return rc;
  GPTQ_CUDA_TRY(cudaEventRecord(q->fork, s));
  GPTQ_CUDA_TRY(cudaStreamWaitEvent(q->hi, q->fork, 0));
  GPTQ_CUDA_TRY(cudaStreamWaitEvent(q->lo, q->fork, 0));
  // With the identity column order (perm NULL) the sweep writes qweight itself and the
  // separate packing launch is skipped.
  int32_t* qweight_fused = perm == nullptr ? qweight : nullptr;
  rc = super_block_loop(q, w, out, n, U, bits, sym, qweight_fused, scales, zeros, err_sq, st, sweep, smem,
                        rows_per_cta, threads);
  // both library streams join the caller's stream, after an error too, so that the
  // caller's stream is ordered after everything this call enqueued
  const int jrc = join_streams(q, s);
  if (rc != GPTQ_OK) return rc;
  if (jrc != GPTQ_OK) return jrc;
  if (qweight_fused == nullptr) {
    rc = launch_pack(w.codes_p, w.invperm, out, n, n, bits, qweight, st, s);
    if (rc != GPTQ_OK) return rc;
  }
  if (codes) {
    dim3 blk(32, 8), grd((unsigned)cdiv(n, 32), (unsigned)cdiv(out, 8));
    codes_out_kernel<<<grd, blk, 0, s>>>(w.codes_p, w.invperm, out, n, codes, st);
    GPTQ_LAUNCH_CHECK();
  }
  return GPTQ_OK;
}

}  // namespace

// The stage's sweeps and trailing updates are a chain of dependent launches on two
// streams: replayed as a CUDA graph when the same arguments come again
// (run_graph_cached).  The key is every argument the launches hold by value.
int launch_quantize(const WRows& W, int w_dtype, int out, int w_cols, int n, const float* U, const int32_t* perm,
                    const uint8_t* dead, int bits, int gs, int sym, int block, int32_t* qweight,
                    uint16_t* scales, uint16_t* zeros, int32_t* g_idx, uint8_t* codes, float* err_sq,
                    void* ws, int32_t* st, cudaStream_t s) {
  (void)block;
  GraphKey key;
  key.add(2).add(W.count);
  for (int i = 0; i < W.count; ++i) key.add(W.W[i]).add(W.row0[i]);
  key.add(W.row0[W.count]).add(w_dtype).add(out).add(w_cols).add(n).add(U).add(perm).add(dead).add(bits).add(gs);
  key.add(sym).add(qweight).add(scales).add(zeros).add(g_idx).add(codes).add(err_sq).add(ws).add(st);
  return run_graph_cached(key, s, [&](cudaStream_t strm) {
    return enqueue_quantize(W, w_dtype, out, w_cols, n, U, perm, dead, bits, gs, sym, qweight, scales, zeros, g_idx,
                            codes, err_sq, ws, st, strm);
  });
}

}  // namespace gptq
