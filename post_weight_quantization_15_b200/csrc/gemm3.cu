// C -= A . B^T in fp32-level precision on the tcgen05 tensor cores (3 x TF32).
//
// The lazy trailing update of the column sweep ("polydesk.ai/glossaire/gptq",
// "Etape 3") and the trailing updates of the blocked Cholesky factorization and
// triangular inverse are dense contractions whose results feed rounding
// decisions; a single TF32 pass (10-bit mantissa) perturbs them too much.  Every
// fp32 operand x is split once, outside this kernel, into hi = x with its low 13
// mantissa bits cleared (exact in TF32) and lo = x - hi (exact in fp32), and
//     A . B^T  ~  A_hi.B_hi^T + A_hi.B_lo^T + A_lo.B_hi^T
// (the dropped A_lo.B_lo^T term is below 2^-20 of the product).
//
// One CTA computes one 128 x GN tile of C (GN = 256; 128, 64 or 32 for narrow C,
// so that a skinny product still spreads over most of the SMs):
//   warp 0      TMA producer: 32-wide K slices of A_hi, A_lo (128 rows) and
//               B_hi, B_lo (GN rows), 128-byte swizzled, 2- or 3-stage ring;
//   warp 1      allocates GN TMEM columns; one thread issues the tcgen05.mma
//               kind::tf32 instructions (M = 128, N = GN, K = 8);
//   warps 2..5  epilogue: TMEM -> registers -> C -= acc, or C = acc, and
//               optionally the TF32 split of the result (Chi, Clo) for a later
//               product.
// All operands are row-major with K contiguous (K-major).  `lower` skips tiles
// that lie entirely above the diagonal of a square C.
// Every wait is bounded (GPTQ_ERR_TIMEOUT).
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

// Timeline marks for probes; empty in the library build.
#ifndef GPTQ_GEMM_MARK
#define GPTQ_GEMM_MARK(i)
#endif

namespace gptq {

namespace {

constexpr int GM = 128;
constexpr int GK = 32;                      // fp32 per 128-byte row
constexpr int A_TILE = GM * GK * 4;         // 16 KB
constexpr int G_THREADS = 192;

// K is accumulated in chunks of CHUNK_KB k-blocks (128) for tiles up to 128 wide:
// the tensor cores' fp32 accumulation is not rounded to nearest and its error grows
// with the accumulation length, so each chunk starts from zero in one of two TMEM
// accumulators and the epilogue warps add the finished chunks in fp32 registers
// (round to nearest) while the next chunk is computed.  256-wide tiles serve
// K <= 128 only (one chunk).
constexpr int CHUNK_KB = 4;

template <int GN>
struct GemmCfg {
  static constexpr int STAGES = GN == 256 ? 2 : (GN == 128 ? 3 : 4);
  static constexpr int B_TILE = GN * GK * 4;
  static constexpr uint32_t IDESC = tc::idesc_f32acc(2, GM, GN);
  static constexpr bool CHUNKED = GN <= 128;
  static constexpr uint32_t TMEM_COLS = CHUNKED ? 2 * GN : GN;
};

template <int GN>
struct GemmSmem {
  static constexpr int ST = GemmCfg<GN>::STAGES;
  uint8_t bhi[ST][GemmCfg<GN>::B_TILE];
  uint8_t blo[ST][GemmCfg<GN>::B_TILE];
  uint8_t ahi[ST][A_TILE];
  uint8_t alo[ST][A_TILE];
  uint64_t full[ST];
  uint64_t empty[ST];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int skip;
};

__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = tc::globaltimer();
  while (!tc::mbar_try_wait(bar, parity)) {
    if (tc::globaltimer() - t0 > 1000000000ull) return false;
  }
  return true;
}

struct GemmMaps {
  CUtensorMap ahi, alo, bhi, blo;
};

struct GemmOut {
  float* C;         // may be null with store = 1 and a split: only the split is written
  int ldc;
  int store;        // 0: C -= acc, 1: C = acc
  float* Chi;       // optional TF32 split of the result (same row/column origin as C)
  float* Clo;
  int ldh;
};

__device__ __forceinline__ float tf32_hi(float x) { return __uint_as_float(__float_as_uint(x) & 0xFFFFE000u); }

template <int GN>
__global__ void __launch_bounds__(G_THREADS, 1)
gemm3_kernel(const __grid_constant__ GemmMaps maps, GemmOut out, int M, int N, int K, int lower, int tiles_n,
             int32_t* st) {
  using Cfg = GemmCfg<GN>;
  constexpr int ST = Cfg::STAGES;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // offset arithmetic on the shared array keeps every access a shared-memory one
  GemmSmem<GN>& S = *reinterpret_cast<GemmSmem<GN>*>(smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ti = blockIdx.x / tiles_n, tj = blockIdx.x % tiles_n;
  const bool skip_tile = lower && (tj * GN > ti * GM + GM - 1);
  if (skip_tile) return;                      // CTA-uniform, before any barrier or TMEM use
  const int kblocks = (int)cdiv(K, GK);
  GPTQ_GEMM_MARK(0);

  if (threadIdx.x == 0) {
    S.skip = has_error(st) ? 1 : 0;
    S.abort = 0;
    for (int s = 0; s < ST; ++s) { tc::mbar_init(&S.full[s], 1); tc::mbar_init(&S.empty[s], 1); }
    for (int b = 0; b < 2; ++b) { tc::mbar_init(&S.acc_full[b], 1); tc::mbar_init(&S.acc_empty[b], 4); }
    tc::mbar_init(&S.drain, 1);
    tc::fence_barrier_init();
  }
  if (warp == 1) tc::tmem_alloc<Cfg::TMEM_COLS>(&S.tmem_base);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  GPTQ_GEMM_MARK(1);
  const uint32_t taddr = S.tmem_base;
  const bool skip = S.skip != 0;
  volatile int* abort_flag = &S.abort;
  int armed[ST] = {};
  bool mma_committed = false;

  if (!skip) {
    if (warp == 0 && lane == 0) {
      for (int kb = 0; kb < kblocks; ++kb) {
        const int s = kb % ST;
        const uint32_t ph = (uint32_t)(kb / ST) & 1u;
        if (!tc::mbar_wait(&S.empty[s], ph ^ 1u, abort_flag)) break;
        tc::mbar_arrive_expect_tx(&S.full[s], 2 * (A_TILE + Cfg::B_TILE));
        tc::tma_load_2d(S.ahi[s], &maps.ahi, &S.full[s], kb * GK, ti * GM);
        tc::tma_load_2d(S.alo[s], &maps.alo, &S.full[s], kb * GK, ti * GM);
        tc::tma_load_2d(S.bhi[s], &maps.bhi, &S.full[s], kb * GK, tj * GN);
        tc::tma_load_2d(S.blo[s], &maps.blo, &S.full[s], kb * GK, tj * GN);
        ++armed[s];
      }
    } else if (warp == 1 && lane == 0) {
      const int chunk_kb = Cfg::CHUNKED ? CHUNK_KB : kblocks;
      const int nchunks = (int)cdiv(kblocks, chunk_kb);
      int kb = 0;
      for (int c = 0; c < nchunks && !*abort_flag; ++c) {
        const int buf = Cfg::CHUNKED ? (c & 1) : 0;
        if (Cfg::CHUNKED && !tc::mbar_wait(&S.acc_empty[buf], ((uint32_t)(c >> 1) & 1u) ^ 1u, abort_flag)) break;
        tc::tc_fence_after();
        const uint32_t dacc = taddr + buf * GN;
        const int kb_end = min(kblocks, (c + 1) * chunk_kb);
        bool first = true;
        for (; kb < kb_end; ++kb) {
          const int s = kb % ST;
          const uint32_t ph = (uint32_t)(kb / ST) & 1u;
          if (!tc::mbar_wait(&S.full[s], ph, abort_flag)) break;
          tc::tc_fence_after();
          if (kb == 0) GPTQ_GEMM_MARK(2);
          const uint32_t ah = tc::smem_u32(S.ahi[s]), al = tc::smem_u32(S.alo[s]);
          const uint32_t bh = tc::smem_u32(S.bhi[s]), bl = tc::smem_u32(S.blo[s]);
#pragma unroll
          for (int kk = 0; kk < GK / 8; ++kk) {
            const uint32_t o = kk * 32;
            tc::mma_tf32(dacc, tc::sdesc_k_sw128(al + o), tc::sdesc_k_sw128(bh + o), Cfg::IDESC, !first);
            tc::mma_tf32(dacc, tc::sdesc_k_sw128(ah + o), tc::sdesc_k_sw128(bl + o), Cfg::IDESC, true);
            tc::mma_tf32(dacc, tc::sdesc_k_sw128(ah + o), tc::sdesc_k_sw128(bh + o), Cfg::IDESC, true);
            first = false;
          }
          tc::mma_commit(&S.empty[s]);
        }
        if (*abort_flag) break;
        tc::mma_commit(&S.acc_full[buf]);
      }
      GPTQ_GEMM_MARK(3);
      tc::mma_commit(&S.drain);
      mma_committed = true;
      if (!*abort_flag) drain_wait(&S.drain, 0);
    } else if (warp >= 2) {
      const int q = warp & 3;
      const uint32_t lane_base = (uint32_t)(q * 32) << 16;
      if (!out.store && warp < 6) {   // this warp's rows of C into L2 while the product runs
        const int r = ti * GM + q * 32 + lane;
        if (r < M)
#pragma unroll
          for (int j = 0; j < GN / 32; ++j)
            if (tj * GN + 32 * j < N) asm volatile("prefetch.global.L2 [%0];" ::"l"(out.C + (int64_t)r * out.ldc + tj * GN + 32 * j));
      }
      // chunked: this thread's row of the tile (TMEM lane) in registers
      float acc[Cfg::CHUNKED ? GN : 1];
      int ready = 1;
      const int nchunks = Cfg::CHUNKED ? (int)cdiv(kblocks, CHUNK_KB) : 1;
      for (int c = 0; c < nchunks && ready; ++c) {
        const int buf = Cfg::CHUNKED ? (c & 1) : 0;
        int ok = 0;
        if (lane == 0) ok = tc::mbar_wait(&S.acc_full[buf], (uint32_t)(c >> 1) & 1u, abort_flag) && !*abort_flag;
        ready = __shfl_sync(0xffffffffu, ok, 0);
        if (!ready) break;
        tc::tc_fence_after();
        if constexpr (Cfg::CHUNKED) {
#pragma unroll
          for (int cc = 0; cc < GN / 32; ++cc) {
            float v[32];
            tc::tmem_ld_32x32b_x32(taddr + lane_base + buf * GN + cc * 32, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) acc[cc * 32 + i] = c == 0 ? v[i] : acc[cc * 32 + i] + v[i];
          }
          tc::tc_fence_before();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&S.acc_empty[buf]);
        }
      }
      if (ready) {
        if (warp == 2 && lane == 0) GPTQ_GEMM_MARK(4);
        // Each warp owns TMEM lanes (rows) [32 q, 32 q + 32).  It stages its 32 x GN
        // slice of C in shared memory (the stage buffers are free once the
        // accumulator is complete): 16-byte pieces, piece p of row rr stored at
        // slot p ^ (rr & 7), so that both the row-wise combine (lane = row) and the
        // coalesced global accesses (lane = piece) stay within 4-way bank sharing.
        constexpr int P = GN / 4;                                    // pieces per row
        float* tile = reinterpret_cast<float*>(S.bhi[0]) + q * (32 * GN);
        const int row0 = ti * GM + q * 32;
        const bool vec = out.C != nullptr && (out.ldc & 3) == 0 && (reinterpret_cast<uintptr_t>(out.C) & 15) == 0;
        auto slot = [](int rr, int p) { return rr * GN + ((p ^ (rr & 7)) << 2); };
        if (!out.store) {
          for (int g = lane; g < 32 * P; g += 32) {
            const int rr = g / P, p = g % P;
            const int r = row0 + rr, col = tj * GN + 4 * p;
            float* dst = tile + slot(rr, p);
            if (vec && r < M && col + 3 < N) {
              asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(tc::smem_u32(dst)),
                           "l"(out.C + (int64_t)r * out.ldc + col)
                           : "memory");
            } else {
#pragma unroll
              for (int e = 0; e < 4; ++e)
                dst[e] = (r < M && col + e < N) ? out.C[(int64_t)r * out.ldc + col + e] : 0.f;
            }
          }
          asm volatile("cp.async.wait_all;" ::: "memory");
          __syncwarp();
        }
#pragma unroll
        for (int c = 0; c < GN / 32; ++c) {
          float v[32];
          if constexpr (Cfg::CHUNKED) {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = acc[c * 32 + i];
          } else {
            tc::tmem_ld_32x32b_x32(taddr + lane_base + c * 32, v);
          }
          // lane = row: combine with C
#pragma unroll
          for (int pp = 0; pp < 8; ++pp) {
            float* e = tile + slot(lane, 8 * c + pp);
            float4 x = *reinterpret_cast<float4*>(e);
            if (out.store) x = make_float4(v[4 * pp], v[4 * pp + 1], v[4 * pp + 2], v[4 * pp + 3]);
            else x = make_float4(x.x - v[4 * pp], x.y - v[4 * pp + 1], x.z - v[4 * pp + 2], x.w - v[4 * pp + 3]);
            *reinterpret_cast<float4*>(e) = x;
          }
        }
        __syncwarp();
        // lane = piece: coalesced stores of C and of its split
        for (int g = lane; g < 32 * P; g += 32) {
          const int rr = g / P, p = g % P;
          const int r = row0 + rr, col = tj * GN + 4 * p;
          if (r >= M || col >= N) continue;
          const float4 x = *reinterpret_cast<const float4*>(tile + slot(rr, p));
          const float xs[4] = {x.x, x.y, x.z, x.w};
          if (out.C == nullptr) {
            // split only
          } else if (vec && col + 3 < N) {
            *reinterpret_cast<float4*>(out.C + (int64_t)r * out.ldc + col) = x;
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (col + e < N) out.C[(int64_t)r * out.ldc + col + e] = xs[e];
          }
          if (out.Chi != nullptr) {
            float hs[4], ls[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) { hs[e] = tf32_hi(xs[e]); ls[e] = xs[e] - hs[e]; }
            if ((out.ldh & 3) == 0 && col + 3 < N) {
              *reinterpret_cast<float4*>(out.Chi + (int64_t)r * out.ldh + col) = make_float4(hs[0], hs[1], hs[2], hs[3]);
              *reinterpret_cast<float4*>(out.Clo + (int64_t)r * out.ldh + col) = make_float4(ls[0], ls[1], ls[2], ls[3]);
            } else {
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                if (col + e < N) {
                  out.Chi[(int64_t)r * out.ldh + col + e] = hs[e];
                  out.Clo[(int64_t)r * out.ldh + col + e] = ls[e];
                }
              }
            }
          }
        }
      }
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  GPTQ_GEMM_MARK(5);
  if (*abort_flag) {
    if (warp == 0 && lane == 0) {
      for (int s = 0; s < ST; ++s)
        if (armed[s] > 0) drain_wait(&S.full[s], (uint32_t)(armed[s] - 1) & 1u);
    }
    if (warp == 1 && lane == 0 && mma_committed) drain_wait(&S.drain, 0);
    if (threadIdx.x == 0) set_error(st, GPTQ_ERR_TIMEOUT, blockIdx.x, STAGE_TRAILING);
    __syncthreads();
  }
  if (warp == 1) {
    __syncwarp();
    tc::tmem_dealloc<Cfg::TMEM_COLS>(taddr);
  }
}

// ---------------------------------------------------------------------------
// The persistent form for products at least 256 columns wide: one CTA per SM walks
// its share of the 128 x 256 output tiles (t = blockIdx.x, blockIdx.x + gridDim.x,
// ...).  The stage ring, the chunk counter and the two TMEM accumulators run on
// across tiles, so the producer loads the next tile's operands and the MMAs start
// it while the epilogue warps still update C with the previous one.
//   warp 0      TMA producer: 16-wide K slices of A hi / lo (128 rows) and B hi / lo
//               (256 rows), 64-byte swizzled, 4-stage ring of 48 KB stages;
//   warp 1      allocates 512 TMEM columns (two 128 x 256 accumulators); one thread
//               issues tcgen05.mma kind::tf32 (M = 128, N = 256, K = 8), three per
//               K step (lo.hi + hi.lo + hi.hi);
//   warps 2..9  epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 32 (its rows) and
//               columns 128 ((w - 2) / 4) .. + 128, adds each 128-deep chunk into fp32
//               registers, releases the accumulator, and at a tile's last chunk
//               updates its rows of C (C -= acc or C = acc; optionally the split of
//               the result), 32 columns at a time turned through a 32 x 32 staging
//               tile in 16-byte pieces (update_c_rows); the tile's rows of C are
//               requested into L2 when the tile starts.
// K is accumulated in chunks of 128 (as in gemm3_kernel), each from zero.  Every
// wait is bounded (GPTQ_ERR_TIMEOUT).
// ---------------------------------------------------------------------------
constexpr int PN = 256;
constexpr int PK = 16;                           // fp32 per 64-byte row: 16-deep K slices
constexpr int PST = 4;
constexpr int P_ATILE = GM * PK * 4;             // 8 KB
constexpr int P_BTILE = PN * PK * 4;             // 16 KB
constexpr int P_CHUNK_KB = CHUNK_KB * GK / PK;   // slices per 128-deep accumulation chunk
constexpr int P_EPI = 8;
constexpr int P_THREADS = 64 + P_EPI * 32;
constexpr uint32_t P_IDESC = tc::idesc_f32acc(2, GM, PN);

constexpr int P_LDT = 33;                       // an epilogue warp's staging tile: 32 x 33 floats

// The L2 lines of this warp's rows of C for the tile, requested when the tile starts so
// that its update at the tile's end reads L2 rather than DRAM.
__device__ __forceinline__ void prefetch_c_rows(const GemmOut& out, int M, int N, int row0, int col0, int lane) {
  const int r = row0 + lane;
  if (out.store || r >= M) return;
  const float* base = out.C + (int64_t)r * out.ldc + col0;
#pragma unroll
  for (int j = 0; j < 4; ++j)
    if (col0 + 32 * j < N) asm volatile("prefetch.global.L2 [%0];" ::"l"(base + 32 * j));
}

// C -= acc (or C = acc; optionally the TF32 split of the result) for this warp's 32 rows
// [row0, +32) and 128 columns [col0, +128), acc holding one row per lane.  32 columns at a
// time go through the warp's 32 x 32 staging tile in 16-byte pieces, piece p of row rr at
// slot p ^ (rr & 7), so that the global accesses are 16-byte and coalesced (lane = piece)
// and the combine (lane = row) shares banks at most 4 ways.
__device__ __forceinline__ void update_c_rows(const GemmOut& out, int M, int N, int row0, int col0,
                                              const float (&acc)[128], float* tile, int lane) {
  auto slot = [](int rr, int p) { return rr * 32 + ((p ^ (rr & 7)) << 2); };
  const bool vec_c = out.C != nullptr && (out.ldc & 3) == 0 && (reinterpret_cast<uintptr_t>(out.C) & 15) == 0;
  const bool vec_h = out.Chi != nullptr && (out.ldh & 3) == 0 && (reinterpret_cast<uintptr_t>(out.Chi) & 15) == 0 &&
                     (reinterpret_cast<uintptr_t>(out.Clo) & 15) == 0;
  const int pr = lane & 7;                     // this lane's piece in the coalesced passes
#pragma unroll
  for (int c4 = 0; c4 < 4; ++c4) {             // unrolled: acc stays in registers
    const int colb = col0 + c4 * 32;
    __syncwarp();
    if (!out.store) {
#pragma unroll 1
      for (int it = 0; it < 8; ++it) {
        const int rr = it * 4 + (lane >> 3);
        const int r = row0 + rr, col = colb + 4 * pr;
        float* dst = tile + slot(rr, pr);
        if (vec_c && r < M && col + 3 < N) {
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(tc::smem_u32(dst)),
                       "l"(out.C + (int64_t)r * out.ldc + col)
                       : "memory");
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = (r < M && col + e < N) ? out.C[(int64_t)r * out.ldc + col + e] : 0.f;
        }
      }
      asm volatile("cp.async.wait_all;" ::: "memory");
    }
    __syncwarp();
    // the row owner combines its 32 values
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      float4* e = reinterpret_cast<float4*>(tile + slot(lane, p));
      const float* a = acc + c4 * 32 + 4 * p;
      float4 x = *e;
      if (out.store) x = make_float4(a[0], a[1], a[2], a[3]);
      else x = make_float4(x.x - a[0], x.y - a[1], x.z - a[2], x.w - a[3]);
      *e = x;
    }
    __syncwarp();
#pragma unroll 1
    for (int it = 0; it < 8; ++it) {
      const int rr = it * 4 + (lane >> 3);
      const int r = row0 + rr, col = colb + 4 * pr;
      if (r >= M || col >= N) continue;
      const float4 x = *reinterpret_cast<const float4*>(tile + slot(rr, pr));
      const float xe[4] = {x.x, x.y, x.z, x.w};
      if (out.C) {
        float* d = out.C + (int64_t)r * out.ldc + col;
        if (vec_c && col + 3 < N) *reinterpret_cast<float4*>(d) = x;
        else
#pragma unroll
          for (int e = 0; e < 4; ++e) if (col + e < N) d[e] = xe[e];
      }
      if (out.Chi != nullptr) {
        float h[4], l[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) { h[e] = tf32_hi(xe[e]); l[e] = xe[e] - h[e]; }
        float* dh = out.Chi + (int64_t)r * out.ldh + col;
        float* dl = out.Clo + (int64_t)r * out.ldh + col;
        if (vec_h && col + 3 < N) {
          *reinterpret_cast<float4*>(dh) = make_float4(h[0], h[1], h[2], h[3]);
          *reinterpret_cast<float4*>(dl) = make_float4(l[0], l[1], l[2], l[3]);
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (col + e < N) { dh[e] = h[e]; dl[e] = l[e]; }
        }
      }
    }
  }
}

struct GemmPSmem {
  uint8_t bhi[PST][P_BTILE];
  uint8_t blo[PST][P_BTILE];
  uint8_t ahi[PST][P_ATILE];
  uint8_t alo[PST][P_ATILE];
  float tr[P_EPI][32 * P_LDT];                  // per epilogue warp: 32 rows x 32 columns, turned
  uint64_t full[PST];
  uint64_t empty[PST];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int skip;
};
constexpr size_t GEMMP_SMEM = sizeof(GemmPSmem) + 1024;

// Tile t of the walk -> (ti, tj).  lower: only tiles that reach the lower triangle of
// square C, tj . 256 <= ti . 128 + 127, i.e. tj <= ti / 2, row by row.
__device__ __forceinline__ void gemmp_tile(int t, int tiles_n, bool lower, int& ti, int& tj) {
  if (!lower) { ti = t / tiles_n; tj = t % tiles_n; return; }
  ti = 0;
  for (;;) {
    const int cnt = min(ti / 2 + 1, tiles_n);
    if (t < cnt) break;
    t -= cnt;
    ++ti;
  }
  tj = t;
}

__global__ void __launch_bounds__(P_THREADS, 1)
gemm3p_kernel(const __grid_constant__ GemmMaps maps, GemmOut out, int M, int N, int K, int lower, int tiles,
              int tiles_n, int32_t* st) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // offset arithmetic on the shared array keeps every access a shared-memory one
  GemmPSmem& S = *reinterpret_cast<GemmPSmem*>(smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kblocks = (int)cdiv(K, PK);
  const int nchunks = (int)cdiv(kblocks, P_CHUNK_KB);      // 128-deep chunks per tile

  if (threadIdx.x == 0) {
    S.skip = has_error(st) ? 1 : 0;
    S.abort = 0;
    for (int s2 = 0; s2 < PST; ++s2) { tc::mbar_init(&S.full[s2], 1); tc::mbar_init(&S.empty[s2], 1); }
    for (int b = 0; b < 2; ++b) { tc::mbar_init(&S.acc_full[b], 1); tc::mbar_init(&S.acc_empty[b], P_EPI); }
    tc::mbar_init(&S.drain, 1);
    tc::fence_barrier_init();
  }
  if (warp == 1) tc::tmem_alloc<512>(&S.tmem_base);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t taddr = S.tmem_base;
  const bool skip = S.skip != 0;
  volatile int* abort_flag = &S.abort;
  int armed[PST] = {};
  bool mma_committed = false;

  if (!skip) {
    if (warp == 0 && lane == 0) {
      // ---------------- producer ----------------
      int q = 0;                                           // stage counter over all tiles
      for (int t = blockIdx.x; t < tiles && !*abort_flag; t += gridDim.x) {
        int ti, tj;
        gemmp_tile(t, tiles_n, lower != 0, ti, tj);
        for (int kb = 0; kb < kblocks; ++kb, ++q) {
          const int s2 = q % PST;
          const uint32_t ph = (uint32_t)(q / PST) & 1u;
          if (!tc::mbar_wait(&S.empty[s2], ph ^ 1u, abort_flag)) break;
          tc::mbar_arrive_expect_tx(&S.full[s2], 2 * (P_ATILE + P_BTILE));
          tc::tma_load_2d(S.ahi[s2], &maps.ahi, &S.full[s2], kb * PK, ti * GM);
          tc::tma_load_2d(S.alo[s2], &maps.alo, &S.full[s2], kb * PK, ti * GM);
          tc::tma_load_2d(S.bhi[s2], &maps.bhi, &S.full[s2], kb * PK, tj * PN);
          tc::tma_load_2d(S.blo[s2], &maps.blo, &S.full[s2], kb * PK, tj * PN);
          ++armed[s2];
        }
      }
    } else if (warp == 1 && lane == 0) {
      // ---------------- MMA issuer ----------------
      int q = 0, g = 0;                                    // stage and chunk counters over all tiles
      for (int t = blockIdx.x; t < tiles && !*abort_flag; t += gridDim.x) {
        int kb = 0;
        for (int c = 0; c < nchunks && !*abort_flag; ++c, ++g) {
          const int buf = g & 1;
          if (!tc::mbar_wait(&S.acc_empty[buf], ((uint32_t)(g >> 1) & 1u) ^ 1u, abort_flag)) break;
          tc::tc_fence_after();
          const uint32_t dacc = taddr + buf * PN;
          const int kb_end = min(kblocks, (c + 1) * P_CHUNK_KB);
          bool first = true;
          for (; kb < kb_end; ++kb, ++q) {
            const int s2 = q % PST;
            const uint32_t ph = (uint32_t)(q / PST) & 1u;
            if (!tc::mbar_wait(&S.full[s2], ph, abort_flag)) break;
            tc::tc_fence_after();
            const uint32_t ah = tc::smem_u32(S.ahi[s2]), al = tc::smem_u32(S.alo[s2]);
            const uint32_t bh = tc::smem_u32(S.bhi[s2]), bl = tc::smem_u32(S.blo[s2]);
#pragma unroll
            for (int kk = 0; kk < PK / 8; ++kk) {
              const uint32_t o = kk * 32;
              tc::mma_tf32(dacc, tc::sdesc_k_sw64(al + o), tc::sdesc_k_sw64(bh + o), P_IDESC, !first);
              tc::mma_tf32(dacc, tc::sdesc_k_sw64(ah + o), tc::sdesc_k_sw64(bl + o), P_IDESC, true);
              tc::mma_tf32(dacc, tc::sdesc_k_sw64(ah + o), tc::sdesc_k_sw64(bh + o), P_IDESC, true);
              first = false;
            }
            tc::mma_commit(&S.empty[s2]);
          }
          if (*abort_flag) break;
          tc::mma_commit(&S.acc_full[buf]);
        }
      }
      tc::mma_commit(&S.drain);
      mma_committed = true;
      if (!*abort_flag) drain_wait(&S.drain, 0);
    } else if (warp >= 2) {
      // ---------------- epilogue ----------------
      const int qq = warp & 3;                   // TMEM lane quarter this warp may access
      const int hc = (warp - 2) >> 2;            // which 128 of the 256 columns
      const uint32_t lane_base = (uint32_t)(qq * 32) << 16;
      int g = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x) {
        int ti, tj;
        gemmp_tile(t, tiles_n, lower != 0, ti, tj);
        // this warp's rows [row0, row0 + 32) and columns [col0, col0 + 128) of C
        const int row0 = ti * GM + qq * 32;
        const int col0 = tj * PN + hc * 128;
        prefetch_c_rows(out, M, N, row0, col0, lane);
        float acc[128];
#pragma unroll
        for (int i = 0; i < 128; ++i) acc[i] = 0.f;
        for (int c = 0; c < nchunks; ++c, ++g) {
          const int buf = g & 1;
          int ready = 0;
          if (lane == 0) ready = tc::mbar_wait(&S.acc_full[buf], (uint32_t)(g >> 1) & 1u, abort_flag) && !*abort_flag;
          ready = __shfl_sync(0xffffffffu, ready, 0);
          if (!ready) { ok = false; break; }
          tc::tc_fence_after();
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            float v[32];
            tc::tmem_ld_32x32b_x32(taddr + lane_base + buf * PN + hc * 128 + c4 * 32, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) acc[c4 * 32 + i] += v[i];
          }
          tc::tc_fence_before();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&S.acc_empty[buf]);   // the MMAs may reuse it now
        }
        if (!ok) break;
        update_c_rows(out, M, N, row0, col0, acc, S.tr[warp - 2], lane);
      }
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    if (warp == 0 && lane == 0) {
      for (int s2 = 0; s2 < PST; ++s2)
        if (armed[s2] > 0) drain_wait(&S.full[s2], (uint32_t)(armed[s2] - 1) & 1u);
    }
    if (warp == 1 && lane == 0 && mma_committed) drain_wait(&S.drain, 0);
    if (threadIdx.x == 0) set_error(st, GPTQ_ERR_TIMEOUT, blockIdx.x, STAGE_TRAILING);
    __syncthreads();
  }
  if (warp == 1) {
    __syncwarp();
    tc::tmem_dealloc<512>(taddr);
  }
}

// ---------------------------------------------------------------------------
// The persistent form on CTA pairs (cta_group::2): a cluster of two CTAs on two SMs
// computes 256 x 256 tiles.  Each CTA loads its own 128 rows of A and its half (128
// rows) of B; the even CTA (the leader) issues tcgen05.mma.cta_group::2 kind::tf32
// M = 256, N = 256, K = 8, which reads both CTAs' shared memory at the same offsets
// and leaves each CTA's 128 rows of the accumulator in its own TMEM.  Per flop each
// CTA loads two thirds of the operand bytes of the 128 x 256 form.  Otherwise as
// gemm3p_kernel: the stage ring (five 32 KB stages of 16-deep K slices), the chunk
// counter and the two TMEM accumulators run on across tiles, and each CTA's eight
// epilogue warps update its 128 rows of C.
// Protocol (that of the Hessian's pair kernel; every wait bounded):
//   full[s]      leader only: the leader's producer arrives with both CTAs' bytes;
//                both producers' loads complete on it.
//   empty[s]     both CTAs, count 1: the leader's commit reaches both.
//   acc_full[b]  both CTAs, count 1: a commit to both after a chunk's MMAs.
//   acc_empty[b] leader only, 2 x P_EPI arrivals (the peer's through the cluster address).
//   drain        leader: every MMA complete before teardown.
// A cluster barrier after the barriers' initialisation and another before TMEM is
// freed.  No load uses cluster multicast.
// ---------------------------------------------------------------------------
constexpr int Q_ST = 5;
constexpr int Q_ATILE = GM * PK * 4;             // 8 KB: this CTA's 128 rows of A (hi or lo)
constexpr int Q_BTILE = (PN / 2) * PK * 4;       // 8 KB: this CTA's 128 rows of B (hi or lo)
constexpr uint32_t Q_IDESC = tc::idesc_f32acc(2, 2 * GM, PN);

struct GemmQSmem {
  uint8_t ahi[Q_ST][Q_ATILE];
  uint8_t alo[Q_ST][Q_ATILE];
  uint8_t bhi[Q_ST][Q_BTILE];
  uint8_t blo[Q_ST][Q_BTILE];
  float tr[P_EPI][32 * P_LDT];
  uint64_t full[Q_ST];
  uint64_t empty[Q_ST];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int skip;
};
constexpr size_t GEMMQ_SMEM = sizeof(GemmQSmem) + 1024;

// Pair tile t -> (ti, tj) over 256 x 256 tiles.  lower: only tiles that reach the lower
// triangle (the diagonal starts top left), tj <= ti, row by row.
__device__ __forceinline__ void gemmq_tile(int t, int tiles_n, bool lower, int& ti, int& tj) {
  if (!lower) { ti = t / tiles_n; tj = t % tiles_n; return; }
  ti = 0;
  for (;;) {
    const int cnt = min(ti + 1, tiles_n);
    if (t < cnt) break;
    t -= cnt;
    ++ti;
  }
  tj = t;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(P_THREADS, 1)
gemm3pp_kernel(const __grid_constant__ GemmMaps maps, GemmOut out, int M, int N, int K, int lower, int tiles,
               int tiles_n, int32_t* st) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // offset arithmetic on the shared array keeps every access a shared-memory one (and
  // gives both CTAs the same offsets)
  GemmQSmem& S = *reinterpret_cast<GemmQSmem*>(smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = tc::cluster_rank();
  const bool leader = rank == 0;
  const int pair = (int)(blockIdx.x >> 1), npairs = (int)(gridDim.x >> 1);
  const int kblocks = (int)cdiv(K, PK);
  const int nchunks = (int)cdiv(kblocks, P_CHUNK_KB);      // 128-deep chunks per tile
  const uint32_t stage_tx = 2u * 2u * (uint32_t)(Q_ATILE + Q_BTILE);   // both CTAs, hi and lo

  if (threadIdx.x == 0) {
    S.skip = has_error(st) ? 1 : 0;
    S.abort = 0;
    for (int s2 = 0; s2 < Q_ST; ++s2) { tc::mbar_init(&S.full[s2], 1); tc::mbar_init(&S.empty[s2], 1); }
    for (int b = 0; b < 2; ++b) { tc::mbar_init(&S.acc_full[b], 1); tc::mbar_init(&S.acc_empty[b], 2 * P_EPI); }
    tc::mbar_init(&S.drain, 1);
    tc::fence_barrier_init();
  }
  if (warp == 1) tc::tmem_alloc_pair<512>(&S.tmem_base);
  tc::tc_fence_before();
  __syncthreads();
  tc::cluster_sync();                            // both CTAs' barriers exist before any remote signal
  tc::tc_fence_after();
  const uint32_t taddr = S.tmem_base;
  // (if the two CTAs disagree here, the waiting side's bounded waits run out)
  const bool skip = S.skip != 0;
  volatile int* abort_flag = &S.abort;
  int armed[Q_ST] = {};
  bool mma_committed = false;

  if (!skip) {
    if (warp == 0 && lane == 0) {
      // ---------------- producer (both CTAs) ----------------
      int q = 0;                                           // stage counter over all tiles
      for (int t = pair; t < tiles && !*abort_flag; t += npairs) {
        int ti, tj;
        gemmq_tile(t, tiles_n, lower != 0, ti, tj);
        const int a_row = ti * 2 * GM + (int)rank * GM;
        const int b_row = tj * PN + (int)rank * (PN / 2);
        for (int kb = 0; kb < kblocks; ++kb, ++q) {
          const int s2 = q % Q_ST;
          const uint32_t ph = (uint32_t)(q / Q_ST) & 1u;
          if (!tc::mbar_wait(&S.empty[s2], ph ^ 1u, abort_flag)) break;
          if (leader) tc::mbar_arrive_expect_tx(&S.full[s2], stage_tx);
          tc::tma_load_2d_pair(S.ahi[s2], &maps.ahi, &S.full[s2], kb * PK, a_row);
          tc::tma_load_2d_pair(S.alo[s2], &maps.alo, &S.full[s2], kb * PK, a_row);
          tc::tma_load_2d_pair(S.bhi[s2], &maps.bhi, &S.full[s2], kb * PK, b_row);
          tc::tma_load_2d_pair(S.blo[s2], &maps.blo, &S.full[s2], kb * PK, b_row);
          ++armed[s2];
        }
      }
    } else if (warp == 1 && lane == 0 && leader) {
      // ---------------- MMA issuer (leader) ----------------
      int q = 0, g = 0;                                    // stage and chunk counters over all tiles
      for (int t = pair; t < tiles && !*abort_flag; t += npairs) {
        int kb = 0;
        for (int c = 0; c < nchunks && !*abort_flag; ++c, ++g) {
          const int buf = g & 1;
          if (!tc::mbar_wait(&S.acc_empty[buf], ((uint32_t)(g >> 1) & 1u) ^ 1u, abort_flag)) break;
          tc::tc_fence_after();
          const uint32_t dacc = taddr + buf * PN;
          const int kb_end = min(kblocks, (c + 1) * P_CHUNK_KB);
          bool first = true;
          for (; kb < kb_end; ++kb, ++q) {
            const int s2 = q % Q_ST;
            const uint32_t ph = (uint32_t)(q / Q_ST) & 1u;
            if (!tc::mbar_wait(&S.full[s2], ph, abort_flag)) break;
            tc::tc_fence_after();
            const uint32_t ah = tc::smem_u32(S.ahi[s2]), al = tc::smem_u32(S.alo[s2]);
            const uint32_t bh = tc::smem_u32(S.bhi[s2]), bl = tc::smem_u32(S.blo[s2]);
#pragma unroll
            for (int kk = 0; kk < PK / 8; ++kk) {
              const uint32_t o = kk * 32;
              tc::mma_tf32_pair(dacc, tc::sdesc_k_sw64(al + o), tc::sdesc_k_sw64(bh + o), Q_IDESC, !first);
              tc::mma_tf32_pair(dacc, tc::sdesc_k_sw64(ah + o), tc::sdesc_k_sw64(bl + o), Q_IDESC, true);
              tc::mma_tf32_pair(dacc, tc::sdesc_k_sw64(ah + o), tc::sdesc_k_sw64(bh + o), Q_IDESC, true);
              first = false;
            }
            tc::mma_commit_pair_both(&S.empty[s2]);
          }
          if (*abort_flag) break;
          tc::mma_commit_pair_both(&S.acc_full[buf]);
        }
      }
      tc::mma_commit_pair_local(&S.drain);
      mma_committed = true;
      if (!*abort_flag) drain_wait(&S.drain, 0);
    } else if (warp >= 2) {
      // ---------------- epilogue (both CTAs) ----------------
      const int qq = warp & 3;                   // TMEM lane quarter this warp may access
      const int hc = (warp - 2) >> 2;            // which 128 of the 256 columns
      const uint32_t lane_base = (uint32_t)(qq * 32) << 16;
      const uint32_t acc_empty_leader[2] = {tc::map_to_cta(tc::smem_u32(&S.acc_empty[0]), 0),
                                            tc::map_to_cta(tc::smem_u32(&S.acc_empty[1]), 0)};
      int g = 0;
      bool ok = true;
      for (int t = pair; t < tiles && ok; t += npairs) {
        int ti, tj;
        gemmq_tile(t, tiles_n, lower != 0, ti, tj);
        // this CTA's and warp's rows [row0, row0 + 32) and columns [col0, col0 + 128) of C
        const int row0 = ti * 2 * GM + (int)rank * GM + qq * 32;
        const int col0 = tj * PN + hc * 128;
        prefetch_c_rows(out, M, N, row0, col0, lane);
        float acc[128];
#pragma unroll
        for (int i = 0; i < 128; ++i) acc[i] = 0.f;
        for (int c = 0; c < nchunks; ++c, ++g) {
          const int buf = g & 1;
          int ready = 0;
          if (lane == 0) ready = tc::mbar_wait(&S.acc_full[buf], (uint32_t)(g >> 1) & 1u, abort_flag) && !*abort_flag;
          ready = __shfl_sync(0xffffffffu, ready, 0);
          if (!ready) { ok = false; break; }
          tc::tc_fence_after();
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            float v[32];
            tc::tmem_ld_32x32b_x32(taddr + lane_base + buf * PN + hc * 128 + c4 * 32, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) acc[c4 * 32 + i] += v[i];
          }
          tc::tc_fence_before();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive_cluster(acc_empty_leader[buf]);   // the MMAs may reuse it now
        }
        if (!ok) break;
        update_c_rows(out, M, N, row0, col0, acc, S.tr[warp - 2], lane);
      }
    }
  }

  // ---------------- teardown ----------------
  tc::tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    if (leader && warp == 0 && lane == 0) {
      // the leader's full barriers count both CTAs' bytes: bounded drain of its armed phases
      for (int s2 = 0; s2 < Q_ST; ++s2)
        if (armed[s2] > 0) drain_wait(&S.full[s2], (uint32_t)(armed[s2] - 1) & 1u);
    }
    if (warp == 1 && lane == 0 && mma_committed) drain_wait(&S.drain, 0);
    if (threadIdx.x == 0) set_error(st, GPTQ_ERR_TIMEOUT, blockIdx.x, STAGE_TRAILING);
    // the peer's loads complete on the leader's barriers, which the peer cannot wait on:
    // give copies in flight a fixed, bounded time before either CTA leaves
    if (threadIdx.x == 0) {
      const uint64_t t0 = tc::globaltimer();
      while (tc::globaltimer() - t0 < 20000000ull) {
      }
    }
    __syncthreads();
  }
  tc::cluster_sync();                            // neither CTA leaves while the other may touch its memory
  tc::tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tc::tmem_dealloc_pair<512>(taddr);
  }
}

// hi = x with the low 13 mantissa bits cleared, lo = x - hi.
__global__ void split_tf32_kernel(const float* X, int rows, int cols, int ldx, float* hi, float* lo, int ldo,
                                  const int32_t* st) {
  if (has_error(st)) return;
  const int c = blockIdx.x * 32 + threadIdx.x;
  const int r = blockIdx.y * 8 + threadIdx.y;
  if (r >= rows || c >= cols) return;
  const float x = X[(int64_t)r * ldx + c];
  const float h = __uint_as_float(__float_as_uint(x) & 0xFFFFE000u);
  hi[(int64_t)r * ldo + c] = h;
  lo[(int64_t)r * ldo + c] = x - h;
}

int launch_split_tf32_impl(const float* X, int rows, int cols, int ldx, float* hi, float* lo, int ldo,
                      const int32_t* st, cudaStream_t s) {
  if (rows <= 0 || cols <= 0) return GPTQ_OK;
  dim3 blk(32, 8), grd((unsigned)cdiv(cols, 32), (unsigned)cdiv(rows, 8));
  split_tf32_kernel<<<grd, blk, 0, s>>>(X, rows, cols, ldx, hi, lo, ldo, st);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

template <int GN>
int launch_gemm3_t(const GemmOut& out, int M, int N, int K, const float* Ahi, const float* Alo, int lda,
                   const float* Bhi, const float* Blo, int ldb, bool lower, int32_t* st, cudaStream_t s) {
  GemmMaps maps;
  int rc = make_tmap_2d(&maps.ahi, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, Ahi, (uint64_t)K, (uint64_t)M,
                        (uint64_t)lda * 4, GK, GM, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc == GPTQ_OK)
    rc = make_tmap_2d(&maps.alo, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, Alo, (uint64_t)K, (uint64_t)M, (uint64_t)lda * 4,
                      GK, GM, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc == GPTQ_OK)
    rc = make_tmap_2d(&maps.bhi, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, Bhi, (uint64_t)K, (uint64_t)N, (uint64_t)ldb * 4,
                      GK, GN, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc == GPTQ_OK)
    rc = make_tmap_2d(&maps.blo, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, Blo, (uint64_t)K, (uint64_t)N, (uint64_t)ldb * 4,
                      GK, GN, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc != GPTQ_OK) return rc;
  const int tm = (int)cdiv(M, GM), tn = (int)cdiv(N, GN);
  const size_t smem = sizeof(GemmSmem<GN>) + 1024;
  GPTQ_CUDA_TRY(cudaFuncSetAttribute(gemm3_kernel<GN>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  gemm3_kernel<GN><<<tm * tn, G_THREADS, smem, s>>>(maps, out, M, N, K, lower ? 1 : 0, tn, st);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

int launch_gemm3p(const GemmOut& out, int M, int N, int K, const float* Ahi, const float* Alo, int lda,
                  const float* Bhi, const float* Blo, int ldb, bool lower, int32_t* st, cudaStream_t s) {
  GemmMaps maps;
  int rc = make_tmap_2d(&maps.ahi, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, Ahi, (uint64_t)K, (uint64_t)M,
                        (uint64_t)lda * 4, PK, GM, CU_TENSOR_MAP_SWIZZLE_64B);
  if (rc == GPTQ_OK)
    rc = make_tmap_2d(&maps.alo, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, Alo, (uint64_t)K, (uint64_t)M, (uint64_t)lda * 4,
                      PK, GM, CU_TENSOR_MAP_SWIZZLE_64B);
  if (rc == GPTQ_OK)
    rc = make_tmap_2d(&maps.bhi, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, Bhi, (uint64_t)K, (uint64_t)N, (uint64_t)ldb * 4,
                      PK, PN, CU_TENSOR_MAP_SWIZZLE_64B);
  if (rc == GPTQ_OK)
    rc = make_tmap_2d(&maps.blo, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, Blo, (uint64_t)K, (uint64_t)N, (uint64_t)ldb * 4,
                      PK, PN, CU_TENSOR_MAP_SWIZZLE_64B);
  if (rc != GPTQ_OK) return rc;
  const int tm = (int)cdiv(M, GM), tn = (int)cdiv(N, PN);
  int tiles = 0;
  if (lower) {
    for (int ti = 0; ti < tm; ++ti) tiles += std::min(ti / 2 + 1, tn);
  } else {
    tiles = tm * tn;
  }
  if (tiles == 0) return GPTQ_OK;
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                 cudaSuccess)
      return GPTQ_ERR_CUDA;
  }
  GPTQ_CUDA_TRY(cudaFuncSetAttribute(gemm3p_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)GEMMP_SMEM));
  gemm3p_kernel<<<std::min(tiles, sms), P_THREADS, GEMMP_SMEM, s>>>(maps, out, M, N, K, lower ? 1 : 0, tiles, tn, st);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

int launch_gemm3pp(const GemmOut& out, int M, int N, int K, const float* Ahi, const float* Alo, int lda,
                   const float* Bhi, const float* Blo, int ldb, bool lower, int64_t tiles, int32_t* st,
                   cudaStream_t s) {
  GemmMaps maps;
  int rc = make_tmap_2d(&maps.ahi, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, Ahi, (uint64_t)K, (uint64_t)M,
                        (uint64_t)lda * 4, PK, GM, CU_TENSOR_MAP_SWIZZLE_64B);
  if (rc == GPTQ_OK)
    rc = make_tmap_2d(&maps.alo, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, Alo, (uint64_t)K, (uint64_t)M, (uint64_t)lda * 4,
                      PK, GM, CU_TENSOR_MAP_SWIZZLE_64B);
  if (rc == GPTQ_OK)
    rc = make_tmap_2d(&maps.bhi, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, Bhi, (uint64_t)K, (uint64_t)N, (uint64_t)ldb * 4,
                      PK, PN / 2, CU_TENSOR_MAP_SWIZZLE_64B);
  if (rc == GPTQ_OK)
    rc = make_tmap_2d(&maps.blo, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, Blo, (uint64_t)K, (uint64_t)N, (uint64_t)ldb * 4,
                      PK, PN / 2, CU_TENSOR_MAP_SWIZZLE_64B);
  if (rc != GPTQ_OK) return rc;
  static int sms = 0;
  if (sms == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
                                                 cudaSuccess)
      return GPTQ_ERR_CUDA;
  }
  const int pairs = (int)std::min<int64_t>(tiles, sms / 2);
  GPTQ_CUDA_TRY(cudaFuncSetAttribute(gemm3pp_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)GEMMQ_SMEM));
  gemm3pp_kernel<<<2 * pairs, P_THREADS, GEMMQ_SMEM, s>>>(maps, out, M, N, K, lower ? 1 : 0, (int)tiles,
                                                           (int)cdiv(N, PN), st);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

}  // namespace

int launch_split_tf32(const float* X, int rows, int cols, int ldx, float* hi, float* lo, int ldo,
                      const int32_t* st, cudaStream_t s) {
  return launch_split_tf32_impl(X, rows, cols, ldx, hi, lo, ldo, st, s);
}

int launch_gemm3(float* C, int ldc, int M, int N, int K, const float* Ahi, const float* Alo, int lda,
                 const float* Bhi, const float* Blo, int ldb, bool lower, int32_t* st, cudaStream_t s,
                 bool store, float* Chi, float* Clo, int ldh, const char* trace) {
  if (M <= 0 || N <= 0 || K <= 0) return GPTQ_OK;
  GemmOut out{C, ldc, store ? 1 : 0, Chi, Clo, ldh};
  // useful flops of the product (lower: about the tiles that reach the lower triangle)
  const double flop = 2.0 * M * N * K * (lower ? 0.5 : 1.0);
  TraceScope ts(trace ? trace : "gemm3", "flop", flop, s);
  // the widest tile that still gives about one CTA per SM; K beyond one chunk takes
  // the chunked (<= 128-wide) tiles
  const int64_t tm = (int64_t)cdiv(M, GM);
  // Products with at least two waves of 128 x 256 tiles (296 on 148 SMs): the persistent
  // form.  Below that, the 128-wide tiles of gemm3_kernel give more CTAs, which the
  // measured layers preferred (1024-row far updates, the trailing updates at n = 4096).
  const int64_t tnw = (int64_t)cdiv(N, PN);
  int64_t wide_tiles = tm * tnw;
  if (lower) {   // the 128 x 256 tiles that reach the lower triangle (tall C: the diagonal starts top left)
    wide_tiles = 0;
    for (int64_t ti = 0; ti < tm; ++ti) wide_tiles += std::min(ti / 2 + 1, tnw);
  }
  // Two waves of 256 x 256 tiles on the CTA pairs (148 on 74 pairs): the pair form
  const int64_t tqm = (int64_t)cdiv(M, 2 * GM);
  int64_t pair_tiles = tqm * tnw;
  if (lower) {
    pair_tiles = 0;
    for (int64_t ti = 0; ti < tqm; ++ti) pair_tiles += std::min(ti + 1, tnw);
  }
  if (N >= PN && pair_tiles >= 148)
    return launch_gemm3pp(out, M, N, K, Ahi, Alo, lda, Bhi, Blo, ldb, lower, pair_tiles, st, s);
  if (N >= PN && wide_tiles >= 296)
    return launch_gemm3p(out, M, N, K, Ahi, Alo, lda, Bhi, Blo, ldb, lower, st, s);
  if (K > CHUNK_KB * GK) return launch_gemm3_t<128>(out, M, N, K, Ahi, Alo, lda, Bhi, Blo, ldb, lower, st, s);
  if (N <= 128 && tm * (int64_t)cdiv(N, 64) < 148)
    return launch_gemm3_t<32>(out, M, N, K, Ahi, Alo, lda, Bhi, Blo, ldb, lower, st, s);
  if (N <= 128 && tm * (int64_t)cdiv(N, 128) < 148)
    return launch_gemm3_t<64>(out, M, N, K, Ahi, Alo, lda, Bhi, Blo, ldb, lower, st, s);
  if (N <= 128) return launch_gemm3_t<128>(out, M, N, K, Ahi, Alo, lda, Bhi, Blo, ldb, lower, st, s);
  return launch_gemm3_t<256>(out, M, N, K, Ahi, Alo, lda, Bhi, Blo, ldb, lower, st, s);
}

}  // namespace gptq
