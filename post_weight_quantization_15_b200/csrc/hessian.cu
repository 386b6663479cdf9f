// K1: H += 2 . X . X^T  ("polydesk.ai/glossaire/gptq", "Etape 2": H = 2.X.X^T),
// a dense contraction over the calibration tokens on the tcgen05 tensor cores.
//
// hessian_diag64_kernel: the act-order key, 2 . sum_t x_it^2 in fp64 (every bf16
// square is exact in fp64).
#include <stdlib.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

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

// ---------------------------------------------------------------------------
// Tensor-core tile product.  One CTA computes one 128 x 256 tile of 2.X.X^T
// (rows [128 bi, +128), columns [256 bj, +256), for tiles that reach the upper
// triangle) over all tokens:
//   warp 0      TMA producer: 64 tokens of the 128 A rows and 256 B rows per
//               stage (128-byte swizzled rows), 4-stage ring;
//   warp 1      allocates 512 TMEM columns (two 128 x 256 fp32 accumulators) and
//               one thread issues tcgen05.mma (bf16 x bf16 -> fp32, M=128, N=256);
//   warps 2..9  epilogue.
// The tensor cores' fp32 accumulation is not rounded to nearest, and its error
// grows with the number of accumulation steps.  So the MMA accumulates chunks of
// 1024 tokens from zero into the two TMEM accumulators alternately, and the
// epilogue warps add each finished chunk into fp32 registers (round to nearest)
// while the next chunk is computed.  At the end H += 2 . acc.
// When the A rows lie inside the B rows (tiles on the diagonal) only the B tile
// is loaded and A reads its half of it.
// Every wait is bounded; a wait that gives up raises GPTQ_ERR_TIMEOUT, drains the
// copies and MMAs in flight (again bounded) and frees TMEM.
// ---------------------------------------------------------------------------
constexpr int HBM_ = 128;                     // tile rows (A)
constexpr int HBN = 256;                      // tile columns (B)
constexpr int HKB = 64;                       // tokens per stage (128 bytes of bf16)
constexpr int HSTAGES = 4;
constexpr int CHUNK_KB = 16;                  // stages per accumulation chunk (1024 tokens)
constexpr int A_BYTES = HBM_ * HKB * 2;       // 16 KB
constexpr int B_BYTES = HBN * HKB * 2;        // 32 KB
constexpr uint32_t HESS_IDESC = tc::idesc_f32acc(1, 128, 256);
constexpr int EPI_WARPS = 8;
constexpr int HESS_THREADS = 64 + EPI_WARPS * 32;

struct HessSmem {
  uint8_t b[HSTAGES][B_BYTES];
  uint8_t a[HSTAGES][A_BYTES];
  uint64_t full[HSTAGES];
  uint64_t empty[HSTAGES];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int skip;
};
constexpr size_t HESS_SMEM = sizeof(HessSmem) + 1024;

__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = tc::globaltimer();
  while (!tc::mbar_try_wait(bar, parity)) {
    if (tc::globaltimer() - t0 > 1000000000ull) return false;
  }
  return true;
}

// Tiles (bi, bj) with 256 bj + 255 >= 128 bi, i.e. bj >= bi / 2, row-major.
__device__ __forceinline__ void hess_tile(int t, int TB, int& bi, int& bj) {
  bi = 0;
  for (;;) {
    const int cnt = TB - bi / 2;
    if (t < cnt) break;
    t -= cnt;
    ++bi;
  }
  bj = bi / 2 + t;
}

__global__ void __launch_bounds__(HESS_THREADS, 1)
hessian_tc_kernel(const __grid_constant__ CUtensorMap tmap, float* H, int n, int kblocks, int32_t* st, int stall,
                  uint64_t wait_ns) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // offset arithmetic on the shared array keeps every access a shared-memory one
  HessSmem& S = *reinterpret_cast<HessSmem*>(smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int TB = (int)cdiv(n, HBN);
  int bi, bj;
  hess_tile(blockIdx.x, TB, bi, bj);
  const bool inside = (bi / 2) == bj;          // A rows are half of the B rows
  const int a_half = bi & 1;
  const int nchunks = (int)cdiv(kblocks, CHUNK_KB);

  if (threadIdx.x == 0) {
    S.skip = has_error(st) ? 1 : 0;
    S.abort = 0;
    for (int s = 0; s < HSTAGES; ++s) { tc::mbar_init(&S.full[s], 1); tc::mbar_init(&S.empty[s], 1); }
    for (int b = 0; b < 2; ++b) { tc::mbar_init(&S.acc_full[b], 1); tc::mbar_init(&S.acc_empty[b], EPI_WARPS); }
    tc::mbar_init(&S.drain, 1);
    tc::fence_barrier_init();
    tc::prefetch_tensormap(&tmap);
  }
  if (warp == 1) tc::tmem_alloc<512>(&S.tmem_base);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t taddr = S.tmem_base;
  const bool skip = S.skip != 0;
  volatile int* abort_flag = &S.abort;

  int armed[HSTAGES] = {0, 0, 0, 0};
  bool mma_committed = false;

  if (!skip) {
    if (warp == 0 && lane == 0) {
      // ---------------- producer ----------------
      // (stall: the failure test withholds every load so that the MMA side's
      // bounded wait runs out)
      for (int kb = 0; kb < kblocks && !stall; ++kb) {
        const int s = kb % HSTAGES;
        const uint32_t ph = (uint32_t)(kb / HSTAGES) & 1u;
        if (!tc::mbar_wait(&S.empty[s], ph ^ 1u, abort_flag, wait_ns)) break;
        tc::mbar_arrive_expect_tx(&S.full[s], inside ? B_BYTES : A_BYTES + B_BYTES);
        tc::tma_load_2d(S.b[s], &tmap, &S.full[s], kb * HKB, bj * HBN);
        tc::tma_load_2d(S.b[s] + A_BYTES, &tmap, &S.full[s], kb * HKB, bj * HBN + HBM_);
        if (!inside) tc::tma_load_2d(S.a[s], &tmap, &S.full[s], kb * HKB, bi * HBM_);
        ++armed[s];
      }
    } else if (warp == 1 && lane == 0) {
      // ---------------- MMA issuer ----------------
      int kb = 0;
      for (int c = 0; c < nchunks && !*abort_flag; ++c) {
        const int buf = c & 1;
        if (!tc::mbar_wait(&S.acc_empty[buf], ((uint32_t)(c >> 1) & 1u) ^ 1u, abort_flag, wait_ns)) break;
        tc::tc_fence_after();
        const int kb_end = min(kblocks, (c + 1) * CHUNK_KB);
        bool first = true;
        for (; kb < kb_end; ++kb) {
          const int s = kb % HSTAGES;
          const uint32_t ph = (uint32_t)(kb / HSTAGES) & 1u;
          if (!tc::mbar_wait(&S.full[s], ph, abort_flag, wait_ns)) break;
          tc::tc_fence_after();
          const uint32_t b0 = tc::smem_u32(S.b[s]);
          const uint32_t a0 = inside ? b0 + a_half * (HBM_ * 128) : tc::smem_u32(S.a[s]);
#pragma unroll
          for (int kk = 0; kk < HKB / 16; ++kk) {
            tc::mma_f16(taddr + buf * HBN, tc::sdesc_k_sw128(a0 + kk * 32), tc::sdesc_k_sw128(b0 + kk * 32),
                        HESS_IDESC, !first);
            first = false;
          }
          tc::mma_commit(&S.empty[s]);
        }
        if (*abort_flag) break;
        tc::mma_commit(&S.acc_full[buf]);
      }
      // Track every MMA this thread issued; wait for them before teardown so that
      // no tcgen05 arrival can land after the CTA's shared memory is released.
      tc::mma_commit(&S.drain);
      mma_committed = true;
      if (!*abort_flag) drain_wait(&S.drain, 0);
    } else if (warp >= 2) {
      // ---------------- epilogue ----------------
      const int q = warp & 3;                  // TMEM lane quarter this warp may access
      const int hc = (warp - 2) >> 2;          // which 128 of the 256 columns
      const uint32_t lane_base = (uint32_t)(q * 32) << 16;
      float acc[128];
#pragma unroll
      for (int i = 0; i < 128; ++i) acc[i] = 0.f;
      bool ok = true;
      for (int c = 0; c < nchunks; ++c) {
        const int buf = c & 1;
        int ready = 0;
        if (lane == 0) ready = tc::mbar_wait(&S.acc_full[buf], (uint32_t)(c >> 1) & 1u, abort_flag, wait_ns);
        ready = __shfl_sync(0xffffffffu, ready, 0);
        if (!ready) { ok = false; break; }
        tc::tc_fence_after();
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          float v[32];
          tc::tmem_ld_32x32b_x32(taddr + lane_base + buf * HBN + hc * 128 + c4 * 32, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) acc[c4 * 32 + i] += v[i];
        }
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&S.acc_empty[buf]);
      }
      if (ok && !*abort_flag) {
        const int row = bi * HBM_ + q * 32 + lane;
        const int col0 = bj * HBN + hc * 128;
        if (row < n && col0 < n) {
          float* dst = H + (int64_t)row * n + col0;
          if ((n & 3) == 0 && col0 + 128 <= n) {
#pragma unroll
            for (int i = 0; i < 128; i += 4) {
              float4 o = *reinterpret_cast<float4*>(dst + i);
              o.x = fmaf(2.f, acc[i], o.x); o.y = fmaf(2.f, acc[i + 1], o.y);
              o.z = fmaf(2.f, acc[i + 2], o.z); o.w = fmaf(2.f, acc[i + 3], o.w);
              *reinterpret_cast<float4*>(dst + i) = o;
            }
          } else {
#pragma unroll
            for (int i = 0; i < 128; ++i)
              if (col0 + i < n) dst[i] = fmaf(2.f, acc[i], dst[i]);
          }
        }
      }
    }
  }

  // ---------------- teardown ----------------
  tc::tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    // drain what this CTA still has in flight before its shared memory and TMEM go away
    if (warp == 0 && lane == 0) {
      for (int s = 0; s < HSTAGES; ++s)
        if (armed[s] > 0) drain_wait(&S.full[s], (uint32_t)(armed[s] - 1) & 1u);
    }
    if (warp == 1 && lane == 0 && mma_committed) drain_wait(&S.drain, 0);
    if (threadIdx.x == 0) set_error(st, GPTQ_ERR_TIMEOUT, blockIdx.x, STAGE_HESSIAN);
    __syncthreads();
  }
  if (warp == 1) {
    __syncwarp();
    tc::tmem_dealloc<512>(taddr);
  }
}

// ---------------------------------------------------------------------------
// The same product on CTA pairs (tcgen05 cta_group::2), for n >= 256.  One cluster
// of two CTAs computes a 256 x 256 tile of 2.X.X^T, (bi, bj) with bi <= bj in
// 256-blocks: CTA r of the pair owns rows [256 bi + 128 r, +128) (its half of A) and
// loads rows [256 bj + 128 r, +128) (its half of B); the leader (r = 0) issues
// M256 x N256 x K16 MMAs that read both halves of A and B from the two CTAs' shared
// memory and leave each CTA's 128 rows x 256 columns in its own TMEM.  Per CTA and
// 64-token stage the TMA writes 32 KB and the MMAs read 32 KB of shared memory,
// against 48 + 48 KB for the single-CTA 128 x 256 tile: shared memory, which bounds
// the single-CTA kernel, moves a third less per flop.  Accumulation as above: chunks
// of 1024 tokens in two alternating TMEM accumulators, added in fp32 registers (a
// chunk's MMAs take much longer than the epilogue's turnaround of the other
// accumulator: measured 0.665 of the bf16 peak with 256-token chunks, 0.744 with 512,
// 0.787 with 1024, the accumulation error bound growing with the chunk).
//
// Protocol (every wait bounded, as in the single-CTA kernel):
//   full[s]      leader only.  The leader's producer arrives with expect_tx of both
//                CTAs' bytes; both producers' loads complete_tx on it.
//   empty[s]     both CTAs, count 1: the leader's commit reaches both.
//   acc_full[b]  both CTAs, count 1: a commit to both after a chunk's MMAs.
//   acc_empty[b] leader only, count 2 x EPI_WARPS: both CTAs' epilogue warps arrive
//                (the peer's through the cluster address) once they have read it.
//   drain        leader: every MMA complete before teardown.
//   Start: barriers initialised and fenced, then a cluster barrier, so no remote
//   arrival precedes an init.  End: a cluster barrier after the leader's drain, so
//   neither CTA leaves while the other's MMAs or arrivals may touch it; then both
//   free TMEM.
// Tiles go in bands of PAIR_BAND block rows, column by column inside a band, so
// that the clusters running at once share their rows of X in L2.
// ---------------------------------------------------------------------------
constexpr int P_M = 128;                        // rows per CTA (A), 256 per pair
constexpr int P_N = 256;                        // tile columns (B), 128 rows of B per CTA
constexpr int P_STAGES = 7;
constexpr int PA_BYTES = P_M * HKB * 2;         // 16 KB
constexpr int PB_BYTES = (P_N / 2) * HKB * 2;   // 16 KB (this CTA's half of B)
constexpr uint32_t PAIR_IDESC = tc::idesc_f32acc(1, 256, 256);
constexpr int PAIR_BAND = 8;

struct PairSmem {
  uint8_t a[P_STAGES][PA_BYTES];
  uint8_t b[P_STAGES][PB_BYTES];
  uint64_t full[P_STAGES];
  uint64_t empty[P_STAGES];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int skip;
};
constexpr size_t PAIR_SMEM = sizeof(PairSmem) + 1024;

// Pair tile t -> (bi, bj), 0 <= bi <= bj < T: bands of PAIR_BAND block rows; inside a
// band, block column by block column, the band's rows that reach the upper triangle.
__device__ __forceinline__ void pair_tile(int t, int T, int& bi, int& bj) {
  for (int b0 = 0; b0 < T; b0 += PAIR_BAND) {
    const int b1 = min(T, b0 + PAIR_BAND), h = b1 - b0;
    const int tri = h * (h + 1) / 2;            // columns inside the band: a triangle
    const int total = tri + (T - b1) * h;
    if (t >= total) { t -= total; continue; }
    if (t < tri) {
      int j = 0;
      while (t >= j + 1) { t -= j + 1; ++j; }
      bi = b0 + t;
      bj = b0 + j;
      return;
    }
    t -= tri;
    bi = b0 + t % h;
    bj = b1 + t / h;
    return;
  }
  bi = bj = 0;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(HESS_THREADS, 1)
hessian_pair_kernel(const __grid_constant__ CUtensorMap tmap, float* H, int n, int kblocks, int32_t* st, int stall,
                    uint64_t wait_ns) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // offset arithmetic on the shared array keeps every access a shared-memory one (and
  // gives both CTAs the same offsets: the same dynamic layout, the same alignment)
  PairSmem& S = *reinterpret_cast<PairSmem*>(smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = tc::cluster_rank();
  const bool leader = rank == 0;

  const int T = (int)cdiv(n, 256);
  int bi, bj;
  pair_tile((int)(blockIdx.x >> 1), T, bi, bj);
  const bool diag = bi == bj;                   // this CTA's A rows are its B rows
  const int a_row0 = bi * 256 + (int)rank * P_M;
  const int b_row0 = bj * 256 + (int)rank * (P_N / 2);
  const int nchunks = (int)cdiv(kblocks, CHUNK_KB);
  const uint32_t stage_tx = 2u * (uint32_t)(diag ? PB_BYTES : PA_BYTES + PB_BYTES);   // both CTAs' bytes

  if (threadIdx.x == 0) {
    S.skip = has_error(st) ? 1 : 0;
    S.abort = 0;
    for (int s2 = 0; s2 < P_STAGES; ++s2) { tc::mbar_init(&S.full[s2], 1); tc::mbar_init(&S.empty[s2], 1); }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&S.acc_full[b], 1);
      tc::mbar_init(&S.acc_empty[b], 2 * EPI_WARPS);
    }
    tc::mbar_init(&S.drain, 1);
    tc::fence_barrier_init();
    tc::prefetch_tensormap(&tmap);
  }
  if (warp == 1) tc::tmem_alloc_pair<512>(&S.tmem_base);
  tc::tc_fence_before();
  __syncthreads();
  tc::cluster_sync();                           // both CTAs' barriers exist before any remote signal
  tc::tc_fence_after();
  const uint32_t taddr = S.tmem_base;
  // (if the two CTAs disagree here, the waiting side's bounded waits run out)
  const bool skip = S.skip != 0;
  volatile int* abort_flag = &S.abort;

  int armed[P_STAGES] = {};
  bool mma_committed = false;

  if (!skip) {
    if (warp == 0 && lane == 0) {
      // ---------------- producer (both CTAs) ----------------
      for (int kb = 0; kb < kblocks && !stall; ++kb) {
        const int s2 = kb % P_STAGES;
        const uint32_t ph = (uint32_t)(kb / P_STAGES) & 1u;
        if (!tc::mbar_wait(&S.empty[s2], ph ^ 1u, abort_flag, wait_ns)) break;
        if (leader) tc::mbar_arrive_expect_tx(&S.full[s2], stage_tx);
        tc::tma_load_2d_pair(S.b[s2], &tmap, &S.full[s2], kb * HKB, b_row0);
        if (!diag) tc::tma_load_2d_pair(S.a[s2], &tmap, &S.full[s2], kb * HKB, a_row0);
        ++armed[s2];
      }
    } else if (warp == 1 && lane == 0 && leader) {
      // ---------------- MMA issuer (leader) ----------------
      int kb = 0;
      for (int c = 0; c < nchunks && !*abort_flag; ++c) {
        const int buf = c & 1;
        if (!tc::mbar_wait(&S.acc_empty[buf], ((uint32_t)(c >> 1) & 1u) ^ 1u, abort_flag, wait_ns)) break;
        tc::tc_fence_after();
        const int kb_end = min(kblocks, (c + 1) * CHUNK_KB);
        bool first = true;
        for (; kb < kb_end; ++kb) {
          const int s2 = kb % P_STAGES;
          const uint32_t ph = (uint32_t)(kb / P_STAGES) & 1u;
          if (!tc::mbar_wait(&S.full[s2], ph, abort_flag, wait_ns)) break;
          tc::tc_fence_after();
          const uint32_t b0 = tc::smem_u32(S.b[s2]);
          const uint32_t a0 = diag ? b0 : tc::smem_u32(S.a[s2]);
#pragma unroll
          for (int kk = 0; kk < HKB / 16; ++kk) {
            tc::mma_f16_pair(taddr + buf * P_N, tc::sdesc_k_sw128(a0 + kk * 32), tc::sdesc_k_sw128(b0 + kk * 32),
                             PAIR_IDESC, !first);
            first = false;
          }
          tc::mma_commit_pair_both(&S.empty[s2]);
        }
        if (*abort_flag) break;
        tc::mma_commit_pair_both(&S.acc_full[buf]);
      }
      tc::mma_commit_pair_local(&S.drain);
      mma_committed = true;
      if (!*abort_flag) drain_wait(&S.drain, 0);
    } else if (warp >= 2) {
      // ---------------- epilogue (both CTAs) ----------------
      const int q = warp & 3;                  // TMEM lane quarter this warp may access
      const int hc = (warp - 2) >> 2;          // which 128 of the 256 columns
      const uint32_t lane_base = (uint32_t)(q * 32) << 16;
      const uint32_t acc_empty_leader[2] = {tc::map_to_cta(tc::smem_u32(&S.acc_empty[0]), 0),
                                            tc::map_to_cta(tc::smem_u32(&S.acc_empty[1]), 0)};
      float acc[128];
#pragma unroll
      for (int i = 0; i < 128; ++i) acc[i] = 0.f;
      bool ok = true;
      for (int c = 0; c < nchunks; ++c) {
        const int buf = c & 1;
        int ready = 0;
        if (lane == 0) ready = tc::mbar_wait(&S.acc_full[buf], (uint32_t)(c >> 1) & 1u, abort_flag, wait_ns);
        ready = __shfl_sync(0xffffffffu, ready, 0);
        if (!ready) { ok = false; break; }
        tc::tc_fence_after();
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          float v[32];
          tc::tmem_ld_32x32b_x32(taddr + lane_base + buf * P_N + hc * 128 + c4 * 32, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) acc[c4 * 32 + i] += v[i];
        }
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive_cluster(acc_empty_leader[buf]);
      }
      if (ok && !*abort_flag) {
        const int row = a_row0 + q * 32 + lane;
        const int col0 = bj * 256 + hc * 128;
        if (row < n && col0 < n) {
          float* dst = H + (int64_t)row * n + col0;
          if ((n & 3) == 0 && col0 + 128 <= n) {
#pragma unroll
            for (int i = 0; i < 128; i += 4) {
              float4 o = *reinterpret_cast<float4*>(dst + i);
              o.x = fmaf(2.f, acc[i], o.x); o.y = fmaf(2.f, acc[i + 1], o.y);
              o.z = fmaf(2.f, acc[i + 2], o.z); o.w = fmaf(2.f, acc[i + 3], o.w);
              *reinterpret_cast<float4*>(dst + i) = o;
            }
          } else {
#pragma unroll
            for (int i = 0; i < 128; ++i)
              if (col0 + i < n) dst[i] = fmaf(2.f, acc[i], dst[i]);
          }
        }
      }
    }
  }

  // ---------------- teardown ----------------
  tc::tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    if (leader && warp == 0 && lane == 0) {
      // the leader's full barriers count both CTAs' bytes: bounded drain of its armed phases
      for (int s2 = 0; s2 < P_STAGES; ++s2)
        if (armed[s2] > 0) drain_wait(&S.full[s2], (uint32_t)(armed[s2] - 1) & 1u);
    }
    if (warp == 1 && lane == 0 && mma_committed) drain_wait(&S.drain, 0);
    if (threadIdx.x == 0) set_error(st, GPTQ_ERR_TIMEOUT, blockIdx.x, STAGE_HESSIAN);
    // the peer's loads complete on the leader's barriers, which the peer cannot wait on,
    // and the leader cannot drain phases it never armed: give copies in flight a fixed,
    // bounded time (they take microseconds) before either CTA leaves
    if (threadIdx.x == 0) {
      const uint64_t t0 = tc::globaltimer();
      while (tc::globaltimer() - t0 < 20000000ull) {
      }
    }
    __syncthreads();
  }
  tc::cluster_sync();                           // neither CTA leaves while the other may touch its memory
  tc::tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tc::tmem_dealloc_pair<512>(taddr);
  }
}

}  // namespace

int launch_hessian_diag64(double* hdiag, int n, const void* X, int64_t ld_x, int64_t tokens,
                          int32_t* st, cudaStream_t s) {
  TraceScope ts("hessian_diag64", "byte", 2.0 * n * (double)tokens, s);
  hessian_diag64_kernel<<<n, DIAG_THREADS, 0, s>>>(hdiag, n, static_cast<const __nv_bfloat16*>(X), ld_x,
                                                   tokens, st);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

int launch_hessian(float* H, int n, const void* X, int x_rows, int64_t ld_x, int64_t tokens, int32_t* st,
                   cudaStream_t s) {
  CUtensorMap map;
  // One map serves both operands: its box is 64 tokens x 128 rows; the B tile is two boxes.
  // The map holds X's x_rows rows; tiles reaching rows x_rows .. n-1 (zero padding) load
  // the map's zero fill, so those rows and columns of H receive nothing.
  int rc = make_tmap_2d(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, (uint64_t)tokens, (uint64_t)x_rows,
                        (uint64_t)ld_x * 2, HKB, HBM_, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc != GPTQ_OK) return rc;
  const int TB = (int)cdiv(n, HBN);
  const int TA = (int)cdiv(n, HBM_);
  int tiles = 0;
  for (int bi = 0; bi < TA; ++bi) tiles += TB - bi / 2;
  const int kblocks = (int)cdiv(tokens, HKB);
  // Failure test switch (host side, read per call): GPTQ_FAULT_INJECT=hessian_stall
  // withholds the operand loads and shortens the wait limit to 200 ms, so the
  // kernel's bounded waits run out and it reports GPTQ_ERR_TIMEOUT.
  const char* fi = getenv("GPTQ_FAULT_INJECT");
  const int stall = (fi != nullptr && strcmp(fi, "hessian_stall") == 0) ? 1 : 0;
  const uint64_t wait_ns = stall ? 200000000ull : tc::kWaitLimitNs;
  // the algorithm's flops: the upper triangle (diagonal included) of the x_rows real rows
  TraceScope ts("hessian_tc", "flop", (double)x_rows * (x_rows + 1) * (double)tokens, s);
  if (n >= 256) {
    // CTA pairs: 256 x 256 tiles of the upper triangle, two CTAs (one cluster) each
    const int T = (int)cdiv(n, 256);
    const int pairs = T * (T + 1) / 2;
    GPTQ_CUDA_TRY(cudaFuncSetAttribute(hessian_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)PAIR_SMEM));
    hessian_pair_kernel<<<2 * pairs, HESS_THREADS, PAIR_SMEM, s>>>(map, H, n, kblocks, st, stall, wait_ns);
    GPTQ_LAUNCH_CHECK();
    return GPTQ_OK;
  }
  GPTQ_CUDA_TRY(cudaFuncSetAttribute(hessian_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)HESS_SMEM));
  hessian_tc_kernel<<<tiles, HESS_THREADS, HESS_SMEM, s>>>(map, H, n, kblocks, st, stall, wait_ns);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

}  // namespace gptq
