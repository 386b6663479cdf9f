// C[M, N] = A[M, K] . B[N, K]^T in bf16 x bf16 -> fp32 on the tcgen05 tensor cores:
// the products of a quantized block's forward pass (the dequantized weights times
// the activations), for the sequential pipeline in which each layer is calibrated on
// the outputs of the layers quantized before it ("polydesk.ai/glossaire/gptq": GPTQ
// proceeds layer by layer).
//
// One CTA computes one 128 x 256 tile of C (rows [128 bi, +128) of A, rows
// [256 bj, +256) of B) over all of K.  Tiles are walked in bands of `band` row
// tiles, column by column inside a band, so that the CTAs running at once share
// their B tiles and the band's rows of A stay in L2: B is read from HBM once per
// band instead of once per row tile (B, the activations, is the large operand).
// The kernel has the structure of the Hessian kernel:
//   warp 0      TMA producer: 64-wide K slices of the 128 A rows and 256 B rows,
//               128-byte swizzled, 4-stage ring;
//   warp 1      allocates 512 TMEM columns (two 128 x 256 fp32 accumulators); one
//               thread issues tcgen05.mma kind::f16 (M = 128, N = 256, K = 16);
//   warps 2..9  epilogue.
// K is accumulated in chunks of 256 from zero in the two TMEM accumulators in turn,
// and the epilogue warps add each finished chunk into fp32 registers (the tensor
// cores' accumulation is not rounded to nearest; its error grows with its length).
// C = acc is stored (fp32, row stride ldc).  Every wait is bounded (GPTQ_ERR_TIMEOUT).
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace gptq {

namespace {

constexpr int LM = 128;
constexpr int LN = 256;
constexpr int LKB = 64;
constexpr int LSTAGES = 4;
constexpr int LCHUNK = 4;
constexpr int LA_BYTES = LM * LKB * 2;
constexpr int LB_BYTES = LN * LKB * 2;
constexpr uint32_t LIN_IDESC = tc::idesc_f32acc(1, LM, LN);
constexpr int LEPI = 8;
constexpr int LTHREADS = 64 + LEPI * 32;

struct LinSmem {
  uint8_t a[LSTAGES][LA_BYTES];
  uint8_t b[LSTAGES][LB_BYTES];
  uint64_t full[LSTAGES];
  uint64_t empty[LSTAGES];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int skip;
};
constexpr size_t LIN_SMEM = sizeof(LinSmem) + 1024;

__device__ __forceinline__ bool lin_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = tc::globaltimer();
  while (!tc::mbar_try_wait(bar, parity)) {
    if (tc::globaltimer() - t0 > 1000000000ull) return false;
  }
  return true;
}

__global__ void __launch_bounds__(LTHREADS, 1)
linear_kernel(const __grid_constant__ CUtensorMap ta, const __grid_constant__ CUtensorMap tb, float* C, int M, int N,
              int64_t ldc, int tiles_m, int tiles_n, int band, int kblocks, int32_t* st) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // offset arithmetic on the shared array keeps every access a shared-memory one
  LinSmem& S = *reinterpret_cast<LinSmem*>(smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per_band = band * tiles_n;
  const int b0 = (int)blockIdx.x / per_band * band;          // the band's first row tile
  const int rows = min(band, tiles_m - b0);                   // row tiles in this band
  const int r = (int)blockIdx.x % per_band;
  const int bi = b0 + r % rows, bj = r / rows;
  const int nchunks = (int)cdiv(kblocks, LCHUNK);

  if (threadIdx.x == 0) {
    S.skip = has_error(st) ? 1 : 0;
    S.abort = 0;
    for (int s = 0; s < LSTAGES; ++s) { tc::mbar_init(&S.full[s], 1); tc::mbar_init(&S.empty[s], 1); }
    for (int b = 0; b < 2; ++b) { tc::mbar_init(&S.acc_full[b], 1); tc::mbar_init(&S.acc_empty[b], LEPI); }
    tc::mbar_init(&S.drain, 1);
    tc::fence_barrier_init();
    tc::prefetch_tensormap(&ta);
    tc::prefetch_tensormap(&tb);
  }
  if (warp == 1) tc::tmem_alloc<512>(&S.tmem_base);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t taddr = S.tmem_base;
  const bool skip = S.skip != 0;
  volatile int* abort_flag = &S.abort;
  int armed[LSTAGES] = {0, 0, 0, 0};
  bool mma_committed = false;

  if (!skip) {
    if (warp == 0 && lane == 0) {
      for (int kb = 0; kb < kblocks; ++kb) {
        const int s = kb % LSTAGES;
        const uint32_t ph = (uint32_t)(kb / LSTAGES) & 1u;
        if (!tc::mbar_wait(&S.empty[s], ph ^ 1u, abort_flag)) break;
        tc::mbar_arrive_expect_tx(&S.full[s], LA_BYTES + LB_BYTES);
        tc::tma_load_2d(S.a[s], &ta, &S.full[s], kb * LKB, bi * LM);
        tc::tma_load_2d(S.b[s], &tb, &S.full[s], kb * LKB, bj * LN);
        tc::tma_load_2d(S.b[s] + LB_BYTES / 2, &tb, &S.full[s], kb * LKB, bj * LN + LN / 2);
        ++armed[s];
      }
    } else if (warp == 1 && lane == 0) {
      int kb = 0;
      for (int c = 0; c < nchunks && !*abort_flag; ++c) {
        const int buf = c & 1;
        if (!tc::mbar_wait(&S.acc_empty[buf], ((uint32_t)(c >> 1) & 1u) ^ 1u, abort_flag)) break;
        tc::tc_fence_after();
        const int kb_end = min(kblocks, (c + 1) * LCHUNK);
        bool first = true;
        for (; kb < kb_end; ++kb) {
          const int s = kb % LSTAGES;
          const uint32_t ph = (uint32_t)(kb / LSTAGES) & 1u;
          if (!tc::mbar_wait(&S.full[s], ph, abort_flag)) break;
          tc::tc_fence_after();
          const uint32_t a0 = tc::smem_u32(S.a[s]), b0 = tc::smem_u32(S.b[s]);
#pragma unroll
          for (int kk = 0; kk < LKB / 16; ++kk) {
            tc::mma_f16(taddr + buf * LN, tc::sdesc_k_sw128(a0 + kk * 32), tc::sdesc_k_sw128(b0 + kk * 32), LIN_IDESC,
                        !first);
            first = false;
          }
          tc::mma_commit(&S.empty[s]);
        }
        if (*abort_flag) break;
        tc::mma_commit(&S.acc_full[buf]);
      }
      tc::mma_commit(&S.drain);
      mma_committed = true;
      if (!*abort_flag) lin_drain(&S.drain, 0);
    } else if (warp >= 2) {
      const int q = warp & 3;
      const int hc = (warp - 2) >> 2;
      const uint32_t lane_base = (uint32_t)(q * 32) << 16;
      float acc[128];
#pragma unroll
      for (int i = 0; i < 128; ++i) acc[i] = 0.f;
      bool ok = true;
      for (int c = 0; c < nchunks; ++c) {
        const int buf = c & 1;
        int ready = 0;
        if (lane == 0) ready = tc::mbar_wait(&S.acc_full[buf], (uint32_t)(c >> 1) & 1u, abort_flag);
        ready = __shfl_sync(0xffffffffu, ready, 0);
        if (!ready) { ok = false; break; }
        tc::tc_fence_after();
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          float v[32];
          tc::tmem_ld_32x32b_x32(taddr + lane_base + buf * LN + hc * 128 + c4 * 32, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) acc[c4 * 32 + i] += v[i];
        }
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&S.acc_empty[buf]);
      }
      if (ok && !*abort_flag) {
        const int row = bi * LM + q * 32 + lane;
        const int col0 = bj * LN + hc * 128;
        if (row < M && col0 < N) {
          float* dst = C + (int64_t)row * ldc + col0;
          if ((ldc & 3) == 0 && col0 + 128 <= N) {
#pragma unroll
            for (int i = 0; i < 128; i += 4)
              *reinterpret_cast<float4*>(dst + i) = make_float4(acc[i], acc[i + 1], acc[i + 2], acc[i + 3]);
          } else {
#pragma unroll
            for (int i = 0; i < 128; ++i)
              if (col0 + i < N) dst[i] = acc[i];
          }
        }
      }
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    if (warp == 0 && lane == 0) {
      for (int s = 0; s < LSTAGES; ++s)
        if (armed[s] > 0) lin_drain(&S.full[s], (uint32_t)(armed[s] - 1) & 1u);
    }
    if (warp == 1 && lane == 0 && mma_committed) lin_drain(&S.drain, 0);
    if (threadIdx.x == 0) set_error(st, GPTQ_ERR_TIMEOUT, blockIdx.x, STAGE_LINEAR);
    __syncthreads();
  }
  if (warp == 1) {
    __syncwarp();
    tc::tmem_dealloc<512>(taddr);
  }
}

}  // namespace

int launch_linear(const void* A, int M, int64_t lda, const void* B, int N, int64_t ldb, int K, float* C, int64_t ldc,
                  int32_t* st, cudaStream_t s) {
  CUtensorMap ta, tb;
  int rc = make_tmap_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, A, (uint64_t)K, (uint64_t)M, (uint64_t)lda * 2, LKB,
                        LM, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc == GPTQ_OK)
    rc = make_tmap_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, B, (uint64_t)K, (uint64_t)N, (uint64_t)ldb * 2, LKB,
                      LN / 2, CU_TENSOR_MAP_SWIZZLE_128B);
  if (rc != GPTQ_OK) return rc;
  const int tm = (int)cdiv(M, LM), tn = (int)cdiv(N, LN);
  const int kblocks = (int)cdiv(K, LKB);
  // a band's rows of A: about 32 MB (a quarter of L2)
  const int band = (int)std::max<int64_t>(1, std::min<int64_t>(tm, (32ll << 20) / ((int64_t)LM * K * 2)));
  TraceScope ts("linear_bf16", "flop", 2.0 * M * (double)N * K, s);
  GPTQ_CUDA_TRY(cudaFuncSetAttribute(linear_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)LIN_SMEM));
  linear_kernel<<<tm * tn, LTHREADS, LIN_SMEM, s>>>(ta, tb, C, M, N, ldc, tm, tn, band, kblocks, st);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

}  // namespace gptq
