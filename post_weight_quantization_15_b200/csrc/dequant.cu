// The consumer side of the stored format: what = s . (code - z), and the product of
// activations with the dequantized weights.
//
// The pages name inference kernels that read GPTQ's packed weights (Marlin, ExLlama:
// "skillmd.com/skills/artubss/gptq", "Backends de inferencia"; "dev.ayinedjimi-
// consultants.fr ... ia-quantization-gptq-gguf-awq", Marlin at about 80 % of the
// memory bandwidth) and store scale and zero point in FP16 (same page, "Calibration et
// dataset").  Those kernels were written for other GPUs and are not the blueprint.
// Here:
//   dequant_kernel   qweight / scales / zeros / g_idx -> What [out, n] (fp32, fp16 or
//                    bf16), one 16-byte load of four output rows' words per thread;
//   qmatvec_kernel   Y[M, out] = X[M, n] . What^T for a few activation rows
//                    (M <= 16, decode): bound by reading qweight once from HBM, so it
//                    runs on the CUDA cores, the weights dequantized in registers,
//                    never written out; the k range is split across CTAs and the
//                    partial sums reduced in a fixed order (deterministic).
// Both take any g_idx (act-order included).  Codes of 2, 4 or 8 bits (a word holds
// 32 / bits whole codes).
#include <algorithm>
#include <climits>
#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace gptq {

namespace {

// ---------------------------------------------------------------------------
// What[o][k] = s[g_idx[k]][o] . (code(o, k) - z[g_idx[k]][o]).  The product of an
// fp16 scale (11 significant bits) and an integer of at most 9 bits is exact in fp32,
// so the fp32 output is exact and the fp16 / bf16 outputs are rounded once (RNE).
// Thread: four consecutive outputs o (one uint4 of qweight row w) and the 32/bits
// input columns of word w; the block's 32 x 8 threads cover 128 outputs x 8 words.
// ---------------------------------------------------------------------------
template <typename TO>
__device__ __forceinline__ TO from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __half from_f32<__half>(float v) { return __float2half_rn(v); }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

template <typename TO, int BITS>
__global__ void __launch_bounds__(256) dequant_kernel(const int32_t* qweight, const uint16_t* scales,
                                                      const uint16_t* zeros, const int32_t* g_idx, int n, int out,
                                                      int groups, TO* What, int32_t* st) {
  if (has_error(st)) return;
  constexpr int PER = 32 / BITS;                       // codes per word
  const int words = n / PER;
  const int o = 4 * (blockIdx.x * 32 + threadIdx.x);
  const int w = blockIdx.y * 8 + threadIdx.y;
  if (o >= out || w >= words) return;
  uint32_t q[4];
  if ((out & 3) == 0) {
    const uint4 v = *reinterpret_cast<const uint4*>(qweight + (int64_t)w * out + o);
    q[0] = v.x; q[1] = v.y; q[2] = v.z; q[3] = v.w;
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j) q[j] = o + j < out ? (uint32_t)qweight[(int64_t)w * out + o + j] : 0u;
  }
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int k = w * PER + i;
    int g = g_idx[k];
    if ((unsigned)g >= (unsigned)groups) {          // a group index the scales do not have
      set_error(st, GPTQ_ERR_INVALID_ARG, k, STAGE_DEQUANT);
      g = 0;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (o + j >= out) break;
      const float s = __half2float(__ushort_as_half(scales[(int64_t)g * out + o + j]));
      const float z = __half2float(__ushort_as_half(zeros[(int64_t)g * out + o + j]));
      const float c = (float)((q[j] >> (i * BITS)) & ((1u << BITS) - 1u));
      What[(int64_t)(o + j) * n + k] = from_f32<TO>(s * (c - z));
    }
  }
}

// ---------------------------------------------------------------------------
// Y = X . What^T for m <= QMV_MAXM activation rows (the kernel is instantiated for
// M = 1, 2, 4, 8, 16 rows; rows m .. M-1 are staged as zeros and never written).
// Block: 8 warps over the same 128 outputs (lane: four outputs, one uint4 of a
// qweight row); the block's k range [k0, k0 + kc) is split between the warps word by
// word, four words in flight per thread.  Staged in shared memory first: X's columns
// of the range as fp32 (column k of the packed layer multiplies X column xperm[k],
// or k), the range's group indices, and - when the range's groups span at most
// QMV_MAXG consecutive groups (groups contiguous in k: no act-order, or a layer
// reordered by gptq_reorder_groups) - their scales and zero points for the block's
// 128 outputs; otherwise the inner loop reads those from global memory.  Per word and
// output the code of each of its 32/bits columns is dequantized once and multiplies
// all rows.  The 8 warps' sums are added in warp order into part[split][m][out]
// (fp32); qmatvec_reduce_kernel adds the splits in order.
// ---------------------------------------------------------------------------
constexpr int QMV_MAXM = 16;
// input columns per block: as many as the staged activations allow (the staging's
// latency is paid once per block, so longer ranges amortise it)
__host__ __device__ constexpr int qmv_kc(int M) { return M <= 2 ? 2048 : M <= 4 ? 1024 : M <= 8 ? 512 : 256; }
constexpr int QMV_UNROLL = 4;         // words in flight per thread
// staged groups: the range's groups when groups of 64 or more columns are contiguous
__host__ __device__ constexpr int qmv_maxg(int M) { return qmv_kc(M) / 64 + 1; }
__host__ __device__ constexpr size_t qmv_smem(int M) {
  return (size_t)M * qmv_kc(M) * 4 + (size_t)qmv_kc(M) * 4 + 8 * 128 * 4 + (size_t)qmv_maxg(M) * 64 * 16 +
         (size_t)M * (qmv_kc(M) + 8) * 2;
}

// ---------------------------------------------------------------------------
// The tensor-core form of the product (4-bit codes, fp16 or bf16 activations, a block
// whose groups are staged and constant over each 32-column tile): per 32 columns and 8
// outputs, two mma.sync m16n8k16 (fp32 accumulate) of the activations (16 rows, the
// rows past M zero) with the codes minus the zero points, exact in fp16 / bf16:
//   lane (g, t) of a warp loads the packed word of columns [8t, 8t + 8) of the tile for
//   output g of the eight, and its nibble pairs (p, p + 4), p = 0..3, become the pairs
//   (B + c_p, B + c_{p+4}) by one mask-or with the bits of B (1024 in fp16, 128 in
//   bf16: c < 16 sits in the mantissa exactly); one packed subtraction of (B + z) leaves
//   the exact integers c - z.  Pair p feeds the k slots of mma p / 2, b-register p % 2,
//   so the tile's k slot s holds column perm(s) = 8t + 2h + j + 4i for s = 16h + 8j +
//   2t + i; the activations are staged in that order, so each product pairs the right
//   column.  The accumulator is scaled by s (per output) and added into fp32 registers
//   at every group change and every 128 columns (at most 8 mma per accumulation).
// ---------------------------------------------------------------------------
__device__ __forceinline__ int qmv_tc_slot(int c) {     // the k slot of tile column c
  const int t = c >> 3, i = (c >> 2) & 1, h = (c >> 1) & 1, j = c & 1;
  return 16 * h + 8 * j + 2 * t + i;
}

template <typename TX>
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1);
template <>
__device__ __forceinline__ void mma_16816<__half>(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
template <>
__device__ __forceinline__ void mma_16816<__nv_bfloat16>(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// (B + c_lo, B + c_hi) - (B + z, B + z) as a packed pair, exactly
template <typename TX>
__device__ __forceinline__ uint32_t qmv_code_pair(uint32_t bits, uint32_t bz);
template <>
__device__ __forceinline__ uint32_t qmv_code_pair<__half>(uint32_t bits, uint32_t bz) {
  const __half2 r = __hsub2(*reinterpret_cast<const __half2*>(&bits), *reinterpret_cast<const __half2*>(&bz));
  return *reinterpret_cast<const uint32_t*>(&r);
}
template <>
__device__ __forceinline__ uint32_t qmv_code_pair<__nv_bfloat16>(uint32_t bits, uint32_t bz) {
  const __nv_bfloat162 r =
      __hsub2(*reinterpret_cast<const __nv_bfloat162*>(&bits), *reinterpret_cast<const __nv_bfloat162*>(&bz));
  return *reinterpret_cast<const uint32_t*>(&r);
}
template <typename TX> struct QmvMagic;
template <> struct QmvMagic<__half> { static constexpr uint32_t bits = 0x64006400u; static constexpr float base = 1024.f; };
template <> struct QmvMagic<__nv_bfloat16> { static constexpr uint32_t bits = 0x43004300u; static constexpr float base = 128.f; };
template <typename TX> __device__ __forceinline__ uint16_t qmv_to_bits(float v);
template <> __device__ __forceinline__ uint16_t qmv_to_bits<__half>(float v) { return __half_as_ushort(__float2half_rn(v)); }
template <> __device__ __forceinline__ uint16_t qmv_to_bits<__nv_bfloat16>(float v) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}

template <typename TX, int BITS, int M>
__global__ void __launch_bounds__(256) qmatvec_kernel(const int32_t* qweight, const uint16_t* scales,
                                                      const uint16_t* zeros, const int32_t* g_idx, int n, int out,
                                                      int groups, const TX* X, const int32_t* xperm, int m_real,
                                                      int ldx, float* part, int32_t* st) {
  if (has_error(st)) return;
  constexpr int PER = 32 / BITS;
  constexpr int kc = qmv_kc(M);
  constexpr int QMV_MAXG = qmv_maxg(M);
  extern __shared__ __align__(16) uint8_t qsm[];
  float* xs = reinterpret_cast<float*>(qsm);                          // [M][kc]
  int* gsm = reinterpret_cast<int*>(xs + M * kc);                     // [kc]
  float* red = reinterpret_cast<float*>(gsm + kc);                    // [8][128]
  // scales, then zero points, of staged group g_lo + gi for the four outputs of lane l:
  // szs[gi][l] = (s0, s1, s2, s3), szs[gi][32 + l] = (z0, z1, z2, z3)
  float4* szs = reinterpret_cast<float4*>(red + 8 * 128);             // [QMV_MAXG][64]
  __shared__ int grange[3];
  // the activations in the tensor-core order (fp16 / bf16 bits), [M][XHS]: rows 16 bytes
  // longer than kc columns, so that the eight rows of a fragment load sit in distinct banks
  constexpr int XHS = kc + 8;
  uint16_t* xh = reinterpret_cast<uint16_t*>(reinterpret_cast<uint8_t*>(szs) + (size_t)QMV_MAXG * 64 * 16);
  // the tensor-core form for one or two rows (measured: from four rows on, the fma form's
  // shorter prologue and reduction win)
  constexpr bool kTC = BITS == 4 && M <= 2 && !std::is_same<TX, float>::value;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int o0 = blockIdx.x * 128;
  const int k0 = blockIdx.y * kc;
  const int k1 = min(n, k0 + kc);
  {
    // the block's packed words (its kc / PER rows, 128 outputs) requested into L2 before the
    // staging below: their DRAM latency overlaps the staging's dependent loads
    const int nl = (min(128, out - o0) + 31) / 32;       // 128-byte lines per row
    const int rows = k1 / PER - k0 / PER;
    for (int i = threadIdx.x; i < rows * nl; i += blockDim.x)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(qweight + (int64_t)(k0 / PER + i / nl) * out + o0 + 32 * (i % nl)));
  }
  if (threadIdx.x == 0) { grange[0] = INT_MAX; grange[1] = -1; grange[2] = 0; }
  // Every global load of the staging is issued before any is used: the range's group
  // indices and its activations (column k of the range multiplies X column xperm[k], or
  // k); thread i holds columns i + 256 r.
  constexpr int KPT = kc / 256;
  int gv[KPT], xk[KPT];
#pragma unroll
  for (int r = 0; r < KPT; ++r) {
    const int k = k0 + threadIdx.x + 256 * r;
    gv[r] = k < k1 ? __ldg(g_idx + k) : -1;
    xk[r] = k < k1 ? (xperm ? __ldg(xperm + k) : k) : -1;
  }
  float xv[M][KPT];
#pragma unroll
  for (int m = 0; m < M; ++m)
#pragma unroll
    for (int r = 0; r < KPT; ++r)
      xv[m][r] = (xk[r] >= 0 && m < m_real) ? load_as_float<TX>(X + (int64_t)m * ldx + xk[r]) : 0.f;
  __syncthreads();
  // the range's groups: their span, and whether every packed word (PER columns; k0 is a
  // multiple of PER) and every 32-column tile holds columns of one group
  int gmin = INT_MAX, gmax = -1, split_word = 0, split_tile = 0;
#pragma unroll
  for (int r = 0; r < KPT; ++r) {
    const int i = threadIdx.x + 256 * r;
    const bool in = k0 + i < k1;
    int g = gv[r];
    if (g >= groups || (g < 0 && in)) {               // a group index the scales do not have
      set_error(st, GPTQ_ERR_INVALID_ARG, k0 + i, STAGE_DEQUANT);
      g = 0;
    }
    g = g < 0 ? 0 : g;
    if (in) { gmin = min(gmin, g); gmax = max(gmax, g); }
    gsm[i] = g;
    const int gw = __shfl_sync(0xffffffffu, g, lane - lane % PER), gt = __shfl_sync(0xffffffffu, g, 0);
    if (in && g != gw) split_word = 1;
    if (in && g != gt) split_tile = 1;
  }
  for (int o = 16; o > 0; o >>= 1) {
    gmin = min(gmin, __shfl_xor_sync(0xffffffffu, gmin, o));
    gmax = max(gmax, __shfl_xor_sync(0xffffffffu, gmax, o));
  }
  split_word = __any_sync(0xffffffffu, split_word);
  split_tile = __any_sync(0xffffffffu, split_tile);
  if (lane == 0) {
    atomicMin(&grange[0], gmin);
    atomicMax(&grange[1], gmax);
    if (split_word | split_tile) atomicOr(&grange[2], split_word | (split_tile << 1));
  }
  __syncthreads();
  const int g_lo = grange[0];
  const bool staged = grange[1] - g_lo < QMV_MAXG;
  const bool uniform = (grange[2] & 1) == 0;
  // the tensor-core form (block-uniform): staged groups constant over each 32-column tile
  bool tc = kTC && staged && (grange[2] & 2) == 0 && ((k1 - k0) & 31) == 0;
  // the staged groups' scales and zero points, loaded before the activations are stored
  constexpr int SZPT = (QMV_MAXG * 128 + 255) / 256;
  const int nsz = staged ? (grange[1] - g_lo + 1) * 128 : 0;
  uint16_t sv[SZPT], zv[SZPT];
#pragma unroll
  for (int r = 0; r < SZPT; ++r) {
    const int i = threadIdx.x + 256 * r, oo = o0 + i % 128;
    const bool in = i < nsz && oo < out;
    sv[r] = in ? __ldg(scales + (int64_t)(g_lo + i / 128) * out + oo) : (uint16_t)0;
    zv[r] = in ? __ldg(zeros + (int64_t)(g_lo + i / 128) * out + oo) : (uint16_t)0;
  }
  auto stage_xs = [&]() {
#pragma unroll
    for (int m = 0; m < M; ++m)
#pragma unroll
      for (int r = 0; r < KPT; ++r) xs[m * kc + threadIdx.x + 256 * r] = xv[m][r];
  };
  if constexpr (kTC) {
    if (tc) {
#pragma unroll
      for (int m = 0; m < M; ++m)
#pragma unroll
        for (int r = 0; r < KPT; ++r) {
          const int c = threadIdx.x + 256 * r;
          xh[m * XHS + (c & ~31) + qmv_tc_slot(c & 31)] = qmv_to_bits<TX>(xv[m][r]);
        }
    } else {
      stage_xs();
    }
  } else {
    stage_xs();
  }
  if (staged) {
    float* szf = reinterpret_cast<float*>(szs);
    int odd_zero = 0;
#pragma unroll
    for (int r = 0; r < SZPT; ++r) {
      const int i = threadIdx.x + 256 * r, gi = i / 128, oi = i % 128;
      if (i < nsz) {
        const float zf = __half2float(__ushort_as_half(zv[r]));
        szf[(gi * 64 + oi / 4) * 4 + oi % 4] = __half2float(__ushort_as_half(sv[r]));
        szf[(gi * 64 + 32 + oi / 4) * 4 + oi % 4] = zf;
        // the tensor-core form subtracts z in fp16 / bf16: exact for integers in [0, 127]
        if (!(zf >= 0.f && zf <= 127.f && zf == rintf(zf))) odd_zero = 1;
      }
    }
    if (kTC && __any_sync(0xffffffffu, odd_zero) && lane == 0) atomicOr(&grange[2], 4);
  }
  __syncthreads();
  if constexpr (kTC) {
    // the tensor-core form also wants integer zero points; a block that finds others (a
    // layer edited by hand) stores the fp32 activations after all and takes the fma form
    if (tc && (grange[2] & 4) != 0) {
      tc = false;
      stage_xs();
      __syncthreads();
    }
    if (tc) {
      const float* szf = reinterpret_cast<const float*>(szs);
      const int g = lane >> 2, t = lane & 3;
      const int qo = warp & 3, kh = warp >> 2;                 // output quarter, k half
      const int ntile = (k1 - k0) >> 5;
      const int tb = kh * ((ntile + 1) >> 1), te = min(ntile, tb + ((ntile + 1) >> 1));
      float yacc[4][4], dacc[4][4];
      uint32_t bz[4];
#pragma unroll
      for (int og = 0; og < 4; ++og)
#pragma unroll
        for (int e = 0; e < 4; ++e) { yacc[og][e] = 0.f; dacc[og][e] = 0.f; }
      int gcur = -1, nacc = 0;
      auto flush = [&]() {
#pragma unroll
        for (int og = 0; og < 4; ++og) {
          const int oi = 32 * qo + 8 * og + 2 * t;             // this lane's two accumulator columns
          const float s0 = szf[(gcur * 64 + oi / 4) * 4 + oi % 4];
          const float s1 = szf[(gcur * 64 + (oi + 1) / 4) * 4 + (oi + 1) % 4];
          yacc[og][0] = fmaf(s0, dacc[og][0], yacc[og][0]);
          yacc[og][1] = fmaf(s1, dacc[og][1], yacc[og][1]);
          yacc[og][2] = fmaf(s0, dacc[og][2], yacc[og][2]);
          yacc[og][3] = fmaf(s1, dacc[og][3], yacc[og][3]);
#pragma unroll
          for (int e = 0; e < 4; ++e) dacc[og][e] = 0.f;
        }
        nacc = 0;
      };
      for (int tq = tb; tq < te; tq += 4) {
      uint32_t q4[4][4];                                       // four tiles' words in flight
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t wrow = (int64_t)((k0 + (tq + u) * 32) / 8 + t) * out;
#pragma unroll
        for (int og = 0; og < 4; ++og) {
          const int oo = o0 + 32 * qo + 8 * og + g;
          q4[u][og] = (tq + u < te && oo < out) ? (uint32_t)__ldg(qweight + wrow + oo) : 0u;
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int tt = tq + u;
        if (tt >= te) break;
        const int c0 = tt * 32;
        const int gi = gsm[c0] - g_lo;
        if (gi != gcur || nacc == 4) {                         // a group change, or 128 columns
          if (gcur >= 0) flush();
          if (gi != gcur) {
            gcur = gi;
#pragma unroll
            for (int og = 0; og < 4; ++og) {                   // B + z for this lane's output
              const int oi = 32 * qo + 8 * og + g;
              const float zb = QmvMagic<TX>::base + szf[(gcur * 64 + 32 + oi / 4) * 4 + oi % 4];
              const uint32_t h = qmv_to_bits<TX>(zb);
              bz[og] = h | (h << 16);
            }
          }
        }
        // the activations: rows g and g + 8 of the two k halves of each mma
        uint32_t a[2][4];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int sb = c0 + 16 * h + 2 * t;
          a[h][0] = g < M ? *reinterpret_cast<const uint32_t*>(xh + g * XHS + sb) : 0u;
          a[h][2] = g < M ? *reinterpret_cast<const uint32_t*>(xh + g * XHS + sb + 8) : 0u;
          a[h][1] = g + 8 < M ? *reinterpret_cast<const uint32_t*>(xh + (g + 8) * XHS + sb) : 0u;
          a[h][3] = g + 8 < M ? *reinterpret_cast<const uint32_t*>(xh + (g + 8) * XHS + sb + 8) : 0u;
        }
        const uint32_t* q = q4[u];
#pragma unroll
        for (int og = 0; og < 4; ++og) {
          uint32_t b[4];
#pragma unroll
          for (int p = 0; p < 4; ++p)
            b[p] = qmv_code_pair<TX>(((q[og] >> (4 * p)) & 0x000F000Fu) | QmvMagic<TX>::bits, bz[og]);
          mma_16816<TX>(dacc[og], a[0], b[0], b[1]);
          mma_16816<TX>(dacc[og], a[1], b[2], b[3]);
        }
        ++nacc;
      }
      }
      if (gcur >= 0) flush();
      // the 8 warps' sums in warp order (each output has two warps' terms, the rest zero)
#pragma unroll 1
      for (int m = 0; m < M; ++m) {
        if (m >= m_real) break;
        __syncthreads();
        for (int i = lane; i < 128; i += 32) red[warp * 128 + i] = 0.f;
        __syncwarp();
        if (g == m || g + 8 == m) {
          const int e0 = g == m ? 0 : 2;
#pragma unroll
          for (int og = 0; og < 4; ++og) {
            red[warp * 128 + 32 * qo + 8 * og + 2 * t] = yacc[og][e0];
            red[warp * 128 + 32 * qo + 8 * og + 2 * t + 1] = yacc[og][e0 + 1];
          }
        }
        __syncthreads();
        if (threadIdx.x < 128) {
          const int oo = o0 + threadIdx.x;
          float tsum = 0.f;
#pragma unroll
          for (int wp = 0; wp < 8; ++wp) tsum += red[wp * 128 + threadIdx.x];
          if (oo < out) part[((int64_t)blockIdx.y * m_real + m) * out + oo] = tsum;
        }
      }
      return;
    }
  }
  const int o = o0 + 4 * lane;
  float acc[M][4];
#pragma unroll
  for (int m = 0; m < M; ++m)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[m][j] = 0.f;
  const bool full = o + 3 < out && (out & 3) == 0;
  const int w0 = k0 / PER, w1 = k1 / PER;
  int g_prev = -1;
  float s[4] = {0.f, 0.f, 0.f, 0.f}, z[4] = {0.f, 0.f, 0.f, 0.f};
  constexpr int I1U = M * PER >= 256 ? 4 : PER;     // the per-column loop's unrolling
  for (int wb = w0 + warp; wb < w1; wb += 8 * QMV_UNROLL) {
    uint32_t q[QMV_UNROLL][4];
#pragma unroll
    for (int u = 0; u < QMV_UNROLL; ++u) {       // the loads first, all in flight together
      const int w = wb + 8 * u;
#pragma unroll
      for (int j = 0; j < 4; ++j) q[u][j] = 0u;
      if (w < w1) {
        if (full) {
          const uint4 v = __ldg(reinterpret_cast<const uint4*>(qweight + (int64_t)w * out + o));
          q[u][0] = v.x; q[u][1] = v.y; q[u][2] = v.z; q[u][3] = v.w;
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j) if (o + j < out) q[u][j] = (uint32_t)__ldg(qweight + (int64_t)w * out + o + j);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < QMV_UNROLL; ++u) {
      const int w = wb + 8 * u;
      if (w >= w1) break;
      if (staged && uniform) {
        // the word's columns share one group: its scales and zero points once, the
        // activations of its PER columns as 16-byte loads
        const int kl0 = w * PER - k0;
        const int gi = gsm[kl0] - g_lo;
        const float4 sv = szs[gi * 64 + lane], zv = szs[gi * 64 + 32 + lane];
        // s (c - z) in one exact fma: the code c placed in the top mantissa bits of 1.0 gives
        // f = 1 + c / 2^BITS without a conversion instruction (a shift and a mask-or), and
        // s (c - z) = (2^BITS s) f - s (2^BITS + z): every product has at most 20 significant
        // bits (an fp16 scale, integers below 2^9), so the fma's one rounding is exact
        const float s4[4] = {sv.x * (float)(1 << BITS), sv.y * (float)(1 << BITS), sv.z * (float)(1 << BITS),
                             sv.w * (float)(1 << BITS)};
        const float n4[4] = {-sv.x * ((float)(1 << BITS) + zv.x), -sv.y * ((float)(1 << BITS) + zv.y),
                             -sv.z * ((float)(1 << BITS) + zv.z), -sv.w * ((float)(1 << BITS) + zv.w)};
        constexpr int POS = 23 - BITS;                 // where the code goes in the mantissa
        // fully unrolled unless the body is large (16 rows of 2-bit codes): then four
        // columns at a time, the shift a register operand
        constexpr int I0U = M * PER >= 256 ? 1 : PER / 4;
#pragma unroll I0U
        for (int i0 = 0; i0 < PER; i0 += 4) {
          float wv[4][4];
#pragma unroll
          for (int ii = 0; ii < 4; ++ii) {
            constexpr uint32_t MASK = ((1u << BITS) - 1u) << POS;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int sh = POS - (i0 + ii) * BITS;   // a compile-time shift after unrolling
              const uint32_t bitsf = (sh >= 0 ? (q[u][j] << sh) : (q[u][j] >> -sh)) & MASK;
              wv[ii][j] = fmaf(s4[j], __uint_as_float(bitsf | 0x3F800000u), n4[j]);
            }
          }
#pragma unroll
          for (int m = 0; m < M; ++m) {
            const float4 x4 = *reinterpret_cast<const float4*>(xs + m * kc + kl0 + i0);
            const float xv[4] = {x4.x, x4.y, x4.z, x4.w};
#pragma unroll
            for (int ii = 0; ii < 4; ++ii)
#pragma unroll
              for (int j = 0; j < 4; ++j) acc[m][j] = fmaf(xv[ii], wv[ii][j], acc[m][j]);
          }
        }
        continue;
      }
#pragma unroll I1U
      for (int i = 0; i < PER; ++i) {
        const int kl = w * PER + i - k0;
        const int g = gsm[kl];
        if (staged) {
          const float4 sv = szs[(g - g_lo) * 64 + lane], zv = szs[(g - g_lo) * 64 + 32 + lane];
          s[0] = sv.x; s[1] = sv.y; s[2] = sv.z; s[3] = sv.w;
          z[0] = zv.x; z[1] = zv.y; z[2] = zv.z; z[3] = zv.w;
        } else if (g != g_prev) {      // a new group: its scales and zero points for the four outputs
          g_prev = g;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const bool in = o + j < out;
            s[j] = in ? __half2float(__ushort_as_half(scales[(int64_t)g * out + o + j])) : 0.f;
            z[j] = in ? __half2float(__ushort_as_half(zeros[(int64_t)g * out + o + j])) : 0.f;
          }
        }
        float wv[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) wv[j] = s[j] * ((float)((q[u][j] >> (i * BITS)) & ((1u << BITS) - 1u)) - z[j]);
#pragma unroll
        for (int m = 0; m < M; ++m) {
          const float xv = xs[m * kc + kl];
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[m][j] = fmaf(xv, wv[j], acc[m][j]);
        }
      }
    }
  }
  // the 8 warps' partial sums, added in warp order, one row at a time
#pragma unroll
  for (int m = 0; m < M; ++m) {
    if (m >= m_real) break;
    __syncthreads();
#pragma unroll
    for (int j = 0; j < 4; ++j) red[warp * 128 + 4 * lane + j] = acc[m][j];
    __syncthreads();
    if (threadIdx.x < 128) {
      const int oo = o0 + threadIdx.x;
      float t = 0.f;
#pragma unroll
      for (int wp = 0; wp < 8; ++wp) t += red[wp * 128 + threadIdx.x];
      if (oo < out) part[((int64_t)blockIdx.y * m_real + m) * out + oo] = t;
    }
  }
}

__global__ void qmatvec_reduce_kernel(const float* part, int splits, int M, int out, float* Y, int ldy,
                                      const int32_t* st) {
  if (has_error(st)) return;
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (int64_t)M * out) return;
  const int m = (int)(i / out), o = (int)(i % out);
  float t = 0.f;
  for (int sp = 0; sp < splits; ++sp) t += part[((int64_t)sp * M + m) * out + o];
  Y[(int64_t)m * ldy + o] = t;
}

template <typename TO>
int dequant_t(const int32_t* qweight, const uint16_t* scales, const uint16_t* zeros, const int32_t* g_idx, int bits,
              int n, int out, int groups, TO* What, int32_t* st, cudaStream_t s) {
  const int words = n * bits / 32;
  dim3 blk(32, 8), grd((unsigned)cdiv(out, 128), (unsigned)cdiv(words, 8));
  if (bits == 2) dequant_kernel<TO, 2><<<grd, blk, 0, s>>>(qweight, scales, zeros, g_idx, n, out, groups, What, st);
  else if (bits == 4) dequant_kernel<TO, 4><<<grd, blk, 0, s>>>(qweight, scales, zeros, g_idx, n, out, groups, What, st);
  else dequant_kernel<TO, 8><<<grd, blk, 0, s>>>(qweight, scales, zeros, g_idx, n, out, groups, What, st);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

template <typename TX, int BITS, int M>
int qmv_launch(const int32_t* qweight, const uint16_t* scales, const uint16_t* zeros, const int32_t* g_idx, int n,
               int out, int groups, const void* X, const int32_t* xperm, int m_real, int ldx, float* part,
               int splits, int32_t* st, cudaStream_t s) {
  (void)splits;
  dim3 grd((unsigned)cdiv(out, 128), (unsigned)cdiv(n, qmv_kc(M)));
  const size_t smem = qmv_smem(M);
  GPTQ_CUDA_TRY(cudaFuncSetAttribute(qmatvec_kernel<TX, BITS, M>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)smem));
  qmatvec_kernel<TX, BITS, M><<<grd, 256, smem, s>>>(qweight, scales, zeros, g_idx, n, out, groups,
                                                   static_cast<const TX*>(X), xperm, m_real, ldx, part, st);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

template <typename TX, int BITS>
int qmv_m(int M, const int32_t* qweight, const uint16_t* scales, const uint16_t* zeros, const int32_t* g_idx, int n,
          int out, int groups, const void* X, const int32_t* xperm, int ldx, float* part, int splits, int32_t* st,
          cudaStream_t s) {
  if (M <= 1) return qmv_launch<TX, BITS, 1>(qweight, scales, zeros, g_idx, n, out, groups, X, xperm, M, ldx, part, splits, st, s);
  if (M <= 2) return qmv_launch<TX, BITS, 2>(qweight, scales, zeros, g_idx, n, out, groups, X, xperm, M, ldx, part, splits, st, s);
  if (M <= 4) return qmv_launch<TX, BITS, 4>(qweight, scales, zeros, g_idx, n, out, groups, X, xperm, M, ldx, part, splits, st, s);
  if (M <= 8) return qmv_launch<TX, BITS, 8>(qweight, scales, zeros, g_idx, n, out, groups, X, xperm, M, ldx, part, splits, st, s);
  return qmv_launch<TX, BITS, 16>(qweight, scales, zeros, g_idx, n, out, groups, X, xperm, M, ldx, part, splits, st, s);
}

// ---------------------------------------------------------------------------
// Reordering a layer so that its groups are contiguous: xperm = the columns sorted by
// group, ties in column order (stable).  One thread per group scans g_idx (staged in
// shared memory in slabs, every thread reading the same word: a broadcast) and writes
// the positions of its group's columns in order, after the counts of the groups
// before it.
// ---------------------------------------------------------------------------
constexpr int RG_SLAB = 8192;

__global__ void __launch_bounds__(1024) group_count_kernel(const int32_t* g_idx, int n, int groups, int* counts,
                                                           int32_t* st) {
  if (has_error(st)) return;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const int g = g_idx[i];
    if ((unsigned)g >= (unsigned)groups) { set_error(st, GPTQ_ERR_INVALID_ARG, i, STAGE_DEQUANT); continue; }
    atomicAdd(counts + g, 1);
  }
}

__global__ void __launch_bounds__(1024) group_scatter_kernel(const int32_t* g_idx, int n, int groups,
                                                             const int* counts, int32_t* xperm, int32_t* g_sorted,
                                                             const int32_t* st) {
  if (has_error(st)) return;
  __shared__ int slab[RG_SLAB];
  const int g = blockIdx.x * blockDim.x + threadIdx.x;
  int pos = 0;                                       // the first position of group g
  if (g < groups)
    for (int h = 0; h < g; ++h) pos += counts[h];
  for (int base = 0; base < n; base += RG_SLAB) {
    const int len = min(RG_SLAB, n - base);
    __syncthreads();
    for (int i = threadIdx.x; i < len; i += blockDim.x) slab[i] = g_idx[base + i];
    __syncthreads();
    if (g < groups) {
      for (int i = 0; i < len; ++i) {
        if (slab[i] == g) {
          xperm[pos] = base + i;
          g_sorted[pos] = g;
          ++pos;
        }
      }
    }
  }
}

// qweight_g[w][o]: the codes of columns xperm[w.PER .. w.PER + PER - 1] for output o.
template <int BITS>
__global__ void repack_kernel(const int32_t* qweight, const int32_t* xperm, int n, int out, int32_t* qweight_g,
                              const int32_t* st) {
  if (has_error(st)) return;
  constexpr int PER = 32 / BITS;
  const int o = blockIdx.x * blockDim.x + threadIdx.x;
  const int w = blockIdx.y;
  if (o >= out || w >= n / PER) return;
  uint32_t word = 0u;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int k = xperm[w * PER + i];
    const uint32_t src = (uint32_t)qweight[(int64_t)(k / PER) * out + o];
    word |= ((src >> ((k % PER) * BITS)) & ((1u << BITS) - 1u)) << (i * BITS);
  }
  qweight_g[(int64_t)w * out + o] = (int32_t)word;
}

}  // namespace

size_t reorder_ws_bytes(int groups) { return align_up((size_t)groups * 4, 256); }

int launch_reorder_groups(const int32_t* qweight, const int32_t* g_idx, int bits, int n, int out, int groups,
                          int32_t* qweight_g, int32_t* g_sorted, int32_t* xperm, void* ws, int32_t* st,
                          cudaStream_t s) {
  int* counts = static_cast<int*>(ws);
  GPTQ_CUDA_TRY(cudaMemsetAsync(counts, 0, (size_t)groups * 4, s));
  group_count_kernel<<<(unsigned)std::min<int64_t>(cdiv(n, 1024), 148), 1024, 0, s>>>(g_idx, n, groups, counts, st);
  GPTQ_LAUNCH_CHECK();
  group_scatter_kernel<<<(unsigned)cdiv(groups, 1024), 1024, 0, s>>>(g_idx, n, groups, counts, xperm, g_sorted, st);
  GPTQ_LAUNCH_CHECK();
  dim3 grd((unsigned)cdiv(out, 256), (unsigned)(n * bits / 32));
  if (bits == 2) repack_kernel<2><<<grd, 256, 0, s>>>(qweight, xperm, n, out, qweight_g, st);
  else if (bits == 4) repack_kernel<4><<<grd, 256, 0, s>>>(qweight, xperm, n, out, qweight_g, st);
  else repack_kernel<8><<<grd, 256, 0, s>>>(qweight, xperm, n, out, qweight_g, st);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

size_t qmatvec_ws_bytes(int M, int n, int out) {
  const int splits = (int)cdiv(n, qmv_kc(M <= 2 ? 2 : M <= 4 ? 4 : M <= 8 ? 8 : 16));
  return align_up((size_t)splits * M * out * 4, 256);
}

int launch_dequant(const int32_t* qweight, const uint16_t* scales, const uint16_t* zeros, const int32_t* g_idx,
                   int bits, int n, int out, int groups, int dtype, void* What, int32_t* st, cudaStream_t s) {
  TraceScope ts("dequant", "byte",
                (double)out * n * bits / 8.0 + 4.0 * n + (double)out * n * (dtype == GPTQ_F32 ? 4.0 : 2.0), s);
  if (dtype == GPTQ_F32) return dequant_t<float>(qweight, scales, zeros, g_idx, bits, n, out, groups, static_cast<float*>(What), st, s);
  if (dtype == GPTQ_F16) return dequant_t<__half>(qweight, scales, zeros, g_idx, bits, n, out, groups, static_cast<__half*>(What), st, s);
  return dequant_t<__nv_bfloat16>(qweight, scales, zeros, g_idx, bits, n, out, groups, static_cast<__nv_bfloat16*>(What), st, s);
}

int launch_qmatvec(const int32_t* qweight, const uint16_t* scales, const uint16_t* zeros, const int32_t* g_idx,
                   int bits, int n, int out, int groups, const void* X, const int32_t* xperm, int x_dtype, int M,
                   int ldx, float* Y, int ldy, void* ws, int32_t* st, cudaStream_t s) {
  const int splits = (int)cdiv(n, qmv_kc(M <= 2 ? 2 : M <= 4 ? 4 : M <= 8 ? 8 : 16));
  float* part = static_cast<float*>(ws);
  // bytes read once: packed weights, scales and zeros, g_idx, X; Y written
  TraceScope ts("qmatvec", "byte",
                (double)out * n * bits / 8.0 + 4.0 * (double)groups * out + 4.0 * n + 2.0 * M * n + 4.0 * M * out, s);
  int rc = GPTQ_ERR_UNSUPPORTED;
  auto go = [&](auto tx_tag) {
    using TX = decltype(tx_tag);
    if (bits == 2) return qmv_m<TX, 2>(M, qweight, scales, zeros, g_idx, n, out, groups, X, xperm, ldx, part, splits, st, s);
    if (bits == 4) return qmv_m<TX, 4>(M, qweight, scales, zeros, g_idx, n, out, groups, X, xperm, ldx, part, splits, st, s);
    return qmv_m<TX, 8>(M, qweight, scales, zeros, g_idx, n, out, groups, X, xperm, ldx, part, splits, st, s);
  };
  if (x_dtype == GPTQ_F16) rc = go(__half{});
  else if (x_dtype == GPTQ_BF16) rc = go(__nv_bfloat16{});
  else rc = go(float{});
  if (rc != GPTQ_OK) return rc;
  qmatvec_reduce_kernel<<<(unsigned)cdiv((int64_t)M * out, 256), 256, 0, s>>>(part, splits, M, out, Y, ldy, st);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

}  // namespace gptq
