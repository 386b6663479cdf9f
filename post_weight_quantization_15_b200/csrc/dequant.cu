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
// word, four words in flight per thread; X's columns of the range sit in shared
// memory as fp32, g_idx beside them.  Per word and output the code of each of its
// 32/bits columns is dequantized once and multiplies all rows.  The 8 warps' sums
// are added in warp order into part[split][m][out] (fp32); qmatvec_reduce_kernel
// adds the splits in order.
// ---------------------------------------------------------------------------
constexpr int QMV_MAXM = 16;
constexpr int QMV_KC = 512;           // input columns per block
constexpr int QMV_UNROLL = 4;         // words in flight per thread

template <typename TX, int BITS, int M>
__global__ void __launch_bounds__(256) qmatvec_kernel(const int32_t* qweight, const uint16_t* scales,
                                                      const uint16_t* zeros, const int32_t* g_idx, int n, int out,
                                                      int groups, const TX* X, int m_real, int ldx, float* part,
                                                      int32_t* st) {
  if (has_error(st)) return;
  constexpr int PER = 32 / BITS;
  constexpr int kc = QMV_KC;
  __shared__ float xs[M * kc];
  __shared__ int gsm[kc];
  __shared__ float red[8 * 128];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int o0 = blockIdx.x * 128;
  const int k0 = blockIdx.y * kc;
  const int k1 = min(n, k0 + kc);
  for (int i = threadIdx.x; i < M * kc; i += blockDim.x) {
    const int m = i / kc, k = k0 + i % kc;
    xs[i] = (k < k1 && m < m_real) ? load_as_float<TX>(X + (int64_t)m * ldx + k) : 0.f;
  }
  for (int i = threadIdx.x; i < kc; i += blockDim.x) {
    int g = k0 + i < k1 ? g_idx[k0 + i] : 0;
    if ((unsigned)g >= (unsigned)groups) {          // a group index the scales do not have
      set_error(st, GPTQ_ERR_INVALID_ARG, k0 + i, STAGE_DEQUANT);
      g = 0;
    }
    gsm[i] = g;
  }
  __syncthreads();
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
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const int kl = w * PER + i - k0;
        const int g = gsm[kl];
        if (g != g_prev) {             // a new group: its scales and zero points for the four outputs
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
               int out, int groups, const void* X, int m_real, int ldx, float* part, int splits, int32_t* st,
               cudaStream_t s) {
  dim3 grd((unsigned)cdiv(out, 128), (unsigned)splits);
  qmatvec_kernel<TX, BITS, M><<<grd, 256, 0, s>>>(qweight, scales, zeros, g_idx, n, out, groups,
                                                   static_cast<const TX*>(X), m_real, ldx, part, st);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

template <typename TX, int BITS>
int qmv_m(int M, const int32_t* qweight, const uint16_t* scales, const uint16_t* zeros, const int32_t* g_idx, int n,
          int out, int groups, const void* X, int ldx, float* part, int splits, int32_t* st, cudaStream_t s) {
  if (M <= 1) return qmv_launch<TX, BITS, 1>(qweight, scales, zeros, g_idx, n, out, groups, X, M, ldx, part, splits, st, s);
  if (M <= 2) return qmv_launch<TX, BITS, 2>(qweight, scales, zeros, g_idx, n, out, groups, X, M, ldx, part, splits, st, s);
  if (M <= 4) return qmv_launch<TX, BITS, 4>(qweight, scales, zeros, g_idx, n, out, groups, X, M, ldx, part, splits, st, s);
  if (M <= 8) return qmv_launch<TX, BITS, 8>(qweight, scales, zeros, g_idx, n, out, groups, X, M, ldx, part, splits, st, s);
  return qmv_launch<TX, BITS, 16>(qweight, scales, zeros, g_idx, n, out, groups, X, M, ldx, part, splits, st, s);
}

}  // namespace

size_t qmatvec_ws_bytes(int M, int n, int out) {
  const int splits = (int)cdiv(n, QMV_KC);
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
                   int bits, int n, int out, int groups, const void* X, int x_dtype, int M, int ldx, float* Y, int ldy,
                   void* ws, int32_t* st, cudaStream_t s) {
  const int splits = (int)cdiv(n, QMV_KC);
  float* part = static_cast<float*>(ws);
  // bytes read once: packed weights, scales and zeros, g_idx, X; Y written
  TraceScope ts("qmatvec", "byte",
                (double)out * n * bits / 8.0 + 4.0 * (double)groups * out + 4.0 * n + 2.0 * M * n + 4.0 * M * out, s);
  int rc = GPTQ_ERR_UNSUPPORTED;
  auto go = [&](auto tx_tag) {
    using TX = decltype(tx_tag);
    if (bits == 2) return qmv_m<TX, 2>(M, qweight, scales, zeros, g_idx, n, out, groups, X, ldx, part, splits, st, s);
    if (bits == 4) return qmv_m<TX, 4>(M, qweight, scales, zeros, g_idx, n, out, groups, X, ldx, part, splits, st, s);
    return qmv_m<TX, 8>(M, qweight, scales, zeros, g_idx, n, out, groups, X, ldx, part, splits, st, s);
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
