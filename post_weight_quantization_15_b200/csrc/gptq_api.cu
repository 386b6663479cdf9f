// The C ABI (include/gptq.h): argument checks, workspace sizes, status block.
// Every call only enqueues kernels on the caller's stream; nothing is allocated.
#include <cuda_runtime.h>

#include <atomic>
#include <climits>

#include "common.cuh"
#include "internal.h"

using namespace gptq;

namespace gptq {
namespace {
std::atomic<uint64_t> g_launches{0};
}
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
void count_launches(int64_t delta) { g_launches.fetch_add((uint64_t)delta, std::memory_order_relaxed); }
}  // namespace gptq

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

bool valid_bits(int bits) { return bits == 2 || bits == 3 || bits == 4 || bits == 8; }
bool valid_gs(int gs) { return gs == -1 || gs == 32 || gs == 64 || gs == 128; }

}  // namespace

extern "C" {

int gptq_version(void) { return GPTQ_ABI_VERSION; }

uint64_t gptq_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

const char* gptq_status_string(int status) {
  switch (status) {
    case GPTQ_OK: return "ok";
    case GPTQ_ERR_INVALID_ARG: return "invalid argument";
    case GPTQ_ERR_UNSUPPORTED: return "unsupported combination";
    case GPTQ_ERR_NOT_SPD: return "damped Hessian is not positive definite";
    case GPTQ_ERR_NONFINITE: return "non-finite value in W or H";
    case GPTQ_ERR_CUDA: return "CUDA runtime error";
    case GPTQ_ERR_TIMEOUT: return "bounded device wait gave up";
    case GPTQ_ERR_WORKSPACE: return "workspace too small or misaligned";
    default: return "unknown status";
  }
}

int gptq_status_reset(int32_t* d_status, void* stream) {
  if (d_status == nullptr) return GPTQ_ERR_INVALID_ARG;
  GPTQ_CUDA_TRY(cudaMemsetAsync(d_status, 0, 4 * sizeof(int32_t), as_stream(stream)));
  return GPTQ_OK;
}

int gptq_status_read(const int32_t* d_status, void* stream, int32_t* info) {
  if (d_status == nullptr) return GPTQ_ERR_INVALID_ARG;
  int32_t h[4] = {0, 0, 0, 0};
  GPTQ_CUDA_TRY(cudaMemcpyAsync(h, d_status, sizeof(h), cudaMemcpyDeviceToHost, as_stream(stream)));
  GPTQ_CUDA_TRY(cudaStreamSynchronize(as_stream(stream)));
  if (info) *info = h[1];
  return h[0];
}

int gptq_hessian_accumulate_padded(float* H, double* hdiag, int n, const void* X, int x_rows, int64_t ld_x,
                                   int64_t tokens, int32_t* d_status, void* stream) {
  if (H == nullptr || n <= 0 || x_rows <= 0 || x_rows > n || tokens < 0) return GPTQ_ERR_INVALID_ARG;
  if (tokens == 0) return GPTQ_OK;
  if (X == nullptr || ld_x < tokens || ld_x % 8 != 0 || !aligned(X, 16)) return GPTQ_ERR_INVALID_ARG;
  int rc = launch_hessian(H, n, X, x_rows, ld_x, tokens, d_status, as_stream(stream));
  if (rc != GPTQ_OK) return rc;
  if (hdiag) rc = launch_hessian_diag64(hdiag, x_rows, X, ld_x, tokens, d_status, as_stream(stream));
  return rc;
}

int gptq_hessian_accumulate(float* H, double* hdiag, int n, const void* X, int64_t ld_x, int64_t tokens,
                            int32_t* d_status, void* stream) {
  return gptq_hessian_accumulate_padded(H, hdiag, n, X, n, ld_x, tokens, d_status, stream);
}

int gptq_hessian_accumulate_host_padded(float* H, double* hdiag, int n, const void* X_host, int x_rows,
                                        int64_t ld_x, int64_t tokens, void* staging, size_t staging_bytes,
                                        int32_t* d_status, void* stream) {
  if (H == nullptr || n <= 0 || x_rows <= 0 || x_rows > n || tokens < 0) return GPTQ_ERR_INVALID_ARG;
  if (tokens == 0) return GPTQ_OK;
  if (X_host == nullptr || ld_x < tokens) return GPTQ_ERR_INVALID_ARG;
  if (staging == nullptr || !aligned(staging, 256) || hessian_host_chunk(x_rows, staging_bytes) < 64)
    return GPTQ_ERR_WORKSPACE;
  return launch_hessian_host(H, hdiag, n, X_host, x_rows, ld_x, tokens, staging, staging_bytes, d_status,
                             as_stream(stream));
}

int gptq_hessian_accumulate_host(float* H, double* hdiag, int n, const void* X_host, int64_t ld_x, int64_t tokens,
                                 void* staging, size_t staging_bytes, int32_t* d_status, void* stream) {
  return gptq_hessian_accumulate_host_padded(H, hdiag, n, X_host, n, ld_x, tokens, staging, staging_bytes, d_status,
                                             stream);
}

size_t gptq_prepare_workspace_size(int n) { return n > 0 ? prepare_ws_bytes(n) : 0; }

int gptq_prepare(const float* H, const double* hdiag, int n, float damp_percent, int desc_act, float* U,
                 int32_t* perm, uint8_t* dead, void* ws, size_t ws_bytes, int32_t* d_status, void* stream) {
  if (H == nullptr || U == nullptr || perm == nullptr || dead == nullptr || d_status == nullptr || n <= 0)
    return GPTQ_ERR_INVALID_ARG;
  if (!(damp_percent >= 0.f) || !(damp_percent < 1e30f)) return GPTQ_ERR_INVALID_ARG;
  if (ws == nullptr || ws_bytes < prepare_ws_bytes(n) || !aligned(ws, 256)) return GPTQ_ERR_WORKSPACE;
  return launch_prepare(H, hdiag, n, damp_percent, desc_act ? 1 : 0, U, perm, dead, ws, d_status,
                        as_stream(stream));
}

int gptq_prepare_set_deferred_min_n(int min_n) { return prepare_set_deferred_min_n(min_n); }

size_t gptq_quantize_workspace_size(int out, int n, int block) {
  if (out <= 0 || n <= 0) return 0;
  return quantize_ws_bytes(out, n, block);
}

}  // extern "C"

namespace gptq {
// Every check of gptq_quantize_layer_padded except the workspace's, in the order the
// ABI reports them; shared with the entry point whose scratch is a static array.
int check_quantize_args(const void* W, int w_dtype, int out, int w_cols, int n, const float* U, int bits,
                        int group_size, int block, const int32_t* qweight, const uint16_t* scales,
                        const uint16_t* zeros, const int32_t* g_idx, const int32_t* d_status) {
  if (W == nullptr || U == nullptr || qweight == nullptr || scales == nullptr || zeros == nullptr ||
      g_idx == nullptr || d_status == nullptr)
    return GPTQ_ERR_INVALID_ARG;
  if (out <= 0 || n <= 0 || w_cols <= 0 || w_cols > n) return GPTQ_ERR_INVALID_ARG;
  if (out > GPTQ_MAX_OUT) return GPTQ_ERR_UNSUPPORTED;
  if (w_dtype != GPTQ_F32 && w_dtype != GPTQ_F16 && w_dtype != GPTQ_BF16) return GPTQ_ERR_INVALID_ARG;
  if (!valid_bits(bits) || !valid_gs(group_size)) return GPTQ_ERR_UNSUPPORTED;
  if (block != 128) return GPTQ_ERR_UNSUPPORTED;
  if (n % 32 != 0) return GPTQ_ERR_UNSUPPORTED;
  if (group_size > 0 && (n % group_size != 0 || block % group_size != 0)) return GPTQ_ERR_UNSUPPORTED;
  return GPTQ_OK;
}
}  // namespace gptq

extern "C" {

int gptq_quantize_layer_padded(const void* W, int w_dtype, int out, int w_cols, int n, const float* U,
                               const int32_t* perm, const uint8_t* dead, int bits, int group_size, int sym, int block,
                               int32_t* qweight, uint16_t* scales, uint16_t* zeros, int32_t* g_idx, uint8_t* codes,
                               float* err_sq, void* ws, size_t ws_bytes, int32_t* d_status, void* stream) {
  const int arc = check_quantize_args(W, w_dtype, out, w_cols, n, U, bits, group_size, block, qweight, scales, zeros,
                                      g_idx, d_status);
  if (arc != GPTQ_OK) return arc;
  if (ws == nullptr || ws_bytes < quantize_ws_bytes(out, n, block) || !aligned(ws, 256)) return GPTQ_ERR_WORKSPACE;
  WRows rows{};
  rows.W[0] = W;
  rows.row0[0] = 0;
  rows.row0[1] = out;
  rows.count = 1;
  return launch_quantize(rows, w_dtype, out, w_cols, n, U, perm, dead, bits, group_size, sym ? 1 : 0, block, qweight,
                         scales, zeros, g_idx, codes, err_sq, ws, d_status, as_stream(stream));
}

int gptq_quantize_layer(const void* W, int w_dtype, int out, int n, const float* U, const int32_t* perm,
                        const uint8_t* dead, int bits, int group_size, int sym, int block, int32_t* qweight,
                        uint16_t* scales, uint16_t* zeros, int32_t* g_idx, uint8_t* codes, float* err_sq,
                        void* ws, size_t ws_bytes, int32_t* d_status, void* stream) {
  return gptq_quantize_layer_padded(W, w_dtype, out, n, n, U, perm, dead, bits, group_size, sym, block, qweight,
                                    scales, zeros, g_idx, codes, err_sq, ws, ws_bytes, d_status, stream);
}

int gptq_quantize_layers(const void* const* W, const int* outs, int count, int w_dtype, int n, const float* U,
                         const int32_t* perm, const uint8_t* dead, int bits, int group_size, int sym, int block,
                         int32_t* qweight, uint16_t* scales, uint16_t* zeros, int32_t* g_idx, uint8_t* codes,
                         float* err_sq, void* ws, size_t ws_bytes, int32_t* d_status, void* stream) {
  if (W == nullptr || outs == nullptr || count < 1 || count > GPTQ_MAX_LAYERS) return GPTQ_ERR_INVALID_ARG;
  WRows rows{};
  int64_t total = 0;
  rows.row0[0] = 0;
  for (int i = 0; i < count; ++i) {
    if (W[i] == nullptr || outs[i] <= 0) return GPTQ_ERR_INVALID_ARG;
    total += outs[i];
    if (total > GPTQ_MAX_OUT) return GPTQ_ERR_UNSUPPORTED;
    rows.W[i] = W[i];
    rows.row0[i + 1] = (int)total;
  }
  rows.count = count;
  const int out = (int)total;
  const int arc = check_quantize_args(W[0], w_dtype, out, n, n, U, bits, group_size, block, qweight, scales, zeros,
                                      g_idx, d_status);
  if (arc != GPTQ_OK) return arc;
  if (ws == nullptr || ws_bytes < quantize_ws_bytes(out, n, block) || !aligned(ws, 256)) return GPTQ_ERR_WORKSPACE;
  return launch_quantize(rows, w_dtype, out, n, n, U, perm, dead, bits, group_size, sym ? 1 : 0, block, qweight,
                         scales, zeros, g_idx, codes, err_sq, ws, d_status, as_stream(stream));
}

namespace {
int check_stored(const int32_t* qweight, const uint16_t* scales, const uint16_t* zeros, const int32_t* g_idx,
                 int bits, int n, int out, int groups) {
  if (qweight == nullptr || scales == nullptr || zeros == nullptr || g_idx == nullptr) return GPTQ_ERR_INVALID_ARG;
  if (n <= 0 || out <= 0 || groups <= 0 || !aligned(qweight, 16)) return GPTQ_ERR_INVALID_ARG;
  if (bits != 2 && bits != 4 && bits != 8) return GPTQ_ERR_UNSUPPORTED;
  if ((n * bits) % 32 != 0) return GPTQ_ERR_UNSUPPORTED;
  if ((int64_t)out * 4 > (int64_t)65535 * 128 * 4) return GPTQ_ERR_UNSUPPORTED;
  return GPTQ_OK;
}
}  // namespace

int gptq_dequantize(const int32_t* qweight, const uint16_t* scales, const uint16_t* zeros, const int32_t* g_idx,
                    int bits, int n, int out, int groups, int out_dtype, void* What, int32_t* d_status,
                    void* stream) {
  const int rc = check_stored(qweight, scales, zeros, g_idx, bits, n, out, groups);
  if (rc != GPTQ_OK) return rc;
  if (What == nullptr) return GPTQ_ERR_INVALID_ARG;
  if (out_dtype != GPTQ_F32 && out_dtype != GPTQ_F16 && out_dtype != GPTQ_BF16) return GPTQ_ERR_INVALID_ARG;
  if ((int64_t)n * bits / 32 > (int64_t)65535 * 8) return GPTQ_ERR_UNSUPPORTED;
  return launch_dequant(qweight, scales, zeros, g_idx, bits, n, out, groups, out_dtype, What, d_status,
                        as_stream(stream));
}

size_t gptq_qmatvec_workspace_size(int M, int n, int out) {
  if (M <= 0 || n <= 0 || out <= 0) return 0;
  return qmatvec_ws_bytes(M, n, out);
}

int gptq_qmatvec(const int32_t* qweight, const uint16_t* scales, const uint16_t* zeros, const int32_t* g_idx,
                 const int32_t* xperm, int bits, int n, int out, int groups, const void* X, int x_dtype, int M,
                 int64_t ld_x, float* Y, int64_t ld_y, void* ws, size_t ws_bytes, int32_t* d_status, void* stream) {
  const int rc = check_stored(qweight, scales, zeros, g_idx, bits, n, out, groups);
  if (rc != GPTQ_OK) return rc;
  if (X == nullptr || Y == nullptr || M < 1 || ld_x < n || ld_y < out || ld_x > INT32_MAX || ld_y > INT32_MAX)
    return GPTQ_ERR_INVALID_ARG;
  if (M > 16) return GPTQ_ERR_UNSUPPORTED;
  if (x_dtype != GPTQ_F32 && x_dtype != GPTQ_F16 && x_dtype != GPTQ_BF16) return GPTQ_ERR_INVALID_ARG;
  if (ws == nullptr || ws_bytes < qmatvec_ws_bytes(M, n, out) || !aligned(ws, 256)) return GPTQ_ERR_WORKSPACE;
  return launch_qmatvec(qweight, scales, zeros, g_idx, bits, n, out, groups, X, xperm, x_dtype, M, (int)ld_x, Y,
                        (int)ld_y, ws, d_status, as_stream(stream));
}

size_t gptq_reorder_groups_workspace_size(int groups) { return groups > 0 ? reorder_ws_bytes(groups) : 0; }

int gptq_reorder_groups(const int32_t* qweight, const int32_t* g_idx, int bits, int n, int out, int groups,
                        int32_t* qweight_g, int32_t* g_idx_g, int32_t* xperm, void* ws, size_t ws_bytes,
                        int32_t* d_status, void* stream) {
  if (qweight == nullptr || g_idx == nullptr || qweight_g == nullptr || g_idx_g == nullptr || xperm == nullptr ||
      d_status == nullptr || n <= 0 || out <= 0 || groups <= 0 || groups > n)
    return GPTQ_ERR_INVALID_ARG;
  if (bits != 2 && bits != 4 && bits != 8) return GPTQ_ERR_UNSUPPORTED;
  if ((n * bits) % 32 != 0 || (int64_t)n * bits / 32 > 65535) return GPTQ_ERR_UNSUPPORTED;
  if (ws == nullptr || ws_bytes < reorder_ws_bytes(groups) || !aligned(ws, 256)) return GPTQ_ERR_WORKSPACE;
  return launch_reorder_groups(qweight, g_idx, bits, n, out, groups, qweight_g, g_idx_g, xperm, ws, d_status,
                               as_stream(stream));
}

int gptq_linear_bf16(const void* A, int M, int64_t lda, const void* B, int N, int64_t ldb, int K, float* C,
                     int64_t ldc, int32_t* d_status, void* stream) {
  if (A == nullptr || B == nullptr || C == nullptr || M <= 0 || N <= 0 || K <= 0) return GPTQ_ERR_INVALID_ARG;
  if (lda < K || ldb < K || ldc < N || lda % 8 != 0 || ldb % 8 != 0 || !aligned(A, 16) || !aligned(B, 16))
    return GPTQ_ERR_INVALID_ARG;
  if (cdiv(M, 128) * cdiv(N, 256) > INT32_MAX) return GPTQ_ERR_UNSUPPORTED;
  return launch_linear(A, M, lda, B, N, ldb, K, C, ldc, d_status, as_stream(stream));
}

int gptq_transpose_bf16(const void* X, int rows, int cols, int64_t ldx, void* Xt, int64_t ldt, int32_t* d_status,
                        void* stream) {
  if (X == nullptr || Xt == nullptr || rows <= 0 || cols <= 0 || ldx < cols || ldt < rows) return GPTQ_ERR_INVALID_ARG;
  if (cdiv(rows, 64) > 65535) return GPTQ_ERR_UNSUPPORTED;
  return launch_transpose_bf16(X, rows, cols, ldx, Xt, ldt, d_status, as_stream(stream));
}

int gptq_silu_mul(const float* G, const float* U, int64_t count, void* h, int32_t* d_status, void* stream) {
  if (G == nullptr || U == nullptr || h == nullptr || count < 0) return GPTQ_ERR_INVALID_ARG;
  if (!aligned(G, 16) || !aligned(U, 16) || !aligned(h, 8)) return GPTQ_ERR_INVALID_ARG;
  if (count == 0) return GPTQ_OK;
  return launch_silu_mul(G, U, count, h, d_status, as_stream(stream));
}

int gptq_residual_add(const void* X, const float* Y, int64_t count, void* Xn, int32_t* d_status, void* stream) {
  if (X == nullptr || Y == nullptr || Xn == nullptr || count < 0) return GPTQ_ERR_INVALID_ARG;
  if (!aligned(X, 8) || !aligned(Y, 16) || !aligned(Xn, 8)) return GPTQ_ERR_INVALID_ARG;
  if (count == 0) return GPTQ_OK;
  return launch_residual_add(X, Y, count, Xn, d_status, as_stream(stream));
}

int gptq_pack(const uint8_t* codes, int out, int n, int bits, int32_t* qweight, void* stream) {
  if (codes == nullptr || qweight == nullptr || out <= 0 || n <= 0) return GPTQ_ERR_INVALID_ARG;
  if (!valid_bits(bits)) return GPTQ_ERR_UNSUPPORTED;
  if (((int64_t)n * bits) % 32 != 0) return GPTQ_ERR_UNSUPPORTED;
  return launch_pack(codes, nullptr, out, n, n, bits, qweight, nullptr, as_stream(stream));
}

int gptq_pack_zeros(const uint16_t* zeros, int groups, int out, int bits, int zero_offset, int32_t* qzeros,
                    int32_t* d_status, void* stream) {
  if (zeros == nullptr || qzeros == nullptr || groups <= 0 || out <= 0) return GPTQ_ERR_INVALID_ARG;
  if (zero_offset != 0 && zero_offset != 1) return GPTQ_ERR_INVALID_ARG;
  if (!valid_bits(bits)) return GPTQ_ERR_UNSUPPORTED;
  if (((int64_t)out * bits) % 32 != 0) return GPTQ_ERR_UNSUPPORTED;
  return launch_pack_zeros(zeros, groups, out, bits, zero_offset, qzeros, d_status, as_stream(stream));
}

}  // extern "C"
