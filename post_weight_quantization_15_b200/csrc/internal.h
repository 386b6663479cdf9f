// Host-side launchers of the individual stages (internal to libgptq.so).
#pragma once

#include <cuda_runtime.h>

#include <cstring>
#include <functional>
#include <stdint.h>

#include "../../include/gptq.h"

namespace gptq {

// ---- timing trace (gptq_trace_enable): events around one launch on its stream ----
// ---- Graph replay of a whole stage (graph.cu) ----------------------------------
// The arguments a stage's launches hold by value, as words.
struct GraphKey {
  static constexpr int kWords = 40;
  uint64_t w[kWords] = {};
  int len = 0;
  bool ok = true;   // false: too many words (the stage then runs launch by launch)
  template <typename T>
  GraphKey& add(T v) {
    uint64_t x = 0;
    static_assert(sizeof(T) <= sizeof(uint64_t), "one word per value");
    memcpy(&x, &v, sizeof(T));
    if (len < kWords) w[len++] = x;
    else ok = false;
    return *this;
  }
  bool operator==(const GraphKey& o) const {
    if (len != o.len) return false;
    for (int i = 0; i < len; ++i)
      if (w[i] != o.w[i]) return false;
    return true;
  }
};
// Runs enqueue(stream) so that its work is ordered after stream s's and s continues
// after it.  The second time the same key (and device) comes, the work is captured as
// a CUDA graph, which later calls with that key replay on a stream of the library:
// launches that wait on one another across streams become graph edges.  Runs
// enqueue(s) directly the first time, with the timing trace on, when s is being
// captured by the caller, when the key does not fit, when the graph cache is full, and
// when a capture fails.
int run_graph_cached(const GraphKey& key, cudaStream_t s, const std::function<int(cudaStream_t)>& enqueue);

bool trace_enabled();   // the kernel timing trace is recording

class TraceScope {
 public:
  // kernel and unit are string literals; work is the launch's algorithmic work in unit
  TraceScope(const char* kernel, const char* unit, double work, cudaStream_t s);
  ~TraceScope();
  TraceScope(const TraceScope&) = delete;
  TraceScope& operator=(const TraceScope&) = delete;

 private:
  const char* kernel_;
  const char* unit_;
  double work_;
  cudaStream_t s_;
  void* a_;
};

// ---- K1: Hessian -----------------------------------------------------------
// H [n, n] from X's first x_rows rows (x_rows <= n; the rows after them are zero padding).
int launch_hessian(float* H, int n, const void* X, int x_rows, int64_t ld_x, int64_t tokens, int32_t* st,
                   cudaStream_t s);
int launch_hessian_diag64(double* hdiag, int n, const void* X, int64_t ld_x, int64_t tokens,
                          int32_t* st, cudaStream_t s);
int64_t hessian_host_chunk(int n, size_t staging_bytes);
int launch_hessian_host(float* H, double* hdiag, int n, const void* X_host, int x_rows, int64_t ld_x_host,
                        int64_t tokens, void* staging, size_t staging_bytes, int32_t* st, cudaStream_t s);

// ---- K2: prepare -------------------------------------------------------------
size_t prepare_ws_bytes(int n);
int prepare_set_deferred_min_n(int min_n);
int launch_prepare(const float* H, const double* hdiag, int n, float damp, int desc_act, float* U,
                   int32_t* perm, uint8_t* dead, void* ws, int32_t* st, cudaStream_t s);

// ---- K0/K3/K4/K5: quantize ---------------------------------------------------
size_t quantize_ws_bytes(int out, int n, int block);
// The argument checks of gptq_quantize_layer_padded, workspace excluded (GPTQ_OK or the error code).
int check_quantize_args(const void* W, int w_dtype, int out, int w_cols, int n, const float* U, int bits,
                        int group_size, int block, const int32_t* qweight, const uint16_t* scales,
                        const uint16_t* zeros, const int32_t* g_idx, const int32_t* d_status);
// The weights of the rows of one quantize call: up to kMaxLayers layers of one input,
// their rows concatenated (layer i holds rows row0[i] .. row0[i+1]-1).
constexpr int kMaxLayers = GPTQ_MAX_LAYERS;
struct WRows {
  const void* W[kMaxLayers];
  int row0[kMaxLayers + 1];
  int count;
};
// W [out, w_cols] (w_cols <= n; columns w_cols .. n-1 are zero padding).
int launch_quantize(const WRows& W, int w_dtype, int out, int w_cols, int n, const float* U, const int32_t* perm,
                    const uint8_t* dead, int bits, int gs, int sym, int block, int32_t* qweight,
                    uint16_t* scales, uint16_t* zeros, int32_t* g_idx, uint8_t* codes, float* err_sq,
                    void* ws, int32_t* st, cudaStream_t s);
int launch_pack(const uint8_t* codes, const int32_t* invperm, int out, int n, int ld_codes, int bits,
                int32_t* qweight, const int32_t* st, cudaStream_t s);
int launch_pack_zeros(const uint16_t* zeros, int groups, int out, int bits, int zero_offset, int32_t* qzeros,
                      int32_t* st, cudaStream_t s);

// ---- the consumer of the stored format (dequant.cu) -----------------------------
int launch_dequant(const int32_t* qweight, const uint16_t* scales, const uint16_t* zeros, const int32_t* g_idx,
                   int bits, int n, int out, int groups, int dtype, void* What, int32_t* st, cudaStream_t s);
size_t qmatvec_ws_bytes(int M, int n, int out);
int launch_qmatvec(const int32_t* qweight, const uint16_t* scales, const uint16_t* zeros, const int32_t* g_idx,
                   int bits, int n, int out, int groups, const void* X, const int32_t* xperm, int x_dtype, int M,
                   int ldx, float* Y, int ldy, void* ws, int32_t* st, cudaStream_t s);
size_t reorder_ws_bytes(int groups);
int launch_reorder_groups(const int32_t* qweight, const int32_t* g_idx, int bits, int n, int out, int groups,
                          int32_t* qweight_g, int32_t* g_sorted, int32_t* xperm, void* ws, int32_t* st,
                          cudaStream_t s);

// ---- a quantized block's forward pass (linear.cu, forward.cu) -----------------------
int launch_linear(const void* A, int M, int64_t lda, const void* B, int N, int64_t ldb, int K, float* C, int64_t ldc,
                  int32_t* st, cudaStream_t s);
int launch_transpose_bf16(const void* X, int rows, int cols, int64_t ldx, void* Xt, int64_t ldt, const int32_t* st,
                          cudaStream_t s);
int launch_silu_mul(const float* G, const float* U, int64_t count, void* h, const int32_t* st, cudaStream_t s);
int launch_residual_add(const void* X, const float* Y, int64_t count, void* Xn, const int32_t* st, cudaStream_t s);

// ---- tensor-core GEMM: C -= A . B^T in 3 x TF32 (operands pre-split) ---------
// store = false: C -= A.B^T; store = true: C = A.B^T (C may be null then, if Chi/Clo are given).
// Chi/Clo (optional, leading dimension ldh) receive the TF32 split of the result.
// lower: only tiles reaching the lower triangle of square C.
// trace: the kernel name the timing trace records this launch under (nullptr: not traced).
int launch_gemm3(float* C, int ldc, int M, int N, int K, const float* Ahi, const float* Alo, int lda,
                 const float* Bhi, const float* Blo, int ldb, bool lower, int32_t* st, cudaStream_t s,
                 bool store = false, float* Chi = nullptr, float* Clo = nullptr, int ldh = 0,
                 const char* trace = nullptr);
int launch_split_tf32(const float* X, int rows, int cols, int ldx, float* hi, float* lo, int ldo,
                      const int32_t* st, cudaStream_t s);

}  // namespace gptq
