/*
 * gptq.h - C ABI of the B200 GPTQ layer-solver library (libgptq.so).
 *
 * GPTQ quantizes one linear layer W [out, in] so that ||W.X - What.X||^2 is small
 * ("polydesk.ai/glossaire/gptq", section "Comment fonctionne l'algorithme GPTQ"):
 * columns are quantized one after another, and each column's rounding error is
 * pushed onto the columns not yet quantized through the upper Cholesky factor of
 * the damped inverse Hessian, in lazy batches of 128 columns (same page, "Etape 2"
 * and "Etape 3").  The calls below are the steps of that path:
 *
 *   gptq_hessian_accumulate   H += 2 . X . X^T                    ("Etape 2")
 *   gptq_prepare              dead inputs, act-order, damping, U  ("Etape 2"; desc_act)
 *   gptq_quantize_layer       column sweep, lazy trailing update,
 *                             packed qweight / fp16 scales, zeros / g_idx
 *   gptq_pack                 the bit-packing step on its own
 *   gptq_pack_zeros           zero points packed into int32 words
 *   *_padded                  the same for a zero-padded layer ("Limites de GPTQ")
 *
 * Conventions shared by every call
 * --------------------------------
 * - All tensor pointers are DEVICE pointers to memory the caller owns.  The
 *   library allocates nothing: calls that need scratch take a caller-provided
 *   workspace whose size the matching *_workspace_size() call reports.
 * - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *   Every call only enqueues work and returns; calls on one stream run in order.
 *   Calls on different streams that share buffers race.  gptq_prepare,
 *   gptq_quantize_layer and the host-memory Hessian run parts of their work on
 *   streams of the library's own (one set per host thread and device, created on
 *   the first call) that fork from `stream` and join it again before the call
 *   returns, so `stream` is ordered after all of a call's work, after an error
 *   too.  Make the first such call on a device outside any stream capture.
 * - Argument errors are returned synchronously (nothing is enqueued).
 *   Errors found on the device (a non-positive Cholesky pivot, non-finite
 *   values, a bounded wait that gave up) are recorded in a caller-provided
 *   device status block `d_status` (int32[4]: code, info, stage, reserved):
 *   the first error wins, and every later kernel that sees a non-zero code
 *   skips its work.  Clear it with gptq_status_reset() before a layer and read
 *   it with gptq_status_read(), which synchronizes the stream.
 * - Matrices are row-major with the stated leading dimensions.
 * - The library targets sm_100a (B200) only.
 */
#ifndef GPTQ_B200_H
#define GPTQ_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GPTQ_ABI_VERSION 1

#if defined(__GNUC__)
#define GPTQ_API __attribute__((visibility("default")))
#else
#define GPTQ_API
#endif

typedef enum {
  GPTQ_OK = 0,
  GPTQ_ERR_INVALID_ARG = -1,  /* a pointer, size or stride is invalid               */
  GPTQ_ERR_UNSUPPORTED = -2,  /* a valid combination the library does not implement */
  GPTQ_ERR_NOT_SPD = -3,      /* damped Hessian not positive definite; info = pivot  */
  GPTQ_ERR_NONFINITE = -4,    /* NaN/Inf in W or H; info = column or pivot           */
  GPTQ_ERR_CUDA = -5,         /* a CUDA runtime call failed                          */
  GPTQ_ERR_TIMEOUT = -6,      /* a bounded on-device wait gave up                    */
  GPTQ_ERR_WORKSPACE = -7     /* workspace too small or misaligned                   */
} gptq_status;

typedef enum { GPTQ_F32 = 0, GPTQ_F16 = 1, GPTQ_BF16 = 2 } gptq_dtype;

/* Largest number of output rows gptq_quantize_layer accepts (8 x 65535). */
#define GPTQ_MAX_OUT 524280

/* Library / ABI version (GPTQ_ABI_VERSION). */
GPTQ_API int gptq_version(void);

/* Number of kernels this library has enqueued since it was loaded (all
 * devices, all streams; host-side counter, for accounting in benchmarks). */
GPTQ_API uint64_t gptq_kernel_launches(void);

/* Human-readable name of a gptq_status code (static string). */
GPTQ_API const char* gptq_status_string(int status);

/* Clears the device status block (int32[4]) on `stream`. */
GPTQ_API int gptq_status_reset(int32_t* d_status, void* stream);

/* Synchronizes `stream`, then returns the code stored in d_status[0]
 * (GPTQ_OK if none) and, when `info` is not NULL, d_status[1] (the failing
 * pivot or column).  Returns GPTQ_ERR_CUDA if the synchronization fails. */
GPTQ_API int gptq_status_read(const int32_t* d_status, void* stream, int32_t* info);

/*
 * gptq_hessian_accumulate - H += 2 . X . X^T on the tensor cores.
 *
 * "polydesk.ai/glossaire/gptq", "Etape 2": the Hessian is approximated by
 * H = 2.X.X^T from the calibration activations.  Calling this once per chunk
 * of tokens accumulates the sum over all chunks.
 *
 *   H        fp32 [n, n], ld = n.  Only the upper triangle (j >= i) is updated
 *            and later read; the lower triangle is left unspecified (diagonal
 *            tiles may write it).  Zero it before the first chunk.
 *   hdiag    optional fp64 [n] (NULL to skip): hdiag[i] += 2 . sum_t X[i,t]^2,
 *            accumulated in fp64 from exact bf16 squares.  gptq_prepare uses it
 *            as the act-order key, so that the order does not depend on the
 *            fp32 summation order of H.
 *   X        bf16 [n, tokens] (features x tokens, tokens contiguous), row
 *            stride ld_x elements; ld_x % 8 == 0 and X 16-byte aligned.
 *   tokens   may be 0 (no-op).  Any n >= 1 and tokens >= 0 are accepted.
 *   d_status may be NULL; bounded waits that give up report GPTQ_ERR_TIMEOUT there.
 */
GPTQ_API int gptq_hessian_accumulate(float* H, double* hdiag, int n, const void* X, int64_t ld_x,
                            int64_t tokens, int32_t* d_status, void* stream);

/*
 * gptq_hessian_accumulate_host - the same accumulation with X in HOST memory.
 *
 * Same computation and arguments as gptq_hessian_accumulate ("polydesk.ai/glossaire/
 * gptq", "Etape 2"), except that X stays on the host: it is copied to the device in
 * chunks of tokens, one strided copy per chunk, into a caller-provided device staging
 * area, and the tile product of each chunk runs while the next one is copied, so
 * that the transfer of the activations hides the contraction.  This is the one call
 * whose X pointer is a host pointer; everything else is as above.
 *
 *   X_host         bf16 [n, tokens] in host memory, row stride ld_x elements
 *                  (ld_x >= tokens).  Page-locked (pinned) memory lets the copies run
 *                  asynchronously; pageable memory still gives the right result but the
 *                  copies then do not overlap the work.  The caller keeps X_host alive
 *                  and unchanged until the stream has passed this call.
 *   staging        device buffer of staging_bytes, 256-byte aligned, owned by the
 *                  caller; it is split in two halves of n x C bf16, C the largest
 *                  multiple of 64 tokens that fits (at least 64, else
 *                  GPTQ_ERR_WORKSPACE).  Larger areas mean fewer, longer chunks.
 *   stream         the tile products run on it; the copies run on a stream of the
 *                  library's own (one per host thread and device, created on first use)
 *                  that is ordered after the work already queued on `stream`, and every
 *                  kernel waits for its chunk's copy, so `stream` is ordered after all of
 *                  this call's copies and kernels.
 * Errors: as gptq_hessian_accumulate; a failed copy returns GPTQ_ERR_CUDA.
 */
GPTQ_API int gptq_hessian_accumulate_host(float* H, double* hdiag, int n, const void* X_host, int64_t ld_x,
                                          int64_t tokens, void* staging, size_t staging_bytes,
                                          int32_t* d_status, void* stream);

/*
 * gptq_prepare - dead inputs, act-order, damping and the Cholesky factor U.
 *
 * In this order (the readings are those of the library's oracle):
 *  1. inputs with diag(H) == 0 are dead: H_ii := 1 and dead[i] = 1;
 *  2. desc_act ("polydesk.ai/glossaire/gptq", desc_act: decreasing activation
 *     magnitude): perm = stable descending order of the key (hdiag if given,
 *     else diag(H); dead inputs have key 1); otherwise perm = identity;
 *  3. damping ("skillmd.com/skills/artubss/gptq", damp_percent): the permuted H
 *     gets lambda = damp_percent . mean(diag H) added to its diagonal;
 *  4. U = the upper-triangular Cholesky factor of the damped, permuted H^-1
 *     (H^-1 = U^T . U), computed in fp32 through a Cholesky factorization
 *     ("polydesk.ai/glossaire/gptq", "Etape 2").
 *
 *   H        fp32 [n, n] (upper triangle read; not modified).
 *   hdiag    optional fp64 [n] act-order key (see gptq_hessian_accumulate).
 *   U        fp32 [n, n] output, row-major, strictly-lower part set to 0.
 *   perm     int32 [n] output: processing position k holds input column perm[k].
 *   dead     uint8 [n] output.
 *   ws       workspace of at least gptq_prepare_workspace_size(n) bytes, 256-byte aligned.
 *   d_status required: GPTQ_ERR_NOT_SPD (info = failing pivot, in processing
 *            order) or GPTQ_ERR_NONFINITE.
 */
GPTQ_API size_t gptq_prepare_workspace_size(int n);
GPTQ_API int gptq_prepare(const float* H, const double* hdiag, int n, float damp_percent, int desc_act,
                 float* U, int32_t* perm, uint8_t* dead, void* ws, size_t ws_bytes,
                 int32_t* d_status, void* stream);

/*
 * gptq_prepare_set_deferred_min_n - how gptq_prepare groups its bulk updates.
 *
 * gptq_prepare factors H in 128-wide panels.  For n >= min_n (default 8192) four
 * panels form a 512-wide outer panel whose trailing and inverse updates are
 * applied once, as rank-512 products, instead of once per panel as rank-128
 * products: the same terms, a quarter of the passes over the trailing matrices.
 * The two forms differ only in the order in which those terms are summed.
 *   min_n    the new threshold; min_n <= 0 only queries.
 * Returns the previous threshold.  Process-wide; a call that races a
 * gptq_prepare on another thread may or may not apply to it.
 */
GPTQ_API int gptq_prepare_set_deferred_min_n(int min_n);

/*
 * gptq_set_graph_replay - whether gptq_prepare and gptq_quantize_layer(s) replay CUDA
 * graphs.
 *
 * Each of those calls enqueues a chain of small dependent launches on several
 * streams.  When replay is on (the default), the second call with exactly the same
 * arguments (every pointer, size and setting, on the same device) captures the call's
 * launches as a CUDA graph (a one-time host cost of milliseconds), and later calls
 * with those arguments replay it: the same kernels on the same data, their
 * cross-stream dependencies turned into graph edges, the same results bit for bit.
 * The data behind the pointers is read when the graph runs.  Calls enqueue launch by
 * launch the first time, while the timing trace is on, while the caller's stream is
 * being captured, and once 32 graphs exist (the library keeps them until unload).
 * Replay pays off in loops that call with the same buffers; a caller that allocates
 * fresh buffers for every call gains nothing from it and pays the captures.
 *   on       1: on; 0: off; < 0: only query.
 * Returns the previous setting.  Per host thread: it governs the calls the calling
 * thread makes (each thread starts with replay on).
 */
GPTQ_API int gptq_set_graph_replay(int on);

/*
 * gptq_quantize_layer - the column sweep, the lazy trailing update and packing.
 *
 * For every column j in processing order ("polydesk.ai/glossaire/gptq",
 * "Etape 2"): at a group start the group's per-row scale and zero point are
 * computed from the current, already compensated weights; the column is
 * quantized (round to nearest even, decided in fp32); e = (w - what) / U_jj;
 * the remaining columns of the block absorb e . U[j, :]; after each block of
 * `block` columns the later columns absorb Err . U[block, later] at once
 * ("Etape 3").  Symmetric codes use the grid [-2^(b-1)+1, 2^(b-1)-1] offset by
 * z = 2^(b-1) ("sym"); asymmetric codes use a zero point in [0, 2^b-1].
 *
 *   W          [out, n] row-major, dtype w_dtype (F32, F16 or BF16); not modified.
 *   U, perm, dead   from gptq_prepare (perm and dead may be NULL: identity / none).
 *              With perm NULL the sweep also packs: it writes qweight itself,
 *              block by block, and the separate packing launch is skipped (the
 *              same bits; the packing then joins the sweep's dependent chain, which
 *              measured slower than the separate launch: pass the identity perm
 *              from gptq_prepare to keep the separate packing).
 *   bits       2, 3, 4 or 8.     group_size 32, 64, 128, or -1 (one group per row).
 *   block      128 (the pages' batch); block % group_size == 0 when group_size > 0.
 *   n % 32 == 0, and n % group_size == 0 when group_size > 0.
 *   1 <= out <= GPTQ_MAX_OUT (GPTQ_ERR_UNSUPPORTED above: the row kernels put
 *   eight rows per block along the grid's second dimension).
 *   qweight    int32 [n*bits/32, out]: per output row, the codes of the input
 *              columns in original order as a little-endian bit stream (column k
 *              at stream bits k*bits ...), word-major.
 *   scales, zeros   fp16 (as uint16) [G, out], G = n / group_size (1 if -1),
 *              in group (processing) order; zeros hold integers.
 *   g_idx      int32 [n]: group of each input column (original order).
 *   codes      optional uint8 [out, n], original column order (NULL to skip).
 *   err_sq     optional fp32 [out]: per row, sum_j e_j^2 (NULL to skip).
 *   ws         >= gptq_quantize_workspace_size(out, n, block) bytes, 256-byte aligned.
 */
GPTQ_API size_t gptq_quantize_workspace_size(int out, int n, int block);
GPTQ_API int gptq_quantize_layer(const void* W, int w_dtype, int out, int n, const float* U,
                        const int32_t* perm, const uint8_t* dead, int bits, int group_size,
                        int sym, int block, int32_t* qweight, uint16_t* scales, uint16_t* zeros,
                        int32_t* g_idx, uint8_t* codes, float* err_sq, void* ws, size_t ws_bytes,
                        int32_t* d_status, void* stream);

/*
 * gptq_quantize_layers - gptq_quantize_layer for several layers that read the same
 * input (a decoder block's q, k and v; its gate and up), in one call.
 *
 * "polydesk.ai/glossaire/gptq", "Etape 1": the order of the columns, and with it the
 * inverse-Hessian work, is shared by every row, and rows are independent given U.
 * So the rows of layers that share H (and U) are quantized as the rows of one layer
 * whose weights are the layers' weights stacked along the outputs: qweight, scales,
 * zeros, g_idx and codes are bit for bit those of one gptq_quantize_layer call per
 * layer (err_sq up to the order of its per-row sum, which depends on the rows per
 * launch), and the row kernels get more rows per launch.
 *
 *   W          HOST array of `count` DEVICE pointers; W[i] is [outs[i], n] row-major,
 *              all of dtype w_dtype.  1 <= count <= GPTQ_MAX_LAYERS.
 *   outs       HOST array of the layers' row counts (each >= 1, sum <= GPTQ_MAX_OUT).
 *   outputs    those of gptq_quantize_layer for the stacked layer, out = sum(outs):
 *              qweight [n*bits/32, out], scales / zeros [G, out], codes [out, n],
 *              err_sq [out]; layer i owns output columns (qweight, scales, zeros) and
 *              rows (codes, err_sq) row0 .. row0 + outs[i] - 1, row0 = outs[0] + ... +
 *              outs[i-1]; g_idx [n] is shared.
 *   ws         >= gptq_quantize_workspace_size(out, n, block) bytes.
 * Everything else, errors included, as gptq_quantize_layer.
 */
#define GPTQ_MAX_LAYERS 8
GPTQ_API int gptq_quantize_layers(const void* const* W, const int* outs, int count, int w_dtype, int n,
                                  const float* U, const int32_t* perm, const uint8_t* dead, int bits,
                                  int group_size, int sym, int block, int32_t* qweight, uint16_t* scales,
                                  uint16_t* zeros, int32_t* g_idx, uint8_t* codes, float* err_sq, void* ws,
                                  size_t ws_bytes, int32_t* d_status, void* stream);

/*
 * gptq_pack - bit-packing on its own: codes uint8 [out, n] (original order)
 * -> qweight int32 [n*bits/32, out], the layout gptq_quantize_layer writes.
 * bits in {2, 3, 4, 8}; n*bits % 32 == 0; codes must be < 2^bits.
 */
GPTQ_API int gptq_pack(const uint8_t* codes, int out, int n, int bits, int32_t* qweight, void* stream);

/*
 * Zero padding of a layer whose width the group size or the packing does not
 * divide.  "polydesk.ai/glossaire/gptq", section "Limites de GPTQ" (problems of
 * divisibility): when a width is not a multiple of the group size, the weights
 * are padded with zeros.  The padded layer has n >= w_cols input columns: W's
 * columns w_cols .. n-1 and X's rows x_rows .. n-1 are zero.  The calls below
 * compute exactly what the unpadded calls compute on those zero-padded arrays,
 * without the arrays being formed:
 *
 * - gptq_hessian_accumulate_padded: H [n, n] from X's x_rows rows
 *   (1 <= x_rows <= n).  Rows and columns x_rows .. n-1 of H receive nothing
 *   (the caller zeroed H, so they stay 0); hdiag entries x_rows .. n-1 are not
 *   touched.  Everything else as gptq_hessian_accumulate (X is [x_rows, ld_x]).
 * - gptq_hessian_accumulate_host_padded: the same with X in host memory; only
 *   x_rows rows cross, and the staging halves hold x_rows x C bf16.
 * - gptq_prepare on that H (n) is the ordinary call: the padded inputs have a
 *   zero diagonal, so step 1 makes them dead inputs, counted in the mean of the
 *   damping like every other input.
 * - gptq_quantize_layer_padded: W is [out, w_cols] (row stride w_cols,
 *   1 <= w_cols <= n); columns w_cols .. n-1 are read as zeros.  Outputs are
 *   those of the padded layer: qweight [n*bits/32, out], scales / zeros [G, out]
 *   with G = n / group_size, g_idx [n], codes [out, n].  A padded column gets the
 *   zero point's code, which dequantizes to 0.
 * Pick n = the next multiple of max(32, group_size) (32 for group_size -1).
 */
GPTQ_API int gptq_hessian_accumulate_padded(float* H, double* hdiag, int n, const void* X, int x_rows,
                                            int64_t ld_x, int64_t tokens, int32_t* d_status, void* stream);
GPTQ_API int gptq_hessian_accumulate_host_padded(float* H, double* hdiag, int n, const void* X_host, int x_rows,
                                                 int64_t ld_x, int64_t tokens, void* staging, size_t staging_bytes,
                                                 int32_t* d_status, void* stream);
GPTQ_API int gptq_quantize_layer_padded(const void* W, int w_dtype, int out, int w_cols, int n, const float* U,
                                        const int32_t* perm, const uint8_t* dead, int bits, int group_size,
                                        int sym, int block, int32_t* qweight, uint16_t* scales, uint16_t* zeros,
                                        int32_t* g_idx, uint8_t* codes, float* err_sq, void* ws, size_t ws_bytes,
                                        int32_t* d_status, void* stream);

/*
 * gptq_pack_zeros - the zero points packed into int32 words along the output
 * dimension, for checkpoint layouts that store them that way.  The pages store
 * scale and zero point in FP16 ("dev.ayinedjimi-consultants.fr ...
 * ia-quantization-gptq-gguf-awq", "Calibration et dataset"), which is what
 * gptq_quantize_layer writes, and warn that checkpoints of different tool
 * versions are not all compatible ("polydesk.ai/glossaire/gptq", "Limites de
 * GPTQ"); this call converts the fp16 zeros to the packed integer form.
 *
 *   zeros        fp16 (as uint16) [groups, out], integers in [0, 2^bits - 1]
 *                (as gptq_quantize_layer writes them).
 *   qzeros       int32 [groups, out*bits/32] output: row g is the little-endian
 *                bit stream of (zeros[g][o] - zero_offset) mod 2^bits, column o
 *                at stream bits o*bits ... (bit (o*bits) mod 32 of word
 *                floor(o*bits/32)); a 3-bit value may continue into the next word.
 *   zero_offset  0: the zero points as they are; 1: zero point - 1, the
 *                convention of older checkpoints (a zero point of 0 wraps to
 *                2^bits - 1).
 *   bits in {2, 3, 4, 8}; out*bits % 32 == 0.
 *   d_status     may be NULL; a zero that is not an integer in [0, 2^bits - 1]
 *                records GPTQ_ERR_INVALID_ARG (info = g*out + o) and is packed
 *                masked to bits.
 */
GPTQ_API int gptq_pack_zeros(const uint16_t* zeros, int groups, int out, int bits, int zero_offset,
                             int32_t* qzeros, int32_t* d_status, void* stream);

/*
 * The consumer side of the stored format.  The pages name the inference kernels
 * that read GPTQ's packed weights (Marlin, ExLlama: "skillmd.com/skills/artubss/gptq",
 * "Backends de inferencia") and store scale and zero point in FP16 ("dev.ayinedjimi-
 * consultants.fr ... ia-quantization-gptq-gguf-awq", "Calibration et dataset").  Both
 * calls read what gptq_quantize_layer writes: qweight int32 [n*bits/32, out], scales
 * and zeros fp16 [groups, out], g_idx int32 [n] (any order, act-order included).
 * bits in {2, 4, 8} (3-bit codes straddle words: GPTQ_ERR_UNSUPPORTED).  A g_idx
 * entry outside [0, groups) is recorded in d_status (GPTQ_ERR_INVALID_ARG, info = its
 * column) and read as group 0.  qweight 16-byte aligned; out % 4 == 0 for the
 * vectorised path (any out works).
 *
 * gptq_dequantize - What[o][k] = scales[g_idx[k]][o] . (code(o, k) - zeros[g_idx[k]][o])
 *   into What [out, n] row-major of dtype out_dtype (GPTQ_F32: exact, the product of an
 *   fp16 scale and a small integer being exact in fp32; GPTQ_F16 / GPTQ_BF16: rounded
 *   once to nearest even).
 *
 * gptq_qmatvec - Y[M, out] = X[M, n] . What^T for 1 <= M <= 16 activation rows (the
 *   decode shapes), the weights dequantized in registers and never written: the call
 *   reads qweight once, so HBM bandwidth bounds it.  X of dtype x_dtype (F16, BF16 or
 *   F32), row stride ld_x; Y fp32, row stride ld_y (>= out).  xperm: NULL, or int32 [n]
 *   (column k of the packed layer multiplies column xperm[k] of X: the form that
 *   gptq_reorder_groups writes).  Sums in fp32, in an order fixed by the shapes and
 *   the data's group layout (deterministic).  With 4-bit codes, M <= 2, F16 / BF16
 *   activations, integer zero points in [0, 127] and every 32 consecutive columns of a
 *   block in one group, the products x . (c - z) (exact) are summed on the tensor cores
 *   (mma.sync, fp32 accumulation, at most 128 columns per accumulation) and scaled in
 *   fp32; otherwise by fp32 fma.  ws: >= gptq_qmatvec_workspace_size(M, n, out) bytes, 256-byte
 *   aligned (the partial sums of the k splits).  Fastest when the groups of nearby
 *   columns are contiguous (no act-order, or a reordered layer): their scales and zero
 *   points are then staged once per block of columns.
 *
 * gptq_reorder_groups - once per layer, for act-order layers (whose g_idx scatters the
 *   groups over the columns): xperm = the columns sorted by group (ties in column
 *   order), g_idx_g[k] = g_idx[xperm[k]] (non-decreasing), and qweight_g [n*bits/32,
 *   out] holding the codes of columns xperm[k] at position k.  The sum over columns does
 *   not depend on their order, so gptq_qmatvec(qweight_g, scales, zeros, g_idx_g,
 *   xperm, ...) is the same product as on the original layer (up to the order of the
 *   fp32 additions).  ws >= gptq_reorder_groups_workspace_size(groups) bytes.
 *   n * bits / 32 <= 65535.
 */
GPTQ_API int gptq_dequantize(const int32_t* qweight, const uint16_t* scales, const uint16_t* zeros,
                             const int32_t* g_idx, int bits, int n, int out, int groups, int out_dtype, void* What,
                             int32_t* d_status, void* stream);
GPTQ_API size_t gptq_qmatvec_workspace_size(int M, int n, int out);
GPTQ_API int gptq_qmatvec(const int32_t* qweight, const uint16_t* scales, const uint16_t* zeros,
                          const int32_t* g_idx, const int32_t* xperm, int bits, int n, int out, int groups,
                          const void* X, int x_dtype, int M, int64_t ld_x, float* Y, int64_t ld_y, void* ws,
                          size_t ws_bytes, int32_t* d_status, void* stream);
GPTQ_API size_t gptq_reorder_groups_workspace_size(int groups);
GPTQ_API int gptq_reorder_groups(const int32_t* qweight, const int32_t* g_idx, int bits, int n, int out, int groups,
                                 int32_t* qweight_g, int32_t* g_idx_g, int32_t* xperm, void* ws, size_t ws_bytes,
                                 int32_t* d_status, void* stream);

/*
 * A quantized block's forward pass, for the sequential pipeline: the pages quantize
 * layer by layer ("polydesk.ai/glossaire/gptq"; "wikiprompt.org", "GPTQ"), each
 * layer calibrated on the activations the layers quantized before it produce.
 * Activations keep the layout of gptq_hessian_accumulate's X: [features, tokens] bf16,
 * tokens contiguous.
 *
 * gptq_linear_bf16 - C[M, N] = A[M, K] . B[N, K]^T on the tensor cores (bf16 in, fp32
 *   accumulate in chunks of 256 added in fp32 registers, fp32 out).  A and B row-major,
 *   K contiguous (lda, ldb >= K, multiples of 8, 16-byte aligned); C fp32, row stride
 *   ldc >= N.  With A = the dequantized weights [out, in] and B = the activations
 *   transposed [tokens, in], C is the layer's output [out, tokens].
 * gptq_transpose_bf16 - Xt[c][r] = X[r][c] for X [rows, cols] (row strides ldx, ldt).
 * gptq_silu_mul - h = bf16(silu(G) . U) elementwise over count fp32 values (G, U
 *   16-byte aligned, h 8-byte aligned), silu(g) = g / (1 + exp(-g)): the gated MLP.
 * gptq_residual_add - Xn = bf16(X + Y) elementwise, X bf16, Y fp32.
 * d_status may be NULL; a bounded wait of the product that gives up reports
 * GPTQ_ERR_TIMEOUT there.
 */
GPTQ_API int gptq_linear_bf16(const void* A, int M, int64_t lda, const void* B, int N, int64_t ldb, int K, float* C,
                              int64_t ldc, int32_t* d_status, void* stream);
GPTQ_API int gptq_transpose_bf16(const void* X, int rows, int cols, int64_t ldx, void* Xt, int64_t ldt,
                                 int32_t* d_status, void* stream);
GPTQ_API int gptq_silu_mul(const float* G, const float* U, int64_t count, void* h, int32_t* d_status, void* stream);
GPTQ_API int gptq_residual_add(const void* X, const float* Y, int64_t count, void* Xn, int32_t* d_status,
                               void* stream);

/*
 * Kernel timing trace.  The GPTQ pages have no counterpart to these calls: they
 * are a measurement aid.  While the trace is on, every kernel the library launches
 * is bracketed by two CUDA events recorded on the stream it is launched on (the
 * caller's or one of the library's own), so that each kernel's device time can be
 * read inside a whole call, where several library streams overlap.
 *
 *   gptq_trace_enable(on)   1: record from now on; 0: stop recording (what was
 *                           recorded stays until read).  Process-wide, all devices.
 *   gptq_trace_read(rows, max_rows, n_rows)
 *                           synchronizes every recorded event, aggregates them per
 *                           kernel (first-launch order) into rows[0 .. *n_rows),
 *                           and clears the record (rows beyond max_rows are
 *                           dropped).  Per row: kernel name, the unit of `work`
 *                           ("flop": useful floating-point operations of the
 *                           algorithm; "byte": algorithmic HBM bytes; "" none),
 *                           launches, summed device milliseconds and summed work.
 *                           Returns GPTQ_ERR_CUDA if an event could not be read.
 * Recording costs two event records per launch; the events are created per
 * launch and destroyed when read.  Make no call with the trace on inside a stream
 * capture.
 */
typedef struct {
  const char* kernel;
  const char* work_unit;
  uint64_t launches;
  double ms;
  double work;
} gptq_trace_row;
GPTQ_API int gptq_trace_enable(int on);
GPTQ_API int gptq_trace_read(gptq_trace_row* rows, int max_rows, int* n_rows);

/*
 * gptq_trace_read_timeline - the same record, launch by launch instead of aggregated:
 * per recorded launch (in the order the launches were enqueued) the kernel name, the
 * stream it went to (an opaque id: launches with equal ids ran in order on one
 * stream) and its start and end in milliseconds from the earliest recorded start
 * (records of the first record's device only).  Start and end are events recorded
 * on the launch's stream just before and after it, so a launch that waited for
 * another stream starts once that wait is over.  Synchronizes every recorded event
 * and clears the record, like gptq_trace_read (launches beyond max_events are
 * dropped).  Returns GPTQ_ERR_CUDA if an event could not be read.
 */
typedef struct {
  const char* kernel;
  uint64_t stream;
  double start_ms;
  double end_ms;
} gptq_trace_event;
GPTQ_API int gptq_trace_read_timeline(gptq_trace_event* events, int max_events, int* n_events);

/*
 * gptq_probe_fp32_peak - measurement aid (no counterpart on the pages): launches
 * `blocks` blocks of 256 threads, each thread running 8 independent chains of
 * iters x 16 fp32 FMAs (2 . blocks . 256 . iters . 128 flop in all) on `stream`;
 * timed by the caller, it gives the FP32 CUDA-core peak that bounds the library's
 * non-tensor kernels.  `out` is device memory of blocks . 256 floats that the
 * kernel may write (it normally writes nothing).
 */
GPTQ_API int gptq_probe_fp32_peak(float* out, int blocks, int iters, void* stream);

/*
 * gptq_quantize_layer_noalloc - gptq_quantize_layer without a caller workspace.
 *
 * The GPTQ pages have no counterpart to this call: it exists for callers that
 * cannot allocate device memory where they quantize (a plugin whose host
 * application owns all device allocations, code that may run while a stream is
 * being captured, a service that must not grow its footprint after start-up).
 * Arguments, layouts, results and errors are those of gptq_quantize_layer; the
 * caller still provides every input and output.  The scratch comes from a
 * static device array of GPTQ_NOALLOC_SCRATCH_BYTES inside the library instead
 * of `ws`:
 *
 * - The arguments are checked first, exactly as gptq_quantize_layer checks them
 *   (same codes, same order); then a layer whose
 *   gptq_quantize_workspace_size(out, n, block) exceeds
 *   GPTQ_NOALLOC_SCRATCH_BYTES is rejected with GPTQ_ERR_WORKSPACE.  Nothing is
 *   enqueued in either case.
 * - Every GPU that loads the library holds one copy of the array until the
 *   process exits.  The first call on a device looks up the array's device
 *   address (cudaGetSymbolAddress, with that device current) and caches it for
 *   the life of the process; make that first call before any stream capture,
 *   and do not use this call across cudaDeviceReset (the cached address would
 *   belong to the destroyed context).
 * - All calls on a device share the array, which keeps the last call's
 *   contents (every byte a call reads from it is written by the same call
 *   first).  Calls whose work overlaps on the GPU - on different streams, or
 *   from host threads that do not order them - race on it.
 * - Nothing is allocated: no cudaMalloc, cudaFree or allocating library call.
 */
#define GPTQ_NOALLOC_SCRATCH_BYTES (32u << 20)
GPTQ_API int gptq_quantize_layer_noalloc(const void* W, int w_dtype, int out, int n, const float* U,
                                         const int32_t* perm, const uint8_t* dead, int bits, int group_size,
                                         int sym, int block, int32_t* qweight, uint16_t* scales,
                                         uint16_t* zeros, int32_t* g_idx, uint8_t* codes, float* err_sq,
                                         int32_t* d_status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* GPTQ_B200_H */
