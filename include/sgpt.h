/*
 * sgpt.h - C ABI of the B200 (sm_100a) SparseGPT layer solver.
 *
 * The operation: given the weights W [d_out x d_in] of one linear layer and
 * calibration inputs X [n_tok x d_in], find a sparse W^ whose outputs W^X stay
 * as close as possible to WX under an N:M or unstructured sparsity pattern,
 * compensating every removed weight in the remaining weights of its row.
 *   - Problem statement: SparseGPT review ("SparseGPT: Massive Language Models
 *     Can Be Accurately Pruned in One-Shot", devpress.csdn.net), section 六.
 *   - Hessian proxy H = X X^T: same page, section 七.
 *   - Optimal-Brain-Surgeon removal with compensation: section 八.
 *   - Layer-wise pipeline, columns processed block by block: section 十一.
 *   - N:M (2:4) semi-structured sparsity: section 十四 14.4. The N:M GPU formats
 *     2:4, 16:32, 16:64 and 16:128: "Sparse Fine-tuning for Inference
 *     Acceleration of Large Language Models" review (tqpw.cn), section 八 8.4.
 *   - 2:4 storage, values plus 2-bit position metadata: "LLM 2:4 structured
 *     sparsity production guide" (oh-bug.com), section "2:4 结构化稀疏的核心机制
 *     与生产状态分类".
 *
 * Conventions for every call below.
 *   - All array arguments are DEVICE pointers into memory the caller owns
 *     (allocated by the caller, e.g. through PyTorch). The library never
 *     allocates, frees or synchronises, except sgpt_sync_status.
 *   - Matrices are row-major. X is bf16 passed as raw 16-bit patterns.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Every call
 *     only enqueues work on that stream.
 *   - `ws`/`ws_bytes` is caller-provided device scratch, at least
 *     sgpt_workspace_bytes() bytes, 256-byte aligned. It is not kept between
 *     calls.
 *   - Argument errors are reported synchronously as the return value, before
 *     anything is enqueued. Numeric errors found on the device (a matrix that
 *     is not positive definite, non-finite values, a bounded wait that ran out,
 *     a mask that breaks 2:4) are written to `*dev_info` (device int). Kernels
 *     record only the first error, and every kernel of a later call that sees
 *     a non-zero *dev_info returns without touching its outputs. Clear it with
 *     sgpt_info_clear, read it with sgpt_sync_status.
 *     dev_info values: 0 ok; k > 0 pivot k (1-based column of H) was not
 *     positive; SGPT_INFO_NONFINITE; SGPT_INFO_TIMEOUT; SGPT_INFO_BAD_MASK.
 *   - Size limits: 32 <= d_in <= 32768 and d_in % 32 == 0; 1 <= d_out <=
 *     16777216; ldw >= d_in and ldw % 4 == 0; every pointer 16-byte aligned.
 */
#ifndef SGPT_H_
#define SGPT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SGPT_ABI_VERSION 2

typedef enum sgpt_status {
  SGPT_OK = 0,
  SGPT_ERR_INVALID_ARG = 1, /* bad pointer, size, alignment or parameter   */
  SGPT_ERR_NOT_PD = 2,      /* damped H has a non-positive pivot           */
  SGPT_ERR_NONFINITE = 3,   /* NaN/Inf met in H, U or W                    */
  SGPT_ERR_TIMEOUT = 4,     /* a bounded device-side wait gave up          */
  SGPT_ERR_CUDA = 5,        /* a CUDA runtime call failed                  */
  SGPT_ERR_UNSUPPORTED = 6, /* valid request this library version does not implement */
  SGPT_ERR_BAD_MASK = 7,    /* pack: a group does not keep exactly n of m  */
  SGPT_ERR_WORKSPACE = 8    /* ws too small or misaligned                  */
} sgpt_status;

/* Non-pivot codes written to *dev_info. */
#define SGPT_INFO_NONFINITE (-1)
#define SGPT_INFO_TIMEOUT (-2)
#define SGPT_INFO_BAD_MASK (-3)

#define SGPT_PATTERN_UNSTRUCTURED 0
#define SGPT_PATTERN_NM 1

typedef struct sgpt_params {
  int pattern;    /* SGPT_PATTERN_UNSTRUCTURED or SGPT_PATTERN_NM            */
  int n, m;       /* N:M - keep n of every m consecutive inputs: m a power
                     of two from 4 to 128, 1 <= n <= m, blocksize % m == 0 and
                     d_in % m == 0 (SGPT_ERR_UNSUPPORTED for other m)        */
  float sparsity; /* unstructured - fraction pruned in each block, [0, 1)    */
  int blocksize;  /* columns per OBS block: 32, 64, 96 or 128; the interval
                     at which an unstructured mask is chosen on the weights
                     compensated so far (the lazy batch of the trailing
                     update is internal and changes only rounding order)    */
  float damp;     /* damping ratio (0.01 = 1% of the mean diagonal), >= 0    */
  int forced;     /* 1: mask_bits is an INPUT and no selection is made       */
  int qbits;      /* 0: prune only. 2..16: joint sparsification and
                     quantization (SparseGPT review, sections 十五 and 十七):
                     every kept weight is replaced by its value on its row's
                     grid of 2^qbits levels as its column is reached, and the
                     difference is compensated like a pruning error          */
  const float* qgrid; /* qbits > 0: the grid [d_out x 2] fp32 (scale, zero
                     point per row, device), e.g. from sgpt_quant_grid; NULL:
                     sgpt_prune computes it from the dense input W           */
} sgpt_params;

/* Human-readable name of a status. Never NULL. */
const char* sgpt_status_string(sgpt_status s);

/* SGPT_ABI_VERSION of the loaded library. */
int sgpt_abi_version(void);

/* Diagnostics: number of kernels this library has enqueued since it was
 * loaded (all devices, all streams). Memsets and copies are not counted. */
uint64_t sgpt_kernel_launches(void);

/* Failure-path testing and diagnostics (no counterpart in the pages): the
 * number of SM clock cycles a device-side wait on other threads or CTAs (a
 * tensor-core pipeline barrier, the selection's grid barrier) polls before
 * it gives up and records SGPT_INFO_TIMEOUT. cycles <= 0 restores the
 * default, 4e9 (about 2 s at the boost clock). Process-wide; read when a
 * kernel is enqueued (a captured graph keeps the value it was captured
 * with). A CTA that gave up still waits for its own copies and tensor-core
 * operations in flight under a fixed limit before it exits, so a tiny value
 * makes kernels report TIMEOUT and return, never leaves work behind. Returns
 * the previous value. */
int64_t sgpt_set_wait_limit(int64_t cycles);

/* Scratch bytes needed by any call below for these sizes (n_tok only matters
 * for the Hessian; pass 0 when H is given). */
size_t sgpt_workspace_bytes(int d_out, int d_in, int64_t n_tok, const sgpt_params* p);

/* *dev_info = 0, enqueued on `stream`. */
sgpt_status sgpt_info_clear(int* dev_info, void* stream);

/* Blocking: waits for `stream`, reads *dev_info and maps it to a status
 * (0 -> OK, k > 0 -> NOT_PD, other codes as named above). */
sgpt_status sgpt_sync_status(const int* dev_info, void* stream);

/* H += X^T X  (SparseGPT review, section 七: H = X X^T with X as channels x
 * tokens; here X is tokens x channels, so the same matrix is X^T X).
 *   H   [d_in x d_in] fp32, full symmetric matrix, updated in place; both
 *       triangles are written. Zero it first (sgpt_hessian_zero) to start a
 *       new accumulation; call repeatedly to stream token chunks.
 *   X   [n_tok x d_in] bf16 bit patterns, row-major, 16-byte aligned rows;
 *       may be NULL when n_tok == 0 (then nothing is launched and H is left
 *       as it is).
 * Products are exact in fp32; sums are fp32 (tensor cores, fixed order). */
sgpt_status sgpt_hessian_zero(float* H, int d_in, void* stream);
sgpt_status sgpt_hessian_accumulate(float* H, const uint16_t* X, int64_t n_tok, int d_in,
                                    void* ws, size_t ws_bytes, int* dev_info, void* stream);

/* H = X^T X: the same sums as sgpt_hessian_zero followed by
 * sgpt_hessian_accumulate, but H is only written (its old contents are never
 * read), which saves the zeroing and a read of H. Same arguments and errors
 * as sgpt_hessian_accumulate; n_tok == 0 gives H = 0. */
sgpt_status sgpt_hessian_compute(float* H, const uint16_t* X, int64_t n_tok, int d_in,
                                 void* ws, size_t ws_bytes, int* dev_info, void* stream);

/* U = upper Cholesky factor of H_d^-1, with H_d = (2/n_total) H + lambda I,
 * lambda = damp * mean(diag((2/n_total) H)); H_d^-1 = U^T U, U_ii > 0.
 *   H   [d_in x d_in] fp32, the accumulated X^T X; only the upper triangle
 *       (i <= j) is read. Not modified (unless U == H).
 *   U   [d_in x d_in] fp32 output; zeros below the diagonal. May alias H.
 * Errors on the device: pivot k not positive -> *dev_info = k (NOT_PD);
 * non-finite diagonal -> NONFINITE. U is then unspecified. */
sgpt_status sgpt_factor(const float* H, int64_t n_total, int d_in, float damp, float* U,
                        void* ws, size_t ws_bytes, int* dev_info, void* stream);

/* The blocked OBS sweep (SparseGPT review, sections 八 and 十一): for each
 * block of p->blocksize columns, select the mask (N:M at the first column of
 * each group of m, on the weights as compensated so far, keeping the n largest
 * w_c^2 / U_cc^2, ties to the lower column; or unstructured: exactly
 * floor(sparsity * d_out * width) of the block's smallest saliencies, ties by
 * row then column), then for each column q: e = (w_q - p_q) / U_qq, subtract
 * e * U[q, q:] from the rest of the block, and after the block subtract
 * Err * U[block, right of block] from every later column.
 *   W          [d_out x ldw] fp32, in: dense weights, out: pruned weights.
 *   U          from sgpt_factor (same d_in).
 *   mask_bits  [d_out x d_in/32] uint32, bit c%32 of word c/32 = 1 if kept;
 *              output, or input when p->forced.
 *   row_loss   [d_out] fp32 or NULL: sum over the row of e^2 (accumulated
 *              in place: zero it first).
 * The result of an N:M run does not depend on blocksize. */
sgpt_status sgpt_prune(float* W, int d_out, int d_in, int ldw, const float* U,
                       const sgpt_params* p, uint32_t* mask_bits, float* row_loss,
                       void* ws, size_t ws_bytes, int* dev_info, void* stream);

/* Allocation-free variant of sgpt_prune. No counterpart in the pages: it
 * exists for callers that cannot provide device memory at the call site -
 * for instance code running in a framework plugin or a real-time loop whose
 * execution path forbids allocation, or a process whose device memory is
 * wholly owned by another allocator - and so cannot pass the workspace
 * sgpt_prune needs. Same arguments, results and device-status behaviour as
 * sgpt_prune, minus ws/ws_bytes: the scratch (the d_out x 128 fp32 error
 * block and the selection state, about 4 MiB) lives in a fixed device array
 * inside the library, which every GPU that loads the library keeps until
 * the process exits. The library allocates nothing here.
 *   - d_out must not exceed SGPT_NOALLOC_MAX_ROWS (else SGPT_ERR_INVALID_ARG).
 *   - The first call on each device looks up that device's copy of the array
 *     (cudaGetSymbolAddress, with the device current); make that first call
 *     before any stream capture on the device.
 *   - All calls share the one array: calls that overlap on the GPU (other
 *     streams, other host threads) race and must be serialised by the
 *     caller. Nothing in the array needs clearing between calls.
 *   - With p->qbits > 0 the caller passes the grid in p->qgrid (the array
 *     has no room for it): SGPT_ERR_UNSUPPORTED when it is NULL. */
#define SGPT_NOALLOC_MAX_ROWS 8192
sgpt_status sgpt_prune_noalloc(float* W, int d_out, int d_in, int ldw, const float* U,
                               const sgpt_params* p, uint32_t* mask_bits, float* row_loss,
                               int* dev_info, void* stream);

/* The per-row quantization grid of the joint sparse + quantized sweep
 * (SparseGPT review, sections 十五 and 十七; the grid itself is this
 * library's reading: uniform and asymmetric, 2^qbits levels over the row's
 * range widened to include 0, so a pruned weight stays exactly 0):
 *   grid [d_out x 2] fp32: grid[2r] = scale = (hi - lo) / (2^qbits - 1),
 *        grid[2r + 1] = zero = rint(-lo / scale), with lo = min(row, 0) and
 *        hi = max(row, 0) of the dense row (a row of zeros: lo = -1, hi = 1),
 *        all in fp32. A weight x maps to scale * (clip(rint(x / scale) +
 *        zero, 0, 2^qbits - 1) - zero); the integer code of a kept weight of
 *        the result is rint(W / scale) + zero exactly.
 * qbits in 2..16. Call it on the dense W before sgpt_prune (or leave
 * qgrid NULL and sgpt_prune computes the same grid). */
sgpt_status sgpt_quant_grid(const float* W, int d_out, int d_in, int ldw, int qbits, float* grid, void* stream);

/* 2:4 packing (2:4 production guide, section on the 2:4 mechanism):
 *   values [d_out x d_in/2] fp32: the two kept weights of each group of four,
 *          in column order;
 *   meta   [d_out x d_in/32] uint32: group g of a row is the 4-bit code
 *          a | (b << 2) (a < b kept positions) in bits [4(g%8), 4(g%8)+4) of
 *          word g/8.
 * A group whose mask does not keep exactly two sets *dev_info = BAD_MASK. */
sgpt_status sgpt_pack24(const float* W, int d_out, int d_in, int ldw, const uint32_t* mask_bits,
                        float* values, uint32_t* meta, int* dev_info, void* stream);

/* N:M packing (sparse fine-tuning review, section 八 8.4: keep N of every M
 * weights and record the kept positions; the 2:4 guide's 2-bit positions
 * generalised to log2(M) bits):
 *   values [d_out x d_in*n/m] fp32: the n kept weights of each group of m,
 *          in column order (value g*n + j of a row is the j-th kept weight
 *          of group g);
 *   meta   [d_out x sgpt_pack_nm_meta_words(d_in, n, m)] uint32: the
 *          in-group position of value k of a row takes log2(m) bits at bit
 *          offset k*log2(m) of the row's bit string, which fills the row's
 *          words least significant bit first (a position may continue into
 *          the next word). For 2:4 the words equal sgpt_pack24's.
 * m a power of two from 4 to 128 (else SGPT_ERR_UNSUPPORTED), 1 <= n <= m,
 * d_in % m == 0. A group whose mask does not keep exactly n sets
 * *dev_info = BAD_MASK. */
sgpt_status sgpt_pack_nm(const float* W, int d_out, int d_in, int ldw, const uint32_t* mask_bits, int n, int m,
                         float* values, uint32_t* meta, int* dev_info, void* stream);

/* Metadata words per row of sgpt_pack_nm: ceil(d_in/m * n * log2(m) / 32),
 * or -1 for arguments sgpt_pack_nm rejects. */
int sgpt_pack_nm_meta_words(int d_in, int n, int m);

/* Layer reconstruction error (SparseGPT review, section 六, the objective):
 * num_den[0] = tr(dW H dW^T), num_den[1] = tr(W0 H W0^T), dW = W0 - W, in
 * fp64 on the device (FP32 products, fp64 sums in a fixed order: the result
 * is the same to the last bit on every call). H is the full symmetric
 * matrix (undamped; any positive scale). Both W0 and W use leading
 * dimension ldw. ws: at least sgpt_workspace_bytes(d_out, d_in, 0, p)
 * bytes (SGPT_ERR_WORKSPACE otherwise). */
sgpt_status sgpt_recon_error(const float* W0, const float* W, int d_out, int d_in, int ldw,
                             const float* H, double* num_den, void* ws, size_t ws_bytes,
                             void* stream);

/* One layer end to end: if X != NULL, H = X^T X over its n_tok rows, else H
 * must already hold that sum; then U = sgpt_factor(H), sgpt_prune, and for
 * N:M sgpt_pack_nm (values/meta sized as sgpt_pack_nm states; NULL to skip
 * packing). U and H must not alias. *dev_info is cleared first. Every
 * argument is checked before the first launch. */
sgpt_status sgpt_prune_layer(float* W, int d_out, int d_in, int ldw, const uint16_t* X,
                             int64_t n_tok, float* H, float* U, const sgpt_params* p,
                             uint32_t* mask_bits, float* values, uint32_t* meta,
                             float* row_loss, void* ws, size_t ws_bytes, int* dev_info,
                             void* stream);

/* ------------------------------------------------------------------------
 * Multi-layer driver. The layer-wise procedure of the SparseGPT review,
 * section 九 (collect the current layer's inputs, form its Hessian, prune
 * and compensate, pass the pruned output to the next layer; section 十一,
 * steps three to six), on one synthetic MLP block of a decoder:
 *   x -> x' = x + W_down (silu(W_gate x) * (W_up x)),
 * x [n_tok x hidden] and z = silu(W_gate x) * (W_up x) [n_tok x inter] bf16,
 * the three products on the tensor cores in bf16 (the weights rounded to
 * bf16) with fp32 accumulation, every rounding to bf16 to nearest even.
 *   SGPT_DRIVER_SEQUENTIAL: gate and up are pruned from x (one Hessian and
 *     factor), z is formed with the PRUNED gate and up, down is pruned from
 *     z, and x' is the pruned block's output.
 *   SGPT_DRIVER_PARALLEL (V-SparseGPT press release, voc.com.cn: the inputs
 *     of every layer of the original model are recorded first, so layers are
 *     sparsified side by side): z and x' come from the DENSE block; gate and
 *     up are pruned from x and down from the recorded z, the down input's
 *     Hessian on a second stream beside gate and up.
 * blk: the three weight matrices (fp32, row-major, in: dense, out: pruned;
 *   W_gate, W_up [inter x hidden], W_down [hidden x inter]) and their masks
 *   ([inter x hidden/32], [hidden x inter/32]).
 * X_next [n_tok x hidden] bf16 out; Z [n_tok x inter] bf16 out (the down
 *   projection's input), or NULL to keep it in ws.
 * p: pattern, block size, damping and qbits as for sgpt_prune (one grid per
 *   matrix from its dense weights); p->forced and p->qgrid must be 0/NULL.
 * ws: sgpt_mlp_block_workspace_bytes(hidden, inter, n_tok) bytes.
 * *dev_info is cleared first; numeric errors as elsewhere. Stacked blocks
 * are pruned by calling this once per block with X = the previous X_next. */
#define SGPT_DRIVER_SEQUENTIAL 0
#define SGPT_DRIVER_PARALLEL 1

typedef struct sgpt_mlp_block {
  float* W_gate;
  float* W_up;
  float* W_down;
  uint32_t* mask_gate;
  uint32_t* mask_up;
  uint32_t* mask_down;
} sgpt_mlp_block;

size_t sgpt_mlp_block_workspace_bytes(int hidden, int inter, int64_t n_tok);
sgpt_status sgpt_prune_mlp_block(const sgpt_mlp_block* blk, int hidden, int inter, const uint16_t* X, int64_t n_tok,
                                 int mode, const sgpt_params* p, uint16_t* X_next, uint16_t* Z, void* ws,
                                 size_t ws_bytes, int* dev_info, void* stream);

/* The forward product of the driver: Y [n x d_out] fp32 = X [n x d_in] bf16
 * times Wb^T, Wb [d_out x d_in] bf16, on the tensor cores
 * (tcgen05.mma.kind::f16, fp32 accumulation in sums of at most 128 of K).
 * d_in and d_out multiples of 32; 1 <= n < 2^31. */
sgpt_status sgpt_linear_bf16(const uint16_t* X, const uint16_t* Wb, int64_t n, int d_in, int d_out, float* Y,
                             int* dev_info, void* stream);

/* A consumer of the 2:4 output (2:4 production guide, section on the 2:4
 * mechanism: two kept weights of every four along the reduction axis and
 * their 2-bit positions): Y [n x d_out] fp32 = X W^T, where W [d_out x d_in]
 * is given ONLY in packed form,
 *   values     [d_out x d_in/2] bf16 (e.g. sgpt_pack24's values through
 *              sgpt_to_bf16),
 *   meta_tiles sgpt_pack24's metadata words re-arranged once per weight
 *              matrix by sgpt_sparse24_tile_meta,
 * and X [n x d_in] bf16. Runs on the sparse tensor cores
 * (tcgen05.mma.sp.kind::f16, fp32 accumulation in one sum over all of K).
 * d_in % 32 == 0; 1 <= n < 2^31. All pointers device, 16-byte aligned; Y is
 * written, nothing else. A bounded wait that runs out sets
 * SGPT_INFO_TIMEOUT in *dev_info.
 *
 * meta_tiles: sgpt_sparse24_meta_tiles_bytes(d_out, d_in) bytes (0 = bad
 * sizes), caller-owned. The layout is the order in which the sparse tensor
 * cores read the metadata from tensor memory, in 4 KB pieces per 256 rows
 * and 128 columns of K (each 4-bit group code unchanged; rows and columns
 * past the matrix hold a valid padding code). sgpt_sparse24_tile_meta
 * reads meta [d_out x d_in/32] uint32 (sgpt_pack24's words) and writes
 * meta_tiles on `stream`; its result is opaque and reusable for every
 * product with the same weights. */
size_t sgpt_sparse24_meta_tiles_bytes(int d_out, int d_in);
sgpt_status sgpt_sparse24_tile_meta(const uint32_t* meta, int d_out, int d_in, uint32_t* meta_tiles, void* stream);
sgpt_status sgpt_sparse24_linear(const uint16_t* values, const uint32_t* meta_tiles, int d_out, int d_in,
                                 const uint16_t* X, int64_t n, float* Y, int* dev_info, void* stream);

/* Wb = W rounded to bf16 (to nearest even), rows x cols, W leading
 * dimension ldw; Wb dense [rows x cols]. */
sgpt_status sgpt_to_bf16(const float* W, int rows, int cols, int ldw, uint16_t* Wb, int* dev_info, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SGPT_H_ */
