// C ABI of the solver: argument checks, workspace carving and launch order.
// Nothing here computes; every step runs in the kernels of the other files.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>

#include "../../include/sgpt.h"
#include "common.cuh"
#include "kernels.h"

#include <atomic>

namespace sgpt {
static std::atomic<unsigned long long> g_launches{0};
void count_launches(unsigned long long n) { g_launches.fetch_add(n, std::memory_order_relaxed); }
static std::atomic<long long> g_wait_cycles{kDefaultWaitCycles};
long long wait_limit_cycles() { return g_wait_cycles.load(std::memory_order_relaxed); }
}  // namespace sgpt

namespace {

using namespace sgpt;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

bool valid_din(int d_in) { return d_in >= 32 && d_in <= 32768 && d_in % 32 == 0; }
bool valid_dout(int d_out) { return d_out >= 1 && d_out <= (1 << 24); }

sgpt_status from_cuda(cudaError_t e) { return e == cudaSuccess ? SGPT_OK : SGPT_ERR_CUDA; }

// Group sizes the N:M sweep and pack support: powers of two from 4 to 128.
bool valid_m(int m) { return m >= 4 && m <= 128 && (m & (m - 1)) == 0; }

sgpt_status check_params(const sgpt_params* p) {
  if (!p) return SGPT_ERR_INVALID_ARG;
  if (p->blocksize < 32 || p->blocksize > kMaxBlock || p->blocksize % 32) return SGPT_ERR_INVALID_ARG;
  if (!(p->damp >= 0.f) || !std::isfinite(p->damp)) return SGPT_ERR_INVALID_ARG;
  if (p->forced != 0 && p->forced != 1) return SGPT_ERR_INVALID_ARG;
  if (p->qbits != 0 && (p->qbits < 2 || p->qbits > 16)) return SGPT_ERR_INVALID_ARG;
  if (p->qbits && p->qgrid && !aligned16(p->qgrid)) return SGPT_ERR_INVALID_ARG;
  if (p->pattern == SGPT_PATTERN_NM) {
    if (p->n <= 0 || p->m <= 0 || p->n > p->m) return SGPT_ERR_INVALID_ARG;
    if (!valid_m(p->m)) return SGPT_ERR_UNSUPPORTED;
    if (p->blocksize % p->m) return SGPT_ERR_INVALID_ARG;
  } else if (p->pattern == SGPT_PATTERN_UNSTRUCTURED) {
    if (!(p->sparsity >= 0.f && p->sparsity < 1.f)) return SGPT_ERR_INVALID_ARG;
  } else {
    return SGPT_ERR_INVALID_ARG;
  }
  return SGPT_OK;
}

sgpt_status check_ws(void* ws, size_t have, size_t need) {
  if (need == 0) return SGPT_OK;
  if (!ws || !aligned256(ws) || have < need) return SGPT_ERR_WORKSPACE;
  return SGPT_OK;
}

}  // namespace

extern "C" {

const char* sgpt_status_string(sgpt_status s) {
  switch (s) {
    case SGPT_OK: return "ok";
    case SGPT_ERR_INVALID_ARG: return "invalid argument";
    case SGPT_ERR_NOT_PD: return "damped Hessian is not positive definite";
    case SGPT_ERR_NONFINITE: return "non-finite value";
    case SGPT_ERR_TIMEOUT: return "device-side wait timed out";
    case SGPT_ERR_CUDA: return "CUDA runtime error";
    case SGPT_ERR_UNSUPPORTED: return "not supported by this library version";
    case SGPT_ERR_BAD_MASK: return "mask breaks the 2:4 pattern";
    case SGPT_ERR_WORKSPACE: return "workspace too small or misaligned";
  }
  return "unknown status";
}

int sgpt_abi_version(void) { return SGPT_ABI_VERSION; }

uint64_t sgpt_kernel_launches(void) { return sgpt::g_launches.load(std::memory_order_relaxed); }

int64_t sgpt_set_wait_limit(int64_t cycles) {
  const long long v = cycles > 0 ? (long long)cycles : kDefaultWaitCycles;
  return (int64_t)sgpt::g_wait_cycles.exchange(v, std::memory_order_relaxed);
}

size_t sgpt_workspace_bytes(int d_out, int d_in, int64_t n_tok, const sgpt_params* p) {
  (void)p;
  if (!valid_din(d_in) || !valid_dout(d_out) || n_tok < 0) return 0;
  size_t need = std::max({factor_ws_bytes(d_in), prune_ws_bytes(d_out, d_in), recon_ws_bytes(d_out, d_in)});
  if (n_tok > 0) need = std::max(need, hessian_ws_bytes(d_in, n_tok));
  return need;
}

sgpt_status sgpt_info_clear(int* dev_info, void* stream) {
  if (!dev_info) return SGPT_ERR_INVALID_ARG;
  return from_cuda(cudaMemsetAsync(dev_info, 0, sizeof(int), as_stream(stream)));
}

sgpt_status sgpt_sync_status(const int* dev_info, void* stream) {
  if (!dev_info) return SGPT_ERR_INVALID_ARG;
  int h = 0;
  if (cudaMemcpyAsync(&h, dev_info, sizeof(int), cudaMemcpyDeviceToHost, as_stream(stream)) != cudaSuccess)
    return SGPT_ERR_CUDA;
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return SGPT_ERR_CUDA;
  if (h == 0) return SGPT_OK;
  if (h > 0) return SGPT_ERR_NOT_PD;
  if (h == SGPT_INFO_NONFINITE) return SGPT_ERR_NONFINITE;
  if (h == SGPT_INFO_TIMEOUT) return SGPT_ERR_TIMEOUT;
  if (h == SGPT_INFO_BAD_MASK) return SGPT_ERR_BAD_MASK;
  return SGPT_ERR_CUDA;
}

sgpt_status sgpt_hessian_zero(float* H, int d_in, void* stream) {
  if (!H || !aligned16(H) || !valid_din(d_in)) return SGPT_ERR_INVALID_ARG;
  return from_cuda(cudaMemsetAsync(H, 0, (size_t)d_in * d_in * sizeof(float), as_stream(stream)));
}

namespace {
sgpt_status hessian(float* H, const uint16_t* X, int64_t n_tok, int d_in, void* ws, size_t ws_bytes, int* dev_info,
                    void* stream, bool set) {
  // X may be NULL when there are no tokens
  if (!H || !aligned16(H) || !valid_din(d_in) || n_tok < 0 || !dev_info) return SGPT_ERR_INVALID_ARG;
  if (n_tok > 0 && (!X || !aligned16(X))) return SGPT_ERR_INVALID_ARG;
  if (n_tok > (int64_t)INT32_MAX) return SGPT_ERR_INVALID_ARG;   // TMA coordinates are 32-bit
  if (n_tok == 0) return set ? sgpt_hessian_zero(H, d_in, stream) : SGPT_OK;
  sgpt_status s = check_ws(ws, ws_bytes, hessian_ws_bytes(d_in, n_tok));
  if (s != SGPT_OK) return s;
  cudaError_t e = launch_hessian_tc(H, X, n_tok, d_in, ws, dev_info, as_stream(stream), set);
  if (e == cudaErrorNotSupported) return SGPT_ERR_UNSUPPORTED;
  return from_cuda(e);
}
}  // namespace

sgpt_status sgpt_hessian_accumulate(float* H, const uint16_t* X, int64_t n_tok, int d_in, void* ws,
                                    size_t ws_bytes, int* dev_info, void* stream) {
  return hessian(H, X, n_tok, d_in, ws, ws_bytes, dev_info, stream, false);
}

sgpt_status sgpt_hessian_compute(float* H, const uint16_t* X, int64_t n_tok, int d_in, void* ws,
                                 size_t ws_bytes, int* dev_info, void* stream) {
  return hessian(H, X, n_tok, d_in, ws, ws_bytes, dev_info, stream, true);
}

sgpt_status sgpt_factor(const float* H, int64_t n_total, int d_in, float damp, float* U, void* ws,
                        size_t ws_bytes, int* dev_info, void* stream) {
  if (!H || !U || !dev_info || !aligned16(H) || !aligned16(U) || !valid_din(d_in) || n_total <= 0)
    return SGPT_ERR_INVALID_ARG;
  if (!(damp >= 0.f) || !std::isfinite(damp)) return SGPT_ERR_INVALID_ARG;
  sgpt_status s = check_ws(ws, ws_bytes, factor_ws_bytes(d_in));
  if (s != SGPT_OK) return s;
  return from_cuda(launch_factor(H, n_total, d_in, damp, U, ws, dev_info, as_stream(stream)));
}

sgpt_status sgpt_prune(float* W, int d_out, int d_in, int ldw, const float* U, const sgpt_params* p,
                       uint32_t* mask_bits, float* row_loss, void* ws, size_t ws_bytes, int* dev_info,
                       void* stream) {
  if (!W || !U || !mask_bits || !dev_info || !aligned16(W) || !aligned16(U) || !aligned16(mask_bits))
    return SGPT_ERR_INVALID_ARG;
  if (!valid_din(d_in) || !valid_dout(d_out) || ldw < d_in || ldw % 4) return SGPT_ERR_INVALID_ARG;
  if (row_loss && !aligned16(row_loss)) return SGPT_ERR_INVALID_ARG;
  sgpt_status s = check_params(p);
  if (s != SGPT_OK) return s;
  if (p->pattern == SGPT_PATTERN_NM && d_in % p->m) return SGPT_ERR_INVALID_ARG;
  s = check_ws(ws, ws_bytes, prune_ws_bytes(d_out, d_in));
  if (s != SGPT_OK) return s;
  return from_cuda(launch_prune(W, d_out, d_in, ldw, U, *p, mask_bits, row_loss, ws, dev_info,
                                as_stream(stream)));
}

sgpt_status sgpt_prune_noalloc(float* W, int d_out, int d_in, int ldw, const float* U, const sgpt_params* p,
                               uint32_t* mask_bits, float* row_loss, int* dev_info, void* stream) {
  if (!W || !U || !mask_bits || !dev_info || !aligned16(W) || !aligned16(U) || !aligned16(mask_bits))
    return SGPT_ERR_INVALID_ARG;
  if (!valid_din(d_in) || !valid_dout(d_out) || ldw < d_in || ldw % 4) return SGPT_ERR_INVALID_ARG;
  if (d_out > SGPT_NOALLOC_MAX_ROWS) return SGPT_ERR_INVALID_ARG;
  if (row_loss && !aligned16(row_loss)) return SGPT_ERR_INVALID_ARG;
  sgpt_status s = check_params(p);
  if (s != SGPT_OK) return s;
  if (p->qbits && !p->qgrid) return SGPT_ERR_UNSUPPORTED;
  if (p->pattern == SGPT_PATTERN_NM && d_in % p->m) return SGPT_ERR_INVALID_ARG;
  return from_cuda(launch_prune_noalloc(W, d_out, d_in, ldw, U, *p, mask_bits, row_loss, dev_info,
                                        as_stream(stream)));
}

sgpt_status sgpt_pack24(const float* W, int d_out, int d_in, int ldw, const uint32_t* mask_bits,
                        float* values, uint32_t* meta, int* dev_info, void* stream) {
  if (!W || !mask_bits || !values || !meta || !dev_info) return SGPT_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(values) || !aligned16(mask_bits) || !aligned16(meta))
    return SGPT_ERR_INVALID_ARG;
  if (!valid_din(d_in) || !valid_dout(d_out) || ldw < d_in || ldw % 4) return SGPT_ERR_INVALID_ARG;
  return from_cuda(launch_pack24(W, ldw, d_out, d_in, mask_bits, values, meta, dev_info, as_stream(stream)));
}

sgpt_status sgpt_quant_grid(const float* W, int d_out, int d_in, int ldw, int qbits, float* grid, void* stream) {
  if (!W || !grid || !aligned16(W) || !aligned16(grid)) return SGPT_ERR_INVALID_ARG;
  if (!valid_din(d_in) || !valid_dout(d_out) || ldw < d_in || ldw % 4) return SGPT_ERR_INVALID_ARG;
  if (qbits < 2 || qbits > 16) return SGPT_ERR_INVALID_ARG;
  return from_cuda(launch_quant_grid(W, ldw, d_out, d_in, qbits, grid, as_stream(stream)));
}

sgpt_status sgpt_to_bf16(const float* W, int rows, int cols, int ldw, uint16_t* Wb, int* dev_info, void* stream) {
  if (!W || !Wb || !aligned16(W) || (reinterpret_cast<uintptr_t>(Wb) & 7u)) return SGPT_ERR_INVALID_ARG;
  if (rows < 1 || cols < 4 || cols % 4 || ldw < cols || ldw % 4) return SGPT_ERR_INVALID_ARG;
  return from_cuda(launch_to_bf16(W, ldw, rows, cols, Wb, dev_info, as_stream(stream)));
}

sgpt_status sgpt_linear_bf16(const uint16_t* X, const uint16_t* Wb, int64_t n, int d_in, int d_out, float* Y,
                             int* dev_info, void* stream) {
  if (!X || !Wb || !Y || !dev_info || !aligned16(X) || !aligned16(Wb) || !aligned16(Y)) return SGPT_ERR_INVALID_ARG;
  if (n < 1 || n > (int64_t)INT32_MAX || !valid_din(d_in) || !valid_din(d_out)) return SGPT_ERR_INVALID_ARG;
  return from_cuda(launch_linear_bf16(X, Wb, n, d_in, d_out, Y, dev_info, as_stream(stream)));
}

size_t sgpt_sparse24_meta_tiles_bytes(int d_out, int d_in) {
  if (!valid_din(d_in) || !valid_dout(d_out)) return 0;
  return sparse24_meta_tiles_bytes(d_out, d_in);
}

sgpt_status sgpt_sparse24_tile_meta(const uint32_t* meta, int d_out, int d_in, uint32_t* meta_tiles, void* stream) {
  if (!meta || !meta_tiles || !aligned16(meta_tiles)) return SGPT_ERR_INVALID_ARG;
  if (!valid_din(d_in) || !valid_dout(d_out)) return SGPT_ERR_INVALID_ARG;
  return from_cuda(launch_tile_meta(meta, d_out, d_in, meta_tiles, as_stream(stream)));
}

sgpt_status sgpt_sparse24_linear(const uint16_t* values, const uint32_t* meta_tiles, int d_out, int d_in,
                                 const uint16_t* X, int64_t n, float* Y, int* dev_info, void* stream) {
  if (!values || !meta_tiles || !X || !Y || !dev_info) return SGPT_ERR_INVALID_ARG;
  if (!aligned16(values) || !aligned16(meta_tiles) || !aligned16(X) || !aligned16(Y)) return SGPT_ERR_INVALID_ARG;
  if (!valid_din(d_in) || !valid_dout(d_out) || n < 1 || n > (int64_t)INT32_MAX) return SGPT_ERR_INVALID_ARG;
  return from_cuda(launch_sparse24_gemm(values, meta_tiles, d_out, d_in, X, n, Y, dev_info, as_stream(stream)));
}

size_t sgpt_mlp_block_workspace_bytes(int hidden, int inter, int64_t n_tok) {
  if (!valid_din(hidden) || !valid_din(inter) || n_tok < 1 || n_tok > (int64_t)INT32_MAX) return 0;
  return mlp_block_ws_bytes(hidden, inter, n_tok);
}

sgpt_status sgpt_prune_mlp_block(const sgpt_mlp_block* blk, int hidden, int inter, const uint16_t* X, int64_t n_tok,
                                 int mode, const sgpt_params* p, uint16_t* X_next, uint16_t* Z, void* ws,
                                 size_t ws_bytes, int* dev_info, void* stream) {
  if (!blk || !X || !X_next || !dev_info) return SGPT_ERR_INVALID_ARG;
  if (!blk->W_gate || !blk->W_up || !blk->W_down || !blk->mask_gate || !blk->mask_up || !blk->mask_down)
    return SGPT_ERR_INVALID_ARG;
  const void* ptrs[] = {blk->W_gate, blk->W_up, blk->W_down, blk->mask_gate, blk->mask_up, blk->mask_down, X, X_next};
  for (const void* q : ptrs)
    if (!aligned16(q)) return SGPT_ERR_INVALID_ARG;
  if (Z && !aligned16(Z)) return SGPT_ERR_INVALID_ARG;
  if (!valid_din(hidden) || !valid_din(inter) || n_tok < 1 || n_tok > (int64_t)INT32_MAX) return SGPT_ERR_INVALID_ARG;
  if (mode != SGPT_DRIVER_SEQUENTIAL && mode != SGPT_DRIVER_PARALLEL) return SGPT_ERR_INVALID_ARG;
  sgpt_status s = check_params(p);
  if (s != SGPT_OK) return s;
  if (p->forced || p->qgrid) return SGPT_ERR_INVALID_ARG;     // each layer decides its own mask and grid
  if (p->pattern == SGPT_PATTERN_NM && (hidden % p->m || inter % p->m)) return SGPT_ERR_INVALID_ARG;
  s = check_ws(ws, ws_bytes, mlp_block_ws_bytes(hidden, inter, n_tok));
  if (s != SGPT_OK) return s;
  if ((s = sgpt_info_clear(dev_info, stream)) != SGPT_OK) return s;
  return from_cuda(launch_prune_mlp_block(*blk, hidden, inter, X, n_tok, mode, *p, X_next, Z, ws, dev_info,
                                          as_stream(stream)));
}

int sgpt_pack_nm_meta_words(int d_in, int n, int m) {
  if (!valid_din(d_in) || !valid_m(m) || n < 1 || n > m || d_in % m) return -1;
  return packnm_meta_words(d_in, n, m);
}

sgpt_status sgpt_pack_nm(const float* W, int d_out, int d_in, int ldw, const uint32_t* mask_bits, int n, int m,
                         float* values, uint32_t* meta, int* dev_info, void* stream) {
  if (!W || !mask_bits || !values || !meta || !dev_info) return SGPT_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(values) || !aligned16(mask_bits) || !aligned16(meta))
    return SGPT_ERR_INVALID_ARG;
  if (!valid_din(d_in) || !valid_dout(d_out) || ldw < d_in || ldw % 4) return SGPT_ERR_INVALID_ARG;
  if (n < 1 || n > m || m < 1) return SGPT_ERR_INVALID_ARG;
  if (!valid_m(m)) return SGPT_ERR_UNSUPPORTED;
  if (d_in % m) return SGPT_ERR_INVALID_ARG;
  if (n == 2 && m == 4)      // the same words, by the 2:4 kernel
    return from_cuda(launch_pack24(W, ldw, d_out, d_in, mask_bits, values, meta, dev_info, as_stream(stream)));
  return from_cuda(launch_packnm(W, ldw, d_out, d_in, mask_bits, n, m, values, meta, dev_info, as_stream(stream)));
}

sgpt_status sgpt_recon_error(const float* W0, const float* W, int d_out, int d_in, int ldw, const float* H,
                             double* num_den, void* ws, size_t ws_bytes, void* stream) {
  if (!W0 || !W || !H || !num_den) return SGPT_ERR_INVALID_ARG;
  if (!aligned16(W0) || !aligned16(W) || !aligned16(H) || (reinterpret_cast<uintptr_t>(num_den) & 7u))
    return SGPT_ERR_INVALID_ARG;
  if (!valid_din(d_in) || !valid_dout(d_out) || ldw < d_in || ldw % 4) return SGPT_ERR_INVALID_ARG;
  const sgpt_status s = check_ws(ws, ws_bytes, recon_ws_bytes(d_out, d_in));
  if (s != SGPT_OK) return s;
  return from_cuda(launch_recon(W0, W, d_out, d_in, ldw, H, num_den, ws, as_stream(stream)));
}

sgpt_status sgpt_prune_layer(float* W, int d_out, int d_in, int ldw, const uint16_t* X, int64_t n_tok,
                             float* H, float* U, const sgpt_params* p, uint32_t* mask_bits, float* values,
                             uint32_t* meta, float* row_loss, void* ws, size_t ws_bytes, int* dev_info,
                             void* stream) {
  // every argument of every step is checked here, before the first launch,
  // so a bad one never leaves H or U half overwritten
  if (!H || !U || H == U || n_tok <= 0 || !dev_info) return SGPT_ERR_INVALID_ARG;
  if (!W || !mask_bits || !aligned16(W) || !aligned16(mask_bits) || !aligned16(H) || !aligned16(U))
    return SGPT_ERR_INVALID_ARG;
  if (X && (!aligned16(X) || n_tok > (int64_t)INT32_MAX)) return SGPT_ERR_INVALID_ARG;
  if (row_loss && !aligned16(row_loss)) return SGPT_ERR_INVALID_ARG;
  sgpt_status s = check_params(p);
  if (s != SGPT_OK) return s;
  if (!valid_din(d_in) || !valid_dout(d_out) || ldw < d_in || ldw % 4) return SGPT_ERR_INVALID_ARG;
  s = check_ws(ws, ws_bytes, sgpt_workspace_bytes(d_out, d_in, X ? n_tok : 0, p));
  if (s != SGPT_OK) return s;
  if (p->pattern == SGPT_PATTERN_NM && d_in % p->m) return SGPT_ERR_INVALID_ARG;
  const bool pack = p->pattern == SGPT_PATTERN_NM && values && meta;
  if ((values || meta) && !pack) return SGPT_ERR_INVALID_ARG;
  if (pack && (!aligned16(values) || !aligned16(meta))) return SGPT_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  if ((s = sgpt_info_clear(dev_info, stream)) != SGPT_OK) return s;
  if (X && (s = sgpt_hessian_compute(H, X, n_tok, d_in, ws, ws_bytes, dev_info, stream)) != SGPT_OK) return s;
  if ((s = sgpt_factor(H, n_tok, d_in, p->damp, U, ws, ws_bytes, dev_info, stream)) != SGPT_OK) return s;
  if (row_loss && cudaMemsetAsync(row_loss, 0, (size_t)d_out * sizeof(float), st) != cudaSuccess)
    return SGPT_ERR_CUDA;
  if ((s = sgpt_prune(W, d_out, d_in, ldw, U, p, mask_bits, row_loss, ws, ws_bytes, dev_info, stream)) != SGPT_OK)
    return s;
  if (pack) s = sgpt_pack_nm(W, d_out, d_in, ldw, mask_bits, p->n, p->m, values, meta, dev_info, stream);
  return s;
}

}  // extern "C"
