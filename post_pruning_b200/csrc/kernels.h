// Internal launchers behind the C ABI (host side, one translation unit each).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <algorithm>

#include "../../include/sgpt.h"

namespace sgpt {

// factor.cu
size_t factor_ws_bytes(int d);
cudaError_t launch_factor(const float* H, long long n_total, int d, float damp, float* U, void* ws,
                          int* info, cudaStream_t st);

// sweep.cu
size_t prune_ws_bytes(int d_out, int d_in);
cudaError_t launch_prune(float* W, int rows, int d, long long ldw, const float* U,
                         const sgpt_params& p, uint32_t* mask, float* row_loss, void* ws,
                         int* info, cudaStream_t st);
cudaError_t launch_quant_grid(const float* W, long long ldw, int rows, int d, int bits, float* grid,
                              cudaStream_t st);
cudaError_t launch_prune_noalloc(float* W, int rows, int d, long long ldw, const float* U,
                                 const sgpt_params& p, uint32_t* mask, float* row_loss, int* info,
                                 cudaStream_t st);

// pack.cu
cudaError_t launch_pack24(const float* W, long long ldw, int rows, int d, const uint32_t* mask,
                          float* values, uint32_t* meta, int* info, cudaStream_t st);
int packnm_meta_words(int d, int n, int m);
cudaError_t launch_packnm(const float* W, long long ldw, int rows, int d, const uint32_t* mask, int n, int m,
                          float* values, uint32_t* meta, int* info, cudaStream_t st);
size_t recon_ws_bytes(int rows, int d);
cudaError_t launch_recon(const float* W0, const float* W, int rows, int d, long long ldw,
                         const float* H, double* num_den, void* ws, cudaStream_t st);

// driver.cu
cudaError_t launch_to_bf16(const float* W, long long ld, long long rows, int cols, uint16_t* Wb, const int* info,
                           cudaStream_t st);
cudaError_t launch_linear_bf16(const uint16_t* X, const uint16_t* Wb, long long n, int d_in, int d_out, float* Y,
                               int* info, cudaStream_t st);
size_t mlp_block_ws_bytes(int h, int f, long long n);
cudaError_t launch_prune_mlp_block(const sgpt_mlp_block& blk, int h, int f, const uint16_t* X, long long n,
                                   int mode, const sgpt_params& p, uint16_t* X_next, uint16_t* Z, void* ws,
                                   int* info, cudaStream_t st);

// consumer.cu
size_t sparse24_meta_tiles_bytes(int rows, int d);
cudaError_t launch_tile_meta(const uint32_t* meta, int rows, int d, uint32_t* tiles, cudaStream_t st);
cudaError_t launch_sparse24_gemm(const uint16_t* values_bf16, const uint32_t* tiles, int rows, int d,
                                 const uint16_t* X, long long n, float* Y, int* info, cudaStream_t st);

// hessian_tc.cu
size_t hessian_ws_bytes(int d, long long n);
cudaError_t launch_hessian_tc(float* H, const uint16_t* X, long long n, int d, void* ws, int* info,
                              cudaStream_t st, bool set);

}  // namespace sgpt
