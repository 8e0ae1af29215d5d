// FP32-accurate tensor-core products (three TF32 products per K step), see
// gemm_tc.cu. Host-side interface used by the factorisation and the sweep.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace sgpt {
namespace tc {

// One fp32 operand as hi/lo planes, both row-major rows x cols with leading
// dimension ld (ld % 4 == 0, 16-byte aligned bases).
struct Operand {
  const float* hi;
  const float* lo;
  long long rows, cols, ld;
};

// What one launch computes; tile sizes are 128 x 128.
//  mode 0: dense grid of mt x nt tiles, K = kdim.
//  mode 1: tiles (i, j), i <= j, enumerated column by column from tile t0, K = kdim.
// A(m, k) is read at (x = a_x0 + k, y = a_y0 + m0 + m); B(k, n) at
// (x = b_x0 + k, y = b_y0 + n0 + n) if K-major, (x = b_x0 + n0 + n, y = b_y0 + k)
// if MN-major. C(m, n) = alpha * acc + beta * C at
// C[(c_row0 + m0 + m) * ldc + c_col0 + n0 + n] for m0+m < Mlim, n0+n < Nlim
// (C may be null: no fp32 result). C_hi/C_lo (optional) receive the hi/lo
// planes of the result at [(c_row0 + m0 + m - p_row0) * ldp + c_col0 + n0 + n
// - p_col0] (ldp = 0: ldc), from every tile or only from the tiles whose
// n0 == planes_n0 (planes_one_col) and whose m0 == planes_m0 (planes_one_row).
struct Job {
  int mode;
  int mt, nt;
  int t0;
  int kdim;
  int a_x0, a_y0, b_x0, b_y0;
  float* C;
  long long ldc;
  int c_row0, c_col0, Mlim, Nlim;
  float alpha, beta;
  float* C_hi;
  float* C_lo;
  long long ldp;
  int p_row0, p_col0;
  int planes_one_col, planes_n0;
  int planes_one_row, planes_m0;
  int max_ctas;      // persistent CTAs at most (0: one per SM)
};

// A bf16 operand: row-major rows x cols, leading dimension ld (ld % 8 == 0,
// 16-byte aligned base); K-major, i.e. K is the column index.
struct OperandBf16 {
  const uint16_t* p;
  long long rows, cols, ld;
};

constexpr int kTileTC = 128;

cudaError_t launch_gemm(const Operand& A, const Operand& B, bool b_mn, const Job& job, int grid, int* info,
                        cudaStream_t st);
// C = alpha * A B^T + beta * C with A [M x K] and B [N x K] bf16 (both
// K-major), fp32 accumulation and C; Job fields as above (mode 0 only, no
// planes needed).
cudaError_t launch_gemm_bf16(const OperandBf16& A, const OperandBf16& B, const Job& job, int grid, int* info,
                             cudaStream_t st);
cudaError_t launch_split(const float* src, long long ld, int rows, int cols, float* hi, float* lo, long long ldo,
                         const int* info, cudaStream_t st);

}  // namespace tc
}  // namespace sgpt
