// Damping and factorisation: U = upper Cholesky factor of H_d^-1.
//
// Route (same U as Cholesky -> inverse -> Cholesky, by uniqueness of the
// factor with positive diagonal): factor H_d = R R^T with R upper triangular
// ("reverse" Cholesky, processed from the last column block to the first),
// then U = R^-1. Indeed H_d^-1 = R^-T R^-1 = U^T U with U = R^-1 upper.
// This costs d^3/3 + d^3/3 flops instead of the 4/3 d^3 of the three-step
// route. The pages (SparseGPT review, section 八) only fix that the inverse
// Hessian drives the compensation; the factor of H_d^-1 is the form in which
// the sweep consumes it.
//
// Blocking: 128 x 128 tiles. Diagonal blocks are factored and inverted in
// float64 in shared memory by one CTA; all off-diagonal work (panel solve,
// rank-128 updates, triangular inverse) runs as FP32 SIMT tile products.
#include <cuda_runtime.h>

#include "common.cuh"
#include "gemm_simt.cuh"
#include "kernels.h"

namespace sgpt {

// ---------------------------------------------------------------- damping

// lam = damp * mean(diag(scale * H)) in float64; flags a non-finite diagonal.
__global__ void __launch_bounds__(1024) damp_lambda_kernel(const float* __restrict__ H, int d,
                                                           double scale, double damp,
                                                           double* __restrict__ lam_out,
                                                           int* info) {
  __shared__ double part[32];
  __shared__ int bad;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  double s = 0.0;
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    const float h = H[(long long)i * d + i];
    if (!isfinite(h)) bad = 1;
    s += scale * (double)h;
  }
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    s = threadIdx.x < (blockDim.x >> 5) ? part[threadIdx.x] : 0.0;
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (threadIdx.x == 0) {
      *lam_out = damp * (s / d);
      if (bad) set_info(info, SGPT_INFO_NONFINITE);
    }
  }
}

// R[i][j] = scale * H[i][j] (+ lam on the diagonal), upper triangle only.
__global__ void scale_damp_kernel(const float* __restrict__ H, float* __restrict__ R, int d,
                                  double scale, const double* __restrict__ lam, const int* info) {
  if (cta_info_set(info)) return;
  const int i = blockIdx.y;
  const double l = *lam;
  for (int j4 = (blockIdx.x * blockDim.x + threadIdx.x) * 4; j4 < d; j4 += gridDim.x * blockDim.x * 4) {
    if (j4 + 3 < i) continue;
    const float4 h = ld4(H + (long long)i * d + j4);
    float v[4] = {h.x, h.y, h.z, h.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      double x = scale * (double)v[t];
      if (j4 + t == i) x += l;
      v[t] = (float)x;
    }
    st4(R + (long long)i * d + j4, make_float4(v[0], v[1], v[2], v[3]));
  }
}

// ------------------------------------------------------- diagonal blocks
//
// One CTA factors the diagonal block A_kk = R_kk R_kk^T (R_kk upper) in
// float64 and inverts it: U_kk = R_kk^-1. Layout in shared memory: one
// 128 x 129 float64 array; R in the strict upper triangle, U transposed in
// the strict lower triangle (A[j][i] = U[i][j], i < j), diagonals apart.

constexpr int kDiagThreads = 512;
constexpr int kDiagLd = kTile + 1;
constexpr size_t kDiagSmem = (size_t)kTile * kDiagLd * sizeof(double) + 2 * kTile * sizeof(double);

__global__ void __launch_bounds__(kDiagThreads) diag_factor_kernel(const float* __restrict__ Rws,
                                                                   int d, int k,
                                                                   float* __restrict__ Ukk,
                                                                   float* __restrict__ U,
                                                                   int* info) {
  if (cta_info_set(info)) return;
  extern __shared__ double sm[];
  double* A = sm;                        // [128][129]
  double* dR = sm + kTile * kDiagLd;     // R_ii
  double* dU = dR + kTile;               // U_ii
  __shared__ int bad;
  const int tid = threadIdx.x;
  const int b0 = k * kTile;
  const int b = min(kTile, d - b0);
  for (int idx = tid; idx < b * b; idx += kDiagThreads) {
    const int i = idx / b, j = idx - (idx / b) * b;
    if (i <= j) A[i * kDiagLd + j] = (double)Rws[(long long)(b0 + i) * d + b0 + j];
  }
  if (tid == 0) bad = 0;
  __syncthreads();

  // Reverse Cholesky: for j = b-1 .. 0: r_jj = sqrt(a_jj); r_ij = a_ij / r_jj
  // (i < j); a_il -= r_ij r_lj for i <= l < j.
  const int ty = tid >> 5, tx = tid & 31;   // 16 x 32 thread grid
  for (int j = b - 1; j >= 0; --j) {
    if (tid == 0) {
      const double piv = A[j * kDiagLd + j];
      if (!(piv > 0.0)) bad = isfinite(piv) ? (b0 + j + 1) : SGPT_INFO_NONFINITE;
      else dR[j] = sqrt(piv);
    }
    __syncthreads();
    if (bad) {
      if (tid == 0) set_info(info, bad);
      return;
    }
    const double rjj = dR[j];
    for (int i = tid; i < j; i += kDiagThreads) A[i * kDiagLd + j] /= rjj;
    __syncthreads();
    for (int i = ty; i < j; i += 16) {
      const double rij = A[i * kDiagLd + j];
      for (int l = i + tx; l < j; l += 32) A[i * kDiagLd + l] -= rij * A[l * kDiagLd + j];
    }
    __syncthreads();
  }

  // Inverse, bottom row first: X[i][j] = B[i][j] / r_ii (j >= i), then
  // B[l][j] -= r_li X[i][j] for l < i <= j. B starts as the identity.
  for (int idx = tid; idx < b * b; idx += kDiagThreads) {
    const int i = idx / b, j = idx - (idx / b) * b;
    if (i > j) A[i * kDiagLd + j] = 0.0;
  }
  for (int i = tid; i < b; i += kDiagThreads) dU[i] = 1.0;
  __syncthreads();
  for (int i = b - 1; i >= 0; --i) {
    const double inv = 1.0 / dR[i];
    for (int j = i + tid; j < b; j += kDiagThreads) {
      if (j == i) dU[i] *= inv;
      else A[j * kDiagLd + i] *= inv;
    }
    __syncthreads();
    // rows l < i, columns j >= i
    for (int l = ty; l < i; l += 16) {
      const double rli = A[l * kDiagLd + i];
      for (int j = i + tx; j < b; j += 32) {
        const double x = (j == i) ? dU[i] : A[j * kDiagLd + i];
        A[j * kDiagLd + l] -= rli * x;
      }
    }
    __syncthreads();
  }

  // Write U_kk (upper, zeros below) to the output and to the block cache.
  for (int idx = tid; idx < kTile * kTile; idx += kDiagThreads) {
    const int i = idx >> 7, j = idx & 127;
    float v = 0.f;
    if (i < b && j < b) {
      if (i == j) v = (float)dU[i];
      else if (i < j) v = (float)A[j * kDiagLd + i];
    }
    Ukk[idx] = v;
    if (i < b && j < b) U[(long long)(b0 + i) * d + b0 + j] = v;
  }
}

// ------------------------------------------------- off-diagonal products

// Panel: R_ik = A_ik U_kk^T for every row block i < k (in place).
__global__ void __launch_bounds__(kGemmThreads) panel_kernel(float* __restrict__ Rws, int d, int k,
                                                             const float* __restrict__ Ukk,
                                                             const int* info) {
  if (cta_info_set(info)) return;
  extern __shared__ float smem[];
  const int i = blockIdx.x;
  const int bk = min(kTile, d - k * kTile);
  float acc[8][8];
  zero_acc(acc);
  const OpKContig A{Rws + k * kTile, d, i * kTile, kTile, bk};
  const OpKContig B{Ukk, kTile, 0, bk, bk};
  gemm_tile(A, B, 0, bk, acc, smem);
  store_tile(Rws + (long long)i * kTile * d + k * kTile, d, kTile, bk, acc, 1.f, 0.f);
}

__device__ __forceinline__ void upper_tile_index(int t, int& i, int& j) {
  // t enumerates (i <= j) row by row: row i holds tiles j = i .. n-1; with n
  // unknown here we enumerate by j instead: column j holds i = 0..j.
  int jj = (int)((sqrtf(8.f * t + 1.f) - 1.f) * 0.5f);
  while ((jj + 1) * (jj + 2) / 2 <= t) ++jj;
  while (jj * (jj + 1) / 2 > t) --jj;
  j = jj;
  i = t - jj * (jj + 1) / 2;
}

// Rank-128 update of the leading part: A_ij -= R_ik R_jk^T, i <= j < k.
__global__ void __launch_bounds__(kGemmThreads) syrk_kernel(float* __restrict__ Rws, int d, int k,
                                                            const int* info) {
  if (cta_info_set(info)) return;
  extern __shared__ float smem[];
  int i, j;
  upper_tile_index(blockIdx.x, i, j);
  const int bk = min(kTile, d - k * kTile);
  float acc[8][8];
  zero_acc(acc);
  const OpKContig A{Rws + k * kTile, d, i * kTile, kTile, bk};
  const OpKContig B{Rws + k * kTile, d, j * kTile, kTile, bk};
  gemm_tile(A, B, 0, bk, acc, smem);
  store_tile(Rws + (long long)i * kTile * d + j * kTile, d, kTile, kTile, acc, -1.f, 1.f);
}

// V_im = U_ii R_im for every off-diagonal block i < m (in place over R).
__global__ void __launch_bounds__(kGemmThreads) vscale_kernel(float* __restrict__ Rws, int d,
                                                              const float* __restrict__ Udiag,
                                                              const int* info) {
  if (cta_info_set(info)) return;
  extern __shared__ float smem[];
  int i, m;
  upper_tile_index(blockIdx.x, i, m);   // i <= m-1 enumerated as (i, m-1)
  m += 1;
  const int bm = min(kTile, d - m * kTile);
  float acc[8][8];
  zero_acc(acc);
  const OpKContig A{Udiag + (size_t)i * kTile * kTile, kTile, 0, kTile, kTile};
  const OpIContig B{Rws + (long long)i * kTile * d, d, m * kTile, bm, kTile};
  gemm_tile(A, B, 0, kTile, acc, smem);
  store_tile(Rws + (long long)i * kTile * d + m * kTile, d, kTile, bm, acc, 1.f, 0.f);
}

// Anti-diagonal s of U: U_ij = -sum_{m=i+1..j} V_im U_mj, j = i + s.
// Split over m into `nsplit` chunks; partial tiles go to `part`, and the CTA
// that finishes a tile last sums its partials in split order (deterministic).
__global__ void __launch_bounds__(kGemmThreads) trtri_kernel(const float* __restrict__ V,
                                                             float* __restrict__ U, int d, int s,
                                                             int nsplit, float* __restrict__ part,
                                                             unsigned int* __restrict__ tickets,
                                                             const int* info) {
  if (cta_info_set(info)) return;
  extern __shared__ float smem[];
  __shared__ unsigned int last;
  const int tile = blockIdx.x / nsplit;
  const int split = blockIdx.x - tile * nsplit;
  const int i = tile, j = tile + s;
  const int bj = min(kTile, d - j * kTile);
  const int k_lo = (i + 1) * kTile, k_hi = min((j + 1) * kTile, d);
  const int nblk = s;                       // blocks m = i+1 .. j
  const int per = cdiv(nblk, nsplit);
  const int kb = k_lo + split * per * kTile;
  const int ke = min(k_hi, kb + per * kTile);
  float acc[8][8];
  zero_acc(acc);
  const OpKContig A{V, d, i * kTile, kTile, k_hi};
  const OpIContig B{U, d, j * kTile, bj, k_hi};
  gemm_tile(A, B, kb, ke, acc, smem);
  float* Ut = U + (long long)i * kTile * d + j * kTile;
  if (nsplit == 1) {
    store_tile(Ut, d, kTile, bj, acc, -1.f, 0.f);
    return;
  }
  float* mine = part + ((size_t)blockIdx.x) * kTile * kTile;
  store_tile(mine, kTile, kTile, bj, acc, 1.f, 0.f);
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last = (atomicAdd(&tickets[tile], 1u) == (unsigned)nsplit - 1);
  __syncthreads();
  if (!last) return;
  __threadfence();
  const float* base = part + (size_t)tile * nsplit * kTile * kTile;
  for (int e = threadIdx.x * 4; e < kTile * bj; e += kGemmThreads * 4) {
    const int r = e / bj, c = e - (e / bj) * bj;
    float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int p = 0; p < nsplit; ++p) {
      const float4 v = __ldcg(reinterpret_cast<const float4*>(base + (size_t)p * kTile * kTile + r * kTile + c));
      sum.x += v.x; sum.y += v.y; sum.z += v.z; sum.w += v.w;
    }
    st4(Ut + (long long)r * d + c, make_float4(-sum.x, -sum.y, -sum.z, -sum.w));
  }
  if (threadIdx.x == 0) tickets[tile] = 0;
}

// ----------------------------------------------------------------- driver

size_t factor_ws_bytes(int d) {
  Carve c(nullptr);
  const int K = cdiv(d, kTile);
  c.take<double>(4);
  c.take<float>((size_t)d * d);                      // R, then V
  c.take<float>((size_t)K * kTile * kTile);          // U_kk cache
  c.take<unsigned int>((size_t)K + 32);              // tickets
  c.take<float>(factor_part_tiles(d) * kTile * kTile);
  return c.off + 256;
}

size_t factor_part_tiles(int d) {
  const int K = cdiv(d, kTile);
  size_t best = 0;
  for (int s = 1; s < K; ++s) {
    const size_t t = (size_t)(K - s) * trtri_splits(K, s);
    if (t > best) best = t;
  }
  return best;
}

int trtri_splits(int K, int s) {
  // aim for two CTAs per SM on each anti-diagonal, at least 2 blocks of m each
  const int tiles = K - s;
  int n = cdiv(2 * kNumSMs, tiles);
  n = min(n, max(1, s / 2));
  return max(1, n);
}

cudaError_t launch_factor(const float* H, long long n_total, int d, float damp, float* U, void* ws,
                          int* info, cudaStream_t st) {
  Carve c(ws);
  const int K = cdiv(d, kTile);
  double* lam = c.take<double>(4);
  float* R = c.take<float>((size_t)d * d);
  float* Udiag = c.take<float>((size_t)K * kTile * kTile);
  unsigned int* tickets = c.take<unsigned int>((size_t)K + 32);
  float* part = c.take<float>(factor_part_tiles(d) * kTile * kTile);
  static bool attr_done = false;
  if (!attr_done) {
    cudaFuncSetAttribute(diag_factor_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDiagSmem);
    attr_done = true;
  }
  const double scale = 2.0 / (double)n_total;
  cudaMemsetAsync(tickets, 0, ((size_t)K + 32) * sizeof(unsigned int), st);
  if (U != H) cudaMemsetAsync(U, 0, (size_t)d * d * sizeof(float), st);
  damp_lambda_kernel<<<1, 1024, 0, st>>>(H, d, scale, (double)damp, lam, info);
  count_launches(1);
  scale_damp_kernel<<<dim3(cdiv(d, 4 * 128), d), 128, 0, st>>>(H, R, d, scale, lam, info);
  count_launches(1);
  if (U == H) cudaMemsetAsync(U, 0, (size_t)d * d * sizeof(float), st);
  for (int k = K - 1; k >= 0; --k) {
    diag_factor_kernel<<<1, kDiagThreads, kDiagSmem, st>>>(R, d, k, Udiag + (size_t)k * kTile * kTile, U, info);
    count_launches(1);
    if (k == 0) break;
    panel_kernel<<<k, kGemmThreads, kGemmSmemBytes, st>>>(R, d, k, Udiag + (size_t)k * kTile * kTile, info);
    count_launches(1);
    syrk_kernel<<<k * (k + 1) / 2, kGemmThreads, kGemmSmemBytes, st>>>(R, d, k, info);
    count_launches(1);
  }
  if (K > 1) {
    vscale_kernel<<<K * (K - 1) / 2, kGemmThreads, kGemmSmemBytes, st>>>(R, d, Udiag, info);
    count_launches(1);
  }
  for (int s = 1; s < K; ++s) {
    const int ns = trtri_splits(K, s);
    trtri_kernel<<<(K - s) * ns, kGemmThreads, kGemmSmemBytes, st>>>(R, U, d, s, ns, part, tickets, info);
    count_launches(1);
  }
  return cudaGetLastError();
}

}  // namespace sgpt
