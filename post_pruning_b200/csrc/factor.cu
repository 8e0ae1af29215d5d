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
// One CTA factors the diagonal block A_kk = R_kk R_kk^T (R_kk upper) and
// inverts it, U_kk = R_kk^-1, in float64. 256 threads form a 16 x 16 grid;
// thread (ty, tx) keeps A[i][l] for i = ty + 16a, l = tx + 16c (a, c < 8) in
// registers (cyclic layout, so the shrinking active triangle stays spread
// over all threads). Each pivot j costs one barrier: column j of the current
// matrix is broadcast through a double-buffered shared vector, every thread
// applies the rank-1 update A[i][l] -= a_ij a_lj / a_jj to its entries with
// i <= l < j, and the owners of column j-1 publish it for the next pivot.
// The inverse runs the same way over rows: X[i][.] = B[i][.] / r_ii, then
// B[l][.] -= r_li X[i][.] for l < i, with B = I initially and R in shared
// memory.

constexpr int kDiagThreads = 256;
constexpr int kDiagLd = kTile + 1;
constexpr size_t kDiagSmem = (size_t)kTile * kDiagLd * sizeof(double);

__global__ void __launch_bounds__(kDiagThreads, 1) diag_factor_kernel(const float* __restrict__ Rws,
                                                                      int d, int k,
                                                                      float* __restrict__ Ukk,
                                                                      float* __restrict__ U,
                                                                      int* info) {
  if (cta_info_set(info)) return;
  extern __shared__ double Rs[];            // [128][129], R after the factorisation
  __shared__ double vec[2][kTile];          // broadcast column (factor) / row (inverse)
  __shared__ double piv[2][3];              // 1/a_jj, 1/sqrt(a_jj), sqrt(a_jj)
  __shared__ int bad;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int b0 = k * kTile;
  const int b = min(kTile, d - b0);
  double r[8][8];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int i = ty + 16 * a, l = tx + 16 * c;
      r[a][c] = (i <= l && l < b) ? (double)Rws[(long long)(b0 + i) * d + b0 + l] : 0.0;
    }
  if (tid == 0) bad = 0;
  __syncthreads();

  // publish column j (entries i <= j) and its pivot into buffer p
  auto publish_col = [&](int j, int p) {
    if (tx != (j & 15)) return;
    const int cj = j >> 4;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      if (c != cj) continue;
#pragma unroll
      for (int a = 0; a < 8; ++a) {
        const int i = ty + 16 * a;
        if (i > j) continue;
        vec[p][i] = r[a][c];
        if (i == j) {
          const double pv = r[a][c];
          if (!(pv > 0.0)) {
            bad = isfinite(pv) ? (b0 + j + 1) : SGPT_INFO_NONFINITE;
            piv[p][0] = piv[p][1] = piv[p][2] = 0.0;
          } else {
            const double sq = sqrt(pv);
            piv[p][0] = 1.0 / pv;
            piv[p][1] = 1.0 / sq;
            piv[p][2] = sq;
          }
        }
      }
    }
  };

  publish_col(b - 1, 0);
  for (int j = b - 1, p = 0; j >= 0; --j, p ^= 1) {
    __syncthreads();
    if (bad) {
      if (tid == 0) set_info(info, bad);
      return;
    }
    const double pinv = piv[p][0], rs = piv[p][1], sq = piv[p][2];
    double ci[8], cl[8];
#pragma unroll
    for (int a = 0; a < 8; ++a) {
      const int i = ty + 16 * a;
      ci[a] = i <= j ? vec[p][i] * pinv : 0.0;
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int l = tx + 16 * c;
      cl[c] = l <= j ? vec[p][l] : 0.0;
    }
    // rank-1 update of the leading j x j upper triangle
#pragma unroll
    for (int a = 0; a < 8; ++a) {
      const int i = ty + 16 * a;
      if (i >= j) continue;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int l = tx + 16 * c;
        if (l >= i && l < j) r[a][c] = fma(-ci[a], cl[c], r[a][c]);
      }
    }
    // column j becomes column j of R
    if (tx == (j & 15)) {
      const int cj = j >> 4;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        if (c != cj) continue;
#pragma unroll
        for (int a = 0; a < 8; ++a) {
          const int i = ty + 16 * a;
          if (i < j) r[a][c] *= rs;
          else if (i == j) r[a][c] = sq;
        }
      }
    }
    if (j > 0) publish_col(j - 1, p ^ 1);
  }

  // R to shared memory; registers become B = I
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int i = ty + 16 * a, l = tx + 16 * c;
      Rs[i * kDiagLd + l] = (i <= l && l < b) ? r[a][c] : 0.0;
      r[a][c] = (i == l && i < b) ? 1.0 : 0.0;
    }

  // publish row i of X = B[i][.] / r_ii (entries j >= i) into buffer p; the
  // owners keep X in their registers.
  auto publish_row = [&](int i, int p) {
    if (ty != (i & 15)) return;
    const int ai = i >> 4;
    const double inv = 1.0 / Rs[i * kDiagLd + i];
#pragma unroll
    for (int a = 0; a < 8; ++a) {
      if (a != ai) continue;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int l = tx + 16 * c;
        if (l < i || l >= b) continue;
        r[a][c] *= inv;
        vec[p][l] = r[a][c];
      }
    }
  };

  __syncthreads();
  publish_row(b - 1, 0);
  for (int i = b - 1, p = 0; i > 0; --i, p ^= 1) {
    __syncthreads();
    double xr[8], rc[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int l = tx + 16 * c;
      xr[c] = (l >= i && l < b) ? vec[p][l] : 0.0;
    }
#pragma unroll
    for (int a = 0; a < 8; ++a) {
      const int row = ty + 16 * a;
      rc[a] = row < i ? Rs[row * kDiagLd + i] : 0.0;
    }
#pragma unroll
    for (int a = 0; a < 8; ++a) {
      const int row = ty + 16 * a;
      if (row >= i) continue;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int l = tx + 16 * c;
        if (l >= i && l < b) r[a][c] = fma(-rc[a], xr[c], r[a][c]);
      }
    }
    publish_row(i - 1, p ^ 1);
  }

  // Write U_kk (upper, zeros below) to the output and to the block cache.
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int i = ty + 16 * a, l = tx + 16 * c;
      const float v = (i <= l && l < b) ? (float)r[a][c] : 0.f;
      Ukk[i * kTile + l] = v;
      if (i < b && l < b) U[(long long)(b0 + i) * d + b0 + l] = v;
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
