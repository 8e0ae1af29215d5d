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
// shared memory by one CTA; the panel solve and the V scaling are FP32 SIMT
// tile products; the rank-128 updates of the leading part and the
// triangular inverse (the d^3/3 + d^3/3 flops) run on the tensor cores as
// FP32-accurate three-product TF32 GEMMs (gemm_tc.cu).
#include <cuda_runtime.h>

#include "common.cuh"
#include "gemm_simt.cuh"
#include "gemm_tc.h"
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
// inverts it, U_kk = R_kk^-1, in FP32 shared memory. The block is treated as
// up to 4 x 4 sub-blocks of 32 (width b = 32..128), processed from the last
// 32-panel to the first:
//   1. warp 0 factors the 32 x 32 diagonal sub-block D_pp = R_pp R_pp^T (lane
//      = row, pivots broadcast by shuffles, no CTA barrier) and inverts R_pp
//      (lane = column, back substitution against R_pp in shared memory);
//   2. panel: R_ip = A_ip U_pp^T for the sub-blocks above (one warp each);
//   3. update: A_ij -= R_ip R_jp^T for the leading sub-blocks (one warp each).
// Then V_pm = U_pp R_pm and the off-diagonal blocks of U along the
// anti-diagonals, U_pq = -sum_{m=p+1..q} V_pm U_mq.
// Warp-level 32 x 32 products keep one operand column per lane in registers
// and read the other operand's rows as broadcast 16-byte loads.

constexpr int kDiagThreads = 256;
constexpr int kDiagLd = kTile + 4;     // 16-byte aligned rows
constexpr size_t kDiagSmem = 2 * (size_t)kTile * kDiagLd * sizeof(float);

// acc[i] = sum_k A[i][k] * b[k] for the 32 rows of A (row stride kDiagLd,
// 16-byte aligned, read as broadcasts), b in registers.
__device__ __forceinline__ void rows_dot32(const float* A, const float (&b)[32], float (&acc)[32]) {
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const float* a = A + i * kDiagLd;
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < 32; k += 4) {
      const float4 x = *reinterpret_cast<const float4*>(a + k);
      s = fmaf(x.x, b[k], s);
      s = fmaf(x.y, b[k + 1], s);
      s = fmaf(x.z, b[k + 2], s);
      s = fmaf(x.w, b[k + 3], s);
    }
    acc[i] = s;
  }
}

__global__ void __launch_bounds__(kDiagThreads, 1) diag_factor_kernel(const float* __restrict__ Rws,
                                                                      int d, int k,
                                                                      float* __restrict__ Ukk,
                                                                      float* __restrict__ U,
                                                                      int* info) {
  if (cta_info_set(info)) return;
  extern __shared__ __align__(16) float dsm[];
  float* S = dsm;                        // A, becoming R (upper)
  float* Ui = dsm + kTile * kDiagLd;     // U (upper)
  __shared__ float rinv[kTile];
  __shared__ int bad;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b0 = k * kTile;
  const int b = min(kTile, d - b0);      // a multiple of 32
  const int np = b >> 5;
  for (int e = tid; e < kTile * kTile; e += kDiagThreads) {
    const int i = e >> 7, l = e & 127;
    S[i * kDiagLd + l] = (i <= l && l < b) ? Rws[(long long)(b0 + i) * d + b0 + l] : 0.f;
    Ui[i * kDiagLd + l] = 0.f;
  }
  if (tid == 0) bad = 0;
  __syncthreads();

  for (int p = np - 1; p >= 0; --p) {
    const int c0 = p * 32;
    if (warp == 0) {
      // ---- reverse Cholesky of the 32 x 32 diagonal sub-block, lane = row
      float dr[32];
      float* row = S + (c0 + lane) * kDiagLd + c0;
#pragma unroll
      for (int l = 0; l < 32; ++l) dr[l] = row[l];
      int fail = 0;
#pragma unroll
      for (int j = 31; j >= 0; --j) {
        const float piv = __shfl_sync(0xffffffffu, dr[j], j);
        if (!(piv > 0.f) && fail == 0) fail = isfinite(piv) ? (b0 + c0 + j + 1) : SGPT_INFO_NONFINITE;
        const float sq = sqrtf(piv);
        const float inv = 1.0f / sq;
        const float rij = lane < j ? dr[j] * inv : (lane == j ? sq : 0.f);
#pragma unroll
        for (int l = 0; l < j; ++l) {
          const float rlj = __shfl_sync(0xffffffffu, rij, l);
          if (lane <= l) dr[l] = fmaf(-rij, rlj, dr[l]);
        }
        dr[j] = rij;
      }
#pragma unroll
      for (int l = 0; l < 32; ++l) row[l] = lane <= l ? dr[l] : 0.f;
      if (fail && lane == 0) bad = fail;
    }
    __syncthreads();
    if (bad) {
      if (tid == 0) set_info(info, bad);
      return;
    }
    if (warp == 0) {
      rinv[c0 + lane] = 1.0f / S[(c0 + lane) * kDiagLd + c0 + lane];
      __syncwarp();
      // ---- U_pp = R_pp^-1, lane = column j: back substitution from the bottom
      float u[32];
      const float* R = S + c0 * kDiagLd + c0;
#pragma unroll
      for (int i = 31; i >= 0; --i) {
        float sacc = (i == lane) ? 1.f : 0.f;
#pragma unroll
        for (int m = i + 1; m < 32; ++m) sacc = fmaf(-R[i * kDiagLd + m], u[m], sacc);
        u[i] = (i <= lane) ? sacc * rinv[c0 + i] : 0.f;
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) Ui[(c0 + i) * kDiagLd + c0 + lane] = u[i];
    }
    __syncthreads();
    if (p == 0) break;
    // ---- panel: R_ip = A_ip U_pp^T, rows blocks i < p (in place)
    if (warp < p) {
      float bcol[32], acc[32];
      const float* ur = Ui + (c0 + lane) * kDiagLd + c0;    // row `lane` of U_pp = column of U_pp^T
#pragma unroll
      for (int m = 0; m < 32; m += 4) {
        const float4 x = *reinterpret_cast<const float4*>(ur + m);
        bcol[m] = x.x; bcol[m + 1] = x.y; bcol[m + 2] = x.z; bcol[m + 3] = x.w;
      }
      float* Ablk = S + (warp * 32) * kDiagLd + c0;
      rows_dot32(Ablk, bcol, acc);
      __syncwarp();
#pragma unroll
      for (int i = 0; i < 32; ++i) Ablk[i * kDiagLd + lane] = acc[i];
    }
    __syncthreads();
    // ---- update of the leading sub-blocks: A_ij -= R_ip R_jp^T, i <= j < p
    {
      const int pairs = p * (p + 1) / 2;
      if (warp < pairs) {
        int jj = 0;
        while ((jj + 1) * (jj + 2) / 2 <= warp) ++jj;
        const int ii = warp - jj * (jj + 1) / 2;          // ii <= jj
        float bcol[32], acc[32];
        const float* rp = S + (jj * 32 + lane) * kDiagLd + c0;   // row of R_jp = column of R_jp^T
#pragma unroll
        for (int m = 0; m < 32; m += 4) {
          const float4 x = *reinterpret_cast<const float4*>(rp + m);
          bcol[m] = x.x; bcol[m + 1] = x.y; bcol[m + 2] = x.z; bcol[m + 3] = x.w;
        }
        rows_dot32(S + (ii * 32) * kDiagLd + c0, bcol, acc);
        float* C = S + (ii * 32) * kDiagLd + jj * 32;
#pragma unroll
        for (int i = 0; i < 32; ++i) C[i * kDiagLd + lane] -= acc[i];
      }
    }
    __syncthreads();
  }

  // ---- V_pm = U_pp R_pm (p < m), in place over R_pm: lane = column of R_pm
  {
    const int pairs = np * (np - 1) / 2;
    if (warp < pairs) {
      int mm = 0;
      while ((mm + 1) * (mm + 2) / 2 <= warp) ++mm;
      const int pp = warp - mm * (mm + 1) / 2;            // pp <= mm
      mm += 1;                                             // pp < mm
      float bcol[32], acc[32];
      float* Rpm = S + (pp * 32) * kDiagLd + mm * 32;
#pragma unroll
      for (int kk = 0; kk < 32; ++kk) bcol[kk] = Rpm[kk * kDiagLd + lane];
      rows_dot32(Ui + (pp * 32) * kDiagLd + pp * 32, bcol, acc);
      __syncwarp();
#pragma unroll
      for (int i = 0; i < 32; ++i) Rpm[i * kDiagLd + lane] = acc[i];
    }
  }
  __syncthreads();
  // ---- off-diagonal blocks of U by anti-diagonals: U_pq = -sum V_pm U_mq
  for (int sd = 1; sd < np; ++sd) {
    if (warp < np - sd) {
      const int pp = warp, qq = warp + sd;
      float acc[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) acc[i] = 0.f;
      for (int mm = pp + 1; mm <= qq; ++mm) {
        float bcol[32], part[32];
        const float* Umq = Ui + (mm * 32) * kDiagLd + qq * 32;
#pragma unroll
        for (int kk = 0; kk < 32; ++kk) bcol[kk] = Umq[kk * kDiagLd + lane];
        rows_dot32(S + (pp * 32) * kDiagLd + mm * 32, bcol, part);
#pragma unroll
        for (int i = 0; i < 32; ++i) acc[i] += part[i];
      }
      float* Upq = Ui + (pp * 32) * kDiagLd + qq * 32;
#pragma unroll
      for (int i = 0; i < 32; ++i) Upq[i * kDiagLd + lane] = -acc[i];
    }
    __syncthreads();
  }

  // Write U_kk (upper, zeros below) to the output and to the block cache.
  for (int e = tid * 4; e < kTile * kTile; e += kDiagThreads * 4) {
    const int i = e >> 7, l = e & 127;
    const float4 v = *reinterpret_cast<const float4*>(Ui + i * kDiagLd + l);
    st4(Ukk + e, v);
    if (i < b && l < b) st4(U + (long long)(b0 + i) * d + b0 + l, v);
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

// ----------------------------------------------------------------- driver

struct FactorWs {
  double* lam;
  float* R;        // H_d, then R, then V; finally the hi plane of V
  float* Udiag;    // U_kk blocks, 128 x 128 each
  float* P_hi;     // hi/lo planes of the current panel (d x 128)
  float* P_lo;
  float* V_lo;     // lo plane of V (d x d)
  float* U_hi;     // hi/lo planes of U (d x d)
  float* U_lo;
  float* part;     // split partials of the triangular inverse
};

static FactorWs carve_factor(void* ws, int d, size_t* bytes) {
  Carve c(ws);
  const int K = cdiv(d, kTile);
  FactorWs w;
  w.lam = c.take<double>(4);
  w.R = c.take<float>((size_t)d * d);
  w.Udiag = c.take<float>((size_t)K * kTile * kTile);
  w.P_hi = c.take<float>((size_t)d * kTile);
  w.P_lo = c.take<float>((size_t)d * kTile);
  w.V_lo = c.take<float>((size_t)d * d);
  w.U_hi = c.take<float>((size_t)d * d);
  w.U_lo = c.take<float>((size_t)d * d);
  w.part = c.take<float>(factor_part_tiles(d) * kTile * kTile);
  if (bytes) *bytes = c.off + 256;
  return w;
}

size_t factor_ws_bytes(int d) {
  size_t b = 0;
  carve_factor(nullptr, d, &b);
  return b;
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
  const int K = cdiv(d, kTile);
  const FactorWs w = carve_factor(ws, d, nullptr);
  static bool attr_done = false;
  if (!attr_done) {
    cudaFuncSetAttribute(diag_factor_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDiagSmem);
    attr_done = true;
  }
  const double scale = 2.0 / (double)n_total;
  if (U != H) cudaMemsetAsync(U, 0, (size_t)d * d * sizeof(float), st);
  damp_lambda_kernel<<<1, 1024, 0, st>>>(H, d, scale, (double)damp, w.lam, info);
  count_launches(1);
  scale_damp_kernel<<<dim3(cdiv(d, 4 * 128), d), 128, 0, st>>>(H, w.R, d, scale, w.lam, info);
  count_launches(1);
  if (U == H) cudaMemsetAsync(U, 0, (size_t)d * d * sizeof(float), st);
  cudaError_t e = cudaSuccess;
  for (int k = K - 1; k >= 0; --k) {
    diag_factor_kernel<<<1, kDiagThreads, kDiagSmem, st>>>(w.R, d, k, w.Udiag + (size_t)k * kTile * kTile, U, info);
    count_launches(1);
    if (k == 0) break;
    const int bk = min(kTile, d - k * kTile);
    panel_kernel<<<k, kGemmThreads, kGemmSmemBytes, st>>>(w.R, d, k, w.Udiag + (size_t)k * kTile * kTile, info);
    count_launches(1);
    // rank-bk update of the leading upper tiles on the tensor cores
    if ((e = tc::launch_split(w.R + k * kTile, d, k * kTile, bk, w.P_hi, w.P_lo, kTile, info, st)) != cudaSuccess)
      return e;
    const tc::Operand P{w.P_hi, w.P_lo, (long long)k * kTile, kTile, kTile};
    tc::Job job{};
    job.mode = 1;
    job.kdim = bk;
    job.C = w.R;
    job.ldc = d;
    job.Mlim = job.Nlim = k * kTile;
    job.alpha = -1.f;
    job.beta = 1.f;
    if ((e = tc::launch_gemm(P, P, false, job, k * (k + 1) / 2, info, st)) != cudaSuccess) return e;
  }
  if (K > 1) {
    vscale_kernel<<<K * (K - 1) / 2, kGemmThreads, kGemmSmemBytes, st>>>(w.R, d, w.Udiag, info);
    count_launches(1);
    // planes of V (hi in place over R) and of U (its diagonal blocks so far)
    if ((e = tc::launch_split(w.R, d, d, d, w.R, w.V_lo, d, info, st)) != cudaSuccess) return e;
    if ((e = tc::launch_split(U, d, d, d, w.U_hi, w.U_lo, d, info, st)) != cudaSuccess) return e;
    const tc::Operand V{w.R, w.V_lo, d, d, d};
    const tc::Operand Up{w.U_hi, w.U_lo, d, d, d};
    for (int s = 1; s < K; ++s) {
      tc::Job job{};
      job.mode = 2;
      job.s = s;
      job.nsplit = trtri_splits(K, s);
      job.nblk = K;
      job.dlim = d;
      job.C = U;
      job.ldc = d;
      job.Mlim = job.Nlim = d;
      job.alpha = -1.f;
      job.beta = 0.f;
      job.C_hi = w.U_hi;
      job.C_lo = w.U_lo;
      job.part = w.part;
      if ((e = tc::launch_gemm(V, Up, true, job, (K - s) * job.nsplit, info, st)) != cudaSuccess) return e;
    }
  }
  return cudaGetLastError();
}

}  // namespace sgpt
