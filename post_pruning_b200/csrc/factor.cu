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
// shared memory by one CTA. The serial chain from one diagonal block to the
// next is diag(k) -> chain step(k) -> diag(k-1): the chain step forms, in
// plain FP32 on 136 CTAs, the one panel tile R_{k-1,k} and the update of
// diagonal block k-1 that diag(k-1) waits for. Every other product (the
// panel R_ik = A_ik U_kk^T of the rows above, the rank-128 to rank-512
// updates of the leading part, the sums T_iq = sum_m R_im U_mq over whole
// rectangles and the block rows U_kq = -U_kk T_kq of the inverse) runs off the chain on the
// tensor cores as an FP32-accurate three-product TF32 GEMM (gemm_tc.cu).
// Operands move between those GEMMs as hi/lo planes written by the producing
// epilogue; the planes of the first column block come from the
// scale-and-damp pass, so no separate split pass runs.
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
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
// In the same pass: zero row i of U_zero (when given: the output, which
// then holds the sums T from zero), and for rows above column block col0
// (>= 0) write the hi/lo planes of R[i][col0..] that the first panel reads.
__global__ void scale_damp_kernel(const float* __restrict__ H, float* __restrict__ R, int d,
                                  double scale, const double* __restrict__ lam, const int* info,
                                  float* __restrict__ U_zero, float* __restrict__ A_hi,
                                  float* __restrict__ A_lo, int col0) {
  if (cta_info_set(info)) return;
  const int i = blockIdx.y;
  const double l = *lam;
  for (int j4 = (blockIdx.x * blockDim.x + threadIdx.x) * 4; j4 < d; j4 += gridDim.x * blockDim.x * 4) {
    if (U_zero) st4(U_zero + (long long)i * d + j4, make_float4(0.f, 0.f, 0.f, 0.f));
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
    if (col0 >= 0 && i < col0 && j4 >= col0) {
      const float4 h = make_float4(tf32_hi(v[0]), tf32_hi(v[1]), tf32_hi(v[2]), tf32_hi(v[3]));
      const long long off = (long long)i * kTile + (j4 - col0);
      st4(A_hi + off, h);
      st4(A_lo + off, make_float4(v[0] - h.x, v[1] - h.y, v[2] - h.z, v[3] - h.w));
    }
  }
}

// ------------------------------------------------------- diagonal blocks
//
// One CTA factors the diagonal block A_kk = R_kk R_kk^T (R_kk upper) and
// inverts it, U_kk = R_kk^-1, in FP32 shared memory. The block is treated as
// up to 4 x 4 sub-blocks of 32 (width b = 32..128), processed from the last
// 32-panel p to the first. The pivots are the only serial chain, so one warp
// runs them while the other seven do everything else around it:
//   warp 0, per panel p: waits until D_pp is fully updated, factors it,
//     D_pp = R_pp R_pp^T (lane = row; each pivot's column of R goes through
//     a small shared buffer that every lane reads as broadcasts), inverts
//     it, U_pp = R_pp^-1 (lane = column, back substitution reading that
//     buffer), and signals;
//   warps 1-4 then form the panel row R_{p-1,p} = A_{p-1,p} U_pp^T and
//     update D_{p-1,p-1} -= R_{p-1,p} R_{p-1,p}^T, the only products the
//     next pivots wait for, and signal warp 0;
//   warps 5-7 meanwhile form the other panel rows R_ip (i < p-1); then all
//     seven do the remaining updates A_ij -= R_ip R_jp^T and block row p of
//     U, U_pq = -U_pp T_pq (q > p), from sums T_pq = sum_{m=p+1..q} R_pm U_mq
//     that earlier panels accumulated; then add the terms R_ip U_pq (q >= p)
//     to the sums T_iq of the rows above, and store the 32 finished rows of
//     U (with their hi/lo planes) while the next panel's pivots run.
// So after the last pivot only U_0q = -U_00 T_0q and the store of 32 rows
// remain. Warp 0 and the workers meet on two named barriers (one each way),
// the workers among themselves on two more. Warp-level 32 x 32 products
// keep one operand column per lane in registers and read the other
// operand's rows as broadcast 16-byte loads, in units of 8 rows.

constexpr int kDiagThreads = 256;
constexpr int kDiagWarps = kDiagThreads / 32;
constexpr int kDiagLd = kTile + 4;     // 16-byte aligned rows
constexpr int kPivLd = 36;             // pivot column buffer: 32 rows of 32 (+4)
constexpr size_t kDiagSmem = (3 * (size_t)kTile * kDiagLd + 32 * kPivLd) * sizeof(float);

// sum_k a[k] * b[k] over 32 entries: a is a shared-memory row (16-byte
// aligned, read as broadcasts), b is in registers.
__device__ __forceinline__ float row_dot32(const float* a, const float (&b)[32]) {
  float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
  for (int k = 0; k < 32; k += 4) {
    const float4 x = *reinterpret_cast<const float4*>(a + k);
    s0 = fmaf(x.x, b[k], s0);
    s1 = fmaf(x.y, b[k + 1], s1);
    s2 = fmaf(x.z, b[k + 2], s2);
    s3 = fmaf(x.w, b[k + 3], s3);
  }
  return (s0 + s1) + (s2 + s3);
}

// Row `lane` of a 32-wide shared-memory block into registers.
__device__ __forceinline__ void load_row32(const float* blk, int lane, float (&b)[32]) {
  const float* r = blk + lane * kDiagLd;
#pragma unroll
  for (int k = 0; k < 32; k += 4) {
    const float4 x = *reinterpret_cast<const float4*>(r + k);
    b[k] = x.x; b[k + 1] = x.y; b[k + 2] = x.z; b[k + 3] = x.w;
  }
}
// Column `lane` of a 32 x 32 shared-memory block into registers.
__device__ __forceinline__ void load_col32(const float* blk, int lane, float (&b)[32]) {
#pragma unroll
  for (int k = 0; k < 32; ++k) b[k] = blk[k * kDiagLd + lane];
}

// 1/sqrt(x) to about 1 ulp: the hardware estimate and one Newton step.
__device__ __forceinline__ float rsqrt_nr(float x) {
  const float y = rsqrtf(x);
  return y * fmaf(-0.5f * x * y, y, 1.5f);
}

// t -> (i, j), i <= j, column by column.
__device__ __forceinline__ void tri_pair(int t, int& i, int& j) {
  int jj = 0;
  while ((jj + 1) * (jj + 2) / 2 <= t) ++jj;
  j = jj;
  i = t - jj * (jj + 1) / 2;
}

// Named CTA barriers: `count` threads take part; bar_arrive does not wait.
__device__ __forceinline__ void bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
__device__ __forceinline__ void bar_arrive(int id, int count) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(count) : "memory");
}
constexpr int kWorkers = kDiagWarps - 1;
constexpr int kCritWarps = 4;                    // workers 0-3: the next pivots' products
constexpr int kBarUReady = 1;    // warp 0 -> workers: U_pp (and R_pp) written        (all 256)
constexpr int kBarDReady = 2;    // workers 0-3 -> warp 0: D_{p-1,p-1} updated       (160)
constexpr int kBarCrit = 3;      // workers 0-3 among themselves                     (128)
constexpr int kBarWorkers = 4;   // the seven workers among themselves               (224)
constexpr int kDReadyCount = 32 * (1 + kCritWarps);

// C[8 rows][lane] (+)= sum_k A[8 rows][k] * b[k] for a unit of 8 rows.
__device__ __forceinline__ void unit_dot8(const float* A, const float (&b)[32], float (&acc)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] += row_dot32(A + i * kDiagLd, b);
}

// Warp 0's part for panel p: factor the 32 x 32 diagonal sub-block at
// (c0, c0) of S in place (reverse Cholesky, lane = row) and write its
// inverse into Ui; Pc is a 32 x kPivLd buffer that ends up holding R_pp^T.
// Returns the first failing column + 1 (or SGPT_INFO_NONFINITE), 0 if every
// pivot was positive.
__device__ __forceinline__ int pivot_panel(float* S, float* Ui, float* Pc, float* rinv, int c0, int col0,
                                           int lane) {
  // Pivot j: r_jj = sqrt(a_jj), r_ij = a_ij / r_jj (i < j), then
  // a_il -= r_ij r_lj for l < j. Lane j-1 forms the next pivot from its own
  // r_{j-1,j} and broadcasts it; column j of R goes to Pc[j][.], from where
  // every lane reads r_lj (l < j) as 16-byte broadcasts for the rest of its
  // update. Entries below the diagonal (l < i) take the update too but are
  // never read, and are zeroed on output.
  float dr[32];
  float* row = S + (c0 + lane) * kDiagLd + c0;
  load_row32(S + c0 * kDiagLd + c0, lane, dr);
  int fail = 0;
  float piv = __shfl_sync(0xffffffffu, dr[31], 31);
#pragma unroll
  for (int j = 31; j >= 0; --j) {
    if (!(piv > 0.f) && fail == 0) fail = isfinite(piv) ? (col0 + j + 1) : SGPT_INFO_NONFINITE;
    const float rs = rsqrt_nr(piv);
    const float rij = lane < j ? dr[j] * rs : (lane == j ? piv * rs : 0.f);
    dr[j] = rij;
    Pc[j * kPivLd + lane] = rij;
    if (j == 0) break;
    const float own = fmaf(-rij, rij, dr[j - 1]);
    const float next = __shfl_sync(0xffffffffu, own, j - 1);
    __syncwarp();
#pragma unroll
    for (int l4 = 0; l4 < j; l4 += 4) {
      const float4 c = *reinterpret_cast<const float4*>(Pc + j * kPivLd + l4);
      dr[l4] = fmaf(-rij, c.x, dr[l4]);
      if (l4 + 1 < j) dr[l4 + 1] = fmaf(-rij, c.y, dr[l4 + 1]);
      if (l4 + 2 < j) dr[l4 + 2] = fmaf(-rij, c.z, dr[l4 + 2]);
      if (l4 + 3 < j) dr[l4 + 3] = fmaf(-rij, c.w, dr[l4 + 3]);
    }
    piv = next;
  }
#pragma unroll
  for (int l = 0; l < 32; l += 4)
    *reinterpret_cast<float4*>(row + l) =
        make_float4(lane <= l ? dr[l] : 0.f, lane <= l + 1 ? dr[l + 1] : 0.f, lane <= l + 2 ? dr[l + 2] : 0.f,
                    lane <= l + 3 ? dr[l + 3] : 0.f);
  rinv[c0 + lane] = 1.0f / Pc[lane * kPivLd + lane];   // 1 / r_ii, written by this lane
  __syncwarp();
  // U_pp = R_pp^-1, lane = column: back substitution from the bottom in
  // column form, u_m = acc_m / r_mm, then acc_i -= r_im u_m for i < m, with
  // r_im = Pc[m][i] read as 16-byte broadcasts.
  float u[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) u[i] = (i == lane) ? 1.f : 0.f;
#pragma unroll
  for (int m = 31; m >= 0; --m) {
    u[m] = (m <= lane) ? u[m] * rinv[c0 + m] : 0.f;
#pragma unroll
    for (int i4 = 0; i4 < m; i4 += 4) {
      const float4 c = *reinterpret_cast<const float4*>(Pc + m * kPivLd + i4);
      u[i4] = fmaf(-c.x, u[m], u[i4]);
      if (i4 + 1 < m) u[i4 + 1] = fmaf(-c.y, u[m], u[i4 + 1]);
      if (i4 + 2 < m) u[i4 + 2] = fmaf(-c.z, u[m], u[i4 + 2]);
      if (i4 + 3 < m) u[i4 + 3] = fmaf(-c.w, u[m], u[i4 + 3]);
    }
  }
#pragma unroll
  for (int i = 0; i < 32; ++i) Ui[(c0 + i) * kDiagLd + c0 + lane] = u[i];
  return fail;
}

__global__ void __launch_bounds__(kDiagThreads, 1) diag_factor_kernel(const float* __restrict__ Rws,
                                                                      int d, int k,
                                                                      float* __restrict__ U,
                                                                      float* __restrict__ U_hi,
                                                                      float* __restrict__ U_lo,
                                                                      int* info) {
  if (cta_info_set(info)) return;
  extern __shared__ __align__(16) float dsm[];
  float* S = dsm;                            // A, becoming R (upper)
  float* Ui = dsm + kTile * kDiagLd;         // U (upper, zeros below)
  float* T = dsm + 2 * kTile * kDiagLd;      // sums T_pq of the block rows of U still to come
  float* Pc = dsm + 3 * kTile * kDiagLd;     // warp 0's pivot columns
  __shared__ float rinv[kTile];
  __shared__ int bad;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b0 = k * kTile;
  const int b = min(kTile, d - b0);          // a multiple of 32
  const int np = b >> 5;
  {
    // all sixteen loads of this thread in flight before the first store
    constexpr int kPer = kTile * kTile / 4 / kDiagThreads;
    float4 v[kPer];
#pragma unroll
    for (int t = 0; t < kPer; ++t) {
      const int e = (tid + t * kDiagThreads) * 4, i = e >> 7, l = e & 127;
      v[t] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (i < b && l < b) v[t] = ld4(Rws + (long long)(b0 + i) * d + b0 + l);
    }
#pragma unroll
    for (int t = 0; t < kPer; ++t) {
      const int e = (tid + t * kDiagThreads) * 4, i = e >> 7, l = e & 127;
      st4(S + i * kDiagLd + l, v[t]);        // only entries i <= l are ever read
      st4(Ui + i * kDiagLd + l, make_float4(0.f, 0.f, 0.f, 0.f));
    }
  }
  if (tid == 0) bad = 0;
  __syncthreads();

  // Every thread runs the same barrier sequence whatever the data; a failed
  // pivot is reported at the end (the values are then meaningless).
  if (warp == 0) {
    for (int p = np - 1; p >= 0; --p) {
      if (p < np - 1) bar_sync(kBarDReady, kDReadyCount);
      const int fail = pivot_panel(S, Ui, Pc, rinv, p * 32, b0 + p * 32, lane);
      if (fail && lane == 0 && bad == 0) bad = fail;
      bar_arrive(kBarUReady, kDiagThreads);
    }
  } else {
    const int w = warp - 1;
    for (int p = np - 1; p >= 0; --p) {
      const int c0 = p * 32;
      bar_sync(kBarUReady, kDiagThreads);
      if (p > 0) {
        // panel R_ip = A_ip U_pp^T in place; lane = column j with row j of
        // U_pp in registers. Workers 0-3 take row block p-1 (the next
        // pivots need it), workers 4-6 the rows above.
        float bu[32];
        load_row32(Ui + c0 * kDiagLd + c0, lane, bu);
        const int first = w < kCritWarps ? (p - 1) * 4 + w : w - kCritWarps;
        const int last = w < kCritWarps ? first + 1 : (p - 1) * 4;
        const int step = w < kCritWarps ? 1 : kWorkers - kCritWarps;
        for (int unit = first; unit < last; unit += step) {
          float* A = S + (unit * 8) * kDiagLd + c0;
          float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
          unit_dot8(A, bu, acc);
          __syncwarp();
#pragma unroll
          for (int i = 0; i < 8; ++i) A[i * kDiagLd + lane] = acc[i];
        }
        if (w < kCritWarps) {
          // D_{p-1,p-1} -= R_{p-1,p} R_{p-1,p}^T, quarter w, then warp 0 may go on
          bar_sync(kBarCrit, 32 * kCritWarps);
          const int r0 = (p - 1) * 32 + w * 8;
          float br[32];
          load_row32(S + ((p - 1) * 32) * kDiagLd + c0, lane, br);   // row `lane` of R_{p-1,p}
          float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
          unit_dot8(S + r0 * kDiagLd + c0, br, acc);
          float* C = S + r0 * kDiagLd + (p - 1) * 32;
#pragma unroll
          for (int i = 0; i < 8; ++i) C[i * kDiagLd + lane] -= acc[i];
          bar_arrive(kBarDReady, kDReadyCount);
        }
        bar_sync(kBarWorkers, kWorkers * 32);   // every panel row is there
      }
      {
        // the other updates A_ij -= R_ip R_jp^T (i <= j < p, but not
        // (p-1, p-1)), then block row p of U: U_pq = -U_pp T_pq (q > p)
        const int n_upd = p > 0 ? (p * (p + 1) / 2 - 1) * 4 : 0;
        const int n_u = (np - 1 - p) * 4;
        for (int unit = w; unit < n_upd + n_u; unit += kWorkers) {
          float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
          if (unit < n_upd) {
            int ii, jj;
            tri_pair(unit >> 2, ii, jj);   // pairs below t = p(p+1)/2 - 1, i.e. all but (p-1, p-1)
            const int r0 = ii * 32 + (unit & 3) * 8;
            float br[32];
            load_row32(S + (jj * 32) * kDiagLd + c0, lane, br);   // row `lane` of R_jp
            unit_dot8(S + r0 * kDiagLd + c0, br, acc);
            float* C = S + r0 * kDiagLd + jj * 32;
#pragma unroll
            for (int i = 0; i < 8; ++i) C[i * kDiagLd + lane] -= acc[i];
          } else {
            const int u = unit - n_upd, q = p + 1 + (u >> 2), r0 = c0 + (u & 3) * 8;
            float bt[32];
            load_col32(T + c0 * kDiagLd + q * 32, lane, bt);      // column `lane` of T_pq
            unit_dot8(Ui + r0 * kDiagLd + c0, bt, acc);
#pragma unroll
            for (int i = 0; i < 8; ++i) Ui[(r0 + i) * kDiagLd + q * 32 + lane] = -acc[i];
          }
        }
      }
      bar_sync(kBarWorkers, kWorkers * 32);   // block row p of U is final
      {
        // T_iq += R_ip U_pq for i < p, q >= p (the first term, q == p,
        // starts the sum), and the store of rows c0..c0+31 of U
        const int n_t = p * (np - p) * 4;
        for (int unit = w; unit < n_t; unit += kWorkers) {
          const int pair = unit >> 2, i = pair / (np - p), q = p + pair % (np - p);
          const int r0 = i * 32 + (unit & 3) * 8;
          float bu2[32];
          load_col32(Ui + c0 * kDiagLd + q * 32, lane, bu2);    // column `lane` of U_pq
          float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
          unit_dot8(S + r0 * kDiagLd + c0, bu2, acc);
          float* C = T + r0 * kDiagLd + q * 32;
#pragma unroll
          for (int x = 0; x < 8; ++x) C[x * kDiagLd + lane] = (q == p ? 0.f : C[x * kDiagLd + lane]) + acc[x];
        }
        for (int e = tid - 32; e < 32 * (kTile / 4); e += kWorkers * 32) {
          const int i = c0 + (e >> 5), l = (e & 31) * 4;
          if (l >= b) continue;
          const float4 v = *reinterpret_cast<const float4*>(Ui + i * kDiagLd + l);
          const float4 h = make_float4(tf32_hi(v.x), tf32_hi(v.y), tf32_hi(v.z), tf32_hi(v.w));
          const long long off = (long long)(b0 + i) * d + b0 + l;
          st4(U + off, v);
          st4(U_hi + off, h);
          st4(U_lo + off, make_float4(v.x - h.x, v.y - h.y, v.z - h.z, v.w - h.w));
        }
      }
    }
  }
  __syncthreads();
  if (bad && tid == 0) set_info(info, bad);
}

// ------------------------------------------------------------- chain step
//
// Right after diag(s), on the critical chain: the next diagonal block is
// made ready without waiting for the panel product and the trailing update
// of block column s, which then run off the chain:
//   R_{s-1,s} = A_{s-1,s} U_ss^T           (its hi/lo planes replace the tile,
//                                           as the panel product does for the
//                                           rows above),
//   D = A_{s-1,s-1} - R_{s-1,s} R_{s-1,s}^T (upper triangle, in place).
// A_{s-1,s} is read from the hi/lo planes of block column s (hi + lo is the
// fp32 value exactly), so the in-place planes of R never race with a read.
// One CTA per 8 x 8 block (I, J), I <= J, of D (136 CTAs, one wave): it
// forms rows I and J of R_{s-1,s} itself in plain FP32 (U_ss has zeros
// below its diagonal, so each dot starts near the diagonal), then its block
// of D; the CTAs with I == J also write the planes of their 8 rows of R.
constexpr int kChainG = 8;
constexpr int kChainBlocks = kTile / kChainG;                       // 16
constexpr int kChainCtas = kChainBlocks * (kChainBlocks + 1) / 2;   // 136
constexpr int kChainThreads = 256;
constexpr int kChainLd = kTile + 4;                                 // 16-byte aligned rows
constexpr size_t kChainSmem = (size_t)(kTile + 4 * kChainG) * kChainLd * sizeof(float);

__global__ void __launch_bounds__(kChainThreads) chain_step_kernel(
    float* __restrict__ Rw, float* __restrict__ V_lo, const float* __restrict__ A_hi,
    const float* __restrict__ A_lo, const float* __restrict__ U, int d, int s, const int* info) {
  if (cta_info_set(info)) return;
  extern __shared__ __align__(16) float csm[];
  float* Us = csm;                                // U_ss rows j, columns l (zeros outside)
  float* As = csm + kTile * kChainLd;             // rows I then J of A_{s-1,s} (hi), then of R
  float* Al = As + 2 * kChainG * kChainLd;        // the same rows, lo plane
  const int tid = threadIdx.x;
  // blockIdx.x -> (I, J), I <= J, column by column
  int J = 0;
  while ((J + 1) * (J + 2) / 2 <= (int)blockIdx.x) ++J;
  const int I = (int)blockIdx.x - J * (J + 1) / 2;
  const int c0 = s * kTile, bk = min(kTile, d - c0), r0 = c0 - kTile;
  const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
  // this thread's entry of the D block (phase 2), fetched early
  const int o = tid >> 2, sl = tid & 3, da = o >> 3, db = o & 7;
  const bool d_out = sl == 0 && (I < J || da <= db);
  float* const d_ptr = Rw + (long long)(r0 + I * kChainG + da) * d + r0 + J * kChainG + db;
  const float a_old = d_out ? *d_ptr : 0.f;
  // U_ss (the chunks that reach the upper triangle) and both planes of the
  // 16 A rows, all copies in flight at once
#pragma unroll
  for (int q = 0; q < kTile * kTile / 4 / kChainThreads; ++q) {
    const int e = tid + q * kChainThreads, j = e >> 5, l = (e & 31) * 4;
    float* dst = Us + j * kChainLd + l;
    if (j < bk && l < bk && l + 4 > j) cp_async16(dst, U + (long long)(c0 + j) * d + c0 + l);
    else *reinterpret_cast<float4*>(dst) = zero;
  }
#pragma unroll
  for (int q = 0; q < 2 * kChainG * kTile / 4 / kChainThreads; ++q) {
    const int e = tid + q * kChainThreads, r = e >> 5, l = (e & 31) * 4;
    const int row = r0 + (r < kChainG ? I * kChainG + r : J * kChainG + r - kChainG);
    if (l < bk) {
      cp_async16(As + r * kChainLd + l, A_hi + (long long)row * kTile + l);
      cp_async16(Al + r * kChainLd + l, A_lo + (long long)row * kTile + l);
    } else {
      *reinterpret_cast<float4*>(As + r * kChainLd + l) = zero;
      *reinterpret_cast<float4*>(Al + r * kChainLd + l) = zero;
    }
  }
  cp_async_commit();
  cp_async_wait_all();
  __syncthreads();
  // A = hi + lo (exact)
#pragma unroll
  for (int q = 0; q < 2 * kChainG * kTile / 4 / kChainThreads; ++q) {
    const int e = tid + q * kChainThreads, r = e >> 5, l = (e & 31) * 4;
    float4* x = reinterpret_cast<float4*>(As + r * kChainLd + l);
    const float4 y = *reinterpret_cast<const float4*>(Al + r * kChainLd + l);
    const float4 v = *x;
    *x = make_float4(v.x + y.x, v.y + y.y, v.z + y.z, v.w + y.w);
  }
  __syncthreads();
  // R[r][j] = sum_l A[r][l] U[j][l]: thread -> column j and half h of the
  // l range, with U[j][64h..64h+64) in registers and the A rows read as
  // broadcasts; warps whose half of U_ss is below the diagonal (h = 0,
  // j >= 64) skip it. The h = 1 sums go through the lo-plane buffer, free by
  // then, and are added to the h = 0 ones.
  {
    const int w = tid >> 5, h = w & 1, j = ((w >> 1) << 5) | (tid & 31);
    float res[2 * kChainG];
#pragma unroll
    for (int r = 0; r < 2 * kChainG; ++r) res[r] = 0.f;
    if (h == 1 || j < 64) {   // warp-uniform
      float u[64];
      const float* ur = Us + j * kChainLd + 64 * h;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float4 v = *reinterpret_cast<const float4*>(ur + 4 * c);
        u[4 * c] = v.x; u[4 * c + 1] = v.y; u[4 * c + 2] = v.z; u[4 * c + 3] = v.w;
      }
#pragma unroll
      for (int r = 0; r < 2 * kChainG; ++r) {
        const float* ar = As + r * kChainLd + 64 * h;
        float p0 = 0.f, p1 = 0.f;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const float4 x = *reinterpret_cast<const float4*>(ar + 4 * c);
          p0 = fmaf(x.x, u[4 * c], p0);
          p1 = fmaf(x.y, u[4 * c + 1], p1);
          p0 = fmaf(x.z, u[4 * c + 2], p0);
          p1 = fmaf(x.w, u[4 * c + 3], p1);
        }
        res[r] = p0 + p1;
      }
    }
    if (h == 1) {
#pragma unroll
      for (int r = 0; r < 2 * kChainG; ++r) Al[r * kChainLd + j] = res[r];
    }
    __syncthreads();   // every thread is done reading the A rows
    if (h == 0) {
#pragma unroll
      for (int r = 0; r < 2 * kChainG; ++r) As[r * kChainLd + j] = res[r] + Al[r * kChainLd + j];
    }
  }
  __syncthreads();
  // planes of rows I of R (the diagonal CTAs), coalesced
  if (I == J) {
    for (int e = tid; e < kChainG * (kTile / 4); e += kChainThreads) {
      const int r = e >> 5, l = (e & 31) * 4;
      if (l >= bk) continue;
      const float4 v = *reinterpret_cast<const float4*>(As + r * kChainLd + l);
      const float4 h = make_float4(tf32_hi(v.x), tf32_hi(v.y), tf32_hi(v.z), tf32_hi(v.w));
      const long long off = (long long)(r0 + I * kChainG + r) * d + c0 + l;
      st4(Rw + off, h);
      st4(V_lo + off, make_float4(v.x - h.x, v.y - h.y, v.z - h.z, v.w - h.w));
    }
  }
  // D block: four threads per entry, a quarter of the K range each
  {
    const float* x = As + da * kChainLd;
    const float* y = As + (kChainG + db) * kChainLd;
    float s0 = 0.f, s1 = 0.f;
    for (int l = 32 * sl; l < min(32 * sl + 32, bk); l += 4) {
      const float4 p = *reinterpret_cast<const float4*>(x + l);
      const float4 q = *reinterpret_cast<const float4*>(y + l);
      s0 = fmaf(p.x, q.x, s0);
      s1 = fmaf(p.y, q.y, s1);
      s0 = fmaf(p.z, q.z, s0);
      s1 = fmaf(p.w, q.w, s1);
    }
    float t = s0 + s1;
    t += __shfl_xor_sync(0xffffffffu, t, 1);
    t += __shfl_xor_sync(0xffffffffu, t, 2);
    if (d_out) *d_ptr = a_old - t;
  }
}

// ----------------------------------------------------------------- driver

struct FactorWs {
  double* lam;
  float* R;        // H_d, then R; the hi plane of R_ik above the diagonal blocks
  float* V_lo;     // lo plane of R_ik (d x d)
  float* U_hi;     // hi/lo planes of U (d x d)
  float* U_lo;
  float* A_hi;     // hi/lo planes of the next column block of the updated H_d (d x 128)
  float* A_lo;
  float* T_hi;     // hi/lo planes of the next block row of the sums T (128 x d)
  float* T_lo;
};

static FactorWs carve_factor(void* ws, int d, size_t* bytes) {
  Carve c(ws);
  FactorWs w;
  w.lam = c.take<double>(4);
  w.R = c.take<float>((size_t)d * d);
  w.V_lo = c.take<float>((size_t)d * d);
  w.U_hi = c.take<float>((size_t)d * d);
  w.U_lo = c.take<float>((size_t)d * d);
  w.A_hi = c.take<float>((size_t)d * kTile);
  w.A_lo = c.take<float>((size_t)d * kTile);
  w.T_hi = c.take<float>((size_t)kTile * d);
  w.T_lo = c.take<float>((size_t)kTile * d);
  if (bytes) *bytes = c.off + 256;
  return w;
}

size_t factor_ws_bytes(int d) {
  size_t b = 0;
  carve_factor(nullptr, d, &b);
  return b;
}

namespace {

// The factorisation's internal streams (per device): the critical chain
// diag(k) -> chain step(k) -> diag(k-1) on `crit`; the panel product of
// the rows above and the update of block column k-1 on `pan`; the rest of
// each trailing update on `upd`; the block rows of U and the sums T they
// come from, which nothing in the chain waits for, on `rows`. They fork
// from and join back to the caller's stream, so the whole factorisation is
// ordered on it (and captures into one graph).
struct FactorStreams {
  cudaStream_t crit = nullptr, pan = nullptr, upd = nullptr, rows = nullptr;
  cudaEvent_t fork = nullptr, diag_done = nullptr, chain_done = nullptr, panel_done = nullptr,
              pan_done = nullptr, upd_done = nullptr;
  cudaEvent_t join[4] = {nullptr, nullptr, nullptr, nullptr};
};

std::mutex g_streams_mu;

cudaError_t factor_streams(FactorStreams** out) {
  static FactorStreams per_dev[64];
  static bool made[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  FactorStreams& f = per_dev[dev];
  if (!made[dev]) {
    int lo = 0, hi = 0;
    if ((e = cudaDeviceGetStreamPriorityRange(&lo, &hi)) != cudaSuccess) return e;
    if ((e = cudaStreamCreateWithPriority(&f.crit, cudaStreamNonBlocking, hi)) != cudaSuccess) return e;
    if ((e = cudaStreamCreateWithPriority(&f.pan, cudaStreamNonBlocking, hi)) != cudaSuccess) return e;
    if ((e = cudaStreamCreateWithPriority(&f.upd, cudaStreamNonBlocking, lo)) != cudaSuccess) return e;
    if ((e = cudaStreamCreateWithPriority(&f.rows, cudaStreamNonBlocking, lo)) != cudaSuccess) return e;
    cudaEvent_t* evs[] = {&f.fork,     &f.diag_done, &f.chain_done, &f.panel_done, &f.pan_done,
                          &f.upd_done, &f.join[0],   &f.join[1],    &f.join[2],    &f.join[3]};
    for (cudaEvent_t* ev : evs)
      if ((e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming)) != cudaSuccess) return e;
    made[dev] = true;
  }
  *out = &f;
  return cudaSuccess;
}

// s2 waits for everything enqueued on s1 so far.
cudaError_t after(cudaStream_t s2, cudaStream_t s1, cudaEvent_t ev) {
  cudaError_t e = cudaEventRecord(ev, s1);
  return e != cudaSuccess ? e : cudaStreamWaitEvent(s2, ev, 0);
}

// Off-chain GEMMs are persistent kernels that would otherwise hold every SM
// for their whole duration; they leave some to the chain's launches
// (d = 25,600: 78.2 ms with 132 CTAs, 78.3-79.2 with 140-148, 80.9 with
// 116, 85.2 with 100).
constexpr int kOffChainCtas = kNumSMs - 16;
// Steps per group of the trailing updates and the sums T, and the number of
// block columns from which they go by groups.
constexpr int kGroup = 4;
constexpr int kGroupFrom = 16;

// Upper tiles of the leading part are numbered column by column: tile
// (i, j), i <= j, is number j (j + 1) / 2 + i.
inline int tri_start(int j) { return j * (j + 1) / 2; }

// The block-column loop (see the file comment). Step k:
//   crit: diag(k); chain step(k) (R_{k-1,k} and the updated diagonal block
//         k-1), after the updates of the step before have written the tiles
//         it reads;
//   pan:  panel R_ik = A_ik U_kk^T for the rows i < k-1, then the update of
//         block column k-1 (rows above its diagonal block), which also
//         writes the planes the next panel reads;
//   upd:  the update of the block columns left of k-1;
//   rows: block row k of U, U_kq = -U_kk T_kq (q > k), then the step's
//         terms R_ik U_kq (i < k, q >= k) of the sums
//         T_iq = sum_{m=i+1..q} R_im U_mq: products over whole
//         rectangles above and right of block k (grouped, below). T lives in the
//         still-unused upper part of U (zero at the start); the product that
//         completes block row k-1 of T also writes its hi/lo planes, which
//         the next block row of U reads.
// From kGroupFrom block columns on, the steps go by groups of kGroup, k0
// down to L (the groups counted from the last block column; the final group
// ends at step 2 for the trailing updates and at step 1 for the sums T).
// Trailing updates: a step k > L applies its own panel (K = 128) to the
// group's block columns left of it, L .. k-1 (all but diagonal tile
// (k-1, k-1), which the chain step updates), and to the diagonal tile
// (L-1, L-1) that the chain step of L reads, writing the planes of block
// column k-1 for the next panel; step L applies all of the group's panels
// (K = up to 512) to block column L-1 above its diagonal tile and, off the
// chain, to every tile left of it. The tiles of the first launch are
// contiguous in the column-by-column numbering: (L-1, L-1) is the one just
// before column L. Sums T: a step k > L adds its term to the group's block
// rows below it (L .. k-1), which the group's next block rows of U need;
// step L adds all of the group's terms to the rows above the group, column
// block q of the group with the terms m <= q (U is upper triangular; its
// planes are not written below the diagonal) and the columns right of the
// group with all of them. So the bulk of the trailing matrix and of the
// sums is read and written once per kGroup block columns.
cudaError_t factor_blocks(const FactorWs& w, int d, float* U, int* info, const FactorStreams& f) {
  const int K = cdiv(d, kTile);
  const tc::Operand Ud{w.U_hi, w.U_lo, d, d, d};
  const tc::Operand Rp{w.R, w.V_lo, d, d, d};
  const tc::Operand Tp{w.T_hi, w.T_lo, kTile, d, d};
  const int G = K >= kGroupFrom ? kGroup : 1;
  cudaError_t e = cudaSuccess;
  bool pan_pending = false, upd_pending = false;
  for (int k = K - 1; k >= 0; --k) {
    const int c0 = k * kTile, bk = min(kTile, d - c0);
    diag_factor_kernel<<<1, kDiagThreads, kDiagSmem, f.crit>>>(w.R, d, k, U, w.U_hi, w.U_lo, info);
    count_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = cudaEventRecord(f.diag_done, f.crit)) != cudaSuccess) return e;
    if (k > 0) {
      // chain step: tiles (k-1, k) and (k-1, k-1) hold every earlier panel's
      // update once the last column update and the last bulk update are done
      if (pan_pending && (e = cudaStreamWaitEvent(f.crit, f.pan_done, 0)) != cudaSuccess) return e;
      if (upd_pending && (e = cudaStreamWaitEvent(f.crit, f.upd_done, 0)) != cudaSuccess) return e;
      chain_step_kernel<<<kChainCtas, kChainThreads, kChainSmem, f.crit>>>(w.R, w.V_lo, w.A_hi, w.A_lo, U, d,
                                                                            k, info);
      count_launches(1);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
      if ((e = cudaEventRecord(f.chain_done, f.crit)) != cudaSuccess) return e;
    }
    if (k >= 2) {   // block 0 is all the chain step of k = 1 touches
      const int k0 = k + (K - 1 - k) % G;              // the group's first step
      const int L = std::max(k0 - G + 1, 2);           // its last step with trailing updates
      const bool last = k == L;
      // K of this step's updates: panel k, or at the group's last step all
      // of the group's panels (the last block may be narrower than 128)
      const int kp = last ? std::min((k0 + 1) * kTile, d) - c0 : bk;
      const tc::Operand P{w.R + c0, w.V_lo + c0, c0, kp, d};
      {
        // panel R_ik = A_ik U_kk^T for i < k-1, as hi/lo planes (hi over R,
        // lo into V_lo)
        if ((e = cudaStreamWaitEvent(f.pan, f.diag_done, 0)) != cudaSuccess) return e;
        const tc::Operand A{w.A_hi, w.A_lo, c0, bk, kTile};
        const tc::Operand B{w.U_hi + (long long)c0 * d + c0, w.U_lo + (long long)c0 * d + c0, bk, bk, d};
        tc::Job job{};
        job.mode = 0;
        job.mt = k - 1;
        job.nt = 1;
        job.kdim = bk;
        job.ldc = d;
        job.c_col0 = c0;
        job.Mlim = c0 - kTile;
        job.Nlim = bk;
        job.alpha = 1.f;
        job.C_hi = w.R;
        job.C_lo = w.V_lo;
        job.max_ctas = kOffChainCtas;
        if ((e = tc::launch_gemm(A, B, false, job, k - 1, info, f.pan)) != cudaSuccess) return e;
        if ((e = cudaEventRecord(f.panel_done, f.pan)) != cudaSuccess) return e;
      }
      {
        // a step before the group's last: the group's block columns left of
        // it and diagonal tile (L-1, L-1), with the planes of block column
        // k-1 for the next panel; the last step: block column k-1 above its
        // diagonal tile, with its planes
        if ((e = cudaStreamWaitEvent(f.pan, f.chain_done, 0)) != cudaSuccess) return e;
        tc::Job job{};
        job.mode = 1;
        job.kdim = kp;
        job.t0 = last ? tri_start(k - 1) : tri_start(L) - 1;
        const int n_tiles = last ? k - 1 : tri_start(k) - tri_start(L);
        job.C = w.R;
        job.ldc = d;
        job.Mlim = job.Nlim = c0;
        job.alpha = -1.f;
        job.beta = 1.f;
        job.C_hi = w.A_hi;
        job.C_lo = w.A_lo;
        job.ldp = kTile;
        job.p_col0 = c0 - kTile;
        job.planes_one_col = last ? 0 : 1;
        job.planes_n0 = c0 - kTile;
        job.max_ctas = kOffChainCtas;
        if ((e = tc::launch_gemm(P, P, false, job, n_tiles, info, f.pan)) != cudaSuccess) return e;
        if ((e = cudaEventRecord(f.pan_done, f.pan)) != cudaSuccess) return e;
        pan_pending = true;
      }
      if (last) {
        // the block columns left of k-1
        if ((e = cudaStreamWaitEvent(f.upd, f.panel_done, 0)) != cudaSuccess) return e;
        tc::Job job{};
        job.mode = 1;
        job.kdim = kp;
        job.C = w.R;
        job.ldc = d;
        job.Mlim = job.Nlim = c0;
        job.alpha = -1.f;
        job.beta = 1.f;
        job.max_ctas = kOffChainCtas;
        if ((e = tc::launch_gemm(P, P, false, job, tri_start(k - 1), info, f.upd)) != cudaSuccess) return e;
        if ((e = cudaEventRecord(f.upd_done, f.upd)) != cudaSuccess) return e;
        upd_pending = true;
      }
    }
    // rows: U_kq = -U_kk T_kq for q > k (T's block row k is complete: its
    // last term came from step k+1, on this stream)
    if ((e = cudaStreamWaitEvent(f.rows, f.diag_done, 0)) != cudaSuccess) return e;
    if (k < K - 1) {
      tc::Job job{};
      job.mode = 0;
      job.mt = 1;
      job.nt = K - 1 - k;
      job.kdim = kTile;
      job.a_x0 = job.a_y0 = c0;
      job.b_x0 = c0 + kTile;
      job.C = U;
      job.ldc = d;
      job.c_row0 = c0;
      job.c_col0 = c0 + kTile;
      job.Mlim = kTile;
      job.Nlim = d - c0 - kTile;
      job.alpha = -1.f;
      job.C_hi = w.U_hi;
      job.C_lo = w.U_lo;
      job.max_ctas = kOffChainCtas;
      if ((e = tc::launch_gemm(Ud, Tp, true, job, K - 1 - k, info, f.rows)) != cudaSuccess) return e;
    }
    if (k > 0) {
      // T_iq += R_ik U_kq for i < k, q >= k (rows [0, c0), columns [c0, d)),
      // with the planes of T's block row k-1, which this term completes.
      // Grouped steps (see above): a step before the group's last adds its
      // term to the group's rows below it; the last adds all of the group's
      // terms to the rows above the group.
      if ((e = cudaStreamWaitEvent(f.rows, f.chain_done, 0)) != cudaSuccess) return e;
      if (k >= 2 && (e = cudaStreamWaitEvent(f.rows, f.panel_done, 0)) != cudaSuccess) return e;
      const int k0 = k + (K - 1 - k) % G;
      const int LT = std::max(k0 - G + 1, 1);
      auto t_job = [&](int row0, int rows, int col0, int cols, int kdim) {
        tc::Job job{};
        job.mode = 0;
        job.mt = rows / kTile;
        job.nt = cdiv(cols, kTile);
        job.kdim = kdim;
        job.a_x0 = c0;
        job.a_y0 = row0;
        job.b_x0 = col0;
        job.b_y0 = c0;
        job.C = U;
        job.ldc = d;
        job.c_row0 = row0;
        job.c_col0 = col0;
        job.Mlim = rows;
        job.Nlim = cols;
        job.alpha = 1.f;
        job.beta = 1.f;
        job.C_hi = w.T_hi;
        job.C_lo = w.T_lo;
        job.ldp = d;
        job.p_row0 = c0 - kTile;
        job.planes_one_row = 1;
        job.planes_m0 = c0 - kTile - row0;
        job.max_ctas = kOffChainCtas;
        return tc::launch_gemm(Rp, Ud, true, job, job.mt * job.nt, info, f.rows);
      };
      if (k > LT) {
        const int r0 = LT * kTile;
        if ((e = t_job(r0, c0 - r0, c0, d - c0, bk)) != cudaSuccess) return e;
      } else {
        // column block q of the group takes the terms m = k .. q; the columns
        // from block k0 on take all of them
        for (int q = k; q < k0; ++q)
          if ((e = t_job(0, c0, q * kTile, kTile, (q + 1) * kTile - c0)) != cudaSuccess) return e;
        const int ck0 = k0 * kTile;
        if ((e = t_job(0, c0, ck0, d - ck0, std::min((k0 + 1) * kTile, d) - c0)) != cudaSuccess) return e;
      }
    }
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_factor(const float* H, long long n_total, int d, float damp, float* U, void* ws,
                          int* info, cudaStream_t st) {
  const int K = cdiv(d, kTile);
  const FactorWs w = carve_factor(ws, d, nullptr);
  std::lock_guard<std::mutex> lock(g_streams_mu);
  static PerDevice attrs;
  cudaError_t e = once_per_device(attrs, [] {
    cudaError_t r = cudaFuncSetAttribute(diag_factor_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kDiagSmem);
    return r != cudaSuccess ? r
                            : cudaFuncSetAttribute(chain_step_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   (int)kChainSmem);
  });
  if (e != cudaSuccess) return e;
  FactorStreams* f = nullptr;
  e = factor_streams(&f);
  if (e != cudaSuccess) return e;
  const double scale = 2.0 / (double)n_total;
  damp_lambda_kernel<<<1, 1024, 0, st>>>(H, d, scale, (double)damp, w.lam, info);
  count_launches(1);
  // scaled, damped H into R; U zeroed in the same pass unless it is H; the
  // planes of the last column block above its diagonal block
  scale_damp_kernel<<<dim3(cdiv(d, 4 * 128), d), 128, 0, st>>>(H, w.R, d, scale, w.lam, info,
                                                               U != H ? U : nullptr, w.A_hi, w.A_lo,
                                                               K > 1 ? (K - 1) * kTile : -1);
  count_launches(1);
  if (U == H && (e = cudaMemsetAsync(U, 0, (size_t)d * d * sizeof(float), st)) != cudaSuccess) return e;
  if ((e = cudaEventRecord(f->fork, st)) != cudaSuccess) return e;
  for (cudaStream_t s : {f->crit, f->pan, f->upd, f->rows})
    if ((e = cudaStreamWaitEvent(s, f->fork, 0)) != cudaSuccess) return e;
  e = factor_blocks(w, d, U, info, *f);
  // always join, also after an error, so that a capture stays well formed
  const cudaStream_t side[4] = {f->crit, f->pan, f->upd, f->rows};
  for (int i = 0; i < 4; ++i) {
    const cudaError_t e2 = after(st, side[i], f->join[i]);
    if (e == cudaSuccess) e = e2;
  }
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace sgpt
