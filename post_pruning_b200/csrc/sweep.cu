// The blocked OBS column sweep (SparseGPT review, sections 八 and 十一).
//
// Per block of `bw` <= 128 columns starting at i1:
//   1. (unstructured) exact k-selection of the block's smallest saliencies
//      over all d_out rows: radix select on a 64-bit key (saliency bits, then
//      row * bw + column), one cooperative launch of select_kernel with a
//      grid barrier per 8-bit digit;
//   2. sweep_kernel: one warp per row, one 4-column group per lane; the
//      groups are processed in order: mask decision (N:M at each group start
//      on the compensated weights), e = (w_q - p_q) / U_qq (as a product with
//      the reciprocal), rank-4 update of the rest of the block with the U
//      rows held in shared memory;
//   3. W[:, i2:] -= Err * U[i1:i2, i2:] as FP32-accurate tensor-core GEMMs
//      (three TF32 products on hi/lo planes of Err and U, gemm_tc.cu): at
//      once for the rest of the block's group of blocks, once per group for
//      the columns right of it (launch_prune).
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <mutex>

#include "common.cuh"
#include "gemm_simt.cuh"
#include "gemm_tc.h"
#include "kernels.h"

namespace sgpt {

// ---------------------------------------------------------------- sweep

constexpr int kSweepWarps = 8;             // warps per CTA
constexpr int kSweepThreads = kSweepWarps * 32;
constexpr size_t kSweepSmem = (size_t)kMaxBlock * kMaxBlock * sizeof(float);

// kModeNM4: N of every 4 (2:4 on the hot path); kModeNMG: N of every M for
// M = 8 .. 128; kModeThreshold: unstructured, prune keys below a threshold
// found by select_kernel; kModeForced: the mask is an input.
enum SweepMode { kModeNM4 = 0, kModeThreshold = 1, kModeForced = 2, kModeNMG = 3 };

// The value of x on a row's quantization grid: scale * (clip(rint(x / scale)
// + zero, 0, maxq) - zero); the code is decided in fp32 with ties to even.
__device__ __forceinline__ float quant_value(float x, float scale, float zero, float maxq) {
  const float c = fminf(fmaxf(rintf(__fdiv_rn(x, scale)) + zero, 0.f), maxq);
  return __fmul_rn(scale, c - zero);
}

__device__ __forceinline__ unsigned long long sal_key(float w, float inv_u, unsigned idx) {
  return ((unsigned long long)__float_as_uint(saliency(w, inv_u)) << 32) | idx;
}

// ROWS rows per warp, 32/ROWS lanes per row; lane l of a row owns the
// 4-column groups l, l + 32/ROWS, ... of its row (an N:M group never
// straddles two lanes; the interleave keeps every shared-memory row read of
// the warp contiguous).
// Groups are taken in order. For group g every lane of the row receives the
// owner lane's four weights, decides the group's mask (2:4: on the
// compensated weights, at the group start) and computes its four errors in
// column order with the in-group updates, all lanes alike; the owner keeps
// the result and applies the group's update to its own later group, and
// every lane right of it applies the rank-4 update to its columns.
// Arithmetically this is the column-by-column sweep with the updates of the
// four columns to the columns right of the group summed together. The chain
// per group is one shuffle, the four in-group steps and one rank-4 update;
// the U values are loaded before the weights arrive. Several rows per warp
// (four for tall layers, two for N:M with M > 4) cut the repeated owner work
// per row; one row per warp gives more parallelism to short layers.
// N:M with M > 4 (kModeNMG): at the first column of each group of M the
// lanes holding the group's columns rank them by saliency on the weights as
// compensated so far (every later column has received the updates of every
// earlier group by then): each member lane receives the group's M
// saliencies by shuffle and counts, for each of its own columns, the group
// columns that beat it (larger saliency, or equal and lower column); the N
// best are kept. An M-group covers M/4 consecutive lanes of one column span,
// or, when M is wider than a span, every lane of M/span consecutive spans.
// The group steps then apply the decided bits like a forced mask.
//
// QUANT (joint sparsification and quantization, SparseGPT review sections
// 十五 and 十七): a kept weight is replaced by its value on the row's grid
// (qgrid[2 * row] = scale, qgrid[2 * row + 1] = zero point) when its column
// is reached, and (w - value) / U_qq is compensated like a pruning error.
template <int MODE, int ROWS, int M, bool QUANT>
__global__ void __launch_bounds__(kSweepThreads) sweep_kernel(
    float* __restrict__ W, long long ldw, int rows, int d, int i1, int bw,
    const float* __restrict__ U, uint32_t* __restrict__ mask, float* __restrict__ row_loss,
    float* __restrict__ Err, float* __restrict__ Err_lo, int err_ld, const unsigned long long* __restrict__ thr,
    int nkeep, const float* __restrict__ qgrid, float qmaxq, int* info) {
  constexpr int LPR = 32 / ROWS;                 // lanes per row
  constexpr int CPL = 4 * ROWS;                  // columns per lane
  if (cta_info_set(info)) return;
  extern __shared__ float Us[];   // [128][128]: U[i1 + a][i1 + b]
  __shared__ float Uinv[kMaxBlock];   // 1 / U_qq of the block's columns
  const int tid = threadIdx.x;
  // U block to shared memory with asynchronous 16-byte copies, all in
  // flight at once (rows are 16-byte aligned: i1 and d are multiples of 32)
  for (int e = tid * 4; e < kMaxBlock * kMaxBlock; e += kSweepThreads * 4) {
    const int a = e >> 7, b = e & 127;
    if (a < bw && b < bw)
      cp_async16(Us + e, U + (long long)(i1 + a) * d + i1 + b);
    else
      st4(Us + e, make_float4(0.f, 0.f, 0.f, 0.f));
  }
  cp_async_commit();
  if (tid < kMaxBlock) Uinv[tid] = tid < bw ? 1.0f / U[(long long)(i1 + tid) * d + i1 + tid] : 0.f;

  const int lane = tid & 31;
  const int sub = lane / LPR, sl = lane % LPR;   // row within the warp, lane within the row
  const int base = sub * LPR;                    // first lane of this row
  const int row = (blockIdx.x * kSweepWarps + (tid >> 5)) * ROWS + sub;
  constexpr int SPAN = 4 * LPR;                  // columns between a lane's groups
  const bool live = row < rows;
  const bool mine = live;
  const int c0 = 4 * sl;                         // block-relative first column of group v: c0 + v * SPAN
  float* wrow = W + (long long)row * ldw + i1 + c0;
  float w[CPL], err[CPL];
#pragma unroll
  for (int j = 0; j < CPL; ++j) {
    w[j] = 0.f;
    err[j] = 0.f;
  }
  if (mine) {
#pragma unroll
    for (int v = 0; v < ROWS; ++v) {
      if (c0 + v * SPAN < bw) {
        const float4 x = ld4(wrow + v * SPAN);
        w[4 * v] = x.x; w[4 * v + 1] = x.y; w[4 * v + 2] = x.z; w[4 * v + 3] = x.w;
      }
    }
  }
  bool bad = false;
#pragma unroll
  for (int j = 0; j < CPL; ++j) bad |= !isfinite(w[j]);
  uint32_t keep = (1u << CPL) - 1u;
  if (MODE == kModeForced && mine) {
    keep = 0;
#pragma unroll
    for (int v = 0; v < ROWS; ++v) {
      const int c = c0 + v * SPAN;
      if (c < bw) {
        const uint32_t word = mask[(long long)row * (d / 32) + (i1 + c) / 32];
        keep |= ((word >> ((i1 + c) & 31)) & 0xfu) << (4 * v);
      }
    }
  }
  cp_async_wait_all();
  __syncthreads();
  if (MODE == kModeThreshold && mine) {
    const unsigned long long t = *thr;
    keep = 0;
#pragma unroll
    for (int j = 0; j < CPL; ++j) {
      const int c = c0 + (j >> 2) * SPAN + (j & 3);
      const unsigned idx = (unsigned)row * (unsigned)bw + (unsigned)c;
      if (c < bw && sal_key(w[j], Uinv[c], idx) >= t) keep |= 1u << j;
    }
  }
  float qs = 1.f, qz = 0.f;
  if (QUANT && mine) {
    qs = qgrid[2 * (long long)row];
    qz = qgrid[2 * (long long)row + 1];
  }
  float loss = 0.f;
  // keep bit j of every lane, for the threshold and forced modes
  uint32_t kb[CPL];
#pragma unroll
  for (int j = 0; j < CPL; ++j) kb[j] = __ballot_sync(0xffffffffu, (keep >> j) & 1u);

#pragma unroll
  for (int gi = 0; gi < ROWS; ++gi) {
    const int gend = min(LPR, (bw - gi * SPAN) / 4);   // groups of this column span inside the block
#pragma unroll 1
    for (int gp = 0; gp < gend; ++gp) {
      const int q0 = gi * SPAN + 4 * gp;         // the group's first column (group order = column order)
      const int owner = base + gp;
      // U values that do not depend on the weights first: the group's four
      // rows at this lane's columns, its in-group entries, the reciprocals
      float4 ur[4][ROWS];
#pragma unroll
      for (int t = 0; t < 4; ++t)
#pragma unroll
        for (int v = 0; v < ROWS; ++v)
          ur[t][v] = (v >= gi) ? ld4(Us + (q0 + t) * kMaxBlock + c0 + v * SPAN) : make_float4(0.f, 0.f, 0.f, 0.f);
      const float4 g0 = ld4(Us + (q0 + 0) * kMaxBlock + q0);
      const float4 g1 = ld4(Us + (q0 + 1) * kMaxBlock + q0);
      const float4 g2 = ld4(Us + (q0 + 2) * kMaxBlock + q0);
      const float4 ri = ld4(Uinv + q0);
      float wo[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) wo[t] = __shfl_sync(0xffffffffu, w[4 * gi + t], owner);
      const float r[4] = {ri.x, ri.y, ri.z, ri.w};
      if (MODE == kModeNMG && (q0 & (M - 1)) == 0) {
        // decide the M-group that starts here
        constexpr int NSPAN = (M > SPAN) ? M / SPAN : 1;    // column spans the group covers
        constexpr int NL = (M > SPAN) ? LPR : M / 4;        // lanes it covers in each span
        const int gl0 = (M > SPAN) ? 0 : (q0 - gi * SPAN) / 4;   // its first lane (row-relative)
        const bool member = sl >= gl0 && sl < gl0 + NL;
        float ms[4 * NSPAN];
        int rk[4 * NSPAN];
#pragma unroll
        for (int vv = 0; vv < NSPAN; ++vv)
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int v = (gi + vv < ROWS) ? gi + vv : gi;
            ms[4 * vv + t] = saliency(w[4 * v + t], Uinv[c0 + v * SPAN + t]);
            rk[4 * vv + t] = 0;
          }
#pragma unroll 1
        for (int k = 0; k < NL; ++k) {
          const int src = base + gl0 + k;
#pragma unroll
          for (int vv = 0; vv < NSPAN; ++vv)
#pragma unroll
            for (int t2 = 0; t2 < 4; ++t2) {
              const float so = __shfl_sync(0xffffffffu, ms[4 * vv + t2], src);
              const int co = (gi + vv) * SPAN + 4 * (gl0 + k) + t2;
#pragma unroll
              for (int vm = 0; vm < NSPAN; ++vm)
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                  const int mc = (gi + vm) * SPAN + c0 + t;
                  const float mv = ms[4 * vm + t];
                  if (so > mv || (so == mv && co < mc)) ++rk[4 * vm + t];
                }
            }
        }
        if (mine && member) {
#pragma unroll
          for (int vm = 0; vm < NSPAN; ++vm)
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              const int j = 4 * (gi + vm) + t;
              if (j < CPL) keep = (keep & ~(1u << j)) | ((rk[4 * vm + t] < nkeep ? 1u : 0u) << j);
            }
        }
#pragma unroll
        for (int j = 0; j < CPL; ++j) kb[j] = __ballot_sync(0xffffffffu, (keep >> j) & 1u);
      }
      uint32_t km;
      if (MODE == kModeNM4) {
        // N of 4 on the compensated weights; ties keep the lower column.
        float slv[4];
#pragma unroll
        for (int t = 0; t < 4; ++t) slv[t] = saliency(wo[t], r[t]);
        km = 0;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          int rank = 0;   // how many of the group beat column t
#pragma unroll
          for (int o = 0; o < 4; ++o)
            if (o != t && (slv[o] > slv[t] || (slv[o] == slv[t] && o < t))) ++rank;
          if (rank < nkeep) km |= 1u << t;
        }
      } else {
        km = 0;
#pragma unroll
        for (int t = 0; t < 4; ++t) km |= ((kb[4 * gi + t] >> owner) & 1u) << t;
      }
      float e[4];
      if constexpr (QUANT) {
        // a kept weight becomes its grid value; the difference is
        // compensated like a pruning error
        float pq[4];
        pq[0] = (km & 1u) ? quant_value(wo[0], qs, qz, qmaxq) : 0.f;
        e[0] = __fmul_rn(__fsub_rn(wo[0], pq[0]), r[0]);
        wo[1] = fmaf(-e[0], g0.y, wo[1]);
        wo[2] = fmaf(-e[0], g0.z, wo[2]);
        wo[3] = fmaf(-e[0], g0.w, wo[3]);
        pq[1] = (km & 2u) ? quant_value(wo[1], qs, qz, qmaxq) : 0.f;
        e[1] = __fmul_rn(__fsub_rn(wo[1], pq[1]), r[1]);
        wo[2] = fmaf(-e[1], g1.z, wo[2]);
        wo[3] = fmaf(-e[1], g1.w, wo[3]);
        pq[2] = (km & 4u) ? quant_value(wo[2], qs, qz, qmaxq) : 0.f;
        e[2] = __fmul_rn(__fsub_rn(wo[2], pq[2]), r[2]);
        wo[3] = fmaf(-e[2], g2.w, wo[3]);
        pq[3] = (km & 8u) ? quant_value(wo[3], qs, qz, qmaxq) : 0.f;
        e[3] = __fmul_rn(__fsub_rn(wo[3], pq[3]), r[3]);
#pragma unroll
        for (int t = 0; t < 4; ++t) wo[t] = pq[t];
      } else {
        e[0] = (km & 1u) ? 0.f : __fmul_rn(wo[0], r[0]);
        wo[1] = fmaf(-e[0], g0.y, wo[1]);
        wo[2] = fmaf(-e[0], g0.z, wo[2]);
        wo[3] = fmaf(-e[0], g0.w, wo[3]);
        e[1] = (km & 2u) ? 0.f : __fmul_rn(wo[1], r[1]);
        wo[2] = fmaf(-e[1], g1.z, wo[2]);
        wo[3] = fmaf(-e[1], g1.w, wo[3]);
        e[2] = (km & 4u) ? 0.f : __fmul_rn(wo[2], r[2]);
        wo[3] = fmaf(-e[2], g2.w, wo[3]);
        e[3] = (km & 8u) ? 0.f : __fmul_rn(wo[3], r[3]);
      }
      if (sl == gp) {
        // the owner keeps its group's result
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          w[4 * gi + t] = ((km >> t) & 1u) ? wo[t] : 0.f;
          err[4 * gi + t] = e[t];
          loss = fmaf(e[t], e[t], loss);
        }
        keep = (keep & ~(0xfu << (4 * gi))) | (km << (4 * gi));
      }
      // the rank-4 update of every column right of the group: this lane's
      // later groups (v > gi) always, group gi if the lane is right of the owner
#pragma unroll
      for (int v = 0; v < ROWS; ++v) {
        if (v > gi || (v == gi && sl > gp)) {
          w[4 * v + 0] = fmaf(-e[3], ur[3][v].x, fmaf(-e[2], ur[2][v].x, fmaf(-e[1], ur[1][v].x, fmaf(-e[0], ur[0][v].x, w[4 * v + 0]))));
          w[4 * v + 1] = fmaf(-e[3], ur[3][v].y, fmaf(-e[2], ur[2][v].y, fmaf(-e[1], ur[1][v].y, fmaf(-e[0], ur[0][v].y, w[4 * v + 1]))));
          w[4 * v + 2] = fmaf(-e[3], ur[3][v].z, fmaf(-e[2], ur[2][v].z, fmaf(-e[1], ur[1][v].z, fmaf(-e[0], ur[0][v].z, w[4 * v + 2]))));
          w[4 * v + 3] = fmaf(-e[3], ur[3][v].w, fmaf(-e[2], ur[2][v].w, fmaf(-e[1], ur[1][v].w, fmaf(-e[0], ur[0][v].w, w[4 * v + 3]))));
        }
      }
    }
  }

  // Loss of the row: sum over its lanes.
  float tot = loss;
#pragma unroll
  for (int o = 1; o < LPR; o <<= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
  bad |= !isfinite(tot);
  // Mask words: for each of its groups v, lanes 8m .. 8m+7 of a row hold the
  // columns of word (v * SPAN) / 32 + m.
  uint32_t bits[ROWS];
#pragma unroll
  for (int v = 0; v < ROWS; ++v) {
    bits[v] = mine ? ((keep >> (4 * v)) & 0xfu) << (4 * (sl & 7)) : 0u;
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) bits[v] |= __shfl_xor_sync(0xffffffffu, bits[v], o);
  }
  if (mine) {
#pragma unroll
    for (int v = 0; v < ROWS; ++v) {
      const int c = c0 + v * SPAN;
      if (c >= bw) continue;
      st4(wrow + v * SPAN, make_float4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]));
      float ev[4] = {err[4 * v], err[4 * v + 1], err[4 * v + 2], err[4 * v + 3]};
      if (Err_lo) {
        // hi/lo planes for the tensor-core trailing update
        float lo[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float h = tf32_hi(ev[j]);
          lo[j] = ev[j] - h;
          ev[j] = h;
        }
        st4(Err_lo + (long long)row * err_ld + c, make_float4(lo[0], lo[1], lo[2], lo[3]));
      }
      st4(Err + (long long)row * err_ld + c, make_float4(ev[0], ev[1], ev[2], ev[3]));
      if (MODE != kModeForced && (sl & 7) == 0) mask[(long long)row * (d / 32) + (i1 + c) / 32] = bits[v];
    }
    if (sl == 0 && row_loss) row_loss[row] += tot;
    if (bad) set_info(info, SGPT_INFO_NONFINITE);
  }
}

// Rows per warp for a layer: four for tall layers (every lane of a row
// repeats the owner group's decision and in-group steps, so fewer lanes per
// row means fewer instructions per row), one for short ones (more warps in
// flight). N:M with M > 4 takes at most two (see launch_sweep_m).
static int sweep_rows_per_warp(int rows) { return rows >= 2048 ? 4 : 1; }

template <int MODE, int M, bool QUANT>
static cudaError_t launch_sweep_m(int rpw, float* W, long long ldw, int rows, int d, int i1, int bw, const float* U,
                                  uint32_t* mask, float* row_loss, float* Err, float* Err_lo, int err_ld,
                                  const unsigned long long* thr, int nkeep, const float* qgrid, float qmaxq,
                                  int* info, cudaStream_t st) {
  // N:M with M > 4 stays at two rows per warp: at four its decision
  // registers leave one CTA per SM and the sweep measured slower (16:64)
  constexpr bool kFour = MODE != kModeNMG;
  static PerDevice attrs;
  const cudaError_t ea = once_per_device(attrs, [] {
    cudaError_t r = cudaFuncSetAttribute(sweep_kernel<MODE, 1, M, QUANT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSweepSmem);
    if (r == cudaSuccess)
      r = cudaFuncSetAttribute(sweep_kernel<MODE, 2, M, QUANT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)kSweepSmem);
    if (r == cudaSuccess && kFour)
      r = cudaFuncSetAttribute(sweep_kernel<MODE, kFour ? 4 : 2, M, QUANT>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSweepSmem);
    return r;
  });
  if (ea != cudaSuccess) return ea;
  if (!kFour && rpw > 2) rpw = 2;
  const int grid = cdiv(rows, kSweepWarps * rpw);
  if (rpw == 4)
    sweep_kernel<MODE, kFour ? 4 : 2, M, QUANT><<<grid, kSweepThreads, kSweepSmem, st>>>(
        W, ldw, rows, d, i1, bw, U, mask, row_loss, Err, Err_lo, err_ld, thr, nkeep, qgrid, qmaxq, info);
  else if (rpw == 2)
    sweep_kernel<MODE, 2, M, QUANT><<<grid, kSweepThreads, kSweepSmem, st>>>(
        W, ldw, rows, d, i1, bw, U, mask, row_loss, Err, Err_lo, err_ld, thr, nkeep, qgrid, qmaxq, info);
  else
    sweep_kernel<MODE, 1, M, QUANT><<<grid, kSweepThreads, kSweepSmem, st>>>(
        W, ldw, rows, d, i1, bw, U, mask, row_loss, Err, Err_lo, err_ld, thr, nkeep, qgrid, qmaxq, info);
  count_launches(1);
  return cudaGetLastError();
}

template <bool QUANT>
static cudaError_t launch_sweep_q(const sgpt_params& p, int rpw, float* W, long long ldw, int rows, int d, int i1,
                                  int bw, const float* U, uint32_t* mask, float* row_loss, float* Err,
                                  float* Err_lo, int err_ld, const unsigned long long* thr, const float* qgrid,
                                  int* info, cudaStream_t st) {
  const float qmaxq = QUANT ? (float)((1 << p.qbits) - 1) : 0.f;
#define SGPT_SWEEP(MODE, M)                                                                                  \
  launch_sweep_m<MODE, M, QUANT>(rpw, W, ldw, rows, d, i1, bw, U, mask, row_loss, Err, Err_lo, err_ld, thr, p.n, \
                                 qgrid, qmaxq, info, st)
  if (p.forced) return SGPT_SWEEP(kModeForced, 4);
  if (p.pattern != SGPT_PATTERN_NM) return SGPT_SWEEP(kModeThreshold, 4);
  switch (p.m) {
    case 4: return SGPT_SWEEP(kModeNM4, 4);
    case 8: return SGPT_SWEEP(kModeNMG, 8);
    case 16: return SGPT_SWEEP(kModeNMG, 16);
    case 32: return SGPT_SWEEP(kModeNMG, 32);
    case 64: return SGPT_SWEEP(kModeNMG, 64);
    case 128: return SGPT_SWEEP(kModeNMG, 128);
  }
#undef SGPT_SWEEP
  return cudaErrorInvalidValue;
}

// The sweep of one block for a pattern: forced mask, unstructured threshold,
// N of 4, or N of M = 8 .. 128; with or without quantization of the kept
// weights (qgrid: the per-row grid, when p.qbits > 0).
static cudaError_t launch_sweep(const sgpt_params& p, int rpw, float* W, long long ldw, int rows, int d, int i1,
                                int bw, const float* U, uint32_t* mask, float* row_loss, float* Err, float* Err_lo,
                                int err_ld, const unsigned long long* thr, const float* qgrid, int* info,
                                cudaStream_t st) {
  if (p.qbits > 0)
    return launch_sweep_q<true>(p, rpw, W, ldw, rows, d, i1, bw, U, mask, row_loss, Err, Err_lo, err_ld, thr, qgrid,
                                info, st);
  return launch_sweep_q<false>(p, rpw, W, ldw, rows, d, i1, bw, U, mask, row_loss, Err, Err_lo, err_ld, thr, nullptr,
                               info, st);
}

// ------------------------------------------------------ quantization grid

// One warp per row: the range of the dense row widened to include 0 (a row
// of zeros takes [-1, 1]); scale = (hi - lo) / maxq and zero =
// rint(-lo / scale), in fp32.
__global__ void __launch_bounds__(256) quant_grid_kernel(const float* __restrict__ W, long long ldw, int rows, int d,
                                                        float maxq, float* __restrict__ grid) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= rows) return;
  const float* w = W + (long long)row * ldw;
  float lo = 0.f, hi = 0.f;
  for (int c = 4 * lane; c < d; c += 128) {
    const float4 x = ld4(w + c);
    lo = fminf(lo, fminf(fminf(x.x, x.y), fminf(x.z, x.w)));
    hi = fmaxf(hi, fmaxf(fmaxf(x.x, x.y), fmaxf(x.z, x.w)));
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if (lane == 0) {
    if (lo == hi) {
      lo = -1.f;
      hi = 1.f;
    }
    const float scale = __fdiv_rn(__fsub_rn(hi, lo), maxq);
    grid[2 * (long long)row] = scale;
    grid[2 * (long long)row + 1] = rintf(__fdiv_rn(-lo, scale));
  }
}

cudaError_t launch_quant_grid(const float* W, long long ldw, int rows, int d, int bits, float* grid,
                              cudaStream_t st) {
  quant_grid_kernel<<<cdiv(rows, 8), 256, 0, st>>>(W, ldw, rows, d, (float)((1 << bits) - 1), grid);
  count_launches(1);
  return cudaGetLastError();
}

// --------------------------------------------------------- trailing update

// W[:, i2:] -= Err[:, :bw] * U[i1:i1+bw, i2:]
__global__ void __launch_bounds__(kGemmThreads) trailing_kernel(
    float* __restrict__ W, long long ldw, int rows, int d, int i1, int bw,
    const float* __restrict__ U, const float* __restrict__ Err, const int* info) {
  if (cta_info_set(info)) return;
  extern __shared__ float smem[];
  const int i2 = i1 + bw;
  const int n0 = i2 + blockIdx.x * kTile;
  const int m0 = blockIdx.y * kTile;
  float acc[8][8];
  zero_acc(acc);
  const OpKContig A{Err, kMaxBlock, m0, rows - m0, bw};
  const OpIContig B{U + (long long)i1 * d, d, n0, d - n0, bw};
  gemm_tile(A, B, 0, bw, acc, smem);
  store_tile(W + (long long)m0 * ldw + n0, ldw, rows - m0, d - n0, acc, -1.f, 1.f);
}

// ------------------------------------------------ unstructured selection

struct SelState {
  unsigned long long thr;      // pruned iff key < thr
  unsigned int arrive;         // grid barrier counter
  unsigned int pad;
  unsigned int hist[8][256];   // one histogram per digit pass
};

constexpr int kSelThreads = 1024;

__device__ __forceinline__ unsigned int ld_acquire(const unsigned int* p) {
  unsigned int v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Barrier over the whole grid (the launch is cooperative, so every CTA is
// resident). The wait is bounded by `limit` SM clock cycles: on timeout the
// CTA records SGPT_INFO_TIMEOUT and the caller returns (a CTA still waiting
// elsewhere gives up on its own limit; none waits on one that returned).
__device__ bool grid_sync(unsigned int* ctr, unsigned int target, int* info, int* failed, long long limit) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(ctr, 1u);
    const long long t0 = clock64();
    while (ld_acquire(ctr) < target) {
      if (clock64() - t0 > limit) {
        set_info(info, SGPT_INFO_TIMEOUT);
        *failed = 1;
        break;
      }
      __nanosleep(64);
    }
    __threadfence();
  }
  __syncthreads();
  return *failed == 0;
}

// Exact k-selection over the block's d_out x bw saliency keys in one
// cooperative launch: a radix select on the 64-bit key, one 8-bit digit per
// pass, most significant first (four passes on the saliency bits, four on
// the index that breaks ties). Each pass histograms the digit of the keys
// that match the prefix fixed so far; after a grid barrier every CTA scans
// the same global histogram and takes the same decision, so a pass needs one
// barrier. It stops as soon as the rank falls on a whole bin (usually after
// the saliency passes). The first pass scores the weights and keeps each
// CTA's saliency bits in shared memory for the later passes (when they fit;
// otherwise every pass rescores W); the index of quad e's element j is
// 4e + j. st must be zeroed before the launch; CTA 0 writes the threshold.
__global__ void __launch_bounds__(kSelThreads) select_kernel(
    const float* __restrict__ W, long long ldw, int rows, int d, int i1, int bw,
    const float* __restrict__ U, SelState* st, unsigned int k, int keep_bits, int* info, long long wait_cycles) {
  if (cta_info_set(info)) return;
  extern __shared__ unsigned int skey[];        // this CTA's saliency bits, if keep_bits
  __shared__ unsigned int h[256];
  __shared__ float ud[kMaxBlock];
  __shared__ unsigned int wsum[kSelThreads / 32];
  __shared__ unsigned long long s_prefix;
  __shared__ unsigned int s_krem;
  __shared__ int s_done, s_failed;
  const int t = threadIdx.x;
  if (t < bw) ud[t] = 1.0f / U[(long long)(i1 + t) * d + i1 + t];   // same reciprocal as the sweep
  if (t == 0) {
    s_prefix = 0;
    s_krem = k;
    s_done = (k == 0);
    s_failed = 0;
  }
  const long long total4 = (long long)rows * (bw / 4);
  for (int pass = 0; pass < 8; ++pass) {
    if (t < 256) h[t] = 0;
    __syncthreads();
    if (s_done) break;
    const int shift = 56 - 8 * pass;
    const unsigned long long prefix = s_prefix;
    // trip count uniform across the CTA: every lane takes part in the match
    int it = 0;
    for (long long base = (long long)blockIdx.x * kSelThreads; base < total4;
         base += (long long)gridDim.x * kSelThreads, ++it) {
      const long long e = base + t;
      const bool act = e < total4;
      unsigned int sb[4] = {0u, 0u, 0u, 0u};
      if (act) {
        if (pass > 0 && keep_bits) {
          const uint4 x = *reinterpret_cast<const uint4*>(skey + 4 * (it * kSelThreads + t));
          sb[0] = x.x; sb[1] = x.y; sb[2] = x.z; sb[3] = x.w;
        } else {
          const int row = (int)(e / (bw / 4));
          const int c = (int)(e - (long long)row * (bw / 4)) * 4;
          const float4 x = ld4(W + (long long)row * ldw + i1 + c);
          const float v[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) sb[j] = (unsigned int)(sal_key(v[j], ud[c + j], 0u) >> 32);
          if (pass == 0 && keep_bits)
            *reinterpret_cast<uint4*>(skey + 4 * (it * kSelThreads + t)) = make_uint4(sb[0], sb[1], sb[2], sb[3]);
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const unsigned long long key = act ? (((unsigned long long)sb[j] << 32) | (unsigned long long)(4 * e + j)) : 0ull;
        const bool mine = act && (pass == 0 || (key >> (shift + 8)) == prefix);
        // saliencies span a narrow exponent range, so a warp holds few
        // distinct digits: one shared atomic per digit and warp
        const unsigned bin = mine ? (unsigned)((key >> shift) & 255u) : 256u;
        const unsigned peers = __match_any_sync(0xffffffffu, bin);
        if (mine && (t & 31) == (__ffs(peers) - 1)) atomicAdd(&h[bin], (unsigned)__popc(peers));
      }
    }
    __syncthreads();
    if (t < 256 && h[t]) atomicAdd(&st->hist[pass][t], h[t]);
    if (!grid_sync(&st->arrive, (unsigned)(pass + 1) * gridDim.x, info, &s_failed, wait_cycles)) return;
    // every CTA: inclusive scan of the 256 bins and the bin holding rank k
    const unsigned int cnt = (t < 256) ? __ldcg(&st->hist[pass][t]) : 0u;
    unsigned int inc = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned int y = __shfl_up_sync(0xffffffffu, inc, o);
      if ((t & 31) >= o) inc += y;
    }
    if ((t & 31) == 31) wsum[t >> 5] = inc;
    __syncthreads();
    for (int w = 0; w < (t >> 5); ++w) inc += wsum[w];
    const unsigned int kr = s_krem;
    const unsigned int exc = inc - cnt;
    __syncthreads();                          // everyone has read s_krem
    if (t < 256 && cnt > 0 && exc < kr && kr <= inc) {
      const unsigned int krem = kr - exc;
      const unsigned long long pre = (prefix << 8) | (unsigned long long)t;
      s_prefix = pre;
      s_krem = krem;
      if (cnt == krem) {
        s_done = 1;
        if (blockIdx.x == 0) st->thr = (pre << shift) + (1ull << shift);   // every key of the bin is pruned
      }
    }
    __syncthreads();
  }
}

constexpr int kSelMaxSmem = 160 * 1024;         // bytes of saliency bits a CTA keeps

static cudaError_t launch_select(const float* W, long long ldw, int rows, int d, int i1, int bw, const float* U,
                                 SelState* sel, unsigned int k, int* info, cudaStream_t st) {
  static PerDevice attrs;
  static int max_grid_dev[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if ((e = once_per_device(attrs, [dev] {
         cudaError_t r = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSelMaxSmem);
         if (r != cudaSuccess) return r;
         int per_sm = 0, sms = 0;
         if ((r = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, select_kernel, kSelThreads, kSelMaxSmem)) !=
             cudaSuccess)
           return r;
         if ((r = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return r;
         max_grid_dev[dev] = std::max(1, std::min(per_sm, 1) * sms);   // one CTA per SM: fewer histogram merges
         return cudaSuccess;
       })) != cudaSuccess)
    return e;
  const int max_grid = max_grid_dev[dev];
  if ((e = cudaMemsetAsync(sel, 0, sizeof(SelState), st)) != cudaSuccess) return e;
  const long long total4 = (long long)rows * (bw / 4);
  const int grid = (int)std::max<long long>(1, std::min<long long>(cdivll(total4, kSelThreads), max_grid));
  const long long iters = cdivll(total4, (long long)grid * kSelThreads);
  const long long bytes = iters * kSelThreads * 16;
  const int keep_bits = bytes <= kSelMaxSmem ? 1 : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kSelThreads);
  cfg.dynamicSmemBytes = keep_bits ? (size_t)bytes : 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, select_kernel, W, ldw, rows, d, i1, bw, U, sel, k, keep_bits, info,
                         wait_limit_cycles());
  count_launches(1);
  return e;
}

// ----------------------------------------------------------------- driver

// The trailing update is applied in two parts. The columns of the blocks
// still to come in the current group (as many whole blocks as fit in
// kGroupCols columns) get each block's error right after its sweep (K = one
// block), since the next sweep reads them; every column right of the group
// gets the errors of the whole group at once when the group ends (K = the
// group's width). Each column receives the same sum of error-times-U terms
// as with one update per block (the lazy batch update of the pages, batched
// over more blocks), in another order; the trailing matrix is read and
// written once per group instead of once per block.
constexpr int kGroupCols = 4 * kMaxBlock;

struct PruneWs {
  float* Err_hi;   // error blocks of the current group, hi/lo planes (d_out x kGroupCols)
  float* Err_lo;
  float* U_hi;     // hi/lo planes of U (d_in x d_in)
  float* U_lo;
  SelState* sel;
  float* qgrid;    // per-row quantization grid (scale, zero), d_out x 2
};
constexpr int kErrLd = kGroupCols;

static PruneWs carve_prune(void* ws, int d_out, int d_in, size_t* bytes) {
  Carve c(ws);
  PruneWs w;
  w.Err_hi = c.take<float>((size_t)d_out * kErrLd);
  w.Err_lo = c.take<float>((size_t)d_out * kErrLd);
  w.U_hi = c.take<float>((size_t)d_in * d_in);
  w.U_lo = c.take<float>((size_t)d_in * d_in);
  w.sel = c.take<SelState>(1);
  w.qgrid = c.take<float>((size_t)d_out * 2);
  if (bytes) *bytes = c.off + 256;
  return w;
}

size_t prune_ws_bytes(int d_out, int d_in) {
  size_t b = 0;
  carve_prune(nullptr, d_out, d_in, &b);
  return b;
}

// W[:, c0:c1] -= Err[:, e0:e0+k] U[u0:u0+k, c0:c1] (FP32-accurate GEMM).
static cudaError_t trailing_update(const tc::Operand& Ep, const tc::Operand& Up, float* W, long long ldw, int rows,
                                   int e0, int u0, int k, int c0, int c1, int* info, cudaStream_t st) {
  if (c1 <= c0 || k <= 0) return cudaSuccess;
  tc::Job job{};
  job.mode = 0;
  job.mt = cdiv(rows, kTile);
  job.nt = cdiv(c1 - c0, kTile);
  job.kdim = k;
  job.a_x0 = e0;
  job.b_x0 = c0;
  job.b_y0 = u0;
  job.C = W;
  job.ldc = ldw;
  job.c_col0 = c0;
  job.Mlim = rows;
  job.Nlim = c1 - c0;
  job.alpha = -1.f;
  job.beta = 1.f;
  return tc::launch_gemm(Ep, Up, true, job, job.mt * job.nt, info, st);
}

cudaError_t launch_prune(float* W, int rows, int d, long long ldw, const float* U,
                         const sgpt_params& p, uint32_t* mask, float* row_loss, void* ws,
                         int* info, cudaStream_t st) {
  const PruneWs w = carve_prune(ws, rows, d, nullptr);
  cudaError_t e = tc::launch_split(U, d, d, d, w.U_hi, w.U_lo, d, info, st);
  if (e != cudaSuccess) return e;
  // the quantization grid of the dense rows, before any column is touched
  const float* qgrid = p.qgrid;
  if (p.qbits > 0 && !qgrid) {
    if ((e = launch_quant_grid(W, ldw, rows, d, p.qbits, w.qgrid, st)) != cudaSuccess) return e;
    qgrid = w.qgrid;
  }
  const tc::Operand Ep{w.Err_hi, w.Err_lo, rows, kErrLd, kErrLd};
  const tc::Operand Up{w.U_hi, w.U_lo, d, d, d};
  const int B = p.blocksize;
  const int rpw = sweep_rows_per_warp(rows);
  const int gw = kGroupCols / B * B;                      // columns per group: whole blocks
  for (int g1 = 0; g1 < d; g1 += gw) {
    const int g2 = std::min(d, g1 + gw);                  // the group's columns [g1, g2)
    for (int i1 = g1; i1 < g2; i1 += B) {
      const int bw = min(B, d - i1), i2 = i1 + bw;
      const int slot = i1 - g1;                           // this block's columns of the error buffer
      if (!p.forced && p.pattern == SGPT_PATTERN_UNSTRUCTURED) {
        const double kk = std::floor((double)p.sparsity * (double)rows * (double)bw);
        if ((e = launch_select(W, ldw, rows, d, i1, bw, U, w.sel, (unsigned int)kk, info, st)) != cudaSuccess)
          return e;
      }
      e = launch_sweep(p, rpw, W, ldw, rows, d, i1, bw, U, mask, row_loss, w.Err_hi + slot, w.Err_lo + slot,
                       kErrLd, &w.sel->thr, qgrid, info, st);
      if (e != cudaSuccess) return e;
      // the group's later blocks need this block's error before their sweeps
      if ((e = trailing_update(Ep, Up, W, ldw, rows, slot, i1, bw, i2, g2, info, st)) != cudaSuccess) return e;
    }
    // the columns right of the group: all of the group's errors at once
    if ((e = trailing_update(Ep, Up, W, ldw, rows, 0, g1, g2 - g1, g2, d, info, st)) != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

// ------------------------------------------------ allocation-free variant
//
// sgpt_prune needs scratch for the error block of the current OBS block
// (d_out x 128 fp32) and for the selection state. The allocation-free entry
// takes that scratch from the fixed device array below instead of a caller
// workspace. Every device that loads this library holds the array until the
// process exits. All calls share it, so calls that overlap on the GPU (two
// streams, or two host threads) race; nothing in it has to start at zero
// (the error block is written before it is read and the selection state is
// re-initialised for every block).

constexpr size_t kNoAllocErrBytes = (size_t)SGPT_NOALLOC_MAX_ROWS * kMaxBlock * sizeof(float);
constexpr size_t kNoAllocScratchBytes = kNoAllocErrBytes + 16384;
static_assert(sizeof(SelState) <= 16384, "selection state must fit the scratch tail");

static __device__ __align__(256) unsigned char g_prune_scratch[kNoAllocScratchBytes];

// In host code g_prune_scratch names a host-side stand-in, not device memory;
// the device address must come from cudaGetSymbolAddress with the device
// current. It is looked up once per device, on the first call there.
static std::mutex g_scratch_mu;
static void* g_scratch_addr[256];

static cudaError_t prune_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 256) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_prune_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

cudaError_t launch_prune_noalloc(float* W, int rows, int d, long long ldw, const float* U,
                                 const sgpt_params& p, uint32_t* mask, float* row_loss, int* info,
                                 cudaStream_t st) {
  if (rows > SGPT_NOALLOC_MAX_ROWS) return cudaErrorInvalidValue;
  void* base = nullptr;
  cudaError_t e = prune_scratch(&base);
  if (e != cudaSuccess) return e;
  float* Err = static_cast<float*>(base);
  SelState* sel = reinterpret_cast<SelState*>(static_cast<char*>(base) + kNoAllocErrBytes);
  const int B = p.blocksize;
  const int rpw = sweep_rows_per_warp(rows);
  for (int i1 = 0; i1 < d; i1 += B) {
    const int bw = min(B, d - i1);
    if (!p.forced && p.pattern == SGPT_PATTERN_UNSTRUCTURED) {
      const double kk = std::floor((double)p.sparsity * (double)rows * (double)bw);
      if ((e = launch_select(W, ldw, rows, d, i1, bw, U, sel, (unsigned int)kk, info, st)) != cudaSuccess)
        return e;
    }
    e = launch_sweep(p, rpw, W, ldw, rows, d, i1, bw, U, mask, row_loss, Err, nullptr, kMaxBlock, &sel->thr, p.qgrid,
                     info, st);
    if (e != cudaSuccess) return e;
    const int i2 = i1 + bw;
    if (i2 < d) {
      dim3 grid(cdiv(d - i2, kTile), cdiv(rows, kTile));
      trailing_kernel<<<grid, kGemmThreads, kGemmSmemBytes, st>>>(W, ldw, rows, d, i1, bw, U, Err, info);
      count_launches(1);
    }
  }
  return cudaGetLastError();
}

}  // namespace sgpt
