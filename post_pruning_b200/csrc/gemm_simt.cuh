// FP32 SIMT tile core: one 256-thread CTA accumulates a 128x128 tile
// C(m, n) = sum_k A(m, k) * B(k, n) in registers (8x8 per thread).
//
// Used where the arithmetic must stay FP32-accurate: the trailing update of
// the OBS sweep, the panel / rank-k / triangular-inverse products of the
// factorisation and the reconstruction-error product. Operands are staged
// through shared memory in k-chunks of 16, double-buffered through registers;
// every operand form below loads 16-byte vectors along its contiguous axis.
#pragma once

#include "common.cuh"

namespace sgpt {

constexpr int kGemmThreads = 256;
constexpr int kGemmBK = 16;
constexpr int kGemmLds = kTile + 4;   // padded row of the staged tiles
constexpr size_t kGemmSmemBytes = 2 * 2 * kGemmBK * kGemmLds * sizeof(float);

// Staged tile: s[k][m] (A) or s[k][n] (B), 16 x (128 + 4) floats.
using Stage = float[kGemmBK][kGemmLds];

// ---- operand forms -------------------------------------------------------
// Each form gives the element (i, k) of a 128-wide operand tile, where i is
// the tile row (m for A, n for B), from a row-major buffer.

// Element (i, k) at p[(i0 + i) * ld + k]: k contiguous ("row form" for A,
// "transposed form" for B). i < I valid rows, k < K valid (K % 4 == 0).
struct OpKContig {
  const float* p;
  long long ld;
  int i0, I, K;
  // thread t fetches rows t/4 and 64 + t/4, k-quad (t%4)*4
  __device__ __forceinline__ void fetch(int k0, float4 (&r)[2]) const {
    const int t = threadIdx.x;
    const int kk = k0 + (t & 3) * 4;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int i = (t >> 2) + 64 * h;
      if (i < I && kk < K) r[h] = ld4(p + (long long)(i0 + i) * ld + kk);
      else r[h] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  __device__ __forceinline__ void stash(Stage& s, const float4 (&r)[2]) const {
    const int t = threadIdx.x;
    const int kq = (t & 3) * 4;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int i = (t >> 2) + 64 * h;
      s[kq + 0][i] = r[h].x;
      s[kq + 1][i] = r[h].y;
      s[kq + 2][i] = r[h].z;
      s[kq + 3][i] = r[h].w;
    }
  }
};

// Element (i, k) at p[k * ld + i0 + i]: i contiguous ("column form" for A,
// "row form" for B). I % 4 == 0.
struct OpIContig {
  const float* p;
  long long ld;
  int i0, I, K;
  // thread t fetches k rows t/32 and 8 + t/32, i-quad (t%32)*4
  __device__ __forceinline__ void fetch(int k0, float4 (&r)[2]) const {
    const int t = threadIdx.x;
    const int i = (t & 31) * 4;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int k = k0 + (t >> 5) + 8 * h;
      if (i < I && k < K) r[h] = ld4(p + (long long)k * ld + i0 + i);
      else r[h] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  __device__ __forceinline__ void stash(Stage& s, const float4 (&r)[2]) const {
    const int t = threadIdx.x;
    const int i = (t & 31) * 4;
#pragma unroll
    for (int h = 0; h < 2; ++h) st4(&s[(t >> 5) + 8 * h][i], r[h]);
  }
};

// Element (i, k) = p[(i0+i)*ld + k] - q[(i0+i)*ld + k] (k contiguous): the
// weight change dW = W0 - W read on the fly by the reconstruction error.
struct OpKContigDiff {
  const float* p;
  const float* q;
  long long ld;
  int i0, I, K;
  __device__ __forceinline__ void fetch(int k0, float4 (&r)[2]) const {
    const int t = threadIdx.x;
    const int kk = k0 + (t & 3) * 4;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int i = (t >> 2) + 64 * h;
      if (i < I && kk < K) {
        const long long o = (long long)(i0 + i) * ld + kk;
        float4 a = ld4(p + o), b = ld4(q + o);
        r[h] = make_float4(a.x - b.x, a.y - b.y, a.z - b.z, a.w - b.w);
      } else {
        r[h] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  }
  __device__ __forceinline__ void stash(Stage& s, const float4 (&r)[2]) const {
    OpKContig{nullptr, 0, 0, 0, 0}.stash(s, r);
  }
};

// ---- main loop -------------------------------------------------------------
// acc[a][b]: thread (ty, tx) = (tid/16, tid%16) holds rows
// m = ty*4 + (a&3) + 64*(a>>2) and columns n = tx*4 + (b&3) + 64*(b>>2).
template <class OA, class OB>
__device__ __forceinline__ void gemm_tile(const OA& A, const OB& B, int k_begin, int k_end,
                                          float (&acc)[8][8], float* smem) {
  Stage* sA = reinterpret_cast<Stage*>(smem);
  Stage* sB = sA + 2;
  const int t = threadIdx.x;
  const int ty = t >> 4, tx = t & 15;
  float4 ra[2], rb[2];
  if (k_begin >= k_end) return;
  A.fetch(k_begin, ra);
  B.fetch(k_begin, rb);
  A.stash(sA[0], ra);
  B.stash(sB[0], rb);
  __syncthreads();
  int buf = 0;
  for (int k0 = k_begin; k0 < k_end; k0 += kGemmBK) {
    const bool more = k0 + kGemmBK < k_end;
    if (more) {
      A.fetch(k0 + kGemmBK, ra);
      B.fetch(k0 + kGemmBK, rb);
    }
#pragma unroll
    for (int k = 0; k < kGemmBK; ++k) {
      float a[8], b[8];
      const float4 a0 = ld4(&sA[buf][k][ty * 4]);
      const float4 a1 = ld4(&sA[buf][k][64 + ty * 4]);
      const float4 b0 = ld4(&sB[buf][k][tx * 4]);
      const float4 b1 = ld4(&sB[buf][k][64 + tx * 4]);
      a[0] = a0.x; a[1] = a0.y; a[2] = a0.z; a[3] = a0.w;
      a[4] = a1.x; a[5] = a1.y; a[6] = a1.z; a[7] = a1.w;
      b[0] = b0.x; b[1] = b0.y; b[2] = b0.z; b[3] = b0.w;
      b[4] = b1.x; b[5] = b1.y; b[6] = b1.z; b[7] = b1.w;
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    if (more) {
      A.stash(sA[buf ^ 1], ra);
      B.stash(sB[buf ^ 1], rb);
    }
    __syncthreads();
    buf ^= 1;
  }
}

__device__ __forceinline__ void zero_acc(float (&acc)[8][8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
}

__device__ __forceinline__ int acc_row(int a) { return (threadIdx.x >> 4) * 4 + (a & 3) + 64 * (a >> 2); }
__device__ __forceinline__ int acc_col(int h) { return (threadIdx.x & 15) * 4 + 64 * h; }

// C[m0 + row][n0 + col] = alpha * acc + beta * C (rows < M, 4-column groups
// with col < N; N % 4 == 0). beta == 0 does not read C.
__device__ __forceinline__ void store_tile(float* C, long long ldc, int M, int N,
                                           const float (&acc)[8][8], float alpha, float beta) {
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    const int m = acc_row(a);
    if (m >= M) continue;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int n = acc_col(h);
      if (n >= N) continue;
      float* p = C + (long long)m * ldc + n;
      float4 v = make_float4(alpha * acc[a][4 * h + 0], alpha * acc[a][4 * h + 1],
                             alpha * acc[a][4 * h + 2], alpha * acc[a][4 * h + 3]);
      if (beta != 0.f) {
        const float4 o = ld4(p);
        v.x = fmaf(beta, o.x, v.x);
        v.y = fmaf(beta, o.y, v.y);
        v.z = fmaf(beta, o.z, v.z);
        v.w = fmaf(beta, o.w, v.w);
      }
      st4(p, v);
    }
  }
}

}  // namespace sgpt
