// 2:4 and N:M packing and the layer reconstruction error.
//
// Packing follows the 2:4 production guide (oh-bug.com, section on the 2:4
// mechanism): of every four consecutive weights along the input dimension two
// are kept, stored in column order, and their positions are recorded as
// 2-bit indices. The N:M formats of the sparse fine-tuning review
// (tqpw.cn, section 八 8.4: 16:32, 16:64, 16:128) keep N of every M and
// record each kept position in log2(M) bits the same way.
#include <cuda_runtime.h>

#include "common.cuh"
#include "gemm_simt.cuh"
#include "kernels.h"

namespace sgpt {

// One thread per (row, 32 columns): 8 groups, one mask word, one meta word,
// 32 weights in, 16 values out.
__global__ void __launch_bounds__(256) pack24_kernel(const float* __restrict__ W, long long ldw,
                                                     int rows, int d,
                                                     const uint32_t* __restrict__ mask,
                                                     float* __restrict__ values,
                                                     uint32_t* __restrict__ meta, int* info) {
  if (info_set(info)) return;
  const int wpr = d / 32;
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= (long long)rows * wpr) return;
  const int row = (int)(t / wpr), wd = (int)(t - (long long)row * wpr);
  const uint32_t m = mask[t];
  const float* src = W + (long long)row * ldw + wd * 32;
  float* dst = values + (long long)row * (d / 2) + wd * 16;
  uint32_t code = 0;
  bool bad = false;
#pragma unroll
  for (int g2 = 0; g2 < 4; ++g2) {           // two groups per float4 pair
    float out[4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int g = 2 * g2 + h;
      const uint32_t nib = (m >> (4 * g)) & 0xfu;
      const float4 x = ld4(src + 4 * g);
      bad |= __popc(nib) != 2;
      const int a = __ffs(nib) - 1;                  // lowest kept
      const int b = 31 - __clz(nib);                 // highest kept
      const int aa = a < 0 ? 0 : a, bb = b < 0 ? 0 : b;
      out[2 * h] = aa == 0 ? x.x : aa == 1 ? x.y : aa == 2 ? x.z : x.w;
      out[2 * h + 1] = bb == 0 ? x.x : bb == 1 ? x.y : bb == 2 ? x.z : x.w;
      code |= (uint32_t)((aa | (bb << 2)) & 0xf) << (4 * g);
    }
    st4(dst + 4 * g2, make_float4(out[0], out[1], out[2], out[3]));
  }
  meta[t] = code;
  if (bad) set_info(info, SGPT_INFO_BAD_MASK);
}

cudaError_t launch_pack24(const float* W, long long ldw, int rows, int d, const uint32_t* mask,
                          float* values, uint32_t* meta, int* info, cudaStream_t st) {
  const long long n = (long long)rows * (d / 32);
  pack24_kernel<<<(unsigned)cdivll(n, 256), 256, 0, st>>>(W, ldw, rows, d, mask, values, meta, info);
  count_launches(1);
  return cudaGetLastError();
}

// General N:M packing: one thread per (row, group of M). The group's mask
// bits (M <= 32: part of one word; M = 64, 128: whole words) give the kept
// positions in column order; kept value j of group g goes to value g*N + j
// of the row and its position (log2(M) bits) to bit offset (g*N + j) *
// log2(M) of the row's metadata bits, least significant first. Positions
// that continue into the next word, and words shared between groups, are
// merged with atomicOr into metadata the launcher zeroed (OR is order-free:
// the result is deterministic).
__global__ void __launch_bounds__(256) packnm_kernel(const float* __restrict__ W, long long ldw, int rows, int d,
                                                     const uint32_t* __restrict__ mask, int n, int m, int lg,
                                                     int meta_words, float* __restrict__ values,
                                                     uint32_t* __restrict__ meta, int* info) {
  if (info_set(info)) return;
  const int groups = d / m;
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= (long long)rows * groups) return;
  const int row = (int)(t / groups), g = (int)(t - (long long)row * groups);
  const uint32_t* mrow = mask + (long long)row * (d / 32);
  const float* wrow = W + (long long)row * ldw + (long long)g * m;
  float* vrow = values + (long long)row * (d / m) * n;
  uint32_t* meta_row = meta + (long long)row * meta_words;
  int cnt = 0;
  for (int w0 = 0; w0 < m; w0 += 32) {
    const int c = g * m + w0;                       // first column of this 32-bit slice
    uint32_t bitsw = mrow[c >> 5] >> (c & 31);
    if (m < 32) bitsw &= (1u << m) - 1u;
    while (bitsw) {
      const int pos = w0 + __ffs(bitsw) - 1;          // in-group position, ascending
      bitsw &= bitsw - 1u;
      if (cnt < n) {
        const long long k = (long long)g * n + cnt;
        vrow[k] = wrow[pos];
        const long long off = k * lg;
        const int word = (int)(off >> 5), sh = (int)(off & 31);
        atomicOr(meta_row + word, (uint32_t)pos << sh);
        if (sh + lg > 32) atomicOr(meta_row + word + 1, (uint32_t)pos >> (32 - sh));
      }
      ++cnt;
    }
  }
  if (cnt != n) set_info(info, SGPT_INFO_BAD_MASK);
}

int packnm_meta_words(int d, int n, int m) {
  int lg = 0;
  while ((1 << lg) < m) ++lg;
  const long long bits = (long long)(d / m) * n * lg;
  return (int)((bits + 31) / 32);
}

cudaError_t launch_packnm(const float* W, long long ldw, int rows, int d, const uint32_t* mask, int n, int m,
                          float* values, uint32_t* meta, int* info, cudaStream_t st) {
  int lg = 0;
  while ((1 << lg) < m) ++lg;
  const int words = packnm_meta_words(d, n, m);
  cudaError_t e = cudaMemsetAsync(meta, 0, (size_t)rows * words * sizeof(uint32_t), st);
  if (e != cudaSuccess) return e;
  const long long threads = (long long)rows * (d / m);
  packnm_kernel<<<(unsigned)cdivll(threads, 256), 256, 0, st>>>(W, ldw, rows, d, mask, n, m, lg, words, values,
                                                                 meta, info);
  count_launches(1);
  return cudaGetLastError();
}

// ------------------------------------------------- reconstruction error

// partial[tile] = sum over the tile of (A H)[m][n] * A[m][n], A = W0 - W
// (diff) or W0; one partial per CTA, summed in a fixed order afterwards, so
// the result is deterministic to the last bit.
template <class OA>
__global__ void __launch_bounds__(kGemmThreads) quad_form_kernel(OA A, const float* __restrict__ H,
                                                                 int d, const float* __restrict__ P,
                                                                 const float* __restrict__ Q,
                                                                 long long ldw, int rows,
                                                                 double* __restrict__ partial) {
  extern __shared__ float smem[];
  __shared__ double red[kGemmThreads / 32];
  const int m0 = blockIdx.x * kTile, n0 = blockIdx.y * kTile;   // row tiles on x: up to 2^17 of them
  A.i0 = m0;
  A.I = rows - m0;
  float acc[8][8];
  zero_acc(acc);
  const OpIContig B{H, d, n0, d - n0, d};
  gemm_tile(A, B, 0, d, acc, smem);
  double s = 0.0;
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    const int m = m0 + acc_row(a);
    if (m >= rows) continue;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int n = n0 + acc_col(h);
      if (n >= d) continue;
      const long long o = (long long)m * ldw + n;
      float4 p = ld4(P + o);
      if (Q) {
        const float4 q = ld4(Q + o);
        p.x -= q.x; p.y -= q.y; p.z -= q.z; p.w -= q.w;
      }
      s += (double)acc[a][4 * h + 0] * p.x + (double)acc[a][4 * h + 1] * p.y +
           (double)acc[a][4 * h + 2] * p.z + (double)acc[a][4 * h + 3] * p.w;
    }
  }
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < kGemmThreads / 32; ++w) t += red[w];
    partial[(long long)blockIdx.x * gridDim.y + blockIdx.y] = t;
  }
}

// out[q] = sum of partial[q * n .. q * n + n) for q = 0, 1 (one CTA per q):
// each thread sums a fixed stride of the partials, then a fixed tree.
constexpr int kSumThreads = 1024;
__global__ void __launch_bounds__(kSumThreads) recon_sum_kernel(const double* __restrict__ partial,
                                                                long long n, double* __restrict__ out) {
  __shared__ double red[kSumThreads];
  const double* p = partial + blockIdx.x * n;
  double s = 0.0;
  for (long long i = threadIdx.x; i < n; i += kSumThreads) s += p[i];
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = kSumThreads / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) out[blockIdx.x] = red[0];
}

size_t recon_ws_bytes(int rows, int d) {
  return 2 * (size_t)cdiv(d, kTile) * (size_t)cdiv(rows, kTile) * sizeof(double) + 256;
}

cudaError_t launch_recon(const float* W0, const float* W, int rows, int d, long long ldw,
                         const float* H, double* num_den, void* ws, cudaStream_t st) {
  dim3 grid(cdiv(rows, kTile), cdiv(d, kTile));
  const long long tiles = (long long)grid.x * grid.y;
  double* partial = static_cast<double*>(ws);
  const OpKContigDiff dA{W0, W, ldw, 0, rows, d};
  quad_form_kernel<<<grid, kGemmThreads, kGemmSmemBytes, st>>>(dA, H, d, W0, W, ldw, rows, partial);
  const OpKContig A0{W0, ldw, 0, rows, d};
  quad_form_kernel<<<grid, kGemmThreads, kGemmSmemBytes, st>>>(A0, H, d, W0, nullptr, ldw, rows, partial + tiles);
  recon_sum_kernel<<<2, kSumThreads, 0, st>>>(partial, tiles, num_den);
  count_launches(3);
  return cudaGetLastError();
}

}  // namespace sgpt
