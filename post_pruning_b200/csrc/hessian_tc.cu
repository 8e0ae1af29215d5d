// H += X^T X, or H = X^T X, on the 5th-generation tensor cores (SparseGPT
// review, section 七: the Hessian proxy of a linear layer is the Gram matrix
// of its inputs).
//
// X is bf16 [n x d] row-major, so both GEMM operands of C = X^T X are the same
// tensor read "MN-major": for C[i][j] = sum_t X[t][i] X[t][j], A(i, t) and
// B(j, t) are contiguous along i and j. H is symmetric: only tiles on the
// upper triangle are computed, and each element is written once, to H[i][j]
// and its mirror H[j][i]. Wide layers use 128 x 256 band tiles whose rows
// i0.. and columns j0.. meet the upper triangle, numbered in super-blocks of
// 2048 x 2048 channels so that the CTAs resident together share most of the
// columns of X they stream (L2 reuse); tokens are split across CTAs when
// there are too few tiles to fill the GPU. Narrow layers use square tiles
// (see PairWork), always token-split. Split partials are summed in split
// order by a separate reduction kernel (deterministic).
//
// Per CTA: warp 0 lane 0 streams 64-token stages with TMA (128-byte swizzle,
// one box = 64 tokens x 64 channels), warp 1 lane 0 issues
// tcgen05.mma.kind::f16 (M=128, N=256, K=16, bf16 in, fp32 accumulate in
// TMEM). The tensor-core accumulator loses a fraction of an ulp per step on
// long sums of positive terms (the diagonal of X^T X drifts low by about 1e-3
// relative over 16k steps), so each TMEM accumulator only ever sums one chunk
// of 512 tokens: two 256-column accumulators alternate, and eight epilogue
// warps drain each finished chunk into FP32 running sums in registers
// (round-to-nearest adds) while the MMAs fill the other one. Every wait is
// bounded; a wait that runs out records SGPT_INFO_TIMEOUT.
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace sgpt {

namespace {

constexpr int kM = 128;              // tile rows (i)
constexpr int kN = 256;              // tile columns (j)
constexpr int kBK = 64;              // tokens per stage
constexpr int kStages = 4;
constexpr int kBox = kBK * 64 * 2;   // bytes of one 64-token x 64-channel box
constexpr int kAStage = 2 * kBox;    // 16 KB
constexpr int kBStage = 4 * kBox;    // 32 KB
constexpr int kStageBytes = kAStage + kBStage;
constexpr int kEpiWarps = 8;                  // warps 2..9 drain TMEM
constexpr int kThreads = 64 + 32 * kEpiWarps;   // warp 0: TMA, warp 1: MMA
constexpr int kChunkIters = 8;                // stages (512 tokens) per TMEM accumulation
constexpr int kTmemCols = 2 * kN;             // two accumulators, double-buffered
constexpr size_t kSmem = (size_t)kStages * kStageBytes + 1024 /*align*/ + 256 /*barriers*/;

// instruction descriptor: D fp32, A/B bf16, both MN-major, N=256, M=128
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                            ((uint32_t)(kN >> 3) << 17) | ((uint32_t)(kM >> 4) << 24);

constexpr uint32_t kIdesc128 = (kIdesc & ~(0x3fu << 17)) | ((uint32_t)(128 >> 3) << 17);

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Shared-memory matrix descriptor, MN-major operand, 128-byte swizzle:
// atoms of 64 channels x 8 tokens (1 KB); LBO = stride between 64-channel
// atoms (one TMA box), SBO = stride between 8-token groups (1 KB).
__device__ __forceinline__ uint64_t mn_desc(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3fff);
  d |= (uint64_t)((kBox >> 4) & 0x3fff) << 16;     // leading byte offset
  d |= (uint64_t)((1024 >> 4) & 0x3fff) << 32;     // stride byte offset
  d |= (uint64_t)1 << 46;                          // descriptor version (sm100)
  d |= (uint64_t)2 << 61;                          // SWIZZLE_128B
  return d;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.b32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Non-suspending test of a barrier phase.
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.b32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: false if the barrier phase did not complete within `limit`
// SM clock cycles. try_wait may suspend the thread for a hardware-defined
// time, longer than a short limit, so short limits (failure-path tests)
// poll with the non-suspending test instead.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, long long limit) {
  if (limit < kShortWaitCycles) {
    const long long t0 = clock64();
    while (!mbar_test(bar, parity))
      if (clock64() - t0 > limit) return false;
    return true;
  }
  if (mbar_try(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try(bar, parity))
    if (clock64() - t0 > limit) return false;
  return true;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x,
                                            int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void mma_bf16(uint32_t tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// 32 consecutive accumulator columns of this thread's TMEM lane (no wait).
__device__ __forceinline__ void tmem_ld32_nowait(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
        "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]),
        "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]),
        "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Number of tiles meeting the upper triangle in the first ti row tiles: row
// tile ti (rows ti*128..) meets the 256-wide column tiles tj >= ti/2, so
// this is ti*tn - floor(ti/2)*floor((ti-1)/2).
__host__ __device__ inline long long band_start(int ti, int tn) {
  return (long long)ti * tn - (long long)(ti / 2) * ((ti - 1) / 2);
}

// Tiles meeting the upper triangle in super-blocks of 2G row tiles by G
// column tiles (G*256 channels each way), super-block rows in order and, in
// each, the diagonal super-block first; tiles row by row inside a
// super-block. CTAs that run together then read a few thousand channels of X
// rather than all of them. G = 8 (2048 channels). At d = 25,600 and 131,072
// tokens, launched alone, G = 2..6 measured 92-97 ms per launch against 100
// for G = 8 or 12 and 106-107 for 16 or 24, but G = 4 read twice the DRAM
// bytes (402 against 193 GB) and inside a whole power-capped step it was no
// faster; narrower layers do not depend on it.
constexpr int kGroup = 8;
__host__ __device__ inline void grouped_tile(long long t, int tm, int tn, int G, int& ti, int& tj) {
  for (int I = 0;; ++I) {
    const int r0 = 2 * G * I, nr = (r0 + 2 * G < tm ? r0 + 2 * G : tm) - r0;
    const int c_hi = G * (I + 1) < tn ? G * (I + 1) : tn;
    long long diag = 0;
    for (int r = r0; r < r0 + nr; ++r) diag += c_hi - r / 2;
    if (t < diag) {
      int r = r0;
      while (t >= c_hi - r / 2) { t -= c_hi - r / 2; ++r; }
      ti = r;
      tj = r / 2 + (int)t;
      return;
    }
    t -= diag;
    const long long rest = (long long)nr * (tn - c_hi > 0 ? tn - c_hi : 0);
    if (t < rest || r0 + nr >= tm) {
      const long long per_sb = (long long)nr * G;
      const int k = (int)(t / per_sb);
      const int w = (int)(t - (long long)k * per_sb);
      const int c0 = c_hi + k * G;
      const int nc = tn - c0 < G ? tn - c0 : G;
      ti = r0 + w / nc;
      tj = c0 + w % nc;
      return;
    }
    t -= rest;
  }
}

// Widths with few 128-blocks (K(K+1)/2 <= one CTA per SM) cover the upper
// triangle with 128 x 128 squares rather than 128 x 256 band tiles, which
// would compute up to a third of their area below the diagonal. Row block a
// takes the squares (a, (a + o) mod K) for o = 0, 1, ...: (K+1)/2 of them
// for odd K; for even K, K/2 + 1 for a < K/2 and K/2 for the others. That
// is every unordered pair {a, c} exactly once; a square with c < a holds
// the transpose of the upper square (c, a). Then rows with an odd count are
// taken two at a time and the one square they share moves to the other
// row, which leaves at most one odd row. Consecutive squares of a row share
// the row block's A and make one 128 x 256 tile (B = column blocks c1 and
// c2, which need not be adjacent); the one odd square left is a 128 x 128
// tile, which takes about as long per token as a full one. Every tile gets
// the same number of token splits, and each CTA writes its partial sums for
// the reduction kernel.
constexpr int kMaxPairCtas = 148;
struct PairWork {
  unsigned char a, c1, c2, nsq;   // row block, column blocks of the one or two squares
  int t0, t1;                     // token range
};
struct PairTile {
  unsigned char a, c1, c2, nsq;
  short first, ns;                // CTAs first .. first + ns - 1, in token order
};
struct PairWorks {
  int ncta;                       // 0: band tiles instead
  PairWork w[kMaxPairCtas];
};
struct PairTiles {
  int ntiles;
  PairTile t[kMaxPairCtas];
};

}  // namespace

// H[i][j] += S[r][c] and, for j != i, H[j][i] += S[r][c] over the upper
// part (j >= i) of the 64 x 64 block at rows i0.., columns j0.. (S in shared
// memory, element (r, c) at r * rs + c * cs: a transposed view passes the
// strides swapped). Both passes are coalesced: rows of H along c, then the
// mirrored rows along r (a column of S).
constexpr int kSLd = 65;
constexpr int kTileLd = kN + 1;
__device__ __forceinline__ float lds1(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}
// (S is a 32-bit shared-memory address: the staging area may have been
// aligned through an integer, which hides its address space from the compiler)
__device__ void flush_block(uint32_t S, int rs, int cs, int i0, int j0, float* __restrict__ H, int d, int t,
                            int nt, bool set) {
  // d is a multiple of 32 and every group starts at a multiple of 4, so a
  // group that starts inside H ends inside it; groups wholly on one side of
  // the diagonal go as one 16-byte access (a store when `set`: H = the sum
  // instead of H += the sum)
  for (int q = t; q < 64 * 16; q += nt) {
    const int r = q >> 4, c4 = (q & 15) * 4, i = i0 + r, j = j0 + c4;
    if (i >= d || j >= d || j + 3 < i) continue;
    float v[4];
#pragma unroll
    for (int x = 0; x < 4; ++x) v[x] = lds1(S + 4u * (uint32_t)(r * rs + (c4 + x) * cs));
    float* p = H + (long long)i * d + j;
    if (j >= i) {
      float4 h = set ? make_float4(0.f, 0.f, 0.f, 0.f) : *reinterpret_cast<float4*>(p);
      h.x += v[0]; h.y += v[1]; h.z += v[2]; h.w += v[3];
      *reinterpret_cast<float4*>(p) = h;
    } else {
#pragma unroll
      for (int x = 0; x < 4; ++x)
        if (j + x >= i) p[x] = (set ? 0.f : p[x]) + v[x];
    }
  }
  for (int q = t; q < 64 * 16; q += nt) {
    const int c = q >> 4, r4 = (q & 15) * 4, j = j0 + c, i = i0 + r4;
    if (j >= d || i >= d || i >= j) continue;
    float v[4];
#pragma unroll
    for (int x = 0; x < 4; ++x) v[x] = lds1(S + 4u * (uint32_t)((r4 + x) * rs + c * cs));
    float* p = H + (long long)j * d + i;
    if (i + 3 < j) {
      float4 h = set ? make_float4(0.f, 0.f, 0.f, 0.f) : *reinterpret_cast<float4*>(p);
      h.x += v[0]; h.y += v[1]; h.z += v[2]; h.w += v[3];
      *reinterpret_cast<float4*>(p) = h;
    } else {
#pragma unroll
      for (int x = 0; x < 4; ++x)
        if (i + x < j) p[x] = (set ? 0.f : p[x]) + v[x];
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1) hessian_tc_kernel(
    const __grid_constant__ CUtensorMap xmap, float* __restrict__ H, int d, long long n,
    int nsplit, long long per, float* __restrict__ part, int* info, const __grid_constant__ PairWorks pw,
    int set, int group, long long wait_cycles) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 5);
  __shared__ int failed;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool paired = pw.ncta > 0;
  int i0, j1, j2, nsq = 2;                    // row channels; B = channels j1.. and j2.. (128 each)
  long long t_begin, t_end;
  if (paired) {
    const PairWork wk = pw.w[blockIdx.x];
    i0 = wk.a * kM;
    nsq = wk.nsq;
    j1 = wk.c1 * kM;
    j2 = wk.c2 * kM;
    t_begin = wk.t0;
    t_end = wk.t1;
  } else {
    const int tile = blockIdx.x / nsplit, split = blockIdx.x - (blockIdx.x / nsplit) * nsplit;
    int ti, tj;
    grouped_tile(tile, (d + kM - 1) / kM, (d + kN - 1) / kN, group, ti, tj);
    i0 = ti * kM;
    j1 = tj * kN;
    j2 = j1 + 128;
    t_begin = (long long)split * per;
    t_end = t_begin + per < n ? t_begin + per : n;
  }
  const int j0 = j1;
  const int iters = (int)((t_end - t_begin + kBK - 1) / kBK);
  const int nchunks = (iters + kChunkIters - 1) / kChunkIters;

  const uint32_t s0 = smem_u32(smem);
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + kStages);
  const uint32_t tfull0 = smem_u32(bars + 2 * kStages), tempty0 = tfull0 + 16;
  const uint32_t mdone = tfull0 + 32;         // every MMA this CTA issued has completed

  if (threadIdx.x == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&xmap)) : "memory");
    failed = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull0 + 8 * b, 1);
      mbar_init(tempty0 + 8 * b, kEpiWarps);
    }
    mbar_init(mdone, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;
  const bool skip = cta_info_set(info) || iters <= 0;

  // Epilogue state: warp w (2..9) owns TMEM lanes 32*(w%4).. (tile rows) and
  // columns 128*((w-2)/4).. of each accumulator; its running sums live in
  // registers and are updated with correctly rounded FP32 adds.
  const int q = warp & 3, h = (warp - 2) >> 2;
  float acc[128];
#pragma unroll
  for (int e = 0; e < 128; ++e) acc[e] = 0.f;

  if (!skip && warp == 0 && lane == 0) {
    // TMA producer
    int issued = 0;
    for (int it = 0; it < iters; ++it) {
      const int s = it % kStages;
      const uint32_t par = ((it / kStages) & 1) ^ 1;
      if (it >= kStages && !mbar_wait(empty0 + 8 * s, par, wait_cycles)) {
        failed = 1;
        break;
      }
      const uint32_t bar = full0 + 8 * s;
      mbar_expect_tx(bar, kAStage + 2 * nsq * kBox);
      const int y = (int)(t_begin + (long long)it * kBK);
      const uint32_t a = s0 + s * kStageBytes, b = a + kAStage;
      tma_load_2d(a, &xmap, bar, i0, y);
      tma_load_2d(a + kBox, &xmap, bar, i0 + 64, y);
#pragma unroll
      for (int c = 0; c < 4; ++c)
        if (c < 2 * nsq) tma_load_2d(b + c * kBox, &xmap, bar, (c < 2 ? j1 : j2) + 64 * (c & 1), y);
      ++issued;
    }
    // never leave with copies in flight: wait for every stage that was armed
    for (int it = (issued > kStages ? issued - kStages : 0); it < issued; ++it)
      if (!mbar_wait(full0 + 8 * (it % kStages), (it / kStages) & 1, kDrainCycles)) failed = 1;
  } else if (!skip && warp == 1 && lane == 0) {
    // MMA issuer: chunk c accumulates kChunkIters stages into buffer c & 1
    const uint32_t idesc = nsq == 2 ? kIdesc : kIdesc128;
    for (int c = 0; c < nchunks && !failed; ++c) {
      const int b = c & 1;
      if (c >= 2 && !mbar_wait(tempty0 + 8 * b, ((c >> 1) - 1) & 1, wait_cycles)) {
        failed = 1;
        break;
      }
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t acc_t = tmem + (uint32_t)(b * kN);
      const int it_end = min(iters, (c + 1) * kChunkIters);
      for (int it = c * kChunkIters; it < it_end; ++it) {
        const int s = it % kStages;
        if (!mbar_wait(full0 + 8 * s, (it / kStages) & 1, wait_cycles)) {
          failed = 1;
          break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t a = s0 + s * kStageBytes, bb = a + kAStage;
#pragma unroll
        for (int ks = 0; ks < kBK / 16; ++ks)
          mma_bf16(acc_t, mn_desc(a + ks * 2048), mn_desc(bb + ks * 2048), idesc,
                   (it != c * kChunkIters) || ks != 0);
        mma_commit(empty0 + 8 * s);
      }
      mma_commit(tfull0 + 8 * b);
    }
    // never free TMEM under a running MMA (after a timeout the epilogue may
    // not have waited for the last ones): wait for all of them
    mma_commit(mdone);
    if (!mbar_wait(mdone, 0, kDrainCycles)) failed = 1;
  } else if (!skip && warp >= 2) {
    // Drain every chunk into the running sums, then hand the buffer back.
    for (int c = 0; c < nchunks; ++c) {
      const int b = c & 1;
      // one decision per warp: the TMEM loads and the __syncwarp below are
      // warp-collective
      if (!__all_sync(0xffffffffu, mbar_wait(tfull0 + 8 * b, (c >> 1) & 1, wait_cycles) ? 1 : 0)) {
        failed = 1;
        break;
      }
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t base = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * kN + h * 128);
      if (h < nsq) {                          // a one-square tile has no second half
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t v[32];
          tmem_ld32_nowait(base + cc * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) acc[cc * 32 + e] += __uint_as_float(v[e]);
        }
      }
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty0 + 8 * b);
    }
  }

  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (failed && threadIdx.x == 0) set_info(info, SGPT_INFO_TIMEOUT);
  if (!skip && !failed && warp >= 2) {
    const int r = q * 32 + lane;              // tile row
    if (paired || nsplit > 1) {
      float* dst = part + (size_t)blockIdx.x * kM * kN + (size_t)r * kN + h * 128;
#pragma unroll
      for (int e = 0; e < 128; e += 4) st4(dst + e, make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]));
    }
  }
  if (!skip && !failed && !paired && nsplit == 1 && warp >= 2) {
    // H += tile (and its mirror) through shared memory, by the epilogue
    // warps (named barrier 1): the whole tile is staged in the stage buffers,
    // free now that every MMA has completed, then flushed 64 x 64 at a time
    const uint32_t S = smem_u32(smem);
    const int et = threadIdx.x - 64;            // epilogue thread 0..255
    const int r = q * 32 + lane;
#pragma unroll
    for (int e = 0; e < 128; ++e)
      asm volatile("st.shared.f32 [%0], %1;" ::"r"(S + 4u * (uint32_t)(r * kTileLd + h * 128 + e)), "f"(acc[e]) : "memory");
    asm volatile("bar.sync 1, 256;" ::: "memory");
    for (int blk = 0; blk < (kM / 64) * (kN / 64); ++blk) {
      const int br = blk / (kN / 64), bc = blk % (kN / 64);
      const int bi0 = i0 + 64 * br, bj0 = j0 + 64 * bc;
      if (bi0 < d && bj0 < d && bj0 + 63 >= bi0)  // the block meets the upper triangle
        flush_block(S + 4u * (uint32_t)((64 * br) * kTileLd + 64 * bc), kTileLd, 1, bi0, bj0, H, d, et, 256,
                    set != 0);
    }
  }
  __syncthreads();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
}

// Split partials -> H: one CTA per 64 x 64 block of a tile, one thread per
// four elements, sums the block's nsplit partials in split order
// (deterministic; up to eight loads in flight per thread), then adds the sum
// to H and to its mirror through shared memory.
constexpr int kReduceThreads = 1024;
__global__ void __launch_bounds__(kReduceThreads) hessian_reduce_kernel(const float* __restrict__ part,
                                                                        float* __restrict__ H, int d, int tiles,
                                                                        int nsplit, const int* info, int set,
                                                                        int group) {
  if (cta_info_set(info)) return;
  __shared__ float S[64 * kSLd];
  const int tn = (d + kN - 1) / kN;
  const int t = threadIdx.x, r = t >> 4, c4 = (t & 15) * 4;
  for (int blk = blockIdx.x; blk < tiles * 8; blk += gridDim.x) {
    const int tile = blk >> 3, br = (blk & 7) >> 2, bc = blk & 3;
    int ti, tj;
    grouped_tile(tile, (d + kM - 1) / kM, tn, group, ti, tj);
    const int bi0 = ti * kM + 64 * br, bj0 = tj * kN + 64 * bc;
    if (!(bi0 < d && bj0 < d && bj0 + 63 >= bi0)) continue;   // block-uniform
    const float* src = part + (size_t)tile * nsplit * kM * kN + (size_t)(64 * br + r) * kN + 64 * bc + c4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int p0 = 0; p0 < nsplit; p0 += 8) {
      float4 v[8];
#pragma unroll
      for (int pp = 0; pp < 8; ++pp)
        v[pp] = (p0 + pp < nsplit) ? __ldcs(reinterpret_cast<const float4*>(src + (size_t)(p0 + pp) * kM * kN))
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int pp = 0; pp < 8; ++pp)
        if (p0 + pp < nsplit) {
          acc.x += v[pp].x; acc.y += v[pp].y; acc.z += v[pp].z; acc.w += v[pp].w;
        }
    }
    S[r * kSLd + c4] = acc.x;
    S[r * kSLd + c4 + 1] = acc.y;
    S[r * kSLd + c4 + 2] = acc.z;
    S[r * kSLd + c4 + 3] = acc.w;
    __syncthreads();
    flush_block(smem_u32(S), kSLd, 1, bi0, bj0, H, d, t, kReduceThreads, set != 0);
    __syncthreads();
  }
}

// Square tiles' partials -> H: one CTA per 64 x 64 block of a square
// (four per square; the lower one of a diagonal square holds nothing
// needed), summing the tile's partials in token order, then adding the sum
// to H and its mirror; a square below the diagonal is flushed through its
// transposed view, which lies above it.
__global__ void __launch_bounds__(kReduceThreads) hessian_pair_reduce_kernel(const float* __restrict__ part,
                                                                             float* __restrict__ H, int d,
                                                                             const __grid_constant__ PairTiles pt,
                                                                             const int* info, int set) {
  if (cta_info_set(info)) return;
  __shared__ float S[64 * kSLd];
  const int t = threadIdx.x, r = t >> 4, c4 = (t & 15) * 4;
  for (int gb = blockIdx.x;; gb += gridDim.x) {
    int ti = 0, base = 0;
    while (ti < pt.ntiles && gb >= base + 4 * pt.t[ti].nsq) base += 4 * pt.t[ti++].nsq;
    if (ti >= pt.ntiles) break;                                // block-uniform
    const PairTile tl = pt.t[ti];
    const int blk = gb - base, sq = blk >> 2, br = (blk >> 1) & 1, bc = blk & 1;
    const int a = tl.a, c = sq ? tl.c2 : tl.c1;
    const int bi0 = a * kM + 64 * br, bj0 = c * kM + 64 * bc;
    if (bi0 >= d || bj0 >= d || (c == a && br > bc)) continue;   // block-uniform
    const float* src = part + (size_t)tl.first * kM * kN + (size_t)(64 * br + r) * kN + 128 * sq + 64 * bc + c4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int p0 = 0; p0 < tl.ns; p0 += 8) {
      float4 v[8];
#pragma unroll
      for (int pp = 0; pp < 8; ++pp)
        v[pp] = (p0 + pp < tl.ns) ? __ldcs(reinterpret_cast<const float4*>(src + (size_t)(p0 + pp) * kM * kN))
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int pp = 0; pp < 8; ++pp)
        if (p0 + pp < tl.ns) {
          acc.x += v[pp].x; acc.y += v[pp].y; acc.z += v[pp].z; acc.w += v[pp].w;
        }
    }
    S[r * kSLd + c4] = acc.x;
    S[r * kSLd + c4 + 1] = acc.y;
    S[r * kSLd + c4 + 2] = acc.z;
    S[r * kSLd + c4 + 3] = acc.w;
    __syncthreads();
    if (c >= a) flush_block(smem_u32(S), kSLd, 1, bi0, bj0, H, d, t, kReduceThreads, set != 0);
    else flush_block(smem_u32(S), 1, kSLd, bj0, bi0, H, d, t, kReduceThreads, set != 0);
    __syncthreads();
  }
}

// ----------------------------------------------------------------- host

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

struct Plan {
  int tiles, nsplit, group;
  long long per;
  PairWorks pw;     // pw.ncta > 0: square tiles (then tiles/nsplit/per are unused)
  PairTiles pt;
  int pair_blocks;  // 64 x 64 blocks of the squares, for the reduction
};

// Square tiles for widths of at most K(K+1)/2 <= kMaxPairCtas squares (see
// PairWork): returns false otherwise.
bool plan_pairs(int d, long long n, Plan& p) {
  const int K = (d + kM - 1) / kM;
  const int squares = K * (K + 1) / 2;
  if (squares > kMaxPairCtas) return false;
  // each row block's squares: list[a][0..cnt[a]), column blocks
  static_assert(kMaxPairCtas < 256, "block numbers are bytes");
  constexpr int kMaxK = 17;                        // K(K+1)/2 <= 148
  unsigned char list[kMaxK][kMaxK + 1];
  int cnt[kMaxK];
  for (int a = 0; a < K; ++a) {
    cnt[a] = (K & 1) ? (K + 1) / 2 : (a < K / 2 ? K / 2 + 1 : K / 2);
    for (int o = 0; o < cnt[a]; ++o) list[a][o] = (unsigned char)((a + o) % K);
  }
  int odd = -1;
  for (int a = 0; a < K; ++a) {
    if (!(cnt[a] & 1)) continue;
    if (odd < 0) {
      odd = a;
      continue;
    }
    // rows odd and a share the square {odd, a}: move it to the other one
    const int b = odd;
    odd = -1;
    int from = -1, at = -1;
    for (int o = 0; o < cnt[b] && from < 0; ++o)
      if (list[b][o] == a && a != b) from = b, at = o;
    for (int o = 0; o < cnt[a] && from < 0; ++o)
      if (list[a][o] == b) from = a, at = o;
    const int to = from == a ? b : a;
    list[to][cnt[to]++] = (unsigned char)(from == a ? a : b);
    for (int o = at; o + 1 < cnt[from]; ++o) list[from][o] = list[from][o + 1];
    --cnt[from];
  }
  int ntiles = 0;
  for (int a = 0; a < K; ++a) ntiles += (cnt[a] + 1) / 2;
  const int s = std::max(1, kMaxPairCtas / ntiles);   // splits per tile
  long long per = ((n + s - 1) / s + kBK - 1) / kBK * kBK;
  per = std::max<long long>(per, 4 * kBK);             // >= 4 stages per split
  const int ns = (int)((n + per - 1) / per);
  p.pw.ncta = 0;
  p.pt.ntiles = 0;
  p.pair_blocks = 0;
  for (int a = 0; a < K; ++a) {
    for (int o = 0; o < cnt[a]; o += 2) {
      PairTile tl;
      tl.a = (unsigned char)a;
      tl.c1 = list[a][o];
      tl.nsq = (unsigned char)(o + 1 < cnt[a] ? 2 : 1);
      tl.c2 = tl.nsq == 2 ? list[a][o + 1] : tl.c1;
      tl.first = (short)p.pw.ncta;
      tl.ns = (short)ns;
      for (int sp = 0; sp < ns; ++sp) {
        PairWork& w = p.pw.w[p.pw.ncta++];
        w.a = tl.a;
        w.c1 = tl.c1;
        w.c2 = tl.c2;
        w.nsq = tl.nsq;
        w.t0 = (int)(sp * per);
        w.t1 = (int)std::min<long long>(n, (sp + 1) * per);
      }
      p.pt.t[p.pt.ntiles++] = tl;
      p.pair_blocks += 4 * tl.nsq;
    }
  }
  return true;
}

Plan plan(int d, long long n) {
  Plan p{};
  if (plan_pairs(d, n, p)) return p;
  p.pw.ncta = 0;
  const int tm = (d + kM - 1) / kM, tn = (d + kN - 1) / kN;
  const int tiles = (int)band_start(tm, tn);
  // split tokens when the tiles alone cannot fill the GPU, keeping the grid
  // within one wave (one CTA per SM: the stages take most of shared memory)
  long long ns = 1;
  if (tiles < kNumSMs) ns = kNumSMs / tiles;
  const long long max_split = (n + 4 * kBK - 1) / (4 * kBK);   // >= 4 stages per split
  ns = std::max<long long>(1, std::min(ns, max_split));
  long long per = ((n + ns - 1) / ns + kBK - 1) / kBK * kBK;
  ns = (n + per - 1) / per;
  p.tiles = tiles;
  p.group = kGroup;
  p.nsplit = (int)std::max<long long>(1, ns);
  p.per = per;
  return p;
}

size_t part_floats(const Plan& p) {
  if (p.pw.ncta > 0) return (size_t)p.pw.ncta * kM * kN;
  return p.nsplit > 1 ? (size_t)p.tiles * p.nsplit * kM * kN : 0;
}

}  // namespace

size_t hessian_ws_bytes(int d, long long n) {
  const Plan p = plan(d, n);
  Carve c(nullptr);
  if (part_floats(p)) c.take<float>(part_floats(p));
  return c.off + 256;
}

cudaError_t launch_hessian_tc(float* H, const uint16_t* X, long long n, int d, void* ws, int* info,
                              cudaStream_t st, bool set) {
  if (n <= 0) return cudaSuccess;
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  const Plan p = plan(d, n);
  Carve c(ws);
  float* part = part_floats(p) ? c.take<float>(part_floats(p)) : nullptr;


  CUtensorMap map;
  const cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)n};
  const cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)kBK};
  const cuuint32_t estr[2] = {1, 1};
  if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(X), dims, strides, box, estr,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  static PerDevice attrs;
  cudaError_t ea = once_per_device(attrs, [] {
    return cudaFuncSetAttribute(hessian_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
  });
  if (ea != cudaSuccess) return ea;
  const int grid = p.pw.ncta > 0 ? p.pw.ncta : p.tiles * p.nsplit;
  hessian_tc_kernel<<<grid, kThreads, kSmem, st>>>(map, H, d, n, p.nsplit, p.per, part, info, p.pw, set ? 1 : 0,
                                                   p.group, wait_limit_cycles());
  count_launches(1);
  if (p.pw.ncta > 0) {
    hessian_pair_reduce_kernel<<<p.pair_blocks, kReduceThreads, 0, st>>>(part, H, d, p.pt, info, set ? 1 : 0);
    count_launches(1);
  } else if (p.nsplit > 1) {
    const int g = (int)std::min<long long>((long long)p.tiles * 8, 8 * kNumSMs);
    hessian_reduce_kernel<<<g, kReduceThreads, 0, st>>>(part, H, d, p.tiles, p.nsplit, info, set ? 1 : 0,
                                                        p.group);
    count_launches(1);
  }
  return cudaGetLastError();
}

}  // namespace sgpt
