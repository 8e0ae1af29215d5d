// FP32-accurate matrix products on the 5th-generation tensor cores.
//
// C = alpha * A B + beta * C with A, B fp32. Each operand is held as two
// planes, x = hi + lo with hi = x rounded to TF32 (10 explicit mantissa
// bits) and lo = x - hi (exact), and every K step issues three
// tcgen05.mma.kind::tf32 products, hi*hi + hi*lo + lo*hi, into one fp32 TMEM
// accumulator (the lo*lo term is below fp32 resolution). The error per
// product is about 2^-21 relative, against 2^-24 for a plain fp32 FMA and
// 2^-11 for a single TF32 product.
//
// Used for the rank-128 updates and the triangular inverse of the
// factorisation and for the lazy trailing update of the OBS sweep.
//
// CTA tile 128 x 128, K in steps of 16 (one 64-byte swizzle row of fp32),
// three-stage TMA ring in 96 KB (no multicast) so that two CTAs share an SM;
// warp 0 lane 0 loads, warp 1 lane 0 issues MMAs, warps 2-5 drain TMEM
// (warp w reads lanes 32*(w%4)..) into a shared staging tile and then update
// C a whole row per warp instruction (coalesced). TMEM accumulates at most
// 128 of K: a longer K alternates between two TMEM accumulators and the
// epilogue warps sum the chunks in FP32 registers (a long accumulation inside
// TMEM loses accuracy).
// A is always K-major (row-major M x K); B is K-major (row-major N x K) or
// MN-major (row-major K x N). Every wait is bounded.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "common.cuh"
#include "gemm_tc.h"
#include "kernels.h"

namespace sgpt {
namespace tc {

namespace {

constexpr int kM = 128, kN = 128, kKC = 16;
constexpr int kStages = 3;
constexpr int kPlane = kM * kKC * 4;            // 8 KB: one operand plane of one stage
constexpr int kStageBytes = 4 * kPlane;         // A hi/lo, B hi/lo
constexpr int kThreads = 192;
constexpr int kStageLd = kN + 4;                // epilogue staging row (floats)
constexpr size_t kSmem = (size_t)kStages * kStageBytes + 1024 + 256;
static_assert((size_t)kM * kStageLd * 4 <= (size_t)kStages * kStageBytes, "staging must fit the stages");
constexpr long long kWaitCycles = 4000000000ll;
constexpr int kChunk = 8;                       // K steps (128 of K) per TMEM accumulation
constexpr int kTmemCols = 2 * kN;               // two accumulators: one fills while one drains

__host__ __device__ constexpr uint32_t make_idesc(bool b_mn) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(kN >> 3) << 17) |
         ((uint32_t)(kM >> 4) << 24);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// K-major operand, 64-byte swizzle (a K chunk of 16 fp32 is one 64-byte
// row): 8-row groups of 512 bytes.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3fff);
  d |= (uint64_t)1 << 16;                         // leading byte offset (unused when swizzled)
  d |= (uint64_t)(512 >> 4) << 32;                // stride byte offset: next 8 rows
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)4 << 61;                         // SWIZZLE_64B
  return d;
}
// MN-major 32-bit operand: the 128-byte swizzle with 32-byte granules
// (descriptor layout SWIZZLE_128B_BASE32B, filled by TMA's
// SWIZZLE_128B_ATOM_32B). Atoms are 32 columns x 4 K rows (512 bytes);
// LBO = next 32 columns (one 32-column x 16-row TMA box, 2 KB), SBO = next
// 4 K rows. The plain 128-byte swizzle (16-byte granules) is not a valid
// MN-major form for 32-bit elements.
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3fff);
  d |= (uint64_t)(2048 >> 4) << 16;
  d |= (uint64_t)(512 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)1 << 61;
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
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try(bar, parity))
    if (clock64() - t0 > kWaitCycles) return false;
  return true;
}
__device__ __forceinline__ void tma_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void mma_tf32(uint32_t tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
        "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]),
        "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]),
        "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tri_index(int t, int& i, int& j) {
  int jj = (int)((sqrtf(8.f * t + 1.f) - 1.f) * 0.5f);
  while ((jj + 1) * (jj + 2) / 2 <= t) ++jj;
  while (jj * (jj + 1) / 2 > t) --jj;
  j = jj;
  i = t - jj * (jj + 1) / 2;
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 2) gemm_tf32x3_kernel(
    const __grid_constant__ CUtensorMap a_hi, const __grid_constant__ CUtensorMap a_lo,
    const __grid_constant__ CUtensorMap b_hi, const __grid_constant__ CUtensorMap b_lo, const Job job,
    const int b_mn, int* info) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 4);
  __shared__ int failed;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- which tile and which K range
  int m0 = 0, n0 = 0, kb = 0, ke = 0, split = 0, tile = 0;
  if (job.mode == 0) {
    m0 = (blockIdx.x / job.nt) * kM;
    n0 = (blockIdx.x % job.nt) * kN;
    ke = job.kdim;
  } else if (job.mode == 1) {
    int i, j;
    tri_index(job.t0 + (int)blockIdx.x, i, j);
    m0 = i * kM;
    n0 = j * kN;
    ke = job.kdim;
  } else if (job.mode == 3) {
    m0 = job.s * kM;
    n0 = (job.s + 1 + (int)blockIdx.x) * kN;
    kb = m0;
    ke = min(m0 + kM, job.dlim);
  } else {
    tile = blockIdx.x / job.nsplit;
    split = blockIdx.x - tile * job.nsplit;
    const int i = job.s, j = job.s + 1 + tile;
    m0 = i * kM;
    n0 = j * kN;
    const int lo = (i + 1) * kM, hi = min((j + 1) * kM, job.dlim);
    const int per = ((j - i + job.nsplit - 1) / job.nsplit) * kM;
    kb = min(hi, lo + split * per);
    ke = min(hi, kb + per);
  }
  const int iters = (ke - kb + kKC - 1) / kKC;
  const uint32_t idesc = make_idesc(b_mn != 0);

  const uint32_t s0 = smem_u32(smem);
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + kStages);
  const uint32_t tfull0 = smem_u32(bars + 2 * kStages), tempty0 = tfull0 + 16;
  const int nchunks = (iters + kChunk - 1) / kChunk;
  if (threadIdx.x == 0) {
    failed = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull0 + 8 * b, 1);
      mbar_init(tempty0 + 8 * b, 4);            // the four epilogue warps
    }
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
  const bool skip = cta_info_set(info);

  if (!skip && iters > 0 && warp == 0 && lane == 0) {
    int issued = 0;
    for (int it = 0; it < iters; ++it) {
      const int s = it % kStages;
      if (it >= kStages && !mbar_wait(empty0 + 8 * s, ((it / kStages) & 1) ^ 1)) {
        failed = 1;
        break;
      }
      const uint32_t bar = full0 + 8 * s;
      mbar_expect_tx(bar, kStageBytes);
      const uint32_t st = s0 + s * kStageBytes;
      const int k = kb + it * kKC;
      tma_2d(st, &a_hi, bar, job.a_x0 + k, job.a_y0 + m0);
      tma_2d(st + kPlane, &a_lo, bar, job.a_x0 + k, job.a_y0 + m0);
      if (b_mn) {
#pragma unroll
        for (int c = 0; c < kN / 32; ++c) {
          tma_2d(st + 2 * kPlane + c * 2048, &b_hi, bar, job.b_x0 + n0 + 32 * c, job.b_y0 + k);
          tma_2d(st + 3 * kPlane + c * 2048, &b_lo, bar, job.b_x0 + n0 + 32 * c, job.b_y0 + k);
        }
      } else {
        tma_2d(st + 2 * kPlane, &b_hi, bar, job.b_x0 + k, job.b_y0 + n0);
        tma_2d(st + 3 * kPlane, &b_lo, bar, job.b_x0 + k, job.b_y0 + n0);
      }
      ++issued;
    }
    for (int it = (issued > kStages ? issued - kStages : 0); it < issued; ++it)
      if (!mbar_wait(full0 + 8 * (it % kStages), (it / kStages) & 1)) failed = 1;
  } else if (!skip && iters > 0 && warp == 1 && lane == 0) {
    // chunk c (kChunk K steps) accumulates into TMEM buffer c & 1; a long K
    // is summed chunk by chunk in FP32 registers by the epilogue warps
    for (int c = 0; c < nchunks && !failed; ++c) {
      const int b = c & 1;
      if (c >= 2 && !mbar_wait(tempty0 + 8 * b, ((c >> 1) - 1) & 1)) {
        failed = 1;
        break;
      }
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t acc_t = tmem + (uint32_t)(b * kN);
      const int it_end = min(iters, (c + 1) * kChunk);
      for (int it = c * kChunk; it < it_end; ++it) {
        const int s = it % kStages;
        if (!mbar_wait(full0 + 8 * s, (it / kStages) & 1)) {
          failed = 1;
          break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t st = s0 + s * kStageBytes;
#pragma unroll
        for (int ks = 0; ks < kKC / 8; ++ks) {
          const uint64_t ah = kmajor_desc(st + ks * 32), al = kmajor_desc(st + kPlane + ks * 32);
          uint64_t bh, bl;
          if (b_mn) {
            bh = mnmajor_desc(st + 2 * kPlane + ks * 1024);
            bl = mnmajor_desc(st + 3 * kPlane + ks * 1024);
          } else {
            bh = kmajor_desc(st + 2 * kPlane + ks * 32);
            bl = kmajor_desc(st + 3 * kPlane + ks * 32);
          }
          const uint32_t first = (it == c * kChunk && ks == 0) ? 0u : 1u;
          mma_tf32(acc_t, al, bh, idesc, first);   // small terms first
          mma_tf32(acc_t, ah, bl, idesc, 1u);
          mma_tf32(acc_t, ah, bh, idesc, 1u);
        }
        mma_commit(empty0 + 8 * s);
      }
      mma_commit(tfull0 + 8 * b);
    }
  }

  const bool partial = job.mode == 2 && job.nsplit > 1;
  const bool read_c = !partial && job.C != nullptr && job.beta != 0.f;
  if (!skip && read_c && warp >= 2) {
    // Bring this warp's 32 rows of C toward L2 while the main loop runs.
    const int row = m0 + (warp - 2) * 32 + lane;
    if (row < job.Mlim && n0 < job.Nlim) {
      const float* p = job.C + (long long)(job.c_row0 + row) * job.ldc + job.c_col0 + n0;
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(min(kN, job.Nlim - n0) * 4)
                   : "memory");
    }
  }
  // Epilogue warps: TMEM -> shared staging tile. Warp w reads TMEM lanes
  // 32*(w%4).. (tile rows). One chunk goes straight to the staging tile;
  // several are summed in FP32 registers first (each thread holds its row).
  // The stage buffers are free for staging once the last chunk is in.
  float* T = reinterpret_cast<float*>(smem);
  const int q = warp & 3;
  const int m = q * 32 + lane;                 // tile row = TMEM lane
  if (!skip && warp >= 2) {
    if (iters == 0) {
#pragma unroll 1
      for (int e = 0; e < kN; e += 4) *reinterpret_cast<float4*>(T + m * kStageLd + e) = make_float4(0.f, 0.f, 0.f, 0.f);
    } else if (nchunks == 1) {
      __syncwarp();
      if (!mbar_wait(tfull0, 0)) failed = 1;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
#pragma unroll 1
      for (int cc = 0; cc < kN / 32 && !failed; ++cc) {
        uint32_t v[32];
        tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + cc * 32, v);
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4*>(T + m * kStageLd + cc * 32 + e) =
              make_float4(__uint_as_float(v[e]), __uint_as_float(v[e + 1]), __uint_as_float(v[e + 2]),
                          __uint_as_float(v[e + 3]));
      }
    } else {
      float acc[kN];
#pragma unroll
      for (int e = 0; e < kN; ++e) acc[e] = 0.f;
      for (int c = 0; c < nchunks; ++c) {
        const int b = c & 1;
        __syncwarp();
        if (!mbar_wait(tfull0 + 8 * b, (c >> 1) & 1)) {
          failed = 1;
          break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
#pragma unroll
        for (int cc = 0; cc < kN / 32; ++cc) {
          uint32_t v[32];
          tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * kN + cc * 32), v);
#pragma unroll
          for (int e = 0; e < 32; ++e) acc[cc * 32 + e] += __uint_as_float(v[e]);
        }
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty0 + 8 * b);
      }
#pragma unroll
      for (int e = 0; e < kN; e += 4)
        *reinterpret_cast<float4*>(T + m * kStageLd + e) = make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (failed && threadIdx.x == 0) set_info(info, SGPT_INFO_TIMEOUT);

  if (!skip && !failed && warp >= 2) {
    const int col = lane * 4;                  // this lane's four columns of a row
    const bool planes = job.C_hi != nullptr && (!job.planes_one_col || n0 == job.planes_n0);
    const long long ldp = job.ldp ? job.ldp : job.ldc;
    const bool col_ok = n0 + col < job.Nlim;
#pragma unroll 1
    for (int r0 = 0; r0 < 32; r0 += 8) {
      float4 a[8], old[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {            // all loads of 8 rows first
        const int mr = (warp - 2) * 32 + r0 + u;
        a[u] = *reinterpret_cast<const float4*>(T + mr * kStageLd + col);
        old[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (read_c && col_ok && m0 + mr < job.Mlim)
          old[u] = ld4(job.C + (long long)(job.c_row0 + m0 + mr) * job.ldc + job.c_col0 + n0 + col);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int mr = (warp - 2) * 32 + r0 + u;
        if (partial) {
          st4(job.part + (size_t)blockIdx.x * kM * kN + (size_t)mr * kN + col, a[u]);
          continue;
        }
        const int row = m0 + mr;
        if (row >= job.Mlim || !col_ok) continue;
        const float o[4] = {fmaf(job.alpha, a[u].x, job.beta * old[u].x), fmaf(job.alpha, a[u].y, job.beta * old[u].y),
                            fmaf(job.alpha, a[u].z, job.beta * old[u].z), fmaf(job.alpha, a[u].w, job.beta * old[u].w)};
        if (job.C)
          st4(job.C + (long long)(job.c_row0 + row) * job.ldc + job.c_col0 + n0 + col,
              make_float4(o[0], o[1], o[2], o[3]));
        if (planes) {
          const long long off = (long long)(job.c_row0 + row) * ldp + job.c_col0 + n0 + col - job.p_col0;
          float h4[4], l4[4];
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            h4[t] = tf32_hi(o[t]);
            l4[t] = o[t] - h4[t];
          }
          st4(job.C_hi + off, make_float4(h4[0], h4[1], h4[2], h4[3]));
          st4(job.C_lo + off, make_float4(l4[0], l4[1], l4[2], l4[3]));
        }
      }
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
}

// Split partials of a block row -> C = alpha * sum (+ hi/lo planes), in split order.
__global__ void __launch_bounds__(256) rowsplit_reduce_kernel(const Job job, const int* info) {
  if (cta_info_set(info)) return;
  const int tiles = job.nblk - 1 - job.s;
  const long long quads = (long long)tiles * (kM * kN / 4);
  for (long long qd = (long long)blockIdx.x * blockDim.x + threadIdx.x; qd < quads;
       qd += (long long)gridDim.x * blockDim.x) {
    const int tile = (int)(qd / (kM * kN / 4));
    const int e = (int)(qd - (long long)tile * (kM * kN / 4)) * 4;
    const int m = e / kN, n = e % kN;
    const int row = job.s * kM + m, col = (job.s + 1 + tile) * kN + n;
    if (row >= job.Mlim || col >= job.Nlim) continue;
    const float* src = job.part + (size_t)tile * job.nsplit * kM * kN + e;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int p = 0; p < job.nsplit; ++p) {
      const float4 v = __ldcs(reinterpret_cast<const float4*>(src + (size_t)p * kM * kN));
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    const float o[4] = {job.alpha * acc.x, job.alpha * acc.y, job.alpha * acc.z, job.alpha * acc.w};
    if (job.C) st4(job.C + (long long)(job.c_row0 + row) * job.ldc + job.c_col0 + col, make_float4(o[0], o[1], o[2], o[3]));
    if (job.C_hi) {
      const long long off = (long long)(job.c_row0 + row) * (job.ldp ? job.ldp : job.ldc) + job.c_col0 + col - job.p_col0;
      float h4[4], l4[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        h4[t] = tf32_hi(o[t]);
        l4[t] = o[t] - h4[t];
      }
      st4(job.C_hi + off, make_float4(h4[0], h4[1], h4[2], h4[3]));
      st4(job.C_lo + off, make_float4(l4[0], l4[1], l4[2], l4[3]));
    }
  }
}

// hi/lo planes of a row-major block: rows x cols (cols % 4 == 0).
// In place is allowed (hi == src): every element is read before it is written.
__global__ void split_planes_kernel(const float* src, long long ld, int rows, int cols, float* hi, float* lo,
                                    long long ldo, const int* info) {
  if (info_set(info)) return;
  const long long quads = (long long)rows * (cols / 4);
  for (long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x; q < quads;
       q += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(q / (cols / 4)), c = (int)(q - (long long)r * (cols / 4)) * 4;
    const float4 x = ld4(src + (long long)r * ld + c);
    const float4 h = make_float4(tf32_hi(x.x), tf32_hi(x.y), tf32_hi(x.z), tf32_hi(x.w));
    st4(hi + (long long)r * ldo + c, h);
    st4(lo + (long long)r * ldo + c, make_float4(x.x - h.x, x.y - h.y, x.z - h.z, x.w - h.w));
  }
}

// ---------------------------------------------------------------- host side

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

// Tensor map over a row-major fp32 matrix [rows x cols] with leading dimension
// ld; box = box_x (inner, fp32 elements) x box_y rows; 64-byte swizzle for
// K-major operands (16-float rows), 128-byte swizzle with 32-byte granules
// for MN-major ones (32-float rows).
bool make_map(CUtensorMap* m, const float* p, long long rows, long long cols, long long ld, int box_x, int box_y,
              bool mn_major) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)ld * 4};
  const cuuint32_t box[2] = {(cuuint32_t)box_x, (cuuint32_t)box_y};
  const cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(p), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE,
             mn_major ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_64B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_split(const float* src, long long ld, int rows, int cols, float* hi, float* lo, long long ldo,
                         const int* info, cudaStream_t st) {
  const long long quads = (long long)rows * (cols / 4);
  if (quads == 0) return cudaSuccess;
  const int g = (int)std::min<long long>((quads + 255) / 256, 8 * kNumSMs);
  split_planes_kernel<<<g, 256, 0, st>>>(src, ld, rows, cols, hi, lo, ldo, info);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_gemm(const Operand& A, const Operand& B, bool b_mn, const Job& job, int grid, int* info,
                        cudaStream_t st) {
  if (grid <= 0) return cudaSuccess;
  CUtensorMap ah, al, bh, bl;
  if (!make_map(&ah, A.hi, A.rows, A.cols, A.ld, kKC, kM, false) ||
      !make_map(&al, A.lo, A.rows, A.cols, A.ld, kKC, kM, false))
    return cudaErrorInvalidValue;
  if (b_mn) {
    if (!make_map(&bh, B.hi, B.rows, B.cols, B.ld, 32, kKC, true) ||
        !make_map(&bl, B.lo, B.rows, B.cols, B.ld, 32, kKC, true))
      return cudaErrorInvalidValue;
  } else {
    if (!make_map(&bh, B.hi, B.rows, B.cols, B.ld, kKC, kN, false) ||
        !make_map(&bl, B.lo, B.rows, B.cols, B.ld, kKC, kN, false))
      return cudaErrorInvalidValue;
  }
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(gemm_tf32x3_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
    attr = true;
  }
  gemm_tf32x3_kernel<<<grid, kThreads, kSmem, st>>>(ah, al, bh, bl, job, b_mn ? 1 : 0, info);
  count_launches(1);
  if (job.mode == 2 && job.nsplit > 1) {
    const long long quads = (long long)(job.nblk - 1 - job.s) * (kM * kN / 4);
    const int g = (int)std::min<long long>((quads + 255) / 256, 8 * kNumSMs);
    rowsplit_reduce_kernel<<<g, 256, 0, st>>>(job, info);
    count_launches(1);
  }
  return cudaGetLastError();
}

}  // namespace tc
}  // namespace sgpt
