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
// Used for the panel products, the rank-128 to rank-512 updates and the
// triangular inverse of the factorisation and for the lazy trailing update of
// the OBS sweep. The same kernel also runs plain bf16 products (one
// tcgen05.mma.kind::f16 per K step of 16, K-major operands, fp32
// accumulation), the forward passes between the layers of a block.
//
// Output tiles of 128 x 128, K in stages of 32 (one 128-byte swizzle row of
// fp32) through a two-stage TMA ring of 64 KB stages (no multicast). Persistent: one CTA per
// SM walks its share of the launch's tiles; warp 0 lane 0 loads, warp 1 lane
// 0 issues MMAs, warps 2-9 drain TMEM, combine it with the C tile that TMA
// brought into shared memory one tile ahead, and write whole rows per warp
// instruction (coalesced). TMEM accumulates at most 128
// of K per accumulator; two accumulators alternate, so a tile's epilogue
// overlaps the next tile's main loop and a longer K is summed chunk by chunk
// in FP32 registers (a long accumulation inside TMEM loses accuracy).
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

constexpr int kM = 128, kN = 128;
// The two arithmetic kinds of the kernel. kKindTf32x3: fp32 operands as hi/lo
// TF32 planes, three tcgen05.mma.kind::tf32 products per K step of 8. kKindBf16:
// bf16 operands, one tcgen05.mma.kind::f16 product per K step of 16. A stage
// holds one 128-byte swizzle row of K per operand row in either case (32
// fp32 or 64 bf16), so a plane is 16 KB; the bf16 ring has four stages in the
// shared memory the fp32 one fills with two.
constexpr int kKindTf32x3 = 0, kKindBf16 = 1;
template <int KIND>
struct Cfg {
  static constexpr int KC = KIND == kKindTf32x3 ? 32 : 64;     // K per stage
  static constexpr int PLANES = KIND == kKindTf32x3 ? 2 : 1;   // planes per operand
  static constexpr int STAGES = KIND == kKindTf32x3 ? 2 : 4;
  static constexpr int KSTEP = KIND == kKindTf32x3 ? 8 : 16;   // K per MMA
};
constexpr int kPlane = kM * 128;                // 16 KB: one operand plane of one stage
template <int KIND>
constexpr int stage_bytes() { return 2 * Cfg<KIND>::PLANES * kPlane; }
constexpr int kRingBytes = 2 * stage_bytes<kKindTf32x3>();   // 128 KB, both kinds
static_assert(Cfg<kKindBf16>::STAGES * stage_bytes<kKindBf16>() == kRingBytes, "same ring for both kinds");
constexpr int kEpiWarps = 8;                    // two per TMEM lane quadrant, 64 columns each
constexpr int kThreads = 64 + 32 * kEpiWarps;   // producer, MMA issuer, epilogue
// Epilogue tile: 128 x 128 fp32 as four 32-column groups of 128 rows x 128
// bytes, 16-byte chunks XOR-swizzled by row % 8 (TMA's 128-byte swizzle).
constexpr size_t kStagingBytes = (size_t)kM * kN * 4;
constexpr size_t kSmem = (size_t)kRingBytes + kStagingBytes + 1024 + 256;
constexpr int kTmemCols = 2 * kN;               // two accumulators: one fills while one drains

template <int KIND>
__host__ __device__ constexpr uint32_t make_idesc(bool b_mn) {
  // D fp32; A and B tf32 (2) or bf16 (1); B MN-major bit 16; N/8, M/16
  return (1u << 4) | ((KIND == kKindTf32x3 ? 2u : 1u) << 7) | ((KIND == kKindTf32x3 ? 2u : 1u) << 10) |
         ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(kN >> 3) << 17) | ((uint32_t)(kM >> 4) << 24);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// K-major operand, 128-byte swizzle (a K stage of 32 fp32 is one 128-byte
// row): 8-row groups of 1024 bytes.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3fff);
  d |= (uint64_t)1 << 16;                         // leading byte offset (unused when swizzled)
  d |= (uint64_t)(1024 >> 4) << 32;               // stride byte offset: next 8 rows
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;                         // SWIZZLE_128B
  return d;
}
// MN-major 32-bit operand: the 128-byte swizzle with 32-byte granules
// (descriptor layout SWIZZLE_128B_BASE32B, filled by TMA's
// SWIZZLE_128B_ATOM_32B). Atoms are 32 columns x 4 K rows (512 bytes);
// LBO = next 32 columns (one 32-column x kKC-row TMA box), SBO = next
// 4 K rows. The plain 128-byte swizzle (16-byte granules) is not a valid
// MN-major form for 32-bit elements.
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3fff);
  d |= (uint64_t)((Cfg<kKindTf32x3>::KC * 128) >> 4) << 16;
  d |= (uint64_t)(512 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)1 << 61;
  return d;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
// 16-byte shared-memory accesses by 32-bit shared address (the epilogue
// tile's address is computed by aligning an integer, which the compiler can
// no longer see as shared memory).
__device__ __forceinline__ float4 lds4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts4(uint32_t addr, float4 v) {
  asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
               : "memory");
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
__device__ __forceinline__ void mma_bf16(uint32_t tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem),
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


// Work item w of a launch: its output tile (m0, n0) and K range [kb, ke).
struct Item {
  int m0, n0, kb, ke;
};

// Dense grids are walked in groups of kGroupRows tile rows, rows fastest
// inside a group: the CTAs resident together share the A panels of the
// group's rows and the B panels of a few tile columns, which stay in L2
// while the CTAs stream K (a row-major order walks every column of B for
// each few rows and reads B from DRAM again and again when it exceeds L2).
constexpr int kGroupRows = 16;

__device__ __forceinline__ Item decode_item(const Job& job, int w) {
  Item it{0, 0, 0, 0};
  if (job.mode == 0) {
    const int per_group = kGroupRows * job.nt;
    const int g = w / per_group;
    const int first = g * kGroupRows;
    const int rows = min(kGroupRows, job.mt - first);
    const int r = w - g * per_group;
    it.m0 = (first + r % rows) * kM;
    it.n0 = (r / rows) * kN;
    it.ke = job.kdim;
  } else if (job.mode == 1) {
    int i, j;
    tri_index(job.t0 + w, i, j);
    it.m0 = i * kM;
    it.n0 = j * kN;
    it.ke = job.kdim;
  }
  return it;
}

// Persistent: CTA c takes items c, c + gridDim.x, ... The TMA ring runs
// through the K steps of all its items without a break; the MMA warp fills
// one TMEM accumulator per unit of at most kChunk K steps, alternating two,
// while the epilogue warps drain the other, so one tile's epilogue overlaps
// the next tile's main loop.
template <int KIND>
__global__ void __launch_bounds__(kThreads, 1) gemm_tc_kernel(
    const __grid_constant__ CUtensorMap a_hi, const __grid_constant__ CUtensorMap a_lo,
    const __grid_constant__ CUtensorMap b_hi, const __grid_constant__ CUtensorMap b_lo, const Job job,
    const __grid_constant__ CUtensorMap c_map, const int b_mn, const int items, int* info,
    const long long wait_cycles) {
  constexpr int kStages = Cfg<KIND>::STAGES, kKC = Cfg<KIND>::KC, kPl = Cfg<KIND>::PLANES;
  constexpr int kStageBytes = stage_bytes<KIND>();
  constexpr int kChunk = 128 / kKC;             // stages (128 of K) per TMEM accumulation
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* T = smem + kStages * kStageBytes;   // epilogue tile (C in, result out)
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes + kStagingBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 6);
  __shared__ int failed;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (cta_info_set(info)) return;

  const uint32_t idesc = make_idesc<KIND>(b_mn != 0);
  const uint32_t s0 = smem_u32(smem);
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + kStages);
  const uint32_t tfull0 = smem_u32(bars + 2 * kStages), tempty0 = tfull0 + 16, cfull = tfull0 + 32;
  const uint32_t mdone = tfull0 + 40;         // every MMA this CTA issued has completed
  if (threadIdx.x == 0) {
    // descriptors into the TMA unit's cache before the first copy needs them
    const CUtensorMap* maps[5] = {&a_hi, &a_lo, &b_hi, &b_lo, &c_map};
    for (int i = 0; i < 5; ++i)
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(maps[i])) : "memory");
    failed = 0;
    for (int st = 0; st < kStages; ++st) {
      mbar_init(full0 + 8 * st, 1);
      mbar_init(empty0 + 8 * st, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull0 + 8 * b, 1);
      mbar_init(tempty0 + 8 * b, kEpiWarps);
    }
    mbar_init(cfull, 1);
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

  if (warp == 0) {
    if (lane == 0) {
      // TMA producer: the K steps of every item, one stage each
      int g = 0;                                  // stage uses so far
      for (int w = blockIdx.x; w < items && !failed; w += gridDim.x) {
        const Item it = decode_item(job, w);
        const int iters = (it.ke - it.kb + kKC - 1) / kKC;
        for (int i = 0; i < iters; ++i, ++g) {
          const int st = g % kStages;
          if (g >= kStages && !mbar_wait(empty0 + 8 * st, ((g / kStages) & 1) ^ 1, wait_cycles)) {
            failed = 1;
            break;
          }
          const uint32_t bar = full0 + 8 * st;
          mbar_expect_tx(bar, kStageBytes);
          const uint32_t sa = s0 + st * kStageBytes;
          const int k = it.kb + i * kKC;
          tma_2d(sa, &a_hi, bar, job.a_x0 + k, job.a_y0 + it.m0);
          if (kPl == 2) tma_2d(sa + kPlane, &a_lo, bar, job.a_x0 + k, job.a_y0 + it.m0);
          if (KIND == kKindBf16) {
            tma_2d(sa + kPlane, &b_hi, bar, job.b_x0 + k, job.b_y0 + it.n0);
          } else if (b_mn) {
#pragma unroll
            for (int c = 0; c < kN / 32; ++c) {
              tma_2d(sa + 2 * kPlane + c * kKC * 128, &b_hi, bar, job.b_x0 + it.n0 + 32 * c, job.b_y0 + k);
              tma_2d(sa + 3 * kPlane + c * kKC * 128, &b_lo, bar, job.b_x0 + it.n0 + 32 * c, job.b_y0 + k);
            }
          } else {
            tma_2d(sa + 2 * kPlane, &b_hi, bar, job.b_x0 + k, job.b_y0 + it.n0);
            tma_2d(sa + 3 * kPlane, &b_lo, bar, job.b_x0 + k, job.b_y0 + it.n0);
          }
        }
      }
      // never leave with copies in flight: wait for every stage still armed
      for (int x = (g > kStages ? g - kStages : 0); x < g; ++x)
        if (!mbar_wait(full0 + 8 * (x % kStages), (x / kStages) & 1, kDrainCycles)) failed = 1;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // MMA issuer: unit u (<= kChunk K steps of one item) into TMEM buffer u & 1
      int g = 0, u = 0;
      for (int w = blockIdx.x; w < items && !failed; w += gridDim.x) {
        const Item it = decode_item(job, w);
        const int iters = (it.ke - it.kb + kKC - 1) / kKC;
        for (int c0 = 0; c0 < iters && !failed; c0 += kChunk, ++u) {
          const int b = u & 1;
          if (u >= 2 && !mbar_wait(tempty0 + 8 * b, ((u >> 1) - 1) & 1, wait_cycles)) {
            failed = 1;
            break;
          }
          asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
          const uint32_t acc_t = tmem + (uint32_t)(b * kN);
          const int c1 = min(iters, c0 + kChunk);
          for (int i = c0; i < c1; ++i, ++g) {
            const int st = g % kStages;
            if (!mbar_wait(full0 + 8 * st, (g / kStages) & 1, wait_cycles)) {
              failed = 1;
              break;
            }
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const uint32_t sa = s0 + st * kStageBytes;
#pragma unroll
            for (int ks = 0; ks < kKC / Cfg<KIND>::KSTEP; ++ks) {
              if constexpr (KIND == kKindBf16) {
                // one K step of 16 bf16 is 32 bytes of each operand row
                mma_bf16(acc_t, kmajor_desc(sa + ks * 32), kmajor_desc(sa + kPlane + ks * 32), idesc,
                         (i == c0 && ks == 0) ? 0u : 1u);
                continue;
              }
              const uint64_t ah = kmajor_desc(sa + ks * 32), al = kmajor_desc(sa + kPlane + ks * 32);
              uint64_t bh, bl;
              if (b_mn) {
                bh = mnmajor_desc(sa + 2 * kPlane + ks * 1024);
                bl = mnmajor_desc(sa + 3 * kPlane + ks * 1024);
              } else {
                bh = kmajor_desc(sa + 2 * kPlane + ks * 32);
                bl = kmajor_desc(sa + 3 * kPlane + ks * 32);
              }
              const uint32_t first = (i == c0 && ks == 0) ? 0u : 1u;
              mma_tf32(acc_t, al, bh, idesc, first);   // small terms first
              mma_tf32(acc_t, ah, bl, idesc, 1u);
              mma_tf32(acc_t, ah, bh, idesc, 1u);
            }
            mma_commit(empty0 + 8 * st);
          }
          mma_commit(tfull0 + 8 * b);
        }
      }
      // never free TMEM under a running MMA (after a timeout the epilogue
      // may not have waited for the last ones): wait for all of them
      mma_commit(mdone);
      if (!mbar_wait(mdone, 0, kDrainCycles)) failed = 1;
    }
  } else {
    // Epilogue warps: warp w reads TMEM lanes 32*(w%4).. (tile rows) and
    // columns 64*h.., h = (w-2)/4, and sums an item's units in FP32
    // registers (one unit: just copied). C arrives by TMA in the epilogue
    // tile, requested one item ahead; each thread forms alpha * acc +
    // beta * C for its row in place, and the warps write whole rows out
    // (coalesced) with the optional hi/lo planes.
    const int q = warp & 3, h = (warp - 2) >> 2;
    const int m = q * 32 + lane;                  // tile row = TMEM lane
    const int ew = warp - 2;                      // 0..7: rows 16*ew.. in the write-out
    const bool read_c = job.C != nullptr && job.beta != 0.f;
    const long long ldp = job.ldp ? job.ldp : job.ldc;
    const bool issuer = (warp == 2 && lane == 0);
    const uint32_t t_s = smem_u32(T);             // the epilogue tile as a shared address
    auto load_c = [&](int ww) {                   // TMA of item ww's C tile (four 32-column groups)
      const Item nx = decode_item(job, ww);
      mbar_expect_tx(cfull, (uint32_t)kStagingBytes);
#pragma unroll
      for (int g4 = 0; g4 < 4; ++g4)
        tma_2d(smem_u32(T) + g4 * (kM * 128), &c_map, cfull, job.c_col0 + nx.n0 + 32 * g4, job.c_row0 + nx.m0);
    };
    int c_issued = 0;                             // C tiles requested (issuer only)
    if (read_c && issuer && (int)blockIdx.x < items) {
      load_c(blockIdx.x);
      ++c_issued;
    }
    int u = 0, nitem = 0;
    for (int w = blockIdx.x; w < items; w += gridDim.x, ++nitem) {
      const Item it = decode_item(job, w);
      const int iters = (it.ke - it.kb + kKC - 1) / kKC;
      float acc[64];
#pragma unroll
      for (int e = 0; e < 64; ++e) acc[e] = 0.f;
      for (int c0 = 0; c0 < iters; c0 += kChunk, ++u) {
        const int b = u & 1;
        // one decision per warp: the TMEM loads below are warp-collective
        int bad = failed;
        if (!bad) bad = !mbar_wait(tfull0 + 8 * b, (u >> 1) & 1, wait_cycles);
        bad = __any_sync(0xffffffffu, bad);
        if (bad) failed = 1;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        if (!bad) {
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            uint32_t v[32];
            tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * kN + h * 64 + cc * 32), v);
#pragma unroll
            for (int e = 0; e < 32; ++e) acc[cc * 32 + e] += __uint_as_float(v[e]);
          }
        }
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty0 + 8 * b);
      }
      if (read_c && !failed && !mbar_wait(cfull, nitem & 1, wait_cycles)) failed = 1;
      // this thread's 64 columns = 16 chunks of 16 bytes in groups 2h, 2h+1
#pragma unroll
      for (int cj = 0; cj < 16; ++cj) {
        const int g4 = 2 * h + (cj >> 3), j = cj & 7;
        const uint32_t pch = t_s + g4 * (kM * 128) + m * 128 + ((j ^ (m & 7)) << 4);
        float4 o = make_float4(acc[4 * cj], acc[4 * cj + 1], acc[4 * cj + 2], acc[4 * cj + 3]);
        const float4 cv = read_c ? lds4(pch) : make_float4(0.f, 0.f, 0.f, 0.f);
        o = make_float4(fmaf(job.alpha, o.x, job.beta * cv.x), fmaf(job.alpha, o.y, job.beta * cv.y),
                        fmaf(job.alpha, o.z, job.beta * cv.z), fmaf(job.alpha, o.w, job.beta * cv.w));
        sts4(pch, o);
      }
      asm volatile("bar.sync 1, %0;" ::"r"(32 * kEpiWarps) : "memory");
      if (!failed) {
        const bool planes = job.C_hi != nullptr && (!job.planes_one_col || it.n0 == job.planes_n0) &&
                            (!job.planes_one_row || it.m0 == job.planes_m0);
        const int cn = lane * 4;                  // lane = 16-byte chunk of the row
        const bool col_ok = it.n0 + cn < job.Nlim;
        const int g4 = lane >> 3, j = lane & 7;
#pragma unroll 4
        for (int x = 0; x < 16; ++x) {
          const int mr = ew * 16 + x;
          const float4 o = lds4(t_s + g4 * (kM * 128) + mr * 128 + ((j ^ (mr & 7)) << 4));
          const int row = it.m0 + mr;
          if (row >= job.Mlim || !col_ok) continue;
          if (job.C) st4(job.C + (long long)(job.c_row0 + row) * job.ldc + job.c_col0 + it.n0 + cn, o);
          if (planes) {
            const long long off =
                (long long)(job.c_row0 + row - job.p_row0) * ldp + job.c_col0 + it.n0 + cn - job.p_col0;
            const float4 hv = make_float4(tf32_hi(o.x), tf32_hi(o.y), tf32_hi(o.z), tf32_hi(o.w));
            st4(job.C_hi + off, hv);
            st4(job.C_lo + off, make_float4(o.x - hv.x, o.y - hv.y, o.z - hv.z, o.w - hv.w));
          }
        }
      }
      // every read of the tile is done: the next item's C may come in
      asm volatile("bar.sync 1, %0;" ::"r"(32 * kEpiWarps) : "memory");
      if (read_c && issuer && !failed && w + (int)gridDim.x < items) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        load_c(w + gridDim.x);
        ++c_issued;
      }
    }
    // never leave with a C copy in flight (after a timeout some were not waited for)
    if (read_c && issuer && c_issued > 0) mbar_wait(cfull, (c_issued - 1) & 1, kDrainCycles);
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (failed && threadIdx.x == 0) set_info(info, SGPT_INFO_TIMEOUT);
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
}

// ------------------------------------------------------------- wide tiles
//
// 128 x 256 output tiles for the bf16 products on dense grids (mode 0). Per
// K stage a CTA loads 128 rows of A and 256 of B, so each byte of operands
// feeds twice the products of a 128 x 128 tile: with 128 x 128 tiles the
// tensor pipe needs more operand bytes per cycle per SM than L2 delivers
// (the 8192 x 5120 x 25600 product: 0.41 -> 0.63 of the bf16 peak). Four
// 48 KB stages of 64 of K (128-byte swizzle); two 256-column TMEM
// accumulators (all 512 columns); warp 0 loads, warp 1 issues N = 256 MMAs,
// warps 2-9 drain TMEM (lane quadrant w % 4, columns 128 (w - 2) / 4 ..) and
// write their rows of C straight from registers (16-byte accesses, each
// thread its own row). The bf16 products have long K and no C to read, so
// the epilogue is a small part of a tile. Every wait is bounded as in the
// kernel above.
namespace {
constexpr int kWN = 256, kWStages = 4, kWKC = 64;
constexpr int kWAPlane = kM * kWKC * 2;          // 16 KB
constexpr int kWBPlane = kWN * kWKC * 2;         // 32 KB
constexpr int kWStage = kWAPlane + kWBPlane;     // 48 KB
constexpr size_t kWideSmem = (size_t)kWStages * kWStage + 1024 + 256;
constexpr int kWTmemCols = 2 * kWN;
}  // namespace

__global__ void __launch_bounds__(kThreads, 1) gemm_wide_bf16_kernel(
    const __grid_constant__ CUtensorMap a_map, const __grid_constant__ CUtensorMap b_map, const Job job,
    const int items, int* info, const long long wait_cycles) {
  constexpr int kChunk = 128 / kWKC;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kWStages * kWStage);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kWStages + 6);
  __shared__ int failed;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (cta_info_set(info)) return;

  // D fp32, A and B bf16, both K-major, N = 256, M = 128
  constexpr uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kWN >> 3) << 17) |
                             ((uint32_t)(kM >> 4) << 24);
  const uint32_t s0 = smem_u32(smem);
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + kWStages);
  const uint32_t tfull0 = smem_u32(bars + 2 * kWStages), tempty0 = tfull0 + 16, mdone = tfull0 + 32;
  if (threadIdx.x == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&a_map)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&b_map)) : "memory");
    failed = 0;
    for (int st = 0; st < kWStages; ++st) {
      mbar_init(full0 + 8 * st, 1);
      mbar_init(empty0 + 8 * st, 1);
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
                 "r"(kWTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;

  auto decode = [&](int w, int& m0, int& n0) {
    const int per_group = kGroupRows * job.nt;
    const int g = w / per_group;
    const int first = g * kGroupRows;
    const int rows = min(kGroupRows, job.mt - first);
    const int r = w - g * per_group;
    m0 = (first + r % rows) * kM;
    n0 = (r / rows) * kWN;
  };
  const int iters = (job.kdim + kWKC - 1) / kWKC;

  if (warp == 0) {
    if (lane == 0) {
      int g = 0;
      for (int w = blockIdx.x; w < items && !failed; w += gridDim.x) {
        int m0, n0;
        decode(w, m0, n0);
        for (int i = 0; i < iters; ++i, ++g) {
          const int st = g % kWStages;
          if (g >= kWStages && !mbar_wait(empty0 + 8 * st, ((g / kWStages) & 1) ^ 1, wait_cycles)) {
            failed = 1;
            break;
          }
          const uint32_t bar = full0 + 8 * st;
          mbar_expect_tx(bar, kWStage);
          const uint32_t sa = s0 + st * kWStage;
          const int k = i * kWKC;
          tma_2d(sa, &a_map, bar, job.a_x0 + k, job.a_y0 + m0);
          tma_2d(sa + kWAPlane, &b_map, bar, job.b_x0 + k, job.b_y0 + n0);
        }
      }
      for (int x = (g > kWStages ? g - kWStages : 0); x < g; ++x)
        if (!mbar_wait(full0 + 8 * (x % kWStages), (x / kWStages) & 1, kDrainCycles)) failed = 1;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int g = 0, u = 0;
      for (int w = blockIdx.x; w < items && !failed; w += gridDim.x) {
        for (int c0 = 0; c0 < iters && !failed; c0 += kChunk, ++u) {
          const int b = u & 1;
          if (u >= 2 && !mbar_wait(tempty0 + 8 * b, ((u >> 1) - 1) & 1, wait_cycles)) {
            failed = 1;
            break;
          }
          asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
          const uint32_t acc_t = tmem + (uint32_t)(b * kWN);
          const int c1 = min(iters, c0 + kChunk);
          for (int i = c0; i < c1; ++i, ++g) {
            const int st = g % kWStages;
            if (!mbar_wait(full0 + 8 * st, (g / kWStages) & 1, wait_cycles)) {
              failed = 1;
              break;
            }
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const uint32_t sa = s0 + st * kWStage;
#pragma unroll
            for (int ks = 0; ks < kWKC / 16; ++ks)   // K steps of 16 bf16 = 32 bytes of each row
              mma_bf16(acc_t, kmajor_desc(sa + ks * 32), kmajor_desc(sa + kWAPlane + ks * 32), idesc,
                       (i == c0 && ks == 0) ? 0u : 1u);
            mma_commit(empty0 + 8 * st);
          }
          mma_commit(tfull0 + 8 * b);
        }
      }
      // never free TMEM under a running MMA
      mma_commit(mdone);
      if (!mbar_wait(mdone, 0, kDrainCycles)) failed = 1;
    }
  } else {
    const int q = warp & 3, h = (warp - 2) >> 2;
    const int m = q * 32 + lane;                    // tile row = TMEM lane
    const bool read_c = job.C != nullptr && job.beta != 0.f;
    int u = 0;
    for (int w = blockIdx.x; w < items; w += gridDim.x) {
      int m0, n0;
      decode(w, m0, n0);
      float acc[128];
#pragma unroll
      for (int e = 0; e < 128; ++e) acc[e] = 0.f;
      for (int c0 = 0; c0 < iters; c0 += kChunk, ++u) {
        const int b = u & 1;
        // one decision per warp: the TMEM loads below are warp-collective
        int bad = failed;
        if (!bad) bad = !mbar_wait(tfull0 + 8 * b, (u >> 1) & 1, wait_cycles);
        bad = __any_sync(0xffffffffu, bad);
        if (bad) failed = 1;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        if (!bad) {
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            uint32_t v[32];
            tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * kWN + h * 128 + cc * 32), v);
#pragma unroll
            for (int e = 0; e < 32; ++e) acc[cc * 32 + e] += __uint_as_float(v[e]);
          }
        }
        asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty0 + 8 * b);
      }
      const int row = m0 + m;
      if (!failed && row < job.Mlim && job.C) {
        float* crow = job.C + (long long)(job.c_row0 + row) * job.ldc + job.c_col0;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int col = n0 + h * 128 + 4 * j;
          if (col >= job.Nlim) continue;
          float4 o = make_float4(acc[4 * j], acc[4 * j + 1], acc[4 * j + 2], acc[4 * j + 3]);
          const float4 cv = read_c ? ld4(crow + col) : make_float4(0.f, 0.f, 0.f, 0.f);
          o = make_float4(fmaf(job.alpha, o.x, job.beta * cv.x), fmaf(job.alpha, o.y, job.beta * cv.y),
                          fmaf(job.alpha, o.z, job.beta * cv.z), fmaf(job.alpha, o.w, job.beta * cv.w));
          st4(crow + col, o);
        }
      }
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (failed && threadIdx.x == 0) set_info(info, SGPT_INFO_TIMEOUT);
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kWTmemCols));
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
// ld; box = box_x (inner, fp32 elements) x box_y rows; 128-byte swizzle for
// K-major operands (32-float rows), 128-byte swizzle with 32-byte granules
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
             mn_major ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor map over a row-major bf16 matrix [rows x cols] (ld in elements):
// boxes of 64 elements (one 128-byte swizzle row) x box_y rows.
bool make_map_bf16(CUtensorMap* m, const uint16_t* p, long long rows, long long cols, long long ld,
                   int box_y = kM) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  const cuuint32_t box[2] = {(cuuint32_t)Cfg<kKindBf16>::KC, (cuuint32_t)box_y};
  const cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(p), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor map over C for the epilogue: boxes of 32 columns x 128 rows with the
// 128-byte swizzle.
bool make_map_c(CUtensorMap* m, const float* p, long long rows, long long cols, long long ld) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)ld * 4};
  const cuuint32_t box[2] = {32, (cuuint32_t)kM};
  const cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(p), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
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

namespace {
// Kernel attributes, the persistent grid, C's map and the launch: shared by
// both arithmetic kinds.
template <int KIND>
cudaError_t launch_kind(const CUtensorMap& ah, const CUtensorMap& al, const CUtensorMap& bh, const CUtensorMap& bl,
                        bool b_mn, const Job& job, int grid, int* info, cudaStream_t st) {
  static PerDevice attrs;
  cudaError_t ea = once_per_device(attrs, [] {
    return cudaFuncSetAttribute(gemm_tc_kernel<KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
  });
  if (ea != cudaSuccess) return ea;
  // persistent: one CTA per SM at most, fewer when the job leaves SMs to others
  const int ctas = std::min(grid, job.max_ctas > 0 ? std::min(job.max_ctas, kNumSMs) : kNumSMs);
  // C comes in by TMA when it is read (beta != 0); otherwise the map is unused
  CUtensorMap cm = ah;
  if (job.C && job.beta != 0.f &&
      !make_map_c(&cm, job.C, (long long)job.c_row0 + job.Mlim, (long long)job.c_col0 + job.Nlim, job.ldc))
    return cudaErrorInvalidValue;
  gemm_tc_kernel<KIND><<<ctas, kThreads, kSmem, st>>>(ah, al, bh, bl, job, cm, b_mn ? 1 : 0, grid, info,
                                                      wait_limit_cycles());
  count_launches(1);
  return cudaGetLastError();
}
}  // namespace

namespace {
cudaError_t launch_wide_bf16(const CUtensorMap& a_map, const CUtensorMap& b_map, const Job& job, int items, int* info,
                             cudaStream_t st) {
  static PerDevice attrs;
  cudaError_t ea = once_per_device(attrs, [] {
    return cudaFuncSetAttribute(gemm_wide_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kWideSmem);
  });
  if (ea != cudaSuccess) return ea;
  const int ctas = std::min(items, job.max_ctas > 0 ? std::min(job.max_ctas, kNumSMs) : kNumSMs);
  gemm_wide_bf16_kernel<<<ctas, kThreads, kWideSmem, st>>>(a_map, b_map, job, items, info, wait_limit_cycles());
  count_launches(1);
  return cudaGetLastError();
}

// bf16 dense grids more than one tile column wide go to the 128 x 256 tiles
// (their job.nt counted in 256-column tiles). The 3xTF32 jobs stay on the
// 128 x 128 tiles: they are read-modify-write updates with short K (128 or
// 256), whose time is in the epilogue's C traffic, and the same wide tiles
// with a register-direct epilogue measured slower for them than the
// TMA-fed, coalesced one (factor 125 -> 149 ms, sweep 64 -> 103 ms on the
// default workload).
bool use_wide_bf16(const Job& job) { return job.mode == 0 && job.Nlim > kN; }
}  // namespace

cudaError_t launch_gemm(const Operand& A, const Operand& B, bool b_mn, const Job& job, int grid, int* info,
                        cudaStream_t st) {
  if (grid <= 0) return cudaSuccess;
  constexpr int kKC = Cfg<kKindTf32x3>::KC;
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
  return launch_kind<kKindTf32x3>(ah, al, bh, bl, b_mn, job, grid, info, st);
}

cudaError_t launch_gemm_bf16(const OperandBf16& A, const OperandBf16& B, const Job& job, int grid, int* info,
                             cudaStream_t st) {
  if (grid <= 0) return cudaSuccess;
  if (use_wide_bf16(job)) {
    CUtensorMap ah, bh;
    if (!make_map_bf16(&ah, A.p, A.rows, A.cols, A.ld) || !make_map_bf16(&bh, B.p, B.rows, B.cols, B.ld, kWN))
      return cudaErrorInvalidValue;
    Job w = job;
    w.nt = cdiv(job.Nlim, kWN);
    return launch_wide_bf16(ah, bh, w, w.mt * w.nt, info, st);
  }
  CUtensorMap ah, bh;
  if (!make_map_bf16(&ah, A.p, A.rows, A.cols, A.ld) || !make_map_bf16(&bh, B.p, B.rows, B.cols, B.ld))
    return cudaErrorInvalidValue;
  return launch_kind<kKindBf16>(ah, ah, bh, bh, false, job, grid, info, st);
}

}  // namespace tc
}  // namespace sgpt
