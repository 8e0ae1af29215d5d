// A consumer of the 2:4 output: Y = X W^T computed from the packed weights
// (the kept values and their 2-bit positions) on the sparse tensor cores,
// tcgen05.mma.sp.kind::f16 (2:4 along K on the A operand). The packing
// follows the 2:4 production guide (oh-bug.com, section on the 2:4
// mechanism: two of every four consecutive weights along the reduction axis
// are kept and their positions recorded in 2-bit metadata); running the
// packed form through the hardware's sparse product checks that format
// semantically.
//
// The sparse operand is A = W^: M = output rows, K = inputs; B = X (N =
// tokens), both K-major, so D = W^ X^T lands in TMEM with one output row per
// lane, and each lane writes its row's values across a token tile, which for
// Y [n x d_out] is 32 consecutive floats per warp instruction.
//
// The hardware reads a K = 32 slab's metadata for 128 rows from one 32-bit
// TMEM column in which rows and K halves are interleaved across lanes: lane
// i = (r % 8) + 8 h + 16 (r / 16) holds, in bits 0-15, the four group codes
// of row r (r % 16 < 8) for K half h, and in bits 16-31 the same for row
// r + 8. A group code is the library's own 4-bit code a | b << 2 (a < b the
// kept positions), so the re-arrangement of the packed metadata words is a
// permutation of 16-bit pieces. It is done once per weight matrix
// (tile_meta_kernel) into "meta tiles": for every 256-row tile and 128-K
// stage, 4 KB holding, for each of the two 128-row halves, 128 lanes x 4
// slab columns, lane-major, in exactly the order tcgen05.cp copies into
// TMEM.
//
// sparse24_gemm_kernel: persistent, one CTA per SM, warp-specialized.
// Output tiles are 256 rows x 128 tokens (two M = 128 accumulators sharing
// each X tile, so an X byte feeds twice the products of a 128-row tile).
// Warp 0 lane 0 issues, per 128-K stage, TMA copies of the two halves' 64
// stored values per row (2 x 16 KB), 128 tokens x 128 K of X (2 x 16 KB)
// and the stage's 4 KB meta tile, into one of three 68 KB stages; warp 1
// lane 0 copies the meta tile into TMEM (tcgen05.cp, ordered before the
// MMAs the same thread issues next) and issues 8 sparse MMAs (2 halves x 4
// K = 32 slabs, N = 128); warps 2-9 drain the accumulators (256 TMEM
// columns) into registers, release them to the next tile's MMAs and write
// their rows of Y while those run. Tiles are walked in groups of 16 tile
// rows (rows fastest) so that resident CTAs share W and X panels in L2.
// Every wait on another role is bounded by the launch's wait limit; a CTA
// that gives up records SGPT_INFO_TIMEOUT, drains its own copies and MMAs
// (kDrainCycles) and frees TMEM.
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/sgpt.h"
#include "common.cuh"
#include "kernels.h"

namespace sgpt {

namespace {

constexpr int kCM = 256, kCN = 128, kCK = 128;      // output tile (rows x tokens), logical K per stage
constexpr int kCStages = 3;
constexpr int kCGroupRows = 16;
constexpr int kCThreads = 320;                      // producer, MMA, 8 epilogue warps
constexpr int kCEpiWarps = 8;
constexpr int kCHalfA = 128 * (kCK / 2) * 2;        // 16 KB: 128 rows x 64 stored bf16
constexpr int kCBox = kCN * 64 * 2;                 // 16 KB: 128 tokens x 64 K
constexpr int kCMeta = 2 * 128 * 16;                // 4 KB: two halves x 128 lanes x 4 words
constexpr int kCOffB = 2 * kCHalfA, kCOffMeta = kCOffB + 2 * kCBox;
constexpr int kCStage = kCOffMeta + kCMeta;         // 68 KB, a multiple of 1024
constexpr size_t kCSmem = (size_t)kCStages * kCStage + 1024 + 256;
constexpr int kCTmemCols = 512;                     // 2 x 128 accumulator columns + metadata
constexpr int kCMetaCol = 256;                      // stage s, half h: columns 256 + 8 s + 4 h ..
constexpr uint32_t kPad = 0x4444u;                  // the valid code 0 | 1 << 2 in every group

static_assert(kCStage % 1024 == 0, "stages keep the 1024-byte swizzle alignment");
static_assert(kCSmem <= 232448, "dynamic shared memory per CTA");
static_assert(kCMetaCol + 8 * kCStages <= kCTmemCols, "metadata columns fit");

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
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
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.b32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait (short limits poll without suspending, as in the GEMMs).
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
// Contiguous global -> shared bulk copy (16-byte aligned, size % 16 == 0).
__device__ __forceinline__ void bulk_copy(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
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

// K-major operand, 128-byte swizzle: 8-row groups of 1024 bytes.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3fff);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}
// The tcgen05.cp source: 128 rows of 16 bytes, row i at byte 16 i (no
// swizzle; 8-row core matrices of 128 bytes, one after the other).
__device__ __forceinline__ uint64_t meta_src_desc(uint32_t addr) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3fff);
  d |= (uint64_t)(128 >> 4) << 16;
  d |= (uint64_t)(128 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  return d;
}

// D fp32, A and B bf16, both K-major, sparse A (bit 2), N/8, M/16.
constexpr uint32_t kSpIdesc = (1u << 2) | (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kCN >> 3) << 17) |
                              ((uint32_t)(128 >> 4) << 24);

__device__ __forceinline__ void mma_sp(uint32_t acc_t, uint64_t ad, uint64_t bd, uint32_t idesc, uint32_t e_addr,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.sp.cta_group::1.kind::f16 [%0], %1, %2, [%5], %3, {%6, %7, %8, %9}, p;\n}\n" ::"r"(acc_t),
      "l"(ad), "l"(bd), "r"(idesc), "r"(accumulate), "r"(e_addr), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}

// One 32-bit word of the meta tiles per thread: tile (mt, kt), half h, lane
// i, slab j at word ((mt * kt_count + kt) * 2 + h) * 512 + 4 i + j.
__global__ void tile_meta_kernel(const uint32_t* __restrict__ meta, int rows, int d, int kt_count, long long words,
                                 uint32_t* __restrict__ tiles) {
  const long long w = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (w >= words) return;
  const int j = (int)(w & 3), i = (int)((w >> 2) & 127);
  const long long t = w >> 9;                   // (mt * kt_count + kt) * 2 + half
  const int half = (int)(t & 1);
  const long long mk = t >> 1;
  const int kt = (int)(mk % kt_count), mt = (int)(mk / kt_count);
  const int r = mt * kCM + half * 128 + (i & 7) + 16 * (i >> 4);
  const int col = kt * kCK + 32 * j + 16 * ((i >> 3) & 1);
  const int mwords = d / 32;
  uint32_t lo = kPad, hi = kPad;
  if (col < d) {
    if (r < rows) lo = (meta[(long long)r * mwords + col / 32] >> (col & 31)) & 0xffffu;
    if (r + 8 < rows) hi = (meta[(long long)(r + 8) * mwords + col / 32] >> (col & 31)) & 0xffffu;
  }
  tiles[w] = lo | (hi << 16);
}

__global__ void __launch_bounds__(kCThreads, 1) sparse24_gemm_kernel(
    const __grid_constant__ CUtensorMap vmap, const __grid_constant__ CUtensorMap xmap,
    const uint32_t* __restrict__ tiles, int rows, int d, int n, float* __restrict__ Y, int* info,
    const long long wait_cycles) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kCStages * kCStage);
  __shared__ uint32_t tmem_slot;
  __shared__ int failed;
  if (cta_info_set(info)) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mt_count = (rows + kCM - 1) / kCM, nt_count = (n + kCN - 1) / kCN;
  const int kt_count = (d + kCK - 1) / kCK;
  const int items = mt_count * nt_count;
  const uint32_t s0 = smem_u32(smem);
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + kCStages);
  const uint32_t tfull = smem_u32(bars + 2 * kCStages), tempty = tfull + 8, mdone = tfull + 16;
  if (threadIdx.x == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&vmap)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&xmap)) : "memory");
    failed = 0;
    for (int st = 0; st < kCStages; ++st) {
      mbar_init(full0 + 8 * st, 1);
      mbar_init(empty0 + 8 * st, 1);
    }
    mbar_init(tfull, 1);
    mbar_init(tempty, kCEpiWarps);
    mbar_init(mdone, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_slot)),
                 "r"(kCTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = tmem_slot;

  auto decode = [&](int w, int& mt, int& nt) {
    const int per_group = kCGroupRows * nt_count;
    const int g = w / per_group;
    const int first = g * kCGroupRows;
    const int grows = min(kCGroupRows, mt_count - first);
    const int r = w - g * per_group;
    mt = first + r % grows;
    nt = r / grows;
  };

  if (warp == 0) {
    if (lane == 0) {
      int g = 0;
      for (int w = blockIdx.x; w < items && !failed; w += gridDim.x) {
        int mt, nt;
        decode(w, mt, nt);
        const uint32_t* tile_meta = tiles + (long long)mt * kt_count * (kCMeta / 4);
        for (int i = 0; i < kt_count; ++i, ++g) {
          const int st = g % kCStages;
          if (g >= kCStages && !mbar_wait(empty0 + 8 * st, ((g / kCStages) & 1) ^ 1, wait_cycles)) {
            failed = 1;
            break;
          }
          const uint32_t bar = full0 + 8 * st;
          asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(kCStage) : "memory");
          const uint32_t sa = s0 + st * kCStage;
          tma_2d(sa, &vmap, bar, i * (kCK / 2), mt * kCM);
          tma_2d(sa + kCHalfA, &vmap, bar, i * (kCK / 2), mt * kCM + 128);
          tma_2d(sa + kCOffB, &xmap, bar, i * kCK, nt * kCN);
          tma_2d(sa + kCOffB + kCBox, &xmap, bar, i * kCK + 64, nt * kCN);
          bulk_copy(sa + kCOffMeta, tile_meta + (long long)i * (kCMeta / 4), kCMeta, bar);
        }
      }
      for (int x = (g > kCStages ? g - kCStages : 0); x < g; ++x)
        if (!mbar_wait(full0 + 8 * (x % kCStages), (x / kCStages) & 1, kDrainCycles)) failed = 1;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int g = 0, u = 0;
      for (int w = blockIdx.x; w < items && !failed; w += gridDim.x, ++u) {
        // the epilogue has read the previous tile's accumulators
        if (u >= 1 && !mbar_wait(tempty, (u - 1) & 1, wait_cycles)) {
          failed = 1;
          break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        for (int i = 0; i < kt_count; ++i, ++g) {
          const int st = g % kCStages;
          if (!mbar_wait(full0 + 8 * st, (g / kCStages) & 1, wait_cycles)) {
            failed = 1;
            break;
          }
          asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
          const uint32_t sa = s0 + st * kCStage;
          const uint32_t mcol = (uint32_t)(kCMetaCol + 8 * st);
#pragma unroll
          for (int h = 0; h < 2; ++h)
            asm volatile("tcgen05.cp.cta_group::1.128x128b [%0], %1;" ::"r"(tmem + mcol + 4 * h),
                         "l"(meta_src_desc(sa + kCOffMeta + h * 2048))
                         : "memory");
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            // B: 32 columns (64 bytes) of box j / 2; A: 16 stored values (32 bytes) per row
            const uint64_t bd = kmajor_desc(sa + kCOffB + (j >> 1) * kCBox + 64 * (j & 1));
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              // slab j's metadata: an even column address and, in the
              // instruction descriptor's sparse selector, the column's low bit
              mma_sp(tmem + (uint32_t)(h * kCN), kmajor_desc(sa + h * kCHalfA + 32 * j), bd,
                     kSpIdesc | (uint32_t)(j & 1), tmem + mcol + 4 * h + (uint32_t)(j & ~1),
                     (i > 0 || j > 0) ? 1u : 0u);
            }
          }
          mma_commit(empty0 + 8 * st);
        }
        if (failed) break;
        mma_commit(tfull);
      }
      // never free TMEM under a running MMA or copy
      mma_commit(mdone);
      if (!mbar_wait(mdone, 0, kDrainCycles)) failed = 1;
    }
  } else {
    const int q = warp & 3, h = (warp - 2) >> 2;
    const int m_in_tile = h * 128 + q * 32 + lane;       // tile row = TMEM lane of accumulator h
    int u = 0;
    for (int w = blockIdx.x; w < items; w += gridDim.x, ++u) {
      int mt, nt;
      decode(w, mt, nt);
      float acc[kCN];
      // one decision per warp: the TMEM loads below are warp-collective
      int bad = failed;
      if (!bad) bad = !mbar_wait(tfull, u & 1, wait_cycles);
      bad = __any_sync(0xffffffffu, bad);
      if (bad) failed = 1;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      if (!bad) {
#pragma unroll
        for (int cc = 0; cc < kCN / 32; ++cc) {
          uint32_t v[32];
          tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(h * kCN + cc * 32), v);
#pragma unroll
          for (int e = 0; e < 32; ++e) acc[cc * 32 + e] = __uint_as_float(v[e]);
        }
      }
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty);
      if (bad) break;
      const int row = mt * kCM + m_in_tile;
      if (row < rows) {
        const int n0 = nt * kCN;
        float* yp = Y + (long long)n0 * rows + row;
#pragma unroll
        for (int e = 0; e < kCN; ++e) {
          if (n0 + e >= n) continue;
          yp[(long long)e * rows] = acc[e];
        }
      }
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (failed && threadIdx.x == 0) set_info(info, SGPT_INFO_TIMEOUT);
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kCTmemCols));
}

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

// bf16 [rows x cols], boxes of 64 x 128 with the 128-byte swizzle (out of
// range elements read as zero).
bool map_bf16(CUtensorMap* m, const uint16_t* p, long long rows, long long cols) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {64, 128};
  const cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(p), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t sparse24_meta_tiles_bytes(int rows, int d) {
  return (size_t)cdiv(rows, kCM) * (size_t)cdiv(d, kCK) * kCMeta;
}

cudaError_t launch_tile_meta(const uint32_t* meta, int rows, int d, uint32_t* tiles, cudaStream_t st) {
  const long long words = (long long)(sparse24_meta_tiles_bytes(rows, d) / 4);
  tile_meta_kernel<<<(unsigned)cdivll(words, 256), 256, 0, st>>>(meta, rows, d, cdiv(d, kCK), words, tiles);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_sparse24_gemm(const uint16_t* values_bf16, const uint32_t* tiles, int rows, int d,
                                 const uint16_t* X, long long n, float* Y, int* info, cudaStream_t st) {
  CUtensorMap vm, xm;
  if (!map_bf16(&vm, values_bf16, rows, d / 2) || !map_bf16(&xm, X, n, d)) return cudaErrorInvalidValue;
  static PerDevice attrs;
  const cudaError_t ea = once_per_device(attrs, [] {
    return cudaFuncSetAttribute(sparse24_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kCSmem);
  });
  if (ea != cudaSuccess) return ea;
  const long long items = (long long)cdiv(rows, kCM) * cdivll(n, kCN);
  const int ctas = (int)(items < kNumSMs ? items : kNumSMs);
  sparse24_gemm_kernel<<<ctas, kCThreads, kCSmem, st>>>(vm, xm, tiles, rows, d, (int)n, Y, info,
                                                        wait_limit_cycles());
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace sgpt
