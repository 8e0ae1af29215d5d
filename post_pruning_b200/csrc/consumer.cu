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
// kept positions), so the conversion from the packed metadata words is a
// re-arrangement, done by every thread for its own lane before each K
// stage and written with tcgen05.st.
//
// One CTA of four warps per 128 x 128 output tile; per K stage of 128: TMA
// brings the tile's 64 stored values per row (A, 16 KB) and 128 columns of X
// (B, two 64-column boxes), the threads store the stage's four metadata
// columns, one thread issues the four sparse MMAs (K = 32 each) and commits
// to an mbarrier the CTA waits on before the next stage reuses the buffers.
// Every wait is on this CTA's own copies and MMAs, bounded by kDrainCycles;
// a wait that runs out records SGPT_INFO_TIMEOUT and the CTA stops issuing.
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/sgpt.h"
#include "common.cuh"
#include "kernels.h"

namespace sgpt {

namespace {

constexpr int kCM = 128, kCN = 128, kCK = 128;      // output tile, logical K per stage
constexpr int kCThreads = 128;
constexpr int kABytes = kCM * (kCK / 2) * 2;        // 16 KB: 64 stored bf16 per row
constexpr int kBBytes = kCN * kCK * 2;              // 32 KB: two 64-column boxes
constexpr int kCBox = 64 * 128 * 2;                 // one TMA box, 16 KB
constexpr int kCTmemCols = 256;                     // 128 accumulator + 4 metadata columns (power of two)
constexpr int kMetaCol = 128;
// 112 KB of dynamic shared memory keeps at most two CTAs (512 TMEM columns) per SM
constexpr size_t kCSmem = 112 * 1024;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
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
__device__ __forceinline__ bool mbar_wait_drain(uint32_t bar, uint32_t parity) {
  if (mbar_try(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try(bar, parity))
    if (clock64() - t0 > kDrainCycles) return false;
  return true;
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

// D fp32, A and B bf16, both K-major, sparse A (bit 2), N/8, M/16.
constexpr uint32_t kSpIdesc = (1u << 2) | (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kCN >> 3) << 17) |
                              ((uint32_t)(kCM >> 4) << 24);

// The metadata column value of this thread's lane for the K = 32 slab that
// starts at column c (a multiple of 32): the 16-bit halves of rows r and
// r + 8 for K half h.
__device__ __forceinline__ uint32_t meta_lane_value(const uint32_t* __restrict__ meta, int rows, int d, int m0,
                                                    int lane_id, int c) {
  const int r = m0 + (lane_id & 7) + 16 * (lane_id >> 4);
  const int h = (lane_id >> 3) & 1;
  const int col = c + 16 * h;                     // first of the 16 columns
  // padding (rows past the layer, columns past d_in, whose A values are the
  // zeros TMA fills in) takes the valid code 0 | 1 << 2 in every group
  constexpr uint32_t kPad = 0x4444u;
  if (col >= d) return kPad | (kPad << 16);
  const int words = d / 32;
  const uint32_t lo = r < rows ? (meta[(long long)r * words + col / 32] >> (col & 31)) & 0xffffu : kPad;
  const uint32_t hi = r + 8 < rows ? (meta[(long long)(r + 8) * words + col / 32] >> (col & 31)) & 0xffffu : kPad;
  return lo | (hi << 16);
}

__global__ void __launch_bounds__(kCThreads) sparse24_gemm_kernel(
    const __grid_constant__ CUtensorMap vmap, const __grid_constant__ CUtensorMap xmap,
    const uint32_t* __restrict__ meta, int rows, int d, long long n, float* __restrict__ Y, int* info) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t bars[2];
  __shared__ uint32_t tmem_slot;
  __shared__ int failed;
  if (cta_info_set(info)) return;
  const int tid = threadIdx.x, warp = tid >> 5;
  const int m0 = blockIdx.x * kCM;
  const long long n0 = (long long)blockIdx.y * kCN;
  const uint32_t sa = smem_u32(smem), sb = sa + kABytes;
  const uint32_t tma_bar = smem_u32(&bars[0]), mma_bar = smem_u32(&bars[1]);
  if (tid == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&vmap)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&xmap)) : "memory");
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(tma_bar));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(mma_bar));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    failed = 0;
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
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;     // this warp's TMEM lane quadrant

  const int stages = (d + kCK - 1) / kCK;
  for (int s = 0; s < stages; ++s) {
    const uint32_t par = s & 1;
    if (tid == 0 && !failed) {
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(tma_bar), "r"(kABytes + kBBytes)
                   : "memory");
      asm volatile(
          "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::
              "r"(sa), "l"(reinterpret_cast<uint64_t>(&vmap)), "r"(tma_bar), "r"(s * (kCK / 2)), "r"(m0)
          : "memory");
#pragma unroll
      for (int b = 0; b < 2; ++b)
        asm volatile(
            "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
            "[%2];" ::"r"(sb + b * kCBox),
            "l"(reinterpret_cast<uint64_t>(&xmap)), "r"(tma_bar), "r"(s * kCK + 64 * b), "r"((int)n0)
            : "memory");
    }
    // this lane's metadata for the stage's four K = 32 slabs
    uint32_t mv[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) mv[j] = meta_lane_value(meta, rows, d, m0, tid, s * kCK + 32 * j);
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(tmem + lane_base + kMetaCol),
                 "r"(mv[0]), "r"(mv[1]), "r"(mv[2]), "r"(mv[3])
                 : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
    if (tid == 0 && !failed && !mbar_wait_drain(tma_bar, par)) failed = 1;
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (failed) break;
    if (tid == 0) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        // A: 16 stored values (32 bytes) per row per slab; B: 32 columns (64 bytes)
        const uint64_t ad = kmajor_desc(sa + 32 * j);
        const uint64_t bd = kmajor_desc(sb + (j >> 1) * kCBox + 64 * (j & 1));
        const uint32_t acc = (s > 0 || j > 0) ? 1u : 0u;
        // the metadata of slab j: an even column address and, in the
        // instruction descriptor's sparse selector, the column's low bit
        const uint32_t e_addr = tmem + kMetaCol + (uint32_t)(j & ~1);
        const uint32_t idesc = kSpIdesc | (uint32_t)(j & 1);
        asm volatile(
            "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
            " tcgen05.mma.sp.cta_group::1.kind::f16 [%0], %1, %2, [%5], %3, {%6, %7, %8, %9}, p;\n}\n" ::"r"(tmem),
            "l"(ad), "l"(bd), "r"(idesc), "r"(acc), "r"(e_addr), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
      }
      asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mma_bar)
                   : "memory");
      if (!mbar_wait_drain(mma_bar, par)) failed = 1;
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (failed) break;
  }
  if (!failed) {
    // lane = output row m0 + tid; columns = tokens n0 ..
    const int m = m0 + tid;
#pragma unroll 1
    for (int cc = 0; cc < kCN / 32; ++cc) {
      uint32_t v[32];
      asm volatile(
          "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
          "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
          : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
            "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
            "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]),
            "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]),
            "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
          : "r"(tmem + lane_base + (uint32_t)(cc * 32)));
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
      if (m < rows) {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const long long tok = n0 + cc * 32 + e;
          if (tok < n) Y[tok * rows + m] = __uint_as_float(v[e]);
        }
      }
    }
  }
  if (failed && tid == 0) set_info(info, SGPT_INFO_TIMEOUT);
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
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

cudaError_t launch_sparse24_gemm(const uint16_t* values_bf16, const uint32_t* meta, int rows, int d,
                                 const uint16_t* X, long long n, float* Y, int* info, cudaStream_t st) {
  CUtensorMap vm, xm;
  if (!map_bf16(&vm, values_bf16, rows, d / 2) || !map_bf16(&xm, X, n, d)) return cudaErrorInvalidValue;
  static PerDevice attrs;
  const cudaError_t ea = once_per_device(attrs, [] {
    return cudaFuncSetAttribute(sparse24_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kCSmem);
  });
  if (ea != cudaSuccess) return ea;
  const dim3 grid(cdiv(rows, kCM), (unsigned)cdivll(n, kCN));
  sparse24_gemm_kernel<<<grid, kCThreads, kCSmem, st>>>(vm, xm, meta, rows, d, n, Y, info);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace sgpt
