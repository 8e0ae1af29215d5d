// Shared device helpers of the SparseGPT solver kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/sgpt.h"

namespace sgpt {

constexpr int kNumSMs = 148;          // B200
constexpr int kTile = 128;            // square tile of H, R, U and the GEMMs
constexpr int kMaxBlock = 128;        // widest OBS block held by the sweep

// Bounded waits. A device-side wait on another role of the same kernel or on
// other CTAs (an mbarrier phase, a grid barrier) gives up after the launch's
// wait limit in SM clock cycles (a kernel argument, from wait_limit_cycles())
// and records SGPT_INFO_TIMEOUT instead of hanging the GPU. A CTA that gave
// up still waits for its own asynchronous work in flight (TMA copies,
// tensor-core MMAs) before it frees TMEM and exits; those drains complete by
// themselves and use the fixed kDrainCycles, never the settable limit.
constexpr long long kDefaultWaitCycles = 4000000000ll;   // ~2 s at the boost clock
constexpr long long kDrainCycles = 4000000000ll;
// Below this limit an mbarrier wait polls without suspending the thread.
constexpr long long kShortWaitCycles = 1000000ll;

// The wait limit kernels are launched with now (sgpt_set_wait_limit).
long long wait_limit_cycles();

// First error wins; later kernels of the chain see it and return early.
__device__ __forceinline__ void set_info(int* info, int code) {
  if (info) atomicCAS(info, 0, code);
}

__device__ __forceinline__ bool info_set(const int* info) {
  return info && *(volatile const int*)info != 0;
}

// The same test taken once per CTA (every thread of the block must call it):
// thread 0 reads the word and the answer is shared, so a CTA never splits
// into threads that return and threads that wait at a barrier.
__device__ __forceinline__ bool cta_info_set(const int* info) {
  return __syncthreads_or(threadIdx.x == 0 && info_set(info)) != 0;
}

__device__ __forceinline__ float4 ld4(const float* p) {
  return *reinterpret_cast<const float4*>(p);
}
__device__ __forceinline__ void st4(float* p, float4 v) {
  *reinterpret_cast<float4*>(p) = v;
}

// 16-byte asynchronous global -> shared copy (both addresses 16-byte aligned),
// its commit and the wait for every copy this thread has committed.
__device__ __forceinline__ void cp_async16(float* dst_smem, const float* src) {
  const unsigned d = static_cast<unsigned>(__cvta_generic_to_shared(dst_smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__host__ __device__ __forceinline__ int cdiv(int a, int b) { return (a + b - 1) / b; }
__host__ __device__ __forceinline__ long long cdivll(long long a, long long b) {
  return (a + b - 1) / b;
}

// Saliency w^2 / U_cc^2 of weight w in a column whose U diagonal has the
// reciprocal inv_u = 1 / U_cc (IEEE-rounded once per column): (w * inv_u)^2
// in fp32. Every kernel that ranks weights calls this one function with the
// same reciprocal, so the selection kernels and the sweep agree bit for bit.
__device__ __forceinline__ float saliency(float w, float inv_u) {
  const float t = __fmul_rn(w, inv_u);
  return __fmul_rn(t, t);
}

// x rounded to TF32 (10 explicit mantissa bits, ties away from zero); the
// remainder x - tf32_hi(x) is exact in fp32. Used to split fp32 operands into
// the hi/lo planes of the three-product tensor-core GEMM.
__device__ __forceinline__ float tf32_hi(float x) {
  return __uint_as_float((__float_as_uint(x) + 0x1000u) & 0xffffe000u);
}

// Host-side count of kernel launches (diagnostics, sgpt_kernel_launches).
void count_launches(unsigned long long n);

// One-time setup per device (kernel attributes such as the dynamic
// shared-memory limit belong to the current device's context): runs `f` the
// first time it is called for the current device, under a lock, and again
// later if it failed.
struct PerDevice {
  std::mutex mu;
  bool done[64] = {};
};
template <class F>
cudaError_t once_per_device(PerDevice& pd, F&& f) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return f();
  std::lock_guard<std::mutex> lock(pd.mu);
  if (pd.done[dev]) return cudaSuccess;
  e = f();
  if (e == cudaSuccess) pd.done[dev] = true;
  return e;
}

// Host-side workspace carving: consecutive 256-byte aligned sub-buffers.
struct Carve {
  char* base;
  size_t off = 0;
  explicit Carve(void* b) : base(static_cast<char*>(b)) {}
  template <class T>
  T* take(size_t count) {
    off = (off + 255) & ~size_t(255);
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += count * sizeof(T);
    return p;
  }
};

}  // namespace sgpt
