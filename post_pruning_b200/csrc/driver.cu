// Multi-layer driver: one synthetic MLP block of a decoder, pruned layer by
// layer (SparseGPT review, section 九: collect the current layer's inputs,
// form its Hessian, prune with compensation, pass the pruned layer's output
// on to the next layer; section 十一, steps three to six), or layer-parallel
// from the dense model's recorded inputs (V-SparseGPT press release: the
// inputs of every layer of the original model are recorded first, so the
// layers can be sparsified side by side).
//
// The block: x -> x + W_down (silu(W_gate x) * (W_up x)), activations bf16,
// the forward products on the tensor cores in bf16 with fp32 accumulation
// (gemm_tc.cu), the weights of each product the bf16 rounding of the fp32
// weights; every rounding to bf16 is to nearest even.
//
// Sequential: H(x), U(x) -> prune gate and up -> z = silu(x Wg^T) * (x Wu^T)
// with the pruned gate and up -> H(z), U(z) -> prune down -> x' = x + z Wd^T.
// Parallel: z and x' from the dense weights first; then gate/up from x and
// down from the recorded z, the down input's Hessian on a second stream while
// gate and up are factored and swept.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "../../include/sgpt.h"
#include "common.cuh"
#include "gemm_tc.h"
#include "kernels.h"

namespace sgpt {

namespace {

__device__ __forceinline__ uint16_t to_bf16_bits(float x) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

// Wb = bf16(W), rows x cols (W leading dimension ld).
__global__ void to_bf16_kernel(const float* __restrict__ W, long long ld, long long rows, int cols,
                               uint16_t* __restrict__ Wb, const int* info) {
  if (info_set(info)) return;
  const long long quads = rows * (cols / 4);
  for (long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x; q < quads;
       q += (long long)gridDim.x * blockDim.x) {
    const long long r = q / (cols / 4);
    const int c = (int)(q - r * (cols / 4)) * 4;
    const float4 x = ld4(W + r * ld + c);
    const ushort4 o = make_ushort4(to_bf16_bits(x.x), to_bf16_bits(x.y), to_bf16_bits(x.z), to_bf16_bits(x.w));
    *reinterpret_cast<ushort4*>(Wb + r * cols + c) = o;
  }
}

// z = bf16(silu(g) * u), silu(g) = g / (1 + e^-g), in fp32.
__global__ void swiglu_kernel(const float* __restrict__ G, const float* __restrict__ Uu, long long count,
                              uint16_t* __restrict__ Z, const int* info) {
  if (info_set(info)) return;
  for (long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x; q < count / 4;
       q += (long long)gridDim.x * blockDim.x) {
    const float4 g = ld4(G + 4 * q), u = ld4(Uu + 4 * q);
    const float v[4] = {g.x / (1.f + expf(-g.x)) * u.x, g.y / (1.f + expf(-g.y)) * u.y,
                        g.z / (1.f + expf(-g.z)) * u.z, g.w / (1.f + expf(-g.w)) * u.w};
    *reinterpret_cast<ushort4*>(Z + 4 * q) =
        make_ushort4(to_bf16_bits(v[0]), to_bf16_bits(v[1]), to_bf16_bits(v[2]), to_bf16_bits(v[3]));
  }
}

// x' = bf16(x + d).
__global__ void residual_kernel(const uint16_t* __restrict__ X, const float* __restrict__ D, long long count,
                                uint16_t* __restrict__ Xn, const int* info) {
  if (info_set(info)) return;
  for (long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x; q < count / 4;
       q += (long long)gridDim.x * blockDim.x) {
    const ushort4 x = *reinterpret_cast<const ushort4*>(X + 4 * q);
    const float4 d = ld4(D + 4 * q);
    *reinterpret_cast<ushort4*>(Xn + 4 * q) =
        make_ushort4(to_bf16_bits(bf16_bits_to_float(x.x) + d.x), to_bf16_bits(bf16_bits_to_float(x.y) + d.y),
                     to_bf16_bits(bf16_bits_to_float(x.z) + d.z), to_bf16_bits(bf16_bits_to_float(x.w) + d.w));
  }
}

int grid_for(long long work) {
  return (int)std::max<long long>(1, std::min<long long>(cdivll(work, 256), 16LL * kNumSMs));
}

}  // namespace

cudaError_t launch_to_bf16(const float* W, long long ld, long long rows, int cols, uint16_t* Wb, const int* info,
                           cudaStream_t st) {
  to_bf16_kernel<<<grid_for(rows * cols / 4), 256, 0, st>>>(W, ld, rows, cols, Wb, info);
  count_launches(1);
  return cudaGetLastError();
}

// Y [n x d_out] fp32 = X [n x d_in] bf16 * Wb [d_out x d_in]^T bf16.
cudaError_t launch_linear_bf16(const uint16_t* X, const uint16_t* Wb, long long n, int d_in, int d_out, float* Y,
                               int* info, cudaStream_t st) {
  const tc::OperandBf16 A{X, n, d_in, d_in};
  const tc::OperandBf16 B{Wb, d_out, d_in, d_in};
  tc::Job job{};
  job.mode = 0;
  job.mt = (int)cdivll(n, kTile);
  job.nt = cdiv(d_out, kTile);
  job.kdim = d_in;
  job.C = Y;
  job.ldc = d_out;
  job.Mlim = (int)std::min<long long>(n, INT32_MAX);
  job.Nlim = d_out;
  job.alpha = 1.f;
  job.beta = 0.f;
  return tc::launch_gemm_bf16(A, B, job, job.mt * job.nt, info, st);
}

namespace {

struct BlockWs {
  float* H1;        // h x h: the block input's X^T X, then (H1, U1) its factor
  float* U1;
  float* H2;        // f x f: the down input's Z^T Z and its factor
  float* U2;
  uint16_t* Wg_b;   // bf16 weights of the forward products
  uint16_t* Wu_b;
  uint16_t* Wd_b;
  float* G;         // n x f fp32: x Wg^T, then x Wu^T in Uu
  float* Uu;
  uint16_t* Z;      // n x f bf16: the down input
  float* D;         // n x h fp32: z Wd^T
  void* inner;      // scratch of the per-layer calls
  size_t inner_bytes;
  void* inner2;     // a second one for the side stream (parallel mode)
  size_t inner2_bytes;
};

size_t inner_bytes_for(int h, int f, long long n) {
  size_t b = std::max({factor_ws_bytes(h), factor_ws_bytes(f), prune_ws_bytes(f, h), prune_ws_bytes(h, f),
                       hessian_ws_bytes(h, n), hessian_ws_bytes(f, n)});
  return b;
}

BlockWs carve_block(void* ws, int h, int f, long long n, uint16_t* Z, size_t* bytes) {
  Carve c(ws);
  BlockWs w;
  w.H1 = c.take<float>((size_t)h * h);
  w.U1 = c.take<float>((size_t)h * h);
  w.H2 = c.take<float>((size_t)f * f);
  w.U2 = c.take<float>((size_t)f * f);
  w.Wg_b = c.take<uint16_t>((size_t)f * h);
  w.Wu_b = c.take<uint16_t>((size_t)f * h);
  w.Wd_b = c.take<uint16_t>((size_t)h * f);
  w.G = c.take<float>((size_t)n * f);
  w.Uu = c.take<float>((size_t)n * f);
  w.Z = Z ? Z : c.take<uint16_t>((size_t)n * f);
  w.D = c.take<float>((size_t)n * h);
  w.inner_bytes = inner_bytes_for(h, f, n);
  w.inner = c.take<unsigned char>(w.inner_bytes);
  w.inner2_bytes = std::max(hessian_ws_bytes(f, n), (size_t)256);
  w.inner2 = c.take<unsigned char>(w.inner2_bytes);
  if (bytes) *bytes = c.off + 256;
  return w;
}

// The block's forward pass with the weights as they are now: z (bf16) and
// x' = x + z Wd^T (bf16).
cudaError_t forward(const sgpt_mlp_block& blk, int h, int f, const uint16_t* X, long long n, uint16_t* X_next,
                    const BlockWs& w, int* info, cudaStream_t st) {
  cudaError_t e;
  if ((e = launch_to_bf16(blk.W_gate, h, f, h, w.Wg_b, info, st)) != cudaSuccess) return e;
  if ((e = launch_to_bf16(blk.W_up, h, f, h, w.Wu_b, info, st)) != cudaSuccess) return e;
  if ((e = launch_linear_bf16(X, w.Wg_b, n, h, f, w.G, info, st)) != cudaSuccess) return e;
  if ((e = launch_linear_bf16(X, w.Wu_b, n, h, f, w.Uu, info, st)) != cudaSuccess) return e;
  swiglu_kernel<<<grid_for(n * f / 4), 256, 0, st>>>(w.G, w.Uu, n * f, w.Z, info);
  count_launches(1);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return cudaSuccess;
}

cudaError_t forward_down(const sgpt_mlp_block& blk, int h, int f, const uint16_t* X, long long n,
                         uint16_t* X_next, const BlockWs& w, int* info, cudaStream_t st) {
  cudaError_t e;
  if ((e = launch_to_bf16(blk.W_down, f, h, f, w.Wd_b, info, st)) != cudaSuccess) return e;
  if ((e = launch_linear_bf16(w.Z, w.Wd_b, n, f, h, w.D, info, st)) != cudaSuccess) return e;
  residual_kernel<<<grid_for(n * h / 4), 256, 0, st>>>(X, w.D, n * h, X_next, info);
  count_launches(1);
  return cudaGetLastError();
}

// Streams and events of the parallel mode (per device).
struct DriverStreams {
  cudaStream_t side = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
std::mutex g_drv_mu;

cudaError_t driver_streams(DriverStreams** out) {
  static DriverStreams per_dev[64];
  static bool made[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  DriverStreams& s = per_dev[dev];
  if (!made[dev]) {
    if ((e = cudaStreamCreateWithFlags(&s.side, cudaStreamNonBlocking)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&s.fork, cudaEventDisableTiming)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&s.join, cudaEventDisableTiming)) != cudaSuccess) return e;
    made[dev] = true;
  }
  *out = &s;
  return cudaSuccess;
}

}  // namespace

size_t mlp_block_ws_bytes(int h, int f, long long n) {
  size_t b = 0;
  carve_block(nullptr, h, f, n, nullptr, &b);
  return b;
}

cudaError_t launch_prune_mlp_block(const sgpt_mlp_block& blk, int h, int f, const uint16_t* X, long long n,
                                   int mode, const sgpt_params& p, uint16_t* X_next, uint16_t* Z, void* ws,
                                   int* info, cudaStream_t st) {
  const BlockWs w = carve_block(ws, h, f, n, Z, nullptr);
  cudaError_t e;
  auto prune_one = [&](float* W, int rows, int d, const float* U, uint32_t* mask, void* inner) {
    return launch_prune(W, rows, d, d, U, p, mask, nullptr, inner, info, st);
  };
  if (mode == SGPT_DRIVER_SEQUENTIAL) {
    // gate and up from the block input
    if ((e = launch_hessian_tc(w.H1, X, n, h, w.inner, info, st, true)) != cudaSuccess) return e;
    if ((e = launch_factor(w.H1, n, h, p.damp, w.U1, w.inner, info, st)) != cudaSuccess) return e;
    if ((e = prune_one(blk.W_gate, f, h, w.U1, blk.mask_gate, w.inner)) != cudaSuccess) return e;
    if ((e = prune_one(blk.W_up, f, h, w.U1, blk.mask_up, w.inner)) != cudaSuccess) return e;
    // the down input from the pruned gate and up
    if ((e = forward(blk, h, f, X, n, X_next, w, info, st)) != cudaSuccess) return e;
    if ((e = launch_hessian_tc(w.H2, w.Z, n, f, w.inner, info, st, true)) != cudaSuccess) return e;
    if ((e = launch_factor(w.H2, n, f, p.damp, w.U2, w.inner, info, st)) != cudaSuccess) return e;
    if ((e = prune_one(blk.W_down, h, f, w.U2, blk.mask_down, w.inner)) != cudaSuccess) return e;
    // the next block's input from the pruned block
    return forward_down(blk, h, f, X, n, X_next, w, info, st);
  }
  // parallel: record the dense block's down input and output first
  if ((e = forward(blk, h, f, X, n, X_next, w, info, st)) != cudaSuccess) return e;
  if ((e = forward_down(blk, h, f, X, n, X_next, w, info, st)) != cudaSuccess) return e;
  DriverStreams* ds = nullptr;
  std::lock_guard<std::mutex> lock(g_drv_mu);
  if ((e = driver_streams(&ds)) != cudaSuccess) return e;
  // the down input's Hessian on the side stream, beside gate and up
  if ((e = cudaEventRecord(ds->fork, st)) != cudaSuccess) return e;
  if ((e = cudaStreamWaitEvent(ds->side, ds->fork, 0)) != cudaSuccess) return e;
  cudaError_t es = launch_hessian_tc(w.H2, w.Z, n, f, w.inner2, info, ds->side, true);
  if (es == cudaSuccess) es = cudaEventRecord(ds->join, ds->side);
  if ((e = launch_hessian_tc(w.H1, X, n, h, w.inner, info, st, true)) == cudaSuccess &&
      (e = launch_factor(w.H1, n, h, p.damp, w.U1, w.inner, info, st)) == cudaSuccess &&
      (e = prune_one(blk.W_gate, f, h, w.U1, blk.mask_gate, w.inner)) == cudaSuccess)
    e = prune_one(blk.W_up, f, h, w.U1, blk.mask_up, w.inner);
  // always join the side stream, also after an error (a capture stays well formed)
  const cudaError_t ej = es == cudaSuccess ? cudaStreamWaitEvent(st, ds->join, 0) : es;
  if (e != cudaSuccess) return e;
  if (ej != cudaSuccess) return ej;
  if ((e = launch_factor(w.H2, n, f, p.damp, w.U2, w.inner, info, st)) != cudaSuccess) return e;
  return prune_one(blk.W_down, h, f, w.U2, blk.mask_down, w.inner);
}

}  // namespace sgpt
