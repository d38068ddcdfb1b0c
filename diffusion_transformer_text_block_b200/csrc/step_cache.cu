// Kernels of the first-block step cache (MossInfer integration guide, What works: Lossy
// accelerators; Per-image settings: Step cache).  A step compares block 0's output o with the
// block-0 output o_ref of the last full call by sum|o - o_ref| / sum|o_ref|; a step that reuses
// the cache adds the stored residual of blocks 1..L-1 to o, a full call stores it.
// All three kernels stream FP32 rows once: HBM-bound.
#include "common.cuh"
#include "internal.h"

namespace moss {

namespace {

constexpr int kThreads = 256;

// partials[2 b] = sum over block b's elements of |a - ref|, partials[2 b + 1] = of |ref|, in FP64.
// The grid size is fixed by the caller and the host adds the partials in block order, so the
// result does not depend on scheduling.
__global__ void __launch_bounds__(kThreads) change_partials_kernel(const float* __restrict__ a,
                                                                   const float* __restrict__ ref, int64_t n,
                                                                   double* __restrict__ partials) {
  double num = 0.0, den = 0.0;
  const int64_t n4 = n >> 2;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const float4* a4 = reinterpret_cast<const float4*>(a);
  const float4* r4 = reinterpret_cast<const float4*>(ref);
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += stride) {
    const float4 u = __ldcs(a4 + i), r = __ldcs(r4 + i);
    num += static_cast<double>(fabsf(u.x - r.x)) + static_cast<double>(fabsf(u.y - r.y)) +
           static_cast<double>(fabsf(u.z - r.z)) + static_cast<double>(fabsf(u.w - r.w));
    den += static_cast<double>(fabsf(r.x)) + static_cast<double>(fabsf(r.y)) + static_cast<double>(fabsf(r.z)) +
           static_cast<double>(fabsf(r.w));
  }
  if (blockIdx.x == 0 && threadIdx.x < (n & 3)) {
    const int64_t i = (n4 << 2) + threadIdx.x;
    num += fabsf(a[i] - ref[i]);
    den += fabsf(ref[i]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    num += __shfl_xor_sync(0xffffffffu, num, o);
    den += __shfl_xor_sync(0xffffffffu, den, o);
  }
  __shared__ double s_num[kThreads / 32], s_den[kThreads / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    s_num[warp] = num;
    s_den[warp] = den;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double tn = 0.0, td = 0.0;
    for (int w = 0; w < kThreads / 32; ++w) {
      tn += s_num[w];
      td += s_den[w];
    }
    partials[2 * blockIdx.x] = tn;
    partials[2 * blockIdx.x + 1] = td;
  }
}

// x += r
__global__ void __launch_bounds__(kThreads) add_kernel(float* __restrict__ x, const float* __restrict__ r,
                                                       int64_t n) {
  const int64_t n4 = n >> 2;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  float4* x4 = reinterpret_cast<float4*>(x);
  const float4* r4 = reinterpret_cast<const float4*>(r);
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 u = x4[i];
    const float4 v = __ldcs(r4 + i);
    u.x += v.x;
    u.y += v.y;
    u.z += v.z;
    u.w += v.w;
    x4[i] = u;
  }
  if (blockIdx.x == 0 && threadIdx.x < (n & 3)) {
    const int64_t i = (n4 << 2) + threadIdx.x;
    x[i] += r[i];
  }
}

// d = a - b
__global__ void __launch_bounds__(kThreads) sub_kernel(float* __restrict__ d, const float* __restrict__ a,
                                                       const float* __restrict__ b, int64_t n) {
  const int64_t n4 = n >> 2;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  float4* d4 = reinterpret_cast<float4*>(d);
  const float4* a4 = reinterpret_cast<const float4*>(a);
  const float4* b4 = reinterpret_cast<const float4*>(b);
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += stride) {
    const float4 u = __ldcs(a4 + i), v = __ldcs(b4 + i);
    d4[i] = make_float4(u.x - v.x, u.y - v.y, u.z - v.z, u.w - v.w);
  }
  if (blockIdx.x == 0 && threadIdx.x < (n & 3)) {
    const int64_t i = (n4 << 2) + threadIdx.x;
    d[i] = a[i] - b[i];
  }
}

unsigned stream_blocks(int64_t n) {
  int64_t blocks = ((n >> 2) + kThreads - 1) / kThreads;
  if (blocks < 1) blocks = 1;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
  return static_cast<unsigned>(blocks > cap ? cap : blocks);
}

}  // namespace

int change_partial_blocks() { return 2 * num_sms(); }

cudaError_t launch_change_partials(const float* a, const float* ref, int64_t n, double* partials, cudaStream_t s) {
  change_partials_kernel<<<change_partial_blocks(), kThreads, 0, s>>>(a, ref, n, partials);
  return cudaGetLastError();
}

cudaError_t launch_add_inplace(float* x, const float* r, int64_t n, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  add_kernel<<<stream_blocks(n), kThreads, 0, s>>>(x, r, n);
  return cudaGetLastError();
}

cudaError_t launch_sub(float* d, const float* a, const float* b, int64_t n, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  sub_kernel<<<stream_blocks(n), kThreads, 0, s>>>(d, a, b, n);
  return cudaGetLastError();
}

}  // namespace moss
