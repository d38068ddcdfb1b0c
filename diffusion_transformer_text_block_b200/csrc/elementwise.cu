// Bandwidth-bound kernels of the denoising step: LN-modulate, CFG + Euler, initial noise,
// timestep conditioning, modulation GEMV, RoPE angle table and patchify.
// All use coalesced, vectorised (16-byte) global accesses.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace moss {

namespace {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---------------------------------------------------------------------------- LN-modulate
// h = LN(x) * (1 + scale) + shift: affine-free LayerNorm with biased variance (SGLang
// cookbook, Qwen-Image 2.1: Lossless LayerNorm modulation).  WPR warps per row; the row stays
// in registers (VPL float4 per lane) so mean and variance are exact two-pass sums; the
// warps of a row combine their partial sums through shared memory.  256 threads per block.
template <int VPL, int WPR>
__global__ void __launch_bounds__(256) ln_mod_kernel(const float* __restrict__ x, const float* __restrict__ shift,
                                                     const float* __restrict__ scale, bf16* __restrict__ h, int rows,
                                                     int gather_n_img, int gather_n_tok, float eps) {
  constexpr int D = VPL * 128 * WPR;
  constexpr int kRowsPerBlock = 8 / WPR;
  __shared__ float part[2][8];
  const int wib = threadIdx.x >> 5;          // warp in block
  const int lane = threadIdx.x & 31;
  const int rib = wib / WPR;                 // row in block
  const int sub = wib % WPR;                 // this warp's slice of the row
  const int row = blockIdx.x * kRowsPerBlock + rib;
  const bool live = row < rows;              // block-uniform barriers below: no early return
  int64_t src = row;
  if (gather_n_img > 0) src = static_cast<int64_t>(row / gather_n_img) * gather_n_tok + row % gather_n_img;
  const float4* xr = reinterpret_cast<const float4*>(x + src * D) + sub * VPL * 32;
  float4 v[VPL];
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    v[i] = live ? __ldcs(xr + lane + 32 * i) : make_float4(0.f, 0.f, 0.f, 0.f);
    s += (v[i].x + v[i].y) + (v[i].z + v[i].w);
  }
  s = warp_sum(s);
  if (WPR > 1) {
    if (lane == 0) part[0][wib] = s;
    __syncthreads();
    s = 0.f;
#pragma unroll
    for (int k = 0; k < WPR; ++k) s += part[0][rib * WPR + k];
  }
  const float mean = s * (1.0f / D);
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const float a = v[i].x - mean, b = v[i].y - mean, c = v[i].z - mean, d = v[i].w - mean;
    q += (a * a + b * b) + (c * c + d * d);
  }
  q = warp_sum(q);
  if (WPR > 1) {
    if (lane == 0) part[1][wib] = q;
    __syncthreads();
    q = 0.f;
#pragma unroll
    for (int k = 0; k < WPR; ++k) q += part[1][rib * WPR + k];
  }
  if (!live) return;
  const float rstd = rsqrtf(q * (1.0f / D) + eps);
  uint2* hr = reinterpret_cast<uint2*>(h + static_cast<int64_t>(row) * D) + sub * VPL * 32;
  const float4* sh = reinterpret_cast<const float4*>(shift) + sub * VPL * 32;
  const float4* sc = reinterpret_cast<const float4*>(scale) + sub * VPL * 32;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int j = lane + 32 * i;
    const float4 a = __ldg(sh + j), m = __ldg(sc + j);
    const float o0 = fmaf((v[i].x - mean) * rstd, 1.0f + m.x, a.x);
    const float o1 = fmaf((v[i].y - mean) * rstd, 1.0f + m.y, a.y);
    const float o2 = fmaf((v[i].z - mean) * rstd, 1.0f + m.z, a.z);
    const float o3 = fmaf((v[i].w - mean) * rstd, 1.0f + m.w, a.w);
    hr[j] = make_uint2(pack_bf16x2(o0, o1), pack_bf16x2(o2, o3));
  }
}

// ---------------------------------------------------------------------------- CFG + Euler
// x <- x + (sigma_next - sigma) * (v_u + cfg * (v_c - v_u)), FP32 (SGLang cookbook,
// MOSS-Image: 3. Guidance and precision).
__global__ void __launch_bounds__(256) cfg_euler_kernel(float* __restrict__ x, const float* __restrict__ vc,
                                                        const float* __restrict__ vu, int64_t n, float cfg,
                                                        float dt) {
  const int64_t n4 = n >> 2;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  float4* x4 = reinterpret_cast<float4*>(x);
  const float4* c4 = reinterpret_cast<const float4*>(vc);
  const float4* u4 = reinterpret_cast<const float4*>(vu);
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 a = x4[i];
    const float4 c = __ldcs(c4 + i), u = __ldcs(u4 + i);
    a.x = fmaf(dt, fmaf(cfg, c.x - u.x, u.x), a.x);
    a.y = fmaf(dt, fmaf(cfg, c.y - u.y, u.y), a.y);
    a.z = fmaf(dt, fmaf(cfg, c.z - u.z, u.z), a.z);
    a.w = fmaf(dt, fmaf(cfg, c.w - u.w, u.w), a.w);
    x4[i] = a;
  }
  if (blockIdx.x == 0 && threadIdx.x < (n & 3)) {
    const int64_t i = (n4 << 2) + threadIdx.x;
    x[i] = fmaf(dt, fmaf(cfg, vc[i] - vu[i], vu[i]), x[i]);
  }
}

// Three-pass skip-layer guidance: the CFG combine plus slg (vc - vcs), then the Euler update.
__global__ void __launch_bounds__(256) cfg_slg_euler_kernel(float* __restrict__ x, const float* __restrict__ vc,
                                                            const float* __restrict__ vcs,
                                                            const float* __restrict__ vu, int64_t n, float cfg,
                                                            float slg, float dt) {
  const int64_t n4 = n >> 2;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  float4* x4 = reinterpret_cast<float4*>(x);
  const float4* c4 = reinterpret_cast<const float4*>(vc);
  const float4* s4 = reinterpret_cast<const float4*>(vcs);
  const float4* u4 = reinterpret_cast<const float4*>(vu);
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 a = x4[i];
    const float4 c = __ldcs(c4 + i), k = __ldcs(s4 + i), u = __ldcs(u4 + i);
    a.x = fmaf(dt, fmaf(slg, c.x - k.x, fmaf(cfg, c.x - u.x, u.x)), a.x);
    a.y = fmaf(dt, fmaf(slg, c.y - k.y, fmaf(cfg, c.y - u.y, u.y)), a.y);
    a.z = fmaf(dt, fmaf(slg, c.z - k.z, fmaf(cfg, c.z - u.z, u.z)), a.z);
    a.w = fmaf(dt, fmaf(slg, c.w - k.w, fmaf(cfg, c.w - u.w, u.w)), a.w);
    x4[i] = a;
  }
  if (blockIdx.x == 0 && threadIdx.x < (n & 3)) {
    const int64_t i = (n4 << 2) + threadIdx.x;
    x[i] = fmaf(dt, fmaf(slg, vc[i] - vcs[i], fmaf(cfg, vc[i] - vu[i], vu[i])), x[i]);
  }
}

// ---------------------------------------------------------------------------- noise
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11): counter (g_lo, g_hi, 0, 0) for the
// group g of four outputs, key (seed_lo, seed_hi); Box-Muller on ((b >> 9) + 1/2) / 2^23.
__device__ __forceinline__ uint4 philox(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint32_t lo0 = 0xD2511F53u * c.x, hi0 = __umulhi(0xD2511F53u, c.x);
    const uint32_t lo1 = 0xCD9E8D57u * c.z, hi1 = __umulhi(0xCD9E8D57u, c.z);
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
  }
  return c;
}

__device__ __forceinline__ float2 box_muller(uint32_t a, uint32_t b) {
  const float ua = (static_cast<float>(a >> 9) + 0.5f) * (1.0f / 8388608.0f);
  const float ub = (static_cast<float>(b >> 9) + 0.5f) * (1.0f / 8388608.0f);
  const float r = sqrtf(-2.0f * logf(ua));
  float s, c;
  sincospif(2.0f * ub, &s, &c);
  return make_float2(r * c, r * s);
}

__global__ void noise_kernel(float* __restrict__ x, int64_t n, uint32_t k0, uint32_t k1) {
  const int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (g * 4 >= n) return;
  const uint4 bits = philox(make_uint4(static_cast<uint32_t>(g), static_cast<uint32_t>(g >> 32), 0u, 0u), k0, k1);
  const float2 z0 = box_muller(bits.x, bits.y);
  const float2 z1 = box_muller(bits.z, bits.w);
  if (g * 4 + 3 < n) {
    reinterpret_cast<float4*>(x)[g] = make_float4(z0.x, z0.y, z1.x, z1.y);
  } else {
    const float z[4] = {z0.x, z0.y, z1.x, z1.y};
    for (int i = 0; g * 4 + i < n; ++i) x[g * 4 + i] = z[i];
  }
}

// ---------------------------------------------------------------------------- conditioning
// c = W2 SiLU(W1 e + b1) + b2 with e = [cos, sin](1000 t exp(-ln(1e4) k / 128)); out SiLU(c),
// the input of every modulation linear (InvokeAI MOSS-Image guide, Transformer formats: the
// time-embedding and modulation layers).  One block per timestep; one warp per output row, its
// lanes reading consecutive pieces of the row (one 16-byte load per lane for the 256-wide first
// layer) and adding up with shuffles.
__global__ void __launch_bounds__(256) cond_kernel(const bf16* __restrict__ w1, const bf16* __restrict__ b1,
                                                   const bf16* __restrict__ w2, const bf16* __restrict__ b2,
                                                   const float* __restrict__ ts, float* __restrict__ sc, int cdim) {
  __shared__ float emb[256];
  __shared__ float hid[256];
  const float t = ts[blockIdx.x];
  for (int k = threadIdx.x; k < 128; k += blockDim.x) {
    const double f = exp(-log(10000.0) * k / 128.0);
    const double arg = 1000.0 * static_cast<double>(t) * f;
    double s, c;
    sincos(arg, &s, &c);
    emb[k] = static_cast<float>(c);
    emb[128 + k] = static_cast<float>(s);
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  for (int j = warp; j < cdim; j += nwarps) {
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(w1 + static_cast<int64_t>(j) * 256) + lane);
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&raw);
    float a = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(p[i]);
      a = fmaf(f.x, emb[lane * 8 + 2 * i], a);
      a = fmaf(f.y, emb[lane * 8 + 2 * i + 1], a);
    }
    a = warp_sum(a);
    if (lane == 0) {
      a += __bfloat162float(b1[j]);
      hid[j] = a / (1.0f + expf(-a));
    }
  }
  __syncthreads();
  const int per_lane = cdim / 32;  // cdim is a multiple of 32, at most 256
  for (int j = warp; j < cdim; j += nwarps) {
    const bf16* wr = w2 + static_cast<int64_t>(j) * cdim + lane * per_lane;
    float a = 0.f;
    for (int i = 0; i < per_lane; ++i) a = fmaf(__bfloat162float(wr[i]), hid[lane * per_lane + i], a);
    a = warp_sum(a);
    if (lane == 0) {
      a += __bfloat162float(b2[j]);
      sc[static_cast<int64_t>(blockIdx.x) * cdim + j] = a / (1.0f + expf(-a));
    }
  }
}

// ---------------------------------------------------------------------------- modulation
// out[t, r] = W[r, :] . sc[t, :] + bias[r], FP32 sums of BF16 weights and FP32 inputs.  One thread
// per weight row, so that a warp's results for one timestep are 32 consecutive floats (one
// coalesced store); the timesteps are taken TC at a time with FP32 accumulators in registers, the
// row read in 16-byte pieces (again from L1/L2 for each further chunk of timesteps), the inputs
// sc[t, :] broadcast from shared memory.
template <int TC>
__global__ void __launch_bounds__(256) mod_gemv_kernel(const bf16* __restrict__ W, const bf16* __restrict__ bias,
                                                       const float* __restrict__ sc, float* __restrict__ out, int R,
                                                       int cdim, int T, int64_t out_stride) {
  extern __shared__ float s_sc[];  // [T, cdim]
  for (int i = threadIdx.x; i < T * cdim; i += blockDim.x) s_sc[i] = sc[i];
  __syncthreads();
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= R) return;
  const uint4* wr = reinterpret_cast<const uint4*>(W + static_cast<int64_t>(r) * cdim);
  const float bv = __bfloat162float(bias[r]);
  for (int t0 = 0; t0 < T; t0 += TC) {
    float acc[TC];
#pragma unroll
    for (int tt = 0; tt < TC; ++tt) acc[tt] = 0.f;
    for (int k8 = 0; k8 < cdim / 8; ++k8) {
      const uint4 raw = __ldg(wr + k8);
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&raw);
      float w[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(p[i]);
        w[2 * i] = f.x;
        w[2 * i + 1] = f.y;
      }
#pragma unroll
      for (int tt = 0; tt < TC; ++tt) {
        if (TC == 1 || t0 + tt < T) {
          const float4* sp = reinterpret_cast<const float4*>(s_sc + (t0 + tt) * cdim + 8 * k8);
          const float4 s0 = sp[0], s1 = sp[1];
          float a = acc[tt];
          a = fmaf(w[0], s0.x, a);
          a = fmaf(w[1], s0.y, a);
          a = fmaf(w[2], s0.z, a);
          a = fmaf(w[3], s0.w, a);
          a = fmaf(w[4], s1.x, a);
          a = fmaf(w[5], s1.y, a);
          a = fmaf(w[6], s1.z, a);
          a = fmaf(w[7], s1.w, a);
          acc[tt] = a;
        }
      }
    }
#pragma unroll
    for (int tt = 0; tt < TC; ++tt)
      if (TC == 1 || t0 + tt < T) out[static_cast<int64_t>(t0 + tt) * out_stride + r] = acc[tt] + bv;
  }
}

// ---------------------------------------------------------------------------- RoPE table
// Angles of the 64 rotation pairs of a 128-wide head: pairs 0..15 (text index), 16..39
// (patch row), 40..63 (patch column), axis dims 32/48/48, theta 1e4; image token (r, c) at
// (0, r, c), text token j at (j + 1, 0, 0).  Stored as (cos, sin) in FP32, computed in FP64,
// pair-major: table[j * N + token], so that consecutive tokens (the rows a warp of the QKV
// epilogue holds) read one contiguous segment.
__global__ void rope_table_kernel(float2* __restrict__ table, int grid_h, int grid_w, int n_txt) {
  const int n_img = grid_h * grid_w;
  const int n_tok = n_img + n_txt;
  const int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= static_cast<int64_t>(n_tok) * 64) return;
  const int j = static_cast<int>(e / n_tok);
  const int tok = static_cast<int>(e % n_tok);
  int p0 = 0, p1 = 0, p2 = 0;
  if (tok < n_img) {
    p1 = tok / grid_w;
    p2 = tok % grid_w;
  } else {
    p0 = tok - n_img + 1;
  }
  double pos, dim;
  int i;
  if (j < 16) {
    pos = p0; dim = 32.0; i = j;
  } else if (j < 40) {
    pos = p1; dim = 48.0; i = j - 16;
  } else {
    pos = p2; dim = 48.0; i = j - 40;
  }
  const double ang = pos * pow(10000.0, -2.0 * i / dim);
  double s, c;
  sincos(ang, &s, &c);
  table[e] = make_float2(static_cast<float>(c), static_cast<float>(s));
}

// ---------------------------------------------------------------------------- patchify
// latent [h8, w8, 32] -> tokens [(h8/2)(w8/2), 128] BF16, feature (dy*2+dx)*32+ch.
__global__ void patchify_kernel(const float* __restrict__ lat, bf16* __restrict__ tok, int h8, int w8) {
  const int gw = w8 / 2;
  const int64_t n = static_cast<int64_t>(h8 / 2) * gw * 32;  // groups of 4 features
  const int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= n) return;
  const int t = static_cast<int>(e / 32);
  const int f4 = static_cast<int>(e % 32);  // features 4*f4 .. 4*f4+3
  const int q = f4 / 8, ch = (f4 % 8) * 4;
  const int r = t / gw, c = t % gw;
  const int dy = q >> 1, dx = q & 1;
  const float4 v = *reinterpret_cast<const float4*>(lat + ((static_cast<int64_t>(2 * r + dy) * w8) + 2 * c + dx) * 32 + ch);
  reinterpret_cast<uint2*>(tok)[e] = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
}

template <int VPL, int WPR>
cudaError_t ln_launch(const float* x, const float* shift, const float* scale, bf16* h, int rows, int gni, int gnt,
                      float eps, cudaStream_t s) {
  constexpr int kRowsPerBlock = 8 / WPR;
  const int blocks = (rows + kRowsPerBlock - 1) / kRowsPerBlock;
  ln_mod_kernel<VPL, WPR><<<blocks, 256, 0, s>>>(x, shift, scale, h, rows, gni, gnt, eps);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ln_mod(const float* x, const float* shift, const float* scale, bf16* h, int rows, int dim,
                          int gather_n_img, int gather_n_tok, float eps, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  // Rows wider than 2048 are split over two warps (at most 48 values per lane).
  switch (dim / 128) {
    case 1: return ln_launch<1, 1>(x, shift, scale, h, rows, gather_n_img, gather_n_tok, eps, s);
    case 2: return ln_launch<2, 1>(x, shift, scale, h, rows, gather_n_img, gather_n_tok, eps, s);
    case 4: return ln_launch<4, 1>(x, shift, scale, h, rows, gather_n_img, gather_n_tok, eps, s);
    case 8: return ln_launch<8, 1>(x, shift, scale, h, rows, gather_n_img, gather_n_tok, eps, s);
    case 16: return ln_launch<8, 2>(x, shift, scale, h, rows, gather_n_img, gather_n_tok, eps, s);
    case 24: return ln_launch<12, 2>(x, shift, scale, h, rows, gather_n_img, gather_n_tok, eps, s);
    case 32: return ln_launch<8, 4>(x, shift, scale, h, rows, gather_n_img, gather_n_tok, eps, s);
    case 48: return ln_launch<12, 4>(x, shift, scale, h, rows, gather_n_img, gather_n_tok, eps, s);
    case 64: return ln_launch<8, 8>(x, shift, scale, h, rows, gather_n_img, gather_n_tok, eps, s);
    default: return cudaErrorInvalidValue;
  }
}

bool ln_mod_supported(int dim) {
  if (dim % 128) return false;
  switch (dim / 128) {
    case 1: case 2: case 4: case 8: case 16: case 24: case 32: case 48: case 64: return true;
    default: return false;
  }
}

cudaError_t launch_cfg_euler(float* x, const float* vc, const float* vu, int64_t n, float cfg, float sigma,
                             float sigma_next, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const float dt = sigma_next - sigma;
  int64_t blocks = ((n >> 2) + 255) / 256;
  if (blocks < 1) blocks = 1;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
  if (blocks > cap) blocks = cap;
  cfg_euler_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(x, vc, vu, n, cfg, dt);
  return cudaGetLastError();
}

cudaError_t launch_cfg_slg_euler(float* x, const float* vc, const float* vcs, const float* vu, int64_t n, float cfg,
                                 float slg, float sigma, float sigma_next, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const float dt = sigma_next - sigma;
  int64_t blocks = ((n >> 2) + 255) / 256;
  if (blocks < 1) blocks = 1;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 8;
  if (blocks > cap) blocks = cap;
  cfg_slg_euler_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(x, vc, vcs, vu, n, cfg, slg, dt);
  return cudaGetLastError();
}

cudaError_t launch_noise(float* x, int64_t n, uint64_t seed, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const int64_t groups = (n + 3) / 4;
  noise_kernel<<<static_cast<unsigned>((groups + 255) / 256), 256, 0, s>>>(
      x, n, static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32));
  return cudaGetLastError();
}

cudaError_t launch_conditioning(const bf16* w1, const bf16* b1, const bf16* w2, const bf16* b2, const float* ts,
                                float* sc, int T, int cdim, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  cond_kernel<<<T, 256, 0, s>>>(w1, b1, w2, b2, ts, sc, cdim);
  return cudaGetLastError();
}

cudaError_t launch_mod_gemv(const bf16* W, const bf16* bias, const float* sc, float* out, int R, int cdim, int T,
                            int64_t out_stride, cudaStream_t s) {
  if (R <= 0 || T <= 0) return cudaSuccess;
  const size_t smem = static_cast<size_t>(T) * cdim * sizeof(float);
  static std::atomic<uint64_t> configured{0};
  if (!configured_on_device(configured)) {
    cudaError_t e = cudaFuncSetAttribute(mod_gemv_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(mod_gemv_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (e != cudaSuccess) return e;
    mark_configured_on_device(configured);
  }
  const unsigned blocks = static_cast<unsigned>((R + 255) / 256);
  if (T == 1)
    mod_gemv_kernel<1><<<blocks, 256, smem, s>>>(W, bias, sc, out, R, cdim, T, out_stride);
  else
    mod_gemv_kernel<16><<<blocks, 256, smem, s>>>(W, bias, sc, out, R, cdim, T, out_stride);
  return cudaGetLastError();
}

cudaError_t launch_rope_table(float2* table, int grid_h, int grid_w, int n_txt, cudaStream_t s) {
  const int64_t n = static_cast<int64_t>(grid_h * grid_w + n_txt) * 64;
  if (n <= 0) return cudaSuccess;
  rope_table_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(table, grid_h, grid_w, n_txt);
  return cudaGetLastError();
}

cudaError_t launch_patchify(const float* latent, bf16* tokens, int h8, int w8, cudaStream_t s) {
  const int64_t n = static_cast<int64_t>(h8 / 2) * (w8 / 2) * 32;
  if (n <= 0) return cudaSuccess;
  patchify_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(latent, tokens, h8, w8);
  return cudaGetLastError();
}

}  // namespace moss
