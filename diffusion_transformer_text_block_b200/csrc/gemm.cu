// BF16 GEMM on the sm_100a tensor cores with the DiT block's fused epilogues.
//
//   D[m, n] = sum_k A[m, k] * B[n, k]      A: activations [M, K], B: weights [N, K] (both
//                                          K-contiguous, BF16), FP32 accumulation in TMEM.
//
// Main kernel (`gemm_pair_kernel`): persistent CTA pairs (clusters of two CTAs on
// neighbouring SMs), 320 threads per CTA, one 256 x 256 output tile per pair at a time.
//   warp 0      TMA producer, in both CTAs: this CTA's 128 rows of A and its 128 rows of the
//               256-row B tile (128-byte swizzle) into a 6-slot ring; every load is counted on
//               the even CTA's "full" barrier of the slot.
//   warp 1      MMA issuer, even CTA only: tcgen05.mma.cta_group::2 256x256x16 (four per 64-wide
//               K slice) reads A and B halves from both CTAs' shared memory and accumulates the
//               128 x 256 quarter of each CTA in that CTA's TMEM (two accumulators, 512 columns);
//               tcgen05.commit frees the slot in both CTAs and hands the accumulator to both
//               epilogues.
//   warps 2..9  epilogue, in both CTAs: tcgen05.ld of the accumulator (thread = output row; two
//               warps per TMEM lane quadrant, each owning half of the tile's columns), the fused
//               element-wise tail of the op, and direct global stores (reductions for the gated
//               residual).  The odd CTA's epilogue releases the accumulator on the even CTA's
//               barrier.  RoPE angles are read before waiting for the accumulator.
// Each CTA streams half of every B tile, so a pair moves 3/4 of the operand bytes per output
// of two independent 128-row CTAs, and a 32 KB slot allows a six-deep ring.
// Tiles are visited in bands of group_m M-tiles (all N-tiles of a band before the next band; the
// launch chooses group_m per GEMM shape, 16 by default).
//
// The 128 x 128 output projection (`gemm_kernel`, BN = 128) keeps the single-CTA form.  In the
// guided step its CFG form (kEpiOutCfg, 128 x 64 tiles) gives each CTA one tile of 128 image tokens
// and one half of the 128 patch features: the MMA warp accumulates the conditional rows into the
// first accumulator and the unconditional rows of the same tokens into the second, and the epilogue
// applies the FP32 CFG combine and Euler update to the latent directly (SGLang cookbook, MOSS-Image: 3. Guidance and precision), so the step needs
// no separate update kernel and no velocity round trip through memory.
//
// Epilogues follow the block of the single-stream DiT (windpaint.ai, MOSS-Image specs:
// 24 heads of 128, FFN 8192) with the fused tails the sibling DiT names on B200 (SGLang
// cookbook, Qwen-Image 2.1: Lossless RoPE fusion, Lossless MLP and residual fusion,
// Lossless Q/K normalization).
#include <cstring>

#include "common.cuh"
#include "internal.h"

namespace moss {

namespace {

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kGroupM = 16;
constexpr int kResidStageBytes = static_cast<int>(kResidBoxCols * kResidBoxRows * 4);  // 2 KB per buffer
constexpr int kThreads = 320;  // warp 0 TMA, warp 1 MMA, warps 2..9 epilogue

// The B map of a single-CTA GEMM has a box of BN rows (kGemmBoxRows for BN = 128, 64 rows for the
// guided output projection's half-width tiles), so that B is one box per slot.
template <int BN>
struct GemmShape {
  static_assert(BN == static_cast<int>(kGemmBoxRows) || BN == 64, "single-CTA tiles load B with one box");
  static constexpr int kStages = 6;
  static constexpr int kABytes = kBM * kBK * 2;
  static constexpr int kBBytes = BN * kBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kTmemCols = 2 * BN;
  static constexpr int kSmemBytes = kStages * kStageBytes + 1024 + 256;
};
static_assert(kBM == static_cast<int>(kGemmBoxRows) && kBK == static_cast<int>(kGemmBoxK), "A box");

// CTA-pair tiles: 256 x 256 per pair; per CTA 128 rows of A and 128 rows of B per slot.
// Only the gated-residual epilogue stages its reductions in shared memory; the other
// epilogues leave that space to L1.
template <int EPI>
struct PairShape {
  static constexpr int kStages = 6;
  static constexpr int kABytes = kBM * kBK * 2;                    // 16 KB
  static constexpr int kBBytes = static_cast<int>(kGemmBoxRows) * kBK * 2;  // 16 KB, half of B
  static constexpr int kStageBytes = kABytes + kBBytes;            // 32 KB per CTA
  static constexpr int kTmemCols = 512;                            // two 256-column accumulators
  static constexpr int kEpiWarps = 8;
  static constexpr int kResidBytes = EPI == kEpiResid ? kEpiWarps * 2 * kResidStageBytes : 0;  // 32 KB
  static constexpr int kSmemBytes = kStages * kStageBytes + kResidBytes + 1024 + 256;
  static_assert(kSmemBytes <= 227 * 1024, "pair GEMM shared memory");
};

__device__ __forceinline__ void tile_coords(int tile, int num_m, int num_n, int& mb, int& nb, int group_m = kGroupM) {
  const int band = tile / (group_m * num_n);
  const int m0 = band * group_m;
  const int bm = min(group_m, num_m - m0);
  const int idx = tile - band * group_m * num_n;
  mb = m0 + idx % bm;
  nb = idx / bm;
}

// 32 BF16 values (16 packed pairs) to global memory with an L2 evict-first hint: the QKV and SwiGLU
// outputs are read by the next kernel, not by later tiles of this launch, so they should not push
// the operand bands out of L2 (1.5 % shorter launches at the 1024^2 shape, DRAM bytes unchanged).
__device__ __forceinline__ void store_bf16x32_ef(bf16* dst, const uint32_t (&pk)[16], uint64_t pol) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
    asm volatile("st.global.L2::cache_hint.v4.b32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(dst + 8 * i), "r"(pk[4 * i]),
                 "r"(pk[4 * i + 1]), "r"(pk[4 * i + 2]), "r"(pk[4 * i + 3]), "l"(pol)
                 : "memory");
}

// ------------------------------------------------------------------------ epilogues
// Eight epilogue warps: warp w reads TMEM lanes 32*(w%4).. (its rows) and owns one half of
// the tile's columns (`half`).  tb is the TMEM address of the warp's lanes at the
// accumulator's first column; row is the thread's output row.
template <int BN>
__device__ __forceinline__ void epi_f32(const EpiParams& ep, uint32_t tb, int row, int nb, int half) {
  constexpr int kChunks = BN / 64;  // 32-column chunks per half
#pragma unroll
  for (int cc = 0; cc < kChunks; ++cc) {
    const int c = half * kChunks + cc;
    const int col = nb * BN + c * 32;
    if (col >= ep.N) break;  // warp-uniform
    float v[32];
    tmem_ld32f(tb + c * 32, v);
    if (row < ep.M) {
      float4* d = reinterpret_cast<float4*>(ep.out_f32 + static_cast<int64_t>(row) * ep.N + col);
#pragma unroll
      for (int i = 0; i < 8; ++i) d[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    }
  }
}

// x += gate * acc through TMA reductions: per 16-column piece of its 32 rows, the warp writes
// gate * acc to one of its two 2 KB staging buffers (64-byte swizzle: the 16-byte chunk k of
// row r sits at chunk k ^ ((r >> 1) & 3), conflict-free) and one lane issues an element-wise
// bulk add into the residual stream.  Each residual element receives exactly one add per
// launch, so the result is deterministic.
__device__ __forceinline__ void epi_resid_tma(const EpiParams& ep, const CUtensorMap* xmap, uint32_t tb, int row0,
                                              int nb, int half, int lane, uint8_t* stage, int& issued) {
  if (row0 >= ep.M) return;  // the whole warp is past the last row
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) {
    const int c = half * 4 + cc;
    const int col = nb * 256 + c * 32;
    if (col >= ep.N) break;
    float v[32];
    tmem_ld32f(tb + c * 32, v);
    const float4* g = reinterpret_cast<const float4*>(ep.gate + col);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 gv = __ldg(g + i);
      v[4 * i] *= gv.x;
      v[4 * i + 1] *= gv.y;
      v[4 * i + 2] *= gv.z;
      v[4 * i + 3] *= gv.w;
    }
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      uint8_t* buf = stage + (issued & 1) * kResidStageBytes;
      if (issued >= 2) {
        if (lane == 0) bulk_wait_group_read<1>();  // the buffer's previous reduction has read it
        __syncwarp();
      }
      float4* rowp = reinterpret_cast<float4*>(buf + lane * 64);
#pragma unroll
      for (int k = 0; k < 4; ++k)
        rowp[k ^ ((lane >> 1) & 3)] =
            make_float4(v[16 * hh + 4 * k], v[16 * hh + 4 * k + 1], v[16 * hh + 4 * k + 2], v[16 * hh + 4 * k + 3]);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_reduce_add_2d(xmap, buf, col + 16 * hh, row0);
        bulk_commit_group();
      }
      ++issued;
    }
  }
}

// Token index (within its branch) of a row of the packed [branch; tokens] activations.
__device__ __forceinline__ int token_of_row(const EpiParams& ep, int row) {
  if (ep.split_rows > 0 && row >= ep.split_rows) return row - ep.split_rows;
  return row % ep.n_tok;
}

// The RoPE table is pair-major ([64][n_tok]): for a fixed pair the 32 lanes (consecutive
// tokens) read one contiguous segment.
constexpr int kRopePrefetch = 16;  // rotation pairs read before the accumulator is ready
struct RopePrefetch {
  float2 cs[kRopePrefetch];
};

__device__ __forceinline__ void qkv_prefetch(const EpiParams& ep, int row, int nb, int half, RopePrefetch& pf) {
  const int col = nb * 256 + half * 128;
  if (col < 2 * ep.hidden && col < ep.N) {
    const float2* rope = ep.rope + token_of_row(ep, row);
#pragma unroll
    for (int i = 0; i < kRopePrefetch; ++i) pf.cs[i] = __ldg(rope + static_cast<int64_t>(i) * ep.rope_stride);
  }
}

__device__ __forceinline__ void epi_qkv(const EpiParams& ep, uint32_t tb, int row, int nb, int half,
                                        const RopePrefetch& pf) {
  const int ld = 3 * ep.hidden;
  const int col = nb * 256 + half * 128;
  if (col >= ep.N) return;
  const int region = col / ep.hidden;  // 0 = q, 1 = k, 2 = v
  const uint32_t th = tb + half * 128;
  bf16* dst = ep.out_bf16 + static_cast<int64_t>(row) * ld + col;
  if (region < 2) {
    float ss[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float v[32];
      tmem_ld32f(th + c * 32, v);
#pragma unroll
      for (int i = 0; i < 32; ++i) ss[i & 3] = fmaf(v[i], v[i], ss[i & 3]);
    }
    const float rinv = rsqrtf(((ss[0] + ss[1]) + (ss[2] + ss[3])) * (1.0f / 128.0f) + ep.eps);
    const float* gain = region == 0 ? ep.q_gain : ep.k_gain;
    const float2* rope = ep.rope + token_of_row(ep, row);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float2 cs[16];
#pragma unroll
      for (int i = 0; i < 16; ++i)
        cs[i] = c * 16 + i < kRopePrefetch ? pf.cs[c * 16 + i] : __ldg(rope + static_cast<int64_t>(c * 16 + i) * ep.rope_stride);
      float v[32];
      tmem_ld32f(th + c * 32, v);
      const float4* g4 = reinterpret_cast<const float4*>(gain + c * 32);
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 g = __ldg(g4 + i);
        const float x0 = v[4 * i] * rinv * g.x, x1 = v[4 * i + 1] * rinv * g.y;
        const float x2 = v[4 * i + 2] * rinv * g.z, x3 = v[4 * i + 3] * rinv * g.w;
        const float2 ca = cs[2 * i], cb = cs[2 * i + 1];
        pk[2 * i] = pack_bf16x2(x0 * ca.x - x1 * ca.y, x0 * ca.y + x1 * ca.x);
        pk[2 * i + 1] = pack_bf16x2(x2 * cb.x - x3 * cb.y, x2 * cb.y + x3 * cb.x);
      }
      if (row < ep.M) store_bf16x32_ef(dst + c * 32, pk, l2_policy(1));
    }
  } else {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float v[32];
      tmem_ld32f(th + c * 32, v);
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
      if (row < ep.M) store_bf16x32_ef(dst + c * 32, pk, l2_policy(1));
    }
  }
}

// Accumulator columns [0,128) = gate rows f0.., [128,256) = up rows f0.. of the same f;
// half h handles f0 + 64h .. f0 + 64h + 63.
__device__ __forceinline__ void epi_swiglu(const EpiParams& ep, uint32_t tb, int row, int nb, int half) {
  const int F = ep.N;
#pragma unroll
  for (int cc = 0; cc < 2; ++cc) {
    const int c = half * 2 + cc;
    const int f = nb * 128 + c * 32;
    if (f >= F) break;
    float g[32], u[32];
    tmem_ld32f(tb + c * 32, g);
    tmem_ld32f(tb + 128 + c * 32, u);
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float a0 = g[2 * i] / (1.0f + __expf(-g[2 * i])) * u[2 * i];
      const float a1 = g[2 * i + 1] / (1.0f + __expf(-g[2 * i + 1])) * u[2 * i + 1];
      pk[i] = pack_bf16x2(a0, a1);
    }
    if (row < ep.M) store_bf16x32_ef(ep.out_bf16 + static_cast<int64_t>(row) * F + f, pk, l2_policy(1));
  }
}

__device__ __forceinline__ void epi_embed(const EpiParams& ep, uint32_t tb, int row, int nb, int half) {
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) {
    const int c = half * 4 + cc;
    const int col = nb * 256 + c * 32;
    if (col >= ep.N) break;
    float v[32];
    tmem_ld32f(tb + c * 32, v);
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] += __bfloat162float(ep.bias[col + i]);
    if (row < ep.M) {
      for (int b = 0; b < ep.n_branch; ++b) {
        float4* d = reinterpret_cast<float4*>(
            ep.out_f32 + (static_cast<int64_t>(b) * ep.n_tok + row) * ep.N + col);
#pragma unroll
        for (int i = 0; i < 8; ++i) d[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
      }
    }
  }
}

// Row = b * n_img + token; column j = (dy*2+dx)*32 + ch -> latent [b, 2r+dy, 2c+dx, ch].
// BN = 128: half h handles dy = h.
__device__ __forceinline__ void epi_out(const EpiParams& ep, uint32_t tb, int row, int half) {
  const int b = row / ep.n_img;
  const int tok = row - b * ep.n_img;
  const int r = tok / ep.grid_w;
  const int cc = tok - r * ep.grid_w;
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const int c = half * 2 + q;
    float v[32];
    tmem_ld32f(tb + c * 32, v);
    if (row < ep.M) {
      const int dy = c >> 1, dx = c & 1;
      float4* d = reinterpret_cast<float4*>(
          ep.out_f32 +
          ((static_cast<int64_t>(b) * ep.lat_h8 + 2 * r + dy) * ep.lat_w8 + 2 * cc + dx) * 32);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int j = c * 32 + 4 * i;
        d[i] = make_float4(v[4 * i] + __bfloat162float(ep.bias[j]), v[4 * i + 1] + __bfloat162float(ep.bias[j + 1]),
                           v[4 * i + 2] + __bfloat162float(ep.bias[j + 2]),
                           v[4 * i + 3] + __bfloat162float(ep.bias[j + 3]));
      }
    }
  }
}

// The guided step's output projection, for one tile of 128 image tokens and one 64-column half nh of
// the 128 patch features: accumulator 0 (TMEM columns 0..63) holds the conditional rows, accumulator
// 1 (columns 64..127) the unconditional rows of the same tokens; warp half h takes the 32 features
// of chunk c = 2 nh + h (dy = nh, dx = h).  x[lat] += dt * (v_u + cfg (v_c - v_u)) with v = acc +
// bias, in the order and rounding of the standalone CFG + Euler kernel.
__device__ __forceinline__ void epi_out_cfg(const EpiParams& ep, uint32_t tb0, int tok, int nh, int half) {
  const bool valid = tok < ep.n_img;
  const int r = tok / ep.grid_w;
  const int cc = tok - r * ep.grid_w;
  const int c = 2 * nh + half;
  float vc[32], vu[32];
  tmem_ld32f(tb0 + half * 32, vc);
  tmem_ld32f(tb0 + 64 + half * 32, vu);
  if (valid) {
    const int dy = c >> 1, dx = c & 1;
    float4* xp = reinterpret_cast<float4*>(ep.x_lat +
                                           ((static_cast<int64_t>(2 * r + dy) * ep.lat_w8) + 2 * cc + dx) * 32);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float4 a = xp[i];
      float cv[4], uv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float bj = __bfloat162float(ep.bias[c * 32 + 4 * i + e]);
        cv[e] = vc[4 * i + e] + bj;
        uv[e] = vu[4 * i + e] + bj;
      }
      a.x = fmaf(ep.dt, fmaf(ep.cfg, cv[0] - uv[0], uv[0]), a.x);
      a.y = fmaf(ep.dt, fmaf(ep.cfg, cv[1] - uv[1], uv[1]), a.y);
      a.z = fmaf(ep.dt, fmaf(ep.cfg, cv[2] - uv[2], uv[2]), a.z);
      a.w = fmaf(ep.dt, fmaf(ep.cfg, cv[3] - uv[3], uv[3]), a.w);
      xp[i] = a;
    }
  }
}

// ------------------------------------------------------------------------ the kernel
// Ten warps: three share one SM sub-partition, whose register file caps them at 168 each.
template <int BN, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmB2, const EpiParams ep, unsigned* err) {
  using S = GemmShape<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + S::kStages * S::kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kStages * S::kStageBytes);
  uint64_t* empty = full + S::kStages;
  uint64_t* tfull = empty + S::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // kEpiOutCfg: a work unit is one tile of 128 image tokens made of two consecutive tiles, the
  // conditional rows (accumulator 0) and the unconditional rows (accumulator 1); otherwise a unit
  // is one output tile.
  constexpr int kPer = EPI == kEpiOutCfg ? 2 : 1;
  const int num_m = (ep.M + kBM - 1) / kBM;
  const int num_n = (ep.N + BN - 1) / BN;
  constexpr int kHalves = EPI == kEpiOutCfg ? 128 / BN : 1;  // N-parts of the 128 patch features
  const int num_units = EPI == kEpiOutCfg ? ((ep.n_img + kBM - 1) / kBM) * kHalves : num_m * num_n;
  const int num_kb = ep.K / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 8);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, S::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int armed[S::kStages];  // parity of the last phase armed on full[s], -1 = never
#pragma unroll
      for (int s2 = 0; s2 < S::kStages; ++s2) armed[s2] = -1;
      for (int unit = blockIdx.x; unit < num_units && ok; unit += gridDim.x)
        for (int sub = 0; sub < kPer && ok; ++sub) {
          int arow, brow;
          if constexpr (EPI == kEpiOutCfg) {
            arow = sub * ep.n_img + (unit / kHalves) * kBM;  // branch `sub`, tokens (unit / kHalves) * 128 ..
            brow = (unit % kHalves) * BN;
          } else {
            int mb, nb;
            tile_coords(unit, num_m, num_n, mb, nb);
            arow = mb * kBM;
            brow = nb * BN;
          }
          for (int kb = 0; kb < num_kb; ++kb) {
            if (!mbar_wait(&empty[stage], phase ^ 1, err, kErrGemmProducer, abort_flag)) {
              ok = false;
              break;
            }
            armed[stage] = static_cast<int>(phase);
            mbar_arrive_expect_tx(&full[stage], S::kStageBytes);
            tma_load_2d(sA + stage * S::kABytes, &tmA, &full[stage], kb * kBK, arow);
            tma_load_2d(sB + stage * S::kBBytes, &tmB, &full[stage], kb * kBK, brow);
            if (++stage == S::kStages) {
              stage = 0;
              phase ^= 1;
            }
          }
        }
      if (!ok) {
        // Let the loads already issued land before the CTA can exit (bounded as well).
        for (int s2 = 0; s2 < S::kStages; ++s2) {
          if (armed[s2] < 0) continue;
          const uint32_t a = smem_u32(&full[s2]);
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(a, static_cast<uint32_t>(armed[s2])) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t kIdesc = idesc_bf16(kBM, BN, false);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int it = 0;
      const int num_tiles = num_units * kPer;  // this CTA's tiles come in runs of kPer (one unit)
      for (int tile = blockIdx.x * kPer; tile < num_tiles && ok;
           tile += (tile % kPer == kPer - 1) ? (gridDim.x - 1) * kPer + 1 : 1, ++it) {
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1, err, kErrGemmMma, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&full[stage], phase, err, kErrGemmMma, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * S::kABytes);
          const uint32_t b0 = smem_u32(sB + stage * S::kBBytes);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            const uint64_t ad = sdesc_sw128(a0 + k * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(b0 + k * 32, 16, 1024);
            mma_ss(d_tmem, ad, bd, kIdesc, (kb | k) != 0 ? 1u : 0u);
          }
          tc_commit(&empty[stage]);
          if (++stage == S::kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (ok) tc_commit(&tfull[acc]);
      }
      // Every MMA issued by this thread has completed once `drain` flips: only then may
      // the TMEM be released, on the normal path and after an abort alike.
      tc_commit(drain);
      const uint32_t a = smem_u32(drain);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(a, 0) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
      }
    }
  } else {
    const int quad = warp & 3;          // TMEM lane quadrant this warp may access
    const int half = (warp - 2) >> 2;   // which half of the tile's columns it owns
    int it = 0;
    if constexpr (EPI == kEpiOutCfg) {
      // Both accumulators of a unit (it even: accumulator 0, then 1 in the same phase).
      for (int unit = blockIdx.x; unit < num_units; unit += gridDim.x, it += 2) {
        const uint32_t acc_phase = (it >> 1) & 1;
        const bool ok = mbar_wait(&tfull[0], acc_phase, err, kErrGemmEpilogue, abort_flag) &&
                        mbar_wait(&tfull[1], acc_phase, err, kErrGemmEpilogue, abort_flag);
        if (!__all_sync(0xffffffffu, ok)) break;  // warp-uniform: TMEM loads are .sync.aligned
        tc_fence_after();
        const uint32_t tb = tmem_base + (static_cast<uint32_t>(quad * 32) << 16);
        epi_out_cfg(ep, tb, (unit / kHalves) * kBM + quad * 32 + lane, unit % kHalves, half);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&tempty[0]);
          mbar_arrive(&tempty[1]);
        }
      }
    }
    for (int tile = blockIdx.x; EPI != kEpiOutCfg && tile < num_units; tile += gridDim.x, ++it) {
      int mb, nb;
      tile_coords(tile, num_m, num_n, mb, nb);
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      const int row = mb * kBM + quad * 32 + lane;
      // Operands of the epilogue that do not depend on the accumulator are fetched first.
      RopePrefetch qp;
      if constexpr (EPI == kEpiQkv) qkv_prefetch(ep, row, nb, half, qp);
      const bool ok = mbar_wait(&tfull[acc], acc_phase, err, kErrGemmEpilogue, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;  // warp-uniform: TMEM loads are .sync.aligned
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * BN;
      if constexpr (EPI == kEpiF32) epi_f32<BN>(ep, tb, row, nb, half);
      if constexpr (EPI == kEpiQkv) epi_qkv(ep, tb, row, nb, half, qp);
      if constexpr (EPI == kEpiSwiglu) epi_swiglu(ep, tb, row, nb, half);
      if constexpr (EPI == kEpiEmbed) epi_embed(ep, tb, row, nb, half);
      if constexpr (EPI == kEpiOut) epi_out(ep, tb, row, half);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, S::kTmemCols);
  }
}

// ------------------------------------------------------------------------ CTA-pair kernel
template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmB2, const __grid_constant__ CUtensorMap tmX,
                     const EpiParams ep, unsigned* err) {
  using S = PairShape<EPI>;
  constexpr int kTileM = 2 * kBM;  // rows per pair tile
  constexpr int kTileN = 256;      // accumulator columns per tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + S::kStages * S::kABytes;
  uint8_t* sResid = smem + S::kStages * S::kStageBytes;  // 1024-aligned: kStageBytes is 32 KB
  uint64_t* full = reinterpret_cast<uint64_t*>(sResid + S::kResidBytes);
  uint64_t* empty = full + S::kStages;
  uint64_t* tfull = empty + S::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: issues the MMAs, 1: its peer
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int num_pairs = gridDim.x >> 1;
  const int num_m = (ep.M + kTileM - 1) / kTileM;
  const int num_n = EPI == kEpiSwiglu ? (ep.N + 127) / 128 : (ep.N + kTileN - 1) / kTileN;
  const int num_tiles = num_m * num_n;
  const int num_kb = ep.K / kBK;
  const int group_m = ep.group_m > 0 ? ep.group_m : kGroupM;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 16);  // eight epilogue warps of each CTA (used in the even CTA)
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (EPI == kEpiSwiglu) tma_prefetch_desc(&tmB2);
    if (EPI == kEpiResid) tma_prefetch_desc(&tmX);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, S::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers are initialised and their TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int armed[S::kStages];  // leader: parity of the last phase armed on full[s], -1 = never
#pragma unroll
      for (int s2 = 0; s2 < S::kStages; ++s2) armed[s2] = -1;
      const CUtensorMap* bmap = (EPI == kEpiSwiglu && !leader) ? &tmB2 : &tmB;
      const uint64_t a_pol = l2_policy(ep.a_l2), b_pol = l2_policy(ep.b_l2);
      for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
        int mb, nb;
        tile_coords(tile, num_m, num_n, mb, nb, group_m);
        // Even CTA: gate rows (SwiGLU) or B rows 0..127 of the tile; odd CTA: up rows or 128..255.
        const int brow = EPI == kEpiSwiglu ? nb * 128 : nb * kTileN + static_cast<int>(rank) * 128;
        const int arow = mb * kTileM + static_cast<int>(rank) * kBM;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, err, kErrGemmProducer, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t full_leader = mapa_shared(smem_u32(&full[stage]), 0);
          if (leader) {
            armed[stage] = static_cast<int>(phase);
            mbar_arrive_expect_tx(&full[stage], 2 * S::kStageBytes);
          }
          if (ep.a_l2)
            tma_load_2d_pair_hint(sA + stage * S::kABytes, &tmA, full_leader, kb * kBK, arow, a_pol);
          else
            tma_load_2d_pair(sA + stage * S::kABytes, &tmA, full_leader, kb * kBK, arow);
          if (ep.b_l2)
            tma_load_2d_pair_hint(sB + stage * S::kBBytes, bmap, full_leader, kb * kBK, brow, b_pol);
          else
            tma_load_2d_pair(sB + stage * S::kBBytes, bmap, full_leader, kb * kBK, brow);
          if (++stage == S::kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok && leader) {
        // Let the loads already issued land before the CTA can exit (bounded as well).
        for (int s2 = 0; s2 < S::kStages; ++s2) {
          if (armed[s2] < 0) continue;
          const uint32_t a = smem_u32(&full[s2]);
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(a, static_cast<uint32_t>(armed[s2])) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      constexpr uint32_t kIdesc = idesc_bf16(kTileM, kTileN, false);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int it = 0;
      for (int tile = pair; tile < num_tiles && ok; tile += num_pairs, ++it) {
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1, err, kErrGemmMma, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kTileN;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&full[stage], phase, err, kErrGemmMma, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * S::kABytes);
          const uint32_t b0 = smem_u32(sB + stage * S::kBBytes);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            const uint64_t ad = sdesc_sw128(a0 + k * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(b0 + k * 32, 16, 1024);
            mma_ss_pair(d_tmem, ad, bd, kIdesc, (kb | k) != 0 ? 1u : 0u);
          }
          tc_commit_pair_both(&empty[stage], 0x3);  // the slot in both CTAs
          if (++stage == S::kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (ok) tc_commit_pair_both(&tfull[acc], 0x3);  // both CTAs' epilogues
      }
      // Every MMA issued by this thread has completed once `drain` flips: only then may
      // either CTA release its TMEM, on the normal path and after an abort alike.
      tc_commit_pair(drain);
      const uint32_t a = smem_u32(drain);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(a, 0) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
      }
    }
  } else {
    const int quad = warp & 3;          // TMEM lane quadrant this warp may access
    const int half = (warp - 2) >> 2;   // which half of the tile's columns it owns
    uint8_t* stage = sResid + (warp - 2) * 2 * kResidStageBytes;
    int issued = 0;                     // residual reductions this warp has issued
    int it = 0;
    for (int tile = pair; tile < num_tiles; tile += num_pairs, ++it) {
      int mb, nb;
      tile_coords(tile, num_m, num_n, mb, nb, group_m);
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      const int row0 = mb * kTileM + static_cast<int>(rank) * kBM + quad * 32;
      const int row = row0 + lane;
      RopePrefetch qp;
      if constexpr (EPI == kEpiQkv) qkv_prefetch(ep, row, nb, half, qp);
      const bool ok = mbar_wait(&tfull[acc], acc_phase, err, kErrGemmEpilogue, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;  // warp-uniform: TMEM loads are .sync.aligned
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * kTileN;
      if constexpr (EPI == kEpiF32) epi_f32<kTileN>(ep, tb, row, nb, half);
      if constexpr (EPI == kEpiResid) epi_resid_tma(ep, &tmX, tb, row0, nb, half, lane, stage, issued);
      if constexpr (EPI == kEpiQkv) epi_qkv(ep, tb, row, nb, half, qp);
      if constexpr (EPI == kEpiSwiglu) epi_swiglu(ep, tb, row, nb, half);
      if constexpr (EPI == kEpiEmbed) epi_embed(ep, tb, row, nb, half);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader)
          mbar_arrive(&tempty[acc]);
        else
          mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));
      }
    }
    // The reductions must have read their staging buffers (and completed) before exit.
    if (EPI == kEpiResid && lane == 0) bulk_wait_group_all();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the even CTA's MMAs into both TMEMs are complete (drained above)
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, S::kTmemCols);
  }
}

template <int BN, int EPI>
cudaError_t launch_single(const CUtensorMap& a, const CUtensorMap& b, const EpiParams& ep, cudaStream_t s,
                          unsigned* err) {
  using S = GemmShape<BN>;
  static std::atomic<uint64_t> configured{0};
  if (!configured_on_device(configured)) {
    cudaError_t e = cudaFuncSetAttribute(gemm_kernel<BN, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         S::kSmemBytes);
    if (e != cudaSuccess) return e;
    mark_configured_on_device(configured);
  }
  const int tiles = EPI == kEpiOutCfg ? ((ep.n_img + kBM - 1) / kBM) * (128 / BN)
                                     : ((ep.M + kBM - 1) / kBM) * ((ep.N + BN - 1) / BN);
  const int grid = tiles < num_sms() ? tiles : num_sms();
  if (grid <= 0) return cudaSuccess;
  gemm_kernel<BN, EPI><<<grid, kThreads, S::kSmemBytes, s>>>(a, b, b, ep, err);
  return cudaGetLastError();
}

template <int EPI>
cudaError_t launch_pair(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& b2, const EpiParams& ep,
                        cudaStream_t s, unsigned* err) {
  using S = PairShape<EPI>;
  static std::atomic<uint64_t> configured{0};
  if (!configured_on_device(configured)) {
    cudaError_t e = cudaFuncSetAttribute(gemm_pair_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         S::kSmemBytes);
    if (e != cudaSuccess) return e;
    mark_configured_on_device(configured);
  }
  // The residual stream's reduction descriptor is built here from the same box constants the
  // epilogue's staging layout uses.
  CUtensorMap xmap;
  std::memset(&xmap, 0, sizeof xmap);
  if (EPI == kEpiResid &&
      !make_tmap_f32_2d_sw64(&xmap, ep.out_f32, ep.N, ep.M, kResidBoxCols, kResidBoxRows, nullptr))
    return cudaErrorInvalidValue;
  const int num_m = (ep.M + 2 * kBM - 1) / (2 * kBM);
  const int num_n = EPI == kEpiSwiglu ? (ep.N + 127) / 128 : (ep.N + 255) / 256;
  const int tiles = num_m * num_n;
  const int pairs = tiles < num_sms() / 2 ? tiles : num_sms() / 2;
  if (pairs <= 0) return cudaSuccess;
  gemm_pair_kernel<EPI><<<2 * pairs, kThreads, S::kSmemBytes, s>>>(a, b, b2, xmap, ep, err);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm(EpiKind kind, const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& b2,
                        const EpiParams& ep, cudaStream_t s, unsigned* err) {
  switch (kind) {
    case kEpiF32: return launch_pair<kEpiF32>(a, b, b2, ep, s, err);
    case kEpiQkv: return launch_pair<kEpiQkv>(a, b, b2, ep, s, err);
    case kEpiResid: return launch_pair<kEpiResid>(a, b, b2, ep, s, err);
    case kEpiSwiglu: return launch_pair<kEpiSwiglu>(a, b, b2, ep, s, err);
    case kEpiEmbed: return launch_pair<kEpiEmbed>(a, b, b2, ep, s, err);
    case kEpiOut: return launch_single<128, kEpiOut>(a, b, ep, s, err);
    case kEpiOutCfg: return launch_single<64, kEpiOutCfg>(a, b, ep, s, err);  // b: box of 64 rows
  }
  return cudaErrorInvalidValue;
}

}  // namespace moss
