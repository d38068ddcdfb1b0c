// Joint (bidirectional) attention of the single-stream DiT on the sm_100a tensor cores.
//
//   O = softmax(Q K^T / sqrt(128)) V    per (branch, head), over the whole [image; text]
//                                       sequence of the branch, no mask.
// (MossInfer integration guide, What works: exact attention; windpaint.ai MOSS-Image specs:
// 24 heads of 128, image and text tokens in one sequence.)
//
// One CTA per (128-query tile, head, branch); two CTAs share an SM so that one CTA's
// softmax overlaps the other's matrix products.  Per CTA (192 threads):
//   warp 0      TMA: the Q tile once, then K_j and V_j (128 keys x 128 dims each, two
//               64-column boxes with 128-byte swizzle) for j = 0.. in order.
//   warp 1      one thread issues S = Q K_j^T (tcgen05, both operands from shared memory,
//               result FP32 in TMEM columns [0,128)) and O += P V_j (P from TMEM, V from
//               shared memory as an MN-major operand, O in TMEM columns [128,256)).
//   warps 2..5  softmax, one query row per thread: online softmax in the log2 domain,
//               P written back as BF16 over the first 64 columns of S, and the lazy
//               rescale of O (only when the running maximum grows by more than 2^8).
//               At the end O / l is stored as BF16.
// Keys past the sequence end (the TMA fills them with zeros) are masked to -inf.
#include "common.cuh"
#include "internal.h"

namespace moss {

namespace {

constexpr int kThreads = 192;
constexpr int kTile = 128;               // queries per CTA and keys per step
constexpr int kHalfBytes = kTile * 128;  // one 64-column (128-byte) box of 128 rows
constexpr int kTileBytes = 2 * kHalfBytes;
constexpr int kSmemBytes = 3 * kTileBytes + 1024 + 256;
constexpr uint32_t kTmemCols = 256;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

__global__ void __launch_bounds__(kThreads, 2)
    attn_kernel(const __grid_constant__ CUtensorMap tm, bf16* __restrict__ out, int n_tok, int heads, int hidden,
                float scale_log2, unsigned* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = smem + kTileBytes;
  uint8_t* sV = smem + 2 * kTileBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 3 * kTileBytes);
  uint64_t* b_q = bars + 0;
  uint64_t* b_kfull = bars + 1;
  uint64_t* b_kempty = bars + 2;
  uint64_t* b_vfull = bars + 3;
  uint64_t* b_vempty = bars + 4;
  uint64_t* b_s = bars + 5;
  uint64_t* b_p = bars + 6;
  uint64_t* b_o = bars + 7;
  uint64_t* b_drain = bars + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 9);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int q0 = blockIdx.x * kTile;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int nkv = (n_tok + kTile - 1) / kTile;

  if (threadIdx.x == 0) {
    mbar_init(b_q, 1);
    mbar_init(b_kfull, 1);
    mbar_init(b_kempty, 1);
    mbar_init(b_vfull, 1);
    mbar_init(b_vempty, 1);
    mbar_init(b_s, 1);
    mbar_init(b_p, 4);
    mbar_init(b_o, 1);
    mbar_init(b_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&tm);
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem;        // S (FP32) and P (BF16 pairs in the first 64 columns)
  const uint32_t tO = tmem + 128;  // O (FP32)

  if (warp == 0) {
    if (lane == 0) {
      const int xq = h * 128, xk = hidden + h * 128, xv = 2 * hidden + h * 128;
      int k_armed = -1, v_armed = -1;  // parity of the last armed phase
      bool ok = true;
      mbar_arrive_expect_tx(b_q, kTileBytes);
      tma_load_3d(sQ, &tm, b_q, xq, q0, b);
      tma_load_3d(sQ + kHalfBytes, &tm, b_q, xq + 64, q0, b);
      for (int j = 0; j < nkv && ok; ++j) {
        if (j > 0 && !mbar_wait(b_kempty, (j - 1) & 1, err, kErrAttnProducer, abort_flag)) {
          ok = false;
          break;
        }
        k_armed = j & 1;
        mbar_arrive_expect_tx(b_kfull, kTileBytes);
        tma_load_3d(sK, &tm, b_kfull, xk, j * kTile, b);
        tma_load_3d(sK + kHalfBytes, &tm, b_kfull, xk + 64, j * kTile, b);
        if (j > 0 && !mbar_wait(b_vempty, (j - 1) & 1, err, kErrAttnProducer, abort_flag)) {
          ok = false;
          break;
        }
        v_armed = j & 1;
        mbar_arrive_expect_tx(b_vfull, kTileBytes);
        tma_load_3d(sV, &tm, b_vfull, xv, j * kTile, b);
        tma_load_3d(sV + kHalfBytes, &tm, b_vfull, xv + 64, j * kTile, b);
      }
      // Before the CTA may exit, every load issued must have landed (bounded wait).
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(smem_u32(b_q), 0) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
      }
      if (k_armed >= 0)
        while (!mbar_try_wait(smem_u32(b_kfull), k_armed) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
        }
      if (v_armed >= 0)
        while (!mbar_try_wait(smem_u32(b_vfull), v_armed) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
        }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t kIdescS = idesc_bf16(128, 128, false);
      constexpr uint32_t kIdescO = idesc_bf16(128, 128, true);
      const uint32_t q_addr = smem_u32(sQ), k_addr = smem_u32(sK), v_addr = smem_u32(sV);
      bool ok = mbar_wait(b_q, 0, err, kErrAttnMma, abort_flag);
      for (int j = 0; j < nkv && ok; ++j) {
        if (!mbar_wait(b_kfull, j & 1, err, kErrAttnMma, abort_flag)) break;
        if (j > 0 && !mbar_wait(b_o, (j - 1) & 1, err, kErrAttnMma, abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < 8; ++k) {  // head dim in steps of 16
          const uint32_t off = (k >> 2) * kHalfBytes + (k & 3) * 32;
          mma_ss(tS, sdesc_sw128(q_addr + off, 16, 1024), sdesc_sw128(k_addr + off, 16, 1024), kIdescS,
                 k > 0 ? 1u : 0u);
        }
        tc_commit(b_s);
        tc_commit(b_kempty);
        if (!mbar_wait(b_p, j & 1, err, kErrAttnMma, abort_flag)) break;
        if (!mbar_wait(b_vfull, j & 1, err, kErrAttnMma, abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < 8; ++k) {  // keys in steps of 16: P columns advance by 8 words
          mma_ts(tO, tS + k * 8, sdesc_sw128(v_addr + k * 16 * 128, kHalfBytes, 1024), kIdescO,
                 (j > 0 || k > 0) ? 1u : 0u);
        }
        tc_commit(b_o);
        tc_commit(b_vempty);
      }
      tc_commit(b_drain);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(smem_u32(b_drain), 0) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
      }
    }
  } else {
    const int quad = warp & 3;
    const int r = quad * 32 + lane;  // query row within the tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    float m_run = -INFINITY;  // running maximum, log2 units (possibly stale by < 2^8)
    float l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      ok = mbar_wait(b_s, j & 1, err, kErrAttnSoftmax, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) {  // warp-uniform: TMEM accesses are .sync.aligned
        ok = false;
        break;
      }
      tc_fence_after();
      const int kvalid = n_tok - j * kTile;  // keys of this step inside the sequence
      float mx = -INFINITY;
      for (int c = 0; c < 4; ++c) {
        float v[32];
        tmem_ld32f(tS + lane_off + c * 32, v);
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (c * 32 + i < kvalid) mx = fmaxf(mx, v[i]);
      }
      mx *= scale_log2;
      const bool grow = mx > m_run + kRescaleThreshold;
      const float m_new = grow ? mx : m_run;
      const float factor = grow ? exp2_approx(m_run - m_new) : 1.0f;  // 0 on the first step
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + lane_off + c * 32, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * factor);
          tmem_st32(tO + lane_off + c * 32, o);
        }
      }
      m_run = m_new;
      float rowsum = 0.f;
      for (int c = 0; c < 4; ++c) {
        float v[32];
        tmem_ld32f(tS + lane_off + c * 32, v);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int k0 = c * 32 + 2 * i;
          const float p0 = k0 < kvalid ? exp2_approx(fmaf(v[2 * i], scale_log2, -m_run)) : 0.f;
          const float p1 = k0 + 1 < kvalid ? exp2_approx(fmaf(v[2 * i + 1], scale_log2, -m_run)) : 0.f;
          rowsum += p0 + p1;
          pk[i] = pack_bf16x2(p0, p1);
        }
        tmem_st16(tS + lane_off + c * 16, pk);
      }
      l_run = l_run * factor + rowsum;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(b_p);
    }
    if (ok) ok = mbar_wait(b_o, (nkv - 1) & 1, err, kErrAttnSoftmax, abort_flag);
    if (__all_sync(0xffffffffu, ok)) {
      tc_fence_after();
      const float inv_l = 1.0f / l_run;
      const int q = q0 + r;
      bf16* dst = out + (static_cast<int64_t>(b) * n_tok + q) * hidden + h * 128;
      for (int c = 0; c < 4; ++c) {
        float v[32];
        tmem_ld32f(tO + lane_off + c * 32, v);
        if (q < n_tok) {
          uint4* d = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            d[i] = make_uint4(pack_bf16x2(v[8 * i] * inv_l, v[8 * i + 1] * inv_l),
                              pack_bf16x2(v[8 * i + 2] * inv_l, v[8 * i + 3] * inv_l),
                              pack_bf16x2(v[8 * i + 4] * inv_l, v[8 * i + 5] * inv_l),
                              pack_bf16x2(v[8 * i + 6] * inv_l, v[8 * i + 7] * inv_l));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_attention(const CUtensorMap& qkv, bf16* o, int batch, int n_tok, int heads, int hidden,
                             cudaStream_t s, unsigned* err) {
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  if (batch <= 0 || n_tok <= 0) return cudaSuccess;
  const float scale_log2 = 1.4426950408889634f / sqrtf(128.0f);
  dim3 grid((n_tok + kTile - 1) / kTile, heads, batch);
  attn_kernel<<<grid, kThreads, kSmemBytes, s>>>(qkv, o, n_tok, heads, hidden, scale_log2, err);
  return cudaGetLastError();
}

}  // namespace moss
