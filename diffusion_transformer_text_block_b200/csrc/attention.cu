// Joint (bidirectional) attention of the single-stream DiT on the sm_100a tensor cores.
//
//   O = softmax(Q K^T / sqrt(128)) V    per (branch, head), over the whole [image; text]
//                                       sequence of the branch, no mask.
// (MossInfer integration guide, What works: exact attention; windpaint.ai MOSS-Image specs:
// 24 heads of 128, image and text tokens in one sequence.)
//
// One CTA per (128-query tile, head, branch); two CTAs share an SM.  Keys are taken 64 at a
// time.  TMEM (256 columns per CTA): S buffers 0 and 1 (64 columns each, FP32) and O (128).
// Per CTA (192 threads):
//   warp 0      TMA: the Q tile once, then K_j and V_j (64 keys x 128 dims, two 64-column
//               boxes with 128-byte swizzle) into two-slot rings.
//   warp 1      one thread issues, in this order, S_0, S_1, PV_0, S_2, PV_1, ...:
//               S_j = Q K_j^T into S buffer j%2 (operands in shared memory) and
//               O += P_j V_j (P_j from TMEM, V_j from shared memory as an MN-major operand).
//               S_j+1 is computed while the softmax warps work on S_j.  S_j+2 is issued
//               right after PV_j without waiting for it: MMAs from one thread run in order.
//   warps 2..5  softmax, one query row per thread: online softmax in the log2 domain, P_j as
//               BF16 over the first 32 columns of its S buffer, lazy rescale of O (only when
//               the running maximum grows by more than 2^8, after waiting for the PV product
//               in flight).  At the end O / l is stored as BF16.
// Keys past the sequence end (the TMA fills them with zeros) are masked to -inf.
#include "common.cuh"
#include "internal.h"

namespace moss {

namespace {

constexpr int kThreads = 192;
constexpr int kQTile = 128;                     // queries per CTA
constexpr int kKTile = 64;                      // keys per step
constexpr int kBox = 64 * 128;                  // one TMA box: 64 rows x 64 BF16 columns
constexpr int kQBytes = 4 * kBox;               // Q: 128 rows x 128 dims
constexpr int kKVBytes = 2 * kBox;              // K_j or V_j: 64 rows x 128 dims
constexpr int kSmemBytes = kQBytes + 4 * kKVBytes + 1024 + 256;
constexpr uint32_t kTmemCols = 256;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

__global__ void __launch_bounds__(kThreads, 2)
    attn_kernel(const __grid_constant__ CUtensorMap tm, bf16* __restrict__ out, int n_tok, int heads, int hidden,
                float scale_log2, unsigned* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // Q halves (dims 0..63, 64..127) are 128 rows x 128 B each: rows 0..63 then 64..127.
  uint8_t* sQ = smem;
  uint8_t* sK = smem + kQBytes;                  // 2 slots
  uint8_t* sV = smem + kQBytes + 2 * kKVBytes;   // 2 slots
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kQBytes + 4 * kKVBytes);
  uint64_t* b_q = bars + 0;
  uint64_t* b_kfull = bars + 1;   // [2]
  uint64_t* b_kempty = bars + 3;  // [2]
  uint64_t* b_vfull = bars + 5;   // [2]
  uint64_t* b_vempty = bars + 7;  // [2]
  uint64_t* b_s = bars + 9;       // [2] S_j complete, per S buffer
  uint64_t* b_p = bars + 11;      // [2] P_j written, per S buffer
  uint64_t* b_o = bars + 13;      // PV_j complete (one phase per j)
  uint64_t* b_drain = bars + 14;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 15);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int q0 = blockIdx.x * kQTile;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int nkv = (n_tok + kKTile - 1) / kKTile;

  if (threadIdx.x == 0) {
    mbar_init(b_q, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&b_kfull[i], 1);
      mbar_init(&b_kempty[i], 1);
      mbar_init(&b_vfull[i], 1);
      mbar_init(&b_vempty[i], 1);
      mbar_init(&b_s[i], 1);
      mbar_init(&b_p[i], 4);
    }
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
  const uint32_t tO = tmem + 128;  // O (FP32); S buffer i at tmem + 64 i

  if (warp == 0) {
    if (lane == 0) {
      const int xq = h * 128, xk = hidden + h * 128, xv = 2 * hidden + h * 128;
      int k_armed[2] = {-1, -1}, v_armed[2] = {-1, -1};  // parity of the last armed phase
      mbar_arrive_expect_tx(b_q, kQBytes);
      for (int half = 0; half < 2; ++half)
        for (int r = 0; r < 2; ++r)
          tma_load_3d(sQ + half * 2 * kBox + r * kBox, &tm, b_q, xq + 64 * half, q0 + 64 * r, b);
      for (int j = 0; j < nkv; ++j) {
        const int slot = j & 1;
        const uint32_t use = (j >> 1) & 1;  // this slot's use count parity
        if (j >= 2 && !mbar_wait(&b_kempty[slot], use ^ 1, err, kErrAttnProducer, abort_flag)) break;
        k_armed[slot] = static_cast<int>(use);
        mbar_arrive_expect_tx(&b_kfull[slot], kKVBytes);
        tma_load_3d(sK + slot * kKVBytes, &tm, &b_kfull[slot], xk, j * kKTile, b);
        tma_load_3d(sK + slot * kKVBytes + kBox, &tm, &b_kfull[slot], xk + 64, j * kKTile, b);
        if (j >= 2 && !mbar_wait(&b_vempty[slot], use ^ 1, err, kErrAttnProducer, abort_flag)) break;
        v_armed[slot] = static_cast<int>(use);
        mbar_arrive_expect_tx(&b_vfull[slot], kKVBytes);
        tma_load_3d(sV + slot * kKVBytes, &tm, &b_vfull[slot], xv, j * kKTile, b);
        tma_load_3d(sV + slot * kKVBytes + kBox, &tm, &b_vfull[slot], xv + 64, j * kKTile, b);
      }
      // Before the CTA may exit, every load issued must have landed (bounded wait).
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(smem_u32(b_q), 0) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
      }
      for (int i = 0; i < 2; ++i) {
        if (k_armed[i] >= 0)
          while (!mbar_try_wait(smem_u32(&b_kfull[i]), k_armed[i]) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
          }
        if (v_armed[i] >= 0)
          while (!mbar_try_wait(smem_u32(&b_vfull[i]), v_armed[i]) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
          }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t kIdescS = idesc_bf16(128, kKTile, false);
      constexpr uint32_t kIdescO = idesc_bf16(128, 128, true);
      const uint32_t q_addr = smem_u32(sQ), k_addr = smem_u32(sK), v_addr = smem_u32(sV);
      bool ok = mbar_wait(b_q, 0, err, kErrAttnMma, abort_flag);
      // PV_{j-1}: O += P_{j-1} V_{j-1}
      auto issue_pv = [&](int jj) -> bool {
        const int slot = jj & 1;
        const uint32_t use = (jj >> 1) & 1;
        if (!mbar_wait(&b_p[slot], use, err, kErrAttnMma, abort_flag)) return false;
        if (!mbar_wait(&b_vfull[slot], use, err, kErrAttnMma, abort_flag)) return false;
        tc_fence_after();
        const uint32_t tP = tmem + 64 * slot;
        const uint32_t vs = v_addr + slot * kKVBytes;
#pragma unroll
        for (int k = 0; k < kKTile / 16; ++k)  // keys in steps of 16: P columns advance by 8 words
          mma_ts(tO, tP + k * 8, sdesc_sw128(vs + k * 16 * 128, kBox, 1024), kIdescO, (jj > 0 || k > 0) ? 1u : 0u);
        tc_commit(b_o);
        tc_commit(&b_vempty[slot]);
        return true;
      };
      for (int j = 0; j < nkv && ok; ++j) {
        const int slot = j & 1;
        const uint32_t use = (j >> 1) & 1;
        // S_j reuses the S buffer whose P_{j-2} the PV_{j-2} product reads.  That product
        // was issued earlier by this thread, and tcgen05.mma operations issued by one thread
        // execute in issue order, so it has read P_{j-2} before S_j is written: no wait.
        if (!mbar_wait(&b_kfull[slot], use, err, kErrAttnMma, abort_flag)) break;
        tc_fence_after();
        const uint32_t ks = k_addr + slot * kKVBytes;
#pragma unroll
        for (int k = 0; k < 8; ++k) {  // head dim in steps of 16
          const uint32_t qoff = (k >> 2) * 2 * kBox + (k & 3) * 32;
          const uint32_t koff = (k >> 2) * kBox + (k & 3) * 32;
          mma_ss(tmem + 64 * slot, sdesc_sw128(q_addr + qoff, 16, 1024), sdesc_sw128(ks + koff, 16, 1024), kIdescS,
                 k > 0 ? 1u : 0u);
        }
        tc_commit(&b_s[slot]);
        tc_commit(&b_kempty[slot]);
        if (j >= 1 && !issue_pv(j - 1)) {
          ok = false;
          break;
        }
      }
      if (ok) issue_pv(nkv - 1);
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
      const int slot = j & 1;
      const uint32_t use = (j >> 1) & 1;
      const uint32_t tS = tmem + 64 * slot + lane_off;
      ok = mbar_wait(&b_s[slot], use, err, kErrAttnSoftmax, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) {  // warp-uniform: TMEM accesses are .sync.aligned
        ok = false;
        break;
      }
      tc_fence_after();
      const int kvalid = n_tok - j * kKTile;  // keys of this step inside the sequence
      const bool full = kvalid >= kKTile;     // warp-uniform
      uint32_t sr[64];
      tmem_ld64(tS, sr);
      float mxp[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) mxp[a] = -INFINITY;
      if (full) {
#pragma unroll
        for (int i = 0; i < 64; ++i) mxp[i & 7] = fmaxf(mxp[i & 7], __uint_as_float(sr[i]));
      } else {
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (i < kvalid) mxp[i & 7] = fmaxf(mxp[i & 7], __uint_as_float(sr[i]));
      }
      const float mx = fmaxf(fmaxf(fmaxf(mxp[0], mxp[1]), fmaxf(mxp[2], mxp[3])),
                             fmaxf(fmaxf(mxp[4], mxp[5]), fmaxf(mxp[6], mxp[7]))) *
                       scale_log2;
      const bool grow = mx > m_run + kRescaleThreshold;
      const float m_new = grow ? mx : m_run;
      const float factor = grow ? exp2_approx(m_run - m_new) : 1.0f;  // 0 on the first step
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
        // O may still be accumulating PV_{j-1}: wait for it before rescaling.
        ok = mbar_wait(b_o, (j - 1) & 1, err, kErrAttnSoftmax, abort_flag);
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + lane_off + c * 32, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * factor);
          tmem_st32(tO + lane_off + c * 32, o);
        }
      }
      m_run = m_new;
      float sump[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t pk[32];
      if (full) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float p0 = exp2_approx(fmaf(__uint_as_float(sr[2 * i]), scale_log2, -m_run));
          const float p1 = exp2_approx(fmaf(__uint_as_float(sr[2 * i + 1]), scale_log2, -m_run));
          sump[i & 3] += p0 + p1;
          pk[i] = pack_bf16x2(p0, p1);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float p0 = 2 * i < kvalid ? exp2_approx(fmaf(__uint_as_float(sr[2 * i]), scale_log2, -m_run)) : 0.f;
          const float p1 =
              2 * i + 1 < kvalid ? exp2_approx(fmaf(__uint_as_float(sr[2 * i + 1]), scale_log2, -m_run)) : 0.f;
          sump[i & 3] += p0 + p1;
          pk[i] = pack_bf16x2(p0, p1);
        }
      }
      // P_j (BF16 pairs) over the first 32 columns of its S buffer: the A operand of PV_j.
      tmem_st32(tS, pk);
      l_run = l_run * factor + ((sump[0] + sump[1]) + (sump[2] + sump[3]));
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&b_p[slot]);
    }
    if (ok) ok = mbar_wait(b_o, (nkv - 1) & 1, err, kErrAttnSoftmax, abort_flag);
    if (__all_sync(0xffffffffu, ok)) {
      tc_fence_after();
      const float inv_l = 1.0f / l_run;
      const int q = q0 + r;
      bf16* dst = out + (static_cast<int64_t>(b) * n_tok + q) * hidden + h * 128;
#pragma unroll
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

cudaError_t launch_attention(const bf16* qkv, bf16* o, int batch, int n_tok, int heads, int hidden, cudaStream_t s,
                             unsigned* err, std::string* emsg) {
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  if (batch <= 0 || n_tok <= 0) return cudaSuccess;
  // The tensor map is built here, from the same box constants the kernel's shared-memory
  // layout and transaction counts use: 64 columns x 64 rows of one branch.
  CUtensorMap tm;
  if (!make_tmap_bf16_3d(&tm, qkv, 3 * static_cast<uint64_t>(hidden), n_tok, batch, 64, kBox / 128, emsg))
    return cudaErrorInvalidValue;
  const float scale_log2 = 1.4426950408889634f / sqrtf(128.0f);
  dim3 grid((n_tok + kQTile - 1) / kQTile, heads, batch);
  attn_kernel<<<grid, kThreads, kSmemBytes, s>>>(tm, o, n_tok, heads, hidden, scale_log2, err);
  return cudaGetLastError();
}

}  // namespace moss
