// Joint (bidirectional) attention of the single-stream DiT on the sm_100a tensor cores.
//
//   O = softmax(Q K^T / sqrt(128)) V    per (branch, head), over the whole [image; text]
//                                       sequence of the branch, no mask.
// (MossInfer integration guide, What works: exact attention; windpaint.ai MOSS-Image specs:
// 24 heads of 128, image and text tokens in one sequence.)
//
// One CTA per SM and per (256-query block, head, branch): two 128-query tiles A and B share
// every K/V tile of 128 keys.  TMEM (512 columns): S_A, S_B (FP32 scores, 128 columns each;
// P as BF16 pairs over the first 64 columns of its S) and O_A, O_B (FP32, 128 each).
// Per CTA (384 threads, three warpgroups):
//   warp 0      TMA: Q_A and Q_B once, then K_j and V_j (128 keys x 128 dims, four 64x64 boxes
//               with 128-byte swizzle) into two-slot rings.
//   warp 1      the MMA warp (one elected lane issues): S_A(0), S_B(0), then per key tile j:
//               PV_A(j) in two halves of 64 keys, S_A(j+1), PV_B(j) likewise, S_B(j+1), so
//               the tensor pipe works for one tile while the other tile's softmax runs.  The
//               first half of PV_t(j) starts as soon as the softmax has written the first
//               half of P_t(j).  S_t(j+1) overwrites the columns PV_t(j) reads P_t(j) from;
//               tcgen05.mma operations issued by one thread execute in issue order, so no
//               wait is needed between them.  This warp waits only on named barriers: an
//               mbarrier poll (or any shared- or global-memory load) issued behind queued
//               MMAs stalls until they have been handed to the tensor pipe and leaves it idle
//               for the poll's latency, about 75 cycles per wait measured.
//   warp 2      waits (bounded) until V_j and K_{j+1} have landed and passes that on to the
//               MMA warp through a named barrier, once per step.
//   warp 3      idle (it only lends its registers, below).
//   warps 4..7  softmax of tile A, warps 8..11 of tile B; one query row per thread: the row
//               of 128 scores in one TMEM load for the maximum, the second half's 64 scores
//               loaded again (still in TMEM) once the first P half is handed over, which frees
//               registers for more exponentials in flight; online softmax in the log2 domain with a lazy
//               rescale of O (only when the running maximum grows by more than 2^8).  Three in
//               eight of the exponentials run on the FMA pipe (a cubic), the rest on MUFU: the
//               MUFU unit alone (16 per clock per SM) needs as many cycles as the tensor pipe.
//               When S_t(j) is complete, the commit that signalled it also covers PV_t(j-1),
//               so O_t is stable for the rescale.  At the end O / l is stored as BF16.
// Registers: the kernel is launched at 168 per thread (384 x 168 = 64512); warps 0..3 give
// theirs down to 80 and the softmax warpgroups take 208 (128 x 80 + 256 x 208 = 63488), enough
// for a row of 128 scores plus the packed P (ptxas reports 8 bytes of spill stores, outside the
// MMA warp).  The launcher checks the compiled register count against that sum before the first
// launch.
// Keys past the sequence end (the TMA fills them with zeros) are masked to -inf.
// A test-only argument makes one CTA skip a V load so that its bounded waits run out (the
// library's failure-path self-test); it is -1 in every other launch.
#include "common.cuh"
#include "internal.h"

namespace moss {

namespace {

constexpr int kThreads = 384;
constexpr int kRegsLow = 80;    // warps 0..3 after setmaxnreg.dec (TMA, MMA, K/V forwarding, idle)
constexpr int kRegsHigh = 208;  // warps 4..11 after setmaxnreg.inc
constexpr int kQTile = 128;                     // queries per tile (two tiles per CTA)
constexpr int kKTile = 128;                     // keys per step
constexpr int kBox = 64 * 128;                  // one TMA box: 64 rows x 64 BF16 columns
constexpr int kTileBytes = 4 * kBox;            // 128 rows x 128 dims
constexpr int kSmemBytes = 2 * kTileBytes + 4 * kTileBytes + 1024 + 256;  // Q_A, Q_B, K x2, V x2
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

// Load a 128-row x 128-dim tile as four 64x64 boxes: dims half h, rows r at h*2*kBox + r*kBox,
// giving for each dims half 128 rows of 128 bytes (the K-major 128-byte-swizzle layout).
__device__ __forceinline__ void load_tile(uint8_t* dst, const CUtensorMap* tm, uint64_t* bar, int x, int y, int b) {
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int r = 0; r < 2; ++r) tma_load_3d(dst + h * 2 * kBox + r * kBox, tm, bar, x + 64 * h, y + 64 * r, b);
}

// 32 lanes x 64 columns of 32-bit TMEM words, waiting for completion in the same statement.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr)
      : "memory");
}

// Packed FP32 pairs: one instruction performs the operation on both halves.
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
// Three-input maximum (one instruction on sm_100).
__device__ __forceinline__ float max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// 2^x for a pair of arguments on the FMA pipe (Cody-Waite split x = n + f, n = round(x),
// f in [-0.5, 0.5]; 2^f by a cubic fitted for minimum relative error, 1.0e-4; 2^n added to the
// exponent field).  Arguments below -126 are clamped there (the result is then < 2^-126).
__device__ __forceinline__ void exp2_poly2(float x0, float x1, float& p0, float& p1) {
  const uint64_t x = f2_pack(fmaxf(x0, -126.0f), fmaxf(x1, -126.0f));
  const uint64_t xr = f2_add(x, f2_pack(12582912.0f, 12582912.0f));  // 1.5 * 2^23: rounds to an integer
  const uint64_t n = f2_add(xr, f2_pack(-12582912.0f, -12582912.0f));
  const uint64_t f = f2_fma(n, f2_pack(-1.0f, -1.0f), x);
  uint64_t p = f2_fma(f2_pack(0.05500893f, 0.05500893f), f, f2_pack(0.24221098f, 0.24221098f));
  p = f2_fma(p, f, f2_pack(0.69328293f, 0.69328293f));
  p = f2_fma(p, f, f2_pack(1.0f, 1.0f));
  float q0, q1, r0, r1;
  f2_unpack(p, q0, q1);
  f2_unpack(xr, r0, r1);
  p0 = __int_as_float(__float_as_int(q0) + (__float_as_int(r0) << 23));
  p1 = __int_as_float(__float_as_int(q1) + (__float_as_int(r1) << 23));
}

// MMA issue with each shared-memory descriptor given as its low word (start address and
// leading byte offset); the high word (stride 1024 bytes, version 1, 128-byte swizzle) is the
// same for every operand here and is joined inside the instruction's asm.
constexpr uint32_t kDescHi = (1024u >> 4) | (1u << 14) | (2u << 29);
__device__ __forceinline__ uint32_t desc_lo(uint32_t saddr, uint32_t lbo) {
  return ((saddr >> 4) & 0x3FFFu) | (((lbo >> 4) & 0x3FFFu) << 16);
}
// Issue forms for a whole warp: one lane, chosen by elect.sync, issues.
__device__ __forceinline__ void mma_ss_lo_e(uint32_t d_tmem, uint32_t a_lo, uint32_t b_lo, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t.reg .b64 ad, bd;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "mov.b64 ad, {%1, %5};\n\t"
      "mov.b64 bd, {%2, %5};\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], ad, bd, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_lo), "r"(b_lo), "r"(idesc), "r"(accumulate), "n"(kDescHi)
      : "memory");
}
__device__ __forceinline__ void mma_ts_lo_e(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_lo, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t.reg .b64 bd;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "mov.b64 bd, {%2, %5};\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], bd, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "r"(b_lo), "r"(idesc), "r"(accumulate), "n"(kDescHi)
      : "memory");
}
__device__ __forceinline__ void tc_commit_e(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}
// Bounded wait taken by a whole warp: every lane polls, the result is warp-uniform.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity, unsigned* err, unsigned code,
                                               volatile int* abort) {
  const uint32_t a = smem_u32(bar);
  if (__all_sync(0xffffffffu, mbar_try_wait(a, parity))) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (__all_sync(0xffffffffu, mbar_try_wait(a, parity))) return true;
    if (__any_sync(0xffffffffu, *abort != 0)) return false;
    if (__any_sync(0xffffffffu, globaltimer_ns() - t0 > kWaitTimeoutNs)) {
      if ((threadIdx.x & 31) == 0) {
        atomicCAS(err, 0u, code);
        *abort = 1;
      }
      __syncwarp();
      return false;
    }
  }
}
// Named barriers: waiting on one does not stall behind the waiting warp's queued MMAs.  Whole
// warps only.  Every barrier gets one generation per key step on every path (arrivals are made
// after an abort too, and the waits before them are bounded), and no side can run a
// generation ahead of the other: the softmax warps pass kBarS + t before they arrive on
// kBarP + 2 t + h, and the MMA warp arrives on kBarS + t for step j + 1 only after it has passed
// both P barriers of step j.  So a named-barrier wait can neither complete without its waiter
// nor be left short of arrivals.
constexpr uint32_t kBarKV = 1;   // warp 2 <-> MMA warp rendezvous: V_j and K_{j+1} have landed (64)
constexpr uint32_t kBarP = 2;    // + 2 t + h: half h of P_t(j) is in TMEM (4 softmax warps arrive, 160)
constexpr uint32_t kBarS = 6;    // + t: S_t(j) has been issued (the MMA warp arrives, 160)
__device__ __forceinline__ void named_sync(uint32_t id, uint32_t n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void named_arrive(uint32_t id, uint32_t n) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// P half c of a key step: exponentials of its 64 scores sv against the maximum m (three in eight
// of the pairs on the FMA pipe; keys at or past kvalid get P = 0 when the step is not full), BF16
// pairs into TMEM at tS + 32 c, row sums into acc2; then the MMA warp is told.
__device__ __forceinline__ void p_half(const uint32_t (&sv)[64], int c, bool full, int kvalid, float m,
                                       float scale_log2, uint64_t scale2, uint64_t negm2, uint32_t tS, uint32_t bar,
                                       uint64_t (&acc2)[2]) {
  uint32_t pk[32];
  if (full) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      float x0, x1, p0, p1;
      f2_unpack(f2_fma(f2_pack(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1])), scale2, negm2), x0, x1);
      if ((i & 7) == 1 || (i & 7) == 4 || (i & 7) == 6) {
        exp2_poly2(x0, x1, p0, p1);
      } else {
        p0 = exp2_approx(x0);
        p1 = exp2_approx(x1);
      }
      acc2[i & 1] = f2_add(acc2[i & 1], f2_pack(p0, p1));
      pk[i] = pack_bf16x2(p0, p1);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int k0 = 64 * c + 2 * i;
      const float p0 = k0 < kvalid ? exp2_approx(fmaf(__uint_as_float(sv[2 * i]), scale_log2, -m)) : 0.f;
      const float p1 = k0 + 1 < kvalid ? exp2_approx(fmaf(__uint_as_float(sv[2 * i + 1]), scale_log2, -m)) : 0.f;
      acc2[i & 1] = f2_add(acc2[i & 1], f2_pack(p0, p1));
      pk[i] = pack_bf16x2(p0, p1);
    }
  }
  tmem_st32(tS + 32 * c, pk);
  tc_fence_before();
  __syncwarp();
  named_arrive(bar, 160);
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tm, bf16* __restrict__ out, int n_tok, int heads, int hidden,
                float scale_log2, unsigned* err, int test_skip_v_step) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                        // [2] tiles A, B
  uint8_t* sK = smem + 2 * kTileBytes;       // [2] slots
  uint8_t* sV = smem + 4 * kTileBytes;       // [2] slots
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 6 * kTileBytes);
  uint64_t* b_q = bars + 0;
  uint64_t* b_kfull = bars + 1;   // [2]
  uint64_t* b_kempty = bars + 3;  // [2]
  uint64_t* b_vfull = bars + 5;   // [2]
  uint64_t* b_vempty = bars + 7;  // [2]
  uint64_t* b_s = bars + 9;       // [2] S_t(j) complete (tile t), one phase per j
  uint64_t* b_done = bars + 11;   // every MMA complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 12);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int q0 = blockIdx.x * 2 * kQTile;
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
    }
    mbar_init(b_done, 1);
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
  // S_t at tmem + 128 t, O_t at tmem + 256 + 128 t.

  // Each warpgroup's role code sits inside the branch that sets its register count.
  if (warp < 4) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow));
  if (warp == 0) {
    if (lane == 0) {
      const int xq = h * 128, xk = hidden + h * 128, xv = 2 * hidden + h * 128;
      int k_armed[2] = {-1, -1}, v_armed[2] = {-1, -1};  // parity of the last armed phase
      mbar_arrive_expect_tx(b_q, 2 * kTileBytes);
      load_tile(sQ, &tm, b_q, xq, q0, b);
      load_tile(sQ + kTileBytes, &tm, b_q, xq, q0 + kQTile, b);
      for (int j = 0; j < nkv; ++j) {
        const int slot = j & 1;
        const uint32_t use = (j >> 1) & 1;
        if (j >= 2 && !mbar_wait(&b_kempty[slot], use ^ 1, err, kErrAttnProducer, abort_flag)) break;
        k_armed[slot] = static_cast<int>(use);
        mbar_arrive_expect_tx(&b_kfull[slot], kTileBytes);
        load_tile(sK + slot * kTileBytes, &tm, &b_kfull[slot], xk, j * kKTile, b);
        if (j >= 2 && !mbar_wait(&b_vempty[slot], use ^ 1, err, kErrAttnProducer, abort_flag)) break;
        // Failure-path self-test only: this V tile never lands, so the waits on it run out.
        if (j == test_skip_v_step && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0) continue;
        v_armed[slot] = static_cast<int>(use);
        mbar_arrive_expect_tx(&b_vfull[slot], kTileBytes);
        load_tile(sV + slot * kTileBytes, &tm, &b_vfull[slot], xv, j * kKTile, b);
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
    {
      constexpr uint32_t kIdescS = idesc_bf16(128, kKTile, false);
      constexpr uint32_t kIdescO = idesc_bf16(128, 128, true);
      const uint32_t q_addr = smem_u32(sQ), k_addr = smem_u32(sK), v_addr = smem_u32(sV);
      // Descriptor low words of the operand bases; an offset inside a tile adds (offset >> 4).
      const uint32_t dq0 = desc_lo(q_addr, 16), dk0 = desc_lo(k_addr, 16), dv0 = desc_lo(v_addr, 2 * kBox);
      constexpr uint32_t kTileLo = kTileBytes >> 4;
      // S_t(j) = Q_t K_j^T into S_t.
      auto issue_s = [&](int t, int j) {
        const uint32_t dq = dq0 + t * kTileLo;
        const uint32_t dk = dk0 + (j & 1) * kTileLo;
        const uint32_t d = tmem + 128 * t;
#pragma unroll
        for (int k = 0; k < 8; ++k) {  // head dim in steps of 16
          const uint32_t off = ((k >> 2) * 2 * kBox + (k & 3) * 32) >> 4;
          mma_ss_lo_e(d, dq + off, dk + off, kIdescS, k > 0 ? 1u : 0u);
        }
        tc_commit_e(&b_s[t]);
      };
      // O_t += P_t(j) V_j over keys 64 h .. 64 h + 63, P from columns 32 h .. 32 h + 31 of S_t.
      auto issue_pv = [&](int t, int j, int h) {
        const uint32_t dv = dv0 + (j & 1) * kTileLo;
        const uint32_t d = tmem + 256 + 128 * t, p = tmem + 128 * t;
#pragma unroll
        for (int k = 4 * h; k < 4 * h + 4; ++k)  // keys in steps of 16: P columns advance by 8 words
          mma_ts_lo_e(d, p + k * 8, dv + ((k * 16 * 128) >> 4), kIdescO, (j > 0 || k > 0) ? 1u : 0u);
      };
      const bool ok = mbar_wait_warp(b_q, 0, err, kErrAttnMma, abort_flag) &&
                      mbar_wait_warp(&b_kfull[0], 0, err, kErrAttnMma, abort_flag);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        issue_s(1, 0);
        tc_commit_e(&b_kempty[0]);
      }
      named_arrive(kBarS + 0, 160);
      named_arrive(kBarS + 1, 160);
      // Every named-barrier wait below is matched by arrivals the other warps make on every
      // step, also after an abort (their own waits are bounded), so none of them can hang.
      for (int j = 0; j < nkv; ++j) {
        const bool more = j + 1 < nkv;
        const int nslot = (j + 1) & 1;
        named_sync(kBarKV, 64);
        // tile A: the two halves of P_A(j)
        named_sync(kBarP + 0, 160);
        if (ok) {
          tc_fence_after();
          issue_pv(0, j, 0);
        }
        named_sync(kBarP + 1, 160);
        if (ok) {
          tc_fence_after();
          issue_pv(0, j, 1);
          if (more) issue_s(0, j + 1);
        }
        if (more) named_arrive(kBarS + 0, 160);
        // tile B
        named_sync(kBarP + 2, 160);
        if (ok) {
          tc_fence_after();
          issue_pv(1, j, 0);
        }
        named_sync(kBarP + 3, 160);
        if (ok) {
          tc_fence_after();
          issue_pv(1, j, 1);
          tc_commit_e(&b_vempty[j & 1]);
          if (more) {
            issue_s(1, j + 1);
            tc_commit_e(&b_kempty[nslot]);
          }
        }
        if (more) named_arrive(kBarS + 1, 160);
      }
      tc_commit_e(b_done);
      const uint32_t a = smem_u32(b_done);
      const uint64_t t0 = globaltimer_ns();
      while (!__all_sync(0xffffffffu, mbar_try_wait(a, 0)) && globaltimer_ns() - t0 < kWaitTimeoutNs) {
      }
    }
  } else if (warp == 2) {
    // Forwards the landing of V_j and K_{j+1} to the MMA warp, once per step, unconditionally
    // (a rendezvous: neither side can run a step ahead).
    for (int j = 0; j < nkv; ++j) {
      mbar_wait_warp(&b_vfull[j & 1], (j >> 1) & 1, err, kErrAttnMma, abort_flag);
      if (j + 1 < nkv) mbar_wait_warp(&b_kfull[(j + 1) & 1], ((j + 1) >> 1) & 1, err, kErrAttnMma, abort_flag);
      named_sync(kBarKV, 64);
    }
  }
  } else {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsHigh));
  {
    const int t = (warp - 4) >> 2;   // query tile: 0 = A (warps 4..7), 1 = B (warps 8..11)
    const int quad = warp & 3;       // TMEM lane quadrant
    const int r = quad * 32 + lane;  // query row within the tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t tS = tmem + 128 * t + lane_off;
    const uint32_t tO = tmem + 256 + 128 * t + lane_off;
    float m_run = -INFINITY;  // running maximum, log2 units (possibly stale by < 2^8)
    float l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      // The MMA warp has issued S_t(j) (and passed both P_t(j-1) barriers): this warp cannot
      // arrive on a P barrier a generation ahead of the MMA warp.
      named_sync(kBarS + t, 160);
      if (ok) ok = mbar_wait(&b_s[t], j & 1, err, kErrAttnSoftmax, abort_flag);
      ok = __all_sync(0xffffffffu, ok);  // warp-uniform: TMEM accesses are .sync.aligned
      if (!ok) {  // after an abort: only the arrivals the MMA warp waits for
        named_arrive(kBarP + 2 * t, 160);
        named_arrive(kBarP + 2 * t + 1, 160);
        continue;
      }
      tc_fence_after();
      const int kvalid = n_tok - j * kKTile;  // keys of this step inside the sequence
      const bool full = kvalid >= kKTile;     // warp-uniform
      // The whole row of 128 scores in one TMEM load.
      uint32_t sr[128];
      tmem_ld128(tS, sr);
      float mxp[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) mxp[a] = -INFINITY;
      if (full) {
#pragma unroll
        for (int i = 0; i < 64; ++i)
          mxp[i & 7] = max3(mxp[i & 7], __uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1]));
      } else {
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (i < kvalid) mxp[i & 7] = fmaxf(mxp[i & 7], __uint_as_float(sr[i]));
      }
      const float mx = fmaxf(fmaxf(fmaxf(mxp[0], mxp[1]), fmaxf(mxp[2], mxp[3])),
                             fmaxf(fmaxf(mxp[4], mxp[5]), fmaxf(mxp[6], mxp[7]))) *
                       scale_log2;
      const bool grow = mx > m_run + kRescaleThreshold;
      const float m_new = grow ? mx : m_run;
      const float factor = grow ? exp2_approx(m_run - m_new) : 1.0f;  // 0 on the first step
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
        // PV_t(j-1) was issued before S_t(j) and covered by its commit: O_t is stable.
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + c * 32, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * factor);
          tmem_st32(tO + c * 32, o);
        }
      }
      m_run = m_new;
      // Exponentials; P_t(j) over the first 64 columns of S_t, in two 32-column halves, each
      // signalled to the MMA thread as soon as it is stored.  Row sums in packed pairs.
      const uint64_t scale2 = f2_pack(scale_log2, scale_log2);
      const uint64_t negm2 = f2_pack(-m_run, -m_run);
      uint64_t acc2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
      p_half(reinterpret_cast<const uint32_t(&)[64]>(sr[0]), 0, full, kvalid, m_run, scale_log2, scale2, negm2, tS,
             kBarP + 2 * t, acc2);
      // Keys 64..127 are still in TMEM (P occupies columns 0..63): reloading them lets their
      // registers go free during the first half.
      uint32_t s1[64];
      tmem_ld64(tS + 64, s1);
      p_half(s1, 1, full, kvalid, m_run, scale_log2, scale2, negm2, tS, kBarP + 2 * t + 1, acc2);
      float a0, a1, b0, b1;
      f2_unpack(acc2[0], a0, a1);
      f2_unpack(acc2[1], b0, b1);
      const float rowsum = (a0 + b0) + (a1 + b1);
      l_run = l_run * factor + rowsum;
    }
    if (ok) ok = mbar_wait(b_done, 0, err, kErrAttnSoftmax, abort_flag);
    if (__all_sync(0xffffffffu, ok)) {
      tc_fence_after();
      const float inv_l = 1.0f / l_run;
      const int q = q0 + kQTile * t + r;
      bf16* dst = out + (static_cast<int64_t>(b) * n_tok + q) * hidden + h * 128;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float v[32];
        tmem_ld32f(tO + c * 32, v);
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
                             unsigned* err, std::string* emsg, int test_skip_v_step) {
  static std::atomic<uint64_t> configured{0};
  if (!configured_on_device(configured)) {
    // setmaxnreg.inc waits until the registers it asks for are free in the CTA's pool (its
    // threads x the registers per thread at launch), so a split that does not fit would never
    // return: refuse to launch unless the compiled count covers it.
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, attn_kernel);
    if (e != cudaSuccess) return e;
    if (fa.numRegs * kThreads < 128 * kRegsLow + 256 * kRegsHigh) {
      if (emsg) *emsg = "attention kernel compiled with too few registers for its register split";
      return cudaErrorInvalidConfiguration;
    }
    e = cudaFuncSetAttribute(attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    mark_configured_on_device(configured);
  }
  if (batch <= 0 || n_tok <= 0) return cudaSuccess;
  // The tensor map is built here, from the same box constants the kernel's shared-memory
  // layout and transaction counts use: 64 columns x 64 rows of one branch.
  CUtensorMap tm;
  if (!make_tmap_bf16_3d(&tm, qkv, 3 * static_cast<uint64_t>(hidden), n_tok, batch, 64, kBox / 128, emsg))
    return cudaErrorInvalidValue;
  const float scale_log2 = 1.4426950408889634f / sqrtf(128.0f);
  dim3 grid((n_tok + 2 * kQTile - 1) / (2 * kQTile), heads, batch);
  attn_kernel<<<grid, kThreads, kSmemBytes, s>>>(tm, o, n_tok, heads, hidden, scale_log2, err,
                                                 test_skip_v_step);
  return cudaGetLastError();
}

}  // namespace moss
