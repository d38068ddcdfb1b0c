// Internal launch interface shared by the library's translation units (not part of the ABI).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <string>

namespace moss {

// One-time per-device setup of a kernel (function attributes are set per device): `done` holds
// one bit per device ordinal.  Two threads may both run the setup the first time; it is
// idempotent.
inline bool configured_on_device(const std::atomic<uint64_t>& done) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  return (done.load(std::memory_order_acquire) >> (dev & 63)) & 1u;
}
inline void mark_configured_on_device(std::atomic<uint64_t>& done) {
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) done.fetch_or(uint64_t{1} << (dev & 63), std::memory_order_release);
}

using bf16 = __nv_bfloat16;

// Residual reduction tiles of the gated-residual epilogue: 16 FP32 columns x 32 rows.
constexpr uint32_t kResidBoxCols = 16;
constexpr uint32_t kResidBoxRows = 32;

// ------------------------------------------------------------------ GEMM epilogue kinds
enum EpiKind : int {
  kEpiF32 = 0,     // C = acc (FP32), test / library GEMM
  kEpiQkv = 1,     // per-head RMSNorm + RoPE on q|k, BF16 store of q|k|v
  kEpiResid = 2,   // x += gate * acc (FP32 read-modify-write)
  kEpiSwiglu = 3,  // act = BF16(SiLU(acc_gate) * acc_up)
  kEpiEmbed = 4,   // x[b, row, :] = acc + bias for every branch b
  kEpiOut = 5,     // unpatchified velocity = acc + bias
  kEpiOutCfg = 6,  // both branches' velocities of one token tile, then the CFG + Euler update of x
};

struct EpiParams {
  int M = 0, N = 0, K = 0;  // GEMM sizes; for kEpiSwiglu N = F (output width)
  float* out_f32 = nullptr;  // kEpiF32: C [M, N]; kEpiResid/kEpiEmbed: x; kEpiOut: v
  bf16* out_bf16 = nullptr;  // kEpiQkv: qkv [M, 3D]; kEpiSwiglu: act [M, F]
  const float* gate = nullptr;       // kEpiResid: [N]
  const bf16* bias = nullptr;        // kEpiEmbed, kEpiOut: [N]
  const float* q_gain = nullptr;     // kEpiQkv: [128]
  const float* k_gain = nullptr;     // kEpiQkv: [128]
  const float2* rope = nullptr;      // kEpiQkv: [64, rope_stride] (cos, sin), pair-major
  int rope_stride = 0;               // kEpiQkv: tokens per pair row of the RoPE table
  int n_tok = 0;                     // tokens per branch (of the first branch when split_rows > 0)
  int split_rows = 0;                // kEpiQkv, a last branch of another length: rows >= split_rows
                                     // belong to it (token = row - split_rows); rows below are
                                     // branches of n_tok tokens (token = row % n_tok)
  int hidden = 0;                    // D
  int n_branch = 0;                  // kEpiEmbed: branches written
  int n_img = 0, grid_w = 0, lat_h8 = 0, lat_w8 = 0;  // kEpiOut, kEpiOutCfg
  float* x_lat = nullptr;            // kEpiOutCfg: the latent [lat_h8, lat_w8, 32], updated in place
  float cfg = 1.0f, dt = 0.0f;       // kEpiOutCfg: guidance scale, sigma_next - sigma
  float eps = 1e-6f;
  int group_m = 16;                  // pair GEMMs: M-tiles per band of the tile order (all N-tiles of
                                     // a band before the next band)
  int a_l2 = 0, b_l2 = 0;            // pair GEMMs: L2 eviction hint of the A and B loads (0 none,
                                     // 1 evict first, 2 evict last)
};

// ------------------------------------------------------------------ tensor maps
bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                       uint32_t box_outer, std::string* err);
bool make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t mid, uint64_t outer,
                       uint32_t box_inner, uint32_t box_mid, std::string* err);

// FP32 [outer, inner] map with a 64-byte swizzle, for TMA reductions into the residual stream.
bool make_tmap_f32_2d_sw64(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                           uint32_t box_outer, std::string* err);

int num_sms();

// Record `msg` as the calling thread's last error (cleared for MOSS_OK) and return `code`.
int set_error(int code, const std::string& msg);
// Add n kernel launches to the library's launch counter.
void count_launches(int n);

// ------------------------------------------------------------------ kernels
// Every GEMM tensor map (A = activations [M, K], B = weights [N, K], BF16) has the box
// {kGemmBoxK, kGemmBoxRows} (the guided output projection: B with 64-row boxes): the kernels' shared-memory layout and transaction counts are
// derived from these two constants.  For kEpiSwiglu, b = gate rows and b2 = up rows.
constexpr uint32_t kGemmBoxK = 64;
constexpr uint32_t kGemmBoxRows = 128;
cudaError_t launch_gemm(EpiKind kind, const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& b2,
                        const EpiParams& ep, cudaStream_t s, unsigned* err);

// qkv: BF16 [batch, n_tok, 3D] (q | k | v); o: BF16 [batch, n_tok, D].  The launcher builds
// the kernel's TMA descriptor itself; on a descriptor error it returns cudaErrorInvalidValue
// with the reason in *emsg.
// test_skip_v_step >= 0 is the failure-path self-test: the CTA of query block 0, head 0, branch 0
// does not load V for that key step, so a bounded wait runs out and the kernel ends with the error
// word set.  -1 in every other call.
cudaError_t launch_attention(const bf16* qkv, bf16* o, int batch, int n_tok, int heads, int hidden, cudaStream_t s,
                             unsigned* err, std::string* emsg, int test_skip_v_step = -1);

// rows of x (FP32, [.., D]) -> h (BF16).  With gather_n_img > 0, output row r reads x row
// (r / gather_n_img) * gather_n_tok + r % gather_n_img (the image rows of every branch).
cudaError_t launch_ln_mod(const float* x, const float* shift, const float* scale, bf16* h, int rows, int dim,
                          int gather_n_img, int gather_n_tok, float eps, cudaStream_t s);

bool ln_mod_supported(int dim);

cudaError_t launch_cfg_euler(float* x, const float* vc, const float* vu, int64_t n, float cfg, float sigma,
                             float sigma_next, cudaStream_t s);

cudaError_t launch_noise(float* x, int64_t n, uint64_t seed, cudaStream_t s);

// Three-pass SLG step: x += (sigma_next - sigma) * (vu + cfg (vc - vu) + slg (vc - vcs)), FP32.
cudaError_t launch_cfg_slg_euler(float* x, const float* vc, const float* vcs, const float* vu, int64_t n, float cfg,
                                 float slg, float sigma, float sigma_next, cudaStream_t s);

// sc[t, :] = SiLU(W2 SiLU(W1 sinusoid(1000 ts[t]) + b1) + b2), t < T.
cudaError_t launch_conditioning(const bf16* w1, const bf16* b1, const bf16* w2, const bf16* b2, const float* ts,
                                float* sc, int T, int cdim, cudaStream_t s);

// out[t * out_stride + r] = W[r, :] . sc[t, :] + bias[r], r < R, t < T.
cudaError_t launch_mod_gemv(const bf16* W, const bf16* bias, const float* sc, float* out, int R, int cdim, int T,
                            int64_t out_stride, cudaStream_t s);

cudaError_t launch_rope_table(float2* table, int grid_h, int grid_w, int n_txt, cudaStream_t s);

cudaError_t launch_patchify(const float* latent, bf16* tokens, int h8, int w8, cudaStream_t s);

// Step cache (first-block cache): per-block FP64 partial sums of |a - ref| and |ref| over n
// elements into partials[2 * change_partial_blocks()]; x += r; d = a - b.
int change_partial_blocks();
cudaError_t launch_change_partials(const float* a, const float* ref, int64_t n, double* partials, cudaStream_t s);
cudaError_t launch_add_inplace(float* x, const float* r, int64_t n, cudaStream_t s);
cudaError_t launch_sub(float* d, const float* a, const float* b, int64_t n, cudaStream_t s);

// Self-test of the device-side wait limit (records kErrSelfTest after about 2 s).
cudaError_t launch_wait_probe(unsigned* err, cudaStream_t s);

}  // namespace moss
