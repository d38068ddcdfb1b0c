// C ABI of the library (declared in include/moss_dit.h): argument checking, the model and
// its workspace, TMA descriptors, per-class kernel timing, and the orchestration of the
// denoising step (block -> forward -> CFG/Euler step -> sampling loop).
//
// The step follows the SGLang cookbook for MOSS-Image (3. Guidance and precision): two DiT
// passes for CFG with an empty negative prompt, the unconditional pass skipping the
// requested layers inside the slg window, FP32 CFG and scheduler arithmetic; and the
// defaults of windpaint.ai's MOSS-Image page (Recommended settings: 50 steps, shift 5,
// CFG 3, uncond_skip_layers [22]).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <limits>
#include <vector>

#include "../../include/moss_dit.h"
#include "internal.h"

namespace moss {

// ------------------------------------------------------------------------------ errors
static thread_local std::string g_last_error;

static int fail(int code, const std::string& msg) {
  g_last_error = msg;
  return code;
}

static int cuda_fail(cudaError_t e, const char* what) {
  const int code = e == cudaErrorMemoryAllocation ? MOSS_ERR_OOM : MOSS_ERR_CUDA;
  return fail(code, std::string(what) + ": " + cudaGetErrorString(e));
}

#define MOSS_CUDA(call, what)                 \
  do {                                        \
    cudaError_t e_ = (call);                  \
    if (e_ != cudaSuccess) return cuda_fail(e_, what); \
  } while (0)

static std::atomic<int64_t> g_launches{0};

int set_error(int code, const std::string& msg) {
  g_last_error = msg;
  return code;
}

void count_launches(int n) { g_launches += n; }

// ------------------------------------------------------------------------------ device info
int num_sms() {
  static int cached[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cached[dev] = n > 0 ? n : 148;
  }
  return cached[dev];
}

// One device error word per device, set by kernels whose bounded wait gave up.
static unsigned* g_err_word[64] = {nullptr};
static std::mutex g_err_mu;

static unsigned* device_error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_err_mu);
  if (!g_err_word[dev]) {
    unsigned* p = nullptr;
    if (cudaMalloc(&p, 256) != cudaSuccess) return nullptr;
    if (cudaMemset(p, 0, 256) != cudaSuccess) return nullptr;
    g_err_word[dev] = p;
  }
  return g_err_word[dev];
}

// ------------------------------------------------------------------------------ TMA maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                       uint32_t box_outer, std::string* err) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) {
    if (err) *err = "cuTensorMapEncodeTiled is not available from the driver";
    return false;
  }
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    if (err) {
      char buf[160];
      snprintf(buf, sizeof buf, "cuTensorMapEncodeTiled failed (%d) for a [%llu, %llu] BF16 tensor", int(r),
               (unsigned long long)outer, (unsigned long long)inner);
      *err = buf;
    }
    return false;
  }
  return true;
}

bool make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t mid, uint64_t outer,
                       uint32_t box_inner, uint32_t box_mid, std::string* err) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) {
    if (err) *err = "cuTensorMapEncodeTiled is not available from the driver";
    return false;
  }
  cuuint64_t dims[3] = {inner, mid, outer};
  cuuint64_t strides[2] = {inner * 2, inner * mid * 2};
  cuuint32_t box[3] = {box_inner, box_mid, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    if (err) *err = "cuTensorMapEncodeTiled failed for a 3-D BF16 tensor";
    return false;
  }
  return true;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool make_tmap_f32_2d_sw64(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                           uint32_t box_outer, std::string* err) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) {
    if (err) *err = "cuTensorMapEncodeTiled is not available from the driver";
    return false;
  }
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 4};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    if (err) *err = "cuTensorMapEncodeTiled failed for an FP32 residual tensor";
    return false;
  }
  return true;
}



}  // namespace moss

using namespace moss;

// ------------------------------------------------------------------------------ the model
struct ProfRec {
  int cls;
  int ev0, ev1;
};

struct moss_model {
  moss_config cfg;
  moss_weights w;
  int device = 0;
  int64_t rows_cap = 0;  // max_batch * max_tokens
  int64_t img_cap = 0;   // max image tokens
  // workspace (owned)
  float* x = nullptr;
  bf16* h = nullptr;
  bf16* qkv = nullptr;
  bf16* attn = nullptr;
  bf16* act = nullptr;
  bf16* patches = nullptr;
  float* v = nullptr;
  float2* rope = nullptr;
  float* mod = nullptr;  // [max_steps, mod_stride]
  float* sc = nullptr;   // [max_steps, C]
  float* tvals = nullptr;
  int64_t mod_stride = 0;
  // The schedule whose per-step modulation m->mod holds (rows 0..steps-1), or steps 0 when it
  // holds something else (one timestep of a forward or block call).
  int mod_sched_steps = 0;
  double mod_sched_shift = 0.0;
  int rope_gh = -1, rope_gw = -1, rope_nt = -1;
  int rope_n = 0;  // tokens of the cached RoPE table (its pair-row stride)
  unsigned* err = nullptr;
  // first-block step cache (allocated on first use): block 0's output at the last full call,
  // the residual of blocks 1..L-1 of that call, and the change partial sums
  float* cache_ref = nullptr;
  float* cache_res = nullptr;
  double* chg_dev = nullptr;
  double* chg_host = nullptr;  // pinned
  // staging of moss_denoise_step_host (allocated on first use): the latent and both prompts
  float* stage_x = nullptr;     // [max_latent_hw * 32]
  float* stage_text = nullptr;  // [2 * max_tokens * D]
  // text path (moss_text_refiner_set): weights, descriptors, the blocks' fixed modulation
  bool has_text = false;
  moss_text_weights tw;
  std::vector<CUtensorMap> tt_qkv, tt_wo, tt_wg, tt_wu, tt_wd;
  CUtensorMap tt_proj;
  float* tt_mod = nullptr;  // [6 D]: shift 0, scale 0, gate 1 (twice)
  // weight descriptors
  std::vector<CUtensorMap> tm_qkv, tm_wo, tm_wg, tm_wu, tm_wd;
  CUtensorMap tm_img, tm_out;
  CUtensorMap tm_out64;  // out_w with a box of 64 rows: the guided output projection's half-width tiles
  // profiling
  bool prof = false;
  unsigned prof_mask = 0xFFFFFFFFu;  // classes timed while prof is on
  std::vector<cudaEvent_t> events;
  size_t next_event = 0;
  std::vector<ProfRec> recs;
};

namespace {

// Weight descriptors of `count` stacked blocks ([count, 3D, D] q|k|v, [count, D, D] out,
// [count, F, D] gate and up, [count, D, F] down), 64 x 128 boxes.
bool build_block_maps(int D, int F, int count, const void* wqkv_v, const void* wo_v, const void* wg_v,
                      const void* wu_v, const void* wd_v, std::vector<CUtensorMap>* tqkv, std::vector<CUtensorMap>* two,
                      std::vector<CUtensorMap>* twg, std::vector<CUtensorMap>* twu, std::vector<CUtensorMap>* twd,
                      std::string* e) {
  tqkv->resize(count);
  two->resize(count);
  twg->resize(count);
  twu->resize(count);
  twd->resize(count);
  const bf16* wqkv = static_cast<const bf16*>(wqkv_v);
  const bf16* wo = static_cast<const bf16*>(wo_v);
  const bf16* wg = static_cast<const bf16*>(wg_v);
  const bf16* wu = static_cast<const bf16*>(wu_v);
  const bf16* wd = static_cast<const bf16*>(wd_v);
  for (int l = 0; l < count; ++l) {
    const int64_t dd = static_cast<int64_t>(D) * D, df = static_cast<int64_t>(D) * F;
    if (!make_tmap_bf16_2d(&(*tqkv)[l], wqkv + l * 3 * dd, D, 3 * D, kGemmBoxK, kGemmBoxRows, e) ||
        !make_tmap_bf16_2d(&(*two)[l], wo + l * dd, D, D, kGemmBoxK, kGemmBoxRows, e) ||
        !make_tmap_bf16_2d(&(*twg)[l], wg + l * df, D, F, kGemmBoxK, kGemmBoxRows, e) ||
        !make_tmap_bf16_2d(&(*twu)[l], wu + l * df, D, F, kGemmBoxK, kGemmBoxRows, e) ||
        !make_tmap_bf16_2d(&(*twd)[l], wd + l * df, F, D, kGemmBoxK, kGemmBoxRows, e))
      return false;
  }
  return true;
}

int prof_begin(moss_model* m, int cls, cudaStream_t s) {
  ++g_launches;
  if (!m || !m->prof || !((m->prof_mask >> cls) & 1u)) return -1;
  if (m->next_event >= m->events.size()) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return -1;
    m->events.push_back(e);
  }
  const int i = static_cast<int>(m->next_event++);
  cudaEventRecord(m->events[i], s);
  return i;
}

void prof_end(moss_model* m, int cls, int i0, cudaStream_t s) {
  if (!m || !m->prof || i0 < 0) return;
  if (m->next_event >= m->events.size()) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return;
    m->events.push_back(e);
  }
  const int i1 = static_cast<int>(m->next_event++);
  cudaEventRecord(m->events[i1], s);
  m->recs.push_back({cls, i0, i1});
}

#define LAUNCH(m, cls, s, call, what)            \
  do {                                           \
    const int ev_ = prof_begin((m), (cls), (s)); \
    cudaError_t e_ = (call);                     \
    prof_end((m), (cls), ev_, (s));              \
    if (e_ != cudaSuccess) return cuda_fail(e_, what); \
  } while (0)

int check_config(const moss_config* c) {
  if (!c) return fail(MOSS_ERR_INVALID_ARGUMENT, "config is NULL");
  if (c->struct_size != sizeof(moss_config))
    return fail(MOSS_ERR_ABI_MISMATCH, "moss_config.struct_size is not sizeof(moss_config) of this library");
  if (c->head_dim != 128) return fail(MOSS_ERR_UNSUPPORTED, "only head_dim 128 is implemented");
  if (c->layers < 1 || c->heads < 1 || c->hidden != c->heads * c->head_dim)
    return fail(MOSS_ERR_INVALID_ARGUMENT, "layers >= 1, heads >= 1 and hidden == heads * head_dim are required");
  if (!ln_mod_supported(c->hidden))
    return fail(MOSS_ERR_UNSUPPORTED, "hidden must be 128 times one of 1,2,4,8,16,24,32,48,64");
  if (c->ffn < 64 || c->ffn % 64)
    return fail(MOSS_ERR_INVALID_ARGUMENT, "ffn must be a positive multiple of 64");
  if (c->cond_dim < 32 || c->cond_dim > 256 || c->cond_dim % 32)
    return fail(MOSS_ERR_INVALID_ARGUMENT, "cond_dim must be a multiple of 32 in [32, 256]");
  if (c->max_tokens < 1 || c->max_batch < 1 || c->max_latent_hw < 4 || c->max_steps < 1)
    return fail(MOSS_ERR_INVALID_ARGUMENT, "workspace capacities must be positive");
  if (c->max_steps * c->cond_dim * 4 > 200 * 1024)
    return fail(MOSS_ERR_INVALID_ARGUMENT, "max_steps * cond_dim is too large for the modulation kernel");
  return MOSS_OK;
}

int check_size(int height, int width) {
  if (height <= 0 || width <= 0 || height % 16 || width % 16)
    return fail(MOSS_ERR_INVALID_ARGUMENT, "Height and width must be positive multiples of 16.");
  if (height > 4096 || width > 4096) return fail(MOSS_ERR_INVALID_ARGUMENT, "Height and width must be at most 4096.");
  if (static_cast<int64_t>(height) * width > 4200000)
    return fail(MOSS_ERR_INVALID_ARGUMENT, "Height times width must be at most 4.2 megapixels.");
  return MOSS_OK;
}

int check_tokens(moss_model* m, int batch, int grid_h, int grid_w, int n_txt) {
  if (grid_h < 1 || grid_w < 1 || n_txt < 0) return fail(MOSS_ERR_INVALID_ARGUMENT, "grid and text sizes must be positive");
  if (batch < 1 || batch > m->cfg.max_batch)
    return fail(MOSS_ERR_INVALID_ARGUMENT, "batch must be in 1..max_batch of the model");
  const int64_t n = static_cast<int64_t>(grid_h) * grid_w + n_txt;
  if (n > m->cfg.max_tokens) return fail(MOSS_ERR_INVALID_ARGUMENT, "image + text tokens exceed max_tokens of the model");
  if (static_cast<int64_t>(grid_h) * grid_w * 4 > m->cfg.max_latent_hw)
    return fail(MOSS_ERR_INVALID_ARGUMENT, "latent exceeds max_latent_hw of the model");
  return MOSS_OK;
}

int ensure_rope(moss_model* m, int gh, int gw, int nt, cudaStream_t s) {
  if (m->rope_gh == gh && m->rope_gw == gw && m->rope_nt == nt) return MOSS_OK;
  LAUNCH(m, MOSS_K_OTHER, s, launch_rope_table(m->rope, gh, gw, nt, s), "rope table");
  m->rope_gh = gh;
  m->rope_gw = gw;
  m->rope_nt = nt;
  m->rope_n = gh * gw + nt;
  return MOSS_OK;
}

// Modulation vectors of all layers and the final layer for T timesteps into m->mod.
int compute_modulation(moss_model* m, const float* ts_host, int T, cudaStream_t s) {
  const moss_config& c = m->cfg;
  const int D = c.hidden, L = c.layers, C = c.cond_dim;
  m->mod_sched_steps = 0;  // the callers that hold a whole schedule record it afterwards
  MOSS_CUDA(cudaMemcpyAsync(m->tvals, ts_host, sizeof(float) * T, cudaMemcpyHostToDevice, s), "copy timesteps");
  LAUNCH(m, MOSS_K_OTHER, s,
         launch_conditioning(static_cast<const bf16*>(m->w.t_w1), static_cast<const bf16*>(m->w.t_b1),
                             static_cast<const bf16*>(m->w.t_w2), static_cast<const bf16*>(m->w.t_b2), m->tvals, m->sc,
                             T, C, s),
         "conditioning");
  LAUNCH(m, MOSS_K_OTHER, s,
         launch_mod_gemv(static_cast<const bf16*>(m->w.mod_w), static_cast<const bf16*>(m->w.mod_b), m->sc, m->mod,
                         L * 6 * D, C, T, m->mod_stride, s),
         "block modulation");
  LAUNCH(m, MOSS_K_OTHER, s,
         launch_mod_gemv(static_cast<const bf16*>(m->w.final_mod_w), static_cast<const bf16*>(m->w.final_mod_b),
                         m->sc, m->mod + static_cast<int64_t>(L) * 6 * D, 2 * D, C, T, m->mod_stride, s),
         "final modulation");
  return MOSS_OK;
}

// Modulation of every step of the (steps, shift) schedule sig in m->mod, computed unless m->mod
// already holds exactly that schedule.  Requires steps <= max_steps.
int ensure_schedule_modulation(moss_model* m, const std::vector<float>& sig, int steps, double shift,
                               cudaStream_t s) {
  if (m->mod_sched_steps == steps && m->mod_sched_shift == shift) return MOSS_OK;
  const int rc = compute_modulation(m, sig.data(), steps, s);
  if (rc) return rc;
  m->mod_sched_steps = steps;
  m->mod_sched_shift = shift;
  return MOSS_OK;
}

// One joint block over consecutive branches of the packed stream x (branch i has lens[i]
// rows, [image; text]); mod_l = [6D] of this layer.  Branches of different lengths are
// supported for two branches (the QKV epilogue maps rows past the first branch onto the
// second branch's tokens; attention runs per branch).
// Tensor maps and Q/K gains of one block's weights (a DiT layer or a text-only block).
struct LayerRes {
  const CUtensorMap* qkv;
  const CUtensorMap* wo;
  const CUtensorMap* wg;
  const CUtensorMap* wu;
  const CUtensorMap* wd;
  const float* q_gain;
  const float* k_gain;
};

// M-tiles per band of the pair GEMMs' tile order and L2 eviction hints of their A and B loads (0
// none, 1 evict first, 2 evict last), per GEMM of the block, chosen by DRAM bytes per launch at the
// 1024^2 shape (M = 9216, 36 pair tiles along M), all with equal launch times.  Down (K = 8192)
// visits all N-tiles of one M-tile before the next, streams its activations (evict first) and keeps
// its 50 MB of weights (evict last): 567 MB read against 751 MB with bands of 16 and no hints.
// O-proj: bands of 8, weights kept (190 against 218 MB).  QKV and gate/up read least with bands of
// 16 and no hints (hints or whole-M bands raised QKV from 237 to 343-436 MB and gate/up from 362 to
// 433-680 MB).
constexpr int kBandQkv = 16, kBandOproj = 8, kBandGateUp = 16, kBandDown = 1;
constexpr int kL2Qkv[2] = {0, 0}, kL2Oproj[2] = {0, 2}, kL2GateUp[2] = {0, 0}, kL2Down[2] = {1, 2};

int block_impl_w(moss_model* m, const LayerRes& lw, float* x, const std::vector<int>& lens, const float* mod_l,
                 cudaStream_t s) {
  const moss_config& c = m->cfg;
  const int D = c.hidden, F = c.ffn, H = c.heads;
  const int nb = static_cast<int>(lens.size());
  bool equal = true;
  int M = 0;
  for (int n : lens) {
    M += n;
    equal = equal && n == lens[0];
  }
  std::string e;
  CUtensorMap tm_h, tm_attn, tm_act;
  if (!make_tmap_bf16_2d(&tm_h, m->h, D, M, kGemmBoxK, kGemmBoxRows, &e) || !make_tmap_bf16_2d(&tm_attn, m->attn, D, M, kGemmBoxK, kGemmBoxRows, &e) ||
      !make_tmap_bf16_2d(&tm_act, m->act, F, M, kGemmBoxK, kGemmBoxRows, &e))
    return fail(MOSS_ERR_CUDA, e);

  LAUNCH(m, MOSS_K_LN_MOD, s, launch_ln_mod(x, mod_l, mod_l + D, m->h, M, D, 0, 0, 1e-6f, s), "ln_modulate 1");

  EpiParams q;
  q.M = M; q.N = 3 * D; q.K = D;
  q.out_bf16 = m->qkv;
  q.q_gain = lw.q_gain;
  q.k_gain = lw.k_gain;
  q.rope = m->rope; q.n_tok = lens[0]; q.hidden = D;
  // Branches of unequal lengths: every branch but the last has lens[0] tokens (the callers
  // order them so), the last one starts at split_rows.
  q.split_rows = equal ? 0 : static_cast<int>(M - lens[nb - 1]);
  q.rope_stride = m->rope_n;
  q.group_m = kBandQkv;
  q.a_l2 = kL2Qkv[0];
  q.b_l2 = kL2Qkv[1];
  LAUNCH(m, MOSS_K_GEMM_QKV, s, launch_gemm(kEpiQkv, tm_h, *lw.qkv, *lw.qkv, q, s, m->err), "qkv gemm");

  if (equal) {
    LAUNCH(m, MOSS_K_ATTENTION, s, launch_attention(m->qkv, m->attn, nb, lens[0], H, D, s, m->err, &e),
           e.empty() ? "attention" : e.c_str());
  } else {
    int64_t off = 0;
    for (int i = 0; i < nb; ++i) {
      LAUNCH(m, MOSS_K_ATTENTION, s,
             launch_attention(m->qkv + off * 3 * D, m->attn + off * D, 1, lens[i], H, D, s, m->err, &e),
             e.empty() ? "attention" : e.c_str());
      off += lens[i];
    }
  }

  EpiParams o;
  o.M = M; o.N = D; o.K = D;
  o.out_f32 = x; o.gate = mod_l + 2 * D;
  o.group_m = kBandOproj;
  o.a_l2 = kL2Oproj[0];
  o.b_l2 = kL2Oproj[1];
  LAUNCH(m, MOSS_K_GEMM_OPROJ, s, launch_gemm(kEpiResid, tm_attn, *lw.wo, *lw.wo, o, s, m->err),
         "out-projection gemm");

  LAUNCH(m, MOSS_K_LN_MOD, s, launch_ln_mod(x, mod_l + 3 * D, mod_l + 4 * D, m->h, M, D, 0, 0, 1e-6f, s),
         "ln_modulate 2");

  EpiParams g;
  g.M = M; g.N = F; g.K = D;
  g.out_bf16 = m->act;
  g.group_m = kBandGateUp;
  g.a_l2 = kL2GateUp[0];
  g.b_l2 = kL2GateUp[1];
  LAUNCH(m, MOSS_K_GEMM_GATEUP, s, launch_gemm(kEpiSwiglu, tm_h, *lw.wg, *lw.wu, g, s, m->err),
         "gate/up gemm");

  EpiParams d;
  d.M = M; d.N = D; d.K = F;
  d.out_f32 = x; d.gate = mod_l + 5 * D;
  d.group_m = kBandDown;
  d.a_l2 = kL2Down[0];
  d.b_l2 = kL2Down[1];
  LAUNCH(m, MOSS_K_GEMM_DOWN, s, launch_gemm(kEpiResid, tm_act, *lw.wd, *lw.wd, d, s, m->err),
         "down gemm");
  return MOSS_OK;
}

int block_impl(moss_model* m, int l, float* x, const std::vector<int>& lens, const float* mod_l, cudaStream_t s) {
  const LayerRes lw{&m->tm_qkv[l], &m->tm_wo[l], &m->tm_wg[l], &m->tm_wu[l], &m->tm_wd[l],
                    m->w.q_gain + static_cast<int64_t>(l) * 128, m->w.k_gain + static_cast<int64_t>(l) * 128};
  return block_impl_w(m, lw, x, lens, mod_l, s);
}

// The DiT for `batch` branches sharing `latent`, branch b with n_txts[b] text tokens (equal
// lengths for any batch, or two branches of different lengths); the branches' rows are packed
// back to back in the residual stream.  skip[b][l] != 0: branch b skips layer l.
// Row layout of one call: branch b has lens[b] = n_img + n_txt[b] rows starting at off[b].
struct CallRows {
  int batch = 0, n_img = 0, gh = 0, gw = 0, h8 = 0, w8 = 0;
  std::vector<int> lens;
  std::vector<int64_t> off;
};

// Patch embedding of the latent into every branch's image rows and the text states into its
// text rows of the residual stream m->x.
int embed_impl(moss_model* m, int batch, const float* latent, const float* const* texts, const int* n_txts,
               int height, int width, CallRows* rows, cudaStream_t s) {
  const int D = m->cfg.hidden;
  CallRows& r = *rows;
  r.batch = batch;
  r.h8 = height / 8; r.w8 = width / 8; r.gh = height / 16; r.gw = width / 16;
  r.n_img = r.gh * r.gw;
  r.lens.assign(batch, 0);
  r.off.assign(batch + 1, 0);
  int n_txt_max = 0;
  for (int b = 0; b < batch; ++b) {
    r.lens[b] = r.n_img + n_txts[b];
    r.off[b + 1] = r.off[b] + r.lens[b];
    n_txt_max = std::max(n_txt_max, n_txts[b]);
  }
  for (int b = 1; b + 1 < batch; ++b)
    if (n_txts[b] != n_txts[0])
      return fail(MOSS_ERR_UNSUPPORTED, "only the last branch may have a text length different from the first's");
  int rc = ensure_rope(m, r.gh, r.gw, n_txt_max, s);
  if (rc) return rc;

  LAUNCH(m, MOSS_K_OTHER, s, launch_patchify(latent, m->patches, r.h8, r.w8, s), "patchify");
  std::string e;
  CUtensorMap tm_p;
  if (!make_tmap_bf16_2d(&tm_p, m->patches, 128, r.n_img, kGemmBoxK, kGemmBoxRows, &e)) return fail(MOSS_ERR_CUDA, e);
  EpiParams pe;
  pe.M = r.n_img; pe.N = D; pe.K = 128;
  pe.out_f32 = m->x; pe.bias = static_cast<const bf16*>(m->w.img_b);
  pe.n_tok = r.lens[0]; pe.n_branch = batch;  // branch b's rows start at b * lens[0] (batch <= 2 if ragged)
  LAUNCH(m, MOSS_K_OTHER, s, launch_gemm(kEpiEmbed, tm_p, m->tm_img, m->tm_img, pe, s, m->err), "patch embed");
  for (int b = 0; b < batch; ++b) {
    if (n_txts[b] == 0) continue;
    MOSS_CUDA(cudaMemcpyAsync(m->x + (r.off[b] + r.n_img) * D, texts[b],
                              sizeof(float) * static_cast<size_t>(n_txts[b]) * D, cudaMemcpyDeviceToDevice, s),
              "copy text states");
  }
  return MOSS_OK;
}

// Blocks l0 .. l1-1 on the residual stream; consecutive branches that run a layer share a call.
int blocks_impl(moss_model* m, int l0, int l1, const CallRows& r, const float* mod,
                const std::vector<std::vector<char>>& skip, cudaStream_t s) {
  const int D = m->cfg.hidden;
  for (int l = l0; l < l1; ++l) {
    int b = 0;
    while (b < r.batch) {
      if (skip[b][l]) {
        ++b;
        continue;
      }
      int e2 = b;
      while (e2 < r.batch && !skip[e2][l]) ++e2;
      const std::vector<int> run(r.lens.begin() + b, r.lens.begin() + e2);
      int rc = block_impl(m, l, m->x + r.off[b] * D, run, mod + static_cast<int64_t>(l) * 6 * D, s);
      if (rc) return rc;
      b = e2;
    }
  }
  return MOSS_OK;
}

// Final LayerNorm-modulation of the image rows and the output projection into v_out.
int final_impl(moss_model* m, const CallRows& r, const float* mod, float* v_out, cudaStream_t s) {
  const int D = m->cfg.hidden, L = m->cfg.layers;
  const float* fmod = mod + static_cast<int64_t>(L) * 6 * D;
  const int rows = r.batch * r.n_img;
  // Image rows of branch b start at b * lens[0] (every branch but the last has lens[0] rows).
  LAUNCH(m, MOSS_K_LN_MOD, s, launch_ln_mod(m->x, fmod, fmod + D, m->h, rows, D, r.n_img, r.lens[0], 1e-6f, s),
         "final ln");
  std::string e;
  CUtensorMap tm_hf;
  if (!make_tmap_bf16_2d(&tm_hf, m->h, D, rows, kGemmBoxK, kGemmBoxRows, &e)) return fail(MOSS_ERR_CUDA, e);
  EpiParams oe;
  oe.M = rows; oe.N = 128; oe.K = D;
  oe.out_f32 = v_out; oe.bias = static_cast<const bf16*>(m->w.out_b);
  oe.n_img = r.n_img; oe.grid_w = r.gw; oe.lat_h8 = r.h8; oe.lat_w8 = r.w8;
  LAUNCH(m, MOSS_K_OTHER, s, launch_gemm(kEpiOut, tm_hf, m->tm_out, m->tm_out, oe, s, m->err), "output projection");
  return MOSS_OK;
}

// Final layer of a guided two-branch step fused with its update: LN-modulate of both branches'
// image rows, then one kernel that projects the conditional and the unconditional rows of each
// token tile (per CTA: 128 tokens, 64 of the 128 patch features) and applies
// x += (sigma_next - sigma) (v_u + cfg (v_c - v_u)) to the latent in FP32.
int final_cfg_impl(moss_model* m, const CallRows& r, const float* mod, float* x, float cfg, float sigma,
                   float sigma_next, cudaStream_t s) {
  const int D = m->cfg.hidden, L = m->cfg.layers;
  const float* fmod = mod + static_cast<int64_t>(L) * 6 * D;
  const int rows = 2 * r.n_img;
  LAUNCH(m, MOSS_K_LN_MOD, s, launch_ln_mod(m->x, fmod, fmod + D, m->h, rows, D, r.n_img, r.lens[0], 1e-6f, s),
         "final ln");
  std::string e;
  CUtensorMap tm_hf;
  if (!make_tmap_bf16_2d(&tm_hf, m->h, D, rows, kGemmBoxK, kGemmBoxRows, &e)) return fail(MOSS_ERR_CUDA, e);
  EpiParams oe;
  oe.M = rows; oe.N = 128; oe.K = D;
  oe.bias = static_cast<const bf16*>(m->w.out_b);
  oe.n_img = r.n_img; oe.grid_w = r.gw; oe.lat_h8 = r.h8; oe.lat_w8 = r.w8;
  oe.x_lat = x; oe.cfg = cfg; oe.dt = sigma_next - sigma;
  LAUNCH(m, MOSS_K_OTHER, s, launch_gemm(kEpiOutCfg, tm_hf, m->tm_out64, m->tm_out64, oe, s, m->err),
         "output projection with cfg euler");
  return MOSS_OK;
}

int forward_impl(moss_model* m, int batch, const float* latent, const float* const* texts, const int* n_txts,
                 int height, int width, const float* mod, const std::vector<std::vector<char>>& skip, float* v_out,
                 cudaStream_t s) {
  CallRows r;
  int rc = embed_impl(m, batch, latent, texts, n_txts, height, width, &r, s);
  if (!rc) rc = blocks_impl(m, 0, m->cfg.layers, r, mod, skip, s);
  if (!rc) rc = final_impl(m, r, mod, v_out, s);
  return rc;
}

int parse_skips(moss_model* m, int batch, const int* skip_layers, int n_skip, std::vector<std::vector<char>>* out) {
  const int L = m->cfg.layers;
  out->assign(batch, std::vector<char>(L, 0));
  if (n_skip < 0) return fail(MOSS_ERR_INVALID_ARGUMENT, "n_skip must be >= 0");
  if (n_skip > 0 && !skip_layers) return fail(MOSS_ERR_INVALID_ARGUMENT, "skip_layers is NULL but n_skip > 0");
  for (int b = 0; b < batch; ++b)
    for (int i = 0; i < n_skip; ++i) {
      const int l = skip_layers[b * n_skip + i];
      if (l == -1) continue;
      if (l < 0 || l >= L) return fail(MOSS_ERR_INVALID_ARGUMENT, "skip layer id out of range 0..layers-1");
      (*out)[b][l] = 1;
    }
  return MOSS_OK;
}

int step_impl(moss_model* m, float* x, const float* text_c, int n_txt_c, const float* text_u, int n_txt_u,
              int height, int width, float sigma, float sigma_next, float cfg, const std::vector<char>& uskip,
              const float* mod, cudaStream_t s) {
  const int batch = cfg == 1.0f ? 1 : 2;
  std::vector<std::vector<char>> skips(batch, std::vector<char>(m->cfg.layers, 0));
  if (batch == 2) skips[1] = uskip;
  const float* texts[2] = {text_c, text_u};
  const int n_txts[2] = {n_txt_c, n_txt_u};
  if (batch == 2) {  // the guided step: the update is part of the output projection
    CallRows r;
    int rc = embed_impl(m, batch, x, texts, n_txts, height, width, &r, s);
    if (!rc) rc = blocks_impl(m, 0, m->cfg.layers, r, mod, skips, s);
    if (!rc) rc = final_cfg_impl(m, r, mod, x, cfg, sigma, sigma_next, s);
    return rc;
  }
  int rc = forward_impl(m, batch, x, texts, n_txts, height, width, mod, skips, m->v, s);
  if (rc) return rc;
  const int64_t n = static_cast<int64_t>(height / 8) * (width / 8) * 32;
  const float* vu = batch == 2 ? m->v + n : m->v;
  LAUNCH(m, MOSS_K_CFG_EULER, s, launch_cfg_euler(x, m->v, vu, n, batch == 2 ? cfg : 1.0f, sigma, sigma_next, s),
         "cfg euler");
  return MOSS_OK;
}

// State of the first-block step cache across the steps of one sampling call.
struct StepCache {
  bool have_ref = false;  // a full call has stored its block-0 output and residual
  int batch = 0;          // its number of branches
  int64_t n = 0;          // and its residual-stream elements
};

int ensure_cache_buffers(moss_model* m) {
  if (m->cache_ref) return MOSS_OK;
  const size_t bytes = sizeof(float) * static_cast<size_t>(m->rows_cap) * m->cfg.hidden;
  const size_t pbytes = sizeof(double) * 2 * change_partial_blocks();
  if (cudaMalloc(&m->cache_ref, bytes) != cudaSuccess || cudaMalloc(&m->cache_res, bytes) != cudaSuccess ||
      cudaMalloc(&m->chg_dev, pbytes) != cudaSuccess || cudaMallocHost(&m->chg_host, pbytes) != cudaSuccess) {
    cudaGetLastError();
    if (m->cache_ref) cudaFree(m->cache_ref);
    if (m->cache_res) cudaFree(m->cache_res);
    if (m->chg_dev) cudaFree(m->chg_dev);
    if (m->chg_host) cudaFreeHost(m->chg_host);
    m->cache_ref = m->cache_res = nullptr;
    m->chg_dev = m->chg_host = nullptr;
    return fail(MOSS_ERR_OOM, "cannot allocate the step-cache buffers");
  }
  return MOSS_OK;
}

// One step of the sampling loop with the lossy accelerators: `two` = run the unconditional
// branch (false once CFG truncation has dropped it); threshold > 0 = first-block step cache.
int accel_step_impl(moss_model* m, float* x, const float* text_c, int n_txt_c, const float* text_u, int n_txt_u,
                    int height, int width, float sigma, float sigma_next, float cfg, bool two, float slg_scale,
                    const std::vector<char>& uskip, const float* mod, double threshold, StepCache* sc, int* cached,
                    float* change, cudaStream_t s) {
  // Branches: conditional, then (three-pass SLG) the conditional with the skip layers left
  // out, then the unconditional; every branch but the last has the prompt's length.
  const bool three = two && slg_scale > 0.0f;
  const int batch = three ? 3 : (two ? 2 : 1);
  const int D = m->cfg.hidden, L = m->cfg.layers;
  std::vector<std::vector<char>> skips(batch, std::vector<char>(L, 0));
  const float* texts[3] = {text_c, text_u, text_u};
  int n_txts[3] = {n_txt_c, n_txt_u, n_txt_u};
  if (two) skips[batch - 1] = uskip;
  if (three) {
    skips[1] = uskip;
    texts[1] = text_c;
    n_txts[1] = n_txt_c;
  }
  CallRows r;
  int rc = embed_impl(m, batch, x, texts, n_txts, height, width, &r, s);
  if (!rc) rc = blocks_impl(m, 0, 1, r, mod, skips, s);
  if (rc) return rc;
  const int64_t n = r.off[batch] * D;
  bool reuse = false;
  double ch = std::numeric_limits<double>::quiet_NaN();
  if (threshold > 0.0 && sc->have_ref && sc->batch == batch && sc->n == n) {
    LAUNCH(m, MOSS_K_OTHER, s, launch_change_partials(m->x, m->cache_ref, n, m->chg_dev, s), "step-cache change");
    const int nb = change_partial_blocks();
    MOSS_CUDA(cudaMemcpyAsync(m->chg_host, m->chg_dev, sizeof(double) * 2 * nb, cudaMemcpyDeviceToHost, s),
              "read step-cache change");
    MOSS_CUDA(cudaStreamSynchronize(s), "wait for step-cache change");
    double num = 0.0, den = 0.0;
    for (int i = 0; i < nb; ++i) {
      num += m->chg_host[2 * i];
      den += m->chg_host[2 * i + 1];
    }
    ch = den > 0.0 ? num / den : (num == 0.0 ? 0.0 : std::numeric_limits<double>::infinity());
    reuse = ch < threshold;
  }
  if (reuse) {
    LAUNCH(m, MOSS_K_OTHER, s, launch_add_inplace(m->x, m->cache_res, n, s), "step-cache reuse");
  } else {
    if (threshold > 0.0)
      MOSS_CUDA(cudaMemcpyAsync(m->cache_ref, m->x, sizeof(float) * n, cudaMemcpyDeviceToDevice, s),
                "store block-0 output");
    rc = blocks_impl(m, 1, L, r, mod, skips, s);
    if (rc) return rc;
    if (threshold > 0.0) {
      LAUNCH(m, MOSS_K_OTHER, s, launch_sub(m->cache_res, m->x, m->cache_ref, n, s), "store block residual");
      sc->have_ref = true;
      sc->batch = batch;
      sc->n = n;
    }
  }
  rc = final_impl(m, r, mod, m->v, s);
  if (rc) return rc;
  const int64_t nl = static_cast<int64_t>(height / 8) * (width / 8) * 32;
  if (three) {
    LAUNCH(m, MOSS_K_CFG_EULER, s,
           launch_cfg_slg_euler(x, m->v, m->v + nl, m->v + 2 * nl, nl, cfg, slg_scale, sigma, sigma_next, s),
           "cfg slg euler");
  } else {
    const float* vu = two ? m->v + nl : m->v;
    LAUNCH(m, MOSS_K_CFG_EULER, s, launch_cfg_euler(x, m->v, vu, nl, two ? cfg : 1.0f, sigma, sigma_next, s),
           "cfg euler");
  }
  *cached = reuse ? 1 : 0;
  *change = static_cast<float>(ch);
  return MOSS_OK;
}

void host_schedule(int steps, double shift, std::vector<float>* sig) {
  sig->resize(steps + 1);
  for (int i = 0; i <= steps; ++i) {
    const double sv = 1.0 - static_cast<double>(i) / steps;
    (*sig)[i] = static_cast<float>(shift * sv / (1.0 + (shift - 1.0) * sv));
  }
}

bool slg_on(int step, int steps, double a, double b) {
  const double p = static_cast<double>(step) / steps;
  return a <= p && p <= b;
}

}  // namespace

// ============================================================================== the C ABI
extern "C" {

int moss_abi_version(void) { return MOSS_ABI_VERSION; }

const char* moss_last_error(void) { return g_last_error.c_str(); }

int moss_validate(int height, int width) {
  g_last_error.clear();
  return check_size(height, width);
}

void moss_config_init(moss_config* c, uint32_t struct_size) {
  if (!c || struct_size < sizeof(uint32_t)) return;
  moss_config d;
  std::memset(&d, 0, sizeof d);
  d.struct_size = sizeof(moss_config);
  d.layers = 42;
  d.hidden = 3072;
  d.heads = 24;
  d.head_dim = 128;
  d.ffn = 8192;
  d.cond_dim = 256;
  d.max_tokens = 4096 + 512;
  d.max_batch = 2;
  d.max_latent_hw = 128 * 128;
  d.max_steps = 50;
  std::memcpy(c, &d, std::min<size_t>(struct_size, sizeof d));
  c->struct_size = struct_size;
}

void moss_weights_init(moss_weights* w, uint32_t struct_size) {
  if (!w || struct_size < sizeof(uint32_t)) return;
  std::memset(w, 0, std::min<size_t>(struct_size, sizeof(moss_weights)));
  w->struct_size = struct_size;
}

int moss_model_create(const moss_config* cfg, const moss_weights* w, moss_model** out) {
  g_last_error.clear();
  if (!out) return fail(MOSS_ERR_INVALID_ARGUMENT, "out is NULL");
  *out = nullptr;
  int rc = check_config(cfg);
  if (rc) return rc;
  if (!w) return fail(MOSS_ERR_INVALID_ARGUMENT, "weights is NULL");
  if (w->struct_size != sizeof(moss_weights))
    return fail(MOSS_ERR_ABI_MISMATCH, "moss_weights.struct_size is not sizeof(moss_weights) of this library");
  const void* ptrs[] = {w->t_w1, w->t_b1, w->t_w2, w->t_b2, w->img_w, w->img_b, w->mod_w, w->mod_b, w->wqkv,
                        w->q_gain, w->k_gain, w->wo, w->wg, w->wu, w->wd, w->final_mod_w, w->final_mod_b,
                        w->out_w, w->out_b};
  for (const void* p : ptrs) {
    if (!p) return fail(MOSS_ERR_INVALID_ARGUMENT, "a weight pointer is NULL");
    if (!aligned16(p)) return fail(MOSS_ERR_INVALID_ARGUMENT, "a weight pointer is not 16-byte aligned");
  }

  moss_model* m = new moss_model();
  m->cfg = *cfg;
  m->w = *w;
  cudaGetDevice(&m->device);
  const int D = cfg->hidden, F = cfg->ffn, L = cfg->layers, C = cfg->cond_dim;
  m->rows_cap = static_cast<int64_t>(cfg->max_batch) * cfg->max_tokens;
  m->img_cap = cfg->max_latent_hw / 4;
  m->mod_stride = static_cast<int64_t>(L) * 6 * D + 2 * D;
  m->err = device_error_word();
  auto cleanup = [&](int code, const std::string& msg) {
    moss_model_free(m);
    return fail(code, msg);
  };
  if (!m->err) return cleanup(MOSS_ERR_CUDA, "could not allocate the device error word");

  struct Alloc {
    void** p;
    size_t bytes;
  } allocs[] = {
      {reinterpret_cast<void**>(&m->x), sizeof(float) * m->rows_cap * D},
      {reinterpret_cast<void**>(&m->h), sizeof(bf16) * m->rows_cap * D},
      {reinterpret_cast<void**>(&m->qkv), sizeof(bf16) * m->rows_cap * 3 * D},
      {reinterpret_cast<void**>(&m->attn), sizeof(bf16) * m->rows_cap * D},
      {reinterpret_cast<void**>(&m->act), sizeof(bf16) * m->rows_cap * F},
      {reinterpret_cast<void**>(&m->patches), sizeof(bf16) * m->img_cap * 128},
      {reinterpret_cast<void**>(&m->v), sizeof(float) * cfg->max_batch * static_cast<int64_t>(cfg->max_latent_hw) * 32},
      {reinterpret_cast<void**>(&m->rope), sizeof(float2) * static_cast<int64_t>(cfg->max_tokens) * 64},
      {reinterpret_cast<void**>(&m->mod), sizeof(float) * cfg->max_steps * m->mod_stride},
      {reinterpret_cast<void**>(&m->sc), sizeof(float) * cfg->max_steps * C},
      {reinterpret_cast<void**>(&m->tvals), sizeof(float) * cfg->max_steps},
  };
  for (auto& a : allocs) {
    cudaError_t e = cudaMalloc(a.p, a.bytes);
    if (e != cudaSuccess) {
      *a.p = nullptr;
      return cleanup(e == cudaErrorMemoryAllocation ? MOSS_ERR_OOM : MOSS_ERR_CUDA,
                     std::string("workspace allocation: ") + cudaGetErrorString(e));
    }
  }
  // Patch-token rows beyond the image are never written; zero them once so that TMA reads
  // of a partial last tile see finite values.
  cudaMemset(m->patches, 0, sizeof(bf16) * m->img_cap * 128);

  std::string e;
  if (!build_block_maps(D, F, L, w->wqkv, w->wo, w->wg, w->wu, w->wd, &m->tm_qkv, &m->tm_wo, &m->tm_wg, &m->tm_wu,
                        &m->tm_wd, &e))
    return cleanup(MOSS_ERR_CUDA, e);
  if (!make_tmap_bf16_2d(&m->tm_img, w->img_w, 128, D, kGemmBoxK, kGemmBoxRows, &e) ||
      !make_tmap_bf16_2d(&m->tm_out, w->out_w, D, 128, kGemmBoxK, kGemmBoxRows, &e) ||
      !make_tmap_bf16_2d(&m->tm_out64, w->out_w, D, 128, kGemmBoxK, 64, &e))
    return cleanup(MOSS_ERR_CUDA, e);
  cudaError_t ce = cudaDeviceSynchronize();
  if (ce != cudaSuccess) return cleanup(MOSS_ERR_CUDA, std::string("model creation: ") + cudaGetErrorString(ce));
  *out = m;
  return MOSS_OK;
}

void moss_model_free(moss_model* m) {
  if (!m) return;
  cudaDeviceSynchronize();
  void* bufs[] = {m->x,   m->h,  m->qkv,   m->attn,      m->act,      m->patches, m->v,       m->rope,
                  m->mod, m->sc, m->tvals, m->cache_ref, m->cache_res, m->chg_dev, m->tt_mod, m->stage_x,
                  m->stage_text};
  for (void* p : bufs)
    if (p) cudaFree(p);
  if (m->chg_host) cudaFreeHost(m->chg_host);
  for (cudaEvent_t e : m->events) cudaEventDestroy(e);
  delete m;
}

int moss_dit_block_forward(moss_model* m, int layer, float* x, int batch, int grid_h, int grid_w, int n_txt, float t,
                           void* stream) {
  g_last_error.clear();
  if (!m || !x) return fail(MOSS_ERR_INVALID_ARGUMENT, "model and x must not be NULL");
  if (!aligned16(x)) return fail(MOSS_ERR_INVALID_ARGUMENT, "x must be 16-byte aligned");
  if (layer < 0 || layer >= m->cfg.layers) return fail(MOSS_ERR_INVALID_ARGUMENT, "layer out of range");
  int rc = check_tokens(m, batch, grid_h, grid_w, n_txt);
  if (rc) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  rc = compute_modulation(m, &t, 1, s);
  if (rc) return rc;
  rc = ensure_rope(m, grid_h, grid_w, n_txt, s);
  if (rc) return rc;
  const int D = m->cfg.hidden;
  const std::vector<int> lens(batch, grid_h * grid_w + n_txt);
  return block_impl(m, layer, x, lens, m->mod + static_cast<int64_t>(layer) * 6 * D, s);
}

int moss_dit_forward(moss_model* m, int batch, const float* latent, const float* text_states, int n_txt, int height,
                     int width, float t, const int* skip_layers, int n_skip, float* v_out, void* stream) {
  g_last_error.clear();
  if (!m || !latent || !v_out || (n_txt > 0 && !text_states))
    return fail(MOSS_ERR_INVALID_ARGUMENT, "model, latent, text_states and v_out must not be NULL");
  if (!aligned16(latent) || !aligned16(v_out) || (text_states && !aligned16(text_states)))
    return fail(MOSS_ERR_INVALID_ARGUMENT, "device buffers must be 16-byte aligned");
  int rc = check_size(height, width);
  if (rc) return rc;
  rc = check_tokens(m, batch, height / 16, width / 16, n_txt);
  if (rc) return rc;
  std::vector<std::vector<char>> skips;
  rc = parse_skips(m, batch, skip_layers, n_skip, &skips);
  if (rc) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  rc = compute_modulation(m, &t, 1, s);
  if (rc) return rc;
  std::vector<const float*> texts(batch);
  for (int b = 0; b < batch; ++b) texts[b] = text_states + static_cast<int64_t>(b) * n_txt * m->cfg.hidden;
  const std::vector<int> n_txts(batch, n_txt);
  return forward_impl(m, batch, latent, texts.data(), n_txts.data(), height, width, m->mod, skips, v_out, s);
}

int moss_cfg_euler_step(float* x, const float* v_c, const float* v_u, int64_t n, float cfg, float sigma,
                        float sigma_next, void* stream) {
  g_last_error.clear();
  if (n < 0) return fail(MOSS_ERR_INVALID_ARGUMENT, "n must be >= 0");
  if (n == 0) return MOSS_OK;
  if (!x || !v_c || !v_u) return fail(MOSS_ERR_INVALID_ARGUMENT, "x, v_c and v_u must not be NULL");
  if (!aligned16(x) || !aligned16(v_c) || !aligned16(v_u))
    return fail(MOSS_ERR_INVALID_ARGUMENT, "x, v_c and v_u must be 16-byte aligned");
  ++g_launches;
  cudaError_t e = launch_cfg_euler(x, v_c, v_u, n, cfg, sigma, sigma_next, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOSS_OK : cuda_fail(e, "cfg euler");
}

int moss_sigma_schedule(int steps, double shift, float* out) {
  g_last_error.clear();
  if (steps < 1 || !(shift > 0.0) || !out) return fail(MOSS_ERR_INVALID_ARGUMENT, "steps >= 1, shift > 0, out != NULL");
  std::vector<float> sig;
  host_schedule(steps, shift, &sig);
  std::memcpy(out, sig.data(), sizeof(float) * (steps + 1));
  return MOSS_OK;
}

int moss_slg_active(int step, int steps, double slg_start, double slg_stop) {
  if (steps < 1 || step < 0 || step >= steps) return -1;
  return slg_on(step, steps, slg_start, slg_stop) ? 1 : 0;
}

int moss_init_noise(float* x, int64_t n, uint64_t seed, void* stream) {
  g_last_error.clear();
  if (n < 0) return fail(MOSS_ERR_INVALID_ARGUMENT, "n must be >= 0");
  if (n == 0) return MOSS_OK;
  if (!x || !aligned16(x)) return fail(MOSS_ERR_INVALID_ARGUMENT, "x must be a 16-byte aligned device pointer");
  ++g_launches;
  cudaError_t e = launch_noise(x, n, seed, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOSS_OK : cuda_fail(e, "noise");
}

static int check_step_args(moss_model* m, float* x, const float* text_c, int n_txt_c, const float* text_u,
                           int n_txt_u, int height, int width, float cfg, const int* uskip, int n_skip,
                           std::vector<char>* skipv) {
  if (!m || !x || (n_txt_c > 0 && !text_c) || (cfg != 1.0f && n_txt_u > 0 && !text_u))
    return fail(MOSS_ERR_INVALID_ARGUMENT, "model, x and text states must not be NULL");
  if (n_txt_c < 0 || n_txt_u < 0) return fail(MOSS_ERR_INVALID_ARGUMENT, "text lengths must be >= 0");
  if (!aligned16(x) || (text_c && !aligned16(text_c)) || (text_u && !aligned16(text_u)))
    return fail(MOSS_ERR_INVALID_ARGUMENT, "device buffers must be 16-byte aligned");
  int rc = check_size(height, width);
  if (rc) return rc;
  rc = check_tokens(m, cfg == 1.0f ? 1 : 2, height / 16, width / 16,
                    cfg == 1.0f ? n_txt_c : std::max(n_txt_c, n_txt_u));
  if (rc) return rc;
  std::vector<std::vector<char>> sk;
  rc = parse_skips(m, 1, uskip, n_skip, &sk);
  if (rc) return rc;
  *skipv = sk[0];
  return MOSS_OK;
}

// The denoising step after its arguments have been checked (uskip: the parsed skip set).
static int denoise_step_impl(moss_model* m, float* x, const float* text_c, int n_txt_c, const float* text_u,
                             int n_txt_u, int height, int width, int step, int steps, float cfg, double shift,
                             std::vector<char> uskip, double slg_start, double slg_stop, cudaStream_t s) {
  int rc = MOSS_OK;
  if (!slg_on(step, steps, slg_start, slg_stop)) std::fill(uskip.begin(), uskip.end(), 0);
  std::vector<float> sig;
  host_schedule(steps, shift, &sig);
  const float* mod = m->mod;
  if (steps <= m->cfg.max_steps) {
    rc = ensure_schedule_modulation(m, sig, steps, shift, s);
    mod = m->mod + static_cast<int64_t>(step) * m->mod_stride;
  } else {
    rc = compute_modulation(m, &sig[step], 1, s);
  }
  if (rc) return rc;
  return step_impl(m, x, text_c, n_txt_c, text_u, n_txt_u, height, width, sig[step], sig[step + 1], cfg, uskip,
                   mod, s);
}

int moss_denoise_step(moss_model* m, float* x, const float* text_c, int n_txt_c, const float* text_u, int n_txt_u,
                      int height, int width, int step, int steps, float cfg, double shift,
                      const int* uncond_skip_layers, int n_skip, double slg_start, double slg_stop, void* stream) {
  g_last_error.clear();
  if (steps < 1 || step < 0 || step >= steps || !(shift > 0.0))
    return fail(MOSS_ERR_INVALID_ARGUMENT, "need 0 <= step < steps and shift > 0");
  std::vector<char> uskip;
  const int rc = check_step_args(m, x, text_c, n_txt_c, text_u, n_txt_u, height, width, cfg, uncond_skip_layers,
                                 n_skip, &uskip);
  if (rc) return rc;
  return denoise_step_impl(m, x, text_c, n_txt_c, text_u, n_txt_u, height, width, step, steps, cfg, shift, uskip,
                           slg_start, slg_stop, static_cast<cudaStream_t>(stream));
}

int moss_denoise_step_host(moss_model* m, float* x_host, const float* text_c_host, int n_txt_c,
                           const float* text_u_host, int n_txt_u, int height, int width, int step, int steps, float cfg,
                           double shift, const int* uncond_skip_layers, int n_skip, double slg_start, double slg_stop,
                           void* stream) {
  g_last_error.clear();
  if (steps < 1 || step < 0 || step >= steps || !(shift > 0.0))
    return fail(MOSS_ERR_INVALID_ARGUMENT, "need 0 <= step < steps and shift > 0");
  if (!m) return fail(MOSS_ERR_INVALID_ARGUMENT, "model is NULL");
  if (!x_host || (n_txt_c > 0 && !text_c_host) || (cfg != 1.0f && n_txt_u > 0 && !text_u_host))
    return fail(MOSS_ERR_INVALID_ARGUMENT, "x and text states must not be NULL");
  if (n_txt_c < 0 || n_txt_u < 0) return fail(MOSS_ERR_INVALID_ARGUMENT, "text lengths must be >= 0");
  int rc = check_size(height, width);
  if (rc) return rc;
  const bool two = cfg != 1.0f;
  rc = check_tokens(m, two ? 2 : 1, height / 16, width / 16, two ? std::max(n_txt_c, n_txt_u) : n_txt_c);
  if (rc) return rc;
  std::vector<std::vector<char>> sk;
  rc = parse_skips(m, 1, uncond_skip_layers, n_skip, &sk);
  if (rc) return rc;
  const int D = m->cfg.hidden;
  if (!m->stage_x) {
    const size_t bx = sizeof(float) * static_cast<size_t>(m->cfg.max_latent_hw) * 32;
    const size_t bt = sizeof(float) * 2 * static_cast<size_t>(m->cfg.max_tokens) * D;
    if (cudaMalloc(&m->stage_x, bx) != cudaSuccess || cudaMalloc(&m->stage_text, bt) != cudaSuccess) {
      cudaGetLastError();
      if (m->stage_x) cudaFree(m->stage_x);
      m->stage_x = nullptr;
      m->stage_text = nullptr;
      return fail(MOSS_ERR_OOM, "cannot allocate the host-step staging buffers");
    }
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t nx = static_cast<size_t>(height / 8) * (width / 8) * 32;
  float* tc = m->stage_text;
  float* tu = m->stage_text + static_cast<size_t>(m->cfg.max_tokens) * D;
  MOSS_CUDA(cudaMemcpyAsync(m->stage_x, x_host, sizeof(float) * nx, cudaMemcpyHostToDevice, s), "copy latent in");
  if (n_txt_c > 0)
    MOSS_CUDA(cudaMemcpyAsync(tc, text_c_host, sizeof(float) * n_txt_c * D, cudaMemcpyHostToDevice, s),
              "copy prompt in");
  if (two && n_txt_u > 0)
    MOSS_CUDA(cudaMemcpyAsync(tu, text_u_host, sizeof(float) * n_txt_u * D, cudaMemcpyHostToDevice, s),
              "copy negative prompt in");
  rc = denoise_step_impl(m, m->stage_x, tc, n_txt_c, tu, two ? n_txt_u : 0, height, width, step, steps, cfg, shift,
                         sk[0], slg_start, slg_stop, s);
  if (rc) return rc;
  MOSS_CUDA(cudaMemcpyAsync(x_host, m->stage_x, sizeof(float) * nx, cudaMemcpyDeviceToHost, s), "copy latent out");
  MOSS_CUDA(cudaStreamSynchronize(s), "host step");
  return MOSS_OK;
}

int moss_sample(moss_model* m, int steps, float cfg, double shift, uint64_t seed, const int* uncond_skip_layers,
                int n_skip, double slg_start, double slg_stop, const float* text_c, int n_txt_c, const float* text_u,
                int n_txt_u, int height, int width, float* latent_out, void* stream) {
  g_last_error.clear();
  if (!m) return fail(MOSS_ERR_INVALID_ARGUMENT, "model is NULL");
  if (steps < 1 || steps > m->cfg.max_steps || !(shift > 0.0))
    return fail(MOSS_ERR_INVALID_ARGUMENT, "need 1 <= steps <= max_steps and shift > 0");
  std::vector<char> uskip;
  int rc = check_step_args(m, latent_out, text_c, n_txt_c, text_u, n_txt_u, height, width, cfg, uncond_skip_layers,
                           n_skip, &uskip);
  if (rc) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t n = static_cast<int64_t>(height / 8) * (width / 8) * 32;
  LAUNCH(m, MOSS_K_OTHER, s, launch_noise(latent_out, n, seed, s), "noise");
  std::vector<float> sig;
  host_schedule(steps, shift, &sig);
  rc = ensure_schedule_modulation(m, sig, steps, shift, s);
  if (rc) return rc;
  const std::vector<char> none(m->cfg.layers, 0);
  for (int i = 0; i < steps; ++i) {
    const bool on = slg_on(i, steps, slg_start, slg_stop);
    rc = step_impl(m, latent_out, text_c, n_txt_c, text_u, n_txt_u, height, width, sig[i], sig[i + 1], cfg,
                   on ? uskip : none, m->mod + static_cast<int64_t>(i) * m->mod_stride, s);
    if (rc) return rc;
  }
  return MOSS_OK;
}

void moss_text_weights_init(moss_text_weights* tw, uint32_t struct_size) {
  if (!tw || struct_size < sizeof(uint32_t)) return;
  moss_text_weights d;
  std::memset(&d, 0, sizeof d);
  d.enc_dim = 4096;
  d.blocks = 2;
  std::memcpy(tw, &d, std::min<size_t>(struct_size, sizeof d));
  tw->struct_size = struct_size;
}

int moss_text_refiner_set(moss_model* m, const moss_text_weights* tw) {
  g_last_error.clear();
  if (!m || !tw) return fail(MOSS_ERR_INVALID_ARGUMENT, "model and text weights must not be NULL");
  if (tw->struct_size != sizeof(moss_text_weights))
    return fail(MOSS_ERR_ABI_MISMATCH, "moss_text_weights.struct_size is not sizeof(moss_text_weights) of this library");
  if (tw->enc_dim <= 0 || tw->enc_dim % 64)
    return fail(MOSS_ERR_INVALID_ARGUMENT, "enc_dim must be a positive multiple of 64");
  if (tw->blocks < 0 || tw->blocks > 8) return fail(MOSS_ERR_INVALID_ARGUMENT, "blocks must lie in 0..8");
  const void* need[] = {tw->proj_w, tw->proj_b};
  const void* blk[] = {tw->wqkv, tw->q_gain, tw->k_gain, tw->wo, tw->wg, tw->wu, tw->wd};
  for (const void* p : need)
    if (!p || !aligned16(p)) return fail(MOSS_ERR_INVALID_ARGUMENT, "a text weight pointer is NULL or misaligned");
  if (tw->blocks > 0)
    for (const void* p : blk)
      if (!p || !aligned16(p)) return fail(MOSS_ERR_INVALID_ARGUMENT, "a text weight pointer is NULL or misaligned");
  const int D = m->cfg.hidden, F = m->cfg.ffn;
  std::string e;
  m->has_text = false;
  if (!make_tmap_bf16_2d(&m->tt_proj, tw->proj_w, tw->enc_dim, D, kGemmBoxK, kGemmBoxRows, &e))
    return fail(MOSS_ERR_CUDA, e);
  if (tw->blocks > 0 && !build_block_maps(D, F, tw->blocks, tw->wqkv, tw->wo, tw->wg, tw->wu, tw->wd, &m->tt_qkv,
                                          &m->tt_wo, &m->tt_wg, &m->tt_wu, &m->tt_wd, &e))
    return fail(MOSS_ERR_CUDA, e);
  if (!m->tt_mod) {
    cudaError_t ce = cudaMalloc(&m->tt_mod, sizeof(float) * 6 * D);
    if (ce != cudaSuccess) {
      m->tt_mod = nullptr;
      return fail(MOSS_ERR_OOM, std::string("text modulation vector: ") + cudaGetErrorString(ce));
    }
    std::vector<float> mod(6 * static_cast<size_t>(D), 0.f);
    std::fill(mod.begin() + 2 * D, mod.begin() + 3 * D, 1.f);
    std::fill(mod.begin() + 5 * D, mod.end(), 1.f);
    ce = cudaMemcpy(m->tt_mod, mod.data(), sizeof(float) * mod.size(), cudaMemcpyHostToDevice);
    if (ce != cudaSuccess) return fail(MOSS_ERR_CUDA, std::string("text modulation vector: ") + cudaGetErrorString(ce));
  }
  m->tw = *tw;
  m->has_text = true;
  return MOSS_OK;
}

int moss_text_refine(moss_model* m, const void* enc_states, int n_txt, float* text_out, void* stream) {
  g_last_error.clear();
  if (!m || !m->has_text) return fail(MOSS_ERR_INVALID_ARGUMENT, "no text path attached to the model");
  if (!enc_states || !text_out || !aligned16(enc_states) || !aligned16(text_out))
    return fail(MOSS_ERR_INVALID_ARGUMENT, "enc_states and text_out must be non-NULL and 16-byte aligned");
  if (n_txt < 1 || n_txt > m->cfg.max_tokens)
    return fail(MOSS_ERR_INVALID_ARGUMENT, "n_txt must lie in 1..max_tokens");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int D = m->cfg.hidden;
  std::string e;
  CUtensorMap tm_e;
  if (!make_tmap_bf16_2d(&tm_e, enc_states, m->tw.enc_dim, n_txt, kGemmBoxK, kGemmBoxRows, &e))
    return fail(MOSS_ERR_CUDA, e);
  EpiParams pe;
  pe.M = n_txt; pe.N = D; pe.K = m->tw.enc_dim;
  pe.out_f32 = text_out; pe.bias = static_cast<const bf16*>(m->tw.proj_b);
  pe.n_tok = n_txt; pe.n_branch = 1;
  LAUNCH(m, MOSS_K_OTHER, s, launch_gemm(kEpiEmbed, tm_e, m->tt_proj, m->tt_proj, pe, s, m->err), "text projection");
  if (m->tw.blocks == 0) return MOSS_OK;
  int rc = ensure_rope(m, 0, 0, n_txt, s);
  if (rc) return rc;
  const std::vector<int> lens(1, n_txt);
  for (int b = 0; b < m->tw.blocks; ++b) {
    const LayerRes lw{&m->tt_qkv[b], &m->tt_wo[b], &m->tt_wg[b], &m->tt_wu[b], &m->tt_wd[b],
                      m->tw.q_gain + static_cast<int64_t>(b) * 128, m->tw.k_gain + static_cast<int64_t>(b) * 128};
    rc = block_impl_w(m, lw, text_out, lens, m->tt_mod, s);
    if (rc) return rc;
  }
  return MOSS_OK;
}

void moss_sample_options_init(moss_sample_options* opt, uint32_t struct_size) {
  if (!opt || struct_size < sizeof(uint32_t)) return;
  moss_sample_options d;
  std::memset(&d, 0, sizeof d);
  d.cfg_truncation = 1.0;
  d.step_cache_threshold = 0.0;
  d.slg_scale = 0.0;
  std::memcpy(opt, &d, std::min<size_t>(struct_size, sizeof d));
  opt->struct_size = struct_size;
}

int moss_sample_ex(moss_model* m, int steps, float cfg, double shift, uint64_t seed, const int* uncond_skip_layers,
                   int n_skip, double slg_start, double slg_stop, const float* text_c, int n_txt_c,
                   const float* text_u, int n_txt_u, int height, int width, const moss_sample_options* opt_in,
                   float* latent_out, void* stream) {
  g_last_error.clear();
  moss_sample_options opt;
  moss_sample_options_init(&opt, sizeof opt);
  if (opt_in) {
    if (opt_in->struct_size != sizeof(moss_sample_options))
      return fail(MOSS_ERR_ABI_MISMATCH,
                  "moss_sample_options.struct_size is not sizeof(moss_sample_options) of this library");
    opt = *opt_in;
  }
  if (!(opt.cfg_truncation >= 0.0 && opt.cfg_truncation <= 1.0))
    return fail(MOSS_ERR_INVALID_ARGUMENT, "cfg_truncation must lie in [0, 1]");
  if (!(opt.step_cache_threshold >= 0.0))
    return fail(MOSS_ERR_INVALID_ARGUMENT, "step_cache_threshold must be >= 0");
  if (!(opt.slg_scale >= 0.0 && opt.slg_scale < 1e30))
    return fail(MOSS_ERR_INVALID_ARGUMENT, "slg_scale must be finite and >= 0");
  if (!m) return fail(MOSS_ERR_INVALID_ARGUMENT, "model is NULL");
  if (steps < 1 || steps > m->cfg.max_steps || !(shift > 0.0))
    return fail(MOSS_ERR_INVALID_ARGUMENT, "need 1 <= steps <= max_steps and shift > 0");
  std::vector<char> uskip;
  int rc = check_step_args(m, latent_out, text_c, n_txt_c, text_u, n_txt_u, height, width, cfg, uncond_skip_layers,
                           n_skip, &uskip);
  if (rc) return rc;
  if (opt.slg_scale > 0.0 && cfg != 1.0f) {
    rc = check_tokens(m, 3, height / 16, width / 16, std::max(n_txt_c, n_txt_u));
    if (rc) return rc;
  }
  const double thr = opt.step_cache_threshold;
  if (thr > 0.0) {
    rc = ensure_cache_buffers(m);
    if (rc) return rc;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t n = static_cast<int64_t>(height / 8) * (width / 8) * 32;
  LAUNCH(m, MOSS_K_OTHER, s, launch_noise(latent_out, n, seed, s), "noise");
  std::vector<float> sig;
  host_schedule(steps, shift, &sig);
  rc = ensure_schedule_modulation(m, sig, steps, shift, s);
  if (rc) return rc;
  const std::vector<char> none(m->cfg.layers, 0);
  StepCache sc;
  for (int i = 0; i < steps; ++i) {
    const bool on = slg_on(i, steps, slg_start, slg_stop);
    const bool two = cfg != 1.0f && !(static_cast<double>(i) >= opt.cfg_truncation * steps);
    int cached = 0;
    float change = 0.f;
    rc = accel_step_impl(m, latent_out, text_c, n_txt_c, text_u, n_txt_u, height, width, sig[i], sig[i + 1], cfg,
                         two, on ? static_cast<float>(opt.slg_scale) : 0.0f, on ? uskip : none, m->mod + static_cast<int64_t>(i) * m->mod_stride, thr, &sc,
                         &cached, &change, s);
    if (rc) return rc;
    if (opt.cached_out) opt.cached_out[i] = cached;
    if (opt.change_out) opt.change_out[i] = change;
  }
  return MOSS_OK;
}

int moss_selftest_wait_timeout(void* stream) {
  g_last_error.clear();
  unsigned* p = device_error_word();
  if (!p) return fail(MOSS_ERR_CUDA, "could not allocate the device error word");
  LAUNCH(static_cast<moss_model*>(nullptr), MOSS_K_OTHER, static_cast<cudaStream_t>(stream),
         launch_wait_probe(p, static_cast<cudaStream_t>(stream)), "wait probe");
  return MOSS_OK;
}

int moss_selftest_attention_timeout(const void* qkv, void* o, int batch, int n_tok, int heads, int step,
                                    void* stream) {
  g_last_error.clear();
  if (!qkv || !o) return fail(MOSS_ERR_INVALID_ARGUMENT, "qkv and o must not be NULL");
  if (!aligned16(qkv) || !aligned16(o)) return fail(MOSS_ERR_INVALID_ARGUMENT, "16-byte alignment required");
  if (batch < 1 || n_tok < 1 || heads < 1) return fail(MOSS_ERR_INVALID_ARGUMENT, "batch, n_tok and heads must be >= 1");
  if (step < 0 || step >= (n_tok + 127) / 128) return fail(MOSS_ERR_INVALID_ARGUMENT, "step must be a key step of the sequence");
  unsigned* err = device_error_word();
  if (!err) return fail(MOSS_ERR_CUDA, "device error word");
  std::string e;
  ++g_launches;
  cudaError_t ce = launch_attention(static_cast<const bf16*>(qkv), static_cast<bf16*>(o), batch, n_tok, heads,
                                    heads * 128, static_cast<cudaStream_t>(stream), err, &e, step);
  return ce == cudaSuccess ? MOSS_OK : cuda_fail(ce, e.empty() ? "attention" : e.c_str());
}

int moss_device_status(int clear) {
  unsigned* p = device_error_word();
  if (!p) return -MOSS_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return -MOSS_ERR_CUDA;
  unsigned v = 0;
  if (cudaMemcpy(&v, p, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return -MOSS_ERR_CUDA;
  if (clear && cudaMemset(p, 0, sizeof v) != cudaSuccess) return -MOSS_ERR_CUDA;
  return static_cast<int>(v & 0x7fffffff);
}

int moss_profile_enable(moss_model* m, int enable) {
  g_last_error.clear();
  if (!m) return fail(MOSS_ERR_INVALID_ARGUMENT, "model is NULL");
  m->prof = enable != 0;
  m->prof_mask = 0xFFFFFFFFu;
  m->next_event = 0;
  m->recs.clear();
  return MOSS_OK;
}

int moss_profile_enable_classes(moss_model* m, unsigned class_mask) {
  g_last_error.clear();
  if (!m) return fail(MOSS_ERR_INVALID_ARGUMENT, "model is NULL");
  m->prof = class_mask != 0;
  m->prof_mask = class_mask;
  m->next_event = 0;
  m->recs.clear();
  return MOSS_OK;
}

int moss_profile_read(moss_model* m, int kclass, int64_t* launches, double* total_ms) {
  g_last_error.clear();
  if (!m || !launches || !total_ms || kclass < 0 || kclass >= MOSS_K_COUNT)
    return fail(MOSS_ERR_INVALID_ARGUMENT, "bad profile query");
  MOSS_CUDA(cudaDeviceSynchronize(), "profile sync");
  int64_t n = 0;
  double ms = 0;
  for (const ProfRec& r : m->recs) {
    if (r.cls != kclass) continue;
    float t = 0;
    MOSS_CUDA(cudaEventElapsedTime(&t, m->events[r.ev0], m->events[r.ev1]), "event time");
    ++n;
    ms += t;
  }
  *launches = n;
  *total_ms = ms;
  return MOSS_OK;
}

int64_t moss_launch_count(int reset) {
  const int64_t v = g_launches.load();
  if (reset) g_launches = 0;
  return v;
}

int moss_op_gemm_bf16(const void* a, const void* b, float* c, int M, int N, int K, void* stream) {
  g_last_error.clear();
  if (!a || !b || !c) return fail(MOSS_ERR_INVALID_ARGUMENT, "a, b and c must not be NULL");
  if (!aligned16(a) || !aligned16(b) || !aligned16(c)) return fail(MOSS_ERR_INVALID_ARGUMENT, "16-byte alignment required");
  if (M < 1 || N < 32 || K < 64 || K % 64 || N % 32) return fail(MOSS_ERR_INVALID_ARGUMENT, "need M >= 1, N % 32 == 0, K % 64 == 0");
  unsigned* err = device_error_word();
  if (!err) return fail(MOSS_ERR_CUDA, "device error word");
  std::string e;
  CUtensorMap ta, tb;
  if (!make_tmap_bf16_2d(&ta, a, K, M, kGemmBoxK, kGemmBoxRows, &e) || !make_tmap_bf16_2d(&tb, b, K, N, kGemmBoxK, kGemmBoxRows, &e))
    return fail(MOSS_ERR_CUDA, e);
  EpiParams ep;
  ep.M = M; ep.N = N; ep.K = K; ep.out_f32 = c;
  ++g_launches;
  cudaError_t ce = launch_gemm(kEpiF32, ta, tb, tb, ep, static_cast<cudaStream_t>(stream), err);
  return ce == cudaSuccess ? MOSS_OK : cuda_fail(ce, "gemm");
}

int moss_op_attention(const void* qkv, void* o, int batch, int n_tok, int heads, void* stream) {
  g_last_error.clear();
  if (!qkv || !o) return fail(MOSS_ERR_INVALID_ARGUMENT, "qkv and o must not be NULL");
  if (!aligned16(qkv) || !aligned16(o)) return fail(MOSS_ERR_INVALID_ARGUMENT, "16-byte alignment required");
  if (batch < 1 || n_tok < 1 || heads < 1) return fail(MOSS_ERR_INVALID_ARGUMENT, "batch, n_tok and heads must be >= 1");
  unsigned* err = device_error_word();
  if (!err) return fail(MOSS_ERR_CUDA, "device error word");
  const int D = heads * 128;
  std::string e;
  ++g_launches;
  cudaError_t ce = launch_attention(static_cast<const bf16*>(qkv), static_cast<bf16*>(o), batch, n_tok, heads, D,
                                    static_cast<cudaStream_t>(stream), err, &e);
  return ce == cudaSuccess ? MOSS_OK : cuda_fail(ce, e.empty() ? "attention" : e.c_str());
}

int moss_op_ln_modulate(const float* x, const float* shift, const float* scale, void* h, int rows, int dim,
                        void* stream) {
  g_last_error.clear();
  if (!x || !shift || !scale || !h) return fail(MOSS_ERR_INVALID_ARGUMENT, "pointers must not be NULL");
  if (!aligned16(x) || !aligned16(shift) || !aligned16(scale) || !aligned16(h))
    return fail(MOSS_ERR_INVALID_ARGUMENT, "16-byte alignment required");
  if (rows < 0 || !ln_mod_supported(dim)) return fail(MOSS_ERR_INVALID_ARGUMENT, "unsupported rows or dim");
  ++g_launches;
  cudaError_t ce = launch_ln_mod(x, shift, scale, static_cast<bf16*>(h), rows, dim, 0, 0, 1e-6f,
                                 static_cast<cudaStream_t>(stream));
  return ce == cudaSuccess ? MOSS_OK : cuda_fail(ce, "ln_modulate");
}

int moss_op_modulation(moss_model* m, float t, float* mod, void* stream) {
  g_last_error.clear();
  if (!m || !mod) return fail(MOSS_ERR_INVALID_ARGUMENT, "model and mod must not be NULL");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int rc = compute_modulation(m, &t, 1, s);
  if (rc) return rc;
  MOSS_CUDA(cudaMemcpyAsync(mod, m->mod, sizeof(float) * m->mod_stride, cudaMemcpyDeviceToDevice, s), "copy modulation");
  return MOSS_OK;
}

}  // extern "C"
