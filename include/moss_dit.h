/*
 * moss_dit.h - C ABI of the B200 (sm_100a) MOSS-Image DiT denoising-step library.
 *
 * The library computes one denoising step of the MOSS-Image single-stream DiT: two DiT
 * passes for classifier-free guidance (conditional and unconditional branch, the latter
 * skipping the requested layers inside the skip-layer window), the FP32 CFG combine and
 * the shifted flow-matching Euler update.
 *
 * Sources, cited by page title and section:
 *   [SGL-MOSS] SGLang cookbook "OpenMOSS/MOSS-Image", 3. Guidance and precision.
 *   [MI]       MossInfer integration guide: Defaults, validation, C API rules.
 *   [INV]      InvokeAI MOSS-Image guide: Transformer formats, Generation settings, Skip layers.
 *   [WP]       windpaint.ai "MOSS-Image: specs, settings, VRAM and text rendering tested":
 *              Architecture and specs table, Recommended settings.
 *   [SGL-QWEN] SGLang cookbook "Qwen-Image 2.1", Lossless RoPE / MLP and residual /
 *              Q/K normalization / LayerNorm modulation fusions (sibling model; used for
 *              the block internals the MOSS-Image pages leave open).
 *
 * Conventions (all entry points):
 *   - Every pointer named "device" is CUDA device memory owned by the caller; the library
 *     never frees it.  Pointers named "host" are ordinary host memory.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is enqueued on it
 *     and the call returns without synchronising, unless stated otherwise.
 *   - Return value: MOSS_OK (0) or a moss_status error.  After an error,
 *     moss_last_error() returns a message for the calling thread.  Arguments are
 *     validated on the host before anything is launched; an invalid call launches nothing.
 *   - After MOSS_ERR_CUDA the model should be freed ([MI] C API rules: after a CUDA error,
 *     free the engine).
 *   - A model holds mutable state: its workspace, the modulation of the last schedule it
 *     computed, the host-step staging buffers.  Calls on one model must not overlap: use it from
 *     one thread at a time and on one stream (or order the streams); separate models are
 *     independent.
 *   - Floating-point layouts are row-major, innermost index last.
 *
 * Model tensors (D = hidden, H = heads, d = head_dim = 128, F = ffn, L = layers,
 * C = conditioning width 256, P = 2x2x32 = 128 patch features):
 *   residual stream x        FP32 [B, N, D], N = n_img + n_txt, rows [image; text]
 *   image tokens             (height/16)*(width/16), row-major over the patch grid
 *   latent                   FP32 [height/8, width/8, 32]
 *   linear weights           BF16 [out_features, in_features]
 */
#ifndef MOSS_DIT_H
#define MOSS_DIT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOSS_ABI_VERSION 1

typedef enum moss_status {
  MOSS_OK = 0,
  MOSS_ERR_INVALID_ARGUMENT = 1, /* a size, pointer or option is out of range            */
  MOSS_ERR_CUDA = 2,             /* a CUDA call failed; free the model                    */
  MOSS_ERR_OOM = 3,              /* workspace allocation failed at model creation         */
  MOSS_ERR_TIMEOUT = 4,          /* a device-side wait gave up (see moss_device_status)   */
  MOSS_ERR_ABI_MISMATCH = 5,     /* struct_size not accepted by this library              */
  MOSS_ERR_UNSUPPORTED = 6       /* shape outside what the kernels implement              */
} moss_status;

/* Library ABI version; a caller refuses to run when it differs from MOSS_ABI_VERSION
 * ([MI] C API rules: check the ABI at start-up). */
int moss_abi_version(void);

/* Message for the last non-OK status returned on the calling thread ("" if none).
 * The pointer stays valid until the next call on that thread. */
const char* moss_last_error(void);

/* Request size check, no GPU needed.  Height and width must be positive multiples of 16,
 * at most 4096 per side and at most 4.2 megapixels ([MI] Defaults and validation;
 * [SGL-MOSS] 3: divisible by 16).  Returns MOSS_OK or MOSS_ERR_INVALID_ARGUMENT with the
 * official wording "Height and width must be positive multiples of 16." for the first rule. */
int moss_validate(int height, int width);

/* ------------------------------------------------------------------------------------ */
/* Model configuration and weights.                                                     */
/* ------------------------------------------------------------------------------------ */
typedef struct moss_config {
  uint32_t struct_size;   /* sizeof(moss_config) as compiled by the caller             */
  int32_t layers;         /* 42 [WP]                                                    */
  int32_t hidden;         /* D = 3072 [WP]; multiple of 128                             */
  int32_t heads;          /* 24 [WP]; heads * head_dim == hidden                        */
  int32_t head_dim;       /* 128 [WP]; only 128 is implemented                          */
  int32_t ffn;            /* F = 8192 [WP]; multiple of 64                              */
  int32_t cond_dim;       /* C = 256, width of the timestep conditioning                */
  int32_t max_tokens;     /* workspace capacity: largest N = n_img + n_txt per branch   */
  int32_t max_batch;      /* workspace capacity: branches per call (2 for CFG)          */
  int32_t max_latent_hw;  /* workspace capacity: largest (height/8)*(width/8)           */
  int32_t max_steps;      /* workspace capacity: steps whose modulation is precomputed  */
} moss_config;

/* Fill `cfg` with the full MOSS-Image DiT (42 x 3072, 24 x 128, FFN 8192, C 256) and a
 * workspace for 1024^2 with a 512-token prompt, batch 2, 50 steps. */
void moss_config_init(moss_config* cfg, uint32_t struct_size);

/* Device pointers to the DiT parameters, stacked over layers.  All BF16 except the two
 * RMSNorm gains (FP32).  The caller owns them and keeps them alive and unchanged while the
 * model exists.  Every pointer must be 16-byte aligned. */
typedef struct moss_weights {
  uint32_t struct_size;
  const void* t_w1;        /* [C, 256]   timestep MLP, first linear                       */
  const void* t_b1;        /* [C]                                                         */
  const void* t_w2;        /* [C, C]     timestep MLP, second linear                      */
  const void* t_b2;        /* [C]                                                         */
  const void* img_w;       /* [D, 128]   patch embedder                                   */
  const void* img_b;       /* [D]                                                         */
  const void* mod_w;       /* [L, 6D, C] per-block modulation (shift1,scale1,gate1,
                                          shift2,scale2,gate2)                             */
  const void* mod_b;       /* [L, 6D]                                                     */
  const void* wqkv;        /* [L, 3D, D] fused q|k|v projection ("proj.qkv", [INV])       */
  const float* q_gain;     /* [L, 128]   FP32 per-head RMSNorm gain of q                  */
  const float* k_gain;     /* [L, 128]   FP32 per-head RMSNorm gain of k                  */
  const void* wo;          /* [L, D, D]  attention output projection                      */
  const void* wg;          /* [L, F, D]  FFN gate projection                              */
  const void* wu;          /* [L, F, D]  FFN up projection                                */
  const void* wd;          /* [L, D, F]  FFN down projection ("proj.ffn_down")            */
  const void* final_mod_w; /* [2D, C]    final-layer modulation (shift_f, scale_f)         */
  const void* final_mod_b; /* [2D]                                                        */
  const void* out_w;       /* [128, D]   output projection to patch velocities             */
  const void* out_b;       /* [128]                                                       */
} moss_weights;

void moss_weights_init(moss_weights* w, uint32_t struct_size);

typedef struct moss_model moss_model;

/* Create a model on the current CUDA device.  Allocates the workspace for the capacities
 * in `cfg` once (no allocation happens in later calls) and builds the TMA descriptors of
 * the weights.  Errors: INVALID_ARGUMENT (shape, null or misaligned pointer),
 * ABI_MISMATCH (struct_size), UNSUPPORTED (head_dim != 128), OOM, CUDA. */
int moss_model_create(const moss_config* cfg, const moss_weights* w, moss_model** out);

/* Free the workspace.  Synchronises the device first.  NULL is accepted. */
void moss_model_free(moss_model* m);

/* ------------------------------------------------------------------------------------ */
/* The hot path.                                                                        */
/* ------------------------------------------------------------------------------------ */

/* One joint DiT block ([WP] 42 joint blocks; [INV] single-stream: image and text tokens
 * in one sequence), applied in place to `x`:
 *   h = LN(x)(1+scale1)+shift1;  q,k,v = h Wqkv^T;  q,k <- RoPE(RMSNorm(q,k));
 *   x += gate1 * (softmax(q k^T / sqrt(128)) v) Wo^T;
 *   h = LN(x)(1+scale2)+shift2;  x += gate2 * ((SiLU(h Wg^T) * (h Wu^T)) Wd^T)
 * with the modulation of layer `layer` at time `t` (sigma in [0, 1]).
 *   x:      device FP32 [batch, N, D], N = grid_h*grid_w + n_txt; modified in place.
 *   batch:  number of branches in x (1..max_batch); every branch runs this layer.
 *           A branch that skips the layer ([SGL-MOSS] 3, [INV] Skip layers) is simply not
 *           passed (the skip is the identity on that branch's stream).
 * Errors: INVALID_ARGUMENT (layer, sizes beyond the workspace, null x), CUDA. */
int moss_dit_block_forward(moss_model* m, int layer, float* x, int batch, int grid_h,
                           int grid_w, int n_txt, float t, void* stream);

/* The DiT velocity prediction for `batch` branches that share one latent:
 * patchify + embed the latent, append each branch's text states, run the L blocks (branch
 * b skips the layers listed in its row of skip_layers), final LN-modulate + output
 * projection of the image tokens, unpatchify.
 *   latent:      device FP32 [height/8, width/8, 32]
 *   text_states: device FP32 [batch, n_txt, D] (the refined prompt states)
 *   t:           sigma of this step
 *   skip_layers: host int [batch, n_skip]; entries in 0..L-1 or -1 (no entry); may be NULL
 *                when n_skip == 0
 *   v_out:       device FP32 [batch, height/8, width/8, 32]
 * Errors: INVALID_ARGUMENT (size rule of moss_validate, layer id out of range, capacities),
 * CUDA. */
int moss_dit_forward(moss_model* m, int batch, const float* latent, const float* text_states,
                     int n_txt, int height, int width, float t, const int* skip_layers,
                     int n_skip, float* v_out, void* stream);

/* FP32 CFG combine and Euler update, in place ([SGL-MOSS] 3: CFG arithmetic and scheduler
 * updates in FP32; flow-matching Euler [WP] Recommended settings):
 *   x[i] <- x[i] + (sigma_next - sigma) * (v_u[i] + cfg * (v_c[i] - v_u[i]))
 *   x, v_c, v_u: device FP32 [n], 16-byte aligned.  n >= 0 (0 launches nothing).
 * Errors: INVALID_ARGUMENT (null or misaligned pointer, n < 0), CUDA. */
int moss_cfg_euler_step(float* x, const float* v_c, const float* v_u, int64_t n, float cfg,
                        float sigma, float sigma_next, void* stream);

/* Shifted flow-matching schedule ("flow-matching Euler, shift 5", [WP]; [SGL-MOSS] 3),
 * host only: sigma_i = shift*s/(1+(shift-1)*s), s = 1 - i/steps, i = 0..steps, computed
 * in double and stored as float.  out: host float [steps+1].  steps >= 1, shift > 0. */
int moss_sigma_schedule(int steps, double shift, float* out);

/* 1 if the unconditional branch skips its layers at `step` of `steps`: the step fraction
 * step/steps lies in [slg_start, slg_stop] ([SGL-MOSS] 3: the default window 0.01..1.0
 * leaves the first step at full CFG; 0.0 starts at step 0), compared in double.  0 otherwise;
 * -1 on bad args. */
int moss_slg_active(int step, int steps, double slg_start, double slg_stop);

/* Initial noise: n standard normals from Philox4x32-10 keyed by `seed` (counter = index/4),
 * Box-Muller on 23-bit uniforms.  x: device FP32 [n], 16-byte aligned. */
int moss_init_noise(float* x, int64_t n, uint64_t seed, void* stream);

/* One denoising step of the default two-pass recipe at step index `step` of `steps`
 * ([SGL-MOSS] 3; [WP] Recommended settings): velocity of the conditional branch
 * (text_c) and, when cfg != 1, of the unconditional branch (text_u) skipping
 * uncond_skip_layers inside the [slg_start, slg_stop] window; then the CFG + Euler update
 * of `x` in place.  cfg == 1 runs no unconditional pass ([INV] Generation settings).
 * The two prompts may differ in length (the default negative prompt is empty); each branch
 * attends over its own tokens, without padding ([SGL-MOSS] 5. Batching).
 *   x: device FP32 [height/8, width/8, 32]
 *   text_c: device FP32 [n_txt_c, D];  text_u: device FP32 [n_txt_u, D] (unused when cfg == 1)
 *   uncond_skip_layers: host int [n_skip] in 0..L-1.
 * Modulation: when steps <= max_steps, the first call for a (steps, shift) schedule computes the
 * modulation vectors of all its steps at once (one pass over the modulation weights, as
 * moss_sample does) and later calls for the same schedule reuse them; a call of
 * moss_dit_forward, moss_dit_block_forward or moss_op_modulation in between drops them.  With
 * steps > max_steps each call computes its own step's vectors.  The weights are read-only for
 * the model's lifetime, so the reused vectors always match them.
 * Errors: as moss_dit_forward; each branch's image + text tokens must fit max_tokens. */
int moss_denoise_step(moss_model* m, float* x, const float* text_c, int n_txt_c, const float* text_u, int n_txt_u,
                      int height, int width, int step, int steps, float cfg, double shift,
                      const int* uncond_skip_layers, int n_skip, double slg_start, double slg_stop, void* stream);

/* moss_denoise_step with host buffers: the same step, with x_host (host FP32 [height/8, width/8,
 * 32], updated in place), text_c_host (host FP32 [n_txt_c, D]) and text_u_host (host FP32
 * [n_txt_u, D], unused when cfg == 1) in host memory.  The call copies the latent and the prompts
 * to the device on `stream`, runs the step there, copies the latent back and waits for the stream,
 * so x_host holds the result when it returns.  Pinned (page-locked) host buffers make the copies
 * asynchronous with the host; pageable ones work too, more slowly.  The device staging buffers
 * (the latent and two prompts at the model's maxima) are allocated on the first call and kept until
 * moss_model_free.  Errors: as moss_denoise_step; OOM if the staging buffers cannot be allocated. */
int moss_denoise_step_host(moss_model* m, float* x_host, const float* text_c_host, int n_txt_c,
                           const float* text_u_host, int n_txt_u, int height, int width, int step, int steps, float cfg,
                           double shift, const int* uncond_skip_layers, int n_skip, double slg_start, double slg_stop,
                           void* stream);

/* The full sampling loop ([SGL-MOSS] 3 defaults: 50 steps, shift 5, CFG 3, empty negative,
 * uncond layer 22 skipped in slg 0.01..1.0): noise from `seed`, then `steps` calls of the
 * denoising step.  Prompt arguments as for moss_denoise_step.  latent_out: device FP32
 * [height/8, width/8, 32] (also the working buffer).  steps <= max_steps of the model's
 * configuration. */
int moss_sample(moss_model* m, int steps, float cfg, double shift, uint64_t seed,
                const int* uncond_skip_layers, int n_skip, double slg_start, double slg_stop,
                const float* text_c, int n_txt_c, const float* text_u, int n_txt_u, int height, int width,
                float* latent_out, void* stream);

/* ------------------------------------------------------------------------------------ */
/* Text path ([WP] Architecture and specs: the frozen text encoder's final-layer states   */
/* pass through a projection and two text-only blocks).                                 */
/* ------------------------------------------------------------------------------------ */
/* Device pointers to the text-path parameters (BF16 except the FP32 gains, 16-byte aligned,
 * caller-owned, kept alive and unchanged while attached to a model). */
typedef struct moss_text_weights {
  uint32_t struct_size;  /* sizeof(moss_text_weights) as compiled by the caller              */
  int32_t enc_dim;       /* width of the encoder's final-layer states: 4096; multiple of 64   */
  int32_t blocks;        /* text-only blocks: 2; 0..8 (0 = projection only)                   */
  const void* proj_w;    /* [D, enc_dim]  projection                                          */
  const void* proj_b;    /* [D]                                                               */
  const void* wqkv;      /* [blocks, 3D, D] the joint blocks' layouts, one per text-only block */
  const float* q_gain;   /* [blocks, 128]                                                     */
  const float* k_gain;   /* [blocks, 128]                                                     */
  const void* wo;        /* [blocks, D, D]                                                    */
  const void* wg;        /* [blocks, F, D]                                                    */
  const void* wu;        /* [blocks, F, D]                                                    */
  const void* wd;        /* [blocks, D, F]                                                    */
} moss_text_weights;

/* Zero pointers, enc_dim 4096, blocks 2; struct_size as given. */
void moss_text_weights_init(moss_text_weights* tw, uint32_t struct_size);

/* Attach the text path to a model (replacing any attached before).  Builds the weight
 * descriptors and a 6*D-float device vector for the blocks' fixed modulation.  Synchronous.
 * Errors: MOSS_ERR_ABI_MISMATCH (struct_size), MOSS_ERR_INVALID_ARGUMENT (NULL model, enc_dim
 * not a positive multiple of 64, blocks outside 0..8, a NULL or misaligned pointer),
 * MOSS_ERR_OOM. */
int moss_text_refiner_set(moss_model* m, const moss_text_weights* tw);

/* The prompt's text states at width D from the encoder's final-layer states: text = enc W_p^T +
 * b_p, then each text-only block in order: the joint block on the prompt's tokens alone
 * (positions (j+1, 0, 0)) without timestep modulation (shifts and scales 0, gates 1), so the
 * result serves every step of a sampling run (readings of the pages' one-line description).
 *   enc_states: device BF16 [n_txt, enc_dim];  text_out: device FP32 [n_txt, D] (also the
 *   blocks' residual stream).  1 <= n_txt <= max_tokens.
 * Uses the model's workspace (calls on one model must not overlap) and replaces its cached
 * RoPE table, which the next image call rebuilds.
 * Errors: MOSS_ERR_INVALID_ARGUMENT (no text path attached, NULL or misaligned buffers, n_txt out
 * of range). */
int moss_text_refine(moss_model* m, const void* enc_states, int n_txt, float* text_out, void* stream);

/* Lossy accelerators of the sampling loop, both off by default ([MI] What works: Lossy
 * accelerators; Per-image settings: CFG truncation, Step cache).  They change the image. */
typedef struct moss_sample_options {
  uint32_t struct_size;        /* sizeof(moss_sample_options) as compiled by the caller       */
  /* CFG truncation, in [0, 1]; 1 (the default) is off.  Step i (0-based) with
   * i >= cfg_truncation * steps (compared in double) runs the conditional branch alone and
   * takes v = v_c.  No effect at cfg 1. */
  double cfg_truncation;
  /* First-block step cache: > 0 turns it on, 0 (the default) is off.  Each step runs block 0;
   * its output o (every row of every branch of the call) is compared with o_ref, block 0's
   * output at the last full call: change = sum|o - o_ref| / sum|o_ref|, summed in FP64.
   * change < threshold reuses the last full call's blocks 1..layers-1 as a residual
   * (stream = o + (x_L - o_ref) of that call); otherwise the step runs every block and becomes
   * the last full call.  The first step, and a step whose number of branches differs from the
   * last full call's (CFG truncation), always runs in full. */
  double step_cache_threshold;
  /* Three-pass skip-layer guidance ([SGL-MOSS] 3: three-pass SLG adds a skipped conditional
   * prediction; the pages give no formula, so this follows the library's reading): > 0 turns
   * it on, 0 (the default) keeps the two-pass recipe.  On a CFG step inside the
   * [slg_start, slg_stop] window a third pass runs the conditional branch with
   * uncond_skip_layers left out (v_cs), and v = v_u + cfg (v_c - v_u) + slg_scale (v_c - v_cs)
   * in FP32.  Needs max_batch >= 3.  Outside the window, and on truncated steps, two-pass. */
  double slg_scale;
  int* cached_out;    /* optional HOST int [steps]: 1 where the step reused the cache, else 0 */
  float* change_out;  /* optional HOST float [steps]: the change measured at the step, NaN where
                         there was no full call to compare with (or the cache is off) */
} moss_sample_options;

/* Defaults: cfg_truncation = 1, step_cache_threshold = 0, slg_scale = 0, no outputs; struct_size
 * as given. */
void moss_sample_options_init(moss_sample_options* opt, uint32_t struct_size);

/* moss_sample with the accelerators of `opt` (NULL = defaults, identical to moss_sample).
 * With the step cache on, the call waits on `stream` once per step (the host reads the change
 * to choose the step's path) and, on first use, allocates two FP32 buffers of
 * max_batch x max_tokens x hidden owned by the model (freed by moss_model_free).
 * Errors: as moss_sample; MOSS_ERR_ABI_MISMATCH when struct_size is not this version's;
 * MOSS_ERR_INVALID_ARGUMENT for cfg_truncation outside [0, 1], a negative or NaN threshold or
 * slg_scale, slg_scale > 0 with cfg != 1 on a model with max_batch < 3;
 * MOSS_ERR_OOM when the cache buffers cannot be allocated. */
int moss_sample_ex(moss_model* m, int steps, float cfg, double shift, uint64_t seed,
                   const int* uncond_skip_layers, int n_skip, double slg_start, double slg_stop,
                   const float* text_c, int n_txt_c, const float* text_u, int n_txt_u, int height, int width,
                   const moss_sample_options* opt, float* latent_out, void* stream);

/* ------------------------------------------------------------------------------------ */
/* Status, profiling and operator-level entry points (used by tests and the benchmark). */
/* ------------------------------------------------------------------------------------ */

/* Device error word set by a kernel whose bounded wait gave up (0 = none).  Synchronises
 * the device.  clear != 0 resets it.  Returns the word (>= 0) or -MOSS_ERR_CUDA. */
int moss_device_status(int clear);

/* Self-test of the device-side wait limit: launches one kernel whose single thread waits on a
 * barrier phase that nothing completes.  After about 2 s the wait gives up, the kernel records
 * 0x301 in the device error word (moss_device_status reads it) and returns; the context stays
 * usable.  Has no counterpart in the pages: it checks the library's own failure path. */
int moss_selftest_wait_timeout(void* stream);

/* Failure-path self-test of the attention kernel: the same call as moss_op_attention, except that
 * the CTA of query block 0, head 0, branch 0 never loads V for key step `step` (0 <= step <
 * ceil(n_tok / 128)).  Its bounded waits run out after 2 s, the device error word reads 0x201 or
 * 0x202 (whichever wait gave up first), o is not meaningful, and every warp of the kernel still
 * finishes (the named-barrier arrivals are unconditional); later launches compute normally.
 * Has no counterpart in the pages. */
int moss_selftest_attention_timeout(const void* qkv, void* o, int batch, int n_tok, int heads, int step,
                                    void* stream);

/* Kernel classes for profiling. */
enum {
  MOSS_K_GEMM_QKV = 0, MOSS_K_GEMM_OPROJ = 1, MOSS_K_GEMM_GATEUP = 2, MOSS_K_GEMM_DOWN = 3,
  MOSS_K_ATTENTION = 4, MOSS_K_LN_MOD = 5, MOSS_K_OTHER = 6, MOSS_K_CFG_EULER = 7, MOSS_K_COUNT = 8
};

/* Enable (1) or disable (0) CUDA-event timing of every launch of the model's kernels, per
 * class.  Resets the accumulators. */
int moss_profile_enable(moss_model* m, int enable);

/* As moss_profile_enable, timing only the launches of the classes whose bit (1 << class) is set
 * in class_mask (0 disables).  Each timed launch adds two event records to the stream, so a
 * caller that times the whole step can restrict the timing to the classes it reports. */
int moss_profile_enable_classes(moss_model* m, unsigned class_mask);

/* Launch count and summed device time (ms) of class `kclass` since the last enable.
 * Synchronises the device. */
int moss_profile_read(moss_model* m, int kclass, int64_t* launches, double* total_ms);

/* Number of kernels this library launched since the last call with reset != 0. */
int64_t moss_launch_count(int reset);

/* Plain BF16 GEMM on the tensor cores: C[M,N] (FP32) = A[M,K] B[N,K]^T.
 * A, B: device BF16, row-major, 16-byte aligned; K multiple of 64, N multiple of 32. */
int moss_op_gemm_bf16(const void* a, const void* b, float* c, int M, int N, int K, void* stream);

/* Joint attention of one block ([MI] What works: exact attention), on the fused
 * projection layout: qkv device BF16 [batch, N, 3*heads*128] (q | k | v, head h at
 * columns h*128 of each part, q and k already normalised and rotated; 16-byte aligned);
 * o device BF16 [batch, N, heads*128] = softmax(q k^T / sqrt(128)) v per head, no mask.
 * Numerics: FP32 scores and softmax statistics, P rounded to BF16 for the P V product,
 * exponentials base 2 (3/8 of them by a cubic with relative error <= 1.0e-4), O
 * normalised in FP32 and rounded to BF16.  N >= 1, any length (keys and queries past N are
 * masked).  Errors: MOSS_ERR_INVALID_ARGUMENT for a null or unaligned pointer or batch,
 * n_tok or heads below 1; MOSS_ERR_CUDA if the launch fails.  A device-side wait that gives
 * up after 2 s sets the device error word (0x201 producer, 0x202 MMA, 0x203 softmax; read
 * with moss_device_status) and the kernel still ends. */
int moss_op_attention(const void* qkv, void* o, int batch, int n_tok, int heads, void* stream);

/* LN-modulate: h[r,:] = BF16(LN(x[r,:]) * (1 + scale) + shift), eps 1e-6, biased
 * variance ([SGL-QWEN] Lossless LayerNorm modulation).  x device FP32 [rows, D];
 * shift, scale device FP32 [D]; h device BF16 [rows, D]; D multiple of 128, <= 8192. */
int moss_op_ln_modulate(const float* x, const float* shift, const float* scale, void* h,
                        int rows, int dim, void* stream);

/* Timestep conditioning of the model at time t: writes the modulation vectors of all
 * layers and of the final layer, mod device FP32 [L*6D + 2D]. */
int moss_op_modulation(moss_model* m, float t, float* mod, void* stream);

/* ------------------------------------------------------------------------------------ */
/* Allocation-free entry point.                                                          */
/* ------------------------------------------------------------------------------------ */

/* Limits of the fixed scratch used by moss_modulation_noalloc. */
#define MOSS_NOALLOC_MAX_TIMESTEPS 64
#define MOSS_NOALLOC_MAX_COND_DIM 256

/* The modulation vectors of moss_op_modulation (all layers, then the final layer) for n_t
 * timesteps, computed without allocating any memory and without a moss_model.  The pages
 * have no counterpart: this exists for callers that must not allocate device memory, such
 * as a serving process whose memory is reserved up front by its own allocator (a cudaMalloc
 * there fails or fragments the reserve), or a latency-critical thread that cannot afford the
 * implicit device synchronisation cudaMalloc may perform.
 *   cfg, w:   model shape and weights as for moss_model_create; only t_w1, t_b1, t_w2, t_b2,
 *             mod_w, mod_b, final_mod_w and final_mod_b are read.
 *   t_host:   host float [n_t], the timesteps (sigma); 1 <= n_t <= MOSS_NOALLOC_MAX_TIMESTEPS.
 *   mod_out:  device FP32 [n_t, L*6D + 2D], caller-owned, 16-byte aligned.
 * Scratch: the timesteps and the n_t conditioning vectors (at most 64 x 256 floats) live in
 * one fixed array in device memory (64 KB + 256 B) that the library reserves on every GPU it
 * is loaded on, for the life of the process.  The first call on a device looks up that
 * array's device address (once per device); make that first call before any stream capture.
 * Every call uses the same array: two calls whose work overlaps on the GPU (on different
 * streams, or from different threads) race on it, so serialise them.  Each call overwrites
 * all the scratch it reads, so results never depend on an earlier call.
 * Errors: INVALID_ARGUMENT (NULL or misaligned pointer, n_t or cond_dim beyond the limits
 * above), ABI_MISMATCH (struct_size), CUDA.  Calls no allocation routine. */
int moss_modulation_noalloc(const moss_config* cfg, const moss_weights* w, const float* t_host, int n_t,
                            float* mod_out, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* MOSS_DIT_H */
