"""Plain CPU oracle of the MOSS-Image DiT denoising step.

TEST INFRASTRUCTURE ONLY.  Nothing in the product library imports, links or runs
this file: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` use it.  It shares no code with the CUDA path.

Written for a reader who checks it against the pages by eye: numpy, float64,
one step of the method per function, no blocking, fusion or reordering.  Library
primitives used as steps: ``@`` (matmul), ``np.exp``/``np.log``/``np.cos``/
``np.sin``, ``np.max``/``np.sum``.

Sources (web pages; each function names the one it follows):
  [SGL-MOSS]  SGLang cookbook, "OpenMOSS/MOSS-Image"
  [MI]        MossInfer (mossimage.cpp) integration guide
  [INV]       InvokeAI MOSS-Image guide
  [WP]        windpaint.ai, "MOSS-Image: specs, settings, VRAM and text rendering tested"
  [SGL-QWEN]  SGLang cookbook, "Qwen-Image 2.1" (a sibling single-stream DiT, used only
              where the MOSS-Image pages are silent)

Readings taken where the pages are silent (each repeated where it is used):
  R1  sigma_i = shift*s_i / (1 + (shift-1)*s_i) with s_i = 1 - i/steps, i = 0..steps.
  R2  Skip-layer window on the step fraction p_i = i/steps, inclusive at both ends.
  R3  Euler x' = x + (sigma' - sigma)*v with v as predicted (flow multiplier 1).
  R4  CFG v = v_u + cfg*(v_c - v_u), in FP32.
  R5  Pre-norm: affine-free LayerNorm (biased variance, eps 1e-6) then *(1+scale)+shift.
  R6  Per-head RMSNorm of q and k (eps 1e-6) with a learned FP32 gain.
  R7  Modulation: c = MLP(sinusoid(1000*t)) of width 256; per block
      Linear(256 -> 6D) on SiLU(c) = [shift1, scale1, gate1, shift2, scale2, gate2];
      final layer Linear(256 -> 2D) = [shift_f, scale_f].  Same for image and text tokens.
  R8  FFN: SwiGLU, (SiLU(h Wg^T) * (h Wu^T)) Wd^T.  No biases in block linears.
  R9  RoPE: 3 axes over the 128-wide head, [32, 48, 48] dims = (text index, patch row,
      patch column), theta 10000, adjacent pairs (2j, 2j+1) rotated as complex numbers;
      image token (r, c) -> (0, r, c), text token j -> (j+1, 0, 0).
  R10 Sequence [image tokens row-major; text tokens]; patch vector index (dy*2+dx)*32+ch.
  R11 Timestep sinusoid on 1000*t with 128 frequencies exp(-ln(1e4) k/128), [cos, sin].
  R12 Attention scale 1/sqrt(128), no mask.
  R13 A skipped layer is the identity on that branch's residual stream.
  R14 Initial noise: Philox4x32-10 (Salmon et al., SC'11) keyed by the seed, counter =
      element-group index, Box-Muller on 23-bit uniforms.
  R15 The two CFG branches each attend over their own prompt tokens; their lengths may
      differ and are never padded.
  R19 CFG truncation X in [0, 1] (1 = off): step i runs the conditional branch alone
      (v = v_c) when cfg != 1 and i >= X * steps.
  R20 Step cache: the quantity watched is block 0's output, the residual stream of every
      branch of the call (image and text rows) right after block 0; its change is
      sum|o - o_ref| / sum|o_ref| against o_ref, block 0's output at the last full call.
  R21 A step reuses the cache when a last full call with the same number of branches exists
      and the change is below the threshold: its stream after the last block is
      o + (x_L - o_ref) of the last full call (blocks 1..L-1 of that call, as a residual).
      Otherwise it runs every block and becomes the last full call.  The first step is
      always a full call.
  R22 Text projection: a linear layer with bias from the encoder's final-layer states
      (width 4096) to D.
  R23 Text-only block: the joint block (R5-R9, R12) on the prompt's tokens alone, positions
      (j+1, 0, 0), without timestep modulation (shift 0, scale 0, gates 1), so the refined
      prompt is the same at every step.
  R24 Three-pass SLG (slg_scale > 0; parity unpinned: the pages give no formula): inside the
      skip window a third pass runs the conditional branch with the skip layers left out
      (v_cs), and v = v_u + cfg (v_c - v_u) + slg_scale (v_c - v_cs) in FP32; outside the
      window, and on CFG-truncated steps, the two-pass rule holds.
"""
from __future__ import annotations

import math

import numpy as np

F64 = np.float64
F32 = np.float32

EPS_LN = 1e-6
EPS_RMS = 1e-6
ROPE_THETA = 10000.0
ROPE_AXES = (32, 48, 48)
TIME_FREQ_DIM = 128  # 128 frequencies -> 256-wide [cos, sin] embedding


# --------------------------------------------------------------------------------------
# Request validation.  [MI] Defaults and validation: width and height multiples of 16,
# at most 4096 per side and at most 4.2 megapixels; [SGL-MOSS] §3: divisible by 16.
# The user-facing message is the official app's wording quoted in [MI] (server errors).
# --------------------------------------------------------------------------------------
SIZE_MESSAGE = "Height and width must be positive multiples of 16."


def validate_size(height: int, width: int) -> tuple[bool, str]:
    if height <= 0 or width <= 0 or height % 16 or width % 16:
        return False, SIZE_MESSAGE
    if height > 4096 or width > 4096:
        return False, "Height and width must be at most 4096."
    if height * width > 4_200_000:
        return False, "Height times width must be at most 4.2 megapixels."
    return True, ""


def image_tokens(height: int, width: int) -> int:
    """(H/16)(W/16) image tokens: one token per 2x2 patch of the 8x-downsampled
    latent ([WP] Architecture and specs: 4,096 image tokens at 1024^2)."""
    return (height // 16) * (width // 16)


# --------------------------------------------------------------------------------------
# Schedule and guidance window.
# --------------------------------------------------------------------------------------
def sigma_schedule(steps: int, shift: float) -> np.ndarray:
    """Shifted flow-matching schedule, reading R1.  "Steps: 50, flow-matching Euler,
    shift 5" ([WP] Recommended settings; [SGL-MOSS] §3).  Computed in float64, returned
    as float32 (scheduler state is FP32 per [SGL-MOSS] §3)."""
    i = np.arange(steps + 1, dtype=F64)
    s = 1.0 - i / steps
    sigma = shift * s / (1.0 + (shift - 1.0) * s)
    return sigma.astype(F32)


def slg_active(step: int, steps: int, slg_start: float, slg_stop: float) -> bool:
    """Whether the unconditional branch skips its layers at ``step`` (reading R2).
    [SGL-MOSS] §3: the default window slg_start=0.01, slg_stop=1.0 leaves the first step
    at full CFG; slg_start=0.0 gives the official pipeline's start-at-zero behaviour."""
    p = step / steps
    return slg_start <= p <= slg_stop


# --------------------------------------------------------------------------------------
# CFG combine and Euler update, FP32 ([SGL-MOSS] §3: CFG arithmetic and scheduler
# updates in FP32; readings R3, R4).
# --------------------------------------------------------------------------------------
def cfg_combine(v_c: np.ndarray, v_u: np.ndarray, cfg: float) -> np.ndarray:
    v_c = np.asarray(v_c, F32)
    v_u = np.asarray(v_u, F32)
    return (v_u + F32(cfg) * (v_c - v_u)).astype(F32)


def euler_update(x: np.ndarray, v: np.ndarray, sigma: float, sigma_next: float) -> np.ndarray:
    dt = F32(sigma_next) - F32(sigma)
    return (np.asarray(x, F32) + dt * np.asarray(v, F32)).astype(F32)


def cfg_euler(x, v_c, v_u, cfg, sigma, sigma_next):
    """One guided Euler step: x + (sigma' - sigma) * (v_u + cfg (v_c - v_u))."""
    return euler_update(x, cfg_combine(v_c, v_u, cfg), sigma, sigma_next)


def slg_combine(v_c: np.ndarray, v_u: np.ndarray, v_cs: np.ndarray, cfg: float, slg_scale: float) -> np.ndarray:
    """R24 (parity unpinned): the CFG combine plus slg_scale (v_c - v_cs), in FP32."""
    v_c = np.asarray(v_c, F32)
    v_cs = np.asarray(v_cs, F32)
    return (cfg_combine(v_c, v_u, cfg) + F32(slg_scale) * (v_c - v_cs)).astype(F32)


# --------------------------------------------------------------------------------------
# Initial noise, reading R14.  Philox4x32-10 as published by Salmon, Moraes, Dror and
# Shaw, "Parallel random numbers: as easy as 1, 2, 3" (SC'11): ten rounds of two
# 32x32->64 multiplies with a Weyl-sequence key schedule.
# --------------------------------------------------------------------------------------
PHILOX_M0 = 0xD2511F53
PHILOX_M1 = 0xCD9E8D57
PHILOX_W0 = 0x9E3779B9
PHILOX_W1 = 0xBB67AE85
_MASK32 = 0xFFFFFFFF


def philox4x32_10(ctr, key) -> np.ndarray:
    """ctr: uint32 array [4, n]; key: two uint32.  Returns uint32 [4, n]."""
    c = [np.asarray(ctr[j], dtype=np.uint64) for j in range(4)]
    k0 = np.uint64(int(key[0]) & _MASK32)
    k1 = np.uint64(int(key[1]) & _MASK32)
    m0 = np.uint64(PHILOX_M0)
    m1 = np.uint64(PHILOX_M1)
    mask = np.uint64(_MASK32)
    for r in range(10):
        if r > 0:
            k0 = (k0 + np.uint64(PHILOX_W0)) & mask
            k1 = (k1 + np.uint64(PHILOX_W1)) & mask
        p0 = m0 * c[0]  # exact: both factors < 2^32
        p1 = m1 * c[2]
        hi0, lo0 = p0 >> np.uint64(32), p0 & mask
        hi1, lo1 = p1 >> np.uint64(32), p1 & mask
        c = [hi1 ^ c[1] ^ k0, lo1, hi0 ^ c[3] ^ k1, lo0]
    return np.stack([x.astype(np.uint32) for x in c])


def uniform23(bits: np.ndarray) -> np.ndarray:
    """Top 23 bits of a uint32 as a uniform in (0, 1): ((b >> 9) + 1/2) / 2^23, a value
    with at most 24 significant bits, so exact in FP32 as well."""
    return ((bits.astype(np.uint64) >> np.uint64(9)).astype(F64) + 0.5) / float(1 << 23)


def gaussian_noise(n: int, seed: int) -> np.ndarray:
    """n standard normals (FP32).  Element e comes from Philox block g = e // 4 with
    counter (g_lo, g_hi, 0, 0) and key (seed_lo, seed_hi); outputs (x0, x1) give elements
    4g, 4g+1 and (x2, x3) give 4g+2, 4g+3 through Box-Muller:
    z = sqrt(-2 ln u_a) * (cos, sin)(2 pi u_b)."""
    groups = (n + 3) // 4
    g = np.arange(groups, dtype=np.uint64)
    ctr = np.stack([g & np.uint64(_MASK32), g >> np.uint64(32),
                    np.zeros_like(g), np.zeros_like(g)])
    key = (seed & _MASK32, (seed >> 32) & _MASK32)
    x = philox4x32_10(ctr, key)
    out = np.empty((groups, 4), dtype=F64)
    for pair in range(2):
        ua = uniform23(x[2 * pair])
        ub = uniform23(x[2 * pair + 1])
        r = np.sqrt(-2.0 * np.log(ua))
        out[:, 2 * pair] = r * np.cos(2.0 * math.pi * ub)
        out[:, 2 * pair + 1] = r * np.sin(2.0 * math.pi * ub)
    return out.reshape(-1)[:n].astype(F32)


# --------------------------------------------------------------------------------------
# Timestep conditioning, readings R7 and R11.  [INV] Transformer formats: the first layer
# of the time embeddings and the modulation layers exist and stay in compute dtype.
# --------------------------------------------------------------------------------------
def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def timestep_embedding(t: float) -> np.ndarray:
    k = np.arange(TIME_FREQ_DIM, dtype=F64)
    freqs = np.exp(-math.log(10000.0) * k / TIME_FREQ_DIM)
    arg = 1000.0 * float(t) * freqs
    return np.concatenate([np.cos(arg), np.sin(arg)])


def conditioning(t: float, w: dict) -> np.ndarray:
    """c = W2 SiLU(W1 emb + b1) + b2 (width c_t)."""
    emb = timestep_embedding(t)
    h = silu(w["t_w1"] @ emb + w["t_b1"])
    return w["t_w2"] @ h + w["t_b2"]


def block_modulation(c: np.ndarray, mod_w: np.ndarray, mod_b: np.ndarray) -> np.ndarray:
    """Per-block modulation vector [6D] = W_mod SiLU(c) + b_mod."""
    return mod_w @ silu(c) + mod_b


# --------------------------------------------------------------------------------------
# Patches, reading R10.  [WP] Architecture and specs: 2x2 latent patches, one token covers
# 16x16 pixels; the FLUX.2 latent has 32 channels at 8x downsampling.
# --------------------------------------------------------------------------------------
def patchify(latent: np.ndarray) -> np.ndarray:
    """latent [H8, W8, 32] -> tokens [(H8/2)(W8/2), 128]; token r*(W8/2)+c holds
    latent[2r+dy, 2c+dx, ch] at feature (dy*2+dx)*32+ch."""
    h8, w8, ch = latent.shape
    hp, wp = h8 // 2, w8 // 2
    tok = np.empty((hp * wp, 4 * ch), dtype=latent.dtype)
    for dy in range(2):
        for dx in range(2):
            f0 = (dy * 2 + dx) * ch
            tok[:, f0:f0 + ch] = latent[dy::2, dx::2, :].reshape(hp * wp, ch)
    return tok


def unpatchify(tokens: np.ndarray, h8: int, w8: int, ch: int = 32) -> np.ndarray:
    """Inverse of :func:`patchify`."""
    hp, wp = h8 // 2, w8 // 2
    lat = np.empty((h8, w8, ch), dtype=tokens.dtype)
    for dy in range(2):
        for dx in range(2):
            f0 = (dy * 2 + dx) * ch
            lat[dy::2, dx::2, :] = tokens[:, f0:f0 + ch].reshape(hp, wp, ch)
    return lat


# --------------------------------------------------------------------------------------
# Normalisation, readings R5 and R6.  [SGL-QWEN] "Lossless LayerNorm modulation"
# (affine-free LayerNorm times (1 + scale)) and "Lossless Q/K normalization" (RMSNorm
# with FP32 mean and a weight multiply) describe the sibling DiT's forms.
# --------------------------------------------------------------------------------------
def layer_norm(x: np.ndarray, eps: float = EPS_LN) -> np.ndarray:
    mean = x.mean(axis=-1, keepdims=True)
    var = ((x - mean) ** 2).mean(axis=-1, keepdims=True)
    return (x - mean) / np.sqrt(var + eps)


def ln_modulate(x: np.ndarray, shift: np.ndarray, scale: np.ndarray, eps: float = EPS_LN):
    return layer_norm(x, eps) * (1.0 + scale) + shift


def rms_norm(x: np.ndarray, gain: np.ndarray, eps: float = EPS_RMS) -> np.ndarray:
    ms = (x * x).mean(axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * gain


# --------------------------------------------------------------------------------------
# Rotary position embedding, reading R9.  [SGL-QWEN] "Lossless RoPE fusion": the sibling
# DiT applies RoPE as a complex rotary multiplication.
# --------------------------------------------------------------------------------------
def token_positions(grid_h: int, grid_w: int, n_txt: int) -> np.ndarray:
    """[N, 3] integer positions (text index, patch row, patch column)."""
    n_img = grid_h * grid_w
    pos = np.zeros((n_img + n_txt, 3), dtype=np.int64)
    r, c = np.divmod(np.arange(n_img), grid_w)
    pos[:n_img, 1] = r
    pos[:n_img, 2] = c
    pos[n_img:, 0] = np.arange(n_txt) + 1
    return pos


def rope_angles(pos: np.ndarray, head_dim: int = 128) -> np.ndarray:
    """[N, head_dim/2] rotation angles; pair j belongs to the axis whose dims cover 2j."""
    assert sum(ROPE_AXES) == head_dim
    cols = []
    for axis, dim in enumerate(ROPE_AXES):
        i = np.arange(dim // 2, dtype=F64)
        omega = ROPE_THETA ** (-2.0 * i / dim)
        cols.append(pos[:, axis:axis + 1].astype(F64) * omega[None, :])
    return np.concatenate(cols, axis=1)


def apply_rope(x: np.ndarray, angles: np.ndarray) -> np.ndarray:
    """x [..., N, 128]: pair (x[2j], x[2j+1]) -> rotated by angles[:, j]."""
    x0 = x[..., 0::2]
    x1 = x[..., 1::2]
    cos, sin = np.cos(angles), np.sin(angles)
    out = np.empty_like(x)
    out[..., 0::2] = x0 * cos - x1 * sin
    out[..., 1::2] = x0 * sin + x1 * cos
    return out


# --------------------------------------------------------------------------------------
# Attention, reading R12.  [MI] What works: exact (FlashAttention-2) attention; the
# single-stream block attends over image and text tokens jointly ([WP], [INV]).
# --------------------------------------------------------------------------------------
def softmax(s: np.ndarray) -> np.ndarray:
    s = s - s.max(axis=-1, keepdims=True)
    e = np.exp(s)
    return e / e.sum(axis=-1, keepdims=True)


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """q, k, v [H, N, d] -> [H, N, d]; scores materialised one head at a time."""
    out = np.empty_like(q)
    scale = 1.0 / math.sqrt(q.shape[-1])
    for h in range(q.shape[0]):
        p = softmax((q[h] @ k[h].T) * scale)
        out[h] = p @ v[h]
    return out


# --------------------------------------------------------------------------------------
# The joint block, readings R5-R8, R12.  [WP]: 42 joint blocks, hidden 3072, 24 heads of
# 128, FFN 8192; image and text tokens in one sequence ([INV]: single-stream).
# --------------------------------------------------------------------------------------
def block_forward(x: np.ndarray, lw: dict, mod: np.ndarray, angles: np.ndarray,
                  heads: int, head_dim: int = 128) -> np.ndarray:
    """x [N, D] (one branch) -> x after the block.

    lw: wqkv [3D, D], q_gain [d], k_gain [d], wo [D, D], wg [F, D], wu [F, D], wd [D, F].
    mod: [6D] = shift1, scale1, gate1, shift2, scale2, gate2.
    """
    n, D = x.shape
    shift1, scale1, gate1, shift2, scale2, gate2 = np.split(mod, 6)

    h = ln_modulate(x, shift1, scale1)
    qkv = h @ lw["wqkv"].T
    q, k, v = np.split(qkv, 3, axis=1)
    q = q.reshape(n, heads, head_dim).transpose(1, 0, 2)
    k = k.reshape(n, heads, head_dim).transpose(1, 0, 2)
    v = v.reshape(n, heads, head_dim).transpose(1, 0, 2)
    q = apply_rope(rms_norm(q, lw["q_gain"]), angles)
    k = apply_rope(rms_norm(k, lw["k_gain"]), angles)
    o = attention(q, k, v).transpose(1, 0, 2).reshape(n, D)
    x = x + gate1 * (o @ lw["wo"].T)

    h2 = ln_modulate(x, shift2, scale2)
    a = silu(h2 @ lw["wg"].T) * (h2 @ lw["wu"].T)
    x = x + gate2 * (a @ lw["wd"].T)
    return x


def block_forward_rows(x: np.ndarray, lw: dict, mod: np.ndarray, angles: np.ndarray, rows,
                       heads: int, head_dim: int = 128) -> np.ndarray:
    """The block's output for the query rows ``rows`` only: the same definition as
    :func:`block_forward`, using that every step but attention acts row by row and that
    attention needs the keys and values of all rows.  Returns [len(rows), D]."""
    n, D = x.shape
    rows = np.asarray(rows)
    shift1, scale1, gate1, shift2, scale2, gate2 = np.split(mod, 6)
    h = ln_modulate(x, shift1, scale1)
    wq, wk, wv = np.split(lw["wqkv"], 3, axis=0)
    q = (h[rows] @ wq.T).reshape(len(rows), heads, head_dim).transpose(1, 0, 2)
    k = (h @ wk.T).reshape(n, heads, head_dim).transpose(1, 0, 2)
    v = (h @ wv.T).reshape(n, heads, head_dim).transpose(1, 0, 2)
    q = apply_rope(rms_norm(q, lw["q_gain"]), angles[rows])
    k = apply_rope(rms_norm(k, lw["k_gain"]), angles)
    o = attention(q, k, v).transpose(1, 0, 2).reshape(len(rows), D)
    xr = x[rows] + gate1 * (o @ lw["wo"].T)
    h2 = ln_modulate(xr, shift2, scale2)
    a = silu(h2 @ lw["wg"].T) * (h2 @ lw["wu"].T)
    return xr + gate2 * (a @ lw["wd"].T)


def layer_weights(w: dict, l: int) -> dict:
    return {k: w[k][l] for k in ("wqkv", "q_gain", "k_gain", "wo", "wg", "wu", "wd")}


def final_layer(x_img: np.ndarray, c: np.ndarray, w: dict) -> np.ndarray:
    """Image rows -> velocity tokens [n_img, 128]: LN-modulate with the final
    [shift_f, scale_f], then the output linear with bias ([INV]: output layers)."""
    shift_f, scale_f = np.split(block_modulation(c, w["final_mod_w"], w["final_mod_b"]), 2)
    return ln_modulate(x_img, shift_f, scale_f) @ w["out_w"].T + w["out_b"]


def dit_forward(latent: np.ndarray, text_states: np.ndarray, t: float, skip_sets, w: dict,
                heads: int, head_dim: int = 128) -> np.ndarray:
    """One DiT pass per branch.

    latent [H8, W8, 32] (shared by the branches), text_states [B, n_txt, D],
    skip_sets: B collections of skipped layer ids (reading R13).
    Returns the predicted velocity [B, H8, W8, 32] (float64).
    """
    h8, w8, _ = latent.shape
    gh, gw = h8 // 2, w8 // 2
    B, n_txt, D = text_states.shape
    L = w["wqkv"].shape[0]
    angles = rope_angles(token_positions(gh, gw, n_txt), head_dim)
    c = conditioning(t, w)
    mods = [block_modulation(c, w["mod_w"][l], w["mod_b"][l]) for l in range(L)]
    img = patchify(np.asarray(latent, F64)) @ w["img_w"].T + w["img_b"]
    out = np.empty((B, h8, w8, latent.shape[2]), dtype=F64)
    for b in range(B):
        x = np.concatenate([img, np.asarray(text_states[b], F64)], axis=0)
        for l in range(L):
            if l in skip_sets[b]:
                continue
            x = block_forward(x, layer_weights(w, l), mods[l], angles, heads, head_dim)
        v_tok = final_layer(x[:gh * gw], c, w)
        out[b] = unpatchify(v_tok, h8, w8, latent.shape[2])
    return out


# --------------------------------------------------------------------------------------
# The sampler.  [SGL-MOSS] §3 and [WP] Recommended settings: 50 steps of flow-matching
# Euler at shift 5, CFG 3 with an empty negative prompt, the negative branch skipping
# block 22 inside the slg window; CFG 1 runs no negative pass ([INV] Generation settings).
# --------------------------------------------------------------------------------------
def sample(w: dict, heads: int, height: int, width: int, text_c: np.ndarray, text_u: np.ndarray,
           steps: int = 50, cfg: float = 3.0, shift: float = 5.0, seed: int = 42,
           uncond_skip_layers=(22,), slg_start: float = 0.01, slg_stop: float = 1.0,
           head_dim: int = 128, x0: np.ndarray | None = None) -> np.ndarray:
    ok, msg = validate_size(height, width)
    if not ok:
        raise ValueError(msg)
    h8, w8 = height // 8, width // 8
    if x0 is None:
        x = gaussian_noise(h8 * w8 * 32, seed).reshape(h8, w8, 32)
    else:
        x = np.asarray(x0, F32).copy()
    sig = sigma_schedule(steps, shift)
    for i in range(steps):
        t = float(sig[i])
        if cfg == 1.0:
            v_c = dit_forward(x, text_c[None], t, [()], w, heads, head_dim)[0]
            x = euler_update(x, v_c.astype(F32), sig[i], sig[i + 1])
            continue
        skip_u = tuple(uncond_skip_layers) if slg_active(i, steps, slg_start, slg_stop) else ()
        # Each branch attends over its own prompt: the two may differ in length (the default
        # negative prompt is empty), with no padding ([SGL-MOSS] 5: samples of different text
        # length run without padding).
        v_c = dit_forward(x, np.asarray(text_c)[None], t, [()], w, heads, head_dim)[0].astype(F32)
        v_u = dit_forward(x, np.asarray(text_u)[None], t, [skip_u], w, heads, head_dim)[0].astype(F32)
        x = cfg_euler(x, v_c, v_u, cfg, sig[i], sig[i + 1])
    return x


# --------------------------------------------------------------------------------------
# Text path.  [WP] Architecture and specs: the frozen text encoder's final-layer states pass
# through a projection and two text-only blocks before they join the image tokens.
# Readings R22, R23.
# --------------------------------------------------------------------------------------
def text_projection(enc_states: np.ndarray, proj_w: np.ndarray, proj_b: np.ndarray) -> np.ndarray:
    """R22: [n, enc_dim] -> [n, D]."""
    return np.asarray(enc_states, F64) @ np.asarray(proj_w, F64).T + np.asarray(proj_b, F64)


def unmodulated(D: int) -> np.ndarray:
    """R23: the modulation vector of a text-only block: shifts and scales 0, gates 1."""
    m = np.zeros(6 * D, dtype=F64)
    m[2 * D:3 * D] = 1.0
    m[5 * D:6 * D] = 1.0
    return m


def text_refine(enc_states: np.ndarray, tw: dict, heads: int, head_dim: int = 128) -> np.ndarray:
    """The prompt's text states at width D: projection, then each text-only block in order."""
    x = text_projection(enc_states, tw["proj_w"], tw["proj_b"])
    angles = rope_angles(token_positions(0, 0, x.shape[0]), head_dim)
    mod = unmodulated(x.shape[1])
    for l in range(tw["wqkv"].shape[0]):
        x = block_forward(x, layer_weights(tw, l), mod, angles, heads, head_dim)
    return x


# --------------------------------------------------------------------------------------
# Lossy accelerators, off by default.  [MI] What works (Lossy accelerators) and the opt-in
# list that follows it; Per-image settings (CFG truncation, Step cache): CFG truncation drops
# the negative branch from step X*steps on; the step cache (First-Block Cache) reuses blocks
# 1..L-1 of the last full call while block 0's output changed by less than a threshold.
# Readings R19-R21.
# --------------------------------------------------------------------------------------
def cfg_truncated(step: int, steps: int, cfg_truncation: float) -> bool:
    """R19: the negative branch is dropped at step `step` (0-based)."""
    return step >= cfg_truncation * steps


def relative_change(outs, refs) -> float:
    """R20: sum |o - o_ref| / sum |o_ref| over every row of every branch."""
    num = sum(float(np.sum(np.abs(np.asarray(o, F64) - np.asarray(r, F64)))) for o, r in zip(outs, refs))
    den = sum(float(np.sum(np.abs(np.asarray(r, F64)))) for r in refs)
    return num / den


def sample_accelerated(w: dict, heads: int, height: int, width: int, text_c: np.ndarray, text_u: np.ndarray,
                       steps: int = 50, cfg: float = 3.0, shift: float = 5.0, seed: int = 42,
                       uncond_skip_layers=(22,), slg_start: float = 0.01, slg_stop: float = 1.0,
                       cfg_truncation: float = 1.0, step_cache_threshold: float = 0.0, decisions=None,
                       slg_scale: float = 0.0, head_dim: int = 128, x0: np.ndarray | None = None):
    """The sampler of `sample` with CFG truncation (R19), the step cache (R20, R21) and
    three-pass SLG (R24; slg_scale 0 keeps the two-pass recipe).  Branch order of a call:
    conditional, skipped conditional (three-pass steps only), unconditional.

    step_cache_threshold <= 0 turns the cache off.  `decisions`, when given, replaces the
    threshold test of each step with decisions[i] (a step without a comparable full call
    still runs in full): a caller that already took the decisions in another precision
    replays them.  Returns (x, cached, change): the final latent, per step whether it reused
    the cache, and the block-0 change measured at that step (NaN when there was nothing to
    compare with).
    """
    ok, msg = validate_size(height, width)
    if not ok:
        raise ValueError(msg)
    h8, w8 = height // 8, width // 8
    gh, gw = h8 // 2, w8 // 2
    n_img = gh * gw
    L = w["wqkv"].shape[0]
    x = gaussian_noise(h8 * w8 * 32, seed).reshape(h8, w8, 32) if x0 is None else np.asarray(x0, F32).copy()
    sig = sigma_schedule(steps, shift)
    use_cache = step_cache_threshold > 0.0 or decisions is not None
    last = None  # (number of branches, block-0 outputs, residuals of blocks 1..L-1)
    cached, change = [], []
    for i in range(steps):
        t = float(sig[i])
        two = cfg != 1.0 and not cfg_truncated(i, steps, cfg_truncation)
        window = slg_active(i, steps, slg_start, slg_stop)
        three = two and slg_scale > 0.0 and window
        skip_u = tuple(uncond_skip_layers) if window else ()
        tc, tu = np.asarray(text_c, F64), np.asarray(text_u, F64)
        if three:
            texts, skips = [tc, tc, tu], [(), skip_u, skip_u]
        elif two:
            texts, skips = [tc, tu], [(), skip_u]
        else:
            texts, skips = [tc], [()]
        c = conditioning(t, w)
        mods = [block_modulation(c, w["mod_w"][l], w["mod_b"][l]) for l in range(L)]
        img = patchify(np.asarray(x, F64)) @ w["img_w"].T + w["img_b"]
        angles = [rope_angles(token_positions(gh, gw, tb.shape[0]), head_dim) for tb in texts]
        o0 = []
        for b, tb in enumerate(texts):
            xb = np.concatenate([img, tb], axis=0)
            if 0 not in skips[b]:
                xb = block_forward(xb, layer_weights(w, 0), mods[0], angles[b], heads, head_dim)
            o0.append(xb)
        ch = float("nan")
        reuse = False
        if use_cache and last is not None and last[0] == len(texts):
            ch = relative_change(o0, last[1])
            reuse = bool(decisions[i]) if decisions is not None else ch < step_cache_threshold
        if reuse:
            xl = [o0[b] + last[2][b] for b in range(len(texts))]
        else:
            xl = []
            for b in range(len(texts)):
                xb = o0[b]
                for l in range(1, L):
                    if l not in skips[b]:
                        xb = block_forward(xb, layer_weights(w, l), mods[l], angles[b], heads, head_dim)
                xl.append(xb)
            if use_cache:
                last = (len(texts), o0, [xl[b] - o0[b] for b in range(len(texts))])
        v = [unpatchify(final_layer(xb[:n_img], c, w), h8, w8, 32).astype(F32) for xb in xl]
        if three:
            x = euler_update(x, slg_combine(v[0], v[2], v[1], cfg, slg_scale), sig[i], sig[i + 1])
        elif two:
            x = cfg_euler(x, v[0], v[1], cfg, sig[i], sig[i + 1])
        else:
            x = euler_update(x, v[0], sig[i], sig[i + 1])
        cached.append(reuse)
        change.append(ch)
    return x, cached, change


def psnr(ref: np.ndarray, test: np.ndarray) -> float:
    """10 log10(range(ref)^2 / MSE), range = max - min of the reference."""
    ref = np.asarray(ref, F64)
    test = np.asarray(test, F64)
    mse = float(np.mean((ref - test) ** 2))
    rng = float(ref.max() - ref.min())
    if mse == 0.0:
        return float("inf")
    return 10.0 * math.log10(rng * rng / mse)
