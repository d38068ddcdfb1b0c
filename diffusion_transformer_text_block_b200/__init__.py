"""Python binding of libmossdit.so, the B200 (sm_100a) MOSS-Image DiT denoising-step library.

Argument marshalling only: every step of the computation runs in the library's CUDA
kernels.  Tensors are PyTorch CUDA tensors (device memory and streams come from torch);
the binding checks their dtype, device and contiguity and passes raw pointers.

There is no fallback: if the shared library is missing or fails to load, every call
raises ``MossError``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmossdit.so")
HEADER_PATH = os.path.join(os.path.dirname(HERE), "include", "moss_dit.h")

ABI_VERSION = 1
STATUS = {0: "OK", 1: "INVALID_ARGUMENT", 2: "CUDA", 3: "OOM", 4: "TIMEOUT", 5: "ABI_MISMATCH", 6: "UNSUPPORTED"}
K_GEMM_QKV, K_GEMM_OPROJ, K_GEMM_GATEUP, K_GEMM_DOWN, K_ATTENTION, K_LN_MOD, K_OTHER, K_CFG_EULER = range(8)
KERNEL_CLASSES = ["gemm_qkv", "gemm_oproj", "gemm_gateup", "gemm_down", "attention", "ln_mod", "other", "cfg_euler"]


class MossError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{STATUS.get(code, code)}: {msg}")
        self.code = code


class Config(ctypes.Structure):
    _fields_ = [("struct_size", ctypes.c_uint32)] + [(n, ctypes.c_int32) for n in (
        "layers", "hidden", "heads", "head_dim", "ffn", "cond_dim", "max_tokens", "max_batch",
        "max_latent_hw", "max_steps")]


WEIGHT_FIELDS = ("t_w1", "t_b1", "t_w2", "t_b2", "img_w", "img_b", "mod_w", "mod_b", "wqkv", "q_gain",
                 "k_gain", "wo", "wg", "wu", "wd", "final_mod_w", "final_mod_b", "out_w", "out_b")


class Weights(ctypes.Structure):
    _fields_ = [("struct_size", ctypes.c_uint32)] + [(n, ctypes.c_void_p) for n in WEIGHT_FIELDS]


TEXT_WEIGHT_FIELDS = ("proj_w", "proj_b", "wqkv", "q_gain", "k_gain", "wo", "wg", "wu", "wd")


class TextWeights(ctypes.Structure):
    _fields_ = [("struct_size", ctypes.c_uint32), ("enc_dim", ctypes.c_int32), ("blocks", ctypes.c_int32)] + \
        [(n, ctypes.c_void_p) for n in TEXT_WEIGHT_FIELDS]


class SampleOptions(ctypes.Structure):
    _fields_ = [("struct_size", ctypes.c_uint32), ("cfg_truncation", ctypes.c_double),
                ("step_cache_threshold", ctypes.c_double), ("slg_scale", ctypes.c_double),
                ("cached_out", ctypes.POINTER(ctypes.c_int)),
                ("change_out", ctypes.POINTER(ctypes.c_float))]


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_F = ctypes.c_float
_D = ctypes.c_double

_SIGS = {
    "moss_abi_version": (_I, []),
    "moss_last_error": (ctypes.c_char_p, []),
    "moss_validate": (_I, [_I, _I]),
    "moss_config_init": (None, [ctypes.POINTER(Config), ctypes.c_uint32]),
    "moss_weights_init": (None, [ctypes.POINTER(Weights), ctypes.c_uint32]),
    "moss_model_create": (_I, [ctypes.POINTER(Config), ctypes.POINTER(Weights), ctypes.POINTER(_P)]),
    "moss_model_free": (None, [_P]),
    "moss_dit_block_forward": (_I, [_P, _I, _P, _I, _I, _I, _I, _F, _P]),
    "moss_dit_forward": (_I, [_P, _I, _P, _P, _I, _I, _I, _F, _P, _I, _P, _P]),
    "moss_cfg_euler_step": (_I, [_P, _P, _P, _I64, _F, _F, _F, _P]),
    "moss_sigma_schedule": (_I, [_I, _D, ctypes.POINTER(_F)]),
    "moss_slg_active": (_I, [_I, _I, _D, _D]),
    "moss_init_noise": (_I, [_P, _I64, ctypes.c_uint64, _P]),
    "moss_denoise_step": (_I, [_P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _F, _D, _P, _I, _D, _D, _P]),
    "moss_denoise_step_host": (_I, [_P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _F, _D, _P, _I, _D, _D, _P]),
    "moss_sample": (_I, [_P, _I, _F, _D, ctypes.c_uint64, _P, _I, _D, _D, _P, _I, _P, _I, _I, _I, _P, _P]),
    "moss_text_weights_init": (None, [ctypes.POINTER(TextWeights), ctypes.c_uint32]),
    "moss_text_refiner_set": (_I, [_P, ctypes.POINTER(TextWeights)]),
    "moss_text_refine": (_I, [_P, _P, _I, _P, _P]),
    "moss_sample_options_init": (None, [ctypes.POINTER(SampleOptions), ctypes.c_uint32]),
    "moss_sample_ex": (_I, [_P, _I, _F, _D, ctypes.c_uint64, _P, _I, _D, _D, _P, _I, _P, _I, _I, _I,
                            ctypes.POINTER(SampleOptions), _P, _P]),
    "moss_device_status": (_I, [_I]),
    "moss_selftest_wait_timeout": (_I, [_P]),
    "moss_selftest_attention_timeout": (_I, [_P, _P, _I, _I, _I, _I, _P]),
    "moss_profile_enable": (_I, [_P, _I]),
    "moss_profile_enable_classes": (_I, [_P, ctypes.c_uint]),
    "moss_profile_read": (_I, [_P, _I, ctypes.POINTER(_I64), ctypes.POINTER(_D)]),
    "moss_launch_count": (_I64, [_I]),
    "moss_op_gemm_bf16": (_I, [_P, _P, _P, _I, _I, _I, _P]),
    "moss_op_attention": (_I, [_P, _P, _I, _I, _I, _P]),
    "moss_op_ln_modulate": (_I, [_P, _P, _P, _P, _I, _I, _P]),
    "moss_op_modulation": (_I, [_P, _F, _P, _P]),
    "moss_modulation_noalloc": (_I, [ctypes.POINTER(Config), ctypes.POINTER(Weights), ctypes.POINTER(_F), _I, _P,
                                     _P]),
}

NOALLOC_MAX_TIMESTEPS = 64


def lib():
    """Load (once) and return the shared library; raise MossError when it is unavailable."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise MossError(2, f"{LIB_PATH} is not built; run __graft_entry__.build()")
        try:
            handle = ctypes.CDLL(LIB_PATH)
        except OSError as e:  # pragma: no cover - depends on the machine
            raise MossError(2, f"cannot load {LIB_PATH}: {e}") from e
        for name, (res, args) in _SIGS.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        if handle.moss_abi_version() != ABI_VERSION:
            raise MossError(5, "library ABI version differs from the binding's")
        _lib = handle
    return _lib


def _check(rc: int):
    if rc != 0:
        raise MossError(rc, lib().moss_last_error().decode())


def _stream(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t, dtype=None, name="tensor"):
    import torch
    if t is None:
        return None
    if not t.is_cuda:
        raise MossError(1, f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise MossError(1, f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise MossError(1, f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def _host_ptr(t, name="tensor"):
    """Address of a contiguous FP32 CPU tensor (pinned or pageable) for the host-buffer calls."""
    import torch
    if t is None:
        return None
    if t.is_cuda:
        raise MossError(1, f"{name} must be a host (CPU) tensor")
    if not t.is_contiguous():
        raise MossError(1, f"{name} must be contiguous")
    if t.dtype != torch.float32:
        raise MossError(1, f"{name} must be torch.float32, got {t.dtype}")
    return t.data_ptr()


# ----------------------------------------------------------------------------- free functions
def validate(height: int, width: int) -> None:
    _check(lib().moss_validate(height, width))


def sigma_schedule(steps: int, shift: float):
    out = (ctypes.c_float * (steps + 1))()
    _check(lib().moss_sigma_schedule(steps, shift, out))
    return list(out)


def slg_active(step: int, steps: int, slg_start: float, slg_stop: float) -> bool:
    r = lib().moss_slg_active(step, steps, slg_start, slg_stop)
    if r < 0:
        raise MossError(1, "bad step arguments")
    return bool(r)


def cfg_euler_step(x, v_c, v_u, cfg: float, sigma: float, sigma_next: float, stream=None) -> None:
    import torch
    f = torch.float32
    _check(lib().moss_cfg_euler_step(_ptr(x, f, "x"), _ptr(v_c, f, "v_c"), _ptr(v_u, f, "v_u"), x.numel(), cfg,
                                     sigma, sigma_next, _stream(stream)))


def init_noise(x, seed: int, stream=None) -> None:
    import torch
    _check(lib().moss_init_noise(_ptr(x, torch.float32, "x"), x.numel(), seed, _stream(stream)))


def selftest_wait_timeout(stream=None) -> None:
    _check(lib().moss_selftest_wait_timeout(_stream(stream)))


def selftest_attention_timeout(qkv, heads: int, step: int, stream=None):
    """Attention with one CTA's V tile for key `step` never loaded (the failure-path self-test);
    returns the (meaningless) output tensor."""
    import torch
    B, N, _ = qkv.shape
    o = torch.empty(B, N, heads * 128, device=qkv.device, dtype=torch.bfloat16)
    _check(lib().moss_selftest_attention_timeout(_ptr(qkv, torch.bfloat16, "qkv"), o.data_ptr(), B, N, heads, step,
                                                 _stream(stream)))
    return o


def device_status(clear: bool = False) -> int:
    return lib().moss_device_status(1 if clear else 0)


def launch_count(reset: bool = False) -> int:
    return lib().moss_launch_count(1 if reset else 0)


def op_gemm_bf16(a, b, stream=None):
    """C = A B^T in FP32 on the tensor cores; A [M, K], B [N, K] BF16."""
    import torch
    M, K = a.shape
    N = b.shape[0]
    c = torch.empty(M, N, device=a.device, dtype=torch.float32)
    _check(lib().moss_op_gemm_bf16(_ptr(a, torch.bfloat16, "a"), _ptr(b, torch.bfloat16, "b"), c.data_ptr(), M, N,
                                   K, _stream(stream)))
    return c


def op_attention(qkv, heads: int, stream=None):
    """qkv [B, N, 3*heads*128] BF16 -> o [B, N, heads*128] BF16."""
    import torch
    B, N, _ = qkv.shape
    o = torch.empty(B, N, heads * 128, device=qkv.device, dtype=torch.bfloat16)
    _check(lib().moss_op_attention(_ptr(qkv, torch.bfloat16, "qkv"), o.data_ptr(), B, N, heads, _stream(stream)))
    return o


def op_ln_modulate(x, shift, scale, stream=None):
    import torch
    rows, dim = x.shape
    h = torch.empty(rows, dim, device=x.device, dtype=torch.bfloat16)
    f = torch.float32
    _check(lib().moss_op_ln_modulate(_ptr(x, f, "x"), _ptr(shift, f, "shift"), _ptr(scale, f, "scale"),
                                     h.data_ptr(), rows, dim, _stream(stream)))
    return h


def _config_for(shape, layers: int) -> Config:
    cfg = Config()
    lib().moss_config_init(ctypes.byref(cfg), ctypes.sizeof(Config))
    cfg.layers, cfg.hidden, cfg.heads, cfg.head_dim = layers, shape.hidden, shape.heads, shape.head_dim
    cfg.ffn, cfg.cond_dim = shape.ffn, shape.c_t
    return cfg


def modulation_noalloc(shape, weights: dict, ts: Sequence[float], out=None, stream=None):
    """Modulation vectors for the timesteps `ts` through the allocation-free entry point:
    returns (or fills) a CUDA FP32 tensor [len(ts), L*6D + 2D].  Only `out` is allocated
    here (by torch, when not given); the library itself allocates nothing."""
    import torch
    L = weights["mod_w"].shape[0]
    D, C = shape.hidden, shape.c_t
    stride = L * 6 * D + 2 * D
    # The library reads these weights and writes len(ts) rows of `stride` floats through raw
    # pointers; nothing below the C ABI can see a buffer's size, so every shape is checked here.
    need = {"t_w1": (C, 256), "t_b1": (C,), "t_w2": (C, C), "t_b2": (C,), "mod_w": (L, 6 * D, C),
            "mod_b": (L, 6 * D), "final_mod_w": (2 * D, C), "final_mod_b": (2 * D,)}
    for name, want_shape in need.items():
        if tuple(weights[name].shape) != want_shape:
            raise MossError(1, f"{name} must have shape {want_shape}, got {tuple(weights[name].shape)}")
    if out is not None and out.numel() < len(ts) * stride:
        raise MossError(1, f"out holds {out.numel()} floats; {len(ts)} timesteps need {len(ts) * stride}")
    if out is None:
        out = torch.empty(len(ts), stride, device="cuda", dtype=torch.float32)
    dev = torch.cuda.current_device()
    for name, t in [("out", out)] + [(k, weights[k]) for k in need]:
        if t.is_cuda and t.device.index != dev:
            raise MossError(1, f"{name} is on cuda:{t.device.index}, not on the current device cuda:{dev}")
    cfg = _config_for(shape, L)
    w = Weights()
    lib().moss_weights_init(ctypes.byref(w), ctypes.sizeof(Weights))
    for name in WEIGHT_FIELDS:
        want = torch.float32 if name in ("q_gain", "k_gain") else torch.bfloat16
        setattr(w, name, _ptr(weights[name], want, name))
    tarr = (ctypes.c_float * max(len(ts), 1))(*ts)
    _check(lib().moss_modulation_noalloc(ctypes.byref(cfg), ctypes.byref(w), tarr, len(ts),
                                         _ptr(out, torch.float32, "out"), _stream(stream)))
    return out


def _skip_array(skips: Sequence[Sequence[int]]):
    width = max([len(s) for s in skips] + [0])
    if width == 0:
        return None, 0
    flat = []
    for s in skips:
        flat += list(s) + [-1] * (width - len(s))
    return (ctypes.c_int * len(flat))(*flat), width


# ----------------------------------------------------------------------------- the model
class Model:
    """A DiT whose weights live in caller-owned CUDA tensors (kept referenced here)."""

    def __init__(self, shape, weights: dict, max_tokens: int, max_batch: int = 2, max_latent_hw: int = 128 * 128,
                 max_steps: int = 50):
        cfg = Config()
        lib().moss_config_init(ctypes.byref(cfg), ctypes.sizeof(Config))
        cfg.layers = weights["wqkv"].shape[0]
        cfg.hidden, cfg.heads, cfg.head_dim, cfg.ffn = shape.hidden, shape.heads, shape.head_dim, shape.ffn
        cfg.cond_dim = shape.c_t
        cfg.max_tokens, cfg.max_batch, cfg.max_latent_hw, cfg.max_steps = max_tokens, max_batch, max_latent_hw, max_steps
        w = Weights()
        lib().moss_weights_init(ctypes.byref(w), ctypes.sizeof(Weights))
        import torch
        for name in WEIGHT_FIELDS:
            t = weights[name]
            want = torch.float32 if name in ("q_gain", "k_gain") else torch.bfloat16
            setattr(w, name, _ptr(t, want, name))
        self._weights = weights
        self.shape = shape
        self.layers = cfg.layers
        self.cfg = cfg
        handle = ctypes.c_void_p()
        _check(lib().moss_model_create(ctypes.byref(cfg), ctypes.byref(w), ctypes.byref(handle)))
        self._h = handle

    def close(self):
        if getattr(self, "_h", None):
            lib().moss_model_free(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def set_text_weights(self, tw: dict):
        """Attach the text path: projection [D, enc_dim] + [D] and the text-only blocks' stacked
        weights (TEXT_WEIGHT_FIELDS; blocks = tw["wqkv"].shape[0], 0 if absent)."""
        import torch
        t = TextWeights()
        lib().moss_text_weights_init(ctypes.byref(t), ctypes.sizeof(TextWeights))
        t.enc_dim = tw["proj_w"].shape[1]
        t.blocks = tw["wqkv"].shape[0] if "wqkv" in tw else 0
        for name in TEXT_WEIGHT_FIELDS:
            if name not in tw:
                continue
            want = torch.float32 if name in ("q_gain", "k_gain") else torch.bfloat16
            setattr(t, name, _ptr(tw[name], want, name))
        _check(lib().moss_text_refiner_set(self._h, ctypes.byref(t)))
        self._text_weights = tw
        self.enc_dim = t.enc_dim

    def text_refine(self, enc_states, stream=None, out=None):
        """enc_states: CUDA BF16 [n_txt, enc_dim] -> FP32 [n_txt, D] text states."""
        import torch
        n = enc_states.shape[0]
        if out is None:
            out = torch.empty(n, self.shape.hidden, device=enc_states.device, dtype=torch.float32)
        _check(lib().moss_text_refine(self._h, _ptr(enc_states, torch.bfloat16, "enc_states"), n,
                                      _ptr(out, torch.float32, "out"), _stream(stream)))
        return out

    def block_forward(self, layer: int, x, grid_h: int, grid_w: int, n_txt: int, t: float, stream=None):
        import torch
        _check(lib().moss_dit_block_forward(self._h, layer, _ptr(x, torch.float32, "x"), x.shape[0], grid_h, grid_w,
                                            n_txt, t, _stream(stream)))
        return x

    def forward(self, latent, text_states, height: int, width: int, t: float,
                skip_layers: Sequence[Sequence[int]] = (), stream=None, out=None):
        import torch
        B, n_txt, _ = text_states.shape
        if out is None:
            out = torch.empty(B, height // 8, width // 8, 32, device=latent.device, dtype=torch.float32)
        skips = list(skip_layers) + [[]] * (B - len(skip_layers))
        arr, width_s = _skip_array(skips)
        _check(lib().moss_dit_forward(self._h, B, _ptr(latent, torch.float32, "latent"),
                                      _ptr(text_states, torch.float32, "text_states"), n_txt, height, width, t, arr,
                                      width_s, _ptr(out, torch.float32, "out"), _stream(stream)))
        return out

    def denoise_step(self, x, text_c, text_u, height: int, width: int, step: int, steps: int = 50, cfg: float = 3.0,
                     shift: float = 5.0, uncond_skip_layers: Sequence[int] = (22,), slg_start: float = 0.01,
                     slg_stop: float = 1.0, stream=None):
        """text_c [n_c, D] and text_u [n_u, D] may differ in length; text_u may be None when cfg == 1."""
        import torch
        arr, n = _skip_array([list(uncond_skip_layers)])
        f = torch.float32
        n_u = text_u.shape[0] if text_u is not None else 0
        _check(lib().moss_denoise_step(self._h, _ptr(x, f, "x"), _ptr(text_c, f, "text_c"), text_c.shape[0],
                                       _ptr(text_u, f, "text_u") if text_u is not None else None, n_u, height,
                                       width, step, steps, cfg, shift, arr, n, slg_start, slg_stop, _stream(stream)))
        return x

    def denoise_step_host(self, x, text_c, text_u, height: int, width: int, step: int, steps: int = 50,
                          cfg: float = 3.0, shift: float = 5.0, uncond_skip_layers: Sequence[int] = (22,),
                          slg_start: float = 0.01, slg_stop: float = 1.0, stream=None):
        """moss_denoise_step_host: x, text_c, text_u are FP32 CPU tensors (pinned for asynchronous
        copies); x is updated in place and holds the result when the call returns."""
        nx = (height // 8) * (width // 8) * 32
        D = self.shape.hidden
        if x.numel() != nx:
            raise MossError(1, f"x must hold {nx} floats")
        n_u = text_u.shape[0] if text_u is not None else 0
        if text_c.numel() != text_c.shape[0] * D or (text_u is not None and text_u.numel() != n_u * D):
            raise MossError(1, f"text states must be [n, {D}]")
        arr, n = _skip_array([list(uncond_skip_layers)])
        _check(lib().moss_denoise_step_host(self._h, _host_ptr(x, "x"), _host_ptr(text_c, "text_c"), text_c.shape[0],
                                            _host_ptr(text_u, "text_u") if text_u is not None else None, n_u, height,
                                            width, step, steps, cfg, shift, arr, n, slg_start, slg_stop,
                                            _stream(stream)))
        return x

    def sample(self, text_c, text_u, height: int, width: int, steps: int = 50, cfg: float = 3.0, shift: float = 5.0,
               seed: int = 42, uncond_skip_layers: Sequence[int] = (22,), slg_start: float = 0.01,
               slg_stop: float = 1.0, stream=None, out=None):
        import torch
        if out is None:
            out = torch.empty(height // 8, width // 8, 32, device=text_c.device, dtype=torch.float32)
        arr, n = _skip_array([list(uncond_skip_layers)])
        f = torch.float32
        n_u = text_u.shape[0] if text_u is not None else 0
        _check(lib().moss_sample(self._h, steps, cfg, shift, seed, arr, n, slg_start, slg_stop,
                                 _ptr(text_c, f, "text_c"), text_c.shape[0],
                                 _ptr(text_u, f, "text_u") if text_u is not None else None, n_u,
                                 height, width, _ptr(out, f, "out"), _stream(stream)))
        return out

    def sample_accelerated(self, text_c, text_u, height: int, width: int, steps: int = 50, cfg: float = 3.0,
                           shift: float = 5.0, seed: int = 42, uncond_skip_layers: Sequence[int] = (22,),
                           slg_start: float = 0.01, slg_stop: float = 1.0, cfg_truncation: float = 1.0,
                           step_cache_threshold: float = 0.0, slg_scale: float = 0.0, stream=None, out=None):
        """moss_sample_ex: returns (latent, cached [steps] list of bool, change [steps] list of float)."""
        import torch
        if out is None:
            out = torch.empty(height // 8, width // 8, 32, device=text_c.device, dtype=torch.float32)
        arr, n = _skip_array([list(uncond_skip_layers)])
        f = torch.float32
        n_u = text_u.shape[0] if text_u is not None else 0
        opt = SampleOptions()
        lib().moss_sample_options_init(ctypes.byref(opt), ctypes.sizeof(SampleOptions))
        opt.cfg_truncation = cfg_truncation
        opt.step_cache_threshold = step_cache_threshold
        opt.slg_scale = slg_scale
        cached = (ctypes.c_int * steps)()
        change = (ctypes.c_float * steps)()
        opt.cached_out = ctypes.cast(cached, ctypes.POINTER(ctypes.c_int))
        opt.change_out = ctypes.cast(change, ctypes.POINTER(ctypes.c_float))
        _check(lib().moss_sample_ex(self._h, steps, cfg, shift, seed, arr, n, slg_start, slg_stop,
                                    _ptr(text_c, f, "text_c"), text_c.shape[0],
                                    _ptr(text_u, f, "text_u") if text_u is not None else None, n_u,
                                    height, width, ctypes.byref(opt), _ptr(out, f, "out"), _stream(stream)))
        return out, [bool(c) for c in cached], [float(c) for c in change]

    def modulation(self, t: float, stream=None):
        import torch
        D, L = self.shape.hidden, self.layers
        mod = torch.empty(L * 6 * D + 2 * D, device="cuda", dtype=torch.float32)
        _check(lib().moss_op_modulation(self._h, t, mod.data_ptr(), _stream(stream)))
        return mod

    def profile_enable(self, enable: bool = True):
        _check(lib().moss_profile_enable(self._h, 1 if enable else 0))

    def profile_enable_classes(self, classes):
        """Time only the launches of the named kernel classes (KERNEL_CLASSES names)."""
        mask = 0
        for c in classes:
            mask |= 1 << KERNEL_CLASSES.index(c)
        _check(lib().moss_profile_enable_classes(self._h, mask))

    def profile_read(self) -> dict:
        out = {}
        for k, name in enumerate(KERNEL_CLASSES):
            n = ctypes.c_int64()
            ms = ctypes.c_double()
            _check(lib().moss_profile_read(self._h, k, ctypes.byref(n), ctypes.byref(ms)))
            out[name] = (n.value, ms.value)
        return out
