"""The Python binding's ctypes signature table against the C header (CPU): every declared entry
point is bound, with the same number of parameters, and each parameter and return value has a
ctypes type of the declared kind (pointer, or the matching integer / floating type)."""
import ctypes
import os
import re

import diffusion_transformer_text_block_b200 as moss

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moss_dit.h")

SCALARS = {
    "int": ctypes.c_int,
    "int64_t": ctypes.c_int64,
    "uint64_t": ctypes.c_uint64,
    "uint32_t": ctypes.c_uint32,
    "unsigned": ctypes.c_uint,
    "float": ctypes.c_float,
    "double": ctypes.c_double,
}


def _declarations():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    decls = {}
    for m in re.finditer(r"^[ \t]*([A-Za-z_][\w \t\*]*?)\b(moss_\w+)\s*\(([^;{]*?)\)\s*;", text, flags=re.S | re.M):
        ret, name, params = " ".join(m.group(1).split()), m.group(2), " ".join(m.group(3).split())
        if ret.startswith("typedef") or ret.endswith("struct"):
            continue
        args = [] if params in ("", "void") else [p.strip() for p in params.split(",")]
        decls[name] = (ret, args)
    return decls


def _kind(ctype_decl):
    """'pointer' for a pointer declaration, else the scalar's base type name."""
    if "*" in ctype_decl:
        return "pointer"
    words = [w for w in ctype_decl.replace("const", " ").split() if w not in ("enum", "struct")]
    return words[0]


def _matches(kind, ct):
    if kind == "pointer":
        return ct in (ctypes.c_void_p, ctypes.c_char_p) or (isinstance(ct, type) and issubclass(ct, ctypes._Pointer))
    if kind == "void":
        return ct is None
    return ct is SCALARS[kind]


def test_header_parses():
    decls = _declarations()
    assert "moss_sample" in decls and "moss_op_attention" in decls
    assert len(decls) >= 30


def test_every_declared_entry_point_is_bound_with_matching_types():
    decls = _declarations()
    sigs = moss._SIGS
    for name, (ret, args) in decls.items():
        assert name in sigs, f"{name} is declared but not bound"
        restype, argtypes = sigs[name]
        assert len(argtypes) == len(args), (name, len(argtypes), len(args))
        for i, (decl, ct) in enumerate(zip(args, argtypes)):
            param_type = decl.rsplit(" ", 1)[0] if "*" not in decl.rsplit(" ", 1)[-1] else decl
            assert _matches(_kind(param_type), ct), (name, i, decl, ct)
        assert _matches(_kind(ret) if "*" not in ret else "pointer", restype), (name, ret, restype)


def test_every_bound_name_is_declared():
    decls = _declarations()
    for name in moss._SIGS:
        assert name in decls, f"{name} is bound but not declared in the header"


def test_modulation_noalloc_checks_buffer_sizes_before_any_call():
    """The allocation-free entry point writes len(ts) rows of L*6D + 2D floats through a raw
    pointer: the binding refuses an `out` that is too short, and weights whose shapes do not match
    the layer count and widths, before it touches the library or a device."""
    import pytest
    import torch

    from synth import TINY, make_weights

    w = make_weights(TINY, 1)
    stride = TINY.layers * 6 * TINY.hidden + 2 * TINY.hidden
    with pytest.raises(moss.MossError, match="out holds"):
        moss.modulation_noalloc(TINY, w, [0.5, 0.25], out=torch.empty(2 * stride - 1))
    bad = dict(w, mod_b=w["mod_b"][:1])
    with pytest.raises(moss.MossError, match="mod_b must have shape"):
        moss.modulation_noalloc(TINY, bad, [0.5], out=torch.empty(stride))
    bad = dict(w, final_mod_w=w["final_mod_w"][:, :128])
    with pytest.raises(moss.MossError, match="final_mod_w must have shape"):
        moss.modulation_noalloc(TINY, bad, [0.5], out=torch.empty(stride))
