"""Host-side checks of the Python binding (no GPU needed).

The binding only marshals arguments: a missing library must raise, and
tensors that are not contiguous CUDA tensors must be rejected before any call
reaches the library -- there is no CPU or PyTorch fallback.
"""
import pytest
import torch

import causal_kernelized_sequence_b200 as la


def test_missing_library_raises(tmp_path, monkeypatch):
    monkeypatch.setattr(la, "_lib", None)
    with pytest.raises(ImportError):
        la.load_library(str(tmp_path / "libla_missing.so"))


def _cpu(*shape, dtype=torch.bfloat16):
    return torch.zeros(*shape, dtype=dtype)


@pytest.mark.parametrize("call", [
    lambda: la.la_forward(_cpu(1, 1, 8, 16), _cpu(1, 1, 8, 16), _cpu(1, 1, 8, 16), la.LA_FMAP_ELU1),
    lambda: la.la_forward_noalloc(_cpu(1, 1, 8, 16), _cpu(1, 1, 8, 16), _cpu(1, 1, 8, 16), la.LA_FMAP_ELU1),
    lambda: la.la_backward(_cpu(1, 1, 8, 16), _cpu(1, 1, 8, 16), _cpu(1, 1, 8, 16), _cpu(1, 1, 8, 16),
                           la.LA_FMAP_ELU1),
    lambda: la.la_backward_decay(_cpu(1, 1, 8, 16), _cpu(1, 1, 8, 16), _cpu(1, 1, 8, 16),
                                 _cpu(1, 1, 8, dtype=torch.float32), _cpu(1, 1, 8, 16), la.LA_FMAP_ELU1),
    lambda: la.la_decode_step(_cpu(1, 1, 16), _cpu(1, 1, 16), _cpu(1, 1, 16), _cpu(1, 1, 16, 16, dtype=torch.float32),
                              _cpu(1, 1, 16, dtype=torch.float32), la.LA_FMAP_ELU1),
    lambda: la.la_forward_varlen(_cpu(1, 8, 16), _cpu(1, 8, 16), _cpu(1, 8, 16),
                                 torch.tensor([0, 8], dtype=torch.int32), 8, la.LA_FMAP_ELU1),
    lambda: la.la_swa_forward(_cpu(1, 1, 8, 64), _cpu(1, 1, 8, 64), _cpu(1, 1, 8, 64), 64),
    lambda: la.la_feature_map(_cpu(4, 16), la.LA_FMAP_TAYLOR2),
])
def test_cpu_tensors_rejected(call):
    la.load_library()
    with pytest.raises(ValueError, match="CUDA"):
        call()


def _header_signatures():
    """{name: (return kind, [parameter kinds])} of every LA_API declaration in
    include/la.h, each kind one of ptr, int, size_t, int64, uint."""
    import os
    import re
    src = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "la.h")).read()
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)

    def kind(decl):
        decl = " ".join(decl.split())
        if "*" in decl:
            return "ptr"
        for word, k in (("size_t", "size_t"), ("int64_t", "int64"), ("unsigned int", "uint"),
                        ("la_status", "int"), ("int", "int")):
            if re.search(r"\b" + word + r"\b", decl):
                return k
        raise AssertionError(f"unclassified declaration {decl!r}")

    sigs = {}
    for m in re.finditer(r"\bLA_API\s+([^;(]*?)\b(la_\w+)\s*\(([^)]*)\)\s*;", src):
        ret, name, params = m.group(1), m.group(2), m.group(3).strip()
        plist = [] if params in ("", "void") else [kind(p) for p in params.split(",")]
        sigs[name] = (kind(ret + " x"), plist)
    return sigs


def _ctypes_kind(t):
    import ctypes
    if t in (ctypes.c_void_p, ctypes.c_char_p):
        return "ptr"
    table = {ctypes.c_int: "int", ctypes.c_size_t: "size_t", ctypes.c_int64: "int64", ctypes.c_uint: "uint"}
    return table[t]


def test_binding_signatures_match_header(monkeypatch):
    # The ctypes declarations in the binding must agree with include/la.h
    # argument by argument: a wrong width or a missing argument is not an
    # error ctypes can see, the call would just pass garbage.
    from causal_kernelized_sequence_b200 import build
    build.build()
    monkeypatch.setattr(la, "_lib", None)   # a fresh CDLL with only the binding's own declarations
    lib = la.load_library()
    sigs = _header_signatures()
    assert len(sigs) >= 25
    for name, (ret, params) in sigs.items():
        fn = getattr(lib, name)
        assert _ctypes_kind(fn.restype) == ret, name
        if params:
            assert fn.argtypes is not None, f"{name}: no argtypes"
            assert [_ctypes_kind(t) for t in fn.argtypes] == params, name
        else:
            assert not fn.argtypes, name


def _f32(*shape):
    return torch.zeros(*shape, dtype=torch.float32)


# Correctly shaped (CPU) tensors pass the binding's shape checks and are then
# refused only for not being CUDA tensors.
@pytest.mark.parametrize("call", [
    lambda: la.la_forward(_cpu(1, 2, 8, 16), _cpu(1, 2, 8, 16), _cpu(1, 2, 8, 64), la.LA_FMAP_TAYLOR2,
                          s_in=_f32(1, 2, 273, 64), z_in=_f32(1, 2, 273), out=_cpu(1, 2, 8, 64)),
    lambda: la.la_forward(_cpu(1, 2, 8, 16), _cpu(1, 2, 8, 16), _cpu(1, 2, 8, 64), la.LA_FMAP_ELU1,
                          log_decay=_f32(1, 2, 8)),
    lambda: la.la_decode_step(_f32(2, 3, 16), _f32(2, 3, 16), _f32(2, 3, 64), _f32(2, 3, 153, 64), _f32(2, 3, 153),
                              la.LA_FMAP_TAYLOR2_SYM, y=_f32(2, 3, 64), log_decay=_f32(2, 3)),
    lambda: la.la_forward_varlen(_cpu(2, 8, 16), _cpu(2, 8, 16), _cpu(2, 8, 64),
                                 torch.tensor([0, 3, 8], dtype=torch.int32), 5, la.LA_FMAP_ELU1,
                                 s_in=_f32(2, 2, 16, 64), z_in=_f32(2, 2, 16), out=_cpu(2, 8, 64)),
    lambda: la.la_swa_cache_fill(_cpu(1, 2, 8, 64), _cpu(1, 2, 8, 64), 16, k_cache=_cpu(1, 2, 16, 64),
                                 v_cache=_cpu(1, 2, 16, 64)),
    lambda: la.la_swa_decode_step(_cpu(1, 2, 64), _cpu(1, 2, 64), _cpu(1, 2, 64), _cpu(1, 2, 16, 64),
                                  _cpu(1, 2, 16, 64), torch.zeros(1, dtype=torch.int32), 16, y=_cpu(1, 2, 64)),
    lambda: la.la_backward(_cpu(1, 1, 8, 16), _cpu(1, 1, 8, 16), _cpu(1, 1, 8, 32), _cpu(1, 1, 8, 32),
                           la.LA_FMAP_ELU1, workspace=torch.zeros(1 << 16, dtype=torch.uint8)),
])
def test_consistent_shapes_reach_the_device_check(call):
    la.load_library()
    with pytest.raises(ValueError, match="CUDA"):
        call()


# A tensor whose shape, dtype or size disagrees with the call is refused before
# its pointer could reach a kernel.
@pytest.mark.parametrize("call,what", [
    (lambda: la.la_forward(_cpu(1, 2, 8, 16), _cpu(1, 2, 7, 16), _cpu(1, 2, 8, 64), la.LA_FMAP_ELU1), "k"),
    (lambda: la.la_forward(_cpu(1, 2, 8, 16), _f32(1, 2, 8, 16), _cpu(1, 2, 8, 64), la.LA_FMAP_ELU1), "k"),
    (lambda: la.la_forward(_cpu(1, 2, 8, 16), _cpu(1, 2, 8, 16), _cpu(1, 2, 8, 64), la.LA_FMAP_ELU1,
                           out=_cpu(1, 2, 8, 32)), "out"),
    (lambda: la.la_forward(_cpu(1, 2, 8, 16), _cpu(1, 2, 8, 16), _cpu(1, 2, 8, 64), la.LA_FMAP_TAYLOR2,
                           s_in=_f32(1, 2, 153, 64), z_in=_f32(1, 2, 153)), "s_in"),
    (lambda: la.la_forward(_cpu(1, 2, 8, 16), _cpu(1, 2, 8, 16), _cpu(1, 2, 8, 64), la.LA_FMAP_ELU1,
                           log_decay=_cpu(1, 2, 8)), "log_decay"),
    (lambda: la.la_decode_step(_f32(2, 3, 16), _f32(2, 3, 16), _f32(2, 3, 64), _f32(2, 3, 273, 64),
                               _f32(2, 3, 273), la.LA_FMAP_TAYLOR2_SYM), "s"),
    (lambda: la.la_decode_step(_f32(2, 3, 16), _f32(2, 3, 16), _f32(2, 3, 64), _f32(2, 3, 16, 64),
                               _f32(2, 3, 16), la.LA_FMAP_ELU1, y=_f32(2, 3, 63)), "y"),
    (lambda: la.la_forward_varlen(_cpu(2, 8, 16), _cpu(2, 8, 16), _cpu(2, 9, 64),
                                  torch.tensor([0, 8], dtype=torch.int32), 8, la.LA_FMAP_ELU1), "v"),
    (lambda: la.la_swa_decode_step(_cpu(1, 2, 64), _cpu(1, 2, 64), _cpu(1, 2, 64), _cpu(1, 2, 32, 64),
                                   _cpu(1, 2, 16, 64), torch.zeros(1, dtype=torch.int32), 16), "k_cache"),
    (lambda: la.la_swa_decode_step(_cpu(1, 2, 64), _cpu(1, 2, 64), _cpu(1, 2, 64), _cpu(1, 2, 16, 64),
                                   _cpu(1, 2, 16, 64), torch.zeros(2, dtype=torch.int32), 16), "pos"),
    (lambda: la.la_backward(_cpu(1, 1, 8, 16), _cpu(1, 1, 8, 16), _cpu(1, 1, 8, 32), _cpu(1, 1, 8, 32),
                            la.LA_FMAP_ELU1, workspace=torch.zeros(16, dtype=torch.uint8)), "workspace"),
])
def test_mismatched_tensors_rejected(call, what):
    la.load_library()
    with pytest.raises(ValueError, match=what):
        call()
