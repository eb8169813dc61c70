"""B200 causal linear attention: Python binding of the C-ABI library libla.so.

This module only marshals arguments: it checks shapes and dtypes of torch
CUDA tensors, makes their device the current one for the call, passes their
device pointers, sizes and that device's current stream to the C entry points
declared in ``include/la.h``, and raises on a non-OK status.  Every step of the computation runs in the library's CUDA kernels;
there is no CPU or PyTorch fallback, and importing the compute functions fails
loudly when the library has not been built.

Entry points (same names as the C ABI):
    la_forward(q, k, v, fmap, *, state=False, den=False, out=None, s_in=None, z_in=None,
               log_decay=None) -> dict   (la_forward / _from_state / _decay)
    la_forward_varlen(q, k, v, cu_seqlens, max_seqlen, fmap, ...) -> dict
    la_forward_noalloc(q, k, v, fmap, ...) -> dict
    la_backward(q, k, v, dout, fmap) -> (dq, dk, dv)
    la_backward_decay(q, k, v, log_decay, dout, fmap) -> (dq, dk, dv, dlog_decay)
    la_decode_step(q, k, v, s, z, fmap, y=None, log_decay=None) -> y   (s, z in place)
    la_swa_forward(q, k, v, window, *, out=None, lse=False) -> dict
    la_swa_cache_fill(k, v, window) -> (k_cache, v_cache)
    la_swa_decode_step(q, k, v, k_cache, v_cache, pos, window, y=None) -> y
    la_feature_map(x, fmap) -> phi
    la_feature_dim(fmap, dqk) -> int
    la_get_device_status() -> None (raises on a recorded device error)
    la_selftest_bounded_wait(wait_us) -> None (a wait that runs out, on purpose)
"""
from __future__ import annotations

import ctypes
import os

import torch

LA_FMAP_ELU1 = 0
LA_FMAP_TAYLOR2 = 1
LA_FMAP_TAYLOR2_SYM = 2
LA_F32 = 0
LA_BF16 = 1

STATUS_NAMES = {0: "LA_OK", 1: "LA_ERR_INVALID_ARG", 2: "LA_ERR_UNSUPPORTED", 3: "LA_ERR_CUDA",
                4: "LA_ERR_TIMEOUT", 5: "LA_ERR_DEVICE_CHECK", 6: "LA_ERR_SCRATCH_LIMIT"}

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_build", "libla.so")
_lib = None


class LAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


def load_library(path: str | None = None):
    """Load libla.so (built by ``causal_kernelized_sequence_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise ImportError(f"libla.so not built ({path}); run python -m causal_kernelized_sequence_b200.build")
    lib = ctypes.CDLL(path)
    vp, sz, i, i64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_int64
    lib.la_version.restype = i
    lib.la_status_string.argtypes = [i]
    lib.la_status_string.restype = ctypes.c_char_p
    lib.la_feature_dim.argtypes = [i, i]
    lib.la_feature_dim.restype = i64
    lib.la_forward_workspace_bytes.argtypes = [i] * 7
    lib.la_forward_workspace_bytes.restype = sz
    lib.la_backward_workspace_bytes.argtypes = [i] * 7
    lib.la_backward_workspace_bytes.restype = sz
    lib.la_forward.argtypes = [vp] * 8 + [sz] + [i] * 7 + [vp]
    lib.la_forward.restype = i
    lib.la_backward.argtypes = [vp] * 8 + [sz] + [i] * 7 + [vp]
    lib.la_backward.restype = i
    lib.la_decode_step.argtypes = [vp] * 6 + [i] * 6 + [vp]
    lib.la_decode_step.restype = i
    lib.la_feature_map.argtypes = [vp, vp, i64, i, i, i, vp]
    lib.la_feature_map.restype = i
    lib.la_get_device_status.argtypes = [vp]
    lib.la_get_device_status.restype = i
    lib.la_forward_from_state.argtypes = [vp] * 10 + [sz] + [i] * 7 + [vp]
    lib.la_forward_from_state.restype = i
    lib.la_forward_noalloc.argtypes = [vp] * 7 + [i] * 7 + [vp]
    lib.la_forward_varlen.argtypes = [vp] * 5 + [i] * 3 + [vp] * 6 + [sz] + [i] * 5 + [vp]
    lib.la_forward_varlen.restype = i
    lib.la_forward_decay.argtypes = [vp] * 11 + [sz] + [i] * 7 + [vp]
    lib.la_forward_decay.restype = i
    lib.la_decode_step_decay.argtypes = [vp] * 7 + [i] * 6 + [vp]
    lib.la_backward_decay.argtypes = [vp] * 10 + [sz] + [i] * 7 + [vp]
    lib.la_backward_decay.restype = i
    lib.la_backward_decay_workspace_bytes.argtypes = [i] * 7
    lib.la_backward_decay_workspace_bytes.restype = sz
    lib.la_decode_step_decay.restype = i
    lib.la_forward_varlen_workspace_bytes.argtypes = [i] * 7
    lib.la_forward_varlen_workspace_bytes.restype = sz
    lib.la_forward_decay_workspace_bytes.argtypes = [i] * 7
    lib.la_forward_decay_workspace_bytes.restype = sz
    lib.la_forward_noalloc.restype = i
    lib.la_swa_forward.argtypes = [vp] * 5 + [i] * 7 + [vp]
    lib.la_swa_forward.restype = i
    lib.la_swa_cache_fill.argtypes = [vp] * 4 + [i] * 7 + [vp]
    lib.la_swa_cache_fill.restype = i
    lib.la_swa_decode_step.argtypes = [vp] * 7 + [i] * 6 + [vp]
    lib.la_swa_decode_step.restype = i
    lib.la_swa_kernel_plan.argtypes = [i] * 8 + [ctypes.c_char_p, sz]
    lib.la_swa_kernel_plan.restype = i
    lib.la_kernel_plan.argtypes = [i] * 8 + [ctypes.c_char_p, sz]
    lib.la_kernel_plan.restype = i
    lib.la_selftest_bounded_wait.argtypes = [ctypes.c_uint, vp]
    lib.la_selftest_bounded_wait.restype = i
    _lib = lib
    return lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _device(device):
    return torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)


def _call(fn, where, device, *args):
    """One library call for tensors on `device`: that device is made current
    for the call (the library launches on the current device) and its
    current stream is passed as the last argument."""
    with torch.cuda.device(device):
        stream = ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)
        _check(fn(*args, stream), where)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return LA_F32
    if t.dtype == torch.bfloat16:
        return LA_BF16
    raise TypeError(f"unsupported dtype {t.dtype}; use float32 or bfloat16")


def _check(status: int, where: str):
    if status != 0:
        raise LAError(status, where)


def _dev(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def _expect(name, t, shape, dtype, device):
    """The library sees only pointers: a tensor of another shape, dtype or
    device than the call implies would be read or written out of bounds, so
    it is refused here (None passes: the argument is optional)."""
    if t is None:
        return
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype:
        raise ValueError(f"{name}: expected {dtype} {list(shape)}, got {t.dtype} {list(t.shape)}")
    if t.device != device:
        raise ValueError(f"{name}: on {t.device}, expected {device}")


def _workspace(ws, need, device):
    """(workspace tensor, its size in bytes): a new one of `need` bytes, or the
    caller's after checking it is large enough and on the right device."""
    if ws is None:
        return (torch.empty(need, dtype=torch.uint8, device=device) if need else None), need
    if ws.device != device or not ws.is_contiguous():
        raise ValueError(f"workspace must be a contiguous tensor on {device}")
    have = ws.numel() * ws.element_size()
    if have < need:
        raise ValueError(f"workspace holds {have} bytes, the call needs {need}")
    return ws, have


def la_feature_dim(fmap: int, dqk: int) -> int:
    return int(load_library().la_feature_dim(fmap, dqk))


def la_forward_workspace_bytes(B, H, N, dqk, dv, fmap, dtype) -> int:
    return int(load_library().la_forward_workspace_bytes(B, H, N, dqk, dv, fmap, dtype))


def la_backward_workspace_bytes(B, H, N, dqk, dv, fmap, dtype) -> int:
    return int(load_library().la_backward_workspace_bytes(B, H, N, dqk, dv, fmap, dtype))


def la_forward(q, k, v, fmap, *, state=False, den=False, out=None, workspace=None, s_in=None, z_in=None,
               log_decay=None):
    """Causal linear attention forward.  q, k [B,H,N,dqk]; v [B,H,N,dv].

    With s_in [B,H,F,dv] and z_in [B,H,F] (fp32) the sequences start from that
    state (la_forward_from_state) instead of zero.  With log_decay [B,H,N]
    (fp32) the gated form runs (la_forward_decay).

    Returns {"o": [B,H,N,dv], and if requested "s": [B,H,F,dv] fp32,
    "z": [B,H,F] fp32, "den": [B,H,N] fp32}.
    """
    lib = load_library()
    B, H, N, dqk = q.shape
    dv = v.shape[-1]
    dt = _dtype_code(q)
    F = la_feature_dim(fmap, dqk)
    if (s_in is None) != (z_in is None):
        raise ValueError("s_in and z_in go together")
    _expect("k", k, (B, H, N, dqk), q.dtype, q.device)
    _expect("v", v, (B, H, N, dv), q.dtype, q.device)
    _expect("out", out, (B, H, N, dv), q.dtype, q.device)
    _expect("s_in", s_in, (B, H, F, dv), torch.float32, q.device)
    _expect("z_in", z_in, (B, H, F), torch.float32, q.device)
    _expect("log_decay", log_decay, (B, H, N), torch.float32, q.device)
    if log_decay is not None:
        wsb = int(lib.la_forward_decay_workspace_bytes(B, H, N, dqk, dv, fmap, dt))
    else:
        wsb = la_forward_workspace_bytes(B, H, N, dqk, dv, fmap, dt)
    workspace, wsb = _workspace(workspace, wsb, q.device)
    _dev(q, k, v, out, s_in, z_in, log_decay)
    o = out if out is not None else torch.empty(B, H, N, dv, dtype=q.dtype, device=q.device)
    res = {"o": o}
    if state:
        res["s"] = torch.empty(B, H, F, dv, dtype=torch.float32, device=q.device)
        res["z"] = torch.empty(B, H, F, dtype=torch.float32, device=q.device)
    if den:
        res["den"] = torch.empty(B, H, N, dtype=torch.float32, device=q.device)
    if log_decay is not None:
        _call(lib.la_forward_decay, "la_forward_decay", q.device,
              _ptr(q), _ptr(k), _ptr(v), _ptr(log_decay), _ptr(o), _ptr(s_in), _ptr(z_in), _ptr(res.get("s")),
              _ptr(res.get("z")), _ptr(res.get("den")), _ptr(workspace), wsb, B, H, N, dqk, dv, fmap, dt)
        return res
    if s_in is not None:
        _call(lib.la_forward_from_state, "la_forward_from_state", q.device,
              _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(s_in), _ptr(z_in), _ptr(res.get("s")), _ptr(res.get("z")),
              _ptr(res.get("den")), _ptr(workspace), wsb, B, H, N, dqk, dv, fmap, dt)
        return res
    _call(lib.la_forward, "la_forward", q.device,
          _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(res.get("s")), _ptr(res.get("z")), _ptr(res.get("den")),
          _ptr(workspace), wsb, B, H, N, dqk, dv, fmap, dt)
    return res


def la_forward_varlen_workspace_bytes(nseq, H, max_seqlen, dqk, dv, fmap, dtype) -> int:
    return int(load_library().la_forward_varlen_workspace_bytes(nseq, H, max_seqlen, dqk, dv, fmap, dtype))


def la_forward_varlen(q, k, v, cu_seqlens, max_seqlen, fmap, *, state=False, den=False, out=None,
                      workspace=None, s_in=None, z_in=None):
    """Forward over sequences packed along the token axis: q, k [H,T,dqk],
    v [H,T,dv]; cu_seqlens int32 [nseq+1] on the device (sequence n is tokens
    cu_seqlens[n] .. cu_seqlens[n+1]-1); max_seqlen bounds every length.

    Returns {"o": [H,T,dv], and if requested "s": [nseq,H,F,dv], "z": [nseq,H,F],
    "den": [H,T]}.  s_in/z_in [nseq,H,F,dv]/[nseq,H,F] start each sequence.
    """
    lib = load_library()
    H, T, dqk = q.shape
    dv = v.shape[-1]
    _expect("k", k, (H, T, dqk), q.dtype, q.device)
    _expect("v", v, (H, T, dv), q.dtype, q.device)
    _expect("out", out, (H, T, dv), q.dtype, q.device)
    if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1 or cu_seqlens.device != q.device:
        raise ValueError("cu_seqlens must be an int32 vector on the device of q")
    nseq = cu_seqlens.numel() - 1
    dt = _dtype_code(q)
    F = la_feature_dim(fmap, dqk)
    if (s_in is None) != (z_in is None):
        raise ValueError("s_in and z_in go together")
    _expect("s_in", s_in, (nseq, H, F, dv), torch.float32, q.device)
    _expect("z_in", z_in, (nseq, H, F), torch.float32, q.device)
    wsb = la_forward_varlen_workspace_bytes(nseq, H, min(max_seqlen, T), dqk, dv, fmap, dt)
    workspace, wsb = _workspace(workspace, wsb, q.device)
    _dev(q, k, v, out, cu_seqlens, s_in, z_in)
    o = out if out is not None else torch.empty(H, T, dv, dtype=q.dtype, device=q.device)
    res = {"o": o}
    if state:
        res["s"] = torch.empty(nseq, H, F, dv, dtype=torch.float32, device=q.device)
        res["z"] = torch.empty(nseq, H, F, dtype=torch.float32, device=q.device)
    if den:
        res["den"] = torch.empty(H, T, dtype=torch.float32, device=q.device)
    _call(lib.la_forward_varlen, "la_forward_varlen", q.device,
          _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(cu_seqlens), nseq, max_seqlen, T, _ptr(s_in), _ptr(z_in),
          _ptr(res.get("s")), _ptr(res.get("z")), _ptr(res.get("den")), _ptr(workspace), wsb, H, dqk, dv, fmap, dt)
    return res


def la_forward_noalloc(q, k, v, fmap, *, state=False, den=False, out=None):
    """la_forward without a workspace argument: the library uses its own
    built-in device scratch (for callers that cannot allocate device memory;
    calls must not overlap on the GPU).  Outputs are allocated here only if
    not given."""
    lib = load_library()
    B, H, N, dqk = q.shape
    dv = v.shape[-1]
    _expect("k", k, (B, H, N, dqk), q.dtype, q.device)
    _expect("v", v, (B, H, N, dv), q.dtype, q.device)
    _expect("out", out, (B, H, N, dv), q.dtype, q.device)
    _dev(q, k, v, out)
    dt = _dtype_code(q)
    F = la_feature_dim(fmap, dqk)
    o = out if out is not None else torch.empty(B, H, N, dv, dtype=q.dtype, device=q.device)
    res = {"o": o}
    if state:
        res["s"] = torch.empty(B, H, F, dv, dtype=torch.float32, device=q.device)
        res["z"] = torch.empty(B, H, F, dtype=torch.float32, device=q.device)
    if den:
        res["den"] = torch.empty(B, H, N, dtype=torch.float32, device=q.device)
    _call(lib.la_forward_noalloc, "la_forward_noalloc", q.device,
          _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(res.get("s")), _ptr(res.get("z")), _ptr(res.get("den")), B, H, N,
          dqk, dv, fmap, dt)
    return res


def la_backward(q, k, v, dout, fmap, *, workspace=None):
    """Gradients (dq, dk, dv) of the forward for upstream gradient dout."""
    lib = load_library()
    B, H, N, dqk = q.shape
    dv = v.shape[-1]
    _expect("k", k, (B, H, N, dqk), q.dtype, q.device)
    _expect("v", v, (B, H, N, dv), q.dtype, q.device)
    _expect("dout", dout, (B, H, N, dv), q.dtype, q.device)
    dt = _dtype_code(q)
    wsb = la_backward_workspace_bytes(B, H, N, dqk, dv, fmap, dt)
    workspace, wsb = _workspace(workspace, wsb, q.device)
    _dev(q, k, v, dout)
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dvv = torch.empty_like(v)
    _call(lib.la_backward, "la_backward", q.device,
          _ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dvv), _ptr(workspace), wsb, B, H, N, dqk,
          dv, fmap, dt)
    return dq, dk, dvv


def la_backward_decay(q, k, v, log_decay, dout, fmap, *, workspace=None):
    """Gradients (dq, dk, dv, dlog_decay) of the gated forward (la_forward with
    log_decay) for upstream gradient dout."""
    lib = load_library()
    B, H, N, dqk = q.shape
    dv = v.shape[-1]
    _expect("k", k, (B, H, N, dqk), q.dtype, q.device)
    _expect("v", v, (B, H, N, dv), q.dtype, q.device)
    _expect("dout", dout, (B, H, N, dv), q.dtype, q.device)
    _expect("log_decay", log_decay, (B, H, N), torch.float32, q.device)
    dt = _dtype_code(q)
    wsb = int(lib.la_backward_decay_workspace_bytes(B, H, N, dqk, dv, fmap, dt))
    workspace, wsb = _workspace(workspace, wsb, q.device)
    _dev(q, k, v, dout, log_decay)
    dq, dk, dvv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dg = torch.empty(B, H, N, dtype=torch.float32, device=q.device)
    _call(lib.la_backward_decay, "la_backward_decay", q.device,
          _ptr(q), _ptr(k), _ptr(v), _ptr(log_decay), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dvv), _ptr(dg),
          _ptr(workspace), wsb, B, H, N, dqk, dv, fmap, dt)
    return dq, dk, dvv, dg


def la_decode_step(q, k, v, s, z, fmap, y=None, log_decay=None):
    """One recurrent step: q, k [B,H,dqk]; v [B,H,dv]; s [B,H,F,dv] and
    z [B,H,F] fp32 updated in place.  Returns y [B,H,dv].  With log_decay
    [B,H] fp32 the state is first multiplied by exp(log_decay)
    (la_decode_step_decay)."""
    lib = load_library()
    B, H, dqk = q.shape
    dv = v.shape[-1]
    F = la_feature_dim(fmap, dqk)
    _expect("k", k, (B, H, dqk), q.dtype, q.device)
    _expect("v", v, (B, H, dv), q.dtype, q.device)
    _expect("s", s, (B, H, F, dv), torch.float32, q.device)
    _expect("z", z, (B, H, F), torch.float32, q.device)
    _expect("y", y, (B, H, dv), q.dtype, q.device)
    _expect("log_decay", log_decay, (B, H), torch.float32, q.device)
    _dev(q, k, v, s, z, y, log_decay)
    dt = _dtype_code(q)
    if y is None:
        y = torch.empty(B, H, dv, dtype=q.dtype, device=q.device)
    if log_decay is not None:
        _call(lib.la_decode_step_decay, "la_decode_step_decay", q.device,
              _ptr(q), _ptr(k), _ptr(v), _ptr(log_decay), _ptr(y), _ptr(s), _ptr(z), B, H, dqk, dv, fmap, dt)
        return y
    _call(lib.la_decode_step, "la_decode_step", q.device,
          _ptr(q), _ptr(k), _ptr(v), _ptr(y), _ptr(s), _ptr(z), B, H, dqk, dv, fmap, dt)
    return y


def la_swa_forward(q, k, v, window, *, out=None, lse=False):
    """Causal sliding-window softmax attention (query i attends to keys
    max(0, i-w+1) .. i).  q, k [B,H,N,dqk]; v [B,H,N,dv].
    Returns {"o": [B,H,N,dv], and if requested "lse": [B,H,N] fp32}."""
    lib = load_library()
    B, H, N, dqk = q.shape
    dv = v.shape[-1]
    _expect("k", k, (B, H, N, dqk), q.dtype, q.device)
    _expect("v", v, (B, H, N, dv), q.dtype, q.device)
    _expect("out", out, (B, H, N, dv), q.dtype, q.device)
    _dev(q, k, v, out)
    o = out if out is not None else torch.empty(B, H, N, dv, dtype=q.dtype, device=q.device)
    res = {"o": o}
    if lse:
        res["lse"] = torch.empty(B, H, N, dtype=torch.float32, device=q.device)
    _call(lib.la_swa_forward, "la_swa_forward", q.device,
          _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(res.get("lse")), B, H, N, dqk, dv, int(window), _dtype_code(q))
    return res


def la_swa_cache_fill(k, v, window, *, k_cache=None, v_cache=None):
    """The w-token cache of a prefill: the last min(N, w) tokens of k, v
    [B,H,N,*] in slots t mod w.  Returns (k_cache [B,H,w,dqk], v_cache [B,H,w,dv])."""
    lib = load_library()
    B, H, N, dqk = k.shape
    dv = v.shape[-1]
    window = int(window)
    _expect("v", v, (B, H, N, dv), k.dtype, k.device)
    _expect("k_cache", k_cache, (B, H, window, dqk), k.dtype, k.device)
    _expect("v_cache", v_cache, (B, H, window, dv), k.dtype, k.device)
    _dev(k, v, k_cache, v_cache)
    if k_cache is None:
        k_cache = torch.zeros(B, H, window, dqk, dtype=k.dtype, device=k.device)
    if v_cache is None:
        v_cache = torch.zeros(B, H, window, dv, dtype=v.dtype, device=v.device)
    _call(lib.la_swa_cache_fill, "la_swa_cache_fill", k.device,
          _ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache), B, H, N, dqk, dv, int(window), _dtype_code(k))
    return k_cache, v_cache


def la_swa_decode_step(q, k, v, k_cache, v_cache, pos, window, y=None):
    """One sliding-window decode step: q, k [B,H,dqk], v [B,H,dv]; the caches
    are updated in place; pos int32 [B] on the device = tokens held before
    this one (not advanced here).  Returns y [B,H,dv]."""
    lib = load_library()
    B, H, dqk = q.shape
    dv = v.shape[-1]
    window = int(window)
    _expect("k", k, (B, H, dqk), q.dtype, q.device)
    _expect("v", v, (B, H, dv), q.dtype, q.device)
    _expect("k_cache", k_cache, (B, H, window, dqk), q.dtype, q.device)
    _expect("v_cache", v_cache, (B, H, window, dv), q.dtype, q.device)
    _expect("pos", pos, (B,), torch.int32, q.device)
    _expect("y", y, (B, H, dv), q.dtype, q.device)
    _dev(q, k, v, k_cache, v_cache, pos, y)
    if y is None:
        y = torch.empty(B, H, dv, dtype=q.dtype, device=q.device)
    _call(lib.la_swa_decode_step, "la_swa_decode_step", q.device,
          _ptr(q), _ptr(k), _ptr(v), _ptr(y), _ptr(k_cache), _ptr(v_cache), _ptr(pos), B, H, dqk, dv, int(window),
          _dtype_code(q))
    return y


def la_feature_map(x, fmap):
    """Materialise phi(x) for x [..., dqk] -> [..., F] (test/baseline helper)."""
    lib = load_library()
    _dev(x)
    dqk = x.shape[-1]
    F = la_feature_dim(fmap, dqk)
    out = torch.empty(*x.shape[:-1], F, dtype=x.dtype, device=x.device)
    rows = x.numel() // dqk
    _call(lib.la_feature_map, "la_feature_map", x.device,
          _ptr(x), _ptr(out), rows, dqk, fmap, _dtype_code(x))
    return out


def la_kernel_plan(op: int, B, H, N, dqk, dv, fmap, dtype):
    """(number of kernel launches, [kernel names]) a call would make."""
    buf = ctypes.create_string_buffer(512)
    n = load_library().la_kernel_plan(op, B, H, N, dqk, dv, fmap, dtype, buf, len(buf))
    return n, [x for x in buf.value.decode().split(",") if x]


def kernel_plan(w):
    """Launches per benchmark step of a workload description (attributes
    B, H, N, dqk, dv, fmap, dtype, backward, decode_steps)."""
    if getattr(w, "window", 0):
        buf = ctypes.create_string_buffer(256)
        n = load_library().la_swa_kernel_plan(1 if w.decode_steps else 0, w.B, w.H, w.N, w.dqk, w.dv, w.window,
                                              w.dtype, buf, len(buf))
        return {"launches_per_step": n * max(1, w.decode_steps), "kernels": buf.value.decode().split(",")}
    if w.decode_steps:
        n, names = la_kernel_plan(2, w.B, w.H, 1, w.dqk, w.dv, w.fmap, w.dtype)
        return {"launches_per_step": n * w.decode_steps, "kernels": names}
    op = 3 if getattr(w, "varlen", False) else 4 if getattr(w, "decay", False) else 0
    n, names = la_kernel_plan(op, w.B, w.H, w.N, w.dqk, w.dv, w.fmap, w.dtype)
    if w.backward:
        decay = getattr(w, "decay", False)
        n2, names2 = la_kernel_plan(5 if decay else 1, w.B, w.H, w.N, w.dqk, w.dv, w.fmap, w.dtype)
        if n2 < 0:   # a gated backward outside the tensor-core shapes: the CUDA-core kernel
            n2, names2 = 1, ["bwd_simt_kernel"]
        n, names = n + n2, names + names2
    return {"launches_per_step": n, "kernels": names}


def la_get_device_status(device=None):
    """Synchronise the current stream of `device` (default: the current CUDA
    device) and raise if a kernel on that device recorded an error."""
    _call(load_library().la_get_device_status, "la_get_device_status", _device(device))


def la_selftest_bounded_wait(wait_us, device=None):
    """Enqueue the library's failure-path self-test on the current stream of
    `device` (default: the current CUDA device): a
    wait of `wait_us` microseconds on an mbarrier nobody arrives on.  The
    following la_get_device_status raises LAError(LA_ERR_TIMEOUT)."""
    _call(load_library().la_selftest_bounded_wait, "la_selftest_bounded_wait", _device(device), int(wait_us))
