"""Python access to the fp64 CPU oracle (``la_oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by the tests, by the smoke check and by the
benchmark's CPU-baseline leg, never by the library itself.  It shares no code
with the CUDA path.  Inputs are converted to float64 numpy arrays (exactly, for
fp32 and bf16 data); outputs are float64.

Every function states the passage it follows; the C source holds the loops.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

ELU1 = 0
TAYLOR2 = 1
TAYLOR2_SYM = 2   # Taylor map with symmetric second-order pairs folded (153 features for d' = 16)

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "la_oracle.c")
_SO = os.path.join(_HERE, "_build", "la_oracle.so")
_lock = threading.Lock()
_lib = None

_d = ctypes.POINTER(ctypes.c_double)
_i64 = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False) -> str:
    """Compile the oracle with gcc -O2 -fopenmp (no -ffast-math: plain IEEE fp64)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        os.makedirs(os.path.dirname(_SO), exist_ok=True)
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            I = ctypes.c_int
            lib.orc_feature_dim.argtypes = [I, I]
            lib.orc_feature_dim.restype = I
            lib.orc_phi.argtypes = [I, I, _d, _d]
            lib.orc_phi_vjp.argtypes = [I, I, _d, _d, _d]
            lib.orc_forward_brute.argtypes = [I, I, I, I, I, I, _d, _d, _d, _d, _d]
            lib.orc_forward_rows.argtypes = [I, I, I, I, _d, _d, _d, _i64, I, _d, _d]
            lib.orc_forward_recurrent.argtypes = [I, I, I, I, I, I, _d, _d, _d, _d, _d, _d, _d, _d, _d]
            lib.orc_decode_step.argtypes = [I, I, I, I, _d, _d, _d, _d, _d, _d]
            lib.orc_backward_brute.argtypes = [I, I, I, I, I, I, _d, _d, _d, _d, _d, _d, _d]
            lib.orc_forward_recurrent_decay.argtypes = [I, I, I, I, I, I] + [_d] * 10
            lib.orc_forward_brute_decay.argtypes = [I, I, I, I, I, I] + [_d] * 6
            lib.orc_decode_step_decay.argtypes = [I, I, I, I] + [_d] * 7
            lib.orc_swa_forward.argtypes = [I, I, I, I, I, I, ctypes.c_double] + [_d] * 5
            lib.orc_backward_brute_decay.argtypes = [I, I, I, I, I, I] + [_d] * 9
            lib.orc_backward_recurrent.argtypes = [I, I, I, I, I, I, _d, _d, _d, _d, _d, _d, _d]
            lib.orc_backward_recurrent_decay.argtypes = [I, I, I, I, I, I] + [_d] * 9
            for f in (lib.orc_phi, lib.orc_phi_vjp, lib.orc_forward_brute, lib.orc_forward_rows,
                      lib.orc_forward_recurrent, lib.orc_decode_step, lib.orc_backward_brute,
                      lib.orc_backward_recurrent, lib.orc_forward_recurrent_decay,
                      lib.orc_forward_brute_decay, lib.orc_decode_step_decay, lib.orc_swa_forward,
                      lib.orc_backward_brute_decay, lib.orc_backward_recurrent_decay):
                f.restype = None
            _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    """Exact conversion of a torch tensor / array to contiguous float64."""
    if hasattr(x, "detach"):
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _p(a):
    return None if a is None else a.ctypes.data_as(_d)


def feature_dim(fmap: int, dqk: int) -> int:
    return _load().orc_feature_dim(fmap, dqk)


def phi(fmap: int, x) -> np.ndarray:
    """Feature map of each row of x[..., dqk] (elu(x)+1, or the BASED Taylor
    map of Knowl 3 with the scaling inside phi)."""
    x = _f64(x)
    dqk = x.shape[-1]
    F = feature_dim(fmap, dqk)
    rows = x.reshape(-1, dqk)
    out = np.empty((rows.shape[0], F))
    lib = _load()
    for r in range(rows.shape[0]):
        xr = np.ascontiguousarray(rows[r])
        o = np.empty(F)
        lib.orc_phi(fmap, dqk, _p(xr), _p(o))
        out[r] = o
    return out.reshape(*x.shape[:-1], F)


def phi_vjp(fmap: int, x, dphi) -> np.ndarray:
    """J_phi(x)^T dphi for each row."""
    x = _f64(x)
    dphi = _f64(dphi)
    dqk = x.shape[-1]
    F = feature_dim(fmap, dqk)
    xr = x.reshape(-1, dqk)
    dr = dphi.reshape(-1, F)
    out = np.empty_like(xr)
    lib = _load()
    for r in range(xr.shape[0]):
        a = np.ascontiguousarray(xr[r]); b = np.ascontiguousarray(dr[r]); o = np.empty(dqk)
        lib.orc_phi_vjp(fmap, dqk, _p(a), _p(b), _p(o))
        out[r] = o
    return out.reshape(x.shape)


def forward_brute(fmap: int, q, k, v):
    """Masked parallel form (Knowl 3, eq. for y_i), O(N^2).  Returns (o, den)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, dqk = q.shape
    dv = v.shape[-1]
    o = np.empty((B, H, N, dv))
    den = np.empty((B, H, N))
    _load().orc_forward_brute(fmap, B, H, N, dqk, dv, _p(q), _p(k), _p(v), _p(o), _p(den))
    return o, den


def forward_rows(fmap: int, q, k, v, rows):
    """Brute-force outputs at positions ``rows`` of one [N, D] slice.
    Returns (o_rows [len(rows), dv], den_rows)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    N, dqk = q.shape
    dv = v.shape[-1]
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    o = np.empty((len(r), dv))
    den = np.empty(len(r))
    _load().orc_forward_rows(fmap, N, dqk, dv, _p(q), _p(k), _p(v),
                             r.ctypes.data_as(_i64), len(r), _p(o), _p(den))
    return o, den


def forward_recurrent(fmap: int, q, k, v, s0=None, z0=None):
    """Recurrent form (Knowl 3, eqs. for s_i, z_i, y_i), optionally from a
    given state.  Returns (o, den, s_final [B,H,F,dv], z_final [B,H,F])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, dqk = q.shape
    dv = v.shape[-1]
    F = feature_dim(fmap, dqk)
    s0 = None if s0 is None else _f64(s0)
    z0 = None if z0 is None else _f64(z0)
    o = np.empty((B, H, N, dv))
    den = np.empty((B, H, N))
    s = np.empty((B, H, F, dv))
    z = np.empty((B, H, F))
    _load().orc_forward_recurrent(fmap, B, H, N, dqk, dv, _p(q), _p(k), _p(v), _p(s0), _p(z0),
                                  _p(o), _p(den), _p(s), _p(z))
    return o, den, s, z


def forward_varlen(fmap: int, q, k, v, cu_seqlens, s0=None, z0=None):
    """A batch of sequences of different lengths packed along the token axis:
    q, k [H, T, dqk], v [H, T, dv], sequence n holding tokens
    cu_seqlens[n] .. cu_seqlens[n+1] - 1 of every head.  Each sequence runs
    the recurrence of Knowl 3 on its own (from zero, or from s0[n], z0[n]);
    nothing crosses a boundary.  Returns (o [H,T,dv], den [H,T],
    s_final [nseq,H,F,dv], z_final [nseq,H,F]); an empty sequence returns its
    starting state."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    H, T, dqk = q.shape
    dv = v.shape[-1]
    F = feature_dim(fmap, dqk)
    cu = [int(c) for c in np.asarray(cu_seqlens).reshape(-1)]
    nseq = len(cu) - 1
    assert cu[0] == 0 and cu[-1] == T and all(a <= b for a, b in zip(cu[:-1], cu[1:]))
    s0 = None if s0 is None else _f64(s0)
    z0 = None if z0 is None else _f64(z0)
    o = np.zeros((H, T, dv))
    den = np.zeros((H, T))
    s = np.zeros((nseq, H, F, dv)) if s0 is None else s0.copy()
    z = np.zeros((nseq, H, F)) if z0 is None else z0.copy()
    for n in range(nseq):
        a, b = cu[n], cu[n + 1]
        if b == a:
            continue
        on, dn, sn, zn = forward_recurrent(fmap, q[None, :, a:b], k[None, :, a:b], v[None, :, a:b],
                                           None if s0 is None else s0[n:n + 1],
                                           None if z0 is None else z0[n:n + 1])
        o[:, a:b], den[:, a:b], s[n], z[n] = on[0], dn[0], sn[0], zn[0]
    return o, den, s, z


def forward_recurrent_decay(fmap: int, q, k, v, g, s0=None, z0=None):
    """Gated recurrent form: a_i = exp(g_i) per token (g [B,H,N]) multiplies
    the state before token i is added (the gated update of the reader
    comments on the 'Transformers are RNNs' discussion page; the BASED page's
    input-dependent decay, Knowl 10).  Returns (o, den, s_final, z_final)."""
    q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(g)
    B, H, N, dqk = q.shape
    dv = v.shape[-1]
    F = feature_dim(fmap, dqk)
    assert g.shape == (B, H, N)
    s0 = None if s0 is None else _f64(s0)
    z0 = None if z0 is None else _f64(z0)
    o = np.empty((B, H, N, dv))
    den = np.empty((B, H, N))
    s = np.empty((B, H, F, dv))
    z = np.empty((B, H, F))
    _load().orc_forward_recurrent_decay(fmap, B, H, N, dqk, dv, _p(q), _p(k), _p(v), _p(g), _p(s0), _p(z0),
                                        _p(o), _p(den), _p(s), _p(z))
    return o, den, s, z


def forward_brute_decay(fmap: int, q, k, v, g):
    """Gated masked form by brute force: weights
    (prod_{l=j+1..i} exp(g_l)) phi(q_i).phi(k_j) for j <= i.  Returns (o, den)."""
    q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(g)
    B, H, N, dqk = q.shape
    dv = v.shape[-1]
    o = np.empty((B, H, N, dv))
    den = np.empty((B, H, N))
    _load().orc_forward_brute_decay(fmap, B, H, N, dqk, dv, _p(q), _p(k), _p(v), _p(g), _p(o), _p(den))
    return o, den


def decode_step_decay(fmap: int, q, k, v, g, s, z):
    """One gated decode step: s <- exp(g) s + phi(k) v^T, z <- exp(g) z + phi(k),
    y = phi(q) s / phi(q) z.  g [..heads]; s, z updated in place (float64)."""
    q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(g)
    dqk, dv = q.shape[-1], v.shape[-1]
    BH = int(np.prod(q.shape[:-1]))
    assert s.dtype == np.float64 and z.dtype == np.float64 and s.flags.c_contiguous and z.flags.c_contiguous
    y = np.empty(q.shape[:-1] + (dv,))
    _load().orc_decode_step_decay(fmap, BH, dqk, dv, _p(q), _p(k), _p(v), _p(g), _p(s), _p(z), _p(y))
    return y


def swa_forward(q, k, v, window: int, scale=None):
    """Causal sliding-window softmax attention (BASED page, Knowl 4): query i
    attends to keys max(0, i-w+1) .. i with softmax weights of scale q_i.k_j,
    scale = 1/sqrt(dqk) unless given.  Returns (o [B,H,N,dv], lse [B,H,N])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, dqk = q.shape
    dv = v.shape[-1]
    scale = 1.0 / np.sqrt(dqk) if scale is None else float(scale)
    o = np.empty((B, H, N, dv))
    lse = np.empty((B, H, N))
    _load().orc_swa_forward(B, H, N, dqk, dv, int(window), scale, _p(q), _p(k), _p(v), _p(o), _p(lse))
    return o, lse


def swa_decode(q, k, v, window: int):
    """Decode-step outputs for tokens q [B,H,T,dqk] arriving one at a time after
    nothing: token t attends to the last min(t+1, w) keys, which is the
    sliding-window forward itself (Knowl 4: a w-token key-value cache during
    generation holds exactly those keys)."""
    return swa_forward(q, k, v, window)[0]


def backward_brute_decay(fmap: int, q, k, v, g, dout):
    """Gradients (dq, dk, dv, dg) of the gated forward by brute force: the
    chain rule through the gated masked form, with dg_l the sum over the pairs
    j < l <= i of dL/dw_ij w_ij (g_l scales each such weight)."""
    q, k, v, g, dout = _f64(q), _f64(k), _f64(v), _f64(g), _f64(dout)
    B, H, N, dqk = q.shape
    dv = v.shape[-1]
    dq = np.empty_like(q); dk = np.empty_like(k); dvv = np.empty_like(v); dg = np.empty_like(g)
    _load().orc_backward_brute_decay(fmap, B, H, N, dqk, dv, _p(q), _p(k), _p(v), _p(g), _p(dout),
                                     _p(dq), _p(dk), _p(dvv), _p(dg))
    return dq, dk, dvv, dg


def backward_recurrent_decay(fmap: int, q, k, v, g, dout):
    """The gated gradients (dq, dk, dv, dg) by a forward scan of the gated
    state (dq) and a backward scan of the gated R (dk, dv); dg from the
    per-token dL/dB_m = phi(q_m).dphiq_m - phi(k_m).dphik_m, summed from the
    end.  O(N F dv) per slice, for the full-size workloads."""
    q, k, v, g, dout = _f64(q), _f64(k), _f64(v), _f64(g), _f64(dout)
    B, H, N, dqk = q.shape
    dv = v.shape[-1]
    dq = np.empty_like(q); dk = np.empty_like(k); dvv = np.empty_like(v); dg = np.empty_like(g)
    _load().orc_backward_recurrent_decay(fmap, B, H, N, dqk, dv, _p(q), _p(k), _p(v), _p(g), _p(dout),
                                         _p(dq), _p(dk), _p(dvv), _p(dg))
    return dq, dk, dvv, dg


def decode_step(fmap: int, q, k, v, s, z):
    """One recurrent step on the state (s, z), updated in place (float64
    arrays [BH,F,dv] / [BH,F]); output from the updated state (Knowl 5)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    dqk = q.shape[-1]
    dv = v.shape[-1]
    BH = q.size // dqk
    assert s.dtype == np.float64 and s.flags.c_contiguous and z.dtype == np.float64 and z.flags.c_contiguous
    y = np.empty(q.shape[:-1] + (dv,))
    _load().orc_decode_step(fmap, BH, dqk, dv, _p(q), _p(k), _p(v), _p(s), _p(z), _p(y))
    return y


def backward_brute(fmap: int, q, k, v, dout):
    """Gradients of the Knowl 3 parallel form (hand-derived), O(N^2).
    Returns (dq, dk, dv)."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, H, N, dqk = q.shape
    dv = v.shape[-1]
    dq = np.empty_like(q); dk = np.empty_like(k); dvv = np.empty_like(v)
    _load().orc_backward_brute(fmap, B, H, N, dqk, dv, _p(q), _p(k), _p(v), _p(dout),
                               _p(dq), _p(dk), _p(dvv))
    return dq, dk, dvv


def backward_recurrent(fmap: int, q, k, v, dout):
    """Same gradients by a forward scan (dq) and a reverse scan (dk, dv)."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, H, N, dqk = q.shape
    dv = v.shape[-1]
    dq = np.empty_like(q); dk = np.empty_like(k); dvv = np.empty_like(v)
    _load().orc_backward_recurrent(fmap, B, H, N, dqk, dv, _p(q), _p(k), _p(v), _p(dout),
                                   _p(dq), _p(dk), _p(dvv))
    return dq, dk, dvv


def max_rel_l2(x, ref, slice_dims: int = 2) -> float:
    """Max over leading ``slice_dims`` indices (the (b,h) slices) of
    ||x - ref||_2 / ||ref||_2."""
    x = _f64(x)
    ref = _f64(ref)
    lead = int(np.prod(ref.shape[:slice_dims])) if slice_dims else 1
    xr = x.reshape(lead, -1)
    rr = ref.reshape(lead, -1)
    num = np.sqrt(((xr - rr) ** 2).sum(axis=1))
    den = np.sqrt((rr ** 2).sum(axis=1))
    den = np.where(den == 0, 1.0, den)
    return float((num / den).max()) if lead else 0.0
