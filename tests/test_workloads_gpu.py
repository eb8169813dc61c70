"""GPU parity at the benchmark workloads' full sizes: every (b,h) slice (every
sequence and head of the packed batch, every head of every decode step) is
compared with the fp64 oracle run on the whole tensors, in the launch
configuration the benchmark times.

Metric and bars as in test_parity_gpu: max over slices of the relative L2
error, <= 1e-2 for bf16 I/O and <= 1e-5 for fp32 I/O.  The decode workloads
are checked per step over the whole [B,H,dv] output (the bar) and per (b,h)
slice of each step (to 1e-4, so that one wrong head cannot hide).

When LA_PARITY_LOG names a file, each test appends one JSON line with its
worst errors and the oracle's host seconds.
"""
import json
import os
import time

import numpy as np
import pytest
import torch

import causal_kernelized_sequence_b200 as la
import workloads as W
from oracle import oracle as orc

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _record(name, **kv):
    path = os.environ.get("LA_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"test": name, **kv}) + "\n")


class _Clock:
    """Host seconds spent in the oracle."""

    def __init__(self):
        self.s = 0.0

    def __call__(self, fn, *a, **kw):
        t0 = time.perf_counter()
        r = fn(*a, **kw)
        self.s += time.perf_counter() - t0
        return r


def _check(errs, tol):
    bad = {n: e for n, e in errs.items() if not e <= tol}
    assert not bad, (bad, tol)


def test_workload_elu_fp32_fwd():
    w = W.BY_NAME["elu_fp32_fwd"]
    q, k, v, _ = W.make_inputs(w)
    r = la.la_forward(q.to(DEV), k.to(DEV), v.to(DEV), w.fmap, den=True)
    torch.cuda.synchronize()
    la.la_get_device_status()
    assert r["o"].shape == (1, 1, 256, 32)
    o_ref, den_ref = orc.forward_brute(w.fmap, q, k, v)
    errs = {"o": orc.max_rel_l2(r["o"].cpu(), o_ref), "den": orc.max_rel_l2(r["den"].cpu(), den_ref)}
    _record("elu_fp32_fwd", slices=1, **errs)
    _check(errs, 1e-5)


def test_workload_elu_bf16_fwd():
    w = W.BY_NAME["elu_bf16_fwd"]
    q, k, v, _ = W.make_inputs(w)
    r = la.la_forward(q.to(DEV), k.to(DEV), v.to(DEV), w.fmap, den=True, state=True)
    torch.cuda.synchronize()
    la.la_get_device_status()
    clk = _Clock()
    o_ref, den_ref, s_ref, z_ref = clk(orc.forward_recurrent, w.fmap, q, k, v)
    errs = {n: orc.max_rel_l2(r[n].cpu(), ref) for n, ref in
            (("o", o_ref), ("den", den_ref), ("s", s_ref), ("z", z_ref))}
    _record("elu_bf16_fwd", slices=w.B * w.H, oracle_s=round(clk.s, 2), **errs)
    _check(errs, 1e-2)
    # brute force on sampled rows cross-checks the recurrent oracle itself
    rows = [0, 1, 63, 64, 2047, 4095]
    ob, _ = orc.forward_rows(w.fmap, q[3, 7], k[3, 7], v[3, 7], rows)
    np.testing.assert_allclose(o_ref[3, 7, rows], ob, rtol=1e-9, atol=1e-12)


def test_workload_taylor_bf16_fwd():
    w = W.BY_NAME["taylor_bf16_fwd"]
    q, k, v, _ = W.make_inputs(w)
    r = la.la_forward(q.to(DEV), k.to(DEV), v.to(DEV), w.fmap, den=True, state=True)
    torch.cuda.synchronize()
    la.la_get_device_status()
    clk = _Clock()
    o_ref, den_ref, s_ref, z_ref = clk(orc.forward_recurrent, w.fmap, q, k, v)
    errs = {n: orc.max_rel_l2(r[n].cpu(), ref) for n, ref in
            (("o", o_ref), ("den", den_ref), ("s", s_ref), ("z", z_ref))}
    _record("taylor_bf16_fwd", slices=w.B * w.H, oracle_s=round(clk.s, 2), **errs)
    _check(errs, 1e-2)
    # Taylor: den_i >= i/2 for every head (1 + s + s^2/2 >= 1/2)
    assert (r["den"].cpu() >= torch.arange(1, w.N + 1) / 2 * (1 - 1e-3)).all()


def test_workload_elu_bf16_train():
    w = W.BY_NAME["elu_bf16_train"]
    q, k, v, do = W.make_inputs(w)
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    fr = la.la_forward(qd, kd, vd, w.fmap, den=True)
    dq, dk, dvv = la.la_backward(qd, kd, vd, dod, w.fmap)
    torch.cuda.synchronize()
    la.la_get_device_status()
    clk = _Clock()
    o_ref, den_ref, _, _ = clk(orc.forward_recurrent, w.fmap, q, k, v)
    rq, rk, rv = clk(orc.backward_recurrent, w.fmap, q, k, v, do)
    errs = {n: orc.max_rel_l2(got.cpu(), ref) for n, got, ref in
            (("o", fr["o"], o_ref), ("den", fr["den"], den_ref), ("dq", dq, rq), ("dk", dk, rk), ("dv", dvv, rv))}
    _record("elu_bf16_train", slices=w.B * w.H, oracle_s=round(clk.s, 2), **errs)
    _check(errs, 1e-2)
    # any-size invariant: sum_j dv_j = sum_i dO_i per slice
    lhs = dvv.float().sum(2)
    rhs = dod.float().sum(2)
    assert ((lhs - rhs).norm() / rhs.norm()).item() < 1e-2


def test_workload_taylor_bf16_train():
    """The BASED Taylor training step at the Taylor prefill's shape: forward
    and the tensor-core backward, every head against the oracle's recurrent
    backward (the 273-feature map)."""
    w = W.BY_NAME["taylor_bf16_train"]
    q, k, v, do = W.make_inputs(w)
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    fr = la.la_forward(qd, kd, vd, w.fmap, den=True)
    dq, dk, dvv = la.la_backward(qd, kd, vd, dod, w.fmap)
    torch.cuda.synchronize()
    la.la_get_device_status()
    clk = _Clock()
    o_ref, den_ref, _, _ = clk(orc.forward_recurrent, w.fmap, q, k, v)
    rq, rk, rv = clk(orc.backward_recurrent, w.fmap, q, k, v, do)
    errs = {n: orc.max_rel_l2(got.cpu(), ref) for n, got, ref in
            (("o", fr["o"], o_ref), ("den", fr["den"], den_ref), ("dq", dq, rq), ("dk", dk, rk), ("dv", dvv, rv))}
    _record("taylor_bf16_train", slices=w.B * w.H, oracle_s=round(clk.s, 2), **errs)
    _check(errs, 1e-2)
    lhs = dvv.float().sum(2)
    rhs = dod.float().sum(2)
    assert ((lhs - rhs).norm() / rhs.norm()).item() < 1e-2


def test_workload_elu_bf16_decay_train():
    """The gated training step on the headline shape: gated forward and the
    gated tensor-core backward, every head against the oracle's gated scans
    (dq, dk, dv and dL/dg)."""
    w = W.BY_NAME["elu_bf16_decay_train"]
    q, k, v, do = W.make_inputs(w)
    g = W.make_gates(w)
    qd, kd, vd, dod, gd = (t.to(DEV) for t in (q, k, v, do, g))
    fr = la.la_forward(qd, kd, vd, w.fmap, den=True, log_decay=gd)
    dq, dk, dvv, dg = la.la_backward_decay(qd, kd, vd, gd, dod, w.fmap)
    torch.cuda.synchronize()
    la.la_get_device_status()
    clk = _Clock()
    o_ref, den_ref, _, _ = clk(orc.forward_recurrent_decay, w.fmap, q, k, v, g)
    rq, rk, rv, rg = clk(orc.backward_recurrent_decay, w.fmap, q, k, v, g, do)
    errs = {n: orc.max_rel_l2(got.cpu(), ref) for n, got, ref in
            (("o", fr["o"], o_ref), ("den", fr["den"], den_ref), ("dq", dq, rq), ("dk", dk, rk), ("dv", dvv, rv),
             ("dg", dg, rg))}
    _record("elu_bf16_decay_train", slices=w.B * w.H, oracle_s=round(clk.s, 2), **errs)
    _check(errs, 1e-2)
    assert (dg[..., 0] == 0).all()


def test_workload_elu_bf16_decay_fwd():
    w = W.BY_NAME["elu_bf16_decay_fwd"]
    q, k, v, _ = W.make_inputs(w)
    g = W.make_gates(w)
    r = la.la_forward(q.to(DEV), k.to(DEV), v.to(DEV), w.fmap, den=True, state=True, log_decay=g.to(DEV))
    torch.cuda.synchronize()
    la.la_get_device_status()
    clk = _Clock()
    o_ref, den_ref, s_ref, z_ref = clk(orc.forward_recurrent_decay, w.fmap, q, k, v, g)
    errs = {n: orc.max_rel_l2(r[n].cpu(), ref) for n, ref in
            (("o", o_ref), ("den", den_ref), ("s", s_ref), ("z", z_ref))}
    _record("elu_bf16_decay_fwd", slices=w.B * w.H, oracle_s=round(clk.s, 2), **errs)
    _check(errs, 1e-2)
    assert (r["den"] > 0).all()


def test_workload_swa_bf16_fwd():
    w = W.BY_NAME["swa_bf16_fwd"]
    q, k, v, _ = W.make_inputs(w)
    r = la.la_swa_forward(q.to(DEV), k.to(DEV), v.to(DEV), w.window, lse=True)
    torch.cuda.synchronize()
    la.la_get_device_status()
    clk = _Clock()
    o_ref, lse_ref = clk(orc.swa_forward, q, k, v, w.window)
    errs = {"o": orc.max_rel_l2(r["o"].cpu(), o_ref), "lse": orc.max_rel_l2(r["lse"].cpu(), lse_ref)}
    _record("swa_bf16_fwd", slices=w.B * w.H, oracle_s=round(clk.s, 2), **errs)
    _check(errs, 1e-2)
    assert torch.isfinite(r["o"].float()).all()


def test_workload_swa_bf16_decode():
    """The decode workload's shapes (1024 sequences x 16 heads, 64-token caches
    filled by a 64-token prompt), 128 steps (the ring of every cache wraps
    twice), every head of every step against the oracle's sliding-window
    forward over prompt + steps."""
    w = W.BY_NAME["swa_bf16_decode"]
    T = 128
    (q, k, v), (sq, sk, sv) = W.make_decode_inputs(w, steps=T)
    kc, vc = la.la_swa_cache_fill(k.to(DEV), v.to(DEV), w.window)
    pos = torch.full((w.B,), w.N, dtype=torch.int32, device=DEV)
    ys = torch.empty(T, w.B, w.H, w.dv, dtype=torch.bfloat16, device=DEV)
    sqd, skd, svd = sq.to(DEV), sk.to(DEV), sv.to(DEV)
    for t in range(T):
        ys[t] = la.la_swa_decode_step(sqd[t], skd[t], svd[t], kc, vc, pos, w.window)
        pos += 1
    torch.cuda.synchronize()
    la.la_get_device_status()
    steps_first = lambda x: x.permute(1, 2, 0, 3)          # [T,B,H,d] -> [B,H,T,d]
    qf = torch.cat([q, steps_first(sq)], 2)
    kf = torch.cat([k, steps_first(sk)], 2)
    vf = torch.cat([v, steps_first(sv)], 2)
    clk = _Clock()
    o_ref, _ = clk(orc.swa_forward, qf, kf, vf, w.window)
    got = steps_first(ys.cpu())                               # [B,H,T,dv]
    err = orc.max_rel_l2(got, o_ref[:, :, w.N:])
    _record("swa_bf16_decode", slices=w.B * w.H, steps=T, oracle_s=round(clk.s, 2), y=err)
    _check({"y": err}, 1e-2)


def test_workload_elu_bf16_varlen():
    w = W.BY_NAME["elu_bf16_varlen"]
    q, k, v, cu = W.make_varlen_inputs(w)
    lens = W.varlen_lengths(w)
    r = la.la_forward_varlen(q.to(DEV), k.to(DEV), v.to(DEV), cu.to(DEV), max(lens), w.fmap, den=True, state=True)
    torch.cuda.synchronize()
    la.la_get_device_status()
    o, den, s, z = (r[n].cpu() for n in ("o", "den", "s", "z"))
    clk = _Clock()
    o_ref, den_ref, s_ref, z_ref = clk(orc.forward_varlen, w.fmap, q, k, v, cu.numpy())
    errs = {"o": 0.0, "den": 0.0, "s": 0.0, "z": 0.0}
    for n, (a, b) in enumerate(zip(cu[:-1].tolist(), cu[1:].tolist())):
        # one slice per (sequence, head)
        errs["o"] = max(errs["o"], orc.max_rel_l2(o[:, a:b], o_ref[:, a:b], slice_dims=1))
        errs["den"] = max(errs["den"], orc.max_rel_l2(den[:, a:b], den_ref[:, a:b], slice_dims=1))
        errs["s"] = max(errs["s"], orc.max_rel_l2(s[n], s_ref[n], slice_dims=1))
        errs["z"] = max(errs["z"], orc.max_rel_l2(z[n], z_ref[n], slice_dims=1))
    _record("elu_bf16_varlen", slices=len(lens) * w.H, oracle_s=round(clk.s, 2), **errs)
    _check(errs, 1e-2)
    assert (den > 0).all()   # elu+1 features are positive: any size


@pytest.mark.parametrize("name", ["taylor_decode", "taylor_decode_sym"])
def test_workload_taylor_decode(name):
    """Prefill of 2048 tokens, then all 1024 decode steps, every one of the
    4096 heads at every step against the oracle's recurrence on the whole
    state (fp64 on the host)."""
    w = W.BY_NAME[name]
    (q, k, v), (sq, sk, sv) = W.make_decode_inputs(w)
    r = la.la_forward(q.to(DEV), k.to(DEV), v.to(DEV), w.fmap, state=True)
    s, z = r["s"], r["z"]
    torch.cuda.synchronize()
    s_pre = s.cpu()
    BH = w.B * w.H
    y_all = torch.empty(w.decode_steps, w.B, w.H, w.dv, device=DEV)
    sqd, skd, svd = sq.to(DEV), sk.to(DEV), sv.to(DEV)
    for t in range(w.decode_steps):
        la.la_decode_step(sqd[t], skd[t], svd[t], s, z, w.fmap, y=y_all[t])
    torch.cuda.synchronize()
    la.la_get_device_status()
    y_all = y_all.cpu().reshape(w.decode_steps, BH, w.dv)
    clk = _Clock()
    _, _, s_o, z_o = clk(orc.forward_recurrent, w.fmap, q, k, v)
    s_o = np.ascontiguousarray(s_o.reshape(BH, *s_o.shape[2:]))
    z_o = np.ascontiguousarray(z_o.reshape(BH, -1))
    err_pre = orc.max_rel_l2(s_pre.reshape(BH, -1), s_o.reshape(BH, -1), slice_dims=1)
    worst_step = worst_head = 0.0
    for t in range(w.decode_steps):
        y_o = clk(orc.decode_step, w.fmap, sq[t].reshape(BH, -1), sk[t].reshape(BH, -1), sv[t].reshape(BH, -1),
                  s_o, z_o)
        yt = y_all[t]
        worst_step = max(worst_step, orc.max_rel_l2(yt[None], y_o[None], slice_dims=1))
        worst_head = max(worst_head, orc.max_rel_l2(yt, y_o, slice_dims=1))
    errs = {"s_prefill": err_pre, "y_step": worst_step, "y_head": worst_head,
            "s_final": orc.max_rel_l2(s.cpu().reshape(BH, -1), s_o.reshape(BH, -1), slice_dims=1),
            "z_final": orc.max_rel_l2(z.cpu().reshape(BH, -1), z_o, slice_dims=1)}
    _record(name, slices=BH, steps=w.decode_steps, oracle_s=round(clk.s, 2), **errs)
    # the bar applies per step over the whole output; each head of each step
    # must also be right to 1e-4 (a wrong head would be off by order 1)
    _check({n: e for n, e in errs.items() if n != "y_head"}, 1e-5)
    _check({"y_head": worst_head}, 1e-4)
