"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle.

Metric: max over (b,h) slices of ||x - x_ref||_2 / ||x_ref||_2 (decode: per
step over the heads compared).  Bars: <= 1e-5 for fp32 I/O, <= 1e-2 for bf16
I/O with fp32 accumulation, gradients included.  For bf16 the oracle runs on
the bf16-rounded inputs, so only the GPU's internal rounding is measured.
"""
import numpy as np
import pytest
import torch

import causal_kernelized_sequence_b200 as la
import workloads as W
from oracle import oracle as orc

pytestmark = pytest.mark.gpu

TOL = {W.F32: 1e-5, W.BF16: 1e-2}
ELU1, TAYLOR2, TAYLOR2_SYM = W.ELU1, W.TAYLOR2, W.TAYLOR2_SYM
DEV = "cuda"

NS = [1, 2, 15, 16, 17, 63, 64, 65, 127, 128, 129, 257, 1000]
DIMS = [(ELU1, 32, 32), (ELU1, 64, 64), (ELU1, 128, 128), (ELU1, 16, 48), (TAYLOR2, 16, 64),
        (TAYLOR2, 4, 8), (TAYLOR2_SYM, 16, 64), (TAYLOR2_SYM, 4, 8)]


def gpu_forward(q, k, v, fmap, **kw):
    r = la.la_forward(q.to(DEV), k.to(DEV), v.to(DEV), fmap, **kw)
    torch.cuda.synchronize()
    la.la_get_device_status()
    return {n: t.cpu() for n, t in r.items()}


@pytest.mark.parametrize("dtype", [W.F32, W.BF16])
@pytest.mark.parametrize("fmap,dqk,dv", DIMS)
def test_forward_small(fmap, dqk, dv, dtype):
    for N in NS:
        q, k, v, _ = W.random_qkv(1000 + N, 2, 2, N, dqk, dv, fmap=fmap, dtype=dtype,
                                  scale=1.0 if fmap != ELU1 else dqk ** -0.5)
        r = gpu_forward(q, k, v, fmap, state=True, den=True)
        o_ref, den_ref = orc.forward_brute(fmap, q, k, v)
        _, _, s_ref, z_ref = orc.forward_recurrent(fmap, q, k, v)
        tol = TOL[dtype]
        assert orc.max_rel_l2(r["o"], o_ref) <= tol, (N, orc.max_rel_l2(r["o"], o_ref))
        assert orc.max_rel_l2(r["den"], den_ref) <= tol, N
        assert orc.max_rel_l2(r["s"], s_ref) <= tol, N
        assert orc.max_rel_l2(r["z"], z_ref) <= tol, N
        assert (r["den"] > 0).all()


FROM_STATE = [(ELU1, 64, 64, W.BF16), (ELU1, 128, 128, W.BF16), (ELU1, 16, 48, W.BF16),
              (ELU1, 32, 32, W.F32), (TAYLOR2, 16, 64, W.BF16), (TAYLOR2, 16, 64, W.F32),
              (TAYLOR2_SYM, 16, 64, W.BF16), (TAYLOR2_SYM, 16, 64, W.F32)]


def _start_state(fmap, dqk, dv, dtype, seed, B, H, skew):
    """A realistic state: the recurrence's state after 300 tokens of other
    random data (fp64), optionally with noise that breaks the symmetry of the
    Taylor pair features (S[(a,b)] != S[(b,a)])."""
    q0, k0, v0, _ = W.random_qkv(seed, B, H, 300, dqk, dv, fmap=fmap, dtype=dtype,
                                 scale=1.0 if fmap != ELU1 else dqk ** -0.5)
    _, _, s0, z0 = orc.forward_recurrent(fmap, q0, k0, v0)
    if skew:
        g = np.random.default_rng(seed)
        s0 = s0 + 0.1 * np.abs(s0).mean() * g.standard_normal(s0.shape)
    return torch.from_numpy(s0).float(), torch.from_numpy(z0).float()


@pytest.mark.parametrize("fmap,dqk,dv,dtype", FROM_STATE)
def test_forward_from_state(fmap, dqk, dv, dtype):
    """la_forward_from_state against the oracle's recurrence started from the
    same state: outputs, denominators and the final state."""
    for B, H, N in ((1, 1, 1), (1, 2, 129), (2, 3, 1000), (1, 2, 3000)):
        s0, z0 = _start_state(fmap, dqk, dv, dtype, 4000 + N, B, H, skew=fmap != ELU1)
        q, k, v, _ = W.random_qkv(5000 + N, B, H, N, dqk, dv, fmap=fmap, dtype=dtype,
                                  scale=1.0 if fmap != ELU1 else dqk ** -0.5)
        r = gpu_forward(q, k, v, fmap, state=True, den=True, s_in=s0.to(DEV), z_in=z0.to(DEV))
        o_ref, den_ref, s_ref, z_ref = orc.forward_recurrent(fmap, q, k, v, s0, z0)
        tol = TOL[dtype]
        for name, ref in (("o", o_ref), ("den", den_ref), ("s", s_ref), ("z", z_ref)):
            err = orc.max_rel_l2(r[name], ref)
            assert err <= tol, (B, H, N, name, err)


@pytest.mark.parametrize("fmap,dqk,dv,dtype", FROM_STATE)
def test_chunked_prefill_matches_one_call(fmap, dqk, dv, dtype):
    """A prompt prefilled in pieces (la_forward, then la_forward_from_state on
    the rest with the returned state) equals the one-call forward."""
    B, H, N = 2, 2, 1100
    q, k, v, _ = W.random_qkv(6000, B, H, N, dqk, dv, fmap=fmap, dtype=dtype,
                              scale=1.0 if fmap != ELU1 else dqk ** -0.5)
    o_ref, den_ref, s_ref, z_ref = orc.forward_recurrent(fmap, q, k, v)
    cuts = [0, 1, 130, 640, N]
    s = z = None
    outs, dens = [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        part = [t[:, :, a:b].contiguous() for t in (q, k, v)]
        kw = {} if s is None else {"s_in": s.to(DEV), "z_in": z.to(DEV)}
        r = gpu_forward(*part, fmap, state=True, den=True, **kw)
        outs.append(r["o"]); dens.append(r["den"]); s, z = r["s"], r["z"]
    tol = TOL[dtype]
    assert orc.max_rel_l2(torch.cat(outs, 2), o_ref) <= tol
    assert orc.max_rel_l2(torch.cat(dens, 2), den_ref) <= tol
    assert orc.max_rel_l2(s, s_ref) <= tol
    assert orc.max_rel_l2(z, z_ref) <= tol


VARLEN = [(ELU1, 64, 64, W.BF16), (ELU1, 128, 128, W.BF16), (TAYLOR2, 16, 64, W.BF16),
          (TAYLOR2_SYM, 16, 64, W.BF16), (ELU1, 16, 48, W.BF16), (ELU1, 32, 32, W.F32),
          (TAYLOR2, 16, 64, W.F32)]


def _packed(seed, lens, H, dqk, dv, fmap, dtype):
    """Packed [H, T, *] inputs for sequences of the given lengths."""
    T = int(sum(lens))
    q, k, v, _ = W.random_qkv(seed, 1, H, T, dqk, dv, fmap=fmap, dtype=dtype,
                              scale=1.0 if fmap != ELU1 else dqk ** -0.5)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    return q[0].contiguous(), k[0].contiguous(), v[0].contiguous(), cu


@pytest.mark.parametrize("fmap,dqk,dv,dtype", VARLEN)
def test_forward_varlen(fmap, dqk, dv, dtype):
    """Packed sequences of mixed lengths (empty, one token, chunk edges, a
    long one that takes several segments) against the oracle's per-sequence
    recurrence, from zero and from given states."""
    H = 3
    for lens, max_len in (([129, 0, 1, 127, 128, 1000, 300], 1000), ([5, 2000], 2048), ([1], 1)):
        q, k, v, cu = _packed(8000 + len(lens), lens, H, dqk, dv, fmap, dtype)
        nseq = len(lens)
        F = la.la_feature_dim(fmap, dqk)
        tol = TOL[dtype]
        for start in (False, True):
            kw = {}
            s0 = z0 = None
            if start:
                s0, z0 = _start_state(fmap, dqk, dv, dtype, 8100 + nseq, nseq, H, skew=fmap != ELU1)
                kw = {"s_in": s0.to(DEV), "z_in": z0.to(DEV)}
            r = la.la_forward_varlen(q.to(DEV), k.to(DEV), v.to(DEV), cu.to(DEV), max_len, fmap,
                                     state=True, den=True, **kw)
            torch.cuda.synchronize()
            la.la_get_device_status()
            o_ref, den_ref, s_ref, z_ref = orc.forward_varlen(fmap, q, k, v, cu.numpy(), s0, z0)
            o, den, s, z = (r[n].cpu() for n in ("o", "den", "s", "z"))
            for n_, (a, b) in enumerate(zip(cu[:-1].tolist(), cu[1:].tolist())):
                if b > a:
                    err = orc.max_rel_l2(o[:, a:b], o_ref[:, a:b], slice_dims=1)
                    assert err <= tol, (lens, start, n_, "o", err)
                    assert orc.max_rel_l2(den[:, a:b], den_ref[:, a:b], slice_dims=1) <= tol
                if b > a or start:
                    assert orc.max_rel_l2(s[n_], s_ref[n_], slice_dims=1) <= tol, (lens, start, n_, "s")
                    assert orc.max_rel_l2(z[n_], z_ref[n_], slice_dims=1) <= tol, (lens, start, n_, "z")
                else:
                    assert (s[n_] == 0).all() and (z[n_] == 0).all()


def test_forward_varlen_matches_fixed_length():
    """Equal lengths packed are the fixed-length batch: same bits from the
    same kernel (Taylor bf16).  A zero start state selects the one-launch
    kernel for the fixed-length call, the one the packed call runs."""
    B, H, N = 3, 2, 700
    q, k, v, _ = W.random_qkv(8200, B, H, N, 16, 64, fmap=TAYLOR2, dtype=W.BF16)
    F = la.la_feature_dim(TAYLOR2, 16)
    fixed = gpu_forward(q, k, v, TAYLOR2, state=True, den=True, s_in=torch.zeros(B, H, F, 64, device=DEV),
                        z_in=torch.zeros(B, H, F, device=DEV))
    pk = lambda t: t.permute(1, 0, 2, 3).reshape(H, B * N, t.shape[-1]).contiguous().to(DEV)
    cu = torch.arange(0, B * N + 1, N, dtype=torch.int32, device=DEV)
    r = la.la_forward_varlen(pk(q), pk(k), pk(v), cu, N, TAYLOR2, state=True, den=True)
    torch.cuda.synchronize()
    unpk = lambda t: t.cpu().reshape(H, B, N, -1).permute(1, 0, 2, 3)
    assert torch.equal(unpk(r["o"]), fixed["o"])
    assert torch.equal(r["s"].cpu().reshape(B, H, *r["s"].shape[2:]), fixed["s"])


def test_forward_varlen_bad_lengths_reported():
    """Lengths live on the device: a decreasing pair or a length above
    max_seqlen is reported through the status word, and nothing is written
    for that sequence; the context stays usable."""
    H, dqk, dv = 2, 16, 64
    q, k, v, _ = _packed(8300, [100, 100], H, dqk, dv, TAYLOR2, W.BF16)
    bad = torch.tensor([0, 150, 120], dtype=torch.int32, device=DEV)     # 150 > 120: decreasing
    o = torch.full((H, 200, dv), 7.0, dtype=torch.bfloat16, device=DEV)
    la.la_forward_varlen(q.to(DEV), k.to(DEV), v.to(DEV), bad, 150, TAYLOR2, out=o)
    torch.cuda.synchronize()
    with pytest.raises(RuntimeError, match="DEVICE_CHECK"):
        la.la_get_device_status()
    assert (o[:, 150:].float() == 7.0).all()                               # sequence 1 untouched
    long = torch.tensor([0, 190, 200], dtype=torch.int32, device=DEV)      # 190 > max_seqlen 100
    la.la_forward_varlen(q.to(DEV), k.to(DEV), v.to(DEV), long, 100, TAYLOR2, out=o)
    torch.cuda.synchronize()
    with pytest.raises(RuntimeError, match="DEVICE_CHECK"):
        la.la_get_device_status()
    ok = torch.tensor([0, 100, 200], dtype=torch.int32, device=DEV)
    r = la.la_forward_varlen(q.to(DEV), k.to(DEV), v.to(DEV), ok, 100, TAYLOR2)
    torch.cuda.synchronize()
    la.la_get_device_status()
    o_ref, _, _, _ = orc.forward_varlen(TAYLOR2, q, k, v, ok.cpu().numpy())
    assert orc.max_rel_l2(r["o"].cpu(), o_ref, slice_dims=1) <= 1e-2


def _log_gates(seed, *shape, lo=-0.5):
    """Seeded log forget gates g <= 0 (a = exp(g) in [e^lo, 1]), some exactly 0."""
    g = torch.Generator().manual_seed(seed)
    x = torch.rand(*shape, generator=g) * lo
    x[..., ::7] = 0.0
    return x


@pytest.mark.parametrize("dtype", [W.F32, W.BF16])
@pytest.mark.parametrize("fmap,dqk,dv", [(ELU1, 32, 32), (ELU1, 64, 64), (ELU1, 128, 128), (TAYLOR2, 16, 64),
                                         (TAYLOR2_SYM, 16, 64), (ELU1, 16, 48)])
def test_forward_decay(fmap, dqk, dv, dtype):
    """The gated forward against the oracle's gated recurrence, from zero and
    from a given state, with ragged lengths; and a strong gate (e^-8 per
    token) that makes the far past vanish."""
    for N, lo in ((1, -0.5), (33, -0.5), (257, -0.5), (700, -8.0)):
        q, k, v, _ = W.random_qkv(9000 + N, 2, 2, N, dqk, dv, fmap=fmap, dtype=dtype,
                                  scale=1.0 if fmap != ELU1 else dqk ** -0.5)
        g = _log_gates(9100 + N, 2, 2, N, lo=lo)
        tol = TOL[dtype]
        for start in (False, True):
            kw = {}
            s0 = z0 = None
            if start:
                s0, z0 = _start_state(fmap, dqk, dv, dtype, 9200 + N, 2, 2, skew=fmap != ELU1)
                kw = {"s_in": s0.to(DEV), "z_in": z0.to(DEV)}
            r = gpu_forward(q, k, v, fmap, state=True, den=True, log_decay=g.to(DEV), **kw)
            o_ref, den_ref, s_ref, z_ref = orc.forward_recurrent_decay(fmap, q, k, v, g, s0, z0)
            for name, ref in (("o", o_ref), ("den", den_ref), ("s", s_ref), ("z", z_ref)):
                err = orc.max_rel_l2(r[name], ref)
                assert err <= tol, (N, lo, start, name, err)


@pytest.mark.parametrize("dtype,fmap,dqk,dv", [(W.F32, ELU1, 32, 32), (W.BF16, ELU1, 64, 64),
                                               (W.BF16, TAYLOR2, 16, 64)])
def test_forward_decay_full_forgetting(dtype, fmap, dqk, dv):
    """Gates of -inf (a = 0) wipe the state: the token after one starts over.
    The oracle takes -inf exactly; the tensor-core path counts it as e^-80."""
    N = 300
    q, k, v, _ = W.random_qkv(9500, 2, 2, N, dqk, dv, fmap=fmap, dtype=dtype,
                              scale=1.0 if fmap != ELU1 else dqk ** -0.5)
    g = _log_gates(9501, 2, 2, N)
    g[..., [0, 5, 127, 128, 200]] = -float("inf")
    r = gpu_forward(q, k, v, fmap, state=True, den=True, log_decay=g.to(DEV))
    o_ref, den_ref, s_ref, _ = orc.forward_recurrent_decay(fmap, q, k, v, g)
    tol = TOL[dtype]
    assert orc.max_rel_l2(r["o"], o_ref) <= tol
    assert orc.max_rel_l2(r["den"], den_ref) <= tol
    assert orc.max_rel_l2(r["s"], s_ref) <= tol
    assert torch.isfinite(r["o"].float()).all()


@pytest.mark.parametrize("dtype", [W.F32, W.BF16])
@pytest.mark.parametrize("fmap,dqk,dv", [(ELU1, 32, 32), (ELU1, 64, 64), (ELU1, 128, 128), (TAYLOR2, 16, 64),
                                         (TAYLOR2_SYM, 16, 64), (TAYLOR2, 4, 8)])
def test_backward_decay(fmap, dqk, dv, dtype):
    """Gated gradients, the gate's included, against the oracle's brute force."""
    for N in (1, 17, 64, 65, 200):
        q, k, v, do = W.random_qkv(9950 + N, 1, 2, N, dqk, dv, fmap=fmap, dtype=dtype,
                                   scale=1.0 if fmap != ELU1 else dqk ** -0.5, with_dout=True)
        g = _log_gates(9960 + N, 1, 2, N)
        dq, dk, dvv, dg = la.la_backward_decay(q.to(DEV), k.to(DEV), v.to(DEV), g.to(DEV), do.to(DEV), fmap)
        torch.cuda.synchronize()
        la.la_get_device_status()
        rq, rk, rv, rg = orc.backward_brute_decay(fmap, q, k, v, g, do)
        tol = TOL[dtype]
        if N == 1:
            # one token: y_1 = v_1, so dq, dk and the gate gradient vanish
            assert dq.abs().max().item() <= 1e-4 and dk.abs().max().item() <= 1e-4
            assert dg.abs().max().item() <= 1e-4   # fp32 rounding of phi(k).dphi(k), exactly 0 in exact arithmetic
            assert orc.max_rel_l2(dvv.cpu(), do) <= tol
            continue
        for got, ref, name in ((dq, rq, "dq"), (dk, rk, "dk"), (dvv, rv, "dv"), (dg, rg, "dg")):
            err = orc.max_rel_l2(got.cpu(), ref)
            assert err <= tol, (N, name, err)
        assert dg[..., 0].abs().max().item() <= 1e-4 * dg.abs().max().item()   # g_1 scales an empty state


@pytest.mark.parametrize("fmap,dqk,dv", [(ELU1, 64, 64), (ELU1, 128, 128), (TAYLOR2, 16, 64), (TAYLOR2_SYM, 16, 64)])
def test_backward_decay_segments(fmap, dqk, dv):
    """The gated tensor-core backward with sequences cut into one-chunk
    segments (2 heads, up to 1000 tokens: 8 segments), so that the S and R
    increments, their gate-decayed sums and the suffix sum for dL/dg all run;
    strong gates (down to e^-2 per token) and gates of exactly 0."""
    for N, lo in ((300, -0.5), (1000, -0.05), (777, -2.0)):
        q, k, v, do = W.random_qkv(9970 + N, 1, 2, N, dqk, dv, fmap=fmap, dtype=W.BF16,
                                   scale=1.0 if fmap != ELU1 else dqk ** -0.5, with_dout=True)
        g = _log_gates(9980 + N, 1, 2, N, lo=lo)
        dq, dk, dvv, dg = la.la_backward_decay(q.to(DEV), k.to(DEV), v.to(DEV), g.to(DEV), do.to(DEV), fmap)
        torch.cuda.synchronize()
        la.la_get_device_status()
        rq, rk, rv, rg = orc.backward_brute_decay(fmap, q, k, v, g, do)
        for got, ref, name in ((dq, rq, "dq"), (dk, rk, "dk"), (dvv, rv, "dv"), (dg, rg, "dg")):
            err = orc.max_rel_l2(got.cpu(), ref)
            assert err <= 1e-2, (N, lo, name, err)
        assert (dg[..., 0] == 0).all()


def test_forward_decay_zero_gate_is_plain_forward():
    """g = 0 gives the ungated exact forward bit for bit (fp32, same kernel)."""
    q, k, v, _ = W.random_qkv(9300, 2, 3, 300, 32, 32, dtype=W.F32, scale=32 ** -0.5)
    a = gpu_forward(q, k, v, ELU1, state=True, den=True)
    b = gpu_forward(q, k, v, ELU1, state=True, den=True, log_decay=torch.zeros(2, 3, 300, device=DEV))
    for n in a:
        assert torch.equal(a[n], b[n]), n


@pytest.mark.parametrize("dtype", [W.F32, W.BF16])
@pytest.mark.parametrize("fmap,dqk,dv", [(TAYLOR2, 16, 64), (TAYLOR2_SYM, 16, 64), (ELU1, 64, 64), (ELU1, 32, 48)])
def test_decode_decay(fmap, dqk, dv, dtype):
    """Gated decode steps continue the gated forward (oracle steps from the
    oracle prefill state)."""
    P, T = 37, 20
    q, k, v, _ = W.random_qkv(9400, 3, 2, P + T, dqk, dv, fmap=fmap, dtype=dtype)
    g = _log_gates(9401, 3, 2, P + T)
    r = la.la_forward(q[:, :, :P].contiguous().to(DEV), k[:, :, :P].contiguous().to(DEV),
                      v[:, :, :P].contiguous().to(DEV), fmap, state=True, log_decay=g[:, :, :P].contiguous().to(DEV))
    s, z = r["s"], r["z"]
    _, _, s_o, z_o = orc.forward_recurrent_decay(fmap, q[:, :, :P], k[:, :, :P], v[:, :, :P], g[:, :, :P])
    s_o = np.ascontiguousarray(s_o.reshape(6, *s_o.shape[2:])); z_o = np.ascontiguousarray(z_o.reshape(6, -1))
    tol = TOL[dtype]
    for t in range(T):
        y = la.la_decode_step(q[:, :, P + t].contiguous().to(DEV), k[:, :, P + t].contiguous().to(DEV),
                              v[:, :, P + t].contiguous().to(DEV), s, z, fmap,
                              log_decay=g[:, :, P + t].contiguous().to(DEV))
        torch.cuda.synchronize()
        y_o = orc.decode_step_decay(fmap, q[:, :, P + t], k[:, :, P + t], v[:, :, P + t], g[:, :, P + t], s_o, z_o)
        err = orc.max_rel_l2(y.cpu().reshape(6, dv)[None], y_o.reshape(6, dv)[None], slice_dims=1)
        assert err <= tol, (t, err)
    la.la_get_device_status()
    assert orc.max_rel_l2(s.cpu().reshape(6, -1), s_o.reshape(6, -1), slice_dims=1) <= tol


SWA = [(W.BF16, 64, 64, 64), (W.BF16, 64, 64, 16), (W.BF16, 64, 64, 128), (W.BF16, 64, 64, 48),
       (W.BF16, 64, 64, 50), (W.F32, 32, 48, 64), (W.F32, 64, 64, 1), (W.BF16, 16, 32, 300)]


@pytest.mark.parametrize("dtype,dqk,dv,w", SWA)
def test_swa_forward(dtype, dqk, dv, w):
    """Sliding-window attention against the oracle: tensor-core tiles (bf16,
    d = 64, w a multiple of 16) with ragged tails and windows reaching before
    the sequence start, and the exact kernel for the other shapes."""
    for N in (1, 15, 127, 128, 129, 300, 1000):
        q, k, v, _ = W.random_qkv(9600 + N + w, 2, 3, N, dqk, dv, dtype=dtype)
        r = la.la_swa_forward(q.to(DEV), k.to(DEV), v.to(DEV), w, lse=True)
        torch.cuda.synchronize()
        la.la_get_device_status()
        o_ref, lse_ref = orc.swa_forward(q, k, v, w)
        tol = TOL[dtype]
        err = orc.max_rel_l2(r["o"].cpu(), o_ref)
        assert err <= tol, (N, err)
        assert orc.max_rel_l2(r["lse"].cpu(), lse_ref) <= tol, N


@pytest.mark.parametrize("dtype,dqk,dv,w", [(W.BF16, 64, 64, 64), (W.F32, 32, 48, 16)])
def test_swa_decode(dtype, dqk, dv, w):
    """Prefill, cache fill, then decode steps: each step equals the oracle's
    sliding-window forward at that position; prompts shorter and longer than
    the window, and sequences at different positions."""
    B, H, T = 2, 3, 40
    for P in (5, w + 37):
        q, k, v, _ = W.random_qkv(9700 + P, B, H, P + T, dqk, dv, dtype=dtype)
        o_ref, _ = orc.swa_forward(q, k, v, w)
        kc, vc = la.la_swa_cache_fill(k[:, :, :P].contiguous().to(DEV), v[:, :, :P].contiguous().to(DEV), w)
        pos = torch.full((B,), P, dtype=torch.int32, device=DEV)
        tol = TOL[dtype]
        for t in range(T):
            y = la.la_swa_decode_step(q[:, :, P + t].contiguous().to(DEV), k[:, :, P + t].contiguous().to(DEV),
                                      v[:, :, P + t].contiguous().to(DEV), kc, vc, pos, w)
            pos += 1
            torch.cuda.synchronize()
            err = orc.max_rel_l2(y.cpu(), o_ref[:, :, P + t])
            assert err <= tol, (P, t, err)
        la.la_get_device_status()
    # sequences at different positions in one call: sequence 1 is one token behind
    q, k, v, _ = W.random_qkv(9800, B, H, 30, dqk, dv, dtype=dtype)
    o_ref, _ = orc.swa_forward(q, k, v, w)
    kc, vc = la.la_swa_cache_fill(k[:, :, :20].contiguous().to(DEV), v[:, :, :20].contiguous().to(DEV), w)
    kc1, vc1 = la.la_swa_cache_fill(k[1:, :, :19].contiguous().to(DEV), v[1:, :, :19].contiguous().to(DEV), w)
    kc[1:], vc[1:] = kc1, vc1
    pos = torch.tensor([20, 19], dtype=torch.int32, device=DEV)
    qt = torch.stack([q[0, :, 20], q[1, :, 19]]).contiguous().to(DEV)
    kt = torch.stack([k[0, :, 20], k[1, :, 19]]).contiguous().to(DEV)
    vt = torch.stack([v[0, :, 20], v[1, :, 19]]).contiguous().to(DEV)
    y = la.la_swa_decode_step(qt, kt, vt, kc, vc, pos, w).cpu()
    ref = torch.stack([torch.from_numpy(o_ref[0, :, 20]), torch.from_numpy(o_ref[1, :, 19])])
    assert orc.max_rel_l2(y, ref) <= TOL[dtype]


def test_swa_decode_bad_position_reported():
    """A negative position writes nothing and is reported; the context stays usable."""
    q, k, v, _ = W.random_qkv(9900, 1, 2, 1, 64, 64, dtype=W.BF16)
    kc = torch.full((1, 2, 64, 64), 3.0, dtype=torch.bfloat16, device=DEV)
    vc = kc.clone()
    pos = torch.tensor([-1], dtype=torch.int32, device=DEV)
    la.la_swa_decode_step(q[:, :, 0].contiguous().to(DEV), k[:, :, 0].contiguous().to(DEV),
                          v[:, :, 0].contiguous().to(DEV), kc, vc, pos, 64)
    torch.cuda.synchronize()
    with pytest.raises(RuntimeError, match="DEVICE_CHECK"):
        la.la_get_device_status()
    assert (kc.float() == 3.0).all()


@pytest.mark.parametrize("dtype", [W.F32, W.BF16])
@pytest.mark.parametrize("fmap,dqk,dv", DIMS)
def test_backward_small(fmap, dqk, dv, dtype):
    for N in (1, 17, 64, 65, 200, 300):
        q, k, v, do = W.random_qkv(2000 + N, 1, 2, N, dqk, dv, fmap=fmap, dtype=dtype,
                                   scale=1.0 if fmap != ELU1 else dqk ** -0.5, with_dout=True)
        qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
        dq, dk, dvv = la.la_backward(qd, kd, vd, dod, fmap)
        torch.cuda.synchronize()
        la.la_get_device_status()
        rq, rk, rv = orc.backward_recurrent(fmap, q, k, v, do)
        tol = TOL[dtype]
        if N == 1:
            # y_1 = v_1 whatever q and k are: dq and dk vanish exactly (the
            # relative metric is undefined there), and dv_1 = dO_1.
            assert dq.abs().max().item() <= 1e-4 and dk.abs().max().item() <= 1e-4
            assert orc.max_rel_l2(dvv.cpu(), do) <= tol
            continue
        for got, ref, name in ((dq, rq, "dq"), (dk, rk, "dk"), (dvv, rv, "dv")):
            err = orc.max_rel_l2(got.cpu(), ref)
            assert err <= tol, (N, name, err)


@pytest.mark.parametrize("dtype", [W.F32, W.BF16])
@pytest.mark.parametrize("fmap,dqk,dv", [(TAYLOR2, 16, 64), (TAYLOR2_SYM, 16, 64), (ELU1, 64, 64), (ELU1, 32, 48)])
def test_decode_small(fmap, dqk, dv, dtype):
    P, T = 37, 20
    q, k, v, _ = W.random_qkv(3000, 3, 2, P + T, dqk, dv, fmap=fmap, dtype=dtype)
    r = la.la_forward(q[:, :, :P].contiguous().to(DEV), k[:, :, :P].contiguous().to(DEV),
                      v[:, :, :P].contiguous().to(DEV), fmap, state=True)
    s, z = r["s"], r["z"]
    o_ref, _, s_ref, z_ref = orc.forward_recurrent(fmap, q, k, v)
    tol = TOL[dtype]
    for t in range(T):
        y = la.la_decode_step(q[:, :, P + t].contiguous().to(DEV), k[:, :, P + t].contiguous().to(DEV),
                              v[:, :, P + t].contiguous().to(DEV), s, z, fmap)
        err = orc.max_rel_l2(y.cpu()[None], o_ref[:, :, P + t][None], slice_dims=1)
        assert err <= tol, (t, err)
    torch.cuda.synchronize()
    la.la_get_device_status()
    assert orc.max_rel_l2(s.cpu(), s_ref) <= tol
    assert orc.max_rel_l2(z.cpu(), z_ref) <= tol


@pytest.mark.parametrize("dtype", [W.F32, W.BF16])
@pytest.mark.parametrize("fmap,dqk", [(ELU1, 64), (TAYLOR2, 16), (TAYLOR2, 3), (TAYLOR2_SYM, 16), (TAYLOR2_SYM, 3)])
def test_feature_map(fmap, dqk, dtype):
    x, _, _, _ = W.random_qkv(4000, 1, 3, 50, dqk, 8, dtype=dtype)
    phi = la.la_feature_map(x.to(DEV), fmap).cpu()
    ref = orc.phi(fmap, x)
    tol = 1e-6 if dtype == W.F32 else 4e-3
    np.testing.assert_allclose(phi.double().numpy(), ref, rtol=tol, atol=tol)


@pytest.mark.parametrize("dtype", [W.F32, W.BF16])
def test_folded_state_is_folded_full_state(dtype):
    # The two Taylor maps give the same outputs; the folded state's pair row is
    # (S[a,b] + S[b,a]) / sqrt(2) of the 273-row state, its square rows S[a,a].
    q, k, v, _ = W.random_qkv(7000, 2, 3, 700, 16, 64, fmap=TAYLOR2, dtype=dtype)
    full = gpu_forward(q, k, v, TAYLOR2, state=True, den=True)
    sym = gpu_forward(q, k, v, TAYLOR2_SYM, state=True, den=True)
    tol = TOL[dtype]
    assert orc.max_rel_l2(sym["o"].double(), full["o"].double()) <= tol
    assert orc.max_rel_l2(sym["den"], full["den"]) <= tol
    d = 16
    sf = full["s"].double()
    rows = [sf[:, :, :1 + d]] + [sf[:, :, 1 + d + a * d + a][:, :, None] for a in range(d)]
    rows += [((sf[:, :, 1 + d + a * d + b] + sf[:, :, 1 + d + b * d + a]) / 2 ** 0.5)[:, :, None]
             for a in range(d) for b in range(a + 1, d)]
    assert orc.max_rel_l2(sym["s"], torch.cat(rows, 2)) <= tol


def test_forward_deterministic():
    q, k, v, _ = W.random_qkv(5000, 2, 4, 777, 16, 64, fmap=TAYLOR2, dtype=W.BF16)
    a = gpu_forward(q, k, v, TAYLOR2, state=True)
    b = gpu_forward(q, k, v, TAYLOR2, state=True)
    for n in a:
        assert torch.equal(a[n], b[n]), n


def _chain(sync):
    """Calls on one stream whose inputs are the previous calls' outputs:
    the split forward (its state launch reading k and v that the previous
    output launch wrote, its output launch reading q), the window prefill,
    the Taylor prefill and a run of decode steps on a resident state."""
    def step():
        if sync:
            torch.cuda.synchronize()
    q, k, v, _ = W.random_qkv(8100, 4, 8, 4096, 64, 64, dtype=W.BF16)
    q, k, v = q.to(DEV), k.to(DEV), v.to(DEV)
    o1 = la.la_forward(q, k, v, ELU1)["o"]
    step()
    o2 = la.la_forward(o1, o1, o1, ELU1)["o"]
    step()
    o3 = la.la_swa_forward(o2, o2, o2, 64)["o"]
    step()
    o4 = la.la_forward(o3, o3, o3, ELU1)["o"]
    step()
    qt, kt, vt, _ = W.random_qkv(8101, 8, 16, 2048, 16, 64, fmap=TAYLOR2, dtype=W.BF16)
    qt, kt, vt = qt.to(DEV), kt.to(DEV), vt.to(DEV)
    t1 = la.la_forward(qt, kt, vt, TAYLOR2)["o"]
    step()
    t2 = la.la_forward(qt, kt, t1, TAYLOR2)["o"]
    step()
    r = la.la_forward(qt[:, :, :1000].contiguous(), kt[:, :, :1000].contiguous(), vt[:, :, :1000].contiguous(),
                      TAYLOR2, state=True)
    s, z = r["s"], r["z"]
    ys = []
    for t in range(1000, 1016):
        step()
        ys.append(la.la_decode_step(qt[:, :, t].contiguous(), kt[:, :, t].contiguous(), vt[:, :, t].contiguous(),
                                    s, z, TAYLOR2))
    torch.cuda.synchronize()
    la.la_get_device_status()
    out = {"o1": o1, "o2": o2, "o3": o3, "o4": o4, "t1": t1, "t2": t2, "s": s, "z": z}
    out.update({f"y{i}": y for i, y in enumerate(ys)})
    return {n: x.cpu() for n, x in out.items()}


def test_back_to_back_calls_see_previous_results():
    """The tensor-core forward and decode kernels are launched as programmatic
    dependents of the kernel before them; each must wait for it before reading
    its results.  Every kernel here is deterministic, so the chain run without
    host synchronisation must match the synchronised one bit for bit."""
    a = _chain(sync=True)
    b = _chain(sync=False)
    for n in a:
        assert torch.equal(a[n], b[n]), n
