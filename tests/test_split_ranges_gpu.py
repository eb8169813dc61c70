"""GPU parity of the chunk-range split of the elu d=64 bf16 forward.

That forward cuts the chunks of all heads, in (head, chunk) order, into at
most 148 contiguous ranges, one thread block each.  A range may end inside a
head (its successor picks the head up through a carried state), cross from
one head into the next, or hold several whole heads.  The small shapes of the
other parity tests give one chunk per range, and the benchmark shape gives
ranges of 6-7 chunks inside 32-chunk heads; these shapes cover the rest:

    B=1 H=37  N=700  6 chunks per head, 222 chunks: ranges of 1-2 chunks,
                     many crossing a head boundary
    B=8 H=16  N=256  2 chunks per head, 256 chunks: ranges that hold a whole
                     head, and ranges that end and start mid-head
    B=1 H=300 N=64   one partial chunk per head, 300 chunks: ranges of 2-3
                     whole heads, each head's final state written from inside
                     a range

Outputs, denominators and final states are compared with the oracle's
recurrence (max relative L2 error per (b, h) slice <= 1e-2, the bf16 bar of
the other parity tests), also when every head starts from a given state.
"""
import pytest
import torch

import causal_kernelized_sequence_b200 as la
import workloads as W
from oracle import oracle as orc

pytestmark = pytest.mark.gpu

TOL = 1e-2
SHAPES = [(1, 37, 700), (8, 16, 256), (1, 300, 64)]


@pytest.mark.parametrize("B,H,N", SHAPES)
@pytest.mark.parametrize("from_state", [False, True])
def test_split_forward_ranges(B, H, N, from_state):
    plan = la.la_kernel_plan(0, B, H, N, 64, 64, la.LA_FMAP_ELU1, la.LA_BF16)
    assert plan == (2, ["fwd_split_state_kernel", "fwd_split_out_kernel"]), plan
    q, k, v, _ = W.random_qkv(7000 + N, B, H, N, 64, 64, fmap=W.ELU1, dtype=W.BF16, scale=0.125)
    kw, s0, z0 = {}, None, None
    if from_state:
        q0, k0, v0, _ = W.random_qkv(7100 + N, B, H, 200, 64, 64, fmap=W.ELU1, dtype=W.BF16, scale=0.125)
        _, _, s0, z0 = orc.forward_recurrent(W.ELU1, q0, k0, v0)
        s0, z0 = torch.from_numpy(s0).float(), torch.from_numpy(z0).float()
        kw = {"s_in": s0.cuda(), "z_in": z0.cuda()}
    r = la.la_forward(q.cuda(), k.cuda(), v.cuda(), W.ELU1, state=True, den=True, **kw)
    torch.cuda.synchronize()
    la.la_get_device_status()
    o_ref, den_ref, s_ref, z_ref = orc.forward_recurrent(W.ELU1, q, k, v, s0, z0)
    for name, ref in (("o", o_ref), ("den", den_ref), ("s", s_ref), ("z", z_ref)):
        err = orc.max_rel_l2(r[name].cpu(), ref)
        assert err <= TOL, (B, H, N, from_state, name, err)
