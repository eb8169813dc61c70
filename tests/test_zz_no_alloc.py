"""The allocation-free forward (la_forward_noalloc) against la_forward.

la_forward_noalloc serves callers that cannot allocate device memory: it
runs the same kernels as la_forward but takes the workspace from a scratch
array built into the library instead of from the caller.  This test calls it
through the C ABI twice in a row, on two different inputs (the second call
finds the first call's data in the shared scratch), and checks each result
against la_forward given a workspace the test allocated.  Both run the same
deterministic kernels on the same stream, so the outputs must agree bit for
bit; a row that read the previous call's leftovers from the scratch would
not.  Two workspace users are covered: the split forward of elu dqk = dv = 64
(phi(K) tiles, snapshots, partial sums) and the one-launch tensor-core
forward's per-segment state increments (elu dqk = dv = 128).  It also checks
that sizes needing more scratch than the library holds are refused before
anything runs.

The file is named so that pytest collects it after every other test.
"""
import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    from causal_kernelized_sequence_b200 import build, load_library
    build.build()
    return load_library()


def _inputs(seed, B, H, N, D):
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    mk = lambda: (torch.randn(B, H, N, D, generator=g) / D ** 0.5).to(torch.bfloat16).cuda()
    return mk(), mk(), mk()


@pytest.mark.parametrize("B,H,N,D", [(4, 8, 4096, 64),     # split forward: phi(K) tiles, snapshots, partial sums
                                     (1, 4, 4096, 128)])   # one-launch forward: per-segment state increments
def test_noalloc_matches_forward_twice(lib, B, H, N, D):
    import causal_kernelized_sequence_b200 as la
    fmap, dtype = 0, 1                                     # elu, bf16
    need = lib.la_forward_workspace_bytes(B, H, N, D, D, fmap, dtype)
    assert 0 < need <= (32 << 20)
    P = lambda t: ctypes.c_void_p(None if t is None else t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for seed in (11, 12):
        q, k, v = _inputs(seed, B, H, N, D)
        ref = la.la_forward(q, k, v, fmap, state=True, den=True)
        o = torch.full_like(v, float("nan"))
        s = torch.full_like(ref["s"], float("nan"))
        z = torch.full_like(ref["z"], float("nan"))
        den = torch.full_like(ref["den"], float("nan"))
        st = lib.la_forward_noalloc(P(q), P(k), P(v), P(o), P(s), P(z), P(den), B, H, N, D, D, fmap, dtype,
                                    stream)
        assert st == 0, la.STATUS_NAMES.get(st, st)
        torch.cuda.synchronize()
        la.la_get_device_status()
        for name, got in (("o", o), ("s", s), ("z", z), ("den", den)):
            assert torch.equal(got, ref[name]), (B, H, N, D, seed, name)


def test_noalloc_rejects_sizes_beyond_scratch(lib):
    # elu bf16 B=4 H=8 N=16384 D=64 needs 48 MB of workspace > 32 MiB.
    B, H, N, D = 4, 8, 16384, 64
    assert lib.la_forward_workspace_bytes(B, H, N, D, D, 0, 1) > (32 << 20)
    P = ctypes.c_void_p
    st = lib.la_forward_noalloc(P(0x1000), P(0x2000), P(0x3000), P(0x4000), P(None), P(None), P(None),
                                B, H, N, D, D, 0, 1, None)
    assert st == 6  # LA_ERR_SCRATCH_LIMIT
    assert lib.la_status_string(6) == b"LA_ERR_SCRATCH_LIMIT"
