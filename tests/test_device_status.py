"""Device-side failure detection: a bounded wait that runs out is reported
through the status word, and the context stays usable afterwards.  The wait
is on an mbarrier that nothing arrives on, with a 2 ms limit; no fault, trap
or unbounded wait is involved."""
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_timeout_reported_and_cleared_then_context_usable():
    import causal_kernelized_sequence_b200 as la
    from oracle import oracle as orc
    import workloads as W
    la.load_library()
    la.la_get_device_status()                      # clean slate
    la.la_selftest_bounded_wait(2000)
    with pytest.raises(la.LAError) as e:
        la.la_get_device_status()
    assert e.value.status == 4                     # LA_ERR_TIMEOUT
    la.la_get_device_status()                      # cleared by the read
    # the context still runs the path correctly
    q, k, v = W.random_qkv(11, 1, 2, 300, 64, 64, fmap=W.ELU1, dtype=W.BF16, scale=0.125)[:3]
    dev = torch.device("cuda", 0)
    y = la.la_forward(q.to(dev), k.to(dev), v.to(dev), W.ELU1)["o"].float().cpu()
    la.la_get_device_status()
    ref = orc.forward_recurrent(W.ELU1, q, k, v)[0]
    assert orc.max_rel_l2(y, ref) <= 1e-2


def test_operand_off_the_current_device_refused_before_launch():
    """A q that is not memory of the current device (here pageable host
    memory, which the device cannot address) is refused with
    LA_ERR_INVALID_ARG by the C entry point itself, before any launch; the
    same call with device memory then runs."""
    import ctypes
    import numpy as np
    import causal_kernelized_sequence_b200 as la
    lib = la.load_library()
    dev = torch.device("cuda", 0)
    B, H, N, D = 1, 2, 64, 64
    host_q = np.zeros(B * H * N * D, dtype=np.float32)          # pageable host memory
    k = torch.zeros(B, H, N, D, dtype=torch.float32, device=dev)
    v = torch.zeros_like(k)
    o = torch.empty_like(k)
    g = [torch.empty_like(k) for _ in range(3)]
    ws = torch.empty(B * H * N * 2, dtype=torch.float32, device=dev)
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    for call in (
        lambda q: lib.la_forward(q, P(k), P(v), P(o), None, None, None, None, 0, B, H, N, D, D, 0, 0, stream),
        lambda q: lib.la_backward(q, P(k), P(v), P(v), P(g[0]), P(g[1]), P(g[2]), P(ws), ws.numel() * 4,
                                  B, H, N, D, D, 0, 0, stream),
        lambda q: lib.la_swa_forward(q, P(k), P(v), P(o), None, B, H, N, D, D, 64, 0, stream),
    ):
        assert call(ctypes.c_void_p(host_q.ctypes.data)) == 1    # LA_ERR_INVALID_ARG
    torch.cuda.synchronize()
    la.la_get_device_status()
    q = torch.zeros_like(k)
    r = la.la_forward(q, k, v, 0)
    torch.cuda.synchronize()
    la.la_get_device_status()
    assert torch.isfinite(r["o"].float()).all()
