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
