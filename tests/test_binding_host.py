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
