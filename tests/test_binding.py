"""Checks of the Python binding's own argument handling that need no GPU: caller-supplied output
tensors are matched against what the kernels write before any launch, and library messages are
attached to errors only when the failing call produced them."""
import numpy as np
import pytest
import torch

import long_context_exact_forward_b200 as ra

FAKE = 0x100000  # 16-byte aligned, never dereferenced: validation fails first


class FakeCuda:
    """Stands in for a CUDA tensor in the binding's host-side checks (no device is touched)."""

    def __init__(self, shape, dtype, device="cuda:0", contiguous=True):
        self.shape = torch.Size(shape)
        self.dtype = dtype
        self.device = torch.device(device)
        self.is_cuda = True
        self._contiguous = contiguous

    def is_contiguous(self):
        return self._contiguous


def test_check_out_accepts_the_written_shape_and_dtype():
    like = FakeCuda((1, 64, 2, 16), torch.bfloat16)
    ra._check_out(FakeCuda((1, 64, 2, 16), torch.bfloat16), like.shape, torch.bfloat16, "out", like)


@pytest.mark.parametrize("t", [
    FakeCuda((1, 63, 2, 16), torch.bfloat16),                     # one token short
    FakeCuda((1, 64, 2, 16), torch.float32),                      # wrong dtype
    FakeCuda((1, 64, 2, 16), torch.bfloat16, device="cuda:1"),    # another device
    FakeCuda((1, 64, 2, 16), torch.bfloat16, contiguous=False),   # strided view
])
def test_check_out_rejects_what_the_kernels_would_overrun(t):
    like = FakeCuda((1, 64, 2, 16), torch.bfloat16)
    with pytest.raises(ValueError):
        ra._check_out(t, like.shape, torch.bfloat16, "out", like)


def test_tensors_of_one_call_must_share_a_device():
    a, b = FakeCuda((4, 8), torch.bfloat16), FakeCuda((4, 8), torch.bfloat16, device="cuda:1")
    ra._check_cuda(a, FakeCuda((4, 8), torch.bfloat16))
    with pytest.raises(ValueError, match="share a device"):
        ra._check_cuda(a, b)


def test_cpu_tensors_are_refused_before_the_library():
    q = torch.zeros(1, 64, 2, 16)
    with pytest.raises(ValueError, match="CUDA"):
        ra.forward(q, q, q, n_ring=4)
    with pytest.raises(ValueError, match="CUDA"):
        ra.rope(q)


def test_plan_tiles_rejects_zero_ring_and_tile():
    with pytest.raises(ValueError):
        ra.plan_tiles(64, 0, "contiguous", True, 16)
    with pytest.raises(ValueError):
        ra.plan_tiles(64, 4, "contiguous", True, 0)


def _backward_head_dim_256():
    """ra_backward_ex with D = 256: refused with RA_ERR_UNSUPPORTED and a message, before any device call."""
    return ra.lib().ra_backward_ex(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 64, 256, 4, 1, 0,
                                   1, 0, 0, 0, None)


def test_error_detail_comes_only_from_the_failing_call():
    lib = ra.lib()
    ra._clear_error()
    rc = _backward_head_dim_256()
    with pytest.raises(ra.RAError, match="head dims above 128"):
        ra._check(rc, "ra_backward_ex")
    # the same failure again still carries its message
    ra._clear_error()
    rc = _backward_head_dim_256()
    with pytest.raises(ra.RAError, match="head dims above 128"):
        ra._check(rc, "ra_backward_ex")
    # a later failure that records no message does not carry the earlier one
    ra._clear_error()
    assert ra._last_error() == ""
    rc = lib.ra_rope(FAKE, FAKE, 1, 4, 1, 3, 0, 10000.0, 0, None)
    with pytest.raises(ra.RAError) as e:
        ra._check(rc, "ra_rope")
    assert e.value.code == -1 and "head dims" not in str(e.value)
