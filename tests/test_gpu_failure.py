"""Failure detection without a GPU fault: every in-kernel wait of the tensor-core kernel is
bounded.  The stall knob makes the load warp issue no copies -- a flag that nothing sets -- so every
consumer wait runs out after `timeout_ns`; the kernel records RA_ERR_DEVICE_TIMEOUT in the status
word, drains, frees its tensor memory and returns.  The host reads the status, and the context
stays usable for the next call."""
import time

import numpy as np
import pytest
import torch

import long_context_exact_forward_b200 as ra
import oracle
from long_context_exact_forward_b200 import inputs

pytestmark = pytest.mark.gpu

RA_ERR_DEVICE_TIMEOUT = -7


@pytest.mark.parametrize("variant", ["fused", "per_step"])
def test_stalled_loads_time_out_and_report(variant):
    q, k, v = inputs.make_qkv(1, 4 * 256, 2, 128, torch.bfloat16, "cuda", seed=3)
    torch.cuda.synchronize()
    assert ra.get_device_status() == 0
    t0 = time.time()
    ra.forward(q, k, v, 4, True, "striped", kernel="tc", variant=variant,
               debug=ra.DEBUG_STALL_LOADS, timeout_ns=100_000_000)
    torch.cuda.synchronize()
    assert time.time() - t0 < 30
    assert ra.get_device_status() == RA_ERR_DEVICE_TIMEOUT
    assert ra.get_device_status() == 0  # reading clears the word
    # the context still works: a normal call right after is correct
    out, lse = ra.forward(q, k, v, 4, True, "striped", kernel="tc", variant=variant)
    torch.cuda.synchronize()
    assert ra.get_device_status() == 0
    ref, ref_lse = oracle.attention(q.cpu(), k.cpu(), v.cpu(), True, threads=8)
    got = out.float().cpu().permute(0, 2, 1, 3).double().numpy()
    assert np.abs(got - ref).max() <= 2e-2
    assert np.abs(lse.cpu().double().numpy() - ref_lse).max() <= 1e-3


def test_host_validation_errors_enqueue_nothing():
    q, k, v = inputs.make_qkv(1, 96, 1, 128, torch.bfloat16, "cuda", seed=1)
    with pytest.raises(ra.RAError) as e:
        ra.forward(q, k, v, 5, True, "contiguous")  # 96 % 5 != 0
    assert e.value.code == -2
    with pytest.raises(ra.RAError) as e:
        ra.forward(q, k, v, 4, True, "contiguous", kernel="tc", out=torch.empty_like(q)[:, :, :, :],
                   lse=torch.empty(1, 1, 96, device="cuda"), variant="auto",
                   workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
    assert e.value.code == -5
    q96 = q[..., :96].contiguous()
    with pytest.raises(ra.RAError) as e:
        ra.forward(q96, q96, q96, 4, True, "contiguous", kernel="tc")  # head dim 96: no tensor-core kernel
    assert e.value.code == -4
    torch.cuda.synchronize()
    assert ra.get_device_status() == 0


def test_backward_stalled_loads_time_out_and_report():
    # the tensor-core backward kernels bound their waits the same way
    q, k, v = inputs.make_qkv(1, 4 * 256, 2, 128, torch.bfloat16, "cuda", seed=4)
    out, lse = ra.forward(q, k, v, 4, True, "striped")
    dout = torch.randn_like(q)
    torch.cuda.synchronize()
    assert ra.get_device_status() == 0
    t0 = time.time()
    ra.backward(q, k, v, out, lse, dout, 4, True, "striped", kernel="tc",
                debug=ra.DEBUG_STALL_LOADS, timeout_ns=100_000_000)
    torch.cuda.synchronize()
    assert time.time() - t0 < 30
    assert ra.get_device_status() == RA_ERR_DEVICE_TIMEOUT
    assert ra.get_device_status() == 0
    # the context still works: the same backward without the knob is correct
    dq, dk, dv = ra.backward(q, k, v, out, lse, dout, 4, True, "striped", kernel="tc")
    torch.cuda.synchronize()
    assert ra.get_device_status() == 0
    ref = oracle.attention_backward(q.cpu(), k.cpu(), v.cpu(), dout.cpu(), True, threads=8)
    for x, r in zip((dq, dk, dv), ref):
        scale = max(1.0, float(np.abs(r).max()))
        assert np.abs(x.float().cpu().double().numpy() - r).max() <= 2e-2 * scale
