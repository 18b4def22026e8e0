"""GPU parity of ra_backward (through the C ABI) against the fp64 backward oracle.

The oracle differentiates the plain definition exactly (fp64, exact lse and Delta); the library
recomputes the weights from its own forward pass's out and lse in fp32.  Errors are measured
against the size of the gradient, max |ref| over the tensor, because gradient entries span
many orders of magnitude:
  fp32 path: max |g - ref| <= 1e-5 * max(1, max |ref|)
  bf16 path: max |g - ref| <= 2e-2 * max(1, max |ref|), mean |g - ref| <= 2e-3 * max(1, max |ref|)
The bf16 bounds are the forward pass's bars on the same scale; the gradients are rounded to bf16
(2^-9 relative) and Delta is formed from the bf16 forward output.
"""
import os

import numpy as np
import pytest
import torch

import long_context_exact_forward_b200 as ra
import oracle
from long_context_exact_forward_b200 import inputs

pytestmark = pytest.mark.gpu

THREADS = os.cpu_count() or 1


def grads_vs_oracle(B, H, S, D, N, causal, layout, dtype, seed=0, kernel="auto", bwd_kernel="auto"):
    q, k, v = inputs.make_qkv(B, S, H, D, dtype=dtype, device="cuda", seed=seed)
    g = torch.Generator(device="cuda").manual_seed(seed + 1000)
    dout = torch.randn((B, S, H, D), generator=g, device="cuda", dtype=torch.float32).to(dtype)
    out, lse = ra.forward(q, k, v, N, causal, layout, kernel=kernel)
    dq, dk, dv = ra.backward(q, k, v, out, lse, dout, N, causal, layout, kernel=bwd_kernel)
    torch.cuda.synchronize()
    assert ra.get_device_status() == 0
    ref = oracle.attention_backward(q.cpu(), k.cpu(), v.cpu(), dout.cpu(), causal, threads=THREADS)
    res = []
    for name, x, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        x = x.float().cpu().double().numpy()
        assert np.isfinite(x).all(), name
        scale = max(1.0, float(np.abs(r).max()))
        err = np.abs(x - r)
        if dtype == torch.float32:
            assert err.max() <= 1e-5 * scale, f"{name}: max abs error {err.max():.3g} (scale {scale:.3g})"
        else:
            assert err.max() <= 2e-2 * scale, f"{name}: max abs error {err.max():.3g} (scale {scale:.3g})"
            assert err.mean() <= 2e-3 * scale, f"{name}: mean abs error {err.mean():.3g} (scale {scale:.3g})"
        res.append((name, err.max() / scale, err.mean() / scale))
    return res


def test_toy_ring_fp32_backward():
    # the ultralytics.com toy's shape: 4 devices x 8 tokens, head dim 16, no mask
    grads_vs_oracle(1, 1, 32, 16, 4, False, "contiguous", torch.float32)


@pytest.mark.parametrize("layout", ["contiguous", "striped", "zigzag"])
@pytest.mark.parametrize("causal", [False, True])
def test_fp32_backward(layout, causal):
    grads_vs_oracle(1, 2, 512, 64, 4, causal, layout, torch.float32, seed=3)


@pytest.mark.parametrize("layout", ["contiguous", "striped", "zigzag"])
def test_bf16_backward_d128_simt(layout):
    # forward on the tensor-core path, backward on CUDA cores
    grads_vs_oracle(1, 2, 1024, 128, 4, True, layout, torch.bfloat16, seed=5, bwd_kernel="simt")


@pytest.mark.parametrize("layout", ["contiguous", "striped", "zigzag"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("D", [64, 128])
def test_bf16_backward_tensor_cores(layout, causal, D):
    grads_vs_oracle(1, 2, 1024, D, 4, causal, layout, torch.bfloat16, seed=6 + D, bwd_kernel="tc")


def test_bf16_backward_tensor_cores_ragged():
    # S_loc = 200: a ragged last 128-row tile in every shard
    grads_vs_oracle(2, 2, 600, 128, 3, True, "striped", torch.bfloat16, seed=21, bwd_kernel="tc")
    grads_vs_oracle(1, 2, 600, 64, 3, True, "contiguous", torch.bfloat16, seed=22, bwd_kernel="tc")


def test_backward_auto_and_refusals():
    # "auto" takes the tensor cores for bf16 zigzag too (through shard-major copies); they refuse
    # fp32 and head dims other than 64 and 128
    grads_vs_oracle(1, 1, 512, 128, 4, True, "zigzag", torch.bfloat16, seed=23)
    q = torch.zeros(1, 512, 1, 128, device="cuda", dtype=torch.float32)
    lse = torch.zeros(1, 1, 512, device="cuda")
    with pytest.raises(ra.RAError):
        ra.backward(q, q, q, q, lse, q, 4, True, "striped", kernel="tc")
    q = torch.zeros(1, 512, 1, 96, device="cuda", dtype=torch.bfloat16)
    with pytest.raises(ra.RAError):
        ra.backward(q, q, q, q, lse, q, 4, True, "striped", kernel="tc")


def test_ragged_tiles_and_odd_head_dim():
    # S_loc = 100 (not a multiple of the 64-row tile), D = 40 (not a multiple of 16)
    grads_vs_oracle(2, 2, 300, 40, 3, True, "striped", torch.float32, seed=7)
    grads_vs_oracle(1, 3, 300, 40, 3, False, "contiguous", torch.bfloat16, seed=8)


def test_single_token_shards():
    # S_loc = 1: every block is one token
    grads_vs_oracle(1, 1, 8, 16, 8, True, "contiguous", torch.float32, seed=9)


def test_backward_rejects_bad_arguments():
    q = torch.zeros(1, 64, 1, 256, device="cuda", dtype=torch.bfloat16)
    lse = torch.zeros(1, 1, 64, device="cuda")
    with pytest.raises(ra.RAError):  # head dim above 128
        ra.backward(q, q, q, q, lse, q, 4, True)
    q = torch.zeros(1, 63, 1, 16, device="cuda")
    lse = torch.zeros(1, 1, 63, device="cuda")
    with pytest.raises(ra.RAError):  # S not divisible by n_ring
        ra.backward(q, q, q, q, lse, q, 4, True)
