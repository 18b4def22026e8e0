"""GPU parity of ra_forward_varlen (packed sequences, through the C ABI) against the fp64 oracle.

Bars as for the forward pass: bf16 max |out - ref| <= 2e-2, mean <= 2e-3, max |lse - ref| <= 1e-3;
fp32 on the CUDA cores 1e-5 for all three.  Length mixes cover sequences shorter than one tile,
ragged tiles, empty sequences and a long sequence beside many short ones.  Both kernels (tensor
cores, CUDA cores) run fused and per step (partials merged in natural packed rows)."""
import numpy as np
import pytest
import torch

import long_context_exact_forward_b200 as ra
import oracle
from long_context_exact_forward_b200 import inputs

pytestmark = pytest.mark.gpu


def run(lengths, H, D, N, causal, layout, seed, dtype=torch.bfloat16, **kw):
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    S = int(cu[-1])
    q, k, v = (x[0] for x in inputs.make_qkv(1, S, H, D, dtype=dtype, device="cuda", seed=seed))
    out, lse = ra.forward_varlen(q, k, v, cu, N, causal, layout, **kw)
    torch.cuda.synchronize()
    assert ra.get_device_status() == 0
    ref, ref_lse = oracle.attention_varlen(q[None].cpu(), k[None].cpu(), v[None].cpu(), cu, causal, threads=16)
    err = np.abs(out.float().cpu().double().numpy() - ref)
    lerr = np.abs(lse.cpu().double().numpy() - ref_lse)
    assert np.isfinite(err).all()
    if dtype == torch.float32:
        assert err.max() <= 1e-5 and lerr.max() <= 1e-5, (err.max(), lerr.max())
    else:
        assert err.max() <= 2e-2 and err.mean() <= 2e-3, (err.max(), err.mean())
        assert lerr.max() <= 1e-3, lerr.max()
    return out, lse


@pytest.mark.parametrize("layout", ["contiguous", "striped", "zigzag"])
@pytest.mark.parametrize("causal", [False, True])
def test_mixed_lengths(layout, causal):
    run([1024, 256, 4096, 512, 64], 2, 128, 4, causal, layout, seed=1)


@pytest.mark.parametrize("layout", ["contiguous", "striped", "zigzag"])
def test_short_ragged_and_empty_sequences(layout):
    run([8, 0, 600, 24, 1200, 8], 2, 64, 4, True, layout, seed=2)


def test_zigzag_one_long_among_many_short():
    run([64] * 20 + [8192] + [48] * 10 + [0], 1, 128, 8, True, "zigzag", seed=5)


def test_one_long_among_many_short():
    run([64] * 30 + [8192] + [128] * 10, 1, 128, 8, True, "striped", seed=3)


@pytest.mark.parametrize("layout", ["striped", "zigzag"])
def test_single_sequence_equals_the_batch_call(layout):
    q, k, v = inputs.make_qkv(1, 2048, 2, 128, dtype=torch.bfloat16, device="cuda", seed=4)
    a, la = ra.forward(q, k, v, 4, True, layout)
    b, lb = ra.forward_varlen(q[0], k[0], v[0], [0, 2048], 4, True, layout)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b) and torch.equal(la[0], lb)


def test_varlen_rejects_bad_arguments():
    q = torch.zeros(100, 1, 128, device="cuda", dtype=torch.bfloat16)
    with pytest.raises(ra.RAError):  # length not a multiple of n_ring
        ra.forward_varlen(q, q, q, [0, 50, 100], 4, True)
    with pytest.raises(ra.RAError):  # zigzag needs lengths divisible by 2 n_ring
        ra.forward_varlen(q, q, q, [0, 4, 100], 4, True, "zigzag")


# CUDA cores: fp32 (exact) and head dims the tensor cores do not take
@pytest.mark.parametrize("layout", ["contiguous", "striped", "zigzag"])
@pytest.mark.parametrize("causal", [False, True])
def test_cuda_cores_fp32(layout, causal):
    run([96, 0, 40, 400, 8, 200], 2, 40, 4, causal, layout, seed=6, dtype=torch.float32)


@pytest.mark.parametrize("D", [16, 64, 200])
def test_cuda_cores_fp32_head_dims(D):
    run([64, 320, 8, 0, 128], 2, D, 4, True, "zigzag", seed=7, dtype=torch.float32)


def test_cuda_cores_bf16_head_dim_outside_the_tensor_cores():
    run([256, 24, 1000, 8], 2, 96, 4, True, "striped", seed=8)  # AUTO: CUDA cores for D = 96


def test_cuda_cores_on_request_for_bf16():
    run([512, 64, 16, 0, 1280], 2, 128, 8, True, "zigzag", seed=9, kernel="simt")


# per-step launches: partial results merged in natural packed rows
@pytest.mark.parametrize("layout", ["contiguous", "striped", "zigzag"])
@pytest.mark.parametrize("steps", [1, 3])
def test_per_step_tensor_cores(layout, steps):
    run([1024, 256, 0, 2048, 512, 64], 2, 128, 4, True, layout, seed=10, variant="per_step",
        steps_per_launch=steps)


@pytest.mark.parametrize("layout", ["striped", "zigzag"])
def test_per_step_cuda_cores_fp32(layout):
    run([96, 0, 40, 400, 8, 200], 2, 40, 4, True, layout, seed=11, dtype=torch.float32, variant="per_step",
        steps_per_launch=1)


def test_per_step_non_causal_head_dim_64():
    run([64, 1024, 8, 320], 3, 64, 8, False, "contiguous", seed=12, variant="per_step", steps_per_launch=2)


def test_single_sequence_equals_the_batch_call_on_the_cuda_cores():
    q, k, v = inputs.make_qkv(1, 640, 2, 48, dtype=torch.float32, device="cuda", seed=13)
    for layout in ("contiguous", "striped", "zigzag"):
        a, la = ra.forward(q, k, v, 4, True, layout, kernel="simt")
        b, lb = ra.forward_varlen(q[0], k[0], v[0], [0, 640], 4, True, layout, kernel="simt")
        torch.cuda.synchronize()
        assert torch.equal(a[0], b) and torch.equal(la[0], lb), layout


def test_single_sequence_equals_the_batch_call_per_step():
    q, k, v = inputs.make_qkv(1, 2048, 2, 128, dtype=torch.bfloat16, device="cuda", seed=14)
    a, la = ra.forward(q, k, v, 4, True, "striped", variant="per_step", steps_per_launch=2)
    b, lb = ra.forward_varlen(q[0], k[0], v[0], [0, 2048], 4, True, "striped", variant="per_step",
                              steps_per_launch=2)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b) and torch.equal(la[0], lb)


def test_caller_workspace_per_step_and_reuse():
    lengths = [256, 0, 1024, 64]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    q, k, v = (x[0] for x in inputs.make_qkv(1, int(cu[-1]), 2, 128, dtype=torch.bfloat16, device="cuda", seed=15))
    n = ra.varlen_workspace_size(cu, 2, 128, 4, "zigzag", 1, "per_step")
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    first = ra.forward_varlen(q, k, v, cu, 4, True, "zigzag", variant="per_step", workspace=ws)
    again = ra.forward_varlen(q, k, v, cu, 4, True, "zigzag", variant="per_step", workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(first[0], again[0]) and torch.equal(first[1], again[1])
    with pytest.raises(ra.RAError):  # per-step launches need the running result: too small
        ra.forward_varlen(q, k, v, cu, 4, True, "zigzag", variant="per_step",
                          workspace=ws[:ra.varlen_workspace_size(cu, 2, 128, 4, "zigzag")])


def test_frozen_max_on_request_for_packed_sequences():
    """Packed sequences this short skip the score-bound pre-pass; on request they take it (and the
    frozen row max), with the same bars."""
    lengths = [1024, 256, 0, 2048, 512]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    q, k, v = (x[0] for x in inputs.make_qkv(1, int(cu[-1]), 2, 128, dtype=torch.bfloat16, device="cuda", seed=16))
    a, la = ra.forward_varlen(q, k, v, cu, 4, True, "striped", debug=ra.DEBUG_FROZEN_MAX)
    torch.cuda.synchronize()
    assert ra.get_device_status() == 0
    ref, ref_lse = oracle.attention_varlen(q[None].cpu(), k[None].cpu(), v[None].cpu(), cu, True, threads=16)
    err = np.abs(a.float().cpu().double().numpy() - ref)
    assert err.max() <= 2e-2 and err.mean() <= 2e-3
    assert np.abs(la.cpu().double().numpy() - ref_lse).max() <= 1e-3

