"""GPU parity of ra_forward_varlen (packed sequences, through the C ABI) against the fp64 oracle.

Bars as for the bf16 forward pass: max |out - ref| <= 2e-2, mean <= 2e-3, max |lse - ref| <= 1e-3.
Length mixes cover sequences shorter than one tile, ragged tiles, empty sequences and a long
sequence beside many short ones."""
import numpy as np
import pytest
import torch

import long_context_exact_forward_b200 as ra
import oracle
from long_context_exact_forward_b200 import inputs

pytestmark = pytest.mark.gpu


def run(lengths, H, D, N, causal, layout, seed):
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    S = int(cu[-1])
    q, k, v = (x[0] for x in inputs.make_qkv(1, S, H, D, dtype=torch.bfloat16, device="cuda", seed=seed))
    out, lse = ra.forward_varlen(q, k, v, cu, N, causal, layout)
    torch.cuda.synchronize()
    assert ra.get_device_status() == 0
    ref, ref_lse = oracle.attention_varlen(q[None].cpu(), k[None].cpu(), v[None].cpu(), cu, causal, threads=16)
    err = np.abs(out.float().cpu().double().numpy() - ref)
    lerr = np.abs(lse.cpu().double().numpy() - ref_lse)
    assert np.isfinite(err).all()
    assert err.max() <= 2e-2 and err.mean() <= 2e-3, (err.max(), err.mean())
    assert lerr.max() <= 1e-3, lerr.max()


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
