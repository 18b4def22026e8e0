"""ra_ring_step and ra_ring_finalize -- the per-device compute of a real ring -- on one B200.

The N ranks of a ring are emulated one after another in this process, each with its own local
buffers: its query shard, the key/value block it holds, and its running (O, lse).  Between steps
every rank's block moves to the next rank by a device-to-device copy, which is what an NCCL
send/recv would deliver into the receiving rank's local buffer.  No kernel waits on another.
The shards are cut from the natural-order inputs with the oracle's own layout map, and each rank's
finalised result, put back in natural order, is compared with the fp64 oracle on every row and with
ra_forward on the whole sequence.
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


def emulated_ring(q, k, v, n, causal, layout, sms_reserved=0):
    B, S, H, D = q.shape
    pos = oracle.layout_positions(S, n, layout)
    idx = [torch.from_numpy(pos[i]).cuda() for i in range(n)]
    qs = [q[:, idx[i]].contiguous() for i in range(n)]
    held = [(k[:, idx[i]].contiguous(), v[:, idx[i]].contiguous()) for i in range(n)]
    S_loc = S // n
    O = [torch.empty((B, S_loc, H, D), dtype=torch.float32, device="cuda") for _ in range(n)]
    lse = [torch.empty((B, S_loc, H), dtype=torch.float32, device="cuda") for _ in range(n)]
    ws = torch.empty(ra.ring_step_workspace_size(B, H, S, D, n, causal, layout, 1 if q.dtype == torch.bfloat16 else 0),
                     dtype=torch.uint8, device="cuda")
    for s in range(n):
        for i in range(n):
            ra.ring_step(qs[i], held[i][0], held[i][1], O[i], lse[i], n, i, s, causal, layout,
                         sms_reserved=sms_reserved, workspace=ws)
        if s + 1 < n:  # rank i receives the block rank i - 1 held
            held = [(held[(i - 1) % n][0].clone(), held[(i - 1) % n][1].clone()) for i in range(n)]
    out = torch.empty_like(q)
    lse_nat = torch.empty((B, H, S), dtype=torch.float32, device="cuda")
    for i in range(n):
        o_i, l_i = ra.ring_finalize(O[i], lse[i], dtype=q.dtype)
        assert o_i.shape == (B, S_loc, H, D) and l_i.shape == (B, H, S_loc)
        out[:, idx[i]] = o_i
        lse_nat[:, :, idx[i]] = l_i
    torch.cuda.synchronize()
    assert ra.get_device_status() == 0
    return out, lse_nat


def check_against_oracle(q, k, v, causal, out, lse, tol_max, tol_mean, tol_lse):
    ref, ref_lse = oracle.attention(q.cpu(), k.cpu(), v.cpu(), causal, threads=THREADS)
    got = out.float().cpu().permute(0, 2, 1, 3).double().numpy()
    err = np.abs(got - ref)
    lerr = np.abs(lse.cpu().double().numpy() - ref_lse)
    assert np.isfinite(got).all()
    assert err.max() <= tol_max and err.mean() <= tol_mean, (err.max(), err.mean())
    assert lerr.max() <= tol_lse, lerr.max()


BF16_CASES = [  # B, H, S, D, n, causal, layout
    (1, 2, 4 * 300, 128, 4, True, "striped"),       # ragged 128-row tiles
    (2, 1, 8 * 256, 64, 8, True, "zigzag"),
    (1, 2, 2 * 1000, 128, 2, True, "contiguous"),   # future blocks masked: nothing enqueued
    (1, 3, 4 * 384, 128, 4, False, "striped"),
    (1, 1, 16 * 40, 64, 16, True, "contiguous"),    # shards shorter than one tile
]


@pytest.mark.parametrize("B, H, S, D, n, causal, layout", BF16_CASES)
def test_ring_steps_bf16_tensor_cores(B, H, S, D, n, causal, layout):
    q, k, v = inputs.make_qkv(B, S, H, D, torch.bfloat16, "cuda", seed=S + D + n)
    out, lse = emulated_ring(q, k, v, n, causal, layout)
    check_against_oracle(q, k, v, causal, out, lse, 2e-2, 2e-3, 1e-3)
    ref, ref_lse = ra.forward(q, k, v, n, causal, layout)
    d = (out.float() - ref.float()).abs()
    assert d.max().item() <= 2e-2 and d.mean().item() <= 2e-3
    assert (lse - ref_lse).abs().max().item() <= 1e-3


def test_toy_ring_fp32_through_ring_steps():
    """The pages' toy (4 devices, block 8, head dim 16, fp32, non-causal) as four real ring ranks."""
    q, k, v = (t.cuda() for t in inputs.toy_qkv())
    out, lse = emulated_ring(q, k, v, 4, False, "contiguous")
    check_against_oracle(q, k, v, False, out, lse, 1e-5, 1e-5, 1e-5)


@pytest.mark.parametrize("layout", ["striped", "zigzag"])
def test_ring_steps_fp32_cuda_cores(layout):
    q, k, v = inputs.make_qkv(1, 4 * 40, 2, 40, torch.float32, "cuda", seed=5)
    out, lse = emulated_ring(q, k, v, 4, True, layout)
    check_against_oracle(q, k, v, True, out, lse, 1e-5, 1e-5, 1e-5)


def test_ring_step_leaves_sms_free_for_a_transfer():
    q, k, v = inputs.make_qkv(1, 4 * 512, 2, 128, torch.bfloat16, "cuda", seed=9)
    out, lse = emulated_ring(q, k, v, 4, True, "striped", sms_reserved=20)
    check_against_oracle(q, k, v, True, out, lse, 2e-2, 2e-3, 1e-3)


def test_ring_step_rejects_bad_arguments():
    q, k, v = inputs.make_qkv(1, 256, 2, 64, torch.bfloat16, "cuda", seed=1)
    O = torch.empty((1, 64, 2, 64), dtype=torch.float32, device="cuda")
    lse = torch.empty((1, 64, 2), dtype=torch.float32, device="cuda")
    qi, ki, vi = (t[:, :64].contiguous() for t in (q, k, v))
    with pytest.raises(ra.RAError):
        ra.ring_step(qi, ki, vi, O, lse, 4, 4, 0, True, "striped")  # shard out of range
    with pytest.raises(ra.RAError):
        ra.ring_step(qi, ki, vi, O, lse, 4, 0, -1, True, "striped")  # step out of range
    with pytest.raises(ra.RAError):
        ra.ring_step(qi, ki, vi, O, lse, 4, 0, 0, True, "striped", sms_reserved=100000)


def test_ring_driver_single_rank_on_the_device():
    """The host driver's default path (ra_ring_step, ra_ring_finalize) in a one-rank NCCL group."""
    import torch.distributed as dist

    from long_context_exact_forward_b200.ring import ring_attention
    q, k, v = inputs.make_qkv(1, 1024, 2, 128, torch.bfloat16, "cuda", seed=21)
    dist.init_process_group("nccl", store=dist.HashStore(), rank=0, world_size=1)
    try:
        out, lse = ring_attention(q, k, v, True, "striped")
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert out.shape == q.shape and lse.shape == (1, 2, 1024)
    check_against_oracle(q, k, v, True, out, lse, 2e-2, 2e-3, 1e-3)
