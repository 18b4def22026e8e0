"""ra_forward_noalloc: the forward pass for callers that cannot let the library allocate GPU
memory (code recording a CUDA graph, engines that own all device memory through their own
allocator, allocation-free hot loops).  Its scratch is one fixed device array shared by all calls
on a device.

The entry point is called through the C ABI and checked twice over: against ra_forward (the
allocating entry point) and against the fp64 oracle, within the bf16 tolerances of the other GPU
tests, on two calls in a row with different problems so that the second call reuses scratch the
first one left behind.  This file is named to be collected last.
"""
import ctypes
import os

import numpy as np
import pytest
import torch

import long_context_exact_forward_b200 as ra
import oracle
from long_context_exact_forward_b200 import inputs

pytestmark = pytest.mark.gpu

THREADS = os.cpu_count() or 1

CASES = [  # B, H, S, D, n_ring, causal, layout
    (1, 4, 4 * 1024, 128, 4, True, "striped"),
    (1, 3, 2 * 1000, 128, 2, True, "contiguous"),
    (2, 2, 8 * 256, 64, 8, False, "zigzag"),
]


def call_noalloc(q, k, v, n_ring, causal, layout):
    B, S, H, D = q.shape
    out = torch.empty_like(q)
    lse = torch.empty((B, H, S), dtype=torch.float32, device=q.device)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = ra.lib().ra_forward_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                     lse.data_ptr(), B, H, S, D, n_ring, int(causal),
                                     ra.LAYOUTS[layout], stream)
    return rc, out, lse


def assert_close_to_library(out, lse, ref, ref_lse):
    d = (out.float() - ref.float()).abs()
    assert d.max().item() <= 2e-2 and d.mean().item() <= 2e-3
    assert (lse - ref_lse).abs().max().item() <= 1e-3


def assert_close_to_oracle(q, k, v, causal, out, lse, rows=None):
    """Compare with the fp64 definition on every row, or on `rows` [B*H, n] per (b, h)."""
    B, S, H, D = q.shape
    ref, ref_lse = oracle.attention(q.cpu(), k.cpu(), v.cpu(), causal, rows=rows, threads=THREADS)
    got = out.float().cpu().permute(0, 2, 1, 3).double().numpy()  # [B, H, S, D]
    got_lse = lse.cpu().double().numpy()
    if rows is not None:
        r = np.asarray(rows).reshape(B, H, -1)
        got = np.take_along_axis(got, r[..., None], axis=2)
        got_lse = np.take_along_axis(got_lse, r, axis=2)
    err = np.abs(got - ref)
    assert err.max() <= 2e-2 and err.mean() <= 2e-3, (err.max(), err.mean())
    assert np.abs(got_lse - ref_lse).max() <= 1e-3


def test_noalloc_matches_allocating_entry_point_twice_in_a_row():
    for rep in range(2):
        for n, (B, H, S, D, N, causal, layout) in enumerate(CASES):
            q, k, v = inputs.make_qkv(B, S, H, D, torch.bfloat16, "cuda", seed=100 * rep + n)
            rc, out, lse = call_noalloc(q, k, v, N, causal, layout)
            assert rc == 0, ra.status_string(rc)
            ref, ref_lse = ra.forward(q, k, v, N, causal, layout)
            torch.cuda.synchronize()
            assert ra.get_device_status() == 0
            assert_close_to_library(out, lse, ref, ref_lse)
            assert_close_to_oracle(q, k, v, causal, out, lse)


def test_noalloc_shard_grouped_order_matches():
    """A head whose K/V exceeds L2 makes the device-built work list group items by shard."""
    q, k, v = inputs.make_qkv(1, 262144, 1, 128, torch.bfloat16, "cuda", seed=7)
    rows = inputs.sample_rows(262144, 1, 256, [0, 262143])
    for rep in range(2):
        rc, out, lse = call_noalloc(q, k, v, 16, True, "contiguous")
        assert rc == 0, ra.status_string(rc)
        ref, ref_lse = ra.forward(q, k, v, 16, True, "contiguous")
        torch.cuda.synchronize()
        assert ra.get_device_status() == 0
        assert_close_to_library(out, lse, ref, ref_lse)
        if rep == 0:
            assert_close_to_oracle(q, k, v, True, out, lse, rows=rows)


def test_noalloc_rejects_problems_beyond_its_scratch():
    # zigzag needs 3 shard-major copies: 3 x 1 x 65536 x 4 x 128 x 2 B = 192 MiB > 64 MiB
    q, k, v = inputs.make_qkv(1, 65536, 4, 128, torch.bfloat16, "cuda", seed=1)
    rc, _, _ = call_noalloc(q, k, v, 8, True, "zigzag")
    assert rc == -5  # RA_ERR_NO_WORKSPACE
    assert b"RA_NOALLOC_SCRATCH_BYTES" in ra.lib().ra_last_error_string()
    q2, k2, v2 = inputs.make_qkv(1, 256, 1, 96, torch.bfloat16, "cuda", seed=2)
    rc, _, _ = call_noalloc(q2, k2, v2, 2, True, "contiguous")
    assert rc == -4  # RA_ERR_UNSUPPORTED: head dim outside the tensor-core kernel


def test_noalloc_rejects_work_lists_beyond_its_shared_memory():
    # 8192 shards of one token pair each: 8192 items per head, but the device list builder's
    # tables (items + shards) need 64 KB of shared memory, above what it is launched with
    q, k, v = inputs.make_qkv(1, 8192 * 256, 1, 64, torch.bfloat16, "cuda", seed=3)
    ra.lib().ra_clear_last_error()
    rc, _, _ = call_noalloc(q, k, v, 8192, True, "contiguous")
    assert rc == -5  # RA_ERR_NO_WORKSPACE, before anything is enqueued
    assert b"work items" in ra.lib().ra_last_error_string()


def test_noalloc_call_replays_from_a_cuda_graph():
    # record the call once in a CUDA graph, then replay the graph on new inputs copied into the
    # same buffers; each replay matches the allocating entry point and the oracle
    B, H, S, D, N = 1, 2, 4 * 512, 128, 4
    q, k, v = inputs.make_qkv(B, S, H, D, torch.bfloat16, "cuda", seed=7)
    out = torch.empty_like(q)
    lse = torch.empty((B, H, S), dtype=torch.float32, device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        # the first call on the device looks up the scratch array; it happens before the capture
        rc = ra.lib().ra_forward_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                         lse.data_ptr(), B, H, S, D, N, 1, ra.LAYOUTS["striped"],
                                         ctypes.c_void_p(side.cuda_stream))
        assert rc == 0
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        rc = ra.lib().ra_forward_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                         lse.data_ptr(), B, H, S, D, N, 1, ra.LAYOUTS["striped"],
                                         ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    for seed in (8, 9):
        nq, nk, nv = inputs.make_qkv(B, S, H, D, torch.bfloat16, "cuda", seed=seed)
        q.copy_(nq)
        k.copy_(nk)
        v.copy_(nv)
        graph.replay()
        ref, ref_lse = ra.forward(q, k, v, N, True, "striped")
        torch.cuda.synchronize()
        assert ra.get_device_status() == 0
        assert_close_to_library(out, lse, ref, ref_lse)
        assert_close_to_oracle(q, k, v, True, out, lse)
