"""GPU parity: the CUDA library (through its C ABI) against the fp64 oracle, element by element.

Tolerances (fixed for the method):
  fp32 path:  max |out - ref| <= 1e-5, max |lse - ref| <= 1e-5
  bf16 path:  max |out - ref| <= 2e-2, mean |out - ref| <= 2e-3, max |lse - ref| <= 1e-3
The oracle sees the exact values handed to the GPU (bf16 -> fp64 is exact), so input rounding is
never counted as error.
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
TOL = {
    torch.float32: dict(max=1e-5, mean=1e-5, lse=1e-5),
    torch.bfloat16: dict(max=2e-2, mean=2e-3, lse=1e-3),
}


def compare(out, lse, ref_out, ref_lse, dtype, rows=None):
    """out [B, S, H, D] (GPU), lse [B, H, S]; ref_* from oracle.attention ([B, H, n, D], [B, H, n])."""
    o = out.float().cpu().permute(0, 2, 1, 3).double().numpy()  # [B, H, S, D]
    l = lse.cpu().double().numpy()
    if rows is not None:
        o = np.stack([np.stack([o[b, h, rows[h]] for h in range(o.shape[1])]) for b in range(o.shape[0])])
        l = np.stack([np.stack([l[b, h, rows[h]] for h in range(l.shape[1])]) for b in range(l.shape[0])])
    err = np.abs(o - ref_out)
    lerr = np.abs(l - ref_lse)
    t = TOL[dtype]
    assert np.isfinite(o).all() and np.isfinite(l).all()
    assert err.max() <= t["max"], f"max abs error {err.max():.3g}"
    assert err.mean() <= t["mean"], f"mean abs error {err.mean():.3g}"
    assert lerr.max() <= t["lse"], f"lse error {lerr.max():.3g}"
    return err.max(), err.mean(), lerr.max()


def run_case(B, H, S, D, N, causal, layout, dtype, variant, kernel="auto", seed=0, qscale=1.0):
    q, k, v = inputs.make_qkv(B, S, H, D, dtype=dtype, device="cuda", seed=seed, scale=qscale)
    out, lse = ra.forward(q, k, v, N, causal, layout, variant=variant, kernel=kernel)
    torch.cuda.synchronize()
    assert ra.get_device_status() == 0
    ref_out, ref_lse = oracle.attention(q.cpu(), k.cpu(), v.cpu(), causal, threads=THREADS)
    return compare(out, lse, ref_out, ref_lse, dtype)


# ---------------------------------------------------------------- the toy ring (fp32)
@pytest.mark.parametrize("variant", ["fused", "per_step"])
def test_toy_ring_fp32(variant):
    q, k, v = (t.cuda() for t in inputs.toy_qkv())
    out, lse = ra.forward(q, k, v, 4, causal=False, layout="contiguous", variant=variant)
    ref_out, ref_lse = oracle.attention(q.cpu(), k.cpu(), v.cpu(), False)
    compare(out, lse, ref_out, ref_lse, torch.float32)
    # the page's own check: allclose to the full softmax at atol 1e-5
    qq, kk, vv = (t.reshape(32, 16).cpu() for t in (q, k, v))
    full = torch.softmax(qq @ kk.T / 4.0, -1) @ vv
    assert torch.allclose(out.reshape(32, 16).cpu(), full, atol=1e-5)


# ---------------------------------------------------------------- SIMT kernel, fp32 and bf16
SIMT_SHAPES = [(1, 2, 3 * 40, 16, 3), (2, 1, 2 * 38, 64, 2), (1, 1, 4 * 50, 128, 4), (1, 2, 2 * 34, 256, 2),
               (1, 1, 1, 8, 1), (1, 1, 2 * 18, 5, 2)]


@pytest.mark.parametrize("shape", SIMT_SHAPES)
@pytest.mark.parametrize("layout", ["contiguous", "striped", "zigzag"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("variant", ["fused", "per_step"])
def test_simt_fp32(shape, layout, causal, variant):
    B, H, S, D, N = shape
    if layout == "zigzag" and S % (2 * N):
        pytest.skip("zigzag needs S % 2N == 0")
    run_case(B, H, S, D, N, causal, layout, torch.float32, variant, kernel="simt", seed=S + D)


# several 64-key tiles per ring step and a ragged last tile: the pipelined CUDA-core form (rows of
# whole 16-byte vectors) prefetches the next tile across tile and step boundaries; D = 200 (fp32)
# takes its single-stage form, D = 256 (bf16) two stages at 210 KB of shared memory, D = 20 (fp32)
# and D = 36 (bf16) the synchronous form
SIMT_MULTI_TILE = [(1, 2, 4 * 300, 64, 4, torch.float32), (1, 1, 2 * 200, 128, 2, torch.float32),
                   (1, 1, 2 * 160, 200, 2, torch.float32), (1, 2, 4 * 200, 64, 4, torch.bfloat16),
                   (1, 1, 2 * 264, 128, 2, torch.bfloat16), (1, 1, 2 * 160, 256, 2, torch.bfloat16),
                   (1, 1, 2 * 150, 20, 2, torch.float32), (1, 1, 2 * 150, 36, 2, torch.bfloat16)]


@pytest.mark.parametrize("shape", SIMT_MULTI_TILE)
@pytest.mark.parametrize("layout", ["contiguous", "striped", "zigzag"])
@pytest.mark.parametrize("causal", [False, True])
def test_simt_multi_tile(shape, layout, causal):
    B, H, S, D, N, dtype = shape
    run_case(B, H, S, D, N, causal, layout, dtype, "fused", kernel="simt", seed=S + 3 * D)


@pytest.mark.parametrize("layout", ["contiguous", "striped", "zigzag"])
@pytest.mark.parametrize("variant", ["fused", "per_step"])
def test_simt_bf16_odd_head_dim(layout, variant):
    run_case(1, 2, 4 * 66, 96, 4, True, layout, torch.bfloat16, variant, seed=5)


# ---------------------------------------------------------------- tcgen05 kernel, bf16
TC_SHAPES = [
    (1, 1, 128, 128, 1),        # one tile
    (1, 2, 2 * 384, 128, 2),    # 3 tiles per shard: one full pair + a half pair
    (1, 1, 3 * 300, 128, 3),    # ragged: 300 = 2 tiles + 44 rows
    (2, 2, 4 * 256, 64, 4),     # head dim 64
    (1, 1, 2 * 1000, 128, 2),   # ragged, several pairs
    (1, 3, 8 * 128, 128, 8),    # many shards, one tile each
    (1, 1, 2 * 40, 128, 2),     # shard shorter than a tile
]


@pytest.mark.parametrize("shape", TC_SHAPES)
@pytest.mark.parametrize("layout", ["contiguous", "striped", "zigzag"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("variant", ["fused", "per_step"])
def test_tc_bf16(shape, layout, causal, variant):
    B, H, S, D, N = shape
    if layout == "zigzag" and S % (2 * N):
        pytest.skip("zigzag needs S % 2N == 0")
    run_case(B, H, S, D, N, causal, layout, torch.bfloat16, variant, kernel="tc", seed=S * 7 + D)


@pytest.mark.parametrize("layout", ["contiguous", "striped"])
def test_tc_bf16_sharp_softmax(layout):
    """q x 4: scores up to ~40, large running-max jumps exercise the lazy O rescale."""
    run_case(1, 2, 4 * 512, 128, 4, True, layout, torch.bfloat16, "fused", kernel="tc", seed=11, qscale=4.0)


def test_tc_planted_dominant_key():
    """One key per row block dominates: the result must pick its value row."""
    B, H, S, D, N = 1, 1, 2 * 512, 128, 2
    q, k, v = inputs.make_qkv(B, S, H, D, dtype=torch.bfloat16, device="cuda", seed=3)
    k[0, 700, 0] = (q[0, 900, 0].float() * 8).to(torch.bfloat16)
    out, lse = ra.forward(q, k, v, N, True, "striped", kernel="tc")
    ref_out, ref_lse = oracle.attention(q.cpu(), k.cpu(), v.cpu(), True, threads=THREADS)
    compare(out, lse, ref_out, ref_lse, torch.bfloat16)


@pytest.mark.parametrize("kernel, dtype, D", [("tc", torch.bfloat16, 128), ("simt", torch.float32, 40)])
@pytest.mark.parametrize("layout", ["contiguous", "striped", "zigzag"])
@pytest.mark.parametrize("steps", [2, 3, 8])
def test_per_step_launches_of_several_ring_steps(kernel, dtype, D, layout, steps):
    """Each attention launch covers `steps` ring steps (the last one what remains of 8); partial
    results merge into the running one after each launch but the first."""
    B, H, S, N = 1, 2, 8 * 256, 8
    q, k, v = inputs.make_qkv(B, S, H, D, dtype=dtype, device="cuda", seed=31 + steps)
    out, lse = ra.forward(q, k, v, N, True, layout, variant="per_step", kernel=kernel, steps_per_launch=steps)
    torch.cuda.synchronize()
    assert ra.get_device_status() == 0
    ref_out, ref_lse = oracle.attention(q.cpu(), k.cpu(), v.cpu(), True, threads=THREADS)
    compare(out, lse, ref_out, ref_lse, dtype)


def test_auto_takes_launches_of_several_steps_for_a_head_beyond_l2():
    """One head of 262144 tokens: its K/V (128 MB) exceed the fused budget, so AUTO runs two
    launches of 16 ring steps and merges them."""
    B, H, S, D, N = 1, 1, 262144, 128, 32
    assert ra.steps_per_launch(S, D, N, "striped", 1, "auto") == 16
    q, k, v = inputs.make_qkv(B, S, H, D, dtype=torch.bfloat16, device="cuda", seed=41)
    out, lse = ra.forward(q, k, v, N, True, "striped")
    torch.cuda.synchronize()
    assert ra.get_device_status() == 0
    rows = inputs.sample_rows(S, H, 256, [0, S - 1, S // 2])
    ref_out, ref_lse = oracle.attention(q.cpu(), k.cpu(), v.cpu(), True, rows=rows, threads=THREADS)
    compare(out, lse, ref_out, ref_lse, torch.bfloat16, rows=rows)


def test_tc_frozen_max_with_a_late_dominant_key():
    """(RA_DEBUG_FROZEN_MAX: the pre-pass and the frozen max at a size that would not take them.)
    Norms of about 16 keep the head's score bound (qmax * kmax / sqrt(D)) within 2^32 of the first
    tile's max, so the kernel freezes each row's max after that tile.  Keys planted parallel to some
    query rows and met only in a later ring step then score up to the bound itself -- about 25
    (log2) above the frozen max -- and those rows must still come out as the exact softmax."""
    B, H, S, D, N = 1, 2, 4 * 512, 128, 4
    q, k, v = inputs.make_qkv(B, S, H, D, dtype=torch.float32, device="cuda", seed=17)
    q, k = q * 1.4, k * 1.4
    for r, late in ((2000, 1001), (1500, 1397), (2043, 2)):  # striped: key `late` is met after row r's first tile
        for h in range(H):
            k[0, late, h] = q[0, r, h] * (k[0, late, h].norm() / q[0, r, h].norm())
    q, k, v = (t.to(torch.bfloat16) for t in (q, k, v))
    # a sequence this short takes the frozen max only on request
    out, lse = ra.forward(q, k, v, N, True, "striped", kernel="tc", debug=ra.DEBUG_FROZEN_MAX)
    torch.cuda.synchronize()
    assert ra.get_device_status() == 0
    ref_out, ref_lse = oracle.attention(q.cpu(), k.cpu(), v.cpu(), True, threads=THREADS)
    compare(out, lse, ref_out, ref_lse, torch.bfloat16)
    # and without the request (no pre-pass, the exact row max on every tile) the same bars hold
    out2, lse2 = ra.forward(q, k, v, N, True, "striped", kernel="tc")
    torch.cuda.synchronize()
    compare(out2, lse2, ref_out, ref_lse, torch.bfloat16)


# ---------------------------------------------------------------- s4k: all rows
@pytest.mark.parametrize("variant", ["fused", "per_step"])
def test_s4k_all_rows(variant):
    w = inputs.WORKLOADS["s4k"]
    q, k, v = inputs.workload_qkv(w)
    out, lse = ra.forward(q, k, v, w.n_ring, True, "contiguous", variant=variant)
    torch.cuda.synchronize()
    ref_out, ref_lse = oracle.attention(q.cpu(), k.cpu(), v.cpu(), True, threads=THREADS)
    compare(out, lse, ref_out, ref_lse, torch.bfloat16)


# ---------------------------------------------------------------- layout invariance on the GPU
def test_layouts_agree():
    q, k, v = inputs.make_qkv(1, 8 * 512, 4, 128, dtype=torch.bfloat16, device="cuda", seed=21)
    outs = [ra.forward(q, k, v, 8, True, lay)[0].float() for lay in ("contiguous", "striped", "zigzag")]
    for o in outs[1:]:
        assert (o - outs[0]).abs().max().item() <= 2e-2


# ---------------------------------------------------------------- permute / merge kernels
@pytest.mark.parametrize("layout", ["contiguous", "striped", "zigzag"])
@pytest.mark.parametrize("dtype, H, D", [(torch.bfloat16, 3, 128), (torch.float32, 2, 5), (torch.bfloat16, 1, 3)])
def test_permute_roundtrip_and_index_map(layout, dtype, H, D):
    B, N, S_loc = 2, 4, 12
    S = N * S_loc
    x = torch.randn(B, S, H, D, device="cuda").to(dtype)
    y = ra.permute(x, N, layout)
    pos = torch.from_numpy(oracle.layout_positions(S, N, layout)).cuda()
    assert torch.equal(y, x[:, pos.reshape(-1)].reshape(B, N, S_loc, H, D))
    assert torch.equal(ra.unpermute(y, N, layout), x)


def test_merge_partials_matches_merge_identities():
    rows, D = 1000, 128
    g = torch.Generator(device="cuda").manual_seed(4)
    O1, O2 = (torch.randn(rows, D, device="cuda", generator=g) for _ in range(2))
    l1, l2 = (torch.randn(rows, device="cuda", generator=g) * 3 for _ in range(2))
    l1[:10] = float("-inf")
    l2[5:15] = float("-inf")
    Or, lr = O1.clone(), l1.clone()
    ra.merge_partials(Or, lr, O2, l2)
    # oracle.merge works on (m, l, un-normalised O); lse-normalised partials map to m = lse, l = 1
    m1, m2 = l1.double().cpu().numpy(), l2.double().cpu().numpy()
    one1 = np.where(np.isinf(m1), 0.0, 1.0)
    one2 = np.where(np.isinf(m2), 0.0, 1.0)
    m, l, O = oracle.merge(m1, one1, O1.double().cpu().numpy() * one1[:, None],
                           m2, one2, O2.double().cpu().numpy() * one2[:, None])
    with np.errstate(divide="ignore", invalid="ignore"):
        ref_O = np.where(l[:, None] > 0, O / l[:, None], 0.0)
        ref_lse = np.where(l > 0, m + np.log(l), -np.inf)
    got_O, got_lse = Or.double().cpu().numpy(), lr.double().cpu().numpy()
    np.testing.assert_allclose(got_O, ref_O, atol=2e-6, rtol=1e-5)
    assert np.array_equal(np.isinf(got_lse), np.isinf(ref_lse))
    fin = np.isfinite(ref_lse)
    np.testing.assert_allclose(got_lse[fin], ref_lse[fin], atol=1e-5)


def test_caller_workspace_and_events():
    B, H, S, D, N = 1, 2, 4 * 256, 128, 4
    q, k, v = inputs.make_qkv(B, S, H, D, dtype=torch.bfloat16, device="cuda", seed=9)
    for variant, layout in (("fused", "striped"), ("per_step", "zigzag")):
        n = ra.workspace_size(B, H, S, D, N, True, layout, 1, variant=variant)
        ws = torch.empty(n, dtype=torch.uint8, device="cuda")
        ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
        out, lse = ra.forward(q, k, v, N, True, layout, variant=variant, workspace=ws, events=ev)
        ev[1].synchronize()
        assert ev[0].elapsed_time(ev[1]) > 0
        ref_out, ref_lse = oracle.attention(q.cpu(), k.cpu(), v.cpu(), True, threads=THREADS)
        compare(out, lse, ref_out, ref_lse, torch.bfloat16)
        small = torch.empty(n // 2, dtype=torch.uint8, device="cuda")
        with pytest.raises(ra.RAError) as e:
            ra.forward(q, k, v, N, True, layout, variant=variant, workspace=small)
        assert e.value.code == -5


def test_caller_outputs_of_the_wrong_size_are_refused_before_launch():
    B, H, S, D, N = 1, 2, 512, 128, 4
    q, k, v = inputs.make_qkv(B, S, H, D, dtype=torch.bfloat16, device="cuda", seed=11)
    short = torch.empty((B, S - 128, H, D), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        ra.forward(q, k, v, N, True, "striped", out=short)
    with pytest.raises(ValueError):
        ra.forward(q, k, v, N, True, "striped", lse=torch.empty((B, H, S - 1), device="cuda"))
    with pytest.raises(ValueError):
        ra.backward(q, k, v, q, torch.zeros((B, H, S), device="cuda"), q, N, True, "striped", dq=short)
    with pytest.raises(ValueError):
        ra.rope(q, out=short)
    with pytest.raises(TypeError):  # fp16 is not a supported dtype
        ra.forward_varlen(q[0].half(), k[0].half(), v[0].half(), [0, S], N)
    with pytest.raises(TypeError):  # mixed dtypes
        ra.forward_varlen(q[0], k[0].float(), v[0], [0, S], N)
    torch.cuda.synchronize()
    assert ra.get_device_status() == 0
