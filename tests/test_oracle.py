"""Pins for the fp64 oracle: each test ties it to something other than itself.

T1 merge identities (troisinh.com "Ring Attention", "Tai sao no hoat dong")
T2 the toy ring of ultralytics.com "Ring Attention" and its printed outcome (tests/golden)
T3 closed forms (single key, first causal row, equal keys, constant values, key permutation)
T4 an independent library routine: torch scaled_dot_product_attention in float64 on the CPU
T5 brute force on tiny inputs in numpy long double
T6 layout invariance of the ring loop (contiguous / striped / zigzag)
T7 per-step work of the ring under the causal mask, in closed form, and the makespan ratio that
   motivates the striped layout (ultralytics.com "Ring Attention": early-query devices idle)
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from long_context_exact_forward_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_qkv(B, S, H, D, seed, dtype=np.float64, scale=1.0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, S, H, D)) * scale
    k = rng.standard_normal((B, S, H, D))
    v = rng.standard_normal((B, S, H, D))
    return q.astype(dtype), k.astype(dtype), v.astype(dtype)


def out_natural(out_bhnd):
    """[B, H, S, D] (oracle row-major per head) -> [B, S, H, D]."""
    return np.transpose(out_bhnd, (0, 2, 1, 3))


# ---------------------------------------------------------------- T1 merge identities
@pytest.mark.parametrize("parts", [2, 3, 5, 8])
def test_t1_merge_identities(parts):
    rng = np.random.default_rng(parts)
    n, L, D = 7, 40, 5
    s = rng.standard_normal((n, L)) * 3.0
    v = rng.standard_normal((L, D))
    # unsplit statistics straight from the definitions
    m_full = s.max(axis=1)
    e = np.exp(s - m_full[:, None])
    l_full, O_full = e.sum(axis=1), e @ v
    cuts = np.sort(rng.choice(np.arange(1, L), size=parts - 1, replace=False))
    bounds = [0, *cuts.tolist(), L]
    m = np.full(n, -np.inf)
    l = np.zeros(n)
    O = np.zeros((n, D))
    for a, b in zip(bounds[:-1], bounds[1:]):
        blk = s[:, a:b]
        mb = blk.max(axis=1)
        eb = np.exp(blk - mb[:, None])
        m, l, O = oracle.merge(m, l, O, mb, eb.sum(axis=1), eb @ v[a:b])
    np.testing.assert_allclose(m, m_full, rtol=0, atol=0)
    np.testing.assert_allclose(l, l_full, rtol=1e-13)
    np.testing.assert_allclose(O, O_full, rtol=1e-13, atol=1e-13)


def test_t1_merge_empty_sides():
    m, l, O = oracle.merge([-np.inf], [0.0], [[0.0, 0.0]], [1.5], [2.0], [[3.0, 4.0]])
    assert m[0] == 1.5 and l[0] == 2.0 and O.tolist() == [[3.0, 4.0]]
    m, l, O = oracle.merge([0.5], [1.0], [[1.0, 2.0]], [-np.inf], [0.0], [[0.0, 0.0]])
    assert m[0] == 0.5 and l[0] == 1.0 and O.tolist() == [[1.0, 2.0]]
    m, l, O = oracle.merge([-np.inf], [0.0], [[0.0]], [-np.inf], [0.0], [[0.0]])
    assert m[0] == -np.inf and l[0] == 0.0 and O.tolist() == [[0.0]]


# ---------------------------------------------------------------- T2 the page's toy ring
def _golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            key, val = line.split(None, 1)
            vals[key] = val.strip()
    return vals


def test_t2_toy_ring_matches_full_attention():
    g = _golden("toy_ring.txt")
    N, block, dim = int(g["n_devices"]), int(g["block"]), int(g["dim"])
    q, k, v = inputs.toy_qkv()
    assert q.shape == (1, N * block, 1, dim)
    ring, ring_lse, pairs = oracle.ring_blockwise(q, k, v, N, causal=False)
    full, full_lse = oracle.attention(q, k, v, causal=False)
    np.testing.assert_allclose(ring, out_natural(full), rtol=0, atol=1e-12)
    np.testing.assert_allclose(ring_lse, full_lse, rtol=0, atol=1e-12)
    # each device scored one block x block tile per step; together they covered the full matrix
    assert g["largest_score_block"] == f"{block}x{block}"
    assert g["full_matrix"] == f"{N * block}x{N * block}"
    assert pairs.tolist() == [[block * block] * N] * N
    assert pairs.sum() == (N * block) ** 2
    # the page's own check: the full softmax in fp32 torch agrees at atol 1e-5 -> True
    qq, kk, vv = (t.reshape(N * block, dim) for t in (q, k, v))
    torch_full = torch.softmax(qq @ kk.T / dim ** 0.5, dim=-1) @ vv
    atol = float(g["matches_full_attention_atol"])
    ok = np.allclose(ring.reshape(N * block, dim), torch_full.double().numpy(), atol=atol, rtol=0)
    assert str(ok) == g["matches_full_attention"]


# ---------------------------------------------------------------- T3 closed forms
def test_t3_single_key():
    q, k, v = rand_qkv(2, 1, 3, 8, seed=1)
    out, lse = oracle.attention(q, k, v, causal=False)
    np.testing.assert_array_equal(out_natural(out), v)
    s = np.einsum("bshd,bshd->bhs", q, k) / math.sqrt(8)
    np.testing.assert_allclose(lse, s, rtol=1e-15, atol=1e-15)


def test_t3_first_causal_row_sees_only_itself():
    q, k, v = rand_qkv(1, 9, 2, 4, seed=2)
    out, lse = oracle.attention(q, k, v, causal=True)
    np.testing.assert_array_equal(out[:, :, 0, :], v[:, 0, :, :])
    np.testing.assert_allclose(lse[:, :, 0], np.einsum("bhd,bhd->bh", q[:, 0], k[:, 0]) / 2.0,
                               rtol=1e-15, atol=1e-15)


def test_t3_equal_keys_give_mean_of_values():
    B, S, H, D = 1, 11, 2, 6
    q, k, v = rand_qkv(B, S, H, D, seed=3)
    k[:] = k[:, :1]  # every key equals key 0
    for causal in (False, True):
        out, lse = oracle.attention(q, k, v, causal=causal)
        for r in range(S):
            n = r + 1 if causal else S
            np.testing.assert_allclose(out[0, :, r, :], v[0, :n].mean(axis=0), rtol=1e-13, atol=1e-14)
            s = np.einsum("hd,hd->h", q[0, r], k[0, 0]) / math.sqrt(D)
            np.testing.assert_allclose(lse[0, :, r], s + math.log(n), rtol=1e-13, atol=1e-13)


def test_t3_constant_values():
    q, k, v = rand_qkv(1, 13, 2, 5, seed=4)
    v[:] = np.array([0.5, -1.0, 2.0, 3.25, 0.0])
    for causal in (False, True):
        out, _ = oracle.attention(q, k, v, causal=causal)
        np.testing.assert_allclose(out, np.broadcast_to(v[0, 0][None, :, None, :], out.shape), rtol=1e-14, atol=1e-14)


def test_t3_key_permutation_invariance():
    q, k, v = rand_qkv(1, 17, 2, 4, seed=5)
    perm = np.random.default_rng(0).permutation(17)
    a, la = oracle.attention(q, k, v, causal=False)
    b, lb = oracle.attention(q, k[:, perm], v[:, perm], causal=False)
    np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(la, lb, rtol=1e-13, atol=1e-14)


# ---------------------------------------------------------------- T4 library routine
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [(1, 64, 2, 16), (2, 96, 3, 32), (1, 300, 1, 128)])
def test_t4_torch_sdpa_float64(shape, causal):
    B, S, H, D = shape
    q, k, v = rand_qkv(B, S, H, D, seed=S + D)
    out, lse = oracle.attention(q, k, v, causal=causal, threads=4)
    tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal)
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-10, atol=1e-12)
    scores = (tq @ tk.transpose(-1, -2)) / math.sqrt(D)
    if causal:
        scores = scores.masked_fill(torch.ones(S, S, dtype=torch.bool).triu(1), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(scores, dim=-1).numpy(), rtol=1e-12, atol=1e-12)


def test_t4_sampled_rows_match_all_rows():
    q, k, v = rand_qkv(2, 50, 3, 8, seed=9)
    full, full_lse = oracle.attention(q, k, v, causal=True)
    rows = np.array([[0, 7, 49], [1, 2, 3], [10, 20, 30], [49, 48, 0], [5, 5, 6], [33, 34, 35]])
    sub, sub_lse = oracle.attention(q, k, v, causal=True, rows=rows, threads=3)
    for bh in range(6):
        b, h = divmod(bh, 3)
        np.testing.assert_array_equal(sub[b, h], full[b, h, rows[bh]])
        np.testing.assert_array_equal(sub_lse[b, h], full_lse[b, h, rows[bh]])


# ---------------------------------------------------------------- T5 brute force
@pytest.mark.parametrize("D", [1, 2, 16])
@pytest.mark.parametrize("causal", [False, True])
def test_t5_brute_force_long_double(D, causal):
    B, S, H = 2, 23, 2
    q, k, v = rand_qkv(B, S, H, D, seed=D * 7 + causal, scale=2.0)
    out, lse = oracle.attention(q, k, v, causal=causal)
    ld = np.longdouble
    for b in range(B):
        for h in range(H):
            for r in range(S):
                keys = range(r + 1) if causal else range(S)
                sc = [sum(ld(q[b, r, h, d]) * ld(k[b, c, h, d]) for d in range(D)) / np.sqrt(ld(D))
                      for c in keys]
                w = [np.exp(x) for x in sc]  # no max shift: long double has the range
                tot = sum(w)
                ref = [sum(wc * ld(v[b, c, h, d]) for wc, c in zip(w, keys)) / tot for d in range(D)]
                np.testing.assert_allclose(out[b, h, r], np.array(ref, dtype=np.float64), rtol=1e-12, atol=1e-13)
                assert abs(float(np.log(tot)) - lse[b, h, r]) < 1e-12


def test_t5_bf16_inputs_are_read_exactly():
    q, k, v = (torch.from_numpy(x) for x in rand_qkv(1, 40, 2, 16, seed=11))
    qb, kb, vb = (x.to(torch.bfloat16) for x in (q, k, v))
    a, la = oracle.attention(qb, kb, vb, causal=True)
    b, lb = oracle.attention(qb.double(), kb.double(), vb.double(), causal=True)
    np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(la, lb)
    c, lc = oracle.attention(qb.float(), kb.float(), vb.float(), causal=True)
    np.testing.assert_array_equal(a, c)


# ---------------------------------------------------------------- T6 layout invariance
@pytest.mark.parametrize("layout", ["contiguous", "striped", "zigzag"])
@pytest.mark.parametrize("N", [1, 2, 3, 4])
@pytest.mark.parametrize("causal", [False, True])
def test_t6_ring_layout_invariance(layout, N, causal):
    S = 24
    q, k, v = rand_qkv(2, S, 2, 8, seed=N * 10 + causal)
    ring, ring_lse, _ = oracle.ring_blockwise(q, k, v, N, causal=causal, layout=layout)
    full, full_lse = oracle.attention(q, k, v, causal=causal)
    np.testing.assert_allclose(ring, out_natural(full), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(ring_lse, full_lse, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("layout", ["contiguous", "striped", "zigzag"])
def test_t6_layout_is_a_bijection_with_monotone_shards(layout):
    S, N = 48, 4
    pos = oracle.layout_positions(S, N, layout)
    assert sorted(pos.ravel().tolist()) == list(range(S))
    assert (np.diff(pos, axis=1) > 0).all()
    if layout == "contiguous":
        assert pos[1, 0] == S // N
    if layout == "striped":
        assert pos[:, 0].tolist() == list(range(N)) and pos[0, 1] == N
    if layout == "zigzag":
        C = S // (2 * N)
        assert pos[0, C] == (2 * N - 1) * C and pos[N - 1, 0] == (N - 1) * C


# ---------------------------------------------------------------- T7 causal work per ring step
def test_t7_per_step_work_closed_forms_and_makespan():
    N, L = 4, 6
    S = N * L
    q, k, v = rand_qkv(1, S, 1, 2, seed=0)
    _, _, contiguous = oracle.ring_blockwise(q, k, v, N, causal=True, layout="contiguous")
    _, _, striped = oracle.ring_blockwise(q, k, v, N, causal=True, layout="striped")
    _, _, zigzag = oracle.ring_blockwise(q, k, v, N, causal=True, layout="zigzag")
    for i in range(N):
        for s in range(N):
            j = (i - s) % N
            # contiguous: own block is a triangle, earlier blocks full, later blocks empty
            want = L * (L + 1) // 2 if j == i else (L * L if j < i else 0)
            assert contiguous[i, s] == want
            # striped: key c*N+j <= query a*N+i  <=>  c < a, or c == a and j <= i
            assert striped[i, s] == L * (L - 1) // 2 + (L if j <= i else 0)
    # every allowed pair is counted once
    for t in (contiguous, striped, zigzag):
        assert t.sum() == S * (S + 1) // 2
    # zigzag: every shard does the same total work
    assert len(set(zigzag.sum(axis=1).tolist())) == 1
    # makespan (sum over steps of the busiest device) ratio, contiguous / striped -> (2N-1)/N
    ratio = contiguous.max(axis=0).sum() / striped.max(axis=0).sum()
    assert ratio == pytest.approx((L * (L + 1) / 2 + (N - 1) * L * L) / (N * L * (L + 1) / 2))
    big_N, big_L = 16, 8192
    big = (big_L * (big_L + 1) / 2 + (big_N - 1) * big_L ** 2) / (big_N * big_L * (big_L + 1) / 2)
    assert big == pytest.approx((2 * big_N - 1) / big_N, rel=1e-3)
