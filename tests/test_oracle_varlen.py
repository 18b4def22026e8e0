"""Pins of the packed-sequence oracle (oracle.attention_varlen) to facts other than itself.

- a library routine: torch scaled_dot_product_attention in float64 with an explicit
  block-diagonal (and causal) boolean mask;
- closed form: a sequence of length one returns its own value row, lse = its own score;
- one sequence covering everything is plain attention (torch SDPA again);
- sequences do not see each other: changing another sequence's keys leaves a row unchanged;
- planted mistakes are caught.
"""
import os

import numpy as np
import pytest
import torch

import oracle

SRC = os.path.join(os.path.dirname(oracle.__file__), "ra_oracle.cpp")


def rand(S, H, D, seed):
    rng = np.random.default_rng(seed)
    return tuple(rng.standard_normal((1, S, H, D)) for _ in range(3))


def sdpa_masked(q, k, v, cu, causal):
    S = q.shape[1]
    seq = np.zeros(S, dtype=np.int64)
    for i in range(len(cu) - 1):
        seq[cu[i]:cu[i + 1]] = i
    allowed = seq[:, None] == seq[None, :]
    if causal:
        allowed &= np.tril(np.ones((S, S), dtype=bool))
    tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=torch.from_numpy(allowed))
    sc = (tq @ tk.transpose(-1, -2)) / np.sqrt(q.shape[-1])
    sc = sc.masked_fill(~torch.from_numpy(allowed), float("-inf"))
    return o.permute(0, 2, 1, 3)[0].numpy(), torch.logsumexp(sc, -1)[0].numpy()


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("cu", [[0, 40], [0, 8, 24, 40], [0, 1, 2, 30, 31, 40], [0, 16, 16, 40]])
def test_matches_masked_sdpa(causal, cu):
    q, k, v = rand(40, 2, 8, seed=len(cu))
    out, lse = oracle.attention_varlen(q, k, v, cu, causal)
    ref, ref_lse = sdpa_masked(q, k, v, cu, causal)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)


def test_length_one_sequences():
    q, k, v = rand(5, 1, 4, seed=9)
    out, lse = oracle.attention_varlen(q, k, v, [0, 1, 2, 3, 4, 5], False)
    np.testing.assert_allclose(out, v[0], rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse[0], (q[0, :, 0] * k[0, :, 0]).sum(-1) / 2.0, rtol=1e-14)


def test_sequences_do_not_see_each_other():
    q, k, v = rand(30, 1, 4, seed=10)
    a, _ = oracle.attention_varlen(q, k, v, [0, 10, 30], True)
    k2, v2 = k.copy(), v.copy()
    k2[0, 10:] += 5.0
    v2[0, 10:] -= 3.0
    b, _ = oracle.attention_varlen(q, k2, v2, [0, 10, 30], True)
    assert np.array_equal(a[:10], b[:10]) and not np.allclose(a[10:], b[10:])


VARLEN_MUTATIONS = {
    "sees_previous_sequence": ("const int64_t lo = cu[seq], hi", "const int64_t lo = 0, hi"),
    "noncausal_sees_next_sequence": ("causal ? r + 1 : cu[seq + 1];", "causal ? r + 1 : S_total;"),
    "causal_excludes_self": ("const int64_t lo = cu[seq], hi = causal ? r + 1", "const int64_t lo = cu[seq], hi = causal ? r"),
}


def pins_pass(lib):
    try:
        for causal in (False, True):
            q, k, v = rand(24, 1, 4, seed=11)
            cu = [0, 5, 17, 24]
            out, lse = oracle.attention_varlen(q, k, v, cu, causal, lib=lib)
            ref, ref_lse = sdpa_masked(q, k, v, cu, causal)
            if not (np.allclose(out, ref, rtol=1e-10, atol=1e-12) and np.allclose(lse, ref_lse, atol=1e-12)):
                return False
    except ValueError:
        return False
    return bool(np.isfinite(out).all())


@pytest.mark.parametrize("name", sorted(VARLEN_MUTATIONS))
def test_planted_varlen_mistake_is_caught(name, tmp_path):
    old, new = VARLEN_MUTATIONS[name]
    text = open(SRC).read()
    assert text.count(old) == 1, f"mutation site for {name} not found"
    assert pins_pass(oracle.load())
    src = tmp_path / "mutant.cpp"
    src.write_text(text.replace(old, new))
    lib_path = oracle.build(str(src), str(tmp_path / "libmutant.so"))
    assert not pins_pass(oracle.load(lib_path)), f"pins did not catch {name}"
