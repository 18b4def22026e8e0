"""Planted mistakes: each plausible slip in the oracle must be caught by an independent pin.

Every case copies ra_oracle.cpp to a temporary directory, applies one textual mutation (a dropped
term, a wrong sign, index or operand), builds the copy, and checks that at least one of the pins
below fails on it.  The committed oracle is never modified.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

SRC = os.path.join(os.path.dirname(oracle.__file__), "ra_oracle.cpp")

MUTATIONS = {
    "drop_scale": ("scores[c] = scale * dot;", "scores[c] = dot;"),
    "causal_excludes_diagonal": ("causal ? r + 1 : S", "causal ? r : S"),
    "key_read_from_query": ("to_f64(k, dtype, at(b, c, h, d, S, H, D))",
                            "to_f64(q, dtype, at(b, c, h, d, S, H, D))"),
    "value_transposed": ("to_f64(v, dtype, at(b, c, h, d, S, H, D))",
                         "to_f64(v, dtype, at(b, d % S, h, c % D, S, H, D))"),
    "lse_without_log": ("*lse_out = m + std::log(l);", "*lse_out = m + l;"),
    "no_division": ("out_row[d] /= l;", "out_row[d] /= 1.0;"),
    "merge_wrong_sign": ("std::exp(mp - mu)", "std::exp(mu - mp)"),
    "merge_drops_new_sum": ("l[r] = ap * l[r] + an * l2[r];", "l[r] = ap * l[r];"),
    "ring_stays_on_own_block": ("const int64_t j = ((i - s) % N + N) % N;", "const int64_t j = i;"),
    "striped_wrong_shard": ("return a * N + i;", "return a * N + (N - 1 - i);"),
    "ring_mask_reversed": ("if (causal && gk > gq)", "if (causal && gk < gq)"),
    "bf16_shift": ("<< 16;", "<< 15;"),
}


def rand(B, S, H, D, seed):
    rng = np.random.default_rng(seed)
    return tuple(rng.standard_normal((B, S, H, D)) for _ in range(3))


def pins_pass(lib):
    """Run a compact set of the independent pins against `lib`; False if any fails."""
    try:
        # library routine (torch SDPA, float64)
        for causal in (False, True):
            q, k, v = rand(1, 40, 2, 16, seed=1)
            out, lse = oracle.attention(q, k, v, causal, lib=lib)
            tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v))
            ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal)
            if not np.allclose(out, ref.numpy(), rtol=1e-10, atol=1e-12):
                return False
            sc = (tq @ tk.transpose(-1, -2)) / 4.0
            if causal:
                sc = sc.masked_fill(torch.ones(40, 40, dtype=torch.bool).triu(1), float("-inf"))
            if not np.allclose(lse, torch.logsumexp(sc, -1).numpy(), rtol=1e-12, atol=1e-12):
                return False
        # bf16 inputs read exactly (torch's own bf16 -> fp32 conversion)
        qb, kb, vb = (torch.from_numpy(x).to(torch.bfloat16) for x in rand(1, 16, 1, 8, seed=2))
        a, _ = oracle.attention(qb, kb, vb, True, lib=lib)
        b, _ = oracle.attention(qb.double(), kb.double(), vb.double(), True, lib=lib)
        if not np.array_equal(a, b):
            return False
        # the ring loop equals the definition (T6) and the merge identities (T1)
        for layout in ("contiguous", "striped", "zigzag"):
            q, k, v = rand(1, 24, 1, 4, seed=3)
            ring, _, _ = oracle.ring_blockwise(q, k, v, 3, True, layout, lib=lib)
            ref = torch.nn.functional.scaled_dot_product_attention(
                *(torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v)), is_causal=True)
            if not np.allclose(ring, ref.permute(0, 2, 1, 3).numpy(), rtol=1e-12, atol=1e-12):
                return False
        rng = np.random.default_rng(4)
        s, vv = rng.standard_normal((3, 10)), rng.standard_normal((10, 2))
        m1, m2 = s[:, :4].max(1), s[:, 4:].max(1)
        e1, e2 = np.exp(s[:, :4] - m1[:, None]), np.exp(s[:, 4:] - m2[:, None])
        m, l, O = oracle.merge(m1, e1.sum(1), e1 @ vv[:4], m2, e2.sum(1), e2 @ vv[4:], lib=lib)
        e = np.exp(s - s.max(1)[:, None])
        if not (np.allclose(l, e.sum(1), rtol=1e-13) and np.allclose(O, e @ vv, rtol=1e-13)):
            return False
        # striped per-step causal work in closed form (T7)
        q, k, v = rand(1, 12, 1, 2, seed=5)
        _, _, pairs = oracle.ring_blockwise(q, k, v, 4, True, "striped", lib=lib)
        for i in range(4):
            for st in range(4):
                j = (i - st) % 4
                if pairs[i, st] != 3 * 2 // 2 + (3 if j <= i else 0):
                    return False
    except ValueError:
        return False
    return True


def test_unmutated_oracle_passes_the_compact_pins():
    assert pins_pass(oracle.load())


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, tmp_path):
    old, new = MUTATIONS[name]
    text = open(SRC).read()
    assert text.count(old) >= 1, f"mutation site for {name} not found"
    src = tmp_path / "mutant.cpp"
    src.write_text(text.replace(old, new))
    lib_path = oracle.build(str(src), str(tmp_path / "libmutant.so"))
    assert not pins_pass(oracle.load(lib_path)), f"pins did not catch {name}"
