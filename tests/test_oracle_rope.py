"""Pins of the fp64 rotary-embedding oracle (oracle.rope) to facts other than itself.

Rotary embedding with global positions (troisinh.com "Ring Attention", "RoPE va Position
Embedding"): each pair (x[2p], x[2p+1]) of the token at position m is rotated by m * theta_p.
Pins: position 0 is the identity; each pair keeps its length; D = 2 has theta_0 = 1 and a closed
form; rotations compose (offset a then b equals offset a + b); the score q . k of two rotated
tokens depends only on the position difference (the point of the embedding); the frequencies
follow base^(-2p/D) (checked on one pair against the formula); planted mistakes are caught.
"""
import math
import os

import numpy as np
import pytest

import oracle

SRC = os.path.join(os.path.dirname(oracle.__file__), "ra_oracle.cpp")


def rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_position_zero_is_identity_and_lengths_are_kept():
    x = rand((2, 7, 3, 8), 1)
    y = oracle.rope(x)
    assert np.array_equal(y[:, 0], x[:, 0])
    pairs_x = np.hypot(x[..., 0::2], x[..., 1::2])
    pairs_y = np.hypot(y[..., 0::2], y[..., 1::2])
    np.testing.assert_allclose(pairs_y, pairs_x, rtol=1e-14, atol=1e-14)


def test_two_dim_closed_form():
    x = rand((1, 9, 1, 2), 2)
    y = oracle.rope(x, pos_offset=5, base=123.0)  # theta_0 = base^0 = 1 for any base
    for g in range(9):
        m = g + 5
        c, s = math.cos(m), math.sin(m)
        x0, x1 = x[0, g, 0]
        np.testing.assert_allclose(y[0, g, 0], [x0 * c - x1 * s, x0 * s + x1 * c], rtol=0, atol=1e-14)


def test_frequencies():
    D, base = 16, 500.0
    x = np.zeros((1, 2, 1, D))
    x[0, 1, 0, 0::2] = 1.0  # unit vectors along each pair's first axis at position 1
    y = oracle.rope(x, base=base)
    for p in range(D // 2):
        theta = base ** (-2.0 * p / D)
        np.testing.assert_allclose(y[0, 1, 0, 2 * p:2 * p + 2], [math.cos(theta), math.sin(theta)], atol=1e-14)


def test_rotations_compose():
    x = rand((1, 6, 2, 12), 3)
    twice = oracle.rope(oracle.rope(x, pos_offset=3), pos_offset=40)
    # rope(x, a) at natural index g rotates by (g + a); applying it twice adds the angles, so it
    # equals one rotation by (2g + 43)
    once = np.empty_like(twice)
    for g in range(6):
        once[:, g] = oracle.rope(x[:, g:g + 1], pos_offset=2 * g + 43)[:, 0]
    np.testing.assert_allclose(twice, once, rtol=1e-12, atol=1e-12)


def test_scores_depend_only_on_the_position_difference():
    q, k = rand((1, 1, 1, 32), 4), rand((1, 1, 1, 32), 5)
    dots = []
    for shift in (0, 17, 1000, 123456):
        rq = oracle.rope(q, pos_offset=shift + 9)
        rk = oracle.rope(k, pos_offset=shift + 2)
        dots.append(float((rq * rk).sum()))
    np.testing.assert_allclose(dots, dots[0], rtol=1e-9, atol=1e-9)
    # and it does change with the difference
    assert abs(float((oracle.rope(q, pos_offset=9) * oracle.rope(k, pos_offset=3)).sum()) - dots[0]) > 1e-6


def test_rejects_odd_head_dim():
    with pytest.raises(ValueError):
        oracle.rope(np.zeros((1, 2, 1, 3)))


ROPE_MUTATIONS = {
    "sin_sign": ("y[at(b, g, h, 2 * p, S, H, D)] = x0 * c - x1 * sn;", "y[at(b, g, h, 2 * p, S, H, D)] = x0 * c + x1 * sn;"),
    "frequency_exponent": ("std::pow(base, -2.0 * (double)p / (double)D)", "std::pow(base, -1.0 * (double)p / (double)D)"),
    "position_ignores_offset": ("const double m = (double)(g + pos_offset);", "const double m = (double)g;"),
    "pair_swapped": ("y[at(b, g, h, 2 * p + 1, S, H, D)] = x0 * sn + x1 * c;", "y[at(b, g, h, 2 * p + 1, S, H, D)] = x1 * sn + x0 * c;"),
}


def rope_pins_pass(lib):
    try:
        x = rand((1, 5, 1, 8), 6)
        y = oracle.rope(x, pos_offset=2, base=100.0, lib=lib)
        for g in range(5):
            m = g + 2
            for p in range(4):
                th = m * 100.0 ** (-2.0 * p / 8)
                x0, x1 = x[0, g, 0, 2 * p], x[0, g, 0, 2 * p + 1]
                want = [x0 * math.cos(th) - x1 * math.sin(th), x0 * math.sin(th) + x1 * math.cos(th)]
                if not np.allclose(y[0, g, 0, 2 * p:2 * p + 2], want, atol=1e-12):
                    return False
    except ValueError:
        return False
    return True


@pytest.mark.parametrize("name", sorted(ROPE_MUTATIONS))
def test_planted_rope_mistake_is_caught(name, tmp_path):
    old, new = ROPE_MUTATIONS[name]
    text = open(SRC).read()
    assert text.count(old) == 1, f"mutation site for {name} not found"
    assert rope_pins_pass(oracle.load())
    src = tmp_path / "mutant.cpp"
    src.write_text(text.replace(old, new))
    lib_path = oracle.build(str(src), str(tmp_path / "libmutant.so"))
    assert not rope_pins_pass(oracle.load(lib_path)), f"pins did not catch {name}"
