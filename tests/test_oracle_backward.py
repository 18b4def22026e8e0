"""Pins of the fp64 backward oracle (oracle.attention_backward) to facts other than itself.

The gradient follows the plain definition of attention by the chain rule (troisinh.com "Ring
Attention", "Blockwise Backward" recomputes the forward statistics in the backward pass).  Pins:
- a library routine: torch autograd through scaled_dot_product_attention in float64 (an
  independent implementation);
- central finite differences of the forward oracle itself (loss = sum(dout * out));
- closed forms: one key (dq = dk = 0, dv = dout), identical keys (dq = 0), and the invariant
  sum_c dv_c = sum_r dout_r (every softmax row sums to one);
- exact reading of bf16 inputs and independence of the host thread count;
- planted mistakes in a copy of the oracle, each caught by these pins.
"""
import os

import numpy as np
import pytest
import torch

import oracle

SRC = os.path.join(os.path.dirname(oracle.__file__), "ra_oracle.cpp")


def rand(B, S, H, D, seed, n=4):
    rng = np.random.default_rng(seed)
    return tuple(rng.standard_normal((B, S, H, D)) for _ in range(n))


def torch_grads(q, k, v, do, causal):
    tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3).clone().requires_grad_(True) for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal)
    o.backward(torch.from_numpy(do).permute(0, 2, 1, 3))
    return tuple(t.grad.permute(0, 2, 1, 3).numpy() for t in (tq, tk, tv))


@pytest.mark.parametrize("shape", [(1, 1, 1, 4), (1, 37, 2, 8), (2, 64, 3, 16), (1, 50, 1, 1)])
@pytest.mark.parametrize("causal", [False, True])
def test_matches_torch_autograd_float64(shape, causal):
    q, k, v, do = rand(*shape, seed=sum(shape))
    ours = oracle.attention_backward(q, k, v, do, causal)
    ref = torch_grads(q, k, v, do, causal)
    for a, b in zip(ours, ref):
        np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_central_finite_differences_of_the_forward_oracle(causal):
    B, S, H, D = 1, 9, 1, 4
    q, k, v, do = rand(B, S, H, D, seed=11)
    grads = oracle.attention_backward(q, k, v, do, causal)

    def loss(qq, kk, vv):
        out, _ = oracle.attention(qq, kk, vv, causal)  # [B, H, S, D]
        return float((out * do.transpose(0, 2, 1, 3)).sum())

    rng = np.random.default_rng(12)
    eps = 1e-6
    for which in range(3):
        for _ in range(6):
            idx = (0, int(rng.integers(S)), 0, int(rng.integers(D)))
            xs = [q.copy(), k.copy(), v.copy()]
            xs[which][idx] += eps
            up = loss(*xs)
            xs[which][idx] -= 2 * eps
            down = loss(*xs)
            fd = (up - down) / (2 * eps)
            assert abs(fd - grads[which][idx]) <= 1e-7 * max(1.0, abs(fd)), (which, idx)


def test_one_key_closed_form():
    q, k, v, do = rand(2, 1, 3, 5, seed=13)
    dq, dk, dv = oracle.attention_backward(q, k, v, do, True)
    assert np.array_equal(dq, np.zeros_like(dq)) and np.array_equal(dk, np.zeros_like(dk))
    np.testing.assert_allclose(dv, do, rtol=0, atol=1e-15)


@pytest.mark.parametrize("causal", [False, True])
def test_identical_keys_give_zero_query_gradient(causal):
    q, k, v, do = rand(1, 20, 2, 6, seed=14)
    k[:] = k[:, :1]  # every key equal: the scores of a row are constant
    dq, _, _ = oracle.attention_backward(q, k, v, do, causal)
    np.testing.assert_allclose(dq, 0.0, atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_value_gradient_sums_to_the_output_gradient(causal):
    q, k, v, do = rand(2, 33, 2, 7, seed=15)
    _, _, dv = oracle.attention_backward(q, k, v, do, causal)
    np.testing.assert_allclose(dv.sum(axis=1), do.sum(axis=1), rtol=1e-12, atol=1e-12)


def test_bf16_inputs_are_read_exactly_and_threads_do_not_matter():
    q, k, v, do = (torch.from_numpy(x).to(torch.bfloat16) for x in rand(2, 24, 2, 8, seed=16))
    a = oracle.attention_backward(q, k, v, do, True, threads=1)
    b = oracle.attention_backward(q.double(), k.double(), v.double(), do.double(), True, threads=3)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


BACKWARD_MUTATIONS = {
    "no_softmax_jacobian_term": ("const double dS = P[c] * (dP[c] - row_dot);",
                                 "const double dS = P[c] * dP[c];"),
    "dk_without_scale": ("dk[at(b, c, h, d, S, H, D)] += scale * dS * qr[d];",
                         "dk[at(b, c, h, d, S, H, D)] += dS * qr[d];"),
    "dv_from_dP": ("dv[at(b, c, h, d, S, H, D)] += P[c] * dor[d];",
                   "dv[at(b, c, h, d, S, H, D)] += dP[c] * dor[d];"),
    "dq_from_query": ("dq[at(b, r, h, d, S, H, D)] += scale * dS * to_f64(k, dtype, at(b, c, h, d, S, H, D));",
                      "dq[at(b, r, h, d, S, H, D)] += scale * dS * qr[d];"),
    "dP_from_keys": ("for (int64_t d = 0; d < D; ++d) dot += dor[d] * to_f64(v, dtype, at(b, c, h, d, S, H, D));",
                     "for (int64_t d = 0; d < D; ++d) dot += dor[d] * to_f64(k, dtype, at(b, c, h, d, S, H, D));"),
    "backward_causal_excludes_diagonal": ("const int64_t n_keys = causal ? r + 1 : S;\n                double m",
                                          "const int64_t n_keys = causal ? r : S;\n                double m"),
}


def backward_pins_pass(lib):
    try:
        for causal in (False, True):
            q, k, v, do = rand(1, 21, 2, 6, seed=17)
            ours = oracle.attention_backward(q, k, v, do, causal, lib=lib)
            for a, b in zip(ours, torch_grads(q, k, v, do, causal)):
                if not np.allclose(a, b, rtol=1e-10, atol=1e-12):
                    return False
    except ValueError:
        return False
    return True


def test_unmutated_backward_oracle_passes():
    assert backward_pins_pass(oracle.load())


@pytest.mark.parametrize("name", sorted(BACKWARD_MUTATIONS))
def test_planted_backward_mistake_is_caught(name, tmp_path):
    old, new = BACKWARD_MUTATIONS[name]
    text = open(SRC).read()
    assert text.count(old) == 1, f"mutation site for {name} not found"
    src = tmp_path / "mutant.cpp"
    src.write_text(text.replace(old, new))
    lib_path = oracle.build(str(src), str(tmp_path / "libmutant.so"))
    assert not backward_pins_pass(oracle.load(lib_path)), f"pins did not catch {name}"
