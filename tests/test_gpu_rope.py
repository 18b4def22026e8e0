"""GPU parity of ra_rope (through the C ABI) against the fp64 rotary-embedding oracle.

Bars: fp32 max |y - ref| <= 1e-5 * max(1, max |ref|); bf16 max <= 2^-8 * max(1, max |ref|) (one
rounding of the output, 2^-9 relative, with margin) and mean <= 2e-3.  The angle is reduced in
fp64 on the GPU, so large positions keep the same accuracy."""
import numpy as np
import pytest
import torch

import long_context_exact_forward_b200 as ra
import oracle
from long_context_exact_forward_b200 import inputs

pytestmark = pytest.mark.gpu


def check(y, ref, dtype):
    y = y.float().cpu().double().numpy()
    scale = max(1.0, float(np.abs(ref).max()))
    err = np.abs(y - ref)
    if dtype == torch.float32:
        assert err.max() <= 1e-5 * scale, err.max()
    else:
        assert err.max() <= 2.0 ** -8 * scale and err.mean() <= 2e-3, (err.max(), err.mean())


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("D, pos_offset", [(128, 0), (64, 1_000_000), (2, 7), (96, 2_000_000_000)])
def test_rope_matches_oracle(dtype, D, pos_offset):
    x, _, _ = inputs.make_qkv(2, 300, 3, D, dtype=dtype, device="cuda", seed=D)
    y = ra.rope(x, pos_offset=pos_offset)
    torch.cuda.synchronize()
    check(y, oracle.rope(x.cpu(), pos_offset=pos_offset), dtype)


def test_rope_in_place_equals_out_of_place():
    x, _, _ = inputs.make_qkv(1, 512, 2, 128, dtype=torch.bfloat16, device="cuda", seed=9)
    y = ra.rope(x, pos_offset=11, base=500000.0)
    z = x.clone()
    ra.rope(z, pos_offset=11, base=500000.0, out=z)
    torch.cuda.synchronize()
    assert torch.equal(y, z)


def test_roped_attention_matches_the_oracle_on_roped_inputs():
    # rotary embedding then the ring forward pass, against the definition on the oracle-roped q, k
    q, k, v = inputs.make_qkv(1, 4 * 256, 2, 128, dtype=torch.bfloat16, device="cuda", seed=10)
    rq, rk = ra.rope(q), ra.rope(k)
    out, lse = ra.forward(rq, rk, v, 4, True, "striped")
    torch.cuda.synchronize()
    ref, ref_lse = oracle.attention(rq.cpu(), rk.cpu(), v.cpu(), True, threads=8)
    got = out.float().cpu().permute(0, 2, 1, 3).double().numpy()
    assert np.abs(got - ref).max() <= 2e-2
    assert np.abs(lse.cpu().double().numpy() - ref_lse).max() <= 1e-3


def test_rope_rejects_bad_arguments():
    x = torch.zeros(1, 4, 1, 3, device="cuda")
    with pytest.raises(ra.RAError):  # odd head dim
        ra.rope(x)
    x = torch.zeros(1, 4, 1, 4, device="cuda")
    with pytest.raises(ra.RAError):  # negative offset
        ra.rope(x, pos_offset=-1)
