"""C-ABI checks that need no GPU: the library loads, exports what include/ra.h declares, and
rejects bad arguments before touching the device."""
import ctypes
import os
import re

import numpy as np
import pytest

import long_context_exact_forward_b200 as ra

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ra.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"RA_API\s+[\w\s\*]+?\b(ra_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = declared_symbols()
    assert "ra_forward" in names and "ra_forward_ex" in names and len(names) >= 12
    lib = ctypes.CDLL(ra.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in ra.h but not exported"


def test_status_strings():
    for code in (0, -1, -2, -3, -4, -5, -6, -7):
        assert ra.status_string(code) and ra.status_string(code) != "unknown status"
    assert ra.status_string(12345) == "unknown status"


FAKE = 0x100000  # 16-byte aligned, never dereferenced: validation fails first


def call(B=1, H=2, S=64, D=16, n_ring=4, causal=1, layout=0, dtype=0, q=FAKE, k=FAKE, v=FAKE,
         out=FAKE, lse=FAKE, variant=0, kernel=0):
    opt = ra.Options()
    opt.variant = variant
    opt.kernel = kernel
    return ra.lib().ra_forward_ex(q, k, v, out, lse, B, H, S, D, n_ring, causal, layout, dtype,
                                  None, ctypes.byref(opt))


@pytest.mark.parametrize("kw, code", [
    (dict(S=63), -2),                    # S % n_ring
    (dict(S=68, layout=2), -2),          # zigzag needs S % 2N
    (dict(D=300), -2),                   # head dim above 256
    (dict(D=0), -1),
    (dict(B=0), -1),
    (dict(n_ring=0), -1),
    (dict(layout=3), -1),
    (dict(dtype=5), -1),
    (dict(q=0), -1),
    (dict(lse=0), -1),
    (dict(k=FAKE + 8), -3),              # misaligned tensor
    (dict(variant=7), -1),
])
def test_validation_rejects_before_any_cuda_call(kw, code):
    assert call(**kw) == code


def test_workspace_size_grows_with_per_step_and_permute():
    args = dict(B=1, H=4, S=4096, D=128, n_ring=4, causal=True, dtype_code=1)
    fused_contig = ra.workspace_size(layout="contiguous", variant="fused", **args)
    fused_striped = ra.workspace_size(layout="striped", variant="fused", **args)
    per_step = ra.workspace_size(layout="contiguous", variant="per_step", **args)
    elems = 1 * 4096 * 4 * 128
    fused_zigzag = ra.workspace_size(layout="zigzag", variant="fused", **args)
    assert fused_striped < fused_contig + elems                    # striped is read in place
    assert fused_zigzag >= fused_contig + 3 * elems * 2           # permuted q, k, v
    assert per_step >= fused_contig + 2 * elems * 4               # running and step partials
    simt = ra.workspace_size(layout="zigzag", variant="fused", kernel="simt", **args)
    assert simt <= fused_contig                                   # SIMT reads natural order


def test_workspace_size_rejects_bad_shape():
    with pytest.raises(ra.RAError):
        ra.workspace_size(1, 1, 10, 16, 3, False, "contiguous", 0)


def test_backward_rope_and_varlen_validate_before_any_cuda_call():
    lib = ra.lib()
    # ra_backward_ex: S not divisible by n_ring; bad kernel code; head dim above 128
    assert lib.ra_backward_ex(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 63, 16, 4, 1, 0, 0,
                              0, 0, 0, None) == -2
    assert lib.ra_backward_ex(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 64, 16, 4, 1, 0, 0,
                              9, 0, 0, None) == -1
    assert lib.ra_backward_ex(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 64, 256, 4, 1, 0, 1,
                              0, 0, 0, None) == -4
    # ra_rope: odd head dim, negative offset, misaligned pointer
    assert lib.ra_rope(FAKE, FAKE, 1, 4, 1, 3, 0, 10000.0, 0, None) == -1
    assert lib.ra_rope(FAKE, FAKE, 1, 4, 1, 4, -1, 10000.0, 0, None) == -1
    assert lib.ra_rope(FAKE + 2, FAKE, 1, 4, 1, 4, 0, 10000.0, 0, None) == -3
    assert lib.ra_rope(FAKE, FAKE, 1, 4, 1 << 21, 256, 0, 10000.0, 0, None) == -2  # H * D above 2^28
    # ra_forward_varlen: a length not divisible by n_ring; under zigzag one not divisible by 2 n_ring;
    # an unknown layout; cu[0] != 0; an unknown dtype; a head dim above 256
    cu = np.array([0, 50, 100], dtype=np.int64)
    assert lib.ra_forward_varlen(FAKE, FAKE, FAKE, FAKE, FAKE, cu.ctypes.data, 2, 1, 128, 4, 1, 0, 1, None) == -2
    cu = np.array([0, 64, 132], dtype=np.int64)
    assert lib.ra_forward_varlen(FAKE, FAKE, FAKE, FAKE, FAKE, cu.ctypes.data, 2, 1, 128, 4, 1, 2, 1, None) == -2
    cu = np.array([0, 64, 128], dtype=np.int64)
    assert lib.ra_forward_varlen(FAKE, FAKE, FAKE, FAKE, FAKE, cu.ctypes.data, 2, 1, 128, 4, 1, 3, 1, None) == -1
    cu = np.array([4, 64, 128], dtype=np.int64)
    assert lib.ra_forward_varlen(FAKE, FAKE, FAKE, FAKE, FAKE, cu.ctypes.data, 2, 1, 128, 4, 1, 0, 1, None) == -1
    cu = np.array([0, 64, 128], dtype=np.int64)
    assert lib.ra_forward_varlen(FAKE, FAKE, FAKE, FAKE, FAKE, cu.ctypes.data, 2, 1, 128, 4, 1, 0, 2, None) == -1
    assert lib.ra_forward_varlen(FAKE, FAKE, FAKE, FAKE, FAKE, cu.ctypes.data, 2, 1, 264, 4, 1, 0, 0, None) == -2


def test_varlen_workspace_size_and_options_validate_on_the_host():
    lib = ra.lib()
    lengths = [1024, 0, 600 * 8, 48, 4096]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    S = int(cu[-1])
    H, D, N = 3, 128, 8
    a256 = lambda x: -(-x // 256) * 256
    # one launch: counter, sequence table, work list, (tensor cores) norms per head
    tc_items = sum(H * N * -(-(n // N) // 256) for n in lengths)
    base = 256 + a256(len(lengths) * 8) + a256(tc_items * 16) + a256(2 * H * 4)
    assert ra.varlen_workspace_size(cu, H, D, N, "contiguous") == base
    assert ra.varlen_workspace_size(cu, H, D, N, "striped") == base
    assert ra.varlen_workspace_size(cu, H, D, N, "zigzag") == base + 3 * a256(S * H * D * 2)
    # per step: one counter per launch (N of them at one step per launch) and the fp32 running and
    # partial results
    acc = 2 * (a256(S * H * D * 4) + a256(S * H * 4))
    assert ra.varlen_workspace_size(cu, H, D, N, "striped", 1, "per_step") == base + acc
    assert ra.varlen_workspace_size(cu, H, D, 1, "striped", 1, "per_step") == \
        256 + a256(len(lengths) * 8) + a256(sum(H * -(-n // 256) for n in lengths) * 16) + a256(2 * H * 4)
    # CUDA cores: 64-row items over every head, no norms, no shard-major copies
    simt_items = sum(N * -(-(n // N) // 64) for n in lengths)
    simt = 256 + a256(len(lengths) * 8) + a256(simt_items * 16)
    for layout in ("contiguous", "zigzag"):
        assert ra.varlen_workspace_size(cu, H, D, N, layout, 1, "auto", "simt") == simt
        assert ra.varlen_workspace_size(cu, H, D, N, layout, 0) == simt  # fp32: CUDA cores
        assert ra.varlen_workspace_size(cu, H, 96, N, layout, 1) == simt  # D outside {64, 128}
        assert ra.varlen_workspace_size(cu, H, D, N, layout, 0, "per_step") == simt + acc
    with pytest.raises(ra.RAError):  # 600 * 8 + 4 is not a multiple of 2N
        ra.varlen_workspace_size([0, 600 * 8 + 4], H, D, N, "zigzag")
    with pytest.raises(ra.RAError):  # the tensor cores take bf16 only
        ra.varlen_workspace_size(cu, H, D, N, "zigzag", 0, "auto", "tc")

    def ex(variant=0, kernel=0, ws=None, nbytes=0, debug=0, dtype=1, spl=0):
        opt = ra.Options()
        opt.variant, opt.kernel, opt.debug, opt.steps_per_launch = variant, kernel, debug, spl
        opt.workspace, opt.workspace_bytes = ws, nbytes
        return lib.ra_forward_varlen_ex(FAKE, FAKE, FAKE, FAKE, FAKE, cu.ctypes.data, len(lengths), H, D, N, 1, 2,
                                        dtype, None, ctypes.byref(opt))
    assert ex(variant=3) == -1                        # unknown variant
    assert ex(kernel=3) == -1                         # unknown kernel
    assert ex(kernel=1, dtype=0) == -4                # tensor cores on fp32
    assert ex(spl=-1, variant=2) == -1
    assert ex(debug=9) == -1
    need = ra.varlen_workspace_size(cu, H, D, N, "zigzag")
    assert ex(ws=FAKE + 16, nbytes=need) == -3        # workspace not 256-byte aligned
    assert ex(ws=FAKE, nbytes=need - 1) == -5         # workspace too small
    need = ra.varlen_workspace_size(cu, H, D, N, "zigzag", 1, "per_step")
    assert ex(variant=2, spl=3, ws=FAKE, nbytes=need - acc) == -5  # 3 launches need the results


def test_ring_step_validates_before_any_cuda_call():
    lib = ra.lib()

    def step(S=64, n_ring=4, shard=0, step=0, reserved=0, q=FAKE, O=FAKE, layout=1):
        return lib.ra_ring_step(q, FAKE, FAKE, O, FAKE, 1, 2, S, 64, n_ring, 1, layout, 1, shard, step, reserved,
                                None, 0, None)
    assert step(S=63) == -2             # S % n_ring
    assert step(shard=4) == -1          # query shard outside the ring
    assert step(shard=-1) == -1
    assert step(step=4) == -1           # ring step outside [0, n_ring)
    assert step(reserved=-1) == -1
    assert step(q=0) == -1
    assert step(O=FAKE + 8) == -3       # running output must be 16-byte aligned
    assert step(layout=5) == -1
    assert lib.ra_ring_finalize(FAKE, FAKE, FAKE, FAKE, 1, 2, 0, 64, 1, None) == -1
    assert lib.ra_ring_finalize(FAKE, FAKE, FAKE + 4, FAKE, 1, 2, 16, 64, 1, None) == -3


def test_ring_step_workspace_covers_every_shard_and_step():
    B, H, D, N = 2, 3, 128, 8
    S = N * 1000
    n = ra.ring_step_workspace_size(B, H, S, D, N, True, "zigzag", 1)
    a256 = lambda x: -(-x // 256) * 256
    rows = B * (S // N) * H
    pairs = -(-(S // N) // 256)
    assert n == 256 + a256(B * H * pairs * 16) + a256(2 * B * H * 4) + a256(rows * D * 4) + a256(rows * 4)
    simt = ra.ring_step_workspace_size(B, H, S, 40, N, True, "zigzag", 0)
    assert simt == a256(rows * 40 * 4) + a256(rows * 4)


def test_steps_per_launch_policy():
    # FUSED covers every step; PER_STEP takes the request (0 -> 1, clamped to n_ring)
    assert ra.steps_per_launch(4096, 128, 8, "striped", 1, "fused") == 8
    assert ra.steps_per_launch(4096, 128, 8, "striped", 1, "per_step", 0) == 1
    assert ra.steps_per_launch(4096, 128, 8, "striped", 1, "per_step", 3) == 3
    assert ra.steps_per_launch(4096, 128, 8, "striped", 1, "per_step", 99) == 8
    # AUTO: fused while a head's K/V (2 * S * D * 2 bytes) fits 96 MB -- s128k (64 MB) stays fused;
    # s1m (512 MB, 16 MB per block) takes launches of 6 steps (96 MB), evened out over 32 steps
    assert ra.steps_per_launch(131072, 128, 16, "striped", 1, "auto") == 16
    assert ra.steps_per_launch(1 << 20, 128, 32, "striped", 1, "auto") == 6
    assert ra.steps_per_launch(262144, 128, 32, "striped", 1, "auto") == 16
    # the workspace of AUTO follows the path it takes: none of the per-step buffers for s128k
    fused = ra.workspace_size(1, 32, 131072, 128, 16, True, "striped", 1, variant="fused")
    assert ra.workspace_size(1, 32, 131072, 128, 16, True, "striped", 1, variant="auto") == fused
    per_step = ra.workspace_size(1, 4, 1 << 20, 128, 32, True, "striped", 1, variant="per_step")
    auto = ra.workspace_size(1, 4, 1 << 20, 128, 32, True, "striped", 1, variant="auto")
    assert auto <= per_step and auto > 2 * (1 << 20) * 4 * 128 * 4  # running and step partials
    assert ra.lib().ra_steps_per_launch(4096, 128, 8, 1, 1, 2, -1, ctypes.byref(ctypes.c_int())) == -1
