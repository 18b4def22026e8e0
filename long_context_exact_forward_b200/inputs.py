"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module holds random-number recipes and shapes only -- no attention arithmetic -- so that
both the CUDA path and the fp64 oracle can be fed identical tensors from it.

Workloads (the sizes the Ring Attention pages talk about, scaled to one B200):

=========  ====================================================================================
toy        4 shards x 8 tokens, head dim 16, 1 head, batch 1, fp32, non-causal: the ultralytics
           "Ring Attention" toy ring; q, k, v = the three slices of randn(3, 32, 16) drawn on the
           CPU after manual_seed(0).
s4k        batch 1, 32 heads, head dim 128, 4 shards x 1024 tokens, bf16, causal, contiguous.
s32k       batch 1, 32 heads, head dim 128, 8 shards x 4096 tokens, bf16, causal or not.
s128k      batch 1, 32 heads, head dim 128, 16 shards x 8192 tokens, bf16, causal; contiguous,
           striped or zigzag.
s1m        batch 1, 4 heads, head dim 128, 32 shards x 32768 tokens, bf16, causal, striped.
=========  ====================================================================================

bf16 inputs are N(0, 1) draws made in bf16 by torch's generator on the target device with seed
2, 3, 4, 5 respectively, packed as randn(3, B, S, H, D) and split into q, k, v.
"""
from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    S: int
    D: int
    n_ring: int
    dtype: str            # "fp32" or "bf16"
    causal: tuple         # causal settings the workload is run with
    layouts: tuple        # token layouts the workload is run with
    seed: int

    @property
    def S_loc(self):
        return self.S // self.n_ring


WORKLOADS = {
    "toy": Workload("toy", 1, 1, 32, 16, 4, "fp32", (False,), ("contiguous",), 0),
    "s4k": Workload("s4k", 1, 32, 4096, 128, 4, "bf16", (True,), ("contiguous",), 2),
    "s32k": Workload("s32k", 1, 32, 32768, 128, 8, "bf16", (False, True), ("contiguous",), 3),
    "s128k": Workload("s128k", 1, 32, 131072, 128, 16, "bf16", (True,),
                      ("contiguous", "striped", "zigzag"), 4),
    "s1m": Workload("s1m", 1, 4, 1048576, 128, 32, "bf16", (True,), ("striped",), 5),
}


def toy_qkv():
    """The toy's q, k, v as [1, 32, 1, 16] fp32 CPU tensors (manual_seed(0), randn(3, 32, 16))."""
    torch.manual_seed(0)
    q, k, v = torch.randn(3, 32, 16)
    return tuple(t.reshape(1, 32, 1, 16).contiguous() for t in (q, k, v))


def make_qkv(B, S, H, D, dtype=torch.bfloat16, device="cpu", seed=0, scale=1.0):
    """q, k, v ~ N(0, 1) drawn as one randn(3, B, S, H, D) with a seeded generator on `device`.

    `scale` multiplies q only (a sharper softmax for robustness cases); 1.0 leaves the draw as is.
    """
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    x = torch.randn((3, B, S, H, D), generator=gen, dtype=dtype, device=device)
    q, k, v = x[0], x[1], x[2]
    if scale != 1.0:
        q = (q.float() * scale).to(dtype)
    return q, k, v


def workload_qkv(w: Workload, device="cuda"):
    if w.name == "toy":
        q, k, v = toy_qkv()
        return q.to(device), k.to(device), v.to(device)
    return make_qkv(w.B, w.S, w.H, w.D, torch.bfloat16, device, w.seed)


def sample_rows(S, H, n=4096, extra_rows=(), seed_base=1000):
    """Per-head query rows to check: `extra_rows` first, then uniform draws without replacement
    from numpy default_rng(seed_base + h) until `n` distinct rows (all rows when S <= n).

    Returns an int64 array [H, n'] (n' = min(n, S)), each row sorted.
    """
    if S <= n:
        return np.tile(np.arange(S, dtype=np.int64), (H, 1))
    out = []
    extra = np.unique(np.asarray([r for r in extra_rows if 0 <= r < S], dtype=np.int64))
    for h in range(H):
        rng = np.random.default_rng(seed_base + h)
        chosen = set(extra.tolist())
        while len(chosen) < n:
            chosen.update(rng.choice(S, size=n - len(chosen), replace=False).tolist())
        rows = np.array(sorted(chosen), dtype=np.int64)[:n] if len(chosen) > n else np.array(sorted(chosen), dtype=np.int64)
        out.append(rows)
    return np.stack(out)
