#!/usr/bin/env python
"""Throughput of the exact ring-attention forward on B200: attention TFLOP/s (causal counted as
half) on the s128k workload -- batch 1, 32 heads, head dim 128, 131072 tokens in 16 shards of
8192, bf16, causal, striped layout -- with synthetic seeded inputs resident in HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  `value` is device-timed (CUDA events around K back-to-back calls,
max over ranks); `e2e` repeats the measurement through the public API with the inputs copied from
pinned host memory and the result copied back inside the timed region; `roofline` is the
attention kernel alone, timed with the library's event hook; `cpu_baseline` is the fp64 oracle on
a bounded sample of the same workload on the host cores.  `--impl reference` times that oracle
as the reference arm.  Inputs (3.2 GB) exceed the 126 MB L2, so no flush is needed.
Under torchrun with N > 1 every rank runs its own replica (the virtual ring lives on one GPU;
there is no data-path collective) and `value` sums the ranks' work over the slowest rank's time.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from long_context_exact_forward_b200 import inputs  # noqa: E402

METRIC = "ring-attn fwd TFLOP/s (bf16, causal) and % of B200 dense BF16 tensor peak"
# --backward runs: gradient flops counted as 2.5x the forward flops (five S x S x D products:
# the recomputed scores, dP, dV, dQ, dK), halved for causal like the forward
METRIC_BWD = "ring-attn bwd TFLOP/s (causal; 2.5x forward flops)"
# --varlen runs: packed sequences, flops summed per sequence (4 * H * len^2 * D, halved for causal)
METRIC_VARLEN = "ring-attn fwd TFLOP/s over packed variable-length sequences (bf16, causal)"


def ring_word(args):
    """How the attention launches walk the ring steps, for the roofline's kernel name."""
    if args.variant != "per_step":
        return "fused ring" if args.varlen or args.variant == "fused" else "ring, variant auto"
    return f"{args.steps_per_launch or 1} ring step(s) per launch"


def varlen_lengths(S, n_ring, seed):
    """A seeded mix of sequence lengths that fills S tokens: multiples of 128 * n_ring between
    S / 64 and S / 4 (the last one takes what is left)."""
    import random
    rng = random.Random(seed)
    unit = 128 * n_ring
    lo, hi = max(1, S // 64 // unit), max(1, S // 4 // unit)
    out, left = [], S
    while left > 0:
        n = min(rng.randint(lo, hi) * unit, left)
        out.append(n)
        left -= n
    return out
UNIT = "TFLOP/s"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM bytes (read + write) per attention launch on s128k striped, from an ncu capture of the
# 4-head case (dram__bytes_read.sum + dram__bytes_write.sum) scaled by heads; valid only while
# the sha256 of the TRAFFIC_SOURCES files, concatenated in that order, starts with the recorded
# prefix -- otherwise traffic is null.
TRAFFIC_RECORD = {"source_sha256_prefix": "489c96f8d0891039", "bytes_per_launch": (3.463295e9 + 0.140089e9) * 8}
# the files whose concatenation the record's hash covers: the kernel, the helpers it inlines and
# the host code that decides the layout it reads
TRAFFIC_SOURCES = ("attn_tc.cu", "sm100.cuh", "layout.cuh", "api.cu")


def recorded_traffic(args):
    """DRAM bytes per launch recorded for this exact kernel and host code (which decides the
    layout the kernel reads), or None."""
    import hashlib
    h = hashlib.sha256()
    for rel in TRAFFIC_SOURCES:
        try:
            h.update(open(os.path.join(ROOT, "long_context_exact_forward_b200", "csrc", rel), "rb").read())
        except OSError:
            return None
    default_run = (args.workload == "s128k" and args.layout == "striped" and args.heads in (0, 32)
                   and args.kernel == "tc" and args.variant == "fused")
    if default_run and h.hexdigest().startswith(TRAFFIC_RECORD["source_sha256_prefix"]):
        return TRAFFIC_RECORD["bytes_per_launch"]
    return None


def attention_flops(B, H, S, D, causal):
    """4 * B * H * S^2 * D, halved when causal (the convention of the target metric)."""
    f = 4.0 * B * H * S * S * D
    return f / 2 if causal else f


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except OSError:
        return PEAKS_FALLBACK, "fallback"


# ------------------------------------------------------------------ clocks during the timed region
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device):
        self.lines = []
        self.proc = None
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", uuid, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, AttributeError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, power, reasons = [], [], [], set()
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for name, val in zip(self.REASONS, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        # samples under load: power within 60% of the run's peak draw
        pmax = max(power)
        loaded = [s for s, p in zip(sm, power) if p >= 0.6 * pmax] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": pmax}


# ------------------------------------------------------------------ distributed plumbing
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(x, world, device="cuda"):
    """The slowest rank's value (timings are reported as the max over ranks)."""
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.item()


def job_throughput(flops_per_rank, world, ms_per_step):
    """Whole-job TFLOP/s: every rank's work over the slowest rank's time (weak scaling)."""
    return world * flops_per_rank / (ms_per_step / 1e3) / 1e12


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


# ------------------------------------------------------------------ oracle on the host cores
def oracle_sample(q, k, v, causal, rows_per_head, seed_base=7000):
    """Time the oracle on `rows_per_head` uniformly drawn query rows of every head."""
    import oracle  # test-side fp64 reference: only this CPU-baseline leg runs it
    B, S, H, D = q.shape
    rows = np.stack([np.sort(np.random.default_rng(seed_base + h).choice(S, rows_per_head, replace=False))
                     for h in range(H)])
    threads = os.cpu_count() or 1
    flops = B * sum(4.0 * D * ((r + 1) if causal else S) for r in rows.ravel())
    t0 = time.perf_counter()
    oracle.attention(q, k, v, causal, rows=rows, threads=threads)
    dt = time.perf_counter() - t0
    return flops, dt, threads, rows.size


def oracle_single_thread(q, k, v, causal, n_rows, seed=7000):
    """The same oracle on one host thread: `n_rows` uniformly drawn query rows of head 0."""
    import oracle  # test-side fp64 reference: only this CPU-baseline leg runs it
    B, S, H, D = q.shape
    rows = np.sort(np.random.default_rng(seed).choice(S, n_rows, replace=False))
    q0, k0, v0 = (t[:, :, :1].contiguous() for t in (q, k, v))
    flops = B * sum(4.0 * D * ((r + 1) if causal else S) for r in rows)
    t0 = time.perf_counter()
    oracle.attention(q0, k0, v0, causal, rows=rows, threads=1)
    return flops, time.perf_counter() - t0


def run_reference(args, w):
    """Reference arm: the fp64 oracle, as it stands, on the host cores (rank 0 only)."""
    world, rank, _ = dist_env()
    if rank != 0:
        return
    q, k, v = inputs.make_qkv(w.B, w.S, w.H, w.D, torch.float32 if args.dtype == "fp32" else torch.bfloat16,
                              "cpu", w.seed)
    rows_per_head = args.ref_rows
    causal = causal_of(args)
    for _ in range(args.warmup):
        oracle_sample(q, k, v, causal, rows_per_head)
    tot_f, tot_t = 0.0, 0.0
    for _ in range(args.steps):
        f, dt, threads, n = oracle_sample(q, k, v, causal, rows_per_head)
        tot_f += f
        tot_t += dt
    value = tot_f / tot_t / 1e12
    sample = (f"{rows_per_head} query rows per head x {w.H} heads of {w.name} ({mask_word(args)}), "
              f"{tot_f / args.steps:.3e} flops per step")
    line = {
        "impl": "reference", "metric": metric_of(args), "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_t / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_dict(w, args),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def causal_of(args):
    return not getattr(args, "non_causal", False)


def mask_word(args):
    return "causal" if causal_of(args) else "non-causal"


def metric_of(args):
    """The metric named by the run: the headline forward metric, or that of a --backward /
    --varlen run; "causal" becomes "non-causal" under --non-causal."""
    m = METRIC_BWD if getattr(args, "backward", False) else METRIC_VARLEN if getattr(args, "varlen", False) else METRIC
    return m if causal_of(args) else m.replace("causal", "non-causal")


def config_dict(w, args):
    return {
        "workload": f"{w.name}: batch {w.B}, {w.H} heads, head dim {w.D}, {w.S} tokens in {w.n_ring} "
                    f"shards of {w.S_loc}, {args.dtype}, {'causal' if causal_of(args) else 'non-causal'}, "
                    f"{args.layout} layout",
        "B": w.B, "H": w.H, "S": w.S, "D": w.D, "n_ring": w.n_ring, "causal": causal_of(args),
        "layout": args.layout, "variant": args.variant, "kernel": args.kernel,
        **({"workspace": "allocated by every call"} if getattr(args, "no_workspace", False) else {}),
        **({"steps_per_launch": args.steps_per_launch} if args.variant == "per_step" else {}),
        "l2": f"inputs (3 x B*S*H*D {args.dtype}) larger than the 126 MB L2; no flush"
              if 3 * w.B * w.S * w.H * w.D * (4 if args.dtype == "fp32" else 2) > 126e6
              else "inputs smaller than the 126 MB L2 (kernel-level runs; not the headline)",
        **({"varlen_lengths": varlen_lengths(w.S, w.n_ring, w.seed)} if getattr(args, "varlen", False) else {}),
    }


def hbm_kernels(ra, q, n_ring, layout, stream, reps=10):
    """Achieved DRAM bandwidth of the permute and merge kernels against the measured copy peak.

    permute: q [B, S, H, D] bf16 -> shard-major copy; algorithmic bytes = read + write of q.
    merge:   one ring step's partial folded into the running result (fp32 [B*S*H, D] and
             lse [B*S*H]); algorithmic bytes = 12 per output element + 12 per row.
    rope:    rotary embedding of q with global positions, out of place; bytes = read + write of q.
    """
    peaks, src = load_peaks()
    res = {"peak_gbs": peaks["hbm_gbs"], "peak_kind": f"copy ({src})"}
    y = torch.empty((q.shape[0], n_ring, q.shape[1] // n_ring, q.shape[2], q.shape[3]), dtype=q.dtype,
                    device=q.device)
    lay = layout if layout != "contiguous" else "striped"

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps

    ms = timed(lambda: ra.permute(q, n_ring, lay, out=y, stream=stream))
    byts = 2.0 * q.numel() * q.element_size()
    res["permute"] = {"layout": lay, "ms": ms, "bytes": byts, "achieved_gbs": byts / ms / 1e6,
                      "frac": byts / ms / 1e6 / peaks["hbm_gbs"]}
    del y
    rows, D = q.numel() // q.shape[-1], q.shape[-1]
    g = torch.Generator(device=q.device).manual_seed(0)
    O_r = torch.randn(rows, D, device=q.device, generator=g)
    O_s = torch.randn(rows, D, device=q.device, generator=g)
    l_r = torch.randn(rows, device=q.device, generator=g)
    l_s = torch.randn(rows, device=q.device, generator=g)
    ms = timed(lambda: ra.merge_partials(O_r, l_r, O_s, l_s, stream=stream))
    byts = 12.0 * rows * D + 12.0 * rows
    res["merge"] = {"rows": rows, "D": D, "ms": ms, "bytes": byts, "achieved_gbs": byts / ms / 1e6,
                    "frac": byts / ms / 1e6 / peaks["hbm_gbs"]}
    del O_r, O_s, l_r, l_s
    yr = torch.empty_like(q)
    ms = timed(lambda: ra.rope(q, out=yr, stream=stream))
    byts = 2.0 * q.numel() * q.element_size()
    res["rope"] = {"ms": ms, "bytes": byts, "achieved_gbs": byts / ms / 1e6, "frac": byts / ms / 1e6 / peaks["hbm_gbs"]}
    return res


# ------------------------------------------------------------------ our arm
def run_ours(args, w):
    import long_context_exact_forward_b200 as ra
    world, rank, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    B, H, S, D, N = w.B, w.H, w.S, w.D, w.n_ring
    fp32 = args.dtype == "fp32"
    q, k, v = inputs.make_qkv(B, S, H, D, torch.float32 if fp32 else torch.bfloat16, dev, w.seed + rank)
    out = torch.empty_like(q)
    lse = torch.empty((B, H, S), dtype=torch.float32, device=dev)
    causal = causal_of(args)
    ws = torch.empty(ra.workspace_size(B, H, S, D, N, causal, args.layout, 0 if fp32 else 1,
                                       variant=args.variant, kernel=args.kernel),
                     dtype=torch.uint8, device=dev)
    flops = attention_flops(B, H, S, D, causal)

    if args.no_workspace:  # every call allocates and frees its own scratch (the library's pool)
        ws = None

    def step(ev=None):
        ra.forward(q, k, v, N, causal, args.layout, variant=args.variant, kernel=args.kernel, out=out,
                   lse=lse, workspace=ws, stream=stream, events=ev, steps_per_launch=args.steps_per_launch)

    if args.varlen:
        lengths = varlen_lengths(S, N, w.seed)
        cu = [0]
        for n in lengths:
            cu.append(cu[-1] + n)
        lse_v = torch.empty((H, S), dtype=torch.float32, device=dev)
        ws_v = torch.empty(ra.varlen_workspace_size(cu, H, D, N, args.layout, 0 if fp32 else 1, args.variant,
                                                    args.kernel), dtype=torch.uint8, device=dev)
        flops = sum(attention_flops(1, H, n, D, causal) for n in lengths)

        def step(ev=None):  # ev: recorded by the library around the attention launches
            ra.forward_varlen(q[0], k[0], v[0], cu, N, causal, args.layout, variant=args.variant, kernel=args.kernel,
                              steps_per_launch=args.steps_per_launch, out=out[0], lse=lse_v, workspace=ws_v,
                              stream=stream, events=ev)

    if args.backward:
        # one forward pass outside the timed region supplies out and lse; a step is one ra_backward
        gen = torch.Generator(device=dev).manual_seed(w.seed + 1000 + rank)
        dout = torch.randn(q.shape, generator=gen, device=dev, dtype=torch.float32).to(q.dtype)
        step()
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        flops = 2.5 * attention_flops(B, H, S, D, causal)

        def step(ev=None):
            if ev is not None:
                ev[0].record(stream)
            ra.backward(q, k, v, out, lse, dout, N, causal, args.layout, kernel=args.bwd_kernel, dq=dq, dk=dk,
                        dv=dv, stream=stream)
            if ev is not None:
                ev[1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert ra.get_device_status() == 0

    # ---- device-timed region: K calls back to back, inputs resident in HBM
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    clocks = ClockSampler(dev)
    start.record(stream)
    for s in range(args.steps):
        step(kev[s])
    end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier(world)
    ms = max_over_ranks(start.elapsed_time(end), world)
    kernel_ms = [a.elapsed_time(b) for a, b in kev]
    status = ra.get_device_status()
    ms_per_step = ms / args.steps
    value = job_throughput(flops, world, ms_per_step)

    # ---- end to end through the public API: every step copies its inputs from pinned host memory
    #      to the device and its result (out, lse) back.  Pipelined: copies run on their own
    #      streams into double-buffered device tensors, so step s+1's inputs travel while step s
    #      computes (what a caller streaming many sequences does).  The serial form, where every
    #      copy waits for the previous call, is reported beside it.
    e2e = None
    if not args.no_e2e:
        qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
        oh = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
        lh = [torch.empty(lse.shape, dtype=lse.dtype).pin_memory() for _ in range(2)]
        dq = [[torch.empty_like(q) for _ in range(3)] for _ in range(2)]
        do = [torch.empty_like(q) for _ in range(2)]
        dl = [torch.empty_like(lse) for _ in range(2)]
        h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_free_in = [torch.cuda.Event() for _ in range(2)]
        ev_free_out = [torch.cuda.Event() for _ in range(2)]

        def pipelined(n_steps):
            for st in range(n_steps):
                b = st % 2
                with torch.cuda.stream(h2d):
                    if st >= 2:
                        h2d.wait_event(ev_free_in[b])
                    for dst, src in zip(dq[b], (qh, kh, vh)):
                        dst.copy_(src, non_blocking=True)
                    ev_in[b].record(h2d)
                stream.wait_event(ev_in[b])
                if st >= 2:
                    stream.wait_event(ev_free_out[b])
                ra.forward(dq[b][0], dq[b][1], dq[b][2], N, causal, args.layout, variant=args.variant, kernel=args.kernel,
                           out=do[b], lse=dl[b], workspace=ws, stream=stream, steps_per_launch=args.steps_per_launch)
                ev_free_in[b].record(stream)
                ev_done[b].record(stream)
                with torch.cuda.stream(d2h):
                    d2h.wait_event(ev_done[b])
                    oh[b].copy_(do[b], non_blocking=True)
                    lh[b].copy_(dl[b], non_blocking=True)
                    ev_free_out[b].record(d2h)

        pipelined(2)
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(h2d)
        pipelined(args.steps)
        e1.record(d2h)
        torch.cuda.synchronize()
        ems = max_over_ranks(e0.elapsed_time(e1), world) / args.steps

        def serial_step():
            for dst, src in zip(dq[0], (qh, kh, vh)):
                dst.copy_(src, non_blocking=True)
            ra.forward(dq[0][0], dq[0][1], dq[0][2], N, causal, args.layout, variant=args.variant, kernel=args.kernel,
                       out=do[0], lse=dl[0], workspace=ws, stream=stream, steps_per_launch=args.steps_per_launch)
            oh[0].copy_(do[0], non_blocking=True)
            lh[0].copy_(dl[0], non_blocking=True)

        serial_step()
        torch.cuda.synchronize()
        barrier(world)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for _ in range(args.steps):
            serial_step()
        s1.record(stream)
        torch.cuda.synchronize()
        sms = max_over_ranks(s0.elapsed_time(s1), world) / args.steps
        bi = 3 * q.numel() * q.element_size()
        bo = out.numel() * out.element_size() + lse.numel() * lse.element_size()
        e2e = {"value": job_throughput(flops, world, ems), "unit": UNIT, "h2d_bytes_per_step": bi,
               "d2h_bytes_per_step": bo, "ms_per_step": ems,
               "form": "copies on their own streams, double-buffered, overlapping the previous step",
               "serial": {"value": job_throughput(flops, world, sms), "ms_per_step": sms}}
        del qh, kh, vh, oh, lh, dq, do, dl

    # ---- the HBM-bound kernels (permute of q into shard-major order; one per-step merge),
    #      timed alone on this workload's sizes, outside the timed region
    hbm = None
    if not args.no_hbm_kernels:
        hbm = hbm_kernels(ra, q, N, args.layout, stream)

    # ---- roofline of the dominant kernel (the attention kernel)
    peaks, peak_src = load_peaks()
    k_ms = statistics.mean(kernel_ms)
    achieved = flops / (k_ms / 1e3) / 1e12
    bwd_tc = args.backward and args.bwd_kernel != "simt" and not fp32 and D in (64, 128)
    if args.kernel == "simt" or (args.backward and not bwd_tc):
        # FP32 pipe: 148 SMs x 128 FMA lanes x 2 flops at the sampled maximum SM clock
        peak = 148 * 128 * 2 * (clk.get("sm_max_mhz") or 1965.0) * 1e6 / 1e12
        roofline = {
            "bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "traffic": args.traffic_bytes,
            "peak_kind": "FP32 FMA pipe (148 SMs x 128 lanes x 2 flops x max SM clock; derived)",
            "kernel": ("bwd_delta + bwd_dq + bwd_dkv kernels (fp32 arithmetic), timed as one ra_backward call"
                       if args.backward else f"attn_simt_kernel<{'float' if fp32 else 'bf16'}> (fp32 arithmetic)"),
            "kernel_ms": k_ms,
            "algorithmic_flops_per_launch": flops,
        }
    else:
        peak = peaks["bf16_tflops_sustained"]
        roofline = {
            "bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "traffic": (args.traffic_bytes if args.traffic_bytes is not None
                        else None if (args.backward or args.varlen) else recorded_traffic(args)),
            "peak_kind": f"bf16 dense cuBLAS, sustained ({peak_src})",
            "frac_of_burst_peak": achieved / peaks["bf16_tflops"],
            "kernel": ("bwd_dq_tc_kernel + bwd_dkv_tc_kernel (tcgen05), timed as one ra_backward call"
                       if args.backward else
                       f"attn_tc_kernel<128, varlen> ({ring_word(args)}, tcgen05)"
                       if args.varlen else f"attn_tc_kernel<128> ({ring_word(args)}, tcgen05)"),
            "kernel_ms": k_ms,
            "algorithmic_flops_per_launch": flops,
        }

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, N = 1 only)
    cpu = None
    if not args.no_cpu_baseline and world == 1 and rank == 0:
        qc, kc, vc = q.cpu(), k.cpu(), v.cpu()
        f, dt, threads, n = oracle_sample(qc, kc, vc, causal, args.cpu_rows)
        cpu = {"value": f / dt / 1e12, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"{args.cpu_rows} query rows per head x {H} heads of {w.name} ({mask_word(args)}), "
                         f"{f:.3e} flops in {dt:.1f} s"}
        if args.cpu_rows_single > 0:
            f1, dt1 = oracle_single_thread(qc, kc, vc, causal, min(args.cpu_rows_single, w.S))
            cpu["single_thread"] = {"value": f1 / dt1 / 1e12, "unit": UNIT, "cores": 1,
                                    "sample": f"{min(args.cpu_rows_single, w.S)} query rows of head 0 of "
                                              f"{w.name} ({mask_word(args)}), {f1:.3e} flops in {dt1:.1f} s"}

    # our kernels per step: the zigzag permute (striped and contiguous are read in place, and the
    # CUDA-core kernel reads natural order) and the attention launch(es) -- with chunks of C ring
    # steps per launch: ceil(N / C) attention launches and one merge after each but the first
    # (2 kernels each, the last one a single final merge)
    # the tensor-core path also launches the query/key norm pre-pass (one kernel per call) when it pays
    chunk = ra.steps_per_launch(S, D, N, args.layout, 0 if fp32 else 1, args.variant, args.steps_per_launch)
    if args.varlen:  # packed sequences: one launch unless per-step launches are asked for
        chunk = min(N, args.steps_per_launch or 1) if args.variant == "per_step" else N
    n_att = -(-N // chunk)
    tc = args.kernel == "tc"
    # the score-bound pre-pass runs when each query row meets >= 32768 keys per launch (RA_DEBUG_FROZEN_MAX
    # in include/ra.h): chunk x S/N keys, or for packed sequences sum(len^2) / S of them per ring pass
    keys_per_row = (sum(n * n for n in varlen_lengths(S, N, w.seed)) / S if args.varlen else S) * chunk / N
    norms = 1 if tc and keys_per_row >= 32768 else 0
    launches_per_step = (1 if args.layout == "zigzag" and tc else 0) + norms + (
        1 if n_att == 1 else n_att + 2 * (n_att - 2) + 1)
    if args.backward:
        # Delta, dq, dk/dv; the tensor-core kernels read zigzag from one shard-major permute launch
        tc_bwd = args.bwd_kernel == "tc" or (args.bwd_kernel == "auto" and args.dtype == "bf16" and D in (64, 128))
        launches_per_step = 3 + (1 if args.layout == "zigzag" and tc_bwd else 0)
    line = {
        "metric": metric_of(args), "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32" if fp32 else "bf16", "data": "synthetic",
        "config": config_dict(w, args),
        "pct_of_bf16_peak": {"burst_measured": value / world / peaks["bf16_tflops"],
                             "sustained_measured": value / world / peaks["bf16_tflops_sustained"],
                             "nvidia_dense_spec_2250": value / world / 2250.0},
        "clocks": clk, "e2e": e2e, "roofline": roofline, "cpu_baseline": cpu, "hbm_kernels": hbm,
        "gpu_launches": launches_per_step * args.steps, "device_status": status,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="s128k", choices=sorted(inputs.WORKLOADS))
    ap.add_argument("--layout", default="striped", choices=["contiguous", "striped", "zigzag"])
    ap.add_argument("--variant", default="fused", choices=["fused", "per_step", "auto"])
    ap.add_argument("--steps-per-launch", type=int, default=0,
                    help="per_step variant: ring steps covered by each attention launch (0 = one)")
    ap.add_argument("--heads", type=int, default=0, help="override the head count (profiling runs)")
    ap.add_argument("--kernel", default="tc", choices=["tc", "simt"],
                    help="tc: the tcgen05 kernel (the headline); simt: the fp32 CUDA-core kernel")
    ap.add_argument("--dtype", default="bf16", choices=["bf16", "fp32"])
    ap.add_argument("--non-causal", action="store_true",
                    help="no causal mask (flops not halved; not the headline)")
    ap.add_argument("--bwd-kernel", default="auto", choices=["auto", "tc", "simt"],
                    help="backward path for --backward runs (auto: tensor cores where they apply)")
    ap.add_argument("--varlen", action="store_true",
                    help="time ra_forward_varlen over a seeded mix of packed sequences filling the workload's "
                         "tokens (needs --no-e2e --no-cpu-baseline; not the headline)")
    ap.add_argument("--backward", action="store_true",
                    help="time ra_backward (needs --no-e2e and --no-cpu-baseline; not the headline)")
    ap.add_argument("--no-workspace", action="store_true",
                    help="call ra_forward without a caller workspace, so that every call allocates its scratch")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-hbm-kernels", action="store_true")
    ap.add_argument("--cpu-rows", type=int, default=256, help="oracle rows per head for cpu_baseline")
    ap.add_argument("--cpu-rows-single", type=int, default=64,
                    help="oracle rows of one head for cpu_baseline's single-thread rate (0: skip)")
    ap.add_argument("--ref-rows", type=int, default=64, help="oracle rows per head per reference step")
    ap.add_argument("--traffic-bytes", type=float, default=None,
                    help="DRAM bytes per attention launch from an ncu capture of this kernel")
    args = ap.parse_args()
    if (args.backward or args.varlen) and not (args.no_e2e and args.no_cpu_baseline):
        ap.error("--backward / --varlen runs time the device call only: add --no-e2e --no-cpu-baseline")
    if args.backward and args.varlen:
        ap.error("--backward and --varlen are separate runs")
    if args.impl == "reference" and (args.backward or args.varlen):
        ap.error("--impl reference times the oracle of the batch forward pass; --backward and --varlen "
                 "have no reference arm")
    if args.kernel == "tc" and args.dtype == "fp32":
        ap.error("the tensor-core kernel takes bf16 inputs; fp32 runs on --kernel simt")
    w = inputs.WORKLOADS[args.workload]
    if args.heads:
        from dataclasses import replace
        w = replace(w, H=args.heads)
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
