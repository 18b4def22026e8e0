"""The host ring driver (long_context_exact_forward_b200.ring) over real process groups: gloo ranks on
the CPU, world sizes 2 to 4.

The compute of one step is a plain fp64 torch implementation written here -- the partial attention
of a query shard against one key/value block, with the causal mask on global positions, merged into
the running result in log-sum-exp form -- so that these tests exercise what the driver owns: which
block each rank holds at each step, the double-buffered exchange with its block index, and the
failure paths (a rank that raises between steps, a dropped message, a rank that never joins, ranks
that disagree on the problem).  The assembled result of a whole ring is compared with the fp64
oracle on the full sequence.
"""
import datetime
import math
import os
import queue
import socket
import sys
import time
import traceback

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def positions(S, N, layout):
    sys.path.insert(0, ROOT)
    import oracle
    return oracle.layout_positions(S, N, layout)


def make_cpu_step(S, N, layout, causal, log, fail_at=None):
    """fp64 step: partial attention of shard `shard` against block j = (shard - step) mod N, merged
    into (O, lse) -- O [B, S_loc, H, D], lse [B, S_loc, H]."""
    pos = positions(S, N, layout)

    def step(q, k_j, v_j, O, lse, n, shard, s):
        if fail_at is not None and s == fail_at:
            raise ValueError(f"planted failure at step {s}")
        j = (shard - s) % n
        log.append(j)
        D = q.shape[-1]
        sc = torch.einsum("bahd,bchd->bhac", q, k_j) / math.sqrt(D)
        if causal:
            allowed = torch.from_numpy(pos[j][None, :] <= pos[shard][:, None])
            sc = sc.masked_fill(~allowed, float("-inf"))
        m = sc.amax(-1, keepdim=True)
        empty = torch.isinf(m)
        p = torch.exp(sc - torch.where(empty, torch.zeros_like(m), m))
        l = p.sum(-1)  # [B, H, Sq]
        o = torch.einsum("bhac,bchd->bahd", p, v_j) / l.permute(0, 2, 1).unsqueeze(-1)
        o = torch.nan_to_num(o, nan=0.0)
        lse_s = (m.squeeze(-1) + torch.log(l)).permute(0, 2, 1)  # [B, Sq, H]; -inf when empty
        if s == 0:
            O.copy_(o)
            lse.copy_(lse_s)
            return
        mx = torch.maximum(lse, lse_s)
        safe = torch.where(torch.isinf(mx), torch.zeros_like(mx), mx)
        wr, ws = torch.exp(lse - safe), torch.exp(lse_s - safe)
        tot = wr + ws
        O.copy_(torch.nan_to_num((wr.unsqueeze(-1) * O + ws.unsqueeze(-1) * o) / tot.unsqueeze(-1), nan=0.0))
        lse.copy_(safe + torch.log(tot))

    return step


def cpu_finalize(O, lse):
    return O.clone(), lse.permute(0, 2, 1).contiguous()


class DroppingExchange:
    """P2P exchange that leaves out the K/V send of one step on one rank (a lost message)."""

    def __init__(self, rank, drop_rank, drop_step):
        from long_context_exact_forward_b200.ring import P2PExchange
        self.inner, self.rank, self.drop_rank, self.drop_step, self.step = P2PExchange(), rank, drop_rank, drop_step, 0

    def start(self, send, send_tag, recv, recv_tag, nxt, prv, group):
        import torch.distributed as dist
        s, self.step = self.step, self.step + 1
        if self.rank == self.drop_rank and s == self.drop_step:
            ops = [dist.P2POp(dist.isend, send_tag, nxt, group), dist.P2POp(dist.irecv, recv, prv, group),
                   dist.P2POp(dist.irecv, recv_tag, prv, group)]
            return dist.batch_isend_irecv(ops)
        return self.inner.start(send, send_tag, recv, recv_tag, nxt, prv, group)

    def finish(self, works, timeout):
        self.inner.finish(works, timeout)


def _worker(rank, world, port, cfg, results):
    code = 0
    store = None
    try:
        sys.path.insert(0, ROOT)
        import torch.distributed as dist
        from long_context_exact_forward_b200 import inputs
        from long_context_exact_forward_b200.ring import RingError, ring_attention
        store = dist.TCPStore("127.0.0.1", port, world, rank == 0, timeout=datetime.timedelta(seconds=30))
        dist.init_process_group("gloo", store=store, rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=cfg.get("pg_timeout", 20)))
        B, S, H, D, layout, causal = cfg["B"], cfg["S"], cfg["H"], cfg["D"], cfg["layout"], cfg["causal"]
        if cfg.get("absent_rank") == rank:
            time.sleep(cfg.get("absent_s", 8))
            results.put((rank, "absent", None))
            return
        if cfg.get("other_mask_rank") == rank:
            causal = not causal
        q, k, v = inputs.make_qkv(B, S, H, D, torch.float64, "cpu", seed=cfg["seed"])
        pos = positions(S, world, layout)[rank]
        qi, ki, vi = (t[:, torch.from_numpy(pos)].contiguous() for t in (q, k, v))
        log = []
        step = make_cpu_step(S, world, layout, causal, log,
                             fail_at=cfg.get("fail_step") if cfg.get("fail_rank") == rank else None)
        exchange = None
        if "drop_rank" in cfg:
            exchange = DroppingExchange(rank, cfg["drop_rank"], cfg["drop_step"])
        try:
            out, lse = ring_attention(qi, ki, vi, causal, layout, store=store, timeout=cfg.get("timeout", 20),
                                      step_fn=step, finalize_fn=cpu_finalize, exchange=exchange,
                                      acc_dtype=torch.float64)
            results.put((rank, "ok", (out.numpy(), lse.numpy(), log)))
        except RingError as exc:
            results.put((rank, "RingError", str(exc)))
        except Exception as exc:
            results.put((rank, type(exc).__name__, str(exc)))
    except Exception:
        results.put((rank, "crash", traceback.format_exc()))
        code = 1
    finally:
        results.close()
        results.join_thread()
        if store is not None:  # rank 0 hosts the store: keep it up until every rank has reported
            try:
                store.add("ring_test/done", 1)
                if rank == 0:
                    deadline = time.time() + 15
                    while store.add("ring_test/done", 0) < world and time.time() < deadline:
                        time.sleep(0.05)
            except Exception:
                pass
        os._exit(code)  # pending gloo requests of a failed ring must not hold the process


def run_ring(world, cfg, limit=90):
    ctx = mp.get_context("spawn")
    results = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, cfg, results)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    deadline = time.time() + limit
    try:
        while len(got) < world and time.time() < deadline:
            try:
                r, kind, payload = results.get(timeout=1.0)
                got[r] = (kind, payload)
            except queue.Empty:
                if all(not p.is_alive() for p in procs) and results.empty():
                    break
    finally:
        for p in procs:
            p.join(timeout=5)
            if p.is_alive():
                p.kill()
                p.join()
    return got


BASE = dict(B=1, H=2, D=8, seed=11)


@pytest.mark.parametrize("world, layout, causal, S", [
    (2, "striped", True, 2 * 24),
    (3, "zigzag", True, 3 * 20),
    (4, "contiguous", False, 4 * 12),
    (4, "striped", True, 4 * 10),
    (4, "contiguous", True, 4 * 9),
])
def test_ring_equals_full_attention(world, layout, causal, S):
    sys.path.insert(0, ROOT)
    import oracle
    from long_context_exact_forward_b200 import inputs
    cfg = dict(BASE, S=S, layout=layout, causal=causal)
    got = run_ring(world, cfg)
    assert sorted(got) == list(range(world)), got
    for r in range(world):
        assert got[r][0] == "ok", got[r]
    q, k, v = inputs.make_qkv(1, S, 2, 8, torch.float64, "cpu", seed=11)
    ref, ref_lse = oracle.attention(q, k, v, causal)
    pos = oracle.layout_positions(S, world, layout)
    out = np.empty((1, S, 2, 8))
    lse = np.empty((1, 2, S))
    for r in range(world):
        o, l, log = got[r][1]
        assert log == [(r - s) % world for s in range(world)]  # block j = (i - s) mod N at step s
        out[:, pos[r]] = o
        lse[:, :, pos[r]] = l
    assert np.abs(out.transpose(0, 2, 1, 3) - ref).max() <= 1e-12
    assert np.abs(lse - ref_lse).max() <= 1e-12


def test_rank_that_raises_stops_the_others():
    cfg = dict(BASE, S=3 * 8, layout="striped", causal=True, fail_rank=1, fail_step=0, timeout=5)
    got = run_ring(3, cfg)
    assert got[1][0] == "ValueError" and "planted failure" in got[1][1]
    for r in (0, 2):
        assert got[r][0] == "RingError", got[r]
        assert "rank 1" in got[r][1]


def test_dropped_message_times_out():
    cfg = dict(BASE, S=2 * 8, layout="contiguous", causal=True, drop_rank=0, drop_step=0, timeout=3)
    got = run_ring(2, cfg)
    assert got[1][0] == "RingError", got[1]
    assert "did not arrive" in got[1][1]


def test_rank_that_never_joins_ends_with_the_group_timeout():
    cfg = dict(BASE, S=2 * 8, layout="striped", causal=True, absent_rank=1, absent_s=10, pg_timeout=3)
    t0 = time.time()
    got = run_ring(2, cfg)
    assert got[0][0] == "RingError" and "could not agree" in got[0][1], got[0]
    assert time.time() - t0 < 60


def test_ranks_that_disagree_on_the_problem_are_named():
    cfg = dict(BASE, S=2 * 8, layout="striped", causal=True, other_mask_rank=1)
    got = run_ring(2, cfg)
    for r in (0, 1):
        assert got[r][0] == "RingError" and "different problem" in got[r][1], got[r]
