"""Ring Attention across devices: one process per GPU, each holding one shard of the sequence.

Device i keeps its query block Q_i for the whole pass.  Its key/value block travels: at step s it
holds the block of device j = (i - s) mod N, computes the partial attention of Q_i against it and
merges the result into its running (O, lse), while that block is already on its way to device
i + 1 and block j - 1 is arriving from device i - 1.  After N steps every device holds exact
attention for its own queries (jisaku.com "Ring Attention", 処理フロー and 通信計算オーバーラップ;
ultralytics.com "Ring Attention", "how ring attention works"; troisinh.com "Ring Attention",
"Ý tưởng cốt lõi").

How this maps onto B200s:
  * K and V of a block travel together in one packed local buffer [2, B, S_loc, H, D], with the
    block's index beside them, by NCCL send/recv (torch.distributed point-to-point, which runs on
    NCCL's own stream).  Two such buffers alternate: step s computes on one while step s + 1's
    block lands in the other.  The per-step compute (ra_ring_step) only ever reads local memory
    through TMA: no peer pointer is a kernel operand and nothing is multicast.
  * The exchange of step s is posted before step s's compute is enqueued, so the transfer runs
    beside the compute; the compute stream waits for it only before the step that needs the block.
    The transfer is hidden when a block's compute takes longer than its send (the pages' overlap
    condition).  `sms_reserved` leaves SMs free for NCCL's kernel while the persistent attention
    kernel runs.
  * Every received block carries its index; a block that is not (i - s - 1) mod N raises
    RingError.  On CUDA the indices are gathered on the device and checked once at the end (no
    host synchronisation per step); on CPU backends they are checked as they arrive.

Failure detection (all on the host; nothing here waits inside a kernel):
  * the ranks first agree on the problem with one all_gather, so a rank that never arrives ends
    the call with the process group's timeout, and a rank with other shapes is named;
  * receives are bounded: `timeout` is passed to Work.wait on backends that honour it (gloo); on
    NCCL the process group's own timeout bounds them;
  * a rank whose step fails writes the reason into `store` (when one is given) before it raises;
    the others look for it before every step and raise RingError naming that rank.

The per-step compute and the final write are pluggable (`step_fn`, `finalize_fn`): by default
they are the library's ra_ring_step and ra_ring_finalize on the tensor's CUDA device.
"""
import datetime
import time

import torch
import torch.distributed as dist

ABORT_KEY = "ring_attention/abort"


class RingError(RuntimeError):
    """A ring pass could not complete: a peer failed, a transfer timed out or a block was wrong."""


def _device_step(layout, causal, sms_reserved, workspace):
    import long_context_exact_forward_b200 as ra

    def step(q, k_j, v_j, O_acc, lse_acc, n_ring, shard, step):
        ra.ring_step(q, k_j, v_j, O_acc, lse_acc, n_ring, shard, step, causal, layout,
                     sms_reserved=sms_reserved, workspace=workspace)

    return step


def _device_finalize(dtype):
    import long_context_exact_forward_b200 as ra

    def finalize(O_acc, lse_acc):
        return ra.ring_finalize(O_acc, lse_acc, dtype=dtype)

    return finalize


class P2PExchange:
    """Send this step's block to the next rank and receive the following one from the previous rank
    (one batch of point-to-point operations: packed K/V plus the block index, each way)."""

    def start(self, send, send_tag, recv, recv_tag, nxt, prv, group):
        ops = [dist.P2POp(dist.isend, send, nxt, group), dist.P2POp(dist.isend, send_tag, nxt, group),
               dist.P2POp(dist.irecv, recv, prv, group), dist.P2POp(dist.irecv, recv_tag, prv, group)]
        return dist.batch_isend_irecv(ops)

    def finish(self, works, timeout):
        for w in works:
            if timeout is None:
                w.wait()
            else:
                w.wait(timeout)


def _abort_reason(store, wait_s=0.0):
    """The reason a failed rank published, or None.  wait_s > 0 polls that long: after a transfer
    failed, the peer that caused it may still be writing its reason."""
    if store is None:
        return None
    deadline = time.monotonic() + wait_s
    while True:
        try:
            if store.check([ABORT_KEY]):
                return store.get(ABORT_KEY).decode(errors="replace")
        except Exception:  # a store that is itself gone tells us nothing more
            return None
        if time.monotonic() >= deadline:
            return None
        time.sleep(0.05)


def _publish_abort(store, rank, exc):
    if store is None:
        return
    try:
        store.set(ABORT_KEY, f"rank {rank}: {type(exc).__name__}: {exc}")
    except Exception:
        pass


def _agree(q, causal, layout, group, rank, n):
    """All ranks hold shards of one problem: same shapes, dtype, mask and layout."""
    code = {"contiguous": 0, "striped": 1, "zigzag": 2}[layout]
    mine = torch.tensor([*q.shape, int(causal), code, {torch.float32: 0, torch.bfloat16: 1}.get(q.dtype, 9)],
                        dtype=torch.int64, device=q.device)
    allv = [torch.empty_like(mine) for _ in range(n)]
    try:
        dist.all_gather(allv, mine, group=group)
    except Exception as exc:  # a rank that never joins ends the collective with the group's timeout
        raise RingError(f"rank {rank}: the ranks could not agree on the problem ({exc})") from exc
    for r, t in enumerate(allv):
        if not torch.equal(t.cpu(), mine.cpu()):
            raise RingError(f"rank {r} holds a different problem {t.tolist()} from rank {rank} {mine.tolist()}")


def ring_attention(q, k, v, causal=True, layout="striped", *, group=None, store=None, timeout=None,
                   sms_reserved=0, step_fn=None, finalize_fn=None, exchange=None, acc_dtype=torch.float32):
    """This rank's part of a Ring Attention forward pass over the ranks of `group`.

    q, k, v: this rank's shard [B, S_loc, H, D] in the layout's local token order: shard i of N
    holds global tokens g(i, 0..S_loc-1) of the layout map (contiguous, striped or zigzag; see
    include/ra.h).  Returns (out [B, S_loc, H, D] in q's dtype, lse [B, H, S_loc] fp32) for those
    tokens, equal to the rows of full attention over the whole sequence.

    timeout: seconds (or a timedelta) for each wait on a transfer where the backend honours it;
    store: a torch.distributed Store shared by the ranks, used to publish and notice failures.
    acc_dtype: dtype of the running (O, lse); the library's step takes fp32, a pluggable CPU step
    may keep fp64.
    """
    rank = dist.get_rank(group)
    n = dist.get_world_size(group)
    nxt = dist.get_global_rank(group, (rank + 1) % n) if group is not None else (rank + 1) % n
    prv = dist.get_global_rank(group, (rank - 1) % n) if group is not None else (rank - 1) % n
    if isinstance(timeout, (int, float)):
        timeout = datetime.timedelta(seconds=timeout)
    if q.dim() != 4 or q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must all be [B, S_loc, H, D]")
    B, S_loc, H, D = q.shape
    dev = q.device
    exchange = exchange or P2PExchange()
    if step_fn is None:
        import long_context_exact_forward_b200 as ra
        ws = torch.empty(ra.ring_step_workspace_size(B, H, S_loc * n, D, n, causal, layout,
                                                     1 if q.dtype == torch.bfloat16 else 0),
                         dtype=torch.uint8, device=dev)
        step_fn = _device_step(layout, causal, sms_reserved, ws)
    finalize_fn = finalize_fn or _device_finalize(q.dtype)

    _agree(q, causal, layout, group, rank, n)
    bufs = [torch.empty((2, B, S_loc, H, D), dtype=q.dtype, device=dev) for _ in range(2)]
    bufs[0][0].copy_(k)
    bufs[0][1].copy_(v)
    tags = [torch.tensor([rank], dtype=torch.int64, device=dev), torch.empty(1, dtype=torch.int64, device=dev)]
    seen = torch.full((n,), -1, dtype=torch.int64, device=dev)  # block index used at each step
    seen[0] = rank
    O_acc = torch.empty((B, S_loc, H, D), dtype=acc_dtype, device=dev)
    lse_acc = torch.empty((B, S_loc, H), dtype=acc_dtype, device=dev)
    check_now = dev.type == "cpu"

    for s in range(n):
        reason = _abort_reason(store)
        if reason is not None:
            raise RingError(f"rank {rank} stops at step {s}: {reason}")
        cur, nb = s % 2, (s + 1) % 2
        works = None
        if s + 1 < n:  # post the next block's transfer before this step's compute
            try:
                works = exchange.start(bufs[cur], tags[cur], bufs[nb], tags[nb], nxt, prv, group)
            except Exception as exc:  # e.g. a peer that failed and closed its connections
                reason = _abort_reason(store, wait_s=2.0)
                raise RingError(f"rank {rank}: the transfer for step {s + 1} could not start"
                                + (f" ({reason})" if reason else f" ({exc})")) from exc
        try:
            step_fn(q, bufs[cur][0], bufs[cur][1], O_acc, lse_acc, n, rank, s)
        except Exception as exc:
            _publish_abort(store, rank, exc)
            raise
        if works is None:
            continue
        try:
            exchange.finish(works, timeout)
        except Exception as exc:
            reason = _abort_reason(store, wait_s=2.0)
            raise RingError(f"rank {rank}: block for step {s + 1} from rank {prv} did not arrive"
                            + (f" ({reason})" if reason else f" ({exc})")) from exc
        if check_now:
            want = (rank - s - 1) % n
            if int(tags[nb].item()) != want:
                raise RingError(f"rank {rank}: step {s + 1} received block {int(tags[nb].item())}, expected {want}")
        else:
            seen[s + 1].copy_(tags[nb][0])

    if not check_now:
        expect = torch.tensor([(rank - s) % n for s in range(n)], dtype=torch.int64)
        got = seen.cpu()
        if not torch.equal(got, expect):
            raise RingError(f"rank {rank}: blocks received in order {got.tolist()}, expected {expect.tolist()}")
    return finalize_fn(O_acc, lse_acc)
