"""The host-side planner (layout maps, causal block-skip tile classes, LPT work list) checked on
the CPU against brute force over the oracle's independent layout positions."""
import numpy as np
import pytest

import long_context_exact_forward_b200 as ra
import oracle

LAYOUT_CASES = [(48, 4, "contiguous"), (48, 4, "striped"), (48, 4, "zigzag"), (40, 5, "contiguous"),
                (40, 5, "striped"), (60, 3, "zigzag"), (7, 1, "contiguous"), (1024, 8, "zigzag")]


@pytest.mark.parametrize("S, N, layout", LAYOUT_CASES)
def test_layout_positions_match_oracle(S, N, layout):
    np.testing.assert_array_equal(ra.layout_positions(S, N, layout), oracle.layout_positions(S, N, layout))


@pytest.mark.parametrize("S, N, layout", LAYOUT_CASES)
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("tile", [1, 3, 4, 8, 64])
def test_tile_classes_are_exact(S, N, layout, causal, tile):
    if S > 100 and tile < 8:
        pytest.skip("large case runs with wide tiles only")
    pos = oracle.layout_positions(S, N, layout)
    S_loc = S // N
    nt = -(-S_loc // tile)
    cls = ra.plan_tiles(S, N, layout, causal, tile)
    assert cls.shape == (N, N, nt, nt)
    covered = np.zeros((S, S), dtype=np.int64)
    for i in range(N):
        for s in range(N):
            j = (i - s) % N
            for qt in range(nt):
                qa = np.arange(qt * tile, min((qt + 1) * tile, S_loc))
                for kt in range(nt):
                    ka = np.arange(kt * tile, (kt + 1) * tile)
                    inside = ka < S_loc
                    gq = pos[i, qa][:, None]
                    gk = np.where(inside, pos[j, np.minimum(ka, S_loc - 1)], S + 1)[None, :]
                    allowed = (gk <= gq) if causal else np.broadcast_to(inside[None, :], (qa.size, ka.size))
                    allowed = allowed & inside[None, :]
                    c = cls[i, s, qt, kt]
                    if c == 0:
                        assert not allowed.any(), "EMPTY tile holds an allowed pair"
                    elif c == 1:
                        assert allowed.all(), "FULL tile holds a masked pair"
                    else:
                        assert c == 2 and allowed.any() and not allowed.all()
                    gqs = np.broadcast_to(gq, allowed.shape)[allowed]
                    gks = np.broadcast_to(gk, allowed.shape)[allowed]
                    np.add.at(covered, (gqs, gks), 1)
    want = np.tril(np.ones((S, S), dtype=np.int64)) if causal else np.ones((S, S), dtype=np.int64)
    np.testing.assert_array_equal(covered, want)  # every allowed pair exactly once


@pytest.mark.parametrize("layout", ["contiguous", "striped", "zigzag"])
@pytest.mark.parametrize("causal", [False, True])
def test_work_list_covers_every_item_once_heaviest_first(layout, causal):
    B, H, N, S_loc = 2, 3, 4, 640  # 640 = 2.5 pairs of 256 rows: a ragged last pair
    S = N * S_loc
    items = ra.plan_items(B, H, S, N, causal, layout)
    pairs = -(-S_loc // 256)
    assert items.shape == (B * H * N * pairs, 5)
    keys = {tuple(r[:4]) for r in items.tolist()}
    assert keys == {(b, h, i, p) for b in range(B) for h in range(H) for i in range(N) for p in range(pairs)}
    # (b, h) major, heaviest first inside a head
    bh = items[:, 0] * H + items[:, 1]
    assert (np.diff(bh) >= 0).all()
    for g in range(B * H):
        cost = items[bh == g, 4]
        assert (np.diff(cost) <= 0).all()
    # cost = live (128-row query tile, 128-key tile) pairs, from the oracle's positions
    pos = oracle.layout_positions(S, N, layout)
    for b, h, i, p, cost in items[:N * pairs].tolist():
        want = 0
        for q in range(2):
            a0 = p * 256 + q * 128
            if a0 >= S_loc:
                continue
            last = min(a0 + 127, S_loc - 1)
            for s in range(N):
                j = (i - s) % N
                n_vis = int((pos[j] <= pos[i, last]).sum()) if causal else S_loc
                want += -(-n_vis // 128)
        assert cost == want


def test_causal_work_totals_match_closed_form():
    # striped spreads the causal triangle evenly: every shard's items cost about the same
    S, N = 8192, 16
    for layout, spread_max in (("striped", 1.10), ("zigzag", 1.25)):
        items = ra.plan_items(1, 1, S, N, True, layout)
        per_shard = np.zeros(N)
        for _, _, i, _, cost in items.tolist():
            per_shard[i] += cost
        assert per_shard.max() / per_shard.min() < spread_max
    items = ra.plan_items(1, 1, S, N, True, "contiguous")
    per_shard = np.zeros(N)
    for _, _, i, _, cost in items.tolist():
        per_shard[i] += cost
    assert per_shard[-1] / per_shard[0] > 10  # the last shard sees every earlier block


def test_work_list_groups_shards_when_a_head_exceeds_l2():
    # one head's K/V = 4 * S * D bytes = 128 MiB > 96 MiB: items of a shard are kept together
    B, H, S, D, N = 1, 2, 262144, 128, 16
    items = ra.plan_items(B, H, S, N, True, "striped", D=D)
    pairs = (S // N + 255) // 256
    assert items.shape == (B * H * N * pairs, 5)
    per_head = N * pairs
    for h in range(H):
        blk = items[h * per_head:(h + 1) * per_head]
        assert (blk[:, 1] == h).all()
        shards = blk[:, 2]
        runs = [shards[0]] + [b for a, b in zip(shards[:-1], shards[1:]) if a != b]
        assert sorted(runs) == list(range(N))  # each shard appears as one contiguous run
        group_cost = [int(blk[shards == i, 4].sum()) for i in runs]
        assert group_cost == sorted(group_cost, reverse=True)
        for i in range(N):
            c = blk[shards == i, 4]
            assert (np.diff(c) <= 0).all()
    # below the threshold the plain heaviest-first order is kept
    small = ra.plan_items(1, 1, 65536, 16, True, "striped", D=128)
    assert (np.diff(small[:, 4]) <= 0).all()


def test_random_shapes_layouts_and_tiles_against_brute_force():
    # seeded random shapes beyond the fixed list: every (query, key) pair of the tile classes agrees
    # with the mask computed from the oracle's positions, and the work list covers each item once
    rng = np.random.default_rng(2024)
    for _ in range(25):
        N = int(rng.integers(1, 7))
        layout = ["contiguous", "striped", "zigzag"][int(rng.integers(3))]
        unit = 2 * N if layout == "zigzag" else N
        S = unit * int(rng.integers(1, 12))
        tile = int(rng.integers(1, 9))
        causal = bool(rng.integers(2))
        pos = oracle.layout_positions(S, N, layout)
        np.testing.assert_array_equal(ra.layout_positions(S, N, layout), pos)
        S_loc = S // N
        nt = -(-S_loc // tile)
        cls = ra.plan_tiles(S, N, layout, causal, tile)
        for i in range(N):
            for s in range(N):
                j = (i - s) % N
                for qt in range(nt):
                    qa = np.arange(qt * tile, min((qt + 1) * tile, S_loc))
                    for kt in range(nt):
                        ka = np.arange(kt * tile, min((kt + 1) * tile, S_loc))
                        gq, gk = pos[i, qa][:, None], pos[j, ka][None, :]
                        allowed = (gk <= gq) if causal else np.ones((qa.size, ka.size), dtype=bool)
                        c = cls[i, s, qt, kt]
                        if c == 0:
                            assert not allowed.any(), (S, N, layout, causal, tile, i, s, qt, kt)
                        elif c == 1:
                            assert allowed.all() and ka.size == tile, (S, N, layout, causal, tile, i, s, qt, kt)
                        else:
                            assert allowed.any(), (S, N, layout, causal, tile, i, s, qt, kt)


def test_plan_cache_keeps_lists_right_past_its_bound():
    """The planner's caches hold a bounded number of shapes (least recently used dropped): a sweep
    over more shapes than that leaves every list, recomputed or cached, as it was."""
    first = ra.plan_items(1, 2, 4096, 4, True, "striped").copy()
    for n in range(1, 90):  # more distinct shapes than the cache keeps
        ra.plan_items(1, 1, 256 * n, 2, True, "contiguous")
    again = ra.plan_items(1, 2, 4096, 4, True, "striped")
    assert np.array_equal(first, again)
