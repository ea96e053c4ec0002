"""Host work order of the prefill queue (sparse_attn_work_order): split tiles.

A tile whose block list is cut into pieces must be covered exactly once by
its pieces (consecutive, in list order, near-equal), every tile must appear
exactly once (whole or split), and the workspace slots of the pieces must be
a permutation laid out per split tile.  No GPU is used.
"""
import numpy as np
import pytest

from block_sparse_attention_29_b200.workloads import random_table


def _lists(product, pat, H, N):
    row_ptr, kb, full, cnt, H_pat, T = product.compile_pattern(pat, H, N)
    return row_ptr, H_pat, T


def _check_cover(product, pat, B, H, Hkv, N, d, mub):
    units, pieces, split = product.work_order(pat, B, H, Hkv, N, d, mub)
    row_ptr, H_pat, T = _lists(product, pat, H, N)
    n_tiles = B * max(pat.dilation, 1) * H * T   # a dilated plan runs B*k residue classes
    length = lambda u: int(row_ptr[((u // T) % H if H_pat > 1 else 0) * T + u % T + 1]
                           - row_ptr[((u // T) % H if H_pat > 1 else 0) * T + u % T])
    whole = units[units >= 0]
    piece_idx = ~units[units < 0]
    # every piece appears once in the queue
    assert np.array_equal(np.sort(piece_idx), np.arange(len(pieces)))
    # every tile once: whole, or split
    split_ids = split[:, 0] if len(split) else np.zeros(0, np.int32)
    assert np.array_equal(np.sort(np.concatenate([whole, split_ids])), np.arange(n_tiles))
    # pieces of a split tile partition its list, slots per tile are consecutive
    slots = []
    for s in split:
        tid, first, npc = int(s[0]), int(s[1]), int(s[2])
        mine = pieces[pieces[:, 0] == tid]
        assert len(mine) == npc
        mine = mine[np.argsort(mine[:, 1])]
        assert mine[0, 1] == 0
        assert np.array_equal(mine[1:, 1], mine[:-1, 1] + mine[:-1, 2])
        assert mine[-1, 1] + mine[-1, 2] == length(tid)
        assert np.array_equal(np.sort(mine[:, 3]), np.arange(first, first + npc))
        assert mine[:, 2].max() - mine[:, 2].min() <= 1      # near-equal pieces
        if mub > 0:
            assert mine[:, 2].max() <= mub
        # queue order: a split tile's pieces in descending list position
        pos = {int(p): k for k, p in enumerate(~units[units < 0])}
        order = [pos[int(np.flatnonzero((pieces[:, 0] == tid) & (pieces[:, 1] == k0))[0])]
                 for k0 in mine[:, 1]]
        assert order == sorted(order, reverse=True)
        slots.extend(mine[:, 3].tolist())
    assert sorted(slots) == list(range(len(slots)))
    if mub > 0:
        for u in whole:
            assert length(int(u)) <= mub
    return units, pieces, split


@pytest.mark.parametrize("mub", [-1, 1, 3, 8, 1000])
@pytest.mark.parametrize("case", [
    dict(B=1, H=2, Hkv=2, N=1000, d=128, causal=1),
    dict(B=2, H=4, Hkv=2, N=700, d=128, causal=0, window=150, n_global=7),
    dict(B=1, H=2, Hkv=1, N=777, d=64, causal=0, window=130, n_global=9),
    dict(B=1, H=3, Hkv=3, N=640, d=128, causal=0, block_local=128),
    dict(B=1, H=8, Hkv=2, N=1, d=128, causal=1),
])
def test_split_covers_every_list_once(product, case, mub):
    c = dict(case)
    B, H, Hkv, N, d = (c.pop(k) for k in ("B", "H", "Hkv", "N", "d"))
    units, pieces, split = _check_cover(product, product.Pattern(**c), B, H, Hkv, N, d, mub)
    if mub < 0:
        assert len(pieces) == 0 and len(split) == 0
    if mub == 1 and N > 128:
        assert len(split) > 0


def test_split_with_random_blocks_and_dilation(product):
    H, N = 3, 700
    tab = random_table(H, N, 64, 3, seed=77)
    pat = product.Pattern(causal=0, window=64, n_global=16, n_random=3, random_block=64,
                          random_table=tab)
    _check_cover(product, pat, 1, H, H, N, 64, 4)
    _check_cover(product, product.Pattern(causal=1, window=64, dilation=4), 2, 2, 1, 1024, 128, 2)


def test_automatic_split_takes_only_the_global_tiles(product):
    """Window + global tokens + random blocks (the BigBird/Longformer mix): the
    automatic rule cuts the tile holding the global rows of every (b, h) -- its
    list covers every key block -- and nothing else."""
    B, H, N, d = 1, 16, 32768, 64   # K + V above half of L2: K/V-group-major order
    tab = random_table(H, N, 64, 3, seed=5)
    pat = product.Pattern(causal=0, window=512, n_global=64, n_random=3, random_block=64,
                          random_table=tab)
    units, pieces, split = _check_cover(product, pat, B, H, H, N, d, 0)
    T = N // 128
    assert sorted(split[:, 0].tolist()) == [bh * T for bh in range(B * H)]
    assert pieces[:, 2].max() <= 64
    # K/V-group-major order (one query head per K/V head here): the tiles of
    # head bh run together, and the pieces of head bh's split tile are queued
    # with the tiles of head bh - 1, before head bh's own tiles
    pos = np.arange(len(units))
    whole_bh = np.where(units >= 0, units // T, -1)
    piece_bh = np.where(units < 0, pieces[~np.minimum(units, -1), 0] // T, -1)
    for bh in range(B * H):
        w = pos[whole_bh == bh]
        pc = pos[piece_bh == bh]
        assert w.max() - w.min() + 1 == len(w)
        assert pc.max() - pc.min() + 1 == len(pc)
        assert pc.max() < w.min()
        if bh >= 1:
            assert pc.max() + 1 == pos[whole_bh == bh - 1].min()
        if bh >= 2:
            assert pc.min() > pos[whole_bh == bh - 2].max()


def test_automatic_split_leaves_even_workloads_alone(product):
    for pat, N in ((product.Pattern(causal=1, window=4096), 8192),
                   (product.Pattern(causal=1), 32768)):
        units, pieces, split = product.work_order(pat, 1, 32, 8, N, 128, 0)
        assert len(split) == 0 and len(units) == 32 * (N // 128)


def _lens(product, pat, H, N, units, T):
    row_ptr, kb, full, cnt, H_pat, _ = product.compile_pattern(pat, H, N)
    out = []
    for u in units:
        h, t = (u // T) % H, u % T
        r = (h if H_pat > 1 else 0) * T + t
        out.append(int(row_ptr[r + 1] - row_ptr[r]))
    return np.array(out)


def test_order_long_units_first_then_tile_major(product):
    """K and V within half of L2 (tile-major): units longer than half a CTA's
    share of the work come first, longest first; the rest by descending tile,
    the query heads of a tile in order."""
    B, H, Hkv, N, d = 1, 4, 2, 8192, 128   # K + V = 8 MiB
    pat = product.Pattern(causal=1)
    units, pieces, split = product.work_order(pat, B, H, Hkv, N, d, -1)
    T = N // 128
    lens = _lens(product, pat, H, N, units, T)
    heavy = max(1, lens.sum() // (2 * 296) // 2)
    n_heavy = int((lens > heavy).sum())
    assert np.all(lens[:n_heavy] > heavy) and np.all(np.diff(lens[:n_heavy]) <= 0)
    rest = units[n_heavy:]
    t = rest % T
    assert np.all(np.diff(t) <= 0)                         # descending tile
    for tt in np.unique(t):
        hs = (rest[t == tt] // T) % H
        assert np.array_equal(hs, np.sort(hs))             # heads of a tile in order


def test_order_kv_group_major_when_kv_exceeds_half_of_l2(product):
    """K and V above half of L2: the tiles of one K/V group (its query heads)
    run together, longest first inside the group."""
    B, H, Hkv, N, d = 1, 8, 4, 65536, 128  # K + V = 128 MiB
    pat = product.Pattern(causal=1, window=1024)
    units, pieces, split = product.work_order(pat, B, H, Hkv, N, d, -1)
    T = N // 128
    group = (units // T) % H // (H // Hkv)
    assert np.all(np.diff(group) >= 0)
    lens = _lens(product, pat, H, N, units, T)
    for g in np.unique(group):
        assert np.all(np.diff(lens[group == g]) <= 0)
