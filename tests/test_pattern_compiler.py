"""The library's host pattern compiler against the oracle's explicit G_i (CPU only).

For every (head, tile): the listed key blocks are exactly those holding at
least one pair (i, j) with j in G_i, the pair count per block matches, and
"full" means every block_q x block_k pair is in G.
"""
import numpy as np
import pytest

from block_sparse_attention_29_b200.workloads import WORKLOADS, random_table


def _expected(oracle_mod, op, H, N, tq, tk):
    T, nkb = -(-N // tq), -(-N // tk)
    exp = {}
    for h in range(H):
        for t in range(T):
            cnt = np.zeros(nkb, np.int64)
            for i in range(t * tq, min(N, t * tq + tq)):
                G = oracle_mod.build_G(op, N, h, i)
                np.add.at(cnt, G // tk, 1)
            exp[(h, t)] = cnt
    return exp


def _cases():
    tab130 = random_table(3, 700, 64, 2, seed=9)
    return [
        dict(causal=1, window=64, n_global=4, block_q=64, block_k=64, N=256, H=2),
        dict(causal=1, window=100, N=700, H=1),
        dict(causal=0, window=130, n_global=9, N=700, H=1),
        dict(causal=1, N=513, H=1),
        dict(causal=0, N=300, H=1),
        dict(causal=0, block_local=96, N=500, H=1),
        dict(causal=1, block_local=128, N=640, H=1),
        dict(causal=0, window=64, n_global=64, n_random=2, random_block=64, random_table=tab130,
             N=700, H=3),
        dict(causal=1, n_random=2, random_block=64, random_table=tab130, N=700, H=3),
        dict(causal=1, window=3, N=1, H=1),
    ]


@pytest.mark.parametrize("case", range(len(_cases())))
@pytest.mark.parametrize("tiles", [(128, 64), (64, 64)])
def test_compiler_matches_oracle(product, oracle_mod, case, tiles):
    c = dict(_cases()[case])
    N, H = c.pop("N"), c.pop("H")
    tq, tk = tiles
    pat = product.Pattern(**c)
    op = oracle_mod.Pattern(**{k: v for k, v in c.items()})
    row_ptr, kb, full, cnt, H_pat, T = product.compile_pattern(pat, H, N, tq, tk)
    assert T == -(-N // tq)
    assert H_pat == (H if c.get("n_random", 0) > 0 else 1)
    exp = _expected(oracle_mod, op, H, N, tq, tk)
    for h in range(H):
        hp = h if H_pat > 1 else 0
        for t in range(T):
            lo, hi = row_ptr[hp * T + t], row_ptr[hp * T + t + 1]
            e = exp[(h, t)]
            listed = np.nonzero(e)[0]
            assert kb[lo:hi].tolist() == listed.tolist(), (case, h, t)
            assert cnt[lo:hi].tolist() == e[listed].tolist()
            assert full[lo:hi].tolist() == (e[listed] == tq * tk).tolist()


def test_workload_block_counts(product):
    """Block counts of the workloads' patterns at 128x64 tiles (closed forms)."""
    w = WORKLOADS["mistral_swa"]
    row_ptr, kb, full, cnt, _, T = product.compile_pattern(
        product.Pattern(**w.pattern_fields()), w.H, w.N)
    # causal window 4096 over 128-row tiles: tile t lists blocks covering
    # [max(0, 128t - 4095), 128t + 127]
    per_tile = [len(range(max(0, 128 * t - 4095) // 64, (128 * t + 127) // 64 + 1)) for t in range(T)]
    assert np.diff(row_ptr).tolist() == per_tile
    assert sum(per_tile) * w.H == 101376
    w = WORKLOADS["bsfa_causal"]
    row_ptr, kb, full, cnt, _, T = product.compile_pattern(
        product.Pattern(**w.pattern_fields()), w.H, w.N)
    assert int(row_ptr[-1]) == sum(2 * t + 2 for t in range(T)) == 65792
    assert int((~full).sum()) == 2 * T     # the two diagonal blocks of each tile


@pytest.mark.parametrize("causal,W,k,N", [(1, 100, 3, 3 * 300), (0, 64, 8, 8 * 200),
                                          (1, 40, 64, 64 * 130), (0, 301, 5, 5 * 257)])
def test_dilated_lists_cover_every_residue_class(product, oracle_mod, causal, W, k, N):
    """A dilated window compiles to the lists of one residue class: for every
    class r, the oracle's G of row m*k + r, renumbered j -> (j - r) / k, gives
    exactly the listed blocks and pair counts of tile m // 128."""
    pat = product.Pattern(causal=causal, window=W, dilation=k)
    row_ptr, kb, full, cnt, H_pat, T = product.compile_pattern(pat, 1, N)
    n = N // k
    assert H_pat == 1 and T == -(-n // 128)
    op = oracle_mod.Pattern(causal=causal, window=W, dilation=k)
    for r in sorted({0, k - 1, k // 2}):
        for t in range(T):
            exp = np.zeros(-(-n // 64), np.int64)
            for m in range(t * 128, min(n, t * 128 + 128)):
                G = oracle_mod.build_G(op, N, 0, m * k + r)
                assert np.all((G - r) % k == 0)
                np.add.at(exp, ((G - r) // k) // 64, 1)
            lo, hi = row_ptr[t], row_ptr[t + 1]
            assert np.array_equal(kb[lo:hi], np.nonzero(exp)[0]), (r, t)
            assert np.array_equal(cnt[lo:hi], exp[kb[lo:hi]]), (r, t)


@pytest.mark.parametrize("bad", [dict(causal=1, window=8, dilation=3, n_global=2),
                                 dict(causal=0, window=8, dilation=2, block_local=64),
                                 dict(causal=1, window=0, dilation=2),
                                 dict(causal=1, window=8, dilation=7),   # 7 does not divide N
                                 dict(causal=1, window=8, dilation=-1)])
def test_dilated_window_rejections(product, bad):
    with pytest.raises(product.SparseAttnError):
        product.compile_pattern(product.Pattern(**bad), 1, 600)
