"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test ties one part of the oracle to something other than itself: values
printed on the pages (tests/golden), closed forms, library routines (torch
float64) and brute-force enumeration written independently in Python.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rand(shape, seed):
    g = np.random.default_rng(seed)
    return g.standard_normal(shape)


# --------------------------------------------------------------- worked example
def test_worked_example_weighted_sum(oracle_mod):
    """1cademy worked question: G={0,2}, alpha=0.6/0.4, v0=[1,0], v2=[0,3] -> [0.6, 1.2]."""
    g = _golden("worked_example_1cademy.json")
    V = np.array(g["V"])
    out = oracle_mod.weighted_sum(g["G"], g["alpha"], V)
    assert np.allclose(out, g["expected_out"], rtol=0, atol=1e-15)
    # v_1 is not in G: changing it must not change the output.
    V2 = V.copy()
    V2[1] = [1e6, -1e6]
    assert np.array_equal(oracle_mod.weighted_sum(g["G"], g["alpha"], V2), out)


def test_worked_example_from_logits(oracle_mod):
    """Same example reached through the softmax: logits ln(1.5) and 0 give 0.6/0.4."""
    g = _golden("worked_example_1cademy.json")
    d = 2
    q = np.array([[[math.sqrt(2.0) * math.log(1.5), 0.0]]])          # [S=1][H=1][d]
    K = np.zeros((1, 1, 4, d))
    K[0, 0, 0] = [1.0, 0.0]                                           # s_0 = ln 1.5
    K[0, 0, 1] = [5.0, 5.0]                                           # not in G
    K[0, 0, 2] = [0.0, 0.0]                                           # s_2 = 0
    V = np.zeros((1, 1, 4, d))
    V[0, 0, :3] = g["V"]
    V[0, 0, 3] = [7.0, 7.0]
    idx = np.array([[g["G"]]], dtype=np.int32)
    out, lse = oracle_mod.gather(q, K, V, idx)
    assert np.allclose(out[0, 0], g["expected_out"], rtol=0, atol=1e-14)
    assert abs(lse[0, 0] - math.log(2.5)) < 1e-14


# ---------------------------------------------------------- dense equivalence
def _torch_dense(Q, K, V, causal, scale):
    q, k, v = (torch.from_numpy(x) for x in (Q, K, V))
    g = q.shape[1] // k.shape[1]
    k = k.repeat_interleave(g, dim=1)
    v = v.repeat_interleave(g, dim=1)
    s = (q @ k.transpose(-1, -2)) * scale
    if causal:
        n = s.shape[-1]
        s = s.masked_fill(torch.ones(n, n, dtype=torch.bool).triu(1), float("-inf"))
    return (torch.softmax(s, dim=-1) @ v).numpy()


@pytest.mark.parametrize("causal", [0, 1])
def test_full_G_is_dense_attention(oracle_mod, causal):
    """A full G (no primitive) reproduces softmax(QK^T/sqrt(d))V (glossary formula)."""
    B, H, Hkv, N, d = 2, 4, 2, 37, 8
    Q, K, V = _rand((B, H, N, d), 1), _rand((B, Hkv, N, d), 2), _rand((B, Hkv, N, d), 3)
    p = oracle_mod.Pattern(causal=causal)
    O, lse = oracle_mod.prefill(p, Q, K, V)
    Od = oracle_mod.dense(Q, K, V, causal=bool(causal))
    Ot = _torch_dense(Q, K, V, causal, 1 / math.sqrt(d))
    assert np.max(np.abs(O - Od)) < 1e-12
    assert np.max(np.abs(O - Ot)) < 1e-12


def test_gqa_equals_mha_on_repeated_kv(oracle_mod):
    """GQA with contiguous head groups == MHA on repeat_interleave'd K/V."""
    B, H, Hkv, N, d = 1, 6, 2, 40, 8
    Q, K, V = _rand((B, H, N, d), 4), _rand((B, Hkv, N, d), 5), _rand((B, Hkv, N, d), 6)
    p = oracle_mod.Pattern(causal=1, window=7, n_global=2, block_q=64, block_k=64)
    O1, _ = oracle_mod.prefill(p, Q, K, V)
    Kr, Vr = np.repeat(K, H // Hkv, axis=1), np.repeat(V, H // Hkv, axis=1)
    O2, _ = oracle_mod.prefill(p, Q, Kr, Vr)
    assert np.array_equal(O1, O2)


# ---------------------------------------------------------------- G enumeration
def _patterns(oracle_mod, N, H):
    tab = np.stack([np.sort(np.random.default_rng(7 + h).choice(-(-N // 64), size=(-(-N // 64), 2),
                                                                  replace=True), axis=-1)
                    for h in range(H)]).astype(np.int32)
    # make entries distinct per row
    for h in range(H):
        for r in range(tab.shape[1]):
            if tab[h, r, 0] == tab[h, r, 1]:
                tab[h, r, 1] = (tab[h, r, 0] + 1) % tab.shape[1]
    P = oracle_mod.Pattern
    return [
        P(),
        P(causal=1),
        P(causal=1, window=5),
        P(causal=0, window=6),
        P(causal=0, window=7),
        P(causal=1, window=9, n_global=3),
        P(causal=0, window=4, n_global=2),
        P(causal=0, block_local=16),
        P(causal=1, block_local=32, window=3),
        P(causal=0, n_random=2, random_block=64, random_table=tab),
        P(causal=1, n_global=1, n_random=2, random_block=64, random_table=tab),
        P(causal=0, window=10, n_global=5, n_random=2, random_block=64, random_table=tab),
        # dilated/strided windows (taps k apart), alone and in unions
        P(causal=1, window=4, dilation=3),
        P(causal=0, window=6, dilation=5),
        P(causal=0, window=7, dilation=2),
        P(causal=1, window=3, dilation=70),
        P(causal=0, window=5, dilation=4, n_global=2),
        P(causal=1, window=6, dilation=3, block_local=16),
    ]


@pytest.mark.parametrize("N", [1, 50, 130])
def test_G_ranges_equal_bruteforce(oracle_mod, N):
    """Range construction == C predicate == an independent Python predicate."""
    H = 2
    for p in _patterns(oracle_mod, N, H):
        for h in range(H):
            for i in range(N):
                G = oracle_mod.build_G(p, N, h, i).tolist()
                brute = [j for j in range(N) if oracle_mod.visible_py(p, N, h, i, j)]
                assert G == brute, (p, h, i)
                cpred = [j for j in range(N) if oracle_mod.visible(p, N, h, i, j)]
                assert G == cpred


def test_window_closed_form(oracle_mod):
    """Mistral rule: |G_i| = min(i + 1, W) for the causal window [max(0, i-W+1), i]."""
    N, W = 300, 64
    p = oracle_mod.Pattern(causal=1, window=W)
    for i in range(N):
        assert len(oracle_mod.build_G(p, N, 0, i)) == min(i + 1, W)


@pytest.mark.parametrize("k", [1, 2, 3, 7, 64])
def test_dilated_window_closed_form(oracle_mod, k):
    """Dilated window (W taps k apart): causal |G_i| = min(floor(i/k) + 1, W);
    non-causal |G_i| = min(floor(i/k), W/2) + 1 + min(floor((N-1-i)/k), W/2);
    every member j has (i - j) mod k == 0."""
    N = 400
    for W in (1, 5, 16):
        pc = oracle_mod.Pattern(causal=1, window=W, dilation=k)
        pn = oracle_mod.Pattern(causal=0, window=W, dilation=k)
        for i in range(0, N, 7):
            G = oracle_mod.build_G(pc, N, 0, i)
            assert len(G) == min(i // k + 1, W)
            assert np.all((i - G) % k == 0) and G.max() == i
            Gn = oracle_mod.build_G(pn, N, 0, i)
            assert len(Gn) == min(i // k, W // 2) + 1 + min((N - 1 - i) // k, W // 2)
            assert np.all((i - Gn) % k == 0)


def test_dilation_zero_and_one_are_the_contiguous_window(oracle_mod):
    N = 200
    for causal, W in ((1, 17), (0, 12)):
        base = oracle_mod.Pattern(causal=causal, window=W)
        for dil in (0, 1):
            p = oracle_mod.Pattern(causal=causal, window=W, dilation=dil)
            for i in range(N):
                assert np.array_equal(oracle_mod.build_G(p, N, 0, i),
                                      oracle_mod.build_G(base, N, 0, i))


@pytest.mark.parametrize("causal", [1, 0])
def test_dilated_window_is_window_on_residue_classes(oracle_mod, causal):
    """A dilated window joins only positions of one residue class i mod k, and
    inside a class (numbered m = i // k) it is the contiguous window: the
    dilated attention's rows of class r equal the contiguous-window attention
    over the subsequence r, r + k, r + 2k, ..."""
    B, H, Hkv, N, d, k, W = 1, 2, 1, 3 * 41, 8, 3, 6
    Q, K, V = _rand((B, H, N, d), 61), _rand((B, Hkv, N, d), 62), _rand((B, Hkv, N, d), 63)
    O, lse = oracle_mod.prefill(oracle_mod.Pattern(causal=causal, window=W, dilation=k), Q, K, V)
    for r in range(k):
        sl = slice(r, None, k)
        Or, lr = oracle_mod.prefill(oracle_mod.Pattern(causal=causal, window=W),
                                    np.ascontiguousarray(Q[:, :, sl]),
                                    np.ascontiguousarray(K[:, :, sl]),
                                    np.ascontiguousarray(V[:, :, sl]), scale=1 / np.sqrt(d))
        assert np.max(np.abs(O[:, :, sl] - Or)) < 1e-13
        assert np.max(np.abs(lse[:, :, sl] - lr)) < 1e-12


def test_tiny_static_pair_count(oracle_mod):
    """causal and (window 64 or globals 0..3), N=256: 15,130 pairs per head (closed form)."""
    N, W, g = 256, 64, 4
    p = oracle_mod.Pattern(causal=1, window=W, n_global=g, block_q=64, block_k=64)
    total = sum(len(oracle_mod.build_G(p, N, 0, i)) for i in range(N))
    closed = sum(i + 1 for i in range(W)) + sum(W + sum(1 for j in range(g) if j < i - W + 1)
                                                 for i in range(W, N))
    assert total == closed == 15130


def test_page_counts(oracle_mod):
    c = _golden("counts.json")
    # dense 5x5: no primitive, non-causal -> all 25 pairs
    p = oracle_mod.Pattern()
    assert sum(len(oracle_mod.build_G(p, 5, 0, i)) for i in range(5)) == c["dense_5x5"]["pairs"]
    # explicit sparse grid: 10 pairs, a 60% reduction; rows through the explicit-set entry
    sp = c["sparse_5x5"]
    assert sum(len(s) for s in sp["G"]) == sp["pairs"]
    assert 1 - sp["pairs"] / c["dense_5x5"]["pairs"] == pytest.approx(sp["reduction"])
    # first token + itself + two preceding: causal window 3 or global 1
    fp = c["first_plus_local"]
    p = oracle_mod.Pattern(causal=1, window=3, n_global=1)
    G = oracle_mod.build_G(p, fp["N"], 0, fp["i"])
    assert len(G) == fp["pairs"] and G.tolist() == [0, fp["i"] - 2, fp["i"] - 1, fp["i"]]


def test_explicit_sets_row_softmax(oracle_mod):
    """Explicit sets (the 5x5 grid) -- each row is the softmax over exactly its set."""
    c = _golden("counts.json")["sparse_5x5"]
    d = 3
    Q = _rand((5, d), 11)
    K = _rand((5, d), 12)
    V = _rand((5, d), 13)
    for i, G in enumerate(c["G"]):
        idx = np.array([[G]], dtype=np.int32)
        out, _ = oracle_mod.gather(Q[i][None, None], K[None, None], V[None, None], idx)
        s = np.array([Q[i] @ K[j] / math.sqrt(d) for j in G])
        a = np.exp(s - s.max()) / np.exp(s - s.max()).sum()
        assert np.allclose(out[0, 0], sum(a[k] * V[j] for k, j in enumerate(G)), atol=1e-14)


def test_exclusion(oracle_mod):
    """1cademy: j outside G_i contributes nothing -- perturbing those K/V rows leaves out_i."""
    B, H, Hkv, N, d = 1, 2, 2, 96, 8
    Q, K, V = _rand((B, H, N, d), 21), _rand((B, Hkv, N, d), 22), _rand((B, Hkv, N, d), 23)
    p = oracle_mod.Pattern(causal=1, window=8, n_global=2, block_q=64, block_k=64)
    i = 70
    rows = np.array([[0, h, i] for h in range(H)], np.int32)
    O1, _ = oracle_mod.prefill(p, Q, K, V, rows=rows)
    G = set(oracle_mod.build_G(p, N, 0, i).tolist())
    K2, V2 = K.copy(), V.copy()
    for j in range(N):
        if j not in G:
            K2[:, :, j] += 100.0
            V2[:, :, j] -= 100.0
    O2, _ = oracle_mod.prefill(p, Q, K2, V2, rows=rows)
    assert np.array_equal(O1, O2)


# ------------------------------------------------------------- block-skip rule
def _bsfa_small(oracle_mod, seed=31):
    B, H, Hkv, N, d = 1, 2, 1, 512, 16
    Q, K, V = _rand((B, H, N, d), seed), _rand((B, Hkv, N, d), seed + 1), _rand((B, Hkv, N, d), seed + 2)
    return B, H, Hkv, N, d, Q, K, V


def test_tile_statistic_bruteforce(oracle_mod):
    """Block statistic, pair count and fullness of a tile against numpy brute force."""
    B, H, Hkv, N, d, Q, K, V = _bsfa_small(oracle_mod)
    p = oracle_mod.Pattern(causal=1, window=150, block_q=128, block_k=64)
    scale = 1 / math.sqrt(d)
    for t in range(N // 128):
        cnt, full, stat, mask = oracle_mod.tile_blocks(p, Q, K, 0, 1, t)
        for kb in range(N // 64):
            vals = [scale * Q[0, 1, i] @ K[0, 0, j]
                    for i in range(t * 128, t * 128 + 128) for j in range(kb * 64, kb * 64 + 64)
                    if oracle_mod.visible_py(p, N, 1, i, j)]
            assert cnt[kb] == len(vals)
            assert full[kb] == (len(vals) == 128 * 64)
            if vals:
                assert stat[kb] == pytest.approx(max(vals), abs=1e-12)
                assert mask[kb] == 1
            else:
                assert mask[kb] == 0


def test_bsfa_threshold_minus_inf_is_dense(oracle_mod):
    """tau = -inf skips nothing: identical to exact causal attention."""
    B, H, Hkv, N, d, Q, K, V = _bsfa_small(oracle_mod)
    p = oracle_mod.Pattern(causal=1, block_q=128, block_k=64)
    O0, l0 = oracle_mod.prefill(p, Q, K, V)
    O1, l1, mask, stat, full = oracle_mod.prefill(p, Q, K, V, thresholds=np.full(H, -np.inf),
                                                  want_blocks=True)
    assert np.array_equal(O0, O1) and np.array_equal(l0, l1)
    assert not (mask == 2).any()
    assert np.max(np.abs(O0 - _torch_dense(Q, K, V, 1, 1 / math.sqrt(d)))) < 1e-12


def test_bsfa_threshold_plus_inf_keeps_partial_blocks_only(oracle_mod):
    """tau = +inf skips every full block; what is left is the diagonal 128x128 block."""
    B, H, Hkv, N, d, Q, K, V = _bsfa_small(oracle_mod)
    p = oracle_mod.Pattern(causal=1, block_q=128, block_k=64)
    O1, _, mask, _, full = oracle_mod.prefill(p, Q, K, V, thresholds=np.full(H, np.inf),
                                              want_blocks=True)
    assert ((mask == 2) == full).all()
    diag = oracle_mod.Pattern(causal=1, block_local=128, block_q=128, block_k=64)
    O2, _ = oracle_mod.prefill(diag, Q, K, V)
    assert np.max(np.abs(O1 - O2)) < 1e-12


def test_bsfa_calibrated_skip_fraction(oracle_mod):
    """Lower-median threshold on the same draw skips floor((n-1)/2) of n full blocks per head."""
    B, H, Hkv, N, d, Q, K, V = _bsfa_small(oracle_mod)
    p = oracle_mod.Pattern(causal=1, block_q=128, block_k=64)
    full, stat, _ = oracle_mod.block_stats(p, Q, K)
    tau = oracle_mod.calibrate_thresholds(full, stat)
    _, _, mask, _, _ = oracle_mod.prefill(p, Q, K, V, thresholds=tau, want_blocks=True)
    for h in range(H):
        n = int(full[:, h].sum())
        assert n == sum(2 * t for t in range(N // 128))   # blocks left of each diagonal
        assert int((mask[:, h] == 2).sum()) == (n - 1) // 2


def test_bsfa_skipped_keys_leave_G(oracle_mod):
    """A skipped block's keys leave G_i of every row of the tile (the rows then equal an
    explicit-set computation without them)."""
    B, H, Hkv, N, d, Q, K, V = _bsfa_small(oracle_mod, seed=41)
    p = oracle_mod.Pattern(causal=1, block_q=128, block_k=64)
    full, stat, _ = oracle_mod.block_stats(p, Q, K)
    tau = oracle_mod.calibrate_thresholds(full, stat)
    O, _, mask, _, _ = oracle_mod.prefill(p, Q, K, V, thresholds=tau, want_blocks=True)
    for h in range(H):
        for i in (200, 383, 500):
            t = i // 128
            G = [j for j in range(i + 1) if mask[0, h, t, j // 64] != 2]
            idx = np.array([[G]], dtype=np.int32)
            og, _ = oracle_mod.gather(Q[0, h][i][None, None], K[0][None, :, : i + 1],
                                      V[0][None, :, : i + 1], idx)
            assert np.max(np.abs(og[0, 0] - O[0, h, i])) < 1e-13


def test_gather_equals_prefill_row(oracle_mod):
    """With idx = static G_i of the last row, the explicit-set entry equals that prefill row."""
    B, H, Hkv, N, d = 1, 4, 2, 200, 8
    Q, K, V = _rand((B, H, N, d), 51), _rand((B, Hkv, N, d), 52), _rand((B, Hkv, N, d), 53)
    p = oracle_mod.Pattern(causal=1, window=20, n_global=3)
    i = N - 1
    O, _ = oracle_mod.prefill(p, Q, K, V)
    G = oracle_mod.build_G(p, N, 0, i)
    idx = np.broadcast_to(G, (1, H, len(G))).astype(np.int32).copy()
    og, _ = oracle_mod.gather(Q[:, :, i], K, V, idx)
    assert np.max(np.abs(og[0] - O[0, :, i])) < 1e-14


def test_bf16_inputs_convert_exactly(oracle_mod):
    """bf16 inputs are converted exactly: the same values as float64 give identical output."""
    B, H, N, d = 1, 1, 64, 8
    g = torch.Generator().manual_seed(3)
    Qb = torch.randn(B, H, N, d, generator=g).bfloat16()
    Kb = torch.randn(B, H, N, d, generator=g).bfloat16()
    Vb = torch.randn(B, H, N, d, generator=g).bfloat16()
    p = oracle_mod.Pattern(causal=1, window=9)
    O1, _ = oracle_mod.prefill(p, Qb, Kb, Vb)
    O2, _ = oracle_mod.prefill(p, Qb.double().numpy(), Kb.double().numpy(), Vb.double().numpy())
    assert np.array_equal(O1, O2)


# ---------------------------------------------------------------- dynamic top-K
def _decode_inputs(S, H, Hkv, L, d, seed):
    return (_rand((S, H, d), seed), _rand((S, Hkv, L, d), seed + 1), _rand((S, Hkv, L, d), seed + 2))


def test_topk_covering_every_key_is_dense_decode(oracle_mod):
    """top_k >= len: G is every key j < len, so the output is the dense softmax
    row (torch float64) of the query over those keys."""
    import torch
    S, H, Hkv, L, d = 2, 4, 2, 60, 16
    Q, K, V = _decode_inputs(S, H, Hkv, L, d, 81)
    lengths = np.array([60, 23])
    idx, n, kth, nxt = oracle_mod.topk_select(Q, K, 64, lengths=lengths)
    assert n.tolist() == [[60] * H, [23] * H] and np.all(np.isnan(nxt))
    O, lse = oracle_mod.gather(Q, K, V, idx, n)
    for s in range(S):
        for h in range(H):
            ln = lengths[s]
            q = torch.from_numpy(Q[s, h])
            k = torch.from_numpy(K[s, h // 2, :ln])
            v = torch.from_numpy(V[s, h // 2, :ln])
            w = torch.softmax(k @ q / np.sqrt(d), dim=0)
            assert np.max(np.abs((w @ v).numpy() - O[s, h])) < 1e-12
            assert abs(torch.logsumexp(k @ q / np.sqrt(d), 0).item() - lse[s, h]) < 1e-12


def test_topk_recovers_planted_keys(oracle_mod):
    """Keys built to score highest (a large multiple of the query direction
    added to a chosen set P) are exactly the selected set."""
    S, H, Hkv, L, d, k = 1, 2, 1, 500, 32, 37
    Q, K, _ = _decode_inputs(S, H, Hkv, L, d, 82)
    Q[0, 1] = Q[0, 0]                        # both heads share the query direction
    P = np.sort(np.random.default_rng(5).choice(L, size=k, replace=False))
    qd = Q[0, 0] / np.linalg.norm(Q[0, 0])
    K[0, 0, P] += 40.0 * qd
    idx, n, kth, nxt = oracle_mod.topk_select(Q, K, k)
    for h in range(H):
        assert n[0, h] == k and np.array_equal(idx[0, h, :k], P)
        assert kth[0, h] > nxt[0, h]


def test_topk_matches_sort_of_numpy_scores(oracle_mod):
    """Against numpy: scores by einsum, order by (score desc, index asc) with
    lexsort; random lengths, all GQA groupings."""
    S, H, Hkv, L, d, k = 3, 8, 2, 300, 24, 41
    Q, K, _ = _decode_inputs(S, H, Hkv, L, d, 83)
    lengths = np.array([300, 41, 7])
    idx, n, kth, nxt = oracle_mod.topk_select(Q, K, k, lengths=lengths, scale=0.3)
    for s in range(S):
        for h in range(H):
            ln = lengths[s]
            sc = 0.3 * np.einsum("jd,d->j", K[s, h // 4, :ln], Q[s, h])
            order = np.lexsort((np.arange(ln), -sc))
            want = np.sort(order[:min(k, ln)])
            assert n[s, h] == len(want) and np.array_equal(idx[s, h, :n[s, h]], want)


def test_topk_ties_go_to_the_smaller_index(oracle_mod):
    """Equal scores (identical key rows) are taken in index order."""
    S, H, Hkv, L, d = 1, 1, 1, 50, 8
    Q, K, _ = _decode_inputs(S, H, Hkv, L, d, 84)
    K[0, 0, :] = K[0, 0, 0]
    K[0, 0, 30] = K[0, 0, 0] + Q[0, 0]       # the one strictly higher score
    idx, n, kth, nxt = oracle_mod.topk_select(Q, K, 5)
    assert idx[0, 0].tolist() == [0, 1, 2, 3, 30]


def test_topk_sets_are_nested_and_exclude_the_rest(oracle_mod):
    """Sets for growing top_k are nested; V rows outside G do not move the output."""
    S, H, Hkv, L, d = 1, 2, 1, 200, 16
    Q, K, V = _decode_inputs(S, H, Hkv, L, d, 85)
    prev = set()
    for k in (1, 5, 17, 64, 200):
        idx, n, _, _ = oracle_mod.topk_select(Q, K, k)
        cur = set(idx[0, 0, :n[0, 0]].tolist())
        assert prev <= cur and len(cur) == k
        prev = cur
    idx, n, _, _ = oracle_mod.topk_select(Q, K, 20)
    O1, _ = oracle_mod.gather(Q, K, V, idx, n)
    out = np.setdiff1d(np.arange(L), idx[0, 0, :20])
    V2 = V.copy()
    V2[0, 0, out] += 100.0
    O2, _ = oracle_mod.gather(Q, K, V2, idx, n)
    assert np.max(np.abs(O1[0, 0] - O2[0, 0])) < 1e-14


def test_bsfa_skipped_keys_in_denominator_variant(oracle_mod):
    """The variant reading (skipped blocks' keys stay in the softmax
    denominator): with every full block skipped (tau = +inf), lse is the dense
    causal lse, and each row's output is the default-rule output scaled by
    exp(lse_default - lse_variant) (same numerator, larger partition sum)."""
    import torch
    B, H, Hkv, N, d, Q, K, V = _bsfa_small(oracle_mod)
    opat = oracle_mod.Pattern(causal=1)
    tau = np.full(H, np.inf)
    O0, l0 = oracle_mod.prefill(opat, Q, K, V, thresholds=tau)
    O1, l1 = oracle_mod.prefill(opat, Q, K, V, thresholds=tau, keep_in_denominator=True)
    s = torch.einsum("bhid,bjd->bhij", torch.from_numpy(Q), torch.from_numpy(K[:, 0])) / np.sqrt(d)
    s = s.masked_fill(torch.triu(torch.ones(N, N, dtype=torch.bool), 1), float("-inf"))
    assert np.max(np.abs(torch.logsumexp(s, -1).numpy() - l1)) < 1e-10
    assert np.max(np.abs(O0 * np.exp(l0 - l1)[..., None] - O1)) < 1e-12
    # a tile whose blocks are all full and all skipped: O = 0, lse from the skipped keys alone
    bl = oracle_mod.Pattern(causal=0, block_local=128)
    Ob, lb = oracle_mod.prefill(bl, Q[:, :, :256], K[:, :, :256], V[:, :, :256], thresholds=tau,
                                keep_in_denominator=True)
    sb = torch.einsum("bhid,bjd->bhij", torch.from_numpy(Q[:, :, :256]),
                      torch.from_numpy(K[:, 0, :256])) / np.sqrt(d)
    blk = torch.arange(256) // 128
    sb = sb.masked_fill(blk[:, None] != blk[None, :], float("-inf"))
    assert np.all(Ob == 0)
    assert np.max(np.abs(torch.logsumexp(sb, -1).numpy() - lb)) < 1e-10


def _row_level_case(oracle_mod):
    """Causal window of 300 over N=512: tiles hold full blocks and partial blocks
    on both window edges."""
    B, H, Hkv, N, d, Q, K, V = _bsfa_small(oracle_mod, seed=47)
    p = oracle_mod.Pattern(causal=1, window=300, block_q=128, block_k=64)
    return B, H, Hkv, N, d, Q, K, V, p


def test_bsfa_row_level_extreme_thresholds(oracle_mod):
    """Row-level reading: tau = -inf drops nothing (the static pattern, bit for
    bit); tau = +inf drops every full block from every row, which is the tile
    rule's result at +inf."""
    B, H, Hkv, N, d, Q, K, V, p = _row_level_case(oracle_mod)
    O0, l0 = oracle_mod.prefill(p, Q, K, V)
    O1, l1 = oracle_mod.prefill(p, Q, K, V, thresholds=np.full(H, -np.inf), row_level=True)
    assert np.array_equal(O0, O1) and np.array_equal(l0, l1)
    O2, l2 = oracle_mod.prefill(p, Q, K, V, thresholds=np.full(H, np.inf), row_level=True)
    O3, l3 = oracle_mod.prefill(p, Q, K, V, thresholds=np.full(H, np.inf))
    assert np.array_equal(O2, O3) and np.array_equal(l2, l3)


def _median_tau(stat, full, H):
    """A threshold per head between two consecutive full-block statistics near
    their median (far from every statistic, so rounding cannot move a decision)."""
    tau = np.empty(H)
    for h in range(H):
        v = np.sort(stat[:, h][full[:, h]])
        k = (len(v) - 1) // 2
        tau[h] = 0.5 * (v[k] + v[k + 1])
    return tau


def test_bsfa_row_level_against_numpy_brute_force(oracle_mod):
    """Row-level reading against a numpy restatement of its definition: scores
    by einsum, G_i by the Python predicate, tile fullness by counting visible
    pairs, each row's maximum over each full block, the dropped blocks' keys
    removed from G_i, softmax over what is left.  Also: the skip set (blocks
    every row drops) is the tile rule's, and a row's per-block maxima reduce to
    the tile statistic."""
    B, H, Hkv, N, d, Q, K, V, p = _row_level_case(oracle_mod)
    scale = 1 / math.sqrt(d)
    _, _, mask_t, stat_t, full_t = oracle_mod.prefill(p, Q, K, V, want_blocks=True,
                                                      thresholds=np.full(H, -np.inf))
    tau = _median_tau(stat_t, full_t, H)
    O, lse, mask_r, stat_r, full_r, rstat = oracle_mod.prefill(
        p, Q, K, V, thresholds=tau, row_level=True, want_blocks=True, want_row_stats=True)
    _, _, mask_tile, _, _ = oracle_mod.prefill(p, Q, K, V, thresholds=tau, want_blocks=True)
    assert np.array_equal(mask_r, mask_tile)
    vis = np.array([[oracle_mod.visible_py(p, N, 0, i, j) for j in range(N)] for i in range(N)])
    T, n_kb = N // 128, N // 64
    full = np.array([[vis[t * 128:(t + 1) * 128, kb * 64:(kb + 1) * 64].all()
                      for kb in range(n_kb)] for t in range(T)])
    assert np.array_equal(full_r[0, 0], full)
    dropped_any = 0
    for h in range(H):
        S = scale * np.einsum("id,jd->ij", Q[0, h], K[0, 0])
        for i in range(N):
            t = i // 128
            keep = vis[i].copy()
            for kb in range(n_kb):
                if not full[t, kb]:
                    assert rstat.reshape(H, N, n_kb)[h, i, kb] == -np.inf
                    continue
                rm = S[i, kb * 64:(kb + 1) * 64].max()
                assert rstat.reshape(H, N, n_kb)[h, i, kb] == pytest.approx(rm, abs=1e-12)
                if rm < tau[h]:
                    keep[kb * 64:(kb + 1) * 64] = False
                    dropped_any += mask_r[0, h, t, kb] == 1
            s = S[i, keep]
            w = np.exp(s - s.max())
            out = (w / w.sum()) @ V[0, 0][keep]
            assert np.max(np.abs(out - O[0, h, i])) < 1e-12
            assert abs(lse[0, h, i] - (s.max() + np.log(w.sum()))) < 1e-12
        # the tile statistic is the largest of its rows' maxima
        rs = rstat.reshape(H, N, n_kb)[h].reshape(T, 128, n_kb).max(axis=1)
        assert np.allclose(rs[full], stat_t[0, h][full], rtol=0, atol=1e-12)
    # the reading changes something: rows drop blocks the tile keeps
    assert dropped_any > 0


def test_bsfa_row_level_override_keep_is_the_tile_rule(oracle_mod):
    """Forcing every row to keep (row override 0) leaves the tile rule's result."""
    B, H, Hkv, N, d, Q, K, V, p = _row_level_case(oracle_mod)
    _, _, _, stat_t, full_t = oracle_mod.prefill(p, Q, K, V, want_blocks=True,
                                                 thresholds=np.full(H, -np.inf))
    tau = _median_tau(stat_t, full_t, H)
    n_kb = N // 64
    keep_all = np.zeros((B * H * N, n_kb), np.int8)
    O1, l1 = oracle_mod.prefill(p, Q, K, V, thresholds=tau, row_level=True, row_override=keep_all)
    O2, l2 = oracle_mod.prefill(p, Q, K, V, thresholds=tau)
    assert np.array_equal(O1, O2) and np.array_equal(l1, l2)
    O3, l3 = oracle_mod.prefill(p, Q, K, V, thresholds=tau, row_level=True)
    assert not np.array_equal(O3, O2)
