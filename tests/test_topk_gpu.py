"""Dynamic top-K decode on the GPU against the fp64 oracle.

The selected sets are compared with the oracle's: where the two differ, every
key in the difference must score within NEAR of the oracle's top_k-th score
(the GPU ranks fp32 scores, the oracle fp64 ones, so keys at the cut may swap).
The GPU's output is then compared element by element with the oracle's output
over the GPU's own set (so the attention itself is checked exactly where the
selection is legitimately ambiguous).  Sets must be ascending, unique, of size
min(top_k, len) and inside [0, len).
"""
import numpy as np
import pytest
import torch

from block_sparse_attention_29_b200.workloads import WORKLOADS, topk_decode_inputs

from _parity import assert_close

pytestmark = pytest.mark.gpu

NEAR = 1e-3   # natural-log scaled-logit units


def _rand(shape, seed, device):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16).to(device)


def _check_sets(oracle_mod, Qc, Kc, top_k, lengths, idx, n, scale):
    """Compares the GPU sets (idx, n) with the oracle's; returns the number of
    keys that differ (all of them near the cut)."""
    S, H, d = Qc.shape
    Hkv = Kc.shape[1]
    L = Kc.shape[2]
    oidx, on, kth, nxt = oracle_mod.topk_select(Qc, Kc, top_k, lengths=lengths, scale=scale)
    assert np.array_equal(n, on)
    q = Qc.double().numpy()
    k = Kc.double().numpy()
    differ = 0
    for s in range(S):
        ln = L if lengths is None else int(lengths[s])
        for h in range(H):
            m = int(n[s, h])
            g = idx[s, h, :m]
            assert m == min(top_k, ln)
            assert np.all(np.diff(g) > 0) and (m == 0 or (g[0] >= 0 and g[-1] < ln))
            diff = np.setxor1d(g, oidx[s, h, :m])
            if diff.size:
                sc = scale * (k[s, h // (H // Hkv), diff] @ q[s, h])
                assert np.all(np.abs(sc - kth[s, h]) <= NEAR), (s, h, diff, sc, kth[s, h])
                differ += diff.size
    return differ


# (S, H, H_kv, L, d, top_k, lengths)
CASES = [
    (2, 4, 2, 1000, 128, 64, None),                 # 2 query heads per K/V head
    (3, 8, 2, 5000, 64, 300, [5000, 17, 2999]),     # d=64, a sequence shorter than top_k
    (1, 2, 1, 100, 128, 200, None),                 # top_k > L: every key
    (2, 4, 4, 4096, 128, 1, None),                  # top-1, one head per K/V head
    (1, 8, 1, 3001, 128, 1024, [3001]),             # 8 heads per K/V head, L not a multiple of 4
    (2, 3, 1, 2000, 64, 100, [0, 2000]),            # 3 heads per K/V head, an empty sequence
    (1, 4, 1, 20000, 128, 2048, None),              # several score chunks
    (1, 2, 2, 9000, 128, 4000, [8193]),             # a length one past a chunk boundary
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_topk_decode_matches_oracle(product, oracle_mod, cuda, case):
    S, H, Hkv, L, d, top_k, lengths = CASES[case]
    seed = 900 + 13 * case
    Q = _rand((S, H, d), seed, cuda)
    K = _rand((S, Hkv, L, d), seed + 1, cuda)
    V = _rand((S, Hkv, L, d), seed + 2, cuda)
    ln = None if lengths is None else torch.tensor(lengths, dtype=torch.int32, device=cuda)
    lse = torch.empty((S, H), dtype=torch.float32, device=cuda)
    O, idx, n = product.sparse_attn_decode_topk(Q, K, V, top_k, lengths=ln, lse=lse)
    product.check_device_error()
    idx, n = idx.cpu().numpy(), n.cpu().numpy()
    scale = 1.0 / np.sqrt(d)
    _check_sets(oracle_mod, Q.cpu(), K.cpu(), top_k, lengths, idx, n, scale)
    Or, lr = oracle_mod.gather(Q.cpu(), K.cpu(), V.cpu(), idx, n)
    assert_close(O, Or)
    assert_close(lse, lr, what="lse")


def test_topk_decode_ties_and_planted_keys(product, oracle_mod, cuda):
    """Equal scores are taken in index order (every key of head group 0 is the
    same row); keys built to score highest (group 1) are found exactly."""
    S, H, Hkv, L, d, top_k = 1, 4, 2, 3000, 128, 50
    Q = _rand((S, H, d), 71, cuda)
    K = _rand((S, Hkv, L, d), 72, cuda)
    V = _rand((S, Hkv, L, d), 73, cuda)
    K[0, 0] = K[0, 0, 7]
    P = torch.from_numpy(np.sort(np.random.default_rng(3).choice(L, top_k, replace=False)))
    Qf = Q.float()
    Q[0, 3] = Q[0, 2]
    qd = Qf[0, 2] / Qf[0, 2].norm()
    K[0, 1, P.to(cuda)] = (K[0, 1, P.to(cuda)].float() + 30.0 * qd).to(torch.bfloat16)
    O, idx, n = product.sparse_attn_decode_topk(Q, K, V, top_k)
    product.check_device_error()
    idx = idx.cpu()
    for h in (0, 1):
        assert idx[0, h].tolist() == list(range(top_k))
    for h in (2, 3):
        assert torch.equal(idx[0, h], P.to(torch.int32))
    Or, _ = oracle_mod.gather(Q.cpu(), K.cpu(), V.cpu(), idx.numpy(), n.cpu().numpy())
    assert_close(O, Or)


def test_topk_decode_repeatable_and_workspace_checked(product, cuda):
    S, H, Hkv, L, d, top_k = 2, 8, 2, 6000, 128, 500
    Q = _rand((S, H, d), 81, cuda)
    K = _rand((S, Hkv, L, d), 82, cuda)
    V = _rand((S, Hkv, L, d), 83, cuda)
    need = product.decode_topk_workspace_bytes(S, H, L, top_k)
    ws = torch.empty(need, dtype=torch.uint8, device=cuda)
    O1, i1, n1 = product.sparse_attn_decode_topk(Q, K, V, top_k, workspace=ws)
    O2, i2, n2 = product.sparse_attn_decode_topk(Q, K, V, top_k, workspace=ws)
    torch.cuda.synchronize()
    product.check_device_error()
    assert torch.equal(O1, O2) and torch.equal(i1, i2) and torch.equal(n1, n2)
    with pytest.raises(product.SparseAttnError):
        product.sparse_attn_decode_topk(Q, K, V, top_k, workspace=ws[: need - 256])
    with pytest.raises(product.SparseAttnError):
        product.sparse_attn_decode_topk(Q, K, V, 0, workspace=ws)


def test_topk_decode_bad_length_is_reported(product, cuda):
    S, H, Hkv, L, d = 2, 2, 1, 500, 64
    Q = _rand((S, H, d), 91, cuda)
    K = _rand((S, Hkv, L, d), 92, cuda)
    V = _rand((S, Hkv, L, d), 93, cuda)
    ln = torch.tensor([500, -3], dtype=torch.int32, device=cuda)
    O, idx, n = product.sparse_attn_decode_topk(Q, K, V, 10, lengths=ln)
    with pytest.raises(product.SparseAttnError):
        product.check_device_error()
    assert n.cpu().tolist() == [[10, 10], [0, 0]]
    assert torch.all(O[1] == 0)


@pytest.mark.slow
def test_topk_decode_full_size_sampled(product, oracle_mod, cuda):
    """The benchmark's workload (64 sequences, 131072 keys, top 2048) in its
    launch configuration; sampled (sequence, head) queries against the oracle."""
    w = WORKLOADS["topk_decode"]
    Q, K, V = topk_decode_inputs(w, device=cuda)
    lse = torch.empty((w.S, w.H), dtype=torch.float32, device=cuda)
    O, idx, n = product.sparse_attn_decode_topk(Q, K, V, w.top_k, lse=lse)
    product.check_device_error()
    assert torch.all(n == w.top_k)
    g = np.random.default_rng(w.seed)
    pairs = sorted({(0, 0), (w.S - 1, w.H - 1)} |
                   {(int(g.integers(w.S)), int(g.integers(w.H))) for _ in range(10)})
    group = w.H // w.H_kv
    for s, h in pairs:
        Qs = Q[s, h][None, None].cpu()
        Ks = K[s, h // group][None, None].cpu()
        Vs = V[s, h // group][None, None].cpu()
        gi = idx[s, h][None, None].cpu().numpy()
        gn = n[s, h].reshape(1, 1).cpu().numpy()
        _check_sets(oracle_mod, Qs, Ks, w.top_k, None, gi, gn, 1.0 / np.sqrt(w.d))
        Or, lr = oracle_mod.gather(Qs, Ks, Vs, gi, gn)
        assert_close(O[s, h][None, None], Or)
        assert_close(lse[s, h].reshape(1, 1), lr, what="lse")


@pytest.mark.parametrize("L,top_k,two_levels", [(4096, 300, False), (20000, 100, False),
                                                 (20000, 12000, True), (32768, 500, "cluster")],
                         ids=["ties-over-segments", "overfull-bin", "overfull-bin-two-levels",
                              "clustered-bin"])
def test_topk_decode_ties_in_index_order(product, oracle_mod, cuda, L, top_k, two_levels):
    """Equal scores are taken in index order when they span several of the
    select pass's row segments, when the threshold's first-level bin holds
    more keys than shared memory keeps (its three-sweep path), and when the
    bin's keys crowd one segment beyond its share of shared memory (1000 equal
    keys in the first of 32 segments).  Checked exactly: the near-cut
    tolerance of the other tests would accept any choice of ties."""
    S, H, Hkv, d = 1, 2, 1, 128
    Q = _rand((S, H, d), L + top_k, cuda)
    Q[0, 1] = Q[0, 0]
    K = _rand((S, Hkv, L, d), L + top_k + 1, cuda)
    V = _rand((S, Hkv, L, d), L + top_k + 2, cuda)
    row_b = K[0, 0, 5].clone()
    K[0, 0] = row_b
    if two_levels == "cluster":
        # keys 0..999 score higher (the same row plus the query direction)
        row_a = (row_b.float() + Q[0, 0].float() / Q[0, 0].float().norm()).to(torch.bfloat16)
        K[0, 0, :1000] = row_a
        want = np.arange(top_k)
    elif two_levels:
        # even keys score higher (the same row plus the query direction)
        row_a = (row_b.float() + Q[0, 0].float() / Q[0, 0].float().norm()).to(torch.bfloat16)
        K[0, 0, 0::2] = row_a
        want = np.sort(np.concatenate([np.arange(0, L, 2), np.arange(1, L, 2)[:top_k - L // 2]]))
    else:
        want = np.arange(top_k)
    O, idx, n = product.sparse_attn_decode_topk(Q, K, V, top_k)
    product.check_device_error()
    idx, n = idx.cpu().numpy(), n.cpu().numpy()
    for h in range(H):
        assert n[0, h] == top_k
        assert np.array_equal(idx[0, h], want)
    Or, _ = oracle_mod.gather(Q.cpu(), K.cpu(), V.cpu(), idx, n)
    assert_close(O, Or)
