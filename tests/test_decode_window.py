"""Decode over a minimum-size cache for a causal window + global tokens pattern.

The CPU part checks the cache layout; the GPU part compares the kernel with the
oracle's prefill row at the query's position over the full sequence (the
definition of the pattern), and bit for bit with the explicit-index gather over
the same cache with the slots of G_p in key order.
"""
import numpy as np
import pytest
import torch

from _parity import assert_close


def test_window_slot_layout(product):
    W, g = 7, 3
    assert [product.window_slot(j, W, g) for j in range(g)] == list(range(g))
    for p in range(g, 60):
        keys = range(max(g, p - W + 1), p + 1)           # the window part of G_p
        slots = [product.window_slot(j, W, g) for j in keys]
        assert len(set(slots)) == len(slots)               # distinct ring slots
        assert all(g <= s < g + W for s in slots)          # inside the W + g slots
    assert product.window_slot(-1, W, g) == -1
    assert product.window_slot(5, 0, g) == -1


def _rand(shape, seed, device):
    gen = torch.Generator(device="cpu").manual_seed(seed)
    return torch.randn(shape, generator=gen).to(torch.bfloat16).to(device)


def _case(product, W, g, H, Hkv, d, positions, seed, device):
    S = len(positions)
    N = max(positions) + 1
    Qf = _rand((S, H, N, d), seed, "cpu")
    Kf = _rand((S, Hkv, N, d), seed + 1, "cpu")
    Vf = _rand((S, Hkv, N, d), seed + 2, "cpu")
    C = W + g
    Kc = torch.zeros((S, Hkv, C, d), dtype=torch.bfloat16)
    Vc = torch.zeros((S, Hkv, C, d), dtype=torch.bfloat16)
    for s, p in enumerate(positions):
        for j in range(p + 1):                             # a decoder writes keys in order
            slot = product.window_slot(j, W, g)
            Kc[s, :, slot] = Kf[s, :, j]
            Vc[s, :, slot] = Vf[s, :, j]
    Q = torch.stack([Qf[s, :, p] for s, p in enumerate(positions)])
    return Qf, Kf, Vf, Kc.to(device), Vc.to(device), Q.to(device)


CASES = [
    dict(W=64, g=4, H=4, Hkv=2, d=128, positions=[0, 2, 3, 63, 67, 68, 200, 517]),
    dict(W=100, g=0, H=2, Hkv=2, d=64, positions=[0, 1, 99, 100, 101, 350]),
    dict(W=33, g=7, H=8, Hkv=2, d=128, positions=[6, 7, 39, 40, 41, 250]),
    dict(W=1, g=2, H=2, Hkv=1, d=64, positions=[0, 1, 2, 9]),
]


@pytest.mark.gpu
@pytest.mark.parametrize("case", range(len(CASES)))
def test_decode_window_matches_oracle_and_gather(product, oracle_mod, cuda, case):
    c = CASES[case]
    W, g, H, Hkv, d, positions = c["W"], c["g"], c["H"], c["Hkv"], c["d"], c["positions"]
    S = len(positions)
    Qf, Kf, Vf, Kc, Vc, Q = _case(product, W, g, H, Hkv, d, positions, 900 + 13 * case, cuda)
    pos_t = torch.tensor(positions, dtype=torch.int32, device=cuda)
    pat = product.Pattern(causal=1, window=W, n_global=g)
    lse = torch.empty((S, H), dtype=torch.float32, device=cuda)
    O = product.sparse_attn_decode_window(Q, Kc, Vc, pos_t, pat, lse=lse)
    product.check_device_error()

    # oracle: row p of the prefill over the full sequence, pattern as defined
    rows = np.array([(s, h, p) for s, p in enumerate(positions) for h in range(H)], np.int32)
    Or, lr = oracle_mod.prefill(oracle_mod.Pattern(causal=1, window=W, n_global=g), Qf, Kf, Vf,
                                rows=rows)
    assert_close(O.cpu().reshape(S * H, d), Or)
    assert_close(lse.cpu().reshape(S * H), lr, what="lse")

    # explicit gather over the same cache, slots of G_p in key order: same bytes
    n_idx = max(min(g, p + 1) + max(0, p - max(g, p - W + 1) + 1) for p in positions)
    idx = np.zeros((S, H, n_idx), np.int32)
    idx_len = np.zeros((S, H), np.int32)
    for s, p in enumerate(positions):
        keys = list(range(min(g, p + 1))) + list(range(max(g, p - W + 1), p + 1))
        sl = [product.window_slot(j, W, g) for j in keys]
        idx[s, :, :len(sl)] = sl
        idx_len[s, :] = len(sl)
    Og = product.sparse_attn_gather(Q, Kc, Vc, torch.from_numpy(idx).to(cuda),
                                    idx_len=torch.from_numpy(idx_len).to(cuda))
    product.check_device_error()
    assert torch.equal(O, Og)


@pytest.mark.gpu
def test_decode_window_negative_position_is_an_error(product, cuda):
    W, g, H, d = 16, 2, 2, 64
    Q = _rand((2, H, d), 5, cuda)
    Kc = _rand((2, H, W + g, d), 6, cuda)
    Vc = _rand((2, H, W + g, d), 7, cuda)
    pos = torch.tensor([-1, 5], dtype=torch.int32, device=cuda)
    O = product.sparse_attn_decode_window(Q, Kc, Vc, pos, product.Pattern(causal=1, window=W,
                                                                          n_global=g))
    with pytest.raises(product.SparseAttnError):
        product.check_device_error()
    assert torch.all(O[0] == 0)
    assert torch.isfinite(O[1].float()).all()


def test_decode_window_rejects_other_patterns(product):
    pat = product.Pattern(causal=0, window=8)
    with pytest.raises(ValueError):
        product.sparse_attn_decode_window(torch.zeros((1, 1, 64), dtype=torch.bfloat16),
                                          torch.zeros((1, 1, 9, 64), dtype=torch.bfloat16),
                                          torch.zeros((1, 1, 9, 64), dtype=torch.bfloat16),
                                          torch.zeros((1,), dtype=torch.int32), pat)


@pytest.mark.gpu
@pytest.mark.slow
def test_decode_window_full_size(product, oracle_mod, cuda):
    """window_decode at its full size (64 sequences, H=32, H_kv=8, d=128, W=4096,
    4 globals, positions up to 131071): every (sequence, head) output and lse
    against the oracle's gather over G_p, with G_p enumerated by the oracle from
    the pattern and its keys read from their cache slots (the layout: key j in
    slot j for j < g, else g + j mod W)."""
    from block_sparse_attention_29_b200.workloads import WORKLOADS, window_decode_inputs
    w = WORKLOADS["window_decode"]
    Q, Kc, Vc, pos = window_decode_inputs(w, device=cuda)
    pat = product.Pattern(causal=1, window=w.window, n_global=w.n_global)
    lse = torch.empty((w.S, w.H), dtype=torch.float32, device=cuda)
    O = product.sparse_attn_decode_window(Q, Kc, Vc, pos, pat, lse=lse)
    product.check_device_error()

    opat = oracle_mod.Pattern(causal=1, window=w.window, n_global=w.n_global)
    positions = pos.cpu().numpy()
    assert positions.max() <= w.max_pos and positions.min() >= w.window + w.n_global
    n = w.window + w.n_global
    Kk = torch.empty((w.S, w.H_kv, n, w.d), dtype=torch.bfloat16)
    Vk = torch.empty_like(Kk)
    for s, p in enumerate(positions):
        G = oracle_mod.build_G(opat, int(p) + 1, 0, int(p))
        assert len(G) == n and G[0] == 0 and G[-1] == p
        slots = np.where(G < w.n_global, G, w.n_global + G % w.window)
        ix = torch.from_numpy(slots.astype(np.int64)).to(cuda)
        Kk[s] = Kc[s][:, ix].cpu()
        Vk[s] = Vc[s][:, ix].cpu()
    idx = np.broadcast_to(np.arange(n, dtype=np.int32), (w.S, w.H, n)).copy()
    Or, lr = oracle_mod.gather(Q.cpu(), Kk, Vk, idx)
    assert_close(O, Or)
    assert_close(lse, lr, what="lse")
