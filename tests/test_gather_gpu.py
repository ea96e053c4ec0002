"""GPU explicit-index gather against the fp64 oracle."""
import numpy as np
import pytest
import torch

from block_sparse_attention_29_b200.workloads import (WORKLOADS, gather_index_sets,
                                                      gather_inputs)

from _parity import assert_close

pytestmark = pytest.mark.gpu


def _rand(shape, seed, device):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16).to(device)


@pytest.mark.parametrize("d,H,Hkv,H_idx,L,n_idx", [
    (128, 8, 2, 8, 1000, 300),
    (128, 8, 2, 2, 1000, 300),      # shared sets, 4 query heads per K/V head
    (128, 4, 2, 2, 700, 129),       # shared sets, 2 per K/V head
    (64, 8, 2, 2, 640, 200),
    (64, 4, 2, 2, 333, 57),
    (64, 4, 4, 4, 517, 517),
    (64, 6, 1, 6, 300, 33),
    (64, 6, 1, 1, 300, 33),         # shared sets, 6 per K/V head (one CTA per query head)
])
def test_gather_small(product, oracle_mod, cuda, d, H, Hkv, H_idx, L, n_idx):
    S = 3
    Q = _rand((S, H, d), 1, cuda)
    K = _rand((S, Hkv, L, d), 2, cuda)
    V = _rand((S, Hkv, L, d), 3, cuda)
    idx = gather_index_sets(S, H_idx, L, n_idx, min(16, n_idx - 1), seed=4).to(cuda)
    lse = torch.empty((S, H), device=cuda)
    O = product.sparse_attn_gather(Q, K, V, idx, lse=lse)
    product.check_device_error()
    Or, lr = oracle_mod.gather(Q.cpu(), K.cpu(), V.cpu(), idx.cpu().numpy())
    assert_close(O, Or)
    assert_close(lse, lr, what="lse")


def test_gather_ragged_lengths(product, oracle_mod, cuda):
    S, H, Hkv, d, L, n_idx = 4, 4, 2, 128, 600, 200
    Q, K, V = _rand((S, H, d), 5, cuda), _rand((S, Hkv, L, d), 6, cuda), _rand((S, Hkv, L, d), 7, cuda)
    idx = gather_index_sets(S, H, L, n_idx, 8, seed=8).to(cuda)
    lens = torch.tensor([[0, 1, 17, 200], [5, 0, 199, 64], [200, 200, 3, 2], [1, 1, 1, 0]],
                        dtype=torch.int32, device=cuda)
    lse = torch.empty((S, H), device=cuda)
    O = product.sparse_attn_gather(Q, K, V, idx, idx_len=lens, lse=lse)
    product.check_device_error()
    Or, lr = oracle_mod.gather(Q.cpu(), K.cpu(), V.cpu(), idx.cpu().numpy(), lens.cpu().numpy())
    assert_close(O, Or)
    assert_close(lse, lr, what="lse")
    assert torch.all(O[lens == 0] == 0)


@pytest.mark.parametrize("d,H,Hkv", [(128, 8, 2), (64, 4, 2)])
def test_gather_shared_sets_same_bytes_as_per_head_sets(product, cuda, d, H, Hkv):
    """Sets shared by the query heads of a K/V head (one CTA reads each row once
    for all of them) give the same bytes as the same sets given per query head."""
    S, L, n_idx = 3, 800, 250
    Q, K, V = _rand((S, H, d), 21, cuda), _rand((S, Hkv, L, d), 22, cuda), _rand((S, Hkv, L, d), 23, cuda)
    idx = gather_index_sets(S, Hkv, L, n_idx, 16, seed=24).to(cuda)
    lens = torch.randint(0, n_idx + 1, (S, Hkv), dtype=torch.int32,
                         generator=torch.Generator().manual_seed(25)).to(cuda)
    l1, l2 = torch.empty((S, H), device=cuda), torch.empty((S, H), device=cuda)
    O1 = product.sparse_attn_gather(Q, K, V, idx, idx_len=lens, lse=l1)
    per_head = idx.repeat_interleave(H // Hkv, dim=1).contiguous()
    lens_h = lens.repeat_interleave(H // Hkv, dim=1).contiguous()
    O2 = product.sparse_attn_gather(Q, K, V, per_head, idx_len=lens_h, lse=l2)
    product.check_device_error()
    assert torch.equal(O1, O2)
    assert torch.equal(l1, l2)


def test_gather_bad_index_is_reported(product, cuda):
    """An index outside [0, L) is skipped and reported through the device error word."""
    S, H, d, L = 1, 2, 64, 100
    Q, K, V = _rand((S, H, d), 9, cuda), _rand((S, H, L, d), 10, cuda), _rand((S, H, L, d), 11, cuda)
    idx = torch.tensor([[[0, 5, 7], [1, 2, 100]]], dtype=torch.int32, device=cuda)
    product.sparse_attn_gather(Q, K, V, idx)
    with pytest.raises(product.SparseAttnError) as e:
        product.check_device_error()
    assert e.value.code == product.SA_ERR_DEVICE_INDEX
    product.check_device_error()          # cleared


@pytest.mark.slow
def test_gather_full_size_sampled(product, oracle_mod, cuda):
    """gather_decode at full size; sampled (sequence, head) pairs checked against the
    oracle on the referenced cache rows only."""
    w = WORKLOADS["gather_decode"]
    Q, K, V, idx = gather_inputs(w, device=cuda)
    O = product.sparse_attn_gather(Q, K, V, idx)
    product.check_device_error()
    g = np.random.default_rng(w.seed)
    pairs = [(0, 0), (w.S - 1, w.H - 1)] + [(int(g.integers(w.S)), int(g.integers(w.H)))
                                            for _ in range(30)]
    group = w.H // w.H_kv
    for s, h in pairs:
        ix = idx[s, h].long()
        Ks = K[s, h // group, ix].cpu()[None, None]
        Vs = V[s, h // group, ix].cpu()[None, None]
        local = np.arange(len(ix), dtype=np.int32)[None, None]
        Or, _ = oracle_mod.gather(Q[s, h].cpu()[None, None], Ks, Vs, local)
        assert_close(O[s, h].cpu()[None, None], Or)
    assert torch.isfinite(O).all()
