"""The prefill entry point that allocates no device memory.

Some callers cannot call cudaMalloc at run time (their device memory belongs
to an external pool or allocator, or their runtime forbids allocation on the
inference path).  sparse_attn_prefill_noalloc serves them from a fixed static
device array.  This file runs last so that, if it fails, a run that stops at
the first failure has already run every other test; it passes alone in a fresh
process too (the entry point sets itself up on first use).
"""
import ctypes

import numpy as np
import pytest
import torch

from block_sparse_attention_29_b200.workloads import random_table


def _rand(shape, seed, device):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16).to(device)


def _noalloc_call(product, Q, K, V, O, pattern, thresholds=None, lse=None):
    """Calls the C ABI directly (ctypes), as a C caller would."""
    L = product._lib.lib()
    B, H, N, d = Q.shape
    st, _tab = pattern.to_c(thresholds.data_ptr() if thresholds is not None else 0)
    rc = L.sparse_attn_prefill_noalloc(Q.data_ptr(), K.data_ptr(), V.data_ptr(), O.data_ptr(),
                                       B, H, K.shape[1], N, d, ctypes.byref(st),
                                       lse.data_ptr() if lse is not None else None,
                                       torch.cuda.current_stream().cuda_stream or None)
    return rc


@pytest.mark.gpu
def test_noalloc_matches_allocating_entry_two_calls(product, cuda):
    # first call: causal window, GQA, d=128, ragged N
    B, H, Hkv, N, d = 1, 4, 2, 1000, 128
    Q, K, V = _rand((B, H, N, d), 1, cuda), _rand((B, Hkv, N, d), 2, cuda), _rand((B, Hkv, N, d), 3, cuda)
    pat1 = product.Pattern(causal=1, window=300, n_global=4)
    ref1 = product.sparse_attn_prefill(Q, K, V, pat1)
    O1 = torch.empty_like(Q)
    assert _noalloc_call(product, Q, K, V, O1, pat1) == product.SA_OK
    # second call in a row: a different pattern (random blocks, d=64) overwrites
    # the shared static array
    B2, H2, N2, d2 = 2, 3, 700, 64
    tab = random_table(H2, N2, 64, 2, seed=5)
    Q2, K2, V2 = (_rand((B2, H2, N2, d2), s, cuda) for s in (4, 5, 6))
    pat2 = product.Pattern(causal=0, window=128, n_global=8, n_random=2, random_block=64,
                           random_table=tab)
    ref2 = product.sparse_attn_prefill(Q2, K2, V2, pat2)
    O2 = torch.empty_like(Q2)
    lse2 = torch.empty((B2, H2, N2), device=cuda)
    assert _noalloc_call(product, Q2, K2, V2, O2, pat2, lse=lse2) == product.SA_OK
    product.check_device_error()
    # the same kernel over the same block lists and work order: the same bytes
    assert torch.equal(O1, ref1)
    assert torch.equal(O2, ref2)
    assert torch.isfinite(lse2).all()
    # and the first pattern again, after the second one
    O3 = torch.empty_like(Q)
    assert _noalloc_call(product, Q, K, V, O3, pat1) == product.SA_OK
    product.check_device_error()
    assert torch.equal(O3, ref1)


@pytest.mark.gpu
def test_noalloc_block_skip_rule(product, cuda):
    B, H, Hkv, N, d = 1, 2, 1, 768, 128
    Q, K, V = _rand((B, H, N, d), 7, cuda), _rand((B, Hkv, N, d), 8, cuda), _rand((B, Hkv, N, d), 9, cuda)
    tau = torch.tensor([0.3, 0.5], dtype=torch.float32, device=cuda)
    pat = product.Pattern(causal=1)
    ref = product.Plan(pat, B, H, Hkv, N, d).prefill(Q, K, V, thresholds=tau)
    O = torch.empty_like(Q)
    assert _noalloc_call(product, Q, K, V, O, pat, thresholds=tau) == product.SA_OK
    product.check_device_error()
    assert torch.equal(O, ref)


def _too_large():
    """A pattern whose plan data exceeds the fixed array: per-head random tables
    grow with H, and 64 heads over N = 262144 with 8 random blocks need more
    than 8 MiB (the random table alone is 8 MiB)."""
    B, H, N, d = 1, 64, 262144, 64
    tab = np.broadcast_to(np.arange(8, dtype=np.int32), (H, N // 64, 8)).copy()
    return B, H, N, d, tab


@pytest.mark.gpu
def test_noalloc_rejects_patterns_beyond_its_limit(product, cuda):
    B, H, N, d, tab = _too_large()
    pat = product.Pattern(causal=0, n_random=8, random_block=64, random_table=tab)
    L = product._lib.lib()
    st, _t = pat.to_c()
    # Tensors of the full declared size (2 GiB each), so that even a launch
    # would stay inside them; O holds a sentinel that any kernel would overwrite.
    Q, K, V = (torch.zeros((B, H, N, d), dtype=torch.bfloat16, device=cuda) for _ in range(3))
    O = torch.full((B, H, N, d), float("nan"), dtype=torch.bfloat16, device=cuda)
    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    rc = L.sparse_attn_prefill_noalloc(Q.data_ptr(), K.data_ptr(), V.data_ptr(), O.data_ptr(),
                                       B, H, H, N, d, ctypes.byref(st), None, s.cuda_stream)
    assert rc == product.SA_ERR_INVALID_ARG
    assert "no-alloc" in L.sparse_attn_last_error().decode()
    assert s.query(), "a rejected call queued device work"
    torch.cuda.synchronize()
    assert torch.isnan(O).all()
    product.check_device_error()


def test_noalloc_size_rule_is_checked_on_the_host(product):
    """Without a GPU: the size rule rejects the call before any CUDA call is
    made, so the (never dereferenced) pointers may be arbitrary aligned values."""
    import torch as _t
    if _t.cuda.is_available():
        pytest.skip("host-only check; the GPU test above covers the same rule with real buffers")
    B, H, N, d, tab = _too_large()
    pat = product.Pattern(causal=0, n_random=8, random_block=64, random_table=tab)
    L = product._lib.lib()
    st, _t2 = pat.to_c()
    fake = 1 << 20
    rc = L.sparse_attn_prefill_noalloc(fake, fake, fake, fake, B, H, H, N, d, ctypes.byref(st),
                                       None, None)
    assert rc == product.SA_ERR_INVALID_ARG
    assert "no-alloc" in L.sparse_attn_last_error().decode()
