"""Host-side argument checks of the Python binding (no GPU needed): a tensor
must have the declared dtype, shape and layout and live on the current CUDA
device before any pointer reaches the library."""
import types

import pytest
import torch


def _fake(shape, dtype, dev_index=0, contiguous=True):
    # stands in for a CUDA tensor: only the attributes the checks read
    t = types.SimpleNamespace(dtype=dtype, shape=torch.Size(shape),
                              device=torch.device("cuda", dev_index))
    t.is_contiguous = lambda: contiguous
    return t


def test_check_tensor_accepts_a_matching_tensor(product, monkeypatch):
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    product._check_tensor("Q", _fake((2, 4, 64, 128), torch.bfloat16), (2, 4, 64, 128),
                          torch.bfloat16)


def test_check_tensor_rejects_each_mismatch(product, monkeypatch):
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    shape = (2, 4, 64, 128)
    with pytest.raises(TypeError, match="Q must be"):
        product._check_tensor("Q", _fake(shape, torch.float16), shape, torch.bfloat16)
    with pytest.raises(ValueError, match="shape"):
        product._check_tensor("Q", _fake((2, 4, 64, 64), torch.bfloat16), shape, torch.bfloat16)
    with pytest.raises(ValueError, match="contiguous"):
        product._check_tensor("Q", _fake(shape, torch.bfloat16, contiguous=False), shape,
                              torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensor"):
        cpu = types.SimpleNamespace(dtype=torch.bfloat16, shape=torch.Size(shape),
                                    device=torch.device("cpu"), is_contiguous=lambda: True)
        product._check_tensor("Q", cpu, shape, torch.bfloat16)


def test_check_tensor_rejects_another_device(product, monkeypatch):
    """A tensor on cuda:1 while cuda:0 is current would hand the kernels a
    pointer into the other device's memory."""
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    shape = (8,)
    with pytest.raises(ValueError, match="cuda:1, the current device is cuda:0"):
        product._check_tensor("thresholds", _fake(shape, torch.float32, dev_index=1), shape,
                              torch.float32)


def test_block_layout_tiles(product):
    """(T_q, n_kb) of the block-mask layout: 128-row query tiles, 64-key blocks."""
    assert product._tiles(1) == (1, 1)
    assert product._tiles(128) == (1, 2)
    assert product._tiles(129) == (2, 3)
    assert product._tiles(32768) == (256, 512)
