"""Split tiles on the GPU: a block list cut into pieces (each a work unit with
an unnormalised partial result) and merged afterwards must give the oracle's
output, and the per-block statistics and decisions of the unsplit plan.
"""
import dataclasses

import numpy as np
import pytest
import torch

from block_sparse_attention_29_b200.workloads import (WORKLOADS, calibration_inputs,
                                                      prefill_inputs, random_table)

from _parity import NEAR_BAND, assert_close, compare_masks

pytestmark = pytest.mark.gpu


def _rand(shape, seed, device):
    g = torch.Generator(device="cpu").manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16).to(device)


SPLIT_CASES = [
    dict(B=1, H=2, Hkv=2, N=1000, d=128, causal=1),
    dict(B=2, H=4, Hkv=2, N=700, d=128, causal=0, window=150, n_global=7),
    dict(B=1, H=2, Hkv=1, N=777, d=64, causal=0, window=130, n_global=9),
    dict(B=1, H=4, Hkv=2, N=1100, d=128, causal=1, window=520, n_global=3),
    dict(B=1, H=8, Hkv=2, N=1, d=128, causal=1),
]


@pytest.mark.parametrize("mub", [1, 3, 7])
@pytest.mark.parametrize("case", range(len(SPLIT_CASES)))
def test_split_matches_oracle(product, oracle_mod, cuda, case, mub):
    c = dict(SPLIT_CASES[case])
    B, H, Hkv, N, d = (c.pop(k) for k in ("B", "H", "Hkv", "N", "d"))
    seed = 500 + 11 * case
    Q, K, V = (_rand(s, seed + k, cuda) for k, s in
               enumerate(((B, H, N, d), (B, Hkv, N, d), (B, Hkv, N, d))))
    pat = product.Pattern(**c)
    plan = product.Plan(pat, B, H, Hkv, N, d, max_unit_blocks=mub)
    if N > 128 or c.get("causal", 0) == 0:
        assert plan.info["split_tiles"] > 0
    lse = torch.empty((B, H, N), dtype=torch.float32, device=cuda)
    O = plan.prefill(Q, K, V, lse=lse)
    product.check_device_error()
    Or, lr = oracle_mod.prefill(oracle_mod.Pattern(**c), Q.cpu(), K.cpu(), V.cpu())
    assert_close(O, Or)
    assert_close(lse, lr, what="lse")
    # repeated launches of the same plan reuse the workspace: same bytes
    O2 = plan.prefill(Q, K, V)
    torch.cuda.synchronize()
    assert torch.equal(O, O2)


def test_split_random_blocks_and_empty_rows(product, oracle_mod, cuda):
    """Pieces whose rows see no key (causal rows before their random block)
    contribute nothing; a row with no key anywhere gives O = 0, lse = -inf."""
    B, H, N, d = 1, 2, 512, 64
    tab = np.full((H, 8, 1), 6, np.int32)       # every 64-row block sees key block 6
    c = dict(causal=1, n_random=1, random_block=64)
    Q, K, V = (_rand((B, H, N, d), 900 + k, cuda) for k in range(3))
    plan = product.Plan(product.Pattern(**c, random_table=tab), B, H, H, N, d, max_unit_blocks=1)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=cuda)
    O = plan.prefill(Q, K, V, lse=lse)
    product.check_device_error()
    Or, lr = oracle_mod.prefill(oracle_mod.Pattern(**c, random_table=tab), Q.cpu(), K.cpu(),
                                V.cpu())
    assert_close(O, Or)
    assert_close(lse, lr, what="lse")
    assert torch.all(O[0, :, :384] == 0) and torch.all(torch.isinf(lse[0, :, :384]))

    tab = random_table(H, N, 64, 3, seed=78)
    c = dict(causal=0, window=64, n_global=16, n_random=3, random_block=64)
    plan = product.Plan(product.Pattern(**c, random_table=tab), B, H, H, N, d, max_unit_blocks=2)
    O = plan.prefill(Q, K, V, lse=lse)
    product.check_device_error()
    Or, lr = oracle_mod.prefill(oracle_mod.Pattern(**c, random_table=tab), Q.cpu(), K.cpu(),
                                V.cpu())
    assert_close(O, Or)
    assert_close(lse, lr, what="lse")


def _bsfa_case(oracle_mod, d):
    w = dataclasses.replace(WORKLOADS["bsfa_causal"], N=1024, H=4, H_kv=2, d=d)
    Qc, Kc, Vc, _ = calibration_inputs(w, device="cpu")
    opat = oracle_mod.Pattern(**w.pattern_fields())
    full_c, stat_c, _ = oracle_mod.block_stats(opat, Qc, Kc)
    tau = oracle_mod.calibrate_thresholds(full_c, stat_c).astype(np.float32).astype(np.float64)
    return w, opat, tau


@pytest.mark.parametrize("variant", ["tile", "denominator", "row_level"])
@pytest.mark.parametrize("d", [128, 64])
def test_split_block_skip_rule(product, oracle_mod, cuda, d, variant):
    """The rule's statistics and decisions are per block: a split plan writes
    the same statistics and masks as the unsplit plan, bit for bit, and its
    output matches the oracle's replay of those decisions."""
    w, opat, tau = _bsfa_case(oracle_mod, d)
    Q, K, V, _ = prefill_inputs(w, device="cpu")
    Q, K, V = Q.to(cuda), K.to(cuda), V.to(cuda)
    extra = {"tile": {}, "denominator": {"skipped_in_denominator": 1},
             "row_level": {"row_level_skip": 1}}[variant]
    pat = product.Pattern(**w.pattern_fields(), **extra)
    tau_d = torch.tensor(tau, dtype=torch.float32, device=cuda)
    res = {}
    for mub in (-1, 3):
        plan = product.Plan(pat, w.B, w.H, w.H_kv, w.N, w.d, max_unit_blocks=mub)
        assert (plan.info["split_tiles"] > 0) == (mub > 0)
        mask = torch.empty((w.B, w.H, plan.T, plan.n_kb), dtype=torch.uint8, device=cuda)
        stat = torch.full((w.B, w.H, plan.T, plan.n_kb), float("-inf"), device=cuda)
        lse = torch.empty((w.B, w.H, w.N), device=cuda)
        O = plan.prefill(Q, K, V, thresholds=tau_d, lse=lse, block_mask=mask, block_stat=stat)
        product.check_device_error()
        res[mub] = (O, lse, mask, stat)
    assert torch.equal(res[-1][2], res[3][2])
    assert torch.equal(res[-1][3], res[3][3])
    O, lse, mask, stat = res[3]
    Qh, Kh, Vh = Q.cpu(), K.cpu(), V.cpu()
    _, _, om, ost, _ = oracle_mod.prefill(opat, Qh, Kh, Vh, thresholds=tau, want_blocks=True)
    n, n_near, override = compare_masks(mask.cpu().numpy(), om, ost, tau)
    kw = dict(thresholds=tau, override=override)
    if variant == "denominator":
        kw["keep_in_denominator"] = True
    ok = np.ones(w.B * w.H * w.N, bool)
    if variant == "row_level":
        # rows with a (row, block) maximum near the threshold may decide either
        # way; the others must match the oracle
        Or, lr, _, _, _, rstat = oracle_mod.prefill(opat, Qh, Kh, Vh, row_level=True,
                                                    want_blocks=True, want_row_stats=True, **kw)
        tau_r = np.repeat(tau, w.N)[:, None]   # per flat row [H*N] (B = 1)
        near = np.isfinite(rstat) & (np.abs(rstat - tau_r) <= NEAR_BAND)
        ok[np.nonzero(near.any(axis=1))[0]] = False
    else:
        Or, lr = oracle_mod.prefill(opat, Qh, Kh, Vh, **kw)
    Og, lg = O.cpu().reshape(-1, w.d), lse.cpu().reshape(-1)
    Or, lr = Or.reshape(-1, w.d), lr.reshape(-1)
    assert ok.mean() > 0.9
    assert_close(Og[torch.from_numpy(ok)], Or[ok])
    assert_close(lg[torch.from_numpy(ok)], lr[ok], what="lse")
    # against the unsplit plan: the same decisions, the same sums in another order
    assert_close(O, res[-1][0].cpu().double().numpy())
    assert_close(lse, res[-1][1].cpu().double().numpy(), what="lse")


def test_split_dilated(product, oracle_mod, cuda):
    B, H, Hkv, N, d = 1, 2, 1, 1024, 128
    c = dict(causal=1, window=100, dilation=4)
    Q, K, V = (_rand(s, 950 + k, cuda) for k, s in
               enumerate(((B, H, N, d), (B, Hkv, N, d), (B, Hkv, N, d))))
    plan = product.Plan(product.Pattern(**c), B, H, Hkv, N, d, max_unit_blocks=1)
    assert plan.info["split_tiles"] > 0
    lse = torch.empty((B, H, N), dtype=torch.float32, device=cuda)
    O = plan.prefill(Q, K, V, lse=lse)
    product.check_device_error()
    Or, lr = oracle_mod.prefill(oracle_mod.Pattern(**c), Q.cpu(), K.cpu(), V.cpu())
    assert_close(O, Or)
    assert_close(lse, lr, what="lse")


def test_split_global_rows_automatic(product, oracle_mod, cuda):
    """The automatic rule on a window + global + random-block pattern (the
    BigBird/Longformer mix) cuts the tile of the global rows; those rows and a
    sample of the others match the oracle."""
    w = dataclasses.replace(WORKLOADS["longformer_bigbird"], B=1, H=2, H_kv=2, N=16384)
    Q, K, V, tab = prefill_inputs(w, device=cuda)
    plan = product.Plan(product.Pattern(**w.pattern_fields(), random_table=tab), w.B, w.H,
                        w.H_kv, w.N, w.d)
    assert plan.info["split_tiles"] == w.B * w.H
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=cuda)
    O = plan.prefill(Q, K, V, lse=lse)
    product.check_device_error()
    rows = np.array([(0, h, i) for h in range(w.H) for i in
                     list(range(0, 128, 5)) + [127, 128, 4000, w.N - 1]], dtype=np.int32)
    opat = oracle_mod.Pattern(**w.pattern_fields(), random_table=tab)
    Or, lr = oracle_mod.prefill(opat, Q.cpu(), K.cpu(), V.cpu(), rows=rows)
    sel = tuple(torch.from_numpy(rows[:, k]).long() for k in range(3))
    assert_close(O.cpu()[sel], Or)
    assert_close(lse.cpu()[sel], lr, what="lse")
