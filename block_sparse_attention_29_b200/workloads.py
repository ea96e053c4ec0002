"""Seeded synthetic inputs for the five workloads (no attention arithmetic here).

Shared by the tests and the benchmark, so that the CUDA path and its checks
see the same bytes.  Everything is drawn from torch
generators seeded as: Q = base, K = base + 1, V = base + 2, structure (unit
directions, marked positions, random-block tables, index sets) = base + 3 ...,
calibration draw = base + 100, with base = 1000 * workload number.  Values
are drawn in float32 and rounded once to bf16.

Workloads (names used by tests and bench):
  tiny_static         B=1 H=H_kv=2 N=256 d=64, causal and (window 64 or globals 0..3),
                      blocks 64x64
  mistral_swa         B=1 H=32 H_kv=8 N=8192 d=128, causal window 4096, blocks 128x64
  bsfa_causal         B=1 H=32 H_kv=8 N=32768 d=128, causal, block-skip rule;
                      K = N(0,1) + 4 u_h on floor(0.02 N) marked positions per K/V head,
                      Q = N(0,1) + 2 u_{h_kv(h)}, u_h a unit vector per K/V head
  longformer_bigbird  B=2 H=H_kv=16 N=65536 d=64, non-causal window 512 + 64 global
                      tokens + 3 random 64-key blocks per 64-query block
  gather_decode       64 sequences x 1 query, H=32 H_kv=8 d=128, cache length 131072,
                      2048 sorted unique indices per (sequence, head) = {0} and the last
                      128 positions and 1919 uniform draws from {1 .. L-129}
  window_decode       64 sequences x 1 query, H=32 H_kv=8 d=128, causal window 4096 +
                      4 global tokens over a cache of 4100 slots, positions past the window
  dilated_swa         B=1 H=32 H_kv=8 N=32768 d=128, causal dilated window: 2048 taps
                      8 apart (receptive field 16384), blocks 128x64
  topk_decode         64 sequences x 1 query, H=32 H_kv=8 d=128, cache length 131072,
                      each query's 2048 highest-scoring keys (dynamic top-K)
  bsfa_denominator    bsfa_causal's inputs and thresholds with the rule's variant that
                      keeps skipped blocks' keys in the softmax denominator
  bsfa_causal_noskip  bsfa_causal's inputs with thresholds of -inf (every block computed
                      and kept: the baseline of the rule's savings)
  bsfa_row_level      bsfa_causal's inputs and thresholds with the row-level reading of
                      the rule (rows also drop kept blocks below the threshold)
  longformer_split    longformer_bigbird's inputs with the global rows' tiles cut into
                      pieces of at most 34 blocks (plan option max_unit_blocks = 34)
  bigbird_two_heads   longformer_bigbird's pattern on B=1 H=H_kv=2: the global rows'
                      tile of each head is longer than a CTA's share of the launch
                      (the automatic split cuts it)
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch


@dataclass
class PrefillWorkload:
    name: str
    B: int
    H: int
    H_kv: int
    N: int
    d: int
    causal: int = 0
    window: int = 0
    n_global: int = 0
    block_local: int = 0
    block_q: int = 128
    block_k: int = 64
    random_block: int = 64
    n_random: int = 0
    bsfa: bool = False
    seed: int = 0
    dilation: int = 1
    skipped_in_denominator: int = 0   # block-skip variant (product pattern field)
    row_level_skip: int = 0           # block-skip rule, per-query reading (product pattern field)
    max_unit_blocks: int = 0          # plan option: split tiles (0 automatic)
    # "calibrated": per-head thresholds from the calibration draw; "minus_inf":
    # thresholds of -inf (the rule computes and keeps every block: the run the
    # rule's savings are measured against)
    thresholds: str = "calibrated"
    extra: dict = field(default_factory=dict)

    def pattern_fields(self):
        return dict(causal=self.causal, window=self.window, n_global=self.n_global,
                    block_local=self.block_local, block_q=self.block_q, block_k=self.block_k,
                    random_block=self.random_block, n_random=self.n_random,
                    dilation=self.dilation)


@dataclass
class GatherWorkload:
    name: str
    S: int
    H: int
    H_kv: int
    d: int
    L: int
    n_idx: int
    H_idx: int
    n_recent: int = 128
    seed: int = 0


@dataclass
class WindowDecodeWorkload:
    """Decode of a causal window + global tokens pattern over a cache of
    window + n_global slots; every query sits past the window (its set is the
    n_global globals and the last `window` keys)."""
    name: str
    S: int
    H: int
    H_kv: int
    d: int
    window: int
    n_global: int
    max_pos: int
    seed: int = 0


@dataclass
class TopkDecodeWorkload:
    """Decode queries attending to their top_k keys by relevance score."""
    name: str
    S: int
    H: int
    H_kv: int
    d: int
    L: int
    top_k: int
    seed: int = 0


WORKLOADS = {
    "tiny_static": PrefillWorkload("tiny_static", B=1, H=2, H_kv=2, N=256, d=64, causal=1,
                                   window=64, n_global=4, block_q=64, block_k=64, seed=1000),
    "mistral_swa": PrefillWorkload("mistral_swa", B=1, H=32, H_kv=8, N=8192, d=128, causal=1,
                                   window=4096, block_q=128, block_k=64, seed=2000),
    "bsfa_causal": PrefillWorkload("bsfa_causal", B=1, H=32, H_kv=8, N=32768, d=128, causal=1,
                                   block_q=128, block_k=64, bsfa=True, seed=3000),
    "longformer_bigbird": PrefillWorkload("longformer_bigbird", B=2, H=16, H_kv=16, N=65536, d=64,
                                          causal=0, window=512, n_global=64, random_block=64,
                                          n_random=3, block_q=128, block_k=64, seed=4000),
    "gather_decode": GatherWorkload("gather_decode", S=64, H=32, H_kv=8, d=128, L=131072,
                                    n_idx=2048, H_idx=32, seed=5000),
    "window_decode": WindowDecodeWorkload("window_decode", S=64, H=32, H_kv=8, d=128,
                                          window=4096, n_global=4, max_pos=131071, seed=6000),
    "topk_decode": TopkDecodeWorkload("topk_decode", S=64, H=32, H_kv=8, d=128, L=131072,
                                      top_k=2048, seed=8000),
    "bsfa_denominator": PrefillWorkload("bsfa_denominator", B=1, H=32, H_kv=8, N=32768, d=128,
                                        causal=1, block_q=128, block_k=64, bsfa=True,
                                        skipped_in_denominator=1, seed=3000),
    "bsfa_causal_noskip": PrefillWorkload("bsfa_causal_noskip", B=1, H=32, H_kv=8, N=32768,
                                          d=128, causal=1, block_q=128, block_k=64, bsfa=True,
                                          thresholds="minus_inf", seed=3000),
    "bsfa_row_level": PrefillWorkload("bsfa_row_level", B=1, H=32, H_kv=8, N=32768, d=128,
                                      causal=1, block_q=128, block_k=64, bsfa=True,
                                      row_level_skip=1, seed=3000),
    "dilated_swa": PrefillWorkload("dilated_swa", B=1, H=32, H_kv=8, N=32768, d=128, causal=1,
                                   window=2048, dilation=8, block_q=128, block_k=64, seed=7000),
    "longformer_split": PrefillWorkload("longformer_split", B=2, H=16, H_kv=16, N=65536, d=64,
                                        causal=0, window=512, n_global=64, random_block=64,
                                        n_random=3, block_q=128, block_k=64, max_unit_blocks=34,
                                        seed=4000),
    "bigbird_two_heads": PrefillWorkload("bigbird_two_heads", B=1, H=2, H_kv=2, N=65536, d=64,
                                         causal=0, window=512, n_global=64, random_block=64,
                                         n_random=3, block_q=128, block_k=64, seed=4000),
}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def randn_bf16(shape, seed: int, device="cpu", chunk_rows: int = 1 << 22) -> torch.Tensor:
    """N(0,1) float32 draws rounded to bf16, generated in chunks along dim 0."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    g = _gen(seed, device)
    flat = out.view(shape[0], -1)
    inner = flat.shape[1]
    step = max(1, chunk_rows // max(inner, 1) * 64)
    for s in range(0, shape[0], step):
        e = min(shape[0], s + step)
        flat[s:e] = torch.randn((e - s, inner), generator=g, device=device,
                                dtype=torch.float32).to(torch.bfloat16)
    return out


def random_table(H: int, N: int, random_block: int, n_random: int, seed: int) -> np.ndarray:
    """n_random distinct key blocks per (head, query block), uniform, ascending."""
    nrb = -(-N // random_block)
    n_random = min(n_random, nrb)
    g = _gen(seed, "cpu")
    keys = torch.rand((H, nrb, nrb), generator=g)
    tab = keys.argsort(dim=-1)[..., :n_random].sort(dim=-1).values
    return tab.to(torch.int32).numpy()


def prefill_inputs(w: PrefillWorkload, device="cpu", seed: Optional[int] = None):
    """(Q, K, V, random_table or None) for a prefill workload."""
    base = w.seed if seed is None else seed
    Q = randn_bf16((w.B, w.H, w.N, w.d), base, device)
    K = randn_bf16((w.B, w.H_kv, w.N, w.d), base + 1, device)
    V = randn_bf16((w.B, w.H_kv, w.N, w.d), base + 2, device)
    if w.bsfa:
        Q, K = _peaked(w, Q, K, base, device)
    tab = None
    if w.n_random > 0:
        tab = random_table(w.H, w.N, w.random_block, w.n_random, base + 4)
    return Q, K, V, tab


def _peaked(w: PrefillWorkload, Q, K, base: int, device):
    """K += 4 u_h on floor(0.02 N) marked positions; Q += 2 u_{h_kv(h)}."""
    g = _gen(base + 3, "cpu")
    u = torch.randn((w.H_kv, w.d), generator=g, dtype=torch.float32)
    u = u / u.norm(dim=-1, keepdim=True)
    n_mark = int(0.02 * w.N)
    group = w.H // w.H_kv
    Kf = K.float()
    for hk in range(w.H_kv):
        pos = torch.randperm(w.N, generator=g)[:n_mark].to(device)
        Kf[:, hk, pos] += 4.0 * u[hk].to(device)
    K = Kf.to(torch.bfloat16)
    del Kf
    for h in range(w.H):
        Qh = Q[:, h].float() + 2.0 * u[h // group].to(device)
        Q[:, h] = Qh.to(torch.bfloat16)
    return Q, K


def calibration_inputs(w: PrefillWorkload, device="cpu"):
    """The calibration draw: same recipe, seed base + 100."""
    return prefill_inputs(w, device=device, seed=w.seed + 100)


def topk_decode_inputs(w: TopkDecodeWorkload, device="cpu", seed: Optional[int] = None):
    """(Q [S][H][d], K, V [S][H_kv][L][d]) -- N(0,1) draws, every key valid."""
    base = w.seed if seed is None else seed
    Q = randn_bf16((w.S, w.H, w.d), base, device)
    K = randn_bf16((w.S, w.H_kv, w.L, w.d), base + 1, device)
    V = randn_bf16((w.S, w.H_kv, w.L, w.d), base + 2, device)
    return Q, K, V


def gather_inputs(w: GatherWorkload, device="cpu", seed: Optional[int] = None):
    """(Q [S][H][d], K, V [S][H_kv][L][d], idx int32 [S][H_idx][n_idx]) -- idx sorted unique."""
    base = w.seed if seed is None else seed
    Q = randn_bf16((w.S, w.H, w.d), base, device)
    K = randn_bf16((w.S, w.H_kv, w.L, w.d), base + 1, device)
    V = randn_bf16((w.S, w.H_kv, w.L, w.d), base + 2, device)
    idx = gather_index_sets(w.S, w.H_idx, w.L, w.n_idx, w.n_recent, base + 3, device)
    return Q, K, V, idx


def window_decode_inputs(w: WindowDecodeWorkload, device="cpu", seed: Optional[int] = None):
    """(Q [S][H][d], K, V [S][H_kv][window + n_global][d] cache, positions int32 [S])
    with positions uniform in [window + n_global, max_pos] (seeded)."""
    base = w.seed if seed is None else seed
    C = w.window + w.n_global
    Q = randn_bf16((w.S, w.H, w.d), base, device)
    K = randn_bf16((w.S, w.H_kv, C, w.d), base + 1, device)
    V = randn_bf16((w.S, w.H_kv, C, w.d), base + 2, device)
    g = _gen(base + 3, "cpu")
    pos = torch.randint(C, w.max_pos + 1, (w.S,), generator=g, dtype=torch.int64)
    return Q, K, V, pos.to(torch.int32).to(device)


def window_slots_in_key_order(p: int, window: int, n_global: int):
    """Cache slots of the index set of a query at position p, in ascending key
    order (globals, then the window), for a cache of window + n_global slots."""
    keys = np.concatenate([np.arange(min(n_global, p + 1)),
                           np.arange(max(n_global, p - window + 1), p + 1)])
    return np.where(keys < n_global, keys, n_global + keys % window).astype(np.int64)


def gather_index_sets(S: int, H_idx: int, L: int, n_idx: int, n_recent: int, seed: int,
                      device="cpu", chunk: int = 64) -> torch.Tensor:
    """{0} and {L-n_recent .. L-1} and (n_idx - n_recent - 1) distinct uniform draws
    from {1 .. L-n_recent-1}, sorted ascending, per (sequence, index head)."""
    n_recent = min(n_recent, L - 1)
    n_draw = n_idx - n_recent - 1
    pool = L - n_recent - 1
    assert 0 <= n_draw <= pool, "index set larger than the cache"
    g = _gen(seed, device)
    rows = S * H_idx
    out = torch.empty((rows, n_idx), dtype=torch.int32, device=device)
    fixed = torch.cat([torch.zeros(1, dtype=torch.int64, device=device),
                       torch.arange(L - n_recent, L, device=device)])
    for s in range(0, rows, chunk):
        e = min(rows, s + chunk)
        keys = torch.rand((e - s, pool), generator=g, device=device)
        draw = keys.topk(n_draw, dim=1).indices + 1 if n_draw > 0 else \
            torch.empty((e - s, 0), dtype=torch.int64, device=device)
        allv = torch.cat([fixed.expand(e - s, -1), draw], dim=1)
        out[s:e] = allv.sort(dim=1).values.to(torch.int32)
    return out.view(S, H_idx, n_idx)
