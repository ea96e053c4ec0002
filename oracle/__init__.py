"""Double-precision CPU oracle for sparse attention (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports, links or calls anything here, and this
package never imports the product package.

The arithmetic lives in ``sa_oracle.c`` (plain C, double precision, OpenMP over
independent rows).  This module compiles it with gcc, wraps it with ctypes and
adds two small steps written in Python:

* ``calibrate_thresholds`` -- the one-time per-head threshold calibration of
  Block Sparse Flash Attention ("Block Sparse Flash Attention", AI Radio
  episode, improvements: thresholds are learned once per layer and head from a
  small calibration set).  Read as: tau_h = the lower median (50th percentile,
  nearest rank) of the block statistics of head h's full blocks on a
  calibration draw.  ``numpy.sort`` is the library step.
* ``visible_py`` -- the membership predicate of G_i written a third time, in
  Python, for brute-force enumeration on tiny inputs.

Sources cited by the functions below are the web pages on sparse attention:
"Sparse Attention Weights Assumption" (1cademy), the "sparse attention
mechanism" glossary (chipfoundryservices), "SAS: Sparse Attention Synthesizer"
(kindchill) and "Block Sparse Flash Attention" (montaan AI Radio).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sa_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "libsa_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile sa_oracle.c into oracle/_build/libsa_oracle.so (gcc, OpenMP)."""
    os.makedirs(_BUILD, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99",
                           "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _Pattern(ctypes.Structure):
    _fields_ = [("causal", ctypes.c_int32), ("window", ctypes.c_int32),
                ("n_global", ctypes.c_int32), ("block_local", ctypes.c_int32),
                ("block_q", ctypes.c_int32), ("block_k", ctypes.c_int32),
                ("random_block", ctypes.c_int32), ("n_random", ctypes.c_int32),
                ("random_table", ctypes.c_void_p), ("dilation", ctypes.c_int32)]


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.POINTER(_Pattern)
        vp, i32, i64, dbl = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.ora_visible.argtypes = [P, i32, i32, i32, i32]
        lib.ora_visible.restype = i32
        lib.ora_build_G.argtypes = [P, i32, i32, i32, vp]
        lib.ora_build_G.restype = i32
        lib.ora_weighted_sum.argtypes = [i32, i32, vp, vp, vp, vp]
        lib.ora_tile_blocks.argtypes = [P, i32, i32, i32, i32, i32, i32, dbl, vp, vp,
                                        i32, i32, i32, vp, vp, vp, vp, vp, vp]
        lib.ora_prefill.argtypes = [P, i32, i32, i32, i32, i32, i32, dbl, vp, vp, vp,
                                    vp, vp, i32, i32, vp, vp, i64, vp, vp, vp, vp, vp, vp, i32]
        lib.ora_dense.argtypes = [i32, i32, i32, i32, i32, i32, dbl, i32, vp, vp, vp, vp]
        lib.ora_gather.argtypes = [i32, i32, i32, i32, i32, i32, i32, i32, dbl, vp, vp, vp,
                                   vp, vp, vp, vp, i32]
        lib.ora_topk_select.argtypes = [i32, i32, i32, i32, i32, i32, dbl, vp, vp, vp, i32,
                                        vp, vp, vp, vp, i32]
        _lib = lib
    return _lib


@dataclass
class Pattern:
    """Static pattern: G_i = causal-cap( window OR global OR block_local OR random ).

    Union of primitives by logical OR ("SAS", Step 5, component 2); primitives
    from the glossary's "Sparse Attention Patterns" table and the Mistral
    sliding-window rule.  No primitive on means every key (dense).
    """
    causal: int = 0
    window: int = 0
    n_global: int = 0
    block_local: int = 0
    block_q: int = 128
    block_k: int = 64
    random_block: int = 64
    n_random: int = 0
    random_table: Optional[np.ndarray] = None   # int32 [H][ceil(N/rb)][n_random]
    dilation: int = 1   # window taps k apart (glossary table, dilated/strided row)

    def _c(self):
        tab = None
        if self.random_table is not None and self.n_random > 0:
            tab = np.ascontiguousarray(self.random_table, dtype=np.int32)
        st = _Pattern(self.causal, self.window, self.n_global, self.block_local,
                      self.block_q, self.block_k, self.random_block,
                      self.n_random if tab is not None else 0,
                      tab.ctypes.data if tab is not None else None, self.dilation)
        return st, tab          # keep tab alive alongside the struct


def _as_input(x):
    """bf16 tensors/arrays -> (kind 0, uint16 bits); float64 -> (kind 1, array)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.bfloat16:
                return 0, x.view(torch.int16).numpy().view(np.uint16)
            return 1, x.to(torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        return 0, x
    return 1, np.ascontiguousarray(x, dtype=np.float64)


def _p(a):
    return None if a is None else a.ctypes.data


def default_scale(d: int) -> float:
    """1/sqrt(d_k), the scale of the glossary's standard attention formula."""
    return 1.0 / math.sqrt(d)


def visible(p: Pattern, N: int, h: int, i: int, j: int) -> bool:
    st, _tab = p._c()
    return bool(_load().ora_visible(ctypes.byref(st), N, h, i, j))


def build_G(p: Pattern, N: int, h: int, i: int) -> np.ndarray:
    """G_i as a sorted int32 array, built from index ranges."""
    st, _tab = p._c()
    out = np.empty(N, dtype=np.int32)
    n = _load().ora_build_G(ctypes.byref(st), N, h, i, out.ctypes.data)
    return out[:n].copy()


def visible_py(p: Pattern, N: int, h: int, i: int, j: int) -> bool:
    """The membership predicate once more, in Python, for brute force."""
    if not (0 <= i < N and 0 <= j < N):
        return False
    if p.causal and j > i:
        return False
    prims = []
    if p.window > 0:
        k = max(1, p.dilation)
        if (i - j) % k:
            prims.append(False)       # not one of the window's taps
        else:
            m = (i - j) // k
            prims.append((0 <= m < p.window) if p.causal else (abs(m) <= p.window // 2))
    if p.n_global > 0:
        prims.append(i < p.n_global or j < p.n_global)
    if p.block_local > 0:
        prims.append(i // p.block_local == j // p.block_local)
    if p.n_random > 0 and p.random_table is not None:
        prims.append(j // p.random_block in set(int(x) for x in p.random_table[h][i // p.random_block]))
    return any(prims) if prims else True


def weighted_sum(G: Sequence[int], alpha: Sequence[float], V: np.ndarray) -> np.ndarray:
    """out = sum_k alpha[k] * V[G[k]] -- the sparse attention output formula
    ("Sparse Attention Weights Assumption", 1cademy) given the weights."""
    V = np.ascontiguousarray(V, dtype=np.float64)
    G = np.ascontiguousarray(G, dtype=np.int32)
    a = np.ascontiguousarray(alpha, dtype=np.float64)
    out = np.empty(V.shape[1], dtype=np.float64)
    _load().ora_weighted_sum(len(G), V.shape[1], G.ctypes.data, a.ctypes.data,
                             V.ctypes.data, out.ctypes.data)
    return out


def tile_blocks(p: Pattern, Q, K, b: int, h: int, t: int, thresholds=None, scale=None,
                override=None):
    """Block-skip bookkeeping of one query tile: (cnt, full, stat, mask) per key block."""
    kq, q = _as_input(Q)
    kk, k = _as_input(K)
    assert kq == kk
    B, H, N, d = q.shape
    Hkv = k.shape[1]
    n_kb = -(-N // p.block_k)
    cnt = np.zeros(n_kb, np.int64)
    full = np.zeros(n_kb, np.uint8)
    stat = np.zeros(n_kb, np.float64)
    mask = np.zeros(n_kb, np.uint8)
    th = None if thresholds is None else np.ascontiguousarray(thresholds, np.float64)
    ov = None if override is None else np.ascontiguousarray(override, np.int8)
    st, _tab = p._c()
    _load().ora_tile_blocks(ctypes.byref(st), kq, B, H, Hkv, N, d,
                            default_scale(d) if scale is None else scale,
                            q.ctypes.data, k.ctypes.data, b, h, t, _p(th), _p(ov),
                            cnt.ctypes.data, full.ctypes.data, stat.ctypes.data, mask.ctypes.data)
    return cnt, full.astype(bool), stat, mask


def prefill(p: Pattern, Q, K, V, thresholds=None, scale=None, rows=None, override=None,
            keep_in_denominator=False, want_blocks=False, nthreads=0, row_level=False,
            row_override=None, want_row_stats=False):
    """Sparse attention prefill over static G_i, optionally with the block-skip rule.

    Q: [B][H][N][d]; K, V: [B][H_kv][N][d] (bf16 tensors or float64 arrays).
    rows: None (every row; returns O [B][H][N][d]) or int array [n][3] of
    (b, h, i) (returns O [n][d]).  Returns (O, lse) or, with want_blocks,
    (O, lse, mask, stat, full) with mask/stat/full shaped [B][H][T][n_kb] (only
    tiles that hold a requested row are filled).

    row_level: the per-query reading of the rule ("Block Sparse Flash
    Attention", paper summary): each row also drops the full blocks of its
    tile whose maximum over its own logits is below the threshold.
    row_override: int8 [n_rows][n_kb] (-1 rule, 0 keep, 1 drop) for the
    requested rows.  want_row_stats appends the rows' per-block maxima
    ([n_rows][n_kb], -inf for blocks that are not full) to the result.
    """
    kq, q = _as_input(Q)
    kk, k = _as_input(K)
    kv, v = _as_input(V)
    assert kq == kk == kv, "Q, K and V must share one input kind"
    B, H, N, d = q.shape
    Hkv = k.shape[1]
    assert H % Hkv == 0
    T = -(-N // p.block_q)
    n_kb = -(-N // p.block_k)
    r = None
    if rows is not None:
        r = np.ascontiguousarray(rows, dtype=np.int32).reshape(-1, 3)
        n = r.shape[0]
    else:
        n = B * H * N
    O = np.zeros((n, d), np.float64)
    lse = np.zeros(n, np.float64)
    if row_level and keep_in_denominator:
        raise ValueError("the row-level reading is not combined with keep_in_denominator")
    rov = None if row_override is None else np.ascontiguousarray(row_override, np.int8)
    if rov is not None:
        assert row_level and rov.shape == (n, n_kb), (rov.shape, (n, n_kb))
    rstat = np.full((n, n_kb), -np.inf) if want_row_stats else None
    th = None if thresholds is None else np.ascontiguousarray(thresholds, np.float64)
    ov = None if override is None else np.ascontiguousarray(override, np.int8)
    mask = stat = full = None
    if want_blocks:
        mask = np.zeros((B, H, T, n_kb), np.uint8)
        stat = np.full((B, H, T, n_kb), -np.inf, np.float64)
        full = np.zeros((B, H, T, n_kb), np.uint8)
    st, _tab = p._c()
    _load().ora_prefill(ctypes.byref(st), kq, B, H, Hkv, N, d,
                        default_scale(d) if scale is None else scale,
                        q.ctypes.data, k.ctypes.data, v.ctypes.data, _p(th), _p(ov),
                        1 if keep_in_denominator else 0, 1 if row_level else 0, _p(rov),
                        _p(rstat), n, _p(r), O.ctypes.data,
                        lse.ctypes.data, _p(mask), _p(stat), _p(full), nthreads)
    if rows is None:
        O = O.reshape(B, H, N, d)
        lse = lse.reshape(B, H, N)
    res = (O, lse)
    if want_blocks:
        res += (mask, stat, full.astype(bool))
    if want_row_stats:
        res += (rstat,)
    return res


def dense(Q, K, V, causal=False, scale=None):
    """softmax(Q K^T * scale) V in matrix form (the glossary's standard formula)."""
    kq, q = _as_input(Q)
    kk, k = _as_input(K)
    kv, v = _as_input(V)
    assert kq == kk == kv
    B, H, N, d = q.shape
    O = np.zeros((B, H, N, d), np.float64)
    _load().ora_dense(kq, B, H, k.shape[1], N, d, default_scale(d) if scale is None else scale,
                      1 if causal else 0, q.ctypes.data, k.ctypes.data, v.ctypes.data,
                      O.ctypes.data)
    return O


def gather(Q, K, V, idx, idx_len=None, scale=None, nthreads=0):
    """Attention of one query per (sequence, head) over explicit index sets.

    Q: [S][H][d]; K, V: [S][H_kv][L][d]; idx: int32 [S][H_idx][n_idx] sorted
    unique; idx_len: [S][H_idx] or None.  Returns (O [S][H][d], lse [S][H]).
    """
    kq, q = _as_input(Q)
    kk, k = _as_input(K)
    kv, v = _as_input(V)
    assert kq == kk == kv
    S, H, d = q.shape
    Hkv, L = k.shape[1], k.shape[2]
    ix = np.ascontiguousarray(idx, dtype=np.int32)
    H_idx, n_idx = ix.shape[1], ix.shape[2]
    il = None if idx_len is None else np.ascontiguousarray(idx_len, dtype=np.int32)
    O = np.zeros((S, H, d), np.float64)
    lse = np.zeros((S, H), np.float64)
    _load().ora_gather(kq, S, H, Hkv, H_idx, L, d, n_idx, default_scale(d) if scale is None else scale,
                       q.ctypes.data, k.ctypes.data, v.ctypes.data, ix.ctypes.data, _p(il),
                       O.ctypes.data, lse.ctypes.data, nthreads)
    return O, lse


def topk_select(Q, K, top_k, lengths=None, scale=None, nthreads=0):
    """Dynamic top-K sets of decode queries ("SAS", component 1, primitive C).

    Q: [S][H][d]; K: [S][H_kv][L][d]; lengths: int [S] keys per sequence (or
    None = L).  G of query (s, h) = the min(top_k, len_s) keys j < len_s with the
    largest scale * q . k_j, ties to the smaller j.  Returns (idx int32
    [S][H][top_k] ascending within the first idx_len entries, idx_len int32
    [S][H], kth [S][H] smallest selected score, nxt [S][H] largest unselected
    score; NaN where there is none).  Feed (idx, idx_len) to gather() for the
    output.
    """
    kq, q = _as_input(Q)
    kk, k = _as_input(K)
    assert kq == kk
    S, H, d = q.shape
    Hkv, L = k.shape[1], k.shape[2]
    ln = None if lengths is None else np.ascontiguousarray(lengths, dtype=np.int32)
    idx = np.zeros((S, H, max(int(top_k), 1)), np.int32)
    idx_len = np.zeros((S, H), np.int32)
    kth = np.zeros((S, H), np.float64)
    nxt = np.zeros((S, H), np.float64)
    _load().ora_topk_select(kq, S, H, Hkv, L, d, default_scale(d) if scale is None else scale,
                            q.ctypes.data, k.ctypes.data, _p(ln), int(top_k), idx.ctypes.data,
                            idx_len.ctypes.data, kth.ctypes.data, nxt.ctypes.data, nthreads)
    return idx[:, :, :top_k], idx_len, kth, nxt


def block_stats(p: Pattern, Q, K, scale=None, tiles=None, nthreads=0):
    """(full, stat) per (b, h, tile, key block) with no threshold applied.

    The rule's statistics need only the tile's scores, so one row per tile is
    requested (its output is discarded).  tiles: None (all) or [n][3] (b, h, t)."""
    kq, q = _as_input(Q)
    B, H, N, d = q.shape
    T = -(-N // p.block_q)
    if tiles is None:
        tiles = np.array([(b, h, t) for b in range(B) for h in range(H) for t in range(T)],
                         dtype=np.int32).reshape(-1, 3)
    tiles = np.asarray(tiles, dtype=np.int32).reshape(-1, 3)
    rows = tiles.copy()
    rows[:, 2] = tiles[:, 2] * p.block_q
    V = K
    _, _, mask, stat, full = prefill(p, Q, K, V, scale=scale, rows=rows, want_blocks=True,
                                     nthreads=nthreads)
    return full, stat, mask


def calibrate_thresholds(full: np.ndarray, stat: np.ndarray) -> np.ndarray:
    """tau_h = lower median (nearest rank) of head h's full-block statistics.

    full, stat: [B][H][T][n_kb].  Returns float64 [H]."""
    H = full.shape[1]
    tau = np.empty(H, np.float64)
    for h in range(H):
        s = np.sort(stat[:, h][full[:, h]])
        tau[h] = s[(len(s) - 1) // 2] if len(s) else -np.inf
    return tau
