"""Block-sparse attention for NVIDIA B200 (sm_100a): Python binding of the C ABI.

The functions here only marshal arguments (torch tensors -> device pointers,
the current CUDA stream) and call libsparse_attn.so; every step of the
computation runs in the library's CUDA kernels.  PyTorch supplies device
memory and streams.

Entry points mirror include/sparse_attn.h:

* ``Plan`` -- sparse_attn_plan_create / _info / _destroy, ``Plan.prefill``
  (sparse_attn_prefill_plan), ``Plan.block_stats`` (sparse_attn_block_stats),
  ``Plan.calibrate`` (sparse_attn_calibrate).
* ``sparse_attn_prefill`` -- one-shot prefill through the library's plan cache;
  ``sparse_attn_prefill_noalloc`` -- the same without device allocation.
* ``sparse_attn_gather`` -- explicit index sets over a KV cache.
* ``sparse_attn_decode_window`` / ``window_slot`` -- decode of a causal window +
  global tokens pattern over a cache of window + globals slots.
* ``sparse_attn_decode_topk`` / ``decode_topk_workspace_bytes`` -- decode over
  each query's top_k keys by relevance score.
* ``compile_pattern`` -- the host pattern compiler (no GPU needed).
* ``check_device_error`` -- reads and clears the device error word.

Example (a causal sliding window of 4096 with GQA, then the block-skip rule
with thresholds calibrated on a calibration draw)::

    import block_sparse_attention_29_b200 as sa
    pat = sa.Pattern(causal=1, window=4096)            # block_q=128, block_k=64
    plan = sa.Plan(pat, B, H, H_kv, N, d)              # compiled once, reusable
    O = plan.prefill(Q, K, V)                          # bf16 [B][H][N][d]
    rule = sa.Plan(sa.Pattern(causal=1), B, H, H_kv, N, d)
    tau = rule.calibrate(rule.block_stats(Qc, Kc), 0.5)   # per-head thresholds
    O = rule.prefill(Q, K, V, thresholds=tau)
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass
from typing import Optional

import numpy as np

from ._lib import (EXPORTS, LIB_PATH, SA_ERR_DEVICE_INDEX, SA_ERR_INVALID_ARG, SA_ERR_TIMEOUT,
                   SA_ERR_UNSUPPORTED, SA_OK, SaPattern, SaPlanInfo, SaPlanOptions, SparseAttnError,
                   check, lib)

__all__ = ["Pattern", "Plan", "KERNEL_AUTO", "KERNEL_SINGLE_HEAD",
           "sparse_attn_prefill", "sparse_attn_prefill_noalloc",
           "sparse_attn_gather", "sparse_attn_decode_window", "window_slot",
           "sparse_attn_decode_topk", "decode_topk_workspace_bytes", "compile_pattern",
           "check_device_error", "SparseAttnError", "EXPORTS", "LIB_PATH", "SA_OK",
           "SA_ERR_INVALID_ARG", "SA_ERR_UNSUPPORTED", "SA_ERR_TIMEOUT", "SA_ERR_DEVICE_INDEX"]


@dataclass
class Pattern:
    """Static pattern descriptor (sa_pattern_t); see include/sparse_attn.h."""
    causal: int = 0
    window: int = 0
    n_global: int = 0
    block_local: int = 0
    block_q: int = 128
    block_k: int = 64
    random_block: int = 64
    n_random: int = 0
    random_table: Optional[np.ndarray] = None   # host int32 [H][ceil(N/rb)][n_random]
    scale: float = 0.0
    dilation: int = 1   # window taps this far apart (dilated/strided window); 1 = contiguous
    skipped_in_denominator: int = 0   # block-skip variant: skipped keys stay in the denominator
    row_level_skip: int = 0   # block-skip rule, per-query reading: rows drop full blocks by their own max

    def to_c(self, thresholds_ptr: int = 0):
        tab = None
        if self.random_table is not None and self.n_random > 0:
            tab = np.ascontiguousarray(np.asarray(self.random_table), dtype=np.int32)
        st = SaPattern(self.causal, self.window, self.n_global, self.block_local, self.block_q,
                       self.block_k, self.random_block, self.n_random if tab is not None else 0,
                       tab.ctypes.data if tab is not None else None,
                       thresholds_ptr or None, self.scale, self.dilation,
                       self.skipped_in_denominator, self.row_level_skip)
        return st, tab   # the caller keeps `tab` alive while the struct is used


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream or None


def _check_tensor(name, t, shape, dtype):
    import torch
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    # the library launches on the current device: a tensor of another device
    # would hand its kernels a pointer into that device's memory
    cur = torch.cuda.current_device()
    if t.device.index != cur:
        raise ValueError(f"{name} is on cuda:{t.device.index}, the current device is cuda:{cur}")


def _tiles(N: int):
    """(T_q, n_kb) of the block-mask and block-statistics layouts: 128-row query
    tiles and 64-key blocks."""
    return (N + 127) // 128, (N + 63) // 64


KERNEL_AUTO = 0            # the kernel measured fastest for the shape (single-head today)
KERNEL_SINGLE_HEAD = 1     # the single-head kernel


class Plan:
    """A compiled pattern for Q [B][H][N][d], K/V [B][H_kv][N][d].

    ``kernel``: KERNEL_AUTO or KERNEL_SINGLE_HEAD; ``max_unit_blocks``: 0 splits a
    tile whose list exceeds one CTA's share of the launch, > 0 cuts every block
    list longer than that into pieces, < 0 splits nothing
    (sparse_attn_plan_create_opts)."""

    def __init__(self, pattern: Pattern, B: int, H: int, H_kv: int, N: int, d: int,
                 kernel: int = KERNEL_AUTO, max_unit_blocks: int = 0):
        self.pattern, self.B, self.H, self.H_kv, self.N, self.d = pattern, B, H, H_kv, N, d
        st, _tab = pattern.to_c()
        h = ctypes.c_void_p()
        opts = SaPlanOptions(kernel, max_unit_blocks)
        check(lib().sparse_attn_plan_create_opts(ctypes.byref(st), B, H, H_kv, N, d,
                                                 ctypes.byref(opts), ctypes.byref(h)))
        self._h = h
        info = SaPlanInfo()
        check(lib().sparse_attn_plan_info(self._h, ctypes.byref(info)))
        self.info = {k: getattr(info, k) for k, _ in SaPlanInfo._fields_}
        self.T = info.T_q
        self.n_kb = info.n_kb

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            lib().sparse_attn_plan_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def prefill(self, Q, K, V, O=None, thresholds=None, lse=None, block_mask=None,
                block_stat=None, stream=None):
        """Launches the prefill; returns O.  Optional outputs are written into
        the tensors given (lse float32 [B][H][N], block_mask uint8 and
        block_stat float32 [B][H][T][n_kb])."""
        import torch
        B, H, Hkv, N, d = self.B, self.H, self.H_kv, self.N, self.d
        _check_tensor("Q", Q, (B, H, N, d), torch.bfloat16)
        _check_tensor("K", K, (B, Hkv, N, d), torch.bfloat16)
        _check_tensor("V", V, (B, Hkv, N, d), torch.bfloat16)
        if O is None:
            O = torch.empty_like(Q)
        _check_tensor("O", O, (B, H, N, d), torch.bfloat16)
        if thresholds is not None:
            _check_tensor("thresholds", thresholds, (H,), torch.float32)
        if lse is not None:
            _check_tensor("lse", lse, (B, H, N), torch.float32)
        if block_mask is not None:
            _check_tensor("block_mask", block_mask, (B, H, self.T, self.n_kb), torch.uint8)
        if block_stat is not None:
            _check_tensor("block_stat", block_stat, (B, H, self.T, self.n_kb), torch.float32)
        check(lib().sparse_attn_prefill_plan(self._h, _ptr(Q), _ptr(K), _ptr(V), _ptr(O),
                                             _ptr(thresholds), _ptr(lse), _ptr(block_mask),
                                             _ptr(block_stat), _stream(stream)))
        return O

    def block_stats(self, Q, K, block_stat=None, block_mask=None, stream=None):
        """Statistics pass of the block-skip rule; returns block_stat."""
        import torch
        _check_tensor("Q", Q, (self.B, self.H, self.N, self.d), torch.bfloat16)
        _check_tensor("K", K, (self.B, self.H_kv, self.N, self.d), torch.bfloat16)
        if block_stat is None:
            block_stat = torch.full((self.B, self.H, self.T, self.n_kb), float("-inf"),
                                    dtype=torch.float32, device=Q.device)
        _check_tensor("block_stat", block_stat, (self.B, self.H, self.T, self.n_kb), torch.float32)
        if block_mask is not None:
            _check_tensor("block_mask", block_mask, (self.B, self.H, self.T, self.n_kb), torch.uint8)
        check(lib().sparse_attn_block_stats(self._h, _ptr(Q), _ptr(K), _ptr(block_stat),
                                            _ptr(block_mask), _stream(stream)))
        return block_stat

    def calibrate(self, block_stat, q: float = 0.5, out=None, stream=None):
        """Per-head thresholds (rank floor((n-1) q) of full-block statistics)."""
        import torch
        _check_tensor("block_stat", block_stat, (self.B, self.H, self.T, self.n_kb), torch.float32)
        if out is None:
            out = torch.empty(self.H, dtype=torch.float32, device=block_stat.device)
        _check_tensor("out", out, (self.H,), torch.float32)
        check(lib().sparse_attn_calibrate(self._h, _ptr(block_stat), float(q), _ptr(out),
                                          _stream(stream)))
        return out


def sparse_attn_prefill(Q, K, V, pattern: Pattern, thresholds=None, O=None, lse=None,
                        block_mask=None, stream=None):
    """One-shot prefill (plans are compiled once and cached by the library)."""
    import torch
    B, H, N, d = Q.shape
    Hkv = K.shape[1]
    _check_tensor("Q", Q, (B, H, N, d), torch.bfloat16)
    _check_tensor("K", K, (B, Hkv, N, d), torch.bfloat16)
    _check_tensor("V", V, (B, Hkv, N, d), torch.bfloat16)
    if O is None:
        O = torch.empty_like(Q)
    _check_tensor("O", O, (B, H, N, d), torch.bfloat16)
    if thresholds is not None:
        _check_tensor("thresholds", thresholds, (H,), torch.float32)
    if lse is not None:
        _check_tensor("lse", lse, (B, H, N), torch.float32)
    if block_mask is not None:
        _check_tensor("block_mask", block_mask, (B, H) + _tiles(N), torch.uint8)
    st, _tab = pattern.to_c(_ptr(thresholds) or 0)
    check(lib().sparse_attn_prefill(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), B, H, Hkv, N, d,
                                    ctypes.byref(st), _ptr(lse), _ptr(block_mask),
                                    _stream(stream)))
    return O


def sparse_attn_prefill_noalloc(Q, K, V, pattern: Pattern, O, thresholds=None, lse=None,
                                stream=None):
    """Prefill through the entry point that allocates no device memory: for
    callers that cannot call cudaMalloc at run time (external pools or
    allocation-free inference runtimes).  The caller supplies O (and lse);
    the library copies the compiled pattern into its fixed 8 MiB static device
    array.  Calls that may overlap on the GPU share that array and race."""
    import torch
    B, H, N, d = Q.shape
    Hkv = K.shape[1]
    _check_tensor("Q", Q, (B, H, N, d), torch.bfloat16)
    _check_tensor("K", K, (B, Hkv, N, d), torch.bfloat16)
    _check_tensor("V", V, (B, Hkv, N, d), torch.bfloat16)
    _check_tensor("O", O, (B, H, N, d), torch.bfloat16)
    if thresholds is not None:
        _check_tensor("thresholds", thresholds, (H,), torch.float32)
    if lse is not None:
        _check_tensor("lse", lse, (B, H, N), torch.float32)
    st, _tab = pattern.to_c(_ptr(thresholds) or 0)
    check(lib().sparse_attn_prefill_noalloc(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), B, H, Hkv, N, d,
                                            ctypes.byref(st), _ptr(lse), _stream(stream)))
    return O


def sparse_attn_gather(Q, K, V, idx, idx_len=None, O=None, scale: float = 0.0, lse=None,
                       stream=None):
    """Q [S][H][d], K/V [S][H_kv][L][d], idx int32 [S][H_idx][n_idx] -> O [S][H][d]."""
    import torch
    S, H, d = Q.shape
    Hkv, L = K.shape[1], K.shape[2]
    H_idx, n_idx = idx.shape[1], idx.shape[2]
    _check_tensor("Q", Q, (S, H, d), torch.bfloat16)
    _check_tensor("K", K, (S, Hkv, L, d), torch.bfloat16)
    _check_tensor("V", V, (S, Hkv, L, d), torch.bfloat16)
    _check_tensor("idx", idx, (S, H_idx, n_idx), torch.int32)
    if idx_len is not None:
        _check_tensor("idx_len", idx_len, (S, H_idx), torch.int32)
    if O is None:
        O = torch.empty_like(Q)
    _check_tensor("O", O, (S, H, d), torch.bfloat16)
    if lse is not None:
        _check_tensor("lse", lse, (S, H), torch.float32)
    check(lib().sparse_attn_gather(_ptr(Q), _ptr(K), _ptr(V), _ptr(idx), _ptr(idx_len), _ptr(O),
                                   S, H, Hkv, H_idx, L, n_idx, d, float(scale), _ptr(lse),
                                   _stream(stream)))
    return O


def sparse_attn_decode_window(Q, K, V, positions, pattern: Pattern, O=None, lse=None,
                              stream=None):
    """Decode over a minimum-size cache for a causal window + global tokens pattern.

    Q [S][H][d]; K/V [S][H_kv][C][d] with C = window + n_global slots (key j in
    slot window_slot(j, window, n_global)); positions int32 [S] -> O [S][H][d]."""
    import torch
    S, H, d = Q.shape
    Hkv, C = K.shape[1], K.shape[2]
    if C != pattern.window + pattern.n_global:
        raise ValueError(f"cache has {C} slots, the pattern needs window + n_global = "
                         f"{pattern.window + pattern.n_global}")
    _check_tensor("Q", Q, (S, H, d), torch.bfloat16)
    _check_tensor("K", K, (S, Hkv, C, d), torch.bfloat16)
    _check_tensor("V", V, (S, Hkv, C, d), torch.bfloat16)
    _check_tensor("positions", positions, (S,), torch.int32)
    if O is None:
        O = torch.empty_like(Q)
    _check_tensor("O", O, (S, H, d), torch.bfloat16)
    if lse is not None:
        _check_tensor("lse", lse, (S, H), torch.float32)
    st, _tab = pattern.to_c()
    check(lib().sparse_attn_decode_window(_ptr(Q), _ptr(K), _ptr(V), _ptr(positions), _ptr(O), S,
                                          H, Hkv, d, ctypes.byref(st), _ptr(lse), _stream(stream)))
    return O


def decode_topk_workspace_bytes(S: int, H: int, L: int, top_k: int) -> int:
    """Workspace bytes sparse_attn_decode_topk needs for these sizes."""
    return int(lib().sparse_attn_decode_topk_workspace(int(S), int(H), int(L), int(top_k)))


def sparse_attn_decode_topk(Q, K, V, top_k: int, lengths=None, O=None, lse=None, idx=None,
                            idx_len=None, scale: float = 0.0, workspace=None, stream=None):
    """Decode attention over each query's top_k keys by relevance score.

    Q [S][H][d]; K/V [S][H_kv][L][d]; lengths int32 [S] (keys per sequence) or
    None.  Returns (O [S][H][d], idx int32 [S][H][top_k], idx_len int32 [S][H]):
    the selected keys of (s, h) are idx[s, h, :idx_len[s, h]], ascending.
    workspace: a uint8 device tensor of decode_topk_workspace_bytes(...) bytes
    (allocated here when None)."""
    import torch
    S, H, d = Q.shape
    Hkv, L = K.shape[1], K.shape[2]
    _check_tensor("Q", Q, (S, H, d), torch.bfloat16)
    _check_tensor("K", K, (S, Hkv, L, d), torch.bfloat16)
    _check_tensor("V", V, (S, Hkv, L, d), torch.bfloat16)
    if lengths is not None:
        _check_tensor("lengths", lengths, (S,), torch.int32)
    if O is None:
        O = torch.empty_like(Q)
    _check_tensor("O", O, (S, H, d), torch.bfloat16)
    if lse is not None:
        _check_tensor("lse", lse, (S, H), torch.float32)
    if idx is None:
        idx = torch.zeros((S, H, top_k), dtype=torch.int32, device=Q.device)
    _check_tensor("idx", idx, (S, H, top_k), torch.int32)
    if idx_len is None:
        idx_len = torch.zeros((S, H), dtype=torch.int32, device=Q.device)
    _check_tensor("idx_len", idx_len, (S, H), torch.int32)
    need = decode_topk_workspace_bytes(S, H, L, top_k)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=Q.device)
    check(lib().sparse_attn_decode_topk(_ptr(Q), _ptr(K), _ptr(V), _ptr(lengths), _ptr(O), S, H,
                                        Hkv, L, d, int(top_k), float(scale), _ptr(idx),
                                        _ptr(idx_len), _ptr(lse), _ptr(workspace),
                                        workspace.numel() * workspace.element_size(),
                                        _stream(stream)))
    return O, idx, idx_len


def window_slot(j: int, window: int, n_global: int) -> int:
    """Cache slot of key j in the layout of sparse_attn_decode_window (-1 if invalid)."""
    return int(lib().sparse_attn_window_slot(int(j), int(window), int(n_global)))


def compile_pattern(pattern: Pattern, H: int, N: int, tile_q: int = 128, tile_k: int = 64):
    """Host pattern compiler: (row_ptr [H_pat*T+1], kb, full, cnt) as numpy arrays."""
    st, _tab = pattern.to_c()
    hp, T, n = ctypes.c_int(), ctypes.c_int(), ctypes.c_int64()
    L = lib()
    check(L.sparse_attn_compile_pattern(ctypes.byref(st), H, N, tile_q, tile_k, ctypes.byref(hp),
                                        ctypes.byref(T), ctypes.byref(n), None, None, None, None))
    row_ptr = np.zeros(hp.value * T.value + 1, np.int32)
    kb = np.zeros(max(n.value, 1), np.int32)
    full = np.zeros(max(n.value, 1), np.uint8)
    cnt = np.zeros(max(n.value, 1), np.int64)
    check(L.sparse_attn_compile_pattern(ctypes.byref(st), H, N, tile_q, tile_k, ctypes.byref(hp),
                                        ctypes.byref(T), ctypes.byref(n), row_ptr.ctypes.data,
                                        kb.ctypes.data, full.ctypes.data, cnt.ctypes.data))
    n = n.value
    return row_ptr, kb[:n], full[:n].astype(bool), cnt[:n], hp.value, T.value


def work_order(pattern: Pattern, B: int, H: int, H_kv: int, N: int, d: int,
               max_unit_blocks: int = 0):
    """Host work order of a plan's prefill queue: (units, pieces [n][4], split [n][4])
    as numpy int32 arrays (sparse_attn_work_order)."""
    st, _tab = pattern.to_c()
    nu, npc, ns = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    L = lib()
    check(L.sparse_attn_work_order(ctypes.byref(st), B, H, H_kv, N, d, max_unit_blocks,
                                   ctypes.byref(nu), ctypes.byref(npc), ctypes.byref(ns),
                                   None, None, None))
    units = np.zeros(max(nu.value, 1), np.int32)
    pieces = np.zeros((max(npc.value, 1), 4), np.int32)
    split = np.zeros((max(ns.value, 1), 4), np.int32)
    check(L.sparse_attn_work_order(ctypes.byref(st), B, H, H_kv, N, d, max_unit_blocks,
                                   ctypes.byref(nu), ctypes.byref(npc), ctypes.byref(ns),
                                   units.ctypes.data, pieces.ctypes.data, split.ctypes.data))
    return units[:nu.value], pieces[:npc.value], split[:ns.value]


def check_device_error(stream=None) -> None:
    """Synchronises `stream` and raises SparseAttnError if a kernel recorded an error."""
    check(lib().sparse_attn_check_device_error(_stream(stream)))
