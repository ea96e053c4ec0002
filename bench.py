#!/usr/bin/env python
"""Benchmark of the block-sparse attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
                    [--no-secondary]

The headline workload (the default) is bsfa_causal: causal prefill at N=32768
with the Block-Sparse-FlashAttention rule.  The same run then times every other
workload of the metric (mistral_swa, longformer_bigbird, gather_decode,
tiny_static) and the extensions (bsfa_denominator, dilated_swa, window_decode,
topk_decode), each with its own roofline, clocks and traffic, under
secondary.workloads of the JSON line (--no-secondary skips them).

One step = one pass of the hot path over one batch of synthetic input: for a
prefill workload one sparse_attn_prefill_plan launch (pattern compile and, for
the block-skip workload, the one-time threshold calibration happen before the
timed region); for gather_decode one sparse_attn_gather launch; for
window_decode one sparse_attn_decode_window launch; for topk_decode one
sparse_attn_decode_topk call (score, select and attend kernels).

Timing: W untimed warm-up steps, then exactly K steps bracketed by a barrier
and torch.cuda.synchronize() on both sides.  L2 is flushed (256 MiB write)
before every step, outside the timed kernel window; each step's kernel is
timed with CUDA events recorded on the stream it is launched on.  Multi-GPU
(torchrun): every rank runs an independent replica (the path has no exchange
step), the time is the max over ranks and `value` aggregates all ranks.

The printed JSON line carries the headline metric, an end-to-end number
through the same C-ABI call with host (pinned) buffers and the host<->device
copies inside the timed region, the roofline of the dominant kernel against
the measured peaks, SM clocks sampled during the timed region and the CPU
baseline (the fp64 oracle on a bounded sample, rank 0, N=1 only; for the
block-skip workloads the oracle uses thresholds it calibrates itself on a
sample of the calibration draw).

--impl reference times the fp64 CPU oracle as it stands on the host cores, on
the same workload and metric (bounded samples per step), and prints the same
JSON line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20
NEAR_BAND = 1e-3   # block statistics this close to the threshold may be decided either way


# ------------------------------------------------------------------ helpers --
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_sha(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "block_sparse_attention_29_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload, sha):
    """DRAM bytes per launch from a committed ncu summary, if the kernel source
    has not changed since it was captured."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)
        e = t[kernel][workload]
        if e.get("source_sha") == sha:
            return e["dram_bytes_per_launch"]
    except (OSError, ValueError, KeyError):
        pass
    return None


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled through NVML every
    ~2 ms on a thread while the timed region runs (read-only queries)."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown"}

    def __init__(self, cuda_index: int):
        self.cuda_index, self.samples, self.reason_bits = cuda_index, [], 0
        self.max_mhz, self.handle, self._stop = None, None, threading.Event()

    def __enter__(self):
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            pr = torch.cuda.get_device_properties(self.cuda_index)
            bus = f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
            self.handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
            self.nvml = pynvml
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
        except Exception as e:  # NVML unavailable: the line says so
            self.error = repr(e)
            self.handle = None
        return self

    def _sample(self):
        n = self.nvml
        self.samples.append(n.nvmlDeviceGetClockInfo(self.handle, n.NVML_CLOCK_SM))
        get = getattr(n, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            n.nvmlDeviceGetCurrentClocksThrottleReasons
        self.reason_bits |= int(get(self.handle))

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                return
            time.sleep(0.002)

    def __exit__(self, *a):
        if self.handle is not None:
            self._stop.set()
            self.thread.join(timeout=2)
            try:
                self._sample()
            except Exception:
                pass

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"],
                    "samples": 0, "error": getattr(self, "error", None)}
        reasons = sorted(v for k, v in self.REASONS.items() if self.reason_bits & k)
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples), "source": "nvml"}


# ------------------------------------------------------------ multi-rank --
def max_over_ranks(x: float, dist=None, device=None) -> float:
    """The largest value of x over all ranks (x itself without a process group)."""
    if dist is None:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(world: int, work_per_rank: float, seconds: float, scale: float) -> float:
    """Whole-job throughput of `world` independent replicas that each did
    `work_per_rank` units of work, timed by the slowest rank (max over ranks)."""
    return world * work_per_rank / seconds / scale


# ---------------------------------------------------------------- workloads --
def prefill_accounting(w, info, kept_desc=None, skipped_pairs=0):
    """FLOPs of one prefill launch: computed-block (descriptor granularity),
    exact-pair and dense-equivalent."""
    bq, bk, d = w.block_q, w.block_k, w.d
    blocks = info["blocks_desc"]
    kept = blocks if kept_desc is None else kept_desc
    computed = 2 * bq * bk * d * (blocks + kept)
    pairs = info["pairs"]
    exact = 2 * d * pairs + 2 * d * (pairs - skipped_pairs)
    p_dense = w.N * (w.N + 1) // 2 if w.causal else w.N * w.N
    dense = 4 * w.B * w.H * d * p_dense
    return computed, exact, dense


def setup_prefill(w, device, torch, sa, workloads):
    Q, K, V, tab = workloads.prefill_inputs(w, device=device)
    pat = sa.Pattern(**w.pattern_fields(), random_table=tab,
                     skipped_in_denominator=w.skipped_in_denominator,
                     row_level_skip=w.row_level_skip)
    plan = sa.Plan(pat, w.B, w.H, w.H_kv, w.N, w.d, max_unit_blocks=w.max_unit_blocks)
    thresholds = None
    extra = {"plan_compile_ms": round(plan.info["compile_ms"], 2)}
    if plan.info["split_tiles"]:
        # tiles cut into pieces (merged inside the same launch)
        extra["split_tiles"] = plan.info["split_tiles"]
        extra["queue_units"] = plan.info["queue_units"]
    kept_desc, skipped_pairs = None, 0
    if w.bsfa and w.thresholds == "minus_inf":
        thresholds = torch.full((w.H,), float("-inf"), dtype=torch.float32, device=device)
    elif w.bsfa:
        Qc, Kc, _, _ = workloads.calibration_inputs(w, device=device)
        # the statistics pass is the same for the rule's variants (they change
        # what a skipped or dropped block contributes, not the block decision)
        thresholds = plan.calibrate(plan.block_stats(Qc, Kc), 0.5)
        del Qc, Kc
    if w.bsfa:
        mask = torch.empty((w.B, w.H, plan.T, plan.n_kb), dtype=torch.uint8, device=device)
        stat = torch.empty((w.B, w.H, plan.T, plan.n_kb), dtype=torch.float32, device=device)
        plan.prefill(Q, K, V, thresholds=thresholds, block_mask=mask, block_stat=stat)
        sa.check_device_error()
        skipped = int((mask == 2).sum())
        # blocks whose statistic lies within NEAR_BAND of their head's threshold: the
        # ones a CPU recomputation in another precision may decide the other way
        # (the parity tests compare whole heads with the oracle outside this band)
        row_ptr, kb, fl, _, H_pat, T = sa.compile_pattern(pat, w.H, w.N)
        full = torch.zeros((H_pat, T, plan.n_kb), dtype=torch.bool)
        for hp in range(H_pat):
            for t in range(T):
                a, e = row_ptr[hp * T + t], row_ptr[hp * T + t + 1]
                full[hp, t, torch.from_numpy(kb[a:e][fl[a:e]]).long()] = True
        full = full.to(device).unsqueeze(0).expand(w.B, w.H if H_pat == 1 else -1, -1, -1)
        near = (stat - thresholds.view(1, -1, 1, 1)).abs() <= NEAR_BAND
        extra["near_threshold_blocks"] = int((near & full).sum())
        del stat, near, full
        kept_desc = plan.info["blocks_desc"] - skipped
        skipped_pairs = skipped * w.block_q * w.block_k
        extra["blocks_skipped"] = skipped
        extra["skip_fraction_of_full"] = round(skipped / max(1, plan.info["blocks_full"]), 4)
        extra["v_loads_issued_fraction"] = round(kept_desc / plan.info["blocks_desc"], 4)
        del mask
    computed, exact, dense = prefill_accounting(w, plan.info, kept_desc, skipped_pairs)
    extra.update({"blocks_listed": plan.info["blocks_desc"], "pairs": plan.info["pairs"]})
    O = torch.empty_like(Q)

    def step(stream=None):
        plan.prefill(Q, K, V, O=O, thresholds=thresholds, stream=stream)

    def e2e_step(host, dev_bufs, stream):
        Qd, Kd, Vd, Od = dev_bufs
        Qd.copy_(host[0], non_blocking=True)
        Kd.copy_(host[1], non_blocking=True)
        Vd.copy_(host[2], non_blocking=True)
        plan.prefill(Qd, Kd, Vd, O=Od, thresholds=thresholds, stream=stream)
        host[3].copy_(Od, non_blocking=True)

    host = [Q.cpu().pin_memory(), K.cpu().pin_memory(), V.cpu().pin_memory(),
            torch.empty(Q.shape, dtype=Q.dtype, pin_memory=True)]
    dev_bufs = [torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V), torch.empty_like(O)]
    h2d = sum(t.numel() * t.element_size() for t in host[:3])
    d2h = host[3].numel() * host[3].element_size()
    algo_bytes = sum(t.numel() * t.element_size() for t in (Q, K, V, O))
    # the same calls over a stream of steps (pipelined_e2e): two device buffer sets,
    # allocated only when the headline's end-to-end run asks for them
    def e2e_pipe():
        return dict(
            host_in=host[:3],
            host_out=[host[3], torch.empty(Q.shape, dtype=Q.dtype, pin_memory=True)],
            dev_sets=[dev_bufs, [torch.empty_like(t) for t in dev_bufs]],
            launch=lambda d, s: plan.prefill(d[0], d[1], d[2], O=d[3], thresholds=thresholds,
                                             stream=s),
            result_dev=O)
    return dict(step=step, e2e_step=lambda s: e2e_step(host, dev_bufs, s), e2e_pipe=e2e_pipe,
                h2d=h2d, d2h=d2h,
                flops=computed, exact_flops=exact, dense_flops=dense, algo_bytes=algo_bytes,
                extra=extra, kernel="prefill_kernel",
                launches_per_step=1,  # split tiles are merged inside the same launch
                kernel_files=["prefill_sm100.cu", "softmax_util.cuh", "ptx.cuh", "common.h",
                              "pattern_compiler.cu"],
                metric="effective TFLOP/s (computed blocks)", unit="TFLOP/s", bound="tensor",
                tensors=(Q, K, V, O), plan=plan, tab=tab, thresholds=thresholds)


def setup_gather(w, device, torch, sa, workloads):
    Q, K, V, idx = workloads.gather_inputs(w, device=device)
    O = torch.empty_like(Q)
    n_sets = w.S * w.H
    rows = n_sets * w.n_idx
    algo_bytes = rows * 2 * w.d * 2 + idx.numel() * 4 + Q.numel() * 2 + O.numel() * 2
    flops = 4 * rows * w.d

    def step(stream=None):
        sa.sparse_attn_gather(Q, K, V, idx, O=O, stream=stream)

    # end to end: the query and index sets come from the host each step, the
    # KV cache stays resident (it is the cache being decoded against)
    host = [Q.cpu().pin_memory(), idx.cpu().pin_memory(),
            torch.empty(O.shape, dtype=O.dtype, pin_memory=True)]
    Qd, idxd, Od = torch.empty_like(Q), torch.empty_like(idx), torch.empty_like(O)

    def e2e_step(stream):
        Qd.copy_(host[0], non_blocking=True)
        idxd.copy_(host[1], non_blocking=True)
        sa.sparse_attn_gather(Qd, K, V, idxd, O=Od, stream=stream)
        host[2].copy_(Od, non_blocking=True)

    h2d = host[0].numel() * 2 + host[1].numel() * 4
    d2h = host[2].numel() * 2
    return dict(step=step, e2e_step=e2e_step, h2d=h2d, d2h=d2h, flops=flops, exact_flops=flops,
                dense_flops=4 * n_sets * w.L * w.d, algo_bytes=algo_bytes,
                extra={"rows_gathered": rows}, kernel="gather_kernel",
                kernel_files=["gather_sm100.cu"], metric="gather GB/s", unit="GB/s", bound="hbm",
                tensors=(Q, K, V, idx, O), idx=idx)


def setup_window_decode(w, device, torch, sa, workloads):
    Q, K, V, pos = workloads.window_decode_inputs(w, device=device)
    O = torch.empty_like(Q)
    pat = sa.Pattern(causal=1, window=w.window, n_global=w.n_global)
    n_rows = w.window + w.n_global                  # every query sits past the window
    # each cached row is needed once per (sequence, K/V head): the query heads
    # of a group read it again from L2
    algo_bytes = (w.S * w.H_kv * n_rows * 2 * w.d * 2 + Q.numel() * 2 + O.numel() * 2
                  + pos.numel() * 4)
    flops = 4 * w.S * w.H * n_rows * w.d

    def step(stream=None):
        sa.sparse_attn_decode_window(Q, K, V, pos, pat, O=O, stream=stream)

    host = [Q.cpu().pin_memory(), pos.cpu().pin_memory(),
            torch.empty(O.shape, dtype=O.dtype, pin_memory=True)]
    Qd, posd, Od = torch.empty_like(Q), torch.empty_like(pos), torch.empty_like(O)

    def e2e_step(stream):
        Qd.copy_(host[0], non_blocking=True)
        posd.copy_(host[1], non_blocking=True)
        sa.sparse_attn_decode_window(Qd, K, V, posd, pat, O=Od, stream=stream)
        host[2].copy_(Od, non_blocking=True)

    h2d = host[0].numel() * 2 + host[1].numel() * 4
    d2h = host[2].numel() * 2
    return dict(step=step, e2e_step=e2e_step, h2d=h2d, d2h=d2h, flops=flops, exact_flops=flops,
                dense_flops=flops, algo_bytes=algo_bytes,
                extra={"rows_per_query": n_rows, "cache_slots": n_rows},
                kernel="window_group_kernel", kernel_files=["gather_sm100.cu", "ptx.cuh"],
                metric="window decode GB/s", unit="GB/s", bound="hbm",
                tensors=(Q, K, V, pos, O), pos=pos)


def setup_topk_decode(w, device, torch, sa, workloads):
    Q, K, V = workloads.topk_decode_inputs(w, device=device)
    O = torch.empty_like(Q)
    idx = torch.zeros((w.S, w.H, w.top_k), dtype=torch.int32, device=device)
    n_sel = torch.zeros((w.S, w.H), dtype=torch.int32, device=device)
    ws = torch.empty(sa.decode_topk_workspace_bytes(w.S, w.H, w.L, w.top_k), dtype=torch.uint8,
                     device=device)
    # every K row is scored once per (sequence, K/V head); the selected V rows
    # are read once per (sequence, query head)
    k_bytes = w.S * w.H_kv * w.L * w.d * 2
    v_bytes = w.S * w.H * w.top_k * w.d * 2
    algo_bytes = k_bytes + v_bytes + Q.numel() * 2 + O.numel() * 2
    flops = 2 * w.S * w.H * w.L * w.d + 2 * w.S * w.H * w.top_k * w.d

    def step(stream=None):
        sa.sparse_attn_decode_topk(Q, K, V, w.top_k, O=O, idx=idx, idx_len=n_sel, workspace=ws,
                                   stream=stream)

    host = [Q.cpu().pin_memory(), torch.empty(O.shape, dtype=O.dtype, pin_memory=True)]
    Qd, Od = torch.empty_like(Q), torch.empty_like(O)

    def e2e_step(stream):
        Qd.copy_(host[0], non_blocking=True)
        sa.sparse_attn_decode_topk(Qd, K, V, w.top_k, O=Od, idx=idx, idx_len=n_sel, workspace=ws,
                                   stream=stream)
        host[1].copy_(Od, non_blocking=True)

    h2d = host[0].numel() * 2
    d2h = host[1].numel() * 2
    return dict(step=step, e2e_step=e2e_step, h2d=h2d, d2h=d2h, flops=flops, exact_flops=flops,
                dense_flops=flops, algo_bytes=algo_bytes,
                extra={"k_bytes_scored": k_bytes, "v_bytes_selected": v_bytes,
                       "workspace_bytes": ws.numel()},
                # the roofline unit is the whole step (score, select and attend
                # kernels): its traffic is the three kernels' DRAM bytes together
                kernel="topk_step", kernel_files=["topk_sm100.cu"],
                launches_per_step=3,
                metric="top-K decode GB/s", unit="GB/s", bound="hbm",
                tensors=(Q, K, V, None, O))


# ------------------------------------------------------------- CPU baseline --
def cpu_oracle_rate(w, seconds, sample_seed=0, device_tensors=None, thresholds=None,
                    threshold_note=""):
    """Times the fp64 oracle as it stands on the host cores over a bounded sample
    of the workload; returns (value in the workload's unit, cores, description).
    thresholds: the block-skip workloads' per-head thresholds (oracle_thresholds)."""
    import numpy as np
    import torch
    import oracle
    from block_sparse_attention_29_b200 import workloads
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    g = np.random.default_rng(1234 + sample_seed)
    if isinstance(w, workloads.WindowDecodeWorkload):
        # window decode: sampled (sequence, head) queries over the oracle's
        # gather with the cache slots of their index sets (same rows, same order)
        Q, K, V, pos = device_tensors
        group = w.H // w.H_kv
        rows_of = {}   # (s, kv head) -> its cache rows in key order, gathered once

        def rows(s, hk):
            if (s, hk) not in rows_of:
                ix = torch.from_numpy(workloads.window_slots_in_key_order(
                    int(pos[s]), w.window, w.n_global)).to(K.device)
                rows_of[(s, hk)] = (K[s, hk, ix].cpu(), V[s, hk, ix].cpu())
            return rows_of[(s, hk)]
        done_rows, t_total, n = 0, 0.0, 8
        while t_total < seconds:
            pairs = [(int(g.integers(w.S)), int(g.integers(w.H))) for _ in range(n)]
            Qh = torch.stack([Q[s, h] for s, h in pairs])[None].cpu()
            Kh = torch.stack([rows(s, h // group)[0] for s, h in pairs])[None]
            Vh = torch.stack([rows(s, h // group)[1] for s, h in pairs])[None]
            m = Kh.shape[2]
            local = np.broadcast_to(np.arange(m, dtype=np.int32), (1, n, m)).copy()
            t0 = time.perf_counter()
            oracle.gather(Qh, Kh, Vh, local, nthreads=cores)
            t_total += time.perf_counter() - t0
            done_rows += n * m
            n = min(32, n * 2)
        gbs = done_rows * (2 * w.d * 2) / t_total / 1e9
        return gbs, cores, f"{done_rows // m} (sequence, head) queries, {done_rows} cache rows"
    if isinstance(w, workloads.TopkDecodeWorkload):
        # top-K decode: sampled (sequence, head) queries, each scored against its
        # K/V head's whole cache, then attending to its selected keys
        Q, K, V, _ = device_tensors
        group = w.H // w.H_kv
        done, t_total, scanned, picked = 0, 0.0, 0, 0
        while t_total < seconds:
            s, h = int(g.integers(w.S)), int(g.integers(w.H))
            Qh = Q[s, h][None, None].cpu()
            Kh = K[s, h // group][None, None].cpu()
            Vh = V[s, h // group][None, None].cpu()
            t0 = time.perf_counter()
            ix, n, _, _ = oracle.topk_select(Qh, Kh, w.top_k, nthreads=cores)
            oracle.gather(Qh, Kh, Vh, ix, n, nthreads=cores)
            t_total += time.perf_counter() - t0
            done += 1
            scanned += w.L
            picked += int(n[0, 0])
        gbs = (scanned * w.d * 2 + picked * w.d * 2) / t_total / 1e9
        return gbs, cores, f"{done} (sequence, head) queries over {w.L} keys each"
    if isinstance(w, workloads.GatherWorkload):
        # gather: sampled (sequence, head) sets, only their referenced rows on the host
        if device_tensors is None:
            raise RuntimeError("gather baseline needs the device tensors")
        Q, K, V, idx = device_tensors
        group = w.H // w.H_kv
        done_rows, t_total = 0, 0.0
        n = 8
        while t_total < seconds:
            pairs = [(int(g.integers(w.S)), int(g.integers(w.H))) for _ in range(n)]
            Qs = torch.stack([Q[s, h] for s, h in pairs])[None]
            ixs = [idx[s, h if w.H_idx == w.H else h // group].long() for s, h in pairs]
            Ks = torch.stack([K[s, h // group, ix] for (s, h), ix in zip(pairs, ixs)])[None]
            Vs = torch.stack([V[s, h // group, ix] for (s, h), ix in zip(pairs, ixs)])[None]
            # one "sequence" whose K/V heads are the sampled sets, one query head per set
            local = np.broadcast_to(np.arange(w.n_idx, dtype=np.int32), (1, n, w.n_idx)).copy()
            Qh, Kh, Vh = Qs.cpu(), Ks.cpu(), Vs.cpu()
            t0 = time.perf_counter()
            oracle.gather(Qh, Kh, Vh, local, nthreads=cores)
            t_total += time.perf_counter() - t0
            done_rows += n * w.n_idx
            n = min(4096, n * 2)
        gbs = done_rows * (2 * w.d * 2 + 4) / t_total / 1e9
        return gbs, cores, f"{done_rows // w.n_idx} (sequence, head) sets, {done_rows} rows"
    # prefill: whole query tiles of the descriptor's height (block_q rows of one
    # residue class for a dilated window).  The computed-block FLOPs of the
    # sample are counted from the oracle's own enumeration of G_i (build_G) at
    # the descriptor's block granularity, and for the block-skip rule from the
    # oracle's own block decisions; nothing here touches the CUDA library.
    Q, K, V, tab = (device_tensors if device_tensors is not None
                    else workloads.prefill_inputs(w, device="cpu"))
    Qh, Kh, Vh = (Q.cpu(), K.cpu(), V.cpu()) if isinstance(Q, torch.Tensor) else (Q, K, V)
    opat = oracle.Pattern(**w.pattern_fields(), random_table=tab)
    if w.bsfa and thresholds is None:
        raise RuntimeError("the block-skip workloads need the oracle's thresholds")
    k = max(1, w.dilation)
    n_pos = w.N // k
    bq, bk = w.block_q, w.block_k
    T = -(-n_pos // bq)
    flops_done, t_total, tiles_done, n, blocks_done = 0, 0.0, 0, 1, 0
    listed_of = {}   # (head or 0, tile, residue class) -> listed blocks (the lists repeat)

    def listed_blocks(h, t, r):
        key = (h if w.n_random > 0 else 0, t, r)
        if key not in listed_of:
            kbs = set()
            for mm in range(t * bq, min(n_pos, t * bq + bq)):
                G = oracle.build_G(opat, w.N, h, mm * k + r)
                kbs.update(np.unique((G // k) // bk).tolist())
            listed_of[key] = len(kbs)
        return listed_of[key]
    while t_total < seconds:
        tiles = [(int(g.integers(w.B)), int(g.integers(w.H)), int(g.integers(T)),
                  int(g.integers(k))) for _ in range(n)]
        rows = np.array([(b, h, m * k + r) for b, h, t, r in tiles
                         for m in range(t * bq, min(n_pos, t * bq + bq))], np.int32)
        t0 = time.perf_counter()
        res = oracle.prefill(opat, Qh, Kh, Vh, thresholds=thresholds, rows=rows, nthreads=cores,
                             keep_in_denominator=bool(w.skipped_in_denominator),
                             row_level=bool(w.row_level_skip), want_blocks=bool(w.bsfa))
        t_total += time.perf_counter() - t0
        for b, h, t, r in tiles:
            if w.bsfa:
                m = res[2][b, h, t]
                listed, kept = int((m != 0).sum()), int((m == 1).sum())
            else:
                listed = kept = listed_blocks(h, t, r)
            flops_done += 2 * bq * bk * w.d * (listed + kept)
            blocks_done += listed
        tiles_done += n
        n = min(64, n * 2)
    what = f"{tiles_done} whole {bq}-row query tiles ({blocks_done} listed {bq}x{bk} blocks)"
    if w.bsfa:
        what += ", thresholds " + threshold_note
    return flops_done / t_total / 1e12, cores, what


def oracle_thresholds(w, tiles_per_head=4, nthreads=0):
    """Per-head thresholds of the block-skip rule computed by the oracle alone:
    the lower median of the full-block statistics of a seeded sample of the
    calibration draw's query tiles (tiles_per_head per head, spread over the
    sequence).  Used by the oracle's timing legs, which cannot afford the
    statistics of the whole calibration draw."""
    import numpy as np
    import oracle
    from block_sparse_attention_29_b200 import workloads
    if w.thresholds == "minus_inf":
        return np.full(w.H, -np.inf), "of -inf (every block kept)"
    Qc, Kc, _, tab = workloads.calibration_inputs(w, device="cpu")
    opat = oracle.Pattern(**w.pattern_fields(), random_table=tab)
    T = -(-w.N // w.block_q)
    g = np.random.default_rng(77)
    tiles = [(b, h, int(t)) for b in range(w.B) for h in range(w.H)
             for t in g.choice(np.arange(T // 4, T), size=tiles_per_head, replace=False)]
    full, stat, _ = oracle.block_stats(opat, Qc, Kc, tiles=np.array(tiles, np.int32),
                                       nthreads=nthreads)
    return (oracle.calibrate_thresholds(full, stat),
            f"from the oracle's statistics of {tiles_per_head} calibration tiles per head")


# --------------------------------------------------------------------- main --
HEADLINE = "bsfa_causal"
# Timed after the headline in the same run: the other four configurations of
# the metric (tiny static pattern, Mistral window, Longformer/BigBird, index-set
# gather), then the block-skip workload with thresholds of -inf (nothing
# skipped: what the rule saves is measured against it), then the extensions (the
# rule's two variants, dilated window, window decode, top-K decode, split tiles
# forced and automatic).
SECONDARY = ("mistral_swa", "longformer_bigbird", "gather_decode", "tiny_static",
             "bsfa_causal_noskip", "bsfa_denominator", "bsfa_row_level", "dilated_swa",
             "window_decode", "topk_decode", "longformer_split", "bigbird_two_heads")
SECONDARY_MIN_S = 0.3   # each secondary workload's timed region lasts at least this long


def pipelined_e2e(P, steps, warmup, torch):
    """End to end over a stream of steps, as a server runs them: step i copies
    its inputs from pinned host memory into device buffer set i % n (copy-in
    stream), makes the library call on them (compute stream) and copies its
    output back to pinned host memory (copy-out stream).  A set's inputs are
    refilled only after the call that read them has finished, and its output
    is overwritten only after it has been copied out, so the copies of steps
    i + 1 and i - 1 overlap the call of step i.  Every step's copies are inside
    the timed region, which runs from before the first timed step's input copy
    to after the last step's output copy.  Returns (ms per timed step, the host
    output of the last step)."""
    n_sets = len(P["dev_sets"])
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    n = warmup + steps
    ev_in = [torch.cuda.Event() for _ in range(n)]
    ev_cmp = [torch.cuda.Event() for _ in range(n)]
    ev_out = [torch.cuda.Event() for _ in range(n)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for i in range(n):
        if i == warmup:
            torch.cuda.synchronize()
            t0.record(s_in)
        dev = P["dev_sets"][i % n_sets]
        if i >= n_sets:
            s_in.wait_event(ev_cmp[i - n_sets])      # the call that read this set is done
        with torch.cuda.stream(s_in):
            for h, d in zip(P["host_in"], dev[:-1]):
                d.copy_(h, non_blocking=True)
        ev_in[i].record(s_in)
        s_cmp.wait_event(ev_in[i])
        if i >= n_sets:
            s_cmp.wait_event(ev_out[i - n_sets])     # this set's output has been copied out
        P["launch"](dev, s_cmp)
        ev_cmp[i].record(s_cmp)
        s_out.wait_event(ev_cmp[i])
        with torch.cuda.stream(s_out):
            P["host_out"][i % n_sets].copy_(dev[-1], non_blocking=True)
        ev_out[i].record(s_out)
    t1.record(s_out)
    torch.cuda.synchronize()
    return t0.elapsed_time(t1) / steps, P["host_out"][(n - 1) % n_sets]


def setup_for(w, workloads):
    if isinstance(w, workloads.WindowDecodeWorkload):
        return setup_window_decode
    if isinstance(w, workloads.TopkDecodeWorkload):
        return setup_topk_decode
    if isinstance(w, workloads.GatherWorkload):
        return setup_gather
    return setup_prefill


def time_steps(S, steps, warmup, stream, flush, torch, sa, dist, device, clock_index):
    """W untimed warm-up steps, then exactly `steps` steps between a barrier and
    a synchronize on both sides; each step's launches are timed with CUDA events
    on their stream, L2 flushed before every step (outside the events).
    Returns (per-step ms, total ms max over ranks, clock summary)."""
    for _ in range(warmup):
        flush.zero_()
        S["step"](stream)
    sa.check_device_error()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(clock_index) as clk:
        for k in range(steps):
            flush.zero_()
            starts[k].record(stream)
            S["step"](stream)
            ends[k].record(stream)
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    sa.check_device_error()
    per_step = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = max_over_ranks(sum(per_step), dist, device)
    return per_step, total_ms, clk.summary()


def summarize(S, w, world, steps, warmup, per_step, total_ms, clocks, peaks, peak_src):
    """Metric value, roofline of the dominant kernel and the secondary figures."""
    ms_per_step = total_ms / steps
    per_launch_s = ms_per_step / 1e3
    if S["unit"] == "TFLOP/s":
        value = aggregate_rate(world, S["flops"], per_launch_s, 1e12)
        achieved = S["flops"] / per_launch_s / 1e12
        peak = peaks["bf16_tflops"]
        roof_unit = "TFLOP/s"
    else:
        value = aggregate_rate(world, S["algo_bytes"], per_launch_s, 1e9)
        achieved = value / world
        peak = peaks["hbm_gbs"]
        roof_unit = "GB/s"
    sha = kernel_source_sha(S["kernel_files"])
    out = {
        "metric": S["metric"], "value": round(value, 3), "unit": S["unit"], "n_gpus": world,
        "steps": steps, "warmup": warmup, "ms_per_step": round(ms_per_step, 5),
        "roofline": {"bound": S["bound"], "achieved": round(achieved, 3), "peak": peak,
                     "unit": roof_unit, "frac": round(achieved / peak, 4),
                     "peak_source": f"{peak_src} ({'bf16_tflops burst' if roof_unit == 'TFLOP/s' else 'hbm_gbs'})",
                     "traffic": recorded_traffic(S["kernel"], w.name, sha),
                     "kernel": S["kernel"], "kernel_source_sha": sha},
        "clocks": clocks,
        "per_step_ms": {"min": round(min(per_step), 5), "median": round(statistics.median(per_step), 5),
                        "max": round(max(per_step), 5)},
    }
    if S["unit"] == "TFLOP/s":
        out["secondary"] = {
            "dense_equiv_tflops": round(world * S["dense_flops"] / per_launch_s / 1e12, 3),
            "exact_pair_tflops": round(world * S["exact_flops"] / per_launch_s / 1e12, 3),
            "pct_bf16_peak_burst": round(100 * achieved / peaks["bf16_tflops"], 2),
            "pct_bf16_peak_sustained": round(100 * achieved / peaks.get("bf16_tflops_sustained", 1400.0), 2),
            "computed_block_flops": S["flops"], **S["extra"]}
    else:
        out["secondary"] = {"pct_hbm_peak": round(100 * achieved / peaks["hbm_gbs"], 2),
                            "algorithmic_bytes": S["algo_bytes"], **S["extra"]}
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=HEADLINE)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true",
                    help="time the chosen workload only (the secondary workloads are timed "
                         "after the headline by default)")
    ap.add_argument("--sequences", type=int, default=0,
                    help="decode workloads: run this many sequences instead of the workload's "
                         "(a reduced case of the same kernels, e.g. for counter captures)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    from block_sparse_attention_29_b200 import workloads
    w = workloads.WORKLOADS[args.workload]
    if args.sequences > 0:
        import dataclasses
        if not hasattr(w, "S"):
            raise SystemExit("--sequences applies to the decode workloads only")
        w = dataclasses.replace(w, S=args.sequences)

    if args.impl == "reference":
        if rank != 0:
            return
        run_reference(args, w, world)
        return

    import torch
    import block_sparse_attention_29_b200 as sa
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", device_id=device, timeout=datetime.timedelta(seconds=120))

    S = setup_for(w, workloads)(w, device, torch, sa, workloads)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()
    peaks, peak_src = load_peaks()

    per_step, total_ms, clocks = time_steps(S, args.steps, args.warmup, stream, flush, torch, sa,
                                            dist, device, local_rank)

    # end to end: the same call with host buffers, copies inside the timed region
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(2):
        S["e2e_step"](stream)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(args.steps):
        S["e2e_step"](stream)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist, device) / args.steps
    sa.check_device_error()
    serial_ms, e2e_mode = e2e_ms, "serial: copy in, call, copy out, one step after another"
    if "e2e_pipe" in S:
        # the stream of steps; its last output must equal the device run's bit for bit
        ok, pipe_ms = 0.0, 0.0
        try:
            if dist:
                dist.barrier()
            P = S["e2e_pipe"]()
            pipe_ms, last = pipelined_e2e(P, args.steps, 2, torch)
            sa.check_device_error()
            ok = 1.0 if torch.equal(last, P["result_dev"].cpu()) else 0.0
        except Exception as ex:   # keep the serial figure; say why
            print(f"pipelined end-to-end run failed: {ex}", file=sys.stderr)
            torch.cuda.synchronize()
        P = None
        ok = -max_over_ranks(-ok, dist, device)           # every rank's output matched
        pipe_ms = max_over_ranks(pipe_ms, dist, device)
        if ok == 1.0 and pipe_ms > 0:
            e2e_ms = pipe_ms
            e2e_mode = ("pipelined over steps: step i+1's input copy and step i-1's output copy "
                        "overlap step i's call (two device buffer sets, a copy stream each way)")
        else:
            e2e_mode += " (the pipelined run failed or its output differed)"

    head = summarize(S, w, world, args.steps, args.warmup, per_step, total_ms, clocks, peaks,
                     peak_src)
    if S["unit"] == "TFLOP/s":
        e2e_value = aggregate_rate(world, S["flops"], e2e_ms / 1e3, 1e12)
    else:
        e2e_value = aggregate_rate(world, S["algo_bytes"], e2e_ms / 1e3, 1e9)
    out = {
        "metric": head["metric"], "value": head["value"], "unit": head["unit"], "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded, device-generated; see block_sparse_attention_29_b200/workloads.py)",
        "config": config_of(w, world),
        "e2e": {"value": round(e2e_value, 3), "unit": S["unit"],
                "h2d_bytes_per_step": S["h2d"], "d2h_bytes_per_step": S["d2h"],
                "ms_per_step": round(e2e_ms, 5), "mode": e2e_mode,
                "serial_ms_per_step": round(serial_ms, 5)},
        "gpu_launches": args.steps * S.get("launches_per_step", 1),
        "roofline": head["roofline"], "clocks": head["clocks"], "per_step_ms": head["per_step_ms"],
        "secondary": head["secondary"],
    }

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        if isinstance(w, (workloads.GatherWorkload, workloads.WindowDecodeWorkload,
                          workloads.TopkDecodeWorkload)):
            Q, K, V, idx, _ = S["tensors"]
            dt = (Q, K, V, idx)
        else:
            Q, K, V, _ = S["tensors"]
            dt = (Q, K, V, S["tab"])
        th, note = (oracle_thresholds(w) if getattr(w, "bsfa", False) else (None, ""))
        val, cores, sample = cpu_oracle_rate(w, args.cpu_seconds, device_tensors=dt,
                                             thresholds=th, threshold_note=note)
        out["cpu_baseline"] = {"value": round(val, 6), "unit": S["unit"], "cores": cores,
                               "kind": "oracle", "sample": sample}
    S = None
    torch.cuda.empty_cache()

    if args.workload == HEADLINE and not args.no_secondary:
        table = {}
        for name in SECONDARY:
            ws = workloads.WORKLOADS[name]
            Ss = setup_for(ws, workloads)(ws, device, torch, sa, workloads)
            # steps: enough for SECONDARY_MIN_S of timed work (clock samples), at least --steps
            probe, _, _ = time_steps(Ss, 3, args.warmup, stream, flush, torch, sa, dist, device,
                                     local_rank)
            est = max(1e-3, statistics.median(probe))
            steps = min(2000, max(args.steps, math.ceil(1e3 * SECONDARY_MIN_S / est)))
            steps = int(max_over_ranks(steps, dist, device))
            ps, tot, clk = time_steps(Ss, steps, 3, stream, flush, torch, sa, dist, device,
                                      local_rank)
            r = summarize(Ss, ws, world, steps, 3, ps, tot, clk, peaks, peak_src)
            r["config"] = config_of(ws, world)
            r["gpu_launches"] = steps * Ss.get("launches_per_step", 1)
            table[name] = r
            Ss = None
            torch.cuda.empty_cache()
        out["secondary"]["workloads"] = table
        if "bsfa_causal_noskip" in table:
            # the rule's saving: the same inputs with nothing skipped, over the headline
            out["secondary"]["block_skip_speedup"] = round(
                table["bsfa_causal_noskip"]["ms_per_step"] / out["ms_per_step"], 4)
        out["secondary"]["workloads_note"] = (
            "each timed like the headline (CUDA events per step, L2 flushed before every step, "
            "clocks sampled during its own timed region); end-to-end and CPU baseline are "
            "measured for the headline only")

    if rank == 0:
        print(json.dumps(out), flush=True)
    if dist:
        dist.destroy_process_group()


def config_of(w, world):
    from block_sparse_attention_29_b200 import workloads
    if isinstance(w, workloads.TopkDecodeWorkload):
        return {"workload": w.name, "sequences": w.S, "H": w.H, "H_kv": w.H_kv, "d": w.d,
                "cache_len": w.L, "top_k": w.top_k, "selection": "dynamic (scores at run time)",
                "per_rank": "one replica per GPU", "l2": "256 MiB flush before every step"}
    if isinstance(w, workloads.WindowDecodeWorkload):
        return {"workload": w.name, "sequences": w.S, "H": w.H, "H_kv": w.H_kv, "d": w.d,
                "pattern": {"causal": 1, "window": w.window, "n_global": w.n_global},
                "cache_slots": w.window + w.n_global, "positions": f"uniform in "
                f"[{w.window + w.n_global}, {w.max_pos}]",
                "per_rank": "one replica per GPU", "l2": "256 MiB flush before every step"}
    if isinstance(w, workloads.GatherWorkload):
        return {"workload": w.name, "sequences": w.S, "H": w.H, "H_kv": w.H_kv, "d": w.d,
                "cache_len": w.L, "n_idx": w.n_idx, "H_idx": w.H_idx,
                "per_rank": "one replica per GPU", "l2": "256 MiB flush before every step"}
    pat = {k: v for k, v in w.pattern_fields().items() if v and not (k == "dilation" and v == 1)}
    return {"workload": w.name, "B": w.B, "H": w.H, "H_kv": w.H_kv, "N": w.N, "d": w.d,
            "pattern": pat, "block_skip_rule": bool(w.bsfa),
            **({"thresholds": w.thresholds} if w.bsfa else {}),
            **({"skipped_keys_in_denominator": True} if w.skipped_in_denominator else {}),
            **({"row_level_skip": True} if w.row_level_skip else {}),
            "per_rank": "one replica per GPU", "l2": "256 MiB flush before every step"}


def run_reference(args, w, world):
    """The fp64 oracle as it stands, on this host's cores (rank 0 only)."""
    import oracle
    oracle.build()
    from block_sparse_attention_29_b200 import workloads
    dt = None
    if isinstance(w, workloads.WindowDecodeWorkload):
        import dataclasses
        ws = dataclasses.replace(w, S=4)
        dt = workloads.window_decode_inputs(ws, device="cpu")
        w = ws
    elif isinstance(w, workloads.TopkDecodeWorkload):
        import dataclasses
        ws = dataclasses.replace(w, S=2)
        Q, K, V = workloads.topk_decode_inputs(ws, device="cpu")
        dt = (Q, K, V, None)
        w = ws
    elif isinstance(w, workloads.GatherWorkload):
        # a cache of the full size does not fit the host budget of this arm: the
        # sampled sets' rows are drawn with the same recipe at reduced length
        import dataclasses
        import torch
        ws = dataclasses.replace(w, S=4, L=max(w.n_idx + w.n_recent + 1, 8192))
        Q, K, V, idx = workloads.gather_inputs(ws, device="cpu")
        dt = (Q, K, V, idx)
        w = ws
    else:
        dt = workloads.prefill_inputs(w, device="cpu")
    # the block-skip rule's thresholds, calibrated by the oracle itself (untimed)
    th, note = (oracle_thresholds(w) if getattr(w, "bsfa", False) else (None, ""))
    budget = 60.0
    per_step = max(1.0, budget / (args.steps + args.warmup))
    for _ in range(args.warmup):
        cpu_oracle_rate(w, per_step / 4, device_tensors=dt, thresholds=th, threshold_note=note)
    vals, cores, sample = [], None, None
    t0 = time.perf_counter()
    for k in range(args.steps):
        v, cores, sample = cpu_oracle_rate(w, per_step, sample_seed=k + 1, device_tensors=dt,
                                           thresholds=th, threshold_note=note)
        vals.append(v)
    elapsed = time.perf_counter() - t0
    value = statistics.mean(vals)
    unit = ("GB/s" if isinstance(w, (workloads.GatherWorkload, workloads.WindowDecodeWorkload,
                                     workloads.TopkDecodeWorkload))
            else "TFLOP/s")
    metric = ("window decode GB/s" if isinstance(w, workloads.WindowDecodeWorkload) else
              "top-K decode GB/s" if isinstance(w, workloads.TopkDecodeWorkload) else
              "gather GB/s" if unit == "GB/s" else "effective TFLOP/s (computed blocks)")
    out = {"impl": "reference", "metric": metric, "value": round(value, 6), "unit": unit,
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": round(1e3 * elapsed / args.steps, 3), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": config_of(w, world),
           "cpu_baseline": {"value": round(value, 6), "unit": unit, "cores": cores,
                            "kind": "oracle", "sample": f"per step: {sample}"},
           "e2e": {"value": round(value, 6), "unit": unit, "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
