"""Benchmark: one step = the whole hot path (pooled block scores -> max-based threshold + CSR ->
block-sparse attention) over one seeded synthetic prefill, through the C ABI.

Default workload: the 131072-token Llama-3-8B-shaped layer (bf16, Hq 32 / Hkv 8, D 128,
block 128, alpha 0.1, 0.2% vertical columns).  Inputs (Q+K+V = 1.6 GB) are larger than L2, so
no L2 flush is needed between steps.

Prints ONE JSON line (rank 0).  `value` is the dense-equivalent throughput of the whole step:
2 * Hq * D * sum(N^2) FLOP (causal dense attention) / step time, summed over ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Multi-GPU (torchrun, one rank per GPU): every rank runs its own copy of the workload (the
prefill's (sequence, KV-head) units are independent; no data-path collective), timed on the
device and reduced as the max over ranks -> weak scaling.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gen import WORKLOADS, default_workers, generate  # noqa: E402

METRIC = "sparse prefill-attn ms & dense-equiv TFLOP/s at 32K/128K; search ms; density"
DEFAULT_WORKLOAD = "llama8b_bf16_n131072"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNELS_PER_STEP = 10  # plan+pool+score, plan+count+scan+emit, plan+order+attention

# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one attention launch per workload,
# from an ncu capture of the kernel built from sources whose digest is ATTN_TRAFFIC_DIGEST.
# Reported as roofline.traffic only while the sources still have that digest; any change to the
# kernel makes it null until it is measured again.
ATTN_SOURCES = ("dynamic_block_sparse_pooled_b200/csrc/fpx_attn_sm100.cu",
                "dynamic_block_sparse_pooled_b200/csrc/fpx_sm100.cuh",
                "dynamic_block_sparse_pooled_b200/csrc/fpx_common.cuh")
ATTN_TRAFFIC_DIGEST = "f88c351c7ee3c84bab085496a3a55124c32d919be05b2a163c66a83baa3ea018"
ATTN_TRAFFIC = {
    "llama8b_bf16_n131072": 3301625856 + 1180681216,
}


def attn_sources_digest() -> str:
    import hashlib
    h = hashlib.sha256()
    for rel in ATTN_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def attn_traffic(workload: str):
    """Measured DRAM bytes of one attention launch, or None (not measured for this workload, or
    the kernel sources changed since the capture)."""
    if workload not in ATTN_TRAFFIC or ATTN_TRAFFIC_DIGEST is None:
        return None
    try:
        return ATTN_TRAFFIC[workload] if attn_sources_digest() == ATTN_TRAFFIC_DIGEST else None
    except OSError:
        return None


def peaks():
    try:
        with open(PEAKS_FILE) as f:
            return json.load(f), "measured"
    except Exception:
        return FALLBACK_PEAKS, "fallback"


def max_over_ranks(values, device="cpu"):
    """Element-wise max of per-rank timings over the process group (identity when single)."""
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if torch.distributed.is_available() and torch.distributed.is_initialized() and \
            torch.distributed.get_world_size() > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def aggregate_value(flops_per_rank: float, world: int, ms_per_step: float) -> float:
    """Whole-job dense-equivalent TFLOP/s: every rank runs its own prefill (weak scaling), the
    step time is the slowest rank's."""
    return world * flops_per_rank / (ms_per_step * 1e-3) / 1e12


def config_of(w, world: int) -> dict:
    """The workload description both arms print (same keys, same values)."""
    return {"workload": w.name, "seqlens": list(w.seqlens), "hq": w.hq, "hkv": w.hkv,
            "d": w.d, "block": w.block, "alpha": w.alpha, "sink_blocks": w.sink_blocks,
            "window_blocks": w.window_blocks,
            "l2": "inputs (Q+K+V) larger than L2; no flush",
            "parallelism": f"replica x{world} (independent prefills)"}


def dense_flops(w) -> float:
    return float(sum(2.0 * w.hq * w.d * n * n for n in w.seqlens))


def pairs(w) -> int:
    return sum((-(-n // w.block)) * (-(-n // w.block) + 1) // 2 for n in w.seqlens)


L2_FLUSH_BELOW = 256 << 20  # Q + K + V below twice the 126 MB L2: flush between timed steps
NEAR_REL = 1e-3  # near-threshold band: |exp(s - m) - alpha| <= NEAR_REL * alpha


def selection_stats(scores, row_ptr, col_idx, cu, hq: int, hkv: int, block: int, alpha: float,
                    sink: int, window: int) -> dict:
    """Figures of one selection, from the device tensors after the timed region:

    * near_threshold_blocks: causal blocks not forced by sink / window whose ratio exp(s - m_I)
      (m_I = the row maximum of the pooled scores) lies within NEAR_REL * alpha of alpha — the
      blocks where an fp32 and an fp64 decision may both be right;
    * kv_tile_loads: K / V tile pairs the attention loads, one per block in the union of the
      two Q heads of a work unit (heads 2p and 2p + 1 of a KV group; an odd last head alone);
    * union_excess_tiles: tiles multiplied for a head that did not keep them (0: the kernel
      issues a tile's MMAs only for the heads that kept it; the union only shares the loads).
    scores: fp32 [hq * TRI] triangular-packed; row_ptr / col_idx: the CSR of fpx_select."""
    dev = scores.device
    nbs = [-(-(int(cu[i + 1]) - int(cu[i])) // block) for i in range(len(cu) - 1)]
    row_i, row_start, tri = [], [], 0
    for nb in nbs:
        for i in range(nb):
            row_i.append(i)
            row_start.append(tri + i * (i + 1) // 2)
        tri += nb * (nb + 1) // 2
    rows_h = len(row_i)
    out = {"near_threshold_blocks": 0, "kv_tile_loads": 0, "union_excess_tiles": 0}
    if rows_h == 0 or tri == 0:
        return out
    row_i = torch.tensor(row_i, dtype=torch.int64, device=dev)
    row_start = torch.tensor(row_start, dtype=torch.int64, device=dev)
    # row (within a head) of every triangular element, and its block indices I, J
    elem_row = torch.repeat_interleave(torch.arange(rows_h, device=dev), row_i + 1)
    elem_j = torch.arange(tri, device=dev) - row_start[elem_row]
    elem_i = row_i[elem_row]
    s = scores[:hq * tri].view(hq, tri).double()
    if alpha > 0:
        m = torch.full((hq, rows_h), float("-inf"), dtype=torch.float64, device=dev)
        m = m.scatter_reduce(1, elem_row.expand(hq, -1), s, reduce="amax", include_self=True)
        ratio = torch.exp(s - m.gather(1, elem_row.expand(hq, -1)))
        forced = (elem_j < sink) | (elem_j > elem_i - window)
        near = (~forced) & ((ratio - alpha).abs() <= NEAR_REL * alpha)
        out["near_threshold_blocks"] = int(near.sum().item())
    # kept flags in the triangular layout, from the CSR
    rp = row_ptr.to(torch.int64)
    nnz = int(rp[-1].item())
    kept = torch.zeros(hq * tri, dtype=torch.bool, device=dev)
    if nnz > 0:
        counts = rp[1:] - rp[:-1]
        row_of = torch.repeat_interleave(torch.arange(hq * rows_h, device=dev), counts)
        pos = (row_of // rows_h) * tri + row_start[row_of % rows_h] + col_idx[:nnz].to(torch.int64)
        kept[pos] = True
    kept = kept.view(hq, tri)
    g = hq // hkv
    loads = 0
    for kvh in range(hkv):
        for h0 in range(kvh * g, (kvh + 1) * g, 2):
            u = kept[h0] | kept[h0 + 1] if h0 + 1 < (kvh + 1) * g else kept[h0]
            loads += int(u.sum().item())
    out["kv_tile_loads"] = loads
    return out


class ClockSampler:
    """Samples the SM clock and the clock-event (throttle) reasons during the timed region, with
    NVML every 10 ms (short regions get at least one sample, taken at exit)."""
    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "sw_power_cap": 0x4}

    def __init__(self, index: int):
        self.index = index
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._nvml = None

    def _sample(self):
        nv = self._nvml
        sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
        try:
            reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except AttributeError:
            reasons = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        self.samples.append((sm, reasons))

    def _run(self):
        while not self._stop.wait(0.01):
            try:
                self._sample()
            except Exception:
                return

    def __enter__(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            self._nvml = nv
            self.h = nv.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
            self._sample()
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()
        except Exception:
            self._nvml = None
        return self

    def __exit__(self, *exc):
        if self._nvml is not None:
            self._stop.set()
            self.thread.join(timeout=1)
            try:
                self._sample()
            except Exception:
                pass

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"],
                    "samples": 0}
        reasons = sorted(name for name, bit in self.REASONS.items()
                         if any(r & bit for _, r in self.samples))
        return {"sm_mhz": statistics.median(s for s, _ in self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(self.samples)}


# ---------------------------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------------------------

def sdpa_baseline(w, dev, cu, device, reps=2):
    """Library baseline on the same inputs: PyTorch SDPA causal attention (dense, i.e. every
    causal tile; grouped K/V taken natively, or expanded to the Q heads where no fused backend
    takes them), restricted to the fused flash / cuDNN backends so that it can never fall back to
    the O(N^2)-memory math path.  bf16 workloads only."""
    if w.dtype != "bf16":
        return {"unavailable": "SDPA takes no e4m3 / fp32-parity configuration here"}
    try:
        from torch.nn.attention import SDPBackend, sdpa_kernel
        F = torch.nn.functional
        g = w.hq // w.hkv
        seqs = [(int(cu[i]), int(cu[i + 1])) for i in range(len(cu) - 1) if cu[i + 1] > cu[i]]

        native = [True]  # grouped K / V taken as they are (no expansion in the timed region)

        def run():
            for a, b in seqs:
                qq = dev["q"][a:b].transpose(0, 1).unsqueeze(0)
                if native[0]:
                    kk = dev["k"][a:b].transpose(0, 1).unsqueeze(0)
                    vv = dev["v"][a:b].transpose(0, 1).unsqueeze(0)
                    F.scaled_dot_product_attention(qq, kk, vv, is_causal=True, enable_gqa=True)
                else:
                    kk = dev["k"][a:b].repeat_interleave(g, dim=1).transpose(0, 1).unsqueeze(0)
                    vv = dev["v"][a:b].repeat_interleave(g, dim=1).transpose(0, 1).unsqueeze(0)
                    F.scaled_dot_product_attention(qq, kk, vv, is_causal=True)

        with sdpa_kernel([SDPBackend.FLASH_ATTENTION, SDPBackend.CUDNN_ATTENTION]):
            try:
                run()
            except (RuntimeError, TypeError):  # no fused backend takes grouped K / V here
                native[0] = False
                run()
            torch.cuda.synchronize(device)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(reps):
                run()
            b.record()
            torch.cuda.synchronize(device)
        ms = a.elapsed_time(b) / reps
        return {"ms": round(ms, 3), "dense_equiv_tflops": round(dense_flops(w) / (ms * 1e-3) / 1e12, 1),
                "what": "torch SDPA is_causal (flash/cuDNN backends), " +
                        ("grouped K/V (enable_gqa)" if native[0] else
                         "K/V expanded to the Q heads inside the timed region")}
    except Exception as e:  # a missing backend is reported, never a fallback
        return {"unavailable": f"{type(e).__name__}: {str(e)[:120]}"}


def extras(fpx, w, pf, dev, cu, ws, scores, row_ptr, col_idx, device, reps=3):
    """Timings of the optional paths on the same inputs (after the timed region): attention with
    K / V in a page cache (pages in reverse order) and the search with the radius rescue branch
    (alpha_rescue 0.1).  Each is the mean of `reps` CUDA-event-timed calls after one warm-up."""
    out = {}
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731

    def timed(fn):
        fn()
        torch.cuda.synchronize(device)
        a, b = ev(), ev()
        a.record()
        for _ in range(reps):
            fn()
        b.record()
        torch.cuda.synchronize(device)
        return round(a.elapsed_time(b) / reps, 4)

    try:
        if fpx.attention_path(pf) == 1:
            nbs = [-(-(int(cu[i + 1]) - int(cu[i])) // w.block) for i in range(len(cu) - 1)]
            npg = sum(nbs)
            table = torch.full((len(nbs), max(1, max(nbs))), -1, dtype=torch.int32)
            kc = torch.zeros((npg * w.block,) + tuple(dev["k"].shape[1:]), dtype=dev["k"].dtype,
                             device=device)
            vc = torch.zeros_like(kc)
            pg = npg
            for s_, nb in enumerate(nbs):
                for J in range(nb):
                    pg -= 1
                    table[s_, J] = pg
                    a_ = int(cu[s_]) + J * w.block
                    b_ = min(int(cu[s_ + 1]), a_ + w.block)
                    kc[pg * w.block: pg * w.block + (b_ - a_)] = dev["k"][a_:b_]
                    vc[pg * w.block: pg * w.block + (b_ - a_)] = dev["v"][a_:b_]
            kv = fpx.paged_kv(table.to(device), npg)
            out["paged_attn_ms"] = timed(lambda: fpx.sparse_prefill_paged(
                pf, dev["q"], kc, vc, kv, row_ptr, col_idx, ws))
            del kc, vc

        def rescue_search():
            sc, qn, rad = fpx.block_scores_rescue(pf, dev["q"], dev["k"], ws)
            fpx.select_rescue(pf, sc, qn, rad, w.alpha, 0.1, ws, w.sink_blocks, w.window_blocks)
        out["rescue_search_ms"] = timed(rescue_search)
        if fpx.status(ws) != 0:
            return {"unavailable": f"device status {fpx.status(ws)}"}
    except Exception as e:  # reported, never hidden
        return {"unavailable": f"{type(e).__name__}: {str(e)[:120]}"}
    return out


class Prefill:
    """One workload resident on the device with every buffer of the path allocated once; step()
    enqueues the whole hot path (fpx_block_scores -> fpx_select -> fpx_sparse_prefill) on the
    current stream and, when asked, records CUDA events around the search and the attention."""

    def __init__(self, fpx, w, data, device, host_copies=False):
        self.fpx, self.w, self.device = fpx, w, device
        self.cu = data["cu_seqlens"]
        if host_copies:
            self.host = {k: data[k].contiguous().pin_memory() for k in ("q", "k", "v")}
            self.dev = {k: self.host[k].to(device, non_blocking=True) for k in self.host}
        else:
            self.host = None
            self.dev = {k: data[k].to(device) for k in ("q", "k", "v")}
        for k in ("q_scale", "k_scale", "v_scale"):
            self.dev[k] = data[k].to(device) if data[k] is not None else None
        torch.cuda.synchronize(device)
        d = self.dev
        self.stream = torch.cuda.current_stream(device)
        self.pf = fpx.problem(d["q"], d["k"], w.block, self.cu, 0.0, d["q_scale"], d["k_scale"],
                              d["v_scale"])
        pf = self.pf
        self.ws = fpx.workspace(pf, -1, device)
        self.scores = torch.empty(w.hq * pf.tri, dtype=torch.float32, device=device)
        self.row_ptr = torch.empty(pf.rows + 1, dtype=torch.int32, device=device)
        self.col_idx = torch.empty(max(1, w.hq * pf.tri), dtype=torch.int32, device=device)
        self.nnz = torch.empty(1, dtype=torch.int64, device=device)
        self.o = torch.empty(d["q"].shape, dtype=torch.float32 if w.dtype == "f32"
                             else torch.bfloat16, device=device)
        self.lse = torch.empty((w.hq, w.total_tokens), dtype=torch.float32, device=device)

    def step(self, timing=None):
        fpx, w, d = self.fpx, self.w, self.dev
        ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
        e0, e1, e2 = ev(), ev(), ev()
        e0.record(self.stream)
        fpx.block_scores(self.pf, d["q"], d["k"], self.ws, scores=self.scores)
        fpx.select(self.pf, self.scores, w.alpha, self.ws, w.sink_blocks, w.window_blocks,
                   row_ptr=self.row_ptr, col_idx=self.col_idx, nnz=self.nnz)
        e1.record(self.stream)
        fpx.sparse_prefill(self.pf, d["q"], d["k"], d["v"], self.row_ptr, self.col_idx, self.ws,
                           o=self.o, lse=self.lse)
        e2.record(self.stream)
        if timing is not None:
            timing.append((e0, e1, e2))

    def check_status(self, when: str):
        st = self.fpx.status(self.ws)
        if st != 0:
            raise RuntimeError(f"device status {st} {when}")

    def metrics(self, search_ms, attn_ms, n_kept):
        """The per-workload figures of the metric, from per-step CUDA-event times."""
        w = self.w
        pk, pk_kind = peaks()
        peak_tf = pk.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
        if w.dtype == "e4m3":
            peak_tf *= 2.0  # fp8 dense is twice bf16 (nominal ratio)
        tri = pairs(w)
        attn = statistics.mean(attn_ms)
        srch = statistics.mean(search_ms)
        exec_tf = 4.0 * w.block * w.block * w.d * n_kept / (attn * 1e-3) / 1e12
        dq, dk = self.dev["q"], self.dev["k"]
        # algorithmic bytes of the search: Q and K read once, the pooled scores written once, the
        # CSR written (the select pass's read-back of the scores is reported apart, not counted)
        sbytes = (dq.numel() * dq.element_size() + dk.numel() * dk.element_size() +
                  4 * w.hq * tri + 4 * (self.pf.rows + 1) + 4 * n_kept)
        gbs = sbytes / (srch * 1e-3) / 1e9
        flops = dense_flops(w)
        return {
            "attn_ms": round(attn, 4), "search_ms": round(srch, 4),
            "density": round(n_kept / (w.hq * tri), 6), "nnz": n_kept,
            "attn_dense_equiv_tflops": round(flops / (attn * 1e-3) / 1e12, 3),
            "step_dense_equiv_tflops": round(flops / ((attn + srch) * 1e-3) / 1e12, 3),
            "attn_executed_tflops": round(exec_tf, 2),
            "attn_executed_frac": round(exec_tf / peak_tf, 4),
            "attn_peak": {"tflops": peak_tf, "kind": f"{pk_kind} bf16 sustained" +
                          (" x2 (fp8, nominal ratio)" if w.dtype == "e4m3" else "")},
            "search_bytes": sbytes, "search_gbs": round(gbs, 1),
            "search_hbm_frac": round(gbs / pk.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]), 4),
        }

    def measure(self, steps, warmup):
        """warmup untimed steps, then `steps` steps with per-step events; the figures above.
        A workload whose Q + K + V would stay in L2 gets L2 flushed before every timed step (a
        256 MB write on the same stream, outside the events)."""
        for _ in range(warmup):
            self.step()
        self.check_status("after warm-up")
        n_kept = int(self.nnz.item())
        inputs = sum(self.dev[k].numel() * self.dev[k].element_size() for k in ("q", "k", "v"))
        flush = torch.empty(64 << 20, dtype=torch.float32, device=self.device) \
            if inputs < L2_FLUSH_BELOW else None
        torch.cuda.synchronize(self.device)
        timing = []
        with ClockSampler(self.device.index if self.device.index is not None else 0) as clk:
            for _ in range(steps):
                if flush is not None:
                    flush.fill_(0.0)
                self.step(timing)
            torch.cuda.synchronize(self.device)
        self.check_status("after the timed steps")
        res = self.metrics([a.elapsed_time(b) for a, b, c in timing],
                           [b.elapsed_time(c) for a, b, c in timing], n_kept)
        res["clocks"] = clk.summary()
        res["l2"] = "flushed before every step (256 MB write)" if flush is not None else \
            "inputs (Q+K+V) larger than L2; no flush"
        del flush
        res.update(self.selection())
        return res

    def measure_graph(self, steps):
        """The same search and attention replayed from two captured CUDA graphs (one launch
        each from the host: what a server that replays its prefill graph sees), CUDA events
        around each replay, L2 flushed before every step as in measure()."""
        fpx, w, d = self.fpx, self.w, self.dev
        s = torch.cuda.Stream(self.device)
        s.wait_stream(torch.cuda.current_stream(self.device))
        g_search, g_attn = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_search, stream=s):
            fpx.block_scores(self.pf, d["q"], d["k"], self.ws, scores=self.scores)
            fpx.select(self.pf, self.scores, w.alpha, self.ws, w.sink_blocks, w.window_blocks,
                       row_ptr=self.row_ptr, col_idx=self.col_idx, nnz=self.nnz)
        with torch.cuda.graph(g_attn, stream=s):
            fpx.sparse_prefill(self.pf, d["q"], d["k"], d["v"], self.row_ptr, self.col_idx,
                               self.ws, o=self.o, lse=self.lse)
        flush = torch.empty(64 << 20, dtype=torch.float32, device=self.device)
        ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
        for _ in range(3):
            g_search.replay()
            g_attn.replay()
        torch.cuda.synchronize(self.device)
        times = []
        for _ in range(steps):
            flush.fill_(0.0)
            e0, e1, e2 = ev(), ev(), ev()
            e0.record()
            g_search.replay()
            e1.record()
            g_attn.replay()
            e2.record()
            times.append((e0, e1, e2))
        torch.cuda.synchronize(self.device)
        self.check_status("after the graph replays")
        srch = statistics.mean(a.elapsed_time(b) for a, b, c in times)
        attn = statistics.mean(b.elapsed_time(c) for a, b, c in times)
        del g_search, g_attn, flush
        return {"search_ms": round(srch, 4), "attn_ms": round(attn, 4),
                "how": "search and attention each replayed from a captured CUDA graph"}

    def selection(self):
        w = self.w
        st = selection_stats(self.scores, self.row_ptr, self.col_idx, self.cu, w.hq, w.hkv,
                             w.block, w.alpha, w.sink_blocks, w.window_blocks)
        n_kept = int(self.nnz.item())
        st["kv_loads_per_kept_tile"] = round(st["kv_tile_loads"] / n_kept, 4) if n_kept else None
        return st


def sub_records(fpx, args, device, sdpa_ms_128k):
    """The other configurations of the metric, timed by the same code after the headline's timed
    region (each: 3 warm-up steps, then args.sub_steps timed steps; every workload's Q + K + V is
    larger than L2 except the 8192-token layer's, which gets L2 flushed before every step).
    * sparse: the 131072-token layer with Q multiplied by q_gain (a labelled supplementary knob
      that widens the pooled-score spread as trained models' logits do): alpha = 0.1 then keeps
      about 50 %, 20 % and 5 % of the causal blocks; speed-up over the same run's dense SDPA;
    * llama8b_bf16_n32768 at alpha 0, 0.05, 0.1, 0.2; llama8b_e4m3_n131072; varlen8_bf16_t264192;
      llama8b_bf16_n8192 (where the search is launch-bound).
    """
    out = {"sparse": [], "configs": []}
    steps = args.sub_steps
    base = WORKLOADS["llama8b_bf16_n131072"]
    # one fp32 draw; Q for each gain is bf16(q_gain * q_fp32), exactly what the generator
    # produces for that gain
    f32 = generate(base.with_(dtype="f32"), workers=default_workers())
    for gain in (290.0, 340.0, 415.0):
        w = base.with_(q_gain=gain)
        data = dict(f32, q=(f32["q"] * np.float32(gain)).to(torch.bfloat16),
                    k=f32["k"].to(torch.bfloat16), v=f32["v"].to(torch.bfloat16))
        run = Prefill(fpx, w, data, device)
        r = run.measure(steps, 3)
        del run, data
        torch.cuda.empty_cache()
        r = {"workload": w.name, "q_gain": gain, "alpha": w.alpha, **r}
        if sdpa_ms_128k:
            r["speedup_vs_sdpa_dense"] = round(sdpa_ms_128k / r["attn_ms"], 3)
        out["sparse"].append(r)
    out["patterns"] = pattern_record(fpx, f32, device, steps)
    del f32
    for name, alphas in (("llama8b_bf16_n32768", (0.0, 0.05, 0.1, 0.2)),
                         ("llama8b_e4m3_n131072", (None,)), ("varlen8_bf16_t264192", (None,)),
                         ("llama8b_bf16_n8192", (None,))):
        w0 = WORKLOADS[name]
        data = generate(w0, workers=default_workers())
        for a in alphas:
            w = w0 if a is None else w0.with_(alpha=a)
            run = Prefill(fpx, w, data, device)
            r = run.measure(steps, 3)
            if name == "llama8b_bf16_n8192":
                r["graph"] = run.measure_graph(steps)
            del run
            torch.cuda.empty_cache()
            out["configs"].append({"workload": w.name, "alpha": w.alpha, **r})
        del data
    return out


def pattern_record(fpx, f32, device, steps, gain=40.0, n_probe=64, alpha_v=0.01, alpha_s=0.01):
    """The query-probe vertical / slash path on the 131072-token layer (Q x q_gain): probe
    discovery, candidate blocks and the token-masked attention, each timed with CUDA events
    (3 warm-up calls, then `steps`), with the sizes of what the probes selected."""
    try:
        w = WORKLOADS["llama8b_bf16_n131072"].with_(q_gain=gain)
        q = (f32["q"] * np.float32(gain)).to(torch.bfloat16).to(device)
        k = f32["k"].to(torch.bfloat16).to(device)
        v = f32["v"].to(torch.bfloat16).to(device)
        cu = f32["cu_seqlens"]
        pf = fpx.problem(q, k, w.block, cu)
        ws = fpx.vs_workspace(pf, n_probe, device)
        vert, slash = fpx.probe_patterns(pf, q, k, n_probe, alpha_v, alpha_s, ws)
        rp, ci, nnz = fpx.vs_select(pf, vert, slash, ws)
        o, lse = fpx.vs_prefill(pf, q, k, v, vert, slash, rp, ci, ws)
        stages = {
            "probe_ms": lambda: fpx.probe_patterns(pf, q, k, n_probe, alpha_v, alpha_s, ws,
                                                   vert=vert, slash=slash),
            "select_ms": lambda: fpx.vs_select(pf, vert, slash, ws, row_ptr=rp, col_idx=ci,
                                               nnz=nnz),
            "attn_ms": lambda: fpx.vs_prefill(pf, q, k, v, vert, slash, rp, ci, ws, o=o, lse=lse),
        }
        res = {"workload": w.name, "q_gain": gain, "n_probe": n_probe, "alpha_v": alpha_v,
               "alpha_s": alpha_s}
        for name, fn in stages.items():
            for _ in range(3):
                fn()
            torch.cuda.synchronize(device)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(steps):
                fn()
            b.record()
            torch.cuda.synchronize(device)
            res[name] = round(a.elapsed_time(b) / steps, 4)
        if fpx.status(ws) != 0:
            return {"unavailable": f"device status {fpx.status(ws)}"}
        bits = lambda t: int(np.unpackbits(t.cpu().numpy().view(np.uint8)).sum())  # noqa: E731
        res["verticals"] = bits(vert)
        res["slashes"] = bits(slash)
        res["candidate_density"] = round(int(nnz.item()) / (w.hq * pairs(w)), 6)
        res["dense_equiv_tflops"] = round(dense_flops(w) / (res["attn_ms"] * 1e-3) / 1e12, 1)
        return res
    except Exception as e:  # reported, never hidden
        return {"unavailable": f"{type(e).__name__}: {str(e)[:120]}"}


def run_ours(args, rank, world, device):
    import dynamic_block_sparse_pooled_b200 as fpx

    w = WORKLOADS[args.workload]
    if args.alpha is not None:
        w = w.with_(alpha=args.alpha)
    if args.q_gain is not None:
        w = w.with_(q_gain=args.q_gain)
    data = generate(w, workers=default_workers())
    run = Prefill(fpx, w, data, device, host_copies=True)
    stream = run.stream
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731

    for _ in range(args.warmup):
        run.step()
    run.check_status("after warm-up")
    n_kept = int(run.nnz.item())

    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    timing = []
    t_start, t_end = ev(), ev()
    with ClockSampler(device.index if device.index is not None else 0) as clk:
        t_start.record(stream)
        for _ in range(args.steps):
            run.step(timing)
        t_end.record(stream)
        torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    total_ms = t_start.elapsed_time(t_end)
    search_ms = [a.elapsed_time(b) for a, b, c in timing]
    attn_ms = [b.elapsed_time(c) for a, b, c in timing]
    run.check_status("after the timed steps")

    # End to end through the public API: every step copies its Q/K/V from pinned host memory to
    # the device, runs the whole path and copies O + LSE back to pinned host memory.  The steps
    # are pipelined the way a server would run them: two sets of device buffers, the inputs of
    # step i + 1 go up on a copy stream while step i computes, and step i's outputs come down on
    # a third stream; the timed region runs from the first upload to the last download.
    host, dev = run.host, run.dev
    run2 = Prefill(fpx, w, data, device)  # the second buffer set
    slots = (run, run2)
    host_o = [torch.empty(run.o.shape, dtype=run.o.dtype, pin_memory=True) for _ in range(2)]
    host_lse = [torch.empty(run.lse.shape, dtype=run.lse.dtype, pin_memory=True)
                for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    e2e_steps = max(3, args.steps)  # as many steps as the device-timed region
    for r in slots:  # warm both buffer sets
        r.step()
    torch.cuda.synchronize(device)
    done_compute, done_out = [None, None], [None, None]
    a, b = ev(), ev()
    a.record(s_in)
    for i in range(e2e_steps):
        r = slots[i % 2]
        with torch.cuda.stream(s_in):
            if done_compute[i % 2] is not None:  # step i - 2 has finished with these inputs
                s_in.wait_event(done_compute[i % 2])
            for k in ("q", "k", "v"):
                r.dev[k].copy_(host[k], non_blocking=True)
            up = ev()
            up.record(s_in)
        stream.wait_event(up)
        if done_out[i % 2] is not None:  # step i - 2's outputs have left these buffers
            stream.wait_event(done_out[i % 2])
        r.step()
        done_compute[i % 2] = ev()
        done_compute[i % 2].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(done_compute[i % 2])
            host_o[i % 2].copy_(r.o, non_blocking=True)
            host_lse[i % 2].copy_(r.lse, non_blocking=True)
            done_out[i % 2] = ev()
            done_out[i % 2].record(s_out)
    b.record(s_out)
    torch.cuda.synchronize(device)
    e2e_ms = a.elapsed_time(b) / e2e_steps
    for r in slots:
        r.check_status("after the end-to-end steps")
    h2d = sum(host[k].numel() * host[k].element_size() for k in host)
    d2h = host_o[0].numel() * host_o[0].element_size() + \
        host_lse[0].numel() * host_lse[0].element_size()
    del run2, slots

    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], device)
    ms_step = total_ms / args.steps
    flops = dense_flops(w)
    m = run.metrics(search_ms, attn_ms, n_kept)
    achieved = m["attn_executed_tflops"]
    peak_tf = m["attn_peak"]["tflops"]
    res = {
        "metric": METRIC,
        "value": round(aggregate_value(flops, world, ms_step), 3),
        "unit": "TFLOP/s (dense-equivalent causal attention, whole step)",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": w.dtype, "data": "synthetic (seeded generator: RoPE + sink + verticals + slash)",
        "config": config_of(w, world),
        "attn_ms": m["attn_ms"], "search_ms": m["search_ms"],
        "attn_dense_equiv_tflops": m["attn_dense_equiv_tflops"],
        "density": m["density"], "nnz": n_kept, "selection": run.selection(),
        "search_bytes": m["search_bytes"], "search_scores_readback_bytes": 4 * w.hq * pairs(w),
        "search_gbs": m["search_gbs"], "search_hbm_frac": m["search_hbm_frac"],
        "roofline": {"bound": "tensor", "kernel": "attn_tc_kernel", "achieved": achieved,
                     "peak": peak_tf, "unit": "TFLOP/s", "frac": round(achieved / peak_tf, 4),
                     "peak_kind": m["attn_peak"]["kind"],
                     "traffic": attn_traffic(w.name) if w.q_gain == 1.0 else None,
                     "traffic_unit": "bytes per launch (ncu dram read + write)",
                     "per_launch": "executed FLOP = 4*B^2*D*nnz (every kept 128x128 tile)"},
        "e2e": {"value": round(aggregate_value(flops, world, e2e_ms), 3),
                "unit": "TFLOP/s (dense-equivalent, host buffers, copies included)",
                "ms_per_step": round(e2e_ms, 3), "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "how": "pinned host Q/K/V up and O + LSE down every step, pipelined over two "
                       "device buffer sets and two copy streams"},
        "gpu_launches": KERNELS_PER_STEP * args.steps,
        "clocks": clk.summary(),
    }
    if not args.no_sdpa:
        res["sdpa_baseline"] = sdpa_baseline(w, dev, run.cu, device)
        res["extras"] = extras(fpx, w, run.pf, dev, run.cu, run.ws, run.scores, run.row_ptr,
                               run.col_idx, device)
    del run, host, dev
    torch.cuda.empty_cache()
    if world == 1 and not args.no_sub and args.workload == DEFAULT_WORKLOAD and \
            args.alpha is None and args.q_gain is None:
        sd = res.get("sdpa_baseline") or {}
        res["sub_records"] = sub_records(fpx, args, device, sd.get("ms"))
    return res, w, data


# ---------------------------------------------------------------------------------------------
# the oracle on the host cores (cpu_baseline leg and the reference arm)
# ---------------------------------------------------------------------------------------------

def oracle_sample(w, data, budget_s: float = 20.0):
    """Times the CPU oracle on a bounded sample of the workload: the pooled scores and the
    selection of one sequence x one head, then exact attention for whole query blocks of that
    head, last blocks first, until ~budget_s.  Returns (dense-equiv FLOP done, seconds, text)."""
    from gen import dequantised
    from oracle import fpx_oracle as O

    s_idx = int(np.argmax(w.seqlens))
    n = w.seqlens[s_idx]
    a = int(data["cu_seqlens"][s_idx])
    g = w.hq // w.hkv
    sl = slice(a, a + n)
    q = dequantised(data["q"][sl, :1], None if data["q_scale"] is None else data["q_scale"][:1])
    k = dequantised(data["k"][sl, :1], None if data["k_scale"] is None else data["k_scale"][:1])
    v = dequantised(data["v"][sl, :1], None if data["v_scale"] is None else data["v_scale"][:1])
    cu = np.array([0, n])
    t0 = time.perf_counter()
    sc = O.block_scores(q, k, cu, w.block)
    keeps, _ = O.select(sc, w.alpha, w.sink_blocks, w.window_blocks)
    rp, ci = O.to_csr(keeps)
    nb = keeps[0].shape[1]
    flop = 0.0
    done = 0
    for I in range(nb - 1, -1, -1):
        O.attention(q, k, v, cu, w.block, rp, ci, blocks=[(0, 0, I)])
        flop += sum(4.0 * w.d * (I * w.block + r + 1) for r in range(min(w.block, n - I * w.block)))
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    text = (f"sequence {s_idx} (N={n}), Q head 0 (KV head 0, group {g}): pooled scores + selection"
            f" of all {nb} query blocks, exact attention of the last {done} query blocks")
    return flop, dt, text


def cpu_cores() -> int:
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = max((x.get("num_threads", 1) for x in info), default=1)
        return int(n)
    except Exception:
        return os.cpu_count() or 1


def run_reference(args):
    w = WORKLOADS[args.workload]
    if args.alpha is not None:
        w = w.with_(alpha=args.alpha)
    data = generate(w, workers=default_workers())
    budget = max(2.0, 150.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_sample(w, data, budget)
    vals = []
    secs = []
    text = ""
    for _ in range(args.steps):
        flop, dt, text = oracle_sample(w, data, budget)
        vals.append(flop / dt / 1e12)
        secs.append(dt)
    v = statistics.mean(vals)
    unit = "TFLOP/s (dense-equivalent causal attention, whole step)"
    return {
        "impl": "reference", "metric": METRIC, "value": v, "unit": unit, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * statistics.mean(secs), 3),
        "ms_per_step_note": "wall time of one bounded oracle sample (see cpu_baseline.sample)",
        "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, 1),
        "cpu_baseline": {"value": v, "unit": unit, "cores": cpu_cores(), "kind": "oracle",
                         "sample": text},
        "e2e": {"value": v, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=None,
                    help="GPUs (one rank each); default: WORLD_SIZE under torchrun, else 1")
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--alpha", type=float, default=None)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sdpa", action="store_true",
                    help="skip the PyTorch SDPA baseline and the paged / rescue timings")
    ap.add_argument("--q-gain", type=float, default=None,
                    help="multiply Q by this gain (the labelled sparse-regime knob)")
    ap.add_argument("--no-sub", action="store_true",
                    help="skip the sub-records (sparse sweep, 32K, e4m3, varlen)")
    ap.add_argument("--sub-steps", type=int, default=5, help="timed steps per sub-record")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    if args.gpus is None:
        args.gpus = int(os.environ.get("WORLD_SIZE", "1"))
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        # one process per GPU: relaunch this command under torchrun on this node
        cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
               f"--nproc-per-node={args.gpus}", "--master-addr=127.0.0.1",
               f"--master-port={os.environ.get('MASTER_PORT', '29517')}",
               os.path.abspath(__file__)] + sys.argv[1:]
        import subprocess
        sys.exit(subprocess.call(cmd))
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world != args.gpus:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={world}: launch one rank per GPU")
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    local = int(os.environ.get("LOCAL_RANK", "0"))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    res, w, data = run_ours(args, rank, world, device)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        flop, dt, text = oracle_sample(w, data, 20.0)
        res["cpu_baseline"] = {"value": flop / dt / 1e12,
                               "unit": "TFLOP/s (dense-equivalent causal attention)",
                               "cores": cpu_cores(), "kind": "oracle", "sample": text,
                               "seconds": round(dt, 2)}
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
