"""Seeded synthetic prefill inputs (Q, K, V) for dynamic block-sparse prefill attention.

This module only *draws inputs*.  It holds none of the method's arithmetic (no pooling,
scoring, thresholding or attention) and is the one piece of code that both the CPU oracle
and the CUDA path consume.

Recipe (one "layer" of a causal prefill, packed THD layout):

* Shapes are those of the attention-layer workloads the FlashPrefill summary evaluates on
  (paperlayer.ai, "FlashPrefill: Instantaneous Pattern Discovery and Thresholding ...",
  §4 Experiments; block 128 from App. A).  Real-model activations are not available, so the
  structure real prefill attention shows -- attention sinks, vertical columns and a local
  slash band (§1 Introduction, §3 Instantaneous Pattern Discovery) -- is planted into
  Gaussian noise.
* Per sequence ``s`` (seed ``seed + s``) and per KV head ``g`` an independent PCG64 stream
  ``default_rng(SeedSequence(seed + s, spawn_key=(g,)))`` draws, in this order:
  K[N, D], V[N, D], Q[group, N, D] (all N(0,1)/sqrt(D)), a sink direction u (unit),
  a vertical direction w (unit, Gram-Schmidt orthogonal to u) and the vertical column
  positions (``round(frac * N)`` distinct tokens, drawn without replacement).
* RoPE (theta = 1e4, rotate-half pairing d <-> d + D/2, positions restart at 0 in every
  sequence) is applied to Q and K.
* After RoPE, in this order: the slash band (optional): k'_j = 0.5 k_j + 0.5 mean(k_{j-64..j-1})
  over the pre-mix rows with the window clipped at token 0 (k'_0 = k_0); the sink: K tokens
  0..3 get +3u and every Q of the group gets +1u; the verticals: the chosen K rows get +2.5w and
  every Q of the group gets +0.8w.  V carries no structure.
* Storage dtype: fp32 as drawn; bf16 by round-to-nearest-even; fp8-e4m3 per head with
  scale = absmax / 448 (1 when absmax == 0), x / scale rounded to nearest even and saturated.

An optional ``q_gain`` multiplies Q after the structure is planted (a supplementary knob that
emulates the larger logit scale of trained models; 1.0 = the recipe above).
"""
from __future__ import annotations

import concurrent.futures as _cf
import dataclasses
import os
from typing import Dict, List, Optional, Sequence

import numpy as np
import torch

ROPE_THETA = 1.0e4
SLASH_WINDOW = 64
SINK_TOKENS = 4
SINK_K_GAIN, SINK_Q_GAIN = 3.0, 1.0
VERT_K_GAIN, VERT_Q_GAIN = 2.5, 0.8
E4M3_MAX = 448.0


@dataclasses.dataclass(frozen=True)
class Workload:
    """One prefill workload: shapes, generator knobs and the selection parameters."""

    name: str
    seqlens: tuple            # tokens per packed sequence
    hq: int
    hkv: int
    d: int
    block: int
    dtype: str                # "f32" | "bf16" | "e4m3"
    alpha: float
    vertical_frac: float = 0.01
    slash: bool = True
    seed: int = 0
    q_gain: float = 1.0
    sink_blocks: int = 1
    window_blocks: int = 1

    @property
    def total_tokens(self) -> int:
        return int(sum(self.seqlens))

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five prefill workloads the measurements and parity tests run on.
WORKLOADS: Dict[str, Workload] = {
    # tiny single-layer causal prefill, fp32, no slash band
    "tiny_fp32_n2048": Workload("tiny_fp32_n2048", (2048,), 2, 1, 64, 64, "f32", 0.1,
                                vertical_frac=0.01, slash=False),
    # Llama-3-8B-shaped layer (GQA 4)
    "llama8b_bf16_n8192": Workload("llama8b_bf16_n8192", (8192,), 32, 8, 128, 128, "bf16", 0.1),
    "llama8b_bf16_n32768": Workload("llama8b_bf16_n32768", (32768,), 32, 8, 128, 128, "bf16", 0.1),
    "llama8b_bf16_n131072": Workload("llama8b_bf16_n131072", (131072,), 32, 8, 128, 128, "bf16",
                                     0.1, vertical_frac=0.002),
    "llama8b_e4m3_n131072": Workload("llama8b_e4m3_n131072", (131072,), 32, 8, 128, 128, "e4m3",
                                     0.1, vertical_frac=0.002),
    # the e4m3 layer at 32K tokens (its Q + K + V, 200 MB, still exceed L2): kernel captures
    "llama8b_e4m3_n32768": Workload("llama8b_e4m3_n32768", (32768,), 32, 8, 128, 128, "e4m3", 0.1),
    # packed varlen batch of eight sequences (continuous-batching shape)
    "varlen8_bf16_t264192": Workload("varlen8_bf16_t264192",
                                     (4096, 8192, 16384, 65536, 2048, 32768, 4096, 131072),
                                     32, 8, 128, 128, "bf16", 0.1),
}


def cu_seqlens_of(seqlens: Sequence[int]) -> np.ndarray:
    cu = np.zeros(len(seqlens) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(np.asarray(seqlens, dtype=np.int64))
    return cu


def _rope(x: np.ndarray) -> np.ndarray:
    """Rotate-half RoPE over the last axis; positions are axis -2 (0..N-1)."""
    n, d = x.shape[-2], x.shape[-1]
    half = d // 2
    inv = ROPE_THETA ** (-np.arange(half, dtype=np.float64) * 2.0 / d)
    ang = np.arange(n, dtype=np.float64)[:, None] * inv[None, :]
    cos = np.cos(ang).astype(np.float32)
    sin = np.sin(ang).astype(np.float32)
    x1, x2 = x[..., :half], x[..., half:]
    out = np.empty_like(x)
    out[..., :half] = x1 * cos - x2 * sin
    out[..., half:] = x2 * cos + x1 * sin
    return out


def _slash_band(k: np.ndarray) -> np.ndarray:
    """k'_j = 0.5 k_j + 0.5 * mean of the (up to) 64 preceding pre-mix rows; k'_0 = k_0."""
    n = k.shape[0]
    csum = np.zeros((n + 1, k.shape[1]), dtype=np.float64)
    np.cumsum(k, axis=0, dtype=np.float64, out=csum[1:])
    j = np.arange(n)
    lo = np.maximum(j - SLASH_WINDOW, 0)
    cnt = (j - lo).astype(np.float64)
    out = k.copy()
    m = j >= 1
    mean = (csum[j[m]] - csum[lo[m]]) / cnt[m][:, None]
    out[m] = (0.5 * k[m] + 0.5 * mean).astype(np.float32)
    return out


def _unit(v: np.ndarray) -> np.ndarray:
    n = float(np.linalg.norm(v))
    return v / n if n > 0 else v


def _gen_group(args):
    """Draw one (sequence, KV head) group: returns (K[N,D], V[N,D], Q[g,N,D]) fp32."""
    seed_s, kvh, n, g, d, frac, slash, q_gain = args
    rng = np.random.default_rng(np.random.SeedSequence(seed_s, spawn_key=(kvh,)))
    inv_sqrt_d = np.float32(1.0 / np.sqrt(d))
    k = rng.standard_normal((n, d), dtype=np.float32) * inv_sqrt_d
    v = rng.standard_normal((n, d), dtype=np.float32) * inv_sqrt_d
    q = rng.standard_normal((g, n, d), dtype=np.float32) * inv_sqrt_d
    u = _unit(rng.standard_normal(d))
    w = rng.standard_normal(d)
    w = _unit(w - np.dot(w, u) * u)
    nvert = int(round(frac * n))
    vert = rng.choice(n, size=nvert, replace=False) if nvert > 0 else np.zeros(0, np.int64)
    if n == 0:
        return k, v, q
    k = _rope(k)
    q = _rope(q)
    if slash:
        k = _slash_band(k)
    u32, w32 = u.astype(np.float32), w.astype(np.float32)
    k[:min(SINK_TOKENS, n)] += np.float32(SINK_K_GAIN) * u32
    q += np.float32(SINK_Q_GAIN) * u32
    if nvert:
        k[vert] += np.float32(VERT_K_GAIN) * w32
    q += np.float32(VERT_Q_GAIN) * w32
    if q_gain != 1.0:
        q *= np.float32(q_gain)
    return k, v, q


def _quant_e4m3(x: torch.Tensor, heads_axis: int = 1):
    """Per-head e4m3 quantisation: scale_h = absmax_h / 448 (1 if 0); returns (codes, scales)."""
    xt = x.movedim(heads_axis, 0)
    amax = xt.reshape(xt.shape[0], -1).abs().amax(dim=1).to(torch.float32) if xt.numel() else \
        torch.zeros(xt.shape[0], dtype=torch.float32)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    shape = [1] * x.dim()
    shape[heads_axis] = -1
    y = (x / scale.view(shape)).clamp_(-E4M3_MAX, E4M3_MAX)
    return y.to(torch.float8_e4m3fn), scale


def generate(w: Workload, workers: int = 0) -> dict:
    """Materialise a workload as CPU tensors in packed THD layout.

    Returns dict(q, k, v: torch tensors [T, H, D] in the storage dtype; q_scale/k_scale/v_scale
    (fp32 [H], e4m3 only, else None); cu_seqlens: int32 numpy [S+1]; workload: w).
    ``workers`` > 1 draws the (sequence, KV head) groups on that many threads (numpy releases
    the GIL inside the array work); every group has its own stream, so the result is the same.
    """
    g = w.hq // w.hkv
    cu = cu_seqlens_of(w.seqlens)
    t = int(cu[-1])
    q = torch.empty((t, w.hq, w.d), dtype=torch.float32)
    k = torch.empty((t, w.hkv, w.d), dtype=torch.float32)
    v = torch.empty((t, w.hkv, w.d), dtype=torch.float32)
    jobs = []
    for s, n in enumerate(w.seqlens):
        for kvh in range(w.hkv):
            jobs.append((w.seed + s, kvh, int(n), g, w.d, w.vertical_frac, w.slash, w.q_gain))

    def place(job, res):
        seed_s, kvh, n = job[0], job[1], job[2]
        s = seed_s - w.seed
        a, b = int(cu[s]), int(cu[s + 1])
        kk, vv, qq = res
        k[a:b, kvh] = torch.from_numpy(kk)
        v[a:b, kvh] = torch.from_numpy(vv)
        q[a:b, kvh * g:(kvh + 1) * g] = torch.from_numpy(np.ascontiguousarray(qq.transpose(1, 0, 2)))

    if workers and workers > 1 and len(jobs) > 1:
        with _cf.ThreadPoolExecutor(max_workers=min(workers, len(jobs))) as ex:
            for job, res in zip(jobs, ex.map(_gen_group, jobs)):
                place(job, res)
    else:
        for job in jobs:
            place(job, _gen_group(job))

    out = dict(workload=w, cu_seqlens=cu, q_scale=None, k_scale=None, v_scale=None)
    if w.dtype == "f32":
        out.update(q=q, k=k, v=v)
    elif w.dtype == "bf16":
        out.update(q=q.to(torch.bfloat16), k=k.to(torch.bfloat16), v=v.to(torch.bfloat16))
    elif w.dtype == "e4m3":
        q8, qs = _quant_e4m3(q)
        k8, ks = _quant_e4m3(k)
        v8, vs = _quant_e4m3(v)
        out.update(q=q8, k=k8, v=v8, q_scale=qs, k_scale=ks, v_scale=vs)
    else:
        raise ValueError(f"unknown dtype {w.dtype}")
    return out


def dequantised(x: torch.Tensor, scale: Optional[torch.Tensor]) -> np.ndarray:
    """Exact fp64 values that a stored tensor [T, H, D] represents (codes x per-head scale)."""
    a = x.to(torch.float64)
    if scale is not None:
        a = a * scale.to(torch.float64).view(1, -1, 1)
    return a.numpy()


def default_workers() -> int:
    return max(1, min(16, (os.cpu_count() or 1)))
