"""Seeded synthetic MoE-layer workloads, shared by the CUDA path's tests/bench and the oracle.

This module only *draws numbers*: it holds the layer shapes, the value distributions and
the seeded random streams.  It contains none of the layer's arithmetic (no routing, no
softmax, no expert FFN), so both sides of a parity test can consume its arrays without
sharing any of the method.

Shapes follow the DeepSeekMoE configurations:
  * "DeepSeekMoE: Towards Ultimate Expert Specialization in Mixture-of-Experts Language
    Models" (deepforge.srivtx.xyz article), section "What the 16B configuration looks like":
    2 shared + 64 routed experts, 6 routed active, hidden 2048; at 145B 4 shared + 128 routed,
    12 routed active.
  * Same article, "Where this sits" / "Reading the evidence carefully": the 2B model is
    compared with GShard at equal total expert parameters (fine-grained m=4 segmentation).
The token counts, hidden sizes, intermediate widths, distributions and the Zipf router
skew of the 145B layer are the workload recipe chosen for this library (no trained
weights or datasets exist here):
  u ~ N(0, 1);  centroids e_i ~ N(0, variance 1/d) so logits are ~N(0, 1);
  expert weights ~ N(0, std 0.02);  seed 0;  PCG64 streams per tensor and expert.
bf16 configurations round the fp32 draws to bf16 (round-to-nearest-even) and keep the
raw 16-bit patterns; both sides widen those patterns exactly.
"""
from __future__ import annotations

import dataclasses
import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

__all__ = ["CONFIGS", "Workload", "make_workload", "f32_to_bf16_bits", "bf16_bits_to_f32",
           "zipf_logit_bias"]

# name -> (T, d, n_shared, n_routed, inter, top_k, dtype, alpha1, zipf_s)
CONFIGS: dict[str, dict] = {
    # tiny fp32 layer: runs through the fp32 SIMT path, oracle in well under a second
    "tiny": dict(T=128, d=256, n_shared=1, n_routed=15, inter=128, top_k=3,
                 dtype="fp32", alpha1=0.01, zipf_s=None),
    # DeepSeekMoE-2B-shaped layer
    "2b": dict(T=8192, d=1280, n_shared=1, n_routed=63, inter=896, top_k=7,
               dtype="bf16", alpha1=0.01, zipf_s=None),
    # GShard-style coarse layer with the same total expert parameters as "2b"
    "gshard": dict(T=8192, d=1280, n_shared=0, n_routed=16, inter=3584, top_k=2,
                   dtype="bf16", alpha1=0.01, zipf_s=None),
    # DeepSeekMoE-16B-shaped layer, prefill and decode token counts
    "16b_prefill": dict(T=16384, d=2048, n_shared=2, n_routed=64, inter=1408, top_k=6,
                        dtype="bf16", alpha1=0.001, zipf_s=None),
    "16b_decode": dict(T=64, d=2048, n_shared=2, n_routed=64, inter=1408, top_k=6,
                       dtype="bf16", alpha1=0.001, zipf_s=None),
    # 145B-shaped layer with a Zipf(1.1) per-expert router bias (skewed load)
    "145b": dict(T=32768, d=4096, n_shared=4, n_routed=128, inter=1536, top_k=12,
                 dtype="bf16", alpha1=0.001, zipf_s=1.1),
    # the 16B-shaped prefill layer with its gate/up GEMM on e4m3 operands (the library's
    # reduced-precision variant; same draws as "16b_prefill")
    "16b_prefill_e4m3": dict(T=16384, d=2048, n_shared=2, n_routed=64, inter=1408, top_k=6,
                             dtype="bf16", alpha1=0.001, zipf_s=None, gate_up_e4m3=True),
    # the same layer with both expert GEMMs on e4m3 operands
    "16b_prefill_e4m3_experts": dict(T=16384, d=2048, n_shared=2, n_routed=64, inter=1408,
                                     top_k=6, dtype="bf16", alpha1=0.001, zipf_s=None,
                                     gate_up_e4m3=True, down_e4m3=True),
}

_STREAMS = ("u", "centroids", "w_gate", "w_up", "w_down")


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return the 16-bit patterns.

    Inputs are finite draws; NaN/Inf are not produced by this module.
    """
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (b >> np.uint32(16)) & np.uint32(1)
    return ((b + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def zipf_logit_bias(n_routed: int, s: float) -> np.ndarray:
    """Per-expert router bias ln(p_i), p_i proportional to (i+1)^-s, normalised (float32).

    Workload structure for the skewed 145B-shaped layer: expert index = popularity rank.
    """
    p = np.arange(1, n_routed + 1, dtype=np.float64) ** (-float(s))
    p /= p.sum()
    return np.log(p).astype(np.float32)


@dataclasses.dataclass
class Workload:
    """One seeded layer instance.

    For dtype "bf16" the tensors hold uint16 bf16 bit patterns; for "fp32" float32 values.
    Layouts (row-major): u [T,d]; centroids [n_routed,d]; w_gate, w_up [G,inter,d];
    w_down [G,d,inter] with G = n_shared + n_routed and the shared experts first;
    logit_bias [n_routed] float32 or None.
    """
    name: str
    T: int
    d: int
    n_shared: int
    n_routed: int
    inter: int
    top_k: int
    dtype: str
    alpha1: float
    u: np.ndarray
    centroids: np.ndarray
    w_gate: np.ndarray
    w_up: np.ndarray
    w_down: np.ndarray
    logit_bias: np.ndarray | None
    gate_up_e4m3: bool = False     # bf16 layer whose gate/up products take e4m3 operands
    down_e4m3: bool = False        # ... and whose down products too (needs gate_up_e4m3)

    @property
    def n_experts(self) -> int:
        return self.n_shared + self.n_routed

    def spec(self) -> dict:
        return dict(T=self.T, d=self.d, n_shared=self.n_shared, n_routed=self.n_routed,
                    inter=self.inter, top_k=self.top_k, dtype=self.dtype, alpha1=self.alpha1,
                    gate_up_e4m3=self.gate_up_e4m3, down_e4m3=self.down_e4m3)


def _draw(seed_seq, shape, std: float, dtype: str) -> np.ndarray:
    x = np.random.Generator(np.random.PCG64(seed_seq)).standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return f32_to_bf16_bits(x) if dtype == "bf16" else x


_ROWS_PER_STREAM = 1024


def make_workload(name: str = "tiny", seed: int = 0, threads: int | None = None,
                  **overrides) -> Workload:
    """Draw the seeded inputs of a named configuration (fields may be overridden).

    Streams: SeedSequence(seed) spawns one child per tensor (u, centroids, w_gate, w_up,
    w_down); each weight tensor's child spawns one PCG64 stream per expert and u's child one
    stream per block of 1024 token rows.  Child i of a SeedSequence does not depend on how
    many children are spawned, so changing T keeps every weight and u's first rows
    identical, and the per-expert streams let the draws run on several threads.
    """
    spec = dict(CONFIGS[name]) if name in CONFIGS else {}
    spec.update(overrides)
    T, d, ks, nr = int(spec["T"]), int(spec["d"]), int(spec["n_shared"]), int(spec["n_routed"])
    inter, top_k, dtype = int(spec["inter"]), int(spec["top_k"]), spec["dtype"]
    g = ks + nr
    ss = dict(zip(_STREAMS, np.random.SeedSequence(seed).spawn(len(_STREAMS))))
    edt = np.uint16 if dtype == "bf16" else np.float32
    u = np.empty((T, d), dtype=edt)
    w_gate = np.empty((g, inter, d), dtype=edt)
    w_up = np.empty((g, inter, d), dtype=edt)
    w_down = np.empty((g, d, inter), dtype=edt)
    jobs = []
    n_chunks = (T + _ROWS_PER_STREAM - 1) // _ROWS_PER_STREAM
    for c, child in enumerate(ss["u"].spawn(n_chunks)):
        r0, r1 = c * _ROWS_PER_STREAM, min(T, (c + 1) * _ROWS_PER_STREAM)
        jobs.append((u, c, slice(r0, r1), child, (r1 - r0, d), 1.0))
    for name_, arr, shape in (("w_gate", w_gate, (inter, d)), ("w_up", w_up, (inter, d)),
                              ("w_down", w_down, (d, inter))):
        for e, child in enumerate(ss[name_].spawn(g)):
            jobs.append((arr, e, None, child, shape, 0.02))

    def run(job):
        arr, i, sl, child, shape, std = job
        x = _draw(child, shape, std, dtype)
        if sl is None:
            arr[i] = x
        else:
            arr[sl] = x

    n_thr = threads or min(32, os.cpu_count() or 1)
    with ThreadPoolExecutor(max_workers=n_thr) as ex:
        list(ex.map(run, jobs))
    cen = _draw(ss["centroids"], (nr, d), 1.0 / math.sqrt(d), dtype)
    zs = spec.get("zipf_s")
    bias = zipf_logit_bias(nr, zs) if zs else None
    return Workload(name=name, T=T, d=d, n_shared=ks, n_routed=nr, inter=inter, top_k=top_k,
                    dtype=dtype, alpha1=float(spec["alpha1"]), u=u, centroids=cen,
                    w_gate=w_gate, w_up=w_up, w_down=w_down, logit_bias=bias,
                    gate_up_e4m3=bool(spec.get("gate_up_e4m3", False)),
                    down_e4m3=bool(spec.get("down_e4m3", False)))
