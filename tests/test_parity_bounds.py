"""The gate tolerance of the parity tests, checked on the CPU.

tests/parity.gate_error_bound bounds |g_gpu / s - 1| from the order in which each router
kernel accumulates its fp32 logits.  Here each of the three orders is emulated in fp32 with
NumPy (every accumulation step rounded explicitly: to nearest, and, for the tensor-core
model whose rounding direction the PTX ISA leaves open, also toward zero), followed by the
fp32 softmax; the emulated gates must stay inside the bound, and the bound must be tight
enough that a plausible mistake in the gates (renormalising them, taking the neighbouring
expert's affinity) fails it.
"""
import numpy as np
import pytest

from mixture_experts_layer_65_b200 import workloads as W
from oracle import moe_oracle as O
from tests import parity as P


def _round_f32(x: np.ndarray, toward_zero: bool) -> np.ndarray:
    y = x.astype(np.float32)
    if toward_zero:
        over = np.abs(y.astype(np.float64)) > np.abs(x)
        y = np.where(over, np.nextafter(y, np.float32(0)), y)
    return y


def _emulate_logits(w, path: str, toward_zero: bool = False) -> np.ndarray:
    """fp32 logits in the accumulation order of router `path` (before the bias)."""
    u, e = O.widen(w.u), O.widen(w.centroids)
    T, d = u.shape
    N = e.shape[0]
    if path == "mma16":
        acc = np.zeros((T, N), np.float32)
        for j in range(d // 16):
            step = u[:, 16 * j:16 * j + 16] @ e[:, 16 * j:16 * j + 16].T     # exact products
            acc = _round_f32(acc.astype(np.float64) + step, toward_zero)
        return acc.astype(np.float64)
    if path == "lanes":
        nv = d // 8
        lane = np.zeros((T, N, 32), np.float32)
        for l in range(32):
            for v in range(l, nv, 32):
                for k in range(8 * v, 8 * v + 8):
                    p = u[:, None, k] * e[None, :, k]
                    lane[:, :, l] = _round_f32(lane[:, :, l].astype(np.float64) + p, False)
        vals = lane
        for m in (16, 8, 4, 2, 1):     # xor butterfly: lane l adds lane l ^ m
            vals = _round_f32(vals.astype(np.float64) +
                              vals[:, :, np.arange(32) ^ m].astype(np.float64), False)
        return vals[:, :, 0].astype(np.float64)
    acc = np.zeros((T, N), np.float32)
    for k in range(d):
        acc = _round_f32(acc.astype(np.float64) + u[:, None, k] * e[None, :, k], False)
    return acc.astype(np.float64)


def _emulate_gates(w, logits32: np.ndarray, idx: np.ndarray) -> np.ndarray:
    b = np.zeros(w.n_routed) if w.logit_bias is None else O.widen(w.logit_bias)
    L = (logits32 + b).astype(np.float32)
    x = (L - L.max(axis=1, keepdims=True)).astype(np.float32)
    ex = np.exp(x)                                         # float32 exp
    den = ex.sum(axis=1, keepdims=True, dtype=np.float32)
    g = (ex * (np.float32(1) / den)).astype(np.float32)
    return np.take_along_axis(g, idx, axis=1).astype(np.float64)


CASES = [
    ("mma16", dict(T=48, d=512, n_routed=64, top_k=6, dtype="bf16"), False),
    ("mma16", dict(T=16, d=512, n_routed=200, top_k=8, dtype="bf16"), True),    # wide rows
    ("mma16", dict(T=48, d=512, n_routed=64, top_k=6, dtype="bf16"), True),
    ("mma16", dict(T=32, d=1024, n_routed=16, top_k=2, dtype="bf16", zipf_s=1.1), True),
    ("lanes", dict(T=16, d=384, n_routed=64, top_k=6, dtype="bf16"), False),
    ("fma_seq", dict(T=40, d=256, n_routed=15, top_k=3, dtype="fp32"), False),
]


@pytest.mark.parametrize("path,spec,toward_zero", CASES,
                         ids=[f"{c[0]}-d{c[1]['d']}-{'rz' if c[2] else 'rn'}" for c in CASES])
def test_emulated_fp32_router_stays_inside_the_gate_bound(path, spec, toward_zero):
    w = W.make_workload("16b_prefill", n_shared=0, inter=64, **spec)
    r = O.route(w.u, w.centroids, w.top_k, w.logit_bias)
    l32 = _emulate_logits(w, path, toward_zero)
    B = P.logit_error_bound(w, path)
    assert np.all(np.abs(l32 - O.router_logits(w.u, w.centroids)) <= B)
    g = _emulate_gates(w, l32, r.topk_idx)
    s_at = r.topk_w
    bound = P.gate_error_bound(w, r.logits, r.topk_idx, path)
    rel = np.abs(g - s_at) / s_at
    assert np.all(rel <= bound)
    assert (rel / bound).max() > 0.01          # the bound is not vacuous
    # plausible mistakes fail it: renormalised gates, the neighbouring expert's affinity
    renorm = s_at / s_at.sum(axis=1, keepdims=True)
    assert np.any(np.abs(renorm - s_at) / s_at > bound)
    nb = np.take_along_axis(r.s, (r.topk_idx + 1) % w.n_routed, axis=1)
    assert np.any(np.abs(nb - s_at) / s_at > bound)


def test_router_path_follows_the_library_dispatch():
    assert P.router_path(W.make_workload("tiny")) == "fma_seq"
    assert P.router_path(W.make_workload("16b_decode", T=8)) == "lanes"
    assert P.router_path(W.make_workload("16b_prefill", T=129, d=256, n_shared=1, n_routed=16,
                                         inter=64, top_k=4)) == "mma16"
    # d % 128 != 0 keeps small batches on the tensor-core router, and so does e4m3 gate/up
    assert P.router_path(W.make_workload("16b_prefill", T=64, d=320, n_shared=1, n_routed=16,
                                         inter=64, top_k=4)) == "mma16"
    assert P.router_path(W.make_workload("16b_prefill", T=64, d=256, n_shared=1, n_routed=16,
                                         inter=64, top_k=4, gate_up_e4m3=True)) == "mma16"
