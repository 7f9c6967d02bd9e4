"""Comparison of the CUDA path's outputs with the fp64 oracle (test helper)."""
from __future__ import annotations

import dataclasses

import numpy as np

from oracle import moe_oracle as O

# Tolerances: max|h - h_ref| <= TOL * max|h_ref| (bf16 and fp32 layers).
TOL = {"bf16": 2e-2, "fp32": 1e-4}
# The expert part (h - u) is also checked against max|h_ref - u| with the same factor
# (after discounting the output's own rounding), so the residual cannot hide an error in
# the experts.
# Gates g = s at the chosen experts are checked against a bound derived per gate from the
# way the router kernel that ran accumulates its fp32 logits (gate_error_bound).
AUX_RTOL = 1e-4
NEAR_TIE = 1e-6
U24 = 2.0 ** -24          # unit roundoff of fp32 (round to nearest)
U23 = 2.0 ** -23          # one fp32 ulp of a value in [1, 2): covers any rounding direction
SMALL_BATCH_MAX_T = 128   # the library's SIMT router runs bf16 batches up to this size


@dataclasses.dataclass
class GpuOut:
    h: np.ndarray          # float64 [T, d]
    topk_idx: np.ndarray   # int64 [T, K]
    topk_w: np.ndarray     # float64 [T, K]
    counts: np.ndarray     # int64 [N_r]
    aux: float


def fetch(out) -> GpuOut:
    return GpuOut(h=out.h.float().cpu().numpy().astype(np.float64),
                  topk_idx=out.topk_idx.cpu().numpy().astype(np.int64),
                  topk_w=out.topk_w.cpu().numpy().astype(np.float64),
                  counts=out.expert_counts.cpu().numpy().astype(np.int64),
                  aux=float(out.aux_loss.cpu().numpy()[0]))


def sample_rows(T: int, n: int = 256, seed: int = 1) -> np.ndarray:
    """Rows checked at full size: both ends, the last (possibly ragged) tile, a random set."""
    rng = np.random.default_rng(seed)
    fixed = [0, 1, 127, 128, T // 2, T - 129, T - 2, T - 1]
    pick = rng.choice(T, size=min(n, T), replace=False)
    rows = np.unique(np.clip(np.concatenate([fixed, pick]), 0, T - 1))
    return rows


# ------------------------------------------------------------------ the gates' error bound
def router_path(w) -> str:
    """Which router kernel computes layer w's logits (the library's dispatch rule):
    'fma_seq' for fp32 layers (one fp32 FMA per element, k in order); 'lanes' for bf16
    batches of at most 128 tokens with d % 128 == 0 (each lane of a warp an FMA chain over
    its 8-element vectors, then a five-level butterfly of adds); 'mma16' for every other
    bf16 layer (tensor-core MMAs of K = 16 in k order into an fp32 accumulator)."""
    if w.dtype != "bf16":
        return "fma_seq"
    if not getattr(w, "gate_up_e4m3", False) and w.T <= SMALL_BATCH_MAX_T and w.d % 128 == 0:
        return "lanes"
    return "mma16"


def _mma16_bound(u, e, block=512):
    """U23 * sum over the d/16 MMA steps of (|running sum before the step| + sum of the
    |products| the step adds).  Model: an MMA adds 16 bf16 products (exact in fp32) to the
    fp32 accumulator and rounds the result once, to within one ulp of the magnitudes it
    adds, whatever the rounding direction (the PTX ISA leaves it unspecified)."""
    T, d = u.shape
    nch = d // 16
    e3 = e.reshape(e.shape[0], nch, 16).transpose(1, 2, 0)             # [nch, 16, N]
    abs_et = np.abs(e).T
    out = np.empty((T, e.shape[0]))
    for t0 in range(0, T, block):
        ub = u[t0:t0 + block]
        u3 = ub.reshape(-1, nch, 16).transpose(1, 0, 2)                   # [nch, n, 16]
        s = np.cumsum(np.matmul(u3, e3), axis=0)                          # running sums
        out[t0:t0 + block] = U23 * (np.abs(s[:-1]).sum(axis=0) + np.abs(ub) @ abs_et)
    return out


def _lanes_bound(u, e, block=32):
    """Lane l runs fmaf over the elements of its 16-byte vectors l, l+32, ... (8 each, in
    order; one rounding to nearest per FMA), then the 32 lane sums meet in a butterfly of
    xor-shuffle adds (offsets 16, 8, 4, 2, 1); every distinct node of the butterfly feeds
    lane 0's result, each with one rounding to nearest."""
    T, d = u.shape
    nv, N = d // 8, e.shape[0]
    lanes = [np.concatenate([np.arange(8 * v, 8 * v + 8) for v in range(l, nv, 32)])
             if l < nv else np.zeros(0, dtype=np.int64) for l in range(32)]
    out = np.empty((T, N))
    for t0 in range(0, T, block):
        ub = u[t0:t0 + block]
        lane_sum = np.zeros((ub.shape[0], N, 32))
        err = np.zeros((ub.shape[0], N))
        for l, idx in enumerate(lanes):
            if idx.size == 0:
                continue
            s = np.cumsum(ub[:, None, idx] * e[None, :, idx], axis=2)
            err += U24 * np.abs(s).sum(axis=2)
            lane_sum[:, :, l] = s[:, :, -1]
        vals = lane_sum
        for m in (16, 8, 4, 2, 1):
            vals = vals[:, :, :m] + vals[:, :, m:2 * m]
            err += U24 * np.abs(vals).sum(axis=2)
        out[t0:t0 + block] = err
    return out


def _fma_seq_bound(u, e, block=64):
    """One fmaf per element in k order, each rounding once to nearest."""
    T = u.shape[0]
    out = np.empty((T, e.shape[0]))
    for t0 in range(0, T, block):
        s = np.cumsum(u[t0:t0 + block, None, :] * e[None, :, :], axis=2)
        out[t0:t0 + block] = U24 * np.abs(s).sum(axis=2)
    return out


def logit_error_bound(w, path: str | None = None) -> np.ndarray:
    """[T, N_r] bound on |fp32 logit - exact logit| (before the bias) for router `path`."""
    u, e = O.widen(w.u), O.widen(w.centroids)
    path = path or router_path(w)
    if path == "mma16":
        return _mma16_bound(u, e)
    if path == "lanes":
        return _lanes_bound(u, e)
    return _fma_seq_bound(u, e)


def gate_error_bound(w, logits: np.ndarray, idx: np.ndarray, path: str | None = None) -> np.ndarray:
    """[T, K] bound on |g_gpu / s - 1| at the chosen experts `idx` (s the exact affinity,
    `logits` the exact logits with the bias).

    The kernels form g = fl(exp(x_i) * fl(1 / sum_j exp(x_j))) with x_j = fl(fl(l_j + b_j)
    - max).  The max cancels in the ratio, so the relative error of g is at most the
    perturbation of x_i plus the largest perturbation of any x_j (each: the accumulation
    bound of the logit, the bias add and the subtraction, half an ulp each), plus the error
    of the fast exponential at x_i and at the worst x_j (2 + 1.2 |x| ulp, its documented
    accuracy), plus N_pad/8 + 5 roundings: the denominator's sum (each of the row's 8
    threads adds its N_pad/8 columns, then a tree of three adds), its reciprocal and the
    product.  First order; the factor 1.01 covers the higher-order terms.
    """
    B = logit_error_bound(w, path)
    x = logits - logits.max(axis=1, keepdims=True)
    per = B + U24 * (np.abs(logits) + np.abs(x)) + U23 * (2.0 + 1.2 * np.abs(x))
    n_pad = (w.n_routed + 15) // 16 * 16
    worst = per.max(axis=1, keepdims=True)
    return 1.01 * (np.take_along_axis(per, idx, axis=1) + worst + U24 * (n_pad // 8 + 5))


# ------------------------------------------------------------------ comparisons
def compare_routing(w, r, topk_idx, topk_w, counts, aux, P_ref, rep: dict,
                    path: str | None = None) -> np.ndarray:
    """Routing outputs against the oracle's routing `r`; returns the kept-token mask."""
    T, K, nr = w.T, w.top_k, w.n_routed
    excl = O.near_tie_tokens(r.s, K, NEAR_TIE)
    keep = ~excl
    rep["excluded_tokens"] = int(excl.sum())

    # every token has K distinct valid indices
    gi = topk_idx
    assert gi.shape == (T, K)
    assert gi.min() >= 0 and gi.max() < nr, "routed index out of range"
    srt = np.sort(gi, axis=1)
    assert np.all(np.diff(srt, axis=1) > 0), "duplicate routed index for a token"
    # sets bit-exact on non-near-tie tokens
    ref_sets = np.sort(r.topk_idx, axis=1)
    bad = np.nonzero(np.any(srt != ref_sets, axis=1) & keep)[0]
    assert bad.size == 0, f"routed sets differ on {bad.size} tokens, first {bad[:5].tolist()}"
    # order: descending oracle affinity up to the near-tie margin
    s_at = np.take_along_axis(r.s, gi, axis=1)
    assert np.all(s_at[:, :-1] >= s_at[:, 1:] - NEAR_TIE), "routed order not descending"
    # gates: g = s at the chosen experts (not renormalised), within the rounding bound
    bound = gate_error_bound(w, r.logits, gi, path)
    rel = np.abs(topk_w - s_at) / s_at
    worst = np.unravel_index(np.argmax(rel / bound), rel.shape)
    rep["gate_rel_err"] = float(rel.max())
    rep["gate_err_over_bound"] = float((rel / bound).max())
    assert np.all(rel <= bound), (
        f"gate error {rel[worst]:.3e} above its bound {bound[worst]:.3e} at token {worst[0]}")

    # counts: the GPU histogram of its own indices, and the oracle's on kept tokens
    own = np.bincount(gi.reshape(-1), minlength=nr)
    np.testing.assert_array_equal(counts, own)
    np.testing.assert_array_equal(np.bincount(gi[keep].reshape(-1), minlength=nr),
                                  np.bincount(r.topk_idx[keep].reshape(-1), minlength=nr))
    if rep["excluded_tokens"] == 0:
        np.testing.assert_array_equal(counts, np.bincount(r.topk_idx.reshape(-1), minlength=nr))
    # balance loss with the GPU's own counts (equal to the oracle's when nothing is
    # excluded) and the oracle's mean affinities
    aux_ref = w.alpha1 * float(np.sum((counts / T) * P_ref))
    assert abs(aux - aux_ref) <= AUX_RTOL * abs(aux_ref) + 1e-12, (aux, aux_ref)
    rep["aux_gpu"] = aux
    return keep


def compare(w, g: GpuOut, rows=None, report: dict | None = None) -> dict:
    """Assert parity of every output; returns a report dict (excluded tokens, errors)."""
    ref = O.moe_forward(w.u, w.centroids, w.w_gate, w.w_up, w.w_down, w.n_shared, w.top_k,
                        w.alpha1, bias=w.logit_bias, rows=rows,
                        gate_up_e4m3=getattr(w, "gate_up_e4m3", False),
                        down_e4m3=getattr(w, "down_e4m3", False))
    rep = report if report is not None else {}
    keep = compare_routing(w, ref.routing, g.topk_idx, g.topk_w, g.counts, g.aux, ref.P, rep)
    rep["aux_ref"] = ref.aux

    # --- outputs on the chosen rows, skipping near-tie tokens
    hr = ref.h
    hg = g.h[ref.rows]
    ok_rows = keep[ref.rows]
    u64 = O.widen(w.u)[ref.rows]
    tol = TOL[w.dtype]
    diff = np.abs(hg[ok_rows] - hr[ok_rows])
    scale = np.abs(hr[ok_rows]).max()
    err = float(diff.max()) / scale if diff.size else 0.0
    # expert part, after discounting the final rounding of h itself (half an ulp of the
    # output type, 2^-8 |h| for bf16 and 2^-24 |h| for fp32)
    eps_out = 2.0 ** -8 if w.dtype == "bf16" else 2.0 ** -24
    ffn_ref = hr[ok_rows] - u64[ok_rows]
    slack = eps_out * np.maximum(np.abs(hr[ok_rows]), np.abs(hg[ok_rows]))
    ffn_err = float(np.maximum(diff - slack, 0.0).max()) / max(
        float(np.abs(ffn_ref).max()), 1e-30) if diff.size else 0.0
    rep["h_rel_err"], rep["ffn_rel_err"] = err, ffn_err
    assert err <= tol, f"max|h - h_ref| / max|h_ref| = {err:.3e} > {tol}"
    assert ffn_err <= tol, f"expert-part relative error {ffn_err:.3e} > {tol}"
    return rep
