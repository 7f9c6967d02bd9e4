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
# Gates g = s come from fp32 logits accumulated over d bf16 products; the accumulated
# rounding error of a logit grows like sqrt(d) (about 1e-5 absolute at d = 4096 for
# logits of unit scale), and a logit error e shifts s by a relative e (plus the same
# through the softmax denominator).  Hence 1e-5 relative up to d = 1024, scaled with d.
GATE_RTOL = 1e-5
AUX_RTOL = 1e-4
NEAR_TIE = 1e-6


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


def compare(w, g: GpuOut, rows=None, report: dict | None = None) -> dict:
    """Assert parity of every output; returns a report dict (excluded tokens, errors)."""
    ref = O.moe_forward(w.u, w.centroids, w.w_gate, w.w_up, w.w_down, w.n_shared, w.top_k,
                        w.alpha1, bias=w.logit_bias, rows=rows,
                        gate_up_e4m3=getattr(w, "gate_up_e4m3", False))
    r = ref.routing
    T, K, nr = w.T, w.top_k, w.n_routed
    rep = report if report is not None else {}
    excl = O.near_tie_tokens(r.s, K, NEAR_TIE)
    keep = ~excl
    rep["excluded_tokens"] = int(excl.sum())

    # --- routing: every token has K distinct valid indices
    gi = g.topk_idx
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
    # gates: g = s at the chosen experts, not renormalised
    gate_rtol = GATE_RTOL * max(1.0, w.d / 1024)
    np.testing.assert_allclose(g.topk_w, s_at, rtol=gate_rtol, atol=1e-7 * np.abs(s_at).max())

    # --- counts: the GPU histogram of its own indices, and the oracle's on kept tokens
    own = np.bincount(gi.reshape(-1), minlength=nr)
    np.testing.assert_array_equal(g.counts, own)
    np.testing.assert_array_equal(np.bincount(gi[keep].reshape(-1), minlength=nr),
                                  np.bincount(r.topk_idx[keep].reshape(-1), minlength=nr))
    if rep["excluded_tokens"] == 0:
        np.testing.assert_array_equal(g.counts, ref.counts)
    # --- balance loss with the GPU's own counts (equal to the oracle's when nothing is
    # excluded) and the oracle's mean affinities
    aux_ref = w.alpha1 * float(np.sum((g.counts / T) * ref.P))
    assert abs(g.aux - aux_ref) <= AUX_RTOL * abs(aux_ref) + 1e-12, (g.aux, aux_ref)
    rep["aux_gpu"], rep["aux_ref"] = g.aux, ref.aux

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
