"""Pins of the oracle's backward pass (CPU only).

The gradients are checked against central finite differences of the forward oracle (the
forward is itself pinned in test_oracle.py), so a dropped term, a wrong sign or a transposed
operand anywhere in the backward shows up as a mismatch; the structural invariants below
(softmax rows, a single expert, segmentation, linearity) pin the same code from other sides.
"""
import numpy as np
import pytest

from mixture_experts_layer_65_b200 import workloads as W
from oracle import moe_oracle as O


def _layer(T=12, d=16, n_shared=1, n_routed=6, inter=8, top_k=2, seed=3, zipf=False):
    w = W.make_workload("tiny", T=T, d=d, n_shared=n_shared, n_routed=n_routed, inter=inter,
                        top_k=top_k, seed=seed)
    # larger weights than the workloads' 0.02 so every term of the gradient is sizeable
    p = dict(u=O.widen(w.u), centroids=O.widen(w.centroids) * 4.0,
             w_gate=O.widen(w.w_gate) * 25.0, w_up=O.widen(w.w_up) * 25.0,
             w_down=O.widen(w.w_down) * 25.0,
             bias=(W.zipf_logit_bias(n_routed, 1.1).astype(np.float64) if zipf
                   else np.zeros(n_routed)))
    return p, dict(n_shared=n_shared, top_k=top_k, alpha1=0.3)


def _loss(p, cfg, dh, d_aux):
    out = O.moe_forward(p["u"], p["centroids"], p["w_gate"], p["w_up"], p["w_down"],
                        cfg["n_shared"], cfg["top_k"], cfg["alpha1"], bias=p["bias"])
    return float(np.sum(dh * out.h)) + d_aux * out.aux, out.routing.topk_idx


def _grads(p, cfg, dh, d_aux):
    return O.moe_backward(p["u"], p["centroids"], p["w_gate"], p["w_up"], p["w_down"],
                          cfg["n_shared"], cfg["top_k"], cfg["alpha1"], dh, d_aux=d_aux,
                          bias=p["bias"])


GRAD_OF = {"u": "du", "centroids": "d_centroids", "bias": "d_bias", "w_gate": "d_w_gate",
           "w_up": "d_w_up", "w_down": "d_w_down"}


@pytest.mark.parametrize("zipf", [False, True], ids=["no_bias", "zipf_bias"])
@pytest.mark.parametrize("d_aux", [0.0, 1.7])
def test_gradients_match_central_differences(zipf, d_aux):
    p, cfg = _layer(zipf=zipf)
    rng = np.random.default_rng(11)
    dh = rng.standard_normal(p["u"].shape)
    g = _grads(p, cfg, dh, d_aux)
    _, idx0 = _loss(p, cfg, dh, d_aux)
    eps = 1e-6
    for name, gname in GRAD_OF.items():
        for _ in range(3):
            v = rng.standard_normal(p[name].shape)
            plus = dict(p, **{name: p[name] + eps * v})
            minus = dict(p, **{name: p[name] - eps * v})
            lp, idx_p = _loss(plus, cfg, dh, d_aux)
            lm, idx_m = _loss(minus, cfg, dh, d_aux)
            # the expert choice must not change inside the difference
            assert np.array_equal(idx_p, idx0) and np.array_equal(idx_m, idx0)
            fd = (lp - lm) / (2 * eps)
            an = float(np.sum(getattr(g, gname) * v))
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


def test_softmax_gradient_rows_sum_to_zero():
    # each token's logit gradient sums to zero over the experts (softmax), so the bias
    # gradient and the centroid gradient also sum to zero over the experts
    p, cfg = _layer(T=40, n_routed=9, top_k=3)
    dh = np.random.default_rng(5).standard_normal(p["u"].shape)
    g = _grads(p, cfg, dh, 0.9)
    assert abs(g.d_bias.sum()) <= 1e-12 * np.abs(g.d_bias).sum()
    assert np.abs(g.d_centroids.sum(axis=0)).max() <= 1e-12 * np.abs(g.d_centroids).sum()


def test_single_expert_layer_has_no_router_gradient():
    # one routed expert, top-1, no shared expert: s = g = 1 exactly, so the softmax passes
    # no gradient back (the layer is a dense FFN plus the residual)
    p, cfg = _layer(n_shared=0, n_routed=1, top_k=1)
    dh = np.random.default_rng(2).standard_normal(p["u"].shape)
    g = _grads(p, cfg, dh, 1.0)
    assert np.all(g.d_centroids == 0.0) and np.all(g.d_bias == 0.0)
    dx, dwg, dwu, dwd = O.swiglu_ffn_backward(p["u"], p["w_gate"][0], p["w_up"][0],
                                              p["w_down"][0], dh)
    np.testing.assert_allclose(g.du, dh + dx, rtol=0, atol=1e-12)
    np.testing.assert_allclose(g.d_w_down[0], dwd, rtol=0, atol=1e-12)


def test_segmented_shared_expert_gradients_are_the_slices():
    # fine-grained segmentation: a shared expert of width I split into m pieces (rows of
    # W_gate / W_up, columns of W_down), all with gate 1, is the same function, so du and
    # the router gradients are unchanged and the pieces' weight gradients are the slices
    # of the unsplit expert's.  The routed experts have width k = I / m in both layers
    # (zero-padded to I in the unsplit one: zero rows and columns add nothing and get a
    # zero gradient).
    m, inter = 4, 8
    k = inter // m
    p, cfg = _layer(n_shared=1, inter=inter)
    dh = np.random.default_rng(8).standard_normal(p["u"].shape)
    wg_r, wu_r, wd_r = p["w_gate"][1:, :k], p["w_up"][1:, :k], p["w_down"][1:, :, :k]
    pad = inter - k
    ref = dict(p,
               w_gate=np.concatenate([p["w_gate"][:1], np.pad(wg_r, ((0, 0), (0, pad), (0, 0)))]),
               w_up=np.concatenate([p["w_up"][:1], np.pad(wu_r, ((0, 0), (0, pad), (0, 0)))]),
               w_down=np.concatenate([p["w_down"][:1], np.pad(wd_r, ((0, 0), (0, 0), (0, pad)))]))
    pieces = np.stack([p["w_down"][0][:, i * k:(i + 1) * k] for i in range(m)])
    split = dict(p,
                 w_gate=np.concatenate([p["w_gate"][0].reshape(m, k, -1), wg_r]),
                 w_up=np.concatenate([p["w_up"][0].reshape(m, k, -1), wu_r]),
                 w_down=np.concatenate([pieces, wd_r]))
    g_ref = _grads(ref, cfg, dh, 0.5)
    g_split = _grads(split, dict(cfg, n_shared=m), dh, 0.5)
    close = dict(rtol=0, atol=1e-12)
    np.testing.assert_allclose(g_split.du, g_ref.du, **close)
    np.testing.assert_allclose(g_split.d_centroids, g_ref.d_centroids, **close)
    np.testing.assert_allclose(g_split.d_w_gate[:m].reshape(inter, -1), g_ref.d_w_gate[0], **close)
    np.testing.assert_allclose(g_split.d_w_up[:m].reshape(inter, -1), g_ref.d_w_up[0], **close)
    np.testing.assert_allclose(np.concatenate(list(g_split.d_w_down[:m]), axis=1),
                               g_ref.d_w_down[0], **close)
    np.testing.assert_allclose(g_split.d_w_gate[m:], g_ref.d_w_gate[1:, :k], **close)
    assert np.all(g_ref.d_w_gate[1:, k:] == 0) and np.all(g_ref.d_w_down[1:, :, k:] == 0)


def test_gradients_are_linear_in_the_upstream_gradients():
    p, cfg = _layer()
    rng = np.random.default_rng(4)
    dh1, dh2 = rng.standard_normal(p["u"].shape), rng.standard_normal(p["u"].shape)
    a = _grads(p, cfg, dh1, 0.3)
    b = _grads(p, cfg, dh2, -1.1)
    c = _grads(p, cfg, dh1 + 2.0 * dh2, 0.3 + 2.0 * -1.1)
    for name in GRAD_OF.values():
        np.testing.assert_allclose(getattr(c, name), getattr(a, name) + 2.0 * getattr(b, name),
                                   rtol=1e-12, atol=1e-12)
