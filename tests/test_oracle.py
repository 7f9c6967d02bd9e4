"""Pins for the fp64 oracle, against things other than itself (CPU only).

Each test ties the oracle to brute force, a closed form, a library routine, or an
invariant that the DeepSeekMoE pages fix, so that a dropped term, a wrong sign or index,
or a transposed operand in the oracle fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

from oracle import moe_oracle as O
from mixture_experts_layer_65_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "deepseekmoe_pages.json")


def _small(seed, T=6, d=12, ks=1, nr=6, inter=8, k=2, bias=False, std_w=0.3):
    rng = np.random.default_rng(seed)
    g = ks + nr
    return dict(
        u=rng.standard_normal((T, d)),
        centroids=rng.standard_normal((nr, d)) / math.sqrt(d),
        w_gate=rng.standard_normal((g, inter, d)) * std_w,
        w_up=rng.standard_normal((g, inter, d)) * std_w,
        w_down=rng.standard_normal((g, d, inter)) * std_w,
        n_shared=ks, top_k=k, alpha1=0.01,
        bias=rng.standard_normal(nr) if bias else None,
    )


# ----------------------------------------------------------------- brute force
@pytest.mark.parametrize("seed,ks,nr,k,bias", [
    (0, 1, 6, 2, False), (1, 0, 5, 1, False), (2, 2, 8, 3, True), (3, 1, 4, 4, False),
    (4, 0, 1, 1, False), (5, 3, 7, 5, True),
])
def test_vectorised_matches_brute_force(seed, ks, nr, k, bias):
    a = _small(seed, ks=ks, nr=nr, k=k, bias=bias)
    out = O.moe_forward(a["u"], a["centroids"], a["w_gate"], a["w_up"], a["w_down"],
                        a["n_shared"], a["top_k"], a["alpha1"], bias=a["bias"])
    H, IDX, Wt, counts, aux = O.brute_force_layer(
        a["u"], a["centroids"], a["w_gate"], a["w_up"], a["w_down"], a["n_shared"],
        a["top_k"], a["alpha1"], bias=a["bias"])
    np.testing.assert_array_equal(out.routing.topk_idx, np.array(IDX))
    np.testing.assert_allclose(out.routing.topk_w, np.array(Wt), rtol=1e-13, atol=0)
    np.testing.assert_allclose(out.h, np.array(H), rtol=1e-12, atol=1e-13)
    np.testing.assert_array_equal(out.counts, np.array(counts))
    assert out.aux == pytest.approx(aux, rel=1e-13)


# ----------------------------------------------------------------- library routines
def test_softmax_matches_scipy():
    rng = np.random.default_rng(7)
    l = rng.standard_normal((50, 17)) * 5
    np.testing.assert_allclose(O.affinity_softmax(l), scipy.special.softmax(l, axis=1),
                               rtol=1e-14, atol=0)


def _llama_mlp(x, wg, wu, wd):
    """SwiGLU FFN as implemented by transformers' LlamaMLP (down(silu(gate x) * up x))."""
    from transformers import LlamaConfig
    from transformers.models.llama.modeling_llama import LlamaMLP
    d, inter = wg.shape[1], wg.shape[0]
    cfg = LlamaConfig(hidden_size=d, intermediate_size=inter, hidden_act="silu",
                      mlp_bias=False, num_attention_heads=1, num_key_value_heads=1,
                      head_dim=d)
    mlp = LlamaMLP(cfg).double()
    with torch.no_grad():
        mlp.gate_proj.weight.copy_(torch.from_numpy(np.asarray(wg, dtype=np.float64)))
        mlp.up_proj.weight.copy_(torch.from_numpy(np.asarray(wu, dtype=np.float64)))
        mlp.down_proj.weight.copy_(torch.from_numpy(np.asarray(wd, dtype=np.float64)))
        return mlp(torch.from_numpy(np.asarray(x, dtype=np.float64))).numpy()


def test_swiglu_matches_llama_mlp():
    a = _small(11, inter=9, d=13)
    y = O.swiglu_ffn(a["u"], a["w_gate"][0], a["w_up"][0], a["w_down"][0])
    ref = _llama_mlp(a["u"], a["w_gate"][0], a["w_up"][0], a["w_down"][0])
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-14)


def test_single_expert_layer_is_dense_swiglu():
    """N_r = 1, top-1, no shared expert: s = g = 1 and h = u + SwiGLU(u)."""
    a = _small(12, ks=0, nr=1, k=1, d=10, inter=7)
    out = O.moe_forward(a["u"], a["centroids"], a["w_gate"], a["w_up"], a["w_down"],
                        0, 1, 0.01)
    assert np.all(out.routing.topk_idx == 0)
    np.testing.assert_allclose(out.routing.topk_w, 1.0, rtol=0, atol=1e-15)
    ref = a["u"] + _llama_mlp(a["u"], a["w_gate"][0], a["w_up"][0], a["w_down"][0])
    np.testing.assert_allclose(out.h, ref, rtol=1e-12, atol=1e-13)
    # f = 1, P = 1 -> aux = alpha1
    assert out.aux == pytest.approx(0.01, rel=1e-15)


def test_shared_expert_has_gate_one():
    """A shared copy of the single routed expert doubles the FFN term: h = u + 2 SwiGLU(u)."""
    a = _small(13, ks=0, nr=1, k=1, d=10, inter=7)
    wg = np.concatenate([a["w_gate"], a["w_gate"]])
    wu = np.concatenate([a["w_up"], a["w_up"]])
    wd = np.concatenate([a["w_down"], a["w_down"]])
    out = O.moe_forward(a["u"], a["centroids"], wg, wu, wd, 1, 1, 0.01)
    ref = a["u"] + 2.0 * _llama_mlp(a["u"], a["w_gate"][0], a["w_up"][0], a["w_down"][0])
    np.testing.assert_allclose(out.h, ref, rtol=1e-12, atol=1e-13)


def test_gate_is_unrenormalised_softmax():
    """Two routed experts, top-1: the kept gate is sigmoid(l0 - l1), not 1."""
    a = _small(14, ks=0, nr=2, k=1, d=8, inter=5)
    out = O.moe_forward(a["u"], a["centroids"], a["w_gate"], a["w_up"], a["w_down"],
                        0, 1, 0.01)
    l = a["u"] @ a["centroids"].T
    for t in range(a["u"].shape[0]):
        e = int(np.argmax(l[t]))
        g = scipy.special.expit(l[t, e] - l[t, 1 - e])
        ref = a["u"][t] + g * _llama_mlp(a["u"][t:t + 1], a["w_gate"][e], a["w_up"][e],
                                         a["w_down"][e])[0]
        assert out.routing.topk_idx[t, 0] == e
        assert out.routing.topk_w[t, 0] == pytest.approx(g, rel=1e-14)
        np.testing.assert_allclose(out.h[t], ref, rtol=1e-12, atol=1e-13)


# ----------------------------------------------------------------- closed forms / special cases
def test_uniform_router_closed_form():
    """All-zero centroids: s = 1/N_r everywhere, ties -> experts 0..K'-1, aux = a1*K'/N_r."""
    a = _small(15, ks=1, nr=6, k=3)
    cen = np.zeros_like(a["centroids"])
    out = O.moe_forward(a["u"], cen, a["w_gate"], a["w_up"], a["w_down"], 1, 3, 0.01)
    T = a["u"].shape[0]
    np.testing.assert_array_equal(out.routing.topk_idx, np.tile(np.arange(3), (T, 1)))
    np.testing.assert_allclose(out.routing.topk_w, 1.0 / 6.0, rtol=1e-15)
    np.testing.assert_array_equal(out.counts, [T, T, T, 0, 0, 0])
    np.testing.assert_allclose(out.P, 1.0 / 6.0, rtol=1e-15)
    assert out.aux == pytest.approx(0.01 * 3 / 6, rel=1e-14)


def test_zero_down_projection_leaves_residual():
    a = _small(16, ks=2, nr=5, k=2)
    out = O.moe_forward(a["u"], a["centroids"], a["w_gate"], a["w_up"],
                        np.zeros_like(a["w_down"]), 2, 2, 0.01)
    np.testing.assert_array_equal(out.h, a["u"])


def test_zero_input_gives_zero_output():
    a = _small(17, ks=1, nr=5, k=2)
    z = np.zeros_like(a["u"])
    out = O.moe_forward(z, a["centroids"], a["w_gate"], a["w_up"], a["w_down"], 1, 2, 0.01)
    np.testing.assert_array_equal(out.h, 0.0)


def test_tie_break_lower_index_wins():
    """Duplicate centroids: equal logits; the stable order keeps the lower index first."""
    rng = np.random.default_rng(18)
    d = 8
    cen = rng.standard_normal((5, d))
    cen[3] = cen[1]
    u = cen[1][None, :] * 3.0            # experts 1 and 3 tie for the largest logit
    l = O.router_logits(u, cen)
    assert l[0, 1] == l[0, 3] and np.argmax(l[0]) in (1, 3)
    idx = O.select_topk(l, 1)
    assert idx[0, 0] == 1
    idx2 = O.select_topk(l, 2)
    np.testing.assert_array_equal(idx2[0], [1, 3])


def test_topk_equal_to_all_experts_gates_sum_to_one():
    a = _small(19, ks=0, nr=5, k=5)
    r = O.route(a["u"], a["centroids"], 5)
    np.testing.assert_allclose(r.topk_w.sum(axis=1), 1.0, rtol=0, atol=1e-15)
    for row in r.topk_idx:
        assert sorted(row.tolist()) == list(range(5))


# ----------------------------------------------------------------- invariants
@pytest.mark.parametrize("name", ["tiny"])
def test_routing_invariants_on_tiny_workload(name):
    w = W.make_workload(name)
    out = O.moe_forward(w.u, w.centroids, w.w_gate, w.w_up, w.w_down, w.n_shared,
                        w.top_k, w.alpha1)
    r = out.routing
    # exactly K' distinct routed indices in [0, N_r)
    assert r.topk_idx.shape == (w.T, w.top_k)
    assert r.topk_idx.min() >= 0 and r.topk_idx.max() < w.n_routed
    assert all(len(set(row)) == w.top_k for row in r.topk_idx.tolist())
    # descending logit order
    ls = np.take_along_axis(r.logits, r.topk_idx, axis=1)
    assert np.all(np.diff(ls, axis=1) <= 0)
    # gates = softmax mass of the selected experts, < 1 since K' < N_r
    gsum = r.topk_w.sum(axis=1)
    sel_mass = np.array([r.s[t, r.topk_idx[t]].sum() for t in range(w.T)])
    np.testing.assert_allclose(gsum, sel_mass, rtol=1e-15)
    assert np.all(gsum < 1.0)
    # balance statistics
    assert out.counts.sum() == w.T * w.top_k
    np.testing.assert_allclose(out.P.sum(), 1.0, rtol=1e-14)
    np.testing.assert_allclose(out.f, out.counts / w.T)
    assert out.aux == pytest.approx(w.alpha1 * float(np.sum(out.f * out.P)), rel=1e-15)


def test_balance_brute_recount():
    a = _small(20, ks=0, nr=7, k=3, T=40)
    out = O.moe_forward(a["u"], a["centroids"], a["w_gate"], a["w_up"], a["w_down"],
                        0, 3, 0.01)
    cnt = [0] * 7
    for row in out.routing.topk_idx.tolist():
        for e in row:
            cnt[e] += 1
    np.testing.assert_array_equal(out.counts, cnt)
    P = [sum(out.routing.s[t, i] for t in range(40)) / 40 for i in range(7)]
    np.testing.assert_allclose(out.P, P, rtol=1e-14)


def test_fine_grained_segmentation_reproduces_unsplit_expert():
    """Split one expert's intermediate dim into m = 4 pieces (rows of W_gate/W_up, columns
    of W_down); the pieces, all routed together with the same gate, sum to the unsplit
    expert.  Shown both on the FFN and at layer level with the pieces as shared experts
    (gate 1), which also justifies running K_s shared experts as one wide group."""
    a = _small(21, ks=1, nr=4, k=2, inter=16, d=10)
    wg, wu, wd = a["w_gate"][0], a["w_up"][0], a["w_down"][0]
    m = 4
    x = a["u"]
    whole = O.swiglu_ffn(x, wg, wu, wd)
    parts = sum(O.swiglu_ffn(x, wg[p::m], wu[p::m], wd[:, p::m]) for p in range(m))
    np.testing.assert_allclose(parts, whole, rtol=1e-13, atol=1e-15)
    # layer level: 1 unsplit shared expert vs m pieces as shared experts
    inter_p = wg.shape[0] // m
    pg = np.stack([wg[p * inter_p:(p + 1) * inter_p] for p in range(m)])
    pu = np.stack([wu[p * inter_p:(p + 1) * inter_p] for p in range(m)])
    pd = np.stack([wd[:, p * inter_p:(p + 1) * inter_p] for p in range(m)])
    # routed experts must share the pieces' width: give them width inter_p
    rg, ru, rd = a["w_gate"][1:, :inter_p], a["w_up"][1:, :inter_p], a["w_down"][1:, :, :inter_p]
    split = O.moe_forward(x, a["centroids"], np.concatenate([pg, rg]),
                          np.concatenate([pu, ru]), np.concatenate([pd, rd]), m, 2, 0.01)
    base = O.moe_forward(x, a["centroids"], rg, ru, rd, 0, 2, 0.01)
    np.testing.assert_allclose(split.h - base.h, whole, rtol=1e-12, atol=1e-14)


def test_rows_subset_matches_full():
    a = _small(22, ks=1, nr=6, k=2, T=12)
    full = O.moe_forward(a["u"], a["centroids"], a["w_gate"], a["w_up"], a["w_down"],
                         1, 2, 0.01)
    sub = O.moe_forward(a["u"], a["centroids"], a["w_gate"], a["w_up"], a["w_down"],
                        1, 2, 0.01, rows=[0, 5, 11])
    np.testing.assert_allclose(sub.h, full.h[[0, 5, 11]], rtol=1e-15, atol=0)
    assert sub.aux == full.aux


def test_near_tie_detection():
    s = np.array([[0.5, 0.3, 0.3 - 5e-7, 0.1], [0.4, 0.3, 0.2, 0.1]])
    np.testing.assert_array_equal(O.near_tie_tokens(s, 2), [True, False])
    np.testing.assert_array_equal(O.near_tie_tokens(s, 4), [False, False])


def test_bf16_bits_widen_exactly():
    x = np.array([1.0, -2.5, 3.140625, 1e-3], dtype=np.float32)
    bits = W.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.widen(bits), ref)


# ----------------------------------------------------------------- numbers the pages print
def test_configs_match_the_pages():
    g = json.load(open(GOLDEN))
    c16 = W.CONFIGS["16b_prefill"]
    assert c16["d"] == g["config_16b"]["hidden"]
    assert c16["n_shared"] == g["config_16b"]["n_shared"]
    assert c16["n_routed"] == g["config_16b"]["n_routed"]
    assert c16["top_k"] == g["config_16b"]["routed_active"]
    assert c16["n_shared"] + c16["top_k"] == g["config_16b"]["expert_passes_per_token"]
    c145 = W.CONFIGS["145b"]
    assert (c145["n_shared"], c145["n_routed"], c145["top_k"]) == (
        g["config_145b"]["n_shared"], g["config_145b"]["n_routed"], g["config_145b"]["routed_active"])
    assert W.CONFIGS["2b"]["alpha1"] == g["alpha1"]["2b"]
    assert c16["alpha1"] == g["alpha1"]["16b"]
    # fine-grained segmentation: same total expert params and per-token FLOPs as GShard
    c2, cg = W.CONFIGS["2b"], W.CONFIGS["gshard"]
    assert (c2["n_shared"] + c2["n_routed"]) * c2["inter"] == cg["n_routed"] * cg["inter"]
    assert (c2["n_shared"] + c2["top_k"]) * c2["inter"] == cg["top_k"] * cg["inter"]
    assert math.comb(16, 2) == g["combinations"]["choose_2_of_16"]
    assert math.comb(64, 8) == g["combinations"]["choose_8_of_64"]


def test_workload_is_seeded_and_prefix_stable():
    a = W.make_workload("tiny")
    b = W.make_workload("tiny", T=64)
    np.testing.assert_array_equal(a.u[:64], b.u)
    np.testing.assert_array_equal(a.w_down, b.w_down)
    c = W.make_workload("tiny", seed=1)
    assert not np.array_equal(a.u, c.u)
    z = W.make_workload("145b", T=4, d=64, inter=64, n_routed=16, n_shared=1, top_k=3)
    assert z.logit_bias is not None and z.logit_bias.shape == (16,)
    assert np.all(np.diff(z.logit_bias) < 0)
    np.testing.assert_allclose(np.exp(z.logit_bias.astype(np.float64)).sum(), 1.0, rtol=1e-6)


# ------------------------------------------------------------------ e4m3 gate/up variant
def _e4m3_values() -> np.ndarray:
    """Every finite e4m3 value, decoded from its bit pattern by torch's float8 type."""
    bits = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    v = bits.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    return np.unique(v[np.isfinite(v)])


def test_e4m3_round_matches_torch_and_the_value_grid():
    grid = _e4m3_values()
    assert grid.size == 253 and grid.max() == O.E4M3_MAX      # 126 per sign, +0 and -0 merge
    np.testing.assert_array_equal(O.e4m3_round(grid), grid)   # representable values stay
    pos = grid[grid >= 0]
    mids = (pos[:-1] + pos[1:]) / 2                           # exact ties: to the even mantissa
    rng = np.random.default_rng(3)
    y = np.concatenate([mids, -mids, rng.uniform(-448, 448, 20000), rng.uniform(-0.03, 0.03, 20000)])
    y = y.astype(np.float32).astype(np.float64)
    ref = torch.from_numpy(y).to(torch.float32).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.e4m3_round(y), ref)
    # saturation beyond the largest finite value
    np.testing.assert_array_equal(O.e4m3_round(np.array([448.5, 463.9, 1e9, -500.0])),
                                  [448.0, 448.0, 448.0, -448.0])


def test_quantize_rows_e4m3_scales_and_error_bound():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((64, 300)).astype(np.float32)
    x[5] = 0.0                                                # an all-zero row
    q, s = O.quantize_rows_e4m3(x)
    grid = set(_e4m3_values().tolist())
    assert set(np.unique(q).tolist()) <= grid
    a = np.abs(x).max(axis=1)
    assert s[5] == 0.0 and np.all(q[5] == 0.0)
    nz = a > 0
    # the row maximum maps to +-448 and the scale is fp32(a / 448)
    np.testing.assert_array_equal(np.abs(q[nz]).max(axis=1), O.E4M3_MAX)
    np.testing.assert_array_equal(s[nz], (a[nz] / np.float32(448)).astype(np.float32))
    # half an e4m3 step: 2^-4 relative in the normal range, 2^-10 * scale below it
    err = np.abs(x.astype(np.float64) - q * s[:, None])
    bound = 2.0 ** -4 * np.abs(x) * (1 + 1e-6) + 2.0 ** -10 * s[:, None] * (1 + 1e-6)
    assert np.all(err <= bound)


def test_e4m3_variant_is_exact_when_quantisation_is_lossless():
    # rows whose entries are e4m3 values times 2^k with the row maximum at 448 * 2^k
    # quantise without loss, so the variant must equal the plain layer
    rng = np.random.default_rng(6)
    grid = _e4m3_values()
    grid = grid[np.abs(grid) > 0.5]

    def lossless(shape, k):
        v = rng.choice(grid, size=shape)
        v[..., 0] = O.E4M3_MAX
        return v * 2.0 ** k

    T, d, ns, nr, I, K = 40, 64, 1, 6, 32, 2
    u = lossless((T, d), -9)
    cen = rng.standard_normal((nr, d)) / 8
    wg = lossless((ns + nr, I, d), -12)
    wu = lossless((ns + nr, I, d), -11)
    wd = rng.standard_normal((ns + nr, d, I)) * 0.02
    a = O.moe_forward(u, cen, wg, wu, wd, ns, K, 0.01)
    b = O.moe_forward(u, cen, wg, wu, wd, ns, K, 0.01, gate_up_e4m3=True)
    np.testing.assert_array_equal(a.routing.topk_idx, b.routing.topk_idx)
    np.testing.assert_allclose(b.h, a.h, rtol=1e-13, atol=1e-13)


def test_e4m3_variant_changes_only_the_expert_part_and_by_little():
    w = W.make_workload("tiny")
    a = O.moe_forward(w.u, w.centroids, w.w_gate, w.w_up, w.w_down, w.n_shared, w.top_k, w.alpha1)
    b = O.moe_forward(w.u, w.centroids, w.w_gate, w.w_up, w.w_down, w.n_shared, w.top_k, w.alpha1,
                      gate_up_e4m3=True)
    np.testing.assert_array_equal(a.routing.topk_idx, b.routing.topk_idx)   # routing untouched
    assert a.aux == b.aux
    u = O.widen(w.u)
    rel = np.abs((b.h - u) - (a.h - u)).max() / np.abs(a.h - u).max()
    assert 1e-4 < rel < 0.1, rel                                           # quantised, not broken


# ---------------------------------------------------------------- e4m3 down variant
def test_bf16_round_matches_torch_and_ties_to_even():
    import torch
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-6, 6, 20000),
                        [0.0, -0.0, 1.0, -3.5, 1e-40]])
    want = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.bf16_round(x), want)
    # exact ties between neighbouring bf16 values go to the even mantissa
    base = np.array([1.0, 1.0 + 2 ** -7, 3.0, 3.0 + 2 ** -6])
    ties = base + np.array([2 ** -8, 2 ** -8, 2 ** -7, 2 ** -7])
    np.testing.assert_array_equal(O.bf16_round(ties), [1.0, 1.0 + 2 ** -6, 3.0, 3.0 + 2 ** -5])
    bf = O.bf16_round(x)
    np.testing.assert_array_equal(O.bf16_round(bf), bf)   # bf16 values stay


def _e4m3_err_bound(x, scale):
    """|deq(x) - x| per entry: half a step of 3 mantissa bits (2^-4 relative) for normal
    e4m3 values, half the subnormal step (2^-10) times the row scale below them."""
    return np.abs(x) * 2.0 ** -4 + 2.0 ** -10 * scale[:, None]


def test_e4m3_down_output_within_the_quantisation_bound():
    """Each routed expert's output with the down product on quantised bf16 hidden rows and
    quantised W_down rows differs from the plain product by at most the sum of the entries'
    rounding bounds (bf16: 2^-9 relative; e4m3: the bound above)."""
    w = W.make_workload("tiny", T=64)
    for e in range(3):
        g = w.n_shared + e
        x = w.u[:32]
        hid = O.swiglu_hidden(x, w.w_gate[g], w.w_up[g])
        wd = O.widen(w.w_down[g])
        y_plain = hid @ wd.T
        y_var = O.swiglu_ffn(x, w.w_gate[g], w.w_up[g], w.w_down[g], down_e4m3=True)
        hb = O.bf16_round(hid)
        _, sh = O.quantize_rows_e4m3(hb)
        _, sw = O.quantize_rows_e4m3(w.w_down[g])
        eh = np.abs(hb - hid) + _e4m3_err_bound(hb, sh)          # hidden entries
        ew = _e4m3_err_bound(wd, sw)                             # weight entries
        bound = eh @ np.abs(wd).T + np.abs(hid) @ ew.T + eh @ ew.T
        err = np.abs(y_var - y_plain)
        assert np.all(err <= bound * (1 + 1e-9))
        assert err.max() > 0                                     # the variant does round
        # a forgotten scale would break it by orders of magnitude
        q, s = O.quantize_rows_e4m3(O.bf16_round(hid))
        assert np.any(np.abs(q @ wd.T - y_plain) > bound)


def test_e4m3_down_quantises_rows_of_w_down():
    """W_down rows that are e4m3 values times a power-of-two row scale quantise without
    loss per row (row maximum 448 * 2^-j); the variant then equals the product of the
    quantised hidden rows with W_down itself.  Quantising per column instead would not be
    lossless here (the columns mix rows of different scales)."""
    rng = np.random.default_rng(9)
    grid = np.array([v for v in np.unique(np.abs(O.e4m3_round(rng.standard_normal(5000) * 100))) if v > 0])
    d, I = 8, 16
    wd = rng.choice(grid, (d, I)) * rng.choice([-1.0, 1.0], (d, I))
    wd[:, 0] = 448.0
    wd = wd * 2.0 ** -rng.integers(3, 12, d)[:, None]
    np.testing.assert_array_equal(O._dequantized(wd), wd)
    assert not np.array_equal(O._dequantized(wd.T).T, wd)
    hid = rng.standard_normal((5, I))
    want = O._dequantized(O.bf16_round(hid)) @ wd.T
    x_rows = O._dequantized(O.bf16_round(hid))
    np.testing.assert_allclose(x_rows @ O._dequantized(wd).T, want, rtol=0, atol=0)


def test_e4m3_down_shared_experts_form_one_group():
    """With the down product quantised, the K_s shared experts run as one group: their part
    of the layer is the quantised concatenation of their bf16 hidden rows times the
    quantised W_down matrices side by side (one scale per row of each concatenation), so
    that the layer equals its routed part (no shared expert) plus that group.  Per-expert
    scales differ from it once the experts' magnitudes do."""
    w = W.make_workload("tiny", T=40, n_shared=2)
    w.w_gate[1] *= 8    # the second shared expert's hidden values are much larger
    a = O.moe_forward(w.u, w.centroids, w.w_gate, w.w_up, w.w_down, 2, w.top_k, w.alpha1,
                      down_e4m3=True)
    routed_only = O.moe_forward(w.u, w.centroids, w.w_gate[2:], w.w_up[2:], w.w_down[2:], 0,
                                w.top_k, w.alpha1, down_e4m3=True)
    x = O.widen(w.u)
    hid = np.concatenate([O.swiglu_hidden(x, w.w_gate[j], w.w_up[j]) for j in range(2)], axis=1)
    wd_joint = np.concatenate([O.widen(w.w_down[0]), O.widen(w.w_down[1])], axis=1)
    shared = O._dequantized(O.bf16_round(hid)) @ O._dequantized(wd_joint).T
    np.testing.assert_allclose(a.h, routed_only.h + shared, rtol=0, atol=1e-12)
    per_expert = sum(O._dequantized(O.bf16_round(O.swiglu_hidden(x, w.w_gate[j], w.w_up[j])))
                     @ O._dequantized(w.w_down[j]).T for j in range(2))
    assert np.abs(per_expert - shared).max() > 1e-6
