"""Plain fp64 CPU oracle of the DeepSeekMoE layer forward pass (and its gradients).

TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check and the CPU
baseline leg of the benchmark may import this module.  It shares no code with the CUDA
path (no kernels, helpers, tables or pre/post-processing); the only thing both sides
consume is the seeded input arrays of the workload generator.

What it computes, and where the pages define it ("DeepSeekMoE: Towards Ultimate Expert
Specialization in Mixture-of-Experts Language Models", deepforge.srivtx.xyz article):

  * section "Routing in a classic MoE layer": affinity s_i = softmax_i(u^T e_i); the gate
    g_i equals s_i when s_i is among the top-K affinities and 0 otherwise; the output is
    h = sum_i g_i FFN_i(u) + u.
  * section "Top-k routing, from affinities to gates": the softmax runs over all routed
    experts *before* the top-k cut, so the kept gates are not renormalised; experts are
    ranked by logit with a stable sort, so on exactly equal logits the lower index wins.
  * section "Where this sits" (shared expert isolation, fine-grained segmentation):
    K_s shared experts run on every token and the routed top-k becomes mK - K_s.
  * section "Expert-level balance loss": L_ExpBal = alpha_1 * sum_i f_i * P_i with f_i the
    fraction of tokens that selected routed expert i and P_i its mean affinity over the
    batch.
  * The expert FFN is SwiGLU, FFN(x) = W_down (SiLU(W_gate x) * (W_up x)), no biases,
    SiLU(z) = z / (1 + exp(-z)) (the GLU-variants form cited by the observer.broadside.tech
    card, "cites"); the pages themselves only say "FFN".

Readings where the pages are silent (each also listed in the design notes):
  * the shared experts carry gate 1 and have no centroid; the softmax domain is the
    routed experts only (plus the optional per-expert logit bias, added before it);
  * f_i = count_i / T and P_i = (1/T) * sum_t s[t, i] over all tokens;
  * the residual +u of the routing equation is included (the page's Python listing
    omits it; the equation is taken as the authority).

All arithmetic is fp64.  bf16 inputs arrive as uint16 bit patterns and are widened
exactly.  Parity is pinned by the CPU tests against brute force, closed forms, library
routines (scipy softmax, transformers' LlamaMLP SwiGLU) and invariants; the backward pass
(moe_backward) against central finite differences of moe_forward and invariants.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

__all__ = ["widen", "router_logits", "affinity_softmax", "select_topk", "route",
           "swiglu_hidden", "swiglu_ffn", "balance_stats", "moe_forward", "near_tie_tokens",
           "brute_force_layer", "Routing", "LayerOut", "E4M3_MAX", "e4m3_round",
           "quantize_rows_e4m3", "bf16_round", "swiglu_ffn_backward", "moe_backward",
           "LayerGrads"]


def widen(a) -> np.ndarray:
    """Exact widening to fp64: uint16 arrays are bf16 bit patterns, floats are values."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return a.astype(np.float64, copy=False)


# ---------------------------------------------------------------- routing (gating)
def router_logits(u, centroids, bias=None) -> np.ndarray:
    """logit[t, i] = u_t . e_i (+ b_i): the token-to-centroid affinity before the softmax.

    deepforge article, "Routing in a classic MoE layer": s_i = softmax_i(u^T e_i).
    """
    l = widen(u) @ widen(centroids).T
    if bias is not None:
        l = l + widen(bias)[None, :]
    return l


def affinity_softmax(logits: np.ndarray) -> np.ndarray:
    """s[t, :] = softmax over the routed experts, max-subtracted (deepforge, same section)."""
    z = logits - logits.max(axis=1, keepdims=True)
    ez = np.exp(z)
    return ez / ez.sum(axis=1, keepdims=True)


def select_topk(logits: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest logits per row, in descending order.

    A stable sort of -logit: on exactly equal logits the lower expert index comes first
    (deepforge, "Top-k routing, from affinities to gates").
    """
    order = np.argsort(-logits, axis=1, kind="stable")
    return order[:, :k].astype(np.int64)


@dataclasses.dataclass
class Routing:
    logits: np.ndarray      # [T, N_r] fp64
    s: np.ndarray           # [T, N_r] fp64 affinities (softmax)
    topk_idx: np.ndarray    # [T, K'] int64, descending logit order
    topk_w: np.ndarray      # [T, K'] fp64 gates g = s at the selected experts


def route(u, centroids, top_k: int, bias=None) -> Routing:
    l = router_logits(u, centroids, bias)
    s = affinity_softmax(l)
    idx = select_topk(l, top_k)
    w = np.take_along_axis(s, idx, axis=1)   # g_i = s_i for selected i, no renormalisation
    return Routing(l, s, idx, w)


# ---------------------------------------------------------------- experts
def _silu(z: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def swiglu_hidden(x, w_gate, w_up, gate_up_e4m3: bool = False) -> np.ndarray:
    """The expert's hidden activation SiLU(W_gate x) * (W_up x); x [n, d], W_gate/W_up [I, d].

    gate_up_e4m3: the e4m3 variant -- x's rows and W_gate's / W_up's rows are replaced by
    their scaled e4m3 approximations (quantize_rows_e4m3) in the two gate/up products."""
    if gate_up_e4m3:
        x, w_gate, w_up = _dequantized(x), _dequantized(w_gate), _dequantized(w_up)
    x = widen(x)
    a = x @ widen(w_gate).T
    b = x @ widen(w_up).T
    return _silu(a) * b


def swiglu_ffn(x, w_gate, w_up, w_down, gate_up_e4m3: bool = False,
               down_e4m3: bool = False) -> np.ndarray:
    """FFN(x) = W_down (SiLU(W_gate x) * (W_up x)); x [n, d], W_gate/W_up [I, d], W_down [d, I].

    down_e4m3: the e4m3 down variant -- the hidden rows (rounded to bf16) and W_down's rows
    are replaced by their scaled e4m3 approximations in the down product."""
    hid = swiglu_hidden(x, w_gate, w_up, gate_up_e4m3)
    if down_e4m3:
        return _dequantized(bf16_round(hid)) @ _dequantized(w_down).T
    return hid @ widen(w_down).T


# ---------------------------------------------------------------- e4m3 gate/up variant
# Not on the pages: a reduced-precision variant of the layer in which the gate/up
# products take e4m3 operands.  Each token row and each gate/up weight row (one output
# channel, d values) is quantised with its own fp32 scale; everything else (router,
# down projection, residual, combine) is the plain layer.  Definition, per row x of
# fp32-valued entries:  a = max_i |x_i|;  if a = 0 every q_i = 0 and the scale is 0;
# otherwise inv = fp32(448 / a), q_i = e4m3(fp32(x_i * inv)) and scale = fp32(a / 448),
# so that x_i ~ q_i * scale.  e4m3 is the 8-bit float with 1 sign, 4 exponent (bias 7)
# and 3 mantissa bits, no infinities, largest finite value 448; e4m3(y) rounds to the
# nearest value, ties to the even mantissa, and clamps |y| > 448 to 448.
E4M3_MAX = 448.0


def e4m3_round(y) -> np.ndarray:
    """Nearest e4m3 value of each entry (ties to even), saturating at +-448."""
    y = np.asarray(y, dtype=np.float64)
    a = np.abs(y)
    out = np.zeros_like(a)
    big = a > E4M3_MAX
    nz = (a > 0) & ~big
    e = np.maximum(np.floor(np.log2(a[nz])), -6.0)   # binade; below 2^-6 the subnormal step
    step = np.exp2(e - 3.0)                          # 3 mantissa bits
    out[nz] = np.rint(a[nz] / step) * step
    out[big] = E4M3_MAX
    return np.copysign(out, y)


def quantize_rows_e4m3(x):
    """Per-row scaled e4m3 quantisation (definition above).  Returns (q [n, m] fp64 with
    e4m3 values, scale [n] fp64 with fp32 values); x_i is approximated by q_i * scale."""
    x32 = np.ascontiguousarray(widen(x), dtype=np.float32)   # bf16/fp32 values are exact
    a = np.max(np.abs(x32), axis=1)
    safe = np.where(a > 0, a, np.float32(1.0)).astype(np.float32)
    inv = (np.float32(E4M3_MAX) / safe).astype(np.float32)
    y = (x32 * inv[:, None]).astype(np.float32)
    q = e4m3_round(y.astype(np.float64))
    q[a == 0] = 0.0
    scale = np.where(a > 0, (safe / np.float32(E4M3_MAX)).astype(np.float32), np.float32(0.0))
    return q, scale.astype(np.float64)


def _dequantized(x) -> np.ndarray:
    q, scale = quantize_rows_e4m3(x)
    return q * scale[:, None]


# The e4m3 down variant (also not on the pages) quantises the down product's operands the
# same way: each hidden row SiLU(W_gate x) * (W_up x), first rounded to bf16 (the precision
# the layer stores it in), and each W_down row (one output channel) get their own scale.
# For the shared experts, which run as one group, the row is the concatenation of the K_s
# experts' hidden rows and the W_down row the concatenation of theirs (one scale each).
def bf16_round(y) -> np.ndarray:
    """Nearest bfloat16 value of each entry (ties to even; fp64 values go through fp32,
    whose rounding cannot change a bf16 decision except for exact ties)."""
    y32 = np.ascontiguousarray(np.asarray(y, dtype=np.float64), dtype=np.float32)
    b = y32.view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
    return b.astype(np.uint32).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------- balance statistics
def balance_stats(s: np.ndarray, topk_idx: np.ndarray, n_routed: int, alpha1: float):
    """Expert-level balance statistics (deepforge, "Expert-level balance loss").

    Returns (counts [N_r] int64, f [N_r], P [N_r], aux) with f_i = count_i / T,
    P_i = mean_t s[t, i] and aux = alpha_1 * sum_i f_i P_i.
    """
    T = s.shape[0]
    counts = np.bincount(topk_idx.reshape(-1), minlength=n_routed).astype(np.int64)
    f = counts / T
    P = s.sum(axis=0) / T
    aux = float(alpha1) * float(np.sum(f * P))
    return counts, f, P, aux


# ---------------------------------------------------------------- the layer
@dataclasses.dataclass
class LayerOut:
    h: np.ndarray           # [T or len(rows), d] fp64
    rows: np.ndarray        # token ids of the rows of h
    routing: Routing
    counts: np.ndarray
    f: np.ndarray
    P: np.ndarray
    aux: float


def moe_forward(u, centroids, w_gate, w_up, w_down, n_shared: int, top_k: int,
                alpha1: float, bias=None, rows=None, gate_up_e4m3: bool = False,
                down_e4m3: bool = False) -> LayerOut:
    """h = u + sum_{j shared} FFN_j(u) + sum_{i routed, selected} g_i FFN_i(u).

    Weights: w_gate/w_up [n_shared + N_r, I, d], w_down [n_shared + N_r, d, I], shared
    experts first; centroids [N_r, d].  Routing and the balance statistics always cover
    all T tokens; `rows` (token ids) restricts only which output rows are computed.
    Per routed expert the selecting tokens are gathered and run as one fp64 GEMM chain
    (the grouping the deepforge article names for production implementations).
    gate_up_e4m3 selects the e4m3 gate/up variant (quantize_rows_e4m3), down_e4m3 the e4m3
    down variant (quantised bf16 hidden rows and W_down rows; the shared experts' rows
    concatenated); routing and the residual use the unquantised values either way.
    """
    u64 = widen(u)
    T = u64.shape[0]
    n_routed = np.asarray(centroids).shape[0]
    r = route(u64, centroids, top_k, bias)
    counts, f, P, aux = balance_stats(r.s, r.topk_idx, n_routed, alpha1)

    rows = np.arange(T) if rows is None else np.asarray(rows, dtype=np.int64)
    x = u64[rows]
    h = x.copy()                                          # residual
    if down_e4m3 and n_shared:                            # shared experts as one group
        hid = np.concatenate([swiglu_hidden(x, w_gate[j], w_up[j], gate_up_e4m3)
                              for j in range(n_shared)], axis=1)
        wd = np.concatenate([widen(w_down[j]) for j in range(n_shared)], axis=1)
        h += _dequantized(bf16_round(hid)) @ _dequantized(wd).T
    else:
        for j in range(n_shared):                         # shared experts, gate 1
            h += swiglu_ffn(x, w_gate[j], w_up[j], w_down[j], gate_up_e4m3)
    sel = r.topk_idx[rows]                                # [n, K']
    gate = r.topk_w[rows]
    for e in range(n_routed):
        hit_r, hit_k = np.nonzero(sel == e)
        if hit_r.size == 0:
            continue
        y = swiglu_ffn(x[hit_r], w_gate[n_shared + e], w_up[n_shared + e],
                       w_down[n_shared + e], gate_up_e4m3, down_e4m3)
        h[hit_r] += gate[hit_r, hit_k][:, None] * y
    return LayerOut(h=h, rows=rows, routing=r, counts=counts, f=f, P=P, aux=aux)


def near_tie_tokens(s: np.ndarray, top_k: int, eps: float = 1e-6) -> np.ndarray:
    """Tokens whose k-th and (k+1)-th largest affinities differ by less than eps.

    Their routed set may legitimately differ between fp32 and fp64 arithmetic, so index
    parity excludes (and reports) them.  With k equal to the number of routed experts no
    token is excluded.
    """
    n = s.shape[1]
    if top_k >= n:
        return np.zeros(s.shape[0], dtype=bool)
    part = -np.sort(-s, axis=1)
    return (part[:, top_k - 1] - part[:, top_k]) < eps


# ---------------------------------------------------------------- backward pass
# Gradients of the layer for training (the full-precision layer only).  The scalar being
# differentiated is L = sum_t dh_t . h_t + d_aux * aux, i.e. dh = dL/dh (the gradient
# arriving from above) and d_aux = dL/daux (the weight of the balance loss in the training
# objective, usually 1).  Readings, where the pages give the forward only:
#   * the top-k choice is piecewise constant in u and the centroids, so no gradient flows
#     through *which* experts are chosen; the chosen gates g_i = s_i ("Routing in a
#     classic MoE layer") carry the gradient into the affinities and through the softmax;
#   * f_i = count_i / T ("Expert-level balance loss") is a step function of the same
#     choice and is held constant; P_i = mean_t s[t, i] carries the balance loss's
#     gradient, d aux / d s[t, i] = alpha_1 * f_i / T;
#   * shared experts have gate 1, so their output gradient is dh itself.
def _sigmoid(z: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-z))


def swiglu_ffn_backward(x, w_gate, w_up, w_down, dy):
    """Gradients of y = W_down (SiLU(W_gate x) * (W_up x)) over rows x [n, d], given
    dy = dL/dy [n, d].  With a = W_gate x, b = W_up x and SiLU'(a) = sigma(a) (1 + a
    (1 - sigma(a))): dhid = dy W_down, da = dhid * b * SiLU'(a), db = dhid * SiLU(a).
    Returns (dx [n, d], dW_gate [I, d], dW_up [I, d], dW_down [d, I])."""
    x = widen(x)
    wg, wu, wd = widen(w_gate), widen(w_up), widen(w_down)
    dy = np.asarray(dy, dtype=np.float64)
    a = x @ wg.T
    b = x @ wu.T
    sg = _sigmoid(a)
    silu = a * sg
    dhid = dy @ wd
    da = dhid * b * (sg * (1.0 + a * (1.0 - sg)))
    db = dhid * silu
    return da @ wg + db @ wu, da.T @ x, db.T @ x, dy.T @ (silu * b)


@dataclasses.dataclass
class LayerGrads:
    du: np.ndarray            # [T, d]
    d_centroids: np.ndarray   # [N_r, d]
    d_bias: np.ndarray        # [N_r] (of the per-expert logit bias, zero or not)
    d_w_gate: np.ndarray      # [n_shared + N_r, I, d]
    d_w_up: np.ndarray        # [n_shared + N_r, I, d]
    d_w_down: np.ndarray      # [n_shared + N_r, d, I]


def moe_backward(u, centroids, w_gate, w_up, w_down, n_shared: int, top_k: int,
                 alpha1: float, dh, d_aux: float = 0.0, bias=None) -> LayerGrads:
    """Gradients of L = sum_t dh_t . h_t + d_aux * aux for the layer of moe_forward (same
    argument layouts; dh [T, d]).  The routing is recomputed exactly as in the forward."""
    x = widen(u)
    T, d = x.shape
    cen = widen(centroids)
    n_routed = cen.shape[0]
    dh = np.asarray(dh, dtype=np.float64)
    r = route(x, centroids, top_k, bias)
    counts, f, P, aux = balance_stats(r.s, r.topk_idx, n_routed, alpha1)
    G = n_shared + n_routed
    inter = np.asarray(w_gate).shape[1]
    d_wg = np.zeros((G, inter, d))
    d_wu = np.zeros((G, inter, d))
    d_wd = np.zeros((G, d, inter))
    du = dh.copy()                                        # the residual
    for j in range(n_shared):                             # gate 1
        dx, d_wg[j], d_wu[j], d_wd[j] = swiglu_ffn_backward(x, w_gate[j], w_up[j], w_down[j], dh)
        du += dx
    dg = np.zeros((T, top_k))                             # dL / d g[t, k]
    for e in range(n_routed):
        tok, slot = np.nonzero(r.topk_idx == e)
        if tok.size == 0:
            continue
        ge = n_shared + e
        xe = x[tok]
        dg[tok, slot] = np.sum(dh[tok] * swiglu_ffn(xe, w_gate[ge], w_up[ge], w_down[ge]), axis=1)
        dy = r.topk_w[tok, slot][:, None] * dh[tok]
        dx, d_wg[ge], d_wu[ge], d_wd[ge] = swiglu_ffn_backward(xe, w_gate[ge], w_up[ge], w_down[ge], dy)
        du[tok] += dx                                     # a token picks an expert once
    # affinities: the chosen gates, and the balance loss through P_i
    ds = np.zeros((T, n_routed))
    ds[np.arange(T)[:, None], r.topk_idx] = dg
    ds += float(d_aux) * float(alpha1) * f[None, :] / T
    # softmax: dl = s * (ds - sum_i s_i ds_i), row by row
    dl = r.s * (ds - np.sum(r.s * ds, axis=1, keepdims=True))
    du += dl @ cen
    return LayerGrads(du=du, d_centroids=dl.T @ x, d_bias=dl.sum(axis=0), d_w_gate=d_wg,
                      d_w_up=d_wu, d_w_down=d_wd)


# ---------------------------------------------------------------- brute force (tiny inputs)
def _py_silu(z: float) -> float:
    if z >= 0.0:
        return z / (1.0 + math.exp(-z))
    ez = math.exp(z)
    return z * ez / (1.0 + ez)


def brute_force_layer(u, centroids, w_gate, w_up, w_down, n_shared: int, top_k: int,
                      alpha1: float, bias=None):
    """Token-at-a-time scalar restatement of the layer in pure Python floats (fp64).

    Routing per token: dot products with every centroid, a max-subtracted softmax over
    the routed experts, then k rounds of "take the largest remaining logit, earliest
    index on equality" (a selection procedure independent of the sort used above).
    For tiny shapes only.  Returns (h, topk_idx, topk_w, counts, aux) as Python lists.
    """
    U = widen(u).tolist()
    E = widen(centroids).tolist()
    B = None if bias is None else widen(bias).tolist()
    Wg, Wu, Wd = widen(w_gate).tolist(), widen(w_up).tolist(), widen(w_down).tolist()
    T, n_routed = len(U), len(E)
    d = len(U[0])
    inter = len(Wg[0])

    def ffn(j, x):
        mid = []
        for a in range(inter):
            g = sum(Wg[j][a][k] * x[k] for k in range(d))
            v = sum(Wu[j][a][k] * x[k] for k in range(d))
            mid.append(_py_silu(g) * v)
        return [sum(Wd[j][o][a] * mid[a] for a in range(inter)) for o in range(d)]

    H, IDX, W = [], [], []
    counts = [0] * n_routed
    psum = [0.0] * n_routed
    for t in range(T):
        x = U[t]
        logit = [sum(x[k] * E[i][k] for k in range(d)) + (B[i] if B else 0.0)
                 for i in range(n_routed)]
        m = max(logit)
        ex = [math.exp(v - m) for v in logit]
        tot = sum(ex)
        s = [v / tot for v in ex]
        taken = [False] * n_routed
        picks = []
        for _ in range(top_k):
            best = -1
            for i in range(n_routed):
                if not taken[i] and (best < 0 or logit[i] > logit[best]):
                    best = i
            taken[best] = True
            picks.append(best)
        out = list(x)
        for j in range(n_shared):
            y = ffn(j, x)
            out = [o + v for o, v in zip(out, y)]
        for i in picks:
            y = ffn(n_shared + i, x)
            out = [o + s[i] * v for o, v in zip(out, y)]
            counts[i] += 1
        for i in range(n_routed):
            psum[i] += s[i]
        H.append(out)
        IDX.append(picks)
        W.append([s[i] for i in picks])
    aux = alpha1 * sum((counts[i] / T) * (psum[i] / T) for i in range(n_routed))
    return H, IDX, W, counts, aux
