"""Per-kernel parity: the intermediates of one forward against the oracle.

Besides the layer outputs (tests/test_gpu_parity.py), the workspace a forward leaves
behind is checked step by step:
  * the row copy (fused into the gate/up GEMM, or the permute kernel): every (token, slot)
    has its own row, inside its expert's group, tokens of an expert in ascending order,
    and the row holds the token's values byte for byte (for e4m3 gate/up layers: the
    oracle's quantised token row, byte for byte);
  * the gate/up GEMM: each routed row's SwiGLU activation, and the shared group's
    activations (experts side by side), against the oracle's;
  * the down GEMM: each routed row's expert output and the shared experts' summed output.
"""
import numpy as np
import pytest
import torch

from mixture_experts_layer_65_b200 import build
from mixture_experts_layer_65_b200 import workloads as W
from mixture_experts_layer_65_b200.layer import MoELayer, to_device_tensor
from oracle import moe_oracle as O
from tests import parity as P

pytestmark = pytest.mark.gpu

SPECS = [
    dict(T=333, d=256, n_shared=2, n_routed=16, inter=192, top_k=4),   # row copy in the GEMM
    dict(T=700, d=256, n_shared=0, n_routed=16, inter=128, top_k=2),   # permute kernel
    dict(T=96, d=256, n_shared=2, n_routed=16, inter=128, top_k=4),    # decode-sized: copy in the GEMM
    # decode-sized with ragged weight tiles: the last gate/up tile holds 64 of its 128
    # features (inter % 128 == 64) and the last down tile 128 of its 256 (d % 256 == 128)
    dict(T=40, d=384, n_shared=1, n_routed=8, inter=192, top_k=2),
    dict(T=17, d=128, n_shared=0, n_routed=8, inter=64, top_k=1),
]


@pytest.fixture(scope="module", autouse=True)
def _lib_ready():
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def _close(got: np.ndarray, ref: np.ndarray, what: str):
    err = np.abs(got - ref).max() / max(np.abs(ref).max(), 1e-30)
    assert err <= P.TOL["bf16"], (what, err)
    return err


@pytest.mark.parametrize("e4m3", [False, True], ids=["bf16", "e4m3_gate_up"])
@pytest.mark.parametrize("spec", SPECS, ids=lambda s: "T{T}_s{n_shared}_r{n_routed}_k{top_k}".format(**s))
def test_intermediates_match_the_oracle(spec, e4m3):
    w = W.make_workload("16b_prefill", alpha1=0.001, gate_up_e4m3=e4m3, **spec)
    layer = MoELayer.from_workload(w)
    out = layer.forward(to_device_tensor(w.u, "cuda"))
    torch.cuda.synchronize()
    layer.device_status()
    T, d, I, K, ks, nr = w.T, w.d, w.inter, w.top_k, w.n_shared, w.n_routed
    idx = out.topk_idx.cpu().numpy()
    slot = layer.debug_buffer("slot_row").cpu().numpy().reshape(T, K)
    grp = layer.debug_buffer("grp_row").cpu().numpy()
    hs_first = 1 if ks else 0

    # row copy: a bijection onto each expert's rows, tokens in ascending order
    assert np.unique(slot).size == slot.size
    for e in range(nr):
        ts, kk = np.nonzero(idx == e)
        order = np.argsort(ts, kind="stable")
        np.testing.assert_array_equal(slot[ts, kk][order], grp[hs_first + e] + np.arange(ts.size))
    xp = layer.debug_buffer("xp").cpu()
    rows = slot.reshape(-1)
    toks = np.repeat(np.arange(T), K)
    row_tok = layer.debug_buffer("row_tok").cpu().numpy()
    if row_tok.size:   # decode-sized layer: the scan recorded the token of every routed row
        np.testing.assert_array_equal(row_tok[rows], toks)
    if e4m3:
        xp8 = xp.view(-1, d)[torch.from_numpy(rows)]
        got = xp8.view(torch.float8_e4m3fn).to(torch.float64).numpy()
        q, _ = O.quantize_rows_e4m3(w.u)
        np.testing.assert_array_equal(got, q[toks])
    else:
        got = xp.view(-1, d)[torch.from_numpy(rows)].view(torch.int16).numpy().view(np.uint16)
        np.testing.assert_array_equal(got, w.u[toks])

    # gate/up and down GEMMs, routed experts
    hr = _f64(layer.debug_buffer("hr")).reshape(-1, I)
    yr = _f64(layer.debug_buffer("yr")).reshape(-1, d)
    for e in range(nr):
        ts, kk = np.nonzero(idx == e)
        if ts.size == 0:
            continue
        x = w.u[ts]
        hid = O.swiglu_hidden(x, w.w_gate[ks + e], w.w_up[ks + e], e4m3)
        y = O.swiglu_ffn(x, w.w_gate[ks + e], w.w_up[ks + e], w.w_down[ks + e], e4m3)
        r = slot[ts, kk]
        _close(hr[r], hid, f"hidden of expert {e}")
        _close(yr[r], y, f"output of expert {e}")

    # shared group
    if ks:
        hs = _f64(layer.debug_buffer("hs")).reshape(-1, ks * I)[:T]
        ys = _f64(layer.debug_buffer("ys")).reshape(-1, d)[:T]
        y_ref = np.zeros((T, d))
        for j in range(ks):
            _close(hs[:, j * I:(j + 1) * I], O.swiglu_hidden(w.u, w.w_gate[j], w.w_up[j], e4m3),
                   f"hidden of shared expert {j}")
            y_ref += O.swiglu_ffn(w.u, w.w_gate[j], w.w_up[j], w.w_down[j], e4m3)
        _close(ys, y_ref, "shared output")
    else:
        assert layer.debug_buffer("hs").numel() == 0


@pytest.mark.parametrize("name", ["16b_prefill", "145b"])
def test_full_size_intermediates_on_sampled_rows_of_every_expert(name):
    """At full size (the launch configuration the benchmark times): for every routed expert,
    its first and last rows and six random ones (the 145B layer's Zipf-skewed expert 0 holds
    ~32 K rows, the longest tile chains), the SwiGLU activation and the expert output
    against the oracle; the shared group's activations and summed output on sampled tokens;
    the row copy byte for byte on those rows."""
    w = W.make_workload(name)
    layer = MoELayer.from_workload(w)
    out = layer.forward(to_device_tensor(w.u, "cuda"))
    torch.cuda.synchronize()
    layer.device_status()
    T, d, I, K, ks, nr = w.T, w.d, w.inter, w.top_k, w.n_shared, w.n_routed
    idx = out.topk_idx.cpu().numpy()
    slot = layer.debug_buffer("slot_row").cpu().numpy().reshape(T, K)
    rng = np.random.default_rng(7)
    picks = []                                  # (token, slot) pairs to check
    for e in range(nr):
        ts, kk = np.nonzero(idx == e)
        if ts.size == 0:
            continue
        order = np.argsort(slot[ts, kk])
        sel = np.unique(np.concatenate([[0, ts.size - 1], rng.integers(0, ts.size, 6)]))
        picks += [(ts[order[i]], kk[order[i]], e) for i in sel]
    picks = np.array(picks)
    rows = torch.from_numpy(slot[picks[:, 0], picks[:, 1]].astype(np.int64)).cuda()
    xp = layer.debug_buffer("xp").view(-1, d)[rows].cpu().view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(xp, w.u[picks[:, 0]])
    hr = _f64(layer.debug_buffer("hr").view(-1, I)[rows])
    yr = _f64(layer.debug_buffer("yr").view(-1, d)[rows])
    worst_h = worst_y = 0.0
    for e in np.unique(picks[:, 2]):
        m = picks[:, 2] == e
        x = w.u[picks[m, 0]]
        g = ks + e
        worst_h = max(worst_h, _close(hr[m], O.swiglu_hidden(x, w.w_gate[g], w.w_up[g]), f"hidden {e}"))
        worst_y = max(worst_y, _close(yr[m], O.swiglu_ffn(x, w.w_gate[g], w.w_up[g], w.w_down[g]),
                                      f"output {e}"))
    toks = np.unique(np.concatenate([[0, T - 1], rng.integers(0, T, 30)]))
    tt = torch.from_numpy(toks).cuda()
    hs = _f64(layer.debug_buffer("hs").view(-1, ks * I)[tt])
    ys = _f64(layer.debug_buffer("ys").view(-1, d)[tt])
    y_ref = np.zeros((toks.size, d))
    for j in range(ks):
        _close(hs[:, j * I:(j + 1) * I], O.swiglu_hidden(w.u[toks], w.w_gate[j], w.w_up[j]),
               f"hidden of shared expert {j}")
        y_ref += O.swiglu_ffn(w.u[toks], w.w_gate[j], w.w_up[j], w.w_down[j])
    _close(ys, y_ref, "shared output")
    print(name, f"{len(picks)} routed rows of {len(np.unique(picks[:, 2]))} experts: "
                f"hidden err {worst_h:.2e}, output err {worst_y:.2e}")
    layer.close()


@pytest.mark.parametrize("name,spec", [
    ("paired_shared", dict(T=333, d=256, n_shared=2, n_routed=16, inter=192, top_k=4)),
    ("paired_no_shared", dict(T=700, d=256, n_shared=0, n_routed=16, inter=128, top_k=2)),
    ("decode_sized", dict(T=96, d=256, n_shared=2, n_routed=16, inter=128, top_k=4)),
])
def test_per_kernel_timing_records_every_slot(name, spec):
    """moe_timing_begin / moe_timing_end (the benchmark's per-kernel slots) on every launch
    path: each slot of each recorded forward is recorded, whether or not a kernel runs in it
    (the permute and, on decode-sized layers, the down GEMM run inside other kernels)."""
    w = W.make_workload("16b_prefill", alpha1=0.001, **spec)
    layer = MoELayer.from_workload(w)
    u = to_device_tensor(w.u, "cuda")
    out = layer.alloc_outputs()
    layer.forward(u, out)
    layer.timing_begin(3)
    for _ in range(3):
        layer.forward(u, out)
    ms, n = layer.timing_end()
    layer.device_status()
    assert n == 3
    assert all(np.isfinite(v) and v >= 0.0 for v in ms.values()), ms
    assert ms["gate_up_gemm"] > 0.0 and (name == "decode_sized" or ms["down_gemm"] > 0.0)
    layer.close()
