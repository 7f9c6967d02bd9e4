"""Backward pass on the GPU against the oracle's pinned moe_backward (fp64).

The library's gradients of L = sum_t dh_t . h_t + d_aux * aux -- du, d_centroids, d_bias and
the expert weight gradients -- element by element against the oracle on the same
bf16-valued inputs and dh.  Tolerance,
the forward's form: max|x - x_ref| <= 2e-2 max|x_ref| for each output, and the same for the
expert part of du (du - dh).  Derivation: the GPU path rounds to bf16 (relative 2^-9) at
most four times on any path into du (dY, dHmid, [da db], dX) with fp32 accumulation in
between, about 4 * 2^-9 = 0.8 % of the expert part; d_centroids and d_bias are fp32 sums of
dl, whose inputs (the gates' gradients dh . Y) carry one bf16 rounding of Y; a weight
gradient is an fp32-accumulated sum over the expert's rows of products of two bf16 factors
that carry at most three such roundings, compared against each expert's own maximum.
"""
import numpy as np
import pytest
import torch

from mixture_experts_layer_65_b200 import build
from mixture_experts_layer_65_b200 import workloads as W
from mixture_experts_layer_65_b200.layer import MoELayer, to_device_tensor
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu
TOL = 2e-2


@pytest.fixture(scope="module", autouse=True)
def _lib_ready():
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _err(got, ref):
    return float(np.abs(got - ref).max()) / max(float(np.abs(ref).max()), 1e-30)


SPECS = [
    ("shared2_r16", dict(T=333, d=256, n_shared=2, n_routed=16, inter=192, top_k=4), 0.0),
    ("no_shared", dict(T=700, d=256, n_shared=0, n_routed=16, inter=128, top_k=2), 1.0),
    ("zipf_bias", dict(T=1000, d=256, n_shared=1, n_routed=16, inter=128, top_k=4, zipf_s=1.1), 1.0),
    ("n63_top7", dict(T=520, d=320, n_shared=1, n_routed=63, inter=128, top_k=7), 1.0),
    ("16b_shape", dict(T=2048, d=2048, n_shared=2, n_routed=64, inter=1408, top_k=6), 1.0),
]


@pytest.mark.parametrize("name,spec,d_aux", SPECS, ids=[s[0] for s in SPECS])
def test_backward_matches_the_oracle(name, spec, d_aux):
    w = W.make_workload("16b_prefill", alpha1=0.001, **spec)
    rng = np.random.default_rng(11)
    dh_bits = W.f32_to_bf16_bits(rng.standard_normal((w.T, w.d), dtype=np.float32))
    layer = MoELayer.from_workload(w)
    layer.backward_prepare()
    u = to_device_tensor(w.u, "cuda")
    out = layer.forward(u)
    dh = to_device_tensor(dh_bits, "cuda")
    grads = [layer.backward(u, out, dh, d_aux) for _ in range(2)]
    torch.cuda.synchronize()
    layer.device_status()
    # deterministic: the second backward is bit for bit the first
    for a, b in zip(grads[0], grads[1]):
        assert torch.equal(a, b)
    du, dcen, dbias, dwg, dwu, dwd = (g.float().cpu().numpy().astype(np.float64) for g in grads[0])
    ref = O.moe_backward(w.u, w.centroids, w.w_gate, w.w_up, w.w_down, w.n_shared, w.top_k,
                         w.alpha1, O.widen(dh_bits), d_aux=d_aux, bias=w.logit_bias)
    dh64 = O.widen(dh_bits)
    e_du = _err(du, ref.du)
    slack = 2.0 ** -8 * np.maximum(np.abs(du), np.abs(ref.du))   # du's own bf16 rounding
    e_part = float(np.maximum(np.abs(du - ref.du) - slack, 0).max()) / float(np.abs(ref.du - dh64).max())
    e_cen, e_bias = _err(dcen, ref.d_centroids), _err(dbias, ref.d_bias)
    # weight gradients per expert (an expert's own scale: routed experts see few tokens)
    e_w = 0.0
    for name_w, got, want in (("d_w_gate", dwg, ref.d_w_gate), ("d_w_up", dwu, ref.d_w_up),
                              ("d_w_down", dwd, ref.d_w_down)):
        for g in range(got.shape[0]):
            if not np.any(want[g]):   # an expert without tokens: exactly zero
                assert not np.any(got[g]), (name_w, g)
                continue
            eg = _err(got[g], want[g])
            e_w = max(e_w, eg)
            assert eg <= TOL, (name_w, g, eg)
    print(f"{name}: du {e_du:.2e}, du expert part {e_part:.2e}, d_centroids {e_cen:.2e}, "
          f"d_bias {e_bias:.2e}, weight gradients (worst expert) {e_w:.2e}")
    assert e_du <= TOL and e_part <= TOL
    assert e_cen <= TOL and e_bias <= TOL
    layer.close()


def test_weight_gradients_into_16_byte_aligned_buffers():
    """The interface asks 16-byte alignment of the gradient buffers; the weight-gradient
    epilogue stores 32 bytes per thread only when all three are 32-byte aligned.  Buffers
    offset by 16 bytes take the other path and must get the same bits."""
    from mixture_experts_layer_65_b200._lib import check, lib
    from mixture_experts_layer_65_b200.layer import _ptr
    w = W.make_workload("16b_prefill", alpha1=0.001, **SPECS[0][1])
    rng = np.random.default_rng(5)
    layer = MoELayer.from_workload(w)
    layer.backward_prepare()
    u = to_device_tensor(w.u, "cuda")
    out = layer.forward(u)
    dh = to_device_tensor(W.f32_to_bf16_bits(rng.standard_normal((w.T, w.d), dtype=np.float32)), "cuda")
    du, dcen, dbias, dwg, dwu, dwd = layer.backward(u, out, dh, 1.0)
    assert all(t.data_ptr() % 32 == 0 for t in (dwg, dwu, dwd))

    def off16(t):   # same shape, storage starting 16 bytes past a 256-byte boundary
        buf = torch.empty(t.numel() + 4, dtype=t.dtype, device=t.device)
        return buf[4:].view(t.shape)

    du2, dcen2, dbias2 = torch.empty_like(du), torch.empty_like(dcen), torch.empty_like(dbias)
    dwg2, dwu2, dwd2 = off16(dwg), off16(dwu), off16(dwd)
    assert all(t.data_ptr() % 32 == 16 for t in (dwg2, dwu2, dwd2))
    s = torch.cuda.current_stream()
    check(lib().moe_backward(layer._h, _ptr(u), _ptr(out.topk_idx), _ptr(out.topk_w),
                             _ptr(out.expert_counts), _ptr(dh), 1.0, _ptr(du2), _ptr(dcen2),
                             _ptr(dbias2), _ptr(dwg2), _ptr(dwu2), _ptr(dwd2), s.cuda_stream))
    torch.cuda.synchronize()
    layer.device_status()
    for a, b in ((du, du2), (dcen, dcen2), (dbias, dbias2), (dwg, dwg2), (dwu, dwu2), (dwd, dwd2)):
        assert torch.equal(a, b)
    layer.close()


def test_backward_refuses_unsupported_layers():
    from mixture_experts_layer_65_b200 import _lib
    w = W.make_workload("tiny")   # fp32 layer
    layer = MoELayer.from_workload(w)
    with pytest.raises(_lib.MoeError) as e:
        layer.backward_prepare()
    assert e.value.status == _lib.MOE_ERR_UNSUPPORTED
    layer.close()
