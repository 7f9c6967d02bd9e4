"""moe_route_noalloc: the router step for callers that cannot allocate device memory.

Callers whose GPU memory belongs to another allocator (a framework's caching allocator
or a serving engine's arena), or that run on a latency-critical path where cudaMalloc
would synchronise the device, cannot let the library allocate a workspace.  This entry
point keeps its scratch in a fixed device array inside the library instead.  The GPU
test calls it through the C-ABI twice in a row and checks every output against the fp64
oracle and against moe_forward's for the same layer; the CPU test checks that oversized
requests are refused before any GPU work.  (Kept in its own file, collected last.)
"""
import ctypes

import numpy as np
import pytest

from mixture_experts_layer_65_b200 import _lib, build
from mixture_experts_layer_65_b200 import workloads as W
from tests import parity as P


@pytest.fixture(scope="module")
def L():
    build.build()
    return _lib.lib()


def test_noalloc_rejects_sizes_beyond_the_maximum(L):
    fake = 1 << 20   # aligned non-NULL stand-ins: the call must fail before using them
    args = dict(u=fake, c=fake, b=None, T=128, d=256, nr=16, k=4)

    def call(**kw):
        a = dict(args, **kw)
        return L.moe_route_noalloc(a["u"], a["c"], a["b"], a["T"], a["d"], a["nr"], a["k"], 0.01,
                                   fake, fake, fake, fake, None, None)

    assert call(T=16385) == _lib.MOE_ERR_UNSUPPORTED
    assert b"16384" in L.moe_last_error()
    assert call(nr=257, k=4) == _lib.MOE_ERR_UNSUPPORTED
    assert call(k=17, nr=64) == _lib.MOE_ERR_UNSUPPORTED
    assert call(d=96) == _lib.MOE_ERR_UNSUPPORTED
    assert call(u=None) == _lib.MOE_ERR_INVALID_ARG
    assert call(c=fake + 8) == _lib.MOE_ERR_INVALID_ARG


CASES = [
    ("16b_prefill", {}),                                            # the 16B router, T = 16384
    ("2b", dict(T=3000)),                                           # N_r = 63, ragged T
    ("145b", dict(T=2000, n_shared=1, inter=64)),                   # d = 4096, N_r = 128, top-12, Zipf bias
    ("16b_decode", {}),                                             # T = 64: moe_forward routes on SIMT
]


@pytest.mark.gpu
@pytest.mark.parametrize("name,overrides", CASES, ids=[c[0] for c in CASES])
def test_noalloc_matches_moe_forward(L, name, overrides):
    """Two calls in a row, each against the fp64 oracle (routing sets exact outside near
    ties, gates within their rounding bound, counts, loss) and against moe_forward on the
    same layer: bit for bit where moe_forward runs the same router (T > 128); for a
    decode-sized batch, where moe_forward sums the logits on a SIMT kernel, the same routed
    sets outside near ties and gates within both kernels' rounding bounds of the oracle."""
    import torch

    from mixture_experts_layer_65_b200.layer import MoELayer, to_device_tensor
    from oracle import moe_oracle as O

    w = W.make_workload(name, **overrides)
    r = O.route(w.u, w.centroids, w.top_k, w.logit_bias)
    _, _, P_ref, _ = O.balance_stats(r.s, r.topk_idx, w.n_routed, w.alpha1)
    layer = MoELayer.from_workload(w)
    u = to_device_tensor(w.u, "cuda")
    ref = layer.forward(u)
    torch.cuda.synchronize()
    layer.device_status()
    same_kernels = P.router_path(w) == "mma16"
    cen = to_device_tensor(w.centroids, "cuda")
    bias = None if w.logit_bias is None else torch.from_numpy(w.logit_bias).cuda()
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):   # two calls in a row share (and overwrite) the scratch array
        idx = torch.full((w.T, w.top_k), -1, dtype=torch.int32, device="cuda")
        wts = torch.full((w.T, w.top_k), float("nan"), dtype=torch.float32, device="cuda")
        cnt = torch.full((w.n_routed,), -1, dtype=torch.int32, device="cuda")
        aux = torch.full((1,), float("nan"), dtype=torch.float32, device="cuda")
        derr = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        st = L.moe_route_noalloc(u.data_ptr(), cen.data_ptr(),
                                 None if bias is None else bias.data_ptr(), w.T, w.d, w.n_routed,
                                 w.top_k, w.alpha1, idx.data_ptr(), wts.data_ptr(),
                                 cnt.data_ptr(), aux.data_ptr(), derr.data_ptr(), stream)
        assert st == _lib.MOE_OK, L.moe_last_error()
        torch.cuda.synchronize()
        assert int(derr.item()) == 0, f"call {call}: device error {int(derr.item()):#x}"
        rep = {}
        keep = P.compare_routing(w, r, idx.cpu().numpy().astype(np.int64),
                                 wts.cpu().numpy().astype(np.float64),
                                 cnt.cpu().numpy().astype(np.int64), float(aux.item()), P_ref,
                                 rep, path="mma16")
        print(name, call, rep)
        if same_kernels:
            assert torch.equal(idx, ref.topk_idx), f"call {call}: routed indices differ"
            assert torch.equal(cnt, ref.expert_counts), f"call {call}: expert counts differ"
            assert torch.equal(wts, ref.topk_w), f"call {call}: gates differ"
            assert torch.equal(aux, ref.aux_loss), f"call {call}: balance loss differs"
        else:
            a = np.sort(idx.cpu().numpy(), axis=1)[keep]
            b = np.sort(ref.topk_idx.cpu().numpy(), axis=1)[keep]
            np.testing.assert_array_equal(a, b)
    layer.close()
