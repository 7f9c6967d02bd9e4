"""Bounded waits give up and report, without faulting or hanging the GPU.

Every spin of the library's kernels (on an mbarrier phase, or on the fused row copy's
grid-wide counter) has a time limit after which the kernel records an error code and
returns.  moe_selftest_wait_timeout runs one tiny kernel whose wait nothing will satisfy,
with a short limit; the test checks the recorded code and that a normal forward still
runs correctly on the same context afterwards.
"""
import ctypes
import time

import pytest
import torch

from mixture_experts_layer_65_b200 import build
from mixture_experts_layer_65_b200 import workloads as W
from mixture_experts_layer_65_b200._lib import MOE_OK, lib
from mixture_experts_layer_65_b200.layer import MoELayer, to_device_tensor
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib_ready():
    build.build()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


@pytest.mark.parametrize("kind,code", [(0, 0x102), (1, 0x105)], ids=["mbarrier", "counter"])
def test_wait_runs_out_and_reports(kind, code):
    torch.cuda.init()
    got = ctypes.c_int32(-1)
    t0 = time.perf_counter()
    st = lib().moe_selftest_wait_timeout(kind, 50_000_000, ctypes.byref(got))   # 50 ms
    dt = time.perf_counter() - t0
    assert st == MOE_OK
    assert got.value == code
    assert 0.04 < dt < 5.0, dt        # it waited about the limit, then gave up


def test_context_usable_after_a_wait_ran_out():
    got = ctypes.c_int32(-1)
    assert lib().moe_selftest_wait_timeout(0, 20_000_000, ctypes.byref(got)) == MOE_OK
    assert got.value == 0x102
    w = W.make_workload("16b_prefill", T=300, d=256, n_shared=1, n_routed=16, inter=128, top_k=4,
                        alpha1=0.01)
    layer = MoELayer.from_workload(w)
    out = layer.forward(to_device_tensor(w.u, "cuda"))
    torch.cuda.synchronize()
    layer.device_status()
    P.compare(w, P.fetch(out))
