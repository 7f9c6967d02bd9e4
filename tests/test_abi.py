"""The C-ABI library: builds for sm_100a, loads, exports every declared entry point, and
rejects bad arguments without touching a GPU (CPU only)."""
import ctypes

import pytest

from mixture_experts_layer_65_b200 import _lib, build


@pytest.fixture(scope="module")
def L():
    build.build()
    return _lib.lib()


def test_every_declared_symbol_is_exported(L):
    syms = _lib.header_symbols()
    assert {"moe_create", "moe_forward", "moe_destroy", "moe_last_error"} <= set(syms)
    missing = [s for s in syms if not hasattr(L, s)]
    assert not missing, missing


def test_abi_version(L):
    assert L.moe_abi_version() == 1


def _cfg(**kw):
    base = dict(T=128, d=256, n_routed=16, n_shared=1, top_k=4, inter=128,
                dtype=_lib.MOE_BF16, alpha1=0.01, centroids=8, logit_bias=None,
                w_gate=8, w_up=8, w_down=8)
    base.update(kw)
    return _lib.MoeCfg(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(T=0), _lib.MOE_ERR_INVALID_ARG),
    (dict(T=(1 << 24) + 1), _lib.MOE_ERR_INVALID_ARG),
    (dict(top_k=17, n_routed=32), _lib.MOE_ERR_UNSUPPORTED),
    (dict(top_k=5, n_routed=4), _lib.MOE_ERR_INVALID_ARG),
    (dict(n_routed=257), _lib.MOE_ERR_UNSUPPORTED),
    (dict(d=100), _lib.MOE_ERR_UNSUPPORTED),
    (dict(inter=96), _lib.MOE_ERR_UNSUPPORTED),
    (dict(dtype=_lib.MOE_FP32, d=6), _lib.MOE_ERR_UNSUPPORTED),
    (dict(dtype=7), _lib.MOE_ERR_INVALID_ARG),
    (dict(w_down=None), _lib.MOE_ERR_INVALID_ARG),
    (dict(n_shared=-1), _lib.MOE_ERR_INVALID_ARG),
    (dict(dtype=_lib.MOE_BF16_E4M3_GATEUP, d=192), _lib.MOE_ERR_UNSUPPORTED),   # d % 128
    (dict(dtype=_lib.MOE_BF16_E4M3_GATEUP, inter=96), _lib.MOE_ERR_UNSUPPORTED),
])
def test_create_rejects_invalid_config(L, kw, status):
    h = ctypes.c_void_p(123)
    cfg = _cfg(**kw)
    assert L.moe_create(ctypes.byref(cfg), ctypes.byref(h)) == status
    assert h.value is None
    assert len(L.moe_last_error()) > 0


def test_null_arguments_are_rejected(L):
    assert L.moe_create(None, ctypes.byref(ctypes.c_void_p())) == _lib.MOE_ERR_INVALID_ARG
    assert b"NULL" in L.moe_last_error()
    assert L.moe_forward(None, 16, 16, 16, 16, 16, 16, None) == _lib.MOE_ERR_INVALID_ARG
    assert L.moe_forward_host(None, 16, 16, 16, 16, 16, 16, None) == _lib.MOE_ERR_INVALID_ARG
    assert L.moe_device_status(None, None) == _lib.MOE_ERR_INVALID_ARG
    assert L.moe_forward_host_pipelined(None, 16, 16, 16, 16, 16, 16, None) == _lib.MOE_ERR_INVALID_ARG
    assert L.moe_pipeline_wait(None, None) == _lib.MOE_ERR_INVALID_ARG
    assert L.moe_expert_psum(None, 16, None) == _lib.MOE_ERR_INVALID_ARG
    assert L.moe_balance_loss(None, 16, 4, 10, 0.01, 16, None) == _lib.MOE_ERR_INVALID_ARG
    assert L.moe_balance_loss(16, 16, 0, 10, 0.01, 16, None) == _lib.MOE_ERR_INVALID_ARG
    assert L.moe_kernels_per_forward(None) == 0
    assert L.moe_device_bytes(None) == 0
    L.moe_destroy(None)   # NULL-safe


def test_product_path_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        _lib.lib()


def test_wait_selftest_validates_arguments_before_touching_the_device():
    L = _lib.lib()
    code = ctypes.c_int32(0)
    assert L.moe_selftest_wait_timeout(2, 50_000_000, ctypes.byref(code)) == _lib.MOE_ERR_INVALID_ARG
    assert L.moe_selftest_wait_timeout(0, 10, ctypes.byref(code)) == _lib.MOE_ERR_INVALID_ARG
    assert L.moe_selftest_wait_timeout(0, 50_000_000, None) == _lib.MOE_ERR_INVALID_ARG


def _unbound_layer():
    """A binding object with the sizes of a small layer but no library handle: argument
    validation must reject bad tensors before anything reaches the library."""
    import torch
    from mixture_experts_layer_65_b200.layer import MoELayer
    L = object.__new__(MoELayer)
    L.T, L.d, L.top_k, L.n_routed = 8, 64, 2, 4
    L.torch_dtype, L.device, L._h = torch.bfloat16, torch.device("cuda", 0), None
    return L


def test_binding_rejects_host_or_misshapen_tensors_before_the_library():
    import torch
    from mixture_experts_layer_65_b200.layer import MoEOutput
    L = _unbound_layer()
    with pytest.raises(ValueError, match="CUDA tensor"):
        L.forward(torch.zeros(8, 64, dtype=torch.bfloat16))          # host input
    host = MoEOutput(h=torch.zeros(8, 64, dtype=torch.bfloat16),
                     topk_idx=torch.zeros(8, 2, dtype=torch.int32),
                     topk_w=torch.zeros(8, 2), expert_counts=torch.zeros(4, dtype=torch.int32),
                     aux_loss=torch.zeros(1))
    with pytest.raises(ValueError, match="CUDA tensor"):
        L._check_outputs(host)                                          # host outputs
    short = host._replace(topk_w=torch.zeros(8, 1))
    with pytest.raises(ValueError, match="topk_w"):
        L._check_host_outputs(short)                                    # too small to copy into
    L._check_host_outputs(host._replace(topk_idx=None, aux_loss=None))  # optional outputs
    with pytest.raises(ValueError, match="contiguous host"):
        L.forward_host(torch.zeros(64, 8, dtype=torch.bfloat16).t(), host)   # not contiguous
