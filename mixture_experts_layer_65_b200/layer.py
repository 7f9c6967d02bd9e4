"""Python face of the C-ABI: a DeepSeekMoE layer whose forward pass runs in libmoe.so.

PyTorch is used for device memory and streams only; every step of the forward pass
(router, scan/permute, grouped expert GEMMs, combine, balance statistics) runs in the
library's CUDA kernels.  There is no CPU or PyTorch fallback: a missing library or a
non-B200 device raises.
"""
from __future__ import annotations

import ctypes
from typing import NamedTuple

import numpy as np
import torch

from . import _lib
from ._lib import MoeCfg, check, lib


class MoEOutput(NamedTuple):
    h: torch.Tensor              # [T, d] layer output (dtype of the layer)
    topk_idx: torch.Tensor       # [T, top_k] int32, descending logit order
    topk_w: torch.Tensor         # [T, top_k] fp32 gates
    expert_counts: torch.Tensor  # [n_routed] int32
    aux_loss: torch.Tensor       # [1] fp32


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def to_device_tensor(a: np.ndarray, device) -> torch.Tensor:
    """Upload a workload array: uint16 arrays are bf16 bit patterns, float32 stays fp32."""
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


class MoELayer:
    """One DeepSeekMoE layer (fixed token count T per instance)."""

    def __init__(self, *, T: int, d: int, n_routed: int, n_shared: int, top_k: int, inter: int,
                 dtype: str, alpha1: float, centroids: torch.Tensor, w_gate: torch.Tensor,
                 w_up: torch.Tensor, w_down: torch.Tensor, logit_bias: torch.Tensor | None = None,
                 gate_up_e4m3: bool = False, down_e4m3: bool = False):
        """gate_up_e4m3 (bf16 layers): the gate/up GEMM runs on per-row scaled e4m3
        operands (MOE_BF16_E4M3_GATEUP in include/moe.h); down_e4m3 (with gate_up_e4m3): the
        down GEMM too (MOE_BF16_E4M3).  The weights are still given in bf16."""
        if gate_up_e4m3 and dtype != "bf16":
            raise ValueError("gate_up_e4m3 needs a bf16 layer")
        if down_e4m3 and not gate_up_e4m3:
            raise ValueError("down_e4m3 comes with gate_up_e4m3 (the MOE_BF16_E4M3 layer)")
        self.gate_up_e4m3 = gate_up_e4m3
        self.down_e4m3 = down_e4m3
        self.T, self.d, self.n_routed, self.n_shared = T, d, n_routed, n_shared
        self.top_k, self.inter, self.alpha1 = top_k, inter, alpha1
        self.dtype = dtype
        self.torch_dtype = torch.bfloat16 if dtype == "bf16" else torch.float32
        self.device = centroids.device
        for t in (centroids, w_gate, w_up, w_down):
            if not t.is_cuda or not t.is_contiguous() or t.dtype != self.torch_dtype:
                raise ValueError("weights must be contiguous CUDA tensors of the layer dtype")
        if logit_bias is not None and (logit_bias.dtype != torch.float32 or not logit_bias.is_cuda):
            raise ValueError("logit_bias must be a float32 CUDA tensor")
        cfg = MoeCfg(T=T, d=d, n_routed=n_routed, n_shared=n_shared, top_k=top_k, inter=inter,
                     dtype=(_lib.MOE_FP32 if dtype != "bf16" else
                            _lib.MOE_BF16_E4M3 if down_e4m3 else
                            _lib.MOE_BF16_E4M3_GATEUP if gate_up_e4m3 else _lib.MOE_BF16),
                     alpha1=alpha1,
                     centroids=_ptr(centroids), logit_bias=_ptr(logit_bias), w_gate=_ptr(w_gate),
                     w_up=_ptr(w_up), w_down=_ptr(w_down))
        handle = ctypes.c_void_p()
        with torch.cuda.device(self.device):
            check(lib().moe_create(ctypes.byref(cfg), ctypes.byref(handle)))
        self._h = handle

    @classmethod
    def from_workload(cls, w, device="cuda") -> "MoELayer":
        dev = torch.device(device)
        bias = None if w.logit_bias is None else torch.from_numpy(w.logit_bias).to(dev)
        return cls(T=w.T, d=w.d, n_routed=w.n_routed, n_shared=w.n_shared, top_k=w.top_k,
                   inter=w.inter, dtype=w.dtype, alpha1=w.alpha1,
                   centroids=to_device_tensor(w.centroids, dev),
                   w_gate=to_device_tensor(w.w_gate, dev), w_up=to_device_tensor(w.w_up, dev),
                   w_down=to_device_tensor(w.w_down, dev), logit_bias=bias,
                   gate_up_e4m3=getattr(w, "gate_up_e4m3", False),
                   down_e4m3=getattr(w, "down_e4m3", False))

    # -------------------------------------------------------------------------- calls
    def alloc_outputs(self) -> MoEOutput:
        dev = self.device
        return MoEOutput(
            h=torch.empty(self.T, self.d, dtype=self.torch_dtype, device=dev),
            topk_idx=torch.empty(self.T, self.top_k, dtype=torch.int32, device=dev),
            topk_w=torch.empty(self.T, self.top_k, dtype=torch.float32, device=dev),
            expert_counts=torch.empty(self.n_routed, dtype=torch.int32, device=dev),
            aux_loss=torch.empty(1, dtype=torch.float32, device=dev))

    def _check_device_tensor(self, name: str, t: torch.Tensor, shape: tuple, dtype) -> None:
        if not isinstance(t, torch.Tensor) or not t.is_cuda or t.device != self.device:
            raise ValueError(f"{name} must be a CUDA tensor on {self.device}")
        if tuple(t.shape) != shape or t.dtype != dtype or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous {list(shape)} {dtype} tensor")

    def _check_outputs(self, out: MoEOutput) -> None:
        """The library writes through these pointers: every output must be device memory of
        the layer's device with the documented shape and dtype."""
        self._check_device_tensor("h", out.h, (self.T, self.d), self.torch_dtype)
        self._check_device_tensor("topk_idx", out.topk_idx, (self.T, self.top_k), torch.int32)
        self._check_device_tensor("topk_w", out.topk_w, (self.T, self.top_k), torch.float32)
        self._check_device_tensor("expert_counts", out.expert_counts, (self.n_routed,), torch.int32)
        self._check_device_tensor("aux_loss", out.aux_loss, (1,), torch.float32)

    def _check_host_outputs(self, out: MoEOutput) -> None:
        """Host outputs are copied into whole: each must be a contiguous host tensor of the
        documented shape and dtype (topk/counts/aux may be None: not copied back)."""
        spec = (("h", (self.T, self.d), self.torch_dtype),
                ("topk_idx", (self.T, self.top_k), torch.int32),
                ("topk_w", (self.T, self.top_k), torch.float32),
                ("expert_counts", (self.n_routed,), torch.int32),
                ("aux_loss", (1,), torch.float32))
        for name, shape, dtype in spec:
            t = getattr(out, name)
            if t is None and name != "h":
                continue
            if (not isinstance(t, torch.Tensor) or t.is_cuda or tuple(t.shape) != shape
                    or t.dtype != dtype or not t.is_contiguous()):
                raise ValueError(f"{name} must be a contiguous host {list(shape)} {dtype} tensor")

    def forward(self, u: torch.Tensor, out: MoEOutput | None = None,
                stream: torch.cuda.Stream | None = None) -> MoEOutput:
        """Enqueue one forward pass on `stream` (default: the current stream)."""
        self._check_device_tensor("u", u, (self.T, self.d), self.torch_dtype)
        if out is None:
            out = self.alloc_outputs()
        else:
            self._check_outputs(out)
        s = stream or torch.cuda.current_stream(self.device)
        check(lib().moe_forward(self._h, _ptr(u), _ptr(out.h), _ptr(out.topk_idx),
                                _ptr(out.topk_w), _ptr(out.expert_counts), _ptr(out.aux_loss),
                                s.cuda_stream))
        return out

    __call__ = forward

    def forward_host(self, u: torch.Tensor, out: MoEOutput | None = None,
                     stream: torch.cuda.Stream | None = None) -> MoEOutput:
        """Forward pass on HOST tensors (pinned for overlap); copies in and out, synchronises."""
        if (u.is_cuda or u.shape != (self.T, self.d) or u.dtype != self.torch_dtype
                or not u.is_contiguous()):
            raise ValueError("u must be a contiguous host tensor of the layer shape and dtype")
        if out is not None:
            self._check_host_outputs(out)
        else:
            out = MoEOutput(
                h=torch.empty(self.T, self.d, dtype=self.torch_dtype, pin_memory=True),
                topk_idx=torch.empty(self.T, self.top_k, dtype=torch.int32, pin_memory=True),
                topk_w=torch.empty(self.T, self.top_k, dtype=torch.float32, pin_memory=True),
                expert_counts=torch.empty(self.n_routed, dtype=torch.int32, pin_memory=True),
                aux_loss=torch.empty(1, dtype=torch.float32, pin_memory=True))
        s = stream or torch.cuda.current_stream(self.device)
        check(lib().moe_forward_host(self._h, _ptr(u), _ptr(out.h), _ptr(out.topk_idx),
                                     _ptr(out.topk_w), _ptr(out.expert_counts),
                                     _ptr(out.aux_loss), s.cuda_stream))
        return out

    def host_outputs(self) -> MoEOutput:
        """Pinned host tensors for the outputs of forward_host / forward_host_pipelined."""
        return MoEOutput(
            h=torch.empty(self.T, self.d, dtype=self.torch_dtype, pin_memory=True),
            topk_idx=torch.empty(self.T, self.top_k, dtype=torch.int32, pin_memory=True),
            topk_w=torch.empty(self.T, self.top_k, dtype=torch.float32, pin_memory=True),
            expert_counts=torch.empty(self.n_routed, dtype=torch.int32, pin_memory=True),
            aux_loss=torch.empty(1, dtype=torch.float32, pin_memory=True))

    def forward_host_pipelined(self, u: torch.Tensor, out: MoEOutput,
                               stream: torch.cuda.Stream | None = None) -> MoEOutput:
        """Enqueue a forward on pinned HOST tensors without waiting (two calls in flight,
        copies overlapped with the neighbouring forwards).  `u` must stay unchanged and
        `out` unread until pipeline_wait() and a synchronisation of `stream`."""
        if (u.is_cuda or u.shape != (self.T, self.d) or u.dtype != self.torch_dtype
                or not u.is_contiguous()):
            raise ValueError("u must be a contiguous host tensor of the layer shape and dtype")
        self._check_host_outputs(out)
        if not (u.is_pinned() and out.h.is_pinned()):
            raise ValueError("forward_host_pipelined needs pinned host tensors")
        s = stream or torch.cuda.current_stream(self.device)
        check(lib().moe_forward_host_pipelined(self._h, _ptr(u), _ptr(out.h), _ptr(out.topk_idx),
                                               _ptr(out.topk_w), _ptr(out.expert_counts),
                                               _ptr(out.aux_loss), s.cuda_stream))
        return out

    def pipeline_wait(self, stream: torch.cuda.Stream | None = None) -> None:
        """Make `stream` wait for every forward_host_pipelined call issued so far."""
        s = stream or torch.cuda.current_stream(self.device)
        check(lib().moe_pipeline_wait(self._h, s.cuda_stream))

    def backward_prepare(self) -> None:
        """Allocate the backward's workspace and transposed weights (once; later forwards also
        keep their logits).  bf16 layers on the paired-GEMM path only."""
        with torch.cuda.device(self.device):
            check(lib().moe_backward_prepare(self._h))

    def backward(self, u: torch.Tensor, out: MoEOutput, dh: torch.Tensor, d_aux: float = 0.0,
                 weights: bool = True, stream: torch.cuda.Stream | None = None):
        """Gradients of sum(dh * h) + d_aux * aux after `forward(u, out)` on this layer (no
        other forward in between): (du [T, d] bf16, d_centroids [n_routed, d] fp32,
        d_bias [n_routed] fp32, d_w_gate, d_w_up [G, inter, d] fp32, d_w_down [G, d, inter]
        fp32), G = n_shared + n_routed; the last three are None with weights=False."""
        self._check_device_tensor("u", u, (self.T, self.d), self.torch_dtype)
        self._check_device_tensor("dh", dh, (self.T, self.d), self.torch_dtype)
        self._check_outputs(out)
        dev = self.device
        du = torch.empty(self.T, self.d, dtype=self.torch_dtype, device=dev)
        d_cen = torch.empty(self.n_routed, self.d, dtype=torch.float32, device=dev)
        d_bias = torch.empty(self.n_routed, dtype=torch.float32, device=dev)
        G = self.n_shared + self.n_routed
        dwg = dwu = dwd = None
        if weights:
            dwg = torch.empty(G, self.inter, self.d, dtype=torch.float32, device=dev)
            dwu = torch.empty(G, self.inter, self.d, dtype=torch.float32, device=dev)
            dwd = torch.empty(G, self.d, self.inter, dtype=torch.float32, device=dev)
        s = stream or torch.cuda.current_stream(dev)
        check(lib().moe_backward(self._h, _ptr(u), _ptr(out.topk_idx), _ptr(out.topk_w),
                                 _ptr(out.expert_counts), _ptr(dh), float(d_aux), _ptr(du),
                                 _ptr(d_cen), _ptr(d_bias), _ptr(dwg), _ptr(dwu), _ptr(dwd),
                                 s.cuda_stream))
        return du, d_cen, d_bias, dwg, dwu, dwd

    DEBUG_BUFFERS = {"slot_row": 0, "xp": 1, "hr": 2, "yr": 3, "hs": 4, "ys": 5, "grp_row": 6,
                     "row_tok": 7}

    def debug_buffer(self, name: str) -> torch.Tensor:
        """A copy (flat, device) of a workspace buffer as the last forward left it: for
        per-kernel tests.  int32 for slot_row/grp_row/row_tok, uint8 bytes for xp of e4m3
        gate/up layers, else the layer dtype.  row_tok is empty except on decode-sized
        layers."""
        which = self.DEBUG_BUFFERS[name]
        size = ctypes.c_size_t(0)
        s = torch.cuda.current_stream(self.device)
        check(lib().moe_debug_copy(self._h, which, None, 0, ctypes.byref(size), s.cuda_stream))
        if name in ("slot_row", "grp_row", "row_tok"):
            dt = torch.int32
        elif name == "xp" and self.gate_up_e4m3:
            dt = torch.uint8
        else:
            dt = self.torch_dtype
        esz = torch.empty(0, dtype=dt).element_size()
        out = torch.empty(size.value // esz, dtype=dt, device=self.device)
        check(lib().moe_debug_copy(self._h, which, _ptr(out), size.value, ctypes.byref(size),
                                   s.cuda_stream))
        return out

    def device_status(self, stream: torch.cuda.Stream | None = None) -> None:
        """Synchronise and raise if a kernel recorded a device-side error."""
        s = stream or torch.cuda.current_stream(self.device)
        check(lib().moe_device_status(self._h, s.cuda_stream))

    def expert_psum(self, out: torch.Tensor | None = None) -> torch.Tensor:
        out = out if out is not None else torch.empty(self.n_routed, dtype=torch.float32,
                                                      device=self.device)
        check(lib().moe_expert_psum(self._h, _ptr(out), torch.cuda.current_stream(self.device).cuda_stream))
        return out

    KERNEL_NAMES = ("router", "scan", "permute", "gate_up_gemm", "down_gemm", "combine")

    def timing_begin(self, max_forwards: int) -> None:
        """Record per-kernel CUDA events in the next `max_forwards` forward calls."""
        check(lib().moe_timing_begin(self._h, int(max_forwards)))

    def timing_end(self) -> tuple[dict, int]:
        """Synchronise; return ({kernel: summed ms}, number of recorded forward calls)."""
        ms = (ctypes.c_double * 6)()
        n = ctypes.c_int32()
        check(lib().moe_timing_end(self._h, ms, ctypes.byref(n)))
        return dict(zip(self.KERNEL_NAMES, list(ms))), int(n.value)

    @property
    def kernels_per_forward(self) -> int:
        return int(lib().moe_kernels_per_forward(self._h))

    @property
    def device_bytes(self) -> int:
        return int(lib().moe_device_bytes(self._h))

    def close(self) -> None:
        if getattr(self, "_h", None):
            lib().moe_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def balance_loss(counts: torch.Tensor, psum: torch.Tensor, n_tokens: int, alpha1: float,
                 out: torch.Tensor | None = None) -> torch.Tensor:
    """aux = alpha1 * sum_i (counts_i / n_tokens) * (psum_i / n_tokens), on the device."""
    out = out if out is not None else torch.empty(1, dtype=torch.float32, device=counts.device)
    check(lib().moe_balance_loss(_ptr(counts), _ptr(psum), counts.numel(), int(n_tokens),
                                 float(alpha1), _ptr(out),
                                 torch.cuda.current_stream(counts.device).cuda_stream))
    return out
