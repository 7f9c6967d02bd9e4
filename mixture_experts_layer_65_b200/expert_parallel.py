"""Expert-parallel DeepSeekMoE layer: the routed experts are split over the ranks, the
tokens stay data-parallel (every rank routes its own T tokens).

DeepSeekMoE (deepforge.srivtx.xyz article), "Where this sits": a layer's experts are spread
over devices, and a device-level balance loss keeps their computation even.  Rank r holds
the shared experts and the routed experts [r * n_local, (r + 1) * n_local).  One forward:

  1. dispatch (library): route the rank's tokens; the row of every (token, slot), ordered
     by expert -- so the rows for rank q are one contiguous block;
  2. all-to-all of the per-expert counts, one host read of the counts (the row exchange
     needs its split sizes on the host), all-to-all of the rows;
  3. experts (library): every received row through its expert's SwiGLU FFN;
  4. the reverse all-to-all;
  5. combine (library): the shared experts on the rank's tokens plus the gated rows;
  6. the balance statistics all-reduced over the ranks for the global expert counts and
     loss.

torch.distributed carries the collectives (NCCL on GPUs: `DistComm`); the arithmetic is the
library's kernels (`LibEPBackend`).  `ep_forward` only moves tensors between them, so it runs
with any backend object that has the same methods (the CPU tests use one built on the
oracle) and any communicator with all_to_all_single / all_reduce.
"""
from __future__ import annotations

import ctypes

import torch
import torch.distributed as dist

from . import _lib
from ._lib import MoeCfg, check, lib
from .layer import MoEOutput, _ptr


def expert_range(n_routed: int, world: int, rank: int) -> tuple[int, int]:
    """The routed experts [e0, e0 + n_local) rank `rank` holds."""
    if n_routed % world:
        raise ValueError(f"n_routed={n_routed} is not a multiple of world={world}")
    n_local = n_routed // world
    return rank * n_local, n_local


class DistComm:
    """The two collectives of the expert-parallel forward, over a torch.distributed group
    (NCCL for CUDA tensors, gloo for CPU tensors)."""

    def __init__(self, group=None):
        self.group = group

    def all_to_all_single(self, out, inp, out_splits=None, in_splits=None):
        dist.all_to_all_single(out, inp, out_splits, in_splits, group=self.group)

    def all_reduce(self, t):
        dist.all_reduce(t, group=self.group)


def ep_forward(backend, u: torch.Tensor, comm=None) -> MoEOutput:
    """One expert-parallel forward on this rank (every rank calls it together).

    backend: dispatch(u) -> (topk_idx, topk_w, counts, aux, send_rows);
             experts(recv_rows, recv_counts, n_recv) -> out_rows;
             combine(u, back_rows, topk_w) -> h;  psum() -> per-expert affinity sums;
             alloc_rows(n) -> an [n, d] buffer for received rows;
             attributes T, n_routed, n_local, alpha1, world.
    comm: all_to_all_single / all_reduce (default: DistComm over the default group).
    Returns h, topk_idx, topk_w of this rank's tokens and the global expert counts and
    balance loss."""
    comm = comm or DistComm()
    world, nl, nr = backend.world, backend.n_local, backend.n_routed
    idx, gates, counts, _, send_rows = backend.dispatch(u)
    # per-expert counts: rank q gets the counts of its n_local experts from every rank
    recv_counts = torch.empty_like(counts)
    comm.all_to_all_single(recv_counts, counts)
    # the row exchange's split sizes, on the host (one read of 2 * n_routed integers)
    both = torch.cat([counts, recv_counts]).cpu()
    send_splits = [int(x) for x in both[:nr].view(world, nl).sum(dim=1)]
    recv_splits = [int(x) for x in both[nr:].view(world, nl).sum(dim=1)]
    n_recv = sum(recv_splits)
    recv_rows = backend.alloc_rows(n_recv)
    comm.all_to_all_single(recv_rows, send_rows, recv_splits, send_splits)
    out_rows = backend.experts(recv_rows, recv_counts, n_recv)
    back_rows = torch.empty_like(send_rows)
    comm.all_to_all_single(back_rows, out_rows, send_splits, recv_splits)
    h = backend.combine(u, back_rows, gates)
    # balance statistics of the global batch: counts, affinity sums and token counts summed
    # over the ranks, then alpha_1 * sum_i (count_i / T) (psum_i / T)
    psum = backend.psum()
    cnt = counts.clone()
    n_tok = torch.tensor([backend.T], dtype=torch.int64, device=cnt.device)
    comm.all_reduce(cnt)
    comm.all_reduce(psum)
    comm.all_reduce(n_tok)
    n_global = float(n_tok.item())
    aux = backend.alpha1 * torch.sum((cnt.double() / n_global) * (psum.double() / n_global))
    return MoEOutput(h=h, topk_idx=idx, topk_w=gates, expert_counts=cnt,
                     aux_loss=aux.to(torch.float32).reshape(1))


class LibEPBackend:
    """This rank's part of an expert-parallel layer in libmoe.so (moe_ep_* in include/moe.h).

    Weights w_gate/w_up [n_shared + n_local, inter, d], w_down [n_shared + n_local, d, inter]
    (the shared experts, then this rank's routed experts); centroids [n_routed, d] and the
    optional logit_bias [n_routed] cover all routed experts.  bf16 layers only."""

    def __init__(self, *, T: int, d: int, n_routed: int, n_shared: int, top_k: int, inter: int,
                 alpha1: float, centroids: torch.Tensor, w_gate: torch.Tensor,
                 w_up: torch.Tensor, w_down: torch.Tensor, rank: int, world: int,
                 logit_bias: torch.Tensor | None = None, recv_capacity: int = 0):
        self.T, self.d, self.n_routed, self.n_shared = T, d, n_routed, n_shared
        self.top_k, self.inter, self.alpha1 = top_k, inter, alpha1
        self.rank, self.world = rank, world
        self.e0, self.n_local = expert_range(n_routed, world, rank)
        self.device = centroids.device
        n_exp = n_shared + self.n_local
        for name, t, shape in (("centroids", centroids, (n_routed, d)),
                               ("w_gate", w_gate, (n_exp, inter, d)),
                               ("w_up", w_up, (n_exp, inter, d)),
                               ("w_down", w_down, (n_exp, d, inter))):
            if (not t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous()
                    or tuple(t.shape) != shape):
                raise ValueError(f"{name} must be a contiguous CUDA bf16 {list(shape)} tensor")
        cfg = MoeCfg(T=T, d=d, n_routed=n_routed, n_shared=n_shared, top_k=top_k, inter=inter,
                     dtype=_lib.MOE_BF16, alpha1=alpha1, centroids=_ptr(centroids),
                     logit_bias=_ptr(logit_bias), w_gate=_ptr(w_gate), w_up=_ptr(w_up),
                     w_down=_ptr(w_down))
        handle = ctypes.c_void_p()
        with torch.cuda.device(self.device):
            check(lib().moe_ep_create(ctypes.byref(cfg), rank, world, int(recv_capacity),
                                      ctypes.byref(handle)))
        self._h = handle
        self.recv_capacity = int(lib().moe_ep_recv_capacity(handle))
        dev = self.device
        self._recv = torch.empty(self.recv_capacity, d, dtype=torch.bfloat16, device=dev)
        self._out = torch.empty(self.recv_capacity, d, dtype=torch.bfloat16, device=dev)

    def _stream(self):
        return torch.cuda.current_stream(self.device).cuda_stream

    def alloc_rows(self, n: int) -> torch.Tensor:
        if n > self.recv_capacity:
            raise ValueError(f"{n} received rows exceed the capacity {self.recv_capacity}")
        return self._recv[:n]

    def dispatch(self, u: torch.Tensor):
        T, K, dev = self.T, self.top_k, self.device
        if tuple(u.shape) != (T, self.d) or u.dtype != torch.bfloat16 or not u.is_contiguous():
            raise ValueError("u must be a contiguous [T, d] bf16 tensor")
        idx = torch.empty(T, K, dtype=torch.int32, device=dev)
        gates = torch.empty(T, K, dtype=torch.float32, device=dev)
        counts = torch.empty(self.n_routed, dtype=torch.int32, device=dev)
        aux = torch.empty(1, dtype=torch.float32, device=dev)
        send = torch.empty(T * K, self.d, dtype=torch.bfloat16, device=dev)
        check(lib().moe_ep_dispatch(self._h, _ptr(u), _ptr(idx), _ptr(gates), _ptr(counts),
                                    _ptr(aux), _ptr(send), self._stream()))
        return idx, gates, counts, aux, send

    def experts(self, recv_rows: torch.Tensor, recv_counts: torch.Tensor, n_recv: int) -> torch.Tensor:
        out = self._out[:n_recv]
        check(lib().moe_ep_experts(self._h, _ptr(recv_rows), _ptr(recv_counts), int(n_recv),
                                   _ptr(out), self._stream()))
        return out

    def combine(self, u: torch.Tensor, back_rows: torch.Tensor, gates: torch.Tensor) -> torch.Tensor:
        h = torch.empty(self.T, self.d, dtype=torch.bfloat16, device=self.device)
        check(lib().moe_ep_combine(self._h, _ptr(u), _ptr(back_rows), _ptr(gates), _ptr(h),
                                   self._stream()))
        return h

    def psum(self) -> torch.Tensor:
        out = torch.empty(self.n_routed, dtype=torch.float32, device=self.device)
        check(lib().moe_ep_expert_psum(self._h, _ptr(out), self._stream()))
        return out

    def device_status(self) -> None:
        check(lib().moe_ep_device_status(self._h, self._stream()))

    def close(self) -> None:
        if getattr(self, "_h", None):
            lib().moe_ep_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def lib_backend_from_workload(w, rank: int, world: int, device="cuda",
                              recv_capacity: int = 0) -> LibEPBackend:
    """This rank's backend for a seeded workload (its slice of the routed experts)."""
    from .layer import to_device_tensor
    e0, nl = expert_range(w.n_routed, world, rank)
    keep = list(range(w.n_shared)) + list(range(w.n_shared + e0, w.n_shared + e0 + nl))
    dev = torch.device(device)
    bias = None if w.logit_bias is None else torch.from_numpy(w.logit_bias).to(dev)
    return LibEPBackend(T=w.T, d=w.d, n_routed=w.n_routed, n_shared=w.n_shared, top_k=w.top_k,
                        inter=w.inter, alpha1=w.alpha1,
                        centroids=to_device_tensor(w.centroids, dev),
                        w_gate=to_device_tensor(w.w_gate[keep], dev),
                        w_up=to_device_tensor(w.w_up[keep], dev),
                        w_down=to_device_tensor(w.w_down[keep], dev),
                        rank=rank, world=world, logit_bias=bias, recv_capacity=recv_capacity)
