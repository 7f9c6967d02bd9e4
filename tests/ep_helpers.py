"""Test helpers for the expert-parallel layer: an oracle-based rank backend (CPU, fp64) and
an in-process communicator for ranks run as host threads."""
from __future__ import annotations

import threading

import numpy as np
import torch

from mixture_experts_layer_65_b200.expert_parallel import expert_range
from oracle import moe_oracle as O


class OracleEPBackend:
    """One rank of the expert-parallel layer restated with the oracle (fp64 torch tensors):
    the dispatch orders each (token, slot) row by expert, tokens ascending; the experts step
    runs block (source s, local expert e) of the received rows through routed expert
    e0 + e; the combine adds the shared experts and the gated returned rows."""

    def __init__(self, w, lo: int, hi: int, rank: int, world: int):
        self.w, self.lo, self.hi = w, lo, hi
        self.T, self.d, self.n_routed, self.alpha1 = hi - lo, w.d, w.n_routed, w.alpha1
        self.rank, self.world = rank, world
        self.e0, self.n_local = expert_range(w.n_routed, world, rank)
        self.r = None
        self.slot = None

    def alloc_rows(self, n):
        return torch.empty(n, self.d, dtype=torch.float64)

    def dispatch(self, u):
        w = self.w
        self.r = O.route(w.u[self.lo:self.hi], w.centroids, w.top_k, w.logit_bias)
        idx = self.r.topk_idx
        order = []
        for e in range(w.n_routed):
            ts, ks = np.nonzero(idx == e)
            order += list(zip(ts.tolist(), ks.tolist()))   # tokens ascending (row-major scan)
        self.slot = np.zeros_like(idx)
        for j, (t, k) in enumerate(order):
            self.slot[t, k] = j
        u64 = O.widen(w.u[self.lo:self.hi])
        send = torch.from_numpy(np.stack([u64[t] for t, _ in order]) if order else
                                np.zeros((0, self.d)))
        counts = torch.from_numpy(np.bincount(idx.reshape(-1), minlength=w.n_routed).astype(np.int64))
        return (torch.from_numpy(idx), torch.from_numpy(self.r.topk_w), counts, None, send)

    def experts(self, recv_rows, recv_counts, n_recv):
        w, ks = self.w, self.w.n_shared
        cnt = recv_counts.numpy().reshape(self.world, self.n_local)
        out = np.zeros((n_recv, self.d))
        x = recv_rows.numpy()
        j = 0
        for s in range(self.world):
            for e in range(self.n_local):
                n = int(cnt[s, e])
                g = ks + self.e0 + e
                if n:
                    out[j:j + n] = O.swiglu_ffn(x[j:j + n], w.w_gate[g], w.w_up[g], w.w_down[g])
                j += n
        return torch.from_numpy(out)

    def combine(self, u, back_rows, gates):
        w = self.w
        u64 = O.widen(w.u[self.lo:self.hi])
        h = u64.copy()
        for j in range(w.n_shared):
            h += O.swiglu_ffn(u64, w.w_gate[j], w.w_up[j], w.w_down[j])
        b = back_rows.numpy()
        g = gates.numpy()
        for k in range(w.top_k):
            h += g[:, k:k + 1] * b[self.slot[:, k]]
        return torch.from_numpy(h)

    def psum(self):
        return torch.from_numpy(self.r.s.sum(axis=0))


class ThreadComm:
    """all_to_all_single / all_reduce between ranks that are host threads of one process
    (one GPU: the ranks' kernels never wait on one another; the threads meet on a host
    barrier between collectives)."""

    def __init__(self, rank: int, world: int, shared: dict):
        self.rank, self.world, self.S = rank, world, shared

    @staticmethod
    def shared(world: int) -> dict:
        return {"barrier": threading.Barrier(world, timeout=120), "slots": [None] * world}

    def all_to_all_single(self, out, inp, out_splits=None, in_splits=None):
        W, S = self.world, self.S
        in_splits = in_splits or [inp.shape[0] // W] * W
        S["slots"][self.rank] = list(torch.split(inp, in_splits))
        S["barrier"].wait()
        parts = [S["slots"][s][self.rank] for s in range(W)]
        if out.shape[0]:
            torch.cat(parts, out=out)
        S["barrier"].wait()

    def all_reduce(self, t):
        S = self.S
        S["slots"][self.rank] = t.clone()
        S["barrier"].wait()
        acc = S["slots"][0].clone()
        for s in range(1, self.world):
            acc += S["slots"][s]
        S["barrier"].wait()
        t.copy_(acc)


def run_threads(world: int, fn):
    """fn(rank, comm) on `world` threads; returns their results (re-raises a failure)."""
    shared = ThreadComm.shared(world)
    res, errs = [None] * world, []

    def body(r):
        try:
            res[r] = fn(r, ThreadComm(r, world, shared))
        except BaseException as e:   # noqa: BLE001 - surfaced below
            errs.append(e)
            shared["barrier"].abort()

    th = [threading.Thread(target=body, args=(r,)) for r in range(world)]
    for t in th:
        t.start()
    for t in th:
        t.join()
    if errs:
        raise errs[0]
    return res
