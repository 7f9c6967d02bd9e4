"""Token-sharded data parallelism on CPU (gloo, world size 2).

Each rank routes its own shard of the tokens; the balance statistics are all-reduced with
the same helper the GPU path uses (`parallel.all_reduce_balance_stats`), and the global
loss and counts must equal those of the unsharded batch.  Uneven shards are included.
`parallel.global_balance_loss` -- the call the benchmark makes after every forward on
N > 1 GPUs -- is also run end to end, with the loss formula restated on the CPU in place
of the library's kernel.
"""
import types
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from mixture_experts_layer_65_b200 import parallel
from mixture_experts_layer_65_b200 import workloads as W
from oracle import moe_oracle as O


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, bounds, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = W.make_workload("tiny")
        lo, hi = bounds[rank], bounds[rank + 1]
        r = O.route(w.u[lo:hi], w.centroids, w.top_k)
        counts = torch.from_numpy(np.bincount(r.topk_idx.reshape(-1), minlength=w.n_routed))
        psum = torch.from_numpy(r.s.sum(axis=0))
        n = parallel.all_reduce_balance_stats(counts, psum, hi - lo)
        aux = w.alpha1 * float(torch.sum((counts / n) * (psum / n)))
        # the same with the global token count computed once up front (no per-step read)
        n_once = parallel.global_token_count(hi - lo, "cpu")
        c2 = torch.from_numpy(np.bincount(r.topk_idx.reshape(-1), minlength=w.n_routed))
        p2 = torch.from_numpy(r.s.sum(axis=0))
        n2 = parallel.all_reduce_balance_stats(c2, p2, hi - lo, n_global=n_once)
        assert n2 == n and torch.equal(c2, counts) and torch.equal(p2, psum)
        # the benchmark's per-step call, end to end: the layer's psum and counts buffers,
        # the all-reduce, then the loss from the global statistics
        layer = types.SimpleNamespace(T=hi - lo, alpha1=w.alpha1,
                                      expert_psum=lambda buf: buf.copy_(torch.from_numpy(r.s.sum(axis=0))))
        out = types.SimpleNamespace(expert_counts=torch.from_numpy(
            np.bincount(r.topk_idx.reshape(-1), minlength=w.n_routed)))

        def cpu_loss(c, p, n_tok, a1, o):
            o.fill_(a1 * float(torch.sum((c / n_tok) * (p / n_tok))))
            return o

        aux_g = parallel.global_balance_loss(
            layer, out, torch.empty(w.n_routed, dtype=torch.float64),
            torch.empty(w.n_routed, dtype=torch.int64), torch.empty(1, dtype=torch.float64),
            loss_fn=cpu_loss)
        aux_g2 = parallel.global_balance_loss(
            layer, out, torch.empty(w.n_routed, dtype=torch.float64),
            torch.empty(w.n_routed, dtype=torch.int64), torch.empty(1, dtype=torch.float64),
            n_global=n_once, loss_fn=cpu_loss)
        assert float(aux_g) == float(aux_g2)
        q.put((rank, n, counts.numpy(), psum.numpy(), aux, r.topk_idx, float(aux_g)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("bounds", [(0, 64, 128), (0, 75, 128)], ids=["even", "uneven"])
def test_sharded_balance_statistics_match_the_full_batch(bounds):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, bounds, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        rank, n, counts, psum, aux, idx, aux_g = q.get(timeout=120)
        res[rank] = (n, counts, psum, aux, idx, aux_g)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w = W.make_workload("tiny")
    full = O.moe_forward(w.u, w.centroids, w.w_gate, w.w_up, w.w_down, w.n_shared, w.top_k,
                         w.alpha1, rows=[0])
    for rank in (0, 1):
        n, counts, psum, aux, _, aux_g = res[rank]
        assert n == w.T
        np.testing.assert_array_equal(counts, full.counts)
        np.testing.assert_allclose(psum / n, full.P, rtol=1e-13)
        assert aux == pytest.approx(full.aux, rel=1e-12)
        assert aux_g == pytest.approx(full.aux, rel=1e-12)
    # routing is per token: the shards' indices are the full batch's rows
    np.testing.assert_array_equal(np.concatenate([res[0][4], res[1][4]]), full.routing.topk_idx)
