"""Expert-parallel forward: routed experts split over ranks, tokens data-parallel.

CPU (gloo, world size 2): the orchestration of mixture_experts_layer_65_b200.expert_parallel
-- the count exchange, the split sizes, both row all-to-alls and the global balance
statistics -- with an oracle-based rank backend, against the oracle's full-batch layer, on
even, uneven and Zipf-skewed loads.  GPU: the library's ranks (moe_ep_*) with 1 rank over
NCCL and with 2 and 4 ranks emulated as host threads on one GPU, bit for bit against
moe_forward on the full batch and against the oracle.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from mixture_experts_layer_65_b200 import workloads as W
from mixture_experts_layer_65_b200.expert_parallel import DistComm, ep_forward, expert_range
from oracle import moe_oracle as O
from tests import parity as P
from tests.ep_helpers import OracleEPBackend, ThreadComm, run_threads

SMALL = dict(d=64, n_shared=1, n_routed=8, inter=32, top_k=3, alpha1=0.01)
LOADS = {
    "even": (dict(T=96, **SMALL), (0, 48, 96)),
    "uneven": (dict(T=96, **SMALL), (0, 71, 96)),
    # Zipf(1.1) logit bias: expert 0 takes most tokens, so rank 0 receives most rows
    "zipf": (dict(T=96, zipf_s=1.1, **dict(SMALL, top_k=2)), (0, 40, 96)),
}


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gloo_worker(rank, world, port, spec, bounds, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = W.make_workload("16b_prefill", **spec)
        be = OracleEPBackend(w, bounds[rank], bounds[rank + 1], rank, world)
        out = ep_forward(be, None, DistComm())
        q.put((rank, out.h.numpy(), out.topk_idx.numpy(), out.expert_counts.numpy(),
               float(out.aux_loss[0])))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("load", list(LOADS))
def test_gloo_two_ranks_match_the_full_batch(load):
    spec, bounds = LOADS[load]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gloo_worker, args=(r, 2, port, spec, bounds, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        r, h, idx, cnt, aux = q.get(timeout=180)
        res[r] = (h, idx, cnt, aux)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    w = W.make_workload("16b_prefill", **spec)
    full = O.moe_forward(w.u, w.centroids, w.w_gate, w.w_up, w.w_down, w.n_shared, w.top_k,
                         w.alpha1, bias=w.logit_bias)
    h = np.concatenate([res[0][0], res[1][0]])
    np.testing.assert_allclose(h, full.h, rtol=0, atol=1e-12 * np.abs(full.h).max())
    np.testing.assert_array_equal(np.concatenate([res[0][1], res[1][1]]), full.routing.topk_idx)
    for r in (0, 1):
        np.testing.assert_array_equal(res[r][2], full.counts)
        assert res[r][3] == pytest.approx(full.aux, rel=2.0 ** -23)   # an fp32 output
    if load == "zipf":   # the skew the test is for: one rank receives most of the rows
        e0, nl = expert_range(w.n_routed, 2, 0)
        assert full.counts[e0:e0 + nl].sum() > 3 * full.counts[nl:].sum()


def test_single_rank_with_local_copies_matches_the_full_batch():
    """The benchmark's one-rank expert-parallel run (`bench.py --expert-parallel`): the
    all-to-alls become local copies and the sums over ranks the rank's own values; with the
    oracle-based rank it reproduces the full-batch oracle."""
    import bench
    spec, _ = LOADS["zipf"]
    w = W.make_workload("16b_prefill", **spec)
    out = ep_forward(OracleEPBackend(w, 0, w.T, 0, 1), None, bench._LocalComm())
    full = O.moe_forward(w.u, w.centroids, w.w_gate, w.w_up, w.w_down, w.n_shared, w.top_k,
                         w.alpha1, bias=w.logit_bias)
    np.testing.assert_allclose(out.h.numpy(), full.h, rtol=0, atol=1e-12 * np.abs(full.h).max())
    np.testing.assert_array_equal(out.topk_idx.numpy(), full.routing.topk_idx)
    np.testing.assert_array_equal(out.expert_counts.numpy(), full.counts)
    assert float(out.aux_loss[0]) == pytest.approx(full.aux, rel=2.0 ** -23)


def test_expert_range_splits_evenly():
    assert expert_range(64, 8, 3) == (24, 8)
    with pytest.raises(ValueError):
        expert_range(63, 2, 0)


def test_thread_comm_matches_the_collective_semantics():
    """The in-process communicator the GPU tests use: uneven all-to-all and all-reduce."""
    def fn(rank, comm):
        x = torch.arange(6, dtype=torch.float64) + 10 * rank
        ins = [2, 4] if rank == 0 else [3, 3]
        outs = [2, 3] if rank == 0 else [4, 3]
        out = torch.empty(sum(outs), dtype=torch.float64)
        comm.all_to_all_single(out, x, outs, ins)
        t = torch.tensor([rank + 1.0])
        comm.all_reduce(t)
        return out.tolist(), float(t)
    r0, r1 = run_threads(2, fn)
    assert r0 == ([0.0, 1.0, 10.0, 11.0, 12.0], 3.0)
    assert r1 == ([2.0, 3.0, 4.0, 5.0, 13.0, 14.0, 15.0], 3.0)


# ------------------------------------------------------------------------------ GPU
def _gpu_full(w):
    from mixture_experts_layer_65_b200.layer import MoELayer, to_device_tensor
    layer = MoELayer.from_workload(w, "cuda")
    out = layer.forward(to_device_tensor(w.u, "cuda"))
    torch.cuda.synchronize()
    layer.device_status()
    layer.close()
    return out


def _run_ep(w, bounds, comm_for_rank):
    """Every rank of `bounds` as a host thread; returns the ranks' outputs (device)."""
    from mixture_experts_layer_65_b200.expert_parallel import LibEPBackend
    from mixture_experts_layer_65_b200.layer import to_device_tensor
    world = len(bounds) - 1

    def fn(rank, tcomm):
        lo, hi = bounds[rank], bounds[rank + 1]
        e0, nl = expert_range(w.n_routed, world, rank)
        keep = list(range(w.n_shared)) + list(range(w.n_shared + e0, w.n_shared + e0 + nl))
        dev = torch.device("cuda")
        bias = None if w.logit_bias is None else torch.from_numpy(w.logit_bias).to(dev)
        be = LibEPBackend(T=hi - lo, d=w.d, n_routed=w.n_routed, n_shared=w.n_shared,
                          top_k=w.top_k, inter=w.inter, alpha1=w.alpha1,
                          centroids=to_device_tensor(w.centroids, dev),
                          w_gate=to_device_tensor(w.w_gate[keep], dev),
                          w_up=to_device_tensor(w.w_up[keep], dev),
                          w_down=to_device_tensor(w.w_down[keep], dev),
                          rank=rank, world=world, logit_bias=bias,
                          recv_capacity=w.T * w.top_k)   # the ranks' token counts differ
        u = to_device_tensor(w.u[lo:hi], dev)
        outs = [ep_forward(be, u, comm_for_rank(rank, tcomm)) for _ in range(2)]
        torch.cuda.synchronize()
        be.device_status()
        be.close()
        return outs
    return run_threads(world, fn) if world > 1 else [fn(0, None)]


def _check(w, bounds, res, full):
    # bit for bit moe_forward's outputs when every rank routes on the same kernel as the
    # full batch (a rank of <= 128 tokens uses the SIMT router, which sums the logits in
    # another order); the oracle comparison below holds either way
    import types
    same = all(P.router_path(types.SimpleNamespace(dtype=w.dtype, T=hi - lo, d=w.d)) ==
               P.router_path(w) for lo, hi in zip(bounds[:-1], bounds[1:]))
    for call in range(2):
        h = torch.cat([r[call].h for r in res])
        idx = torch.cat([r[call].topk_idx for r in res])
        gates = torch.cat([r[call].topk_w for r in res])
        if same:
            assert torch.equal(idx, full.topk_idx), f"call {call}: routed indices differ"
            assert torch.equal(gates, full.topk_w), f"call {call}: gates differ"
            assert torch.equal(h, full.h), f"call {call}: h differs from moe_forward"
            for r in res:
                assert torch.equal(r[call].expert_counts, full.expert_counts)
        for r in res:   # every rank holds the same global counts
            assert torch.equal(r[call].expert_counts, res[0][call].expert_counts)
        g = P.GpuOut(h=h.float().cpu().numpy().astype(np.float64),
                     topk_idx=idx.cpu().numpy().astype(np.int64),
                     topk_w=gates.cpu().numpy().astype(np.float64),
                     counts=res[0][call].expert_counts.cpu().numpy().astype(np.int64),
                     aux=float(res[0][call].aux_loss[0]))
        rows = None if w.T <= 1024 else P.sample_rows(w.T)
        rep = P.compare(w, g, rows=rows)
        print(w.name, bounds, call, rep)


EP_GPU = [
    ("two_ranks", dict(T=600, d=256, n_shared=2, n_routed=16, inter=192, top_k=4), (0, 300, 600)),
    ("four_ranks_uneven", dict(T=700, d=256, n_shared=1, n_routed=16, inter=128, top_k=4),
     (0, 100, 350, 351, 700)),
    ("zipf_two_ranks", dict(T=1000, d=256, n_shared=1, n_routed=16, inter=128, top_k=2, zipf_s=1.1),
     (0, 500, 1000)),
    ("no_shared_two_ranks", dict(T=500, d=256, n_shared=0, n_routed=16, inter=128, top_k=2), (0, 250, 500)),
    ("decode_sized_two_ranks", dict(T=128, d=256, n_shared=2, n_routed=16, inter=192, top_k=4), (0, 64, 128)),
]


@pytest.mark.gpu
@pytest.mark.parametrize("name,spec,bounds", EP_GPU, ids=[c[0] for c in EP_GPU])
def test_ep_ranks_as_threads_match_moe_forward(name, spec, bounds):
    w = W.make_workload("16b_prefill", alpha1=0.001, **spec)
    full = _gpu_full(w)
    res = _run_ep(w, bounds, lambda rank, tcomm: tcomm)
    _check(w, bounds, res, full)


@pytest.mark.gpu
def test_ep_16b_layer_four_ranks():
    """The 16B-shaped layer (64 routed experts, 16 per rank) at 4096 tokens per rank."""
    w = W.make_workload("16b_prefill")
    full = _gpu_full(w)
    bounds = (0, 4096, 8192, 12288, 16384)
    res = _run_ep(w, bounds, lambda rank, tcomm: tcomm)
    _check(w, bounds, res, full)


@pytest.mark.gpu
def test_ep_one_rank_over_nccl():
    """World size 1 through torch.distributed's NCCL backend (the collectives a multi-GPU
    run makes), the 2B-shaped layer."""
    if not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        os.environ["MASTER_PORT"] = str(_free_port())
        dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        w = W.make_workload("2b", T=3000)
        full = _gpu_full(w)
        res = _run_ep(w, (0, w.T), lambda rank, tcomm: DistComm())
        _check(w, (0, w.T), res, full)
    finally:
        dist.destroy_process_group()
