"""Data-parallel (token-sharded) use of the layer: the global expert-level balance loss.

Each rank runs the layer on its own tokens with replicated weights; routing and the
expert FFNs are per token, so nothing crosses ranks except the balance statistics.  The
expert-level balance loss of the DeepSeekMoE article ("Expert-level balance loss",
L_ExpBal = alpha_1 * sum_i f_i P_i) is defined over the whole batch, so its per-expert
counts and affinity sums are summed over the ranks (one all-reduce each) before
f_i = count_i / T_global and P_i = psum_i / T_global are formed.  torch.distributed
(NCCL on GPUs, gloo on CPUs) carries the all-reduce; the loss itself is one kernel of the
library (`balance_loss`).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def all_reduce_balance_stats(counts: torch.Tensor, psum: torch.Tensor, n_tokens: int,
                             group=None) -> int:
    """Sum `counts` [N_r] and `psum` [N_r] over the ranks of `group`, in place.

    Returns the global token count (the sum of every rank's `n_tokens`).  Every rank must
    call this in the same order (it issues three all-reduces).
    """
    dist.all_reduce(counts, group=group)
    dist.all_reduce(psum, group=group)
    t = torch.tensor([int(n_tokens)], dtype=torch.int64, device=counts.device)
    dist.all_reduce(t, group=group)
    return int(t.item())


def global_balance_loss(layer, out, psum_buf: torch.Tensor, counts_buf: torch.Tensor,
                        aux_buf: torch.Tensor, group=None) -> torch.Tensor:
    """After `layer.forward(u, out)`: the balance loss of the global batch into `aux_buf`."""
    from .layer import balance_loss
    layer.expert_psum(psum_buf)
    counts_buf.copy_(out.expert_counts)
    n_global = all_reduce_balance_stats(counts_buf, psum_buf, layer.T, group)
    return balance_loss(counts_buf, psum_buf, n_global, layer.alpha1, aux_buf)
