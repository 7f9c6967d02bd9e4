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


def global_token_count(n_tokens: int, device, group=None) -> int:
    """The sum of every rank's `n_tokens` (one all-reduce and a host read: call it once,
    not per step, when the per-rank token counts do not change)."""
    t = torch.tensor([int(n_tokens)], dtype=torch.int64, device=device)
    dist.all_reduce(t, group=group)
    return int(t.item())


def all_reduce_balance_stats(counts: torch.Tensor, psum: torch.Tensor, n_tokens: int,
                             group=None, n_global: int | None = None) -> int:
    """Sum `counts` [N_r] and `psum` [N_r] over the ranks of `group`, in place.

    Returns the global token count: `n_global` when the caller already knows it (then no
    host synchronisation happens here), else the sum of every rank's `n_tokens`.  Every
    rank must call this in the same order and with the same choice of `n_global`.
    """
    dist.all_reduce(counts, group=group)
    dist.all_reduce(psum, group=group)
    if n_global is not None:
        return int(n_global)
    return global_token_count(n_tokens, counts.device, group)


def global_balance_loss(layer, out, psum_buf: torch.Tensor, counts_buf: torch.Tensor,
                        aux_buf: torch.Tensor, group=None, n_global: int | None = None,
                        loss_fn=None) -> torch.Tensor:
    """After `layer.forward(u, out)`: the balance loss of the global batch into `aux_buf`
    (`n_global`: the global token count, if known -- see global_token_count).

    `loss_fn(counts, psum, n_tokens, alpha1, out)` computes the loss from the all-reduced
    statistics; the default is the library's kernel (`layer.balance_loss`).  `layer` needs
    `expert_psum(buf)`, `T` and `alpha1`; `out` needs `expert_counts`."""
    if loss_fn is None:
        from .layer import balance_loss as loss_fn
    layer.expert_psum(psum_buf)
    counts_buf.copy_(out.expert_counts)
    n_global = all_reduce_balance_stats(counts_buf, psum_buf, layer.T, group, n_global)
    return loss_fn(counts_buf, psum_buf, n_global, layer.alpha1, aux_buf)
