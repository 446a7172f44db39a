"""Data-parallel replicas of the layer: the one exchange the pages define between them.

Each rank runs the whole layer forward on its own tokens with its own copy of the experts
(nothing crosses ranks on the data path). The global-batch statistics of "Qwen global-batch
load balance for MoE LLM training" (agentlenshq.com) pool the routed counts, and with them f_i,
P_i, the loss and the Loss-Free update, over every rank's tokens. That takes one all-reduce of
a [2, n] fp64 buffer per forward, between `moe_balance_totals` and `moe_balance_global`. Summing
the rank totals and dividing by the tokens of all ranks gives the same numbers as one rank
holding the whole global batch: counts are exact integers in fp64, and the probability sums
differ only by the order of the fp64 additions.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def sum_over_ranks(t: torch.Tensor, group=None) -> torch.Tensor:
    """Element-wise sum of `t` over the ranks of `group`, in place (identity without a process group)."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
    return t


def tokens_over_ranks(m_local: int, group=None, device="cpu") -> int:
    """Tokens of the global batch: the sum of every rank's m."""
    t = torch.tensor([m_local], dtype=torch.int64, device=device)
    return int(sum_over_ranks(t, group).item())


def global_batch_stats(probs, topk_idx, n, m_total, alpha=1e-2, bias_inout=None, gamma=1e-3, group=None,
                       totals=None, workspace=None, out=None, stream=None):
    """f, P, aux and violations of the global batch over every rank (and the shared Loss-Free update).

    Every rank calls this with its own probs / topk_idx; all ranks get the same results."""
    from . import moe_balance_global, moe_balance_totals

    totals = moe_balance_totals(probs, topk_idx, n, totals=totals, workspace=workspace, stream=stream)
    if stream is not None:
        with torch.cuda.stream(stream):
            sum_over_ranks(totals, group)
    else:
        sum_over_ranks(totals, group)
    return moe_balance_global(totals, m_total, topk_idx.shape[1], has_probs=probs is not None, alpha=alpha,
                              bias_inout=bias_inout, gamma=gamma, out=out, stream=stream)
