"""Global-batch statistics across data-parallel ranks (gloo, world size 2, CPU).

Each rank holds half of one batch. The exchange plan of `load_balanced_dispatch_b200.dp` sums
every rank's [2, n] totals (routed copies, probability sums) and the token counts over the
ranks. Normalised by the tokens of all ranks, the sums must give the oracle's whole-batch row
computed on the concatenated batch: f and the Loss-Free update exactly, P and the loss to
rounding ("Qwen global-batch load balance for MoE LLM training", the three steps: synchronise
f, compute, aggregate)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

M, N, K = 1536, 24, 3


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _batch():
    import workloads as W
    rng = np.random.default_rng(17)
    p = rng.random((M, N)).astype(np.float32)
    p /= p.sum(1, keepdims=True)
    idx = W.make_topk_idx(M, N, K, seed=5, skew=1.5)
    b = rng.uniform(-0.05, 0.05, N).astype(np.float32)
    return p, idx, b


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from load_balanced_dispatch_b200 import dp
    p, idx, _ = _batch()
    lo, hi = rank * M // world, (rank + 1) * M // world
    # this rank's totals, from their definitions: routed copies per expert, probability sums
    totals = torch.tensor(np.stack([np.bincount(idx[lo:hi].ravel(), minlength=N).astype(np.float64),
                                    p[lo:hi].astype(np.float64).sum(0)]))
    dp.sum_over_ranks(totals)
    m_total = dp.tokens_over_ranks(hi - lo)
    out[rank] = (totals.numpy().copy(), m_total)
    dist.barrier()
    dist.destroy_process_group()


def test_rank_totals_sum_to_the_global_batch():
    import oracle
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    t0, m0 = out[0]
    t1, m1 = out[1]
    assert m0 == m1 == M
    assert (t0 == t1).all()  # every rank holds the same sums
    p, idx, b = _batch()
    ref = oracle.balance_stats(p, idx, M, N, K, M, 1e-2, bias=b, gamma=1e-3)
    f = t0[0] / (K * m0)
    P = t0[1] / m0
    assert (f == ref["f"][-1]).all()
    assert np.allclose(P, ref["P"][-1], rtol=1e-12, atol=0)
    assert 1e-2 * N * (f * P).sum() == pytest.approx(ref["aux"][-2], rel=1e-12)  # the global-batch loss
    # the Loss-Free update from the pooled counts, decided on integers
    c = t0[0].astype(np.int64)
    step = np.where(c * N > M * K, -1, np.where(c * N < M * K, 1, 0))
    upd = np.where(step < 0, b - np.float32(1e-3), np.where(step > 0, b + np.float32(1e-3), b)).astype(np.float32)
    assert (upd == ref["bias"]).all()


def test_sum_over_ranks_without_a_process_group_is_identity():
    from load_balanced_dispatch_b200 import dp
    t = torch.arange(6, dtype=torch.float64).reshape(2, 3)
    assert (dp.sum_over_ranks(t.clone()) == t).all()
    assert dp.tokens_over_ranks(123) == 123
