"""Expert parallelism, the exchange plan on gloo ranks (world size 2, CPU).

Each rank routes its own half of one batch and assigns capacity slots over its own tokens (the
oracle stands in for the rank's kernels). `ep.gather_offsets` then gathers every rank's
expert_offsets in rank order, the one collective of the plan. The gathered rows must describe
the oracle's layout of the whole batch with one capacity segment per rank: for every expert the
kept rows of all ranks add up to the whole batch's rows of that expert, and rank 0's rows come
first ("Switch Transformer read for implementation", Expert Parallelism: the dispatch
permutation becomes an exchange between devices, capacity decided where the tokens are)."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

M, N, K, CAP = 768, 16, 2, 90


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _routing():
    import workloads as W
    return W.make_topk_idx(M, N, K, seed=21, skew=1.3)


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import oracle
    from load_balanced_dispatch_b200 import ep
    idx = _routing()
    lo, hi = rank * M // world, (rank + 1) * M // world
    cap = oracle.capacity(idx[lo:hi], hi - lo, K, N, CAP, hi - lo)
    gathered = ep.gather_offsets(torch.from_numpy(cap["expert_offsets"].copy()))
    out[rank] = (gathered.numpy().copy(), cap["expert_offsets"].copy(), cap["dest_row"].copy())
    dist.barrier()
    dist.destroy_process_group()


def test_gathered_offsets_describe_the_whole_batch_layout():
    import oracle
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    g0, off0, dest0 = out[0]
    g1, off1, dest1 = out[1]
    assert (g0 == g1).all()                      # every rank holds the same plan
    assert (g0[0] == off0).all() and (g0[1] == off1).all()  # in rank order
    whole = oracle.capacity(_routing(), M, K, N, CAP, M // world)
    woff = whole["expert_offsets"]
    kept = np.diff(g0, axis=1)                   # [ranks, n] kept rows per expert
    assert (kept.sum(0) == np.diff(woff)).all()
    # a row of rank r for expert e sits in the whole layout at: the expert's start, then the
    # rows of the ranks before r, then its place among its own rank's rows of e
    idx = _routing()
    for r, (dest, off) in enumerate(((dest0, off0), (dest1, off1))):
        lo = r * M // world
        for i in range(dest.shape[0]):
            for t in range(K):
                if dest[i, t] < 0:
                    assert whole["dest_row"][lo + i, t] < 0
                    continue
                e = idx[lo + i, t]
                row = woff[e] + kept[:r, e].sum() + dest[i, t] - off[e]
                assert whole["dest_row"][lo + i, t] == row
