"""Expert parallelism: the layer's n experts split over G ranks, rows moved through peer memory.

"Switch Transformer read for implementation" (molayo1419.me), Expert Parallelism: experts sit on
different devices and the two permutations of the layer become exchanges between them;
"Switch Transformers paper review" (tildalice.io/?p=118): one all-to-all before the experts and
one after. Rank q owns experts q E .. q E + E - 1 (E = n / G) and holds only their weights.

One forward of rank r (every step runs in the library's kernels; this module only orders the
calls and the one collective):
  1. route its own tokens over all n experts, capacity slots over its own tokens;
  2. gather every rank's expert_offsets [n + 1] (one all-gather of n + 1 int32);
  3. moe_ep_plan: where this rank's rows go in each owner's receive buffer, and where the rows
     of its own experts lie in its receive buffer;
  4. moe_ep_dispatch: each token read once, stored into its picks' owners' receive buffers;
  5. (all ranks) moe_expert_ffn of the owner on its receive buffer with its E experts;
  6. (all ranks) moe_ep_combine: gated sum of the owners' output rows, read from peer memory.
Steps 4 -> 5 -> 6 cross ranks, so every rank finishes a step before any rank starts the next
(a device synchronisation and a barrier here). The owner's receive buffer holds, per local
expert, the rows of source rank 0, then rank 1, ...: the rows the one-GPU layer gives that
expert on the concatenated batch with one capacity segment per rank, so the results are bit for
bit those of the one-GPU moe_expert_ffn + moe_combine on that batch.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import (MOE_SIGMOID, MOE_SOFTMAX, lib, moe_capacity_slots, moe_ep_combine, moe_ep_dispatch, moe_ep_plan,
               moe_expert_ffn, moe_router_prepare, moe_router_topk)
from .layer import LayerShape


def gather_offsets(expert_offsets: torch.Tensor, group=None) -> torch.Tensor:
    """Every rank's expert_offsets [n + 1], stacked by rank: [G, n + 1] (one all-gather)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return expert_offsets.reshape(1, -1).clone()
    G = dist.get_world_size(group)
    n1 = expert_offsets.numel()
    out = torch.empty((G * n1,), dtype=expert_offsets.dtype, device=expert_offsets.device)
    dist.all_gather_into_tensor(out, expert_offsets.contiguous().reshape(-1), group=group)
    return out.reshape(G, n1)


def local_experts(weights: dict, rank: int, G: int, n: int) -> dict:
    """The slices of the expert weights rank `rank` owns (views, no copy), plus the router weight."""
    E = n // G
    lo, hi = rank * E, (rank + 1) * E
    out = {key: weights[key][lo:hi] for key in ("w1", "b1", "w2", "b2")}
    out["w_r"] = weights["w_r"]
    if weights.get("rank_bias") is not None:
        out["rank_bias"] = weights["rank_bias"]
    return out


class EPShard:
    """One rank's buffers: its routing and capacity outputs, its receive buffer and its experts' output.

    max_recv_rows bounds the rows any owner can receive: G ranks x m tokens x k picks in the worst
    case; with capacity C per expert per segment, at most G x nseg x C x E."""

    def __init__(self, shape: LayerShape, weights_local: dict, rank: int, G: int, max_recv_rows: int,
                 device="cuda", alloc=None):
        s = self.shape = shape
        if s.n % G:
            raise ValueError("n must be divisible by the number of ranks")
        self.rank, self.G, self.E = rank, G, s.n // G
        self.w = weights_local
        self.device = torch.device(device)
        m, n, k, d = s.m, s.n, s.k, s.d
        self.seg_len = s.seg_len or m
        nseg = m // self.seg_len
        i32, f32, dev = torch.int32, torch.float32, self.device
        alloc = alloc or (lambda shp, dt: torch.empty(shp, dtype=dt, device=dev))
        self.max_recv_rows = max_recv_rows
        self.buf = dict(
            topk_idx=torch.empty((m, k), dtype=i32, device=dev),
            topk_gate=torch.empty((m, k), dtype=f32, device=dev),
            probs=torch.empty((m, n), dtype=f32, device=dev),
            slot=torch.empty((m, k), dtype=i32, device=dev),
            dest_row=torch.empty((m, k), dtype=i32, device=dev),
            src_token=torch.empty((m * k,), dtype=i32, device=dev),
            expert_offsets=torch.empty((n + 1,), dtype=i32, device=dev),
            routed_count=torch.empty((nseg, n), dtype=i32, device=dev),
            kept_count=torch.empty((nseg, n), dtype=i32, device=dev),
            send_base=torch.empty((n,), dtype=i32, device=dev),
            recv_offsets=torch.empty((self.E + 1,), dtype=i32, device=dev),
            ep_row=torch.empty((m, k), dtype=i32, device=dev),
            y=torch.empty((m, d), dtype=s.dtype, device=dev),
        )
        # the two buffers other ranks read or write: from `alloc` (symmetric memory across GPUs)
        self.xrecv = alloc((max_recv_rows, d), s.dtype)
        self.yrecv = alloc((max_recv_rows, d), s.dtype)
        L = lib()
        dt = 1 if s.dtype == torch.bfloat16 else 0
        self.ws_router = torch.empty((max(L.moe_router_topk_workspace_size(d, n, k, dt), 1),), dtype=torch.uint8,
                                     device=dev)
        self.ws_cap = torch.empty((max(L.moe_capacity_slots_workspace_size(m, k, n, self.seg_len), 1),),
                                  dtype=torch.uint8, device=dev)
        self.ws_ffn = torch.empty((L.moe_expert_ffn_workspace_size(dt, max_recv_rows, s.d_ff),), dtype=torch.uint8,
                                  device=dev)
        self.router_prepared = L.moe_router_topk_workspace_size(d, n, k, dt) > 0
        if self.router_prepared:
            moe_router_prepare(self.w["w_r"], k, s.dtype, workspace=self.ws_router)

    def route(self, x: torch.Tensor, stream=None) -> None:
        """Router and capacity slots over this rank's tokens (all n experts)."""
        s, b = self.shape, self.buf
        fn = MOE_SOFTMAX if s.score_fn == "softmax" else MOE_SIGMOID
        moe_router_topk(x, None if self.router_prepared else self.w["w_r"], s.n, s.k, fn, s.renorm_topk,
                        rank_bias=self.w.get("rank_bias"), probs_out=b["probs"], topk_idx=b["topk_idx"],
                        topk_gate=b["topk_gate"], workspace=self.ws_router, stream=stream)
        moe_capacity_slots(b["topk_idx"], s.n, s.capacity, self.seg_len, out=b, workspace=self.ws_cap, stream=stream)

    def plan(self, offsets_all: torch.Tensor, stream=None) -> None:
        moe_ep_plan(offsets_all, self.rank, send_base=self.buf["send_base"], recv_offsets=self.buf["recv_offsets"],
                    stream=stream)

    def dispatch(self, x: torch.Tensor, peer_xrecv: torch.Tensor, stream=None) -> None:
        b = self.buf
        moe_ep_dispatch(x, b["topk_idx"], b["dest_row"], b["expert_offsets"], b["send_base"], peer_xrecv, self.G,
                        self.max_recv_rows, ep_row=b["ep_row"], stream=stream)

    def ffn(self, stream=None) -> None:
        """The owner's FFN on its receive buffer with its E experts."""
        w = self.w
        moe_expert_ffn(self.xrecv, w["w1"], w["b1"], w["w2"], w["b2"], self.buf["recv_offsets"], ybuf=self.yrecv,
                       workspace=self.ws_ffn, stream=stream)

    def combine(self, peer_yrecv: torch.Tensor, residual=None, stream=None) -> torch.Tensor:
        b, s = self.buf, self.shape
        return moe_ep_combine(peer_yrecv, s.dtype, b["ep_row"], b["topk_idx"], s.n, self.G, b["topk_gate"],
                              residual=residual, y=b["y"], stream=stream)


def pointer_array(tensors, device) -> torch.Tensor:
    """A device int64 array of the tensors' addresses (the peer arrays of moe_ep_dispatch / combine)."""
    return torch.tensor([t.data_ptr() for t in tensors], dtype=torch.int64, device=device)


def forward_ranks_on_one_device(shards, xs, residual=False):
    """All G ranks of an expert-parallel forward run by one process on one GPU, one step after the
    other (every rank's dispatch, then every owner's FFN, then every combine): the same kernels and
    the same stores, with the ranks' buffers side by side in one device's memory. Returns the ys."""
    dev = xs[0].device
    for sh, x in zip(shards, xs):
        sh.route(x)
    offsets_all = torch.stack([sh.buf["expert_offsets"] for sh in shards])
    for sh in shards:
        sh.plan(offsets_all)
    peer_x = pointer_array([sh.xrecv for sh in shards], dev)
    peer_y = pointer_array([sh.yrecv for sh in shards], dev)
    for sh, x in zip(shards, xs):
        sh.dispatch(x, peer_x)
    for sh in shards:
        sh.ffn()
    return [sh.combine(peer_y, residual=x if residual else None) for sh, x in zip(shards, xs)]


class SymmetricBuffers:
    """Receive and output buffers in torch symmetric memory: every rank can store into and load from
    every other rank's buffers; buffer_ptrs_dev is the device array of the G buffer addresses."""

    def __init__(self, group=None):
        self.group = group if group is not None else dist.group.WORLD
        self.handles = []

    def alloc(self, shape, dtype):
        from torch.distributed import _symmetric_memory as symm
        t = symm.empty(*shape, dtype=dtype, device=torch.device("cuda", torch.cuda.current_device()))
        self.handles.append((t, symm.rendezvous(t, self.group)))
        return t

    def peers(self, t: torch.Tensor) -> torch.Tensor:
        for buf, h in self.handles:
            if buf is t:
                return torch.tensor(list(h.buffer_ptrs), dtype=torch.int64, device=t.device)
        raise KeyError("not a symmetric buffer of this group")


def forward_rank(shard: EPShard, x: torch.Tensor, peer_x: torch.Tensor, peer_y: torch.Tensor, group=None,
                 residual=False) -> torch.Tensor:
    """One rank of a multi-GPU expert-parallel forward (one process per GPU, NCCL process group).
    The steps that cross ranks are separated by a device synchronisation and a barrier."""
    shard.route(x)
    offsets_all = gather_offsets(shard.buf["expert_offsets"], group)
    shard.plan(offsets_all)
    shard.dispatch(x, peer_x)
    torch.cuda.synchronize()
    dist.barrier(group=group)
    shard.ffn()
    torch.cuda.synchronize()
    dist.barrier(group=group)
    y = shard.combine(peer_y, residual=x if residual else None)
    torch.cuda.synchronize()
    dist.barrier(group=group)  # no rank reuses its buffers while another still reads them
    return y
