"""One MoE-layer forward through the C ABI: buffers owned by torch, stages run in order.

The runner only allocates device buffers once and calls the library's entry
points in the order the layer defines (router -> [balance] -> capacity ->
dispatch -> expert FFN -> combine, and the statistics beside them once the
router is done). All arithmetic happens in the library's kernels.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import (MOE_QB_MIDPOINT, MOE_QB_STEP, MOE_SIGMOID, MOE_SOFTMAX, moe_balance_assign, moe_balance_stats,
               moe_capacity_slots, moe_combine, moe_dispatch_tokens, moe_expert_ffn, moe_expert_ffn_combine,
               moe_expert_ffn_gather, moe_router_prepare, moe_router_topk, lib)


@dataclass
class LayerShape:
    m: int
    d: int
    n: int
    k: int
    d_ff: int
    score_fn: str = "softmax"
    dtype: torch.dtype = torch.bfloat16
    capacity: int = 0
    seg_len: int = 0
    renorm_topk: int = 0
    alpha: float = 1e-2
    gamma: float = 1e-3
    residual: bool = False
    lossfree: bool = False   # update the Loss-Free ranking bias after each forward


class MoELayer:
    """Device-resident weights and preallocated buffers for repeated forwards."""

    def __init__(self, shape: LayerShape, weights: dict, device="cuda"):
        s = self.shape = shape
        self.device = torch.device(device)
        self.w = weights  # x-independent tensors on the device: w_r, w1, b1, w2, b2, rank_bias (optional)
        m, n, k, d = s.m, s.n, s.k, s.d
        seg = s.seg_len or m
        self.seg_len = seg
        nseg = m // seg
        dev = self.device
        i32, f32 = torch.int32, torch.float32
        bf16 = s.dtype == torch.bfloat16
        self.rows_max = m * k
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
            xbuf=torch.empty((self.rows_max, d), dtype=s.dtype, device=dev),  # k = 1 bf16 needs no ybuf
            ybuf=torch.empty((0 if (bf16 and k == 1) else self.rows_max, d), dtype=s.dtype, device=dev),
            y=torch.empty((m, d), dtype=s.dtype, device=dev),
            f=torch.empty((nseg + 1, n), dtype=f32, device=dev),
            P=torch.empty((nseg + 1, n), dtype=f32, device=dev),
            aux=torch.empty((nseg + 3,), dtype=f32, device=dev),
            vio=torch.empty((3,), dtype=f32, device=dev),
        )
        L = lib()
        dt = 1 if s.dtype == torch.bfloat16 else 0
        self.ws = dict(
            router=torch.empty((max(L.moe_router_topk_workspace_size(d, n, k, dt), 1),), dtype=torch.uint8,
                               device=dev),
            cap=torch.empty((max(L.moe_capacity_slots_workspace_size(m, k, n, seg), 1),), dtype=torch.uint8, device=dev),
            ffn=torch.empty((L.moe_expert_ffn_workspace_size(dt, self.rows_max, s.d_ff),), dtype=torch.uint8,
                            device=dev),
            stats=torch.empty((max(L.moe_balance_stats_workspace_size(m, n, seg), 1),), dtype=torch.uint8,
                              device=dev),
        )
        # the router weight is static: on the tensor-core path its bf16 split is made once, here
        self.router_prepared = L.moe_router_topk_workspace_size(d, n, k, dt) > 0
        if self.router_prepared:
            moe_router_prepare(self.w["w_r"], k, s.dtype, workspace=self.ws["router"])
        # one pick per token in bf16: the combine runs in the FFN's second GEMM (moe_expert_ffn_combine).
        # gather = True would let the FFN read its rows from x (moe_expert_ffn_gather: no dispatch, no
        # xbuf); measured slower, it is off
        self.gather = False
        self.ffn_combine = s.k == 1 and s.dtype == torch.bfloat16
        # data-parallel replicas: set by enable_global_stats(); the Loss-Free bias then follows the
        # pooled counts of every rank instead of this rank's
        self.global_stats = None

    STAGES = ("router", "capacity", "dispatch", "ffn", "combine", "stats")

    def _stage(self, i: int, x: torch.Tensor, st) -> None:
        s, b, w = self.shape, self.buf, self.w
        if i == 0:
            fn = MOE_SOFTMAX if s.score_fn == "softmax" else MOE_SIGMOID
            moe_router_topk(x, None if self.router_prepared else w["w_r"], s.n, s.k, fn, s.renorm_topk,
                            rank_bias=w.get("rank_bias"),
                            probs_out=b["probs"], topk_idx=b["topk_idx"], topk_gate=b["topk_gate"],
                            workspace=self.ws["router"], stream=st)
        elif i == 1:
            moe_capacity_slots(b["topk_idx"], s.n, s.capacity, self.seg_len, out=b, workspace=self.ws["cap"], stream=st)
        elif i == 2:
            if self.uses_dispatch():  # otherwise the FFN gathers its rows from x
                # token-major: each token read once, written to each of its kept rows
                moe_dispatch_tokens(x, b["dest_row"], self.rows_max, xbuf=b["xbuf"], stream=st)
        elif i == 3:
            if self.ffn_combine:
                moe_expert_ffn_combine(b["xbuf"], w["w1"], w["b1"], w["w2"], w["b2"], b["expert_offsets"],
                                       b["src_token"], b["dest_row"], b["topk_gate"],
                                       residual=x if s.residual else None, y=b["y"], workspace=self.ws["ffn"],
                                       stream=st)
            elif self.gather:
                moe_expert_ffn_gather(x, w["w1"], w["b1"], w["w2"], w["b2"], b["expert_offsets"], b["src_token"],
                                      max_rows=self.rows_max, ybuf=b["ybuf"], workspace=self.ws["ffn"], stream=st)
            else:
                moe_expert_ffn(b["xbuf"], w["w1"], w["b1"], w["w2"], w["b2"], b["expert_offsets"], ybuf=b["ybuf"],
                               workspace=self.ws["ffn"], stream=st)
        elif i == 4:
            if not self.ffn_combine:  # otherwise done by the FFN's second GEMM
                moe_combine(b["ybuf"], b["dest_row"], b["topk_gate"], residual=x if s.residual else None, y=b["y"],
                            stream=st)
        else:
            local_bias = s.lossfree and self.global_stats is None
            moe_balance_stats(b["probs"], b["topk_idx"], s.n, self.seg_len, s.alpha,
                              bias_inout=w.get("rank_bias") if local_bias else None, gamma=s.gamma, out=b,
                              workspace=self.ws["stats"], stream=st)

    def forward(self, x: torch.Tensor, stream=None, events=None) -> torch.Tensor:
        """One forward through the C ABI on `stream`. The statistics read only the router's outputs, so
        they run on a side stream (forked after the router, joined at the end) beside capacity, dispatch,
        FFN and combine. `events`: optional 7 CUDA events; then the 6 stages run one after another on
        `stream` with the events recorded between them (per-stage timing)."""
        st = stream if stream is not None else torch.cuda.current_stream()
        if events is not None:
            for i in range(len(self.STAGES)):
                events[i].record(st)
                self._stage(i, x, st)
            events[len(self.STAGES)].record(st)
            return self.buf["y"]
        if not hasattr(self, "_side"):
            self._side = torch.cuda.Stream(device=self.device)
            self._fork, self._join = torch.cuda.Event(), torch.cuda.Event()
        self._stage(0, x, st)
        self._fork.record(st)
        self._side.wait_event(self._fork)
        self._stage(5, x, self._side)
        for i in range(1, 5):
            self._stage(i, x, st)
        self._join.record(self._side)
        st.wait_event(self._join)
        return self.buf["y"]

    def uses_dispatch(self) -> bool:
        """Whether the forward forms xbuf with moe_dispatch (the fused-combine FFN always reads xbuf)."""
        return self.ffn_combine or not self.gather

    def capture(self, x: torch.Tensor) -> None:
        """Record forward(x) as one CUDA graph, and each stage into a graph of its own for per-stage
        timing (x's address is baked in). The first forward runs eagerly so one-time host set-up
        happens outside the capture."""
        self.forward(x)
        torch.cuda.synchronize()
        self.graphs = []
        for i in range(len(self.STAGES)):
            if (i == 4 and self.ffn_combine) or (i == 2 and not self.uses_dispatch()):  # done inside the FFN stage
                self.graphs.append(None)
                continue
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self._stage(i, x, torch.cuda.current_stream())
            self.graphs.append(g)
        self.graph_all = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph_all):
            self.forward(x, stream=torch.cuda.current_stream())
        torch.cuda.synchronize()

    def replay(self, events=None) -> torch.Tensor:
        """Replay the captured forward on the current stream: the whole-forward graph, or with
        `events` (7 CUDA events) the per-stage graphs with the events recorded between them."""
        st = torch.cuda.current_stream()
        if events is None:
            self.graph_all.replay()
            return self.buf["y"]
        for i, g in enumerate(self.graphs):
            events[i].record(st)
            if g is not None:
                g.replay()
        events[len(self.graphs)].record(st)
        return self.buf["y"]

    def enable_global_stats(self, m_total: int, group=None) -> None:
        """Pool the statistics over data-parallel ranks: after each forward, `sync_global_stats`
        sums this rank's totals with every other rank's (one all-reduce of 2 n doubles) and
        computes the global-batch f, P, loss and violations, and the Loss-Free update, which
        then no longer follows this rank's counts alone."""
        from . import lib as _lib
        n, m = self.shape.n, self.shape.m
        dev = self.device
        self.global_stats = dict(
            m_total=m_total, group=group,
            totals=torch.empty((2, n), dtype=torch.float64, device=dev),
            ws=torch.empty((max(_lib().moe_balance_totals_workspace_size(m, n), 1),), dtype=torch.uint8, device=dev),
            out=dict(f=torch.empty((n,), dtype=torch.float32, device=dev),
                     P=torch.empty((n,), dtype=torch.float32, device=dev),
                     aux=torch.empty((1,), dtype=torch.float32, device=dev),
                     vio=torch.empty((3,), dtype=torch.float32, device=dev)))

    def sync_global_stats(self, stream=None) -> dict:
        """The cross-rank step of a data-parallel forward (see enable_global_stats)."""
        from .dp import global_batch_stats
        g, s, b = self.global_stats, self.shape, self.buf
        return global_batch_stats(b["probs"], b["topk_idx"], s.n, g["m_total"], alpha=s.alpha,
                                  bias_inout=self.w.get("rank_bias") if s.lossfree else None, gamma=s.gamma,
                                  group=g["group"], totals=g["totals"], workspace=g["ws"], out=g["out"],
                                  stream=stream)

    def launches_per_forward(self) -> int:
        """Kernel launches of one forward: router (bf16 with n <= 128: projection and finish, 2, except
        n <= 64 with more 128-token tiles than SMs, where the projection kernel finishes the rows, 1;
        else 1), capacity 2 (count + scan, assign), dispatch 1 (0 when the FFN
        gathers its rows from x), FFN (bf16: one fused launch, after a memset of its counters; fp32: 2),
        combine 1, statistics 1. With one pick per token in bf16 the combine is the FFN's epilogue plus
        one launch for the dropped tokens' rows (which also clears the FFN's counters)."""
        s = self.shape
        bf16 = s.dtype == torch.bfloat16
        # bf16 with n <= 128: tensor-core logits tiles + the finish kernel (the W_r split is made
        # once, at construction), or one launch when the projection kernel finishes whole rows
        # (n <= 64 and more 128-token tiles than SMs); otherwise the fp32 FMA kernel
        sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
        rows_mode = s.n <= 64 and (s.m + 127) // 128 > sms
        router = 2 if (bf16 and s.n <= 128 and not rows_mode) else 1
        capacity = 2
        dispatch = 1 if self.uses_dispatch() else 0
        if self.ffn_combine:  # the FFN with the combine in its epilogue, plus the dropped rows
            ffn, combine = 2, 0
        else:
            ffn, combine = (1 if bf16 else 2), 1
        return router + capacity + dispatch + ffn + combine + 1


def weights_to_device(inp: dict, dtype: torch.dtype, device="cuda") -> dict:
    """Move numpy inputs from `workloads.make_layer_inputs` to the device (bf16-representable values convert exactly)."""
    out = {}
    for key in ("w1", "b1", "w2", "b2"):
        out[key] = torch.from_numpy(inp[key]).to(device=device, dtype=dtype).contiguous()
    out["w_r"] = torch.from_numpy(inp["w_r"]).to(device=device, dtype=torch.float32).contiguous()
    if inp.get("rank_bias") is not None:
        out["rank_bias"] = torch.from_numpy(inp["rank_bias"]).to(device=device, dtype=torch.float32).contiguous()
    return out
