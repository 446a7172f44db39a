"""Expert parallelism through the C ABI: G ranks run by one process on one GPU.

Each rank routes its own tokens, then moe_ep_plan / moe_ep_dispatch store its rows into the
owners' receive buffers, each owner runs moe_expert_ffn on its E experts, and moe_ep_combine
gathers the outputs back (the ranks' buffers side by side in one device's memory; the kernels
wait on nothing, the steps run one after the other). Checked against:
  - the oracle's dispatch of the concatenated batch (one capacity segment per rank), taken on
    the GPU's own routing: every owner's receive buffer holds exactly those rows of its experts;
  - the one-GPU path on the concatenated batch (moe_expert_ffn + moe_combine, which the layer
    itself takes for k >= 2): outputs bit for bit (each expert's rows reach the same FFN tile
    positions and the combine takes the same operations in the same order).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from gpu_util import dev, host

pytestmark = pytest.mark.gpu

lb = pytest.importorskip("load_balanced_dispatch_b200")
from load_balanced_dispatch_b200 import ep  # noqa: E402
from load_balanced_dispatch_b200.layer import LayerShape, MoELayer, weights_to_device  # noqa: E402


def _cfg(m_rank, G, n, k, d, d_ff, seg_per_rank, cf, score_fn="softmax", renorm=1):
    m = m_rank * G
    seg = m_rank // seg_per_rank
    return W.LayerConfig("ep", m=m, d=d, n=n, k=k, d_ff=d_ff, score_fn=score_fn, dtype="bf16",
                         capacity=W.capacity_from_factor(cf, seg, k, n), seg_len=seg,
                         wr_std=1.0 / np.sqrt(d), renorm_topk=renorm)


def _shape(cfg, m):
    return LayerShape(m=m, d=cfg.d, n=cfg.n, k=cfg.k, d_ff=cfg.d_ff, score_fn=cfg.score_fn, dtype=torch.bfloat16,
                      capacity=cfg.capacity, seg_len=cfg.seg_len, renorm_topk=cfg.renorm_topk)


@pytest.mark.parametrize("G,m_rank,n,k,d,d_ff,seg_per_rank,cf", [(2, 1024, 16, 2, 256, 512, 1, 2.0),
                                                                (4, 512, 32, 2, 256, 384, 2, 1.25),
                                                                (2, 640, 8, 1, 512, 1024, 1, 1.25),
                                                                (4, 256, 64, 6, 128, 256, 1, 10.0)])
@pytest.mark.parametrize("residual", [False, True])
def test_ep_matches_one_gpu_layer_and_oracle_layout(G, m_rank, n, k, d, d_ff, seg_per_rank, cf, residual):
    cfg = _cfg(m_rank, G, n, k, d, d_ff, seg_per_rank, cf)
    inp = W.make_layer_inputs(cfg, seed=G + n, bias_std=0.05)
    w = weights_to_device(inp, torch.bfloat16)
    x_all = dev(inp["x"], torch.bfloat16)
    # the one-GPU layer on the concatenated batch
    layer = MoELayer(_shape(cfg, cfg.m), w)
    layer.shape.residual = residual
    y_one = layer.forward(x_all).clone()
    lb.sync_status()
    # G ranks, each with its tokens and its experts
    max_recv = cfg.m * k
    shards = [ep.EPShard(_shape(cfg, m_rank), ep.local_experts(w, r, G, n), r, G, max_recv) for r in range(G)]
    xs = [x_all[r * m_rank:(r + 1) * m_rank] for r in range(G)]
    ys = ep.forward_ranks_on_one_device(shards, xs, residual=residual)
    torch.cuda.synchronize()
    lb.sync_status()
    # routing and capacity per rank = the one-GPU layer's on that rank's tokens (segments align)
    idx_all = torch.cat([sh.buf["topk_idx"] for sh in shards])
    assert torch.equal(idx_all, layer.buf["topk_idx"])
    # each owner's receive buffer = the oracle's dispatch rows of its experts
    idx_h = host(idx_all)
    cap = oracle.capacity(idx_h, cfg.m, k, n, cfg.capacity, cfg.seg_len)
    off = cap["expert_offsets"]
    xbuf = oracle.dispatch(inp["x"], cap["src_token"], int(off[-1]))
    E = n // G
    for q, sh in enumerate(shards):
        lo, hi = int(off[q * E]), int(off[(q + 1) * E])
        ro = host(sh.buf["recv_offsets"])
        assert (ro == off[q * E:(q + 1) * E + 1] - lo).all()
        assert (host(sh.xrecv)[: hi - lo] == xbuf[lo:hi]).all()
    # outputs: bit for bit the one-GPU path's moe_expert_ffn + moe_combine on the same batch
    ybuf = lb.moe_expert_ffn(layer.buf["xbuf"], w["w1"], w["b1"], w["w2"], w["b2"], layer.buf["expert_offsets"])
    y_ref = lb.moe_combine(ybuf, layer.buf["dest_row"], layer.buf["topk_gate"], residual=x_all if residual else None)
    torch.cuda.synchronize()
    y_ep = torch.cat(ys)
    assert torch.equal(y_ep, y_ref)
    if k > 1:  # the layer itself takes the same two calls
        assert torch.equal(y_ep, y_one)


def test_ep_single_rank_is_the_layer():
    # G = 1: every expert local, the plan is the identity layout
    cfg = _cfg(768, 1, 16, 2, 256, 512, 3, 1.5)
    inp = W.make_layer_inputs(cfg, seed=3)
    w = weights_to_device(inp, torch.bfloat16)
    x = dev(inp["x"], torch.bfloat16)
    layer = MoELayer(_shape(cfg, cfg.m), w)
    y_one = layer.forward(x).clone()
    sh = ep.EPShard(_shape(cfg, cfg.m), ep.local_experts(w, 0, 1, 16), 0, 1, cfg.m * 2)
    (y,) = ep.forward_ranks_on_one_device([sh], [x])
    torch.cuda.synchronize()
    lb.sync_status()
    assert (host(sh.buf["send_base"]) == host(layer.buf["expert_offsets"])[:-1]).all()
    assert (host(sh.buf["recv_offsets"]) == host(layer.buf["expert_offsets"])).all()
    assert torch.equal(y, y_one)
