"""Pins for the oracle's expert FFN and load statistics.

FFN: a hand-computed case, special cases (identity weights, one expert with no
drop = the dense FFN, checked with torch's CPU linear layers). Statistics: the
golden balanced-loss identity, sum f = 1, micro = global for identical
micro-batches, hand-computed MaxVio and the exact Loss-Free update.
Sources: "Switch Transformers paper review" (tildalice.io/?p=118), Switch Layer
FFN and the auxiliary load balancing loss; "Qwen global-batch load balance"
(agentlenshq.com); "MoE travelogue 6" (kexue.fm/archives/11619), eq. (2) and
Demo code.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W


def test_ffn_hand_example():
    # d = 2, d_ff = 2, one expert. W1^T rows: [1, -1], [2, 0]; b1 = [0, -1];
    # x = [3, 1]: pre = [3-1+0, 6+0-1] = [2, 5]; relu -> [2, 5].
    # W2^T rows: [1, 1], [0, -1]; b2 = [0.5, 0]: y = [2+5+0.5, -5+0] = [7.5, -5].
    w1 = np.array([[[1.0, -1.0], [2.0, 0.0]]], np.float32)
    b1 = np.array([[0.0, -1.0]], np.float32)
    w2 = np.array([[[1.0, 1.0], [0.0, -1.0]]], np.float32)
    b2 = np.array([[0.5, 0.0]], np.float32)
    y = oracle.expert_ffn(np.array([[3.0, 1.0], [-1.0, 0.0]]), np.array([0, 2], np.int32), w1, b1, w2, b2)
    assert y[0].tolist() == [7.5, -5.0]
    # x = [-1, 0]: pre = [-1, -2-1] -> relu [0, 0]; y = b2
    assert y[1].tolist() == [0.5, 0.0]


def test_ffn_identity_weights_give_relu():
    d = 5
    eye = np.eye(d, dtype=np.float32)[None]
    x = np.array([[1.0, -2.0, 0.5, -0.25, 3.0]])
    b2 = np.full((1, d), 0.125, np.float32)
    y = oracle.expert_ffn(x, np.array([0, 1], np.int32), eye, np.zeros((1, d), np.float32), eye, b2)
    assert y[0].tolist() == (np.maximum(x[0], 0) + 0.125).tolist()


def test_one_expert_no_drop_equals_dense_ffn():
    cfg = W.scaled_config("tiny", m=48, d=16, n=1, d_ff=24, capacity=48, seg_len=48)
    inp = W.make_layer_inputs(cfg, seed=5, bias_std=0.1)
    out = oracle.layer_forward(inp, cfg)
    assert (out["topk_idx"] == 0).all() and np.allclose(out["topk_gate"], 1.0)
    lin1 = torch.nn.functional.linear(torch.from_numpy(inp["x"]).double(), torch.from_numpy(inp["w1"][0]).double(),
                                      torch.from_numpy(inp["b1"][0]).double())
    ref = torch.nn.functional.linear(torch.relu(lin1), torch.from_numpy(inp["w2"][0]).double(),
                                     torch.from_numpy(inp["b2"][0]).double()).numpy()
    assert np.allclose(out["y"], ref, rtol=1e-12, atol=1e-12)


def test_expert_rows_use_their_own_weights():
    # two experts with different constant weights: each row must use its expert's matrices
    d, d_ff = 3, 2
    w1 = np.stack([np.ones((d_ff, d)), 2 * np.ones((d_ff, d))]).astype(np.float32)
    w2 = np.stack([np.ones((d, d_ff)), -np.ones((d, d_ff))]).astype(np.float32)
    z1, z2 = np.zeros((2, d_ff), np.float32), np.zeros((2, d), np.float32)
    x = np.ones((3, d))
    y = oracle.expert_ffn(x, np.array([0, 1, 3], np.int32), w1, z1, w2, z2)
    assert y[0].tolist() == [6.0] * 3  # hidden [3, 3] -> 6
    assert y[1].tolist() == [-12.0] * 3 and y[2].tolist() == [-12.0] * 3  # hidden [6, 6] -> -12


def test_aux_balanced_golden(golden):
    g = golden("aux_balanced.txt")
    alpha = float(g["alpha"][0])
    for n in (int(v) for v in g["experts"]):
        for k in (1, 2):
            m = 4 * n
            st = oracle.balance_stats(W.make_uniform_probs(m, n), W.make_round_robin_idx(m, n, k), m, n, k, m // 2,
                                      alpha=alpha)
            # per segment, micro-batch mean and global loss equal alpha; the hybrid loss adds
            # 0.01 x the micro-batch loss to the global one: alpha (1 + 0.01)
            assert (st["aux"][:-1] == float(g["expected_aux"][0])).all()
            assert st["aux"][-1] == pytest.approx(alpha * 1.01, rel=1e-15)
            assert (st["f"] == 1.0 / n).all() and (st["P"] == 1.0 / n).all()
            assert (st["vio"] == 0).all()


def test_stats_hand_example():
    # m = 4 tokens, n = 2 experts, top-1 routes [0, 0, 0, 1]; probs rows below.
    probs = np.array([[0.9, 0.1], [0.6, 0.4], [0.7, 0.3], [0.2, 0.8]])
    idx = np.array([[0], [0], [0], [1]], np.int32)
    st = oracle.balance_stats(probs, idx, 4, 2, 1, 2, alpha=0.01)
    # segment 0 = tokens 0,1: f = [1, 0], P = [0.75, 0.25] -> aux = 0.01*2*0.75 = 0.015
    # segment 1 = tokens 2,3: f = [.5, .5], P = [0.45, 0.55] -> aux = 0.01*2*0.5 = 0.01
    # global: f = [.75, .25], P = [0.6, 0.4] -> aux = 0.01*2*(0.45+0.1) = 0.011
    assert st["f"].tolist() == [[1.0, 0.0], [0.5, 0.5], [0.75, 0.25]]
    assert np.allclose(st["P"], [[0.75, 0.25], [0.45, 0.55], [0.6, 0.4]], rtol=1e-15)
    # hybrid ("Qwen global-batch load balance", balancing efficiency and effectiveness): the global
    # loss plus the micro-batch loss with weight 0.01: 0.011 + 0.01 * 0.0125 = 0.011125
    assert np.allclose(st["aux"], [0.015, 0.01, 0.0125, 0.011, 0.011125], rtol=1e-14)
    # MaxVio/MinVio/AvgVio of pooled counts [3, 1]: F = [3/4*2-1, 1/4*2-1] = [0.5, -0.5]
    assert st["vio"].tolist() == [0.5, -0.5, 0.5]


def test_f_sums_to_one_and_micro_equals_global_for_identical_segments():
    rng = np.random.default_rng(2)
    seg, n, k = 32, 8, 2
    p_seg = rng.random((seg, n))
    p_seg /= p_seg.sum(1, keepdims=True)
    i_seg = W.make_topk_idx(seg, n, k, seed=3)
    probs = np.concatenate([p_seg] * 4)
    idx = np.concatenate([i_seg] * 4)
    st = oracle.balance_stats(probs, idx, 4 * seg, n, k, seg)
    assert np.allclose(st["f"].sum(1), 1.0, rtol=1e-15)
    assert np.allclose(st["aux"][:4], st["aux"][0], rtol=1e-14)
    assert st["aux"][4] == pytest.approx(st["aux"][5], rel=1e-12)  # micro mean = global
    # each micro-batch specialised on its own experts: loss per micro-batch is large, pooled loss is not.
    # segment a routes to experts {0,1} with probs 0.5 there, segment b to {2,3}: f and P coincide per segment,
    # micro aux = alpha*n*(2 * 0.5*0.5) = alpha*n/2; globally f = P = 1/4 on 4 experts -> alpha*n/4.
    pa = np.zeros((seg, n)); pa[:, :2] = 0.5
    pb = np.zeros((seg, n)); pb[:, 2:4] = 0.5
    ia = np.tile(np.array([0, 1], np.int32), (seg, 1))
    ib = np.tile(np.array([2, 3], np.int32), (seg, 1))
    st2 = oracle.balance_stats(np.concatenate([pa, pb]), np.concatenate([ia, ib]), 2 * seg, n, 2, seg, alpha=0.01)
    assert st2["aux"][2] == pytest.approx(0.01 * n / 2, rel=1e-15)
    assert st2["aux"][3] == pytest.approx(0.01 * n / 4, rel=1e-15)
    # the hybrid keeps a small pull towards micro-batch balance: global + 0.01 x micro
    assert st2["aux"][4] == pytest.approx(0.01 * n / 4 + 0.01 * 0.01 * n / 2, rel=1e-14)


def test_lossfree_bias_update_exact():
    # counts [5, 3, 4, 0] with m*k = 12, n = 4: mean 3 -> signs [+1, 0, +1, -1]
    idx = np.array([[0], [0], [0], [0], [0], [1], [1], [1], [2], [2], [2], [2]], np.int32)
    b = np.array([0.0, 0.25, -0.05, 0.01], np.float32)
    st = oracle.balance_stats(None, idx, 12, 4, 1, 12, bias=b, gamma=1e-3)
    g = np.float32(1e-3)
    exp = np.array([b[0] - g, b[1], b[2] - g, b[3] + g], np.float32)
    assert st["bias"].tolist() == exp.tolist()
    assert st["P"] is None and st["aux"] is None


# ---------------------------------------------------------------- router gradient of the balance loss
def _loss(h, idx, m, n, k, seg, fn, w_micro, w_global, alpha=1e-2):
    """The balance loss at logits h with the routing (hence f) held fixed: the oracle's router
    scores from h, then the oracle's micro-batch and global-batch losses."""
    probs = oracle.router(None, None, m, 0, n, k, fn, 0, None, logits_in=h)[0]
    aux = oracle.balance_stats(probs, idx, m, n, k, seg, alpha)["aux"]
    nseg = m // seg
    return w_global * aux[nseg + 1] + w_micro * aux[nseg]


@pytest.mark.parametrize("fn,w_micro,w_global", [(oracle.SOFTMAX, 0.01, 1.0), (oracle.SOFTMAX, 1.0, 0.0),
                                                 (oracle.SIGMOID, 0.0, 1.0)])
def test_loss_grad_matches_finite_differences(fn, w_micro, w_global):
    # "Switch Transformers paper review", auxiliary loss: f_i is fixed by the argmax, the gradient
    # flows through P_i. Central differences of the oracle's own loss, routing held fixed.
    m, n, k, seg = 48, 8, 2, 16
    rng = np.random.default_rng(4)
    h = rng.standard_normal((m, n)).astype(np.float32)
    idx = W.make_topk_idx(m, n, k, seed=8, skew=1.0)
    probs = oracle.router(None, None, m, 0, n, k, fn, 0, None, logits_in=h)[0]
    g = oracle.balance_loss_grad(probs, idx, m, n, k, seg, fn, 1e-2, w_micro, w_global)
    for t, j in [(0, 0), (5, 3), (17, 7), (33, 1), (47, 6)]:
        hp, hm = h.copy(), h.copy()
        hp[t, j] = np.float32(h[t, j] + np.float32(2e-3))
        hm[t, j] = np.float32(h[t, j] - np.float32(2e-3))
        step = float(hp[t, j]) - float(hm[t, j])
        fd = (_loss(hp, idx, m, n, k, seg, fn, w_micro, w_global) -
              _loss(hm, idx, m, n, k, seg, fn, w_micro, w_global)) / step
        assert fd == pytest.approx(g[t, j], rel=1e-4, abs=1e-12)


def test_loss_grad_softmax_rows_sum_to_zero_and_vanish_at_balance():
    m, n, k, seg = 64, 8, 2, 32
    rng = np.random.default_rng(5)
    p = rng.random((m, n))
    p /= p.sum(1, keepdims=True)
    g = oracle.balance_loss_grad(p, W.make_topk_idx(m, n, k, seed=2), m, n, k, seg, oracle.SOFTMAX, 1e-2, 0.01, 1.0)
    # softmax is unchanged by adding a constant to a token's logits: each gradient row sums to 0
    assert np.abs(g.sum(1)).max() < 1e-18
    assert np.abs(g).max() > 1e-6
    # f_i = 1/n in every segment: dL/dp is the same for every expert, so the gradient vanishes
    g0 = oracle.balance_loss_grad(p, W.make_round_robin_idx(m, n, k), m, n, k, seg, oracle.SOFTMAX, 1e-2, 0.01, 1.0)
    assert np.abs(g0).max() < 1e-18
