"""Pins for the oracle's router (projection, score function, top-k, gate).

Each check is fixed by something other than the oracle itself: hand-computed
closed forms, the brute-force characterisation of a top-k set, invariances of
softmax, and torch's CPU softmax as an independent library routine.
Sources: "Switch Transformers paper review" (tildalice.io/?p=118), Switch
Routing Steps 1-3 and the Shazeer top-k gate; "MoE travelogue 6"
(kexue.fm/archives/11619), Method review eq. (1) (bias ranks only).
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle


def test_projection_orientation_hand_example():
    # h = x W_r with W_r [d, n]: x = [1, 2], W_r = [[0, 3], [1, 0]] -> h = [2, 3] (top-1 = expert 1).
    # The transposed product would give h = [6, 1] (top-1 = expert 0).
    x = np.array([[1.0, 2.0]], np.float32)
    w = np.array([[0.0, 3.0], [1.0, 0.0]], np.float32)
    probs, idx, gate, margin = oracle.router(x, w, 1, 2, 2, 1)
    assert idx.tolist() == [[1]]
    e2, e3 = math.exp(2.0), math.exp(3.0)
    assert probs[0] == pytest.approx([e2 / (e2 + e3), e3 / (e2 + e3)], rel=1e-15)
    assert gate[0, 0] == pytest.approx(e3 / (e2 + e3), rel=1e-15)
    assert margin[0] == pytest.approx(1.0, abs=1e-15)


def test_softmax_closed_form():
    logits = np.log(np.array([[1.0, 2.0, 3.0, 4.0]], np.float64)).astype(np.float32)
    probs, idx, gate, _ = oracle.router(None, None, 1, 0, 4, 1, logits_in=logits)
    ref = np.array([1, 2, 3, 4], np.float64) / 10.0
    assert np.allclose(probs[0], ref, rtol=1e-6)
    assert idx.tolist() == [[3]]
    assert gate[0, 0] == pytest.approx(0.4, rel=1e-6)


def test_sigmoid_closed_form():
    logits = np.array([[0.0, math.log(3.0), -math.log(3.0)]], np.float32)
    probs, idx, gate, _ = oracle.router(None, None, 1, 0, 3, 2, fn=oracle.SIGMOID, logits_in=logits)
    assert np.allclose(probs[0], [0.5, 0.75, 0.25], rtol=1e-6)
    assert idx.tolist() == [[1, 0]]
    assert np.allclose(gate[0], [0.75, 0.5], rtol=1e-6)


def test_renormalised_topk_gate_closed_form():
    # Softmax(TopK(h)) with h = ln[1,2,3,4], k = 2: selected experts 3, 2 with gates 4/7, 3/7.
    logits = np.log(np.array([[1.0, 2.0, 3.0, 4.0]], np.float64)).astype(np.float32)
    _, idx, gate, _ = oracle.router(None, None, 1, 0, 4, 2, renorm=1, logits_in=logits)
    assert idx.tolist() == [[3, 2]]
    assert np.allclose(gate[0], [4 / 7, 3 / 7], rtol=1e-6)
    # without renormalisation the gate is the full-softmax probability
    _, _, gate0, _ = oracle.router(None, None, 1, 0, 4, 2, renorm=0, logits_in=logits)
    assert np.allclose(gate0[0], [0.4, 0.3], rtol=1e-6)


def test_ties_go_to_lowest_index():
    logits = np.zeros((3, 8), np.float32)
    for k in (1, 3, 8):
        _, idx, gate, margin = oracle.router(None, None, 3, 0, 8, k, logits_in=logits)
        assert (idx == np.arange(k)[None, :]).all()
        assert np.allclose(gate, 1 / 8)
        if k < 8:
            assert (margin == 0).all()


def _is_topk_set(key, S):
    """A set S is the top-k iff every member outranks every non-member (larger key, or equal key and lower index)."""
    out = [j for j in range(len(key)) if j not in S]
    return all(key[a] > key[b] or (key[a] == key[b] and a < b) for a in S for b in out)


@pytest.mark.parametrize("seed", range(6))
def test_topk_matches_bruteforce_characterisation(seed):
    rng = np.random.default_rng(seed)
    n, k, m = 7, 3, 40
    # coarse values force many exact ties
    logits = rng.integers(-3, 4, size=(m, n)).astype(np.float32)
    _, idx, _, _ = oracle.router(None, None, m, 0, n, k, logits_in=logits)
    for i in range(m):
        sets = [set(S) for S in itertools.combinations(range(n), k) if _is_topk_set(logits[i], set(S))]
        assert len(sets) == 1
        assert set(idx[i].tolist()) == sets[0]
        # listed best first
        order = sorted(idx[i].tolist(), key=lambda j: (-logits[i, j], j))
        assert idx[i].tolist() == order


def test_softmax_matches_torch_and_shift_invariance():
    rng = np.random.default_rng(3)
    m, d, n = 16, 12, 9
    x = rng.standard_normal((m, d)).astype(np.float32)
    w = rng.standard_normal((d, n)).astype(np.float32)
    probs, idx, gate, _ = oracle.router(x, w, m, d, n, 1)
    h = torch.from_numpy(x).double() @ torch.from_numpy(w).double()
    ref = torch.softmax(h, dim=-1).numpy()
    assert np.allclose(probs, ref, rtol=1e-12, atol=1e-15)
    assert (idx[:, 0] == ref.argmax(1)).all()
    assert np.allclose(gate[:, 0], ref.max(1), rtol=1e-12)
    # adding a constant to every logit changes nothing (shift invariance of softmax)
    logits = (h.numpy() + 0.0).astype(np.float32)
    p1, i1, _, _ = oracle.router(None, None, m, 0, n, 2, logits_in=logits)
    p2, i2, _, _ = oracle.router(None, None, m, 0, n, 2, logits_in=logits + np.float32(4.0))
    assert (i1 == i2).all()
    assert np.allclose(p1, p2, rtol=1e-5)


def test_expert_permutation_equivariance():
    rng = np.random.default_rng(4)
    m, d, n, k = 10, 6, 8, 2
    x = rng.standard_normal((m, d)).astype(np.float32)
    w = rng.standard_normal((d, n)).astype(np.float32)
    perm = rng.permutation(n)
    p, i, g, _ = oracle.router(x, w, m, d, n, k)
    pp, ip, gp, _ = oracle.router(x, w[:, perm], m, d, n, k)
    assert np.allclose(pp, p[:, perm], rtol=1e-14)
    assert (perm[ip] == i).all()
    assert np.allclose(gp, g)


def test_lossfree_bias_changes_ranking_not_gate():
    # rho = sigmoid(h): expert 0 has the larger score, but the bias lifts expert 1 above it.
    logits = np.array([[1.0, 0.9, -2.0]], np.float32)
    bias = np.array([0.0, 0.1, 0.0], np.float32)
    probs, idx, gate, _ = oracle.router(None, None, 1, 0, 3, 1, fn=oracle.SIGMOID, rank_bias=bias, logits_in=logits)
    assert idx.tolist() == [[1]]
    assert gate[0, 0] == pytest.approx(1 / (1 + math.exp(-0.9)), rel=1e-6)
    _, idx0, gate0, _ = oracle.router(None, None, 1, 0, 3, 1, fn=oracle.SIGMOID, logits_in=logits)
    assert idx0.tolist() == [[0]]
    assert gate0[0, 0] == pytest.approx(1 / (1 + math.exp(-1.0)), rel=1e-6)


def test_margin_definition():
    logits = np.array([[0.5, 2.0, 1.25, 1.0]], np.float32)
    _, idx, _, margin = oracle.router(None, None, 1, 0, 4, 2, logits_in=logits)
    assert idx.tolist() == [[1, 2]]
    assert margin[0] == pytest.approx(0.25)
    _, _, _, margin_all = oracle.router(None, None, 1, 0, 4, 4, logits_in=logits)
    assert math.isinf(margin_all[0])
