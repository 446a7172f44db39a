"""Whole-layer parity: router -> capacity -> dispatch -> FFN -> combine -> statistics
through the C ABI, against the oracle on the same seeded inputs.

Routing computed from GPU logits (fp32) can legitimately differ from the
oracle's (fp64) on a token whose top-k is decided by a near tie. Such a token
is accepted only when the oracle's keys leave the choice open: every expert the
GPU picked lies within MARGIN of the oracle's k-th key. Its routing is then
adopted into the reference (the oracle's capacity, layout and statistics are
recomputed from the adopted routing), so that every segment's slots, rows and
counts, the whole batch's f, P and loss, and the Loss-Free update are compared
in full; the outputs of adopted tokens are left out of the y comparison (their
oracle gates belong to the oracle's picks), and their number is printed.
Reduced sizes compare every token's output; full sizes compare sampled tokens,
each computed one by one by the oracle.
"""
import hashlib

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from gpu_util import MARGIN, TOL_STATS, dev, host, norm_err, tol, torch_dtype

pytestmark = pytest.mark.gpu

lb = pytest.importorskip("load_balanced_dispatch_b200")
from load_balanced_dispatch_b200.layer import LayerShape, MoELayer, weights_to_device  # noqa: E402


def _shape(cfg, residual=False):
    return LayerShape(m=cfg.m, d=cfg.d, n=cfg.n, k=cfg.k, d_ff=cfg.d_ff, score_fn=cfg.score_fn,
                      dtype=torch_dtype(cfg.dtype), capacity=cfg.capacity, seg_len=cfg.seg_len,
                      renorm_topk=cfg.renorm_topk, alpha=cfg.alpha, gamma=cfg.gamma, residual=residual,
                      lossfree=cfg.lossfree_bias > 0)


def _run_gpu(cfg, inp, residual=False):
    w = weights_to_device(inp, torch_dtype(cfg.dtype))
    layer = MoELayer(_shape(cfg, residual), w)
    x = dev(inp["x"], torch_dtype(cfg.dtype))
    layer.forward(x)
    lb.sync_status()
    out = {k: host(v) for k, v in layer.buf.items()}
    if "rank_bias" in w:
        out["rank_bias_new"] = host(w["rank_bias"])
    return out


def _scaled(name, **kw):
    c = W.CONFIGS[name]
    base = dict(m=c.m, d=c.d, d_ff=c.d_ff, seg_len=c.seg_len)
    base.update(kw)
    cf = {"tiny": 1.25, "switch": 1.25, "global": 2.0}.get(name)
    seg = base["seg_len"] if base["seg_len"] <= base["m"] else base["m"]
    base["seg_len"] = seg
    cap = W.capacity_from_factor(cf, seg, c.k, c.n) if cf else seg * c.k
    return W.scaled_config(name, capacity=cap, **base)


def _keys(probs, cfg, bias):
    """The ranking key of every (token, expert) from the oracle's fp64 scores: the logit up to a
    per-token constant (log p) for softmax, rho for sigmoid, fp32(fp32(score) + b) with a bias."""
    if bias is not None:
        return (probs.astype(np.float32) + bias[None, :].astype(np.float32)).astype(np.float64)
    if cfg.score_fn == "softmax":
        with np.errstate(divide="ignore"):
            return np.log(probs)
    return probs


def _adopt_near_ties(cfg, got_idx, ref_idx, probs, bias):
    """The routing to compare against: the oracle's, with the GPU's rows adopted where they differ
    and the oracle's keys leave the choice open (each GPU pick within MARGIN of the k-th key; the
    picks distinct). Returns (routing [m,k], mask of adopted tokens)."""
    idx = ref_idx.copy()
    diff = (got_idx != ref_idx).any(1)
    rows = np.nonzero(diff)[0]
    if len(rows):
        keys = _keys(probs[rows], cfg, bias)
        kth = -np.sort(-keys, axis=1)[:, cfg.k - 1]
        picked = np.take_along_axis(keys, got_idx[rows].astype(np.int64), axis=1)
        assert (picked >= kth[:, None] - MARGIN).all(), "a GPU pick differs from the oracle's by more than a near tie"
        assert all(len(set(r)) == cfg.k for r in got_idx[rows].tolist())
        idx[rows] = got_idx[rows]
    return idx, diff


def _reference(cfg, inp, got, residual=False, sample=None):
    """Oracle router; GPU near-tie choices adopted; then capacity, statistics, and the FFN + combine
    of every token (sample None) or of the sampled tokens only."""
    m, d, n, k = cfg.m, cfg.d, cfg.n, cfg.k
    fn = oracle.SOFTMAX if cfg.score_fn == "softmax" else oracle.SIGMOID
    bias = inp.get("rank_bias")
    probs, r_idx, gate, margin = oracle.router(inp["x"], inp["w_r"], m, d, n, k, fn, cfg.renorm_topk, bias)
    idx, adopted = _adopt_near_ties(cfg, got["topk_idx"], r_idx, probs, bias)
    cap = oracle.capacity(idx, m, k, n, cfg.capacity, cfg.seg_len)
    gbf = int(cfg.dtype == "bf16")
    res = inp["x"] if residual else None
    if sample is None:
        rows = int(cap["expert_offsets"][-1])
        xbuf = oracle.dispatch(inp["x"], cap["src_token"], rows)
        ybuf = oracle.expert_ffn(xbuf, cap["expert_offsets"], inp["w1"], inp["b1"], inp["w2"], inp["b2"])
        y = oracle.combine(ybuf, cap["dest_row"], gate, res, m, k, d, gate_bf16=gbf)
    else:
        # the sampled tokens' kept picks as rows of their own, grouped by expert
        pairs = sorted((int(idx[i, r]), j, r) for j, i in enumerate(sample) for r in range(k)
                       if cap["slot"][i, r] >= 0)
        xs = np.array([inp["x"][sample[j]] for _, j, _ in pairs], np.float64).reshape(-1, d)
        off = np.zeros(n + 1, np.int64)
        for e, _, _ in pairs:
            off[e + 1] += 1
        off = np.cumsum(off).astype(np.int32)
        ys = oracle.expert_ffn(xs, off, inp["w1"], inp["b1"], inp["w2"], inp["b2"]) if pairs else np.zeros((1, d))
        dest = -np.ones((len(sample), k), np.int32)
        for row, (_, j, r) in enumerate(pairs):
            dest[j, r] = row
        y = oracle.combine(ys, dest, gate[sample], None if res is None else res[sample], len(sample), k, d,
                           gate_bf16=gbf)
    st = oracle.balance_stats(probs, idx, m, n, k, cfg.seg_len, cfg.alpha, bias, cfg.gamma)
    return dict(probs=probs, oracle_idx=r_idx, topk_idx=idx, adopted=adopted, topk_gate=gate, margin=margin,
                cap=cap, y=y, stats=st)


def _compare_layer(cfg, got, ref, sample=None):
    """Every routing decision, slot, row and count, f, P, loss and bias update against the oracle;
    y on every (or every sampled) token whose routing was not adopted. Returns the adopted count."""
    margin_ok = ref["margin"] > MARGIN
    assert (got["topk_idx"][margin_ok] == ref["oracle_idx"][margin_ok]).all(), \
        "routing differs on a token with a clear margin"
    assert (ref["margin"] > MARGIN).mean() > 0.95
    adopted = ref["adopted"]
    cap = ref["cap"]
    for key in ("slot", "dest_row", "expert_offsets", "routed_count", "kept_count"):
        assert (got[key] == cap[key]).all(), key
    rows = int(cap["expert_offsets"][-1])
    assert (got["src_token"][:rows] == cap["src_token"][:rows]).all()
    same = ~adopted
    assert np.allclose(got["topk_gate"][same & margin_ok], ref["topk_gate"][same & margin_ok], rtol=1e-5, atol=1e-7)
    toks = np.nonzero(same)[0] if sample is None else sample[same[sample]]
    assert len(toks) > 0
    y_got = got["y"][toks]
    y_exp = ref["y"][toks] if sample is None else ref["y"][np.searchsorted(sample, toks)]
    assert norm_err(y_got, y_exp) <= tol(cfg.dtype)
    st = ref["stats"]
    assert (got["f"] == st["f"].astype(np.float32)).all()
    assert np.allclose(got["P"], st["P"], rtol=TOL_STATS, atol=1e-9)
    assert np.allclose(got["aux"], st["aux"], rtol=TOL_STATS)
    if "rank_bias_new" in got:
        assert (got["rank_bias_new"] == st["bias"]).all()
    return int(adopted.sum())


@pytest.mark.parametrize("name,kw", [("tiny", {}), ("switch", dict(m=1024, d=256, d_ff=512)),
                                     ("lossfree", dict(m=1024, d=256, d_ff=352)),
                                     ("global", dict(m=2048, d=256, d_ff=512, seg_len=512)),
                                     # more 128-token tiles than SMs (the router finishes whole rows),
                                     # rows of 16 vectors in dispatch and combine, half-width GEMM2 tiles
                                     ("global", dict(m=19456, d=128, d_ff=256, seg_len=4864,
                                                     wr_std=1.0 / np.sqrt(128)))])
@pytest.mark.parametrize("residual", [False, True])
def test_layer_reduced(name, kw, residual):
    cfg = _scaled(name, **kw)
    inp = W.make_layer_inputs(cfg, seed=0, bias_std=0.05)
    got = _run_gpu(cfg, inp, residual=residual)
    ref = _reference(cfg, inp, got, residual=residual)
    adopted = _compare_layer(cfg, got, ref)
    print(f"{name} reduced: near-tie tokens adopted: {adopted}")


@pytest.mark.parametrize("name", ["tiny", "switch", "lossfree", "global"])
def test_layer_full_size(name):
    """Every workload at its full size. The global-batch layer (16 micro-batches x 4096 tokens) has
    all 65536 tokens routed by the oracle, capacity per micro-batch for all 16, and the whole
    batch's f, P and loss (and the micro-batch mean) compared."""
    cfg = W.CONFIGS[name]
    inp = W.make_layer_inputs(cfg, seed=0)
    got = _run_gpu(cfg, inp)
    sample = np.unique(np.random.default_rng(1).integers(0, cfg.m, 48))
    ref = _reference(cfg, inp, got, sample=sample)
    adopted = _compare_layer(cfg, got, ref, sample=sample)
    nseg = cfg.m // cfg.seg_len
    print(f"{name} full size: {nseg} segment(s), near-tie tokens adopted: {adopted}, "
          f"tokens with margin <= {MARGIN}: {int((ref['margin'] <= MARGIN).sum())}")
    if nseg > 1:
        # the identities that tie the global row to the segments, on the GPU's own numbers
        f = got["f"].astype(np.float64)
        assert abs(f[-1].sum() - 1.0) < 1e-5
        assert np.allclose(f[:-1].mean(0), f[-1], atol=1e-6)
        assert got["aux"][nseg] == pytest.approx(got["aux"][:nseg].astype(np.float64).mean(), rel=1e-5)


def test_balance_full_size_step_and_solve(golden):
    """Balanced assignment at 65536 x 256, k = 8: one STEP bit-exact against the oracle run here,
    and the whole SOLVE (32 beta updates at most, then the exact repair) bit-exact against the
    oracle's stored result (tests/golden/qb_solve_65536x256_k8.txt, written by the oracle alone):
    picks (SHA-256 of the [m, k] int32 array), beta bits and info."""
    cfg = W.QB_CONFIG
    g = golden("qb_solve_65536x256_k8.txt")
    s = W.make_qb_scores(cfg["m"], cfg["n"], seed=0, skew_std=cfg["skew_std"])
    k, n, m = cfg["k"], cfg["n"], cfg["m"]
    assert (int(g["m"][0]), int(g["n"][0]), int(g["k"][0]), int(g["max_iters"][0])) == (m, n, k, 32)
    sd = dev(s)
    i_ref, b_ref, _, _ = oracle.balance_assign(s, k, mode=oracle.QB_STEP)
    idx, beta, info = lb.moe_balance_assign(sd, k, mode=lb.MOE_QB_STEP)
    torch.cuda.synchronize()
    assert (host(idx) == i_ref).all() and (host(beta) == b_ref).all()
    idx, beta, info = lb.moe_balance_assign(sd, k, mode=lb.MOE_QB_SOLVE, max_iters=32)
    torch.cuda.synchronize()
    got = host(idx)
    assert hashlib.sha256(np.ascontiguousarray(got, dtype="<i4").tobytes()).hexdigest() == g["picks_sha256"][0]
    assert [f"{int(b):08x}" for b in host(beta).view(np.uint32)] == g["beta_bits"]
    assert host(info).tolist() == [int(v) for v in g["info"]]
    assert (np.bincount(got.ravel(), minlength=n) == m * k // n).all()
    assert oracle.is_optimal(s, got)
    plain = oracle.qb_row(s, k, np.zeros(n, np.float32))[1]
    vio_plain = oracle.balance_stats(None, plain, m, n, k, m)["vio"]
    print(f"qb full size: info={host(info).tolist()} MaxVio plain top-k {vio_plain[0]:.3f} -> 0")
