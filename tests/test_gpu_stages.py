"""Per-call parity of the CUDA library against the CPU oracle, on the same seeded inputs.

Integer outputs (selections, slots, rows, counts) and fp32 decisions are
bit-exact; floating-point values are within the stated tolerances. Sizes span
several tiles and a ragged tail; edge cases: empty experts, capacity 0 and
>= m, k = n - 1, ties, several segments.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from gpu_util import MARGIN, TOL_STATS, dev, host, norm_err, tol, torch_dtype

pytestmark = pytest.mark.gpu

lb = pytest.importorskip("load_balanced_dispatch_b200")


@pytest.fixture(scope="module", autouse=True)
def _built():
    from load_balanced_dispatch_b200 import build
    build.build()
    assert torch.cuda.is_available()
    yield
    lb.sync_status()


# ---------------------------------------------------------------- router
@pytest.mark.parametrize("m,n,k,renorm", [(1000, 8, 1, 0), (777, 64, 2, 1), (513, 128, 1, 0), (300, 200, 6, 0),
                                          (256, 256, 8, 1), (97, 16, 15, 0), (64, 256, 40, 1)])
def test_router_logits_in_softmax_bitexact(m, n, k, renorm):
    rng = np.random.default_rng(m + n)
    logits = rng.standard_normal((m, n)).astype(np.float32)
    logits[::7] = np.round(logits[::7] * 2) / 2  # exact ties on some rows
    p_ref, i_ref, g_ref, _ = oracle.router(None, None, m, 0, n, k, renorm=renorm, logits_in=logits)
    idx, gate, probs = lb.moe_router_topk(None, None, n, k, lb.MOE_SOFTMAX, renorm, logits_in=dev(logits))
    torch.cuda.synchronize()
    assert (host(idx) == i_ref).all()
    assert np.allclose(host(gate), g_ref, rtol=1e-5, atol=1e-7)
    assert np.allclose(host(probs), p_ref, rtol=1e-5, atol=1e-8)


@pytest.mark.parametrize("m,n,k,bias", [(1000, 64, 6, True), (333, 32, 4, False), (128, 256, 8, True)])
def test_router_logits_in_sigmoid(m, n, k, bias):
    rng = np.random.default_rng(n + k)
    logits = rng.standard_normal((m, n)).astype(np.float32)
    b = rng.uniform(-0.05, 0.05, n).astype(np.float32) if bias else None
    p_ref, i_ref, g_ref, margin = oracle.router(None, None, m, 0, n, k, fn=oracle.SIGMOID, rank_bias=b,
                                                logits_in=logits)
    idx, gate, probs = lb.moe_router_topk(None, None, n, k, lb.MOE_SIGMOID, 0, rank_bias=None if b is None else dev(b),
                                          logits_in=dev(logits))
    torch.cuda.synchronize()
    ok = margin > MARGIN
    assert ok.mean() > 0.9
    assert (host(idx)[ok] == i_ref[ok]).all()
    assert np.allclose(host(gate)[ok], g_ref[ok], rtol=1e-6)
    assert np.allclose(host(probs), p_ref, rtol=1e-6)


@pytest.mark.parametrize("dtype,m,d,n,k,fn,renorm,bias", [
    ("fp32", 1000, 64, 8, 1, 0, 0, False), ("bf16", 517, 768, 128, 1, 0, 0, False),
    ("bf16", 300, 200, 64, 6, 0, 1, False), ("fp32", 129, 36, 256, 8, 0, 0, False),
    ("bf16", 700, 2048, 64, 6, 1, 0, True), ("bf16", 259, 128, 256, 8, 0, 1, False),
    ("bf16", 1000, 96, 40, 3, 1, 0, False), ("bf16", 131, 4096, 64, 2, 0, 1, False),
    ("bf16", 64, 64, 16, 12, 0, 0, False), ("bf16", 600, 256, 100, 8, 0, 1, False),
    ("bf16", 300, 128, 96, 5, 1, 0, True), ("bf16", 257, 192, 65, 2, 0, 0, False),
    ("bf16", 200, 64, 128, 4, 0, 0, True)])
def test_router_projection(dtype, m, d, n, k, fn, renorm, bias):
    rng = np.random.default_rng(d + n)
    x = rng.standard_normal((m, d)).astype(np.float32)
    if dtype == "bf16":
        x = W.round_to_bf16(x)
    w = (rng.standard_normal((d, n)) / np.sqrt(d)).astype(np.float32)
    b = rng.uniform(-0.05, 0.05, n).astype(np.float32) if bias else None
    p_ref, i_ref, g_ref, margin = oracle.router(x, w, m, d, n, k, fn, renorm, b)
    idx, gate, probs = lb.moe_router_topk(dev(x, torch_dtype(dtype)), dev(w), n, k, fn, renorm,
                                          rank_bias=None if b is None else dev(b))
    torch.cuda.synchronize()
    ok = margin > MARGIN
    assert ok.mean() > 0.97
    assert (host(idx)[ok] == i_ref[ok]).all()
    assert np.allclose(host(gate)[ok], g_ref[ok], rtol=1e-5)
    assert np.allclose(host(probs), p_ref, rtol=1e-5, atol=1e-9)


@pytest.mark.parametrize("m,d,n,k,fn,renorm,bias", [(517, 768, 128, 1, 0, 0, False), (300, 200, 64, 6, 0, 1, False),
                                                      (700, 512, 64, 6, 1, 0, True), (64, 64, 16, 12, 0, 0, False),
                                                      (400, 128, 100, 8, 1, 0, True)])
def test_router_projection_without_scores(m, d, n, k, fn, renorm, bias):
    # no probs_out: the tensor-core path keeps whole rows per CTA and a warp finishes each row in
    # the kernel; nothing but the picks and gates is stored
    rng = np.random.default_rng(d * 3 + n)
    x = W.round_to_bf16(rng.standard_normal((m, d)).astype(np.float32))
    w = (rng.standard_normal((d, n)) / np.sqrt(d)).astype(np.float32)
    b = rng.uniform(-0.05, 0.05, n).astype(np.float32) if bias else None
    _, i_ref, g_ref, margin = oracle.router(x, w, m, d, n, k, fn, renorm, b)
    idx, gate, probs = lb.moe_router_topk(dev(x, torch.bfloat16), dev(w), n, k, fn, renorm,
                                          rank_bias=None if b is None else dev(b), want_probs=False)
    torch.cuda.synchronize()
    assert probs is None
    ok = margin > MARGIN
    assert ok.mean() > 0.97
    assert (host(idx)[ok] == i_ref[ok]).all()
    assert np.allclose(host(gate)[ok], g_ref[ok], rtol=1e-5)


@pytest.mark.parametrize("m,d,n,k,fn,renorm,bias", [(40000, 256, 64, 2, 0, 1, False), (20000, 512, 128, 1, 0, 0, False),
                                                      (19100, 192, 96, 6, 1, 0, True), (30001, 128, 32, 4, 0, 0, False),
                                                      # the per-thread row finish with sigmoid scores and a
                                                      # ranking bias, and with k = 8 renormalised gates
                                                      (25000, 128, 64, 6, 1, 0, True), (20000, 64, 64, 8, 0, 1, False)])
def test_router_many_blocks_and_prepared_split(m, d, n, k, fn, renorm, bias):
    # more 128-token blocks than two waves of CTAs (ragged last block); the call with w_r = None
    # on a workspace from moe_router_prepare gives the same bits as the call that splits W_r itself
    rng = np.random.default_rng(m + d)
    x = W.round_to_bf16(rng.standard_normal((m, d)).astype(np.float32))
    w = (rng.standard_normal((d, n)) / np.sqrt(d)).astype(np.float32)
    b = rng.uniform(-0.05, 0.05, n).astype(np.float32) if bias else None
    p_ref, i_ref, g_ref, margin = oracle.router(x, w, m, d, n, k, fn, renorm, b)
    xd, wd, bd = dev(x, torch.bfloat16), dev(w), None if b is None else dev(b)
    idx, gate, probs = lb.moe_router_topk(xd, wd, n, k, fn, renorm, rank_bias=bd)
    ws = lb.moe_router_prepare(wd, k, torch.bfloat16)
    idx2, gate2, probs2 = lb.moe_router_topk(xd, None, n, k, fn, renorm, rank_bias=bd, workspace=ws)
    torch.cuda.synchronize()
    lb.sync_status()
    assert torch.equal(idx, idx2) and torch.equal(gate, gate2) and torch.equal(probs, probs2)
    ok = margin > MARGIN
    assert ok.mean() > 0.97
    assert (host(idx)[ok] == i_ref[ok]).all()
    assert np.allclose(host(gate)[ok], g_ref[ok], rtol=1e-5)
    assert np.allclose(host(probs), p_ref, rtol=1e-5, atol=1e-9)


# ---------------------------------------------------------------- capacity
@pytest.mark.parametrize("m,n,k,cap,seg", [(1000, 8, 1, 160, 1000), (8192, 128, 1, 80, 8192), (4096, 64, 2, 256, 512),
                                           (777, 16, 3, 40, 777), (1536, 256, 8, 30, 256), (600, 5, 2, 0, 300),
                                           (300, 4, 2, 10 ** 6, 100), (64, 64, 63, 1, 64),
                                           # a large one-segment shape (many chunks in one segment)
                                           (16384, 64, 6, 16384 * 6, 16384),
                                           # more (segment, expert) pairs than the pair scan holds
                                           (32768, 64, 2, 40, 256)])
def test_capacity_bitexact(m, n, k, cap, seg):
    idx = W.make_topk_idx(m, n, k, seed=m * 7 + n)
    ref = oracle.capacity(idx, m, k, n, cap, seg)
    out = lb.moe_capacity_slots(dev(idx), n, cap, seg)
    torch.cuda.synchronize()
    rows = int(ref["expert_offsets"][-1])
    for key in ("slot", "dest_row", "expert_offsets", "routed_count", "kept_count"):
        assert (host(out[key]) == ref[key]).all(), key
    assert (host(out["src_token"])[:rows] == ref["src_token"][:rows]).all()


def test_capacity_golden_example(golden):
    g = golden("capacity_example.txt")
    routed = [int(v) for v in g["routed"]]
    route = np.concatenate([np.full(c, e) for e, c in enumerate(routed)])
    route = np.random.default_rng(0).permutation(route).astype(np.int32)[:, None]
    for cf in ("1.0", "1.25"):
        out = lb.moe_capacity_slots(dev(route), 4, int(g["capacity_" + cf][0]))
        assert host(out["kept_count"])[0].tolist() == [int(v) for v in g["kept_" + cf]]
        assert int((host(out["slot"]) < 0).sum()) == int(g["dropped_" + cf][0])


def test_capacity_rejects_bad_expert_ids():
    idx = np.array([[0], [9], [1]], np.int32)
    lb.moe_capacity_slots(dev(idx), 4, 8)
    with pytest.raises(lb.MoEError):
        lb.sync_status()


# ---------------------------------------------------------------- dispatch / combine
@pytest.mark.parametrize("dtype,m,d,n,k,cap", [("bf16", 1000, 768, 16, 2, 100), ("fp32", 513, 64, 8, 1, 80),
                                               ("bf16", 300, 4096, 64, 2, 0),
                                               # rows of fewer than 32 16-byte vectors with several picks
                                               ("bf16", 777, 128, 64, 2, 40), ("bf16", 500, 64, 8, 3, 150),
                                               ("bf16", 400, 8, 4, 3, 1000), ("fp32", 333, 20, 16, 5, 90)])
def test_dispatch_combine(dtype, m, d, n, k, cap):
    rng = np.random.default_rng(d)
    x = rng.standard_normal((m, d)).astype(np.float32)
    if dtype == "bf16":
        x = W.round_to_bf16(x)
    idx = W.make_topk_idx(m, n, k, seed=1)
    ref = oracle.capacity(idx, m, k, n, cap, m)
    rows = int(ref["expert_offsets"][-1])
    td = torch_dtype(dtype)
    xd = dev(x, td)
    out = lb.moe_capacity_slots(dev(idx), n, cap)
    xbuf = lb.moe_dispatch(xd, out["src_token"], out["expert_offsets"], n, m * k)
    torch.cuda.synchronize()
    assert (host(xbuf)[:rows] == oracle.dispatch(x, ref["src_token"], rows)).all()
    # token-major dispatch: the same rows, each token read once
    xbuf_t = lb.moe_dispatch_tokens(xd, out["dest_row"], m * k)
    torch.cuda.synchronize()
    assert (host(xbuf_t)[:rows] == oracle.dispatch(x, ref["src_token"], rows)).all()
    ybuf = rng.standard_normal((m * k, d)).astype(np.float32)
    if dtype == "bf16":
        ybuf = W.round_to_bf16(ybuf)
    gate = rng.random((m, k)).astype(np.float32)
    for residual in (None, xd):
        y = lb.moe_combine(dev(ybuf, td), out["dest_row"], dev(gate), residual=residual)
        torch.cuda.synchronize()
        y_ref = oracle.combine(ybuf[:max(rows, 1)] if rows else np.zeros((1, d)), ref["dest_row"], gate,
                               None if residual is None else x, m, k, d, gate_bf16=int(dtype == "bf16"))
        assert norm_err(host(y), y_ref) <= (2 ** -8 if dtype == "bf16" else 1e-6)


# ---------------------------------------------------------------- expert FFN
@pytest.mark.parametrize("dtype,rows_per,d,d_ff", [("fp32", [100, 0, 37, 256, 1], 64, 256),
                                                   ("bf16", [64, 80, 0, 3, 129, 77], 768, 3072),
                                                   ("bf16", [130, 1, 0, 256], 2048, 1408),
                                                   ("bf16", [0, 300], 256, 512),
                                                   # 512-column tiles (d and d_ff multiples of 512)
                                                   ("bf16", [300, 0, 17, 513, 256], 512, 1024)])
def test_expert_ffn(dtype, rows_per, d, d_ff):
    n = len(rows_per)
    rng = np.random.default_rng(d + d_ff)
    off = np.concatenate([[0], np.cumsum(rows_per)]).astype(np.int32)
    rows = int(off[-1])
    max_rows = rows + 19
    st = (lambda a: W.round_to_bf16(a)) if dtype == "bf16" else (lambda a: a.astype(np.float32))
    xbuf = st(rng.standard_normal((max_rows, d)).astype(np.float32))
    w1 = st((rng.standard_normal((n, d_ff, d)) / np.sqrt(d)).astype(np.float32))
    b1 = st((0.1 * rng.standard_normal((n, d_ff))).astype(np.float32))
    w2 = st((rng.standard_normal((n, d, d_ff)) / np.sqrt(d_ff)).astype(np.float32))
    b2 = st((0.1 * rng.standard_normal((n, d))).astype(np.float32))
    td = torch_dtype(dtype)
    ybuf = lb.moe_expert_ffn(dev(xbuf, td), dev(w1, td), dev(b1, td), dev(w2, td), dev(b2, td), dev(off))
    torch.cuda.synchronize()
    ref = oracle.expert_ffn(xbuf[:rows], off, w1, b1, w2, b2)
    assert norm_err(host(ybuf)[:rows], ref) <= tol(dtype)


@pytest.mark.parametrize("m,n,d,d_ff,cap", [(2048, 16, 768, 3072, 150), (1000, 8, 256, 512, 100),
                                            (513, 5, 2048, 1408, 1000), (300, 4, 256, 256, 0)])
def test_expert_ffn_combine_matches_two_calls(m, n, d, d_ff, cap):
    # k = 1: the FFN's second GEMM writes the gated combine straight into y. Bit for bit the
    # result of moe_expert_ffn followed by moe_combine, with and without the residual; capacity
    # 0 drops every token (no FFN rows at all)
    rng = np.random.default_rng(m + d)
    x = W.round_to_bf16(rng.standard_normal((m, d)).astype(np.float32))
    idx = W.make_topk_idx(m, n, 1, seed=4, skew=1.5)
    gate = rng.random((m, 1)).astype(np.float32)
    w1 = W.round_to_bf16((rng.standard_normal((n, d_ff, d)) / np.sqrt(d)).astype(np.float32))
    b1 = W.round_to_bf16((0.1 * rng.standard_normal((n, d_ff))).astype(np.float32))
    w2 = W.round_to_bf16((rng.standard_normal((n, d, d_ff)) / np.sqrt(d_ff)).astype(np.float32))
    b2 = W.round_to_bf16((0.1 * rng.standard_normal((n, d))).astype(np.float32))
    bf = torch.bfloat16
    xd = dev(x, bf)
    out = lb.moe_capacity_slots(dev(idx), n, cap)
    xbuf = lb.moe_dispatch(xd, out["src_token"], out["expert_offsets"], n, m)
    wd = [dev(a, bf) for a in (w1, b1, w2, b2)]
    ybuf = lb.moe_expert_ffn(xbuf, *wd, out["expert_offsets"])
    for residual in (None, xd):
        y2 = lb.moe_combine(ybuf, out["dest_row"], dev(gate), residual=residual)
        y1 = lb.moe_expert_ffn_combine(xbuf, *wd, out["expert_offsets"], out["src_token"], out["dest_row"],
                                       dev(gate), residual=residual)
        torch.cuda.synchronize()
        lb.sync_status()
        assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


@pytest.mark.parametrize("m,n,k,d,d_ff,cap", [(2000, 16, 2, 768, 3072, 300), (1000, 64, 6, 2048, 1408, 10 ** 6),
                                              (777, 8, 3, 256, 512, 40), (512, 4, 1, 128, 256, 0),
                                              (1500, 8, 2, 1024, 512, 300)])
def test_expert_ffn_gather_matches_dispatch(m, n, k, d, d_ff, cap):
    # the FFN loading its rows from x by src_token gives bit for bit the FFN of the dispatched
    # copy, including dropped picks, ragged experts and a capacity that empties every expert
    rng = np.random.default_rng(m * 3 + d)
    x = W.round_to_bf16(rng.standard_normal((m, d)).astype(np.float32))
    idx = W.make_topk_idx(m, n, k, seed=6, skew=1.3)
    bf = torch.bfloat16
    wd = [dev(W.round_to_bf16(a), bf) for a in (
        (rng.standard_normal((n, d_ff, d)) / np.sqrt(d)).astype(np.float32),
        (0.1 * rng.standard_normal((n, d_ff))).astype(np.float32),
        (rng.standard_normal((n, d, d_ff)) / np.sqrt(d_ff)).astype(np.float32),
        (0.1 * rng.standard_normal((n, d))).astype(np.float32))]
    xd = dev(x, bf)
    out = lb.moe_capacity_slots(dev(idx), n, cap)
    xbuf = lb.moe_dispatch(xd, out["src_token"], out["expert_offsets"], n, m * k)
    y_ref = lb.moe_expert_ffn(xbuf, *wd, out["expert_offsets"])
    y = lb.moe_expert_ffn_gather(xd, *wd, out["expert_offsets"], out["src_token"], max_rows=m * k)
    torch.cuda.synchronize()
    lb.sync_status()
    rows = int(host(out["expert_offsets"])[-1])
    assert torch.equal(y[:rows].view(torch.int16), y_ref[:rows].view(torch.int16))


# ---------------------------------------------------------------- statistics
@pytest.mark.parametrize("m,n,k,seg", [(8192, 128, 1, 8192), (65536, 64, 2, 4096), (1000, 8, 1, 250),
                                       (777, 256, 8, 777)])
def test_balance_stats(m, n, k, seg):
    rng = np.random.default_rng(n)
    p = rng.random((m, n)).astype(np.float32)
    p /= p.sum(1, keepdims=True)
    idx = W.make_topk_idx(m, n, k, seed=3)
    b = rng.uniform(-0.05, 0.05, n).astype(np.float32)
    ref = oracle.balance_stats(p, idx, m, n, k, seg, 1e-2, bias=b, gamma=1e-3)
    bd = dev(b)
    out = lb.moe_balance_stats(dev(p), dev(idx), n, seg, 1e-2, bias_inout=bd, gamma=1e-3)
    torch.cuda.synchronize()
    assert (host(out["f"]) == ref["f"].astype(np.float32)).all()
    assert np.allclose(host(out["P"]), ref["P"], rtol=TOL_STATS, atol=0)
    assert np.allclose(host(out["aux"]), ref["aux"], rtol=TOL_STATS, atol=0)
    assert np.allclose(host(out["vio"]), ref["vio"], rtol=1e-6, atol=1e-7)
    assert (host(bd) == ref["bias"]).all()


def test_balance_stats_golden_identity(golden):
    g = golden("aux_balanced.txt")
    for n in (int(v) for v in g["experts"]):
        m = 4 * n
        out = lb.moe_balance_stats(dev(W.make_uniform_probs(m, n)), dev(W.make_round_robin_idx(m, n, 2)), n, m // 2,
                                   float(g["alpha"][0]))
        torch.cuda.synchronize()
        aux = host(out["aux"])
        assert (aux[:-1] == np.float32(g["expected_aux"][0])).all()
        # the hybrid loss: the global loss + 0.01 x the micro-batch loss = 1.01 alpha at balance
        assert aux[-1] == pytest.approx(1.01 * float(g["alpha"][0]), rel=TOL_STATS)
        assert (host(out["vio"]) == 0).all()


@pytest.mark.parametrize("m,n,k,ranks,with_probs", [(8192, 128, 1, 2, True), (6000, 64, 6, 3, True),
                                                   (4096, 24, 3, 4, False)])
def test_balance_global_across_ranks(m, n, k, ranks, with_probs):
    # one batch split over `ranks` pretend ranks: per-rank totals, summed, then the global
    # statistics = the oracle's whole-batch row on the unsplit batch
    rng = np.random.default_rng(m + n)
    p = rng.random((m, n)).astype(np.float32)
    p /= p.sum(1, keepdims=True)
    idx = W.make_topk_idx(m, n, k, seed=9, skew=1.2)
    b = rng.uniform(-0.05, 0.05, n).astype(np.float32)
    ref = oracle.balance_stats(p if with_probs else None, idx, m, n, k, m, 1e-2, bias=b, gamma=1e-3)
    total = torch.zeros((2, n), dtype=torch.float64, device="cuda")
    cuts = [r * m // ranks for r in range(ranks + 1)]
    for r in range(ranks):
        lo, hi = cuts[r], cuts[r + 1]
        t = lb.moe_balance_totals(dev(p[lo:hi]) if with_probs else None, dev(idx[lo:hi]), n)
        total += t
    bd = dev(b)
    out = lb.moe_balance_global(total, m, k, has_probs=with_probs, alpha=1e-2, bias_inout=bd, gamma=1e-3)
    torch.cuda.synchronize()
    lb.sync_status()
    assert (host(total)[0] == np.bincount(idx.ravel(), minlength=n)).all()
    assert (host(out["f"]) == ref["f"][-1].astype(np.float32)).all()
    if with_probs:
        assert np.allclose(host(out["P"]), ref["P"][-1], rtol=TOL_STATS, atol=0)
        assert np.allclose(host(out["aux"])[0], ref["aux"][-2], rtol=TOL_STATS, atol=0)  # the global-batch loss
    assert np.allclose(host(out["vio"]), ref["vio"], rtol=1e-6, atol=1e-7)
    assert (host(bd) == ref["bias"]).all()


# ---------------------------------------------------------------- router gradient of the balance loss
@pytest.mark.parametrize("m,n,k,seg,fn,w_micro,w_global", [(4096, 64, 2, 512, 0, 0.01, 1.0), (2000, 8, 1, 250, 0, 1.0, 0.0),
                                                          (3000, 256, 8, 3000, 0, 0.0, 1.0),
                                                          (1024, 100, 6, 128, 1, 0.01, 1.0)])
def test_balance_loss_grad(m, n, k, seg, fn, w_micro, w_global):
    rng = np.random.default_rng(m + n)
    logits = rng.standard_normal((m, n)).astype(np.float32)
    idx, _, probs = lb.moe_router_topk(None, None, n, k, fn, 0, logits_in=dev(logits))
    st = lb.moe_balance_stats(probs, idx, n, seg, 1e-2)
    g = lb.moe_balance_loss_grad(probs, st["f"], seg, fn, 1e-2, w_micro, w_global)
    torch.cuda.synchronize()
    ref = oracle.balance_loss_grad(host(probs), host(idx), m, n, k, seg, fn, 1e-2, w_micro, w_global)
    assert norm_err(host(g), ref) <= TOL_STATS


# ---------------------------------------------------------------- mini-batch beta
@pytest.mark.parametrize("m,n,k,seg,rule", [(65536, 256, 8, 4096, 0), (65536, 256, 8, 32768, 0),
                                            (6144, 64, 6, 1024, 1), (4000, 16, 4, 500, 2), (2048, 32, 2, 2048, 0),
                                            (1024, 8, 1, 8, 0), (12000, 24, 3, 24000 // 8, 0)])
def test_balance_step_minibatch_bitexact(m, n, k, seg, rule):
    # picks, beta and info bit-exact against the oracle: mini-batches kept in shared memory
    # (seg <= 16384), the full radix path (32768), many tiny mini-batches (seg = 8), one (seg = m)
    s = W.make_qb_scores(m, n, seed=m + n + seg, skew_std=1.0)
    b0 = np.random.default_rng(seg).uniform(-0.5, 0.5, n).astype(np.float32)
    i_ref, b_ref, f_ref = oracle.balance_step_minibatch(s, k, b0, seg, rule=rule)
    beta = dev(b0)
    idx, beta, info = lb.moe_balance_step_minibatch(dev(s), k, beta, seg, rule=rule)
    torch.cuda.synchronize()
    lb.sync_status()
    assert (host(idx) == i_ref).all()
    assert (host(beta) == b_ref).all()
    assert (host(info) == f_ref).all()


def test_balance_step_minibatch_ties():
    # coarse scores: many equal keys inside each mini-batch's column
    m, n, k, seg = 8192, 32, 4, 1024
    s = (np.round(W.make_qb_scores(m, n, seed=3) * 4) / 4).astype(np.float32)
    i_ref, b_ref, f_ref = oracle.balance_step_minibatch(s, k, np.zeros(n, np.float32), seg)
    idx, beta, info = lb.moe_balance_step_minibatch(dev(s), k, torch.zeros(n, device="cuda"), seg)
    torch.cuda.synchronize()
    assert (host(idx) == i_ref).all() and (host(beta) == b_ref).all() and (host(info) == f_ref).all()


# ---------------------------------------------------------------- balanced assignment
@pytest.mark.parametrize("m,n,k,rule", [(2048, 32, 4, 0), (4096, 64, 6, 1), (1000, 8, 2, 0), (768, 256, 8, 0),
                                        (2560, 16, 15, 0)])
def test_balance_step_bitexact(m, n, k, rule):
    s = W.make_qb_scores(m, n, seed=m + k)
    beta0 = (0.3 * np.random.default_rng(5).standard_normal(n)).astype(np.float32)
    i_ref, b_ref, info_ref, _ = oracle.balance_assign(s, k, beta=beta0, mode=oracle.QB_STEP, rule=rule)
    idx, beta, info = lb.moe_balance_assign(dev(s), k, beta=dev(beta0), mode=lb.MOE_QB_STEP, rule=rule)
    torch.cuda.synchronize()
    assert (host(idx) == i_ref).all()
    assert (host(beta) == b_ref).all()
    assert host(info)[2] == info_ref[2] and host(info)[3] == info_ref[3]


@pytest.mark.parametrize("m,n,k", [(8192, 64, 4), (65536, 256, 8), (3000, 24, 5), (1002, 6, 3)])
def test_balance_step_chain(m, n, k):
    # each STEP starts from the previous one's beta, so the column pass finds the new thresholds
    # inside its window around the old ones (the first step, from beta = 0, takes the full select)
    s = W.make_qb_scores(m, n, seed=11)
    b = np.zeros(n, dtype=np.float32)
    for _ in range(3):
        i_ref, b_ref, info_ref, _ = oracle.balance_assign(s, k, beta=b, mode=oracle.QB_STEP)
        idx, beta, info = lb.moe_balance_assign(dev(s), k, beta=dev(b), mode=lb.MOE_QB_STEP)
        torch.cuda.synchronize()
        assert (host(idx) == i_ref).all()
        assert (host(beta) == b_ref).all()
        assert host(info)[2] == info_ref[2] and host(info)[3] == info_ref[3]
        b = b_ref


@pytest.mark.parametrize("m,n,k", [(65536, 4, 1), (32768, 8, 2)])
def test_balance_step_heavy_ties(m, n, k):
    # integer-grid scores: u = s - alpha repeats a few values thousands of times per column (signed
    # zeros among them); at (65536, 4, 1) the selected key alone outnumbers the shared-memory
    # candidate list, so the column pass streams its last digits from global memory
    s = np.round(W.make_qb_scores(m, n, seed=7, skew_std=0.0)).astype(np.float32)
    b = np.zeros(n, dtype=np.float32)
    for _ in range(2):
        i_ref, b_ref, info_ref, _ = oracle.balance_assign(s, k, beta=b, mode=oracle.QB_STEP)
        idx, beta, info = lb.moe_balance_assign(dev(s), k, beta=dev(b), mode=lb.MOE_QB_STEP)
        torch.cuda.synchronize()
        assert (host(idx) == i_ref).all()
        assert (host(beta) == b_ref).all()
        b = b_ref


@pytest.mark.parametrize("m,n,k,shift", [(4096, 32, 4, 0.0), (2048, 16, 2, -1.0), (65536, 256, 8, 0.0),
                                         (1002, 6, 3, 2.0)])
def test_balance_bip_steps_bitexact(m, n, k, shift):
    # BIP thresholds (the (k+1)-th / (C+1)-th values clipped at zero), three chained STEPs
    s = W.make_qb_scores(m, n, seed=m + n) + np.float32(shift)
    b = np.zeros(n, dtype=np.float32)
    for _ in range(3):
        i_ref, b_ref, info_ref, _ = oracle.balance_assign(s, k, beta=b, mode=oracle.QB_STEP, rule=oracle.QB_BIP)
        idx, beta, info = lb.moe_balance_assign(dev(s), k, beta=dev(b), mode=lb.MOE_QB_STEP, rule=lb.MOE_QB_BIP)
        torch.cuda.synchronize()
        assert (host(idx) == i_ref).all()
        assert (host(beta) == b_ref).all()
        assert (host(info) == info_ref).all()
        b = b_ref


def test_balance_bip_solve_bitexact():
    s = W.make_qb_scores(2048, 16, seed=9)
    i_ref, b_ref, info_ref, rc = oracle.balance_assign(s, 2, mode=oracle.QB_SOLVE, rule=oracle.QB_BIP, max_iters=12)
    assert rc == oracle.OK
    idx, beta, info = lb.moe_balance_assign(dev(s), 2, mode=lb.MOE_QB_SOLVE, rule=lb.MOE_QB_BIP, max_iters=12)
    torch.cuda.synchronize()
    assert (host(info) == info_ref).all()
    assert (host(beta) == b_ref).all()
    assert (host(idx) == i_ref).all()


@pytest.mark.parametrize("m,n,k,gamma,rule", [(4096, 32, 4, 0.05, 0), (65536, 256, 8, 0.01, 0), (1002, 6, 3, 0.1, 1),
                                              (2048, 16, 2, 0.02, 2)])
def test_balance_sign_steps_bitexact(m, n, k, gamma, rule):
    # SignSGD on beta: five chained steps, picks, beta and info identical to the oracle
    s = W.make_qb_scores(m, n, seed=m * 5 + n)
    b = np.zeros(n, dtype=np.float32)
    for _ in range(5):
        i_ref, b_ref, info_ref = oracle.qb_sign_step(s, k, b, gamma, rule=rule)
        bd = dev(b)
        idx, _, info = lb.moe_balance_sign_step(dev(s), k, bd, gamma, rule=rule)
        torch.cuda.synchronize()
        assert (host(idx) == i_ref).all()
        assert (host(bd) == b_ref).all()
        assert (host(info) == info_ref).all()
        b = b_ref


@pytest.mark.parametrize("m,n,k,iters,rule", [(2048, 32, 4, 8, 0), (2048, 32, 4, 0, 0), (1024, 16, 2, 3, 1),
                                              (4096, 64, 8, 20, 0), (512, 8, 1, 2, 0), (4096, 64, 8, 40, 0),
                                              (2048, 16, 3, 33, 1)])
def test_balance_solve_bitexact(m, n, k, iters, rule):
    s = W.make_qb_scores(m, n, seed=m * 3 + n)
    i_ref, b_ref, info_ref, rc = oracle.balance_assign(s, k, mode=oracle.QB_SOLVE, rule=rule, max_iters=iters)
    assert rc == oracle.OK
    idx, beta, info = lb.moe_balance_assign(dev(s), k, mode=lb.MOE_QB_SOLVE, rule=rule, max_iters=iters)
    torch.cuda.synchronize()
    assert (host(info) == info_ref).all()
    assert (host(beta) == b_ref).all()
    assert (host(idx) == i_ref).all()
    assert (np.bincount(host(idx).ravel(), minlength=n) == m * k // n).all()


@pytest.mark.parametrize("m,n,k", [(4096, 64, 4), (1000, 32, 8)])
def test_balance_misaligned_scores(m, n, k):
    # s starting 4 bytes past a 16-byte boundary: the row pass loads its tiles without bulk copies
    # and the window sweep reads scalars; two chained STEPs and a SOLVE stay bit-exact
    s = W.make_qb_scores(m, n, seed=m + 5)
    buf = torch.empty((m * n + 1,), dtype=torch.float32, device="cuda")
    sd = buf[1:].view(m, n)
    sd.copy_(torch.from_numpy(s))
    assert sd.data_ptr() % 16 == 4
    b = np.zeros(n, dtype=np.float32)
    for _ in range(2):
        i_ref, b_ref, info_ref, _ = oracle.balance_assign(s, k, beta=b, mode=oracle.QB_STEP)
        idx, beta, info = lb.moe_balance_assign(sd, k, beta=dev(b), mode=lb.MOE_QB_STEP)
        torch.cuda.synchronize()
        assert (host(idx) == i_ref).all()
        assert (host(beta) == b_ref).all()
        b = b_ref
    i_ref, b_ref, info_ref, rc = oracle.balance_assign(s, k, mode=oracle.QB_SOLVE, max_iters=12)
    idx, beta, info = lb.moe_balance_assign(sd, k, mode=lb.MOE_QB_SOLVE, max_iters=12)
    torch.cuda.synchronize()
    assert (host(info) == info_ref).all()
    assert (host(beta) == b_ref).all()
    assert (host(idx) == i_ref).all()


@pytest.mark.parametrize("m,n,k,kind", [(8192, 256, 8, "tied_rows"), (4040, 101, 5, "odd_n"),
                                        (4096, 256, 40, "large_k"), (1024, 64, 40, "large_k"),
                                        (6048, 96, 23, "k_at_groups"), (2016, 32, 31, "k_at_groups")])
def test_balance_row_pass_forms(m, n, k, kind):
    # the row pass's two forms: the thread-per-row selection (k + 1 <= the number of column groups)
    # with its warp-per-row fallback for rows whose listed elements overflow (every 7th row constant,
    # every 5th on a coarse grid: many equal values), rows of n not a multiple of 4 (plain loads),
    # and the warp-per-row kernel when k + 1 exceeds the groups; chained STEPs and a SOLVE
    s = W.make_qb_scores(m, n, seed=m + n + k)
    if kind == "tied_rows":
        s[3::7] = np.float32(0.5)
        s[1::5] = np.round(s[1::5] * 2) / 2
    b = np.zeros(n, dtype=np.float32)
    for _ in range(3):
        i_ref, b_ref, info_ref, _ = oracle.balance_assign(s, k, beta=b, mode=oracle.QB_STEP)
        idx, beta, info = lb.moe_balance_assign(dev(s), k, beta=dev(b), mode=lb.MOE_QB_STEP)
        torch.cuda.synchronize()
        assert (host(idx) == i_ref).all()
        assert (host(beta) == b_ref).all()
        assert (host(info) == info_ref).all()
        b = b_ref
    if kind == "tied_rows":
        return  # the SOLVE of heavily tied scores: test_balance_solve_zero_cost_cycles
    i_ref, b_ref, info_ref, rc = oracle.balance_assign(s, k, mode=oracle.QB_SOLVE, max_iters=10)
    assert rc == oracle.OK
    idx, beta, info = lb.moe_balance_assign(dev(s), k, mode=lb.MOE_QB_SOLVE, max_iters=10)
    torch.cuda.synchronize()
    assert (host(info) == info_ref).all()
    assert (host(beta) == b_ref).all()
    assert (host(idx) == i_ref).all()


@pytest.mark.parametrize("m,n,k,seed", [(1024, 16, 2, 0), (2048, 32, 4, 1), (1536, 64, 8, 2)])
def test_balance_solve_zero_cost_cycles(m, n, k, seed):
    # half-integer scores with every third row constant: the exact finish runs thousands of moves on
    # an expert graph with zero-cost cycles (several tight arcs into an expert); the predecessor
    # settled in the earlier round keeps every path acyclic. Picks, beta and info bit-exact.
    s = (np.round(np.random.default_rng(seed).standard_normal((m, n)) * 2) / 2).astype(np.float32)
    s[::3] = np.float32(0.5)
    i_ref, b_ref, info_ref, rc = oracle.balance_assign(s, k, mode=oracle.QB_SOLVE, max_iters=6)
    assert rc == oracle.OK and info_ref[1] > 0
    idx, beta, info = lb.moe_balance_assign(dev(s), k, mode=lb.MOE_QB_SOLVE, max_iters=6)
    torch.cuda.synchronize()
    assert (host(info) == info_ref).all()
    assert (host(beta) == b_ref).all()
    assert (host(idx) == i_ref).all()


@pytest.mark.parametrize("m,n,k,seed", [(1024, 8, 2, 0), (2048, 16, 2, 2), (4096, 32, 4, 1), (512, 4, 1, 0)])
def test_balance_solve_converges_inside_a_batch(m, n, k, seed):
    # mild skew: QB alone reaches exact balance after 6..45 beta updates (no repair), so the
    # early exit happens inside, or at the edge of, a batch of enqueued iterations
    s = W.make_qb_scores(m, n, seed=seed, skew_std=0.5)
    i_ref, b_ref, info_ref, rc = oracle.balance_assign(s, k, mode=oracle.QB_SOLVE, max_iters=60)
    assert rc == oracle.OK and info_ref[1] == 0 and info_ref[0] < 60
    idx, beta, info = lb.moe_balance_assign(dev(s), k, mode=lb.MOE_QB_SOLVE, max_iters=60)
    torch.cuda.synchronize()
    assert (host(info) == info_ref).all()
    assert (host(beta) == b_ref).all()
    assert (host(idx) == i_ref).all()


# ---------------------------------------------------------------- bounded waits
def test_bounded_wait_gives_up_and_the_context_stays_usable():
    # a wait (the FFN's counter wait) on a flag that nothing sets runs out after its limit,
    # reports the pipeline timeout through the device error word, and the context keeps working
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    lb.moe_selftest_wait(flag, 20_000_000)  # about 10 ms of SM clock cycles
    with pytest.raises(lb.MoEError, match="timed out"):
        lb.sync_status()
    lb.sync_status()  # reading the word cleared it
    flag.fill_(1)
    lb.moe_selftest_wait(flag, 20_000_000)  # the flag is set: no wait, no error
    lb.sync_status()
    # a regular call after the timeout still gives the oracle's bits
    m, n, k, cap = 1000, 8, 2, 200
    idx = W.make_topk_idx(m, n, k, seed=3)
    ref = oracle.capacity(idx, m, k, n, cap, m)
    out = lb.moe_capacity_slots(dev(idx), n, cap)
    lb.sync_status()
    assert (host(out["slot"]) == ref["slot"]).all()
    assert (host(out["expert_offsets"]) == ref["expert_offsets"]).all()
