"""Pins for the oracle's capacity slots, dispatch layout and combine.

Fixed by the pages' worked examples (golden files), by a brute-force recount
of every slot, and by closed-form invariants of the expert-major layout.
Sources: "Switch Transformer read for implementation" (molayo1419.me),
dispatch and capacity sections; "Switch Transformers paper review"
(tildalice.io/?p=118), Expert Capacity and token drop.
"""
import numpy as np
import pytest

import oracle
import workloads as W


def test_dispatch_example(golden):
    g = golden("dispatch_example.txt")
    m, n = int(g["tokens"][0]), int(g["experts"][0])
    route = np.array([int(v) for v in g["route"]], np.int32)[:, None]
    out = oracle.capacity(route, m, 1, n, m, m)
    assert out["expert_offsets"].tolist() == [int(v) for v in g["expert_offsets"]]
    assert out["src_token"][:m].tolist() == [int(v) for v in g["src_token"]]
    assert (out["slot"] >= 0).all()


@pytest.mark.parametrize("cf", ["1.0", "1.25"])
def test_capacity_example(golden, cf):
    g = golden("capacity_example.txt")
    m, n = int(g["tokens"][0]), int(g["experts"][0])
    routed = [int(v) for v in g["routed"]]
    cap = int(g["capacity_" + cf][0])
    assert cap == W.capacity_from_factor(float(cf), m, 1, n)
    # tokens in an interleaved order that realises the counts
    route = np.concatenate([np.full(c, e) for e, c in enumerate(routed)])
    route = np.random.default_rng(0).permutation(route).astype(np.int32)[:, None]
    out = oracle.capacity(route, m, 1, n, cap, m)
    assert out["routed_count"][0].tolist() == routed
    assert out["kept_count"][0].tolist() == [int(v) for v in g["kept_" + cf]]
    assert int((out["slot"] < 0).sum()) == int(g["dropped_" + cf][0])
    # the dropped tokens of an expert are its last arrivals in token order
    for e in range(n):
        toks = np.nonzero(route[:, 0] == e)[0]
        assert (out["slot"][toks, 0] == np.where(np.arange(len(toks)) < cap, np.arange(len(toks)), -1)).all()


def _brute_slots(idx, seg_len, cap):
    m, k = idx.shape
    slot = np.empty_like(idx)
    for i in range(m):
        s0 = (i // seg_len) * seg_len
        for r in range(k):
            e = idx[i, r]
            earlier = int((idx[s0:i] == e).sum())  # a token never picks an expert twice
            slot[i, r] = earlier if earlier < cap else -1
    return slot


@pytest.mark.parametrize("m,n,k,cap,seg", [(96, 8, 2, 20, 96), (96, 8, 2, 7, 32), (64, 16, 3, 0, 64),
                                           (60, 5, 1, 100, 20), (128, 4, 4, 30, 64)])
def test_slots_bruteforce_and_layout(m, n, k, cap, seg):
    idx = W.make_topk_idx(m, n, k, seed=m + n + k)
    out = oracle.capacity(idx, m, k, n, cap, seg)
    assert (out["slot"] == _brute_slots(idx, seg, cap)).all()
    nseg = m // seg
    for s in range(nseg):
        cnt = np.bincount(idx[s * seg:(s + 1) * seg].ravel(), minlength=n)
        assert out["routed_count"][s].tolist() == cnt.tolist()
        assert out["kept_count"][s].tolist() == np.minimum(cnt, cap).tolist()
    off = out["expert_offsets"]
    rows = int(off[-1])
    assert rows == int(out["kept_count"].sum())
    kept = out["dest_row"][out["dest_row"] >= 0]
    assert sorted(kept.tolist()) == list(range(rows))  # a bijection onto [0, rows)
    assert ((out["dest_row"] >= 0) == (out["slot"] >= 0)).all()
    for e in range(n):
        toks = out["src_token"][off[e]:off[e + 1]]
        assert (np.diff(toks) > 0).all()  # token order inside an expert
        assert all(e in idx[t] for t in toks)
    i, r = np.nonzero(out["dest_row"] >= 0)
    assert (out["src_token"][out["dest_row"][i, r]] == i).all()
    assert (out["src_token"][rows:] == -1).all()


def test_capacity_bounds():
    idx = W.make_topk_idx(32, 4, 2, seed=1)
    none = oracle.capacity(idx, 32, 2, 4, 0, 32)
    assert none["expert_offsets"][-1] == 0 and (none["slot"] == -1).all()
    allk = oracle.capacity(idx, 32, 2, 4, 32 * 2, 32)
    assert allk["expert_offsets"][-1] == 64 and (allk["slot"] >= 0).all()
    with pytest.raises(oracle.OracleError):
        oracle.capacity(idx, 32, 2, 4, 5, 10)  # seg_len must divide m


def test_dispatch_and_combine_small():
    # two tokens, experts chosen [1], [0]; only expert 0 has room (capacity 1 each, token 1 dropped? no: distinct)
    x = np.array([[1.0, -2.0], [3.0, 4.0], [5.0, 6.0]], np.float32)
    idx = np.array([[1], [0], [1]], np.int32)
    cap = oracle.capacity(idx, 3, 1, 2, 1, 3)  # expert 1 keeps token 0, drops token 2
    assert cap["slot"][:, 0].tolist() == [0, 0, -1]
    assert cap["src_token"][:2].tolist() == [1, 0]
    xbuf = oracle.dispatch(x, cap["src_token"], 2)
    assert xbuf.tolist() == [[3.0, 4.0], [1.0, -2.0]]
    ybuf = np.array([[10.0, 20.0], [30.0, 40.0]])
    gate = np.array([[0.5], [0.25], [0.75]])
    y = oracle.combine(ybuf, cap["dest_row"], gate, None, 3, 1, 2)
    assert y.tolist() == [[15.0, 20.0], [2.5, 5.0], [0.0, 0.0]]  # the dropped token contributes nothing
    y_res = oracle.combine(ybuf, cap["dest_row"], gate, x, 3, 1, 2)
    assert y_res.tolist() == [[16.0, 18.0], [5.5, 9.0], [5.0, 6.0]]  # dropped token keeps its residual


def test_combine_gate_bf16_rounding_matches_rne():
    gate = np.array([[1.0 + 2.0 ** -9], [1.0 + 3 * 2.0 ** -9], [0.3]])
    ybuf = np.ones((3, 1))
    dest = np.array([[0], [1], [2]], np.int32)
    y = oracle.combine(ybuf, dest, gate, None, 3, 1, 1, gate_bf16=1)
    ref = W.round_to_bf16(gate.astype(np.float32)).astype(np.float64)
    assert y[:, 0].tolist() == ref[:, 0].tolist()
    assert y[0, 0] == 1.0 and y[1, 0] == 1.0 + 2.0 ** -7  # ties to even
