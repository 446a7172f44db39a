"""CPU oracle of the MoE-layer forward (test infrastructure).

Only the test suite, `__graft_entry__.smoke()` and the benchmark's CPU-baseline
leg may import this package. The CUDA library never calls it, and it never
calls the CUDA library. The arithmetic lives in `moe_oracle.c` (plain C, one
thread, fp64 accumulation); this module compiles it with gcc and marshals
numpy arrays.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")

SOFTMAX, SIGMOID = 0, 1
QB_STEP, QB_SOLVE = 0, 1
QB_MIDPOINT, QB_BOUNDARY, QB_BIP = 0, 1, 2
OK, ERR_ARG, ERR_NOT_CONVERGED, ERR_INTERNAL = 0, 1, 5, 6


def build(force: bool = False) -> str:
    """Compile the oracle into oracle/libmoe_oracle.so (plain -O2, no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c99", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared",
               "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        P = C.c_void_p
        L, I, D, F = C.c_int64, C.c_int, C.c_double, C.c_float
        _lib.orc_router.argtypes = [P, P, P, L, I, I, I, I, I, P, P, P, P, P]
        _lib.orc_capacity.argtypes = [P, L, I, I, C.c_int32, L, P, P, P, P, P, P]
        _lib.orc_dispatch.argtypes = [P, L, I, P, L, P]
        _lib.orc_dispatch.restype = None
        _lib.orc_expert_ffn.argtypes = [P, P, I, I, I, P, P, P, P, P]
        _lib.orc_expert_ffn.restype = None
        _lib.orc_combine.argtypes = [P, P, P, P, L, I, I, I, P]
        _lib.orc_combine.restype = None
        _lib.orc_balance_stats.argtypes = [P, P, L, I, I, L, D, P, P, P, P, P, F, P]
        _lib.orc_balance_assign.argtypes = [P, L, I, I, P, I, I, I, I, P, P]
        _lib.orc_qb_row.argtypes = [P, L, I, I, P, I, P, P, P]
        _lib.orc_qb_row.restype = None
        _lib.orc_qb_col.argtypes = [P, L, I, L, P, I, P]
        _lib.orc_qb_col.restype = None
        _lib.orc_is_optimal.argtypes = [P, L, I, P, I, D]
        _lib.orc_qb_sign_step.argtypes = [P, L, I, I, P, F, I, P, P]
        _lib.orc_balance_step_minibatch.argtypes = [P, L, I, I, P, I, L, P, P]
        _lib.orc_balance_loss_grad.argtypes = [P, P, L, I, I, L, I, D, D, D, P]
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _f32(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float32)


def _i32(a):
    return np.ascontiguousarray(a, dtype=np.int32)


class OracleError(RuntimeError):
    def __init__(self, fn, code):
        super().__init__(f"{fn} returned status {code}")
        self.code = code


def router(x, w_r, m, d, n, k, fn=SOFTMAX, renorm=0, rank_bias=None, logits_in=None):
    """Returns (probs [m,n] f64, topk_idx [m,k] i32, topk_gate [m,k] f64, margin [m] f64)."""
    x, w_r, rank_bias, logits_in = _f32(x), _f32(w_r), _f32(rank_bias), _f32(logits_in)
    probs = np.empty((m, n), np.float64)
    idx = np.empty((m, k), np.int32)
    gate = np.empty((m, k), np.float64)
    margin = np.empty(m, np.float64)
    rc = lib().orc_router(_p(x), _p(w_r), _p(logits_in), m, d, n, k, fn, renorm, _p(rank_bias),
                          _p(probs), _p(idx), _p(gate), _p(margin))
    if rc:
        raise OracleError("orc_router", rc)
    return probs, idx, gate, margin


def capacity(topk_idx, m, k, n, cap, seg_len):
    """Returns dict(slot, dest_row, src_token, expert_offsets, routed_count, kept_count)."""
    topk_idx = _i32(topk_idx)
    nseg = m // seg_len if seg_len > 0 else 0
    out = dict(slot=np.empty((m, k), np.int32), dest_row=np.empty((m, k), np.int32),
               src_token=np.empty(m * k, np.int32), expert_offsets=np.empty(n + 1, np.int32),
               routed_count=np.empty((max(nseg, 1), n), np.int32), kept_count=np.empty((max(nseg, 1), n), np.int32))
    rc = lib().orc_capacity(_p(topk_idx), m, k, n, cap, seg_len, _p(out["slot"]), _p(out["dest_row"]),
                            _p(out["src_token"]), _p(out["expert_offsets"]), _p(out["routed_count"]),
                            _p(out["kept_count"]))
    if rc:
        raise OracleError("orc_capacity", rc)
    return out


def dispatch(x, src_token, rows):
    x = _f32(x)
    m, d = x.shape
    src_token = _i32(src_token)
    xbuf = np.empty((rows, d), np.float64)
    lib().orc_dispatch(_p(x), m, d, _p(src_token), rows, _p(xbuf))
    return xbuf


def expert_ffn(xbuf, expert_offsets, w1, b1, w2, b2):
    xbuf = np.ascontiguousarray(xbuf, dtype=np.float64)
    n, d_ff, d = w1.shape
    off = _i32(expert_offsets)
    ybuf = np.zeros((xbuf.shape[0], d), np.float64)
    lib().orc_expert_ffn(_p(xbuf), _p(off), n, d, d_ff, _p(_f32(w1)), _p(_f32(b1)), _p(_f32(w2)), _p(_f32(b2)),
                         _p(ybuf))
    return ybuf


def combine(ybuf, dest_row, topk_gate, residual, m, k, d, gate_bf16=0):
    ybuf = np.ascontiguousarray(ybuf, dtype=np.float64)
    gate = np.ascontiguousarray(topk_gate, dtype=np.float64)
    y = np.empty((m, d), np.float64)
    lib().orc_combine(_p(ybuf), _p(_i32(dest_row)), _p(gate), _p(_f32(residual)), m, k, d, gate_bf16, _p(y))
    return y


def balance_stats(probs, topk_idx, m, n, k, seg_len, alpha=1e-2, bias=None, gamma=1e-3):
    """Returns dict(f [nseg+1,n], P [nseg+1,n] or None, aux [nseg+3] or None, vio [3], bias_new or None).
    aux: per segment, micro-batch mean, global-batch, hybrid (global + 0.01 micro)."""
    nseg = m // seg_len
    probs = None if probs is None else np.ascontiguousarray(probs, dtype=np.float64)
    f = np.empty((nseg + 1, n), np.float64)
    P = np.empty((nseg + 1, n), np.float64)
    aux = np.empty(nseg + 3, np.float64)
    vio = np.empty(3, np.float64)
    bias = _f32(bias)
    bias_out = None if bias is None else np.empty(n, np.float32)
    rc = lib().orc_balance_stats(_p(probs), _p(_i32(topk_idx)), m, n, k, seg_len, alpha, _p(f), _p(P), _p(aux),
                                 _p(vio), _p(bias), np.float32(gamma), _p(bias_out))
    if rc:
        raise OracleError("orc_balance_stats", rc)
    return dict(f=f, P=None if probs is None else P, aux=None if probs is None else aux, vio=vio,
                bias=bias_out)


def balance_loss_grad(probs, topk_idx, m, n, k, seg_len, fn=SOFTMAX, alpha=1e-2, w_micro=0.0, w_global=1.0):
    """Gradient of w_global L_global + w_micro L_micro with respect to the router logits: [m, n] f64."""
    probs = np.ascontiguousarray(probs, dtype=np.float64)
    out = np.empty((m, n), np.float64)
    rc = lib().orc_balance_loss_grad(_p(probs), _p(_i32(topk_idx)), m, n, k, seg_len, fn, alpha, w_micro, w_global,
                                     _p(out))
    if rc:
        raise OracleError("orc_balance_loss_grad", rc)
    return out


def balance_assign(s, k, beta=None, mode=QB_SOLVE, rule=QB_MIDPOINT, max_iters=64, max_repair=1 << 20,
                   check=True):
    """Returns (topk_idx [m,k] ascending experts, beta_out [n] f32, info [4], status)."""
    s = _f32(s)
    m, n = s.shape
    beta = np.zeros(n, np.float32) if beta is None else np.array(beta, dtype=np.float32, copy=True)
    idx = np.empty((m, k), np.int32)
    info = np.zeros(4, np.int32)
    rc = lib().orc_balance_assign(_p(s), m, n, k, _p(beta), mode, rule, max_iters, max_repair, _p(idx), _p(info))
    if check and rc not in (OK, ERR_NOT_CONVERGED):
        raise OracleError("orc_balance_assign", rc)
    return idx, beta, info, rc


def qb_sign_step(s, k, beta, gamma, rule=QB_MIDPOINT):
    """One SignSGD-on-beta step: returns (topk_idx [m,k] ascending experts, beta_out [n] f32, info [4])."""
    s = _f32(s)
    m, n = s.shape
    beta = np.array(beta, dtype=np.float32, copy=True)
    idx = np.empty((m, k), np.int32)
    info = np.zeros(4, np.int32)
    rc = lib().orc_qb_sign_step(_p(s), m, n, k, _p(beta), np.float32(gamma), rule, _p(idx), _p(info))
    if rc:
        raise OracleError("orc_qb_sign_step", rc)
    return idx, beta, info


def balance_step_minibatch(s, k, beta, seg_len, rule=QB_MIDPOINT):
    """The practical QB step with beta computed per mini-batch of seg_len tokens and averaged:
    returns (topk_idx [m,k] ascending experts, beta_out [n] f32, info [4])."""
    s = _f32(s)
    m, n = s.shape
    beta = np.array(beta, dtype=np.float32, copy=True)
    idx = np.empty((m, k), np.int32)
    info = np.zeros(4, np.int32)
    rc = lib().orc_balance_step_minibatch(_p(s), m, n, k, _p(beta), rule, seg_len, _p(idx), _p(info))
    if rc:
        raise OracleError("orc_balance_step_minibatch", rc)
    return idx, beta, info


def qb_row(s, k, beta, rule=QB_MIDPOINT):
    """One row pass: (alpha [m] f32, topk_idx [m,k] best first, counts [n])."""
    s = _f32(s)
    m, n = s.shape
    alpha = np.empty(m, np.float32)
    idx = np.empty((m, k), np.int32)
    counts = np.empty(n, np.int64)
    lib().orc_qb_row(_p(s), m, n, k, _p(_f32(beta)), rule, _p(alpha), _p(idx), _p(counts))
    return alpha, idx, counts


def qb_col(s, k, alpha, rule=QB_MIDPOINT):
    """One column pass: beta [n] f32 with C = m k / n."""
    s = _f32(s)
    m, n = s.shape
    beta = np.empty(n, np.float32)
    lib().orc_qb_col(_p(s), m, n, m * k // n, _p(_f32(alpha)), rule, _p(beta))
    return beta


def is_optimal(s, topk_idx, tol=1e-9):
    s = _f32(s)
    m, n = s.shape
    idx = _i32(topk_idx)
    return bool(lib().orc_is_optimal(_p(s), m, n, _p(idx), idx.shape[1], tol))


def layer_forward(inp: dict, cfg, residual=None, probs_needed=True):
    """Whole layer through the oracle: router -> capacity -> dispatch -> FFN -> combine -> stats.

    `inp` is the dict of `workloads.make_layer_inputs`; `cfg` a `workloads.LayerConfig`.
    Returns a dict with every intermediate.
    """
    m, d, n, k = cfg.m, cfg.d, cfg.n, cfg.k
    fn = SOFTMAX if cfg.score_fn == "softmax" else SIGMOID
    probs, idx, gate, margin = router(inp["x"], inp["w_r"], m, d, n, k, fn, cfg.renorm_topk, inp.get("rank_bias"))
    cap = capacity(idx, m, k, n, cfg.capacity, cfg.seg_len)
    rows = int(cap["expert_offsets"][-1])
    xbuf = dispatch(inp["x"], cap["src_token"], rows)
    ybuf = expert_ffn(xbuf, cap["expert_offsets"], inp["w1"], inp["b1"], inp["w2"], inp["b2"])
    res = inp["x"] if residual else None
    y = combine(ybuf, cap["dest_row"], gate, res, m, k, d, gate_bf16=int(cfg.dtype == "bf16"))
    st = balance_stats(probs if probs_needed else None, idx, m, n, k, cfg.seg_len, cfg.alpha,
                       inp.get("rank_bias"), cfg.gamma)
    return dict(probs=probs, topk_idx=idx, topk_gate=gate, margin=margin, cap=cap, rows=rows, xbuf=xbuf,
                ybuf=ybuf, y=y, stats=st)
