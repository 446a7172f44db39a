"""Python binding of the B200 MoE-layer forward library (libmoe_b200.so).

Argument marshalling only: each function takes torch tensors, checks dtypes,
devices and shapes, optionally allocates outputs and workspaces through torch
(device memory is PyTorch's job here), and calls the C entry point of the same
name on the current CUDA stream. Every step of the computation runs in the
library's CUDA kernels; there is no fallback. If the library is missing, the
import of any function raises immediately.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_F32, MOE_BF16 = 0, 1
MOE_SOFTMAX, MOE_SIGMOID = 0, 1
MOE_QB_STEP, MOE_QB_SOLVE = 0, 1
MOE_QB_MIDPOINT, MOE_QB_BOUNDARY, MOE_QB_BIP = 0, 1, 2
STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE",
          4: "MOE_ERR_CUDA", 5: "MOE_ERR_NOT_CONVERGED", 6: "MOE_ERR_INTERNAL"}

# every symbol the C header declares
EXPORTS = ("moe_last_error", "moe_sync_status", "moe_router_topk_workspace_size", "moe_router_topk", "moe_balance_assign_workspace_size",
           "moe_balance_assign", "moe_capacity_slots_workspace_size", "moe_capacity_slots", "moe_dispatch",
           "moe_expert_ffn_workspace_size", "moe_expert_ffn", "moe_combine", "moe_balance_stats_workspace_size",
           "moe_balance_stats", "moe_capacity_slots_static", "moe_balance_totals_workspace_size",
           "moe_balance_totals", "moe_balance_global", "moe_expert_ffn_combine", "moe_balance_sign_step",
           "moe_expert_ffn_gather", "moe_dispatch_tokens", "moe_router_prepare",
           "moe_balance_step_minibatch", "moe_ep_plan", "moe_ep_dispatch", "moe_ep_combine",
           "moe_balance_loss_grad")


class MoEError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn}: {STATUS.get(code, code)}: {msg}")
        self.code = code


_lib = None


def lib() -> C.CDLL:
    """Load libmoe_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m load_balanced_dispatch_b200.build`")
        L = C.CDLL(LIB_PATH)
        P, I64, I32, F, SZ = C.c_void_p, C.c_int64, C.c_int32, C.c_float, C.c_size_t
        L.moe_last_error.argtypes = [C.c_char_p, SZ]
        L.moe_last_error.restype = None
        L.moe_sync_status.argtypes = [P]
        L.moe_selftest_wait.argtypes = [P, I64, P]
        L.moe_router_topk_workspace_size.argtypes = [I32, I32, I32, I32]
        L.moe_router_topk_workspace_size.restype = SZ
        L.moe_router_topk.argtypes = [P, I32, P, P, I64, I32, I32, I32, I32, I32, P, P, P, P, P, SZ, P]
        L.moe_router_prepare.argtypes = [P, I32, I32, I32, I32, P, SZ, P]
        L.moe_balance_assign_workspace_size.argtypes = [I64, I32, I32, I32]
        L.moe_balance_assign_workspace_size.restype = SZ
        L.moe_balance_assign.argtypes = [P, I64, I32, I32, P, I32, I32, I32, I32, P, P, P, SZ, P]
        L.moe_capacity_slots_workspace_size.argtypes = [I64, I32, I32, I64]
        L.moe_capacity_slots_workspace_size.restype = SZ
        L.moe_capacity_slots.argtypes = [P, I64, I32, I32, I32, I64, P, P, P, P, P, P, P, SZ, P]
        L.moe_capacity_slots_static.argtypes = [P, I64, I32, I32, I32, I64, P, P, P, P, P, P, P]
        L.moe_dispatch.argtypes = [P, I32, I64, I32, P, P, I32, I64, P, P]
        L.moe_dispatch_tokens.argtypes = [P, I32, I64, I32, I32, P, I64, P, P]
        L.moe_ep_plan.argtypes = [P, I32, I32, I32, P, P, P]
        L.moe_balance_loss_grad.argtypes = [P, I32, P, I64, I32, I64, F, F, F, P, P]
        L.moe_ep_dispatch.argtypes = [P, I32, I64, I32, I32, I32, I32, P, P, P, P, P, I64, P, P]
        L.moe_ep_combine.argtypes = [P, I32, P, P, I32, I32, P, P, I64, I32, I32, P, P]
        L.moe_expert_ffn_workspace_size.argtypes = [I32, I64, I32]
        L.moe_expert_ffn_workspace_size.restype = SZ
        L.moe_expert_ffn.argtypes = [P, I32, P, P, P, P, P, I32, I32, I32, I64, P, P, SZ, P]
        L.moe_combine.argtypes = [P, I32, P, P, P, I64, I32, I32, P, P]
        L.moe_expert_ffn_combine.argtypes = [P, I32, P, P, P, P, P, I32, I32, I32, I64, P, P, P, P, I64, P, P, SZ,
                                             P]
        L.moe_expert_ffn_gather.argtypes = [P, I32, P, P, P, P, P, I32, I32, I32, I64, P, I64, P, P, SZ, P]
        L.moe_balance_stats_workspace_size.argtypes = [I64, I32, I64]
        L.moe_balance_stats_workspace_size.restype = SZ
        L.moe_balance_stats.argtypes = [P, P, I64, I32, I32, I64, F, P, P, P, P, P, F, P, SZ, P]
        L.moe_balance_sign_step.argtypes = [P, I64, I32, I32, P, F, I32, P, P, P, SZ, P]
        L.moe_balance_step_minibatch.argtypes = [P, I64, I32, I32, P, I32, I64, P, P, P, SZ, P]
        L.moe_balance_totals_workspace_size.argtypes = [I64, I32]
        L.moe_balance_totals_workspace_size.restype = SZ
        L.moe_balance_totals.argtypes = [P, P, I64, I32, I32, P, P, SZ, P]
        L.moe_balance_global.argtypes = [P, I64, I32, I32, I32, F, P, P, P, P, P, F, P]
        for name in EXPORTS:
            if name not in ("moe_last_error",) and not name.endswith("_workspace_size"):
                getattr(L, name).restype = C.c_int
        _lib = L
    return _lib


def last_error() -> str:
    buf = C.create_string_buffer(512)
    lib().moe_last_error(buf, 512)
    return buf.value.decode()


def _check(fn: str, code: int):
    if code != 0:
        raise MoEError(fn, code, last_error())


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return MOE_BF16
    if t.dtype == torch.float32:
        return MOE_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _need(t, dtype, shape, name):
    if t is None:
        return
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous() or not t.is_cuda:
        raise ValueError(f"{name}: expected contiguous CUDA {dtype} {tuple(shape)}, got {t.dtype} {tuple(t.shape)}")


def sync_status(stream=None):
    """Synchronise the stream and raise if a kernel recorded a device-side error."""
    _check("moe_sync_status", lib().moe_sync_status(_stream(stream)))


def moe_selftest_wait(flag, limit_cycles, stream=None):
    """One warp waits (at most limit_cycles SM cycles) for the int32 device scalar `flag` to reach 1;
    if nothing sets it, the device error word records a pipeline timeout (see sync_status)."""
    _need(flag, torch.int32, (1,), "flag")
    _check("moe_selftest_wait", lib().moe_selftest_wait(_ptr(flag), int(limit_cycles), _stream(stream)))


def moe_router_topk(x, w_r, n, k, score_fn=MOE_SOFTMAX, renorm_topk=0, rank_bias=None, logits_in=None,
                    probs_out=None, topk_idx=None, topk_gate=None, want_probs=True, workspace=None, stream=None):
    """Router + top-k. Returns (topk_idx [m,k] int32, topk_gate [m,k] fp32, probs [m,n] fp32 or None).
    w_r None: the workspace holds the split made by moe_router_prepare (tensor-core path only)."""
    if logits_in is not None:
        m, d = logits_in.shape[0], 0
        dev = logits_in.device
        _need(logits_in, torch.float32, (m, n), "logits_in")
        xdt = MOE_F32
    else:
        m, d = x.shape
        dev = x.device
        xdt = _dtype_code(x)
        _need(x, x.dtype, (m, d), "x")
        _need(w_r, torch.float32, (d, n), "w_r")
        if w_r is None and workspace is None:
            raise ValueError("w_r None needs the workspace prepared by moe_router_prepare")
    _need(rank_bias, torch.float32, (n,), "rank_bias")
    if topk_idx is None:
        topk_idx = torch.empty((m, k), dtype=torch.int32, device=dev)
    if topk_gate is None:
        topk_gate = torch.empty((m, k), dtype=torch.float32, device=dev)
    if probs_out is None and want_probs:
        probs_out = torch.empty((m, n), dtype=torch.float32, device=dev)
    ws_bytes = lib().moe_router_topk_workspace_size(d, n, k, xdt) if logits_in is None else 0
    if workspace is None and ws_bytes:
        workspace = torch.empty((ws_bytes,), dtype=torch.uint8, device=dev)
    _check("moe_router_topk", lib().moe_router_topk(
        _ptr(x), xdt, _ptr(w_r), _ptr(logits_in), m, d, n, k, score_fn, renorm_topk, _ptr(rank_bias),
        _ptr(probs_out), _ptr(topk_idx), _ptr(topk_gate), _ptr(workspace),
        0 if workspace is None else workspace.numel(), _stream(stream)))
    return topk_idx, topk_gate, probs_out


def moe_router_prepare(w_r, k, x_dtype=torch.bfloat16, workspace=None, stream=None):
    """Split the static router weight once into the router workspace (tensor-core path). Returns the
    workspace, for moe_router_topk(x, None, ..., workspace=ws)."""
    d, n = w_r.shape
    _need(w_r, torch.float32, (d, n), "w_r")
    xdt = MOE_BF16 if x_dtype == torch.bfloat16 else MOE_F32
    ws_bytes = lib().moe_router_topk_workspace_size(d, n, k, xdt)
    if workspace is None:
        workspace = torch.empty((max(ws_bytes, 1),), dtype=torch.uint8, device=w_r.device)
    _check("moe_router_prepare", lib().moe_router_prepare(_ptr(w_r), d, n, k, xdt, _ptr(workspace),
                                                          workspace.numel(), _stream(stream)))
    return workspace


def moe_capacity_slots(topk_idx, n, capacity, seg_len=None, out=None, workspace=None, stream=None):
    """Capacity slots. Returns dict(slot, dest_row, src_token, expert_offsets, routed_count, kept_count)."""
    m, k = topk_idx.shape
    seg_len = m if seg_len is None else seg_len
    dev = topk_idx.device
    nseg = m // seg_len if seg_len > 0 else 1
    if out is None:
        out = dict(slot=torch.empty((m, k), dtype=torch.int32, device=dev),
                   dest_row=torch.empty((m, k), dtype=torch.int32, device=dev),
                   src_token=torch.empty((m * k,), dtype=torch.int32, device=dev),
                   expert_offsets=torch.empty((n + 1,), dtype=torch.int32, device=dev),
                   routed_count=torch.empty((nseg, n), dtype=torch.int32, device=dev),
                   kept_count=torch.empty((nseg, n), dtype=torch.int32, device=dev))
    ws_bytes = lib().moe_capacity_slots_workspace_size(m, k, n, seg_len)
    if workspace is None:
        workspace = torch.empty((max(ws_bytes, 1),), dtype=torch.uint8, device=dev)
    _check("moe_capacity_slots", lib().moe_capacity_slots(
        _ptr(topk_idx), m, k, n, capacity, seg_len, _ptr(out["slot"]), _ptr(out["dest_row"]), _ptr(out["src_token"]),
        _ptr(out["expert_offsets"]), _ptr(out["routed_count"]), _ptr(out["kept_count"]), _ptr(workspace),
        workspace.numel(), _stream(stream)))
    return out


def moe_capacity_slots_static(topk_idx, n, capacity, seg_len=None, out=None, stream=None):
    """moe_capacity_slots without a workspace: the library's fixed 1 MiB scratch array is used
    instead, for callers that cannot allocate device memory. Same outputs as moe_capacity_slots."""
    m, k = topk_idx.shape
    seg_len = m if seg_len is None else seg_len
    dev = topk_idx.device
    nseg = m // seg_len if seg_len > 0 else 1
    if out is None:
        out = dict(slot=torch.empty((m, k), dtype=torch.int32, device=dev),
                   dest_row=torch.empty((m, k), dtype=torch.int32, device=dev),
                   src_token=torch.empty((m * k,), dtype=torch.int32, device=dev),
                   expert_offsets=torch.empty((n + 1,), dtype=torch.int32, device=dev),
                   routed_count=torch.empty((nseg, n), dtype=torch.int32, device=dev),
                   kept_count=torch.empty((nseg, n), dtype=torch.int32, device=dev))
    _check("moe_capacity_slots_static", lib().moe_capacity_slots_static(
        _ptr(topk_idx), m, k, n, capacity, seg_len, _ptr(out["slot"]), _ptr(out["dest_row"]), _ptr(out["src_token"]),
        _ptr(out["expert_offsets"]), _ptr(out["routed_count"]), _ptr(out["kept_count"]), _stream(stream)))
    return out


def moe_dispatch(x, src_token, expert_offsets, n, max_rows=None, xbuf=None, stream=None):
    """xbuf[r] = x[src_token[r]] for the kept rows (expert-major). Returns xbuf [max_rows, d]."""
    m, d = x.shape
    max_rows = src_token.numel() if max_rows is None else max_rows
    if xbuf is None:
        xbuf = torch.empty((max_rows, d), dtype=x.dtype, device=x.device)
    _check("moe_dispatch", lib().moe_dispatch(_ptr(x), _dtype_code(x), m, d, _ptr(src_token), _ptr(expert_offsets),
                                              n, max_rows, _ptr(xbuf), _stream(stream)))
    return xbuf


def moe_dispatch_tokens(x, dest_row, max_rows=None, xbuf=None, stream=None):
    """xbuf[dest_row[i, r]] = x[i] for the kept picks, visiting tokens (each x row read once).
    Returns xbuf [max_rows, d]; the same rows as moe_dispatch."""
    m, d = x.shape
    k = dest_row.shape[1]
    max_rows = m * k if max_rows is None else max_rows
    if xbuf is None:
        xbuf = torch.empty((max_rows, d), dtype=x.dtype, device=x.device)
    _check("moe_dispatch_tokens", lib().moe_dispatch_tokens(_ptr(x), _dtype_code(x), m, d, k, _ptr(dest_row),
                                                            max_rows, _ptr(xbuf), _stream(stream)))
    return xbuf


def moe_ep_plan(offsets_all, rank, send_base=None, recv_offsets=None, stream=None):
    """Expert parallelism, the exchange plan of one rank from every rank's expert_offsets
    offsets_all [G, n+1]: (send_base [n], recv_offsets [n/G + 1])."""
    G, n1 = offsets_all.shape
    n = n1 - 1
    dev = offsets_all.device
    _need(offsets_all, torch.int32, (G, n + 1), "offsets_all")
    if send_base is None:
        send_base = torch.empty((n,), dtype=torch.int32, device=dev)
    if recv_offsets is None:
        recv_offsets = torch.empty((n // G + 1,), dtype=torch.int32, device=dev)
    _check("moe_ep_plan", lib().moe_ep_plan(_ptr(offsets_all), G, n, rank, _ptr(send_base), _ptr(recv_offsets),
                                            _stream(stream)))
    return send_base, recv_offsets


def moe_ep_dispatch(x, topk_idx, dest_row, expert_offsets, send_base, peer_xrecv, G, max_recv_rows, ep_row=None,
                    stream=None):
    """Store each kept row of this rank's tokens into its expert owner's receive buffer. peer_xrecv:
    a device int64 tensor [G] of buffer addresses (this GPU's view). Returns ep_row [m, k]."""
    m, d = x.shape
    k = topk_idx.shape[1]
    n = expert_offsets.numel() - 1
    if ep_row is None:
        ep_row = torch.empty((m, k), dtype=torch.int32, device=x.device)
    _check("moe_ep_dispatch", lib().moe_ep_dispatch(
        _ptr(x), _dtype_code(x), m, d, k, n, G, _ptr(topk_idx), _ptr(dest_row), _ptr(expert_offsets),
        _ptr(send_base), _ptr(peer_xrecv), max_recv_rows, _ptr(ep_row), _stream(stream)))
    return ep_row


def moe_ep_combine(peer_yrecv, dtype, ep_row, topk_idx, n, G, topk_gate, residual=None, y=None, d=None, stream=None):
    """y = (residual) + gated sum of the owners' output rows (peer loads). peer_yrecv: device int64 [G]."""
    m, k = ep_row.shape
    if y is None:
        y = torch.empty((m, d), dtype=dtype, device=ep_row.device)
    d = y.shape[1]
    code = MOE_BF16 if dtype == torch.bfloat16 else MOE_F32
    _check("moe_ep_combine", lib().moe_ep_combine(
        _ptr(peer_yrecv), code, _ptr(ep_row), _ptr(topk_idx), n, G, _ptr(topk_gate), _ptr(residual), m, k, d,
        _ptr(y), _stream(stream)))
    return y


def moe_expert_ffn(xbuf, w1, b1, w2, b2, expert_offsets, ybuf=None, workspace=None, stream=None):
    """ybuf = max(0, xbuf W1_e + b1_e) W2_e + b2_e per expert group. w1 [n,d_ff,d], w2 [n,d,d_ff]."""
    max_rows, d = xbuf.shape
    n, d_ff, _ = w1.shape
    dt = _dtype_code(xbuf)
    for t, shp, name in ((w1, (n, d_ff, d), "w1"), (b1, (n, d_ff), "b1"), (w2, (n, d, d_ff), "w2"), (b2, (n, d), "b2")):
        _need(t, xbuf.dtype, shp, name)
    if ybuf is None:
        ybuf = torch.empty((max_rows, d), dtype=xbuf.dtype, device=xbuf.device)
    ws_bytes = lib().moe_expert_ffn_workspace_size(dt, max_rows, d_ff)
    if workspace is None:
        workspace = torch.empty((ws_bytes,), dtype=torch.uint8, device=xbuf.device)
    _check("moe_expert_ffn", lib().moe_expert_ffn(
        _ptr(xbuf), dt, _ptr(w1), _ptr(b1), _ptr(w2), _ptr(b2), _ptr(expert_offsets), n, d, d_ff, max_rows,
        _ptr(ybuf), _ptr(workspace), workspace.numel(), _stream(stream)))
    return ybuf


def moe_expert_ffn_gather(x, w1, b1, w2, b2, expert_offsets, src_token, max_rows=None, ybuf=None, workspace=None,
                          stream=None):
    """bf16: ybuf = the FFN of x[src_token[r]] per expert group, rows gathered by the FFN itself (no xbuf)."""
    m, d = x.shape
    n, d_ff, _ = w1.shape
    max_rows = src_token.numel() if max_rows is None else max_rows
    dt = _dtype_code(x)
    for t, shp, name in ((w1, (n, d_ff, d), "w1"), (b1, (n, d_ff), "b1"), (w2, (n, d, d_ff), "w2"), (b2, (n, d), "b2")):
        _need(t, x.dtype, shp, name)
    if ybuf is None:
        ybuf = torch.empty((max_rows, d), dtype=x.dtype, device=x.device)
    ws_bytes = lib().moe_expert_ffn_workspace_size(dt, max_rows, d_ff)
    if workspace is None:
        workspace = torch.empty((ws_bytes,), dtype=torch.uint8, device=x.device)
    _check("moe_expert_ffn_gather", lib().moe_expert_ffn_gather(
        _ptr(x), dt, _ptr(w1), _ptr(b1), _ptr(w2), _ptr(b2), _ptr(expert_offsets), n, d, d_ff, max_rows,
        _ptr(src_token), m, _ptr(ybuf), _ptr(workspace), workspace.numel(), _stream(stream)))
    return ybuf


def moe_expert_ffn_combine(xbuf, w1, b1, w2, b2, expert_offsets, src_token, dest_row, topk_gate, residual=None,
                           y=None, workspace=None, stream=None):
    """k = 1, bf16: y[t] = residual[t] + g_t FFN_e(xbuf[row of t]) with the combine done by the FFN's second
    GEMM (no ybuf); tokens without a kept row get the residual or zeros. Returns y [m, d]."""
    max_rows, d = xbuf.shape
    n, d_ff, _ = w1.shape
    m, k = dest_row.shape
    if k != 1:
        raise ValueError("moe_expert_ffn_combine: one pick per token (k = 1)")
    max_rows = min(max_rows, m)
    dt = _dtype_code(xbuf)
    for t, shp, name in ((w1, (n, d_ff, d), "w1"), (b1, (n, d_ff), "b1"), (w2, (n, d, d_ff), "w2"), (b2, (n, d), "b2")):
        _need(t, xbuf.dtype, shp, name)
    _need(residual, xbuf.dtype, (m, d), "residual")
    if y is None:
        y = torch.empty((m, d), dtype=xbuf.dtype, device=xbuf.device)
    ws_bytes = lib().moe_expert_ffn_workspace_size(dt, max_rows, d_ff)
    if workspace is None:
        workspace = torch.empty((ws_bytes,), dtype=torch.uint8, device=xbuf.device)
    _check("moe_expert_ffn_combine", lib().moe_expert_ffn_combine(
        _ptr(xbuf), dt, _ptr(w1), _ptr(b1), _ptr(w2), _ptr(b2), _ptr(expert_offsets), n, d, d_ff, max_rows,
        _ptr(src_token), _ptr(dest_row), _ptr(topk_gate), _ptr(residual), m, _ptr(y), _ptr(workspace),
        workspace.numel(), _stream(stream)))
    return y


def moe_combine(ybuf, dest_row, topk_gate, residual=None, y=None, stream=None):
    """y[i] = residual[i] + sum_r g_ir ybuf[dest_row[i,r]] (kept picks only). Returns y [m, d]."""
    m, k = dest_row.shape
    d = ybuf.shape[1]
    if y is None:
        y = torch.empty((m, d), dtype=ybuf.dtype, device=ybuf.device)
    _check("moe_combine", lib().moe_combine(_ptr(ybuf), _dtype_code(ybuf), _ptr(dest_row), _ptr(topk_gate),
                                            _ptr(residual), m, k, d, _ptr(y), _stream(stream)))
    return y


def moe_balance_stats(probs, topk_idx, n, seg_len=None, alpha=1e-2, bias_inout=None, gamma=1e-3, out=None,
                      workspace=None, stream=None):
    """f, P [nseg+1, n], aux [nseg+3], vio [3]; updates bias_inout in place when given."""
    m, k = topk_idx.shape
    seg_len = m if seg_len is None else seg_len
    nseg = m // seg_len
    dev = topk_idx.device
    if out is None:
        out = dict(f=torch.empty((nseg + 1, n), dtype=torch.float32, device=dev),
                   P=torch.empty((nseg + 1, n), dtype=torch.float32, device=dev),
                   aux=torch.empty((nseg + 3,), dtype=torch.float32, device=dev),
                   vio=torch.empty((3,), dtype=torch.float32, device=dev))
    ws_bytes = lib().moe_balance_stats_workspace_size(m, n, seg_len)
    if workspace is None:
        workspace = torch.empty((max(ws_bytes, 1),), dtype=torch.uint8, device=dev)
    _check("moe_balance_stats", lib().moe_balance_stats(
        _ptr(probs), _ptr(topk_idx), m, n, k, seg_len, alpha, _ptr(out["f"]), _ptr(out["P"] if probs is not None else None),
        _ptr(out["aux"] if probs is not None else None), _ptr(out["vio"]), _ptr(bias_inout), gamma, _ptr(workspace),
        workspace.numel(), _stream(stream)))
    return out


def moe_balance_loss_grad(probs, f, seg_len=None, score_fn=MOE_SOFTMAX, alpha=1e-2, w_micro=0.01, w_global=1.0,
                          dlogits=None, stream=None):
    """Router-logit gradient of w_global L_global + w_micro L_micro, f held fixed. Returns dlogits [m, n]."""
    m, n = probs.shape
    seg_len = m if seg_len is None else seg_len
    _need(probs, torch.float32, (m, n), "probs")
    _need(f, torch.float32, (m // seg_len + 1, n), "f")
    if dlogits is None:
        dlogits = torch.empty((m, n), dtype=torch.float32, device=probs.device)
    _check("moe_balance_loss_grad", lib().moe_balance_loss_grad(
        _ptr(probs), score_fn, _ptr(f), m, n, seg_len, alpha, w_micro, w_global, _ptr(dlogits), _stream(stream)))
    return dlogits


def moe_balance_totals(probs, topk_idx, n, totals=None, workspace=None, stream=None):
    """This rank's [2, n] fp64 totals: routed copies per expert and probability sums (row 1 is 0 without probs)."""
    m, k = topk_idx.shape
    dev = topk_idx.device
    _need(topk_idx, torch.int32, (m, k), "topk_idx")
    _need(probs, torch.float32, (m, n), "probs")
    if totals is None:
        totals = torch.empty((2, n), dtype=torch.float64, device=dev)
    _need(totals, torch.float64, (2, n), "totals")
    ws_bytes = lib().moe_balance_totals_workspace_size(m, n)
    if workspace is None:
        workspace = torch.empty((max(ws_bytes, 1),), dtype=torch.uint8, device=dev)
    _check("moe_balance_totals", lib().moe_balance_totals(
        _ptr(probs), _ptr(topk_idx), m, n, k, _ptr(totals), _ptr(workspace), workspace.numel(), _stream(stream)))
    return totals


def moe_balance_global(totals, m_total, k, has_probs=True, alpha=1e-2, bias_inout=None, gamma=1e-3, out=None,
                       stream=None):
    """Global-batch f, P [n], aux [1], vio [3] from totals summed over the ranks (m_total tokens in all)."""
    n = totals.shape[1]
    dev = totals.device
    _need(totals, torch.float64, (2, n), "totals")
    _need(bias_inout, torch.float32, (n,), "bias_inout")
    if out is None:
        out = dict(f=torch.empty((n,), dtype=torch.float32, device=dev),
                   P=torch.empty((n,), dtype=torch.float32, device=dev),
                   aux=torch.empty((1,), dtype=torch.float32, device=dev),
                   vio=torch.empty((3,), dtype=torch.float32, device=dev))
    _check("moe_balance_global", lib().moe_balance_global(
        _ptr(totals), m_total, n, k, 1 if has_probs else 0, alpha, _ptr(out["f"]), _ptr(out["P"]), _ptr(out["aux"]),
        _ptr(out["vio"]), _ptr(bias_inout), gamma, _stream(stream)))
    return out


def moe_balance_sign_step(s, k, beta, gamma, rule=MOE_QB_MIDPOINT, topk_idx=None, info=None, workspace=None,
                          stream=None):
    """One SignSGD step on beta (in place): (topk_idx [m,k] ascending experts, beta, info [4])."""
    m, n = s.shape
    dev = s.device
    _need(s, torch.float32, (m, n), "s")
    _need(beta, torch.float32, (n,), "beta")
    if topk_idx is None:
        topk_idx = torch.empty((m, k), dtype=torch.int32, device=dev)
    if info is None:
        info = torch.zeros((4,), dtype=torch.int32, device=dev)
    ws_bytes = lib().moe_balance_assign_workspace_size(m, n, k, MOE_QB_STEP)
    if workspace is None:
        workspace = torch.empty((ws_bytes,), dtype=torch.uint8, device=dev)
    _check("moe_balance_sign_step", lib().moe_balance_sign_step(
        _ptr(s), m, n, k, _ptr(beta), gamma, rule, _ptr(topk_idx), _ptr(info), _ptr(workspace), workspace.numel(),
        _stream(stream)))
    return topk_idx, beta, info


def moe_balance_step_minibatch(s, k, beta, seg_len, rule=MOE_QB_MIDPOINT, topk_idx=None, info=None, workspace=None,
                               stream=None):
    """The practical QB step with beta averaged over mini-batches of seg_len tokens (beta updated in
    place): (topk_idx [m,k] ascending experts, beta, info [4])."""
    m, n = s.shape
    dev = s.device
    _need(s, torch.float32, (m, n), "s")
    _need(beta, torch.float32, (n,), "beta")
    if topk_idx is None:
        topk_idx = torch.empty((m, k), dtype=torch.int32, device=dev)
    if info is None:
        info = torch.zeros((4,), dtype=torch.int32, device=dev)
    ws_bytes = lib().moe_balance_assign_workspace_size(m, n, k, MOE_QB_STEP)
    if workspace is None:
        workspace = torch.empty((ws_bytes,), dtype=torch.uint8, device=dev)
    _check("moe_balance_step_minibatch", lib().moe_balance_step_minibatch(
        _ptr(s), m, n, k, _ptr(beta), rule, seg_len, _ptr(topk_idx), _ptr(info), _ptr(workspace), workspace.numel(),
        _stream(stream)))
    return topk_idx, beta, info


def moe_balance_assign(s, k, beta=None, mode=MOE_QB_SOLVE, rule=MOE_QB_MIDPOINT, max_iters=64, max_repair=1 << 20,
                       topk_idx=None, info=None, workspace=None, stream=None):
    """Balanced assignment. Returns (topk_idx [m,k] ascending experts, beta [n] (updated in place), info [4])."""
    m, n = s.shape
    dev = s.device
    if beta is None:
        beta = torch.zeros((n,), dtype=torch.float32, device=dev)
    if topk_idx is None:
        topk_idx = torch.empty((m, k), dtype=torch.int32, device=dev)
    if info is None:
        info = torch.zeros((4,), dtype=torch.int32, device=dev)
    ws_bytes = lib().moe_balance_assign_workspace_size(m, n, k, mode)
    if workspace is None:
        workspace = torch.empty((max(ws_bytes, 1),), dtype=torch.uint8, device=dev)
    _check("moe_balance_assign", lib().moe_balance_assign(
        _ptr(s), m, n, k, _ptr(beta), mode, rule, max_iters, max_repair, _ptr(topk_idx), _ptr(info), _ptr(workspace),
        workspace.numel(), _stream(stream)))
    return topk_idx, beta, info
