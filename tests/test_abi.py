"""The C-ABI library loads and exports every symbol include/moe.h declares; host-side
argument validation and workspace queries work without a GPU (no compute calls)."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_symbols():
    syms = []
    for name in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if name.endswith(".h"):
            text = open(os.path.join(ROOT, "include", name)).read()
            syms += re.findall(r"^MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text, flags=re.M)
    return syms


@pytest.fixture(scope="module")
def L():
    from load_balanced_dispatch_b200 import build
    build.build()
    import load_balanced_dispatch_b200 as lb
    return lb.lib()


def test_header_declares_the_seven_calls():
    syms = set(header_symbols())
    for call in ("moe_router_topk", "moe_balance_assign", "moe_capacity_slots", "moe_dispatch", "moe_expert_ffn",
                 "moe_combine", "moe_balance_stats"):
        assert call in syms


def test_library_exports_every_declared_symbol(L):
    import load_balanced_dispatch_b200 as lb
    syms = header_symbols()
    assert syms
    for s in syms:
        assert hasattr(L, s), s
    assert set(lb.EXPORTS) <= set(syms)


def test_workspace_queries_are_host_only(L):
    assert L.moe_router_topk_workspace_size(768, 128, 1, 1) >= 3 * 768 * 128 * 2
    assert L.moe_router_topk_workspace_size(64, 8, 1, 0) == 0  # fp32 activations: FMA path, no scratch
    assert L.moe_capacity_slots_workspace_size(8192, 1, 128, 8192) > 0
    assert L.moe_expert_ffn_workspace_size(1, 8192, 3072) >= 8192 * 3072 * 2
    assert L.moe_balance_stats_workspace_size(65536, 64, 4096) > 0
    assert L.moe_balance_assign_workspace_size(65536, 256, 8, 1) >= 65536 * 256 * 4


def _err(L):
    buf = C.create_string_buffer(256)
    L.moe_last_error(buf, 256)
    return buf.value.decode()


def test_invalid_arguments_rejected_before_any_launch(L):
    P = C.c_void_p
    fake = P(256)  # never dereferenced: validation fails first
    # seg_len does not divide m
    rc = L.moe_capacity_slots(fake, 100, 1, 8, 10, 30, fake, fake, fake, fake, fake, fake, fake, 1 << 20, None)
    assert rc == 1 and "seg_len" in _err(L)
    # k > n
    rc = L.moe_router_topk(fake, 1, fake, None, 16, 8, 4, 5, 0, 0, None, None, fake, fake, None, 0, None)
    assert rc == 1 and "k must be" in _err(L)
    # m*k not divisible by n for the balanced assignment
    rc = L.moe_balance_assign(fake, 10, 4, 1, fake, 1, 0, 4, 4, fake, fake, fake, 1 << 30, None)
    assert rc == 1 and "divisible" in _err(L)
    # k must be < n for the balanced assignment
    rc = L.moe_balance_assign(fake, 8, 4, 4, fake, 1, 0, 4, 4, fake, fake, fake, 1 << 30, None)
    assert rc == 1
    # bf16 router without its workspace
    rc = L.moe_router_topk(fake, 1, fake, None, 16, 64, 8, 2, 0, 0, None, None, fake, fake, None, 0, None)
    assert rc == 3 and "workspace" in _err(L)
    # w_r NULL (a prepared split) is only for the tensor-core path: not for fp32 activations
    rc = L.moe_router_topk(fake, 0, None, None, 16, 64, 8, 2, 0, 0, None, None, fake, fake, None, 0, None)
    assert rc == 1 and "moe_router_prepare" in _err(L)
    # preparing the split on the fp32 FMA path: nothing to prepare
    rc = L.moe_router_prepare(fake, 64, 8, 2, 0, fake, 1 << 20, None)
    assert rc == 2 and "FMA" in _err(L)
    # preparing without a workspace
    rc = L.moe_router_prepare(fake, 64, 8, 2, 1, None, 0, None)
    assert rc == 3 and "workspace" in _err(L)
    # workspace too small
    rc = L.moe_capacity_slots(fake, 64, 1, 8, 10, 64, fake, fake, fake, fake, fake, fake, fake, 0, None)
    assert rc == 3 and "workspace" in _err(L)
    # global-batch statistics: totals required, m_total >= 1, workspace sized by the query
    rc = L.moe_balance_totals(fake, fake, 64, 8, 2, None, fake, 1 << 20, None)
    assert rc == 1 and "totals" in _err(L)
    rc = L.moe_balance_totals(fake, fake, 64, 8, 2, fake, fake, 0, None)
    assert rc == 3 and "workspace" in _err(L)
    assert L.moe_balance_totals_workspace_size(64, 8) > 0
    rc = L.moe_balance_global(fake, 0, 8, 2, 1, C.c_float(0.01), fake, fake, fake, None, None, C.c_float(1e-3), None)
    assert rc == 1 and "m_total" in _err(L)
    rc = L.moe_balance_global(fake, 64, 8, 2, 1, C.c_float(0.01), fake, None, None, None, None, C.c_float(1e-3), None)
    assert rc == 1 and "P and aux" in _err(L)
    # d not a multiple of 8 for bf16 dispatch
    rc = L.moe_dispatch(fake, 1, 4, 12, fake, fake, 8, 4, fake, None)
    assert rc == 1
    # misaligned expert buffers
    rc = L.moe_expert_ffn(P(258), 1, fake, fake, fake, fake, fake, 4, 64, 64, 16, fake, fake, 1 << 20, None)
    assert rc == 1 and "aligned" in _err(L)
    # residual aliasing the output
    rc = L.moe_combine(fake, 1, fake, fake, fake, 4, 1, 64, fake, None)
    assert rc == 1 and "alias" in _err(L)
    # the bounded-wait self-test: a flag is required, and the limit is at most the library's own
    rc = L.moe_selftest_wait(None, C.c_int64(1000), None)
    assert rc == 1 and "flag" in _err(L)
    rc = L.moe_selftest_wait(fake, C.c_int64(5_000_000_000), None)
    assert rc == 1 and "limit_cycles" in _err(L)
