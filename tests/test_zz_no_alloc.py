"""moe_capacity_slots_static: capacity slots for callers that cannot allocate device memory.

Some callers cannot hand the library a workspace -- code reached through a fixed
foreign-function signature that carries only inputs and outputs, or a host
framework that owns all device memory and forbids its plugins to call
cudaMalloc. For them the library runs the capacity kernels on a fixed 1 MiB
scratch array of its own. This test calls that entry point through the C ABI
twice in a row, on different problems (the second smaller than the first, so
stale scratch contents from the first call are present), and checks that every
output equals the one of moe_capacity_slots with a caller workspace, bit for
bit (these are integer results). A second pair runs small-then-large (so the
large call uses scratch words the small one never touched), then an empty problem.
It also checks that a problem needing more than the fixed array, or one with
invalid arguments, is rejected before anything runs.
"""
import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu

lb = pytest.importorskip("load_balanced_dispatch_b200")


@pytest.fixture(scope="module")
def lib():
    from load_balanced_dispatch_b200 import build
    build.build()
    assert torch.cuda.is_available()
    torch.cuda.set_device(0)
    return lb.lib()


KEYS = ("slot", "dest_row", "expert_offsets", "routed_count", "kept_count")


def _compare(idx, n, cap, seg):
    m, k = idx.shape
    d_idx = torch.from_numpy(idx).cuda()
    ref = lb.moe_capacity_slots(d_idx, n, cap, seg)
    got = lb.moe_capacity_slots_static(d_idx, n, cap, seg)
    torch.cuda.synchronize()
    lb.sync_status()
    rows = int(ref["expert_offsets"][-1].item())
    for key in KEYS:
        assert torch.equal(got[key], ref[key]), key
    assert torch.equal(got["src_token"][:rows], ref["src_token"][:rows])


def test_static_scratch_matches_workspace_version_on_two_calls(lib):
    # call 1: 16 micro-batches of 4096 tokens, top-2 over 64 experts (the global-batch shape)
    _compare(W.make_topk_idx(65536, 64, 2, seed=11), 64, 256, 4096)
    # call 2: a smaller single-segment top-1 problem over 128 experts with heavy drops
    _compare(W.make_topk_idx(8192, 128, 1, seed=12), 128, 40, 8192)


def test_static_scratch_small_then_large_and_empty(lib):
    # small first, then large: the large call's per-chunk words lie past anything the small one wrote
    _compare(W.make_topk_idx(1024, 16, 2, seed=13), 16, 100, 512)
    _compare(W.make_topk_idx(32768, 64, 4, seed=14), 64, 300, 8192)
    # no tokens: the empty layout (all offsets 0), from both entry points
    n = 32
    empty = torch.empty((0, 2), dtype=torch.int32, device="cuda")

    def outs():
        return dict(slot=torch.empty((0, 2), dtype=torch.int32, device="cuda"),
                    dest_row=torch.empty((0, 2), dtype=torch.int32, device="cuda"),
                    src_token=torch.empty((1,), dtype=torch.int32, device="cuda"),
                    expert_offsets=torch.full((n + 1,), 7, dtype=torch.int32, device="cuda"),
                    routed_count=torch.empty((1, n), dtype=torch.int32, device="cuda"),
                    kept_count=torch.empty((1, n), dtype=torch.int32, device="cuda"))
    ref = lb.moe_capacity_slots(empty, n, 10, 1, out=outs())
    got = lb.moe_capacity_slots_static(empty, n, 10, 1, out=outs())
    torch.cuda.synchronize()
    lb.sync_status()
    assert torch.equal(got["expert_offsets"], ref["expert_offsets"])
    assert int(got["expert_offsets"].abs().sum().item()) == 0


def test_static_scratch_rejects_invalid_arguments_first(lib):
    # seg_len that does not divide m: the same MOE_ERR_INVALID_ARG as moe_capacity_slots
    fake = torch.empty(16, dtype=torch.int32, device="cuda")
    p = fake.data_ptr()
    rc = lib.moe_capacity_slots_static(p, 10, 1, 4, 2, 3, p, p, p, p, p, p, None)
    assert rc == 1
    assert "seg_len" in lb.last_error()


def test_static_scratch_rejects_problems_larger_than_the_array(lib):
    m, k, n = 1 << 20, 8, 256  # needs ~16 MiB of scratch as one segment
    assert lib.moe_capacity_slots_workspace_size(m, k, n, m) > (1 << 20)
    fake = torch.empty(1, dtype=torch.int32, device="cuda")
    p = fake.data_ptr()
    rc = lib.moe_capacity_slots_static(p, m, k, n, 10, m, p, p, p, p, p, p, None)
    assert rc == 3  # MOE_ERR_WORKSPACE
    assert "fixed" in lb.last_error()
