"""The allocation-free layout entry point, moedisp_moe_dispatch_layout_noalloc.

It serves callers that cannot allocate device memory for a workspace (an allocator that
owns all device memory, a region where allocation is not allowed, a real-time caller
that allocates nothing after start-up): its scratch is an array inside the library's own
device memory. The test calls it through the C ABI, several times in a row with changing
geometry (other experts, tile counts and masks, no tokens at all, a tiny problem, and a
problem whose scratch fills most of the array), and checks every output against both the
regular entry point (with a caller-allocated workspace) and the CPU oracle. A counter or
flag that one call left in the shared array and the next call read would show up as a
mismatch. The file's name makes pytest collect it last.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from tests.gpu_cases import assert_layout_equal

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def md():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import combine_a2a_exchange_b200 as md
    return md


def _outputs(L):
    return {k: getattr(L, k).cpu().numpy() for k in
            ("cnt", "occ", "dst_row", "assist_info", "expert_base", "rank_base", "send_splits")}


def _near_limit_T(md, W, K, E):
    """The largest T (a multiple of 64) whose layout scratch still fits the array."""
    best = 0
    for T in range(64, 1 << 16, 64):
        if md.layout_workspace_size(W, T, K, E) <= md.NOALLOC_SCRATCH_BYTES:
            best = T
    return best


def _check_call(md, name, seed, over):
    w = wl.moe_workload(name, seed=seed, **over)
    ids = torch.from_numpy(w.expert_ids.reshape(-1)).cuda()
    act = None if w.active is None else torch.from_numpy(w.active).cuda()

    ref = md.LayoutBuffers.allocate(w.W, w.T, w.K, w.E)
    st_ref = torch.zeros(1, dtype=torch.int32, device="cuda")
    md.moe_dispatch_layout(ids, act, ref, st_ref)

    got = md.LayoutBuffers.allocate(w.W, w.T, w.K, w.E)
    for t in (got.cnt, got.occ, got.dst_row, got.assist_info, got.expert_base,
              got.rank_base, got.send_splits):
        t.fill_(-7)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    md.moe_dispatch_layout_noalloc(ids, act, got, st)
    torch.cuda.synchronize()

    assert int(st.item()) == 0 and int(st_ref.item()) == 0, (name, over)
    a, b = _outputs(got), _outputs(ref)
    R = int(b["expert_base"][-1])
    for k in ("cnt", "occ", "dst_row", "expert_base", "rank_base", "send_splits"):
        assert np.array_equal(a[k], b[k]), (name, over, k)
    assert np.array_equal(a["assist_info"][:R], b["assist_info"][:R]), (name, over)
    orc = oracle.moe_dispatch_layout(w.W, w.T, w.K, w.E, w.expert_ids, w.active)
    assert orc["flags"] == 0
    assert_layout_equal(a, orc, orc["R"], got.rows_cap)


def test_noalloc_layout_matches_regular_entry_point_and_oracle(md):
    Tn = _near_limit_T(md, 8, 8, 1024)
    assert Tn > 0
    ws = md.layout_workspace_size(8, Tn, 8, 1024)
    assert ws > 0.9 * md.NOALLOC_SCRATCH_BYTES
    calls = [
        ("tiny", 900, dict(W=4, T=1500, K=6, E=24, active_p=0.7)),
        ("tiny", 901, dict(W=8, T=700, K=8, E=64)),                 # other E, other tiling
        ("tiny", 902, dict(W=8, T=0, K=2, E=16)),                   # no tokens
        ("tiny", 903, {}),                                          # the tiny configuration
        ("tiny", 904, dict(W=8, T=Tn, K=8, E=1024)),                # scratch nearly full
        ("tiny", 905, dict(W=3, T=900, K=4, E=12, slot_active_p=0.5)),
    ]
    for name, seed, over in calls:
        _check_call(md, name, seed, over)


def test_noalloc_layout_rejects_oversized_problems(md):
    # E = 1024 experts over 8 ranks with 2^20 slots needs more scratch than the array holds
    W, T, K, E = 8, 16384, 8, 1024
    assert md.layout_workspace_size(W, T, K, E) > md.NOALLOC_SCRATCH_BYTES
    L = md.Layout(1 << 40, 1 << 41, 1 << 42, 1 << 43, 1 << 44, 1 << 45, 1 << 46, W * T * K)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    import ctypes
    rc = md.raw_call("moedisp_moe_dispatch_layout_noalloc", 1 << 47, None, 0, 0, md.Dims(W, T, K, E),
                     ctypes.byref(L), st.data_ptr(), None)
    assert rc == md.MOEDISP_ERR_UNSUPPORTED
