"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI on
seeded inputs and return host copies of every output."""
from __future__ import annotations

import numpy as np
import torch

import workloads as wl


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def bf16_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def bits_host(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def new_status():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def run_layout(md, w: wl.MoEWorkload, rows_cap=None, ids=None, active="default", major_align=0):
    ids = w.expert_ids if ids is None else ids
    act = w.active if isinstance(active, str) else active
    L = md.LayoutBuffers.allocate(w.W, w.T, w.K, w.E, rows_cap=rows_cap, major_align=major_align)
    st = new_status()
    ids_d = dev(ids.reshape(-1).astype(np.int32))
    act_d = None if act is None else dev(act.astype(np.uint8))
    md.moe_dispatch_layout(ids_d, act_d, L, st)
    torch.cuda.synchronize()
    return L, int(st.item())


def layout_host(L) -> dict:
    return dict(cnt=L.cnt.cpu().numpy(), occ=L.occ.cpu().numpy(), dst_row=L.dst_row.cpu().numpy(),
                assist_info=L.assist_info.cpu().numpy(), expert_base=L.expert_base.cpu().numpy(),
                rank_base=L.rank_base.cpu().numpy(), send_splits=L.send_splits.cpu().numpy())


def assert_layout_equal(got: dict, ref: dict, R: int, rows_cap: int):
    for k in ("cnt", "occ", "dst_row", "expert_base", "rank_base", "send_splits"):
        assert np.array_equal(got[k], ref[k]), k
    n = min(R, rows_cap)
    assert np.array_equal(got["assist_info"][:n], ref["assist_info"][:n]), "assist_info"


def alloc_expand(L, H, quant_mode, guard_rows=2):
    """expand_x with guard rows around it (filled with a canary) to catch stray writes."""
    cap = L.rows_cap
    if quant_mode == 0:
        full = torch.full((cap + 2 * guard_rows, H), -12345, dtype=torch.int16, device="cuda")
    else:
        full = torch.full((cap + 2 * guard_rows, H), 0x5A, dtype=torch.uint8, device="cuda")
    scales = torch.full((cap + 2 * guard_rows,), -1.0, dtype=torch.float32, device="cuda")
    return full, scales, guard_rows
