"""Host-side tests of the C ABI: the library loads without a GPU, exports every function
include/*.h declares, and rejects bad arguments before touching the GPU (so these run on
a CPU-only machine; the pointers below are never dereferenced)."""
import ctypes
import glob
import os
import re
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="session")
def md():
    import __graft_entry__
    __graft_entry__.build()
    import combine_a2a_exchange_b200 as md
    return md


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"\b(moedisp_\w+)\s*\(", text):
            names.add(m.group(1))
    return sorted(names)


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("moedisp_a2a_exchange_plan", "moedisp_a2a_v", "moedisp_moe_dispatch_layout",
                     "moedisp_moe_dispatch", "moedisp_moe_combine", "moedisp_moe_combine_rmsnorm",
                     "moedisp_layout_workspace_size", "moedisp_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(md):
    lib = ctypes.CDLL(md.LIBRARY_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", md.LIBRARY_PATH], capture_output=True,
                         text=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    assert set(declared_functions()) <= exported


def test_status_strings(md):
    assert md.version() == 3
    assert md.status_string(0) == "ok"
    assert md.status_string(-1) == "null pointer"
    assert md.status_string(md.STATUS_CAPACITY | md.STATUS_TIMEOUT) == "capacity | timeout"
    assert md.status_string(12345) == "unknown code"


FAKE = 0x7f0000000000          # 16-byte aligned, never dereferenced on the host paths


def test_plan_rejections(md):
    call = lambda *a: md.raw_call("moedisp_a2a_exchange_plan", *a)
    ok = [FAKE, 4, FAKE + 0x1000, FAKE + 0x2000, FAKE + 0x3000, FAKE + 0x4000, None]
    a = list(ok); a[0] = None
    assert call(*a) == md.MOEDISP_ERR_NULLPTR
    a = list(ok); a[5] = None
    assert call(*a) == md.MOEDISP_ERR_NULLPTR
    a = list(ok); a[1] = 0
    assert call(*a) == md.MOEDISP_ERR_INVALID
    a = list(ok); a[1] = 70000
    assert call(*a) == md.MOEDISP_ERR_UNSUPPORTED
    a = list(ok); a[2] = FAKE + 0x1004
    assert call(*a) == md.MOEDISP_ERR_MISALIGNED
    a = list(ok); a[3] = FAKE + 0x1008          # out_splits overlaps src_offsets
    assert call(*a) == md.MOEDISP_ERR_ALIASED
    a = list(ok); a[2] = FAKE + 0x10            # src_offsets overlaps in_splits
    assert call(*a) == md.MOEDISP_ERR_ALIASED


def test_a2a_v_rejections(md):
    call = lambda *a: md.raw_call("moedisp_a2a_v", *a)
    # in, stride, out, cap, row_bytes, W, src, splits, dst, status, stream
    ok = [FAKE, 10, FAKE + (1 << 30), 10, 64, 2, FAKE + (2 << 30), FAKE + (2 << 30) + 64,
          FAKE + (2 << 30) + 128, FAKE + (2 << 30) + 256, None]
    a = list(ok); a[4] = 24
    assert call(*a) == md.MOEDISP_ERR_MISALIGNED
    a = list(ok); a[0] = FAKE + 8
    assert call(*a) == md.MOEDISP_ERR_MISALIGNED
    a = list(ok); a[4] = 0
    assert call(*a) == md.MOEDISP_ERR_INVALID
    a = list(ok); a[1] = -1
    assert call(*a) == md.MOEDISP_ERR_INVALID
    a = list(ok); a[0] = None
    assert call(*a) == md.MOEDISP_ERR_NULLPTR
    a = list(ok); a[2] = FAKE + 640            # out overlaps in (2 ranks x 10 rows x 64 B)
    assert call(*a) == md.MOEDISP_ERR_ALIASED
    a = list(ok); a[7] = None
    assert call(*a) == md.MOEDISP_ERR_NULLPTR


def _layout(md, base=FAKE, rows_cap=64):
    step = 1 << 20
    return md.Layout(base, base + step, base + 2 * step, base + 3 * step, base + 4 * step,
                     base + 5 * step, base + 6 * step, rows_cap)


def test_layout_rejections(md):
    ws_ok = md.layout_workspace_size(4, 8, 2, 8)
    assert ws_ok > 0
    with pytest.raises(md.MoedispError):
        md.layout_workspace_size(3, 8, 2, 8)                 # E % W != 0
    with pytest.raises(md.MoedispError):
        md.layout_workspace_size(4, 8, 17, 8)                # K > 16
    L = _layout(md)
    call = lambda ids, dims, L, ws, nws, st, act=None, ad=0, al=0: md.raw_call(
        "moedisp_moe_dispatch_layout", ids, act, ad, al, dims, ctypes.byref(L), ws, nws, st, None)
    ids, ws, st = FAKE + (64 << 20), FAKE + (128 << 20), FAKE + (256 << 20)
    d = md.Dims(4, 8, 2, 8)
    assert call(ids, d, L, ws, ws_ok - 1, st) == md.MOEDISP_ERR_WORKSPACE
    assert call(ids, d, L, None, ws_ok, st) == md.MOEDISP_ERR_WORKSPACE
    assert call(None, d, L, ws, ws_ok, st) == md.MOEDISP_ERR_NULLPTR
    assert call(ids, md.Dims(4, 8, 0, 8), L, ws, ws_ok, st) == md.MOEDISP_ERR_INVALID
    assert call(ids, md.Dims(4, 8, 2, 2048), L, ws, ws_ok, st) == md.MOEDISP_ERR_UNSUPPORTED
    assert call(ids, md.Dims(4, 1 << 28, 2, 8), L, ws, ws_ok, st) == md.MOEDISP_ERR_UNSUPPORTED
    assert call(ids + 2, d, L, ws, ws_ok, st) == md.MOEDISP_ERR_MISALIGNED
    bad = _layout(md); bad.dst_row = bad.occ + 16       # dst_row overlaps occ
    assert call(ids, d, bad, ws, ws_ok, st) == md.MOEDISP_ERR_ALIASED
    bad = _layout(md, rows_cap=-1)
    assert call(ids, d, bad, ws, ws_ok, st) == md.MOEDISP_ERR_INVALID
    assert call(ids, d, L, L.cnt, ws_ok, st) == md.MOEDISP_ERR_ALIASED   # workspace over cnt
    act = FAKE + (300 << 20)
    assert call(ids, d, L, ws, ws_ok, st, act, 0) == md.MOEDISP_ERR_INVALID    # mask dims
    assert call(ids, d, L, ws, ws_ok, st, act, 3) == md.MOEDISP_ERR_INVALID
    assert call(ids, d, L, ws, ws_ok, st, al=-1) == md.MOEDISP_ERR_INVALID        # major_align
    assert call(ids, d, L, ws, ws_ok, st, al=(1 << 16) + 1) == md.MOEDISP_ERR_UNSUPPORTED
    # a per-slot mask [G][K] spans G*K bytes: one starting G*K - 1 bytes before occ overlaps it
    G, K = 4 * 8, 2
    assert call(ids, d, L, ws, ws_ok, st, L.occ - (G * K - 1), 2) == md.MOEDISP_ERR_ALIASED


def test_dispatch_and_combine_rejections(md):
    L = _layout(md)
    d = md.Dims(4, 8, 2, 8)
    x, ex, sc, st = FAKE + (64 << 20), FAKE + (128 << 20), FAKE + (192 << 20), FAKE + (256 << 20)
    disp = lambda x, H, q, ex, sc, st, etn=None, t=1, sm=None, lay=None: md.raw_call(
        "moedisp_moe_dispatch", x, H, d, ctypes.byref(lay or L), q, sm, ex, sc, etn, t, None, st, None)
    assert disp(x, 128, 1, ex, sc, st) == md.MOEDISP_ERR_INVALID           # quant mode
    assert disp(x, 120, 2, ex, sc, st) == md.MOEDISP_ERR_MISALIGNED        # H % 16 (quant)
    assert disp(x, 124, 0, ex, sc, st) == md.MOEDISP_ERR_MISALIGNED        # H % 8
    assert disp(x, 32768, 0, ex, sc, st) == md.MOEDISP_ERR_UNSUPPORTED
    assert disp(x, 128, 2, ex, None, st) == md.MOEDISP_ERR_NULLPTR          # scales needed
    assert disp(None, 128, 0, ex, None, st) == md.MOEDISP_ERR_NULLPTR
    assert disp(x, 128, 0, x + 256, None, st) == md.MOEDISP_ERR_ALIASED     # out over x
    assert disp(x + 8, 128, 0, ex, None, st) == md.MOEDISP_ERR_MISALIGNED
    assert disp(x, 128, 0, ex, None, None) == md.MOEDISP_ERR_NULLPTR
    assert disp(x, 128, 0, ex, None, st, etn=FAKE + (300 << 20), t=5) == md.MOEDISP_ERR_INVALID
    sm = FAKE + (320 << 20)
    assert disp(x, 128, 0, ex, None, st, sm=sm) == md.MOEDISP_ERR_INVALID   # smoothing, no quant
    assert disp(x, 128, 2, ex, sc, st, sm=sm + 4) == md.MOEDISP_ERR_MISALIGNED
    assert disp(x, 128, 2, sm + 256, sc, st, sm=sm) == md.MOEDISP_ERR_ALIASED  # out over smooth
    noassist = _layout(md); noassist.assist_info = None
    assert disp(x, 128, 2, ex, sc, st, sm=sm, lay=noassist) == md.MOEDISP_ERR_NULLPTR
    comb = lambda eo, H, w, y, st: md.raw_call(
        "moedisp_moe_combine", eo, H, d, ctypes.byref(L), w, y, st, None)
    assert comb(ex, 100, x, sc, st) == md.MOEDISP_ERR_MISALIGNED
    assert comb(ex, 0, x, sc, st) == md.MOEDISP_ERR_INVALID
    assert comb(ex, 128, None, sc, st) == md.MOEDISP_ERR_NULLPTR
    assert comb(ex, 128, x, ex + 512, st) == md.MOEDISP_ERR_ALIASED        # y over expert_out
    assert comb(ex + 4, 128, x, sc, st) == md.MOEDISP_ERR_MISALIGNED
    # no tokens: a valid no-op that launches nothing
    assert md.raw_call("moedisp_moe_combine", None, 128, md.Dims(4, 0, 2, 8), ctypes.byref(L),
                       None, None, st, None) == md.MOEDISP_OK
    res, gm, ro = FAKE + (320 << 20), FAKE + (384 << 20), FAKE + (448 << 20)
    rms = lambda eo, H, res, gm, eps, ro, y, st: md.raw_call(
        "moedisp_moe_combine_rmsnorm", eo, H, d, ctypes.byref(L), x, res, gm, eps, ro, y, st, None)
    assert rms(ex, 100, res, gm, 1e-6, ro, sc, st) == md.MOEDISP_ERR_MISALIGNED   # H % 8
    assert rms(ex, 128, res, gm, -1.0, ro, sc, st) == md.MOEDISP_ERR_INVALID      # eps < 0
    assert rms(ex, 128, res, gm, float("nan"), ro, sc, st) == md.MOEDISP_ERR_INVALID
    assert rms(ex, 32768, res, gm, 1e-6, ro, sc, st) == md.MOEDISP_ERR_UNSUPPORTED
    assert rms(ex, 128, None, gm, 1e-6, ro, sc, st) == md.MOEDISP_ERR_NULLPTR
    assert rms(ex, 128, res, None, 1e-6, ro, sc, st) == md.MOEDISP_ERR_NULLPTR
    assert rms(ex, 128, res, gm + 4, 1e-6, ro, sc, st) == md.MOEDISP_ERR_MISALIGNED
    assert rms(ex, 128, res, gm, 1e-6, ro + 8, sc, st) == md.MOEDISP_ERR_MISALIGNED
    assert rms(ex, 128, res, gm, 1e-6, res + 512, sc, st) == md.MOEDISP_ERR_ALIASED  # rout over residual
    assert rms(ex, 128, res, gm, 1e-6, ro, ro + 1024, st) == md.MOEDISP_ERR_ALIASED  # y over rout
    assert rms(ex, 128, res, gm, 1e-6, ro, gm, st) == md.MOEDISP_ERR_ALIASED         # y over gamma
    assert rms(ex, 128, res, gm, 1e-6, ro, sc, None) == md.MOEDISP_ERR_NULLPTR
    assert md.raw_call("moedisp_moe_combine_rmsnorm", None, 128, md.Dims(4, 0, 2, 8),
                       ctypes.byref(L), None, None, None, 1e-6, None, None, st, None) == md.MOEDISP_OK


def test_selftest_rejections(md):
    assert md.raw_selftest(10, None) == md.MOEDISP_ERR_NULLPTR
    assert md.raw_selftest(0, FAKE) == md.MOEDISP_ERR_INVALID
    assert md.raw_selftest(10, FAKE + 2) == md.MOEDISP_ERR_MISALIGNED


def test_binding_has_no_fallback():
    """The package refuses to import without the compiled library."""
    src = open(os.path.join(ROOT, "combine_a2a_exchange_b200", "__init__.py")).read()
    assert "raise ImportError" in src
    for f in glob.glob(os.path.join(ROOT, "combine_a2a_exchange_b200", "**", "*.py"), recursive=True):
        text = open(f).read()
        assert "import oracle" not in text and "from oracle" not in text, f


def test_shared_expert_routing_rejections(md):
    ids, w, eo, ew, st = (FAKE + (i << 20) for i in (64, 128, 192, 256, 320))
    call = lambda W, T, K, E, N, S, ids=ids, w=w, eo=eo, ew=ew, st=st: md.raw_call(
        "moedisp_shared_expert_routing", ids, w, W, T, K, E, N, S, eo, ew, st, None)
    assert call(8, 4, 2, 64, 1, 0) == md.MOEDISP_ERR_INVALID        # N without shared ranks
    assert call(8, 4, 2, 64, 0, 4) == md.MOEDISP_ERR_INVALID        # shared ranks, N = 0
    assert call(8, 4, 2, 64, 3, 4) == md.MOEDISP_ERR_INVALID        # S % N
    assert call(8, 4, 2, 64, 1, 3) == md.MOEDISP_ERR_INVALID        # W % S
    assert call(8, 4, 2, 62, 1, 4) == md.MOEDISP_ERR_INVALID        # E % (W - S)
    assert call(8, 4, 2, 64, 1, 8) == md.MOEDISP_ERR_INVALID        # S < W
    assert call(8, 4, 16, 64, 1, 4) == md.MOEDISP_ERR_UNSUPPORTED   # K + N > 16
    assert call(8, 4, 2, 1024, 1, 4) == md.MOEDISP_ERR_UNSUPPORTED  # W * ne > 1024
    assert call(8, 4, 2, 64, 1, 4, ids=None) == md.MOEDISP_ERR_NULLPTR
    assert call(8, 4, 2, 64, 1, 4, st=None) == md.MOEDISP_ERR_NULLPTR
    assert call(8, 4, 2, 64, 1, 4, eo=ids + 64) == md.MOEDISP_ERR_ALIASED
    assert call(8, 4, 2, 64, 1, 4, ew=eo + 4) == md.MOEDISP_ERR_ALIASED   # outputs overlap
    assert call(8, 4, 2, 64, 1, 4, eo=eo + 2) == md.MOEDISP_ERR_MISALIGNED
    assert call(8, 0, 2, 64, 1, 4, ids=None, w=None, eo=None, ew=None) == md.MOEDISP_OK


def test_gather_and_token_rows_rejections(md):
    L = _layout(md)
    d = md.Dims(4, 8, 2, 8)
    x, rows, ex, sc, st = (FAKE + (i << 20) for i in (64, 96, 128, 192, 256))
    g = lambda x, xr, rows, st=st: md.raw_call(
        "moedisp_moe_dispatch_gather", x, xr, rows, 128, d, ctypes.byref(L), 0, None, ex, None,
        None, 1, None, st, None)
    assert g(x, 100, None) == md.MOEDISP_ERR_NULLPTR                 # no token map
    assert g(x, -1, rows) == md.MOEDISP_ERR_INVALID                  # x_rows < 0
    assert g(x, 100, rows + 4) == md.MOEDISP_ERR_MISALIGNED
    assert g(x, 100, ex + 64) == md.MOEDISP_ERR_ALIASED              # map inside expand_x
    assert g(x, 1 << 20, rows) == md.MOEDISP_ERR_ALIASED             # x reaches expand_x
    so, os_, do, tr, act = (FAKE + (i << 20) for i in (300, 320, 340, 360, 380))
    t = lambda W, T, stride, so=so, tr=tr, act=act, st=st: md.raw_call(
        "moedisp_a2a_token_rows", so, os_, do, W, T, stride, tr, act, st, None)
    assert t(0, 4, 10) == md.MOEDISP_ERR_INVALID
    assert t(4, -1, 10) == md.MOEDISP_ERR_INVALID
    assert t(4, 4, -1) == md.MOEDISP_ERR_INVALID
    assert t(4, 4, 10, so=None) == md.MOEDISP_ERR_NULLPTR
    assert t(4, 4, 10, st=None) == md.MOEDISP_ERR_NULLPTR
    assert t(4, 4, 10, tr=tr + 4) == md.MOEDISP_ERR_MISALIGNED
    assert t(4, 4, 10, tr=so) == md.MOEDISP_ERR_ALIASED
    assert t(4, 4, 10, act=do + 8) == md.MOEDISP_ERR_ALIASED
    assert t(4, 0, 10, so=None, tr=None) == md.MOEDISP_OK


def test_peers_rejections(md):
    L = _layout(md)
    d = md.Dims(4, 8, 2, 8)
    x, ids, tab, stab, st, y, w = (FAKE + (i << 20) for i in (64, 96, 128, 160, 256, 300, 340))
    disp = lambda rank, q, tab=tab, stab=stab, st=st, H=128: md.raw_call(
        "moedisp_moe_dispatch_peers", x, H, d, rank, ids, ctypes.byref(L), q, tab, stab, 100, st, None)
    assert disp(4, 0) == md.MOEDISP_ERR_INVALID                   # rank >= W
    assert disp(-1, 0) == md.MOEDISP_ERR_INVALID
    assert disp(0, 1) == md.MOEDISP_ERR_INVALID                   # quant mode
    assert disp(0, 0, tab=None) == md.MOEDISP_ERR_NULLPTR
    assert disp(0, 2, stab=None) == md.MOEDISP_ERR_NULLPTR        # scales table for quant
    assert disp(0, 0, tab=tab + 4) == md.MOEDISP_ERR_MISALIGNED
    assert disp(0, 0, st=None) == md.MOEDISP_ERR_NULLPTR
    assert disp(0, 2, H=136) == md.MOEDISP_ERR_MISALIGNED
    comb = lambda rank, y=y, tab=tab: md.raw_call(
        "moedisp_moe_combine_peers", tab, 100, 128, d, rank, ids, ctypes.byref(L), w, y, st, None)
    assert comb(4) == md.MOEDISP_ERR_INVALID
    assert comb(0, tab=None) == md.MOEDISP_ERR_NULLPTR
    assert comb(0, y=y + 8) == md.MOEDISP_ERR_MISALIGNED
    assert comb(0, y=w) == md.MOEDISP_ERR_ALIASED                 # y over the weights


def test_binding_host_logic(md):
    """Argument marshalling that happens in Python: the active mask's form is read from
    its shape, and the default capacity covers major_align padding."""
    import torch
    d = md.Dims(4, 8, 3, 8)
    assert md._mask_dims(None, d, None) == 0
    assert md._mask_dims(torch.zeros(32, dtype=torch.uint8), d, None) == 1
    assert md._mask_dims(torch.zeros(32, 3, dtype=torch.uint8), d, None) == 2
    assert md._mask_dims(torch.zeros(96, dtype=torch.uint8), d, None) == 2      # flat [G*K]
    assert md._mask_dims(torch.zeros(32, dtype=torch.uint8), md.Dims(4, 8, 1, 8), None) == 1
    assert md._mask_dims(torch.zeros(32, dtype=torch.uint8), d, 2) == 2          # explicit
    with pytest.raises(ValueError):
        md._mask_dims(FAKE, d, None)                                           # raw pointer
    L = md.LayoutBuffers.allocate(4, 8, 3, 8, device="cpu")
    assert L.rows_cap == 4 * 8 * 3 and L.major_align == 0
    L = md.LayoutBuffers.allocate(4, 8, 3, 8, device="cpu", major_align=16)
    assert L.rows_cap == 4 * 8 * 3 + 8 * 16 and L.assist_info.numel() == L.rows_cap
    L = md.LayoutBuffers.allocate(4, 8, 3, 8, device="cpu", major_align=1)
    assert L.rows_cap == 4 * 8 * 3


def test_ep_barrier_rejections(md):
    tab, st = FAKE + (1 << 20), FAKE + (2 << 20)
    b = lambda tab=tab, W=2, rank=0, to=1000, st=st, ep=1: md.raw_call(
        "moedisp_ep_barrier", tab, W, rank, ep, to, st, None)
    assert b(tab=None) == md.MOEDISP_ERR_NULLPTR
    assert b(ep=0) == md.MOEDISP_ERR_INVALID                   # zeroed words would pass
    assert b(st=None) == md.MOEDISP_ERR_NULLPTR
    assert b(W=0) == md.MOEDISP_ERR_INVALID
    assert b(rank=2) == md.MOEDISP_ERR_INVALID
    assert b(rank=-1) == md.MOEDISP_ERR_INVALID
    assert b(to=0) == md.MOEDISP_ERR_INVALID                   # no limit is not allowed
    assert b(to=10000001) == md.MOEDISP_ERR_INVALID
    assert b(W=70000, rank=1) == md.MOEDISP_ERR_UNSUPPORTED
    assert b(tab=tab + 4) == md.MOEDISP_ERR_MISALIGNED
    assert b(st=st + 2) == md.MOEDISP_ERR_MISALIGNED


def test_pipelined_rejections(md):
    L = _layout(md)
    d = md.Dims(4, 8, 2, 8)
    ws_need = md.a2a_dispatch_pipelined_workspace_size(4)
    assert ws_need > 0
    inp, so, os_, do, recv, ex, sc, ready, ws, st = (FAKE + (i << 20) for i in range(64, 74))

    def p(inp=inp, stride=10, so=so, recv=recv, H=128, d=d, q=0, ex=ex, sc=None, ready=ready,
          roles=3, lim=1000, ws=ws, wsb=ws_need, st=st, ep=1):
        return md.raw_call("moedisp_a2a_dispatch_pipelined", inp, stride, so, os_, do, recv, H, d,
                           ctypes.byref(L), q, ex, sc, None, 1, None, ready, ep, roles, lim, ws,
                           wsb, st, None)
    assert p(ep=0) == md.MOEDISP_ERR_INVALID                   # zeroed words would read as published
    assert p(st=None) == md.MOEDISP_ERR_NULLPTR
    assert p(ready=None) == md.MOEDISP_ERR_NULLPTR
    assert p(ws=None) == md.MOEDISP_ERR_NULLPTR
    assert p(so=None) == md.MOEDISP_ERR_NULLPTR
    assert p(recv=None) == md.MOEDISP_ERR_NULLPTR
    assert p(inp=None) == md.MOEDISP_ERR_NULLPTR
    assert p(q=2) == md.MOEDISP_ERR_NULLPTR                    # quantising without scales
    assert p(roles=0) == md.MOEDISP_ERR_INVALID
    assert p(roles=4) == md.MOEDISP_ERR_INVALID
    assert p(lim=0) == md.MOEDISP_ERR_INVALID
    assert p(stride=-1) == md.MOEDISP_ERR_INVALID
    assert p(q=1) == md.MOEDISP_ERR_INVALID
    assert p(H=100) == md.MOEDISP_ERR_MISALIGNED
    assert p(H=136, q=3, sc=sc) == md.MOEDISP_ERR_MISALIGNED   # quantised rows need H % 16
    assert p(H=32768) == md.MOEDISP_ERR_UNSUPPORTED
    assert p(wsb=ws_need - 1) == md.MOEDISP_ERR_WORKSPACE
    assert p(recv=recv + 8) == md.MOEDISP_ERR_MISALIGNED
    assert p(ws=ws + 8) == md.MOEDISP_ERR_MISALIGNED
    assert p(recv=inp) == md.MOEDISP_ERR_ALIASED              # receive buffer over the send rows
    assert p(ready=ex) == md.MOEDISP_ERR_ALIASED              # ready words inside expand_x
    assert p(d=md.Dims(4, 0, 2, 8), so=None) == md.MOEDISP_OK  # no positions, no plan


def test_ipc_rejections(md):
    h = ctypes.create_string_buffer(64)
    off = ctypes.c_int64(0)
    p = ctypes.c_void_p(0)
    lib = ctypes.CDLL(md.LIBRARY_PATH)
    lib.moedisp_ipc_export.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(ctypes.c_int64)]
    lib.moedisp_ipc_import.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.POINTER(ctypes.c_void_p)]
    lib.moedisp_ipc_close.argtypes = [ctypes.c_void_p]
    assert lib.moedisp_ipc_export(None, h, ctypes.byref(off)) == md.MOEDISP_ERR_NULLPTR
    assert lib.moedisp_ipc_export(FAKE, None, ctypes.byref(off)) == md.MOEDISP_ERR_NULLPTR
    assert lib.moedisp_ipc_export(FAKE, h, None) == md.MOEDISP_ERR_NULLPTR
    assert lib.moedisp_ipc_import(None, 0, ctypes.byref(p)) == md.MOEDISP_ERR_NULLPTR
    assert lib.moedisp_ipc_import(h, 0, None) == md.MOEDISP_ERR_NULLPTR
    assert lib.moedisp_ipc_import(h, -1, ctypes.byref(p)) == md.MOEDISP_ERR_INVALID
    assert lib.moedisp_ipc_close(None) == md.MOEDISP_ERR_NULLPTR
    assert lib.moedisp_ipc_close(FAKE) == md.MOEDISP_ERR_INVALID       # never imported


def test_slot_division_by_k_multiply_shift():
    """The smoothing dispatch divides a slot (< 2^30) by K (<= 16) as (slot * ceil(2^34 / K))
    >> 34: with M = 2^34 / K + e (0 <= e < 1) the quotient is slot / K + slot * e / 2^34, whose
    excess stays below 2^-4 <= 1 / K, so the floor is exact. Every K, both ends of the slot
    range and a seeded sample between them."""
    rng = np.random.default_rng(5)
    slots = np.concatenate([np.arange(0, 4096), (1 << 30) - 1 - np.arange(0, 4096),
                            rng.integers(0, 1 << 30, 50000)]).astype(object)
    for K in range(1, 17):
        M = ((1 << 34) + K - 1) // K
        assert all((int(s) * M) >> 34 == int(s) // K for s in slots), K


def test_window_quantisation_brackets_the_ieee_quotient():
    """The quantisers' window: with inv = RN(1/scale), lo = RN(inv * RN(1 - 2^-22)) and
    hi = RN(inv * RN(1 + 2^-22)) in fp32, the exact products x*lo and x*hi must bracket the
    IEEE quotient RN(x/scale) for every normal scale: lo < (1/scale)(1 - 2^-24) and
    hi > (1/scale)(1 + 2^-24), which the quotient's own rounding (|RN(q) - q| <= q 2^-24)
    cannot cross. Checked in exact rational arithmetic on seeded scales spanning the normal
    range (both ends included) and on mantissas next to powers of two."""
    from fractions import Fraction
    rng = np.random.default_rng(11)
    f32 = np.float32
    one_m, one_p = f32(1 - 2.0 ** -22), f32(1 + 2.0 ** -22)
    assert Fraction(float(one_m)) == 1 - Fraction(1, 2 ** 22)
    assert Fraction(float(one_p)) == 1 + Fraction(1, 2 ** 22)
    exps = rng.integers(-126, 122, 3000)
    mant = rng.random(3000) + 1.0
    scales = np.concatenate([(mant * 2.0 ** exps).astype(f32),
                             np.array([np.finfo(f32).tiny, f32(2.0 ** 121), f32(1.0), f32(1.5),
                                       np.nextafter(f32(1.0), f32(2.0)), np.nextafter(f32(2.0), f32(1.0))],
                                      f32)])
    eps = Fraction(1, 2 ** 24)
    for sc in scales:
        assert np.isfinite(sc) and sc >= np.finfo(f32).tiny
        inv = f32(1.0) / sc                                   # IEEE round to nearest
        lo, hi = inv * one_m, inv * one_p
        q = 1 / Fraction(float(sc))
        assert Fraction(float(lo)) < q * (1 - eps), sc
        assert Fraction(float(hi)) > q * (1 + eps), sc
