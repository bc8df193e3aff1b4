"""CPU oracle for the EP MoE dispatch / combine path and the all-to-all-v exchange.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU baseline
of ``bench.py`` may call it; the CUDA library never does. The arithmetic lives in
``moe_oracle.c`` (plain C, built with gcc -O2 -ffp-contract=off); this module only
compiles it and marshals numpy arrays through ctypes. It imports nothing from the
CUDA library, and the CUDA library imports nothing from here.

Each function cites the passage it follows in ``moe_oracle.c``. Pins (tests that tie
the oracle to the pages and to mathematics rather than to itself) are in
``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

ORC_CAPACITY = 1
ORC_BAD_EXPERT = 2
ORC_BAD_SPLIT = 8
ORC_BAD_ARG = 16


def build_oracle(force: bool = False) -> str:
    """Compile moe_oracle.c into liboracle.so (next to the source)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= max(
            os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "moe_oracle.h"))):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
           "-Wall", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build_oracle()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i32, i64 = ctypes.c_int, ctypes.c_int64
        L.orc_bf16_from_f32.argtypes = [ctypes.c_float]
        L.orc_bf16_from_f32.restype = ctypes.c_uint16
        L.orc_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.orc_bf16_to_f32.restype = ctypes.c_float
        L.orc_e4m3_from_f32.argtypes = [ctypes.c_float]
        L.orc_e4m3_from_f32.restype = ctypes.c_uint8
        L.orc_e4m3_to_f32.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_to_f32.restype = ctypes.c_float
        L.orc_a2a_exchange_plan.argtypes = [i32, P, P, P, P]
        L.orc_a2a_v.argtypes = [i32, P, i64, P, i64, i64, P, P, P]
        L.orc_moe_dispatch_layout.argtypes = [i32, i32, i32, i32, P, P, i32, i64, i64, P, P, P, P, P,
                                              P, P]
        L.orc_moe_recv_counts.argtypes = [i32, i32, P, i64, i32, P, P]
        L.orc_moe_dispatch.argtypes = [i32, i32, i32, P, P, i64, i32, P, P, P, i32, P]
        L.orc_quant_row.argtypes = [i32, P, i32, P]
        L.orc_quant_row.restype = ctypes.c_float
        L.orc_quant_row_f32.argtypes = [i32, P, i32, P]
        L.orc_quant_row_f32.restype = ctypes.c_float
        L.orc_moe_combine_f64.argtypes = [i32, i32, i32, P, i64, P, P, P]
        L.orc_moe_combine_f32.argtypes = [i32, i32, i32, P, i64, P, P, P]
        L.orc_moe_combine_rmsnorm_f64.argtypes = [i32, i32, i32, P, i64, P, P, P, P, ctypes.c_float, P, P]
        L.orc_moe_combine_rmsnorm_f32.argtypes = [i32, i32, i32, P, i64, P, P, P, P, ctypes.c_float, P, P]
        L.orc_shared_expert_routing.argtypes = [i32, i32, i32, i32, i32, i32, P, P, P, P]
        for f in ("orc_shared_expert_routing", "orc_moe_combine_rmsnorm_f64", "orc_moe_combine_rmsnorm_f32",
                  "orc_a2a_exchange_plan", "orc_a2a_v", "orc_moe_dispatch_layout",
                  "orc_moe_recv_counts", "orc_moe_dispatch", "orc_moe_combine_f64",
                  "orc_moe_combine_f32"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


def _p(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


# ----------------------------------------------------------------- conversions

def bf16_from_f32(v: float) -> int:
    return int(lib().orc_bf16_from_f32(ctypes.c_float(v)))


def bf16_to_f32(b: int) -> float:
    return float(lib().orc_bf16_to_f32(ctypes.c_uint16(b)))


def e4m3_from_f32(v: float) -> int:
    return int(lib().orc_e4m3_from_f32(ctypes.c_float(v)))


def e4m3_to_f32(c: int) -> float:
    return float(lib().orc_e4m3_to_f32(ctypes.c_uint8(c)))


# ------------------------------------------------------------------- O1 / O2

def a2a_exchange_plan(in_splits: np.ndarray):
    """Returns (src_offsets, out_splits, dst_offsets, flags), each [W, W] int64."""
    S = _c(in_splits, np.int64)
    W = S.shape[0]
    src = np.zeros((W, W), np.int64)
    out = np.zeros((W, W), np.int64)
    dst = np.zeros((W, W), np.int64)
    fl = lib().orc_a2a_exchange_plan(W, _p(S), _p(src), _p(out), _p(dst))
    return src, out, dst, fl


def a2a_v(inp: np.ndarray, out: np.ndarray, src_offsets, out_splits, dst_offsets) -> int:
    """inp: [W, in_rows, row_bytes-like]; out: [W, out_cap, ...] (modified in place)."""
    W = inp.shape[0]
    assert out.shape[0] == W and inp.dtype == out.dtype
    row_bytes = int(np.prod(inp.shape[2:])) * inp.itemsize
    assert int(np.prod(out.shape[2:])) * out.itemsize == row_bytes
    so, os_, do = (_c(a, np.int64) for a in (src_offsets, out_splits, dst_offsets))
    return lib().orc_a2a_v(W, _p(inp), inp.shape[1], _p(out), out.shape[1], row_bytes,
                           _p(so), _p(os_), _p(do))


# ----------------------------------------------------------------------- O3

def moe_dispatch_layout(W: int, T: int, K: int, E: int, expert_ids, active=None,
                        rows_cap: int | None = None, major_align: int = 0) -> dict:
    """active: None, a per-token mask [G], or a per-slot mask [G, K] (told apart by size;
    with K = 1 the two readings coincide). major_align >= 2 pads expert segments."""
    ids = _c(expert_ids, np.int32).reshape(-1)
    G = W * T
    assert ids.size == G * K
    act = None if active is None else _c(active, np.uint8).reshape(-1)
    active_dims = 1 if act is None or act.size == G else 2
    assert act is None or act.size == (G if active_dims == 1 else G * K)
    if rows_cap is None:
        A = max(int(major_align), 1)
        rows_cap = G * K + (E * A if A > 1 else 0)
    out = dict(
        cnt=np.zeros((W, E), np.int32),
        occ=np.zeros(G * K, np.int32),
        dst_row=np.zeros(G * K, np.int32),
        assist_info=np.full(max(rows_cap, 1), -1, np.int32),
        expert_base=np.zeros(E + 1, np.int64),
        rank_base=np.zeros(W + 1, np.int64),
        send_splits=np.zeros((W, W), np.int64),
    )
    fl = lib().orc_moe_dispatch_layout(W, T, K, E, _p(ids), _p(act), active_dims, int(major_align),
                                       rows_cap,
                                       _p(out["cnt"]), _p(out["occ"]), _p(out["dst_row"]),
                                       _p(out["assist_info"]), _p(out["expert_base"]),
                                       _p(out["rank_base"]), _p(out["send_splits"]))
    out["flags"] = fl
    out["R"] = int(out["expert_base"][E])
    out["rows_cap"] = rows_cap
    return out


def moe_recv_counts(W: int, E: int, cnt, expert_token_nums_type: int = 1, major_align: int = 0):
    ne = E // W
    c = _c(cnt, np.int32)
    etn = np.zeros((W, ne), np.int64)
    erc = np.zeros((W, ne, W), np.int32)
    fl = lib().orc_moe_recv_counts(W, E, _p(c), int(major_align), expert_token_nums_type,
                                   _p(etn), _p(erc))
    return etn, erc, fl


# ----------------------------------------------------------------------- O4

def quant_row(x_bits_row, quant_mode: int):
    x = _c(x_bits_row, np.uint16)
    q = np.zeros(x.size, np.uint8)
    s = lib().orc_quant_row(x.size, _p(x), quant_mode, _p(q))
    return q, float(np.float32(s))


def quant_row_f32(x_row, quant_mode: int):
    x = _c(x_row, np.float32)
    q = np.zeros(x.size, np.uint8)
    s = lib().orc_quant_row_f32(x.size, _p(x), quant_mode, _p(q))
    return q, float(np.float32(s))


def moe_dispatch(x_bits, dst_row, K: int, rows_cap: int, quant_mode: int = 0,
                 expand_x=None, dynamic_scales=None, smooth=None, expert_ids=None):
    """smooth: per-expert smoothing factors [E, H] fp32 (quantising modes), with the
    routing's expert_ids [G, K]."""
    x = _c(x_bits, np.uint16)
    G, H = x.shape
    dr = _c(dst_row, np.int32).reshape(-1)
    sm = None if smooth is None else _c(smooth, np.float32)
    ids = None if expert_ids is None else _c(expert_ids, np.int32).reshape(-1)
    E = 0 if sm is None else sm.shape[0]
    assert sm is None or (sm.shape == (E, H) and ids is not None and ids.size == G * K)
    if expand_x is None:
        expand_x = (np.zeros((rows_cap, H), np.uint16) if quant_mode == 0
                    else np.zeros((rows_cap, H), np.uint8))
    if dynamic_scales is None and quant_mode != 0:
        dynamic_scales = np.zeros(rows_cap, np.float32)
    fl = lib().orc_moe_dispatch(G, K, H, _p(x), _p(dr), rows_cap, quant_mode,
                                _p(expand_x), _p(dynamic_scales), _p(sm), E, _p(ids))
    return expand_x, dynamic_scales, fl


# ----------------------------------------------------------------------- O5

def moe_combine_f64(expert_out_bits, dst_row, weights, K: int, rows_cap: int | None = None):
    eo = _c(expert_out_bits, np.uint16)
    dr = _c(dst_row, np.int32).reshape(-1)
    w = _c(weights, np.float32).reshape(-1)
    G = dr.size // K
    H = eo.shape[1]
    if rows_cap is None:
        rows_cap = eo.shape[0]
    y = np.zeros((G, H), np.float64)
    fl = lib().orc_moe_combine_f64(G, K, H, _p(eo), rows_cap, _p(dr), _p(w), _p(y))
    return y, fl


def moe_combine_f32(expert_out_bits, dst_row, weights, K: int, rows_cap: int | None = None):
    eo = _c(expert_out_bits, np.uint16)
    dr = _c(dst_row, np.int32).reshape(-1)
    w = _c(weights, np.float32).reshape(-1)
    G = dr.size // K
    H = eo.shape[1]
    if rows_cap is None:
        rows_cap = eo.shape[0]
    y = np.zeros((G, H), np.uint16)
    fl = lib().orc_moe_combine_f32(G, K, H, _p(eo), rows_cap, _p(dr), _p(w), _p(y))
    return y, fl


# ------------------------------------------------------------- fused tail

def moe_combine_rmsnorm(expert_out_bits, dst_row, weights, K: int, residual_bits, gamma,
                        eps: float, rows_cap: int | None = None, exact: str = "f64"):
    """Returns (residual_out bf16 bits, y) with y fp64 (exact='f64') or bf16 bits ('f32')."""
    eo = _c(expert_out_bits, np.uint16)
    dr = _c(dst_row, np.int32).reshape(-1)
    w = _c(weights, np.float32).reshape(-1)
    res = _c(residual_bits, np.uint16)
    gm = _c(gamma, np.float32)
    G = dr.size // K
    H = res.shape[1]
    if rows_cap is None:
        rows_cap = eo.shape[0]
    rout = np.zeros((G, H), np.uint16)
    if exact == "f64":
        y = np.zeros((G, H), np.float64)
        fl = lib().orc_moe_combine_rmsnorm_f64(G, K, H, _p(eo), rows_cap, _p(dr), _p(w), _p(res),
                                               _p(gm), eps, _p(rout), _p(y))
    else:
        y = np.zeros((G, H), np.uint16)
        fl = lib().orc_moe_combine_rmsnorm_f32(G, K, H, _p(eo), rows_cap, _p(dr), _p(w), _p(res),
                                               _p(gm), eps, _p(rout), _p(y))
    return rout, y, fl


# ------------------------------------------------------------ shared experts

def shared_expert_routing(W: int, T: int, K: int, E: int, N: int, S: int, expert_ids, weights):
    """Returns (ext_ids [G, K+N] int32, ext_w [G, K+N] fp32, E_total, flags)."""
    ids = _c(expert_ids, np.int32).reshape(-1)
    w = _c(weights, np.float32).reshape(-1)
    G = W * T
    ext_ids = np.zeros((G, K + N), np.int32)
    ext_w = np.zeros((G, K + N), np.float32)
    fl = lib().orc_shared_expert_routing(W, T, K, E, N, S, _p(ids), _p(w), _p(ext_ids), _p(ext_w))
    E_total = W * (E // (W - S)) if 0 <= S < W and E % (W - S) == 0 else 0
    return ext_ids, ext_w, E_total, fl
