"""Python binding of libmoedisp: EP MoE dispatch / combine and the all-to-all-v exchange
on NVIDIA B200 (sm_100a).

This module only marshals arguments: torch tensors (device memory allocated by torch)
become raw pointers, the current torch CUDA stream becomes the cudaStream_t, and every
step of the path runs in the CUDA kernels of ``libmoedisp.so``. The functions carry the
names of the C ABI (``include/moedisp.h``) without its ``moedisp_`` prefix. There is no
CPU fallback: importing this package fails if the library has not been built.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

_HERE = os.path.dirname(os.path.abspath(__file__))
LIBRARY_PATH = os.path.join(_HERE, "libmoedisp.so")

if not os.path.exists(LIBRARY_PATH):
    raise ImportError(
        f"{LIBRARY_PATH} is missing: build it with `python combine_a2a_exchange_b200/_build.py` "
        "(or __graft_entry__.build()); this package has no fallback implementation")

_lib = ctypes.CDLL(LIBRARY_PATH)

MOEDISP_OK = 0
MOEDISP_ERR_NULLPTR = -1
MOEDISP_ERR_INVALID = -2
MOEDISP_ERR_MISALIGNED = -3
MOEDISP_ERR_ALIASED = -4
MOEDISP_ERR_UNSUPPORTED = -5
MOEDISP_ERR_WORKSPACE = -6
MOEDISP_ERR_CUDA = -7

STATUS_CAPACITY = 1
STATUS_BAD_EXPERT_ID = 2
STATUS_TIMEOUT = 4
STATUS_BAD_SPLIT = 8

NOALLOC_SCRATCH_BYTES = 2 << 20

QUANT_NONE = 0
QUANT_INT8 = 2
QUANT_FP8_E4M3 = 3

_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64


class Dims(ctypes.Structure):
    _fields_ = [("W", _I), ("T", _I), ("K", _I), ("E", _I)]


class Layout(ctypes.Structure):
    _fields_ = [("cnt", _P), ("occ", _P), ("dst_row", _P), ("assist_info", _P),
                ("expert_base", _P), ("rank_base", _P), ("send_splits", _P),
                ("rows_cap", _I64)]


def _sig(name, argtypes, restype=ctypes.c_int):
    f = getattr(_lib, name)
    f.argtypes = argtypes
    f.restype = restype
    return f


_status_string = _sig("moedisp_status_string", [_I], ctypes.c_char_p)
_version = _sig("moedisp_version", [])
_selftest_wait = _sig("moedisp_selftest_bounded_wait", [ctypes.c_uint32, _P, _P])
_plan = _sig("moedisp_a2a_exchange_plan", [_P, _I, _P, _P, _P, _P, _P])
_a2a_v = _sig("moedisp_a2a_v", [_P, _I64, _P, _I64, _I64, _I, _P, _P, _P, _P, _P])
_ws_size = _sig("moedisp_layout_workspace_size", [Dims, ctypes.POINTER(ctypes.c_size_t)])
_layout = _sig("moedisp_moe_dispatch_layout",
               [_P, _P, _I, _I, Dims, ctypes.POINTER(Layout), _P, ctypes.c_size_t, _P, _P])
_layout_noalloc = _sig("moedisp_moe_dispatch_layout_noalloc",
                       [_P, _P, _I, _I, Dims, ctypes.POINTER(Layout), _P, _P])
_dispatch = _sig("moedisp_moe_dispatch",
                 [_P, _I, Dims, ctypes.POINTER(Layout), _I, _P, _P, _P, _P, _I, _P, _P, _P])
_combine = _sig("moedisp_moe_combine", [_P, _I, Dims, ctypes.POINTER(Layout), _P, _P, _P, _P])
_dispatch_gather = _sig("moedisp_moe_dispatch_gather",
                        [_P, ctypes.c_int64, _P, _I, Dims, ctypes.POINTER(Layout), _I, _P, _P, _P,
                         _P, _I, _P, _P, _P])
_token_rows = _sig("moedisp_a2a_token_rows",
                   [_P, _P, _P, _I, ctypes.c_int64, ctypes.c_int64, _P, _P, _P, _P])
_dispatch_peers = _sig("moedisp_moe_dispatch_peers",
                       [_P, _I, Dims, _I, _P, ctypes.POINTER(Layout), _I, _P, _P, ctypes.c_int64,
                        _P, _P])
_combine_peers = _sig("moedisp_moe_combine_peers",
                      [_P, ctypes.c_int64, _I, Dims, _I, _P, ctypes.POINTER(Layout), _P, _P, _P,
                       _P])
_pipe_ws = _sig("moedisp_a2a_dispatch_pipelined_workspace_size", [_I, ctypes.POINTER(ctypes.c_size_t)])
_pipe = _sig("moedisp_a2a_dispatch_pipelined",
             [_P, _I64, _P, _P, _P, _P, _I, Dims, ctypes.POINTER(Layout), _I, _P, _P, _P, _I, _P,
              _P, ctypes.c_uint32, _I, ctypes.c_uint32, _P, ctypes.c_size_t, _P, _P])
IPC_HANDLE_BYTES = 64
_ipc_export = _sig("moedisp_ipc_export", [_P, _P, ctypes.POINTER(ctypes.c_int64)])
_ipc_import = _sig("moedisp_ipc_import", [_P, ctypes.c_int64, ctypes.POINTER(ctypes.c_void_p)])
_ipc_close = _sig("moedisp_ipc_close", [_P])
_ep_barrier = _sig("moedisp_ep_barrier", [_P, _I, _I, ctypes.c_uint32, ctypes.c_uint32, _P, _P])
_shared = _sig("moedisp_shared_expert_routing",
               [_P, _P, _I, _I, _I, _I, _I, _I, _P, _P, _P, _P])
_combine_rms = _sig("moedisp_moe_combine_rmsnorm",
                    [_P, _I, Dims, ctypes.POINTER(Layout), _P, _P, _P, ctypes.c_float, _P, _P, _P, _P])


class MoedispError(RuntimeError):
    def __init__(self, code: int, call: str):
        super().__init__(f"{call} failed: {status_string(code)} ({code})")
        self.code = code


def status_string(code: int) -> str:
    return _status_string(int(code)).decode()


def version() -> int:
    return int(_version())


def _ptr(t):
    """Device pointer of a tensor (None stays NULL; ints pass through)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int, call: str, raise_on_error: bool) -> int:
    if rc < 0 and raise_on_error:
        raise MoedispError(rc, call)
    return rc


def selftest_bounded_wait(limit_us, status, stream=None, raise_on_error=True) -> int:
    """Runs the device-side wait time-out diagnostic (see include/moedisp.h)."""
    rc = _selftest_wait(int(limit_us), _ptr(status), _stream(stream))
    return _check(rc, "selftest_bounded_wait", raise_on_error)


# ------------------------------------------------------------------ exchange

def a2a_exchange_plan(in_splits, src_offsets, out_splits, dst_offsets, status, W=None,
                      stream=None, raise_on_error=True) -> int:
    W = int(in_splits.shape[0]) if W is None else W
    rc = _plan(_ptr(in_splits), W, _ptr(src_offsets), _ptr(out_splits), _ptr(dst_offsets),
               _ptr(status), _stream(stream))
    return _check(rc, "a2a_exchange_plan", raise_on_error)


def a2a_v(inp, in_rank_stride_rows, out, out_cap_rows, row_bytes, W, src_offsets, out_splits,
          dst_offsets, status, stream=None, raise_on_error=True) -> int:
    rc = _a2a_v(_ptr(inp), int(in_rank_stride_rows), _ptr(out), int(out_cap_rows),
                int(row_bytes), int(W), _ptr(src_offsets), _ptr(out_splits), _ptr(dst_offsets),
                _ptr(status), _stream(stream))
    return _check(rc, "a2a_v", raise_on_error)


# -------------------------------------------------------------------- layout

def layout_workspace_size(W: int, T: int, K: int, E: int) -> int:
    n = ctypes.c_size_t(0)
    rc = _ws_size(Dims(W, T, K, E), ctypes.byref(n))
    _check(rc, "layout_workspace_size", True)
    return int(n.value)


@dataclass
class LayoutBuffers:
    """The caller-owned device buffers of one dispatch layout (allocated with torch)."""
    W: int
    T: int
    K: int
    E: int
    rows_cap: int
    cnt: object
    occ: object
    dst_row: object
    assist_info: object
    expert_base: object
    rank_base: object
    send_splits: object
    workspace: object
    major_align: int = 0

    @classmethod
    def allocate(cls, W, T, K, E, rows_cap=None, device="cuda", major_align=0):
        """rows_cap defaults to the most rows the layout can produce: G*K, plus E*A with
        major_align A >= 2."""
        import torch
        G = W * T
        if rows_cap is None:
            rows_cap = G * K + (E * major_align if major_align > 1 else 0)
        z = dict(device=device)
        return cls(W=W, T=T, K=K, E=E, rows_cap=rows_cap, major_align=major_align,
                   cnt=torch.zeros((W, E), dtype=torch.int32, **z),
                   occ=torch.zeros(G * K, dtype=torch.int32, **z),
                   dst_row=torch.zeros(G * K, dtype=torch.int32, **z),
                   assist_info=torch.zeros(max(rows_cap, 1), dtype=torch.int32, **z),
                   expert_base=torch.zeros(E + 1, dtype=torch.int64, **z),
                   rank_base=torch.zeros(W + 1, dtype=torch.int64, **z),
                   send_splits=torch.zeros((W, W), dtype=torch.int64, **z),
                   workspace=torch.zeros(layout_workspace_size(W, T, K, E), dtype=torch.uint8, **z))

    @property
    def dims(self) -> Dims:
        return Dims(self.W, self.T, self.K, self.E)

    def struct(self) -> Layout:
        return Layout(_ptr(self.cnt), _ptr(self.occ), _ptr(self.dst_row), _ptr(self.assist_info),
                      _ptr(self.expert_base), _ptr(self.rank_base), _ptr(self.send_splits),
                      int(self.rows_cap))


def _mask_dims(active_mask, dims: Dims, given) -> int:
    """1 for a per-token mask [G], 2 for a per-slot mask [G, K]: from the tensor's shape
    unless given (raw pointers need it given)."""
    if given is not None:
        return int(given)
    if active_mask is None:
        return 0
    if isinstance(active_mask, int):
        raise ValueError("active_mask_dims is required with a raw active_mask pointer")
    if active_mask.dim() == 2:
        return 2
    return 2 if (dims.K > 1 and active_mask.numel() == dims.W * dims.T * dims.K) else 1


def moe_dispatch_layout(expert_ids, active_mask, layout: LayoutBuffers, status, stream=None,
                        raise_on_error=True, workspace=None, workspace_bytes=None,
                        active_mask_dims=None) -> int:
    """active_mask: None, uint8 [G] (per token) or [G, K] (per slot)."""
    ws = layout.workspace if workspace is None else workspace
    nbytes = (ws.numel() * ws.element_size()) if workspace_bytes is None else workspace_bytes
    L = layout.struct()
    rc = _layout(_ptr(expert_ids), _ptr(active_mask),
                 _mask_dims(active_mask, layout.dims, active_mask_dims), int(layout.major_align),
                 layout.dims, ctypes.byref(L), _ptr(ws), int(nbytes), _ptr(status), _stream(stream))
    return _check(rc, "moe_dispatch_layout", raise_on_error)


def moe_dispatch_layout_noalloc(expert_ids, active_mask, layout: LayoutBuffers, status,
                                stream=None, raise_on_error=True, active_mask_dims=None) -> int:
    """moe_dispatch_layout without a workspace argument: the scratch lives in the
    library's own device memory (see include/moedisp.h). Allocates nothing."""
    L = layout.struct()
    rc = _layout_noalloc(_ptr(expert_ids), _ptr(active_mask),
                         _mask_dims(active_mask, layout.dims, active_mask_dims),
                         int(layout.major_align), layout.dims, ctypes.byref(L), _ptr(status),
                         _stream(stream))
    return _check(rc, "moe_dispatch_layout_noalloc", raise_on_error)


def moe_dispatch(x, H, layout: LayoutBuffers, quant_mode, expand_x, dynamic_scales, status,
                 expert_token_nums=None, expert_token_nums_type=1, ep_recv_counts=None,
                 stream=None, raise_on_error=True, smooth_scales=None) -> int:
    """smooth_scales: fp32 [E, H] per-expert smoothing before quantisation (quantising
    modes)."""
    L = layout.struct()
    rc = _dispatch(_ptr(x), int(H), layout.dims, ctypes.byref(L), int(quant_mode),
                   _ptr(smooth_scales), _ptr(expand_x),
                   _ptr(dynamic_scales), _ptr(expert_token_nums), int(expert_token_nums_type),
                   _ptr(ep_recv_counts), _ptr(status), _stream(stream))
    return _check(rc, "moe_dispatch", raise_on_error)


def moe_combine(expert_out, H, layout: LayoutBuffers, expert_scales, y, status, stream=None,
                raise_on_error=True) -> int:
    L = layout.struct()
    rc = _combine(_ptr(expert_out), int(H), layout.dims, ctypes.byref(L), _ptr(expert_scales),
                  _ptr(y), _ptr(status), _stream(stream))
    return _check(rc, "moe_combine", raise_on_error)


def moe_combine_rmsnorm(expert_out, H, layout: LayoutBuffers, expert_scales, residual, gamma,
                        eps, y, status, residual_out=None, stream=None, raise_on_error=True) -> int:
    L = layout.struct()
    rc = _combine_rms(_ptr(expert_out), int(H), layout.dims, ctypes.byref(L), _ptr(expert_scales),
                      _ptr(residual), _ptr(gamma), float(eps), _ptr(residual_out), _ptr(y),
                      _ptr(status), _stream(stream))
    return _check(rc, "moe_combine_rmsnorm", raise_on_error)


def moe_dispatch_gather(x, x_rows, token_rows, H, layout: LayoutBuffers, quant_mode, expand_x,
                        dynamic_scales, status, expert_token_nums=None, expert_token_nums_type=1,
                        ep_recv_counts=None, stream=None, raise_on_error=True,
                        smooth_scales=None) -> int:
    """moe_dispatch with token g read from row token_rows[g] of x ([x_rows, H])."""
    L = layout.struct()
    rc = _dispatch_gather(_ptr(x), int(x_rows), _ptr(token_rows), int(H), layout.dims,
                          ctypes.byref(L), int(quant_mode), _ptr(smooth_scales), _ptr(expand_x),
                          _ptr(dynamic_scales), _ptr(expert_token_nums),
                          int(expert_token_nums_type), _ptr(ep_recv_counts), _ptr(status),
                          _stream(stream))
    return _check(rc, "moe_dispatch_gather", raise_on_error)


def a2a_token_rows(src_offsets, out_splits, dst_offsets, W, T, in_rank_stride_rows, token_rows,
                   status, active=None, stream=None, raise_on_error=True) -> int:
    """Source row of every receive position of an exchange plan (-1 where none)."""
    rc = _token_rows(_ptr(src_offsets), _ptr(out_splits), _ptr(dst_offsets), int(W), int(T),
                     int(in_rank_stride_rows), _ptr(token_rows), _ptr(active), _ptr(status),
                     _stream(stream))
    return _check(rc, "a2a_token_rows", raise_on_error)


def moe_dispatch_peers(x, H, layout: LayoutBuffers, rank, expert_ids, quant_mode, peer_expand_x,
                       peer_rows_cap, status, peer_scales=None, stream=None,
                       raise_on_error=True) -> int:
    """Rank `rank`'s dispatch over W GPUs: peer_expand_x / peer_scales are device int64
    tensors [W] of the ranks' buffer addresses (peer memory mapped into this GPU)."""
    L = layout.struct()
    rc = _dispatch_peers(_ptr(x), int(H), layout.dims, int(rank), _ptr(expert_ids),
                         ctypes.byref(L), int(quant_mode), _ptr(peer_expand_x),
                         _ptr(peer_scales), int(peer_rows_cap), _ptr(status), _stream(stream))
    return _check(rc, "moe_dispatch_peers", raise_on_error)


PIPE_PRODUCE = 1
PIPE_CONSUME = 2
PIPE_BOTH = 3


def a2a_dispatch_pipelined_workspace_size(W: int) -> int:
    n = ctypes.c_size_t(0)
    _check(_pipe_ws(int(W), ctypes.byref(n)), "a2a_dispatch_pipelined_workspace_size", True)
    return int(n.value)


def a2a_dispatch_pipelined(inp, in_rank_stride_rows, src_offsets, out_splits, dst_offsets, recv,
                           H, layout: LayoutBuffers, quant_mode, expand_x, dynamic_scales, ready,
                           epoch, workspace, status, roles=PIPE_BOTH, wait_limit_us=2_000_000,
                           expert_token_nums=None, expert_token_nums_type=1,
                           ep_recv_counts=None, stream=None, raise_on_error=True) -> int:
    """The exchange (a2a_v into recv [W][T][H]) and the dispatch of the received tokens
    (layout over the W*T receive positions), pipelined through per-segment ready words
    (uint32 [W][W], zeroed once; a new epoch 1, 2, ... per exchange -- or, for a CUDA
    graph, ready zeroed in stream order before every call and epoch 1 each time).
    workspace: a device buffer of a2a_dispatch_pipelined_workspace_size(W) bytes."""
    L = layout.struct()
    rc = _pipe(_ptr(inp), int(in_rank_stride_rows), _ptr(src_offsets), _ptr(out_splits),
               _ptr(dst_offsets), _ptr(recv), int(H), layout.dims, ctypes.byref(L), int(quant_mode),
               _ptr(expand_x), _ptr(dynamic_scales), _ptr(expert_token_nums),
               int(expert_token_nums_type), _ptr(ep_recv_counts), _ptr(ready),
               ctypes.c_uint32(int(epoch) & 0xFFFFFFFF), int(roles), ctypes.c_uint32(int(wait_limit_us)),
               _ptr(workspace), 0 if workspace is None else workspace.numel() * workspace.element_size(),
               _ptr(status), _stream(stream))
    return _check(rc, "a2a_dispatch_pipelined", raise_on_error)


def ipc_export(t) -> tuple[bytes, int]:
    """(IPC handle bytes, byte offset) of a device tensor's memory, for another process."""
    buf = ctypes.create_string_buffer(IPC_HANDLE_BYTES)
    off = ctypes.c_int64(0)
    _check(_ipc_export(_ptr(t), buf, ctypes.byref(off)), "ipc_export", True)
    return bytes(buf.raw), int(off.value)


def ipc_import(handle: bytes, offset: int) -> int:
    """Address, in this process, of a buffer another process exported (a plain peer
    mapping, no multicast); release it with ipc_close."""
    assert len(handle) == IPC_HANDLE_BYTES
    p = ctypes.c_void_p(0)
    _check(_ipc_import(ctypes.c_char_p(handle), int(offset), ctypes.byref(p)), "ipc_import", True)
    return int(p.value)


def ipc_close(ptr: int) -> None:
    _check(_ipc_close(ctypes.c_void_p(int(ptr))), "ipc_close", True)


def ep_barrier(peer_signals, W, rank, epoch, timeout_us, status, stream=None,
               raise_on_error=True) -> int:
    """Barrier across the W expert-parallel ranks: peer_signals is a device int64 tensor [W]
    of the ranks' signal-array addresses (uint32 [W] each, peer memory mapped into this
    GPU); a wait beyond timeout_us sets STATUS_TIMEOUT in `status` instead of hanging."""
    rc = _ep_barrier(_ptr(peer_signals), int(W), int(rank), ctypes.c_uint32(int(epoch) & 0xFFFFFFFF),
                     ctypes.c_uint32(int(timeout_us)), _ptr(status), _stream(stream))
    return _check(rc, "ep_barrier", raise_on_error)


def moe_combine_peers(peer_expert_out, peer_rows_cap, H, layout: LayoutBuffers, rank, expert_ids,
                      expert_scales, y, status, stream=None, raise_on_error=True) -> int:
    """Rank `rank`'s combine over W GPUs: peer_expert_out is a device int64 tensor [W] of
    the ranks' expert-output buffer addresses."""
    L = layout.struct()
    rc = _combine_peers(_ptr(peer_expert_out), int(peer_rows_cap), int(H), layout.dims, int(rank),
                        _ptr(expert_ids), ctypes.byref(L), _ptr(expert_scales), _ptr(y),
                        _ptr(status), _stream(stream))
    return _check(rc, "moe_combine_peers", raise_on_error)


def shared_expert_routing(expert_ids, expert_scales, W, T, K, E, shared_expert_num,
                          shared_expert_rank_num, ext_ids, ext_scales, status, stream=None,
                          raise_on_error=True) -> int:
    """Widens the routing with the shared experts: ext_ids / ext_scales are [G, K + N];
    the layout then takes dims (W, T, K + N, W * (E // (W - S)))."""
    rc = _shared(_ptr(expert_ids), _ptr(expert_scales), int(W), int(T), int(K), int(E),
                 int(shared_expert_num), int(shared_expert_rank_num), _ptr(ext_ids),
                 _ptr(ext_scales), _ptr(status), _stream(stream))
    return _check(rc, "shared_expert_routing", raise_on_error)


def raw_selftest(limit_us, status_ptr) -> int:
    return int(_selftest_wait(int(limit_us), status_ptr, None))


def raw_call(name: str, *args) -> int:
    """Calls an exported C function with already-marshalled arguments (for ABI tests)."""
    return int({"moedisp_a2a_exchange_plan": _plan, "moedisp_a2a_v": _a2a_v,
                "moedisp_moe_dispatch_layout": _layout,
                "moedisp_moe_dispatch_layout_noalloc": _layout_noalloc,
                "moedisp_moe_dispatch": _dispatch, "moedisp_moe_combine": _combine,
                "moedisp_moe_combine_rmsnorm": _combine_rms,
                "moedisp_shared_expert_routing": _shared,
                "moedisp_moe_dispatch_gather": _dispatch_gather,
                "moedisp_a2a_token_rows": _token_rows,
                "moedisp_moe_dispatch_peers": _dispatch_peers,
                "moedisp_moe_combine_peers": _combine_peers,
                "moedisp_ep_barrier": _ep_barrier,
                "moedisp_a2a_dispatch_pipelined": _pipe}[name](*args))


__all__ = [
    "a2a_exchange_plan", "a2a_v", "layout_workspace_size", "LayoutBuffers",
    "moe_dispatch_layout", "moe_dispatch_layout_noalloc", "moe_dispatch", "moe_combine",
    "selftest_bounded_wait", "moe_combine_rmsnorm", "shared_expert_routing",
    "moe_dispatch_gather", "a2a_token_rows", "moe_dispatch_peers", "moe_combine_peers",
    "status_string", "version", "NOALLOC_SCRATCH_BYTES",
    "Dims", "Layout", "MoedispError", "LIBRARY_PATH",
    "QUANT_NONE", "QUANT_INT8", "QUANT_FP8_E4M3",
    "STATUS_CAPACITY", "STATUS_BAD_EXPERT_ID", "STATUS_TIMEOUT", "STATUS_BAD_SPLIT",
]
