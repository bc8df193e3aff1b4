"""Benchmark of the EP MoE dispatch / combine hot path on B200.

One step = one pass of the whole path over one batch of the ``cfg3`` workload, the
largest configuration (W=8 virtual EP ranks x T=4096 tokens, H=7168 bf16 with 1 %
outlier rows, E=256, K=8 Zipf(1.2)-skewed experts, per-token dynamic int8 quantisation):
dispatch layout (three kernels: tile histograms, column scans, ranking + scatter),
exchange plan of the layout's send counts (1 kernel, on a side-stream branch), quantising
dispatch (1 kernel), combine (1 kernel) of N(0,1) bf16 expert outputs. Inputs are resident
in HBM when the timed region starts; L2 is flushed before every timed step (a 512 MiB
write, then a 256 MiB read of another buffer so no dirty line is left to be written
back), outside the per-step CUDA-event pair. ``--workload cfg2|cfg4`` runs another
configuration as the step.

Prints ONE JSON line (rank 0). ``value`` = tokens/s over all ranks (each rank runs an
independent replica: weak scaling, no data-path collective); ``e2e`` = the same metric
with the step's inputs copied host->device from pinned memory and the result copied
back inside the timed region. ``roofline`` = the dominant kernel's algorithmic bytes /
its CUDA-event duration against the measured HBM copy bandwidth; ``ops`` = per-kernel
figures for the other workloads (int8 / fp8 dispatch, the W=64 all-to-all-v).

``--impl reference`` times the plain CPU oracle (the reference arm of this build) on the
same workload and metric instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "dispatch+combine tokens/s and achieved HBM GB/s (% of B200 peak), 1 GPU"
UNIT = "tokens/s"
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 512 << 20     # written, then a separate 256 MiB buffer is read
L2_READ_BYTES = 256 << 20
CPU_SAMPLE_T = 256             # tokens per rank of the oracle's bounded sample


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        try:
            d = json.load(open(p))
            return float(d["hbm_gbs"]), "measured"
        except Exception:
            pass
    return FALLBACK_HBM_GBS, "fallback"


def source_sha(path):
    return hashlib.sha256(open(os.path.join(ROOT, path), "rb").read()).hexdigest()[:16]


def ncu_traffic(kernel_key, workload):
    """dram read+write bytes per launch of `kernel_key` on `workload` from a committed ncu
    capture (scaled to the full launch when the capture ran a smaller case), when the
    kernel's source has not changed since (else None)."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p)).get(f"{kernel_key} @ {workload}")
        if not d or d.get("source_sha") != source_sha(d["source"]):
            return None
        return float(d["bytes_per_launch"])
    except Exception:
        return None


# ------------------------------------------------------------------ clocks

class ClockSampler:
    def __init__(self, enabled=True):
        self.enabled = enabled
        self.proc = None
        self.path = None

    def start(self):
        if not self.enabled:
            return
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        q = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self, uuids):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        mhz, maxes, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            if uuids and not any(u and u in f[1] for u in uuids):
                continue
            try:
                mhz.append(float(f[2]))
                maxes.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        if not mhz:
            return None
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": max(maxes),
                "reasons": sorted(reasons), "samples": len(mhz)}


# --------------------------------------------------------------- workloads

def algorithmic_bytes(op, w=None, R=None, a2a=None):
    """Bytes an op must move at minimum (each input byte read once, each output byte
    written once)."""
    if op == "a2a_v":
        return 2 * a2a.moved_rows() * a2a.row_bytes
    G, K, H = w.G, w.K, w.H
    n_act = G if w.active is None else int(w.active.sum())
    out_elem = 2 if w.quant_mode == 0 else 1
    if op == "dispatch":
        return (n_act * H * 2 + R * H * out_elem + (R * 4 if w.quant_mode else 0)
                + G * K * 4)
    if op == "combine":
        return R * H * 2 + G * H * 2 + G * K * 8
    if op == "layout":
        return G * K * 4 + (0 if w.active is None else G) + 2 * G * K * 4 + R * 4
    if op == "dispatch_smooth":
        # the dispatch's bytes + the smoothing table, read once
        return algorithmic_bytes("dispatch", w, R) + w.E * H * 4
    if op == "dispatch_smooth_gather":
        # as walked by the row-order kernel: one token row per output row, the rows'
        # assist_info, the codes and scales, the smoothing table
        out_elem = 2 if w.quant_mode == 0 else 1
        return R * H * 2 + R * 4 + R * H * out_elem + R * 4 + w.E * H * 4
    if op == "combine_rmsnorm":
        # expert rows + residual read, residual_out + y written, gamma, routing
        return R * H * 2 + 3 * G * H * 2 + H * 4 + G * K * 8
    raise ValueError(op)


class MoEStep:
    """Device-resident buffers of one workload and the five launches of one step."""

    def __init__(self, md, torch, w, device):
        self.md, self.torch, self.w = md, torch, w
        t = torch
        self.ids = t.from_numpy(w.expert_ids.reshape(-1)).to(device)
        self.active = None if w.active is None else t.from_numpy(w.active).to(device)
        self.x = t.from_numpy(w.x_bits.view(np.int16)).to(device).view(t.bfloat16)
        self.wts = t.from_numpy(w.weights.reshape(-1)).to(device)
        self.L = md.LayoutBuffers.allocate(w.W, w.T, w.K, w.E, device=device)
        cap = self.L.rows_cap
        if w.quant_mode == 0:
            self.ex = t.empty((cap, w.H), dtype=t.bfloat16, device=device)
            self.scales = None
            self.expert_out = self.ex                    # identity expert
        else:
            self.ex = t.empty((cap, w.H), dtype=t.uint8, device=device)
            self.scales = t.empty(cap, dtype=t.float32, device=device)
            g = t.Generator(device=device).manual_seed(7)
            self.expert_out = t.randn((cap, w.H), generator=g, device=device).to(t.bfloat16)
        ne = w.E // w.W
        self.etn = t.empty((w.W, ne), dtype=t.int64, device=device)
        self.erc = t.empty((w.W, ne, w.W), dtype=t.int32, device=device)
        self.plan = [t.empty((w.W, w.W), dtype=t.int64, device=device) for _ in range(3)]
        self.y = t.empty((w.G, w.H), dtype=t.bfloat16, device=device)
        self.status = t.zeros(1, dtype=t.int32, device=device)
        self.side = t.cuda.Stream(device=device)

    def op_layout(self):
        self.md.moe_dispatch_layout(self.ids, self.active, self.L, self.status)

    def op_plan(self):
        L = self.L
        self.md.a2a_exchange_plan(L.send_splits, self.plan[0], self.plan[1], self.plan[2],
                                  self.status)

    def op_dispatch(self):
        w = self.w
        self.md.moe_dispatch(self.x, w.H, self.L, w.quant_mode, self.ex, self.scales, self.status,
                             expert_token_nums=self.etn, expert_token_nums_type=0,
                             ep_recv_counts=self.erc)

    def op_combine(self):
        self.md.moe_combine(self.expert_out, self.w.H, self.L, self.wts, self.y, self.status)

    def run(self):
        """layout -> dispatch -> combine on the current stream; the exchange plan of the
        layout's send counts runs beside dispatch on a side stream (nothing in the step
        consumes it), joined before the step ends."""
        torch = self.torch
        main = torch.cuda.current_stream()
        self.op_layout()
        self.side.wait_stream(main)
        with torch.cuda.stream(self.side):
            self.op_plan()
        self.op_dispatch()
        self.op_combine()
        main.wait_stream(self.side)


def max_over_ranks(torch, value: float, device=None) -> float:
    """The largest of every rank's value (no-op without a multi-rank process group)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: int, world: int, ms: float) -> float:
    """Units per second over all ranks, for a step time that is the max over ranks."""
    return world * units_per_rank / (ms / 1e3)


def capture(torch, fn):
    """CUDA graph of fn's launches (one eager run first, outside the capture)."""
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def kernel_launches(torch, fn):
    """Kernel nodes in a CUDA graph of fn (the library's kernels of one step; the graph
    holds nothing else), or None if the runtime cannot be asked."""
    import ctypes
    try:
        rt = ctypes.CDLL("libcudart.so.12")
        g = torch.cuda.CUDAGraph(keep_graph=True)
        with torch.cuda.graph(g):
            fn()
        torch.cuda.synchronize()
        h = ctypes.c_void_p(g.raw_cuda_graph())
        n = ctypes.c_size_t(0)
        if rt.cudaGraphGetNodes(h, None, ctypes.byref(n)) != 0:
            return None
        nodes = (ctypes.c_void_p * max(n.value, 1))()
        if rt.cudaGraphGetNodes(h, nodes, ctypes.byref(n)) != 0:
            return None
        kinds = ctypes.c_int(0)
        k = 0
        for i in range(n.value):
            if rt.cudaGraphNodeGetType(ctypes.c_void_p(nodes[i]), ctypes.byref(kinds)) != 0:
                return None
            k += kinds.value == 0                    # cudaGraphNodeTypeKernel
        del g
        return k
    except Exception:
        return None


class L2Flush:
    """Writes a 512 MiB buffer (> 4x L2), then reads a separate 256 MiB one: the read
    evicts the dirty lines of the write, so the timed region starts with L2 holding
    nothing of ours and nothing left to write back."""

    def __init__(self, torch, device):
        self.w = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=device)
        self.r = torch.ones(L2_READ_BYTES // 4, dtype=torch.float32, device=device)
        self.sink = torch.empty((), dtype=torch.float32, device=device)

    def zero_(self):
        self.w.zero_()
        torch_sum = self.r.sum()
        self.sink.copy_(torch_sum)


def time_graph(torch, g, reps, warmup, flush):
    """CUDA-event time (ms) of each of `reps` replays, L2 flushed before each."""
    E = torch.cuda.Event
    for _ in range(warmup):
        flush.zero_()
        g.replay()
    torch.cuda.synchronize()
    evs = []
    for _ in range(reps):
        flush.zero_()
        a, b = E(enable_timing=True), E(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        evs.append((a, b))
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def time_ops(torch, step, reps, warmup, flush):
    """Per-op CUDA-event times (ms). Each op is launched on its own right behind the L2
    flush: the flush keeps the GPU busy while the host enqueues the event pair and the
    op, so the pair brackets the op's kernels only."""
    E = torch.cuda.Event
    out = {}
    for op in ("layout", "plan", "dispatch", "combine"):
        fn = getattr(step, "op_" + op)
        for _ in range(warmup):
            flush.zero_()
            fn()
        torch.cuda.synchronize()
        evs = []
        for _ in range(reps):
            flush.zero_()
            a, b = E(enable_timing=True), E(enable_timing=True)
            a.record()
            fn()
            b.record()
            evs.append((a, b))
        torch.cuda.synchronize()
        out[op] = [a.elapsed_time(b) for a, b in evs]
    return out


def time_ops_in_graph(torch, step, reps, warmup, flush):
    """Per-op device times (ms) inside one graph of the step (the plan serialised between
    layout and dispatch): an external event-record node after each op, so each pair of
    events brackets exactly that op's kernels as the graph runs them (no host launch
    latency). Returns None if the runtime does not support event nodes."""
    import ctypes
    try:
        rt = ctypes.CDLL("libcudart.so.12")
        rec_fn = rt.cudaEventRecordWithFlags
    except (OSError, AttributeError):
        return None
    rec_fn.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_uint]
    rec_fn.restype = ctypes.c_int
    rt.cudaGetLastError.restype = ctypes.c_int
    ops = ("layout", "plan", "dispatch", "combine")
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(ops) + 1)]
    for ev in evs:                 # torch creates the CUDA event at its first record
        ev.record()
    torch.cuda.synchronize()
    if any(not ev.cuda_event for ev in evs):
        return None

    def body(capturing):
        s = torch.cuda.current_stream().cuda_stream
        flags = 1 if capturing else 0       # external (a graph node) only inside a capture
        def rec(ev):
            rc = rec_fn(ctypes.c_void_p(ev.cuda_event), ctypes.c_void_p(s), flags)
            if rc != 0:
                raise RuntimeError(f"cudaEventRecordWithFlags failed ({rc})")
        rec(evs[0])
        for i, op in enumerate(ops):
            getattr(step, "op_" + op)()
            rec(evs[i + 1])

    try:
        body(False)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            body(True)
        out = {op: [] for op in ops}
        for it in range(warmup + reps):
            flush.zero_()
            g.replay()
            torch.cuda.synchronize()
            if it >= warmup:
                for i, op in enumerate(ops):
                    out[op].append(evs[i].elapsed_time(evs[i + 1]))
        del g
        return out
    except RuntimeError:
        rt.cudaGetLastError()      # clear the refused call's error state
        torch.cuda.synchronize()
        return None


def time_e2e(torch, md, step, steps, warmup, flush, device):
    """The step through the public API with host buffers: every step copies its inputs in
    from pinned host memory and its result y out to pinned host memory, inside the timed
    region. Steps are pipelined as a serving loop would run them: a copy-in stream, a
    compute stream and a copy-out stream over two sets of device buffers, so that step
    i+1's inputs cross PCIe while step i computes and step i-1's y comes back (PCIe is
    full duplex). The L2 flush stays on the compute stream before every step, inside the
    timed region. Returns (ms per step = total / steps, h2d bytes, d2h bytes)."""
    w = step.w
    steps_ = [step, MoEStep(md, torch, w, device)]
    h_x = torch.from_numpy(w.x_bits.view(np.int16)).pin_memory()
    h_ids = torch.from_numpy(w.expert_ids.reshape(-1)).pin_memory()
    h_w = torch.from_numpy(w.weights.reshape(-1)).pin_memory()
    h_act = None if w.active is None else torch.from_numpy(w.active).pin_memory()
    h_y = [torch.empty((w.G, w.H), dtype=torch.int16).pin_memory() for _ in range(2)]
    h2d = h_x.numel() * 2 + h_ids.numel() * 4 + h_w.numel() * 4 + (0 if h_act is None else h_act.numel())
    d2h = h_y[0].numel() * 2
    s_in, s_comp, s_out = (torch.cuda.Stream(device=device) for _ in range(3))
    E = torch.cuda.Event

    def run(n):
        ev_in = [E(), E()]
        ev_comp = [None, None]
        ev_out = [None, None]
        start, end = E(enable_timing=True), E(enable_timing=True)
        start.record(s_in)
        for i in range(n):
            b = i % 2
            st = steps_[b]
            with torch.cuda.stream(s_in):
                if ev_comp[b] is not None:
                    s_in.wait_event(ev_comp[b])            # step i-2 is done with buffers b
                st.x.view(torch.int16).copy_(h_x, non_blocking=True)
                st.ids.copy_(h_ids, non_blocking=True)
                st.wts.copy_(h_w, non_blocking=True)
                if h_act is not None:
                    st.active.copy_(h_act, non_blocking=True)
                ev_in[b].record(s_in)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(ev_in[b])
                if ev_out[b] is not None:
                    s_comp.wait_event(ev_out[b])           # y of step i-2 has left
                flush.zero_()
                st.run()
                ev_comp[b] = E()
                ev_comp[b].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[b])
                h_y[b].copy_(st.y.view(torch.int16), non_blocking=True)
                ev_out[b] = E()
                ev_out[b].record(s_out)
        end.record(s_out)
        torch.cuda.synchronize()
        return start.elapsed_time(end)

    run(max(warmup, 2))
    ms = run(steps) / steps
    del steps_[1]
    return ms, h2d, d2h


def oracle_step(oracle, w):
    lay = oracle.moe_dispatch_layout(w.W, w.T, w.K, w.E, w.expert_ids, w.active)
    oracle.a2a_exchange_plan(lay["send_splits"])
    ex, sc, _ = oracle.moe_dispatch(w.x_bits, lay["dst_row"], w.K, lay["rows_cap"], w.quant_mode)
    oracle.moe_recv_counts(w.W, w.E, lay["cnt"], 0)
    if w.quant_mode == 0:
        oracle.moe_combine_f32(ex, lay["dst_row"], w.weights, w.K)
    else:
        eo = np.zeros((lay["rows_cap"], w.H), np.uint16)
        oracle.moe_combine_f32(eo, lay["dst_row"], w.weights, w.K)


def cpu_sample(w, T_s=CPU_SAMPLE_T):
    """A bounded sample of workload w for the CPU oracle: the first T_s tokens of every
    source rank (same ranks, experts, routing, hidden size and quantisation), so that one
    oracle step takes about a second however large w is."""
    import workloads as wl
    if w.T <= T_s:
        return w
    rows = np.concatenate([np.arange(r * w.T, r * w.T + T_s) for r in range(w.W)])
    act = None if w.active is None else np.ascontiguousarray(w.active[rows])
    return wl.MoEWorkload(name=w.name, W=w.W, T=T_s, H=w.H, E=w.E, K=w.K,
                          quant_mode=w.quant_mode, x_bits=np.ascontiguousarray(w.x_bits[rows]),
                          expert_ids=np.ascontiguousarray(w.expert_ids[rows]),
                          weights=np.ascontiguousarray(w.weights[rows]), active=act,
                          recipe=dict(w.recipe, sample_T=T_s))


def sample_note(w, s):
    return (f"the first {s.T} of each rank's {w.T} tokens of {w.name} ({s.G} of {w.G} tokens; "
            f"same W, H, E, K, routing and quantisation), full oracle steps (layout, plan, "
            f"dispatch, fp32 combine) on one host thread")


def cpu_baseline(w, budget_s=10.0):
    import oracle
    cores = len(os.sched_getaffinity(0))
    s = cpu_sample(w)
    oracle_step(oracle, s)                       # warm-up (builds the library if needed)
    t0 = time.perf_counter()
    n = 0
    while True:
        oracle_step(oracle, s)
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return {"value": n * s.G / el, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{n} steps of {sample_note(w, s)}, {el:.1f} s; {cores} cores visible"}


def dtype_of(w):
    """Arithmetic types of the step: bf16 rows, the dispatch codes, fp32 combine sums."""
    return {0: "bf16", 2: "bf16 in, int8 codes + f32 scales, f32 combine",
            3: "bf16 in, e4m3 codes + f32 scales, f32 combine"}[w.quant_mode]


def config_of(w):
    return {"workload": f"{w.name}: W={w.W} virtual EP ranks x T={w.T} tokens, H={w.H} bf16, "
                        f"E={w.E}, K={w.K}, quant={'none' if w.quant_mode == 0 else w.quant_mode}",
            "global_batch": w.G, "seq_len": 1, "parallelism": "ep-virtual (one GPU)",
            "l2": "flushed before every timed step (512 MiB write, then 256 MiB read of another buffer)"}


# --------------------------------------------------------------- per-op sweep

def dispatch_kernel_name(w):
    return {0: "dispatch_copy_kernel", 2: "dispatch_quant_kernel (int8)",
            3: "dispatch_quant_kernel (e4m3)"}[w.quant_mode]


def op_sweep(md, torch, device, hbm, reps=10, main_workload="cfg3"):
    import workloads as wl
    out = []
    flush = L2Flush(torch, device)
    cache = {}

    def moe(name):
        if name not in cache:
            cache[name] = wl.moe_workload(name, seed=0)
        return cache[name]

    for name in ("cfg2", "cfg3", "cfg4"):
        if name == main_workload:
            continue
        w = moe(name)
        st = MoEStep(md, torch, w, device)
        g = capture(torch, st.run)
        t_step = time_graph(torch, g, reps, 3, flush)
        del g
        t = time_ops_in_graph(torch, st, reps, 3, flush) or time_ops(torch, st, reps, 3, flush)
        R = int(st.L.expert_base[-1].item())
        for op in ("layout", "dispatch", "combine"):
            ms = statistics.mean(t[op])
            b = algorithmic_bytes(op, w, R)
            out.append({"workload": name, "op": op, "us": round(ms * 1e3, 2),
                        "bytes": b, "GB/s": round(b / ms / 1e6, 1),
                        "frac": round(b / ms / 1e6 / hbm, 4)})
        out.append({"workload": name, "op": "step", "us": round(statistics.mean(t_step) * 1e3, 2),
                    "tokens/s": round(w.G / (statistics.mean(t_step) / 1e3), 1)})
        assert int(st.status.item()) == 0, md.status_string(int(st.status.item()))
        del st
        torch.cuda.empty_cache()
    # fused tail: combine + residual add + RMSNorm (residual_out written), after the step's
    # layout and dispatch
    for name in ("cfg2", "cfg3"):
        w = moe(name)
        st = MoEStep(md, torch, w, device)
        st.run()
        g = torch.Generator(device=device).manual_seed(11)
        res = torch.randn((w.G, w.H), generator=g, device=device).to(torch.bfloat16)
        gamma = 0.5 + torch.rand((w.H,), generator=g, device=device)
        rout = torch.empty_like(res)
        Ev = torch.cuda.Event
        pairs = []
        for r in range(reps + 3):
            flush.zero_()
            e0, e1 = Ev(enable_timing=True), Ev(enable_timing=True)
            e0.record()
            md.moe_combine_rmsnorm(st.expert_out, w.H, st.L, st.wts, res, gamma, 1e-6, st.y,
                                   st.status, residual_out=rout)
            e1.record()
            if r >= 3:
                pairs.append((e0, e1))
        torch.cuda.synchronize()
        assert int(st.status.item()) == 0, md.status_string(int(st.status.item()))
        ms = statistics.mean(a.elapsed_time(b) for a, b in pairs)
        R = int(st.L.expert_base[-1].item())
        b = algorithmic_bytes("combine_rmsnorm", w, R)
        out.append({"workload": name, "op": "combine_rmsnorm", "us": round(ms * 1e3, 2),
                    "bytes": b, "GB/s": round(b / ms / 1e6, 1),
                    "frac": round(b / ms / 1e6 / hbm, 4)})
        del st, res, rout
        torch.cuda.empty_cache()
    # dispatch with per-expert smoothing before the dynamic quantisation
    for name in ("cfg3", "cfg4"):
        w = moe(name)
        st = MoEStep(md, torch, w, device)
        st.run()
        sm = torch.from_numpy(wl.smooth_scales(w.E, w.H, seed=1)).to(device)
        Ev = torch.cuda.Event
        pairs = []
        for r in range(reps + 3):
            flush.zero_()
            e0, e1 = Ev(enable_timing=True), Ev(enable_timing=True)
            e0.record()
            md.moe_dispatch(st.x, w.H, st.L, w.quant_mode, st.ex, st.scales, st.status,
                            smooth_scales=sm)
            e1.record()
            if r >= 3:
                pairs.append((e0, e1))
        torch.cuda.synchronize()
        assert int(st.status.item()) == 0, md.status_string(int(st.status.item()))
        ms = statistics.mean(a.elapsed_time(b) for a, b in pairs)
        R = int(st.L.expert_base[-1].item())
        b = algorithmic_bytes("dispatch_smooth", w, R)
        bg = algorithmic_bytes("dispatch_smooth_gather", w, R)
        out.append({"workload": name, "op": "dispatch_smooth", "us": round(ms * 1e3, 2),
                    "bytes": b, "GB/s": round(b / ms / 1e6, 1),
                    "frac": round(b / ms / 1e6 / hbm, 4),
                    "gather_bytes": bg, "gather_frac": round(bg / ms / 1e6 / hbm, 4)})
        del st, sm
        torch.cuda.empty_cache()
    # layout with expert segments padded to multiples of 128 rows (grouped-GEMM tiles),
    # beside the unpadded layout timed the same way (eager launches, flushed L2)
    for name, A in (("cfg2", 0), ("cfg2", 128), ("cfg3", 0), ("cfg3", 128)):
        w = moe(name)
        L = md.LayoutBuffers.allocate(w.W, w.T, w.K, w.E, device=device, major_align=A)
        ids = torch.from_numpy(w.expert_ids.reshape(-1)).to(device)
        act = None if w.active is None else torch.from_numpy(w.active).to(device)
        status = torch.zeros(1, dtype=torch.int32, device=device)
        Ev = torch.cuda.Event
        pairs = []
        for r in range(reps + 3):
            flush.zero_()
            e0, e1 = Ev(enable_timing=True), Ev(enable_timing=True)
            e0.record()
            md.moe_dispatch_layout(ids, act, L, status)
            e1.record()
            if r >= 3:
                pairs.append((e0, e1))
        torch.cuda.synchronize()
        assert int(status.item()) == 0, md.status_string(int(status.item()))
        ms = statistics.mean(a.elapsed_time(b) for a, b in pairs)
        R = int(L.expert_base[-1].item())
        out.append({"workload": name, "op": f"layout_eager_align{A}", "us": round(ms * 1e3, 2),
                    "rows": R})
        del L
        torch.cuda.empty_cache()
    # cfg2 with shared experts: 4 of the 8 ranks host one shared-expert replica each
    # (sharedExpertNum 1), the 64 routed experts live on the other 4; every token also
    # goes to its shared replica (9 rows per token). Step: widened routing -> layout ->
    # dispatch -> combine, one graph.
    w = moe("cfg2")
    S_, N_ = 4, 1
    ne_ = w.E // (w.W - S_)
    Kw, Ew = w.K + N_, w.W * ne_
    ids = torch.from_numpy(w.expert_ids).to(device)
    wts = torch.from_numpy(w.weights).to(device)
    x = torch.from_numpy(w.x_bits.view(np.int16)).to(device).view(torch.bfloat16)
    ext = torch.empty((w.G, Kw), dtype=torch.int32, device=device)
    extw = torch.empty((w.G, Kw), dtype=torch.float32, device=device)
    L = md.LayoutBuffers.allocate(w.W, w.T, Kw, Ew, device=device)
    ex = torch.empty((L.rows_cap, w.H), dtype=torch.bfloat16, device=device)
    y = torch.empty((w.G, w.H), dtype=torch.bfloat16, device=device)
    status = torch.zeros(1, dtype=torch.int32, device=device)

    def shared_step():
        md.shared_expert_routing(ids, wts, w.W, w.T, w.K, w.E, N_, S_, ext, extw, status)
        md.moe_dispatch_layout(ext, None, L, status)
        md.moe_dispatch(x, w.H, L, 0, ex, None, status)
        md.moe_combine(ex, w.H, L, extw, y, status)

    g = capture(torch, shared_step)
    t = time_graph(torch, g, reps, 3, flush)
    del g
    torch.cuda.synchronize()
    assert int(status.item()) == 0, md.status_string(int(status.item()))
    ms = statistics.mean(t)
    R = w.G * Kw
    b = (w.G * w.H * 2 + R * w.H * 2) * 2 + w.G * w.K * 8 + w.G * Kw * 16
    out.append({"workload": "cfg2+shared(S=4,N=1)", "op": "step", "us": round(ms * 1e3, 2),
                "tokens/s": round(w.G / (ms / 1e3), 1), "bytes": b,
                "frac": round(b / ms / 1e6 / hbm, 4)})
    del ids, wts, x, ext, extw, L, ex, y
    torch.cuda.empty_cache()
    # exchange -> dispatch: the tokens of W = 8 ranks are first exchanged (splits ~
    # randint[0, 512)), then dispatched by the receivers' routing (H = 4096 bf16, E = 64,
    # K = 8). Sequential: a2a_v into a receive buffer, then dispatch from it. Without a
    # receive buffer: a2a_token_rows, then moe_dispatch_gather straight from the senders'
    # buffer. Both graphs: plan, receive map (the layout's mask), layout, exchange/dispatch.
    a = wl.a2a_workload(seed=3, W=8, max_split=512, zero_frac=0.1, row_elems=4096)
    W_, H_, K_, E_ = a.W, 4096, 8, 64
    cap_in, T_ = a.cap_in, a.cap_out
    w = wl.moe_workload("tiny", seed=4, W=W_, T=T_, K=K_, E=E_, H=8)
    S = torch.from_numpy(a.in_splits).to(device)
    g0 = torch.Generator(device=device).manual_seed(5)
    xin = torch.randn((W_ * cap_in, H_), generator=g0, device=device).to(torch.bfloat16)
    recv = torch.empty((W_ * T_, H_), dtype=torch.bfloat16, device=device)
    ids = torch.from_numpy(w.expert_ids.reshape(-1)).to(device)
    plan = [torch.empty((W_, W_), dtype=torch.int64, device=device) for _ in range(3)]
    tr = torch.empty(W_ * T_, dtype=torch.int64, device=device)
    act = torch.empty(W_ * T_, dtype=torch.uint8, device=device)
    L = md.LayoutBuffers.allocate(W_, T_, K_, E_, device=device)
    ex = torch.empty((L.rows_cap, H_), dtype=torch.bfloat16, device=device)
    status = torch.zeros(1, dtype=torch.int32, device=device)

    def front():
        md.a2a_exchange_plan(S, plan[0], plan[1], plan[2], status)
        md.a2a_token_rows(plan[0], plan[1], plan[2], W_, T_, cap_in, tr, status, active=act)
        md.moe_dispatch_layout(ids, act, L, status)

    def sequential():
        front()
        md.a2a_v(xin, cap_in, recv, T_, 2 * H_, W_, plan[0], plan[1], plan[2], status)
        md.moe_dispatch(recv, H_, L, 0, ex, None, status)

    def fused():
        front()
        md.moe_dispatch_gather(xin, W_ * cap_in, tr, H_, L, 0, ex, None, status)

    ready = torch.zeros((W_, W_), dtype=torch.int32, device=device)
    pws = torch.empty(md.a2a_dispatch_pipelined_workspace_size(W_), dtype=torch.uint8, device=device)

    def pipelined():
        front()
        # the graph replays one epoch: the ready words are zeroed in stream order first
        ready.zero_()
        md.a2a_dispatch_pipelined(xin, cap_in, plan[0], plan[1], plan[2], recv, H_, L, 0, ex, None,
                                  ready, 1, pws, status)

    res = {}
    for nm, fn in (("sequential", sequential), ("no_receive_buffer", fused),
                   ("pipelined_ready_words", pipelined)):
        g = capture(torch, fn)
        res[nm] = statistics.mean(time_graph(torch, g, reps, 3, flush))
        del g
    torch.cuda.synchronize()
    assert int(status.item()) == 0, md.status_string(int(status.item()))
    n_recv = int(a.in_splits.sum())
    R = int(L.expert_base[-1].item())
    b_fused = n_recv * H_ * 2 + R * H_ * 2
    b_recv = b_fused + n_recv * H_ * 2          # the receive buffer is an output too
    for nm, ms in res.items():
        bm = b_recv if nm != "no_receive_buffer" else b_fused
        out.append({"workload": "a2a8->dispatch", "op": nm, "us": round(ms * 1e3, 2),
                    "tokens/s": round(n_recv / (ms / 1e3), 1),
                    "bytes_min": bm, "frac_of_min": round(bm / ms / 1e6 / hbm, 4)})
    del xin, recv, ex, L, ready, pws
    torch.cuda.empty_cache()
    # expert parallelism through per-rank buffers: cfg2's 8 ranks each dispatch their own
    # tokens into the 8 ranks' separate buffers through a pointer table, then each combines
    # its own tokens from them (one stream per rank; on one GPU the "peers" are local
    # allocations, so this measures the kernels' addressing, not NVLink)
    w = moe("cfg2")
    st = MoEStep(md, torch, w, device)
    st.run()
    rb = st.L.rank_base.cpu().numpy()
    cap = int(np.diff(rb).max())
    bufs = [torch.empty((cap, w.H), dtype=torch.bfloat16, device=device) for _ in range(w.W)]
    table = torch.tensor([b.data_ptr() for b in bufs], dtype=torch.int64, device=device)
    ys = [torch.empty((w.T, w.H), dtype=torch.bfloat16, device=device) for _ in range(w.W)]
    streams = [torch.cuda.Stream(device=device) for _ in range(w.W)]
    ids = st.ids
    wts = st.wts.view(w.G, w.K)

    def peers_step():
        main = torch.cuda.current_stream()
        for r, s_ in enumerate(streams):
            s_.wait_stream(main)
            with torch.cuda.stream(s_):
                md.moe_dispatch_peers(st.x[r * w.T:(r + 1) * w.T], w.H, st.L, r, ids, 0, table, cap,
                                      st.status)
        for s_ in streams:
            main.wait_stream(s_)
        for r, s_ in enumerate(streams):
            s_.wait_stream(main)
            with torch.cuda.stream(s_):
                md.moe_combine_peers(table, cap, w.H, st.L, r, ids, wts[r * w.T:(r + 1) * w.T],
                                     ys[r], st.status)
        for s_ in streams:
            main.wait_stream(s_)

    g = capture(torch, peers_step)
    t = statistics.mean(time_graph(torch, g, reps, 3, flush))
    del g
    torch.cuda.synchronize()
    assert int(st.status.item()) == 0, md.status_string(int(st.status.item()))
    b = algorithmic_bytes("dispatch", w, w.G * w.K) + algorithmic_bytes("combine", w, w.G * w.K)
    out.append({"workload": "cfg2 over 8 per-rank buffers", "op": "dispatch_peers+combine_peers",
                "us": round(t * 1e3, 2), "bytes": b, "frac": round(b / t / 1e6 / hbm, 4)})
    del st, bufs, ys
    torch.cuda.empty_cache()
    # raw all-to-all-v, W = 64
    a = wl.a2a_workload(seed=0)
    W, E_ = a.W, a.row_elems
    cap_in, cap_out = a.cap_in, a.cap_out
    S = torch.from_numpy(a.in_splits).to(device)
    plan = [torch.empty((W, W), dtype=torch.int64, device=device) for _ in range(3)]
    status = torch.zeros(1, dtype=torch.int32, device=device)
    i = torch.arange(W, device=device, dtype=torch.float32)[:, None]
    k = torch.arange(cap_in, device=device, dtype=torch.float32)[None, :]
    inp = (10.0 * i + k).to(torch.bfloat16)[:, :, None].expand(W, cap_in, E_).contiguous()
    outb = torch.empty((W, cap_out, E_), dtype=torch.bfloat16, device=device)
    Ev = torch.cuda.Event
    times_plan, times_a2a = [], []
    for r in range(reps + 3):
        flush.zero_()
        e0, e1, e2 = Ev(enable_timing=True), Ev(enable_timing=True), Ev(enable_timing=True)
        e0.record()
        md.a2a_exchange_plan(S, plan[0], plan[1], plan[2], status)
        e1.record()
        md.a2a_v(inp, cap_in, outb, cap_out, 2 * E_, W, plan[0], plan[1], plan[2], status)
        e2.record()
        if r >= 3:
            times_plan.append((e0, e1))
            times_a2a.append((e1, e2))
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ms_p = statistics.mean(a.elapsed_time(b) for a, b in times_plan)
    ms_a = statistics.mean(x.elapsed_time(y) for x, y in times_a2a)
    b = algorithmic_bytes("a2a_v", a2a=a)
    out.append({"workload": "a2a64", "op": "plan", "us": round(ms_p * 1e3, 2)})
    out.append({"workload": "a2a64", "op": "a2a_v", "us": round(ms_a * 1e3, 2), "bytes": b,
                "GB/s": round(b / ms_a / 1e6, 1), "frac": round(b / ms_a / 1e6 / hbm, 4),
                "rows/s": round(a.moved_rows() / (ms_a / 1e3), 1)})
    del inp, outb
    torch.cuda.empty_cache()
    return out


# ---------------------------------------------------------------------- main

def run_gather_op(args, wl, md, torch, device, flush):
    """The dispatch of W = 8 ranks' exchanged tokens (splits ~ randint[0, 512), H = 4096
    bf16, E = 64, K = 8) after the plan, the receive map and the layout ran once:
    moe_dispatch_gather reading the tokens in place, or (--op dispatch_pipelined) the
    exchange into a receive buffer and the dispatch pipelined through ready words, a new
    epoch per call."""
    a = wl.a2a_workload(seed=3, W=8, max_split=512, zero_frac=0.1, row_elems=4096)
    W_, H_, K_, E_ = a.W, 4096, 8, 64
    cap_in, T_ = a.cap_in, a.cap_out
    w = wl.moe_workload("tiny", seed=4, W=W_, T=T_, K=K_, E=E_, H=8)
    g0 = torch.Generator(device=device).manual_seed(5)
    xin = torch.randn((W_ * cap_in, H_), generator=g0, device=device).to(torch.bfloat16)
    plan = [torch.empty((W_, W_), dtype=torch.int64, device=device) for _ in range(3)]
    tr = torch.empty(W_ * T_, dtype=torch.int64, device=device)
    act = torch.empty(W_ * T_, dtype=torch.uint8, device=device)
    L = md.LayoutBuffers.allocate(W_, T_, K_, E_, device=device)
    ex = torch.empty((L.rows_cap, H_), dtype=torch.bfloat16, device=device)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    md.a2a_exchange_plan(torch.from_numpy(a.in_splits).to(device), plan[0], plan[1], plan[2], status)
    md.a2a_token_rows(plan[0], plan[1], plan[2], W_, T_, cap_in, tr, status, active=act)
    md.moe_dispatch_layout(torch.from_numpy(w.expert_ids.reshape(-1)).to(device), act, L, status)
    Ev = torch.cuda.Event
    if args.op == "dispatch_pipelined":
        recv = torch.empty((W_ * T_, H_), dtype=torch.bfloat16, device=device)
        ready = torch.zeros((W_, W_), dtype=torch.int32, device=device)
        pws = torch.empty(md.a2a_dispatch_pipelined_workspace_size(W_), dtype=torch.uint8,
                          device=device)
        epoch = [0]

        def op():
            epoch[0] += 1
            md.a2a_dispatch_pipelined(xin, cap_in, plan[0], plan[1], plan[2], recv, H_, L, 0, ex,
                                      None, ready, epoch[0], pws, status)
    else:
        def op():
            md.moe_dispatch_gather(xin, W_ * cap_in, tr, H_, L, 0, ex, None, status)
    for _ in range(args.warmup):
        flush.zero_()
        op()
    pairs = []
    for _ in range(args.steps):
        flush.zero_()
        e0, e1 = Ev(enable_timing=True), Ev(enable_timing=True)
        e0.record()
        op()
        e1.record()
        pairs.append((e0, e1))
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise SystemExit(f"status {md.status_string(int(status.item()))}")
    us = statistics.mean(x.elapsed_time(y) for x, y in pairs) * 1e3
    print(json.dumps({"op": args.op, "workload": "a2a8->dispatch", "us": round(us, 2),
                      "steps": args.steps, "warmup": args.warmup}))
    return 0


def run_single_op(args, wl, md, torch):
    """Times one op of the widened path on --workload after the step's layout (and
    dispatch) ran once: warm-up launches, then --steps launches, each behind an L2 flush.
    Prints one JSON line. Launch order: the step's kernels once, then the op's."""
    device = torch.device("cuda", torch.cuda.current_device())
    flush = L2Flush(torch, device)
    if args.op in ("dispatch_gather", "dispatch_pipelined"):
        return run_gather_op(args, wl, md, torch, device, flush)
    w = wl.moe_workload(args.workload, seed=0, **({"T": args.T} if args.T else {}))
    st = MoEStep(md, torch, w, device)
    st.run()
    if args.op == "peers":
        # every rank's dispatch into the W ranks' separate buffers, then every rank's
        # combine from them (rank by rank on one stream)
        rb = st.L.rank_base.cpu().numpy()
        cap = int(np.diff(rb).max())
        bufs = [torch.empty((cap, w.H), dtype=torch.bfloat16, device=device) for _ in range(w.W)]
        table = torch.tensor([b.data_ptr() for b in bufs], dtype=torch.int64, device=device)
        wts = st.wts.view(w.G, w.K)

        def op():
            for r in range(w.W):
                md.moe_dispatch_peers(st.x[r * w.T:(r + 1) * w.T], w.H, st.L, r, st.ids, 0, table,
                                      cap, st.status)
            for r in range(w.W):
                md.moe_combine_peers(table, cap, w.H, st.L, r, st.ids, wts[r * w.T:(r + 1) * w.T],
                                     st.y[r * w.T:(r + 1) * w.T], st.status)
    elif args.op == "combine":
        def op():
            st.op_combine()
    elif args.op == "dispatch":
        def op():
            st.op_dispatch()
    elif args.op == "layout":
        def op():
            st.op_layout()
    elif args.op == "dispatch_smooth":
        if w.quant_mode == 0:
            raise SystemExit("dispatch_smooth needs a quantising workload (cfg3, cfg4)")
        sm = torch.from_numpy(wl.smooth_scales(w.E, w.H, seed=1)).to(device)

        def op():
            md.moe_dispatch(st.x, w.H, st.L, w.quant_mode, st.ex, st.scales, st.status,
                            smooth_scales=sm)
    else:
        g = torch.Generator(device=device).manual_seed(11)
        res = torch.randn((w.G, w.H), generator=g, device=device).to(torch.bfloat16)
        gamma = 0.5 + torch.rand((w.H,), generator=g, device=device)
        rout = torch.empty_like(res)

        def op():
            md.moe_combine_rmsnorm(st.expert_out, w.H, st.L, st.wts, res, gamma, 1e-6, st.y,
                                   st.status, residual_out=rout)
    Ev = torch.cuda.Event
    for _ in range(args.warmup):
        flush.zero_()
        op()
    pairs = []
    for _ in range(args.steps):
        flush.zero_()
        a, b = Ev(enable_timing=True), Ev(enable_timing=True)
        a.record()
        op()
        b.record()
        pairs.append((a, b))
    torch.cuda.synchronize()
    stt = int(st.status.item())
    if stt != 0:
        raise SystemExit(f"status {md.status_string(stt)}")
    us = statistics.mean(x.elapsed_time(y) for x, y in pairs) * 1e3
    line = {"op": args.op, "workload": args.workload, "us": round(us, 2),
            "steps": args.steps, "warmup": args.warmup}
    if args.op in ("layout", "dispatch", "combine", "dispatch_smooth", "combine_rmsnorm"):
        hbm, src = measured_peaks()
        b = algorithmic_bytes(args.op, w, int(st.L.expert_base[-1].item()))
        line.update({"bytes": b, "GB/s": round(b / us / 1e3, 1),
                     "frac": round(b / us / 1e3 / hbm, 4), "peak_source": src})
    print(json.dumps(line))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="cfg3")
    ap.add_argument("--T", type=int, default=None,
                    help="tokens per rank override (smaller cases for profiling)")
    ap.add_argument("--a2a-W", type=int, default=64, help="ranks of the a2a64 workload")
    ap.add_argument("--a2a-max-split", type=int, default=512, help="split bound of a2a64")
    ap.add_argument("--no-ops", action="store_true", help="skip the per-op sweep of other workloads")
    ap.add_argument("--ep", action="store_true",
                    help="expert parallelism across the N GPUs (the real exchange over NVLink) "
                         "instead of one independent replica per GPU")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--op", choices=["step", "layout", "dispatch", "combine", "dispatch_smooth",
                                     "combine_rmsnorm", "dispatch_gather", "dispatch_pipelined",
                                     "peers"], default="step",
                    help="time one op alone on --workload (one GPU, eager launches behind an L2 "
                         "flush), e.g. to profile it")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    import workloads as wl

    if args.impl == "reference":
        if rank != 0:
            return 0
        return run_reference(args, wl)
    if args.workload == "a2a64":
        return run_a2a(args, wl, world, rank, local_rank)
    if args.ep:
        return run_ep(args, wl, world, rank, local_rank)

    import torch
    import torch.distributed as dist
    import combine_a2a_exchange_b200 as md

    torch.cuda.set_device(local_rank)
    if args.op != "step":
        return run_single_op(args, wl, md, torch)
    device = torch.device("cuda", local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=device)

    hbm, peak_src = measured_peaks()
    over = {} if args.T is None else {"T": args.T}
    w = wl.moe_workload(args.workload, seed=rank, **over)
    step = MoEStep(md, torch, w, device)
    flush = L2Flush(torch, device)

    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(device).uuid)
    except Exception:
        pass
    sampler = ClockSampler(enabled=(rank == 0))

    launches = kernel_launches(torch, step.run)
    g_step = capture(torch, step.run)
    sampler.start()                    # clocks sampled over warm-up, timed steps, per-op timing
    for _ in range(args.warmup):
        flush.zero_()
        g_step.replay()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_step = time_graph(torch, g_step, args.steps, 0, flush)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    del g_step
    t = time_ops_in_graph(torch, step, args.steps, args.warmup, flush)
    op_timing = "event-record nodes inside a graph of the step"
    if t is None:
        t = time_ops(torch, step, args.steps, args.warmup, flush)
        op_timing = "eager launches right behind the L2 flush"
    clocks = sampler.stop([uuid.replace("GPU-", "")] if uuid else None) if rank == 0 else None
    status = int(step.status.item())
    if status != 0:
        raise RuntimeError(f"device status after the timed steps: {md.status_string(status)}")

    ms_step = max_over_ranks(torch, statistics.mean(t_step), device)
    R = int(step.L.expert_base[-1].item())
    per_op = {op: statistics.mean(t[op]) for op in ("layout", "plan", "dispatch", "combine")}
    dom = max(("dispatch", "combine"), key=lambda o: per_op[o])
    dom_bytes = algorithmic_bytes(dom, w, R)
    achieved = dom_bytes / (per_op[dom] * 1e-3) / 1e9
    kernel_key = {"dispatch": dispatch_kernel_name(w), "combine": f"combine_kernel<{w.K}>"}[dom]
    traffic = ncu_traffic(kernel_key, w.name)

    e2e = None
    if not args.no_e2e:
        ms_e2e, h2d, d2h = time_e2e(torch, md, step, args.steps, args.warmup, flush, device)
        ms_e2e = max_over_ranks(torch, ms_e2e, device)
        e2e = {"value": round(whole_job_rate(w.G, world, ms_e2e), 1), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": round(ms_e2e, 4),
               "mode": "pinned host in/out every step; copy-in, compute and copy-out streams "
                       "over two buffer sets (steps overlap on PCIe, both directions)"}

    ops = None
    if rank == 0 and world == 1 and not args.no_ops:
        del step
        torch.cuda.empty_cache()
        ops = op_sweep(md, torch, device, hbm, main_workload=w.name)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    step_bytes = sum(algorithmic_bytes(op, w, R) for op in ("layout", "dispatch", "combine"))
    line = {
        "metric": METRIC,
        "value": round(whole_job_rate(w.G, world, ms_step), 1),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": dtype_of(w),
        "data": "synthetic (seeded generator; no dataset)",
        "config": config_of(w),
        "timing": "CUDA-graph replay of the step (exchange plan on a side-stream branch beside "
                  "dispatch); per-op times from " + op_timing,
        "hbm_GBps_step": round(step_bytes / (ms_step * 1e-3) / 1e9, 1),
        "frac_of_peak_step": round(step_bytes / (ms_step * 1e-3) / 1e9 / hbm, 4),
        "per_op_us": {k: round(v * 1e3, 2) for k, v in per_op.items()},
        "per_op_frac": {op: round(algorithmic_bytes(op, w, R) / (per_op[op] * 1e-3) / 1e9 / hbm, 4)
                        for op in ("dispatch", "combine")},
        "roofline": {"bound": "hbm", "kernel": kernel_key, "achieved": round(achieved, 1),
                     "peak": hbm, "peak_source": peak_src, "unit": "GB/s",
                     "frac": round(achieved / hbm, 4), "traffic": traffic,
                     "algorithmic_bytes": dom_bytes},
        "gpu_launches": None if launches is None else launches * args.steps,
        "launches_per_step": launches,
        "clocks": clocks,
        "e2e": e2e,
        "cpu_baseline": cpu,
        "ops": ops,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_a2a(args, wl, world, rank, local_rank):
    """The raw uneven all-to-all-v workload as the step: exchange plan + a2a_v over W
    virtual ranks (rows of 4096 bf16 labelled 10*i+k). Metric: moved rows/s and GB/s."""
    import torch
    import combine_a2a_exchange_b200 as md
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    hbm, peak_src = measured_peaks()
    a = wl.a2a_workload(seed=rank, W=args.a2a_W, max_split=args.a2a_max_split)
    W, E_ = a.W, a.row_elems
    cap_in, cap_out = a.cap_in, a.cap_out
    S = torch.from_numpy(a.in_splits).to(device)
    plan = [torch.empty((W, W), dtype=torch.int64, device=device) for _ in range(3)]
    status = torch.zeros(1, dtype=torch.int32, device=device)
    i = torch.arange(W, device=device, dtype=torch.float32)[:, None]
    k = torch.arange(cap_in, device=device, dtype=torch.float32)[None, :]
    inp = (10.0 * i + k).to(torch.bfloat16)[:, :, None].expand(W, cap_in, E_).contiguous()
    out = torch.empty((W, cap_out, E_), dtype=torch.bfloat16, device=device)

    def step():
        md.a2a_exchange_plan(S, plan[0], plan[1], plan[2], status)
        md.a2a_v(inp, cap_in, out, cap_out, 2 * E_, W, plan[0], plan[1], plan[2], status)

    flush = L2Flush(torch, device)
    g = capture(torch, step)
    ms = statistics.mean(time_graph(torch, g, args.steps, args.warmup, flush))
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise RuntimeError(md.status_string(int(status.item())))
    ms = max_over_ranks(torch, ms, device)
    if rank == 0:
        b = algorithmic_bytes("a2a_v", a2a=a)
        print(json.dumps({
            "metric": "a2a_v moved rows/s (plan + exchange), 1 GPU", "value":
            round(whole_job_rate(a.moved_rows(), world, ms), 1), "unit": "rows/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16 rows (copied as bytes)", "data": "synthetic",
            "config": {"workload": f"a2a: W={W}, splits ~ randint[0,{args.a2a_max_split}) with 10% "
                                   f"zeros, rows of {E_} bf16", "moved_rows": a.moved_rows()},
            "hbm_GBps": round(b / (ms * 1e-3) / 1e9, 1), "peak": hbm, "peak_source": peak_src,
            "gpu_launches": 2 * args.steps}), flush=True)
    return 0


def run_ep(args, wl, world, rank, local_rank):
    """Expert parallelism across the GPUs: the workload's W virtual ranks are spread over
    the N processes (W/N each, so GPU r holds tokens [r*G/N, (r+1)*G/N) and experts
    [r*E/N, (r+1)*E/N)), and one step is EPDispatcher's real exchange -- routing
    all-gather (NCCL), global layout, peer-table dispatch into the owners' buffers, bounded
    device barriers, peer-table combine -- with the experts' outputs fixed (N(0,1) rows).
    Strong scaling: the total work is the configuration's at every N. Inputs are larger
    than L2 on every GPU, so no flush between steps; device time per step is the max over
    ranks. NVLink bytes are the rows this rank sends to other GPUs in the dispatch plus the
    rows it reads from other GPUs in the combine."""
    from datetime import timedelta

    import torch
    import torch.distributed as dist
    import combine_a2a_exchange_b200 as md
    from combine_a2a_exchange_b200.ep import EPDispatcher

    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ.setdefault("MASTER_PORT", "29517")
    os.environ.setdefault("RANK", str(rank))
    os.environ.setdefault("WORLD_SIZE", str(world))
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=device)
    w = wl.moe_workload(args.workload, seed=0)
    if w.W % world or w.E % world:
        raise SystemExit(f"--ep needs N dividing W={w.W} and E={w.E}")
    Tr = w.G // world
    sl = slice(rank * Tr, (rank + 1) * Tr)
    ep = EPDispatcher(md, dist.group.WORLD, Tr, w.K, w.E, w.H, quant_mode=w.quant_mode,
                      device=device)
    x = torch.from_numpy(np.ascontiguousarray(w.x_bits[sl]).view(np.int16)).to(device).view(torch.bfloat16)
    ids = torch.from_numpy(np.ascontiguousarray(w.expert_ids[sl])).to(device)
    act = None if w.active is None else torch.from_numpy(np.ascontiguousarray(w.active[sl])).to(device)
    wts = torch.from_numpy(np.ascontiguousarray(w.weights[sl])).to(device)
    y = torch.empty((Tr, w.H), dtype=torch.bfloat16, device=device)
    g = torch.Generator(device=device).manual_seed(7 + rank)
    ep.expert_out.copy_(torch.randn(ep.expert_out.shape, generator=g, device=device).to(torch.bfloat16))

    def step():
        ep.dispatch(x, ids, act)
        ep.combine(wts, y, check=False)

    for _ in range(args.warmup):
        step()
    ep.check()
    dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    ep.check()
    dist.barrier()
    torch.cuda.synchronize()
    ms = max_over_ranks(torch, e0.elapsed_time(e1) / args.steps, device)
    # bytes this rank moves over NVLink per step
    ne = w.E // world
    mine = w.expert_ids[sl]
    live = np.ones(mine.shape, bool) if w.active is None else (
        np.broadcast_to(w.active[sl][:, None], mine.shape).astype(bool) if w.active.ndim == 1
        else w.active[sl].astype(bool))
    remote = int(((mine // ne != rank) & live).sum())
    out_row = w.H * (2 if w.quant_mode == 0 else 1) + (4 if w.quant_mode else 0)
    nvl = remote * (out_row + 2 * w.H)
    nvl_t = torch.tensor([float(nvl)], dtype=torch.float64, device=device)
    dist.all_reduce(nvl_t, op=dist.ReduceOp.MAX)
    ep.close()
    dist.barrier()
    dist.destroy_process_group()
    if rank != 0:
        return 0
    print(json.dumps({
        "metric": METRIC, "value": round(w.G / (ms / 1e3), 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": dtype_of(w),
        "data": "synthetic (seeded generator; no dataset)",
        "config": dict(config_of(w), parallelism=f"ep{world} (expert parallel over GPUs)",
                       l2="inputs larger than L2 on every GPU; no flush"),
        "mode": "ep: routing all-gather, global layout, peer-table dispatch and combine over "
                "IPC-mapped buffers, bounded device barriers",
        "nvlink_bytes_per_rank_step_max": int(nvl_t.item()),
        "nvlink_GBps_per_rank": round(nvl_t.item() / (ms * 1e-3) / 1e9, 1),
        "gpu_launches": None}), flush=True)
    return 0


def run_reference(args, wl):
    import oracle
    w = wl.moe_workload(args.workload, seed=0)
    s = cpu_sample(w)
    cores = len(os.sched_getaffinity(0))
    for _ in range(args.warmup):
        oracle_step(oracle, s)
    ts = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle_step(oracle, s)
        ts.append(time.perf_counter() - t0)
    ms = statistics.mean(ts) * 1e3
    value = round(s.G / (ms / 1e3), 1)
    line = {
        "impl": "reference",
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": dtype_of(w),
        "data": "synthetic (seeded generator; no dataset)", "config": config_of(w),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": f"each step: {sample_note(w, s)}; {cores} cores visible"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
