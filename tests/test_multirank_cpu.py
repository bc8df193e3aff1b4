"""The N > 1 path of bench.py on CPU: two gloo ranks (127.0.0.1). Each rank runs an
independent replica, so the only cross-rank steps are the max over ranks of the step
time and rank 0's report; the reference arm runs on rank 0 alone."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, values, out):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        m = bench.max_over_ranks(torch, values[rank])
        out.put((rank, m, bench.whole_job_rate(2048, world, m)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_rate_gloo():
    world, port = 2, _free_port()
    values = [1.25, 3.5]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, values, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for _, m, rate in res:
        assert m == 3.5                                  # every rank sees the slowest rank
        assert rate == pytest.approx(2 * 2048 / 3.5e-3)  # tokens of both ranks / max time


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3", "--gpus", "2"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
    env = dict(os.environ, RANK="0", WORLD_SIZE="2", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3", "--gpus", "2"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


def _routing_worker(rank, world, port, out):
    import numpy as np
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    import workloads as wl
    from combine_a2a_exchange_b200.ep import gather_routing
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = wl.moe_workload("tiny", seed=5, W=world, T=37, K=3, E=6, active_p=0.7)
        T = w.T
        ids = torch.from_numpy(w.expert_ids[rank * T:(rank + 1) * T].copy())
        act = torch.from_numpy(w.active[rank * T:(rank + 1) * T].copy())
        ids_all, act_all = gather_routing(ids, act, None)
        same = bool((ids_all.numpy() == w.expert_ids).all() and (act_all.numpy() == w.active).all())
        lay = oracle.moe_dispatch_layout(world, T, w.K, w.E, ids_all.numpy(), act_all.numpy())
        ref = oracle.moe_dispatch_layout(world, T, w.K, w.E, w.expert_ids, w.active)
        out.put((rank, same, bool(np.array_equal(lay["dst_row"], ref["dst_row"])),
                 lay["rank_base"].tolist()))
    finally:
        dist.destroy_process_group()


def test_ep_routing_all_gather_gives_every_rank_the_global_layout():
    """Expert parallelism's only host exchange: each rank all-gathers the routing and then
    computes the same global layout (here with the oracle standing in for the kernels)."""
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_routing_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(r[1] and r[2] for r in res)
    assert res[0][3] == res[1][3]                        # the same receive ranges everywhere
