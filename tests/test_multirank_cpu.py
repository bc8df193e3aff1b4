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


def _leaving_worker(rank, world, port, out):
    """Step 1 on every rank; then rank 1 leaves (the process ends without a word) and rank
    0 runs step 2's routing all-gather, which must fail within the group's timeout."""
    import time
    from datetime import timedelta

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import workloads as wl
    from combine_a2a_exchange_b200.ep import gather_routing
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=5))
    w = wl.moe_workload("tiny", seed=6, W=world, T=16, K=2, E=4)
    T = w.T
    ids = torch.from_numpy(w.expert_ids[rank * T:(rank + 1) * T].copy())
    ids_all, _ = gather_routing(ids, None, None)
    ok1 = bool((ids_all.numpy() == w.expert_ids).all())
    if rank == 1:
        out.put((rank, ok1, None, None))
        out.close()
        out.join_thread()                 # the message is out before the process ends
        os._exit(0)                       # leaves between steps: no goodbye, no destroy
    time.sleep(1.0)                       # rank 1 is gone by now
    t0 = time.monotonic()
    err = None
    try:
        gather_routing(ids, None, None)
    except Exception as e:                # gloo reports the lost peer or the timeout
        err = type(e).__name__
    out.put((rank, ok1, err, time.monotonic() - t0))
    out.close()
    out.join_thread()
    os._exit(0)


def test_ep_rank_leaving_between_steps_fails_the_survivor_in_bounded_time():
    """Failure detection on the host: after a completed step one rank exits; the other
    rank's next routing all-gather raises within the process group's 5 s timeout (plus a
    margin) instead of waiting for good. No GPU is involved."""
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_leaving_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
    assert res[0][1] and res[1][1]                       # step 1 ran on both ranks
    rank0 = res[0]
    assert rank0[2] is not None, "the survivor's all-gather did not fail"
    assert rank0[3] < 30.0, rank0[3]
