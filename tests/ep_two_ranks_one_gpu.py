"""Two expert-parallel ranks as two processes sharing GPU 0, run by the GPU tests: a gloo
process group, EPDispatcher with every rank's buffers mapped into the other process through
the library's IPC calls, and host barriers (each rank synchronises its stream, then the
group meets) -- so no kernel ever waits for the other process. Each rank dispatches its
tokens into both ranks' buffers through the peer tables, an identity-like expert output is
written, and each rank combines its own tokens back; rows, scales and y against the CPU
oracle, over two steps. Prints one JSON line per rank; exit code 0 when both match."""
import json
import os
import socket
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def worker(rank, world, port, q_mode, out):
    import numpy as np
    import torch
    import torch.distributed as dist
    from datetime import timedelta

    import combine_a2a_exchange_b200 as md
    import oracle
    import workloads as wl
    from combine_a2a_exchange_b200.ep import EPDispatcher

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    res = {"rank": rank, "quant": q_mode}
    try:
        W, T, K, E, H = world, 200, 4, 8 * world, 384
        w = wl.moe_workload("tiny", seed=21, W=W, T=T, K=K, E=E, H=H, active_p=0.8)
        ep = EPDispatcher(md, dist.group.WORLD, T, K, E, H, quant_mode=q_mode, device=dev,
                          barrier="host")
        sl = slice(rank * T, (rank + 1) * T)
        x = torch.from_numpy(w.x_bits[sl].view(np.int16).copy()).to(dev).view(torch.bfloat16)
        ids = torch.from_numpy(w.expert_ids[sl].copy()).to(dev)
        act = torch.from_numpy(w.active[sl].copy()).to(dev)
        wts = torch.from_numpy(w.weights[sl].copy()).to(dev)
        ref = oracle.moe_dispatch_layout(W, T, K, E, w.expert_ids, w.active)
        rb = ref["rank_base"]
        R = ref["R"]
        rex, rsc, _ = oracle.moe_dispatch(w.x_bits, ref["dst_row"], K, ref["rows_cap"], q_mode)
        eo = wl.expert_rows(max(R, 1), H, seed=22)          # expert outputs, global row order
        lo, hi = int(rb[rank]), int(rb[rank + 1])
        for step in range(2):
            ex, sc = ep.dispatch(x, ids, act)
            torch.cuda.synchronize()
            n = int(ep.local_rows().item())
            got = ex[:n].view(torch.int16 if q_mode == 0 else torch.uint8).cpu().numpy()
            if q_mode == 0:
                got = got.view(np.uint16)
            res[f"rows_{step}"] = bool(n == hi - lo and np.array_equal(got, rex[lo:hi]))
            if q_mode:
                res[f"scales_{step}"] = bool(np.array_equal(
                    sc[:n].cpu().numpy().view(np.uint32), rsc[lo:hi].view(np.uint32)))
            # this rank's experts: their outputs for its rows of the global order
            ep.expert_out[:n].copy_(torch.from_numpy(eo[lo:hi].view(np.int16).copy()).to(dev)
                                    .view(torch.bfloat16))
            y = torch.full((T, H), 7, dtype=torch.int16, device=dev).view(torch.bfloat16)
            ep.combine(wts, y)
            y32, _ = oracle.moe_combine_f32(eo, ref["dst_row"][rank * T * K:(rank + 1) * T * K],
                                            w.weights[sl], K, max(R, 1))
            res[f"combine_{step}"] = bool(np.array_equal(
                y.view(torch.int16).cpu().numpy().view(np.uint16), y32))
            ep.barrier()                      # both ranks are done with this step's buffers
        res["ok"] = all(v for k, v in res.items() if k.startswith(("rows", "scales", "combine")))
        ep.close()
        dist.barrier()
    except Exception as e:                    # reported, not hidden
        res["error"] = f"{type(e).__name__}: {e}"
        res["ok"] = False
    finally:
        dist.destroy_process_group()
    out.put(res)


def main():
    import torch.multiprocessing as mp
    q_mode = int(sys.argv[1]) if len(sys.argv) > 1 else 0
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=worker, args=(r, 2, port, q_mode, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=240) for _ in procs), key=lambda r: r["rank"])
    for p in procs:
        p.join(timeout=60)
    for r in res:
        print(json.dumps(r), flush=True)
    return 0 if all(r.get("ok") for r in res) and all(p.exitcode == 0 for p in procs) else 1


if __name__ == "__main__":
    sys.exit(main())
