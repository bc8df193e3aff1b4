"""One expert-parallel rank on one GPU, run as its own process by the GPU tests: a NCCL
process group of world size 1, EPDispatcher's symmetric buffers, bounded rank barriers,
the peer-table dispatch into the (own) mapped buffer, an identity expert and the combine
back, checked against the CPU oracle. Prints one JSON line; exit code 0 when it matches."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def main():
    from datetime import timedelta

    import numpy as np
    import torch
    import torch.distributed as dist

    import combine_a2a_exchange_b200 as md
    import oracle
    import workloads as wl
    from combine_a2a_exchange_b200.ep import EPDispatcher

    q = int(sys.argv[1]) if len(sys.argv) > 1 else 0
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=timedelta(seconds=60),
                            device_id=dev)
    res = {"quant": q}
    try:
        w = wl.moe_workload("tiny", seed=12, W=1, T=300, K=4, E=16, H=512, active_p=0.8)
        ep = EPDispatcher(md, dist.group.WORLD, w.T, w.K, w.E, w.H, quant_mode=q, device=dev)
        x = torch.from_numpy(w.x_bits.view(np.int16)).to(dev).view(torch.bfloat16)
        ids = torch.from_numpy(w.expert_ids).to(dev)
        act = torch.from_numpy(w.active).to(dev)
        wts = torch.from_numpy(w.weights).to(dev)
        ref = oracle.moe_dispatch_layout(1, w.T, w.K, w.E, w.expert_ids, w.active)
        R = ref["R"]
        rex, rsc, _ = oracle.moe_dispatch(w.x_bits, ref["dst_row"], w.K, ref["rows_cap"], q)
        eo = wl.expert_rows(max(R, 1), w.H, seed=13)
        for step in range(2):                      # two steps: the barrier epochs advance
            ex, sc = ep.dispatch(x, ids, act)
            torch.cuda.synchronize()
            n = int(ep.local_rows().item())
            got = ex[:n].view(torch.int16 if q == 0 else torch.uint8).cpu().numpy()
            if q == 0:
                got = got.view(np.uint16)
            res[f"rows_{step}"] = bool(n == R and np.array_equal(got, rex[:R]))
            if q:
                res[f"scales_{step}"] = bool(np.array_equal(sc[:n].cpu().numpy().view(np.uint32),
                                                            rsc[:R].view(np.uint32)))
            ep.expert_out[:R].copy_(torch.from_numpy(eo[:R].view(np.int16)).to(dev).view(torch.bfloat16))
            y = torch.empty((w.T, w.H), dtype=torch.bfloat16, device=dev)
            ep.combine(wts, y)                     # waits and raises on any status bit
            y32, _ = oracle.moe_combine_f32(eo, ref["dst_row"], w.weights, w.K, max(R, 1))
            res[f"combine_{step}"] = bool(np.array_equal(
                y.view(torch.int16).cpu().numpy().view(np.uint16), y32))
        res["epoch"] = ep.epoch
        res["ok"] = all(v for k, v in res.items() if k.startswith(("rows", "scales", "combine")))
    finally:
        dist.destroy_process_group()
    print(json.dumps(res), flush=True)
    return 0 if res.get("ok") else 1


if __name__ == "__main__":
    sys.exit(main())
