"""Expert-parallel decomposition of one MoE layer on CPU, gloo, world size 2:
each rank adds up the routed experts it holds (plus the shared expert on rank
0) with the oracle, one all-reduce sums the partials, and every rank must get
the whole layer's output.  The ownership rule is the library's
(moe_expert_gemv_b200.qmoe.expert_owner, the same rule moe_expert_qmlp_ep
applies on the device)."""
import json
import os
import socket
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist

    import oracle
    from moe_expert_gemv_b200 import qmoe, synth

    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank,
                            world_size=world)
    E, H, I, k = 16, 256, 64, 4
    m = synth.moe_layer(3, 0, E=E, H=H, I=I)
    L = oracle.Layer(m, E, H, I)
    x16 = synth.activations(3, 1, H)
    _, idx, wt = oracle.router(*m["router"], E, H, 8, x16, k)
    part = L.expert(-1, x16) if rank == 0 else np.zeros(H)
    held = []
    for j in range(k):
        e = int(idx[0, j])
        if qmoe.expert_owner(e, E, world) == rank:
            held.append(e)
            part = part + wt[0, j] * L.expert(e, x16)
    t = torch.from_numpy(part.copy())
    dist.all_reduce(t)
    y64, _ = L.moe(x16, idx, wt)
    owners = [qmoe.expert_owner(e, E, world) for e in range(E)]
    dist.barrier()
    dist.destroy_process_group()
    with open(os.path.join(out_dir, "r%d.json" % rank), "w") as f:
        json.dump({"err": float(np.abs(t.numpy() - y64[0]).max() / np.abs(y64[0]).max()),
                   "held": held, "owners": owners, "idx": [int(e) for e in idx[0]]}, f)


def test_expert_parallel_partials_sum_to_layer(tmp_path):
    import torch.multiprocessing as mp
    world, port = 2, free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, str(tmp_path)))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], codes
    res = [json.load(open(tmp_path / ("r%d.json" % r))) for r in range(world)]
    for r in res:
        assert r["err"] < 1e-12
    # contiguous blocks of E/world experts; every chosen expert held exactly once
    assert res[0]["owners"] == [0] * 8 + [1] * 8
    held = sorted(res[0]["held"] + res[1]["held"])
    assert held == sorted(res[0]["idx"])


def _plumbing_main(rank, world, port, out_dir):
    """moe_layer_ep's host side under gloo: each rank's share (a stand-in for
    the device kernel: a vector of rank + 1), the all-reduce over the group,
    the fp16 conversion (a stand-in for the library's kernel)."""
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist

    from moe_expert_gemv_b200 import qmoe

    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank,
                            world_size=world)
    seen = {}

    def share(G, x, idx, weights, r, w, workspace=None):
        seen["rank"], seen["world"] = r, w
        return torch.full((8,), float(r + 1), dtype=torch.float32)

    qmoe.moe_expert_qmlp_ep = share
    qmoe.f32_to_f16 = lambda t: t.half()
    y = qmoe.moe_layer_ep(None, None, None, None)
    dist.barrier()
    dist.destroy_process_group()
    with open(os.path.join(out_dir, "p%d.json" % rank), "w") as f:
        json.dump({"y": y.float().tolist(), "dtype": str(y.dtype), **seen}, f)


def test_moe_layer_ep_plumbing(tmp_path):
    import torch.multiprocessing as mp
    world, port = 2, free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_plumbing_main, args=(r, world, port, str(tmp_path)))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], codes
    for r in range(world):
        d = json.load(open(tmp_path / ("p%d.json" % r)))
        assert d["rank"] == r and d["world"] == world
        assert d["dtype"] == "torch.float16"
        assert d["y"] == [3.0] * 8          # 1 + 2 summed over the two ranks
