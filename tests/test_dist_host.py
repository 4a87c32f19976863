"""Host side of the multi-rank bench path, on CPU with the gloo backend and
world size 2: every rank is an independent replica (the decode path has no
exchange step), the timed region is bracketed by a barrier, and the reported
time is the maximum over ranks."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    d = bench.Dist(want_gpu=False)
    assert d.pg and d.world == world and d.rank == rank
    d.barrier()
    # each rank "measures" a different device time; all must see the maximum
    ms = 10.0 + 5.0 * rank
    ms_max = d.max(ms)
    rate = bench.whole_job_rate(30 * 100, d.world, ms_max)
    d.barrier()
    d.close()
    with open(os.path.join(out_dir, "r%d.json" % rank), "w") as f:
        json.dump({"ms_max": ms_max, "rate": rate}, f)


def test_max_over_ranks_and_whole_job_rate(tmp_path):
    import torch.multiprocessing as mp
    world, port = 2, free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, str(tmp_path)))
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
    res = [json.load(open(tmp_path / ("r%d.json" % r))) for r in range(world)]
    slowest = 10.0 + 5.0 * (world - 1)
    for r in res:
        assert r["ms_max"] == slowest
        # 2 replicas x 3000 layers over the slowest rank's 15 ms
        assert r["rate"] == pytest.approx(2 * 3000 / 0.015)


def test_single_rank_needs_no_process_group(monkeypatch):
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    sys.path.insert(0, ROOT)
    import bench
    d = bench.Dist(want_gpu=False)
    assert not d.pg and d.world == 1
    assert d.max(3.25) == 3.25
    d.barrier()
    d.close()


def test_reference_arm_under_torchrun_prints_once():
    """`bench.py --impl reference` under a 2-rank launch: rank 0 times the CPU
    oracle and prints one JSON line; rank 1 exits 0 without work."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--steps", "3", "--warmup", "1"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "layers/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
