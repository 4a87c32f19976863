#!/usr/bin/env python
"""Benchmark of the MoE decode hot path on B200.

Default workload (one "step"): one decode token through 30 MoE layers back to
back, each layer = 8-bit router GEMV -> softmax -> top-8 of 128 experts ->
8 gathered routed SwiGLU experts + the resident shared expert (affine 4-bit,
group 64, hidden 2816, intermediate 704) -> weighted combine.  Every layer has
its own seeded weights (12.96 GB in total, far larger than the 126 MB L2, so
each step streams its 915 MB of weights from HBM) and its own seeded input.

Metric: MoE decode layers/s (whole job, all ranks).  The JSON line also gives
the weight-stream GB/s of the dominant kernel against the measured HBM peak
(`roofline`), the same metric end to end through host buffers (`e2e`), and the
CPU oracle timed on a bounded sample (`cpu_baseline`).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload moe_decode|qgemv|qgemv_fmt|router|prefill|
                              expert_cache|expert_parallel]
                  [--layers L] [--qgemv-batch 1,4,8,16,32] [--router-tokens 1,...,128]

The other workloads print one JSON line of per-kernel numbers each: dense
qGEMV at batch 1..32 (one pass over the weights from batch 9 on), the
bf16-scale formats, the router, the 128-token prefill chunk, expert streaming
from host memory, and one rank's share of an expert-parallel layer.

Under torchrun every rank runs an independent replica (weak scaling); the
timed region is bracketed by a barrier and device synchronisation, and the
slowest rank's time is reported.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

E, H, I, TOPK, LAYERS = 128, 2816, 704, 8, 30
# algorithmic bytes (packed codes + fp16 scales + fp16 biases)
MAT_BYTES = I * H // 2 + 2 * I * (H // 64) * 2            # one 704x2816 4-bit matrix
EXPERT_BYTES = 3 * MAT_BYTES                                # gate + up + down
ROUTER_BYTES = E * H + 2 * E * (H // 64) * 2                # 128x2816 8-bit
LAYER_BYTES = ROUTER_BYTES + (TOPK + 1) * EXPERT_BYTES      # 30,491,648
GATEUP_BYTES = (TOPK + 1) * 2 * MAT_BYTES + H * 2 + (TOPK + 1) * I * 4
DOWN_BYTES = (TOPK + 1) * MAT_BYTES + (TOPK + 1) * I * 4 + H * 2
ROUTER_CALL_BYTES = ROUTER_BYTES + H * 2 + TOPK * 8

# DRAM traffic per launch of the dominant kernel from an ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum), valid only for the kernel
# source it was taken on (sha256 of csrc/decode.cu); otherwise reported null.
NCU_TRAFFIC = {
    # 6-layer capture (183,180,800 B read + 4,709,632 B written) scaled to
    # the 30 layers of one launch; the hash covers decode.cu and common.cuh
    # (the dequantisation the kernel inlines; comments of both files have
    # changed since the capture, the code has not)
    "moe_decode_kernel": {"bytes": 939452160, "sha": "8ec6d2a74df41ac6"},
}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["moe_decode", "qgemv", "qgemv_fmt", "router", "prefill",
                                           "expert_cache", "expert_parallel"],
                    default="moe_decode")
    ap.add_argument("--layers", type=int, default=LAYERS)
    ap.add_argument("--qgemv-batch", default="1,4,8,16,32",
                    help="batch sizes of the qgemv workload (comma-separated)")
    ap.add_argument("--router-tokens", default="1,2,4,8,16,32,64,128",
                    help="token counts of the router workload (comma-separated)")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="time budget of the CPU-oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


# --------------------------------------------------------------- helpers --
def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 1590.0, "fallback"


def source_sha(*names):
    """sha256[:16] of the named csrc files, concatenated in order."""
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(ROOT, "moe_expert_gemv_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.device_index = device_index

    def start(self):
        try:
            import torch
            uuid = "GPU-" + str(torch.cuda.get_device_properties(self.device_index).uuid)
            cmd = ["nvidia-smi", "-i", uuid, "--query-gpu=" + self.FIELDS,
                   "--format=csv,noheader,nounits", "-lms", "100"]
            self.proc = subprocess.Popen(cmd, stdout=self.file, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, AttributeError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [r.split(", ") for r in self.file.read().strip().splitlines() if r.strip()]
        os.unlink(self.file.name)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


class Dist:
    def __init__(self, want_gpu=True):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = False
        if self.world > 1:
            import datetime
            import torch
            import torch.distributed as dist
            backend = "nccl" if (want_gpu and torch.cuda.is_available()) else "gloo"
            if backend == "nccl":
                torch.cuda.set_device(self.local)
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
            self.pg = True

    def barrier(self):
        if self.pg:
            import torch.distributed as dist
            dist.barrier()

    def max(self, v):
        if not self.pg:
            return v
        import torch
        import torch.distributed as dist
        dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
        t = torch.tensor([float(v)], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            import torch.distributed as dist
            dist.destroy_process_group()


def whole_job_rate(units_per_rank, n_ranks, ms_max):
    """Units all ranks processed per second, over the slowest rank's time."""
    return units_per_rank * n_ranks / (ms_max / 1e3)


def timed_replays(fn, iters, dist=None):
    """Device time (ms) of `iters` calls of fn on the current stream."""
    import torch
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    s.record()
    for _ in range(iters):
        fn()
    e.record()
    e.synchronize()
    torch.cuda.synchronize()
    return s.elapsed_time(e)


# ---------------------------------------------------- CPU oracle baseline --
def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def host_threads():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline_line(seconds, seed, m):
    """The oracle on bounded samples of decode layers: the threaded build on
    every host thread (the reported value) and the plain single-threaded
    build beside it."""
    import oracle
    half = seconds / 2.0
    d1, e1 = oracle_decode_layers(half, seed, m=m)
    nt = host_threads()
    oracle.use_threads(True)
    try:
        dn, en = oracle_decode_layers(half, seed, m=m)
    finally:
        oracle.use_threads(False)
    return {"value": round(dn / en, 3), "unit": "layers/s", "cores": nt, "kind": "oracle",
            "sample": "%d decode layers (router + shared + 8 routed experts) of layer 0's "
                      "weights, fresh seeded tokens, %.1f s, OpenMP over output rows on %d "
                      "threads" % (dn, en, nt),
            "cpu_model": cpu_model(),
            "single_thread": {"value": round(d1 / e1, 3), "unit": "layers/s", "cores": 1,
                              "sample": "%d layers, %.1f s" % (d1, e1)}}


def oracle_decode_layers(seconds, seed, max_layers=None, m=None):
    """Run the CPU oracle on decode layers (router + shared + 8 routed experts)
    of one layer's weights with fresh seeded tokens until `seconds` elapse.
    Returns (layers done, elapsed s)."""
    import oracle
    from moe_expert_gemv_b200 import synth
    if m is None:
        m = synth.moe_layer(seed, 0)
    L = oracle.Layer(m, E, H, I)
    done, t0 = 0, time.perf_counter()
    while True:
        x16 = synth.activations(seed + 1000 + done, 1, H)
        _, idx, wt = oracle.router(*m["router"], E, H, 8, x16, TOPK)
        L.moe(x16, idx, wt)
        done += 1
        el = time.perf_counter() - t0
        if (el >= seconds and done >= 3) or (max_layers and done >= max_layers):
            return done, el


# --------------------------------------------------------- MoE decode run --
def build_decode(args, dev):
    import concurrent.futures as cf
    import torch
    from moe_expert_gemv_b200 import qmoe, synth

    def gen(l):
        m = synth.moe_layer(args.seed, l)
        G = qmoe.MoELayer.from_numpy(m, E, H, I, device=dev)
        return G, (m if l == 0 else None)

    with cf.ThreadPoolExecutor(8) as ex:
        res = list(ex.map(gen, range(args.layers)))
    layers = [r[0] for r in res]
    m0 = res[0][1]
    xs = np.stack([synth.activations(args.seed, 1, H, layer=l)[0] for l in range(args.layers)])
    x = torch.from_numpy(xs.view(np.float16).copy()).to(dev)
    idx = torch.zeros(args.layers, TOPK, dtype=torch.int32, device=dev)
    wt = torch.zeros(args.layers, TOPK, dtype=torch.float32, device=dev)
    y = torch.zeros(args.layers, H, dtype=torch.float16, device=dev)
    ws = [qmoe.expert_workspace(layers[0], TOPK, dev) for _ in range(args.layers)]
    torch.cuda.synchronize()
    return layers, m0, x, idx, wt, y, ws


def run_decode(args, dist):
    import torch
    from moe_expert_gemv_b200 import qmoe

    dev = torch.device("cuda", dist.local if dist.world > 1 else 0)
    torch.cuda.set_device(dev)
    layers, m0, x, idx, wt, y, ws = build_decode(args, dev)
    nl = args.layers
    stack = qmoe.DecodeStack(layers, TOPK, dev)

    def fused_step():
        qmoe.moe_decode_layers(stack, x, y, idx, wt)

    # the same step as per-layer calls (router, gate/up, down kernels)
    def unfused_step():
        for l in range(nl):
            qmoe.moe_router_topk(layers[l].router, x[l:l + 1], TOPK, idx[l:l + 1], wt[l:l + 1])
            qmoe.moe_expert_qmlp(layers[l], x[l], idx[l], wt[l], y[l], ws[l])

    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        fused_step()
        unfused_step()
        torch.cuda.synchronize()
        assert qmoe.qmoe_check_status() == 0
        g_unfused = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_unfused, stream=stream):
            unfused_step()
        torch.cuda.synchronize()

        for _ in range(args.warmup):
            fused_step()
        torch.cuda.synchronize()
        clocks = ClockSampler(dev.index) if dist.rank == 0 else None
        if clocks:
            clocks.start()
        ms = timed_replays(fused_step, args.steps, dist)
        clk = clocks.stop() if clocks else None
        ms = dist.max(ms)
        flags = qmoe.qmoe_check_status()

        # the per-layer kernel path, for comparison
        reps = max(20, args.steps // 10)
        for _ in range(3):
            g_unfused.replay()
        unfused_ms = timed_replays(g_unfused.replay, reps) / reps

        # end to end through host buffers with the C call that takes them
        # (moe_decode_layers_host): H2D of every layer's input token, the
        # step, D2H of every layer's output, each step
        x_host = x.cpu().pin_memory()
        y_host = torch.empty_like(y, device="cpu").pin_memory()

        def e2e_step():
            qmoe.moe_decode_layers_host(stack, x_host, y_host, x, y)

        for _ in range(3):
            e2e_step()
        e2e_steps = max(10, args.steps // 4)
        e2e_ms = dist.max(timed_replays(e2e_step, e2e_steps, dist))
    del g_unfused
    return dict(ms=ms, unfused_ms=unfused_ms, clk=clk, flags=flags, e2e_ms=e2e_ms,
                e2e_steps=e2e_steps, m0=m0, h2d=x.numel() * 2, d2h=y.numel() * 2)


def decode_config(nl, n_ranks):
    return {
        "workload": "moe_decode: 1 token x %d MoE layers (router 8-bit 128x%d, top-%d of %d "
                    "SwiGLU experts %dx%d 4-bit g64 + shared expert)" % (nl, H, TOPK, E, I, H),
        "layers": nl, "experts": E, "hidden": H, "inter": I, "top_k": TOPK,
        "bytes_per_layer": LAYER_BYTES,
        "l2": "inputs larger than L2: %.2f GB of weights, each step streams %.0f MB"
              % (nl * (ROUTER_BYTES + (E + 1) * EXPERT_BYTES) / 1e9, nl * LAYER_BYTES / 1e6),
        "path": "moe_decode_layers: one persistent cooperative launch per step",
        "parallelism": "replicas x%d" % n_ranks if n_ranks > 1 else "single GPU",
    }


def main_decode(args):
    dist = Dist()
    r = run_decode(args, dist)
    if dist.rank != 0:
        dist.close()
        return
    hbm, _, peak_kind = peaks()
    nl, K, N = args.layers, args.steps, dist.world
    value = whole_job_rate(nl * K, N, r["ms"])
    launch_ms = r["ms"] / K
    step_bytes = nl * (LAYER_BYTES + 2 * H * 2)
    gbs = step_bytes / (launch_ms / 1e3) / 1e9
    trf = NCU_TRAFFIC.get("moe_decode_kernel")
    # traffic grows in proportion to the layers a launch streams
    traffic = (round(trf["bytes"] * nl / 30) if trf and trf["sha"] == source_sha("decode.cu", "common.cuh")
               else None)
    line = {
        "metric": "qGEMV/MoE-layer weight-stream GB/s vs HBM peak; MoE decode layers/s",
        "value": round(value, 1),
        "unit": "layers/s",
        "n_gpus": N,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(launch_ms, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f16xf16->f32 (affine int4 weights)",
        "data": "synthetic (seeded; value distributions of the pages' workloads)",
        "config": dict(decode_config(nl, N),
                       weight_stream_gbs=round(LAYER_BYTES * nl / (launch_ms / 1e3) / 1e9, 1)),
        "roofline": {
            "bound": "hbm", "kernel": "moe_decode_kernel",
            "achieved": round(gbs, 1), "peak": hbm, "peak_kind": peak_kind, "unit": "GB/s",
            "frac": round(gbs / hbm, 4), "traffic": traffic,
            "algorithmic_bytes_per_launch": step_bytes,
            "launch_us": round(launch_ms * 1e3, 2),
        },
        "unfused_layers_per_s": round(nl / (r["unfused_ms"] / 1e3), 1),
        "e2e": {"value": round(whole_job_rate(nl * r["e2e_steps"], N, r["e2e_ms"]), 1),
                "unit": "layers/s", "h2d_bytes_per_step": r["h2d"],
                "d2h_bytes_per_step": r["d2h"]},
        "gpu_launches": K,
        "device_flags": r["flags"],
    }
    if r["clk"]:
        line["clocks"] = r["clk"]
    if N == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_line(args.cpu_seconds, args.seed, r["m0"])
    print(json.dumps(line), flush=True)
    dist.close()


# ----------------------------------------------------- reference (oracle) --
def main_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    budget = 150.0
    per_layer = 0.25
    steps = max(3, min(args.steps, int(budget / per_layer)))
    warm = min(args.warmup, 2)
    import oracle
    from moe_expert_gemv_b200 import synth
    m = synth.moe_layer(args.seed, 0)
    nt = host_threads()
    oracle.use_threads(True)   # the oracle's OpenMP build on every host thread
    oracle_decode_layers(0.0, args.seed, max_layers=max(1, warm), m=m)
    done, el = oracle_decode_layers(1e9, args.seed, max_layers=steps, m=m)
    oracle.use_threads(False)
    value = done / el
    line = {
        "impl": "reference",
        "metric": "qGEMV/MoE-layer weight-stream GB/s vs HBM peak; MoE decode layers/s",
        "value": round(value, 3), "unit": "layers/s",
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": done,
        "warmup": warm, "ms_per_step": round(el / done * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(decode_config(args.layers, 1),
                       path="CPU oracle (fp64), one layer of the stack per step"),
        "cpu_baseline": {"value": round(value, 3), "unit": "layers/s", "cores": nt,
                         "kind": "oracle", "cpu_model": cpu_model(),
                         "sample": "%d decode layers (router + shared + 8 routed experts) "
                                   "of layer 0's weights, fresh seeded tokens, OpenMP over "
                                   "output rows on %d threads" % (done, nt)},
        "e2e": {"value": round(value, 3), "unit": "layers/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------- secondary workloads --
def main_other(args):
    """Single-kernel workloads used for the per-kernel roofline notes."""
    import torch
    from moe_expert_gemv_b200 import qmoe, synth
    dev = torch.device("cuda", 0)
    hbm, tflops, peak_kind = peaks()
    out = {"workload": args.workload, "peak_gbs": hbm, "peak_kind": peak_kind, "results": []}
    if args.workload == "qgemv":
        for N in (14336, 4096):
            K = 4096
            copies = max(2, int(4 * 126e6 // (N * K * 9 // 16)) + 1)
            Ws = []
            for c in range(copies):
                P, S, B = synth.dense(c, N, K)
                Ws.append(qmoe.QMatrix.from_numpy(P, S, B, N, K, 4, dev))
            nbytes = N * K // 2 + 2 * N * (K // 64) * 2
            for Bt in [int(b) for b in args.qgemv_batch.split(",")]:
                x = torch.from_numpy(synth.activations(Bt, Bt, K).view(np.float16).copy()).to(dev)
                y = torch.empty(Bt, N, dtype=torch.float16, device=dev)

                def run():
                    for W in Ws:
                        qmoe.qgemv_affine(W, x, y)
                run()
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    run()
                for _ in range(3):
                    g.replay()
                reps = max(10, args.steps // 10)
                ms = timed_replays(g.replay, reps) / (reps * copies)
                gbs = (nbytes + Bt * K * 2 + Bt * N * 2) / (ms / 1e3) / 1e9
                out["results"].append({"N": N, "K": K, "B": Bt, "us": round(ms * 1e3, 3),
                                       "GB/s": round(gbs, 1), "frac": round(gbs / hbm, 4),
                                       "rotated_copies": copies})
        # the small case: N=512, K=1024, batch 1 (295 KB of weights, which fit
        # L2): hot (the same matrix every call) and cold (L2 flushed by a
        # 2 x L2 write before each call, the call alone timed)
        N, K = 512, 1024
        P, S, B = synth.dense(0, N, K)
        W = qmoe.QMatrix.from_numpy(P, S, B, N, K, 4, dev)
        x = torch.from_numpy(synth.activations(1, 1, K).view(np.float16).copy()).to(dev)
        y = torch.empty(1, N, dtype=torch.float16, device=dev)
        nbytes = N * K // 2 + 2 * N * (K // 64) * 2 + (K + N) * 2

        def run_small():
            for _ in range(20):
                qmoe.qgemv_affine(W, x, y)
        run_small()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            run_small()
        for _ in range(3):
            g.replay()
        reps = max(10, args.steps // 10)
        hot_ms = timed_replays(g.replay, reps) / (reps * 20)
        flush = torch.empty(2 * torch.cuda.get_device_properties(dev).L2_cache_size,
                            dtype=torch.uint8, device=dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        cold = []
        for i in range(max(20, args.steps // 5)):
            flush.fill_(i & 255)
            e0.record()
            qmoe.qgemv_affine(W, x, y)
            e1.record()
            e1.synchronize()
            cold.append(e0.elapsed_time(e1))
        cold_ms = float(np.median(cold))
        out["results"].append({"N": N, "K": K, "B": 1, "us_hot": round(hot_ms * 1e3, 3),
                               "us_cold": round(cold_ms * 1e3, 3),
                               "GB/s_cold": round(nbytes / (cold_ms / 1e3) / 1e9, 1),
                               "frac_cold": round(nbytes / (cold_ms / 1e3) / 1e9 / hbm, 4)})
    elif args.workload == "qgemv_fmt":
        # bf16-scale formats with the block-32 rotation of x, the K=4096 dense shapes
        for fmt, name in ((qmoe.FMT_ZP4_BF16, "zp4_bf16"), (qmoe.FMT_SYM8_BF16, "sym8_bf16")):
            bits = 4 if fmt == qmoe.FMT_ZP4_BF16 else 8
            for N in (14336, 4096):
                K = 4096
                nbytes = N * K * bits // 8 + N * (K // 64) * 4
                copies = max(2, int(4 * 126e6 // nbytes) + 1)
                Ws = []
                for c in range(copies):
                    P, prm, sg = synth.qmatrix_fmt(synth.rng(c, N, fmt), N, K, fmt)
                    Ws.append(qmoe.QMatrixFmt.from_numpy(P, prm, sg, N, K, fmt, device=dev))
                for Bt in (1, 8, 32):
                    x = torch.from_numpy(synth.activations(Bt, Bt, K).view(np.float16).copy()).to(dev)
                    y = torch.empty(Bt, N, dtype=torch.float16, device=dev)

                    def run():
                        for W in Ws:
                            qmoe.qgemv_fmt(W, x, y)
                    run()
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g):
                        run()
                    for _ in range(3):
                        g.replay()
                    reps = max(10, args.steps // 10)
                    ms = timed_replays(g.replay, reps) / (reps * copies)
                    gbs = (nbytes + K // 8 + Bt * K * 2 + Bt * N * 2) / (ms / 1e3) / 1e9
                    out["results"].append({"format": name, "rotation": True, "N": N, "K": K,
                                           "B": Bt, "us": round(ms * 1e3, 3),
                                           "GB/s": round(gbs, 1), "frac": round(gbs / hbm, 4),
                                           "rotated_copies": copies})
                del Ws
    elif args.workload == "expert_parallel":
        # one 128-expert layer split over `world` ranks: every rank's share
        # (moe_expert_qmlp_ep) timed on this GPU, rotating over 8 layers so the
        # weights come from HBM; the all-reduce of the 11 KB partial is not
        # included (it needs the other GPUs)
        nl = 8
        ms_l = [synth.moe_layer(args.seed, l) for l in range(nl)]
        xs = [torch.from_numpy(synth.activations(args.seed, 1, H, layer=l).view(np.float16).copy())
              .to(dev).reshape(-1) for l in range(nl)]
        routed = []
        for l in range(nl):
            G = qmoe.MoELayer.from_numpy(ms_l[l], E, H, I, device=dev)
            idx, wt, _ = qmoe.moe_router_topk(G.router, xs[l].reshape(1, -1), TOPK)
            routed.append((idx.reshape(-1), wt.reshape(-1)))
            del G
        for world in (1, 2, 4, 8):
            times = []
            for r in range(world):
                Gs = [qmoe.MoELayer.from_numpy(ms_l[l], E, H, I, device=dev, rank=r, world=world)
                      for l in range(nl)]
                ws = qmoe.expert_workspace(Gs[0], TOPK, dev)
                yp = torch.empty(H, dtype=torch.float32, device=dev)

                def run():
                    for l in range(nl):
                        qmoe.moe_expert_qmlp_ep(Gs[l], xs[l], routed[l][0], routed[l][1], r, world,
                                                yp, ws)
                run()
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    run()
                for _ in range(3):
                    g.replay()
                reps = max(10, args.steps // 10)
                times.append(timed_replays(g.replay, reps) / (reps * nl) * 1e3)
                del Gs, g
            out["results"].append({"world": world, "us_per_rank": [round(t, 2) for t in times],
                                   "us_max_rank": round(max(times), 2)})
    elif args.workload == "expert_cache":
        # one 128-expert H=2816 layer with its routed experts in pinned host memory and
        # 16 device slots; decode tokens whose routing locality is set by rho
        m = synth.moe_layer(args.seed, 0)
        for rho in (0.0, 0.9, 0.99):
            layer = qmoe.ExpertCacheLayer(m, E, H, I, nslots=16, device=dev)
            T = 48
            x16 = synth.correlated_tokens(args.seed, T, H, rho)
            xs = torch.from_numpy(x16.view(np.float16).copy()).to(dev)
            y = torch.empty(H, dtype=torch.float16, device=dev)
            for t in range(8):   # warm-up: fills the cache
                layer.forward(xs[t], TOPK, y)
            h0, m0, b0, _ = layer.stats()
            torch.cuda.synchronize()
            t0 = time.perf_counter()
            for t in range(8, T):
                layer.forward(xs[t], TOPK, y)
            torch.cuda.synchronize()
            el = time.perf_counter() - t0
            h1, m1, b1, _ = layer.stats()
            n = T - 8
            out["results"].append({
                "rho": rho, "tokens": n, "us_per_layer": round(el / n * 1e6, 1),
                "layers_per_s": round(n / el, 1),
                "hit_rate": round((h1 - h0) / max(1, (h1 - h0) + (m1 - m0)), 4),
                "misses_per_layer": round((m1 - m0) / n, 2),
                "h2d_GB/s": round((b1 - b0) / el / 1e9, 2)})
            del layer
    elif args.workload == "router":
        P, S, B = synth.router(args.seed)
        R = qmoe.QMatrix.from_numpy(P, S, B, E, H, 8, dev)
        for T in [int(t) for t in args.router_tokens.split(",")]:
            x = torch.from_numpy(synth.activations(T, T, H).view(np.float16).copy()).to(dev)
            idx = torch.empty(T, TOPK, dtype=torch.int32, device=dev)
            wt = torch.empty(T, TOPK, dtype=torch.float32, device=dev)

            def run():
                qmoe.moe_router_topk(R, x, TOPK, idx, wt)
            run()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for _ in range(20):
                    run()
            g.replay()
            reps = 50
            ms = timed_replays(g.replay, reps) / (reps * 20)
            out["results"].append({"T": T, "us": round(ms * 1e3, 3),
                                   "tokens_per_s": round(T / (ms / 1e3), 1)})
    elif args.workload == "prefill":
        # 128-token chunk through one 128-expert layer, rotating over 4 layers
        # (1.7 GB of weights) so consecutive calls do not find their experts in
        # L2.  Routings: the pages' Zipf(1.1) draw, and a dense one (every token
        # to experts 0..7: nine 128-token slots, the tensor-bound case).  Paths:
        # streaming kernels only, and experts with >= 16 tokens on tcgen05.
        nl = 4
        Gs = [qmoe.MoELayer.from_numpy(synth.moe_layer(args.seed, l), E, H, I, dev)
              for l in range(nl)]
        idx_z, wt_z = synth.zipf_routing(args.seed)
        T = idx_z.shape[0]
        idx_d = np.tile(np.arange(TOPK, dtype=np.int32), (T, 1))
        x = torch.from_numpy(synth.activations(args.seed, T, H).view(np.float16).copy()).to(dev)
        y = torch.empty(T, H, dtype=torch.float16, device=dev)
        ws = torch.empty(qmoe.moe_prefill_workspace_bytes(Gs[0], T, TOPK), dtype=torch.uint8,
                         device=dev)
        flops = 2.0 * (T * TOPK + T) * 3 * I * H
        old_min = qmoe.qmoe_set_prefill_tensor_min(0)
        try:
            for routing, idx_np in (("zipf1.1", idx_z), ("dense_experts_0_7", idx_d)):
                idx = torch.from_numpy(idx_np).to(dev)
                wt = torch.from_numpy(wt_z).to(dev)
                for tmin in (0, qmoe.TENSOR_MIN_DEFAULT):
                    qmoe.qmoe_set_prefill_tensor_min(tmin)

                    def run():
                        for G in Gs:
                            qmoe.moe_prefill_qgemm(G, x, idx, wt, y, ws)
                    run()
                    torch.cuda.synchronize()
                    assert qmoe.qmoe_check_status() == 0
                    for _ in range(3):
                        run()
                    reps = max(5, args.steps // 50)
                    ms = timed_replays(run, reps) / (reps * nl)
                    counts = np.bincount(idx_np.ravel(), minlength=E)
                    touched = int((counts > 0).sum())
                    heavy = int((counts >= tmin).sum() + (T >= tmin)) if tmin else 0
                    nbytes = (touched + 1) * EXPERT_BYTES
                    gbs = nbytes / (ms / 1e3) / 1e9
                    # the attainable time: the slower of streaming the touched
                    # weights at the HBM peak and the useful flops at the
                    # dense bf16 peak
                    att_us = max(nbytes / (hbm * 1e9), flops / (tflops * 1e12)) * 1e6
                    out["results"].append({
                        "T": T, "routing": routing, "tensor_min_tokens": tmin,
                        "tensor_core_slots": heavy, "experts_touched": touched,
                        "us": round(ms * 1e3, 2), "tokens_per_s": round(T / (ms / 1e3), 1),
                        "weight_GB/s": round(gbs, 1), "frac_hbm": round(gbs / hbm, 4),
                        "useful_TFLOP/s": round(flops / (ms / 1e3) / 1e12, 2),
                        "attainable_us": round(att_us, 2),
                        "frac_attainable": round(att_us / (ms * 1e3), 4)})
        finally:
            qmoe.qmoe_set_prefill_tensor_min(old_min)
    else:
        out["error"] = "workload not available"
    print(json.dumps(out), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        main_reference(args)
    elif args.workload == "moe_decode":
        main_decode(args)
    else:
        main_other(args)


if __name__ == "__main__":
    main()
