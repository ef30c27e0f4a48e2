"""Benchmark of the fused 2-bit LLVQ GEMV on B200.

Workload: one 4096 x 4096 linear layer (K zero-padded to 4104 = 171 blocks of 24), 2-bit
budget (48-bit Leech index + 8-bit gain code per block, per-row 256-entry fp16 chi(24) gain
table), fp16 N(0,1) activations, batch 1.  Synthetic seeded data stands in for trained
weights.  One step = the fused GEMV over R distinct copies of the layer (together larger than
L2, so every launch streams its words from HBM), captured in one CUDA graph.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference]

N > 1 runs under torchrun as independent replicas (the product does not shard: one layer fits
one GPU); each rank times its own graph and rank 0 prints the max over ranks.  The reference
arm (--impl reference) times the CPU oracle on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fused 2-bit LLVQ GEMV effective GB/s and % of HBM roofline; decoded vectors/s"
ROWS, K = 4096, 4096
NB = -(-K // 24)
CONFIG_ID = 2
WORKLOAD = "llvq 2-bit fused GEMV, 4096x4096 layer (K padded to 4104), u8 gain table, batch 1"


def algorithmic_bytes(rows=ROWS, nb=NB, batch=1) -> int:
    """Bytes one launch must move: packed words (8 B/block), per-row gain tables (512 B),
    activations (fp16) and outputs (fp32)."""
    return rows * nb * 8 + rows * 512 + batch * nb * 24 * 2 + batch * rows * 4


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while the timed region runs."""

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        try:
            for line in open(self.path):
                f = [x.strip() for x in line.split(",")]
                if len(f) < 9:
                    continue
                try:
                    sm.append(float(f[1]))
                    mx = float(f[2])
                except ValueError:
                    continue
                for n, v in zip(names, f[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
            os.unlink(self.path)
        except Exception:
            pass
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def make_layer_copies(torch, codec, R, dev):
    from codebook_free_lattice_b200 import synth
    n = ROWS * NB
    lo, _ = synth.uniform_indices(synth.rng(CONFIG_ID, 0), n * R, codec.n_points, 48)
    codes = synth.gain_codes(synth.rng(CONFIG_ID, 1), n * R)
    words = torch.from_numpy(synth.pack_words(lo, None, codes, 48).view(np.int64)).to(dev)
    words = words.view(R, ROWS, NB)
    gains = torch.from_numpy(synth.chi24_tables(synth.rng(CONFIG_ID, 2), ROWS).view(np.int16)).to(dev)
    xs = synth.activations(synth.rng(CONFIG_ID, 3), R, K)       # one activation row per copy
    return words, gains, xs


def decode_throughput(torch, codec, dev, n, steps, warmup):
    """llvq_decode on n seeded uniform 48-bit indices (int8 [n, 24] out), CUDA-event timed."""
    from codebook_free_lattice_b200 import synth
    lo, _ = synth.uniform_indices(synth.rng(4, 0), n, codec.n_points, 48)
    w = torch.from_numpy(lo.view(np.int64)).to(dev)
    out = torch.empty((n, 24), dtype=torch.int8, device=dev)
    for _ in range(max(warmup, 1)):
        codec.decode(w, out)
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(steps):
        codec.decode(w, out)
    e.record()
    torch.cuda.synchronize()
    t = s.elapsed_time(e) / 1e3 / max(steps, 1)
    return {"n": n, "us_per_launch": t * 1e6, "decoded_vectors_per_s": n / t,
            "GBps": n * 32 / t / 1e9}


def cpu_baseline(steps_seconds=12.0):
    """The oracle (fp64, plain C) on a bounded sample of the same workload: whole rows of the
    layer, decoded and multiplied on every host core, timed until ~steps_seconds of work."""
    import oracle
    from codebook_free_lattice_b200 import synth
    oc = oracle.Codec(48)
    cores = os.cpu_count() or 1
    rows = min(64 * cores, ROWS)
    n = rows * NB
    lo, _ = synth.uniform_indices(synth.rng(CONFIG_ID, 0), n, oc.n_points, 48)
    codes = synth.gain_codes(synth.rng(CONFIG_ID, 1), n)
    words = synth.pack_words(lo, None, codes, 48).reshape(rows, NB)
    gains = synth.chi24_tables(synth.rng(CONFIG_ID, 2), ROWS)[:rows]
    x = synth.activations(synth.rng(CONFIG_ID, 3), 1, K)
    done_rows, t0 = 0, time.perf_counter()
    while True:
        oc.gemm(words, NB, 1, gains, x, 1, threads=cores)
        done_rows += rows
        el = time.perf_counter() - t0
        if el > steps_seconds:
            break
    bytes_per_row = NB * 8 + 512
    gbs = done_rows * bytes_per_row / el / 1e9
    return {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{done_rows} rows of the 4096x4104 layer ({rows} rows per pass, all cores), "
                      f"{el:.1f} s; GB/s of packed words + gain tables processed",
            "vectors_per_s": done_rows * NB / el}


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    t0 = time.perf_counter()
    per_step = max(2.0, min(20.0, 150.0 / max(args.steps + args.warmup, 1)))
    for _ in range(args.warmup):
        cpu_baseline(per_step / 4)
    vals = [cpu_baseline(per_step) for _ in range(args.steps)]
    v = statistics.median(x["value"] for x in vals)
    ms = statistics.median(algorithmic_bytes() / (x["value"] * 1e9) * 1e3 for x in vals)
    cb = dict(vals[0])
    cb["value"] = v
    line = {"metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": WORKLOAD, "rows": ROWS, "cols": K, "batch": 1, "index_bits": 48},
            "cpu_baseline": cb,
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "wall_s": time.perf_counter() - t0}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="llvq", choices=["llvq", "reference"])
    ap.add_argument("--copies", type=int, default=0, help="layer copies per step (0: > 3x L2)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--decode-n", type=int, default=28672 * 342,
                    help="indices for the llvq_decode throughput line (default: the 28672x8192 layer)")
    ap.add_argument("--mode", default="gemv", choices=["gemv", "decode"],
                    help="decode: time llvq_decode alone (profiling aid)")
    args = ap.parse_args()

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch
    import torch.distributed as dist
    if world > 1:
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    import codebook_free_lattice_b200 as L
    codec = L.Codec(48)
    if args.mode == "decode":
        r = decode_throughput(torch, codec, dev, args.decode_n, args.steps, args.warmup)
        if rank == 0:
            print(json.dumps({"mode": "decode", **r}), flush=True)
        return 0

    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    layer_bytes = ROWS * NB * 8
    R = args.copies or int(np.ceil(3 * l2 / layer_bytes)) + 1
    words, gains, xs = make_layer_copies(torch, codec, R, dev)
    x_dev = torch.from_numpy(xs.view(np.int16)).to(dev)                 # [R, K_pad]
    y_dev = torch.empty((R, ROWS), dtype=torch.float32, device=dev)
    ws = [codec.weight(words[i], gains, ROWS, K, L.LLVQ_GAIN_U8_TABLE) for i in range(R)]

    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        for i in range(R):                                              # warm the path once
            codec.gemv(ws[i], x_dev[i], y_dev[i], stream=stream)
    stream.synchronize()
    assert codec.get_error(stream) == 0
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(R):
            codec.gemv(ws[i], x_dev[i], y_dev[i], stream=stream)

    def barrier():
        if world > 1:
            dist.barrier()

    def time_steps(n, body):
        barrier()
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        for _ in range(n):
            body()
        e.record(stream)
        torch.cuda.synchronize()
        barrier()
        return s.elapsed_time(e) / 1e3

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            graph.replay()
        with ClockSampler(torch.cuda.current_device()) as clocks:
            secs = time_steps(args.steps, graph.replay)
    clk = clocks.summary()

    # end to end through the public API: pinned host activations in, outputs back out
    x_host = torch.from_numpy(xs.view(np.int16)).pin_memory()
    y_host = torch.empty((R, ROWS), dtype=torch.float32).pin_memory()

    def e2e_step():
        x_dev.copy_(x_host, non_blocking=True)
        graph.replay()
        y_host.copy_(y_dev, non_blocking=True)

    with torch.cuda.stream(stream):
        for _ in range(max(args.warmup, 1)):
            e2e_step()
        secs_e2e = time_steps(args.steps, e2e_step)

    if world > 1:
        t = torch.tensor([secs, secs_e2e], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        secs, secs_e2e = t.tolist()

    launches = args.steps * R
    bytes_launch = algorithmic_bytes()
    per_launch_s = secs / launches
    gbs = bytes_launch / per_launch_s / 1e9
    value = gbs * world
    peak, peak_kind = measured_peaks()
    h2d = R * NB * 24 * 2
    d2h = R * ROWS * 4
    e2e_gbs = bytes_launch * launches / secs_e2e / 1e9 * world

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": WORKLOAD, "rows": ROWS, "cols": K, "blocks_per_row": NB,
                       "batch": 1, "index_bits": 48, "layer_copies_per_step": R,
                       "l2_policy": f"inputs larger than L2: {R} distinct layer copies "
                                    f"({R * layer_bytes / 2**20:.0f} MiB of words) per step",
                       "parallelism": f"replicas x{world}"},
            "us_per_layer": per_launch_s * 1e6,
            "decoded_vectors_per_s": ROWS * NB / per_launch_s * world,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s",
                         "frac": gbs / peak, "traffic": None,
                         "peak_source": f"{peak_kind} hbm_gbs (MEASURED_PEAKS.json)"},
            "e2e": {"value": e2e_gbs, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": launches,
            "clocks": clk,
        }
        line["decode"] = decode_throughput(torch, codec, dev, args.decode_n, 5, 2)
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline()
        print(json.dumps(line), flush=True)
    del graph
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
