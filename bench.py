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


def workload(rows=None, cols=None, batch=1) -> str:
    rows, cols = rows or ROWS, cols or K
    return (f"llvq 2-bit fused GEMV, {rows}x{cols} layer (K padded to {-(-cols // 24) * 24}), u8 gain table, "
            f"batch {batch}")


WORKLOAD = workload()


def algorithmic_bytes(rows=None, nb=None, batch=1) -> int:
    """Bytes one launch must move: packed words (8 B/block), per-row gain tables (512 B),
    activations (fp16) and outputs (fp32)."""
    rows, nb = rows or ROWS, nb or NB
    return rows * nb * 8 + rows * 512 + batch * nb * 24 * 2 + batch * rows * 4


def max_over_ranks(dist, values, device):
    """Each timing's maximum over all ranks (every rank runs the same steps; the slowest one
    bounds the whole job)."""
    import torch
    t = torch.tensor(list(values), device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_gbps(bytes_per_launch, launches_per_rank, secs, world):
    """Whole-job throughput: every rank streams the same number of launches, the time is the
    max over ranks, so the job moves world times the per-rank bytes in that time."""
    return bytes_per_launch * launches_per_rank * world / secs / 1e9


def kernel_sources_hash() -> str:
    """Hash of the library sources with comments and blank lines removed, so that the committed
    ncu record stays tied to the code it was measured on and not to its comments."""
    import glob
    import hashlib
    import re
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "codebook_free_lattice_b200", "csrc", "*"))):
        h.update(os.path.basename(f).encode())
        with open(f, encoding="utf-8") as fh:
            src = fh.read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        lines = [" ".join(line.split()) for line in src.splitlines()]
        h.update("\n".join(line for line in lines if line).encode())
    return h.hexdigest()


def profile_record():
    """The committed ncu record of the metric's kernel (DRAM bytes and warp instructions per
    launch), or None when the kernel sources changed since the capture."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)
        if rec.get("kernel_sources_sha256") == kernel_sources_hash():
            return rec
    except Exception:
        pass
    return None


def search_record():
    """The committed ncu record of the search kernel ("search" in profiles/traffic.json), keyed by
    the kernel sources like profile_record, or None when they changed since the capture."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f).get("search")
        if rec and rec.get("kernel_sources_sha256") == kernel_sources_hash():
            return rec
    except Exception:
        pass
    return None


def measured_traffic():
    rec = profile_record()
    return int(rec["traffic_bytes_per_launch"]) if rec else None


def issue_roofline(per_launch_s, sm_mhz, sms):
    """Instruction-issue roofline of the metric's kernel: thread-instructions per second (ncu count
    of one launch / the measured launch time) against sms SMs x 4 schedulers x 32 lanes x the SM
    clock measured during the timed region (one warp-instruction per scheduler and cycle)."""
    rec = profile_record()
    if not rec or "warp_instructions_per_launch" not in rec or not sm_mhz:
        return None
    achieved = rec["warp_instructions_per_launch"] * 32 / per_launch_s
    peak = sms * 4 * 32 * sm_mhz * 1e6
    return {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "thread-instructions/s",
            "frac": achieved / peak,
            "peak_source": f"{sms} SMs x 4 schedulers x 32 lanes x {sm_mhz:.0f} MHz (clock measured under load)"}


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


def make_layer_copies(torch, codec, R, dev, batch=1):
    from codebook_free_lattice_b200 import synth
    n = ROWS * NB
    lo, _ = synth.uniform_indices(synth.rng(CONFIG_ID, 0), n * R, codec.n_points, 48)
    codes = synth.gain_codes(synth.rng(CONFIG_ID, 1), n * R)
    words = torch.from_numpy(synth.pack_words(lo, None, codes, 48).view(np.int64)).to(dev)
    words = words.view(R, ROWS, NB)
    gains = torch.from_numpy(synth.chi24_tables(synth.rng(CONFIG_ID, 2), ROWS).view(np.int16)).to(dev)
    xs = synth.activations(synth.rng(CONFIG_ID, 3), R * batch, K).reshape(R, batch, -1)  # per copy
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


def encode_throughput(torch, codec, dev, n, steps, warmup):
    """llvq_encode on the n lattice points llvq_decode gives for seeded uniform 48-bit indices
    (int8 [n, 24] in, packed words out), CUDA-event timed; the round trip must return the indices."""
    from codebook_free_lattice_b200 import synth
    lo, _ = synth.uniform_indices(synth.rng(5, 0), n, codec.n_points, 48)
    w = torch.from_numpy(lo.view(np.int64)).to(dev)
    vecs = torch.empty((n, 24), dtype=torch.int8, device=dev)
    codec.decode(w, vecs)
    out = torch.empty(n, dtype=torch.int64, device=dev)
    for _ in range(max(warmup, 1)):
        codec.encode(vecs, out)
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(steps):
        codec.encode(vecs, out)
    e.record()
    torch.cuda.synchronize()
    if not torch.equal(out, w) or codec.get_error() != 0:
        raise RuntimeError("llvq_encode did not invert llvq_decode")
    t = s.elapsed_time(e) / 1e3 / max(steps, 1)
    return {"n": n, "us_per_launch": t * 1e6, "encoded_vectors_per_s": n / t, "GBps": n * 32 / t / 1e9}


def cpu_model() -> str:
    """The host CPU's model name (first /proc/cpuinfo entry)."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def cpu_baseline(steps_seconds=12.0, one_core_seconds=3.0):
    """The oracle (fp64, plain C) on a bounded sample of the same workload: whole rows of the
    layer, decoded and multiplied on every host core, timed until ~steps_seconds of work; then,
    when one_core_seconds > 0, the same on one core for ~one_core_seconds."""
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
    out = {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle",
           "sample": f"{done_rows} rows of the 4096x4104 layer ({rows} rows per pass, all cores), "
                     f"{el:.1f} s; GB/s of packed words + gain tables processed",
           "vectors_per_s": done_rows * NB / el, "cpu_model": cpu_model()}
    if one_core_seconds > 0:
        r1 = min(8, rows)
        done1, t1 = 0, time.perf_counter()
        while True:
            oc.gemm(words[:r1], NB, 1, gains[:r1], x, 1, threads=1)
            done1 += r1
            el1 = time.perf_counter() - t1
            if el1 > one_core_seconds:
                break
        out["one_core"] = {"value": done1 * bytes_per_row / el1 / 1e9, "unit": "GB/s",
                           "vectors_per_s": done1 * NB / el1,
                           "sample": f"{done1} rows, {el1:.1f} s on one core"}
    return out


# ------------------------------------------------------------------ nearest-point search
# The pages' Gaussian-source experiment at 2 bits per dimension: spherical clipping spends all
# 48 bits of a block on the index (shells 2..13, Euclidean criterion, reconstruction c v); the
# shape-gain split gives 1 or 2 bits to a scalar gain and the rest to the direction (angular
# criterion over shells 2..12, 46.66 bits, or 2..11, 45.20 bits).
SEARCH_N = 1 << 17
SEARCH_TRAIN = 1 << 16
# Algorithmic fp64 FMAs per searched vector: over every (class, codeword) pair of shells 2..M
# (4096 codewords for an odd class, those of weight k for an even one), one FMA per nonzero
# magnitude group and one for the criterion (the even classes' data-dependent sign turn is left
# out).  Counted from the class list of the 48-bit union: 921,486 pairs at M = 13.
SEARCH_FMAS = {11: 2081740, 12: 2857480, 13: 3805180}
FP64_FMA_PER_SM_CLK = 64      # ncu: sm__sass_thread_inst_executed_op_dfma_pred_on.sum.peak_sustained / SMs
SEARCH_CONFIGS = [
    # name, criterion, max_shell, gain bits
    ("spherical clipping", 1, 13, 0),
    ("shape-gain, 1 gain bit", 0, 12, 1),
    ("shape-gain, 2 gain bits", 0, 11, 2),
]


def _search(torch, codec, X, max_shell, mode, scale, levels=None):
    n = X.shape[0]
    P = torch.empty((n, 24), dtype=torch.int8, device=X.device)
    D = torch.empty(n, dtype=torch.float64, device=X.device)
    codes = None if levels is None else torch.empty(n, dtype=torch.uint8, device=X.device)
    codec.search(X, P, max_shell, mode, scale, dots=D, levels=levels, codes=codes)
    return P, D, codes


def search_quality(torch, codec, dev):
    """MSE per dimension, SQNR (bits) and share of the Shannon bound (2 bits) on SEARCH_N test
    blocks; the scale c (clipping) and the gain levels (shape-gain, Lloyd-Max on the best gains
    <x, v> / |v|) are fitted on SEARCH_TRAIN other blocks."""
    from codebook_free_lattice_b200 import synth
    import math
    Xtr = torch.from_numpy(synth.gaussian_blocks(synth.rng(60, 4), SEARCH_TRAIN)).to(dev)
    Xte = torch.from_numpy(synth.gaussian_blocks(synth.rng(61, 4), SEARCH_N)).to(dev)
    out = []
    for name, mode, ms, gbits in SEARCH_CONFIGS:
        if mode == 1:
            def mse(c, X):
                P, _, _ = _search(torch, codec, X, ms, 1, c)
                return float(((X.double() - c * P.double()) ** 2).mean())
            lo, hi = 0.15, 0.60                                   # golden-section search for c
            r = (math.sqrt(5) - 1) / 2
            a, b = hi - r * (hi - lo), lo + r * (hi - lo)
            fa, fb = mse(a, Xtr), mse(b, Xtr)
            for _ in range(18):
                if fa < fb:
                    hi, b, fb = b, a, fa
                    a = hi - r * (hi - lo)
                    fa = mse(a, Xtr)
                else:
                    lo, a, fa = a, b, fb
                    b = lo + r * (hi - lo)
                    fb = mse(b, Xtr)
            c = (lo + hi) / 2
            m = mse(c, Xte)
            extra = {"scale": c}
            index_bits = 47.997
        else:
            P, D, _ = _search(torch, codec, Xtr, ms, 0, 1.0)
            g = (D / P.double().pow(2).sum(1).sqrt()).cpu().numpy()
            L = np.quantile(g, (np.arange(2 ** gbits) + 0.5) / 2 ** gbits)   # Lloyd-Max levels
            for _ in range(100):
                idx = np.argmin(np.abs(g[:, None] - L[None, :]), axis=1)
                L = np.array([g[idx == k].mean() if (idx == k).any() else L[k] for k in range(L.size)])
            lev = torch.tensor(L, dtype=torch.float64, device=dev)
            P, D, codes = _search(torch, codec, Xte, ms, 0, 1.0, lev)
            V = P.double()
            Xh = lev[codes.long()][:, None] * V / V.pow(2).sum(1, keepdim=True).sqrt()
            m = float(((Xte.double() - Xh) ** 2).mean())
            g_exact = D / V.pow(2).sum(1).sqrt()
            shape_only = float(((Xte.double() - g_exact[:, None] * V / V.pow(2).sum(1, keepdim=True).sqrt()) ** 2).mean())
            extra = {"gain_levels": [round(float(x), 4) for x in L], "mse_exact_gain": shape_only}
            index_bits = {11: 45.205, 12: 46.658}[ms]
        sq = -0.5 * math.log2(m)
        out.append({"config": name, "max_shell": ms, "bits_per_dim": (index_bits + gbits) / 24,
                    "mse": m, "sqnr_bits": sq, "shannon_retention": sq / 2.0, **extra})
    return {"source": f"N(0, I_24), {SEARCH_N} test blocks (fit on {SEARCH_TRAIN} others)", "results": out}


def search_throughput(torch, codec, dev, steps, warmup, max_shell=13, mode=1, scale=0.3):
    """llvq_search on SEARCH_N Gaussian blocks, CUDA events around each launch on the launching
    stream; L2 flushed (a 3x L2 buffer written) before every launch, outside the timed span."""
    from codebook_free_lattice_b200 import synth
    X = torch.from_numpy(synth.gaussian_blocks(synth.rng(62, 4), SEARCH_N)).to(dev)
    P = torch.empty((SEARCH_N, 24), dtype=torch.int8, device=dev)
    D = torch.empty(SEARCH_N, dtype=torch.float64, device=dev)
    flush = torch.empty(3 * torch.cuda.get_device_properties(dev).L2_cache_size // 4, dtype=torch.int32, device=dev)
    stream = torch.cuda.Stream(device=dev)
    total = 0.0
    with torch.cuda.stream(stream):
        for i in range(warmup + steps):
            flush.fill_(i)
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record(stream)
            codec.search(X, P, max_shell, mode, scale, dots=D, stream=stream)
            e.record(stream)
            e.synchronize()
            if i >= warmup:
                total += s.elapsed_time(e) / 1e3
    if codec.get_error(stream) != 0:
        raise RuntimeError("llvq_search raised a device flag")
    t = total / steps
    return {"n": SEARCH_N, "max_shell": max_shell, "criterion": "euclidean" if mode else "angular",
            "ms_per_launch": t * 1e3, "vectors_per_s": SEARCH_N / t}


def search_roofline(r, sm_mhz, sms):
    """fp64 roofline of the search kernel: algorithmic FMAs (SEARCH_FMAS) x 2 per second against
    sms x 64 fp64 FMA lanes x 2 x the SM clock measured under load; DRAM traffic per launch from
    the committed ncu record when it matches the sources."""
    flops = 2.0 * SEARCH_FMAS[r["max_shell"]] * r["n"]
    achieved = flops / (r["ms_per_launch"] / 1e3) / 1e12
    peak = sms * FP64_FMA_PER_SM_CLK * 2 * sm_mhz * 1e6 / 1e12
    rec = search_record()
    return {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "traffic": rec["traffic_bytes_per_launch"] if rec and rec.get("n") == r["n"] else None,
            "peak_source": f"{sms} SMs x {FP64_FMA_PER_SM_CLK} fp64 FMA/clk x 2 x {sm_mhz:.0f} MHz (clock under load)",
            "algorithmic": f"{SEARCH_FMAS[r['max_shell']]} fp64 FMAs per vector (class-codeword pairs x (groups + 1))"}


def search_cpu_baseline(seconds=12.0, max_shell=13, mode=1, scale=0.3):
    """The oracle's search (plain C, fp64) on all host cores, on a bounded sample of the same
    Gaussian blocks, timed until ~seconds of work."""
    import oracle
    from codebook_free_lattice_b200 import synth
    oc = oracle.Codec(48)
    cores = os.cpu_count() or 1
    X = synth.gaussian_blocks(synth.rng(62, 4), 4 * cores)
    done, t0 = 0, time.perf_counter()
    while True:
        oc.search(X, max_shell, mode, scale, threads=cores)
        done += X.shape[0]
        el = time.perf_counter() - t0
        if el > seconds:
            break
    return {"value": done / el, "unit": "vectors/s", "cores": cores, "kind": "oracle",
            "sample": f"{done} of the Gaussian blocks ({X.shape[0]} per pass, all cores), {el:.1f} s",
            "cpu_model": cpu_model()}


# ------------------------------------------------------------------ Spherical GPTQ pass
GPTQ_ROWS, GPTQ_COLS, GPTQ_SHELL = 4096, 4104, 12


def gptq_inputs(torch, dev, rows, cols, seed=70):
    """Gaussian weights and the Cholesky factor U (H^-1 = U^T U) of a synthetic calibration
    Hessian H = X X^T / n + damping over correlated inputs; U is prepared with library routines
    (torch.linalg) outside any timed region."""
    from codebook_free_lattice_b200 import synth
    g = synth.rng(seed, 4)
    W = torch.from_numpy(g.standard_normal((rows, cols))).to(dev)
    X = torch.from_numpy(g.standard_normal((cols, 2 * cols))).to(dev)
    X = X * torch.linspace(0.3, 2.0, cols, dtype=torch.float64, device=dev)[:, None]
    X[1:] += 0.5 * X[:-1].clone()
    H = X @ X.T / X.shape[1]
    H += 0.05 * H.diagonal().mean() * torch.eye(cols, dtype=torch.float64, device=dev)
    U = torch.linalg.cholesky(torch.linalg.inv(H)).T.contiguous()
    return W, U


def gptq_throughput(torch, codec, dev, steps, warmup):
    """One Spherical GPTQ pass over a 4096 x 4104 layer per step (fp64), CUDA events per pass; each
    pass starts from a fresh copy of the weights (the copy is outside the timed span)."""
    rows, cols = GPTQ_ROWS, GPTQ_COLS
    W0, U = gptq_inputs(torch, dev, rows, cols)
    W = torch.empty_like(W0)
    nb = cols // 24
    P = torch.empty((rows, nb, 24), dtype=torch.int8, device=dev)
    N = torch.empty((rows, nb), dtype=torch.float64, device=dev)
    ws = None
    stream = torch.cuda.Stream(device=dev)
    total = 0.0
    with torch.cuda.stream(stream):
        for i in range(warmup + steps):
            W.copy_(W0)
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record(stream)
            ws = codec.spherical_gptq(W, U, P, N, GPTQ_SHELL, workspace=ws, stream=stream)
            e.record(stream)
            e.synchronize()
            if i >= warmup:
                total += s.elapsed_time(e) / 1e3
    if codec.get_error(stream) != 0:
        raise RuntimeError("llvq_spherical_gptq raised a device flag")
    t = total / steps
    upd = rows * 24 * sum(cols - 24 * (b + 1) for b in range(nb))        # propagation FMAs
    gmat = sum((cols - 24 * (b + 1)) * 276 for b in range(nb))             # back substitution FMAs
    fmas = rows * nb * SEARCH_FMAS[GPTQ_SHELL] + upd + gmat
    return {"rows": rows, "cols": cols, "max_shell": GPTQ_SHELL, "ms_per_pass": t * 1e3,
            "weights_per_s": rows * cols / t, "fp64_fmas_per_pass": fmas,
            "search_share_of_fmas": rows * nb * SEARCH_FMAS[GPTQ_SHELL] / fmas}


def gptq_cpu_baseline(rows=2, cols=960):
    """The oracle's pass on a bounded sample (rows x cols of the same kind of layer, one core)."""
    import oracle
    import torch
    W, U = gptq_inputs(torch, torch.device("cpu"), rows, cols)
    oc = oracle.Codec(48)
    t0 = time.perf_counter()
    oc.spherical_gptq(W.numpy(), U.numpy(), GPTQ_SHELL)
    el = time.perf_counter() - t0
    return {"value": rows * cols / el, "unit": "weights/s", "cores": 1, "kind": "oracle",
            "sample": f"one pass over a {rows} x {cols} layer ({rows * cols // 24} blocks), {el:.1f} s",
            "cpu_model": cpu_model()}


# ------------------------------------------------------------------ secondary measurements
SWEEP_CASES = [
    # (name, rows, K, index_bits, batch)
    ("4096x4096", 4096, 4096, 48, 1),
    ("11008x4096 (gate/up)", 11008, 4096, 48, 1),
    ("11008x4096 (gate/up)", 11008, 4096, 48, 4),
    ("4096x11008 (down)", 4096, 11008, 48, 1),
    ("4096x11008 (down)", 4096, 11008, 48, 4),
    ("28672x8192", 28672, 8192, 48, 1),
    ("28672x8192", 28672, 8192, 48, 8),
    ("28672x8192", 28672, 8192, 48, 16),
    ("8192x28672", 8192, 28672, 48, 1),
    ("8192x28672", 8192, 28672, 48, 16),
    ("28672x8192", 28672, 8192, 72, 1),
    ("28672x8192", 28672, 8192, 72, 16),
    ("8192x28672", 8192, 28672, 72, 1),
    ("8192x28672", 8192, 28672, 72, 8),
    ("4096x4096", 4096, 4096, 96, 1),
    ("28672x8192", 28672, 8192, 96, 1),
    ("28672x8192", 28672, 8192, 96, 16),
    ("8192x28672", 8192, 28672, 96, 1),
    ("8192x28672", 8192, 28672, 96, 8),
]
LLAMA7B_LAYER = [("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
                 ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008)]


def _graph_time(torch, stream, body, reps=10, warm=3):
    with torch.cuda.stream(stream):
        body()
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        body()
    with torch.cuda.stream(stream):
        for _ in range(warm):
            g.replay()
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        for _ in range(reps):
            g.replay()
        e.record(stream)
    torch.cuda.synchronize()
    del g
    return s.elapsed_time(e) / 1e3 / reps


def _layers(torch, codec, dev, shapes, bits, batch, seed):
    """Packed words, table gains and activations for each (rows, K) in shapes (distinct data)."""
    import codebook_free_lattice_b200 as L
    from codebook_free_lattice_b200 import synth
    out = []
    for i, (rows, K) in enumerate(shapes):
        nb = -(-K // 24)
        lo, hi = synth.uniform_indices(synth.rng(seed + i, 0), rows * nb, codec.n_points, bits)
        codes = synth.gain_codes(synth.rng(seed + i, 1), rows * nb)
        w = torch.from_numpy(np.ascontiguousarray(synth.pack_words(lo, hi, codes, bits)).view(np.int64)).to(dev)
        g = torch.from_numpy(synth.chi24_tables(synth.rng(seed + i, 2), rows).view(np.int16)).to(dev)
        x = torch.from_numpy(synth.activations(synth.rng(seed + i, 3), batch, K).view(np.int16)).to(dev)
        y = torch.empty((batch, rows), dtype=torch.float32, device=dev)
        out.append((codec.weight(w, g, rows, K, L.LLVQ_GAIN_U8_TABLE), w, g, x, y))
    return out


def _run_layers(codec, layers, batch, stream):
    for wt, _, _, x, y in layers:
        if batch == 1:
            codec.gemv(wt, x, y, stream=stream)
        else:
            codec.gemm(wt, x, y, batch, stream=stream)


def sweep(torch, dev):
    """One JSON line per (layer, bits, batch): fused LLVQ product time against cuBLAS fp16
    (torch.matmul on identical shapes), inputs larger than L2 in both arms; then the full
    Llama-2-7B-shaped decoder stack (32 layers x q,k,v,o,gate,up,down) at 2, 3 and 4 bits."""
    import codebook_free_lattice_b200 as L
    peak, _ = measured_peaks()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    stream = torch.cuda.Stream(device=dev)
    codecs = {48: L.Codec(48), 72: L.Codec(72), 96: L.Codec(96)}
    for name, rows, K, bits, batch in SWEEP_CASES:
        codec = codecs[bits]
        nb = -(-K // 24)
        wb = 8 if bits == 48 else 16
        copies = max(1, int(np.ceil(3 * l2 / (rows * nb * wb))))
        layers = _layers(torch, codec, dev, [(rows, K)] * copies, bits, batch, 500 + rows % 97)
        t = _graph_time(torch, stream, lambda: _run_layers(codec, layers, batch, stream)) / copies
        assert codec.get_error(stream) == 0
        alg = rows * nb * wb + rows * 512 + batch * nb * 48 + batch * rows * 4
        del layers
        fcopies = max(1, int(np.ceil(3 * l2 / (rows * K * 2))))
        Ws = [torch.randn(rows, K, dtype=torch.float16, device=dev) for _ in range(fcopies)]
        xs = torch.randn(batch, K, dtype=torch.float16, device=dev)
        tc = _graph_time(torch, stream, lambda: [torch.matmul(xs, W.t()) for W in Ws]) / fcopies
        del Ws
        print(json.dumps({"sweep": name, "index_bits": bits, "batch": batch, "us": t * 1e6,
                          "GBps": alg / t / 1e9, "frac_hbm": alg / t / 1e9 / peak,
                          "fp16_equivalent_GBps": 2 * rows * K / t / 1e9,
                          "decoded_vectors_per_s": rows * nb / t, "cublas_fp16_us": tc * 1e6,
                          "speedup_vs_fp16": tc / t, "layer_copies": copies}), flush=True)
        torch.cuda.empty_cache()
    for bits in (48, 72, 96):
        codec = codecs[bits]
        shapes = [(r, k) for _ in range(32) for (_, r, k) in LLAMA7B_LAYER]
        layers = _layers(torch, codec, dev, shapes, bits, 1, 900 + bits)
        t = _graph_time(torch, stream, lambda: _run_layers(codec, layers, 1, stream), reps=5)
        assert codec.get_error(stream) == 0
        wb = 8 if bits == 48 else 16
        alg = sum(r * -(-k // 24) * wb + r * 512 + -(-k // 24) * 48 + r * 4 for r, k in shapes)
        del layers
        torch.cuda.empty_cache()
        Ws = [torch.randn(r, k, dtype=torch.float16, device=dev) for r, k in shapes]
        xs = {k: torch.randn(1, k, dtype=torch.float16, device=dev) for k in (4096, 11008)}
        tc = _graph_time(torch, stream, lambda: [torch.matmul(xs[W.shape[1]], W.t()) for W in Ws], reps=5)
        del Ws
        torch.cuda.empty_cache()
        print(json.dumps({"sweep": "llama-2-7b stack (224 GEMVs)", "index_bits": bits, "batch": 1,
                          "ms": t * 1e3, "GBps": alg / t / 1e9, "frac_hbm": alg / t / 1e9 / peak,
                          "cublas_fp16_ms": tc * 1e3, "speedup_vs_fp16": tc / t}), flush=True)
    print(json.dumps(oracle_stack(48)), flush=True)


def oracle_stack(bits=48):
    """The oracle (fp64, all host cores) on one Llama-2-7B-shaped decoder layer (q, k, v, o, gate,
    up, down GEMVs, u8 gain tables), times 32 for the stack: the whole stack would take minutes."""
    import oracle
    from codebook_free_lattice_b200 import synth
    oc = oracle.Codec(bits)
    cores = os.cpu_count() or 1
    secs, nbytes, blocks = 0.0, 0, 0
    for i, (_, rows, k) in enumerate(LLAMA7B_LAYER):
        nb = -(-k // 24)
        lo, hi = synth.uniform_indices(synth.rng(950 + i, 0), rows * nb, oc.n_points, bits)
        codes = synth.gain_codes(synth.rng(950 + i, 1), rows * nb)
        w = synth.pack_words(lo, hi, codes, bits)
        w = w.reshape((rows, nb) + w.shape[1:])
        gains = synth.chi24_tables(synth.rng(950 + i, 2), rows)
        x = synth.activations(synth.rng(950 + i, 3), 1, k)
        t0 = time.perf_counter()
        oc.gemm(w, nb, 1, gains, x, 1, threads=cores)
        secs += time.perf_counter() - t0
        nbytes += rows * nb * (8 if bits == 48 else 16) + rows * 512 + nb * 48 + rows * 4
        blocks += rows * nb
    return {"sweep": "llama-2-7b stack, oracle (one decoder layer x 32)", "index_bits": bits, "batch": 1,
            "ms": 32 * secs * 1e3, "GBps": nbytes / secs / 1e9, "decoded_vectors_per_s": blocks / secs,
            "cores": cores, "cpu_model": cpu_model()}


def build_line(steps, warmup, R, B, world, secs, secs_e2e, clk, sms, gpu_name):
    """The bench's JSON record from the timings of one run: secs and secs_e2e are the device
    times (max over ranks) of `steps` graph replays of R layer launches each, without and with
    the host copies; clk is the clock summary sampled during the timed region."""
    launches = steps * R
    bytes_launch = algorithmic_bytes(batch=B)
    per_launch_s = secs / launches
    gbs = bytes_launch / per_launch_s / 1e9                            # one GPU's kernel, for the roofline
    value = whole_job_gbps(bytes_launch, launches, secs, world)
    peak, peak_kind = measured_peaks()
    h2d = R * B * NB * 24 * 2
    d2h = R * B * ROWS * 4
    e2e_gbs = whole_job_gbps(bytes_launch, launches, secs_e2e, world)
    layer_bytes = ROWS * NB * 8
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": steps,
        "warmup": warmup, "ms_per_step": secs / steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": workload(batch=B),
                   "rows": ROWS, "cols": K, "blocks_per_row": NB,
                   "batch": B, "index_bits": 48, "layer_copies_per_step": R,
                   "l2_policy": f"inputs larger than L2: {R} distinct layer copies "
                                f"({R * layer_bytes / 2**20:.0f} MiB of words) per step",
                   "parallelism": f"replicas x{world}"},
        "us_per_layer": per_launch_s * 1e6,
        "fp16_equivalent_GBps": 2 * ROWS * K / per_launch_s / 1e9 * world,
        "decoded_vectors_per_s": ROWS * NB / per_launch_s * world,
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s",
                     "frac": gbs / peak, "traffic": measured_traffic() if B == 1 else None,
                     "peak_source": f"{peak_kind} hbm_gbs (MEASURED_PEAKS.json)"},
        "e2e": {"value": e2e_gbs, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": launches,
        "clocks": clk,
        "gpu_name": gpu_name,
    }
    if B == 1:
        line["issue_roofline"] = issue_roofline(per_launch_s, clk.get("sm_mhz") if clk else None, sms)
    return line


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    t0 = time.perf_counter()
    per_step = max(2.0, min(20.0, 150.0 / max(args.steps + args.warmup, 1)))
    for _ in range(args.warmup):
        cpu_baseline(per_step / 4, one_core_seconds=0)
    vals = [cpu_baseline(per_step, one_core_seconds=0) for _ in range(args.steps)]
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
    ap.add_argument("--mode", default="gemv", choices=["gemv", "decode", "encode", "sweep", "search", "gptq"],
                    help="decode: time llvq_decode alone (profiling aid); sweep: every layer shape, "
                         "budget and batch against cuBLAS fp16, plus the full 7B stack; search: "
                         "the nearest-point search on the Gaussian source (throughput and quality); gptq: "
                         "one Spherical GPTQ pass over a 4096 x 4104 layer")
    ap.add_argument("--search-quality", type=int, default=1, help="search mode: run the quality experiment")
    ap.add_argument("--batch", type=int, default=1, help="gemv mode: batch (1 = the metric's workload)")
    ap.add_argument("--rows", type=int, default=4096, help="gemv mode: layer rows (4096 = the metric's workload)")
    ap.add_argument("--cols", type=int, default=4096, help="gemv mode: layer columns (4096 = the metric's workload)")
    args = ap.parse_args()
    global ROWS, K, NB, WORKLOAD
    ROWS, K = args.rows, args.cols
    NB = -(-K // 24)
    WORKLOAD = workload()

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
    if args.mode == "encode":
        r = encode_throughput(torch, codec, dev, args.decode_n, args.steps, args.warmup)
        if rank == 0:
            print(json.dumps({"mode": "encode", **r}), flush=True)
        return 0
    if args.mode == "sweep":
        if rank == 0:
            sweep(torch, dev)
        return 0
    if args.mode == "gptq":
        if rank == 0:
            with ClockSampler(torch.cuda.current_device()) as clocks:
                r = gptq_throughput(torch, codec, dev, args.steps, args.warmup)
            clk = clocks.summary()
            props = torch.cuda.get_device_properties(dev)
            sm = clk.get("sm_mhz") or 1965.0
            achieved = 2.0 * r["fp64_fmas_per_pass"] / (r["ms_per_pass"] / 1e3) / 1e12
            peak = props.multi_processor_count * FP64_FMA_PER_SM_CLK * 2 * sm * 1e6 / 1e12
            line = {"metric": "gptq_weights_per_s", "value": r["weights_per_s"], "unit": "weights/s",
                    "steps": args.steps, "warmup": args.warmup,
                    "config": {"workload": f"one Spherical GPTQ pass, {GPTQ_ROWS} x {GPTQ_COLS} Gaussian layer, "
                                           f"synthetic SPD Hessian, angular search over shells 2..{GPTQ_SHELL}"},
                    "dtype": "f64", "data": "synthetic", **r, "clocks": clk,
                    "roofline": {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                                 "frac": achieved / peak, "traffic": None,
                                 "peak_source": f"{props.multi_processor_count} SMs x {FP64_FMA_PER_SM_CLK} fp64 FMA/clk x 2 x {sm:.0f} MHz"}}
            if not args.no_cpu_baseline:
                line["cpu_baseline"] = gptq_cpu_baseline()
            print(json.dumps(line), flush=True)
        return 0
    if args.mode == "search":
        if rank == 0:
            with ClockSampler(torch.cuda.current_device()) as clocks:
                r = search_throughput(torch, codec, dev, args.steps, args.warmup)
            line = {"metric": "search_vectors_per_s", "value": r["vectors_per_s"],
                    "unit": "vectors/s", "steps": args.steps, "warmup": args.warmup,
                    "config": {"workload": f"nearest point of Leech shells 2..13 (Euclidean, c = 0.3) "
                                           f"for {SEARCH_N} N(0, I_24) blocks", "l2": "flushed"},
                    "dtype": "f64", "data": "synthetic", **r, "clocks": clocks.summary()}
            props = torch.cuda.get_device_properties(dev)
            line["roofline"] = search_roofline(r, line["clocks"].get("sm_mhz") or 1965.0,
                                               props.multi_processor_count)
            if args.search_quality:
                line["quality"] = search_quality(torch, codec, dev)
            if not args.no_cpu_baseline:
                line["cpu_baseline"] = search_cpu_baseline()
            print(json.dumps(line), flush=True)
        return 0

    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    layer_bytes = ROWS * NB * 8
    R = args.copies or int(np.ceil(3 * l2 / layer_bytes)) + 1
    B = args.batch
    words, gains, xs = make_layer_copies(torch, codec, R, dev, B)
    x_dev = torch.from_numpy(xs.view(np.int16)).to(dev)                 # [R, B, K_pad]
    y_dev = torch.empty((R, B, ROWS), dtype=torch.float32, device=dev)
    ws = [codec.weight(words[i], gains, ROWS, K, L.LLVQ_GAIN_U8_TABLE) for i in range(R)]

    def run_all():
        for i in range(R):
            if B == 1:
                codec.gemv(ws[i], x_dev[i], y_dev[i], stream=stream)
            else:
                codec.gemm(ws[i], x_dev[i], y_dev[i], B, stream=stream)

    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        run_all()                                                       # warm the path once
    stream.synchronize()
    assert codec.get_error(stream) == 0
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        run_all()

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
    y_host = torch.empty((R, B, ROWS), dtype=torch.float32).pin_memory()

    def e2e_step():
        x_dev.copy_(x_host, non_blocking=True)
        graph.replay()
        y_host.copy_(y_dev, non_blocking=True)

    with torch.cuda.stream(stream):
        for _ in range(max(args.warmup, 1)):
            e2e_step()
        secs_e2e = time_steps(args.steps, e2e_step)

    if world > 1:
        secs, secs_e2e = max_over_ranks(dist, [secs, secs_e2e], dev)

    if rank == 0:
        props = torch.cuda.get_device_properties(dev)
        line = build_line(args.steps, args.warmup, R, B, world, secs, secs_e2e, clk,
                          props.multi_processor_count, torch.cuda.get_device_name(dev))
        line["decode"] = decode_throughput(torch, codec, dev, args.decode_n, 5, 2)
        line["encode"] = encode_throughput(torch, codec, dev, args.decode_n, 5, 2)
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
