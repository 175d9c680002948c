#!/usr/bin/env python
"""Decode throughput of libdf11 on B200: decompressed BF16 GB/s, fraction of
the HBM roofline, and compression ratio, on seeded synthetic weights shaped
like a whole Llama-3-8B model (32 transformer blocks + embedding + LM head,
8,029,995,008 BF16 weights, one codebook per block, one decode launch per
block, 34 launches back to back per step).

  python bench.py [--gpus N --steps K --warmup W] [--impl reference] [--workload ...]

One step = one decode of the whole model (every launch of the hot path) with
the compressed images resident in HBM.  The groups are independent, so each
launch may start while the previous one finishes (programmatic dependent
launch; `--no-overlap` for plain stream order).  Inputs (10.8 GB compressed,
16 GB decoded) are far larger than the 126 MB L2, so no flush is needed.  Rank 0
prints one JSON line.  Multi-GPU (torchrun): every rank decodes its own
replica of the model (weak scaling, no collective on the data path); the
timed region is bracketed by barriers and the reported time is the max over
ranks.  `--impl reference` times the CPU oracle decoder (the method written
out plainly, single-threaded) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from entropy_decoding_b200 import synth  # noqa: E402

METRIC = "decompressed BF16 GB/s"
HBM_FALLBACK_GBS = 6650.0
# the decode kernels' source: decode.cu and the device headers it includes
KERNEL_SRC = [os.path.join(ROOT, "entropy_decoding_b200", "csrc", f)
              for f in ("decode.cu", "walk.cuh", "merge.cuh", "check.cuh", "df11_internal.h")]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "decode_traffic.json")


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", choices=["whole_model", "block", "e4m3"], default="whole_model")
    p.add_argument("--seed", type=int, default=0)
    p.add_argument("--e2e-steps", type=int, default=3)
    p.add_argument("--cpu-seconds", type=float, default=6.0)
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu", action="store_true")
    p.add_argument("--no-encode", action="store_true", help="skip the GPU encoder measurement")
    p.add_argument("--no-extra", action="store_true",
                   help="skip the extra measurements of the default line (sustained, two-phase, block, single "
                        "matrices with an L2 flush, E4M3, rANS)")
    p.add_argument("--chunk-bits", type=int, default=128)
    p.add_argument("--tile-threads", type=int, default=32)
    p.add_argument("--chunks-per-thread", type=int, default=0, help="decode launch option (0 = library default)")
    p.add_argument("--ctas-per-sm", type=int, default=0, help="decode launch option (0 = as many as fit)")
    p.add_argument("--warps-per-cta", type=int, default=0,
                   help="decode launch option, warp tiles (0 = library default for the walker)")
    p.add_argument("--walker", choices=["auto", "window", "byte_step"], default="auto",
                   help="decode launch option, warp tiles: how a thread walks its chunk")
    p.add_argument("--no-chunk-counts", dest="chunk_counts", action="store_false",
                   help="encode without the chunk-counts section (the pages' sections only): the decode "
                        "counts each chunk's codes with a first walk")
    p.add_argument("--count-walk", action="store_true",
                   help="decode launch option: count each chunk's codes with a first walk even though the "
                        "images store chunk counts")
    p.add_argument("--coder", choices=["huffman", "rans", "fused_gemm"], default="huffman",
                   help="exponent coder: the Huffman container (default) or the rANS variant (decode from HBM "
                        "only; no end-to-end, streaming, encoder or CPU measurements); fused_gemm: the decode "
                        "fused into the consuming GEMM alone (y += x W on the block's seven matrices at M = "
                        "--gemm-m, one launch per step, the Huffman container in operand-tile order)")
    p.add_argument("--gemm-m", type=int, default=16, help="rows of x for --coder fused_gemm (1..64)")
    p.add_argument("--rans-tile", type=int, default=0, help="rANS symbols per tile (0 = library default)")
    p.add_argument("--no-overlap", dest="overlap", action="store_false",
                   help="launch the groups in plain stream order (default: each group's decode may start "
                        "while the previous one finishes, the groups being independent; the roofline then "
                        "uses the whole step's time, else each launch's own)")
    return p.parse_args()


# ------------------------------------------------------------------ workload description

def workload_config(name: str) -> dict:
    if name == "whole_model":
        n = sum(s[0] * s[1] for _, ts in synth.whole_model_specs() for _, s, _ in ts)
        return {"workload": "whole Llama-3-8B-shaped model: 32 blocks (q,k,v,o,gate,up,down) + embedding + "
                            "LM head, per-block codebooks, 34 decode launches per step",
                "n_weights": n, "launches_per_step": 34, "dtype_in": "bf16"}
    if name == "block":
        n = sum(s[0] * s[1] for _, s in synth.BLOCK_SHAPES)
        return {"workload": "one Llama-3-8B-shaped transformer block, shared codebook, 1 launch",
                "n_weights": n, "launches_per_step": 1, "dtype_in": "bf16"}
    return {"workload": "8192x28672 FP8 E4M3, N(0,0.02) scaled to E4M3 range, 1 launch",
            "n_weights": 8192 * 28672, "launches_per_step": 1, "dtype_in": "e4m3"}


def full_config(args, world: int) -> dict:
    """The `config` object of the JSON line (identical for both arms)."""
    cfg = workload_config(args.workload)
    out_gb = cfg["n_weights"] * (2 if cfg["dtype_in"] == "bf16" else 1) / 1e9
    return {**cfg, "seed": args.seed, "chunk_bits": args.chunk_bits, "tile_threads": args.tile_threads,
            "chunks_per_thread": args.chunks_per_thread or 1, "ctas_per_sm": args.ctas_per_sm or "max",
            "warps_per_cta": (args.warps_per_cta or "library default") if args.tile_threads == 32 else None,
            "walker": args.walker if args.tile_threads == 32 else "window",
            "chunk_counts": bool(args.chunk_counts) and args.chunk_bits <= 128,
            "count_walk": bool(args.count_walk),  # the device-resident decode's launch option
            "overlap_launches": bool(args.overlap),
            "l2": f"no flush: inputs larger than L2 (decoded output {out_gb:.1f} GB, compressed images "
                  f"about 0.68x that, vs 126 MB L2)",
            "parallelism": f"replicas x{world} (each GPU decodes its own copy)"}


def group_count(name: str) -> int:
    return len(synth.whole_model_specs()) if name == "whole_model" else 1


def make_group(name: str, seed: int, gi: int) -> synth.Group:
    if name == "whole_model":
        return synth.whole_model_group(seed, gi)
    if name == "block":
        return synth.transformer_block(seed)[0]
    return synth.e4m3_matrix(seed)[0]


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""
    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="df11_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) == len(self.FIELDS):
                    rows.append(parts)
        os.unlink(self.path)
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max((float(r[2]) for r in rows if r[2].replace(".", "").isdigit()), default=None)}


# ------------------------------------------------------------------ helpers

def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, copy bandwidth)"
    except (OSError, KeyError, ValueError):
        return HBM_FALLBACK_GBS, "fallback (profiling recipe: 6.65 TB/s)"


def kernel_hash() -> str:
    h = hashlib.sha256()
    for path in KERNEL_SRC:
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_per_weight():
    """DRAM bytes per weight from a committed ncu capture of the current
    kernel source, or None when the kernel changed since."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None, None
    if t.get("kernel_sha256_16") != kernel_hash():
        return None, "stale"
    return float(t["dram_bytes_per_weight"]), t.get("source")


def rank_env() -> tuple[int, int, int]:
    """(rank, world size, local rank) from the torchrun environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(x: float, device) -> float:
    """Max of a per-rank number over all ranks (identity for one rank)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(bytes_per_rank: float, world: int, steps: int, max_ms: float) -> float:
    """Whole-job GB/s: bytes decoded by all ranks over the slowest rank's time."""
    return world * bytes_per_rank * steps / (max_ms / 1e3) / 1e9


def host_threads(world: int) -> int:
    try:
        c = len(os.sched_getaffinity(0))
    except AttributeError:
        c = os.cpu_count() or 1
    return max(1, c // max(world, 1))


# ------------------------------------------------------------------ CPU oracle

def oracle_prepare(groups_host, chunk_bits: int, tile_threads: int, budget: int):
    """Compresses whole tensors of the workload with the oracle itself (its
    own code lengths, one code per group), in order, until `budget` weights:
    the oracle decodes streams it wrote, so no library code is involved."""
    import oracle
    oracle.build()
    out = []
    for gname, dt, lengths, tensors in groups_host:
        for tname, bits in tensors:
            out.append((f"{gname}.{tname}", oracle.compress(bits, dt, lengths=lengths, chunk_bits=chunk_bits,
                                                            tile_threads=tile_threads), bits))
            if sum(c.n for _, c, _ in out) >= budget:
                return out
    return out


def oracle_decode_sample(prepared, seconds: float):
    """Times the CPU oracle decoder (single-threaded) on whole tensors, in
    order, until `seconds` of decode time have accumulated; each result is
    checked against the source weights outside the timed part."""
    import oracle
    done_w, spent, names = 0, 0.0, []
    for name, c, bits in prepared:
        t0 = time.perf_counter()
        got = oracle.decompress(c)
        spent += time.perf_counter() - t0
        assert np.array_equal(got, bits), name
        done_w += c.n
        names.append(name)
        if spent >= seconds:
            break
    return done_w, spent, names


def _oracle_decode_task(c):
    """Worker of oracle_decode_parallel: one whole tensor through the oracle."""
    import oracle
    t0 = time.perf_counter()
    oracle.decompress(c)
    return c.n, time.perf_counter() - t0


def oracle_decode_parallel(prepared, cores: int):
    """The same oracle decode on every host core at once: whole tensors, one
    per task, in a pool of `cores` processes started with spawn.  Returns
    (weights, wall seconds around the whole map, tensors)."""
    import multiprocessing as mp
    tasks = sorted((c for _, c, _ in prepared), key=lambda c: -c.n)  # longest first
    with mp.get_context("spawn").Pool(cores) as pool:
        pool.map(_oracle_decode_task, tasks[-1:])  # workers up before the clock starts
        t0 = time.perf_counter()
        done = pool.map(_oracle_decode_task, tasks, chunksize=1)
        wall = time.perf_counter() - t0
    return sum(d[0] for d in done), wall, len(tasks)


# ------------------------------------------------------------------ reference arm

def run_reference(args, rank: int, world: int):
    """The oracle end to end: it builds its own code for the group, compresses
    the group's first tensor and, per step, decodes it on one host core.  The
    library is not loaded."""
    if rank != 0:
        return
    cfg = full_config(args, world)
    gi = 1 if args.workload == "whole_model" else 0
    g = make_group(args.workload, args.seed, gi)
    import oracle
    oracle.build()
    t = g.tensors[0]
    dt = "bf16" if t.bits.dtype == np.uint16 else "e4m3"
    lengths = oracle.build_lengths([x.bits for x in g.tensors], dt)
    c = oracle.compress(t.bits, dt, lengths=lengths, chunk_bits=args.chunk_bits, tile_threads=args.tile_threads)
    n = t.bits.size
    for _ in range(args.warmup):
        oracle.decompress(c)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        out = oracle.decompress(c)
    el = time.perf_counter() - t0
    assert np.array_equal(out, t.bits)
    out_bytes = n * (2 if dt == "bf16" else 1)
    value = out_bytes * args.steps / el / 1e9
    sample = (f"{g.name}.{t.name} ({n} weights) per step: compressed by the oracle with its own code for the "
              f"group, decoded by the single-threaded CPU oracle (bit-by-bit code walk + field merge)")
    line = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "u32", "data": "synthetic",
            "config": cfg, "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ single-launch measurements

L2_FLUSH_BYTES = 256 << 20  # written between timed launches: more than 2 x the 126 MB L2


def timed_launches(torch, stream, launch, flush, smi_index: int, min_s: float = 0.3, min_reps: int = 20,
                   max_reps: int = 5000):
    """CUDA-event times of single launches on `stream`, each preceded by an
    L2 flush outside its events; at least min_reps launches and about min_s
    seconds, with the SM clocks sampled meanwhile.  Returns (median ms, min
    ms, reps, clocks)."""
    for _ in range(3):
        flush()
        launch()
    stream.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(3)]
    for a, b in ev:
        flush()
        a.record(stream)
        launch()
        b.record(stream)
    stream.synchronize()
    est = statistics.median(a.elapsed_time(b) for a, b in ev)
    reps = int(min(max_reps, max(min_reps, min_s * 1e3 / (est + 0.06))))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    clocks = ClockSampler(smi_index)
    clocks.start()
    time.sleep(0.3)
    for a, b in ev:
        flush()
        a.record(stream)
        launch()
        b.record(stream)
    stream.synchronize()
    clk = clocks.stop()
    ms = [a.elapsed_time(b) for a, b in ev]
    return statistics.median(ms), min(ms), reps, clk


def huffman_single(df11, torch, stream, dev, xs, dt, flush, smi_index, peak, label, threads, count_walk=0):
    """One group (one codebook, one launch) encoded on the host, decoded from
    HBM: median launch time with an L2 flush between launches, the roofline
    fraction of the algorithmic bytes, and a full comparison with the source."""
    cb = df11.df11_build_codebook(dt, xs)
    blobs = [df11.df11_encode(cb, x, 128, 32, threads) for x in xs]
    with torch.cuda.stream(stream):
        for b in blobs:
            df11.upload(b, stream)
        outs = [torch.empty(max(16, x.size * x.itemsize + 64), dtype=torch.uint8, device=dev) for x in xs]
        err = torch.zeros(1, dtype=torch.int32, device=dev)
    stream.synchronize()
    shape = df11.df11_decode_launch_shape(blobs, with_walk=True, count_walk=count_walk)
    algo = 0
    for b in blobs:
        i = b.info()
        algo += i.stream_bytes + i.plane_bytes + i.gaps_bytes + i.out_off_bytes + i.uncompressed_bytes
        algo += i.counts_bytes if shape[4] else 0
    out_bytes = sum(x.size * x.itemsize for x in xs)

    def launch():
        df11.df11_decode_ex(blobs, [o.data_ptr() for o in outs], err.data_ptr(), stream.cuda_stream,
                            count_walk=count_walk)

    med, mn, reps, clk = timed_launches(torch, stream, launch, flush, smi_index)
    assert int(err.item()) == 0, f"{label}: device error word {int(err.item())}"
    for x, o in zip(xs, outs):
        src = torch.from_numpy(x.view(np.int16) if x.dtype == np.uint16 else x).to(dev)
        got = o[: x.size * x.itemsize].view(torch.int16 if x.dtype == np.uint16 else torch.uint8)
        assert torch.equal(got, src), f"{label}: output differs from the source"
    ser = sum(b.info().serialized_bytes for b in blobs)
    nw = sum(x.size for x in xs)
    nwarp = shape[1] // 32
    kern = (f"decode_fsm_kernel<{dt},128,{nwarp},{'true' if shape[4] else 'false'}>" if shape[3] == 2
            else f"decode_warp_kernel<{dt},128,{nwarp}>")
    return {"value": out_bytes / (med / 1e3) / 1e9, "unit": "GB/s", "ms": med, "ms_min": mn, "reps": reps,
            "weights_per_s": nw / (med / 1e3), "weights": nw, "compression_ratio": ser / out_bytes,
            "roofline": {"bound": "hbm", "achieved": algo / (med / 1e3) / 1e9, "peak": peak, "unit": "GB/s",
                         "frac": algo / (med / 1e3) / 1e9 / peak, "algorithmic_bytes": algo, "kernel": kern,
                         "stored_counts": bool(shape[4])},
            "l2": f"flushed: {L2_FLUSH_BYTES >> 20} MB written between launches", "clocks": clk,
            "workload": label, "checked": "every output equal to the source"}


def rans_single(df11, torch, stream, dev, xs, dt, flush, smi_index, peak, label, threads):
    """The rANS variant on one group: one launch, timed and checked as huffman_single."""
    rg = df11.df11_rans_encode_group(dt, xs, 0, threads)
    with torch.cuda.stream(stream):
        df11.rans_upload(rg, stream)
        outs = [torch.empty(max(16, x.size * x.itemsize + 64), dtype=torch.uint8, device=dev) for x in xs]
        err = torch.zeros(1, dtype=torch.int32, device=dev)
    stream.synchronize()
    coded = sum(rg.info(i).coded_bytes + rg.info(i).plane_bytes for i in range(len(xs)))
    out_bytes = sum(x.size * x.itemsize for x in xs)
    algo = coded + out_bytes

    def launch():
        df11.df11_rans_decode(rg, [o.data_ptr() for o in outs], err.data_ptr(), stream.cuda_stream)

    med, mn, reps, clk = timed_launches(torch, stream, launch, flush, smi_index)
    assert int(err.item()) == 0, f"{label}: device error word {int(err.item())}"
    for x, o in zip(xs, outs):
        src = torch.from_numpy(x.view(np.int16) if x.dtype == np.uint16 else x).to(dev)
        got = o[: x.size * x.itemsize].view(torch.int16 if x.dtype == np.uint16 else torch.uint8)
        assert torch.equal(got, src), f"{label}: output differs from the source"
    nw = sum(x.size for x in xs)
    freq_bytes = 2 * (256 if dt == "bf16" else 16)
    return {"value": out_bytes / (med / 1e3) / 1e9, "unit": "GB/s", "ms": med, "ms_min": mn, "reps": reps,
            "weights_per_s": nw / (med / 1e3), "weights": nw,
            "bits_per_weight": 8 * (coded + freq_bytes) / nw,
            "roofline": {"bound": "hbm", "achieved": algo / (med / 1e3) / 1e9, "peak": peak, "unit": "GB/s",
                         "frac": algo / (med / 1e3) / 1e9 / peak, "algorithmic_bytes": algo,
                         "kernel": f"rans_decode_kernel<{dt},32>"},
            "l2": f"flushed: {L2_FLUSH_BYTES >> 20} MB written between launches", "clocks": clk,
            "workload": label, "checked": "every output equal to the source"}


def fused_gemm_block(df11, torch, stream, dev, tensors, flush, smi_index, peak, threads, m=16):
    """The decode fused into the consuming GEMM (y += x W) on the block's
    seven matrices, one launch at batch M = m, against the unfused path on
    the same weights: the decode launch of the row-major block followed by
    one cuBLAS BF16 GEMM per matrix (torch.matmul).  Both timed with CUDA
    events, an L2 flush before every timed launch sequence."""
    shapes = [tuple(t.shape) for t in tensors]
    ws = [t.bits for t in tensors]
    g = np.random.default_rng(2024)
    xs = [synth.to_bf16_bits(g.standard_normal(m * k).astype(np.float32)) for k, _ in shapes]
    tiled = [df11.df11_gemm_tile_weights(w, k, n) for w, (k, n) in zip(ws, shapes)]
    cbt = df11.df11_build_codebook("bf16", tiled)
    blobs_t = [df11.df11_encode(cbt, t, 128, 32, threads) for t in tiled]
    del tiled
    cb = df11.df11_build_codebook("bf16", ws)
    blobs = [df11.df11_encode(cb, w, 128, 32, threads) for w in ws]
    with torch.cuda.stream(stream):
        for b in blobs_t + blobs:
            df11.upload(b, stream)
        xd = [torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16).reshape(m, k)
              for x, (k, _) in zip(xs, shapes)]
        ys = [torch.zeros(m * n, dtype=torch.float32, device=dev) for _, n in shapes]
        wout = [torch.empty(2 * k * n, dtype=torch.uint8, device=dev) for k, n in shapes]
        err = torch.zeros(1, dtype=torch.int32, device=dev)
    stream.synchronize()
    mats = [(b, k, n, x.data_ptr(), y.data_ptr()) for b, (k, n), x, y in zip(blobs_t, shapes, xd, ys)]
    wviews = [o.view(torch.bfloat16).reshape(k, n) for o, (k, n) in zip(wout, shapes)]

    def fused():
        for y in ys:
            y.zero_()
        df11.df11_decode_gemm(mats, m, err.data_ptr(), stream.cuda_stream)

    def unfused():
        df11.df11_decode(blobs, [o.data_ptr() for o in wout], err.data_ptr(), stream.cuda_stream)
        for x, wv in zip(xd, wviews):
            torch.matmul(x, wv)

    def gemm_only():
        for x, wv in zip(xd, wviews):
            torch.matmul(x, wv)

    with torch.cuda.stream(stream):
        f_ms, f_min, f_reps, f_clk = timed_launches(torch, stream, fused, flush, smi_index)
        u_ms, u_min, u_reps, u_clk = timed_launches(torch, stream, unfused, flush, smi_index)
        g_ms, _, _, _ = timed_launches(torch, stream, gemm_only, flush, smi_index)
        # correctness outside the timed region: one clean launch against float32 matmuls
        fused()
        stream.synchronize()
        assert int(err.item()) == 0, f"fused gemm: device error word {int(err.item())}"
        for y, x, wv, (k, n) in zip(ys, xd, wviews, shapes):
            ref = x.float() @ wv.float()
            scale = x.float().abs() @ wv.float().abs()
            assert bool((( y.reshape(m, n) - ref).abs() <= 2 * (k + 16) * 2.0 ** -24 * scale).all()), "fused gemm"
    nw = sum(k * n for k, n in shapes)
    comp = 0
    for b in blobs_t:
        i = b.info()
        comp += i.stream_bytes + i.plane_bytes + i.gaps_bytes + i.out_off_bytes + i.counts_bytes
    act = sum(2 * m * k + 8 * m * n for k, n in shapes)  # x read; y read and written (fp32)
    algo = comp + act
    dec_algo = 0
    for b in blobs:
        i = b.info()
        dec_algo += i.stream_bytes + i.plane_bytes + i.gaps_bytes + i.out_off_bytes + i.counts_bytes + 2 * i.n_elems
    unfused_bytes = dec_algo + 2 * nw + sum(2 * m * k + 2 * m * n for k, n in shapes)
    shape = df11.df11_decode_gemm_launch_shape([(b, k, n, 0, 0) for b, (k, n) in zip(blobs_t, shapes)], m)
    return {"value": nw / (f_ms / 1e3), "unit": "weights/s", "ms": f_ms, "ms_min": f_min, "reps": f_reps,
            "batch_m": m, "weights": nw,
            "unfused_ms": u_ms, "unfused_gemm_ms": g_ms, "speedup_vs_unfused": u_ms / f_ms,
            "bytes_per_weight": algo / nw, "unfused_bytes_per_weight": unfused_bytes / nw,
            "roofline": {"bound": "hbm", "achieved": algo / (f_ms / 1e3) / 1e9, "peak": peak, "unit": "GB/s",
                         "frac": algo / (f_ms / 1e3) / 1e9 / peak, "algorithmic_bytes": algo,
                         "kernel": "decode_gemm_kernel", "launch": {"grid": shape[0], "block": shape[1],
                                                                    "smem_bytes": shape[2]}},
            "clocks": f_clk, "unfused_clocks": u_clk,
            "l2": f"flushed: {L2_FLUSH_BYTES >> 20} MB written before every timed launch sequence",
            "workload": f"one Llama-3-8B-shaped transformer block, 7 matrices [in, out], y += x W at M = {m}, "
                        f"one fused launch; unfused = one decode launch + 7 cuBLAS BF16 GEMMs (torch.matmul)",
            "checked": "every output within (K + 16) 2^-24 sum|x w| of float32 matmuls of the decoded weights"}


# ------------------------------------------------------------------ our arm

def kernel_name(args, cfg: dict, shape) -> str:
    """Name of the decode kernel the library launched for these options."""
    dt = cfg["dtype_in"]
    if args.tile_threads != 32:
        cpt = args.chunks_per_thread or 1
        return f"decode_kernel<{dt},{args.chunk_bits},{cpt},{args.tile_threads // cpt}>"
    nw = shape[1] // 32
    if shape[3] == 2:  # DF11_WALKER_BYTE_STEP; shape[4]: reads the stored chunk counts
        return f"decode_fsm_kernel<{dt},{args.chunk_bits},{nw},{'true' if shape[4] else 'false'}>"
    return f"decode_warp_kernel<{dt},{args.chunk_bits},{nw}>"


def run_ours(args, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist
    from entropy_decoding_b200 import df11

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    cfg = workload_config(args.workload)
    threads = host_threads(world)

    # ---- build: generate, encode, upload, one group at a time (host memory stays bounded)
    t_setup = time.time()
    groups = []  # (name, blobs, dsts, algo bytes, n weights, out bytes)
    host_for_cpu = []
    samples = []  # (group index, tensor index, positions, values)
    out_bytes_total = 0
    ser_total = 0
    dev_total = 0
    uncompressed_total = 0
    max_len = 0
    tensors_meta = []
    rng = np.random.default_rng(12345)
    for gi in range(group_count(args.workload)):
        g = make_group(args.workload, args.seed, gi)
        dt = "bf16" if g.tensors[0].bits.dtype == np.uint16 else "e4m3"
        cb = df11.df11_build_codebook(dt, [t.bits for t in g.tensors])
        blobs = [df11.df11_encode(cb, t.bits, args.chunk_bits, args.tile_threads, threads,
                                  chunk_counts=args.chunk_counts) for t in g.tensors]
        for ti, (t, b) in enumerate(zip(g.tensors, blobs)):
            pos = np.unique(np.concatenate([np.arange(min(4096, t.bits.size)),
                                            np.arange(max(0, t.bits.size - 4096), t.bits.size),
                                            rng.integers(0, t.bits.size, 32768)]))
            samples.append((gi, ti, pos, t.bits[pos].copy()))
            i = b.info()
            ser_total += i.serialized_bytes
            dev_total += i.device_bytes
            uncompressed_total += i.uncompressed_bytes
            max_len = max(max_len, i.max_code_len)
            tensors_meta.append(i)
        if rank == 0 and world == 1 and not args.no_cpu and gi in (1, 2, 3):
            # raw weights for the oracle baseline, which compresses them itself
            host_for_cpu.append((g.name, dt, [(t.name, t.bits) for t in g.tensors]))
        groups.append([g.name, blobs, dt])
        del g
    setup_s = time.time() - t_setup

    # device images (torch-owned memory) and one output buffer, 256-byte aligned slices
    with torch.cuda.stream(stream):
        for _, blobs, _ in groups:
            for b in blobs:
                df11.upload(b, stream)
        sizes = []
        for _, blobs, dt in groups:
            sizes.append([b.info().n_elems * (2 if dt == "bf16" else 1) for b in blobs])
        total_out = sum(((s + 255) // 256) * 256 for ss in sizes for s in ss)
        out = torch.empty(total_out, dtype=torch.uint8, device=dev)
        base = out.data_ptr()
        off = 0
        for gi, (ss, grp) in enumerate(zip(sizes, groups)):
            dsts = []
            for s in ss:
                dsts.append((base + off, off, s))
                off += ((s + 255) // 256) * 256
            grp.append(dsts)
        err = torch.zeros(1, dtype=torch.int32, device=dev)
    stream.synchronize()
    out_bytes_total = sum(sum(ss) for ss in sizes)

    walker = {"auto": 0, "window": 1, "byte_step": 2}[args.walker]
    # the launch shape of the largest group (what the library picked for these options)
    big = max(range(len(groups)), key=lambda gi: sum(b.info().n_elems for b in groups[gi][1]))
    shape = df11.df11_decode_launch_shape(groups[big][1], args.chunks_per_thread, args.ctas_per_sm,
                                          args.warps_per_cta, walker, with_walk=True,
                                          count_walk=int(args.count_walk))

    # algorithmic bytes per launch: compressed sections read (the chunk counts
    # when the kernel reads them) + output written
    algo = []
    k = 0
    for name, blobs, dt, dsts in groups:
        a = 0
        for b in blobs:
            i = tensors_meta[k]
            k += 1
            a += i.stream_bytes + i.plane_bytes + i.gaps_bytes + i.out_off_bytes + i.uncompressed_bytes
            if shape[4]:
                a += i.counts_bytes
        algo.append(a)

    def one_step(events=None):
        for gi, (name, blobs, dt, dsts) in enumerate(groups):
            if events is not None and not args.overlap:
                events[gi][0].record(stream)
            df11.df11_decode_ex(blobs, [d[0] for d in dsts], err.data_ptr(), stream.cuda_stream,
                                args.chunks_per_thread, args.ctas_per_sm, args.warps_per_cta, walker, 0,
                                int(args.overlap), count_walk=int(args.count_walk))
            if events is not None and not args.overlap:
                events[gi][1].record(stream)

    for _ in range(args.warmup):
        one_step()
    stream.synchronize()

    ev = [[[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)]
           for _ in groups] for _ in range(args.steps)]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ
                          else local_rank)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)  # let the sampler attach before the region
    start.record(stream)
    for s_ in range(args.steps):
        one_step(ev[s_])
    end.record(stream)
    end.synchronize()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    elapsed_ms = max_over_ranks(start.elapsed_time(end), dev)
    if args.overlap:  # launches overlap: each one's share of the step
        launch_ms = [[elapsed_ms / args.steps / len(groups)] * len(groups) for _ in ev]
    else:
        launch_ms = [[e[0].elapsed_time(e[1]) for e in step] for step in ev]

    # ---- correctness outside the timed region: error word + sampled positions
    def check_samples(what: str):
        e = int(err.item())
        bad = 0
        for gi, ti, pos, vals in samples:
            name, blobs, dt, dsts = groups[gi]
            ptr, o, s_ = dsts[ti]
            if dt == "bf16":
                v = out[o:o + s_].view(torch.int16)
                got = v[torch.from_numpy(pos).to(dev)].cpu().numpy().view(np.uint16)
            else:
                got = out[o:o + s_][torch.from_numpy(pos).to(dev)].cpu().numpy()
            bad += int((got != vals).sum())
        assert e == 0, f"{what}: device error word {e}"
        assert bad == 0, f"{what}: {bad} sampled outputs differ from the source weights"

    check_samples("decode")
    smi_index = torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ else local_rank
    peak, peak_src = hbm_peak()
    extras = world == 1 and not args.no_extra

    # ---- the same step held for seconds (clocks settle under the power cap),
    # and the pages' two phases: each chunk's codes counted by a first walk
    def whole_run(nsteps: int, count_walk: int):
        def step():
            for name, blobs, dt, dsts in groups:
                df11.df11_decode_ex(blobs, [d[0] for d in dsts], err.data_ptr(), stream.cuda_stream,
                                    args.chunks_per_thread, args.ctas_per_sm, args.warps_per_cta, walker, 0,
                                    int(args.overlap), count_walk=count_walk)
        for _ in range(3):
            step()
        stream.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        cs = ClockSampler(smi_index)
        cs.start()
        time.sleep(0.3)
        a.record(stream)
        for _ in range(nsteps):
            step()
        b.record(stream)
        b.synchronize()
        c = cs.stop()
        ms = a.elapsed_time(b) / nsteps
        counts_read = df11.df11_decode_launch_shape(groups[big][1], args.chunks_per_thread, args.ctas_per_sm,
                                                    args.warps_per_cta, walker, with_walk=True,
                                                    count_walk=count_walk)[4]
        algo_b = 0
        for i in tensors_meta:
            algo_b += i.stream_bytes + i.plane_bytes + i.gaps_bytes + i.out_off_bytes + i.uncompressed_bytes
            algo_b += i.counts_bytes if counts_read else 0
        return {"value": out_bytes_total / (ms / 1e3) / 1e9, "unit": "GB/s", "ms_per_step": ms, "steps": nsteps,
                "seconds": ms * nsteps / 1e3,
                "roofline": {"bound": "hbm", "achieved": algo_b / (ms / 1e3) / 1e9, "peak": peak, "unit": "GB/s",
                             "frac": algo_b / (ms / 1e3) / 1e9 / peak, "algorithmic_bytes_per_step": algo_b,
                             "stored_counts": bool(counts_read)},
                "clocks": c}

    sub = {}
    if extras:
        n_sus = max(args.steps, int(math.ceil(2.0 / (elapsed_ms / args.steps / 1e3))))
        sub["sustained"] = {**whole_run(n_sus, int(args.count_walk)),
                            "what": "the headline step repeated for about 2 s (steady state under the power cap)"}
        check_samples("sustained")
        if not args.count_walk and shape[3] == 2:
            tp = whole_run(args.steps, 1)
            tp_s = whole_run(n_sus, 1)
            check_samples("two_phase")
            sub["two_phase"] = {**tp, "sustained": tp_s,
                                "what": "whole model, each chunk's codes counted by a first walk (phase 1), "
                                        "warp scan, then the decoding walk (phase 2): the two-phase kernel of "
                                        "the DFloat11 Abstract, item (ii); the images keep their stored counts "
                                        "but the launches do not read them"}
        # the block workload: one launch of the first transformer block alone
        gb = 1 if len(groups) > 2 else big
        _, blobs_b, dt_b, dsts_b = groups[gb]
        flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

        def flush():
            with torch.cuda.stream(stream):
                flush_buf.fill_(1)

        for cw in (0, 1):
            def launch_b(cw=cw):
                df11.df11_decode_ex(blobs_b, [d[0] for d in dsts_b], err.data_ptr(), stream.cuda_stream,
                                    count_walk=cw)
            med, mn, reps, clk_b = timed_launches(torch, stream, launch_b, flush, smi_index)
            cr = df11.df11_decode_launch_shape(blobs_b, with_walk=True, count_walk=cw)[4]
            ab = 0
            for b in blobs_b:
                i = b.info()
                ab += i.stream_bytes + i.plane_bytes + i.gaps_bytes + i.out_off_bytes + i.uncompressed_bytes
                ab += i.counts_bytes if cr else 0
            ob = sum(d[2] for d in dsts_b)
            sub["block" if cw == 0 else "block_two_phase"] = {
                "value": ob / (med / 1e3) / 1e9, "unit": "GB/s", "ms": med, "ms_min": mn, "reps": reps,
                "weights_per_s": sum(b.info().n_elems for b in blobs_b) / (med / 1e3),
                "roofline": {"bound": "hbm", "achieved": ab / (med / 1e3) / 1e9, "peak": peak, "unit": "GB/s",
                             "frac": ab / (med / 1e3) / 1e9 / peak, "algorithmic_bytes": ab,
                             "stored_counts": bool(cr)},
                "l2": f"flushed: {L2_FLUSH_BYTES >> 20} MB written between launches", "clocks": clk_b,
                "workload": f"one Llama-3-8B-shaped transformer block ({groups[gb][0]}), shared code, 1 launch"}
        check_samples("block")

    # ---- end to end through the C-ABI with host buffers (pinned)
    e2e = None
    streamed = None
    if not args.no_e2e:
        himgs = []
        for name, blobs, dt, dsts in groups:
            hs = []
            for b in blobs:
                nb = b.info().device_bytes
                h = torch.empty(nb, dtype=torch.uint8, pin_memory=True)
                df11.df11_blob_device_image(b, h.data_ptr(), nb)
                hs.append(h)
            himgs.append(hs)
        max_group_out = max(sum(((s + 255) // 256) * 256 for s in ss) for ss in sizes)
        hout = torch.empty(max_group_out, dtype=torch.uint8, pin_memory=True)
        h2d = sum(h.numel() for hs in himgs for h in hs)
        d2h = out_bytes_total

        def e2e_step():
            for gi, (name, blobs, dt, dsts) in enumerate(groups):
                hp = []
                o = 0
                for (_, _, s) in dsts:
                    hp.append(hout.data_ptr() + o)
                    o += ((s + 255) // 256) * 256
                dimg = [b._keep.data_ptr() + (-b._keep.data_ptr()) % 256 for b in blobs]
                df11.df11_decode_host(blobs, [h.data_ptr() for h in himgs[gi]], dimg, [d[0] for d in dsts], hp,
                                      err.data_ptr(), stream.cuda_stream)

        e2e_step()
        stream.synchronize()
        if world > 1:
            dist.barrier()
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        s1.record(stream)
        s1.synchronize()
        e2e_ms = max_over_ranks(s0.elapsed_time(s1) / args.e2e_steps, dev)
        assert int(err.item()) == 0
        e2e = {"value": job_throughput(out_bytes_total, world, 1, e2e_ms), "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
               "path": "df11_decode_host: pinned host image -> H2D -> decode launch -> D2H of every output"}
        check_samples("e2e")

        # ---- decode of weights kept in host memory (offloaded): images stay in
        # pinned host memory and stream through device staging slots, each
        # group's copy overlapping earlier groups' decodes; outputs stay on the
        # device (where the layers would consume them)
        slot_cap = max(sum(((b.info().device_bytes + 255) // 256) * 256 for b in blobs) for _, blobs, _, _ in groups)
        slot_bufs = [torch.empty(slot_cap + 256, dtype=torch.uint8, device=dev) for _ in range(2)]
        slot_ptrs = [x.data_ptr() + (-x.data_ptr()) % 256 for x in slot_bufs]
        cstream = torch.cuda.Stream(device=dev)
        flat_imgs = [h.data_ptr() for hs in himgs for h in hs]
        flat_dst = [d[0] for _, _, _, dsts in groups for d in dsts]
        glist = [blobs for _, blobs, _, _ in groups]
        st_ms = {}
        for nslots in (2, 1):
            def streamed_step():
                df11.df11_decode_streamed(glist, flat_imgs, slot_ptrs[:nslots], slot_cap, flat_dst, err.data_ptr(),
                                          cstream.cuda_stream, stream.cuda_stream)
            streamed_step()
            stream.synchronize()
            cstream.synchronize()
            if world > 1:
                dist.barrier()
            a0 = torch.cuda.Event(enable_timing=True)
            a1 = torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            cstream.wait_event(a0)
            for _ in range(args.e2e_steps):
                streamed_step()
            a1.record(stream)
            a1.synchronize()
            cstream.synchronize()
            st_ms[nslots] = max_over_ranks(a0.elapsed_time(a1) / args.e2e_steps, dev)
        check_samples("streamed")
        streamed = {"value": job_throughput(out_bytes_total, world, 1, st_ms[2]), "unit": "GB/s",
                    "ms_per_step": st_ms[2], "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": 0, "slots": 2,
                    "one_slot": {"value": job_throughput(out_bytes_total, world, 1, st_ms[1]), "ms_per_step": st_ms[1]},
                    "path": "df11_decode_streamed: pinned host images -> device staging slots on a copy stream, "
                            "decodes on the bench stream, outputs on the device; one_slot = copy and decode "
                            "in turn"}
        del himgs, hout, slot_bufs

    # ---- CPU oracle baseline (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu and host_for_cpu:
        import oracle
        oracle.build()
        ghost = [(gname, dt, oracle.build_lengths([b for _, b in ts], dt), ts) for gname, dt, ts in host_for_cpu]
        prepared = oracle_prepare(ghost, args.chunk_bits, args.tile_threads, int(args.cpu_seconds * 1.2e8))
        del ghost, host_for_cpu
        w, sec, names = oracle_decode_sample(prepared, args.cpu_seconds)
        cpu = {"value": 2 * w / sec / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
               "sample": f"{w} weights ({len(names)} whole tensors from blocks 0-2, {names[0]} ... {names[-1]}), "
                         f"compressed by the oracle with its own per-block code, then single-threaded "
                         f"bit-by-bit oracle decode + field merge, {sec:.1f} s"}
        cores = host_threads(1)
        if cores > 1:
            prepared = [p_ for p_ in prepared if p_[0] in names]
            wa, wall, nt = oracle_decode_parallel(prepared, cores)
            cpu["all_cores"] = {"value": 2 * wa / wall / 1e9, "unit": "GB/s", "cores": cores,
                                "weights_per_s": wa / wall,
                                "sample": f"{wa} weights ({nt} whole tensors of blocks 0-2), one tensor per "
                                          f"task on {cores} spawned processes, {wall:.1f} s wall"}

    # ---- the GPU encoder on the largest group (histogram, code, packing, aux),
    # its source being the decoded output (bit-identical to the weights)
    enc = None
    if rank == 0 and not args.no_encode:
        ge = 1 if len(groups) > 2 else big  # a transformer block for the whole model
        _, blobs_b, dt_b, dsts_b = groups[ge]
        srcs = [out[o:o + s_].view(torch.int16 if dt_b == "bf16" else torch.uint8) for _, o, s_ in dsts_b]
        n_b = sum(x.numel() for x in srcs)

        def encode_group():
            counts = torch.zeros(256, dtype=torch.int64, device=dev)
            with torch.cuda.stream(stream):
                for x in srcs:
                    df11.df11_histogram_device(dt_b, x.data_ptr(), x.numel(), counts.data_ptr(), stream.cuda_stream)
                nsym = 256 if dt_b == "bf16" else 16
                cb_g = df11.df11_codebook_from_counts(dt_b, counts.cpu().numpy().view(np.uint64)[:nsym])
                return [df11.encode_on_device(cb_g, x, args.chunk_bits, args.tile_threads, stream,
                                              chunk_counts=args.chunk_counts) for x in srcs]

        encode_group()
        stream.synchronize()
        t0 = time.perf_counter()
        reps = 5
        for _ in range(reps):
            res = encode_group()
        stream.synchronize()
        enc_s = (time.perf_counter() - t0) / reps
        same = all(r.info().device_bytes == b.info().device_bytes for r, b in zip(res, blobs_b))
        enc = {"value": n_b * (2 if dt_b == "bf16" else 1) / enc_s / 1e9, "unit": "GB/s of source",
               "ms": enc_s * 1e3, "weights": n_b, "same_size_as_host_encoding": same,
               "sample": f"group {groups[ge][0]}: device histogram, host code from the 256 counts, device "
                         f"bit packing and gap/out_off, one image per tensor; wall clock over {reps} repetitions"}
        del res

    # ---- the other workloads, one launch each, with an L2 flush between
    # launches (the whole model's memory is released first)
    if extras:
        for _, blobs, _, _ in groups:
            for b in blobs:
                b._keep = None
        del out
        torch.cuda.empty_cache()
        wl = [("c1_l2_flushed", "bf16", lambda: synth.single_matrix(args.seed)[0],
               "single 1024x1024 BF16 matrix, N(0, 0.02)"),
              ("c2_l2_flushed", "bf16", lambda: synth.heavy_tail_matrix(args.seed)[0],
               "4096x4096 BF16, 0.02 t(3) with 0.1% N(0,1) outliers"),
              ("e4m3", "e4m3", lambda: synth.e4m3_matrix(args.seed)[0],
               "8192x28672 FP8 E4M3, N(0, 0.02) scaled to the E4M3 range")]
        for key, dt_w, make, label in wl:
            xs = [t.bits for t in make().tensors]
            sub[key] = huffman_single(df11, torch, stream, dev, xs, dt_w, flush, smi_index, peak, label, threads)
            del xs
        blk = synth.transformer_block(args.seed)[0]
        xs = [t.bits for t in blk.tensors]
        sub["rans"] = rans_single(df11, torch, stream, dev, xs, "bf16", flush, smi_index, peak,
                                  "the transformer block, rANS-coded exponents (16,384-symbol tiles, 32 "
                                  "interleaved coders)", threads)
        del xs
        torch.cuda.empty_cache()
        sub["fused_gemm"] = fused_gemm_block(df11, torch, stream, dev, blk.tensors, flush, smi_index, peak, threads)
        del blk

    if rank != 0:
        return
    ms_per_step = elapsed_ms / args.steps
    value = job_throughput(out_bytes_total, world, args.steps, elapsed_ms)
    per_launch = np.array(launch_ms)  # steps x groups
    tot_launch_s = per_launch.sum() / 1e3
    algo_step = float(sum(algo))
    achieved = algo_step * args.steps / tot_launch_s / 1e9
    tpw, tsrc = traffic_per_weight()
    n_w = cfg["n_weights"]
    traffic = tpw * n_w / len(groups) if tpw is not None else None
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "u32", "data": "synthetic (seeded N(0,1/sqrt(fan_in)) / N(0,0.02) weights, "
                                                     "random init, no trained checkpoint)",
        "config": full_config(args, world),
        "weights_per_s": world * n_w * args.steps / (elapsed_ms / 1e3),
        "compression_ratio": ser_total / uncompressed_total,
        "bits_per_weight": 8 * ser_total / n_w,
        "max_code_len": max_len,
        "hbm_roofline_frac": achieved / peak,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "peak_source": peak_src,
                     "peak_datasheet": 8000.0, "frac_datasheet": achieved / 8000.0,
                     "kernel": kernel_name(args, cfg, shape),
                     "launch": {"grid": shape[0], "block": shape[1], "smem_bytes": shape[2],
                                "walker": {1: "window", 2: "byte_step"}.get(shape[3], shape[3]),
                                "stored_counts": bool(shape[4])},
                     "algorithmic_bytes_per_launch": algo_step / len(groups),
                     "launch_ms_mean": float(per_launch.mean()),
                     "launch_ms_by_group": {"first": float(per_launch[:, 0].mean()),
                                            "block_mean": float(per_launch[:, 1:-1].mean()) if len(groups) > 2
                                            else None,
                                            "last": float(per_launch[:, -1].mean())},
                     "traffic_source": tsrc},
        "cpu_baseline": cpu,
        "encode_gpu": enc,
        "e2e": e2e,
        "streamed_from_host": streamed,
        **sub,
        "gpu_launches": len(groups) * args.steps,
        "clocks": clk,
        "setup_s": setup_s,
    }
    print(json.dumps(line), flush=True)


def run_rans(args, rank: int, world: int, local_rank: int):
    """The rANS variant of the exponent coder on the same workload: every
    group encoded with one frequency table on the host, then per step one
    decode launch per group from HBM, timed and checked as the Huffman arm."""
    import torch
    import torch.distributed as dist
    from entropy_decoding_b200 import df11

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    threads = host_threads(world)
    t_setup = time.time()
    groups, samples = [], []
    rng = np.random.default_rng(12345)
    coded = plane = uncompressed = 0
    n_w = 0
    for gi in range(group_count(args.workload)):
        g = make_group(args.workload, args.seed, gi)
        dt = "bf16" if g.tensors[0].bits.dtype == np.uint16 else "e4m3"
        xs = [t.bits for t in g.tensors]
        rg = df11.df11_rans_encode_group(dt, xs, args.rans_tile, threads)
        for ti, x in enumerate(xs):
            pos = np.unique(np.concatenate([np.arange(min(4096, x.size)), np.arange(max(0, x.size - 4096), x.size),
                                            rng.integers(0, x.size, 32768)]))
            samples.append((gi, ti, pos, x[pos].copy()))
            inf = rg.info(ti)
            coded += inf.coded_bytes
            plane += inf.plane_bytes
            uncompressed += inf.uncompressed_bytes
            n_w += x.size
        with torch.cuda.stream(stream):
            df11.rans_upload(rg, stream)
        groups.append([g.name, rg, dt, [x.size * x.itemsize for x in xs]])
        del g, xs
    setup_s = time.time() - t_setup
    total_out = sum(((s_ + 255) // 256) * 256 for grp in groups for s_ in grp[3])
    out = torch.empty(total_out, dtype=torch.uint8, device=dev)
    off = 0
    for grp in groups:
        dsts = []
        for s_ in grp[3]:
            dsts.append((out.data_ptr() + off, off, s_))
            off += ((s_ + 255) // 256) * 256
        grp.append(dsts)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    stream.synchronize()
    out_bytes = sum(sum(grp[3]) for grp in groups)

    def one_step():
        for name, rg, dt, sizes, dsts in groups:
            df11.df11_rans_decode(rg, [d[0] for d in dsts], err.data_ptr(), stream.cuda_stream)

    for _ in range(args.warmup):
        one_step()
    stream.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ else local_rank)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    start.record(stream)
    for _ in range(args.steps):
        one_step()
    end.record(stream)
    end.synchronize()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    elapsed_ms = max_over_ranks(start.elapsed_time(end), dev)
    e = int(err.item())
    bad = 0
    for gi, ti, pos, vals in samples:
        ptr, o, s_ = groups[gi][4][ti]
        v = out[o:o + s_]
        if groups[gi][2] == "bf16":
            got = v.view(torch.int16)[torch.from_numpy(pos).to(dev)].cpu().numpy().view(np.uint16)
        else:
            got = v[torch.from_numpy(pos).to(dev)].cpu().numpy()
        bad += int((got != vals).sum())
    assert e == 0, f"rans decode: device error word {e}"
    assert bad == 0, f"rans decode: {bad} sampled outputs differ from the source weights"
    if rank != 0:
        return
    value = job_throughput(out_bytes, world, args.steps, elapsed_ms)
    algo = coded + plane + out_bytes
    achieved = algo * args.steps / (elapsed_ms / 1e3) / 1e9
    peak, peak_src = hbm_peak()
    freq_bytes = 2 * (256 if groups[0][2] == "bf16" else 16) * len(groups)  # the stored form of each table
    shape = df11.df11_rans_decode_launch_shape(groups[0][1])
    dtn = groups[0][2]
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "u32", "data": "synthetic (seeded N(0,1/sqrt(fan_in)) / N(0,0.02) weights, "
                                                     "random init, no trained checkpoint)",
        "config": {**full_config(args, world), "coder": "rans",
                   "rans_tile_symbols": args.rans_tile or df11.RANS_TILE_DEFAULT},
        "weights_per_s": world * n_w * args.steps / (elapsed_ms / 1e3),
        "compression_ratio": (coded + plane + freq_bytes) / uncompressed,
        "bits_per_weight": 8 * (coded + plane + freq_bytes) / n_w,
        "hbm_roofline_frac": achieved / peak,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": None, "peak_source": peak_src, "peak_datasheet": 8000.0,
                     "frac_datasheet": achieved / 8000.0,
                     "kernel": f"rans_decode_kernel<{dtn},32>",
                     "launch": {"grid": shape[0], "block": shape[1], "smem_bytes": shape[2]},
                     "algorithmic_bytes_per_step": algo, "traffic_source": "not captured for this kernel"},
        "cpu_baseline": None, "e2e": None, "gpu_launches": len(groups) * args.steps, "clocks": clk,
        "setup_s": setup_s,
    }
    print(json.dumps(line), flush=True)


def run_fused_gemm(args, rank: int, world: int, local_rank: int):
    """The decode fused into the consuming GEMM alone: the block's seven
    matrices encoded in operand-tile order with one code, then per step one
    df11_decode_gemm launch (y += x W at M = --gemm-m), each after an L2
    flush and timed with CUDA events; checked once against float32 matmuls
    of the source weights (the exact decoded weights)."""
    import torch
    from entropy_decoding_b200 import df11

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    threads = host_threads(world)
    m = args.gemm_m
    t_setup = time.time()
    blk = synth.transformer_block(args.seed)[0]
    shapes = [tuple(t.shape) for t in blk.tensors]
    ws = [t.bits for t in blk.tensors]
    tiled = [df11.df11_gemm_tile_weights(w, k, n) for w, (k, n) in zip(ws, shapes)]
    cb = df11.df11_build_codebook("bf16", tiled)
    blobs = [df11.df11_encode(cb, t, 128, 32, threads) for t in tiled]
    del tiled
    g = np.random.default_rng(2024)
    xs = [synth.to_bf16_bits(g.standard_normal(m * k).astype(np.float32)) for k, _ in shapes]
    with torch.cuda.stream(stream):
        for b in blobs:
            df11.upload(b, stream)
        xd = [torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16).reshape(m, k)
              for x, (k, _) in zip(xs, shapes)]
        ys = [torch.zeros(m * n, dtype=torch.float32, device=dev) for _, n in shapes]
        err = torch.zeros(1, dtype=torch.int32, device=dev)
        flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream.synchronize()
    setup_s = time.time() - t_setup
    mats = [(b, k, n, x.data_ptr(), y.data_ptr()) for b, (k, n), x, y in zip(blobs, shapes, xd, ys)]

    def launch():
        df11.df11_decode_gemm(mats, m, err.data_ptr(), stream.cuda_stream)

    smi_index = torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ else local_rank
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            flush_buf.fill_(1)
            launch()
        stream.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        clocks = ClockSampler(smi_index)
        clocks.start()
        time.sleep(0.3)
        for a, b in ev:
            flush_buf.fill_(1)
            a.record(stream)
            launch()
            b.record(stream)
        stream.synchronize()
        clk = clocks.stop()
        ms = [a.elapsed_time(b) for a, b in ev]
        for y in ys:
            y.zero_()
        launch()
        stream.synchronize()
    e = int(err.item())
    assert e == 0, f"fused gemm: device error word {e}"
    for y, x, w, (k, n) in zip(ys, xd, ws, shapes):
        wv = torch.from_numpy(w.view(np.int16)).to(dev).view(torch.bfloat16).reshape(k, n).float()
        ref = x.float() @ wv
        scale = x.float().abs() @ wv.abs()
        assert bool(((y.reshape(m, n) - ref).abs() <= 2 * (k + 16) * 2.0 ** -24 * scale).all()), "fused gemm"
    if rank != 0:
        return
    nw = sum(k * n for k, n in shapes)
    comp = 0
    for b in blobs:
        i = b.info()
        comp += i.stream_bytes + i.plane_bytes + i.gaps_bytes + i.out_off_bytes + i.counts_bytes
    algo = comp + sum(2 * m * k + 8 * m * n for k, n in shapes)
    med = statistics.median(ms)
    peak, peak_src = hbm_peak()
    shape = df11.df11_decode_gemm_launch_shape([(b, k, n, 0, 0) for b, (k, n) in zip(blobs, shapes)], m)
    line = {
        "metric": "fused decode + GEMM weights/s", "value": world * nw / (med / 1e3), "unit": "weights/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": med,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1/sqrt(fan_in)) weights and N(0,1) activations, random init)",
        "config": {"workload": f"one Llama-3-8B-shaped transformer block, 7 matrices [in, out], y += x W at "
                               f"M = {m}, one fused launch per step", "batch_m": m, "seed": args.seed,
                   "l2": f"flushed: {L2_FLUSH_BYTES >> 20} MB written before every timed launch"},
        "bytes_per_weight": algo / nw,
        "roofline": {"bound": "hbm", "achieved": algo / (med / 1e3) / 1e9, "peak": peak, "unit": "GB/s",
                     "frac": algo / (med / 1e3) / 1e9 / peak, "peak_source": peak_src, "traffic": None,
                     "algorithmic_bytes": algo, "kernel": "decode_gemm_kernel",
                     "launch": {"grid": shape[0], "block": shape[1], "smem_bytes": shape[2]}},
        "ms_min": min(ms), "cpu_baseline": None, "e2e": None, "gpu_launches": args.steps, "clocks": clk,
        "setup_s": setup_s,
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    rank, world, local_rank = rank_env()
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.coder == "rans":
            run_rans(args, rank, world, local_rank)
        elif args.coder == "fused_gemm":
            run_fused_gemm(args, rank, world, local_rank)
        else:
            run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
