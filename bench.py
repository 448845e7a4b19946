"""Benchmark of the fused lattice-rANS tile decode on B200.

One step = the fused decode (tables staged per CTA, rANS tiles, E8 reconstruction, container
stores) of every tensor of a workload: by default the 4096x4096 BF16 matrix with per-row
log-normal std at 4 bits per weight, the configuration the headline metric is quoted on;
``--workload`` selects the DiT weight set (112 tensors), the INT8 / FP8 code matrices or the
outlier matrix, and ``--target`` the rate.  Streams, tables and outputs are resident in HBM;
workloads smaller than twice the 126 MB L2 rotate over device copies so that every step reads
its streams from HBM.  Launches are replayed from a CUDA graph so that host launch cost does not
gate the GPU.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--workload W]

N > 1 runs N independent replicas (the decode has no exchange step, so there is no collective):
one process per GPU under torchrun, timed on the device, max over ranks.  The reference arm
(--impl reference) is the CPU oracle: it encodes the workload's first tensor with the oracle's
compressor and times the oracle's decoder on every host core the process may use.  Both arms
print the same ``config`` (the workload and how the timed region defeats the L2).
"""
import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fused decode GB/s (container out) & Gweights/s at 4 bpp; % of HBM roofline"
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "decode_kernel_traffic.json")
KERNEL_SRCS = {"decode_kernel": ("decode.cu", "decode_core.cuh", "device_util.cuh", "format.h"),
               "linear_kernel": ("linear.cu", "decode_core.cuh", "device_util.cuh", "format.h"),
               "ans_decode_kernel": ("tile_ans.cu", "device_util.cuh", "tile_ans.h")}
L2_BYTES = 126 * 2 ** 20

# The workloads (synthetic, seeded; shapes and distributions as stated).  The default is the
# 4096x4096 matrix the headline metric is quoted on; the others are the remaining workloads of
# the decode, one JSON line each.
WORKLOADS = {
    "lognormal_rows_4096x4096_bf16": dict(
        layers=lambda: [("w", lambda: _synth().row_lognormal(4096, 4096, 1))], target=4.0, container=0,
        dims=[(4096, 4096)], distribution="N(0, s_r^2), s_r = 0.02 exp(0.3 g), seed 1", shape="4096x4096"),
    "dit_28blocks_hidden3072_bf16": dict(
        layers=lambda: [(f"block{b}.{n}", (lambda b=b, l=l: _synth().dit_layer(b, l)))
                        for b in range(28) for l, n in enumerate(("qkv", "out", "mlp_up", "mlp_down"))],
        target=4.0, container=0, shape="28 x {3072x9216, 3072x3072, 3072x12288, 12288x3072}",
        dims=[(3072, 9216), (3072, 3072), (3072, 12288), (12288, 3072)] * 28,
        distribution="Student-t(5) / sqrt(5/3) * 0.02 * per-row exp(0.3 g), seed 100 + 4 block + layer"),
    "int8_codes_8192x8192": dict(
        layers=lambda: [("w", lambda: _synth().gaussian(8192, 8192, 0.02, 2))], target=3.0, container="int8",
        dims=[(8192, 8192)],
        distribution="N(0, 0.02^2), seed 2, per-row absmax INT8 codes", shape="8192x8192"),
    "fp8_codes_8192x8192": dict(
        layers=lambda: [("w", lambda: _synth().gaussian(8192, 8192, 0.02, 2))], target=3.0, container="fp8_e4m3",
        dims=[(8192, 8192)],
        distribution="N(0, 0.02^2), seed 2, per-row absmax FP8 E4M3 codes", shape="8192x8192"),
    "tile_ans_lognormal_4096x4096_bf16": dict(
        layers=lambda: [("w", lambda: _synth().row_lognormal(4096, 4096, 1))], target=16.0, container=0,
        dims=[(4096, 4096)], scheme="tile_ans", shape="4096x4096",
        distribution="N(0, s_r^2), s_r = 0.02 exp(0.3 g), seed 1; lossless Tile-ANS (every bit kept)"),
    "linear_fused_dit_block_16tok_bf16": dict(
        layers=lambda: [(f"block0.{n}", (lambda l=l: _synth().dit_layer(0, l)))
                        for l, n in enumerate(("qkv", "out", "mlp_up", "mlp_down"))],
        target=4.0, container=0, scheme="linear_fused", tokens=16,
        dims=[(3072, 9216), (3072, 3072), (3072, 12288), (12288, 3072)],
        shape="block 0 linears {3072x9216, 3072x3072, 3072x12288, 12288x3072} (out x in), 16 tokens",
        distribution="DiT block 0 weights (as dit_28blocks_hidden3072_bf16), GEMM block order; "
                     "x = 0.5 N(0, 1) BF16, seed 5"),
    "linear_fused_dit_block_16tok_int8": dict(
        layers=lambda: [(f"block0.{n}", (lambda l=l: _synth().dit_layer(0, l)))
                        for l, n in enumerate(("qkv", "out", "mlp_up", "mlp_down"))],
        target=4.0, container="int8", scheme="linear_fused", tokens=16,
        dims=[(3072, 9216), (3072, 3072), (3072, 12288), (12288, 3072)],
        shape="block 0 linears {3072x9216, 3072x3072, 3072x12288, 12288x3072} (out x in), 16 tokens",
        distribution="DiT block 0 weights as per-row absmax INT8 codes, GEMM block order; x = 0.5 N(0, 1) BF16, "
                     "seed 5, quantized per token (W8A8)"),
    "linear_fused_dit_block_16tok_fp8": dict(
        layers=lambda: [(f"block0.{n}", (lambda l=l: _synth().dit_layer(0, l)))
                        for l, n in enumerate(("qkv", "out", "mlp_up", "mlp_down"))],
        target=4.0, container="fp8_e4m3", scheme="linear_fused", tokens=16,
        dims=[(3072, 9216), (3072, 3072), (3072, 12288), (12288, 3072)],
        shape="block 0 linears {3072x9216, 3072x3072, 3072x12288, 12288x3072} (out x in), 16 tokens",
        distribution="DiT block 0 weights as per-row absmax FP8 E4M3 codes, GEMM block order; x = 0.5 N(0, 1) "
                     "BF16, seed 5, quantized per token (W8A8)"),
    "outliers_8192x28672_bf16": dict(
        layers=lambda: [("w", lambda: _synth().gaussian_outliers(8192, 28672, 3))], target=4.0, container=0,
        dims=[(8192, 28672)],
        distribution="N(0, 0.02^2), seed 3, 0.1% of entries set to +-8 sigma", shape="8192x28672"),
}
DEFAULT_WORKLOAD = "lognormal_rows_4096x4096_bf16"
TILE_ANS_METRIC = "lossless Tile-ANS decode GB/s (tensor out) & Gelements/s; % of HBM roofline"


def is_tile_ans(a):
    return WORKLOADS[a.workload].get("scheme") == "tile_ans"


def is_linear(a):
    return WORKLOADS[a.workload].get("scheme") == "linear_fused"


def _synth():
    from dit_weight_compression_tile_b200 import synth
    return synth


def args_():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=40000)
    p.add_argument("--warmup", type=int, default=16)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    p.add_argument("--target", type=float, default=None, help="bits per weight (default: the workload's)")
    p.add_argument("--cpu-seconds", type=float, default=12.0)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--shape", default=None,
                   help="RxC: the workload's first R rows and C columns instead of the whole tensor "
                        "(single-tensor workloads; a smaller case of the same kernel for profiler captures)")
    a = p.parse_args()
    wl = WORKLOADS[a.workload]
    a.target = wl["target"] if a.target is None else a.target
    if a.shape:
        if len(wl["dims"]) != 1:
            raise SystemExit("--shape applies to single-tensor workloads")
        R, Cc = (int(v) for v in a.shape.lower().split("x"))
        full = wl["layers"]()[0][1]
        sub = dict(wl)
        sub["layers"] = lambda: [("w", lambda: full()[:R, :Cc].contiguous())]
        sub["dims"] = [(R, Cc)]
        sub["shape"] = f"{R}x{Cc} (top-left part of {wl['shape']})"
        WORKLOADS[a.workload] = sub
    return a


def coding_label(infos):
    """how the workload's streams code coordinates 1..6: paired, single or mixed"""
    paired = sum(1 for i in infos if i.paired)
    return "paired" if paired == len(infos) else ("single" if paired == 0 else "mixed")


def workload_config(a):
    wl = WORKLOADS[a.workload]
    cfg = {"workload": a.workload, "shape": wl["shape"],
           "target_bpp": "lossless" if wl.get("scheme") == "tile_ans" else a.target,
           "distribution": wl["distribution"], "container": wl["container"] or "bf16"}
    if wl.get("scheme") == "linear_fused":
        cfg["tokens"] = wl["tokens"]
    return cfg


def l2_policy(a):
    """(device copies to rotate over, the sentence that says how the timed region defeats the
    L2), from the workload's nominal bytes (target rate in, container out) so that both arms
    state the same policy: workloads smaller than twice the L2 rotate over copies whose streams
    and outputs together exceed twice the L2"""
    wl = WORKLOADS[a.workload]
    # bytes per weight a step moves besides the stream: the container written (none for the fused
    # GEMM, whose weight stays on chip)
    esz = 0 if wl.get("scheme") == "linear_fused" else (1 if wl["container"] in ("int8", "fp8_e4m3") else 2)
    nominal = sum(r * c for r, c in wl["dims"]) * (a.target / 8.0 + esz)
    if nominal >= 2 * L2_BYTES:
        return 1, f"inputs larger than L2: {nominal / 1e6:.0f} MB per step"
    rot = min(8, -(-2 * L2_BYTES // int(nominal)))
    what = "stream" if esz == 0 else "stream+output"
    return rot, f"inputs larger than L2: {rot} rotating {what} copies ({rot * nominal / 1e6:.0f} MB)"


def bench_config(a, world):
    """the ``config`` both arms print: the workload and the L2 policy of the timed region"""
    return dict(workload_config(a), l2=l2_policy(a)[1], parallelism="replicas" if world > 1 else "single")


def compress_layers(a):
    """the workload's streams, encoded once on the GPU (ep_compress_device: the host compressor's
    bytes), untimed for the metric; returns [(name, host copy of the blob)], the encode seconds
    and the relative L2 error of the decoded weights against the source tensors,
    sqrt(sum (W - What)^2 / sum W^2) over the whole workload (INT8 / FP8 codes dequantized with
    the stream's row scales)"""
    from dit_weight_compression_tile_b200 import binding as B
    wl = WORKLOADS[a.workload]
    out, t = [], 0.0
    err2 = ref2 = 0.0
    for name, make in wl["layers"]():
        w = make().cuda()
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        blob = B.compress_device(w, a.target, container=wl["container"])
        torch.cuda.synchronize()
        t += time.perf_counter() - t0
        host = blob.cpu()
        info = B.stream_info(host)
        dec = B.decompress(blob, info).double()
        if info.container_dtype in (B.INT8, B.FP8E4M3):
            scales = blob[info.off_scales: info.off_scales + 4 * info.rows].view(torch.float32).double()
            dec = dec * scales[:, None]
        w64 = w.double()
        err2 += float(((w64 - dec) ** 2).sum())
        ref2 += float((w64 ** 2).sum())
        out.append((name, host))
        del w, w64, blob, dec
    return out, t, (err2 / ref2) ** 0.5 if ref2 > 0 else 0.0


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ------------------------------------------------------------------ clocks during the timed region
NVML_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
                0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
                0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, device_index):
        self.samples, self.reasons, self.max_mhz = [], 0, None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = None
            try:  # CUDA and NVML number devices differently when only some are visible
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
                self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:  # no NVML: clocks are reported as unknown
            self.nv = None

    def _sample(self):
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            self.reasons |= self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            pass

    def _run(self):
        # every 5 ms while the timed region runs, plus one sample as it ends (a short region
        # still gets two)
        while not self._stop.is_set():
            self._sample()
            time.sleep(0.005)

    def __enter__(self):
        if self.nv:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.nv:
            self.t.join()
            self._sample()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"], "samples": 0}
        names = [n for bit, n in NVML_REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


# ------------------------------------------------------------------ ranks (replicas, no data exchange)
def max_over_ranks(x, world, device):
    """the slowest rank's time: every rank decodes its own replica, the job ends with the last"""
    if world <= 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_rate(per_rank_bytes, world, seconds):
    """whole-job throughput: all ranks' bytes over the slowest rank's time"""
    return world * per_rank_bytes / seconds


# ------------------------------------------------------------------ CPU oracle leg
def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_oracle_decode(blob_np, seconds, threads=1):
    """the oracle decoder, as it stands, on `threads` host cores: each thread decodes runs of 16
    consecutive tiles of one stream (threads start at different tiles; the oracle keeps no global
    state and ctypes releases the GIL) until the time is up; returns (weights decoded, seconds,
    tiles)"""
    from concurrent.futures import ThreadPoolExecutor
    from oracle import oracle as O
    rc, info = O.parse(blob_np)
    per_tile = 32 * info.blocks_per_lane * 8
    n_w = info.rows * info.cols
    t0 = time.perf_counter()

    def worker(i):
        done, tiles, lo = 0, 0, (i * info.n_tiles) // threads
        while time.perf_counter() - t0 < seconds:
            lo = lo % info.n_tiles
            hi = min(info.n_tiles, lo + 16)
            rc, st, _, _ = O.decode(blob_np, lo, hi, want_v=False)
            assert rc == 0 and st == 0
            done += min(hi * per_tile, n_w) - lo * per_tile
            tiles += hi - lo
            lo = hi
        return done, tiles

    with ThreadPoolExecutor(threads) as ex:
        res = list(ex.map(worker, range(threads)))
    t = time.perf_counter() - t0
    return sum(r[0] for r in res), t, sum(r[1] for r in res)


def kernel_source_hash(kernel):
    """sha256 (16 hex digits) of the sources that make up a kernel"""
    h = hashlib.sha256()
    for name in KERNEL_SRCS[kernel]:
        with open(os.path.join(ROOT, "dit_weight_compression_tile_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_for_kernel(kernel, key):
    """DRAM bytes per launch (read + write) from the committed ncu record for this workload key,
    if it was captured on the kernel's current sources; None otherwise"""
    if not os.path.exists(PROFILE_TRAFFIC) or kernel not in KERNEL_SRCS:
        return None
    with open(PROFILE_TRAFFIC) as f:
        d = json.load(f)
    rec = d.get(kernel, {})
    if rec.get("sources_sha256_16") != kernel_source_hash(kernel):
        return None
    w = rec.get("workloads", {}).get(key)
    return None if w is None else w.get("dram_bytes_per_launch")


def traffic_key(a):
    """the record's key for a workload: its name, plus the rate and shape when they differ from the
    workload's own"""
    wl = WORKLOADS[a.workload]
    key = a.workload
    if a.target != wl["target"]:
        key += f"@{a.target:g}"
    if getattr(a, "shape", None):
        key += f"[{a.shape}]"
    return key


# ------------------------------------------------------------------ the reference arm
def run_reference(a, rank, world):
    """the CPU oracle decoder as the reference arm: each step decodes a bounded, rotating range
    of tiles of the workload's first stream, sized so that the whole run stays near a minute"""
    if rank != 0:
        return
    from oracle import oracle as O
    blob = oracle_first_stream(a)
    rc, info = O.parse(blob)
    T, per_tile_w = info.n_tiles, 32 * info.blocks_per_lane * 8
    esz = 2 if WORKLOADS[a.workload]["container"] in (0, "bf16") else 1
    from concurrent.futures import ThreadPoolExecutor
    ncores = host_cores()
    n_cal = min(16, T)
    t0 = time.perf_counter()
    O.decode(blob, 0, n_cal, want_v=False)
    sec_per_tile = (time.perf_counter() - t0) / n_cal
    budget = 60.0 / max(1, a.steps + a.warmup)
    tiles = max(1, min(T - 1, int(budget * ncores / sec_per_tile))) if T > 1 else 1
    start = 0
    pool = ThreadPoolExecutor(ncores)

    def one(r):
        rc, st, _, _ = O.decode(blob, r[0], r[1], want_v=False)
        assert rc == 0 and st == 0

    def step():
        # a step: `tiles` consecutive tiles split into one range per host core
        nonlocal start
        if start + tiles > max(1, T - 1):
            start = 0
        cuts = [start + (tiles * i) // ncores for i in range(ncores + 1)]
        list(pool.map(one, [(cuts[i], cuts[i + 1]) for i in range(ncores) if cuts[i + 1] > cuts[i]]))
        start += tiles

    for _ in range(a.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(a.steps):
        step()
    t = time.perf_counter() - t0
    pool.shutdown()
    out_bytes = tiles * per_tile_w * esz * a.steps
    gbs = out_bytes / t / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s",
            "n_gpus": world, "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(1e3 * t / a.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u32+f32",
            "data": "synthetic", "config": bench_config(a, world),
            "stream": {"actual_bpp": round(info.actual_bpp, 4), "coding": "paired" if info.paired else "single",
                       "n_tiles": info.n_tiles, "blocks_per_lane": info.blocks_per_lane,
                       "encoder": "the oracle's compressor (first tensor of the workload)"},
            "gweights_per_s": round(tiles * per_tile_w * a.steps / t / 1e9, 4),
            "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": ncores, "kind": "oracle",
                             "sample": f"{tiles} of {T} tiles ({tiles * per_tile_w} weights) of the first "
                                       f"stream per step, decoded by the C oracle on {ncores} threads"},
            "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def oracle_first_stream(a):
    """the workload's first tensor encoded by the oracle's own compressor (the reference arm decodes
    a sample of it; the oracle's bytes equal the library's, and this arm loads no library code)"""
    from oracle import oracle as O
    wl = WORKLOADS[a.workload]
    name, make = wl["layers"]()[0]
    container = {0: 0, "bf16": O.BF16, "int8": O.INT8, "fp8_e4m3": O.FP8E4M3}[wl["container"]]
    rc, blob = O.compress(make(), a.target, container=container)
    assert rc == O.OK, rc
    return blob


# ------------------------------------------------------------------ our arm
def run_ours(a, rank, world, local_rank):
    from dit_weight_compression_tile_b200 import binding as B
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    layers, t_enc, rel_l2 = compress_layers(a)
    infos = [B.stream_info(blob) for _, blob in layers]
    n_weights = sum(i.rows * i.cols for i in infos)
    in_bytes = sum(i.storage_nbytes for i in infos)
    out_bytes = sum(i.out_nbytes for i in infos)
    # rotate device copies so that every step reads and writes more than the L2 holds
    rot = l2_policy(a)[0]
    stream = torch.cuda.Stream(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    blobs, works, outs = [], [], []
    with torch.cuda.stream(stream):
        for r in range(rot):
            for (_, blob), info in zip(layers, infos):
                d = blob.to(dev)
                blobs.append(d)
                # each device copy gets its slot tables once (ep_prepare), as when weights land
                works.append(B.prepare(d, info, status=status, stream=stream))
                outs.append(torch.empty(info.shape, dtype=info.dtype, device=dev))
    per = [infos[i % len(infos)] for i in range(len(blobs))]

    ntens = len(infos)

    def decode_steps(first, count):
        # `count` steps from copy `first` on: each step decodes every tensor of one copy
        for j in range(count):
            r = (first + j) % rot
            for i in range(ntens):
                k = r * ntens + i
                B.decompress(blobs[k], per[k], workspace=works[k], out=outs[k], status=status, stream=stream)

    # first calls outside capture: sets the kernel attributes, checks the output
    with torch.cuda.stream(stream):
        decode_steps(0, rot)
    torch.cuda.synchronize(dev)
    assert int(status.item()) == 0, "decode reported stream damage"
    # exactly a.steps timed steps: whole replays of a graph of `rot` steps, then a graph of the rest
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        decode_steps(0, rot)
    replays, rest = divmod(a.steps, rot)
    tail = None
    if rest:
        tail = torch.cuda.CUDAGraph()
        with torch.cuda.graph(tail, stream=stream):
            decode_steps(0, rest)
    steps = a.steps
    with torch.cuda.stream(stream):
        for _ in range(max(1, -(-a.warmup // rot))):
            graph.replay()
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(replays + 2)]
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index if dev.index is not None else 0) as clk:
        with torch.cuda.stream(stream):
            ev[0].record(stream)
            for r in range(replays):
                graph.replay()
                ev[r + 1].record(stream)
            if tail is not None:
                tail.replay()
            ev[-1].record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    per_replay = [ev[r].elapsed_time(ev[r + 1]) for r in range(replays)]
    total_ms = max_over_ranks(ev[0].elapsed_time(ev[-1]), world, dev)
    assert int(status.item()) == 0
    step_s = total_ms / steps / 1e3
    # the decode launches of one step run back to back on one stream: the mean launch time is
    # the timed region over its launches; median and minimum come from whole replays
    kernel_s = ev[0].elapsed_time(ev[-1]) / steps / 1e3
    per_launch_us = sorted(1e3 * x / (rot * ntens) for x in per_replay)
    value = job_rate(out_bytes, world, step_s) / 1e9
    peak, peak_kind = measured_peaks()
    achieved = (in_bytes + out_bytes) / kernel_s / 1e9
    traffic = traffic_for_kernel("decode_kernel", traffic_key(a))

    # the tables' preparation by itself (once per device copy of a stream)
    prep_reps = max(1, 200 // len(infos))
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        p0.record(stream)
        for _ in range(prep_reps):
            for i, info in enumerate(infos):
                B.prepare(blobs[i], info, workspace=works[i], stream=stream)
        p1.record(stream)
    torch.cuda.synchronize(dev)
    prepare_us = p0.elapsed_time(p1) * 1e3 / (prep_reps * len(infos))

    # end to end through the C ABI with host buffers (ep_decompress_host): every step, for every
    # tensor, the pinned stream copied in, the tables, the decode and the container copied back
    # into pinned memory.  Consecutive (step, tensor) units alternate between two CUDA streams with
    # their own device scratch, so that one unit's device-to-host read overlaps the next unit's
    # host-to-device copy
    host_blobs = [blob.pin_memory() for _, blob in layers]
    biggest = max(range(len(infos)), key=lambda i: infos[i].out_nbytes)
    host_outs = [torch.empty(infos[biggest].shape, dtype=infos[biggest].dtype).pin_memory() for _ in range(2)]
    streams = [stream, torch.cuda.Stream(dev)]
    scratch_nbytes = max(B.decompress_host_scratch(info) for info in infos)
    scratches = [torch.empty(scratch_nbytes, dtype=torch.uint8, device=dev) for _ in range(2)]
    unit = [0]

    def e2e_step():
        for i, info in enumerate(infos):
            j = unit[0] % 2
            unit[0] += 1
            o = host_outs[j].view(-1)[: info.rows * info.cols].view(info.shape)
            B.decompress_host(host_blobs[i], info, out=o, scratch=scratches[j], stream=streams[j], sync=False)

    e2e_steps = max(2, min(200, int(0.5 / max(1e-9, (in_bytes + out_bytes) / 40e9))))
    e2e_step()
    torch.cuda.synchronize(dev)
    e0, e1, ej = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
                  torch.cuda.Event())
    e0.record(streams[0])
    streams[1].wait_event(e0)
    for _ in range(e2e_steps):
        e2e_step()
    ej.record(streams[1])
    streams[0].wait_event(ej)
    e1.record(streams[0])
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e_value = job_rate(out_bytes * e2e_steps, world, e2e_ms / 1e3) / 1e9

    if rank != 0:
        return
    i0 = infos[0]
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": steps,
        "warmup": a.warmup, "ms_per_step": round(step_s * 1e3, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "u32+f32", "data": "synthetic",
        "config": bench_config(a, world),
        "stream": {"actual_bpp": round(8.0 * in_bytes / n_weights, 4), "coding": coding_label(infos),
                   "n_tensors": len(infos), "n_tiles": sum(i.n_tiles for i in infos),
                   "blocks_per_lane": i0.blocks_per_lane, "rel_l2": round(rel_l2, 5),
                   "rel_l2_note": "||W - What|| / ||W|| against the source weights over the whole workload"},
        "gweights_per_s": round(job_rate(n_weights, world, step_s) / 1e9, 3),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic, "peak_kind": peak_kind,
                     "algorithmic_bytes_per_launch": (in_bytes + out_bytes) // len(infos),
                     "kernel_us": round(kernel_s * 1e6 / len(infos), 3),
                     "kernel_us_median": round(statistics.median(per_launch_us), 3) if per_launch_us else None,
                     "kernel_us_min": round(per_launch_us[0], 3) if per_launch_us else None},
        "e2e": {"value": round(e2e_value, 3), "unit": "GB/s", "h2d_bytes_per_step": in_bytes,
                "d2h_bytes_per_step": out_bytes},
        "gpu_launches": steps * len(infos),
        "tables": {"prepare_us": round(prepare_us, 3), "note": "slot tables built once per device copy of "
                   "a stream (ep_prepare); each step stages them into shared memory and decodes"},
        "clocks": clk.summary(),
        "encode_s": round(t_enc, 3),
    }
    if world == 1 and not a.no_cpu_baseline:
        esz = i0.out_nbytes // (i0.rows * i0.cols)
        ncores = host_cores()
        d1, e1, t1 = cpu_oracle_decode(layers[0][1].numpy(), a.cpu_seconds / 2, 1)
        done, el, tiles = cpu_oracle_decode(layers[0][1].numpy(), a.cpu_seconds / 2, ncores)
        line["cpu_baseline"] = {"value": round(done * esz / el / 1e9, 4), "unit": "GB/s", "cores": ncores,
                                "kind": "oracle",
                                "sample": f"{tiles} tiles ({done} weights) of the first stream, decoded by the "
                                          f"C oracle on {ncores} threads in {el:.1f} s",
                                "single_core": {"value": round(d1 * esz / e1 / 1e9, 4), "unit": "GB/s",
                                                "sample": f"{t1} tiles in {e1:.1f} s on one thread"}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ the lossless Tile-ANS workload
def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16) if t.element_size() == 2 else \
        t.contiguous().view(torch.uint8).numpy()


def run_ours_tile_ans(a, rank, world, local_rank):
    """the lossless scheme's decode (ep_ans_decompress) of the workload's tensor, timed as the
    lattice decode is: streams, tables and outputs resident, rotating copies past the L2, CUDA-graph
    replays of exactly --steps decodes; e2e copies the stream in and the tensor out every step"""
    from dit_weight_compression_tile_b200 import binding as B
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    name, make = WORKLOADS[a.workload]["layers"]()[0]
    w = make()
    t0 = time.perf_counter()
    blob = B.ans_compress(w)
    t_enc = time.perf_counter() - t0
    info = B.ans_stream_info(blob)
    in_bytes, out_bytes, n = info.storage_nbytes, info.out_nbytes, info.n_elems
    rot = l2_policy(a)[0]
    stream = torch.cuda.Stream(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    with torch.cuda.stream(stream):
        blobs = [blob.to(dev) for _ in range(rot)]
        works = [B.ans_prepare(d, info, status=status, stream=stream) for d in blobs]
        outs = [torch.empty(info.shape, dtype=info.torch_dtype, device=dev) for _ in range(rot)]

    def steps_(first, count):
        for j in range(count):
            r = (first + j) % rot
            B.ans_decompress(blobs[r], info, workspace=works[r], out=outs[r], status=status, stream=stream)

    with torch.cuda.stream(stream):
        steps_(0, rot)
    torch.cuda.synchronize(dev)
    assert int(status.item()) == 0 and torch.equal(outs[0].cpu().view(torch.int16), w.view(torch.int16)), \
        "lossless decode differs from the input"
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        steps_(0, rot)
    replays, rest = divmod(a.steps, rot)
    tail = None
    if rest:
        tail = torch.cuda.CUDAGraph()
        with torch.cuda.graph(tail, stream=stream):
            steps_(0, rest)
    with torch.cuda.stream(stream):
        for _ in range(max(1, -(-a.warmup // rot))):
            graph.replay()
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(replays + 2)]
    with ClockSampler(dev.index if dev.index is not None else 0) as clk:
        with torch.cuda.stream(stream):
            ev[0].record(stream)
            for r in range(replays):
                graph.replay()
                ev[r + 1].record(stream)
            if tail is not None:
                tail.replay()
            ev[-1].record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    per_launch_us = sorted(1e3 * ev[r].elapsed_time(ev[r + 1]) / rot for r in range(replays))
    total_ms = max_over_ranks(ev[0].elapsed_time(ev[-1]), world, dev)
    assert int(status.item()) == 0
    step_s = total_ms / a.steps / 1e3
    kernel_s = ev[0].elapsed_time(ev[-1]) / a.steps / 1e3
    peak, peak_kind = measured_peaks()
    achieved = (in_bytes + out_bytes) / kernel_s / 1e9

    # end to end through the public API's host-resident path: the pinned stream copied in, the
    # decode, the tensor copied back into pinned memory, on two CUDA streams so that one step's
    # copy-out overlaps the next step's copy-in
    host_blob = blob.pin_memory()
    host_outs = [torch.empty(info.shape, dtype=info.torch_dtype).pin_memory() for _ in range(2)]
    streams = [stream, torch.cuda.Stream(dev)]
    dblobs = [torch.empty_like(blobs[0]) for _ in range(2)]
    douts = [torch.empty_like(outs[0]) for _ in range(2)]
    dworks = [torch.empty_like(works[0]) for _ in range(2)]
    e2e_steps = max(2, min(200, int(0.5 / max(1e-9, (in_bytes + out_bytes) / 40e9))))

    def e2e_step(j):
        s_ = streams[j % 2]
        with torch.cuda.stream(s_):
            dblobs[j % 2].copy_(host_blob, non_blocking=True)
            B.ans_prepare(dblobs[j % 2], info, workspace=dworks[j % 2], stream=s_)
            B.ans_decompress(dblobs[j % 2], info, workspace=dworks[j % 2], out=douts[j % 2], stream=s_)
            host_outs[j % 2].copy_(douts[j % 2], non_blocking=True)

    e2e_step(0)
    torch.cuda.synchronize(dev)
    e0, e1, ej = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True), torch.cuda.Event())
    e0.record(streams[0])
    streams[1].wait_event(e0)
    for j in range(e2e_steps):
        e2e_step(j)
    ej.record(streams[1])
    streams[0].wait_event(ej)
    e1.record(streams[0])
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    if rank != 0:
        return
    line = {
        "metric": TILE_ANS_METRIC, "value": round(job_rate(out_bytes, world, step_s) / 1e9, 2), "unit": "GB/s",
        "n_gpus": world, "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(step_s * 1e3, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u32+u8", "data": "synthetic",
        "config": bench_config(a, world),
        "stream": {"ratio": round(info.ratio, 5), "bits_per_element": round(8.0 * in_bytes / n, 4),
                   "n_tiles": info.n_tiles, "blocks_per_lane": info.blocks_per_lane, "lossless": True},
        "gelements_per_s": round(job_rate(n, world, step_s) / 1e9, 3),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic_for_kernel("ans_decode_kernel", traffic_key(a)),
                     "peak_kind": peak_kind,
                     "algorithmic_bytes_per_launch": in_bytes + out_bytes, "kernel_us": round(kernel_s * 1e6, 3),
                     "kernel_us_median": round(statistics.median(per_launch_us), 3) if per_launch_us else None,
                     "kernel_us_min": round(per_launch_us[0], 3) if per_launch_us else None},
        "e2e": {"value": round(job_rate(out_bytes * e2e_steps, world, e2e_ms / 1e3) / 1e9, 3), "unit": "GB/s",
                "h2d_bytes_per_step": in_bytes, "d2h_bytes_per_step": out_bytes},
        "gpu_launches": a.steps,
        "clocks": clk.summary(),
        "encode_s": round(t_enc, 3),
    }
    if world == 1 and not a.no_cpu_baseline:
        from concurrent.futures import ThreadPoolExecutor
        from oracle import oracle as O
        ncores = host_cores()
        b_np = blob.numpy()
        t0 = time.perf_counter()
        done = 0
        with ThreadPoolExecutor(ncores) as ex:
            while time.perf_counter() - t0 < a.cpu_seconds:
                cuts = [(info.n_tiles * i) // ncores for i in range(ncores + 1)]
                list(ex.map(lambda i: O.ta_decode(b_np, cuts[i], cuts[i + 1]), range(ncores)))
                done += 1
        el = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": round(done * out_bytes / el / 1e9, 4), "unit": "GB/s", "cores": ncores,
                                "kind": "oracle", "sample": f"{done} whole-stream decodes by the C oracle on "
                                                            f"{ncores} threads in {el:.1f} s"}
    print(json.dumps(line), flush=True)


def run_reference_tile_ans(a, rank, world):
    """the oracle's Tile-ANS decoder on every host core, on the oracle's own stream of the workload"""
    if rank != 0:
        return
    from concurrent.futures import ThreadPoolExecutor
    from oracle import oracle as O
    name, make = WORKLOADS[a.workload]["layers"]()[0]
    w = make()
    rc, blob = O.ta_compress(_bits(w), O.BF16, shape=tuple(w.shape))
    assert rc == O.OK
    rc, info = O.ta_parse(blob)
    ncores = host_cores()
    out_bytes = info.n * 2
    pool = ThreadPoolExecutor(ncores)
    cuts = [(info.n_tiles * i) // ncores for i in range(ncores + 1)]

    def step():
        list(pool.map(lambda i: O.ta_decode(blob, cuts[i], cuts[i + 1]), range(ncores)))

    for _ in range(a.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(a.steps):
        step()
    t = time.perf_counter() - t0
    pool.shutdown()
    gbs = out_bytes * a.steps / t / 1e9
    line = {"impl": "reference", "metric": TILE_ANS_METRIC, "value": round(gbs, 4), "unit": "GB/s",
            "n_gpus": world, "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(1e3 * t / a.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u32+u8",
            "data": "synthetic", "config": bench_config(a, world),
            "gelements_per_s": round(info.n * a.steps / t / 1e9, 4),
            "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": ncores, "kind": "oracle",
                             "sample": f"the whole stream ({info.n_tiles} tiles) per step, decoded by the C oracle "
                                       f"on {ncores} threads"},
            "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)

LINEAR_METRIC = "fused decode + tcgen05 GEMM Gweights/s (DiT block linears, 16 tokens); % of HBM roofline"


def run_ours_linear(a, rank, world, local_rank):
    """the decode fused into the tcgen05 GEMM (ep_linear_fused) on one DiT block's four linear
    layers at a small token count: one step = the four products Y = X W^T, W from GEMM-ordered
    streams, streams rotating past the L2 as in the other workloads.  Beside it, timed the same way
    for context: the decode into a buffer followed by the library GEMM, and the library GEMM on
    the BF16 weights (nn.Linear).  The decode-then-GEMM leg reads the same weights' row-ordered
    streams at the same rate"""
    import torch.nn.functional as F
    from dit_weight_compression_tile_b200 import binding as B
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = WORKLOADS[a.workload]
    m = wl["tokens"]
    rot = l2_policy(a)[0]
    stream = torch.cuda.Stream(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    g = torch.Generator().manual_seed(5)
    layers, t_enc = [], 0.0
    code_dtype = {"int8": torch.int8, "fp8_e4m3": torch.float8_e4m3fn}.get(wl["container"])
    for name, make in wl["layers"]():
        w = make().to(dev)
        torch.cuda.synchronize(dev)
        t0 = time.perf_counter()
        blob = B.compress_device(w, a.target, container=wl["container"], layout=B.LAYOUT_GEMM)
        torch.cuda.synchronize(dev)
        t_enc += time.perf_counter() - t0
        info = B.stream_info(blob.cpu())
        # the same weights in the row order, for the decode-then-GEMM comparison (its decode stores
        # whole rows, the faster order for a decode into memory)
        rblob = B.compress_device(w, a.target, container=wl["container"])
        rinfo = B.stream_info(rblob.cpu())
        x = (torch.randn(m, info.cols, generator=g) * 0.5).to(torch.bfloat16)
        with torch.cuda.stream(stream):
            blobs = [blob.clone() for _ in range(rot)]
            tables = B.prepare(blobs[0], info, status=status, stream=stream)  # the copies hold the same stream
            rblobs = [rblob.clone() for _ in range(rot)]
            rtables = B.prepare(rblobs[0], rinfo, status=status, stream=stream)
        layers.append(dict(name=name, w=w, info=info, blobs=blobs, tables=tables, rinfo=rinfo, rblobs=rblobs,
                           rtables=rtables, x_host=x, x=x.to(dev),
                           y=torch.empty(m, info.rows, dtype=torch.bfloat16, device=dev),
                           work=torch.zeros(B.linear_fused_workspace(info, m), dtype=torch.uint8, device=dev),
                           wbuf=torch.empty(info.rows, info.cols, dtype=code_dtype or torch.bfloat16, device=dev),
                           sw=rblob[rinfo.off_scales: rinfo.off_scales + 4 * rinfo.rows].view(torch.float32)
                           if code_dtype else None))
    torch.cuda.synchronize(dev)

    def fused(r, s_=stream):
        for L in layers:
            B.linear_fused(L["x"], L["blobs"][r], L["info"], L["tables"], out=L["y"], work=L["work"],
                           status=status, stream=s_)

    def library_w8a8(L, codes):
        """what the per-row-quantized layers do unfused: the activations quantized per token with
        torch ops, then torch._int_mm (INT8, tokens padded to 32: it takes more than 16 rows) or
        torch._scaled_mm (FP8), and the two scales"""
        x2 = L["x"]
        amax = x2.abs().amax(dim=1, keepdim=True).float()
        bound = 127.0 if code_dtype == torch.int8 else 448.0
        sx = torch.where(amax > 0, amax / torch.full_like(amax, bound), torch.ones_like(amax))  # rounded division
        q = x2.float() / sx
        if code_dtype == torch.int8:
            qp = torch.zeros(32, x2.shape[1], dtype=torch.int8, device=x2.device)
            qp[:m] = q.round().clamp(-127, 127).to(torch.int8)
            acc = torch._int_mm(qp, codes.t())[:m]
            return (acc.float() * sx * L["sw"][None, :]).to(torch.bfloat16)
        q = q.clamp(-448.0, 448.0).to(torch.float8_e4m3fn)
        return torch._scaled_mm(q, codes.t(), scale_a=sx, scale_b=L["sw"][None, :].contiguous(),
                                out_dtype=torch.bfloat16)

    def unfused(r):
        for L in layers:
            wd = B.decompress(L["rblobs"][r], L["rinfo"], workspace=L["rtables"], out=L["wbuf"], stream=stream)
            if code_dtype is None:
                F.linear(L["x"], wd)
            else:
                library_w8a8(L, wd)

    def dense(r):
        for L in layers:
            F.linear(L["x"], L["w"])

    # the fused result against the library GEMM on the decoded weight: the same BF16 products summed
    # in fp32 in another order (bound K 2^-24 sum |x w| + one BF16 rounding each)
    with torch.cuda.stream(stream):
        fused(0)
    torch.cuda.synchronize(dev)
    assert int(status.item()) == 0, "fused GEMM status"
    for L in layers:
        wd = B.decompress(L["blobs"][0], L["info"], workspace=L["tables"])
        if code_dtype is not None:
            # INT8: the same bits as the layer's unfused arithmetic; FP8: the same up to the order
            # of the fp32 sums
            lib_y = library_w8a8(L, wd)
            if code_dtype == torch.int8:
                assert torch.equal(L["y"], lib_y), L["name"]
            else:
                assert torch.allclose(L["y"].float(), lib_y.float(), rtol=2 ** -6, atol=1e-3), L["name"]
            continue
        wd = wd.float()
        ref = L["x"].float() @ wd.T
        mag = L["x"].float().abs() @ wd.abs().T
        tol = L["info"].cols * 2.0 ** -24 * mag + 2.0 ** -8 * ref.abs()
        assert bool(((L["y"].float() - ref).abs() <= tol + 2.0 ** -8 * L["y"].float().abs()).all()), L["name"]

    def timed(body, steps):
        # once outside the capture: libraries create their per-stream handles on first use, which a
        # capture does not allow
        with torch.cuda.stream(stream):
            body(0)
        torch.cuda.synchronize(dev)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for r in range(rot):
                body(r)
        replays, rest = divmod(steps, rot)
        tail = None
        if rest:
            tail = torch.cuda.CUDAGraph()
            with torch.cuda.graph(tail, stream=stream):
                for r in range(rest):
                    body(r)
        with torch.cuda.stream(stream):
            for _ in range(max(1, -(-a.warmup // rot))):
                graph.replay()
        torch.cuda.synchronize(dev)
        if world > 1:
            torch.distributed.barrier()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(replays + 2)]
        with torch.cuda.stream(stream):
            ev[0].record(stream)
            for r in range(replays):
                graph.replay()
                ev[r + 1].record(stream)
            if tail is not None:
                tail.replay()
            ev[-1].record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            torch.distributed.barrier()
        per_step = sorted(1e3 * ev[r].elapsed_time(ev[r + 1]) / rot for r in range(replays))
        return ev[0].elapsed_time(ev[-1]), per_step

    with ClockSampler(dev.index if dev.index is not None else 0) as clk:
        fused_ms, per_step = timed(fused, a.steps)
    total_ms = max_over_ranks(fused_ms, world, dev)
    assert int(status.item()) == 0
    unfused_ms, _ = timed(unfused, a.steps)
    dense_ms, _ = timed(dense, a.steps)
    # each layer alone, the same three ways (fewer steps: context, not the metric)
    per_layer = {}
    n_layer = max(a.warmup + 1, min(a.steps, 100))
    for L in layers:
        one = [L]

        def f1(r, one=one):
            for L_ in one:
                B.linear_fused(L_["x"], L_["blobs"][r], L_["info"], L_["tables"], out=L_["y"], work=L_["work"],
                               status=status, stream=stream)

        def u1(r, one=one):
            for L_ in one:
                wd = B.decompress(L_["rblobs"][r], L_["rinfo"], workspace=L_["rtables"], out=L_["wbuf"],
                                  stream=stream)
                if code_dtype is None:
                    F.linear(L_["x"], wd)
                else:
                    library_w8a8(L_, wd)

        def d1(r, one=one):
            for L_ in one:
                F.linear(L_["x"], L_["w"])

        per_layer[f'{L["info"].rows}x{L["info"].cols}'] = [round(1e3 * timed(fn, n_layer)[0] / n_layer, 2)
                                                          for fn in (f1, u1, d1)]
    nweights = sum(L["info"].rows * L["info"].cols for L in layers)
    stream_bytes = sum(L["info"].storage_nbytes for L in layers)
    act_bytes = sum(2 * m * (L["info"].cols + L["info"].rows) for L in layers)
    step_s = total_ms / a.steps / 1e3
    kernel_s = fused_ms / a.steps / 1e3
    peak, peak_kind = measured_peaks()
    achieved = (stream_bytes + act_bytes) / kernel_s / 1e9

    # end to end through the public API: x copied in from pinned memory, the four fused products,
    # y copied back into pinned memory, every step
    xs_host = [L["x_host"].pin_memory() for L in layers]
    ys_host = [torch.empty(m, L["info"].rows, dtype=torch.bfloat16).pin_memory() for L in layers]
    e2e_steps = max(4, min(400, a.steps))
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for j in range(e2e_steps):
            for L, xh, yh in zip(layers, xs_host, ys_host):
                L["x"].copy_(xh, non_blocking=True)
                B.linear_fused(L["x"], L["blobs"][j % rot], L["info"], L["tables"], out=L["y"], work=L["work"],
                               stream=stream)
                yh.copy_(L["y"], non_blocking=True)
        e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    if rank != 0:
        return
    line = {
        "metric": LINEAR_METRIC, "value": round(job_rate(nweights, world, step_s) / 1e9, 2), "unit": "Gweights/s",
        "n_gpus": world, "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(step_s * 1e3, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": bench_config(a, world),
        "stream": {"bpp": [round(L["info"].actual_bpp, 4) for L in layers], "paired": [L["info"].paired for L in layers],
                   "layout": "gemm"},
        "step_us": {"fused": round(1e3 * fused_ms / a.steps, 2),
                    ("decode_row_stream_then_library_gemm" if code_dtype is None else
                     "decode_row_stream_then_library_w8a8"): round(1e3 * unfused_ms / a.steps, 2),
                    "library_gemm_bf16_weights": round(1e3 * dense_ms / a.steps, 2),
                    "per_layer_fused_unfused_bf16": per_layer},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic_for_kernel("linear_kernel", traffic_key(a)),
                     "peak_kind": peak_kind, "algorithmic_bytes_per_step": stream_bytes + act_bytes,
                     "note": "four linear_kernel launches per step; the fused kernel is bound by its decoding "
                             "warps, not by HBM",
                     "step_us_median": round(statistics.median(per_step), 3) if per_step else None,
                     "step_us_min": round(per_step[0], 3) if per_step else None},
        "e2e": {"value": round(job_rate(nweights * e2e_steps, world, e2e_ms / 1e3) / 1e9, 3), "unit": "Gweights/s",
                "h2d_bytes_per_step": sum(2 * m * L["info"].cols for L in layers),
                "d2h_bytes_per_step": sum(2 * m * L["info"].rows for L in layers)},
        "gpu_launches": len(layers) * a.steps,
        "clocks": clk.summary(),
        "encode_s": round(t_enc, 3),
    }
    if world == 1 and not a.no_cpu_baseline:
        line["cpu_baseline"] = cpu_linear_baseline(a, layers, m)
    print(json.dumps(line), flush=True)


def _oracle_weights_f32(O, blob_np, wd):
    """the oracle's decoded container as fp32 weights: BF16 as it is, INT8 / FP8 codes times the
    stream's row scales"""
    rc, info = O.parse(blob_np)
    if info.container_dtype == O.BF16:
        return (wd.view(np.uint16).astype(np.uint32) << 16).view(np.float32)
    scales = np.frombuffer(blob_np.tobytes(), np.float32, count=info.rows, offset=info.off_scales)
    if info.container_dtype == O.INT8:
        codes = wd.astype(np.float32)
    else:
        codes = torch.from_numpy(wd.view(np.uint8).copy()).view(torch.float8_e4m3fn).float().numpy()
    return codes * scales[:, None]


def cpu_linear_baseline(a, layers, m):
    """the oracle (tile-parallel decode on every host core) plus a numpy fp32 GEMM, on a bounded
    sample: the 3072x3072 layer's stream, whole, repeated for about --cpu-seconds"""
    from oracle import oracle as O
    L = min(layers, key=lambda L: L["info"].rows * L["info"].cols)
    blob_np = L["blobs"][0].cpu().numpy()
    rc, oinfo = O.parse(blob_np)
    assert rc == 0
    x_np = L["x_host"].float().numpy()
    ncores = host_cores()
    done = 0
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < a.cpu_seconds:
        rc, st, _, wd = O.decode_parallel(blob_np, threads=ncores, want_v=False)
        assert rc == 0 and st == 0
        _ = x_np @ _oracle_weights_f32(O, blob_np, wd).T
        done += 1
    el = time.perf_counter() - t0
    n = oinfo.rows * oinfo.cols
    return {"value": round(done * n / el / 1e9, 4), "unit": "Gweights/s", "cores": ncores, "kind": "oracle",
            "sample": f"{done} decodes of the {oinfo.rows}x{oinfo.cols} layer's stream by the C oracle on {ncores} "
                      f"threads, each followed by x W^T in numpy fp32 ({m} tokens), in {el:.1f} s"}


def run_reference_linear(a, rank, world):
    """the oracle as the reference arm of the fused GEMM: the oracle's own GEMM-ordered stream of the
    block's 3072x3072 layer, decoded on every host core and multiplied in numpy fp32, each step"""
    if rank != 0:
        return
    from oracle import oracle as O
    wl = WORKLOADS[a.workload]
    m = wl["tokens"]
    name, make = [(n, f) for n, f in wl["layers"]() if n.endswith(".out")][0]
    w = make()
    rc, blob = O.compress(w, a.target, container={0: 0, "int8": O.INT8, "fp8_e4m3": O.FP8E4M3}[wl["container"]],
                          layout=1)
    assert rc == 0
    rc, oinfo = O.parse(blob)
    g = torch.Generator().manual_seed(5)
    x_np = (torch.randn(m, oinfo.cols, generator=g) * 0.5).to(torch.bfloat16).float().numpy()
    ncores = host_cores()

    def step():
        rc_, st_, _, wd = O.decode_parallel(blob, threads=ncores, want_v=False)
        assert rc_ == 0 and st_ == 0
        return x_np @ _oracle_weights_f32(O, blob, wd).T

    for _ in range(a.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(a.steps):
        step()
    t = time.perf_counter() - t0
    n = oinfo.rows * oinfo.cols
    rate = n * a.steps / t / 1e9
    line = {"impl": "reference", "metric": LINEAR_METRIC, "value": round(rate, 4), "unit": "Gweights/s",
            "n_gpus": world, "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(1e3 * t / a.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": bench_config(a, world),
            "cpu_baseline": {"value": round(rate, 4), "unit": "Gweights/s", "cores": ncores, "kind": "oracle",
                             "sample": f"the {oinfo.rows}x{oinfo.cols} layer's stream per step, decoded by the C oracle "
                                       f"on {ncores} threads, then x W^T in numpy fp32 with the decoded weights "
                                       f"({m} tokens)"},
            "e2e": {"value": round(rate, 4), "unit": "Gweights/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    a = args_()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if a.impl == "reference":
        (run_reference_tile_ans if is_tile_ans(a) else run_reference_linear if is_linear(a) else run_reference)(
            a, rank, world)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        (run_ours_tile_ans if is_tile_ans(a) else run_ours_linear if is_linear(a) else run_ours)(
            a, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
