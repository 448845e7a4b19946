"""Benchmark of the fused lattice-rANS tile decode on B200.

One step = one fused decode (the whole hot path: tables, rANS tiles, E8 reconstruction,
container stores) of the 4096x4096 BF16 weight matrix with per-row log-normal std,
compressed at 4 bits per weight.  Streams and outputs rotate over 8 device copies
(8 x 41.8 MB > the 126 MB L2), so every step reads its stream from HBM.  Launches are
replayed from a CUDA graph of 8 decodes so that host launch cost does not gate the GPU.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

N > 1 runs N independent replicas (the decode has no exchange step; see the design notes):
one process per GPU under torchrun, timed on the device, max over ranks.
The reference arm (--impl reference) is the CPU oracle decoder, timed on the host cores.
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

WORKLOAD = {"workload": "lognormal_rows_4096x4096_bf16", "rows": 4096, "cols": 4096, "target_bpp": 4.0,
            "distribution": "N(0, s_r^2), s_r = 0.02 exp(0.3 g), seed 1", "container": "bf16"}
METRIC = "fused decode GB/s (container out) & Gweights/s at 4 bpp; % of HBM roofline"
ROTATE = 8
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "decode_kernel_traffic.json")
KERNEL_SRC = os.path.join(ROOT, "dit_weight_compression_tile_b200", "csrc", "decode.cu")


def args_():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=40000)
    p.add_argument("--warmup", type=int, default=16)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--cpu-seconds", type=float, default=12.0)
    p.add_argument("--no-cpu-baseline", action="store_true")
    return p.parse_args()


def workload_tensor():
    from dit_weight_compression_tile_b200 import synth
    return synth.row_lognormal(WORKLOAD["rows"], WORKLOAD["cols"], 1)


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

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                pass
            time.sleep(0.02)

    def __enter__(self):
        if self.nv:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.nv:
            self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"], "samples": 0}
        names = [n for bit, n in NVML_REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


# ------------------------------------------------------------------ CPU oracle leg
def cpu_oracle_decode(blob_np, seconds):
    """the oracle decoder, as it stands, on one host core, repeated for a bounded time"""
    from oracle import oracle as O
    n, t0 = 0, time.perf_counter()
    while True:
        rc, st, _, out = O.decode(blob_np, want_v=False)
        assert rc == 0 and st == 0
        n += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return n, el, out


def traffic_for_kernel():
    """DRAM bytes per launch from the committed ncu summary, if it was taken on this kernel source"""
    if not os.path.exists(PROFILE_TRAFFIC):
        return None
    with open(PROFILE_TRAFFIC) as f:
        d = json.load(f)
    with open(KERNEL_SRC, "rb") as f:
        h = hashlib.sha256(f.read()).hexdigest()[:16]
    if d.get("kernel_sha256_16") != h or d.get("workload") != WORKLOAD["workload"]:
        return None
    return d.get("dram_bytes_per_launch")


# ------------------------------------------------------------------ the reference arm
def run_reference(a, rank, world):
    """the CPU oracle decoder as the reference arm: each step decodes a bounded, rotating range
    of tiles of the same stream, sized so that the whole run stays near a minute"""
    if rank != 0:
        return
    from dit_weight_compression_tile_b200 import binding as B
    from oracle import oracle as O
    w = workload_tensor()
    blob = B.compress(w, WORKLOAD["target_bpp"]).numpy()
    info = B.stream_info(torch.from_numpy(blob))
    T, per_tile_w = info.n_tiles, 32 * info.blocks_per_lane * 8
    n_cal = min(64, T)
    t0 = time.perf_counter()
    O.decode(blob, 0, n_cal, want_v=False)
    sec_per_tile = (time.perf_counter() - t0) / n_cal
    budget = 60.0 / max(1, a.steps + a.warmup)
    tiles = max(1, min(T - 1, int(budget / sec_per_tile)))  # full tiles only (the last may be partial)
    start = 0
    buf = np.zeros(info.shape, np.uint16)

    def step():
        nonlocal start
        if start + tiles > T - 1:
            start = 0
        rc, st, _, _ = O.decode(blob, start, start + tiles, want_v=False, out_buf=buf)
        assert rc == 0 and st == 0
        start += tiles

    for _ in range(a.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(a.steps):
        step()
    t = time.perf_counter() - t0
    out_bytes = tiles * per_tile_w * 2 * a.steps
    gbs = out_bytes / t / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s",
            "n_gpus": world, "steps": a.steps, "warmup": a.warmup, "ms_per_step": round(1e3 * t / a.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u32+f32",
            "data": "synthetic", "config": dict(WORKLOAD, l2="n/a (host)"),
            "gweights_per_s": round(tiles * per_tile_w * a.steps / t / 1e9, 4),
            "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": f"{tiles} of {T} tiles ({tiles * per_tile_w} weights) of the 4096x4096 "
                                       "stream per step, decoded by the C oracle"},
            "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ our arm
def run_ours(a, rank, world, local_rank):
    from dit_weight_compression_tile_b200 import binding as B
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = workload_tensor()
    t_enc = time.perf_counter()
    blob_cpu = B.compress(w, WORKLOAD["target_bpp"])
    t_enc = time.perf_counter() - t_enc
    info = B.stream_info(blob_cpu)
    n_weights = info.rows * info.cols
    out_bytes, in_bytes = info.out_nbytes, info.storage_nbytes
    blobs = [blob_cpu.to(dev) for _ in range(ROTATE)]
    outs = [torch.empty(info.shape, dtype=info.dtype, device=dev) for _ in range(ROTATE)]
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.Stream(dev)
    # each device copy of the stream gets its slot tables once (ep_prepare), as when weights land
    # on the device; every step then decodes with them
    with torch.cuda.stream(stream):
        works = [B.prepare(blobs[i], info, status=status, stream=stream) for i in range(ROTATE)]
    # first calls outside capture: sets the kernel attributes, checks the output
    with torch.cuda.stream(stream):
        for i in range(ROTATE):
            B.decompress(blobs[i], info, workspace=works[i], out=outs[i], status=status, stream=stream)
    torch.cuda.synchronize(dev)
    assert int(status.item()) == 0, "decode reported stream damage"
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(ROTATE):
            B.decompress(blobs[i], info, workspace=works[i], out=outs[i], status=status, stream=stream)
    replays = max(1, -(-a.steps // ROTATE))
    steps = replays * ROTATE
    with torch.cuda.stream(stream):
        for _ in range(max(1, -(-a.warmup // ROTATE))):
            graph.replay()
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(replays + 1)]
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index if dev.index is not None else 0) as clk:
        with torch.cuda.stream(stream):
            ev[0].record(stream)
            for r in range(replays):
                graph.replay()
                ev[r + 1].record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    per_replay = [ev[r].elapsed_time(ev[r + 1]) for r in range(replays)]
    total_ms = ev[0].elapsed_time(ev[-1])
    if world > 1:
        t = torch.tensor([total_ms], device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        total_ms = float(t.item())
    assert int(status.item()) == 0
    kernel_s = statistics.mean(per_replay) / ROTATE / 1e3
    step_s = total_ms / steps / 1e3
    value = world * out_bytes / step_s / 1e9
    peak, peak_kind = measured_peaks()
    achieved = (in_bytes + out_bytes) / kernel_s / 1e9
    traffic = traffic_for_kernel()

    # the tables' preparation by itself (once per device copy of a stream)
    prep_reps = 200
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        p0.record(stream)
        for r in range(prep_reps):
            B.prepare(blobs[r % ROTATE], info, workspace=works[r % ROTATE], stream=stream)
        p1.record(stream)
    torch.cuda.synchronize(dev)
    prepare_us = p0.elapsed_time(p1) * 1e3 / prep_reps

    # end to end through the public API with host buffers: pinned H2D of the stream, the tables,
    # the decode, D2H of the container into pinned memory, every step
    host_blob = blob_cpu.pin_memory()
    host_out = torch.empty(info.shape, dtype=info.dtype).pin_memory()
    e2e_steps = max(8, min(200, a.steps // 200))
    dblob, dout, dwork = blobs[0], outs[0], works[0]

    def e2e_step():
        dblob.copy_(host_blob, non_blocking=True)
        B.prepare(dblob, info, workspace=dwork, stream=stream)
        B.decompress(dblob, info, workspace=dwork, out=dout, stream=stream)
        host_out.copy_(dout, non_blocking=True)

    for _ in range(3):
        with torch.cuda.stream(stream):
            e2e_step()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1)
    if world > 1:
        t = torch.tensor([e2e_ms], device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        e2e_ms = float(t.item())
    e2e_value = world * out_bytes * e2e_steps / (e2e_ms / 1e3) / 1e9

    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": steps,
        "warmup": a.warmup, "ms_per_step": round(step_s * 1e3, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "u32+f32", "data": "synthetic",
        "config": dict(WORKLOAD, l2=f"inputs larger than L2: {ROTATE} rotating stream+output copies "
                                    f"({ROTATE * (in_bytes + out_bytes) / 1e6:.0f} MB)",
                       actual_bpp=round(info.actual_bpp, 4), n_tiles=info.n_tiles,
                       blocks_per_lane=info.blocks_per_lane, parallelism="replicas" if world > 1 else "single"),
        "gweights_per_s": round(world * n_weights / step_s / 1e9, 3),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic, "peak_kind": peak_kind,
                     "algorithmic_bytes_per_launch": in_bytes + out_bytes,
                     "kernel_us": round(kernel_s * 1e6, 3)},
        "e2e": {"value": round(e2e_value, 3), "unit": "GB/s", "h2d_bytes_per_step": in_bytes,
                "d2h_bytes_per_step": out_bytes},
        "gpu_launches": steps,
        "tables": {"prepare_us": round(prepare_us, 3), "note": "slot tables built once per device copy of "
                   "the stream (ep_prepare); each step stages them into shared memory and decodes"},
        "clocks": clk.summary(),
        "encode_s": round(t_enc, 3),
    }
    if world == 1 and not a.no_cpu_baseline:
        n, el, _ = cpu_oracle_decode(blob_cpu.numpy(), a.cpu_seconds)
        line["cpu_baseline"] = {"value": round(out_bytes * n / el / 1e9, 4), "unit": "GB/s", "cores": 1,
                                "kind": "oracle",
                                "sample": f"{n} full decodes of the 4096x4096 stream by the C oracle ({el:.1f} s)"}
    print(json.dumps(line), flush=True)


def main():
    a = args_()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if a.impl == "reference":
        run_reference(a, rank, world)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_ours(a, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
