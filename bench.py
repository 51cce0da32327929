"""Benchmark of the fused lattice-rANS decode (ep_decompress) on B200.

One step = one ep_decompress call over the whole workload matrix: every tile's rANS streams
decoded to fields, lattice points, row-scaled and written as BF16.  Default workload: 4096 x 4096
BF16, rows N(0, sigma_r^2) with sigma_r log-uniform in [0.005, 0.05], compressed at 4.0 bits per
element by the library's own encoder (synthetic data; no model weights are involved).

Timing: W untimed warm-up steps, then exactly K steps between a barrier + synchronize on both
sides, timed by CUDA events on the launching stream; the maximum over ranks is reported.  The K
launches are queued behind a short device-side delay recorded before the start event, so the
timed region holds K back-to-back decodes and no host launch cost.  The steps rotate over R
independent blob/output copies whose total exceeds 3x the 126 MB L2, so each step reads its blob
and writes its output through HBM.  nvidia-smi samples clocks and throttle reasons from the
warm-up through the timed region.

Multi-GPU (torchrun): every rank decodes its own copy of the workload; no data-path collective
(tiles are independent), so scaling is weak and the value is the sum over ranks.

Arms:
  default             the CUDA path through the C ABI;
  --impl reference    the oracle (plain single-threaded C) on the host cores, each step a
                      bounded sample of the same workload; rank 0 only.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decompressed output GB/s and % of HBM roofline (fused rANS+E8 decode), 1×B200"
NOMINAL_HBM_GBS = 8000.0          # the roofline the metric names
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--steps-per-tile", type=int, default=0, help="encoder S override (0 = default)")
    ap.add_argument("--prob-bits", type=int, default=12, choices=[10, 12],
                    help="frequency totals 2^prob_bits: 12 (the format's choice) or 10")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="CPU-baseline sample length")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-cores", type=int, default=0,
                    help="also time the oracle tile-parallel on this many host cores (0 = all, 1 = skip)")
    ap.add_argument("--workload", default="square",
                    help="square (default) | small | dit-set | sweep:<bpp> | large")
    ap.add_argument("--out-dtype", default="",
                    help="output container(s), comma-separated, decoded back to back every step: "
                         "bf16, fp16, e4m3, f32, int8 (default: the input's)")
    ap.add_argument("--decode", choices=["grouped", "single"], default="grouped",
                    help="for a set of matrices: one ep_decompress_group call per step, or one "
                         "ep_decompress call per matrix")
    ap.add_argument("--matrices", type=int, default=0,
                    help="for a set of matrices: use only the first K (0 = all), e.g. to keep a profiled "
                         "case to a few GB on the device")
    return ap.parse_args()


def workload(name: str = "square"):
    """The matrices one step decodes, and a description."""
    import workloads as W
    if name == "square":
        return [W.square()], ("square 4096x4096 BF16, row r i.i.d. N(0, sigma_r^2), sigma_r log-uniform in "
                              "[0.005, 0.05], target 4.0 bpp, output BF16")
    if name == "small":
        return [W.small()], "small 256x256 BF16 N(0, 0.02^2), target 3.5 bpp, output BF16"
    if name == "dit-set":
        return ([W.dit(j) for j in range(len(W.DIT_SHAPES))],
                "dit-set: a DiT block's linear layers (4 x 3072x3072, 3072x8192, 8192x3072) BF16, Student-t(5) "
                "x 0.02/sqrt(5/3) with 1% of rows x10, target 2.5 bpp, output BF16")
    if name.startswith("sweep:"):
        rate = float(name.split(":", 1)[1])
        return [W.sweep(rate)], f"sweep 4096x11008 FP16 N(0, 0.02^2), target {rate} bpp, output FP16"
    if name == "large":
        return ([W.large(j) for j in range(4)],
                "large: 4 x 28672x8192 BF16, N(0, 0.015^2) x per-column scale log-uniform in [0.5, 2], "
                "target 4.0 bpp, output BF16")
    raise SystemExit(f"unknown workload {name!r}")


# ---------------------------------------------------------------------------------------------
# Clocks during the timed region.
# ---------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.proc = None
        self.path = None
        self.gpu_id = gpu_id

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50"]
            if self.gpu_id:
                cmd += ["-i", self.gpu_id]
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        # nvidia-smi takes a moment to start: wait for its first sample (up to 5 s), so that even a
        # short timed region lies inside the sampled interval
        t0 = time.time()
        while time.time() - t0 < 5.0 and self.proc.poll() is None:
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.02)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.12)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------------------------
# Peaks and the committed ncu traffic figure.
# ---------------------------------------------------------------------------------------------
def hbm_peak():
    try:
        d = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        return float(d["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


KERNEL_SOURCES = ("decode_device.cuh", "decode_launch.h", "format.h")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "decode_traffic.json")


def kernel_source_hash() -> str:
    """Hash of the decode kernel's code (comments and blank space removed): a DRAM traffic figure
    is valid only for this code, and an edit to a comment does not change the kernel."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        text = open(os.path.join(ROOT, "dit_weight_compression_b200", "csrc", f), encoding="utf-8").read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def measured_traffic(key: str):
    """DRAM bytes (read + write) per decode launch from the ncu capture of consecutive launches
    summarised in profiles/decode_traffic.json, if it was taken on this kernel source; else None."""
    try:
        d = json.load(open(TRAFFIC_FILE))
    except (OSError, ValueError):
        return None
    if d.get("kernel_source_sha") != kernel_source_hash():
        return None
    w = d.get("workloads", {}).get(key)
    if not w:
        return None
    return int(w["dram_bytes_read_per_launch"]) + int(w["dram_bytes_write_per_launch"])


# ---------------------------------------------------------------------------------------------
# Multi-rank plumbing: the job's time is the slowest rank's; the value counts every rank's units.
# ---------------------------------------------------------------------------------------------
def max_over_ranks(values, world: int, device: str = "cuda"):
    """Elementwise maximum of a list of floats over all ranks (identity for one rank)."""
    if world <= 1:
        return list(values)
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_throughput(world: int, bytes_per_step_per_rank: float, steps: int, max_ms: float) -> float:
    """Whole-job GB/s: every rank's bytes over the slowest rank's time."""
    return world * bytes_per_step_per_rank * steps / (max_ms * 1e-3) / 1e9


# ---------------------------------------------------------------------------------------------
# CPU baseline: the oracle decoder on the host.
# ---------------------------------------------------------------------------------------------
def cpu_oracle_rate(blob: bytes, seconds: float, max_tiles: int | None = None):
    import oracle
    info = oracle.blob_info(blob)
    out = np.zeros((info["rows"], info["cols"]), np.uint16)
    n_tiles = info["n_tiles"] if max_tiles is None else min(max_tiles, info["n_tiles"])
    per = 32 * info["S"]
    elems = min(n_tiles * per, info["V"]) * 8
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle.decompress_tiles(blob, 0, n_tiles, oracle.BF16, out)
        reps += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    return elems * 2 * reps / dt / 1e9, reps, n_tiles, dt


_POOL_BLOB = None


def _pool_init(blob: bytes):
    global _POOL_BLOB
    _POOL_BLOB = blob


def _pool_decode(job):
    """One worker's share: decode tiles [t0, t1) repeatedly for about `seconds`."""
    import oracle
    t0, t1, seconds = job
    info = oracle.blob_info(_POOL_BLOB)
    out = np.zeros((info["rows"], info["cols"]), np.uint16)
    per = 32 * info["S"]
    elems = (min(t1 * per, info["V"]) - t0 * per) * 8
    start = time.perf_counter()
    reps = 0
    while True:
        oracle.decompress_tiles(_POOL_BLOB, t0, t1, oracle.BF16, out)
        reps += 1
        if time.perf_counter() - start >= seconds:
            break
    return elems * reps, time.perf_counter() - start


def cpu_oracle_rate_parallel(blob: bytes, seconds: float, cores: int):
    """The same oracle decode, tile-parallel: `cores` processes (spawned, so no CUDA state is
    inherited), each on a contiguous tile range.  GB/s of output over the slowest worker."""
    import multiprocessing as mp
    import oracle
    info = oracle.blob_info(blob)
    n = info["n_tiles"]
    cores = max(1, min(cores, n))
    bounds = [n * i // cores for i in range(cores + 1)]
    jobs = [(bounds[i], bounds[i + 1], seconds) for i in range(cores)]
    with mp.get_context("spawn").Pool(cores, initializer=_pool_init, initargs=(blob,)) as pool:
        res = pool.map(_pool_decode, jobs)
    elems = sum(r[0] for r in res)
    dt = max(r[1] for r in res)
    return elems * 2 / dt / 1e9, cores, dt


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def reference_arm(args, m, desc):
    """The oracle as it stands, timed on the host cores with the same metric and workload."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    blob = oracle.compress(m.bits, m.dtype, m.target_bpp, prob_bits=args.prob_bits)
    info = oracle.blob_info(blob)
    # size each step's sample so that warm-up + steps take about a minute
    t = time.perf_counter()
    oracle.decompress_tiles(blob, 0, 8, oracle.BF16, np.zeros((info["rows"], info["cols"]), np.uint16))
    per_tile = max((time.perf_counter() - t) / 8, 1e-6)
    tiles = int(max(1, min(info["n_tiles"], 60.0 / (args.steps + args.warmup) / per_tile)))
    out = np.zeros((info["rows"], info["cols"]), np.uint16)
    for i in range(args.warmup):
        oracle.decompress_tiles(blob, 0, tiles, oracle.BF16, out)
    t0 = time.perf_counter()
    for i in range(args.steps):
        t_lo = (i * tiles) % max(1, info["n_tiles"] - tiles + 1)
        oracle.decompress_tiles(blob, t_lo, t_lo + tiles, oracle.BF16, out)
    dt = time.perf_counter() - t0
    elems = tiles * 32 * info["S"] * 8
    value = elems * 2 * args.steps / dt / 1e9
    sample = f"{tiles} of {info['n_tiles']} tiles ({elems} elements) per step"
    line = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "u32/f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": desc, "rows": m.shape[0], "cols": m.shape[1], "target_bpp": m.target_bpp,
                       "actual_bpp": oracle.actual_bpp(blob), "sample": sample},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------------------------
# The CUDA arm.
# ---------------------------------------------------------------------------------------------
OUT_DTYPES = {"bf16": "bfloat16", "fp16": "float16", "e4m3": "float8_e4m3fn", "f32": "float32",
              "int8": "int8", "e4m3row": "float8_e4m3fn"}


def out_containers(arg: str, default):
    """The containers each step decodes into, in order (the input's own by default), as
    (name, torch dtype, row-scaled FP8?)."""
    import torch
    if not arg:
        return [(str(default).replace("torch.", ""), default, False)]
    out = []
    for name in arg.split(","):
        name = name.strip().lower()
        if name not in OUT_DTYPES:
            raise SystemExit(f"unknown output container {name!r} (one of {', '.join(OUT_DTYPES)})")
        out.append((name if name == "e4m3row" else OUT_DTYPES[name], getattr(torch, OUT_DTYPES[name]),
                    name == "e4m3row"))
    return out


def queue_delay_cycles(launches: int) -> int:
    """Length of the device-side delay queued before the timed region: long enough for the host
    to enqueue the first launches behind it (about 10 us each through ctypes), so host launch
    cost and idle gaps stay out of the timed region."""
    return int(max(1e-3, min(launches, 2048) * 10e-6) * 2.0e9)


def main():
    args = parse_args()
    mats, desc = workload(args.workload)
    subset = ""
    if 0 < args.matrices < len(mats):
        subset = f"; the first {args.matrices} of its {len(mats)} matrices"
        mats = mats[:args.matrices]
    if args.impl == "reference":
        reference_arm(args, mats[0], desc + subset)
        return

    import torch
    import torch.distributed as dist

    import dit_weight_compression_b200 as ep
    import workloads as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    # compress with the library's host encoder
    cfg = ep.LatticeRANSConfig(mats[0].target_bpp, steps_per_tile=args.steps_per_tile, prob_bits=args.prob_bits)
    t = time.perf_counter()
    comps = [ep.compress(W.bits_to_torch(m.bits, m.dtype), cfg) for m in mats]
    enc_s = time.perf_counter() - t
    blobs = [c.to_bytes() for c in comps]
    # the same matrices encoded on the GPU from device tensors (byte-identical blobs)
    dev_in = [W.bits_to_torch(m.bits, m.dtype).cuda() for m in mats]
    ep.compress(dev_in[0], cfg)  # first use: context and kernel set-up
    torch.cuda.synchronize()
    t = time.perf_counter()
    gcomps = [ep.compress(x, cfg) for x in dev_in]
    enc_gpu_s = time.perf_counter() - t
    if [g.to_bytes() for g in gcomps] != blobs:
        raise SystemExit("GPU encoder blob differs from the host encoder's")
    del gcomps, dev_in
    n = len(comps)
    out_dts = out_containers(args.out_dtype, comps[0].dtype)
    nd = len(out_dts)
    out_bytes = sum(c.shape[0] * c.shape[1] * torch.empty((), dtype=dt).element_size() + (4 * c.shape[0] if rs else 0)
                    for c in comps for _, dt, rs in out_dts)
    blob_bytes = sum(len(b) for b in blobs)
    moved = nd * blob_bytes + out_bytes          # every decode reads its blob once
    grouped = n > 1 and args.decode == "grouped" and not any(rs for _, _, rs in out_dts)

    # R independent device copies of the whole set so that consecutive steps miss L2
    R = max(2, math.ceil(3 * L2_BYTES / moved))
    stream = torch.cuda.current_stream()
    copies = [[ep.CompressedTensor.from_bytes(b) for b in blobs] for _ in range(R)]
    outs = [[[torch.empty(c.shape, dtype=dt, device="cuda") for c in comps] for _, dt, _ in out_dts] for _ in range(R)]
    sigmas = [[torch.empty(c.shape[0], dtype=torch.float32, device="cuda") for c in comps] for _ in range(R)]
    for cs in copies:
        for c in cs:
            c.prepare(stream=stream)
    L = ep.lib()
    views = [[[ep.tensor_view(o) for o in od] for od in os_] for os_ in outs]
    handles = [[c.handle for c in cs] for cs in copies]
    g_handles = [(ctypes.c_void_p * n)(*[h.value for h in hs]) for hs in handles]
    g_views = [[(ep.EpTensor * n)(*vs) for vs in vd] for vd in views]
    sh = ctypes.c_void_p(stream.cuda_stream)
    launches_per_step = nd * (math.ceil(n / 28) if grouped else n)
    sig_ptrs = [[ctypes.c_void_p(t.data_ptr()) for t in ts] for ts in sigmas]

    def step(i):
        j = i % R
        for d in range(nd):
            if grouped:
                rc = L.ep_decompress_group(g_handles[j], g_views[j][d], n, sh)
                if rc != 0:
                    raise ep.EPError(rc, "ep_decompress_group")
                continue
            rowscaled = out_dts[d][2]
            for b, (h, v) in enumerate(zip(handles[j], views[j][d])):
                if rowscaled:
                    rc = L.ep_decompress_fp8_rowscaled(h, ctypes.byref(v), sig_ptrs[j][b], sh)
                else:
                    rc = L.ep_decompress(h, ctypes.byref(v), sh)
                if rc != 0:
                    raise ep.EPError(rc, "decode")

    # a first step, checked by the kernels' own integrity checks
    step(0)
    torch.cuda.synchronize()
    for c in copies[0]:
        ep.decode_status(c)

    gpu_uuid = None
    try:
        gpu_uuid = str(torch.cuda.get_device_properties(local).uuid)
        if not gpu_uuid.startswith("GPU-"):
            gpu_uuid = "GPU-" + gpu_uuid
    except Exception:
        gpu_uuid = None
    clocks = ClockSampler(gpu_uuid)
    clocks.start()  # samples warm-up and timed region alike: the GPU is never idle in between
    for i in range(args.warmup):
        step(i)
    K = args.steps
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    # The K launches queue up behind a device-side delay recorded before the start event, so the
    # timed region holds exactly K back-to-back decodes (each may overlap the previous one's drain,
    # see the kernel) and neither host launch cost nor a gap after the barrier.
    torch.cuda._sleep(queue_delay_cycles(K * launches_per_step))
    start.record(stream)
    for i in range(K):
        step(args.warmup + i)
    end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier()
    torch.cuda.synchronize()
    total_ms = start.elapsed_time(end)
    avg_step_ms = total_ms / K
    for cs in copies:
        for c in cs:
            ep.decode_status(c)

    total_ms, avg_step_ms = max_over_ranks([total_ms, avg_step_ms], world)

    # end to end through the public call with host buffers: upload each blob, decode, download
    host_outs = [[torch.empty(c.shape, dtype=dt).pin_memory() for c in comps] for _, dt, _ in out_dts]
    host_sig = [torch.empty(c.shape[0], dtype=torch.float32).pin_memory() for c in comps]

    def e2e_step():
        for (_, _, rowscaled), ho in zip(out_dts, host_outs):
            for c, o, hs in zip(comps, ho, host_sig):
                if rowscaled:
                    ep.decompress_fp8_rowscaled(c, out=o, row_scale=hs)
                else:
                    ep.decompress(c, out=o)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    e_s, e_e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_s.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    e_e.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e_s.elapsed_time(e_e)
    (e2e_ms,) = max_over_ranks([e2e_ms], world)
    for c in comps:
        ep.decode_status(c)

    if rank == 0:
        peak, peak_kind = hbm_peak()
        achieved = moved / (avg_step_ms * 1e-3) / 1e9   # algorithmic bytes over the step's device time
        value = job_throughput(world, out_bytes, K, total_ms)
        symbols = nd * sum(c.info.n_vectors for c in comps) * 8   # a vector is 8 rANS symbols
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            gbs, reps, nt, secs = cpu_oracle_rate(blobs[0], args.cpu_seconds)
            r0, c0 = comps[0].shape
            what = "matrix" if n == 1 else f"first matrix of the {n}"
            cpu = {"value": gbs, "unit": "GB/s", "cores": 1, "kind": "oracle",
                   "sample": f"whole {r0}x{c0} {what} ({nt} tiles) decoded {reps} times, {secs:.1f} s, "
                             f"single-threaded oracle, BF16 output"}
            if args.cpu_cores != 1:
                want = host_cores() if args.cpu_cores <= 0 else args.cpu_cores
                pg, used, psecs = cpu_oracle_rate_parallel(blobs[0], args.cpu_seconds, want)
                cpu["all_cores"] = {"value": pg, "unit": "GB/s", "cores": used, "kind": "oracle",
                                    "sample": f"the same {what}, tile-parallel over {used} processes, "
                                              f"{psecs:.1f} s"}
        traffic = None
        if launches_per_step == 1:
            traffic = measured_traffic(f"{args.workload}:{out_dts[0][0]}:pb{args.prob_bits}")
        info = comps[0].info
        dt_names = [name for name, _, _ in out_dts]
        config = {
            "workload": (desc if not args.out_dtype else f"{desc.rsplit(', output', 1)[0]}, output "
                                                         f"{' then '.join(dt_names)}") + subset,
            "matrices": n,
            "shapes": [list(c.shape) for c in comps],
            "target_bpp": mats[0].target_bpp,
            "prob_bits": args.prob_bits,
            "actual_bpp": 8.0 * blob_bytes / sum(c.shape[0] * c.shape[1] for c in comps),
            "steps_per_tile": sorted({c.info.steps_per_tile for c in comps}),
            "n_tiles": sum(c.info.n_tiles for c in comps), "blob_bytes": blob_bytes, "out_bytes": out_bytes,
            "out_containers": dt_names,
            "l2": f"rotating {R} blob/output copies ({R * moved / 1e6:.0f} MB > 3x L2)",
            "rans_symbols_per_s": world * symbols * K / (total_ms * 1e-3),
            "step_avg_us": avg_step_ms * 1e3, "encode_s": enc_s, "encode_gpu_s": enc_gpu_s,
            "decode": ("ep_decompress_group, one launch per container per step" if grouped else
                       f"ep_decompress, {launches_per_step} launch(es) per step"),
            "timing": "K launches queued behind a device-side delay; CUDA events around exactly K steps",
            "parallelism": f"weak, {world} independent rank(s)",
        }
        if n == 1 and nd == 1:
            config.update(rows=info.rows, cols=info.cols, kernel_avg_us=avg_step_ms * 1e3)
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": total_ms / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "u32/f32", "data": "synthetic",
            "config": config,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "peak_kind": peak_kind, "nominal_8tbs_frac": achieved / NOMINAL_HBM_GBS,
                         "algorithmic_bytes_per_launch" if launches_per_step == 1 else "algorithmic_bytes_per_step": moved},
            "cpu_baseline": cpu,
            "e2e": {"value": job_throughput(world, out_bytes, args.e2e_steps, e2e_ms), "unit": "GB/s",
                    "h2d_bytes_per_step": nd * blob_bytes, "d2h_bytes_per_step": out_bytes},
            "gpu_launches": K * launches_per_step,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    del copies
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
