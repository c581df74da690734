"""Benchmark of the PACK3D attention forward on B200 (one process per GPU).

A step is one pass of the operator's hot path over one batch of synthetic input: block
summaries with the rotated keys written in the same pass (pack3d_summarize_rotated), the local
branch on those keys (pack3d_attn_local with PACK3D_K_ROTATED), then the global branch with the
mixer (pack3d_attn_global) -- the two halves of pack3d_attn_fwd, called separately so that each
kernel is timed with CUDA events on the stream it runs on -- the index of
the packed field is built once per geometry before timing, as it is amortised over layers,
heads and batches. Default workload: the 65,536-token field (32x32x64 grid, batch 2, 8 heads,
head_dim 96, bf16, 4x4x4 blocks -> 1,024 summaries, raster-block packing).

The line's `roofline` is the whole step's: the slower of the step's algorithmic bytes at the
measured HBM peak and its global-contraction flops at the measured bf16 peak, against the step
time; the per-kernel rooflines sit under `kernels` (and the slowest under
`roofline.dominant_kernel`). On one GPU the same run also reports the forward + backward of
the headline field (`fwd_bwd`, `attn_bwd`), the 262,144-token field (`field262k_bf16`) and the
pages' 1M-token point (`field1m_bf16`: 64x128x128, 4,096 summaries after a second pooling
stage).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl pack3d|reference]

With N > 1 the script is launched by torch.distributed.run, one rank per GPU; every rank runs
its own batch (weak scaling, no data-path collective) and rank 0 prints one JSON line.
``--impl reference`` times the float64 CPU oracle on the host cores instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import inputs  # noqa: E402

METRIC = "PACK3D attn fwd tokens/s at 65,536 tokens bf16 (1×B200) + % of roofline"
UNIT = "tokens/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="pack3d", choices=["pack3d", "reference"])
    ap.add_argument("--workload", default="field65k_bf16", choices=sorted(inputs.WORKLOADS))
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--skip-bwd", action="store_true",
                    help="skip the (untimed-step) backward and index-build measurements")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (smaller cases for profiler captures)")
    return ap.parse_args()


def workload_config(name, w):
    return {"workload": name, "grid": list(w["grid"]), "block": list(w["block"]),
            "batch": w["batch"], "heads": w["heads"], "head_dim": w["d"],
            "tokens": int(np.prod(w["grid"])), "summaries": _sizes(w)[3],
            "pool2": list(w.get("pool2", (1, 1, 1))),
            "packing": w["packing"], "exclude_near": w["exclude_near"],
            "l2": "inputs larger than L2: q, k, v alone are "
                  f"{3 * w['batch'] * w['heads'] * int(np.prod(w['grid'])) * w['d'] * 2 / 1e6:.0f}"
                  " MB per step"}


# ------------------------------------------------------------------------------ clocks
class ClockSampler:
    """SM clock, power and clock-event reasons of one GPU while the timed region runs: NVML
    polled every 2 ms from a thread (read-only queries), or nvidia-smi at 100 ms when NVML is
    not available."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap"}

    def __init__(self, device_index):
        self.idx = device_index
        self.proc = None
        self.path = None
        self.thread = None
        self.rows = []
        self.source = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            uuid = str(torch.cuda.get_device_properties(self.idx).uuid)
            return pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(self.idx)

    def start(self):
        try:
            import threading

            import pynvml
            h = self._nvml_handle()
            smax = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            self.stop_flag = threading.Event()

            def poll():
                while not self.stop_flag.is_set():
                    try:
                        self.rows.append(dict(
                            sm=float(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)),
                            smax=smax,
                            power=pynvml.nvmlDeviceGetPowerUsage(h) / 1000.0,
                            bits=int(pynvml.nvmlDeviceGetCurrentClocksEventReasons(h))))
                    except Exception:
                        break
                    time.sleep(0.002)

            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            # the sampler is live before the caller's timed region starts (up to 1 s)
            t_end = time.time() + 1.0
            while not self.rows and time.time() < t_end and self.thread.is_alive():
                time.sleep(0.001)
            self.source = "nvml, 2 ms"
            return
        except Exception:
            self.thread = None
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
            self.source = "nvidia-smi, 100 ms"
        except Exception:
            self.proc = None

    def stop(self):
        rows = []
        if self.thread is not None:
            self.stop_flag.set()
            self.thread.join(timeout=5)
            for r in self.rows:
                rows.append(dict(sm=r["sm"], smax=r["smax"], power=r["power"],
                                 reasons={n for bit, n in self.REASONS.items() if r["bits"] & bit}))
        elif self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 8:
                    continue
                try:
                    rows.append(dict(sm=float(parts[0]), smax=float(parts[1]),
                                     power=float(parts[2]) if parts[2] not in ("[N/A]", "") else 0.0,
                                     reasons={n for n, v in zip(names, parts[4:8])
                                              if v.lower() == "active"}))
                except ValueError:
                    continue
            os.unlink(self.path)
        if not rows:
            return None
        load = [r for r in rows if r["power"] > 0.25 * max(x["power"] for x in rows)] or rows
        reasons = set()
        for r in rows:
            reasons |= r["reasons"]
        return {"sm_mhz": statistics.median(r["sm"] for r in load),
                "sm_max_mhz": max(r["smax"] for r in rows), "reasons": sorted(reasons),
                "samples": len(rows), "source": self.source}


# ---------------------------------------------------------------------------- roofline
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d["bf16_tflops_sustained"],
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, source="fallback")


def kernel_traffic(kernel_key):
    """DRAM bytes per launch from a committed ncu summary, if the kernel source is unchanged."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(kernel_key)
    if not d:
        return None
    h = hashlib.sha256()
    for f in d["sources"]:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    if h.hexdigest() != d["sources_sha256"]:
        return None
    return d["bytes_per_launch_full"]


def _sizes(w):
    """B, H, N, M, d of a workload (M: the summaries the global branch attends to, after the
    second pooling stage when there is one)."""
    B, H, d = w["batch"], w["heads"], w["d"]
    N = int(np.prod(w["grid"]))
    pool2 = w.get("pool2", (1, 1, 1))
    M = int(np.prod([-(-(-(-g // b)) // p) for g, b, p in zip(w["grid"], w["block"], pool2)]))
    return B, H, N, M, d


def algorithmic(w):
    """Per-launch algorithmic work of the three kernels of a step (each row read or written
    once; index tables read once)."""
    B, H, N, M, d = _sizes(w)
    el = 2  # bf16
    e = B * H * N * d * el  # bytes of one [B, H, N, d] tensor
    return {
        # k, v read; summary tiles and the rotated keys written; members + coords read
        "summarize": {"bytes": 3 * e + 2 * B * H * M * d * el + N * 4 * 2},
        # q, rotated k, v read; o_loc written; inverse map read
        "local": {"bytes": 4 * e + N * 4},
        # the global contraction: 2 N M d (QK) + 2 N M d (PV) per (batch, head)
        "global": {"flops": 4.0 * N * M * d * B * H,
                   "bytes": 3 * e + B * H * N * el + 2 * B * H * M * d * el},
    }


def step_algorithmic(w, index_bytes):
    """Algorithmic work of one forward step whatever the kernel split: q, k, v read and o
    written once, the gate logits read, the summaries written and read back once, the index
    tables read once; the global contraction's 4 N M d flops per (batch, head)."""
    B, H, N, M, d = _sizes(w)
    el = 2
    e = B * H * N * d * el
    summ = B * H * M * d * el
    return {"bytes": 4 * e + B * H * N * el + 2 * 2 * summ + index_bytes,
            "flops": 4.0 * N * M * d * B * H}


def step_roofline(alg, ms, peaks):
    """Roofline of a whole step: the slower of its bytes at the HBM peak and its flops at the
    bf16 tensor peak, against the measured step time."""
    t_hbm = alg["bytes"] / (peaks["hbm"] * 1e9)
    t_mma = alg["flops"] / (peaks["bf16"] * 1e12)
    sec = ms / 1e3
    if t_mma >= t_hbm:
        ach = alg["flops"] / sec / 1e12
        return {"bound": "tensor", "achieved": ach, "peak": peaks["bf16"], "unit": "TFLOP/s",
                "frac": ach / peaks["bf16"], "roofline_ms": t_mma * 1e3,
                "algorithmic_flops_per_step": alg["flops"],
                "algorithmic_bytes_per_step": alg["bytes"],
                "peak_source": f"{peaks['source']} bf16 dense burst"}
    ach = alg["bytes"] / sec / 1e9
    return {"bound": "hbm", "achieved": ach, "peak": peaks["hbm"], "unit": "GB/s",
            "frac": ach / peaks["hbm"], "roofline_ms": t_hbm * 1e3,
            "algorithmic_flops_per_step": alg["flops"], "algorithmic_bytes_per_step": alg["bytes"],
            "peak_source": f"{peaks['source']} HBM copy"}


# -------------------------------------------------------------------------------- oracle
def oracle_sample(w, idx, head=(0, 0)):
    """Time the float64 oracle on one (batch, head) of the workload: summaries + all rows.
    Returns (wall seconds, process CPU seconds)."""
    from oracle import pack3d_oracle as orc
    b, h = head
    sl = lambda t: t[b:b + 1, h:h + 1].numpy()  # noqa: E731
    q, k, v, a = sl(w["q"]), sl(w["k"]), sl(w["v"]), sl(w["a"])
    c0, t0 = time.process_time(), time.perf_counter()
    orc.forward(q, k, v, a, w["coords"], w["grid"], w["block"], exclude_near=w["exclude_near"],
                index=idx)
    return time.perf_counter() - t0, time.process_time() - c0


def cores_used(wall, cpu):
    """Threads the oracle actually kept busy: process CPU time over wall time (at least 1)."""
    return max(1, int(round(cpu / wall))) if wall > 0 else 1


def cpu_baseline(w, reps=3):
    from oracle import pack3d_oracle as orc
    idx = orc.build_index(w["coords"], w["grid"], w["block"])
    runs = [oracle_sample(w, idx) for _ in range(reps)]
    t = statistics.median(r[0] for r in runs)
    cores = cores_used(sum(r[0] for r in runs), sum(r[1] for r in runs))
    B, H, N, _, _ = _sizes(w)
    # one head of one batch element is 1/(B*H) of a step
    value = (B * N) / (t * B * H)
    return {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"float64 numpy oracle on 1 of {B * H} (batch, head) pairs of the workload "
                      f"(summaries + local + global + mixer for all {N} tokens), median of "
                      f"{reps} runs ({t:.2f} s), scaled by {B * H}; cores = process CPU time / "
                      f"wall time"}


def run_reference(args, rank):
    if rank != 0:
        return
    w = inputs.make_workload(args.workload)
    from oracle import pack3d_oracle as orc
    idx = orc.build_index(w["coords"], w["grid"], w["block"])
    for _ in range(args.warmup):
        oracle_sample(w, idx)
    runs = [oracle_sample(w, idx, head=(s % w["batch"], s % w["heads"]))
            for s in range(args.steps)]
    B, H, N, _, _ = _sizes(w)
    # a step is the oracle on one (batch, head): N tokens of one head = N / H token-equivalents
    # of the metric (a token of the metric carries all H heads)
    step = float(np.mean([r[0] for r in runs]))
    value = (N / H) / step
    cores = cores_used(sum(r[0] for r in runs), sum(r[1] for r in runs))
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference", "config": workload_config(args.workload, w),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"each timed step: the float64 oracle on one (batch, head) "
                                       f"of {B * H}, all {N} tokens (= {N // H} tokens of all "
                                       f"{H} heads); cores = process CPU time / wall time"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------ multi-rank
def max_over_ranks(values, dist=None, device=None):
    """Element-wise max of per-rank timings (ms) over every rank of the default process group
    (identity on one rank): the job is as slow as its slowest rank."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return [float(x) for x in values]
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_throughput(world, tokens_per_rank, ms):
    """Whole-job tokens/s when each of `world` ranks processes `tokens_per_rank` tokens per step
    and a step takes `ms` (the max over ranks)."""
    return world * tokens_per_rank / (ms / 1e3)


# ------------------------------------------------------------------------------- GPU arm
def device_workload(name, dev):
    """A named workload with its q, k, v, a drawn on the device (N(0, sigma^2) and N(0, 1) from
    a seeded CUDA generator, rounded to bf16, in memory order): the large fields of the extra
    measurements, whose CPU generation would take longer than their timing. The packing and
    coordinates come from the same host generator as every other workload."""
    cfg = dict(inputs.WORKLOADS[name])
    grid, block = tuple(cfg["grid"]), tuple(cfg["block"])
    perm = inputs.packing(cfg["packing"], grid, block)
    B, H, N, d = cfg["batch"], cfg["heads"], int(np.prod(grid)), cfg["d"]
    g = torch.Generator(device=dev).manual_seed(0)
    shape = (B, H, N, d)
    out = dict(cfg)
    out.update(perm=perm, coords=inputs.coords_of(perm, grid))
    for n in "qkv":
        out[n] = (torch.randn(shape, generator=g, device=dev) * cfg["qkv_std"]).to(torch.bfloat16)
    out["a"] = torch.randn(shape[:3], generator=g, device=dev).to(torch.bfloat16)
    return out


class Forward:
    """The timed forward step of one workload on one device: summaries + rotated keys, local
    branch, global branch + mixer, each call's kernel timed with CUDA events on its stream."""

    def __init__(self, p3d, w, dev):
        self.p3d, self.w = p3d, w
        B, H, d = w["batch"], w["heads"], w["d"]
        dt = torch.bfloat16
        self.geom = p3d.make_geom(w["grid"], w["block"], d, pool2=w.get("pool2", (1, 1, 1)))
        self.ix = p3d.pack3d_build_index(self.geom, coords=torch.from_numpy(w["coords"]).to(dev))
        self.q, self.k, self.v, self.a = (w[n].to(dt).to(dev).contiguous() for n in "qkva")
        self.ksum = torch.empty(p3d.summary_tiles_shape(self.ix, B, H, d), dtype=dt, device=dev)
        self.vsum = torch.empty_like(self.ksum)
        self.k_rot = torch.empty_like(self.k)
        self.o = torch.empty_like(self.q)
        self.stream = torch.cuda.current_stream()

    def step(self, ev=None):
        p3d, st = self.p3d, self.stream
        if ev is not None:
            ev[0].record(st)
        p3d.pack3d_summarize_rotated(self.ix, self.k, self.v, self.ksum, self.vsum, self.k_rot)
        n = p3d.pack3d_last_launch_count()
        if ev is not None:
            ev[1].record(st)
        p3d.pack3d_attn_local(self.ix, self.q, self.k_rot, self.v, k_rotated=True, o_loc=self.o)
        n += p3d.pack3d_last_launch_count()
        if ev is not None:
            ev[2].record(st)
        p3d.pack3d_attn_global(self.ix, self.q, self.a, self.ksum, self.vsum, self.o,
                               exclude_near=self.w["exclude_near"], o=self.o)
        n += p3d.pack3d_last_launch_count()
        if ev is not None:
            ev[3].record(st)
        return n

    def time(self, steps, warmup, sync=None):
        for _ in range(max(warmup, 0)):
            self.step()
        torch.cuda.synchronize()
        if sync:
            sync()
        torch.cuda.synchronize()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        launches = 0
        t0.record(self.stream)
        for s in range(steps):
            launches += self.step(evs[s])
        t1.record(self.stream)
        torch.cuda.synchronize()
        if sync:
            sync()
        torch.cuda.synchronize()
        ms = t0.elapsed_time(t1) / steps
        ms_k = {name: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in evs)
                for i, name in enumerate(("summarize", "local", "global"))}
        return ms, ms_k, launches

    def index_bytes(self):
        return self.p3d.pack3d_index_bytes(self.geom, int(np.prod(self.w["grid"])))


KERNEL_NAMES = {"summarize": "k_summarize (pack3d_summarize_rotated)",
                "local": "k_local_tma (pack3d_attn_local)",
                "global": "k_global_tc (pack3d_attn_global)"}


def kernel_rooflines(w, ms_k, peaks, workload):
    alg = algorithmic(w)
    kernels = {}
    for name in ("summarize", "local", "global"):
        sec = ms_k[name] / 1e3
        if "flops" in alg[name]:
            ach = alg[name]["flops"] / sec / 1e12
            ent = {"bound": "tensor", "achieved": ach, "peak": peaks["bf16"], "unit": "TFLOP/s",
                   "frac": ach / peaks["bf16"],
                   "algorithmic_flops_per_launch": alg[name]["flops"],
                   "peak_source": f"{peaks['source']} bf16 dense burst"}
        else:
            ach = alg[name]["bytes"] / sec / 1e9
            ent = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm"], "unit": "GB/s",
                   "frac": ach / peaks["hbm"], "peak_source": f"{peaks['source']} HBM copy"}
        ent.update({"kernel": KERNEL_NAMES[name], "ms_per_launch": ms_k[name],
                    "algorithmic_bytes_per_launch": alg[name]["bytes"],
                    "traffic": kernel_traffic(f"{name}_{workload}")})
        kernels[name] = ent
    return kernels


def forward_line(w, workload, ms, ms_k, index_bytes, peaks):
    """Step-level roofline (the headline) plus the per-kernel rooflines."""
    kernels = kernel_rooflines(w, ms_k, peaks, workload)
    roof = step_roofline(step_algorithmic(w, index_bytes), ms, peaks)
    tr = [kernels[n]["traffic"] for n in kernels]
    roof["traffic"] = float(sum(tr)) if all(t is not None for t in tr) else None
    roof["traffic_note"] = "DRAM bytes per step: sum of the step kernels' ncu dram__bytes"
    dominant = max(kernels, key=lambda n: kernels[n]["ms_per_launch"])
    roof["dominant_kernel"] = dict(kernels[dominant])
    return roof, kernels


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    import datetime

    import torch.distributed as dist

    import geometry_aware_local_pack3d_b200 as p3d

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    sync = dist.barrier if world > 1 else None

    if args.batch is not None:
        cfg = dict(inputs.WORKLOADS[args.workload])
        cfg["batch"] = args.batch
        w = inputs.make_workload(cfg)
    else:
        w = inputs.make_workload(args.workload)
    B, H, N, M, d = _sizes(w)
    F = Forward(p3d, w, dev)

    clocks = ClockSampler(local) if (rank == 0 and not args.no_clocks) else None
    if clocks:
        clocks.start()
    ms, ms_k, launches = F.time(args.steps, args.warmup, sync)
    clk = clocks.stop() if clocks else None
    vals = max_over_ranks([ms] + [ms_k[n] for n in ("summarize", "local", "global")],
                          dist if world > 1 else None, dev)
    ms, ms_k = vals[0], dict(zip(("summarize", "local", "global"), vals[1:]))
    peaks = measured_peaks()

    # Outside the headline step (rank 0's GPU alone): the index build (once per geometry), the
    # forward + backward of the same field (dO ~ N(0, 1), seed 2) and the 262,144-token field,
    # each timed with CUDA events on this stream.
    extra = {}
    if not args.skip_bwd and world == 1:
        stream = F.stream
        coords_d = torch.from_numpy(w["coords"]).to(dev)
        ie0, ie1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        p3d.pack3d_build_index(F.geom, coords=coords_d)
        ie0.record(stream)
        for _ in range(3):
            p3d.pack3d_build_index(F.geom, coords=coords_d)
        ie1.record(stream)
        torch.cuda.synchronize()
        extra["index_build"] = {"ms": ie0.elapsed_time(ie1) / 3,
                                "note": "inverse map, neighbour and block tables, RoPE table; "
                                        "includes the call's one host synchronisation"}
        excl = w["exclude_near"]
        dO = inputs.pack(inputs.upstream_grad(B, H, w["grid"], d), w["perm"]).to(
            torch.bfloat16).to(dev)
        ws = torch.empty(p3d.pack3d_bwd_workspace_bytes(F.ix, 1, B, H), dtype=torch.uint8,
                         device=dev)

        def fwd_saving():
            p3d.pack3d_summarize_rotated(F.ix, F.k, F.v, F.ksum, F.vsum, F.k_rot)
            return p3d.pack3d_attn_fwd(F.ix, F.q, F.k_rot, F.v, F.a, F.ksum, F.vsum,
                                       exclude_near=excl, k_rotated=True, save_for_backward=True)

        saved = fwd_saving()
        p3d.pack3d_attn_bwd(F.ix, F.q, F.k, F.v, F.a, F.ksum, F.vsum, saved, dO,
                            exclude_near=excl, workspace=ws)
        torch.cuda.synchronize()
        nb = 3
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(nb)]
        for i in range(nb):
            ev[i][0].record(stream)
            saved = fwd_saving()
            ev[i][1].record(stream)
            p3d.pack3d_attn_bwd(F.ix, F.q, F.k, F.v, F.a, F.ksum, F.vsum, saved, dO,
                                exclude_near=excl, workspace=ws)
            ev[i][2].record(stream)
        torch.cuda.synchronize()
        fms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
        bms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
        # the global branch's backward: five products of N x M x d per (batch, head) (S
        # recomputed, dP, dq, dK_sum, dV_sum), 2.5x its forward contraction
        bflops = 10.0 * N * M * d * B * H
        fflops = 4.0 * N * M * d * B * H
        extra["attn_bwd"] = {"ms": bms, "tokens_per_s": B * N / (bms / 1e3),
                             "roofline": {"bound": "tensor", "algorithmic_flops": bflops,
                                          "achieved": bflops / (bms / 1e3) / 1e12,
                                          "peak": peaks["bf16"], "unit": "TFLOP/s",
                                          "frac": bflops / (bms / 1e3) / 1e12 / peaks["bf16"]},
                             "path": "tensor cores: global branch (k_bwd_dsum_tc, "
                                     "k_bwd_dq_tc) and local branch (k_bwd_local_dq_tc, "
                                     "k_bwd_local_dkv_tc, with the un-pooling and inverse RoPE "
                                     "in their epilogues); the row prologue on CUDA cores "
                                     "(k_bwd_prep)"}
        extra["fwd_bwd"] = {"workload": "field65k_fwdbwd_bf16 (the headline field, forward "
                                        "saving o_loc, o_glob and both lse, then the backward)",
                            "ms": fms + bms, "fwd_ms": fms, "bwd_ms": bms,
                            "tokens_per_s": B * N / ((fms + bms) / 1e3),
                            "roofline": {"bound": "tensor",
                                         "algorithmic_flops": fflops + bflops,
                                         "achieved": (fflops + bflops) / ((fms + bms) / 1e3) / 1e12,
                                         "peak": peaks["bf16"], "unit": "TFLOP/s",
                                         "frac": (fflops + bflops) / ((fms + bms) / 1e3) / 1e12
                                         / peaks["bf16"]}}
        del saved, dO, ws

        # the 262,144-token field (64^3, batch 1, 8 heads, 4,096 summaries)
        name = "field262k_bf16"
        w2 = device_workload(name, dev)
        F2 = Forward(p3d, w2, dev)
        ms2, ms2_k, _ = F2.time(10, 3)
        roof2, kern2 = forward_line(w2, name, ms2, ms2_k, F2.index_bytes(), peaks)
        B2, H2, N2, _, _ = _sizes(w2)
        extra[name] = {"config": workload_config(name, w2), "ms_per_step": ms2,
                       "tokens_per_s": B2 * N2 / (ms2 / 1e3), "roofline": roof2,
                       "kernels": kern2, "steps": 10, "warmup": 3,
                       "data": "synthetic, drawn on the device (seeded CUDA generator)"}
        del F2, w2
        torch.cuda.empty_cache()

        # the pages' high-token point: 1,048,576 tokens, 4,096 summaries per KV head
        name = "field1m_bf16"
        w3 = device_workload(name, dev)
        F3 = Forward(p3d, w3, dev)
        ms3, ms3_k, _ = F3.time(5, 2)
        roof3, kern3 = forward_line(w3, name, ms3, ms3_k, F3.index_bytes(), peaks)
        B3, H3, N3, _, _ = _sizes(w3)
        extra[name] = {"config": workload_config(name, w3), "ms_per_step": ms3,
                       "tokens_per_s": B3 * N3 / (ms3 / 1e3), "roofline": roof3,
                       "kernels": kern3, "steps": 5, "warmup": 2,
                       "data": "synthetic, drawn on the device (seeded CUDA generator)"}
        del F3, w3
        torch.cuda.empty_cache()

    # End to end through the public API with host buffers: every step copies its inputs q, k,
    # v, a from pinned host memory to the device and its output o back. Steps are pipelined as
    # a serving loop would run them: two device input/output sets, host->device copies on one
    # stream, the operator on the compute stream, device->host copies on a third, so a step's
    # input upload, the previous step's compute and an earlier step's download overlap (PCIe
    # is full duplex). The timed region runs from the first upload to the last download.
    e2e = None
    if not args.skip_e2e:
        dt = torch.bfloat16
        hq, hk, hv, ha = (t.to(dt).pin_memory() for t in (w["q"], w["k"], w["v"], w["a"]))
        ho = [torch.empty(F.o.shape, dtype=dt).pin_memory() for _ in range(2)]
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, ha))
        d2h = ho[0].numel() * ho[0].element_size()
        sets = [dict(q=F.q, k=F.k, v=F.v, a=F.a, o=F.o)]
        sets.append({n: torch.empty_like(sets[0][n]) for n in ("q", "k", "v", "a", "o")})
        s_up, s_down = torch.cuda.Stream(), torch.cuda.Stream()
        s_comp = F.stream

        def e2e_run(k_steps):
            up = [torch.cuda.Event() for _ in range(k_steps)]
            done = [torch.cuda.Event() for _ in range(k_steps)]
            down = [torch.cuda.Event() for _ in range(k_steps)]
            for i in range(k_steps):
                bufs = sets[i % 2]
                with torch.cuda.stream(s_up):
                    if i >= 2:
                        s_up.wait_event(done[i - 2])  # the set's previous compute has read it
                    for n, h in (("q", hq), ("k", hk), ("v", hv), ("a", ha)):
                        bufs[n].copy_(h, non_blocking=True)
                    up[i].record(s_up)
                s_comp.wait_event(up[i])
                if i >= 2:
                    s_comp.wait_event(down[i - 2])  # the set's previous output has left
                F.q, F.k, F.v, F.a, F.o = (bufs[n] for n in ("q", "k", "v", "a", "o"))
                F.step()
                done[i].record(s_comp)
                with torch.cuda.stream(s_down):
                    s_down.wait_event(done[i])
                    ho[i % 2].copy_(bufs["o"], non_blocking=True)
                    down[i].record(s_down)
            return down[-1]

        e2e_run(2)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        k_e2e = max(3, min(args.steps, 10))
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(s_up)
        last = e2e_run(k_e2e)
        s_down.wait_event(last)
        e1.record(s_down)
        torch.cuda.synchronize()
        ems = e0.elapsed_time(e1) / k_e2e
        ems = max_over_ranks([ems], dist if world > 1 else None, dev)[0]
        F.q, F.k, F.v, F.a, F.o = (sets[0][n] for n in ("q", "k", "v", "a", "o"))
        e2e = {"value": job_throughput(world, B * N, ems), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": ems, "steps": k_e2e,
               "pipelining": "uploads, compute and downloads of consecutive steps overlap on "
                             "three streams (two device input/output sets)"}

    if rank == 0:
        roof, kernels = forward_line(w, args.workload, ms, ms_k, F.index_bytes(), peaks)
        line = {
            "metric": METRIC, "value": job_throughput(world, B * N, ms), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": workload_config(args.workload, w),
            "roofline": roof,
            "kernels": kernels,
            "gpu_launches": launches,
            "clocks": clk,
            "e2e": e2e,
        }
        line.update(extra)
        if not args.skip_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(w)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
