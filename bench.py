"""Benchmark of the PACK3D attention forward on B200 (one process per GPU).

A step is one pass of the operator's hot path over one batch of synthetic input: block
summaries with the rotated keys written in the same pass (pack3d_summarize_rotated), the local
branch on those keys (pack3d_attn_local with PACK3D_K_ROTATED), then the global branch with the
mixer (pack3d_attn_global) -- the two halves of pack3d_attn_fwd, called separately so that each
kernel is timed with CUDA events on the stream it runs on -- the index of
the packed field is built once per geometry before timing, as it is amortised over layers,
heads and batches. Default workload: the 65,536-token field (32x32x64 grid, batch 2, 8 heads,
head_dim 96, bf16, 4x4x4 blocks -> 1,024 summaries, raster-block packing).

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
    return ap.parse_args()


def workload_config(name, w):
    return {"workload": name, "grid": list(w["grid"]), "block": list(w["block"]),
            "batch": w["batch"], "heads": w["heads"], "head_dim": w["d"],
            "tokens": int(np.prod(w["grid"])), "summaries": int(np.prod(
                [g // b for g, b in zip(w["grid"], w["block"])])),
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


def algorithmic(w):
    """Per-launch algorithmic work of the three kernels of a step (each row read or written
    once; index tables read once)."""
    B, H, d = w["batch"], w["heads"], w["d"]
    N = int(np.prod(w["grid"]))
    M = int(np.prod([g // b for g, b in zip(w["grid"], w["block"])]))
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


# -------------------------------------------------------------------------------- oracle
def oracle_sample(w, idx, head=(0, 0)):
    """Time the float64 oracle on one (batch, head) of the workload: summaries + all rows."""
    from oracle import pack3d_oracle as orc
    b, h = head
    sl = lambda t: t[b:b + 1, h:h + 1].numpy()  # noqa: E731
    q, k, v, a = sl(w["q"]), sl(w["k"]), sl(w["v"]), sl(w["a"])
    t0 = time.perf_counter()
    orc.forward(q, k, v, a, w["coords"], w["grid"], w["block"], exclude_near=w["exclude_near"],
                index=idx)
    return time.perf_counter() - t0


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info()]
        return max(n) if n else 1
    except Exception:
        return 1


def cpu_baseline(w, reps=1):
    from oracle import pack3d_oracle as orc
    idx = orc.build_index(w["coords"], w["grid"], w["block"])
    ts = [oracle_sample(w, idx) for _ in range(reps)]
    t = statistics.median(ts)
    B, H = w["batch"], w["heads"]
    N = int(np.prod(w["grid"]))
    # one head of one batch element is 1/(B*H) of a step
    value = (B * N) / (t * B * H)
    return {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"float64 numpy oracle on 1 of {B * H} (batch, head) pairs of the workload "
                      f"(summaries + local + global + mixer for all {N} tokens), {reps} rep(s), "
                      f"{t:.2f} s each, scaled by {B * H}"}


def run_reference(args, rank):
    if rank != 0:
        return
    w = inputs.make_workload(args.workload)
    from oracle import pack3d_oracle as orc
    idx = orc.build_index(w["coords"], w["grid"], w["block"])
    for _ in range(args.warmup):
        oracle_sample(w, idx)
    ts = [oracle_sample(w, idx, head=(s % w["batch"], s % w["heads"])) for s in range(args.steps)]
    B, H = w["batch"], w["heads"]
    N = int(np.prod(w["grid"]))
    step = float(np.mean(ts)) * B * H
    value = B * N / step
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference", "config": workload_config(args.workload, w),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(),
                             "kind": "oracle",
                             "sample": f"each step: the float64 oracle on one (batch, head) of "
                                       f"{B * H}, all {N} tokens; value scaled by {B * H}"},
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

    w = inputs.make_workload(args.workload)
    B, H, d = w["batch"], w["heads"], w["d"]
    N = int(np.prod(w["grid"]))
    dt = torch.bfloat16 if w["dtype"] == "bf16" else torch.float32
    geom = p3d.make_geom(w["grid"], w["block"], d)
    ix = p3d.pack3d_build_index(geom, coords=torch.from_numpy(w["coords"]).to(dev))
    q, k, v, a = (w[n].to(dt).to(dev).contiguous() for n in "qkva")
    ksum = torch.empty(p3d.summary_tiles_shape(ix, B, H, d), dtype=dt, device=dev)
    vsum = torch.empty_like(ksum)
    k_rot = torch.empty_like(k)
    o = torch.empty_like(q)
    excl = w["exclude_near"]
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        p3d.pack3d_summarize_rotated(ix, k, v, ksum, vsum, k_rot)
        n = p3d.pack3d_last_launch_count()
        if ev is not None:
            ev[1].record(stream)
        p3d.pack3d_attn_local(ix, q, k_rot, v, k_rotated=True, o_loc=o)
        n += p3d.pack3d_last_launch_count()
        if ev is not None:
            ev[2].record(stream)
        p3d.pack3d_attn_global(ix, q, a, ksum, vsum, o, exclude_near=excl, o=o)
        n += p3d.pack3d_last_launch_count()
        if ev is not None:
            ev[3].record(stream)
        return n

    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()

    clocks = ClockSampler(local) if (rank == 0 and not args.no_clocks) else None
    if clocks:
        clocks.start()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches = 0
    t0.record(stream)
    for s in range(args.steps):
        launches += step(evs[s])
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clk = clocks.stop() if clocks else None

    ms = t0.elapsed_time(t1) / args.steps
    ms_k = {name: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in evs)
            for i, name in enumerate(("summarize", "local", "global"))}
    vals = max_over_ranks([ms] + [ms_k[n] for n in ("summarize", "local", "global")],
                          dist if world > 1 else None, dev)
    ms, ms_k = vals[0], dict(zip(("summarize", "local", "global"), vals[1:]))

    # Outside the headline step: the index build (once per geometry) and the backward of the
    # same field (dO ~ N(0, 1), seed 2), each timed with CUDA events on this stream.
    extra = {}
    if not args.skip_bwd and world == 1:
        coords_d = torch.from_numpy(w["coords"]).to(dev)
        ie0, ie1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        p3d.pack3d_build_index(geom, coords=coords_d)
        ie0.record(stream)
        for _ in range(3):
            p3d.pack3d_build_index(geom, coords=coords_d)
        ie1.record(stream)
        torch.cuda.synchronize()
        extra["index_build"] = {"ms": ie0.elapsed_time(ie1) / 3,
                                "note": "inverse map, neighbour and block tables, RoPE table; "
                                        "includes the call's one host synchronisation"}
        saved = p3d.pack3d_attn_fwd(ix, q, k, v, a, ksum, vsum, exclude_near=excl,
                                    save_for_backward=True)
        dO = inputs.pack(inputs.upstream_grad(B, H, w["grid"], d), w["perm"]).to(dt).to(dev)
        ws = torch.empty(p3d.pack3d_bwd_workspace_bytes(ix, 1 if dt == torch.bfloat16 else 0,
                                                        B, H), dtype=torch.uint8, device=dev)
        p3d.pack3d_attn_bwd(ix, q, k, v, a, ksum, vsum, saved, dO, exclude_near=excl, workspace=ws)
        be0, be1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        be0.record(stream)
        nb = 3
        for _ in range(nb):
            p3d.pack3d_attn_bwd(ix, q, k, v, a, ksum, vsum, saved, dO, exclude_near=excl,
                                workspace=ws)
        be1.record(stream)
        torch.cuda.synchronize()
        bms = be0.elapsed_time(be1) / nb
        M = int(np.prod([g_ // b_ for g_, b_ in zip(w["grid"], w["block"])]))
        # the global branch's backward: five products of N x M x d per (batch, head) (S
        # recomputed, dP, dq, dK_sum, dV_sum), 2.5x its forward contraction
        bflops = 10.0 * N * M * d * B * H
        peaks_b = measured_peaks()
        extra["attn_bwd"] = {"ms": bms, "tokens_per_s": B * N / (bms / 1e3),
                             "roofline": {"bound": "tensor", "algorithmic_flops": bflops,
                                          "achieved": bflops / (bms / 1e3) / 1e12,
                                          "peak": peaks_b["bf16"], "unit": "TFLOP/s",
                                          "frac": bflops / (bms / 1e3) / 1e12 / peaks_b["bf16"]},
                             "path": "global branch on tensor cores (k_bwd_dsum_tc, "
                                     "k_bwd_dq_tc); row prologue, local branch, un-pooling and "
                                     "inverse RoPE on CUDA cores (k_bwd_prep, k_bwd_dq, "
                                     "k_bwd_dkv)"}
        del saved, dO, ws

    # end to end through the public API with host buffers: H2D of the inputs and D2H of o
    e2e = None
    if not args.skip_e2e:
        hq, hk, hv, ha = (t.to(dt).pin_memory() for t in (w["q"], w["k"], w["v"], w["a"]))
        ho = torch.empty(o.shape, dtype=dt).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, ha))
        d2h = ho.numel() * ho.element_size()

        def e2e_step():
            q.copy_(hq, non_blocking=True)
            k.copy_(hk, non_blocking=True)
            v.copy_(hv, non_blocking=True)
            a.copy_(ha, non_blocking=True)
            step()
            ho.copy_(o, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        k_e2e = max(3, min(args.steps, 10))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(k_e2e):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        ems = e0.elapsed_time(e1) / k_e2e
        ems = max_over_ranks([ems], dist if world > 1 else None, dev)[0]
        e2e = {"value": job_throughput(world, B * N, ems), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": ems, "steps": k_e2e}

    if rank == 0:
        peaks = measured_peaks()
        alg = algorithmic(w)
        kernel_names = {"summarize": "k_summarize (pack3d_summarize_rotated)",
                        "local": "k_local_tma (pack3d_attn_local)",
                        "global": "k_global_tc (pack3d_attn_global)"}
        kernels = {}
        for name in ("summarize", "local", "global"):
            sec = ms_k[name] / 1e3
            if "flops" in alg[name]:
                ach = alg[name]["flops"] / sec / 1e12
                ent = {"bound": "tensor", "achieved": ach, "peak": peaks["bf16"],
                       "unit": "TFLOP/s", "frac": ach / peaks["bf16"],
                       "algorithmic_flops_per_launch": alg[name]["flops"],
                       "peak_source": f"{peaks['source']} bf16 dense burst"}
            else:
                ach = alg[name]["bytes"] / sec / 1e9
                ent = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm"], "unit": "GB/s",
                       "frac": ach / peaks["hbm"],
                       "peak_source": f"{peaks['source']} HBM copy"}
            ent.update({"kernel": kernel_names[name], "ms_per_launch": ms_k[name],
                        "algorithmic_bytes_per_launch": alg[name]["bytes"],
                        "traffic": kernel_traffic(f"{name}_{args.workload}")})
            kernels[name] = ent
        dominant = max(kernels, key=lambda n: kernels[n]["ms_per_launch"])
        roof = dict(kernels[dominant])
        line = {
            "metric": METRIC, "value": job_throughput(world, B * N, ms), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": workload_config(args.workload, w),
            "roofline": roof,
            "kernels": kernels,
            # the global contraction's flops over the whole forward (local + global kernels)
            "fwd_tflops": alg["global"]["flops"] / ((ms_k["local"] + ms_k["global"]) / 1e3) / 1e12,
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
