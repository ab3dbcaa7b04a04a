#!/usr/bin/env python
"""Benchmark of the pair-biased attention hot path on B200.

One step = the "large" workload: pba_forward at N=16384, H=16, D=64 bf16 with a
5% random key mask (bias [H,N,N] = 8.6 GB), then triangle attention on a pair
tensor of N=1024, H=4, D=32 in both orientations.  Inputs are synthetic and
seeded (workloads.py) and resident in HBM before the timed region; every input
is larger than L2, so no flush is needed between iterations.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  Under torchrun each rank runs the same
workload on its own GPU (weak scaling, no collective on the data path); the
step time is the maximum over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "pair-bias attention TFLOP/s & bias HBM GB/s vs roofline at N=16K; tri-attn rows/s"
UNIT = "TFLOP/s"


def attn_flops(B, H, Nq, Nk, D) -> float:
    """Q K^T and P V: 2 * 2 * B*H*Nq*Nk*D (Fold-CP Table 1 serial time B H N^2 D)."""
    return 4.0 * B * H * Nq * Nk * D


def tri_ceilings(N, H, D, ms_per_call, tensor_tflops, hbm_gbs, sm_mhz, n_sms) -> dict:
    """The three ceilings of one triangle-attention call on a pair tensor of
    N x N rows (one orientation, gate and lse written) and the measured call's
    fraction of each: the tensor cores (4 N^3 H D FLOPs), HBM (q, k, v, gate
    read and out written as bf16 [N,N,H,D], lse [N,N,H] fp32, bias [H,N,N]
    bf16) and the exp2 unit (one exponential per score, N^3 H of them, at 16
    per clock per SM).  frac = ceiling time / measured time."""
    flops = 4.0 * N * N * N * H * D
    nbytes = 5.0 * N * N * H * D * 2 + N * N * H * 4 + H * N * N * 2
    exps = float(N) * N * N * H
    floors = {"tensor": flops / (tensor_tflops * 1e12) * 1e3,
              "hbm": nbytes / (hbm_gbs * 1e9) * 1e3,
              "exp2": exps / (16.0 * n_sms * sm_mhz * 1e6) * 1e3}
    return {"ms_per_call": ms_per_call, "floor_ms": floors,
            "frac": {k: v / ms_per_call for k, v in floors.items()},
            "flops_per_call": flops, "bytes_per_call": nbytes, "exps_per_call": exps}


def attn_bytes(B, H, Nq, Nk, D, elt=2, mask=True) -> float:
    """Algorithmic HBM bytes of one pass: bias, Q, K, V read once, O and the
    log-sum-exp written once, the key mask read once."""
    return (B * H * Nq * Nk * elt + B * H * (Nq + 2 * Nk) * D * elt + B * H * Nq * D * elt + B * H * Nq * 4 +
            (B * Nk if mask else 0))


def roofline_entry(flops, nbytes, seconds, peaks, traffic, kernel):
    """Roofline of one launch: the slower of the dense-bf16 floor (flops at the
    burst tensor peak) and the HBM floor (algorithmic bytes at the copy
    bandwidth) sets the bound; achieved and frac are in that bound's unit."""
    t_tensor = flops / (peaks["bf16_tflops"] * 1e12)
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    tflops = flops / seconds / 1e12
    gbs = nbytes / seconds / 1e9
    if t_hbm >= t_tensor:
        e = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
             "frac": gbs / peaks["hbm_gbs"]}
    else:
        e = {"bound": "tensor", "achieved": tflops, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
             "frac": tflops / peaks["bf16_tflops"]}
    e.update({"traffic": traffic, "kernel": kernel, "algorithmic_bytes_per_launch": nbytes,
              "flops_per_launch": flops, "floor_ms": {"tensor": t_tensor * 1e3, "hbm": t_hbm * 1e3},
              "peak_source": peaks["source"], "tensor_frac": tflops / peaks["bf16_tflops"],
              "tensor_frac_sustained": tflops / peaks["bf16_tflops_sustained"], "hbm_frac": gbs / peaks["hbm_gbs"]})
    return e


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def kernel_source_sha256() -> str:
    import glob
    import hashlib

    h = hashlib.sha256()
    # the attention kernel's own sources: other kernels of the library do not change its traffic
    files = [os.path.join(ROOT, "pair_biased_attention_b200", "csrc", n) for n in ("pba_attn_sm100.cuh", "pba_ptx.cuh")]
    for f in files:
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def measured_traffic():
    """DRAM bytes per large16k launch from the last ncu capture, or None when
    the kernel sources changed since that capture."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    if rec.get("kernel_source_sha256") != kernel_source_sha256():
        return None
    return rec.get("pba_attn_sm100_large16k_bytes_per_launch")


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.proc = None
        self.uuid = None
        try:
            self.uuid = str(torch.cuda.get_device_properties(device).uuid).replace("-", "").lower()
        except Exception:
            pass

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons, power = [], None, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            uid = parts[0].replace("GPU-", "").replace("-", "").lower()
            if self.uuid and self.uuid not in uid and uid not in self.uuid:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
                power.append(float(parts[3]))
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        loaded = [s for s, p in zip(sm, power) if p > 300] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power) if power else None}


# ------------------------------------------------------------------ distributed plumbing
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = False
    if world > 1 and args.impl == "ours":
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        pg = True
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local, pg


def max_over_ranks(x: float, pg: bool, device: str = "cuda") -> float:
    """Largest value over the ranks (the step time every rank waits for)."""
    if not pg:
        return x
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, work_per_rank_step: float, steps: int, t_max_ms: float) -> float:
    """Whole-job rate: every rank does the same work per step (weak scaling);
    the job time is the slowest rank's."""
    return world * work_per_rank_step * steps / (t_max_ms / 1e3)


def barrier(pg: bool):
    torch.cuda.synchronize()
    if pg:
        import torch.distributed as dist

        dist.barrier()
        torch.cuda.synchronize()


# ------------------------------------------------------------------ CPU oracle timing
ORACLE_CHUNK_ROWS = 1024


def oracle_chunks(q, k, v, bias, mask, n_chunks, chunk_rows=ORACLE_CHUNK_ROWS, seed=77):
    """Seeded chunks of query rows of the large workload, one head per chunk
    round robin, each against all keys, converted to fp64 host arrays before
    any timing (the conversion is not the oracle's work)."""
    import numpy as np

    H, N = q.shape[1], q.shape[2]
    g = torch.Generator("cpu").manual_seed(seed)
    ms = None if mask is None else mask.cpu().numpy().astype(np.uint8)
    f64 = lambda t: np.ascontiguousarray(t.cpu().double().numpy())
    kv = {}
    for c in range(n_chunks):
        h = c % H
        rows = torch.randperm(N, generator=g)[:chunk_rows].to(q.device)
        if h not in kv:
            kv[h] = (f64(k[:, h:h + 1]), f64(v[:, h:h + 1]))
        yield (f64(q[:, h:h + 1].index_select(2, rows)), kv[h][0], kv[h][1],
               f64(bias[:, h:h + 1].index_select(2, rows)), ms)


def time_oracle_chunk(chunk) -> float:
    """Seconds of one oracle call on one chunk (all host cores)."""
    import oracle

    t0 = time.perf_counter()
    oracle.pba(*chunk)
    return time.perf_counter() - t0


def oracle_sample(q, k, v, bias, mask, target_s=10.0, chunk_rows=ORACLE_CHUNK_ROWS):
    """Times the fp64 oracle on sampled query rows of the large workload (all
    16384 keys each), chunk by chunk, until about target_s seconds of oracle
    time.  Returns (TFLOP/s, threads, description, seconds)."""
    import oracle

    N, D = q.shape[2], q.shape[3]
    flops, t, nrows = 0.0, 0.0, 0
    chunks = oracle_chunks(q, k, v, bias, mask, 256, chunk_rows)
    for ch in chunks:
        if t >= target_s:
            break
        t += time_oracle_chunk(ch)
        flops += attn_flops(1, 1, chunk_rows, N, D)
        nrows += chunk_rows
    return (flops / t / 1e12, oracle.threads_used(),
            f"{nrows} query rows x {N} keys of large16k, {chunk_rows}-row chunks over the heads (fp64 oracle)", t)


# ------------------------------------------------------------------ the reference arm
def run_reference(args, world, rank):
    """The oracle as the reference arm: each step is one 1024-row chunk of the
    large workload's query rows against all keys (the chunking of the
    cpu_baseline leg, so both report one oracle rate)."""
    if rank != 0:
        return 0
    import oracle

    oracle.build()
    cfg = W.LARGE16K
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    q, k, v, bias, mask = W.attn_inputs(cfg, dev)
    H, N, D = cfg.H, cfg.N, cfg.D
    warm = max(1, args.warmup)
    chunks = oracle_chunks(q, k, v, bias, mask, warm + args.steps)
    times = []
    for c, ch in enumerate(chunks):  # each chunk converted before its timed call
        t = time_oracle_chunk(ch)
        if c >= warm:
            times.append(t)
    total = sum(times)
    flops_step = attn_flops(1, 1, ORACLE_CHUNK_ROWS, N, D)
    value = flops_step * args.steps / total / 1e12
    cores = oracle.threads_used()
    desc = (f"{ORACLE_CHUNK_ROWS} query rows x {N} keys of large16k per step, one head per step round robin "
            f"(fp64 oracle, {cores} threads)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": warm, "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "large16k: pair-biased attention N=16384 H=16 D=64, 5% random key mask (sampled rows)",
                   "B": 1, "N": N, "H": H, "D": D},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ our arm
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=60)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--profile", choices=["none", "pba4k", "tri512", "proj1024", "oproj1024", "pwa4k", "bwd4k", "f32_4k",
                                          "merge8k"],
                    default="none",
                    help="run one small case only (for ncu captures); prints no JSON line")
    args = ap.parse_args()
    world, rank, local, pg = dist_setup(args)
    if args.impl == "reference":
        return run_reference(args, world, rank)

    import pair_biased_attention_b200 as pba

    pba.load_library()
    dev = torch.device("cuda", local)

    if args.profile != "none":
        return run_profile_case(args, pba, dev)

    peaks = load_peaks()
    cfg = W.LARGE16K
    tcfg = W.TRI1024
    q, k, v, bias, mask = W.attn_inputs(cfg, dev)
    tq, tk, tv, tg, tb = W.tri_inputs(tcfg, dev)
    out = torch.empty_like(q)
    lse = torch.empty((cfg.B, cfg.H, cfg.N), dtype=torch.float32, device=dev)
    tout = torch.empty_like(tq)
    tlse = torch.empty((tcfg.N, tcfg.N, tcfg.H), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        pba.pba_forward(q, k, v, bias, mask, out, lse, stream=stream)
        if ev:
            ev[1].record(stream)
        pba.tri_attn_forward(tq, tk, tv, tb, tg, None, "starting", tout, tlse, stream=stream)
        pba.tri_attn_forward(tq, tk, tv, tb, tg, None, "ending", tout, tlse, stream=stream)
        if ev:
            ev[2].record(stream)

    for _ in range(max(3, args.warmup)):
        step()
    assert pba.pba_last_device_error(stream) == pba.PBA_OK
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    clocks = ClockSampler(dev)
    barrier(pg)
    clocks.start()
    for i in range(args.steps):
        step(evs[i])
    barrier(pg)
    clk = clocks.stop()
    if pba.pba_last_device_error(stream) != pba.PBA_OK:
        raise RuntimeError("a kernel recorded a device error during the timed steps")
    pba_ms = [e[0].elapsed_time(e[1]) for e in evs]
    tri_ms = [e[1].elapsed_time(e[2]) for e in evs]
    step_ms = [e[0].elapsed_time(e[2]) for e in evs]
    t_pba = max_over_ranks(sum(pba_ms), pg)
    t_tri = max_over_ranks(sum(tri_ms), pg)
    t_step = max_over_ranks(sum(step_ms), pg)

    flops = attn_flops(cfg.B, cfg.H, cfg.N, cfg.N, cfg.D)
    nbytes = attn_bytes(cfg.B, cfg.H, cfg.N, cfg.N, cfg.D)
    value = job_throughput(world, flops, args.steps, t_pba) / 1e12
    avg_launch_s = sum(pba_ms) / len(pba_ms) / 1e3
    achieved_gbs = nbytes / avg_launch_s / 1e9
    tri_rows = 2 * tcfg.N  # pair-tensor rows per step (starting + ending)
    tri_rows_per_s = job_throughput(world, tri_rows, args.steps, t_tri)
    tri_flops = 2 * attn_flops(tcfg.N, tcfg.H, tcfg.N, tcfg.N, tcfg.D)

    traffic = measured_traffic()

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": t_step / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "large16k: pair-biased attention N=16384 H=16 D=64 bf16, bias [H,N,N] ~N(0,1), "
                               "5% random key mask; plus triangle attention N=1024 c=128 H=4 D=32 (starting+ending)",
                   "B": cfg.B, "N": cfg.N, "H": cfg.H, "D": cfg.D, "tri_N": tcfg.N, "tri_H": tcfg.H, "tri_D": tcfg.D,
                   "l2": "no flush: every input is larger than L2 (bias 8.6 GB, tri q/k/v/g 1.07 GB)",
                   "parallelism": f"replicas x{world} (independent problems per GPU)"},
        "pba_ms_per_launch": sum(pba_ms) / len(pba_ms),
        "bias_hbm_gbs": cfg.B * cfg.H * cfg.N * cfg.N * 2 / avg_launch_s / 1e9,
        "tri_attn_rows_per_s": tri_rows_per_s,
        "tri_attn_ms_per_call": sum(tri_ms) / len(tri_ms) / 2,
        "tri_attn_tflops": world * tri_flops * args.steps / (t_tri / 1e3) / 1e12,
        "tri_attn_ceilings": tri_ceilings(tcfg.N, tcfg.H, tcfg.D, sum(tri_ms) / len(tri_ms) / 2,
                                          peaks["bf16_tflops_sustained"], peaks["hbm_gbs"],
                                          (clk.get("sm_mhz") or 1965.0) if isinstance(clk, dict) else 1965.0,
                                          torch.cuda.get_device_properties(dev).multi_processor_count),
        "roofline": roofline_entry(flops, nbytes, avg_launch_s, peaks, traffic,
                                   "pba_attn_sm100_kernel (pba_forward, large16k)"),
        "gpu_launches": 3 * args.steps,
        "clocks": clk,
    }

    line["tri_proj"] = run_proj(args, pba, tcfg, dev, stream, pg, peaks)
    line["tri_out_proj"] = run_out_proj(args, pba, tcfg, dev, stream, pg, peaks)
    line["pwa"] = run_pwa(args, pba, dev, stream, pg, peaks, clk)
    line["backward"] = run_bwd(args, pba, dev, stream, pg, peaks)
    line["ring8k"] = run_ring8k(args, pba, dev, stream, pg, peaks)
    line["f32"] = run_f32(args, pba, dev, stream, pg, peaks)
    line["configs"] = run_configs(args, pba, dev, stream, pg, peaks, line, clk)
    if not args.no_e2e:
        line["e2e"] = run_e2e(args, pba, cfg, q, k, v, bias, mask, out, lse, stream, pg, world, flops)
    if not args.no_cpu and rank == 0 and world == 1:
        val, cores, desc, secs = oracle_sample(q, k, v, bias, mask, target_s=args.cpu_seconds)
        line["cpu_baseline"] = {"value": val, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc,
                                "seconds": secs, "per_config": oracle_per_config(dev, val, cores)}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg:
        import torch.distributed as dist

        dist.destroy_process_group()
    return 0


def run_proj(args, pba, tcfg, dev, stream, pg, peaks):
    """The triangle projections of the triangle workload (tri_proj_forward:
    z [N,N,c] -> q, k, v, g [N,N,H,D] and bias [H,N,N]), timed on their own
    after the step: K calls after 3 warm-up calls, CUDA events on the stream.
    HBM-bound: algorithmic bytes = z read once + the five outputs written."""
    z, w, wb = W.tri_pair_inputs(tcfg, dev)
    N2 = tcfg.N * tcfg.N
    outs = tuple(torch.empty((tcfg.N, tcfg.N, tcfg.H, tcfg.D), dtype=torch.bfloat16, device=dev) for _ in range(4))
    pb = torch.empty((tcfg.H, tcfg.N, tcfg.N), dtype=torch.bfloat16, device=dev)
    call = lambda: pba.tri_proj_forward(z, w, wb, tcfg.H, out=outs, bias=pb, stream=stream)
    for _ in range(3):
        call()
    barrier(pg)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(args.steps):
        call()
    e.record(stream)
    barrier(pg)
    if pba.pba_last_device_error(stream) != pba.PBA_OK:
        raise RuntimeError("the projection kernel recorded a device error")
    ms = max_over_ranks(s.elapsed_time(e), pg) / args.steps
    nbytes = N2 * tcfg.c * 2 + 4 * N2 * tcfg.H * tcfg.D * 2 + tcfg.H * N2 * 2
    flops = 2.0 * N2 * tcfg.c * (4 * tcfg.H * tcfg.D + tcfg.H)
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"ms_per_call": ms, "calls": args.steps, "gpu_launches": args.steps,
            "workload": f"tri{tcfg.N}: z [{tcfg.N},{tcfg.N},{tcfg.c}] bf16 -> q,k,v,g [N,N,{tcfg.H},{tcfg.D}] + bias [{tcfg.H},N,N]",
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "algorithmic_bytes_per_call": nbytes,
                         "kernel": "pba_proj_sm100_kernel (tri_proj_forward)", "peak_source": peaks["source"],
                         "tensor_frac": (flops / (ms / 1e3) / 1e12) / peaks["bf16_tflops"]}}


def run_out_proj(args, pba, tcfg, dev, stream, pg, peaks):
    """The output projection of the triangle workload (tri_out_proj_forward:
    o [N,N,H,D] -> out [N,N,c] = o W_o), timed on its own after the step: K
    calls after 3 warm-up calls, CUDA events on the stream.  HBM-bound:
    algorithmic bytes = o read once + out written once (+ W_o)."""
    g = torch.Generator(dev.type).manual_seed(tcfg.seed + 100)
    HD = tcfg.H * tcfg.D
    o = torch.randn((tcfg.N, tcfg.N, tcfg.H, tcfg.D), generator=g, device=dev).to(torch.bfloat16)
    w_o = (torch.randn((HD, tcfg.c), generator=g, device=dev) / HD ** 0.5).to(torch.bfloat16)
    out = torch.empty((tcfg.N, tcfg.N, tcfg.c), dtype=torch.bfloat16, device=dev)
    call = lambda: pba.tri_out_proj_forward(o, w_o, out=out, stream=stream)
    for _ in range(3):
        call()
    barrier(pg)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(args.steps):
        call()
    e.record(stream)
    barrier(pg)
    if pba.pba_last_device_error(stream) != pba.PBA_OK:
        raise RuntimeError("the output projection kernel recorded a device error")
    ms = max_over_ranks(s.elapsed_time(e), pg) / args.steps
    N2 = tcfg.N * tcfg.N
    nbytes = N2 * HD * 2 + N2 * tcfg.c * 2 + HD * tcfg.c * 2
    flops = 2.0 * N2 * HD * tcfg.c
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"ms_per_call": ms, "calls": args.steps, "gpu_launches": args.steps,
            "workload": f"tri{tcfg.N}: o [{tcfg.N},{tcfg.N},{tcfg.H},{tcfg.D}] bf16 -> out [N,N,{tcfg.c}]",
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "algorithmic_bytes_per_call": nbytes,
                         "kernel": "pba_oproj_sm100_kernel (tri_out_proj_forward)", "peak_source": peaks["source"],
                         "tensor_frac": (flops / (ms / 1e3) / 1e12) / peaks["bf16_tflops"]}}


def run_pwa(args, pba, dev, stream, pg, peaks, clk):
    """Pair weighted averaging on pwa4k (S=64 sequences, N=4096, H=8, D=32,
    gate, 5% key padding), timed on its own after the step: K calls after 3
    warm-up calls, CUDA events on the stream; a call is the row log-sum-exp
    pass and the weights-times-values kernel (2 launches).  Compute-bound:
    2*H*S*N^2*D FLOPs on the tensor cores; H*N^2 exps in the first pass and
    H*N^2 per 256-feature tile in the second on the exp2 unit (16 per clock
    per SM)."""
    cfg = W.PWA4K
    v, bias, mask, gate = W.pwa_inputs(cfg, dev)
    out = torch.empty_like(v)
    lse = torch.empty((cfg.H, cfg.N), dtype=torch.float32, device=dev)
    call = lambda: pba.pwa_forward(v, bias, mask, gate, out, lse, stream=stream)
    for _ in range(3):
        call()
    barrier(pg)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(args.steps):
        call()
    e.record(stream)
    barrier(pg)
    if pba.pba_last_device_error(stream) != pba.PBA_OK:
        raise RuntimeError("the pair weighted averaging kernel recorded a device error")
    ms = max_over_ranks(s.elapsed_time(e), pg) / args.steps
    flops = 2.0 * cfg.H * cfg.S * cfg.N * cfg.N * cfg.D
    ftiles = -(-cfg.S // (256 // cfg.D))
    exps = cfg.H * cfg.N * cfg.N * (ftiles + 1)
    tflops = flops / (ms / 1e3) / 1e12
    sm_hz = (clk.get("sm_mhz") or 1965.0) * 1e6 if isinstance(clk, dict) else 1965e6
    exp_floor_ms = exps / (16 * torch.cuda.get_device_properties(dev).multi_processor_count * sm_hz) * 1e3
    return {"ms_per_call": ms, "calls": args.steps, "gpu_launches": 2 * args.steps, "tflops": tflops,
            "workload": f"pwa4k: S={cfg.S} N={cfg.N} H={cfg.H} D={cfg.D}, gate, 5% key padding, bias [H,N,N]",
            "roofline": {"bound": "tensor", "achieved": tflops, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": tflops / peaks["bf16_tflops"], "kernel": "pba_pwa_sm100_kernel (pwa_forward)",
                         "peak_source": peaks["source"], "exp2_floor_ms": exp_floor_ms,
                         "exp2_frac": exp_floor_ms / ms}}


def run_bwd(args, pba, dev, stream, pg, peaks):
    """Backward of pair-biased attention on the ring8k shapes (N=8192, H=16,
    D=64, bf16, no mask), timed on its own after the step: forward once, then
    K backward calls after 2 warm-up calls, CUDA events on the stream.
    Algorithmic work: 10*B*H*N^2*D FLOPs (S recomputed, dP, dV, dQ, dK) and
    the bias read once plus dbias written, with Q, K, V, O, dO read and dQ,
    dK, dV (fp32) written once."""
    cfg = W.RING8K
    q, k, v, bias, mask = W.attn_inputs(cfg, dev)
    out, lse = pba.pba_forward(q, k, v, bias, mask, stream=stream)
    dout = torch.randn(q.shape, generator=torch.Generator(dev.type).manual_seed(11), device=dev).to(torch.bfloat16)
    call = lambda: pba.pba_backward(q, k, v, bias, mask, out, lse, dout, stream=stream)
    steps = max(3, args.steps // 6)
    for _ in range(2):
        call()
    barrier(pg)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(steps):
        call()
    e.record(stream)
    barrier(pg)
    if pba.pba_last_device_error(stream) != pba.PBA_OK:
        raise RuntimeError("a backward kernel recorded a device error")
    ms = max_over_ranks(s.elapsed_time(e), pg) / steps
    B, H, N, D = cfg.B, cfg.H, cfg.N, cfg.D
    flops = 10.0 * B * H * N * N * D
    nbytes = 2 * B * H * N * N * 2 + 5 * B * H * N * D * 2 + 3 * B * H * N * D * 4 + 2 * B * H * N * 4
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"ms_per_call": ms, "calls": steps, "gpu_launches": 3 * steps,
            "tflops_algorithmic": flops / (ms / 1e3) / 1e12,
            "workload": f"ring8k shapes: N={N} H={H} D={D} bf16, bias ~N(0,1); dq, dk, dv fp32, dbias bf16",
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "algorithmic_bytes_per_call": nbytes,
                         "kernel": "pba_bwd_sm100_kernel (pba_backward: dq/dbias and dk/dv kernels)",
                         "peak_source": peaks["source"],
                         "tensor_frac": (flops / (ms / 1e3) / 1e12) / peaks["bf16_tflops"]}}


# Nominal dense tf32 : bf16 tensor rate of the B200 (1.1 : 2.25 PFLOP/s): the
# tf32 peak is the measured bf16 peak times this ratio.
TF32_PER_BF16 = 1.1 / 2.25


def run_f32(args, pba, dev, stream, pg, peaks):
    """pba_forward with fp32 inputs on the ring8k shapes (N=8192, H=16, D=64,
    bias ~N(0,1), no mask), timed on its own after the step: K calls after 3
    warm-up calls, CUDA events on the stream; plus the pr1 config (fp32, N=256,
    H=4, D=32), which is a single wave of 8 CTAs and measures launch latency
    more than throughput.  The path runs three tf32 products per product
    (high and low parts of both operands), so its tensor-core work is three
    times the algorithmic 4*H*N^2*D FLOPs; that work is reported against the
    tf32 peak (the measured bf16 peak times the nominal tf32 : bf16 ratio)."""
    cfg = W.RING8K
    q, k, v, bias = (t.float() for t in W.attn_inputs(cfg, dev)[:4])
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)

    def timed(call, n):
        for _ in range(3):
            call()
        barrier(pg)
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        for _ in range(n):
            call()
        e.record(stream)
        barrier(pg)
        return max_over_ranks(s.elapsed_time(e), pg) / n

    ms = timed(lambda: pba.pba_forward(q, k, v, bias, None, out, lse, stream=stream), args.steps)
    del q, k, v, bias, out, lse
    pq, pk, pv, pb, _ = W.attn_inputs(W.PR1, dev)
    pout = torch.empty_like(pq)
    plse = torch.empty(pq.shape[:3], dtype=torch.float32, device=dev)
    pr1_ms = timed(lambda: pba.pba_forward(pq, pk, pv, pb, None, pout, plse, stream=stream), args.steps)
    if pba.pba_last_device_error(stream) != pba.PBA_OK:
        raise RuntimeError("the fp32 attention kernel recorded a device error")
    flops = attn_flops(cfg.B, cfg.H, cfg.N, cfg.N, cfg.D)
    alg = flops / (ms / 1e3) / 1e12
    peak = peaks["bf16_tflops"] * TF32_PER_BF16
    return {"ms_per_call": ms, "calls": args.steps, "gpu_launches": args.steps, "tflops_algorithmic": alg,
            "workload": f"ring8k shapes in fp32: N={cfg.N} H={cfg.H} D={cfg.D}, bias ~N(0,1), no mask",
            "pr1_ms_per_call": pr1_ms,
            "roofline": {"bound": "tensor", "achieved": 3 * alg, "peak": peak, "unit": "TFLOP/s",
                         "frac": 3 * alg / peak, "kernel": "pba_attn_tf32_sm100_kernel (pba_forward, fp32)",
                         "peak_source": peaks["source"] + " bf16 x 1.1/2.25",
                         "note": "achieved = tf32 tensor-core work, 3x the algorithmic FLOPs"}}


def per_call_ms(call, n, stream, pg, flush=None):
    """Median over n calls of one call's CUDA-event time on the stream, after
    3 warm-up calls.  With `flush` (a buffer larger than L2) rewritten before
    each call, no input is left in L2 by the call before."""
    for _ in range(3):
        call()
    barrier(pg)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for i, (s, e) in enumerate(ev):
        if flush is not None:
            flush.fill_(i & 0xFF)
        s.record(stream)
        call()
        e.record(stream)
    barrier(pg)
    return max_over_ranks(statistics.median(s.elapsed_time(e) for s, e in ev), pg)


def run_configs(args, pba, dev, stream, pg, peaks, line, clk):
    """Each workload of the benchmark plan on its own: ms per call (median of
    20 calls, each after a 256 MB L2 flush), TFLOP/s, GB/s and the roofline
    fraction; for triangle attention also pair-tensor rows/s (lines of the
    pair tensor) and softmax rows/s (one per line, query and head).  pr1,
    apb2k and tri512 are timed here; ring8k, large16k and tri1024 repeat the
    figures of their own entries of the line."""
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    n = 20
    res = {}

    # pr1: fp32, one pass and the four 64-key blocks merged
    cfg = W.PR1
    q, k, v, b, _ = W.attn_inputs(cfg, dev)
    B, H, N, D, P = cfg.B, cfg.H, cfg.N, cfg.D, cfg.blocks
    out, lse = torch.empty_like(q), torch.empty((B, H, N), dtype=torch.float32, device=dev)
    ms = per_call_ms(lambda: pba.pba_forward(q, k, v, b, None, out, lse, stream=stream), n, stream, pg, flush)
    L = N // P
    o_p = torch.empty((P, B, H, N, D), dtype=torch.float32, device=dev)
    m_p, l_p = torch.empty((P, B, H, N), dtype=torch.float32, device=dev), torch.empty((P, B, H, N), dtype=torch.float32, device=dev)
    mout, mlse = torch.empty_like(out), torch.empty_like(lse)
    views = [(k[:, :, j * L:(j + 1) * L], v[:, :, j * L:(j + 1) * L], b[..., j * L:(j + 1) * L]) for j in W.block_order(cfg)]

    def blocks():
        for slot, (kb, vb, bb) in enumerate(views):
            pba.pba_partial(q, kb, vb, bb, None, o_p[slot], m_p[slot], l_p[slot], stream=stream)
        pba.softmax_merge(o_p, m_p, l_p, out_dtype=torch.float32, out=mout, lse=mlse, stream=stream)

    ms_blocks = per_call_ms(blocks, n, stream, pg, flush)
    flops = attn_flops(B, H, N, N, D)
    res["pr1"] = {"ms_per_call": ms, "tflops": flops / (ms / 1e3) / 1e12,
                  "gbs": attn_bytes(B, H, N, N, D, elt=4, mask=False) / (ms / 1e3) / 1e9,
                  "ms_4_blocks_and_merge": ms_blocks, "gpu_launches_per_call": 1,
                  "bound": "launch (one wave of 8 CTAs; the roofline floors are below 2 us)",
                  "workload": "pr1: fp32 N=256 H=4 D=32, no mask; also 4 key blocks of 64 in seeded order + merge"}
    del q, k, v, b, out, lse, o_p, m_p, l_p, mout, mlse, views

    # apb2k: bf16, last 10 % of the keys masked
    cfg = W.APB2K
    q, k, v, b, mask = W.attn_inputs(cfg, dev)
    B, H, N, D = cfg.B, cfg.H, cfg.N, cfg.D
    out, lse = torch.empty_like(q), torch.empty((B, H, N), dtype=torch.float32, device=dev)
    ms = per_call_ms(lambda: pba.pba_forward(q, k, v, b, mask, out, lse, stream=stream), n, stream, pg, flush)
    flops, nbytes = attn_flops(B, H, N, N, D), attn_bytes(B, H, N, N, D)
    n_valid = int(mask[0].sum().item())
    res["apb2k"] = {"ms_per_call": ms, "tflops": flops / (ms / 1e3) / 1e12,
                    "tflops_valid_keys": flops * n_valid / N / (ms / 1e3) / 1e12, "valid_keys": n_valid,
                    "gbs": nbytes / (ms / 1e3) / 1e9,
                    "roofline": roofline_entry(flops, nbytes, ms / 1e3, peaks, None, "pba_attn_sm100_kernel (pba_forward, apb2k)"),
                    "workload": "apb2k: bf16 N=2048 H=16 D=64, bias ~N(0,2), last 204 keys masked"}
    del q, k, v, b, mask, out, lse

    # tri512: both orientations, gate on
    tcfg = W.TRI512
    tq, tk, tv, tg, tb = W.tri_inputs(tcfg, dev)
    tout = torch.empty_like(tq)
    tlse = torch.empty((tcfg.N, tcfg.N, tcfg.H), dtype=torch.float32, device=dev)
    sm_mhz = (clk.get("sm_mhz") or 1965.0) if isinstance(clk, dict) else 1965.0
    n_sms = torch.cuda.get_device_properties(dev).multi_processor_count
    tri = {}
    for orient in ("starting", "ending"):
        ms = per_call_ms(lambda: pba.tri_attn_forward(tq, tk, tv, tb, tg, None, orient, tout, tlse, stream=stream),
                         n, stream, pg, flush)
        tri[orient] = tri_ceilings(tcfg.N, tcfg.H, tcfg.D, ms, peaks["bf16_tflops_sustained"], peaks["hbm_gbs"],
                                   sm_mhz, n_sms)
        tri[orient]["pair_rows_per_s"] = tcfg.N / (ms / 1e3)
        tri[orient]["softmax_rows_per_s"] = tcfg.N * tcfg.N * tcfg.H / (ms / 1e3)
        tri[orient]["tflops"] = tri[orient]["flops_per_call"] / (ms / 1e3) / 1e12
    tri["workload"] = "tri512: pair tensor N=512 c=128, H=4 D=32 bf16, gate on, no pair mask"
    res["tri512"] = tri
    del tq, tk, tv, tg, tb, tout, tlse

    r8 = line.get("ring8k", {})
    res["ring8k"] = {k2: r8.get(k2) for k2 in ("partials_ms", "merge_ms_l2_flushed", "pba_forward_ms_same_shape",
                                               "partials_tflops")}
    res["ring8k"]["partials_frac"] = r8.get("partials_roofline", {}).get("frac")
    res["ring8k"]["merge_frac"] = r8.get("merge_roofline", {}).get("frac")
    rl = line["roofline"]
    res["large16k"] = {"ms_per_call": line["pba_ms_per_launch"], "tflops": line["value"],
                       "gbs": rl["hbm_frac"] * peaks["hbm_gbs"], "frac": rl["frac"], "bound": rl["bound"]}
    t1 = W.TRI1024
    ms = line["tri_attn_ms_per_call"]
    res["tri1024"] = {"ms_per_call": ms, "tflops": line["tri_attn_ceilings"]["flops_per_call"] / (ms / 1e3) / 1e12,
                      "pair_rows_per_s": t1.N / (ms / 1e3), "softmax_rows_per_s": t1.N * t1.N * t1.H / (ms / 1e3),
                      "frac": line["tri_attn_ceilings"]["frac"]}
    res["timing"] = f"median of {n} calls, CUDA events, 256 MB L2 flush before each call (pr1, apb2k, tri512)"
    if pba.pba_last_device_error(stream) != pba.PBA_OK:
        raise RuntimeError("a kernel recorded a device error in the per-workload timings")
    return res


def oracle_per_config(dev, large_tflops, large_cores):
    """The fp64 oracle's rate on every workload of the benchmark plan, in
    softmax rows per second (a row = one query of one head, against all its
    keys), on the host cores: pr1 and apb2k in full, the others on seeded
    samples that include the tile-boundary rows (ring8k 512 query rows of
    every head, tri512 16 lines, tri1024 8 lines); large16k from the
    cpu_baseline sample.  Inputs are converted to fp64 before each timed
    call.  The full-size time of a sampled workload is extrapolated and
    labelled so."""
    import numpy as np

    import oracle

    f64 = lambda t: np.ascontiguousarray(t.detach().cpu().double().numpy())
    u8 = lambda t: None if t is None else np.ascontiguousarray(t.detach().cpu().numpy().astype(np.uint8))
    res = {}

    def timed(fn):
        t0 = time.perf_counter()
        fn()
        return time.perf_counter() - t0

    for cfg in (W.PR1, W.APB2K, W.RING8K):
        q, k, v, b, mask = W.attn_inputs(cfg, dev)
        B, H, N = cfg.B, cfg.H, cfg.N
        if cfg is W.RING8K:
            rows = torch.as_tensor(W.sample_rows(N, 512, seed=3), device=dev)
            q, b = q.index_select(2, rows), b.index_select(2, rows)
        args = (f64(q), f64(k), f64(v), f64(b), u8(mask))
        nrows = B * H * args[0].shape[2]
        t = timed(lambda: oracle.pba(*args))
        e = {"softmax_rows_per_s": nrows / t, "rows": nrows, "seconds": t}
        if cfg is W.RING8K:
            e["extrapolated_full_s"] = B * H * N * t / nrows
            e["sample"] = "512 query rows (incl. 0, 127, 128, 255, 8191) of every head, all 8192 keys"
        else:
            e["sample"] = "full"
        res[cfg.name] = e
        del q, k, v, b, mask, args
    for tcfg, count in ((W.TRI512, 16), (W.TRI1024, 8)):
        tq, tk, tv, tg, tb = W.tri_inputs(tcfg, dev)
        lines = torch.as_tensor(W.sample_rows(tcfg.N, count, seed=tcfg.seed), device=dev)
        sel = lambda x: f64(x.index_select(0, lines))
        args = (sel(tq), sel(tk), sel(tv), f64(tb), sel(tg))
        t = timed(lambda: oracle.tri_attn_lines(*args))
        nrows = count * tcfg.N * tcfg.H
        res[tcfg.name] = {"softmax_rows_per_s": nrows / t, "pair_rows_per_s": count / t, "rows": nrows,
                          "seconds": t, "extrapolated_full_s_per_orientation": tcfg.N * t / count,
                          "sample": f"{count} starting-node lines (incl. 0, 127, 128, 255, {tcfg.N - 1})"}
        del tq, tk, tv, tg, tb, args
    L = W.LARGE16K
    res["large16k"] = {"softmax_rows_per_s": large_tflops * 1e12 / (4.0 * L.N * L.D),
                       "extrapolated_full_s": L.B * L.H * L.N * 4.0 * L.N * L.D / (large_tflops * 1e12),
                       "sample": "the cpu_baseline sample"}
    res["cores"] = large_cores
    return res


def merge_bytes(P, rows, D, out_elt=2):
    """Algorithmic bytes of softmax_merge: the P partials (O_p fp32, m_p, l_p)
    read once, out and lse written once."""
    return P * rows * (4 * D + 8) + rows * (out_elt * D + 4)


def run_ring8k(args, pba, dev, stream, pg, peaks):
    """The ring-step emulation on one GPU (ring8k: N=8192, H=16, D=64, bf16,
    bias ~N(0,1), no mask): P=8 pba_partial calls over key blocks of 1024 in
    randperm(8) order, each into its slot of one preallocated [8,B,H,N,D]
    buffer, then softmax_merge into bf16 out and the lse.  The partials and the
    merge are timed in their own CUDA-event regions; the merge also alone,
    after an L2 flush each time (its 277 MB input otherwise partly sits in L2
    from the last partial).  pba_forward at the same shape is timed beside."""
    cfg = W.RING8K
    q, k, v, bias, mask = W.attn_inputs(cfg, dev)
    B, H, N, D, P = cfg.B, cfg.H, cfg.N, cfg.D, cfg.blocks
    L = N // P
    order = W.block_order(cfg)
    o_parts = torch.empty((P, B, H, N, D), dtype=torch.float32, device=dev)
    m_parts = torch.empty((P, B, H, N), dtype=torch.float32, device=dev)
    l_parts = torch.empty_like(m_parts)
    out = torch.empty((B, H, N, D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    views = [(k[:, :, b * L:(b + 1) * L], v[:, :, b * L:(b + 1) * L], bias[..., b * L:(b + 1) * L]) for b in order]

    def partials():
        for slot, (kb, vb, bb) in enumerate(views):
            pba.pba_partial(q, kb, vb, bb, None, o_parts[slot], m_parts[slot], l_parts[slot], stream=stream)

    merge = lambda: pba.softmax_merge(o_parts, m_parts, l_parts, out_dtype=torch.bfloat16, out=out, lse=lse,
                                      stream=stream)
    fwd_out, fwd_lse = torch.empty_like(out), torch.empty_like(lse)
    fwd = lambda: pba.pba_forward(q, k, v, bias, None, fwd_out, fwd_lse, stream=stream)
    for _ in range(3):
        partials()
        merge()
        fwd()
    barrier(pg)
    steps = max(3, args.steps // 4)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for i in range(steps):
        ev[i][0].record(stream)
        partials()
        ev[i][1].record(stream)
        merge()
        ev[i][2].record(stream)
    fs, fe = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    fs.record(stream)
    for _ in range(steps):
        fwd()
    fe.record(stream)
    # the merge alone, L2 flushed before each call
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    mev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    for i in range(steps):
        flush.fill_(i & 0xFF)
        mev[i][0].record(stream)
        merge()
        mev[i][1].record(stream)
    barrier(pg)
    if pba.pba_last_device_error(stream) != pba.PBA_OK:
        raise RuntimeError("a ring-step kernel recorded a device error")
    part_ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ev), pg) / steps
    merge_ms = max_over_ranks(sum(e[1].elapsed_time(e[2]) for e in ev), pg) / steps
    merge_cold_ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in mev), pg) / steps
    fwd_ms = max_over_ranks(fs.elapsed_time(fe), pg) / steps
    flops = attn_flops(B, H, N, N, D)
    # partials: every block reads its bias columns, Q, its K/V block; writes O_p fp32, m_p, l_p
    part_bytes = B * H * N * N * 2 + P * B * H * N * D * 2 + 2 * B * H * N * D * 2 + P * B * H * N * (4 * D + 8)
    mbytes = merge_bytes(P, B * H * N, D)
    return {"partials_ms": part_ms, "merge_ms_in_step": merge_ms, "merge_ms_l2_flushed": merge_cold_ms,
            "pba_forward_ms_same_shape": fwd_ms, "steps": steps, "gpu_launches": steps * (P + 1),
            "workload": f"ring8k: N={N} H={H} D={D} bf16, P={P} key blocks of {L} in order {order}, "
                        f"partials into one preallocated [P,B,H,N,D] buffer, then softmax_merge",
            "partials_tflops": flops / (part_ms / 1e3) / 1e12,
            "partials_roofline": roofline_entry(flops, part_bytes, part_ms / 1e3, peaks, None,
                                                "pba_attn_sm100_kernel (pba_partial x 8)"),
            "merge_roofline": {"bound": "hbm", "achieved": mbytes / (merge_cold_ms / 1e3) / 1e9,
                               "peak": peaks["hbm_gbs"], "unit": "GB/s",
                               "frac": mbytes / (merge_cold_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                               "algorithmic_bytes_per_call": mbytes, "kernel": "softmax_merge_kernel",
                               "peak_source": peaks["source"],
                               "in_step_gbs": mbytes / (merge_ms / 1e3) / 1e9}}


def run_e2e(args, pba, cfg, q, k, v, bias, mask, out, lse, stream, pg, world, flops):
    """Same metric through the public call with the inputs starting in pinned
    host memory and the outputs read back each step."""
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    hb = torch.empty(bias.shape, dtype=bias.dtype, pin_memory=True)
    hb.copy_(bias)
    hm = mask.cpu().pin_memory()
    ho = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    hl = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hb, hm))
    d2h = ho.numel() * ho.element_size() + hl.numel() * hl.element_size()

    def e2e_step():
        q.copy_(hq, non_blocking=True)
        k.copy_(hk, non_blocking=True)
        v.copy_(hv, non_blocking=True)
        bias.copy_(hb, non_blocking=True)
        mask.copy_(hm, non_blocking=True)
        pba.pba_forward(q, k, v, bias, mask, out, lse, stream=stream)
        ho.copy_(out, non_blocking=True)
        hl.copy_(lse, non_blocking=True)

    e2e_step()
    barrier(pg)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    e.record(stream)
    barrier(pg)
    t = max_over_ranks(s.elapsed_time(e), pg)
    assert torch.isfinite(hl[hl > -math.inf]).all()
    return {"value": world * flops * args.e2e_steps / (t / 1e3) / 1e12, "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": args.e2e_steps}


def run_profile_case(args, pba, dev):
    """One small case for ncu, each kernel launched twice (a warm-up launch,
    then the captured one): pba4k = pba_forward at N=4096 (bias 512 MB, larger
    than L2); merge8k = softmax_merge of the ring8k partials (L2 flushed
    before each merge); tri512 = triangle attention N=512 both orientations; proj1024 /
    oproj1024 = the input / output projections at tri1024; pwa4k = pwa_forward;
    bwd4k = pba_backward at N=4096, H=4; f32_4k = pba_forward with fp32 inputs
    at N=4096, H=16, D=64 (bias 1 GB)."""
    if args.profile == "merge8k":
        cfg = W.RING8K
        q, k, v, bias, _ = W.attn_inputs(cfg, dev)
        P, L = cfg.blocks, cfg.N // cfg.blocks
        o_parts = torch.empty((P,) + tuple(q.shape), dtype=torch.float32, device=dev)
        m_parts = torch.empty((P,) + tuple(q.shape[:3]), dtype=torch.float32, device=dev)
        l_parts = torch.empty_like(m_parts)
        for slot, b in enumerate(W.block_order(cfg)):
            sl = slice(b * L, (b + 1) * L)
            pba.pba_partial(q, k[:, :, sl], v[:, :, sl], bias[..., sl], None, o_parts[slot], m_parts[slot],
                            l_parts[slot])
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        for i in range(2):
            flush.fill_(i)
            pba.softmax_merge(o_parts, m_parts, l_parts, out_dtype=torch.bfloat16)
    elif args.profile == "bwd4k":
        q, k, v, bias, mask = W.random_attn(1, 4, 4096, 4096, 64, seed=12, device=dev, mask_frac=0.05)
        out, lse = pba.pba_forward(q, k, v, bias, mask)
        dout = torch.randn(q.shape, generator=torch.Generator(dev.type).manual_seed(13), device=dev).to(torch.bfloat16)
        for _ in range(2):
            pba.pba_backward(q, k, v, bias, mask, out, lse, dout)
    elif args.profile == "pwa4k":
        v, bias, mask, gate = W.pwa_inputs(W.PWA4K, dev)
        for _ in range(2):
            pba.pwa_forward(v, bias, mask, gate)
    elif args.profile == "proj1024":
        z, w, wb = W.tri_pair_inputs(W.TRI1024, dev)
        for _ in range(2):
            pba.tri_proj_forward(z, w, wb, W.TRI1024.H)
    elif args.profile == "oproj1024":
        cfg = W.TRI1024
        g = torch.Generator(dev.type).manual_seed(cfg.seed + 100)
        o = torch.randn((cfg.N, cfg.N, cfg.H, cfg.D), generator=g, device=dev).to(torch.bfloat16)
        w_o = (torch.randn((cfg.H * cfg.D, cfg.c), generator=g, device=dev) / (cfg.H * cfg.D) ** 0.5).to(torch.bfloat16)
        for _ in range(2):
            pba.tri_out_proj_forward(o, w_o)
    elif args.profile == "f32_4k":
        q, k, v, bias, _ = W.random_attn(1, 16, 4096, 4096, 64, dtype=torch.float32, seed=1, device=dev)
        for _ in range(2):
            pba.pba_forward(q, k, v, bias)
    elif args.profile == "pba4k":
        cfg = W.AttnConfig("pba4k", B=1, N=4096, H=16, D=64, dtype=torch.bfloat16, seed=4, mask="random5")
        q, k, v, bias, mask = W.attn_inputs(cfg, dev)
        for _ in range(2):
            pba.pba_forward(q, k, v, bias, mask)
    else:
        q, k, v, g, b = W.tri_inputs(W.TRI512, dev)
        for _ in range(2):
            pba.tri_attn_forward(q, k, v, b, g, None, "starting")
            pba.tri_attn_forward(q, k, v, b, g, None, "ending")
    torch.cuda.synchronize()
    assert pba.pba_last_device_error() == pba.PBA_OK
    print(f"profile case {args.profile} done")
    return 0


if __name__ == "__main__":
    sys.exit(main())
