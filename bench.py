#!/usr/bin/env python
"""Bench of the ReLU linear-attention forward at the 4096px Sana shape.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

One step = the whole forward (state phi(K)^T[V|1] over all tokens, fixed-order
chunk reduction, apply phi(Q)S and normalise) over one synthetic batch of the
4096px workload: B=2 (CFG pair), N=16384 tokens (128x128 latent), H=70, d=32,
bf16 Q/K/V, bf16 output. Inputs are 440 MB and the output 147 MB per step, more
than the 126 MB L2, so no explicit L2 flush is done between steps.

Prints one JSON line (rank 0). `value` is GB/s of algorithmic traffic (Q, K, V
read once, O written once) over the device-timed steps, summed over ranks and
divided by the slowest rank's time. Multi-GPU runs give every rank its own
4096px problem (independent batches: weak scaling, no data-path collective);
`--scaling strong` splits one problem over the ranks instead, by batches and
then by ranges of whole head groups (still no collective: the (b, h) problems
are independent), and `value` is that one problem's bytes over the slowest
rank's time.

`--impl reference` times the fp64 CPU oracle (the only reference there is) on
bounded samples of the same workload, on the host cores, rank 0 only.

`--workload` selects another named workload (other sizes, the ELU+1 and cos
feature maps, the block-causal video shapes). `--op kvproj` times the key-value
projection with the state in its epilogue and `--op mixffn` the Mix-FFN, each
next to the unfused pipeline it replaces (one GPU, TFLOP/s).
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ReLU linear-attn GB/s (% of B200 HBM peak) and Mtokens/s at 4096px shape"
UNIT = "GB/s"
WORKLOAD = "4096px"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
# dram__bytes_read.sum + dram__bytes_write.sum per launch from an ncu capture of
# the same build and workload, keyed by (kernel set, workload, kernel, output
# bytes per element); absent when the kernels changed since the counters were
# taken
TRAFFIC_PER_LAUNCH = {
    # fwd_fused_tc at 4096px, bf16 out: 440.70 MB read + 90.81 MB written
    ("tcgen05-tma", "4096px", "fwd_fused_tc", 2): 531.52e6,
}
SMS = 148
FP32_LANES_PER_SM = 128


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=5000,
                   help="timed steps (about 1 s at 4096px, long enough to sample clocks)")
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--op", choices=["forward", "kvproj", "mixffn"], default="forward",
                   help="kvproj: the key-value projection with the state in its epilogue (one GPU), "
                        "against a cuBLAS projection followed by kv_state; mixffn: the Mix-FFN after "
                        "the attention (one GPU), against torch (cuBLAS + cuDNN depthwise conv)")
    p.add_argument("--e2e-steps", type=int, default=10)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--workload", default=WORKLOAD,
                   help="named workload (profiling runs use smaller ones; the bench line is 4096px)")
    p.add_argument("--cpu-seconds", type=float, default=12.0,
                   help="target CPU time of the oracle baseline sample")
    p.add_argument("--scaling", choices=["weak", "strong"], default="weak",
                   help="weak: every rank its own batch of the workload; strong: one workload split "
                        "over the ranks by batches and head groups (no data-path collective)")
    args = p.parse_args(argv)
    if args.warmup < 3:
        p.error("--warmup must be >= 3")
    if args.steps < 1:
        p.error("--steps must be >= 1")
    return args


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d.get("sm_max_mhz", 1965.0)), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, 1965.0, "fallback"


# ------------------------------------------------------------ distributed --

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(x: float, device=None) -> float:
    """Largest value of x over all ranks (identity when not distributed)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard(world: int, rank: int, B: int, H: int, G: int):
    """Strong scaling: the batches [b0, b1) and heads [h0, h1) of rank `rank`
    when one job of B batches of H heads is split over `world` GPUs. Whole
    batches when world divides B; when world = k B, each batch is split into k
    ranges of whole head groups (G heads each, one slab of the kernels). The
    (b, h) problems are independent, so the ranks exchange nothing."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of {world}")
    if B % world == 0:
        per = B // world
        return rank * per, (rank + 1) * per, 0, H
    if world % B == 0:
        k = world // B
        groups = -(-H // G)
        if groups < k:
            raise ValueError(f"{H} heads ({groups} groups of {G}) cannot be split {k} ways")
        b, j = divmod(rank, k)
        g0, g1 = j * groups // k, (j + 1) * groups // k
        return b, b + 1, g0 * G, min(g1 * G, H)
    raise ValueError(f"{world} GPUs neither divide {B} batches nor are a multiple of them")


def rank_workload(w, world: int, rank: int, scaling: str):
    """This rank's workload and its (b0, b1, h0, h1) part of the job (None for
    weak scaling, where every rank runs the whole workload `w`)."""
    if scaling != "strong" or world == 1:
        return w, None
    part = shard(world, rank, w.B, w.H, 128 // w.d)
    b0, b1, h0, h1 = part
    return dataclasses.replace(w, name=f"{w.name}[b{b0}:{b1},h{h0}:{h1}]", B=b1 - b0, H=h1 - h0), part


def aggregate_gbs(bytes_per_rank: int, world: int, max_seconds: float) -> float:
    """Whole-job GB/s: all ranks' bytes over the slowest rank's time."""
    return bytes_per_rank * world / max_seconds / 1e9


# ---------------------------------------------------------------- clocks --

class ClockSampler:
    """nvidia-smi clock and throttle-reason samples during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.5)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [r.split(",") for r in self.file.read().strip().splitlines() if r.strip()]
        os.unlink(self.file.name)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [x.strip() for x in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                smax.append(float(r[2]))
            except ValueError:
                continue
            for name, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        busy = [s for s in sm if smax and s > 0.5 * max(smax)] or sm
        return {"sm_mhz": statistics.median(busy) if busy else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------- CPU oracle --

def input_generator(w) -> str:
    """Where the workload's inputs are drawn: the seeded CUDA generator for the
    largest shapes (a host draw of billions of values takes minutes), else the
    host generator."""
    import torch
    big = w.token_heads * w.d * 3 > 2_000_000_000
    return "cuda" if big and torch.cuda.is_available() else "cpu"


def oracle_sample(w, seconds: float, max_heads: int | None = None):
    """Time the fp64 oracle (as it stands) on whole heads of workload w, all N
    tokens each, adding heads until about `seconds` of CPU work is done.
    Returns (GB/s, Mtokens/s, threads, sample description, seconds)."""
    import numpy as np
    import torch
    from oracle import default
    from linear_attention_diffusion_relu_b200.workloads import make_inputs
    orc = default()
    Q, K, V = (t.cpu() for t in make_inputs(w, generator_device=input_generator(w)))   # bf16
    pairs = [(b, h) for b in range(w.B) for h in range(w.H)]
    if max_heads is not None:
        pairs = pairs[:max_heads]
    done, elapsed = [], 0.0
    step = 2
    while done != pairs and elapsed < seconds:
        batch = pairs[len(done):len(done) + step]
        sl = [(torch.stack([t[b, :, h, :] for b, h in batch], dim=1)[None]
               .to(torch.float64).numpy()) for t in (Q, K, V)]
        t0 = time.perf_counter()
        if w.block:
            O = orc.block_causal_apply(sl[0], orc.block_causal_state(sl[1], sl[2], w.block), w.block, w.eps)
        elif w.feature != "relu":
            O = orc.apply_fm(sl[0], orc.state_fm(sl[1], sl[2], w.feature), w.feature, w.eps)
        else:
            O = orc.apply(sl[0], orc.state(sl[1], sl[2]), w.eps)
        elapsed += time.perf_counter() - t0
        assert np.isfinite(O).all()
        done += batch
        step = min(step * 2, 16)
    token_heads = len(done) * w.N
    nbytes = token_heads * w.d * (3 * 2 + 2)
    desc = (f"{w.name}: {len(done)} of {w.B * w.H} (b,h) pairs, all {w.N} tokens each "
            f"({token_heads} token-heads), fp64 oracle state+apply"
            + (f", block-causal L={w.block}" if w.block else ""))
    return nbytes / elapsed / 1e9, token_heads / w.H / elapsed / 1e6, orc.num_threads(), desc, elapsed


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    from linear_attention_diffusion_relu_b200.workloads import WORKLOADS
    w = WORKLOADS[args.workload]
    per_step = max(2.0, min(20.0, 150.0 / (args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(w, per_step / 4, max_heads=2)
    vals, mts, secs = [], [], []
    desc, cores = "", 0
    for _ in range(args.steps):
        gbs, mtok, cores, desc, s = oracle_sample(w, per_step)
        vals.append(gbs)
        mts.append(mtok)
        secs.append(s)
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * statistics.median(secs), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "mtokens_per_s": statistics.median(mts),
        "config": {"workload": w.name, "B": w.B, "N": w.N, "H": w.H, "d": w.d,
                   "sample_per_step": desc},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- GPU arm --

def run_ours(args):
    import torch
    import torch.distributed as dist
    from linear_attention_diffusion_relu_b200 import ops
    from linear_attention_diffusion_relu_b200.workloads import WORKLOADS, make_inputs

    world, rank, local = dist_env()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", device_id=dev, timeout=timedelta(seconds=120))
    ops.load_library()

    w = WORKLOADS[args.workload]
    # the whole job: weak scaling, one workload per rank; strong, one workload
    # split over the ranks (this rank's part becomes `w`)
    strong = args.scaling == "strong"
    job = w
    job_copies = 1 if strong else world
    w, part = rank_workload(job, world, rank, args.scaling)
    B, N, H, d, L = w.B, w.N, w.H, w.d, w.block
    Q, K, V = make_inputs(w, device=dev, generator_device=input_generator(w))
    if rank > 0 and not strong:   # every rank its own independent batch of the same shape
        Q, K, V = (t.roll(shifts=rank, dims=1).contiguous() for t in (Q, K, V))
    out = torch.empty((B, N, H, d), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    if L:   # block-causal: prefix states of blocks of L tokens
        state = torch.empty((B, H, ops.num_blocks(N, L), d, d + 1), dtype=torch.float32, device=dev)
        ws = ops.make_block_causal_workspace(B, N, H, d, L, dev)
    else:
        state = torch.empty((B, H, d, d + 1), dtype=torch.float32, device=dev)
        ws = ops.make_workspace(B, N, H, d, dev)

    fm = w.feature
    if L and fm != "relu":
        raise SystemExit("the block-causal form runs with phi = ReLU only")

    def step():
        if L:
            ops.block_causal_forward(Q, K, V, L, out_dtype=torch.bfloat16, eps=w.eps, out=out, workspace=ws)
        else:
            ops.forward(Q, K, V, out_dtype=torch.bfloat16, eps=w.eps, out=out, workspace=ws, feature_map=fm)

    def split_step(ev):
        ev[0].record(stream)
        if L:
            ops.block_causal_kv_state(K, V, L, states=state, workspace=ws)
        else:
            ops.kv_state(K, V, state=state, workspace=ws, feature_map=fm)
        ev[1].record(stream)
        if L:
            ops.block_causal_apply(Q, state, L, out_dtype=torch.bfloat16, eps=w.eps, out=out)
        else:
            ops.apply(Q, state, out_dtype=torch.bfloat16, eps=w.eps, out=out, feature_map=fm)
        ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()

    # ---- timed region: K forward passes
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    start.record(stream)
    for k in range(args.steps):
        step()
    end.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    ms = start.elapsed_time(end) / args.steps
    ms_max = max_over_ranks(ms, dev)
    # the per-step distribution from a second loop with an event between
    # steps (an event record between two launches adds ~2 us at the small
    # shapes, so the timed region above has none)
    per_step = per_step_times(step, stream, min(args.steps, 1000))
    bytes_per_step = w.algorithmic_bytes(2)
    # whole-job bytes and tokens over the slowest rank's time
    value = aggregate_gbs(job.algorithmic_bytes(2), job_copies, ms_max / 1e3)
    mtok = job.B * job.N * job_copies / (ms_max / 1e3) / 1e6

    # ---- breakdown: the same phases as separate kernels through the two-call
    # API, with events between the state half and the apply half
    n_split = min(args.steps, 2000)
    for _ in range(3):
        split_step([torch.cuda.Event(enable_timing=True) for _ in range(3)])
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n_split)]
    torch.cuda.synchronize(dev)
    for i in range(n_split):
        split_step(events[i])
    torch.cuda.synchronize(dev)
    ks_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in events)
    ka_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in events)
    hbm_peak, sm_max_mhz, peak_src = measured_peaks()
    impl = ops.implementation()
    launches = ops.block_causal_forward_launches(B, N, H, d, L) if L else ops.forward_launches(B, N, H, d)
    if launches == 1:
        # the step is one launch of fwd_fused_tc: its average launch duration
        # is the timed region's time per step
        dom, dom_ms, dom_bytes = "fwd_fused_tc", ms, bytes_per_step
    else:   # three-kernel forward: the larger half (128 B per token-head each)
        half_bytes = w.token_heads * d * 4
        halves = {"kv_state(KS+KR)": ks_ms, "apply(KA)": ka_ms}
        dom = max(halves, key=halves.get)
        dom_ms, dom_bytes = halves[dom], half_bytes
    if impl["bound"] == "alu":
        flops = w.token_heads * 2 * d * (d + 1)
        achieved = flops / (dom_ms / 1e3) / 1e12
        peak = SMS * FP32_LANES_PER_SM * 2 * sm_max_mhz * 1e6 / 1e12
        roof = {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": None, "kernel": dom,
                "peak_source": "FP32 FFMA: 148 SMs x 128 lanes x 2 flop x max SM clock"}
    else:
        achieved = dom_bytes / (dom_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                "frac": achieved / hbm_peak, "traffic": TRAFFIC_PER_LAUNCH.get((impl["name"], w.name, dom, 2)),
                "kernel": dom, "peak_source": f"{peak_src} copy bandwidth (burst)"}
    roof["ms_per_launch"] = dom_ms
    roof["algorithmic_bytes_per_launch"] = dom_bytes
    if launches == 1:
        roof["ms_per_launch_median"] = statistics.median(per_step)
        roof["ms_per_launch_min"] = min(per_step)
    roof["split_api_ms"] = {"kv_state(KS+KR)": ks_ms, "apply(KA)": ka_ms}
    roof["timing"] = ("launch duration: CUDA events over the timed region / steps (one launch per "
                      "step); median and min: per-step events in a second loop of "
                      f"{min(args.steps, 1000)} steps; split_api_ms: events around kv_state and apply in a "
                      f"{n_split}-step loop of the two-call API after the timed region")

    fp32 = None if L else run_fp32_out(args, w, Q, K, V, ws, dev, stream, job, job_copies, hbm_peak, peak_src,
                                       impl)

    # block-causal: the one-launch form (bit-identical), timed the same way
    single = None
    if L:
        def single_step():
            ops.block_causal_forward(Q, K, V, L, out_dtype=torch.bfloat16, eps=w.eps, out=out, workspace=ws,
                                     single_launch=True)
        n_single = min(args.steps, 200)
        for _ in range(args.warmup):
            single_step()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(n_single + 1)]
        torch.cuda.synchronize(dev)
        ev[0].record(stream)
        for k in range(n_single):
            single_step()
            ev[k + 1].record(stream)
        torch.cuda.synchronize(dev)
        per = [ev[k].elapsed_time(ev[k + 1]) for k in range(n_single)]
        s_ms = ev[0].elapsed_time(ev[-1]) / n_single
        s_gbs = bytes_per_step / (s_ms / 1e3) / 1e9
        single = {"ms_per_step": s_ms, "ms_per_step_median": statistics.median(per), "ms_per_step_min": min(per),
                  "value": s_gbs, "unit": UNIT, "frac": s_gbs / hbm_peak, "steps": n_single,
                  "kernel": "fwd_fused_tc (block-causal instance)",
                  "gpu_launches": ops.block_causal_forward_launches(B, N, H, d, L, single_launch=True) * n_single,
                  "call": "block_causal_forward_single"}

    e2e = None if args.no_e2e else run_e2e(args, w, dev, stream, job, job_copies)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        gbs, mt, cores, desc, _ = oracle_sample(w, args.cpu_seconds)
        cpu = {"value": gbs, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc,
               "mtokens_per_s": mt}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
            "higher_is_better": True, "scaling": args.scaling, "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "mtokens_per_s": mtok, "pct_of_hbm_peak": 100.0 * value / (hbm_peak * world),
            "config": {"workload": job.name, "B": job.B, "N": N, "H": job.H, "d": d,
                       **({"form": "block-causal", "block": L} if L else {}),
                       **({"feature_map": fm} if fm != "relu" else {}),
                       "io": "bf16 Q/K/V in, bf16 O out, fp32 state and accumulation",
                       "eps": w.eps,
                       "per_rank": (f"one independent {w.name} batch" if part is None else
                                    f"rank 0: batches {part[0]}-{part[1] - 1}, heads {part[2]}-{part[3] - 1}"),
                       "parallelism": f"dp{world}" if part is None else f"batch/head-group split over {world}",
                       "l2": (f"inputs {w.token_heads * d * 6 / 1e6:.0f} MB + output "
                              f"{w.token_heads * d * 2 / 1e6:.0f} MB per step vs the 126 MB L2; no flush"),
                       "kernel_impl": impl["name"]},
            "ms_per_step_median": statistics.median(per_step), "ms_per_step_min": min(per_step),
            "roofline": roof, "fp32_out": fp32, "e2e": e2e, "clocks": clk,
            "gpu_launches": launches * args.steps,
        }
        if single is not None:
            line["single_launch"] = single
        if cpu is not None:
            line["cpu_baseline"] = cpu
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def per_step_times(step, stream, n):
    """Milliseconds of each of n consecutive calls of step(), from an event
    recorded between every two steps on `stream`."""
    import torch
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(n + 1)]
    ev[0].record(stream)
    for k in range(n):
        step()
        ev[k + 1].record(stream)
    torch.cuda.synchronize()
    return [ev[k].elapsed_time(ev[k + 1]) for k in range(n)]


def run_fp32_out(args, w, Q, K, V, ws, dev, stream, job, job_copies, hbm_peak, peak_src, impl):
    """The same forward with O in fp32 (the output type the 1e-4 per-row
    tolerance is stated for): its own timed loop after the main one, the same
    step count, algorithmic bytes with 4-byte outputs."""
    import torch
    from linear_attention_diffusion_relu_b200 import ops
    out32 = torch.empty((w.B, w.N, w.H, w.d), dtype=torch.float32, device=dev)

    def step():
        ops.forward(Q, K, V, out_dtype=torch.float32, eps=w.eps, out=out32, workspace=ws, feature_map=w.feature)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for k in range(args.steps):
        step()
    b.record(stream)
    torch.cuda.synchronize(dev)
    ms = a.elapsed_time(b) / args.steps
    ms_max = max_over_ranks(ms, dev)
    per_step = per_step_times(step, stream, min(args.steps, 1000))
    nbytes = w.algorithmic_bytes(4)
    achieved = nbytes / (ms / 1e3) / 1e9
    return {
        "value": aggregate_gbs(job.algorithmic_bytes(4), job_copies, ms_max / 1e3), "unit": UNIT,
        "ms_per_step": ms_max,
        "ms_per_step_median": statistics.median(per_step), "ms_per_step_min": min(per_step),
        "mtokens_per_s": job.B * job.N * job_copies / (ms_max / 1e3) / 1e6,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "kernel": "fwd_fused_tc",
                     "traffic": TRAFFIC_PER_LAUNCH.get((impl["name"], w.name, "fwd_fused_tc", 4)),
                     "algorithmic_bytes_per_launch": nbytes,
                     "peak_source": f"{peak_src} copy bandwidth (burst)"},
        "io": "bf16 Q/K/V in, fp32 O out",
    }


def run_e2e(args, w, dev, stream, job, job_copies):
    """Same metric through the public call with host buffers: every step copies
    Q, K, V from pinned host memory to the device and O back, the copies made
    by the library (ops.forward_host, or ops.block_causal_forward_host): K and
    V in, the state (or the blocks' prefix states), then Q streamed through in
    chunks whose outputs are copied back while the next chunk comes in."""
    import torch
    from linear_attention_diffusion_relu_b200 import ops
    from linear_attention_diffusion_relu_b200.workloads import make_inputs
    hQ, hK, hV = (t.cpu().pin_memory() for t in make_inputs(w, generator_device=input_generator(w)))
    hO = torch.empty(hQ.shape, dtype=torch.bfloat16).pin_memory()
    L = w.block
    if L:
        ws = torch.empty(ops.block_causal_forward_host_workspace_bytes(w.B, w.N, w.H, w.d, L, torch.bfloat16),
                         dtype=torch.uint8, device=dev)
    else:
        ws = torch.empty(ops.forward_host_workspace_bytes(w.B, w.N, w.H, w.d, torch.bfloat16),
                         dtype=torch.uint8, device=dev)

    def one():
        if L:
            ops.block_causal_forward_host(hQ, hK, hV, L, out_dtype=torch.bfloat16, eps=w.eps, out=hO,
                                          workspace=ws, device=dev)
        else:
            ops.forward_host(hQ, hK, hV, out_dtype=torch.bfloat16, eps=w.eps, out=hO, workspace=ws,
                             feature_map=w.feature, device=dev)

    for _ in range(3):
        one()
    torch.cuda.synchronize(dev)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(args.e2e_steps):
        one()
    e.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(s.elapsed_time(e) / args.e2e_steps, dev)
    h2d = 3 * hQ.numel() * hQ.element_size()
    d2h = hO.numel() * hO.element_size()
    return {"value": aggregate_gbs(job.algorithmic_bytes(2), job_copies, ms / 1e3), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms,
            "call": ("block_causal_forward_host" if L else "forward_host") + " (copies by the library)"}


def run_kvproj(args):
    """The key-value projection with the state in its epilogue at a Sana
    shape (X (B, N, C) with C = H*d), timed per call with CUDA events, next to
    the unfused pipeline it replaces: K and V from torch's bf16 matmul (cuBLAS,
    stored), then kv_state. Metric: TFLOP/s of the projection GEMM (the state
    product adds < 1 %), roofline against the measured cuBLAS bf16 peak."""
    import torch
    from linear_attention_diffusion_relu_b200 import ops
    from linear_attention_diffusion_relu_b200.workloads import WORKLOADS
    if args.gpus != 1:
        raise SystemExit("--op kvproj runs on one GPU")
    w = WORKLOADS[args.workload]
    B, N, H, d = w.B, w.N, w.H, w.d
    C = H * d
    dev = torch.device("cuda", 0)
    g = torch.Generator(device="cuda").manual_seed(w.seed)
    X = torch.randn((B, N, C), generator=g, device=dev).to(torch.bfloat16)
    Wk = (torch.randn((H * d, C), generator=g, device=dev) / C ** 0.5).to(torch.bfloat16)
    Wv = (torch.randn((H * d, C), generator=g, device=dev) / C ** 0.5).to(torch.bfloat16)
    state = torch.empty((B, H, d, d + 1), dtype=torch.float32, device=dev)
    ws = torch.empty(ops.kv_projection_workspace_bytes(B, N, C, H, d), dtype=torch.uint8, device=dev)
    K = torch.empty((B, N, H, d), dtype=torch.bfloat16, device=dev)
    V = torch.empty_like(K)
    ws2 = ops.make_workspace(B, N, H, d, dev)

    def fused():
        ops.kv_projection_state(X, Wk, Wv, H, state=state, workspace=ws)

    def unfused():
        torch.matmul(X, Wk.T, out=K.view(B, N, H * d))
        torch.matmul(X, Wv.T, out=V.view(B, N, H * d))
        ops.kv_state(K, V, state=state, workspace=ws2)

    def timed(fn, steps):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(steps):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / steps

    steps = max(1, min(args.steps, 200))
    clocks = ClockSampler(0)
    clocks.start()
    ms = timed(fused, steps)
    clk = clocks.stop()
    ms_unfused = timed(unfused, steps)
    flops = 2.0 * B * N * C * (2 * H * d)
    tflops = flops / (ms / 1e3) / 1e12
    peak = FALLBACK_BF16_TFLOPS
    src = "fallback"
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peak, src = float(json.load(f)["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        pass
    line = {
        "metric": "key-value projection with the state in its epilogue, TFLOP/s", "value": tflops,
        "unit": "TFLOP/s", "n_gpus": 1, "steps": steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": f"{w.name} key-value projection", "B": B, "N": N, "C": C, "H": H, "d": d},
        "roofline": {"bound": "tensor", "achieved": tflops, "peak": peak, "unit": "TFLOP/s",
                     "frac": tflops / peak, "traffic": None, "kernel": "kvproj_state_tc",
                     "peak_source": f"{src} cuBLAS bf16 (burst)"},
        "unfused": {"ms_per_step": ms_unfused, "what": "torch bf16 matmul for K and V (stored) + kv_state",
                    "tflops": flops / (ms_unfused / 1e3) / 1e12},
        "clocks": clk,
        "gpu_launches": ops.load_library().sana_linattn_kv_projection_state_launches(B, N, C, H, d) * steps,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_mixffn(args):
    """The Mix-FFN at a Sana shape: tokens on a square grid (N = Hg * Wg), C = H*d,
    hidden Ch = 2.5 C (a workload choice; the pages give no expansion ratio).
    Metric: TFLOP/s of the two 1x1 convolutions (the depthwise conv adds < 1 %),
    roofline against the measured cuBLAS bf16 peak; torch's unfused pipeline
    (cuBLAS, cuDNN depthwise conv, GLU) is timed beside it."""
    import math
    import torch
    from linear_attention_diffusion_relu_b200 import ops
    from linear_attention_diffusion_relu_b200.workloads import WORKLOADS
    if args.gpus != 1:
        raise SystemExit("--op mixffn runs on one GPU")
    w = WORKLOADS[args.workload]
    B, N = w.B, w.N
    C = w.H * w.d
    Ch = int(round(2.5 * C / 8)) * 8
    Hg = Wg = int(math.isqrt(N))
    if Hg * Wg != N:
        raise SystemExit(f"{w.name}: N = {N} is not a square grid")
    dev = torch.device("cuda", 0)
    g = torch.Generator(device="cuda").manual_seed(w.seed)
    X = torch.randn((B, N, C), generator=g, device=dev).to(torch.bfloat16)
    W1 = (torch.randn((2 * Ch, C), generator=g, device=dev) / C ** 0.5).to(torch.bfloat16)
    Kdw = (torch.randn((2 * Ch, 3, 3), generator=g, device=dev) / 3.0).float()
    W2 = (torch.randn((C, Ch), generator=g, device=dev) / Ch ** 0.5).to(torch.bfloat16)
    Y = torch.empty((B, N, C), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(ops.mix_ffn_workspace_bytes(B, Hg, Wg, C, Ch), dtype=torch.uint8, device=dev)
    Kt = Kdw.to(torch.bfloat16).view(2 * Ch, 1, 3, 3)

    def ours():
        ops.mix_ffn(X, W1, Kdw, W2, (Hg, Wg), out=Y, workspace=ws)

    def torch_ref():
        U = (X @ W1.T).view(B, Hg, Wg, 2 * Ch).permute(0, 3, 1, 2)
        D = torch.nn.functional.conv2d(U, Kt, padding=1, groups=2 * Ch)
        a, gt = D.permute(0, 2, 3, 1).reshape(B, N, 2 * Ch).chunk(2, dim=-1)
        return (a * torch.sigmoid(gt)) @ W2.T

    def timed(fn, steps):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(steps):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / steps

    steps = max(1, min(args.steps, 100))
    clocks = ClockSampler(0)
    clocks.start()
    ms = timed(ours, steps)
    clk = clocks.stop()
    ms_torch = timed(torch_ref, max(1, steps // 4))
    flops = 2.0 * B * N * C * (2 * Ch) + 2.0 * B * N * Ch * C
    tflops = flops / (ms / 1e3) / 1e12
    peak, src = FALLBACK_BF16_TFLOPS, "fallback"
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peak, src = float(json.load(f)["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        pass
    line = {
        "metric": "Mix-FFN (expand, depthwise 3x3 + GLU, project), TFLOP/s", "value": tflops,
        "unit": "TFLOP/s", "n_gpus": 1, "steps": steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": f"{w.name} Mix-FFN", "B": B, "grid": [Hg, Wg], "C": C, "Ch": Ch},
        "roofline": {"bound": "tensor", "achieved": tflops, "peak": peak, "unit": "TFLOP/s",
                     "frac": tflops / peak, "traffic": None, "kernel": "gemm_bf16_tc (x2) + dwconv_glu",
                     "peak_source": f"{src} cuBLAS bf16 (burst)"},
        "torch_unfused": {"ms_per_step": ms_torch,
                          "what": "cuBLAS matmul, cuDNN depthwise conv2d, sigmoid gate, cuBLAS matmul"},
        "clocks": clk,
        "gpu_launches": ops.load_library().sana_linattn_mix_ffn_launches(B, Hg, Wg, C, Ch) * steps,
    }
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.op == "kvproj":
        return run_kvproj(args)
    if args.op == "mixffn":
        return run_mixffn(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
