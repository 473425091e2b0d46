"""Benchmark of the HSTU layer hot path (forward + backward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload training|long_history|mfalcon|academic|pr1_ref]

One step = one pass of the whole path over one batch: for the default
`training` workload, 8 HSTU layers forward (projection + SiLU, pointwise
attention with rab buckets and causal masking, LayerNorm*U, output
projection) then backward with fp32 gradient accumulation, on 64 jagged
sequences with lengths U[1024, 8192], d=1024, 8 heads of 128, bf16.  Inputs
are synthetic (seeded) and resident in HBM; with N GPUs each rank processes
its own 64 sequences (weak scaling) and the fp32 gradients are all-reduced
over NCCL.  Rank 0 prints one JSON line.

With N GPUs each rank processes its own 64 sequences (weak scaling) and each
layer's fp32 gradients are all-reduced over NCCL as soon as that layer's
backward has been issued (overlapping the layers below).  --split instead
shards ONE batch's 64 sequences across the ranks, balanced by n^2 with LPT
(strong scaling).  The default line also carries `attention_8k`: the two
attention kernels alone on 16 sequences of exactly 8,192 tokens (H=8,
dh=128), measured on rank 0 after the timed steps.

--impl reference times the fp64 CPU oracle on a bounded sample of the same
workload on this host's cores (rank 0 only).

--attention-8k prints only that attention measurement, on its own line;
--softmax-8k the same measurement with the softmax comparison kernel's
forward as the value (the pointwise forward beside it).

--sampler measures the Stochastic Length sampler instead (selection plus the
gathers of the fp32 rows and timestamps of the training batch, alpha 1.6 by
default) and prints its own line; with --impl reference it times the oracle
sampler on the same batch.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from hstu_sequential_transducer_b200 import workloads as W  # noqa: E402

METRIC = "HSTU layer fwd+bwd tokens/s and TFLOP/s at max_len 8192; % of B200 BF16 peak"
FP32_FMA_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
MUFU_TOPS = 148 * 16 * 1.965e9 / 1e12          # tanh.approx results per second, T/s


def pairs_allowed(lengths, num_targets=None):
    tot = 0
    for i, n in enumerate(lengths):
        n = int(n)
        m = 0 if num_targets is None else int(num_targets[i])
        if m == 0:
            tot += n * (n + 1) // 2
        else:
            h = n - m
            tot += h * (h + 1) // 2 + m * h + m
    return tot


def workload_flops(w: W.Workload, backward: bool):
    """Algorithmic flops of one step: per layer F_fwd = 10 T d^2 + 4 d sum|allowed|,
    F_bwd = 2 F_fwd (masked pairs, padding and recompute not counted)."""
    d, T = w.d_model, w.T
    pairs = pairs_allowed(w.lengths, w.num_targets)
    f_fwd = 10 * T * d * d + 4 * d * pairs
    per_layer = f_fwd * (3 if backward else 1)
    return per_layer * w.num_layers, pairs


def describe(w: W.Workload):
    return {
        "training": "8 HSTU layers fwd+bwd, bf16, fp32 grad accumulation; 64 jagged sequences "
                    "n~U[1024,8192]; d=1024, H=8, dh=128; causal, rab pos+time; N=8192",
        "long_history": "4 HSTU layers fwd, bf16; 32 jagged sequences, power-law n on [256,8192]; "
                        "d=512, H=4, dh=128; N=8192",
        "mfalcon": "M-FALCON: 16 users x (4096 history + 1024 candidates), 3 layers fwd, "
                   "candidates in microbatches of 256 against cached history K/V; d=512, H=4",
        "academic": "2 HSTU layers fwd, bf16; 128 jagged sequences n~U[20,200]; d=64, H=2, dh=32",
        "pr1_ref": "1 HSTU layer fwd, fp32; 4 sequences n~U[8,64]; d=64, H=2, dh=32",
    }[w.name.replace("_subset", "")]


# ----------------------------------------------------------------------------
# Data-parallel pieces (weak scaling: every rank its own sequences, one
# all-reduce of the flat fp32 gradient buffer per step, max-over-ranks time)
# ----------------------------------------------------------------------------

def rank_data_seed(rank: int) -> int:
    """Seed of rank `rank`'s sequences; the weights come from the common seed."""
    return 5 + 1000 * rank


def allreduce_grads(flat, dist):
    """Sums the ranks' gradient buffers in place (one collective)."""
    dist.all_reduce(flat)


def split_shard(w: W.Workload, rank: int, world: int) -> W.Workload:
    """Rank `rank`'s part of one batch shared by all ranks: LPT by n^2."""
    from hstu_sequential_transducer_b200 import dp
    return W.subset(w, dp.lpt_shards(w.lengths, world)[rank])


def max_over_ranks(ms: float, dist, device) -> float:
    """The slowest rank's time: the job's step time."""
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def make_workload(name, rank, batch=None, layers=None, split_world=None):
    """The named workload; `batch` keeps only its first sequences and
    `layers` its first layers (a small case of the same shapes, e.g. for
    profiler captures).  With `split_world`, every rank draws the same batch
    and keeps its LPT shard of it."""
    if name == "training":
        w = W.training(data_seed=rank_data_seed(0 if split_world else rank))
    else:
        w = W.WORKLOADS[name]()
    if batch is not None and batch < w.B:
        w = W.subset(w, list(range(batch)))
    if split_world:
        w = split_shard(w, rank, split_world)
    if layers is not None and layers < w.num_layers:
        w.params = w.params[:layers]
        w.num_layers = layers
    return w


# ----------------------------------------------------------------------------
# Clock sampling during the timed region
# ----------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.idx = device_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
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
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[5 + k] == "Active"})
        power = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max(power) if power else None}


# kernel class -> the source file its traffic figure was captured from
_KERNEL_SOURCES = {"attn_fwd": "attn_tc.cu", "attn_bwd": "attn_bwd_tc.cu",
                   "sl_gather": "stoch_len.cu"}


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes (read + write) per launch of `kernel` on the full training
    workload, from the ncu capture summarised under profiles/ (a line
    `traffic_per_full_launch_bytes: <kernel> <bytes> <source hash>`); None
    when there is none or the kernel's source changed since the capture."""
    import glob
    import hashlib
    src = _KERNEL_SOURCES.get(kernel)
    if src is None or workload != "training":       # scaled to the full workload only
        return None
    path = os.path.join(ROOT, "hstu_sequential_transducer_b200", "csrc", src)
    try:
        digest = hashlib.sha256(open(path, "rb").read()).hexdigest()[:12]
    except OSError:
        return None
    for md in glob.glob(os.path.join(ROOT, "profiles", "*.md")):
        for line in open(md):
            parts = line.split()
            if len(parts) == 4 and parts[0] == "traffic_per_full_launch_bytes:" and parts[1] == kernel:
                if parts[3] == digest:
                    return int(parts[2])
    return None


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# ----------------------------------------------------------------------------
# CPU baseline (the fp64 oracle as it stands)
# ----------------------------------------------------------------------------

def oracle_sample(w: W.Workload, budget_s: float):
    """Times the oracle on a bounded sample of the workload: the shortest
    sequences, as many as fit the budget (at least one).  Returns
    (layer-tokens/s, description, threads)."""
    from oracle import hstu_ref as R
    plist = [R.LayerParams(p.W1, p.W2, p.rab_pos, p.rab_time, p.b1, p.b2, p.gamma, p.beta)
             for p in w.params]
    cfg = R.LayerConfig(w.num_heads, w.norm_N, w.num_pos_buckets, w.num_time_buckets, w.ln_eps)
    order = np.argsort(w.lengths)
    done_tokens, t_used, seqs = 0, 0.0, 0
    for b in order:
        sub = W.subset(w, [int(b)])
        if w.name.startswith("training") and sub.T > 1024:
            # the sample is a 1024-token prefix of a sequence
            pref = 1024
            sub.x, sub.timestamps, sub.dy = sub.x[:pref], sub.timestamps[:pref], sub.dy[:pref]
            sub.seq_offsets = np.array([0, pref], np.int64)
        t0 = time.perf_counter()
        if w.backward:
            R.stack_forward_backward(sub.x, sub.seq_offsets, sub.timestamps, sub.num_targets, plist,
                                     cfg, sub.dy)
        else:
            R.stack_forward(sub.x, sub.seq_offsets, sub.timestamps, sub.num_targets, plist, cfg)
        t_used += time.perf_counter() - t0
        done_tokens += sub.T
        seqs += 1
        if t_used >= budget_s:
            break
    threads = os.cpu_count()
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        if info:
            threads = max(i.get("num_threads", 1) for i in info)
    except Exception:
        pass
    desc = (f"{seqs} sequence(s), {done_tokens} tokens, {w.num_layers} layers "
            f"{'fwd+bwd' if w.backward else 'fwd'} (shortest first"
            f"{'; 1024-token prefix' if w.name.startswith('training') else ''})")
    return done_tokens * w.num_layers / t_used, desc, threads, t_used


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = make_workload(args.workload, 0, args.batch, args.layers)
    for _ in range(args.warmup):
        oracle_sample(w, 0.0)
    vals, times = [], []
    desc, threads = "", os.cpu_count()
    for _ in range(args.steps):
        v, desc, threads, t = oracle_sample(w, 0.0)
        vals.append(v)
        times.append(t)
    value = float(np.median(vals))
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": float(np.median(times) * 1000), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{args.workload}: {describe(w)}",
                       "sample": desc, "parallelism": "host cores"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads,
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------
# Our arm
# ----------------------------------------------------------------------------

def run_ours(args):
    import torch
    import torch.distributed as dist

    from hstu_sequential_transducer_b200 import build
    from hstu_sequential_transducer_b200 import hstu as H
    from hstu_sequential_transducer_b200 import stack as S

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300))
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    H.lib()

    from hstu_sequential_transducer_b200 import dp
    split = bool(args.split) and args.workload == "training"
    w = make_workload(args.workload, rank, args.batch, args.layers,
                      split_world=world if split else None)
    dw = S.DeviceWorkload.from_workload(w)
    backward = w.backward
    flops, pairs = workload_flops(w, backward)
    dev = torch.device("cuda", local)
    # whole-job work: the sum over ranks (ranks' batches differ in size)
    job = torch.tensor([float(w.T * w.num_layers), float(flops)], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(job)
    job_tokens, job_flops = float(job[0].item()), float(job[1].item())

    if args.workload == "mfalcon" and args.batch is None:
        hist, cand = w.meta["history"], w.meta["candidates"]

        def step():
            S.mfalcon_score(dw, hist, cand, w.microbatch)
    elif backward:
        ts = S.TrainStep(dw)
        # each layer's gradients are summed across ranks as soon as its
        # backward is issued, overlapping the backward of the layers below
        bk = dp.default_group_bucketing(ts)

        def step():
            ts.zero_grads()
            ts.run(on_layer_grads=bk.layer_done if bk else None)
            if bk:
                bk.wait()
    else:
        def step():
            S.forward_stack(dw)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()

    clocks = ClockSampler(local)
    clocks.start()
    H.profiler_reset()
    H.profiler_enable(True)
    launches0 = H.launch_count()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step()
    e1.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    launches = H.launch_count() - launches0
    H.profiler_enable(False)
    clk = clocks.stop()
    ms = e0.elapsed_time(e1) / args.steps
    if world > 1:
        ms = max_over_ranks(ms, dist, dev)

    kern = {}
    for k, name in enumerate(H.KERNEL_NAMES):
        n, tot = H.profiler_collect(k)
        if n:
            kern[name] = {"launches": n, "total_ms": tot, "avg_ms": tot / n}
    H.profiler_reset()

    value = job_tokens / (ms / 1000.0)
    tflops = job_flops / (ms / 1000.0) / 1e12
    peaks, peak_src = read_peaks()

    # dominant kernel and its roofline (algorithmic flops or bytes per launch)
    d = w.d_model
    per_launch = {
        "attn_fwd": ("tensor", 4 * d * pairs),
        "attn_bwd": ("tensor", 8 * d * pairs),
        "proj_in": ("tensor", 8 * w.T * d * d),
        "proj_out": ("tensor", 2 * w.T * d * d),
        "proj_in_bwd": ("tensor", 16 * w.T * d * d),
        "proj_out_bwd": ("tensor", 4 * w.T * d * d),
        # read O (fp32) and U, write Z, row statistics
        "ln_fwd": ("hbm", w.T * (8 * d + 8)),
        # read dZ, O (fp32), U, Pre_U, statistics; write dO and dPre_U
        "ln_bwd": ("hbm", w.T * (14 * d + 8)),
    }
    # contractions that run on the FP32 pipes (fp32 layers) are held against
    # the FP32 FMA peak: 148 SMs x 128 lanes x 2 flops x 1.965 GHz = 74.4
    # TFLOP/s.  bf16 heads of 32 run on the tensor cores zero-padded to 64
    # columns, where one tanh per allowed score (the MUFU unit) binds before
    # the tensor pipe: held against 148 SMs x 16 MUFU results x 1.965 GHz
    dh = d // w.num_heads
    if w.dtype == "f32":
        for k in ("attn_fwd", "attn_bwd"):
            per_launch[k] = ("alu", per_launch[k][1])
    elif dh == 32:
        per_launch["attn_fwd"] = ("mufu", w.num_heads * pairs)
        per_launch["attn_bwd"] = ("mufu", w.num_heads * pairs)
    if w.dtype == "f32":
        for k in ("proj_in", "proj_out", "proj_in_bwd", "proj_out_bwd"):
            per_launch[k] = ("alu", per_launch[k][1])
    if args.workload == "mfalcon" and args.batch is None:
        # the history pass runs attn_fwd (causal over each user's history);
        # each candidate microbatch runs attn_cached (history + self per
        # candidate); the projections see history and microbatch rows
        hist, cand, mb = w.meta["history"], w.meta["candidates"], w.microbatch
        per_launch["attn_fwd"] = ("tensor", 4 * d * w.B * hist * (hist + 1) // 2)
        per_launch["attn_cached"] = ("tensor", 4 * d * w.B * mb * (hist + 1))
        per_launch.pop("proj_in")
        per_launch.pop("proj_out")
        per_launch.pop("ln_fwd")
    roof = None
    if kern:
        top = max((k for k in kern if k in per_launch), key=lambda k: kern[k]["total_ms"],
                  default=None)
        if top:
            bound, work = per_launch[top]
            avg_s = kern[top]["avg_ms"] / 1000.0
            if bound == "tensor":
                ach = work / avg_s / 1e12
                peak = peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops"))
                unit, src = "TFLOP/s", f"{peak_src} (bf16_tflops_sustained)"
            elif bound == "alu":
                ach = work / avg_s / 1e12
                peak = FP32_FMA_TFLOPS
                unit, src = "TFLOP/s", "derived: 148 SMs x 128 FP32 lanes x 2 x 1.965 GHz"
            elif bound == "mufu":
                ach = work / avg_s / 1e12
                peak = MUFU_TOPS
                unit, src = "Ttanh/s", "derived: 148 SMs x 16 MUFU results/clk x 1.965 GHz"
            else:
                ach = work / avg_s / 1e9
                peak = peaks.get("hbm_gbs")
                unit, src = "GB/s", f"{peak_src} (hbm_gbs)"
            roof = {"kernel": top, "bound": "alu" if bound == "mufu" else bound,
                    "achieved": ach, "peak": peak, "unit": unit,
                    "frac": ach / peak, "traffic": profiled_traffic(top, w.name),
                    "peak_source": src, "work_per_launch": work}
            if bound == "mufu":
                # the same launch against the bf16 tensor roof (algorithmic
                # flops 4 d per allowed pair; the padded columns not counted)
                fl = (4 if top == "attn_fwd" else 8) * d * pairs
                tpk = peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops"))
                roof["tensor"] = {"achieved": fl / avg_s / 1e12, "peak": tpk, "unit": "TFLOP/s",
                                  "frac": fl / avg_s / 1e12 / tpk}

    # end to end through the public API with host buffers
    e2e = None
    if backward and args.workload == "training" and not args.skip_e2e and args.batch is None:
        e2e = e2e_training(args, ts, dw, world, dist, bk, job_tokens)

    # the attention kernels alone at the length the throughput target names
    # (rank 0; the other ranks wait at the barrier below)
    attn8k = None
    if args.workload == "training" and not args.skip_attention_8k and rank == 0:
        attn8k = attention8k_measure(args, dev)
    if world > 1:
        dist.barrier()

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "strong" if split else "weak",
            "vs_baseline": None,
            "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
            "config": {"workload": f"{args.workload}: {describe(w)}",
                       "global_batch": (64 if split else w.B * world),
                       "tokens_per_step": int(job_tokens) // w.num_layers,
                       "seq_len": int(w.lengths.max()), "max_len": 8192,
                       "layers": w.num_layers, "parallelism": f"dp{world}",
                       "sharding": ("one batch split across ranks by n^2 (LPT)" if split else
                                    "each rank its own batch"),
                       "grad_allreduce": "per-layer buckets, overlapped with the backward",
                       "l2": "inputs larger than L2 (no flush)"},
            "tflops": tflops, "pct_bf16_peak": tflops / peaks.get("bf16_tflops_sustained", 1400.0),
            "roofline": roof, "kernels": kern, "gpu_launches": launches,
            "clocks": clk, "e2e": e2e, "attention_8k": attn8k}
    if rank == 0 and world == 1 and not args.skip_cpu:
        v, desc, threads, _ = oracle_sample(w, args.cpu_budget)
        line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                                "sample": desc}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def e2e_training(args, ts, dw, world, dist, bk, job_tokens):
    """The same training step through the public API, with each step's inputs
    (x, offsets, timestamps, dY; x and dY as bf16) copied from pinned host
    memory and its result (dX, as bf16) read back, all inside the timed
    region.  Copies run on a second stream, double-buffered like a data
    loader with a prefetch depth of one: step k+1's inputs are uploaded while
    step k computes, and step k's dX is downloaded while step k+1 computes."""
    import torch
    w = dw.w
    dev = dw.x.device
    hx = torch.from_numpy(w.x).to(torch.bfloat16).pin_memory()
    hoff = torch.from_numpy(w.seq_offsets).pin_memory()
    hts = torch.from_numpy(w.timestamps).pin_memory()
    hdy = torch.from_numpy(w.dy).to(torch.bfloat16).pin_memory()
    hdx = [torch.empty(hx.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    h2d = hx.numel() * 2 + hoff.numel() * 8 + hts.numel() * 8 + hdy.numel() * 2
    d2h = hdx[0].numel() * 2
    comp = torch.cuda.current_stream(dev)
    copy = torch.cuda.Stream(device=dev)
    bufs = [(dw.x, dw.offsets, dw.timestamps, dw.dy),
            (torch.empty_like(dw.x), torch.empty_like(dw.offsets),
             torch.empty_like(dw.timestamps), torch.empty_like(dw.dy))]
    stage = [torch.empty(dw.x.shape, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    loaded = [torch.cuda.Event() for _ in range(2)]    # set s holds a step's inputs
    consumed = [torch.cuda.Event() for _ in range(2)]  # the step using set s is done
    drained = [torch.cuda.Event() for _ in range(2)]   # stage[s] has been read back
    saved_inputs = (dw.x, dw.offsets, dw.timestamps, dw.dy, ts.acts[0])

    def load(s):
        with torch.cuda.stream(copy):
            copy.wait_event(consumed[s])
            x, off, tst, dy = bufs[s]
            x.copy_(hx, non_blocking=True)
            off.copy_(hoff, non_blocking=True)
            tst.copy_(hts, non_blocking=True)
            dy.copy_(hdy, non_blocking=True)
            loaded[s].record(copy)

    def step(k, last):
        s = k % 2
        comp.wait_event(loaded[s])
        x, off, tst, dy = bufs[s]
        dw.offsets, dw.timestamps, dw.dy = off, tst, dy
        ts.acts[0] = x
        ts.zero_grads()
        dx = ts.run(on_layer_grads=bk.layer_done if bk else None)
        if bk:
            bk.wait()
        comp.wait_event(drained[s])
        stage[s].copy_(dx)
        consumed[s].record(comp)
        if not last:
            load((k + 1) % 2)
        with torch.cuda.stream(copy):
            copy.wait_event(consumed[s])
            hdx[s].copy_(stage[s], non_blocking=True)
            drained[s].record(copy)

    def run(n):
        copy.wait_stream(comp)
        load(0)
        for k in range(n):
            step(k, k == n - 1)
        comp.wait_stream(copy)

    run(2)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    run(args.steps)
    e1.record(comp)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    if world > 1:
        ms = max_over_ranks(ms, dist, dev)
    dw.x, dw.offsets, dw.timestamps, dw.dy, ts.acts[0] = saved_inputs
    return {"value": job_tokens / (ms / 1000.0), "unit": "tokens/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "ms_per_step": ms,
            "copies": "second stream, double-buffered: next step's inputs uploaded and the "
                      "previous step's dX downloaded while a step computes"}


# ----------------------------------------------------------------------------
# Stochastic Length sampler (--sampler): its own measurement line
# ----------------------------------------------------------------------------

SAMPLER_METRIC = ("Stochastic Length sampler input tokens/s (training batch: 64 sequences "
                  "U[1024, 8192], d=1024 fp32 rows, max_len 8192)")


def sampler_inputs(rank: int, batch=None):
    """The training batch's lengths and timestamps (same draws as the training
    workload), fp32 rows of width 1024 (the residual stream entering layer 1)
    and the sampler's random inputs; `batch` keeps the first sequences."""
    seed = rank_data_seed(rank)
    rng = np.random.default_rng(seed)
    lengths = rng.integers(1024, 8193, size=64)
    ts = W.draw_timestamps(rng, lengths)
    if batch is not None and batch < len(lengths):
        ts = ts[:int(lengths[:batch].sum())]
        lengths = lengths[:batch]
    offs = W.offsets_from_lengths(lengths)
    T = int(offs[-1])
    x = np.random.default_rng(seed + 1).standard_normal((T, 1024), dtype=np.float32)
    keep, keys = W.sl_draws(seed + 2, len(lengths), T)
    return offs, ts, x, keep, keys


def sampler_oracle(offs, ts, x, keep, keys, L):
    """One pass of the oracle sampler (selection, then gathers of the rows
    and timestamps) over the whole batch; returns seconds."""
    from oracle import stochastic_length as SL
    t0 = time.perf_counter()
    new_offs, gi = SL.sample(offs, None, L, keep, keys)
    SL.gather(x, gi)
    SL.gather(ts, gi)
    return time.perf_counter() - t0


def run_sampler(args):
    import torch
    import torch.distributed as dist

    from hstu_sequential_transducer_b200 import build
    from hstu_sequential_transducer_b200 import hstu as H

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    offs, ts, x, keep, keys = sampler_inputs(rank, args.batch)
    B, T = len(offs) - 1, int(offs[-1])
    if args.impl == "reference":
        if rank != 0:
            return 0
        from oracle import stochastic_length as SL
        L = SL.subsequence_length(8192, args.alpha)
        for _ in range(args.warmup):
            sampler_oracle(offs, ts, x, keep, keys, L)
        times = [sampler_oracle(offs, ts, x, keep, keys, L) for _ in range(args.steps)]
        sec = float(np.median(times))
        value = T / sec
        desc = f"whole batch ({B} sequences, {T} tokens), alpha {args.alpha}"
        print(json.dumps({
            "metric": SAMPLER_METRIC, "value": value, "unit": "tokens/s", "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": sec * 1000, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int64", "data": "synthetic",
            "config": {"workload": f"stochastic_length: {desc}", "parallelism": "host cores"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}), flush=True)
        return 0

    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300))
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    H.lib()
    dev = torch.device("cuda", local)
    L = H.sl_subsequence_length(8192, args.alpha)
    hoffs = torch.from_numpy(offs).pin_memory()
    hts = torch.from_numpy(ts).pin_memory()
    hx = torch.from_numpy(x).pin_memory()
    hkeep = torch.from_numpy(keep.view(np.int32)).pin_memory()
    hkeys = torch.from_numpy(keys.view(np.int32)).pin_memory()
    d_offs, d_ts, d_x = hoffs.to(dev), hts.to(dev), hx.to(dev)
    d_keep, d_keys = hkeep.to(dev), hkeys.to(dev)
    new_offs = torch.empty(B + 1, dtype=torch.int64, device=dev)
    gidx = torch.empty(T, dtype=torch.int64, device=dev)
    x_out, ts_out = torch.empty_like(d_x), torch.empty_like(d_ts)
    hnew = torch.empty(B + 1, dtype=torch.int64).pin_memory()
    gather_events = []

    def step(timed=False):
        H.stochastic_length(d_offs, None, L, d_keep, d_keys, new_offs, gidx)
        if timed:
            g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            g0.record()
        H.gather_rows(d_x, gidx, new_offs[B:], x_out)
        if timed:
            g1.record()
            gather_events.append((g0, g1))
        H.gather_rows(d_ts, gidx, new_offs[B:], ts_out)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    t_new = int(new_offs[B].item())
    if world > 1:
        dist.barrier()
    clocks = ClockSampler(local)
    clocks.start()
    launches0 = H.launch_count()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        step(timed=True)
    e1.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    launches = H.launch_count() - launches0
    clk = clocks.stop()
    ms = e0.elapsed_time(e1) / args.steps
    if world > 1:
        ms = max_over_ranks(ms, dist, dev)
    g_ms = float(np.mean([a.elapsed_time(b) for a, b in gather_events]))
    peaks, peak_src = read_peaks()
    # the row gather: read T' rows of 4 KiB and their indices, write T' rows
    work = t_new * (2 * 1024 * 4 + 8)
    ach = work / (g_ms / 1000.0) / 1e9
    roof = {"kernel": "sl_gather", "bound": "hbm", "achieved": ach, "peak": peaks.get("hbm_gbs"),
            "unit": "GB/s", "frac": ach / peaks.get("hbm_gbs"),
            "traffic": profiled_traffic("sl_gather", "training"),
            "peak_source": f"{peak_src} (hbm_gbs)", "work_per_launch": work,
            "avg_launch_ms": g_ms}

    e2e = None
    if not args.skip_e2e:
        def e2e_step():
            d_offs.copy_(hoffs, non_blocking=True)
            d_ts.copy_(hts, non_blocking=True)
            d_x.copy_(hx, non_blocking=True)
            d_keep.copy_(hkeep, non_blocking=True)
            d_keys.copy_(hkeys, non_blocking=True)
            step()
            hnew.copy_(new_offs, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(args.steps):
            e2e_step()
        b.record()
        torch.cuda.synchronize()
        ems = a.elapsed_time(b) / args.steps
        if world > 1:
            ems = max_over_ranks(ems, dist, dev)
        h2d = (hoffs.numel() + hts.numel()) * 8 + hx.numel() * 4 + (hkeep.numel() + hkeys.numel()) * 4
        e2e = {"value": T * world / (ems / 1000.0), "unit": "tokens/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(hnew.numel() * 8),
               "ms_per_step": ems}

    line = {"metric": SAMPLER_METRIC, "value": T * world / (ms / 1000.0), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int64",
            "data": "synthetic",
            "config": {"workload": f"stochastic_length: training batch, B={B}, T={T}, "
                                   f"alpha {args.alpha} (L={L}), sampled T'={t_new}",
                       "global_batch": B * world, "tokens_per_step": T * world,
                       "l2": "inputs larger than L2 (no flush)", "parallelism": f"dp{world}"},
            "roofline": roof, "gpu_launches": launches, "clocks": clk, "e2e": e2e}
    if rank == 0 and world == 1 and not args.skip_cpu:
        sec = sampler_oracle(offs, ts, x, keep, keys, L)
        line["cpu_baseline"] = {"value": T / sec, "unit": "tokens/s", "cores": 1,
                                "kind": "oracle", "sample": "whole batch, one pass"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


# ----------------------------------------------------------------------------
# The attention kernels alone at length 8,192 (--attention-8k)
# ----------------------------------------------------------------------------

ATTN8K_METRIC = ("HSTU attention fwd+bwd TFLOP/s at length 8192 (16 x 8192 tokens, H=8, dh=128, "
                 "causal, pos+time rab, bf16)")
SOFTMAX8K_METRIC = ("softmax attention fwd TFLOP/s at length 8192 (16 x 8192 tokens, H=8, dh=128, "
                    "causal, pos+time rab, bf16; the comparison kernel)")


def attn8k_oracle(seconds: float):
    """The oracle's attention forward and backward on 1,024-token prefixes
    (d = 1,024, H = 8) for about `seconds`; returns (algorithmic TFLOP/s,
    sample description)."""
    from oracle import hstu_ref as R
    rng = np.random.default_rng(41)
    n, d, H = 1024, 1024, 8
    offs = np.array([0, n], np.int64)
    ts = W.draw_timestamps(rng, [n])
    g = rng.standard_normal((n, 4 * d)) * 0.5
    do = rng.standard_normal((n, d))
    rp, rt = rng.normal(0, 0.1, (H, 32)), rng.normal(0, 0.1, (H, 32))
    cfg = R.LayerConfig(H, 8192.0, 32, 32, 1e-5)
    t_used, reps = 0.0, 0
    while t_used < seconds or reps == 0:
        t0 = time.perf_counter()
        R.attention_forward(g, offs, ts, None, rp, rt, cfg)
        R.attention_backward(g, do, offs, ts, None, rp, rt, cfg)
        t_used += time.perf_counter() - t0
        reps += 1
    flops = 12 * d * (n * (n + 1) // 2) * reps
    return flops / t_used / 1e12, f"{reps} x one 1,024-token sequence, fwd+bwd, d=1024, H=8"


def softmax8k_oracle(seconds: float):
    """The softmax oracle's forward on one 1,024-token sequence (d = 1,024,
    H = 8) for about `seconds`; returns (algorithmic TFLOP/s, sample)."""
    from oracle import hstu_ref as R
    from oracle import softmax_ref as SR
    rng = np.random.default_rng(43)
    n, d, H = 1024, 1024, 8
    offs = np.array([0, n], np.int64)
    ts = W.draw_timestamps(rng, [n])
    g = rng.standard_normal((n, 4 * d)) * 0.5
    rp, rt = rng.normal(0, 0.1, (H, 32)), rng.normal(0, 0.1, (H, 32))
    cfg = R.LayerConfig(H, 8192.0, 32, 32, 1e-5)
    t_used, reps = 0.0, 0
    while t_used < seconds or reps == 0:
        t0 = time.perf_counter()
        SR.softmax_attention_forward(g, offs, ts, None, rp, rt, cfg)
        t_used += time.perf_counter() - t0
        reps += 1
    flops = 4 * d * (n * (n + 1) // 2) * reps
    return flops / t_used / 1e12, f"{reps} x one 1,024-token sequence, softmax fwd, d=1024, H=8"


def run_attention8k(args, softmax=False):
    """--attention-8k (the pointwise kernels; value = fwd+bwd TFLOP/s) or
    --softmax-8k (value = the softmax comparison kernel's forward TFLOP/s,
    the pointwise forward beside it)."""
    import torch

    from hstu_sequential_transducer_b200 import build
    from hstu_sequential_transducer_b200 import hstu as H

    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        if rank != 0:
            return 0
        v, desc = (softmax8k_oracle if softmax else attn8k_oracle)(args.cpu_budget)
        print(json.dumps({
            "metric": SOFTMAX8K_METRIC if softmax else ATTN8K_METRIC, "value": v, "unit": "TFLOP/s",
            "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": None, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"attention at 8192: {desc}", "parallelism": "host cores"},
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": os.cpu_count(),
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}), flush=True)
        return 0

    if rank != 0:          # a single-GPU measurement: under torchrun only rank 0 runs it
        return 0
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    build.build()
    H.lib()
    dev = torch.device("cuda", local)
    clocks = ClockSampler(local)
    clocks.start()
    launches0 = H.launch_count()
    m = attention8k_measure(args, dev)
    launches = H.launch_count() - launches0
    clk = clocks.stop()
    peaks, peak_src = read_peaks()
    peak = peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops"))
    sm = m["softmax_fwd"]
    line = {"metric": SOFTMAX8K_METRIC if softmax else ATTN8K_METRIC,
            "value": sm["tflops"] if softmax else m["tflops"], "unit": "TFLOP/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": sm["ms"] if softmax else m["ms"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": m["workload"], "tokens_per_step": m["tokens"],
                       "l2": "inputs larger than L2 (no flush)", "parallelism": "dp1"},
            "attn_fwd": m["attn_fwd"], "attn_bwd": m["attn_bwd"], "softmax_fwd": m["softmax_fwd"],
            "pointwise_fwd_speedup_over_softmax": m["pointwise_fwd_speedup_over_softmax"],
            "roofline": {"kernel": "attn_bwd", "bound": "tensor", "achieved": m["attn_bwd"]["tflops"],
                         "peak": peak, "unit": "TFLOP/s", "frac": m["attn_bwd"]["frac"],
                         "traffic": None, "peak_source": f"{peak_src} (bf16_tflops_sustained)",
                         "work_per_launch": m["attn_bwd"]["flops"]},
            "gpu_launches": launches, "clocks": clk, "e2e": None}
    if softmax:
        line["roofline"] = {"kernel": "softmax_fwd", "bound": "tensor", "achieved": sm["tflops"],
                            "peak": peak, "unit": "TFLOP/s", "frac": sm["frac"], "traffic": None,
                            "peak_source": f"{peak_src} (bf16_tflops_sustained)",
                            "work_per_launch": sm["flops"]}
    if not args.skip_cpu:
        v, desc = (softmax8k_oracle if softmax else attn8k_oracle)(args.cpu_budget)
        line["cpu_baseline"] = {"value": v, "unit": "TFLOP/s", "cores": os.cpu_count(),
                                "kind": "oracle", "sample": desc}
    print(json.dumps(line), flush=True)
    return 0


def attention8k_measure(args, dev):
    """The attention forward and backward kernels alone on B sequences of
    exactly 8,192 tokens (d = 1,024, H = 8, dh = 128, causal, position and time
    rab, N = 8,192), each timed with CUDA events around its launch on the
    current stream; median over the timed steps."""
    import torch

    from hstu_sequential_transducer_b200 import hstu as H
    B, n, d, nh = (args.batch or 16), 8192, 1024, 8
    T = B * n
    rng = np.random.default_rng(7)
    cfg = H.make_config(d, nh, 8192.0, H.HSTU_BF16, 32, 32, 8192)
    offs = torch.arange(B + 1, dtype=torch.int64, device=dev) * n
    ts = torch.from_numpy(W.draw_timestamps(rng, [n] * B)).to(dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(11)
    g = (torch.randn(T, 4 * d, device=dev, generator=gen) * 0.5).to(torch.bfloat16)
    pre = torch.randn(T, 4 * d, device=dev, generator=gen).to(torch.bfloat16)
    dout = torch.randn(T, d, device=dev, generator=gen).to(torch.bfloat16)
    rab_pos = torch.from_numpy(rng.normal(0, 0.1, (nh, 32)).astype(np.float32)).to(dev)
    rab_time = torch.from_numpy(rng.normal(0, 0.1, (nh, 32)).astype(np.float32)).to(dev)
    o = torch.empty(T, d, dtype=torch.float32, device=dev)
    dpre = torch.zeros(T, 4 * d, dtype=torch.bfloat16, device=dev)
    drp, drt = torch.zeros_like(rab_pos), torch.zeros_like(rab_time)
    pairs = B * n * (n + 1) // 2
    f_fwd, f_bwd = 4 * d * pairs, 8 * d * pairs
    ev = []

    def step(timed=False):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(4)] if timed else None
        if timed:
            e[0].record()
        H.attention_fwd(cfg, rab_pos, rab_time, g, offs, ts, None, o)
        if timed:
            e[1].record()
        H.attention_bwd(cfg, rab_pos, rab_time, g, pre, dout, offs, ts, None, dpre, drp, drt)
        if timed:
            e[2].record()
        # the softmax comparison kernel on the same inputs (not part of the step's
        # HSTU work: timed on its own and reported beside the pointwise forward)
        H.softmax_attention_fwd(cfg, rab_pos, rab_time, g, offs, ts, None, o)
        if timed:
            e[3].record()
            ev.append(e)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    steps = max(args.steps, 5)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        step(timed=True)
    e1.record()
    torch.cuda.synchronize()
    fwd_ms = float(np.median([a.elapsed_time(b) for a, b, _, _ in ev]))
    bwd_ms = float(np.median([b.elapsed_time(c) for _, b, c, _ in ev]))
    smx_ms = float(np.median([c.elapsed_time(d) for _, _, c, d in ev]))
    ms = e0.elapsed_time(e1) / steps - smx_ms
    peaks, peak_src = read_peaks()
    peak = peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops"))
    fwd_tf, bwd_tf = f_fwd / fwd_ms / 1e9, f_bwd / bwd_ms / 1e9
    out = {"workload": f"attention at 8192: B={B} sequences of 8,192 tokens, d=1024, H=8, dh=128, "
                       "causal, 32+32 rab buckets, N=8192",
           "tokens": T, "steps": steps, "ms": ms, "tflops": (f_fwd + f_bwd) / ms / 1e9,
           "attn_fwd": {"ms": fwd_ms, "tflops": fwd_tf, "frac": fwd_tf / peak, "flops": f_fwd},
           "attn_bwd": {"ms": bwd_ms, "tflops": bwd_tf, "frac": bwd_tf / peak, "flops": f_bwd},
           "softmax_fwd": {"ms": smx_ms, "tflops": f_fwd / smx_ms / 1e9,
                           "frac": f_fwd / smx_ms / 1e9 / peak, "flops": f_fwd,
                           "what": "softmax comparison kernel, same score, mask and tiling"},
           "pointwise_fwd_speedup_over_softmax": smx_ms / fwd_ms,
           "peak": peak, "peak_source": f"{peak_src} (bf16_tflops_sustained)"}
    del g, pre, dout, o, dpre
    torch.cuda.empty_cache()
    return out


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="training", choices=list(W.WORKLOADS))
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--skip-cpu", action="store_true")
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--batch", type=int, default=None,
                    help="keep only the first B sequences (a small case for profiler captures)")
    ap.add_argument("--layers", type=int, default=None,
                    help="keep only the first L layers (a small case for profiler captures)")
    ap.add_argument("--sampler", action="store_true",
                    help="measure the Stochastic Length sampler on the training batch instead")
    ap.add_argument("--alpha", type=float, default=1.6)
    ap.add_argument("--attention-8k", action="store_true",
                    help="measure the attention kernels alone on 16 sequences of 8,192 tokens")
    ap.add_argument("--softmax-8k", action="store_true",
                    help="the softmax comparison kernel alone on 16 sequences of 8,192 tokens")
    ap.add_argument("--skip-attention-8k", action="store_true",
                    help="leave the attention_8k measurement out of the default line")
    ap.add_argument("--split", action="store_true",
                    help="shard one training batch across the ranks (LPT by n^2; strong scaling)")
    args = ap.parse_args(argv)
    if args.attention_8k or args.softmax_8k:
        return run_attention8k(args, softmax=args.softmax_8k)
    if args.sampler:
        return run_sampler(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
