#!/usr/bin/env python
"""Throughput of the tensor-parallel layer and the vocab-parallel loss on B200.

One step = forward + backward of the 8.3B-scale GPT layer (batch 4, seq 1024,
hidden 3072, 32 heads, MLP 12288, t = 8 logical partitions, causal), the
headline workload; a second timed loop runs the vocab-parallel cross-entropy
forward + backward (8192 tokens, hidden 1024, vocab 50304, t = 8) and is
reported under "xent".  Inputs are seeded synthetic bf16 tensors already in
HBM when timing starts; "e2e" repeats each measurement through the same
C-ABI calls with pinned host buffers, copies included.

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Multi-GPU (N > 1) runs under torchrun: every rank runs an independent replica
of the step on its own GPU (the layer's partitions live on one device), the
timed region is bracketed by barriers and the slowest rank's time is used.

--impl reference times the fp64 CPU oracle on the host cores (rank 0 only) on
a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import csv
import datetime
import hashlib
import io
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import tp_inputs as TI  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
GEMM_SOURCES = ("gemm.cu", "gemm.cuh", "tp_common.cuh")
XENT_SOURCES = ("xent.cu",)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_hash(names) -> str:
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "tensor_transformer_layer_tp_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(profile_name: str, sources, key: str = "dram_bytes_per_launch") -> float | None:
    """DRAM bytes (per launch, or per step for `key` = dram_bytes_per_step) from
    a committed ncu summary, if it was taken on the current kernel source (the
    summary records the source hash)."""
    p = os.path.join(ROOT, "profiles", profile_name)
    if not os.path.exists(p):
        return None
    want = source_hash(sources)
    traffic, src = None, None
    with open(p) as f:
        for line in f:
            if line.startswith("source_hash:"):
                src = line.split(":", 1)[1].strip()
            if line.startswith(key + ":"):
                traffic = float(line.split(":", 1)[1].strip())
    return traffic if src == want else None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        rows = [r for r in csv.reader(io.StringIO(out)) if len(r) >= 9]
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.strip() == "Active"})
        power = [float(r[3]) for r in rows if r[3].strip().replace(".", "").isdigit()]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "power_w_max": max(power) if power else None,
                "samples": len(rows), "reasons": reasons}


# --------------------------------------------------------------------- distributed

def dist_setup(backend: str = "nccl"):
    """Join the process group torchrun describes (RANK / WORLD_SIZE / MASTER_*).

    The layer's t partitions live on one GPU, so ranks run independent
    replicas: the only collectives are the barrier and the max of the timings.
    """
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300), **kw)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int, device: str = "cuda") -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank_step: float, steps: int, world: int, max_ms: float) -> float:
    """Whole-job rate: units all ranks processed / slowest rank's time (per second)."""
    return world * units_per_rank_step * steps / (max_ms / 1e3)


def timed_loop(step, steps, world):
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(steps):
        step()
    e1.record(s)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    return max_over_ranks(e0.elapsed_time(e1), world)


# --------------------------------------------------------------------- our implementation

def bench_layer(d: TI.LayerDims, steps, warmup, world, B, runner_mod):
    inp = TI.make_layer_inputs(d, seed=0)
    dims = B.make_dims(d.t, d.batch, d.seq, d.hidden, d.heads, d.ffn, d.causal, d.ln_eps)
    params = runner_mod.params_to(TI.partition_layer_params(inp, d.t, d.heads), "cuda")
    r = runner_mod.LayerRunner(dims, params)
    x, dy = inp["x"].cuda(), inp["dy"].cuda()
    vl = inp["valid_len"].cuda() if "valid_len" in inp else None
    flops = TI.layer_flops(d, inp.get("valid_len"))
    n, h, f = d.tokens, d.hidden, d.ffn
    gemm_flops = 3 * 2 * n * (3 * h * h + h * h + 2 * h * f)

    def step():
        r.forward(x, vl)
        r.backward(x, dy, vl)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    B.tp_device_status()
    B.tp_profile_reset()
    ms_eager = timed_loop(step, steps, world)   # per-kernel breakdown from these launches
    prof = B.tp_profile_summary()
    B.tp_device_status()

    # The same step recorded once as a CUDA graph and replayed: the headline
    # device number (same kernels, same buffers, no per-launch host gaps).
    graph = r.capture_step(x, dy, vl)
    for _ in range(warmup):
        graph.replay()
    torch.cuda.synchronize()
    ms = timed_loop(graph.replay, steps, world)
    B.tp_device_status()
    del graph
    # (profiling stays off for the end-to-end loop: a user's calls carry no events)

    # End to end through the same calls: every step copies its inputs in from
    # pinned host memory and reads dX back.  Copies run on their own stream:
    # step k+1's inputs go into a second device buffer while step k computes,
    # and step k's dX is read back before step k+1's backward overwrites it.
    xh, dyh = inp["x"].pin_memory(), inp["dy"].pin_memory()
    dxh = torch.empty_like(inp["x"]).pin_memory()
    xd = [torch.empty_like(x) for _ in range(2)]
    dyd = [torch.empty_like(dy) for _ in range(2)]

    def e2e_steps(n):
        comp, copy = torch.cuda.current_stream(), torch.cuda.Stream()
        ev = lambda: torch.cuda.Event()
        in_ready, in_free = [ev(), ev()], [ev(), ev()]
        dx_read = ev()
        start = ev()
        start.record(comp)
        copy.wait_event(start)

        def copy_in(k):
            b = k % 2
            with torch.cuda.stream(copy):
                if k >= 2:
                    copy.wait_event(in_free[b])
                xd[b].copy_(xh, non_blocking=True)
                dyd[b].copy_(dyh, non_blocking=True)
                in_ready[b].record(copy)

        copy_in(0)
        for k in range(n):
            b = k % 2
            comp.wait_event(in_ready[b])
            r.forward(xd[b], vl)
            if k + 1 < n:
                copy_in(k + 1)
            if k >= 1:
                comp.wait_event(dx_read)       # previous dX is on the host
            r.backward(xd[b], dyd[b], vl)
            in_free[b].record(comp)
            done = ev()
            done.record(comp)
            with torch.cuda.stream(copy):
                copy.wait_event(done)
                dxh.copy_(r.dx, non_blocking=True)
                dx_read.record(copy)
        comp.wait_event(dx_read)

    e2e_steps(max(1, warmup // 2))
    ms_e2e = timed_loop(lambda: e2e_steps(steps), 1, world)
    bytes_in = (x.numel() + dy.numel()) * 2
    return dict(ms=ms, ms_eager=ms_eager, prof=prof, flops=flops, gemm_flops=gemm_flops,
                ms_e2e=ms_e2e, h2d=bytes_in, d2h=dxh.numel() * 2)


def bench_partition_sum(d: TI.LayerDims, steps, warmup, world, B):
    """The FC2 all-reduce point of the layer two ways: summed inside the GEMM's
    K-loop (what the layer runs) and explicitly (per-partition fp32 partials,
    then tp_partition_sum with bias and residual)."""
    n, h, fw, t = d.tokens, d.hidden, d.ffn // d.t, d.t
    g = torch.Generator().manual_seed(0)
    A = [(torch.randn(n, fw, generator=g) * 0.5).to(torch.bfloat16).cuda() for _ in range(t)]
    W = [(torch.randn(fw, h, generator=g) * 0.02).to(torch.bfloat16).cuda() for _ in range(t)]
    bias = torch.zeros(h, dtype=torch.bfloat16, device="cuda")
    res = torch.zeros(n, h, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(n, h, dtype=torch.bfloat16, device="cuda")
    parts = [torch.empty(n, h, dtype=torch.float32, device="cuda") for _ in range(t)]

    def fused():
        B.tp_gemm(t, 1, n, h, fw, A, 0, W, 0, [out], 0)

    def explicit():
        B.tp_gemm(t, 0, n, h, fw, A, 0, W, 0, parts, 1)
        B.tp_partition_sum(parts, out, bias, res)

    res_ms = {}
    for name, fn in (("fused_ms", fused), ("explicit_ms", explicit)):
        for _ in range(warmup):
            fn()
        res_ms[name] = timed_loop(fn, steps, world) / steps
    B.tp_device_status()
    return dict(res_ms, shape=f"FC2 of the layer: sum over t={t} of [{n}x{fw}].[{fw}x{h}] + b2 + residual",
                partial_bytes=t * n * h * 4,
                note="explicit = fp32 partial per partition, then one summing pass; "
                     "fused = one fp32 TMEM accumulator over all partitions' K ranges")


def bench_xent(d: TI.XentDims, steps, warmup, world, B, runner_mod):
    inp = TI.make_xent_inputs(d, seed=0)
    xr = runner_mod.XentRunner(d.t, d.tokens, d.hidden, d.vocab)
    x = inp["x"].cuda()
    emb = [e.cuda() for e in TI.partition_vocab(inp["emb"], d.t)]
    tgt = inp["target"].cuda()

    def step():
        xr(x, emb, tgt)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    B.tp_device_status()
    B.tp_profile_enable(4096)
    ms = timed_loop(step, steps, world)
    prof = B.tp_profile_summary()
    B.tp_device_status()

    # End to end: inputs copied in from pinned host memory and the loss read
    # back every step, with the next step's inputs copied on a second stream.
    xh, th = inp["x"].pin_memory(), inp["target"].pin_memory()
    lossh = torch.empty(1, dtype=torch.float32).pin_memory()
    xd = [torch.empty_like(x) for _ in range(2)]
    td = [torch.empty_like(tgt) for _ in range(2)]

    def e2e_steps(n):
        comp, copy = torch.cuda.current_stream(), torch.cuda.Stream()
        in_ready, in_free = [torch.cuda.Event(), torch.cuda.Event()], [torch.cuda.Event(), torch.cuda.Event()]
        start = torch.cuda.Event()
        start.record(comp)
        copy.wait_event(start)

        def copy_in(k):
            b = k % 2
            with torch.cuda.stream(copy):
                if k >= 2:
                    copy.wait_event(in_free[b])
                xd[b].copy_(xh, non_blocking=True)
                td[b].copy_(th, non_blocking=True)
                in_ready[b].record(copy)

        copy_in(0)
        for k in range(n):
            b = k % 2
            comp.wait_event(in_ready[b])
            if k + 1 < n:
                copy_in(k + 1)
            xr(xd[b], emb, td[b])
            in_free[b].record(comp)
            lossh.copy_(xr.loss, non_blocking=True)   # 4 bytes, on the compute stream

    B.tp_profile_enable(0)   # a user's calls carry no profiling events
    e2e_steps(max(1, warmup // 2))
    ms_e2e = timed_loop(lambda: e2e_steps(steps), 1, world)
    return dict(ms=ms, prof=prof, ms_e2e=ms_e2e, h2d=x.numel() * 2 + tgt.numel() * 4, d2h=4)


# --------------------------------------------------------------------- CPU oracle

def oracle_layer_sample(d: TI.LayerDims, batch: int = 1):
    """fp64 oracle forward + backward of `batch` sequences of the layer workload."""
    from oracle import tp_oracle as O
    sd = TI.LayerDims(batch=batch, seq=d.seq, hidden=d.hidden, heads=d.heads, ffn=d.ffn, t=d.t,
                      causal=d.causal, padding=d.padding)
    inp = TI.make_layer_inputs(sd, seed=0)
    names = [k for k in TI.LAYER_PARAM_ORDER]
    p = O.to_f64({k: inp[k] for k in names})
    x = inp["x"].double().numpy()
    dy = inp["dy"].double().numpy()
    vl = inp["valid_len"].numpy() if "valid_len" in inp else None
    t0 = time.perf_counter()
    y, cache = O.layer_forward(x, p, sd.heads, sd.causal, vl, sd.ln_eps)
    O.layer_backward(dy, cache, p, sd.heads, sd.causal, vl)
    dt = time.perf_counter() - t0
    return TI.layer_flops(sd, inp.get("valid_len")), dt, sd


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    d = TI.WORKLOADS[args.workload]
    for _ in range(args.warmup):
        oracle_layer_sample(d)
    times = []
    flops = sd = None
    for _ in range(args.steps):
        flops, dt, sd = oracle_layer_sample(d)
        times.append(dt)
    total = sum(times)
    value = flops * args.steps / total / 1e12
    sample = (f"one sequence (batch 1 x seq {sd.seq} = {sd.tokens} tokens) of the {args.workload} "
              f"workload per step, fp64 layer forward + backward")
    line = {
        "impl": "reference", "metric": LAYER_METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": layer_config(d),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


LAYER_METRIC = "layer fwd+bwd TFLOP/s"
XENT_METRIC = "vocab-parallel xent tokens/s"


def layer_config(d: TI.LayerDims):
    return {"workload": "8.3B-scale GPT layer fwd+bwd" if d.hidden == 3072 else "layer fwd+bwd",
            "name": [k for k, v in TI.WORKLOADS.items() if v == d][0],
            "batch": d.batch, "seq": d.seq, "hidden": d.hidden, "heads": d.heads, "ffn": d.ffn,
            "t": d.t, "causal": d.causal, "global_batch": d.batch, "seq_len": d.seq,
            "parallelism": f"tp{d.t} logical partitions on one GPU; replicas across GPUs"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="gpt_8p3b_t8", choices=sorted(TI.WORKLOADS))
    ap.add_argument("--xent-workload", default="xent_50k_t8", choices=sorted(TI.XENT_WORKLOADS))
    ap.add_argument("--no-xent", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world, rank, local = dist_setup()
    if args.impl == "reference":
        rc = run_reference(args, world, rank)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return rc

    from tensor_transformer_layer_tp_b200 import binding as B
    from tensor_transformer_layer_tp_b200 import runner as R

    peaks, peak_kind = load_peaks()
    B.tp_profile_enable(4096)
    d = TI.WORKLOADS[args.workload]
    sampler = ClockSampler(local)
    sampler.start()
    L = bench_layer(d, args.steps, args.warmup, world, B, R)
    X = None if args.no_xent else bench_xent(TI.XENT_WORKLOADS[args.xent_workload], args.steps,
                                             args.warmup, world, B, R)
    PS = bench_partition_sum(d, min(args.steps, 10), args.warmup, world, B)
    clocks = sampler.stop()

    ms_step = L["ms"] / args.steps
    value = job_throughput(L["flops"], args.steps, world, L["ms"]) / 1e12
    gemm_k, gemm_ms = L["prof"]["gemm"]
    gemm_launches_per_step = gemm_k / args.steps
    gemm_ms_launch = gemm_ms / max(gemm_k, 1)
    gemm_flops_launch = L["gemm_flops"] / gemm_launches_per_step
    achieved = gemm_flops_launch / (gemm_ms_launch / 1e3) / 1e12
    peak = float(peaks["bf16_tflops"])
    traffic = profiled_traffic("gemm_tc_gpt_8p3b_t8.md", GEMM_SOURCES)
    kernels = {}
    total_prof_ms = sum(ms for _, ms in L["prof"].values())
    for name, (k, ms) in L["prof"].items():
        if k:
            kernels[name] = {"launches_per_step": k / args.steps, "ms_per_step": ms / args.steps,
                             "share": ms / total_prof_ms if total_prof_ms else None}
    line = {
        "metric": LAYER_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": dict(layer_config(d), flops_per_step=L["flops"],
                       l2="no flush: a step streams ~0.75 GB of activations and weights, > 126 MB L2"),
        "frac_of_peak": {"value": value / world / peak, "peak_tflops": peak, "peak": f"bf16 burst, {peak_kind}"},
        "roofline": {"kernel": "gemm_tc (tcgen05 GEMM, every linear of the layer)", "bound": "tensor",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_source": f"bf16_tflops ({peak_kind}, burst)",
                     "traffic": traffic, "launches_per_step": gemm_launches_per_step,
                     "flops_per_launch": gemm_flops_launch, "ms_per_launch": gemm_ms_launch},
        "e2e": {"value": job_throughput(L["flops"], args.steps, world, L["ms_e2e"]) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": L["h2d"], "d2h_bytes_per_step": L["d2h"]},
        "eager": {"value": job_throughput(L["flops"], args.steps, world, L["ms_eager"]) / 1e12,
                  "ms_per_step": L["ms_eager"] / args.steps,
                  "note": "the same step launched call by call (value: replayed as a CUDA graph)"},
        "gpu_launches": sum(k for k, _ in L["prof"].values()),
        "kernels": kernels,
        "clocks": clocks,
        "partition_sum": PS,
    }
    if X is not None:
        xd = TI.XENT_WORKLOADS[args.xent_workload]
        st_k, st_ms = X["prof"]["xent_stats"]
        gr_k, gr_ms = X["prof"]["xent_grad"]
        stream_ms = (st_ms + gr_ms) / args.steps
        sbytes = TI.xent_stream_bytes(xd)
        hbm = float(peaks["hbm_gbs"])
        xk, xms = X["prof"]["gemm"]
        line["xent"] = {
            "metric": XENT_METRIC, "value": job_throughput(xd.tokens, args.steps, world, X["ms"]),
            "unit": "tokens/s", "ms_per_step": X["ms"] / args.steps,
            "config": {"workload": "vocab-parallel output embedding + cross-entropy fwd+bwd",
                       "name": args.xent_workload, "tokens": xd.tokens, "hidden": xd.hidden,
                       "vocab": xd.vocab, "t": xd.t},
            "roofline": {"kernel": "xent_stats + xent_grad (logit streaming)", "bound": "hbm",
                         "achieved": sbytes / (stream_ms / 1e3) / 1e9, "peak": hbm, "unit": "GB/s",
                         "frac": sbytes / (stream_ms / 1e3) / 1e9 / hbm,
                         "peak_source": f"hbm_gbs ({peak_kind})",
                         "traffic": profiled_traffic("xent_stream_50k_t8.md", XENT_SOURCES,
                                                     "dram_bytes_per_step"),
                         "bytes_per_step": sbytes, "ms_per_step": stream_ms},
            "gemm_tflops": xent_gemm_tflops(xd, xms / args.steps),
            "e2e": {"value": job_throughput(xd.tokens, args.steps, world, X["ms_e2e"]), "unit": "tokens/s",
                    "h2d_bytes_per_step": X["h2d"], "d2h_bytes_per_step": X["d2h"]},
            "gpu_launches": sum(k for k, _ in X["prof"].values()),
            "kernels": {n: {"launches_per_step": k / args.steps, "ms_per_step": ms / args.steps}
                        for n, (k, ms) in X["prof"].items() if k},
        }
    B.tp_profile_enable(0)

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        flops, dt, sd = oracle_layer_sample(d, batch=d.batch)
        line["cpu_baseline"] = {
            "value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
            "sample": f"the whole layer batch ({sd.tokens} tokens), fp64 fwd+bwd once, {dt:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def xent_gemm_tflops(xd: TI.XentDims, ms):
    return TI.xent_flops(xd) / (ms / 1e3) / 1e12 if ms > 0 else None


if __name__ == "__main__":
    sys.exit(main())
