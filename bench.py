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
import dataclasses
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

def layer_setup(d: TI.LayerDims, B, runner_mod, **opts):
    inp = TI.make_layer_inputs(d, seed=0)
    dims = B.make_dims(d.t, d.batch, d.seq, d.hidden, d.heads, d.ffn, d.causal, d.ln_eps, **opts)
    params = runner_mod.params_to(TI.partition_layer_params(inp, d.t, d.heads), "cuda")
    r = runner_mod.LayerRunner(dims, params)
    x, dy = inp["x"].cuda(), inp["dy"].cuda()
    vl = inp["valid_len"].cuda() if "valid_len" in inp else None
    return inp, r, x, dy, vl


def gemm_flops_per_step(d: TI.LayerDims) -> float:
    n, h, f = d.tokens, d.hidden, d.ffn
    return float(3 * 2 * n * (3 * h * h + h * h + 2 * h * f))


def time_layer(r, x, dy, vl, steps, warmup, world, B):
    """Device time of `steps` forward+backward steps, two ways: call by call
    with the library's per-launch event profiler on (the per-kernel
    breakdown), and the same step captured once as a CUDA graph and replayed
    with profiling off (the headline number)."""
    def step():
        r.forward(x, vl)
        r.backward(x, dy, vl)

    B.tp_profile_enable(0)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    B.tp_device_status()
    B.tp_profile_enable(4096)
    ms_eager = timed_loop(step, steps, world)
    prof = B.tp_profile_summary()
    B.tp_profile_enable(0)
    B.tp_device_status()

    graph = r.capture_step(x, dy, vl)
    for _ in range(warmup):
        graph.replay()
    torch.cuda.synchronize()
    ms = timed_loop(graph.replay, steps, world)
    B.tp_device_status()
    del graph
    return ms, ms_eager, prof


def bench_layer(d: TI.LayerDims, steps, warmup, world, B, runner_mod, e2e=True):
    inp, r, x, dy, vl = layer_setup(d, B, runner_mod)
    flops = TI.layer_flops(d, inp.get("valid_len"))
    ms, ms_eager, prof = time_layer(r, x, dy, vl, steps, warmup, world, B)
    out = dict(ms=ms, ms_eager=ms_eager, prof=prof, flops=flops, gemm_flops=gemm_flops_per_step(d))
    if not e2e:
        return out

    # End to end through the public API: every step copies its inputs in from
    # pinned host memory and reads dX back.  Copies run on their own stream:
    # step k+1's inputs go into a second device buffer while step k computes,
    # and step k's dX is read back before step k+1's backward overwrites it.
    # Each input buffer pair has its forward and its backward call recorded
    # once as CUDA graphs (as a training loop would; separately, so that the
    # next forward can start while the previous dX is still being read back);
    # profiling stays off (a user's calls carry no events).
    xh, dyh = inp["x"].pin_memory(), inp["dy"].pin_memory()
    dxh = torch.empty_like(inp["x"]).pin_memory()
    xd = [torch.empty_like(x) for _ in range(2)]
    dyd = [torch.empty_like(dy) for _ in range(2)]
    for b in range(2):
        xd[b].copy_(x)
        dyd[b].copy_(dy)
    B.tp_profile_enable(0)

    def capture(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        return g

    gfwd = [capture(lambda b=b: r.forward(xd[b], vl)) for b in range(2)]
    gbwd = [capture(lambda b=b: r.backward(xd[b], dyd[b], vl)) for b in range(2)]
    torch.cuda.synchronize()

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
            gfwd[b].replay()
            if k + 1 < n:
                copy_in(k + 1)
            if k >= 1:
                comp.wait_event(dx_read)       # previous dX is on the host
            gbwd[b].replay()
            in_free[b].record(comp)
            done = ev()
            done.record(comp)
            with torch.cuda.stream(copy):
                copy.wait_event(done)
                dxh.copy_(r.dx, non_blocking=True)
                dx_read.record(copy)
        comp.wait_event(dx_read)

    e2e_steps(max(1, warmup // 2))
    out["ms_e2e"] = timed_loop(lambda: e2e_steps(steps), 1, world)
    out["h2d"] = (x.numel() + dy.numel()) * 2
    out["d2h"] = dxh.numel() * 2
    del gfwd, gbwd
    return out


def gemm_roofline(prof, steps, gemm_flops_step, peak, peak_kind):
    """The tcgen05 GEMM kernel against the bf16 peak: algorithmic GEMM flops
    per launch over its mean launch time from the event profiler."""
    k, ms = prof["gemm"]
    per_step = k / steps
    ms_launch = ms / max(k, 1)
    fl = gemm_flops_step / per_step
    achieved = fl / (ms_launch / 1e3) / 1e12
    return {"kernel": "gemm_tc (tcgen05 GEMM, every linear of the layer)", "bound": "tensor",
            "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "peak_source": f"bf16_tflops ({peak_kind}, burst)",
            "launches_per_step": per_step, "flops_per_launch": fl, "ms_per_launch": ms_launch}


def attention_roofline(d: TI.LayerDims, prof, steps, peak, peak_kind, valid_len=None):
    """The tcgen05 attention kernels against the bf16 peak: algorithmic flops
    (4 d per kept (query, key) pair per head forward, 8 d backward) over their
    measured time per step."""
    if d.causal:
        pairs = d.batch * d.seq * (d.seq + 1) // 2
    elif valid_len is not None:
        pairs = d.seq * int(sum(int(v) for v in valid_len))
    else:
        pairs = d.batch * d.seq * d.seq
    fwd_fl, bwd_fl = 4.0 * d.hidden * pairs, 8.0 * d.hidden * pairs
    out = {}
    for name, fl in (("attn_fwd", fwd_fl), ("attn_bwd", bwd_fl)):
        k, ms = prof[name]
        if k:
            ms_step = ms / steps
            tf = fl / (ms_step / 1e3) / 1e12
            out[name] = {"flops_per_step": fl, "ms_per_step": ms_step, "achieved": tf,
                         "peak": peak, "unit": "TFLOP/s", "frac": tf / peak,
                         "peak_source": f"bf16_tflops ({peak_kind}, burst)"}
    return out


def kernel_breakdown(prof, steps):
    total = sum(ms for _, ms in prof.values())
    return {name: {"launches_per_step": k / steps, "ms_per_step": ms / steps,
                   "share": ms / total if total else None}
            for name, (k, ms) in prof.items() if k}


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


def bench_xent(d: TI.XentDims, steps, warmup, world, B, runner_mod, e2e=True, explicit=False):
    inp = TI.make_xent_inputs(d, seed=0)
    xr = runner_mod.XentRunner(d.t, d.tokens, d.hidden, d.vocab, explicit=explicit)
    x = inp["x"].cuda()
    emb = [e.cuda() for e in TI.partition_vocab(inp["emb"], d.t)]
    tgt = inp["target"].cuda()

    def step():
        xr(x, emb, tgt)

    B.tp_profile_enable(0)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    B.tp_device_status()
    ms = timed_loop(step, steps, world)          # no profiling events in the timed loop
    B.tp_device_status()
    # per-kernel breakdown from a separate loop of the same steps, profiled
    B.tp_profile_enable(4096)
    timed_loop(step, steps, world)
    prof = B.tp_profile_summary()
    B.tp_profile_enable(0)
    B.tp_device_status()
    out = dict(ms=ms, prof=prof)
    if not e2e:
        return out

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

    e2e_steps(max(1, warmup // 2))
    out["ms_e2e"] = timed_loop(lambda: e2e_steps(steps), 1, world)
    out["h2d"] = x.numel() * 2 + tgt.numel() * 4
    out["d2h"] = 4
    return out


# --------------------------------------------------------------------- CPU oracle

def oracle_layer_sample(d: TI.LayerDims, batch: int | None = None):
    """fp64 oracle forward + backward of the first `batch` sequences of the
    layer workload (all of them by default).  Returns (flops, seconds, dims)."""
    from oracle import tp_oracle as O
    batch = d.batch if batch is None else batch
    d = dataclasses.replace(d, vocab=0)     # layer-only: the upstream gradient is drawn
    inp = TI.make_layer_inputs(d, seed=0)
    sd = dataclasses.replace(d, batch=batch)
    p = O.to_f64({k: inp[k] for k in TI.LAYER_PARAM_ORDER})
    x = inp["x"][:batch].double().numpy()
    dy = inp["dy"][:batch].double().numpy()
    vl = inp["valid_len"][:batch].numpy() if "valid_len" in inp else None
    t0 = time.perf_counter()
    y, cache = O.layer_forward(x, p, sd.heads, sd.causal, vl, sd.ln_eps)
    O.layer_backward(dy, cache, p, sd.heads, sd.causal, vl)
    dt = time.perf_counter() - t0
    return TI.layer_flops(sd, vl), dt, sd


def oracle_xent_sample(d: TI.XentDims, tokens: int):
    """fp64 oracle loss forward + backward on the first `tokens` tokens of the
    loss workload.  Returns (tokens, seconds)."""
    from oracle import tp_oracle as O
    inp = TI.make_xent_inputs(d, seed=0)
    x = inp["x"][:tokens].double().numpy()
    e = inp["emb"].double().numpy()
    y = inp["target"][:tokens].numpy()
    t0 = time.perf_counter()
    _, _, lse = O.cross_entropy(x, e, y)
    O.cross_entropy_backward(x, e, y, lse)
    return tokens, time.perf_counter() - t0


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def layer_cpu_baseline(d: TI.LayerDims, batch: int | None = None):
    flops, dt, sd = oracle_layer_sample(d, batch)
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
            "sample": f"{sd.batch} of {d.batch} sequences ({sd.tokens} tokens) of the workload, "
                      f"fp64 layer fwd+bwd once, {dt:.1f} s"}


def xent_cpu_baseline(d: TI.XentDims, tokens: int = 1024):
    n, dt = oracle_xent_sample(d, tokens)
    return {"value": n / dt, "unit": "tokens/s", "cores": cpu_cores(), "kind": "oracle",
            "sample": f"{n} of {d.tokens} tokens of the workload (the unpartitioned loss; every t "
                      f"computes the same function), fp64 fwd+bwd once, {dt:.1f} s"}


LAYER_METRIC = "layer fwd+bwd TFLOP/s"
XENT_METRIC = "vocab-parallel xent tokens/s"


def layer_config(d: TI.LayerDims, name: str):
    workload = {"gpt_8p3b_t8": "8.3B-scale GPT layer fwd+bwd",
                "bert_3p9b_t4": "3.9B-scale BERT layer fwd+bwd (bidirectional, key padding)"}.get(
        name, "GPT-2 355M-shape layer fwd+bwd" if d.hidden == 1024 else "layer fwd+bwd")
    return {"workload": workload, "name": name,
            "batch": d.batch, "seq": d.seq, "hidden": d.hidden, "heads": d.heads, "ffn": d.ffn,
            "t": d.t, "causal": d.causal, "padding": d.padding, "global_batch": d.batch,
            "seq_len": d.seq,
            "parallelism": f"tp{d.t} logical partitions on one GPU; replicas across GPUs",
            "l2": "no flush: a step streams its activations and weights, far more than the 126 MB L2"}


def xent_config(d: TI.XentDims, name: str):
    return {"workload": "vocab-parallel output embedding + cross-entropy fwd+bwd", "name": name,
            "tokens": d.tokens, "hidden": d.hidden, "vocab": d.vocab, "t": d.t,
            "l2": "no flush: the logits alone are 1.6 GB, far more than the 126 MB L2"}


def run_reference(args, world, rank):
    """The reference arm: the fp64 CPU oracle of the same workload on the host
    cores.  A timed step is the whole batch (the same work as one GPU step);
    warm-up steps are one-sequence samples (they only warm the host's caches
    and allocator)."""
    if rank != 0:
        return 0
    d = TI.WORKLOADS[args.workload]
    for _ in range(args.warmup):
        oracle_layer_sample(d, batch=1)
    times = []
    flops = None
    for _ in range(args.steps):
        flops, dt, _ = oracle_layer_sample(d)
        times.append(dt)
    total = sum(times)
    value = flops * args.steps / total / 1e12
    sample = (f"the whole batch ({d.batch} x seq {d.seq} = {d.tokens} tokens) of the workload "
              f"per timed step, fp64 layer forward + backward; warm-up steps one sequence")
    line = {
        "impl": "reference", "metric": LAYER_METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": layer_config(d, args.workload),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


SUB_LAYER_WORKLOADS = ("gpt2_355m_t1", "gpt2_355m_t2", "gpt2_355m_t4", "bert_3p9b_t4")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="gpt_8p3b_t8", choices=sorted(TI.WORKLOADS))
    ap.add_argument("--xent-workload", default="xent_50k_t8", choices=sorted(TI.XENT_WORKLOADS))
    ap.add_argument("--no-xent", action="store_true")
    ap.add_argument("--no-sub", action="store_true", help="skip the other workloads' lines")
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
    peak = float(peaks["bf16_tflops"])
    hbm = float(peaks["hbm_gbs"])
    d = TI.WORKLOADS[args.workload]
    sampler = ClockSampler(local)
    sampler.start()
    L = bench_layer(d, args.steps, args.warmup, world, B, R)
    xd = TI.XENT_WORKLOADS[args.xent_workload]
    X = None if args.no_xent else bench_xent(xd, args.steps, args.warmup, world, B, R)
    XE = None if args.no_xent else bench_xent(xd, min(args.steps, 20), args.warmup, world, B, R,
                                              e2e=False, explicit=True)
    PS = bench_partition_sum(d, min(args.steps, 10), args.warmup, world, B)
    variants = {}
    if not args.no_sub:
        # the same workload with the layer's options on: Philox dropout (0.1 on
        # the attention probabilities and the hidden outputs), and activation
        # recomputation (the forward saves only LN statistics and lse; the
        # backward rebuilds the rest).  Same algorithmic flop count, so the
        # extra work of each shows as a lower rate.
        for vname, opts in (("dropout_0.1", dict(dropout_attn=0.1, dropout_hidden=0.1, seed=1234)),
                            ("recompute", dict(recompute=True))):
            vinp, vr, vx, vdy, vvl = layer_setup(d, B, R, **opts)
            vflops = TI.layer_flops(d, vinp.get("valid_len"))
            vms, _, vprof = time_layer(vr, vx, vdy, vvl, min(args.steps, 20), args.warmup, world, B)
            vsteps = min(args.steps, 20)
            variants[vname] = {"metric": LAYER_METRIC,
                               "value": job_throughput(vflops, vsteps, world, vms) / 1e12,
                               "unit": "TFLOP/s", "ms_per_step": vms / vsteps, "steps": vsteps,
                               "options": {k: v for k, v in opts.items()},
                               "saved_bytes": vr.saved.numel(),
                               "kernels": kernel_breakdown(vprof, vsteps)}
            del vr
        torch.cuda.empty_cache()
    sub_steps = min(args.steps, 20)
    subs, xsubs = {}, {}
    if not args.no_sub:
        for name in SUB_LAYER_WORKLOADS:
            if name == args.workload:
                continue
            sd = TI.WORKLOADS[name]
            inp, r, x, dy, vl = layer_setup(sd, B, R)
            flops = TI.layer_flops(sd, inp.get("valid_len"))
            ms, ms_eager, prof = time_layer(r, x, dy, vl, sub_steps, args.warmup, world, B)
            del r
            val = job_throughput(flops, sub_steps, world, ms) / 1e12
            subs[name] = {"metric": LAYER_METRIC, "value": val, "unit": "TFLOP/s",
                          "ms_per_step": ms / sub_steps, "steps": sub_steps,
                          "config": dict(layer_config(sd, name), flops_per_step=flops),
                          "frac_of_peak": val / world / peak,
                          "roofline": gemm_roofline(prof, sub_steps, gemm_flops_per_step(sd), peak,
                                                    peak_kind),
                          "attention": attention_roofline(sd, prof, sub_steps, peak, peak_kind,
                                                          inp.get("valid_len")),
                          "kernels": kernel_breakdown(prof, sub_steps)}
            if "valid_len" in inp:
                subs[name]["config"]["valid_len"] = TI.padded_len_summary(inp["valid_len"])
        if not args.no_xent:
            for name, sx in TI.XENT_WORKLOADS.items():
                if name == args.xent_workload:
                    continue
                XS = bench_xent(sx, sub_steps, args.warmup, world, B, R, e2e=False)
                xsubs[name] = xent_line(sx, name, XS, sub_steps, world, hbm, peak, peak_kind)
        torch.cuda.empty_cache()
    clocks = sampler.stop()

    ms_step = L["ms"] / args.steps
    value = job_throughput(L["flops"], args.steps, world, L["ms"]) / 1e12
    roof = gemm_roofline(L["prof"], args.steps, L["gemm_flops"], peak, peak_kind)
    roof["traffic"] = profiled_traffic("gemm_tc_gpt_8p3b_t8.md", GEMM_SOURCES)
    launches_per_step = sum(k for k, _ in L["prof"].values()) / args.steps
    line = {
        "metric": LAYER_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": layer_config(d, args.workload),
        "flops_per_step": L["flops"],
        "frac_of_peak": {"value": value / world / peak, "peak_tflops": peak, "peak": f"bf16 burst, {peak_kind}"},
        "roofline": roof,
        "e2e": {"value": job_throughput(L["flops"], args.steps, world, L["ms_e2e"]) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": L["h2d"], "d2h_bytes_per_step": L["d2h"]},
        "eager": {"value": job_throughput(L["flops"], args.steps, world, L["ms_eager"]) / 1e12,
                  "ms_per_step": L["ms_eager"] / args.steps,
                  "note": "the same step launched call by call with per-launch profiling events, "
                          "every launch on one stream (value: replayed as a CUDA graph, no events, "
                          "weight-gradient GEMMs on the backward's side stream)"},
        "gpu_launches": int(round(launches_per_step * args.steps)),
        "gpu_launches_per_step": launches_per_step,
        "kernels": kernel_breakdown(L["prof"], args.steps),
        "attention": attention_roofline(d, L["prof"], args.steps, peak, peak_kind),
        "clocks": clocks,
        "partition_sum": PS,
    }
    if variants:
        line["variants"] = variants
    if X is not None:
        line["xent"] = xent_line(xd, args.xent_workload, X, args.steps, world, hbm, peak, peak_kind)
        line["xent_explicit"] = xent_line(xd, args.xent_workload, XE, min(args.steps, 20), world, hbm,
                                          peak, peak_kind, explicit=True)
    if subs:
        line["configs"] = subs
    if xsubs:
        line["xent_configs"] = xsubs

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = layer_cpu_baseline(d)
        for name, sub in subs.items():
            sd = TI.WORKLOADS[name]
            # BERT: 2 of 16 sequences bound the CPU time; the 355M batch runs whole
            sub["cpu_baseline"] = layer_cpu_baseline(sd, None if sd.hidden <= 1024 else 2)
        if X is not None:
            xb = xent_cpu_baseline(xd)
            line["xent"]["cpu_baseline"] = xb
            for sub in xsubs.values():
                sub["cpu_baseline"] = xb
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def xent_line(xd: TI.XentDims, name, X, steps, world, hbm, peak, peak_kind, explicit=False):
    """The loss line.  Fused path: the dominant kernel is the logits GEMM with
    the statistics epilogue (tensor roofline over all three GEMMs' flops); the
    one bandwidth-bound pass is the bf16 gradient.  Explicit path: the fp32
    logit streams (statistics + gradient) against HBM."""
    gr_k, gr_ms = X["prof"]["xent_grad"]
    st_k, st_ms = X["prof"]["xent_stats"]
    xk, xms = X["prof"]["gemm"]
    gemm_ms = xms / steps
    gemm_tf = xent_gemm_tflops(xd, gemm_ms)
    if explicit:
        stream_ms = (st_ms + gr_ms) / steps
        sbytes = TI.xent_stream_bytes(xd)
        skernel = "xent_stats + xent_grad (fp32 logit streaming)"
    else:
        stream_ms = gr_ms / steps
        sbytes = TI.xent_fused_stream_bytes(xd)
        skernel = "xent_grad_bf16 (bf16 logits -> bf16 gradient, in place)"
    stream = {"kernel": skernel, "bound": "hbm", "achieved": sbytes / (stream_ms / 1e3) / 1e9,
              "peak": hbm, "unit": "GB/s", "frac": sbytes / (stream_ms / 1e3) / 1e9 / hbm,
              "peak_source": f"hbm_gbs ({peak_kind})", "bytes_per_step": sbytes,
              "ms_per_step": stream_ms}
    gemm = {"kernel": "gemm_tc (logits GEMM with the loss-statistics epilogue, dE and dX GEMMs)",
            "bound": "tensor", "achieved": gemm_tf, "peak": peak, "unit": "TFLOP/s",
            "frac": gemm_tf / peak if gemm_tf else None, "peak_source": f"bf16_tflops ({peak_kind}, burst)",
            "flops_per_step": TI.xent_flops(xd), "ms_per_step": gemm_ms, "launches_per_step": xk / steps}
    if explicit:
        stream["traffic"] = (profiled_traffic("xent_stream_50k_t8.md", XENT_SOURCES, "dram_bytes_per_step")
                             if xd.t == 8 else None)
        roof, other = stream, gemm
    else:
        gemm["traffic"] = None
        roof, other = gemm, stream
    out = {
        "metric": XENT_METRIC, "value": job_throughput(xd.tokens, steps, world, X["ms"]),
        "unit": "tokens/s", "ms_per_step": X["ms"] / steps, "steps": steps,
        "config": dict(xent_config(xd, name), path="explicit fp32 logits" if explicit else "fused"),
        "roofline": roof,
        "roofline_other": other,
        "gpu_launches_per_step": sum(k for k, _ in X["prof"].values()) / steps,
        "kernels": {n: {"launches_per_step": k / steps, "ms_per_step": ms / steps}
                    for n, (k, ms) in X["prof"].items() if k},
    }
    if "ms_e2e" in X:
        out["e2e"] = {"value": job_throughput(xd.tokens, steps, world, X["ms_e2e"]), "unit": "tokens/s",
                      "h2d_bytes_per_step": X["h2d"], "d2h_bytes_per_step": X["d2h"]}
    return out


def xent_gemm_tflops(xd: TI.XentDims, ms):
    return TI.xent_flops(xd) / (ms / 1e3) / 1e12 if ms > 0 else None


if __name__ == "__main__":
    sys.exit(main())
