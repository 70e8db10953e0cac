#!/usr/bin/env python
"""Benchmark of the DoRA hot path on B200: factored row norm + fused compose
forward + compose backward on the 8192 x 8192, r = 384, bf16 module with
8192 tokens (synthetic, seeded inputs).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    torchrun --nproc-per-node N bench.py --gpus N ...        (N > 1)

One step = dora_factored_norm -> dora_compose_fwd -> dora_compose_bwd on
inputs already resident in HBM.  The headline value is the factored norm's
TFLOP/s (algorithmic FLOPs over the norm launches' CUDA-event time, summed
over ranks); compose forward / backward HBM GB/s and every kernel's
roofline fraction ride along in the same JSON line.  Multi-GPU runs are
independent replicas (weak scaling): the path has no exchange step.

``--impl reference`` times the fp64 CPU oracle (the reference arm) on the
host cores on a bounded sample of the same workload.  ``--sweep`` runs the
rank/shape sweep instead (the norm over ranks 16..768, the compose over
token counts 1024..65536, each call timed alone after an L2 flush) and
prints its points.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from factored_weight_norm_b200 import workloads as WL  # noqa: E402

METRIC = "factored-norm TFLOP/s + fused-compose HBM GB/s (d=8192, r=384, bf16), % roofline"
# bounded oracle sample per step: norm rows, compose tokens (about 1 s of CPU work)
ORACLE_SAMPLE = (1024, 512)
ORACLE_MIN_SECONDS = 10.0  # repeat the sample until this much CPU time is measured
ORACLE_MAX_REPS = 200
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------ algorithmic work
def norm_flops(d_out, d_in, r):
    """Fixed count: cross GEMM + Gram + Gram quadratic form + base norm + row dot."""
    return 2 * d_out * d_in * r + 2 * r * r * d_in + 2 * d_out * r * r + 2 * d_out * d_in + 2 * d_out * r


def norm_bytes(d_out, d_in, r, e=2):
    return e * (d_out * d_in + r * d_in + d_out * r) + 4 * d_out


def fwd_bytes(T, d_out, e=2):
    return 3 * e * T * d_out + 8 * d_out


def bwd_bytes(T, d_out, e=2):
    return 5 * e * T * d_out + 12 * d_out


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# the sources that define each measured kernel family's code and launches
TRAFFIC_SOURCES = {
    "norm": ("sm100_ptx.cuh", "norm_tc.cuh", "gram_cluster.cuh", "dora_api.cu"),
    "compose_fwd": ("sm100_ptx.cuh", "compose.cuh", "dora_api.cu"),
    "compose_bwd": ("sm100_ptx.cuh", "compose.cuh", "dora_api.cu"),
}


def source_digest(names=None):
    """sha256 prefix of the listed csrc files (all .cu/.cuh files by default)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "factored_weight_norm_b200", "csrc")
    if names is None:
        names = [n for n in os.listdir(csrc) if n.endswith((".cu", ".cuh"))]
    for name in sorted(names):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_traffic():
    """DRAM bytes per launch from the committed ncu summary, keyed by (kernel,
    workload label): valid only for the workload it was captured on and for
    the kernel sources it was captured from."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    out = {}
    if not os.path.exists(p):
        return out
    for line in open(p):
        parts = line.split()
        if len(parts) >= 4 and not line.startswith("#") and parts[0] in TRAFFIC_SOURCES:
            if parts[1] == source_digest(TRAFFIC_SOURCES[parts[0]]):
                out[(parts[0], parts[3])] = float(parts[2])
    return out


def traffic_labels(wl):
    """Workload labels of the traffic rows: the norm's depends on the weights'
    shape, the compose kernels' on the token count too."""
    return {"norm": wl.name, "compose_fwd": f"{wl.name}_T{wl.tokens}", "compose_bwd": f"{wl.name}_T{wl.tokens}"}


L2_BYTES = 126 << 20


def step_bytes(wl):
    e = 2 if wl.dtype == "bf16" else 4
    return norm_bytes(wl.d_out, wl.d_in, wl.r, e) + fwd_bytes(wl.tokens, wl.d_out, e) + bwd_bytes(wl.tokens, wl.d_out, e)


def l2_statement(wl, flushed):
    mb = step_bytes(wl) / 1e6
    if flushed:
        return (f"L2 cleaned before every step (256 MB written, then another 256 MB read; untimed), so a step "
                f"neither finds its inputs in L2 nor pays for the previous step's dirty lines; a step streams "
                f"{mb:.0f} MB; its three calls run back to back")
    return f"no flush: each step streams {mb:.0f} MB (norm inputs, then 3 activation reads + 1 write, then 3 reads + 2 writes)"


DTYPE_LABEL = {"bf16": "bf16", "f32": "f32"}


# ---------------------------------------------------------------- clocks
class ClockSampler:
    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        self.path = f"/tmp/dora_clocks_{os.getpid()}.csv"
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={q}", "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        self.proc.wait(timeout=10)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                cur, mx, pw = float(f[1]), float(f[2]), float(f[3])
            except ValueError:
                continue
            smax = mx
            if pw > 250 or cur > 0.5 * mx:  # under load
                sm.append(cur)
                for nm, v in zip(names, f[5:9]):
                    if v.lower() == "active":
                        reasons.add(nm)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "samples_under_load": len(sm), "reasons": sorted(reasons)}


# ------------------------------------------------------------- our arm
def max_over_ranks(values, world, device):
    """Element-wise maximum of a list of floats over all ranks (the slowest
    rank's time decides every multi-GPU number); identity when world == 1."""
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def workload_of(args):
    wl = WL.WORKLOADS[args.workload]
    tokens = getattr(args, "tokens", None)
    return wl.with_(tokens=tokens) if tokens else wl


def run_ours(args, rank, world, local_rank):
    from factored_weight_norm_b200 import dora as D

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = workload_of(args)
    T, d_out, d_in, r, s = wl.tokens, wl.d_out, wl.d_in, wl.r, wl.s
    W, A, B, m = WL.make_weights(wl, dev)
    _, base, lora = WL.make_activations(wl, W, A, B, dev)
    dy = WL.make_grad(wl, dev)
    n = torch.empty(d_out, dtype=torch.float32, device=dev)
    y = torch.empty_like(base)
    d_base = torch.empty_like(base)
    d_lora = torch.empty_like(base)
    d_m = torch.empty(d_out, dtype=torch.float32, device=dev)
    ws_n = torch.empty(D.dora_factored_norm_workspace_size(d_out, d_in, r), dtype=torch.uint8, device=dev)
    ws_b = torch.empty(D.dora_compose_bwd_workspace_size(T, d_out), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    # L2 is cleaned before every timed step (untimed): the norm then streams W
    # without also writing back the previous step's compose-backward output;
    # a second pass without the clean is reported beside it
    flush = L2Flush(dev)

    def step(ev=None, clean=True):
        if clean:
            flush()
        if ev is not None:
            ev[0].record(stream)
        D.dora_factored_norm(W, A, B, s, n_out=n, workspace=ws_n)
        if ev is not None:
            ev[1].record(stream)
        D.dora_compose_fwd(base, lora, m, n, s, y=y)
        if ev is not None:
            ev[2].record(stream)
        D.dora_compose_bwd(dy, base, lora, m, n, s, d_base, d_lora, d_m, ws_b)
        if ev is not None:
            ev[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if D.dora_device_status() != D.DORA_OK:
        raise RuntimeError("device status not OK after warm-up")

    sampler = ClockSampler(local_rank) if rank == 0 else None
    if sampler:
        sampler.start()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    # an untimed ~1 ms spin first, so that the host enqueues the timed steps
    # ahead of the GPU: no launch of a timed step waits on the host (the
    # clock sampler's process start, the first calls' host work)
    head_start = getattr(torch.cuda, "_sleep", None)
    if head_start is not None:
        head_start(2_000_000)
    launches0 = D.dora_launch_count()
    for k in range(args.steps):
        step(evs[k])
    launches = D.dora_launch_count() - launches0
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop() if sampler else None
    status = D.dora_device_status()

    per_step = {k: [e[i].elapsed_time(e[i + 1]) * 1e-3 for e in evs] for i, k in enumerate(("norm", "fwd", "bwd"))}
    t_norm = sum(per_step["norm"]) / args.steps
    t_fwd = sum(per_step["fwd"]) / args.steps
    t_bwd = sum(per_step["bwd"]) / args.steps
    t_total = (t_norm + t_fwd + t_bwd) * args.steps  # the cleans between steps are not the step's
    spread = {k: {"median_us": statistics.median(v) * 1e6, "min_us": min(v) * 1e6, "max_us": max(v) * 1e6}
              for k, v in per_step.items()}

    # the same steps back to back without the clean: the norm then also
    # writes back what the previous compose backward left dirty in L2
    evs2 = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    for k in range(min(3, args.steps)):
        step(clean=False)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    if head_start is not None:
        head_start(2_000_000)
    for k in range(args.steps):
        step(evs2[k], clean=False)
    torch.cuda.synchronize()
    u_norm = sum(e[0].elapsed_time(e[1]) for e in evs2) / args.steps * 1e-3
    u_fwd = sum(e[1].elapsed_time(e[2]) for e in evs2) / args.steps * 1e-3
    u_bwd = sum(e[2].elapsed_time(e[3]) for e in evs2) / args.steps * 1e-3
    u_total = evs2[0][0].elapsed_time(evs2[-1][3]) * 1e-3
    t_total, t_norm, t_fwd, t_bwd, u_total, u_norm, u_fwd, u_bwd = max_over_ranks(
        [t_total, t_norm, t_fwd, t_bwd, u_total, u_norm, u_fwd, u_bwd], world, dev)

    # ---- end to end through the Python API with pinned host buffers
    e2e = run_e2e(args, D, dev, wl, W, A, B, m, base, lora, dy, n, y, d_base, d_lora, d_m, ws_n, ws_b, world)
    ctx = rank == 0 and not getattr(args, "no_context", False)
    bf16_ctx = ctx and wl.dtype == "bf16"  # the fused linear and the norm backward take bf16 only
    # each context measurement starts from an idle GPU (a short host pause),
    # and the power-hungry fused-linear GEMMs run last
    def idle_then(f):
        torch.cuda.synchronize()
        time.sleep(0.25)
        return f()

    dense = idle_then(lambda: run_dense_comparator(D, dev, W, A, B, s, ws_n)) if ctx else None
    batched = idle_then(lambda: run_batched_context(D, dev)) if ctx else None
    norm_bwd = idle_then(lambda: run_norm_backward_context(D, dev, wl, W, A, B, n)) if bf16_ctx else None
    fused = idle_then(lambda: run_fused_linear_context(D, dev, wl, W, A, B, m, n)) if bf16_ctx else None
    return dict(t_total=t_total, t_norm=t_norm, t_fwd=t_fwd, t_bwd=t_bwd, clocks=clocks, status=status, e2e=e2e,
                wl=wl, dense=dense, batched=batched, fused=fused, norm_bwd=norm_bwd, launches=launches,
                flushed=True, unflushed=dict(t_total=u_total, t_norm=u_norm, t_fwd=u_fwd, t_bwd=u_bwd), spread=spread)


def run_dense_comparator(D, dev, W, A, B, s, ws_n, reps=10):
    """Context, not our path: the row norm as the frameworks the pages survey
    compute it, by materialising the dense [d_out, d_in] product B A in the
    weight dtype (torch matmul, i.e. cuBLAS) and taking ||W + s B A||_row.
    Returns its time and transient memory beside the factored norm's."""
    def dense():
        return torch.linalg.vector_norm((W + s * (B @ A)).float(), dim=1)

    def timed(f):
        for _ in range(3):
            f()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            f()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps * 1e3

    n = torch.empty(W.shape[0], dtype=torch.float32, device=dev)
    t_dense = timed(dense)
    t_factored = timed(lambda: D.dora_factored_norm(W, A, B, s, n_out=n, workspace=ws_n))
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats(dev)
    before = torch.cuda.memory_allocated(dev)
    dense()
    torch.cuda.synchronize()
    dense_peak = torch.cuda.max_memory_allocated(dev) - before
    return {"what": "row norm by materialising B A (torch matmul, bf16) vs the factored norm; context only",
            "dense_time_us": t_dense, "factored_time_us": t_factored,
            "dense_transient_bytes": dense_peak, "factored_workspace_bytes": ws_n.numel()}


def linear_flops(T, d_in, d_out, r):
    """Algorithmic FLOPs of the fused linear forward: x W^T and P B^T (K = d_in + r
    over T x d_out outputs) plus P = x A^T (T x r x d_in)."""
    return 2.0 * T * d_out * (d_in + r) + 2.0 * T * r * d_in


def run_fused_linear_context(D, dev, wl, W, A, B, m, n, reps=10):
    """The compose fused into the producing GEMMs (dora_fused_linear_fwd) at the
    workload's shape (tokens x d_in -> d_out, rank r, with a bias), against the
    unfused path a framework runs: cuBLAS x W^T (+ b), cuBLAS (x A^T) B^T, then
    dora_compose_fwd.  Inputs and outputs (x, W, y: 134 MB each at 8192^2) are
    larger than L2.  Context beside the step, timed with CUDA events."""
    g = torch.Generator(device=dev)
    g.manual_seed(4321)
    T = wl.tokens
    x = torch.randn(T, wl.d_in, generator=g, device=dev).to(torch.bfloat16)
    b = (0.1 * torch.randn(wl.d_out, generator=g, device=dev)).to(torch.bfloat16)
    mf = m.float().contiguous()
    y = torch.empty(T, wl.d_out, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(D.dora_fused_linear_fwd_workspace_size(T, wl.r), dtype=torch.uint8, device=dev)
    base = torch.empty_like(y)
    lora = torch.empty_like(y)

    def fused():
        D.dora_fused_linear_fwd(x, W, A, B, mf, n, wl.s, bias=b, y=y, workspace=ws)

    def unfused():
        torch.matmul(x, W.t(), out=base)
        base.add_(b)
        torch.matmul(torch.matmul(x, A.t()), B.t(), out=lora)
        D.dora_compose_fwd(base, lora, mf, n, wl.s, y=y, bias=b)

    def timed(f):
        for _ in range(3):
            f()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            f()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps * 1e-3

    t_f = timed(fused)
    t_u = timed(unfused)
    F = linear_flops(T, wl.d_in, wl.d_out, wl.r)
    return {"what": f"y = b + (m/n)(x W^T + s (x A^T) B^T) for {T} tokens, {wl.d_in} -> {wl.d_out}, r = {wl.r}, bf16, "
                    "bias: dora_fused_linear_fwd vs cuBLAS GEMMs + dora_compose_fwd; context only",
            "fused_us": t_f * 1e6, "unfused_us": t_u * 1e6, "flops": F, "fused_tflops": F / t_f / 1e12,
            "speedup_vs_unfused": t_u / t_f, "gpu_launches_per_call": 2, "device_status": D.dora_device_status()}


def norm_backward_flops(d_out, d_in, r):
    """Algorithmic FLOPs of the attached-norm backward: dB = s c * ([W | B] [A | sG]^T)
    and dA = [(s c B)^T | s^2 H] [W ; A], plus G = A A^T and H = (c B)^T B."""
    return 4.0 * d_out * r * (d_in + r) + 2.0 * r * r * (d_in + d_out)


def run_norm_backward_context(D, dev, wl, W, A, B, n, reps=10):
    """Gradients of the row norms into A and B (norm kept attached):
    dora_factored_norm_bwd against torch.autograd through the dense
    ||W + s B A||_row (bf16 product, fp32 norm) that frameworks would run.
    Context beside the step, CUDA events."""
    g = torch.Generator(device=dev)
    g.manual_seed(2468)
    d_n = torch.randn(wl.d_out, generator=g, device=dev)
    dA = torch.empty(wl.r, wl.d_in, device=dev)
    dB = torch.empty(wl.d_out, wl.r, device=dev)
    ws = torch.empty(D.dora_factored_norm_bwd_workspace_size(wl.d_out, wl.d_in, wl.r), dtype=torch.uint8, device=dev)
    Ab = A.detach().clone().requires_grad_()
    Bb = B.detach().clone().requires_grad_()

    def factored():
        D.dora_factored_norm_bwd(W, A, B, wl.s, n, d_n, dA=dA, dB=dB, workspace=ws)

    def dense():
        Ab.grad = None
        Bb.grad = None
        torch.linalg.vector_norm((W + wl.s * (Bb @ Ab)).float(), dim=1).backward(d_n)

    def timed(f):
        for _ in range(3):
            f()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            f()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps * 1e-3

    t_f = timed(factored)
    t_d = timed(dense)
    F = norm_backward_flops(wl.d_out, wl.d_in, wl.r)
    return {"what": f"dL/dA, dL/dB through n = ||W + sBA||_row at {wl.d_out} x {wl.d_in}, r = {wl.r}, bf16: "
                    "dora_factored_norm_bwd vs torch.autograd of the dense norm; context only",
            "factored_us": t_f * 1e6, "dense_us": t_d * 1e6, "flops": F, "factored_tflops": F / t_f / 1e12,
            "speedup_vs_dense": t_d / t_f, "workspace_bytes": ws.numel(), "gpu_launches_per_call": 5,
            "device_status": D.dora_device_status()}


# the seven adapted projections of one decoder block of an 8B-class model
# (q, k, v, o, gate, up, down) as (d_out, d_in)
BLOCK_SHAPES = [(4096, 4096), (1024, 4096), (1024, 4096), (4096, 4096), (14336, 4096), (14336, 4096), (4096, 14336)]


def run_batched_context(D, dev, blocks=16, r=384, s=0.5, reps=3):
    """Context for the many-module path: the norms of every adapted module
    of `blocks` decoder blocks (7 modules each, bf16, r = 384, synthetic),
    computed by one dora_factored_norm_batched call versus one
    dora_factored_norm call per module, both timed with CUDA events."""
    g = torch.Generator(device=dev)
    g.manual_seed(1234)
    mods = []
    for _ in range(blocks):
        for d_out, d_in in BLOCK_SHAPES:
            W = (torch.randn(d_out, d_in, generator=g, device=dev) * 0.02).bfloat16()
            A = ((torch.rand(r, d_in, generator=g, device=dev) * 2 - 1) / d_in ** 0.5).bfloat16()
            B = (torch.randn(d_out, r, generator=g, device=dev) * 0.002).bfloat16()
            mods.append((W, A, B, s))
    outs = [torch.empty(m[0].shape[0], dtype=torch.float32, device=dev) for m in mods]
    ws_b = torch.empty(D.dora_factored_norm_batched_workspace_size(mods), dtype=torch.uint8, device=dev)
    ws_1 = torch.empty(max(D.dora_factored_norm_workspace_size(m[0].shape[0], m[0].shape[1], r) for m in mods),
                       dtype=torch.uint8, device=dev)

    def batched():
        D.dora_factored_norm_batched(mods, n_outs=outs, workspace=ws_b)

    def one_by_one():
        for (W, A, B, sm), n in zip(mods, outs):
            D.dora_factored_norm(W, A, B, sm, n_out=n, workspace=ws_1)

    def timed(f):
        f()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            f()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps * 1e3

    t_b, t_1 = timed(batched), timed(one_by_one)
    F = sum(norm_flops(m[0].shape[0], m[0].shape[1], r) for m in mods)
    return {"what": f"norms of {len(mods)} modules ({blocks} decoder blocks x q,k,v,o,gate,up,down of an "
                    f"8B-class model, r = {r}, bf16, synthetic): one batched call vs one call per module",
            "modules": len(mods), "batched_us": t_b, "one_by_one_us": t_1,
            "batched_tflops": F / (t_b * 1e-6) / 1e12, "one_by_one_tflops": F / (t_1 * 1e-6) / 1e12,
            "device_status": D.dora_device_status()}


def run_e2e(args, D, dev, wl, W, A, B, m, base, lora, dy, n, y, d_base, d_lora, d_m, ws_n, ws_b, world):
    T, d_out, s = wl.tokens, wl.d_out, wl.s
    h = {k: v.cpu().pin_memory() for k, v in dict(W=W, A=A, B=B, m=m, base=base, lora=lora, dy=dy).items()}
    o = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in
         dict(n=n, y=y, d_base=d_base, d_lora=d_lora, d_m=d_m).items()}
    h2d = sum(v.numel() * v.element_size() for v in h.values())
    d2h = sum(v.numel() * v.element_size() for v in o.values())
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        rec = (lambda i: ev[i].record(stream)) if ev is not None else (lambda i: None)
        rec(0)
        W.copy_(h["W"], non_blocking=True)
        A.copy_(h["A"], non_blocking=True)
        B.copy_(h["B"], non_blocking=True)
        D.dora_factored_norm(W, A, B, s, n_out=n, workspace=ws_n)
        o["n"].copy_(n, non_blocking=True)
        rec(1)
        m.copy_(h["m"], non_blocking=True)
        base.copy_(h["base"], non_blocking=True)
        lora.copy_(h["lora"], non_blocking=True)
        D.dora_compose_fwd(base, lora, m, n, s, y=y)
        o["y"].copy_(y, non_blocking=True)
        rec(2)
        dy.copy_(h["dy"], non_blocking=True)
        D.dora_compose_bwd(dy, base, lora, m, n, s, d_base, d_lora, d_m, ws_b)
        o["d_base"].copy_(d_base, non_blocking=True)
        o["d_lora"].copy_(d_lora, non_blocking=True)
        o["d_m"].copy_(d_m, non_blocking=True)
        rec(3)

    for _ in range(max(1, min(args.warmup, 2))):
        step()
    torch.cuda.synchronize()
    k = max(1, min(args.steps, 5))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(k)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    for i in range(k):
        step(evs[i])
    torch.cuda.synchronize()
    t_norm, t_fwd, t_bwd = max_over_ranks([sum(e[0].elapsed_time(e[1]) for e in evs) / k * 1e-3,
                                           sum(e[1].elapsed_time(e[2]) for e in evs) / k * 1e-3,
                                           sum(e[2].elapsed_time(e[3]) for e in evs) / k * 1e-3], world, dev)
    return dict(t_norm=t_norm, t_fwd=t_fwd, t_bwd=t_bwd, h2d=h2d, d2h=d2h, steps=k)


# ------------------------------------------------------- oracle (CPU) arm
def oracle_threads():
    try:
        from threadpoolctl import threadpool_info

        return max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        return os.cpu_count() or 1


def time_oracle(wl, norm_rows, compose_tokens, seed=0):
    """Oracle norm on `norm_rows` rows and compose fwd/bwd on `compose_tokens`
    tokens of the workload; returns (norm TFLOP/s, fwd GB/s, bwd GB/s, sample)."""
    import numpy as np

    import oracle

    W, A, B, m = WL.make_weights(wl.with_(d_out=norm_rows))
    W64, A64, B64 = (t.double().numpy() for t in (W, A, B))
    t0 = time.perf_counter()
    n = oracle.row_norm(W64, A64, B64, wl.s)
    t_norm = time.perf_counter() - t0
    rng = np.random.default_rng(seed)
    T, d = compose_tokens, wl.d_out
    base = rng.standard_normal((T, d)).astype(np.float32).astype(np.float64)
    lora = rng.standard_normal((T, d)).astype(np.float32).astype(np.float64) * 0.02
    dy = rng.standard_normal((T, d)).astype(np.float32).astype(np.float64)
    mm = np.ones(d)
    nn = np.ones(d) * (1 + 1e-4)
    t0 = time.perf_counter()
    oracle.compose_forward(base, lora, mm, nn, wl.s)
    t_fwd = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.compose_backward(dy, base, lora, mm, nn, wl.s)
    t_bwd = time.perf_counter() - t0
    del n
    tf = norm_flops(norm_rows, wl.d_in, wl.r) / t_norm / 1e12
    return dict(
        norm_tflops=tf, fwd_gbs=fwd_bytes(T, d) / t_fwd / 1e9, bwd_gbs=bwd_bytes(T, d) / t_bwd / 1e9,
        t=t_norm + t_fwd + t_bwd,
        sample=f"norm on {norm_rows} of {wl.d_out} rows (full d_in, r); compose fwd/bwd on {T} of {wl.tokens} tokens",
    )


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    wl = workload_of(args)
    for _ in range(args.warmup):
        time_oracle(wl, *ORACLE_SAMPLE)
    res = []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        res.append(time_oracle(wl, *ORACLE_SAMPLE))
    wall = time.perf_counter() - t0
    v = statistics.median(r["norm_tflops"] for r in res)
    cores = oracle_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": wall / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "d_out": wl.d_out, "d_in": wl.d_in, "r": wl.r, "tokens": wl.tokens,
                   "s": wl.s, "sample": res[0]["sample"]},
        "compose": {"fwd_gbs": statistics.median(r["fwd_gbs"] for r in res),
                    "bwd_gbs": statistics.median(r["bwd_gbs"] for r in res)},
        "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": res[0]["sample"]},
        "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


def build_line(args, res, N, peaks, peak_src, traffic, cpu):
    """The JSON line of our arm from the max-over-ranks times in `res`; N ranks
    each ran one replica of the workload, so every rate is the whole job's."""
    wl = res["wl"]
    e = 2 if wl.dtype == "bf16" else 4
    F = norm_flops(wl.d_out, wl.d_in, wl.r)
    Bn = norm_bytes(wl.d_out, wl.d_in, wl.r, e)
    Bf = fwd_bytes(wl.tokens, wl.d_out, e)
    Bb = bwd_bytes(wl.tokens, wl.d_out, e)
    labels = traffic_labels(wl)

    def roof(kernel, t, work, bound):
        if bound == "tensor":
            ach = work / t / 1e12
            pk = peaks["bf16_tflops"]
            unit = "TFLOP/s"
        else:
            ach = work / t / 1e9
            pk = peaks["hbm_gbs"]
            unit = "GB/s"
        return {"kernel": kernel, "bound": bound, "achieved": ach, "peak": pk, "unit": unit, "frac": ach / pk,
                "traffic": traffic.get((kernel, labels[kernel])),
                "peak_source": f"{peak_src} (burst)" if bound == "tensor" else peak_src, "time_us": t * 1e6}

    # norm bound: slower of FLOPs at tensor peak and bytes at HBM bandwidth
    norm_bound = "tensor" if F / (peaks["bf16_tflops"] * 1e12) >= Bn / (peaks["hbm_gbs"] * 1e9) else "hbm"
    rl = [
        roof("norm", res["t_norm"], F if norm_bound == "tensor" else Bn, norm_bound),
        roof("compose_fwd", res["t_fwd"], Bf, "hbm"),
        roof("compose_bwd", res["t_bwd"], Bb, "hbm"),
    ]
    dominant = max(rl, key=lambda x: x["time_us"])
    e2e = res["e2e"]
    e2e_norm = F * N / (e2e["t_norm"]) / 1e12

    line = {
        "metric": METRIC,
        "value": F * N / res["t_norm"] / 1e12,
        "unit": "TFLOP/s",
        "n_gpus": N,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": res["t_total"] / args.steps * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": DTYPE_LABEL[wl.dtype],
        "data": "synthetic",
        "config": {"workload": wl.name, "d_out": wl.d_out, "d_in": wl.d_in, "r": wl.r, "tokens": wl.tokens,
                   "s": wl.s, "parallelism": f"replicas x{N}", "l2": l2_statement(wl, res["flushed"])},
        "value_basis": "norm FLOPs x ranks / max-over-ranks mean CUDA-event time of the norm launches in the timed steps",
        "compose": {
            "fwd": {"value": Bf * N / res["t_fwd"] / 1e9, "unit": "GB/s", "frac": rl[1]["frac"],
                    "time_us": res["t_fwd"] * 1e6},
            "bwd": {"value": Bb * N / res["t_bwd"] / 1e9, "unit": "GB/s", "frac": rl[2]["frac"],
                    "time_us": res["t_bwd"] * 1e6},
        },
        "norm": {"tflops": F / res["t_norm"] / 1e12, "frac": rl[0]["frac"], "bound": norm_bound,
                 "time_us": res["t_norm"] * 1e6, "flops": F, "bytes": Bn},
        "step_time_spread": res.get("spread"),
        "roofline": {k: dominant[k] for k in ("bound", "achieved", "peak", "unit", "frac", "traffic")}
                    | {"kernel": dominant["kernel"], "peak_source": dominant["peak_source"]},
        "rooflines": rl,
        "step_roofline_frac": (
            max(F / (peaks["bf16_tflops"] * 1e12), Bn / (peaks["hbm_gbs"] * 1e9))
            + Bf / (peaks["hbm_gbs"] * 1e9) + Bb / (peaks["hbm_gbs"] * 1e9)) / (res["t_total"] / args.steps),
        "e2e": {"value": e2e_norm, "unit": "TFLOP/s", "h2d_bytes_per_step": e2e["h2d"],
                "d2h_bytes_per_step": e2e["d2h"], "steps": e2e["steps"],
                "basis": "norm FLOPs / (H2D of W, A, B + norm + D2H of n), pinned host buffers",
                "compose_fwd_gbs": Bf * N / e2e["t_fwd"] / 1e9, "compose_bwd_gbs": Bb * N / e2e["t_bwd"] / 1e9},
        "cpu_baseline": cpu,
        "gpu_launches": res["launches"],
        "gpu_launches_basis": "dora_launch_count() after the timed steps minus before them (this rank)",
        "memset_nodes": 0,  # the compose backward's counters are tagged per call, nothing is cleared
        "clocks": res["clocks"],
        "device_status": res["status"],
    }
    if res.get("unflushed"):
        u = res["unflushed"]
        line["steps_without_clean"] = {
            "what": "the same steps back to back with no L2 clean between them (each step's norm also writes "
                    "back the previous compose backward's dirty lines)",
            "ms_per_step": u["t_total"] / args.steps * 1e3,
            "norm": {"time_us": u["t_norm"] * 1e6, "tflops": F / u["t_norm"] / 1e12,
                     "frac": F / u["t_norm"] / 1e12 / peaks["bf16_tflops"]},
            "compose_fwd": {"time_us": u["t_fwd"] * 1e6, "gbs": Bf / u["t_fwd"] / 1e9,
                            "frac": Bf / u["t_fwd"] / 1e9 / peaks["hbm_gbs"]},
            "compose_bwd": {"time_us": u["t_bwd"] * 1e6, "gbs": Bb / u["t_bwd"] / 1e9,
                            "frac": Bb / u["t_bwd"] / 1e9 / peaks["hbm_gbs"]},
        }
    if res.get("dense") is not None:
        line["dense_comparator"] = res["dense"]
    if res.get("batched") is not None:
        line["many_modules"] = res["batched"]
    if res.get("norm_bwd"):
        nb = dict(res["norm_bwd"])
        nb["frac"] = nb["factored_tflops"] / peaks["bf16_tflops"]
        nb["peak"] = peaks["bf16_tflops"]
        nb["bound"] = "tensor"
        line["norm_backward"] = nb
    if res.get("fused"):
        fl = dict(res["fused"])
        # ten calls back to back (~8 ms): between the burst and the sustained
        # (seconds-long, power-capped) measured GEMM figures; both are given
        fl["frac"] = fl["fused_tflops"] / peaks["bf16_tflops"]
        fl["peak"] = peaks["bf16_tflops"]
        fl["frac_of_sustained"] = fl["fused_tflops"] / peaks["bf16_tflops_sustained"]
        fl["peak_sustained"] = peaks["bf16_tflops_sustained"]
        fl["bound"] = "tensor"
        line["fused_linear"] = fl
    return line


# ------------------------------------------------------------------ sweep
SWEEP_FLUSH_BYTES = 256 << 20  # twice the 126 MB L2


class L2Flush:
    """Writes one buffer larger than L2, then reads another: the read evicts
    the written lines (their write-back happens here, untimed) and leaves L2
    holding clean lines of the second buffer, so the next call neither finds
    its inputs in L2 nor pays for someone else's dirty lines."""

    def __init__(self, dev):
        self.w = torch.empty(SWEEP_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        self.r = torch.zeros(SWEEP_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        self.acc = torch.empty((), dtype=torch.float32, device=dev)

    def __call__(self):
        self.w.fill_(1.0)
        torch.sum(self.r, dim=0, out=self.acc)


def time_alone(f, reps, flush, stream):
    """Median CUDA-event time (s) of f() over reps calls, each timed alone on
    ``stream`` after ``flush()``, which is not timed."""
    for _ in range(3):
        flush()
        f()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for e0, e1 in evs:
        flush()
        e0.record(stream)
        f()
        e1.record(stream)
    torch.cuda.synchronize()
    return statistics.median(e0.elapsed_time(e1) for e0, e1 in evs) * 1e-3


def run_sweep(args):
    """The rank/shape sweep workload on one GPU: the factored norm at
    d_out = d_in = 8192 for every rank of RANK_SWEEP, then the compose forward
    and backward at d_out = 8192 for every token count of TOKEN_SWEEP (m, n
    with m / n = 1 + N(0, 1e-4)).  Each point's time is the median of calls
    timed alone after an L2 flush (L2Flush); each point gives its throughput and its
    fraction of the roofline time (the slower of its algorithmic FLOPs at the
    measured bf16 peak and its algorithmic bytes at the measured copy
    bandwidth).  Prints one JSON line {"sweep": [...], ...}; it is not the
    benchmark line."""
    from factored_weight_norm_b200 import dora as D

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    reps = max(5, min(args.steps, 50))
    sampler = ClockSampler(0)
    sampler.start()
    pts = sweep_points(D, dev, reps, peaks)
    clocks = sampler.stop()
    status = D.dora_device_status()
    print(json.dumps({"sweep": pts, "reps_per_point": reps, "l2": "before every timed call 256 MB written, then another 256 MB read",
                      "peaks": {"bf16_tflops": peaks["bf16_tflops"], "hbm_gbs": peaks["hbm_gbs"],
                                "source": peak_src}, "clocks": clocks, "device_status": status}), flush=True)
    return 0 if status == D.DORA_OK else 1


def sweep_points(D, dev, reps, peaks):
    """Points of the rank/shape sweep (see run_sweep)."""
    stream = torch.cuda.current_stream(dev)
    flush = L2Flush(dev)
    pts = []
    for wl in WL.RANK_SWEEP:
        W, A, B, _ = WL.make_weights(wl, dev)
        n = torch.empty(wl.d_out, dtype=torch.float32, device=dev)
        ws = torch.empty(D.dora_factored_norm_workspace_size(wl.d_out, wl.d_in, wl.r), dtype=torch.uint8,
                         device=dev)
        t = time_alone(lambda: D.dora_factored_norm(W, A, B, wl.s, n_out=n, workspace=ws), reps, flush, stream)
        fl, by = norm_flops(wl.d_out, wl.d_in, wl.r), norm_bytes(wl.d_out, wl.d_in, wl.r)
        t_roof = max(fl / (peaks["bf16_tflops"] * 1e12), by / (peaks["hbm_gbs"] * 1e9))
        pts.append({"op": "factored_norm", "d_out": wl.d_out, "d_in": wl.d_in, "r": wl.r, "us": t * 1e6,
                    "tflops": fl / t * 1e-12, "gbs": by / t * 1e-9,
                    "bound": "tensor" if fl / (peaks["bf16_tflops"] * 1e12) >= by / (peaks["hbm_gbs"] * 1e9)
                    else "hbm", "roofline_frac": t_roof / t})
        del W, A, B, ws
    base_wl = WL.TOKEN_SWEEP[0]
    W, A, B, _ = WL.make_weights(base_wl, dev)
    m, n = WL.make_near_unity_mn(base_wl, W, dev)
    for wl in WL.TOKEN_SWEEP:
        _, base, lora = WL.make_activations(wl, W, A, B, dev)
        dy = WL.make_grad(wl, dev)
        y, d_base, d_lora = torch.empty_like(base), torch.empty_like(base), torch.empty_like(base)
        d_m = torch.empty(wl.d_out, dtype=torch.float32, device=dev)
        ws = torch.empty(D.dora_compose_bwd_workspace_size(wl.tokens, wl.d_out), dtype=torch.uint8, device=dev)
        t_f = time_alone(lambda: D.dora_compose_fwd(base, lora, m, n, wl.s, y=y), reps, flush, stream)
        t_b = time_alone(lambda: D.dora_compose_bwd(dy, base, lora, m, n, wl.s, d_base, d_lora, d_m, ws), reps,
                         flush, stream)
        for op, t, by in (("compose_fwd", t_f, fwd_bytes(wl.tokens, wl.d_out)),
                          ("compose_bwd", t_b, bwd_bytes(wl.tokens, wl.d_out))):
            pts.append({"op": op, "tokens": wl.tokens, "d_out": wl.d_out, "us": t * 1e6, "gbs": by / t * 1e-9,
                        "bound": "hbm", "roofline_frac": by / t * 1e-9 / peaks["hbm_gbs"]})
        del base, lora, dy, y, d_base, d_lora, ws
    return pts


# --------------------------------------------------- the other configs
def kernel_point(kernel, t, flops, nbytes, peaks, traffic, label):
    """One kernel's time against its roofline time: the slower of its FLOPs
    at the measured bf16 peak and its bytes at the measured copy bandwidth."""
    t_tensor = flops / (peaks["bf16_tflops"] * 1e12) if flops else 0.0
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    bound = "tensor" if t_tensor >= t_hbm else "hbm"
    pt = {"kernel": kernel, "time_us": t * 1e6, "bound": bound, "roofline_time_us": max(t_tensor, t_hbm) * 1e6,
          "frac": max(t_tensor, t_hbm) / t, "gbs": nbytes / t / 1e9,
          "traffic": traffic.get((kernel, label))}
    if flops:
        pt["tflops"] = flops / t / 1e12
    return pt


def config_line(D, dev, wl, what, peaks, traffic, reps, full_step=False):
    """Norm, compose forward and compose backward of workload `wl`, each timed
    alone after an L2 flush (median of `reps` calls); with `full_step`, also
    the three back to back, as one training step of the adapter path."""
    stream = torch.cuda.current_stream(dev)
    flush = L2Flush(dev)
    e = 2 if wl.dtype == "bf16" else 4
    W, A, B, _ = WL.make_weights(wl, dev)
    m, n_ref = WL.make_near_unity_mn(wl, W, dev)
    _, base, lora = WL.make_activations(wl, W, A, B, dev)
    dy = WL.make_grad(wl, dev)
    n = torch.empty(wl.d_out, dtype=torch.float32, device=dev)
    y, d_base, d_lora = torch.empty_like(base), torch.empty_like(base), torch.empty_like(base)
    d_m = torch.empty(wl.d_out, dtype=torch.float32, device=dev)
    ws_n = torch.empty(D.dora_factored_norm_workspace_size(wl.d_out, wl.d_in, wl.r, WL.torch_dtype(wl)),
                       dtype=torch.uint8, device=dev)
    ws_b = torch.empty(D.dora_compose_bwd_workspace_size(wl.tokens, wl.d_out), dtype=torch.uint8, device=dev)
    norm = lambda: D.dora_factored_norm(W, A, B, wl.s, n_out=n, workspace=ws_n)  # noqa: E731
    fwd = lambda: D.dora_compose_fwd(base, lora, m, n_ref, wl.s, y=y)  # noqa: E731
    bwd = lambda: D.dora_compose_bwd(dy, base, lora, m, n_ref, wl.s, d_base, d_lora, d_m, ws_b)  # noqa: E731
    launches0 = D.dora_launch_count()
    t_n = time_alone(norm, reps, flush, stream)
    t_f = time_alone(fwd, reps, flush, stream)
    t_b = time_alone(bwd, reps, flush, stream)
    labels = traffic_labels(wl)
    line = {
        "config_line": what, "workload": wl.name, "dtype": DTYPE_LABEL[wl.dtype],
        "config": {"d_out": wl.d_out, "d_in": wl.d_in, "r": wl.r, "tokens": wl.tokens, "s": wl.s},
        "l2": "every call timed alone after 256 MB written, then another 256 MB read (untimed)",
        "reps_per_kernel": reps,
        "kernels": [
            kernel_point("norm", t_n, norm_flops(wl.d_out, wl.d_in, wl.r), norm_bytes(wl.d_out, wl.d_in, wl.r, e),
                         peaks, traffic, labels["norm"]),
            kernel_point("compose_fwd", t_f, 0, fwd_bytes(wl.tokens, wl.d_out, e), peaks, traffic, labels["compose_fwd"]),
            kernel_point("compose_bwd", t_b, 0, bwd_bytes(wl.tokens, wl.d_out, e), peaks, traffic, labels["compose_bwd"]),
        ],
    }
    if full_step:
        def step():
            norm()
            fwd()
            bwd()
        t_s = time_alone(step, reps, flush, stream)
        roof = sum(k["roofline_time_us"] for k in line["kernels"])
        line["full_step"] = {"time_us": t_s * 1e6, "roofline_time_us": roof, "frac": roof / (t_s * 1e6),
                             "what": "norm -> compose fwd -> compose bwd back to back after one flush"}
    line["gpu_launches"] = D.dora_launch_count() - launches0
    line["device_status"] = D.dora_device_status()
    return line


def oracle_single_thread_line(wl):
    """The oracle on the whole tiny workload with its BLAS limited to one
    thread: norm, compose forward, compose backward (median of 20 runs)."""
    import numpy as np

    import oracle

    try:
        from threadpoolctl import threadpool_limits
    except Exception:  # pragma: no cover - threadpoolctl is in the image
        threadpool_limits = None
    W, A, B, m = WL.make_weights(wl)
    W64, A64, B64 = (t.double().numpy() for t in (W, A, B))
    rng = np.random.default_rng(0)
    base = rng.standard_normal((wl.tokens, wl.d_out))
    lora = rng.standard_normal((wl.tokens, wl.d_out)) * 0.02
    dy = rng.standard_normal((wl.tokens, wl.d_out))
    mm = m.double().numpy()

    def timed(f):
        ts = []
        for _ in range(20):
            t0 = time.perf_counter()
            f()
            ts.append(time.perf_counter() - t0)
        return statistics.median(ts)

    def run():
        n = oracle.row_norm(W64, A64, B64, wl.s)
        return (timed(lambda: oracle.row_norm(W64, A64, B64, wl.s)),
                timed(lambda: oracle.compose_forward(base, lora, mm, n, wl.s)),
                timed(lambda: oracle.compose_backward(dy, base, lora, mm, n, wl.s)))

    if threadpool_limits is not None:
        with threadpool_limits(limits=1):
            t_n, t_f, t_b = run()
    else:
        t_n, t_f, t_b = run()
    return {"config_line": "config-1 oracle, one thread", "workload": wl.name, "kind": "oracle", "cores": 1,
            "config": {"d_out": wl.d_out, "d_in": wl.d_in, "r": wl.r, "tokens": wl.tokens, "s": wl.s},
            "norm_us": t_n * 1e6, "compose_fwd_us": t_f * 1e6, "compose_bwd_us": t_b * 1e6,
            "norm_tflops": norm_flops(wl.d_out, wl.d_in, wl.r) / t_n / 1e12,
            "sample": "the whole workload, median of 20 runs each"}


def run_config_lines(args, peaks):
    """The other configs on this GPU, one JSON line each, after the headline line."""
    from factored_weight_norm_b200 import dora as D

    dev = torch.device("cuda", 0)
    traffic = load_traffic()
    reps = max(5, min(args.steps, 20))
    lines = [
        config_line(D, dev, WL.TINY_F32, "config-1 tiny fp32", peaks, traffic, reps),
        config_line(D, dev, WL.SINGLE_4096, "config-2 bf16 single module", peaks, traffic, reps),
        config_line(D, dev, WL.MLP_UP_32B, "config-4 bf16 MLP up-projection, training step", peaks, traffic, reps,
                    full_step=True),
    ]
    sampler = ClockSampler(0)
    sampler.start()
    pts = sweep_points(D, dev, reps, peaks)
    lines.append({"config_line": "config-5 rank/token sweep", "sweep": pts, "reps_per_point": reps,
                  "l2": "every call timed alone after 256 MB written, then another 256 MB read (untimed)",
                  "clocks": sampler.stop(), "device_status": D.dora_device_status()})
    if not args.no_cpu_baseline:
        lines.append(oracle_single_thread_line(WL.TINY_F32))
    return lines


# ------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WL.HEADLINE.name, choices=sorted(WL.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the timed CPU oracle sample")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override the workload's token count (compose and fused-linear activations)")
    ap.add_argument("--no-context", action="store_true",
                    help="skip the context measurements after the timed step (dense comparator, many modules, "
                         "fused linear, attached-norm backward), e.g. for a profiler's launch list")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the lines of the other configs (tiny fp32, 4096 single module, MLP up-projection "
                         "step, rank/token sweep, single-thread oracle) after the headline line")
    ap.add_argument("--sweep", action="store_true",
                    help="run the rank/shape sweep (norm over ranks, compose over token counts) on one GPU "
                         "and print its points instead of the benchmark line")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.sweep:
        if world > 1:
            raise SystemExit("--sweep measures one GPU; run it without torchrun")
        return run_sweep(args)

    if world > 1:
        import datetime

        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    res = run_ours(args, rank, world, local_rank)
    wl = res["wl"]
    N = world
    peaks, peak_src = load_peaks()
    traffic = load_traffic()
    cpu = None
    if rank == 0 and N == 1 and not args.no_cpu_baseline:
        obs = []
        while len(obs) < ORACLE_MAX_REPS and sum(o["t"] for o in obs) < ORACLE_MIN_SECONDS:
            obs.append(time_oracle(wl, *ORACLE_SAMPLE, seed=len(obs)))
        cpu = {"value": statistics.median(o["norm_tflops"] for o in obs), "unit": "TFLOP/s",
               "cores": oracle_threads(), "kind": "oracle",
               "sample": f"{obs[0]['sample']}; median of {len(obs)} repetitions",
               "cpu_seconds": sum(o["t"] for o in obs),
               "compose_fwd_gbs": statistics.median(o["fwd_gbs"] for o in obs),
               "compose_bwd_gbs": statistics.median(o["bwd_gbs"] for o in obs)}

    if rank == 0:
        print(json.dumps(build_line(args, res, N, peaks, peak_src, traffic, cpu)), flush=True)
    if rank == 0 and N == 1 and not args.no_configs and wl.name == WL.HEADLINE.name and args.tokens is None:
        for line in run_config_lines(args, peaks):
            print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
