"""Benchmark: MoE-layer tokens/s and packed-weight HBM GB/s against the roofline.

Default workload (--workload 5): dynamic repaging at full size, the largest
single-GPU configuration -- 256 experts, hidden 7168, SwiGLU ffn 2048, 22.5 GB
of fp16 masters ~N(0, 0.02), top-8 routing. Quantize at 8 bits average, then 10
phases, each a run of decode steps (one forward pass of a 128-token batch:
route, page-table gather + unpack/dequant fused into the gate/up and down
contractions, SwiGLU, top-k combine) followed by a budget change (average bits
7, 6, 5, 4, 3, 3.75, 4.5, 5.25, 6, 6) whose repage re-quantizes only the
experts whose width changed. Exactly K decode steps are timed, spread over the
phases; value = decode tokens/s; the quantize and repage rates are reported
beside it against the HBM roofline.

--workload 2 / 3: one decode layer (Mixtral-shaped 8 x 4096 x 14336 with 16
tokens top-2; fine-grained 128 x 2048 x 768 with 64 tokens top-8); a step is
one forward pass over a fresh batch with the pages resident.

--workload 4 times the fine-grained prefill layer (128 experts, hidden 2048,
ffn 768, 8192 tokens top-8, 3.5 bits average), which runs on the tensor-core
path; its roofline is the gate/up kernel's bf16 FLOP rate.

--width B / --experts E / --tokens T / --topk k time one layer of the
workload's shape instead (with --workload 5: one decode layer, not the
schedule): every expert at B bits rather than the allocator's widths, and/or
another expert count, batch or top-k -- the decode rate by width, or a case
small enough for a multi-pass profiler capture. The line names the layer.
--path decode|prefill forces one contraction path on a one-layer run.

The value comes from a timed region without per-kernel events; the kernel
durations behind the roofline come from a second pass over the same batches
with CUDA events around each kernel on the context stream.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 5]
    python bench.py --impl reference ...   # the float64 CPU oracle arm

With N > 1 (torchrun), every rank runs an independent replica of the layer on
its own GPU (the path needs no collective); value = tokens of all ranks / the
slowest rank's device time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "MoE-layer tokens/s & packed-weight HBM GB/s vs roofline (mixed 3/4/8-bit)"
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: 2000 decode, 400 prefill)")
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["mpe", "reference"], default="mpe")
    ap.add_argument("--workload", type=int, default=5, choices=[1, 2, 3, 4, 5])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--variant", choices=["packed", "prefix"], default="packed",
                    help="prefix: the layered prefix-compatible store on a decode workload")
    ap.add_argument("--width", type=int, choices=[3, 4, 8], default=None,
                    help="every expert at this width instead of the allocator's widths: one "
                         "layer of the workload's shape (with --workload 5, one decode layer "
                         "instead of the repaging schedule)")
    ap.add_argument("--experts", type=int, default=None,
                    help="one layer with this many experts (a smaller case of the same shape)")
    ap.add_argument("--tokens", type=int, default=None, help="one layer, tokens per step")
    ap.add_argument("--topk", type=int, default=None, help="one layer, experts per token")
    ap.add_argument("--path", choices=["auto", "decode", "prefill"], default="auto",
                    help="contraction path of a one-layer run (auto: the library's rule)")
    args = ap.parse_args()
    layer_flags = (args.width, args.experts, args.tokens, args.topk)
    if args.variant == "prefix" and any(v is not None for v in layer_flags):
        ap.error("--width/--experts/--tokens/--topk time the packed format's layer")
    if args.path != "auto" and (args.variant == "prefix" or (
            args.workload == 5 and all(v is None for v in layer_flags))):
        ap.error("--path applies to one layer (not the schedule or the prefix variant)")
    E = args.experts
    if (E is not None and E < 1) or (args.tokens is not None and args.tokens < 1) or \
            (args.topk is not None and not 1 <= args.topk <= 32):
        ap.error("need --experts >= 1, --tokens >= 1 and --topk in 1..32")
    if args.steps is None:
        args.steps = {4: 400, 5: 200}.get(args.workload, 2000)
    # at least 3 untimed warm-up steps whatever is asked (the JSON line
    # reports the number run)
    args.warmup = max(3, args.warmup)
    return args


# ---------------------------------------------------------------------------
# distributed plumbing (replicas: barriers and a max over ranks only)
# ---------------------------------------------------------------------------
class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        self.device = "cuda"

    def init(self, backend: str):
        if self.world > 1:
            import datetime

            import torch.distributed as dist
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
            self.pg = dist
            self.device = "cpu" if backend == "gloo" else "cuda"

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, v: float) -> float:
        if not self.pg:
            return v
        import torch
        t = torch.tensor([v], dtype=torch.float64, device=self.device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines: list[str] = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict | None:
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# shared helpers
# ---------------------------------------------------------------------------
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0


def measured_peaks() -> tuple[dict, str]:
    """HBM GB/s and dense bf16 TFLOP/s (burst, sustained) measured on this machine."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return ({"hbm_gbs": float(pk["hbm_gbs"]), "bf16_tflops": float(pk["bf16_tflops"]),
                 "bf16_tflops_sustained": float(pk["bf16_tflops_sustained"])}, "measured")
    except (OSError, KeyError, ValueError):
        return ({"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                 "bf16_tflops_sustained": FALLBACK_BF16_TFLOPS_SUSTAINED}, "fallback")


# the source files each profiled kernel is built from: its device code and the
# types and constants it uses (context.h, the host-side context, is not one)
KERNEL_SOURCES = {
    "k_decode_gateup": ["decode.cu", "common.cuh", "internal.h"],
    "k_prefill_gateup": ["prefill.cu", "common.cuh", "internal.h"],
}


E2E_API = ("mpe_moe_ffn_host_async + mpe_host_wait: pinned host x, ids, w in and out back "
           "every step, step i's result waited for after step i+1 is queued (two host buffer "
           "sets), the last one waited for inside the timed region")


def e2e_pipeline(ctx, hb, n: int) -> None:
    """n host-buffer steps through the library's asynchronous entry point:
    step i is queued, then step i-1's result is waited for (its output is in
    host memory when the wait returns); the buffer sets hb are used in turn,
    so a set is reused only after its previous step was waited for."""
    prev = None
    for i in range(n):
        xh, ih, wh, oh = hb[i % len(hb)]
        t = ctx.moe_ffn_host_async(xh, ih, wh, oh)
        if prev is not None:
            ctx.wait_host(prev)
        prev = t
    ctx.wait_host(prev)


def kernel_source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "mixed_precision_expert_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic_ratio(kernel: str, workload: str) -> float | None:
    """DRAM bytes over algorithmic bytes per launch from a committed ncu
    summary (profiles/traffic.json), if it was taken on the kernel's current
    sources: for a workload too large to capture whole, the capture runs a
    smaller case of the same kernel and the ratio scales it."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    ent = rec.get(f"{kernel}:{workload}")
    if not ent or ent.get("source_hash") != kernel_source_hash(kernel) or \
            "traffic_over_algorithmic" not in ent:
        return None
    return float(ent["traffic_over_algorithmic"])


def recorded_traffic(kernel: str, workload: str) -> float | None:
    """DRAM bytes per launch from a committed ncu summary (profiles/traffic.json),
    if it was taken on the kernel's current sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    ent = rec.get(f"{kernel}:{workload}")
    if not ent or ent.get("source_hash") != kernel_source_hash(kernel):
        return None
    return float(ent["dram_bytes_per_launch"])


PREFILL_MIN_AVG = 32  # the library's automatic path rule: tensor cores when T*k >= 32 E


def bench_workload(workload: int, experts=None, tokens=None, topk=None, width=None):
    """The workload the flags name: one of the five, or one layer of its shape
    with another expert count, batch or top-k, or with every expert at one
    width (named after the workload it comes from, its sizes and the width)."""
    import synth
    wl = synth.WORKLOADS[workload]
    ch = {n: v for n, v in (("E", experts), ("T", tokens), ("k", topk)) if v is not None}
    if not ch and width is None:
        return wl
    E, T, k = ch.get("E", wl.E), ch.get("T", wl.T), ch.get("k", wl.k)
    if k > E:
        raise ValueError(f"top-{k} routing over {E} experts")
    name = f"{wl.name.split('-')[0]}-layer-e{E}-h{wl.H}-f{wl.F}-t{T}-top{k}"
    if width is not None:
        name += f"-w{width}"
    return synth.scaled(wl, name=name, **ch)


def args_workload(args):
    return bench_workload(args.workload, args.experts, args.tokens, args.topk, args.width)


def is_schedule(wl) -> bool:
    """The repaging schedule itself (not one layer of its shape)."""
    return wl.cfg == 5 and wl.name.startswith("repage-e")


def bench_config(wl, width=None, path_flag: str = "auto") -> dict:
    """The workload as both arms print it: static, so the two lines carry the
    same dict (measured values go in keys of their own)."""
    path = "tensor-core" if wl.T * wl.k >= PREFILL_MIN_AVG * wl.E else "streaming"
    if path_flag != "auto":
        path = {"decode": "streaming", "prefill": "tensor-core"}[path_flag]
    cfg = {"workload": wl.name, "E": wl.E, "H": wl.H, "F": wl.F, "tokens_per_step": wl.T,
           "top_k": wl.k, "avg_bits_budget": None if width else wl.avg_bits,
           "page_bytes": 65536, "parallelism": "replicas", "path": path}
    if width:
        cfg["width"] = width
    if "-layer-" in wl.name:
        pages_mb = wl.sum_W * (width or wl.avg_bits) / 8 / 1e6
        cfg["l2"] = (f"no flush: the layer's packed pages total {pages_mb:.0f} MB (a step "
                     f"reads those of its active experts; L2 holds 126 MB)")
    elif is_schedule(wl):
        cfg["schedule"] = ("quantize at 8 bits average, then 10 phases: decode steps of 128 "
                           "tokens, then a budget change (repage) to 7, 6, 5, 4, 3, 3.75, 4.5, "
                           "5.25, 6, 6 bits average")
        cfg["l2"] = ("no flush: each decode step reads the active experts' pages (4-11 GB) "
                     "and each repage the changed experts' masters, far above the 126 MB L2")
    elif wl.cfg == 1:
        cfg["l2"] = "no flush: a correctness-size layer (1.8 MB of pages) that fits in L2"
    elif wl.cfg == 4:
        cfg["l2"] = ("no flush: each step reads the packed pages of every expert (264 MB) and "
                     "the routed tokens (256 MB), above the 126 MB L2")
    else:
        cfg["l2"] = "no flush: the active experts' packed pages read per step exceed the 126 MB L2"
    return cfg


def bits_hist(bits) -> dict:
    return {str(b): int((np.asarray(bits) == b).sum()) for b in (3, 4, 8)}


def cores_used() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def oracle_widths(wl, width=None) -> np.ndarray:
    """The oracle's widths for the workload: its allocator's, or one width for all."""
    import synth
    from oracle import allocate as oa
    if width:
        return np.full(wl.E, width, dtype=np.uint8)
    return oa.allocate_bits(synth.importance(wl), [wl.W_e] * wl.E, wl.budget_bits)


class OracleSample:
    """Bounded sample of the oracle's forward work: one token through one expert,
    in slices of rows of F (SwiGLU separates over F, so the slices of all F rows
    sum to the expert's output). Input generation and the oracle's quantization
    of the expert (the resident pages) happen once, untimed; each slice
    dequantizes its rows and runs the float64 SwiGLU."""

    def __init__(self, wl, e: int = 0, token: int = 0, width=None):
        import synth
        from oracle import quantize as oq
        self.wl = wl
        bits = oracle_widths(wl, width)
        master = synth.expert_weights(wl, e).numpy()
        self.m, self.s, k = oq.quantize_expert(master, int(bits[e]))
        H, F = wl.H, wl.F
        self.k1 = k[:F * H].reshape(F, H)
        self.k3 = k[F * H:2 * F * H].reshape(F, H)
        self.k2 = k[2 * F * H:].reshape(H, F)
        self.x = synth.activations(wl, T=token + 1)[token:token + 1].double().numpy()

    def run(self, n_slices: int, slice_rows: int):
        """(seconds, tokens of layer work done)."""
        from oracle import ffn as of
        from oracle import quantize as oq
        F = self.wl.F
        t0 = time.perf_counter()
        y = np.zeros((1, self.wl.H))
        for i in range(n_slices):
            f0 = (i * slice_rows) % F
            sl = slice(f0, f0 + slice_rows)
            y += of.expert_ffn(self.x, oq.dequantize(self.k1[sl], self.s),
                               oq.dequantize(self.k3[sl], self.s),
                               oq.dequantize(self.k2[:, sl], self.s))
        return time.perf_counter() - t0, n_slices * slice_rows / F / self.wl.k


def oracle_quantize_rate(wl, n_weights: int = 1 << 21, width=None) -> dict:
    """The oracle's quantizer on a bounded sample (the first n_weights fp16
    weights of expert 0 at its width): absmax, scale, codes, offset codes.
    Rate in the quantize pass's bytes: 4 per weight (two reads of the master)
    + b / 8 written."""
    import synth
    from oracle import quantize as oq
    b = int(oracle_widths(wl, width)[0])
    n = min(n_weights, wl.W_e)
    master = synth.expert_weights(wl, 0, count=n).numpy()
    t0 = time.perf_counter()
    m, s, k = oq.quantize_expert(master, b)
    oq.offset_codes(k, b)
    dt = time.perf_counter() - t0
    nbytes = 4 * n + b * n // 8
    return {"GB/s": nbytes / dt / 1e9, "sample": f"{n} weights of expert 0 at {b} bits"}


# ---------------------------------------------------------------------------
# reference arm: the float64 oracle on the host cores
# ---------------------------------------------------------------------------
def run_reference(args, dist: Dist):
    import synth
    if dist.rank != 0:
        return
    wl = args_workload(args)
    slice_rows = 128
    sample = OracleSample(wl, width=args.width)
    # warm-up and timed steps: each step = one 128-row F-slice of one token-slot
    sample.run(max(1, args.warmup), slice_rows)
    dt, frac = sample.run(args.steps, slice_rows)
    value = frac / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(wl, args.width, args.path),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores_used(),
                         "kind": "oracle",
                         "sample": f"each step: one {slice_rows}-row slice of ffn for one token "
                                   f"through one expert (dequantize + SwiGLU, float64); "
                                   f"{args.steps} steps = {frac:.4f} tokens of layer work",
                         "quantize": oracle_quantize_rate(wl, width=args.width)},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# the library arm
# ---------------------------------------------------------------------------
def run_mpe(args, dist: Dist):
    import torch

    from mixed_precision_expert_b200.build import build
    if dist.rank == 0:
        build()
    dist.barrier()
    import mixed_precision_expert_b200 as mpe
    import synth

    dev = dist.local_rank
    torch.cuda.set_device(dev)
    wl = args_workload(args)
    E, H, F, T, k = wl.E, wl.H, wl.F, wl.T, wl.k

    # resident state: fp16 masters -> bit allocation -> quantized pages
    masters = []
    for e in range(E):
        t = torch.empty(wl.W_e, dtype=torch.float16, device="cuda")
        synth.fill_expert_weights(wl, e, t)
        masters.append(t)
    if args.width:
        bits = np.full(E, args.width, dtype=np.uint8)
    else:
        bits = mpe.allocate_bits(synth.importance(wl), [wl.W_e] * E, wl.budget_bits)
    ctx = mpe.Context(E, H, F, path={"auto": mpe.PATH_AUTO, "decode": mpe.PATH_DECODE,
                                     "prefill": mpe.PATH_PREFILL}[args.path])
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    q_ms = []
    for _ in range(3):
        torch.cuda.synchronize()
        ev0.record()
        ctx.quantize_experts(masters, bits)
        ev1.record()
        torch.cuda.synchronize()
        q_ms.append(ev0.elapsed_time(ev1))
    q_bytes = 4 * wl.sum_W + sum(int(b) * wl.W_e // 8 for b in bits)  # absmax + encode passes
    if ctx.status() != 0:
        raise RuntimeError(f"device status {ctx.status():#x} after quantize")
    # measured per-expert loss (exact MSE at 3/4/8 bits; one read of the masters);
    # a quantize call invalidates the context's cached values, so each rep re-quantizes
    ml_ms = []
    for _ in range(3):
        ctx.quantize_experts(masters, bits)
        torch.cuda.synchronize()
        ev0.record()
        ctx.measure_loss()
        ev1.record()
        torch.cuda.synchronize()
        ml_ms.append(ev0.elapsed_time(ev1))
    ml_bytes = 2 * wl.sum_W

    # per-step batches, resident in HBM (distinct seeds, cycled)
    nb = min(64, args.steps + args.warmup)
    batches = []
    for i in range(nb):
        seed = 7_000_000 + 1000 * dist.rank + i
        ids, w = synth.routing(wl, seed=seed)
        x = synth.activations(wl, seed=seed, device="cuda")
        batches.append((x, torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda(), ids))
    out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")

    def valid_assignments(ids_np):
        return int(((ids_np >= 0) & (ids_np < E)).sum())

    def gateup_bytes(ids_np):
        act = np.unique(ids_np)
        wbytes = sum(int(bits[e]) * 2 * F * H // 8 for e in act)
        return wbytes + T * H * 2 + T * k * F * 2

    def layer_bytes(ids_np):
        act = np.unique(ids_np)
        return sum(int(bits[e]) * wl.W_e // 8 for e in act) + 2 * T * H * 2

    def run_steps(n):
        for i in range(n):
            x, idt, wt, _ = batches[i % nb]
            ctx.moe_ffn(x, idt, wt, out)

    run_steps(args.warmup)
    torch.cuda.synchronize()

    # timed region: the whole forward path, no per-kernel events
    clocks = ClockSampler(dev)
    clocks.start()
    time.sleep(0.3)  # let the sampler attach before the timed region
    launches0 = ctx.kernel_launches()
    dist.barrier()
    torch.cuda.synchronize()
    ev0.record()
    run_steps(args.steps)
    ev1.record()
    torch.cuda.synchronize()
    dist.barrier()
    ms_local = ev0.elapsed_time(ev1)
    launches = ctx.kernel_launches() - launches0
    clk = clocks.stop()
    ms = dist.max(ms_local)
    if ctx.status() != 0:
        raise RuntimeError(f"device status {ctx.status():#x} after the timed region")

    # kernel durations: the same steps again with events around each kernel
    ctx.profile(True)
    run_steps(args.steps)
    prof = ctx.profile_read(reset=True)
    ctx.profile(False)

    tokens = T * args.steps * dist.world
    value = tokens / (ms / 1e3)
    alg_layer = np.mean([layer_bytes(batches[i % nb][3]) for i in range(args.steps)])
    peaks, peak_kind = measured_peaks()
    if prof["tc_gate_up"][1]:
        # tensor-core path: bf16 FLOPs of the gate/up contraction (2 matrices, 2 FLOP/MAC)
        gu_ms, gu_n = prof["tc_gate_up"]
        flops = np.mean([4.0 * valid_assignments(batches[i % nb][3]) * H * F
                         for i in range(args.steps)])
        achieved = flops / (gu_ms / gu_n / 1e3) / 1e12
        # burst peak: the clocks stay at their maximum through these runs (see
        # "clocks"); the power-capped sustained figure is given for context
        peak = peaks["bf16_tflops"]
        roofline = {"bound": "tensor", "kernel": "tensor-core gate/up (k_prefill<1>)",
                    "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak,
                    "peak_source": f"{peak_kind} bf16 dense, burst; frac of the sustained "
                                   f"{peaks['bf16_tflops_sustained']:.0f} TFLOP/s: "
                                   f"{achieved / peaks['bf16_tflops_sustained']:.3f}",
                    "traffic": recorded_traffic("k_prefill_gateup", wl.name),
                    "algorithmic_flops_per_launch": flops,
                    "avg_launch_us": gu_ms / gu_n * 1e3}
    else:
        gu_ms, gu_n = prof["gate_up"]
        alg_gu = np.mean([gateup_bytes(batches[i % nb][3]) for i in range(args.steps)])
        achieved = alg_gu / (gu_ms / gu_n / 1e3) / 1e9
        peak = peaks["hbm_gbs"]
        roofline = {"bound": "hbm", "kernel": "decode gate/up (k_decode<1, 0>)",
                    "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                    "peak_source": peak_kind,
                    "traffic": recorded_traffic("k_decode_gateup", wl.name),
                    "algorithmic_bytes_per_launch": alg_gu,
                    "avg_launch_us": gu_ms / gu_n * 1e3}
    layer_gbs = alg_layer / (ms_local / args.steps / 1e3) / 1e9
    total_prof = max(sum(v[0] for v in prof.values()), 1e-9)
    kernel_us = {kname: round(v[0] / v[1] * 1e3, 2) for kname, v in prof.items() if v[1]}
    kernel_share = {kname: round(v[0] / total_prof, 4) for kname, v in prof.items() if v[1]}
    layer_tflops = 6.0 * np.mean([valid_assignments(batches[i % nb][3])
                                  for i in range(args.steps)]) * H * F / (ms_local / args.steps / 1e3) / 1e12

    # end to end through the C ABI with host buffers (pinned), copies in the timed region
    e2e = None
    hb = []
    for i in range(min(nb, 16)):
        x, idt, wt, ids_np = batches[i]
        hb.append((x.cpu().pin_memory(), torch.from_numpy(ids_np).pin_memory(),
                   wt.cpu().pin_memory(), torch.empty(T, H, dtype=torch.bfloat16).pin_memory()))
    n_e2e = max(10, min(args.steps, 500))
    for i in range(5):
        xh, ih, wh, oh = hb[i % len(hb)]
        ctx.moe_ffn_host(xh, ih, wh, oh)
    dist.barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    e2e_pipeline(ctx, hb, n_e2e)
    e2e_s = dist.max(time.perf_counter() - t0)
    h2d = T * H * 2 + T * k * 4 + T * k * 4
    d2h = T * H * 2
    e2e = {"value": T * n_e2e * dist.world / e2e_s, "unit": "tokens/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n_e2e,
           "api": E2E_API}

    # salient-channel compensation on the streaming path (timed apart from the
    # headline value): step time with n channels kept per row, store in device
    # or mapped host memory
    comp = None
    # one GPU only: a rank whose store allocation failed would otherwise skip
    # the max over ranks the others wait in
    if not prof["tc_gate_up"][1] and dist.world == 1:
        comp = {"n_channels": [], "store": [], "step_us": []}
        ev_a, ev_b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_comp = max(20, min(args.steps, 200))
        try:
            for n_ch, store in ((16, mpe.STORE_DEVICE), (64, mpe.STORE_DEVICE),
                                (16, mpe.STORE_HOST)):
                ctx.set_compensation(n_ch, store)
                for i in range(3):
                    x, idt, wt, _ = batches[i % nb]
                    ctx.moe_ffn(x, idt, wt, out)
                torch.cuda.synchronize()
                ev_a.record()
                for i in range(n_comp):
                    x, idt, wt, _ = batches[i % nb]
                    ctx.moe_ffn(x, idt, wt, out)
                ev_b.record()
                torch.cuda.synchronize()
                comp["n_channels"].append(n_ch)
                comp["store"].append("host" if store == mpe.STORE_HOST else "device")
                comp["step_us"].append(ev_a.elapsed_time(ev_b) / n_comp * 1e3)
            ctx.set_compensation(0)
            comp["plain_step_us"] = ms / args.steps * 1e3
        except mpe.MpeError as err:
            comp = {"unavailable": str(err)}
            ctx.set_compensation(0)

    cpu = None
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        slice_rows = 128
        n_slices = max(1, F // slice_rows)
        dt, frac = OracleSample(wl, width=args.width).run(n_slices, slice_rows)
        cpu = {"value": frac / dt, "unit": "tokens/s", "cores": cores_used(), "kind": "oracle",
               "sample": f"one token through one expert (all {F} ffn rows in {n_slices} slices; "
                         f"dequantize + SwiGLU in float64) = {frac:.3f} tokens of layer work",
               "quantize": oracle_quantize_rate(wl, width=args.width)}

    qms = float(np.median(q_ms))
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": bench_config(wl, args.width, args.path),
        "bits_hist": bits_hist(bits),
        "path_taken": "tensor-core" if prof["tc_gate_up"][1] else "streaming",
        "packed_bytes_per_step": alg_layer,
        "packed_weight_gbs": layer_gbs,
        "packed_weight_frac_of_peak": layer_gbs / peaks["hbm_gbs"],
        "layer_tflops": layer_tflops,
        "roofline": roofline,
        "kernel_us": kernel_us,
        "kernel_time_share": kernel_share,
        "quantize": {"ms": qms, "GB/s": q_bytes / (qms / 1e3) / 1e9,
                     "frac": q_bytes / (qms / 1e3) / 1e9 / peaks["hbm_gbs"],
                     "bytes": q_bytes, "passes": "absmax read + encode read/write"},
        "measure_loss": {"ms": min(ml_ms), "GB/s": ml_bytes / (min(ml_ms) / 1e3) / 1e9,
                         "frac_hbm": ml_bytes / (min(ml_ms) / 1e3) / 1e9 / peaks["hbm_gbs"],
                         "bytes": ml_bytes,
                         "note": "exact MSE of every expert at 3, 4 and 8 bits; one read "
                                 "of the fp16 masters; integer-ALU bound"},
        "compensation": comp,
        "gpu_launches": launches,
        "clocks": clk,
        "e2e": e2e,
        "cpu_baseline": cpu,
    }
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    ctx.close()


# ---------------------------------------------------------------------------
# the dynamic-repaging schedule (workload 5)
# ---------------------------------------------------------------------------
def phase_steps(K: int, phases: int) -> list[int]:
    """K timed decode steps spread over the schedule's phases (earlier phases
    take the remainder)."""
    return [K // phases + (1 if i < K % phases else 0) for i in range(phases)]


def run_repage_schedule(args, dist: Dist):
    """The dynamic-repaging workload (the largest single-GPU configuration):
    256 experts, hidden 7168, ffn 2048, 22.5 GB of fp16 masters. After the
    initial quantize at 8 bits average, 10 phases: decode steps (one forward
    pass of 128 tokens, top-8, each), then a budget change whose repage
    re-quantizes only the experts whose width changed. Exactly K decode steps
    are timed, spread over the phases, inside one region that also holds the
    repages (each timed on its own); value = decode tokens / decode device
    time. The roofline is the decode gate/up kernel's, over every launch of
    the schedule (a second pass with per-kernel events)."""
    import torch

    from mixed_precision_expert_b200.build import build
    if dist.rank == 0:
        build()
    dist.barrier()
    import mixed_precision_expert_b200 as mpe
    import synth

    dev = dist.local_rank
    torch.cuda.set_device(dev)
    wl = synth.WORKLOADS[5]
    E, H, F, T, k = wl.E, wl.H, wl.F, wl.T, wl.k
    masters = []
    for e in range(E):
        t = torch.empty(wl.W_e, dtype=torch.float16, device="cuda")
        synth.fill_expert_weights(wl, e, t)
        masters.append(t)
    p = synth.importance(wl)
    W = [wl.W_e] * E
    # a quarter of headroom beside the all-8-bit pages: the overlapped repage
    # keeps the changed experts' old pages until its commit
    pages8 = -(-3 * (F // 16) * (H // 128) // (65536 // (256 * 8)))
    ctx = mpe.Context(E, H, F, pool_pages=(5 * E * pages8) // 4)
    peaks, peak_kind = measured_peaks()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed(fn):
        torch.cuda.synchronize()
        ev0.record()
        r = fn()
        ev1.record()
        torch.cuda.synchronize()
        return r, ev0.elapsed_time(ev1)

    sched = synth.schedule(wl)
    phases = [(sched[2 * i][1], sched[2 * i + 1][1]) for i in range(len(sched) // 2)]
    # every phase's batch resident in HBM before the timed region
    batches = []
    for seed, _ in phases:
        ids, w = synth.routing(wl, seed=seed + 1000 * dist.rank)
        x = synth.activations(wl, seed=seed + 1000 * dist.rank, device="cuda")
        batches.append((x, torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda(), ids))
    out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    steps = phase_steps(args.steps, len(phases))
    B0 = synth.budget_for(wl, wl.avg_bits)
    bits0 = mpe.allocate_bits(p, W, B0)

    # initial quantize (timed), then W untimed warm-up steps on the first batch
    _, q_ms = timed(lambda: ctx.quantize_experts(masters, bits0))
    q_bytes = 4 * wl.sum_W + sum(int(b) * wl.W_e // 8 for b in bits0)
    if ctx.status() != 0:
        raise RuntimeError(f"device status {ctx.status():#x} after quantize")
    for _ in range(args.warmup):
        ctx.moe_ffn(batches[0][0], batches[0][1], batches[0][2], out)
    torch.cuda.synchronize()

    def pages_read(ids_np, cur):
        return sum(int(cur[e]) * wl.W_e // 8 for e in np.unique(ids_np))

    def gateup_bytes(ids_np, cur):
        act = np.unique(ids_np[(ids_np >= 0) & (ids_np < E)])
        return sum(int(cur[e]) * 2 * F * H // 8 for e in act) + T * H * 2 + T * k * F * 2

    # the timed region: K decode steps over the 10 phases, the repages between
    clocks = ClockSampler(dev)
    clocks.start()
    time.sleep(0.3)
    launches0 = ctx.kernel_launches()
    ev_d = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in phases]
    ev_r = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in phases]
    n_changed, widths = [], []
    dist.barrier()
    torch.cuda.synchronize()
    ev0.record()
    for i, (_, avg) in enumerate(phases):
        x, idt, wt, _ = batches[i]
        ev_d[i][0].record()
        for _ in range(steps[i]):
            ctx.moe_ffn(x, idt, wt, out)
        ev_d[i][1].record()
        widths.append(ctx.bits())
        ev_r[i][0].record()
        n_changed.append(ctx.repage(synth.budget_for(wl, avg), p))
        ev_r[i][1].record()
    ev1.record()
    torch.cuda.synchronize()
    dist.barrier()
    launches = ctx.kernel_launches() - launches0
    clk = clocks.stop()
    final_bits = ctx.bits()
    if ctx.status() != 0:
        raise RuntimeError(f"device status {ctx.status():#x} after the schedule")
    dec_ms_ph = [a.elapsed_time(b_) for a, b_ in ev_d]
    rep_ms_ph = [a.elapsed_time(b_) for a, b_ in ev_r]
    dec_ms_local = sum(dec_ms_ph)
    dec_ms = dist.max(dec_ms_local)
    region_ms = dist.max(ev0.elapsed_time(ev1))
    value = T * args.steps * dist.world / (dec_ms / 1e3)
    q_gbs = q_bytes / (q_ms / 1e3) / 1e9

    decode, repages = [], []
    for i, (_, avg) in enumerate(phases):
        cur = widths[i]
        pb = pages_read(batches[i][3], cur)
        ms = dec_ms_ph[i] / max(steps[i], 1)
        decode.append({"avg_bits": float(cur.mean()), "steps": steps[i],
                       "us_per_step": ms * 1e3 if steps[i] else None,
                       "packed_GB/s": pb / (ms / 1e3) / 1e9 if steps[i] else None})
        after = widths[i + 1] if i + 1 < len(widths) else final_bits
        changed = np.nonzero(after != cur)[0]
        nbytes = sum(2 * wl.W_e + int(after[e]) * wl.W_e // 8 for e in changed)
        rms = rep_ms_ph[i]
        repages.append({"avg_bits": avg, "changed": int(n_changed[i]), "ms": rms,
                        "bytes": nbytes,
                        "GB/s": nbytes / (rms / 1e3) / 1e9 if n_changed[i] else None,
                        "frac": nbytes / (rms / 1e3) / 1e9 / peaks["hbm_gbs"]
                        if n_changed[i] else None})
    moved = [r for r in repages if r["changed"]]
    rp_bytes = sum(r["bytes"] for r in moved)
    rp_ms = sum(r["ms"] for r in moved)
    dec_pages = sum(pages_read(batches[i][3], widths[i]) * steps[i] for i in range(len(phases)))

    # kernel durations: the same schedule again from the initial widths, with
    # CUDA events around each forward kernel on the context stream
    ctx.repage(B0, p)
    ctx.profile(True)
    gu_ms, gu_n, gu_bytes = 0.0, 0, 0.0
    tot = {}
    for i, (_, avg) in enumerate(phases):
        x, idt, wt, ids_np = batches[i]
        cur = ctx.bits()
        for _ in range(steps[i]):
            ctx.moe_ffn(x, idt, wt, out)
        prof = ctx.profile_read(reset=True)
        gu_ms += prof["gate_up"][0]
        gu_n += prof["gate_up"][1]
        gu_bytes += gateup_bytes(ids_np, cur) * prof["gate_up"][1]
        for kname, v in prof.items():
            a = tot.setdefault(kname, [0.0, 0])
            a[0] += v[0]
            a[1] += v[1]
        ctx.repage(synth.budget_for(wl, avg), p)
    ctx.profile(False)
    achieved = (gu_bytes / gu_n) / (gu_ms / gu_n / 1e3) / 1e9 if gu_n else None
    traffic_ratio = recorded_traffic_ratio("k_decode_gateup", wl.name)
    roofline = {"bound": "hbm", "kernel": "decode gate/up (k_decode<1, 0>), every launch of "
                "the schedule (3-, 4- and 8-bit pages)",
                "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"] if achieved else None,
                "peak_source": peak_kind,
                "traffic": traffic_ratio * gu_bytes / gu_n if (traffic_ratio and gu_n) else None,
                "algorithmic_bytes_per_launch": gu_bytes / gu_n if gu_n else None,
                "avg_launch_us": gu_ms / gu_n * 1e3 if gu_n else None}
    total_prof = max(sum(v[0] for v in tot.values()), 1e-9)
    kernel_us = {kn: round(v[0] / v[1] * 1e3, 2) for kn, v in tot.items() if v[1]}
    kernel_share = {kn: round(v[0] / total_prof, 4) for kn, v in tot.items() if v[1]}

    # a budget change while decode batches are served: synchronous repage then
    # the batches, against the overlapped repage (forward passes keep the old
    # pages until the commit); device time from the first call to the commit
    overlap = None
    x_l, idt_l, wt_l, ids_l = batches[-1]
    w_l = wt_l.cpu().numpy()
    n_dec = 5
    ev_first = torch.cuda.Event(enable_timing=True)
    # forwards on a high-priority stream: the library's side stream has the
    # lowest priority, so decode CTAs are scheduled ahead of the re-encode's
    hp = torch.cuda.Stream(priority=-1)
    torch.cuda.synchronize()
    try:
        with torch.cuda.stream(hp):
            res = {"sequential": [], "overlapped": []}
            first = {"sequential": [], "overlapped": []}
            for mode in ("sequential", "overlapped", "sequential", "overlapped"):
                for avg in (4.5, 6.0):
                    torch.cuda.synchronize()
                    ev0.record()
                    if mode == "sequential":
                        ctx.repage(synth.budget_for(wl, avg), p)
                    else:
                        ctx.repage_async(synth.budget_for(wl, avg), p)
                    for i in range(n_dec):
                        ctx.moe_ffn(x_l, idt_l, wt_l, out)
                        if i == 0:
                            ev_first.record()
                    if mode == "overlapped":
                        ctx.repage_commit(wait=True)
                    ev1.record()
                    torch.cuda.synchronize()
                    res[mode].append(ev0.elapsed_time(ev1))
                    first[mode].append(ev0.elapsed_time(ev_first))
            overlap = {"decode_batches": n_dec, "budget_changes": "6 -> 4.5 -> 6 avg bits, twice",
                       "forward_stream": "priority -1 (side stream: lowest)",
                       "sequential_ms": float(np.median(res["sequential"])),
                       "overlapped_ms": float(np.median(res["overlapped"])),
                       "first_batch_sequential_ms": float(np.median(first["sequential"])),
                       "first_batch_overlapped_ms": float(np.median(first["overlapped"]))}
    except mpe.MpeError as err:
        overlap = {"unavailable": str(err)}

    # the prefix-compatible variant on the same width sequence: a layered store
    # quantized at the initial widths, then the schedule's widths; a change
    # that only lowers widths drops layers and moves nothing
    prefix = None
    try:
        store = mpe.PrefixStore(E, H, F)
        _, pq_ms = timed(lambda: store.quantize(masters, bits0))
        psteps = []
        for wbits, r in zip(widths[1:] + [final_bits], repages):
            moved_b, pr_ms = timed(lambda: store.repage(wbits))
            psteps.append({"avg_bits": r["avg_bits"], "ms": pr_ms, "bytes": moved_b,
                           "packed_ms": r["ms"], "packed_bytes": r["bytes"]})
        for _ in range(3):
            store.moe_ffn(x_l, idt_l, wt_l, out)
        _, pd_ms = timed(lambda: [store.moe_ffn(x_l, idt_l, wt_l, out) for _ in range(5)])
        prefix = {"quantize_ms": pq_ms, "repage": psteps,
                  "repage_total_ms": sum(st["ms"] for st in psteps),
                  "repage_total_bytes": sum(st["bytes"] for st in psteps),
                  "packed_repage_total_ms": sum(st["packed_ms"] for st in psteps),
                  "packed_repage_total_bytes": sum(st["packed_bytes"] for st in psteps),
                  "decode_us_final_widths": pd_ms / 5 * 1e3}
        store.close()
        del store
    except mpe.MpeError as err:
        prefix = {"unavailable": str(err)}

    # end to end: the last phase's batch through the host-buffer entry point
    # (pinned host x, ids, w in; out back; copies inside the timed loop)
    hb = [(x_l.cpu().pin_memory(), torch.from_numpy(ids_l).pin_memory(),
           torch.from_numpy(w_l).pin_memory(), torch.empty(T, H, dtype=torch.bfloat16).pin_memory())
          for _ in range(2)]
    n_e2e = max(10, min(args.steps, 200))
    for i in range(3):
        ctx.moe_ffn_host(*hb[i % 2])
    dist.barrier()
    t0 = time.perf_counter()
    e2e_pipeline(ctx, hb, n_e2e)
    e2e_s = dist.max(time.perf_counter() - t0)
    e2e = {"value": T * n_e2e * dist.world / e2e_s, "unit": "tokens/s",
           "h2d_bytes_per_step": T * H * 2 + 2 * T * k * 4, "d2h_bytes_per_step": T * H * 2,
           "steps": n_e2e, "widths": "the schedule's final widths (6 bits average)",
           "api": E2E_API}

    cpu = None
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        slice_rows = 128
        n_slices = max(1, F // slice_rows)
        dt, frac = OracleSample(wl).run(n_slices, slice_rows)
        cpu = {"value": frac / dt, "unit": "tokens/s", "cores": cores_used(), "kind": "oracle",
               "sample": f"one token through one expert at 8 bits (all {F} ffn rows in "
                         f"{n_slices} slices; dequantize + SwiGLU in float64) = {frac:.4f} "
                         f"tokens of layer work",
               "quantize": oracle_quantize_rate(wl)}

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": dist.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dec_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": bench_config(wl),
        "bits_hist": bits_hist(bits0),
        "packed_weight_gbs": dec_pages / (dec_ms_local / 1e3) / 1e9,
        "packed_weight_frac_of_peak": dec_pages / (dec_ms_local / 1e3) / 1e9 / peaks["hbm_gbs"],
        "roofline": roofline,
        "kernel_us": kernel_us,
        "kernel_time_share": kernel_share,
        "schedule": {"region_ms": region_ms, "decode_ms": dec_ms,
                     "repage_ms": sum(rep_ms_ph),
                     "tokens_per_s_with_repages": T * args.steps * dist.world / (region_ms / 1e3)},
        "quantize": {"ms": q_ms, "GB/s": q_gbs, "frac": q_gbs / peaks["hbm_gbs"], "bytes": q_bytes,
                     "passes": "absmax read + encode read/write of the 22.5 GB master"},
        "repage_total": {"ms": rp_ms, "GB/s": rp_bytes / (rp_ms / 1e3) / 1e9 if rp_ms else None,
                         "frac": rp_bytes / (rp_ms / 1e3) / 1e9 / peaks["hbm_gbs"] if rp_ms else None,
                         "bytes": rp_bytes,
                         "timing": "CUDA events on the context stream around each mpe_repage call: "
                                   "the page-table upload, scales and encode of the changed experts; "
                                   "the width solve runs beside the decode steps queued before it "
                                   "(high-priority internal stream), its cost lands in the decode "
                                   "and schedule figures"},
        "repage": repages,
        "decode": decode,
        "repage_overlap": overlap,
        "prefix_variant": prefix,
        "gpu_launches": launches,
        "clocks": clk,
        "e2e": e2e,
        "cpu_baseline": cpu,
    }
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    ctx.close()


def run_prefix_variant(args, dist: Dist):
    """The prefix-compatible layered store on a decode workload: forward
    tokens/s at the workload's widths, plus one lowering and one raising width
    change (time and bytes moved). Inputs as for the packed format."""
    import torch

    from mixed_precision_expert_b200.build import build
    if dist.rank == 0:
        build()
    dist.barrier()
    import mixed_precision_expert_b200 as mpe
    import synth

    dev = dist.local_rank
    torch.cuda.set_device(dev)
    wl = synth.WORKLOADS[args.workload]
    if args.workload in (4, 5):
        raise SystemExit("the prefix variant runs on the decode workloads 1-3")
    E, H, F, T, k = wl.E, wl.H, wl.F, wl.T, wl.k
    masters = []
    for e in range(E):
        t = torch.empty(wl.W_e, dtype=torch.float16, device="cuda")
        synth.fill_expert_weights(wl, e, t)
        masters.append(t)
    bits = mpe.allocate_bits(synth.importance(wl), [wl.W_e] * E, wl.budget_bits)
    store = mpe.PrefixStore(E, H, F)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed(fn):
        torch.cuda.synchronize()
        ev0.record()
        r = fn()
        ev1.record()
        torch.cuda.synchronize()
        return r, ev0.elapsed_time(ev1)

    _, q_ms = timed(lambda: store.quantize(masters, np.full(E, 8, np.uint8)))
    low, low_ms = timed(lambda: store.repage(np.full(E, 3, np.uint8)))
    up, up_ms = timed(lambda: store.repage(bits))
    nb = min(16, args.steps + args.warmup)
    batches = []
    for i in range(nb):
        seed = 7_000_000 + 1000 * dist.rank + i
        ids, w = synth.routing(wl, seed=seed)
        x = synth.activations(wl, seed=seed, device="cuda")
        batches.append((x, torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda()))
    out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    for i in range(args.warmup):
        x, idt, wt = batches[i % nb]
        store.moe_ffn(x, idt, wt, out)
    dist.barrier()
    clocks = ClockSampler(dev)
    clocks.start()
    time.sleep(0.2)
    torch.cuda.synchronize()
    ev0.record()
    for i in range(args.steps):
        x, idt, wt = batches[i % nb]
        store.moe_ffn(x, idt, wt, out)
    ev1.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = dist.max(ev0.elapsed_time(ev1))
    # the packed format on the same masters, widths and batches, for comparison
    ctx = mpe.Context(E, H, F, path=mpe.PATH_DECODE)
    ctx.quantize_experts(masters, bits)
    for i in range(args.warmup):
        x, idt, wt = batches[i % nb]
        ctx.moe_ffn(x, idt, wt, out)
    torch.cuda.synchronize()
    ev0.record()
    for i in range(args.steps):
        x, idt, wt = batches[i % nb]
        ctx.moe_ffn(x, idt, wt, out)
    ev1.record()
    torch.cuda.synchronize()
    packed_ms = dist.max(ev0.elapsed_time(ev1))
    ctx.close()
    stored = sum(int(b) * wl.W_e // 8 for b in bits)
    line = {
        "metric": METRIC, "value": T * args.steps * dist.world / (ms / 1e3), "unit": "tokens/s",
        "n_gpus": dist.world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {**bench_config(wl), "variant": "prefix-compatible layered store"},
        "bits_hist": bits_hist(bits),
        "roofline": None,
        "stored_bytes": stored,
        "quantize_8bit_ms": q_ms,
        "repage_lower_to_3bit": {"ms": low_ms, "bytes_moved": low},
        "repage_raise_to_widths": {"ms": up_ms, "bytes_moved": up,
                                   "GB/s": up / (up_ms / 1e3) / 1e9 if up else None},
        "clocks": clk,
        "packed_ms_per_step": packed_ms / args.steps,
        "vs_packed_step": ms / packed_ms,
        "note": "forward pass of the variant: the streaming kernels (bulk copies into a "
                "shared-memory ring, mma.sync) reading each chunk's stored layers, merged in "
                "registers",
    }
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    store.close()


def main():
    args = parse_args()
    dist = Dist()
    if args.impl == "reference":
        run_reference(args, dist)
        return
    import torch
    torch.cuda.set_device(dist.local_rank)
    dist.init("nccl")
    try:
        if args.variant == "prefix":
            run_prefix_variant(args, dist)
        elif is_schedule(args_workload(args)):
            run_repage_schedule(args, dist)
        else:
            run_mpe(args, dist)
    finally:
        dist.close()


if __name__ == "__main__":
    main()
