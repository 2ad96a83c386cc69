"""Benchmark of the MoE layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
                    [--gemm-tiles auto|single|pair] [--no-backward] [--no-sweep] [--no-cpu-baseline]

One step is one whole layer forward (route, permute, grouped SwiGLU FFN,
unpermute/combine) over one batch of T synthetic tokens, through the C ABI
entry point moe_layer_forward_timed, which also records a CUDA event between
the stages so every stage is timed inside the steps. Under torchrun each rank
runs its own batch on its own GPU (token-sharded replicas: weak scaling, no
collective on the data path); `value` is the tokens of all ranks divided by
the slowest rank's device time. Rank 0 prints one JSON line, which also
carries the end-to-end figure (pinned host buffers, transfers inside the
timed region), the grouped GEMM's roofline, the SM clocks seen during the
timed region and a CPU-oracle baseline.

On one GPU the same line also carries:
  backward  ms per moe_layer_backward call on the headline workload and its
            GEMM rate (--no-backward leaves it out);
  sweep     every other workload (the scaled Mixtral layer, the skewed layer
            dropless, with capacity 1920 in the compact and the padded layout,
            many small experts with SwiGLU and with identity experts, and the
            tiny fp32 layer), each timed the same way with per-stage us,
            GB/s or TFLOP/s and fractions of the peaks (--no-sweep leaves it
            out).

--impl reference times the CPU oracle (fp64, numpy) on the host cores on a
bounded token sample of the same workload; under torchrun only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE layer tokens/s; dispatch+combine HBM GB/s; grouped-GEMM TFLOPS (1 B200)"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "mixtral_8x7b"
# tokens of the bounded CPU sample per workload (about 10-30 s of oracle work)
CPU_SAMPLE = {"mixtral_8x7b": 8192, "mixtral_scaled": 4096, "skewed": 4096, "many_small": 4096,
              "tiny_f32": 64}
# tokens per step of the reference arm (a few seconds of oracle work per step)
REF_STEP_SAMPLE = {"mixtral_8x7b": 1024, "mixtral_scaled": 1024, "skewed": 1024, "many_small": 1024,
                   "tiny_f32": 64}
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
L2_BYTES = 126 * 1000 * 1000
# Spin-kernel length (SM clock cycles, about 2 ms) that keeps the device busy
# while the host queues a timed sequence of launches.
HOST_LEAD_CYCLES = 4_000_000
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}



def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--gemm-tiles", choices=["auto", "single", "pair"], default="auto")
    ap.add_argument("--no-backward", action="store_true",
                    help="leave out the moe_layer_backward timing of the headline workload")
    ap.add_argument("--shape", default="",
                    help="override workload sizes, e.g. T=8192,E=2 (a smaller slice of the same layer for profiling)")
    ap.add_argument("--precision", choices=["bf16", "mxfp8"], default="bf16",
                    help="operands of the expert GEMMs of the timed layer")
    ap.add_argument("--no-sweep", action="store_true",
                    help="leave out the per-workload sweep that follows the headline on one GPU")
    return ap.parse_args()


def peaks():
    if os.path.exists(PEAKS_PATH):
        with open(PEAKS_PATH) as f:
            p = json.load(f)
        return p, "measured"
    return FALLBACK_PEAKS, "fallback"


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_id), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------- CPU oracle
def oracle_sample(wl, n_tokens, seed=0):
    """The first n_tokens of the workload as their own batch (drawn once)."""
    import workloads as W
    return W.draw(wl.with_(T=min(n_tokens, wl.T)), seed)


def oracle_time(inp):
    """Oracle (as it stands) on one sample: route, dispatch metadata, experts
    and combine. Returns (tokens/s, seconds, BLAS/OpenMP threads)."""
    import oracle as O
    from oracle import cases
    from threadpoolctl import threadpool_info

    wl = inp.wl
    t0 = time.perf_counter()
    O.layer_forward(cases.as64(inp.h), cases.as64(inp.w_router), cases.as64(inp.bias), wl.k, wl.expert_kind,
                    cases.weights_fn(inp) if wl.expert_kind == "swiglu" else None, wl.capacity)
    dt = time.perf_counter() - t0
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    return wl.T / dt, dt, threads


def run_reference(args, wl, rank):
    if rank != 0:
        return
    n = REF_STEP_SAMPLE.get(wl.name, 256)
    inp = oracle_sample(wl, n, args.seed)
    for _ in range(args.warmup):
        oracle_time(inp)
    times = []
    threads = 1
    for _ in range(args.steps):
        _, dt, threads = oracle_time(inp)
        times.append(dt)
    total = sum(times)
    value = inp.wl.T * args.steps / total
    sample = (f"first {inp.wl.T} tokens of {wl.name} as their own batch per step, {args.steps} steps; the oracle "
              f"batches tokens per expert, so its rate grows with the sample size (the cpu_baseline of the GPU "
              f"arm uses a larger sample)")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded)", "config": config_dict(wl, args.gpus),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": os.cpu_count(), "blas_threads": threads,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def combine_ranks(ms_local, tokens_per_rank, steps, world, device=None):
    """Whole-job throughput of token-sharded replicas: every rank processed
    tokens_per_rank tokens per step; the job took as long as its slowest rank.
    Returns (max device ms over ranks, tokens/s of all ranks)."""
    import torch
    import torch.distributed as dist

    ms = float(ms_local)
    if world > 1:
        t = torch.tensor([ms], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    return ms, tokens_per_rank * world * steps / (ms / 1e3)


def tiles_used(M, cfg):
    """Tile shape the grouped GEMMs take for cfg (AUTO resolved by the library)."""
    return {M.MOE_GEMM_TILES_SINGLE: "single (128x256)", M.MOE_GEMM_TILES_PAIR: "pair (256x256, 2 SMs)"}[
        M.moe_gemm_tiles_used(cfg)]


def config_dict(wl, n, flush=None):
    c = {"workload": wl.name, "T": wl.T, "d": wl.d, "E": wl.E, "k": wl.k, "d_ff": wl.F, "dtype": wl.dtype,
         "expert_kind": wl.expert_kind, "capacity": wl.capacity, "layout": wl.layout, "global_batch": wl.T * n,
         "parallelism": f"token-sharded replicas x{n}"}
    if flush is not None:
        c["l2"] = ("flushed between steps (256 MB write), steps timed one by one" if flush
                   else "not flushed: step inputs larger than 2x L2 (126 MB)")
    return c


# ---------------------------------------------------------------------------- GPU arm
# Workloads of the sweep that rides along with the headline line on one GPU
# (parity-test workloads, timed the same way as the headline).
SWEEP = ["mixtral_scaled", "skewed", "skewed_capacity", "skewed_capacity_padded", "many_small",
         "many_small_identity", "tiny_f32"]
SWEEP_STEPS, SWEEP_WARMUP = 10, 3


class Layer:
    """Device copies of one workload's inputs and the buffers of its steps."""

    def __init__(self, M, W, wl, seed, rank, dev, gemm_tiles="auto", host_h=True, precision="bf16"):
        import torch

        self.wl = wl
        self.dev = dev
        inp = W.draw(wl, seed)
        self.h_host = None
        if host_h:
            self.h_host = W.draw_h(wl, seed + rank).pin_memory() if rank else inp.h.pin_memory()
            self.h = self.h_host.to(dev)
        else:
            self.h = inp.h.to(dev)
        self.cfg = M.config(wl.T, wl.d, wl.E, wl.k, wl.F, wl.dtype, wl.expert_kind, wl.capacity, gemm_tiles,
                            wl.layout, precision=precision)
        self.wr = inp.w_router.to(dev)
        self.bias = None if inp.bias is None else inp.bias.to(dev)
        self.w13 = self.wd = None
        if wl.expert_kind == "swiglu":
            wg, wu = inp.w_gate.to(dev), inp.w_up.to(dev)
            self.w13 = M.moe_pack_weights(self.cfg, wg, wu)
            del wg, wu
            self.wd = inp.w_down.to(dev)
            if precision == "mxfp8":
                self.w13, self.wd = M.moe_pack_weights_mxfp8(self.cfg, self.w13, self.wd)
        del inp
        self.y = torch.empty((wl.T, wl.d), dtype=wl.torch_dtype, device=dev)
        self.counts = torch.empty(wl.E, dtype=torch.int32, device=dev)
        self.routed = torch.empty(wl.E, dtype=torch.int32, device=dev)
        self.ws = M.workspace(self.cfg, M.MOE_OP_LAYER, dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.M = M

    def step(self, stream, stage_events=None):
        self.M.moe_layer_forward(self.cfg, self.h, self.wr, self.bias, self.w13, self.wd, y=self.y,
                                 routed_counts=self.routed, counts=self.counts, ws=self.ws, status=self.status,
                                 stream=stream, stage_events=stage_events)

    def input_bytes(self):
        n = self.wl.T * self.wl.d * self.wl.elem_bytes + self.wr.numel() * self.wr.element_size()
        if self.w13 is not None:
            n += self.w13.numel() * self.w13.element_size() + self.wd.numel() * self.wd.element_size()
        return n


def _timed_pass(L, steps, stream, barrier, flush, scrub, with_stages, sampler=None):
    """One timed pass of `steps` layer steps. Without stages, two events per
    step bracket the moe_layer_forward call, so nothing is recorded inside the
    layer and its kernels chain as in use (programmatic dependent launches);
    with stages, the layer records its 5 stage events. Returns (ms, stage
    means or None)."""
    import contextlib

    import torch

    n_ev = 5 if with_stages else 2
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(steps)]
    for row in ev:
        for e in row:
            e.record(stream)
    torch.cuda.synchronize()
    with (sampler if sampler is not None else contextlib.nullcontext()):
        barrier()
        torch.cuda.synchronize()
        # a spin kernel ahead of the first event lets the host queue the timed
        # launches before the device reaches them, so the events bracket device
        # work only (host launch cost is part of the end-to-end figure)
        torch.cuda._sleep(HOST_LEAD_CYCLES)
        for i in range(steps):
            if flush:
                scrub.fill_(1)
            if with_stages:
                L.step(stream, ev[i])
            else:
                ev[i][0].record(stream)
                L.step(stream)
                ev[i][1].record(stream)
        torch.cuda.synchronize()
        barrier()
    if flush:
        ms = sum(row[0].elapsed_time(row[-1]) for row in ev)   # each step alone, scrub excluded
    else:
        ms = ev[0][0].elapsed_time(ev[-1][-1])                 # steps back to back
    stages = None
    if with_stages:
        stages = {name: statistics.mean(row[i].elapsed_time(row[i + 1]) for row in ev)
                  for i, name in enumerate(("route", "permute", "grouped_ffn", "combine"))}
    return ms, stages


def time_steps(L, steps, warmup, stream, barrier, sampler=None):
    """Device time of `steps` layer steps, timed as a user runs the layer (no
    events inside it), then a second pass of `steps` steps that records the
    layer's 5 stage events for the per-stage breakdown. When the step's
    inputs could stay in L2 (126 MB) between steps, a 256 MB buffer is
    written between steps and each step is timed alone.
    Returns (total ms of the first pass, mean in-step ms per stage of the
    second, whether L2 was flushed)."""
    import torch

    for _ in range(max(warmup, 3)):
        L.step(stream)
    torch.cuda.synchronize()
    flush = L.input_bytes() < 2 * L2_BYTES
    scrub = torch.empty(256 << 20, dtype=torch.uint8, device=L.dev) if flush else None
    ms, _ = _timed_pass(L, steps, stream, barrier, flush, scrub, False, sampler)
    _, stages = _timed_pass(L, steps, stream, barrier, flush, scrub, True)
    return ms, stages, flush


def main():
    args = parse()
    import torch

    import workloads as W

    wl = W.get(args.workload)
    if args.shape:
        kw = {k: int(v) for k, v in (item.split("=") for item in args.shape.split(","))}
        wl = wl.with_(name=f"{wl.name}[{args.shape}]", **kw)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, wl, rank)
        return

    import datetime

    import torch.distributed as dist

    import combine_router_gemm_softmax_b200 as M

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    # inputs: each rank draws its own batch (seed + rank), weights are the same
    M.lib()
    L = Layer(M, W, wl, args.seed, rank, dev, args.gemm_tiles, precision=args.precision)
    stream = torch.cuda.current_stream(dev)

    # ------------------------------------------------ timed region (device events)
    gpu_uuid = torch.cuda.get_device_properties(dev).uuid
    sampler = ClockSampler(f"GPU-{gpu_uuid}")
    ms, stages, flush = time_steps(L, args.steps, args.warmup, stream, barrier, sampler)
    ms_max, value = combine_ranks(ms, wl.T, args.steps, world, dev)
    launches_per_step = launches(L.cfg)
    st = int(L.status.item())

    # ------------------------------------------------ end to end: host buffers, copies inside the timed region
    # Every step copies its tokens from pinned host memory to the device, runs
    # the layer and copies its result back. Two device slots and separate copy
    # streams let step i+1's upload and step i-1's download overlap step i's
    # compute, as a serving loop would run it.
    e2e_ms = run_e2e(M, L.cfg, wl, L.h_host, L.h, L.y, L.wr, L.bias, L.w13, L.wd, L.ws, stream, dev, args.steps,
                     barrier)
    e2e_ms, e2e_value = combine_ranks(e2e_ms, wl.T, args.steps, world, dev)
    row_bytes = wl.d * wl.elem_bytes

    barrier()
    do_bwd = not args.no_backward and wl.expert_kind == "swiglu" and wl.dtype == "bf16" and args.precision == "bf16"
    bwd = run_backward(M, L.cfg, wl, L.h, L.wr, L.bias, L.w13, L.wd, L.ws, stream, dev, args.steps,
                       args.seed + rank) if do_bwd else None
    barrier()

    if rank == 0:
        pk, pk_kind = peaks()
        counts_np = L.counts.cpu().numpy()
        A_kept = int(counts_np.sum())
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": ms_max / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype if args.precision == "bf16" else "mxfp8",
            "data": "synthetic: seeded N(0,1) tokens, N(0,1/fan_in) random-init weights",
            "config": {**config_dict(wl, world, flush), "gemm_tiles": args.gemm_tiles,
                       "gemm_tiles_used": tiles_used(M, L.cfg), "precision": args.precision,
                       "combine": "fused into the down projection" if fused_combine(L.cfg) else "separate kernel"},
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": wl.T * row_bytes,
                    "d2h_bytes_per_step": wl.T * row_bytes, "ms_per_step": e2e_ms / args.steps,
                    "path": "pinned host h -> device, moe_layer_forward, device y -> pinned host; "
                            "two device slots, upload and download on their own streams overlap the "
                            "neighbouring steps' compute"},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": sampler.summary(),
            "status_word": st,
        }
        line["stages"] = stage_report(stages, wl, A_kept, pk, pk_kind, fused_combine(L.cfg), args.precision)
        line["stages"]["pass"] = ("a second pass of the same number of steps with the layer's 5 stage events "
                                  "recorded inside it; value and ms_per_step come from steps without them")
        line["roofline"] = roofline(stages, wl, A_kept, pk, pk_kind, args.precision)
        if bwd is not None:
            flops = 16.0 * A_kept * wl.d * wl.F          # incl. the recomputed gate/up GEMM
            bwd, bwd_saved, fwd_saving = bwd
            line["backward"] = {"ms_per_step": bwd, "tokens_per_s": wl.T / (bwd / 1e3),
                                "gemm_tflops": flops / (bwd / 1e3) / 1e12,
                                "frac_bf16": flops / (bwd / 1e3) / 1e12 / pk["bf16_tflops_sustained"],
                                "train_step_tokens_per_s": wl.T / ((bwd + ms_max / args.steps) / 1e3),
                                "steps": args.steps,
                                "note": "moe_layer_backward after one forward, steps back to back; "
                                        "gemm_tflops counts 16*A*d*F (dgrad, wgrad and the gate/up recompute) "
                                        "over the whole backward time",
                                "saved_preact": {
                                    "ms_per_step": bwd_saved, "forward_ms_per_step": fwd_saving,
                                    "gemm_tflops": 12.0 * A_kept * wl.d * wl.F / (bwd_saved / 1e3) / 1e12,
                                    "train_step_tokens_per_s": wl.T / ((bwd_saved + fwd_saving) / 1e3),
                                    "note": "forward keeps the gate/up pre-activations (MOE_PREACT_SAVE), the "
                                            "backward skips their recompute; gemm_tflops counts 12*A*d*F; "
                                            "forward_ms_per_step is that forward, 5 steps back to back"}}
        line["routing"] = {"routed_counts_max": int(L.routed.max().item()),
                           "routed_counts_mean": float(L.routed.float().mean().item()),
                           "empty_experts": int((L.routed == 0).sum().item()), "kept": A_kept,
                           "dropped": wl.T * wl.k - A_kept}
    if rank == 0 and world == 1 and not args.no_sweep:
        line["combine_separate"] = run_combine_separate(M, L, stream, barrier)
        if L.input_bytes() >= 2 * L2_BYTES:
            line["ops_alone"] = run_ops_alone(M, L, stream, barrier)
        if args.precision == "bf16" and wl.expert_kind == "swiglu" and wl.dtype == "bf16":
            line["mxfp8"] = run_mxfp8(M, L, stream, barrier)
    del L
    torch.cuda.empty_cache()

    if rank == 0 and world == 1 and not args.no_sweep:
        line["sweep"] = run_sweep(M, W, [n for n in SWEEP if n != wl.name], args.seed, dev, stream, barrier)
    if rank == 0:
        if not args.no_cpu_baseline and world == 1:
            n = CPU_SAMPLE.get(wl.name, 256)
            v, dt, threads = oracle_time(oracle_sample(wl, n, args.seed))
            line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": os.cpu_count(), "blas_threads": threads,
                                    "kind": "oracle",
                                    "sample": f"first {min(n, wl.T)} tokens of {wl.name} as their own batch, "
                                              f"{dt:.1f} s; the oracle batches tokens per expert, so its rate "
                                              f"grows with the sample size"}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def run_combine_separate(M, L, stream, barrier):
    """The headline layer again with the combine as its own kernel (the
    separate dispatch + combine HBM rate), same inputs, SWEEP_STEPS steps."""
    import copy

    pk, pk_kind = peaks()
    cfg0 = L.cfg
    L.cfg = copy.copy(cfg0)
    L.cfg.combine = M.MOE_COMBINE_SEPARATE
    try:
        ms, st, flush = time_steps(L, SWEEP_STEPS, SWEEP_WARMUP, stream, barrier)
    finally:
        L.cfg = cfg0
    A_kept = int(L.counts.sum().item())
    rep = stage_report(st, L.wl, A_kept, pk, pk_kind)
    return {"ms_per_step": ms / SWEEP_STEPS, "steps": SWEEP_STEPS, "permute": rep["permute"],
            "combine": rep["combine"], "dispatch_combine": rep["dispatch_combine"],
            "grouped_ffn_us": rep["grouped_ffn"]["us"]}


def run_ops_alone(M, L, stream, barrier, reps=20):
    """The three HBM-bound entry points of the headline layer, each called
    alone: 3 warm-up calls, then `reps` calls back to back on one stream
    between two events. Inside a layer step the router also pays for writing
    back the previous step's combine output (up to L2's 126 MB of dirty
    lines), and the combine leaves part of its own output in L2; called back
    to back, each op pays for its own writes."""
    import torch

    pk, pk_kind = peaks()
    cfg, wl = L.cfg, L.wl
    s = wl.elem_bytes
    T, d, E, k = wl.T, wl.d, wl.E, wl.k
    dev = L.dev
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    gates = torch.empty((T, k), dtype=torch.float32, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    ws = M.workspace(cfg, M.MOE_OP_PERMUTE, dev)
    M.moe_route(cfg, L.h, L.wr, L.bias, topk_idx=idx, topk_gate=gates, status=st, stream=stream)
    out = M.moe_permute(cfg, L.h, idx, ws=ws, status=st, stream=stream)
    A_kept = int(out["counts"].sum().item())
    y = torch.empty_like(L.y)
    calls = {
        "route": (lambda: M.moe_route(cfg, L.h, L.wr, L.bias, topk_idx=idx, topk_gate=gates, status=st,
                                      stream=stream),
                  T * d * s + E * d * s + T * k * 8),
        "permute": (lambda: M.moe_permute(cfg, L.h, idx, out=out, ws=ws, status=st, stream=stream),
                    T * k * 4 + T * d * s + A_kept * d * s),
        "combine": (lambda: M.moe_unpermute_combine(cfg, out["x_perm"], out["dest_row"], gates, y=y, status=st,
                                                    stream=stream),
                    A_kept * d * s + T * d * s + T * k * 8),
    }
    res = {}
    for name, (fn, nbytes) in calls.items():
        for _ in range(3):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        barrier()
        torch.cuda._sleep(HOST_LEAD_CYCLES)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        us = 1e3 * e0.elapsed_time(e1) / reps
        res[name] = {"us": us, "GB/s": nbytes / us / 1e3, "frac_hbm": nbytes / us / 1e3 / pk["hbm_gbs"],
                     "bytes": nbytes}
    if int(st.item()) & ~(M.MOE_STATUS_MX_SATURATED | M.MOE_STATUS_MX_UNDERFLOW):
        raise RuntimeError(f"ops alone: status word {int(st.item())}")
    res["reps"] = reps
    res["note"] = ("each entry point alone (moe_route; moe_permute with its own count kernel; "
                   "moe_unpermute_combine of x_perm as y_perm), calls back to back, inputs larger than L2")
    return res


def run_mxfp8(M, L, stream, barrier):
    """The headline workload with MXFP8 expert GEMMs (weights quantised from
    the same bf16 weights), SWEEP_STEPS steps; GEMM rate against an fp8 peak
    of twice the measured bf16 one (the nominal ratio)."""
    import copy

    import torch

    pk, pk_kind = peaks()
    cfg = copy.copy(L.cfg)
    cfg.precision = M.MOE_PRECISION_MXFP8
    cfg.combine = M.MOE_COMBINE_AUTO
    wcounts = torch.zeros(2, dtype=torch.int32, device=L.dev)
    w13, wd = M.moe_pack_weights_mxfp8(cfg, L.w13, L.wd, counts=wcounts)
    ws = M.workspace(cfg, M.MOE_OP_LAYER, L.dev)
    saved = (L.cfg, L.w13, L.wd, L.ws)
    L.cfg, L.w13, L.wd, L.ws = cfg, w13, wd, ws
    gpu_uuid = torch.cuda.get_device_properties(L.dev).uuid
    sampler = ClockSampler(f"GPU-{gpu_uuid}")
    try:
        ms, st, flush = time_steps(L, SWEEP_STEPS, SWEEP_WARMUP, stream, barrier, sampler)
        counters = M.mx_counters(ws)
    finally:
        L.cfg, L.w13, L.wd, L.ws = saved
    A_kept = int(L.counts.sum().item())
    del w13, wd, ws
    torch.cuda.empty_cache()
    # compact layout: the dispatch stage quantises the rows; padded: it copies
    # bf16 rows and the expert stage quantises them
    rep = stage_report(st, L.wl, A_kept, pk, pk_kind, False,
                       "mxfp8" if L.wl.layout == "compact" else "mxfp8, bf16 dispatch")
    wl = L.wl
    return {"ms_per_step": ms / SWEEP_STEPS, "tokens_per_s": wl.T * SWEEP_STEPS / (ms / 1e3), "steps": SWEEP_STEPS,
            "dtype": "mxfp8 (E4M3 elements, E8M0 scale per 32) with fp32 accumulation, bf16 y",
            "stages": rep, "gpu_launches_per_step": launches(cfg), "clocks": sampler.summary(),
            "counts": {"x_saturated": counters[0], "x_underflow": counters[1], "h_mid_saturated": counters[2],
                       "h_mid_underflow": counters[3], "weights_saturated": int(wcounts[0].item()),
                       "weights_underflow": int(wcounts[1].item())},
            "elements": {"x": A_kept * wl.d, "h_mid": A_kept * wl.F, "weights": 3 * wl.E * wl.d * wl.F},
            "peak_note": "frac_fp8 = TFLOP/s / (2 x bf16_tflops_sustained): the nominal dense fp8:bf16 ratio "
                         "applied to the measured bf16 peak"}


def run_sweep(M, W, names, seed, dev, stream, barrier):
    """Every other workload timed like the headline (in-step stage events,
    L2 flushed between steps when the inputs fit in it), one entry each."""
    import torch

    out = {}
    pk, pk_kind = peaks()
    for name in names:
        wl = W.get(name)
        L = Layer(M, W, wl, seed, 0, dev, host_h=False)
        gpu_uuid = torch.cuda.get_device_properties(dev).uuid
        sampler = ClockSampler(f"GPU-{gpu_uuid}")
        ms, stages, flush = time_steps(L, SWEEP_STEPS, SWEEP_WARMUP, stream, barrier, sampler)
        A_kept = int(L.counts.sum().item())
        entry = {"ms_per_step": ms / SWEEP_STEPS, "tokens_per_s": wl.T * SWEEP_STEPS / (ms / 1e3),
                 "steps": SWEEP_STEPS, "config": {**config_dict(wl, 1, flush), "gemm_tiles_used": tiles_used(M, L.cfg)},
                 "kept": A_kept,
                 "status_word": int(L.status.item()), "clocks": sampler.summary(),
                 "gpu_launches_per_step": launches(L.cfg)}
        if wl.dtype == "bf16":
            entry["stages"] = stage_report(stages, wl, A_kept, pk, pk_kind, fused_combine(L.cfg))
            if wl.expert_kind == "swiglu":
                mx = run_mxfp8(M, L, stream, barrier)
                entry["mxfp8"] = {"ms_per_step": mx["ms_per_step"], "tokens_per_s": mx["tokens_per_s"],
                                  "grouped_ffn": mx["stages"]["grouped_ffn"], "counts": mx["counts"]}
        else:
            entry["stages"] = {k: {"us": 1e3 * v} for k, v in stages.items()}
            entry["note"] = "fp32 SIMT path, sized for correctness, not rooflined"
        out[name] = entry
        del L
        torch.cuda.empty_cache()
    return out


def run_e2e(M, cfg, wl, h_host, h0, y0, wr, bias, w13, wd, ws, stream, dev, steps, barrier):
    """Device time of `steps` host-to-host layer steps (upload, layer, download),
    double-buffered over two device slots. Returns milliseconds."""
    import torch

    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    h_dev = [h0, torch.empty_like(h0)]
    y_dev = [y0, torch.empty_like(y0)]
    y_host = [torch.empty(y0.shape, dtype=y0.dtype, pin_memory=True) for _ in range(2)]
    ev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("in", "comp", "out")}

    def run(n):
        for i in range(n):
            sl = i % 2
            if i >= 2:
                s_in.wait_event(ev["comp"][sl])          # slot's previous step has read its tokens
            with torch.cuda.stream(s_in):
                h_dev[sl].copy_(h_host, non_blocking=True)
            ev["in"][sl].record(s_in)
            stream.wait_event(ev["in"][sl])
            if i >= 2:
                stream.wait_event(ev["out"][sl])         # slot's previous result has been downloaded
            M.moe_layer_forward(cfg, h_dev[sl], wr, bias, w13, wd, y=y_dev[sl], ws=ws, stream=stream)
            ev["comp"][sl].record(stream)
            s_out.wait_event(ev["comp"][sl])
            with torch.cuda.stream(s_out):
                y_host[sl].copy_(y_dev[sl], non_blocking=True)
            ev["out"][sl].record(s_out)
        for sl in range(min(n, 2)):
            stream.wait_event(ev["out"][sl])

    run(2)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    run(steps)
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def run_backward(M, cfg, wl, h, wr, bias, w13, wd, ws, stream, dev, steps, seed):
    """Device time (ms per call) of moe_layer_backward on the forward state
    left in ws, CUDA events around `steps` back-to-back calls. Returns
    (recompute ms, saved-pre-activation ms, forward ms with the
    pre-activations kept): the second form runs on a forward that kept
    them (MOE_PREACT_SAVE), timed the same way."""
    import copy

    import torch

    import workloads as W

    w13_t, wd_t = M.moe_pack_weights_backward(cfg, w13, wd, stream=stream)
    dy = W.draw_dy(wl, seed).to(dev)

    def timed(fn, n):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda._sleep(HOST_LEAD_CYCLES)
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n

    out = []
    for preact in (M.MOE_PREACT_RECOMPUTE, M.MOE_PREACT_SAVE):
        c = copy.copy(cfg)
        c.preact = preact
        fws = ws if preact == M.MOE_PREACT_RECOMPUTE else M.workspace(c, M.MOE_OP_LAYER, dev)
        fwd_ms = timed(lambda: M.moe_layer_forward(c, h, wr, bias, w13, wd, ws=fws, stream=stream), 5)
        bws = M.workspace(c, M.MOE_OP_BACKWARD, dev)
        out.append(timed(lambda: M.moe_layer_backward(c, h, wr, w13, w13_t, wd_t, dy, fws, with_bias=bias is not None,
                                                      ws=bws, stream=stream), steps))
        if preact == M.MOE_PREACT_SAVE:
            out.append(fwd_ms)
        del bws
        if fws is not ws:
            del fws
        torch.cuda.empty_cache()
    return tuple(out)


def fused_combine(cfg):
    """Whether moe_layer_forward lets the down projection write y (the rule in
    include/moe.h at MOE_COMBINE_*)."""
    return (cfg.combine == 2 and cfg.k <= 2 and cfg.dtype == 0 and cfg.expert_kind == 0 and cfg.gemm_tiles != 2
            and cfg.precision == 0)


def launches(cfg):
    """Kernels one moe_layer_forward launches: router (which also counts the
    experts per 128-token tile on the bf16 path; the fp32 path adds a count
    kernel), a separate scan only for large E * ceil(T/128), rank, row copy
    (in MXFP8 with the compact layout replaced by the dispatch that quantises
    the rows), the zero fill of the padded layout, the MXFP8 row quantisation
    of the padded layout, the expert stage and the combine (none when fused
    into the down projection)."""
    n_chunks = (cfg.T + 127) // 128
    count = 0 if cfg.dtype == 0 else 1
    scan = 0 if cfg.E * n_chunks <= 8192 else 1
    pad = 1 if cfg.layout == 1 and cfg.capacity > 0 else 0
    copy = 1
    ffn = {0: 2, 1: 0, 2: 1}[cfg.expert_kind]
    if cfg.precision == 1:
        ffn += 1                                     # the row quantisation (or the quantising dispatch)
        copy = 1 if cfg.layout == 1 else 0
    combine = 0 if fused_combine(cfg) else 1
    return 1 + count + scan + 1 + copy + pad + ffn + combine


def stage_report(st, wl, A_kept, pk, pk_kind, fused=False, precision="bf16"):
    """Per-stage us and rates of one timed run. fused: the combine ran inside
    the down projection (its interval is empty and grouped_ffn includes it).
    precision mxfp8: the expert GEMMs are compared with an fp8 peak taken as
    twice the measured bf16 one (the nominal dense fp8 : bf16 ratio)."""
    s = wl.elem_bytes
    T, d, E, k, F = wl.T, wl.d, wl.E, wl.k, wl.F
    hbm = pk["hbm_gbs"]
    tf = pk["bf16_tflops_sustained"]
    router_b = T * d * s + E * d * s + T * k * 8
    # the dispatch writes bf16 rows, or in MXFP8 E4M3 rows and a scale byte per 32
    permute_b = T * d * s + (A_kept * d * (1 + 1 / 32) if precision == "mxfp8" else A_kept * d * s)
    combine_b = A_kept * d * s + T * d * s + T * k * 8
    flops = 6.0 * A_kept * d * F if wl.expert_kind == "swiglu" else 0.0
    out = {
        "route": {"us": 1e3 * st["route"], "GB/s": router_b / st["route"] / 1e6},
        "permute": {"us": 1e3 * st["permute"], "GB/s": permute_b / st["permute"] / 1e6},
        "grouped_ffn": {"us": 1e3 * st["grouped_ffn"]},
        "combine": {"us": 1e3 * st["combine"], "GB/s": combine_b / st["combine"] / 1e6},
    }
    for key in ("route", "permute", "combine"):
        out[key]["frac_hbm"] = out[key]["GB/s"] / hbm
    if flops:
        out["grouped_ffn"]["TFLOP/s"] = flops / st["grouped_ffn"] / 1e9
        if precision.startswith("mxfp8"):
            out["grouped_ffn"]["frac_fp8"] = out["grouped_ffn"]["TFLOP/s"] / (2.0 * tf)
        else:
            out["grouped_ffn"]["frac_bf16"] = out["grouped_ffn"]["TFLOP/s"] / tf
    if fused:
        out["combine"] = {"us": 1e3 * st["combine"],
                          "fused": "written by the down projection's epilogue; its time is inside grouped_ffn"}
        out["dispatch_combine"] = {"note": "combine fused; see the combine_separate object for the separate kernel"}
    else:
        dc = (permute_b + combine_b) / ((st["permute"] + st["combine"]) / 1e3) / 1e9
        out["dispatch_combine"] = {"GB/s": dc, "frac_hbm": dc / hbm}
    out["peaks"] = {"hbm_gbs": hbm, "bf16_tflops_sustained": tf, "source": f"{pk_kind} (MEASURED_PEAKS.json)"
                    if pk_kind == "measured" else "fallback"}
    return out


def roofline(st, wl, A_kept, pk, pk_kind, precision="bf16"):
    if wl.expert_kind == "swiglu":
        flops = 6.0 * A_kept * wl.d * wl.F
        ach = flops / (st["grouped_ffn"] / 1e3) / 1e12
        peak = pk["bf16_tflops_sustained"] * (2.0 if precision == "mxfp8" else 1.0)
        return {"bound": "tensor", "kernel": "grouped_gemm (SwiGLU GEMM1 + GEMM2, one call)", "achieved": ach,
                "peak": peak, "unit": "TFLOP/s", "frac": ach / peak, "traffic": None,
                "traffic_note": "DRAM bytes come from ncu captures kept as summaries under profiles/; "
                                "this run does not measure them",
                "peak_source": (f"2 x bf16_tflops_sustained (nominal fp8:bf16 ratio), {pk_kind}"
                                if precision == "mxfp8" else f"bf16_tflops_sustained, {pk_kind}")}
    s = wl.elem_bytes
    b = wl.T * wl.d * s + A_kept * wl.d * s
    ach = b / (st["permute"] / 1e3) / 1e9
    return {"bound": "hbm", "kernel": "permute", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": ach / pk["hbm_gbs"], "traffic": None, "peak_source": f"hbm_gbs, {pk_kind}"}


if __name__ == "__main__":
    main()
