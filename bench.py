"""Benchmark of the DiT-MoE sparse expert layer forward on B200 (one process per GPU).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole layer (router, dispatch, expert GEMM1 with
GELU, expert GEMM2 with gates, combine) over one batch of the workload, inputs
resident in HBM.  Each step is timed on the device with CUDA events on the
launching stream; L2 is flushed between steps by a 256 MB write outside the
step's events.  With N > 1 (torchrun) every rank runs its own batch (weak
scaling; the batches are independent, so there is no data-path collective),
the timed region is bracketed by a barrier and a synchronize, and the max over
ranks is reported.  Rank 0 prints one JSON line.

The line's headline is the XL/2-8E2A workload; the key ``workloads`` adds the
device time of the other four workloads of the method (fewer steps, same
timing rules).  ``--gpus N`` without torchrun relaunches itself under
torch.distributed.run with N ranks on 127.0.0.1.

--impl reference times the fp64 CPU oracle (the only other implementation of
the method here) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from sparse_moe_layer_03_b200 import inputs as I  # noqa: E402
from sparse_moe_layer_03_b200 import metrics as M  # noqa: E402

METRIC = "MoE-layer tokens/sec and TFLOP/s on 1 B200; % of bf16 peak and % HBM BW"
DEFAULT_WORKLOAD = "xl2_8e2a_512"
L2_FLUSH_BYTES = 256 << 20
SPACER_CYCLES = 400_000          # ~0.2 ms of GPU sleep after each flush, outside the timed events
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NOMINAL_BF16_TFLOPS = 2250.0     # dense bf16 tensor rate, vendor figure
NOMINAL_HBM_GBS = 8000.0         # HBM3e bandwidth named by the workload's targets
# DRAM read + write bytes of one launch of each expert GEMM at the default workload (ncu, one pass,
# full size), valid only for the GEMM sources they were measured on: GEMM_SOURCES hashed to
# TRAFFIC_SOURCES_SHA.  Any change to those files makes the reported traffic null until re-measured.
GEMM_SOURCES = ("sparse_moe_layer_03_b200/csrc/gemm_tc2.cu", "sparse_moe_layer_03_b200/csrc/common.cuh",
                "sparse_moe_layer_03_b200/csrc/kernels.h",
                "sparse_moe_layer_03_b200/csrc/api.cu")      # api.cu builds the tensor maps the GEMMs load through
TRAFFIC_SOURCES_SHA = "a7f379751030705b"
MEASURED_TRAFFIC = {
    # second forward pass of profile_layer at XL (ncu, gpu__time_duration + dram__bytes_read/write)
    ("xl2_8e2a_512", "gemm1"): 335290112 + 1168311040,
    ("xl2_8e2a_512", "gemm2_combine"): 1495313920 + 220181760,
}
EXTRA_STEPS = 10                 # timed steps of each other workload in the ``workloads`` key


def gemm_sources_sha() -> str:
    h = hashlib.sha256()
    for rel in GEMM_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_traffic(workload: str, stage: str):
    """ncu DRAM bytes of one launch, or None when the GEMM sources changed since the capture."""
    if not TRAFFIC_SOURCES_SHA or gemm_sources_sha() != TRAFFIC_SOURCES_SHA:
        return None
    return MEASURED_TRAFFIC.get((workload, stage))


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


# ------------------------------------------------------------------ distributed plumbing

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def reduce_max(value: float, world: int, device=None) -> float:
    """Max of a per-rank float over all ranks (identity when world == 1)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: str):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", str(self.gpu), "-lms", "100"], stdout=open(self.path, "w"),
                                         stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.25)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        rows = []
        try:
            for line in open(self.path):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        finally:
            if self.path and os.path.exists(self.path):
                os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no nvidia-smi samples"]}

        def num(s):
            try:
                return float(s)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        loaded = [s for s in sm if s is not None and s > 0.5 * max(sm)] if sm else []
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def gpu_index_for(local_rank: int) -> str:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local_rank < len(ids):
            return ids[local_rank]
    return str(local_rank)


# ------------------------------------------------------------------ oracle timing (CPU baseline / reference arm)

def oracle_rate(w: I.Workload, inp: dict, n_tokens: int):
    """Time the fp64 oracle on a contiguous slice of the workload; returns tokens/s, seconds, cores."""
    from oracle import moe_oracle as O
    sl = {k: v for k, v in inp.items()}
    sl["x"] = inp["x"][:n_tokens]
    t0 = time.perf_counter()
    O.layer(sl, w.K, w.routing, w.alpha)
    dt = time.perf_counter() - t0
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        cores = os.cpu_count() or 1
    return n_tokens / dt, dt, cores


def calibrated_tokens(w: I.Workload, inp: dict, target_s: float) -> int:
    """Tokens of oracle work that take about target_s seconds on this host."""
    rate, _, _ = oracle_rate(w, inp, 128)
    return int(max(128, min(w.T, rate * target_s)))


# ------------------------------------------------------------------ our arm

def time_steps(stages, calls, stream, steps, flush_l2):
    """Run `steps` steps (each stage between CUDA events on `stream`, L2 flushed before every
    step outside the events); returns per-stage ms lists and per-step totals."""
    import torch
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)] for _ in range(steps)]
    for i in range(steps):
        flush_l2(i)
        for j, st in enumerate(stages):
            ev[i][j].record(stream)
            calls[st]()
        ev[i][len(stages)].record(stream)
    torch.cuda.synchronize()
    per_stage = {st: [ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(steps)] for j, st in enumerate(stages)}
    totals = [ev[i][0].elapsed_time(ev[i][len(stages)]) for i in range(steps)]
    return per_stage, totals


def other_workloads(args, device, world, flush_l2) -> dict:
    """Device time of every workload besides the headline one, on this rank (max over ranks)."""
    import torch
    from sparse_moe_layer_03_b200.layer import LayerShape, MoELayer
    peaks, _ = load_peaks()
    out = {}
    for key in I.WORKLOAD_ORDER:
        if key == args.workload:
            continue
        w = I.WORKLOADS[key]
        inp = I.make_inputs(w)
        L = MoELayer(LayerShape(w.T, w.D, w.H, w.E, w.K, w.n_shared, w.dtype, w.routing, w.alpha), inp, device)
        x = torch.as_tensor(inp["x"]).to(device=device, dtype=L.act_dtype)
        stages = ["route", "dispatch", "gemm1"] + (["gemm2_combine"] if L.fused else ["gemm2", "combine"])
        calls = {"route": lambda: L.route(x), "dispatch": lambda: L.dispatch(x), "gemm1": lambda: L.gemm1(x),
                 "gemm2": L.gemm2, "combine": L.combine, "gemm2_combine": L.gemm2_combine}
        stream = torch.cuda.current_stream(device)
        time_steps(stages, calls, stream, max(3, args.warmup), flush_l2)
        steps = min(args.steps, EXTRA_STEPS)
        per_stage, totals = time_steps(stages, calls, stream, steps, flush_l2)
        L.check()
        ms = reduce_max(sum(totals), world, device) / steps
        elem = 2 if w.dtype in ("bf16", "f16") else 4
        race = w.routing == "race"
        avg = {st: float(np.mean(v)) for st, v in per_stage.items()}
        g1 = M.gemm1_flops(w.T, w.D, w.H, w.K, w.n_shared)
        g2 = M.gemm2_flops(w.T, w.D, w.H, w.K, w.n_shared)
        work = {"route": ("GB/s", M.route_bytes(w.T, w.D, w.E, w.K, elem, race)),
                "dispatch": ("GB/s", M.dispatch_bytes(w.T, w.D, w.E, w.K, elem, race)),
                "gemm1": ("TFLOP/s", g1), "gemm2": ("TFLOP/s", g2), "gemm2_combine": ("TFLOP/s", g2),
                "combine": ("GB/s", M.combine_bytes(w.T, w.D, w.K, w.n_shared, elem))}
        st_out = {}
        for st in stages:
            unit, amount = work[st]
            rate = amount / (avg[st] * 1e-3) / (1e9 if unit == "GB/s" else 1e12)
            frac = rate / (peaks["hbm_gbs"] if unit == "GB/s" else peaks["bf16_tflops"])
            st_out[st] = {"ms": round(avg[st], 4), unit: round(rate, 1),
                          ("frac_hbm" if unit == "GB/s" else "frac_bf16"): round(frac, 3)}
        out[key] = {"workload": w.name, "dtype": w.dtype, "T": w.T, "steps": steps,
                    "ms_per_step": round(ms, 4), "tokens/s": round(w.T * world / (ms * 1e-3), 1),
                    "layer_tflops": round(M.gemm_flops(w.T, w.D, w.H, w.K, w.n_shared) / (ms * 1e-3) / 1e12, 1),
                    "stages": st_out}
        del L, x, inp
        torch.cuda.empty_cache()
    return out


def run_ours(args, w: I.Workload, rank: int, world: int, local: int) -> dict:
    import torch
    from sparse_moe_layer_03_b200 import binding as B
    from sparse_moe_layer_03_b200.layer import LayerShape, MoELayer, global_balance_loss

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)

    # each rank draws its own batch (seed offset by rank); the weights are the workload's
    inp = I.make_inputs(w)
    if rank > 0:
        inp["x"] = I.make_inputs(I.Workload(**{**w.__dict__, "seed": w.seed + 1000 * rank}))["x"]
    shape = LayerShape(w.T, w.D, w.H, w.E, w.K, w.n_shared, w.dtype, w.routing, w.alpha,
                       seq_len=getattr(args, "seq_len", 0), fuse_combine=args.fuse_combine == "on")
    L = MoELayer(shape, inp, device)
    dt = L.act_dtype
    x_host = torch.as_tensor(inp["x"]).to(dt).pin_memory()
    x = x_host.to(device, non_blocking=False)
    out_host = torch.empty((w.T, w.D), dtype=dt).pin_memory()
    aux_host = torch.empty((1,), dtype=torch.float32).pin_memory()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    flush_clean = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)

    # with the combine folded into GEMM2 (bf16, n_s >= 1) the step has four stages
    stages = (["route", "dispatch", "gemm1", "gemm2_combine"] if L.fused
              else ["route", "dispatch", "gemm1", "gemm2", "combine"])
    mod = res = None
    x_in = x
    if args.adaln == "on":
        # per-image adaLN parameters (the synthetic conditioning of the workload's images)
        g = torch.Generator().manual_seed(w.seed + 77)
        nimg = w.T // w.tokens_per_image
        per_img = lambda scale, shift: (torch.randn((nimg, w.D), generator=g) * scale + shift).to(dt).to(device)
        gamma, beta, alpha = per_img(0.3, 1.0), per_img(0.3, 0.0), per_img(0.5, 0.0)
        L.x_mod = torch.empty_like(x)
        mod = B.make_adaln(gamma, beta, w.tokens_per_image, 1e-5, L.x_mod)
        res = B.make_residual(x, alpha, w.tokens_per_image)
        x_in = L.x_mod
    if args.global_aux == "on":
        # the balance loss of the whole batch over every rank: statistics, one all-reduce of 2E values, loss
        stages.insert(1, "balance_exchange")
    calls = {"route": lambda: L.route(x, mod), "dispatch": lambda: L.dispatch(x_in), "gemm1": lambda: L.gemm1(x_in),
             "gemm2": L.gemm2, "combine": lambda: L.combine(res), "gemm2_combine": lambda: L.gemm2_combine(res),
             "balance_exchange": lambda: global_balance_loss(L)}

    def flush_l2(i):
        # write a buffer larger than L2; then read another one as large, so the written lines
        # go back to DRAM here and not inside the next stage's events (a write-back L2 keeps
        # them dirty until evicted); then idle the GPU briefly so the host has enqueued the
        # whole step before the GPU reaches it (every stage is then timed as device time alone)
        flush.fill_(float(i))
        flush_clean.sum()
        torch.cuda._sleep(SPACER_CYCLES)

    time_steps(stages, calls, stream, args.warmup, flush_l2)
    L.check()

    barrier(world, device)
    torch.cuda.synchronize(device)
    with ClockSampler(gpu_index_for(local)) as clk:
        per_stage, totals = time_steps(stages, calls, stream, args.steps, flush_l2)
    barrier(world, device)
    L.check()
    clocks = clk.summary()
    my_ms = sum(totals)
    max_ms = reduce_max(my_ms, world, device)
    ms_per_step = max_ms / args.steps

    # ---- end to end through the public API: pinned host x in, host out + loss back, per step.
    # MoELayer.forward_host_pipelined overlaps step i+1's input copy and step i-1's output copy
    # with step i's compute (two device buffers); the timed region holds all K steps with
    # every copy, measured on the device from the first copy in to the last copy out.
    xs_host = [x_host] * args.steps
    outs_host = [torch.empty((w.T, w.D), dtype=dt).pin_memory() for _ in range(2)]
    auxs_host = [torch.empty((1,), dtype=torch.float32).pin_memory() for _ in range(2)]
    L.forward_host_pipelined(xs_host[:3], [outs_host[i % 2] for i in range(3)], [auxs_host[i % 2] for i in range(3)])
    torch.cuda.synchronize(device)
    barrier(world, device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    L.forward_host_pipelined(xs_host, [outs_host[i % 2] for i in range(args.steps)],
                             [auxs_host[i % 2] for i in range(args.steps)])
    e1.record(stream)                      # after the call returned: every copy out has finished
    torch.cuda.synchronize(device)
    e2e_ms = reduce_max(e0.elapsed_time(e1), world, device) / args.steps

    # the balance loss's gradient through the router (not part of the forward step): timed on its own
    bwd_ms = None
    if w.routing in ("topk", "race") and not getattr(args, "seq_len", 0):   # covers the whole-call loss only
        bws = torch.empty(B.moe_backward_workspace_size(L.cfg), dtype=torch.uint8, device=device)
        dwg = torch.empty((w.E, w.D), dtype=torch.float32, device=device)
        dbias = torch.empty((w.E,), dtype=torch.float32, device=device)
        dx = torch.empty_like(x)
        run_bwd = lambda: B.moe_balance_loss_backward(L.cfg, x, L.wg, L.router_bias, L.counts, 1.0, dwg, dbias, dx,
                                                      bws, bws.numel(), L.stream())
        for _ in range(3):
            run_bwd()
        b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        times = []
        for i in range(5):
            flush_l2(i)
            b0.record(stream)
            run_bwd()
            b1.record(stream)
            torch.cuda.synchronize(device)
            times.append(b0.elapsed_time(b1))
        bwd_ms = float(np.median(times))

    # the whole layer's backward (experts, gates, router; not part of the forward step): on its own
    layer_bwd = None
    if w.dtype in ("bf16", "f16") and not getattr(args, "seq_len", 0) and L.x_perm is not None:
        L.forward(x)
        dout = torch.randn((w.T, w.D), generator=torch.Generator().manual_seed(5)).to(device=device, dtype=dt)
        for _ in range(2):
            L.backward(x, dout)
        torch.cuda.synchronize(device)
        times = []
        for i in range(5):
            flush_l2(i)
            b0 = torch.cuda.Event(enable_timing=True)
            b1 = torch.cuda.Event(enable_timing=True)
            b0.record(stream)
            L.backward(x, dout)
            b1.record(stream)
            torch.cuda.synchronize(device)
            times.append(b0.elapsed_time(b1))
        L.check()
        layer_bwd = float(np.median(times))

    # expert-selection frequency per patch position of the last routing (not part of the step): on its own
    freq_ms = None
    if w.tokens_per_image and w.T % w.tokens_per_image == 0:
        for _ in range(3):
            L.expert_frequency(w.tokens_per_image)
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        times = []
        for i in range(5):
            flush_l2(i)
            f0.record(stream)
            L.expert_frequency(w.tokens_per_image)
            f1.record(stream)
            torch.cuda.synchronize(device)
            times.append(f0.elapsed_time(f1))
        freq_ms = float(np.median(times))
        L.check()

    others = other_workloads(args, device, world, flush_l2) if args.other_workloads == "on" else None

    result = None
    if rank == 0:
        result = report(args, w, L, per_stage, ms_per_step, e2e_ms, clocks, world, inp)
        if others is not None:
            result["workloads"] = others
        if freq_ms is not None:
            kmax = w.E if w.routing == "race" else w.K
            moved = w.T * kmax * 4 + (w.T * 4 if w.routing == "race" else 0) + w.tokens_per_image * w.E * 4
            result["expert_frequency"] = {"ms": round(freq_ms, 4), "GB/s": round(moved / (freq_ms * 1e-3) / 1e9, 1),
                                          "what": "moe_expert_frequency per patch position (selection read once, "
                                                  "[positions, E] counts written), timed separately"}
        if layer_bwd is not None:
            # five GEMMs of GEMM1's size: the pre-activations again, dU, dx, dW2, dW1
            bflops = 5 * M.gemm1_flops(w.T, w.D, w.H, w.K, w.n_shared)
            result["layer_backward"] = {"ms": round(layer_bwd, 4),
                                        "gemm_TFLOP/s": round(bflops / (layer_bwd * 1e-3) / 1e12, 1),
                                        "what": "MoELayer.backward: moe_expert_backward (gather of dY, five "
                                                "tcgen05 GEMMs with MN-major operands, bias column sums, gate "
                                                "gradient) + moe_router_backward; timed separately; TFLOP/s counts "
                                                "the five GEMMs over the whole time"}
        if bwd_ms is not None:
            elem = 2 if w.dtype in ("bf16", "f16") else 4
            moved = 2 * w.T * w.D * elem + w.E * w.D * (elem + 4)
            result["balance_backward"] = {"ms": round(bwd_ms, 4), "GB/s": round(moved / (bwd_ms * 1e-3) / 1e9, 1),
                                          "what": "moe_balance_loss_backward (dWg, db, dx of the balance loss), "
                                                  "timed separately; x read and dx written once"}
    if world > 1:
        import torch.distributed as dist
        barrier(world, device)
        dist.destroy_process_group()
    return result


def report(args, w, L, per_stage, ms_per_step, e2e_ms, clocks, world, inp) -> dict:
    peaks, peak_kind = load_peaks()
    elem = 2 if w.dtype in ("bf16", "f16") else 4
    race = w.routing == "race"
    avg = {s: float(np.mean(v)) for s, v in per_stage.items()}
    g1 = M.gemm1_flops(w.T, w.D, w.H, w.K, w.n_shared)
    g2 = M.gemm2_flops(w.T, w.D, w.H, w.K, w.n_shared)
    fused = "gemm2_combine" in avg
    stage_work = {
        "route": ("GB/s", M.route_bytes(w.T, w.D, w.E, w.K, elem, race)),
        "dispatch": ("GB/s", M.dispatch_bytes(w.T, w.D, w.E, w.K, elem, race)),
        "gemm1": ("TFLOP/s", g1),
    }
    if fused:
        stage_work["gemm2_combine"] = ("TFLOP/s", g2)
    else:
        stage_work["gemm2"] = ("TFLOP/s", g2)
        stage_work["combine"] = ("GB/s", M.combine_bytes(w.T, w.D, w.K, w.n_shared, elem))
    g2_stage = "gemm2_combine" if fused else "gemm2"
    mem_stages = ("route", "dispatch") if fused else ("route", "dispatch", "combine")
    hbm = peaks["hbm_gbs"]
    tc_peak = peaks["bf16_tflops_sustained"]
    tc_burst = peaks["bf16_tflops"]
    stages_out = {}
    for s, (unit, work) in stage_work.items():
        ms = avg[s]
        if unit == "GB/s":
            a = work / (ms * 1e-3) / 1e9
            stages_out[s] = {"ms": round(ms, 4), "GB/s": round(a, 1), "frac_hbm": round(a / hbm, 3)}
        else:
            a = work / (ms * 1e-3) / 1e12
            stages_out[s] = {"ms": round(ms, 4), "TFLOP/s": round(a, 1), "frac_bf16": round(a / tc_peak, 3)}
    if "balance_exchange" in avg:
        stages_out["balance_exchange"] = {
            "ms": round(avg["balance_exchange"], 4),
            "what": "moe_balance_stats, an all-reduce of the 2E statistics over the ranks (NCCL; none at one "
                    "process), moe_balance_loss_from_stats"}
    dom = "gemm1" if avg["gemm1"] >= avg[g2_stage] else g2_stage
    dom_flops = g1 if dom == "gemm1" else g2
    achieved = dom_flops / (avg[dom] * 1e-3) / 1e12
    gemm_ms = avg["gemm1"] + avg[g2_stage]
    mem_ms = sum(avg[s] for s in mem_stages)
    mem_bytes = sum(stage_work[s][1] for s in mem_stages)
    total_tokens = w.T * world
    value = total_tokens / (ms_per_step * 1e-3)
    ntok = calibrated_tokens(w, inp, 15.0)
    rate, secs, cores = oracle_rate(w, inp, ntok)
    h2d = w.T * w.D * elem
    d2h = w.T * w.D * elem + 4
    # route (finalize fused; race: + one cooperative select-and-finalize launch), dispatch count +
    # gather, GEMM1, GEMM2 (+ combine unless folded into GEMM2)
    launches_per_step = (1 + (1 if race else 0)) + 2 + 1 + 1 + (0 if fused else 1)
    if getattr(args, "seq_len", 0):
        launches_per_step += 1                  # the per-image loss kernel after the router
    if "balance_exchange" in avg:
        launches_per_step += 2                  # statistics and loss kernels (the all-reduce is NCCL's)
    return {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name, "T": w.T, "D": w.D, "H": w.H, "E": w.E, "K": w.K, "n_shared": w.n_shared,
                   "routing": w.routing, "batch": w.batch, "tokens_per_image": w.tokens_per_image,
                   "global_batch_tokens": total_tokens, "parallelism": f"dp{world}" if world > 1 else "single",
                   "adaln": ("modulation in the router and the gated residual in the combine (e2e: the plain "
                             "layer)") if args.adaln == "on" else "off",
                   "balance_loss": ("whole batch over all ranks (one all-reduce of 2E statistics per step; e2e: "
                                    "per rank)") if args.global_aux == "on" else
                                   (f"per rank, mean over images of {args.seq_len} tokens (router stores P; "
                                    f"one more launch)" if getattr(args, "seq_len", 0) else
                                    "per rank (this rank's batch)"),
                   "l2": "flushed between steps (256 MB written, then another 256 MB read so the written lines "
                         "return to DRAM before the step, then a 0.2 ms GPU sleep so the host is ahead; all "
                         "outside each step's events)"},
        "layer_tflops": round(M.gemm_flops(w.T, w.D, w.H, w.K, w.n_shared) / (ms_per_step * 1e-3) / 1e12, 1),
        "gemm_tflops": round((g1 + g2) / (gemm_ms * 1e-3) / 1e12, 1),
        "gemm_frac_bf16": round((g1 + g2) / (gemm_ms * 1e-3) / 1e12 / tc_peak, 3),
        "mem_stages_GBps": round(mem_bytes / (mem_ms * 1e-3) / 1e9, 1),
        "mem_stages_frac_hbm": round(mem_bytes / (mem_ms * 1e-3) / 1e9 / hbm, 3),
        "vs_nominal": {"gemm_frac": round((g1 + g2) / (gemm_ms * 1e-3) / 1e12 / NOMINAL_BF16_TFLOPS, 3),
                       "mem_stages_frac": round(mem_bytes / (mem_ms * 1e-3) / 1e9 / NOMINAL_HBM_GBS, 3),
                       "denominators": f"{NOMINAL_BF16_TFLOPS} TFLOP/s dense bf16, {NOMINAL_HBM_GBS} GB/s HBM "
                                       "(nominal B200 figures; the fractions above use the measured peaks)"},
        "stages": stages_out,
        "roofline": {"kernel": f"tcgen05 CTA-pair grouped expert GEMM ({dom}, one launch per step"
                               + (", combine folded into the shared experts' tiles)" if dom == "gemm2_combine" else ")"),
                     "bound": "tensor", "achieved": round(achieved, 1), "peak": tc_burst, "unit": "TFLOP/s",
                     "frac": round(achieved / tc_burst, 3),
                     "traffic": measured_traffic(args.workload, dom) if w.dtype == "bf16" else None,
                     "peak_source": f"{peak_kind} bf16_tflops (burst: the timed region is short and the "
                                    f"sampled SM clock stays at its maximum); vs sustained "
                                    f"{tc_peak}: {round(achieved / tc_peak, 3)}"
                                    + ("; fp16 takes the bf16 figure (equal nominal dense rates)"
                                       if w.dtype == "f16" else "")},
        "cpu_baseline": {"value": round(rate, 2), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{ntok} contiguous tokens of this workload through the whole fp64 oracle "
                                   f"layer (router, selection, experts, combine); {secs:.1f} s"},
        "e2e": {"value": round(total_tokens / (e2e_ms * 1e-3), 1), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4),
                "how": "MoELayer.forward_host_pipelined over K host batches: pinned x in, out and "
                       "balance loss back every step; copies overlap neighbouring steps' compute"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }


# ------------------------------------------------------------------ reference arm (the oracle)

def run_reference(args, w: I.Workload, rank: int, world: int) -> dict:
    if rank != 0:
        return None
    inp = I.make_inputs(w)
    ntok = calibrated_tokens(w, inp, 6.0)
    times = []
    cores = 1
    for i in range(args.warmup + args.steps):
        rate, secs, cores = oracle_rate(w, inp, ntok)
        if i >= args.warmup:
            times.append(secs)
    secs = sum(times) / len(times)
    value = ntok / secs
    return {"impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(secs * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "T": w.T, "D": w.D, "H": w.H, "E": w.E, "K": w.K,
                       "n_shared": w.n_shared, "routing": w.routing},
            "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": f"each step: {ntok} contiguous tokens of the workload through the whole "
                                       f"fp64 oracle layer on the host cores"},
            "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def relaunch(n: int, argv: list):
    """Start this script under torch.distributed.run with n ranks (one per GPU) on 127.0.0.1 and
    exit with its status; rank 0 prints the line."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__), *argv]
    sys.exit(subprocess.call(cmd))


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(I.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--fuse-combine", default="on", choices=["on", "off"],
                    help="fold the combine into the shared experts' GEMM2 (bf16, n_s >= 1)")
    ap.add_argument("--adaln", default="off", choices=["on", "off"],
                    help="time the layer inside its DiT block: adaLN modulation in the router and the "
                         "adaLN-Zero gated residual in the combine (per-image gamma, beta, alpha)")
    ap.add_argument("--global-aux", default="off", choices=["on", "off"],
                    help="balance loss of the whole batch over every rank (statistics all-reduced each step) "
                         "instead of each rank's own")
    ap.add_argument("--dtype", default=None, choices=["bf16", "f16"],
                    help="storage type of activations and weights (default: the workload's); f16 is the "
                         "pages' inference type")
    ap.add_argument("--seq-len", type=int, default=0,
                    help="balance loss per image of this many tokens, averaged over the images (0: over the "
                         "whole call)")
    ap.add_argument("--other-workloads", default="on", choices=["on", "off"],
                    help="also time the method's other workloads (key `workloads` of the line)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.global_aux == "on" and args.seq_len:
        ap.error("--global-aux gives the whole-batch loss; it does not combine with --seq-len")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        relaunch(args.gpus, sys.argv[1:] if argv is None else list(argv))
        return
    rank, world, local = dist_env()
    if world != args.gpus:
        ap.error(f"--gpus {args.gpus} but the launcher started {world} rank(s)")
    w = I.WORKLOADS[args.workload]
    if args.seq_len and (args.seq_len < 0 or w.T % args.seq_len):
        ap.error(f"--seq-len must divide T={w.T}")
    if args.dtype and args.dtype != w.dtype:
        base = w.name[: -len(", " + w.dtype)] if w.name.endswith(", " + w.dtype) else w.name
        w = dataclasses.replace(w, dtype=args.dtype, name=f"{base}, {args.dtype}")
    if args.impl == "reference":
        res = run_reference(args, w, rank, world)
    else:
        res = run_ours(args, w, rank, world, local)
    if rank == 0 and res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
