#!/usr/bin/env python
"""Throughput of the full MoE layer forward on B200 (one JSON line on rank 0).

Workload (full_layer_bf16): T=16384 tokens, hidden 2048, 256 routed SwiGLU
experts (intermediate 512), top-8, capacity factor 1.25 (C=640), one always-on
shared SwiGLU expert (intermediate 512), router bias skew, aux coefficient 0.001.
One step = router GEMM, softmax/top-k/gates, slot scan, gather, routed experts,
shared expert, combine and load statistics over one batch.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torchrun, one rank per GPU, each rank on its own batch
(weak scaling; no collective on the data path).  Timing: CUDA events on the
launch stream around every step, an L2 flush (a 256 MiB write) between steps,
a barrier + synchronize on both sides of the timed loop, max over ranks.
``--impl reference`` times the fp64 CPU oracle on a bounded token sample of the
same workload (rank 0 only).  The JSON line also carries the other workloads
(router only, top-1 dispatch/combine, tiny fp32 GELU layer and its training
step, fp32 fwd+bwd, the expert-parallel step with 4 ranks on one GPU, and the
full-layer training step); ``--workload NAME`` times one of them alone (with
``--tokens/--experts`` for smaller full-layer shapes), for profiling captures.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE layer tokens/sec fwd(+bwd) on 1 B200; % of HBM and bf16 tensor-core roofline"
UNIT = "tokens/s"
WORKLOAD = dict(workload="full_layer_bf16", T=16384, hidden=2048, experts=256, top_k=8, expert_intermediate=512,
                shared_experts=1, shared_intermediate=512, capacity_factor=1.25, capacity=640, aux_coef=0.001)
KERNELS_PER_STEP = 10  # fused router, reduce, scan, gather, 2 routed GEMMs, 2 shared GEMMs, combine, aux
# DRAM bytes (read + write) per algorithmic byte of the two routed expert-FFN kernels (the SwiGLU
# gate/up tcw_kernel and the down projection tc_gemm_kernel<BF16>), from one ncu capture of
# dram__bytes_read.sum + dram__bytes_write.sum on the T=8192, E=128 case (two launches of each;
# profiles/routed_ffn_dram_traffic_T8192_E128.md); the bench scales it by its own algorithmic
# bytes.  Set back to None when either kernel changes.
TRAFFIC_PER_ALG_BYTE = {"gate_up": 1.024, "down": 0.943}


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return dict(hbm=p["hbm_gbs"], bf16=p["bf16_tflops"], bf16_sustained=p["bf16_tflops_sustained"],
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


class ClockSampler:
    """Polls NVML (SM clock, max clock, power, clock-event reasons) in a thread."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int):
        self.samples, self.reasons, self.ok = [], set(), False
        self.max_mhz = None
        try:
            import pynvml

            pynvml.nvmlInit()
            uuid = None
            try:
                uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            except Exception:
                pass
            h = None
            if uuid:
                for i in range(pynvml.nvmlDeviceGetCount()):
                    hh = pynvml.nvmlDeviceGetHandleByIndex(i)
                    u = pynvml.nvmlDeviceGetUUID(hh)
                    u = u.decode() if isinstance(u, bytes) else u
                    if u.replace("GPU-", "") == uuid.replace("GPU-", ""):
                        h = hh
            if h is None:
                h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nv, self.h = pynvml, h
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append(mhz)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.ok:
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(v: float, world: int, device="cuda") -> float:
    """Largest per-rank value (the slowest rank's time decides the job time)."""
    if world == 1:
        return v
    import torch.distributed as dist

    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank_step: int, steps: int, world: int, max_ms: float) -> float:
    """Whole-job tokens/s: every rank's tokens over the slowest rank's device time."""
    return tokens_per_rank_step * steps * world / (max_ms / 1e3)


def rank_seed(rank: int) -> int:
    """Weak scaling: each rank draws its own batch (and its own random-init weights) from its seed."""
    return rank


# ------------------------------------------------------------------------------------------------
def oracle_step(cfg64, S: int):
    """The fp64 CPU oracle over the first S tokens of the batch (route .. combine, aux)."""
    from oracle import oracle as O

    xs = cfg64["x"][:S]
    s = O.router_logits(xs, cfg64["w_router_de"], cfg64["bias"])
    _, sel, gates, counts, psum = O.route(s, WORKLOAD["top_k"])
    C = O.capacity(S, WORKLOAD["top_k"], WORKLOAD["experts"], WORKLOAD["capacity_factor"])
    disp = O.dispatch(sel, WORKLOAD["experts"], C)
    shared = O.expert_rows("swiglu", xs, np.arange(S), np.zeros(S, np.int64), cfg64["shared"])
    y = O.layer_rows("swiglu", xs, sel, disp["kept"], gates, cfg64["experts"], base_kind="tensor", base=shared)
    O.aux(counts, psum, S, WORKLOAD["top_k"])
    return y


def oracle_inputs(cfg):
    from sparse_mixture_experts_stable_b200.inputs import pages_layout

    return dict(
        x=cfg["x"].double().numpy(), w_router_de=cfg["w_router"].double().numpy().T.copy(),
        bias=cfg["router_bias"].double().numpy(),
        experts=dict(w1=pages_layout(cfg["w_gate"]), w3=pages_layout(cfg["w_up"]), w2=pages_layout(cfg["w_down"])),
        shared=dict(w1=pages_layout(cfg["s_gate"]), w3=pages_layout(cfg["s_up"]), w2=pages_layout(cfg["s_down"])),
    )


def time_oracle(cfg64, budget_s: float):
    """Pick a token sample that takes about budget_s, then time it.  Returns (tokens/s, S, seconds)."""
    t0 = time.perf_counter()
    oracle_step(cfg64, 16)
    per_tok = (time.perf_counter() - t0) / 16
    S = int(max(16, min(WORKLOAD["T"], budget_s / max(per_tok, 1e-6))))
    t0 = time.perf_counter()
    oracle_step(cfg64, S)
    dt = time.perf_counter() - t0
    return S / dt, S, dt


def run_reference(args, world, rank):
    from sparse_mixture_experts_stable_b200 import inputs as I

    if rank != 0:
        return
    cfg = I.full_layer_bf16(seed=0)
    cfg64 = oracle_inputs(cfg)
    budget = max(2.0, 150.0 / max(1, args.steps + args.warmup))
    t0 = time.perf_counter()
    oracle_step(cfg64, 16)
    per_tok = (time.perf_counter() - t0) / 16
    S = int(max(16, min(WORKLOAD["T"], budget / max(per_tok, 1e-6))))
    for _ in range(args.warmup):
        oracle_step(cfg64, S)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle_step(cfg64, S)
        times.append(time.perf_counter() - t0)
    total = sum(times)
    value = S * args.steps / total
    line = dict(impl="reference", metric=METRIC, value=value, unit=UNIT, n_gpus=args.gpus, steps=args.steps,
                warmup=args.warmup, ms_per_step=1e3 * total / args.steps, higher_is_better=True, scaling="weak",
                vs_baseline=None, dtype="f64", data="synthetic",
                config=dict(WORKLOAD, sample_tokens_per_step=S, l2="n/a (CPU)"),
                cpu_baseline=dict(value=value, unit=UNIT, cores=os.cpu_count(), kind="oracle",
                                  sample=f"first {S} tokens of the batch per step, capacity from the sample's T"),
                e2e=dict(value=value, unit=UNIT, h2d_bytes_per_step=0, d2h_bytes_per_step=0))
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------------------
def run_ours(args, world, rank, local):
    import sparse_mixture_experts_stable_b200 as moe
    from sparse_mixture_experts_stable_b200 import inputs as I
    from sparse_mixture_experts_stable_b200.layer import SwiGLUMoE

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    moe.lib()  # fail loudly if the CUDA library is missing
    cfg = I.full_layer_bf16(seed=rank_seed(rank), T=args.tokens, E=args.experts)
    T, H, E, F, k = cfg["T"], cfg["H"], cfg["E"], cfg["F"], cfg["k"]
    names = ("x", "w_router", "router_bias", "w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down")
    dv = {n: cfg[n].to(dev) for n in names}
    layer = SwiGLUMoE(T, H, E, F, k, cfg["capacity_factor"], F_shared=cfg["F_shared"], aux_coef=cfg["aux_coef"],
                      device=dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    ffn_ev = []

    side = torch.cuda.Stream(device=dev)
    ev_x, ev_shared = torch.cuda.Event(), torch.cuda.Event()

    def step(x, time_ffn=True, y_out=None):
        # shared expert on a second stream, overlapping the routing chain (as SwiGLUMoE.forward does)
        cur = torch.cuda.current_stream(dev)
        ev_x.record(cur)
        side.wait_event(ev_x)
        moe.moe_expert_ffn("swiglu", x.view(1, T, H), None, dv["s_gate"], w2=dv["s_down"], w3=dv["s_up"],
                           ybuf=layer.shared.view(1, T, H), dev_status=layer.status, workspace=layer.ws_shared,
                           stream=side)
        ev_shared.record(side)
        r = moe.moe_route(x, k, w_router=dv["w_router"], layout="ED", logit_bias=dv["router_bias"],
                          out=layer.route_out, dev_status=layer.status, workspace=layer.ws_route)
        d = moe.moe_dispatch(r["selected"], E, layer.C, x=x, out=layer.disp_out, dev_status=layer.status,
                             workspace=layer.ws_disp)
        if time_ffn:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(cur)
        moe.moe_expert_ffn("swiglu", d["xbuf"], d["used"], dv["w_gate"], w2=dv["w_down"], w3=dv["w_up"],
                           ybuf=layer.ybuf, dev_status=layer.status, workspace=layer.ws_ffn)
        if time_ffn:
            e1.record(cur)
            ffn_ev.append((e0, e1))
        cur.wait_event(ev_shared)
        y = moe.moe_combine(layer.ybuf, r["selected"], d["slot"], r["gates_f32"], base_kind="tensor",
                            base=layer.shared, y=layer.y if y_out is None else y_out, dev_status=layer.status)
        f, P, aux = moe.moe_aux_stats(r["counts"], r["prob_sum"], T, k, True, cfg["aux_coef"],
                                      out_dtype=torch.bfloat16)
        return y, aux

    for _ in range(args.warmup):
        flush_l2(flush)
        step(dv["x"])
    torch.cuda.synchronize()
    assert moe.moe_read_status(layer.status) == 0, "device status reported an error"
    ffn_ev.clear()
    # the routed FFN's own time for the roofline: the same launches, timed with events on their stream
    for _ in range(max(args.warmup, 5)):
        flush_l2(flush)
        step(dv["x"])
    torch.cuda.synchronize()
    ffn_ms = [a.elapsed_time(b) for a, b in ffn_ev]

    # ---- device-timed loop ----
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        for i in range(args.steps):
            flush_l2(flush)
            starts[i].record(stream)
            step(dv["x"], time_ffn=False)
            ends[i].record(stream)
        torch.cuda.synchronize()
    barrier(world)
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = max_over_ranks(sum(step_ms), world)
    value = job_throughput(T, args.steps, world, total_ms)

    # the same steps back to back with a warm L2 (no flush between them), beside the flushed figure
    n_warm = min(args.steps, 20)
    barrier(world)
    torch.cuda.synchronize()
    w0, w1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    w0.record(stream)
    for _ in range(n_warm):
        step(dv["x"], time_ffn=False)
    w1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    warm_ms = max_over_ranks(w0.elapsed_time(w1), world)
    warm = dict(value=job_throughput(T, n_warm, world, warm_ms), unit=UNIT, ms_per_step=warm_ms / n_warm,
                steps=n_warm, l2="warm: no flush between steps")

    if args.no_e2e:
        e2e_value = None
    else:
        e2e_value = run_e2e(args, world, cfg, dv, flush, stream)
    assert moe.moe_read_status(layer.status) == 0

    # ---- roofline of the dominant kernel (routed SwiGLU grouped GEMMs) ----
    kept = int(layer.disp_out["used"].sum().item())
    flops = 2.0 * kept * (2 * H * F) + 2.0 * kept * F * H
    ffn_avg_s = statistics.mean(ffn_ms) / 1e3
    pk = measured_peaks()
    achieved = flops / ffn_avg_s / 1e12
    alg_gate_up = E * 2 * F * H * 2 + kept * H * 2 + kept * F * 2  # weights, gathered rows, h written
    alg_down = E * H * F * 2 + kept * F * 2 + kept * H * 2
    if TRAFFIC_PER_ALG_BYTE is None:
        traffic, traffic_source = None, "not captured for the current kernels"
    else:
        traffic = TRAFFIC_PER_ALG_BYTE["gate_up"] * alg_gate_up + TRAFFIC_PER_ALG_BYTE["down"] * alg_down
        traffic_source = ("ncu DRAM bytes per algorithmic byte of each kernel on the T=8192, E=128 case, "
                          "times this workload's algorithmic bytes")
    # the routed FFN is timed inside ~1 ms steps, so the burst peak (a kernel timed alone) applies
    roof = dict(bound="tensor", kernel="routed expert FFN: tcw_kernel<SWIGLU> gate/up + tc_gemm_kernel<BF16> down",
                achieved=achieved, peak=pk["bf16"], unit="TFLOP/s", frac=achieved / pk["bf16"],
                traffic=traffic, traffic_source=traffic_source, bytes_alg=alg_gate_up + alg_down,
                peak_source=f"{pk['source']} bf16 burst (cuBLAS)", frac_of_sustained=achieved / pk["bf16_sustained"],
                flops_per_launch=flops, kept_rows=kept, avg_launch_ms=1e3 * ffn_avg_s)

    if rank != 0:
        return
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cfg64 = oracle_inputs(cfg)
        tps, S, dt = time_oracle(cfg64, args.cpu_seconds)
        cpu = dict(value=tps, unit=UNIT, cores=os.cpu_count(), kind="oracle",
                   sample=f"first {S} tokens of the batch ({dt:.1f} s), capacity from the sample's T")
    others = None
    if world == 1 and not args.no_other_workloads:
        others = run_other_workloads(min(args.steps, 20), max(3, min(args.warmup, 5)), flush, stream, dev)
    wl = dict(WORKLOAD, T=T, experts=E, capacity=layer.C)
    line = dict(
        metric=METRIC, value=value, unit=UNIT, n_gpus=world, steps=args.steps, warmup=args.warmup,
        ms_per_step=total_ms / args.steps, higher_is_better=True, scaling="weak", vs_baseline=None, dtype="bf16",
        data="synthetic",
        config=dict(wl, parallelism=f"replicas{world}", global_batch=T * world,
                    l2="flushed between steps (256 MiB write)", tokens_kept=kept),
        e2e=None if e2e_value is None else dict(value=e2e_value, unit=UNIT, h2d_bytes_per_step=T * H * 2,
                                                d2h_bytes_per_step=T * H * 2 + 8,
                                                api="moe_swiglu_layer_forward (C ABI) with pinned host x, y, aux"),
        gpu_launches=KERNELS_PER_STEP * args.steps,
        roofline=roof, cpu_baseline=cpu, clocks=clocks.summary(), warm_l2=warm, workloads=others,
    )
    print(json.dumps(line), flush=True)


def run_e2e(args, world, cfg, dv, flush, stream):
    """The same layer through the library's one-call entry point moe_swiglu_layer_forward with HOST
    buffers: every step hands the call a pinned host x and a pinned host y (and aux), and the library
    copies x in (one cudaMemcpyAsync on a copy-in stream) and y and the aux loss out (on a copy-out
    stream).  Two workspaces alternate, each with its own event, so one batch's copies overlap the
    neighbouring batches' kernels.  The timed region spans all steps, copies included."""
    from sparse_mixture_experts_stable_b200.layer import SwiGLULayer

    T, H = cfg["T"], cfg["H"]
    dev = dv["x"].device
    layer = SwiGLULayer(T, H, cfg["E"], cfg["F"], cfg["k"], cfg["capacity_factor"], dv["w_router"],
                        dv["router_bias"], dv["w_gate"], dv["w_up"], dv["w_down"], dv["s_gate"], dv["s_up"],
                        dv["s_down"], aux_coef=cfg["aux_coef"], n_workspaces=2, device=dev)
    x_host = [cfg["x"].pin_memory(), cfg["x"].clone().pin_memory()]
    y_host = [torch.empty(T, H, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    aux_host = [torch.empty(2, dtype=torch.float32).pin_memory() for _ in range(2)]
    side, cin, cout = (torch.cuda.Stream(device=dev) for _ in range(3))

    def run(n):
        for i in range(n):
            flush.zero_()  # inside the timed region: no launch cover here, the host's cost is part of e2e
            layer.forward(x_host[i % 2], y_host[i % 2], aux_host[i % 2], slot=i % 2, stream=stream,
                          side_stream=side, copy_in_stream=cin, copy_out_stream=cout)
        done = torch.cuda.Event()
        done.record(cout)
        stream.wait_event(done)

    run(max(2, min(args.warmup, 4)))
    torch.cuda.synchronize()
    n = args.steps
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    start.record(stream)
    run(n)
    end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    assert moe_status_ok(layer.status), "device status reported an error in the e2e run"
    e2e_ms = max_over_ranks(start.elapsed_time(end), world)
    return job_throughput(T, n, world, e2e_ms)


def moe_status_ok(status) -> bool:
    import sparse_mixture_experts_stable_b200 as moe

    return moe.moe_read_status(status) == 0


# ------------------------------------------------------------------------------------------------
# The other workloads of the pages, timed the same way (events around every step, L2 flush between
# steps) and reported in the "workloads" field.  Each names its dominant kernel call and roofline.
TF32_PEAK_SOURCE = "measured here: cuBLAS fp32 GEMM 8192^3 on TF32 tensor cores, best of 10 (burst)"
_TF32_PEAK = {}


def tf32_peak(pk, dev=None):
    """Dense tf32 tensor peak in TFLOP/s, measured on this GPU once per process.

    A library GEMM (torch.matmul, fp32 with TF32 allowed) of 8192^3, timed with
    CUDA events, best of 10 after 3 warm-ups: the same kind of calibration the
    measured bf16 peak is.
    """
    if "v" not in _TF32_PEAK:
        n = 8192
        a = torch.randn(n, n, device=dev or "cuda")
        b = torch.randn(n, n, device=dev or "cuda")
        prev = torch.backends.cuda.matmul.allow_tf32
        torch.backends.cuda.matmul.allow_tf32 = True
        try:
            for _ in range(3):
                torch.matmul(a, b)
            best = float("inf")
            for _ in range(10):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                torch.matmul(a, b)
                e1.record()
                e1.synchronize()
                best = min(best, e0.elapsed_time(e1) / 1e3)
        finally:
            torch.backends.cuda.matmul.allow_tf32 = prev
        _TF32_PEAK["v"] = 2.0 * n ** 3 / best / 1e12
        del a, b
    return _TF32_PEAK["v"]


# A spin of about a millisecond on the GPU after each L2 flush, outside the timed
# events: while it runs the host enqueues the step's launches, so the events
# measure device time and not the Python and ctypes overhead of issuing them.
LAUNCH_COVER_CYCLES = 2_000_000


def flush_l2(flush):
    flush.zero_()
    torch.cuda._sleep(LAUNCH_COVER_CYCLES)


def _time_steps(step, steps, warmup, flush, stream, inner=None):
    """Device time of `steps` calls of step() (ms each) and of the inner event pair step() records."""
    for _ in range(warmup):
        flush_l2(flush)
        step()
    torch.cuda.synchronize()
    if inner is not None:
        inner.clear()
    st = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    en = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for i in range(steps):
        flush_l2(flush)
        st[i].record(stream)
        step()
        en[i].record(stream)
    torch.cuda.synchronize()
    step_ms = [a.elapsed_time(b) for a, b in zip(st, en)]
    inner_ms = [a.elapsed_time(b) for a, b in inner] if inner is not None else []
    return step_ms, inner_ms


def run_other_workloads(steps, warmup, flush, stream, dev, only=None, layer_sizes=None):
    import sparse_mixture_experts_stable_b200 as moe
    from sparse_mixture_experts_stable_b200 import binding as B
    from sparse_mixture_experts_stable_b200 import inputs as I

    pk = measured_peaks()
    out = {}

    def want(name):  # the tiny fp32 block also times its training-step line
        return only is None or name == only or (name == "tiny_gelu_fp32" and only == "tiny_gelu_fp32_train")

    def events(lst):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        lst.append((e0, e1))
        return e0, e1

    if want("router_bf16"):
        # router-only with load statistics (router GEMM + softmax/top-k/gates + statistics)
        c = I.router_bf16(seed=0)
        T, D, E, k = c["T"], c["D"], c["E"], c["k"]
        x, w = c["x"].to(dev), c["w_router"].to(dev)
        ro = dict(selected=torch.empty(T, k, dtype=torch.int64, device=dev),
                  gates=torch.empty(T, k, dtype=torch.bfloat16, device=dev),
                  gates_f32=torch.empty(T, k, dtype=torch.float32, device=dev),
                  counts=torch.empty(E, dtype=torch.int32, device=dev), prob_sum=torch.empty(E, device=dev))
        ws = torch.empty(B.moe_route_workspace_size(T, D, E, B.MOE_BF16, True, "ED"), dtype=torch.uint8, device=dev)
        inner = []

        def step_router():
            e0, e1 = events(inner)
            e0.record(stream)
            moe.moe_route(x, k, w_router=w, out=ro, workspace=ws)
            e1.record(stream)
            moe.moe_aux_stats(ro["counts"], ro["prob_sum"], T, k, out_dtype=torch.bfloat16)

        sm, im = _time_steps(step_router, steps, warmup, flush, stream, inner)
        r_s = statistics.mean(im) / 1e3
        bytes_alg = T * D * 2 + E * D * 2 + T * k * (8 + 2 + 4) + E * 8
        flops = 2.0 * T * D * E
        out["router_bf16"] = dict(
            value=T * steps / (sum(sm) / 1e3), unit=UNIT, ms_per_step=sum(sm) / steps, steps=steps,
            config=dict(T=T, D=D, E=E, k=k),
            roofline=dict(bound="hbm/tensor ridge", kernel="moe_route: route_fused_kernel (scores on tcgen05, softmax, top-k, gates) + route_reduce_kernel",
                          achieved=bytes_alg / r_s / 1e9, peak=pk["hbm"], unit="GB/s", frac=bytes_alg / r_s / 1e9 / pk["hbm"],
                          tflops=flops / r_s / 1e12, frac_tensor=flops / r_s / 1e12 / pk["bf16"], traffic=None,
                          bytes_per_launch=bytes_alg, flops_per_launch=flops, avg_launch_ms=1e3 * r_s))
        del x, w, ws, ro

    if want("dispatch_top1_bf16"):
        # capacity-limited top-1 dispatch/combine with linear experts
        c = I.dispatch_top1_bf16(seed=0)
        T, D, E = c["T"], c["D"], c["E"]
        C = moe.moe_capacity(T, 1, E, c["capacity_factor"])
        idx = c["expert_idx"].view(T, 1).to(dev)
        x, w, gate = c["x"].to(dev), c["w"].to(dev), c["gate"].view(T, 1).to(dev)
        do = dict(slot=torch.empty(T, 1, dtype=torch.int64, device=dev), kept=torch.empty(T, 1, dtype=torch.uint8, device=dev),
                  used=torch.empty(E, dtype=torch.int32, device=dev), overflow=torch.empty(E, dtype=torch.int32, device=dev),
                  drops=torch.empty(T, dtype=torch.int32, device=dev),
                  token_of_slot=torch.empty(E, C, dtype=torch.int32, device=dev),
                  xbuf=torch.empty(E, C, D, dtype=torch.bfloat16, device=dev))
        ybuf = torch.empty(E, C, D, dtype=torch.bfloat16, device=dev)
        y = torch.empty(T, D, dtype=torch.bfloat16, device=dev)
        wsd = torch.empty(B.moe_dispatch_workspace_size(T, 1, E), dtype=torch.uint8, device=dev)
        inner = []

        def step_top1():
            moe.moe_dispatch(idx, E, C, x=x, out=do, workspace=wsd)
            e0, e1 = events(inner)
            e0.record(stream)
            moe.moe_expert_ffn("linear", do["xbuf"], do["used"], w, ybuf=ybuf)
            e1.record(stream)
            moe.moe_combine(ybuf, idx, do["slot"], gate, y=y)

        sm, im = _time_steps(step_top1, steps, warmup, flush, stream, inner)
        used = do["used"].cpu()
        kept = int(used.sum())
        active = int((used > 0).sum())
        f_s = statistics.mean(im) / 1e3
        bytes_alg = kept * D * 2 + active * D * D * 2 + kept * D * 2
        out["dispatch_top1_bf16"] = dict(
            value=T * steps / (sum(sm) / 1e3), unit=UNIT, ms_per_step=sum(sm) / steps, steps=steps,
            config=dict(T=T, D=D, E=E, k=1, capacity=C, kept=kept),
            roofline=dict(bound="hbm", kernel="tcx_kernel: linear experts (moe_expert_ffn)", achieved=bytes_alg / f_s / 1e9,
                          peak=pk["hbm"], unit="GB/s", frac=bytes_alg / f_s / 1e9 / pk["hbm"], traffic=None,
                          tflops=2.0 * kept * D * D / f_s / 1e12, bytes_per_launch=bytes_alg, avg_launch_ms=1e3 * f_s))
        del x, w, gate, do, ybuf, y

    if want("tiny_gelu_fp32"):
        # tiny top-2 GELU layer, fp32
        c = I.tiny_gelu_fp32(seed=0)
        T, D, E, F, k = c["T"], c["D"], c["E"], c["F"], c["k"]
        C = moe.moe_capacity(T, k, E, c["capacity_factor"])
        dv = {n: c[n].to(dev) for n in ("x", "w_router", "w1", "b1", "w2", "b2")}
        inner = []

        def step_tiny():
            r = moe.moe_route(dv["x"], k, w_router=dv["w_router"])
            d = moe.moe_dispatch(r["selected"], E, C, x=dv["x"])
            e0, e1 = events(inner)
            e0.record(stream)
            yb = moe.moe_expert_ffn("gelu_mlp", d["xbuf"], d["used"], dv["w1"], b1=dv["b1"], w2=dv["w2"], b2=dv["b2"])
            e1.record(stream)
            moe.moe_combine(yb, r["selected"], d["slot"], r["gates_f32"], base_kind="input", base=dv["x"])
            moe.moe_aux_stats(r["counts"], r["prob_sum"], T, k, True, 0.01)

        sm, im = _time_steps(step_tiny, steps, warmup, flush, stream, inner)
        f_s = statistics.mean(im) / 1e3
        flops = 2.0 * T * k * (D * F + F * D)
        out["tiny_gelu_fp32"] = dict(
            value=T * steps / (sum(sm) / 1e3), unit=UNIT, ms_per_step=sum(sm) / steps, steps=steps,
            config=dict(T=T, D=D, E=E, F=F, k=k, capacity=C),
            roofline=dict(bound="tensor", kernel="tf32x3_kernel: GELU MLP experts (moe_expert_ffn, split-tf32)",
                          achieved=3 * flops / f_s / 1e12, peak=tf32_peak(pk), unit="TFLOP/s",
                          frac=3 * flops / f_s / 1e12 / tf32_peak(pk), traffic=None, avg_launch_ms=1e3 * f_s,
                          fp32_tflops=flops / f_s / 1e12, peak_source=TF32_PEAK_SOURCE,
                          note="three tf32 MMAs per fp32 product; launch-latency bound at this size"))

        # the same layer's training step: forward, GELU-expert backward, router backward (fp32)
        dyg = torch.randn(T, D, generator=torch.Generator().manual_seed(2)).to(dev)
        wsg = torch.empty(B.moe_backward_gelu_workspace_size(E, C, D, F, D), dtype=torch.uint8, device=dev)
        inner = []
        kept_box = {}

        def step_tiny_train():
            r = moe.moe_route(dv["x"], k, w_router=dv["w_router"], want_logits=True)
            d = moe.moe_dispatch(r["selected"], E, C, x=dv["x"])
            yb = moe.moe_expert_ffn("gelu_mlp", d["xbuf"], d["used"], dv["w1"], b1=dv["b1"], w2=dv["w2"], b2=dv["b2"])
            moe.moe_combine(yb, r["selected"], d["slot"], r["gates_f32"], base_kind="input", base=dv["x"])
            e0, e1 = events(inner)
            e0.record(stream)
            g = moe.moe_backward_gelu(dyg, r["logits"], r["selected"], r["gates_f32"], d["slot"], d["used"], d["xbuf"],
                                      yb, dv["w1"], dv["b1"], dv["w2"], C, use_residual=True, workspace=wsg)
            e1.record(stream)
            moe.moe_router_backward(dv["x"], dv["w_router"], g[5])
            kept_box["used"] = d["used"]

        sm, im = _time_steps(step_tiny_train, steps, warmup, flush, stream, inner)
        kept = int(kept_box["used"].sum())
        b_s = statistics.mean(im) / 1e3
        flops_b = 2.0 * kept * D * F * 5  # recomputed z, dh, dW2, dW1, dx: 2*kept*D*F each
        out["tiny_gelu_fp32_train"] = dict(
            value=T * steps / (sum(sm) / 1e3), unit=UNIT, ms_per_step=sum(sm) / steps, steps=steps,
            config=dict(T=T, D=D, E=E, F=F, k=k, capacity=C, kept=kept,
                        step="forward + moe_backward_gelu + moe_router_backward"),
            roofline=dict(bound="tensor", kernel="moe_backward_gelu (tf32x3_kernel x5, elementwise, sums, combine)",
                          achieved=3 * flops_b / b_s / 1e12, peak=tf32_peak(pk), unit="TFLOP/s",
                          frac=3 * flops_b / b_s / 1e12 / tf32_peak(pk), traffic=None, avg_launch_ms=1e3 * b_s,
                          fp32_tflops=flops_b / b_s / 1e12, peak_source=TF32_PEAK_SOURCE,
                          note="launch-latency bound at this size"))
        del dv, dyg, wsg

    if want("fwd_bwd_fp32"):
        # forward + backward, fp32, linear experts with residual
        c = I.fwd_bwd_fp32(seed=0)
        T, D, E, k = c["T"], c["D"], c["E"], c["k"]
        C = moe.moe_capacity(T, k, E, c["capacity_factor"])
        lg, x, w, dy = (c[n].to(dev) for n in ("logits", "x", "w", "dy"))
        inner = []
        wsb = torch.empty(B.moe_backward_workspace_size(E, C, D, D), dtype=torch.uint8, device=dev)
        state = {}

        def step_fb():
            r = moe.moe_route(lg, k)
            d = moe.moe_dispatch(r["selected"], E, C, x=x)
            yb = moe.moe_expert_ffn("linear", d["xbuf"], d["used"], w)
            moe.moe_combine(yb, r["selected"], d["slot"], r["gates_f32"], base_kind="input", base=x)
            e0, e1 = events(inner)
            e0.record(stream)
            moe.moe_backward(dy, x, lg, r["selected"], r["gates_f32"], d["slot"], d["used"], d["token_of_slot"],
                             d["xbuf"], yb, w, C, workspace=wsb)
            e1.record(stream)
            state["used"] = d["used"]

        sm, im = _time_steps(step_fb, steps, warmup, flush, stream, inner)
        kept = int(state["used"].sum())
        b_s = statistics.mean(im) / 1e3
        flops_b = 2.0 * kept * D * D * 2 + 2.0 * kept * D
        out["fwd_bwd_fp32"] = dict(
            value=T * steps / (sum(sm) / 1e3), unit=UNIT, ms_per_step=sum(sm) / steps, steps=steps,
            config=dict(T=T, D=D, E=E, k=k, capacity=C, kept=kept),
            roofline=dict(bound="tensor", kernel="moe_backward (tf32x3_kernel dW + dx, dgate/dlogits, combine)",
                          achieved=3 * flops_b / b_s / 1e12, peak=tf32_peak(pk), unit="TFLOP/s",
                          frac=3 * flops_b / b_s / 1e12 / tf32_peak(pk), traffic=None, avg_launch_ms=1e3 * b_s,
                          fp32_tflops=flops_b / b_s / 1e12, peak_source=TF32_PEAK_SOURCE))
        del lg, x, w, dy, wsb, state

    if want("full_layer_bf16_ep4_one_device"):
        # expert parallelism, 4 ranks emulated on this GPU: the full-layer batch split over the ranks, every rank's
        # rows written into and read from the other ranks' buffers through the peer-pointer tables
        from sparse_mixture_experts_stable_b200 import ep
        c = I.full_layer_bf16(seed=0, **(layer_sizes or {}))
        T, H, E, F, k = c["T"], c["H"], c["E"], c["F"], c["k"]
        R, epr = 4, c["E"] // 4
        C = moe.moe_capacity(T, k, E, c["capacity_factor"])
        dv = {n: c[n].to(dev) for n in ("x", "w_router", "router_bias", "w_gate", "w_up", "w_down")}
        xs = [t.contiguous() for t in torch.chunk(dv["x"], R)]
        wr = [{"w1": dv["w_gate"][q * epr:(q + 1) * epr], "w3": dv["w_up"][q * epr:(q + 1) * epr],
               "w2": dv["w_down"][q * epr:(q + 1) * epr]} for q in range(R)]
        xbufs = [torch.empty(epr, C, H, dtype=torch.bfloat16, device=dev) for _ in range(R)]
        ybufs = [torch.empty(epr, C, H, dtype=torch.bfloat16, device=dev) for _ in range(R)]
        ys = [torch.empty_like(t) for t in xs]
        tb = ep.token_bases([t.shape[0] for t in xs])
        wsd = torch.empty(B.moe_dispatch_workspace_size(T // R, k, E), dtype=torch.uint8, device=dev)
        inner_d, inner_c = [], []
        kept_box = {}

        def step_ep():
            routes = [moe.moe_route(xs[q], k, w_router=dv["w_router"], logit_bias=dv["router_bias"]) for q in range(R)]
            counts_all = torch.stack([r["counts"] for r in routes])
            plans = [moe.moe_ep_plan(counts_all, q, C) for q in range(R)]
            e0, e1 = events(inner_d)
            e0.record(stream)
            disp = [moe.moe_ep_dispatch(routes[q]["selected"], E, C, plans[q]["rank_base"], tb[q], xs[q], xbufs,
                                        workspace=wsd) for q in range(R)]
            e1.record(stream)
            for q in range(R):
                moe.moe_expert_ffn("swiglu", xbufs[q], plans[q]["used"][q * epr:(q + 1) * epr], wr[q]["w1"],
                                   w2=wr[q]["w2"], w3=wr[q]["w3"], ybuf=ybufs[q])
            e0, e1 = events(inner_c)
            e0.record(stream)
            for q in range(R):
                moe.moe_ep_combine(ybufs, routes[q]["selected"], disp[q]["slot"], routes[q]["gates_f32"], E, C, H,
                                   torch.bfloat16, base_kind="input", base=xs[q], y=ys[q])
            e1.record(stream)
            kept_box["used"] = plans[0]["used"]

        sm, _ = _time_steps(step_ep, steps, warmup, flush, stream)
        kept = int(kept_box["used"].sum())
        d_s = statistics.mean(a.elapsed_time(b) for a, b in inner_d[-steps:]) / 1e3
        c_s = statistics.mean(a.elapsed_time(b) for a, b in inner_c[-steps:]) / 1e3
        moved = 2 * kept * H * 2  # kept rows out to their owner ranks and back (bf16)
        bytes_alg = (T * H * 2 + kept * H * 2) + (kept * H * 2 + 2 * T * H * 2)  # dispatch + combine (x and y base/out)
        out["full_layer_bf16_ep4_one_device"] = dict(
            value=T * steps / (sum(sm) / 1e3), unit=UNIT, ms_per_step=sum(sm) / steps, steps=steps,
            config=dict(T=T, H=H, E=E, F=F, k=k, capacity=C, kept=kept, ranks=R, experts_per_rank=epr,
                        step="4 ranks on one GPU: route, counts, moe_ep_plan, moe_ep_dispatch, experts, moe_ep_combine",
                        shared_experts=0),
            roofline=dict(bound="hbm", kernel="moe_ep_dispatch gather + moe_ep_combine (peer-pointer row exchange)",
                          achieved=bytes_alg / (d_s + c_s) / 1e9, peak=pk["hbm"], unit="GB/s",
                          frac=bytes_alg / (d_s + c_s) / 1e9 / pk["hbm"], traffic=None,
                          dispatch_ms=1e3 * d_s, combine_ms=1e3 * c_s, bytes_per_step=bytes_alg,
                          exchanged_bytes=moved, payload_bytes_no_drops=ep.payload_bytes(T, H, k, 2),
                          note="on one GPU the peer buffers are local HBM; across GPUs the exchanged bytes cross NVLink"))
        del dv, xs, wr, xbufs, ybufs, ys, wsd

    if want("full_layer_bf16_train"):
        # training step of the full layer: forward, SwiGLU-expert backward and router backward (bf16)
        from sparse_mixture_experts_stable_b200.layer import SwiGLUMoE
        c = I.full_layer_bf16(seed=0, **(layer_sizes or {}))
        T, H, E, F, k = c["T"], c["H"], c["E"], c["F"], c["k"]
        dv = {n: c[n].to(dev) for n in ("x", "w_router", "router_bias", "w_gate", "w_up", "w_down")}
        dyt = (torch.randn(T, H, generator=torch.Generator().manual_seed(1)) * 0.1).to(torch.bfloat16).to(dev)
        layer = SwiGLUMoE(T, H, E, F, k, c["capacity_factor"], F_shared=0, aux_coef=c["aux_coef"], device=dev,
                          save_for_backward=True)
        wsbs = torch.empty(B.moe_backward_swiglu_workspace_size(E, layer.C, H, F), dtype=torch.uint8, device=dev)
        kept_box = {}
        inner = []

        def step_train():
            o = layer.forward(dv["x"], dv["w_router"], dv["router_bias"], dv["w_gate"], dv["w_up"], dv["w_down"])
            lg_t = layer.route_out.get("logits")
            e0, e1 = events(inner)
            e0.record(stream)
            dxe, dwg, dwu, dwd, dl, dg = moe.moe_backward_swiglu(
                dyt, lg_t, o["selected"], o["gates_f32"], o["slot"], o["used"], o["xbuf"], layer.ybuf, dv["w_gate"],
                dv["w_up"], dv["w_down"], layer.C, aux_coef=c["aux_coef"], counts=o["counts"], workspace=wsbs,
                saved_ab=layer.saved_ab)
            e1.record(stream)
            moe.moe_router_backward(dv["x"], dv["w_router"], dl)
            kept_box["used"] = o["used"]

        layer.route_out["logits"] = torch.empty(T, E, dtype=torch.float32, device=dev)
        sm, im = _time_steps(step_train, max(steps // 5, 3), warmup, flush, stream, inner)
        kept = int(kept_box["used"].sum())
        bw_s = statistics.mean(im) / 1e3
        flops_bw = 16.0 * kept * H * F  # recomputed gate/up (4), dh (2), three weight gradients (6), dx (4): x kept*H*F
        out["full_layer_bf16_train"] = dict(
            value=T * len(sm) / (sum(sm) / 1e3), unit=UNIT, ms_per_step=sum(sm) / len(sm), steps=len(sm),
            config=dict(T=T, H=H, E=E, F=F, k=k, capacity=layer.C, kept=kept, shared_experts=0,
                        step="forward (moe_expert_ffn_save) + moe_backward_swiglu + moe_router_backward"),
            roofline=dict(bound="tensor", kernel="moe_backward_swiglu (tcgen05 GEMMs + transposes)",
                          achieved=flops_bw / bw_s / 1e12, peak=pk["bf16"], unit="TFLOP/s",
                          frac=flops_bw / bw_s / 1e12 / pk["bf16"], traffic=None, avg_launch_ms=1e3 * bw_s,
                          peak_source=f"{pk['source']} bf16 burst (cuBLAS); the backward runs ~2 ms"))

    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--tokens", type=int, default=WORKLOAD["T"], help="tokens per rank (smaller for profiling)")
    ap.add_argument("--experts", type=int, default=WORKLOAD["experts"], help="routed experts (smaller for profiling)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-other-workloads", action="store_true",
                    help="skip timing the router-only, top-1, tiny fp32 and fp32 fwd+bwd workloads")
    ap.add_argument("--workload", default=None,
                    help="time only this secondary workload (e.g. full_layer_bf16_train) and print its line; "
                         "for profiling captures")
    args = ap.parse_args()
    world, rank, local = dist_setup()
    try:
        if args.workload is not None:
            import sparse_mixture_experts_stable_b200 as moe

            dev = torch.device("cuda", local)
            torch.cuda.set_device(dev)
            moe.lib()
            flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
            sizes = None
            if args.tokens != WORKLOAD["T"] or args.experts != WORKLOAD["experts"]:
                sizes = dict(T=args.tokens, E=args.experts)  # smaller full-layer shapes for profiling captures
            out = run_other_workloads(args.steps, args.warmup, flush, torch.cuda.current_stream(dev), dev,
                                      only=args.workload, layer_sizes=sizes)
            if args.workload not in out:
                raise SystemExit(f"unknown workload {args.workload}; known: {sorted(out)}")
            print(json.dumps(dict(workload=args.workload, **out[args.workload])), flush=True)
        elif args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
