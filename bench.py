"""Throughput benchmark of the ring attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--schedule S] [--impl reference]

One step = one ``ra_ring_fwd`` call (the whole hot path: TMA tile staging, QK^T and PV on the
tensor cores, causal masks from global positions, online softmax, partial (O, LSE) results and
their LSE merges, the P-step ring) over the workload's synthetic inputs, resident in HBM.
Timing: CUDA events on the launching stream around every step, L2 flushed (a 256 MiB write)
between steps outside the events, W untimed warm-up steps, max over ranks.  N > 1 runs N
independent replicas (one per GPU, weak scaling; the method needs no collective on one GPU).

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU fp64 oracle on the host
cores instead (each step a bounded sample of query rows of the same workload).
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention fwd TFLOP/s (bf16, ring P shards) and % of B200 dense BF16 peak"
METRIC_BWD = ("attention bwd TFLOP/s (weights recomputed from the saved LSE; bf16 inputs on the tensor cores) "
              "and % of B200 dense BF16 peak")
SPEC_BF16_TFLOPS = 2250.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


FMHA_SOURCES = ("ra_common.cuh", "ra_fmha_sm100.cuh", "ra_fmha_launch.cu", "ra_attn.cu")


def kernel_sources_hash() -> str:
    """sha256 over the attention kernel's sources without blank and whole-line comment lines
    (identifies the kernel code a capture is of; editing a comment does not invalidate it)."""
    import hashlib

    h = hashlib.sha256()
    for name in FMHA_SOURCES:
        with open(os.path.join(ROOT, "ring_blockwise_softmax_b200", "csrc", name), "rb") as fh:
            code = [ln.strip() for ln in fh.read().splitlines()]
        code = [ln for ln in code if ln and not ln.startswith(b"//")]
        h.update(name.encode() + b"\0" + b"\n".join(code))
    return h.hexdigest()


# Exponential throughput of the MUFU unit: 16 ex2 per clock per SM (4 per sub-partition; a
# micro-benchmark of the softmax's exponential loop on this GPU reaches ~3.8 per sub-partition).
MUFU_EX2_PER_CLK_PER_SM = 16
B200_SMS = 148


def mufu_roofline(w, ms: float, world: int, clocks: dict):
    """Second roofline for head dims <= 64, where the softmax exponentials (one per visible
    query-key pair: algorithmic FLOPs / (4 d)) bind before the tensor core does.  Peak at the
    median SM clock sampled during the timed region (the maximum clock when none was sampled)."""
    if w.dtype != "bf16":
        return None
    mhz = clocks.get("sm_mhz") or clocks.get("sm_max_mhz") or 1965.0
    exps = w.flops() / (4.0 * w.d)
    achieved = world * exps / (ms * 1e-3) / 1e12
    peak = world * MUFU_EX2_PER_CLK_PER_SM * B200_SMS * mhz * 1e6 / 1e12
    return {"bound": "mufu", "achieved": achieved, "peak": peak, "unit": "Tex2/s", "frac": achieved / peak,
            "note": "one exponential per visible (query, key) pair; peak = 16 ex2/clk/SM x 148 SMs x sampled SM clock"}


BWD_NOTE = ("algorithmic FLOPs 10*d per visible query-key pair (S, dP, dV, dK, dQ products of 2*d each) / the "
            "step's 2 serialised launches; the kernels execute 14*d (S and dP are recomputed by both the dQ and "
            "the dK/dV instance)")


def fp32_roofline(achieved: float, clocks: dict):
    """The fp32-input backward kernels run their products as fp32 FMAs on the SIMT pipes: peak 128 FMA per
    clock per SM (256 flops) x 148 SMs at the sampled SM clock."""
    mhz = clocks.get("sm_mhz") or clocks.get("sm_max_mhz") or 1965.0
    peak = 256 * B200_SMS * mhz * 1e6 / 1e12
    return {"bound": "alu", "kernel": "attn_bwd_dq + attn_bwd_dkv", "achieved": achieved, "peak": peak,
            "unit": "TFLOP/s", "frac": achieved / peak,
            "note": "10*d algorithmic flops per visible pair; peak = 128 fp32 FMA/clk/SM x 2 x 148 SMs x SM clock"}


def recorded_traffic(workload: str, schedule: str):
    """DRAM bytes per launch of the attention kernel from profiles/fmha_traffic.json, if that
    capture was taken of the current kernel sources on this workload and schedule; else None."""
    p = os.path.join(ROOT, "profiles", "fmha_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    if rec.get("kernel_sources_sha256") != kernel_sources_hash():
        return None
    for e in rec.get("captures", []):
        if e.get("workload") == workload and e.get("schedule") == schedule:
            return e.get("dram_bytes_per_launch")
    return None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------------------------
# clocks sampled during the timed region (NVML reads only; no setting is changed)
# ---------------------------------------------------------------------------------------------
class ClockSampler:
    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, device_index: int, period_s: float = 0.02):
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception as e:  # no NVML: report that instead of clocks
            self.error = repr(e)
        self.period = period_s
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        n = self._nvml
        while not self._stop.is_set():
            try:
                self.samples.append(n.nvmlDeviceGetClockInfo(self._h, n.NVML_CLOCK_SM))
                mask = n.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for name, bit in self.REASONS.items():
                    if mask & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._ok:
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._ok:
            self._t.join()

    def summary(self):
        if not self._ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": getattr(self, "error", "")}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------------------------------------
# distributed plumbing (replicas; barrier + max over ranks only)
# ---------------------------------------------------------------------------------------------
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world: int, backend: str):
    import datetime

    import torch.distributed as dist

    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Max of a scalar over all ranks (a barrier + all-reduce MAX); x itself when world == 1."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


# ---------------------------------------------------------------------------------------------
# the reference arm and the CPU baseline: the fp64 oracle on a bounded sample of rows
# ---------------------------------------------------------------------------------------------
def _blas_threads():
    try:
        from threadpoolctl import threadpool_info

        return max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        return os.cpu_count() or 1


class OracleSampler:
    """Evaluates the oracle on successive chunks of query rows of the workload (cycling heads)."""

    def __init__(self, w, rows_per_step: int):
        import numpy as np

        from ring_blockwise_softmax_b200 import inputs as I

        self.np = np
        self.w = w
        self.rows = rows_per_step
        # Host copies of the inputs (the workload's dtype); the oracle widens the exact bf16/fp32
        # values of one head at a time to fp64.
        self.q, self.k, self.v = I.make_qkv(w)
        self.cursor = 0
        self.flops = 0.0
        self.rng = np.random.default_rng(w.seed)

    def step(self):
        import oracle

        np = self.np
        w = self.w
        n_heads = w.B * w.H
        head = self.cursor % n_heads
        self.cursor += 1
        b, h = divmod(head, w.H)
        # query rows drawn uniformly (seeded), so causal rows see N/2 keys on average
        rows = np.sort(self.rng.choice(w.N, size=min(self.rows, w.N), replace=False))
        pos = np.arange(w.N)
        hk = oracle.kv_head(h, w.H, self.k.shape[1])  # K/V head (grouped-query K/V)
        k = self.k[b, hk].float().numpy().astype(np.float64)
        v = self.v[b, hk].float().numpy().astype(np.float64)
        q = self.q[b, h].float().numpy()[rows].astype(np.float64)
        oracle.attention_rows(q, k, v, w.scale, rows, pos, w.causal, window=w.window)
        if w.window is not None:
            keys = np.minimum(rows + 1, w.window).sum()
        elif w.causal:
            keys = (rows + 1).sum()
        else:
            keys = self.rows * w.N
        self.flops += 4.0 * w.d * float(keys)


def cpu_baseline(w, budget_s: float = 12.0, rows_per_step: int = 64, single_s: float = 3.0):
    """The oracle on the host's cores (BLAS threads), then the same on one thread for single_s."""
    s = OracleSampler(w, rows_per_step)
    t0 = time.perf_counter()
    n = 0
    while time.perf_counter() - t0 < budget_s:
        s.step()
        n += 1
    dt = time.perf_counter() - t0
    out = {"value": s.flops / dt / 1e12, "unit": "TFLOP/s", "cores": _blas_threads(), "kind": "oracle",
           "sample": f"{n * rows_per_step} query rows ({rows_per_step} seeded uniform rows per chunk, cycling the "
                     f"{w.B * w.H} heads) of the workload, fp64 numpy oracle, {dt:.1f} s"}
    if single_s > 0:
        from threadpoolctl import threadpool_limits

        with threadpool_limits(limits=1):
            s.flops = 0.0
            n1 = 0
            t1 = time.perf_counter()
            while time.perf_counter() - t1 < single_s:
                s.step()
                n1 += 1
            dt1 = time.perf_counter() - t1
        out["single_thread"] = {"value": s.flops / dt1 / 1e12, "unit": "TFLOP/s", "cores": 1,
                                "sample": f"{n1 * rows_per_step} query rows, same sampling, {dt1:.1f} s"}
    return out


def run_reference(args, w):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    s = OracleSampler(w, args.ref_rows)
    for _ in range(args.warmup):
        s.step()
    s.flops = 0.0
    t0 = time.perf_counter()
    for _ in range(args.steps):
        s.step()
    dt = time.perf_counter() - t0
    value = s.flops / dt / 1e12
    cores = _blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(w, args),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"each step: {args.ref_rows} seeded uniform query rows of one head (cycling heads) "
                                   f"of the workload"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------------------------
# the GPU arm
# ---------------------------------------------------------------------------------------------
def config_dict(w, args):
    name = w.name if w.H_kv is None else f"{w.name}, grouped-query K/V with {w.H_kv} heads"
    if w.window is not None:
        name += f", sliding window of {w.window} positions"
    from ring_blockwise_softmax_b200 import inputs as I

    if w.N != I.WORKLOADS[w.cfg].N:
        name += f", sequence length reduced to {w.N}"
    if w.layout != I.WORKLOADS[w.cfg].layout:
        name += f", {w.layout} shards instead"
    return {"workload": f"cfg{w.cfg}: {name}", "B": w.B, "H": w.H, "H_kv": w.H_kv or w.H, "N": w.N, "d": w.d,
            "causal": w.causal, "window": w.window,
            "P": w.P, "layout": w.layout, "schedule": args.schedule, "striped_walk": args.striped_walk,
            "l2": "flushed between timed steps (256 MiB write outside the events)",
            "parallelism": f"replicas x{args.gpus}" if args.gpus > 1 else "single GPU"}


def time_forward(w, args, dev, stream, flush, world, steps: int, warmup: int):
    """Time `steps` ring-forward steps of workload w (inputs resident in HBM, L2 flushed between
    steps outside the events).  Returns (mean ms over ranks' max, per-step ms, clocks, launches per
    step, device tensors)."""
    import torch

    from ring_blockwise_softmax_b200 import inputs as I
    from ring_blockwise_softmax_b200 import ra_attn as ra

    q_h, k_h, v_h = I.make_qkv(w)
    q, k, v = (t.to(dev) for t in (q_h, k_h, v_h))
    assert q.stride() == q_h.stride()
    B, H, N, d = q.shape
    o = torch.empty((B, H, N, d), dtype=q.dtype, device=dev)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    ws_bytes = ra.ring_workspace_size(q, w.P, args.schedule)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev) if ws_bytes else None

    def step():
        ra.ring_fwd(q, k, v, w.P, w.layout, w.causal, o, lse, 0.0, args.schedule, [stream], ws, w.window or 0)

    launches = 1 if (args.schedule == "fused" or w.P == 1) else w.P
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    assert ra.get_device_status(stream) == ra.RA_OK
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clocks:
        for i in range(steps):
            flush.zero_()
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        torch.cuda.synchronize()
    barrier(world)
    per_step = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    ms = max_over_ranks(sum(per_step) / len(per_step), world, dev)
    status = ra.get_device_status(stream)
    bufs = {"host": (q_h, k_h, v_h), "dev": (q, k, v), "o": o, "lse": lse, "ws": ws, "step": step}
    return ms, per_step, clocks.summary(), launches, status, bufs


def forward_roofline(w, ms: float, world: int, peak: float, peak_kind: str, launches: int, traffic):
    value = world * w.flops() / (ms * 1e-3) / 1e12
    return value, {
        "bound": "tensor", "kernel": "fmha_fwd_sm100", "achieved": value / world, "peak": peak,
        "peak_kind": f"{peak_kind} bf16 burst", "unit": "TFLOP/s", "frac": (value / world) / peak,
        "traffic": traffic,
        "note": ("algorithmic FLOPs (4*d per visible query-key pair: 4*B*H*N^2*d, halved when causal; "
                 "sum_i min(i+1, w) pairs per head with a sliding window w) / summed duration of the "
                 f"step's {launches} serialised launches (CUDA events on the launch stream)")}


def traffic_key(w, backward: bool = False, walk: str = "shard") -> str:
    """Key of a workload's recorded DRAM traffic: the configuration plus every override that
    changes what the attention kernel reads (reduced lengths are never recorded)."""
    from ring_blockwise_softmax_b200 import inputs as I

    key = f"cfg{w.cfg}" + ("" if w.H_kv is None else f"-kv{w.H_kv}") + ("" if w.window is None else f"-w{w.window}")
    if w.layout != I.WORKLOADS[w.cfg].layout:
        key += f"-{w.layout}"
    if w.N != I.WORKLOADS[w.cfg].N:
        key += f"-n{w.N}"
    if walk != "shard" and w.layout == "striped" and w.d > 64:
        key += f"-{walk}walk"
    return key + ("-bwd" if backward else "")


def run_gpu(args, w):
    import torch

    from ring_blockwise_softmax_b200 import inputs as I
    from ring_blockwise_softmax_b200 import ra_attn as ra

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist(world, "nccl")
    peaks, peak_kind = load_peaks()
    peak = peaks["bf16_tflops"]
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    ms, per_step_ms, clk, launches_per_step, status, bufs = time_forward(
        w, args, dev, stream, flush, world, args.steps, args.warmup)
    q_h, k_h, v_h = bufs["host"]
    q, k, v = bufs["dev"]
    o, lse, ws = bufs["o"], bufs["lse"], bufs["ws"]
    flops = w.flops()
    if args.backward:
        # Backward of the ring forward = backward on the full tensors (same function of global
        # positions): ra_attn_bwd from the forward's saved O and LSE, dO drawn like the inputs.
        bufs["step"]()
        do_ = I.draw(tuple(q.shape), w.seed, 3, "normal", 1.0, w.dtype).to(dev)
        dq_ = torch.empty(q.shape, dtype=torch.float32, device=dev)
        dk_ = torch.empty(k.shape, dtype=torch.float32, device=dev)
        dv_ = torch.empty(v.shape, dtype=torch.float32, device=dev)
        o_saved, lse_saved = o.clone(), lse.clone()

        def bstep():
            ra.attn_bwd(q, k, v, o_saved, lse_saved, do_, dq_, dk_, dv_, 0.0, w.causal, w.window or 0, stream)

        for _ in range(args.warmup):
            bstep()
        torch.cuda.synchronize()
        assert ra.get_device_status(stream) == ra.RA_OK
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        barrier(world)
        torch.cuda.synchronize()
        with ClockSampler(local) as clocks_b:
            for i in range(args.steps):
                flush.zero_()
                starts[i].record(stream)
                bstep()
                ends[i].record(stream)
            torch.cuda.synchronize()
        barrier(world)
        per_step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
        ms = max_over_ranks(sum(per_step_ms) / len(per_step_ms), world, dev)
        status = ra.get_device_status(stream)
        clk = clocks_b.summary()
        launches_per_step = 2
        flops = w.flops() * 2.5  # backward: 5 products of 2*d per pair
    value = world * flops / (ms * 1e-3) / 1e12

    # End to end through the public API: pinned host inputs -> device, ring forward, result -> host.
    qp, kp, vp = (t.pin_memory() for t in (q_h, k_h, v_h))
    qd, kd, vd = (torch.empty_strided(t.shape, t.stride(), dtype=t.dtype, device=dev) for t in (q_h, k_h, v_h))
    o_host = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    lse_host = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in (qp, kp, vp))
    d2h = o_host.numel() * o_host.element_size() + lse_host.numel() * lse_host.element_size()
    e2e_steps = max(3, min(args.steps, args.e2e_steps))

    # Host-resident tensors go through ra_ring_fwd_host, which overlaps the copies of one chunk of
    # heads with the kernels of another (three streams; the compute stream is the timed one).
    # Strided host views (the tabular layout) and the stepwise / windowed variants copy whole
    # tensors around one ra_ring_fwd call instead.
    pipelined = (all(t.is_contiguous() for t in (qp, kp, vp)) and args.schedule == "fused" and w.window is None
                 and not args.backward)
    if pipelined:
        copy_in, copy_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        od = torch.empty_like(o)
        e2e_streams = [copy_in, stream, copy_out]

    def e2e_step():
        if pipelined:
            ra.ring_fwd_host(qp, kp, vp, w.P, w.layout, w.causal, o_host, lse_host, qd, kd, vd, od, lse, 0.0,
                             args.e2e_chunks, e2e_streams)
            return
        for dst, src in zip((qd, kd, vd), (qp, kp, vp)):
            dst.copy_(src, non_blocking=True)
        ra.ring_fwd(qd, kd, vd, w.P, w.layout, w.causal, o, lse, 0.0, args.schedule, [stream], ws, w.window or 0)
        o_host.copy_(o, non_blocking=True)
        lse_host.copy_(lse, non_blocking=True)

    if args.backward:
        # End to end for the backward: Q, K, V, O, LSE, dO in from pinned host memory, dQ, dK, dV out.
        extra_in = [(x.to("cpu").pin_memory(), torch.empty_like(x)) for x in (o_saved, lse_saved, do_)]
        grads_host = [torch.empty(g.shape, dtype=g.dtype, pin_memory=True) for g in (dq_, dk_, dv_)]
        h2d += sum(src.numel() * src.element_size() for src, _ in extra_in)
        d2h = sum(g.numel() * g.element_size() for g in grads_host)

        def e2e_step():  # noqa: F811 - the backward mode's end-to-end step
            for dst, src in zip((qd, kd, vd), (qp, kp, vp)):
                dst.copy_(src, non_blocking=True)
            for src, dst in extra_in:
                dst.copy_(src, non_blocking=True)
            ra.attn_bwd(qd, kd, vd, extra_in[0][1], extra_in[1][1], extra_in[2][1], dq_, dk_, dv_, 0.0, w.causal,
                        w.window or 0, stream)
            for host, dev_t in zip(grads_host, (dq_, dk_, dv_)):
                host.copy_(dev_t, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world, dev)
    e2e_value = world * flops / (e2e_ms * 1e-3) / 1e12
    del qp, kp, vp, qd, kd, vd, o_host, lse_host, bufs, q, k, v, o, lse, ws
    if args.backward:
        del extra_in, grads_host, dq_, dk_, dv_, do_, o_saved, lse_saved
    torch.cuda.empty_cache()

    # Standalone LSE merge of 16 fp32 partials O[1,8,16384,128] + LSE (the k-way merge kernel).
    merge = None
    if not args.skip_merge:
        kparts, rows, dm = 16, 8 * 16384, 128
        mo, ml = I.make_merge_inputs(kparts, rows, dm, seed=1104, empty_frac=0.01)
        mo_l = [x.to(dev) for x in mo]
        ml_l = [x.to(dev) for x in ml]
        out_o = torch.empty(rows, dm, device=dev)
        out_l = torch.empty(rows, device=dev)
        for _ in range(3):
            ra.lse_merge_n(mo_l, ml_l, out_o, out_l, stream)
        torch.cuda.synchronize()
        times = []
        for _ in range(20):
            flush.zero_()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            ra.lse_merge_n(mo_l, ml_l, out_o, out_l, stream)
            b.record(stream)
            times.append((a, b))
        torch.cuda.synchronize()
        mms = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in times), world, dev)
        mbytes = (kparts + 1) * rows * (dm + 1) * 4
        gbs = mbytes / (mms * 1e-3) / 1e9
        merge = {"kernel": "lse_merge_n_kernel", "workload": "16 x fp32 O[1,8,16384,128] + LSE[1,8,16384]",
                 "algorithmic_bytes": mbytes, "ms": mms, "achieved_gbs": gbs, "peak_gbs": peaks["hbm_gbs"],
                 "frac": gbs / peaks["hbm_gbs"], "frac_of_8000": gbs / 8000.0, "launches": 20}
        del mo_l, ml_l, out_o, out_l, mo, ml
        torch.cuda.empty_cache()

    # The other bf16 workloads, each timed the same way (the headline keys stay on the main one).
    others = {}
    if not args.backward and args.configs:
        for c in [int(x) for x in args.configs.split(",") if x.strip().isdigit()]:
            if c == w.cfg:
                continue
            wc = I.WORKLOADS[c]
            steps_c = max(3, min(args.steps, args.config_steps))
            ms_c, per_c, clk_c, l_c, st_c, bufs_c = time_forward(wc, args, dev, stream, flush, world, steps_c,
                                                                 args.warmup)
            del bufs_c
            torch.cuda.empty_cache()
            v_c, roof_c = forward_roofline(wc, ms_c, world, peak, peak_kind, l_c,
                                           recorded_traffic(traffic_key(wc, walk=args.striped_walk), args.schedule))
            others[f"cfg{c}"] = {
                "workload": wc.name, "steps": steps_c, "ms_per_step": ms_c, "value": v_c, "unit": "TFLOP/s",
                "flops_per_step": wc.flops(), "pct_of_spec_bf16_peak": 100.0 * (v_c / world) / SPEC_BF16_TFLOPS,
                "roofline": roof_c, "mufu_roofline": mufu_roofline(wc, ms_c, world, clk_c),
                "gpu_launches": l_c * steps_c, "clocks": clk_c, "device_status": ra.status_string(st_c),
                "step_ms_min": min(per_c), "step_ms_median": statistics.median(per_c)}

    if rank != 0:
        return 0
    if args.backward:
        roof = {"bound": "tensor", "kernel": "attn_bwd_sm100 (dQ + dK/dV instances)", "achieved": value / world,
                "peak": peak, "peak_kind": f"{peak_kind} bf16 burst", "unit": "TFLOP/s",
                "frac": (value / world) / peak,
                "traffic": args.traffic if args.traffic is not None else recorded_traffic(traffic_key(w, True),
                                                                                           args.schedule),
                "note": BWD_NOTE}
    else:
        _, roof = forward_roofline(w, ms, world, peak, peak_kind, launches_per_step,
                                   args.traffic if args.traffic is not None
                                   else recorded_traffic(traffic_key(w, walk=args.striped_walk), args.schedule))
    line = {
        "metric": METRIC_BWD if args.backward else METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic (seeded, shapes and distributions of the workload)",
        "config": config_dict(w, args),
        "pct_of_spec_bf16_peak": 100.0 * (value / world) / SPEC_BF16_TFLOPS,
        "pct_of_measured_bf16_peak": 100.0 * (value / world) / peak,
        "roofline": roof,
        "mufu_roofline": None if args.backward else mufu_roofline(w, ms, world, clk),
        "fp32_roofline": (fp32_roofline(value / world, clk) if args.backward and w.dtype == "f32" else None),
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms,
                "call": (f"ra_ring_fwd_host ({args.e2e_chunks} chunks of heads, copies overlapped with the kernels)"
                         if pipelined else "copies in, one ring / backward call, copies out (one stream)")},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
        "device_status": ra.status_string(status),
        "step_ms_min": min(per_step_ms), "step_ms_median": statistics.median(per_step_ms),
    }
    if merge is not None:
        line["merge"] = merge
    if others:
        line["configs"] = others
    if not args.skip_cpu and world == 1 and not args.backward:
        line["cpu_baseline"] = cpu_baseline(w, args.cpu_budget)
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=3,
                    help="headline workload (default 3: the largest bf16 causal ring, B=1 H=32 N=32768 d=128)")
    ap.add_argument("--configs", default="2,4,5",
                    help="other workloads timed in the same run, reported under 'configs' ('' for none)")
    ap.add_argument("--config-steps", type=int, default=20,
                    help="timed steps per workload under 'configs' (at most --steps)")
    ap.add_argument("--schedule", choices=["stepwise", "fused"], default="fused")
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--e2e-chunks", type=int, default=8,
                    help="chunks of heads in the end-to-end call (ra_ring_fwd_host)")
    ap.add_argument("--ref-rows", type=int, default=64)
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--skip-cpu", action="store_true")
    ap.add_argument("--skip-merge", action="store_true")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward pass (ra_attn_bwd) instead of the forward")
    ap.add_argument("--window", type=int, default=None,
                    help="causal sliding-window variant of a causal workload (window in positions)")
    ap.add_argument("--kv-heads", type=int, default=None,
                    help="grouped-query variant of the workload: K and V with this many heads (must divide H)")
    ap.add_argument("--layout", choices=["contiguous", "striped"], default=None,
                    help="ring shard layout override (the workload's own by default)")
    ap.add_argument("--striped-walk", choices=["shard", "tile"], default="shard",
                    help="K/V walk order of fused rings over striped shards (ra_set_striped_walk)")
    ap.add_argument("--n", type=int, default=None,
                    help="sequence length override: a smaller case of the workload's layout (profiling)")
    ap.add_argument("--traffic", type=float, default=None,
                    help="DRAM bytes per launch of the attention kernel, from an ncu capture of the current kernel")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    from ring_blockwise_softmax_b200 import inputs as I

    if args.striped_walk != "shard" and args.impl != "reference":
        from ring_blockwise_softmax_b200 import ra_attn as ra_walk

        ra_walk.set_striped_walk(args.striped_walk)

    w = I.WORKLOADS[args.config]
    if args.layout is not None:
        import dataclasses

        w = dataclasses.replace(w, layout=args.layout)
    if args.n is not None:
        import dataclasses

        if args.n < w.P or args.n % w.P != 0:
            raise SystemExit("--n must be a positive multiple of the workload's P")
        w = dataclasses.replace(w, N=args.n)
    if args.kv_heads is not None:
        if w.tabular is not None or args.kv_heads < 1 or w.H % args.kv_heads != 0:
            raise SystemExit("--kv-heads must divide H and does not apply to the tabular workload")
        import dataclasses

        w = dataclasses.replace(w, H_kv=args.kv_heads)
    if args.window is not None:
        if not w.causal or args.window < 1:
            raise SystemExit("--window needs a causal workload and a window >= 1")
        import dataclasses

        w = dataclasses.replace(w, window=args.window)
    if args.impl == "reference":
        return run_reference(args, w)
    return run_gpu(args, w)


if __name__ == "__main__":
    sys.exit(main())
