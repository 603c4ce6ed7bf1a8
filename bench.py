#!/usr/bin/env python
"""Benchmark of the VGG-T^3 TTT layer on B200.

One step = one ``ttt_layer`` call over the whole workload: ShortConv2D of V,
`steps` SGD write steps (forward residual, backward partials, reduce+update)
and the read of Q.  Default workload: 1000 views x (37x37 + 5) tokens
(1,374,000 tokens), 16 heads, d=64, h=256, 2 steps, lr 0.05, bf16 operands.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (under torchrun) the ranks run the write of ONE collection sharded
by views: each rank holds 1000 views of an N x 1000-view collection,
convolves and reads its own views, and per SGD step the ranks all-gather
their gradient sums (NCCL, 3*heads*d*h floats each) and apply the same
fixed-order update (test_layer_reconstruction_b200.sharded).  Per-GPU work is
fixed, so the scaling is weak; value = all ranks' tokens / max-over-ranks
time.  ``--replicas`` runs independent scenes instead (no exchange).
``--impl reference`` times the float64 CPU oracle on bounded samples of the
same workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "TTT layer tokens/s (write 2 steps + read) at 1000 views; % BF16 TC & HBM peak"
DEFAULT_CONFIG = "views1000_37x37p5_h16_d64_h256"


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            return None
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- oracle timing
def _blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        info = [i for i in threadpool_info() if i.get("user_api") == "blas"]
        if info:
            return int(info[0]["num_threads"])
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def _oracle_sample(cfg, n_views_sample: int, head: int = 0) -> float:
    """Seconds of the float64 oracle on `n_views_sample` views x 1 head of the workload."""
    import numpy as np  # noqa: F401
    from oracle import ttt_oracle as orc
    from test_layer_reconstruction_b200 import inputs as tin
    sub = cfg.with_views(n_views_sample)
    inp = tin.make_inputs(sub)
    d = cfg.d
    ch = slice(head * d, (head + 1) * d)
    K = inp["K"][:, head].double().numpy()
    Q = inp["Q"][:, head].double().numpy()
    V = inp["V"][:, head].double().numpy()
    w = inp["conv_w"][ch].double().numpy()
    th0 = (inp["W1"][head].double().numpy(), inp["W3"][head].double().numpy(), inp["W2"][head].double().numpy())
    dims = orc.Dims(sub.n_views, sub.grid_h, sub.grid_w, sub.n_special)
    t0 = time.perf_counter()
    Vp = orc.shortconv2d(V, w, dims)
    th, _ = orc.sgd_write(K, Vp, th0, sub.lr, sub.steps)
    orc.read(Q, *th)
    return time.perf_counter() - t0


def _oracle_tokens_per_s(cfg, seconds_budget: float):
    """Time the oracle on a bounded sample; returns (tokens/s in layer tokens, description)."""
    t_small = _oracle_sample(cfg, 2)
    per_view = t_small / 2
    views = max(2, min(cfg.n_views, int(seconds_budget / max(per_view, 1e-6))))
    t = _oracle_sample(cfg, views)
    tokens = views * cfg.tokens_per_view
    # one head of `heads`: a full-layer token costs `heads` times the per-head work
    value = tokens / (t * cfg.heads)
    desc = (f"float64 numpy oracle, 1 of {cfg.heads} heads x {views} of {cfg.n_views} views "
            f"({tokens} tokens, {cfg.steps} steps), {t:.2f} s; tokens/s = tokens / (time * heads)")
    return value, desc, t


# ----------------------------------------------------------------------------- arms
def replica_config(cfg, rank: int):
    """The workload of `rank` in a multi-GPU run: the same shape, its own scene
    (seed offset by rank)."""
    from test_layer_reconstruction_b200 import inputs as tin
    return tin.LayerConfig(cfg.name, cfg.n_views, cfg.grid_h, cfg.grid_w, cfg.n_special, cfg.heads, cfg.d, cfg.h,
                           cfg.steps, cfg.lr, cfg.seed + 1000 * rank)


def shard_views(cfg, rank: int, world: int):
    """The collection of a sharded multi-GPU run (world x cfg.n_views views, the
    workload's seed) and the contiguous views of `rank`."""
    scene = cfg.with_views(cfg.n_views * world)
    return scene, range(rank * cfg.n_views, (rank + 1) * cfg.n_views)


def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's time (all ranks call it, in the same order)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tokens_per_s(world: int, tokens_per_rank: int, ms_max: float) -> float:
    """All ranks' tokens over the slowest rank's time (weak scaling)."""
    return world * tokens_per_rank / (ms_max / 1e3)


def run_reference(args, cfg):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    per_step_budget = max(2.0, min(20.0, 150.0 / max(1, args.steps + args.warmup)))
    t_small = _oracle_sample(cfg, 2)
    views = max(2, min(cfg.n_views, int(per_step_budget / max(t_small / 2, 1e-6))))
    for _ in range(args.warmup):
        _oracle_sample(cfg, views)
    times = [_oracle_sample(cfg, views) for _ in range(args.steps)]
    t = sum(times) / len(times)
    tokens = views * cfg.tokens_per_view
    value = tokens / (t * cfg.heads)
    cores = _blas_threads()
    sample = (f"float64 numpy oracle, 1 of {cfg.heads} heads x {views} of {cfg.n_views} views "
              f"({tokens} tokens, {cfg.steps} steps) per step; tokens/s = tokens / (time * heads)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg.name, "n_views": cfg.n_views, "tokens": cfg.n, "heads": cfg.heads, "d": cfg.d,
                   "h": cfg.h, "steps": cfg.steps, "lr": cfg.lr},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def _kernel_work(cfg, n_read=None):
    """Algorithmic work of each kernel kind in ONE step (a layer call, plus the
    held-out read where the workload has one): bytes for the HBM-bound kinds,
    FLOPs for the tensor-core ones.  `n_read` is the number of tokens read
    (the layer's Q plus held-out queries)."""
    n, H, d, h, st = cfg.n, cfg.heads, cfg.d, cfg.h, cfg.steps
    n_read = n if n_read is None else n_read
    tok = n * H * d * 2
    theta = 3 * H * d * h * 4
    hidp = 128 * math.ceil(h / 128)
    return {
        "shortconv2d": ("hbm", 2 * tok + H * d * 9 * 4),                 # read V, write V'
        "swiglu_fwd_residual": ("tensor", st * 6.0 * d * h * n * H),     # Z1, Z3, Y
        "swiglu_bwd_partials": ("tensor", st * 8.0 * d * h * n * H),     # dA, dW1, dW3, dW2
        "swiglu_fwd_read": ("tensor", 6.0 * d * h * n_read * H),
        # read theta (f32); write the operand images (bf16 W1|W3, bf16 and f16 W2)
        "pack_theta": ("hbm", (st + 1) * (theta + 4 * H * hidp * d * 2)),
        # read theta, write theta* (the split-K partials it also reads are a by-product of the tiling)
        "reduce_sgd": ("hbm", st * 2 * theta),
        # the tensor-core GEMMs of the wide-head path and the surround
        "gemm_gate": ("tensor", 4.0 * d * h * H * (st * n + n_read)),     # Z1, Z3
        "gemm_residual": ("tensor", st * 2.0 * d * h * n * H),            # Y = A W2
        "gemm_dz": ("tensor", st * 2.0 * d * h * n * H),                  # dA = E W2^T
        "gemm_wgrad": ("tensor", st * 6.0 * d * h * n * H),               # dW1, dW3, dW2
        "gemm_store": ("tensor", 2.0 * d * h * n_read * H),               # O = A W2
        "gemm_qkv_l2norm": ("tensor", 3 * 2.0 * n * (H * d) ** 2),        # X Wq, X Wk, X Wv
    }


def _kernel_table(prof, work, steps, peaks):
    """Per kernel kind: launches and time per step, achieved rate on its
    algorithmic work per step, fraction of the measured peak."""
    total = sum(r["total_ms"] for k, r in prof.items() if not k.startswith("_"))
    kernels = {}
    for name, rec in prof.items():
        if name.startswith("_") or rec["launches"] == 0 or name not in work:
            continue
        bound, amount = work[name]
        ms_step = rec["total_ms"] / steps
        extra = {}
        if bound == "tensor":
            # each launch is timed on its own (CUDA events around every launch), so the
            # burst GEMM peak is the denominator; the sustained figure is a second number
            achieved = amount / (ms_step / 1e3) / 1e12
            peak = peaks["bf16_tflops"]
            unit = "TFLOP/s"
            extra = {"peak_sustained": peaks["bf16_tflops_sustained"],
                     "frac_sustained": achieved / peaks["bf16_tflops_sustained"]}
        else:
            achieved = amount / (ms_step / 1e3) / 1e9
            peak = peaks["hbm_gbs"]
            unit = "GB/s"
        kernels[name] = {"launches_per_step": rec["launches"] / steps,
                         "ms_per_launch": rec["total_ms"] / rec["launches"], "ms_per_step": ms_step,
                         "share": rec["total_ms"] / max(1e-9, total), "bound": bound, "achieved": achieved,
                         "peak": peak, "unit": unit, "frac": achieved / peak if peak else None, **extra}
    return kernels


def run_ours(args, cfg):
    import torch
    import torch.distributed as dist
    from test_layer_reconstruction_b200 import build as tbuild
    from test_layer_reconstruction_b200 import inputs as tin
    from test_layer_reconstruction_b200 import sharded, ttt

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    distributed = world > 1 or (args.shard and "MASTER_ADDR" in os.environ)
    if distributed:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    tbuild.build()
    ttt.load_library()

    def barrier():
        if world > 1:
            dist.barrier()

    # N > 1: this rank's views of one collection (or, with --replicas, its own scene).
    shard = (world > 1 and not args.replicas) or args.shard
    if shard:
        scene, views = shard_views(cfg, rank, world)
        inp = tin.make_inputs(scene, device="cuda", views=views)
    else:
        inp = tin.make_inputs(replica_config(cfg, rank), device="cuda")
    Q = inp["Q"].to(torch.bfloat16).contiguous()
    K = inp["K"].to(torch.bfloat16).contiguous()
    V = inp["V"].to(torch.bfloat16).contiguous()
    conv_w = inp["conv_w"].contiguous()
    theta0 = tin.pack_theta(inp["W1"], inp["W3"], inp["W2"]).cuda()
    del inp
    torch.cuda.empty_cache()
    theta = torch.empty_like(theta0)
    O = torch.empty_like(Q)
    ws = ttt.make_workspace(cfg, ttt.OP_LAYER)
    if shard:
        n_total = cfg.n * world
        gather = sharded.all_gather_rows() if distributed else (lambda t: t.reshape(1, -1))
        ops = sharded.ShardOps(
            conv=lambda V_, w_, dm: ttt.shortconv2d(V_, w_, dm),
            grad=lambda K_, Vp_, th_, dm: ttt.grad(K_, Vp_, th_, dm, workspace=ws),
            update=lambda th_, g_, sc_, dm: ttt.sgd_update(th_, g_, sc_, dm),
            read=lambda Q_, th_, dm: ttt.read(Q_, th_, dm, O=O, workspace=ws))

        def layer_call(Q_, K_, V_, w_, th0_):
            return sharded.layer_sharded(Q_, K_, V_, w_, th0_, cfg.lr, cfg.steps, cfg, n_total, gather, ops)
    elif args.inner == "muon":
        # the pages' own inner loop: dot-product loss, Muon steps at their lr 0.1
        def layer_call(Q_, K_, V_, w_, th0_):
            return ttt.layer_muon(Q_, K_, V_, w_, th0_, 0.1, cfg.steps, cfg, theta_out=theta, O=O, workspace=ws)
    else:
        def layer_call(Q_, K_, V_, w_, th0_):
            return ttt.layer(Q_, K_, V_, w_, th0_, cfg.lr, cfg.steps, cfg, theta_out=theta, O=O, workspace=ws)

    # Workloads with held-out views: each step also reads their queries with
    # the frozen theta* (the localisation-style query path).
    n_read = cfg.n
    held = None
    if cfg.heldout_views > 0:
        hcfg = cfg.with_views(cfg.heldout_views)
        Qh = tin.make_inputs(cfg, device="cuda", heldout=True)["Q"].to(torch.bfloat16).contiguous()
        held = (hcfg, Qh, torch.empty_like(Qh), ttt.make_workspace(hcfg, ttt.OP_READ))
        n_read += hcfg.n

    def step():
        th_, _ = layer_call(Q, K, V, conv_w, theta0)
        if held is not None:
            hcfg_, Qh_, Oh_, wsr_ = held
            ttt.read(Qh_, th_, hcfg_, O=Oh_, workspace=wsr_)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if ttt.check_status(ws) != 0:
        raise SystemExit("device status word set during warm-up")

    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(torch.cuda.current_device())
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    ttt.profile_start()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    prof = ttt.profile_stop()
    clk = clocks.stop()
    barrier()
    ms = e0.elapsed_time(e1) / args.steps
    if ttt.check_status(ws) != 0:
        raise SystemExit("device status word set during the timed steps")
    ms_max = max_over_ranks(ms, world, "cuda")
    value = whole_job_tokens_per_s(world, cfg.n, ms_max)

    # per-kernel roofline from the live event timings
    peaks = _peaks()
    kernels = _kernel_table(prof, _kernel_work(cfg, n_read), args.steps, peaks)
    dom = max(kernels, key=lambda k: kernels[k]["ms_per_step"])
    dk = kernels[dom]
    traffic = _traffic_from_profiles(dom, cfg.name)
    roofline = {"kernel": dom, "bound": dk["bound"], "achieved": dk["achieved"], "peak": dk["peak"],
                "unit": dk["unit"], "frac": dk["frac"], "traffic": traffic,
                "peak_source": f"{peaks['source']} ({'burst bf16 GEMM' if dk['bound'] == 'tensor' else 'HBM copy'})"}
    if dk["bound"] == "tensor":
        roofline["frac_sustained"] = dk["frac_sustained"]
    gpu_launches = sum(r["launches"] for k, r in prof.items() if not k.startswith("_"))

    # end to end through the host-buffer entry point
    e2e = None
    if args.e2e_steps > 0 and shard:
        # the sharded layer from pinned host buffers: this rank's inputs up, O and theta* back
        hq, hk, hv = (t.cpu().pin_memory() for t in (Q, K, V))
        hw = conv_w.cpu().pin_memory()
        ht0 = theta0.cpu().pin_memory()
        hth = torch.empty_like(ht0).pin_memory()
        ho = torch.empty_like(hq).pin_memory()
        h2d = 3 * hq.numel() * 2 + hw.numel() * 4 + ht0.numel() * 4
        d2h = ho.numel() * 2 + hth.numel() * 4
        dq, dk, dv, dw, dt = (torch.empty_like(t) for t in (Q, K, V, conv_w, theta0))

        def host_call():
            for dst, src in ((dq, hq), (dk, hk), (dv, hv), (dw, hw), (dt, ht0)):
                dst.copy_(src, non_blocking=True)
            th_, O_ = layer_call(dq, dk, dv, dw, dt)
            hth.copy_(th_, non_blocking=True)
            ho.copy_(O_, non_blocking=True)

        host_call()
        torch.cuda.synchronize()
        barrier()
        t0 = time.perf_counter()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(args.e2e_steps):
            host_call()
        f1.record(stream)
        torch.cuda.synchronize()
        e_ms = f0.elapsed_time(f1) / args.e2e_steps
        e_max = max_over_ranks(e_ms, world, "cuda")
        e2e = {"value": whole_job_tokens_per_s(world, cfg.n, e_max), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
               "wall_s_per_step": (time.perf_counter() - t0) / args.e2e_steps}
    elif args.e2e_steps > 0:
        ws_h = ttt.make_workspace(cfg, ttt.OP_LAYER_HOST)
        hq, hk, hv = (t.cpu().pin_memory() for t in (Q, K, V))
        hw = conv_w.cpu().pin_memory()
        ht0 = theta0.cpu().pin_memory()
        hth = torch.empty_like(ht0).pin_memory()
        ho = torch.empty_like(hq).pin_memory()
        h2d = 3 * hq.numel() * 2 + hw.numel() * 4 + ht0.numel() * 4
        d2h = ho.numel() * 2 + hth.numel() * 4
        ttt.layer_host(hq, hk, hv, hw, ht0, cfg.lr, cfg.steps, cfg, hth, ho, ws_h)
        torch.cuda.synchronize()
        barrier()
        t0 = time.perf_counter()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(args.e2e_steps):
            ttt.layer_host(hq, hk, hv, hw, ht0, cfg.lr, cfg.steps, cfg, hth, ho, ws_h)
        f1.record(stream)
        torch.cuda.synchronize()
        e_ms = f0.elapsed_time(f1) / args.e2e_steps
        e_max = max_over_ranks(e_ms, world, "cuda")
        e2e = {"value": whole_job_tokens_per_s(world, cfg.n, e_max), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
               "wall_s_per_step": (time.perf_counter() - t0) / args.e2e_steps}
        del ws_h

    # Linear-scaling sweep over view counts (prefixes of the same inputs: views
    # are contiguous token ranges) and the write-only / read-only split at 100
    # views, each timed with CUDA events like the main run.
    sweep, paths = None, None
    if rank == 0 and world == 1 and not args.no_sweep and cfg.name == DEFAULT_CONFIG:
        T = cfg.tokens_per_view

        def time_calls(fn, reps=3, warm=2):
            for _ in range(warm):
                fn()
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(reps):
                fn()
            b.record(stream)
            torch.cuda.synchronize()
            return a.elapsed_time(b) / reps

        pts = []
        for v in (100, 250, 500):
            if v >= cfg.n_views:
                continue
            sub, nt = cfg.with_views(v), v * T
            q, k, vv = Q[:nt], K[:nt], V[:nt]
            th, o = torch.empty_like(theta0), torch.empty_like(q)
            wsv = ttt.make_workspace(sub, ttt.OP_LAYER)
            ms_v = time_calls(lambda: ttt.layer(q, k, vv, conv_w, theta0, cfg.lr, cfg.steps, sub, theta_out=th, O=o,
                                                workspace=wsv))
            pts.append((v, ms_v))
            if ttt.check_status(wsv) != 0:
                raise SystemExit(f"device status word set during the {v}-view sweep point")
            del wsv
        pts.append((cfg.n_views, ms_max))
        sweep = {"views": [v for v, _ in pts], "ms_per_call": [round(m, 3) for _, m in pts],
                 "tokens_per_s": [v * T / (m / 1e3) for v, m in pts]}
        v = min(100, cfg.n_views)
        sub, nt = cfg.with_views(v), v * T
        q, k, vv = Q[:nt], K[:nt], V[:nt]
        th, o = torch.empty_like(theta0), torch.empty_like(q)
        wsw, wsr = ttt.make_workspace(sub, ttt.OP_WRITE), ttt.make_workspace(sub, ttt.OP_READ)
        ms_w = time_calls(lambda: ttt.write(k, vv, conv_w, theta0, cfg.lr, cfg.steps, sub, theta_out=th, workspace=wsw))
        ms_r = time_calls(lambda: ttt.read(q, th, sub, O=o, workspace=wsr))
        paths = {"views": v, "write_ms": round(ms_w, 3), "write_tokens_per_s": nt / (ms_w / 1e3),
                 "read_ms": round(ms_r, 3), "read_tokens_per_s": nt / (ms_r / 1e3)}
        if ttt.check_status(wsw) != 0 or ttt.check_status(wsr) != 0:
            raise SystemExit("device status word set during the write/read split")
        del wsw, wsr
        # The pages' own inner loop on the whole workload: dot-product loss, Muon
        # steps (lr 0.1, as the pages give it), same steps and read.
        ttt.profile_start()
        ms_mu = time_calls(lambda: ttt.layer_muon(Q, K, V, conv_w, theta0, 0.1, cfg.steps, cfg, theta_out=theta, O=O,
                                                  workspace=ws))
        prof_mu = ttt.profile_stop()
        if ttt.check_status(ws) != 0:
            raise SystemExit("device status word set during the Muon layer")
        calls = 5   # time_calls: 2 warm-up + 3 timed
        paths["dot_loss_muon"] = {
            "views": cfg.n_views, "lr": 0.1, "steps": cfg.steps, "ms_per_call": round(ms_mu, 3),
            "tokens_per_s": cfg.n / (ms_mu / 1e3),
            "ms_per_call_by_kernel": {k: round(r["total_ms"] / calls, 3) for k, r in prof_mu.items()
                                      if not k.startswith("_") and r["launches"]}}
        # The same layer with Q, K, V left in pinned host memory and streamed in
        # chunks of 100 views (the offload path for collections beyond HBM).
        from test_layer_reconstruction_b200 import stream as tstream
        hq, hk, hv = (t.cpu().pin_memory() for t in (Q, K, V))
        chunk = min(100, cfg.n_views)

        def streamed_call():
            th_ = tstream.write_streamed(hk, hv, conv_w, theta0, cfg.lr, cfg.steps, cfg, chunk)
            tstream.read_streamed(hq, th_, cfg, chunk)

        ms_st = time_calls(streamed_call, reps=2, warm=1)
        paths["streamed_from_host"] = {
            "views": cfg.n_views, "chunk_views": chunk, "ms_per_call": round(ms_st, 1),
            "tokens_per_s": cfg.n / (ms_st / 1e3),
            "host_bytes_per_call": int((cfg.steps * 2 + 2) * hq.numel() * 2)}
        del hq, hk, hv
    if rank == 0 and world == 1 and not args.no_sweep and cfg.name == DEFAULT_CONFIG and not args.no_surround:
        # The layer's surround on the same workload: q = L2(X Wq), k = L2(X Wk),
        # v = X Wv (one GEMM launch, the normalisation in its epilogue), the
        # layer, out = O Wo.
        sx = tin.make_surround(cfg, device="cuda")
        sdev = {k: sx[k].to(torch.bfloat16).contiguous() for k in ("X", "Wq", "Wk", "Wv", "Wo")}
        del sx
        torch.cuda.empty_cache()
        ws_a = ttt.make_workspace(cfg, ttt.OP_ATTENTION)
        s_out = torch.empty_like(sdev["X"])
        ttt.profile_start()
        ms_att = time_calls(lambda: ttt.attention(sdev["X"], sdev["Wq"], sdev["Wk"], sdev["Wv"], sdev["Wo"], conv_w,
                                                  theta0, cfg.lr, cfg.steps, cfg, theta_out=theta, out=s_out,
                                                  workspace=ws_a))
        prof_att = ttt.profile_stop()
        if ttt.check_status(ws_a) != 0:
            raise SystemExit("device status word set during the attention layer")
        work_att = _kernel_work(cfg)
        work_att["gemm_store"] = ("tensor", 2.0 * cfg.n * (cfg.heads * cfg.d) ** 2)   # out = O Wo
        tab = _kernel_table(prof_att, work_att, calls, _peaks())
        paths["attention_surround"] = {
            "views": cfg.n_views, "ms_per_call": round(ms_att, 3), "tokens_per_s": cfg.n / (ms_att / 1e3),
            "qkv_projection": tab.get("gemm_qkv_l2norm"), "output_projection": tab.get("gemm_store")}
        del sdev, s_out, ws_a

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, desc, _ = _oracle_tokens_per_s(cfg, args.cpu_seconds)
        cpu = {"value": v, "unit": "tokens/s", "cores": _blas_threads(), "kind": "oracle", "sample": desc}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": cfg.name, "n_views": cfg.n_views, "tokens": cfg.n, "heads": cfg.heads,
                       "d": cfg.d, "h": cfg.h, "steps": cfg.steps, "lr": cfg.lr,
                       "l2": f"no flush: every token tensor ({cfg.n * cfg.heads * cfg.d * 2 / 1e9:.2f} GB) exceeds the 126 MB L2",
                       "parallelism": (f"{world} GPUs: one {cfg.n_views * world}-view collection sharded by views "
                                       f"({cfg.n_views} per GPU), gradient all-gather per step (NCCL)" if shard
                                       else f"{world} independent replicas" if world > 1 else "1 GPU"),
                       **({"inner": "dot-product loss + Muon steps, lr 0.1"} if args.inner == "muon" else {}),
                       **({"heldout_views": cfg.heldout_views, "tokens_read": n_read,
                           "value_counts": "the layer's tokens (the held-out read is extra work in each step)"}
                          if cfg.heldout_views else {})},
            "roofline": roofline, "kernels": kernels, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": gpu_launches, "clocks": clk, "sweep": sweep, "paths": paths,
        }
        print(json.dumps(line), flush=True)
    if distributed:
        dist.destroy_process_group()
    return 0


def _source_digest(files) -> str:
    """sha256 over the named CUDA sources (test_layer_reconstruction_b200/csrc), in the given order."""
    import hashlib
    d = os.path.join(ROOT, "test_layer_reconstruction_b200", "csrc")
    h = hashlib.sha256()
    for name in files:
        h.update(name.encode())
        with open(os.path.join(d, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def _traffic_from_profiles(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary
    (profiles/traffic.json), or None when the counters were taken on another
    workload or the kernel's sources have changed since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    try:
        with open(path) as f:
            t = json.load(f)
        e = t["kernels"].get(kernel)
        if t.get("workload") != workload or e is None or e["sha256"] != _source_digest(e["sources"]):
            return None
        return e["bytes_per_launch"]
    except Exception:
        return None


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default=DEFAULT_CONFIG)
    ap.add_argument("--views", type=int, default=0,
                    help="run the workload's shape on this many views instead (small cases for profiling)")
    ap.add_argument("--e2e-steps", type=int, default=2)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sweep", action="store_true", help="skip the view-count sweep and write/read split")
    ap.add_argument("--no-surround", action="store_true", help="skip the attention-surround measurement")
    ap.add_argument("--inner", default="sgd", choices=["sgd", "muon"],
                    help="inner loop of the timed layer: mean-squared loss + SGD, or dot-product loss + Muon")
    ap.add_argument("--replicas", action="store_true",
                    help="with N > 1: independent scenes per GPU instead of one collection sharded by views")
    ap.add_argument("--shard", action="store_true",
                    help="run the view-sharded layer even on one GPU (under torchrun: with the NCCL all-gather)")
    args = ap.parse_args()
    from test_layer_reconstruction_b200 import inputs as tin
    cfg = tin.CONFIGS[args.config]
    if args.views > 0:
        import dataclasses
        cfg = dataclasses.replace(cfg.with_views(args.views), name=f"{cfg.name}@{args.views}views",
                                  heldout_views=min(cfg.heldout_views, args.views))
    if args.impl == "reference":
        return run_reference(args, cfg)
    return run_ours(args, cfg)


if __name__ == "__main__":
    sys.exit(main())
