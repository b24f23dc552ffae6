#!/usr/bin/env python
"""Throughput of the pi0 flow-matching action sampler (libpi0x) on B200.

One bench "step" is one whole sampler call: all Euler steps (one action chunk per
sample) over one batch of synthetic inputs, inputs resident in HBM.  The default
workload is the full pi0 action expert at B=1 with 10 Euler steps and an
816-token prefix; ``--workload`` selects another of the five workloads.

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle on the
same workload instead (host cores, bounded samples).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from vla_flow_matching_b200 import synth  # noqa: E402

METRIC = "action chunks/sec and µs per 10-step chunk at B=1/32/128; % HBM/TC roofline"
UNIT = "chunks/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------------------------------
def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def algorithmic_work(wl):
    """Per call: (GEMM bytes, GEMM flops, attention flops), algorithmic counts.

    GEMM bytes per launch: the bf16 weight once, the bf16 activation operand once
    and the output once in the type the method needs next (bf16 q/k/v, u and the
    GeGLU product; fp32 residual stream read and written for O-proj and down-proj,
    fp32 written for the time-MLP output).  Rows: every sample's 1 + H suffix
    tokens at the first Euler step, its H action tokens afterwards (the state
    token's hidden states and K/V depend on neither x_t nor t).
    """
    d, B, N = wl.dims, wl.batch, wl.num_steps
    W, F, Q, Dh, L, H = d.width, d.mlp_dim, d.num_heads * d.head_dim, d.head_dim, d.depth, d.horizon
    n = synth.make_mask(wl).sum(axis=1).astype(np.int64)
    byt = flo = att = 0
    for k in range(N):
        M = B * (H + 1) if k == 0 else B * H
        # (rows, out features, in features, output bytes per element)
        gemms = [(B * H, W, W, 2), (B * H, W, W, 4)]
        for _ in range(L):
            gemms += [(M, Q + 2 * Dh, W, 2), (M, W, Q, 8), (M, 2 * F, W, 1), (M, W, F, 8)]
        for (m, nn, kk, ob) in gemms:
            byt += nn * kk * 2 + m * kk * 2 + m * nn * ob
            flo += 2 * m * nn * kk
        # attention (QK^T and PV): action queries see n_b + 1 + H keys, the state
        # query (first step only) n_b + 1
        keys = H * (n + 1 + H) + ((n + 1) if k == 0 else 0)
        att += int(4 * d.num_heads * Dh * keys.sum()) * L
    return byt, flo, att


def sample_clocks_start():
    q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    try:
        return subprocess.Popen(["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                text=True)
    except (OSError, FileNotFoundError):
        return None


def sample_clocks_stop(proc, gpu_index):
    if proc is None:
        return None
    proc.terminate()
    try:
        out, _ = proc.communicate(timeout=5)
    except subprocess.TimeoutExpired:
        proc.kill()
        out, _ = proc.communicate()
    sm, mx, reasons = [], None, set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for line in out.splitlines():
        f = [x.strip() for x in line.split(",")]
        if len(f) < 9 or not f[0].isdigit() or int(f[0]) != gpu_index:
            continue
        try:
            sm.append(float(f[1]))
            mx = float(f[2])
        except ValueError:
            continue
        for name, v in zip(names, f[5:9]):
            if v.lower().startswith("active"):
                reasons.add(name)
    if not sm:
        return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": 0}
    return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
            "samples": len(sm)}


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = [p for p in threadpool_info() if p.get("user_api") == "blas"]
        if info:
            return int(info[0]["num_threads"])
    except Exception:
        pass
    return os.cpu_count() or 1


def slowest_rank_ms(ms, dist, device="cuda"):
    """The device time of the slowest rank: every rank passes its own CUDA-event time
    and all take the same collective step (a MAX all-reduce); without a process
    group the time is returned as is."""
    if dist is None:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, batch, calls, ms):
    """Whole-job chunks/s: every rank (one GPU) runs `calls` calls of `batch`
    samples (replicas with a fixed per-GPU batch), all done in `ms`."""
    return world * batch * calls / (ms / 1000.0)


def variant_of(args):
    """The solver / convention variant the run uses (oracle keyword arguments)."""
    return dict(time_convention=args.time_grid, x_prediction=args.x_prediction,
                causal_actions=args.causal_actions)


def time_oracle(wl, budget_s=12.0, max_reps=50, variant=None):
    """The CPU oracle, as it stands, on bounded samples of the workload.

    Each repetition runs all Euler steps of one sample (one action chunk).
    Returns (chunks per second, description, cores).
    """
    from oracle import pi0_oracle as O
    w = synth.make_weights(wl.dims, wl.seed)
    reps, t_total, b = 0, 0.0, 0
    while reps < max_reps and (t_total < budget_s or reps == 0):
        inp = synth.make_inputs(wl, samples=[b % wl.batch], weights=w)
        t0 = time.perf_counter()
        O.sample_actions(inp.weights, inp.prefix_k, inp.prefix_v, inp.mask, inp.state, inp.x1,
                         wl.num_steps, **(variant or {}))
        t_total += time.perf_counter() - t0
        reps += 1
        b += 1
    desc = (f"{reps} whole action chunk(s) ({wl.num_steps} Euler steps, 1 sample each) of "
            f"workload {wl.name}, fp32 numpy oracle, {t_total:.1f} s")
    return reps / t_total, desc, blas_threads()


# ---------------------------------------------------------------------------------------
def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from oracle import pi0_oracle as O
    w = synth.make_weights(wl.dims, wl.seed)
    inps = [synth.make_inputs(wl, samples=[i % wl.batch], weights=w) for i in range(min(wl.batch, 4))]

    def one(i):
        inp = inps[i % len(inps)]
        O.sample_actions(inp.weights, inp.prefix_k, inp.prefix_v, inp.mask, inp.state, inp.x1,
                         wl.num_steps, **variant_of(args))
    for i in range(args.warmup):
        one(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        one(i)
    dt = time.perf_counter() - t0
    value = args.steps / dt
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "config": config_of(wl, args),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"each step: all {wl.num_steps} Euler steps of one sample of "
                                   f"workload {wl.name} (fp32 numpy oracle on {cores} threads)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_of(wl, args):
    d = wl.dims
    return {"workload": wl.name, "batch": wl.batch, "prefix_len": wl.prefix_len,
            "num_steps": wl.num_steps, "depth": d.depth, "horizon": d.horizon,
            "action_dim": d.action_dim, "width": d.width, "precision": args.precision,
            "time_grid": args.time_grid, "x_prediction": args.x_prediction,
            "causal_actions": args.causal_actions,
            "l2": "inputs larger than L2: every Euler step streams the 629 MB of bf16 expert "
                  "weights (126 MB L2)"}


def main():
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="full_b1", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--precision", default="bf16", choices=["bf16", "fp32"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-steps", type=int, default=3)
    # solver / convention variant (pi0x_set_variant); the default is pi0's own loop
    ap.add_argument("--time-grid", default="pi0", choices=["pi0", "linspace"])
    ap.add_argument("--x-prediction", action="store_true")
    ap.add_argument("--causal-actions", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = synth.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, wl)

    import torch
    from vla_flow_matching_b200 import build, pi0x

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    if rank == 0:
        build.build()
    if dist is not None:
        dist.barrier()

    precision = pi0x.PI0X_BF16 if args.precision == "bf16" else pi0x.PI0X_FP32
    inp = synth.make_inputs(wl)
    sampler = pi0x.Sampler(wl.dims, inp.weights, precision)
    sampler.set_variant(pi0x.PI0X_TIME_LINSPACE if args.time_grid == "linspace" else pi0x.PI0X_TIME_PI0,
                        args.x_prediction, args.causal_actions)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    pk = [dev(k.view(np.int16)) for k in inp.prefix_k]
    pv = [dev(v.view(np.int16)) for v in inp.prefix_v]
    mask, state, x1 = dev(inp.mask), dev(inp.state), dev(inp.x1)
    x0 = torch.empty_like(x1)
    stream = torch.cuda.current_stream()
    sid = stream.cuda_stream
    B, N = wl.batch, wl.num_steps

    def call():
        sampler.sample(pk, pv, mask, state, x1, N, x0=x0, stream=sid)

    for _ in range(args.warmup):
        call()
    sampler.sync()

    # ---- timed region: K whole calls, device-timed, max over ranks ----
    clk = sample_clocks_start() if rank == 0 else None
    time.sleep(0.3 if clk else 0)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        call()
    e1.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    clocks = sample_clocks_stop(clk, local) if clk else None
    sampler.sync()
    ms = slowest_rank_ms(e0.elapsed_time(e1), dist)
    ms_per = ms / args.steps
    value = job_throughput(world, B, args.steps, ms)
    if rank == 0:
        print(f"[bench] {wl.name} {args.precision}: {1000 * ms_per:.1f} us per call, "
              f"{value:.1f} {UNIT}", file=sys.stderr, flush=True)

    # ---- end to end through the public call with host buffers ----
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a)).pin_memory()
    hk = [pin(k.view(np.int16)) for k in inp.prefix_k]
    hv = [pin(v.view(np.int16)) for v in inp.prefix_v]
    hm, hs, hx = pin(inp.mask), pin(inp.state), pin(inp.x1)
    hx0 = torch.empty(inp.x1.shape, dtype=torch.float32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in hk + hv + [hm, hs, hx])
    d2h = hx0.numel() * 4
    e2e_steps = max(3, min(args.steps, 50))
    for _ in range(3):
        sampler.sample(hk, hv, hm, hs, hx, N, x0=hx0, stream=sid)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    e0.record(stream)
    for _ in range(e2e_steps):
        sampler.sample(hk, hv, hm, hs, hx, N, x0=hx0, stream=sid)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = slowest_rank_ms(e0.elapsed_time(e1), dist)
    e2e_value = job_throughput(world, B, e2e_steps, e2e_ms)

    # ---- per-kernel device time from the profiling graph (same workload) ----
    sampler.profile(True)
    acc = {}
    for _ in range(max(1, args.profile_steps)):
        call()
        for kname, (n, t) in sampler.profile_read().items():
            a = acc.setdefault(kname, [0, 0.0])
            a[0] += n
            a[1] += t
    sampler.profile(False)
    sampler.sync()
    if rank == 0:
        print("[bench] per-call kernel ms (launches): " + ", ".join(
            f"{k}={v[1] / max(1, args.profile_steps):.3f} ({v[0] // max(1, args.profile_steps)})"
            for k, v in acc.items()), file=sys.stderr, flush=True)

    roofline = None
    kernel_ms = {}
    if rank == 0:
        pk_, src = peaks()
        byt, flo, att = algorithmic_work(wl)
        n_g, t_g = acc["gemm"]
        t_g_per_call = t_g / max(1, args.profile_steps)
        kernel_ms = {k: round(v[1] / max(1, args.profile_steps), 4) for k, v in acc.items()}
        ridge = pk_["bf16_tflops"] * 1e12 / (pk_["hbm_gbs"] * 1e9)
        if flo / byt < ridge:
            achieved = byt / (t_g_per_call / 1000) / 1e9
            roofline = {"kernel": "k_gemm_tc (all expert and time-MLP Linears)", "bound": "hbm",
                        "achieved": achieved, "peak": pk_["hbm_gbs"], "unit": "GB/s",
                        "frac": achieved / pk_["hbm_gbs"], "traffic": None,
                        "peak_source": f"{src} hbm_gbs"}
        else:
            achieved = flo / (t_g_per_call / 1000) / 1e12
            peak = pk_.get("bf16_tflops_sustained", pk_["bf16_tflops"])
            roofline = {"kernel": "k_gemm_tc (all expert and time-MLP Linears)", "bound": "tensor",
                        "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                        "frac": achieved / peak, "traffic": None,
                        "peak_source": f"{src} bf16_tflops_sustained"}
        roofline["launches_per_call"] = n_g // max(1, args.profile_steps)
        roofline["algorithmic_per_call"] = {"gemm_bytes": byt, "gemm_flops": flo, "attn_flops": att}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, desc, cores = time_oracle(wl, variant=variant_of(args))
        cpu = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per, "us_per_chunk": 1000 * ms_per,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": args.precision, "data": "synthetic (seeded numpy PCG64, bf16-rounded N(0,0.02) "
                                               "weights, N(0,1) prefix K/V, state, noise)",
            "config": dict(config_of(wl, args), parallelism=f"replicas x{world} (batch per GPU fixed)"),
            "parallelism": f"replicas x{world} (batch per GPU fixed)",
            "gpu_launches": sampler.launch_count(B, wl.prefix_len, N) * args.steps,
            "clocks": clocks,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps},
            "roofline": roofline, "kernel_ms_per_call": kernel_ms, "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    sampler.close()
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
