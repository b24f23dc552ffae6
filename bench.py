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


def hbm_bytes(wl):
    """Compulsory HBM bytes of one call: every weight of the expert and of the
    suffix embedding / out-projection read once per Euler step (bf16 matrices; the
    fp32 out-projection, biases and norm gains), plus the valid prefix K/V of every
    layer read once per step."""
    d, N = wl.dims, wl.num_steps
    W, F, Q, Dh, L, A = d.width, d.mlp_dim, d.num_heads * d.head_dim, d.head_dim, d.depth, d.action_dim
    per_layer = 2 * (W * (Q + 2 * Dh) + W * Q + 2 * F * W + W * F) + 4 * 2 * W
    embed = 2 * (W * A + 2 * W * W + W * W) + 4 * (4 * W) + 4 * (A * W + A + W)
    n = synth.make_mask(wl).sum(axis=1).astype(np.int64)
    kv = int(n.sum()) * L * Dh * 2 * 2
    return N * (L * per_layer + embed + kv)


def roofline_of(wl, kernel_ms, call_ms):
    """Roofline of the kernel class with the most device time.

    The class's time per call is its share of the profiled (serialised, one event
    pair per kernel) device time times the graph-timed call, so it can never exceed
    the call.  Work per call is algorithmic: the loop kernel (every step of a small
    batch) moves the call's compulsory HBM bytes and runs all of its FLOPs; the GEMM
    class moves its weights and operands (``algorithmic_work``)."""
    pk_, src = peaks()
    total = sum(kernel_ms.values())
    dom = max(kernel_ms, key=kernel_ms.get)
    t_ms = call_ms * kernel_ms[dom] / total
    gbytes, gflops, aflops = algorithmic_work(wl)
    if dom == "loop":
        byt, flo, name = hbm_bytes(wl), gflops + aflops, "k_loop (persistent: every Euler step of the call)"
    elif dom == "attn":
        n = synth.make_mask(wl).sum(axis=1).astype(np.int64)
        byt = int(n.sum()) * wl.dims.depth * wl.dims.head_dim * 4 * wl.num_steps
        flo, name = aflops, "k_attn_tc (masked MQA attention)"
    else:
        byt, flo, name = gbytes, gflops, "k_gemm_tc (all expert and time-MLP Linears)"
    ridge = pk_["bf16_tflops"] * 1e12 / (pk_["hbm_gbs"] * 1e9)
    if flo / byt < ridge:
        bound, peak, unit, psrc = "hbm", pk_["hbm_gbs"], "GB/s", f"{src} hbm_gbs"
        ach, whole = byt / (t_ms / 1e3) / 1e9, hbm_bytes(wl) / (call_ms / 1e3) / 1e9
    else:
        bound, unit, psrc = "tensor", "TFLOP/s", f"{src} bf16_tflops_sustained"
        peak = pk_.get("bf16_tflops_sustained", pk_["bf16_tflops"])
        ach, whole = flo / (t_ms / 1e3) / 1e12, (gflops + aflops) / (call_ms / 1e3) / 1e12
    traffic = TRAFFIC.get((wl.name, dom))
    return {"kernel": name, "bound": bound, "achieved": ach, "peak": peak, "unit": unit, "frac": ach / peak,
            "traffic": traffic, "peak_source": psrc, "kernel_ms_per_call": t_ms,
            "kernel_share_of_profile": kernel_ms[dom] / total,
            "whole_call": {"achieved": whole, "frac": whole / peak},
            "algorithmic_per_call": {"bytes": byt, "flops": flo, "hbm_bytes": hbm_bytes(wl),
                                     "gemm_bytes": gbytes, "gemm_flops": gflops, "attn_flops": aflops}}


# DRAM bytes (read + write) per launch of the dominant kernel from an ncu capture of
# the same build, keyed by (workload, kernel class); None when not captured.  full_b1:
# k_loop over one Euler step (the full_b1_1step profiling case) read 734,413,056 B and
# wrote 12,787,968 B; every step streams all weights (629 MB, more than L2), so the
# ten-step launch moves ten times that.
TRAFFIC = {("full_b1", "loop"): 10 * (709838336 + 7940096)}


def measure(wl, args, sampler, inp, rank, dist, clocks_on):
    """Device-timed throughput of whole calls on one workload (inputs resident)."""
    import torch
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    pk = [dev(k.view(np.int16)) for k in inp.prefix_k]
    pv = [dev(v.view(np.int16)) for v in inp.prefix_v]
    mask, state, x1 = dev(inp.mask), dev(inp.state), dev(inp.x1)
    x0 = torch.empty_like(x1)
    stream = torch.cuda.current_stream()
    sid = stream.cuda_stream
    N = wl.num_steps
    steps = args.steps if wl.name == args.workload else max(5, min(args.steps, 20))

    def call():
        sampler.sample(pk, pv, mask, state, x1, N, x0=x0, stream=sid)

    for _ in range(args.warmup):
        call()
    sampler.sync()
    clk = sample_clocks_start() if (rank == 0 and clocks_on) else None
    time.sleep(0.3 if clk else 0)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        call()
    e1.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    clocks = sample_clocks_stop(clk, int(os.environ.get("LOCAL_RANK", "0"))) if clk else None
    sampler.sync()
    ms = slowest_rank_ms(e0.elapsed_time(e1), dist)
    # per-kernel-class device time of the same call shape (serialised profile)
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
    ps = max(1, args.profile_steps)
    kernel_ms = {k: v[1] / ps for k, v in acc.items() if v[0] > 0}
    launches = {k: v[0] // ps for k, v in acc.items() if v[0] > 0}
    out = {"ms": ms, "steps": steps, "clocks": clocks, "kernel_ms": kernel_ms, "launches": launches,
           "tensors": (pk, pv, mask, state, x1, x0, sid)}
    return out


def main():
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="full_b1",
                    choices=sorted(synth.WORKLOADS) + sorted(synth.PROFILE_WORKLOADS))
    ap.add_argument("--precision", default="bf16", choices=["bf16", "fp32"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-by-workload", action="store_true",
                    help="skip the per-workload lines (short_b8, full_b32, full_b128) of a 1-GPU run")
    ap.add_argument("--profile-steps", type=int, default=3)
    # solver / convention variant (pi0x_set_variant); the default is pi0's own loop
    ap.add_argument("--time-grid", default="pi0", choices=["pi0", "linspace"])
    ap.add_argument("--x-prediction", action="store_true")
    ap.add_argument("--causal-actions", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.gpus != world:
        print(f"bench.py: --gpus {args.gpus} needs {args.gpus} ranks (WORLD_SIZE={world}); launch it with "
              f"python -m torch.distributed.run --nproc-per-node {args.gpus} bench.py --gpus {args.gpus}",
              file=sys.stderr)
        return 2
    wl = {**synth.WORKLOADS, **synth.PROFILE_WORKLOADS}[args.workload]
    if args.impl == "reference":
        return run_reference(args, wl)

    import torch
    from vla_flow_matching_b200 import build, pi0x

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
    variant = (pi0x.PI0X_TIME_LINSPACE if args.time_grid == "linspace" else pi0x.PI0X_TIME_PI0,
               args.x_prediction, args.causal_actions)

    def sampler_for(w, inp):
        s = pi0x.Sampler(w.dims, inp.weights, precision)
        s.set_variant(*variant)
        return s

    inp = synth.make_inputs(wl)
    sampler = sampler_for(wl, inp)
    B, N = wl.batch, wl.num_steps
    r = measure(wl, args, sampler, inp, rank, dist, clocks_on=True)
    ms, steps = r["ms"], r["steps"]
    ms_per = ms / steps
    value = job_throughput(world, B, steps, ms)
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
    sid = r["tensors"][-1]
    stream = torch.cuda.current_stream()
    e2e_steps = max(3, min(args.steps, 50))
    for _ in range(3):
        sampler.sample(hk, hv, hm, hs, hx, N, x0=hx0, stream=sid)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        sampler.sample(hk, hv, hm, hs, hx, N, x0=hx0, stream=sid)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = slowest_rank_ms(e0.elapsed_time(e1), dist)
    e2e_value = job_throughput(world, B, e2e_steps, e2e_ms)
    sampler.sync()
    if rank == 0:
        print("[bench] per-call kernel ms (launches): " + ", ".join(
            f"{k}={v:.3f} ({r['launches'][k]})" for k, v in r["kernel_ms"].items()), file=sys.stderr, flush=True)
    launches_per_call = sampler.launch_count(B, wl.prefix_len, N)
    roof = roofline_of(wl, r["kernel_ms"], ms_per) if rank == 0 else None
    clocks = r["clocks"]
    del r
    sampler.close()

    # ---- the other workloads of the metric (B = 8, 32, 128), device-timed, 1 GPU ----
    by_workload = {}
    if world == 1 and not args.no_by_workload and args.workload == "full_b1":
        for name in ("short_b8", "full_b32", "full_b128"):
            w2 = synth.WORKLOADS[name]
            inp2 = synth.make_inputs(w2)
            s2 = sampler_for(w2, inp2)
            r2 = measure(w2, args, s2, inp2, rank, None, clocks_on=True)
            mp = r2["ms"] / r2["steps"]
            by_workload[name] = {
                "batch": w2.batch, "prefix_len": w2.prefix_len, "num_steps": w2.num_steps,
                "horizon": w2.dims.horizon, "value": w2.batch * r2["steps"] / (r2["ms"] / 1000.0), "unit": UNIT,
                "ms_per_step": mp, "us_per_chunk": 1000 * mp, "steps": r2["steps"],
                "gpu_launches": s2.launch_count(w2.batch, w2.prefix_len, w2.num_steps) * r2["steps"],
                "clocks": r2["clocks"], "roofline": roofline_of(w2, r2["kernel_ms"], mp),
                "profiled_kernel_ms_per_call": {k: round(v, 4) for k, v in r2["kernel_ms"].items()},
            }
            print(f"[bench] {name}: {1000 * mp:.1f} us per call, "
                  f"{by_workload[name]['value']:.1f} {UNIT}", file=sys.stderr, flush=True)
            del r2, inp2
            s2.close()
            torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, desc, cores = time_oracle(wl, variant=variant_of(args))
        cpu = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": steps,
            "warmup": args.warmup, "ms_per_step": ms_per, "us_per_chunk": 1000 * ms_per,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": args.precision, "data": "synthetic (seeded numpy PCG64, bf16-rounded N(0,0.02) "
                                               "weights, N(0,1) prefix K/V, state, noise)",
            "config": dict(config_of(wl, args), parallelism=f"replicas x{world} (batch per GPU fixed)"),
            "parallelism": f"replicas x{world} (batch per GPU fixed)",
            "gpu_launches": launches_per_call * steps,
            "clocks": clocks,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps},
            "roofline": roof, "cpu_baseline": cpu, "by_workload": by_workload or None,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
