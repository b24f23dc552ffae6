"""Parity of the CUDA path (through the C ABI) with the CPU oracle on seeded inputs.

Bars: bf16 mode max|dx0| <= 3e-2 and relative L2 <= 1e-2; fp32 mode max|dx0| <= 1e-4.
Full-size workloads are checked on sampled batch elements (samples are
independent, so the oracle runs only those), at the launch configuration the
benchmark times (the whole batch in one call).
"""
from __future__ import annotations

import dataclasses
import functools

import numpy as np
import pytest

from vla_flow_matching_b200 import synth

pytestmark = pytest.mark.gpu

BF16_MAX, BF16_REL, FP32_MAX = 3e-2, 1e-2, 1e-4


def _torch():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


@functools.lru_cache(maxsize=None)
def _sampler(dims, seed, precision):
    from vla_flow_matching_b200 import build, pi0x
    build.build()
    return pi0x.Sampler(dims, synth.make_weights(dims, seed), precision)


@functools.lru_cache(maxsize=4)
def _weights(dims, seed):
    return synth.make_weights(dims, seed)


def to_dev(inp):
    torch = _torch()
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    pk = [dev(k.view(np.int16)) for k in inp.prefix_k]
    pv = [dev(v.view(np.int16)) for v in inp.prefix_v]
    return pk, pv, dev(inp.mask), dev(inp.state), dev(inp.x1)


def run_gpu(sampler, inp, num_steps=None):
    torch = _torch()
    pk, pv, m, s, x1 = to_dev(inp)
    x0 = sampler.sample(pk, pv, m, s, x1, num_steps or inp.workload.num_steps)
    sampler.sync()
    torch.cuda.synchronize()
    return x0.cpu().numpy()


def oracle_x0(inp, weights=None, pk=None, pv=None):
    from oracle import pi0_oracle as O
    return O.sample_actions(weights or inp.weights, pk or inp.prefix_k, pv or inp.prefix_v, inp.mask,
                            inp.state, inp.x1, inp.workload.num_steps)


def check(gpu, ref, precision, what=""):
    d = np.abs(gpu.astype(np.float64) - ref.astype(np.float64))
    rel = np.linalg.norm(gpu - ref) / np.linalg.norm(ref)
    if precision == 1:
        assert d.max() <= FP32_MAX, f"{what} fp32 max|d|={d.max():.3g}"
    else:
        assert d.max() <= BF16_MAX and rel <= BF16_REL, f"{what} bf16 max|d|={d.max():.3g} rel={rel:.3g}"
    return float(d.max()), float(rel)


# ---- the five workloads --------------------------------------------------------------
@pytest.mark.parametrize("precision", [0, 1], ids=["bf16", "fp32"])
def test_tiny_workload(precision):
    wl = synth.WORKLOADS["tiny"]
    inp = synth.make_inputs(wl, weights=_weights(wl.dims, wl.seed))
    s = _sampler(wl.dims, wl.seed, precision)
    check(run_gpu(s, inp), oracle_x0(inp), precision, "tiny")


@pytest.mark.parametrize("precision", [0, 1], ids=["bf16", "fp32"])
def test_full_b1_workload(precision):
    wl = synth.WORKLOADS["full_b1"]
    inp = synth.make_inputs(wl, weights=_weights(wl.dims, wl.seed))
    s = _sampler(wl.dims, wl.seed, precision)
    check(run_gpu(s, inp), oracle_x0(inp), precision, "full_b1")


@pytest.mark.parametrize("precision", [0, 1], ids=["bf16", "fp32"])
def test_short_b8_workload(precision):
    wl = synth.WORKLOADS["short_b8"]
    inp = synth.make_inputs(wl, weights=_weights(wl.dims, wl.seed))
    s = _sampler(wl.dims, wl.seed, precision)
    check(run_gpu(s, inp), oracle_x0(inp), precision, "short_b8")


@pytest.mark.parametrize("name,samples", [("full_b32", [0, 13, 31]), ("full_b128", [0, 77, 127])])
@pytest.mark.parametrize("precision", [0, 1], ids=["bf16", "fp32"])
def test_full_batch_workloads_on_sampled_outputs(name, samples, precision):
    wl = synth.WORKLOADS[name]
    w = _weights(wl.dims, wl.seed)
    full = synth.make_inputs(wl, weights=w)
    s = _sampler(wl.dims, wl.seed, precision)
    gpu = run_gpu(s, full)
    sub = synth.make_inputs(wl, samples=samples, weights=w)
    ref = oracle_x0(sub)
    check(gpu[samples], ref, precision, name)
    # every output is finite and the full batch moved away from the noise
    assert np.isfinite(gpu).all()


# ---- invariants and edge cases on the GPU ---------------------------------------------
def small_wl(B=3, P=77, masked=0, horizon=50, depth=2, steps=3, kind="prefix_len", seed=21):
    dims = dataclasses.replace(synth.ExpertDims(), depth=depth, horizon=horizon)
    return synth.Workload("edge", dims, batch=B, prefix_len=P, num_steps=steps, seed=seed,
                          mask_kind=kind, mask_a=masked)


@pytest.mark.parametrize("precision", [0, 1], ids=["bf16", "fp32"])
def test_ragged_batch_and_prefix(precision):
    wl = small_wl(B=3, P=77, masked=40)          # valid lengths in [40, 77]
    inp = synth.make_inputs(wl)
    inp.mask[1, 5] = 0                           # a hole inside the valid prefix
    s = _sampler(wl.dims, wl.seed, precision)
    check(run_gpu(s, inp), oracle_x0(inp), precision, "ragged")


@pytest.mark.parametrize("precision", [0, 1], ids=["bf16", "fp32"])
def test_empty_prefix_and_all_masked_row(precision):
    wl = small_wl(B=2, P=0, kind="all")
    inp = synth.make_inputs(wl)
    s = _sampler(wl.dims, wl.seed, precision)
    check(run_gpu(s, inp), oracle_x0(inp), precision, "P=0")
    wl2 = small_wl(B=2, P=33, kind="all")
    inp2 = synth.make_inputs(wl2)
    inp2.mask[0, :] = 0
    check(run_gpu(s, inp2), oracle_x0(inp2), precision, "all-masked row")


@pytest.mark.parametrize("precision", [0, 1], ids=["bf16", "fp32"])
def test_zero_outproj_returns_noise_bitwise(precision):
    from vla_flow_matching_b200 import pi0x
    wl = small_wl(B=2, P=40)
    w = dict(synth.make_weights(wl.dims, wl.seed))
    w["action_out_w"] = np.zeros_like(w["action_out_w"])
    w["action_out_b"] = np.zeros_like(w["action_out_b"])
    s = pi0x.Sampler(wl.dims, w, precision)
    inp = synth.make_inputs(wl, weights=w)
    assert np.array_equal(run_gpu(s, inp), inp.x1)


@pytest.mark.parametrize("precision", [0, 1], ids=["bf16", "fp32"])
def test_bias_only_outproj(precision):
    from vla_flow_matching_b200 import pi0x
    wl = small_wl(B=2, P=40, steps=10)
    w = dict(synth.make_weights(wl.dims, wl.seed))
    w["action_out_w"] = np.zeros_like(w["action_out_w"])
    b = synth.f32_to_bf16_bits(np.linspace(-2, 2, 32).astype(np.float32))
    w["action_out_b"] = b
    s = pi0x.Sampler(wl.dims, w, precision)
    inp = synth.make_inputs(wl, weights=w)
    bf = synth.bf16_bits_to_f32(b)
    x = inp.x1.copy()
    dt = np.float32(-0.1)
    for _ in range(10):                  # x <- x + dt*b, fp32 rounding per step
        x = x + dt * bf
    assert np.array_equal(run_gpu(s, inp), x)
    assert np.allclose(x, inp.x1 - bf, atol=1e-5)


@pytest.mark.parametrize("precision", [0, 1], ids=["bf16", "fp32"])
def test_masked_prefix_values_are_never_read(precision):
    wl = small_wl(B=3, P=64, masked=30)
    inp = synth.make_inputs(wl)
    s = _sampler(wl.dims, wl.seed, precision)
    a = run_gpu(s, inp)
    rng = np.random.default_rng(5)
    for k in inp.prefix_k + inp.prefix_v:
        noise = synth.f32_to_bf16_bits(rng.normal(0, 100, k.shape).astype(np.float32))
        m = inp.mask[:, None, :, None].astype(bool)
        k[...] = np.where(m, k, noise)
    assert np.array_equal(run_gpu(s, inp), a)


def test_host_buffers_give_the_same_result():
    torch = _torch()
    wl = small_wl(B=2, P=50)
    inp = synth.make_inputs(wl)
    s = _sampler(wl.dims, wl.seed, 0)
    dev = run_gpu(s, inp)
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a)).pin_memory()
    x0 = torch.empty(inp.x1.shape, dtype=torch.float32).pin_memory()
    s.sample([pin(k.view(np.int16)) for k in inp.prefix_k], [pin(v.view(np.int16)) for v in inp.prefix_v],
             pin(inp.mask), pin(inp.state), pin(inp.x1), wl.num_steps, x0=x0)
    s.sync()
    assert np.array_equal(x0.numpy(), dev)
    # pageable numpy arrays too
    x0n = s.sample(inp.prefix_k, inp.prefix_v, inp.mask, inp.state, inp.x1, wl.num_steps)
    s.sync()
    assert np.array_equal(x0n, dev)


def test_x0_may_alias_x1_and_calls_repeat_bitwise():
    torch = _torch()
    wl = small_wl(B=2, P=50)
    inp = synth.make_inputs(wl)
    s = _sampler(wl.dims, wl.seed, 0)
    ref = run_gpu(s, inp)
    pk, pv, m, st, x1 = to_dev(inp)
    s.sample(pk, pv, m, st, x1, wl.num_steps, x0=x1)
    s.sync()
    assert np.array_equal(x1.cpu().numpy(), ref)


def test_invalid_arguments_return_status():
    from vla_flow_matching_b200 import pi0x
    wl = small_wl(B=1, P=8)
    inp = synth.make_inputs(wl)
    s = _sampler(wl.dims, wl.seed, 0)
    with pytest.raises(pi0x.Pi0xError) as e:
        s.sample(inp.prefix_k, inp.prefix_v, inp.mask, inp.state, inp.x1, 0)
    assert e.value.status == pi0x.PI0X_EINVAL
