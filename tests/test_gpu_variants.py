"""Solver / convention variants through the C ABI against the oracle.

The variants are the Wall-X sampler's conventions (``pi0x_set_variant``): the time
grid 0 -> 1 on linspace, x-prediction (velocity = prediction - noise) and the
causal action mask.  Same bars as the default loop: bf16 mode max|dx0| <= 3e-2 and
relative L2 <= 1e-2, fp32 mode max|dx0| <= 1e-4.
"""
from __future__ import annotations

import dataclasses

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


def run_gpu(sampler, inp):
    torch = _torch()
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    pk = [dev(k.view(np.int16)) for k in inp.prefix_k]
    pv = [dev(v.view(np.int16)) for v in inp.prefix_v]
    x0 = sampler.sample(pk, pv, dev(inp.mask), dev(inp.state), dev(inp.x1), inp.workload.num_steps)
    sampler.sync()
    torch.cuda.synchronize()
    return x0.cpu().numpy()


def check(gpu, ref, precision, what=""):
    d = np.abs(gpu.astype(np.float64) - ref.astype(np.float64))
    rel = np.linalg.norm(gpu - ref) / np.linalg.norm(ref)
    if precision == 1:
        assert d.max() <= FP32_MAX, f"{what} fp32 max|d|={d.max():.3g}"
    else:
        assert d.max() <= BF16_MAX and rel <= BF16_REL, f"{what} bf16 max|d|={d.max():.3g} rel={rel:.3g}"

VARIANTS = {
    "linspace": dict(time_convention="linspace"),
    "x_pred": dict(x_prediction=True),
    "causal": dict(causal_actions=True),
    "all": dict(time_convention="linspace", x_prediction=True, causal_actions=True),
}


def _sampler(wl, precision, variant):
    from vla_flow_matching_b200 import build, pi0x
    _torch()
    build.build()
    s = pi0x.Sampler(wl.dims, synth.make_weights(wl.dims, wl.seed), precision)
    s.set_variant(pi0x.PI0X_TIME_LINSPACE if variant.get("time_convention") == "linspace" else pi0x.PI0X_TIME_PI0,
                  variant.get("x_prediction", False), variant.get("causal_actions", False))
    return s


def _oracle(inp, variant):
    from oracle import pi0_oracle as O
    return O.sample_actions(inp.weights, inp.prefix_k, inp.prefix_v, inp.mask, inp.state, inp.x1,
                            inp.workload.num_steps, **variant)


@pytest.mark.parametrize("precision", [0, 1], ids=["bf16", "fp32"])
@pytest.mark.parametrize("name", sorted(VARIANTS))
def test_tiny_workload_variants(name, precision):
    wl = synth.WORKLOADS["tiny"]
    inp = synth.make_inputs(wl)
    s = _sampler(wl, precision, VARIANTS[name])
    check(run_gpu(s, inp), _oracle(inp, VARIANTS[name]), precision, f"tiny {name}")
    s.close()


# Full size in bf16: the combinations whose x_0 is the noise plus the integrated
# velocity, like the pi0 loop's.  With x-prediction on the 0 -> 1 grid x_0 is the
# average of the network's predictions, so the relative L2 measures the bf16 network
# error itself (1.4 % on full_b1, max|dx0| 0.009): that combination is held to the
# fp32 bar in fp32 mode and to max|dx0| (2 % relative guard) in bf16 below.
BF16_FULL = {
    "full_b1": dict(time_convention="linspace", causal_actions=True),
    "short_b8": dict(x_prediction=True, causal_actions=True),
}


@pytest.mark.parametrize("workload", sorted(BF16_FULL))
def test_full_size_variants_bf16(workload):
    wl = synth.WORKLOADS[workload]
    inp = synth.make_inputs(wl)
    s = _sampler(wl, 0, BF16_FULL[workload])
    check(run_gpu(s, inp), _oracle(inp, BF16_FULL[workload]), 0, f"{workload} {BF16_FULL[workload]}")
    s.close()


def test_full_size_all_variants_fp32():
    wl = synth.WORKLOADS["short_b8"]
    inp = synth.make_inputs(wl)
    s = _sampler(wl, 1, VARIANTS["all"])
    check(run_gpu(s, inp), _oracle(inp, VARIANTS["all"]), 1, "short_b8 all variants")
    s.close()


def test_x_prediction_linspace_full_b1_fp32():
    """Linspace grid + x-prediction + causal mask at full_b1 in fp32 mode, held to the
    fp32 bar.  Same kernels and control flow as the bf16 run below, so a pass here
    says the bf16 relative-L2 excess is bf16 rounding of the network, not a logic error."""
    wl = synth.WORKLOADS["full_b1"]
    inp = synth.make_inputs(wl)
    s = _sampler(wl, 1, VARIANTS["all"])
    check(run_gpu(s, inp), _oracle(inp, VARIANTS["all"]), 1, "full_b1 all variants")
    s.close()


def test_x_prediction_linspace_full_b1_bf16_max_error():
    """The x-prediction / 0 -> 1 combination at full size in bf16, held to the max|dx0|
    bar with a 2 % relative-L2 guard: with x-prediction on the 0 -> 1 grid the noise
    cancels (the step sizes sum to 1), so x_0 is the average of the network's
    predictions rather than the noise plus a small correction, and its relative L2
    measures the bf16 error of the network itself (1.4 % measured).
    The fp32 run of the same combination above meets the 1e-4 bar, which rules out a
    logic error."""
    wl = synth.WORKLOADS["full_b1"]
    inp = synth.make_inputs(wl)
    s = _sampler(wl, 0, VARIANTS["all"])
    gpu, ref = run_gpu(s, inp), _oracle(inp, VARIANTS["all"])
    d = np.abs(gpu.astype(np.float64) - ref)
    rel = np.linalg.norm(gpu - ref) / np.linalg.norm(ref)
    assert d.max() <= BF16_MAX and rel <= 2e-2, f"max|d|={d.max():.3g} rel={rel:.3g}"
    s.close()


@pytest.mark.parametrize("precision", [0, 1], ids=["bf16", "fp32"])
def test_causal_first_action_ignores_later_noise(precision):
    """Under the causal mask action 0's trajectory does not depend on the other
    actions' noise (row-independent GEMMs, deterministic reductions: bitwise)."""
    wl = synth.WORKLOADS["tiny"]
    inp = synth.make_inputs(wl)
    s = _sampler(wl, precision, VARIANTS["causal"])
    a = run_gpu(s, inp)
    x1b = inp.x1.copy()
    x1b[:, 1:] += np.float32(0.5)
    b = run_gpu(s, dataclasses.replace(inp, x1=x1b))
    assert np.array_equal(a[:, 0], b[:, 0])
    assert np.max(np.abs(a[:, 1:] - b[:, 1:])) > 1e-3
    s.close()


def test_switching_back_restores_the_default_loop():
    from vla_flow_matching_b200 import pi0x
    wl = synth.WORKLOADS["tiny"]
    inp = synth.make_inputs(wl)
    s = _sampler(wl, 0, {})
    base = run_gpu(s, inp)
    s.set_variant(pi0x.PI0X_TIME_LINSPACE, True, True)
    other = run_gpu(s, inp)
    assert np.max(np.abs(other - base)) > 1e-2
    s.set_variant(pi0x.PI0X_TIME_PI0, False, False)
    assert np.array_equal(run_gpu(s, inp), base)
    with pytest.raises(pi0x.Pi0xError):
        s.set_variant(7, False, False)
    s.close()
