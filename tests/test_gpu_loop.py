"""The persistent small-batch loop kernel (bf16 mode, B * (horizon + 1) <= 128).

Small batches run every Euler step in one cooperative kernel; larger batches take
the multi-kernel path.  The default-path parity tests already hold the small
workloads to the oracle bars; here the loop is also compared with the multi-kernel
path on the same inputs, checked for run-to-run determinism (every cross-CTA
reduction adds in a fixed order), and driven through its failure path: a stage
that waits on a done-counter nothing raises must end the call with PI0X_ETIMEOUT,
leave the context usable, and the next call must reproduce the reference result
bit for bit.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import pytest

from tests.test_gpu_parity import BF16_MAX, _torch, check, oracle_x0, run_gpu, small_wl, to_dev
from vla_flow_matching_b200 import synth

pytestmark = pytest.mark.gpu


def _sampler(dims, seed):
    from vla_flow_matching_b200 import build, pi0x
    _torch()
    build.build()
    s = pi0x.Sampler(dims, synth.make_weights(dims, seed), pi0x.PI0X_BF16)
    assert s.uses_loop(1), pi0x.load().pi0x_last_error().decode()
    return s


@pytest.mark.parametrize("name", ["tiny", "full_b1", "short_b8"])
def test_loop_matches_oracle_multi_kernel_path_and_itself(name):
    wl = synth.WORKLOADS[name]
    inp = synth.make_inputs(wl)
    s = _sampler(wl.dims, wl.seed)
    assert s.uses_loop(wl.batch)
    a = run_gpu(s, inp)
    assert np.array_equal(run_gpu(s, inp), a), "the loop kernel is not deterministic"
    check(a, oracle_x0(inp), 0, f"{name} loop")
    s.debug_set_loop(False)
    assert not s.uses_loop(wl.batch)
    b = run_gpu(s, inp)
    assert np.abs(a.astype(np.float64) - b).max() <= BF16_MAX
    s.debug_set_loop(True)
    assert np.array_equal(run_gpu(s, inp), a)
    s.close()


def test_only_batches_that_fit_one_tile_use_the_loop():
    dims = dataclasses.replace(synth.ExpertDims(), depth=1)
    s = _sampler(dims, 3)
    assert s.uses_loop(1) and s.uses_loop(2)          # 51 and 102 rows
    assert not s.uses_loop(3) and not s.uses_loop(32)  # 153 and 1632 rows
    assert s.launch_count(1, 816, 10) == 6
    assert s.launch_count(32, 816, 10) > 50       # one kernel per projection, attention, small step
    s.close()


@pytest.mark.parametrize("masked,hole", [(0, False), (30, True)])
def test_loop_two_samples_ragged_prefix(masked, hole):
    wl = small_wl(B=2, P=70, masked=masked, steps=3)
    inp = synth.make_inputs(wl)
    if hole:
        inp.mask[0, 4] = 0
    s = _sampler(wl.dims, wl.seed)
    assert s.uses_loop(2)
    check(run_gpu(s, inp), oracle_x0(inp), 0, "B=2 loop")
    s.close()


def test_loop_full_128_row_tile():
    """B=2 at horizon 63: 128 rows, the largest tile the loop takes (N = 128 tokens per
    MMA, two accumulator chains per GEMM unit, an 8-slot activation ring, the largest
    split-K slices); against the oracle, the multi-kernel path and itself."""
    wl = small_wl(B=2, P=40, masked=20, horizon=63, depth=2, steps=2)
    inp = synth.make_inputs(wl)
    s = _sampler(wl.dims, wl.seed)
    assert s.uses_loop(2) and not s.uses_loop(3)
    a = run_gpu(s, inp)
    assert np.array_equal(run_gpu(s, inp), a)
    check(a, oracle_x0(inp), 0, "128-row loop")
    s.debug_set_loop(False)
    b = run_gpu(s, inp)
    assert np.abs(a.astype(np.float64) - b).max() <= BF16_MAX
    s.close()


def test_loop_empty_prefix():
    """No prefix keys at all: attention over the suffix only (state and action keys)."""
    wl = small_wl(B=1, P=0, kind="all", depth=2, steps=2)
    inp = synth.make_inputs(wl)
    s = _sampler(wl.dims, wl.seed)
    assert s.uses_loop(1)
    check(run_gpu(s, inp), oracle_x0(inp), 0, "P=0 loop")
    s.close()


def test_loop_four_ragged_samples_short_horizon():
    """B=4 at horizon 20 (84 rows, N = 96 tokens): ragged valid prefixes per sample."""
    wl = small_wl(B=4, P=90, masked=35, horizon=20, depth=2, steps=3)
    inp = synth.make_inputs(wl)
    s = _sampler(wl.dims, wl.seed)
    assert s.uses_loop(4)
    check(run_gpu(s, inp), oracle_x0(inp), 0, "B=4 loop")
    s.close()


@pytest.mark.parametrize("stage", [1, 9], ids=["step0_mlp_out", "step0_layer1"])
def test_stalled_stage_times_out_and_next_call_is_exact(stage):
    """Stage 1 is the action-time MLP output GEMM of step 0; stage 9 lies in layer 1
    of step 0, so layer 0's units and every CTA's later waits are in flight when the
    error word is raised."""
    from vla_flow_matching_b200 import pi0x
    torch = _torch()
    wl = small_wl(B=1, P=77, steps=2, depth=2)
    inp = synth.make_inputs(wl)
    s = _sampler(wl.dims, wl.seed)
    assert s.uses_loop(1)
    ref = run_gpu(s, inp)
    s.debug_loop_stall(stage, 20_000_000)   # 20 ms limit for that call
    pk, pv, m, st, x1 = to_dev(inp)
    s.sample(pk, pv, m, st, x1, wl.num_steps)
    with pytest.raises(pi0x.Pi0xError) as e:
        s.sync()
    assert e.value.status == pi0x.PI0X_ETIMEOUT
    torch.cuda.synchronize()
    for _ in range(2):
        assert np.array_equal(run_gpu(s, inp), ref)
    s.close()
