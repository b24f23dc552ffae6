"""The seeded input module that the oracle and the CUDA path share."""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

from vla_flow_matching_b200 import synth


def test_bf16_rounding_matches_torch_round_to_nearest_even():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.normal(0, 1, 100000), rng.normal(0, 1e30, 1000), rng.normal(0, 1e-30, 1000),
        np.array([0.0, -0.0, 1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 3.3895314e38, -3.4e38, np.inf, -np.inf,
                  2.0 ** -130, -(2.0 ** -140)]),
    ]).astype(np.float32)
    ours = synth.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_bf16_rounding_keeps_nan():
    x = np.array([0x7FC00000, 0x7FFFFFFF, 0xFFFFFFFF, 0x7F800001], np.uint32).view(np.float32)
    back = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(x))
    assert np.all(np.isnan(back))
    assert np.signbit(back[2]) and not np.signbit(back[0])


def test_bf16_widening_is_exact():
    bits = np.arange(0, 1 << 16, 97, dtype=np.uint16)
    f = synth.bf16_bits_to_f32(bits)
    finite = np.isfinite(f)
    assert np.array_equal(synth.f32_to_bf16_bits(f[finite]), bits[finite])


def test_a_sample_regenerates_alone():
    """Sampled parity checks regenerate single samples of a big batch; every
    per-sample input must equal the same sample of the whole batch."""
    dims = dataclasses.replace(synth.ExpertDims(), depth=2, horizon=6)
    wl = synth.Workload("regen", dims, batch=5, prefix_len=40, num_steps=2, seed=21,
                        mask_kind="prefix_len", mask_a=20, mask_b=40)
    w = synth.make_weights(dims, wl.seed)
    full = synth.make_inputs(wl, weights=w)
    for b in (0, 3, 4):
        one = synth.make_inputs(wl, samples=[b], weights=w)
        assert np.array_equal(one.mask[0], full.mask[b])
        assert np.array_equal(one.state[0], full.state[b])
        assert np.array_equal(one.x1[0], full.x1[b])
        for l in range(dims.depth):
            assert np.array_equal(one.prefix_k[l][0], full.prefix_k[l][b])
            assert np.array_equal(one.prefix_v[l][0], full.prefix_v[l][b])
