"""Pins of the CPU oracle against facts fixed by the pages and by mathematics.

Each pin is independent of the oracle's own code: closed forms, invariants,
special cases that reduce to a library routine (torch / transformers on CPU),
hand-computed values and a float64 brute force written separately
(``tests/brute_f64.py``).  ``test_planted_mistakes_are_caught`` plants plausible
mistakes into the oracle (on the CPU) and checks that a pin fails for each.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import pytest
import torch

from oracle import pi0_oracle as O
from tests.brute_f64 import brute_sample
from vla_flow_matching_b200 import synth


# --- helpers -------------------------------------------------------------------
def tiny_float_inputs(dims, B=2, P=5, n_masked=(1, 3), std=0.3, seed=11, steps=2):
    """Random float64 inputs at tiny dims (weights large enough that every term matters)."""
    rng = np.random.default_rng(seed)
    shapes = synth.weight_shapes(dims)
    w = {k: rng.normal(0, std, shapes[k]) for k in synth.WEIGHT_ORDER + synth.TAIL_ORDER}
    w["layers"] = [{k: rng.normal(0, std, shapes[k]) for k in synth.LAYER_ORDER}
                   for _ in range(dims.depth)]
    kv = (dims.num_kv_heads, P, dims.head_dim)
    pk = [rng.normal(0, 1, (B,) + kv) for _ in range(dims.depth)]
    pv = [rng.normal(0, 1, (B,) + kv) for _ in range(dims.depth)]
    mask = np.ones((B, P), np.uint8)
    for b in range(B):
        if n_masked[b % len(n_masked)]:
            mask[b, -n_masked[b % len(n_masked)]:] = 0
    mask[0, 1] = 0   # a hole inside the prefix, not only tail padding
    state = rng.normal(0, 1, (B, dims.state_dim))
    x1 = rng.normal(0, 1, (B, dims.horizon, dims.action_dim))
    return w, pk, pv, mask, state, x1, steps


def full_width_small(depth=2, B=1, P=64, masked=10, horizon=50):
    wl = synth.Workload("pin", dataclasses.replace(synth.ExpertDims(), depth=depth, horizon=horizon),
                        batch=B, prefix_len=P, num_steps=2, seed=7,
                        mask_kind="tail_pad" if masked else "all", mask_a=masked)
    return synth.make_inputs(wl)


def run_oracle(inp, dtype=np.float32, weights=None, pk=None, pv=None, **variant):
    return O.sample_actions(weights if weights is not None else inp.weights,
                            pk if pk is not None else inp.prefix_k,
                            pv if pv is not None else inp.prefix_v,
                            inp.mask, inp.state, inp.x1, inp.workload.num_steps, dtype=dtype, **variant)


# --- timestep embedding ----------------------------------------------------------
def test_time_embedding_closed_forms():
    W = 1024
    e0 = O.time_embedding(np.array([0.0]), W)[0]
    assert np.array_equal(e0[:512], np.zeros(512)) and np.array_equal(e0[512:], np.ones(512))
    # t = 1: the fastest period is 0.004 -> angle 500*pi; the slowest is 4 -> pi/2.
    e1 = O.time_embedding(np.array([1.0]), W)[0]
    assert abs(e1[0] - math.sin(500 * math.pi)) < 1e-12 and abs(e1[512] - 1.0) < 1e-12
    assert abs(e1[511] - 1.0) < 1e-15 and abs(e1[1023]) < 1e-15
    # t = 0.5: slowest angle pi/4
    e5 = O.time_embedding(np.array([0.5]), W)[0]
    assert abs(e5[511] - math.sqrt(0.5)) < 1e-15 and abs(e5[1023] - math.sqrt(0.5)) < 1e-15
    # small t: no wrap-around, so angles follow a geometric sweep with ratio 1000^(1/511)
    t = 1e-5
    e = O.time_embedding(np.array([t]), W)[0]
    ang = np.arctan2(e[:512], e[512:])
    assert abs(ang[0] - 2 * math.pi * t / 0.004) < 1e-13
    ratio = ang[:-1] / ang[1:]
    assert np.allclose(ratio, 1000.0 ** (1.0 / 511), rtol=1e-9)


def test_time_embedding_rejects_odd_dim():
    with pytest.raises(ValueError):
        O.time_embedding(np.array([0.5]), 7)


# --- RoPE ------------------------------------------------------------------------
def test_rope_hand_example_and_identity():
    # head_dim 4, theta 1e4: inverse frequencies [1, 0.01]; x = e_0 at position 1
    x = np.array([[[1.0, 0.0, 0.0, 0.0]]])             # (T=1, heads=1, D=4)
    out = O.apply_rope(x, np.array([1]), np.float64)[0, 0]
    assert np.allclose(out, [math.cos(1.0), 0.0, math.sin(1.0), 0.0], atol=1e-15)
    y = np.array([[[0.0, 1.0, 0.0, 0.0]]])
    out = O.apply_rope(y, np.array([3]), np.float64)[0, 0]
    assert np.allclose(out, [0.0, math.cos(0.03), 0.0, math.sin(0.03)], atol=1e-15)
    r = np.random.default_rng(0).normal(size=(5, 2, 256))
    assert np.array_equal(O.apply_rope(r, np.zeros(5, np.int64), np.float64), r)


def test_rope_relative_position_invariance():
    rng = np.random.default_rng(1)
    q = rng.normal(size=(1, 1, 256))
    k = rng.normal(size=(1, 1, 256))
    dots = []
    for m, n in [(10, 3), (507, 500), (870, 863)]:
        qm = O.apply_rope(q, np.array([m]), np.float64)[0, 0]
        kn = O.apply_rope(k, np.array([n]), np.float64)[0, 0]
        dots.append(qm @ kn)
    assert np.allclose(dots, dots[0], rtol=1e-9)


def test_rope_matches_transformers():
    from transformers import GemmaConfig
    from transformers.models.gemma.modeling_gemma import GemmaRotaryEmbedding, apply_rotary_pos_emb
    cfg = GemmaConfig(head_dim=256, hidden_size=1024, num_attention_heads=8,
                      num_key_value_heads=1, hidden_activation="gelu_pytorch_tanh")
    rot = GemmaRotaryEmbedding(cfg)
    rng = np.random.default_rng(2)
    q = rng.normal(size=(1, 8, 6, 256)).astype(np.float32)
    k = rng.normal(size=(1, 1, 6, 256)).astype(np.float32)
    pos = np.array([[0, 1, 300, 806, 857, 900]])
    cos, sin = rot(torch.from_numpy(q), torch.from_numpy(pos))
    qt, kt = apply_rotary_pos_emb(torch.from_numpy(q), torch.from_numpy(k), cos, sin)
    qo = O.apply_rope(q[0].transpose(1, 0, 2), pos[0], np.float32).transpose(1, 0, 2)
    ko = O.apply_rope(k[0].transpose(1, 0, 2), pos[0], np.float32).transpose(1, 0, 2)
    # float32 angles: a 1-ulp difference in an inverse frequency moves the angle
    # by pos * 2^-24 and rounding the angle adds ulp(angle)/2, so the bound grows
    # with the position; at positions 0 and 1 the two must agree to rounding.
    ang_err = pos[0] * 2.0 ** -23 + np.spacing(np.float32(pos[0])) * 2.0 + 1e-7
    bound = (np.abs(q[0]).max() * 2 * ang_err)[None, :, None] + 1e-6
    assert np.all(np.abs(qo - qt[0].numpy()) <= bound)
    assert np.all(np.abs(ko - kt[0].numpy()) <= (np.abs(k[0]).max() * 2 * ang_err)[None, :, None] + 1e-6)
    assert np.allclose(qo[:, :2], qt[0].numpy()[:, :2], atol=1e-6)


# --- bf16 widening of weights and prefix K/V -------------------------------------
def _torch_bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """torch's own bf16 -> float32 conversion of uint16 bit patterns."""
    return torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).float().numpy()


def _widening_agrees_with_torch(widen) -> bool:
    """Every one of the 65536 bf16 bit patterns widens to torch's float32 value,
    bit for bit (so +0 / -0, subnormals and infinities too); NaN patterns stay NaN."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = _torch_bf16_to_f32(bits)
    with np.errstate(invalid="ignore"):   # signalling-NaN patterns
        got = np.asarray(widen(bits, np.float32))
        wide = np.asarray(widen(bits, np.float64))
    if got.dtype != np.float32 or got.shape != ref.shape:
        return False
    nan = np.isnan(ref)
    if not np.array_equal(np.isnan(got), nan):
        return False
    if not np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32)):
        return False
    return wide.dtype == np.float64 and np.array_equal(wide[~nan], ref[~nan].astype(np.float64))


def test_bf16_widening_matches_torch_on_every_bit_pattern():
    # the vllm-omni page casts the bf16 prefix cache to the expert's dtype before the
    # attention (`_compute_layer_suffix_only`); weights enter the float32 model the same way
    assert _widening_agrees_with_torch(O.as_float)
    f = np.array([1.5, -2.25], np.float32)
    assert O.as_float(f, np.float64).dtype == np.float64 and np.array_equal(O.as_float(f, np.float32), f)


@pytest.mark.parametrize("mutant", ["int16_value", "no_shift", "shift_15", "byteswap"])
def test_bf16_widening_pin_catches_planted_mistakes(mutant):
    """Plausible widening mistakes, each of which the pin above must reject."""
    def int16_value(a, dtype):          # sign-extending int16 view taken as a number
        return np.asarray(a).view(np.int16).astype(dtype)

    def no_shift(a, dtype):             # bits placed in the low half of the float32
        return np.asarray(a).astype(np.uint32).view(np.float32).astype(dtype)

    def shift_15(a, dtype):
        return (np.asarray(a).astype(np.uint32) << np.uint32(15)).view(np.float32).astype(dtype)

    def byteswap(a, dtype):
        return (np.asarray(a).byteswap().astype(np.uint32) << np.uint32(16)).view(np.float32).astype(dtype)

    fn = {"int16_value": int16_value, "no_shift": no_shift, "shift_15": shift_15, "byteswap": byteswap}[mutant]
    assert not _widening_agrees_with_torch(fn)


def test_convert_weights_widens_every_array():
    dims = dataclasses.replace(synth.ExpertDims(), depth=2)
    w = synth.make_weights(dims, seed=5)
    for dtype in (np.float32, np.float64):
        c = O.convert_weights(w, dtype)
        assert set(c) == set(w)
        assert len(c["layers"]) == len(w["layers"])
        pairs = [(c[k], w[k]) for k in w if k != "layers"]
        pairs += [(cl[k], wl[k]) for cl, wl in zip(c["layers"], w["layers"]) for k in wl]
        assert len(pairs) == len(synth.WEIGHT_ORDER + synth.TAIL_ORDER) + 2 * len(synth.LAYER_ORDER)
        for got, bits in pairs:
            assert bits.dtype == np.uint16 and got.dtype == dtype and got.shape == bits.shape
            assert np.array_equal(got, _torch_bf16_to_f32(bits).astype(dtype))


# --- RMSNorm, activations ----------------------------------------------------------
def test_rms_norm_unit_rms_and_gain():
    rng = np.random.default_rng(3)
    x = rng.normal(0, 5, size=(4, 1024)).astype(np.float32)
    y = O.rms_norm(x, np.zeros(1024, np.float32))
    assert np.allclose(np.sqrt((y.astype(np.float64) ** 2).mean(-1)), 1.0, atol=1e-5)
    y2 = O.rms_norm(x, np.ones(1024, np.float32))
    assert np.allclose(y2, 2 * y, rtol=1e-6)


def test_rms_norm_matches_transformers():
    from transformers.models.gemma.modeling_gemma import GemmaRMSNorm
    rng = np.random.default_rng(4)
    x = rng.normal(0, 0.7, size=(3, 1024)).astype(np.float32)
    g = rng.normal(0, 0.02, size=1024).astype(np.float32)
    m = GemmaRMSNorm(1024, eps=1e-6)
    with torch.no_grad():
        m.weight.copy_(torch.from_numpy(g))
        ref = m(torch.from_numpy(x)).numpy()
    assert np.allclose(O.rms_norm(x, g), ref, atol=2e-6)


def test_activations_match_torch():
    x = np.linspace(-8, 8, 4001).astype(np.float32)
    ref_g = torch.nn.functional.gelu(torch.from_numpy(x), approximate="tanh").numpy()
    ref_s = torch.nn.functional.silu(torch.from_numpy(x)).numpy()
    assert np.allclose(O.gelu_tanh(x), ref_g, atol=2e-6)
    assert np.allclose(O.silu(x), ref_s, atol=2e-6)


def test_gated_mlp_matches_transformers():
    from transformers import GemmaConfig
    from transformers.models.gemma.modeling_gemma import GemmaMLP
    cfg = GemmaConfig(hidden_size=64, intermediate_size=128, hidden_activation="gelu_pytorch_tanh")
    mlp = GemmaMLP(cfg)
    rng = np.random.default_rng(5)
    y = rng.normal(size=(3, 64)).astype(np.float32)
    with torch.no_grad():
        ref = mlp(torch.from_numpy(y)).numpy()
    gw, uw, dw = (p.detach().numpy() for p in (mlp.gate_proj.weight, mlp.up_proj.weight, mlp.down_proj.weight))
    ours = O.linear(O.gelu_tanh(O.linear(y, gw)) * O.linear(y, uw), dw)
    assert np.allclose(ours, ref, atol=1e-5)


# --- attention, masks, positions --------------------------------------------------
def test_single_visible_key_returns_its_value():
    rng = np.random.default_rng(6)
    q = rng.normal(size=(3, 8, 256)).astype(np.float32)
    k = rng.normal(size=(10, 256)).astype(np.float32)
    v = rng.normal(size=(10, 256)).astype(np.float32)
    vis = np.zeros((3, 10), bool)
    vis[0, 4] = vis[1, 0] = vis[2, 9] = True
    out = O.attend(q, k, v, vis)
    for i, key in enumerate([4, 0, 9]):
        assert np.array_equal(out[i], np.broadcast_to(v[key], (8, 256)))


def test_attention_matches_torch_sdpa():
    rng = np.random.default_rng(7)
    q = rng.normal(size=(51, 8, 256))
    k = rng.normal(size=(90, 256))
    v = rng.normal(size=(90, 256))
    vis = rng.random((51, 90)) < 0.7
    vis[:, 0] = True
    ours = O.attend(q, k, v, vis, np.float64)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q).transpose(0, 1), torch.from_numpy(k)[None].expand(8, -1, -1),
        torch.from_numpy(v)[None].expand(8, -1, -1), attn_mask=torch.from_numpy(vis)[None])
    assert np.allclose(ours, ref.transpose(0, 1).numpy(), atol=1e-12)


def test_block_mask_and_positions():
    mask = np.array([[1, 1, 0, 1, 0], [0, 0, 0, 0, 0]], np.uint8)
    vis = O.suffix_visibility(mask, horizon=3)          # (2, 4, 9)
    assert vis.shape == (2, 4, 9)
    # prefix block = valid mask for every query
    assert np.array_equal(vis[0, :, :5], np.broadcast_to(mask[0].astype(bool), (4, 5)))
    assert not vis[1, :, :5].any()
    # state query sees only the state among suffix keys; action queries see all
    assert vis[0, 0, 5:].tolist() == [True, False, False, False]
    assert vis[0, 1:, 5:].all()
    pos = O.suffix_positions(mask, horizon=3)
    assert pos.tolist() == [[3, 4, 5, 6], [0, 1, 2, 3]]


# --- end-to-end invariants -----------------------------------------------------------
def test_zero_outproj_keeps_noise_bitwise():
    inp = full_width_small()
    w = dict(inp.weights)
    w["action_out_w"] = np.zeros_like(O.as_float(w["action_out_w"], np.float32))
    w["action_out_b"] = np.zeros_like(O.as_float(w["action_out_b"], np.float32))
    x0 = run_oracle(inp, weights=w)
    assert np.array_equal(x0, inp.x1)


@pytest.mark.parametrize("steps", [1, 3, 10])
def test_bias_only_outproj_moves_by_minus_b(steps):
    inp = full_width_small()
    inp = dataclasses.replace(inp, workload=dataclasses.replace(inp.workload, num_steps=steps))
    w = dict(inp.weights)
    b = np.random.default_rng(8).normal(0, 1, 32).astype(np.float32)
    w["action_out_w"] = np.zeros((32, 1024), np.float32)
    w["action_out_b"] = b
    x0 = run_oracle(inp, weights=w)
    expect = inp.x1 - b[None, None, :]
    tol = steps * 1.2e-7 * (np.abs(inp.x1) + np.abs(b))
    assert np.all(np.abs(x0 - expect) <= tol + 1e-30)


def test_masked_prefix_positions_do_not_matter():
    inp = full_width_small(P=64, masked=10)
    x0 = run_oracle(inp)
    rng = np.random.default_rng(9)
    pk2, pv2 = [], []
    for k, v in zip(inp.prefix_k, inp.prefix_v):
        k2, v2 = O.as_float(k, np.float32).copy(), O.as_float(v, np.float32).copy()
        k2[:, :, -10:] = rng.normal(0, 30, k2[:, :, -10:].shape)
        v2[:, :, -10:] = rng.normal(0, 30, v2[:, :, -10:].shape)
        pk2.append(k2)
        pv2.append(v2)
    assert np.array_equal(run_oracle(inp, pk=pk2, pv=pv2), x0)
    # ...while changing a valid position does change the result
    pk3 = [O.as_float(k, np.float32).copy() for k in inp.prefix_k]
    pk3[0][:, :, 0] += 1.0
    assert not np.array_equal(run_oracle(inp, pk=pk3), x0)


def test_fp32_and_fp64_agree_on_full_width():
    inp = full_width_small(P=64, masked=5)
    a = run_oracle(inp, np.float32)
    b = run_oracle(inp, np.float64)
    assert np.max(np.abs(a - b)) < 1e-5


# --- float64 brute force ---------------------------------------------------------------
def _brute_and_oracle(dtype=np.float64, oracle=None):
    dims = synth.TINY_BRUTE_DIMS
    w, pk, pv, mask, state, x1, steps = tiny_float_inputs(dims)
    ref = np.array(brute_sample(w, pk, pv, mask, state, x1, steps, dims.num_heads))
    mod = oracle or O
    ours = mod.sample_actions(w, pk, pv, mask, state, x1, steps, num_heads=dims.num_heads, dtype=dtype)
    return ours, ref


def test_brute_force_float64_matches():
    ours, ref = _brute_and_oracle(np.float64)
    assert np.max(np.abs(ours - ref)) < 1e-11


def test_brute_force_float32_matches():
    ours, ref = _brute_and_oracle(np.float32)
    assert np.max(np.abs(ours - ref)) < 2e-5


def test_brute_force_sees_the_mask_hole():
    """The tiny case puts a masked hole inside sample 0's prefix; a changed value there is ignored."""
    dims = synth.TINY_BRUTE_DIMS
    w, pk, pv, mask, state, x1, steps = tiny_float_inputs(dims)
    a = O.sample_actions(w, pk, pv, mask, state, x1, steps, num_heads=2, dtype=np.float64)
    pk[0][0, 0, 1] += 5.0
    b = O.sample_actions(w, pk, pv, mask, state, x1, steps, num_heads=2, dtype=np.float64)
    assert np.array_equal(a, b)


# --- edge shapes against the float64 brute force --------------------------------------
EDGE_CASES = {
    # name: (horizon, P, mask rows (1 = valid), steps)
    "horizon_1": (1, 5, [[1, 1, 0, 1, 1], [1, 1, 1, 1, 0]], 2),
    "no_valid_prefix": (3, 4, [[0, 0, 0, 0], [1, 0, 1, 1]], 2),
    "one_position_prefix": (3, 1, [[1], [0]], 3),
    "single_step": (3, 5, [[1, 1, 1, 1, 1], [1, 0, 0, 0, 0]], 1),
}


@pytest.mark.parametrize("variant", [{}, VARIANTS_ALL := dict(time_convention="linspace", x_prediction=True,
                                                            causal_actions=True)],
                         ids=["pi0", "variants"])
@pytest.mark.parametrize("case", sorted(EDGE_CASES))
def test_brute_force_float64_matches_edge_shapes(case, variant):
    H, P, rows, steps = EDGE_CASES[case]
    dims = dataclasses.replace(synth.TINY_BRUTE_DIMS, horizon=H)
    w, pk, pv, _, state, x1, _ = tiny_float_inputs(dims, B=2, P=max(P, 2), n_masked=(0,))
    pk = [k[:, :, :P] for k in pk]
    pv = [v[:, :, :P] for v in pv]
    mask = np.array(rows, np.uint8)
    ref = np.array(brute_sample(w, pk, pv, mask, state, x1, steps, dims.num_heads, **variant))
    ours = O.sample_actions(w, pk, pv, mask, state, x1, steps, num_heads=dims.num_heads, dtype=np.float64,
                            **variant)
    assert ours.shape == (2, H, dims.action_dim)
    assert np.max(np.abs(ours - ref)) < 1e-11


# --- solver / convention variants (the Wall-X page) -------------------------------------
VARIANTS = [dict(time_convention="linspace"), dict(x_prediction=True), dict(causal_actions=True),
            dict(time_convention="linspace", x_prediction=True, causal_actions=True)]


@pytest.mark.parametrize("variant", VARIANTS, ids=lambda v: "+".join(f"{k}={x}" for k, x in v.items()))
def test_brute_force_float64_matches_variants(variant):
    dims = synth.TINY_BRUTE_DIMS
    w, pk, pv, mask, state, x1, steps = tiny_float_inputs(dims)
    ref = np.array(brute_sample(w, pk, pv, mask, state, x1, steps, dims.num_heads, **variant))
    ours = O.sample_actions(w, pk, pv, mask, state, x1, steps, num_heads=dims.num_heads, dtype=np.float64,
                            **variant)
    assert np.max(np.abs(ours - ref)) < 1e-11


@pytest.mark.parametrize("steps", [1, 3, 10])
def test_linspace_grid_runs_zero_to_one(steps):
    """t_0 = 0, each t_k within fp32 rounding of k/N, and the float32 step sizes
    are exact differences, so they add up to exactly +1 (the pi0 grid: -1)."""
    ts, dts = O.time_grid(steps, "linspace")
    assert ts[0] == 0.0 and len(ts) == len(dts) == steps
    for k, t in enumerate(ts):
        assert abs(float(t) - k / steps) <= 2.0 ** -24 * (k / steps)  # unit roundoff of fp32
    assert math.fsum(float(d) for d in dts) == 1.0
    ts_pi0, dts_pi0 = O.time_grid(steps, "pi0")
    assert ts_pi0[0] == 1.0 and abs(math.fsum(float(d) for d in dts_pi0) + 1.0) < steps * 1e-7


@pytest.mark.parametrize("steps", [1, 3, 10])
def test_linspace_bias_only_outproj_moves_by_plus_b(steps):
    inp = full_width_small()
    inp = dataclasses.replace(inp, workload=dataclasses.replace(inp.workload, num_steps=steps))
    w = dict(inp.weights)
    b = np.random.default_rng(8).normal(0, 1, 32).astype(np.float32)
    w["action_out_w"] = np.zeros((32, 1024), np.float32)
    w["action_out_b"] = b
    x0 = run_oracle(inp, weights=w, time_convention="linspace")
    tol = steps * 1.2e-7 * (np.abs(inp.x1) + np.abs(b))
    assert np.all(np.abs(x0 - (inp.x1 + b[None, None, :])) <= tol + 1e-30)


@pytest.mark.parametrize("grid,expect", [("linspace", "b"), ("pi0", "2x1-b")])
def test_x_prediction_with_a_constant_prediction(grid, expect):
    """x_hat == b at every step: the velocity is b - x_1, so on the 0 -> 1 grid the
    chunk lands on b and on the 1 -> 0 grid on x_1 - (b - x_1)."""
    inp = full_width_small()
    w = dict(inp.weights)
    b = np.random.default_rng(12).normal(0, 1, 32).astype(np.float32)
    w["action_out_w"] = np.zeros((32, 1024), np.float32)
    w["action_out_b"] = b
    x0 = run_oracle(inp, weights=w, time_convention=grid, x_prediction=True)
    want = b[None, None, :] + 0 * inp.x1 if expect == "b" else 2 * inp.x1 - b[None, None, :]
    steps = inp.workload.num_steps
    assert np.all(np.abs(x0 - want) <= steps * 2.5e-7 * (np.abs(inp.x1) + np.abs(b)) + 1e-30)


def test_causal_mask_first_action_ignores_later_actions():
    """Under the causal action mask action 0 sees the prefix, the state and itself
    only, so its whole trajectory is independent of the other actions' noise; with
    the pi0 mask it is not."""
    inp = full_width_small(horizon=6)
    x1b = inp.x1.copy()
    x1b[:, 1:] = np.random.default_rng(13).normal(0, 1, x1b[:, 1:].shape).astype(np.float32)
    inp_b = dataclasses.replace(inp, x1=x1b)
    a = run_oracle(inp, np.float64, causal_actions=True)
    b = run_oracle(inp_b, np.float64, causal_actions=True)
    assert np.max(np.abs(a[:, 0] - b[:, 0])) < 1e-12
    assert np.max(np.abs(a[:, 1:] - b[:, 1:])) > 1e-3
    a2 = run_oracle(inp, np.float64)
    b2 = run_oracle(inp_b, np.float64)
    assert np.max(np.abs(a2[:, 0] - b2[:, 0])) > 1e-6


# --- planted mistakes: each must make a pin fail --------------------------------------
def _mutations():
    def rope_sign(x, pos, dtype=np.float32):
        y = O.__dict__["_orig_apply_rope"](x, -pos, dtype)
        return y

    def rms_no_one(x, gain, dtype=np.float32, eps=O.RMS_EPS):
        return O.__dict__["_orig_rms_norm"](x, gain - 1.0, dtype, eps)

    def temb_swapped(t, dim, min_period=4e-3, max_period=4.0):
        e = O.__dict__["_orig_time_embedding"](t, dim, min_period, max_period)
        h = dim // 2
        return np.concatenate([e[:, h:], e[:, :h]], axis=1)

    def vis_state_sees_all(prefix_valid, horizon, causal_actions=False):
        v = O.__dict__["_orig_suffix_visibility"](prefix_valid, horizon, causal_actions).copy()
        v[:, 0, :] = v[:, 1, :]
        return v

    def pos_off_by_one(prefix_valid, horizon):
        return O.__dict__["_orig_suffix_positions"](prefix_valid, horizon) + 1

    def vis_causal_ignored(prefix_valid, horizon, causal_actions=False):
        return O.__dict__["_orig_suffix_visibility"](prefix_valid, horizon, False)

    def xpred_sign(out, noise, x_prediction):
        return noise - out if x_prediction else out

    def grid_reversed(num_steps, convention="pi0", dtype=np.float32):
        t, dt = O.__dict__["_orig_time_grid"](num_steps, convention, dtype)
        if convention == "linspace":
            t = [np.float32(1.0) - x for x in t]
        return t, dt

    def gelu_erf(x):
        import scipy.special
        return 0.5 * x * (1.0 + scipy.special.erf(x / math.sqrt(2.0)))

    return {
        # label: (oracle function replaced, mutant, variant the brute-force comparison runs)
        "apply_rope": ("apply_rope", rope_sign, {}),
        "rms_norm": ("rms_norm", rms_no_one, {}),
        "time_embedding": ("time_embedding", temb_swapped, {}),
        "suffix_visibility": ("suffix_visibility", vis_state_sees_all, {}),
        "suffix_positions": ("suffix_positions", pos_off_by_one, {}),
        "gelu_tanh": ("gelu_tanh", gelu_erf, {}),
        "causal_mask_ignored": ("suffix_visibility", vis_causal_ignored, {"causal_actions": True}),
        "x_prediction_sign": ("output_to_velocity", xpred_sign, {"x_prediction": True}),
        "time_grid_reversed": ("time_grid", grid_reversed, {"time_convention": "linspace"}),
    }


@pytest.mark.parametrize("label", sorted(_mutations()))
def test_planted_mistakes_are_caught(label, monkeypatch):
    name, fn, variant = _mutations()[label]
    monkeypatch.setitem(O.__dict__, "_orig_" + name, getattr(O, name))
    monkeypatch.setattr(O, name, fn)
    dims = synth.TINY_BRUTE_DIMS
    w, pk, pv, mask, state, x1, steps = tiny_float_inputs(dims)
    ref = np.array(brute_sample(w, pk, pv, mask, state, x1, steps, dims.num_heads, **variant))
    ours = O.sample_actions(w, pk, pv, mask, state, x1, steps, num_heads=dims.num_heads, dtype=np.float64,
                            **variant)
    assert np.max(np.abs(ours - ref)) > 1e-6, f"planted mistake {label} went unnoticed"
