"""Seeded synthetic inputs for the pi0 action-expert denoising loop.

This module is shared by the CPU oracle's tests and by the CUDA path's tests and
benchmark. It holds none of the method's arithmetic: only random draws
(numpy ``PCG64`` streams), the bf16 round-to-nearest-even used to *store*
weights and prefix K/V, and the prefix valid-mask recipes of the five workloads.

Shapes and distributions follow the pi0 action expert ("gemma_300m": width 1024,
depth 18, MLP 4096, 8 query heads, 1 KV head, head_dim 256; horizon 50,
action/state dim 32) described on the vllm-omni ``modeling_pi0.py`` page
(``get_gemma_config`` and the module constants).

Stream layout (every stream is independent, so any subset of samples can be
regenerated without drawing the rest):

* ``SeedSequence(seed).spawn(4)`` -> ``[weights, prefix_kv, masks, io]``
* weights: one generator, tensors drawn in :data:`WEIGHT_ORDER` order,
  N(0, 0.02) then rounded to bf16 (norm gains and Linear biases included).
* prefix K/V: ``prefix_kv.spawn(batch)[b]`` draws, for layer 0..depth-1, the
  K then the V block of sample ``b``: (P, head_dim) N(0, 1) rounded to bf16.
* masks: one generator, one integer per sample where the recipe needs it.
* io: one generator; ``state`` (B, state_dim) then ``x_1`` (B, H, A), N(0, 1) fp32.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Sequence

import numpy as np

__all__ = [
    "ExpertDims", "Workload", "WORKLOADS", "TINY_BRUTE_DIMS", "Inputs",
    "f32_to_bf16_bits", "bf16_bits_to_f32", "make_weights", "make_prefix_kv",
    "make_mask", "make_io", "make_inputs", "WEIGHT_ORDER", "LAYER_ORDER",
]


@dataclasses.dataclass(frozen=True)
class ExpertDims:
    """Dimensions of the action expert and of the action chunk."""
    width: int = 1024
    depth: int = 18
    mlp_dim: int = 4096
    num_heads: int = 8
    num_kv_heads: int = 1
    head_dim: int = 256
    horizon: int = 50
    action_dim: int = 32
    state_dim: int = 32

    @property
    def suffix_len(self) -> int:
        return self.horizon + 1


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: dims, batch, prefix layout and Euler steps.

    ``mask_kind``:
      * ``"all"``: every prefix position valid.
      * ``"tail_pad"``: the last ``mask_a`` positions padded.
      * ``"text_len"``: ``mask_b`` image tokens always valid, then a text
        segment whose valid length is drawn uniform in [mask_a, P - mask_b]
        per sample, padding at the end of the segment.
      * ``"prefix_len"``: valid prefix length drawn uniform in [mask_a, P]
        per sample (the first ``len`` positions valid).
    ``state_zero_from``: state dims at and after this index are set to 0.
    """
    name: str
    dims: ExpertDims
    batch: int
    prefix_len: int
    num_steps: int
    seed: int
    mask_kind: str = "all"
    mask_a: int = 0
    mask_b: int = 0
    state_zero_from: Optional[int] = None


_FULL = ExpertDims()

#: The five workloads: a tiny depth-2 case, the full expert at B=1, B=32, a
#: short-horizon B=8 variant and the large-batch B=128 case.  Prefix lengths
#: are 256 tokens per camera plus 48 text tokens (3 cameras: 816; 2: 560).
WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", dataclasses.replace(_FULL, depth=2), batch=1,
                     prefix_len=128, num_steps=2, seed=0),
    "full_b1": Workload("full_b1", _FULL, batch=1, prefix_len=816, num_steps=10,
                        seed=1, mask_kind="tail_pad", mask_a=10),
    "full_b32": Workload("full_b32", _FULL, batch=32, prefix_len=816,
                         num_steps=10, seed=2, mask_kind="text_len",
                         mask_a=20, mask_b=768),
    "short_b8": Workload("short_b8", dataclasses.replace(_FULL, horizon=10),
                         batch=8, prefix_len=560, num_steps=5, seed=3,
                         state_zero_from=7),
    "full_b128": Workload("full_b128", _FULL, batch=128, prefix_len=816,
                          num_steps=10, seed=4, mask_kind="prefix_len",
                          mask_a=600),
}

#: Profiling case, not a benchmark config: one Euler step of full_b1.  Every step
#: streams all of the expert's weights (629 MB against a 126 MB L2), so DRAM counters
#: taken on it scale to full_b1's ten steps by the step count.
PROFILE_WORKLOADS: Dict[str, Workload] = {
    "full_b1_1step": dataclasses.replace(WORKLOADS["full_b1"], name="full_b1_1step", num_steps=1),
}

#: Tiny dims for the float64 brute force (pure-Python loops stay fast).
TINY_BRUTE_DIMS = ExpertDims(width=16, depth=2, mlp_dim=32, num_heads=2,
                             num_kv_heads=1, head_dim=8, horizon=3,
                             action_dim=4, state_dim=4)

#: Order in which the non-layer weight tensors are drawn (layers in between).
WEIGHT_ORDER = ["state_proj_w", "state_proj_b", "action_in_w", "action_in_b",
                "time_in_w", "time_in_b", "time_out_w", "time_out_b"]
LAYER_ORDER = ["in_norm_w", "q_w", "k_w", "v_w", "o_w", "post_norm_w",
               "gate_w", "up_w", "down_w"]
TAIL_ORDER = ["final_norm_w", "action_out_w", "action_out_b"]


def weight_shapes(d: ExpertDims) -> Dict[str, tuple]:
    """nn.Linear layout (out, in) for every tensor of the expert + projections."""
    w, q = d.width, d.num_heads * d.head_dim
    kv = d.num_kv_heads * d.head_dim
    return {
        "state_proj_w": (w, d.state_dim), "state_proj_b": (w,),
        "action_in_w": (w, d.action_dim), "action_in_b": (w,),
        "time_in_w": (w, 2 * w), "time_in_b": (w,),
        "time_out_w": (w, w), "time_out_b": (w,),
        "in_norm_w": (w,), "q_w": (q, w), "k_w": (kv, w), "v_w": (kv, w),
        "o_w": (w, q), "post_norm_w": (w,), "gate_w": (d.mlp_dim, w),
        "up_w": (d.mlp_dim, w), "down_w": (w, d.mlp_dim),
        "final_norm_w": (w,), "action_out_w": (d.action_dim, w),
        "action_out_b": (d.action_dim,),
    }


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); returns the uint16 bit pattern.
    NaN stays NaN (quiet, sign kept); overflow rounds to infinity."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = u + (np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1)))
    out = (rounded >> np.uint32(16)).astype(np.uint16)
    nan = (u & np.uint32(0x7FFFFFFF)) > np.uint32(0x7F800000)
    return np.where(nan, ((u >> np.uint32(16)) | np.uint32(0x0040)).astype(np.uint16), out)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen a bf16 bit pattern (uint16) to fp32 exactly."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _streams(seed: int):
    return np.random.SeedSequence(seed).spawn(4)


def make_weights(d: ExpertDims, seed: int, std: float = 0.02) -> dict:
    """All expert weights as bf16 bit patterns (uint16), nn.Linear (out, in) layout.

    Returns ``{"state_proj_w": ..., ..., "layers": [{"q_w": ...}, ...], ...}``.
    """
    rng = np.random.Generator(np.random.PCG64(_streams(seed)[0]))
    shapes = weight_shapes(d)

    def draw(name):
        x = rng.standard_normal(shapes[name], dtype=np.float32) * np.float32(std)
        return f32_to_bf16_bits(x)

    out = {name: draw(name) for name in WEIGHT_ORDER}
    out["layers"] = [{name: draw(name) for name in LAYER_ORDER} for _ in range(d.depth)]
    for name in TAIL_ORDER:
        out[name] = draw(name)
    return out


def make_prefix_kv(d: ExpertDims, seed: int, batch: int, prefix_len: int,
                   samples: Optional[Sequence[int]] = None):
    """Per-layer prefix K and V as bf16 bits, shape (B', 1, P, head_dim) each.

    ``samples`` selects which of the ``batch`` samples to generate (default all);
    sample ``b`` always gets the same values whatever subset is asked for.
    """
    if samples is None:
        samples = range(batch)
    samples = list(samples)
    subs = _streams(seed)[1].spawn(batch)
    kv_shape = (d.num_kv_heads, prefix_len, d.head_dim)
    ks = [np.empty((len(samples),) + kv_shape, np.uint16) for _ in range(d.depth)]
    vs = [np.empty((len(samples),) + kv_shape, np.uint16) for _ in range(d.depth)]
    for i, b in enumerate(samples):
        rng = np.random.Generator(np.random.PCG64(subs[b]))
        for layer in range(d.depth):
            ks[layer][i] = f32_to_bf16_bits(rng.standard_normal(kv_shape, dtype=np.float32))
            vs[layer][i] = f32_to_bf16_bits(rng.standard_normal(kv_shape, dtype=np.float32))
    return ks, vs


def make_mask(wl: Workload) -> np.ndarray:
    """Prefix valid mask (B, P) uint8 (1 = valid key) for the workload's recipe."""
    rng = np.random.Generator(np.random.PCG64(_streams(wl.seed)[2]))
    B, P = wl.batch, wl.prefix_len
    m = np.zeros((B, P), np.uint8)
    if wl.mask_kind == "all":
        m[:] = 1
    elif wl.mask_kind == "tail_pad":
        m[:, : P - wl.mask_a] = 1
    elif wl.mask_kind == "text_len":
        lens = rng.integers(wl.mask_a, P - wl.mask_b, size=B, endpoint=True)
        for b in range(B):
            m[b, : wl.mask_b + int(lens[b])] = 1
    elif wl.mask_kind == "prefix_len":
        lens = rng.integers(wl.mask_a, P, size=B, endpoint=True)
        for b in range(B):
            m[b, : int(lens[b])] = 1
    else:
        raise ValueError(f"unknown mask kind {wl.mask_kind!r}")
    return m


def make_io(wl: Workload):
    """Robot state (B, state_dim) and the t=1 noise x_1 (B, H, A), fp32 N(0, 1)."""
    d = wl.dims
    rng = np.random.Generator(np.random.PCG64(_streams(wl.seed)[3]))
    state = rng.standard_normal((wl.batch, d.state_dim), dtype=np.float32)
    if wl.state_zero_from is not None:
        state[:, wl.state_zero_from:] = 0.0
    x1 = rng.standard_normal((wl.batch, d.horizon, d.action_dim), dtype=np.float32)
    return state, x1


@dataclasses.dataclass
class Inputs:
    """Everything one call of the sampler consumes (host numpy arrays)."""
    workload: Workload
    weights: dict
    prefix_k: List[np.ndarray]   # depth x (B', 1, P, Dh) uint16 (bf16 bits)
    prefix_v: List[np.ndarray]
    mask: np.ndarray             # (B', P) uint8
    state: np.ndarray            # (B', S) float32
    x1: np.ndarray               # (B', H, A) float32
    samples: List[int]

    @property
    def batch(self) -> int:
        return len(self.samples)


def make_inputs(wl: Workload, samples: Optional[Sequence[int]] = None,
                weights: Optional[dict] = None) -> Inputs:
    """Generate the workload's inputs, optionally for a subset of samples."""
    if samples is None:
        samples = list(range(wl.batch))
    samples = list(samples)
    w = weights if weights is not None else make_weights(wl.dims, wl.seed)
    ks, vs = make_prefix_kv(wl.dims, wl.seed, wl.batch, wl.prefix_len, samples)
    mask = make_mask(wl)[samples]
    state, x1 = make_io(wl)
    return Inputs(wl, w, ks, vs, np.ascontiguousarray(mask),
                  np.ascontiguousarray(state[samples]),
                  np.ascontiguousarray(x1[samples]), samples)
