"""Constants the pi0 page prints (tests/golden/pi0_page_constants.txt) against the
dimensions, workloads and oracle defaults used here."""
from __future__ import annotations

import inspect
import os

from oracle import pi0_oracle as O
from vla_flow_matching_b200 import synth


def _golden():
    out = {}
    with open(os.path.join(os.path.dirname(__file__), "golden", "pi0_page_constants.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = (x.strip() for x in line.split("=", 1))
                out[k] = float(v)
    return out


def test_expert_dims_are_the_gemma_300m_variant():
    g, d = _golden(), synth.ExpertDims()
    for f in ("width", "depth", "mlp_dim", "num_heads", "num_kv_heads", "head_dim"):
        assert getattr(d, f) == g[f"gemma_300m.{f}"], f
    assert d.horizon == g["DEFAULT_ACTION_HORIZON"] and d.action_dim == g["DEFAULT_ACTION_DIM"]


def test_full_workloads_use_the_default_step_count_and_text_length():
    g = _golden()
    for name in ("full_b1", "full_b32", "full_b128"):
        wl = synth.WORKLOADS[name]
        assert wl.num_steps == g["DEFAULT_NUM_INFERENCE_STEPS"]
        assert wl.prefix_len == 3 * 256 + g["DEFAULT_MAX_TOKEN_LEN"]   # three 224x224 cameras + text


def test_oracle_mask_fill_and_sinusoid_periods():
    g = _golden()
    assert O.MASK_FILL == g["OPENPI_ATTENTION_MASK_VALUE"]
    sig = inspect.signature(O.time_embedding)
    assert sig.parameters["min_period"].default == g["sinusoid.min_period"]
    assert sig.parameters["max_period"].default == g["sinusoid.max_period"]
