"""CPU oracle for the pi0 flow-matching denoising loop.  TEST INFRASTRUCTURE.

This is a plain, slow, step-by-step restatement of what the loop computes, used
only to check the CUDA path.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it;
the product path (``vla_flow_matching_b200``) never imports, calls or links it,
and this module imports nothing from the product path.

Source: the vllm-omni page "vllm_omni/diffusion/models/pi0/modeling_pi0.py"
(an inference-only pi0 "math kernel"), cited below by function name, and the
VersatIL ``GenerativeVLM`` page for the rotate-half RoPE and residual+FFN order.
The solver and convention variants (time grid 0 -> 1, x-prediction, causal
action mask) follow the Wall-X flow-matching page (its ODE integration of the
sampler, ``use_x_pred`` and ``causal_action_attention_mask``).

Precision follows that page: the expert runs in float32 (its Gemma config is
built with ``dtype="float32"``), the timestep embedding is formed in float64 and
then cast to the model dtype, RoPE angles and the softmax are float32.
``dtype=np.float64`` runs every step in float64 instead.

Library primitives used as steps: ``numpy.matmul`` (each Linear), ``np.exp``,
``np.sin``/``np.cos``, ``np.tanh``.  No step is fused, blocked or reordered
beyond what the page states.

Parity pins for every function live in ``tests/test_oracle_pins.py``; none of
the functions here is "parity unpinned".
"""
from __future__ import annotations

import math
from typing import List, Sequence

import numpy as np

# Fill value the page adds to masked attention logits (OpenPI's constant).
MASK_FILL = -2.3819763e38
RMS_EPS = 1e-6          # Gemma RMSNorm epsilon (transformers GemmaConfig default)
ROPE_THETA = 10000.0    # Gemma rotary base (transformers GemmaConfig default)


def as_float(a, dtype):
    """bf16 bit patterns (uint16) widen exactly; float arrays are cast."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        a = (a.astype(np.uint32) << np.uint32(16)).view(np.float32)
    return a.astype(dtype, copy=False)


# --- timestep embedding ------------------------------------------------------
def time_embedding(t: np.ndarray, dim: int, min_period: float = 4e-3,
                   max_period: float = 4.0) -> np.ndarray:
    """Sine/cosine embedding of scalar times, float64 (``create_sinusoidal_pos_embedding``).

    For half = dim/2 frequencies, the i-th period sweeps log-linearly from
    ``min_period`` (i = 0) to ``max_period`` (i = half-1):
    period_i = min_period * (max_period/min_period)^(i/(half-1)).  The angle is
    2*pi*t/period_i; the output is [sin(angles), cos(angles)] (sin block first).
    """
    if dim % 2 != 0:
        raise ValueError("embedding dimension must be even")
    t = np.asarray(t)
    if t.ndim != 1:
        raise ValueError("times must be a 1-D array")
    half = dim // 2
    out = np.empty((t.shape[0], dim), np.float64)
    for i in range(half):
        frac = i / (half - 1) if half > 1 else 0.0
        period = min_period * (max_period / min_period) ** frac
        ang = (2.0 * math.pi / period) * t.astype(np.float64)
        out[:, i] = np.sin(ang)
        out[:, half + i] = np.cos(ang)
    return out


# --- Gemma primitives ---------------------------------------------------------
def rms_norm(x: np.ndarray, gain: np.ndarray, dtype=np.float32, eps: float = RMS_EPS):
    """Gemma RMSNorm: x / sqrt(mean(x^2) + eps) * (1 + gain), in float32 or wider."""
    x = x.astype(dtype, copy=False)
    ms = np.mean(x * x, axis=-1, keepdims=True, dtype=dtype)
    inv = (1.0 / np.sqrt(ms + dtype(eps))).astype(dtype)
    return (x * inv) * (dtype(1.0) + gain.astype(dtype))


def rope_inv_freq(head_dim: int, dtype=np.float32, theta: float = ROPE_THETA):
    """Per-pair inverse frequency theta^(-2i/head_dim), i < head_dim/2.

    The page builds these in float32 (the Gemma rotary module); the oracle takes
    the value of the formula evaluated in float64 and rounded once to the rotary
    dtype, i.e. the correctly rounded float32 number (a float32 ``pow`` may be
    1 ulp away from it).
    """
    i = np.arange(head_dim // 2, dtype=np.float64)
    return (theta ** (-2.0 * i / head_dim)).astype(dtype)


def apply_rope(x: np.ndarray, pos: np.ndarray, dtype=np.float32):
    """Rotate-half RoPE on the last axis (HF ``apply_rotary_pos_emb``).

    ``x``: (..., T, heads, head_dim) with positions ``pos`` (..., T).  With
    a = x[:half], b = x[half:], angle = pos * inv_freq:
    out[:half] = a*cos - b*sin,  out[half:] = b*cos + a*sin.
    """
    d = x.shape[-1]
    half = d // 2
    ang = pos.astype(dtype)[..., None] * rope_inv_freq(d, dtype)  # (..., T, half)
    c = np.cos(ang).astype(dtype)[..., None, :]
    s = np.sin(ang).astype(dtype)[..., None, :]
    a, b = x[..., :half], x[..., half:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1).astype(dtype)


def gelu_tanh(x: np.ndarray):
    """GELU, tanh form (``gelu_pytorch_tanh``): 0.5 x (1 + tanh(sqrt(2/pi)(x + 0.044715 x^3)))."""
    dt = x.dtype.type
    k = dt(math.sqrt(2.0 / math.pi))
    return dt(0.5) * x * (dt(1.0) + np.tanh(k * (x + dt(0.044715) * x * x * x)))


def silu(x: np.ndarray):
    """SiLU / swish: x * sigmoid(x)."""
    dt = x.dtype.type
    return x / (dt(1.0) + np.exp(-x))


def linear(x, w, b=None):
    """nn.Linear: x @ w^T (+ b), w in (out, in) layout."""
    y = np.matmul(x, w.T)
    return y if b is None else y + b


# --- masks and positions -----------------------------------------------------
def suffix_visibility(prefix_valid: np.ndarray, horizon: int, causal_actions: bool = False) -> np.ndarray:
    """Boolean (B, T, P+T) mask of which key each suffix query may attend to.

    From ``denoise_step``/``embed_suffix``/``make_att_2d_masks``: prefix keys are
    visible to every suffix query iff valid; inside the suffix the AR flags are
    [1, 1, 0, ..., 0] and key j is visible to query i iff cumsum[j] <= cumsum[i]
    (all suffix tokens are non-padding).

    ``causal_actions`` (the Wall-X ``causal_action_attention_mask``): the
    suffix-to-suffix block is lower triangular, key j visible to query i iff
    j <= i, so action token i sees the state and actions 0..i.
    """
    B, P = prefix_valid.shape
    T = horizon + 1
    if causal_actions:
        suf = np.tril(np.ones((T, T), dtype=bool))          # [query, key]
    else:
        ar = np.array([1, 1] + [0] * (horizon - 1), dtype=np.int64)
        cum = np.cumsum(ar)
        suf = cum[None, :] <= cum[:, None]                  # [query, key]
    pre = np.broadcast_to(prefix_valid.astype(bool)[:, None, :], (B, T, P))
    return np.concatenate([pre, np.broadcast_to(suf, (B, T, T))], axis=2)


def suffix_positions(prefix_valid: np.ndarray, horizon: int) -> np.ndarray:
    """Position ids (B, T): number of valid prefix tokens + cumsum(suffix pad) - 1."""
    n = prefix_valid.astype(np.int64).sum(axis=1)
    return n[:, None] + np.arange(horizon + 1, dtype=np.int64)[None, :]


# --- attention and layer -----------------------------------------------------
def attend(q, k, v, visible, dtype=np.float32):
    """Eager masked attention (``_attend``), one KV head shared by all q heads.

    q (T, H, D), k/v (S, D), visible (T, S).  Logits = (q . k) / sqrt(D) plus the
    additive fill where not visible, softmax in float32 (or float64), then the
    probabilities (already in the query dtype) times V.  Returns (T, H, D).
    """
    D = q.shape[-1]
    scale = dtype(1.0 / math.sqrt(D))
    fill = np.where(visible, dtype(0.0), dtype(MASK_FILL)).astype(dtype)   # (T, S)
    out = np.empty_like(q)
    for h in range(q.shape[1]):
        logits = np.matmul(q[:, h, :], k.T) * scale + fill
        m = logits.max(axis=-1, keepdims=True)
        e = np.exp(logits - m)
        p = e / e.sum(axis=-1, keepdims=True)
        out[:, h, :] = np.matmul(p.astype(dtype), v)
    return out


def expert_layer(h, lw, k_pref, v_pref, visible, pos, n_heads, head_dim, dtype):
    """One action-expert layer on the suffix (``_compute_layer_suffix_only``).

    h (B, T, W); k_pref/v_pref (B, P, D) already rotated; visible (B, T, P+T);
    pos (B, T).  RMSNorm -> q/k/v -> RoPE(q, k_suffix) -> concat prefix and suffix
    K/V -> attention (scale 1/sqrt(D)) -> o_proj + residual -> post-attention
    RMSNorm -> gated-GELU(tanh) MLP + residual.
    """
    B, T, W = h.shape
    x = rms_norm(h, lw["in_norm_w"], dtype)
    q = linear(x, lw["q_w"]).reshape(B, T, n_heads, head_dim)
    k = linear(x, lw["k_w"]).reshape(B, T, 1, head_dim)
    v = linear(x, lw["v_w"]).reshape(B, T, head_dim)
    q = apply_rope(q, pos, dtype)
    k = apply_rope(k, pos, dtype)[:, :, 0, :]
    o = np.empty((B, T, n_heads, head_dim), dtype)
    for b in range(B):
        kk = np.concatenate([k_pref[b], k[b]], axis=0)
        vv = np.concatenate([v_pref[b], v[b]], axis=0)
        o[b] = attend(q[b], kk, vv, visible[b], dtype)
    h = linear(o.reshape(B, T, n_heads * head_dim), lw["o_w"]) + h
    y = rms_norm(h, lw["post_norm_w"], dtype)
    mlp = linear(gelu_tanh(linear(y, lw["gate_w"])) * linear(y, lw["up_w"]), lw["down_w"])
    return mlp + h


# --- suffix embedding, one denoising step, the Euler loop --------------------
def embed_suffix(w, state, x_t, t, dtype):
    """Suffix tokens [state_proj(state), mlp_out(silu(mlp_in([a; temb])))] (``embed_suffix``).

    a = action_in_proj(x_t) per action token; temb is the float64 sinusoid of
    the step time cast to the model dtype, broadcast over the horizon.
    """
    B, H, _ = x_t.shape
    W = w["action_in_w"].shape[0]
    s_tok = linear(state.astype(dtype), w["state_proj_w"], w["state_proj_b"])[:, None, :]
    temb = time_embedding(np.full((B,), t, np.float32), W).astype(dtype)
    a = linear(x_t.astype(dtype), w["action_in_w"], w["action_in_b"])
    at = np.concatenate([a, np.broadcast_to(temb[:, None, :], a.shape)], axis=2)
    u = silu(linear(at, w["time_in_w"], w["time_in_b"]))
    act_tok = linear(u, w["time_out_w"], w["time_out_b"])
    return np.concatenate([s_tok, act_tok], axis=1)


def denoise_step(w, prefix_k, prefix_v, prefix_valid, state, x_t, t, dims, dtype, causal_actions=False):
    """v_t for one Euler step (``denoise_step``): suffix through all expert layers,
    final RMSNorm, keep the last ``horizon`` tokens, action_out_proj."""
    n_heads, head_dim = dims
    H = x_t.shape[1]
    h = embed_suffix(w, state, x_t, t, dtype)
    visible = suffix_visibility(prefix_valid, H, causal_actions)
    pos = suffix_positions(prefix_valid, H)
    for layer, lw in enumerate(w["layers"]):
        h = expert_layer(h, lw, prefix_k[layer], prefix_v[layer], visible, pos,
                         n_heads, head_dim, dtype)
    h = rms_norm(h, w["final_norm_w"], dtype)
    return linear(h[:, -H:, :], w["action_out_w"], w["action_out_b"])


def convert_weights(weights: dict, dtype) -> dict:
    """bf16 bits or float arrays -> arrays of ``dtype`` (same nesting)."""
    out = {k: as_float(v, dtype) for k, v in weights.items() if k != "layers"}
    out["layers"] = [{k: as_float(v, dtype) for k, v in lw.items()} for lw in weights["layers"]]
    return out


def time_grid(num_steps: int, convention: str = "pi0", dtype=np.float32):
    """Step times t_k (k < N; float32, the value the time embedding receives) and
    step sizes dt_k (in the model dtype).

    "pi0" (``sample_actions``): t runs from 1 (noise) to 0; t_k = float32(1 + k*(-1/N))
    with the product formed in float64, dt = -1/N (a Python double) taken in the
    model dtype.
    "linspace" (the Wall-X sampler: ``torch.linspace(0, 1, N + 1)`` in the model
    dtype, integrated with a fixed-grid Euler step): grid points dtype(k/N),
    correctly rounded, dt_k = their difference in the model dtype, and t_k =
    float32(k/N), so the noise sits at t = 0 and the action at t = 1.
    """
    if num_steps <= 0:
        raise ValueError("num_steps must be positive")
    if convention == "pi0":
        dt_exact = -1.0 / num_steps
        t = [np.float32(1.0 + k * dt_exact) for k in range(num_steps)]
        dt = [dtype(dt_exact)] * num_steps
    elif convention == "linspace":
        pts = [dtype(k / num_steps) for k in range(num_steps + 1)]
        t = [np.float32(k / num_steps) for k in range(num_steps)]
        dt = [dtype(pts[k + 1] - pts[k]) for k in range(num_steps)]
    else:
        raise ValueError(f"unknown time grid {convention!r}")
    return t, dt


def output_to_velocity(out: np.ndarray, noise: np.ndarray, x_prediction: bool) -> np.ndarray:
    """The network output read as the velocity (pi0), or as the clean action
    x_hat with velocity x_hat - noise (the Wall-X ``use_x_pred`` branch)."""
    return out - noise if x_prediction else out


def sample_actions(weights: dict, prefix_k: Sequence[np.ndarray],
                   prefix_v: Sequence[np.ndarray], prefix_valid: np.ndarray,
                   state: np.ndarray, x1: np.ndarray, num_steps: int,
                   num_heads: int = 8, dtype=np.float32, time_convention: str = "pi0",
                   x_prediction: bool = False, causal_actions: bool = False) -> np.ndarray:
    """Euler integration from t = 1 (noise x_1) to t = 0 (``sample_actions``).

    dt = -1/num_steps; at step k the time is t = 1 + k*dt (stored as float32),
    v_t comes from :func:`denoise_step` and x <- x + dt*v_t (dt taken in the
    model dtype).  Returns x_0 with the shape of ``x1``.

    Variants (the Wall-X page): ``time_convention="linspace"`` integrates from
    t = 0 (noise) to 1 on the grid of :func:`time_grid`; ``x_prediction``
    reads the network output as the clean action x_hat and uses the velocity
    x_hat - x_1 (``use_x_pred``: prediction minus the noise); ``causal_actions``
    makes the suffix attention lower triangular (:func:`suffix_visibility`).

    ``prefix_k``/``prefix_v``: per layer (B, 1, P, head_dim), already rotated,
    bf16 bits or floats.  ``prefix_valid``: (B, P), nonzero = valid key.
    """
    if num_steps <= 0:
        raise ValueError("num_steps must be positive")
    if len(prefix_k) != len(weights["layers"]) or len(prefix_v) != len(prefix_k):
        raise ValueError("one prefix K and V per expert layer is required")
    w = convert_weights(weights, dtype)
    head_dim = prefix_k[0].shape[-1]
    kp = [as_float(k, dtype)[:, 0] for k in prefix_k]
    vp = [as_float(v, dtype)[:, 0] for v in prefix_v]
    ts, dts = time_grid(num_steps, time_convention, dtype)
    noise = np.asarray(x1).astype(dtype)
    x = noise.copy()
    for step in range(num_steps):
        v = denoise_step(w, kp, vp, prefix_valid, state, x, ts[step], (num_heads, head_dim), dtype,
                         causal_actions).astype(dtype)
        v = output_to_velocity(v, noise, x_prediction)
        x = x + dtype(dts[step]) * v
    return x
