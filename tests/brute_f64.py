"""Float64 brute force of the pi0 denoising loop, pure-Python loops, tiny dims only.

Written independently of ``oracle/pi0_oracle.py`` (no shared helpers): it skips
masked keys instead of adding a fill value, counts valid prefix tokens by hand,
rotates RoPE pairs explicitly and evaluates every dot product with a Python loop.
It restates the vllm-omni ``modeling_pi0.py`` page (``sample_actions``,
``denoise_step``, ``embed_suffix``, ``_compute_layer_suffix_only``).
"""
from __future__ import annotations

import math


def _vec(a):
    return [float(x) for x in a]


def _mat(a):
    return [[float(x) for x in row] for row in a]


def _matvec(w, x, b=None):
    out = []
    for r, row in enumerate(w):
        s = 0.0
        for c, wc in enumerate(row):
            s += wc * x[c]
        out.append(s + (b[r] if b is not None else 0.0))
    return out


def _rmsnorm(x, g, eps=1e-6):
    ms = sum(v * v for v in x) / len(x)
    r = 1.0 / math.sqrt(ms + eps)
    return [x[i] * r * (1.0 + g[i]) for i in range(len(x))]


def _rope(x, p, theta=10000.0):
    d = len(x)
    half = d // 2
    out = [0.0] * d
    for i in range(half):
        f = p * theta ** (-(2.0 * i) / d)
        c, s = math.cos(f), math.sin(f)
        out[i] = x[i] * c - x[i + half] * s
        out[i + half] = x[i + half] * c + x[i] * s
    return out


def _gelu_tanh(x):
    return 0.5 * x * (1.0 + math.tanh(math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)))


def _silu(x):
    return x / (1.0 + math.exp(-x))


def _temb(t, dim):
    half = dim // 2
    sins, coss = [], []
    for i in range(half):
        period = 0.004 * (1000.0 ** (i / (half - 1)))
        a = t * 2.0 * math.pi / period
        sins.append(math.sin(a))
        coss.append(math.cos(a))
    return sins + coss


def brute_sample(weights, prefix_k, prefix_v, mask, state, x1, num_steps, num_heads, time_convention="pi0",
                 x_prediction=False, causal_actions=False):
    """weights: float arrays (nn.Linear layout); prefix_k/v: per layer (B,1,P,D) floats.

    Variants (the Wall-X page): time_convention "linspace" steps t from 0 to 1 on the
    grid k/N (the time embedding sees float32(k/N)); x_prediction takes the
    output as the clean action and moves along output - initial noise;
    causal_actions lets suffix query i see suffix keys 0..i only."""
    W = _mat(weights["state_proj_w"])
    depth = len(weights["layers"])
    B = len(x1)
    H = len(x1[0])
    D = len(prefix_k[0][0][0][0])
    width = len(W)
    np = __import__("numpy")
    dt = -1.0 / num_steps
    if time_convention == "linspace":
        grid = [k / num_steps for k in range(num_steps + 1)]
    x = [[_vec(row) for row in x1[b]] for b in range(B)]
    noise = [[_vec(row) for row in x1[b]] for b in range(B)]
    layers = [{k: (_mat(v) if getattr(v, "ndim", 1) == 2 else _vec(v)) for k, v in lw.items()}
              for lw in weights["layers"]]
    g = {k: (_mat(v) if getattr(v, "ndim", 1) == 2 else _vec(v))
         for k, v in weights.items() if k != "layers"}
    for step in range(num_steps):
        if time_convention == "linspace":
            t = float(np.float32(grid[step]))
            h_step = grid[step + 1] - grid[step]
        else:
            t = float(np.float32(1.0 + step * dt))
            h_step = dt
        te = _temb(t, width)
        for b in range(B):
            n_valid = 0
            valid_idx = []
            for p, m in enumerate(mask[b]):
                if m:
                    valid_idx.append(p)
                    n_valid += 1
            toks = [_matvec(g["state_proj_w"], _vec(state[b]), g["state_proj_b"])]
            for j in range(H):
                a = _matvec(g["action_in_w"], x[b][j], g["action_in_b"])
                u = [_silu(v) for v in _matvec(g["time_in_w"], a + te, g["time_in_b"])]
                toks.append(_matvec(g["time_out_w"], u, g["time_out_b"]))
            T = H + 1
            for li in range(depth):
                lw = layers[li]
                kp = prefix_k[li][b][0]
                vp = prefix_v[li][b][0]
                xs = [_rmsnorm(h, lw["in_norm_w"]) for h in toks]
                qs = [_matvec(lw["q_w"], xx) for xx in xs]
                ks = [_rope(_matvec(lw["k_w"], xx), n_valid + i) for i, xx in enumerate(xs)]
                vs = [_matvec(lw["v_w"], xx) for xx in xs]
                new = []
                for i in range(T):
                    # keys this query may see: valid prefix, then the suffix block rule
                    keys = [(_vec(kp[p]), _vec(vp[p])) for p in valid_idx]
                    if causal_actions:
                        suffix_keys = list(range(i + 1))
                    else:
                        suffix_keys = [0] if i == 0 else list(range(T))
                    keys += [(ks[j], vs[j]) for j in suffix_keys]
                    o = []
                    for hd in range(num_heads):
                        q = _rope(qs[i][hd * D:(hd + 1) * D], n_valid + i)
                        logits = [sum(q[d] * kk[d] for d in range(D)) / math.sqrt(D) for kk, _ in keys]
                        mx = max(logits)
                        e = [math.exp(l - mx) for l in logits]
                        z = sum(e)
                        o += [sum(e[k] * keys[k][1][d] for k in range(len(keys))) / z for d in range(D)]
                    att = _matvec(lw["o_w"], o)
                    h1 = [toks[i][c] + att[c] for c in range(width)]
                    y = _rmsnorm(h1, lw["post_norm_w"])
                    gt = _matvec(lw["gate_w"], y)
                    up = _matvec(lw["up_w"], y)
                    m = _matvec(lw["down_w"], [_gelu_tanh(gt[f]) * up[f] for f in range(len(gt))])
                    new.append([h1[c] + m[c] for c in range(width)])
                toks = new
            for j in range(H):
                y = _rmsnorm(toks[1 + j], g["final_norm_w"])
                vel = _matvec(g["action_out_w"], y, g["action_out_b"])
                if x_prediction:
                    vel = [vel[a] - noise[b][j][a] for a in range(len(vel))]
                x[b][j] = [x[b][j][a] + h_step * vel[a] for a in range(len(vel))]
    return x
