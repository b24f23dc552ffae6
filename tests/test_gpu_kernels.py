"""Unit parity of single kernels through the debug C ABI (include/pi0x_debug.h).

The tcgen05 GEMM is checked against a plain fp32 matmul of the same bf16
operands (torch on the GPU, fp32 accumulate, TF32 off).
"""
import pytest

pytestmark = pytest.mark.gpu


def _torch():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _attention_reference(torch, q, ks, vs, pk, pv, mask, B, H, P, step0):
    """fp32 masked MQA attention written out per sample (skipping masked keys)."""
    out = {}
    for b in range(B):
        valid = mask[b].nonzero().flatten() if P > 0 else torch.zeros(0, dtype=torch.long, device=q.device)
        arows = [B + b * H + j for j in range(H)]
        K = torch.cat([pk[b][valid].float(), ks[b:b + 1].float(), ks[arows].float()])
        V = torch.cat([pv[b][valid].float(), vs[b:b + 1].float(), vs[arows].float()])
        nv = valid.numel()
        toks = ([b] if step0 else []) + arows
        for t in toks:
            qq = q[t].float().view(8, 256)
            lim = nv + 1 if (step0 and t == b) else K.shape[0]
            p = torch.softmax(qq @ K[:lim].T / 16.0, dim=-1)
            out[t] = (p @ V[:lim]).reshape(-1)
    return out


@pytest.mark.parametrize("B,H,P,masked,step0", [
    (1, 50, 816, 10, 1), (1, 50, 816, 10, 0), (3, 50, 77, 30, 1), (8, 10, 560, 0, 0),
    (2, 50, 0, 0, 1), (5, 50, 300, 150, 0)])
@pytest.mark.parametrize("impl", [0, 1, 2], ids=["simt", "tc_split", "tc"])
def test_attention_kernels_match_reference(B, H, P, masked, step0, impl):
    torch = _torch()
    from vla_flow_matching_b200 import build, pi0x
    build.build()
    g = torch.Generator(device="cuda").manual_seed(B * 1000 + P + H)
    R = B + B * H
    q = (0.6 * torch.randn(R, 2048, device="cuda", generator=g)).to(torch.bfloat16)
    ks = (0.6 * torch.randn(R, 256, device="cuda", generator=g)).to(torch.bfloat16)
    vs = torch.randn(R, 256, device="cuda", generator=g).to(torch.bfloat16)
    pk = torch.randn(B, max(P, 1), 256, device="cuda", generator=g).to(torch.bfloat16)
    pv = torch.randn(B, max(P, 1), 256, device="cuda", generator=g).to(torch.bfloat16)
    mask = torch.ones(B, max(P, 1), dtype=torch.uint8, device="cuda")
    for b in range(B):
        if masked:
            cut = P - (masked * (b + 1)) % max(P, 1)
            mask[b, cut:] = 0
        if P > 8:
            mask[b, 3 + b] = 0   # a hole
    out = torch.zeros(R, 2048, dtype=torch.bfloat16, device="cuda")
    pi0x.debug_attention(q, ks, vs, pk, pv, mask, B, H, P, step0, out, impl=impl,
                         stream=torch.cuda.current_stream().cuda_stream)
    ref = _attention_reference(torch, q, ks, vs, pk, pv, mask, B, H, P, step0)
    for t, r in ref.items():
        d = (out[t].float() - r).abs().max().item()
        assert d <= 1.5e-2 * max(1.0, r.abs().max().item()), (t, d)
    rows = sorted(ref)
    got = out[rows].float()
    want = torch.stack([ref[t] for t in rows])
    assert (torch.linalg.norm(got - want) / torch.linalg.norm(want)).item() < 6e-3


@pytest.mark.parametrize("M,N,K,bn,splits", [
    (128, 128, 64, 128, 1),      # one tile, one K block
    (51, 2560, 1024, 256, 1),    # B=1 suffix rows, QKV shape
    (300, 1024, 2048, 128, 1),   # ragged M over three tiles, O-proj shape
    (77, 256, 4096, 64, 1),      # ragged tail, long K (ring wraps many times)
    (1000, 8192, 1024, 256, 1),  # gate/up shape
    (40, 256, 512, 32, 1),       # narrowest tile
    (51, 2560, 1024, 64, 3),     # split-K as planned for B=1 QKV (uneven last split)
    (51, 1024, 4096, 64, 8),     # split-K as planned for B=1 down-proj
    (200, 512, 2048, 64, 9),     # two row tiles, uneven splits
])
def test_tc_gemm_matches_fp32_matmul(M, N, K, bn, splits):
    torch = _torch()
    from vla_flow_matching_b200 import build, pi0x
    build.build()
    g = torch.Generator(device="cuda").manual_seed(M * 7 + N)
    A = torch.randn(M, K, device="cuda", generator=g).to(torch.bfloat16)
    W = (0.05 * torch.randn(N, K, device="cuda", generator=g)).to(torch.bfloat16)
    D = torch.full((M, N), float("nan"), device="cuda")
    for _ in range(2):   # twice: the split-K counters must be back at zero
        pi0x.debug_gemm_bf16(A, W, D, bn=bn, splits=splits, stream=torch.cuda.current_stream().cuda_stream)
    torch.backends.cuda.matmul.allow_tf32 = False
    ref = A.float() @ W.float().T
    err = (D - ref).abs().max().item()
    scale = ref.abs().max().item()
    assert err <= 2e-5 * scale * (K / 64) ** 0.5 + 1e-5, (err, scale)
