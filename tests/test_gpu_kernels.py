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


@pytest.mark.parametrize("M,N,K,bn", [
    (128, 128, 64, 128),      # one tile, one K block
    (51, 2560, 1024, 256),    # B=1 suffix rows, QKV shape
    (300, 1024, 2048, 128),   # ragged M over three tiles, O-proj shape
    (77, 256, 4096, 64),      # ragged tail, long K (ring wraps many times)
    (1000, 8192, 1024, 256),  # gate/up shape
])
def test_tc_gemm_matches_fp32_matmul(M, N, K, bn):
    torch = _torch()
    from vla_flow_matching_b200 import build, pi0x
    build.build()
    g = torch.Generator(device="cuda").manual_seed(M * 7 + N)
    A = torch.randn(M, K, device="cuda", generator=g).to(torch.bfloat16)
    W = (0.05 * torch.randn(N, K, device="cuda", generator=g)).to(torch.bfloat16)
    D = torch.full((M, N), float("nan"), device="cuda")
    pi0x.debug_gemm_bf16(A, W, D, bn=bn, stream=torch.cuda.current_stream().cuda_stream)
    torch.backends.cuda.matmul.allow_tf32 = False
    ref = A.float() @ W.float().T
    err = (D - ref).abs().max().item()
    scale = ref.abs().max().item()
    assert err <= 2e-5 * scale * (K / 64) ** 0.5 + 1e-5, (err, scale)
