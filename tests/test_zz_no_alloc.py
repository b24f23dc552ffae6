"""pi0x_attention_noalloc: the attention entry point that allocates no device memory.

Some callers cannot call cudaMalloc while they run: a real-time robot control loop
(cudaMalloc can block for milliseconds and synchronises the device) or an
application whose device memory belongs to its own pool.  For them the library
keeps this one variant of the tcgen05 attention, whose scratch lives in a static
device array.  This test calls it through the C ABI twice in a row and checks each
result against an independent fp32 attention written out per sample and against
the allocating entry point (pi0x_debug_attention, tcgen05 path), within the
tolerance of the attention kernel tests; it also checks that a call leaves the
device's free memory unchanged.  The file name makes pytest collect it last.
"""
import pytest

from tests.test_gpu_kernels import _attention_reference

pytestmark = pytest.mark.gpu


def _torch():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _inputs(torch, B, H, P, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    R = B + B * H
    Pb = max(P, 1)
    q = (0.6 * torch.randn(R, 2048, device="cuda", generator=g)).to(torch.bfloat16)
    ks = (0.6 * torch.randn(R, 256, device="cuda", generator=g)).to(torch.bfloat16)
    vs = torch.randn(R, 256, device="cuda", generator=g).to(torch.bfloat16)
    pk = torch.randn(B, Pb, 256, device="cuda", generator=g).to(torch.bfloat16)
    pv = torch.randn(B, Pb, 256, device="cuda", generator=g).to(torch.bfloat16)
    mask = torch.ones(B, Pb, dtype=torch.uint8, device="cuda")
    if P > 10:
        mask[:, P - 10:] = 0
        mask[:, 5] = 0
    return q, ks, vs, pk, pv, mask


def _check_rows(torch, out, ref, tol_scale=1.5e-2):
    for t, r in ref.items():
        d = (out[t].float() - r).abs().max().item()
        assert d <= tol_scale * max(1.0, r.abs().max().item()), (t, d)
    rows = sorted(ref)
    got = out[rows].float()
    want = torch.stack([ref[t] for t in rows])
    assert (torch.linalg.norm(got - want) / torch.linalg.norm(want)).item() < 6e-3


@pytest.mark.parametrize("B,H,P,step0", [(1, 50, 816, 1), (1, 50, 816, 0), (4, 10, 560, 1), (8, 50, 816, 1),
                                         (2, 50, 0, 1)])
def test_noalloc_attention_matches_reference_twice(B, H, P, step0):
    torch = _torch()
    from vla_flow_matching_b200 import build, pi0x
    build.build()
    stream = torch.cuda.current_stream().cuda_stream
    R = B + B * H
    for call in range(2):
        q, ks, vs, pk, pv, mask = _inputs(torch, B, H, P, seed=100 * call + B + P)
        out = torch.zeros(R, 2048, dtype=torch.bfloat16, device="cuda")
        pi0x.attention_noalloc(q, ks, vs, pk, pv, mask, B, H, P, step0, out, stream=stream)
        ref = _attention_reference(torch, q, ks, vs, pk, pv, mask, B, H, P, step0)
        _check_rows(torch, out, ref)
        alloc = torch.zeros(R, 2048, dtype=torch.bfloat16, device="cuda")
        pi0x.debug_attention(q, ks, vs, pk, pv, mask, B, H, P, step0, alloc, impl=1, stream=stream)
        rows = sorted(ref)
        d = (out[rows].float() - alloc[rows].float()).abs().max().item()
        assert d <= 1.5e-2 * max(1.0, alloc[rows].float().abs().max().item()), (call, d)


def test_noalloc_call_leaves_free_device_memory_unchanged():
    torch = _torch()
    from vla_flow_matching_b200 import build, pi0x
    build.build()
    stream = torch.cuda.current_stream().cuda_stream
    B, H, P = 1, 50, 816
    q, ks, vs, pk, pv, mask = _inputs(torch, B, H, P, seed=7)
    out = torch.zeros(B + B * H, 2048, dtype=torch.bfloat16, device="cuda")
    pi0x.attention_noalloc(q, ks, vs, pk, pv, mask, B, H, P, 1, out, stream=stream)  # loads the module
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    pi0x.attention_noalloc(q, ks, vs, pk, pv, mask, B, H, P, 1, out, stream=stream)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0


def test_noalloc_rejects_problems_larger_than_its_scratch():
    torch = _torch()
    from vla_flow_matching_b200 import build, pi0x
    build.build()
    B, H, P = 2048, 50, 8192   # the valid-index list alone needs 64 MiB; rejected before any launch
    dummy = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(pi0x.Pi0xError) as e:
        pi0x.attention_noalloc(dummy, dummy, dummy, dummy, dummy, dummy, B, H, P, 1, dummy)
    assert e.value.status == pi0x.PI0X_EINVAL
