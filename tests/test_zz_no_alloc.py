"""pi0x_attention_noalloc: the attention entry point that allocates no device memory.

Some callers (a real-time robot control loop, an application whose device memory
belongs to its own pool) cannot call cudaMalloc while they run.  For them the
library keeps this one variant of the tcgen05 attention whose scratch lives in a
static device array.  This test calls it through the C ABI twice in a row and
checks each result against the allocating entry point (pi0x_debug_attention,
tcgen05 path) within the tolerance of the attention kernel tests.  The file name
makes pytest collect it last.
"""
import ctypes

import pytest

pytestmark = pytest.mark.gpu


def _torch():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


def _inputs(torch, B, H, P, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    R = B + B * H
    q = (0.6 * torch.randn(R, 2048, device="cuda", generator=g)).to(torch.bfloat16)
    ks = (0.6 * torch.randn(R, 256, device="cuda", generator=g)).to(torch.bfloat16)
    vs = torch.randn(R, 256, device="cuda", generator=g).to(torch.bfloat16)
    pk = torch.randn(B, P, 256, device="cuda", generator=g).to(torch.bfloat16)
    pv = torch.randn(B, P, 256, device="cuda", generator=g).to(torch.bfloat16)
    mask = torch.ones(B, P, dtype=torch.uint8, device="cuda")
    mask[:, P - 10:] = 0
    mask[:, 5] = 0
    return q, ks, vs, pk, pv, mask


@pytest.mark.parametrize("B,H,P,step0", [(1, 50, 816, 1), (1, 50, 816, 0), (4, 10, 560, 1), (8, 50, 816, 1)])
def test_noalloc_attention_matches_allocating_entry_point(B, H, P, step0):
    torch = _torch()
    from vla_flow_matching_b200 import build, pi0x
    build.build()
    lib = pi0x.load()
    f = lib.pi0x_attention_noalloc
    f.argtypes = [ctypes.c_void_p] * 6 + [ctypes.c_int] * 4 + [ctypes.c_void_p] * 2
    f.restype = ctypes.c_int
    stream = torch.cuda.current_stream().cuda_stream
    R = B + B * H
    for call in range(2):
        q, ks, vs, pk, pv, mask = _inputs(torch, B, H, P, seed=100 * call + B + P)
        ref = torch.zeros(R, 2048, dtype=torch.bfloat16, device="cuda")
        pi0x.debug_attention(q, ks, vs, pk, pv, mask, B, H, P, step0, ref, impl=1, stream=stream)
        out = torch.zeros(R, 2048, dtype=torch.bfloat16, device="cuda")
        st = f(q.data_ptr(), ks.data_ptr(), vs.data_ptr(), pk.data_ptr(), pv.data_ptr(), mask.data_ptr(),
               B, H, P, step0, out.data_ptr(), ctypes.c_void_p(stream))
        assert st == pi0x.PI0X_OK, lib.pi0x_status_string(st)
        rows = list(range(B)) if step0 else []
        rows += list(range(B, R))
        d = (out[rows].float() - ref[rows].float()).abs().max().item()
        scale = max(1.0, ref[rows].float().abs().max().item())
        assert d <= 1.5e-2 * scale, (call, d)


def test_noalloc_rejects_problems_larger_than_its_scratch():
    torch = _torch()
    from vla_flow_matching_b200 import build, pi0x
    build.build()
    f = pi0x.load().pi0x_attention_noalloc
    f.argtypes = [ctypes.c_void_p] * 6 + [ctypes.c_int] * 4 + [ctypes.c_void_p] * 2
    f.restype = ctypes.c_int
    B, H, P = 2048, 50, 8192   # the valid-index list alone needs 64 MiB; rejected before any launch
    dummy = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    st = f(dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr(),
           dummy.data_ptr(), B, H, P, 1, dummy.data_ptr(), None)
    assert st == pi0x.PI0X_EINVAL
