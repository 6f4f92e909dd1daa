"""The allocation-free backward entry point against the workspace-taking one.

s2attn_bwd_noalloc serves callers that cannot allocate device memory on the call
path (their allocator already holds the device, or their enqueue step must not
allocate), so it takes its scratch from a fixed array inside the library.  This
file is collected last on purpose; it must pass alone in a fresh process and after
the other tests.  Both calls go through the C ABI with identical inputs; the second
call checks that scratch contents left by the first do not leak into the result.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

# The tolerance the other bf16 backward parity tests use (relative L2 per tensor);
# both paths run the same kernels, so in practice they agree far more closely.
TOL_REL_L2 = 2e-2


def _rel_l2(a, b):
    a, b = a.double(), b.double()
    return float((a - b).norm() / b.norm().clamp_min(1e-30))


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import shifted_sparse_attention_s2attn_b200 as s2
    return s2.capi()


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("B,N,H,G,sh", [(1, 2048, 4, 1024, 2), (2, 1024, 2, 256, 1)])
def test_noalloc_matches_workspace_backward(lib, B, N, H, G, sh):
    D = 128
    gen = torch.Generator(device="cpu").manual_seed(1234 + N)
    q, k, v, do = (torch.randn((B, N, H, D), generator=gen).to(torch.bfloat16).cuda() for _ in range(4))
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    assert lib.s2attn_fwd(_p(q), _p(k), _p(v), _p(o), _p(lse), B, N, H, D, G, sh, stream) == 0

    ref = [torch.empty_like(q) for _ in range(3)]
    ws_bytes = lib.s2attn_bwd_workspace_bytes(B, N, H, D)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    assert lib.s2attn_bwd(_p(q), _p(k), _p(v), _p(o), _p(do), _p(lse), *(_p(t) for t in ref), B, N, H, D, G, sh,
                          _p(ws), ws_bytes, stream) == 0

    for call in range(2):  # two calls in a row: the shared scratch must not carry over
        out = [torch.full_like(q, float("nan")) for _ in range(3)]
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        assert lib.s2attn_bwd_noalloc(_p(q), _p(k), _p(v), _p(o), _p(do), _p(lse), *(_p(t) for t in out),
                                      B, N, H, D, G, sh, stream) == 0
        torch.cuda.synchronize()
        if call == 1:
            # the first call on the device may load the module that holds the scratch (lazy
            # loading); from then on a call takes no device memory at all
            assert torch.cuda.mem_get_info()[0] == free_before
        for name, got, want in zip(("dq", "dk", "dv"), out, ref):
            assert torch.isfinite(got).all(), name
            err = _rel_l2(got.float(), want.float())
            assert err <= TOL_REL_L2, (name, err)
    detail = ctypes.c_int(0)
    assert lib.s2attn_get_device_error(ctypes.byref(detail)) == 0, hex(detail.value)


def test_noalloc_rejects_problems_beyond_the_scratch(lib):
    # B*N*H*D*4 bytes of fp32 accumulator: 1 x 65536 x 4 x 128 x 4 = 128 MiB > 64 MiB
    t = torch.zeros(16, dtype=torch.uint8, device="cuda")
    p = _p(t)
    rc = lib.s2attn_bwd_noalloc(p, p, p, p, p, p, p, p, p, 1, 65536, 4, 128, 8192, 2, None)
    assert rc == -3
