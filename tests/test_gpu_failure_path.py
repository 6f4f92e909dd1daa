"""Device-side failure detection without a GPU fault.

Every wait in the kernels is bounded; when one runs out, the kernel records a code in
the library's error word and returns, so the host sees a status instead of a hung
GPU.  The self-test kernel waits on a barrier that nothing arrives at, with a short
limit, and the context must stay usable afterwards.
"""
import numpy as np
import pytest
import torch

import oracle
import shifted_sparse_attention_s2attn_b200 as s2
from shifted_sparse_attention_s2attn_b200.synthetic import f32_to_bf16_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def test_bounded_wait_times_out_and_reports():
    s2.clear_device_error()
    s2.s2attn_selftest_bounded_wait(20000)  # 20 ms
    torch.cuda.synchronize()
    rc, detail = s2.get_device_error()
    assert rc == -5 and detail == (3 << 8) | 1
    s2.clear_device_error()
    assert s2.get_device_error() == (0, 0)


def test_context_usable_after_timeout():
    s2.clear_device_error()
    s2.s2attn_selftest_bounded_wait(5000)
    torch.cuda.synchronize()
    assert s2.get_device_error()[0] == -5
    s2.clear_device_error()
    B, N, H, D, G, sh = 1, 512, 2, 128, 256, 1
    rng = np.random.default_rng(5)
    bits = [f32_to_bf16_bits(rng.standard_normal((B, N, H, D)).astype(np.float32)) for _ in range(3)]
    q, k, v = (torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).cuda() for b in bits)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    s2.s2attn_fwd(q, k, v, o, lse, G, sh)
    torch.cuda.synchronize()
    assert s2.get_device_error()[0] == 0
    ro, _ = oracle.s2attn_fwd(bits[0], bits[1], bits[2], G, sh)
    assert np.abs(o.float().cpu().numpy() - ro).max() <= 2e-2


def test_selftest_rejects_bad_limits():
    with pytest.raises(s2.S2AttnError):
        s2.s2attn_selftest_bounded_wait(0)
    with pytest.raises(s2.S2AttnError):
        s2.s2attn_selftest_bounded_wait(2_000_000)
