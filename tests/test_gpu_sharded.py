"""The sequence-sharded path on one GPU with this library's kernels: one rank's halo is its
own first G/2 rows (the cyclic wrap), so the shifted heads run as plain groups of the local
layout.  Its results must equal the direct call with the shift: the forward bit for bit
(every group sees the same rows in the same order), the backward within the bf16 bounds.
Runs with more than one GPU exchange the halos over NCCL; every run here has one GPU."""
import numpy as np
import pytest
import torch

import shifted_sparse_attention_s2attn_b200 as s2
from shifted_sparse_attention_s2attn_b200.sharded import sharded_bwd, sharded_fwd
from shifted_sparse_attention_s2attn_b200.synthetic import f32_to_bf16_bits
from parity_utils import TOL_REL_L2_BF16, bits_to_device, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    s2.clear_device_error()
    yield


@pytest.mark.parametrize("N,H,G,sh", [(1024, 2, 512, 1), (2048, 4, 256, 2)])
def test_one_rank_sharded_equals_direct(N, H, G, sh):
    B, D = 1, 128
    rng = np.random.default_rng(5)
    q, k, v, do = (bits_to_device(f32_to_bf16_bits(rng.standard_normal((B, N, H, D)).astype(np.float32)))
                   for _ in range(4))
    o, lse = sharded_fwd(q, k, v, G, sh)
    o_ref = torch.empty_like(q)
    lse_ref = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    s2.s2attn_fwd(q, k, v, o_ref, lse_ref, G, sh)
    dq, dk, dv = sharded_bwd(q, k, v, o, do, lse, G, sh)
    dq_r, dk_r, dv_r = (torch.empty_like(q) for _ in range(3))
    ws = torch.empty(s2.s2attn_bwd_workspace_bytes(B, N, H, D), dtype=torch.uint8, device="cuda")
    s2.s2attn_bwd(q, k, v, o_ref, do, lse_ref, dq_r, dk_r, dv_r, G, sh, ws)
    torch.cuda.synchronize()
    rc, detail = s2.get_device_error()
    assert rc == 0, f"device error word set: {detail:#x}"
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
    for got, ref in ((dq, dq_r), (dk, dk_r), (dv, dv_r)):
        assert rel_l2(got.float().cpu().numpy(), ref.float().cpu().numpy().astype(np.float64)) <= TOL_REL_L2_BF16 / 10
