"""CPU checks of the Python binding's argument checks.  The C entry points see only
pointers, so the binding checks every tensor's element count, dtype and contiguity
against the call's shape, and checks that it lives on a CUDA device (last).  With CPU
tensors a call whose extents are right therefore fails only on the device check, and one
whose extents are wrong fails before it; nothing reaches the library.  The shapes below
are those of the library's own callers (tests, smoke, bench, the sharded path)."""
import pytest
import torch

import shifted_sparse_attention_s2attn_b200 as s2

BF, F32 = torch.bfloat16, torch.float32
ON_DEVICE = "CUDA device"


def _attn(B=1, N=256, H=2, D=128, dtype=BF):
    t = lambda: torch.zeros((B, N, H, D), dtype=dtype)  # noqa: E731
    return dict(q=t(), k=t(), v=t(), o=t(), dout=t(), dq=t(), dk=t(), dv=t(),
                lse=torch.zeros((B, H, N), dtype=F32), ws=torch.zeros(1024, dtype=torch.uint8))


def _only_device_check_fails(fn, *args, **kw):
    with pytest.raises(ValueError, match=ON_DEVICE):
        fn(*args, **kw)


def _extent_check_fails(fn, *args, **kw):
    with pytest.raises(ValueError) as e:
        fn(*args, **kw)
    assert ON_DEVICE not in str(e.value), str(e.value)


def test_forward_and_backward_accept_their_shapes():
    a = _attn()
    _only_device_check_fails(s2.s2attn_fwd, a["q"], a["k"], a["v"], a["o"], a["lse"], 128, 1)
    _only_device_check_fails(s2.s2attn_bwd, a["q"], a["k"], a["v"], a["o"], a["dout"], a["lse"], a["dq"], a["dk"],
                             a["dv"], 128, 1, a["ws"])
    _only_device_check_fails(s2.s2attn_bwd_noalloc, a["q"], a["k"], a["v"], a["o"], a["dout"], a["lse"], a["dq"],
                             a["dk"], a["dv"], 128, 1)
    f = _attn(N=90, H=3, D=40, dtype=F32)
    _only_device_check_fails(s2.s2attn_fwd_f32, f["q"], f["k"], f["v"], f["o"], f["lse"], 18, 1)
    _only_device_check_fails(s2.s2attn_bwd_f32, f["q"], f["k"], f["v"], f["o"], f["dout"], f["lse"], f["dq"],
                             f["dk"], f["dv"], 18, 1, f["ws"])


def test_split_backward_accepts_flat_workspace_views():
    """The bench passes dq_acc and delta as flat fp32 views of the backward workspace."""
    B, N, H, D = 1, 256, 2, 128
    a = _attn(B, N, H, D)
    ws = torch.zeros(B * N * H * D * 4 + 256 + B * H * N * 4, dtype=torch.uint8)
    dq_acc = ws[: B * N * H * D * 4].view(F32)
    off = ((B * N * H * D * 4 + 255) // 256) * 256
    delta = ws[off: off + B * H * N * 4].view(F32)
    _only_device_check_fails(s2.s2attn_bwd_preprocess, a["o"], a["dout"], delta, dq_acc)
    _only_device_check_fails(s2.s2attn_bwd_main, a["q"], a["k"], a["v"], a["dout"], a["lse"], delta, dq_acc,
                             a["dk"], a["dv"], 128, 1)
    _only_device_check_fails(s2.s2attn_bwd_dq_convert, dq_acc, a["dq"])


def test_decode_and_rope_accept_their_shapes():
    B, M, N, H, D = 2, 3, 1000, 4, 128
    q = torch.zeros((B, M, H, D), dtype=BF)
    k, v = torch.zeros((B, N, H, D), dtype=BF), torch.zeros((B, N, H, D), dtype=BF)
    o, lse = torch.zeros_like(q), torch.zeros((B, H, M), dtype=F32)
    ws = torch.zeros(4096, dtype=torch.uint8)
    _only_device_check_fails(s2.s2attn_decode, q, k, v, o, lse, ws)
    _only_device_check_fails(s2.rope_pi_apply, k, v, 0.5)
    _only_device_check_fails(s2.rope_pi_apply, None, k, 0.5)
    _only_device_check_fails(s2.rope_pi_apply_offset, q, None, 997, 0.5)


def test_mismatched_extents_are_rejected_before_the_device_check():
    a = _attn()
    short = torch.zeros((1, 255, 2, 128), dtype=BF)
    _extent_check_fails(s2.s2attn_fwd, a["q"], short, a["v"], a["o"], a["lse"], 128, 1)       # k too short
    _extent_check_fails(s2.s2attn_fwd, a["q"], a["k"], a["v"], a["o"], a["lse"][:, :, :128].contiguous(), 128, 1)
    _extent_check_fails(s2.s2attn_fwd, a["q"], a["k"], a["v"], a["o"].float(), a["lse"], 128, 1)   # fp32 o
    _extent_check_fails(s2.s2attn_bwd, a["q"], a["k"], a["v"], a["o"], a["dout"], a["lse"], a["dq"], short,
                        a["dv"], 128, 1, a["ws"])
    _extent_check_fails(s2.s2attn_fwd_f32, a["q"], a["k"], a["v"], a["o"], a["lse"], 128, 1)    # bf16 on fp32 path
    q = torch.zeros((2, 3, 4, 128), dtype=BF)
    k = torch.zeros((2, 1000, 4, 128), dtype=BF)
    lse = torch.zeros((2, 4, 3), dtype=F32)
    ws = torch.zeros(4096, dtype=torch.uint8)
    _extent_check_fails(s2.s2attn_decode, q, torch.zeros((2, 1000, 2, 128), dtype=BF), k, q.clone(), lse, ws)
    _extent_check_fails(s2.s2attn_decode, q, k, k[:, :999].contiguous(), q.clone(), lse, ws)     # v too short
    _extent_check_fails(s2.rope_pi_apply, a["q"], short, 0.5)
    nc = torch.zeros((1, 2, 256, 128), dtype=BF).transpose(1, 2)                                 # not contiguous
    _extent_check_fails(s2.s2attn_fwd, a["q"], nc, a["v"], a["o"], a["lse"], 128, 1)


def test_halo_copies_check_their_buffers():
    """The sequence-sharded path's halo copies: one [B, G/2, shift_heads, D] buffer per
    [B,N,H,D] tensor, one [B, shift_heads, G/2] buffer per [B,H,N] lse."""
    B, N, H, D, G, sh = 2, 1024, 4, 128, 512, 2
    xs = [torch.zeros((B, N, H, D), dtype=BF) for _ in range(3)]
    bufs = [torch.zeros((B, G // 2, sh, D), dtype=BF) for _ in range(3)]
    _only_device_check_fails(s2.s2attn_halo_rows, xs, bufs, True, G, sh)
    lse, lbuf = torch.zeros((B, H, N), dtype=F32), torch.zeros((B, sh, G // 2), dtype=F32)
    _only_device_check_fails(s2.s2attn_halo_lse, [lse], [lbuf], False, G, sh)
    _extent_check_fails(s2.s2attn_halo_rows, xs, bufs[:2] + [torch.zeros((B, G // 2, sh + 1, D), dtype=BF)], True, G,
                        sh)                                                                        # buffer too big
    _extent_check_fails(s2.s2attn_halo_lse, [lse], [lbuf[:, :1].contiguous()], True, G, sh)        # buffer too small
    with pytest.raises(ValueError):
        s2.s2attn_halo_rows(xs, bufs[:2], True, G, sh)                                             # unequal lists
