"""One LongLoRA attention layer (layer.py) on the GPU against the fp64 oracle composed step
by step: the LoRA-adapted q/k/v projection, RoPE-PI on q and k, S^2-Attn, the LoRA-adapted o
projection, and the backward of all four (W frozen).  The oracle keeps every intermediate
exact; the CUDA path rounds q, k, v, o, the attention gradients and the projection
outputs to bf16 between the calls, so the bound is the bf16 gradient tolerance of the
attention (relative L2 2e-2 per tensor), for the output and for every gradient.

The forward has no separate rotation pass: RoPE-PI runs in the q/k projection's epilogue,
and the rotated q, k equal the unfused projection followed by rope_pi_apply, bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import shifted_sparse_attention_s2attn_b200 as s2
from shifted_sparse_attention_s2attn_b200.layer import LayerBuffers, LayerShape, LayerWeights, layer_bwd, layer_fwd
from shifted_sparse_attention_s2attn_b200.synthetic import f32_to_bf16_bits, make_lora_inputs
from parity_utils import TOL_REL_L2_BF16, bf16_tensor_to_f64, bits_to_device, device_to_bits, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    s2.clear_device_error()
    yield


def _oracle_layer(s, x, w_qkv, a_qkv, b_qkv, w_o, a_o, b_o, dy):
    T, n = s.T, s.width
    qkv = oracle.lora_proj(x, w_qkv, a_qkv, b_qkv, s.scaling, 3).reshape(3, s.B, s.N, s.H, s.D)
    q, k, v = oracle.rope_pi_f64(qkv[0], s.pos_scale, s.base), oracle.rope_pi_f64(qkv[1], s.pos_scale, s.base), qkv[2]
    o, _ = oracle.s2attn_fwd(q, k, v, s.G, s.shift_heads)
    y = oracle.lora_proj(o.reshape(T, n), w_o, a_o, b_o, s.scaling, 1)
    do, da_o, db_o = oracle.lora_proj_bwd(o.reshape(T, n), w_o, a_o, b_o, dy, s.scaling, 1)
    dq, dk, dv = oracle.s2attn_bwd(q, k, v, do.reshape(s.B, s.N, s.H, s.D), s.G, s.shift_heads)
    dqkv = np.stack([oracle.rope_pi_bwd_f64(dq, s.pos_scale, s.base), oracle.rope_pi_bwd_f64(dk, s.pos_scale, s.base),
                     dv]).reshape(3, T, n)
    dx, da, db = oracle.lora_proj_bwd(x, w_qkv, a_qkv, b_qkv, dqkv, s.scaling, 3)
    return {"y": y, "dx": dx, "da_qkv": da, "db_qkv": db, "da_o": da_o, "db_o": db_o}


@pytest.mark.parametrize("B,N,H,G,sh,r", [(1, 1024, 2, 512, 1, 8), (2, 512, 2, 256, 2, 16)])
def test_layer_matches_oracle(B, N, H, G, sh, r):
    D = 128
    s = LayerShape(B=B, N=N, H=H, D=D, G=G, shift_heads=sh, r=r, scaling=2.0, pos_scale=0.5)
    T, n = s.T, s.width
    x, w_qkv, a_qkv, b_qkv = make_lora_inputs(T, n, n, 3, r, seed=N + r)
    _, w_o, a_o, b_o = make_lora_inputs(T, n, n, 1, r, seed=N + r + 1)
    dy = f32_to_bf16_bits(np.random.default_rng(N).standard_normal((1, T, n)).astype(np.float32))
    dev = {k: bits_to_device(v) for k, v in dict(x=x, w_qkv=w_qkv, a_qkv=a_qkv, b_qkv=b_qkv, w_o=w_o, a_o=a_o,
                                                 b_o=b_o, dy=dy).items()}
    w = LayerWeights(dev["w_qkv"], dev["w_o"], dev["a_qkv"], dev["b_qkv"], dev["a_o"], dev["b_o"])
    buf = LayerBuffers(s, "cuda")
    layer_fwd(s, w, dev["x"], buf)
    layer_bwd(s, w, dev["x"], dev["dy"], buf)
    torch.cuda.synchronize()
    rc, detail = s2.get_device_error()
    assert rc == 0, f"device error word set: {detail:#x}"

    # the fused rotation equals the projection followed by rope_pi_apply, bit for bit
    plain = torch.empty_like(buf.qkv)
    ws = torch.empty(max(256, s2.lora_proj_workspace_bytes(T, n, n, 3, r)), dtype=torch.uint8, device="cuda")
    s2.lora_proj_fwd(dev["x"], w.w_qkv, w.a_qkv, w.b_qkv, plain, 3, s.scaling, workspace=ws)
    s2.rope_pi_apply(plain[0], plain[1], s.pos_scale, s.base)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(device_to_bits(plain), device_to_bits(buf.qkv))

    ref = _oracle_layer(s, x, w_qkv, a_qkv, b_qkv, w_o, a_o, b_o, dy)
    got = {"y": buf.y, "dx": buf.dx, "da_qkv": buf.da_qkv, "db_qkv": buf.db_qkv, "da_o": buf.da_o, "db_o": buf.db_o}
    for name, t in got.items():
        e = rel_l2(bf16_tensor_to_f64(t), ref[name])
        assert e <= TOL_REL_L2_BF16, (name, e)
