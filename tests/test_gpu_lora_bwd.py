"""GPU parity of the LoRA-projection backward (lora_proj_bwd) against the fp64 oracle:
ragged token counts, K and ranks (0, 5, 8, 16, 64) on whole tensors, and the LLaMA2-7B
q/k/v layer at 32k tokens (dx on sampled rows, dA and dB whole)."""
import numpy as np
import pytest
import torch

import oracle
import shifted_sparse_attention_s2attn_b200 as s2
from shifted_sparse_attention_s2attn_b200.synthetic import LORA_LLAMA2_7B, f32_to_bf16_bits, make_lora_inputs
from parity_utils import bits_to_device, bf16_tensor_to_f64, rel_l2

pytestmark = pytest.mark.gpu


def _dy(parts, T, n_out, seed):
    return f32_to_bf16_bits(np.random.default_rng(seed).standard_normal((parts, T, n_out)).astype(np.float32))


def _run(x, w, a, b, dy, parts, s):
    X, W, DY = bits_to_device(x), bits_to_device(w), bits_to_device(dy)
    A = None if a is None else bits_to_device(a)
    Bm = None if b is None else bits_to_device(b)
    T, K = X.shape
    n_out = W.shape[0] // parts
    r = 0 if A is None else A.shape[0] // parts
    dx = torch.empty_like(X)
    da = None if A is None else torch.empty_like(A)
    db = None if Bm is None else torch.empty_like(Bm)
    ws = torch.empty(s2.lora_proj_bwd_workspace_bytes(T, K, n_out, parts, r), dtype=torch.uint8, device="cuda")
    s2.lora_proj_bwd(X, W, A, Bm, DY, dx, da, db, parts, s, ws)
    torch.cuda.synchronize()
    rc, detail = s2.get_device_error()
    assert rc == 0, f"device error word set: {detail:#x}"
    return dx, da, db


@pytest.mark.parametrize("T,K,n_out,parts,r", [
    (300, 520, 256, 3, 8), (129, 64, 512, 1, 5), (256, 256, 256, 2, 64), (1000, 264, 256, 3, 16),
    (300, 520, 256, 3, 0),
])
def test_lora_bwd_matches_oracle(T, K, n_out, parts, r):
    x, w, a, b = make_lora_inputs(T, K, n_out, parts, r, seed=T + r)
    dy = _dy(parts, T, n_out, T)
    dx, da, db = _run(x, w, a, b, dy, parts, 2.0)
    rdx, rda, rdb = oracle.lora_proj_bwd(x, w, a, b, dy, 2.0, parts)
    # bf16 rounding of g, u and the outputs (2^-8 each); fp32 accumulation over <= 32k terms
    assert rel_l2(bf16_tensor_to_f64(dx), rdx) <= 1e-2
    if r:
        assert rel_l2(bf16_tensor_to_f64(da), rda) <= 1e-2
        assert rel_l2(bf16_tensor_to_f64(db), rdb) <= 1e-2


def test_lora_bwd_llama2_7b_32k_qkv():
    T, c = 32768, LORA_LLAMA2_7B
    x, w, a, b = make_lora_inputs(T, c["K"], c["n_out"], 3, c["r"], seed=2)
    dy = _dy(3, T, c["n_out"], 3)
    dx, da, db = _run(x, w, a, b, dy, 3, c["scaling"])
    rows = np.unique(np.r_[0, 127, 128, T // 2, T - 1, np.random.default_rng(1).choice(T, 27, replace=False)])
    rdx, rda, rdb = oracle.lora_proj_bwd(x, w, a, b, dy, c["scaling"], 3)
    assert rel_l2(bf16_tensor_to_f64(dx)[rows], rdx[rows]) <= 1e-2
    assert rel_l2(bf16_tensor_to_f64(da), rda) <= 1e-2
    assert rel_l2(bf16_tensor_to_f64(db), rdb) <= 1e-2
