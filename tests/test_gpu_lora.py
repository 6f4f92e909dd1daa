"""GPU parity of the LoRA-adapted projections (lora_proj_fwd) against the fp64 oracle,
through the C ABI ("LongLoRA paper notes", section 3.2: adapters on the Q, K, V and O
projections; section 3.4: RoPE with position interpolation on q and k).

Tolerance, per element, from the arithmetic of the CUDA path: y is rounded once to bf16
(8 significant bits: at most 2^-8 |y|), the rank-r intermediate is held in bf16 (at most
2^-8 of each adapter product s*u_j*B_cj), and the fp32 accumulation over K stays far below
2^-14 of sum_k |x_k W_ck|.  The rounding bounds are doubled:
    |y - y_ref| <= 2^-7 |y_ref| + 2^-7 sum_j |s u_j B_cj| + 2^-14 sum_k |x_k W_ck| + 1e-6.
A rotated pair (y1, y2) mixes the errors of both elements (|cos|, |sin| <= 1), adds its own
bf16 rounding, and its angle differs from the exact one by the fp32 rounding of
t * pos_scale * theta (below 2^-11 radian for positions up to 2^12 after interpolation):
    |y1' - y1'_ref| <= tol(y1) + tol(y2) + 2^-10 (|y1_ref| + |y2_ref|) + 2^-7 |y1'_ref|.
The fused RoPE is also compared bit for bit with the projection followed by rope_pi_apply
(two CUDA paths, same rounding by construction).
"""
import numpy as np
import pytest
import torch

import oracle
import shifted_sparse_attention_s2attn_b200 as s2
from shifted_sparse_attention_s2attn_b200.synthetic import LORA_LLAMA2_7B, make_lora_inputs
from parity_utils import bits_to_device, bf16_tensor_to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    s2.clear_device_error()
    yield


def _f64(bits):
    return (np.asarray(bits).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _run(x_bits, w_bits, a_bits, b_bits, parts, scaling, rope_parts=0, head_dim=128, seq_len=None,
         pos_scale=1.0, check=True):
    x, w = bits_to_device(x_bits), bits_to_device(w_bits)
    a = None if a_bits is None else bits_to_device(a_bits)
    b = None if b_bits is None else bits_to_device(b_bits)
    T, K = x.shape
    n_out = w.shape[0] // parts
    r = 0 if a is None else a.shape[0] // parts
    y = torch.empty((parts, T, n_out), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(max(256, s2.lora_proj_workspace_bytes(T, K, n_out, parts, r)), dtype=torch.uint8, device="cuda")
    s2.lora_proj_fwd(x, w, a, b, y, parts, scaling, rope_parts=rope_parts, head_dim=head_dim,
                     seq_len=seq_len if seq_len is not None else T, pos_scale=pos_scale, workspace=ws)
    if check:
        torch.cuda.synchronize()
        rc, detail = s2.get_device_error()
        assert rc == 0, f"device error word set: {detail:#x}"
    return y


def _tol(x_bits, w_bits, a_bits, b_bits, scaling, parts, rows, ref):
    x = _f64(x_bits)[rows]
    w = _f64(w_bits)
    n_out = w.shape[0] // parts
    tol = 2.0 ** -7 * np.abs(ref) + 1e-6
    for p in range(parts):
        tol[p] += 2.0 ** -14 * (np.abs(x) @ np.abs(w[p * n_out:(p + 1) * n_out]).T)
        if a_bits is not None:
            a, b = _f64(a_bits), _f64(b_bits)
            r = a.shape[0] // parts
            u = np.abs(scaling * (x @ a[p * r:(p + 1) * r].T))
            tol[p] += 2.0 ** -7 * (u @ np.abs(b[p * n_out:(p + 1) * n_out]).T)
    return tol


def _check(y, x_bits, w_bits, a_bits, b_bits, scaling, parts, rows=None):
    rows = np.arange(y.shape[1]) if rows is None else np.asarray(rows)
    ref = oracle.lora_proj(x_bits, w_bits, a_bits, b_bits, scaling, parts, rows=rows)
    got = bf16_tensor_to_f64(y[:, torch.as_tensor(rows, device=y.device)])
    tol = _tol(x_bits, w_bits, a_bits, b_bits, scaling, parts, rows, ref)
    bad = np.abs(got - ref) > tol
    assert not bad.any(), f"{int(bad.sum())} elements out of tolerance; worst excess " \
                          f"{float((np.abs(got - ref) - tol).max()):.3e}"
    return ref, tol


def _rope_ref(ref, tol, seq_len, head_dim, pos_scale):
    """fp64 RoPE-PI of the oracle's outputs (all rows; row t is position t mod seq_len) and
    the bound for each rotated element."""
    parts_, T, n_out = ref.shape
    B, H, half = T // seq_len, n_out // head_dim, head_dim // 2
    out, out_tol = np.empty_like(ref), np.empty_like(ref)
    for p in range(parts_):
        y = ref[p].reshape(B, seq_len, H, head_dim)
        e = tol[p].reshape(B, seq_len, H, head_dim)
        rot = oracle.rope_pi_f64(y, pos_scale)
        pair = e[..., :half] + e[..., half:] + 2.0 ** -10 * (np.abs(y[..., :half]) + np.abs(y[..., half:]))
        out[p] = rot.reshape(T, n_out)
        out_tol[p] = (np.concatenate([pair, pair], axis=-1) + 2.0 ** -7 * np.abs(rot)).reshape(T, n_out)
    return out, out_tol


@pytest.mark.parametrize("T,K,n_out,parts,r", [
    (300, 520, 256, 3, 8),       # ragged rows (44 in the last block) and K (8 in the last block)
    (129, 64, 512, 1, 0),        # no adapter: the plain projection, one K block
    (256, 1024, 256, 2, 64),     # the largest rank (four K=16 steps in the rank block)
    (200, 136, 256, 1, 5),       # a rank that is not a multiple of 8 or 16
    (384, 256, 768, 1, 24),      # two K=16 steps in the rank block
    (2597, 264, 768, 3, 8),      # 189 output tiles: persistent CTAs take two, both accumulators
])
def test_lora_proj_matches_oracle(T, K, n_out, parts, r):
    x, w, a, b = make_lora_inputs(T, K, n_out, parts, r, seed=T)
    y = _run(x, w, a, b, parts, 2.0)
    _check(y, x, w, a, b, 2.0, parts)


@pytest.mark.parametrize("T,seq_len,K,n_out,parts,rope_parts,head_dim,pos_scale", [
    (300, 100, 520, 256, 3, 2, 128, 0.5),    # q, k rotated, v not; 3 sequences of 100
    (256, 256, 128, 512, 1, 1, 64, 0.125),   # head_dim 64: four heads per 256-column tile
])
def test_fused_rope_equals_projection_then_rope_pi_apply(T, seq_len, K, n_out, parts, rope_parts, head_dim,
                                                          pos_scale):
    x, w, a, b = make_lora_inputs(T, K, n_out, parts, 8, seed=7)
    plain = _run(x, w, a, b, parts, 2.0)
    fused = _run(x, w, a, b, parts, 2.0, rope_parts=rope_parts, head_dim=head_dim, seq_len=seq_len,
                 pos_scale=pos_scale)
    B, H = T // seq_len, n_out // head_dim
    for p in range(parts):
        if p < rope_parts:
            q = plain[p].clone().view(B, seq_len, H, head_dim)
            s2.rope_pi_apply(q, None, pos_scale)
            torch.cuda.synchronize()
            assert torch.equal(fused[p].view(B, seq_len, H, head_dim), q), f"part {p}"
        else:
            assert torch.equal(fused[p], plain[p]), f"part {p}"
    # and against the oracle: fp64 projection, then fp64 RoPE-PI
    ref, tol = _check(plain, x, w, a, b, 2.0, parts)
    rref, rtol = _rope_ref(ref[:rope_parts], tol[:rope_parts], seq_len, head_dim, pos_scale)
    got = bf16_tensor_to_f64(fused[:rope_parts])
    bad = np.abs(got - rref) > rtol
    assert not bad.any(), f"{int(bad.sum())} rotated elements out of tolerance"


def _sample_rows(T, n=40, seed=3):
    rng = np.random.default_rng(seed)
    fixed = [0, 1, 127, 128, 129, 2047, 2048, T // 2, T - 129, T - 128, T - 1]
    return np.unique(np.concatenate([fixed, rng.choice(T, n - len(fixed), replace=False)]))


def test_lora_llama2_7b_32k_qkv_full_size():
    """The LLaMA2-7B layer at 32k tokens: q, k, v stacked (12288 outputs), rank 8, RoPE-PI
    (pos_scale = 4096/32768) fused on q and k.  Sampled rows against the oracle; the whole
    output against the projection followed by rope_pi_apply, bit for bit."""
    T, L0 = 32768, 4096
    c = LORA_LLAMA2_7B
    x, w, a, b = make_lora_inputs(T, c["K"], c["n_out"], 3, c["r"], seed=2)
    plain = _run(x, w, a, b, 3, c["scaling"])
    fused = _run(x, w, a, b, 3, c["scaling"], rope_parts=2, head_dim=128, seq_len=T, pos_scale=L0 / T)
    q = plain[0].clone().view(1, T, 32, 128)
    k = plain[1].clone().view(1, T, 32, 128)
    s2.rope_pi_apply(q, k, L0 / T)
    torch.cuda.synchronize()
    assert torch.equal(fused[0].view(1, T, 32, 128), q)
    assert torch.equal(fused[1].view(1, T, 32, 128), k)
    assert torch.equal(fused[2], plain[2])
    _check(plain, x, w, a, b, c["scaling"], 3, rows=_sample_rows(T))


def test_lora_llama2_7b_32k_o_proj_full_size():
    T = 32768
    c = LORA_LLAMA2_7B
    x, w, a, b = make_lora_inputs(T, c["K"], c["n_out"], 1, c["r"], seed=4)
    y = _run(x, w, a, b, 1, c["scaling"])
    _check(y, x, w, a, b, c["scaling"], 1, rows=_sample_rows(T))


def test_lora_back_to_back_calls_are_deterministic():
    """Ten calls queued without synchronisation: no bounded wait gives up and every result
    equals the first (no atomics; the K order of the accumulation is fixed)."""
    x, w, a, b = make_lora_inputs(1000, 512, 512, 3, 16, seed=9)
    first = _run(x, w, a, b, 3, 2.0, rope_parts=2, head_dim=128, seq_len=500, pos_scale=0.25)
    xs, ws_, as_, bs = bits_to_device(x), bits_to_device(w), bits_to_device(a), bits_to_device(b)
    y = torch.empty_like(first)
    ws = torch.empty(s2.lora_proj_workspace_bytes(1000, 512, 512, 3, 16), dtype=torch.uint8, device="cuda")
    for _ in range(10):
        s2.lora_proj_fwd(xs, ws_, as_, bs, y, 3, 2.0, rope_parts=2, head_dim=128, seq_len=500, pos_scale=0.25,
                         workspace=ws)
    torch.cuda.synchronize()
    rc, detail = s2.get_device_error()
    assert rc == 0, f"device error word set: {detail:#x}"
    assert torch.equal(y, first)


def test_projection_output_feeds_s2attn_fwd_without_copies():
    """y[p] of the stacked q, k, v projection is a contiguous [B, N, H, D] tensor: the
    forward reads it in place and gives the same result as on separate copies."""
    T, H, D = 2048, 2, 128
    x, w, a, b = make_lora_inputs(T, 256, H * D, 3, 8, seed=11)
    y = _run(x, w, a, b, 3, 2.0, rope_parts=2, head_dim=D, seq_len=T, pos_scale=0.5)
    q, k, v = (y[p].view(1, T, H, D) for p in range(3))
    outs = []
    for args in ((q, k, v), (q.clone(), k.clone(), v.clone())):
        o = torch.empty_like(args[0])
        lse = torch.empty((1, H, T), dtype=torch.float32, device="cuda")
        s2.s2attn_fwd(*args, o, lse, 1024, 1)
        outs.append((o, lse))
    torch.cuda.synchronize()
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
