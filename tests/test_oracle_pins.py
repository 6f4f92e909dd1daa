"""Pins the fp64 oracle to things other than itself (CPU only).

Each check is an independent formulation: torch's SDPA for full causal attention,
brute-force softmax with an explicit N x N mask matrix for grouped / shifted
heads, the shift example printed on the "LongLoRA paper notes" page (section 3.3),
central finite differences for the gradients, RoPE as complex multiplication, and
the FLOP table of the nearauto.com article (Table 7).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import flops

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _brute_force(q, k, v, mask):
    """Masked softmax attention with an explicit [N,N] boolean mask (True = visible)."""
    B, N, H, D = q.shape
    o = np.zeros_like(q)
    lse = np.zeros((B, H, N))
    for b in range(B):
        for h in range(H):
            s = (q[b, :, h, :] @ k[b, :, h, :].T) / math.sqrt(D)
            s = np.where(mask[h], s, -np.inf)
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            lse[b, h] = (m[:, 0] + np.log(e.sum(axis=1)))
            o[b, :, h, :] = (e / e.sum(axis=1, keepdims=True)) @ v[b, :, h, :]
    return o, lse


def _mask_for_head(N, G, shift):
    """Visible pairs for one head: same group and causal, both in the shifted frame.

    Token t sits at position (t - shift) mod N of the shifted sequence.
    """
    pos = (np.arange(N) - shift) % N
    grp = pos // G
    same = grp[:, None] == grp[None, :]
    causal = pos[None, :] <= pos[:, None]
    return same & causal


def _masks(N, H, G, shift_heads, sign=+1):
    return [_mask_for_head(N, G, sign * (G // 2) if h >= H - shift_heads else 0) for h in range(H)]


def test_full_causal_equals_textbook_sdpa():
    B, N, H, D = 2, 16, 3, 8
    q, k, v = (_rand((B, N, H, D), s) for s in (1, 2, 3))
    o, lse = oracle.s2attn_fwd(q, k, v, G=N, shift_heads=0)
    t = lambda x: torch.from_numpy(x).permute(0, 2, 1, 3)  # [B,H,N,D]
    ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), is_causal=True)
    np.testing.assert_allclose(o, ref.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-12)
    s = (t(q) @ t(k).transpose(-1, -2)) / math.sqrt(D)
    s = s.masked_fill(~torch.ones(N, N, dtype=torch.bool).tril(), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(s, dim=-1).numpy(), rtol=0, atol=1e-12)


def test_unshifted_heads_equal_block_diagonal_causal():
    B, N, H, D, G = 1, 24, 2, 8, 6
    q, k, v = (_rand((B, N, H, D), s) for s in (4, 5, 6))
    o, lse = oracle.s2attn_fwd(q, k, v, G=G, shift_heads=0)
    ref_o, ref_lse = _brute_force(q, k, v, _masks(N, H, G, 0))
    np.testing.assert_allclose(o, ref_o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


@pytest.mark.parametrize("sign", [+1, -1])
def test_shifted_heads_equal_explicit_mask(sign):
    """Shifted heads == brute force with the N x N mask; the roll direction does not matter."""
    B, N, H, D, G = 2, 24, 4, 8, 6
    q, k, v = (_rand((B, N, H, D), s) for s in (7, 8, 9))
    o, lse = oracle.s2attn_fwd(q, k, v, G=G, shift_heads=2)
    ref_o, ref_lse = _brute_force(q, k, v, _masks(N, H, G, 2, sign))
    np.testing.assert_allclose(o, ref_o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_shifted_differs_from_unshifted():
    B, N, H, D, G = 1, 24, 2, 8, 6
    q, k, v = (_rand((B, N, H, D), s) for s in (10, 11, 12))
    o_s, _ = oracle.s2attn_fwd(q, k, v, G=G, shift_heads=1)
    o_u, _ = oracle.s2attn_fwd(q, k, v, G=G, shift_heads=0)
    np.testing.assert_array_equal(o_s[:, :, 0], o_u[:, :, 0])
    assert np.abs(o_s[:, :, 1] - o_u[:, :, 1]).max() > 1e-3


def test_page_shift_example_groups():
    g = json.load(open(os.path.join(GOLDEN, "p3_shift_example.json")))
    N, G = g["N"], g["G"]
    x = _rand((1, N, 2, 4), 13)
    for head, key in ((0, "unshifted_groups_1indexed"), (1, "shifted_groups_1indexed")):
        groups = []
        for j in range(N // G):
            r = oracle.s2attn_unit(x, x, x, G, 1, 0, head, j, qrows=range(G))
            groups.append(sorted((r["qtok"] + 1).tolist()))
        assert sorted(groups) == sorted(sorted(gr) for gr in g[key])


def test_unit_rows_match_full():
    B, N, H, D, G = 1, 32, 2, 8, 8
    q, k, v, do = (_rand((B, N, H, D), s) for s in (14, 15, 16, 17))
    o, lse = oracle.s2attn_fwd(q, k, v, G, 1)
    dq, dk, dv = oracle.s2attn_bwd(q, k, v, do, G, 1)
    r = oracle.s2attn_unit(q, k, v, G, 1, 0, 1, 3, qrows=[0, 5, 7], krows=[1, 6], dout=do)
    np.testing.assert_array_equal(r["o"], o[0, r["qtok"], 1])
    np.testing.assert_array_equal(r["lse"], lse[0, 1, r["qtok"]])
    np.testing.assert_array_equal(r["dq"], dq[0, r["qtok"], 1])
    np.testing.assert_array_equal(r["dk"], dk[0, r["ktok"], 1])
    np.testing.assert_array_equal(r["dv"], dv[0, r["ktok"], 1])
    # the last group of the shifted head wraps around the end of the sequence
    assert sorted(oracle.s2attn_unit(q, k, v, G, 1, 0, 1, 3, qrows=range(G))["qtok"].tolist()) == \
        [0, 1, 2, 3, 28, 29, 30, 31]


def test_gradients_match_finite_differences():
    B, N, H, D, G = 1, 16, 2, 4, 4
    q, k, v, do = (_rand((B, N, H, D), s) for s in (18, 19, 20, 21))
    dq, dk, dv = oracle.s2attn_bwd(q, k, v, do, G, 1)

    def loss(qq, kk, vv):
        return float((oracle.s2attn_fwd(qq, kk, vv, G, 1)[0] * do).sum())

    eps = 1e-6
    for name, grad in (("q", dq), ("k", dk), ("v", dv)):
        num = np.zeros_like(grad)
        for idx in np.ndindex(*grad.shape):
            args = {"q": q.copy(), "k": k.copy(), "v": v.copy()}
            args[name][idx] += eps
            up = loss(args["q"], args["k"], args["v"])
            args[name][idx] -= 2 * eps
            dn = loss(args["q"], args["k"], args["v"])
            num[idx] = (up - dn) / (2 * eps)
        rel = np.linalg.norm(num - grad) / np.linalg.norm(grad)
        assert rel < 1e-6, (name, rel)


def test_gradient_of_full_causal_matches_torch_autograd():
    B, N, H, D = 1, 12, 2, 8
    q, k, v, do = (_rand((B, N, H, D), s) for s in (22, 23, 24, 25))
    dq, dk, dv = oracle.s2attn_bwd(q, k, v, do, G=N, shift_heads=0)
    tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3).requires_grad_() for x in (q, k, v))
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True)
    o.backward(torch.from_numpy(do).permute(0, 2, 1, 3))
    for mine, ref in ((dq, tq), (dk, tk), (dv, tv)):
        np.testing.assert_allclose(mine, ref.grad.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-12)


def test_bf16_and_f32_inputs_widen_exactly():
    B, N, H, D, G = 1, 16, 2, 8, 8
    x32 = _rand((B, N, H, D), 26).astype(np.float32)
    bits = (x32.view(np.uint32) >> 16).astype(np.uint16)  # truncation: an exact bf16 value
    as64 = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    o_b, _ = oracle.s2attn_fwd(bits, bits, bits, G, 1)
    o_d, _ = oracle.s2attn_fwd(as64, as64, as64, G, 1)
    np.testing.assert_array_equal(o_b, o_d)
    o_f, _ = oracle.s2attn_fwd(x32, x32, x32, G, 1)
    o_fd, _ = oracle.s2attn_fwd(x32.astype(np.float64), x32.astype(np.float64), x32.astype(np.float64), G, 1)
    np.testing.assert_array_equal(o_f, o_fd)


def test_invalid_shapes_rejected():
    x = _rand((1, 12, 2, 4), 27)
    with pytest.raises(ValueError):
        oracle.s2attn_fwd(x, x, x, G=5, shift_heads=0)   # G does not divide N
    with pytest.raises(ValueError):
        oracle.s2attn_fwd(x, x, x, G=3, shift_heads=1)   # odd G cannot shift by G/2
    with pytest.raises(ValueError):
        oracle.s2attn_fwd(x, x, x, G=4, shift_heads=3)   # more shifted heads than heads


# ---- work counts -------------------------------------------------------------

def test_useful_pairs_brute_force():
    for N, G, H in ((24, 6, 3), (16, 16, 2), (12, 4, 1)):
        count = sum(int(m.sum()) for m in _masks(N, H, G, H // 2))
        assert flops.useful_pairs(1, N, H, G) == count
        assert flops.fwd_flops(2, N, H, 8, G) == 2 * 4 * 8 * count


def test_table7_attention_shares():
    g = json.load(open(os.path.join(GOLDEN, "table7_flop_shares.json")))
    want = g["attention_share_percent"]
    got = {
        "full_8192": flops.llama2_7b_attention_share(8192, 8192),
        "full_65536": flops.llama2_7b_attention_share(65536, 65536),
        "s2attn_65536": flops.llama2_7b_attention_share(65536, 65536 // 4),
    }
    for key, pct in want.items():
        assert round(100 * got[key], g["decimals"]) == pct, (key, 100 * got[key])


def test_context_compute_ratio():
    g = json.load(open(os.path.join(GOLDEN, "context_compute_ratio.json")))
    s, l = g["short_context"], g["long_context"]
    # non-causal counting of the attention pair work, as in the article's ratio
    ratio = (l * l) / (s * s)
    assert ratio == g["attention_compute_ratio"]
    # grouped attention keeps the per-token cost fixed: O(L^2/g) with g = L/G groups
    assert flops.useful_pairs(1, l, 1, 2048) == 4 * flops.useful_pairs(1, s, 1, 2048)


# ---- RoPE with position interpolation -----------------------------------------

def _rope_complex(x, positions, base):
    """RoPE as complex multiplication: z_i = x_i + 1j*x_{i+D/2}, z_i *= exp(1j*pos*theta_i)."""
    D = x.shape[-1]
    half = D // 2
    theta = base ** (-2.0 * np.arange(half) / D)
    z = x[..., :half] + 1j * x[..., half:]
    rot = np.exp(1j * positions[None, :, None, None] * theta[None, None, None, :])
    z = z * rot
    return np.concatenate([z.real, z.imag], axis=-1)


def test_rope_matches_complex_rotation_and_interpolation():
    B, N, H, D = 2, 32, 3, 16
    x = _rand((B, N, H, D), 28)
    for scale in (1.0, 0.5, 1 / 8):
        y = oracle.rope_pi_f64(x, scale, 10000.0)
        ref = _rope_complex(x, np.arange(N) * scale, 10000.0)
        np.testing.assert_allclose(y, ref, rtol=0, atol=1e-12)
    # interpolation: token 2m at scale 1/2 sits where token m sits without interpolation
    y_half = oracle.rope_pi_f64(x, 0.5, 10000.0)
    y_one = oracle.rope_pi_f64(x, 1.0, 10000.0)
    x_even = x[:, ::2]
    y_even_one = oracle.rope_pi_f64(np.ascontiguousarray(x_even), 1.0, 10000.0)
    np.testing.assert_allclose(y_half[:, ::2], y_even_one, rtol=0, atol=1e-12)
    assert np.abs(y_half - y_one).max() > 1e-3


def test_rope_invariants():
    B, N, H, D = 1, 40, 2, 16
    x = _rand((B, N, H, D), 29)
    y = oracle.rope_pi_f64(x, 0.25, 10000.0)
    np.testing.assert_array_equal(y[:, 0], x[:, 0])                       # position 0: identity
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)
    # relative position: <R(m) q, R(n) k> depends on m - n only
    q1 = np.broadcast_to(_rand((1, 1, 1, D), 30), (1, N, 1, D)).copy()
    k1 = np.broadcast_to(_rand((1, 1, 1, D), 31), (1, N, 1, D)).copy()
    rq, rk = oracle.rope_pi_f64(q1, 1.0, 10000.0), oracle.rope_pi_f64(k1, 1.0, 10000.0)
    dots = {}
    for m in range(N):
        for n in range(N):
            dots.setdefault(m - n, []).append(float(rq[0, m, 0] @ rk[0, n, 0]))
    for vals in dots.values():
        assert max(vals) - min(vals) < 1e-10


def test_rope_f32_order_within_bf16_rounding_of_f64():
    from shifted_sparse_attention_s2attn_b200.synthetic import bf16_bits_to_f32, f32_to_bf16_bits
    B, N, H, D = 1, 512, 2, 128
    bits = f32_to_bf16_bits(_rand((B, N, H, D), 32).astype(np.float32))
    x = bf16_bits_to_f32(bits).astype(np.float64).reshape(B, N, H, D)
    for scale in (1.0, 0.125):
        y32 = bf16_bits_to_f32(oracle.rope_pi_bf16(bits, scale)).reshape(B, N, H, D)
        y64 = oracle.rope_pi_f64(x, scale, 10000.0)
        # one bf16 rounding (2^-9 relative) plus fp32 angle error (< 1e-6 * |pos*theta|)
        tol = np.abs(y64) * 2.0 ** -8 + 2e-3 * np.linalg.norm(x, axis=-1, keepdims=True) / np.sqrt(D)
        assert np.all(np.abs(y32 - y64) <= tol)
    np.testing.assert_array_equal(oracle.rope_pi_bf16(bits, 0.5)[:, 0], bits[:, 0])


def test_rope_bf16_commutes_with_power_of_two_scaling():
    """K rows scaled by 8 before or after the rotation give identical bits."""
    from shifted_sparse_attention_s2attn_b200.synthetic import bf16_bits_to_f32, f32_to_bf16_bits
    B, N, H, D = 1, 256, 2, 128
    x = _rand((B, N, H, D), 33).astype(np.float32)
    bits = f32_to_bf16_bits(x)
    times8 = lambda b: f32_to_bf16_bits(bf16_bits_to_f32(b) * np.float32(8)).reshape(b.shape)
    a = oracle.rope_pi_bf16(times8(bits), 1 / 25)
    b = times8(oracle.rope_pi_bf16(bits, 1 / 25))
    np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("pos0,scale", [(0, 0.5), (7, 1.0), (4093, 0.125), (32760, 1 / 8)])
def test_rope_at_offset_equals_rows_of_the_longer_sequence(pos0, scale):
    """Rotating rows t of a short tensor as tokens pos0 + t (a decoding step's new rows) gives
    exactly rows pos0 .. pos0+N-1 of the same rows rotated as part of the whole sequence."""
    from shifted_sparse_attention_s2attn_b200.synthetic import f32_to_bf16_bits
    B, N, H, D = 1, 5, 2, 64
    rows = f32_to_bf16_bits(_rand((B, N, H, D), 31).astype(np.float32))
    full = np.zeros((B, pos0 + N, H, D), dtype=np.uint16)
    full[:, pos0:] = rows
    np.testing.assert_array_equal(oracle.rope_pi_bf16_at(rows, pos0, scale), oracle.rope_pi_bf16(full, scale)[:, pos0:])
    if pos0 == 0:
        np.testing.assert_array_equal(oracle.rope_pi_bf16_at(rows, 0, scale), oracle.rope_pi_bf16(rows, scale))
