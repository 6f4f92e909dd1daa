"""Pins the oracle's decoding step (full causal attention of the last M positions) to
things other than itself (CPU only).

Inference runs ordinary full attention ("LongLoRA paper notes", section 3.1; the model
page's features list).  A decoding step appends M queries at positions N-M .. N-1 to a
sequence whose keys and values hold all N positions.  The checks: torch SDPA with an
explicit boolean mask, the last rows of the (separately pinned) full-causal forward,
closed forms (a single key; identical keys), causality, and exact bf16 widening.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from shifted_sparse_attention_s2attn_b200.synthetic import bf16_bits_to_f32, f32_to_bf16_bits


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


@pytest.mark.parametrize("B,M,N,H,D", [(1, 1, 9, 2, 8), (2, 4, 13, 3, 16), (1, 7, 7, 1, 4)])
def test_decode_equals_sdpa_with_explicit_mask(B, M, N, H, D):
    q, k, v = _rand((B, M, H, D), 1), _rand((B, N, H, D), 2), _rand((B, N, H, D), 3)
    o, lse = oracle.decode(q, k, v)
    t = lambda x: torch.from_numpy(x).permute(0, 2, 1, 3)  # [B,H,len,D]
    mask = torch.from_numpy(np.arange(N)[None, :] <= (N - M + np.arange(M))[:, None])  # [M,N]
    ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), attn_mask=mask)
    np.testing.assert_allclose(o, ref.permute(0, 2, 1, 3).numpy(), rtol=0, atol=1e-12)
    s = (t(q) @ t(k).transpose(-1, -2)) / math.sqrt(D)
    ref_lse = torch.logsumexp(s.masked_fill(~mask, float("-inf")), dim=-1)
    np.testing.assert_allclose(lse, ref_lse.numpy(), rtol=0, atol=1e-12)


def test_decode_equals_last_rows_of_full_causal_forward():
    B, N, H, D, M = 1, 24, 2, 8, 5
    qf, k, v = _rand((B, N, H, D), 4), _rand((B, N, H, D), 5), _rand((B, N, H, D), 6)
    of, lsef = oracle.s2attn_fwd(qf, k, v, G=N, shift_heads=0)
    o, lse = oracle.decode(qf[:, N - M:], k, v)
    np.testing.assert_allclose(o, of[:, N - M:], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lsef[:, :, N - M:], rtol=0, atol=1e-12)


def test_single_key_closed_form():
    q, k, v = _rand((1, 1, 1, 8), 7), _rand((1, 1, 1, 8), 8), _rand((1, 1, 1, 8), 9)
    o, lse = oracle.decode(q, k, v)
    np.testing.assert_array_equal(o, v)
    assert lse[0, 0, 0] == pytest.approx(float(q.ravel() @ k.ravel()) / math.sqrt(8), abs=1e-14)


def test_identical_keys_average_the_visible_values():
    B, M, N, H, D = 1, 3, 10, 2, 8
    q, v = _rand((B, M, H, D), 10), _rand((B, N, H, D), 11)
    k = np.broadcast_to(_rand((B, 1, H, D), 12), (B, N, H, D)).copy()
    o, lse = oracle.decode(q, k, v)
    for m in range(M):
        n_vis = N - M + m + 1
        np.testing.assert_allclose(o[:, m], v[:, :n_vis].mean(axis=1), rtol=0, atol=1e-13)
        s = np.einsum("bhd,bhd->bh", q[:, m], k[:, 0]) / math.sqrt(D)
        np.testing.assert_allclose(lse[:, :, m], s + math.log(n_vis), rtol=0, atol=1e-13)


def test_later_keys_are_invisible_to_earlier_queries():
    B, M, N, H, D = 1, 4, 12, 2, 8
    q, k, v = _rand((B, M, H, D), 13), _rand((B, N, H, D), 14), _rand((B, N, H, D), 15)
    o, lse = oracle.decode(q, k, v)
    k2, v2 = k.copy(), v.copy()
    k2[:, N - 1] += 5.0
    v2[:, N - 1] -= 3.0
    o2, lse2 = oracle.decode(q, k2, v2)
    np.testing.assert_array_equal(o2[:, : M - 1], o[:, : M - 1])
    np.testing.assert_array_equal(lse2[:, :, : M - 1], lse[:, :, : M - 1])
    assert np.abs(o2[:, M - 1] - o[:, M - 1]).max() > 1e-3


def test_bf16_inputs_widen_exactly():
    B, M, N, H, D = 1, 2, 9, 2, 16
    bits = [f32_to_bf16_bits(_rand(s, i).astype(np.float32)) for i, s in
            enumerate([(B, M, H, D), (B, N, H, D), (B, N, H, D)], start=16)]
    o_b, lse_b = oracle.decode(*bits)
    o_f, lse_f = oracle.decode(*(bf16_bits_to_f32(b).astype(np.float64) for b in bits))
    np.testing.assert_array_equal(o_b, o_f)
    np.testing.assert_array_equal(lse_b, lse_f)


def test_rejects_more_queries_than_positions():
    with pytest.raises(ValueError):
        oracle.decode(_rand((1, 5, 1, 4), 1), _rand((1, 4, 1, 4), 2), _rand((1, 4, 1, 4), 3))
