"""Pins of the LoRA-projection oracle (oracle/lora.py) to facts that do not come from the
oracle: a hand-worked example, brute-force loops, the merged-weight identity of a
low-rank update, a zero adapter, linearity in the scaling, and the independence of the
stacked projections ("LongLoRA paper notes", section 3.2: adapters on the Q, K, V and O
projections)."""
import numpy as np
import pytest

import oracle
from shifted_sparse_attention_s2attn_b200.synthetic import bf16_bits_to_f32, make_lora_inputs


def _rand(seed, T, K, n_out, parts, r):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((T, K)), rng.standard_normal((parts * n_out, K)),
            rng.standard_normal((parts * r, K)), rng.standard_normal((parts * n_out, r)))


def test_hand_worked_example():
    x = np.array([[1.0, 2.0]])
    w = np.array([[3.0, 4.0], [5.0, 6.0]])
    a = np.array([[1.0, -1.0]])
    b = np.array([[2.0], [0.5]])
    # x W^T = [1*3 + 2*4, 1*5 + 2*6] = [11, 17]; x A^T = 1 - 2 = -1;
    # 3 * (-1) * [2, 0.5] = [-6, -1.5]; y = [5, 15.5]
    np.testing.assert_array_equal(oracle.lora_proj(x, w, a, b, 3.0, parts=1), [[[5.0, 15.5]]])


def test_brute_force_loops():
    T, K, n_out, parts, r, s = 5, 7, 3, 2, 2, 1.75
    x, w, a, b = _rand(5, T, K, n_out, parts, r)
    y = oracle.lora_proj(x, w, a, b, s, parts)
    assert y.shape == (parts, T, n_out)
    for p in range(parts):
        for t in range(T):
            for c in range(n_out):
                acc = 0.0
                for k in range(K):
                    acc += x[t, k] * w[p * n_out + c, k]
                for j in range(r):
                    u = 0.0
                    for k in range(K):
                        u += x[t, k] * a[p * r + j, k]
                    acc += s * u * b[p * n_out + c, j]
                assert abs(y[p, t, c] - acc) <= 1e-12 * (1 + abs(acc))


def test_merged_weight_identity():
    """A low-rank update folds into the weight: x (W + s B A)^T, merged first."""
    T, K, n_out, parts, r, s = 9, 16, 8, 3, 4, 0.5
    x, w, a, b = _rand(6, T, K, n_out, parts, r)
    y = oracle.lora_proj(x, w, a, b, s, parts)
    for p in range(parts):
        merged = w[p * n_out:(p + 1) * n_out] + s * (b[p * n_out:(p + 1) * n_out] @ a[p * r:(p + 1) * r])
        np.testing.assert_allclose(y[p], x @ merged.T, rtol=1e-12, atol=1e-12)


def test_zero_adapter_and_rank_zero_give_the_plain_projection():
    T, K, n_out, parts, r = 4, 6, 5, 2, 3
    x, w, a, b = _rand(7, T, K, n_out, parts, r)
    plain = np.stack([x @ w[p * n_out:(p + 1) * n_out].T for p in range(parts)])
    np.testing.assert_array_equal(oracle.lora_proj(x, w, a, np.zeros_like(b), 2.0, parts), plain)
    np.testing.assert_array_equal(oracle.lora_proj(x, w, None, None, 2.0, parts), plain)


def test_linear_in_the_scaling():
    T, K, n_out, parts, r = 6, 10, 4, 1, 2
    x, w, a, b = _rand(8, T, K, n_out, parts, r)
    y0, y1, y3 = (oracle.lora_proj(x, w, a, b, s, parts) for s in (0.0, 1.0, 3.0))
    np.testing.assert_allclose(y3 - y0, 3.0 * (y1 - y0), rtol=1e-12, atol=1e-12)
    assert np.abs(y1 - y0).max() > 0.1


def test_stacked_parts_are_independent_projections():
    T, K, n_out, parts, r, s = 5, 8, 3, 3, 2, 1.5
    x, w, a, b = _rand(9, T, K, n_out, parts, r)
    y = oracle.lora_proj(x, w, a, b, s, parts)
    for p in range(parts):
        one = oracle.lora_proj(x, w[p * n_out:(p + 1) * n_out], a[p * r:(p + 1) * r],
                               b[p * n_out:(p + 1) * n_out], s, 1)
        np.testing.assert_array_equal(y[p], one[0])
    a2, b2 = a.copy(), b.copy()
    a2[r:] += 1.0       # change the adapters of parts 1 and 2 only
    b2[n_out:] -= 1.0
    np.testing.assert_array_equal(oracle.lora_proj(x, w, a2, b2, s, parts)[0], y[0])


def test_rows_select_rows_and_bf16_is_widened_exactly():
    x, w, a, b = make_lora_inputs(12, 24, 8, 2, 3, seed=1)
    full = oracle.lora_proj(x, w, a, b, 2.0, 2)
    rows = [0, 5, 11]
    np.testing.assert_array_equal(oracle.lora_proj(x, w, a, b, 2.0, 2, rows=rows), full[:, rows])
    as_f32 = [bf16_bits_to_f32(t).astype(np.float64) for t in (x, w, a, b)]
    np.testing.assert_array_equal(oracle.lora_proj(*as_f32, 2.0, 2), full)


def test_rejects_mismatched_shapes():
    x, w, a, b = _rand(10, 3, 4, 2, 1, 2)
    with pytest.raises(ValueError):
        oracle.lora_proj(x, w[:, :3], a, b, 1.0, 1)
    with pytest.raises(ValueError):
        oracle.lora_proj(x, w, a, b[:, :1], 1.0, 1)


# ---- backward ------------------------------------------------------------------------

def _loss(x, w, a, b, s, parts, dy):
    """<y, dy>: its gradient with respect to any input is what lora_proj_bwd returns."""
    return float((oracle.lora_proj(x, w, a, b, s, parts) * dy).sum())


def test_backward_equals_central_finite_differences():
    T, K, n_out, parts, r, s = 3, 5, 4, 2, 2, 1.25
    x, w, a, b = _rand(11, T, K, n_out, parts, r)
    dy = np.random.default_rng(12).standard_normal((parts, T, n_out))
    dx, da, db = oracle.lora_proj_bwd(x, w, a, b, dy, s, parts)
    h = 1e-6
    for name, arr, grad in (("x", x, dx), ("a", a, da), ("b", b, db)):
        num = np.empty_like(arr)
        for idx in np.ndindex(arr.shape):
            saved = arr[idx]
            arr[idx] = saved + h
            fp = _loss(x, w, a, b, s, parts, dy)
            arr[idx] = saved - h
            fm = _loss(x, w, a, b, s, parts, dy)
            arr[idx] = saved
            num[idx] = (fp - fm) / (2 * h)
        rel = np.abs(num - grad).max() / np.abs(grad).max()
        assert rel < 1e-7, (name, rel)


def test_backward_hand_worked_example():
    # the forward example above: x = [1, 2], W = [[3, 4], [5, 6]], A = [[1, -1]], B = [[2], [0.5]], s = 3
    x = np.array([[1.0, 2.0]])
    w = np.array([[3.0, 4.0], [5.0, 6.0]])
    a = np.array([[1.0, -1.0]])
    b = np.array([[2.0], [0.5]])
    dy = np.array([[[1.0, -2.0]]])
    dx, da, db = oracle.lora_proj_bwd(x, w, a, b, dy, 3.0, 1)
    # dy B = 1*2 - 2*0.5 = 1;  dx = dy W + 3 * 1 * A = [3 - 10, 4 - 12] + [3, -3] = [-4, -11]
    np.testing.assert_array_equal(dx, [[-4.0, -11.0]])
    # dA = 3 * (dy B)^T x = 3 * [1, 2];  dB = 3 * dy^T (x A^T) = 3 * [1, -2]^T * (-1)
    np.testing.assert_array_equal(da, [[3.0, 6.0]])
    np.testing.assert_array_equal(db, [[-3.0], [6.0]])


def test_backward_without_adapter_is_the_plain_linear_backward():
    T, K, n_out, parts = 4, 6, 3, 3
    x, w, _, _ = _rand(13, T, K, n_out, parts, 1)
    dy = np.random.default_rng(14).standard_normal((parts, T, n_out))
    dx, da, db = oracle.lora_proj_bwd(x, w, None, None, dy, 2.0, parts)
    assert da is None and db is None
    want = sum(dy[p] @ w[p * n_out:(p + 1) * n_out] for p in range(parts))
    np.testing.assert_allclose(dx, want, rtol=1e-13, atol=1e-13)


def test_rope_backward_undoes_the_forward_rotation():
    """The rotation is orthogonal, so its transposed rotation (the backward) inverts the
    C oracle's fp64 forward: rope_bwd(rope(y)) = y; and <rope(y), g> = <y, rope_bwd(g)>."""
    rng = np.random.default_rng(15)
    y = rng.standard_normal((2, 50, 3, 64))
    g = rng.standard_normal(y.shape)
    for ps in (1.0, 0.125):
        np.testing.assert_allclose(oracle.rope_pi_bwd_f64(oracle.rope_pi_f64(y, ps), ps), y, rtol=0, atol=1e-12)
        lhs = float((oracle.rope_pi_f64(y, ps) * g).sum())
        rhs = float((y * oracle.rope_pi_bwd_f64(g, ps)).sum())
        assert abs(lhs - rhs) <= 1e-10 * abs(lhs)
    # position 0 is the identity
    z = np.zeros((1, 1, 1, 8)); z[..., 3] = 1.0
    np.testing.assert_array_equal(oracle.rope_pi_bwd_f64(z, 0.5), z)


def test_rope_backward_is_rope_with_negated_pos_scale():
    """Rotating by -a is the transposed rotation, and every step of the fp32 evaluation order
    flips sign exactly when pos_scale does (t * ps and (t * ps) * theta round symmetrically,
    cos is even, sin is odd), so RoPE-PI with -pos_scale is the RoPE backward: in fp64 equal to
    rope_pi_bwd_f64, and in the bit-exact fp32 order within one bf16 rounding of it."""
    import math
    from shifted_sparse_attention_s2attn_b200.synthetic import f32_to_bf16_bits
    rng = np.random.default_rng(16)
    g = rng.standard_normal((1, 300, 2, 128))
    for ps in (1.0, 0.125, 0.04):
        np.testing.assert_allclose(oracle.rope_pi_f64(g, -ps), oracle.rope_pi_bwd_f64(g, ps), rtol=0, atol=1e-12)
        bits = f32_to_bf16_bits(g.astype(np.float32))
        inv = bf16_bits_to_f32(oracle.rope_pi_bf16(bits, -ps)).astype(np.float64)
        ref = oracle.rope_pi_bwd_f64(bf16_bits_to_f32(bits).astype(np.float64), ps)
        # bf16 rounding of each output, plus the fp32 angle's rounding (half an fp32 ulp of angles
        # up to 300 rad here, ~1.5e-5 rad) times the pair's size
        err = np.abs(inv - ref)
        assert np.all(err <= 2.0 ** -8 * np.abs(ref) + 2.0 ** -12 * np.abs(g).max())
        assert np.abs(inv - bf16_bits_to_f32(oracle.rope_pi_bf16(bits, ps)).astype(np.float64)).max() > 0.5
    # the host libm the tables are built with: (float) cos / sin of +-a in double, over many a
    for a in np.linspace(-5000.0, 5000.0, 20011):
        a32 = float(np.float32(a))
        assert np.float32(math.cos(-a32)) == np.float32(math.cos(a32))
        assert np.float32(math.sin(-a32)) == -np.float32(math.sin(a32))
