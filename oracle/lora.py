"""fp64 oracle of the LoRA-adapted projections -- TEST INFRASTRUCTURE ONLY.

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline / reference leg use
this module; the CUDA library never does, and this module never imports it.

What it computes ("LongLoRA paper notes", section 3.2: low-rank adapters on the Q, K, V
and O projections; nearauto.com article, "long-context LoRA improvement"): a frozen
weight W plus a trainable update of rank r.  The pages do not write the update out; the
plain reading, taken here, is the usual one -- the update is B A with A of shape [r, K]
and B of shape [n_out, r], scaled by a constant s (alpha / r):

    y_p = x W_p^T + s (x A_p^T) B_p^T        for each stacked projection p < parts,

every input widened exactly from bf16 to fp64, the products and sums in fp64 (numpy
matmul as the contraction step).  No rounding of the intermediate: the oracle is the
exact value, and the tests' tolerance covers the CUDA path's bf16 intermediate and
output.

Pinned by tests/test_oracle_lora_pins.py: a hand-worked example, brute-force loops,
the merged-weight identity x (W + s B A)^T, a zero adapter, linearity in s, and the
independence of the stacked parts.  The backward (lora_proj_bwd, rope_pi_bwd_f64) is pinned
there by central finite differences of <y, dy>, a hand-worked example, and the RoPE
backward undoing the forward rotation of the C oracle.
"""
import numpy as np


def _f64(a):
    """bf16 bit patterns (uint16) or floats -> float64, exactly."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def lora_proj(x, w, lora_a, lora_b, scaling, parts, rows=None):
    """y [parts, len(rows), n_out] (fp64) for x [T, K], w [parts*n_out, K],
    lora_a [parts*r, K], lora_b [parts*n_out, r] (lora_a / lora_b None: r = 0).
    `rows` selects rows of x (default: all)."""
    x = _f64(x)
    if rows is not None:
        x = x[np.asarray(rows)]
    w = _f64(w)
    n_out = w.shape[0] // parts
    if w.shape[0] != parts * n_out or w.shape[1] != x.shape[1]:
        raise ValueError("w must be [parts*n_out, K]")
    y = np.empty((parts, x.shape[0], n_out))
    if lora_a is None:
        a = b = None
        r = 0
    else:
        a, b = _f64(lora_a), _f64(lora_b)
        r = a.shape[0] // parts
        if a.shape != (parts * r, x.shape[1]) or b.shape != (parts * n_out, r):
            raise ValueError("lora_a must be [parts*r, K] and lora_b [parts*n_out, r]")
    for p in range(parts):
        wp = w[p * n_out:(p + 1) * n_out]
        y[p] = x @ wp.T
        if r:
            ap = a[p * r:(p + 1) * r]
            bp = b[p * n_out:(p + 1) * n_out]
            y[p] += scaling * ((x @ ap.T) @ bp.T)
    return y


def lora_proj_bwd(x, w, lora_a, lora_b, dy, scaling, parts):
    """Gradients of the projection for an upstream gradient dy [parts, T, n_out] (of y, before
    any RoPE).  W is frozen -- only the adapters and the input get gradients (notes section 3.2:
    the adapters are what trains; LoRA+ adds embeddings and norms, not W):

        dx     = sum_p  dy_p W_p + s (dy_p B_p) A_p          [T, K]
        dA_p   = s (dy_p B_p)^T x                            [r, K]
        dB_p   = s dy_p^T (x A_p^T)                          [n_out, r]

    Returns (dx, dA [parts*r, K], dB [parts*n_out, r]) in fp64; dA, dB are None when r == 0."""
    x, w, dy = _f64(x), _f64(w), _f64(dy)
    n_out = w.shape[0] // parts
    if dy.shape != (parts, x.shape[0], n_out):
        raise ValueError("dy must be [parts, T, n_out]")
    dx = np.zeros_like(x)
    if lora_a is None:
        for p in range(parts):
            dx += dy[p] @ w[p * n_out:(p + 1) * n_out]
        return dx, None, None
    a, b = _f64(lora_a), _f64(lora_b)
    r = a.shape[0] // parts
    da, db = np.empty_like(a), np.empty_like(b)
    for p in range(parts):
        wp, ap, bp = w[p * n_out:(p + 1) * n_out], a[p * r:(p + 1) * r], b[p * n_out:(p + 1) * n_out]
        g = dy[p] @ bp                      # [T, r]: the gradient reaching the rank-r intermediate / s
        dx += dy[p] @ wp + scaling * (g @ ap)
        da[p * r:(p + 1) * r] = scaling * (g.T @ x)
        db[p * n_out:(p + 1) * n_out] = scaling * (dy[p].T @ (x @ ap.T))
    return dx, da, db


def rope_pi_bwd_f64(dy_rot, pos_scale, base=10000.0):
    """Gradient through RoPE-PI ("LongLoRA paper notes", section 3.4): the rotation of each pair
    (i, i + D/2) by angle a = (t * pos_scale) * base^(-2i/D) is orthogonal, so the gradient of
    the unrotated pair is the transposed rotation of the rotated pair's gradient:
        dy1 = cos(a) dy1' + sin(a) dy2',   dy2 = -sin(a) dy1' + cos(a) dy2'.
    dy_rot: [B, N, H, D] (row t is position t); fp64 throughout."""
    g = _f64(dy_rot)
    B, N, H, D = g.shape
    half = D // 2
    theta = base ** (-2.0 * np.arange(half) / D)
    ang = (np.arange(N, dtype=np.float64) * pos_scale)[:, None] * theta[None, :]   # [N, half]
    c, s = np.cos(ang)[None, :, None, :], np.sin(ang)[None, :, None, :]
    g1, g2 = g[..., :half], g[..., half:]
    return np.concatenate([c * g1 + s * g2, -s * g1 + c * g2], axis=-1)
