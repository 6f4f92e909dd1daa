"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Small shapes are compared element by element over whole tensors; the LLaMA2-shaped
workloads are compared on sampled rows that the oracle computes one group at a time
(the rows include the group edges, the diagonal tiles and the wrap-around group of
the shifted heads).  All inputs are the seeded synthetic recipe; Q and K go through
RoPE-PI on the GPU and, independently, through the oracle's RoPE on the host.
"""
import numpy as np
import pytest
import torch

import oracle
import shifted_sparse_attention_s2attn_b200 as s2
from shifted_sparse_attention_s2attn_b200.synthetic import (WORKLOADS, FULL_CAUSAL_32K, bf16_bits_to_f32,
                                                            f32_to_bf16_bits, make_inputs)
from parity_utils import (TOL_F32, TOL_LSE_BF16, TOL_O_BF16, TOL_REL_L2_BF16, bf16_tensor_to_f64,
                          device_to_bits, rel_l2, run_bf16)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    s2.clear_device_error()
    yield


def _bits(shape, seed):
    x = np.random.default_rng(seed).standard_normal(shape).astype(np.float32)
    return f32_to_bf16_bits(x)


# ---- RoPE-PI: bit-exact -------------------------------------------------------------

@pytest.mark.parametrize("B,N,H,D,scale", [(1, 512, 4, 128, 0.5), (2, 300, 3, 64, 1 / 8), (1, 8192, 32, 128, 0.5)])
def test_rope_pi_bit_exact(B, N, H, D, scale):
    q_bits, k_bits = _bits((B, N, H, D), 1), _bits((B, N, H, D), 2)
    from parity_utils import bits_to_device
    q, k = bits_to_device(q_bits), bits_to_device(k_bits)
    s2.rope_pi_apply(q, k, scale, 10000.0)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(device_to_bits(q), oracle.rope_pi_bf16(q_bits, scale))
    np.testing.assert_array_equal(device_to_bits(k), oracle.rope_pi_bf16(k_bits, scale))


@pytest.mark.parametrize("N,H,D,scale", [(512, 4, 128, 0.5), (32768, 2, 128, 1 / 8)])
def test_rope_backward_is_rope_with_negated_scale(N, H, D, scale):
    """The gradient through RoPE-PI (the transposed rotation) is rope_pi_apply with -pos_scale:
    bit-exact to the fp32-order oracle at -pos_scale, and the forward followed by it returns the
    input to within two bf16 roundings of the pair's size (doubled)."""
    from parity_utils import bits_to_device
    g_bits = _bits((1, N, H, D), 3)
    g = bits_to_device(g_bits)
    s2.rope_pi_apply(g, None, -scale)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(device_to_bits(g), oracle.rope_pi_bf16(g_bits, -scale))
    y = bits_to_device(g_bits)
    s2.rope_pi_apply(y, None, scale)
    s2.rope_pi_apply(y, None, -scale)
    torch.cuda.synchronize()
    x = bf16_bits_to_f32(g_bits).astype(np.float64)
    back = y.float().cpu().numpy().astype(np.float64)
    # each bf16 rounding is at most 2^-8 of a rotated element, which is at most |x1| + |x2| of its pair
    half = D // 2
    pair = np.abs(x[..., :half]) + np.abs(x[..., half:])
    pair = np.concatenate([pair, pair], axis=-1)
    assert np.all(np.abs(back - x) <= 2.0 ** -6 * pair + 2.0 ** -20)


def test_rope_pi_k_only_and_repeat():
    from parity_utils import bits_to_device
    k_bits = _bits((1, 256, 2, 128), 3)
    k = bits_to_device(k_bits)
    s2.rope_pi_apply(None, k, 0.25)
    s2.rope_pi_apply(None, k, 0.25)   # cached table, applied twice
    torch.cuda.synchronize()
    once = oracle.rope_pi_bf16(k_bits, 0.25)
    np.testing.assert_array_equal(device_to_bits(k), oracle.rope_pi_bf16(once, 0.25))


# ---- fp32 path ---------------------------------------------------------------------

def _run_f32(q, k, v, do, G, sh):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    tq, tk, tv, tdo = t(q), t(k), t(v), t(do)
    B, N, H, D = q.shape
    o = torch.empty_like(tq)
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    s2.s2attn_fwd_f32(tq, tk, tv, o, lse, G, sh)
    dq, dk, dv = torch.empty_like(tq), torch.empty_like(tq), torch.empty_like(tq)
    ws = torch.empty(s2.s2attn_bwd_workspace_bytes(B, N, H, D), dtype=torch.uint8, device="cuda")
    s2.s2attn_bwd_f32(tq, tk, tv, o, tdo, lse, dq, dk, dv, G, sh, ws)
    torch.cuda.synchronize()
    assert s2.get_device_error()[0] == 0
    return [x.cpu().numpy().astype(np.float64) for x in (o, lse, dq, dk, dv)]


@pytest.mark.parametrize("case", ["tiny", "ragged", "full_causal", "all_shifted"])
def test_f32_path_matches_oracle(case):
    if case == "tiny":
        w = WORKLOADS["tiny_fp32"]
        inp = make_inputs(w)
        q, k, v, do = inp["q"], inp["k"], inp["v"], inp["dout"]
        G, sh = w.G, w.shift_heads
    else:
        shape, G, sh = {"ragged": ((2, 90, 3, 40), 18, 1), "full_causal": ((1, 64, 2, 128), 64, 0),
                        "all_shifted": ((1, 120, 2, 16), 30, 2)}[case]
        rng = np.random.default_rng(7)
        q, k, v, do = (rng.standard_normal(shape).astype(np.float32) for _ in range(4))
    o, lse, dq, dk, dv = _run_f32(q, k, v, do, G, sh)
    ro, rlse = oracle.s2attn_fwd(q, k, v, G, sh)
    rdq, rdk, rdv = oracle.s2attn_bwd(q, k, v, do, G, sh)
    for name, got, ref in (("o", o, ro), ("lse", lse, rlse), ("dq", dq, rdq), ("dk", dk, rdk), ("dv", dv, rdv)):
        err = np.abs(got - ref).max()
        assert err <= TOL_F32, (case, name, err)


# ---- bf16 tensor-core path, whole tensors --------------------------------------------

SMALL = {
    # name: (B, N, H, G, shift_heads, rope pos_scale)
    "shifted_4tiles": (1, 1024, 4, 512, 2, 0.5),
    "two_batches": (2, 768, 2, 256, 1, None),
    "odd_tile_count": (1, 768, 2, 384, 0, None),
    "full_causal": (1, 1024, 2, 1024, 0, 0.25),
    "one_tile_groups": (1, 512, 2, 128, 0, None),
    "all_heads_shifted": (1, 512, 2, 256, 2, None),
    "one_group_shifted": (1, 512, 2, 512, 1, None),   # G = N with a shifted head: causal in half-rolled order
    # 256 query-tile pairs on the forward's persistent snake grid (a full round, then a partial
    # odd one) and 256 backward folds on its persistent grid (some CTAs take two folds, some one)
    "multi_round_schedules": (1, 8192, 8, 512, 4, None),
    # the forward's folded grid (two pairs per CTA, 288 CTAs) with the backward's persistent grid
    # taking 576 folds
    "fold_schedule": (1, 8192, 18, 512, 9, None),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_bf16_small_matches_oracle(name):
    B, N, H, G, sh, scale = SMALL[name]
    D = 128
    q_bits, k_bits, v_bits, do_bits = (_bits((B, N, H, D), 10 + i) for i in range(4))
    out = run_bf16(q_bits, k_bits, v_bits, do_bits, G, sh, rope_scale=scale)
    if scale is not None:
        q_bits, k_bits = oracle.rope_pi_bf16(q_bits, scale), oracle.rope_pi_bf16(k_bits, scale)
        np.testing.assert_array_equal(device_to_bits(out["q"]), q_bits)
    ro, rlse = oracle.s2attn_fwd(q_bits, k_bits, v_bits, G, sh)
    o_err = np.abs(bf16_tensor_to_f64(out["o"]) - ro).max()
    lse_err = np.abs(out["lse"].cpu().numpy() - rlse).max()
    assert o_err <= TOL_O_BF16, (name, "o", o_err)
    assert lse_err <= TOL_LSE_BF16, (name, "lse", lse_err)
    rdq, rdk, rdv = oracle.s2attn_bwd(q_bits, k_bits, v_bits, do_bits, G, sh)
    for g, ref in (("dq", rdq), ("dk", rdk), ("dv", rdv)):
        e = rel_l2(bf16_tensor_to_f64(out[g]), ref)
        assert e <= TOL_REL_L2_BF16, (name, g, e)


def test_bf16_forward_is_deterministic():
    B, N, H, G, sh = 1, 1024, 2, 512, 1
    bits = [_bits((B, N, H, 128), 30 + i) for i in range(4)]
    a = run_bf16(*bits, G, sh, bwd=False)
    b = run_bf16(*bits, G, sh, bwd=False)
    assert torch.equal(a["o"], b["o"]) and torch.equal(a["lse"], b["lse"])


def test_bf16_rejects_unsupported_shapes():
    q = torch.zeros((1, 768, 2, 128), dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty((1, 2, 768), dtype=torch.float32, device="cuda")
    with pytest.raises(s2.S2AttnError) as e:
        s2.s2attn_fwd(q, q, q, o, lse, 384, 1)      # G/2 = 192 is not a multiple of 128
    assert e.value.status == -2
    with pytest.raises(s2.S2AttnError) as e:
        s2.s2attn_fwd(q, q, q, o, lse, 96, 0)       # G not a multiple of 128
    assert e.value.status == -2
    q64 = torch.zeros((1, 256, 2, 64), dtype=torch.bfloat16, device="cuda")
    lse64 = torch.empty((1, 2, 256), dtype=torch.float32, device="cuda")
    with pytest.raises(s2.S2AttnError) as e:
        s2.s2attn_fwd(q64, q64, q64, torch.empty_like(q64), lse64, 128, 0)   # D = 64: fp32 path only
    assert e.value.status == -2


# ---- the LLaMA2-shaped workloads at full size, sampled rows ---------------------------

def _sample_units(w):
    last = w.groups - 1
    shifted = w.H - 1
    first_shifted = min(w.H - w.shift_heads, w.H - 1)
    units = {(0, 0, 0), (0, 0, last), (0, shifted, last), (0, shifted, 0), (0, first_shifted, min(1, last))}
    return sorted(units)


def _sample_rows(G, seed):
    """Query rows and key rows (rolled-local) of one group.  The key rows cover the whole walk
    of the backward: key tile 0 (seen by every query tile of the group: the longest dK/dV
    accumulation), the tile starting at G/2 (the wrap point of a shifted head's roll) and the
    one before it, a random middle tile, and the last two tiles (seen by one or two query tiles)."""
    rng = np.random.default_rng(seed)
    qrows = sorted({0, 1, 63, 64, 127, 128, 129, G // 2 - 1, G // 2, G - 129, G - 128, G - 2, G - 1,
                    *rng.integers(0, G, 6).tolist()})
    n_kt = G // 128
    mid = int(rng.integers(1, max(2, n_kt - 1))) * 128
    krows = sorted({0, 1, 2, 63, 64, 126, 127,                      # key tile 0
                    G // 2 - 1, G // 2, G // 2 + 1, G // 2 + 127,   # around the wrap point
                    mid, mid + 1 + int(rng.integers(0, 126)),       # a middle tile
                    G - 1, G - 2, G - 64, G - 65, G - 127, G - 128, *rng.integers(G - 256, G, 4).tolist()})
    return qrows, [r for r in krows if 0 <= r < G]


@pytest.mark.parametrize("wname", ["llama2_7b_8k", "llama2_7b_32k", "llama2_7b_32k_full_causal",
                                   "llama2_13b_64k", "llama2_7b_100k"])
def test_bf16_full_size_sampled(wname):
    w = FULL_CAUSAL_32K if wname == "llama2_7b_32k_full_causal" else WORKLOADS[wname]
    bwd = wname != "llama2_7b_32k_full_causal"   # the inference case is forward only
    inp = make_inputs(w)
    out = run_bf16(inp["q"], inp["k"], inp["v"], inp["dout"], w.G, w.shift_heads, rope_scale=w.pos_scale,
                   base=w.base, bwd=bwd)
    q_bits, k_bits = oracle.rope_pi_bf16(inp["q"], w.pos_scale, w.base), oracle.rope_pi_bf16(inp["k"], w.pos_scale,
                                                                                            w.base)
    # RoPE bit-exactness on a slab of rows (whole-tensor equality would copy GBs back)
    np.testing.assert_array_equal(device_to_bits(out["q"][:, :1024]), q_bits[:, :1024])
    np.testing.assert_array_equal(device_to_bits(out["k"][:, -1024:]), k_bits[:, -1024:])
    worst = {"o": 0.0, "lse": 0.0}
    got_g = {g: [] for g in ("dq", "dk", "dv")}
    ref_g = {g: [] for g in ("dq", "dk", "dv")}
    got_t0, ref_t0 = {"dk": [], "dv": []}, {"dk": [], "dv": []}
    for (b, h, j) in _sample_units(w):
        qrows, krows = _sample_rows(w.G, 1000 * h + j)
        r = oracle.s2attn_unit(q_bits, k_bits, inp["v"], w.G, w.shift_heads, b, h, j, qrows=qrows,
                               krows=krows if bwd else (), dout=inp["dout"] if bwd else None)
        qt = torch.from_numpy(r["qtok"]).cuda()
        o_rows = out["o"][b, qt, h].float().cpu().numpy()
        worst["o"] = max(worst["o"], float(np.abs(o_rows - r["o"]).max()))
        worst["lse"] = max(worst["lse"], float(np.abs(out["lse"][b, h, qt].cpu().numpy() - r["lse"]).max()))
        if bwd:
            kt = torch.from_numpy(r["ktok"]).cuda()
            got_g["dq"].append(out["dq"][b, qt, h].float().cpu().numpy()); ref_g["dq"].append(r["dq"])
            got_g["dk"].append(out["dk"][b, kt, h].float().cpu().numpy()); ref_g["dk"].append(r["dk"])
            got_g["dv"].append(out["dv"][b, kt, h].float().cpu().numpy()); ref_g["dv"].append(r["dv"])
            # key tile 0 alone: the longest accumulation must not hide behind the short ones
            t0 = np.asarray(krows) < 128
            got_t0["dk"].append(got_g["dk"][-1][t0]); ref_t0["dk"].append(r["dk"][t0])
            got_t0["dv"].append(got_g["dv"][-1][t0]); ref_t0["dv"].append(r["dv"][t0])
    assert worst["o"] <= TOL_O_BF16, (wname, worst)
    assert worst["lse"] <= TOL_LSE_BF16, (wname, worst)
    if bwd:
        for g in ("dq", "dk", "dv"):
            e = rel_l2(np.concatenate(got_g[g]), np.concatenate(ref_g[g]))
            assert e <= TOL_REL_L2_BF16, (wname, g, e)
        for g in ("dk", "dv"):
            e = rel_l2(np.concatenate(got_t0[g]), np.concatenate(ref_t0[g]))
            assert e <= TOL_REL_L2_BF16, (wname, g, "key tile 0", e)
    # properties that hold at any size, over the whole output
    assert torch.isfinite(out["o"]).all() and torch.isfinite(out["lse"]).all()
    if bwd:
        for g in ("dq", "dk", "dv"):
            assert torch.isfinite(out[g]).all(), g


@pytest.mark.parametrize("pos0,N,H,D,scale", [(0, 64, 2, 128, 0.5), (4090, 16, 32, 128, 1 / 8),
                                               (32752, 16, 32, 128, 1 / 8), (1000, 33, 3, 64, 1.0)])
def test_rope_pi_offset_bit_exact(pos0, N, H, D, scale):
    """Rows at positions pos0 .. pos0+N-1 (a decoding step's new tokens): bit-exact to the
    oracle and to the same rows of rope_pi_apply over the whole sequence."""
    from parity_utils import bits_to_device
    q_bits, k_bits = _bits((1, N, H, D), 50), _bits((1, N, H, D), 51)
    q, k = bits_to_device(q_bits), bits_to_device(k_bits)
    s2.rope_pi_apply_offset(q, k, pos0, scale)
    full = torch.zeros((1, pos0 + N, H, D), dtype=torch.bfloat16, device="cuda")
    full[:, pos0:] = bits_to_device(q_bits)
    s2.rope_pi_apply(full, None, scale)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(device_to_bits(q), oracle.rope_pi_bf16_at(q_bits, pos0, scale))
    np.testing.assert_array_equal(device_to_bits(k), oracle.rope_pi_bf16_at(k_bits, pos0, scale))
    np.testing.assert_array_equal(device_to_bits(q), device_to_bits(full[:, pos0:]))
