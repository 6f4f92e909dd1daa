"""GPU parity of the decoding step (full causal attention of the last M positions)
against the fp64 oracle, through the C ABI: the CUDA-core kernel (M = 1) and the
tensor-core kernel (2 <= M <= 128).

Inference runs ordinary full attention ("LongLoRA paper notes", section 3.1): the
decoding queries are the last M positions of a sequence whose K/V hold all N
positions.  Small and ragged shapes exercise partial tiles, several splits and every
query-count specialisation; the LLaMA2-7B 32k shape runs at full size (the oracle's
cost here is M*N per head, so it compares every output).
"""
import numpy as np
import pytest
import torch

import oracle
import shifted_sparse_attention_s2attn_b200 as s2
from shifted_sparse_attention_s2attn_b200.synthetic import WORKLOADS, f32_to_bf16_bits, make_tensor
from parity_utils import TOL_LSE_BF16, TOL_O_BF16, bf16_tensor_to_f64, bits_to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    s2.clear_device_error()
    yield


def _bits(shape, seed):
    return f32_to_bf16_bits(np.random.default_rng(seed).standard_normal(shape).astype(np.float32))


def _run(q_bits, k_bits, v_bits):
    q, k, v = bits_to_device(q_bits), bits_to_device(k_bits), bits_to_device(v_bits)
    B, M, H, D = q.shape
    N = k.shape[1]
    o = torch.empty_like(q)
    lse = torch.empty((B, H, M), dtype=torch.float32, device="cuda")
    ws = torch.empty(s2.s2attn_decode_workspace_bytes(B, M, N, H, D), dtype=torch.uint8, device="cuda")
    s2.s2attn_decode(q, k, v, o, lse, ws)
    torch.cuda.synchronize()
    rc, detail = s2.get_device_error()
    assert rc == 0, f"device error word set: {detail:#x}"
    return o, lse


def _check(o, lse, ref_o, ref_lse):
    err_o = float(np.abs(bf16_tensor_to_f64(o) - ref_o).max())
    err_l = float(np.abs(lse.cpu().numpy() - ref_lse).max())
    assert err_o <= TOL_O_BF16, f"O max abs error {err_o}"
    assert err_l <= TOL_LSE_BF16, f"lse max abs error {err_l}"


@pytest.mark.parametrize("B,M,N,H", [
    (1, 1, 1, 1),        # one position: o = v
    (1, 1, 128, 2),      # exactly one tile
    (1, 1, 20000, 2),    # many tiles per split
    (3, 1, 777, 5),
    # tensor-core path (2 <= M <= 128)
    (2, 3, 1000, 4),     # ragged tail, several splits
    (1, 5, 4099, 3),     # tail of 3 keys
    (1, 16, 300, 2),     # M > the last tile's tail
    (1, 2, 20000, 2),    # many tiles per split
    (3, 8, 777, 5),
    (1, 17, 300, 2),     # the last split starts past some queries' limits
    (2, 32, 1000, 3),
    (1, 64, 4099, 2),
    (1, 100, 100, 2),    # M = N: the first query sees one key
    (1, 128, 2048, 2),   # a whole query tile
    (3, 40, 777, 5),
])
def test_decode_matches_oracle(B, M, N, H):
    D = 128
    q, k, v = _bits((B, M, H, D), 1), _bits((B, N, H, D), 2), _bits((B, N, H, D), 3)
    o, lse = _run(q, k, v)
    ref_o, ref_lse = oracle.decode(q, k, v)
    _check(o, lse, ref_o, ref_lse)


def test_decode_equals_last_rows_of_full_causal_forward():
    """Two of this library's kernels agree: the decoding step and the tensor-core forward
    with G = N and no shift (full causal attention), on the last M rows."""
    B, N, H, D, M = 1, 2048, 4, 128, 4
    q, k, v = _bits((B, N, H, D), 4), _bits((B, N, H, D), 5), _bits((B, N, H, D), 6)
    qd, kd, vd = bits_to_device(q), bits_to_device(k), bits_to_device(v)
    of = torch.empty_like(qd)
    lsef = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    s2.s2attn_fwd(qd, kd, vd, of, lsef, N, 0)
    o, lse = _run(np.ascontiguousarray(q[:, N - M:]), k, v)
    assert float((o.float() - of[:, N - M:].float()).abs().max()) <= 2 * TOL_O_BF16
    assert float((lse - lsef[:, :, N - M:]).abs().max()) <= 2 * TOL_LSE_BF16


def test_decode_repeated_calls_and_nonfinite_free():
    B, M, N, H, D = 1, 4, 3000, 2, 128
    q, k, v = _bits((B, M, H, D), 7), _bits((B, N, H, D), 8), _bits((B, N, H, D), 9)
    o1, l1 = _run(q, k, v)
    o2, l2 = _run(q, k, v)
    assert torch.isfinite(o1.float()).all() and torch.isfinite(l1).all()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)  # no atomics: the result is deterministic


@pytest.mark.parametrize("M", [1, 16, 128])
def test_decode_llama2_7b_32k_full_size(M):
    """The 32k LLaMA2-7B layer (H=32, D=128): the decoding queries are the last M rows of
    the workload's Q, against the workload's whole K and V."""
    w = WORKLOADS["llama2_7b_32k"]
    q = np.ascontiguousarray(make_tensor(w, "q")[:, w.N - M:])
    k, v = make_tensor(w, "k"), make_tensor(w, "v")
    o, lse = _run(q, k, v)
    ref_o, ref_lse = oracle.decode(q, k, v)
    _check(o, lse, ref_o, ref_lse)


@pytest.mark.parametrize("M", [1, 16, 128])
def test_decode_back_to_back_calls(M):
    """Thirty calls queued back to back (no synchronisation in between, so kernels of one
    call overlap the launches of the next): no bounded wait may give up (the device error
    word stays clear) and the result equals a single synchronised call's."""
    B, N, H, D = 1, 8192, 8, 128
    q, k, v = (bits_to_device(_bits(s, 40 + i)) for i, s in enumerate([(B, M, H, D), (B, N, H, D), (B, N, H, D)]))
    o_ref = torch.empty_like(q)
    lse_ref = torch.empty((B, H, M), dtype=torch.float32, device="cuda")
    ws = torch.empty(s2.s2attn_decode_workspace_bytes(B, M, N, H, D), dtype=torch.uint8, device="cuda")
    s2.s2attn_decode(q, k, v, o_ref, lse_ref, ws)
    torch.cuda.synchronize()
    o, lse = torch.empty_like(o_ref), torch.empty_like(lse_ref)
    for _ in range(30):
        s2.s2attn_decode(q, k, v, o, lse, ws)
    torch.cuda.synchronize()
    rc, detail = s2.get_device_error()
    assert rc == 0, f"device error word set: {detail:#x}"
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
