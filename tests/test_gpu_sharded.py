"""The sequence-sharded path on one GPU with this library's kernels.

* The halo copies (s2attn_halo_rows / s2attn_halo_lse) move exactly rows [0, G/2) of the
  shifted heads, bit for bit, in both directions (index work: compared with slicing).
* One rank: its halo is its own first G/2 rows (the cyclic wrap).  sharded_fwd and
  sharded_bwd must equal the fp64 oracle of the unsharded sequence, and the direct call
  (the forward bit for bit), and leave their inputs unchanged.
* Two ranks emulated on one GPU: the two halves of a sequence run the same steps one after
  the other, with the exchange done by handing the buffers over (no kernel waits on
  another); the rows put side by side must equal the oracle of the whole sequence.
Runs with more than one GPU exchange the halos over NCCL; every run here has one GPU.
"""
import numpy as np
import pytest
import torch

import oracle
import shifted_sparse_attention_s2attn_b200 as s2
from shifted_sparse_attention_s2attn_b200 import sharded
from shifted_sparse_attention_s2attn_b200.synthetic import f32_to_bf16_bits
from parity_utils import TOL_LSE_BF16, TOL_O_BF16, TOL_REL_L2_BF16, bits_to_device, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    s2.clear_device_error()
    yield


def _no_device_error():
    torch.cuda.synchronize()
    rc, detail = s2.get_device_error()
    assert rc == 0, f"device error word set: {detail:#x}"


def _bits(shape, seed):
    return f32_to_bf16_bits(np.random.default_rng(seed).standard_normal(shape).astype(np.float32))


@pytest.mark.parametrize("B,N,H,D,G,sh", [(2, 1024, 4, 128, 512, 2), (1, 768, 3, 64, 256, 1), (1, 512, 2, 128, 512, 2)])
def test_halo_copies_move_exactly_the_halo_rows(B, N, H, D, G, sh):
    half, hs = G // 2, H - sh
    xs = [bits_to_device(_bits((B, N, H, D), 70 + i)) for i in range(3)]
    ref = [x.clone() for x in xs]
    bufs = sharded.halo_rows(xs, G, sh)
    for x, b in zip(xs, bufs):
        assert torch.equal(b, x[:, :half, hs:])
    new = [bits_to_device(_bits((B, half, sh, D), 80 + i)) for i in range(3)]
    sharded.put_halo_rows(new, xs, G, sh)
    for x, r, n in zip(xs, ref, new):
        want = r.clone()
        want[:, :half, hs:] = n
        assert torch.equal(x, want)      # only the halo rows changed
    lse = torch.randn((B, H, N), device="cuda")
    lse_ref = lse.clone()
    (lb,) = sharded.halo_lse([lse], G, sh)
    assert torch.equal(lb, lse[:, hs:, :half])
    nl = torch.randn((B, sh, half), device="cuda")
    sharded.put_halo_lse([nl], [lse], G, sh)
    lse_ref[:, hs:, :half] = nl
    assert torch.equal(lse, lse_ref)
    _no_device_error()


def _inputs(B, N, H, seed):
    return [_bits((B, N, H, 128), seed + i) for i in range(4)]


def _sampled(o, lse, dq, dk, dv, bits, G, sh, units):
    """Max abs errors of o and lse and the relative L2 of dq, dk, dv on the rows of the
    given units (every row of each group) against the oracle."""
    q, k, v, do = bits
    worst_o = worst_lse = 0.0
    got = {g: [] for g in ("dq", "dk", "dv")}
    ref = {g: [] for g in ("dq", "dk", "dv")}
    rows = list(range(G))
    for (b, h, j) in units:
        r = oracle.s2attn_unit(q, k, v, G, sh, b, h, j, qrows=rows, krows=rows, dout=do)
        qt = torch.from_numpy(r["qtok"]).cuda()
        kt = torch.from_numpy(r["ktok"]).cuda()
        worst_o = max(worst_o, float(np.abs(o[b, qt, h].float().cpu().numpy() - r["o"]).max()))
        worst_lse = max(worst_lse, float(np.abs(lse[b, h, qt].cpu().numpy() - r["lse"]).max()))
        got["dq"].append(dq[b, qt, h].float().cpu().numpy()); ref["dq"].append(r["dq"])
        got["dk"].append(dk[b, kt, h].float().cpu().numpy()); ref["dk"].append(r["dk"])
        got["dv"].append(dv[b, kt, h].float().cpu().numpy()); ref["dv"].append(r["dv"])
    errs = {g: rel_l2(np.concatenate(got[g]), np.concatenate(ref[g])) for g in got}
    return worst_o, worst_lse, errs


@pytest.mark.parametrize("N,H,G,sh", [(1024, 2, 512, 1), (2048, 4, 256, 2)])
def test_one_rank_sharded_matches_oracle_and_direct(N, H, G, sh):
    B = 1
    bits = _inputs(B, N, H, 5)
    q, k, v, do = (bits_to_device(x) for x in bits)
    before = [x.clone() for x in (q, k, v, do)]
    o, lse = sharded.sharded_fwd(q, k, v, G, sh)
    o_in, lse_in = o.clone(), lse.clone()
    dq, dk, dv = sharded.sharded_bwd(q, k, v, o, do, lse, G, sh)
    _no_device_error()
    for a, b in zip((q, k, v, do, o, lse), before + [o_in, lse_in]):
        assert torch.equal(a, b)          # inputs restored
    # the oracle: every group of an unshifted head and of the last shifted head (the wrap group included)
    units = [(0, 0, j) for j in range(N // G)] + [(0, H - 1, j) for j in range(N // G)]
    eo, el, eg = _sampled(o, lse, dq, dk, dv, bits, G, sh, units)
    assert eo <= TOL_O_BF16 and el <= TOL_LSE_BF16, (eo, el)
    for g, e in eg.items():
        assert e <= TOL_REL_L2_BF16, (g, e)
    # the direct call: the forward bit for bit (same groups, same rows, same order)
    o_ref = torch.empty_like(q)
    lse_ref = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    s2.s2attn_fwd(q, k, v, o_ref, lse_ref, G, sh)
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)


def test_two_ranks_emulated_on_one_gpu_match_the_unsharded_oracle():
    """Rank 0 holds tokens [0, N/2), rank 1 tokens [N/2, N).  The steps of sharded_fwd and
    sharded_bwd run for both ranks in turn; 'exchange' hands rank p's buffers to its ring
    neighbour.  The shifted heads' wrap groups then mix both ranks' rows."""
    B, N, H, G, sh = 1, 2048, 4, 512, 2
    bits = _inputs(B, N, H, 40)
    full = [bits_to_device(x) for x in bits]
    P, Np = 2, N // 2
    ranks = [[x[:, p * Np:(p + 1) * Np].contiguous() for x in full] for p in range(P)]

    def ring(bufs_by_rank, step):       # what rank p receives from rank (p - step) mod P
        return [bufs_by_rank[(p - step) % P] for p in range(P)]

    # forward
    own = [sharded.halo_rows(r[:3], G, sh) for r in ranks]
    halo = ring(own, -1)
    for p in range(P):
        sharded.put_halo_rows(halo[p], ranks[p][:3], G, sh)
    outs = [sharded._attn_fwd(*ranks[p][:3], G, sh) for p in range(P)]
    for p in range(P):
        sharded.put_halo_rows(own[p], ranks[p][:3], G, sh)
    res = [sharded.halo_rows([o], G, sh) + sharded.halo_lse([lse], G, sh) for (o, lse) in outs]
    back = ring(res, +1)
    for p in range(P):
        sharded.put_halo_rows(back[p][:1], [outs[p][0]], G, sh)
        sharded.put_halo_lse(back[p][1:], [outs[p][1]], G, sh)
    # backward
    xs = [ranks[p][:3] + [outs[p][0], ranks[p][3]] for p in range(P)]
    own = [sharded.halo_rows(xs[p], G, sh) + sharded.halo_lse([outs[p][1]], G, sh) for p in range(P)]
    got = ring(own, -1)
    for p in range(P):
        sharded.put_halo_rows(got[p][:5], xs[p], G, sh)
        sharded.put_halo_lse(got[p][5:], [outs[p][1]], G, sh)
    grads = [sharded._attn_bwd(*xs[p], outs[p][1], G, sh) for p in range(P)]
    for p in range(P):
        sharded.put_halo_rows(own[p][:5], xs[p], G, sh)
        sharded.put_halo_lse(own[p][5:], [outs[p][1]], G, sh)
    res = [sharded.halo_rows(list(g), G, sh) for g in grads]
    back = ring(res, +1)
    for p in range(P):
        sharded.put_halo_rows(back[p], list(grads[p]), G, sh)
    _no_device_error()
    o = torch.cat([outs[p][0] for p in range(P)], dim=1)
    lse = torch.cat([outs[p][1] for p in range(P)], dim=2)
    dq, dk, dv = (torch.cat([grads[p][i] for p in range(P)], dim=1) for i in range(3))
    for p in range(P):                    # inputs restored
        for a, b in zip(ranks[p], full):
            assert torch.equal(a, b[:, p * Np:(p + 1) * Np])
    # every group of an unshifted head and of a shifted head, incl. the wrap group across ranks
    units = [(0, 0, j) for j in range(N // G)] + [(0, H - 1, j) for j in range(N // G)]
    eo, el, eg = _sampled(o, lse, dq, dk, dv, bits, G, sh, units)
    assert eo <= TOL_O_BF16 and el <= TOL_LSE_BF16, (eo, el)
    for g, e in eg.items():
        assert e <= TOL_REL_L2_BF16, (g, e)
