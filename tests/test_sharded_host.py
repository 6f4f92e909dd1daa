"""Sequence-sharded S^2-Attn on CPU: gloo ranks run the library's sharded_fwd / sharded_bwd
with their four device primitives replaced by CPU stand-ins that this test defines -- the
halo copies by tensor slicing and the attention calls by the fp64 oracle with the shift.
The exchange steps (which rows go to which rank, in which direction, and the restore of
the inputs) are the library's own.  The rows of all ranks, put side by side, must equal
the oracle on the whole sequence with the shift -- forward (o, lse) and backward (dq, dk,
dv) -- and every input must come back unchanged.  tests/test_gpu_sharded.py runs the same
steps with the CUDA kernels."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

B, H, D, G, SH = 2, 3, 4, 8, 2   # N (sequence length) per test: 64 for 1, 2 and 4 ranks, 48 for 3


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(N):
    rng = np.random.default_rng(77)
    return [rng.standard_normal((B, N, H, D)) for _ in range(4)]


def _cpu_primitives(sharded):
    """CPU stand-ins for the halo copies (slicing) and the attention calls (the oracle)."""
    import oracle

    def rows_copy(xs, bufs, to_buf, G_, sh):
        for x, b in zip(xs, bufs):
            hs = x.shape[2] - sh
            if to_buf:
                b.copy_(x[:, : G_ // 2, hs:])
            else:
                x[:, : G_ // 2, hs:] = b

    def lse_copy(lses, bufs, to_buf, G_, sh):
        for x, b in zip(lses, bufs):
            hs = x.shape[1] - sh
            if to_buf:
                b.copy_(x[:, hs:, : G_ // 2])
            else:
                x[:, hs:, : G_ // 2] = b

    def attn_fwd(q, k, v, G_, sh):
        return tuple(torch.from_numpy(a) for a in oracle.s2attn_fwd(q.numpy(), k.numpy(), v.numpy(), G_, sh))

    def attn_bwd(q, k, v, o, dout, lse, G_, sh):
        return tuple(torch.from_numpy(a) for a in oracle.s2attn_bwd(q.numpy(), k.numpy(), v.numpy(), dout.numpy(),
                                                                     G_, sh))

    sharded._rows_copy, sharded._lse_copy = rows_copy, lse_copy
    sharded._attn_fwd, sharded._attn_bwd = attn_fwd, attn_bwd


def _run_rank(rank, world, N):
    import sys
    sys.path.insert(0, ROOT)
    from shifted_sparse_attention_s2attn_b200 import sharded
    _cpu_primitives(sharded)
    t0, t1 = sharded.shard_range(N, G, world, rank)
    q, k, v, do = (torch.from_numpy(x[:, t0:t1].copy()) for x in _inputs(N))
    before = [x.clone() for x in (q, k, v, do)]
    o, lse = sharded.sharded_fwd(q, k, v, G, SH)
    o_in, lse_in = o.clone(), lse.clone()
    dq, dk, dv = sharded.sharded_bwd(q, k, v, o, do, lse, G, SH)
    # every input comes back as it was given (the halo rows are swapped back)
    for a, b in zip((q, k, v, do, o, lse), before + [o_in, lse_in]):
        assert torch.equal(a, b)
    return [x.numpy() for x in (o, lse, dq, dk, dv)]


def _worker(rank, world, N, port, q):
    import torch.distributed as dist
    from datetime import timedelta
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=timedelta(seconds=60))
    try:
        q.put((rank, _run_rank(rank, world, N)))
    finally:
        dist.destroy_process_group()


def _check(parts, N):
    import sys
    sys.path.insert(0, ROOT)
    import oracle
    o = np.concatenate([p[0] for p in parts], axis=1)
    lse = np.concatenate([p[1] for p in parts], axis=2)
    dq, dk, dv = (np.concatenate([p[i] for p in parts], axis=1) for i in (2, 3, 4))
    qf, kf, vf, dof = _inputs(N)
    ro, rlse = oracle.s2attn_fwd(qf, kf, vf, G, SH)
    rdq, rdk, rdv = oracle.s2attn_bwd(qf, kf, vf, dof, G, SH)
    for got, ref in ((o, ro), (lse, rlse), (dq, rdq), (dk, rdk), (dv, rdv)):
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_one_rank_wraps_onto_itself():
    _check([_run_rank(0, 1, 64)], 64)


@pytest.mark.parametrize("world,N", [(2, 64), (3, 48), (4, 64)])
def test_gloo_ranks_match_the_unsharded_oracle(world, N):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, N, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    try:
        results = dict(q.get(timeout=120) for _ in range(world))
    finally:
        for p in procs:
            p.join(timeout=60)
    assert all(p.exitcode == 0 for p in procs)
    _check([results[r] for r in range(world)], N)


def test_shard_range_rejects_partial_groups():
    from shifted_sparse_attention_s2attn_b200.sharded import shard_range
    assert shard_range(64, 8, 4, 3) == (48, 64)
    with pytest.raises(ValueError):
        shard_range(64, 8, 3, 0)      # 64 tokens do not split over 3 ranks
    with pytest.raises(ValueError):
        shard_range(48, 16, 2, 0)     # 24 tokens per rank is not a whole number of 16-token groups
