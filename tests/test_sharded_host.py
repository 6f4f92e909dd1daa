"""Sequence-sharded S^2-Attn on CPU: gloo ranks exchange the G/2 halos of the shifted heads
(to_local), the test runs the fp64 oracle with shift_heads = 0 on each rank's local layout,
and the results go back to their owners (to_owner); the rows, put side by side, must equal
the oracle on the whole sequence with the shift -- forward (o, lse) and backward (dq, dk,
dv).  The library's sharded_fwd / sharded_bwd compose the same steps with the CUDA kernels
(tests/test_gpu_sharded.py)."""
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


def _run_rank(rank, world, N):
    import sys
    sys.path.insert(0, ROOT)
    import oracle
    from shifted_sparse_attention_s2attn_b200.sharded import shard_range, to_local, to_owner
    t0, t1 = shard_range(N, G, world, rank)
    q, k, v, do = (torch.from_numpy(x[:, t0:t1].copy()) for x in _inputs(N))
    # forward: local layout, oracle with shift 0, results back to their owners
    qz, kz, vz = to_local((q, k, v), G, SH)
    oz, lse_z = (torch.from_numpy(a) for a in oracle.s2attn_fwd(qz.numpy(), kz.numpy(), vz.numpy(), G, 0))
    (o,), lse = to_owner([oz], G, SH, lse=lse_z)
    # backward: o and lse travel through the exchange too; they must come back as the local layout's
    (qz2, kz2, vz2, oz2, dz), lse_z2 = to_local((q, k, v, o, do), G, SH, lse=lse)
    assert torch.equal(oz2, oz) and torch.equal(lse_z2, lse_z)
    grads = oracle.s2attn_bwd(qz2.numpy(), kz2.numpy(), vz2.numpy(), dz.numpy(), G, 0)
    dq, dk, dv = to_owner([torch.from_numpy(a) for a in grads], G, SH)
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
