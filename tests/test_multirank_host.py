"""The multi-GPU bench path on CPU: two gloo ranks run the host-side timing logic.

Each GPU runs an independent replica of the workload (the path does not shard), so
the only cross-rank steps are the barrier and the max over ranks of the timed region;
the reported value counts the work of every rank over the slowest rank's time.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    from datetime import timedelta
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=timedelta(seconds=60))
    try:
        local_ms = [12.5, 17.25][rank]
        ms_max = bench.max_over_ranks(local_ms)
        dist.barrier()
        value = bench.whole_job_tflops(7.7e12, 10, world, ms_max)
        q.put((rank, ms_max, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, ms_max, value in res:
        assert ms_max == 17.25
        assert value == pytest.approx(2 * 7.7e12 * 10 / 17.25e-3 / 1e12)


def test_single_process_helpers():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.0) == 3.0
    assert bench.whole_job_tflops(1e12, 5, 1, 1000.0) == pytest.approx(5.0)
    from shifted_sparse_attention_s2attn_b200.synthetic import WORKLOADS
    w = WORKLOADS["llama2_7b_32k"]
    from oracle import flops
    assert bench.step_flops(w) == 3.5 * flops.fwd_flops(w.B, w.N, w.H, w.D, w.G)
    assert bench.oracle_sample_flops(w, w.G) == 3.5 * flops.fwd_flops(1, w.G, 1, w.D, w.G)
