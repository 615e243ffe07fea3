"""Host logic of the multi-GPU benchmark path on two CPU ranks (gloo).

Decode of different sequences needs no exchange, so N ranks run N independent
batches (weak scaling) and only the control path talks: a barrier and the max
of the per-rank step time. These ranks run the oracle on CPU, never a GPU.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from oracle import ORACLE
        from paged_kv_cache_339_b200 import workloads as W
        b = W.mha("cpu", seed=1002 + 100 * rank, num_seqs=3, num_heads=2, min_len=5,
                  max_len=40, num_blocks=30)
        f = lambda t: t.float().numpy().astype(np.float64)
        out = ORACLE.decode(f(b.q), f(b.k_cache), f(b.v_cache), b.block_tables.numpy(),
                            b.context_lens.numpy(), b.scale)
        my_ms = 1.0 + rank                           # rank 1 is the slow one
        bench.barrier(world)
        ms = bench.max_over_ranks(my_ms, world)
        total = bench.sum_over_ranks(b.kv_bytes_logical(), world)
        value = bench.weak_scaling_value(total, ms)
        # per-step times: rank 1's are uniformly 10x rank 0's
        pct = bench.percentiles([(1 + 9 * rank) * x for x in range(1, 11)], world)
        q.put((rank, ms, value, float(out.sum()), b.kv_bytes_logical(), pct))
    finally:
        dist.destroy_process_group()


def test_two_ranks_weak_scaling_control_path():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=120) for _ in procs), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, ms0, v0, s0, b0, p0), (r1, ms1, v1, s1, b1, p1) = res
    assert ms0 == ms1 == 2.0                         # max over ranks, on every rank
    assert v0 == v1                                  # every rank reports the same job value
    assert v0 == pytest.approx((b0 + b1) / 2.0e-3)   # units of both ranks / slowest time
    assert s0 != s1                                  # independent batches (different seeds)
    # percentiles of 10x(1..10): linear interpolation gives 19, 55, 91 on both ranks
    assert p0 == p1 == {"p10": 19.0, "p50": 55.0, "p90": 91.0}
