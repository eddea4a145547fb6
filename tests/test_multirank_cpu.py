"""The multi-rank host logic of bench.py (weak scaling, max-over-ranks timing) on two
gloo ranks on the CPU.  The data path has no collective: each rank draws its own batch."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import bench
    from gqa_attention_paged_b200 import inputs
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        case = inputs.sweep_decode(2, seed=bench.rank_seed(0, rank), ctx=64)
        ms = 1.0 + rank  # rank 1 is the slow one
        ms_max = bench.max_over_ranks(ms, dist)
        step = bench.decode_step_bytes([int(x) for x in case.kv.seq_lens], 32, 8, 128, 2)
        gbs = bench.aggregate_gbs(step, world, ms_max)
        dist.barrier()
        q.put((rank, ms_max, gbs, float(case.q.float().sum())))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_weak_scaling():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, m0, g0, s0), (r1, m1, g1, s1) = res
    assert m0 == m1 == 2.0                      # both ranks see the slowest rank's time
    step = 2 * 2 * 64 * 8 * 128 * 2 + 2 * 2 * 32 * 128 * 2
    assert g0 == g1 == pytest.approx(world * step / 2e-3 / 1e9)
    assert s0 != s1                             # independent batches per rank
