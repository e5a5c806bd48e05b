"""Host-side logic of the multi-GPU benchmark path on CPU: two gloo ranks.

`bench.py --gpus N` runs N independent replicas (one batch per rank, no
exchange); the only cross-rank steps are a barrier and the max-over-ranks
reduction of the device times, which these tests exercise with gloo.
"""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    import sys

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        # rank r reports a slower dispatch on rank 1 and a slower combine on rank 0
        out = bench.reduce_max_over_ranks([100.0 + rank, 50.0 - 10 * rank, 7.0], world, "cpu")
        dist.barrier()
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got[0] == got[1] == [101.0, 50.0, 7.0]


def test_single_rank_needs_no_process_group():
    import bench

    assert bench.reduce_max_over_ranks([3.0, 1.0], 1, "cpu") == [3.0, 1.0]


def test_algorithmic_bytes_normal_workload():
    import bench

    # 4096 x 7168, top-8 of 256 experts, 8 partitions, every slot valid: R = 32768
    d, c = bench.algorithmic_bytes(4096, 7168, 8, 256, 8, 32768, True)
    x = 4096 * 7168 * 2
    payload = 32768 * 7168
    scales = 32768 * 56 * 4
    meta = 4096 * 8 * 12 + 32768 * 12 + 4096 * 8 * 4 + 257 * 4 + 256 * 4 + 8 * 4 + 4096 * 8
    assert d == x + payload + scales + meta == 301_893_668
    assert c == 32768 * 7168 * 2 + x + 4096 * 8 * 8 == 528_744_448
    # BF16 path: two bytes per payload element, no scales
    d16, _ = bench.algorithmic_bytes(8192, 4096, 6, 64, 16, 49152, False)
    assert d16 == (8192 * 4096 * 2 + 49152 * 4096 * 2 + 8192 * 6 * 12 + 49152 * 12
                   + 8192 * 6 * 4 + 65 * 4 + 64 * 4 + 16 * 4 + 8192 * 16)
