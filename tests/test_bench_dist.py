"""Multi-process plumbing of bench.py on the CPU: two gloo ranks rendezvous
on 127.0.0.1, pass the timing barriers and agree on the max over ranks,
the way ``bench.py --gpus 2`` does under torch.distributed.run with NCCL."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench

    w, r, local = bench.dist_env()
    assert (w, r, local) == (world, rank, rank)
    dist = bench.init_dist(w, "gloo")
    bench.barrier(dist)
    got = bench.max_over_ranks(dist, 1.5 + rank, "cpu")
    bench.barrier(dist)
    out[rank] = got
    dist.destroy_process_group()


def test_two_ranks_agree_on_max():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert dict(out) == {0: 2.5, 1: 2.5}


def test_single_rank_is_identity():
    import bench
    assert bench.init_dist(1, "gloo") is None
    assert bench.max_over_ranks(None, 3.25) == 3.25


def test_accounting_matches_the_pages_conventions():
    """FLOPs count only the unmasked causal pairs; decode bytes count K and
    V of every context token plus q, o and the used table entries."""
    import bench
    from exact_io_aware_86_b200 import inputs
    assert bench.prefill_flops([2048] * 4, 16, 128) == 4 * 128 * 16 * 4 * 2048 * 2049 // 2
    assert bench.prefill_flops([3], 1, 2, causal=False) == 4 * 2 * 9
    d = inputs.make_decode([17, 32], 4, 2, 16, 16, seed=1)
    # 49 tokens x Hkv 2 x d 16 x 2 B x (K, V); q and o; ceil(17/16) + ceil(32/16) = 4 pages; 2 lengths
    assert bench.decode_bytes(d) == (49 * 2 * 16 * 2 * 2) + 2 * 2 * 4 * 16 * 2 + 4 * 4 + 4 * 2
