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


def test_gpus_flag_launches_that_many_ranks():
    """`bench.py --gpus 2` outside torchrun re-launches itself under
    torch.distributed.run with two ranks; with --plumbing (gloo, no kernels)
    rank 0 prints a line whose n_gpus is 2, and only rank 0 prints."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2", "--plumbing",
                        "--steps", "3", "--warmup", "3"], capture_output=True, text=True, env=env,
                       timeout=300, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["n_gpus"] == 2 and line["steps"] == 3


def test_gpus_flag_must_match_the_launcher():
    """Under a launcher that set WORLD_SIZE, --gpus must agree with it."""
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "2", "--plumbing"],
                       capture_output=True, text=True, env=env, timeout=120, cwd=root)
    assert r.returncode != 0 and "WORLD_SIZE=1" in r.stderr


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


def _pairs_by_mask(L, causal, left, right):
    """Brute-force count of the (query, key) pairs a mask leaves visible."""
    n = 0
    for i in range(L):
        for j in range(L):
            if causal and j > i:
                continue
            if left >= 0 and j < i - left:
                continue
            if right >= 0 and j > i + right:
                continue
            n += 1
    return n


@pytest.mark.parametrize("L", [1, 2, 7, 33, 130])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("window", [(-1, -1), (0, 0), (3, -1), (-1, 5), (4, 2), (40, 0), (200, 7)])
def test_visible_pairs_equal_the_mask(L, causal, window):
    """The work a prefill workload is credited with counts exactly the pairs
    the mask (causal and/or window) leaves visible."""
    import bench
    assert bench.visible_pairs(L, causal, window) == _pairs_by_mask(L, causal, *window)


def test_append_decode_bytes():
    """An appended token joins the context; the call also moves k_new, v_new
    (read), the new k, v (written) and one cos and one sin row per request."""
    import bench
    from exact_io_aware_86_b200 import inputs
    a = inputs.make_append_decode([15, 40], 4, 2, 16, 16, seed=2, rotary_dim=8, max_pos=64)
    ctx = [16, 41]
    kv = sum(ctx) * 2 * 16 * 2 * 2
    qo = 2 * 2 * 4 * 16 * 2
    pages = 1 + 3
    extra = 2 * (2 * 2 * 2 * 16 * 2) + 2 * 2 * 4 * 4
    assert bench.decode_bytes(a) == kv + qo + 4 * pages + 4 * 2 + extra


def test_l2_flush_writes_then_reads():
    """The benchmark's flush writes one buffer and reads another (so the
    dirty lines of the write are gone before a timed call); checked on a
    small CPU buffer."""
    import torch
    import bench
    f = bench.L2Flush(torch.device("cpu"), 1 << 16)
    f.r.fill_(0.5)
    f(3.0)
    assert float(f.w.min()) == 3.0 and float(f.w.max()) == 3.0
    assert float(f.acc) == 0.5 * f.r.numel()
