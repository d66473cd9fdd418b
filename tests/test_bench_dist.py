"""Multi-rank host logic of bench.py on CPU: two gloo ranks.

The benchmark's N-GPU mode runs independent replicas and only uses the
process group for barriers and the max/sum over ranks of the timed values;
those helpers, and the reference arm's rank handling, are exercised here.
"""
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
    import torch.distributed as dist
    r, w, local = bench.dist_init()
    assert (r, w, local) == (rank, world, rank)
    bench.dist_setup(w, "gloo")
    bench.dist_barrier(w)
    mx = bench.dist_max(float(rank + 1) * 1.5, w)
    sm = bench.dist_sum(float(rank + 1), w)
    # the reference arm runs on rank 0 only; the other ranks return 0 without work
    rc = bench.run_reference(_Args()) if rank != 0 else 0
    bench.dist_barrier(w)
    dist.destroy_process_group()
    out.put((rank, mx, sm, rc))


class _Args:
    workload = "prefill_n16k"
    steps = 3
    warmup = 3
    gpus = 2


def test_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(world))
    for rank, mx, sm, rc in res:
        assert mx == pytest.approx(3.0)   # max over ranks of 1.5 * (rank + 1)
        assert sm == pytest.approx(3.0)   # 1 + 2
        assert rc == 0


def test_single_process_helpers_are_identities():
    import bench
    assert bench.dist_max(2.5, 1) == 2.5
    assert bench.dist_sum(2.5, 1) == 2.5
    bench.dist_barrier(1)
    assert bench.tiled_flops_per_token_head(128, 128) == 131072
    assert bench.prefill_bytes(131072, 64, 128) == 8589934592
    assert bench.decode_bytes(256, 64, 128) == 2164260864
