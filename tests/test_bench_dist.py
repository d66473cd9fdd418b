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


class _Event:
    clock = 0.0

    def __init__(self, enable_timing=True):
        self.t = None

    def record(self, stream=None):
        _Event.clock += 1.0
        self.t = _Event.clock

    def elapsed_time(self, other):
        return (other.t - self.t) * 1000.0


class _FakeTorch:
    import torch as _torch
    zeros = staticmethod(_torch.zeros)
    float32 = _torch.float32

    class cuda:
        Event = _Event

        @staticmethod
        def synchronize():
            pass


class _FakeStream:
    def synchronize(self):
        pass


class _FakeApi:
    def __init__(self):
        self.shapes = []
        self.options = []

    def prefill(self, q, k, v, beta=128, out=None, stream=None, rmsnorm=False, initial_state=None):
        assert q.shape == k.shape == v.shape == out.shape and out.data_ptr() == self.o_ptr
        assert beta in (64, 128)
        if initial_state is not None:
            assert tuple(initial_state.shape) == (q.shape[0], q.shape[2], q.shape[3], q.shape[3])
        self.shapes.append(tuple(q.shape))
        self.options.append((beta, rmsnorm, initial_state is not None))

    def device_status(self, stream=None):
        return 0

    def status_string(self, status):
        return "LA_OK"


def test_length_sweep_control_flow():
    """The sweep's host logic with stand-ins for CUDA events, the stream and the library:
    views of the one workload as B = T / N sequences, warm-up + timed launches per N, and
    one row per N that divides T."""
    import torch

    import bench
    T, H, D = 4096, 2, 8
    q, k, v, o = (torch.zeros(1, T, H, D) for _ in range(4))
    api = _FakeApi()
    api.o_ptr = o.data_ptr()
    res = bench.bench_length_sweep(api, _FakeTorch, _FakeStream(), q, k, v, o, 128, 6544.0, reps=4, warm=2)
    assert [r["N"] for r in res["rows"]] == [1024, 2048, 4096]
    assert [r["B"] for r in res["rows"]] == [4, 2, 1]
    assert api.shapes.count((4, 1024, H, D)) == 6 and api.shapes.count((1, 4096, H, D)) == 6
    r = res["rows"][0]
    assert r["ms_per_launch"] == pytest.approx(1000.0 / 4)    # one fake second over 4 launches
    assert r["tokens_per_s"] == pytest.approx(T / 0.25)
    assert r["hbm_frac"] == pytest.approx(8 * T * H * D / 0.25 / 1e9 / 6544.0)
    assert r["status"] == "LA_OK" and res["tokens_per_launch"] == T


def test_prefill_options_control_flow():
    import torch

    import bench
    T, H, D = 2048, 2, 8
    q, k, v, o = (torch.zeros(1, T, H, D) for _ in range(4))
    api = _FakeApi()
    api.o_ptr = o.data_ptr()
    res = bench.bench_prefill_options(api, _FakeTorch, _FakeStream(), q, k, v, o, 6544.0, reps=3, warm=1)
    assert set(res) == {"rmsnorm", "beta64", "initial_state", "launches_per_option"}
    assert api.options.count((128, True, False)) == 4
    assert api.options.count((64, False, False)) == 4
    assert api.options.count((128, False, True)) == 4
    assert res["beta64"]["ms_per_launch"] == pytest.approx(1000.0 / 3)
