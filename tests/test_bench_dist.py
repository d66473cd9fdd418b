"""Multi-rank host logic of bench.py on CPU: two gloo ranks.

The benchmark's N-GPU mode runs independent replicas and only uses the
process group for barriers and the max/sum over ranks of the timed values;
those helpers, and the reference arm's rank handling, are exercised here.
"""
import contextlib
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

        @staticmethod
        def stream(s):
            return contextlib.nullcontext()


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
    assert set(res) == {"plain", "rmsnorm", "beta64", "initial_state", "launches_per_option",
                        "status", "order"}
    assert api.options.count((128, False, False)) == 4
    assert api.options.count((128, True, False)) == 4
    assert api.options.count((64, False, False)) == 4
    assert api.options.count((128, False, True)) == 4
    # the options take turns launch by launch: plain, rmsnorm, beta64, initial_state, ...
    assert api.options[4:8] == [(128, False, False), (128, True, False), (64, False, False),
                                (128, False, True)]
    assert res["beta64"]["ms_per_launch"] == pytest.approx(1000.0)   # one fake tick per launch
    assert res["rmsnorm"]["vs_plain"] == pytest.approx(1.0)


class _LaspApi:
    """fp64 CPU stand-ins (the oracle) for the three kernels of a LASP+ step; each call is
    logged so that the test can check the order of the steps."""

    def __init__(self):
        self.calls = []

    def chunk_state(self, k, v, state_out=None, stream=None):
        import oracle
        st = torch_from(oracle.final_state(k[0].numpy(), v[0].numpy()))
        self.calls.append("chunk_state")
        if state_out is None:
            return st
        state_out.copy_(st)
        return state_out

    def state_prefix(self, gathered, rank, out=None, stream=None):
        self.calls.append(("state_prefix", tuple(gathered.shape)))
        out.zero_()
        for r in range(rank):
            out += gathered[r]
        return out

    def prefill(self, q, k, v, beta=128, out=None, initial_state=None, stream=None):
        import oracle
        o, _ = oracle.recurrent(q[0].numpy(), k[0].numpy(), v[0].numpy(),
                                initial_state=initial_state.numpy())
        out[0].copy_(torch_from(o))
        self.calls.append("prefill")

    def device_status(self, stream=None):
        return 0

    def status_string(self, status):
        return "LA_OK"


def torch_from(a):
    import torch
    return torch.from_numpy(a)


LASP_L, LASP_H, LASP_D = 96, 2, 8


def _lasp_inputs(world):
    import numpy as np
    g = np.random.default_rng(11)
    return tuple(g.standard_normal((world * LASP_L, LASP_H, LASP_D)) / np.sqrt(LASP_D)
                 for _ in range(3))


def _lasp_worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch
    import torch.distributed as dist

    import bench
    from long_context_04_b200 import lasp
    bench.dist_setup(world, "gloo")
    rows = slice(rank * LASP_L, (rank + 1) * LASP_L)
    q, k, v = (torch.from_numpy(x[rows]).unsqueeze(0).contiguous() for x in _lasp_inputs(world))
    o = torch.empty_like(q)
    api = _LaspApi()
    res = bench.bench_lasp(api, lasp, _FakeTorch, _FakeStream(), q, k, v, o, rank, world, 6544.0,
                           reps=2, warm=1)
    dist.destroy_process_group()
    out.put((rank, res, o[0].numpy(), api.calls))


@pytest.mark.parametrize("world", [2, 3])
def test_lasp_leg_gloo_ranks(world):
    """bench.py's LASP+ leg on gloo ranks, through lasp.all_gather_states itself, with the
    oracle standing in for the kernels: each rank's rows equal the oracle's single pass
    over the whole sequence, the steps run in the method's order, and the per-rank table
    has one row per rank."""
    import oracle
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_lasp_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in range(world)), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    qq, kk, vv = _lasp_inputs(world)
    ref, _ = oracle.recurrent(qq, kk, vv)
    for rank, r, o, calls in res:
        assert oracle.rel_l2(o, ref[rank * LASP_L:(rank + 1) * LASP_L]) <= 1e-12, rank
        step = ["chunk_state", ("state_prefix", (world, 1, LASP_H, LASP_D, LASP_D)), "prefill"]
        assert calls == ["chunk_state"] + step * 3     # allocation call, 1 warm-up, 2 timed
        assert len(r["per_rank_ms_median"]) == world
        assert set(r["per_rank_ms_median"][0]) == set(bench_parts())
        assert r["status"] == "LA_OK"
        assert r["gathered_bytes_per_rank"] == world * LASP_H * LASP_D * LASP_D * 4
        assert r["tokens_per_s"] > 0 and r["slowest_rank_ms_per_step"] > 0


def bench_parts():
    import bench
    return bench.LASP_PARTS
