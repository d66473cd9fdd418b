"""LASP+ orchestration across ranks on CPU: two and three gloo ranks.

``lasp.lasp_prefill`` is run with the four kernel-facing operations replaced by fp64
stand-ins built on the oracle (chunk state = K^T V, prefix = ordered sum, prefill from an
initial state), so that what is checked is the driver itself: that every rank gathers the
chunk states in rank order, takes the sum of the ranks before it, and returns its own rows
and the state after the whole sequence.  Each rank's rows and the final state must equal
the oracle's single run over the whole sequences.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleOps:
    """fp64 CPU stand-ins for api.chunk_state / api.state_prefix / api.prefill."""

    @staticmethod
    def chunk_state(k, v, cu_seqlens=None, stream=None):
        import oracle
        return torch.from_numpy(oracle.final_state(k.numpy(), v.numpy(), cu_seqlens))

    @staticmethod
    def state_prefix(gathered, rank, stream=None):
        out = torch.zeros_like(gathered[0])
        for r in range(rank):
            out += gathered[r]
        return out

    @staticmethod
    def prefill(q, k, v, beta=128, cu_seqlens=None, rmsnorm=False, initial_state=None, stream=None):
        import oracle
        o, _ = oracle.recurrent(q.numpy(), k.numpy(), v.numpy(), cu_seqlens, rmsnorm=rmsnorm,
                                initial_state=initial_state.numpy())
        return torch.from_numpy(o)


LENS = [200, 95]                            # two packed sequences
CHUNKS = {2: [[120, 80], [0, 95]], 3: [[50, 0, 150], [40, 40, 15]]}
H, D = 2, 8


def _inputs():
    g = np.random.default_rng(7)
    T = sum(LENS)
    return tuple(g.standard_normal((T, H, D)) / np.sqrt(D) for _ in range(3))


def _rows(world, rank):
    starts, idx, cu = [0, LENS[0]], [], [0]
    for s in range(2):
        a = starts[s] + sum(CHUNKS[world][s][:rank])
        idx += list(range(a, a + CHUNKS[world][s][rank]))
        cu.append(cu[-1] + CHUNKS[world][s][rank])
    return idx, cu


def _worker(rank, world, port, rms, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from long_context_04_b200 import lasp
    q, k, v = (torch.from_numpy(x) for x in _inputs())
    idx, cu = _rows(world, rank)
    o, st = lasp.lasp_prefill(q[idx], k[idx], v[idx], cu_seqlens=cu, rmsnorm=rms,
                              return_state=True, ops=OracleOps)
    dist.barrier()
    dist.destroy_process_group()
    out.put((rank, idx, o.numpy(), st.numpy()))


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("rms", [False, True], ids=["plain", "rmsnorm"])
def test_lasp_prefill_gloo_ranks(world, rms):
    import oracle
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, rms, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    qq, kk, vv = _inputs()
    cu_full = [0, LENS[0], sum(LENS)]
    ref_o, ref_s = oracle.recurrent(qq, kk, vv, cu_full, rmsnorm=rms)
    for rank, idx, o, st in res:
        if idx:
            assert oracle.rel_l2(o, ref_o[idx]) <= 1e-12, f"rank {rank} rows"
        assert oracle.rel_l2(st, ref_s) <= 1e-12, f"rank {rank} final state"
