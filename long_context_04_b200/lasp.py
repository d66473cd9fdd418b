"""LASP+ sequence parallelism: long sequences split into contiguous chunks, one per rank.

The pages name LASP+ as lightning attention's sequence-parallel scheme (mizuki blog,
section 5 "pretraining" and appendix "key concepts"; jvyan.cn article, section 3):
local prefix sums of the chunk states, an all-gather, and the serial dependency across
chunks becomes parallel work.  For rank r holding rows [r L, (r+1) L) of every sequence:

 1. local state       S_r = K_r^T V_r                   ``api.chunk_state``
 2. all-gather        [S_0, ..., S_{R-1}] on every rank   the only exchange (NCCL)
 3. initial state     X_r = sum_{r' < r} S_{r'}           ``api.state_prefix``
 4. chunk prefill     O_r from X_r                        ``api.prefill(initial_state=X_r)``

Step 2 moves S*H*D*D*4 bytes per rank (4 MiB for one sequence, H = 64, D = 128).  Every
arithmetic step runs in the library's kernels; torch.distributed only moves bytes.

``ops`` names the four operations (default: this package's C-ABI binding); tests
substitute other implementations to check the orchestration itself.
"""
from __future__ import annotations

import contextlib

import torch

from . import api


def all_gather_states(local: torch.Tensor, group=None) -> torch.Tensor:
    """[R, *local.shape]: every rank's local state, in rank order, on every rank.

    One ``all_gather_into_tensor`` into a buffer that holds the R local states one after
    the other along the first axis: the layout both NCCL and gloo accept, so that the CPU
    tests run the same call as the GPU ranks."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    local = local.contiguous()
    flat = local.new_empty((world * local.shape[0],) + tuple(local.shape[1:]))
    dist.all_gather_into_tensor(flat, local, group=group)
    return flat.view((world,) + tuple(local.shape))


def chunk_prefill(q, k, v, gathered, rank: int, *, beta: int = 128, cu_seqlens=None,
                  rmsnorm: bool = False, ops=api, stream=None):
    """Step 3 and 4 for chunk ``rank``: its initial state from the gathered chunk states,
    then the prefill of its rows from that state.  Returns ``o``."""
    init = ops.state_prefix(gathered, rank, stream=stream)
    return ops.prefill(q, k, v, beta=beta, cu_seqlens=cu_seqlens, rmsnorm=rmsnorm,
                       initial_state=init, stream=stream)


def lasp_prefill(q, k, v, *, group=None, beta: int = 128, cu_seqlens=None, rmsnorm: bool = False,
                 return_state: bool = False, ops=api, stream=None):
    """Prefill of this rank's chunk of every sequence.

    ``q, k, v``: this rank's rows, ``[B, L, H, D]`` or packed ``[T_r, H, D]`` with
    ``cu_seqlens`` (the chunk of each sequence; a chunk may be empty).  Every rank holds
    the same sequences in the same order.  Returns ``o`` (this rank's rows), or
    ``(o, state)`` with ``return_state``: the state after the whole of every sequence,
    the same on every rank.
    """
    import torch.distributed as dist
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    # the collective runs on the stream the kernels use, so that it is ordered with them
    ctx = torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()
    with ctx:
        local = ops.chunk_state(k, v, cu_seqlens=cu_seqlens, stream=stream)
        gathered = all_gather_states(local, group)
        o = chunk_prefill(q, k, v, gathered, rank, beta=beta, cu_seqlens=cu_seqlens,
                          rmsnorm=rmsnorm, ops=ops, stream=stream)
        if return_state:
            return o, ops.state_prefix(gathered, world, stream=stream)
    return o
