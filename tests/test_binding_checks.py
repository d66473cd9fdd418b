"""Argument checks of the Python binding, on the CPU.

Outputs are handed to the library as raw pointers, so the binding must reject a wrong
shape before any call: a short output buffer would be written out of bounds.  Here the
device check is relaxed (CPU tensors stand in for CUDA ones) and the library loader is
replaced by a stub, so each case shows either a ValueError raised by the binding or that
the call got as far as the library with valid arguments.
"""
import pytest
import torch

from long_context_04_b200 import api


class Reached(Exception):
    pass


@pytest.fixture(autouse=True)
def cpu_binding(monkeypatch):
    monkeypatch.setattr(api, "_on_gpu", lambda t: True)

    def stub():
        raise Reached()
    monkeypatch.setattr(api, "lib", stub)


def bf(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def f32(*shape):
    return torch.zeros(shape, dtype=torch.float32)


def test_prefill_shapes():
    q = bf(10, 2, 64)
    with pytest.raises(Reached):
        api.prefill(q, q, q, beta=64, cu_seqlens=[0, 4, 10], out=bf(10, 2, 64), state_out=f32(2, 2, 64, 64))
    with pytest.raises(ValueError, match="out must have shape"):
        api.prefill(q, q, q, beta=64, out=bf(9, 2, 64))
    with pytest.raises(ValueError, match="state_out must have shape"):
        api.prefill(q, q, q, beta=64, cu_seqlens=[0, 4, 10], state_out=f32(1, 2, 64, 64))
    with pytest.raises(ValueError, match="initial_state"):
        api.prefill(q, q, q, beta=64, initial_state=f32(2, 2, 64, 64))
    with pytest.raises(ValueError, match="one shape"):
        api.prefill(q, bf(10, 2, 128), q)
    with pytest.raises(ValueError, match="must be"):
        api.prefill(q, q, q, out=f32(10, 2, 64))              # dtype of out
    q4 = bf(2, 5, 2, 64)
    with pytest.raises(ValueError, match="state_out must have shape"):
        api.prefill(q4, q4, q4, beta=64, state_out=f32(1, 2, 64, 64))
    with pytest.raises(Reached):
        api.prefill(q4, q4, q4, beta=64, return_state=True)


def test_decode_step_shapes():
    q = bf(3, 2, 64)
    with pytest.raises(Reached):
        api.decode_step(q, q, q, f32(3, 2, 64, 64), out=bf(3, 2, 64))
    with pytest.raises(ValueError, match="out must have shape"):
        api.decode_step(q, q, q, f32(3, 2, 64, 64), out=bf(2, 2, 64))
    with pytest.raises(ValueError, match="state must be"):
        api.decode_step(q, q, q, f32(3, 2, 64, 32))
    with pytest.raises(ValueError, match=r"q must be \[B, H, D\]"):
        api.decode_step(bf(3, 2, 1, 64), bf(3, 2, 1, 64), bf(3, 2, 1, 64), f32(3, 2, 64, 64))


def test_state_out_shapes():
    ws = f32(4, 2, 64, 64)
    with pytest.raises(Reached):
        api.state_out(ws, f32(9, 2, 64, 64), torch.zeros(4, dtype=torch.int32))
    with pytest.raises(ValueError, match="state_dst must have shape"):
        api.state_out(ws, f32(9, 2, 128, 128))
    with pytest.raises(ValueError, match="seq_to_slot must have shape"):
        api.state_out(ws, f32(9, 2, 64, 64), torch.zeros(3, dtype=torch.int32))
    with pytest.raises(ValueError, match="seq_to_slot must be"):
        api.state_out(ws, f32(9, 2, 64, 64), torch.zeros(4, dtype=torch.int64))


def test_chunk_state_and_prefix_shapes():
    k = bf(10, 2, 64)
    with pytest.raises(Reached):
        api.chunk_state(k, k, cu_seqlens=[0, 3, 10], state_out=f32(2, 2, 64, 64))
    with pytest.raises(ValueError, match="state_out must have shape"):
        api.chunk_state(k, k, cu_seqlens=[0, 3, 10], state_out=f32(1, 2, 64, 64))
    g = f32(3, 2, 2, 64, 64)
    with pytest.raises(Reached):
        api.state_prefix(g, 1, out=f32(2, 2, 64, 64))
    with pytest.raises(ValueError, match="out must have shape"):
        api.state_prefix(g, 1, out=f32(2, 2, 64, 32))
    with pytest.raises(ValueError, match="gathered must be"):
        api.state_prefix(f32(2, 2, 64, 64), 1)


def test_one_device_per_call():
    """Every tensor of a call must be on q's device (the library launches there); a
    tensor elsewhere is rejected before the library is reached.  ``meta`` tensors stand
    in for a second device."""
    q = bf(10, 2, 64)
    other = torch.zeros((10, 2, 64), dtype=torch.bfloat16, device="meta")
    with pytest.raises(ValueError, match="is on meta"):
        api.prefill(q, other, q, beta=64)
    with pytest.raises(ValueError, match="is on meta"):
        api.prefill(q, q, q, beta=64, out=other)
    with pytest.raises(ValueError, match="is on meta"):
        api.prefill(q, q, q, beta=64, state_out=torch.zeros((1, 2, 64, 64), device="meta"))
    with pytest.raises(ValueError, match="is on meta"):
        api.prefill(q, q, q, beta=64, initial_state=torch.zeros((1, 2, 64, 64), device="meta"))
    qd = bf(3, 2, 64)
    with pytest.raises(ValueError, match="is on meta"):
        api.decode_step(qd, qd, qd, torch.zeros((3, 2, 64, 64), device="meta"))
    ws = f32(4, 2, 64, 64)
    with pytest.raises(ValueError, match="is on meta"):
        api.state_out(ws, torch.zeros((4, 2, 64, 64), device="meta"))
    with pytest.raises(ValueError, match="is on meta"):
        api.state_out(ws, f32(4, 2, 64, 64), torch.zeros(4, dtype=torch.int32, device="meta"))
    with pytest.raises(ValueError, match="is on meta"):
        api.chunk_state(q, other)
    with pytest.raises(ValueError, match="is on meta"):
        api.state_prefix(f32(2, 1, 2, 64, 64), 1, out=torch.zeros((1, 2, 64, 64), device="meta"))


def test_overlapping_state_buffers():
    """initial_state is copied into a separate state_out before the in-place update, so
    two views that overlap without coinciding would corrupt it: rejected."""
    q = bf(10, 2, 64)
    n = 2 * 64 * 64
    buf = f32(3 * n)
    init = buf[:2 * n].view(2, 2, 64, 64)
    shifted = buf[n:3 * n].view(2, 2, 64, 64)
    with pytest.raises(ValueError, match="overlap"):
        api.prefill(q, q, q, beta=64, cu_seqlens=[0, 4, 10], initial_state=init, state_out=shifted)
    with pytest.raises(Reached):       # the same tensor: an in-place update, allowed
        api.prefill(q, q, q, beta=64, cu_seqlens=[0, 4, 10], initial_state=init, state_out=init)
    with pytest.raises(Reached):       # disjoint
        api.prefill(q, q, q, beta=64, cu_seqlens=[0, 4, 10], initial_state=init,
                    state_out=f32(2, 2, 64, 64))
    with pytest.raises(ValueError, match="overlap"):
        api.state_out(init, shifted)
    g = f32(3, 1, 2, 64, 64)
    with pytest.raises(ValueError, match="overlap"):
        api.state_prefix(g, 1, out=g[1])
