"""Decode parity (one token per sequence) and the prefill -> decode state hand-off."""
import numpy as np
import pytest
import torch

import oracle
from long_context_04_b200 import api, synth

pytestmark = pytest.mark.gpu


def _rand_state(B, H, D, seed):
    g = synth.generator(seed, "cuda")
    return torch.randn(B, H, D, D, generator=g, device="cuda", dtype=torch.float32)


@pytest.mark.parametrize("dtype,tol", [(torch.float32, 1e-5), (torch.bfloat16, 2e-2)])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("rmsnorm", [False, True])
def test_decode_step_all_heads(dtype, tol, D, rmsnorm):
    B, H = 5, 3
    st = _rand_state(B, H, D, 7)
    st0 = st.cpu().double().numpy()
    q, k, v = synth.decode_tokens(B, H, D, step=0, seed=1, dtype=dtype, device="cuda")
    o = api.decode_step(q, k, v, st, rmsnorm=rmsnorm)
    torch.cuda.synchronize()
    o_ref, st_ref = oracle.decode_step(q, k, v, st0, rmsnorm=rmsnorm)
    assert oracle.max_rel_l2_per_head(o, o_ref) <= tol
    # the fp32 state update is one FMA per element: within a few ulp
    assert oracle.rel_l2(st, st_ref) <= 1e-6


def test_decode_equals_next_prefill_row():
    """decode(state of prefill_N, token N+1) = row N+1 of prefill_{N+1} (bf16 path)."""
    N, H, D = 1000, 4, 128
    q, k, v = synth.qkv(N + 1, H, D, seed=11, dtype=torch.bfloat16, device="cuda")
    _, st = api.prefill(q[:N].contiguous(), k[:N].contiguous(), v[:N].contiguous(), beta=128,
                        return_state=True)
    o_full = api.prefill(q, k, v, beta=128)
    o_dec = api.decode_step(q[N:].contiguous(), k[N:].contiguous(), v[N:].contiguous(), st)
    torch.cuda.synchronize()
    o_ref, _ = oracle.recurrent(q, k, v)
    assert oracle.max_rel_l2_per_head(o_dec, o_ref[N:]) <= 2e-2
    assert oracle.max_rel_l2_per_head(o_full[N:], o_ref[N:]) <= 2e-2


def test_state_out_with_slot_map():
    S, H, D, slots = 5, 3, 128, 9
    ws = _rand_state(S, H, D, 12)
    dst = torch.zeros(slots, H, D, D, device="cuda")
    m = torch.tensor([8, 0, 3, 4, 6], dtype=torch.int32, device="cuda")
    api.state_out(ws, dst, m)
    torch.cuda.synchronize()
    assert api.device_status() == api.LA_OK
    for s, slot in enumerate(m.tolist()):
        assert torch.equal(dst[slot], ws[s])
    untouched = [i for i in range(slots) if i not in m.tolist()]
    assert bool((dst[untouched] == 0).all())


def test_state_out_out_of_range_slot_is_reported():
    S, H, D = 2, 2, 64
    ws = _rand_state(S, H, D, 13)
    dst = torch.zeros(2, H, D, D, device="cuda")
    m = torch.tensor([1, 7], dtype=torch.int32, device="cuda")
    api.state_out(ws, dst, m)
    assert api.device_status() == api.LA_ERR_DEVICE_RANGE
    assert api.device_status() == api.LA_OK  # cleared
    assert torch.equal(dst[1], ws[0])


def test_config5_decode_from_prefill_state():
    """B=256, H=64, D=128: state from seeded N=4096 prefills (8 chunks of 32 sequences,
    handed over with la_state_out), then 64 decode steps.  Checks: step 1 for every (b, h)
    from the exact GPU input state; 64 sampled (b, h) from scratch in fp64 over all 64 steps."""
    B, H, D, N, steps, chunk = 256, 64, 128, 4096, 64, 32
    state = torch.empty(B, H, D, D, device="cuda")
    # 64 pairs with distinct b (37 is odd, so i -> 37 i + 5 mod 256 is one-to-one), corners included
    sample = [(0, 0), (255, 63)] + [((37 * i + 5) % 256, (29 * i + 3) % 64) for i in range(62)]
    kept = {}
    for c in range(B // chunk):
        q, k, v = synth.qkv(chunk * N, H, D, seed=100 + c, dtype=torch.bfloat16, device="cuda")
        q4, k4, v4 = (x.view(chunk, N, H, D) for x in (q, k, v))
        _, ws = api.prefill(q4, k4, v4, beta=128, return_state=True)
        slots = torch.arange(c * chunk, (c + 1) * chunk, dtype=torch.int32, device="cuda")
        api.state_out(ws, state, slots)
        for (b, h) in sample:
            if c * chunk <= b < (c + 1) * chunk:
                lb = b - c * chunk
                kept[(b, h)] = tuple(x[lb, :, h:h + 1].cpu() for x in (q4, k4, v4))
        del q, k, v, q4, k4, v4, ws
    torch.cuda.synchronize()
    assert api.device_status() == api.LA_OK

    st_in = state.cpu().double().numpy()
    toks = [synth.decode_tokens(B, H, D, step=t, seed=0, device="cuda") for t in range(steps)]
    outs = []
    for t in range(steps):
        outs.append(api.decode_step(*toks[t], state))
    torch.cuda.synchronize()

    # (a) step 1 for every (b, h), from the exact input state
    o1_ref, _ = oracle.decode_step(*toks[0], st_in)
    assert oracle.max_rel_l2_per_head(outs[0], o1_ref) <= 2e-2

    # (b) sampled (b, h): fp64 prefill of the 4096 tokens, then the 64 decode steps
    for (b, h), (qs, ks, vs) in kept.items():
        _, st = oracle.recurrent(qs, ks, vs, want_o=False)
        for t in range(steps):
            qt, kt, vt = (x[b:b + 1, h:h + 1] for x in toks[t])
            o_ref, st = oracle.decode_step(qt, kt, vt, st)
            err = oracle.rel_l2(outs[t][b, h].cpu().double().numpy(), o_ref[0, 0])
            assert err <= 2e-2, (b, h, t, err)
