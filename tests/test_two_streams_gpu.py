"""Prefill and decode on two CUDA streams at once.

The jvyan.cn article (section 2, "compute optimisation") runs length-1 and length>1
requests as two kernels on two CUDA streams, in parallel.  Here a prefill of the
MiniMax-layer size (B=1, N=8192, H=64, D=128, bf16, RMSNorm, final state exported)
is enqueued on one stream and 16 decode steps (B=16, H=64, D=128) on another, with no
synchronisation between them.  Events show that decode steps ran while the prefill
ran; afterwards every output and state is compared with the fp64 oracle per
(sequence, head), and the device status (one word per device) is read on both streams.
"""
import pytest
import torch

import oracle
from long_context_04_b200 import api, synth

pytestmark = pytest.mark.gpu


def test_prefill_and_decode_on_two_streams():
    N, H, D = 8192, 64, 128
    B, steps = 16, 16
    dev = torch.device("cuda", 0)
    q, k, v = synth.qkv(N, H, D, seed=21, dtype=torch.bfloat16, device=dev)
    o = torch.empty_like(q)
    st = torch.empty(1, H, D, D, dtype=torch.float32, device=dev)
    X = synth.initial_state(B, H, D, tokens=4096, seed=22, device=dev)
    state = X.clone()
    toks = [synth.decode_tokens(B, H, D, step=t, seed=23, device=dev) for t in range(steps)]
    outs = [torch.empty(B, H, D, dtype=torch.bfloat16, device=dev) for _ in range(steps)]
    torch.cuda.synchronize()

    pa, pb = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ea = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    eb = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    ea[0].record(pa)
    api.prefill(q, k, v, beta=128, rmsnorm=True, state_out=st, out=o, stream=pa)
    ea[1].record(pa)
    for t in range(steps):
        eb[t].record(pb)
        api.decode_step(*toks[t], state, out=outs[t], stream=pb)
    eb[steps].record(pb)
    assert api.device_status(pa) == api.LA_OK
    assert api.device_status(pb) == api.LA_OK
    torch.cuda.synchronize()

    # decode step t ran during the prefill if [eb[t], eb[t+1]] meets [ea[0], ea[1]]
    during = [t for t in range(steps)
              if eb[t].elapsed_time(ea[1]) > 0 and ea[0].elapsed_time(eb[t + 1]) > 0]
    assert during, "no decode step overlapped the prefill"

    o_ref, st_ref = oracle.recurrent(q, k, v, rmsnorm=True)
    assert oracle.max_rel_l2_per_head(o, o_ref) <= 2e-2
    assert oracle.max_rel_l2_per_state(st, st_ref) <= 1e-5

    ref_state = X.cpu().double().numpy()
    for t in range(steps):
        od_ref, ref_state = oracle.decode_step(*toks[t], ref_state)
        assert oracle.max_rel_l2_per_head(outs[t], od_ref) <= 2e-2, f"decode step {t}"
    assert oracle.max_rel_l2_per_state(state, ref_state) <= 1e-5
