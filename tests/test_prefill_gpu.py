"""Prefill parity: the CUDA path (through the C ABI) against the fp64 oracle.

Error metric: relative L2 per (sequence, head), maximum reported.  Bounds:
1e-5 for the fp32 path, 2e-2 for bf16 inputs with fp32 accumulation.
"""
import pytest
import torch

import oracle
from long_context_04_b200 import api, synth

pytestmark = pytest.mark.gpu

TOL = {torch.float32: 1e-5, torch.bfloat16: 2e-2}
SENTINEL = 12288.0  # exactly representable in bf16 and fp32


def _packed_out(T, H, D, dtype, pad=64):
    """Output buffer followed by sentinel rows, to catch stores past the end."""
    buf = torch.full((T + pad, H, D), SENTINEL, dtype=dtype, device="cuda")
    return buf, buf[:T]


def _check_canary(buf, T):
    assert bool((buf[T:].float() == SENTINEL).all()), "kernel wrote past the output"


def _state_err(st_gpu, st_ref):
    return oracle.max_rel_l2_per_state(st_gpu, st_ref)


def _run_and_compare(T, H, D, beta, dtype, cu, rmsnorm, seed=0, form="recurrent"):
    q, k, v = synth.qkv(T, H, D, seed=seed, dtype=dtype, device="cuda")
    buf, o = _packed_out(T, H, D, dtype)
    o, st = api.prefill(q, k, v, beta=beta, cu_seqlens=cu, rmsnorm=rmsnorm, return_state=True,
                        out=o)
    torch.cuda.synchronize()
    assert api.device_status() == api.LA_OK
    _check_canary(buf, T)
    fn = oracle.quadratic if form == "quadratic" else oracle.recurrent
    o_ref, st_ref = fn(q, k, v, cu, rmsnorm=rmsnorm)
    err = oracle.max_rel_l2_per_head(o, o_ref, cu)
    st_err = _state_err(st.cpu().double().numpy(), st_ref)
    return err, st_err


def test_config1_tiny_fp32():
    """B=1, H=2, N=256, D=64, beta=64, fp32, no norm; quadratic-form oracle."""
    err, st_err = _run_and_compare(256, 2, 64, 64, torch.float32, None, False, form="quadratic")
    assert err <= 1e-5 and st_err <= 1e-5, (err, st_err)


RAGGED = [0, 1, 64, 64, 127, 255, 384, 1000]  # empty, 1 token, exact block, tails


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("beta", [64, 128])
@pytest.mark.parametrize("rmsnorm", [False, True])
def test_fp32_ragged_varlen(D, beta, rmsnorm):
    cu = RAGGED
    err, st_err = _run_and_compare(cu[-1], 3, D, beta, torch.float32, cu, rmsnorm, seed=1)
    assert err <= 1e-5 and st_err <= 1e-5, (err, st_err)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("beta", [64, 128])
@pytest.mark.parametrize("rmsnorm", [False, True])
def test_bf16_ragged_varlen(D, beta, rmsnorm):
    cu = RAGGED
    err, st_err = _run_and_compare(cu[-1], 4, D, beta, torch.bfloat16, cu, rmsnorm, seed=2)
    assert err <= 2e-2 and st_err <= 2e-2, (err, st_err)


@pytest.mark.parametrize("N", [1, 63, 65, 127, 129, 1000])
def test_bf16_uniform_batch_odd_lengths(N):
    """B=3 equal sequences (no cu_seqlens), lengths around the block size."""
    B, H, D = 3, 2, 128
    q, k, v = synth.qkv(B * N, H, D, seed=3, dtype=torch.bfloat16, device="cuda")
    q4, k4, v4 = (x.view(B, N, H, D) for x in (q, k, v))
    o, st = api.prefill(q4, k4, v4, beta=128, return_state=True)
    torch.cuda.synchronize()
    cu = [b * N for b in range(B + 1)]
    o_ref, st_ref = oracle.recurrent(q, k, v, cu)
    assert oracle.max_rel_l2_per_head(o.view(B * N, H, D), o_ref, cu) <= 2e-2
    assert _state_err(st.cpu().double().numpy(), st_ref) <= 2e-2


def test_bf16_beta_independence():
    """beta = 64 and beta = 128 agree with each other and with the oracle."""
    T, H, D = 2048, 4, 128
    q, k, v = synth.qkv(T, H, D, seed=4, dtype=torch.bfloat16, device="cuda")
    o64 = api.prefill(q, k, v, beta=64)
    o128 = api.prefill(q, k, v, beta=128)
    torch.cuda.synchronize()
    o_ref, _ = oracle.recurrent(q, k, v)
    assert oracle.max_rel_l2_per_head(o64, o_ref) <= 2e-2
    assert oracle.max_rel_l2_per_head(o128, o_ref) <= 2e-2
    assert oracle.max_rel_l2_per_head(o64, o128.double().cpu().numpy()) <= 2e-2


def test_bf16_packed_equals_separate():
    """A packed batch gives each sequence the result of running it alone (state reset)."""
    cu = [0, 300, 301, 777, 1500]
    H, D = 2, 128
    q, k, v = synth.qkv(cu[-1], H, D, seed=5, dtype=torch.bfloat16, device="cuda")
    o, st = api.prefill(q, k, v, beta=128, cu_seqlens=cu, return_state=True)
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        o_s, st_s = api.prefill(q[a:b].contiguous(), k[a:b].contiguous(), v[a:b].contiguous(),
                                beta=128, return_state=True)
        torch.cuda.synchronize()
        assert torch.equal(o[a:b], o_s), f"sequence {s}"
        assert torch.equal(st[s], st_s[0]), f"state {s}"


@pytest.mark.parametrize("beta", [64, 128])
def test_config2_layer_prefill(beta):
    """B=1, H=64, N=8192, D=128, bf16, RMSNorm: sampled heads + all final states."""
    T, H, D = 8192, 64, 128
    q, k, v = synth.qkv(T, H, D, seed=0, dtype=torch.bfloat16, device="cuda")
    o, st = api.prefill(q, k, v, beta=beta, rmsnorm=True, return_state=True)
    torch.cuda.synchronize()
    heads = [0, 17, 38, 63]
    o_ref, _ = oracle.recurrent(q[:, heads], k[:, heads], v[:, heads], rmsnorm=True)
    assert oracle.max_rel_l2_per_head(o[:, heads], o_ref) <= 2e-2
    st_ref = oracle.final_state(k, v)
    assert _state_err(st.cpu().double().numpy(), st_ref) <= 2e-2


def test_config3_long_context():
    """B=1, H=64, N=131072, D=128, beta=128: heads {0, 37} in full + every head's final state."""
    T, H, D = 131072, 64, 128
    q, k, v = synth.qkv(T, H, D, seed=0, dtype=torch.bfloat16, device="cuda")
    o, st = api.prefill(q, k, v, beta=128, return_state=True)
    torch.cuda.synchronize()
    assert api.device_status() == api.LA_OK
    heads = [0, 37]
    o_ref, st_ref = oracle.recurrent(q[:, heads], k[:, heads], v[:, heads])
    assert oracle.max_rel_l2_per_head(o[:, heads], o_ref) <= 2e-2
    assert _state_err(st[:, heads].cpu().double().numpy(), st_ref) <= 2e-2
    for h0 in range(0, H, 16):  # 16 heads at a time keeps the fp64 copies of K, V near 4 GB
        hs = list(range(h0, h0 + 16))
        st_ref2 = oracle.final_state(k[:, hs], v[:, hs])
        assert _state_err(st[:, hs].cpu().double().numpy(), st_ref2) <= 2e-2
    assert bool(torch.isfinite(o).all())


def test_config4_packed_varlen():
    """262144 tokens, 8 seeded sequences, H=64: all sequences on 2 heads + sampled states."""
    T, H, D, S = 262144, 64, 128, 8
    cu = synth.cu_seqlens_uniform(T, S, seed=0)
    q, k, v = synth.qkv(T, H, D, seed=0, dtype=torch.bfloat16, device="cuda")
    o, st = api.prefill(q, k, v, beta=128, cu_seqlens=cu, return_state=True)
    torch.cuda.synchronize()
    assert api.device_status() == api.LA_OK
    heads = [5, 60]
    o_ref, st_ref = oracle.recurrent(q[:, heads], k[:, heads], v[:, heads], cu)
    assert oracle.max_rel_l2_per_head(o[:, heads], o_ref, cu) <= 2e-2
    assert _state_err(st[:, heads].cpu().double().numpy(), st_ref) <= 2e-2
    sample = [0, 21, 42, 63]
    st_ref2 = oracle.final_state(k[:, sample], v[:, sample], cu)
    assert _state_err(st[:, sample].cpu().double().numpy(), st_ref2) <= 2e-2
