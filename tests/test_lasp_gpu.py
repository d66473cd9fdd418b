"""LASP+ on one GPU: the chunk-state and prefix kernels against the oracle, and the whole
scheme with the ranks run one after another (the all-gather is the stacking of the chunk
states in rank order, which is what it produces on every rank).

Bounds: states 1e-5 (bf16 inputs, fp32 accumulation) and 1e-6 (fp32 path), relative L2 per
(sequence, head); outputs 2e-2 (bf16) and 1e-5 (fp32); the prefix sum bit-exact against a
float32 loop in the same order.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_04_b200 import api, lasp, synth

pytestmark = pytest.mark.gpu

TOL = {torch.float32: 1e-5, torch.bfloat16: 2e-2}
STOL = {torch.float32: 1e-6, torch.bfloat16: 1e-5}
CASES = [(torch.bfloat16, 128), (torch.bfloat16, 64), (torch.float32, 128), (torch.float32, 64)]
IDS = [f"{'bf16' if d == torch.bfloat16 else 'fp32'}-d{D}" for d, D in CASES]


def _state_err(st_gpu, st_ref):
    return oracle.max_rel_l2_per_state(st_gpu, st_ref)


@pytest.mark.parametrize("dtype,D", CASES, ids=IDS)
def test_chunk_state_against_oracle(dtype, D):
    H = 3
    cu = [0, 1, 1, 128, 300, 1000, 1129]        # 1 token, empty, exact block, tails
    q, k, v = synth.qkv(cu[-1], H, D, seed=41, dtype=dtype, device="cuda")
    st = api.chunk_state(k, v, cu_seqlens=cu)
    torch.cuda.synchronize()
    assert api.device_status() == api.LA_OK
    assert _state_err(st.cpu().numpy(), oracle.final_state(k, v, cu)) <= STOL[dtype]
    # uniform batch form
    kb, vb = (x[:1000].reshape(4, 250, H, D) for x in (k, v))
    st = api.chunk_state(kb.contiguous(), vb.contiguous())
    torch.cuda.synchronize()
    ref = np.stack([oracle.final_state(kb[b], vb[b])[0] for b in range(4)])
    assert _state_err(st.cpu().numpy(), ref) <= STOL[dtype]


def test_chunk_state_long_sequence():
    N, H, D = 65536, 4, 128
    _, k, v = synth.qkv(N, H, D, seed=42, dtype=torch.bfloat16, device="cuda")
    st = api.chunk_state(k, v)
    torch.cuda.synchronize()
    assert api.device_status() == api.LA_OK
    assert _state_err(st.cpu().numpy(), oracle.final_state(k, v)) <= 1e-5


@pytest.mark.parametrize("rank", [0, 1, 3, 4])
def test_state_prefix_is_ordered_sum(rank):
    R, S, H, D = 4, 2, 3, 64
    g = torch.randn((R, S, H, D, D), generator=synth.generator(43, "cuda"), device="cuda")
    out = api.state_prefix(g, rank)
    torch.cuda.synchronize()
    gh = g.cpu().numpy()
    ref = np.zeros((S, H, D, D), np.float32)
    for r in range(rank):
        ref = (ref + gh[r]).astype(np.float32)
    assert np.array_equal(out.cpu().numpy(), ref)


@pytest.mark.parametrize("dtype,D", CASES, ids=IDS)
@pytest.mark.parametrize("rmsnorm", [False, True], ids=["plain", "rmsnorm"])
def test_lasp_ranks_in_sequence(dtype, D, rmsnorm):
    """Four chunks of two packed sequences (uneven chunk lengths, an empty chunk): each
    rank's rows against the oracle's single run, and the state after the whole."""
    H, R = 2, 4
    lens = [1500, 700]
    chunks = [[400, 0, 700, 400], [129, 300, 1, 270]]   # rows of each sequence per rank
    q, k, v = synth.qkv(sum(lens), H, D, seed=44, dtype=dtype, device="cuda")
    starts = [0, lens[0]]
    rows, cus = [], []
    for r in range(R):
        idx, cu = [], [0]
        for s in range(2):
            a = starts[s] + sum(chunks[s][:r])
            idx += list(range(a, a + chunks[s][r]))
            cu.append(cu[-1] + chunks[s][r])
        rows.append(torch.as_tensor(idx, dtype=torch.long, device="cuda"))
        cus.append(cu)
    # step 1 on every rank, step 2 = stacking in rank order
    local = [api.chunk_state(k[rows[r]], v[rows[r]], cu_seqlens=cus[r]) for r in range(R)]
    gathered = torch.stack(local)
    o = torch.empty_like(q)
    for r in range(R):
        o[rows[r]] = lasp.chunk_prefill(q[rows[r]], k[rows[r]], v[rows[r]], gathered, r,
                                        beta=128, cu_seqlens=cus[r], rmsnorm=rmsnorm)
    final = api.state_prefix(gathered, R)
    torch.cuda.synchronize()
    assert api.device_status() == api.LA_OK
    cu_full = [0, lens[0], sum(lens)]
    ref_o, ref_s = oracle.recurrent(q, k, v, cu_full, rmsnorm=rmsnorm)
    assert oracle.max_rel_l2_per_head(o, ref_o, cu_full) <= TOL[dtype]
    assert _state_err(final.cpu().numpy(), ref_s) <= STOL[dtype]


def test_lasp_prefill_one_nccl_rank():
    """lasp.lasp_prefill itself on a one-rank NCCL group, on a side stream: the all-gather
    runs on the kernels' stream between la_chunk_state and la_state_prefix, and the rows and
    the final state match the oracle's single pass (three packed sequences, bf16, D = 128)."""
    import datetime

    import torch.distributed as dist
    if dist.is_initialized():
        pytest.skip("a process group is already set up in this process")
    dist.init_process_group("nccl", store=dist.HashStore(), rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        H, D = 4, 128
        cu = [0, 1000, 1000, 2333]
        q, k, v = synth.qkv(cu[-1], H, D, seed=45, dtype=torch.bfloat16, device="cuda")
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        o, st = lasp.lasp_prefill(q, k, v, cu_seqlens=cu, return_state=True, stream=s)
        s.synchronize()
        assert api.device_status(s) == api.LA_OK
    finally:
        dist.destroy_process_group()
    ref_o, ref_s = oracle.recurrent(q, k, v, cu)
    assert oracle.max_rel_l2_per_head(o, ref_o, cu) <= TOL[torch.bfloat16]
    assert _state_err(st.cpu().numpy(), ref_s) <= STOL[torch.bfloat16]
