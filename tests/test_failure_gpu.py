"""Failure detection on the GPU without a fault: a bounded wait that runs out.

Every device wait in the library gives up after a limit and records
LA_ERR_DEVICE_TIMEOUT in a per-device status word instead of spinning forever.
``la_selftest_wait`` launches one kernel whose only wait can never complete (a
barrier nothing arrives on, nothing else in flight); the test checks that the timeout
surfaces through ``la_get_device_status``, that reading it clears it, and that the
context stays usable for a normal prefill afterwards.
"""
import pytest
import torch

import oracle
from long_context_04_b200 import api, synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("limit_ns", [1_000, 20_000_000], ids=["1us", "20ms"])
def test_bounded_wait_surfaces_as_timeout(limit_ns):
    assert api.device_status() == api.LA_OK           # nothing pending
    api.selftest_wait(limit_ns)
    assert api.device_status() == api.LA_ERR_DEVICE_TIMEOUT
    assert api.device_status() == api.LA_OK           # reading it cleared it
    q, k, v = synth.qkv(300, 2, 128, seed=51, dtype=torch.bfloat16, device="cuda")
    o = api.prefill(q, k, v, beta=128)
    torch.cuda.synchronize()
    assert api.device_status() == api.LA_OK
    ref, _ = oracle.recurrent(q, k, v)
    assert oracle.max_rel_l2_per_head(o, ref) <= 2e-2
