"""The unpaired prefill kernel's barrier protocol (two MMA issuers, scores two blocks ahead),
checked on the CPU by its executable model (``tc_protocol.py``): random schedules of the
producer, both issuers and the epilogue warps of one CTA or of the two value-slice CTAs of a
cluster, with TMA landings, MMA completions, commit arrivals and remote arrivals in random
order.

Checked: the kernel's protocol is clean for every block count shape (empty, one block,
partial last block, initial state, RMSNorm; one CTA and a cluster pair) and for every stage
count the kernel accepts (and, the bound being for prefetch depth, for two stages); and each
planted protocol mistake is caught.
"""
import pytest

from pair_protocol import ProtocolError
from tc_protocol import TcModel

SEEDS = 8


@pytest.mark.parametrize("nb", [0, 1, 2, 3, 5, 8])
@pytest.mark.parametrize("tail", [False, True], ids=["full", "tail"])
@pytest.mark.parametrize("init", [False, True], ids=["zero", "init"])
@pytest.mark.parametrize("rms", [False, True], ids=["plain", "rms"])
@pytest.mark.parametrize("pair", [True, False], ids=["d128", "d64"])
def test_default_protocol(nb, tail, init, rms, pair):
    for seed in range(SEEDS):
        TcModel(nb, tail=tail, init=init, rms=rms, pair=pair).run(seed)


def test_every_accepted_stage_count():
    for nst in (3, 4, 5):
        assert TcModel.compiles(nst)
        for seed in range(6):
            TcModel(7, tail=bool(seed & 1), init=bool(seed & 2), rms=bool(seed & 4),
                    nst=nst).run(seed)


def _first_violation(seeds=300, **kw):
    for seed in range(seeds):
        try:
            TcModel(**kw).run(seed)
        except ProtocolError as e:
            return str(e)
    return None


def test_two_stages_still_safe():
    """The kernel asserts at least three stages so that block b + 2 can load while blocks b
    and b + 1 are in use; that bound is for prefetch depth, not for correctness: with two
    stages the load of block b + 2 waits for block b's release and the protocol stays clean."""
    assert not TcModel.compiles(2)
    with pytest.raises(ValueError):
        TcModel(5, nst=2)
    assert _first_violation(seeds=60, nb=6, nst=2, tail=True, static_checks=False) is None


# mutation -> (shape, words of which the first violation must name one)
MUTANTS = {
    # issuer A issues dKV_b and S_{b+2} without waiting for P_b V_b: dKV_b may read the value
    # tile before issuer B zeroed its tail rows, S_{b+2} may overwrite P_b under P V, and
    # group KV may write snapshot b + 1 over snapshot b - 1 before Q_{b-1} snap_{b-1} read it
    "a_no_pv_done_wait": (dict(nb=6, tail=True), ("another issuer", "tmS", "zeroed", "snap")),
    # issuer B adds the inter-block term before P V, which initialises the accumulator
    "b_qkv_first": (dict(nb=5, init=True), ("tmO", "another issuer")),
    # issuer B's P V overwrites O before group O loaded it
    "b_no_o_free_wait": (dict(nb=7), ("tmO",)),
    # only issuer A releases a stage: the producer reloads it under issuer B's products
    "single_empty_arrival": (dict(nb=9, init=True), ("TMA", "Q", "V")),
    # one P-ready barrier instead of a ring of two: with the scores two blocks ahead, group P
    # can complete the next phase before issuer B waits on this one
    "p_ready_single": (dict(nb=8), ("p_ready",)),
    # the value rows past the sequence end zeroed after P V read them
    "zero_after_pv": (dict(nb=3, tail=True), ("zeroed",)),
    # one snapshot buffer
    "snap_one_buffer": (dict(nb=7, init=True), ("snap",)),
    # group O reads the partner's partial sum without waiting for it
    "rms_no_wait": (dict(nb=4, rms=True), ("partial sum",)),
}


@pytest.mark.parametrize("mutation", sorted(MUTANTS))
def test_planted_mistakes_are_caught(mutation):
    kw, words = MUTANTS[mutation]
    msg = _first_violation(mutations=(mutation,), **kw)
    assert msg is not None, f"{mutation} not caught"
    assert any(w in msg for w in words), msg
