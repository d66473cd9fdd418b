"""The paired prefill kernel's barrier protocol, checked on the CPU by its executable model
(``pair_protocol.py``): random schedules of the producers, the two MMA issuers and the
epilogue warps of both CTAs, with TMA landings, MMA completions, commit arrivals and
remote arrivals in random order.

Three things are checked:
  * the kernel's protocol is clean (no parity-alias, data or ordering violation, no
    deadlock) for every block count shape (empty, one block, partial last block, initial
    state, RMSNorm) and for every ring depth the kernel's static_assert accepts;
  * ring depths that assert rejects do fail in the model;
  * each planted protocol mistake (one wait taken out, a slot released by the wrong
    product, the output loaded after the wrong product) is caught.
"""
import itertools

import pytest

from pair_protocol import NDK, NF, PairModel, ProtocolError

SEEDS = 8


@pytest.mark.parametrize("nb", [0, 1, 2, 3, 5, 8])
@pytest.mark.parametrize("tail", [False, True], ids=["full", "tail"])
@pytest.mark.parametrize("init", [False, True], ids=["zero", "init"])
@pytest.mark.parametrize("rms", [False, True], ids=["plain", "rms"])
def test_default_rings(nb, tail, init, rms):
    for seed in range(SEEDS):
        PairModel(nb, tail=tail, init=init, rms=rms).run(seed)


def _depths(hi=4):
    return itertools.product(range(1, hi + 1), range(1, hi + 1), range(1, hi), range(1, hi + 1),
                             range(1, hi + 1))


def test_every_accepted_ring_depth():
    accepted = [d for d in _depths() if PairModel.compiles(*d)]
    assert (2, 2, 2, 4, 1) in accepted            # the kernel's depths
    for i, (nq, nks, nkd, nv, npb) in enumerate(accepted):
        for nb, seed in ((3, i), (7, i + 1)):
            PairModel(nb, tail=bool(seed & 1), init=bool(seed & 2), rms=bool(seed & 4), nq=nq,
                      nks=nks, nkd=nkd, nv=nv, npb=npb).run(seed)


def _first_violation(seeds=300, **kw):
    for seed in range(seeds):
        try:
            PairModel(**kw).run(seed)
        except ProtocolError as e:
            return str(e)
    return None


@pytest.mark.parametrize("depths,barrier", [
    (dict(nkd=NDK + 1), "dkv_done"),      # key-dim slots tested on a 2-deep dkv_done ring
    (dict(nq=NF + 1, npb=2), "f1_done"),  # query slots tested on the f1_done ring
    (dict(nks=NF + 1), "f1_done"),        # key-row slots tested on the f1_done ring
    (dict(nv=1), "full_v"),               # group KV's tail wait meets an open previous phase
])
def test_rejected_ring_depths_do_fail(depths, barrier):
    """A ring deeper than the done-barrier ring its slots are released on: the producer's
    test of a slot can meet a barrier already lapped by the block one ring further on (for
    the query ring the model reaches that schedule with two P buffers; with one, group P's
    wait for the previous P V holds F1 back far enough, but the bound does not rely on it).  And
    a one-slot value ring: group KV's wait for the partial last block's value tile starts
    while the slot's previous phase is still open."""
    with pytest.raises(ValueError):
        PairModel(6, **depths)
    msg = _first_violation(nb=8, tail=True, static_checks=False, **depths)
    assert msg is not None and (barrier in msg or "deadlock" in msg), (depths, msg)


# mutation -> (shape, words of which the first violation must name one: the mistake's symptoms)
MUTANTS = {
    # the dKV issuer overwrites a dKV accumulator before group KV loaded it
    "no_dkv_free_wait": (dict(nb=6), ("tmDKV",)),
    # the F1 issuer overwrites an [S | O] region before groups P and O loaded it
    "no_f1_free_wait": (dict(nb=7), ("tmS", "tmO", "f1_free")),
    # group P stores P_j before P_{j-1} V has completed (one P buffer: with two, F1_j's
    # completion, which group P waits for, already implies P_{j-2} V's, as one thread issues
    # both in that order)
    "no_o_done_wait_p": (dict(nb=5, npb=1), ("P0.", "P1.", "p_ready")),
    # dKV reads the partial last block before group KV zeroed its value rows (and, in
    # CTA 1, before its tile landed: only the zeroing implies that)
    "no_tail_zeroed_wait": (dict(nb=3, tail=True), ("zeroed", "V")),
    # group KV writes the next snapshot into a key-row slot that F1 still reads
    "no_snap_slot_wait": (dict(nb=6), ("KS", "snap")),
    # value slots released when dKV completes, though P V still reads them
    "v_release_on_dkv": (dict(nb=6), ("V", "full_v", "dkv_done")),
    # group O frees the value slot before it has seen P V complete
    "v_free_early": (dict(nb=7), ("V", "v_free", "full_v")),
    # one RMSNorm partial-sum buffer: a fast warp overwrites it before its partner read it
    "ss_one_buffer": (dict(nb=6, rms=True), ("partial sum",)),
    # group O loads O_b once F1_b completes, before P_b V_b has added to it
    "o_after_f1": (dict(nb=4), ("tmO",)),
}


@pytest.mark.parametrize("mutation", sorted(MUTANTS))
def test_planted_mistakes_are_caught(mutation):
    kw, words = MUTANTS[mutation]
    msg = _first_violation(mutations=(mutation,), **kw)
    assert msg is not None, f"{mutation} not caught"
    assert any(w in msg for w in words), msg
