"""The paired prefill kernel's barrier protocol, checked on the CPU by its executable model
(``pair_protocol.py``): random schedules of the producer, the two MMA issuers and the
epilogue warps of both CTAs, with TMA landings, MMA completions, commit arrivals and
remote arrivals in random order.

Three things are checked:
  * the kernel's protocol is clean (no parity-alias, data or ordering violation, no
    deadlock) for every block count shape (empty, one block, partial last block, initial
    state, RMSNorm) and for every ring depth the kernel's static_asserts accept;
  * the ring depths those asserts reject do fail in the model, where they can;
  * each planted protocol mistake (one wait or barrier taken out or merged) is caught.
"""
import itertools

import pytest

from pair_protocol import PairModel, ProtocolError

SEEDS = 8


@pytest.mark.parametrize("nb", [0, 1, 2, 3, 5, 8])
@pytest.mark.parametrize("tail", [False, True], ids=["full", "tail"])
@pytest.mark.parametrize("init", [False, True], ids=["zero", "init"])
@pytest.mark.parametrize("rms", [False, True], ids=["plain", "rms"])
def test_default_rings(nb, tail, init, rms):
    for seed in range(SEEDS):
        PairModel(nb, tail=tail, init=init, rms=rms).run(seed)


def _depths():
    for sahead in (1, 2):
        for kk, qh, kv, pb in itertools.product(range(1, sahead + 2), range(1, 5), range(1, 5),
                                                range(1, 5)):
            yield kk, qh, kv, pb, sahead


def test_every_accepted_ring_depth():
    accepted = [d for d in _depths() if PairModel.compiles(*d)]
    assert (2, 4, 2, 1, 1) in accepted            # the kernel's default depths
    for i, (kk, qh, kv, pb, sahead) in enumerate(accepted):
        for nb, seed in ((3, i), (6, i + 1)):
            PairModel(nb, tail=True, init=bool(seed & 1), rms=bool(seed & 2), kk=kk, qh=qh, kv=kv,
                      pbufs=pb, sahead=sahead).run(seed)


def _first_violation(seeds=200, **kw):
    for seed in range(seeds):
        try:
            PairModel(**kw).run(seed)
        except ProtocolError as e:
            return str(e)
    return None


def test_rejected_ring_depths_do_fail():
    """Look-ahead 2 with one K/V slot and two or more P buffers: CTA 0's group P may start its
    wait on the partial last block's load while the slot's previous phase is still open.
    The check is conservative for a single query slot: then S_b cannot start before
    O_{b-1} has completed, which implies that load, and the model finds nothing."""
    rejected = [d for d in _depths() if not PairModel.compiles(*d)]
    assert rejected and all(d[4] == 2 and d[2] == 1 and d[3] >= 2 for d in rejected)
    for kk, qh, kv, pb, sahead in rejected:
        with pytest.raises(ValueError):
            PairModel(3, kk=kk, qh=qh, kv=kv, pbufs=pb, sahead=sahead)
        msg = _first_violation(nb=3, tail=True, kk=kk, qh=qh, kv=kv, pbufs=pb, sahead=sahead,
                               static_checks=False)
        if qh == 1:
            assert msg is None, (kk, qh, kv, pb, sahead, msg)
        else:
            assert msg is not None and "full_kv" in msg, (kk, qh, kv, pb, sahead)


# mutation -> (shape, words of which the first violation must name one: the mistake's symptoms)
MUTANTS = {
    # issuer B issues Q_b snap_b without waiting for the query tile to land
    "no_qh_wait_b": (dict(nb=4, init=True), ("QH",)),
    # issuer A overwrites a dKV accumulator before group O loaded it
    "no_dkv_free_wait": (dict(nb=5), ("tmDKV",)),
    # group P stores P_b before P_{b-1} V has completed
    "no_o_done_wait_p": (dict(nb=4), ("p_ready", "P0.", "P1.")),
    # two P buffers behind one p_ready barrier (phases alias)
    "single_p_ready": (dict(nb=5, pbufs=2), ("p_ready",)),
    # issuer A reads the partial last block before group P zeroed its value rows (and, in
    # CTA 1, before its tiles landed: only the zeroing implies that)
    "no_tail_zeroed_wait": (dict(nb=3, tail=True), ("zeroed", "KV")),
    # one snapshot buffer: snapshot b+1 overwrites snapshot b under Q_b snap_b, and the
    # buffer's one barrier aliases phases
    "one_snapshot": (dict(nb=5), ("SNAP", "snap_ready")),
    # query slots released when S_j completes, though Q_j snap_j still reads them (and the
    # 4-deep query ring then laps the 2-deep s_full ring)
    "qh_release_on_s_full": (dict(nb=5), ("full_qh", "QH", "s_full")),
}


@pytest.mark.parametrize("mutation", sorted(MUTANTS))
def test_planted_mistakes_are_caught(mutation):
    kw, words = MUTANTS[mutation]
    msg = _first_violation(mutations=(mutation,), **kw)
    assert msg is not None, f"{mutation} not caught"
    assert any(w in msg for w in words), msg
