"""Executable model of the synchronisation in ``prefill_pair_kernel``
(long_context_04_b200/csrc/prefill_pair.cuh), checked under random schedules.

The model has no arithmetic: it tracks which block's data each shared-memory slot, P
buffer, state snapshot and TMEM accumulator holds, and the mbarriers that order them.
Each agent is a generator that mirrors one role of the kernel, one step per wait,
arrival, TMA issue, store or MMA issue, in the kernel's order:

    producer0, producer1   warp 0 of CTA 0 / CTA 1 (the four TMA rings)
    A                      CTA 0's issuer of F1 = Q [K ; snap]^T and P V
    D                      CTA 0's issuer of dKV^T = V^T K
    P<c>.<w>, KV<c>.<w>, O<c>.<w>
                           warp w (0..3) of group P / KV / O in CTA c

Asynchronous work is a pool of pending events that fire in random order, interleaved at
random with the agents' steps: each TMA tile landing (its transaction bytes on its
barrier), each MMA's completion (in issue order per issuing thread, the two threads
independent), each commit's arrival on each CTA's barrier, and each arrival that a
CTA 1 thread sends to a CTA 0 barrier.  Every schedule draws a speed for each agent and
each kind of event, so that some schedules starve one role for long stretches.

Every schedule is checked for:
  * the parity-wait rules: a wait (or the producer's non-blocking test) on phase n of a
    barrier starts only once phase n - 1 has completed, and phase n + 1 does not
    complete before the wait has returned (otherwise the parity bit would alias);
  * every arrival and every transaction-byte count landing in the phase its sender means;
  * an MMA issued only on operands that hold the intended block's data, fully landed,
    with the value rows past the sequence end zeroed for the partial last block, and
    never overwriting an accumulator that a warp still has to load;
  * the O accumulator loaded only after both of its products (F1, then P V) completed;
  * a TMEM load only of the intended block's accumulator, with all its MMAs complete;
  * no shared-memory write (TMA or store) to a buffer that an in-flight MMA reads;
  * the RMSNorm partial sums read only after their writer stored them, and never
    overwritten before the partner lane read them (the four warps of group O meet at a
    named barrier once per block, modelled as a barrier of four arrivals per block);
  * no deadlock, and nothing in flight once every agent has finished.

Not modelled: the timeout / abort paths, TMEM allocation, the numerical content, the
output's TMA store (its staging buffer is read by no MMA).
"""
from __future__ import annotations

import random

BETA = 128
HBOX = 64 * 128          # one 64-row x 128-byte TMA tile
FBOX = 128 * 128         # one 128-row x 128-byte TMA tile
NF = 3                   # F1 TMEM regions [S | O] (and the f1_done / o_done / f1_free rings)
NDK = 2                  # dKV TMEM buffers (and the dkv_done / dkv_free rings)
WARPS = 4                # warps per epilogue group


class ProtocolError(AssertionError):
    pass


class Barrier:
    """An mbarrier: expected arrivals, the pending arrivals and transaction bytes of the
    current phase, and the number of completed phases."""

    def __init__(self, name: str, count: int):
        self.name, self.count = name, count
        self.pending, self.tx, self.done = count, 0, 0

    def _phase(self, phase, who, what):
        if self.done != phase:
            raise ProtocolError(f"{who}: {what} meant for phase {phase} of {self.name} "
                                f"lands in phase {self.done}")

    def _maybe_complete(self):
        if self.pending == 0 and self.tx == 0:
            self.done += 1
            self.pending = self.count

    def arrive(self, phase, who, expect_tx=0):
        self._phase(phase, who, "an arrival")
        if self.pending == 0:
            raise ProtocolError(f"{who}: one arrival too many in phase {phase} of {self.name}")
        self.pending -= 1
        self.tx += expect_tx
        self._maybe_complete()

    def complete_tx(self, phase, nbytes, who):
        self._phase(phase, who, f"{nbytes} transaction bytes")
        self.tx -= nbytes
        self._maybe_complete()


class Buf:
    """A shared-memory tile (or part of one) or a TMEM accumulator."""

    def __init__(self, name: str, consumers=()):
        self.name = name
        self.tag = None                  # the data it holds, e.g. ("q", 3)
        self.writing = 0                 # writes in flight (TMA tiles, MMAs)
        self.reading = 0                 # MMA reads in flight
        self.consumer_ids = frozenset(consumers)
        self.consumers = set()           # TMEM: warps that must still load the current data
        self.zeroed = set()              # group-P warps that zeroed their rows of the tail


class _Ev:
    __slots__ = ("kind", "args")

    def __init__(self, kind, *args):
        self.kind, self.args = kind, args


STEP = ("step",)


class PairModel:
    """One CTA pair working on one (sequence, head) of ``nb`` blocks.

    tail: the last block is partial.  init: the kernel starts from an initial state.
    nq, nks, nkd, nv, npb: ring depths (PairCfg::NQ, NKS, NKD, NV, NPB).  ``mutations``
    names deliberate protocol mistakes, for checking that the model catches them.
    """

    def __init__(self, nb, tail=False, init=False, rms=False, nq=2, nks=2, nkd=2, nv=4, npb=1,
                 mutations=(), static_checks=True):
        self.nb, self.tail, self.init, self.rms = nb, tail and nb > 0, init, rms
        self.NQ, self.NKS, self.NKD, self.NV, self.NPB = nq, nks, nkd, nv, npb
        self.mut = frozenset(mutations)
        if static_checks and not self.compiles(nq, nks, nkd, nv, npb):
            raise ValueError("ring depths rejected by the kernel's static_assert")
        self.bars = [self._cta_bars(c) for c in (0, 1)]
        P_ids = [{("P", c, w) for w in range(WARPS)} for c in (0, 1)]
        KV_ids = [{("KV", c, w) for w in range(WARPS)} for c in (0, 1)]
        O_ids = [{("O", c, w) for w in range(WARPS)} for c in (0, 1)]
        self.Q = [[[Buf(f"Q{s}.{h}@{c}") for h in (0, 1)] for s in range(nq)] for c in (0, 1)]
        # key-row slot: the TMA'd key rows (per dim half) and the snapshot rows (per KV warp)
        self.KSK = [[[Buf(f"KS{s}.K{h}@{c}") for h in (0, 1)] for s in range(nks)] for c in (0, 1)]
        self.KSS = [[[Buf(f"KS{s}.snap{w}@{c}") for w in range(WARPS)] for s in range(nks)]
                    for c in (0, 1)]
        self.KD = [[Buf(f"KD{s}@{c}") for s in range(nkd)] for c in (0, 1)]
        self.V = [[Buf(f"V{s}@{c}") for s in range(nv)] for c in (0, 1)]
        self.P = [[[Buf(f"P{s}.{w}@{c}") for w in range(WARPS)] for s in range(npb)] for c in (0, 1)]
        self.S = [[Buf(f"tmS{f}@{c}", P_ids[c]) for f in range(NF)] for c in (0, 1)]
        self.O = [[Buf(f"tmO{f}@{c}", O_ids[c]) for f in range(NF)] for c in (0, 1)]
        self.DKV = [[Buf(f"tmDKV{s}@{c}", KV_ids[c]) for s in range(NDK)] for c in (0, 1)]
        self.ssx = [[[None] * WARPS for _ in range(2)] for _ in (0, 1)]
        self.inflight: list[_Ev] = []
        self.fifo = {"A": [], "D": []}
        self.issued = {"A": 0, "D": 0}
        self.completed = {"A": 0, "D": 0}
        self.commits: list[_Ev] = []

    @staticmethod
    def compiles(nq, nks, nkd, nv, npb):
        """The kernel's static_asserts on the ring depths (PairCfg in prefill_pair.cuh): a
        ring's slot of block x is tested free on the done barrier of block x, which must not
        have been lapped when the producer tests it (the value ring has a release ring of
        its own, v_free, as deep as itself); and group KV's wait for the value tile of a
        partial last block (one block before its dKV) is exact only if the slot's previous
        load fed a dKV that group has seen complete."""
        return nq <= NF and nks <= NF and nkd <= NDK and npb <= NF and nv >= 2

    # ------------------------------------------------------------------ set-up
    def _cta_bars(self, c):
        G = 2 * WARPS            # arrivals from one epilogue group in each of the two CTAs

        def ring(name, n, count):
            return [Barrier(f"{name}[{i}]@{c}", count) for i in range(n)]
        return {
            "full_q": ring("full_q", self.NQ, 1),
            "full_ks": ring("full_ks", self.NKS, 1),
            "full_kd": ring("full_kd", self.NKD, 1),
            "full_v": ring("full_v", self.NV, 1),
            "tail_v": Barrier(f"tail_v@{c}", 1),
            "tail_zeroed": Barrier(f"tail_zeroed@{c}", G),
            "f1_done": ring("f1_done", NF, 1),
            "dkv_done": ring("dkv_done", NDK, 1),
            "o_done": ring("o_done", NF, 1),
            "f1_free": ring("f1_free", NF, 2 * G),
            "dkv_free": ring("dkv_free", NDK, G),
            "p_ready": ring("p_ready", self.NPB, G),
            "snap_ready": ring("snap_ready", self.NKS, G),
            "drain": Barrier(f"drain@{c}", 2),
            "v_free": ring("v_free", self.NV, 1),
            "ss_sync": Barrier(f"ss_sync@{c}", WARPS),
        }

    # ------------------------------------------------------------------ primitives
    def _check_wait(self, who, bar, n, start):
        c = bar.done
        if start and c < n:
            raise ProtocolError(f"{who}: waits on phase {n} of {bar.name} before phase {n - 1} "
                                f"completed ({c} phases done)")
        if c > n + 1:
            raise ProtocolError(f"{who}: phase {n + 1} of {bar.name} completed before the wait "
                                f"on phase {n} returned")

    def arrive(self, who, c, bar, phase, expect_tx=0):
        """Arrival on a CTA 0 barrier: immediate from CTA 0, in flight from CTA 1."""
        if c == 0:
            bar.arrive(phase, who, expect_tx)
        else:
            self.inflight.append(_Ev("arrive", bar, phase, who))

    def tma(self, who, buf, tag, bar, phase, nbytes):
        if buf.reading or buf.writing:
            raise ProtocolError(f"{who}: TMA load of {tag} into {buf.name} while "
                                f"{'an MMA reads' if buf.reading else 'a write lands in'} it")
        buf.tag, buf.writing, buf.zeroed = tag, 1, set()
        self.inflight.append(_Ev("tma", buf, bar, phase, nbytes, who))

    def store(self, who, buf, tag):
        if buf.reading or buf.writing:
            raise ProtocolError(f"{who}: stores {tag} into {buf.name} while an MMA reads {buf.tag}")
        buf.tag = tag

    def zero_tail(self, who, w, buf, tag):
        if buf.tag != tag or buf.writing:
            raise ProtocolError(f"{who}: zeroes rows of {buf.name} before {tag} has landed")
        if buf.reading:
            raise ProtocolError(f"{who}: zeroes rows of {buf.name} while an MMA reads it")
        buf.zeroed.add(w)

    def mma(self, issuer, what, reads, writes, zeroed=()):
        """writes: (buf, tag, acc, new_tag): an accumulating write expects ``tag`` in the
        buffer and leaves ``new_tag`` (the next stage of the same accumulator)."""
        for buf, tag in reads:
            if buf.tag != tag or buf.writing:
                state = " (still being written)" if buf.writing else ""
                raise ProtocolError(f"{issuer}: {what} reads {buf.name} holding {buf.tag}{state}, "
                                    f"wants {tag}")
        for buf in zeroed:
            if buf.zeroed != set(range(WARPS)):
                raise ProtocolError(f"{issuer}: {what} reads {buf.name} before the rows past the "
                                    f"sequence end were zeroed")
        for buf, tag, acc, new_tag in writes:
            if acc:
                if buf.tag != tag:
                    raise ProtocolError(f"{issuer}: {what} accumulates onto {buf.name} holding "
                                        f"{buf.tag}, wants {tag}")
                buf.tag = new_tag
            else:
                if buf.consumers:
                    raise ProtocolError(f"{issuer}: {what} overwrites {buf.name} ({buf.tag}) before "
                                        f"{sorted(buf.consumers)} loaded it")
                buf.tag, buf.consumers = new_tag, set(buf.consumer_ids)
            buf.writing += 1
        for buf, _ in reads:
            buf.reading += 1
        self.fifo[issuer].append((reads, [(b, t, a) for b, t, a, _ in writes]))
        self.issued[issuer] += 1

    def commit(self, issuer, targets):
        for bar, phase in targets:
            self.commits.append(_Ev("commit", issuer, self.issued[issuer], bar, phase))

    def tmem_ld(self, who, wid, buf, tag):
        if buf.tag != tag or buf.writing:
            state = " (MMA in flight)" if buf.writing else ""
            raise ProtocolError(f"{who}: loads {buf.name} holding {buf.tag}{state}, wants {tag}")
        if wid not in buf.consumers:
            raise ProtocolError(f"{who}: loads {buf.name} ({tag}) twice")
        buf.consumers.discard(wid)

    def _both(self, name, i, phase):
        return [(self.bars[c][name][i], phase) for c in (0, 1)]

    # ------------------------------------------------------------------ agents
    def producer(self, c):
        who = f"producer{c}"
        B0, Bc = self.bars[0], self.bars[c]
        nb, NQ, NKS, NKD, NV = self.nb, self.NQ, self.NKS, self.NKD, self.NV
        jq = js = jd = jv = 0
        # value slots are released once group O has seen P V complete (v_free); the
        # mutation releases them when dKV completes
        if "v_release_on_dkv" in self.mut:
            v_ring, v_n = Bc["dkv_done"], NDK
        else:
            v_ring, v_n = Bc["v_free"], NV

        def freed(ring, nring, j, depth):
            x = j - depth
            if x < 0:
                return True
            bar, n = ring[x % nring], x // nring
            self._check_wait(who, bar, n, start=True)
            if bar.done > n + 1:   # the parity test would read the lapped phase
                raise ProtocolError(f"{who}: tests phase {n} of {bar.name} after phase {n + 1} "
                                    f"completed")
            return bar.done >= n + 1

        def cond(ring, nring, j, depth):
            x = j - depth
            return [] if x < 0 else [(ring[x % nring], x // nring)]

        while jq < nb or js < nb or jd < nb or jv < nb:
            progressed = False
            if jd < nb and freed(Bc["dkv_done"], NDK, jd, NKD):
                slot, ph, bar = jd % NKD, jd // NKD, B0["full_kd"][jd % NKD]
                if c == 0:
                    self.arrive(who, 0, bar, ph, expect_tx=2 * FBOX)
                self.tma(who, self.KD[c][slot], ("kd", jd), bar, ph, FBOX)
                jd += 1
                progressed = True
            if jv < nb and freed(v_ring, v_n, jv, NV):
                slot, ph = jv % NV, jv // NV
                last_partial = self.tail and jv == nb - 1
                if c == 0:
                    bar = B0["full_v"][slot]
                    self.arrive(who, 0, bar, ph, expect_tx=(1 if last_partial else 2) * FBOX)
                elif last_partial:
                    bar, ph = Bc["tail_v"], 0
                    bar.arrive(0, who, FBOX)
                else:
                    bar = B0["full_v"][slot]
                self.tma(who, self.V[c][slot], ("v", jv), bar, ph, FBOX)
                jv += 1
                progressed = True
            if js < nb and freed(Bc["f1_done"], NF, js, NKS):
                slot, ph, bar = js % NKS, js // NKS, B0["full_ks"][js % NKS]
                if c == 0:
                    self.arrive(who, 0, bar, ph, expect_tx=4 * HBOX)
                for h in (0, 1):
                    self.tma(who, self.KSK[c][slot][h], ("k", js), bar, ph, HBOX)
                js += 1
                progressed = True
            if jq < nb and freed(Bc["f1_done"], NF, jq, NQ):
                slot, ph, bar = jq % NQ, jq // NQ, B0["full_q"][jq % NQ]
                if c == 0:
                    self.arrive(who, 0, bar, ph, expect_tx=4 * HBOX)
                for h in (0, 1):
                    self.tma(who, self.Q[c][slot][h], ("q", jq), bar, ph, HBOX)
                jq += 1
                progressed = True
            if progressed:
                yield STEP
            else:
                conds = []
                if jd < nb:
                    conds.append(cond(Bc["dkv_done"], NDK, jd, NKD))
                if jv < nb:
                    conds.append(cond(v_ring, v_n, jv, NV))
                if js < nb:
                    conds.append(cond(Bc["f1_done"], NF, js, NKS))
                if jq < nb:
                    conds.append(cond(Bc["f1_done"], NF, jq, NQ))
                yield ("poll", conds)
        # drain: the last loads of each ring have landed before the CTA exits
        if c == 0:
            for ring, n, j in (("full_q", NQ, jq), ("full_ks", NKS, js), ("full_kd", NKD, jd),
                               ("full_v", NV, jv)):
                for x in range(max(0, j - n), j):
                    yield ("wait", B0[ring][x % n], x // n)
        elif self.tail and jv == nb:
            yield ("wait", Bc["tail_v"], 0)

    def issuer_d(self):
        B0 = self.bars[0]
        nb = self.nb
        for j in range(nb):
            last_tail = self.tail and j == nb - 1
            yield ("wait", B0["full_kd"][j % self.NKD], j // self.NKD)
            yield ("wait", B0["full_v"][j % self.NV], j // self.NV)
            if j >= NDK and "no_dkv_free_wait" not in self.mut:
                yield ("wait", B0["dkv_free"][j % NDK], (j - NDK) // NDK)
            if last_tail and "no_tail_zeroed_wait" not in self.mut:
                yield ("wait", B0["tail_zeroed"], 0)
            reads = [(self.KD[c][j % self.NKD], ("kd", j)) for c in (0, 1)]
            reads += [(self.V[c][j % self.NV], ("v", j)) for c in (0, 1)]
            zeroed = [self.V[c][j % self.NV] for c in (0, 1)] if last_tail else []
            self.mma("D", f"dKV_{j}", reads,
                     [(self.DKV[c][j % NDK], None, False, ("dkv", j)) for c in (0, 1)], zeroed)
            self.commit("D", self._both("dkv_done", j % NDK, j // NDK))
            yield STEP
        self.commit("D", [(B0["drain"], 0)])
        yield ("wait", B0["drain"], 0)

    def issuer_a(self):
        B0 = self.bars[0]
        nb, NKS = self.nb, self.NKS

        def f1(j):   # [S_j | O_j] = Q_j [K_j ; snap_j]^T
            yield ("wait", B0["full_q"][j % self.NQ], j // self.NQ)
            yield ("wait", B0["full_ks"][j % NKS], j // NKS)
            yield ("wait", B0["snap_ready"][j % NKS], j // NKS)
            if j >= NF and "no_f1_free_wait" not in self.mut:
                yield ("wait", B0["f1_free"][j % NF], (j - NF) // NF)
            reads = [(self.Q[c][j % self.NQ][h], ("q", j)) for c in (0, 1) for h in (0, 1)]
            reads += [(self.KSK[c][j % NKS][h], ("k", j)) for c in (0, 1) for h in (0, 1)]
            reads += [(self.KSS[c][j % NKS][w], ("snap", j)) for c in (0, 1) for w in range(WARPS)]
            writes = [(self.S[c][j % NF], None, False, ("S", j)) for c in (0, 1)]
            writes += [(self.O[c][j % NF], None, False, ("oi", j)) for c in (0, 1)]
            self.mma("A", f"F1_{j}", reads, writes)
            self.commit("A", self._both("f1_done", j % NF, j // NF))
            yield STEP

        def pv(j):   # O_j += P_j V_j
            yield ("wait", B0["p_ready"][j % self.NPB], j // self.NPB)
            yield ("wait", B0["full_v"][j % self.NV], j // self.NV)
            reads = [(self.P[c][j % self.NPB][w], ("p", j)) for c in (0, 1) for w in range(WARPS)]
            reads += [(self.V[c][j % self.NV], ("v", j)) for c in (0, 1)]
            self.mma("A", f"PV_{j}", reads, [(self.O[c][j % NF], ("oi", j), True, ("o", j)) for c in (0, 1)])
            self.commit("A", self._both("o_done", j % NF, j // NF))
            yield STEP

        if nb > 0:
            yield from f1(0)
        for b in range(nb):
            if b + 1 < nb:
                yield from f1(b + 1)
            yield from pv(b)
        self.commit("A", [(B0["drain"], 0)])
        yield ("wait", B0["drain"], 0)

    def group_p(self, c, w):
        who = f"P{c}.{w}"
        B0, Bc = self.bars[0], self.bars[c]
        for j in range(self.nb):
            yield ("wait", Bc["f1_done"][j % NF], j // NF)
            self.tmem_ld(who, ("P", c, w), self.S[c][j % NF], ("S", j))
            self.arrive(who, c, B0["f1_free"][j % NF], j // NF)
            yield STEP
            pb = j - self.NPB
            if pb >= 0 and "no_o_done_wait_p" not in self.mut:
                yield ("wait", Bc["o_done"][pb % NF], pb // NF)
            self.store(who, self.P[c][j % self.NPB][w], ("p", j))
            self.arrive(who, c, B0["p_ready"][j % self.NPB], j // self.NPB)
            yield STEP

    def group_kv(self, c, w):
        who = f"KV{c}.{w}"
        B0, Bc = self.bars[0], self.bars[c]
        nb, NKS = self.nb, self.NKS

        def write_snap(u):
            self.store(who, self.KSS[c][u % NKS][w], ("snap", u))
            self.arrive(who, c, B0["snap_ready"][u % NKS], u // NKS)

        def zero_tail():
            b = nb - 1
            if c == 0:
                yield ("wait", B0["full_v"][b % self.NV], b // self.NV)
            else:
                yield ("wait", Bc["tail_v"], 0)
            self.zero_tail(who, w, self.V[c][b % self.NV], ("v", b))
            self.arrive(who, c, B0["tail_zeroed"], 0)
            yield STEP

        if nb > 0:
            write_snap(0)
            yield STEP
            if self.tail and nb == 1:
                yield from zero_tail()
        for b in range(nb):
            if self.tail and nb >= 2 and b == nb - 2:
                yield from zero_tail()
            yield ("wait", Bc["dkv_done"][b % NDK], b // NDK)
            self.tmem_ld(who, ("KV", c, w), self.DKV[c][b % NDK], ("dkv", b))
            self.arrive(who, c, B0["dkv_free"][b % NDK], b // NDK)
            yield STEP
            if b + 1 < nb:
                x = b + 1 - NKS
                if x >= 0 and "no_snap_slot_wait" not in self.mut:
                    yield ("wait", Bc["f1_done"][x % NF], x // NF)
                write_snap(b + 1)
                yield STEP

    def group_o(self, c, w):
        who = f"O{c}.{w}"
        B0, Bc = self.bars[0], self.bars[c]
        for b in range(self.nb):
            if "v_free_early" in self.mut and w == 0:   # frees the value slot before P V is done
                Bc["v_free"][b % self.NV].arrive(b // self.NV, who)
            if "o_after_f1" in self.mut:      # waits for F1_b instead of P_b V_b
                yield ("wait", Bc["f1_done"][b % NF], b // NF)
            else:
                yield ("wait", Bc["o_done"][b % NF], b // NF)
            if w == 0 and "v_free_early" not in self.mut:   # P V of block b read its value slot
                Bc["v_free"][b % self.NV].arrive(b // self.NV, who)
            self.tmem_ld(who, ("O", c, w), self.O[c][b % NF], ("o", b))
            self.arrive(who, c, B0["f1_free"][b % NF], b // NF)
            yield STEP
            if self.rms:   # exchange of the row's partial sum of squares with warp w ^ 2
                slot = 0 if "ss_one_buffer" in self.mut else b & 1
                prev = self.ssx[c][slot][w]
                if prev is not None and not prev[1]:
                    raise ProtocolError(f"{who}: overwrites its partial sum of block {prev[0]} "
                                        f"before warp {w ^ 2} read it")
                self.ssx[c][slot][w] = [b, False]
                Bc["ss_sync"].arrive(b, who)          # the group's named barrier, block b
                yield ("wait", Bc["ss_sync"], b)
                other = self.ssx[c][slot][w ^ 2]
                if other is None or other[0] != b:
                    raise ProtocolError(f"{who}: reads the partial sum of warp {w ^ 2} for block "
                                        f"{None if other is None else other[0]}, wants {b}")
                other[1] = True
                yield STEP

    def agents(self):
        """name -> generator, one per role of the kernel."""
        agents = {"producer0": self.producer(0), "producer1": self.producer(1),
                  "A": self.issuer_a(), "D": self.issuer_d()}
        for c in (0, 1):
            for w in range(WARPS):
                agents[f"P{c}.{w}"] = self.group_p(c, w)
                agents[f"KV{c}.{w}"] = self.group_kv(c, w)
                agents[f"O{c}.{w}"] = self.group_o(c, w)
        return agents

    # ------------------------------------------------------------------ scheduler
    def _events(self):
        evs = list(self.inflight)
        for who in ("A", "D"):
            if self.fifo[who]:
                evs.append(_Ev("mma", who))
        evs += [e for e in self.commits if self.completed[e.args[0]] >= e.args[1]]
        return evs

    def _fire(self, ev):
        if ev.kind == "tma":
            buf, bar, phase, nbytes, who = ev.args
            self.inflight.remove(ev)
            buf.writing -= 1
            bar.complete_tx(phase, nbytes, f"{who} (TMA into {buf.name})")
        elif ev.kind == "arrive":
            bar, phase, who = ev.args
            self.inflight.remove(ev)
            bar.arrive(phase, who)
        elif ev.kind == "mma":
            who = ev.args[0]
            reads, writes = self.fifo[who].pop(0)
            for buf, _ in reads:
                buf.reading -= 1
            for buf, _, _ in writes:
                buf.writing -= 1
            self.completed[who] += 1
        else:
            who, _, bar, phase = ev.args
            self.commits.remove(ev)
            bar.arrive(phase, f"{who} commit")

    @staticmethod
    def _runnable(st):
        if st[0] == "ready":
            return True
        if st[0] == "wait":
            return st[1].done >= st[2] + 1
        if st[0] == "poll":
            return any(all(bar.done >= n + 1 for bar, n in conj) for conj in st[1])
        return False

    def run(self, seed: int, max_steps: int = 1_000_000):
        """Run every agent to completion under one random schedule; raise ProtocolError on
        the first violation."""
        rng = random.Random(seed)
        bias = rng.uniform(0.05, 0.95)      # how eagerly asynchronous work completes
        agents = self.agents()
        state = {name: ("ready",) for name in agents}
        # Each agent and each kind of asynchronous event gets a speed for this schedule, so
        # that some schedules starve one role (a slow warp, late TMA tiles, a slow issuer).
        speeds = (0.02, 0.2, 1.0, 1.0, 5.0)
        w_agent = {name: rng.choice(speeds) for name in agents}
        w_event = {kind: rng.choice(speeds) for kind in ("tma", "arrive", "mma", "commit")}
        for _ in range(max_steps):
            live = [n for n, st in state.items() if st[0] != "done"]
            runnable = [n for n in live if self._runnable(state[n])]
            events = self._events()
            if not runnable and not events:
                if not live:
                    break
                raise ProtocolError("deadlock: " + "; ".join(
                    f"{n} waits on phase {state[n][2]} of {state[n][1].name}" if state[n][0] == "wait"
                    else f"{n} polls" for n in live))
            if events and (not runnable or rng.random() < bias):
                self._fire(rng.choices(events, weights=[w_event[e.kind] for e in events])[0])
            else:
                name = rng.choices(runnable, weights=[w_agent[n] for n in runnable])[0]
                try:
                    instr = next(agents[name])
                except StopIteration:
                    state[name] = ("done",)
                    continue
                if instr[0] == "wait":
                    self._check_wait(name, instr[1], instr[2], start=True)
                    state[name] = ("wait", instr[1], instr[2])
                elif instr[0] == "poll":
                    state[name] = ("poll", instr[1])
                else:
                    state[name] = ("ready",)
            for n, st in state.items():     # phase n + 1 must not complete under a pending wait
                if st[0] == "wait":
                    self._check_wait(n, st[1], st[2], start=False)
                elif st[0] == "poll":
                    for conj in st[1]:
                        for bar, k in conj:
                            self._check_wait(n, bar, k, start=False)
        else:
            raise ProtocolError("no end after max_steps")
        if self.inflight or self.fifo["A"] or self.fifo["D"] or self.commits:
            raise ProtocolError("work still in flight after every agent finished")
