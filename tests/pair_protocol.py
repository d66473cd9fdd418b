"""Executable model of the synchronisation in ``prefill_pair_kernel``
(long_context_04_b200/csrc/prefill_pair.cuh), checked under random schedules.

The model has no arithmetic: it tracks which block's data each shared-memory slot, P
buffer, state snapshot and TMEM accumulator holds, and the mbarriers that order them.
Each agent is a generator that mirrors one role of the kernel, one step per wait,
arrival, TMA issue, store or MMA issue, in the kernel's order:

    producer0, producer1   warp 0 of CTA 0 / CTA 1 (the three TMA rings)
    A, B                   the two MMA-issuing warps of CTA 0
    P<c>.<w>, O<c>.<w>     warp w (0..3) of group P / group O in CTA c

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
  * a TMEM load only of the intended block's accumulator, with all its MMAs complete;
  * no shared-memory write (TMA or store) to a buffer that an in-flight MMA reads;
  * the RMSNorm partial sums read only after their writer stored them, and never
    overwritten before the partner lane read them;
  * no deadlock, and nothing in flight once every agent has finished.

Not modelled: the timeout / abort paths, TMEM allocation, the numerical content.
"""
from __future__ import annotations

import random

BETA = 128
HBOX = 64 * 128          # one 64-row x 128-byte TMA tile
FBOX = 128 * 128         # one 128-row x 128-byte TMA tile
KK_BYTES = QH_BYTES = 2 * HBOX
KV_BYTES = 2 * FBOX
NDONE = 4                # ring of block-completion barriers (kv_done, o_done)
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
    kk, qh, kv, pbufs, sahead: ring depths (LA_PAIR_KK_DEPTH, LA_PAIR_QH_DEPTH,
    LA_PAIR_KV_DEPTH, LA_PAIR_P_BUFS, LA_PAIR_S_AHEAD).  ``mutations`` names deliberate
    protocol mistakes, for checking that the model catches them.
    """

    def __init__(self, nb, tail=False, init=False, rms=False, kk=2, qh=4, kv=2, pbufs=1,
                 sahead=1, mutations=(), static_checks=True):
        self.nb, self.tail, self.init, self.rms = nb, tail and nb > 0, init, rms
        self.NKK, self.NQH, self.NKV, self.NPB = kk, qh, kv, pbufs
        self.SAHEAD, self.NS = sahead, sahead + 1
        self.mut = frozenset(mutations)
        if static_checks and not self.compiles(kk, qh, kv, pbufs, sahead):
            raise ValueError("ring depths rejected by the kernel's static_asserts")
        self.u0 = 0 if init else 1
        self.bars = [self._cta_bars(c) for c in (0, 1)]
        P_ids = [{("P", c, w) for w in range(WARPS)} for c in (0, 1)]
        O_ids = [{("O", c, w) for w in range(WARPS)} for c in (0, 1)]
        self.KK = [[[Buf(f"KK{s}.{h}@{c}") for h in (0, 1)] for s in range(self.NKK)] for c in (0, 1)]
        self.QH = [[[Buf(f"QH{s}.{h}@{c}") for h in (0, 1)] for s in range(self.NQH)] for c in (0, 1)]
        self.KV = [[{"K": Buf(f"KV{s}.K@{c}"), "V": Buf(f"KV{s}.V@{c}")} for s in range(self.NKV)]
                   for c in (0, 1)]
        self.P = [[[Buf(f"P{s}.{w}@{c}") for w in range(WARPS)] for s in range(self.NPB)] for c in (0, 1)]
        nsnap = 1 if "one_snapshot" in self.mut else 2
        self.NSNAP = nsnap
        self.SNAP = [[[Buf(f"SNAP{s}.{w}@{c}") for w in range(WARPS)] for s in range(nsnap)]
                     for c in (0, 1)]
        self.S = [[Buf(f"tmS{s}@{c}", P_ids[c]) for s in range(self.NS)] for c in (0, 1)]
        self.O = [[Buf(f"tmO{s}@{c}", O_ids[c]) for s in range(2)] for c in (0, 1)]
        self.DKV = [[Buf(f"tmDKV{s}@{c}", O_ids[c]) for s in range(2)] for c in (0, 1)]
        self.ssx = [[[None] * WARPS for _ in range(2)] for _ in (0, 1)]
        self.inflight: list[_Ev] = []
        self.fifo = {"A": [], "B": []}
        self.issued = {"A": 0, "B": 0}
        self.completed = {"A": 0, "B": 0}
        self.commits: list[_Ev] = []

    @staticmethod
    def compiles(kk, qh, kv, pbufs, sahead):
        """The compile-time checks on the ring depths (PairCfg in prefill_pair.cuh and the
        pair kernel's launch in lightning.cu)."""
        ns = sahead + 1
        return (kk <= ns and qh <= NDONE and kv <= NDONE and pbufs <= NDONE
                and (sahead <= kv or pbufs <= kv))

    # ------------------------------------------------------------------ set-up
    def _cta_bars(self, c):
        G = 2 * WARPS            # arrivals from one epilogue group in each of the two CTAs

        def ring(name, n, count):
            return [Barrier(f"{name}[{i}]@{c}", count) for i in range(n)]
        single_p = "single_p_ready" in self.mut
        return {
            "full_kk": ring("full_kk", self.NKK, 1),
            "full_qh": ring("full_qh", self.NQH, 1),
            "full_kv": ring("full_kv", self.NKV, 1),
            "tail_kv": Barrier(f"tail_kv@{c}", 1),
            "tail_zeroed": Barrier(f"tail_zeroed@{c}", G),
            "s_full": ring("s_full", self.NS, 1),
            "s_free": ring("s_free", self.NS, G),
            "kv_done": ring("kv_done", NDONE, 1),
            "o_done": ring("o_done", NDONE, 1),
            "o_free": ring("o_free", 2, G),
            "dkv_free": ring("dkv_free", 2, G),
            "p_ready": ring("p_ready", 1 if single_p else self.NPB, G),
            "snap_ready": ring("snap_ready", 2, G),
            "drain": Barrier(f"drain@{c}", 2),
            "ss_bar": ring("ss_bar", 2, WARPS),
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
        for buf, tag in reads:
            if buf.tag != tag or buf.writing:
                state = " (still being written)" if buf.writing else ""
                raise ProtocolError(f"{issuer}: {what} reads {buf.name} holding {buf.tag}{state}, "
                                    f"wants {tag}")
        for buf in zeroed:
            if buf.zeroed != set(range(WARPS)):
                raise ProtocolError(f"{issuer}: {what} reads {buf.name} before the rows past the "
                                    f"sequence end were zeroed")
        for buf, tag, acc in writes:
            if acc:
                if buf.tag != tag:
                    raise ProtocolError(f"{issuer}: {what} accumulates onto {buf.name} holding "
                                        f"{buf.tag}, wants {tag}")
            else:
                if buf.consumers:
                    raise ProtocolError(f"{issuer}: {what} overwrites {buf.name} ({buf.tag}) before "
                                        f"{sorted(buf.consumers)} loaded it")
                buf.tag, buf.consumers = tag, set(buf.consumer_ids)
            buf.writing += 1
        for buf, _ in reads:
            buf.reading += 1
        self.fifo[issuer].append((reads, writes))
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

    # ------------------------------------------------------------------ agents
    def producer(self, c):
        who = f"producer{c}"
        B0, Bc = self.bars[0], self.bars[c]
        nb, NKK, NQH, NKV, NS = self.nb, self.NKK, self.NQH, self.NKV, self.NS
        jk = jq = jv = 0
        # a query slot is released by O_j (o_done); the mutation releases it at S_j instead
        if "qh_release_on_s_full" in self.mut:
            qh_ring, qh_n = Bc["s_full"], NS
        else:
            qh_ring, qh_n = Bc["o_done"], NDONE

        def freed(ring, nring, j, depth):
            x = j - depth
            if x < 0:
                return True
            bar, n = ring[x % nring], x // nring
            self._check_wait(who, bar, n, start=True)
            return bar.done >= n + 1

        def cond(ring, nring, j, depth):
            x = j - depth
            return [] if x < 0 else [(ring[x % nring], x // nring)]

        while jk < nb or jq < nb or jv < nb:
            progressed = False
            if jk < nb and freed(Bc["s_full"], NS, jk, NKK):
                slot, ph, bar = jk % NKK, jk // NKK, B0["full_kk"][jk % NKK]
                if c == 0:
                    self.arrive(who, 0, bar, ph, expect_tx=2 * KK_BYTES)
                for h in (0, 1):
                    self.tma(who, self.KK[c][slot][h], ("k", jk), bar, ph, HBOX)
                jk += 1
                progressed = True
            if jq < nb and freed(qh_ring, qh_n, jq, NQH):
                slot, ph, bar = jq % NQH, jq // NQH, B0["full_qh"][jq % NQH]
                if c == 0:
                    self.arrive(who, 0, bar, ph, expect_tx=2 * QH_BYTES)
                for h in (0, 1):
                    self.tma(who, self.QH[c][slot][h], ("q", jq), bar, ph, HBOX)
                jq += 1
                progressed = True
            if jv < nb and freed(Bc["kv_done"], NDONE, jv, NKV) and freed(Bc["o_done"], NDONE, jv, NKV):
                slot, ph = jv % NKV, jv // NKV
                last_partial = self.tail and jv == nb - 1
                if c == 0:
                    bar = B0["full_kv"][slot]
                    self.arrive(who, 0, bar, ph, expect_tx=(1 if last_partial else 2) * KV_BYTES)
                elif last_partial:
                    bar, ph = Bc["tail_kv"], 0
                    bar.arrive(0, who, KV_BYTES)
                else:
                    bar = B0["full_kv"][slot]
                self.tma(who, self.KV[c][slot]["K"], ("kv", jv), bar, ph, FBOX)
                self.tma(who, self.KV[c][slot]["V"], ("kv", jv), bar, ph, FBOX)
                jv += 1
                progressed = True
            if progressed:
                yield STEP
            else:
                conds = []
                if jk < nb:
                    conds.append(cond(Bc["s_full"], NS, jk, NKK))
                if jq < nb:
                    conds.append(cond(qh_ring, qh_n, jq, NQH))
                if jv < nb:
                    conds.append(cond(Bc["kv_done"], NDONE, jv, NKV) + cond(Bc["o_done"], NDONE, jv, NKV))
                yield ("poll", conds)
        # drain: the last loads of each ring have landed before the CTA exits
        if c == 0:
            for j in range(max(0, jk - NKK), jk):
                yield ("wait", B0["full_kk"][j % NKK], j // NKK)
            for j in range(max(0, jq - NQH), jq):
                yield ("wait", B0["full_qh"][j % NQH], j // NQH)
            for j in range(max(0, jv - NKV), jv):
                yield ("wait", B0["full_kv"][j % NKV], j // NKV)
        elif self.tail and jv == nb:
            yield ("wait", Bc["tail_kv"], 0)

    def _kk(self, j):
        return [(self.KK[c][j % self.NKK][h], ("k", j)) for c in (0, 1) for h in (0, 1)]

    def _qh(self, j):
        return [(self.QH[c][j % self.NQH][h], ("q", j)) for c in (0, 1) for h in (0, 1)]

    def issuer_a(self):
        B0 = self.bars[0]
        nb, NS = self.nb, self.NS

        def stage_in(j):   # S_j = Q_j K_j^T
            yield ("wait", B0["full_kk"][j % self.NKK], j // self.NKK)
            yield ("wait", B0["full_qh"][j % self.NQH], j // self.NQH)
            if j >= NS:
                yield ("wait", B0["s_free"][j % NS], (j - NS) // NS)
            self.mma("A", f"S_{j}", self._kk(j) + self._qh(j),
                     [(self.S[c][j % NS], ("S", j), False) for c in (0, 1)])
            self.commit("A", [(self.bars[c]["s_full"][j % NS], j // NS) for c in (0, 1)])
            yield STEP

        for j in range(min(self.SAHEAD, nb)):
            yield from stage_in(j)
        for b in range(nb):
            slot = b % self.NKV
            zero_tail = self.tail and b == nb - 1
            if zero_tail and "no_tail_zeroed_wait" not in self.mut:
                yield ("wait", B0["tail_zeroed"], 0)
            yield ("wait", B0["full_kv"][slot], b // self.NKV)
            if b >= 2 and "no_dkv_free_wait" not in self.mut:
                yield ("wait", B0["dkv_free"][b & 1], (b - 2) >> 1)
            reads = [(self.KV[c][slot][p], ("kv", b)) for c in (0, 1) for p in ("K", "V")]
            zeroed = [self.KV[c][slot]["V"] for c in (0, 1)] if zero_tail else []
            self.mma("A", f"dKV_{b}", reads, [(self.DKV[c][b & 1], ("dkv", b), False) for c in (0, 1)],
                     zeroed)
            self.commit("A", [(self.bars[c]["kv_done"][b % NDONE], b // NDONE) for c in (0, 1)])
            yield STEP
            if b + self.SAHEAD < nb:
                yield from stage_in(b + self.SAHEAD)
        self.commit("A", [(B0["drain"], 0)])
        yield ("wait", B0["drain"], 0)

    def _snap(self, u):
        return [(self.SNAP[c][u % self.NSNAP][w], ("snap", u)) for c in (0, 1) for w in range(WARPS)]

    def _snap_ready(self, u):
        if self.NSNAP == 1:
            return self.bars[0]["snap_ready"][0], u - self.u0
        return self.bars[0]["snap_ready"][u & 1], (u - self.u0) >> 1

    def _p_ready(self, b):
        if "single_p_ready" in self.mut:
            return self.bars[0]["p_ready"][0], b
        return self.bars[0]["p_ready"][b % self.NPB], b // self.NPB

    def issuer_b(self):
        B0 = self.bars[0]
        for b in range(self.nb):
            if b >= 2:
                yield ("wait", B0["o_free"][b & 1], (b - 2) >> 1)
            if "no_qh_wait_b" not in self.mut:
                yield ("wait", B0["full_qh"][b % self.NQH], b // self.NQH)
            if b >= self.u0:
                yield ("wait", *self._snap_ready(b))
                self.mma("B", f"Qsnap_{b}", self._qh(b) + self._snap(b),
                         [(self.O[c][b & 1], ("o", b), False) for c in (0, 1)])
                yield STEP
            yield ("wait", *self._p_ready(b))
            yield ("wait", B0["full_kv"][b % self.NKV], b // self.NKV)
            reads = [(self.P[c][b % self.NPB][w], ("p", b)) for c in (0, 1) for w in range(WARPS)]
            reads += [(self.KV[c][b % self.NKV]["V"], ("kv", b)) for c in (0, 1)]
            self.mma("B", f"PV_{b}", reads, [(self.O[c][b & 1], ("o", b), b >= self.u0) for c in (0, 1)])
            self.commit("B", [(self.bars[c]["o_done"][b % NDONE], b // NDONE) for c in (0, 1)])
            yield STEP
        self.commit("B", [(B0["drain"], 0)])
        yield ("wait", B0["drain"], 0)

    def group_p(self, c, w):
        who = f"P{c}.{w}"
        B0, Bc = self.bars[0], self.bars[c]
        NS = self.NS
        for b in range(self.nb):
            yield ("wait", Bc["s_full"][b % NS], b // NS)
            self.tmem_ld(who, ("P", c, w), self.S[c][b % NS], ("S", b))
            self.arrive(who, c, B0["s_free"][b % NS], b // NS)
            yield STEP
            pb = b - self.NPB
            if pb >= 0 and "no_o_done_wait_p" not in self.mut:
                yield ("wait", Bc["o_done"][pb % NDONE], pb // NDONE)
            self.store(who, self.P[c][b % self.NPB][w], ("p", b))
            yield STEP
            if self.tail and b == self.nb - 1:
                if c == 0:
                    yield ("wait", B0["full_kv"][b % self.NKV], b // self.NKV)
                else:
                    yield ("wait", Bc["tail_kv"], 0)
                self.zero_tail(who, w, self.KV[c][b % self.NKV]["V"], ("kv", b))
                self.arrive(who, c, B0["tail_zeroed"], 0)
                yield STEP
            self.arrive(who, c, *self._p_ready(b))
            yield STEP

    def group_o(self, c, w):
        who = f"O{c}.{w}"
        B0, Bc = self.bars[0], self.bars[c]

        def write_snap(u):
            self.store(who, self.SNAP[c][u % self.NSNAP][w], ("snap", u))
            self.arrive(who, c, *self._snap_ready(u))

        if self.init:
            write_snap(0)
            yield STEP
        for b in range(self.nb):
            yield ("wait", Bc["kv_done"][b % NDONE], b // NDONE)
            self.tmem_ld(who, ("O", c, w), self.DKV[c][b & 1], ("dkv", b))
            self.arrive(who, c, B0["dkv_free"][b & 1], b >> 1)
            yield STEP
            if b + 1 < self.nb:
                write_snap(b + 1)
                yield STEP
            yield ("wait", Bc["o_done"][b % NDONE], b // NDONE)
            self.tmem_ld(who, ("O", c, w), self.O[c][b & 1], ("o", b))
            self.arrive(who, c, B0["o_free"][b & 1], b >> 1)
            yield STEP
            if self.rms:   # exchange of the row's partial sum of squares with warp w ^ 2
                prev = self.ssx[c][b & 1][w]
                if prev is not None and not prev[1]:
                    raise ProtocolError(f"{who}: overwrites its partial sum of block {prev[0]} "
                                        f"before warp {w ^ 2} read it")
                self.ssx[c][b & 1][w] = [b, False]
                Bc["ss_bar"][b & 1].arrive(b >> 1, who)
                yield ("wait", Bc["ss_bar"][b & 1], b >> 1)
                other = self.ssx[c][b & 1][w ^ 2]
                if other is None or other[0] != b:
                    raise ProtocolError(f"{who}: reads the partial sum of warp {w ^ 2} for block "
                                        f"{None if other is None else other[0]}, wants {b}")
                other[1] = True
                yield STEP

    def agents(self):
        """name -> generator, one per role of the kernel."""
        agents = {"producer0": self.producer(0), "producer1": self.producer(1),
                  "A": self.issuer_a(), "B": self.issuer_b()}
        for c in (0, 1):
            for w in range(WARPS):
                agents[f"P{c}.{w}"] = self.group_p(c, w)
                agents[f"O{c}.{w}"] = self.group_o(c, w)
        return agents

    # ------------------------------------------------------------------ scheduler
    def _events(self):
        evs = list(self.inflight)
        for who in ("A", "B"):
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
        if self.inflight or self.fifo["A"] or self.fifo["B"] or self.commits:
            raise ProtocolError("work still in flight after every agent finished")
