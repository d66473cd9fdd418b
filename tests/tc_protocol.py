"""Executable model of the synchronisation in ``prefill_tc_kernel``
(long_context_04_b200/csrc/prefill_tc.cuh), checked under random schedules.

Like ``pair_protocol.py`` for the paired kernel, the model has no arithmetic: it tracks which
block's data each shared-memory tile, snapshot buffer and TMEM accumulator holds, and the
mbarriers that order them.  Each agent is a generator mirroring one role of the kernel in the
kernel's order, one step per wait, arrival, TMA issue, store or MMA issue:

    producer<c>        warp 0: Q, K and the value slice of every block into a ring of stages
    A<c>               issuer A: the scores S_b (two blocks ahead) and dKV_b = K_b^T V_b,
                       once issuer B's O_b = P_b V_b has completed
    B<c>               issuer B: O_b = P_b V_b (it zeroes the value rows past the sequence
                       end first), then O_b += Q_b snap_b on the same accumulator
    P<c>.<w>, O<c>.<w>, KV<c>.<w>
                       warp w (0..3) of group P (S -> P in TMEM), group O (O -> RMSNorm ->
                       store) and group KV (state, snapshots) of CTA c

With D = 128 the two value slices of a head are two CTAs of a cluster (c = 0, 1) that only
meet in the RMSNorm exchange; with D = 64 there is one CTA.  Asynchronous work is a pool of
events fired in random order, interleaved with the agents' steps: TMA landings, MMA
completions (in issue order per issuing thread; the issuers of one CTA are independent),
commit arrivals and the partner CTA's remote arrivals.  Every schedule is checked for:
  * the parity-wait rules on every wait (phase n - 1 complete when it starts, phase n + 1
    not complete before it returns), and each arrival landing in the phase its sender means;
  * MMA operands landed and for the intended block, the value rows past the sequence end
    zeroed before any product reads them;
  * no accumulator overwritten before its warps loaded it, and no MMA of one issuer writing
    a TMEM buffer that an in-flight MMA of the other issuer reads or writes (one issuer's
    MMAs run in order, so its own earlier reads are safe);
  * O loaded only once both of its products completed; no shared-memory or TMEM store, and
    no TMA load, into a buffer an in-flight MMA reads;
  * the RMSNorm partial sums read only after the partner wrote them, never overwritten
    before they were read;
  * no deadlock, nothing in flight at exit.
Not modelled: the timeout / abort paths, TMEM allocation, the numerical content.
"""
from __future__ import annotations

import random

from pair_protocol import STEP, Barrier, ProtocolError, _Ev

WARPS = 4


class TBuf:
    """A shared-memory tile or TMEM buffer; in-flight MMA reads and writes per issuer."""

    def __init__(self, name: str, consumers=()):
        self.name = name
        self.tag = None
        self.reading: dict[str, int] = {}
        self.writing: dict[str, int] = {}
        self.consumer_ids = frozenset(consumers)
        self.consumers = set()
        self.zeroed = False

    def busy(self, exclude=None):
        return any(n for who, n in self.reading.items() if who != exclude) or \
            any(n for who, n in self.writing.items() if who != exclude)


class TcModel:
    """One (sequence, head) of ``nb`` blocks: one CTA (D = 64) or the two value-slice CTAs
    of a cluster (D = 128).  tail: partial last block; init: start from an initial state;
    rms: the fused RMSNorm (its exchange only exists with two CTAs); nst: TMA stages."""

    def __init__(self, nb, tail=False, init=False, rms=False, pair=True, nst=4, mutations=(),
                 static_checks=True):
        self.nb, self.tail, self.init, self.rms = nb, tail and nb > 0, init, rms
        self.ctas = (0, 1) if pair else (0,)
        self.NST = nst
        self.u0 = 0 if init else 1
        self.mut = frozenset(mutations)
        if static_checks and not self.compiles(nst):
            raise ValueError("stage count rejected by the kernel's static_assert")
        self.bars = {c: self._bars(c) for c in self.ctas}
        self.Q = {c: [TBuf(f"Q{s}@{c}") for s in range(nst)] for c in self.ctas}
        self.K = {c: [TBuf(f"K{s}@{c}") for s in range(nst)] for c in self.ctas}
        self.V = {c: [TBuf(f"V{s}@{c}") for s in range(nst)] for c in self.ctas}
        self.SNAP = {c: [TBuf(f"snap{s}@{c}") for s in range(2)] for c in self.ctas}
        # S and P share a TMEM buffer; each group-P warp owns one lane quadrant of it
        self.SQ = {c: [[TBuf(f"tmS{s}.{w}@{c}", {("P", c, w)}) for w in range(WARPS)]
                       for s in range(2)] for c in self.ctas}
        self.O = {c: [TBuf(f"tmO{s}@{c}", {("O", c, w) for w in range(WARPS)}) for s in range(2)]
                  for c in self.ctas}
        self.DKV = {c: [TBuf(f"tmDKV{s}@{c}", {("KV", c, w) for w in range(WARPS)})
                        for s in range(2)] for c in self.ctas}
        self.ssx = {c: [[None] * WARPS for _ in range(2)] for c in self.ctas}
        self.inflight: list[_Ev] = []
        issuers = [f"{r}{c}" for c in self.ctas for r in "AB"]
        self.fifo = {i: [] for i in issuers}
        self.issued = {i: 0 for i in issuers}
        self.completed = {i: 0 for i in issuers}
        self.commits: list[_Ev] = []

    @staticmethod
    def compiles(nst):
        """The kernel's static_assert (NST >= 3): the scores run two blocks ahead, so three
        stages (blocks b, b + 1 and b + 2) are resident at once for the load of b + 2 to
        overlap block b.  (A prefetch-depth bound: the protocol itself is also clean with two.)"""
        return nst >= 3

    def _bars(self, c):
        def ring(name, n, count):
            return [Barrier(f"{name}[{i}]@{c}", count) for i in range(n)]
        empty_count = 1 if "single_empty_arrival" in self.mut else 2
        return {
            "full": ring("full", self.NST, 1),
            "empty": ring("empty", self.NST, empty_count),
            "s_full": ring("s_full", 2, 1),
            "p_ready": ring("p_ready", 2, WARPS),
            "pv_done": ring("pv_done", 2, 1),
            "o_full": ring("o_full", 2, 1),
            "o_free": ring("o_free", 2, WARPS),
            "dkv_full": ring("dkv_full", 2, 1),
            "dkv_free": ring("dkv_free", 2, WARPS),
            "snap_ready": ring("snap_ready", 2, WARPS),
            "ss_full": ring("ss_full", 2, WARPS),
            "drain": Barrier(f"drain@{c}", 2),
            "tail_zeroed": Barrier(f"tail_zeroed@{c}", 1),
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

    def tma(self, who, buf, tag, bar, phase):
        if buf.busy():
            raise ProtocolError(f"{who}: TMA load of {tag} into {buf.name} while an MMA "
                                f"reads or writes it")
        buf.tag, buf.zeroed = tag, False
        buf.writing["tma"] = buf.writing.get("tma", 0) + 1
        self.inflight.append(_Ev("tma", buf, bar, phase, who))

    def store(self, who, buf, tag):
        if buf.busy():
            raise ProtocolError(f"{who}: stores {tag} into {buf.name} while an MMA reads or "
                                f"writes {buf.tag}")
        buf.tag = tag

    def mma(self, issuer, what, reads, writes, zeroed=()):
        """writes: (buf, expected tag or None, accumulate, new tag)."""
        for buf, tag in reads:
            if buf.tag != tag or buf.writing.get("tma"):
                raise ProtocolError(f"{issuer}: {what} reads {buf.name} holding {buf.tag}"
                                    f"{' (still landing)' if buf.writing.get('tma') else ''}, "
                                    f"wants {tag}")
            if any(n for who, n in buf.writing.items() if who not in (issuer, "tma")):
                raise ProtocolError(f"{issuer}: {what} reads {buf.name} while another issuer's "
                                    f"MMA writes it")
        for buf in zeroed:
            if not buf.zeroed:
                raise ProtocolError(f"{issuer}: {what} reads {buf.name} before the rows past the "
                                    f"sequence end were zeroed")
        for buf, tag, acc, new_tag in writes:
            if buf.busy(exclude=issuer):
                raise ProtocolError(f"{issuer}: {what} writes {buf.name} while another issuer's "
                                    f"MMA reads or writes it")
            if acc:
                if buf.tag != tag:
                    raise ProtocolError(f"{issuer}: {what} accumulates onto {buf.name} holding "
                                        f"{buf.tag}, wants {tag}")
            elif buf.consumers:
                raise ProtocolError(f"{issuer}: {what} overwrites {buf.name} ({buf.tag}) before "
                                    f"{sorted(buf.consumers)} loaded it")
            else:
                buf.consumers = set(buf.consumer_ids)
            buf.tag = new_tag
            buf.writing[issuer] = buf.writing.get(issuer, 0) + 1
        for buf, _ in reads:
            buf.reading[issuer] = buf.reading.get(issuer, 0) + 1
        self.fifo[issuer].append(([b for b, _ in reads], [w[0] for w in writes]))
        self.issued[issuer] += 1

    def commit(self, issuer, bar, phase):
        self.commits.append(_Ev("commit", issuer, self.issued[issuer], bar, phase))

    def tmem_ld(self, who, wid, buf, tag):
        if buf.tag != tag or any(buf.writing.values()):
            raise ProtocolError(f"{who}: loads {buf.name} holding {buf.tag}"
                                f"{' (MMA in flight)' if any(buf.writing.values()) else ''}, "
                                f"wants {tag}")
        if wid not in buf.consumers:
            raise ProtocolError(f"{who}: loads {buf.name} ({tag}) twice")
        buf.consumers.discard(wid)

    # ------------------------------------------------------------------ agents
    def producer(self, c):
        who, B, NST = f"producer{c}", self.bars[c], self.NST
        for b in range(self.nb):
            st = b % NST
            if b >= NST:
                yield ("wait", B["empty"][st], b // NST - 1)
            B["full"][st].arrive(b // NST, who, 3)
            for ring, t in ((self.Q, "q"), (self.K, "k"), (self.V, "v")):
                self.tma(who, ring[c][st], (t, b), B["full"][st], b // NST)
            yield STEP
        for b in range(max(0, self.nb - NST), self.nb):
            yield ("wait", B["full"][b % NST], b // NST)

    def issuer_a(self, c):
        """The scores (two blocks ahead) and dKV_b, once P_b V_b has completed: issuer B zeroes
        the tail rows before it, and issues Q_{b-1} snap_{b-1} before it (so group KV may write
        snapshot b + 1 into that snapshot's buffer once dKV_b is done)."""
        who, B, NST, nb = f"A{c}", self.bars[c], self.NST, self.nb

        def stage_in(j):
            yield ("wait", B["full"][j % NST], j // NST)
            st = j % NST
            self.mma(who, f"S_{j}", [(self.Q[c][st], ("q", j)), (self.K[c][st], ("k", j))],
                     [(self.SQ[c][j & 1][w], None, False, ("S", j)) for w in range(WARPS)])
            self.commit(who, B["s_full"][j & 1], j >> 1)
            yield STEP

        if nb > 0:
            yield from stage_in(0)
        if nb > 1:
            yield from stage_in(1)
        for b in range(nb):
            st = b % NST
            last_tail = self.tail and b == nb - 1
            if "a_no_pv_done_wait" not in self.mut:
                yield ("wait", B["pv_done"][b & 1], b >> 1)
            if b >= 2:
                yield ("wait", B["dkv_free"][b & 1], (b - 2) >> 1)
            if last_tail:
                yield ("wait", B["tail_zeroed"], 0)
            vbuf = self.V[c][st]
            self.mma(who, f"dKV_{b}", [(self.K[c][st], ("k", b)), (vbuf, ("v", b))],
                     [(self.DKV[c][b & 1], None, False, ("dkv", b))],
                     zeroed=[vbuf] if last_tail else [])
            self.commit(who, B["dkv_full"][b & 1], b >> 1)
            self.commit(who, B["empty"][st], b // NST)
            yield STEP
            if b + 2 < nb:
                yield from stage_in(b + 2)
        self.commit(who, B["drain"], 0)
        yield ("wait", B["drain"], 0)

    def issuer_b(self, c):
        """P_b V_b (zeroing the tail rows first), then, in order on the same accumulator,
        O_b += Q_b snap_b."""
        who, B, NST, nb = f"B{c}", self.bars[c], self.NST, self.nb
        qkv_first = "b_qkv_first" in self.mut
        for b in range(nb):
            st = b % NST
            yield ("wait", B["full"][st], b // NST)
            if "p_ready_single" in self.mut:
                yield ("wait", B["p_ready"][0], b)
            else:
                yield ("wait", B["p_ready"][b & 1], b >> 1)
            if b >= 2 and "b_no_o_free_wait" not in self.mut:
                yield ("wait", B["o_free"][b & 1], (b - 2) >> 1)
            last_tail = self.tail and b == nb - 1
            vbuf = self.V[c][st]
            if qkv_first and b >= self.u0:     # the inter-block term issued before P V
                yield ("wait", B["snap_ready"][b & 1], (b - self.u0) >> 1)
                self.mma(who, f"QKV_{b}", [(self.Q[c][st], ("q", b)), (self.SNAP[c][b & 1], ("snap", b))],
                         [(self.O[c][b & 1], ("o_pv", b), True, ("o", b))])
            if last_tail and "zero_after_pv" not in self.mut:
                self._zero(who, vbuf, ("v", b))
                B["tail_zeroed"].arrive(0, who)
            self.mma(who, f"PV_{b}", [(self.SQ[c][b & 1][w], ("P", b)) for w in range(WARPS)] +
                     [(vbuf, ("v", b))], [(self.O[c][b & 1], None, False, ("o_pv", b))],
                     zeroed=[vbuf] if last_tail else [])
            self.commit(who, B["pv_done"][b & 1], b >> 1)
            yield STEP
            if last_tail and "zero_after_pv" in self.mut:
                self._zero(who, vbuf, ("v", b))
                B["tail_zeroed"].arrive(0, who)
            if b >= self.u0 and not qkv_first:
                one = "snap_one_buffer" in self.mut
                yield ("wait", B["snap_ready"][0 if one else b & 1],
                       (b - self.u0) if one else (b - self.u0) >> 1)
                sbuf = self.SNAP[c][0 if one else b & 1]
                self.mma(who, f"QKV_{b}", [(self.Q[c][st], ("q", b)), (sbuf, ("snap", b))],
                         [(self.O[c][b & 1], ("o_pv", b), True, ("o", b))])
            self.commit(who, B["o_full"][b & 1], b >> 1)
            if "single_empty_arrival" not in self.mut:
                self.commit(who, B["empty"][st], b // NST)
            yield STEP
        self.commit(who, B["drain"], 0)
        yield ("wait", B["drain"], 0)

    def _zero(self, who, buf, tag):
        if buf.tag != tag or buf.writing.get("tma"):
            raise ProtocolError(f"{who}: zeroes rows of {buf.name} before {tag} has landed")
        if buf.busy():
            raise ProtocolError(f"{who}: zeroes rows of {buf.name} while an MMA reads it")
        buf.zeroed = True

    def group_p(self, c, w):
        who, B = f"P{c}.{w}", self.bars[c]
        for b in range(self.nb):
            yield ("wait", B["s_full"][b & 1], b >> 1)
            buf = self.SQ[c][b & 1][w]
            self.tmem_ld(who, ("P", c, w), buf, ("S", b))
            self.store(who, buf, ("P", b))          # P over S, in this warp's lanes
            if "p_ready_single" in self.mut:
                B["p_ready"][0].arrive(b, who)
            else:
                B["p_ready"][b & 1].arrive(b >> 1, who)
            yield STEP

    def group_o(self, c, w):
        who, B = f"O{c}.{w}", self.bars[c]
        pair = len(self.ctas) == 2
        for b in range(self.nb):
            yield ("wait", B["o_full"][b & 1], b >> 1)
            self.tmem_ld(who, ("O", c, w), self.O[c][b & 1], ("o", b) if b >= self.u0 else ("o_pv", b))
            B["o_free"][b & 1].arrive(b >> 1, who)
            yield STEP
            if self.rms and pair:
                p = 1 - c
                slot = self.ssx[p][b & 1]
                prev = slot[w]
                if prev is not None and not prev[1]:
                    raise ProtocolError(f"{who}: overwrites the partner's partial sum of block "
                                        f"{prev[0]} before it was read")
                slot[w] = [b, False]
                self.inflight.append(_Ev("arrive", self.bars[p]["ss_full"][b & 1], b >> 1, who))
                if "rms_no_wait" not in self.mut:
                    yield ("wait", B["ss_full"][b & 1], b >> 1)
                mine = self.ssx[c][b & 1][w]
                if mine is None or mine[0] != b:
                    raise ProtocolError(f"{who}: reads the partner's partial sum for block "
                                        f"{None if mine is None else mine[0]}, wants {b}")
                mine[1] = True
                yield STEP

    def group_kv(self, c, w):
        who, B = f"KV{c}.{w}", self.bars[c]

        def write_snap(u):
            one = "snap_one_buffer" in self.mut
            self.store(who, self.SNAP[c][0 if one else u & 1], ("snap", u))
            B["snap_ready"][0 if one else u & 1].arrive(
                (u - self.u0) if one else (u - self.u0) >> 1, who)

        if self.init and self.nb > 0:
            write_snap(0)
            yield STEP
        for b in range(self.nb):
            yield ("wait", B["dkv_full"][b & 1], b >> 1)
            self.tmem_ld(who, ("KV", c, w), self.DKV[c][b & 1], ("dkv", b))
            B["dkv_free"][b & 1].arrive(b >> 1, who)
            yield STEP
            if b + 1 < self.nb:
                write_snap(b + 1)
                yield STEP

    def agents(self):
        agents = {}
        for c in self.ctas:
            agents[f"producer{c}"] = self.producer(c)
            agents[f"A{c}"] = self.issuer_a(c)
            agents[f"B{c}"] = self.issuer_b(c)
            for w in range(WARPS):
                agents[f"P{c}.{w}"] = self.group_p(c, w)
                agents[f"O{c}.{w}"] = self.group_o(c, w)
                agents[f"KV{c}.{w}"] = self.group_kv(c, w)
        return agents

    # ------------------------------------------------------------------ scheduler
    def _events(self):
        evs = list(self.inflight)
        for who, q in self.fifo.items():
            if q:
                evs.append(_Ev("mma", who))
        evs += [e for e in self.commits if self.completed[e.args[0]] >= e.args[1]]
        return evs

    def _fire(self, ev):
        if ev.kind == "tma":
            buf, bar, phase, who = ev.args
            self.inflight.remove(ev)
            buf.writing["tma"] -= 1
            bar.complete_tx(phase, 1, f"{who} (TMA into {buf.name})")
        elif ev.kind == "arrive":
            bar, phase, who = ev.args
            self.inflight.remove(ev)
            bar.arrive(phase, who)
        elif ev.kind == "mma":
            who = ev.args[0]
            reads, writes = self.fifo[who].pop(0)
            for buf in reads:
                buf.reading[who] -= 1
            for buf in writes:
                buf.writing[who] -= 1
            self.completed[who] += 1
        else:
            who, _, bar, phase = ev.args
            self.commits.remove(ev)
            bar.arrive(phase, f"{who} commit")

    def run(self, seed: int, max_steps: int = 1_000_000):
        rng = random.Random(seed)
        bias = rng.uniform(0.05, 0.95)
        agents = self.agents()
        state = {name: ("ready",) for name in agents}
        speeds = (0.02, 0.2, 1.0, 1.0, 5.0)
        w_agent = {name: rng.choice(speeds) for name in agents}
        w_event = {kind: rng.choice(speeds) for kind in ("tma", "arrive", "mma", "commit")}
        for _ in range(max_steps):
            live = [n for n, st in state.items() if st[0] != "done"]
            runnable = [n for n in live if state[n][0] == "ready" or
                        (state[n][0] == "wait" and state[n][1].done >= state[n][2] + 1)]
            events = self._events()
            if not runnable and not events:
                if not live:
                    break
                raise ProtocolError("deadlock: " + "; ".join(
                    f"{n} waits on phase {state[n][2]} of {state[n][1].name}" for n in live))
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
                    if instr[2] >= 0:
                        self._check_wait(name, instr[1], instr[2], start=True)
                    state[name] = ("wait", instr[1], instr[2])
                else:
                    state[name] = ("ready",)
            for n, st in state.items():
                if st[0] == "wait":
                    self._check_wait(n, st[1], st[2], start=False)
        else:
            raise ProtocolError("no end after max_steps")
        if self.inflight or any(self.fifo.values()) or self.commits:
            raise ProtocolError("work still in flight after every agent finished")
