"""Model check of the decision kernel's mbarrier protocol (CPU only).

A small discrete model of the persistent decision_attn_kernel.cuh: one CTA
claiming pairs of query tiles (one per stream) that walk one shared dense
sequence of KV blocks twice (first sweep: score MMAs only, for each row's
log-sum-exp; second: P, O and the pooled mass), with the TMA producer, one MMA
issuer per stream and four softmax warps per stream, the tensor core and the
TMA engine, connected by mbarriers with phase counters.  Random interleavings
(TMA loads landing in any order, the roles advancing in any order) are explored
for many pair sequences (one to four KV blocks, missing second tiles) and ring
sizes, checking

* that no schedule deadlocks;
* that every parity wait only observes its own phase or the next one (a barrier
  two phases ahead, or one behind, would make ``try_wait.parity`` lie); and
* that no buffer is used out of turn: an MMA reads the Q tile and ring slot it
  was issued for; the softmax reads its block's scores and the PV its block's P;
  a tile's first PV (which overwrites O) comes after the epilogue of the
  stream's previous tile has read O; an epilogue reads O after the tile's last
  PV; each stream's score MMAs see its own blocks in its own order.

The model follows the kernel step for step.  The producer claims a pair,
publishes it in the pair queue for the softmax warps, and loads, into slot
(item mod NS) once the MMAs that read the slot's previous item are complete:
each stream's Q once that stream's previous tile's last score MMA is complete
(q_free), the K of the first entry, then per entry u: V(u) (second sweep only)
and K(u + 1); each item carries flags saying which streams use it and whether
it is a stream's first or last score / PV item of its tile; a final item marks
the end.  Each issuer takes a V item together with the K item after it (entry
n) and, when its stream uses the entry, its P (and, for a tile's first score
MMA, its Q) is ready and it is the stream's turn (stream 0 after stream 1's
group of entry n - 1, stream 1 after stream 0's of entry n), issues the
stream's group: PV on V [o_done after the tile's last], S on K [q_free after
the tile's last; s_full].  Then it passes the turn and releases the entry's
slots; a slot is free once both issuers have released it.  A commit fires when
the MMAs its own thread issued before it have run.  Known-bad variants (an
epilogue that reads O only after the next tile's first P, no q_free wait, no
wait for the previous use of a ring slot, releasing a slot before the MMA that
reads it) are checked to be caught, so the checker is not vacuous.
"""
import random

import pytest

N_WARPS = 4  # softmax warps per stream (each arrives once on p_full)


class Bar:
    def __init__(self, count=1):
        self.count, self.arr, self.done = count, 0, 0

    def arrive(self):
        self.arr += 1
        if self.arr == self.count:
            self.arr = 0
            self.done += 1


class Hazard(AssertionError):
    pass


def decision_entries(nkb, second):
    """A pair's entries: blocks 0..nkb-1 twice, shared by the pair's tiles; PV in the
    second sweep only."""
    return [(kb % nkb, True, second, kb >= nkb) for kb in range(2 * nkb)]


class Model:
    def __init__(self, units, ns, seed, tq=4, bad=None):
        """units: a list of (nkb, second tile exists)."""
        self.rng = random.Random(seed)
        self.ns, self.tq, self.bad = ns, tq, bad or set()
        self.units = [decision_entries(*u) for u in units]
        self.bars = {"drain": Bar(2), ("turn", 0): Bar(), ("turn", 1): Bar()}
        for s in (0, 1):
            for name, cnt in (("q_full", 1), ("q_free", 1), ("s_full", 1), ("p_full", N_WARPS),
                              ("o_done", 1)):
                self.bars[(s, name)] = Bar(cnt)
        for i in range(ns):
            self.bars[("full", i)] = Bar()
            self.bars[("empty", i)] = Bar(2)
        for i in range(tq):
            self.bars[("tq_full", i)] = Bar()
            self.bars[("tq_empty", i)] = Bar(2 * N_WARPS)
        self.queue = {}
        self.q_buf = {0: None, 1: None}
        self.slot = {i: None for i in range(ns)}
        self.sbuf = {0: None, 1: None}
        self.o = {0: ("free", -1), 1: ("free", -1)}
        self.pv_inflight = {0: 0, 1: 0}
        self.o_reads = {}
        self.seen = {0: [], 1: []}  # KV blocks each stream's score MMAs read, in order
        self.meta = {}  # ring item number -> flags
        self.item_kb = {}  # ring item number -> KV block
        self.groups = []  # (entry, stream) of each group, in the order the groups are issued
        self.tc = []  # the tensor-core queue: (role, "mma" | "commit", what), in issue order
        self.tma = []
        self.roles = [self.producer(), self.issuer(0), self.issuer(1)]
        for s in (0, 1):
            for w in range(N_WARPS):
                self.roles.append(self.softmax(s, w))
        self.cur = [next(r) for r in self.roles]

    def stream_blocks(self, u, s):
        return [kb for kb, i0, i1, _ in self.units[u] if (i0, i1)[s]]

    # ---------------------------------------------------------------- roles
    def producer(self):
        e, items, kq = 0, 0, [0, 0]

        def load(kb, meta):
            nonlocal items
            i = items % self.ns
            if items >= self.ns and "no_slot_wait" not in self.bad:
                yield ("wait", ("empty", i), items // self.ns - 1)
            self.meta[items] = meta
            self.item_kb[items] = kb
            if meta["kind"] == "end":
                yield ("arrive", ("full", i))
            else:
                yield ("tma", ("full", i), ("slot", i, (items, kb)))
            items += 1

        def flags(kind, ent, cnt, tot):
            f = {"kind": kind, "use": [False, False], "first": [False, False],
                 "last": [False, False]}
            for s in (0, 1):
                if ent[1 + s]:
                    f["use"][s] = True
                    f["first"][s] = cnt[s] == 0
                    cnt[s] += 1
                    f["last"][s] = cnt[s] == tot[s]
            return f

        for u in list(range(len(self.units))) + [None]:
            q = e % self.tq
            if e >= self.tq:
                yield ("wait", ("tq_empty", q), e // self.tq - 1)
            self.queue[e] = u
            yield ("arrive", ("tq_full", q))
            e += 1
            if u is None:
                break
            ent = self.units[u]
            if not ent:
                continue
            n = [sum(1 for x in ent if x[1 + s]) for s in (0, 1)]
            npv = [sum(1 for x in ent if x[1 + s] and x[3]) for s in (0, 1)]
            ns_, nv = [0, 0], [0, 0]
            for s in (0, 1):
                if n[s]:
                    if kq[s] > 0 and "no_q_free" not in self.bad:
                        yield ("wait", (s, "q_free"), kq[s] - 1)
                    yield ("tma", (s, "q_full"), ("q", s, (s, kq[s])))
                    kq[s] += 1
            yield from load(ent[0][0], flags("K", ent[0], ns_, n))
            for i, x in enumerate(ent):
                if x[3]:
                    yield from load(x[0], flags("V", x, nv, npv))
                if i + 1 < len(ent):
                    y = ent[i + 1]
                    yield from load(y[0], flags("K", y, ns_, n))
        yield from load(None, {"kind": "end"})
        yield ("end",)

    def issuer(self, st):
        """Issuer st: a V item together with the K item after it (entry n); when stream
        st uses it, its group [PV on V, S on K] once its P (and, for a tile's first
        score MMA, its Q) is ready and it is the stream's turn; then it passes the turn
        and releases the entry's slots."""
        items, J, k, kpv, pp = 0, 0, 0, 0, False

        def take():
            nonlocal items
            i = items % self.ns
            yield ("wait", ("full", i), items // self.ns)
            it = items
            items += 1
            return i, it, self.meta[it]

        n = 0
        while True:
            i1, it1, m1 = yield from take()
            if m1["kind"] == "end":
                break
            v = k_ = None
            end = False
            if m1["kind"] == "V":
                v = (i1, it1, m1)
                i2, it2, m2 = yield from take()
                if m2["kind"] == "end":
                    end = True
                else:
                    k_ = (i2, it2, m2)
            else:
                k_ = (i1, it1, m1)
            use_v = v is not None and v[2]["use"][st]
            use_k = k_ is not None and k_[2]["use"][st]
            if use_v or (use_k and pp):
                yield ("wait", (st, "p_full"), J)
                J += 1
                pp = False
            if use_k and k_[2]["first"][st]:
                yield ("wait", (st, "q_full"), k)
            if (st == 1 or n > 0) and "no_turns" not in self.bad:
                yield ("wait", ("turn", 1 - st), n if st == 1 else n - 1)
            if use_v or use_k:
                self.groups.append((n, st))
            if use_v:
                i, it, m = v
                yield ("mma", ("PV", st, J - 1, (st, kpv), i, it, m["first"][st],
                               self.item_kb[it]))
                if m["last"][st]:
                    yield ("commit", (st, "o_done"))
                    kpv += 1
            if use_k:
                i, it, m = k_
                yield ("mma", ("S", st, J, (st, k), i, it, self.item_kb[it]))
                if m["last"][st]:
                    yield ("commit", (st, "q_free"))
                    k += 1
                yield ("commit", (st, "s_full"))
                pp = True
            yield ("arrive", ("turn", st))
            if v is not None:
                if "early_release" in self.bad:
                    yield ("arrive", ("empty", v[0]))
                else:
                    yield ("commit", ("empty", v[0]))
            if k_ is not None:
                yield ("commit", ("empty", k_[0]))
            n += 1
            if end:
                break
        yield ("commit", "drain")
        yield ("wait", "drain", 0)
        yield ("end",)

    def softmax(self, s, w):
        e, J, k = 0, 0, 0
        late = None  # an epilogue read deferred by the bad variant
        while True:
            q = e % self.tq
            yield ("wait", ("tq_full", q), e // self.tq)
            u = self.queue[e]
            yield ("arrive", ("tq_empty", q))
            e += 1
            if u is None:
                break
            ent = self.units[u]
            if s == 1 and not ent[0][2]:
                continue  # the pair's second tile does not exist
            mine = [y for y in ent if y[1 + s]]
            n, npv = len(mine), sum(1 for y in mine if y[3])
            for j, y in enumerate(mine):
                yield ("wait", (s, "s_full"), J)
                yield ("read_s", s, J)
                if y[3]:
                    yield ("write_p", s, J)
                yield ("arrive", (s, "p_full"))
                J += 1
                if late is not None and y[3]:
                    yield late
                    late = None
            if n > 0:
                yield ("wait", (s, "o_done"), k)
                k += 1
            if n > 0:
                r = ("read_o", s, s, k - 1, npv)
                if "late_epilogue" in self.bad:
                    late = r
                else:
                    yield r
        if late is not None:
            yield late
        yield ("end",)

    # ---------------------------------------------------------------- engine
    def check(self, cond, what):
        if not cond:
            raise Hazard(what)

    def exec_mma(self, op):
        if op[0] == "S":
            _, s, J, qk, i, it, kb = op
            self.check(self.q_buf[s] == qk, f"S({J}) of stream {s} reads Q {self.q_buf[s]}, wants {qk}")
            self.check(self.slot[i] == (it, kb), f"S({J}) reads slot {self.slot[i]}, wants {(it, kb)}")
            self.sbuf[s] = ("S", J)
            self.seen[s].append(kb)
        else:
            _, s, J, qk, i, it, first, kb = op
            self.check(self.slot[i] == (it, kb), f"PV({J}) reads slot {self.slot[i]}, wants {(it, kb)}")
            self.check(self.sbuf[s] == ("P", J, N_WARPS), f"PV({J}) of stream {s} reads {self.sbuf[s]}")
            k = qk[1]
            if first:
                self.check(self.o[s] in (("free", k - 1), ("free", -1)),
                           f"first PV of tile {k} of stream {s} overwrites O in state {self.o[s]}")
                self.o[s] = ("acc", k, 1)
            else:
                self.check(self.o[s][:2] == ("acc", k), f"PV of tile {k} into O {self.o[s]}")
                self.o[s] = ("acc", k, self.o[s][2] + 1)
            self.pv_inflight[s] -= 1

    def effect(self, op):
        kind = op[0]
        if kind == "read_s":
            _, s, J = op
            cur = self.sbuf[s]
            self.check(cur == ("S", J) or (cur is not None and cur[0] == "P" and cur[1] == J),
                       f"softmax {s} reads S({J}) from {cur}")
        elif kind == "write_p":
            _, s, J = op
            cur = self.sbuf[s]
            self.sbuf[s] = ("P", J, 1) if cur == ("S", J) else ("P", J, cur[2] + 1)
        elif kind == "read_o":
            _, reader, s, k, n = op
            self.check(self.o[s] == ("acc", k, n),
                       f"stream {reader} reads O_{s} of tile {k} in state {self.o[s]}")
            self.check(self.pv_inflight[s] == 0, "O read with a PV in flight")
            self.o_reads[(s, k)] = self.o_reads.get((s, k), 0) + 1
            if self.o_reads[(s, k)] == N_WARPS:
                self.o[s] = ("free", k)

    def ready(self, op):
        if op[0] != "wait":
            return True
        done = self.bars[op[1]].done
        if not op[2] <= done <= op[2] + 1:
            raise AssertionError(f"parity ambiguity on {op[1]}: phase {op[2]}, done {done}")
        return done == op[2] + 1

    def run(self, max_steps=2000000):
        for _ in range(max_steps):
            live = [i for i, op in enumerate(self.cur) if op[0] != "end"]
            if not live and not self.tc and not self.tma:
                want = [[kb for u in range(len(self.units)) for kb in self.stream_blocks(u, s)]
                        for s in (0, 1)]
                self.check(self.seen[0] == want[0] and self.seen[1] == want[1],
                           "a stream's score MMAs did not follow its own blocks")
                return True
            choices = [("role", i) for i in live if self.ready(self.cur[i])]
            if self.tc:
                choices.append(("tc", None))
            if self.tma:
                choices.append(("tma", None))
            if not choices:
                return False
            kind, i = self.rng.choice(choices)
            if kind == "tc":
                # MMAs run in issue order; a commit fires once the MMAs its own
                # thread issued before it have run, whatever the other issuer queued
                fire = [0] + [p for p, it in enumerate(self.tc) if p > 0 and it[1] == "commit"
                              and not any(x[0] == it[0] and x[1] == "mma" for x in self.tc[:p])]
                item = self.tc.pop(self.rng.choice(fire))
                if item[1] == "commit":
                    self.bars[item[2]].arrive()
                else:
                    self.exec_mma(item[2])
            elif kind == "tma":
                bar, what = self.tma.pop(self.rng.randrange(len(self.tma)))
                if what[0] == "q":
                    self.q_buf[what[1]] = what[2]
                else:
                    self.slot[what[1]] = what[2]
                self.bars[bar].arrive()
            else:
                op = self.cur[i]
                if op[0] == "tma":
                    self.tma.append((op[1], op[2]))
                elif op[0] == "mma":
                    if op[1][0] == "PV":
                        self.pv_inflight[op[1][1]] += 1
                    self.tc.append((i, "mma", op[1]))
                elif op[0] == "commit":
                    self.tc.append((i, "commit", op[1]))
                elif op[0] == "arrive":
                    self.bars[op[1]].arrive()
                elif op[0] != "wait":
                    self.effect(op)
                self.cur[i] = next(self.roles[i])
        raise AssertionError("model did not finish")


def _pair_sequences(seed, count):
    rng = random.Random(seed)
    seqs = [[(1, True)], [(1, False)], [(2, True), (1, False)], [(3, True)] * 3]
    for _ in range(count):
        seqs.append([(rng.randint(1, 4), rng.random() < 0.8) for _ in range(rng.randint(1, 3))])
    return seqs


@pytest.mark.parametrize("ns", [2, 3, 4])
def test_never_deadlocks_and_keeps_buffers_in_turn(ns):
    for t, units in enumerate(_pair_sequences(ns, 30)):
        for seed in range(3):
            assert Model(units, ns, seed * 1000 + t).run(), (units, seed)


def test_short_pair_queue_still_completes():
    for seed in range(30):
        assert Model([(2, True), (1, False), (3, True), (1, True)], 2, seed, tq=2).run()


def test_entries_walk_the_prefix_twice():
    assert decision_entries(2, False) == [(0, True, False, False), (1, True, False, False),
                                          (0, True, False, True), (1, True, False, True)]


def _caught(bad, units, ns, seeds=200):
    caught = 0
    for seed in range(seeds):
        try:
            if not Model(units, ns, seed, bad=set(bad.split("+"))).run():
                caught += 1
        except AssertionError:
            caught += 1
    return caught


def test_late_epilogue_is_caught():
    """An epilogue that read O only after handing over the next tile's first P (of its
    second sweep) would let that tile's first PV overwrite O before it is read."""
    assert _caught("late_epilogue", [(2, True), (1, True), (2, False)], 2) > 0


def test_missing_q_free_wait_is_caught():
    """Without the q_free wait the next tile's Q can land while a score MMA of the
    current tile still reads the buffer."""
    assert _caught("no_q_free", [(2, True), (2, True), (1, True)], 4) > 0


def test_missing_slot_wait_is_caught():
    """Without waiting for the previous use of a ring slot a load can overwrite an
    operand before its MMA has run."""
    assert _caught("no_slot_wait", [(4, True), (3, True)], 2) > 0


def test_release_before_the_mma_is_caught():
    """An issuer that released a V slot with a plain arrival (instead of a commit that
    fires when its PV has read the slot) would let the next load overwrite V early."""
    assert _caught("early_release", [(4, True), (3, True)], 2) > 0


def test_groups_take_turns():
    """The issuers' groups reach the tensor core entry by entry, stream 0 first."""
    for t, units in enumerate(_pair_sequences(5, 20)):
        for seed in range(3):
            m = Model(units, 4, seed * 100 + t)
            assert m.run()
            assert m.groups == sorted(m.groups), (units, seed)
