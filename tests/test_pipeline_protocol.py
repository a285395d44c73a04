"""Model check of the attention kernel's mbarrier protocol (CPU only).

A small discrete model of the persistent attn_fwd_kernel.cuh: one CTA claiming
pairs of query tiles (two streams, one tile each) that share one K/V stream:
the TMA producer, the MMA issuer and four softmax warps per stream, with the
tensor core and the TMA engine, connected by mbarriers with phase counters.
Random interleavings (TMA loads landing in any order, random "raise the
reference max" decisions) are explored for many pair sequences (empty lists,
missing second tiles, one-block tiles, disjoint and overlapping lists, lists out
of order) and ring sizes, checking

* that no schedule deadlocks;
* that every parity wait only observes its own phase or the next one (a barrier
  two phases ahead, or one behind, would make ``try_wait.parity`` lie); and
* that no buffer is used out of turn: an MMA reads the Q tile and ring slot it
  was issued for; the softmax reads its block's scores and the PV its block's P;
  a tile's first PV (which overwrites O) comes after the epilogue of the
  stream's previous tile has read O; the softmax rescales O only when no PV of
  its stream is in flight; the epilogue reads O after the tile's last PV; each
  stream's MMAs see its own list in its own order.

The model follows the kernel step for step.  The producer claims a pair,
publishes it in the pair queue, loads each stream's Q once that stream's
previous tile's last score MMA is complete (q_free), and loads ring items in the
order K of the first merged entry, then per entry: V and the K of the next
entry, each into slot (item mod NS) once the MMAs that read the slot's previous
item are complete.  The issuer waits for the streams' Q, issues the score MMAs
of the first entry, then per entry, for stream 0 then 1: wait P (if the stream
keeps the entry), PV [o_done after the stream's last PV of the pair], the
stream's next score MMA if it keeps the next entry [q_free after its last one;
s_full]; then it frees the entry's two slots.  Each softmax warp waits
s_full(J), may rescale O, writes P and arrives on p_full; after a tile's last
block it waits o_done and reads O, before it can arrive on p_full for its next
tile's first block.  Known-bad variants (the epilogue's O read deferred past
the next tile's first block, no q_free wait, no wait for the previous use of a
ring slot) are checked to be caught, so the checker is not vacuous.
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


def merge(l0, l1):
    """The merged sequence: (kb, in0, in1); equal next blocks are shared."""
    out, i0, i1 = [], 0, 0
    while i0 < len(l0) or i1 < len(l1):
        h0, h1 = i0 < len(l0), i1 < len(l1)
        x = l0[i0] if h0 else None
        y = l1[i1] if h1 else None
        if h0 and h1 and x == y:
            out.append((x, True, True))
            i0, i1 = i0 + 1, i1 + 1
        elif h0 and (not h1 or x < y):
            out.append((x, True, False))
            i0 += 1
        else:
            out.append((y, False, True))
            i1 += 1
    return out


class Model:
    def __init__(self, pairs, ns, p_raise, seed, tq=4, bad=None):
        """pairs: [(list0, list1)], a list None when that query block does not exist."""
        self.rng = random.Random(seed)
        self.pairs, self.ns, self.p_raise, self.tq, self.bad = pairs, ns, p_raise, tq, bad or set()
        self.bars = {"drain": Bar()}
        for s in (0, 1):
            for name, cnt in (("q_full", 1), ("q_free", 1), ("s_full", 1), ("p_full", N_WARPS),
                              ("o_done", 1)):
                self.bars[(s, name)] = Bar(cnt)
        for i in range(ns):
            self.bars[("full", i)] = Bar()
            self.bars[("empty", i)] = Bar()
        for i in range(tq):
            self.bars[("tq_full", i)] = Bar()
            self.bars[("tq_empty", i)] = Bar(1 + 2 * N_WARPS)
        self.queue = {}
        self.q_buf = {0: None, 1: None}
        self.slot = {i: None for i in range(ns)}
        self.sbuf = {0: None, 1: None}
        self.o = {0: ("free", -1), 1: ("free", -1)}
        self.pv_inflight = {0: 0, 1: 0}
        self.o_reads = {}
        self.seen = {0: [], 1: []}  # KV blocks each stream's score MMAs read, in order
        self.tc = []  # the issuer's tensor-core queue (in order)
        self.tma = []
        self.roles = [self.producer(), self.issuer()]
        for s in (0, 1):
            for w in range(N_WARPS):
                self.roles.append(self.softmax(s, w))
        self.cur = [next(r) for r in self.roles]

    def lists(self, p):
        l0, l1 = self.pairs[p]
        return [l0 or [], l1 or []]

    # ---------------------------------------------------------------- roles
    def producer(self):
        e, items, kq = 0, 0, [0, 0]

        def load(kb):
            nonlocal items
            i = items % self.ns
            if items >= self.ns and "no_slot_wait" not in self.bad:
                yield ("wait", ("empty", i), items // self.ns - 1)
            yield ("tma", ("full", i), ("slot", i, (items, kb)))
            items += 1

        for p in list(range(len(self.pairs))) + [None]:
            q = e % self.tq
            if e >= self.tq:
                yield ("wait", ("tq_empty", q), e // self.tq - 1)
            self.queue[e] = p
            yield ("arrive", ("tq_full", q))
            e += 1
            if p is None:
                break
            ls = self.lists(p)
            for s in (0, 1):
                if ls[s]:
                    if kq[s] > 0 and "no_q_free" not in self.bad:
                        yield ("wait", (s, "q_free"), kq[s] - 1)
                    yield ("tma", (s, "q_full"), ("q", s, (s, kq[s])))
                    kq[s] += 1
            ent = merge(*ls)
            if not ent:
                continue
            yield from load(ent[0][0])
            for u, (kb, _, _) in enumerate(ent):
                yield from load(kb)  # V
                if u + 1 < len(ent):
                    yield from load(ent[u + 1][0])  # K of the next entry
        yield ("end",)

    def issuer(self):
        e, items = 0, 0
        J, k = [0, 0], [0, 0]

        def wait_item():
            nonlocal items
            i = items % self.ns
            yield ("wait", ("full", i), items // self.ns)
            items += 1
            return i, items - 1

        while True:
            q = e % self.tq
            yield ("wait", ("tq_full", q), e // self.tq)
            p = self.queue[e]
            yield ("arrive", ("tq_empty", q))
            e += 1
            if p is None:
                break
            ls = self.lists(p)
            ent = merge(*ls)
            if not ent:
                continue
            n = [len(ls[0]), len(ls[1])]
            ns_, nv = [0, 0], [0, 0]
            for s in (0, 1):
                if n[s]:
                    yield ("wait", (s, "q_full"), k[s])
            ik, it = yield from wait_item()
            for s in (0, 1):
                if ent[0][1 + s]:
                    yield ("mma", ("S", s, J[s] + ns_[s], (s, k[s]), ik, it, ent[0][0]))
                    ns_[s] += 1
                    if ns_[s] == n[s]:
                        yield ("commit", (s, "q_free"))
                    yield ("commit", (s, "s_full"))
            yield ("commit", ("empty", ik))
            for u, (kb, a0, a1) in enumerate(ent):
                ins = (a0, a1)
                nxt = ent[u + 1] if u + 1 < len(ent) else None
                iv, itv = yield from wait_item()
                ik = None
                for s in (0, 1):
                    if ins[s]:
                        yield ("wait", (s, "p_full"), J[s])
                        yield ("mma", ("PV", s, J[s], (s, k[s]), iv, itv, nv[s] == 0, kb))
                        J[s] += 1
                        nv[s] += 1
                        if nv[s] == n[s]:
                            yield ("commit", (s, "o_done"))
                    if nxt is not None and nxt[1 + s]:
                        if ik is None:
                            ik, itk = yield from wait_item()
                        yield ("mma", ("S", s, J[s], (s, k[s]), ik, itk, nxt[0]))
                        ns_[s] += 1
                        if ns_[s] == n[s]:
                            yield ("commit", (s, "q_free"))
                        yield ("commit", (s, "s_full"))
                yield ("commit", ("empty", iv))
                if ik is not None:
                    yield ("commit", ("empty", ik))
            for s in (0, 1):
                if n[s]:
                    k[s] += 1
        yield ("commit", "drain")
        yield ("wait", "drain", 0)
        yield ("end",)

    def softmax(self, s, w):
        e, J, k = 0, 0, 0
        late = None  # (tile number, blocks) of an epilogue deferred by the bad variant
        while True:
            q = e % self.tq
            yield ("wait", ("tq_full", q), e // self.tq)
            p = self.queue[e]
            yield ("arrive", ("tq_empty", q))
            e += 1
            if p is None:
                break
            if self.pairs[p][s] is None:
                continue
            n = len(self.lists(p)[s])
            for j in range(n):
                yield ("wait", (s, "s_full"), J)
                yield ("read_s", s, J)
                if j > 0 and self.rng.random() < self.p_raise:
                    yield ("rescale_o", s)
                yield ("write_p", s, J)
                yield ("arrive", (s, "p_full"))
                J += 1
                if late is not None:
                    yield ("read_o", s, late[0], late[1])
                    late = None
            if n > 0:
                yield ("wait", (s, "o_done"), k)
                if "late_epilogue" in self.bad:
                    late = (k, n)
                else:
                    yield ("read_o", s, k, n)
                k += 1
        if late is not None:
            yield ("read_o", s, late[0], late[1])
        yield ("end",)

    # ---------------------------------------------------------------- effects
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
                           f"first PV of tile {k} overwrites O in state {self.o[s]}")
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
        elif kind == "rescale_o":
            self.check(self.pv_inflight[op[1]] == 0, "O rescaled while a PV is in flight")
        elif kind == "read_o":
            _, s, k, n = op
            self.check(self.o[s] == ("acc", k, n),
                       f"epilogue of tile {k} of stream {s} reads O {self.o[s]}")
            self.check(self.pv_inflight[s] == 0, "epilogue reads O with a PV in flight")
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
                want = [[kb for p in range(len(self.pairs)) for kb in self.lists(p)[s]]
                        for s in (0, 1)]
                self.check(self.seen[0] == want[0] and self.seen[1] == want[1],
                           "a stream's score MMAs did not follow its own list")
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
                item = self.tc.pop(0)
                if item[0] == "commit":
                    self.bars[item[1]].arrive()
                else:
                    self.exec_mma(item[1])
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
                    self.tc.append(("mma", op[1]))
                elif op[0] == "commit":
                    self.tc.append(op)
                elif op[0] == "arrive":
                    self.bars[op[1]].arrive()
                elif op[0] != "wait":
                    self.effect(op)
                self.cur[i] = next(self.roles[i])
        raise AssertionError("model did not finish")


def _pair_sequences(seed, count):
    rng = random.Random(seed)

    def rlist(nkb=12):
        n = rng.choice([0, 1, 1, 2, 3, 5, 8])
        return sorted(rng.sample(range(nkb), n))

    seqs = [
        [([0], [0])], [([0, 1, 2], [1, 2, 3])], [([0, 5], [1, 2, 3, 4])], [([], [0, 1])],
        [([0, 1], None)], [([], [])], [([3], [])], [([0, 1, 2, 3], [0, 1, 2, 3])] * 3,
        [([0, 2, 4], [1, 3, 5]), ([7], [7]), ([], None)],
        [([5, 1, 3], [1, 3, 5])],  # a list out of order: less sharing, still correct
    ]
    for _ in range(count):
        seqs.append([(rlist(), rlist() if rng.random() < 0.85 else None)
                     for _ in range(rng.randint(1, 5))])
    return seqs


@pytest.mark.parametrize("ns", [2, 4])
@pytest.mark.parametrize("p_raise", [0.0, 0.5])
def test_protocol_never_deadlocks_and_keeps_buffers_in_turn(ns, p_raise):
    for t, pairs in enumerate(_pair_sequences(ns * 10 + int(p_raise * 10), 40)):
        for seed in range(3):
            assert Model(pairs, ns, p_raise, seed * 1000 + t).run(), (pairs, seed)


def test_merge_shares_equal_blocks_and_keeps_each_list():
    assert merge([0, 2, 5], [1, 2, 3]) == [(0, True, False), (1, False, True), (2, True, True),
                                          (3, False, True), (5, True, False)]
    # out of order: each list still comes out whole and in its own order
    ent = merge([5, 1], [1, 5])
    assert [kb for kb, a, _ in ent if a] == [5, 1] and [kb for kb, _, b in ent if b] == [1, 5]


def test_short_pair_queue_still_completes():
    for seed in range(30):
        assert Model([([0, 1], [1]), ([], [2]), ([3], None), ([0], [0, 4])], 2, 0.3, seed,
                     tq=2).run()


def _caught(bad, pairs, ns, seeds=200):
    caught = 0
    for seed in range(seeds):
        try:
            if not Model(pairs, ns, 0.3, seed, bad={bad}).run():
                caught += 1
        except AssertionError:
            caught += 1
    return caught


def test_late_epilogue_is_caught():
    """An epilogue that read O only after handing over the next tile's first P would
    let that tile's first PV overwrite O before it is read."""
    assert _caught("late_epilogue", [([0, 1, 2], [1]), ([0], [2]), ([1, 2], [0, 1])], 2) > 0


def test_missing_q_free_wait_is_caught():
    """Without the q_free wait the next tile's Q can land while a score MMA of the
    current tile still reads the buffer."""
    assert _caught("no_q_free", [([0, 1], [1, 2]), ([0], [0]), ([2, 3], [1])], 2) > 0


def test_missing_slot_wait_is_caught():
    """Without waiting for the previous use of a ring slot a load can overwrite an
    operand before its MMA has run."""
    assert _caught("no_slot_wait", [([0, 1, 2, 3, 4], [2, 3, 4, 5, 6])], 2) > 0
