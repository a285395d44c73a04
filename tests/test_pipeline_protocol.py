"""Model check of the attention kernel's mbarrier protocol (CPU only).

A small discrete model of the persistent attn_fwd_kernel.cuh: one CTA claiming
pairs of query tiles (two streams, one tile each) that share one K/V stream:
the TMA producer, the MMA issuer and four softmax warps per stream, with the
tensor core and the TMA engine, connected by mbarriers with phase counters.
Random interleavings (either stream's MMA group first when both are ready, TMA
loads landing in any order, random "raise the reference max" decisions) are explored
for many pair sequences (empty lists, missing second tiles, one-block tiles,
disjoint and overlapping lists, lists out of order) and ring sizes, checking

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
publishes it in the pair queue for the softmax warps, loads each stream's Q once
that stream's previous tile's last score MMA is complete (q_free), and loads
ring items in the order K of the first merged entry, then per entry: V and the
K of the next entry, each into slot (item mod NS) once the MMAs that read the
slot's previous item are complete, with flags saying which streams use the
item and whether it is a stream's first or last score / PV item of its tile;
a final item marks the end.  The issuer takes a V item together with the K item
after it and, for each stream that uses them, as soon as that stream's P (and,
for a tile's first score MMA, its Q) is ready, issues the stream's group: PV on
V [o_done after the tile's last], S on K [q_free after the tile's last;
s_full]; a K item alone (a pair's first) waits for the previous block's P when
no PV did.  Then it releases both slots.  Each softmax
warp waits s_full(J), may rescale O, writes P and arrives on p_full; after a
tile's last block it waits o_done and reads O, before it can arrive on p_full
for its next tile's first block.  Known-bad variants (the epilogue's O read
deferred past the next tile's first block, no q_free wait, no wait for the
previous use of a ring slot, releasing a slot before the MMA that reads it)
are checked to be caught, so the checker is not vacuous.
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
        self.tc = []  # the issuer's tensor-core queue (in order)
        self.tma = []
        self.roles = [self.producer(), self.issuer()]
        for s in (0, 1):
            for w in range(N_WARPS):
                self.roles.append(self.softmax(s, w))
        self.cur = [next(r) for r in self.roles]

    def slot_kb(self, item):
        return self.item_kb[item]

    def lists(self, p):
        l0, l1 = self.pairs[p]
        return [l0 or [], l1 or []]

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
            n = [len(ls[0]), len(ls[1])]
            ns_, nv = [0, 0], [0, 0]

            def flags(kind, ins, cnt, tot):
                f = {"kind": kind, "use": [False, False], "first": [False, False],
                     "last": [False, False]}
                for s in (0, 1):
                    if ins[s]:
                        f["use"][s] = True
                        f["first"][s] = cnt[s] == 0
                        cnt[s] += 1
                        f["last"][s] = cnt[s] == tot[s]
                return f

            yield from load(ent[0][0], flags("K", ent[0][1:], ns_, n))
            for u, (kb, a0, a1) in enumerate(ent):
                yield from load(kb, flags("V", (a0, a1), nv, n))
                if u + 1 < len(ent):
                    yield from load(ent[u + 1][0], flags("K", ent[u + 1][1:], ns_, n))
        yield from load(None, {"kind": "end"})
        yield ("end",)

    def issuer(self):
        """The single issuer: a V item together with the K item after it; each stream's
        group [PV on V, S on K] as soon as that stream is ready, in either order."""
        items = 0
        J, k, kpv = [0, 0], [0, 0], [0, 0]
        pp = [False, False]

        def next_item():
            nonlocal items
            i = items % self.ns
            yield ("wait", ("full", i), items // self.ns)
            it = items
            items += 1
            return i, it, self.meta[it]

        end = False
        while not end:
            i1, it1, m1 = yield from next_item()
            if m1["kind"] == "end":
                break
            v = k_ = None
            if m1["kind"] == "V":
                v = (i1, it1, m1)
                i2, it2, m2 = yield from next_item()
                if m2["kind"] == "end":
                    end = True
                else:
                    k_ = (i2, it2, m2)
            else:
                k_ = (i1, it1, m1)
            todo = [s for s in (0, 1) if (v and v[2]["use"][s]) or (k_ and k_[2]["use"][s])]
            while todo:
                # the streams whose group can go now (P and Q ready); the model lets any
                # ready stream go first
                ready = []
                for s in todo:
                    use_v = v is not None and v[2]["use"][s]
                    use_k = k_ is not None and k_[2]["use"][s]
                    need = []
                    if use_v or (use_k and pp[s]):
                        need.append(((s, "p_full"), J[s]))
                    if use_k and k_[2]["first"][s]:
                        need.append(((s, "q_full"), k[s]))
                    if all(self.ready(("wait", b, ph)) for b, ph in need):
                        ready.append(s)
                if not ready:
                    yield ("poll",)
                    continue
                s = self.rng.choice(ready)
                todo.remove(s)
                use_v = v is not None and v[2]["use"][s]
                use_k = k_ is not None and k_[2]["use"][s]
                if use_v or (use_k and pp[s]):
                    J[s] += 1
                    pp[s] = False
                if use_v:
                    i, it, m = v
                    yield ("mma", ("PV", s, J[s] - 1, (s, kpv[s]), i, it, m["first"][s],
                                   self.slot_kb(it)))
                    if m["last"][s]:
                        yield ("commit", (s, "o_done"))
                        kpv[s] += 1
                if use_k:
                    i, it, m = k_
                    yield ("mma", ("S", s, J[s], (s, k[s]), i, it, self.slot_kb(it)))
                    if m["last"][s]:
                        yield ("commit", (s, "q_free"))
                        k[s] += 1
                    yield ("commit", (s, "s_full"))
                    pp[s] = True
            if v is not None:
                if "early_release" in self.bad:
                    yield ("arrive", ("empty", v[0]))
                else:
                    yield ("commit", ("empty", v[0]))
            if k_ is not None:
                yield ("commit", ("empty", k_[0]))
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
                elif op[0] not in ("wait", "poll"):
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
    assert _caught("no_q_free", [([0, 1], [1, 2]), ([0], [0]), ([2, 3], [1])], 4) > 0


def test_missing_slot_wait_is_caught():
    """Without waiting for the previous use of a ring slot a load can overwrite an
    operand before its MMA has run."""
    assert _caught("no_slot_wait", [([0, 1, 2, 3, 4], [2, 3, 4, 5, 6])], 2) > 0


def test_release_before_the_mma_is_caught():
    """An issuer that released a V slot with a plain arrival (instead of a commit that
    fires when its PV has read the slot) would let the next load overwrite V early."""
    assert _caught("early_release", [([0, 1, 2, 3, 4], [1, 2, 3, 4, 5])], 2) > 0
