"""Model check of the attention kernel's mbarrier protocol (CPU only).

A small discrete model of the persistent attn_fwd_kernel.cuh: one CTA walking
several query tiles with the TMA producer, the two MMA issuers, the two softmax
groups and the tensor core, connected by mbarriers with phase counters.
Random interleavings (and random "raise the reference max" decisions) are
explored for many tile sequences (empty tiles included) and ring sizes,
checking

* that no schedule deadlocks, and
* that every parity wait only ever observes its own phase or the next one
  (a barrier two phases ahead would make `try_wait.parity` lie).

The model follows the kernel's protocol step for step: block J of the CTA's
sequence goes to softmax group and issuer J mod 2, a tile's prologue group
(its first score MMAs) is issued by issuer 0 after the previous tile's MMAs,
MMA group G commits on rel[G mod 16], an issuer waits for its block's P
before the block's V and K ring slots (a slot may be two loads behind before
then), the producer waits for the group that last used a ring slot, and Q
buffers alternate between non-empty tiles with an epilogue hand-back.  Known-bad variants (waiting for P of the next block
inside the current MMA group; fewer release barriers than the protocol needs;
waiting for the ring slots before P) are checked to fail, so the checker is
not vacuous.
"""
import random

import pytest


class Bar:
    def __init__(self, count=1):
        self.count, self.arr, self.done = count, 0, 0

    def arrive(self):
        self.arr += 1
        if self.arr == self.count:
            self.arr = 0
            self.done += 1


class Model:
    def __init__(self, tiles, ns, p_raise, seed, n_rel=16, bad_next_p=False, bad_slots_first=False):
        self.rng = random.Random(seed)
        self.ns, self.p_raise, self.n_rel = ns, p_raise, n_rel
        self.bars = {"drain": Bar(2)}
        for i in range(2):
            self.bars[f"q_full{i}"] = Bar()
            self.bars[f"epi{i}"] = Bar()
        for i in range(ns):
            self.bars[f"full{i}"] = Bar()
        for i in range(n_rel):
            self.bars[f"rel{i}"] = Bar()
        for i in range(3):
            self.bars[f"s_full{i}"] = Bar()
            self.bars[f"p_full{i}"] = Bar()
        # per-tile sequence counters, as the kernel's cursor advances them
        self.desc = []
        J0 = pos0 = k = 0
        for n in tiles:
            n0, nk = min(n, 3), max(n - 3, 0)
            self.desc.append(dict(n=n, J0=J0, pos0=pos0, k=k, n0=n0, nk=nk))
            if n > 0:
                J0, pos0, k = J0 + n, pos0 + n0 + n + nk, k + 1
        self.tc, self.tma, self.passed = [], [], set()
        self.bad_slots_first = bad_slots_first
        issuer = self.issuer_bad if bad_next_p else self.issuer
        self.roles = [self.loader(), issuer(0), issuer(1), self.softmax(0), self.softmax(1)]
        self.cur = [next(r) for r in self.roles]

    @staticmethod
    def pos_v(d, j):
        return d["pos0"] + d["n0"] + j + min(j, d["nk"])

    @staticmethod
    def group(d, j):  # MMA group of block j of tile d
        return d["J0"] + d["k"] + 1 + j

    @staticmethod
    def prologue_group(d):
        return d["J0"] + d["k"]

    def rel(self, g):
        return ("wait", f"rel{g % self.n_rel}", g // self.n_rel)

    def full(self, p):
        return ("wait", f"full{p % self.ns}", p // self.ns)

    def loader(self):
        owner = [None] * self.ns  # group that frees each slot
        w = 0
        for d in self.desc:
            if d["n"] == 0:
                continue
            k = d["k"]
            if k >= 2:
                yield ("wait", f"epi{k % 2}", (k - 2) // 2)
            yield ("tma", f"q_full{k % 2}")
            items = [self.prologue_group(d)] * d["n0"]
            for j in range(d["n"]):
                items.append(self.group(d, j))  # V_j
                if j + 3 < d["n"]:
                    items.append(self.group(d, j))  # K_{j+3}
            for g in items:
                s = w % self.ns
                if owner[s] is not None:
                    yield self.rel(owner[s])
                owner[s] = g
                yield ("tma", f"full{s}")
                w += 1
        yield ("end",)

    def prologue(self, d, prev):
        yield ("wait", f"q_full{d['k'] % 2}", d["k"] // 2)
        if prev is not None:
            yield self.rel(self.group(prev, prev["n"] - 1))
            if prev["n"] >= 2:
                yield self.rel(self.group(prev, prev["n"] - 2))
        for jj in range(d["n0"]):
            yield self.full(d["pos0"] + jj)
            yield ("issue",)
            yield ("commit", f"s_full{(d['J0'] + jj) % 3}")
        yield ("commit", f"rel{self.prologue_group(d) % self.n_rel}")

    def issuer(self, me):
        prev = None
        for d in self.desc:
            n = d["n"]
            if n == 0:
                continue
            if me == 0:
                yield from self.prologue(d, prev)
            for j in range(n):
                J = d["J0"] + j
                if J % 2 != me:
                    continue
                pv = self.pos_v(d, j)
                if not self.bad_slots_first:
                    yield ("wait", f"p_full{J % 3}", J // 3)
                yield self.full(pv)
                if j + 3 < n:
                    yield self.full(pv + 1)
                if self.bad_slots_first:
                    yield ("wait", f"p_full{J % 3}", J // 3)
                yield ("issue",)
                if j + 3 < n:
                    yield ("issue",)
                    yield ("commit", f"s_full{J % 3}")
                yield ("commit", f"rel{self.group(d, j) % self.n_rel}")
            prev = d
        yield ("commit", "drain")
        yield ("wait", "drain", 0)
        yield ("end",)

    def issuer_bad(self, me):
        """Issuer 0 alone, waiting for P_{J+1} inside group J (deadlocks on a raise)."""
        if me == 1:
            yield ("commit", "drain")
            yield ("wait", "drain", 0)
            yield ("end",)
            return
        prev = None
        for d in self.desc:
            n = d["n"]
            if n == 0:
                continue
            yield from self.prologue(d, prev)
            yield ("wait", f"p_full{d['J0'] % 3}", d["J0"] // 3)
            for j in range(n):
                J = d["J0"] + j
                yield ("issue",)
                if j + 1 < n:
                    yield ("wait", f"p_full{(J + 1) % 3}", (J + 1) // 3)
                pv = self.pos_v(d, j)
                yield self.full(pv)
                if j + 3 < n:
                    yield self.full(pv + 1)
                    yield ("issue",)
                    yield ("commit", f"s_full{J % 3}")
                yield ("commit", f"rel{self.group(d, j) % self.n_rel}")
            prev = d
        yield ("commit", "drain")
        yield ("wait", "drain", 0)
        yield ("end",)

    def softmax(self, g):
        for u, d in enumerate(self.desc):
            n = d["n"]
            for j in range(n):
                J = d["J0"] + j
                if J % 2 != g:
                    continue
                yield ("wait", f"s_full{J % 3}", J // 3)
                if J > 0:
                    yield ("wait", f"p_full{(J - 1) % 3}", (J - 1) // 3)
                if j > 0 and self.rng.random() < self.p_raise:
                    # O rescale: the latest group of each issuer must have completed
                    yield self.rel(self.group(d, j - 1))
                    if j > 1:
                        yield self.rel(self.group(d, j - 2))
                yield ("arrive", f"p_full{J % 3}")
            if n > 0:  # epilogue: every MMA of the tile has completed
                yield self.rel(self.group(d, n - 1))
                if n >= 2:
                    yield self.rel(self.group(d, n - 2))
            yield ("bar", u)  # 256-thread named barrier of both groups
            if g == 0 and n > 0:
                yield ("arrive", f"epi{d['k'] % 2}")
        yield ("end",)

    def ready(self, i, op):
        if op[0] == "bar":
            other = 4 if i == 3 else 3
            o = self.cur[other]
            return (o[0] == "bar" and o[1] == op[1]) or (other, op[1]) in self.passed
        if op[0] != "wait":
            return True
        done = self.bars[op[1]].done
        assert op[2] <= done <= op[2] + 1, f"parity ambiguity on {op[1]}: phase {op[2]}, done {done}"
        return done == op[2] + 1

    def run(self, max_steps=400000):
        for _ in range(max_steps):
            live = [i for i, op in enumerate(self.cur) if op[0] != "end"]
            if not live and not self.tc and not self.tma:
                return True
            choices = [("role", i) for i in live if self.ready(i, self.cur[i])]
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
            elif kind == "tma":
                self.bars[self.tma.pop(self.rng.randrange(len(self.tma)))].arrive()
            else:
                op = self.cur[i]
                if op[0] == "tma":
                    self.tma.append(op[1])
                elif op[0] in ("issue", "commit"):
                    self.tc.append(op)
                elif op[0] == "arrive":
                    self.bars[op[1]].arrive()
                elif op[0] == "bar":
                    self.passed.add((i, op[1]))
                self.cur[i] = next(self.roles[i])
        raise AssertionError("model did not finish")


def _tile_sequences(seed, count):
    rng = random.Random(seed)
    seqs = [[n] for n in list(range(0, 26)) + [41, 83]]
    seqs += [[0, 0], [1, 1, 1, 1, 1], [2, 0, 2, 0, 2], [3, 21, 3, 21]]
    for _ in range(count):
        seqs.append([rng.choice([0, 1, 2, 3, 4, 5, 7, 9, 15, 21]) for _ in range(rng.randint(2, 7))])
    return seqs


@pytest.mark.parametrize("ns", [5, 12])
@pytest.mark.parametrize("p_raise", [0.0, 0.3, 1.0])
def test_protocol_never_deadlocks(ns, p_raise):
    for t, tiles in enumerate(_tile_sequences(ns * 10 + int(p_raise * 10), 60)):
        for seed in range(4):
            assert Model(tiles, ns, p_raise, seed * 1000 + t).run(), (tiles, seed)


def test_known_bad_next_p_wait_is_caught():
    failures = sum(not Model([n], 5, 0.5, seed, bad_next_p=True).run()
                   for n in range(4, 16) for seed in range(10))
    assert failures > 0


def test_too_few_release_barriers_is_caught():
    caught = 0
    for seed in range(200):
        try:
            Model([21, 21, 21], 12, 0.3, seed, n_rel=4).run()
        except AssertionError as e:
            assert "parity ambiguity" in str(e)
            caught += 1
    assert caught > 0


def test_ring_wait_before_p_is_caught():
    """Waiting for a block's ring slots before its P can see a slot two loads
    behind (parity ambiguity) at the start of a sequence."""
    caught = 0
    for seed in range(100):
        try:
            Model([9, 9], 5, 0.3, seed, bad_slots_first=True).run()
        except AssertionError as e:
            assert "parity ambiguity" in str(e)
            caught += 1
    assert caught > 0
