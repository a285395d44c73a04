"""Model check of the attention kernel's mbarrier protocol (CPU only).

A small discrete model of the persistent attn_fwd_kernel.cuh: one CTA walking
several query tiles with the TMA producer, the two MMA issuers, the two softmax
groups and the tensor core, connected by mbarriers with phase counters.
Random interleavings (and random "raise the reference max" decisions) are
explored for many tile sequences (empty and short tiles included) and ring
sizes, checking

* that no schedule deadlocks, and
* that every parity wait only ever observes its own phase or the next one
  (a barrier two phases ahead would make `try_wait.parity` lie).

The model follows the kernel's protocol step for step: block J of the CTA's
sequence goes to softmax group and issuer J mod 2; MMA group J is PV_J then
the score MMA of block J + 3, also across a tile boundary when the tile has at
least three blocks (it then feeds the next tile: the next tile's Q and first
K blocks are loaded in its ring stream); a tile whose predecessor is shorter
starts with a prologue group issued by issuer 0 after the predecessor's MMAs;
groups commit on rel[G mod 16], and on rel_v[G mod 16] once their PV MMAs are
issued (a prologue group, which has none, commits it with rel); each issuer
signs a per-tile o_done after its last PV of the tile, which the epilogue waits
for; an issuer waits for its block's P and V slot, issues the PV MMAs, and only
then waits for the K slot (and the next Q when it feeds); the producer waits,
for a ring slot, on rel_v of the group that last read a V block from it and on
rel of the group that last read a K block; an O rescale waits on rel_v of the
latest group of each issuer; Q buffers alternate between non-empty tiles and
come back after each tile's epilogue.  Known-bad
variants (waiting for P of the next block inside the current MMA group; fewer
release barriers than the protocol needs; waiting for ring slots before P) are
checked to fail, so the checker is not vacuous.
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


def plan(tiles):
    """Per non-empty tile: first block J0, tile number k, prologue flag, groups."""
    desc, J0, k, G, prev_n = [], 0, 0, 0, None
    for n in tiles:
        if n == 0:
            continue
        d = dict(n=n, J0=J0, k=k, pro=prev_n is None or prev_n < 3, n0=min(n, 3))
        if d["pro"]:
            d["Gpro"] = G
            G += 1
        d["G0"] = G  # group of block j is G0 + j
        G += n
        desc.append(d)
        J0, k, prev_n = J0 + n, k + 1, n
    for i, d in enumerate(desc):
        d["next"] = desc[i + 1] if i + 1 < len(desc) else None
        d["feeds"] = d["next"] is not None and not d["next"]["pro"]
    return desc


class Model:
    def __init__(self, tiles, ns, p_raise, seed, n_rel=16, bad_next_p=False,
                 bad_slots_first=False):
        self.rng = random.Random(seed)
        self.ns, self.p_raise, self.n_rel = ns, p_raise, n_rel
        self.bad_slots_first = bad_slots_first
        self.bars = {"drain": Bar(2)}
        for i in range(2):
            self.bars[f"q_full{i}"] = Bar()
            self.bars[f"epi{i}"] = Bar()
            self.bars[f"o_done{i}"] = Bar(2)
        for i in range(ns):
            self.bars[f"full{i}"] = Bar()
        for i in range(n_rel):
            self.bars[f"rel{i}"] = Bar()
            self.bars[f"rel_v{i}"] = Bar()
        for i in range(3):
            self.bars[f"s_full{i}"] = Bar()
            self.bars[f"p_full{i}"] = Bar()
        self.desc = plan(tiles)
        self.items = self.ring_items()
        self.pos = {}
        p = 0
        for kind, x, _ in self.items:
            if kind != "Q":
                self.pos[(kind, x)] = p
                p += 1
        self.tc, self.tma, self.passed = [], [], set()
        issuer = self.issuer_bad if bad_next_p else self.issuer
        self.roles = [self.loader(), issuer(0), issuer(1), self.softmax(0), self.softmax(1)]
        self.cur = [next(r) for r in self.roles]

    @staticmethod
    def k_after(d, j):
        """Block whose K follows V_j in the ring, or None."""
        if j + 3 < d["n"]:
            return d["J0"] + j + 3
        if d["feeds"] and j + 3 - d["n"] < d["next"]["n"]:
            return d["J0"] + j + 3
        return None

    def ring_items(self):
        items = []
        for d in self.desc:
            if d["pro"]:
                items.append(("Q", d["k"], None))
                items += [("K", d["J0"] + jj, d["Gpro"]) for jj in range(d["n0"])]
            for j in range(d["n"]):
                g = d["G0"] + j
                items.append(("V", d["J0"] + j, g))
                x = self.k_after(d, j)
                if x is not None:
                    if j + 3 == d["n"]:
                        items.append(("Q", d["next"]["k"], None))
                    items.append(("K", x, g))
        return items

    def rel(self, g):
        return ("wait", f"rel{g % self.n_rel}", g // self.n_rel)

    def rel_v(self, g):
        return ("wait", f"rel_v{g % self.n_rel}", g // self.n_rel)

    def full(self, p):
        return ("wait", f"full{p % self.ns}", p // self.ns)

    def loader(self):
        owner, w = [None] * self.ns, 0
        for kind, x, g in self.items:
            if kind == "Q":
                if x >= 2:
                    yield ("wait", f"epi{x % 2}", (x - 2) // 2)
                yield ("tma", f"q_full{x % 2}")
                continue
            s = w % self.ns
            if owner[s] is not None:
                og, ov = owner[s]
                yield self.rel_v(og) if ov else self.rel(og)
            owner[s] = (g, kind == "V")
            yield ("tma", f"full{s}")
            w += 1
        yield ("end",)

    def prologue(self, d, prev):
        yield ("wait", f"q_full{d['k'] % 2}", d["k"] // 2)
        if prev is not None:
            yield self.rel(prev["G0"] + prev["n"] - 1)
            if prev["n"] >= 2:
                yield self.rel(prev["G0"] + prev["n"] - 2)
        for jj in range(d["n0"]):
            yield self.full(self.pos[("K", d["J0"] + jj)])
            yield ("issue",)
            yield ("commit", f"s_full{(d['J0'] + jj) % 3}")
        yield ("commit", f"rel_v{d['Gpro'] % self.n_rel}")
        yield ("commit", f"rel{d['Gpro'] % self.n_rel}")

    def issuer(self, me):
        prev = None
        for d in self.desc:
            if d["pro"] and me == 0:
                yield from self.prologue(d, prev)
            for j in range(d["n"]):
                X = d["J0"] + j
                if X % 2 != me:
                    continue
                x = self.k_after(d, j)
                if self.bad_slots_first:
                    yield self.full(self.pos[("V", X)])
                    if x is not None:
                        yield self.full(self.pos[("K", x)])
                yield ("wait", f"p_full{X % 3}", X // 3)
                if not self.bad_slots_first:
                    yield self.full(self.pos[("V", X)])
                yield ("issue",)
                if j + 2 >= d["n"]:  # this issuer's last PV of the tile
                    yield ("commit", f"o_done{d['k'] % 2}")
                yield ("commit", f"rel_v{(d['G0'] + j) % self.n_rel}")
                if x is not None:
                    if not self.bad_slots_first:
                        yield self.full(self.pos[("K", x)])
                    if j + 3 >= d["n"]:
                        yield ("wait", f"q_full{d['next']['k'] % 2}", d["next"]["k"] // 2)
                    yield ("issue",)
                    yield ("commit", f"s_full{X % 3}")
                yield ("commit", f"rel{(d['G0'] + j) % self.n_rel}")
            if d["n"] == 1 and d["J0"] % 2 != me:
                yield ("commit", f"o_done{d['k'] % 2}")
            prev = d
        yield ("commit", "drain")
        yield ("wait", "drain", 0)
        yield ("end",)

    def issuer_bad(self, me):
        """Issuer 0 alone, waiting for P_{J+1} inside group J, before the group's
        commits (deadlocks on a raise)."""
        if me == 1:
            for d in self.desc:
                yield ("commit", f"o_done{d['k'] % 2}")
            yield ("commit", "drain")
            yield ("wait", "drain", 0)
            yield ("end",)
            return
        prev = None
        for d in self.desc:
            if d["pro"]:
                yield from self.prologue(d, prev)
            yield ("wait", f"p_full{d['J0'] % 3}", d["J0"] // 3)
            for j in range(d["n"]):
                X = d["J0"] + j
                yield ("issue",)
                if j + 1 == d["n"]:
                    yield ("commit", f"o_done{d['k'] % 2}")
                if j + 1 < d["n"]:
                    yield ("wait", f"p_full{(X + 1) % 3}", (X + 1) // 3)
                yield self.full(self.pos[("V", X)])
                x = self.k_after(d, j)
                if x is not None:
                    yield self.full(self.pos[("K", x)])
                    if j + 3 >= d["n"]:
                        yield ("wait", f"q_full{d['next']['k'] % 2}", d["next"]["k"] // 2)
                    yield ("issue",)
                    yield ("commit", f"s_full{X % 3}")
                yield ("commit", f"rel_v{(d['G0'] + j) % self.n_rel}")
                yield ("commit", f"rel{(d['G0'] + j) % self.n_rel}")
            prev = d
        yield ("commit", "drain")
        yield ("wait", "drain", 0)
        yield ("end",)

    def softmax(self, g):
        for u, d in enumerate(self.desc):
            for j in range(d["n"]):
                X = d["J0"] + j
                if X % 2 != g:
                    continue
                yield ("wait", f"s_full{X % 3}", X // 3)
                if X > 0:
                    yield ("wait", f"p_full{(X - 1) % 3}", (X - 1) // 3)
                if j > 0 and self.rng.random() < self.p_raise:
                    # O rescale: the PVs of the latest group of each issuer must have completed
                    yield self.rel_v(d["G0"] + j - 1)
                    if j > 1:
                        yield self.rel_v(d["G0"] + j - 2)
                yield ("arrive", f"p_full{X % 3}")
            # epilogue: every PV of the tile has completed (o_done), then a named
            # barrier of both groups, then the Q buffer goes back to the producer
            yield ("wait", f"o_done{d['k'] % 2}", d["k"] // 2)
            yield ("bar", u)
            if g == 0:
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

    def run(self, max_steps=500000):
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
    seqs += [[0, 0], [1, 1, 1, 1, 1], [2, 0, 2, 0, 2], [3, 21, 3, 21], [3, 3, 3, 3],
             [21, 1, 21, 2, 21, 3, 21], [4, 0, 0, 5, 2, 3]]
    for _ in range(count):
        seqs.append([rng.choice([0, 1, 2, 3, 4, 5, 7, 9, 15, 21]) for _ in range(rng.randint(2, 8))])
    return seqs


@pytest.mark.parametrize("ns", [5, 12])
@pytest.mark.parametrize("p_raise", [0.0, 0.3, 1.0])
def test_protocol_never_deadlocks(ns, p_raise):
    for t, tiles in enumerate(_tile_sequences(ns * 10 + int(p_raise * 10), 80)):
        for seed in range(4):
            assert Model(tiles, ns, p_raise, seed * 1000 + t).run(), (tiles, seed)


def test_fed_and_prologue_tiles():
    desc = plan([21, 2, 5, 0, 3, 1])
    assert [d["pro"] for d in desc] == [True, False, True, False, False]
    assert [d["feeds"] for d in desc] == [True, False, True, True, False]


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


def test_longest_first_orders():
    """The kernel can take its tiles in a given order (longest list first within
    each wave, dealt in a serpentine over the CTAs), so a CTA's sequence of list
    lengths can have any shape; the extreme ones, falling (with empty tiles last)
    and rising, run clean, as do the random sequences of the other tests."""
    rng = random.Random(11)
    for t in range(40):
        tiles = [rng.choice([0, 0, 1, 2, 3, 4, 6, 9]) for _ in range(rng.randint(2, 8))]
        for seq in (sorted(tiles, reverse=True), sorted(tiles)):
            for ns in (5, 6):
                assert Model(seq, ns, 0.3, t).run(), (seq, ns)
