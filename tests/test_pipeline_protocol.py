"""Model check of the attention kernel's mbarrier protocol (CPU only).

A small discrete model of attn_fwd_kernel.cuh: the TMA producer, the two MMA
issuers, the two softmax groups and the tensor core, connected by mbarriers
with phase counters.  Random interleavings (and random "raise the reference
max" decisions) are explored for many list lengths and ring sizes, checking

* that no schedule deadlocks, and
* that every parity wait only ever observes its own phase or the next one
  (a barrier two phases ahead would make `try_wait.parity` lie).

The model must follow the kernel's protocol step for step; a known-bad
variant (waiting for P of the next block inside the current MMA group, which
deadlocks with a rescale) is checked to fail, so the checker is not vacuous.
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
    def __init__(self, n, ns, p_raise, seed, bad_variant=False):
        self.rng = random.Random(seed)
        self.n, self.ns, self.p_raise = n, ns, p_raise
        self.n0, self.nk = min(n, 3), max(n - 3, 0)
        self.bars = {"q_full": Bar(), "pro_done": Bar(), "o_done": Bar(2), "drain": Bar(2)}
        for i in range(ns):
            self.bars[f"full{i}"] = Bar()
        for i in range(8):
            self.bars[f"rel{i}"] = Bar()
        for i in range(3):
            self.bars[f"s_full{i}"] = Bar()
            self.bars[f"p_full{i}"] = Bar()
        self.tc, self.tma = [], []
        issuers = ([self.issuer_bad()] if bad_variant else [self.issuer(0), self.issuer(1)])
        if bad_variant:
            self.bars["o_done"].count = 1
            self.bars["drain"].count = 1
        self.roles = [self.loader(), *issuers, self.softmax(0), self.softmax(1)]
        self.cur = [next(r) for r in self.roles]

    # ring layout: K_0..K_{n0-1}, then V_j and (j + 3 < n) K_{j+3}
    def pos_v(self, j):
        return self.n0 + j + min(j, self.nk)

    def ring_block(self, p):
        q = p - self.n0
        return q >> 1 if q < 2 * self.nk else self.nk + (q - 2 * self.nk)

    def wait_pos(self, p):
        return ("wait", f"full{p % self.ns}", p // self.ns)

    def loader(self):
        yield ("tma", "q_full")
        w = 0
        order = [None] * self.n0
        for j in range(self.n):
            order.append(None)
            if j + 3 < self.n:
                order.append(None)
        for _ in order:
            if w >= self.ns:
                prev = w - self.ns
                if prev < self.n0:
                    yield ("wait", "pro_done", 0)
                else:
                    jb = self.ring_block(prev)
                    yield ("wait", f"rel{jb % 8}", jb // 8)
            yield ("tma", f"full{w % self.ns}")
            w += 1
        yield ("end",)

    def issuer(self, me):
        n = self.n
        if n == 0:
            yield ("end",)
            return
        if me == 0:
            yield ("wait", "q_full", 0)
            for jj in range(self.n0):
                yield self.wait_pos(jj)
                yield ("issue",)
                yield ("commit", f"s_full{jj}")
            yield ("commit", "pro_done")
        for j in range(me, n, 2):
            yield ("wait", f"p_full{j % 3}", j // 3)
            pv = self.pos_v(j)
            yield self.wait_pos(pv)
            if j + 3 < n:
                yield self.wait_pos(pv + 1)
            yield ("issue",)
            if j + 3 < n:
                yield ("issue",)
                yield ("commit", f"s_full{j % 3}")
            yield ("commit", f"rel{j % 8}")
        yield ("commit", "o_done")
        yield ("commit", "drain")
        yield ("wait", "drain", 0)
        yield ("end",)

    def issuer_bad(self):
        """Single issuer that waits for P_{j+1} inside group j (deadlocks on a raise)."""
        n = self.n
        if n == 0:
            yield ("end",)
            return
        yield ("wait", "q_full", 0)
        for jj in range(self.n0):
            yield self.wait_pos(jj)
            yield ("issue",)
            yield ("commit", f"s_full{jj}")
        yield ("commit", "pro_done")
        yield ("wait", "p_full0", 0)
        for j in range(n):
            yield ("issue",)
            if j + 1 < n:
                yield ("wait", f"p_full{(j + 1) % 3}", (j + 1) // 3)
            pv = self.pos_v(j)
            yield self.wait_pos(pv)
            if j + 3 < n:
                yield self.wait_pos(pv + 1)
                yield ("issue",)
                yield ("commit", f"s_full{j % 3}")
            yield ("commit", f"rel{j % 8}")
        yield ("commit", "o_done")
        yield ("commit", "drain")
        yield ("wait", "drain", 0)
        yield ("end",)

    def softmax(self, g):
        n = self.n
        for j in range(g, n, 2):
            yield ("wait", f"s_full{j % 3}", j // 3)
            if j > 0:
                yield ("wait", f"p_full{(j - 1) % 3}", (j - 1) // 3)
                if self.rng.random() < self.p_raise:
                    # O rescale: the latest group of each issuer must have completed
                    yield ("wait", f"rel{(j - 1) % 8}", (j - 1) // 8)
                    if j > 1:
                        yield ("wait", f"rel{(j - 2) % 8}", (j - 2) // 8)
            yield ("arrive", f"p_full{j % 3}")
        if n > 0:
            yield ("wait", "o_done", 0)
        yield ("end",)

    def ready(self, op):
        if op[0] != "wait":
            return True
        done = self.bars[op[1]].done
        assert op[2] <= done <= op[2] + 1, f"parity ambiguity on {op[1]}: phase {op[2]}, done {done}"
        return done == op[2] + 1

    def run(self, max_steps=200000):
        for _ in range(max_steps):
            live = [i for i, op in enumerate(self.cur) if op[0] != "end"]
            if not live and not self.tc and not self.tma:
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
                self.cur[i] = next(self.roles[i])
        raise AssertionError("model did not finish")


@pytest.mark.parametrize("ns", [6, 12])
@pytest.mark.parametrize("p_raise", [0.0, 0.3, 1.0])
def test_protocol_never_deadlocks(ns, p_raise):
    for n in list(range(0, 26)) + [41, 83]:
        for seed in range(12):
            assert Model(n, ns, p_raise, seed).run(), (n, seed)


def test_known_bad_protocol_is_caught():
    failures = sum(not Model(n, 6, 0.5, seed, bad_variant=True).run()
                   for n in range(4, 16) for seed in range(10))
    assert failures > 0
