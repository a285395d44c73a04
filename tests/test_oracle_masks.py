"""Pins for the oracle's mask builders: CSLA, CS4A selection and index mapping.

Pinned against hand-derived fixtures under tests/golden/, an exact-rational
restatement of the mapping on token level, and invariants that the method's
description fixes (sinks always kept, own token always kept, radius >= side is
dense, mapping identity, ranges, monotonicity).
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from block_sparse_cross_sparvar_b200 import inputs
from oracle import sparvar_oracle as orc
from tests.conftest import GOLDEN

INF_SIDES = (1, 2, 4, 6, 8, 12, 16, 20, 24, 32, 40, 48, 64)


def _read_csla_cases():
    cases = []
    for line in open(os.path.join(GOLDEN, "csla_tiny.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        if line.startswith("case"):
            parts = line.split()
            kv = dict(p.split("=") for p in parts[2:])
            cases.append(dict(sides=tuple(int(x) for x in kv["sides"].split(",")),
                              q_scale=int(kv["q_scale"]), n_sink=int(kv["n_sink"]),
                              r_prev=int(kv["r_prev"]), r_own=int(kv["r_own"]), rows={}))
        else:
            head, keys = line.split(":")
            cases[-1]["rows"][int(head.split()[1])] = [int(x) for x in keys.split()]
    return cases


@pytest.mark.parametrize("case", _read_csla_cases(), ids=lambda c: f"{c['sides']}-{c['r_prev']}-{c['r_own']}")
def test_csla_token_mask_golden(case):
    T = orc.csla_token_mask(case["sides"], case["q_scale"], case["n_sink"], case["r_prev"], case["r_own"])
    for q, keys in case["rows"].items():
        assert list(np.nonzero(T[q])[0]) == keys, q


def test_csla_block_aggregation_golden():
    cnt, idx, blk = orc.build_csla_mask((1, 2, 4), 2, 1, 0, 0, 4, 4)
    want = {}
    for line in open(os.path.join(GOLDEN, "csla_tiny_blocks.txt")):
        if line.startswith("qb"):
            head, keys = line.split(":")
            want[int(head.split()[1])] = [int(x) for x in keys.split()]
    assert blk.shape == (4, 6)
    for qb, kbs in want.items():
        assert list(np.nonzero(blk[qb])[0]) == kbs
        assert cnt[qb] == len(kbs)
        assert list(idx[qb, :cnt[qb]]) == kbs and np.all(idx[qb, cnt[qb]:] == -1)


@pytest.mark.parametrize("sides,k,n_sink", [((1, 2, 4, 8, 16), 4, 2), (INF_SIDES, 9, 5), ((1, 3, 5, 7), 3, 1)])
def test_csla_invariants(sides, k, n_sink):
    off = orc.scale_offsets(sides)
    T = orc.csla_token_mask(sides, k, n_sink, 1, 2)
    sk = sides[k]
    # sink keys kept for every query
    assert T[:, :off[n_sink]].all()
    # every query keeps its own token
    assert T[np.arange(sk * sk), off[k] + np.arange(sk * sk)].all()
    # nothing beyond the prefix
    assert T.shape == (sk * sk, off[k + 1])
    # radius >= largest side keeps everything
    Td = orc.csla_token_mask(sides, k, n_sink, max(sides), max(sides))
    assert Td.all()
    # monotone in the radius
    T2 = orc.csla_token_mask(sides, k, n_sink, 2, 3)
    assert np.all(T2 >= T)
    # per query, kept keys of each non-sink earlier scale form a (2r+1)^2 window clipped to the grid
    for m in range(n_sink, k):
        sm = sides[m]
        w = T[:, off[m]:off[m + 1]].sum(axis=1)
        assert w.min() >= min(2, sm) ** 2 and w.max() <= min(3, sm) ** 2


def test_csla_blocks_match_tokenwise_or():
    sides = INF_SIDES
    T = orc.csla_token_mask(sides, 10, 5, 2, 4)
    blk = orc.aggregate_to_blocks(T, 128, 128)
    nq, L = T.shape
    rng = np.random.default_rng(0)
    for _ in range(200):
        qb = rng.integers(blk.shape[0])
        kb = rng.integers(blk.shape[1])
        tile = T[qb * 128:(qb + 1) * 128, kb * 128:(kb + 1) * 128]
        assert blk[qb, kb] == bool(tile.any())
    # sink block 0 always kept
    assert blk[:, 0].all()


# ---------------------------------------------------------------- CS4A selection
def test_select_golden():
    for line in open(os.path.join(GOLDEN, "select_mass.txt")):
        if not line.startswith("tau"):
            continue
        a, b, c = line.split("|")
        tau = float(a.split()[1])
        M = np.array([[float(x) for x in b.split()]])
        want = [int(x) for x in c.split()]
        blk, margin = orc.select_blocks_by_mass(M, tau)
        assert list(np.nonzero(blk[0])[0]) == want, line


def test_select_topk_golden():
    for line in open(os.path.join(GOLDEN, "select_topk.txt")):
        if not line.startswith("ratio"):
            continue
        a, b, c = line.split("|")
        ratio = float(a.split()[1])
        M = np.array([[float(x) for x in b.split()]])
        want = [int(x) for x in c.split()]
        blk, margin = orc.select_blocks_topk(M, ratio)
        assert list(np.nonzero(blk[0])[0]) == want, line


@pytest.mark.parametrize("ratio,nkb,k", [(0.2, 20, 4), (np.float32(0.2), 20, 4), (0.2, 83, 17),
                                         (0.2, 51, 11), (0.2, 5, 1), (0.2, 1, 1), (1e-9, 40, 1),
                                         (1.0, 33, 33), (0.5, 7, 4), (0.25, 8, 2)])
def test_topk_count(ratio, nkb, k):
    assert orc.topk_count(float(ratio), nkb) == k


def test_topk_special_cases_and_order():
    q, k = _rand(6, 64, 16), _rand(7, 100, 16)
    M = orc.decision_block_mass(q, k, 16, 16)
    blk1, _ = orc.select_blocks_topk(M, 1e-9)
    assert np.array_equal(np.nonzero(blk1)[1], np.argmax(M, axis=1))
    blk_all, margin = orc.select_blocks_topk(M, 1.0)
    assert blk_all.all() and np.isinf(margin).all()
    blk, margin = orc.select_blocks_topk(M, 0.3)
    kk = orc.topk_count(0.3, M.shape[1])
    for qb in range(M.shape[0]):
        assert blk[qb].sum() == kk
        # every kept block is at least as heavy as every dropped one, by the margin
        assert M[qb][blk[qb]].min() - M[qb][~blk[qb]].max() == pytest.approx(margin[qb])
        assert margin[qb] >= 0
    # the mass rule's set for a row is the Top-K set with k = its size
    blk_m, _ = orc.select_blocks_by_mass(M, 0.8)
    for qb in range(M.shape[0]):
        n = int(blk_m[qb].sum())
        bk, _ = orc.select_blocks_topk(M[qb:qb + 1], (n - 0.5) / M.shape[1])
        assert np.array_equal(bk[0], blk_m[qb])


def _rand(seed, *shape):
    return np.random.default_rng(seed).standard_normal(shape)


def test_mass_uniform_closed_form():
    # q = 0 gives uniform attention: M[qb, kb] = n_k(kb) / L
    q = np.zeros((50, 8))
    k = _rand(1, 70, 8)
    M = orc.decision_block_mass(q, k, 16, 16)
    want = np.array([min(16, 70 - kb * 16) / 70 for kb in range(5)])
    np.testing.assert_allclose(M, want[None].repeat(4, 0), atol=1e-15)


def test_mass_rows_sum_to_one_and_bruteforce():
    q, k = _rand(2, 11, 4), _rand(3, 17, 4)
    M = orc.decision_block_mass(q, k, 4, 5, scale=0.9)
    np.testing.assert_allclose(M.sum(axis=1), 1.0, atol=1e-14)
    for qb in range(M.shape[0]):
        rows = range(qb * 4, min(qb * 4 + 4, 11))
        for kb in range(M.shape[1]):
            tot = 0.0
            for i in rows:
                s = [0.9 * sum(q[i][d] * k[j][d] for d in range(4)) for j in range(17)]
                mx = max(s)
                z = sum(math.exp(x - mx) for x in s)
                tot += sum(math.exp(s[j] - mx) for j in range(kb * 5, min(kb * 5 + 5, 17))) / z
            assert abs(M[qb, kb] - tot / len(rows)) < 1e-13


def test_mass_concentrated_key():
    # one key whose score dominates every row -> its block holds ~all the mass
    q = np.ones((16, 4)) * 10.0
    k = np.zeros((40, 4))
    k[27] = 10.0
    M = orc.decision_block_mass(q, k, 8, 8)
    assert np.all(M[:, 3] > 1 - 1e-12)


def test_decide_thresholds():
    q, k = _rand(4, 64, 16), _rand(5, 100, 16)
    _, _, blk_all, M, _ = orc.decide_blocks(q, k, 16, 16, 2.0)
    assert blk_all.all()
    _, _, blk_one, _, _ = orc.decide_blocks(q, k, 16, 16, 1e-9)
    assert np.all(blk_one.sum(1) == 1)
    assert np.all(np.argmax(M, axis=1) == np.nonzero(blk_one)[1])
    cnt, idx, blk, M, margin = orc.decide_blocks(q, k, 16, 16, 0.95)
    for qb in range(blk.shape[0]):
        assert M[qb][blk[qb]].sum() >= 0.95
        # dropping the smallest kept block falls below the threshold
        kept = np.sort(M[qb][blk[qb]])
        assert kept[1:].sum() < 0.95
        # every dropped block is no heavier than every kept block
        if (~blk[qb]).any():
            assert M[qb][~blk[qb]].max() <= kept[0]


def test_decide_head_permutation():
    qs = [_rand(10 + h, 32, 8) for h in range(3)]
    ks = [_rand(20 + h, 48, 8) for h in range(3)]
    res = [orc.decide_blocks(qs[h], ks[h], 8, 8, 0.9)[2] for h in range(3)]
    perm = [2, 0, 1]
    res_p = [orc.decide_blocks(qs[p], ks[p], 8, 8, 0.9)[2] for p in perm]
    for i, p in enumerate(perm):
        assert np.array_equal(res_p[i], res[p])


# ---------------------------------------------------------------- CS4A mapping
def _read_map_cases():
    cases = []
    for line in open(os.path.join(GOLDEN, "map_indices_tiny.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        if line.startswith("case"):
            p = line.split()
            cases.append(dict(args=tuple(int(x) for x in p[2:]), src=[], dst={}))
        elif line.startswith("src"):
            _, a, b = line.split()
            cases[-1]["src"].append((int(a), int(b)))
        else:
            head, kbs = line.split(":")
            cases[-1]["dst"][int(head.split()[1])] = [int(x) for x in kbs.split()]
    return cases


@pytest.mark.parametrize("case", _read_map_cases())
def test_map_golden(case):
    src_nq, src_lkv, dst_nq, dst_lkv, bq, bk, n_sink = case["args"]
    src = np.zeros((orc.n_blocks(src_nq, bq), orc.n_blocks(src_lkv, bk)), dtype=bool)
    for a, b in case["src"]:
        src[a, b] = True
    dst = orc.map_block_mask(src, src_nq, src_lkv, dst_nq, dst_lkv, bq, bk, n_sink)
    for qb, kbs in case["dst"].items():
        assert list(np.nonzero(dst[qb])[0]) == kbs


def _covered_tokens_exact(lo, hi, n_src, n_dst):
    """Destination tokens t whose unit cell [t, t+1), carried back to source
    coordinates by the ratio n_src/n_dst, overlaps the source interval [lo, hi)."""
    r = Fraction(n_dst, n_src)
    return [t for t in range(n_dst) if Fraction(t) < hi * r and Fraction(t + 1) > lo * r]


@pytest.mark.parametrize("geom", [(9, 30, 25, 61, 4, 8, 3), (1024, 2521, 4096, 10521, 128, 128, 121),
                                  (1024, 2521, 1600, 4121, 128, 128, 121), (7, 11, 13, 29, 2, 3, 0)])
def test_map_matches_exact_rational_cover(geom):
    src_nq, src_lkv, dst_nq, dst_lkv, bq, bk, n_sink = geom
    rng = np.random.default_rng(sum(geom))
    snqb, snkb = orc.n_blocks(src_nq, bq), orc.n_blocks(src_lkv, bk)
    src = rng.random((snqb, snkb)) < 0.3
    dst = orc.map_block_mask(src, src_nq, src_lkv, dst_nq, dst_lkv, bq, bk, n_sink)
    want = np.zeros_like(dst)
    for qb, kb in zip(*np.nonzero(src)):
        tq = _covered_tokens_exact(qb * bq, min(qb * bq + bq, src_nq), src_nq, dst_nq)
        tk = _covered_tokens_exact(kb * bk, min(kb * bk + bk, src_lkv), src_lkv, dst_lkv)
        for a in sorted({t // bq for t in tq}):
            for b in sorted({t // bk for t in tk}):
                want[a, b] = True
    want[:, :orc.n_blocks(n_sink, bk)] = True
    assert np.array_equal(dst, want)


def test_map_identity_and_invariants():
    rng = np.random.default_rng(3)
    src = rng.random((8, 20)) < 0.3
    same = orc.map_block_mask(src, 1024, 2521, 1024, 2521, 128, 128, 0)
    assert np.array_equal(same, src)
    full = orc.map_block_mask(np.ones((8, 20), bool), 1024, 2521, 4096, 10521, 128, 128, 0)
    assert full.all()
    a = orc.map_block_mask(src, 1024, 2521, 4096, 10521, 128, 128, 121)
    more = src | (rng.random((8, 20)) < 0.2)
    b = orc.map_block_mask(more, 1024, 2521, 4096, 10521, 128, 128, 121)
    assert np.all(b >= a)
    assert a[:, 0].all()
    cnt, idx, blk = orc.map_indices(*orc.block_lists(src), 1024, 2521, 4096, 10521, 128, 128, 121)
    assert np.array_equal(blk, a)
    assert np.all((idx == -1) | ((idx >= 0) & (idx < 83)))
    for qb in range(32):
        row = idx[qb, :cnt[qb]]
        assert np.all(np.diff(row) > 0)


# ---------------------------------------------------------------- CS4A 2-D mapping
def test_map_2d_golden():
    for line in open(os.path.join(GOLDEN, "map_2d_tiny.txt")):
        if not line.startswith("case"):
            continue
        parts = [p.strip() for p in line.split("|")]
        sink = int(parts[1].split()[1])
        src = np.zeros((2, 3), bool)
        for pr in parts[2].split():
            a, b = pr.split(":")
            src[int(a), int(b)] = True
        want = np.zeros((8, 11), bool)
        for pr in parts[3].split():
            a, b = pr.split(":")
            for x in filter(None, b.split(",")):
                want[int(a), int(x)] = True
        dst = orc.map_block_mask_2d(src, (1, 2, 4), 1, 2, 2, 2, sink)
        assert np.array_equal(dst, want), parts[0]


def test_upscale_cell():
    assert orc.upscale_cell(3, 4, 8) == (6, 8)          # exact 2x
    assert orc.upscale_cell(0, 32, 40) == (0, 2)        # 1.25x: [0, 1.25) -> rows 0, 1
    assert orc.upscale_cell(3, 32, 40) == (3, 5)        # [3.75, 5)
    assert orc.upscale_cell(31, 32, 48) == (46, 48)
    assert orc.upscale_cell(5, 7, 7) == (5, 6)          # same side: identity


def _token_level_2d(src, sides, d, t, bq, bk, n_sink):
    """Brute force: token pairs of kept source blocks carried to the target, then blocks."""
    off = orc.scale_offsets(sides)
    s_d, s_t = sides[d], sides[t]
    n_t, l_t = s_t * s_t, off[t + 1]
    tok = np.zeros((n_t, l_t), bool)

    def img_q(q):
        i, j = divmod(q, s_d)
        r0, r1 = orc.upscale_cell(i, s_d, s_t)
        c0, c1 = orc.upscale_cell(j, s_d, s_t)
        return [r * s_t + c for r in range(r0, r1) for c in range(c0, c1)]

    def img_k(key):
        if key < off[d]:
            return [key]
        a, b = divmod(key - off[d], s_d)
        r0, r1 = orc.upscale_cell(a, s_d, s_t)
        c0, c1 = orc.upscale_cell(b, s_d, s_t)
        return [off[t] + r * s_t + c for r in range(r0, r1) for c in range(c0, c1)]

    for qb, kb in zip(*np.nonzero(src)):
        qs = sorted({x for q in range(qb * bq, min(qb * bq + bq, s_d * s_d)) for x in img_q(q)})
        ks = sorted({x for k in range(kb * bk, min(kb * bk + bk, off[d + 1])) for x in img_k(k)})
        tok[np.ix_(qs, ks)] = True
    tok[:, :min(n_sink, l_t)] = True
    nqb, nkb = orc.n_blocks(n_t, bq), orc.n_blocks(l_t, bk)
    return np.array([[tok[a * bq:(a + 1) * bq, b * bk:(b + 1) * bk].any() for b in range(nkb)]
                     for a in range(nqb)])


@pytest.mark.parametrize("sides,d,t,bq,bk,sink", [
    ((1, 2, 4, 6, 8), 2, 4, 4, 4, 1),
    ((1, 2, 4, 6, 8), 3, 4, 8, 4, 5),
    ((1, 2, 3, 5, 7), 2, 4, 4, 8, 0),
    ((1, 2, 4, 6, 8, 12), 3, 5, 16, 16, 21),
])
def test_map_2d_matches_token_level(sides, d, t, bq, bk, sink):
    off = orc.scale_offsets(sides)
    rng = np.random.default_rng(d * 10 + t)
    src = rng.random((orc.n_blocks(sides[d] ** 2, bq), orc.n_blocks(off[d + 1], bk))) < 0.35
    dst = orc.map_block_mask_2d(src, sides, d, t, bq, bk, sink)
    assert np.array_equal(dst, _token_level_2d(src, sides, d, t, bq, bk, sink))


def test_map_2d_identity_and_invariants():
    sides = inputs.INFINITY_SIDES
    off = orc.scale_offsets(sides)
    rng = np.random.default_rng(11)
    src = rng.random((8, 20)) < 0.3
    # same scale: every token maps to itself
    assert np.array_equal(orc.map_block_mask_2d(src, sides, 9, 9, 128, 128, 0), src)
    dst = orc.map_block_mask_2d(src, sides, 9, 12, 128, 128, 121)
    assert dst[:, 0].all()
    # keys of the scales strictly between the two are reached only by the sink
    mid = [kb for kb in range(83) if kb * 128 >= off[10] and (kb + 1) * 128 <= off[12]]
    assert mid and not dst[:, mid].any()
    # a full source covers the earlier scales and the target's own scale, for every query block
    full = orc.map_block_mask_2d(np.ones((8, 20), bool), sides, 9, 12, 128, 128, 0)
    keep = [kb for kb in range(83) if kb * 128 < off[9] or (kb + 1) * 128 > off[12]]
    assert full[:, keep].all()
    # monotone in the source
    more = src | (rng.random((8, 20)) < 0.2)
    assert np.all(orc.map_block_mask_2d(more, sides, 9, 12, 128, 128, 121) >= dst)
    cnt, idx, blk = orc.map_indices_2d(*orc.block_lists(src), sides, 9, 12, 128, 128, 121)
    assert np.array_equal(blk, dst)


def test_block_lists_layout_and_inverse():
    """Lists are ascending with a -1 tail and counts equal to the kept blocks per
    row (a hand-made mask); lists_to_blocks inverts them and ignores entry order
    and the tail."""
    blk = np.array([[1, 0, 1, 1], [0, 0, 0, 0], [0, 1, 0, 0]], dtype=bool)
    cnt, idx = orc.block_lists(blk)
    assert cnt.tolist() == [3, 0, 1]
    assert idx.tolist() == [[0, 2, 3, -1], [-1, -1, -1, -1], [1, -1, -1, -1]]
    assert np.array_equal(orc.lists_to_blocks(cnt, idx, 4), blk)
    shuffled = np.array([[3, 0, 2, -1], [-1, -1, -1, -1], [1, -1, -1, -1]], dtype=np.int32)
    assert np.array_equal(orc.lists_to_blocks(cnt, shuffled, 4), blk)
    rng = np.random.default_rng(4)
    for _ in range(20):
        r = rng.random((5, 9)) < rng.random()
        assert np.array_equal(orc.lists_to_blocks(*orc.block_lists(r), 9), r)
