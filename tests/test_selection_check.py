"""The CS4A selection validity checker used by the GPU parity tests, on the CPU.

The oracle's own selections must pass; planted mistakes (an extra block, a
missing block, a lighter block swapped in, a wrong Top-K count, a broken list
layout) must fail.
"""
import numpy as np
import pytest

from oracle import sparvar_oracle as orc
from tests.selection_check import mass_selection_error, topk_selection_error


def _rows(seed, nqb=64, nkb=20):
    rng = np.random.default_rng(seed)
    # peaked rows (a few heavy blocks) and flat rows, each summing to one
    M = rng.dirichlet(np.full(nkb, 0.3), size=nqb // 2)
    M = np.concatenate([M, rng.dirichlet(np.full(nkb, 5.0), size=nqb - nqb // 2)])
    return M


def _lists(blk):
    cnt, idx = orc.block_lists(blk)
    return cnt, idx


@pytest.mark.parametrize("tau", [0.5, 0.95, 0.99])
def test_oracle_mass_selection_passes(tau):
    M = _rows(1)
    blk, _ = orc.select_blocks_by_mass(M, tau)
    cnt, idx = _lists(blk)
    for qb in range(M.shape[0]):
        assert mass_selection_error(cnt[qb], idx[qb], M[qb], tau) == ""


def test_threshold_never_reached_keeps_everything():
    M = _rows(2) * 0.5  # rows sum to 0.5 < tau
    blk, _ = orc.select_blocks_by_mass(M, 0.95)
    cnt, idx = _lists(blk)
    assert np.all(cnt == M.shape[1])
    for qb in range(M.shape[0]):
        assert mass_selection_error(cnt[qb], idx[qb], M[qb], 0.95) == ""


def _replant(row_kept, nkb):
    idx = np.full(nkb, -1, np.int32)
    kept = np.sort(np.asarray(row_kept, np.int32))
    idx[:kept.size] = kept
    return kept.size, idx


def test_planted_superset_fails():
    """One extra block appended (the heaviest dropped one, so the set is still
    heaviest first): the selection is no longer minimal."""
    tau = 0.95
    M = _rows(3)
    blk, margin = orc.select_blocks_by_mass(M, tau)
    cnt, idx = _lists(blk)
    failed = 0
    for qb in range(M.shape[0]):
        if cnt[qb] == M.shape[1] or margin[qb] < 1e-3:
            continue
        kept = list(idx[qb, :cnt[qb]])
        dropped = [kb for kb in range(M.shape[1]) if kb not in kept]
        extra = max(dropped, key=lambda kb: M[qb, kb])
        c2, i2 = _replant(kept + [extra], M.shape[1])
        assert mass_selection_error(c2, i2, M[qb], tau) != ""
        failed += 1
    assert failed > 20


def test_planted_missing_block_fails():
    tau = 0.95
    M = _rows(4)
    blk, margin = orc.select_blocks_by_mass(M, tau)
    cnt, idx = _lists(blk)
    n = 0
    for qb in range(M.shape[0]):
        if cnt[qb] < 2 or margin[qb] < 1e-3:
            continue
        kept = list(idx[qb, :cnt[qb]])
        lightest = min(kept, key=lambda kb: M[qb, kb])
        c2, i2 = _replant([kb for kb in kept if kb != lightest], M.shape[1])
        assert mass_selection_error(c2, i2, M[qb], tau) != ""
        n += 1
    assert n > 20


def test_planted_lighter_swap_fails():
    """The lightest kept block replaced by a strictly lighter dropped one."""
    tau = 0.95
    M = _rows(5)
    blk, _ = orc.select_blocks_by_mass(M, tau)
    cnt, idx = _lists(blk)
    n = 0
    for qb in range(M.shape[0]):
        kept = list(idx[qb, :cnt[qb]])
        dropped = [kb for kb in range(M.shape[1]) if kb not in kept]
        if not dropped:
            continue
        lightest = min(kept, key=lambda kb: M[qb, kb])
        lighter = min(dropped, key=lambda kb: M[qb, kb])
        if M[qb, lightest] - M[qb, lighter] < 1e-3:
            continue
        c2, i2 = _replant([kb for kb in kept if kb != lightest] + [lighter], M.shape[1])
        assert mass_selection_error(c2, i2, M[qb], tau) != ""
        n += 1
    assert n > 20


def test_layout_mistakes_fail():
    M = _rows(6)[0]
    blk, _ = orc.select_blocks_by_mass(M[None], 0.95)
    cnt, idx = _lists(blk)
    c, row = int(cnt[0]), idx[0].copy()
    assert mass_selection_error(c, row, M, 0.95) == ""
    bad = row.copy()
    bad[c:] = 0  # tail not -1
    if c < M.size:
        assert mass_selection_error(c, bad, M, 0.95) != ""
    bad = row.copy()
    if c >= 2:
        bad[0], bad[1] = bad[1], bad[0]  # not ascending
        assert mass_selection_error(c, bad, M, 0.95) != ""
    bad = row.copy()
    bad[0] = M.size  # out of range
    assert mass_selection_error(c, bad, M, 0.95) != ""


@pytest.mark.parametrize("ratio", [0.2, 0.5, 1e-6, 1.0])
def test_topk_checker(ratio):
    M = _rows(7)
    nkb = M.shape[1]
    k = orc.topk_count(ratio, nkb)
    blk, margin = orc.select_blocks_topk(M, ratio)
    cnt, idx = _lists(blk)
    for qb in range(M.shape[0]):
        assert topk_selection_error(cnt[qb], idx[qb], M[qb], k) == ""
        kept = list(idx[qb, :k])
        dropped = [kb for kb in range(nkb) if kb not in kept]
        if dropped:
            # one block too many
            extra = max(dropped, key=lambda kb: M[qb, kb])
            c2, i2 = _replant(kept + [extra], nkb)
            assert topk_selection_error(c2, i2, M[qb], k) != ""
            # a lighter block swapped in
            lightest = min(kept, key=lambda kb: M[qb, kb])
            lighter = min(dropped, key=lambda kb: M[qb, kb])
            if margin[qb] > 1e-3 and M[qb, lightest] - M[qb, lighter] > 1e-3:
                c3, i3 = _replant([kb for kb in kept if kb != lightest] + [lighter], nkb)
                assert topk_selection_error(c3, i3, M[qb], k) != ""
