"""Pins for the oracle's masked attention (CPU only).

The oracle's result is tied to things other than itself: torch's own fp64
scaled-dot-product attention, element-by-element Python loops, and closed
forms (Q = 0, constant V, one-hot V, empty rows).
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import sparvar_oracle as orc
from tests.conftest import GOLDEN


def _rand(seed, *shape):
    return np.random.default_rng(seed).standard_normal(shape)


def test_all_kept_equals_torch_sdpa():
    q, k, v = _rand(1, 150, 32), _rand(2, 333, 32), _rand(3, 333, 32)
    blk = np.ones((orc.n_blocks(150, 64), orc.n_blocks(333, 64)), dtype=bool)
    O, lse = orc.masked_attention(q, k, v, blk, 64, 64)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None], torch.from_numpy(k)[None, None], torch.from_numpy(v)[None, None])
    np.testing.assert_allclose(O, ref[0, 0].numpy(), rtol=0, atol=1e-12)
    s = (q @ k.T) / math.sqrt(32)
    np.testing.assert_allclose(lse, torch.logsumexp(torch.from_numpy(s), dim=1).numpy(), atol=1e-12)


def test_block_mask_equals_torch_sdpa_with_boolean_mask():
    rng = np.random.default_rng(7)
    q, k, v = _rand(4, 70, 16), _rand(5, 90, 16), _rand(6, 90, 16)
    blk = rng.random((orc.n_blocks(70, 16), orc.n_blocks(90, 8))) < 0.5
    blk[:, 0] = True
    O, _ = orc.masked_attention(q, k, v, blk, 16, 8, scale=0.3)
    E = np.repeat(np.repeat(blk, 16, axis=0), 8, axis=1)[:70, :90]
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None],
        attn_mask=torch.from_numpy(E)[None], scale=0.3)
    np.testing.assert_allclose(O, ref[0].numpy(), atol=1e-12)


def test_bruteforce_loops_tiny():
    rng = np.random.default_rng(11)
    nq, L, D, bq, bk = 9, 13, 4, 4, 5
    q, k, v = _rand(12, nq, D), _rand(13, L, D), _rand(14, L, D)
    blk = rng.random((orc.n_blocks(nq, bq), orc.n_blocks(L, bk))) < 0.6
    blk[:, 1] = True
    scale = 0.7
    O, lse = orc.masked_attention(q, k, v, blk, bq, bk, scale=scale)
    for i in range(nq):
        keys = [j for j in range(L) if blk[i // bq][j // bk]]
        scores = [scale * sum(q[i][d] * k[j][d] for d in range(D)) for j in keys]
        mx = max(scores)
        w = [math.exp(s - mx) for s in scores]
        tot = sum(w)
        for d in range(D):
            ref = sum(wi * v[j][d] for wi, j in zip(w, keys)) / tot
            assert abs(O[i][d] - ref) < 1e-12
        assert abs(lse[i] - (mx + math.log(tot))) < 1e-12


def test_rows_of_p_sum_to_one_and_masked_entries_zero():
    rng = np.random.default_rng(3)
    q, k, v = _rand(20, 40, 8), _rand(21, 57, 8), _rand(22, 57, 8)
    blk = rng.random((5, 8)) < 0.5
    blk[:, 2] = True
    _, _, P = orc.masked_attention(q, k, v, blk, 8, 8, return_p=True)
    np.testing.assert_allclose(P.sum(axis=1), 1.0, atol=1e-13)
    E = orc.expand_block_mask(blk, 40, 57, 8, 8)
    assert np.all(P[~E] == 0.0)


def test_zero_query_gives_mean_of_kept_values():
    v = _rand(30, 50, 6)
    k = _rand(31, 50, 6)
    q = np.zeros((20, 6))
    blk = np.zeros((2, 5), dtype=bool)
    blk[0, [0, 3]] = True
    blk[1, [4]] = True
    O, _ = orc.masked_attention(q, k, v, blk, 10, 10)
    np.testing.assert_allclose(O[:10], np.concatenate([v[0:10], v[30:40]]).mean(0)[None].repeat(10, 0), atol=1e-13)
    np.testing.assert_allclose(O[10:], v[40:50].mean(0)[None].repeat(10, 0), atol=1e-13)


def test_constant_value_rows_give_the_constant():
    q, k = _rand(40, 33, 8), _rand(41, 77, 8)
    v = np.full((77, 8), 2.5)
    blk = np.random.default_rng(0).random((3, 5)) < 0.5
    blk[:, 4] = True
    O, _ = orc.masked_attention(q, k, v, blk, 16, 16)
    np.testing.assert_allclose(O, 2.5, atol=1e-13)


def test_one_hot_values_give_block_sums_of_p():
    q, k = _rand(50, 24, 8), _rand(51, 40, 8)
    nkb = 5
    v = np.zeros((40, nkb))
    for key in range(40):
        v[key, key // 8] = 1.0
    blk = np.random.default_rng(2).random((3, nkb)) < 0.6
    blk[:, 0] = True
    O, _, P = orc.masked_attention(q, k, v, blk, 8, 8, return_p=True)
    for kb in range(nkb):
        np.testing.assert_allclose(O[:, kb], P[:, kb * 8:(kb + 1) * 8].sum(1), atol=1e-13)
        assert np.all(O[:, kb][~np.repeat(blk[:, kb], 8)] == 0.0)


def test_empty_rows_give_zero_and_minus_inf():
    q, k, v = _rand(60, 16, 4), _rand(61, 16, 4), _rand(62, 16, 4)
    blk = np.array([[True, False], [False, False]])
    O, lse = orc.masked_attention(q, k, v, blk, 8, 8)
    assert np.all(O[8:] == 0.0) and np.all(np.isneginf(lse[8:]))
    assert np.all(np.isfinite(lse[:8]))


def test_rows_variant_matches_full():
    q, k, v = _rand(70, 100, 16), _rand(71, 130, 16), _rand(72, 130, 16)
    blk = np.random.default_rng(5).random((4, 5)) < 0.5
    blk[:, 0] = True
    O, lse = orc.masked_attention(q, k, v, blk, 32, 32)
    rows = np.array([0, 17, 31, 32, 99])
    O2, lse2 = orc.masked_attention_rows(rows, q, k, v, blk, 32, 32)
    np.testing.assert_allclose(O2, O[rows], atol=1e-13)
    np.testing.assert_allclose(lse2, lse[rows], atol=1e-13)


def test_kept_flops_closed_form():
    blk = np.ones((3, 4), dtype=bool)
    assert orc.kept_flops(blk, 300, 500, 128, 128, 64) == 4 * 300 * 500 * 64
    blk = np.zeros((3, 4), dtype=bool)
    blk[2, 3] = True  # 44 query rows x 116 keys
    assert orc.kept_flops(blk, 300, 500, 128, 128, 64) == 4 * 44 * 116 * 64


@pytest.mark.parametrize("planted", ["drop_scale", "swap_block_sizes", "no_max_shift_sign"])
def test_plausible_mistakes_are_caught(planted):
    """Planted mistakes (in a copy of the arithmetic, on the CPU) fail the torch pin."""
    q, k, v = _rand(80, 24, 8), _rand(81, 40, 8), _rand(82, 40, 8)
    blk = np.random.default_rng(9).random((3, 8)) < 0.5
    blk[:, 0] = True
    E = orc.expand_block_mask(blk, 24, 40, 8, 5)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None],
        attn_mask=torch.from_numpy(E)[None])[0].numpy()
    good, _ = orc.masked_attention(q, k, v, blk, 8, 5)
    assert np.abs(good - ref).max() < 1e-12
    S = (q @ k.T) / math.sqrt(8)
    if planted == "drop_scale":
        S = q @ k.T
        Sm = np.where(E, S, -np.inf)
    elif planted == "swap_block_sizes":
        Eb = blk[np.minimum(np.arange(24) // 5, 2)][:, np.arange(40) // 8]
        Sm = np.where(Eb, S, -np.inf)
    else:
        Sm = np.where(E, -S, -np.inf)
    P = np.exp(Sm - Sm.max(1, keepdims=True))
    bad = (P / P.sum(1, keepdims=True)) @ v
    assert np.abs(bad - ref).max() > 1e-3


# ---------------------------------------------------------------- CS4A output cache
def test_ocache_golden():
    od = np.array([[1.0], [2.0], [3.0], [4.0]])
    osp = np.array([[0.5], [2.0], [2.0], [5.0]])
    for line in open(os.path.join(GOLDEN, "ocache_tiny.txt")):
        if not line.startswith("side"):
            continue
        a, b, c = [x.strip() for x in line.split("|")]
        s_dst = int(a.split()[1])
        ot = np.array([[float(x)] for x in b.split()])
        want = np.array([float(x) for x in c.split()])
        np.testing.assert_allclose(orc.ocache_apply(ot, od, osp, 2, s_dst)[:, 0], want, atol=0)


def test_ocache_closed_forms():
    rng = np.random.default_rng(3)
    # every block kept: the sparse output is the dense one, the residual is zero
    q, k, v = rng.standard_normal((64, 16)), rng.standard_normal((100, 16)), rng.standard_normal((100, 16))
    full = np.ones((4, 7), bool)
    o_dense, _ = orc.masked_attention(q, k, v, full, 16, 16)
    o_sparse, _ = orc.masked_attention(q, k, v, full, 16, 16)
    assert np.abs(orc.ocache_residual(o_dense, o_sparse)).max() == 0.0
    r = rng.standard_normal((36, 5))
    # same side: identity; constant field stays constant; integer factor replicates
    np.testing.assert_array_equal(orc.ocache_upsample(r, 6, 6), r)
    c = np.full((36, 5), 2.5)
    np.testing.assert_array_equal(orc.ocache_upsample(c, 6, 10), np.full((100, 5), 2.5))
    up = orc.ocache_upsample(r, 6, 12).reshape(12, 12, 5)
    for i in range(12):
        for j in range(12):
            np.testing.assert_array_equal(up[i, j], r[(i // 2) * 6 + j // 2])
    # linear in the residual, and every source token used when upsampling
    r2 = rng.standard_normal((36, 5))
    np.testing.assert_allclose(orc.ocache_upsample(r + 2 * r2, 6, 9),
                               orc.ocache_upsample(r, 6, 9) + 2 * orc.ocache_upsample(r2, 6, 9))
    used = {orc.nearest_source(i, 32, 48) for i in range(48)}
    assert used == set(range(32))


# ---------------------------------------------------------------- token-level masks
def test_token_mask_attention_pins():
    rng = np.random.default_rng(21)
    q, k, v = rng.standard_normal((40, 8)), rng.standard_normal((70, 8)), rng.standard_normal((70, 8))
    # a block-structured token mask gives the block function's result
    blk = rng.random((3, 5)) < 0.5
    blk[:, 0] = True
    E = orc.expand_block_mask(blk, 40, 70, 16, 16)
    O1, L1 = orc.masked_attention_tokens(q, k, v, E)
    O2, L2 = orc.masked_attention(q, k, v, blk, 16, 16)
    np.testing.assert_allclose(O1, O2, atol=1e-14)
    np.testing.assert_allclose(L1, L2, atol=1e-14)
    # brute force on a random token mask, element by element
    T = rng.random((40, 70)) < 0.3
    T[5] = False  # an empty row
    O, lse = orc.masked_attention_tokens(q, k, v, T, scale=0.4)
    for i in range(40):
        keys = np.nonzero(T[i])[0]
        if keys.size == 0:
            assert np.all(O[i] == 0) and lse[i] == -np.inf
            continue
        s = [0.4 * sum(q[i, d] * k[j, d] for d in range(8)) for j in keys]
        mx = max(s)
        w = [math.exp(x - mx) for x in s]
        z = sum(w)
        for d in range(8):
            assert abs(O[i, d] - sum(w[t] * v[j, d] for t, j in enumerate(keys)) / z) < 1e-12
        assert abs(lse[i] - (mx + math.log(z))) < 1e-12


def test_csla_token_mask_inside_its_blocks():
    # the CSLA block mask is the token mask's aggregate, so masking by tokens inside the
    # kept blocks is masking by tokens
    sides = (1, 2, 4, 8, 16)
    T = orc.csla_token_mask(sides, 4, 2, 1, 1)
    cnt, idx, blk = orc.build_csla_mask(sides, 4, 2, 1, 1, 16, 16)
    E = orc.expand_block_mask(blk, T.shape[0], T.shape[1], 16, 16)
    assert np.all(E[T]) and (E & ~T).any()
