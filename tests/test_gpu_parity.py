"""CUDA path vs the CPU fp64 oracle, through the C-ABI (needs a B200).

Masks and index lists must match bit-exactly (the CS4A selection under the
margin rule: rows whose decision sits within 1e-4 of a flip are checked for
validity instead).  Attention outputs must match with max-abs <= 2e-2 and
mean-abs <= 2e-3 against fp64 on the same bf16 inputs.
"""

import numpy as np
import pytest
import torch

from block_sparse_cross_sparvar_b200 import inputs, ops
from oracle import sparvar_oracle as orc
from tests.selection_check import mass_selection_error, topk_selection_error

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3
INF = inputs.INFINITY_SIDES
TINY = inputs.TINY_SIDES


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _status():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


# ------------------------------------------------------------------ CSLA masks
MASK_CASES = [
    (TINY, 4, 2, 1, 1, 16, 16),
    (TINY, 3, 2, 1, 1, 16, 16),
    (TINY, 4, 2, 1, 1, 128, 128),
    (INF, 12, 5, 2, 4, 128, 128),
    (INF, 11, 5, 2, 4, 128, 128),
    (INF, 10, 5, 2, 4, 128, 128),
    (INF, 12, 5, 1, 4, 128, 128),
    (INF, 12, 5, 4, 4, 128, 128),
    (INF, 11, 5, 1, 4, 128, 128),
    (INF, 11, 5, 4, 4, 128, 128),
    (INF, 12, 5, 2, 4, 64, 64),
    (INF, 12, 8, 2, 4, 128, 128),
    (INF, 12, 5, 3, 5, 32, 16),
    (INF, 3, 5, 2, 4, 16, 16),
    ((1, 3, 5, 7, 11), 4, 1, 1, 2, 16, 32),
]


@pytest.mark.parametrize("case", MASK_CASES, ids=lambda c: "-".join(map(str, c[1:])))
def test_csla_mask_bit_exact(case):
    sides, k, ns, rp, ro, bq, bk = case
    cnt, idx, mask = ops.sparvar_build_csla_mask(sides, k, ns, rp, ro, bq, bk, with_mask=True)
    ocnt, oidx, oblk = orc.build_csla_mask(sides, k, ns, rp, ro, bq, bk)
    assert np.array_equal(cnt.cpu().numpy(), ocnt)
    assert np.array_equal(idx.cpu().numpy(), oidx)
    assert np.array_equal(mask.cpu().numpy().astype(bool), oblk)


def test_csla_every_scale_and_block_size():
    for bq in (16, 32, 64, 128):
        for k in range(len(INF)):
            cnt, idx, _ = ops.sparvar_build_csla_mask(INF, k, 5, 2, 4, bq, bq)
            ocnt, oidx, _ = orc.build_csla_mask(INF, k, 5, 2, 4, bq, bq)
            assert np.array_equal(cnt.cpu().numpy(), ocnt), (bq, k)
            assert np.array_equal(idx.cpu().numpy(), oidx), (bq, k)


# ------------------------------------------------------------------ attention
def _check_attention(q_bits, k_bits, v_bits, blk_lists, bq, bk, D, lse_check=True, scale=None,
                     ordered=False):
    """q/k/v bits [B,H,*,D]; blk_lists = (cnt, idx) torch (shared or per (b,h));
    ordered: the kernel takes the query tiles longest list first."""
    B, H, Lq, _ = q_bits.shape
    Lkv = k_bits.shape[2]
    q, k, v = _dev(q_bits), _dev(k_bits), _dev(v_bits)
    cnt, idx = blk_lists
    st = _status()
    order = ops.sparvar_tile_order(cnt, B, H, Lq) if ordered else None
    o, lse = ops.sparvar_block_sparse_attn_fwd(q, k, v, cnt, idx, bq, bk, softmax_scale=scale,
                                               return_lse=True, dev_status=st, tile_order=order)
    torch.cuda.synchronize()
    assert st.item() == 0
    o = o.float().cpu().numpy()
    lse = lse.cpu().numpy()
    cnt_np, idx_np = cnt.cpu().numpy(), idx.cpu().numpy()
    nkb = -(-Lkv // bk)
    worst = 0.0
    for b in range(B):
        for h in range(H):
            if cnt_np.ndim == 1:
                c, ix = cnt_np, idx_np
            else:
                c, ix = cnt_np[b, h], idx_np[b, h]
            blk = orc.lists_to_blocks(c, ix, nkb)
            O, L = orc.masked_attention(q_bits_f(q_bits, b, h), q_bits_f(k_bits, b, h),
                                        q_bits_f(v_bits, b, h), blk, bq, bk, scale=scale)
            err = np.abs(o[b, h] - O)
            assert err.max() <= MAX_ABS, (b, h, err.max())
            assert err.mean() <= MEAN_ABS, (b, h, err.mean())
            worst = max(worst, err.max())
            if lse_check:
                fin = np.isfinite(L)
                assert np.array_equal(np.isfinite(lse[b, h]), fin)
                assert np.abs(lse[b, h][fin] - L[fin]).max() < 1e-3
    return worst


def q_bits_f(bits, b, h):
    return (bits[b, h].astype(np.uint32) << 16).view(np.float32).astype(np.float64)


@pytest.mark.parametrize("D", [64, 128])
def test_attention_tiny_schedule_block128(D):
    d = inputs.make_qkv(1, 1, 2, TINY, D, 2, pe=False)
    off = d["offsets"]
    k = len(TINY) - 1
    q_bits = d["q"][:, :, off[k]:off[k + 1]]
    kv = slice(0, off[k + 1])
    cnt, idx, _ = ops.sparvar_build_csla_mask(TINY, k, 2, 1, 1, 128, 128)
    _check_attention(q_bits, d["k"][:, :, kv], d["v"][:, :, kv], (cnt, idx), 128, 128, D)


@pytest.mark.parametrize("q_scale", [2, 3, 4])
def test_attention_tiny_schedule_block16(q_scale):
    """The tiny schedule with 16x16 CSLA blocks (sink = scales 1-2, radius 1), B1 H2
    D64: fine lists go through coarsening to 128x128 tiles with per-tile masks."""
    d = inputs.make_qkv(6, 1, 2, TINY, 64, 2, pe=False)
    off = d["offsets"]
    q_bits = d["q"][:, :, off[q_scale]:off[q_scale + 1]]
    kv = slice(0, off[q_scale + 1])
    cnt, idx, _ = ops.sparvar_build_csla_mask(TINY, q_scale, 2, 1, 1, 16, 16)
    _check_attention(q_bits, d["k"][:, :, kv], d["v"][:, :, kv], (cnt, idx), 16, 16, 64)


def _random_lists(rng, B, H, nqb, nkb, p):
    blk = rng.random((B, H, nqb, nkb)) < p
    cnt = torch.from_numpy(blk.sum(-1).astype(np.int32)).cuda()
    idx_np = np.full((B, H, nqb, nkb), -1, np.int32)
    for b in range(B):
        for h in range(H):
            for qb in range(nqb):
                kept = np.nonzero(blk[b, h, qb])[0]
                idx_np[b, h, qb, :kept.size] = kept
    return blk, cnt, torch.from_numpy(idx_np).cuda()


@pytest.mark.parametrize("block,D", [(16, 64), (32, 128), (64, 128), (16, 128)])
def test_attention_fine_blocks_random_lists(block, D):
    """Random per-(b, h) fine lists with ragged query and key tails, an empty row
    and a row whose only blocks sit in the ragged last tile."""
    rng = np.random.default_rng(block + D)
    B, H, Lq, Lkv = 2, 2, 300, 777
    bits = {n: inputs.bf16_round(rng.standard_normal((B, H, L, D)).astype(np.float32))[0]
            for n, L in (("q", Lq), ("k", Lkv), ("v", Lkv))}
    nqb, nkb = -(-Lq // block), -(-Lkv // block)
    blk, cnt, idx = _random_lists(rng, B, H, nqb, nkb, 0.3)
    cnt[0, 0, 1] = 0
    cnt[1, 1, nqb - 1] = 1
    idx[1, 1, nqb - 1, 0] = nkb - 1
    _check_attention(bits["q"], bits["k"], bits["v"], (cnt, idx), block, block, D, scale=0.1)


@pytest.mark.parametrize("block", [16, 32, 64])
def test_coarsen_lists_bit_exact(block):
    """Tile lists and masks expand to exactly the fine block mask."""
    rng = np.random.default_rng(7 * block)
    B, H, Lq, Lkv = 2, 3, 1000, 2100
    nqb, nkb = -(-Lq // block), -(-Lkv // block)
    blk, cnt, idx = _random_lists(rng, B, H, nqb, nkb, 0.2)
    st = _status()
    t_cnt, t_idx, t_mask = ops.sparvar_coarsen_lists(cnt, idx, B, H, Lq, Lkv, block, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    t_cnt, t_idx = t_cnt.cpu().numpy(), t_idx.cpu().numpy()
    t_mask = t_mask.cpu().numpy().view(np.uint64)
    g, nqt, nkt = 128 // block, -(-Lq // 128), -(-Lkv // 128)
    for b in range(B):
        for h in range(H):
            got = np.zeros((nqt * g, nkt * g), bool)
            for T in range(nqt):
                c = t_cnt[b, h, T]
                row = t_idx[b, h, T]
                assert np.all(np.diff(row[:c]) > 0) and np.all(row[c:] == -1)
                assert np.all(t_mask[b, h, T, c:] == 0)
                for e in range(c):
                    m = int(t_mask[b, h, T, e])
                    assert m != 0
                    for qi in range(g):
                        for ki in range(g):
                            if (m >> (qi * g + ki)) & 1:
                                got[T * g + qi, row[e] * g + ki] = True
            assert np.array_equal(got[:nqb, :nkb], blk[b, h])
            assert not got[nqb:].any() and not got[:, nkb:].any()


def test_coarsen_shared_lists_stay_shared():
    cnt, idx, blk = ops.sparvar_build_csla_mask(TINY, 4, 2, 1, 1, 16, 16, with_mask=True)
    t_cnt, t_idx, t_mask = ops.sparvar_coarsen_lists(cnt, idx, 2, 4, 256, 341, 16)
    assert tuple(t_cnt.shape) == (1, 1, 2) and tuple(t_idx.shape) == (1, 1, 2, 3)
    ocnt, oidx, oblk = orc.build_csla_mask(TINY, 4, 2, 1, 1, 16, 16)
    m = t_mask.cpu().numpy().view(np.uint64)[0, 0]
    ti = t_idx.cpu().numpy()[0, 0]
    for T in range(2):
        for e in range(int(t_cnt[0, 0, T])):
            for qi in range(8):
                for ki in range(8):
                    qb, kb = T * 8 + qi, ti[T, e] * 8 + ki
                    bit = bool((int(m[T, e]) >> (qi * 8 + ki)) & 1)
                    exp = qb < oblk.shape[0] and kb < oblk.shape[1] and bool(oblk[qb, kb])
                    assert bit == exp


@pytest.mark.parametrize("q_scale,D", [(9, 128), (10, 128), (10, 64), (8, 128)])
def test_attention_infinity_mid_scales(q_scale, D):
    d = inputs.make_qkv(2, 1, 2, INF, D, 5)
    off = d["offsets"]
    q_bits = d["q"][:, :, off[q_scale]:off[q_scale + 1]]
    kv = slice(0, off[q_scale + 1])
    cnt, idx, _ = ops.sparvar_build_csla_mask(INF, q_scale, 5, 2, 4, 128, 128)
    _check_attention(q_bits, d["k"][:, :, kv], d["v"][:, :, kv], (cnt, idx), 128, 128, D)


def test_attention_dense_lists_and_random_lists_per_head():
    rng = np.random.default_rng(5)
    B, H, Lq, Lkv, D = 2, 2, 300, 777, 128
    bits = {n: inputs.bf16_round(rng.standard_normal((B, H, L, D)).astype(np.float32))[0]
            for n, L in (("q", Lq), ("k", Lkv), ("v", Lkv))}
    nqb, nkb = 3, 7
    blk = rng.random((B, H, nqb, nkb)) < 0.4
    blk[..., 0, :] = True  # one fully dense query block
    blk[0, 0, 1, :] = False  # one empty list -> O = 0, lse = -inf
    blk[1, 1, 2, :] = False
    blk[1, 1, 2, 6] = True  # only the ragged last block
    cnt = torch.from_numpy(blk.sum(-1).astype(np.int32)).cuda()
    idx_np = np.full((B, H, nqb, nkb), -1, np.int32)
    for b in range(B):
        for h in range(H):
            for qb in range(nqb):
                kept = np.nonzero(blk[b, h, qb])[0]
                idx_np[b, h, qb, :kept.size] = kept
    idx = torch.from_numpy(idx_np).cuda()
    _check_attention(bits["q"], bits["k"], bits["v"], (cnt, idx), 128, 128, D, scale=0.11)


@pytest.mark.parametrize("D", [64, 128])
def test_attention_persistent_short_and_empty_lists(D):
    """Many query tiles per CTA (2 x 16 x 40 = 1280 tiles on at most one CTA per SM)
    with lists of 0-6 blocks in random order, so that each CTA walks every kind of
    transition: empty tiles between others, tiles of one or two blocks (whose
    first score MMAs are issued on their own) and tiles of three or more (which
    feed the next one); ragged query and key tails; every row of every head."""
    rng = np.random.default_rng(17 + D)
    B, H = 2, 16
    nqb, nkb = 40, 6
    Lq, Lkv = nqb * 128 - 37, nkb * 128 - 50
    bits = {n: inputs.bf16_round(rng.standard_normal((B, H, L, D)).astype(np.float32))[0]
            for n, L in (("q", Lq), ("k", Lkv), ("v", Lkv))}
    lens = rng.choice(nkb + 1, size=(B, H, nqb), p=[0.15, 0.2, 0.2, 0.15, 0.1, 0.1, 0.1])
    # CTA 1 walks tiles 1, 1 + G, 1 + 2G, ... (G = one CTA per SM): a tile that
    # feeds the next, two empty tiles, a two-block tile, a feeding tile again
    G = torch.cuda.get_device_properties(0).multi_processor_count
    flat = lens.reshape(-1)
    for i, n in enumerate([3, 0, 0, 2, 4]):
        if 1 + i * G < flat.size:
            flat[1 + i * G] = n
    idx_np = np.full((B, H, nqb, nkb), -1, np.int32)
    for b in range(B):
        for h in range(H):
            for qb in range(nqb):
                idx_np[b, h, qb, :lens[b, h, qb]] = rng.permutation(nkb)[:lens[b, h, qb]]
    cnt = torch.from_numpy(lens.astype(np.int32)).cuda()
    idx = torch.from_numpy(idx_np).cuda()
    _check_attention(bits["q"], bits["k"], bits["v"], (cnt, idx), 128, 128, D)


def test_tile_order_longest_first_serpentine():
    """The order is a permutation of the tiles; round r of G positions holds the
    natural tiles r*G .. r*G + G - 1, longest list first, then by query block, then
    by tile id, dealt to CTAs 0..G-1 for even r and G-1..0 for odd r."""
    rng = np.random.default_rng(5)
    B, H, nqb = 2, 16, 40
    lens = rng.integers(0, 30, size=(B, H, nqb)).astype(np.int32)
    cnt = torch.from_numpy(lens).cuda()
    order = ops.sparvar_tile_order(cnt, B, H, nqb * 128).cpu().numpy()
    T = B * H * nqb
    G = min(T, torch.cuda.get_device_properties(0).multi_processor_count)
    assert sorted(order.tolist()) == list(range(T))
    flat = lens.reshape(-1)
    for r in range(-(-T // G)):
        pos = order[r * G:(r + 1) * G]
        tiles = np.arange(r * G, min(T, (r + 1) * G))
        want = sorted(tiles.tolist(), key=lambda t: (-flat[t], t % nqb, t))
        dealt = pos if r % 2 == 0 else pos[::-1]
        assert dealt.tolist() == want


def test_csla_build_with_tile_order():
    """The list builder's last CTA writes the same order as the order call, the
    lists are those of the plain builder, and the counter is back at zero, so the
    next call can use it again."""
    done = torch.zeros(1, dtype=torch.int32, device="cuda")
    wide = (1, 2, 4, 8, 16, 32, 64, 128)  # 128 query blocks at the last scale: several
    #                                       chunks of 32 in each round's walk
    for sides, q_scale, csla, B, H in ((INF, 9, (5, 2, 4), 2, 16), (INF, 12, (5, 2, 4), 2, 16),
                                       (INF, 12, (5, 2, 4), 1, 5), (INF, 11, (2, 1, 2), 3, 25),
                                       (wide, 7, (2, 1, 2), 1, 3), (wide, 7, (3, 1, 3), 2, 5)):
        cnt0, idx0, _ = ops.sparvar_build_csla_mask(sides, q_scale, *csla, 128, 128)
        for _ in range(2):
            cnt, idx, order = ops.sparvar_build_csla_mask_ordered(sides, q_scale, *csla, B, H,
                                                                  done=done)
            torch.cuda.synchronize()
            assert torch.equal(cnt, cnt0) and torch.equal(idx, idx0)
            assert int(done.item()) == 0
            nqb = cnt.numel()
            ref = ops.sparvar_tile_order(cnt, B, H, nqb * 128)
            assert torch.equal(order, ref)


def test_attention_in_tile_order():
    """Taking the query tiles longest first changes which CTA runs a tile and what
    comes before it (and so which softmax group takes which of its blocks, and the
    order in which the two groups' PVs add into O): the output matches the oracle
    as in natural order, and the two agree to within rounding."""
    rng = np.random.default_rng(23)
    B, H, D = 2, 16, 128
    nqb, nkb = 40, 6
    Lq, Lkv = nqb * 128 - 37, nkb * 128 - 50
    bits = {n: inputs.bf16_round(rng.standard_normal((B, H, L, D)).astype(np.float32))[0]
            for n, L in (("q", Lq), ("k", Lkv), ("v", Lkv))}
    lens = rng.choice(nkb + 1, size=(B, H, nqb), p=[0.15, 0.2, 0.2, 0.15, 0.1, 0.1, 0.1])
    idx_np = np.full((B, H, nqb, nkb), -1, np.int32)
    for b in range(B):
        for h in range(H):
            for qb in range(nqb):
                idx_np[b, h, qb, :lens[b, h, qb]] = rng.permutation(nkb)[:lens[b, h, qb]]
    cnt = torch.from_numpy(lens.astype(np.int32)).cuda()
    idx = torch.from_numpy(idx_np).cuda()
    q, k, v = _dev(bits["q"]), _dev(bits["k"]), _dev(bits["v"])
    o1, l1 = ops.sparvar_block_sparse_attn_fwd(q, k, v, cnt, idx, return_lse=True)
    order = ops.sparvar_tile_order(cnt, B, H, Lq)
    st = _status()
    o2, l2 = ops.sparvar_block_sparse_attn_fwd(q, k, v, cnt, idx, return_lse=True,
                                               tile_order=order, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert (o1.float() - o2.float()).abs().max().item() <= 1e-2
    fin = torch.isfinite(l1)
    assert torch.equal(fin, torch.isfinite(l2))
    assert (l1[fin] - l2[fin]).abs().max().item() < 1e-4
    _check_attention(bits["q"], bits["k"], bits["v"], (cnt, idx), 128, 128, D, ordered=True)


def test_attention_unordered_lists_give_same_result():
    d = inputs.make_qkv(3, 1, 2, INF, 128, 5)
    off = d["offsets"]
    qk = 10
    q = _dev(d["q"][:, :, off[qk]:off[qk + 1]])
    k = _dev(d["k"][:, :, :off[qk + 1]])
    v = _dev(d["v"][:, :, :off[qk + 1]])
    cnt, idx, _ = ops.sparvar_build_csla_mask(INF, qk, 5, 2, 4, 128, 128)
    o1 = ops.sparvar_block_sparse_attn_fwd(q, k, v, cnt, idx)
    rev = idx.clone()
    for qb in range(cnt.shape[0]):
        c = int(cnt[qb])
        rev[qb, :c] = idx[qb, :c].flip(0)
    o2 = ops.sparvar_block_sparse_attn_fwd(q, k, v, cnt, rev)
    assert (o1.float() - o2.float()).abs().max().item() < 2e-2


def test_attention_bad_list_entries_flagged_not_trapped():
    d = inputs.make_qkv(4, 1, 1, TINY, 64, 2, pe=False)
    off = d["offsets"]
    q = _dev(d["q"][:, :, off[4]:off[5]])
    k = _dev(d["k"][:, :, :off[5]])
    v = _dev(d["v"][:, :, :off[5]])
    cnt = torch.tensor([2, 2], dtype=torch.int32, device="cuda")
    idx = torch.tensor([[0, 99, -1], [1, -5, -1]], dtype=torch.int32, device="cuda")
    st = _status()
    o = ops.sparvar_block_sparse_attn_fwd(q, k, v, cnt, idx, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() & ops.SPARVAR_DEV_BAD_LIST
    # the valid entries alone give the same output
    cnt1 = torch.tensor([1, 1], dtype=torch.int32, device="cuda")
    idx1 = torch.tensor([[0, -1, -1], [1, -1, -1]], dtype=torch.int32, device="cuda")
    o1 = ops.sparvar_block_sparse_attn_fwd(q, k, v, cnt1, idx1)
    assert torch.equal(o, o1)
    assert ops.sparvar_validate_lists(cnt, idx, 3) & ops.SPARVAR_DEV_BAD_LIST
    assert ops.sparvar_validate_lists(cnt1, idx1, 3) == 0
    bad_order = torch.tensor([[1, 0, -1], [0, 2, -1]], dtype=torch.int32, device="cuda")
    assert ops.sparvar_validate_lists(cnt, bad_order, 3) == ops.SPARVAR_DEV_NOT_ASCENDING
    over = torch.tensor([5, 1], dtype=torch.int32, device="cuda")
    assert ops.sparvar_validate_lists(over, idx1, 3) & ops.SPARVAR_DEV_BAD_LIST


def test_attention_full_size_sampled_rows():
    """Infinity-2B last scale (B2 H16, 4096 x 10521, D128) in the bench's launch
    configuration (the list builder's tile order); sampled rows against the oracle
    evaluated row by row, and the natural tile order within rounding."""
    d = inputs.make_qkv(0, 2, 16, INF, 128, 5)
    off = d["offsets"]
    q_bits = d["q"][:, :, off[12]:off[13]]
    q, k, v = _dev(q_bits), _dev(d["k"]), _dev(d["v"])
    done = torch.zeros(1, dtype=torch.int32, device="cuda")
    cnt, idx, order = ops.sparvar_build_csla_mask_ordered(INF, 12, 5, 2, 4, 2, 16, done=done)
    st = _status()
    o, lse = ops.sparvar_block_sparse_attn_fwd(q, k, v, cnt, idx, return_lse=True, dev_status=st,
                                               tile_order=order)
    o_nat = ops.sparvar_block_sparse_attn_fwd(q, k, v, cnt, idx, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert (o.float() - o_nat.float()).abs().max().item() <= 1e-2
    ocnt, oidx, blk = orc.build_csla_mask(INF, 12, 5, 2, 4, 128, 128)
    assert np.array_equal(cnt.cpu().numpy(), ocnt) and np.array_equal(idx.cpu().numpy(), oidx)
    rng = np.random.default_rng(0)
    errs = []
    for b, h in [(0, 0), (1, 15), (0, 7), (1, 3)]:
        rows = np.unique(np.concatenate([rng.integers(0, 4096, 60), [0, 127, 128, 4095]]))
        O, L = orc.masked_attention_rows(rows, q_bits_f(q_bits, b, h), q_bits_f(d["k"], b, h),
                                         q_bits_f(d["v"], b, h), blk, 128, 128)
        got = o[b, h, torch.from_numpy(rows).cuda()].float().cpu().numpy()
        err = np.abs(got - O)
        errs.append(err)
        assert np.abs(lse[b, h, torch.from_numpy(rows).cuda()].cpu().numpy() - L).max() < 1e-3
    err = np.concatenate(errs)
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS
    assert torch.isfinite(o.float()).all()


# ------------------------------------------------------------------ CS4A
def _decide_compare(q_bits, k_bits, tau, lse_dev=None):
    B, H, Lq, D = q_bits.shape
    q, k = _dev(q_bits), _dev(k_bits)
    st = _status()
    cnt, idx, mass = ops.sparvar_decide_blocks(q, k, tau, lse=lse_dev, return_mass=True,
                                               dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    cnt, idx, mass = cnt.cpu().numpy(), idx.cpu().numpy(), mass.cpu().numpy()
    n_margin = 0
    for b in range(B):
        for h in range(H):
            ocnt, oidx, oblk, M, margin = orc.decide_blocks(q_bits_f(q_bits, b, h),
                                                             q_bits_f(k_bits, b, h), 128, 128, tau)
            assert np.abs(mass[b, h] - M).max() < 2e-5
            for qb in range(M.shape[0]):
                # every row: a valid selection of the kernel's own masses (heaviest first,
                # minimal, reaching tau); beyond the margin also the oracle's exact list
                err = mass_selection_error(cnt[b, h, qb], idx[b, h, qb], mass[b, h, qb], tau)
                assert err == "", (b, h, qb, err)
                if margin[qb] > 1e-4:
                    assert cnt[b, h, qb] == ocnt[qb]
                    assert np.array_equal(idx[b, h, qb], oidx[qb])
                else:
                    n_margin += 1
    return n_margin


def test_decide_blocks_decision_scale():
    d = inputs.make_qkv(0, 1, 4, INF, 128, 5)
    off = d["offsets"]
    s = 9  # 32x32 decision scale
    _decide_compare(d["q"][:, :, off[s]:off[s + 1]], d["k"][:, :, :off[s + 1]], 0.95)


def test_decide_blocks_with_lse_from_attention():
    d = inputs.make_qkv(1, 2, 2, INF, 128, 5)
    off = d["offsets"]
    s = 9
    q = _dev(d["q"][:, :, off[s]:off[s + 1]])
    k = _dev(d["k"][:, :, :off[s + 1]])
    v = _dev(d["v"][:, :, :off[s + 1]])
    nkb = -(-off[s + 1] // 128)
    cnt = torch.full((8,), nkb, dtype=torch.int32, device="cuda")
    idx = torch.arange(nkb, dtype=torch.int32, device="cuda").repeat(8, 1)
    _, lse = ops.sparvar_block_sparse_attn_fwd(q, k, v, cnt, idx, return_lse=True)
    _decide_compare(d["q"][:, :, off[s]:off[s + 1]], d["k"][:, :, :off[s + 1]], 0.95, lse_dev=lse)


@pytest.mark.parametrize("ratio,D", [(0.2, 128), (0.5, 64), (1e-6, 128), (1.0, 128)])
def test_decide_blocks_topk_ratio(ratio, D):
    """Top-K-ratio mode: exactly ceil(ratio * NKB) blocks, the heaviest ones; bit-exact
    where the gap between the last kept and first dropped mass exceeds 1e-4."""
    d = inputs.make_qkv(8, 1, 3, INF, D, 5)
    off = d["offsets"]
    s = 9
    q_bits, k_bits = d["q"][:, :, off[s]:off[s + 1]], d["k"][:, :, :off[s + 1]]
    B, H = q_bits.shape[:2]
    st = _status()
    cnt, idx, mass = ops.sparvar_decide_blocks(_dev(q_bits), _dev(k_bits), 0.95, topk_ratio=ratio,
                                               return_mass=True, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    cnt, idx, mass = cnt.cpu().numpy(), idx.cpu().numpy(), mass.cpu().numpy()
    nkb = mass.shape[-1]
    kk = orc.topk_count(ratio, nkb)
    assert np.all(cnt == kk)
    for b in range(B):
        for h in range(H):
            ocnt, oidx, oblk, M, margin = orc.decide_blocks(
                q_bits_f(q_bits, b, h), q_bits_f(k_bits, b, h), 128, 128, None, topk_ratio=ratio)
            assert np.abs(mass[b, h] - M).max() < 2e-5
            for qb in range(M.shape[0]):
                # every row: exactly k of the heaviest of the kernel's own masses, ascending,
                # -1 padded; beyond the margin also the oracle's exact list
                err = topk_selection_error(cnt[b, h, qb], idx[b, h, qb], mass[b, h, qb], kk)
                assert err == "", (b, h, qb, err)
                if margin[qb] > 1e-4:
                    assert np.array_equal(idx[b, h, qb, :kk], oidx[qb, :kk])


@pytest.mark.parametrize("scale_idx,D,B,H,tau,ratio", [
    (9, 128, 1, 4, 0.95, 0.0),   # the 32x32 decision scale over its 2521-key prefix
    (9, 128, 2, 2, 0.0, 0.2),    # the same with the Top-K rule
    (8, 64, 1, 3, 0.9, 0.0),     # 24x24: 576 queries (a ragged last query tile), 1497 keys
    (10, 128, 1, 2, 0.5, 0.0),   # 40x40: 1600 queries, 4121 keys (33 KV blocks)
])
def test_decision_attn_fwd_fused(scale_idx, D, B, H, tau, ratio):
    """Dense attention with the CS4A decision fused in (one launch): O and LSE against
    the fp64 oracle's dense attention, the pooled mass against the oracle's, every
    list a valid selection of the kernel's own masses and bit-exact beyond the
    margin, and the same masses as the stand-alone decision kernel."""
    d = inputs.make_qkv(20 + scale_idx, B, H, INF, D, 5)
    off = d["offsets"]
    s = scale_idx
    q_bits = d["q"][:, :, off[s]:off[s + 1]]
    k_bits, v_bits = d["k"][:, :, :off[s + 1]], d["v"][:, :, :off[s + 1]]
    st = _status()
    o, lse, cnt, idx, mass = ops.sparvar_decision_attn_fwd(_dev(q_bits), _dev(k_bits), _dev(v_bits),
                                                           tau, topk_ratio=ratio, return_mass=True,
                                                           dev_status=st)
    c2, i2, m2 = ops.sparvar_decide_blocks(_dev(q_bits), _dev(k_bits), tau, lse=lse,
                                           topk_ratio=ratio, return_mass=True)
    torch.cuda.synchronize()
    assert st.item() == 0
    o, lse = o.float().cpu().numpy(), lse.cpu().numpy()
    cnt, idx, mass, m2 = cnt.cpu().numpy(), idx.cpu().numpy(), mass.cpu().numpy(), m2.cpu().numpy()
    assert np.abs(mass - m2).max() < 2e-5
    Lq, Lkv = q_bits.shape[2], k_bits.shape[2]
    nqb, nkb = -(-Lq // 128), -(-Lkv // 128)
    for b in range(B):
        for h in range(H):
            qf, kf, vf = q_bits_f(q_bits, b, h), q_bits_f(k_bits, b, h), q_bits_f(v_bits, b, h)
            O, L = orc.masked_attention(qf, kf, vf, np.ones((nqb, nkb), bool), 128, 128)
            err = np.abs(o[b, h] - O)
            assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (b, h, err.max(), err.mean())
            assert np.abs(lse[b, h] - L).max() < 1e-3
            if ratio > 0:
                oc, oi, _, M, margin = orc.decide_blocks(qf, kf, 128, 128, None, topk_ratio=ratio)
            else:
                oc, oi, _, M, margin = orc.decide_blocks(qf, kf, 128, 128, tau)
            assert np.abs(mass[b, h] - M).max() < 2e-5
            for qb in range(nqb):
                if ratio > 0:
                    err_s = topk_selection_error(cnt[b, h, qb], idx[b, h, qb], mass[b, h, qb],
                                                 orc.topk_count(ratio, nkb))
                else:
                    err_s = mass_selection_error(cnt[b, h, qb], idx[b, h, qb], mass[b, h, qb], tau)
                assert err_s == "", (b, h, qb, err_s)
                if margin[qb] > 1e-4:
                    assert cnt[b, h, qb] == oc[qb] and np.array_equal(idx[b, h, qb], oi[qb])


@pytest.mark.parametrize("tau", [0.5, 0.99, 2.0])
def test_decide_blocks_thresholds_d64(tau):
    d = inputs.make_qkv(2, 1, 2, INF, 64, 5)
    off = d["offsets"]
    s = 8
    _decide_compare(d["q"][:, :, off[s]:off[s + 1]], d["k"][:, :, :off[s + 1]], tau)


@pytest.mark.parametrize("dst_scale", [10, 11, 12])
def test_map_indices_bit_exact(dst_scale):
    off = inputs.token_offsets(INF)
    rng = np.random.default_rng(dst_scale)
    B, H = 2, 3
    s_nq, s_lkv = 1024, off[10]
    s_nqb, s_nkb = 8, -(-s_lkv // 128)
    blk = rng.random((B, H, s_nqb, s_nkb)) < 0.3
    cnt = blk.sum(-1).astype(np.int32)
    idx = np.full((B, H, s_nqb, s_nkb), -1, np.int32)
    for b in range(B):
        for h in range(H):
            for qb in range(s_nqb):
                kept = np.nonzero(blk[b, h, qb])[0]
                idx[b, h, qb, :kept.size] = kept
    d_nq, d_lkv = INF[dst_scale] ** 2, off[dst_scale + 1]
    st = _status()
    dc, di, dm = ops.sparvar_map_indices(torch.from_numpy(cnt).cuda(), torch.from_numpy(idx).cuda(),
                                         s_nq, s_lkv, d_nq, d_lkv, 128, 128, off[5], with_mask=True,
                                         dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    for b in range(B):
        for h in range(H):
            oc, oi, ob = orc.map_indices(cnt[b, h], idx[b, h], s_nq, s_lkv, d_nq, d_lkv, 128, 128, off[5])
            assert np.array_equal(dc[b, h].cpu().numpy(), oc)
            assert np.array_equal(di[b, h].cpu().numpy(), oi)
            assert np.array_equal(dm[b, h].cpu().numpy().astype(bool), ob)


def test_map_indices_small_blocks_and_bad_entries():
    # golden case P of tests/golden/map_indices_tiny.txt with every size times 16
    # (block 32 instead of 2): the same destination blocks must come out.
    cnt = torch.tensor([[[2, 1]]], dtype=torch.int32, device="cuda")
    idx = torch.tensor([[[[1, 7, -1], [2, -1, -1]]]], dtype=torch.int32, device="cuda")
    st = _status()
    dc, di, _ = ops.sparvar_map_indices(cnt, idx, 64, 96, 128, 240, 32, 32, n_sink_tokens=16,
                                        dev_status=st)
    torch.cuda.synchronize()
    assert st.item() & ops.SPARVAR_DEV_BAD_LIST  # entry 7 is out of range and skipped
    want = [[0, 2, 3, 4], [0, 2, 3, 4], [0, 5, 6, 7], [0, 5, 6, 7]]
    for qb, w in enumerate(want):
        assert di[0, 0, qb, :dc[0, 0, qb]].tolist() == w


# ------------------------------------------------------------------ CS4A 2-D mapping
def _lists_from_blk(blk):
    B, H, nqb, nkb = blk.shape
    cnt = blk.sum(-1).astype(np.int32)
    idx = np.full((B, H, nqb, nkb), -1, np.int32)
    for b in range(B):
        for h in range(H):
            for qb in range(nqb):
                kept = np.nonzero(blk[b, h, qb])[0]
                idx[b, h, qb, :kept.size] = kept
    return cnt, idx


@pytest.mark.parametrize("sides,src,dst,bq,bk,sink", [
    (INF, 9, 10, 128, 128, 121),
    (INF, 9, 11, 128, 128, 121),
    (INF, 9, 12, 128, 128, 121),
    (INF, 9, 12, 64, 64, 121),
    (INF, 9, 9, 128, 128, 0),
    (TINY, 3, 4, 16, 16, 5),
    ((1, 2, 3, 5, 7, 11), 3, 5, 16, 32, 1),
])
def test_map_indices_2d_bit_exact(sides, src, dst, bq, bk, sink):
    off = inputs.token_offsets(sides)
    rng = np.random.default_rng(src * 100 + dst + bq)
    B, H = 2, 2
    s_nqb, s_nkb = -(-sides[src] ** 2 // bq), -(-off[src + 1] // bk)
    blk = rng.random((B, H, s_nqb, s_nkb)) < 0.25
    cnt, idx = _lists_from_blk(blk)
    st = _status()
    dc, di, dm = ops.sparvar_map_indices_2d(torch.from_numpy(cnt).cuda(),
                                            torch.from_numpy(idx).cuda(), sides, src, dst, bq, bk,
                                            sink, with_mask=True, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    for b in range(B):
        for h in range(H):
            oc, oi, ob = orc.map_indices_2d(cnt[b, h], idx[b, h], sides, src, dst, bq, bk, sink)
            assert np.array_equal(dc[b, h].cpu().numpy(), oc)
            assert np.array_equal(di[b, h].cpu().numpy(), oi)
            assert np.array_equal(dm[b, h].cpu().numpy().astype(bool), ob)


def test_cs4a_topk_2d_pipeline_attention():
    """Decision at the 32x32 scale with the Top-K rule, 2-D mapping to 64x64, then the
    block-sparse attention on the mapped lists, against the oracle end to end."""
    d = inputs.make_qkv(9, 1, 2, INF, 128, 5)
    off = d["offsets"]
    s, t = 9, 12
    qd, kd = d["q"][:, :, off[s]:off[s + 1]], d["k"][:, :, :off[s + 1]]
    dc, di, _ = ops.sparvar_decide_blocks(_dev(qd), _dev(kd), 0.95, topk_ratio=0.2)
    mc, mi, _ = ops.sparvar_map_indices_2d(dc, di, INF, s, t, 128, 128, off[5])
    q_bits = d["q"][:, :, off[t]:off[t + 1]]
    kv = slice(0, off[t + 1])
    _check_attention(q_bits, d["k"][:, :, kv], d["v"][:, :, kv], (mc, mi), 128, 128, 128,
                     lse_check=False)
    # the mapped lists equal the oracle's mapping of the kernel's own decision
    dcn, din = dc.cpu().numpy(), di.cpu().numpy()
    for h in range(2):
        oc, oi, _ = orc.map_indices_2d(dcn[0, h], din[0, h], INF, s, t, 128, 128, off[5])
        assert np.array_equal(mc[0, h].cpu().numpy(), oc)
        assert np.array_equal(mi[0, h].cpu().numpy(), oi)


# ------------------------------------------------------------------ CS4A output cache
@pytest.mark.parametrize("s_src,s_dst,D", [(32, 64, 128), (32, 40, 128), (32, 48, 64), (7, 7, 128),
                                           (5, 13, 64), (3, 17, 8), (6, 9, 72), (4, 7, 1024),
                                           (13, 5, 128)])
def test_ocache_apply_elementwise(s_src, s_dst, D):
    rng = np.random.default_rng(s_src * s_dst + D)
    B, H = 2, 3
    mk = lambda n: inputs.bf16_round(rng.standard_normal((B, H, n, D)).astype(np.float32))[0]  # noqa: E731
    t_bits, d_bits, s_bits = mk(s_dst * s_dst), mk(s_src * s_src), mk(s_src * s_src)
    t_dev = _dev(t_bits)
    # strided view for the target: every other head of a wider tensor
    wide = torch.zeros(B, 2 * H, s_dst * s_dst, D, dtype=torch.bfloat16, device="cuda")
    wide[:, ::2] = t_dev
    out = ops.sparvar_ocache_apply(wide[:, ::2], _dev(d_bits), _dev(s_bits), s_src, s_dst)
    inplace = t_dev.clone()
    ops.sparvar_ocache_apply(inplace, _dev(d_bits), _dev(s_bits), s_src, s_dst, out=inplace)
    torch.cuda.synchronize()
    assert torch.equal(out, inplace)
    got = out.float().cpu().numpy()
    for b in range(B):
        for h in range(H):
            want = orc.ocache_apply(q_bits_f(t_bits, b, h), q_bits_f(d_bits, b, h),
                                    q_bits_f(s_bits, b, h), s_src, s_dst)
            assert np.all(np.abs(got[b, h] - want) <= np.abs(want) * 2.0 ** -8 + 1e-6)


def test_cs4a_with_ocache_pipeline():
    """Decision at 32x32, the decision scale's sparse output, mapping to 40x40, the
    sparse output there corrected by the cache, against the oracle chain in fp64."""
    d = inputs.make_qkv(12, 1, 2, INF, 128, 5)
    off = d["offsets"]
    s, t = 9, 10
    qd, kd, vd = d["q"][:, :, off[s]:off[s + 1]], d["k"][:, :, :off[s + 1]], d["v"][:, :, :off[s + 1]]
    nqb, nkb = 8, -(-off[s + 1] // 128)
    dense_c = torch.full((nqb,), nkb, dtype=torch.int32, device="cuda")
    dense_i = torch.arange(nkb, dtype=torch.int32, device="cuda").repeat(nqb, 1).contiguous()
    o_dense, lse = ops.sparvar_block_sparse_attn_fwd(_dev(qd), _dev(kd), _dev(vd), dense_c, dense_i,
                                                     return_lse=True)
    dc, di, _ = ops.sparvar_decide_blocks(_dev(qd), _dev(kd), 0.0, lse=lse, topk_ratio=0.2)
    o_sparse = ops.sparvar_block_sparse_attn_fwd(_dev(qd), _dev(kd), _dev(vd), dc, di)
    qt, kt, vt = d["q"][:, :, off[t]:off[t + 1]], d["k"][:, :, :off[t + 1]], d["v"][:, :, :off[t + 1]]
    mc, mi, _ = ops.sparvar_map_indices(dc, di, 1024, off[s + 1], 1600, off[t + 1], 128, 128, off[5])
    o_t = ops.sparvar_block_sparse_attn_fwd(_dev(qt), _dev(kt), _dev(vt), mc, mi)
    out = ops.sparvar_ocache_apply(o_t, o_dense, o_sparse, INF[s], INF[t])
    torch.cuda.synchronize()
    dcn, din, mcn, min_ = dc.cpu().numpy(), di.cpu().numpy(), mc.cpu().numpy(), mi.cpu().numpy()
    for h in range(2):
        Od, _ = orc.masked_attention(q_bits_f(qd, 0, h), q_bits_f(kd, 0, h), q_bits_f(vd, 0, h),
                                     np.ones((nqb, nkb), bool), 128, 128)
        Os, _ = orc.masked_attention(q_bits_f(qd, 0, h), q_bits_f(kd, 0, h), q_bits_f(vd, 0, h),
                                     orc.lists_to_blocks(dcn[0, h], din[0, h], nkb), 128, 128)
        Ot, _ = orc.masked_attention(q_bits_f(qt, 0, h), q_bits_f(kt, 0, h), q_bits_f(vt, 0, h),
                                     orc.lists_to_blocks(mcn[0, h], min_[0, h], -(-off[t + 1] // 128)),
                                     128, 128)
        want = orc.ocache_apply(Ot, Od, Os, INF[s], INF[t])
        err = np.abs(out[0, h].float().cpu().numpy() - want)
        assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())


# ------------------------------------------------------------------ CSLA token mask
def _token_check(sides, q_scale, ns, rp, ro, B, H, D, seed, rows=None, pe=True):
    d = inputs.make_qkv(seed, B, H, sides, D, ns, pe=pe)
    off = d["offsets"]
    q_bits = d["q"][:, :, off[q_scale]:off[q_scale + 1]]
    L = off[q_scale + 1]
    cnt, idx, _ = ops.sparvar_build_csla_mask(sides, q_scale, ns, rp, ro, 128, 128)
    st = _status()
    o, lse = ops.sparvar_csla_token_attn_fwd(_dev(q_bits), _dev(d["k"][:, :, :L]),
                                             _dev(d["v"][:, :, :L]), sides, q_scale, ns, rp, ro,
                                             cnt, idx, return_lse=True, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    T = orc.csla_token_mask(sides, q_scale, ns, rp, ro)
    if rows is None:
        rows = np.arange(T.shape[0])
    o, lse = o.float().cpu().numpy(), lse.cpu().numpy()
    for b in range(B):
        for h in range(H):
            O, Lo = orc.masked_attention_tokens(q_bits_f(q_bits, b, h)[rows], q_bits_f(d["k"][:, :, :L], b, h),
                                                q_bits_f(d["v"][:, :, :L], b, h), T[rows])
            err = np.abs(o[b, h, rows] - O)
            assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (b, h, err.max(), err.mean())
            assert np.abs(lse[b, h, rows] - Lo).max() < 1e-3
    # the token mask drops keys the block path keeps: the outputs differ
    o_blk = ops.sparvar_block_sparse_attn_fwd(_dev(q_bits), _dev(d["k"][:, :, :L]),
                                              _dev(d["v"][:, :, :L]), cnt, idx).float().cpu().numpy()
    assert np.abs(o_blk - o).max() > 1e-3


@pytest.mark.parametrize("q_scale,D", [(3, 64), (4, 64), (4, 128)])
def test_csla_token_attention_tiny(q_scale, D):
    _token_check(TINY, q_scale, 2, 1, 1, 1, 2, D, 31 + q_scale, pe=False)


@pytest.mark.parametrize("q_scale,rp", [(9, 2), (10, 1), (11, 4)])
def test_csla_token_attention_infinity(q_scale, rp):
    _token_check(INF, q_scale, 5, rp, 4, 1, 2, 128, q_scale)


def test_csla_token_attention_last_scale_sampled_rows():
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([rng.integers(0, 4096, 48), [0, 63, 64, 4095]]))
    _token_check(INF, 12, 5, 2, 4, 2, 2, 128, 7, rows=rows)


# ------------------------------------------------------------------ several problems per launch
def _dense_lists(nq, L):
    nqb, nkb = -(-nq // 128), -(-L // 128)
    cnt = torch.full((nqb,), nkb, dtype=torch.int32, device="cuda")
    idx = torch.arange(nkb, dtype=torch.int32, device="cuda").repeat(nqb, 1).contiguous()
    return cnt, idx, np.ones((nqb, nkb), bool)


@pytest.mark.parametrize("sides,first_sparse,D,B,H", [(INF, 10, 128, 1, 2), (TINY, 3, 64, 1, 2)])
def test_multi_problem_launch(sides, first_sparse, D, B, H):
    """Every scale of a schedule in one launch over the shared multi-scale Q/K/V:
    dense for the early scales, CSLA lists for the late ones; each scale's rows,
    including the ragged last tile next to the following scale, against the oracle."""
    ns = 5 if sides is INF else 2
    rp, ro = (2, 4) if sides is INF else (1, 1)
    d = inputs.make_qkv(40 + D, B, H, sides, D, ns, pe=sides is INF)
    off = d["offsets"]
    q, k, v = _dev(d["q"]), _dev(d["k"]), _dev(d["v"])
    problems, blks = [], []
    for s in range(len(sides)):
        nq, L = off[s + 1] - off[s], off[s + 1]
        if s < first_sparse:
            cnt, idx, blk = _dense_lists(nq, L)
        else:
            cnt, idx, _ = ops.sparvar_build_csla_mask(sides, s, ns, rp, ro, 128, 128)
            _, _, blk = orc.build_csla_mask(sides, s, ns, rp, ro, 128, 128)
        problems.append((off[s], nq, L, cnt, idx))
        blks.append(blk)
    st = _status()
    o, lse = ops.sparvar_block_sparse_attn_fwd_multi(q, k, v, problems, return_lse=True, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    o, lse = o.float().cpu().numpy(), lse.cpu().numpy()
    rng = np.random.default_rng(D)
    for s in range(len(sides)):
        nq, L = off[s + 1] - off[s], off[s + 1]
        rows = np.arange(nq) if nq <= 600 else np.unique(np.concatenate(
            [rng.integers(0, nq, 40), [0, nq - 1, (nq - 1) // 128 * 128]]))
        for b in range(B):
            for h in range(H):
                O, Lo = orc.masked_attention_rows(rows, q_bits_f(d["q"][:, :, off[s]:off[s + 1]], b, h),
                                                  q_bits_f(d["k"][:, :, :L], b, h),
                                                  q_bits_f(d["v"][:, :, :L], b, h), blks[s], 128, 128)
                err = np.abs(o[b, h, off[s] + rows] - O)
                assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (s, b, h, err.max())
                assert np.abs(lse[b, h, off[s] + rows] - Lo).max() < 1e-3


def test_multi_problem_launch_full_size_sampled():
    """The 13 Infinity scales at B2 H16 D128 in one launch (2784 query tiles, about
    19 per CTA, so CTAs cross from one problem to the next mid-sequence): dense
    lists for scales 1-10, CSLA lists for the last three; sampled rows of every
    scale for three (batch, head) pairs, and the LSE."""
    B, H, D = 2, 16, 128
    d = inputs.make_qkv(7, B, H, INF, D, 5)
    off = d["offsets"]
    q, k, v = _dev(d["q"]), _dev(d["k"]), _dev(d["v"])
    problems, blks = [], []
    for s in range(len(INF)):
        nq, L = off[s + 1] - off[s], off[s + 1]
        if s < 10:
            cnt, idx, blk = _dense_lists(nq, L)
        else:
            cnt, idx, _ = ops.sparvar_build_csla_mask(INF, s, 5, 2, 4, 128, 128)
            _, _, blk = orc.build_csla_mask(INF, s, 5, 2, 4, 128, 128)
        problems.append((off[s], nq, L, cnt, idx))
        blks.append(blk)
    st = _status()
    o, lse = ops.sparvar_block_sparse_attn_fwd_multi(q, k, v, problems, return_lse=True, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    rng = np.random.default_rng(77)
    for s in range(len(INF)):
        nq, L = off[s + 1] - off[s], off[s + 1]
        rows = np.arange(nq) if nq <= 64 else np.unique(np.concatenate(
            [rng.integers(0, nq, 12), [0, nq - 1, (nq - 1) // 128 * 128]]))
        sel = torch.from_numpy(off[s] + rows).cuda()
        for b, h in [(0, 0), (1, 9), (0, 15)]:
            O, Lo = orc.masked_attention_rows(rows, q_bits_f(d["q"][:, :, off[s]:off[s + 1]], b, h),
                                              q_bits_f(d["k"][:, :, :L], b, h),
                                              q_bits_f(d["v"][:, :, :L], b, h), blks[s], 128, 128)
            err = np.abs(o[b, h, sel].float().cpu().numpy() - O)
            assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (s, b, h, err.max())
            assert np.abs(lse[b, h, sel].cpu().numpy() - Lo).max() < 1e-3


# ------------------------------------------------------------------ failure path
def test_bounded_wait_gives_up_and_the_context_stays_usable():
    """A wait that nothing completes gives up after its limit, raises the abort
    flag and reports SPARVAR_DEV_TIMEOUT; attention launched right after on the
    same context is still correct."""
    limit_ns = 2_000_000
    status, completed, abort, waited_us = ops.sparvar_wait_timeout_probe(limit_ns)
    assert status == 0x2 and completed == 0 and abort == 1
    assert limit_ns // 1000 <= waited_us < 1_000_000
    rng = np.random.default_rng(23)
    B, H, Lq, Lkv, D = 1, 2, 200, 300, 128
    bits = {n: inputs.bf16_round(rng.standard_normal((B, H, L, D)).astype(np.float32))[0]
            for n, L in (("q", Lq), ("k", Lkv), ("v", Lkv))}
    cnt = torch.tensor([3, 2], dtype=torch.int32, device="cuda")
    idx = torch.tensor([[0, 1, 2], [2, 0, -1]], dtype=torch.int32, device="cuda")
    _check_attention(bits["q"], bits["k"], bits["v"], (cnt, idx), 128, 128, D)
