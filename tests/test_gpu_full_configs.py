"""Parity at the full workload sizes the bench and its extra lines time (needs a B200).

Each test runs the library on the full-size synthetic inputs of one workload,
in the same launch configuration, and checks sampled query rows against the
CPU fp64 oracle evaluated row by row (masks and lists are checked whole where
the oracle computes them in seconds).  Tolerances as everywhere: max-abs 2e-2,
mean-abs 2e-3; lists bit-exact.
"""
import numpy as np
import pytest
import torch

from block_sparse_cross_sparvar_b200 import inputs, ops
from oracle import sparvar_oracle as orc
from tests.selection_check import mass_selection_error

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3
INF = inputs.INFINITY_SIDES
TINY = inputs.TINY_SIDES


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _f(bits):
    return (np.asarray(bits).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _sampled_check(o, q_bits, k_bits, v_bits, blk_of, pairs, rng, bq=128, bk=128, n_rows=24):
    """o: device output [B,H,Lq,D]; blk_of(b, h) -> block mask for that pair."""
    Lq = q_bits.shape[2]
    errs = []
    for b, h in pairs:
        rows = np.unique(np.concatenate([rng.integers(0, Lq, n_rows), [0, Lq - 1]]))
        O, _ = orc.masked_attention_rows(rows, _f(q_bits[b, h]), _f(k_bits[b, h]),
                                         _f(v_bits[b, h]), blk_of(b, h), bq, bk)
        got = o[b, h, torch.from_numpy(rows).cuda()].float().cpu().numpy()
        errs.append(np.abs(got - O))
    err = np.concatenate(errs)
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())
    return err.max()


def test_tiny_schedule_dense_check_block16():
    """The tiny workload with every 16x16 block kept is plain causal-by-scale attention."""
    d = inputs.make_qkv(11, 1, 2, TINY, 64, 2, pe=False)
    off = d["offsets"]
    for s in range(len(TINY)):
        q_bits = d["q"][:, :, off[s]:off[s + 1]]
        L = off[s + 1]
        nqb, nkb = -(-q_bits.shape[2] // 16), -(-L // 16)
        cnt = torch.full((nqb,), nkb, dtype=torch.int32, device="cuda")
        idx = torch.arange(nkb, dtype=torch.int32, device="cuda").repeat(nqb, 1).contiguous()
        o = ops.sparvar_block_sparse_attn_fwd(_dev(q_bits), _dev(d["k"][:, :, :L]),
                                              _dev(d["v"][:, :, :L]), cnt, idx, 16, 16)
        full = np.ones((nqb, nkb), bool)
        for h in range(2):
            O, _ = orc.masked_attention(_f(q_bits[0, h]), _f(d["k"][0, h, :L]), _f(d["v"][0, h, :L]),
                                        full, 16, 16)
            err = np.abs(o[0, h].float().cpu().numpy() - O)
            assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS


def test_cs4a_full_pass_every_scale():
    """The 13-scale CS4A pass at full size (B2 H16 D128): dense scales 1-10 with the
    decision scale's LSE, the decision (mass >= 0.95) against the oracle's, the mapped
    lists of 40x40 / 48x48 / 64x64 bit-exact against the oracle's mapping of the
    kernel's decision, and sampled rows of every scale's output."""
    B, H, D = 2, 16, 128
    d = inputs.make_qkv(0, B, H, INF, D, 5)
    off = d["offsets"]
    q_all, k_all, v_all = _dev(d["q"]), _dev(d["k"]), _dev(d["v"])
    rng = np.random.default_rng(1)
    pairs = [(0, 0), (1, 11)]
    dec = 9
    for s in range(dec + 1):
        nq, L = off[s + 1] - off[s], off[s + 1]
        nqb, nkb = -(-nq // 128), -(-L // 128)
        cnt = torch.full((nqb,), nkb, dtype=torch.int32, device="cuda")
        idx = torch.arange(nkb, dtype=torch.int32, device="cuda").repeat(nqb, 1).contiguous()
        o, lse = ops.sparvar_block_sparse_attn_fwd(q_all[:, :, off[s]:off[s + 1]], k_all[:, :, :L],
                                                   v_all[:, :, :L], cnt, idx, return_lse=True)
        _sampled_check(o, d["q"][:, :, off[s]:off[s + 1]], d["k"][:, :, :L], d["v"][:, :, :L],
                       lambda b, h: np.ones((nqb, nkb), bool), pairs, rng, n_rows=8)
    dc, di, mass = ops.sparvar_decide_blocks(q_all[:, :, off[dec]:off[dec + 1]],
                                             k_all[:, :, :off[dec + 1]], 0.95, lse=lse,
                                             return_mass=True)
    dcn, din, massn = dc.cpu().numpy(), di.cpu().numpy(), mass.cpu().numpy()
    # the decision of every (batch, head) pair: masses against the oracle's; every row a
    # valid selection of the kernel's own masses; beyond the margin the oracle's exact list
    for b in range(B):
        for h in range(H):
            oc, oi, _, M, margin = orc.decide_blocks(_f(d["q"][b, h, off[dec]:off[dec + 1]]),
                                                     _f(d["k"][b, h, :off[dec + 1]]), 128, 128, 0.95)
            assert np.abs(massn[b, h] - M).max() < 2e-5
            for qb in range(M.shape[0]):
                err = mass_selection_error(dcn[b, h, qb], din[b, h, qb], massn[b, h, qb], 0.95)
                assert err == "", (b, h, qb, err)
                if margin[qb] > 1e-4:
                    assert dcn[b, h, qb] == oc[qb] and np.array_equal(din[b, h, qb], oi[qb])
    src_nq, src_lkv = off[dec + 1] - off[dec], off[dec + 1]
    for s in range(dec + 1, len(INF)):
        nq, L = off[s + 1] - off[s], off[s + 1]
        mc, mi, _ = ops.sparvar_map_indices(dc, di, src_nq, src_lkv, nq, L, 128, 128, off[5])
        mcn, min_ = mc.cpu().numpy(), mi.cpu().numpy()
        blks = {}
        for b, h in pairs:
            oc, oi, ob = orc.map_indices(dcn[b, h], din[b, h], src_nq, src_lkv, nq, L, 128, 128,
                                         off[5])
            assert np.array_equal(mcn[b, h], oc) and np.array_equal(min_[b, h], oi)
            blks[(b, h)] = ob
        o = ops.sparvar_block_sparse_attn_fwd(q_all[:, :, off[s]:off[s + 1]], k_all[:, :, :L],
                                              v_all[:, :, :L], mc, mi)
        _sampled_check(o, d["q"][:, :, off[s]:off[s + 1]], d["k"][:, :, :L], d["v"][:, :, :L],
                       lambda b, h: blks[(b, h)], pairs, rng, n_rows=12)


@pytest.mark.parametrize("radius", [1, 4])
def test_infinity8b_last_two_scales(radius):
    """B2 H32 D128, 48x48 and 64x64 over their prefixes, CSLA with r_prev swept."""
    B, H, D = 2, 32, 128
    d = inputs.make_qkv(3, B, H, INF, D, 5)
    off = d["offsets"]
    k_all, v_all = _dev(d["k"]), _dev(d["v"])
    rng = np.random.default_rng(radius)
    for s in (11, 12):
        L = off[s + 1]
        cnt, idx, _ = ops.sparvar_build_csla_mask(INF, s, 5, radius, 4, 128, 128)
        ocnt, oidx, oblk = orc.build_csla_mask(INF, s, 5, radius, 4, 128, 128)
        assert np.array_equal(cnt.cpu().numpy(), ocnt) and np.array_equal(idx.cpu().numpy(), oidx)
        o = ops.sparvar_block_sparse_attn_fwd(_dev(d["q"][:, :, off[s]:off[s + 1]]),
                                              k_all[:, :, :L], v_all[:, :, :L], cnt, idx)
        _sampled_check(o, d["q"][:, :, off[s]:off[s + 1]], d["k"][:, :, :L], d["v"][:, :, :L],
                       lambda b, h: oblk, [(0, 0), (1, 31), (0, 17)], rng, n_rows=16)


@pytest.mark.parametrize("prefix,density", [("full", 0.05), ("full", 1.0), ("skip", 0.2),
                                            ("skip", 1.0)])
def test_density_sweep_lists(prefix, density):
    """Last scale, B2 H16 D128, Bernoulli block lists with the sink block kept, over
    the full 10521-key prefix or with the 40x40 and 48x48 scales skipped (6617 keys)."""
    B, H, D = 2, 16, 128
    d = inputs.make_qkv(0, B, H, INF, D, 5)
    off = d["offsets"]
    keys = np.arange(off[13]) if prefix == "full" else \
        np.concatenate([np.arange(off[10]), np.arange(off[12], off[13])])
    q_bits = d["q"][:, :, off[12]:off[13]]
    k_bits = np.ascontiguousarray(d["k"][:, :, keys])
    v_bits = np.ascontiguousarray(d["v"][:, :, keys])
    L = keys.size
    nqb, nkb = 32, -(-L // 128)
    rng = np.random.default_rng(int(density * 100) + L)
    keep = inputs.bernoulli_keep(rng, (B, H, nqb, nkb), density)
    keep[..., 0] = True
    cnt = torch.from_numpy(keep.sum(-1).astype(np.int32)).cuda()
    idx_np = np.full((B, H, nqb, nkb), -1, np.int32)
    for b in range(B):
        for h in range(H):
            for qb in range(nqb):
                kept = np.nonzero(keep[b, h, qb])[0]
                idx_np[b, h, qb, :kept.size] = kept
    o = ops.sparvar_block_sparse_attn_fwd(_dev(q_bits), _dev(k_bits), _dev(v_bits), cnt,
                                          torch.from_numpy(idx_np).cuda())
    _sampled_check(o, q_bits, k_bits, v_bits, lambda b, h: keep[b, h], [(0, 3), (1, 9)], rng,
                   n_rows=16)
