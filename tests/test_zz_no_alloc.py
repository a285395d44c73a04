"""The allocation-free fine-grid attention entry point (tile lists in the
library's static device scratch) against the allocating path, which coarsens
into caller buffers.  Collected last, so it also runs after every other test
has used the library."""
import ctypes

import numpy as np
import pytest
import torch

from block_sparse_cross_sparvar_b200 import build, inputs, ops


def _lists(rng, B, H, nqb, nkb, p):
    blk = rng.random((B, H, nqb, nkb)) < p
    blk[..., 0] = True
    cnt = blk.sum(-1).astype(np.int32)
    idx = np.full((B, H, nqb, nkb), -1, np.int32)
    for b in range(B):
        for h in range(H):
            for qb in range(nqb):
                kept = np.nonzero(blk[b, h, qb])[0]
                idx[b, h, qb, :kept.size] = kept
    return torch.from_numpy(cnt).cuda(), torch.from_numpy(idx).cuda()


def _problem(seed, B, H, Lq, Lkv, D):
    rng = np.random.default_rng(seed)
    t = {}
    for name, L in (("q", Lq), ("k", Lkv), ("v", Lkv)):
        bits = inputs.bf16_round(rng.standard_normal((B, H, L, D)).astype(np.float32))[0]
        t[name] = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()
    return rng, t


@pytest.mark.gpu
def test_static_scratch_matches_allocating_path_two_calls_in_a_row():
    # two different problems back to back: the second call reuses the scratch the
    # first one wrote, with other shapes, and must not see its leftovers
    cases = [(1, 2, 2, 300, 777, 128, 16), (2, 2, 3, 200, 1500, 64, 32)]
    outs = []
    for seed, B, H, Lq, Lkv, D, block in cases:
        rng, t = _problem(seed, B, H, Lq, Lkv, D)
        cnt, idx = _lists(rng, B, H, -(-Lq // block), -(-Lkv // block), 0.3)
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        o_s, lse_s = ops.sparvar_block_sparse_attn_fwd_static(t["q"], t["k"], t["v"], cnt, idx,
                                                              block, return_lse=True, dev_status=st)
        outs.append((t, cnt, idx, block, o_s, lse_s, st))
    torch.cuda.synchronize()
    for t, cnt, idx, block, o_s, lse_s, st in outs:
        assert st.item() == 0
        o_a, lse_a = ops.sparvar_block_sparse_attn_fwd(t["q"], t["k"], t["v"], cnt, idx, block,
                                                       block, return_lse=True)
        torch.cuda.synchronize()
        # the same kernels on the same tile lists: the row sums and LSE are exact; O may
        # differ by the order in which the two MMA issuers' PV products reach the
        # accumulator, a rounding-level difference
        assert torch.equal(lse_s, lse_a)
        diff = (o_s.float() - o_a.float()).abs()
        assert diff.max().item() <= 1e-2 and diff.mean().item() <= 1e-5


@pytest.mark.gpu
def test_static_scratch_shared_lists():
    # one CSLA list set shared by every batch item and head (zero list strides)
    d = inputs.make_qkv(3, 2, 2, inputs.TINY_SIDES, 64, 2, pe=False)
    off = d["offsets"]
    dev = lambda b: torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16).cuda()  # noqa: E731
    q, k, v = dev(d["q"][:, :, off[4]:off[5]]), dev(d["k"]), dev(d["v"])
    cnt, idx, _ = ops.sparvar_build_csla_mask(inputs.TINY_SIDES, 4, 2, 1, 1, 16, 16)
    o_s = ops.sparvar_block_sparse_attn_fwd_static(q, k, v, cnt, idx, 16)
    o_a = ops.sparvar_block_sparse_attn_fwd(q, k, v, cnt, idx, 16, 16)
    torch.cuda.synchronize()
    diff = (o_s.float() - o_a.float()).abs()
    assert diff.max().item() <= 1e-2 and diff.mean().item() <= 1e-5


def test_static_scratch_rejects_oversize_and_bad_blocks_on_host():
    build.build()
    lib = ops.lib()
    vp = ctypes.c_void_p
    i64 = lambda *x: (ctypes.c_int64 * len(x))(*x)  # noqa: E731

    def call(B=1, H=1, Lq=128, Lkv=128, block=16, ls=(1, 1)):
        return lib.sparvar_block_sparse_attn_fwd_static(
            vp(16), vp(16), vp(16), vp(16), vp(0), B, H, Lq, Lkv, 128, i64(0, 0, 128),
            i64(0, 0, 128), i64(0, 0, 128), i64(0, 0, 128), vp(16), vp(16), i64(*ls), 1, block,
            0.1, vp(0), vp(0))

    # 64 x 64 rows x 4096 KV tiles of 12 bytes is far above 8 MiB: refused before any launch
    assert call(B=64, H=64, Lq=128, Lkv=4096 * 128) == 2
    assert "static scratch" in lib.sparvar_last_error().decode()
    assert call(block=128) == 2 and "block=128" in lib.sparvar_last_error().decode()
    assert call(block=8) == 2
    assert call(Lq=0) == 1
    assert call(ls=(-1, 0)) == 1
