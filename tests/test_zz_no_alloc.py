"""The allocation-free fine-grid attention entry point (tile lists in the
library's static device scratch) against the CPU fp64 oracle and against the
allocating path, which coarsens into caller buffers.  It serves callers that
may not allocate device memory (for instance a host that hands the library
pre-sized buffers from its own pool and forbids cudaMalloc while its steps
run).  Collected last, so it also runs after every other test has used the
library."""
import ctypes

import numpy as np
import pytest
import torch

from block_sparse_cross_sparvar_b200 import build, inputs, ops
from oracle import sparvar_oracle as orc

MAX_ABS, MEAN_ABS = 2e-2, 2e-3


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
        # against the oracle: fp64 attention under the fine block mask, every row
        B, H, Lq, D = t["q"].shape
        nkb = -(-t["k"].shape[2] // block)
        f = lambda x, b, h: x[b, h].double().cpu().numpy()  # noqa: E731
        for b in range(B):
            for h in range(H):
                blk = orc.lists_to_blocks(cnt[b, h].cpu().numpy(), idx[b, h].cpu().numpy(), nkb)
                O, L = orc.masked_attention(f(t["q"], b, h), f(t["k"], b, h), f(t["v"], b, h), blk,
                                            block, block)
                err = np.abs(o_s[b, h].double().cpu().numpy() - O)
                assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (b, h, err.max())
                got = lse_s[b, h].double().cpu().numpy()
                assert np.array_equal(np.isfinite(got), np.isfinite(L))
                assert np.abs(got[np.isfinite(L)] - L[np.isfinite(L)]).max() < 1e-3
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
    _, _, blk = orc.build_csla_mask(inputs.TINY_SIDES, 4, 2, 1, 1, 16, 16)
    f = lambda bits, b, h: (bits[b, h].astype(np.uint32) << 16).view(np.float32).astype(np.float64)  # noqa: E731
    for b in range(2):
        for h in range(2):
            O, _ = orc.masked_attention(f(d["q"][:, :, off[4]:off[5]], b, h), f(d["k"], b, h),
                                        f(d["v"], b, h), blk, 16, 16)
            err = np.abs(o_s[b, h].double().cpu().numpy() - O)
            assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS


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

    # an attention argument the kernel cannot take (D = 96) is refused on the host,
    # before the scratch is looked up or the coarsening enqueued
    def call_d(D):
        return lib.sparvar_block_sparse_attn_fwd_static(
            vp(16), vp(16), vp(16), vp(16), vp(0), 1, 1, 128, 128, D, i64(0, 0, 128),
            i64(0, 0, 128), i64(0, 0, 128), i64(0, 0, 128), vp(16), vp(16), i64(1, 1), 8, 16,
            0.1, vp(0), vp(0))
    assert call_d(96) == 2 and "D=96" in lib.sparvar_last_error().decode()
    # a bad stride of q is refused the same way
    assert lib.sparvar_block_sparse_attn_fwd_static(
        vp(16), vp(16), vp(16), vp(16), vp(0), 1, 1, 128, 128, 128, i64(0, 0, 100),
        i64(0, 0, 128), i64(0, 0, 128), i64(0, 0, 128), vp(16), vp(16), i64(1, 1), 8, 16, 0.1,
        vp(0), vp(0)) == 1


def test_static_binding_refuses_lists_of_another_block_size():
    """Lists built over 64-token blocks passed with block=16 would make the coarsening
    read past the end of kv_cnt and kv_idx: the binding refuses them before any call."""
    Lq, Lkv, D = 300, 777, 64
    q = torch.zeros(1, 1, Lq, D, dtype=torch.bfloat16)
    k = torch.zeros(1, 1, Lkv, D, dtype=torch.bfloat16)
    cnt = torch.ones(-(-Lq // 64), dtype=torch.int32)
    idx = torch.zeros(-(-Lq // 64), -(-Lkv // 64), dtype=torch.int32)
    with pytest.raises(ops.SparvarError, match="query blocks"):
        ops.sparvar_block_sparse_attn_fwd_static(q, k, k, cnt, idx, 16)
    with pytest.raises(ops.SparvarError, match="block=128"):
        ops.sparvar_block_sparse_attn_fwd_static(q, k, k, cnt, idx, 128)
