"""The C-ABI library loads, exports every declared symbol, and rejects bad
arguments on the host (no GPU needed: nothing is enqueued on failure)."""
import ctypes
import os
import re

import pytest

from block_sparse_cross_sparvar_b200 import build, ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return ops.lib()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "sparvar.h")).read()
    return sorted(set(re.findall(r"SPARVAR_API\s+(?:const\s+)?\w+\*?\s+(sparvar_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert len(names) >= 8
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(ops.EXPORTS), "binding and header disagree"


def test_version(lib):
    assert b"sm_100a" in lib.sparvar_version()


def test_scale_blocks_host_only(lib):
    assert ops.scale_blocks([1, 2, 4, 6, 8, 12, 16, 20, 24, 32, 40, 48, 64], 12, 128, 128) == (32, 83)
    assert ops.scale_blocks([1, 2, 4, 8, 16], 4, 16, 16) == (16, 22)
    with pytest.raises(ops.SparvarError, match="q_scale"):
        ops.scale_blocks([1, 2], 5, 128, 128)


def _attn_call(lib, **over):
    i64 = lambda *v: (ctypes.c_int64 * len(v))(*v)  # noqa: E731
    args = dict(q=16, k=16, v=16, o=16, lse=0, B=1, H=1, Lq=128, Lkv=128, D=128,
                qs=i64(0, 0, 128), ks=i64(0, 0, 128), vs=i64(0, 0, 128), os=i64(0, 0, 128),
                cnt=16, idx=16, ls=i64(0, 0), row=1, tm=0, mb=0, bq=128, bk=128, scale=0.1, st=0,
                stream=0)
    args.update(over)
    vp = ctypes.c_void_p
    return lib.sparvar_block_sparse_attn_fwd(
        vp(args["q"]), vp(args["k"]), vp(args["v"]), vp(args["o"]), vp(args["lse"]), args["B"],
        args["H"], args["Lq"], args["Lkv"], args["D"], args["qs"], args["ks"], args["vs"], args["os"],
        vp(args["cnt"]), vp(args["idx"]), args["ls"], args["row"], vp(args["tm"]), args["mb"],
        args["bq"], args["bk"], args["scale"], vp(args["st"]), vp(args["stream"]))


@pytest.mark.parametrize("over,code,msg", [
    (dict(D=96), 2, "D=96"),
    (dict(bq=64), 2, "128 x 128"),
    (dict(q=0), 1, "q is NULL"),
    (dict(k=8), 1, "not 16-byte aligned"),
    (dict(Lq=0), 1, "Lq=0"),
    (dict(cnt=0), 1, "kv_cnt"),
    (dict(row=-1), 1, "idx_row_len"),
    (dict(scale=float("inf")), 1, "softmax_scale"),
    (dict(tm=16, mb=8), 2, "mask_block=8"),
    (dict(tm=16, mb=128), 2, "mask_block=128"),
])
def test_attention_rejects_bad_arguments_on_host(lib, over, code, msg):
    assert _attn_call(lib, **over) == code
    assert msg in lib.sparvar_last_error().decode()


def test_attention_rejects_bad_strides(lib):
    i64 = lambda *v: (ctypes.c_int64 * len(v))(*v)  # noqa: E731
    assert _attn_call(lib, qs=i64(0, 0, 100)) == 1
    assert "row stride" in lib.sparvar_last_error().decode()
    assert _attn_call(lib, H=2, ks=i64(0, 0, 128)) == 1
    assert "head stride" in lib.sparvar_last_error().decode()


def test_csla_rejects_bad_arguments(lib):
    sides = (ctypes.c_int32 * 3)(1, 2, 4)
    vp = ctypes.c_void_p
    assert lib.sparvar_build_csla_mask(sides, 3, 2, 1, 0, 0, 48, 128, vp(16), vp(16), vp(0), vp(0)) == 2
    assert lib.sparvar_build_csla_mask(sides, 3, 3, 1, 0, 0, 128, 128, vp(16), vp(16), vp(0), vp(0)) == 1
    assert lib.sparvar_build_csla_mask(sides, 3, 2, 1, -1, 0, 128, 128, vp(16), vp(16), vp(0), vp(0)) == 1
    bad = (ctypes.c_int32 * 3)(1, 0, 4)
    assert lib.sparvar_build_csla_mask(bad, 3, 2, 1, 0, 0, 128, 128, vp(16), vp(16), vp(0), vp(0)) == 1
    assert "sides[1]" in lib.sparvar_last_error().decode()


def test_map_and_decide_reject_bad_arguments(lib):
    vp = ctypes.c_void_p
    assert lib.sparvar_map_indices(vp(16), vp(16), 1, 1, 10, 10, 20, 20, 100, 128, 0, vp(16), vp(16),
                                   vp(0), vp(0), vp(0)) == 2
    assert lib.sparvar_map_indices(vp(0), vp(16), 1, 1, 10, 10, 20, 20, 128, 128, 0, vp(16), vp(16),
                                   vp(0), vp(0), vp(0)) == 1
    i64 = lambda *v: (ctypes.c_int64 * len(v))(*v)  # noqa: E731
    assert lib.sparvar_decide_blocks(vp(16), vp(16), 1, 1, 128, 600000, 128, i64(0, 0, 128),
                                     i64(0, 0, 128), 0.1, vp(0), 128, 128, 0.95, 0.0, vp(16),
                                     vp(16), vp(0), vp(0), vp(0)) == 2
    assert "KV blocks" in lib.sparvar_last_error().decode()
    for bad in (1.5, -0.1, float("nan")):
        assert lib.sparvar_decide_blocks(vp(16), vp(16), 1, 1, 128, 1000, 128, i64(0, 0, 128),
                                         i64(0, 0, 128), 0.1, vp(0), 128, 128, 0.95, bad, vp(16),
                                         vp(16), vp(0), vp(0), vp(0)) == 1
        assert "topk_ratio" in lib.sparvar_last_error().decode()
    assert lib.sparvar_validate_lists(vp(16), vp(16), 4, 4, 4, vp(0), vp(0)) == 1


def test_coarsen_rejects_bad_arguments(lib):
    vp = ctypes.c_void_p
    i64 = lambda *v: (ctypes.c_int64 * len(v))(*v)  # noqa: E731

    def call(block=16, B=1, H=1, Lq=256, Lkv=256, cnt=16, ls=None, row=16, lkv_ok=True):
        return lib.sparvar_coarsen_lists(vp(cnt), vp(16), ls if ls is not None else i64(0, 0), row,
                                         B, H, Lq, Lkv, block, vp(16), vp(16), vp(16), vp(0), vp(0))

    assert call(block=128) == 2 and "block=128" in lib.sparvar_last_error().decode()
    assert call(block=8) == 2
    assert call(cnt=0) == 1 and "NULL" in lib.sparvar_last_error().decode()
    assert call(Lq=0) == 1
    assert call(ls=i64(-1, 0)) == 1
    assert call(row=-1) == 1
    assert call(Lkv=4097 * 128) == 2 and "KV tiles" in lib.sparvar_last_error().decode()


def test_map_2d_rejects_bad_arguments(lib):
    vp = ctypes.c_void_p
    sides = (ctypes.c_int32 * 4)(1, 2, 4, 8)

    def call(src=2, dst=3, bq=16, bk=16, sink=0, cnt=16):
        return lib.sparvar_map_indices_2d(vp(cnt), vp(16), 1, 1, sides, 4, src, dst, bq, bk, sink,
                                          vp(16), vp(16), vp(0), vp(0), vp(0))

    assert call(src=3, dst=2) == 1 and "scales" in lib.sparvar_last_error().decode()
    assert call(dst=4) == 1
    assert call(bq=8) == 2
    assert call(sink=-1) == 1
    assert call(cnt=0) == 1


def test_ocache_rejects_bad_arguments(lib):
    vp = ctypes.c_void_p
    i64 = lambda *x: (ctypes.c_int64 * len(x))(*x)  # noqa: E731
    st = i64(0, 0, 128)

    def call(D=128, s_src=32, s_dst=64, ot=16, od=16):
        return lib.sparvar_ocache_apply(vp(ot), vp(od), vp(16), vp(16), 1, 1, s_src, s_dst, D, st, st,
                                        st, st, vp(0))

    assert call(D=12) == 2 and "D=12" in lib.sparvar_last_error().decode()
    assert call(s_src=0) == 1
    assert call(ot=0) == 1 and "o_target" in lib.sparvar_last_error().decode()
    assert call(od=8) == 1 and "aligned" in lib.sparvar_last_error().decode()


def test_multi_rejects_bad_arguments(lib):
    vp = ctypes.c_void_p
    i64 = lambda *x: (ctypes.c_int64 * len(x))(*x)  # noqa: E731
    i32 = lambda *x: (ctypes.c_int32 * len(x))(*x)  # noqa: E731
    st = i64(0, 0, 128)
    ptrs = (ctypes.c_void_p * 2)(16, 16)

    def call(n=2, r0=(0, 100), lq=(100, 200), lkv=(300, 500), q_rows=300, D=128):
        return lib.sparvar_block_sparse_attn_fwd_multi(
            vp(16), vp(16), vp(16), vp(16), vp(0), 1, 1, q_rows, 500, D, st, st, st, st, n, i32(*r0),
            i32(*lq), i32(*lkv), ctypes.cast(ptrs, vp), ctypes.cast(ptrs, vp), i64(0, 0, 0, 0),
            i32(4, 4), 0.1, vp(0), vp(0))

    assert call(n=17) == 2 and "n_problems" in lib.sparvar_last_error().decode()
    assert call(n=0) == 2
    assert call(r0=(0, 250)) == 1 and "problem 1" in lib.sparvar_last_error().decode()
    assert call(lkv=(300, 501)) == 1 and "Lkv=501" in lib.sparvar_last_error().decode()
    assert call(D=96) == 2


def test_wait_probe_rejects_bad_arguments(lib):
    vp = ctypes.c_void_p
    assert lib.sparvar_wait_timeout_probe(10**6, vp(0), vp(16), vp(0)) == 1
    assert lib.sparvar_wait_timeout_probe(10**6, vp(16), vp(0), vp(0)) == 1
    assert lib.sparvar_wait_timeout_probe(999, vp(16), vp(16), vp(0)) == 1
    assert "limit_ns=999" in lib.sparvar_last_error().decode()
    assert lib.sparvar_wait_timeout_probe(10**9 + 1, vp(16), vp(16), vp(0)) == 1


def test_tile_order_rejects_bad_arguments(lib):
    i64 = lambda *v: (ctypes.c_int64 * len(v))(*v)  # noqa: E731
    vp = ctypes.c_void_p
    cases = [((vp(0), 1, 1, 128, i64(0, 0), 1, vp(16), vp(0)), "bad lists"),
             ((vp(16), 1, 1, 128, i64(0, 0), 1, vp(0), vp(0)), "bad lists"),
             ((vp(16), 0, 1, 128, i64(0, 0), 1, vp(16), vp(0)), "B=0"),
             ((vp(16), 1, 1, 0, i64(0, 0), 1, vp(16), vp(0)), "Lq=0"),
             ((vp(16), 1, 1, 128, i64(-1, 0), 1, vp(16), vp(0)), "bad lists")]
    for args, msg in cases:
        assert lib.sparvar_tile_order(*args) == 1
        assert msg in lib.sparvar_last_error().decode()


def test_ordered_attention_rejects_bad_arguments(lib):
    i64 = lambda *v: (ctypes.c_int64 * len(v))(*v)  # noqa: E731
    vp = ctypes.c_void_p

    def call(order, D=128):
        return lib.sparvar_block_sparse_attn_fwd_ordered(
            vp(16), vp(16), vp(16), vp(16), vp(0), 1, 1, 128, 128, D, i64(0, 0, 128),
            i64(0, 0, 128), i64(0, 0, 128), i64(0, 0, 128), vp(16), vp(16), i64(0, 0), 1,
            vp(order), ctypes.c_float(0.1), vp(0), vp(0))

    assert call(0) == 1
    assert "tile_order is NULL" in lib.sparvar_last_error().decode()
    assert call(16, D=96) == 2
    assert "D=96" in lib.sparvar_last_error().decode()


def test_ordered_csla_build_rejects_bad_arguments(lib):
    vp = ctypes.c_void_p
    sides = (ctypes.c_int32 * 3)(1, 2, 4)

    def call(B=1, order=16, done=16, q_scale=2):
        return lib.sparvar_build_csla_mask_ordered(sides, 3, q_scale, 1, 1, 1, B, 1, vp(16),
                                                   vp(16), vp(order), vp(done), vp(0))

    assert call(order=0) == 1 and "order/done is NULL" in lib.sparvar_last_error().decode()
    assert call(done=0) == 1 and "order/done is NULL" in lib.sparvar_last_error().decode()
    assert call(B=0) == 1 and "B=0" in lib.sparvar_last_error().decode()
    assert call(q_scale=3) == 1 and "q_scale" in lib.sparvar_last_error().decode()
    # the order is written by one CTA that ranks at most 1024 query blocks
    wide = (ctypes.c_int32 * 2)(1, 400)  # 160000 queries: 1250 blocks of 128
    rc = lib.sparvar_build_csla_mask_ordered(wide, 2, 1, 1, 1, 1, 1, 1, vp(16), vp(16), vp(16),
                                             vp(16), vp(0))
    assert rc == 2 and "1024 query blocks" in lib.sparvar_last_error().decode()
