"""Python binding of libsparvar.so: the C-ABI calls under the same names.

Argument marshalling only: tensors are allocated by torch (device memory,
current stream), every step of the computation runs in the library's CUDA
kernels.  A missing library raises immediately; there is no fallback.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libsparvar.so")

SPARVAR_DEV_BAD_LIST = 0x1
SPARVAR_DEV_TIMEOUT = 0x2
SPARVAR_DEV_NOT_ASCENDING = 0x4

_lib = None

_i32p = ctypes.POINTER(ctypes.c_int32)
_i64p = ctypes.POINTER(ctypes.c_int64)
_vp = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float

EXPORTS = {
    "sparvar_last_error": ([], ctypes.c_char_p),
    "sparvar_version": ([], ctypes.c_char_p),
    "sparvar_scale_blocks": ([_i32p, _i, _i, _i, _i, _i32p, _i32p], _i),
    "sparvar_build_csla_mask": ([_i32p, _i, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp], _i),
    "sparvar_decide_blocks": ([_vp, _vp, _i, _i, _i, _i, _i, _i64p, _i64p, _f, _vp, _i, _i, _f,
                               _f, _vp, _vp, _vp, _vp, _vp], _i),
    "sparvar_map_indices": ([_vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp,
                             _vp], _i),
    "sparvar_block_sparse_attn_fwd": ([_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i64p, _i64p,
                                       _i64p, _i64p, _vp, _vp, _i64p, _i, _vp, _i, _i, _i, _f, _vp,
                                       _vp], _i),
    "sparvar_tile_order": ([_vp, _i, _i, _i, _i64p, _i, _vp, _vp], _i),
    "sparvar_build_csla_mask_ordered": ([_i32p, _i, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp,
                                         _vp], _i),
    "sparvar_block_sparse_attn_fwd_ordered": ([_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i64p,
                                               _i64p, _i64p, _i64p, _vp, _vp, _i64p, _i, _vp, _f,
                                               _vp, _vp], _i),
    "sparvar_map_indices_2d": ([_vp, _vp, _i, _i, _i32p, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp,
                                _vp, _vp], _i),
    "sparvar_block_sparse_attn_fwd_static": ([_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i64p,
                                              _i64p, _i64p, _i64p, _vp, _vp, _i64p, _i, _i, _f,
                                              _vp, _vp], _i),
    "sparvar_ocache_apply": ([_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i64p, _i64p, _i64p, _i64p,
                              _vp], _i),
    "sparvar_csla_token_attn_fwd": ([_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i64p, _i64p, _i64p,
                                     _i64p, _i32p, _i, _i, _i, _i, _i, _vp, _vp, _i64p, _i, _f,
                                     _vp, _vp], _i),
    "sparvar_block_sparse_attn_fwd_multi": ([_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i64p,
                                             _i64p, _i64p, _i64p, _i, _i32p, _i32p, _i32p, _vp,
                                             _vp, _i64p, _i32p, _f, _vp, _vp], _i),
    "sparvar_coarsen_lists": ([_vp, _vp, _i64p, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp],
                              _i),
    "sparvar_validate_lists": ([_vp, _vp, _i, _i, _i, _vp, _vp], _i),
    "sparvar_wait_timeout_probe": ([ctypes.c_uint64, _vp, _vp, _vp], _i),
    "sparvar_decision_attn_fwd": ([_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i64p, _i64p, _i64p,
                                   _i64p, _f, _f, _f, _vp, _vp, _vp, _vp, _vp], _i),
}


class SparvarError(RuntimeError):
    pass


def lib():
    """Load libsparvar.so (built in-tree) and declare its signatures."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise SparvarError(
                f"{LIB_PATH} is missing: build it with `python -m block_sparse_cross_sparvar_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in EXPORTS.items():
            fn = getattr(handle, name)
            fn.argtypes = args
            fn.restype = res
        _lib = handle
    return _lib


def _check(rc: int, name: str):
    if rc != 0:
        msg = lib().sparvar_last_error().decode()
        raise SparvarError(f"{name} failed (status {rc}): {msg}")


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _i64(vals):
    return (ctypes.c_int64 * len(vals))(*[int(v) for v in vals])


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _bhrd(t, name):
    if t.dim() != 4:
        raise SparvarError(f"{name} must be [B, H, rows, D], got {tuple(t.shape)}")
    if t.dtype != torch.bfloat16 or not t.is_cuda:
        raise SparvarError(f"{name} must be a CUDA bf16 tensor")
    if t.stride(3) != 1:
        raise SparvarError(f"{name} must have a contiguous last dimension")
    return _i64([t.stride(0), t.stride(1), t.stride(2)])


def scale_blocks(sides, q_scale, block_q, block_kv):
    arr = (ctypes.c_int32 * len(sides))(*sides)
    nqb, nkb = ctypes.c_int32(), ctypes.c_int32()
    _check(lib().sparvar_scale_blocks(arr, len(sides), q_scale, block_q, block_kv,
                                      ctypes.byref(nqb), ctypes.byref(nkb)), "sparvar_scale_blocks")
    return nqb.value, nkb.value


def sparvar_build_csla_mask(sides, q_scale, n_sink_scales, radius_prev, radius_own,
                            block_q=128, block_kv=128, device="cuda", with_mask=False):
    """CSLA block lists for one query scale: (kv_cnt [NQB], kv_idx [NQB, NKB], blk_mask|None)."""
    nqb, nkb = scale_blocks(sides, q_scale, block_q, block_kv)
    cnt = torch.empty(nqb, dtype=torch.int32, device=device)
    idx = torch.empty(nqb, nkb, dtype=torch.int32, device=device)
    mask = torch.empty(nqb, nkb, dtype=torch.uint8, device=device) if with_mask else None
    arr = (ctypes.c_int32 * len(sides))(*sides)
    _check(lib().sparvar_build_csla_mask(arr, len(sides), q_scale, n_sink_scales, radius_prev,
                                         radius_own, block_q, block_kv, _ptr(cnt), _ptr(idx),
                                         _ptr(mask), _stream(cnt.device)), "sparvar_build_csla_mask")
    return cnt, idx, mask


def sparvar_build_csla_mask_ordered(sides, q_scale, n_sink_scales, radius_prev, radius_own, B, H,
                                    device="cuda", done=None, out=None):
    """CSLA lists over 128x128 blocks and, from the same launch, the longest-first
    tile order for a (B, H) attention call over them: (kv_cnt, kv_idx, order).
    ``done`` is a zeroed int32 device counter the launch leaves at zero (one per
    call site that may run concurrently); allocated here when not given."""
    nqb, nkb = scale_blocks(sides, q_scale, 128, 128)
    cnt = torch.empty(nqb, dtype=torch.int32, device=device)
    idx = torch.empty(nqb, nkb, dtype=torch.int32, device=device)
    order = out if out is not None else torch.empty(B * H * nqb, dtype=torch.int32, device=device)
    if order.dtype != torch.int32 or order.numel() != B * H * nqb or not order.is_contiguous():
        raise SparvarError(f"out must be a contiguous int32 tensor of {B * H * nqb}")
    if done is None:
        done = torch.zeros(1, dtype=torch.int32, device=device)
    if done.dtype != torch.int32 or done.numel() != 1:
        raise SparvarError("done must be one int32")
    arr = (ctypes.c_int32 * len(sides))(*sides)
    _check(lib().sparvar_build_csla_mask_ordered(arr, len(sides), q_scale, n_sink_scales, radius_prev,
                                                 radius_own, B, H, _ptr(cnt), _ptr(idx), _ptr(order),
                                                 _ptr(done), _stream(cnt.device)),
           "sparvar_build_csla_mask_ordered")
    return cnt, idx, order


def _list_strides(kv_cnt, B, H):
    """List-row strides (b, h) for counts shaped [NQB], [H, NQB] or [B, H, NQB]."""
    if not kv_cnt.is_contiguous():
        raise SparvarError("kv_cnt must be contiguous")
    nqb = kv_cnt.shape[-1]
    if kv_cnt.dim() == 1:
        return (0, 0)
    if kv_cnt.dim() == 2:
        if kv_cnt.shape[0] not in (1, H):
            raise SparvarError("kv_cnt [H, NQB] does not match H")
        return (0, nqb if kv_cnt.shape[0] == H else 0)
    if kv_cnt.dim() == 3:
        if kv_cnt.shape[0] not in (1, B) or kv_cnt.shape[1] not in (1, H):
            raise SparvarError("kv_cnt [B, H, NQB] does not match B, H")
        sh = nqb if kv_cnt.shape[1] == H else 0
        sb = kv_cnt.shape[1] * nqb if kv_cnt.shape[0] == B else 0
        return (sb, sh)
    raise SparvarError("kv_cnt must be 1-, 2- or 3-D")


def sparvar_coarsen_lists(kv_cnt, kv_idx, B, H, Lq, Lkv, block, dev_status=None):
    """Fine (16/32/64) block lists -> 128x128 tile lists and per-tile masks.

    Returns (tile_cnt [Bo, Ho, NQT], tile_idx [Bo, Ho, NQT, NKT], tile_mask, same
    shape, int64 holding the uint64 bits), Bo/Ho = 1 where the input lists are
    shared across batch items/heads."""
    if kv_cnt.dtype != torch.int32 or kv_idx.dtype != torch.int32:
        raise SparvarError("kv_cnt/kv_idx must be int32")
    if kv_idx.shape[:-1] != kv_cnt.shape or not kv_idx.is_contiguous():
        raise SparvarError("kv_idx must be contiguous with shape (*kv_cnt.shape, row_len)")
    if kv_cnt.shape[-1] != -(-Lq // block):
        raise SparvarError(f"kv_cnt has {kv_cnt.shape[-1]} query blocks, expected {-(-Lq // block)}")
    sb, sh = _list_strides(kv_cnt, B, H)
    Bo, Ho = (1 if sb == 0 else B), (1 if sh == 0 else H)
    nqt, nkt = -(-Lq // 128), -(-Lkv // 128)
    dev = kv_cnt.device
    t_cnt = torch.empty(Bo, Ho, nqt, dtype=torch.int32, device=dev)
    t_idx = torch.empty(Bo, Ho, nqt, nkt, dtype=torch.int32, device=dev)
    t_mask = torch.empty(Bo, Ho, nqt, nkt, dtype=torch.int64, device=dev)
    _check(lib().sparvar_coarsen_lists(_ptr(kv_cnt), _ptr(kv_idx), _i64([sb, sh]), kv_idx.shape[-1],
                                       B, H, Lq, Lkv, block, _ptr(t_cnt), _ptr(t_idx), _ptr(t_mask),
                                       _ptr(dev_status), _stream(dev)), "sparvar_coarsen_lists")
    return t_cnt, t_idx, t_mask


def sparvar_tile_order(kv_cnt, B, H, Lq, out=None):
    """Query tiles longest list first, dealt in a serpentine to the attention
    kernel's CTAs (lists over 128x128 blocks): int32 [B * H * ceil(Lq / 128)]."""
    if kv_cnt.dtype != torch.int32:
        raise SparvarError("kv_cnt must be int32")
    nqb = -(-Lq // 128)
    if kv_cnt.shape[-1] != nqb:
        raise SparvarError(f"kv_cnt has {kv_cnt.shape[-1]} query blocks, expected {nqb}")
    T = B * H * nqb
    if out is None:
        out = torch.empty(T, dtype=torch.int32, device=kv_cnt.device)
    if out.dtype != torch.int32 or out.numel() != T or not out.is_contiguous():
        raise SparvarError(f"out must be a contiguous int32 tensor of {T} elements")
    sb, sh = _list_strides(kv_cnt, B, H)
    # counts are only ranked here (the attention call checks them against its lists)
    _check(lib().sparvar_tile_order(_ptr(kv_cnt), B, H, Lq, _i64([sb, sh]), 1 << 30, _ptr(out),
                                    _stream(kv_cnt.device)), "sparvar_tile_order")
    return out


def sparvar_block_sparse_attn_fwd(q, k, v, kv_cnt, kv_idx, block_q=128, block_kv=128,
                                  softmax_scale=None, out=None, return_lse=False, dev_status=None,
                                  tile_order=None):
    """Block-sparse attention forward: returns O (and the row LSE when asked).

    Lists over 128x128 blocks go to the kernel as they are; lists over square
    16/32/64 blocks are first coarsened to 128x128 tiles with per-tile masks.
    ``tile_order`` (from sparvar_tile_order on the same lists; 128x128 blocks only)
    sets the order in which the kernel's CTAs take the query tiles."""
    B, H, Lq, D = q.shape
    Lkv = k.shape[2]
    if k.shape != (B, H, Lkv, D) or v.shape != (B, H, Lkv, D):
        raise SparvarError("k/v must be [B, H, Lkv, D] matching q")
    qs, ks, vs = _bhrd(q, "q"), _bhrd(k, "k"), _bhrd(v, "v")
    if out is None:
        out = torch.empty_like(q, memory_format=torch.contiguous_format)
    os_ = _bhrd(out, "out")
    if kv_cnt.dtype != torch.int32 or kv_idx.dtype != torch.int32:
        raise SparvarError("kv_cnt/kv_idx must be int32")
    if kv_idx.shape[:-1] != kv_cnt.shape or not kv_idx.is_contiguous():
        raise SparvarError("kv_idx must be contiguous with shape (*kv_cnt.shape, row_len)")
    nqb = -(-Lq // block_q)
    if kv_cnt.shape[-1] != nqb:
        raise SparvarError(f"kv_cnt has {kv_cnt.shape[-1]} query blocks, expected {nqb}")
    tile_mask, mask_block = None, 0
    if (block_q, block_kv) != (128, 128):
        if block_q != block_kv or block_q not in (16, 32, 64):
            raise SparvarError(f"blocks ({block_q}, {block_kv}): 128 x 128 or square 16/32/64")
        kv_cnt, kv_idx, tile_mask = sparvar_coarsen_lists(kv_cnt, kv_idx, B, H, Lq, Lkv, block_q,
                                                          dev_status)
        mask_block = block_q
    lse = torch.empty(B, H, Lq, dtype=torch.float32, device=q.device) if return_lse else None
    scale = 1.0 / math.sqrt(D) if softmax_scale is None else float(softmax_scale)
    sb, sh = _list_strides(kv_cnt, B, H)
    if tile_order is not None:
        if tile_mask is not None:
            raise SparvarError("tile_order needs lists over 128x128 blocks")
        if (tile_order.dtype != torch.int32 or tile_order.numel() != B * H * nqb
                or not tile_order.is_contiguous()):
            raise SparvarError(f"tile_order must be a contiguous int32 tensor of {B * H * nqb}")
        _check(lib().sparvar_block_sparse_attn_fwd_ordered(
            _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Lq, Lkv, D, qs, ks, vs, os_,
            _ptr(kv_cnt), _ptr(kv_idx), _i64([sb, sh]), kv_idx.shape[-1], _ptr(tile_order), scale,
            _ptr(dev_status), _stream(q.device)), "sparvar_block_sparse_attn_fwd_ordered")
        return (out, lse) if return_lse else out
    _check(lib().sparvar_block_sparse_attn_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Lq, Lkv, D, qs, ks, vs, os_,
        _ptr(kv_cnt), _ptr(kv_idx), _i64([sb, sh]), kv_idx.shape[-1], _ptr(tile_mask), mask_block,
        128, 128, scale, _ptr(dev_status), _stream(q.device)), "sparvar_block_sparse_attn_fwd")
    return (out, lse) if return_lse else out


def sparvar_block_sparse_attn_fwd_static(q, k, v, kv_cnt, kv_idx, block, softmax_scale=None,
                                         out=None, return_lse=False, dev_status=None):
    """Fine-grid (16/32/64) attention whose tile lists live in the library's static
    device scratch: the only allocations here are the outputs, made by torch.

    The lists are checked first: the C call cannot see their shapes, and lists
    built for another block size would make the coarsening read past their end."""
    B, H, Lq, D = q.shape
    Lkv = k.shape[2]
    if block not in (16, 32, 64):
        raise SparvarError(f"block={block} not in (16, 32, 64)")
    if kv_cnt.dtype != torch.int32 or kv_idx.dtype != torch.int32:
        raise SparvarError("kv_cnt/kv_idx must be int32")
    if kv_idx.shape[:-1] != kv_cnt.shape or not kv_idx.is_contiguous():
        raise SparvarError("kv_idx must be contiguous with shape (*kv_cnt.shape, row_len)")
    if kv_cnt.shape[-1] != -(-Lq // block):
        raise SparvarError(f"kv_cnt has {kv_cnt.shape[-1]} query blocks, expected "
                           f"{-(-Lq // block)} for block={block}")
    if k.shape != (B, H, Lkv, D) or v.shape != (B, H, Lkv, D):
        raise SparvarError("k/v must be [B, H, Lkv, D] matching q")
    qs, ks, vs = _bhrd(q, "q"), _bhrd(k, "k"), _bhrd(v, "v")
    if out is None:
        out = torch.empty_like(q, memory_format=torch.contiguous_format)
    os_ = _bhrd(out, "out")
    lse = torch.empty(B, H, Lq, dtype=torch.float32, device=q.device) if return_lse else None
    scale = 1.0 / math.sqrt(D) if softmax_scale is None else float(softmax_scale)
    sb, sh = _list_strides(kv_cnt, B, H)
    _check(lib().sparvar_block_sparse_attn_fwd_static(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Lq, Lkv, D, qs, ks, vs, os_,
        _ptr(kv_cnt), _ptr(kv_idx), _i64([sb, sh]), kv_idx.shape[-1], block, scale,
        _ptr(dev_status), _stream(q.device)), "sparvar_block_sparse_attn_fwd_static")
    return (out, lse) if return_lse else out


def sparvar_csla_token_attn_fwd(q, k, v, sides, q_scale, n_sink_scales, radius_prev, radius_own,
                                kv_cnt, kv_idx, softmax_scale=None, out=None, return_lse=False,
                                dev_status=None):
    """Attention under the CSLA token mask inside the listed 128x128 tiles."""
    B, H, Lq, D = q.shape
    Lkv = k.shape[2]
    off = [0]
    for s_ in sides:
        off.append(off[-1] + s_ * s_)
    if Lq != sides[q_scale] ** 2 or Lkv != off[q_scale + 1]:
        raise SparvarError("q must hold the query scale's tokens and k/v its prefix")
    qs, ks, vs = _bhrd(q, "q"), _bhrd(k, "k"), _bhrd(v, "v")
    if out is None:
        out = torch.empty_like(q, memory_format=torch.contiguous_format)
    if kv_cnt.dtype != torch.int32 or kv_idx.dtype != torch.int32 or not kv_idx.is_contiguous():
        raise SparvarError("kv_cnt/kv_idx must be int32, kv_idx contiguous")
    lse = torch.empty(B, H, Lq, dtype=torch.float32, device=q.device) if return_lse else None
    scale = 1.0 / math.sqrt(D) if softmax_scale is None else float(softmax_scale)
    sb, sh = _list_strides(kv_cnt, B, H)
    arr = (ctypes.c_int32 * len(sides))(*sides)
    _check(lib().sparvar_csla_token_attn_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, D, qs, ks, vs, _bhrd(out, "out"), arr,
        len(sides), q_scale, n_sink_scales, radius_prev, radius_own, _ptr(kv_cnt), _ptr(kv_idx),
        _i64([sb, sh]), kv_idx.shape[-1], scale, _ptr(dev_status), _stream(q.device)),
        "sparvar_csla_token_attn_fwd")
    return (out, lse) if return_lse else out


def sparvar_block_sparse_attn_fwd_multi(q, k, v, problems, softmax_scale=None, out=None,
                                        return_lse=False, dev_status=None):
    """Several problems in one launch.  q [B,H,q_rows,D], k/v [B,H,kv_rows,D] shared;
    problems = [(q_row0, lq, lkv, kv_cnt, kv_idx), ...] with 128x128 block lists.
    Returns O [B,H,q_rows,D] (rows of no problem untouched) and, when asked, the LSE."""
    B, H, q_rows, D = q.shape
    kv_rows = k.shape[2]
    if k.shape != (B, H, kv_rows, D) or v.shape != (B, H, kv_rows, D):
        raise SparvarError("k/v must be [B, H, kv_rows, D] matching q")
    qs, ks, vs = _bhrd(q, "q"), _bhrd(k, "k"), _bhrd(v, "v")
    if out is None:
        out = torch.zeros_like(q, memory_format=torch.contiguous_format)
    os_ = _bhrd(out, "out")
    n = len(problems)
    lse = torch.full((B, H, q_rows), float("-inf"), dtype=torch.float32, device=q.device) \
        if return_lse else None
    r0 = (ctypes.c_int32 * n)(*[p[0] for p in problems])
    lq = (ctypes.c_int32 * n)(*[p[1] for p in problems])
    lkv = (ctypes.c_int32 * n)(*[p[2] for p in problems])
    cnts = (ctypes.c_void_p * n)(*[p[3].data_ptr() for p in problems])
    idxs = (ctypes.c_void_p * n)(*[p[4].data_ptr() for p in problems])
    strides, rows = [], []
    for (_, _, _, cnt, idx) in problems:
        if cnt.dtype != torch.int32 or idx.dtype != torch.int32 or not idx.is_contiguous():
            raise SparvarError("kv_cnt/kv_idx must be int32, kv_idx contiguous")
        strides += list(_list_strides(cnt, B, H))
        rows.append(idx.shape[-1])
    scale = 1.0 / math.sqrt(D) if softmax_scale is None else float(softmax_scale)
    _check(lib().sparvar_block_sparse_attn_fwd_multi(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, q_rows, kv_rows, D, qs, ks, vs, os_,
        n, r0, lq, lkv, ctypes.cast(cnts, ctypes.c_void_p), ctypes.cast(idxs, ctypes.c_void_p),
        _i64(strides), (ctypes.c_int32 * n)(*rows), scale, _ptr(dev_status), _stream(q.device)),
        "sparvar_block_sparse_attn_fwd_multi")
    return (out, lse) if return_lse else out


def sparvar_ocache_apply(o_target, o_dense, o_sparse, side_src, side_dst, out=None):
    """CS4A output cache: o_target + nearest-upsampled (o_dense - o_sparse)."""
    B, H, n_dst, D = o_target.shape
    if n_dst != side_dst * side_dst or o_dense.shape != (B, H, side_src * side_src, D) \
            or o_sparse.shape != o_dense.shape:
        raise SparvarError("o_target [B, H, side_dst^2, D]; o_dense, o_sparse [B, H, side_src^2, D]")
    if out is None:
        out = torch.empty_like(o_target, memory_format=torch.contiguous_format)
    _check(lib().sparvar_ocache_apply(
        _ptr(o_target), _ptr(o_dense), _ptr(o_sparse), _ptr(out), B, H, side_src, side_dst, D,
        _bhrd(o_target, "o_target"), _bhrd(o_dense, "o_dense"), _bhrd(o_sparse, "o_sparse"),
        _bhrd(out, "out"), _stream(o_target.device)), "sparvar_ocache_apply")
    return out


def sparvar_decide_blocks(q, k, mass_threshold, lse=None, softmax_scale=None, block_q=128,
                          block_kv=128, return_mass=False, dev_status=None, topk_ratio=0.0):
    """CS4A decision: (kv_cnt [B,H,NQB], kv_idx [B,H,NQB,NKB], mass|None).

    mass_threshold rule by default; topk_ratio > 0 keeps ceil(ratio * NKB) blocks."""
    B, H, Lq, D = q.shape
    Lkv = k.shape[2]
    qs, ks = _bhrd(q, "q"), _bhrd(k, "k")
    nqb, nkb = -(-Lq // block_q), -(-Lkv // block_kv)
    cnt = torch.empty(B, H, nqb, dtype=torch.int32, device=q.device)
    idx = torch.empty(B, H, nqb, nkb, dtype=torch.int32, device=q.device)
    mass = torch.empty(B, H, nqb, nkb, dtype=torch.float32, device=q.device) if return_mass else None
    if lse is not None and (lse.dtype != torch.float32 or not lse.is_contiguous()
                            or lse.shape != (B, H, Lq)):
        raise SparvarError("lse must be contiguous fp32 [B, H, Lq]")
    scale = 1.0 / math.sqrt(D) if softmax_scale is None else float(softmax_scale)
    _check(lib().sparvar_decide_blocks(
        _ptr(q), _ptr(k), B, H, Lq, Lkv, D, qs, ks, scale, _ptr(lse), block_q, block_kv,
        float(mass_threshold), float(topk_ratio), _ptr(cnt), _ptr(idx), _ptr(mass),
        _ptr(dev_status),
        _stream(q.device)), "sparvar_decide_blocks")
    return cnt, idx, mass


def sparvar_decision_attn_fwd(q, k, v, mass_threshold, topk_ratio=0.0, softmax_scale=None,
                              out=None, return_mass=False, dev_status=None):
    """Dense attention at the decision scale with the CS4A decision fused in.

    Returns (O [B,H,Lq,D], LSE [B,H,Lq], kv_cnt [B,H,NQB], kv_idx [B,H,NQB,NKB],
    mass [B,H,NQB,NKB] or None), 128 x 128 blocks."""
    B, H, Lq, D = q.shape
    Lkv = k.shape[2]
    if k.shape != (B, H, Lkv, D) or v.shape != (B, H, Lkv, D):
        raise SparvarError("k/v must be [B, H, Lkv, D] matching q")
    qs, ks, vs = _bhrd(q, "q"), _bhrd(k, "k"), _bhrd(v, "v")
    if out is None:
        out = torch.empty_like(q, memory_format=torch.contiguous_format)
    os_ = _bhrd(out, "out")
    nqb, nkb = -(-Lq // 128), -(-Lkv // 128)
    dev = q.device
    lse = torch.empty(B, H, Lq, dtype=torch.float32, device=dev)
    cnt = torch.empty(B, H, nqb, dtype=torch.int32, device=dev)
    idx = torch.empty(B, H, nqb, nkb, dtype=torch.int32, device=dev)
    mass = torch.empty(B, H, nqb, nkb, dtype=torch.float32, device=dev) if return_mass else None
    scale = 1.0 / math.sqrt(D) if softmax_scale is None else float(softmax_scale)
    _check(lib().sparvar_decision_attn_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Lq, Lkv, D, qs, ks, vs, os_, scale,
        float(mass_threshold), float(topk_ratio), _ptr(cnt), _ptr(idx), _ptr(mass),
        _ptr(dev_status), _stream(dev)), "sparvar_decision_attn_fwd")
    return out, lse, cnt, idx, mass


def sparvar_map_indices(src_cnt, src_idx, src_nq, src_lkv, dst_nq, dst_lkv, block_q=128,
                        block_kv=128, n_sink_tokens=0, with_mask=False, dev_status=None):
    """CS4A mapping of [B, H, NQB_src] lists onto a later scale: (cnt, idx, mask|None)."""
    if src_cnt.dim() != 3 or not src_cnt.is_contiguous() or not src_idx.is_contiguous():
        raise SparvarError("src_cnt must be contiguous [B, H, NQB_src]; src_idx contiguous")
    B, H, s_nqb = src_cnt.shape
    s_nkb = -(-src_lkv // block_kv)
    if src_idx.shape != (B, H, s_nqb, s_nkb):
        raise SparvarError(f"src_idx must be [B, H, {s_nqb}, {s_nkb}]")
    d_nqb, d_nkb = -(-dst_nq // block_q), -(-dst_lkv // block_kv)
    dev = src_cnt.device
    cnt = torch.empty(B, H, d_nqb, dtype=torch.int32, device=dev)
    idx = torch.empty(B, H, d_nqb, d_nkb, dtype=torch.int32, device=dev)
    mask = torch.empty(B, H, d_nqb, d_nkb, dtype=torch.uint8, device=dev) if with_mask else None
    _check(lib().sparvar_map_indices(
        _ptr(src_cnt), _ptr(src_idx), B, H, src_nq, src_lkv, dst_nq, dst_lkv, block_q, block_kv,
        n_sink_tokens, _ptr(cnt), _ptr(idx), _ptr(mask), _ptr(dev_status), _stream(dev)),
        "sparvar_map_indices")
    return cnt, idx, mask


def sparvar_map_indices_2d(src_cnt, src_idx, sides, src_scale, dst_scale, block_q=128,
                           block_kv=128, n_sink_tokens=0, with_mask=False, dev_status=None):
    """CS4A scale-aware 2-D mapping of [B, H, NQB_src] lists from scale src_scale to
    dst_scale of the schedule ``sides``: (cnt, idx, mask|None)."""
    if src_cnt.dim() != 3 or not src_cnt.is_contiguous() or not src_idx.is_contiguous():
        raise SparvarError("src_cnt must be contiguous [B, H, NQB_src]; src_idx contiguous")
    B, H, s_nqb = src_cnt.shape
    off = [0]
    for s in sides:
        off.append(off[-1] + s * s)
    if s_nqb != -(-sides[src_scale] ** 2 // block_q):
        raise SparvarError("src_cnt does not match the source scale's query blocks")
    s_nkb = -(-off[src_scale + 1] // block_kv)
    if src_idx.shape != (B, H, s_nqb, s_nkb):
        raise SparvarError(f"src_idx must be [B, H, {s_nqb}, {s_nkb}]")
    d_nqb, d_nkb = -(-sides[dst_scale] ** 2 // block_q), -(-off[dst_scale + 1] // block_kv)
    dev = src_cnt.device
    cnt = torch.empty(B, H, d_nqb, dtype=torch.int32, device=dev)
    idx = torch.empty(B, H, d_nqb, d_nkb, dtype=torch.int32, device=dev)
    mask = torch.empty(B, H, d_nqb, d_nkb, dtype=torch.uint8, device=dev) if with_mask else None
    arr = (ctypes.c_int32 * len(sides))(*sides)
    _check(lib().sparvar_map_indices_2d(
        _ptr(src_cnt), _ptr(src_idx), B, H, arr, len(sides), src_scale, dst_scale, block_q,
        block_kv, n_sink_tokens, _ptr(cnt), _ptr(idx), _ptr(mask), _ptr(dev_status), _stream(dev)),
        "sparvar_map_indices_2d")
    return cnt, idx, mask


def sparvar_wait_timeout_probe(limit_ns, device="cuda"):
    """Run the bounded-wait self-test on `device`: a wait that nothing completes
    gives up after `limit_ns`.  Returns (status bits, completed, abort flag,
    microseconds waited) (synchronises)."""
    device = torch.device(device)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    result = torch.full((3,), -1, dtype=torch.int32, device=device)
    _check(lib().sparvar_wait_timeout_probe(int(limit_ns), _ptr(status), _ptr(result),
                                            _stream(device)),
           "sparvar_wait_timeout_probe")
    r = result.cpu().tolist()
    return int(status.item()), r[0], r[1], r[2]


def sparvar_validate_lists(kv_cnt, kv_idx, nkb):
    """Device check of lists; returns the SPARVAR_DEV_* bits found (synchronises)."""
    status = torch.zeros(1, dtype=torch.int32, device=kv_cnt.device)
    n_rows = kv_cnt.numel()
    _check(lib().sparvar_validate_lists(_ptr(kv_cnt), _ptr(kv_idx), n_rows, kv_idx.shape[-1], nkb,
                                        _ptr(status), _stream(kv_cnt.device)),
           "sparvar_validate_lists")
    return int(status.item())
