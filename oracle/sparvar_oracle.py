"""CPU float64 oracle for SparVAR block-sparse cross-scale attention.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The CUDA library
never calls it, and it shares no code with the CUDA library: every piece of
geometry, masking and attention arithmetic below is written out again here, in
the plainest form, from the method's description.

Sources (the SparVAR pages):
  [M]   "SparVAR: Exploring Sparsity in Visual AutoRegressive Modeling for
        Training-Free Acceleration", ai.info summary, section "Methodology in
        Plain English" (CS4A and CSLA paragraphs).
  [F]   same page, section "Main Findings" (sparse decision scale 10, Top-K,
        sinks = scales <= 5, block sizes 64/128).
  [W]   same page, section "What This Paper Is About" (each scale's tokens
        attend to all tokens of all previous scales).
  [K]   same page, section "Key Contributions" items 2 and 3 (block-wise mask,
        block-wise sparse kernel).

Conventions (the plainest reading where the pages are silent):
  * scales are square; scale m (0-based) holds tokens [off[m], off[m+1]) of the
    concatenated sequence, row-major (token = off[m] + a * s_m + b);
  * queries of scale k attend to keys [0, off[k+1]) ([W]);
  * query blocks are numbered locally inside the query scale, KV blocks
    globally over the key prefix;
  * the softmax scale defaults to 1/sqrt(D);
  * inside a kept block attention is dense; the token mask only decides which
    blocks are kept ([M] CSLA: the token rule is reduced to a block rule).

Parity status: every function here is pinned by tests under ``tests/``
(closed forms, brute force, hand-derived golden fixtures, invariants).
"""
from __future__ import annotations

import math

import numpy as np


# ----------------------------------------------------------------------------
# geometry
# ----------------------------------------------------------------------------
def scale_offsets(sides):
    """off[m] = number of tokens in scales 0..m-1 (length n_scales + 1)."""
    off = [0]
    for s in sides:
        off.append(off[-1] + s * s)
    return off


def n_blocks(n, block):
    return (n + block - 1) // block


# ----------------------------------------------------------------------------
# CSLA: sink prior + cross-scale locality prior, token-wise, then blocks  [M]
# ----------------------------------------------------------------------------
def csla_token_mask(sides, q_scale, n_sink_scales, radius_prev, radius_own):
    """Token-wise CSLA mask T[q, key] for the queries of scale ``q_scale``.

    [M] CSLA: a query of a large scale is mapped to its position on the grid of
    every earlier scale and may attend there only to keys near that position,
    within a radius chosen per scale; besides, a few early tokens (the sink)
    stay visible to every query.

    * sink: keys of the first ``n_sink_scales`` scales ([F]: scale <= 5);
    * every later scale m <= q_scale: query (i, j) of the side-s_k grid projects
      to (floor(i*s_m/s_k), floor(j*s_m/s_k)); keys (a, b) of scale m with
      Chebyshev distance <= r_m from that point are kept, where
      r_m = radius_own for m == q_scale and radius_prev otherwise.

    Returns a bool array [s_k^2, off[q_scale+1]].
    """
    off = scale_offsets(sides)
    sk = sides[q_scale]
    nq = sk * sk
    L = off[q_scale + 1]
    T = np.zeros((nq, L), dtype=bool)
    n_sink_tok = off[min(n_sink_scales, q_scale + 1)]
    T[:, :n_sink_tok] = True
    qi, qj = np.divmod(np.arange(nq), sk)
    for m in range(n_sink_scales, q_scale + 1):
        sm = sides[m]
        r = radius_own if m == q_scale else radius_prev
        ci = (qi * sm) // sk
        cj = (qj * sm) // sk
        ka, kb = np.divmod(np.arange(sm * sm), sm)
        near = (np.abs(ka[None, :] - ci[:, None]) <= r) & (np.abs(kb[None, :] - cj[:, None]) <= r)
        T[:, off[m]:off[m + 1]] = near
    return T


def aggregate_to_blocks(token_mask, block_q, block_kv):
    """blk[qb, kb] = any(T) over the (block_q x block_kv) tile ([M] CSLA)."""
    nq, L = token_mask.shape
    nqb, nkb = n_blocks(nq, block_q), n_blocks(L, block_kv)
    blk = np.zeros((nqb, nkb), dtype=bool)
    for qb in range(nqb):
        rows = token_mask[qb * block_q:(qb + 1) * block_q]
        for kb in range(nkb):
            blk[qb, kb] = rows[:, kb * block_kv:(kb + 1) * block_kv].any()
    return blk


def block_lists(blk):
    """Compacted ascending KV-block lists: cnt [NQB] int32, idx [NQB, NKB] (-1 tail)."""
    nqb, nkb = blk.shape
    cnt = blk.sum(axis=1).astype(np.int32)
    idx = np.full((nqb, nkb), -1, dtype=np.int32)
    for qb in range(nqb):
        kept = np.nonzero(blk[qb])[0]
        idx[qb, :kept.size] = kept
    return cnt, idx


def build_csla_mask(sides, q_scale, n_sink_scales, radius_prev, radius_own, block_q, block_kv):
    """CSLA block mask and lists for one query scale: (cnt, idx, blk)."""
    T = csla_token_mask(sides, q_scale, n_sink_scales, radius_prev, radius_own)
    blk = aggregate_to_blocks(T, block_q, block_kv)
    cnt, idx = block_lists(blk)
    return cnt, idx, blk


def lists_to_blocks(cnt, idx, nkb):
    """Inverse of ``block_lists`` (for lists produced elsewhere)."""
    nqb = cnt.shape[0]
    blk = np.zeros((nqb, nkb), dtype=bool)
    for qb in range(nqb):
        for j in range(int(cnt[qb])):
            blk[qb, int(idx[qb, j])] = True
    return blk


# ----------------------------------------------------------------------------
# masked attention (the block-wise sparse kernel's result)  [K], [W]
# ----------------------------------------------------------------------------
def expand_block_mask(blk, nq, L, block_q, block_kv):
    """Element mask E[q, key] = blk[q // block_q, key // block_kv]."""
    rq = np.arange(nq) // block_q
    rk = np.arange(L) // block_kv
    return blk[rq][:, rk]


def masked_attention(q, k, v, blk, block_q, block_kv, scale=None, return_p=False):
    """O = softmax(scale * q k^T, masked to -inf outside kept blocks) v, in fp64.

    q [Nq, D], k [L, D], v [L, D] for one (batch, head).  Rows whose every key
    is masked give O = 0 and LSE = -inf.  Returns (O, lse[, P]).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    nq, D = q.shape
    L = k.shape[0]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    S = scale * (q @ k.T)
    E = expand_block_mask(blk, nq, L, block_q, block_kv)
    S = np.where(E, S, -np.inf)
    m = S.max(axis=1)
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    P = np.exp(S - m_safe[:, None])
    l = P.sum(axis=1)
    l_safe = np.where(empty, 1.0, l)
    P = P / l_safe[:, None]
    O = P @ v
    lse = np.where(empty, -np.inf, m_safe + np.log(l_safe))
    if return_p:
        return O, lse, P
    return O, lse


def masked_attention_tokens(q, k, v, token_mask, scale=None):
    """O = softmax(scale * q k^T, -inf where token_mask is False) v, in fp64: the
    CSLA token mask applied exactly instead of through its blocks.  Rows whose
    every key is masked give O = 0 and LSE = -inf.  Returns (O, lse)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[1])
    S = np.where(token_mask, scale * (q @ k.T), -np.inf)
    m = S.max(axis=1)
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    P = np.exp(S - m_safe[:, None])
    l = P.sum(axis=1)
    l_safe = np.where(empty, 1.0, l)
    O = (P / l_safe[:, None]) @ v
    return O, np.where(empty, -np.inf, m_safe + np.log(l_safe))


def masked_attention_rows(rows, q, k, v, blk, block_q, block_kv, scale=None):
    """The same definition evaluated for selected query rows only."""
    rows = np.asarray(rows)
    q = np.asarray(q, dtype=np.float64)
    D = q.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    L = k.shape[0]
    S = scale * (q[rows] @ k.T)
    rk = np.arange(L) // block_kv
    E = blk[rows // block_q][:, rk]
    S = np.where(E, S, -np.inf)
    m = S.max(axis=1)
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    P = np.exp(S - m_safe[:, None])
    l = P.sum(axis=1)
    l_safe = np.where(empty, 1.0, l)
    O = (P / l_safe[:, None]) @ v
    lse = np.where(empty, -np.inf, m_safe + np.log(l_safe))
    return O, lse


# ----------------------------------------------------------------------------
# CS4A: sparse decision scale -> pooled softmax mass -> block selection  [M], [F]
# ----------------------------------------------------------------------------
def decision_block_mass(q, k, block_q, block_kv, scale=None):
    """M[qb, kb] = (1/n_q(qb)) * sum_{q in qb, key in kb} softmax_row(q)[key].

    [M] CS4A: full attention at the decision scale; the map is split into
    query blocks and the attention weights are summed inside each block.  The
    softmax is the unmasked dense one over the whole key prefix.  The sum is
    divided by the number of query rows in the block so that each row of M
    sums to one.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    nq, D = q.shape
    L = k.shape[0]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    S = scale * (q @ k.T)
    S = S - S.max(axis=1, keepdims=True)
    P = np.exp(S)
    P = P / P.sum(axis=1, keepdims=True)
    nqb, nkb = n_blocks(nq, block_q), n_blocks(L, block_kv)
    M = np.zeros((nqb, nkb))
    for qb in range(nqb):
        rows = P[qb * block_q:(qb + 1) * block_q]
        for kb in range(nkb):
            M[qb, kb] = rows[:, kb * block_kv:(kb + 1) * block_kv].sum() / rows.shape[0]
    return M


def select_blocks_by_mass(M, mass_threshold):
    """Per query block keep the smallest mass-sorted set whose sum >= threshold.

    Blocks are ordered by mass, descending, ties to the smaller index; the
    shortest prefix whose running sum reaches ``mass_threshold`` is kept (all
    blocks if the total never reaches it).  Returns (blk, margin) where margin
    [NQB] is the distance of this decision from a flip: the smaller of the
    running-sum gaps around the threshold and the mass gap between the last
    kept and the first dropped block.
    """
    nqb, nkb = M.shape
    blk = np.zeros((nqb, nkb), dtype=bool)
    margin = np.full(nqb, np.inf)
    for qb in range(nqb):
        order = sorted(range(nkb), key=lambda kb: (-M[qb, kb], kb))
        run = 0.0
        t = nkb
        sums = []
        for pos, kb in enumerate(order):
            run += M[qb, kb]
            sums.append(run)
            if run >= mass_threshold:
                t = pos + 1
                break
        for kb in order[:t]:
            blk[qb, kb] = True
        gaps = []
        if t <= len(sums):
            gaps.append(abs(sums[t - 1] - mass_threshold))
        if t >= 2:
            gaps.append(abs(mass_threshold - sums[t - 2]))
        if t < nkb:
            gaps.append(M[qb, order[t - 1]] - M[qb, order[t]])
        margin[qb] = min(gaps) if gaps else np.inf
    return blk, margin


def topk_count(ratio, nkb):
    """Blocks kept per query block in the Top-K mode.

    [M] CS4A keeps the most important key blocks by a Top-K choice, and [F]
    gives 0.2 as its usual ratio; read as a ratio of the key blocks:
    k = ceil(ratio * NKB), at least 1 and at most NKB.  The product is taken with
    a 1e-6 allowance so that a ratio given in binary floating point (0.2 is
    0.2000000030 as a float32) does not round 0.2 * 20 up to 5.
    """
    return int(min(nkb, max(1, math.ceil(ratio * nkb - 1e-6))))


def select_blocks_topk(M, ratio):
    """Per query block keep the topk_count(ratio, NKB) blocks of largest mass.

    Ties are broken towards the smaller block index.  Returns (blk, margin) with
    margin [NQB] the mass gap between the last kept and the first dropped block
    (inf when every block is kept): the decision flips only if masses move by
    more than that.
    """
    nqb, nkb = M.shape
    k = topk_count(ratio, nkb)
    blk = np.zeros((nqb, nkb), dtype=bool)
    margin = np.full(nqb, np.inf)
    for qb in range(nqb):
        order = sorted(range(nkb), key=lambda kb: (-M[qb, kb], kb))
        for kb in order[:k]:
            blk[qb, kb] = True
        if k < nkb:
            margin[qb] = M[qb, order[k - 1]] - M[qb, order[k]]
    return blk, margin


def decide_blocks(q, k, block_q, block_kv, mass_threshold, scale=None, topk_ratio=None):
    """Decision-scale block selection for one (batch, head): (cnt, idx, blk, M, margin).

    The mass-threshold rule by default; the Top-K-ratio rule when ``topk_ratio``
    is given."""
    M = decision_block_mass(q, k, block_q, block_kv, scale)
    if topk_ratio is not None:
        blk, margin = select_blocks_topk(M, topk_ratio)
    else:
        blk, margin = select_blocks_by_mass(M, mass_threshold)
    cnt, idx = block_lists(blk)
    return cnt, idx, blk, M, margin


# ----------------------------------------------------------------------------
# CS4A cross-scale index mapping  [M]
# ----------------------------------------------------------------------------
def map_block_mask(src_blk, src_nq, src_lkv, dst_nq, dst_lkv, block_q, block_kv, n_sink_tokens):
    """Map kept decision-scale blocks onto a later scale's block grid.

    [M] CS4A: the kept block positions found at the decision scale are carried
    to each later, larger scale by scaling their coordinates, and the sink
    region may be appended.  Reading: each kept (qb, kb) covers the query-token interval
    [qlo, qhi) and key-token interval [klo, khi); both are rescaled
    proportionally, [floor(lo * N_dst / N_src), ceil(hi * N_dst / N_src)),
    with N the query count for the query axis and the key-prefix length for the
    key axis.  Every destination block meeting both rescaled intervals is kept;
    the union is taken over all kept source pairs, and every destination KV
    block holding a token below ``n_sink_tokens`` is added to every row.
    """
    s_nqb, s_nkb = src_blk.shape
    d_nqb, d_nkb = n_blocks(dst_nq, block_q), n_blocks(dst_lkv, block_kv)
    dst = np.zeros((d_nqb, d_nkb), dtype=bool)
    for qb in range(s_nqb):
        qlo, qhi = qb * block_q, min((qb + 1) * block_q, src_nq)
        tq_lo = (qlo * dst_nq) // src_nq
        tq_hi = -((-qhi * dst_nq) // src_nq)
        for kb in range(s_nkb):
            if not src_blk[qb, kb]:
                continue
            klo, khi = kb * block_kv, min((kb + 1) * block_kv, src_lkv)
            tk_lo = (klo * dst_lkv) // src_lkv
            tk_hi = -((-khi * dst_lkv) // src_lkv)
            for tqb in range(d_nqb):
                a, b = tqb * block_q, min((tqb + 1) * block_q, dst_nq)
                if not (a < tq_hi and tq_lo < b):
                    continue
                for tkb in range(d_nkb):
                    c, d = tkb * block_kv, min((tkb + 1) * block_kv, dst_lkv)
                    if c < tk_hi and tk_lo < d:
                        dst[tqb, tkb] = True
    for tkb in range(d_nkb):
        if tkb * block_kv < n_sink_tokens:
            dst[:, tkb] = True
    return dst


def map_indices(src_cnt, src_idx, src_nq, src_lkv, dst_nq, dst_lkv, block_q, block_kv, n_sink_tokens):
    """List form of ``map_block_mask``: (cnt, idx, blk) on the destination grid."""
    src_blk = lists_to_blocks(src_cnt, src_idx, n_blocks(src_lkv, block_kv))
    dst = map_block_mask(src_blk, src_nq, src_lkv, dst_nq, dst_lkv, block_q, block_kv, n_sink_tokens)
    cnt, idx = block_lists(dst)
    return cnt, idx, dst


def upscale_cell(i, s_src, s_dst):
    """Rows (or columns) [floor(i*s_dst/s_src), ceil((i+1)*s_dst/s_src)) of a
    side-s_dst grid covered by row (column) i of a side-s_src grid."""
    return (i * s_dst) // s_src, -((-(i + 1) * s_dst) // s_src)


def map_block_mask_2d(src_blk, sides, src_scale, dst_scale, block_q, block_kv, n_sink_tokens):
    """Scale-aware 2-D reading of the CS4A mapping (the alternative to
    ``map_block_mask``).

    [M] CS4A carries the kept positions to later, larger scales by scaling their
    coordinates, relying on the attention pattern looking alike from scale to
    scale.  Reading: a query
    token (i, j) of the decision scale (side s_d) stands for its upscaled cell of
    the target scale (side s_t): rows upscale_cell(i), columns upscale_cell(j).  A
    key keeps its position when it lies in a scale before the decision scale (the
    target's prefix holds the same tokens), and a key of the decision scale
    itself at (a, b) stands for the cell of (a, b) in the target scale's own
    tokens.  Keys of the scales between the two are reached only through the
    sink.  Every destination (query block, KV block) pair holding a mapped query
    and a mapped key of one kept source pair is kept; the union is taken over
    kept source pairs, and every KV block holding a key below ``n_sink_tokens``
    is added to every row.
    """
    off = scale_offsets(sides)
    s_d, s_t = sides[src_scale], sides[dst_scale]
    n_d, n_t = s_d * s_d, s_t * s_t
    l_d, l_t = off[src_scale + 1], off[dst_scale + 1]
    d_nqb, d_nkb = n_blocks(n_t, block_q), n_blocks(l_t, block_kv)
    dst = np.zeros((d_nqb, d_nkb), dtype=bool)

    def query_blocks(qb):
        out = set()
        for q in range(qb * block_q, min((qb + 1) * block_q, n_d)):
            i, j = divmod(q, s_d)
            r0, r1 = upscale_cell(i, s_d, s_t)
            c0, c1 = upscale_cell(j, s_d, s_t)
            for r in range(r0, r1):
                for c in range(c0, c1):
                    out.add((r * s_t + c) // block_q)
        return out

    def key_blocks(kb):
        out = set()
        for key in range(kb * block_kv, min((kb + 1) * block_kv, l_d)):
            if key < off[src_scale]:
                out.add(key // block_kv)
                continue
            a, b = divmod(key - off[src_scale], s_d)
            r0, r1 = upscale_cell(a, s_d, s_t)
            c0, c1 = upscale_cell(b, s_d, s_t)
            for r in range(r0, r1):
                for c in range(c0, c1):
                    out.add((off[dst_scale] + r * s_t + c) // block_kv)
        return out

    qsets = [query_blocks(qb) for qb in range(src_blk.shape[0])]
    ksets = [key_blocks(kb) for kb in range(src_blk.shape[1])]
    for qb, kb in zip(*np.nonzero(src_blk)):
        for tq in qsets[qb]:
            for tk in ksets[kb]:
                dst[tq, tk] = True
    if n_sink_tokens > 0:
        dst[:, :n_blocks(min(n_sink_tokens, l_t), block_kv)] = True
    return dst


def map_indices_2d(src_cnt, src_idx, sides, src_scale, dst_scale, block_q, block_kv,
                   n_sink_tokens):
    """List form of ``map_block_mask_2d``: (cnt, idx, blk) on the destination grid."""
    off = scale_offsets(sides)
    src_blk = lists_to_blocks(src_cnt, src_idx, n_blocks(off[src_scale + 1], block_kv))
    dst = map_block_mask_2d(src_blk, sides, src_scale, dst_scale, block_q, block_kv,
                            n_sink_tokens)
    cnt, idx = block_lists(dst)
    return cnt, idx, dst


# ----------------------------------------------------------------------------
# CS4A output cache  [M]
# ----------------------------------------------------------------------------
def nearest_source(i, s_src, s_dst):
    """Row (or column) of a side-s_src grid that row i of a side-s_dst grid
    upsamples from: floor(i * s_src / s_dst)."""
    return (i * s_src) // s_dst


def ocache_residual(o_dense, o_sparse):
    """[M] CS4A caches what the sparse computation leaves out at the decision
    scale.  Reading: the part of the decision scale's dense attention output that
    its own block-sparse output (with the blocks the decision keeps) misses,
    R = O_dense - O_sparse, per token and channel."""
    return np.asarray(o_dense, dtype=np.float64) - np.asarray(o_sparse, dtype=np.float64)


def ocache_upsample(r, s_src, s_dst):
    """Nearest-neighbour 2-D upsampling of a [s_src*s_src, D] token grid to
    [s_dst*s_dst, D]: target token (i, j) takes source token
    (nearest_source(i), nearest_source(j))."""
    r = np.asarray(r, dtype=np.float64)
    out = np.empty((s_dst * s_dst, r.shape[1]))
    for i in range(s_dst):
        for j in range(s_dst):
            a, b = nearest_source(i, s_src, s_dst), nearest_source(j, s_src, s_dst)
            out[i * s_dst + j] = r[a * s_src + b]
    return out


def ocache_apply(o_target, o_dense, o_sparse, s_src, s_dst):
    """[M] the cached residual, brought up to a later scale's grid, is added to
    that scale's block-sparse output."""
    return np.asarray(o_target, dtype=np.float64) + ocache_upsample(
        ocache_residual(o_dense, o_sparse), s_src, s_dst)


# ----------------------------------------------------------------------------
# FLOP accounting for the kept blocks (metric definition)
# ----------------------------------------------------------------------------
def kept_flops(blk, nq, L, block_q, block_kv, D):
    """4 * n_q(qb) * n_k(kb) * D summed over kept blocks (valid elements only)."""
    total = 0
    for qb, kb in zip(*np.nonzero(blk)):
        nqr = min((qb + 1) * block_q, nq) - qb * block_q
        nkr = min((kb + 1) * block_kv, L) - kb * block_kv
        total += 4 * nqr * nkr * D
    return total
