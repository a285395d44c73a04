/*
 * sparvar.h - C ABI of libsparvar.so: block-sparse cross-scale attention for
 * next-scale-prediction (VAR) transformers on NVIDIA B200 (sm_100a).
 *
 * The operations follow the SparVAR pages ("SparVAR: Exploring Sparsity in
 * Visual AutoRegressive Modeling for Training-Free Acceleration", ai.info
 * summary): section "Methodology in Plain English" defines CSLA (sink +
 * cross-scale locality mask aggregated into blocks) and CS4A (block pooling
 * of dense attention at a sparse decision scale, top-block selection, index
 * rescaling to later scales); sections "Key Contributions" (item 3) and
 * "Main Findings" (block sizes 64/128) define the block-wise sparse kernel;
 * section "What This Paper Is About" fixes that a scale's queries attend to
 * all tokens of all earlier scales and of their own scale.
 *
 * Conventions shared by every call
 *  - Scales are square; scale m (0-based) has side sides[m] and holds tokens
 *    [off[m], off[m+1]) of the concatenated sequence, off[m] = sum_{i<m} side_i^2,
 *    row-major inside a scale.
 *  - Query blocks are numbered locally inside the query scale: qb covers query
 *    rows [qb*block_q, min((qb+1)*block_q, Lq)).  KV blocks are numbered
 *    globally over the key prefix: kb covers keys [kb*block_kv, min(.., Lkv)).
 *  - A block list for one query block is an int32 count plus an int32 row of
 *    KV-block indices; the first `count` entries are used.  Lists written by
 *    this library are ascending and padded with -1.
 *  - Tensors are bf16, laid out [B][H][rows][D] with arbitrary element strides
 *    for B, H and rows and a contiguous last dimension.
 *  - Device pointers are plain CUDA device addresses; "host" marks the few
 *    arguments read from host memory during the call.
 *  - The caller allocates and owns every buffer.  Calls enqueue work on
 *    `stream` (a cudaStream_t; NULL = legacy default stream), never
 *    synchronise, and never allocate device memory.
 *  - Every call returns a sparvar_status.  Arguments are checked on the host
 *    before anything is enqueued; on failure nothing is enqueued and
 *    sparvar_last_error() describes the problem.  Problems that can only be
 *    seen on the device (a list entry out of range, a bounded wait that gave
 *    up) are OR-ed into the optional `dev_status` word as SPARVAR_DEV_* bits;
 *    kernels never trap.
 */
#ifndef SPARVAR_H_
#define SPARVAR_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SPARVAR_API __attribute__((visibility("default")))
#else
#define SPARVAR_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SPARVAR_OK = 0,
  SPARVAR_ERR_INVALID_ARG = 1,  /* bad pointer, size, stride or alignment      */
  SPARVAR_ERR_UNSUPPORTED = 2,  /* valid request outside what is implemented  */
  SPARVAR_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed           */
} sparvar_status;

/* Bits OR-ed into *dev_status by kernels. */
#define SPARVAR_DEV_BAD_LIST 0x1 /* count < 0, count > row length, or an index outside [0, nkb) */
#define SPARVAR_DEV_TIMEOUT 0x2  /* a bounded wait inside a kernel gave up; outputs are invalid  */
#define SPARVAR_DEV_NOT_ASCENDING 0x4 /* (validate only) indices not strictly ascending   */

#define SPARVAR_MAX_SCALES 32

/* Thread-local description of the last failing call on this thread. */
SPARVAR_API const char* sparvar_last_error(void);

/* Library version string. */
SPARVAR_API const char* sparvar_version(void);

/*
 * Number of query blocks and KV blocks for query scale `q_scale`:
 *   *nqb = ceil(sides[q_scale]^2 / block_q), *nkb = ceil(off[q_scale+1] / block_kv).
 * sides: host array of n_scales side lengths.  Pure host computation.
 */
SPARVAR_API int sparvar_scale_blocks(const int32_t* sides, int n_scales, int q_scale, int block_q,
                         int block_kv, int32_t* nqb, int32_t* nkb);

/*
 * CSLA block mask for the queries of scale `q_scale`
 * ("Methodology in Plain English", CSLA paragraph; sinks and windows from
 * "Main Findings").
 *
 * Token rule: query (i, j) of the side-s_k query scale keeps key token t when
 *   t < off[n_sink_scales]                                   (sink prior), or
 *   t lies in scale m, n_sink_scales <= m <= q_scale, at (a, b), with
 *   max(|a - floor(i*s_m/s_k)|, |b - floor(j*s_m/s_k)|) <= r_m, where
 *   r_m = radius_own if m == q_scale else radius_prev   (locality prior).
 * A (query block, KV block) is kept when any of its token pairs is kept.
 * The mask depends only on the geometry, so one list serves every batch item
 * and head (pass zero list strides to the attention call).
 *
 * sides      host, n_scales int32 side lengths (1 <= n_scales <= SPARVAR_MAX_SCALES).
 * block_q, block_kv  in {16, 32, 64, 128}.
 * kv_cnt     device, int32[nqb]          out: kept KV blocks per query block.
 * kv_idx     device, int32[nqb * nkb]    out: ascending kept indices, -1 padded.
 * blk_mask   device, uint8[nqb * nkb] or NULL; out: 1 = kept.
 * The kernel lets a programmatically serialized launch behind it on the stream
 * (the attention call) start at once; that launch waits for it before reading.
 */
SPARVAR_API int sparvar_build_csla_mask(const int32_t* sides, int n_scales, int q_scale,
                            int n_sink_scales, int radius_prev, int radius_own,
                            int block_q, int block_kv, int32_t* kv_cnt, int32_t* kv_idx,
                            uint8_t* blk_mask, void* stream);

/*
 * sparvar_build_csla_mask at block_q = block_kv = 128 (no blk_mask), which lets
 * the attention launch behind it start early (see sparvar_block_sparse_attn_fwd),
 * that also writes, in the same launch, the tile order of sparvar_tile_order
 * for an attention call over B batch items and H heads sharing these lists
 * (order: device int32 [B * H * nqb]; for launches on the current device).  The
 * CTA that finishes last ranks the lists: done is a device int32 the caller sets
 * to 0 once; the launch leaves it at 0.  Calls that may run at the same time
 * need their own `done`.  Errors as for sparvar_build_csla_mask, and a NULL
 * order or done is refused.
 */
SPARVAR_API int sparvar_build_csla_mask_ordered(const int32_t* sides, int n_scales, int q_scale,
                                                int n_sink_scales, int radius_prev,
                                                int radius_own, int B, int H, int32_t* kv_cnt,
                                                int32_t* kv_idx, int32_t* order, int32_t* done,
                                                void* stream);

/*
 * CS4A decision: pooled softmax mass of dense attention at the sparse decision
 * scale and per-query-block selection ("Methodology in Plain English", CS4A
 * paragraph: split the dense map into query blocks, sum the attention weights
 * in each block, keep the top blocks; decision scale from "Main Findings").
 *
 *   mass[qb, kb] = (1 / n_q(qb)) * sum_{q in qb} sum_{key in kb} exp(s(q,key) - lse(q)),
 *   s = softmax_scale * q . key over all Lkv keys (no mask), lse = log-sum-exp of row q.
 * Per query block, KV blocks are ordered by mass (descending, ties to the lower
 * index) and the shortest prefix whose running sum reaches mass_threshold is
 * kept (every block when the total stays below it).  With topk_ratio > 0 the
 * first k = ceil(topk_ratio * nkb) blocks of that order are kept instead (at
 * least one; the product is taken with a 1e-6 allowance so 0.2 * 20 gives 4):
 * the Top-K rule of the same paragraph, with the ratio 0.2 of "Main Findings".
 * Kept lists are written in ascending order.
 *
 * q [B][H][Lq][D], k [B][H][Lkv][D]: device bf16; strides in elements for
 *   (b, h, row) given by host arrays q_strides[3], k_strides[3]; row strides and
 *   base addresses 16-byte aligned; D in {64, 128}.
 * lse        device fp32 [B][H][Lq] contiguous (natural log), or NULL to have the
 *            call compute it (one extra sweep over the keys).
 * block_q = block_kv = 128.
 * mass_threshold  used when topk_ratio == 0.  topk_ratio in [0, 1].
 * kv_cnt     device int32 [B][H][nqb]; kv_idx device int32 [B][H][nqb][nkb] (-1 padded).
 * mass       device fp32 [B][H][nqb][nkb] or NULL.
 * dev_status device int32 or NULL.
 */
SPARVAR_API int sparvar_decide_blocks(const void* q, const void* k, int B, int H, int Lq, int Lkv, int D,
                          const int64_t* q_strides, const int64_t* k_strides,
                          float softmax_scale, const float* lse, int block_q, int block_kv,
                          float mass_threshold, float topk_ratio, int32_t* kv_cnt,
                          int32_t* kv_idx, float* mass, int32_t* dev_status, void* stream);

/*
 * Dense attention at the CS4A decision scale with the decision fused in: one
 * launch computes O and the row LSE of attention over the whole key prefix
 * (every KV block, no mask) and, from the same score tiles, the pooled mass and
 * the selected lists of sparvar_decide_blocks ("Methodology in Plain English",
 * CS4A paragraph: full attention at the decision scale, its weights summed per
 * block, the top blocks kept).  Each 128-row query tile walks the prefix twice:
 * a first sweep of score MMAs forms each row's log-sum-exp, the second computes
 * P = exp(s - lse) (normalised), O += P V and the per-block sums of P.
 *
 * q, o [B][H][Lq][D], k, v [B][H][Lkv][D]: device bf16 with element strides for
 *   (b, h, row) in host arrays *_strides[3]; last dim contiguous; base addresses
 *   and row strides 16-byte aligned; D in {64, 128}.  ceil(Lkv / 128) <= 128.
 * lse        device fp32 [B][H][Lq] (natural log) or NULL.
 * softmax_scale, mass_threshold, topk_ratio: as for sparvar_decide_blocks
 *   (blocks of 128 x 128).
 * kv_cnt     device int32 [B][H][nqb]; kv_idx device int32 [B][H][nqb][nkb]: out.
 * mass       device fp32 [B][H][nqb][nkb] or NULL: out.
 * dev_status device int32 or NULL (SPARVAR_DEV_TIMEOUT on a wait that gave up).
 * Errors: SPARVAR_ERR_UNSUPPORTED for D or the key count, SPARVAR_ERR_INVALID_ARG
 * for bad pointers, strides or sizes; nothing is enqueued on an error return.
 */
SPARVAR_API int sparvar_decision_attn_fwd(const void* q, const void* k, const void* v, void* o,
                                          float* lse, int B, int H, int Lq, int Lkv, int D,
                                          const int64_t* q_strides, const int64_t* k_strides,
                                          const int64_t* v_strides, const int64_t* o_strides,
                                          float softmax_scale, float mass_threshold,
                                          float topk_ratio, int32_t* kv_cnt, int32_t* kv_idx,
                                          float* mass, int32_t* dev_status, void* stream);

/*
 * CS4A cross-scale index mapping ("Methodology in Plain English", CS4A
 * paragraph: kept positions are rescaled to a later, larger scale, optionally
 * adding the sink region).
 *
 * A kept source block covering query rows [qlo, qhi) and keys [klo, khi) covers
 * destination query rows [floor(qlo*dst_nq/src_nq), ceil(qhi*dst_nq/src_nq)) and
 * keys [floor(klo*dst_lkv/src_lkv), ceil(khi*dst_lkv/src_lkv)); every destination
 * block meeting both ranges is kept.  The union over all kept source blocks is
 * taken, and every destination KV block holding a key < n_sink_tokens is kept in
 * every row.
 *
 * src_cnt  device int32 [B][H][src_nqb]; src_idx device int32 [B][H][src_nqb][src_nkb]
 *          (src_nqb = ceil(src_nq/block_q), src_nkb = ceil(src_lkv/block_kv)).
 * dst_cnt  device int32 [B][H][dst_nqb]; dst_idx device int32 [B][H][dst_nqb][dst_nkb].
 * dst_blk_mask device uint8 [B][H][dst_nqb][dst_nkb] or NULL.
 * block_q, block_kv in {16, 32, 64, 128}.  dev_status device int32 or NULL
 * (SPARVAR_DEV_BAD_LIST for source entries out of range; they are skipped).
 */
SPARVAR_API int sparvar_map_indices(const int32_t* src_cnt, const int32_t* src_idx, int B, int H,
                        int src_nq, int src_lkv, int dst_nq, int dst_lkv, int block_q,
                        int block_kv, int n_sink_tokens, int32_t* dst_cnt, int32_t* dst_idx,
                        uint8_t* dst_blk_mask, int32_t* dev_status, void* stream);

/*
 * CS4A cross-scale index mapping, scale-aware 2-D reading ("Methodology in
 * Plain English", CS4A paragraph: kept positions rescaled to a later, larger
 * scale, which the pages call scale self-similar; this library's alternative
 * to the proportional 1-D reading of sparvar_map_indices).
 *
 * On the schedule `sides` (host, n_scales int32), the decision scale src_scale
 * (side s_d) and a target dst_scale >= src_scale (side s_t): a decision-scale
 * query (i, j) stands for the target queries in rows
 * [floor(i*s_t/s_d), ceil((i+1)*s_t/s_d)) and the same range of columns; a key
 * of a scale before src_scale keeps its index; a decision-scale key (a, b)
 * stands for the same upscaled cell of the target scale's own tokens.  For
 * each kept source (qb, kb) every destination (query block, KV block) holding a
 * mapped query and a mapped key of that pair is kept; the union over kept
 * pairs is taken and every destination KV block holding a key < n_sink_tokens
 * is kept in every row.  Keys of the scales between the two are reached only
 * through the sink.
 *
 * src_cnt  device int32 [B][H][src_nqb]; src_idx device int32 [B][H][src_nqb][src_nkb]
 *          (src_nqb = ceil(s_d^2/block_q), src_nkb = ceil(prefix(src_scale)/block_kv)).
 * dst_cnt  device int32 [B][H][dst_nqb]; dst_idx device int32 [B][H][dst_nqb][dst_nkb]
 *          (dst_nqb = ceil(s_t^2/block_q), dst_nkb = ceil(prefix(dst_scale)/block_kv)),
 *          ascending, -1 padded.  dst_blk_mask device uint8 [B][H][dst_nqb][dst_nkb] or NULL.
 * block_q, block_kv in {16, 32, 64, 128}.  dev_status device int32 or NULL
 * (SPARVAR_DEV_BAD_LIST for source counts or entries out of range; skipped).
 */
SPARVAR_API int sparvar_map_indices_2d(const int32_t* src_cnt, const int32_t* src_idx, int B,
                                       int H, const int32_t* sides, int n_scales, int src_scale,
                                       int dst_scale, int block_q, int block_kv, int n_sink_tokens,
                                       int32_t* dst_cnt, int32_t* dst_idx, uint8_t* dst_blk_mask,
                                       int32_t* dev_status, void* stream);

/*
 * Block-sparse attention forward ("Key Contributions" item 3, "Main
 * Findings" block-size rows; scale-causal prefix from "What This Paper Is
 * About"):
 *
 *   O[q] = sum_key softmax_key(s(q,key)) V[key],  s = softmax_scale * Q[q].K[key],
 *   keys restricted to the KV blocks listed for q's query block (dense inside a
 *   block, key < Lkv).  A row with an empty list gives O = 0 and lse = -inf.
 *
 * q [B][H][Lq][D], k and v [B][H][Lkv][D], o [B][H][Lq][D]: device bf16, strides in
 *   elements for (b, h, row) from host arrays *_strides[3]; last dim contiguous;
 *   base addresses and row strides 16-byte aligned.  D in {64, 128}.
 * lse        device fp32 [B][H][Lq] contiguous (natural log) or NULL.
 * kv_cnt     device int32; the count of (b, h, qb) is at
 *            kv_cnt[b*list_strides[0] + h*list_strides[1] + qb].
 * kv_idx     device int32; its list is the idx_row_len entries starting at
 *            kv_idx[(b*list_strides[0] + h*list_strides[1] + qb) * idx_row_len].
 *            list_strides (host, 2 values, in list rows) may be 0 to share one
 *            list set across batch items or heads.
 * tile_mask  device uint64 or NULL.  NULL: the lists name whole 128x128 blocks.
 *            Otherwise the lists name 128x128 tiles of a finer square block grid
 *            of side mask_block (16, 32 or 64; g = 128 / mask_block), as written
 *            by sparvar_coarsen_lists: entry e of list row r has its mask at
 *            tile_mask[r * idx_row_len + e], and bit (qi * g + ki) keeps fine KV
 *            block ki of the tile for the tile's fine query block qi.  Keys of a
 *            fine block whose bit is clear are excluded for that block's rows.
 * mask_block ignored when tile_mask is NULL.
 * block_q = block_kv = 128 (the tile size of the lists).
 * dev_status device int32 or NULL: SPARVAR_DEV_BAD_LIST when an entry is out of
 *            range (the entry contributes nothing), SPARVAR_DEV_TIMEOUT when a
 *            bounded wait gave up.
 * Stream order: the kernel is launched with programmatic stream serialization,
 *   so its CTAs may start while the kernel ahead of it on `stream` finishes (when
 *   that kernel allows it, as the list builders do); they read no input before
 *   that kernel has completed, so the usual stream order holds for every buffer.
 */
SPARVAR_API int sparvar_block_sparse_attn_fwd(const void* q, const void* k, const void* v, void* o,
                                  float* lse, int B, int H, int Lq, int Lkv, int D,
                                  const int64_t* q_strides, const int64_t* k_strides,
                                  const int64_t* v_strides, const int64_t* o_strides,
                                  const int32_t* kv_cnt, const int32_t* kv_idx,
                                  const int64_t* list_strides, int idx_row_len,
                                  const uint64_t* tile_mask, int mask_block, int block_q,
                                  int block_kv, float softmax_scale, int32_t* dev_status,
                                  void* stream);

/*
 * Longest lists first, wave by wave (a scheduling aid for the persistent
 * attention kernel; the pages fix no tile order): writes into order[T], T = B * H *
 * ceil(Lq / 128), the tile ids (b * H + h) * nqb + qb for the kernel's
 * G = min(T, SMs of the current device) CTAs, CTA c taking positions c, c + G, ...
 * Round r holds the natural tiles r*G .. r*G + G - 1 (so that each wave of the
 * kernel touches the same heads' K/V as in natural order), ranked longest list
 * first, then by query block qb, then by tile id, and dealt to CTAs 0..G-1 for
 * even r and G-1..0 for odd
 * r, so that each CTA's total work is close to the mean.  kv_cnt, list_strides
 * and idx_row_len as for sparvar_block_sparse_attn_fwd with 128x128 blocks;
 * order is device int32 owned by the caller.  One launch of one CTA on `stream`
 * (G compares per tile); the order depends on the device's SM count, so it is for
 * launches on that device.  Errors: a bad shape or pointer is refused before
 * anything is enqueued.
 */
SPARVAR_API int sparvar_tile_order(const int32_t* kv_cnt, int B, int H, int Lq,
                                   const int64_t* list_strides, int idx_row_len, int32_t* order,
                                   void* stream);

/*
 * sparvar_block_sparse_attn_fwd over 128x128 block lists (no tile mask), the
 * kernel's CTAs taking the query tiles in the order written by sparvar_tile_order
 * for the same lists and device (tile_order, device int32 [T], not NULL).  The
 * result does not depend on the order; only the balance of the CTAs' work does.
 */
SPARVAR_API int sparvar_block_sparse_attn_fwd_ordered(
    const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Lq,
    int Lkv, int D, const int64_t* q_strides, const int64_t* k_strides, const int64_t* v_strides,
    const int64_t* o_strides, const int32_t* kv_cnt, const int32_t* kv_idx,
    const int64_t* list_strides, int idx_row_len, const int32_t* tile_order, float softmax_scale,
    int32_t* dev_status, void* stream);

/*
 * Fine block lists to 128x128 tile lists with per-tile bitmasks, the form the
 * attention call takes for block sizes below 128 ("Main Findings" block-size
 * rows: the mask is defined on a fine grid, the contraction runs on 128x128
 * tensor-core tiles).
 *
 * Input: lists over square blocks of side `block` (16, 32 or 64) for queries
 *   [0, Lq) and keys [0, Lkv): count of (b, h, fine query block qb) at
 *   kv_cnt[b*list_strides[0] + h*list_strides[1] + qb], entries (fine KV block
 *   indices) from kv_idx[(that row) * idx_row_len]; list_strides (host, 2 values)
 *   may be 0 to share lists.
 * Output, for Bo = (list_strides[0] == 0 ? 1 : B) and Ho = (list_strides[1] == 0
 *   ? 1 : H), NQT = ceil(Lq/128), NKT = ceil(Lkv/128) (NKT <= 4096):
 *   tile_cnt int32 [Bo][Ho][NQT], tile_idx int32 [Bo][Ho][NQT][NKT] (ascending,
 *   -1 padded), tile_mask uint64 [Bo][Ho][NQT][NKT] (0 padded), all device,
 *   caller-allocated.  Pass them to sparvar_block_sparse_attn_fwd with
 *   list_strides {Bo > 1 ? Ho*NQT : 0, Ho > 1 ? NQT : 0}, idx_row_len NKT and
 *   mask_block = block.
 * dev_status device int32 or NULL: SPARVAR_DEV_BAD_LIST for counts or entries out
 *   of range (skipped).  Duplicated entries are harmless.
 */
SPARVAR_API int sparvar_coarsen_lists(const int32_t* kv_cnt, const int32_t* kv_idx,
                                      const int64_t* list_strides, int idx_row_len, int B, int H,
                                      int Lq, int Lkv, int block, int32_t* tile_cnt,
                                      int32_t* tile_idx, uint64_t* tile_mask,
                                      int32_t* dev_status, void* stream);

/*
 * Several block-sparse attention problems in one launch (for instance the scales
 * of one generation step, which share the Q, K and V tensors of the whole
 * multi-scale sequence): the persistent kernel walks the query tiles of all
 * problems as one work list, so small scales do not each pay a launch and a
 * tail.  Problem i is sparvar_block_sparse_attn_fwd on query rows
 * [q_row0[i], q_row0[i] + lq[i]) of q and o, keys [0, lkv[i]) of k and v, with
 * lists kv_cnt[i], kv_idx[i] (device pointers in host arrays), list strides
 * list_strides[2i], list_strides[2i+1] and row length idx_row_len[i]; the blocks
 * are 128 x 128 (no fine grids).
 *
 * q, o [B][H][q_rows][D]; k, v [B][H][kv_rows][D]: device bf16, strides and
 * alignment as for sparvar_block_sparse_attn_fwd, D in {64, 128}.  lse device
 * fp32 [B][H][q_rows] or NULL (rows of no problem are not written).  1 <=
 * n_problems <= 16; query row ranges must not overlap.  The problems' results
 * are those of separate calls (up to the order in which PV products reach the
 * accumulator).
 */
SPARVAR_API int sparvar_block_sparse_attn_fwd_multi(
    const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int q_rows,
    int kv_rows, int D, const int64_t* q_strides, const int64_t* k_strides,
    const int64_t* v_strides, const int64_t* o_strides, int n_problems, const int32_t* q_row0,
    const int32_t* lq, const int32_t* lkv, const int32_t* const* kv_cnt,
    const int32_t* const* kv_idx, const int64_t* list_strides, const int32_t* idx_row_len,
    float softmax_scale, int32_t* dev_status, void* stream);

/*
 * Block-sparse attention with the CSLA token mask applied inside the kept tiles
 * ("Methodology in Plain English", CSLA paragraph: the token-wise mask, here used
 * as it is rather than only through its blocks): O[q] = sum_key softmax(s(q,key)) V[key] over the keys the CSLA token
 * rule of sparvar_build_csla_mask keeps for q, taken from the listed 128x128
 * tiles (pass the lists sparvar_build_csla_mask writes at block 128; a key the
 * rule keeps outside the listed tiles does not contribute).
 *
 * Geometry (host sides[n_scales], q_scale, n_sink_scales, radius_prev,
 * radius_own) as for sparvar_build_csla_mask; Lq = sides[q_scale]^2 and Lkv =
 * the prefix length through q_scale.  q, k, v, o, lse, the lists, the scale and
 * dev_status as for sparvar_block_sparse_attn_fwd (D in {64, 128}).  A query
 * whose kept keys all fall outside the listed tiles gets O = 0, lse = -inf.
 */
SPARVAR_API int sparvar_csla_token_attn_fwd(const void* q, const void* k, const void* v, void* o,
                                            float* lse, int B, int H, int D,
                                            const int64_t* q_strides, const int64_t* k_strides,
                                            const int64_t* v_strides, const int64_t* o_strides,
                                            const int32_t* sides, int n_scales, int q_scale,
                                            int n_sink_scales, int radius_prev, int radius_own,
                                            const int32_t* kv_cnt, const int32_t* kv_idx,
                                            const int64_t* list_strides, int idx_row_len,
                                            float softmax_scale, int32_t* dev_status,
                                            void* stream);

/*
 * CS4A output cache ("Methodology in Plain English", CS4A paragraph: what the
 * sparse computation misses at the decision scale is kept and, brought to a
 * later scale's grid, corrects that scale's sparse output; "Main Findings":
 * the cache is worth about 0.7 dB of PSNR):
 *
 *   out[t] = o_target[t] + o_dense[src(t)] - o_sparse[src(t)],
 *
 * for target token t = (i, j) of the side-side_dst scale and src(t) the token
 * (floor(i*side_src/side_dst), floor(j*side_src/side_dst)) of the side-side_src
 * decision scale (nearest-neighbour upsampling); o_dense and o_sparse are the
 * decision scale's dense output and its block-sparse output with the lists the
 * decision keeps.  Computed in fp32 from the bf16 inputs, rounded to bf16.
 *
 * o_target, out [B][H][side_dst^2][D]; o_dense, o_sparse [B][H][side_src^2][D]: device
 *   bf16 with element strides for (b, h, row) from host arrays *_strides[3]; last dim
 *   contiguous; base addresses and strides 16-byte aligned.  D a multiple of 8 in
 *   [8, 1024].  out may be o_target (in place); it must not overlap the other inputs.
 */
SPARVAR_API int sparvar_ocache_apply(const void* o_target, const void* o_dense,
                                     const void* o_sparse, void* out, int B, int H,
                                     int side_src, int side_dst, int D,
                                     const int64_t* t_strides, const int64_t* d_strides,
                                     const int64_t* s_strides, const int64_t* out_strides,
                                     void* stream);

/*
 * Fine-grid attention that allocates nothing: the same result as
 * sparvar_coarsen_lists followed by sparvar_block_sparse_attn_fwd with
 * mask_block = block, with the tile lists and masks held in a static device
 * array of the library (8 MiB per device, its address looked up once per
 * device).  The pages have no counterpart; this is for callers that cannot
 * allocate device memory.
 *
 * Arguments as for sparvar_block_sparse_attn_fwd, with kv_cnt/kv_idx/list_strides/
 * idx_row_len describing lists over square blocks of side `block` (16, 32 or 64)
 * as for sparvar_coarsen_lists.  Returns SPARVAR_ERR_UNSUPPORTED, enqueuing
 * nothing, when the tile lists would not fit: Bo*Ho*ceil(Lq/128) rows of
 * 4 + 12*ceil(Lkv/128) bytes (each part rounded up to 256 bytes), with Bo and Ho
 * as for sparvar_coarsen_lists.
 *
 * The scratch is shared by every call on the device: calls must be ordered
 * (one stream, or ordered by events); two calls in flight at once on different
 * streams or host threads overwrite each other's tile lists.  Each call's
 * coarsening writes every scratch byte its attention launch reads, so nothing
 * must start at zero.
 */
SPARVAR_API int sparvar_block_sparse_attn_fwd_static(
    const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Lq,
    int Lkv, int D, const int64_t* q_strides, const int64_t* k_strides, const int64_t* v_strides,
    const int64_t* o_strides, const int32_t* kv_cnt, const int32_t* kv_idx,
    const int64_t* list_strides, int idx_row_len, int block, float softmax_scale,
    int32_t* dev_status, void* stream);

/*
 * Device-side check of block lists: for each of n_rows rows,
 * 0 <= cnt <= min(idx_row_len, nkb), entries in [0, nkb) and strictly ascending.
 * ORs SPARVAR_DEV_BAD_LIST / SPARVAR_DEV_NOT_ASCENDING into *dev_status (required).
 * kv_cnt int32[n_rows], kv_idx int32[n_rows * idx_row_len], both device.
 */
SPARVAR_API int sparvar_validate_lists(const int32_t* kv_cnt, const int32_t* kv_idx, int n_rows,
                           int idx_row_len, int nkb, int32_t* dev_status, void* stream);

/*
 * Self-test of the failure path every kernel of the library shares (no
 * counterpart in the pages): one GPU thread waits on a shared-memory mbarrier
 * that nothing completes, using the same bounded wait as the attention
 * pipeline.  After limit_ns nanoseconds (1e3 <= limit_ns <= 1e9) it gives up,
 * ORs SPARVAR_DEV_TIMEOUT into *dev_status and returns; the CUDA context stays
 * usable.  result (device int32[3], written): [0] 1 if the wait completed
 * (never expected), 0 if it gave up; [1] the CTA's abort flag afterwards (1);
 * [2] microseconds spent waiting.  dev_status and result are device pointers
 * owned by the caller; nothing is synchronised.  Returns SPARVAR_ERR_INVALID_ARG
 * for null pointers or a limit outside the range, SPARVAR_ERR_CUDA on a launch
 * failure.
 */
SPARVAR_API int sparvar_wait_timeout_probe(uint64_t limit_ns, int32_t* dev_status,
                                           int32_t* result, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SPARVAR_H_ */
