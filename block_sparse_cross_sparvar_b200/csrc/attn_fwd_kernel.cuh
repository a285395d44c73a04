// Block-sparse attention forward on sm_100a: a persistent kernel.
//
// Each CTA owns one SM and walks the query tiles t = blockIdx.x, blockIdx.x +
// gridDim.x, ... (a tile is one 128-row query block of one batch item and
// head).  The KV blocks of all its tiles form one block sequence J = 0, 1, ...
// (tile after tile), and the pipeline runs across tile boundaries: the next
// tile's Q, first K blocks and first score MMAs overlap the current tile's last
// blocks and its epilogue.  Roles:
//   warps 0-3   softmax group 0: blocks with J even (thread t: query row t,
//               TMEM lane t)
//   warps 4-7   softmax group 1: blocks with J odd
//   warp  8     MMA issue for even J (one lane), tile prologues, TMEM owner
//   warp  9     TMA producer (one lane)
//   warp  10    MMA issue for odd J (one lane)
// TMEM (512 columns): three score buffers S_b = [128b, 128b+128), b = J mod 3,
// and the output accumulator O = [384, 384+D).  P_J is written as packed bf16
// over the first 64 columns of its score buffer and feeds the PV MMA from TMEM.
// Shared memory: two Q buffers (the k-th non-empty tile uses Q[k mod 2]) and a
// ring of K/V slots.  Within a tile of n blocks the ring order is K_0..K_{n0-1}
// (n0 = min(n, 3)), then V_j and, while j + 3 < n, K_{j+3}.
//
// MMA groups.  A tile's prologue (S_0 .. S_{n0-1}) is one group, issued by
// issuer 0 once the previous tile's MMAs have all completed.  Block j's group
// is PV_j followed by S_{j+3} into the buffer PV_j has just read (one issuer's
// MMAs run in issue order); issuer J mod 2 runs it, so while one issuer waits
// on a barrier the other keeps the tensor core's short queue filled.  The issuer
// waits for P_J and V_j, issues the PV MMAs and commits on rel_v[G mod 16] (G
// numbers the groups of the sequence in order), which frees V_j's slot; only then
// does it wait for K_{j+3}, whose load is the one most often late, and after the
// score MMAs it commits on rel[G mod 16], which frees K_{j+3}'s slot.  The
// producer records, per slot, the group that must release it and whether it held
// a V block.  Release barriers outnumber ring slots, so no waiter can fall two
// phases behind a barrier.
//
// Softmax.  Both groups add into one O, so they share a per-row reference max
// m (log2 units) in shared memory, reset at each tile.  Block J is computed
// against the reference read when it starts and finalised in block order: its
// group waits until P_{J-1} has been handed over, re-reads m, and either raises
// m (block max more than 2^8 above it: O is rescaled in place once the tile's
// earlier PVs have completed) or, if m moved meanwhile, rescales its own P in
// TMEM.  O is zeroed before a tile's first PV, so the two issuers' PVs may
// accumulate in either order.  Each issuer signs o_done after its last PV of a
// tile, so the epilogue need not wait for the next tile's score MMAs issued in
// the same groups.  Each block's softmax takes two passes over S in
// TMEM: the row max, then P in packed f32x2 arithmetic from the 96 columns kept
// in registers plus the last 32 re-read.  The epilogue waits for o_done,
// merges the two groups' row sums against the final m
// (exchanging them through the tile's Q buffer, which no MMA reads any more),
// stages the normalised bf16 output in that buffer in the output tensor map's
// swizzled layout, sends it with one TMA store per 64 columns, writes the LSE,
// and hands the buffer back to the producer once the store has read it.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx.cuh"
#include "tmem_io.cuh"

namespace sparvar {
namespace fwd {

constexpr int kTile = 128;
constexpr int kThreads = 352;
constexpr int kMmaWarp = 8;    // MMA issuer 0 (even J), tile prologues, TMEM owner
constexpr int kLoadWarp = 9;
constexpr int kMmaWarp1 = 10;  // MMA issuer 1 (odd J), on another SM sub-partition
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 384;
constexpr float kLazyRescale = 8.0f;          // log2 units
constexpr uint64_t kWaitNs = 1000000000ull;   // 1 s per wait
constexpr uint64_t kDrainNs = 500000000ull;   // 0.5 s per drain
constexpr int kMaxSlots = 12;
constexpr int kRel = 16;                      // release barriers (more than ring slots)

// CSLA token mask applied inside the kept tiles (enabled != 0): the query scale,
// the sink length in tokens and the locality radii over the schedule.
struct CslaTokens {
  int enabled;
  int q_scale, n_sink_scales, n_sink_tok, r_prev, r_own;
  int side[32];
  int off[33];
};

// One attention problem of a launch: queries [q_row0, q_row0 + Lq) of the Q, O
// and LSE row space attend to keys [0, Lkv) under their own block lists.  A
// launch walks the tiles of all its problems (one problem unless several
// scales share a launch).
constexpr int kMaxProblems = 16;
struct Problem {
  int Lq, Lkv, nqb, nkb;
  int q_row0;
  int tile0;  // first tile id of the problem in the launch
  int idx_row_len;
  const int32_t* kv_cnt;
  const int32_t* kv_idx;
  int64_t list_sb, list_sh;
};

struct Args {
  int B, H, n_problems, total_tiles;
  float scale_log2;  // softmax_scale * log2(e)
  Problem prob[kMaxProblems];
  const uint64_t* tile_mask;  // per list entry, fine-block bits; null: whole tiles
  const int32_t* tile_order;  // ORD instantiation: the tile id at each position
  int mask_shift;             // log2 of the fine block side (4, 5 or 6)
  __nv_bfloat16* o;
  int64_t o_sb, o_sh, o_sr;
  float* lse;    // [B][H][lse_rows] or null
  int lse_rows;
  int32_t* dev_status;
  CslaTokens tok;
};

// output tensor map of each problem (its rows only, so ragged tiles are clipped)
struct OutMaps {
  CUtensorMap m[kMaxProblems];
};

struct __align__(8) Bars {
  uint64_t q_full[2];             // Q of non-empty tile k landed: [k & 1], phase k >> 1
  uint64_t epi[2];                // epilogue of non-empty tile k done: [k & 1], phase k >> 1
  uint64_t full[kMaxSlots];       // ring slot loaded (TMA transaction count)
  uint64_t rel[kRel];             // MMA group G done: [G % kRel], phase G / kRel
  uint64_t rel_v[kRel];           // the PV MMAs of group G done (its V slot free): same indexing
  uint64_t s_full[3], p_full[3];  // block J: [J % 3], phase J / 3
  uint64_t o_done[2];             // every PV of non-empty tile k done: [k & 1], phase k >> 1
  uint64_t drain;
};

template <int D>
struct Layout {
  static constexpr uint32_t kTileBytes = kTile * D * 2;
  static constexpr uint32_t kChunkBytes = kTile * 128;  // 128 rows x 64 bf16
  static constexpr int kChunks = D / 64;
  static constexpr int kSlots = D == 128 ? 5 : 12;
  static constexpr uint32_t kQ = 0;  // two Q buffers
  static constexpr uint32_t kRing = 2 * kTileBytes;
  static constexpr uint32_t kBytes = (2 + kSlots) * kTileBytes + 1024;
};

// One tile of this CTA's sequence, with the sequence counters at its start.
// A tile whose predecessor (the previous non-empty tile) has at least three
// blocks is fed by it: the predecessor's last three MMA groups issue the tile's
// first score MMAs, and its K blocks and Q are loaded in the predecessor's ring
// stream.  Any other non-empty tile starts with a prologue group (its first
// score MMAs, issued once the predecessor's MMAs are done).
struct TileCursor {
  int t;  // position in the launch's tile sequence: the tile id (problem tile0 + (b * H + h) *
          // nqb + qb), or for a single problem given an order, its index into that
          // order; >= total when the CTA is done
  int p;  // problem of the tile
  int n;  // list length (clamped to [0, idx_row_len])
  const int32_t* list;
  int J0;      // sequence index of the tile's first block
  int pos0;    // ring position of the tile's first operand
  int k;       // number of non-empty tiles before this one
  int G;       // first MMA group of the tile
  int prev_n;  // list length of the previous non-empty tile, -1 before the first
  int next_n;  // list length of the next non-empty tile, 0 after the last
};

struct TileCoord {
  int p, b, h, qb;
  int nkb, row0;  // the problem's key-block count and first query row
};
// How a launch numbers its tiles: one problem in natural order, several
// problems (a problem table), or one problem in a given order (args.tile_order).
constexpr int kSingle = 0, kProblems = 1, kOrdered = 2;
template <int PM>
__device__ __forceinline__ TileCoord tile_coord(int t, const Args& a) {
  int p = 0;
  if constexpr (PM == kProblems) {
    while (p + 1 < a.n_problems && t >= a.prob[p + 1].tile0) ++p;
  }
  const int nqb = a.prob[p].nqb;
  // a single problem starts at tile 0, row 0; its tiles may run in a given order
  const int lt = PM == kProblems ? t - a.prob[p].tile0
                                 : (PM == kOrdered ? __ldg(a.tile_order + t) : t);
  const int bh = lt / nqb;
  return TileCoord{p, bh / a.H, bh % a.H, lt % nqb, a.prob[p].nkb,
                   PM == kProblems ? a.prob[p].q_row0 : 0};
}

template <int PM>
__device__ __forceinline__ int tile_count(int t, const Args& a, bool report,
                                          const int32_t** list, int* prob) {
  const TileCoord tc = tile_coord<PM>(t, a);
  const Problem& pr = a.prob[tc.p];
  const int64_t lrow = tc.b * pr.list_sb + tc.h * pr.list_sh + tc.qb;
  int n = __ldg(pr.kv_cnt + lrow);
  if (n < 0 || n > pr.idx_row_len) {
    if (report && a.dev_status) atomicOr(a.dev_status, 0x1);
    n = n < 0 ? 0 : pr.idx_row_len;
  }
  if (list) *list = pr.kv_idx + lrow * pr.idx_row_len;
  if (prob) *prob = tc.p;
  return n;
}

template <int PM>
__device__ __forceinline__ void cursor_load(TileCursor& c, const Args& a, int total, bool report) {
  if (c.t >= total) return;
  c.n = tile_count<PM>(c.t, a, report, &c.list, &c.p);
  c.next_n = 0;
  for (int t = c.t + gridDim.x; t < total && c.next_n == 0; t += gridDim.x)
    c.next_n = tile_count<PM>(t, a, false, nullptr, nullptr);
}

__device__ __forceinline__ bool has_prologue(const TileCursor& c) { return c.prev_n < 3; }
__device__ __forceinline__ bool feeds_next(const TileCursor& c) { return c.n >= 3 && c.next_n > 0; }
__device__ __forceinline__ int own_k(const TileCursor& c) { return c.n > 3 ? c.n - 3 : 0; }
__device__ __forceinline__ int n_prologue(const TileCursor& c) {
  return has_prologue(c) ? (c.n < 3 ? c.n : 3) : 0;
}
// ring positions of a tile: prologue K's, then V_j followed, when it exists, by
// the K block whose score MMA group j issues (K_{j+3} of this tile or, for the
// last three blocks of a feeding tile, the next tile's first K's)
__device__ __forceinline__ bool has_k_after(const TileCursor& c, int j) {
  return j < own_k(c) || (feeds_next(c) && j - own_k(c) < c.next_n);
}
__device__ __forceinline__ int ring_pos_v(const TileCursor& c, int j) {
  const int nk = own_k(c);
  int p = c.pos0 + n_prologue(c) + j + (j < nk ? j : nk);
  if (feeds_next(c) && j > nk) p += (j - nk < c.next_n ? j - nk : c.next_n);
  return p;
}
__device__ __forceinline__ int ring_items(const TileCursor& c) {
  return n_prologue(c) + c.n + own_k(c) + (feeds_next(c) ? (c.next_n < 3 ? c.next_n : 3) : 0);
}
__device__ __forceinline__ int group_of_prologue(const TileCursor& c) { return c.G; }
__device__ __forceinline__ int group_of_block(const TileCursor& c, int j) {
  return c.G + (has_prologue(c) ? 1 : 0) + j;
}

template <int PM>
__device__ __forceinline__ void cursor_next(TileCursor& c, const Args& a, int total, bool report) {
  if (c.n > 0) {
    c.pos0 += ring_items(c);
    c.G += c.n + (has_prologue(c) ? 1 : 0);
    c.J0 += c.n;
    c.k += 1;
    c.prev_n = c.n;
  }
  c.t += gridDim.x;
  cursor_load<PM>(c, a, total, report);
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          int32_t* st) {
  const bool ok = mbar_wait(bar, parity, abort, st, 0x2, kWaitNs);
  return __all_sync(0xffffffffu, ok);
}
__device__ __forceinline__ bool wait_group(uint64_t* rel, int grp, volatile int* abort,
                                           int32_t* st) {
  return mbar_wait(&rel[grp % kRel], (grp / kRel) & 1, abort, st, 0x2, kWaitNs);
}
__device__ __forceinline__ bool warp_wait_group(uint64_t* rel, int grp, volatile int* abort,
                                                int32_t* st) {
  return warp_wait(&rel[grp % kRel], (grp / kRel) & 1, abort, st);
}

// OR columns [lo, hi) (0 <= lo < hi <= 128) into a 128-bit row mask
__device__ __forceinline__ void set_cols(uint32_t (&km)[4], int lo, int hi) {
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const int a = max(lo, w * 32), b = min(hi, w * 32 + 32);
    if (a < b) km[w] |= (b - a == 32 ? 0xffffffffu : ((1u << (b - a)) - 1u)) << (a - w * 32);
  }
}

// CSLA token mask of query (i, j) of the query scale over keys [k0, k1): the sink,
// and for every scale m from the first non-sink one up to the query scale, the keys
// within Chebyshev radius r_m of the query's projection (floor(i*s_m/s_k),
// floor(j*s_m/s_k)); the rows of that window meeting [k0, k1) are contiguous
// column ranges.
__device__ __forceinline__ void csla_row_mask(const CslaTokens& t, int i, int j, int k0, int k1,
                                              uint32_t (&km)[4]) {
  km[0] = km[1] = km[2] = km[3] = 0u;
  if (k0 < t.n_sink_tok) set_cols(km, 0, min(t.n_sink_tok, k1) - k0);
  const int sk = t.side[t.q_scale];
  for (int m = t.n_sink_scales; m <= t.q_scale; ++m) {
    const int o0 = t.off[m], o1 = t.off[m + 1];
    if (o1 <= k0 || o0 >= k1) continue;
    const int sm = t.side[m];
    const int r = m == t.q_scale ? t.r_own : t.r_prev;
    // (32-bit unsigned arithmetic: sides are at most 46340, so i * sm < 2^32)
    const uint32_t usm = static_cast<uint32_t>(sm), usk = static_cast<uint32_t>(sk);
    const int ci = static_cast<int>(static_cast<uint32_t>(i) * usm / usk);
    const int cj = static_cast<int>(static_cast<uint32_t>(j) * usm / usk);
    const int c0 = max(cj - r, 0), c1 = min(cj + r, sm - 1);
    const int a0 = max(max(ci - r, 0), static_cast<int>(static_cast<uint32_t>(max(k0, o0) - o0) / usm));
    const int a1 = min(min(ci + r, sm - 1),
                       static_cast<int>(static_cast<uint32_t>(min(k1, o1) - 1 - o0) / usm));
    for (int a = a0; a <= a1; ++a) {
      const int lo = max(o0 + a * sm + c0, k0) - k0;
      const int hi = min(o0 + a * sm + c1 + 1, k1) - k0;
      if (lo < hi) set_cols(km, lo, hi);
    }
  }
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// TOK: apply the CSLA token mask (args.tok) inside the kept tiles.  MULTI: the
// launch holds several problems (args.prob), one output map each.
template <int D, bool TOK, bool MULTI, bool ORD = false, bool FINE = true>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ OutMaps tm_os, const __grid_constant__ Args args) {
  constexpr int PM = MULTI ? kProblems : (ORD ? kOrdered : kSingle);
  using L = Layout<D>;
  constexpr int NS = L::kSlots;
  extern __shared__ uint8_t smem_raw[];
  __shared__ Bars bars;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  __shared__ float m_sh[kTile];      // shared reference max per row
  __shared__ int relg_sh[kMaxSlots];  // producer: group that frees each ring slot (-1: unused)
  __shared__ int relv_sh[kMaxSlots];  // producer: the slot holds a V block (freed by rel_v)

  const uint32_t smem_base = (smem_addr(smem_raw) + 1023u) & ~1023u;
  uint8_t* smem_gen = smem_raw + (smem_base - smem_addr(smem_raw));
  const int warp = warp_id();
  const int lane = lane_id();
  volatile int* abort_flag = &abort_sh;
  int32_t* dev_status = args.dev_status;
  // a single problem's tile count is its shape's (equal to total_tiles); written so,
  // the compiler relates tile ids to tile coordinates and emits shorter tile code
  const int total = MULTI ? args.total_tiles : args.B * args.H * args.prob[0].nqb;

  if (threadIdx.x == 0) {
    abort_sh = 0;
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars.q_full[i], 1);
      mbar_init(&bars.epi[i], 1);
    }
    for (int s = 0; s < NS; ++s) mbar_init(&bars.full[s], 1);
    for (int i = 0; i < kRel; ++i) {
      mbar_init(&bars.rel[i], 1);
      mbar_init(&bars.rel_v[i], 1);
    }
    for (int i = 0; i < 3; ++i) {
      mbar_init(&bars.s_full[i], 1);
      mbar_init(&bars.p_full[i], 128);
    }
    for (int i = 0; i < 2; ++i) mbar_init(&bars.o_done[i], 2);  // one commit per issuer
    mbar_init(&bars.drain, 2);  // one commit per issuer
    fence_barrier_init();
  }
  if (threadIdx.x < kTile) m_sh[threadIdx.x] = -INFINITY;
  if (threadIdx.x < kMaxSlots) {
    relg_sh[threadIdx.x] = -1;
    relv_sh[threadIdx.x] = 0;
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&tmem_base_sh, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kLoadWarp && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_os.m[0]);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // launched behind the list builder with programmatic serialization: its lists and
  // tile order are read only after it has completed
  griddep_wait();
  const uint32_t tmem = tmem_base_sh;
  auto sQ = [&](int k) { return smem_base + L::kQ + (k & 1) * L::kTileBytes; };
  auto sSlot = [&](int s) { return smem_base + L::kRing + s * L::kTileBytes; };

  TileCursor first{};
  first.t = blockIdx.x;
  first.prev_n = -1;
  cursor_load<PM>(first, args, total, threadIdx.x == 0);

  if (warp == kLoadWarp) {
    // ================================================================ producer
    if (lane == 0) {
      int w = 0;  // ring position
      int q_issued0 = 0, q_issued1 = 0;  // Q loads into each buffer
      bool ok = true;
      auto produce = [&](const CUtensorMap* tm, int kb, int grp, const TileCoord& tc) {
        const int s = w % NS;
        const int prev = relg_sh[s];
        if (prev >= 0 &&
            !wait_group(relv_sh[s] ? bars.rel_v : bars.rel, prev, abort_flag, dev_status)) {
          ok = false;
          return;
        }
        relg_sh[s] = grp;
        relv_sh[s] = tm == &tm_v;
        kb = kb < 0 ? -1 : (kb > tc.nkb ? tc.nkb : kb);
        mbar_arrive_expect_tx(&bars.full[s], L::kTileBytes);
#pragma unroll
        for (int c = 0; c < L::kChunks; ++c)
          tma_load_4d(sSlot(s) + c * L::kChunkBytes, tm, &bars.full[s], c * 64, kb * kTile, tc.h,
                      tc.b);
        ++w;
      };
      // Q of non-empty tile k into buffer k & 1, free once tile k - 2's epilogue is done
      auto load_q = [&](int k, const TileCoord& tq) {
        const int qs = k & 1;
        if (k >= 2 &&
            !mbar_wait(&bars.epi[qs], ((k - 2) >> 1) & 1, abort_flag, dev_status, 0x2, kWaitNs)) {
          ok = false;
          return;
        }
        mbar_arrive_expect_tx(&bars.q_full[qs], L::kTileBytes);
#pragma unroll
        for (int cc = 0; cc < L::kChunks; ++cc)
          tma_load_4d(sQ(k) + cc * L::kChunkBytes, &tm_q, &bars.q_full[qs], cc * 64,
                      tq.row0 + tq.qb * kTile, tq.h, tq.b);
        if (qs) ++q_issued1; else ++q_issued0;
      };
      for (TileCursor c = first; c.t < total && ok; cursor_next<PM>(c, args, total, false)) {
        if (c.n == 0) continue;
        const TileCoord tc = tile_coord<PM>(c.t, args);
        if (has_prologue(c)) {
          load_q(c.k, tc);
          for (int jj = 0; jj < n_prologue(c) && ok; ++jj)
            produce(&tm_k, __ldg(c.list + jj), group_of_prologue(c), tc);
        }
        // the next non-empty tile, when this one feeds it
        TileCursor nx = c;
        TileCoord tn{};
        if (feeds_next(c)) {
          do {
            cursor_next<PM>(nx, args, total, false);
          } while (nx.t < total && nx.n == 0);
          tn = tile_coord<PM>(nx.t, args);
        }
        const int nk = own_k(c);
        for (int j = 0; j < c.n && ok; ++j) {
          const int grp = group_of_block(c, j);
          produce(&tm_v, __ldg(c.list + j), grp, tc);
          if (!ok) break;
          if (j < nk) {
            produce(&tm_k, __ldg(c.list + j + 3), grp, tc);
          } else if (has_k_after(c, j)) {
            if (j == nk) load_q(c.k + 1, tn);
            if (ok) produce(&tm_k, __ldg(nx.list + (j - nk)), grp, tn);
          }
        }
      }
      // drain: every issued TMA write lands before the CTA exits
      if (q_issued0) mbar_drain(&bars.q_full[0], (q_issued0 - 1) & 1, kDrainNs);
      if (q_issued1) mbar_drain(&bars.q_full[1], (q_issued1 - 1) & 1, kDrainNs);
      for (int s = 0; s < NS; ++s) {
        const int issued = w > s ? (w - 1 - s) / NS + 1 : 0;  // loads that used slot s
        if (issued) mbar_drain(&bars.full[s], (issued - 1) & 1, kDrainNs);
      }
    }
  } else if (warp == kMmaWarp || warp == kMmaWarp1) {
    // ================================================================ MMA issue
    const int me = warp == kMmaWarp ? 0 : 1;
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(kTile, kTile, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kTile, D, 1);
      constexpr uint32_t kBufStep = L::kTileBytes >> 4;  // descriptor units per buffer
      const uint64_t dq = smem_desc_sw128(sQ(0), 16, 1024);
      const uint64_t dk = smem_desc_sw128(sSlot(0), 16, 1024);
      const uint64_t dv = smem_desc_sw128(sSlot(0), L::kChunkBytes, 1024);
      bool ok = true;
      auto wait_pos = [&](int pos) {
        ok = ok && mbar_wait(&bars.full[pos % NS], (pos / NS) & 1, abort_flag, dev_status, 0x2,
                             kWaitNs);
      };
      // S_J = Q(tile k) K^T, K from ring position pos, into score buffer J mod 3
      auto issue_s = [&](int J, int k, int pos) {
        const uint64_t dqs = dq + static_cast<uint64_t>((k & 1) * kBufStep);
        const uint64_t dks = dk + static_cast<uint64_t>((pos % NS) * kBufStep);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * L::kChunkBytes + (kk & 3) * 32) >> 4;
          mma_ss(tmem + (J % 3) * 128, dqs + off, dks + off, idesc_s, kk > 0 ? 1u : 0u);
        }
      };
      int last1 = -1, last2 = -1;  // last two groups of the previous non-empty tile
      for (TileCursor c = first; c.t < total && ok; cursor_next<PM>(c, args, total, false)) {
        if (c.n == 0) continue;
        const int nk = own_k(c);
        if (me == 0 && has_prologue(c)) {
          // prologue: the score buffers are free once the previous tile's MMAs are done
          ok = mbar_wait(&bars.q_full[c.k & 1], (c.k >> 1) & 1, abort_flag, dev_status, 0x2,
                         kWaitNs);
          if (ok && last1 >= 0) ok = wait_group(bars.rel, last1, abort_flag, dev_status);
          if (ok && last2 >= 0) ok = wait_group(bars.rel, last2, abort_flag, dev_status);
          for (int jj = 0; jj < n_prologue(c) && ok; ++jj) {
            wait_pos(c.pos0 + jj);
            if (!ok) break;
            tc_fence_after();
            issue_s(c.J0 + jj, c.k, c.pos0 + jj);
            mma_commit(&bars.s_full[(c.J0 + jj) % 3]);
          }
          if (!ok) break;
          mma_commit(&bars.rel_v[group_of_prologue(c) % kRel]);  // (no PV: keeps the phases)
          mma_commit(&bars.rel[group_of_prologue(c) % kRel]);
        }
        for (int j = ((c.J0 & 1) == me) ? 0 : 1; j < c.n && ok; j += 2) {
          const int J = c.J0 + j;
          ok = mbar_wait(&bars.p_full[J % 3], (J / 3) & 1, abort_flag, dev_status, 0x2, kWaitNs);
          const int pv = ring_pos_v(c, j);
          const bool more = has_k_after(c, j);
          const bool feed = more && j >= nk;  // S of the next tile's block j - nk
          wait_pos(pv);
          if (!ok) break;
          const uint64_t dvs = dv + static_cast<uint64_t>((pv % NS) * kBufStep);
          const uint32_t a_col = tmem + (J % 3) * 128;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            mma_ts(tmem + kColO, a_col + kk * 8, dvs + static_cast<uint64_t>(kk * (2048 >> 4)),
                   idesc_pv, 1u);
          // this issuer's last PV of the tile: O is final once both issuers' are done
          if (j + 2 >= c.n) mma_commit(&bars.o_done[c.k & 1]);
          mma_commit(&bars.rel_v[group_of_block(c, j) % kRel]);
          // the score MMAs' operands are waited for only now, behind the PV MMAs
          if (more) wait_pos(pv + 1);
          if (feed)
            ok = ok && mbar_wait(&bars.q_full[(c.k + 1) & 1], ((c.k + 1) >> 1) & 1, abort_flag,
                                 dev_status, 0x2, kWaitNs);
          if (!ok) break;
          if (more) {
            tc_fence_after();
            // buffer J mod 3 is free once PV_J has read P_J (this issuer's MMAs run in order)
            issue_s(J + 3, feed ? c.k + 1 : c.k, pv + 1);
            mma_commit(&bars.s_full[J % 3]);
          }
          mma_commit(&bars.rel[group_of_block(c, j) % kRel]);
        }
        // an issuer with no block in this (one-block) tile still signs for O
        if (ok && c.n == 1 && ((c.J0 & 1) != me)) mma_commit(&bars.o_done[c.k & 1]);
        last1 = group_of_block(c, c.n - 1);
        last2 = c.n >= 2 ? group_of_block(c, c.n - 2) : -1;
      }
      mma_commit(&bars.drain);
      mbar_drain(&bars.drain, 0, kDrainNs);
    }
    __syncwarp();
  } else {
    // ================================================================ softmax
    const int g = warp >> 2;  // group: blocks with J % 2 == g
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t o_addr = tmem + lane_off + kColO;
    const float csc = args.scale_log2;
    bool good = true;

    for (TileCursor c = first; c.t < total; cursor_next<PM>(c, args, total, threadIdx.x == 0)) {
      // the tile's problem, read once per tile into registers
      const int pi = MULTI ? c.p : 0;
      const int p_nkb = args.prob[pi].nkb, p_lkv = args.prob[pi].Lkv, p_lq = args.prob[pi].Lq;
      const int p_row0 = MULTI ? args.prob[pi].q_row0 : 0;
      float m_own = -INFINITY;  // reference of this group's row sum
      float l_own = 0.f;
      const int c_qb = TOK ? (c.t - args.prob[pi].tile0) % args.prob[pi].nqb : 0;
      for (int j = ((c.J0 & 1) == g) ? 0 : 1; j < c.n && good; j += 2) {
        const int J = c.J0 + j;
        const int kb = __ldg(c.list + j);
        const int buf = J % 3;
        const uint32_t s_addr = tmem + lane_off + buf * 128;
        if (!warp_wait(&bars.s_full[buf], (J / 3) & 1, abort_flag, dev_status)) {
          good = false;
          break;
        }
        tc_fence_after();
        int valid = kTile;
        if (kb < 0 || kb >= p_nkb) {
          valid = 0;
          if (row == 0 && dev_status) atomicOr(dev_status, 0x1);
        } else if ((kb + 1) * kTile > p_lkv) {
          valid = p_lkv - kb * kTile;
        }
        // with a fine block grid, bit i of `keep` keeps this row's columns
        // [i << mask_shift, (i + 1) << mask_shift) of the tile
        uint32_t keep = 0xffu;
        bool fine = false;
        if constexpr (FINE) {  // (instantiated without it for launches with no tile masks)
          if (args.tile_mask) {
            const int fg = kTile >> args.mask_shift;
            const uint32_t full = (1u << fg) - 1u;
            const uint64_t mk = __ldg(args.tile_mask + (c.list - args.prob[pi].kv_idx) + j);
            keep = static_cast<uint32_t>(mk >> ((row >> args.mask_shift) * fg)) & full;
            fine = __any_sync(0xffffffffu, keep != full);
            keep |= ~full;
          }
        }
        // with the CSLA token mask on, bit c of km keeps column c of this row
        uint32_t km[4] = {~0u, ~0u, ~0u, ~0u};
        if constexpr (TOK) {
          const int grow = c_qb * kTile + row;
          const int sk = args.tok.side[args.tok.q_scale];
          const int gq = grow < p_lq ? grow : 0;
          if (valid > 0)
            csla_row_mask(args.tok, gq / sk, gq % sk, kb * kTile, kb * kTile + valid, km);
          fine = true;
        }
        // columns at or past the prefix end (the same for every row): -inf in TMEM
        // before S is read, with whole-warp stores (the token-mask instantiation masks
        // its rows in registers anyway)
        constexpr bool kTmemMask = !TOK;
        if constexpr (kTmemMask) {
         if (__builtin_expect(valid < kTile, 0)) {
          const uint32_t ninf = __float_as_uint(-INFINITY);
          const int v8 = (valid + 7) & ~7;
          for (int col = valid; col < v8; ++col) tmem_st1(s_addr + col, ninf);
          for (int col = v8; col < kTile; col += 8) tmem_st8_fill(s_addr + col, ninf);
          tmem_wait_st();
         }
        }
        // fine blocks of 32 or 64 rows: the rows of one warp share their keep bits, so
        // the dropped fine KV blocks are set to -inf in TMEM as well (whole-warp stores)
        // and the registers need no mask
        if constexpr (FINE && kTmemMask) {
          if (fine && args.mask_shift >= 5) {
            const uint32_t ninf = __float_as_uint(-INFINITY);
            const int w = 1 << args.mask_shift;
            for (int i = 0; i < (kTile >> args.mask_shift); ++i)
              if (!((keep >> i) & 1u))
                for (int col = i * w; col < (i + 1) * w; col += 8) tmem_st8_fill(s_addr + col, ninf);
            tmem_wait_st();
            fine = false;
          }
        }
        auto dropped = [&](int col) {
          return col >= valid || !((keep >> (col >> args.mask_shift)) & 1u) ||
                 !((km[col >> 5] >> (col & 31)) & 1u);
        };
        // pass 1: the block's row max.  Columns 0-95 stay in registers for pass 2.
        float bm;
        uint32_t s0[32], s1[32], s2[32];
        {
          uint32_t sr[kTile];
          tmem_ld128_wait(s_addr, sr);
          if ((!kTmemMask && valid < kTile) || fine) {
#pragma unroll
            for (int k = 0; k < kTile; ++k)
              if (dropped(k)) sr[k] = __float_as_uint(-INFINITY);
          }
          float mx0 = fmaxf(__uint_as_float(sr[0]), __uint_as_float(sr[4]));
          float mx1 = fmaxf(__uint_as_float(sr[1]), __uint_as_float(sr[5]));
          float mx2 = fmaxf(__uint_as_float(sr[2]), __uint_as_float(sr[6]));
          float mx3 = fmaxf(__uint_as_float(sr[3]), __uint_as_float(sr[7]));
#pragma unroll
          for (int k = 8; k < kTile; k += 8) {
            mx0 = max3(mx0, __uint_as_float(sr[k]), __uint_as_float(sr[k + 4]));
            mx1 = max3(mx1, __uint_as_float(sr[k + 1]), __uint_as_float(sr[k + 5]));
            mx2 = max3(mx2, __uint_as_float(sr[k + 2]), __uint_as_float(sr[k + 6]));
            mx3 = max3(mx3, __uint_as_float(sr[k + 3]), __uint_as_float(sr[k + 7]));
          }
          bm = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * csc;
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            s0[k] = sr[k];
            s1[k] = sr[32 + k];
            s2[k] = sr[64 + k];
          }
        }
        // provisional reference: the shared one, raised to bm if bm is far above it
        const float m_cur = m_sh[row];
        const float m_use = (m_cur == -INFINITY || bm > m_cur + kLazyRescale) ? bm : m_cur;
        const float neg = (m_use == -INFINITY) ? 0.f : -m_use;
        // pass 2: P = 2^(s * scale - m) in packed pairs.  Columns 96-127 are re-read
        // while the columns held in registers are worked on; P chunk cc (packed bf16)
        // overwrites TMEM columns [16cc, 16cc + 16), already read.
        const uint64_t sc2 = f2_pack(csc, csc), neg2 = f2_pack(neg, neg);
        uint64_t acc0 = 0, acc1 = 0;  // (0.f, 0.f)
        auto p_chunk = [&](const uint32_t(&cur)[32], int cc) {
          uint32_t pk[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            float e0, e1, p0, p1;
            f2_unpack(f2_fma(f2_pack(__uint_as_float(cur[2 * k]), __uint_as_float(cur[2 * k + 1])),
                             sc2, neg2),
                      e0, e1);
            p0 = ex2_approx(e0);
            p1 = ex2_approx(e1);
            if (k & 1) {
              acc1 = f2_add(acc1, f2_pack(p0, p1));
            } else {
              acc0 = f2_add(acc0, f2_pack(p0, p1));
            }
            pk[k] = pack_bf16x2(p0, p1);
          }
          tmem_st16(s_addr + cc * 16, pk);
        };
        auto mask_chunk = [&](uint32_t(&cur)[32], int cc) {
          if ((!kTmemMask && valid < kTile) || fine) {
#pragma unroll
            for (int k = 0; k < 32; ++k)
              if (dropped(cc * 32 + k)) cur[k] = __float_as_uint(-INFINITY);
          }
        };
        {
          uint32_t s3[32];
          tmem_ld32_async(s_addr + 96, s3, __float_as_uint(neg));
          p_chunk(s0, 0);
          p_chunk(s1, 1);
          p_chunk(s2, 2);
          tmem_wait_ld_tied(s3);
          mask_chunk(s3, 3);
          p_chunk(s3, 3);
        }
        float lb;
        {
          float a0, a1;
          f2_unpack(f2_add(acc0, acc1), a0, a1);
          lb = a0 + a1;
        }

        // ---- finalise block J in sequence order
        if (J > 0 &&
            !warp_wait(&bars.p_full[(J - 1) % 3], ((J - 1) / 3) & 1, abort_flag, dev_status)) {
          good = false;
          break;
        }
        const float m_fin = m_sh[row];
        const bool raise = m_fin == -INFINITY ? (bm != -INFINITY) : (bm > m_fin + kLazyRescale);
        const float m_blk = raise ? bm : m_fin;  // reference of block J from now on
        // O holds non-zero values only once an earlier block of the tile had a finite reference
        const bool o_live = raise && m_fin != -INFINITY;
        if (__builtin_expect(__any_sync(0xffffffffu, o_live), 0)) {  // rare: laid out of line
          // every earlier PV of the tile is complete once the PV MMAs of the latest
          // group of each issuer (blocks j-1 and j-2) have completed
          if (!warp_wait_group(bars.rel_v, group_of_block(c, j - 1), abort_flag, dev_status) ||
              (j >= 2 &&
               !warp_wait_group(bars.rel_v, group_of_block(c, j - 2), abort_flag, dev_status))) {
            good = false;
            break;
          }
          tc_fence_after();
          const float alpha = o_live ? ex2_approx(m_fin - bm) : 1.f;
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t orr[32];
            tmem_ld32_wait(o_addr + cc * 32, orr);
#pragma unroll
            for (int k = 0; k < 32; ++k) orr[k] = __float_as_uint(__uint_as_float(orr[k]) * alpha);
            tmem_st32(o_addr + cc * 32, orr);
          }
        }
        const bool fix_p = (m_use != m_blk) && m_use != -INFINITY;
        if (__builtin_expect(__any_sync(0xffffffffu, fix_p), 0)) {
          // the shared reference moved while P_J was computed: rescale P_J to m_blk
          tmem_wait_st();
          const float beta = fix_p ? ex2_approx(m_use - m_blk) : 1.f;
          if (fix_p) lb *= beta;
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            uint32_t pr[32];
            tmem_ld32_wait(s_addr + cc * 32, pr);
#pragma unroll
            for (int k = 0; k < 32; ++k) {
              const float lo = __uint_as_float(pr[k] << 16) * beta;
              const float hi = __uint_as_float(pr[k] & 0xffff0000u) * beta;
              pr[k] = pack_bf16x2(lo, hi);
            }
            tmem_st32(s_addr + cc * 32, pr);
          }
        }
        if (raise) m_sh[row] = m_blk;
        // this group's running sum, moved to the block's reference
        if (m_blk != m_own) {
          l_own *= (m_own == -INFINITY) ? 0.f : ex2_approx(m_own - m_blk);
          m_own = m_blk;
        }
        l_own += lb;
        if (j == 0) {
          // O starts at zero: the two issuers' PV MMAs accumulate in either order
          uint32_t zr[32];
#pragma unroll
          for (int k = 0; k < 32; ++k) zr[k] = 0u;
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) tmem_st32(o_addr + cc * 32, zr);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars.p_full[buf]);
      }

      // ---- epilogue of the tile
      if (good && c.n > 0)
        good = warp_wait(&bars.o_done[c.k & 1], (c.k >> 1) & 1, abort_flag, dev_status);
      // every MMA of the tile is done and its Q buffer is free: it takes first the two
      // groups' sums, then the bf16 output tile, which leaves through a TMA store
      uint8_t* qbuf = smem_gen + L::kQ + (c.k & 1) * L::kTileBytes;
      float* xch = reinterpret_cast<float*>(qbuf);
      if (c.n > 0) {
        xch[g * kTile + row] = m_own;
        xch[(2 + g) * kTile + row] = l_own;
      }
      tc_fence_before();
      asm volatile("bar.sync 1, 256;" ::: "memory");
      tc_fence_after();
      const int aborted = __shfl_sync(0xffffffffu, *abort_flag, 0);
      const TileCoord tc = tile_coord<PM>(c.t, args);
      const int grow = tc.qb * kTile + row;
      float l = 0.f, m = -INFINITY, inv_l = 0.f;
      if (c.n > 0) {
        m = m_sh[row];
        const float ma = xch[row], mb = xch[kTile + row];
        const float sa = (ma == -INFINITY) ? 0.f : ex2_approx(ma - m);
        const float sb = (mb == -INFINITY) ? 0.f : ex2_approx(mb - m);
        l = xch[2 * kTile + row] * sa + xch[3 * kTile + row] * sb;
        inv_l = l > 0.f ? 1.f / l : 0.f;
      }
      if (!aborted && g == 0 && args.lse && grow < p_lq) {
        args.lse[(static_cast<int64_t>(tc.b) * args.H + tc.h) * args.lse_rows + p_row0 + grow] =
            l > 0.f ? (m + __log2f(l)) * 0.6931471805599453f : -INFINITY;
      }
      if (c.n > 0) {
        asm volatile("bar.sync 1, 256;" ::: "memory");  // the sums are read: reuse the buffer
        if (!aborted) {
          // row `row`, columns [g D/2, (g+1) D/2), into the 128B-swizzled layout of the
          // output tensor map: 64-column chunks of 128 rows x 128 bytes, 16-byte unit u of
          // row r at position u ^ (r mod 8)
          auto stage = [&](const uint32_t* ro, int col) {  // 32 columns from `col`
            uint32_t pk[16];
#pragma unroll
            for (int k = 0; k < 16; ++k)
              pk[k] = pack_bf16x2(__uint_as_float(ro[2 * k]) * inv_l,
                                  __uint_as_float(ro[2 * k + 1]) * inv_l);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const int cv = col + 8 * v;
              const int unit = (cv & 63) >> 3;
              uint4* dst = reinterpret_cast<uint4*>(qbuf + (cv >> 6) * L::kChunkBytes + row * 128 +
                                                    ((unit ^ (row & 7)) << 4));
              *dst = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
            }
          };
          // this thread's D/2 columns of O in one TMEM load
          if constexpr (D == 128) {
            uint32_t ro[64];
            tmem_ld64_wait(o_addr + g * 64, ro);
            stage(ro, g * 64);
            stage(ro + 32, g * 64 + 32);
          } else {
            uint32_t ro[32];
            tmem_ld32_wait(o_addr + g * 32, ro);
            stage(ro, g * 32);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        asm volatile("bar.sync 1, 256;" ::: "memory");
        if (threadIdx.x == 0 && !aborted) {
#pragma unroll
          for (int ch = 0; ch < L::kChunks; ++ch)
            tma_store_4d(&tm_os.m[MULTI ? tc.p : 0], sQ(c.k) + ch * L::kChunkBytes, ch * 64,
                         tc.qb * kTile, tc.h, tc.b);
          bulk_commit_group();
        }
      } else if (!aborted && grow < p_lq) {
        // empty list: zero rows (the Q buffer may already hold the next tile's Q)
        __nv_bfloat16* orow =
            args.o + tc.b * args.o_sb + tc.h * args.o_sh + (p_row0 + grow) * args.o_sr;
#pragma unroll
        for (int v = 0; v < D / 16; ++v)
          reinterpret_cast<uint4*>(orow + g * (D / 2))[v] = make_uint4(0u, 0u, 0u, 0u);
      }
      // reset m for the next tile once everyone has read it
      asm volatile("bar.sync 1, 256;" ::: "memory");
      if (g == 0) m_sh[row] = -INFINITY;
      asm volatile("bar.sync 1, 256;" ::: "memory");
      if (threadIdx.x == 0 && c.n > 0) {
        bulk_wait_read_all();  // the output tile has left the buffer: hand it back
        mbar_arrive(&bars.epi[c.k & 1]);
      }
      tc_fence_after();
    }
  }

  if (threadIdx.x == 0) bulk_wait_all();  // output stores complete before the CTA exits
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace fwd
}  // namespace sparvar
