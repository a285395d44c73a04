// Block-sparse attention forward on sm_100a: a persistent kernel over pairs of
// query tiles that share one K/V stream.
//
// A query tile is one 128-row query block of one batch item and head, with its
// list of kept 128-key blocks.  The tiles of query blocks 2i and 2i + 1 of one
// (batch, head) form a pair; their lists overlap (nearby queries keep nearby
// keys), and the pair walks the merge of the two lists once: each K/V block of
// the merged sequence is loaded into shared memory once and used by one or both
// tiles, so the K/V bytes per FLOP are about half those of tiles run alone.  Each
// CTA owns one SM and claims pairs one at a time.  Stream s = 0, 1 of a CTA runs
// tile 2i + s of every pair.  Roles:
//   warps 4s..4s+3   softmax of stream s (thread t: query row t, TMEM lane t)
//   warp  8          MMA issue (one lane) and TMEM owner
//   warp  9          TMA producer (one lane): claims pairs, loads Q and K/V
//   warps 10, 11     idle (they complete the control warpgroup)
// TMEM (512 columns): stream s has its score buffer S_s = [256s, 256s + 128) and
// its output accumulator O_s = [256s + 128, 256s + 128 + D).  P (packed bf16)
// is written over the first 64 columns of S_s and feeds the PV MMA from TMEM.
// Shared memory: Q of each stream, a ring of K/V slots shared by the streams,
// and a 64-column output staging buffer per stream.
//
// MMA order.  For each entry u of the merged sequence (a KV block and the
// streams that keep it): for s = 0, 1, PV_s(u) if s keeps u, then S_s of the
// stream's next block when that is entry u + 1.  The issuer's MMAs run in issue
// order, so S_s may overwrite the P that PV_s has read, and the completion of
// S_s(j) implies that of PV_s of the stream's previous block: once S_s(j) is
// complete no MMA touches O_s until P_s(j) is handed over, which lets the
// softmax rescale O_s in place.  The two streams' groups alternate on the
// tensor core while each stream's softmax works on its next block.
//
// Softmax per block: the 128 scores of a row stay in registers; P = 2^(s * scale
// - m) in packed f32x2 arithmetic against a lazily raised reference m, with the
// block's row max formed alongside; only when the block max exceeds the
// reference by more than 2^8 (rare after a tile's first block) are O and the row
// sum rescaled and the block redone.  A tile's first block takes its max first.  Keys past the
// prefix, keys of fine blocks the tile mask drops and, with the token mask, keys
// outside the CSLA rule are set to -inf first (one 128-bit keep mask per row).
// Epilogue per tile: wait until the stream's last PV of the pair is complete and
// read O into registers; the warp's P of the next tile's first block comes after
// that read, so the PV that overwrites O cannot start before it.  Then each warp
// normalises its 32 rows, stages them as bf16 in the 128B-swizzled layout and
// stores them by TMA, with no barrier across warps.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include <type_traits>

#include "ptx.cuh"
#include "select.cuh"
#include "tmem_io.cuh"

namespace sparvar {
namespace fwd {

constexpr int kTile = 128;
constexpr int kThreads = 384;  // 12 warps
constexpr int kIssuerWarp = 8;
constexpr int kProducerWarp = 9;
// flags of a ring item (item_meta_sh): kItemV a V block (else K); per stream st,
// shifted by st: kItemUse the stream's MMA reads it, kItemFirst its first score /
// PV MMA of the tile, kItemLast its last one; kItemEnd: no more items
constexpr uint32_t kItemV = 1u << 8, kItemEnd = 1u << 9;
constexpr uint32_t kItemUse = 1u << 0, kItemFirst = 1u << 2, kItemLast = 1u << 4;
constexpr uint32_t kTmemCols = 512;
constexpr float kLazyRescale = 8.0f;          // log2 units
constexpr uint64_t kWaitNs = 1000000000ull;   // 1 s per wait
constexpr uint64_t kDrainNs = 500000000ull;   // 0.5 s per drain
constexpr int kMaxSlots = 8;                  // K/V ring slots
constexpr int kTq = 4;                        // pair queue entries
constexpr int kOutBoxRows = 32;               // rows of one output TMA store (one warp's)
constexpr int kMaxDecBlocks = 128;            // KV blocks of a decision-scale prefix
// Register budgets: the kernel is launched with kLaunchRegs per thread (the host
// checks the compiled count); warps 8-11 (issuers, producers) give registers back
// and the two softmax warpgroups take them: 2 * 128 * 200 + 128 * 104 = 384 * 168.
constexpr int kLaunchRegs = 168;
constexpr uint32_t kSoftmaxRegs = 200, kControlRegs = 104;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kControlRegs <= kThreads * kLaunchRegs,
              "register budgets exceed the launch allocation");

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
  int pair0;  // first pair id of the problem in the launch
  int idx_row_len;
  const int32_t* kv_cnt;
  const int32_t* kv_idx;
  int64_t list_sb, list_sh;
};

struct Args {
  int B, H, n_problems, total_pairs;
  float scale_log2;  // softmax_scale * log2(e)
  Problem prob[kMaxProblems];
  const uint64_t* tile_mask;  // per list entry, fine-block bits; null: whole tiles
  int mask_shift;             // log2 of the fine block side (4, 5 or 6)
  __nv_bfloat16* o;
  int64_t o_sb, o_sh, o_sr;
  float* lse;    // [B][H][lse_rows] or null
  int lse_rows;
  int32_t* dev_status;
  CslaTokens tok;
  // decision instantiation: pooled mass [B][H][nqb][nkb] (or null), selection rule
  // (topk > 0: keep topk blocks; else the smallest heaviest-first set reaching
  // mass_threshold) and the selected lists [B][H][nqb] / [B][H][nqb][nkb]
  float* mass_out;
  int topk;
  float mass_threshold;
  int32_t* sel_cnt;
  int32_t* sel_idx;
};

// output tensor map of each problem (its rows only, so ragged tiles are clipped);
// box: 64 columns x kOutBoxRows rows
struct OutMaps {
  CUtensorMap m[kMaxProblems];
};

// The mbarriers of one stream.  Phases: k counts the stream's non-empty tiles,
// J its blocks over all its tiles.
struct __align__(8) StreamBars {
  uint64_t q_full;             // Q of tile k landed                              [k]
  uint64_t q_free;             // last score MMA of tile k complete                [k]
  uint64_t s_full;             // S of block J in TMEM                             [J]
  uint64_t p_full;             // P of block J in TMEM (128 arrivals)              [J]
  uint64_t o_done;             // every PV of tile k complete                      [k]
  uint64_t mass_done;          // decision: the tile's block sums are in (128 arrivals) [k]
};
// The mbarriers the streams share.  Phases: u counts the uses of a ring slot, e
// the entries of the pair queue.
struct __align__(8) SharedBars {
  uint64_t full[kMaxSlots];    // ring slot loaded                                 [u]
  uint64_t empty[kMaxSlots];   // the MMAs reading the slot are complete          [u]
  uint64_t tq_full[kTq];       // pair queue entry written                         [e]
  uint64_t tq_empty[kTq];      // entry read by the 256 softmax threads
  uint64_t drain;              // the issuer's MMAs are complete
};

template <int D>
struct Layout {
  static constexpr uint32_t kTileBytes = kTile * D * 2;
  static constexpr uint32_t kChunkBytes = kTile * 128;  // 128 rows x 64 bf16
  static constexpr int kChunks = D / 64;
  static constexpr int kSlots = D == 128 ? 4 : 8;       // shared K/V ring
  // Q of stream 0 and 1, the ring, then one 64-column staging chunk per stream
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kRing = 2 * kTileBytes;
  static constexpr uint32_t kStage = kRing + kSlots * kTileBytes;
  static constexpr uint32_t kBytes = kStage + 2 * kChunkBytes + 1024;
};

// A pair: query blocks 2 pp and 2 pp + 1 of (batch b, head h) of problem p.
struct PairCoord {
  int p, b, h, pp;
  int nqb, nkb, row0;  // the problem's query and key block counts and first query row
};
template <bool MULTI>
__device__ __forceinline__ PairCoord pair_coord(int P, const Args& a) {
  int p = 0;
  if constexpr (MULTI) {
    while (p + 1 < a.n_problems && P >= a.prob[p + 1].pair0) ++p;
  }
  const int nqb = a.prob[p].nqb;
  const int npp = (nqb + 1) >> 1;
  const int lp = MULTI ? P - a.prob[p].pair0 : P;  // a single problem starts at pair 0, row 0
  const int bh = lp / npp;
  return PairCoord{p, bh / a.H, bh % a.H, lp % npp, nqb, a.prob[p].nkb,
                   MULTI ? a.prob[p].q_row0 : 0};
}

// Number of blocks stream s runs in pair pc (0 when its query block does not
// exist or its list is empty) and its list.  A bad count is reported by the
// producer, which reads every pair first; it is clamped to [0, idx_row_len].  The
// decision instantiation attends densely over the problem's whole key prefix and
// walks it twice: a first sweep (score MMAs only) for each row's log-sum-exp, then
// a second with P and O.
template <bool DEC>
__device__ __forceinline__ int stream_list(const PairCoord& pc, int s, const Args& a, bool report,
                                           const int32_t** list) {
  const int qb = 2 * pc.pp + s;
  if (list) *list = nullptr;
  if (qb >= pc.nqb) return 0;
  if constexpr (DEC) {
    return 2 * pc.nkb;
  } else {
    const Problem& pr = a.prob[pc.p];
    const int64_t lrow = pc.b * pr.list_sb + pc.h * pr.list_sh + qb;
    int n = __ldg(pr.kv_cnt + lrow);
    if (n < 0 || n > pr.idx_row_len) {
      if (report && a.dev_status) atomicOr(a.dev_status, 0x1);
      n = n < 0 ? 0 : pr.idx_row_len;
    }
    if (list) *list = pr.kv_idx + lrow * pr.idx_row_len;
    return n;
  }
}

// KV block of entry j of a stream's sequence of length n, and whether the entry
// has a PV MMA (every entry, except those of the first decision sweep)
template <bool DEC>
__device__ __forceinline__ int seq_kb(const int32_t* list, int j, int n) {
  if constexpr (DEC) {
    return j < n / 2 ? j : j - n / 2;
  } else {
    return __ldg(list + j);
  }
}
template <bool DEC>
__device__ __forceinline__ bool seq_pv(int j, int n) {
  return !DEC || j >= n / 2;
}

// The merged sequence of a pair: the two streams' sequences walked together, an
// entry shared when both streams' next blocks are equal, else the smaller one
// alone.  Ascending lists (the library's layout) merge into their union; any
// other order still gives each stream its own list in its own order.  In the
// decision instantiation both sequences are the same and every entry is shared.
// One stream's tile of a pair.
struct TileCoord {
  int p, b, h, qb;
  int nkb, row0;  // the problem's key-block count and first query row
};

template <bool DEC>
struct Merge {
  const int32_t* l0;
  const int32_t* l1;
  int n0, n1, i0, i1;
  int kb;        // the entry's KV block
  bool in0, in1;  // the streams that run it
  bool pv;       // whether it has PV MMAs
  __device__ __forceinline__ bool next() {
    const bool h0 = i0 < n0, h1 = i1 < n1;
    if (!h0 && !h1) return false;
    if constexpr (DEC) {
      const int n = h0 ? n0 : n1;
      const int j = h0 ? i0 : i1;
      kb = seq_kb<DEC>(nullptr, j, n);
      pv = seq_pv<DEC>(j, n);
      in0 = h0;
      in1 = h1;
      i0 += h0;
      i1 += h1;
      return true;
    } else {
      const int x = h0 ? __ldg(l0 + i0) : 0, y = h1 ? __ldg(l1 + i1) : 0;
      pv = true;
      if (h0 && h1 && x == y) {
        kb = x;
        in0 = in1 = true;
        ++i0;
        ++i1;
      } else if (h0 && (!h1 || x < y)) {
        kb = x;
        in0 = true;
        in1 = false;
        ++i0;
      } else {
        kb = y;
        in0 = false;
        in1 = true;
        ++i1;
      }
      return true;
    }
  }
};

// Warp-uniform bounded wait (the softmax's tcgen05.ld/st are warp-collective).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          int32_t* st) {
  const bool ok = mbar_wait(bar, parity, abort, st, 0x2, kWaitNs);
  return __all_sync(0xffffffffu, ok);
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
    const int ci = static_cast<int>(static_cast<int64_t>(i) * sm / sk);
    const int cj = static_cast<int>(static_cast<int64_t>(j) * sm / sk);
    const int c0 = max(cj - r, 0), c1 = min(cj + r, sm - 1);
    const int a0 = max(max(ci - r, 0), (max(k0, o0) - o0) / sm);
    const int a1 = min(min(ci + r, sm - 1), (min(k1, o1) - 1 - o0) / sm);
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
// launch holds several problems (args.prob), one output map each.  DEC: dense
// attention over each problem's prefix that also pools the attention weights per
// (query block, KV block) and selects the kept blocks (CS4A decision scale).
template <int D, bool TOK, bool MULTI, bool DEC>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ OutMaps tm_os, const __grid_constant__ Args args) {
  using L = Layout<D>;
  constexpr int NS = L::kSlots;
  extern __shared__ uint8_t smem_raw[];
  __shared__ StreamBars bars_sh[2];
  __shared__ SharedBars sb;
  __shared__ int tq_pair_sh[kTq];
  __shared__ uint32_t item_meta_sh[kMaxSlots];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  __shared__ float mass_sh[DEC ? 2 : 1][DEC ? kMaxDecBlocks : 1];     // decision: block sums
  __shared__ uint8_t kept_sh[DEC ? 2 : 1][DEC ? kMaxDecBlocks : 1];   // decision: selection

  const uint32_t smem_base = (smem_addr(smem_raw) + 1023u) & ~1023u;
  uint8_t* smem_gen = smem_raw + (smem_base - smem_addr(smem_raw));
  const int warp = warp_id();
  const int lane = lane_id();
  volatile int* abort_flag = &abort_sh;
  int32_t* dev_status = args.dev_status;
  // a single problem's pair count is its shape's (equal to total_pairs); written so,
  // the compiler relates pair ids to pair coordinates
  const int total = MULTI ? args.total_pairs : args.B * args.H * ((args.prob[0].nqb + 1) >> 1);

  if constexpr (DEC) {
    for (int i = threadIdx.x; i < 2 * kMaxDecBlocks; i += kThreads) {
      mass_sh[i / kMaxDecBlocks][i % kMaxDecBlocks] = 0.f;
      kept_sh[i / kMaxDecBlocks][i % kMaxDecBlocks] = 0;
    }
  }
  if (threadIdx.x == 0) {
    abort_sh = 0;
    for (int s = 0; s < 2; ++s) {
      StreamBars& b = bars_sh[s];
      mbar_init(&b.q_full, 1);
      mbar_init(&b.q_free, 1);
      mbar_init(&b.s_full, 1);
      mbar_init(&b.p_full, 128);
      mbar_init(&b.o_done, 1);
      mbar_init(&b.mass_done, 128);
    }
    for (int i = 0; i < NS; ++i) {
      mbar_init(&sb.full[i], 1);
      mbar_init(&sb.empty[i], 1);
    }
    for (int i = 0; i < kTq; ++i) {
      mbar_init(&sb.tq_full[i], 1);
      mbar_init(&sb.tq_empty[i], 256);
    }
    mbar_init(&sb.drain, 1);
    fence_barrier_init();
  }
  if (warp == kIssuerWarp) {
    tmem_alloc(&tmem_base_sh, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_os.m[0]);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  auto sQ = [&](int st) { return smem_base + L::kQ + st * L::kTileBytes; };
  auto sSlot = [&](int i) { return smem_base + L::kRing + i * L::kTileBytes; };

  if (warp >= 8) {
   setmaxnreg_dec<kControlRegs>();
   if (warp == kProducerWarp) {
    // ================================================================ producer
    if (lane == 0) {
      int e = 0;                  // pair queue entries written
      int items = 0;              // ring items issued
      int kq[2] = {0, 0};         // Q loads issued per stream (one per non-empty tile)
      int pos = 0;                // pairs claimed
      bool ok = true;
      // the next ring slot, once the MMAs that read its previous item are complete
      auto acquire_slot = [&]() -> int {
        const int i = items % NS;
        if (!mbar_wait(&sb.empty[i], ((items / NS) & 1) ^ 1, abort_flag, dev_status, 0x2,
                       kWaitNs)) {
          ok = false;
          return -1;
        }
        return i;
      };
      // one K or V block into the next slot, with the item's flags for the issuers
      auto load = [&](const CUtensorMap* tm, int kb, const PairCoord& pc, uint32_t meta) {
        const int i = acquire_slot();
        if (i < 0) return;
        kb = kb < 0 ? -1 : (kb > pc.nkb ? pc.nkb : kb);  // out of range: zero-filled, masked
        item_meta_sh[i] = meta;
        mbar_arrive_expect_tx(&sb.full[i], L::kTileBytes);
#pragma unroll
        for (int c = 0; c < L::kChunks; ++c)
          tma_load_4d(sSlot(i) + c * L::kChunkBytes, tm, &sb.full[i], c * 64, kb * kTile, pc.h,
                      pc.b);
        ++items;
      };
      // Q of stream st's tile, once its previous tile's last score MMA no longer reads the buffer
      auto load_q = [&](int st, const PairCoord& pc) {
        StreamBars& bs = bars_sh[st];
        if (kq[st] > 0 &&
            !mbar_wait(&bs.q_free, (kq[st] - 1) & 1, abort_flag, dev_status, 0x2, kWaitNs)) {
          ok = false;
          return;
        }
        mbar_arrive_expect_tx(&bs.q_full, L::kTileBytes);
#pragma unroll
        for (int c = 0; c < L::kChunks; ++c)
          tma_load_4d(sQ(st) + c * L::kChunkBytes, &tm_q, &bs.q_full, c * 64,
                      pc.row0 + (2 * pc.pp + st) * kTile, pc.h, pc.b);
        ++kq[st];
      };
      while (ok) {
        // claim the CTA's next pair and publish it to the softmax warps
        const int64_t P64 = blockIdx.x + static_cast<int64_t>(pos++) * gridDim.x;
        const int P = P64 < total ? static_cast<int>(P64) : -1;
        const int q = e % kTq;
        if (!mbar_wait(&sb.tq_empty[q], ((e / kTq) & 1) ^ 1, abort_flag, dev_status, 0x2,
                       kWaitNs))
          break;
        tq_pair_sh[q] = P;
        mbar_arrive(&sb.tq_full[q]);
        ++e;
        if (P < 0) break;
        const PairCoord pc = pair_coord<MULTI>(P, args);
        {
          // the next pair's Q tiles into L2 now, so that their loads after this pair's
          // last score MMAs are short
          const int64_t Pn = P64 + gridDim.x;
          if (Pn < total) {
            const PairCoord pn = pair_coord<MULTI>(static_cast<int>(Pn), args);
            for (int st = 0; st < 2; ++st) {
              if (2 * pn.pp + st >= pn.nqb) continue;
#pragma unroll
              for (int c = 0; c < L::kChunks; ++c)
                tma_prefetch_4d(&tm_q, c * 64, pn.row0 + (2 * pn.pp + st) * kTile, pn.h, pn.b);
            }
          }
        }
        Merge<DEC> m{};
        m.n0 = stream_list<DEC>(pc, 0, args, true, &m.l0);
        m.n1 = stream_list<DEC>(pc, 1, args, true, &m.l1);
        if (m.n0 + m.n1 == 0) continue;
        const int n[2] = {m.n0, m.n1};
        const int npv[2] = {DEC ? m.n0 / 2 : m.n0, DEC ? m.n1 / 2 : m.n1};
        int ns[2] = {0, 0}, nv[2] = {0, 0};  // score and PV items per stream so far
        if (m.n0 > 0) load_q(0, pc);
        if (ok && m.n1 > 0) load_q(1, pc);
        // flags of the K item of the current entry and of the V item
        auto k_meta = [&]() {
          uint32_t f = 0;
          const bool in[2] = {m.in0, m.in1};
          for (int st = 0; st < 2; ++st) {
            if (!in[st]) continue;
            f |= kItemUse << st;
            if (ns[st] == 0) f |= kItemFirst << st;
            if (++ns[st] == n[st]) f |= kItemLast << st;
          }
          return f;
        };
        // ring order: K of the first entry, then per entry: V (if the entry has PV
        // MMAs) and the K of the next entry
        m.next();
        if (ok) load(&tm_k, m.kb, pc, k_meta());
        while (ok) {
          const int kb = m.kb;
          const bool pv = m.pv;
          const bool in[2] = {m.in0, m.in1};
          const bool more = m.next();
          if (pv) {
            uint32_t f = kItemV;
            for (int st = 0; st < 2; ++st) {
              if (!in[st]) continue;
              f |= kItemUse << st;
              if (nv[st] == 0) f |= kItemFirst << st;
              if (++nv[st] == npv[st]) f |= kItemLast << st;
            }
            load(&tm_v, kb, pc, f);
          }
          if (!more || !ok) break;
          load(&tm_k, m.kb, pc, k_meta());
        }
      }
      // the end of the item stream for the issuers
      if (ok) {
        const int i = acquire_slot();
        if (i >= 0) {
          item_meta_sh[i] = kItemEnd;
          mbar_arrive(&sb.full[i]);
          ++items;
        }
      }
      // drain: every issued TMA write lands before the CTA exits
      for (int st = 0; st < 2; ++st)
        if (kq[st] > 0) mbar_drain(&bars_sh[st].q_full, (kq[st] - 1) & 1, kDrainNs);
      for (int i = 0; i < NS; ++i) {
        const int issued = items > i ? (items - 1 - i) / NS + 1 : 0;  // items in slot i
        if (issued) mbar_drain(&sb.full[i], (issued - 1) & 1, kDrainNs);
      }
    }
    __syncwarp();
   } else if (warp == kIssuerWarp) {
    // ================================================================ MMA issue
    // The issuer follows the ring items in order, taking a V item together with the
    // K item after it.  For each stream that uses them it issues the group [PV of
    // the stream's block on V, S of its next block on K]; the streams' groups go to
    // the tensor core one after the other, whichever stream's P is ready first.
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(kTile, kTile, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kTile, D, 1);
      constexpr uint32_t kBufStep = L::kTileBytes >> 4;  // descriptor units per slot
      const uint64_t dq = smem_desc_sw128(sQ(0), 16, 1024);
      const uint64_t dk = smem_desc_sw128(sSlot(0), 16, 1024);
      const uint64_t dv = smem_desc_sw128(sSlot(0), L::kChunkBytes, 1024);
      int items = 0;
      // per stream: p_full waits (one per block), tiles (q_full / q_free phases), and
      // whether a block's P has not been waited for yet (no PV since its S)
      int J0 = 0, J1 = 0, k0 = 0, k1 = 0;
      bool pp0 = false, pp1 = false;
      bool ok = true, end = false;
      auto next_item = [&](uint32_t& meta) -> int {
        const int i = items % NS;
        ok = ok && mbar_wait(&sb.full[i], (items / NS) & 1, abort_flag, dev_status, 0x2, kWaitNs);
        ++items;
        meta = ok ? item_meta_sh[i] : kItemEnd;
        return i;
      };
      // stream st's group on V slot iv (flags vm) and K slot ik (flags km), if it is
      // ready; returns whether it was issued
      auto group = [&](auto stc, uint32_t vm, uint32_t km, int iv, int ik, int& J, int& k,
                       bool& pp) -> bool {
        constexpr int st = decltype(stc)::value;
        StreamBars& bs = bars_sh[st];
        const bool use_v = (vm >> st) & kItemUse, use_k = (km >> st) & kItemUse;
        const bool need_p = use_v || (use_k && pp);
        if (need_p && !mbar_try_wait(&bs.p_full, J & 1)) return false;
        if (use_k && ((km >> st) & kItemFirst) && !mbar_try_wait(&bs.q_full, k & 1)) return false;
        if (need_p) {
          ++J;
          pp = false;
        }
        tc_fence_after();
        const uint32_t s_col = tmem + 256u * st;
        if (use_v) {
          const uint64_t dvs = dv + static_cast<uint64_t>(iv * kBufStep);
          const uint32_t acc0 = ((vm >> st) & kItemFirst) ? 0u : 1u;
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            mma_ts(s_col + 128, s_col + kk * 8, dvs + static_cast<uint64_t>(kk * (2048 >> 4)),
                   idesc_pv, kk > 0 ? 1u : acc0);
          if ((vm >> st) & kItemLast) mma_commit(&bs.o_done);
        }
        if (use_k) {
          const uint64_t dqs = dq + static_cast<uint64_t>(st * kBufStep);
          const uint64_t dks = dk + static_cast<uint64_t>(ik * kBufStep);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = ((kk >> 2) * L::kChunkBytes + (kk & 3) * 32) >> 4;
            mma_ss(s_col, dqs + off, dks + off, idesc_s, kk > 0 ? 1u : 0u);
          }
          if ((km >> st) & kItemLast) {
            mma_commit(&bs.q_free);
            ++k;
          }
          mma_commit(&bs.s_full);
          pp = true;
        }
        return true;
      };
      while (ok && !end) {
        uint32_t m1, m2 = 0;
        const int i1 = next_item(m1);
        if (m1 & kItemEnd) break;
        int iv = -1, ik = i1;
        uint32_t vm = 0, km = m1;
        if (m1 & kItemV) {
          iv = i1;
          vm = m1;
          ik = next_item(m2);
          km = m2;
          if (m2 & kItemEnd) {
            end = true;
            ik = -1;
            km = 0;
          }
        }
        if (!ok) break;
        // each stream's group, in the order the streams become ready
        bool todo0 = (vm | km) & kItemUse, todo1 = ((vm | km) >> 1) & kItemUse;
        const uint64_t t0 = global_timer_ns();
        for (uint32_t spin = 0; todo0 || todo1; ++spin) {
          if (todo0 && group(std::integral_constant<int, 0>{}, vm, km, iv, ik, J0, k0, pp0))
            todo0 = false;
          if (todo1 && group(std::integral_constant<int, 1>{}, vm, km, iv, ik, J1, k1, pp1))
            todo1 = false;
          if ((spin & 15u) == 15u && (todo0 || todo1)) {
            if (*abort_flag) {
              ok = false;
              break;
            }
            if (global_timer_ns() - t0 > kWaitNs) {
              *abort_flag = 1;
              if (dev_status) atomicOr(dev_status, 0x2);
              ok = false;
              break;
            }
          }
        }
        if (!ok) break;
        if (iv >= 0) mma_commit(&sb.empty[iv]);
        if (ik >= 0) mma_commit(&sb.empty[ik]);
      }
      mma_commit(&sb.drain);
      mbar_drain(&sb.drain, 0, kDrainNs);
    }
    __syncwarp();
   }
  } else {
    setmaxnreg_inc<kSoftmaxRegs>();
    const int s = warp >> 2;  // the stream this warpgroup serves
    StreamBars& bs = bars_sh[s];
    const uint32_t tmem_s = tmem + 256u * s;        // S_s
    const uint32_t tmem_o = tmem + 256u * s + 128;  // O_s
    // ================================================================ softmax
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t s_addr = tmem_s + lane_off;
    const uint32_t o_addr = tmem_o + lane_off;
    const float csc = args.scale_log2;
    // this warp's 32 rows of the stream's staging chunk (4 KB, 1024-byte aligned)
    const uint32_t stage_off = L::kStage + s * L::kChunkBytes + quad * (kOutBoxRows * 128);
    uint8_t* stage = smem_gen + stage_off;
    const uint32_t stage_addr = smem_base + stage_off;
    int e = 0, J = 0, k = 0;
    bool good = true;
    bool store_pending = false;  // lane 0: a TMA store may still read the warp's stage

    while (good) {
      // next pair from the queue; this stream runs its query block 2 pp + s
      const int q = e % kTq;
      if (!warp_wait(&sb.tq_full[q], (e / kTq) & 1, abort_flag, dev_status)) break;
      const int P = tq_pair_sh[q];
      mbar_arrive(&sb.tq_empty[q]);
      ++e;
      if (P < 0) break;
      const PairCoord pc = pair_coord<MULTI>(P, args);
      const TileCoord tc{pc.p, pc.b, pc.h, 2 * pc.pp + s, pc.nkb, pc.row0};
      if (tc.qb >= pc.nqb) continue;  // the pair's second query block does not exist
      const int32_t* list = nullptr;
      const int n = stream_list<DEC>(pc, s, args, false, &list);
      const Problem& pr = args.prob[MULTI ? tc.p : 0];
      const int p_lkv = pr.Lkv, p_lq = pr.Lq;
      const int grow = tc.qb * kTile + row;
      float m_run = -INFINITY;  // reference of the row (log2 units)
      float l_run = 0.f;

      for (int j = 0; j < n; ++j, ++J) {
        const int kb = seq_kb<DEC>(list, j, n);
        const bool sweep_a = DEC && j < n / 2;  // decision: log-sum-exp sweep, no P
        if (!warp_wait(&bs.s_full, J & 1, abort_flag, dev_status)) {
          good = false;
          break;
        }
        tc_fence_after();
        // this row's keep mask over the block's 128 columns
        uint32_t km[4] = {~0u, ~0u, ~0u, ~0u};
        if (kb < 0 || kb >= tc.nkb) {
          km[0] = km[1] = km[2] = km[3] = 0u;
          if (row == 0 && dev_status) atomicOr(dev_status, 0x1);
        } else if ((kb + 1) * kTile > p_lkv) {
          const int valid = p_lkv - kb * kTile;
#pragma unroll
          for (int w = 0; w < 4; ++w)
            km[w] = valid >= 32 * (w + 1) ? ~0u
                                          : (valid <= 32 * w ? 0u : ((1u << (valid - 32 * w)) - 1u));
        }
        if (args.tile_mask) {
          // bit i of the row's fine-block bits keeps columns [i << shift, (i + 1) << shift)
          const int sh = args.mask_shift;
          const int fg = kTile >> sh;
          const uint64_t mk = __ldg(args.tile_mask + (list - pr.kv_idx) + j);
          const uint32_t keep = static_cast<uint32_t>(mk >> ((row >> sh) * fg)) & ((1u << fg) - 1u);
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            uint32_t wm;
            if (sh == 4) {
              wm = (((keep >> (2 * w)) & 1u) ? 0x0000ffffu : 0u) |
                   (((keep >> (2 * w + 1)) & 1u) ? 0xffff0000u : 0u);
            } else if (sh == 5) {
              wm = ((keep >> w) & 1u) ? ~0u : 0u;
            } else {
              wm = ((keep >> (w >> 1)) & 1u) ? ~0u : 0u;
            }
            km[w] &= wm;
          }
        }
        if constexpr (TOK) {
          const int sk = args.tok.side[args.tok.q_scale];
          const int gq = grow < p_lq ? grow : 0;
          if (kb >= 0 && kb < tc.nkb) {
            uint32_t kt[4];
            csla_row_mask(args.tok, gq / sk, gq % sk, kb * kTile, min(kb * kTile + kTile, p_lkv),
                          kt);
#pragma unroll
            for (int w = 0; w < 4; ++w) km[w] &= kt[w];
          }
        }
        const bool masked = __any_sync(0xffffffffu, (km[0] & km[1] & km[2] & km[3]) != ~0u);
        // the block's 128 scores of this row, in registers for the whole block
        uint32_t sr[kTile];
        tmem_ld128_wait(s_addr, sr);
        if (masked) {
#pragma unroll
          for (int c = 0; c < kTile; ++c)
            if (!((km[c >> 5] >> (c & 31)) & 1u)) sr[c] = __float_as_uint(-INFINITY);
        }
        auto row_max = [&]() {
          float mx0 = fmaxf(__uint_as_float(sr[0]), __uint_as_float(sr[4]));
          float mx1 = fmaxf(__uint_as_float(sr[1]), __uint_as_float(sr[5]));
          float mx2 = fmaxf(__uint_as_float(sr[2]), __uint_as_float(sr[6]));
          float mx3 = fmaxf(__uint_as_float(sr[3]), __uint_as_float(sr[7]));
#pragma unroll
          for (int c = 8; c < kTile; c += 8) {
            mx0 = max3(mx0, __uint_as_float(sr[c]), __uint_as_float(sr[c + 4]));
            mx1 = max3(mx1, __uint_as_float(sr[c + 1]), __uint_as_float(sr[c + 5]));
            mx2 = max3(mx2, __uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 6]));
            mx3 = max3(mx3, __uint_as_float(sr[c + 3]), __uint_as_float(sr[c + 7]));
          }
          return fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * csc;
        };
        if (sweep_a) {
          // decision, first sweep: the row's running log-sum-exp, reference max(m, bm),
          // the sum rescaled exactly; S has been read, so the next score MMA may
          // overwrite it
          const float bm = row_max();
          const float m_new = fmaxf(m_run, bm);
          const float nm = m_new == -INFINITY ? 0.f : -m_new;
          const uint64_t sc2 = f2_pack(csc, csc), nm2 = f2_pack(nm, nm);
          uint64_t a0 = 0, a1 = 0;
#pragma unroll
          for (int c = 0; c < kTile; c += 4) {
            float e0, e1, e2, e3;
            f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sc2, nm2),
                      e0, e1);
            f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3])), sc2,
                             nm2),
                      e2, e3);
            a0 = f2_add(a0, f2_pack(ex2_approx(e0), ex2_approx(e1)));
            a1 = f2_add(a1, f2_pack(ex2_approx(e2), ex2_approx(e3)));
          }
          float x0, x1;
          f2_unpack(f2_add(a0, a1), x0, x1);
          l_run = (m_run == -INFINITY ? 0.f : l_run * ex2_approx(m_run - m_new)) + x0 + x1;
          m_run = m_new;
          if (j + 1 == n / 2) {
            // end of the sweep: the row's log-sum-exp is the fixed reference of the
            // second sweep, whose P is then already normalised
            m_run = l_run > 0.f ? m_run + __log2f(l_run) : -INFINITY;
            l_run = 1.f;
          }
          tc_fence_before();
          mbar_arrive(&bs.p_full);
          continue;
        }
        // O and the row sum move to a new reference m_new (per lane; O is quiescent:
        // S(j) complete implies PV(j - 1) complete)
        auto raise_to = [&](bool raise, float m_new) {
          const bool o_live = raise && m_run != -INFINITY;
          if (__any_sync(0xffffffffu, o_live)) {
            const float alpha = o_live ? ex2_approx(m_run - m_new) : 1.f;
            l_run *= alpha;
#pragma unroll 1
            for (int cc = 0; cc < D / 16; ++cc) {
              uint32_t orr[16];
              tmem_ld16_wait(o_addr + cc * 16, orr);
#pragma unroll
              for (int c = 0; c < 16; ++c) orr[c] = __float_as_uint(__uint_as_float(orr[c]) * alpha);
              tmem_st16(o_addr + cc * 16, orr);
            }
          }
          if (raise) m_run = m_new;
        };
        // P = 2^(s * scale - m) in packed pairs, written over TMEM columns [8cc, 8cc + 8)
        // of the scores (already in registers) as packed bf16; with TRACK the raw row max
        // is formed alongside (it fills issue slots the exponentials leave free)
        const uint64_t sc2 = f2_pack(csc, csc);
        uint64_t acc0 = 0, acc1 = 0;  // (0.f, 0.f)
        auto exp_pass = [&](auto track) {
          const float neg = (m_run == -INFINITY) ? 0.f : -m_run;
          const uint64_t neg2 = f2_pack(neg, neg);
          float t0 = -INFINITY, t1 = -INFINITY;
          acc0 = acc1 = 0;
#pragma unroll
          for (int cc = 0; cc < kTile / 16; ++cc) {
            uint32_t pk[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const float x0 = __uint_as_float(sr[cc * 16 + 2 * c]);
              const float x1 = __uint_as_float(sr[cc * 16 + 2 * c + 1]);
              if constexpr (decltype(track)::value) {
                if (c & 1) {
                  t1 = max3(t1, x0, x1);
                } else {
                  t0 = max3(t0, x0, x1);
                }
              }
              float e0, e1;
              f2_unpack(f2_fma(f2_pack(x0, x1), sc2, neg2), e0, e1);
              const float p0 = ex2_approx(e0);
              const float p1 = ex2_approx(e1);
              if (c & 1) {
                acc1 = f2_add(acc1, f2_pack(p0, p1));
              } else {
                acc0 = f2_add(acc0, f2_pack(p0, p1));
              }
              pk[c] = pack_bf16x2(p0, p1);
            }
            tmem_st8(s_addr + cc * 8, pk);
          }
          return fmaxf(t0, t1) * csc;
        };
        if (DEC) {
          // decision, second sweep: the fixed reference is the row's log-sum-exp
          exp_pass(std::false_type{});
        } else if (__any_sync(0xffffffffu, m_run == -INFINITY)) {
          // a row without a reference yet (a tile's first block): the block max first
          const float bm = row_max();
          raise_to(m_run == -INFINITY ? (bm != -INFINITY) : (bm > m_run + kLazyRescale), bm);
          exp_pass(std::false_type{});
        } else {
          // against the current reference, the block max formed alongside; in the rare
          // case that it exceeds the reference by more than 2^8 the reference is raised
          // and the block redone
          const float bm = exp_pass(std::true_type{});
          const bool raise = bm > m_run + kLazyRescale;
          if (__any_sync(0xffffffffu, raise)) {
            tmem_wait_st();
            raise_to(raise, bm);
            exp_pass(std::false_type{});
          }
        }
        {
          float a0, a1;
          f2_unpack(f2_add(acc0, acc1), a0, a1);
          if constexpr (DEC) {
            // decision: the block's share of the attention weights, summed over the
            // tile's valid rows
            float part = grow < p_lq ? a0 + a1 : 0.f;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
            if (lane == 0) atomicAdd(&mass_sh[s][kb], part);
            if (j + 1 == n) mbar_arrive(&bs.mass_done);
          } else {
            l_run += a0 + a1;
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bs.p_full);
      }
      if (!good) break;

      // ---- epilogue of the tile
      const float l = l_run;
      if (n > 0) {
        if (!warp_wait(&bs.o_done, k & 1, abort_flag, dev_status)) break;
        tc_fence_after();
        // O into registers as normalised packed bf16
        const float inv_l = l > 0.f ? 1.f / l : 0.f;
        uint32_t pk[D / 2];
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t ro[32];
          tmem_ld32_wait(o_addr + cc * 32, ro);
#pragma unroll
          for (int c = 0; c < 16; ++c)
            pk[cc * 16 + c] = pack_bf16x2(__uint_as_float(ro[2 * c]) * inv_l,
                                          __uint_as_float(ro[2 * c + 1]) * inv_l);
        }
        if constexpr (DEC) {
          // warp 0 of the stream: pooled mass and selection once every warp's sums are in
          if (quad == 0) {
            if (!warp_wait(&bs.mass_done, k & 1, abort_flag, dev_status)) break;
            const int64_t rowid =
                (static_cast<int64_t>(tc.b) * args.H + tc.h) * pr.nqb + tc.qb;
            select_blocks_warp(mass_sh[s], kept_sh[s], tc.nkb, min(kTile, p_lq - tc.qb * kTile),
                               args.topk, args.mass_threshold,
                               args.mass_out ? args.mass_out + rowid * tc.nkb : nullptr,
                               args.sel_idx + rowid * tc.nkb, args.sel_cnt + rowid);
          }
        }
        ++k;
        // each 64-column chunk of the warp's 32 rows into the warp's stage, in the output
        // map's 128B-swizzled layout (16-byte unit u of row r at position u ^ (r mod 8)),
        // then one TMA store of 64 columns x 32 rows
        const int row0 = tc.qb * kTile + quad * kOutBoxRows;  // the warp's first row
        if (row0 < p_lq) {
#pragma unroll
          for (int ch = 0; ch < L::kChunks; ++ch) {
            if (lane == 0 && store_pending) bulk_wait_read_all();
            __syncwarp();
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              uint4* dst = reinterpret_cast<uint4*>(stage + lane * 128 + ((u ^ (lane & 7)) << 4));
              const int w = ch * 32 + 4 * u;
              *dst = make_uint4(pk[w], pk[w + 1], pk[w + 2], pk[w + 3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_4d(&tm_os.m[MULTI ? tc.p : 0], stage_addr, ch * 64, row0, tc.h, tc.b);
              bulk_commit_group();
              store_pending = true;
            }
          }
        }
      } else if (grow < p_lq) {
        // empty list: zero rows
        __nv_bfloat16* orow = args.o + tc.b * args.o_sb + tc.h * args.o_sh +
                              (static_cast<int64_t>(tc.row0) + grow) * args.o_sr;
#pragma unroll
        for (int v = 0; v < D / 8; ++v)
          reinterpret_cast<uint4*>(orow)[v] = make_uint4(0u, 0u, 0u, 0u);
      }
      if (args.lse && grow < p_lq) {
        args.lse[(static_cast<int64_t>(tc.b) * args.H + tc.h) * args.lse_rows + tc.row0 + grow] =
            (n > 0 && l > 0.f) ? (m_run + __log2f(l)) * 0.6931471805599453f : -INFINITY;
      }
    }
    if (lane == 0 && store_pending) bulk_wait_all();  // output stores complete before exit
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kIssuerWarp) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace fwd
}  // namespace sparvar
