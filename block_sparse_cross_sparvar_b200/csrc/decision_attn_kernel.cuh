// The CS4A decision scale on sm_100a: dense attention over each problem's key
// prefix with the pooled attention mass per (query block, KV block) and the block
// selection fused in, as a persistent kernel over pairs of query tiles that share
// one K/V stream.
//
// A query tile is one 128-row query block of one batch item and head.  The tiles
// of query blocks 2i and 2i + 1 of one (batch, head) form a pair; both attend to
// every key block of the prefix, so each K/V block is loaded into shared memory
// once for the two.  Each tile walks the prefix twice: a first sweep of score
// MMAs only gives each row's log-sum-exp; the second computes P normalised by it,
// O, and each block's share of the attention weights, summed over the tile's rows
// (the pooled mass); after the last block the tile's blocks are selected by mass
// (heaviest first until the threshold, or the Top-K count).  Each CTA owns one SM
// and claims pairs one at a time.  Stream s = 0, 1 of a CTA runs tile 2i + s.
// Roles:
//   warps 4s..4s+3   softmax of stream s (thread t: query row t, TMEM lane t)
//   warp  8          MMA issue of stream 0 (one lane) and TMEM owner
//   warp  9          TMA producer (one lane): claims pairs, loads Q and K/V
//   warp  10         MMA issue of stream 1 (one lane)
//   warp  11         idle (it completes the control warpgroup)
// TMEM (512 columns): stream s has its score buffer S_s = [256s, 256s + 128) and
// its output accumulator O_s = [256s + 128, 256s + 128 + D).  P (packed bf16)
// is written over the first 64 columns of S_s and feeds the PV MMA from TMEM.
// Shared memory: Q of each stream, a ring of K/V slots shared by the streams,
// and a 64-column output staging buffer per stream.
//
// MMA order.  For each entry u of the pair's sequence (a KV block and the streams
// that run it), issuer s issues PV_s(u) if the entry has PV MMAs, then S_s of
// the stream's next block (entry u + 1).  One thread's MMAs run in issue order,
// so S_s may overwrite the P that PV_s has read, and the completion of S_s(j)
// implies that of PV_s of the stream's previous block: once S_s(j) is complete
// no MMA touches O_s until P_s(j) is handed over, which lets the softmax rescale
// O_s in place.  The two streams' groups take turns on the tensor core (stream
// 0's of entry u, stream 1's of u, stream 0's of u + 1, ...) while each stream's
// softmax works on its next block.
//
// Softmax per block: the 128 scores of a row stay in registers.  First sweep:
// the row's running log-sum-exp (reference max(m, block max), the sum rescaled
// exactly).  Second sweep: P = 2^(s * scale - lse) in packed f32x2 arithmetic,
// already normalised; the block's mass is the sum of P over the tile's valid
// rows.  Keys past the prefix are set to -inf first.  Epilogue per tile: wait
// until the stream's last PV of the pair is complete and read O into registers;
// the warp's P of the next tile's first block comes after that read, so the PV
// that overwrites O cannot start before it.  Warp 0 of the stream selects the
// blocks once every warp's sums are in.  Then each warp stages its 32 rows as
// bf16 in the 128B-swizzled layout and stores them by TMA.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx.cuh"
#include "select.cuh"
#include "tmem_io.cuh"

namespace sparvar {
namespace dec {

constexpr int kTile = 128;
constexpr int kThreads = 384;  // 12 warps
constexpr int kIssuerWarp = 8;
constexpr int kProducerWarp = 9;
constexpr int kIssuerWarp1 = 10;  // MMA issue of stream 1
// flags of a ring item (item_meta_sh): kItemV a V block (else K); per stream st,
// shifted by st: kItemUse the stream's MMA reads it, kItemFirst its first score /
// PV MMA of the tile, kItemLast its last one; kItemEnd: no more items
constexpr uint32_t kItemV = 1u << 8, kItemEnd = 1u << 9;
constexpr uint32_t kItemUse = 1u << 0, kItemFirst = 1u << 2, kItemLast = 1u << 4;
constexpr uint32_t kTmemCols = 512;
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

// One launch: queries [0, Lq) of every (batch, head) attend densely to keys
// [0, Lkv); the pooled mass, the selection and the attention output are written.
struct Args {
  int B, H, Lq, Lkv, nqb, nkb;
  int total_pairs;   // B * H * ceil(nqb / 2)
  float scale_log2;  // softmax_scale * log2(e)
  __nv_bfloat16* o;
  int64_t o_sb, o_sh, o_sr;
  float* lse;  // [B][H][Lq] or null
  int32_t* dev_status;
  // pooled mass [B][H][nqb][nkb] (or null), selection rule (topk > 0: keep topk
  // blocks; else the smallest heaviest-first set reaching mass_threshold) and the
  // selected lists [B][H][nqb] / [B][H][nqb][nkb]
  float* mass_out;
  int topk;
  float mass_threshold;
  int32_t* sel_cnt;
  int32_t* sel_idx;
};

// The mbarriers of one stream.  Phases: k counts the stream's non-empty tiles,
// J its blocks over all its tiles.
struct __align__(8) StreamBars {
  uint64_t q_full;             // Q of tile k landed                              [k]
  uint64_t q_free;             // last score MMA of tile k complete                [k]
  uint64_t s_full;             // S of block J in TMEM                             [J]
  uint64_t p_full;             // P of block J in TMEM (128 arrivals)              [J]
  uint64_t o_done;             // every PV of tile k complete                      [k]
  uint64_t mass_done;          // the tile's block sums are in (128 arrivals)      [k]
};
// The mbarriers the streams share.  Phases: u counts the uses of a ring slot, e
// the entries of the pair queue.
struct __align__(8) SharedBars {
  uint64_t full[kMaxSlots];    // ring slot loaded                                 [u]
  uint64_t empty[kMaxSlots];   // both issuers are done with the slot's item        [u]
  uint64_t tq_full[kTq];       // pair queue entry written                         [e]
  uint64_t tq_empty[kTq];      // entry read by the 256 softmax threads
  uint64_t turn[2];            // issuer st has issued its group of entry n        [n]
  uint64_t drain;              // both issuers' MMAs are complete
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

// A pair: query blocks 2 pp and 2 pp + 1 of (batch b, head h).
struct PairCoord {
  int b, h, pp;
};
__device__ __forceinline__ PairCoord pair_coord(int P, const Args& a) {
  const int npp = (a.nqb + 1) >> 1;
  const int bh = P / npp;
  return PairCoord{bh / a.H, bh % a.H, P % npp};
}

// The walk of a pair: every KV block of the prefix twice (a first sweep of score
// MMAs only for each row's log-sum-exp, then a second with P and O), the entries
// shared by both streams (stream 0 alone when the pair's second tile does not
// exist); only the second sweep's entries have PV MMAs.
struct Walk {
  int nkb;
  bool two;  // the pair's second tile exists
  int i;     // entries walked
  int kb;    // the entry's KV block
  bool in0, in1;  // the streams that run it
  bool pv;        // whether it has PV MMAs
  __device__ __forceinline__ bool next() {
    if (i >= 2 * nkb) return false;
    kb = i < nkb ? i : i - nkb;
    pv = i >= nkb;
    in0 = true;
    in1 = two;
    ++i;
    return true;
  }
};

// Warp-uniform bounded wait (the softmax's tcgen05.ld/st are warp-collective).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          int32_t* st) {
  const bool ok = mbar_wait(bar, parity, abort, st, 0x2, kWaitNs);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    decision_attn_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ CUtensorMap tm_o, const __grid_constant__ Args args) {
  using L = Layout<D>;
  constexpr int NS = L::kSlots;
  static_assert(NS >= 2, "the ring holds at least one entry of two items");
  extern __shared__ uint8_t smem_raw[];
  __shared__ StreamBars bars_sh[2];
  __shared__ SharedBars sb;
  __shared__ int tq_pair_sh[kTq];
  __shared__ uint32_t item_meta_sh[kMaxSlots];
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  __shared__ float mass_sh[2][kMaxDecBlocks];     // block sums of each stream's tile
  __shared__ uint8_t kept_sh[2][kMaxDecBlocks];   // selection scratch

  const uint32_t smem_base = (smem_addr(smem_raw) + 1023u) & ~1023u;
  uint8_t* smem_gen = smem_raw + (smem_base - smem_addr(smem_raw));
  const int warp = warp_id();
  const int lane = lane_id();
  volatile int* abort_flag = &abort_sh;
  int32_t* dev_status = args.dev_status;
  const int total = args.total_pairs;

  for (int i = threadIdx.x; i < 2 * kMaxDecBlocks; i += kThreads) {
    mass_sh[i / kMaxDecBlocks][i % kMaxDecBlocks] = 0.f;
    kept_sh[i / kMaxDecBlocks][i % kMaxDecBlocks] = 0;
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
      mbar_init(&sb.empty[i], 2);
    }
    for (int i = 0; i < kTq; ++i) {
      mbar_init(&sb.tq_full[i], 1);
      mbar_init(&sb.tq_empty[i], 256);
    }
    mbar_init(&sb.turn[0], 1);
    mbar_init(&sb.turn[1], 1);
    mbar_init(&sb.drain, 2);
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
    prefetch_tmap(&tm_o);
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
                      (2 * pc.pp + st) * kTile, pc.h, pc.b);
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
        const PairCoord pc = pair_coord(P, args);
        {
          // the next pair's Q tiles into L2 now, so that their loads after this pair's
          // last score MMAs are short
          const int64_t Pn = P64 + gridDim.x;
          if (Pn < total) {
            const PairCoord pn = pair_coord(static_cast<int>(Pn), args);
            for (int st = 0; st < 2; ++st) {
              if (2 * pn.pp + st >= args.nqb) continue;
#pragma unroll
              for (int c = 0; c < L::kChunks; ++c)
                tma_prefetch_4d(&tm_q, c * 64, (2 * pn.pp + st) * kTile, pn.h, pn.b);
            }
          }
        }
        Walk wk{args.nkb, 2 * pc.pp + 1 < args.nqb, 0, 0, false, false, false};
        Walk wv = wk;  // the V items follow the K items one entry behind
        const int n[2] = {2 * args.nkb, wk.two ? 2 * args.nkb : 0};
        const int npv[2] = {args.nkb, wk.two ? args.nkb : 0};
        int ns[2] = {0, 0}, nv[2] = {0, 0};  // score and PV items per stream so far
        auto flags = [&](const Walk& w, int (&cnt)[2], const int (&tot)[2], uint32_t f) {
          const bool in[2] = {w.in0, w.in1};
          for (int st = 0; st < 2; ++st) {
            if (!in[st]) continue;
            f |= kItemUse << st;
            if (cnt[st] == 0) f |= kItemFirst << st;
            if (++cnt[st] == tot[st]) f |= kItemLast << st;
          }
          return f;
        };
        // ring order: the pair's Q tiles, the K of the first entry, then per entry u:
        // V(u) (if it has PV MMAs) and K(u + 1)
        load_q(0, pc);
        if (ok && wk.two) load_q(1, pc);
        bool kmore = ok && wk.next();
        if (kmore) load(&tm_k, wk.kb, pc, flags(wk, ns, n, 0u));
        while (ok && wv.next()) {
          if (wv.pv) load(&tm_v, wv.kb, pc, flags(wv, nv, npv, kItemV));
          if (ok && kmore && (kmore = wk.next())) load(&tm_k, wk.kb, pc, flags(wk, ns, n, 0u));
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
   } else if (warp == kIssuerWarp || warp == kIssuerWarp1) {
    // ================================================================ MMA issue
    // Issuer st (warp 8: stream 0, warp 10: stream 1) follows the ring items in
    // order, taking a V item together with the K item after it (an entry n).  When
    // its stream uses the entry it issues the group [PV of the stream's block on V,
    // S of its next block on K].  The groups take turns: stream 0's group of entry
    // n goes after stream 1's of entry n - 1, stream 1's after stream 0's of entry
    // n (turn barriers), so each stream's softmax overlaps the other's MMAs; the
    // issuer that is not issuing meanwhile takes its next items and releases its
    // slots.  Each issuer releases every slot once (empty counts two arrivals).
    if (lane == 0) {
      const int st = warp == kIssuerWarp ? 0 : 1;
      StreamBars& bs = bars_sh[st];
      constexpr uint32_t idesc_s = idesc_bf16_f32(kTile, kTile, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kTile, D, 1);
      constexpr uint32_t kBufStep = L::kTileBytes >> 4;  // descriptor units per slot
      const uint64_t dq = smem_desc_sw128(sQ(st), 16, 1024);
      const uint64_t dk = smem_desc_sw128(sSlot(0), 16, 1024);
      const uint64_t dv = smem_desc_sw128(sSlot(0), L::kChunkBytes, 1024);
      const uint32_t s_col = tmem + 256u * st;
      int items = 0;
      int J = 0, k = 0;  // p_full waits (one per block), tiles (q_full / q_free phases)
      bool pp = false;   // a block's P not waited for yet (no PV since its S)
      bool ok = true, end = false;
      auto next_item = [&](uint32_t& meta) -> int {
        const int i = items % NS;
        ok = ok && mbar_wait(&sb.full[i], (items / NS) & 1, abort_flag, dev_status, 0x2, kWaitNs);
        ++items;
        meta = ok ? item_meta_sh[i] : kItemEnd;
        return i;
      };
      for (int n = 0; ok && !end; ++n) {
        uint32_t m1, m2 = 0;
        const int i1 = next_item(m1);
        if (!ok || (m1 & kItemEnd)) break;
        int iv = -1, ik = i1;
        uint32_t vm = 0, km = m1;
        if (m1 & kItemV) {
          // a V item is followed by the K of the next entry (or the end)
          iv = i1;
          vm = m1;
          ik = next_item(m2);
          km = m2;
          if (!ok) break;
          if (m2 & kItemEnd) {
            end = true;
            ik = -1;
            km = 0;
          }
        }
        vm >>= st;
        km >>= st;
        const bool use_v = vm & kItemUse, use_k = km & kItemUse;
        if (use_v || (use_k && pp)) {
          if (!mbar_wait(&bs.p_full, J & 1, abort_flag, dev_status, 0x2, kWaitNs)) break;
          ++J;
          pp = false;
        }
        if (use_k && (km & kItemFirst) &&
            !mbar_wait(&bs.q_full, k & 1, abort_flag, dev_status, 0x2, kWaitNs))
          break;
        // this stream's turn: after the other stream's group of the previous entry
        // (stream 0) or of this entry (stream 1)
        if (st == 1 || n > 0) {
          const int tn = st == 1 ? n : n - 1;
          if (!mbar_wait(&sb.turn[st ^ 1], tn & 1, abort_flag, dev_status, 0x2, kWaitNs)) break;
        }
        if (use_v || use_k) {
          tc_fence_after();
          if (use_v) {
            const uint64_t dvs = dv + static_cast<uint64_t>(iv * kBufStep);
            const uint32_t acc0 = (vm & kItemFirst) ? 0u : 1u;
#pragma unroll
            for (int kk = 0; kk < kTile / 16; ++kk)
              mma_ts(s_col + 128, s_col + kk * 8, dvs + static_cast<uint64_t>(kk * (2048 >> 4)),
                     idesc_pv, kk > 0 ? 1u : acc0);
            if (vm & kItemLast) mma_commit(&bs.o_done);
          }
          if (use_k) {
            const uint64_t dks = dk + static_cast<uint64_t>(ik * kBufStep);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = ((kk >> 2) * L::kChunkBytes + (kk & 3) * 32) >> 4;
              mma_ss(s_col, dq + off, dks + off, idesc_s, kk > 0 ? 1u : 0u);
            }
            if (km & kItemLast) {
              mma_commit(&bs.q_free);
              ++k;
            }
            mma_commit(&bs.s_full);
            pp = true;
          }
        }
        mbar_arrive(&sb.turn[st]);
        if (iv >= 0) mma_commit(&sb.empty[iv]);
        if (ik >= 0) mma_commit(&sb.empty[ik]);
      }
    }
    if (lane == 0) {
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

    const int nkb = args.nkb, p_lkv = args.Lkv, p_lq = args.Lq;
    while (good) {
      // next pair from the queue; this stream runs its query block 2 pp + s
      const int q = e % kTq;
      if (!warp_wait(&sb.tq_full[q], (e / kTq) & 1, abort_flag, dev_status)) break;
      const int P = tq_pair_sh[q];
      mbar_arrive(&sb.tq_empty[q]);
      ++e;
      if (P < 0) break;
      const PairCoord pc = pair_coord(P, args);
      const int qb = 2 * pc.pp + s;
      if (qb >= args.nqb) continue;  // the pair's second query block does not exist
      const int n = 2 * nkb;         // two sweeps over the prefix
      const int grow = qb * kTile + row;
      float m_run = -INFINITY;  // reference of the row (log2 units)
      float l_run = 0.f;

      for (int j = 0; j < n; ++j, ++J) {
        const int kb = j < nkb ? j : j - nkb;
        const bool sweep_a = j < nkb;  // the log-sum-exp sweep, no P
        if (!warp_wait(&bs.s_full, J & 1, abort_flag, dev_status)) {
          good = false;
          break;
        }
        tc_fence_after();
        // the columns past the prefix end (the same for every row): -inf in TMEM with
        // whole-warp stores before the scores are read
        if (__builtin_expect((kb + 1) * kTile > p_lkv, 0)) {
          const int valid = p_lkv - kb * kTile;
          const uint32_t ninf = __float_as_uint(-INFINITY);
          const int v8 = (valid + 7) & ~7;
          for (int col = valid; col < v8; ++col) tmem_st1(s_addr + col, ninf);
          for (int col = v8; col < kTile; col += 8) tmem_st8_fill(s_addr + col, ninf);
          tmem_wait_st();
        }
        // the block's 128 scores of this row, in registers for the whole block
        uint32_t sr[kTile];
        tmem_ld128_wait(s_addr, sr);
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
          // first sweep: the row's running log-sum-exp, reference max(m, bm),
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
        // second sweep: P = 2^(s * scale - lse) in packed pairs, already normalised,
        // written over TMEM columns [8cc, 8cc + 8) of the scores (in registers) as
        // packed bf16
        const uint64_t sc2 = f2_pack(csc, csc);
        uint64_t acc0 = 0, acc1 = 0;  // (0.f, 0.f)
        {
          const float neg = (m_run == -INFINITY) ? 0.f : -m_run;
          const uint64_t neg2 = f2_pack(neg, neg);
#pragma unroll
          for (int cc = 0; cc < kTile / 16; ++cc) {
            uint32_t pk[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const float x0 = __uint_as_float(sr[cc * 16 + 2 * c]);
              const float x1 = __uint_as_float(sr[cc * 16 + 2 * c + 1]);
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
        }
        {
          float a0, a1;
          f2_unpack(f2_add(acc0, acc1), a0, a1);
          // the block's share of the attention weights, summed over the tile's valid rows
          float part = grow < p_lq ? a0 + a1 : 0.f;
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
          if (lane == 0) atomicAdd(&mass_sh[s][kb], part);
          if (j + 1 == n) mbar_arrive(&bs.mass_done);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bs.p_full);
      }
      if (!good) break;

      // ---- epilogue of the tile: P was normalised, so O is the output
      if (!warp_wait(&bs.o_done, k & 1, abort_flag, dev_status)) break;
      tc_fence_after();
      uint32_t pk[D / 2];
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t ro[32];
        tmem_ld32_wait(o_addr + cc * 32, ro);
#pragma unroll
        for (int c = 0; c < 16; ++c)
          pk[cc * 16 + c] = pack_bf16x2(__uint_as_float(ro[2 * c]), __uint_as_float(ro[2 * c + 1]));
      }
      // warp 0 of the stream: pooled mass and selection once every warp's sums are in
      if (quad == 0) {
        if (!warp_wait(&bs.mass_done, k & 1, abort_flag, dev_status)) break;
        const int64_t rowid = (static_cast<int64_t>(pc.b) * args.H + pc.h) * args.nqb + qb;
        select_blocks_warp(mass_sh[s], kept_sh[s], nkb, min(kTile, p_lq - qb * kTile), args.topk,
                           args.mass_threshold,
                           args.mass_out ? args.mass_out + rowid * nkb : nullptr,
                           args.sel_idx + rowid * nkb, args.sel_cnt + rowid);
      }
      ++k;
      // each 64-column chunk of the warp's 32 rows into the warp's stage, in the output
      // map's 128B-swizzled layout (16-byte unit u of row r at position u ^ (r mod 8)),
      // then one TMA store of 64 columns x 32 rows
      const int row0 = qb * kTile + quad * kOutBoxRows;  // the warp's first row
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
            tma_store_4d(&tm_o, stage_addr, ch * 64, row0, pc.h, pc.b);
            bulk_commit_group();
            store_pending = true;
          }
        }
      }
      if (args.lse && grow < p_lq) {
        args.lse[(static_cast<int64_t>(pc.b) * args.H + pc.h) * p_lq + grow] =
            m_run * 0.6931471805599453f;  // the row's log-sum-exp (log2 units before)
      }
    }
    if (lane == 0 && store_pending) bulk_wait_all();  // output stores complete before exit
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kIssuerWarp) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace dec
}  // namespace sparvar
