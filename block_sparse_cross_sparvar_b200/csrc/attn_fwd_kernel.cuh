// Block-sparse attention forward on sm_100a.
//
// One CTA owns one 128-row query tile (one query block of one batch item and
// head) and walks that tile's list of KV blocks j = 0 .. n-1.  Roles:
//   warps 0-3   softmax group 0: blocks j = 0, 2, 4, ... (thread t: query row t,
//               TMEM lane t)
//   warps 4-7   softmax group 1: blocks j = 1, 3, 5, ...
//   warp  8     MMA issue for even blocks (one lane) and TMEM owner
//   warp  9     TMA producer (one lane)
//   warp  10    MMA issue for odd blocks (one lane)
// TMEM (512 columns): three score buffers S_b = [128b, 128b+128), b = j mod 3,
// and the output accumulator O = [384, 384+D).  P_j is written as packed bf16
// over the first 64 columns of its score buffer and feeds the PV MMA from TMEM.
// The MMA warp keeps three score blocks in flight (S_{j+3} is issued right
// after PV_j, which frees buffer j mod 3), so a softmax group finds its next S
// already computed and the tensor core never waits for a softmax round trip.
// Q is loaded once; K and V blocks pass through a ring of shared-memory slots
// in the order the MMA warp needs them: K_0, K_1, K_2, then V_j, K_{j+3}.  The
// MMA warp issues PV_j and S_{j+3} as one group and frees both slots with one
// commit.
//
// Both groups add into the one O accumulator, so they share a per-row
// reference max m (log2 units) in shared memory.  Block j is computed against
// the reference read when it starts and finalised in block order: its group
// waits until block j-1 has been handed to the MMA warp, re-reads m, and either
// raises m (when the block's max exceeds m by more than 2^8: O is rescaled in
// place once PV_{j-1} has completed, i.e. once group j-1 has released its slots)
// or, if m moved meanwhile, rescales its own
// P in TMEM.  Each group keeps its row sum relative to its own last reference;
// the epilogue combines the two sums against the final m.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx.cuh"
#include "tmem_io.cuh"

namespace sparvar {
namespace fwd {

constexpr int kTile = 128;
constexpr int kThreads = 352;
constexpr int kMmaWarp = 8;    // MMA issuer 0 (even blocks) and TMEM owner
constexpr int kLoadWarp = 9;
constexpr int kMmaWarp1 = 10;  // MMA issuer 1 (odd blocks), on another SM sub-partition
constexpr uint32_t kTmemCols = 512;
constexpr float kLazyRescale = 8.0f;          // log2 units
constexpr uint64_t kWaitNs = 1000000000ull;   // 1 s per wait
constexpr uint64_t kDrainNs = 500000000ull;   // 0.5 s per drain
constexpr int kMaxSlots = 12;

struct Args {
  int B, H, Lq, Lkv, nqb, nkb;
  float scale_log2;  // softmax_scale * log2(e)
  const int32_t* kv_cnt;
  const int32_t* kv_idx;
  int64_t list_sb, list_sh;
  int idx_row_len;
  __nv_bfloat16* o;
  int64_t o_sb, o_sh, o_sr;
  float* lse;  // [B][H][Lq] or null
  int32_t* dev_status;
};

struct __align__(8) Bars {
  uint64_t q_full;
  uint64_t full[kMaxSlots];       // ring slot loaded (TMA transaction count)
  uint64_t rel[8];                // group j (PV_j and S_{j+3}) done: its ring slots are free
  uint64_t pro_done;              // prologue score groups done: K_0..K_2 slots are free
  uint64_t s_full[3], p_full[3];  // per score buffer
  uint64_t o_done;
  uint64_t drain;
};

// Ring positions: K_0 .. K_{n0-1} (n0 = min(n, 3)), then V_j and, while j + 3 < n,
// K_{j+3}, for j = 0 .. n-1.  The group that consumes position p (or the prologue)
// is what frees its slot.  Group j commits on rel[j % 8]: a slot is reused five
// positions later, so its user is at most ~3 groups ahead of the group that
// freed it and a waiter can never be two phases behind on that barrier.
__device__ __forceinline__ int ring_pos_v(int j, int n) {
  const int n0 = n < 3 ? n : 3;
  const int nk = n > 3 ? n - 3 : 0;
  return n0 + j + (j < nk ? j : nk);
}
// block whose group consumes ring position p >= n0
__device__ __forceinline__ int ring_block(int p, int n) {
  const int n0 = n < 3 ? n : 3;
  const int nk = n > 3 ? n - 3 : 0;
  const int q = p - n0;
  return q < 2 * nk ? (q >> 1) : nk + (q - 2 * nk);
}

template <int D>
struct Layout {
  static constexpr uint32_t kTileBytes = kTile * D * 2;
  static constexpr uint32_t kChunkBytes = kTile * 128;  // 128 rows x 64 bf16
  static constexpr int kChunks = D / 64;
  static constexpr int kSlots = D == 128 ? 6 : 12;
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kRing = kTileBytes;
  static constexpr uint32_t kColO = 384;
  static constexpr uint32_t kBytes = (1 + kSlots) * kTileBytes + 1024;
};

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
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ Args args) {
  using L = Layout<D>;
  constexpr int NS = L::kSlots;
  extern __shared__ uint8_t smem_raw[];
  __shared__ Bars bars;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;
  __shared__ float m_sh[kTile];  // shared reference max per row

  const uint32_t smem_base = (smem_addr(smem_raw) + 1023u) & ~1023u;
  const int warp = warp_id();
  const int lane = lane_id();
  const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  volatile int* abort_flag = &abort_sh;
  int32_t* dev_status = args.dev_status;

  const int64_t lrow = b * args.list_sb + h * args.list_sh + qb;
  int n = __ldg(args.kv_cnt + lrow);
  if (n < 0 || n > args.idx_row_len) {
    if (threadIdx.x == 0 && dev_status) atomicOr(dev_status, 0x1);
    n = n < 0 ? 0 : args.idx_row_len;
  }
  const int32_t* list = args.kv_idx + lrow * args.idx_row_len;

  if (threadIdx.x == 0) {
    abort_sh = 0;
    mbar_init(&bars.q_full, 1);
    for (int i = 0; i < 3; ++i) {
      mbar_init(&bars.s_full[i], 1);
      mbar_init(&bars.p_full[i], 128);
    }
    mbar_init(&bars.o_done, 2);  // one commit per issuer
    for (int s = 0; s < NS; ++s) mbar_init(&bars.full[s], 1);
    for (int i = 0; i < 8; ++i) mbar_init(&bars.rel[i], 1);
    mbar_init(&bars.pro_done, 1);
    mbar_init(&bars.drain, 2);  // one commit per issuer
    fence_barrier_init();
  }
  if (threadIdx.x < kTile) m_sh[threadIdx.x] = -INFINITY;
  if (warp == kMmaWarp) {
    tmem_alloc(&tmem_base_sh, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kLoadWarp && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  const uint32_t sQ = smem_base + L::kQ;
  auto sSlot = [&](int s) { return smem_base + L::kRing + s * L::kTileBytes; };

  if (warp == kLoadWarp) {
    // ================================================================ producer
    if (lane == 0 && n > 0) {
      const int n0 = n < 3 ? n : 3;
      int w = 0;  // ring position
      bool ok = true;
      auto produce = [&](const CUtensorMap* tm, int kb) {
        const int s = w % NS;
        if (w >= NS) {
          // wait until the group that consumed position w - NS has completed
          const int prev = w - NS;
          bool got;
          if (prev < n0) {
            got = mbar_wait(&bars.pro_done, 0, abort_flag, dev_status, 0x2, kWaitNs);
          } else {
            const int jb = ring_block(prev, n);
            got = mbar_wait(&bars.rel[jb & 7], (jb >> 3) & 1, abort_flag, dev_status, 0x2, kWaitNs);
          }
          if (!got) {
            ok = false;
            return;
          }
        }
        kb = kb < 0 ? -1 : (kb > args.nkb ? args.nkb : kb);
        mbar_arrive_expect_tx(&bars.full[s], L::kTileBytes);
#pragma unroll
        for (int c = 0; c < L::kChunks; ++c)
          tma_load_4d(sSlot(s) + c * L::kChunkBytes, tm, &bars.full[s], c * 64, kb * kTile, h, b);
        ++w;
      };
      mbar_arrive_expect_tx(&bars.q_full, L::kTileBytes);
#pragma unroll
      for (int c = 0; c < L::kChunks; ++c)
        tma_load_4d(sQ + c * L::kChunkBytes, &tm_q, &bars.q_full, c * 64, qb * kTile, h, b);
      for (int j = 0; j < n0 && ok; ++j) produce(&tm_k, __ldg(list + j));
      for (int j = 0; j < n && ok; ++j) {
        produce(&tm_v, __ldg(list + j));
        if (ok && j + 3 < n) produce(&tm_k, __ldg(list + j + 3));
      }
      // drain: every issued TMA write lands before the CTA exits
      mbar_drain(&bars.q_full, 0, kDrainNs);
      for (int s = 0; s < NS; ++s) {
        const int issued = w > s ? (w - 1 - s) / NS + 1 : 0;  // loads that used slot s
        if (issued) mbar_drain(&bars.full[s], (issued - 1) & 1, kDrainNs);
      }
    }
  } else if (warp == kMmaWarp || warp == kMmaWarp1) {
    // ================================================================ MMA issue
    // The tensor core queues only a few MMAs ahead of the one it executes, so
    // a single issuing thread loses tensor time whenever it waits on a barrier
    // or commits.  Two issuers on different SM sub-partitions therefore take
    // alternate blocks: issuer i runs group j (PV_j, then S_{j+3} into the
    // buffer PV_j has just read) for j = i, i + 2, ...; while one waits, the
    // other keeps the queue filled.  O is zeroed before the first PV, so the
    // two issuers' PV MMAs may accumulate in either order.  Each group's
    // commit frees both of its ring slots.
    const int me = warp == kMmaWarp ? 0 : 1;
    if (lane == 0 && n > 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(kTile, kTile, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kTile, D, 1);
      constexpr uint32_t kSlotStep = L::kTileBytes >> 4;  // descriptor units per slot
      const uint64_t dq = smem_desc_sw128(sQ, 16, 1024);
      const uint64_t dk = smem_desc_sw128(sSlot(0), 16, 1024);
      const uint64_t dv = smem_desc_sw128(sSlot(0), L::kChunkBytes, 1024);
      const int n0 = n < 3 ? n : 3;
      bool ok = true;
      auto wait_pos = [&](int pos) {
        ok = ok && mbar_wait(&bars.full[pos % NS], (pos / NS) & 1, abort_flag, dev_status, 0x2, kWaitNs);
      };
      auto mma_s = [&](int jj, int kslot, int kk) {
        const uint32_t off = ((kk >> 2) * L::kChunkBytes + (kk & 3) * 32) >> 4;
        mma_ss(tmem + (jj % 3) * 128, dq + off, dk + static_cast<uint64_t>(kslot * kSlotStep) + off,
               idesc_s, kk > 0 ? 1u : 0u);
      };
      if (me == 0) {
        // prologue: S_0 .. S_{n0-1}
        ok = mbar_wait(&bars.q_full, 0, abort_flag, dev_status, 0x2, kWaitNs);
        for (int jj = 0; jj < n0 && ok; ++jj) {
          wait_pos(jj);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) mma_s(jj, jj % NS, kk);
          mma_commit(&bars.s_full[jj]);
        }
        mma_commit(&bars.pro_done);
      }
      // (issuer 1 needs no prologue wait: P_1 exists only after S_1 and Q were used)
      for (int j = me; j < n && ok; j += 2) {
        ok = mbar_wait(&bars.p_full[j % 3], (j / 3) & 1, abort_flag, dev_status, 0x2, kWaitNs);
        const int pv = ring_pos_v(j, n);
        const bool more = j + 3 < n;
        wait_pos(pv);
        if (more) wait_pos(pv + 1);
        if (!ok) break;
        const uint64_t dvs = dv + static_cast<uint64_t>((pv % NS) * kSlotStep);
        const uint32_t a_col = tmem + (j % 3) * 128;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          mma_ts(tmem + L::kColO, a_col + kk * 8, dvs + static_cast<uint64_t>(kk * (2048 >> 4)),
                 idesc_pv, 1u);
        if (more) {
          // buffer j mod 3 is free once PV_j has read P_j (one issuer's MMAs run in order)
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) mma_s(j + 3, (pv + 1) % NS, kk);
          mma_commit(&bars.s_full[j % 3]);
        }
        mma_commit(&bars.rel[j & 7]);
      }
      mma_commit(&bars.o_done);
      mma_commit(&bars.drain);
      mbar_drain(&bars.drain, 0, kDrainNs);
    }
    __syncwarp();
  } else {
    // ================================================================ softmax
    const int g = warp >> 2;  // group: blocks j = g, g + 2, ...
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t o_addr = tmem + lane_off + L::kColO;
    const int grow = qb * kTile + row;
    const float c = args.scale_log2;
    float m_own = -INFINITY;  // reference of this group's l_sum
    float l0 = 0.f, l1 = 0.f;
    bool good = true;

    for (int j = g; j < n && good; j += 2) {
      const int kb = __ldg(list + j);
      const int buf = j % 3;
      const uint32_t s_addr = tmem + lane_off + buf * 128;
      if (!warp_wait(&bars.s_full[buf], (j / 3) & 1, abort_flag, dev_status)) { good = false; break; }
      tc_fence_after();
      float x[kTile];
      {
        uint32_t sr[kTile];
        tmem_ld128_wait(s_addr, sr);
#pragma unroll
        for (int k = 0; k < kTile; ++k) x[k] = __uint_as_float(sr[k]);
      }
      int valid = kTile;
      if (kb < 0 || kb >= args.nkb) {
        valid = 0;
        if (row == 0 && dev_status) atomicOr(dev_status, 0x1);
      } else if ((kb + 1) * kTile > args.Lkv) {
        valid = args.Lkv - kb * kTile;
      }
      if (valid < kTile) {
#pragma unroll
        for (int k = 0; k < kTile; ++k)
          if (k >= valid) x[k] = -INFINITY;
      }
      float mx0 = fmaxf(x[0], x[4]), mx1 = fmaxf(x[1], x[5]);
      float mx2 = fmaxf(x[2], x[6]), mx3 = fmaxf(x[3], x[7]);
#pragma unroll
      for (int k = 8; k < kTile; k += 8) {
        mx0 = max3(mx0, x[k], x[k + 4]);
        mx1 = max3(mx1, x[k + 1], x[k + 5]);
        mx2 = max3(mx2, x[k + 2], x[k + 6]);
        mx3 = max3(mx3, x[k + 3], x[k + 7]);
      }
      const float bm = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3)) * c;  // block row max
      // provisional reference: the shared one, raised to bm if bm is far above it
      const float m_cur = m_sh[row];
      const float m_use = (m_cur == -INFINITY || bm > m_cur + kLazyRescale) ? bm : m_cur;
      const float neg = (m_use == -INFINITY) ? 0.f : -m_use;
      float lb0 = 0.f, lb1 = 0.f;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t pk[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const float p0 = ex2_approx(fmaf(x[cc * 32 + 2 * k], c, neg));
          const float p1 = ex2_approx(fmaf(x[cc * 32 + 2 * k + 1], c, neg));
          lb0 += p0;
          lb1 += p1;
          pk[k] = pack_bf16x2(p0, p1);
        }
        tmem_st16(s_addr + cc * 16, pk);
      }
      float lb = lb0 + lb1;

      // ---- finalise block j in block order
      if (j > 0) {
        const int pj = j - 1;
        if (!warp_wait(&bars.p_full[pj % 3], (pj / 3) & 1, abort_flag, dev_status)) { good = false; break; }
      }
      const float m_fin = m_sh[row];
      const bool raise = m_fin == -INFINITY ? (bm != -INFINITY) : (bm > m_fin + kLazyRescale);
      const float m_blk = raise ? bm : m_fin;  // reference of block j from now on
      // O holds non-zero values only once some earlier block had a finite reference
      const bool o_live = raise && m_fin != -INFINITY;
      if (__any_sync(0xffffffffu, o_live)) {
        // PV_{j-1} must have completed before O is rewritten
        // every earlier PV is complete once groups j-1 and j-2 (the latest of each
        // issuer) have released their ring slots
        const int pj = j - 1;
        if (!warp_wait(&bars.rel[pj & 7], (pj >> 3) & 1, abort_flag, dev_status)) { good = false; break; }
        if (pj >= 1 &&
            !warp_wait(&bars.rel[(pj - 1) & 7], ((pj - 1) >> 3) & 1, abort_flag, dev_status)) {
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
      if (__any_sync(0xffffffffu, fix_p)) {
        // the shared reference moved while P_j was computed: rescale P_j to m_blk
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
        const float f = (m_own == -INFINITY) ? 0.f : ex2_approx(m_own - m_blk);
        l0 *= f;
        l1 *= f;
        m_own = m_blk;
      }
      l0 += lb;
      if (j == 0) {
        // O starts at zero: PV MMAs of the two issuers accumulate in either order
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

    // ---- epilogue: both groups' sums against the final reference.  Once o_done
    // has fired every MMA has finished and every TMA load has landed, so the
    // first ring slot is free for the exchange.
    if (good && n > 0) good = warp_wait(&bars.o_done, 0, abort_flag, dev_status);
    float* merge_m = reinterpret_cast<float*>(smem_raw + (smem_base - smem_addr(smem_raw)) + L::kRing);
    float* merge_l = merge_m + 2 * kTile;
    merge_m[g * kTile + row] = m_own;
    merge_l[g * kTile + row] = l0 + l1;
    tc_fence_before();
    asm volatile("bar.sync 1, 256;" ::: "memory");
    tc_fence_after();
    const int aborted = __shfl_sync(0xffffffffu, *abort_flag, 0);
    if (!aborted) {
      const float m = m_sh[row];
      const float ma = merge_m[row], mb = merge_m[kTile + row];
      const float sa = (ma == -INFINITY) ? 0.f : ex2_approx(ma - m);
      const float sb = (mb == -INFINITY) ? 0.f : ex2_approx(mb - m);
      const float l = merge_l[row] * sa + merge_l[kTile + row] * sb;
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* orow = args.o + b * args.o_sb + h * args.o_sh + grow * args.o_sr;
      // group 0 writes columns [0, D/2), group 1 writes [D/2, D)
#pragma unroll
      for (int cc = 0; cc < D / 64; ++cc) {
        const int col = g * (D / 2) + cc * 32;
        uint32_t ro[32];
        if (n > 0) {
          tmem_ld32_wait(o_addr + col, ro);
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) ro[k] = 0u;
        }
        uint32_t pk[16];
#pragma unroll
        for (int k = 0; k < 16; ++k)
          pk[k] = pack_bf16x2(__uint_as_float(ro[2 * k]) * inv_l,
                              __uint_as_float(ro[2 * k + 1]) * inv_l);
        if (grow < args.Lq) {
          uint4* dst = reinterpret_cast<uint4*>(orow + col);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
      }
      if (g == 0 && args.lse && grow < args.Lq) {
        args.lse[(static_cast<int64_t>(b) * args.H + h) * args.Lq + grow] =
            l > 0.f ? (m + __log2f(l)) * 0.6931471805599453f : -INFINITY;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace fwd
}  // namespace sparvar
