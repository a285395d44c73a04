// CS4A decision on sm_100a: the pooled softmax mass of dense attention per
// (query block, KV block) and the selection of the kept KV blocks ("SparVAR",
// ai.info summary, "Methodology in Plain English", CS4A paragraph: full attention
// at the decision scale, attention weights summed per block, the most important
// blocks kept).  tcgen05 MMAs with TMEM accumulators, TMA staging of Q and K,
// warp-specialised roles.
//
// One CTA owns one 128-row query tile of one (batch, head):
//   warps 0-3  softmax: thread t owns query row t of the tile and TMEM lane t
//   warp  4    MMA issue (one elected lane) + TMEM allocation
//   warp  5    TMA producer (one elected lane)
// TMEM: two score buffers S0 [0,128), S1 [128,256).
//
// Sweeps over every KV block kb of the prefix, S_kb = Q K_kb^T in buffer kb % 2:
//   without a given LSE, a first sweep forms each row's log-sum-exp online;
//   the last sweep adds exp(s - lse) over the block's keys, reduced over the
//   tile's rows into a per-block sum in shared memory.
// Warp 0 then divides by the tile's query count (the pooled mass) and selects.
#pragma once

#include <cuda_bf16.h>
#include <cuda.h>

#include "ptx.cuh"
#include "select.cuh"
#include "tmem_io.cuh"

namespace sparvar {

constexpr int kTile = 128;
constexpr int kThreads = 192;
constexpr int kMmaWarp = 4;
constexpr int kLoadWarp = 5;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128;
constexpr uint64_t kWaitNs = 1000000000ull;   // 1 s per wait
constexpr uint64_t kDrainNs = 500000000ull;   // 0.5 s per drain
constexpr int kMaxMassBlocks = 4096;

struct DecideArgs {
  int B, H, Lq, Lkv, nqb, nkb;
  float scale_log2;  // softmax_scale * log2(e)
  const float* lse_in;  // [B][H][Lq] natural log, or null -> computed in a first sweep
  float mass_threshold;
  int topk;          // > 0: keep exactly this many blocks per query block (Top-K mode)
  int32_t* sel_cnt;  // [B][H][nqb]
  int32_t* sel_idx;  // [B][H][nqb][nkb]
  float* mass_out;   // [B][H][nqb][nkb] or null
  int32_t* dev_status;
};

struct __align__(8) Barriers {
  uint64_t q_full;
  uint64_t k_full[2], k_empty[2];
  uint64_t s_full[2], s_free[2];
  uint64_t drain;
};

template <int D>
struct Smem {
  static constexpr uint32_t kTileBytes = kTile * D * 2;  // 128 rows x D bf16
  static constexpr uint32_t kChunkBytes = kTile * 128;   // 128 rows x 64 cols
  static constexpr uint32_t kChunks = D / 64;
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kK0 = kTileBytes;
  static constexpr uint32_t kMassBytes = 3 * kTileBytes + kMaxMassBlocks * 4 + kMaxMassBlocks;
  // Every CTA allocates all 512 TMEM columns, so at most one may live on an SM:
  // asking for more than half of the SM's shared memory guarantees that.
  static constexpr uint32_t kMinBytes = 116 * 1024;
  static constexpr uint32_t dyn_bytes() {
    return (kMassBytes > kMinBytes ? kMassBytes : kMinBytes) + 1024;
  }
};

// Warp-uniform wait for the softmax warps: their tcgen05.ld/st are warp-collective,
// so every lane must take the same branch even when a wait gives up.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          int32_t* dev_status) {
  const bool ok = mbar_wait(bar, parity, abort, dev_status, 0x2, kWaitNs);
  return __all_sync(0xffffffffu, ok);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    decide_blocks_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ DecideArgs args) {
  using L = Smem<D>;
  extern __shared__ uint8_t smem_raw[];
  __shared__ Barriers bars;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  const uint32_t smem_base = (smem_addr(smem_raw) + 1023u) & ~1023u;
  uint8_t* smem_gen = smem_raw + (smem_base - smem_addr(smem_raw));
  const int warp = warp_id();
  const int lane = lane_id();
  const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  volatile int* abort_flag = &abort_sh;
  int32_t* dev_status = args.dev_status;

  // every KV block of the prefix, once per sweep
  const int sweeps = args.lse_in ? 1 : 2;
  const int n_blocks = args.nkb * sweeps;

  if (threadIdx.x == 0) {
    abort_sh = 0;
    mbar_init(&bars.q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars.k_full[s], 1);
      mbar_init(&bars.k_empty[s], 1);
      mbar_init(&bars.s_full[s], 1);
      mbar_init(&bars.s_free[s], 128);
    }
    mbar_init(&bars.drain, 1);
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&tmem_base_sh, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kLoadWarp && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  const uint32_t sQ = smem_base + L::kQ;
  auto sK = [&](int s) { return smem_base + L::kK0 + s * L::kTileBytes; };

  if (warp == kLoadWarp) {
    // ================================================================ producer
    if (lane == 0 && n_blocks > 0) {
      int issued_k[2] = {0, 0};
      mbar_arrive_expect_tx(&bars.q_full, L::kTileBytes);
#pragma unroll
      for (int c = 0; c < (int)L::kChunks; ++c)
        tma_load_4d(sQ + c * L::kChunkBytes, &tm_q, &bars.q_full, c * 64, qb * kTile, h, b);
      for (int j = 0; j < n_blocks; ++j) {
        const int s = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        const int kb = j % args.nkb;
        if (!mbar_wait(&bars.k_empty[s], ph ^ 1, abort_flag, dev_status, 0x2, kWaitNs)) break;
        mbar_arrive_expect_tx(&bars.k_full[s], L::kTileBytes);
#pragma unroll
        for (int c = 0; c < (int)L::kChunks; ++c)
          tma_load_4d(sK(s) + c * L::kChunkBytes, &tm_k, &bars.k_full[s], c * 64, kb * kTile, h, b);
        ++issued_k[s];
      }
      // Drain: every TMA write into shared memory lands before the CTA exits.
      mbar_drain(&bars.q_full, 0, kDrainNs);
      for (int s = 0; s < 2; ++s)
        if (issued_k[s]) mbar_drain(&bars.k_full[s], (issued_k[s] - 1) & 1, kDrainNs);
    }
  } else if (warp == kMmaWarp) {
    // ================================================================ MMA issue
    if (lane == 0 && n_blocks > 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(kTile, kTile, 0);
      bool ok = mbar_wait(&bars.q_full, 0, abort_flag, dev_status, 0x2, kWaitNs);
      for (int j = 0; ok && j < n_blocks; ++j) {
        const int s = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (!mbar_wait(&bars.k_full[s], ph, abort_flag, dev_status, 0x2, kWaitNs)) break;
        // S buffer s is free once the softmax warps have read S_{j-2}
        if (j >= 2 &&
            !mbar_wait(&bars.s_free[s], ((j - 2) >> 1) & 1, abort_flag, dev_status, 0x2, kWaitNs))
          break;
        tc_fence_after();
        const uint32_t d_col = tmem + (s ? kColS1 : kColS0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * L::kChunkBytes + (kk & 3) * 32;
          const uint64_t adesc = smem_desc_sw128(sQ + off, 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(sK(s) + off, 16, 1024);
          mma_ss(d_col, adesc, bdesc, idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bars.s_full[s]);
        mma_commit(&bars.k_empty[s]);
      }
      // Drain: no MMA may still read shared memory or TMEM when the CTA exits.
      mma_commit(&bars.drain);
      mbar_drain(&bars.drain, 0, kDrainNs);
    }
    __syncwarp();
  } else {
    // ================================================================ softmax
    const int row = warp * 32 + lane;  // tile row == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const int grow = qb * kTile + row;
    const float c = args.scale_log2;
    float m_run = -INFINITY;  // log2-domain running max of the first sweep
    float l_sum = 0.f;
    bool good = true;

    float* mass_sh = reinterpret_cast<float*>(smem_gen + 3 * L::kTileBytes);
    uint8_t* kept_sh = reinterpret_cast<uint8_t*>(mass_sh + kMaxMassBlocks);
    for (int i = threadIdx.x; i < args.nkb; i += 128) {
      mass_sh[i] = 0.f;
      kept_sh[i] = 0;
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    float lse2 = 0.f;  // the row's log-sum-exp, log2 units
    if (args.lse_in && grow < args.Lq)
      lse2 = args.lse_in[(static_cast<int64_t>(b) * args.H + h) * args.Lq + grow] *
             1.4426950408889634f;

    for (int j = 0; j < n_blocks; ++j) {
      const int s = j & 1;
      const uint32_t ph = (j >> 1) & 1;
      const int kb = j % args.nkb;
      if (!warp_wait(&bars.s_full[s], ph, abort_flag, dev_status)) { good = false; break; }
      tc_fence_after();
      const uint32_t s_addr = tmem + lane_off + (s ? kColS1 : kColS0);
      float x[kTile];
      {
        uint32_t r[32];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          tmem_ld32_wait(s_addr + cc * 32, r);
#pragma unroll
          for (int i = 0; i < 32; ++i) x[cc * 32 + i] = __uint_as_float(r[i]) * c;
        }
      }
      // S has been read into registers: release the buffer
      tc_fence_before();
      mbar_arrive(&bars.s_free[s]);
      // keys past the prefix in a ragged last block
      const int valid = (kb + 1) * kTile > args.Lkv ? args.Lkv - kb * kTile : kTile;
      if (valid < kTile) {
#pragma unroll
        for (int i = 0; i < kTile; ++i)
          if (i >= valid) x[i] = -INFINITY;
      }
      if (j < n_blocks - args.nkb) {
        // sweep 0 (no lse given): online log-sum-exp of the row
        float mx = -INFINITY;
#pragma unroll
        for (int i = 0; i < kTile; ++i) mx = fmaxf(mx, x[i]);
        const float m_new = fmaxf(m_run, mx);
        const float mref = (m_new == -INFINITY) ? 0.f : m_new;
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < kTile; ++i) acc += ex2_approx(x[i] - mref);
        l_sum = l_sum * ex2_approx(((m_run == -INFINITY) ? mref : m_run) - mref) + acc;
        m_run = m_new;
        if (j == n_blocks - args.nkb - 1) lse2 = m_run + __log2f(l_sum);
      } else {
        float acc = 0.f;
        if (grow < args.Lq) {
#pragma unroll
          for (int i = 0; i < kTile; ++i) acc += ex2_approx(x[i] - lse2);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) atomicAdd(&mass_sh[kb], acc);
      }
    }

    // ---- CS4A selection for this query block (warp 0 of the softmax group)
    asm volatile("bar.sync 1, 128;" ::: "memory");
    const int aborted = __shfl_sync(0xffffffffu, *abort_flag, 0);
    if (warp == 0 && !aborted && good) {
      const int64_t rowid = (static_cast<int64_t>(b) * args.H + h) * args.nqb + qb;
      select_blocks_warp(mass_sh, kept_sh, args.nkb, min(kTile, args.Lq - qb * kTile), args.topk,
                         args.mass_threshold,
                         args.mass_out ? args.mass_out + rowid * args.nkb : nullptr,
                         args.sel_idx + rowid * args.nkb, args.sel_cnt + rowid);
    }
  }

  // ---- teardown: every role has left its loop and drained its async work
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace sparvar
