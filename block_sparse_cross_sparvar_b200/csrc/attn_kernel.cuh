// Block-sparse attention on sm_100a: tcgen05 MMAs with TMEM accumulators, TMA
// staging of the K/V blocks named by a per-query-block list, warp-specialised
// roles.  The same kernel, in "mass" mode, computes the pooled softmax mass of
// dense attention per (query block, KV block) and selects blocks for CS4A.
//
// One CTA owns one 128-row query tile of one (batch, head):
//   warps 0-3  softmax: thread t owns query row t of the tile and TMEM lane t
//   warp  4    MMA issue (one elected lane) + TMEM allocation
//   warp  5    TMA producer (one elected lane)
// TMEM (512 columns): S0 [0,128), S1 [128,256), O [256, 256+D).  P_j is written
// as packed bf16 over the first 64 columns of S_{j%2} and fed to the PV MMA
// straight from TMEM.
//
// Per KV block j of the list:
//   S_j = Q K_j^T                       (SS MMA, M=128 N=128, K=D)
//   row max / lazy rescale / P_j = exp2(S_j*c - m)   (softmax warps)
//   O  += P_j V_j                       (TS MMA, M=128 N=D, K=128)
// S_{j+1} is issued before PV_j so the tensor core runs while the softmax
// warps work.  The running max is only moved (and O rescaled) when it grows by
// more than 2^8, so most blocks need no O round trip through registers.
#pragma once

#include <cuda_bf16.h>
#include <cuda.h>

#include "ptx.cuh"
#include "tmem_io.cuh"

namespace sparvar {

constexpr int kTile = 128;
constexpr int kThreads = 192;
constexpr int kMmaWarp = 4;
constexpr int kLoadWarp = 5;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;
constexpr float kLazyRescale = 8.0f;          // log2 units
constexpr uint64_t kWaitNs = 1000000000ull;   // 1 s per wait
constexpr uint64_t kDrainNs = 500000000ull;   // 0.5 s per drain
constexpr int kMaxMassBlocks = 4096;

enum : int { kModeAttn = 0, kModeMass = 1 };

struct AttnArgs {
  int B, H, Lq, Lkv, nqb, nkb;
  float scale_log2;  // softmax_scale * log2(e)
  // lists (attention mode)
  const int32_t* kv_cnt;
  const int32_t* kv_idx;
  int64_t list_sb, list_sh;
  int idx_row_len;
  // output (attention mode)
  __nv_bfloat16* o;
  int64_t o_sb, o_sh, o_sr;
  float* lse_out;  // [B][H][Lq] or null
  // mass mode
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
  uint64_t v_full[2], v_empty[2];
  uint64_t s_full[2], p_full[2], pv_done[2];
  uint64_t drain;
};

template <int D>
struct Smem {
  static constexpr uint32_t kTileBytes = kTile * D * 2;  // 128 rows x D bf16
  static constexpr uint32_t kChunkBytes = kTile * 128;   // 128 rows x 64 cols
  static constexpr uint32_t kChunks = D / 64;
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kK0 = kTileBytes;
  static constexpr uint32_t kV0 = 3 * kTileBytes;
  static constexpr uint32_t kAttnBytes = 5 * kTileBytes;
  static constexpr uint32_t kMassBytes = 3 * kTileBytes + kMaxMassBlocks * 4 + kMaxMassBlocks;
  // Every CTA allocates all 512 TMEM columns, so at most one may live on an SM:
  // asking for more than half of the SM's shared memory guarantees that.
  static constexpr uint32_t kMinBytes = 116 * 1024;
  static constexpr uint32_t dyn_bytes(int mode) {
    const uint32_t need = mode == kModeAttn ? kAttnBytes : kMassBytes;
    return (need > kMinBytes ? need : kMinBytes) + 1024;
  }
};

// Warp-uniform wait for the softmax warps: their tcgen05.ld/st are warp-collective,
// so every lane must take the same branch even when a wait gives up.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          int32_t* dev_status) {
  const bool ok = mbar_wait(bar, parity, abort, dev_status, 0x2, kWaitNs);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ int clamp_block(int kb, int nkb) {
  // An out-of-range entry is moved fully outside the tensor: TMA then zero-fills
  // it and the softmax masks every key of it.
  return kb < 0 ? -1 : (kb > nkb ? nkb : kb);
}

template <int D, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    block_sparse_attn_kernel(const __grid_constant__ CUtensorMap tm_q,
                             const __grid_constant__ CUtensorMap tm_k,
                             const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ AttnArgs args) {
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

  // ---- list of KV blocks for this query tile
  int n_blocks;
  const int32_t* list = nullptr;
  int sweeps = 1;
  if constexpr (MODE == kModeAttn) {
    const int64_t row = b * args.list_sb + h * args.list_sh + qb;
    int cnt = __ldg(args.kv_cnt + row);
    if (cnt < 0 || cnt > args.idx_row_len) {
      if (threadIdx.x == 0 && dev_status) atomicOr(dev_status, 0x1);
      cnt = cnt < 0 ? 0 : args.idx_row_len;
    }
    n_blocks = cnt;
    list = args.kv_idx + row * args.idx_row_len;
  } else {
    sweeps = args.lse_in ? 1 : 2;
    n_blocks = args.nkb * sweeps;
  }

  if (threadIdx.x == 0) {
    abort_sh = 0;
    mbar_init(&bars.q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars.k_full[s], 1);
      mbar_init(&bars.k_empty[s], 1);
      mbar_init(&bars.v_full[s], 1);
      mbar_init(&bars.v_empty[s], 1);
      mbar_init(&bars.s_full[s], 1);
      mbar_init(&bars.p_full[s], 128);
      mbar_init(&bars.pv_done[s], 1);
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
    if constexpr (MODE == kModeAttn) prefetch_tmap(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  const uint32_t sQ = smem_base + L::kQ;
  auto sK = [&](int s) { return smem_base + L::kK0 + s * L::kTileBytes; };
  auto sV = [&](int s) { return smem_base + L::kV0 + s * L::kTileBytes; };

  auto block_at = [&](int j) -> int {
    if constexpr (MODE == kModeAttn) {
      return __ldg(list + j);
    } else {
      return j % args.nkb;
    }
  };

  if (warp == kLoadWarp) {
    // ================================================================ producer
    if (lane == 0 && n_blocks > 0) {
      int issued_k[2] = {0, 0}, issued_v[2] = {0, 0};
      mbar_arrive_expect_tx(&bars.q_full, L::kTileBytes);
#pragma unroll
      for (int c = 0; c < (int)L::kChunks; ++c)
        tma_load_4d(sQ + c * L::kChunkBytes, &tm_q, &bars.q_full, c * 64, qb * kTile, h, b);
      for (int j = 0; j < n_blocks; ++j) {
        const int s = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        const int kb = clamp_block(block_at(j), args.nkb);
        if (!mbar_wait(&bars.k_empty[s], ph ^ 1, abort_flag, dev_status, 0x2, kWaitNs)) break;
        mbar_arrive_expect_tx(&bars.k_full[s], L::kTileBytes);
#pragma unroll
        for (int c = 0; c < (int)L::kChunks; ++c)
          tma_load_4d(sK(s) + c * L::kChunkBytes, &tm_k, &bars.k_full[s], c * 64, kb * kTile, h, b);
        ++issued_k[s];
        if constexpr (MODE == kModeAttn) {
          if (!mbar_wait(&bars.v_empty[s], ph ^ 1, abort_flag, dev_status, 0x2, kWaitNs)) break;
          mbar_arrive_expect_tx(&bars.v_full[s], L::kTileBytes);
#pragma unroll
          for (int c = 0; c < (int)L::kChunks; ++c)
            tma_load_4d(sV(s) + c * L::kChunkBytes, &tm_v, &bars.v_full[s], c * 64, kb * kTile, h,
                        b);
          ++issued_v[s];
        }
      }
      // Drain: every TMA write into shared memory lands before the CTA exits.
      mbar_drain(&bars.q_full, 0, kDrainNs);
      for (int s = 0; s < 2; ++s) {
        if (issued_k[s]) mbar_drain(&bars.k_full[s], (issued_k[s] - 1) & 1, kDrainNs);
        if (issued_v[s]) mbar_drain(&bars.v_full[s], (issued_v[s] - 1) & 1, kDrainNs);
      }
    }
  } else if (warp == kMmaWarp) {
    // ================================================================ MMA issue
    if (lane == 0 && n_blocks > 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(kTile, kTile, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kTile, D, 1);
      bool ok = mbar_wait(&bars.q_full, 0, abort_flag, dev_status, 0x2, kWaitNs);
      auto issue_pv = [&](int i) -> bool {
        const int s = i & 1;
        const uint32_t ph = (i >> 1) & 1;
        if (!mbar_wait(&bars.p_full[s], ph, abort_flag, dev_status, 0x2, kWaitNs)) return false;
        if (!mbar_wait(&bars.v_full[s], ph, abort_flag, dev_status, 0x2, kWaitNs)) return false;
        tc_fence_after();
        const uint32_t a_col = tmem + (s ? kColS1 : kColS0);
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk) {
          // V tile: keys are the K dimension (128 B rows), D is the N dimension (64-wide chunks).
          const uint64_t bdesc = smem_desc_sw128(sV(s) + kk * 2048, L::kChunkBytes, 1024);
          mma_ts(tmem + kColO, a_col + kk * 8, bdesc, idesc_pv, (i > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&bars.v_empty[s]);
        mma_commit(&bars.pv_done[s]);
        return true;
      };
      for (int j = 0; ok && j < n_blocks; ++j) {
        const int s = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (!mbar_wait(&bars.k_full[s], ph, abort_flag, dev_status, 0x2, kWaitNs)) { ok = false; break; }
        if constexpr (MODE == kModeMass) {
          // S buffer s is free once the softmax warps have read S_{j-2}.
          if (j >= 2 && !mbar_wait(&bars.p_full[s], ((j - 2) >> 1) & 1, abort_flag, dev_status, 0x2,
                                   kWaitNs)) { ok = false; break; }
        }
        // (attention mode: S_j overwrites P_{j-2}, whose PV MMA was issued earlier
        //  by this thread; tcgen05 MMAs from one thread execute in issue order.)
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
        if constexpr (MODE == kModeAttn) {
          if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
        }
      }
      if constexpr (MODE == kModeAttn) {
        if (ok) issue_pv(n_blocks - 1);
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
    float m_ref = -INFINITY;  // log2-domain reference (lazy running max)
    float l_sum = 0.f;
    bool good = true;

    float* mass_sh = nullptr;
    uint8_t* kept_sh = nullptr;
    float lse2 = 0.f;
    if constexpr (MODE == kModeMass) {
      mass_sh = reinterpret_cast<float*>(smem_gen + 3 * L::kTileBytes);
      kept_sh = reinterpret_cast<uint8_t*>(mass_sh + kMaxMassBlocks);
      for (int i = threadIdx.x; i < args.nkb; i += 128) {
        mass_sh[i] = 0.f;
        kept_sh[i] = 0;
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (args.lse_in && grow < args.Lq)
        lse2 = args.lse_in[(static_cast<int64_t>(b) * args.H + h) * args.Lq + grow] *
               1.4426950408889634f;
    }

    for (int j = 0; j < n_blocks; ++j) {
      const int s = j & 1;
      const uint32_t ph = (j >> 1) & 1;
      const int kb_raw = block_at(j);
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
      // keys past the prefix (ragged last block) or of an out-of-range entry
      int valid = kTile;
      if (kb_raw < 0 || kb_raw >= args.nkb) {
        valid = 0;
        if (MODE == kModeAttn && row == 0 && dev_status) atomicOr(dev_status, 0x1);
      } else if ((kb_raw + 1) * kTile > args.Lkv) {
        valid = args.Lkv - kb_raw * kTile;
      }
      if (valid < kTile) {
#pragma unroll
        for (int i = 0; i < kTile; ++i)
          if (i >= valid) x[i] = -INFINITY;
      }
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < kTile; ++i) mx = fmaxf(mx, x[i]);

      if constexpr (MODE == kModeAttn) {
        bool need = (j > 0) && (mx > m_ref + kLazyRescale);
        if (j == 0 || m_ref == -INFINITY) {
          // first block (or nothing seen yet): set the reference, O is not live
          m_ref = fmaxf(m_ref, mx);
          need = false;
        }
        if (__any_sync(0xffffffffu, need)) {
          // O must be quiescent: wait for PV_{j-1}.
          const int i = j - 1;
          if (!warp_wait(&bars.pv_done[i & 1], (i >> 1) & 1, abort_flag, dev_status)) {
            good = false;
            break;
          }
          tc_fence_after();
          float alpha = 1.f;
          if (need) {
            alpha = ex2_approx(m_ref - mx);
            m_ref = mx;
            l_sum *= alpha;
          }
          const uint32_t o_addr = tmem + lane_off + kColO;
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t r[32];
            tmem_ld32_wait(o_addr + cc * 32, r);
#pragma unroll
            for (int i2 = 0; i2 < 32; ++i2) r[i2] = __float_as_uint(__uint_as_float(r[i2]) * alpha);
            tmem_st32(o_addr + cc * 32, r);
          }
          tmem_wait_st();
        }
        const float mref = (m_ref == -INFINITY) ? 0.f : m_ref;
        uint32_t p[64];
        float lsum_blk = 0.f;
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const float p0 = ex2_approx(x[2 * i] - mref);
          const float p1 = ex2_approx(x[2 * i + 1] - mref);
          lsum_blk += p0 + p1;
          p[i] = pack_bf16x2(p0, p1);
        }
        l_sum += lsum_blk;
        uint32_t (&p_lo)[32] = *reinterpret_cast<uint32_t(*)[32]>(&p[0]);
        uint32_t (&p_hi)[32] = *reinterpret_cast<uint32_t(*)[32]>(&p[32]);
        tmem_st32(s_addr, p_lo);
        tmem_st32(s_addr + 32, p_hi);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars.p_full[s]);
      } else {
        // S has been read into registers: release the buffer first.
        tc_fence_before();
        mbar_arrive(&bars.p_full[s]);
        if (j < n_blocks - args.nkb) {
          // sweep 0 (no lse given): online log-sum-exp of the row
          const float m_new = fmaxf(m_ref, mx);
          const float mref = (m_new == -INFINITY) ? 0.f : m_new;
          float acc = 0.f;
#pragma unroll
          for (int i = 0; i < kTile; ++i) acc += ex2_approx(x[i] - mref);
          l_sum = l_sum * ex2_approx(((m_ref == -INFINITY) ? mref : m_ref) - mref) + acc;
          m_ref = m_new;
          if (j == n_blocks - args.nkb - 1) lse2 = m_ref + __log2f(l_sum);
        } else {
          float acc = 0.f;
          if (grow < args.Lq) {
#pragma unroll
            for (int i = 0; i < kTile; ++i) acc += ex2_approx(x[i] - lse2);
          }
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
          if (lane == 0 && kb_raw >= 0 && kb_raw < args.nkb) atomicAdd(&mass_sh[kb_raw], acc);
        }
      }
    }

    if constexpr (MODE == kModeAttn) {
      const int64_t bh = static_cast<int64_t>(b) * args.H + h;
      if (good && n_blocks > 0) {
        const int i = n_blocks - 1;
        good = warp_wait(&bars.pv_done[i & 1], (i >> 1) & 1, abort_flag, dev_status);
      }
      if (good) {
        tc_fence_after();
        const float inv_l = (n_blocks > 0 && l_sum > 0.f) ? 1.f / l_sum : 0.f;
        __nv_bfloat16* orow = args.o + b * args.o_sb + h * args.o_sh + grow * args.o_sr;
        const uint32_t o_addr = tmem + lane_off + kColO;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t r[32];
          if (n_blocks > 0) {
            tmem_ld32_wait(o_addr + cc * 32, r);
          } else {
#pragma unroll
            for (int i2 = 0; i2 < 32; ++i2) r[i2] = 0u;
          }
          uint32_t pk[16];
#pragma unroll
          for (int i2 = 0; i2 < 16; ++i2)
            pk[i2] = pack_bf16x2(__uint_as_float(r[2 * i2]) * inv_l,
                                 __uint_as_float(r[2 * i2 + 1]) * inv_l);
          if (grow < args.Lq) {
            uint4* dst = reinterpret_cast<uint4*>(orow + cc * 32);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4)
              dst[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
          }
        }
        if (args.lse_out && grow < args.Lq) {
          const float lse = (n_blocks > 0 && l_sum > 0.f)
                                ? (m_ref + __log2f(l_sum)) * 0.6931471805599453f
                                : -INFINITY;
          args.lse_out[bh * args.Lq + grow] = lse;
        }
      }
    } else {
      // ---- CS4A selection for this query block (warp 0 of the softmax group)
      asm volatile("bar.sync 1, 128;" ::: "memory");
      const int aborted = __shfl_sync(0xffffffffu, *abort_flag, 0);
      if (warp == 0 && !aborted) {
        const int nkb = args.nkb;
        const int nq_blk = min(kTile, args.Lq - qb * kTile);
        const float inv_nq = 1.f / static_cast<float>(nq_blk);
        const int64_t rowid = (static_cast<int64_t>(b) * args.H + h) * args.nqb + qb;
        for (int i = lane; i < nkb; i += 32) {
          const float mval = mass_sh[i] * inv_nq;
          mass_sh[i] = mval;
          if (args.mass_out) args.mass_out[rowid * nkb + i] = mval;
        }
        __syncwarp();
        float run = 0.f;
        int taken = 0;
        const int limit = args.topk > 0 ? min(args.topk, nkb) : nkb;
        while (taken < limit) {
          float best = -1.f;
          int best_i = 0x7fffffff;
          for (int i = lane; i < nkb; i += 32) {
            if (!kept_sh[i]) {
              const float mv = mass_sh[i];
              if (mv > best || (mv == best && i < best_i)) { best = mv; best_i = i; }
            }
          }
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) {
            const float ob = __shfl_xor_sync(0xffffffffu, best, off);
            const int oi = __shfl_xor_sync(0xffffffffu, best_i, off);
            if (ob > best || (ob == best && oi < best_i)) { best = ob; best_i = oi; }
          }
          if (lane == 0) kept_sh[best_i] = 1;
          __syncwarp();
          run += best;
          ++taken;
          if (args.topk <= 0 && run >= args.mass_threshold) break;
        }
        // ascending compaction
        int base = 0;
        int32_t* out = args.sel_idx + rowid * nkb;
        for (int i0 = 0; i0 < nkb; i0 += 32) {
          const int i = i0 + lane;
          const bool k = i < nkb && kept_sh[i];
          const uint32_t bal = __ballot_sync(0xffffffffu, k);
          if (k) out[base + __popc(bal & ((1u << lane) - 1u))] = i;
          base += __popc(bal);
        }
        for (int i = base + lane; i < nkb; i += 32) out[i] = -1;
        if (lane == 0) args.sel_cnt[rowid] = base;
      }
    }
  }

  // ---- teardown: every role has left its loop and drained its async work
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace sparvar
