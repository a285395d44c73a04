// Integer kernels that build and check KV-block lists:
//   csla_mask_kernel      CSLA sink + cross-scale locality mask, one CTA per query block
//   map_indices_kernel    CS4A proportional index mapping, one CTA per (b, h, dst query block)
//   map_2d_kernel         CS4A scale-aware 2-D index mapping, same grid
//   validate_lists_kernel range / order check of block lists, one warp per list
//   coarsen_lists_kernel  fine (16/32/64) block lists -> 128x128 tile lists with
//                         per-tile bitmasks, one CTA per (b, h, query tile)
// They build a KV-block bitset in shared memory with atomicOr and then compact
// it into an ascending list (-1 padded) with warp ballots.  Integer only, so
// results are exact.
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace sparvar {

constexpr int kMaskThreads = 256;

struct ScaleGeometry {
  int n_scales;
  int side[32];
  int off[33];
};

// Set bits [k0, k1] (inclusive) of a shared bitset.
__device__ __forceinline__ void set_bit_range(uint32_t* bits, int k0, int k1) {
  if (k1 < k0) return;
  for (int w = k0 >> 5; w <= (k1 >> 5); ++w) {
    const int lo = max(k0 - w * 32, 0);
    const int hi = min(k1 - w * 32, 31);
    const uint32_t upto = hi == 31 ? 0xffffffffu : ((1u << (hi + 1)) - 1u);
    const uint32_t from = ~((1u << lo) - 1u);
    atomicOr(&bits[w], upto & from);
  }
}

// Compact a bitset of nkb bits into an ascending index row (warp 0 only).
__device__ __forceinline__ void compact_bitset(const uint32_t* bits, int nkb, int32_t* idx_row,
                                               int32_t* cnt_out, uint8_t* mask_row) {
  const int lane = threadIdx.x & 31;
  const int nwords = (nkb + 31) >> 5;
  int base = 0;
  for (int w0 = 0; w0 < nwords; w0 += 32) {
    const int w = w0 + lane;
    const uint32_t word = w < nwords ? bits[w] : 0u;
    const int c = __popc(word);
    int incl = c;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    int pos = base + incl - c;
    uint32_t rest = word;
    while (rest) {
      const int bit = __ffs(rest) - 1;
      rest &= rest - 1;
      idx_row[pos++] = w * 32 + bit;
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  for (int i = base + lane; i < nkb; i += 32) idx_row[i] = -1;
  if (mask_row) {
    for (int i = lane; i < nkb; i += 32) mask_row[i] = (bits[i >> 5] >> (i & 31)) & 1u;
  }
  if (lane == 0) *cnt_out = base;
}

// Order of the query tiles for the persistent attention kernel on G CTAs, whose
// CTA c takes the tiles at positions c, c + G, c + 2G, ... of `order` (tile id =
// (b * H + h) * nqb + qb).  Round r is the natural tiles r*G .. r*G + G - 1 (the
// kernel's r-th wave, so the waves keep touching the K/V of the same heads); a
// round's tiles are ranked longest list first, then by query block, then by tile
// id, and dealt in a serpentine: to CTAs 0..G-1 in even rounds and G-1..0 in odd
// ones, so that each CTA's total work is close to the mean.  The counts are read
// through L2 (they may have been written by other CTAs of the same launch).
constexpr int kOrderMaxG = 1024;
constexpr int kOrderSlots = 4096;  // list lengths held in shared memory at a time
constexpr int kOrderMaxQb = 1024;

__device__ __forceinline__ int clamp_len(int n, int idx_row_len) {
  return n < 0 ? 0 : (n > idx_row_len ? idx_row_len : n);
}

// Lists per (b, h, query block): the lengths of a run of whole rounds go to shared
// memory, then each tile's rank is the number of its round's tiles ranked before
// it (G compares per tile).
__device__ void order_tiles_block(const int32_t* kv_cnt, int64_t sb, int64_t sh, int B, int H,
                                  int nqb, int idx_row_len, int G, int32_t* order) {
  __shared__ int len[kOrderSlots];
  const int T = B * H * nqb;
  const int span = (kOrderSlots / G) * G;
  for (int c0 = 0; c0 < T; c0 += span) {
    const int n = min(span, T - c0);
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      const int t = c0 + i, qb = t % nqb, bh = t / nqb;
      len[i] = clamp_len(__ldcg(kv_cnt + (bh / H) * sb + (bh % H) * sh + qb), idx_row_len);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
      const int rs = (i / G) * G, nr = min(G, n - rs), own = i - rs;
      const int li = len[i], qi = (c0 + i) % nqb;
      int qu = (c0 + rs) % nqb, rank = 0;
#pragma unroll 4
      for (int u = 0; u < nr; ++u) {
        const int lu = len[rs + u];
        rank += (lu > li) | ((lu == li) & ((qu < qi) | ((qu == qi) & (u < own))));
        qu = qu + 1 == nqb ? 0 : qu + 1;
      }
      const bool odd = ((c0 + rs) / G) & 1;
      order[c0 + rs + (odd ? nr - 1 - rank : rank)] = c0 + i;
    }
    __syncthreads();
  }
}

// The same order for lists shared by every (b, h) (kv_cnt[qb]): the query blocks
// are ranked once (longest first, then by index); then one warp per round takes
// them in that order, 32 at a time: a query block's tiles in the round (every
// nqb-th tile) take, in tile-id order, the positions after those of the query
// blocks ranked before it (a warp scan of the per-block counts).  nqb <= kOrderMaxQb.
__device__ void order_tiles_shared_lists(const int32_t* kv_cnt, int B, int H, int nqb,
                                         int idx_row_len, int G, int32_t* order) {
  __shared__ int len_q[kOrderMaxQb];
  __shared__ int qb_at[kOrderMaxQb];
  for (int q = threadIdx.x; q < nqb; q += blockDim.x) len_q[q] = clamp_len(__ldcg(kv_cnt + q), idx_row_len);
  __syncthreads();
  for (int q = threadIdx.x; q < nqb; q += blockDim.x) {
    const int lq = len_q[q];
    int rank = 0;
#pragma unroll 8
    for (int u = 0; u < nqb; ++u) rank += (len_q[u] > lq) | ((len_q[u] == lq) & (u < q));
    qb_at[rank] = q;
  }
  __syncthreads();
  const int T = B * H * nqb, rounds = (T + G - 1) / G;
  const int lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  for (int r = threadIdx.x >> 5; r < rounds; r += nwarps) {
    const int r0 = r * G, nr = min(G, T - r0), r1 = r0 + nr, rm = r0 % nqb;
    const bool odd = r & 1;
    int p = 0;  // positions taken by the query blocks ranked before this chunk of 32
    for (int s0 = 0; s0 < nqb; s0 += 32) {
      int u0 = 0, c = 0;
      if (s0 + lane < nqb) {
        const int q = qb_at[s0 + lane];
        u0 = r0 + (q >= rm ? q - rm : q - rm + nqb);  // the round's first tile of query block q
        c = u0 < r1 ? (r1 - 1 - u0) / nqb + 1 : 0;
      }
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      for (int k = 0; k < c; ++k) {
        const int pos = p + incl - c + k;
        order[r0 + (odd ? nr - 1 - pos : pos)] = u0 + k * nqb;
      }
      p += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
  __syncthreads();
}

// The order on its own: one CTA of 1024 threads.
__global__ void __launch_bounds__(1024)
    tile_order_kernel(const int32_t* kv_cnt, int64_t sb, int64_t sh, int B, int H, int nqb,
                      int idx_row_len, int G, int32_t* order) {
  order_tiles_block(kv_cnt, sb, sh, B, H, nqb, idx_row_len, G, order);
}

// ---------------------------------------------------------------- CSLA
// For the query block's rows, each (query row i, scale m) pair contributes the
// keys of scale m in rows [ci - r, ci + r] and columns [cl - r, ch + r], where
// ci = floor(i*s_m/s_k) and [cl, ch] is the projection of the block's columns in
// row i (the projection of consecutive columns moves by 0 or 1, so the union of
// the per-query windows is that rectangle).  Each key row of the rectangle is a
// contiguous token range, which sets a contiguous range of KV-block bits.
// With `order` set, the CTA that finishes last (counted in *done, which it sets
// back to zero) also writes the tile order of the lists for a
// (B, H) launch of the attention kernel on G CTAs (the lists are shared by every
// batch item and head).
struct TileOrderOut {
  int32_t* order;  // null: no order
  int32_t* done;   // zero before the launch, zero after it
  int B, H, G;
};
__global__ void __launch_bounds__(kMaskThreads)
    csla_mask_kernel(const ScaleGeometry g, int q_scale, int n_sink, int r_prev, int r_own,
                     int block_q, int block_kv, int nkb, int32_t* kv_cnt, int32_t* kv_idx,
                     uint8_t* blk_mask, const TileOrderOut ord) {
  // the attention launch behind it may start its prologue now; it reads the lists
  // only after this grid has completed
  griddep_launch_dependents();
  extern __shared__ uint32_t bits[];
  const int qb = blockIdx.x;
  const int nwords = (nkb + 31) >> 5;
  for (int w = threadIdx.x; w < nwords; w += blockDim.x) bits[w] = 0u;
  __syncthreads();

  const int sk = g.side[q_scale];
  const int nq = sk * sk;
  const int q0 = qb * block_q;
  const int q1 = min(q0 + block_q, nq) - 1;
  const int i0 = q0 / sk, i1 = q1 / sk;
  const int sink_scales = min(n_sink, q_scale + 1);
  const int n_sink_tok = g.off[sink_scales];
  if (threadIdx.x == 0 && n_sink_tok > 0) set_bit_range(bits, 0, (n_sink_tok - 1) / block_kv);

  const int m_first = n_sink;
  const int num_m = q_scale - m_first + 1;
  if (num_m > 0) {
    const int num_rows = i1 - i0 + 1;
    for (int t = threadIdx.x; t < num_rows * num_m; t += blockDim.x) {
      const int i = i0 + t / num_m;
      const int m = m_first + t % num_m;
      const int j_lo = (i == i0) ? q0 - i * sk : 0;
      const int j_hi = (i == i1) ? q1 - i * sk : sk - 1;
      const int sm = g.side[m];
      const int r = (m == q_scale) ? r_own : r_prev;
      // (32-bit unsigned: sides are at most 46340, so the products stay below 2^32)
      const uint32_t usm = static_cast<uint32_t>(sm), usk = static_cast<uint32_t>(sk);
      const int ci = static_cast<int>(static_cast<uint32_t>(i) * usm / usk);
      const int cl = static_cast<int>(static_cast<uint32_t>(j_lo) * usm / usk);
      const int ch = static_cast<int>(static_cast<uint32_t>(j_hi) * usm / usk);
      const int a_lo = max(0, ci - r), a_hi = min(sm - 1, ci + r);
      const int b_lo = max(0, cl - r), b_hi = min(sm - 1, ch + r);
      for (int a = a_lo; a <= a_hi; ++a) {
        const int t_lo = g.off[m] + a * sm + b_lo;
        const int t_hi = g.off[m] + a * sm + b_hi;
        set_bit_range(bits, t_lo / block_kv, t_hi / block_kv);
      }
    }
  }
  __syncthreads();
  if (threadIdx.x < 32)
    compact_bitset(bits, nkb, kv_idx + static_cast<int64_t>(qb) * nkb, kv_cnt + qb,
                   blk_mask ? blk_mask + static_cast<int64_t>(qb) * nkb : nullptr);
  if (ord.order) {
    __shared__ int last;
    __threadfence();  // this CTA's count is visible before it is counted as done
    __syncthreads();
    if (threadIdx.x == 0) last = atomicAdd(ord.done, 1) == static_cast<int>(gridDim.x) - 1;
    __syncthreads();
    if (last) {
      __threadfence();
      order_tiles_shared_lists(kv_cnt, ord.B, ord.H, gridDim.x, nkb, ord.G, ord.order);
      if (threadIdx.x == 0) *ord.done = 0;
    }
  }
}

// ---------------------------------------------------------------- CS4A mapping
__device__ __forceinline__ int64_t floor_scale(int64_t x, int64_t num, int64_t den) {
  return (x * num) / den;
}
__device__ __forceinline__ int64_t ceil_scale(int64_t x, int64_t num, int64_t den) {
  return (x * num + den - 1) / den;
}

__global__ void __launch_bounds__(kMaskThreads)
    map_indices_kernel(const int32_t* src_cnt, const int32_t* src_idx, int H, int s_nq,
                       int s_lkv, int d_nq, int d_lkv, int block_q, int block_kv, int s_nqb,
                       int s_nkb, int d_nqb, int d_nkb, int n_sink_tok, int32_t* d_cnt,
                       int32_t* d_idx, uint8_t* d_mask, int32_t* dev_status) {
  extern __shared__ uint32_t bits[];
  const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int64_t bh = static_cast<int64_t>(b) * H + h;
  const int nwords = (d_nkb + 31) >> 5;
  for (int w = threadIdx.x; w < nwords; w += blockDim.x) bits[w] = 0u;
  __syncthreads();

  const int a = qb * block_q;
  const int bnd = min(a + block_q, d_nq);
  for (int t = threadIdx.x; t < s_nqb * s_nkb; t += blockDim.x) {
    const int qs = t / s_nkb, e = t % s_nkb;
    const int64_t srow = bh * s_nqb + qs;
    int cnt = src_cnt[srow];
    if (cnt < 0 || cnt > s_nkb) {
      if (e == 0 && dev_status) atomicOr(dev_status, 0x1);
      cnt = cnt < 0 ? 0 : s_nkb;
    }
    if (e >= cnt) continue;
    const int qlo = qs * block_q, qhi = min(qlo + block_q, s_nq);
    const int64_t tq_lo = floor_scale(qlo, d_nq, s_nq);
    const int64_t tq_hi = ceil_scale(qhi, d_nq, s_nq);
    if (!(a < tq_hi && tq_lo < bnd)) continue;
    const int kb = src_idx[srow * s_nkb + e];
    if (kb < 0 || kb >= s_nkb) {
      if (dev_status) atomicOr(dev_status, 0x1);
      continue;
    }
    const int klo = kb * block_kv, khi = min(klo + block_kv, s_lkv);
    const int64_t tk_lo = floor_scale(klo, d_lkv, s_lkv);
    const int64_t tk_hi = min(ceil_scale(khi, d_lkv, s_lkv), static_cast<int64_t>(d_lkv));
    if (tk_hi > tk_lo)
      set_bit_range(bits, static_cast<int>(tk_lo / block_kv),
                    static_cast<int>((tk_hi - 1) / block_kv));
  }
  if (threadIdx.x == 0 && n_sink_tok > 0)
    set_bit_range(bits, 0, min(d_nkb - 1, (n_sink_tok - 1) / block_kv));
  __syncthreads();
  if (threadIdx.x < 32) {
    const int64_t drow = bh * d_nqb + qb;
    compact_bitset(bits, d_nkb, d_idx + drow * d_nkb, d_cnt + drow,
                   d_mask ? d_mask + drow * d_nkb : nullptr);
  }
}

// ---------------------------------------------------------------- CS4A 2-D mapping
// Rows (columns) [lo, hi) of a side-s_dst grid covered by row (column) i of a
// side-s_src grid: lo = floor(i*s_dst/s_src), hi = ceil((i+1)*s_dst/s_src).
__device__ __forceinline__ void cell_range(int64_t i, int64_t s_src, int64_t s_dst, int64_t* lo,
                                           int64_t* hi) {
  *lo = (i * s_dst) / s_src;
  *hi = ((i + 1) * s_dst + s_src - 1) / s_src;
}

// A decision-scale query (i, j) (side s_d) stands for its upscaled cell of the
// target scale (side s_t); a key below off_d keeps its index; a decision-scale
// key (a, b) stands for its cell in the target's own tokens (from off_t).
// Source query blocks whose cells meet this CTA's destination query block are
// flagged first; every kept entry of a flagged block then sets the destination
// KV blocks of its mapped keys.
__global__ void __launch_bounds__(kMaskThreads)
    map_2d_kernel(const int32_t* src_cnt, const int32_t* src_idx, int H, int s_d, int s_t,
                  int off_d, int l_d, int off_t, int block_q, int block_kv, int s_nqb, int s_nkb,
                  int d_nqb, int d_nkb, int n_sink_tok, int32_t* d_cnt, int32_t* d_idx,
                  uint8_t* d_mask, int32_t* dev_status) {
  extern __shared__ uint32_t bits[];
  const int nwords = (d_nkb + 31) >> 5;
  int* flag = reinterpret_cast<int*>(bits + nwords);
  const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int64_t bh = static_cast<int64_t>(b) * H + h;
  for (int w = threadIdx.x; w < nwords; w += blockDim.x) bits[w] = 0u;
  for (int w = threadIdx.x; w < s_nqb; w += blockDim.x) flag[w] = 0;
  __syncthreads();

  // source query blocks reaching destination tokens [a, bnd)
  const int64_t a = static_cast<int64_t>(qb) * block_q;
  const int64_t bnd = min(a + block_q, static_cast<int64_t>(s_t) * s_t);
  const int n_d = s_d * s_d;
  for (int q = threadIdx.x; q < n_d; q += blockDim.x) {
    int64_t r0, r1, c0, c1;
    cell_range(q / s_d, s_d, s_t, &r0, &r1);
    cell_range(q % s_d, s_d, s_t, &c0, &c1);
    bool hit = false;
    for (int64_t r = r0; r < r1 && !hit; ++r) hit = (r * s_t + c0 < bnd) && (a < r * s_t + c1);
    if (hit) flag[q / block_q] = 1;
  }
  __syncthreads();

  for (int t = threadIdx.x; t < s_nqb * s_nkb; t += blockDim.x) {
    const int qs = t / s_nkb, e = t % s_nkb;
    const int64_t srow = bh * s_nqb + qs;
    int cnt = src_cnt[srow];
    if (cnt < 0 || cnt > s_nkb) {
      if (e == 0 && dev_status) atomicOr(dev_status, 0x1);
      cnt = cnt < 0 ? 0 : s_nkb;
    }
    if (e >= cnt || !flag[qs]) continue;
    const int kb = src_idx[srow * s_nkb + e];
    if (kb < 0 || kb >= s_nkb) {
      if (dev_status) atomicOr(dev_status, 0x1);
      continue;
    }
    const int klo = kb * block_kv, khi = min(klo + block_kv, l_d);
    // earlier scales: same keys
    const int ihi = min(khi, off_d);
    if (ihi > klo) set_bit_range(bits, klo / block_kv, (ihi - 1) / block_kv);
    // decision-scale keys: their cells in the target scale's own tokens
    const int u0 = max(klo, off_d) - off_d, u1 = khi - off_d;
    for (int row = u0 / s_d; u1 > u0 && row <= (u1 - 1) / s_d; ++row) {
      const int b0 = row == u0 / s_d ? u0 % s_d : 0;
      const int b1 = row == (u1 - 1) / s_d ? (u1 - 1) % s_d : s_d - 1;
      int64_t r0, r1, c0, c1, cx, cy;
      cell_range(row, s_d, s_t, &r0, &r1);
      cell_range(b0, s_d, s_t, &c0, &cx);
      cell_range(b1, s_d, s_t, &cy, &c1);
      for (int64_t r = r0; r < r1; ++r) {
        const int64_t k0 = off_t + r * s_t + c0, k1 = off_t + r * s_t + c1 - 1;
        set_bit_range(bits, static_cast<int>(k0 / block_kv), static_cast<int>(k1 / block_kv));
      }
    }
  }
  if (threadIdx.x == 0 && n_sink_tok > 0)
    set_bit_range(bits, 0, min(d_nkb - 1, (n_sink_tok - 1) / block_kv));
  __syncthreads();
  if (threadIdx.x < 32) {
    const int64_t drow = bh * d_nqb + qb;
    compact_bitset(bits, d_nkb, d_idx + drow * d_nkb, d_cnt + drow,
                   d_mask ? d_mask + drow * d_nkb : nullptr);
  }
}

// ---------------------------------------------------------------- coarsening
// Fine square blocks of side 128/g (g = 2, 4 or 8) grouped into 128x128 tiles.
// For query tile T and KV tile kt, bit (qi * g + ki) of the tile mask is set
// when fine KV block kt*g + ki is listed for fine query block T*g + qi; the tile
// list holds, ascending, every kt whose mask is not zero.  Fine entries outside
// [0, nkb_f) are flagged (SPARVAR_DEV_BAD_LIST) and skipped.  Dynamic shared
// memory: nkt 64-bit masks, then ceil(nkt / 32) bitset words.
__global__ void __launch_bounds__(kMaskThreads)
    coarsen_lists_kernel(const int32_t* kv_cnt, const int32_t* kv_idx, int64_t l_sb, int64_t l_sh,
                         int idx_row_len, int nqb_f, int nkb_f, int g, int nqt, int nkt,
                         int32_t* t_cnt, int32_t* t_idx, uint64_t* t_mask, int32_t* dev_status) {
  extern __shared__ uint64_t masks[];
  uint32_t* bits = reinterpret_cast<uint32_t*>(masks + nkt);
  const int T = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int nwords = (nkt + 31) >> 5;
  for (int i = threadIdx.x; i < nkt; i += blockDim.x) masks[i] = 0ull;
  __syncthreads();
  int bad = 0;
  for (int qi = 0; qi < g; ++qi) {
    const int qbf = T * g + qi;
    if (qbf >= nqb_f) break;
    const int64_t row = b * l_sb + h * l_sh + qbf;
    int n = kv_cnt[row];
    if (n < 0 || n > idx_row_len) {
      bad = 1;
      n = n < 0 ? 0 : idx_row_len;
    }
    const int32_t* list = kv_idx + row * idx_row_len;
    for (int e = threadIdx.x; e < n; e += blockDim.x) {
      const int kb = list[e];
      if (kb < 0 || kb >= nkb_f) {
        bad = 1;
        continue;
      }
      atomicOr(reinterpret_cast<unsigned long long*>(&masks[kb / g]),
               1ull << (qi * g + kb % g));
    }
  }
  if (bad && dev_status) atomicOr(dev_status, 0x1);
  __syncthreads();
  for (int w = threadIdx.x; w < nwords; w += blockDim.x) {
    uint32_t word = 0u;
    for (int i = 0; i < 32; ++i) {
      const int kt = w * 32 + i;
      if (kt < nkt && masks[kt] != 0ull) word |= 1u << i;
    }
    bits[w] = word;
  }
  __syncthreads();
  if (threadIdx.x >= 32) return;
  const int64_t orow = (static_cast<int64_t>(b) * gridDim.y + h) * nqt + T;
  int32_t* idx_row = t_idx + orow * nkt;
  uint64_t* mask_row = t_mask + orow * nkt;
  const int lane = threadIdx.x;
  int base = 0;
  for (int w0 = 0; w0 < nwords; w0 += 32) {
    const int w = w0 + lane;
    const uint32_t word = w < nwords ? bits[w] : 0u;
    const int c = __popc(word);
    int incl = c;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    int pos = base + incl - c;
    uint32_t rest = word;
    while (rest) {
      const int kt = w * 32 + __ffs(rest) - 1;
      rest &= rest - 1;
      idx_row[pos] = kt;
      mask_row[pos] = masks[kt];
      ++pos;
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  for (int i = base + lane; i < nkt; i += 32) {
    idx_row[i] = -1;
    mask_row[i] = 0ull;
  }
  if (lane == 0) t_cnt[orow] = base;
}

// ---------------------------------------------------------------- validation
__global__ void validate_lists_kernel(const int32_t* kv_cnt, const int32_t* kv_idx, int n_rows,
                                      int row_len, int nkb, int32_t* dev_status) {
  const int warps = blockDim.x >> 5;
  const int row = blockIdx.x * warps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= n_rows) return;
  int flags = 0;
  int cnt = kv_cnt[row];
  if (cnt < 0 || cnt > row_len || cnt > nkb) {
    flags |= 0x1;
    cnt = cnt < 0 ? 0 : min(row_len, nkb);
  }
  const int32_t* r = kv_idx + static_cast<int64_t>(row) * row_len;
  for (int e = lane; e < cnt; e += 32) {
    const int v = r[e];
    if (v < 0 || v >= nkb) flags |= 0x1;
    if (e > 0 && r[e - 1] >= v) flags |= 0x4;
  }
  flags = __reduce_or_sync(0xffffffffu, flags);
  if (lane == 0 && flags) atomicOr(dev_status, flags);
}

}  // namespace sparvar
