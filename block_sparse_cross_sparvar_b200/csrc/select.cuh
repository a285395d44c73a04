// CS4A block selection by one warp ("SparVAR", ai.info summary, "Methodology in
// Plain English", CS4A paragraph: the attention weights pooled per block decide
// which key blocks a query block keeps).  Shared by the stand-alone decision
// kernel and the decision instantiation of the attention kernel.
#pragma once

#include <cstdint>

namespace sparvar {

// mass_sh[kb] holds, for one query block, the sum over its nq rows and over the
// keys of KV block kb of the normalised attention weights; kept_sh[0, nkb) is
// zero on entry.  One warp (all 32 lanes): divides by nq (the pooled mass),
// writes it to mass_out (if given), keeps blocks heaviest first (ties to the
// lower index) until topk are kept (topk > 0) or the kept mass reaches tau
// (every block when it never does), and writes the ascending list, padded with
// -1, to idx_out[0, nkb) and its length to *cnt_out.  Leaves mass_sh and
// kept_sh zeroed for the next query block.
__device__ __forceinline__ void select_blocks_warp(float* mass_sh, uint8_t* kept_sh, int nkb,
                                                   int nq, int topk, float tau, float* mass_out,
                                                   int32_t* idx_out, int32_t* cnt_out) {
  const int lane = threadIdx.x & 31;
  const float inv_nq = 1.f / static_cast<float>(nq);
  for (int i = lane; i < nkb; i += 32) {
    const float mval = mass_sh[i] * inv_nq;
    mass_sh[i] = mval;
    if (mass_out) mass_out[i] = mval;
  }
  __syncwarp();
  float run = 0.f;
  int taken = 0;
  const int limit = topk > 0 ? min(topk, nkb) : nkb;
  while (taken < limit) {
    float best = -1.f;
    int best_i = 0x7fffffff;
    for (int i = lane; i < nkb; i += 32) {
      if (!kept_sh[i]) {
        const float mv = mass_sh[i];
        if (mv > best || (mv == best && i < best_i)) {
          best = mv;
          best_i = i;
        }
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, off);
      const int oi = __shfl_xor_sync(0xffffffffu, best_i, off);
      if (ob > best || (ob == best && oi < best_i)) {
        best = ob;
        best_i = oi;
      }
    }
    if (lane == 0) kept_sh[best_i] = 1;
    __syncwarp();
    run += best;
    ++taken;
    if (topk <= 0 && run >= tau) break;
  }
  // ascending compaction
  int base = 0;
  for (int i0 = 0; i0 < nkb; i0 += 32) {
    const int i = i0 + lane;
    const bool k = i < nkb && kept_sh[i];
    const uint32_t bal = __ballot_sync(0xffffffffu, k);
    if (k) idx_out[base + __popc(bal & ((1u << lane) - 1u))] = i;
    base += __popc(bal);
  }
  for (int i = base + lane; i < nkb; i += 32) idx_out[i] = -1;
  if (lane == 0) *cnt_out = base;
  __syncwarp();
  for (int i = lane; i < nkb; i += 32) {
    mass_sh[i] = 0.f;
    kept_sh[i] = 0;
  }
  __syncwarp();
}

}  // namespace sparvar
