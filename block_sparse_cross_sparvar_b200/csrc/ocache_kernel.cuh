// CS4A output cache: a later scale's block-sparse output corrected by the
// decision scale's residual (dense output minus sparse output), upsampled to
// the later scale's grid by nearest neighbour.  Elementwise and bound by HBM.
// One CTA per target row i of one (batch, head), whose nearest source row is
// fixed; thread x takes 8 channels (16 bytes), thread y every ty-th token of
// the row, four of them per pass.  The nearest source column of token j,
// floor(j * s_src / s_dst), is carried from token to token as a quotient and
// remainder, so the loop holds no integer division.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace sparvar {

struct OcacheArgs {
  const __nv_bfloat16* o_t;   // [B][H][s_dst^2][D]
  const __nv_bfloat16* o_d;   // [B][H][s_src^2][D] dense output at the decision scale
  const __nv_bfloat16* o_s;   // [B][H][s_src^2][D] sparse output at the decision scale
  __nv_bfloat16* out;         // [B][H][s_dst^2][D], may be o_t
  int B, H, s_src, s_dst, D;
  int64_t t_sb, t_sh, t_sr, d_sb, d_sh, d_sr, s_sb, s_sh, s_sr, u_sb, u_sh, u_sr;
};

// two bf16 (low half first) as an f32 pair
__device__ __forceinline__ uint64_t bf16x2_to_f2(uint32_t w) {
  return f2_pack(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// grid (s_dst, H, B), block (D / 8, ty) with ty * D / 8 <= 256
__global__ void __launch_bounds__(256) ocache_apply_kernel(const OcacheArgs a) {
  const int i = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int c = threadIdx.x * 8;
  const int ty = blockDim.y;
  const int si = static_cast<int>(static_cast<int64_t>(i) * a.s_src / a.s_dst);
  const int64_t row_t = static_cast<int64_t>(i) * a.s_dst, row_s = static_cast<int64_t>(si) * a.s_src;
  // j * s_src == sj * s_dst + rem, 0 <= rem < s_dst (j * s_src < 2^31 for sides <= 46340)
  int j = threadIdx.y;
  const int sj = j * a.s_src / a.s_dst;
  int rem = j * a.s_src - sj * a.s_dst;
  const int step_q = ty * a.s_src / a.s_dst, step_r = ty * a.s_src - step_q * a.s_dst;
  // running pointers at token j and its source column sj; a step of ty tokens
  // moves the source column by step_q, or step_q + 1 when the remainder wraps
  const __nv_bfloat16* pt = a.o_t + b * a.t_sb + h * a.t_sh + (row_t + j) * a.t_sr + c;
  __nv_bfloat16* pu = a.out + b * a.u_sb + h * a.u_sh + (row_t + j) * a.u_sr + c;
  const __nv_bfloat16* pd = a.o_d + b * a.d_sb + h * a.d_sh + (row_s + sj) * a.d_sr + c;
  const __nv_bfloat16* ps = a.o_s + b * a.s_sb + h * a.s_sh + (row_s + sj) * a.s_sr + c;
  const int64_t t_step = ty * a.t_sr, u_step = ty * a.u_sr;
  const int64_t d_step = step_q * a.d_sr, s_step = step_q * a.s_sr;
  const uint64_t neg1 = f2_pack(-1.f, -1.f);
  // four tokens per pass: every load of the pass is issued before its first store
  constexpr int kU = 4;
  for (; j < a.s_dst; j += kU * ty) {
    uint4 vt[kU], vd[kU], vs[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      if (j + u * ty < a.s_dst) {
        vt[u] = *reinterpret_cast<const uint4*>(pt);
        vd[u] = __ldg(reinterpret_cast<const uint4*>(pd));
        vs[u] = __ldg(reinterpret_cast<const uint4*>(ps));
      }
      pt += t_step;
      pd += d_step;
      ps += s_step;
      rem += step_r;
      if (rem >= a.s_dst) {
        rem -= a.s_dst;
        pd += a.d_sr;
        ps += a.s_sr;
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      if (j + u * ty < a.s_dst) {
        const uint32_t wt[4] = {vt[u].x, vt[u].y, vt[u].z, vt[u].w};
        const uint32_t wd[4] = {vd[u].x, vd[u].y, vd[u].z, vd[u].w};
        const uint32_t ws[4] = {vs[u].x, vs[u].y, vs[u].z, vs[u].w};
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          // (lo, hi) channel pairs in f32: t + (d - s), each step rounded once
          const uint64_t r = f2_fma(bf16x2_to_f2(ws[k]), neg1, bf16x2_to_f2(wd[k]));
          float lo, hi;
          f2_unpack(f2_add(bf16x2_to_f2(wt[k]), r), lo, hi);
          w[k] = pack_bf16x2(lo, hi);
        }
        *reinterpret_cast<uint4*>(pu) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      pu += u_step;
    }
  }
}

}  // namespace sparvar
