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

namespace sparvar {

struct OcacheArgs {
  const __nv_bfloat16* o_t;   // [B][H][s_dst^2][D]
  const __nv_bfloat16* o_d;   // [B][H][s_src^2][D] dense output at the decision scale
  const __nv_bfloat16* o_s;   // [B][H][s_src^2][D] sparse output at the decision scale
  __nv_bfloat16* out;         // [B][H][s_dst^2][D], may be o_t
  int B, H, s_src, s_dst, D;
  int64_t t_sb, t_sh, t_sr, d_sb, d_sh, d_sr, s_sb, s_sh, s_sr, u_sb, u_sh, u_sr;
};

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// grid (s_dst, H, B), block (D / 8, ty) with ty * D / 8 <= 256
__global__ void __launch_bounds__(256) ocache_apply_kernel(const OcacheArgs a) {
  const int i = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int c = threadIdx.x * 8;
  const int ty = blockDim.y;
  const int si = static_cast<int>(static_cast<int64_t>(i) * a.s_src / a.s_dst);
  const int64_t row_t = static_cast<int64_t>(i) * a.s_dst, row_s = static_cast<int64_t>(si) * a.s_src;
  const __nv_bfloat16* pt = a.o_t + b * a.t_sb + h * a.t_sh + row_t * a.t_sr + c;
  __nv_bfloat16* pu = a.out + b * a.u_sb + h * a.u_sh + row_t * a.u_sr + c;
  const __nv_bfloat16* pd = a.o_d + b * a.d_sb + h * a.d_sh + row_s * a.d_sr + c;
  const __nv_bfloat16* ps = a.o_s + b * a.s_sb + h * a.s_sh + row_s * a.s_sr + c;
  // j * s_src == sj * s_dst + rem, 0 <= rem < s_dst (j * s_src < 2^31 for sides <= 46340)
  int j = threadIdx.y;
  int sj = j * a.s_src / a.s_dst;
  int rem = j * a.s_src - sj * a.s_dst;
  const int step_q = ty * a.s_src / a.s_dst, step_r = ty * a.s_src - step_q * a.s_dst;
  // four tokens per pass: every load of the pass is issued before its first store
  constexpr int kU = 4;
  for (; j < a.s_dst; j += kU * ty) {
    uint4 vt[kU], vd[kU], vs[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int ju = j + u * ty;
      if (ju < a.s_dst) {
        vt[u] = *reinterpret_cast<const uint4*>(pt + ju * a.t_sr);
        vd[u] = __ldg(reinterpret_cast<const uint4*>(pd + sj * a.d_sr));
        vs[u] = __ldg(reinterpret_cast<const uint4*>(ps + sj * a.s_sr));
      }
      sj += step_q;
      rem += step_r;
      if (rem >= a.s_dst) {
        rem -= a.s_dst;
        ++sj;
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int ju = j + u * ty;
      if (ju < a.s_dst) {
        float ft[8], fd[8], fs[8];
        bf16x8_to_f32(vt[u], ft);
        bf16x8_to_f32(vd[u], fd);
        bf16x8_to_f32(vs[u], fs);
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const __nv_bfloat162 p = __floats2bfloat162_rn(
              ft[2 * k] + (fd[2 * k] - fs[2 * k]), ft[2 * k + 1] + (fd[2 * k + 1] - fs[2 * k + 1]));
          w[k] = *reinterpret_cast<const uint32_t*>(&p);
        }
        *reinterpret_cast<uint4*>(pu + ju * a.u_sr) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
}

}  // namespace sparvar
