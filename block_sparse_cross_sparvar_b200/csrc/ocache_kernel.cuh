// CS4A output cache: a later scale's block-sparse output corrected by the
// decision scale's residual (dense output minus sparse output), upsampled to
// the later scale's grid by nearest neighbour.  Elementwise and bound by HBM:
// each thread takes 8 channels (16 bytes) of one target token.
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

__global__ void __launch_bounds__(256) ocache_apply_kernel(const OcacheArgs a) {
  const int vecs = a.D / 8;
  const int64_t n_t = static_cast<int64_t>(a.s_dst) * a.s_dst;
  const int64_t total = static_cast<int64_t>(a.B) * a.H * n_t * vecs;
  for (int64_t x = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; x < total;
       x += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int c8 = static_cast<int>(x % vecs);
    const int64_t tok = (x / vecs) % n_t;
    const int64_t bh = x / (vecs * n_t);
    const int h = static_cast<int>(bh % a.H), b = static_cast<int>(bh / a.H);
    const int i = static_cast<int>(tok / a.s_dst), j = static_cast<int>(tok % a.s_dst);
    // nearest source token: row floor(i * s_src / s_dst), column likewise
    const int64_t src = static_cast<int64_t>(i) * a.s_src / a.s_dst * a.s_src +
                        static_cast<int64_t>(j) * a.s_src / a.s_dst;
    const uint4 vt = *reinterpret_cast<const uint4*>(a.o_t + b * a.t_sb + h * a.t_sh + tok * a.t_sr + c8 * 8);
    const uint4 vd = __ldg(reinterpret_cast<const uint4*>(a.o_d + b * a.d_sb + h * a.d_sh + src * a.d_sr + c8 * 8));
    const uint4 vs = __ldg(reinterpret_cast<const uint4*>(a.o_s + b * a.s_sb + h * a.s_sh + src * a.s_sr + c8 * 8));
    float ft[8], fd[8], fs[8];
    bf16x8_to_f32(vt, ft);
    bf16x8_to_f32(vd, fd);
    bf16x8_to_f32(vs, fs);
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const __nv_bfloat162 p = __floats2bfloat162_rn(ft[2 * k] + (fd[2 * k] - fs[2 * k]),
                                                     ft[2 * k + 1] + (fd[2 * k + 1] - fs[2 * k + 1]));
      w[k] = *reinterpret_cast<const uint32_t*>(&p);
    }
    *reinterpret_cast<uint4*>(a.out + b * a.u_sb + h * a.u_sh + tok * a.u_sr + c8 * 8) =
        make_uint4(w[0], w[1], w[2], w[3]);
  }
}

}  // namespace sparvar
