// C-ABI entry points of libsparvar.so (declared in include/sparvar.h).
// Host-side argument checks, TMA tensor-map encoding and kernel launches.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "../../include/sparvar.h"
#include "attn_fwd_kernel.cuh"
#include "decide_kernel.cuh"
#include "decision_attn_kernel.cuh"
#include "mask_kernels.cuh"
#include "ocache_kernel.cuh"
#include "wait_probe_kernel.cuh"

// Scratch of sparvar_block_sparse_attn_fwd_static: one array per device, in the
// library's own module, shared by every call on that device.
constexpr size_t kStaticScratchBytes = size_t{8} << 20;
static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(SPARVAR_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool block_ok(int b) { return b == 16 || b == 32 || b == 64 || b == 128; }

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

int build_geometry(const int32_t* sides, int n_scales, sparvar::ScaleGeometry* g) {
  if (!sides) return fail(SPARVAR_ERR_INVALID_ARG, "sides is NULL");
  if (n_scales < 1 || n_scales > SPARVAR_MAX_SCALES)
    return fail(SPARVAR_ERR_INVALID_ARG, "n_scales=%d outside [1, %d]", n_scales,
                SPARVAR_MAX_SCALES);
  g->n_scales = n_scales;
  int64_t off = 0;
  g->off[0] = 0;
  for (int m = 0; m < n_scales; ++m) {
    if (sides[m] < 1 || sides[m] > 46340)
      return fail(SPARVAR_ERR_INVALID_ARG, "sides[%d]=%d outside [1, 46340]", m, sides[m]);
    g->side[m] = sides[m];
    off += static_cast<int64_t>(sides[m]) * sides[m];
    if (off > (1ll << 30)) return fail(SPARVAR_ERR_INVALID_ARG, "total tokens exceed 2^30");
    g->off[m + 1] = static_cast<int>(off);
  }
  return SPARVAR_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 4-D map over a [B][H][rows][D] bf16 tensor: box = 64 columns x box_rows rows
// (128, a query or key tile; 32, one warp's rows of the decision kernel's output),
// 128-byte swizzle, zero fill outside the tensor.
int make_tmap(CUtensorMap* m, const void* base, int D, int rows, int H, int B, int64_t sr,
              int64_t sh, int64_t sb, const char* name, int box_rows = 128) {
  auto enc = tensor_map_encoder();
  if (!enc) return fail(SPARVAR_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  if (H == 1) sh = static_cast<int64_t>(rows) * sr;
  if (B == 1) sb = static_cast<int64_t>(H) * sh;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(sr * 2), static_cast<cuuint64_t>(sh * 2),
                           static_cast<cuuint64_t>(sb * 2)};
  cuuint32_t box[4] = {64, static_cast<cuuint32_t>(box_rows), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(SPARVAR_ERR_INVALID_ARG, "tensor map for %s rejected (CUresult %d)", name,
                static_cast<int>(r));
  return SPARVAR_OK;
}

// Row stride, head stride and batch stride of one [B][H][rows][D] operand.
int check_operand(const void* p, const int64_t* st, int B, int H, int rows, int D,
                  const char* name) {
  if (!p) return fail(SPARVAR_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned16(p)) return fail(SPARVAR_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  if (!st) return fail(SPARVAR_ERR_INVALID_ARG, "%s strides are NULL", name);
  const int64_t sb = st[0], sh = st[1], sr = st[2];
  if (sr < D || (sr % 8) != 0)
    return fail(SPARVAR_ERR_INVALID_ARG, "%s row stride %lld must be >= D and a multiple of 8",
                name, static_cast<long long>(sr));
  if (H > 1 && (sh <= 0 || (sh % 8) != 0))
    return fail(SPARVAR_ERR_INVALID_ARG, "%s head stride %lld must be a positive multiple of 8",
                name, static_cast<long long>(sh));
  if (B > 1 && (sb <= 0 || (sb % 8) != 0))
    return fail(SPARVAR_ERR_INVALID_ARG, "%s batch stride %lld must be a positive multiple of 8",
                name, static_cast<long long>(sb));
  if (sr * 2 >= (1ll << 40) || sh * 2 >= (1ll << 40) || sb * 2 >= (1ll << 40))
    return fail(SPARVAR_ERR_INVALID_ARG, "%s strides too large", name);
  (void)rows;
  return SPARVAR_OK;
}

template <int D>
int launch_decide_kernel(const CUtensorMap& tq, const CUtensorMap& tk, const sparvar::DecideArgs& a,
                         cudaStream_t stream) {
  auto kern = sparvar::decide_blocks_kernel<D>;
  const uint32_t smem = sparvar::Smem<D>::dyn_bytes();
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  dim3 grid(a.nqb, a.H, a.B);
  kern<<<grid, sparvar::kThreads, smem, stream>>>(tq, tk, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "decide_blocks_kernel launch");
  return SPARVAR_OK;
}

template <int D, bool TOK, bool MULTI, bool ORD = false, bool FINE = true>
int launch_fwd_kernel(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                      const sparvar::fwd::OutMaps& to, const sparvar::fwd::Args& a,
                      cudaStream_t stream) {
  auto kern = sparvar::fwd::attn_fwd_kernel<D, TOK, MULTI, ORD, FINE>;
  const uint32_t smem = sparvar::fwd::Layout<D>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  // persistent: one CTA per SM, each walking tiles blockIdx.x, blockIdx.x + gridDim.x, ...
  int dev = 0, sms = 0;
  e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e, "multiprocessor count");
  const int64_t tiles = a.total_tiles;
  const int64_t grid = tiles < sms ? tiles : sms;
  // the kernel's per-CTA sequence counters (blocks, ring positions) are 32-bit
  int64_t row_len = 0;
  for (int i = 0; i < a.n_problems; ++i) row_len = std::max<int64_t>(row_len, a.prob[i].idx_row_len);
  if (ceil_div(tiles, grid) * (3 * row_len + 1) >= (int64_t{1} << 31))
    return fail(SPARVAR_ERR_UNSUPPORTED, "%lld query tiles x idx_row_len %lld too large per SM",
                static_cast<long long>(tiles), static_cast<long long>(row_len));
  // programmatic stream serialization: the CTAs may start (barriers, TMEM, tensor
  // maps) while the kernel ahead of them on the stream (the list builder) finishes;
  // the kernel waits for that kernel before it reads any list
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(sparvar::fwd::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, tq, tk, tv, to, a);
  if (e != cudaSuccess) return cuda_fail(e, "attn_fwd_kernel launch");
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "attn_fwd_kernel launch");
  return SPARVAR_OK;
}

template <int D>
int launch_decision_kernel(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                           const CUtensorMap& to, const sparvar::dec::Args& a,
                           cudaStream_t stream) {
  auto kern = sparvar::dec::decision_attn_kernel<D>;
  const uint32_t smem = sparvar::dec::Layout<D>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  // the kernel's warpgroups trade registers (setmaxnreg) on the assumption that each
  // thread was launched with exactly kLaunchRegs; any other count could leave a
  // warpgroup waiting for registers that never come, so it is refused
  cudaFuncAttributes fa{};
  e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncGetAttributes");
  if (fa.numRegs != sparvar::dec::kLaunchRegs)
    return fail(SPARVAR_ERR_UNSUPPORTED, "decision_attn_kernel compiled with %d registers per "
                "thread, its register budgets assume %d", fa.numRegs, sparvar::dec::kLaunchRegs);
  // persistent: one CTA per SM, claiming the pairs blockIdx.x, blockIdx.x + gridDim.x, ...
  int dev = 0, sms = 0;
  e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e, "multiprocessor count");
  const int64_t pairs = a.total_pairs;
  const int64_t grid = pairs < sms ? pairs : sms;
  // the kernel's per-CTA sequence counters (blocks, ring loads) are 32-bit
  if (ceil_div(pairs, grid) * (8 * static_cast<int64_t>(a.nkb) + 8) >= (int64_t{1} << 31))
    return fail(SPARVAR_ERR_UNSUPPORTED, "%lld query tile pairs too many per SM",
                static_cast<long long>(pairs));
  kern<<<static_cast<unsigned>(grid), sparvar::dec::kThreads, smem, stream>>>(tq, tk, tv, to, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "decision_attn_kernel launch");
  return SPARVAR_OK;
}

}  // namespace

extern "C" {

const char* sparvar_last_error(void) { return g_last_error.c_str(); }

const char* sparvar_version(void) { return "sparvar-b200 0.1 (sm_100a)"; }

int sparvar_scale_blocks(const int32_t* sides, int n_scales, int q_scale, int block_q,
                         int block_kv, int32_t* nqb, int32_t* nkb) {
  sparvar::ScaleGeometry g;
  int rc = build_geometry(sides, n_scales, &g);
  if (rc) return rc;
  if (q_scale < 0 || q_scale >= n_scales)
    return fail(SPARVAR_ERR_INVALID_ARG, "q_scale=%d outside [0, %d)", q_scale, n_scales);
  if (block_q < 1 || block_kv < 1) return fail(SPARVAR_ERR_INVALID_ARG, "block sizes must be >= 1");
  if (!nqb || !nkb) return fail(SPARVAR_ERR_INVALID_ARG, "output pointers are NULL");
  const int64_t nq = static_cast<int64_t>(g.side[q_scale]) * g.side[q_scale];
  *nqb = static_cast<int32_t>(ceil_div(nq, block_q));
  *nkb = static_cast<int32_t>(ceil_div(g.off[q_scale + 1], block_kv));
  return SPARVAR_OK;
}

static int csla_mask_impl(const int32_t* sides, int n_scales, int q_scale, int n_sink_scales,
                          int radius_prev, int radius_own, int block_q, int block_kv,
                          int32_t* kv_cnt, int32_t* kv_idx, uint8_t* blk_mask, void* stream,
                          sparvar::TileOrderOut ord);

int sparvar_build_csla_mask(const int32_t* sides, int n_scales, int q_scale, int n_sink_scales,
                            int radius_prev, int radius_own, int block_q, int block_kv,
                            int32_t* kv_cnt, int32_t* kv_idx, uint8_t* blk_mask, void* stream) {
  return csla_mask_impl(sides, n_scales, q_scale, n_sink_scales, radius_prev, radius_own, block_q,
                        block_kv, kv_cnt, kv_idx, blk_mask, stream,
                        sparvar::TileOrderOut{nullptr, nullptr, 0, 0, 0});
}

static int attn_grid(int64_t T, int* grid);

int sparvar_build_csla_mask_ordered(const int32_t* sides, int n_scales, int q_scale,
                                    int n_sink_scales, int radius_prev, int radius_own, int B,
                                    int H, int32_t* kv_cnt, int32_t* kv_idx, int32_t* order,
                                    int32_t* done, void* stream) {
  if (B < 1 || H < 1 || B > 65535 || H > 65535)
    return fail(SPARVAR_ERR_INVALID_ARG, "B=%d H=%d outside [1, 65535]", B, H);
  if (!order || !done) return fail(SPARVAR_ERR_INVALID_ARG, "order/done is NULL");
  if (!sides || n_scales < 1 || q_scale < 0 || q_scale >= n_scales)
    return fail(SPARVAR_ERR_INVALID_ARG, "bad schedule or q_scale");
  const int64_t side = sides[q_scale];
  const int64_t nqb = ceil_div(side * side, 128);
  if (nqb > sparvar::kOrderMaxQb)
    return fail(SPARVAR_ERR_UNSUPPORTED, "more than %d query blocks", sparvar::kOrderMaxQb);
  const int64_t T = static_cast<int64_t>(B) * H * nqb;
  if (T > (int64_t{1} << 30)) return fail(SPARVAR_ERR_UNSUPPORTED, "more than 2^30 query tiles");
  int G = 0;
  int rc = attn_grid(T, &G);
  if (rc) return rc;
  if (G > sparvar::kOrderMaxG) return fail(SPARVAR_ERR_UNSUPPORTED, "more than %d SMs", G);
  return csla_mask_impl(sides, n_scales, q_scale, n_sink_scales, radius_prev, radius_own, 128, 128,
                        kv_cnt, kv_idx, nullptr, stream, sparvar::TileOrderOut{order, done, B, H, G});
}

static int csla_mask_impl(const int32_t* sides, int n_scales, int q_scale, int n_sink_scales,
                          int radius_prev, int radius_own, int block_q, int block_kv,
                          int32_t* kv_cnt, int32_t* kv_idx, uint8_t* blk_mask, void* stream,
                          sparvar::TileOrderOut ord) {
  sparvar::ScaleGeometry g;
  int rc = build_geometry(sides, n_scales, &g);
  if (rc) return rc;
  if (q_scale < 0 || q_scale >= n_scales)
    return fail(SPARVAR_ERR_INVALID_ARG, "q_scale=%d outside [0, %d)", q_scale, n_scales);
  if (n_sink_scales < 0) return fail(SPARVAR_ERR_INVALID_ARG, "n_sink_scales < 0");
  if (radius_prev < 0 || radius_own < 0) return fail(SPARVAR_ERR_INVALID_ARG, "radius < 0");
  if (!block_ok(block_q) || !block_ok(block_kv))
    return fail(SPARVAR_ERR_UNSUPPORTED, "block sizes (%d, %d) not in {16, 32, 64, 128}", block_q,
                block_kv);
  if (!kv_cnt || !kv_idx) return fail(SPARVAR_ERR_INVALID_ARG, "kv_cnt/kv_idx is NULL");
  const int64_t nq = static_cast<int64_t>(g.side[q_scale]) * g.side[q_scale];
  const int nqb = static_cast<int>(ceil_div(nq, block_q));
  const int nkb = static_cast<int>(ceil_div(g.off[q_scale + 1], block_kv));
  const size_t smem = static_cast<size_t>((nkb + 31) / 32) * 4;
  // the kernel's static shared memory (the order's 8 KB) and the bitset share 48 KB
  if (smem > 40 * 1024) return fail(SPARVAR_ERR_UNSUPPORTED, "too many KV blocks (%d)", nkb);
  sparvar::csla_mask_kernel<<<nqb, sparvar::kMaskThreads, smem,
                              static_cast<cudaStream_t>(stream)>>>(
      g, q_scale, n_sink_scales, radius_prev, radius_own, block_q, block_kv, nkb, kv_cnt, kv_idx,
      blk_mask, ord);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "csla_mask_kernel launch");
  return SPARVAR_OK;
}

int sparvar_map_indices(const int32_t* src_cnt, const int32_t* src_idx, int B, int H, int src_nq,
                        int src_lkv, int dst_nq, int dst_lkv, int block_q, int block_kv,
                        int n_sink_tokens, int32_t* dst_cnt, int32_t* dst_idx,
                        uint8_t* dst_blk_mask, int32_t* dev_status, void* stream) {
  if (!src_cnt || !src_idx || !dst_cnt || !dst_idx)
    return fail(SPARVAR_ERR_INVALID_ARG, "list pointer is NULL");
  if (B < 1 || H < 1 || B > 65535 || H > 65535)
    return fail(SPARVAR_ERR_INVALID_ARG, "B=%d H=%d outside [1, 65535]", B, H);
  if (src_nq < 1 || src_lkv < 1 || dst_nq < 1 || dst_lkv < 1)
    return fail(SPARVAR_ERR_INVALID_ARG, "sizes must be >= 1");
  if (src_nq > (1 << 30) || src_lkv > (1 << 30) || dst_nq > (1 << 30) || dst_lkv > (1 << 30))
    return fail(SPARVAR_ERR_INVALID_ARG, "sizes must be <= 2^30");
  if (!block_ok(block_q) || !block_ok(block_kv))
    return fail(SPARVAR_ERR_UNSUPPORTED, "block sizes (%d, %d) not in {16, 32, 64, 128}", block_q,
                block_kv);
  if (n_sink_tokens < 0) return fail(SPARVAR_ERR_INVALID_ARG, "n_sink_tokens < 0");
  const int s_nqb = static_cast<int>(ceil_div(src_nq, block_q));
  const int s_nkb = static_cast<int>(ceil_div(src_lkv, block_kv));
  const int d_nqb = static_cast<int>(ceil_div(dst_nq, block_q));
  const int d_nkb = static_cast<int>(ceil_div(dst_lkv, block_kv));
  const size_t smem = static_cast<size_t>((d_nkb + 31) / 32) * 4;
  if (smem > 48 * 1024) return fail(SPARVAR_ERR_UNSUPPORTED, "too many KV blocks (%d)", d_nkb);
  if (static_cast<int64_t>(s_nqb) * s_nkb > (1ll << 30))
    return fail(SPARVAR_ERR_UNSUPPORTED, "source block grid too large");
  dim3 grid(d_nqb, H, B);
  sparvar::map_indices_kernel<<<grid, sparvar::kMaskThreads, smem,
                                static_cast<cudaStream_t>(stream)>>>(
      src_cnt, src_idx, H, src_nq, src_lkv, dst_nq, dst_lkv, block_q, block_kv, s_nqb, s_nkb,
      d_nqb, d_nkb, n_sink_tokens, dst_cnt, dst_idx, dst_blk_mask, dev_status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "map_indices_kernel launch");
  return SPARVAR_OK;
}

int sparvar_map_indices_2d(const int32_t* src_cnt, const int32_t* src_idx, int B, int H,
                           const int32_t* sides, int n_scales, int src_scale, int dst_scale,
                           int block_q, int block_kv, int n_sink_tokens, int32_t* dst_cnt,
                           int32_t* dst_idx, uint8_t* dst_blk_mask, int32_t* dev_status,
                           void* stream) {
  sparvar::ScaleGeometry g;
  int rc = build_geometry(sides, n_scales, &g);
  if (rc) return rc;
  if (!src_cnt || !src_idx || !dst_cnt || !dst_idx)
    return fail(SPARVAR_ERR_INVALID_ARG, "list pointer is NULL");
  if (B < 1 || H < 1 || B > 65535 || H > 65535)
    return fail(SPARVAR_ERR_INVALID_ARG, "B=%d H=%d outside [1, 65535]", B, H);
  if (src_scale < 0 || dst_scale < src_scale || dst_scale >= n_scales)
    return fail(SPARVAR_ERR_INVALID_ARG, "scales %d -> %d: need 0 <= src <= dst < %d", src_scale,
                dst_scale, n_scales);
  if (!block_ok(block_q) || !block_ok(block_kv))
    return fail(SPARVAR_ERR_UNSUPPORTED, "block sizes (%d, %d) not in {16, 32, 64, 128}", block_q,
                block_kv);
  if (n_sink_tokens < 0) return fail(SPARVAR_ERR_INVALID_ARG, "n_sink_tokens < 0");
  const int s_d = g.side[src_scale], s_t = g.side[dst_scale];
  const int s_nqb = static_cast<int>(ceil_div(static_cast<int64_t>(s_d) * s_d, block_q));
  const int s_nkb = static_cast<int>(ceil_div(g.off[src_scale + 1], block_kv));
  const int d_nqb = static_cast<int>(ceil_div(static_cast<int64_t>(s_t) * s_t, block_q));
  const int d_nkb = static_cast<int>(ceil_div(g.off[dst_scale + 1], block_kv));
  const size_t smem = static_cast<size_t>((d_nkb + 31) / 32) * 4 + static_cast<size_t>(s_nqb) * 4;
  if (smem > 48 * 1024) return fail(SPARVAR_ERR_UNSUPPORTED, "block grids too large");
  if (static_cast<int64_t>(s_nqb) * s_nkb > (1ll << 30))
    return fail(SPARVAR_ERR_UNSUPPORTED, "source block grid too large");
  dim3 grid(d_nqb, H, B);
  sparvar::map_2d_kernel<<<grid, sparvar::kMaskThreads, smem, static_cast<cudaStream_t>(stream)>>>(
      src_cnt, src_idx, H, s_d, s_t, g.off[src_scale], g.off[src_scale + 1], g.off[dst_scale],
      block_q, block_kv, s_nqb, s_nkb, d_nqb, d_nkb, n_sink_tokens, dst_cnt, dst_idx,
      dst_blk_mask, dev_status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "map_2d_kernel launch");
  return SPARVAR_OK;
}

int sparvar_coarsen_lists(const int32_t* kv_cnt, const int32_t* kv_idx,
                          const int64_t* list_strides, int idx_row_len, int B, int H, int Lq,
                          int Lkv, int block, int32_t* tile_cnt, int32_t* tile_idx,
                          uint64_t* tile_mask, int32_t* dev_status, void* stream) {
  if (block != 16 && block != 32 && block != 64)
    return fail(SPARVAR_ERR_UNSUPPORTED, "block=%d not in {16, 32, 64}", block);
  if (B < 1 || H < 1 || B > 65535 || H > 65535)
    return fail(SPARVAR_ERR_INVALID_ARG, "B=%d H=%d outside [1, 65535]", B, H);
  if (Lq < 1 || Lkv < 1 || Lq > (1 << 30) || Lkv > (1 << 30))
    return fail(SPARVAR_ERR_INVALID_ARG, "Lq=%d Lkv=%d outside [1, 2^30]", Lq, Lkv);
  if (!kv_cnt || !kv_idx || !list_strides || !tile_cnt || !tile_idx || !tile_mask)
    return fail(SPARVAR_ERR_INVALID_ARG, "a list pointer is NULL");
  if (list_strides[0] < 0 || list_strides[1] < 0)
    return fail(SPARVAR_ERR_INVALID_ARG, "list strides must be >= 0");
  if (idx_row_len < 0) return fail(SPARVAR_ERR_INVALID_ARG, "idx_row_len < 0");
  const int nqt = static_cast<int>(ceil_div(Lq, 128));
  const int nkt = static_cast<int>(ceil_div(Lkv, 128));
  if (nkt > 4096)
    return fail(SPARVAR_ERR_UNSUPPORTED, "Lkv=%d gives %d KV tiles (max 4096)", Lkv, nkt);
  if (nqt > 65535) return fail(SPARVAR_ERR_UNSUPPORTED, "Lq=%d gives too many query tiles", Lq);
  const int Bo = list_strides[0] == 0 ? 1 : B;
  const int Ho = list_strides[1] == 0 ? 1 : H;
  const int g = 128 / block;
  const size_t smem = static_cast<size_t>(nkt) * 8 + static_cast<size_t>((nkt + 31) / 32) * 4;
  cudaError_t e = cudaFuncSetAttribute(sparvar::coarsen_lists_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  dim3 grid(nqt, Ho, Bo);
  sparvar::coarsen_lists_kernel<<<grid, sparvar::kMaskThreads, smem,
                                  static_cast<cudaStream_t>(stream)>>>(
      kv_cnt, kv_idx, list_strides[0], list_strides[1], idx_row_len,
      static_cast<int>(ceil_div(Lq, block)), static_cast<int>(ceil_div(Lkv, block)), g, nqt, nkt,
      tile_cnt, tile_idx, tile_mask, dev_status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "coarsen_lists_kernel launch");
  return SPARVAR_OK;
}

int sparvar_validate_lists(const int32_t* kv_cnt, const int32_t* kv_idx, int n_rows,
                           int idx_row_len, int nkb, int32_t* dev_status, void* stream) {
  if (!kv_cnt || !kv_idx || !dev_status)
    return fail(SPARVAR_ERR_INVALID_ARG, "kv_cnt/kv_idx/dev_status is NULL");
  if (n_rows < 0 || idx_row_len < 0 || nkb < 0)
    return fail(SPARVAR_ERR_INVALID_ARG, "negative size");
  if (n_rows == 0) return SPARVAR_OK;
  const int warps = 8;
  sparvar::validate_lists_kernel<<<static_cast<unsigned>(ceil_div(n_rows, warps)), warps * 32, 0,
                                   static_cast<cudaStream_t>(stream)>>>(
      kv_cnt, kv_idx, n_rows, idx_row_len, nkb, dev_status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "validate_lists_kernel launch");
  return SPARVAR_OK;
}

int sparvar_wait_timeout_probe(uint64_t limit_ns, int32_t* dev_status, int32_t* result,
                               void* stream) {
  if (!dev_status || !result) return fail(SPARVAR_ERR_INVALID_ARG, "dev_status/result is NULL");
  if (limit_ns < 1000u || limit_ns > 1000000000u)
    return fail(SPARVAR_ERR_INVALID_ARG, "limit_ns=%llu outside [1e3, 1e9]",
                static_cast<unsigned long long>(limit_ns));
  sparvar::wait_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      limit_ns, SPARVAR_DEV_TIMEOUT, dev_status, result);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "wait_probe_kernel launch");
  return SPARVAR_OK;
}

// A checked single-problem launch of attn_fwd_kernel: arguments, tensor maps.
struct FwdLaunch {
  sparvar::fwd::Args a;
  CUtensorMap tq, tk, tv;
  sparvar::fwd::OutMaps to;
  int D;
  bool tok;
};

// Checks every argument of a single-problem attention call and encodes its tensor
// maps; enqueues nothing.
static int attn_fwd_prepare(FwdLaunch* L, const void* q, const void* k, const void* v, void* o,
                            float* lse, int B, int H, int Lq, int Lkv, int D,
                            const int64_t* q_strides, const int64_t* k_strides,
                            const int64_t* v_strides, const int64_t* o_strides,
                            const int32_t* kv_cnt, const int32_t* kv_idx,
                            const int64_t* list_strides, int idx_row_len,
                            const uint64_t* tile_mask, int mask_block, int block_q, int block_kv,
                            float softmax_scale, int32_t* dev_status,
                            const sparvar::fwd::CslaTokens* tok) {
  if (D != 64 && D != 128) return fail(SPARVAR_ERR_UNSUPPORTED, "D=%d not in {64, 128}", D);
  if (block_q != 128 || block_kv != 128)
    return fail(SPARVAR_ERR_UNSUPPORTED,
                "attention blocks (%d, %d): this kernel takes 128 x 128 blocks", block_q,
                block_kv);
  if (B < 1 || H < 1 || B > 65535 || H > 65535)
    return fail(SPARVAR_ERR_INVALID_ARG, "B=%d H=%d outside [1, 65535]", B, H);
  if (Lq < 1 || Lkv < 1 || Lq > (1 << 30) || Lkv > (1 << 30))
    return fail(SPARVAR_ERR_INVALID_ARG, "Lq=%d Lkv=%d outside [1, 2^30]", Lq, Lkv);
  if (static_cast<int64_t>(B) * H * ceil_div(Lq, 128) > (int64_t{1} << 30))
    return fail(SPARVAR_ERR_UNSUPPORTED, "B*H*ceil(Lq/128) above 2^30 query tiles");
  int rc;
  if ((rc = check_operand(q, q_strides, B, H, Lq, D, "q"))) return rc;
  if ((rc = check_operand(k, k_strides, B, H, Lkv, D, "k"))) return rc;
  if ((rc = check_operand(v, v_strides, B, H, Lkv, D, "v"))) return rc;
  if ((rc = check_operand(o, o_strides, B, H, Lq, D, "o"))) return rc;
  if (!kv_cnt || !kv_idx || !list_strides)
    return fail(SPARVAR_ERR_INVALID_ARG, "kv_cnt/kv_idx/list_strides is NULL");
  if (list_strides[0] < 0 || list_strides[1] < 0)
    return fail(SPARVAR_ERR_INVALID_ARG, "list strides must be >= 0");
  if (idx_row_len < 0) return fail(SPARVAR_ERR_INVALID_ARG, "idx_row_len < 0");
  int mask_shift = 7;
  if (tile_mask) {
    if (mask_block != 16 && mask_block != 32 && mask_block != 64)
      return fail(SPARVAR_ERR_UNSUPPORTED, "mask_block=%d not in {16, 32, 64}", mask_block);
    mask_shift = mask_block == 16 ? 4 : (mask_block == 32 ? 5 : 6);
  }
  if (!std::isfinite(softmax_scale) || !(softmax_scale > 0.f))
    return fail(SPARVAR_ERR_INVALID_ARG, "softmax_scale must be finite and > 0");

  *L = FwdLaunch{};
  sparvar::fwd::Args& a = L->a;
  a.B = B; a.H = H; a.n_problems = 1;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  sparvar::fwd::Problem& pr = a.prob[0];
  pr.Lq = Lq; pr.Lkv = Lkv;
  pr.nqb = static_cast<int>(ceil_div(Lq, 128));
  pr.nkb = static_cast<int>(ceil_div(Lkv, 128));
  pr.q_row0 = 0; pr.tile0 = 0;
  pr.kv_cnt = kv_cnt; pr.kv_idx = kv_idx;
  pr.list_sb = list_strides[0]; pr.list_sh = list_strides[1];
  pr.idx_row_len = idx_row_len;
  a.total_tiles = static_cast<int>(static_cast<int64_t>(B) * H * pr.nqb);
  a.tile_mask = tile_mask;
  a.mask_shift = mask_shift;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.o_sb = o_strides[0]; a.o_sh = o_strides[1]; a.o_sr = o_strides[2];
  a.lse = lse;
  a.lse_rows = Lq;
  a.dev_status = dev_status;
  if (tok) a.tok = *tok;

  if ((rc = make_tmap(&L->tq, q, D, Lq, H, B, q_strides[2], q_strides[1], q_strides[0], "q")))
    return rc;
  if ((rc = make_tmap(&L->tk, k, D, Lkv, H, B, k_strides[2], k_strides[1], k_strides[0], "k")))
    return rc;
  if ((rc = make_tmap(&L->tv, v, D, Lkv, H, B, v_strides[2], v_strides[1], v_strides[0], "v")))
    return rc;
  if ((rc = make_tmap(&L->to.m[0], o, D, Lq, H, B, o_strides[2], o_strides[1], o_strides[0], "o")))
    return rc;
  L->D = D;
  L->tok = tok != nullptr;
  return SPARVAR_OK;
}

static int attn_fwd_launch(const FwdLaunch& L, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (L.tok) {
    if (L.D == 128) return launch_fwd_kernel<128, true, false>(L.tq, L.tk, L.tv, L.to, L.a, st);
    return launch_fwd_kernel<64, true, false>(L.tq, L.tk, L.tv, L.to, L.a, st);
  }
  // launches without tile masks (every launch in a given order) run instantiations
  // compiled without the fine-mask code
  if (L.a.tile_order) {
    if (L.D == 128)
      return launch_fwd_kernel<128, false, false, true, false>(L.tq, L.tk, L.tv, L.to, L.a, st);
    return launch_fwd_kernel<64, false, false, true, false>(L.tq, L.tk, L.tv, L.to, L.a, st);
  }
  if (!L.a.tile_mask) {
    if (L.D == 128)
      return launch_fwd_kernel<128, false, false, false, false>(L.tq, L.tk, L.tv, L.to, L.a, st);
    return launch_fwd_kernel<64, false, false, false, false>(L.tq, L.tk, L.tv, L.to, L.a, st);
  }
  if (L.D == 128) return launch_fwd_kernel<128, false, false>(L.tq, L.tk, L.tv, L.to, L.a, st);
  return launch_fwd_kernel<64, false, false>(L.tq, L.tk, L.tv, L.to, L.a, st);
}

// Device address of g_static_scratch in the current context.  Looked up with
// cudaGetSymbolAddress once per (device, context) and cached: a new primary context
// (after cudaDeviceReset) loads the module again, possibly elsewhere, so the cache
// is keyed on the context as well as the device.
using PFN_ctx_get_current = CUresult (*)(CUcontext*);
static int static_scratch_address(void** out) {
  static std::mutex mu;
  static PFN_ctx_get_current get_ctx = nullptr;
  static CUcontext ctx_of[128] = {};
  static void* addr_of[128] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 128) return fail(SPARVAR_ERR_UNSUPPORTED, "device %d", dev);
  std::lock_guard<std::mutex> lock(mu);
  if (!get_ctx) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &qr) != cudaSuccess ||
        qr != cudaDriverEntryPointSuccess || !fn)
      return fail(SPARVAR_ERR_CUDA, "cuCtxGetCurrent unavailable");
    get_ctx = reinterpret_cast<PFN_ctx_get_current>(fn);
  }
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS) ctx = nullptr;
  if (!ctx || ctx_of[dev] != ctx || !addr_of[dev]) {
    // the lookup also binds the device's primary context when none is current yet
    void* a = nullptr;
    e = cudaGetSymbolAddress(&a, g_static_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress");
    if (get_ctx(&ctx) != CUDA_SUCCESS || !ctx)
      return fail(SPARVAR_ERR_CUDA, "no current CUDA context");
    ctx_of[dev] = ctx;
    addr_of[dev] = a;
  }
  *out = addr_of[dev];
  return SPARVAR_OK;
}

static int attn_fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                         int H, int Lq, int Lkv, int D, const int64_t* q_strides,
                         const int64_t* k_strides, const int64_t* v_strides,
                         const int64_t* o_strides, const int32_t* kv_cnt, const int32_t* kv_idx,
                         const int64_t* list_strides, int idx_row_len, const uint64_t* tile_mask,
                         int mask_block, int block_q, int block_kv, float softmax_scale,
                         int32_t* dev_status, void* stream,
                         const sparvar::fwd::CslaTokens* tok,
                         const int32_t* tile_order = nullptr) {
  FwdLaunch L;
  int rc = attn_fwd_prepare(&L, q, k, v, o, lse, B, H, Lq, Lkv, D, q_strides, k_strides,
                            v_strides, o_strides, kv_cnt, kv_idx, list_strides, idx_row_len,
                            tile_mask, mask_block, block_q, block_kv, softmax_scale, dev_status,
                            tok);
  if (rc) return rc;
  L.a.tile_order = tile_order;
  return attn_fwd_launch(L, stream);
}

// the persistent attention kernel's grid for T query tiles on the current device
static int attn_grid(int64_t T, int* grid) {
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e, "multiprocessor count");
  *grid = static_cast<int>(T < sms ? T : sms);
  return SPARVAR_OK;
}

int sparvar_tile_order(const int32_t* kv_cnt, int B, int H, int Lq,
                       const int64_t* list_strides, int idx_row_len, int32_t* order,
                       void* stream) {
  if (B < 1 || H < 1 || B > 65535 || H > 65535)
    return fail(SPARVAR_ERR_INVALID_ARG, "B=%d H=%d outside [1, 65535]", B, H);
  if (Lq < 1 || Lq > (1 << 30)) return fail(SPARVAR_ERR_INVALID_ARG, "Lq=%d outside [1, 2^30]", Lq);
  if (!kv_cnt || !order || !list_strides || list_strides[0] < 0 || list_strides[1] < 0 ||
      idx_row_len < 0)
    return fail(SPARVAR_ERR_INVALID_ARG, "bad lists or order buffer");
  const int64_t nqb = ceil_div(Lq, 128);
  const int64_t T = static_cast<int64_t>(B) * H * nqb;
  if (T > (int64_t{1} << 30)) return fail(SPARVAR_ERR_UNSUPPORTED, "more than 2^30 query tiles");
  int G = 0, rc;
  if ((rc = attn_grid(T, &G))) return rc;
  if (G > sparvar::kOrderMaxG) return fail(SPARVAR_ERR_UNSUPPORTED, "more than %d SMs", G);
  sparvar::tile_order_kernel<<<1, 1024, 0, static_cast<cudaStream_t>(stream)>>>(
      kv_cnt, list_strides[0], list_strides[1], B, H, static_cast<int>(nqb), idx_row_len, G, order);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "tile_order_kernel launch");
  return SPARVAR_OK;
}

int sparvar_block_sparse_attn_fwd_ordered(const void* q, const void* k, const void* v, void* o,
                                          float* lse, int B, int H, int Lq, int Lkv, int D,
                                          const int64_t* q_strides, const int64_t* k_strides,
                                          const int64_t* v_strides, const int64_t* o_strides,
                                          const int32_t* kv_cnt, const int32_t* kv_idx,
                                          const int64_t* list_strides, int idx_row_len,
                                          const int32_t* tile_order, float softmax_scale,
                                          int32_t* dev_status, void* stream) {
  if (!tile_order) return fail(SPARVAR_ERR_INVALID_ARG, "tile_order is NULL");
  return attn_fwd_impl(q, k, v, o, lse, B, H, Lq, Lkv, D, q_strides, k_strides, v_strides,
                       o_strides, kv_cnt, kv_idx, list_strides, idx_row_len, nullptr, 0, 128, 128,
                       softmax_scale, dev_status, stream, nullptr, tile_order);
}

int sparvar_block_sparse_attn_fwd(const void* q, const void* k, const void* v, void* o,
                                  float* lse, int B, int H, int Lq, int Lkv, int D,
                                  const int64_t* q_strides, const int64_t* k_strides,
                                  const int64_t* v_strides, const int64_t* o_strides,
                                  const int32_t* kv_cnt, const int32_t* kv_idx,
                                  const int64_t* list_strides, int idx_row_len,
                                  const uint64_t* tile_mask, int mask_block, int block_q,
                                  int block_kv, float softmax_scale, int32_t* dev_status,
                                  void* stream) {
  return attn_fwd_impl(q, k, v, o, lse, B, H, Lq, Lkv, D, q_strides, k_strides, v_strides,
                       o_strides, kv_cnt, kv_idx, list_strides, idx_row_len, tile_mask, mask_block,
                       block_q, block_kv, softmax_scale, dev_status, stream, nullptr);
}

int sparvar_block_sparse_attn_fwd_multi(
    const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int q_rows,
    int kv_rows, int D, const int64_t* q_strides, const int64_t* k_strides,
    const int64_t* v_strides, const int64_t* o_strides, int n_problems, const int32_t* q_row0,
    const int32_t* lq, const int32_t* lkv, const int32_t* const* kv_cnt,
    const int32_t* const* kv_idx, const int64_t* list_strides, const int32_t* idx_row_len,
    float softmax_scale, int32_t* dev_status, void* stream) {
  if (D != 64 && D != 128) return fail(SPARVAR_ERR_UNSUPPORTED, "D=%d not in {64, 128}", D);
  if (B < 1 || H < 1 || B > 65535 || H > 65535)
    return fail(SPARVAR_ERR_INVALID_ARG, "B=%d H=%d outside [1, 65535]", B, H);
  if (q_rows < 1 || kv_rows < 1 || q_rows > (1 << 30) || kv_rows > (1 << 30))
    return fail(SPARVAR_ERR_INVALID_ARG, "q_rows=%d kv_rows=%d outside [1, 2^30]", q_rows, kv_rows);
  if (n_problems < 1 || n_problems > sparvar::fwd::kMaxProblems)
    return fail(SPARVAR_ERR_UNSUPPORTED, "n_problems=%d outside [1, %d]", n_problems,
                sparvar::fwd::kMaxProblems);
  if (!q_row0 || !lq || !lkv || !kv_cnt || !kv_idx || !list_strides || !idx_row_len)
    return fail(SPARVAR_ERR_INVALID_ARG, "a problem array is NULL");
  if (!std::isfinite(softmax_scale) || !(softmax_scale > 0.f))
    return fail(SPARVAR_ERR_INVALID_ARG, "softmax_scale must be finite and > 0");
  int rc;
  if ((rc = check_operand(q, q_strides, B, H, q_rows, D, "q"))) return rc;
  if ((rc = check_operand(k, k_strides, B, H, kv_rows, D, "k"))) return rc;
  if ((rc = check_operand(v, v_strides, B, H, kv_rows, D, "v"))) return rc;
  if ((rc = check_operand(o, o_strides, B, H, q_rows, D, "o"))) return rc;
  sparvar::fwd::Args a{};
  a.B = B; a.H = H; a.n_problems = n_problems;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  int64_t tiles = 0;
  for (int i = 0; i < n_problems; ++i) {
    if (q_row0[i] < 0 || lq[i] < 1 || static_cast<int64_t>(q_row0[i]) + lq[i] > q_rows)
      return fail(SPARVAR_ERR_INVALID_ARG, "problem %d: query rows [%d, %d + %d) outside [0, %d)", i,
                  q_row0[i], q_row0[i], lq[i], q_rows);
    if (lkv[i] < 1 || lkv[i] > kv_rows)
      return fail(SPARVAR_ERR_INVALID_ARG, "problem %d: Lkv=%d outside [1, %d]", i, lkv[i], kv_rows);
    if (!kv_cnt[i] || !kv_idx[i] || list_strides[2 * i] < 0 || list_strides[2 * i + 1] < 0 ||
        idx_row_len[i] < 0)
      return fail(SPARVAR_ERR_INVALID_ARG, "problem %d: bad lists", i);
    sparvar::fwd::Problem& pr = a.prob[i];
    pr.Lq = lq[i]; pr.Lkv = lkv[i];
    pr.nqb = static_cast<int>(ceil_div(lq[i], 128));
    pr.nkb = static_cast<int>(ceil_div(lkv[i], 128));
    pr.q_row0 = q_row0[i];
    pr.tile0 = static_cast<int>(tiles);
    pr.kv_cnt = kv_cnt[i]; pr.kv_idx = kv_idx[i];
    pr.list_sb = list_strides[2 * i]; pr.list_sh = list_strides[2 * i + 1];
    pr.idx_row_len = idx_row_len[i];
    tiles += static_cast<int64_t>(B) * H * pr.nqb;
    if (tiles > (int64_t{1} << 30))
      return fail(SPARVAR_ERR_UNSUPPORTED, "more than 2^30 query tiles");
  }
  a.total_tiles = static_cast<int>(tiles);
  a.tile_mask = nullptr;
  a.mask_shift = 7;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.o_sb = o_strides[0]; a.o_sh = o_strides[1]; a.o_sr = o_strides[2];
  a.lse = lse;
  a.lse_rows = q_rows;
  a.dev_status = dev_status;

  CUtensorMap tq, tk, tv;
  sparvar::fwd::OutMaps to{};
  if ((rc = make_tmap(&tq, q, D, q_rows, H, B, q_strides[2], q_strides[1], q_strides[0], "q")))
    return rc;
  if ((rc = make_tmap(&tk, k, D, kv_rows, H, B, k_strides[2], k_strides[1], k_strides[0], "k")))
    return rc;
  if ((rc = make_tmap(&tv, v, D, kv_rows, H, B, v_strides[2], v_strides[1], v_strides[0], "v")))
    return rc;
  for (int i = 0; i < n_problems; ++i) {
    // the problem's own rows only, so the last tile's rows past its end are clipped
    const void* base = static_cast<const __nv_bfloat16*>(o) + q_row0[i] * o_strides[2];
    if ((rc = make_tmap(&to.m[i], base, D, lq[i], H, B, o_strides[2], o_strides[1], o_strides[0],
                        "o")))
      return rc;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // (multi-problem launches take no tile masks)
  if (D == 128) return launch_fwd_kernel<128, false, true, false, false>(tq, tk, tv, to, a, st);
  return launch_fwd_kernel<64, false, true, false, false>(tq, tk, tv, to, a, st);
}

int sparvar_csla_token_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                                int B, int H, int D, const int64_t* q_strides,
                                const int64_t* k_strides, const int64_t* v_strides,
                                const int64_t* o_strides, const int32_t* sides, int n_scales,
                                int q_scale, int n_sink_scales, int radius_prev, int radius_own,
                                const int32_t* kv_cnt, const int32_t* kv_idx,
                                const int64_t* list_strides, int idx_row_len,
                                float softmax_scale, int32_t* dev_status, void* stream) {
  sparvar::ScaleGeometry g;
  int rc = build_geometry(sides, n_scales, &g);
  if (rc) return rc;
  if (q_scale < 0 || q_scale >= n_scales)
    return fail(SPARVAR_ERR_INVALID_ARG, "q_scale=%d outside [0, %d)", q_scale, n_scales);
  if (n_sink_scales < 0 || radius_prev < 0 || radius_own < 0)
    return fail(SPARVAR_ERR_INVALID_ARG, "n_sink_scales and radii must be >= 0");
  sparvar::fwd::CslaTokens t{};
  t.enabled = 1;
  t.q_scale = q_scale;
  t.n_sink_scales = n_sink_scales;
  t.n_sink_tok = g.off[std::min(n_sink_scales, q_scale + 1)];
  t.r_prev = radius_prev;
  t.r_own = radius_own;
  for (int m = 0; m < n_scales; ++m) t.side[m] = g.side[m];
  for (int m = 0; m <= n_scales; ++m) t.off[m] = g.off[m];
  const int Lq = g.side[q_scale] * g.side[q_scale], Lkv = g.off[q_scale + 1];
  return attn_fwd_impl(q, k, v, o, lse, B, H, Lq, Lkv, D, q_strides, k_strides, v_strides,
                       o_strides, kv_cnt, kv_idx, list_strides, idx_row_len, nullptr, 0, 128, 128,
                       softmax_scale, dev_status, stream, &t);
}

int sparvar_decide_blocks(const void* q, const void* k, int B, int H, int Lq, int Lkv, int D,
                          const int64_t* q_strides, const int64_t* k_strides, float softmax_scale,
                          const float* lse, int block_q, int block_kv, float mass_threshold,
                          float topk_ratio, int32_t* kv_cnt, int32_t* kv_idx, float* mass,
                          int32_t* dev_status, void* stream) {
  if (D != 64 && D != 128) return fail(SPARVAR_ERR_UNSUPPORTED, "D=%d not in {64, 128}", D);
  if (block_q != 128 || block_kv != 128)
    return fail(SPARVAR_ERR_UNSUPPORTED, "decision blocks (%d, %d): 128 x 128 only", block_q,
                block_kv);
  if (B < 1 || H < 1 || B > 65535 || H > 65535)
    return fail(SPARVAR_ERR_INVALID_ARG, "B=%d H=%d outside [1, 65535]", B, H);
  if (Lq < 1 || Lkv < 1 || Lq > (1 << 30) || Lkv > (1 << 30))
    return fail(SPARVAR_ERR_INVALID_ARG, "Lq=%d Lkv=%d outside [1, 2^30]", Lq, Lkv);
  const int nkb = static_cast<int>(ceil_div(Lkv, 128));
  if (nkb > sparvar::kMaxMassBlocks)
    return fail(SPARVAR_ERR_UNSUPPORTED, "Lkv=%d gives %d KV blocks (max %d)", Lkv, nkb,
                sparvar::kMaxMassBlocks);
  int rc;
  if ((rc = check_operand(q, q_strides, B, H, Lq, D, "q"))) return rc;
  if ((rc = check_operand(k, k_strides, B, H, Lkv, D, "k"))) return rc;
  if (!kv_cnt || !kv_idx) return fail(SPARVAR_ERR_INVALID_ARG, "kv_cnt/kv_idx is NULL");
  if (!std::isfinite(softmax_scale) || !(softmax_scale > 0.f) || std::isnan(mass_threshold))
    return fail(SPARVAR_ERR_INVALID_ARG, "softmax_scale must be finite and > 0, mass_threshold a number");
  if (!(topk_ratio >= 0.f && topk_ratio <= 1.f))
    return fail(SPARVAR_ERR_INVALID_ARG, "topk_ratio must be in [0, 1] (0: mass threshold)");

  sparvar::DecideArgs a{};
  a.B = B; a.H = H; a.Lq = Lq; a.Lkv = Lkv;
  a.nqb = static_cast<int>(ceil_div(Lq, 128));
  a.nkb = nkb;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  a.lse_in = lse;
  a.mass_threshold = mass_threshold;
  // k = ceil(ratio * NKB), at least one; the allowance keeps 0.2f * 20 at 4
  a.topk = topk_ratio > 0.f
               ? static_cast<int>(std::min<double>(
                     nkb, std::max<double>(1.0, std::ceil(static_cast<double>(topk_ratio) * nkb - 1e-6))))
               : 0;
  a.sel_cnt = kv_cnt; a.sel_idx = kv_idx; a.mass_out = mass;
  a.dev_status = dev_status;
  CUtensorMap tq, tk;
  if ((rc = make_tmap(&tq, q, D, Lq, H, B, q_strides[2], q_strides[1], q_strides[0], "q"))) return rc;
  if ((rc = make_tmap(&tk, k, D, Lkv, H, B, k_strides[2], k_strides[1], k_strides[0], "k"))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (D == 128) return launch_decide_kernel<128>(tq, tk, a, st);
  return launch_decide_kernel<64>(tq, tk, a, st);
}

int sparvar_decision_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                              int B, int H, int Lq, int Lkv, int D, const int64_t* q_strides,
                              const int64_t* k_strides, const int64_t* v_strides,
                              const int64_t* o_strides, float softmax_scale, float mass_threshold,
                              float topk_ratio, int32_t* kv_cnt, int32_t* kv_idx, float* mass,
                              int32_t* dev_status, void* stream) {
  if (D != 64 && D != 128) return fail(SPARVAR_ERR_UNSUPPORTED, "D=%d not in {64, 128}", D);
  if (B < 1 || H < 1 || B > 65535 || H > 65535)
    return fail(SPARVAR_ERR_INVALID_ARG, "B=%d H=%d outside [1, 65535]", B, H);
  if (Lq < 1 || Lkv < 1 || Lq > (1 << 30) || Lkv > (1 << 30))
    return fail(SPARVAR_ERR_INVALID_ARG, "Lq=%d Lkv=%d outside [1, 2^30]", Lq, Lkv);
  const int nkb = static_cast<int>(ceil_div(Lkv, 128));
  if (nkb > sparvar::dec::kMaxDecBlocks)
    return fail(SPARVAR_ERR_UNSUPPORTED, "Lkv=%d gives %d KV blocks (max %d)", Lkv, nkb,
                sparvar::dec::kMaxDecBlocks);
  if (static_cast<int64_t>(B) * H * ceil_div(Lq, 128) > (int64_t{1} << 30))
    return fail(SPARVAR_ERR_UNSUPPORTED, "B*H*ceil(Lq/128) above 2^30 query tiles");
  int rc;
  if ((rc = check_operand(q, q_strides, B, H, Lq, D, "q"))) return rc;
  if ((rc = check_operand(k, k_strides, B, H, Lkv, D, "k"))) return rc;
  if ((rc = check_operand(v, v_strides, B, H, Lkv, D, "v"))) return rc;
  if ((rc = check_operand(o, o_strides, B, H, Lq, D, "o"))) return rc;
  if (!kv_cnt || !kv_idx) return fail(SPARVAR_ERR_INVALID_ARG, "kv_cnt/kv_idx is NULL");
  if (!std::isfinite(softmax_scale) || !(softmax_scale > 0.f) || std::isnan(mass_threshold))
    return fail(SPARVAR_ERR_INVALID_ARG,
                "softmax_scale must be finite and > 0, mass_threshold a number");
  if (!(topk_ratio >= 0.f && topk_ratio <= 1.f))
    return fail(SPARVAR_ERR_INVALID_ARG, "topk_ratio must be in [0, 1] (0: mass threshold)");

  sparvar::dec::Args a{};
  a.B = B; a.H = H; a.Lq = Lq; a.Lkv = Lkv;
  a.nqb = static_cast<int>(ceil_div(Lq, 128));
  a.nkb = nkb;
  a.total_pairs = static_cast<int>(static_cast<int64_t>(B) * H * ((a.nqb + 1) / 2));
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.o_sb = o_strides[0]; a.o_sh = o_strides[1]; a.o_sr = o_strides[2];
  a.lse = lse;
  a.dev_status = dev_status;
  a.mass_out = mass;
  a.mass_threshold = mass_threshold;
  // k = ceil(ratio * NKB), at least one; the allowance keeps 0.2f * 20 at 4
  a.topk = topk_ratio > 0.f
               ? static_cast<int>(std::min<double>(
                     nkb, std::max<double>(1.0, std::ceil(static_cast<double>(topk_ratio) * nkb - 1e-6))))
               : 0;
  a.sel_cnt = kv_cnt;
  a.sel_idx = kv_idx;
  CUtensorMap tq, tk, tv, to;
  if ((rc = make_tmap(&tq, q, D, Lq, H, B, q_strides[2], q_strides[1], q_strides[0], "q"))) return rc;
  if ((rc = make_tmap(&tk, k, D, Lkv, H, B, k_strides[2], k_strides[1], k_strides[0], "k"))) return rc;
  if ((rc = make_tmap(&tv, v, D, Lkv, H, B, v_strides[2], v_strides[1], v_strides[0], "v"))) return rc;
  if ((rc = make_tmap(&to, o, D, Lq, H, B, o_strides[2], o_strides[1], o_strides[0], "o",
                      sparvar::dec::kOutBoxRows)))
    return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (D == 128) return launch_decision_kernel<128>(tq, tk, tv, to, a, st);
  return launch_decision_kernel<64>(tq, tk, tv, to, a, st);
}

int sparvar_ocache_apply(const void* o_target, const void* o_dense, const void* o_sparse, void* out,
                         int B, int H, int side_src, int side_dst, int D,
                         const int64_t* t_strides, const int64_t* d_strides,
                         const int64_t* s_strides, const int64_t* out_strides, void* stream) {
  if (B < 1 || H < 1 || B > 65535 || H > 65535)
    return fail(SPARVAR_ERR_INVALID_ARG, "B=%d H=%d outside [1, 65535]", B, H);
  if (side_src < 1 || side_dst < 1 || side_src > 46340 || side_dst > 46340)
    return fail(SPARVAR_ERR_INVALID_ARG, "sides %d, %d outside [1, 46340]", side_src, side_dst);
  if (D < 8 || D > 1024 || D % 8 != 0)
    return fail(SPARVAR_ERR_UNSUPPORTED, "D=%d: a multiple of 8 in [8, 1024]", D);
  const int n_src = side_src * side_src, n_dst = side_dst * side_dst;
  int rc;
  if ((rc = check_operand(o_target, t_strides, B, H, n_dst, D, "o_target"))) return rc;
  if ((rc = check_operand(o_dense, d_strides, B, H, n_src, D, "o_dense"))) return rc;
  if ((rc = check_operand(o_sparse, s_strides, B, H, n_src, D, "o_sparse"))) return rc;
  if ((rc = check_operand(out, out_strides, B, H, n_dst, D, "out"))) return rc;
  sparvar::OcacheArgs a{};
  a.o_t = static_cast<const __nv_bfloat16*>(o_target);
  a.o_d = static_cast<const __nv_bfloat16*>(o_dense);
  a.o_s = static_cast<const __nv_bfloat16*>(o_sparse);
  a.out = static_cast<__nv_bfloat16*>(out);
  a.B = B; a.H = H; a.s_src = side_src; a.s_dst = side_dst; a.D = D;
  a.t_sb = t_strides[0]; a.t_sh = t_strides[1]; a.t_sr = t_strides[2];
  a.d_sb = d_strides[0]; a.d_sh = d_strides[1]; a.d_sr = d_strides[2];
  a.s_sb = s_strides[0]; a.s_sh = s_strides[1]; a.s_sr = s_strides[2];
  a.u_sb = out_strides[0]; a.u_sh = out_strides[1]; a.u_sr = out_strides[2];
  // one CTA per target row of one (batch, head): D / 8 threads across the channels,
  // up to 256 / (D / 8) tokens of the row at a time
  const int vecs = D / 8;
  const int ty = std::max(1, std::min(256 / vecs, side_dst));
  sparvar::ocache_apply_kernel<<<dim3(side_dst, H, B), dim3(vecs, ty), 0,
                                 static_cast<cudaStream_t>(stream)>>>(a);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "ocache_apply_kernel launch");
  return SPARVAR_OK;
}

int sparvar_block_sparse_attn_fwd_static(
    const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Lq,
    int Lkv, int D, const int64_t* q_strides, const int64_t* k_strides, const int64_t* v_strides,
    const int64_t* o_strides, const int32_t* kv_cnt, const int32_t* kv_idx,
    const int64_t* list_strides, int idx_row_len, int block, float softmax_scale,
    int32_t* dev_status, void* stream) {
  if (block != 16 && block != 32 && block != 64)
    return fail(SPARVAR_ERR_UNSUPPORTED, "block=%d not in {16, 32, 64}", block);
  if (B < 1 || H < 1 || B > 65535 || H > 65535)
    return fail(SPARVAR_ERR_INVALID_ARG, "B=%d H=%d outside [1, 65535]", B, H);
  if (Lq < 1 || Lkv < 1 || Lq > (1 << 30) || Lkv > (1 << 30))
    return fail(SPARVAR_ERR_INVALID_ARG, "Lq=%d Lkv=%d outside [1, 2^30]", Lq, Lkv);
  if (!list_strides) return fail(SPARVAR_ERR_INVALID_ARG, "list_strides is NULL");
  if (list_strides[0] < 0 || list_strides[1] < 0)
    return fail(SPARVAR_ERR_INVALID_ARG, "list strides must be >= 0");
  if (idx_row_len < 0) return fail(SPARVAR_ERR_INVALID_ARG, "idx_row_len < 0");
  if (ceil_div(Lkv, 128) > 4096)
    return fail(SPARVAR_ERR_UNSUPPORTED, "Lkv=%d gives more than 4096 KV tiles", Lkv);
  // tile counts, tile lists and tile masks, each 256-byte aligned, as sparvar_coarsen_lists
  // writes them
  const int64_t Bo = list_strides[0] == 0 ? 1 : B, Ho = list_strides[1] == 0 ? 1 : H;
  const int64_t nqt = ceil_div(Lq, 128), nkt = ceil_div(Lkv, 128);
  const int64_t rows = Bo * Ho * nqt;
  auto up = [](int64_t x) { return (x + 255) / 256 * 256; };
  const int64_t cnt_bytes = up(rows * 4), idx_bytes = up(rows * nkt * 4);
  const int64_t need = cnt_bytes + idx_bytes + up(rows * nkt * 8);
  if (need > static_cast<int64_t>(kStaticScratchBytes))
    return fail(SPARVAR_ERR_UNSUPPORTED,
                "tile lists need %lld bytes, the static scratch holds %zu",
                static_cast<long long>(need), kStaticScratchBytes);
  const int64_t t_strides[2] = {Bo > 1 ? Ho * nqt : 0, Ho > 1 ? nqt : 0};
  // every argument of the attention launch is checked (on the host) before the scratch
  // is looked up or the coarsening enqueued, so a refused call touches neither the
  // scratch nor dev_status; the tile-list pointers are filled in afterwards
  FwdLaunch L;
  int rc = attn_fwd_prepare(&L, q, k, v, o, lse, B, H, Lq, Lkv, D, q_strides, k_strides,
                            v_strides, o_strides, kv_cnt, kv_idx, t_strides,
                            static_cast<int>(nkt), reinterpret_cast<const uint64_t*>(kv_idx),
                            block, 128, 128, softmax_scale, dev_status, nullptr);
  if (rc) return rc;
  void* base = nullptr;
  rc = static_scratch_address(&base);
  if (rc) return rc;
  uint8_t* p = static_cast<uint8_t*>(base);
  int32_t* t_cnt = reinterpret_cast<int32_t*>(p);
  int32_t* t_idx = reinterpret_cast<int32_t*>(p + cnt_bytes);
  uint64_t* t_mask = reinterpret_cast<uint64_t*>(p + cnt_bytes + idx_bytes);
  L.a.prob[0].kv_cnt = t_cnt;
  L.a.prob[0].kv_idx = t_idx;
  L.a.tile_mask = t_mask;
  rc = sparvar_coarsen_lists(kv_cnt, kv_idx, list_strides, idx_row_len, B, H, Lq, Lkv, block,
                             t_cnt, t_idx, t_mask, dev_status, stream);
  if (rc) return rc;
  return attn_fwd_launch(L, stream);
}

}  // extern "C"
