// ig4_api.cu - C ABI of the Ideogram 4 DiT block library (see include/ig4.h).
//
// Host side: argument validation (before anything is launched), TMA
// descriptor encoding, the workspace layout, and the launch sequence of the
// block and of the stack on the caller's stream.  The device code lives in
// the ig4_*.cuh headers.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <utility>

#include "ig4.h"
#include "ig4_attention.cuh"
#include "ig4_gemm.cuh"
#include "ig4_mx8.cuh"
#include "ig4_nvf4.cuh"
#include "ig4_parallel.cuh"
#include "ig4_small.cuh"

using namespace ig4;

namespace {

constexpr int ABI_VERSION = 2;

// ------------------------------------------------------------------ utils

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
inline cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

// Launch with programmatic stream serialization: the kernel may be scheduled
// while the previous kernel on the stream drains; every kernel launched this
// way waits (griddepcontrol.wait, pdl_wait()) before touching global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args &&...args) {
  cudaLaunchConfig_t lc = {};
  lc.gridDim = grid;
  lc.blockDim = block;
  lc.dynamicSmemBytes = smem;
  lc.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  return cudaLaunchKernelEx(&lc, kern, std::forward<Args>(args)...);
}

// Inverse of the standard normal CDF Phi(x) = erfc(-x / sqrt 2) / 2 for
// 0 < p < 1, by bisection (Phi is monotone; 200 halvings reach the spacing of
// doubles), +-infinity at p = 1 and p = 0.  The upper half uses the symmetry
// Phi^-1(p) = -Phi^-1(1 - p), so the bisection always works in the lower
// tail, where erfc keeps full relative precision.
inline double normal_quantile(double p) {
  if (p <= 0.0) return -INFINITY;
  if (p >= 1.0) return INFINITY;
  if (p > 0.5) return -normal_quantile(1.0 - p);
  double lo = -40.0, hi = 0.0;
  for (int it = 0; it < 200; ++it) {
    const double mid = 0.5 * (lo + hi);
    if (mid == lo || mid == hi) break;
    if (0.5 * std::erfc(-mid / std::sqrt(2.0)) < p)
      lo = mid;
    else
      hi = mid;
  }
  return 0.5 * (lo + hi);
}

ig4_status last_launch_status() {
  return cudaGetLastError() == cudaSuccess ? IG4_OK : IG4_ERR_CUDA;
}

#define IG4_TRY(expr)                       \
  do {                                      \
    const ig4_status st_ = (expr);          \
    if (st_ != IG4_OK) return st_;          \
  } while (0)

// Per-device facts queried once.
struct DeviceInfo {
  int sms = 0;
};
constexpr int MAX_DEVICES = 64;
DeviceInfo g_dev[MAX_DEVICES];
std::mutex g_dev_mu;

ig4_status device_info(DeviceInfo **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return IG4_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (g_dev[dev].sms == 0) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return IG4_ERR_CUDA;
    g_dev[dev].sms = sms;
  }
  *out = &g_dev[dev];
  return IG4_OK;
}

// Raise a kernel's dynamic shared-memory limit (idempotent, cheap).
template <typename K>
ig4_status allow_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) ==
                 cudaSuccess
             ? IG4_OK
             : IG4_ERR_CUDA;
}

// --------------------------------------------------------- tensor maps

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Row-major matrix [rows][cols] of esize-byte elements (row stride ld
// elements), box [box_rows][box_cols] with box_cols * esize == 128 bytes.
ig4_status map_2d(CUtensorMap *m, const void *base, int esize, long rows, long cols, long ld,
                  int box_rows, int box_cols) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return IG4_ERR_CUDA;
  const CUtensorMapDataType dt =
      esize == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * esize};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? IG4_OK : IG4_ERR_CUDA;
}

// bf16 tensor [d2][d1][d0] (d0 contiguous, row stride ld0 elements, plane
// stride ld1 elements), box [1][b1][b0], b0 * 2 == 128 bytes.
ig4_status map_3d_bf16(CUtensorMap *m, const void *base, long d0, long d1, long d2, long ld0,
                       long ld1, int b0, int b1) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return IG4_ERR_CUDA;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d0), static_cast<cuuint64_t>(d1),
                        static_cast<cuuint64_t>(d2)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(ld0) * 2, static_cast<cuuint64_t>(ld1) * 2};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(b0), static_cast<cuuint32_t>(b1), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? IG4_OK : IG4_ERR_CUDA;
}

// -------------------------------------------------------------- GEMMs

// 256- and 192-wide tiles over more than one 128-row block run on CTA pairs
// (M = 256 per pair tile, B rows split between the two CTAs); the B tensor
// map's box is then BN / 2 rows.
inline bool use_pair(int BN, int M) { return (BN == 256 || BN == 240 || BN == 192) && M > GEMM_BM; }
inline int b_box_rows(int BN, int M) { return use_pair(BN, M) ? BN / 2 : BN; }

// Tile order of the persistent GEMMs: plain m-fastest while A fits easily in
// L2 (the 126 MB L2 then serves every re-read of A), groups of 10 m tiles
// once A is larger, so that consecutive rounds of pair tiles share A rows
// (which the pair kernel's K-snake then finds in L2).  DRAM reads of the
// 1024 px down-projection (A = 113 MB, 240-wide pair tiles), ncu: groups of
// 4 m tiles 634 MB, 6 576 MB, 8 610 MB, 10 542 MB, 12 570 MB, m-fastest 578
// MB (with 256-wide tiles, groups of 12: 536 MB; 649 MB for groups of 8
// before the K-snake); times within 1%, and the other GEMMs of the block
// moved by less than 1%.
inline int gemm_group_m(long M, long K, int esize) {
  return M * K * esize <= (64L << 20) ? (1 << 30) : 10;
}

template <int BN, bool FP8, bool DUAL_B, class Epi>
ig4_status launch_gemm(const CUtensorMap &A, const CUtensorMap &B, const CUtensorMap &B2, int M,
                       int n_tiles_n, int K, const Epi &epi, cudaStream_t st) {
  DeviceInfo *di = nullptr;
  IG4_TRY(device_info(&di));
  const int group_m = gemm_group_m(M, K, FP8 ? 1 : 2);
  if constexpr (BN == 256 || BN == 240 || BN == 192) {
    if (use_pair(BN, M)) {
      auto kern = gemm_pair_kernel<BN, FP8, DUAL_B, Epi>;
      constexpr int PAIR_SMEM_BYTES = PairShape<BN>::SMEM_BYTES;
      IG4_TRY(allow_smem(kern, PAIR_SMEM_BYTES));
      const long tiles = static_cast<long>((M + 2 * GEMM_BM - 1) / (2 * GEMM_BM)) * n_tiles_n;
      const int pairs = static_cast<int>(std::min<long>(tiles, di->sms / 2));
      cudaLaunchConfig_t lc = {};
      lc.gridDim = dim3(2 * pairs);
      lc.blockDim = dim3(GEMM_THREADS);
      lc.dynamicSmemBytes = PAIR_SMEM_BYTES;
      lc.stream = st;
      cudaLaunchAttribute attr[2];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[1].val.programmaticStreamSerializationAllowed = 1;
      lc.attrs = attr;
      lc.numAttrs = 2;
      if (cudaLaunchKernelEx(&lc, kern, A, B, B2, M, n_tiles_n, K, group_m, epi) != cudaSuccess)
        return IG4_ERR_CUDA;
      return last_launch_status();
    }
  }
  if constexpr (BN == 240) {
    return IG4_ERR_UNSUPPORTED;  // 240-wide tiles run on CTA pairs only
  } else {
  auto kern = gemm_tc_kernel<BN, FP8, DUAL_B, Epi>;
  constexpr int SMEM = GemmShape<BN>::SMEM_BYTES;
  IG4_TRY(allow_smem(kern, SMEM));
  const long tiles = static_cast<long>((M + GEMM_BM - 1) / GEMM_BM) * n_tiles_n;
  const int grid = static_cast<int>(std::min<long>(tiles, di->sms));
  if (launch_pdl(kern, dim3(grid), dim3(GEMM_THREADS), SMEM, st, A, B, B2, M, n_tiles_n, K,
                 group_m, epi) != cudaSuccess)
    return IG4_ERR_CUDA;
  return last_launch_status();
  }
}

// A [M][K] and W [N][K] maps for one GEMM (esize 2 = bf16, 1 = e4m3).
ig4_status gemm_maps(CUtensorMap *ma, CUtensorMap *mb, const void *a, const void *w, int esize,
                     long M, long N, long K, int b_rows) {
  const int bk = 128 / esize;
  IG4_TRY(map_2d(ma, a, esize, M, K, K, GEMM_BM, bk));
  IG4_TRY(map_2d(mb, w, esize, N, K, K, b_rows, bk));
  return IG4_OK;
}

// E4M3 linears (all of them, or all but the NVFP4 FFN of the mixed format)
bool is_fp8(int dt) { return dt == IG4_E4M3 || dt == IG4_NVFP4_MIXED; }
bool is_nvf4_mixed(int dt) { return dt == IG4_NVFP4_MIXED; }

// ------------------------------------------------------------ validation

bool valid_dtype_x(int d) { return d == IG4_F32 || d == IG4_BF16; }
bool valid_dtype_w(int d) { return d == IG4_BF16 || d == IG4_E4M3; }

ig4_status check_config(const ig4_config *c) {
  if (!c) return IG4_ERR_INVALID_ARG;
  if (c->B < 1 || c->T_text < 0 || c->grid_t < 0 || c->grid_h < 0 || c->grid_w < 0)
    return IG4_ERR_INVALID_ARG;
  const long L = static_cast<long>(c->T_text) + static_cast<long>(c->grid_t) * c->grid_h * c->grid_w;
  if (L < 1 || L > (1L << 24)) return IG4_ERR_INVALID_ARG;
  if (static_cast<long>(c->B) * L > (1L << 26)) return IG4_ERR_UNSUPPORTED;
  if (c->H < 1 || c->D < 1 || c->I < 1 || c->adaln_dim < 1) return IG4_ERR_INVALID_ARG;
  if (c->sections[0] < 0 || c->sections[1] < 0 || c->sections[2] < 0 ||
      c->sections[0] + c->sections[1] + c->sections[2] != 64)
    return IG4_ERR_INVALID_ARG;
  if (!(c->rope_theta > 0.0) || !(c->eps > 0.0f)) return IG4_ERR_INVALID_ARG;
  if (!valid_dtype_x(c->x_dtype) || !(valid_dtype_w(c->w_dtype) || is_nvf4_mixed(c->w_dtype)))
    return IG4_ERR_INVALID_ARG;
  if (c->head_dim != 256 || c->D != 256 * c->H) return IG4_ERR_UNSUPPORTED;
  // the NVFP4 FFN runs on CTA pairs with K-steps of 256
  if (is_nvf4_mixed(c->w_dtype) && (c->I % 256 != 0 || static_cast<long>(c->B) * L <= 128))
    return IG4_ERR_UNSUPPORTED;
  if (c->D > 6144) return IG4_ERR_UNSUPPORTED;
  if (c->I % 128 != 0) return IG4_ERR_UNSUPPORTED;
  if (c->adaln_dim % 16 != 0 || c->adaln_dim > 1024 || c->B > 8) return IG4_ERR_UNSUPPORTED;
  return IG4_OK;
}

// ------------------------------------------------------------- launchers

ig4_status launch_adaln(int B, int A, int N, const float *temb, const void *w, int w_dtype,
                        const float *w_scale, const float *bias, float *mod, cudaStream_t st) {
  const int rows_per_cta = (ADALN_THREADS / 32) * ADALN_ROWS_PER_WARP;
  const int grid = (N + rows_per_cta - 1) / rows_per_cta;
  const int smem = B * A * 4;
  const bool f8 = is_fp8(w_dtype);
  const int mv = (A * (f8 ? 1 : 2) + 511) / 512;  // 16-byte vectors per lane and row
  cudaError_t e;
  if (f8)
    e = mv <= 1 ? launch_pdl(adaln_kernel<true, 1>, dim3(grid), dim3(ADALN_THREADS), smem, st,
                             temb, w, w_scale, bias, mod, B, A, N)
                : launch_pdl(adaln_kernel<true, 2>, dim3(grid), dim3(ADALN_THREADS), smem, st,
                             temb, w, w_scale, bias, mod, B, A, N);
  else
    e = mv <= 2 ? launch_pdl(adaln_kernel<false, 2>, dim3(grid), dim3(ADALN_THREADS), smem, st,
                             temb, w, w_scale, bias, mod, B, A, N)
                : launch_pdl(adaln_kernel<false, 4>, dim3(grid), dim3(ADALN_THREADS), smem, st,
                             temb, w, w_scale, bias, mod, B, A, N);
  if (e != cudaSuccess) return IG4_ERR_CUDA;
  return last_launch_status();
}

template <typename XT, bool FP8>
ig4_status launch_norm_t(int rows, int L, int D, const void *x, const float *shift,
                         const float *scale, int mod_stride, float eps, void *h, float *hs,
                         int remap_n, int remap_L, int remap_off, cudaStream_t st) {
  DeviceInfo *di = nullptr;
  IG4_TRY(device_info(&di));
  // rows of one sample, and samples; one chunk of rows per CTA, about one CTA per SM
  const int nb = remap_n > 0 ? remap_n : L;
  const int B = rows / nb;
  if (B < 1 || B * nb != rows) return IG4_ERR_INVALID_ARG;
  const long per_cta = (static_cast<long>(rows) + di->sms - 1) / di->sms;
  const int rows_per_cta =
      static_cast<int>(std::max<long>(NORM_WARPS, (per_cta + NORM_WARPS - 1) / NORM_WARPS * NORM_WARPS));
  const dim3 grid((nb + rows_per_cta - 1) / rows_per_cta, B);
  const size_t smem = 2ull * D * sizeof(float);
  if (smem > 48 * 1024) return IG4_ERR_UNSUPPORTED;
  const int nv = (D / 8 + 31) / 32;
  const XT *xp = static_cast<const XT *>(x);
  if constexpr (sizeof(XT) == 2) {
    // bf16 stream up to D = 4608: 16 warps per CTA, a row per warp
    const long per_cta2 = (static_cast<long>(rows) + di->sms - 1) / di->sms;
    const int rpc2 = static_cast<int>(std::max<long>(NORM2_WARPS, per_cta2));
    const dim3 grid2((nb + rpc2 - 1) / rpc2, B);
    const size_t smem2 = norm2_smem_bytes(D);
#define IG4_NORM2_CASE(NV)                                                                      \
  if (nv <= NV) {                                                                              \
    IG4_TRY(allow_smem(norm_modulate_rows_kernel<FP8, NV>, static_cast<int>(smem2)));          \
    if (launch_pdl(norm_modulate_rows_kernel<FP8, NV>, grid2, dim3(NORM2_THREADS), smem2, st,  \
                   xp, shift, scale, mod_stride, L, D, eps, h, hs, remap_n, remap_L,           \
                   remap_off, rpc2) != cudaSuccess)                                            \
      return IG4_ERR_CUDA;                                                                     \
    return last_launch_status();                                                               \
  }
    IG4_NORM2_CASE(2)
    IG4_NORM2_CASE(4)
    IG4_NORM2_CASE(8)
    IG4_NORM2_CASE(12)
    IG4_NORM2_CASE(18)
#undef IG4_NORM2_CASE
  }
#define IG4_NORM_CASE(NV)                                                                        \
  if (nv <= NV) {                                                                                \
    if (launch_pdl(norm_modulate_kernel<XT, FP8, NV>, grid, dim3(NORM_THREADS), smem, st, xp,   \
                   shift, scale, mod_stride, L, D, eps, h, hs, remap_n, remap_L, remap_off,     \
                   rows_per_cta) != cudaSuccess)                                                 \
      return IG4_ERR_CUDA;                                                                       \
    return last_launch_status();                                                                 \
  }
  IG4_NORM_CASE(2)
  IG4_NORM_CASE(4)
  IG4_NORM_CASE(8)
  IG4_NORM_CASE(12)
  IG4_NORM_CASE(18)
  IG4_NORM_CASE(24)
#undef IG4_NORM_CASE
  return IG4_ERR_UNSUPPORTED;
}

ig4_status launch_norm(int rows, int L, int D, const void *x, int x_dtype, const float *shift,
                       const float *scale, int mod_stride, float eps, void *h, int h_dtype,
                       float *hs, int remap_n, int remap_L, int remap_off, cudaStream_t st) {
  const bool f8 = is_fp8(h_dtype);
  if (x_dtype == IG4_F32)
    return f8 ? launch_norm_t<float, true>(rows, L, D, x, shift, scale, mod_stride, eps, h, hs,
                                           remap_n, remap_L, remap_off, st)
              : launch_norm_t<float, false>(rows, L, D, x, shift, scale, mod_stride, eps, h, hs,
                                            remap_n, remap_L, remap_off, st);
  return f8 ? launch_norm_t<__nv_bfloat16, true>(rows, L, D, x, shift, scale, mod_stride, eps, h,
                                                 hs, remap_n, remap_L, remap_off, st)
            : launch_norm_t<__nv_bfloat16, false>(rows, L, D, x, shift, scale, mod_stride, eps, h,
                                                  hs, remap_n, remap_L, remap_off, st);
}

ig4_status launch_rope_table(int L, const int32_t *pos, double theta, const int sec[3], float *c,
                             float *s, cudaStream_t st) {
  const int n = L * 64;
  if (launch_pdl(rope_table_kernel, dim3((n + 255) / 256), dim3(256), 0, st, pos, L, theta, sec[0],
                 sec[1], c, s) != cudaSuccess)
    return IG4_ERR_CUDA;
  return last_launch_status();
}

ig4_status launch_quantize(int M, int K, const void *x, void *q, float *scale, cudaStream_t st) {
  const int nv = (K / 8 + QUANT_THREADS - 1) / QUANT_THREADS;
  const __nv_bfloat16 *xp = static_cast<const __nv_bfloat16 *>(x);
  uint8_t *qp = static_cast<uint8_t *>(q);
#define IG4_Q_CASE(NV)                                                                   \
  if (nv <= NV) {                                                                        \
    if (launch_pdl(quantize_rows_kernel<NV>, dim3(M), dim3(QUANT_THREADS), 0, st, xp, qp,  \
                   scale, K) != cudaSuccess)                                             \
      return IG4_ERR_CUDA;                                                               \
    return last_launch_status();                                                         \
  }
  IG4_Q_CASE(1)
  IG4_Q_CASE(2)
  IG4_Q_CASE(4)
  IG4_Q_CASE(6)
  IG4_Q_CASE(8)
#undef IG4_Q_CASE
  return IG4_ERR_UNSUPPORTED;
}

// q, k, v of H heads (3 * 256 * H weight rows) from h [B*L][D]; a
// tensor-parallel shard passes its own head count.
ig4_status launch_qkv(int B, int L, int D, int H, const void *h, int h_dtype, const float *h_scale,
                      const void *w, const float *w_scale, const float *g_q, const float *g_k,
                      float eps, const float *cs, const float *sn, void *q, void *k, void *vt,
                      int vt_ld, cudaStream_t st) {
  const int M = B * L;
  const bool f8 = is_fp8(h_dtype);
  const int esize = f8 ? 1 : 2;
  CUtensorMap ma, mb;
  IG4_TRY(gemm_maps(&ma, &mb, h, w, esize, M, 3L * 256 * H, D, b_box_rows(256, M)));
  const int ntn = 3 * H;
  if (f8) {
    EpiQKV<true> e{static_cast<__nv_bfloat16 *>(q), static_cast<__nv_bfloat16 *>(k),
                   static_cast<__nv_bfloat16 *>(vt), vt_ld, L, H, M, g_q, g_k, eps, cs, sn,
                   h_scale, w_scale};
    return launch_gemm<256, true, false>(ma, mb, mb, M, ntn, D, e, st);
  }
  EpiQKV<false> e{static_cast<__nv_bfloat16 *>(q), static_cast<__nv_bfloat16 *>(k),
                  static_cast<__nv_bfloat16 *>(vt), vt_ld, L, H, M, g_q, g_k, eps, cs, sn,
                  nullptr, nullptr};
  return launch_gemm<256, false, false>(ma, mb, mb, M, ntn, D, e, st);
}

// The attention kernel's launch.  With two or more query tiles the kernel
// runs on CTA pairs (an item is two query tiles of one (b, h)), else on
// single CTAs (an item is the one query tile).  Workers (pairs or CTAs): one
// per item when there are no more items than workers fit on the device (or
// no partial slots), else one per SM (pair) taking the items round-robin,
// with the last partial round's items split into pieces of key tiles (the
// kernel's AttSched).
struct AttPlan {
  bool pair;
  long items;
  int workers;  // pairs or CTAs
  int split;    // tail items split into pieces (0: none)
};
AttPlan att_plan(int B, int H, int L, int sms, bool have_part) {
  AttPlan p{};
  const int nkv = (L + ATT_BN - 1) / ATT_BN;
  p.pair = nkv >= 2;
  const int ctas = p.pair ? 2 : 1;
  p.items = static_cast<long>(B) * H * (p.pair ? (nkv + 1) / 2 : nkv);
  const int g = std::max(1, std::min(sms, ATT_MAX_CTAS) / ctas);
  p.workers = (!have_part || p.items <= g) ? static_cast<int>(p.items) : g;
  const long rem = p.items % p.workers;
  const long k = rem ? std::max<long>(1, std::min<long>(nkv, p.workers / rem)) : 1;
  p.split = k > 1 ? static_cast<int>(rem) : 0;
  return p;
}
// Bytes of partial slots the grid may need: one per CTA (0 when no item can
// be split: a single key tile per item).
size_t att_part_bytes(int B, int H, int L) {
  const long nkv = (L + ATT_BN - 1) / ATT_BN;
  if (nkv <= 1 || static_cast<long>(B) * H * nkv <= 1) return 0;
  return static_cast<size_t>(ATT_MAX_CTAS) * ATT_PART_BYTES;
}

// part: att_part_bytes(B, H, L) bytes of workspace for the balanced grid, or
// nullptr (one worker per item).  o_sf != nullptr: o receives MX8 (E4M3
// codes [B*L][H*256] and the packed scales in o_sf) instead of bf16.
ig4_status launch_attention(int B, int H, int L, const void *q, const void *k, const void *vt,
                            int vt_ld, void *o, void *part, cudaStream_t st,
                            void *o_sf = nullptr) {
  DeviceInfo *di = nullptr;
  IG4_TRY(device_info(&di));
  const long BH = static_cast<long>(B) * H;
  const bool have_part = part != nullptr && att_part_bytes(B, H, L) > 0;
  const AttPlan plan = att_plan(B, H, L, di->sms, have_part);
  if (BH > (1L << 30) || plan.items > (1L << 29)) return IG4_ERR_UNSUPPORTED;
  CUtensorMap mq, mk, mv;
  IG4_TRY(map_3d_bf16(&mq, q, 256, L, BH, 256, static_cast<long>(L) * 256, 64, ATT_BM));
  // K boxes: 64 head dims (128 bytes, the swizzle span) x the keys one CTA
  // loads per tile (all 128, or its 64 of a pair's tile).  V^T boxes: 64 keys
  // x the head dims one CTA loads (all 256, or its 128 of a pair's).
  IG4_TRY(map_3d_bf16(&mk, k, 256, L, BH, 256, static_cast<long>(L) * 256, 64,
                      plan.pair ? ATT_BN / 2 : ATT_BN));
  IG4_TRY(map_3d_bf16(&mv, vt, L, 256, BH, vt_ld, 256L * vt_ld, 64,
                      plan.pair ? ATT_DH / 2 : ATT_DH));
  __nv_bfloat16 *op = static_cast<__nv_bfloat16 *>(o);
  uint8_t *pp = static_cast<uint8_t *>(part);
  if (plan.pair) {
    IG4_TRY(allow_smem(attention_kernel<true>, ATT_SMEM_BYTES));
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(2 * plan.workers);
    lc.blockDim = dim3(ATT_THREADS);
    lc.dynamicSmemBytes = ATT_SMEM_BYTES;
    lc.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = attr;
    lc.numAttrs = 2;
    if (cudaLaunchKernelEx(&lc, attention_kernel<true>, mq, mk, mv, op, L, H,
                           static_cast<int>(BH), pp, static_cast<uint8_t *>(o_sf)) != cudaSuccess)
      return IG4_ERR_CUDA;
  } else {
    IG4_TRY(allow_smem(attention_kernel<false>, ATT_SMEM_BYTES));
    if (launch_pdl(attention_kernel<false>, dim3(plan.workers), dim3(ATT_THREADS),
                   ATT_SMEM_BYTES, st, mq, mk, mv, op, L, H, static_cast<int>(BH), pp,
                   static_cast<uint8_t *>(o_sf)) != cudaSuccess)
      return IG4_ERR_CUDA;
  }
  IG4_TRY(last_launch_status());
  if (plan.split > 0) {
    // merge the pieces of the split tail items
    const int rows = (plan.pair ? 2 : 1) * ATT_BM;
    const dim3 grid(plan.split, rows / ATT_COMBINE_ROWS);
    const cudaError_t e =
        plan.pair ? launch_pdl(attention_combine_kernel<true>, grid, dim3(ATT_COMBINE_THREADS), 0,
                               st, static_cast<const uint8_t *>(pp), op, L, H,
                               static_cast<int>(BH), plan.workers, static_cast<uint8_t *>(o_sf))
                  : launch_pdl(attention_combine_kernel<false>, grid, dim3(ATT_COMBINE_THREADS),
                               0, st, static_cast<const uint8_t *>(pp), op, L, H,
                               static_cast<int>(BH), plan.workers, static_cast<uint8_t *>(o_sf));
    if (e != cudaSuccess) return IG4_ERR_CUDA;
    IG4_TRY(last_launch_status());
  }
  return IG4_OK;
}

// Tile width for an output of N columns: the candidate with the best product
// of wave efficiency (tiles / (waves * workers), where a worker is a CTA pair
// for the 256-, 240- and 192-wide tiles over more than 128 rows and a single
// CTA otherwise), useful columns (240-wide tiles need not divide N: the last
// one is partial) and per-tile MMA efficiency.  Single-CTA 192- and 128-wide
// tiles read more shared memory per flop (measured on the 4608 x 4608 x 4608
// out-projection, single-CTA 192-wide tiles ran 10% slower per tile than
// 256-wide ones); 192-wide pair tiles ran at 0.79 of the 256-wide pair rate
// per flop on the 4608 x 4608 out- and down-projections (a pair tile of 192
// needs ~75 operand bytes per cycle per SM from L2 against 64 at 256); 240
// needs ~66.  On N = 4608 the 256-wide tiles leave the last of 4.4 rounds of
// 74 pairs 62% idle, the 240-wide ones (20 column tiles, 4% of them past N)
// the last of 4.86 rounds 14% idle.
// allow240: the epilogue handles a partial last tile (the gated residual).
int choose_bn(int M, int N, int sms, bool allow240 = false) {
  const int cand[4] = {256, 240, 192, 128};
  const double mma_eff_single[4] = {1.0, 0.0, 0.88, 0.8};
  const double mma_eff_pair[4] = {1.0, 0.97, 0.8, 0.0};
  int best = 0;
  double best_score = -1.0;
  for (int i = 0; i < 4; ++i) {
    const int bn = cand[i];
    const bool pair = use_pair(bn, M);
    if (bn == 240 ? (!allow240 || !pair || N % 16) : (N % bn)) continue;
    const int bm = pair ? 2 * GEMM_BM : GEMM_BM;
    const int workers = pair ? sms / 2 : sms;
    const long tiles_n = (N + bn - 1) / bn;
    const long tiles = static_cast<long>((M + bm - 1) / bm) * tiles_n;
    const long waves = (tiles + workers - 1) / workers;
    const double eff = pair ? mma_eff_pair[i] : mma_eff_single[i];
    const double useful = static_cast<double>(N) / static_cast<double>(tiles_n * bn);
    const double score = eff * useful * static_cast<double>(tiles) / static_cast<double>(waves * workers);
    if (score > best_score + 1e-9) {
      best_score = score;
      best = bn;
    }
  }
  return best;
}

template <int BN, typename XT>
ig4_status launch_resid_bn(int B, int L, int N, int K, const void *a, bool f8, const float *a_scale,
                           const void *w, const float *w_scale, const float *gate, int gate_stride,
                           const void *x_res, void *x_out, cudaStream_t st) {
  const int M = B * L;
  CUtensorMap ma, mb;
  IG4_TRY(gemm_maps(&ma, &mb, a, w, f8 ? 1 : 2, M, N, K, b_box_rows(BN, M)));
  if (f8) {
    EpiResidGate<BN, true, XT> e{static_cast<const XT *>(x_res), static_cast<XT *>(x_out), gate,
                                  gate_stride, L, M, N, a_scale, w_scale};
    return launch_gemm<BN, true, false>(ma, mb, mb, M, (N + BN - 1) / BN, K, e, st);
  }
  EpiResidGate<BN, false, XT> e{static_cast<const XT *>(x_res), static_cast<XT *>(x_out), gate,
                                 gate_stride, L, M, N, nullptr, nullptr};
  return launch_gemm<BN, false, false>(ma, mb, mb, M, (N + BN - 1) / BN, K, e, st);
}

template <typename XT>
ig4_status launch_resid_t(int B, int L, int N, int K, const void *a, bool f8, const float *a_scale,
                          const void *w, const float *w_scale, const float *gate, int gate_stride,
                          const void *x_res, void *x_out, cudaStream_t st) {
  DeviceInfo *di = nullptr;
  IG4_TRY(device_info(&di));
  switch (choose_bn(B * L, N, di->sms, true)) {
    case 256:
      return launch_resid_bn<256, XT>(B, L, N, K, a, f8, a_scale, w, w_scale, gate, gate_stride,
                                      x_res, x_out, st);
    case 240:
      return launch_resid_bn<240, XT>(B, L, N, K, a, f8, a_scale, w, w_scale, gate, gate_stride,
                                      x_res, x_out, st);
    case 192:
      return launch_resid_bn<192, XT>(B, L, N, K, a, f8, a_scale, w, w_scale, gate, gate_stride,
                                      x_res, x_out, st);
    case 128:
      return launch_resid_bn<128, XT>(B, L, N, K, a, f8, a_scale, w, w_scale, gate, gate_stride,
                                      x_res, x_out, st);
    default:
      return IG4_ERR_UNSUPPORTED;
  }
}

ig4_status launch_resid(int B, int L, int N, int K, const void *a, bool f8, const float *a_scale,
                        const void *w, const float *w_scale, const float *gate, int gate_stride,
                        const void *x_res, void *x_out, int x_dtype, cudaStream_t st) {
  if (x_dtype == IG4_F32)
    return launch_resid_t<float>(B, L, N, K, a, f8, a_scale, w, w_scale, gate, gate_stride, x_res,
                                 x_out, st);
  return launch_resid_t<__nv_bfloat16>(B, L, N, K, a, f8, a_scale, w, w_scale, gate, gate_stride,
                                       x_res, x_out, st);
}

ig4_status launch_swiglu(int M, int I, int K, const void *h, bool f8, const float *h_scale,
                         const void *wg, const void *wu, const float *sg, const float *su, void *u,
                         cudaStream_t st) {
  const int esize = f8 ? 1 : 2;
  CUtensorMap ma, mg, mu;
  IG4_TRY(map_2d(&ma, h, esize, M, K, K, GEMM_BM, 128 / esize));
  IG4_TRY(map_2d(&mg, wg, esize, I, K, K, 128, 128 / esize));
  IG4_TRY(map_2d(&mu, wu, esize, I, K, K, 128, 128 / esize));
  if (f8) {
    EpiSwiGLU<true> e{static_cast<__nv_bfloat16 *>(u), I, M, h_scale, sg, su};
    return launch_gemm<256, true, true>(ma, mg, mu, M, I / 128, K, e, st);
  }
  EpiSwiGLU<false> e{static_cast<__nv_bfloat16 *>(u), I, M, nullptr, nullptr, nullptr};
  return launch_gemm<256, false, true>(ma, mg, mu, M, I / 128, K, e, st);
}

// ------------------------------------------------- MX8 (FP8, 1x32 scales)
// The FP8 block feeds the out- and down-projections MX8 activations (E4M3
// with a UE8M0 scale per 32 elements, written by the attention and SwiGLU
// epilogues) through the block-scaled pair GEMM.  K % 128 == 0, N % 16 == 0.
inline bool mx8_ok(long N, long K) { return K % 128 == 0 && N % 16 == 0; }

// bytes of packed MX8 scales of an [M][K] operand (rows padded to 128)
inline size_t mx8_sf_bytes(long M, long K) { return static_cast<size_t>((M + 127) / 128) * (K / 128) * 512; }

ig4_status launch_mx8_quantize(int M, int K, const void *x, void *codes, void *sf,
                               cudaStream_t st) {
  if (K % 128) return IG4_ERR_UNSUPPORTED;
  const int rows_per_cta = MX8Q_THREADS / 32;
  if (launch_pdl(quantize_mx8_kernel, dim3((M + rows_per_cta - 1) / rows_per_cta),
                 dim3(MX8Q_THREADS), 0, st, static_cast<const __nv_bfloat16 *>(x), M, K,
                 static_cast<uint8_t *>(codes), static_cast<uint8_t *>(sf)) != cudaSuccess)
    return IG4_ERR_CUDA;
  return last_launch_status();
}

// scale chunks [row blocks][K/128][128 words]; a box is one chunk
ig4_status map_mx8_sf(CUtensorMap *m, const void *base, long rows, long K) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return IG4_ERR_CUDA;
  const long rb = (rows + 127) / 128;
  cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(K / 128), static_cast<cuuint64_t>(rb)};
  cuuint64_t strides[2] = {512, static_cast<cuuint64_t>(K / 128) * 512};
  cuuint32_t box[3] = {128, 1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void *>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? IG4_OK : IG4_ERR_CUDA;
}

// Block-scaled pair GEMM with A in MX8: gemm_pair_kernel's MX8A variant on
// 240-wide tiles (or 192-wide where the tile chooser prefers them): two
// accumulators of at most 240 columns leave TMEM room for the scales.
template <int BN, class Epi>
ig4_status launch_mx8_gemm(const void *a_codes, const void *a_sf, const void *w, int M, int N,
                           int K, const Epi &ep, cudaStream_t st) {
  static_assert(BN == 192 || BN == 240, "MX8 tile width");
  if (K % 128 || N % 16 || (BN == 192 && N % 192)) return IG4_ERR_UNSUPPORTED;
  CUtensorMap ma, mb, msa;
  IG4_TRY(map_2d(&ma, a_codes, 1, M, K, K, GEMM_BM, 128));
  IG4_TRY(map_2d(&mb, w, 1, N, K, K, BN / 2, 128));
  IG4_TRY(map_mx8_sf(&msa, a_sf, M, K));
  DeviceInfo *di = nullptr;
  IG4_TRY(device_info(&di));
  const int n_tiles_n = (N + BN - 1) / BN;
  const long tiles = static_cast<long>((M + 2 * GEMM_BM - 1) / (2 * GEMM_BM)) * n_tiles_n;
  const int pairs = static_cast<int>(std::min<long>(tiles, di->sms / 2));
  const int group_m = gemm_group_m(M, K, 1);
  auto kern = gemm_pair_kernel<BN, true, false, Epi, true>;
  constexpr int SMEM = PairShape<BN, true>::SMEM_BYTES;
  IG4_TRY(allow_smem(kern, SMEM));
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(2 * pairs);
  lc.blockDim = dim3(GEMM_THREADS);
  lc.dynamicSmemBytes = SMEM;
  lc.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = 2;
  if (cudaLaunchKernelEx(&lc, kern, ma, mb, msa, M, n_tiles_n, K, group_m, ep) != cudaSuccess)
    return IG4_ERR_CUDA;
  return last_launch_status();
}

template <int BN, typename XT>
ig4_status launch_mx8_resid_bn(int B, int L, int N, int K, const void *a_codes, const void *a_sf,
                               const void *w, const float *w_scale, const float *gate,
                               int gate_stride, const void *x_res, void *x_out, cudaStream_t st) {
  const int M = B * L;
  EpiResidGate<BN, true, XT> e{static_cast<const XT *>(x_res), static_cast<XT *>(x_out), gate,
                               gate_stride, L, M, N, nullptr, w_scale};
  return launch_mx8_gemm<BN>(a_codes, a_sf, w, M, N, K, e, st);
}

// x_out = x_res + gate * (w_scale (A W^T)) with A in MX8.
ig4_status launch_mx8_resid(int B, int L, int N, int K, const void *a_codes, const void *a_sf,
                            const void *w, const float *w_scale, const float *gate,
                            int gate_stride, const void *x_res, void *x_out, int x_dtype,
                            cudaStream_t st) {
  const bool f32 = x_dtype == IG4_F32;
  DeviceInfo *di = nullptr;
  IG4_TRY(device_info(&di));
  // 192-wide where it divides N and the chooser prefers it, else 240-wide
  const int M = B * L;
  if (M > GEMM_BM && choose_bn(M, N, di->sms, true) == 192)
    return f32 ? launch_mx8_resid_bn<192, float>(B, L, N, K, a_codes, a_sf, w, w_scale, gate,
                                                 gate_stride, x_res, x_out, st)
               : launch_mx8_resid_bn<192, __nv_bfloat16>(B, L, N, K, a_codes, a_sf, w, w_scale,
                                                         gate, gate_stride, x_res, x_out, st);
  return f32 ? launch_mx8_resid_bn<240, float>(B, L, N, K, a_codes, a_sf, w, w_scale, gate,
                                               gate_stride, x_res, x_out, st)
             : launch_mx8_resid_bn<240, __nv_bfloat16>(B, L, N, K, a_codes, a_sf, w, w_scale,
                                                       gate, gate_stride, x_res, x_out, st);
}

// FP8 SwiGLU writing u as MX8 (codes [M][I], packed scales).  I % 128 == 0.
ig4_status launch_swiglu_mx8(int M, int I, int K, const void *h, const float *h_scale,
                             const void *wg, const void *wu, const float *sg, const float *su,
                             void *uq, void *usf, cudaStream_t st) {
  if (I % 128) return IG4_ERR_UNSUPPORTED;
  CUtensorMap ma, mg, mu;
  IG4_TRY(map_2d(&ma, h, 1, M, K, K, GEMM_BM, 128));
  IG4_TRY(map_2d(&mg, wg, 1, I, K, K, 128, 128));
  IG4_TRY(map_2d(&mu, wu, 1, I, K, K, 128, 128));
  EpiSwiGLUMx8 e{static_cast<uint8_t *>(uq), static_cast<uint8_t *>(usf), I, M, h_scale, sg, su};
  return launch_gemm<256, true, true>(ma, mg, mu, M, I / 128, K, e, st);
}

// E4M3 weight [N][K] with per-row scale -> bf16 [N][K].  K % 16 == 0.
ig4_status launch_dequant(int N, int K, const void *q, const float *s, void *out, cudaStream_t st) {
  const long total16 = static_cast<long>(N) * K / 16;
  const int grid = static_cast<int>(std::min<long>((total16 + 255) / 256, 148L * 16));
  if (launch_pdl(dequant_e4m3_rows_kernel, dim3(grid), dim3(256), 0, st,
                 static_cast<const uint8_t *>(q), s, static_cast<__nv_bfloat16 *>(out), K,
                 total16) != cudaSuccess)
    return IG4_ERR_CUDA;
  return last_launch_status();
}

// Plain linear with bias (stack in/out projections).  N % 128 == 0.
ig4_status launch_linear_store(int M, int N, int K, const void *a, bool f8, const float *a_scale,
                               const void *w, const float *w_scale, const float *bias, void *out,
                               int out_dtype, int ldo, int remap_n, int remap_L, int remap_off,
                               cudaStream_t st) {
  CUtensorMap ma, mb;
  IG4_TRY(gemm_maps(&ma, &mb, a, w, f8 ? 1 : 2, M, N, K, 128));
  if (out_dtype == IG4_F32) {
    if (f8) {
      EpiStore<128, true, float> e{static_cast<float *>(out), ldo, M, N, bias, a_scale, w_scale,
                                   remap_n, remap_L, remap_off};
      return launch_gemm<128, true, false>(ma, mb, mb, M, N / 128, K, e, st);
    }
    EpiStore<128, false, float> e{static_cast<float *>(out), ldo, M, N, bias, nullptr, nullptr,
                                  remap_n, remap_L, remap_off};
    return launch_gemm<128, false, false>(ma, mb, mb, M, N / 128, K, e, st);
  }
  if (f8) {
    EpiStore<128, true, __nv_bfloat16> e{static_cast<__nv_bfloat16 *>(out), ldo, M, N, bias,
                                         a_scale, w_scale, remap_n, remap_L, remap_off};
    return launch_gemm<128, true, false>(ma, mb, mb, M, N / 128, K, e, st);
  }
  EpiStore<128, false, __nv_bfloat16> e{static_cast<__nv_bfloat16 *>(out), ldo, M, N, bias,
                                        nullptr, nullptr, remap_n, remap_L, remap_off};
  return launch_gemm<128, false, false>(ma, mb, mb, M, N / 128, K, e, st);
}

// Plain linear layer into bf16 with a bias, tile width chosen for the shape
// (the text conditioning projection: K = 53248, N = 4608, M = tokens).
template <int BN, bool FP8>
ig4_status launch_store_bf16_bn(int M, int N, int K, const void *a, const float *a_scale,
                                const void *w, const float *w_scale, const float *bias, void *out,
                                cudaStream_t st) {
  CUtensorMap ma, mb;
  IG4_TRY(gemm_maps(&ma, &mb, a, w, FP8 ? 1 : 2, M, N, K, b_box_rows(BN, M)));
  EpiStore<BN, FP8, __nv_bfloat16> e{static_cast<__nv_bfloat16 *>(out), N, M, N, bias,
                                     FP8 ? a_scale : nullptr, FP8 ? w_scale : nullptr, 0, 0, 0};
  return launch_gemm<BN, FP8, false>(ma, mb, mb, M, N / BN, K, e, st);
}

template <bool FP8>
ig4_status launch_store_bf16(int M, int N, int K, const void *a, const float *a_scale,
                             const void *w, const float *w_scale, const float *bias, void *out,
                             cudaStream_t st) {
  DeviceInfo *di = nullptr;
  IG4_TRY(device_info(&di));
  switch (choose_bn(M, N, di->sms)) {
    case 256:
      return launch_store_bf16_bn<256, FP8>(M, N, K, a, a_scale, w, w_scale, bias, out, st);
    case 192:
      return launch_store_bf16_bn<192, FP8>(M, N, K, a, a_scale, w, w_scale, bias, out, st);
    case 128:
      return launch_store_bf16_bn<128, FP8>(M, N, K, a, a_scale, w, w_scale, bias, out, st);
    default:
      return IG4_ERR_UNSUPPORTED;
  }
}

// Packed NVFP4 scale blocks as a 3D tensor of 4-byte words: [row blocks of
// 128][K/64 chunks][128 words]; a box takes 4 chunks (one stage) of
// `blocks` row blocks.
ig4_status map_sf_3d(CUtensorMap *m, const void *base, long rows, long K, int blocks) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return IG4_ERR_CUDA;
  const long rb = (rows + 127) / 128;
  cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(K / 64), static_cast<cuuint64_t>(rb)};
  cuuint64_t strides[2] = {512, static_cast<cuuint64_t>(K / 64) * 512};
  cuuint32_t box[3] = {128, 4, static_cast<cuuint32_t>(blocks)};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void *>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? IG4_OK : IG4_ERR_CUDA;
}

// NVFP4 GEMM on CTA pairs (256 x 256 tiles), maps built by the caller.
template <bool DUAL_B, class Epi>
ig4_status launch_nvf4_pair_maps(const CUtensorMap &ma, const CUtensorMap &mb,
                                 const CUtensorMap &mb2, const CUtensorMap &msa,
                                 const CUtensorMap &msb, const CUtensorMap &msb2, int M,
                                 int n_tiles_n, int K, const Epi &ep, cudaStream_t st) {
  DeviceInfo *di = nullptr;
  IG4_TRY(device_info(&di));
  const long tiles = static_cast<long>((M + 2 * GEMM_BM - 1) / (2 * GEMM_BM)) * n_tiles_n;
  const int pairs = static_cast<int>(std::min<long>(tiles, di->sms / 2));
  const int group_m = gemm_group_m(M, K / 2, 1);
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(2 * pairs);
  lc.blockDim = dim3(NVF4P_THREADS);
  lc.dynamicSmemBytes = NVF4P_SMEM_BYTES;
  lc.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = 2;
  auto kern = gemm_nvf4_pair_kernel<DUAL_B, Epi>;
  IG4_TRY(allow_smem(kern, NVF4P_SMEM_BYTES));
  if (cudaLaunchKernelEx(&lc, kern, ma, mb, mb2, msa, msb, msb2, M, n_tiles_n, K, group_m, ep) !=
      cudaSuccess)
    return IG4_ERR_CUDA;
  return last_launch_status();
}

// A operand maps of an NVFP4 GEMM: codes [M][K/2] and packed scales.
ig4_status nvf4_a_maps(CUtensorMap *ma, CUtensorMap *msa, const void *codes, const void *sf,
                       int M, int K) {
  IG4_TRY(map_2d(ma, codes, 1, M, K / 2, K / 2, GEMM_BM, 128));
  return map_sf_3d(msa, sf, M, K, 1);
}

// NVFP4 linear layer on CTA pairs: out = a_scale w_scale (A W^T) (+ bias).
ig4_status launch_nvf4_pair(int M, int N, int K, const void *a_codes, const void *a_sf,
                            const float *a_scale, const void *w_codes, const void *w_sf,
                            const float *w_scale, const float *bias, void *out, int out_dtype,
                            cudaStream_t st) {
  CUtensorMap ma, mb, msa, msb;
  IG4_TRY(nvf4_a_maps(&ma, &msa, a_codes, a_sf, M, K));
  IG4_TRY(map_2d(&mb, w_codes, 1, N, K / 2, K / 2, 128, 128));
  IG4_TRY(map_sf_3d(&msb, w_sf, N, K, 2));
  if (out_dtype == IG4_F32) {
    EpiStore<256, true, float> ep{static_cast<float *>(out), N, M, N, bias, a_scale, w_scale, 0, 0, 0};
    return launch_nvf4_pair_maps<false>(ma, mb, mb, msa, msb, msb, M, N / 256, K, ep, st);
  }
  EpiStore<256, true, __nv_bfloat16> ep{static_cast<__nv_bfloat16 *>(out), N, M, N, bias,
                                        a_scale, w_scale, 0, 0, 0};
  return launch_nvf4_pair_maps<false>(ma, mb, mb, msa, msb, msb, M, N / 256, K, ep, st);
}

// NVFP4 gate/up + SwiGLU: u = silu(a_scale s_g (h W_g^T)) * (a_scale s_u (h W_u^T)), bf16.
ig4_status launch_nvf4_swiglu(int M, int I, int K, const void *h_codes, const void *h_sf,
                              const float *h_scale, const void *wg, const void *sfg,
                              const float *sg, const void *wu, const void *sfu, const float *su,
                              void *u, cudaStream_t st) {
  CUtensorMap ma, msa, mg, mu, msg, msu;
  IG4_TRY(nvf4_a_maps(&ma, &msa, h_codes, h_sf, M, K));
  IG4_TRY(map_2d(&mg, wg, 1, I, K / 2, K / 2, 128, 128));
  IG4_TRY(map_2d(&mu, wu, 1, I, K / 2, K / 2, 128, 128));
  IG4_TRY(map_sf_3d(&msg, sfg, I, K, 1));
  IG4_TRY(map_sf_3d(&msu, sfu, I, K, 1));
  EpiSwiGLU<true> ep{static_cast<__nv_bfloat16 *>(u), I, M, h_scale, sg, su};
  return launch_nvf4_pair_maps<true>(ma, mg, mu, msa, msg, msu, M, I / 128, K, ep, st);
}

// NVFP4 down-projection + gated residual: x_out = x_res + gate * (a_scale w_scale (u W^T)).
template <typename XT>
ig4_status launch_nvf4_resid_t(int B, int L, int N, int K, const void *a_codes, const void *a_sf,
                               const float *a_scale, const void *w, const void *w_sf,
                               const float *w_scale, const float *gate, int gate_stride,
                               const void *x_res, void *x_out, cudaStream_t st) {
  const int M = B * L;
  CUtensorMap ma, msa, mb, msb;
  IG4_TRY(nvf4_a_maps(&ma, &msa, a_codes, a_sf, M, K));
  IG4_TRY(map_2d(&mb, w, 1, N, K / 2, K / 2, 128, 128));
  IG4_TRY(map_sf_3d(&msb, w_sf, N, K, 2));
  EpiResidGate<256, true, XT> ep{static_cast<const XT *>(x_res), static_cast<XT *>(x_out), gate,
                                 gate_stride, L, M, N, a_scale, w_scale};
  return launch_nvf4_pair_maps<false>(ma, mb, mb, msa, msb, msb, M, N / 256, K, ep, st);
}

ig4_status launch_nvf4_resid(int B, int L, int N, int K, const void *a_codes, const void *a_sf,
                             const float *a_scale, const void *w, const void *w_sf,
                             const float *w_scale, const float *gate, int gate_stride,
                             const void *x_res, void *x_out, int x_dtype, cudaStream_t st) {
  if (x_dtype == IG4_F32)
    return launch_nvf4_resid_t<float>(B, L, N, K, a_codes, a_sf, a_scale, w, w_sf, w_scale, gate,
                                      gate_stride, x_res, x_out, st);
  return launch_nvf4_resid_t<__nv_bfloat16>(B, L, N, K, a_codes, a_sf, a_scale, w, w_sf, w_scale,
                                            gate, gate_stride, x_res, x_out, st);
}

// bf16 rows -> NVFP4 codes, packed scales and row scales (one warp per row).
ig4_status launch_nvf4_quantize(int M, int K, const void *x, void *codes, void *sf,
                                float *row_scale, cudaStream_t st) {
  const int rows_per_cta = NVF4Q_THREADS / 32;
  if (launch_pdl(nvf4_quantize_kernel, dim3((M + rows_per_cta - 1) / rows_per_cta),
                 dim3(NVF4Q_THREADS), 0, st, static_cast<const __nv_bfloat16 *>(x), M, K,
                 static_cast<uint8_t *>(codes), static_cast<uint8_t *>(sf), row_scale) !=
      cudaSuccess)
    return IG4_ERR_CUDA;
  return last_launch_status();
}

// NVFP4 linear layer on 128- or 256-wide tiles.
template <int BN>
ig4_status launch_nvf4(int M, int N, int K, const void *a_codes, const void *a_sf,
                       const float *a_scale, const void *w_codes, const void *w_sf,
                       const float *w_scale, const float *bias, void *out, int out_dtype, int sms,
                       cudaStream_t st) {
  CUtensorMap ma, mb;
  IG4_TRY(map_2d(&ma, a_codes, 1, M, K / 2, K / 2, GEMM_BM, 128));
  IG4_TRY(map_2d(&mb, w_codes, 1, N, K / 2, K / 2, BN, 128));
  const int n_tiles_n = N / BN;
  const long tiles = static_cast<long>((M + GEMM_BM - 1) / GEMM_BM) * n_tiles_n;
  const int grid = static_cast<int>(std::min<long>(tiles, sms));
  const int group_m = gemm_group_m(M, K / 2, 1);
  const uint8_t *sa = static_cast<const uint8_t *>(a_sf);
  const uint8_t *sw = static_cast<const uint8_t *>(w_sf);
  constexpr int SMEM = Nvf4Shape<BN>::SMEM_BYTES;
  if (out_dtype == IG4_F32) {
    EpiStore<BN, true, float> e{static_cast<float *>(out), N, M, N, bias, a_scale, w_scale, 0, 0, 0};
    auto kern = gemm_nvf4_kernel<BN, decltype(e)>;
    IG4_TRY(allow_smem(kern, SMEM));
    if (launch_pdl(kern, dim3(grid), dim3(GEMM_THREADS), SMEM, st, ma, mb, sa, sw, M, n_tiles_n, K,
                   group_m, e) != cudaSuccess)
      return IG4_ERR_CUDA;
  } else {
    EpiStore<BN, true, __nv_bfloat16> e{static_cast<__nv_bfloat16 *>(out), N, M, N, bias, a_scale,
                                        w_scale, 0, 0, 0};
    auto kern = gemm_nvf4_kernel<BN, decltype(e)>;
    IG4_TRY(allow_smem(kern, SMEM));
    if (launch_pdl(kern, dim3(grid), dim3(GEMM_THREADS), SMEM, st, ma, mb, sa, sw, M, n_tiles_n, K,
                   group_m, e) != cudaSuccess)
      return IG4_ERR_CUDA;
  }
  return last_launch_status();
}

// ------------------------------------------------------- workspace layout

struct BlockWs {
  float *mod, *cos, *sin;
  void *h;        // bf16 [M][D] or e4m3 [M][D]
  float *h_scale; // [M] (E4M3)
  void *q, *k, *vt;
  void *o;        // bf16 [M][D]
  void *oq;       // e4m3 [M][D]
  float *o_scale;
  void *u;        // bf16 [M][I]
  void *uq;       // e4m3 [M][I]
  float *u_scale;
  void *h_sf, *u_sf;  // packed NVFP4 scales of h2 and u (NVFP4-mixed FFN); u_sf: MX8 scales of u (FP8)
  void *o_sf;         // MX8 scales of the attention output (FP8 weights)
  void *att_part;     // attention partial slots: the u buffer (u is written after attention)
  int vt_ld;
  size_t bytes;
};

// The FP8 block's MX8 stages: the attention output into the out-projection
// (N = K = D), u into the down-projection (N = D, K = I; not with the NVFP4
// FFN).
inline bool mx8_attn_out(const ig4_config *c) { return is_fp8(c->w_dtype) && mx8_ok(c->D, c->D); }
inline bool mx8_ffn(const ig4_config *c) {
  return is_fp8(c->w_dtype) && !is_nvf4_mixed(c->w_dtype) && mx8_ok(c->D, c->I);
}

// Lays the block's buffers out from `base` (nullptr: only count bytes).
BlockWs block_ws_layout(const ig4_config *c, uint8_t *base) {
  BlockWs w{};
  const long L = c->T_text + static_cast<long>(c->grid_t) * c->grid_h * c->grid_w;
  const long M = c->B * L;
  const long D = c->D, I = c->I, H = c->H;
  const bool f8 = is_fp8(c->w_dtype);
  const bool nv4 = is_nvf4_mixed(c->w_dtype);
  w.vt_ld = static_cast<int>(round_up(L, 8));
  size_t off = 0;
  auto take = [&](size_t n) -> uint8_t * {
    uint8_t *p = base ? base + off : nullptr;
    off += round_up(n, 256);
    return p;
  };
  w.mod = reinterpret_cast<float *>(take(sizeof(float) * c->B * 6 * D));
  w.cos = reinterpret_cast<float *>(take(sizeof(float) * L * 64));
  w.sin = reinterpret_cast<float *>(take(sizeof(float) * L * 64));
  w.h = take((f8 && !nv4 ? 1 : 2) * M * D);  // NVFP4 FFN: h2 in bf16 before quantising
  w.h_scale = reinterpret_cast<float *>(take(f8 ? sizeof(float) * M : 0));
  w.q = take(2 * c->B * H * L * 256);
  w.k = take(2 * c->B * H * L * 256);
  w.vt = take(2 * c->B * H * 256 * static_cast<long>(w.vt_ld));
  w.o = take(2 * M * D);
  w.oq = take(f8 ? M * D : 0);
  w.o_scale = reinterpret_cast<float *>(take(f8 ? sizeof(float) * M : 0));
  w.u = take(std::max<size_t>(2 * M * I, att_part_bytes(c->B, static_cast<int>(H),
                                                         static_cast<int>(L))));
  w.att_part = att_part_bytes(c->B, static_cast<int>(H), static_cast<int>(L)) ? w.u : nullptr;
  w.uq = take(f8 ? M * I : 0);
  w.u_scale = reinterpret_cast<float *>(take(f8 ? sizeof(float) * M : 0));
  // NVFP4 FFN: h2 codes reuse oq (M D / 2 bytes), u codes reuse uq
  const long rb = (M + 127) / 128;
  w.h_sf = take(nv4 ? rb * (D / 64) * 512 : 0);
  w.u_sf = take(nv4 ? rb * (I / 64) * 512 : (mx8_ffn(c) ? mx8_sf_bytes(M, I) : 0));
  w.o_sf = take(mx8_attn_out(c) ? mx8_sf_bytes(M, D) : 0);
  w.bytes = off;
  return w;
}

ig4_status check_block_weights(const ig4_config *c, const ig4_block_weights *w) {
  if (!w) return IG4_ERR_INVALID_ARG;
  const void *ptrs[] = {w->w_ada, w->w_qkv, w->w_o, w->w_gate, w->w_up, w->w_down,
                        w->b_ada, w->g_q, w->g_k};
  for (const void *p : ptrs)
    if (!p || !aligned16(p)) return IG4_ERR_INVALID_ARG;
  if (is_fp8(c->w_dtype)) {
    const void *s[] = {w->s_ada, w->s_qkv, w->s_o, w->s_gate, w->s_up, w->s_down};
    for (const void *p : s)
      if (!p || !aligned16(p)) return IG4_ERR_INVALID_ARG;
  }
  if (is_nvf4_mixed(c->w_dtype)) {
    const void *sf[] = {w->sf_gate, w->sf_up, w->sf_down};
    for (const void *p : sf)
      if (!p || !aligned16(p)) return IG4_ERR_INVALID_ARG;
  }
  return IG4_OK;
}

// Event recording for the traced block forward.
struct Tracer {
  void *const *ev;
  int n;
  int next;
  cudaStream_t st;
  ig4_status mark() {
    if (!ev || next >= n) return IG4_OK;
    void *e = ev[next++];
    if (!e) return IG4_OK;  // this boundary is not recorded
    return cudaEventRecord(reinterpret_cast<cudaEvent_t>(e), st) == cudaSuccess ? IG4_OK
                                                                                 : IG4_ERR_CUDA;
  }
};

// The block's steps before attention: AdaLN, rotary table (unless
// rope_ready: ws.cos / ws.sin already hold the table of these positions, as
// in the stack's blocks after the first), norm1, QKV with QK-norm and MRoPE
// into ws.q, ws.k, ws.vt.  Records trace marks 0..4.
ig4_status block_pre_attention(const ig4_config *c, const ig4_block_weights *w, const void *x_in,
                               const int32_t *pos, const float *temb, const BlockWs &ws,
                               cudaStream_t st, Tracer &t, bool rope_ready) {
  const int L = c->T_text + c->grid_t * c->grid_h * c->grid_w;
  const int M = c->B * L;
  const int D = c->D, H = c->H;
  const bool f8 = is_fp8(c->w_dtype);
  const int hdt = f8 ? IG4_E4M3 : IG4_BF16;
  const int ms = 6 * D;
  IG4_TRY(t.mark());
  IG4_TRY(launch_adaln(c->B, c->adaln_dim, 6 * D, temb, w->w_ada, c->w_dtype, w->s_ada, w->b_ada,
                       ws.mod, st));
  IG4_TRY(t.mark());
  if (!rope_ready)
    IG4_TRY(launch_rope_table(L, pos, c->rope_theta, c->sections, ws.cos, ws.sin, st));
  IG4_TRY(t.mark());
  IG4_TRY(launch_norm(M, L, D, x_in, c->x_dtype, ws.mod + 0 * D, ws.mod + 1 * D, ms, c->eps, ws.h,
                      hdt, ws.h_scale, 0, 0, 0, st));
  IG4_TRY(t.mark());
  IG4_TRY(launch_qkv(c->B, L, D, H, ws.h, hdt, ws.h_scale, w->w_qkv, w->s_qkv, w->g_q, w->g_k,
                     c->eps, ws.cos, ws.sin, ws.q, ws.k, ws.vt, ws.vt_ld, st));
  IG4_TRY(t.mark());
  return IG4_OK;
}

// The block's steps after attention, with o in ws.o: out-projection + gated
// residual (x_in -> x_out), norm2, SwiGLU, down-projection + gated residual
// (in place in x_out).  The AdaLN modulation is read from ws.mod.
ig4_status block_post_attention(const ig4_config *c, const ig4_block_weights *w, const void *x_in,
                                void *x_out, const BlockWs &ws, cudaStream_t st, Tracer &t,
                                bool o_is_mx8 = false) {
  const int L = c->T_text + c->grid_t * c->grid_h * c->grid_w;
  const int M = c->B * L;
  const int D = c->D, I = c->I;
  const bool f8 = is_fp8(c->w_dtype);
  const int hdt = f8 ? IG4_E4M3 : IG4_BF16;
  const int ms = 6 * D;
  if (f8 && mx8_attn_out(c)) {
    // MX8 attention output: written by the attention epilogue, or encoded here
    if (!o_is_mx8) IG4_TRY(launch_mx8_quantize(M, D, ws.o, ws.oq, ws.o_sf, st));
    IG4_TRY(t.mark());
    IG4_TRY(launch_mx8_resid(c->B, L, D, D, ws.oq, ws.o_sf, w->w_o, w->s_o, ws.mod + 2 * D, ms,
                             x_in, x_out, c->x_dtype, st));
  } else {
    if (f8) {
      IG4_TRY(launch_quantize(M, D, ws.o, ws.oq, ws.o_scale, st));
      IG4_TRY(t.mark());
    }
    IG4_TRY(launch_resid(c->B, L, D, D, f8 ? ws.oq : ws.o, f8, ws.o_scale, w->w_o, w->s_o,
                         ws.mod + 2 * D, ms, x_in, x_out, c->x_dtype, st));
  }
  IG4_TRY(t.mark());
  if (is_nvf4_mixed(c->w_dtype)) {
    // FFN in NVFP4: h2 (bf16) and u (bf16) are quantised to NVFP4 for the
    // block-scaled FP4 GEMMs; the h2 quantiser shares the norm's trace slot
    IG4_TRY(launch_norm(M, L, D, x_out, c->x_dtype, ws.mod + 3 * D, ws.mod + 4 * D, ms, c->eps,
                        ws.h, IG4_BF16, nullptr, 0, 0, 0, st));
    IG4_TRY(launch_nvf4_quantize(M, D, ws.h, ws.oq, ws.h_sf, ws.h_scale, st));
    IG4_TRY(t.mark());
    IG4_TRY(launch_nvf4_swiglu(M, I, D, ws.oq, ws.h_sf, ws.h_scale, w->w_gate, w->sf_gate,
                               w->s_gate, w->w_up, w->sf_up, w->s_up, ws.u, st));
    IG4_TRY(t.mark());
    IG4_TRY(launch_nvf4_quantize(M, I, ws.u, ws.uq, ws.u_sf, ws.u_scale, st));
    IG4_TRY(t.mark());
    IG4_TRY(launch_nvf4_resid(c->B, L, D, I, ws.uq, ws.u_sf, ws.u_scale, w->w_down, w->sf_down,
                              w->s_down, ws.mod + 5 * D, ms, x_out, x_out, c->x_dtype, st));
    IG4_TRY(t.mark());
    return IG4_OK;
  }
  IG4_TRY(launch_norm(M, L, D, x_out, c->x_dtype, ws.mod + 3 * D, ws.mod + 4 * D, ms, c->eps,
                      ws.h, hdt, ws.h_scale, 0, 0, 0, st));
  IG4_TRY(t.mark());
  if (mx8_ffn(c)) {
    // u leaves the SwiGLU epilogue as MX8 (its trace slot after it stays empty)
    IG4_TRY(launch_swiglu_mx8(M, I, D, ws.h, ws.h_scale, w->w_gate, w->w_up, w->s_gate, w->s_up,
                              ws.uq, ws.u_sf, st));
    IG4_TRY(t.mark());
    IG4_TRY(t.mark());
    IG4_TRY(launch_mx8_resid(c->B, L, D, I, ws.uq, ws.u_sf, w->w_down, w->s_down, ws.mod + 5 * D,
                             ms, x_out, x_out, c->x_dtype, st));
    IG4_TRY(t.mark());
    return IG4_OK;
  }
  IG4_TRY(launch_swiglu(M, I, D, ws.h, f8, ws.h_scale, w->w_gate, w->w_up, w->s_gate, w->s_up,
                        ws.u, st));
  IG4_TRY(t.mark());
  if (f8) {
    IG4_TRY(launch_quantize(M, I, ws.u, ws.uq, ws.u_scale, st));
    IG4_TRY(t.mark());
  }
  IG4_TRY(launch_resid(c->B, L, D, I, f8 ? ws.uq : ws.u, f8, ws.u_scale, w->w_down, w->s_down,
                       ws.mod + 5 * D, ms, x_out, x_out, c->x_dtype, st));
  IG4_TRY(t.mark());
  return IG4_OK;
}

// The block on already validated arguments.
// rope_ready: ws.cos / ws.sin already hold the table of these positions (the
// stack computes it for its first block only; every block shares it).
ig4_status block_forward_impl(const ig4_config *c, const ig4_block_weights *w, const void *x_in,
                              void *x_out, const int32_t *pos, const float *temb,
                              const BlockWs &ws, cudaStream_t st, Tracer *tr,
                              bool rope_ready = false) {
  const int L = c->T_text + c->grid_t * c->grid_h * c->grid_w;
  Tracer none{nullptr, 0, 0, st};
  Tracer &t = tr ? *tr : none;
  IG4_TRY(block_pre_attention(c, w, x_in, pos, temb, ws, st, t, rope_ready));
  const bool mx8 = mx8_attn_out(c);  // FP8: the attention epilogue writes MX8
  IG4_TRY(launch_attention(c->B, c->H, L, ws.q, ws.k, ws.vt, ws.vt_ld, mx8 ? ws.oq : ws.o,
                           ws.att_part, st, mx8 ? ws.o_sf : nullptr));
  IG4_TRY(t.mark());
  return block_post_attention(c, w, x_in, x_out, ws, st, t, mx8);
}

// Stack workspace: two sequence buffers, the block workspace, final-layer buffers.
struct StackWs {
  void *s0, *s1;
  BlockWs blk;
  float *mod_f;
  void *hf;  // bf16 [B*N][D]
  void *w_in16, *w_out16;  // bf16 copies of E4M3 in/out projection weights
  size_t bytes;
};

StackWs stack_ws_layout(const ig4_config *c, int C, uint8_t *base) {
  StackWs w{};
  const long L = c->T_text + static_cast<long>(c->grid_t) * c->grid_h * c->grid_w;
  const long N = static_cast<long>(c->grid_t) * c->grid_h * c->grid_w;
  const long M = c->B * L;
  const bool f8 = is_fp8(c->w_dtype);
  const long xs = c->x_dtype == IG4_F32 ? 4 : 2;
  size_t off = 0;
  auto take = [&](size_t n) -> uint8_t * {
    uint8_t *p = base ? base + off : nullptr;
    off += round_up(n, 256);
    return p;
  };
  w.s0 = take(xs * M * c->D);
  w.s1 = take(xs * M * c->D);
  w.mod_f = reinterpret_cast<float *>(take(sizeof(float) * c->B * 2 * c->D));
  w.hf = take(2 * c->B * N * c->D);
  w.w_in16 = take(f8 ? 2L * c->D * C : 0);
  w.w_out16 = take(f8 ? 2L * C * c->D : 0);
  uint8_t *blk_base = base ? base + off : nullptr;
  w.blk = block_ws_layout(c, blk_base);
  off += w.blk.bytes;
  w.bytes = off;
  return w;
}

}  // namespace

// =================================================================== C ABI

extern "C" {

const char *ig4_status_string(int s) {
  switch (s) {
    case IG4_OK: return "IG4_OK";
    case IG4_ERR_INVALID_ARG: return "IG4_ERR_INVALID_ARG";
    case IG4_ERR_UNSUPPORTED: return "IG4_ERR_UNSUPPORTED";
    case IG4_ERR_WORKSPACE: return "IG4_ERR_WORKSPACE";
    case IG4_ERR_CUDA: return "IG4_ERR_CUDA";
    case IG4_ERR_TIMEOUT: return "IG4_ERR_TIMEOUT";
    default: return "IG4_ERR_UNKNOWN";
  }
}

int ig4_abi_version(void) { return ABI_VERSION; }

ig4_status ig4_mrope_positions(int T, int gt, int gh, int gw, int32_t *pos, int on_device,
                               void *stream) {
  if (!pos || T < 0 || gt < 0 || gh < 0 || gw < 0) return IG4_ERR_INVALID_ARG;
  const long L = static_cast<long>(T) + static_cast<long>(gt) * gh * gw;
  if (L < 1 || L > (1L << 24)) return IG4_ERR_INVALID_ARG;
  if (on_device) {
    if (!aligned16(pos)) return IG4_ERR_INVALID_ARG;
    mrope_positions_kernel<<<static_cast<int>((L + 255) / 256), 256, 0, as_stream(stream)>>>(
        T, gt, gh, gw, 0, gt * gh * gw, pos);
    return last_launch_status();
  }
  for (long l = 0; l < T; ++l) pos[l] = pos[L + l] = pos[2 * L + l] = static_cast<int32_t>(l);
  long n = T;
  for (int t = 0; t < gt; ++t)
    for (int i = 0; i < gh; ++i)
      for (int j = 0; j < gw; ++j, ++n) {
        pos[n] = T + t;
        pos[L + n] = T + i;
        pos[2 * L + n] = T + j;
      }
  return IG4_OK;
}

ig4_status ig4_rope_table(int L, const int32_t *pos, double theta, const int sections[3],
                          float *cos_out, float *sin_out, void *stream) {
  if (L < 1 || !pos || !sections || !cos_out || !sin_out || !(theta > 0.0))
    return IG4_ERR_INVALID_ARG;
  if (sections[0] < 0 || sections[1] < 0 || sections[2] < 0 ||
      sections[0] + sections[1] + sections[2] != 64)
    return IG4_ERR_INVALID_ARG;
  return launch_rope_table(L, pos, theta, sections, cos_out, sin_out, as_stream(stream));
}

ig4_status ig4_adaln_modulation(int B, int A, int N, const float *temb, const void *w, int w_dtype,
                                const float *w_scale, const float *bias, float *mod_out,
                                void *stream) {
  if (!temb || !w || !mod_out || B < 1 || B > 8 || A < 16 || A % 16 || A > 1024 || N < 1)
    return IG4_ERR_INVALID_ARG;
  if (!valid_dtype_w(w_dtype) || (is_fp8(w_dtype) && !w_scale) || !aligned16(w))
    return IG4_ERR_INVALID_ARG;
  return launch_adaln(B, A, N, temb, w, w_dtype, w_scale, bias, mod_out, as_stream(stream));
}

ig4_status ig4_norm_modulate(int B, int L, int D, const void *x, int x_dtype, const float *shift,
                             const float *scale, int mod_stride, float eps, void *h_out,
                             int h_dtype, float *h_scale_out, void *stream) {
  if (!x || !shift || !scale || !h_out || B < 1 || L < 1 || D < 8 || D % 8 || D > 6144 ||
      !(eps > 0.0f) || mod_stride < D)
    return IG4_ERR_INVALID_ARG;
  if (!valid_dtype_x(x_dtype) || (h_dtype != IG4_BF16 && h_dtype != IG4_E4M3))
    return IG4_ERR_INVALID_ARG;
  if (h_dtype == IG4_E4M3 && !h_scale_out) return IG4_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(shift) || !aligned16(scale) || !aligned16(h_out) ||
      mod_stride % 4)
    return IG4_ERR_INVALID_ARG;
  return launch_norm(B * L, L, D, x, x_dtype, shift, scale, mod_stride, eps, h_out, h_dtype,
                     h_scale_out, 0, 0, 0, as_stream(stream));
}

ig4_status ig4_qkv_project(int B, int L, int D, int H, const void *h, int h_dtype,
                           const float *h_scale, const void *w_qkv, int w_dtype,
                           const float *w_scale, const float *g_q, const float *g_k, float eps,
                           const float *rope_cos, const float *rope_sin, void *q_out, void *k_out,
                           void *vt_out, int vt_ld, void *stream) {
  if (B < 1 || L < 1 || H < 1 || !h || !w_qkv || !g_q || !g_k || !rope_cos || !rope_sin ||
      !q_out || !k_out || !vt_out || !(eps > 0.0f) || vt_ld < L || vt_ld % 8)
    return IG4_ERR_INVALID_ARG;
  if (D != 256 * H) return IG4_ERR_UNSUPPORTED;
  if (!valid_dtype_w(w_dtype) || h_dtype != (is_fp8(w_dtype) ? IG4_E4M3 : IG4_BF16))
    return IG4_ERR_UNSUPPORTED;
  if (is_fp8(w_dtype) && (!h_scale || !w_scale)) return IG4_ERR_INVALID_ARG;
  const void *al[] = {h, w_qkv, g_q, g_k, rope_cos, rope_sin, q_out, k_out, vt_out};
  for (const void *p : al)
    if (!aligned16(p)) return IG4_ERR_INVALID_ARG;
  return launch_qkv(B, L, D, H, h, h_dtype, h_scale, w_qkv, w_scale, g_q, g_k, eps, rope_cos,
                    rope_sin, q_out, k_out, vt_out, vt_ld, as_stream(stream));
}

ig4_status ig4_joint_attention(int B, int H, int L, const void *q, const void *k, const void *vt,
                               int vt_ld, void *o_out, void *stream) {
  return ig4_joint_attention_ws(B, H, L, q, k, vt, vt_ld, o_out, nullptr, 0, stream);
}

size_t ig4_joint_attention_workspace_size(int B, int H, int L) {
  if (B < 1 || H < 1 || L < 1) return 0;
  return att_part_bytes(B, H, L);
}

ig4_status ig4_joint_attention_ws(int B, int H, int L, const void *q, const void *k,
                                  const void *vt, int vt_ld, void *o_out, void *workspace,
                                  size_t ws_bytes, void *stream) {
  if (B < 1 || H < 1 || L < 1 || !q || !k || !vt || !o_out || vt_ld < L || vt_ld % 8)
    return IG4_ERR_INVALID_ARG;
  if (H > 65535 || B > 65535) return IG4_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(vt) || !aligned16(o_out))
    return IG4_ERR_INVALID_ARG;
  if (workspace != nullptr) {
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return IG4_ERR_WORKSPACE;
    if (ws_bytes < att_part_bytes(B, H, L)) return IG4_ERR_WORKSPACE;
  }
  return launch_attention(B, H, L, q, k, vt, vt_ld, o_out, workspace, as_stream(stream));
}

ig4_status ig4_gated_residual_linear(int B, int L, int N, int K, const void *a, int a_dtype,
                                     const float *a_scale, const void *w, int w_dtype,
                                     const float *w_scale, const float *gate, int gate_stride,
                                     const void *x_res, void *x_out, int x_dtype, void *stream) {
  if (B < 1 || L < 1 || N < 1 || K < 1 || !a || !w || !gate || !x_res || !x_out ||
      gate_stride < N || gate_stride % 4)
    return IG4_ERR_INVALID_ARG;
  if (!valid_dtype_w(w_dtype) || !valid_dtype_x(x_dtype)) return IG4_ERR_INVALID_ARG;
  const bool f8 = is_fp8(w_dtype);
  if (a_dtype != (f8 ? IG4_E4M3 : IG4_BF16)) return IG4_ERR_UNSUPPORTED;
  if (f8 && (!a_scale || !w_scale)) return IG4_ERR_INVALID_ARG;
  if (N % 128 || K % (f8 ? 128 : 64)) return IG4_ERR_UNSUPPORTED;
  if (!aligned16(a) || !aligned16(w) || !aligned16(gate) || !aligned16(x_res) ||
      !aligned16(x_out))
    return IG4_ERR_INVALID_ARG;
  return launch_resid(B, L, N, K, a, f8, a_scale, w, w_scale, gate, gate_stride, x_res, x_out,
                      x_dtype, as_stream(stream));
}

ig4_status ig4_swiglu(int M, int I, int K, const void *h, int h_dtype, const float *h_scale,
                      const void *w_gate, const void *w_up, int w_dtype, const float *s_gate,
                      const float *s_up, void *u_out, void *stream) {
  if (M < 1 || I < 1 || K < 1 || !h || !w_gate || !w_up || !u_out) return IG4_ERR_INVALID_ARG;
  if (!valid_dtype_w(w_dtype)) return IG4_ERR_INVALID_ARG;
  const bool f8 = is_fp8(w_dtype);
  if (h_dtype != (f8 ? IG4_E4M3 : IG4_BF16)) return IG4_ERR_UNSUPPORTED;
  if (f8 && (!h_scale || !s_gate || !s_up)) return IG4_ERR_INVALID_ARG;
  if (I % 128 || K % (f8 ? 128 : 64)) return IG4_ERR_UNSUPPORTED;
  if (!aligned16(h) || !aligned16(w_gate) || !aligned16(w_up) || !aligned16(u_out))
    return IG4_ERR_INVALID_ARG;
  return launch_swiglu(M, I, K, h, f8, h_scale, w_gate, w_up, s_gate, s_up, u_out,
                       as_stream(stream));
}

ig4_status ig4_quantize_rows(int M, int K, const void *x, void *q_out, float *scale_out,
                             void *stream) {
  if (M < 1 || K < 8 || K % 8 || K > 16384 || !x || !q_out || !scale_out)
    return IG4_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(q_out)) return IG4_ERR_INVALID_ARG;
  return launch_quantize(M, K, x, q_out, scale_out, as_stream(stream));
}

ig4_status ig4_quantize_mx8(int M, int K, const void *x, void *codes_out, void *sf_out,
                            void *stream) {
  if (M < 1 || K < 128 || K % 128 || K > 65536 || !x || !codes_out || !sf_out)
    return IG4_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(codes_out)) return IG4_ERR_INVALID_ARG;
  return launch_mx8_quantize(M, K, x, codes_out, sf_out, as_stream(stream));
}

size_t ig4_mx8_scale_bytes(int M, int K) {
  if (M < 1 || K < 128 || K % 128) return 0;
  return mx8_sf_bytes(M, K);
}

size_t ig4_workspace_size(const ig4_config *cfg) {
  if (check_config(cfg) != IG4_OK) return 0;
  return block_ws_layout(cfg, nullptr).bytes;
}

static ig4_status block_forward_checked(const ig4_config *cfg, const ig4_block_weights *w,
                                        const void *x_in, void *x_out, const int32_t *pos,
                                        const float *temb, void *workspace, size_t ws_bytes,
                                        void *stream, void *const *events, int n_events) {
  IG4_TRY(check_config(cfg));
  IG4_TRY(check_block_weights(cfg, w));
  if (!x_in || !x_out || !pos || !temb || !workspace) return IG4_ERR_INVALID_ARG;
  if (!aligned16(x_in) || !aligned16(x_out) || !aligned16(temb)) return IG4_ERR_INVALID_ARG;
  if (n_events != 0 && (n_events != IG4_BLOCK_TRACE_EVENTS || !events)) return IG4_ERR_INVALID_ARG;
  const long L = cfg->T_text + static_cast<long>(cfg->grid_t) * cfg->grid_h * cfg->grid_w;
  const size_t xbytes = (cfg->x_dtype == IG4_F32 ? 4 : 2) * static_cast<size_t>(cfg->B) * L * cfg->D;
  const uint8_t *xi = static_cast<const uint8_t *>(x_in);
  const uint8_t *xo = static_cast<const uint8_t *>(x_out);
  if (xi < xo + xbytes && xo < xi + xbytes) return IG4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return IG4_ERR_WORKSPACE;
  const BlockWs ws = block_ws_layout(cfg, static_cast<uint8_t *>(workspace));
  if (ws_bytes < ws.bytes) return IG4_ERR_WORKSPACE;
  Tracer tr{events, n_events, 0, as_stream(stream)};
  return block_forward_impl(cfg, w, x_in, x_out, pos, temb, ws, as_stream(stream),
                            n_events ? &tr : nullptr);
}

ig4_status ig4_block_forward(const ig4_config *cfg, const ig4_block_weights *w, const void *x_in,
                             void *x_out, const int32_t *pos, const float *temb, void *workspace,
                             size_t ws_bytes, void *stream) {
  return block_forward_checked(cfg, w, x_in, x_out, pos, temb, workspace, ws_bytes, stream,
                               nullptr, 0);
}

ig4_status ig4_block_forward_traced(const ig4_config *cfg, const ig4_block_weights *w,
                                    const void *x_in, void *x_out, const int32_t *pos,
                                    const float *temb, void *workspace, size_t ws_bytes,
                                    void *stream, void *const *events, int n_events) {
  return block_forward_checked(cfg, w, x_in, x_out, pos, temb, workspace, ws_bytes, stream,
                               events, n_events);
}

size_t ig4_stack_workspace_size(const ig4_config *cfg, int latent_ch) {
  if (check_config(cfg) != IG4_OK || latent_ch < 128 || latent_ch % 128 ||
      cfg->x_dtype != IG4_BF16)
    return 0;
  return stack_ws_layout(cfg, latent_ch, nullptr).bytes;
}

}  // extern "C"

namespace {

// The stack on the caller's arguments; taps (may be empty) copy the sequence
// entering the listed blocks into caller buffers.
ig4_status stack_forward_checked(const ig4_config *cfg, const ig4_stack_weights *sw,
                                 const void *x_latent, const void *text, void *out_latent,
                                 const int32_t *pos, const float *temb, void *workspace,
                                 size_t ws_bytes, void *stream, const int *tap_blocks,
                                 void *const *tap_out, int n_taps) {
  IG4_TRY(check_config(cfg));
  if (!sw || !x_latent || !out_latent || !pos || !temb || !workspace) return IG4_ERR_INVALID_ARG;
  if (cfg->x_dtype != IG4_BF16) return IG4_ERR_UNSUPPORTED;
  const int C = sw->latent_ch;
  if (C < 128 || C % 128 || sw->n_blocks < 0 || (sw->n_blocks > 0 && !sw->blocks))
    return IG4_ERR_INVALID_ARG;
  const int N = cfg->grid_t * cfg->grid_h * cfg->grid_w;
  const int T = cfg->T_text;
  if (N < 1 || (T > 0 && !text)) return IG4_ERR_INVALID_ARG;
  const bool f8 = is_fp8(cfg->w_dtype);
  const void *need[] = {sw->w_in, sw->b_in, sw->w_f, sw->b_f, sw->w_out, sw->b_out};
  for (const void *p : need)
    if (!p || !aligned16(p)) return IG4_ERR_INVALID_ARG;
  if (f8 && (!sw->s_in || !sw->s_f || !sw->s_out)) return IG4_ERR_INVALID_ARG;
  for (int i = 0; i < sw->n_blocks; ++i) IG4_TRY(check_block_weights(cfg, &sw->blocks[i]));
  if (!aligned16(x_latent) || !aligned16(out_latent) || !aligned16(temb) ||
      (text && !aligned16(text)))
    return IG4_ERR_INVALID_ARG;
  if (n_taps < 0 || (n_taps > 0 && (!tap_blocks || !tap_out))) return IG4_ERR_INVALID_ARG;
  for (int t = 0; t < n_taps; ++t)
    if (tap_blocks[t] < 0 || tap_blocks[t] > sw->n_blocks || !tap_out[t] || !aligned16(tap_out[t]))
      return IG4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return IG4_ERR_WORKSPACE;
  const StackWs ws = stack_ws_layout(cfg, C, static_cast<uint8_t *>(workspace));
  if (ws_bytes < ws.bytes) return IG4_ERR_WORKSPACE;

  cudaStream_t st = as_stream(stream);
  const int L = T + N;
  const int D = cfg->D;
  const int B = cfg->B;
  const size_t seq_bytes = 2ull * B * L * D;  // the stack's stream is bf16
  // copy the sequence entering block i (i == n_blocks: after the last block)
  auto tap = [&](int i, const void *seq) -> ig4_status {
    for (int t = 0; t < n_taps; ++t)
      if (tap_blocks[t] == i &&
          cudaMemcpyAsync(tap_out[t], seq, seq_bytes, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return IG4_ERR_CUDA;
    return IG4_OK;
  };
  // [text | image] sequence in s0: the text prefix, then the latent in-projection.
  if (T > 0) {
    const int vpr = D * 2 / 16;
    const long total = static_cast<long>(B) * T * vpr;
    const int grid = static_cast<int>(std::min<long>((total + 255) / 256, 148L * 8));
    if (launch_pdl(copy_rows_kernel, dim3(grid), dim3(256), 0, st,
                   static_cast<const uint4 *>(text), static_cast<uint4 *>(ws.s0), T, L, 0, vpr,
                   total) != cudaSuccess)
      return IG4_ERR_CUDA;
    IG4_TRY(last_launch_status());
  }
  // The latent in/out projections are 0.01% of the step's work: they run in
  // bf16 (E4M3 weights decoded into the workspace) so that they add no
  // activation-quantisation error.
  const void *w_in = sw->w_in;
  const void *w_out = sw->w_out;
  if (f8) {
    IG4_TRY(launch_dequant(D, C, sw->w_in, sw->s_in, ws.w_in16, st));
    IG4_TRY(launch_dequant(C, D, sw->w_out, sw->s_out, ws.w_out16, st));
    w_in = ws.w_in16;
    w_out = ws.w_out16;
  }
  IG4_TRY(launch_linear_store(B * N, D, C, x_latent, false, nullptr, w_in, nullptr, sw->b_in,
                              ws.s0, IG4_BF16, D, N, L, T, st));
  void *cur = ws.s0;
  void *nxt = ws.s1;
  for (int i = 0; i < sw->n_blocks; ++i) {
    IG4_TRY(tap(i, cur));
    IG4_TRY(block_forward_impl(cfg, &sw->blocks[i], cur, nxt, pos, temb, ws.blk, st, nullptr,
                               i > 0));
    std::swap(cur, nxt);
  }
  IG4_TRY(tap(sw->n_blocks, cur));
  // Final layer on the image tokens: RMSNorm + (shift, scale), then D -> C.
  IG4_TRY(launch_adaln(B, cfg->adaln_dim, 2 * D, temb, sw->w_f, cfg->w_dtype, sw->s_f, sw->b_f,
                       ws.mod_f, st));
  IG4_TRY(launch_norm(B * N, L, D, cur, IG4_BF16, ws.mod_f, ws.mod_f + D, 2 * D, cfg->eps, ws.hf,
                      IG4_BF16, nullptr, N, L, T, st));
  IG4_TRY(launch_linear_store(B * N, C, D, ws.hf, false, nullptr, w_out, nullptr, sw->b_out,
                              out_latent, IG4_BF16, C, 0, 0, 0, st));
  return IG4_OK;
}

}  // namespace

extern "C" {

ig4_status ig4_stack_forward(const ig4_config *cfg, const ig4_stack_weights *sw,
                             const void *x_latent, const void *text, void *out_latent,
                             const int32_t *pos, const float *temb, void *workspace,
                             size_t ws_bytes, void *stream) {
  return stack_forward_checked(cfg, sw, x_latent, text, out_latent, pos, temb, workspace,
                               ws_bytes, stream, nullptr, nullptr, 0);
}

ig4_status ig4_stack_forward_tapped(const ig4_config *cfg, const ig4_stack_weights *sw,
                                    const void *x_latent, const void *text, void *out_latent,
                                    const int32_t *pos, const float *temb, void *workspace,
                                    size_t ws_bytes, void *stream, const int *tap_blocks,
                                    void *const *tap_out, int n_taps) {
  return stack_forward_checked(cfg, sw, x_latent, text, out_latent, pos, temb, workspace,
                               ws_bytes, stream, tap_blocks, tap_out, n_taps);
}

// ----------------------------------------------------------------- NVFP4


size_t ig4_nvfp4_scale_bytes(int rows, int K) {
  if (rows < 1 || K < 64 || K % 64) return 0;
  return static_cast<size_t>((rows + 127) / 128) * (K / 64) * 512;
}

ig4_status ig4_nvfp4_pack_scales(int rows, int K, const void *sf_rows, void *sf_packed,
                                 void *stream) {
  if (rows < 1 || K < 64 || K % 64 || !sf_rows || !sf_packed) return IG4_ERR_INVALID_ARG;
  const long total = static_cast<long>(ig4_nvfp4_scale_bytes(rows, K));
  DeviceInfo *di = nullptr;
  IG4_TRY(device_info(&di));
  const int grid = static_cast<int>(std::min<long>((total + 255) / 256, 8L * di->sms));
  nvf4_pack_scales_kernel<<<grid, 256, 0, as_stream(stream)>>>(
      static_cast<const uint8_t *>(sf_rows), static_cast<uint8_t *>(sf_packed), rows, K, total);
  return last_launch_status();
}

ig4_status ig4_nvfp4_linear(int M, int N, int K, const void *a_codes, const void *a_sf,
                            const float *a_scale, const void *w_codes, const void *w_sf,
                            const float *w_scale, const float *bias, void *out, int out_dtype,
                            void *stream) {
  if (M < 1 || N < 128 || N % 128 || K < 256 || K % 256) return IG4_ERR_INVALID_ARG;
  if (out_dtype != IG4_F32 && out_dtype != IG4_BF16) return IG4_ERR_INVALID_ARG;
  const void *ptrs[] = {a_codes, a_sf, a_scale, w_codes, w_sf, w_scale, out};
  for (const void *p : ptrs)
    if (!p || !aligned16(p)) return IG4_ERR_INVALID_ARG;
  if (bias && !aligned16(bias)) return IG4_ERR_INVALID_ARG;
  DeviceInfo *di = nullptr;
  IG4_TRY(device_info(&di));
  // CTA pairs with 256 x 256 tiles (half the B bytes per CTA) for more than one
  // 128-row block; else single CTAs with 256-wide tiles (one accumulator) once
  // there are two waves of them, or 128-wide tiles
  if (N % 256 == 0 && M > GEMM_BM)
    return launch_nvf4_pair(M, N, K, a_codes, a_sf, a_scale, w_codes, w_sf, w_scale, bias, out,
                            out_dtype, as_stream(stream));
  const long tiles256 = static_cast<long>((M + GEMM_BM - 1) / GEMM_BM) * (N / 256);
  if (N % 256 == 0 && tiles256 >= 2L * di->sms)
    return launch_nvf4<256>(M, N, K, a_codes, a_sf, a_scale, w_codes, w_sf, w_scale, bias, out,
                            out_dtype, di->sms, as_stream(stream));
  return launch_nvf4<128>(M, N, K, a_codes, a_sf, a_scale, w_codes, w_sf, w_scale, bias, out,
                          out_dtype, di->sms, as_stream(stream));
}

ig4_status ig4_nvfp4_quantize(int M, int K, const void *x, void *codes, void *sf_packed,
                              float *row_scale, void *stream) {
  if (M < 1 || K < 64 || K % 64) return IG4_ERR_INVALID_ARG;
  const void *ptrs[] = {x, codes, sf_packed, row_scale};
  for (const void *p : ptrs)
    if (!p || !aligned16(p)) return IG4_ERR_INVALID_ARG;
  return launch_nvf4_quantize(M, K, x, codes, sf_packed, row_scale, as_stream(stream));
}

// --------------------------------------------------- text conditioning

size_t ig4_text_cond_workspace_size(int M, int K_raw, int w_dtype) {
  if (M < 1 || K_raw < 128 || K_raw % 128 || !valid_dtype_w(w_dtype)) return 0;
  const size_t es = is_fp8(w_dtype) ? 1 : 2;
  return round_up(es * M * static_cast<size_t>(K_raw), 256) +
         round_up(sizeof(float) * static_cast<size_t>(M), 256);
}

ig4_status ig4_text_cond_project(int M, int K_raw, int D, const float *raw, const float *g_norm,
                                 float eps, const void *w_proj, const float *w_scale, int w_dtype,
                                 const float *b_proj, void *text_out, void *workspace,
                                 size_t ws_bytes, void *stream) {
  if (M < 1 || K_raw < 128 || K_raw % 128 || D < 128 || D % 128 || !(eps > 0.0f))
    return IG4_ERR_INVALID_ARG;
  if (!valid_dtype_w(w_dtype)) return IG4_ERR_INVALID_ARG;
  const bool f8 = is_fp8(w_dtype);
  if (!raw || !g_norm || !w_proj || !b_proj || !text_out || !workspace || (f8 && !w_scale))
    return IG4_ERR_INVALID_ARG;
  const void *ptrs[] = {raw, g_norm, w_proj, b_proj, text_out};
  for (const void *p : ptrs)
    if (!aligned16(p)) return IG4_ERR_INVALID_ARG;
  if (f8 && !aligned16(w_scale)) return IG4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return IG4_ERR_WORKSPACE;
  if (ws_bytes < ig4_text_cond_workspace_size(M, K_raw, w_dtype)) return IG4_ERR_WORKSPACE;
  cudaStream_t st = as_stream(stream);
  uint8_t *h = static_cast<uint8_t *>(workspace);
  float *h_scale = reinterpret_cast<float *>(
      h + round_up((f8 ? 1 : 2) * static_cast<size_t>(M) * K_raw, 256));
  // llm_cond_norm: RMSNorm over the concatenated features, into bf16 / E4M3
  const cudaError_t e =
      f8 ? launch_pdl(wide_rmsnorm_kernel<true>, dim3(M), dim3(WIDE_NORM_THREADS), 0, st, raw,
                      g_norm, K_raw, eps, static_cast<void *>(h), h_scale)
         : launch_pdl(wide_rmsnorm_kernel<false>, dim3(M), dim3(WIDE_NORM_THREADS), 0, st, raw,
                      g_norm, K_raw, eps, static_cast<void *>(h), static_cast<float *>(nullptr));
  if (e != cudaSuccess) return IG4_ERR_CUDA;
  IG4_TRY(last_launch_status());
  // llm_cond_proj: K_raw -> D with bias, bf16 out
  if (f8) return launch_store_bf16<true>(M, D, K_raw, h, h_scale, w_proj, w_scale, b_proj, text_out, st);
  return launch_store_bf16<false>(M, D, K_raw, h, nullptr, w_proj, nullptr, b_proj, text_out, st);
}

// ---------------------------------------------------------------- sampler

ig4_status ig4_flow_schedule(int num_steps, double mu_base, double std_dev, int height_px,
                             int width_px, double *t_out) {
  if (num_steps < 1 || num_steps > 100000 || !(std_dev > 0.0) || !std::isfinite(mu_base) ||
      !std::isfinite(std_dev) || height_px < 1 || width_px < 1 || !t_out)
    return IG4_ERR_INVALID_ARG;
  const double mu =
      mu_base + 0.5 * std::log(static_cast<double>(height_px) * static_cast<double>(width_px) /
                               (512.0 * 512.0));
  t_out[0] = 1.0;
  t_out[num_steps] = 0.0;
  for (int i = 1; i < num_steps; ++i) {
    // the (1 - i/N) quantile: Phi^-1(1 - q) = -Phi^-1(q), q = i/N
    const double x = -normal_quantile(static_cast<double>(i) / num_steps);
    t_out[i] = 1.0 / (1.0 + std::exp(-(mu + std_dev * x)));
  }
  return IG4_OK;
}

ig4_status ig4_guidance_schedule(int num_steps, int n_polish, float gw_main, float gw_polish,
                                 float *gw_out) {
  if (num_steps < 1 || n_polish < 0 || n_polish > num_steps || !gw_out ||
      !std::isfinite(gw_main) || !std::isfinite(gw_polish))
    return IG4_ERR_INVALID_ARG;
  for (int i = 0; i < num_steps; ++i) gw_out[i] = i < num_steps - n_polish ? gw_main : gw_polish;
  return IG4_OK;
}

ig4_status ig4_cfg_euler(long long n, const void *v_cond, const void *v_uncond, float gw, float dt,
                         const float *z_in, float *z_out, void *z16_out, void *stream) {
  if (n < 0 || n % 8 || !z_in || (!z_out && !z16_out) || (!v_cond) != (!v_uncond) ||
      (v_cond && !z_out))
    return IG4_ERR_INVALID_ARG;
  const void *ptrs[] = {v_cond, v_uncond, z_in, z_out, z16_out};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return IG4_ERR_INVALID_ARG;
  if (!std::isfinite(gw) || !std::isfinite(dt)) return IG4_ERR_INVALID_ARG;
  if (n == 0) return IG4_OK;
  DeviceInfo *di = nullptr;
  IG4_TRY(device_info(&di));
  const long n8 = n / 8;
  const int grid = static_cast<int>(std::min<long>((n8 + 255) / 256, 8L * di->sms));
  if (launch_pdl(cfg_euler_kernel, dim3(grid), dim3(256), 0, as_stream(stream),
                 static_cast<const uint4 *>(v_cond), static_cast<const uint4 *>(v_uncond), gw, dt,
                 reinterpret_cast<const float4 *>(z_in), reinterpret_cast<float4 *>(z_out),
                 static_cast<uint4 *>(z16_out), n8) != cudaSuccess)
    return IG4_ERR_CUDA;
  return last_launch_status();
}

namespace {
struct DenoiseWs {
  void *z16, *v_c, *v_u;
  uint8_t *stack;
  size_t bytes;
};

DenoiseWs denoise_ws_layout(const ig4_config *c, int C, uint8_t *base) {
  DenoiseWs w{};
  const size_t lat = round_up(2ull * c->B * c->grid_t * c->grid_h * c->grid_w * C, 256);
  w.z16 = base;
  w.v_c = base ? base + lat : nullptr;
  w.v_u = base ? base + 2 * lat : nullptr;
  w.stack = base ? base + 3 * lat : nullptr;
  w.bytes = 3 * lat + stack_ws_layout(c, C, nullptr).bytes;
  return w;
}
}  // namespace

size_t ig4_denoise_workspace_size(const ig4_config *cfg, int latent_ch) {
  if (ig4_stack_workspace_size(cfg, latent_ch) == 0) return 0;
  return denoise_ws_layout(cfg, latent_ch, nullptr).bytes;
}

ig4_status ig4_denoise_step(const ig4_config *cfg, const ig4_stack_weights *cond,
                            const ig4_stack_weights *uncond, float *z, const void *text,
                            const int32_t *pos_cond, const int32_t *pos_uncond,
                            const float *temb_cond, const float *temb_uncond, float t_cur,
                            float t_next, float gw, void *workspace, size_t ws_bytes,
                            void *stream) {
  IG4_TRY(check_config(cfg));
  if (!cond || !uncond || !z || !pos_cond || !pos_uncond || !temb_cond || !temb_uncond ||
      !workspace)
    return IG4_ERR_INVALID_ARG;
  if (cfg->x_dtype != IG4_BF16) return IG4_ERR_UNSUPPORTED;
  const int C = cond->latent_ch;
  if (uncond->latent_ch != C || C < 128 || C % 128) return IG4_ERR_INVALID_ARG;
  if (!std::isfinite(t_cur) || !std::isfinite(t_next) || !std::isfinite(gw))
    return IG4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return IG4_ERR_WORKSPACE;
  const DenoiseWs ws = denoise_ws_layout(cfg, C, static_cast<uint8_t *>(workspace));
  if (ws_bytes < ws.bytes) return IG4_ERR_WORKSPACE;
  const size_t stack_bytes = ws_bytes - (ws.stack - static_cast<uint8_t *>(workspace));
  const long long n = static_cast<long long>(cfg->B) * cfg->grid_t * cfg->grid_h * cfg->grid_w * C;
  // the stacks read the latent in bf16
  IG4_TRY(ig4_cfg_euler(n, nullptr, nullptr, 0.0f, 0.0f, z, nullptr, ws.z16, stream));
  // conditional transformer over [text | image]
  IG4_TRY(ig4_stack_forward(cfg, cond, ws.z16, text, ws.v_c, pos_cond, temb_cond, ws.stack,
                            stack_bytes, stream));
  // separate unconditional transformer over the image tokens alone
  ig4_config cu = *cfg;
  cu.T_text = 0;
  IG4_TRY(ig4_stack_forward(&cu, uncond, ws.z16, nullptr, ws.v_u, pos_uncond, temb_uncond,
                            ws.stack, stack_bytes, stream));
  // v = v_u + gw (v_c - v_u); z += (t_cur - t_next) v
  return ig4_cfg_euler(n, ws.v_c, ws.v_u, gw, t_cur - t_next, z, z, nullptr, stream);
}

}  // extern "C"

// ------------------------------------------------------ multi-GPU layouts
// Tensor parallelism over heads (TP) and Ulysses sequence parallelism over
// image tokens (SP), "SGLang cookbook: Ideogram 4", section 3.  The library
// computes each rank's share and packs / reduces the exchanged data; the
// transfers between GPUs are the caller's collectives (or peer-mapped
// pointers handed to ig4_tp_reduce).
namespace {

constexpr int SP_MAX_RANKS = 8;

// Image tokens [*off, *off + *cnt) of Ulysses rank r of P: contiguous shares
// in the grid's row-major order, the first N % P ranks one token more.
void sp_range(long N, int P, int r, long *off, long *cnt) {
  const long base = N / P, rem = N % P;
  *cnt = base + (r < rem ? 1 : 0);
  *off = r * base + std::min<long>(r, rem);
}

ig4_status check_tp(const ig4_config *c, int rank, int size) {
  IG4_TRY(check_config(c));
  if (size < 1 || size > TP_MAX_RANKS || rank < 0 || rank >= size) return IG4_ERR_INVALID_ARG;
  if (c->H % size != 0 || c->I % size != 0 || (c->I / size) % 128 != 0) return IG4_ERR_UNSUPPORTED;
  if (is_nvf4_mixed(c->w_dtype)) return IG4_ERR_UNSUPPORTED;
  return IG4_OK;
}

// A TP shard's block: H / size heads, I / size FFN columns, full width D.
ig4_config tp_local(const ig4_config *c, int size) {
  ig4_config t = *c;
  t.H = c->H / size;
  t.I = c->I / size;
  return t;
}

// TP partial output [B*L][D] fp32: (x_res or 0) + gate * (a W^T), 256-wide tiles.
template <typename XT>
ig4_status launch_partial_t(int B, int L, int N, int K, const void *a, bool f8,
                            const float *a_scale, const void *w, const float *w_scale,
                            const float *gate, int gate_stride, const void *x_res, float *out,
                            cudaStream_t st) {
  const int M = B * L;
  CUtensorMap ma, mb;
  IG4_TRY(gemm_maps(&ma, &mb, a, w, f8 ? 1 : 2, M, N, K, b_box_rows(256, M)));
  if (f8) {
    EpiResidGate<256, true, XT, float> e{static_cast<const XT *>(x_res), out, gate, gate_stride,
                                         L, M, N, a_scale, w_scale};
    return launch_gemm<256, true, false>(ma, mb, mb, M, N / 256, K, e, st);
  }
  EpiResidGate<256, false, XT, float> e{static_cast<const XT *>(x_res), out, gate, gate_stride, L,
                                        M, N, nullptr, nullptr};
  return launch_gemm<256, false, false>(ma, mb, mb, M, N / 256, K, e, st);
}

ig4_status launch_partial(int B, int L, int N, int K, const void *a, bool f8, const float *a_scale,
                          const void *w, const float *w_scale, const float *gate, int gate_stride,
                          const void *x_res, int x_dtype, float *out, cudaStream_t st) {
  if (x_dtype == IG4_F32)
    return launch_partial_t<float>(B, L, N, K, a, f8, a_scale, w, w_scale, gate, gate_stride,
                                   x_res, out, st);
  return launch_partial_t<__nv_bfloat16>(B, L, N, K, a, f8, a_scale, w, w_scale, gate,
                                         gate_stride, x_res, out, st);
}

ig4_status check_tp_call(const ig4_config *cfg, int rank, int size, const ig4_block_weights *w,
                         const void *x, const float *partial, const void *workspace,
                         size_t ws_bytes, BlockWs *ws) {
  IG4_TRY(check_tp(cfg, rank, size));
  IG4_TRY(check_block_weights(cfg, w));
  if (!x || !partial || !workspace || !aligned16(x) || !aligned16(partial))
    return IG4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return IG4_ERR_WORKSPACE;
  const ig4_config t = tp_local(cfg, size);
  *ws = block_ws_layout(&t, static_cast<uint8_t *>(const_cast<void *>(workspace)));
  if (ws_bytes < ws->bytes) return IG4_ERR_WORKSPACE;
  return IG4_OK;
}

// ----------------------------------------------------------- Ulysses SP

ig4_status check_sp(const ig4_config *c, int rank, int size) {
  IG4_TRY(check_config(c));
  if (size < 1 || size > SP_MAX_RANKS || rank < 0 || rank >= size) return IG4_ERR_INVALID_ARG;
  if (c->H % size != 0) return IG4_ERR_UNSUPPORTED;
  const long N = static_cast<long>(c->grid_t) * c->grid_h * c->grid_w;
  if (N < size) return IG4_ERR_UNSUPPORTED;  // every rank holds image tokens
  return IG4_OK;
}

// The block a Ulysses rank runs outside attention: the text tokens and its
// share of the image tokens, as one flat image row.
ig4_config sp_local(const ig4_config *c, int size, int rank) {
  long off = 0, cnt = 0;
  sp_range(static_cast<long>(c->grid_t) * c->grid_h * c->grid_w, size, rank, &off, &cnt);
  ig4_config t = *c;
  t.grid_t = 1;
  t.grid_h = 1;
  t.grid_w = static_cast<int>(cnt);
  return t;
}

struct SpWs {
  BlockWs loc;            // the local block's buffers (q, k, vt, o of the local tokens)
  void *qg, *kg, *vtg;    // the rank's head group over all L tokens
  void *og;               // attention output of the head group [B*L][Hg*256]
  void *part;             // its attention partial slots (or nullptr)
  int vtg_ld;
  size_t bytes;
};

SpWs sp_ws_layout(const ig4_config *c, int size, int rank, uint8_t *base) {
  SpWs w{};
  const ig4_config t = sp_local(c, size, rank);
  w.loc = block_ws_layout(&t, base);
  size_t off = w.loc.bytes;
  const long L = c->T_text + static_cast<long>(c->grid_t) * c->grid_h * c->grid_w;
  const long Hg = c->H / size;
  w.vtg_ld = static_cast<int>(round_up(L, 8));
  auto take = [&](size_t n) -> uint8_t * {
    uint8_t *p = base ? base + off : nullptr;
    off += round_up(n, 256);
    return p;
  };
  w.qg = take(2 * c->B * Hg * L * 256);
  w.kg = take(2 * c->B * Hg * L * 256);
  w.vtg = take(2 * c->B * Hg * 256 * static_cast<long>(w.vtg_ld));
  w.og = take(2 * c->B * L * Hg * 256);
  const size_t pb = att_part_bytes(c->B, static_cast<int>(Hg), static_cast<int>(L));
  w.part = pb ? take(pb) : nullptr;
  w.bytes = off;
  return w;
}

// Bytes of one exchange chunk from rank s to rank d.  Phase 0 (before
// attention): q, k [B][Hg][N_s][256] and v^T [B][Hg][256][N_s] of d's head
// group over s's image tokens.  Phase 1 (after attention): o [B][T + N_d]
// [Hg*256] of s's head group over d's text and image tokens.
size_t sp_chunk_bytes(const ig4_config *c, int size, int phase, int s, int d) {
  const long N = static_cast<long>(c->grid_t) * c->grid_h * c->grid_w;
  long off = 0, cnt = 0;
  sp_range(N, size, phase == 0 ? s : d, &off, &cnt);
  const long Hg = c->H / size;
  if (phase == 0) return 3ull * 2 * c->B * Hg * cnt * 256;
  return 2ull * c->B * (c->T_text + cnt) * Hg * 256;
}

// Offset of the chunk for (s, d) in s's send buffer (chunks ordered by d)
// or in d's receive buffer (ordered by s).
size_t sp_chunk_offset(const ig4_config *c, int size, int phase, int s, int d, bool in_send) {
  size_t off = 0;
  for (int k = 0; k < (in_send ? d : s); ++k)
    off += in_send ? sp_chunk_bytes(c, size, phase, s, k) : sp_chunk_bytes(c, size, phase, k, d);
  return off;
}

struct JobList {
  CopyJobs jobs;
  int n = 0;
  bool overflow = false;
  // element offsets and strides; bases are 2-byte element pointers
  void add(const void *src, long long src_off, void *dst, long long dst_off, int n_b, int n_h,
           int rows, int row_elems, long long s_b, long long s_h, long long s_r, long long d_b,
           long long d_h, long long d_r) {
    if (n_b < 1 || n_h < 1 || rows < 1 || row_elems < 1) return;
    if (n >= EXCHANGE_MAX_JOBS) {
      overflow = true;
      return;
    }
    CopyJob &j = jobs.j[n++];
    j.src = static_cast<const uint16_t *>(src) + src_off;
    j.dst = static_cast<uint16_t *>(dst) + dst_off;
    j.n_b = n_b;
    j.n_h = n_h;
    j.rows = rows;
    j.row_elems = row_elems;
    j.s_b = s_b;
    j.s_h = s_h;
    j.s_r = s_r;
    j.d_b = d_b;
    j.d_h = d_h;
    j.d_r = d_r;
    const long long all = (s_b | s_h | s_r | d_b | d_h | d_r | row_elems);
    j.vec = (all % 8 == 0) && aligned16(j.src) && aligned16(j.dst);
  }
  ig4_status launch(cudaStream_t st, int sms) const {
    if (overflow) return IG4_ERR_UNSUPPORTED;
    if (n == 0) return IG4_OK;
    long most = 0;
    for (int i = 0; i < n; ++i) {
      const CopyJob &j = jobs.j[i];
      const long units = static_cast<long>(j.n_b) * j.n_h * j.rows * (j.vec ? j.row_elems / 8 : j.row_elems);
      most = std::max(most, units);
    }
    const int gx = static_cast<int>(std::max<long>(1, std::min<long>((most + 255) / 256, 4L * sms)));
    if (launch_pdl(exchange_copy_kernel, dim3(gx, n), dim3(256), 0, st, jobs) != cudaSuccess)
      return IG4_ERR_CUDA;
    return last_launch_status();
  }
};

}  // namespace

extern "C" {

size_t ig4_tp_workspace_size(const ig4_config *cfg, int tp_size) {
  if (check_tp(cfg, 0, tp_size) != IG4_OK) return 0;
  const ig4_config t = tp_local(cfg, tp_size);
  return block_ws_layout(&t, nullptr).bytes;
}

ig4_status ig4_block_tp_attention(const ig4_config *cfg, int tp_rank, int tp_size,
                                  const ig4_block_weights *w, const void *x_in,
                                  const int32_t *pos, const float *temb, float *partial,
                                  void *workspace, size_t ws_bytes, void *stream) {
  BlockWs ws;
  IG4_TRY(check_tp_call(cfg, tp_rank, tp_size, w, x_in, partial, workspace, ws_bytes, &ws));
  if (!pos || !temb || !aligned16(temb)) return IG4_ERR_INVALID_ARG;
  const ig4_config t = tp_local(cfg, tp_size);
  const int L = cfg->T_text + cfg->grid_t * cfg->grid_h * cfg->grid_w;
  const int M = cfg->B * L;
  const int D = cfg->D;
  const int Ks = t.H * 256;  // this shard's attention output width
  const bool f8 = is_fp8(cfg->w_dtype);
  cudaStream_t st = as_stream(stream);
  Tracer none{nullptr, 0, 0, st};
  IG4_TRY(block_pre_attention(&t, w, x_in, pos, temb, ws, st, none, false));
  IG4_TRY(launch_attention(cfg->B, t.H, L, ws.q, ws.k, ws.vt, ws.vt_ld, ws.o, ws.att_part, st));
  if (f8) IG4_TRY(launch_quantize(M, Ks, ws.o, ws.oq, ws.o_scale, st));
  return launch_partial(cfg->B, L, D, Ks, f8 ? ws.oq : ws.o, f8, ws.o_scale, w->w_o, w->s_o,
                        ws.mod + 2 * D, 6 * D, tp_rank == 0 ? x_in : nullptr, cfg->x_dtype,
                        partial, st);
}

ig4_status ig4_block_tp_mlp(const ig4_config *cfg, int tp_rank, int tp_size,
                            const ig4_block_weights *w, const void *x1, float *partial,
                            void *workspace, size_t ws_bytes, void *stream) {
  BlockWs ws;
  IG4_TRY(check_tp_call(cfg, tp_rank, tp_size, w, x1, partial, workspace, ws_bytes, &ws));
  const ig4_config t = tp_local(cfg, tp_size);
  const int L = cfg->T_text + cfg->grid_t * cfg->grid_h * cfg->grid_w;
  const int M = cfg->B * L;
  const int D = cfg->D, Is = t.I;
  const bool f8 = is_fp8(cfg->w_dtype);
  const int hdt = f8 ? IG4_E4M3 : IG4_BF16;
  cudaStream_t st = as_stream(stream);
  IG4_TRY(launch_norm(M, L, D, x1, cfg->x_dtype, ws.mod + 3 * D, ws.mod + 4 * D, 6 * D, cfg->eps,
                      ws.h, hdt, ws.h_scale, 0, 0, 0, st));
  IG4_TRY(launch_swiglu(M, Is, D, ws.h, f8, ws.h_scale, w->w_gate, w->w_up, w->s_gate, w->s_up,
                        ws.u, st));
  if (f8) IG4_TRY(launch_quantize(M, Is, ws.u, ws.uq, ws.u_scale, st));
  return launch_partial(cfg->B, L, D, Is, f8 ? ws.uq : ws.u, f8, ws.u_scale, w->w_down,
                        w->s_down, ws.mod + 5 * D, 6 * D, tp_rank == 0 ? x1 : nullptr,
                        cfg->x_dtype, partial, st);
}

ig4_status ig4_tp_reduce(long long n, int n_src, const float *const *src, void *out,
                         int out_dtype, void *stream) {
  if (n < 0 || n % 8 || n_src < 1 || n_src > TP_MAX_RANKS || !src || !out || !aligned16(out))
    return IG4_ERR_INVALID_ARG;
  if (out_dtype != IG4_F32 && out_dtype != IG4_BF16) return IG4_ERR_INVALID_ARG;
  TpSources ps{};
  for (int r = 0; r < n_src; ++r) {
    if (!src[r] || !aligned16(src[r])) return IG4_ERR_INVALID_ARG;
    ps.p[r] = src[r];
  }
  if (n == 0) return IG4_OK;
  DeviceInfo *di = nullptr;
  IG4_TRY(device_info(&di));
  const long n8 = n / 8;
  const int grid = static_cast<int>(std::min<long>((n8 + 255) / 256, 8L * di->sms));
  const cudaError_t e =
      out_dtype == IG4_F32
          ? launch_pdl(tp_reduce_kernel<float>, dim3(grid), dim3(256), 0, as_stream(stream), ps,
                       n_src, static_cast<float *>(out), n8)
          : launch_pdl(tp_reduce_kernel<__nv_bfloat16>, dim3(grid), dim3(256), 0,
                       as_stream(stream), ps, n_src, static_cast<__nv_bfloat16 *>(out), n8);
  if (e != cudaSuccess) return IG4_ERR_CUDA;
  return last_launch_status();
}

ig4_status ig4_sp_image_range(const ig4_config *cfg, int sp_size, int sp_rank, int *img_off,
                              int *img_count) {
  IG4_TRY(check_sp(cfg, sp_rank, sp_size));
  if (!img_off || !img_count) return IG4_ERR_INVALID_ARG;
  long off = 0, cnt = 0;
  sp_range(static_cast<long>(cfg->grid_t) * cfg->grid_h * cfg->grid_w, sp_size, sp_rank, &off,
           &cnt);
  *img_off = static_cast<int>(off);
  *img_count = static_cast<int>(cnt);
  return IG4_OK;
}

ig4_status ig4_sp_positions(const ig4_config *cfg, int sp_size, int sp_rank, int32_t *pos_out,
                            int out_on_device, void *stream) {
  IG4_TRY(check_sp(cfg, sp_rank, sp_size));
  if (!pos_out) return IG4_ERR_INVALID_ARG;
  long off = 0, cnt = 0;
  sp_range(static_cast<long>(cfg->grid_t) * cfg->grid_h * cfg->grid_w, sp_size, sp_rank, &off,
           &cnt);
  const int T = cfg->T_text;
  const long Ls = T + cnt;
  if (out_on_device) {
    if (!aligned16(pos_out)) return IG4_ERR_INVALID_ARG;
    mrope_positions_kernel<<<static_cast<int>((Ls + 255) / 256), 256, 0, as_stream(stream)>>>(
        T, cfg->grid_t, cfg->grid_h, cfg->grid_w, static_cast<int>(off), static_cast<int>(cnt),
        pos_out);
    return last_launch_status();
  }
  const long hw = static_cast<long>(cfg->grid_h) * cfg->grid_w;
  for (long l = 0; l < T; ++l)
    pos_out[l] = pos_out[Ls + l] = pos_out[2 * Ls + l] = static_cast<int32_t>(l);
  for (long i = 0; i < cnt; ++i) {
    const long n = off + i;
    const long tt = n / hw, rem = n % hw;
    pos_out[T + i] = static_cast<int32_t>(T + tt);
    pos_out[Ls + T + i] = static_cast<int32_t>(T + rem / cfg->grid_w);
    pos_out[2 * Ls + T + i] = static_cast<int32_t>(T + rem % cfg->grid_w);
  }
  return IG4_OK;
}

size_t ig4_sp_workspace_size(const ig4_config *cfg, int sp_size, int sp_rank) {
  if (check_sp(cfg, sp_rank, sp_size) != IG4_OK) return 0;
  return sp_ws_layout(cfg, sp_size, sp_rank, nullptr).bytes;
}

size_t ig4_sp_exchange_bytes(const ig4_config *cfg, int sp_size, int phase, int src_rank,
                             int dst_rank) {
  if (check_sp(cfg, 0, sp_size) != IG4_OK || (phase != 0 && phase != 1) || src_rank < 0 ||
      src_rank >= sp_size || dst_rank < 0 || dst_rank >= sp_size)
    return 0;
  return sp_chunk_bytes(cfg, sp_size, phase, src_rank, dst_rank);
}

ig4_status ig4_block_sp_pre(const ig4_config *cfg, int sp_rank, int sp_size,
                            const ig4_block_weights *w, const void *x_local,
                            const int32_t *pos_local, const float *temb, void *send,
                            void *workspace, size_t ws_bytes, void *stream) {
  IG4_TRY(check_sp(cfg, sp_rank, sp_size));
  IG4_TRY(check_block_weights(cfg, w));
  if (!x_local || !pos_local || !temb || !send || !workspace) return IG4_ERR_INVALID_ARG;
  if (!aligned16(x_local) || !aligned16(temb) || !aligned16(send)) return IG4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return IG4_ERR_WORKSPACE;
  const SpWs ws = sp_ws_layout(cfg, sp_size, sp_rank, static_cast<uint8_t *>(workspace));
  if (ws_bytes < ws.bytes) return IG4_ERR_WORKSPACE;
  DeviceInfo *di = nullptr;
  IG4_TRY(device_info(&di));
  cudaStream_t st = as_stream(stream);
  const ig4_config t = sp_local(cfg, sp_size, sp_rank);
  Tracer none{nullptr, 0, 0, st};
  IG4_TRY(block_pre_attention(&t, w, x_local, pos_local, temb, ws.loc, st, none, false));
  // pack: to rank d, head group d of q, k, v^T over this rank's image tokens
  const int T = cfg->T_text, B = cfg->B, H = cfg->H, Hg = H / sp_size;
  const long Ls = T + t.grid_w, Ns = t.grid_w;
  const long vld = ws.loc.vt_ld;
  JobList jl;
  for (int d = 0; d < sp_size; ++d) {
    uint8_t *ch = static_cast<uint8_t *>(send) + sp_chunk_offset(cfg, sp_size, 0, sp_rank, d, true);
    const long part = static_cast<long>(B) * Hg * Ns * 256;  // elements per part
    for (int which = 0; which < 2; ++which)
      jl.add(which == 0 ? ws.loc.q : ws.loc.k, (static_cast<long>(d) * Hg * Ls + T) * 256,
             ch + which * 2 * part, 0, B, Hg, static_cast<int>(Ns), 256, H * Ls * 256, Ls * 256,
             256, Hg * Ns * 256, Ns * 256, 256);
    jl.add(ws.loc.vt, static_cast<long>(d) * Hg * 256 * vld + T, ch + 2 * 2 * part, 0, B, Hg, 256,
           static_cast<int>(Ns), H * 256 * vld, 256 * vld, vld, Hg * 256 * Ns, 256 * Ns, Ns);
  }
  return jl.launch(st, di->sms);
}

ig4_status ig4_block_sp_attention(const ig4_config *cfg, int sp_rank, int sp_size,
                                  const void *recv, void *send_o, void *workspace,
                                  size_t ws_bytes, void *stream) {
  IG4_TRY(check_sp(cfg, sp_rank, sp_size));
  if (!recv || !send_o || !workspace || !aligned16(recv) || !aligned16(send_o))
    return IG4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return IG4_ERR_WORKSPACE;
  const SpWs ws = sp_ws_layout(cfg, sp_size, sp_rank, static_cast<uint8_t *>(workspace));
  if (ws_bytes < ws.bytes) return IG4_ERR_WORKSPACE;
  DeviceInfo *di = nullptr;
  IG4_TRY(device_info(&di));
  cudaStream_t st = as_stream(stream);
  const int T = cfg->T_text, B = cfg->B, H = cfg->H, Hg = H / sp_size, r = sp_rank;
  const long N = static_cast<long>(cfg->grid_t) * cfg->grid_h * cfg->grid_w;
  const long L = T + N;
  const ig4_config t = sp_local(cfg, sp_size, r);
  const long Ls = T + t.grid_w;
  const long vld = ws.loc.vt_ld, gld = ws.vtg_ld;
  // unpack: text rows from this rank's own q, k, v^T (head group r), image
  // rows of every source rank from its chunk
  JobList jl;
  for (int which = 0; which < 2; ++which)
    jl.add(which == 0 ? ws.loc.q : ws.loc.k, static_cast<long>(r) * Hg * Ls * 256,
           which == 0 ? ws.qg : ws.kg, 0, B, Hg, T, 256, H * Ls * 256, Ls * 256, 256,
           Hg * L * 256, L * 256, 256);
  jl.add(ws.loc.vt, static_cast<long>(r) * Hg * 256 * vld, ws.vtg, 0, B, Hg, 256, T,
         H * 256 * vld, 256 * vld, vld, Hg * 256 * gld, 256 * gld, gld);
  for (int s = 0; s < sp_size; ++s) {
    long off = 0, Ns = 0;
    sp_range(N, sp_size, s, &off, &Ns);
    const uint8_t *ch =
        static_cast<const uint8_t *>(recv) + sp_chunk_offset(cfg, sp_size, 0, s, r, false);
    const long part = static_cast<long>(B) * Hg * Ns * 256;
    for (int which = 0; which < 2; ++which)
      jl.add(ch + which * 2 * part, 0, which == 0 ? ws.qg : ws.kg, (T + off) * 256, B, Hg,
             static_cast<int>(Ns), 256, Hg * Ns * 256, Ns * 256, 256, Hg * L * 256, L * 256, 256);
    jl.add(ch + 2 * 2 * part, 0, ws.vtg, T + off, B, Hg, 256, static_cast<int>(Ns),
           Hg * 256 * Ns, 256 * Ns, Ns, Hg * 256 * gld, 256 * gld, gld);
  }
  IG4_TRY(jl.launch(st, di->sms));
  // attention of head group r over all L tokens
  IG4_TRY(launch_attention(B, Hg, static_cast<int>(L), ws.qg, ws.kg, ws.vtg, ws.vtg_ld, ws.og,
                           ws.part, st));
  // pack: to rank d, the text rows and d's image rows of o (head group r)
  JobList jo;
  const long W = static_cast<long>(Hg) * 256;
  for (int d = 0; d < sp_size; ++d) {
    long off = 0, Nd = 0;
    sp_range(N, sp_size, d, &off, &Nd);
    uint8_t *ch = static_cast<uint8_t *>(send_o) + sp_chunk_offset(cfg, sp_size, 1, r, d, true);
    jo.add(ws.og, 0, ch, 0, B, 1, T, static_cast<int>(W), L * W, 0, W, (T + Nd) * W, 0, W);
    jo.add(ws.og, (T + off) * W, ch, T * W, B, 1, static_cast<int>(Nd), static_cast<int>(W),
           L * W, 0, W, (T + Nd) * W, 0, W);
  }
  return jo.launch(st, di->sms);
}

ig4_status ig4_block_sp_post(const ig4_config *cfg, int sp_rank, int sp_size,
                             const ig4_block_weights *w, const void *x_local, void *x_out_local,
                             const void *recv_o, void *workspace, size_t ws_bytes,
                             void *stream) {
  IG4_TRY(check_sp(cfg, sp_rank, sp_size));
  IG4_TRY(check_block_weights(cfg, w));
  if (!x_local || !x_out_local || !recv_o || !workspace) return IG4_ERR_INVALID_ARG;
  if (!aligned16(x_local) || !aligned16(x_out_local) || !aligned16(recv_o))
    return IG4_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return IG4_ERR_WORKSPACE;
  const SpWs ws = sp_ws_layout(cfg, sp_size, sp_rank, static_cast<uint8_t *>(workspace));
  if (ws_bytes < ws.bytes) return IG4_ERR_WORKSPACE;
  const ig4_config t = sp_local(cfg, sp_size, sp_rank);
  const long Ls = cfg->T_text + static_cast<long>(t.grid_w);
  const size_t xbytes = (cfg->x_dtype == IG4_F32 ? 4 : 2) * static_cast<size_t>(cfg->B) * Ls * cfg->D;
  const uint8_t *xi = static_cast<const uint8_t *>(x_local);
  const uint8_t *xo = static_cast<const uint8_t *>(x_out_local);
  if (xi < xo + xbytes && xo < xi + xbytes) return IG4_ERR_INVALID_ARG;
  DeviceInfo *di = nullptr;
  IG4_TRY(device_info(&di));
  cudaStream_t st = as_stream(stream);
  const int B = cfg->B, Hg = cfg->H / sp_size;
  const long W = static_cast<long>(Hg) * 256, D = cfg->D;
  // unpack: o columns of head group s from rank s's chunk
  JobList jl;
  for (int s = 0; s < sp_size; ++s) {
    const uint8_t *ch = static_cast<const uint8_t *>(recv_o) +
                        sp_chunk_offset(cfg, sp_size, 1, s, sp_rank, false);
    jl.add(ch, 0, ws.loc.o, s * W, B, 1, static_cast<int>(Ls), static_cast<int>(W), Ls * W, 0, W,
           Ls * D, 0, D);
  }
  IG4_TRY(jl.launch(st, di->sms));
  Tracer none{nullptr, 0, 0, st};
  return block_post_attention(&t, w, x_local, x_out_local, ws.loc, st, none);
}

}  // extern "C"

// ------------------------------------------------ block without a workspace
// Scratch for ig4_block_forward_noalloc: a static device array, so the entry
// point never allocates.  In host code `g_noalloc_scratch` names a host-side
// stand-in, not device memory; its device address comes from
// cudaGetSymbolAddress, looked up on the first call for each device (with
// that device current) and again whenever the device's current context has
// changed since (a device reset loads the module anew, possibly elsewhere).
__device__ __align__(256) uint8_t g_noalloc_scratch[IG4_NOALLOC_SCRATCH_BYTES];

namespace {
struct NoallocSlot {
  void *ptr = nullptr;
  unsigned long long ctx_id = 0;
};
NoallocSlot g_noalloc[MAX_DEVICES];
std::mutex g_noalloc_mu;

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

// Unique id of the calling thread's current context (0 if there is none or
// the driver cannot tell).
unsigned long long current_ctx_id() {
  static CtxGetCurrentFn get_cur = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  if (!get_cur || !get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_cur(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of the scratch array on the current device.
ig4_status noalloc_scratch(uint8_t **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return IG4_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  NoallocSlot &slot = g_noalloc[dev];
  const unsigned long long id = current_ctx_id();
  if (slot.ptr == nullptr || id == 0 || id != slot.ctx_id) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return IG4_ERR_CUDA;
    slot.ptr = p;
    slot.ctx_id = current_ctx_id();  // the lookup made the primary context current
  }
  *out = static_cast<uint8_t *>(slot.ptr);
  return IG4_OK;
}
}  // namespace

// ------------------------------------------------------------ SM clock
// One thread counts SM cycles across a window of the global nanosecond
// timer; cycles / ns is the SM clock of that moment.  Under a power cap the
// clock drops within a millisecond of heavy tensor work, faster than a
// polled driver reading follows.  The loop is bounded by an iteration cap as
// well as by the window.
__device__ unsigned long long g_clock_probe[2];

__global__ void sm_clock_probe_kernel(unsigned long long window_ns) {
  unsigned long long t0, t1;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
  const long long c0 = clock64();
  long it = 0;
  do {
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t1));
  } while (t1 - t0 < window_ns && ++it < (1L << 26));
  const long long c1 = clock64();
  g_clock_probe[0] = static_cast<unsigned long long>(c1 - c0);
  g_clock_probe[1] = t1 - t0;
}

extern "C" {

ig4_status ig4_block_forward_noalloc(const ig4_config *cfg, const ig4_block_weights *w,
                                     const void *x_in, void *x_out, const int32_t *pos,
                                     const float *temb, void *stream) {
  IG4_TRY(check_config(cfg));
  IG4_TRY(check_block_weights(cfg, w));
  if (!x_in || !x_out || !pos || !temb) return IG4_ERR_INVALID_ARG;
  if (!aligned16(x_in) || !aligned16(x_out) || !aligned16(temb)) return IG4_ERR_INVALID_ARG;
  const long L = cfg->T_text + static_cast<long>(cfg->grid_t) * cfg->grid_h * cfg->grid_w;
  const size_t xbytes = (cfg->x_dtype == IG4_F32 ? 4 : 2) * static_cast<size_t>(cfg->B) * L * cfg->D;
  const uint8_t *xi = static_cast<const uint8_t *>(x_in);
  const uint8_t *xo = static_cast<const uint8_t *>(x_out);
  if (xi < xo + xbytes && xo < xi + xbytes) return IG4_ERR_INVALID_ARG;
  if (block_ws_layout(cfg, nullptr).bytes > IG4_NOALLOC_SCRATCH_BYTES) return IG4_ERR_WORKSPACE;
  uint8_t *scratch = nullptr;
  IG4_TRY(noalloc_scratch(&scratch));
  const BlockWs ws = block_ws_layout(cfg, scratch);
  return block_forward_impl(cfg, w, x_in, x_out, pos, temb, ws, as_stream(stream), nullptr);
}

ig4_status ig4_last_device_error(void *stream) {
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return IG4_ERR_CUDA;
  unsigned int word = 0;
  if (cudaMemcpyFromSymbol(&word, g_device_error, sizeof(word)) != cudaSuccess)
    return IG4_ERR_CUDA;
  if (word) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess)
      return IG4_ERR_CUDA;
    return IG4_ERR_TIMEOUT;
  }
  return IG4_OK;
}

ig4_status ig4_sm_clock_mhz(int window_us, void *stream, double *mhz) {
  if (window_us < 1 || window_us > 100000 || mhz == nullptr) return IG4_ERR_INVALID_ARG;
  cudaStream_t st = as_stream(stream);
  sm_clock_probe_kernel<<<1, 1, 0, st>>>(static_cast<unsigned long long>(window_us) * 1000ull);
  IG4_TRY(last_launch_status());
  unsigned long long v[2] = {0, 0};
  if (cudaMemcpyFromSymbolAsync(v, g_clock_probe, sizeof(v), 0, cudaMemcpyDeviceToHost, st) !=
          cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return IG4_ERR_CUDA;
  if (v[1] == 0) return IG4_ERR_CUDA;
  *mhz = 1e3 * static_cast<double>(v[0]) / static_cast<double>(v[1]);
  return IG4_OK;
}

ig4_status ig4_selftest_timeout(int wait_us, void *stream) {
  if (wait_us < 1 || wait_us > 5000000) return IG4_ERR_INVALID_ARG;
  selftest_timeout_kernel<<<1, 32, 0, as_stream(stream)>>>(
      static_cast<unsigned long long>(wait_us) * 1000ull);
  return last_launch_status();
}

}  // extern "C"
