// ig4_gemm.cuh - persistent tcgen05 GEMM C = A B^T for sm_100a with fused
// epilogues for the block's linears.
//
// A [M, K] and B [N, K] are K-major (row-major, K contiguous) in bf16, or both
// in FP8 E4M3 for the FP8-weight path (activation codes + per-row scale,
// weight codes + per-output-channel scale).  One CTA per SM walks the output
// tiles (128 x BN) in m-fastest order so that the CTAs in flight share the
// same few B column blocks and all of A through L2.
//
// Warp roles (192 threads):
//   warp 4      TMA producer: A and B tiles (128-byte swizzle) into a STAGES
//               deep shared-memory ring, one mbarrier per stage;
//   warp 5      TMEM allocator and MMA issuer (one thread): 4 tcgen05.mma per
//               stage into one of two TMEM accumulators (2 x BN fp32 columns),
//               tcgen05.commit frees the stage / publishes the accumulator;
//   warps 0-3   epilogue: each warp owns 32 accumulator rows (TMEM lanes
//               32*(warp%4) ..), reads 32 columns at a time with tcgen05.ld,
//               applies the fused epilogue and stores to global memory, then
//               releases the accumulator so the MMA of tile t+2 can reuse it.
#pragma once

#include "ig4_ptx.cuh"

namespace ig4 {

constexpr int GEMM_BM = 128;
constexpr int GEMM_THREADS = 192;

template <int BN>
struct GemmShape {
  static_assert(BN == 256 || BN == 192 || BN == 128, "tile width");
  static constexpr int A_BYTES = GEMM_BM * 128;
  static constexpr int B_BYTES = BN * 128;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  // as many stages as fit in ~200 KB of shared memory
  static constexpr int STAGES = (BN == 256) ? 4 : (BN == 192 ? 5 : 6);
  // two accumulators of BN fp32 columns, rounded up to a power of two
  static constexpr int TMEM_COLS = (2 * BN <= 256) ? 256 : 512;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
};

// Tile t of a persistent GEMM -> (m tile, n tile).  Tiles are taken in
// groups of group_m m tiles: within a group the m tile runs fastest, then
// the n tile.  group_m >= m_tiles is plain m-fastest order, right when A fits
// in L2 (every wave re-reads A from L2 and streams B once); a group of 8
// makes the tiles that run at the same time share ~8 A slabs and ~10 B slabs
// when A is too large to stay resident.  A bijection for any sizes.
__device__ __forceinline__ void tile_coords(int t, int m_tiles, int n_tiles_n, int group_m,
                                            int *mt, int *nt) {
  const int gsize = min(group_m, m_tiles);
  const int group = gsize * n_tiles_n;
  const int first_m = (t / group) * gsize;
  const int gm = min(m_tiles - first_m, gsize);
  const int local = t - (t / group) * group;
  *mt = first_m + local % gm;
  *nt = local / gm;
}

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(p);
  return reinterpret_cast<uint8_t *>((a + 1023) & ~static_cast<uintptr_t>(1023));
}

// ----------------------------------------------------------- store helpers

__device__ __forceinline__ void store32_bf16(__nv_bfloat16 *dst, const float (&v)[32]) {
  uint4 *d = reinterpret_cast<uint4 *>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 w;
    w.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
    w.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
    w.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
    w.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
    d[q] = w;
  }
}

__device__ __forceinline__ void store32_f32(float *dst, const float (&v)[32]) {
  float4 *d = reinterpret_cast<float4 *>(dst);
#pragma unroll
  for (int q = 0; q < 8; ++q) d[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

__device__ __forceinline__ void load32_bf16(const __nv_bfloat16 *src, float (&v)[32]) {
  const uint4 *s = reinterpret_cast<const uint4 *>(src);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 w = s[q];
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[8 * q + 2 * e] = __uint_as_float(u[e] << 16);
      v[8 * q + 2 * e + 1] = __uint_as_float(u[e] & 0xFFFF0000u);
    }
  }
}

__device__ __forceinline__ void load32_f32(const float *src, float (&v)[32]) {
  const float4 *s = reinterpret_cast<const float4 *>(src);
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float4 w = s[q];
    v[4 * q] = w.x;
    v[4 * q + 1] = w.y;
    v[4 * q + 2] = w.z;
    v[4 * q + 3] = w.w;
  }
}

__device__ __forceinline__ void load32_f32_ldg(const float *src, float (&v)[32]) {
  const float4 *s = reinterpret_cast<const float4 *>(src);
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float4 w = __ldg(s + q);
    v[4 * q] = w.x;
    v[4 * q + 1] = w.y;
    v[4 * q + 2] = w.z;
    v[4 * q + 3] = w.w;
  }
}

template <typename T>
__device__ __forceinline__ void load32_x(const T *src, float (&v)[32]);
template <>
__device__ __forceinline__ void load32_x<float>(const float *src, float (&v)[32]) {
  load32_f32(src, v);
}
template <>
__device__ __forceinline__ void load32_x<__nv_bfloat16>(const __nv_bfloat16 *src, float (&v)[32]) {
  load32_bf16(src, v);
}
template <typename T>
__device__ __forceinline__ void store32_x(T *dst, const float (&v)[32]);
template <>
__device__ __forceinline__ void store32_x<float>(float *dst, const float (&v)[32]) {
  store32_f32(dst, v);
}
template <>
__device__ __forceinline__ void store32_x<__nv_bfloat16>(__nv_bfloat16 *dst, const float (&v)[32]) {
  store32_bf16(dst, v);
}

// Dequantisation factors of the FP8 path: acc * a_scale[row] * b_scale[col].
template <bool FP8>
__device__ __forceinline__ void apply_scales(float (&v)[32], float rs, const float *bs) {
  if constexpr (FP8) {
    float s[32];
    load32_f32_ldg(bs, s);
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] *= rs * s[i];
  }
}

// W-wide (16 or 32) versions of the loads and stores above, for the chunks
// of the gated-residual epilogue (a 240-wide tile ends in a 16-column chunk).
template <int W>
__device__ __forceinline__ void load_f32_w(const float *src, float (&v)[32]) {
  const float4 *s = reinterpret_cast<const float4 *>(src);
#pragma unroll
  for (int q = 0; q < W / 4; ++q) {
    const float4 w = __ldg(s + q);
    v[4 * q] = w.x;
    v[4 * q + 1] = w.y;
    v[4 * q + 2] = w.z;
    v[4 * q + 3] = w.w;
  }
}
template <int W, typename T>
__device__ __forceinline__ void load_x_w(const T *src, float (&v)[32]) {
  if constexpr (sizeof(T) == 4) {
    const float4 *s = reinterpret_cast<const float4 *>(src);
#pragma unroll
    for (int q = 0; q < W / 4; ++q) {
      const float4 w = s[q];
      v[4 * q] = w.x;
      v[4 * q + 1] = w.y;
      v[4 * q + 2] = w.z;
      v[4 * q + 3] = w.w;
    }
  } else {
    const uint4 *s = reinterpret_cast<const uint4 *>(src);
#pragma unroll
    for (int q = 0; q < W / 8; ++q) {
      const uint4 w = s[q];
      const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[8 * q + 2 * e] = __uint_as_float(u[e] << 16);
        v[8 * q + 2 * e + 1] = __uint_as_float(u[e] & 0xFFFF0000u);
      }
    }
  }
}
template <int W, typename T>
__device__ __forceinline__ void store_x_w(T *dst, const float (&v)[32]) {
  if constexpr (sizeof(T) == 4) {
    float4 *d = reinterpret_cast<float4 *>(dst);
#pragma unroll
    for (int q = 0; q < W / 4; ++q) d[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
  } else {
    uint4 *d = reinterpret_cast<uint4 *>(dst);
#pragma unroll
    for (int q = 0; q < W / 8; ++q)
      d[q] = make_uint4(pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                        pack_bf16x2(v[8 * q + 4], v[8 * q + 5]),
                        pack_bf16x2(v[8 * q + 6], v[8 * q + 7]));
  }
}

// ------------------------------------------------------------- epilogues
// Each epilogue is called by the 128 epilogue threads for one output tile;
// `tacc` is the TMEM address of this warp's 32 lanes at column 0 of the
// tile's accumulator and `r` the thread's row inside the tile.

// out[row', col] = acc (* scales) (+ bias[col]); row' = row, or, with
// remap_n > 0, (row / remap_n) * remap_L + remap_off + row % remap_n (writes
// the latent in-projection straight into the image part of the sequence).
template <int BN, bool FP8, typename OT>
struct EpiStore {
  OT *out;
  int ldo;
  int M, N;
  const float *bias;
  const float *a_scale, *b_scale;
  int remap_n, remap_L, remap_off;
  static constexpr int COLS = BN;

  __device__ __forceinline__ void operator()(int m0, int n0, uint32_t tacc, int r) const {
    part(m0, n0, tacc, r, 0, BN);
  }

  // columns [lo, hi) of the tile (multiples of 32)
  __device__ __forceinline__ void part(int m0, int n0, uint32_t tacc, int r, int lo, int hi) const {
    const int row = m0 + r;
    const bool valid = row < M;
    long orow = row;
    if (remap_n > 0) orow = static_cast<long>(row / remap_n) * remap_L + remap_off + row % remap_n;
    const float rs = (FP8 && valid) ? __ldg(a_scale + row) : 1.0f;
#pragma unroll 1
    for (int c = lo; c < hi; c += 32) {
      float v[32];
      tmem_ld32(tacc + c, v);
      tmem_ld_wait();
      if (n0 + c >= N) continue;
      apply_scales<FP8>(v, rs, b_scale + n0 + c);
      if (bias != nullptr) {
        float bb[32];
        load32_f32_ldg(bias + n0 + c, bb);
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] += bb[i];
      }
      if (valid) store32_x<OT>(out + orow * ldo + n0 + c, v);
    }
  }
};

// Gated residual: x_out[row, col] = x_res[row, col] + gate[b, col] * acc,
// b = row / L (the AdaLN gate of the row's sample).  x_res may be null (no
// residual: a tensor-parallel shard's partial sum); x_out may have another
// type than x_res (fp32 partial sums).
template <int BN, bool FP8, typename XT, typename OT = XT>
struct EpiResidGate {
  const XT *x_res;
  OT *x_out;
  const float *gate;
  int gate_stride;
  int L, M, N;
  const float *a_scale, *b_scale;
  static constexpr int COLS = BN;

  __device__ __forceinline__ void operator()(int m0, int n0, uint32_t tacc, int r) const {
    part(m0, n0, tacc, r, 0, BN);
  }

  // columns [lo, hi) of the tile (multiples of 16); columns at or past N (the
  // last tile of a 240-wide tiling) are skipped
  __device__ __forceinline__ void part(int m0, int n0, uint32_t tacc, int r, int lo, int hi) const {
    const int row = m0 + r;
    const bool valid = row < M;
    const int b = valid ? row / L : 0;
    // a_scale == nullptr: A's scales were applied by the tensor cores (MX8)
    const float rs = (FP8 && valid && a_scale != nullptr) ? __ldg(a_scale + row) : 1.0f;
    const float *grow = gate + static_cast<long>(b) * gate_stride + n0;
    const int cmax = min(hi, N - n0);
#pragma unroll 1
    for (int c = lo; c < cmax; c += 32) {
      if (cmax - c >= 32)
        chunk<32>(n0, tacc, row, valid, rs, grow, c);
      else
        chunk<16>(n0, tacc, row, valid, rs, grow, c);
    }
  }

  template <int W>
  __device__ __forceinline__ void chunk(int n0, uint32_t tacc, int row, bool valid, float rs,
                                        const float *grow, int c) const {
    float v[32];
    tmem_ld32(tacc + c, v);  // (a 16-wide chunk reads 16 spare columns)
    tmem_ld_wait();
    if (!valid) return;
    if constexpr (FP8) {
      float sc[32];
      load_f32_w<W>(b_scale + n0 + c, sc);
#pragma unroll
      for (int i = 0; i < W; ++i) v[i] *= rs * sc[i];
    }
    float g[32], x[32];
    load_f32_w<W>(grow + c, g);
    const long off = static_cast<long>(row) * N + n0 + c;
    if (x_res != nullptr) {
      load_x_w<W>(x_res + off, x);
    } else {
#pragma unroll
      for (int i = 0; i < W; ++i) x[i] = 0.0f;
    }
#pragma unroll
    for (int i = 0; i < W; ++i) x[i] = fmaf(g[i], v[i], x[i]);
    store_x_w<W>(x_out + off, x);
  }
};

// SwiGLU: the 256-column tile holds gate rows [n, n+128) in columns [0,128)
// and up rows [n, n+128) in columns [128,256); u[row, n + c] =
// silu(gate) * up.  (Two TMA loads fill the two halves of the B tile.)
template <bool FP8>
struct EpiSwiGLU {
  __nv_bfloat16 *u;
  int I, M;
  const float *a_scale, *s_gate, *s_up;
  static constexpr int COLS = 128;  // output columns per tile

  __device__ __forceinline__ void operator()(int m0, int n0, uint32_t tacc, int r) const {
    part(m0, n0, tacc, r, 0, 128);
  }

  // output columns [lo, hi) of the tile: accumulator columns [lo, hi) (gate)
  // and [128 + lo, 128 + hi) (up)
  __device__ __forceinline__ void part(int m0, int n0, uint32_t tacc, int r, int lo, int hi) const {
    const int row = m0 + r;
    const bool valid = row < M;
    const float rs = (FP8 && valid) ? __ldg(a_scale + row) : 1.0f;
    const int n = n0 / 2;  // tile index * 128
#pragma unroll 1
    for (int c = lo; c < hi; c += 32) {
      float g[32], up[32];
      tmem_ld32(tacc + c, g);
      tmem_ld32(tacc + 128 + c, up);
      tmem_ld_wait();
      if (!valid) continue;
      apply_scales<FP8>(g, rs, s_gate + n + c);
      apply_scales<FP8>(up, rs, s_up + n + c);
#pragma unroll
      for (int i = 0; i < 32; ++i) g[i] = silu_f(g[i]) * up[i];
      store32_bf16(u + static_cast<long>(row) * I + n + c, g);
    }
  }
};

// QKV projection with per-head QK-RMSNorm and MRoPE.  Tile columns
// [n0, n0+256) are one head of q (n-tile < H), k (< 2H) or v.  q, k are
// normalised over the 256 values, scaled by g, and the pairs (j, j+64),
// j < 64, are rotated by the row's table angle; they are stored as
// [B, H, L, 256].  v is stored transposed, [B, H, 256, vt_ld].
template <bool FP8>
struct EpiQKV {
  __nv_bfloat16 *q, *k, *vt;
  int vt_ld;
  int L, H, M;
  const float *g_q, *g_k;
  float eps;
  const float *rope_cos, *rope_sin;
  const float *a_scale, *b_scale;

  __device__ __forceinline__ void operator()(int m0, int n0, uint32_t tacc, int r) const {
    const int row = m0 + r;
    const bool valid = row < M;
    const int b = valid ? row / L : 0;
    const int l = valid ? row - b * L : 0;
    const int nt = n0 >> 8;
    const int sec = nt / H;
    const int h = nt - sec * H;
    const float rs = (FP8 && valid) ? __ldg(a_scale + row) : 1.0f;
    const float *bs = b_scale + n0;

    if (sec == 2) {
      __nv_bfloat16 *dst = vt + static_cast<long>(b * H + h) * 256 * vt_ld + l;
#pragma unroll 1
      for (int c = 0; c < 256; c += 32) {
        float v[32];
        tmem_ld32(tacc + c, v);
        tmem_ld_wait();
        if (!valid) continue;
        apply_scales<FP8>(v, rs, bs + c);
#pragma unroll
        for (int i = 0; i < 32; ++i) dst[static_cast<long>(c + i) * vt_ld] = __float2bfloat16_rn(v[i]);
      }
      return;
    }

    float ss = 0.0f;
#pragma unroll 1
    for (int c = 0; c < 256; c += 32) {
      float v[32];
      tmem_ld32(tacc + c, v);
      tmem_ld_wait();
      apply_scales<FP8>(v, rs, bs + c);
#pragma unroll
      for (int i = 0; i < 32; ++i) ss = fmaf(v[i], v[i], ss);
    }
    const float rstd = rsqrtf(ss * (1.0f / 256.0f) + eps);
    const float *g = (sec == 0) ? g_q : g_k;
    __nv_bfloat16 *dst = ((sec == 0) ? q : k) + (static_cast<long>(b * H + h) * L + l) * 256;
    const float *cs = rope_cos + static_cast<long>(l) * 64;
    const float *sn = rope_sin + static_cast<long>(l) * 64;

#pragma unroll 1
    for (int j0 = 0; j0 < 64; j0 += 32) {
      float a[32], bv[32];
      tmem_ld32(tacc + j0, a);
      tmem_ld32(tacc + j0 + 64, bv);
      tmem_ld_wait();
      if (!valid) continue;
      apply_scales<FP8>(a, rs, bs + j0);
      apply_scales<FP8>(bv, rs, bs + j0 + 64);
      float ga[32], gb[32], c32[32], s32[32];
      load32_f32_ldg(g + j0, ga);
      load32_f32_ldg(g + j0 + 64, gb);
      load32_f32_ldg(cs + j0, c32);
      load32_f32_ldg(sn + j0, s32);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float x1 = a[i] * rstd * ga[i];
        const float x2 = bv[i] * rstd * gb[i];
        a[i] = x1 * c32[i] - x2 * s32[i];
        bv[i] = x2 * c32[i] + x1 * s32[i];
      }
      store32_bf16(dst + j0, a);
      store32_bf16(dst + j0 + 64, bv);
    }
#pragma unroll 1
    for (int c = 128; c < 256; c += 32) {
      float v[32];
      tmem_ld32(tacc + c, v);
      tmem_ld_wait();
      if (!valid) continue;
      apply_scales<FP8>(v, rs, bs + c);
      float gg[32];
      load32_f32_ldg(g + c, gg);
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] *= rstd * gg[i];
      store32_bf16(dst + c, v);
    }
  }
};

// ---------------------------------------------------------------- kernel
// BN: accumulator columns per tile (256 or 128).  DUAL_B: the B tile is two
// 128-row halves from two tensors (tmB rows, then tmB2 rows, same row index).
// n_cols_tile: output columns one n-tile advances (BN, or 128 with DUAL_B).
template <int BN, bool FP8, bool DUAL_B, class Epi>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmB2, int M, int n_tiles_n, int K,
                   int group_m, const Epi epi) {
  using S = GemmShape<BN>;
  constexpr int STAGES = S::STAGES;
  constexpr int BK = FP8 ? 128 : 64;  // K elements per stage: one 128-byte row
  constexpr int UK_BYTES = 32;        // K bytes per MMA instruction (16 bf16 / 32 e4m3)
  constexpr uint32_t IDESC = FP8 ? idesc_e4m3(GEMM_BM, BN) : idesc_bf16(GEMM_BM, BN);
  constexpr int B_ROWS_HALF = BN / 2;

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = align1024(smem_raw);
  uint8_t *sA = smem;
  uint8_t *sB = smem + STAGES * S::A_BYTES;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + STAGES * S::STAGE_BYTES);
  uint64_t *empty = full + STAGES;
  uint64_t *tfull = empty + STAGES;
  uint64_t *tempty = tfull + 2;
  uint64_t *drain = tempty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m_tiles = (M + GEMM_BM - 1) / GEMM_BM;
  const int n_tiles = m_tiles * n_tiles_n;
  const int kblocks = (K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (DUAL_B) tma_prefetch_desc(&tmB2);
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, S::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();
  pdl_trigger();

  if (warp == 4) {
    if (lane == 0) {
      // ---------------- TMA producer
      int s = 0;
      uint32_t ph = 0;
      long issued = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
        int mt, nt;
        tile_coords(t, m_tiles, n_tiles_n, group_m, &mt, &nt);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], S::STAGE_BYTES);
          tma_load_2d(sA + s * S::A_BYTES, &tmA, &full[s], kb * BK, mt * GEMM_BM);
          if (DUAL_B) {
            tma_load_2d(sB + s * S::B_BYTES, &tmB, &full[s], kb * BK, nt * B_ROWS_HALF);
            tma_load_2d(sB + s * S::B_BYTES + B_ROWS_HALF * 128, &tmB2, &full[s], kb * BK,
                        nt * B_ROWS_HALF);
          } else {
            tma_load_2d(sB + s * S::B_BYTES, &tmB, &full[s], kb * BK, nt * BN);
          }
          ++issued;
          if (++s == STAGES) {
            s = 0;
            ph ^= 1;
          }
        }
      }
      if (!ok) {
        // Let the loads already issued land before the CTA's shared memory goes away.
        for (long i = (issued > STAGES ? issued - STAGES : 0); i < issued; ++i)
          mbar_wait(&full[i % STAGES], static_cast<uint32_t>((i / STAGES) & 1), nullptr,
                    WAIT_LIMIT_NS / 4);
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      // ---------------- MMA issuer
      int s = 0;
      uint32_t ph = 0;
      int local = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++local) {
        const int buf = local & 1;
        const uint32_t use = static_cast<uint32_t>(local >> 1);
        if (!mbar_wait(&tempty[buf], (use & 1) ^ 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * BN;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&full[s], ph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + s * S::A_BYTES);
          const uint32_t b_base = smem_u32(sB + s * S::B_BYTES);
#pragma unroll
          for (int kk = 0; kk < 128 / UK_BYTES; ++kk) {
            const uint64_t ad = sdesc_kmajor_sw128(a_base + kk * UK_BYTES);
            const uint64_t bd = sdesc_kmajor_sw128(b_base + kk * UK_BYTES);
            if (FP8)
              umma_f8(d_tmem, ad, bd, IDESC, (kb | kk) != 0);
            else
              umma_bf16(d_tmem, ad, bd, IDESC, (kb | kk) != 0);
          }
          umma_commit(&empty[s]);
          if (++s == STAGES) {
            s = 0;
            ph ^= 1;
          }
        }
        if (ok) umma_commit(&tfull[buf]);
      }
      // Every MMA issued above has finished once `drain` completes.
      umma_commit(drain);
      mbar_wait(drain, 0, nullptr, WAIT_LIMIT_NS / 4);
    }
  } else {
    // ---------------- epilogue warps 0..3
    const int r = warp * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    int local = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++local) {
      const int buf = local & 1;
      const uint32_t use = static_cast<uint32_t>(local >> 1);
      if (!mbar_wait_warp(&tfull[buf], use & 1, abort_flag)) break;
      tc_fence_after();
      int mt, nt;
      tile_coords(t, m_tiles, n_tiles_n, group_m, &mt, &nt);
      epi(mt * GEMM_BM, nt * BN, tmem_base + lane_base + buf * BN, r);
      tc_fence_before();
      mbar_arrive(&tempty[buf]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) tmem_dealloc(tmem_base, S::TMEM_COLS);
}

// ------------------------------------------------------ CTA-pair kernel
// The same GEMM on a 2-CTA cluster: a pair tile is 256 rows x BN columns
// (BN = 256, or 192 where 256-wide tiles leave the last wave of pairs mostly
// idle); each CTA loads its own 128 A rows and HALF of the BN B rows (so with
// DUAL_B the first CTA loads the gate rows and the second the up rows), the
// leader issues tcgen05.mma.cta_group::2 with M = 256, and each CTA's
// epilogue warps handle its own 128 accumulator rows exactly as above.  Per
// 128-clock MMA each SM reads 8 KB of operands instead of 12 KB, and each SM
// loads a third fewer bytes per flop.
//
// K-snake: a pair's odd-numbered tiles sweep K from the last k-block down.
// All pairs move from tile to tile at about the same time, so each round of
// tiles starts on the k-blocks the previous round read last, which are still
// in L2 where the two rounds share A rows or B rows.
//
// Barriers: full[s] in the leader (its producer posts the bytes of both
// CTAs; both CTAs' loads complete on it); empty[s] and tfull[b] in both CTAs
// (arrived by the leader's multicast commits); tempty[b] in the leader (one
// arrival per epilogue warp of the pair).
template <int BN, bool MX8A = false>
struct PairShape {
  static_assert(BN == 256 || BN == 240 || BN == 192, "pair tile width");
  static constexpr int A_BYTES = GEMM_BM * 128;          // 16 KB
  static constexpr int BH_BYTES = (BN / 2) * 128;        // 16, 15 or 12 KB (a multiple of 1 KB)
  static constexpr int SF_BYTES = MX8A ? 512 : 0;        // A's scale chunk (MX8)
  static constexpr int STAGE_BYTES = A_BYTES + BH_BYTES + SF_BYTES;
  static constexpr int STAGES = BN == 256 ? 6 : 7;       // 190-227 KB of shared memory
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
};

// MX8A: A in MX8 (E4M3 with a UE8M0 scale per 32 elements, see ig4_mx8.cuh)
// and B in E4M3 with unit block scales: tcgen05.mma kind::mxf8f6f4 with
// block_scale; tmB2 then maps A's 512-byte scale chunks, which the leader
// copies into TMEM once per k-block (one tcgen05.cp); B's scales (byte 127)
// are written into TMEM once.  192-wide tiles only: the two accumulators
// (384 columns) leave room for the scales.
template <int BN, bool FP8, bool DUAL_B, class Epi, bool MX8A = false>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmB2, int M, int n_tiles_n, int K,
                     int group_m, const Epi epi) {
  static_assert(!DUAL_B || BN == 256, "SwiGLU pairs split 128 gate / 128 up rows");
  static_assert(!MX8A || (FP8 && !DUAL_B && (BN == 192 || BN == 240)),
                "MX8 A: FP8, single B, 192- or 240-wide tiles");
  using P = PairShape<BN, MX8A>;
  // TMEM: accumulator b at column b * ACC_STRIDE (a 240-wide tile's second
  // accumulator starts at 256); MX8A scale columns after both
  constexpr uint32_t ACC_STRIDE = BN == 240 ? 256 : BN;
  constexpr uint32_t SFA_COL = BN == 240 ? 496 : 448;
  constexpr uint32_t SFB_COL = BN == 240 ? 500 : 464;
  constexpr uint32_t SF_INIT_COL = BN == 240 ? 480 : 464;  // 32 columns of byte 127
  constexpr int PAIR_STAGES = P::STAGES;
  constexpr int PAIR_STAGE_BYTES = P::STAGE_BYTES;
  constexpr int A_BYTES = P::A_BYTES;
  constexpr int BH_BYTES = P::BH_BYTES;
  constexpr int BK = FP8 ? 128 : 64;
  constexpr int UK_BYTES = 32;
  constexpr uint32_t IDESC = FP8 ? idesc_e4m3(2 * GEMM_BM, BN) : idesc_bf16(2 * GEMM_BM, BN);
  constexpr uint32_t TMEM_COLS = 512;

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = align1024(smem_raw);
  uint8_t *sA = smem;
  uint8_t *sB = smem + PAIR_STAGES * A_BYTES;
  uint8_t *sSF = sB + PAIR_STAGES * BH_BYTES;  // MX8A only
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + PAIR_STAGES * PAIR_STAGE_BYTES);
  uint64_t *empty = full + PAIR_STAGES;
  uint64_t *tfull = empty + PAIR_STAGES;
  uint64_t *tempty = tfull + 2;
  uint64_t *drain = tempty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  const int n_pairs = gridDim.x >> 1;
  const int m_tiles = (M + 2 * GEMM_BM - 1) / (2 * GEMM_BM);
  const int n_tiles = m_tiles * n_tiles_n;
  const int kblocks = (K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < PAIR_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 2 * 4);  // one arrival per epilogue warp of the pair
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (DUAL_B) tma_prefetch_desc(&tmB2);
  }
  if (warp == 5) {
    tmem_alloc_pair(tmem_slot, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  if constexpr (MX8A) {
    // B's unit scales (byte 127) in every lane of the B scale columns
    if (warp < 4) {
      uint32_t ones[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) ones[i] = 0x7F7F7F7Fu;
      tmem_st32_u(tmem_base + (static_cast<uint32_t>(warp * 32) << 16) + SF_INIT_COL, ones);
      tmem_st_wait();
    }
    tc_fence_before();
    cluster_sync_all();
    tc_fence_after();
  }
  pdl_wait();
  pdl_trigger();

  if (warp == 4) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs)
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      int local = 0;
      for (int t = pair; t < n_tiles && ok; t += n_pairs, ++local) {
        int mt, nt;
        tile_coords(t, m_tiles, n_tiles_n, group_m, &mt, &nt);
        for (int it = 0; it < kblocks; ++it) {
          const int kb = (local & 1) ? kblocks - 1 - it : it;  // K-snake
          if (!mbar_wait_cluster(&empty[s], ph ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * PAIR_STAGE_BYTES);
          const uint32_t bar = map_shared_to_rank(&full[s], 0);
          tma_load_2d_pair(sA + s * A_BYTES, &tmA, bar, kb * BK,
                           mt * 2 * GEMM_BM + static_cast<int>(rank) * GEMM_BM);
          if (DUAL_B)
            tma_load_2d_pair(sB + s * BH_BYTES, rank == 0 ? &tmB : &tmB2, bar, kb * BK,
                             nt * (BN / 2));
          else
            tma_load_2d_pair(sB + s * BH_BYTES, &tmB, bar, kb * BK,
                             nt * BN + static_cast<int>(rank) * (BN / 2));
          if constexpr (MX8A)
            tma_load_3d_pair(sSF + s * 512, &tmB2, bar, 0, kb,
                             mt * 2 + static_cast<int>(rank));
          if (++s == PAIR_STAGES) {
            s = 0;
            ph ^= 1;
          }
        }
      }
      if (!ok) sleep_ns(50000);  // let the loads already issued land
    }
  } else if (warp == 5) {
    if (lane == 0 && rank == 0) {
      // ---------------- MMA issuer (leader CTA)
      int s = 0;
      uint32_t ph = 0;
      int local = 0;
      bool ok = true;
      for (int t = pair; t < n_tiles && ok; t += n_pairs, ++local) {
        const int buf = local & 1;
        const uint32_t use = static_cast<uint32_t>(local >> 1);
        if (!mbar_wait_cluster(&tempty[buf], (use & 1) ^ 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * ACC_STRIDE;
        for (int it = 0; it < kblocks; ++it) {  // k-blocks in the producer's order
          if (!mbar_wait_cluster(&full[s], ph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + s * A_BYTES);
          const uint32_t b_base = smem_u32(sB + s * BH_BYTES);
          if constexpr (MX8A)
            tmem_cp_sf_pair(tmem_base + SFA_COL, sdesc_kmajor_none(smem_u32(sSF + s * 512), 128));
#pragma unroll
          for (int kk = 0; kk < 128 / UK_BYTES; ++kk) {
            const uint64_t ad = sdesc_kmajor_sw128(a_base + kk * UK_BYTES);
            const uint64_t bd = sdesc_kmajor_sw128(b_base + kk * UK_BYTES);
            if constexpr (MX8A)
              umma_mx8_pair(d_tmem, ad, bd, idesc_mx8(2 * GEMM_BM, BN, kk), tmem_base + SFA_COL,
                            tmem_base + SFB_COL, (it | kk) != 0);
            else if (FP8)
              umma_f8_pair(d_tmem, ad, bd, IDESC, (it | kk) != 0);
            else
              umma_bf16_pair(d_tmem, ad, bd, IDESC, (it | kk) != 0);
          }
          umma_commit_pair_both(&empty[s]);
          if (++s == PAIR_STAGES) {
            s = 0;
            ph ^= 1;
          }
        }
        if (ok) umma_commit_pair_both(&tfull[buf]);
      }
      umma_commit_pair_both(drain);
      mbar_wait_cluster(drain, 0, nullptr, WAIT_LIMIT_NS / 4);
    }
  } else {
    // ---------------- epilogue warps 0..3 (both CTAs, own 128 rows)
    const int r = warp * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t tempty_leader0 = map_shared_to_rank(&tempty[0], 0);
    const uint32_t tempty_leader1 = map_shared_to_rank(&tempty[1], 0);
    int local = 0;
    for (int t = pair; t < n_tiles; t += n_pairs, ++local) {
      const int buf = local & 1;
      const uint32_t use = static_cast<uint32_t>(local >> 1);
      const bool ok = mbar_wait_cluster(&tfull[buf], use & 1, abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      int mt, nt;
      tile_coords(t, m_tiles, n_tiles_n, group_m, &mt, &nt);
      epi(mt * 2 * GEMM_BM + static_cast<int>(rank) * GEMM_BM, nt * BN,
          tmem_base + lane_base + buf * ACC_STRIDE, r);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(buf ? tempty_leader1 : tempty_leader0);
    }
  }

  __syncwarp();
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  if (warp == 5) tmem_dealloc_pair(tmem_base, TMEM_COLS);
}

}  // namespace ig4
