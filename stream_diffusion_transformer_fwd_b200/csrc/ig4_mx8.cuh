// ig4_mx8.cuh - FP8 activations with 1x32 block scales (MX format) for the
// FP8 path's two activation-side GEMM inputs (the attention output feeding
// the out-projection, u feeding the down-projection), and the block-scaled
// FP8 GEMM on CTA pairs (tcgen05 kind::mxf8f6f4) that consumes them.
//
// Source: "Ideogram 4 快速开始", section on hardware and precision: the
// release weights are FP8 E4M3 with per-output-channel scales.  How the
// activations reach the FP8 tensor cores is not fixed there; here every 32
// consecutive elements of a row share a power-of-two scale (UE8M0), which
// the producing kernel (attention epilogue, SwiGLU epilogue) can compute on
// its own - no pass over the whole row is needed - and which the tensor
// cores apply themselves (block_scale), so the GEMM epilogue only applies
// the weights' per-channel scale.
//
// Encoding of a block of 32 values v (every step one float32 operation):
//   amax  = max |v|;
//   e     = ceil(log2(amax / 448)) (the smallest power of two that brings
//           the block into E4M3's range), at least -126; e = 0 for an
//           all-zero block;
//   code  = RNE_E4M3(v * 2^-e) (saturating at +-448);
//   scale byte = e + 127,
// so v ~= 2^(byte - 127) * e4m3(code).
//
// Scale layout: the tensor cores read the scales of a 128-row block and a
// 128-element k-block (4 scales per row) from one 512-byte chunk, row r's
// 4 bytes at 16 (r % 32) + 4 ((r % 128) / 32); chunk (row block rb, k-block
// kb) sits at byte 512 (rb * K/128 + kb).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ig4_gemm.cuh"
#include "ig4_ptx.cuh"

namespace ig4 {

constexpr int MX8_BLOCK = 32;

// Byte offset of the scale of (row r, 32-element block b) for a K-wide operand.
__device__ __forceinline__ long mx8_sf_offset(int r, int b, int K) {
  const long chunk = static_cast<long>(r >> 7) * (K >> 7) + (b >> 2);
  return chunk * 512 + 16 * (r & 31) + 4 * ((r & 127) >> 5) + (b & 3);
}

// Scale exponent of a block with this amax (see the encoding above).
__device__ __forceinline__ int mx8_exponent(float amax) {
  if (!(amax > 0.0f)) return 0;
  const uint32_t bits = __float_as_uint(amax / 448.0f);
  const int ef = static_cast<int>((bits >> 23) & 0xFF);
  if (ef == 0) return -126;  // subnormal quotient: 2^-126 covers it
  return ef - 127 + ((bits & 0x7FFFFF) != 0 ? 1 : 0);
}

// 2^-e as a float, e in [-126, 126] (finite inputs give e <= 120).
__device__ __forceinline__ float mx8_inv_scale(int e) {
  return __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
}

// The bf16 value of a float (round to nearest even): the producers encode
// the bf16 activation, as a separate quantiser of the stored bf16 tensor
// would, so every path that reaches MX8 takes the same decisions.
__device__ __forceinline__ float bf16_round(float x) {
  return __bfloat162float(__float2bfloat16_rn(x));
}

// Encodes the bf16 roundings of 32 values: codes into out[0..1] (16 bytes
// each), returns the scale byte.  v is overwritten with the rounded values.
__device__ __forceinline__ uint8_t mx8_encode32(float (&v)[32], uint4 (&out)[2]) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    v[i] = bf16_round(v[i]);
    amax = fmaxf(amax, fabsf(v[i]));
  }
  const int e = mx8_exponent(amax);
  const float inv = mx8_inv_scale(e);
  uint32_t w[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    w[i] = static_cast<uint32_t>(pack_e4m3x2(v[4 * i] * inv, v[4 * i + 1] * inv)) |
           (static_cast<uint32_t>(pack_e4m3x2(v[4 * i + 2] * inv, v[4 * i + 3] * inv)) << 16);
  out[0] = make_uint4(w[0], w[1], w[2], w[3]);
  out[1] = make_uint4(w[4], w[5], w[6], w[7]);
  return static_cast<uint8_t>(e + 127);
}

// bf16 [M][K] (K % 128 == 0) -> codes [M][K] and packed scales (rows padded
// to a multiple of 128; the padding's scales are left as they are).  One
// warp per row; lane i takes elements 8i .. 8i + 7 of every 256, four lanes
// share a block's amax by shuffle.
constexpr int MX8Q_THREADS = 256;

__global__ void __launch_bounds__(MX8Q_THREADS)
    quantize_mx8_kernel(const __nv_bfloat16 *__restrict__ x, int M, int K,
                        uint8_t *__restrict__ codes, uint8_t *__restrict__ sf) {
  pdl_wait();
  pdl_trigger();
  const int row = blockIdx.x * (MX8Q_THREADS / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  const uint4 *xr = reinterpret_cast<const uint4 *>(x + static_cast<long>(row) * K);
  uint2 *cr = reinterpret_cast<uint2 *>(codes + static_cast<long>(row) * K);
  for (int base = 0; base < K; base += 256) {
    const int k = base + 8 * lane;
    const bool in = k < K;  // whole 32-element blocks (K % 128 == 0)
    const uint4 q = in ? __ldg(xr + k / 8) : make_uint4(0, 0, 0, 0);
    const uint32_t u[4] = {q.x, q.y, q.z, q.w};
    float f[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(u[i] << 16);
      f[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    const int e = mx8_exponent(amax);
    const float inv = mx8_inv_scale(e);
    uint2 w;
    w.x = static_cast<uint32_t>(pack_e4m3x2(f[0] * inv, f[1] * inv)) |
          (static_cast<uint32_t>(pack_e4m3x2(f[2] * inv, f[3] * inv)) << 16);
    w.y = static_cast<uint32_t>(pack_e4m3x2(f[4] * inv, f[5] * inv)) |
          (static_cast<uint32_t>(pack_e4m3x2(f[6] * inv, f[7] * inv)) << 16);
    if (in) {
      cr[k / 8] = w;
      if ((lane & 3) == 0) sf[mx8_sf_offset(row, k / MX8_BLOCK, K)] = static_cast<uint8_t>(e + 127);
    }
  }
}

// SwiGLU epilogue writing u as MX8 (the FP8 block's down-projection input):
// as EpiSwiGLU<true>, each 32-column chunk of a row encoded on the spot.
struct EpiSwiGLUMx8 {
  uint8_t *uq, *usf;
  int I, M;
  const float *a_scale, *s_gate, *s_up;
  static constexpr int COLS = 128;  // output columns per tile

  __device__ __forceinline__ void operator()(int m0, int n0, uint32_t tacc, int r) const {
    part(m0, n0, tacc, r, 0, 128);
  }

  __device__ __forceinline__ void part(int m0, int n0, uint32_t tacc, int r, int lo, int hi) const {
    const int row = m0 + r;
    const bool valid = row < M;
    const float rs = valid ? __ldg(a_scale + row) : 1.0f;
    const int n = n0 / 2;  // tile index * 128
#pragma unroll 1
    for (int c = lo; c < hi; c += 32) {
      float g[32], up[32];
      tmem_ld32(tacc + c, g);
      tmem_ld32(tacc + 128 + c, up);
      tmem_ld_wait();
      if (!valid) continue;
      apply_scales<true>(g, rs, s_gate + n + c);
      apply_scales<true>(up, rs, s_up + n + c);
#pragma unroll
      for (int i = 0; i < 32; ++i) g[i] = silu_f(g[i]) * up[i];
      uint4 q[2];
      const uint8_t sb = mx8_encode32(g, q);
      uint4 *dst = reinterpret_cast<uint4 *>(uq + static_cast<long>(row) * I + n + c);
      dst[0] = q[0];
      dst[1] = q[1];
      usf[mx8_sf_offset(row, (n + c) / MX8_BLOCK, I)] = sb;
    }
  }
};

// ------------------------------------------------- block-scaled FP8 GEMM
// The CTA-pair GEMM (see gemm_pair_kernel) with A in MX8 (E4M3 codes and a
// UE8M0 scale per 32 elements) and B in E4M3 with unit block scales (the
// weights' per-channel fp32 scale stays in the epilogue): tcgen05.mma
// kind::mxf8f6f4 with block_scale.  Per 128-element k-block a stage holds
// A (128 rows x 128 B), half of B (128 rows x 128 B) and A's 512-byte
// scale chunk; the leader copies that chunk into TMEM (one tcgen05.cp) and
// issues 4 MMAs of K = 32, the j-th reading scale byte j of each row (scale
// factor id j).  B's scales are the constant 1.0 (byte 127), written into
// TMEM once.  The two 256-column accumulators overlap by 64 columns to leave
// room for the scales: accumulator 1 starts at column 192, and the epilogue
// of a tile drains the overlapped columns first and reports it (barrier
// ovl), so the next tile's MMAs may start while the rest drains.  K-snake
// as in gemm_pair_kernel.
constexpr int MX8P_STAGES = 6;
constexpr int MX8P_A_BYTES = GEMM_BM * 128;
constexpr int MX8P_BH_BYTES = 128 * 128;
constexpr int MX8P_SFA_BYTES = 512;
constexpr int MX8P_STAGE_BYTES = MX8P_A_BYTES + MX8P_BH_BYTES + MX8P_SFA_BYTES;
constexpr int MX8P_SMEM_BYTES = MX8P_STAGES * MX8P_STAGE_BYTES + 1024 + 256;
constexpr uint32_t MX8P_ACC1_COL = 192;
constexpr uint32_t MX8P_SFA_COL = 448;  // 4 columns
constexpr uint32_t MX8P_SFB_COL = 464;  // 32 columns of byte 127
static_assert(MX8P_ACC1_COL + 256 <= MX8P_SFA_COL && MX8P_SFB_COL + 32 <= 512, "TMEM");

template <class Epi>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_mx8_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                         const __grid_constant__ CUtensorMap tmSFA, int M, int n_tiles_n, int K,
                         int group_m, const Epi epi) {
  constexpr int BN = 256;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = align1024(smem_raw);
  uint8_t *sA = smem;
  uint8_t *sB = sA + MX8P_STAGES * MX8P_A_BYTES;
  uint8_t *sSFA = sB + MX8P_STAGES * MX8P_BH_BYTES;
  uint64_t *full = reinterpret_cast<uint64_t *>(sSFA + MX8P_STAGES * MX8P_SFA_BYTES);
  uint64_t *empty = full + MX8P_STAGES;
  uint64_t *tfull = empty + MX8P_STAGES;  // [2]: accumulator ready
  uint64_t *tempty = tfull + 2;           // [2]: accumulator drained
  uint64_t *ovl = tempty + 2;             // overlapped columns drained
  uint64_t *drain = ovl + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  const int n_pairs = gridDim.x >> 1;
  const int m_tiles = (M + 2 * GEMM_BM - 1) / (2 * GEMM_BM);
  const int n_tiles = m_tiles * n_tiles_n;
  const int kblocks = K / 128;

  if (threadIdx.x == 0) {
    for (int s = 0; s < MX8P_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * 4);  // one arrival per epilogue warp of the pair
    }
    mbar_init(ovl, 2 * 4);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmSFA);
  }
  if (warp == 5) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  if (warp < 4) {
    // B's unit scales (byte 127) in every lane of the B scale columns
    uint32_t ones[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) ones[i] = 0x7F7F7F7Fu;
    tmem_st32_u(tmem_base + (static_cast<uint32_t>(warp * 32) << 16) + MX8P_SFB_COL, ones);
    tmem_st_wait();
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  pdl_wait();
  pdl_trigger();

  if (warp == 4) {
    if (lane == 0) {
      // ---------------- loads (both CTAs), completing on the leader's barrier
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      int local = 0;
      for (int t = pair; t < n_tiles && ok; t += n_pairs, ++local) {
        int mt, nt;
        tile_coords(t, m_tiles, n_tiles_n, group_m, &mt, &nt);
        const int mrow = mt * 2 * GEMM_BM + static_cast<int>(rank) * GEMM_BM;
        for (int it = 0; it < kblocks; ++it) {
          const int kb = (local & 1) ? kblocks - 1 - it : it;  // K-snake
          if (!mbar_wait_cluster(&empty[s], ph ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * MX8P_STAGE_BYTES);
          const uint32_t bar = map_shared_to_rank(&full[s], 0);
          tma_load_2d_pair(sA + s * MX8P_A_BYTES, &tmA, bar, kb * 128, mrow);
          tma_load_3d_pair(sSFA + s * MX8P_SFA_BYTES, &tmSFA, bar, 0, kb, mrow / 128);
          tma_load_2d_pair(sB + s * MX8P_BH_BYTES, &tmB, bar, kb * 128,
                           nt * BN + static_cast<int>(rank) * (BN / 2));
          if (++s == MX8P_STAGES) {
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
      bool ok = true;
      const uint32_t sfa = tmem_base + MX8P_SFA_COL;
      const uint32_t sfb = tmem_base + MX8P_SFB_COL;
      for (int t = pair, i = 0; t < n_tiles && ok; t += n_pairs, ++i) {
        const int acc = i & 1;
        // this accumulator's own columns: drained by the epilogue of tile i - 2;
        // the overlapped ones: by the epilogue of tile i - 1
        if (!mbar_wait_cluster(&tempty[acc], static_cast<uint32_t>((i >> 1) & 1) ^ 1, abort_flag))
          break;
        if (i > 0 && !mbar_wait_cluster(ovl, static_cast<uint32_t>((i - 1) & 1), abort_flag)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + (acc ? MX8P_ACC1_COL : 0);
        for (int it = 0; it < kblocks; ++it) {  // k-blocks in the producer's order
          if (!mbar_wait_cluster(&full[s], ph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          tmem_cp_sf_pair(sfa, sdesc_kmajor_none(smem_u32(sSFA + s * MX8P_SFA_BYTES), 128));
          const uint64_t ad = sdesc_kmajor_sw128(smem_u32(sA + s * MX8P_A_BYTES));
          const uint64_t bd = sdesc_kmajor_sw128(smem_u32(sB + s * MX8P_BH_BYTES));
#pragma unroll
          for (int j = 0; j < 4; ++j)
            umma_mx8_pair(d, ad + 2 * j, bd + 2 * j, idesc_mx8(2 * GEMM_BM, BN, j), sfa, sfb,
                          (it | j) != 0);
          umma_commit_pair_both(&empty[s]);
          if (++s == MX8P_STAGES) {
            s = 0;
            ph ^= 1;
          }
        }
        if (ok) umma_commit_pair_both(&tfull[acc]);
      }
      umma_commit_pair_both(drain);
      mbar_wait_cluster(drain, 0, nullptr, WAIT_LIMIT_NS / 4);
    }
  } else {
    // ---------------- epilogue warps 0..3 (both CTAs, own 128 rows)
    const int r = warp * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t ovl_leader = map_shared_to_rank(ovl, 0);
    constexpr int C = Epi::COLS;  // 64 accumulator columns overlap: the top 64 of
    constexpr int OV = C - 64;    // acc 0's epilogue columns, the bottom 64 of acc 1's
    for (int t = pair, i = 0; t < n_tiles; t += n_pairs, ++i) {
      const int acc = i & 1;
      const bool ok =
          mbar_wait_cluster(&tfull[acc], static_cast<uint32_t>((i >> 1) & 1), abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      int mt, nt;
      tile_coords(t, m_tiles, n_tiles_n, group_m, &mt, &nt);
      const int m0 = mt * 2 * GEMM_BM + static_cast<int>(rank) * GEMM_BM;
      const uint32_t tacc = tmem_base + (acc ? MX8P_ACC1_COL : 0) + lane_base;
      epi.part(m0, nt * BN, tacc, r, acc ? 0 : OV, acc ? 64 : C);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(ovl_leader);
      epi.part(m0, nt * BN, tacc, r, acc ? 64 : 0, acc ? C : OV);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(map_shared_to_rank(&tempty[acc], 0));
    }
  }

  __syncwarp();
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  if (warp == 5) tmem_dealloc_pair(tmem_base, 512);
}

}  // namespace ig4
