// NVFP4 (block-scaled FP4) kernels: the GEMMs on tcgen05 kind::mxf4nvf4
// (single CTAs and CTA pairs), the packing of block scales into the order
// the tensor cores read, and the activation quantiser.
//
// NVFP4 activations: bf16 rows -> E2M1 codes, E4M3 block scales (one per 16
// elements, written in the tensor cores' scale-block order) and an fp32 row
// scale, for the block-scaled FP4 GEMMs.
//
// Source: "不用再充会员！Ideogram 4.0 NF4 免费本地部署" (deployment article),
// section "2.2 NVFP4 Mixed": the FFN linears run in NVFP4 (4-bit E2M1 values
// sharing an E4M3 scale per block), the attention projections and the time
// embedding in FP8.  The tensor cores' block is 16 elements.
//
// Recipe per row m (every step one float32 operation):
//   s[m]       = amax_k |x[m, k]| / (6 * 448), or 1 for an all-zero row;
//   sc[m, b]   = RNE_E4M3(amax over block b of |x[m, :]| / (6 * s[m]));
//   code[m, k] = RNE_E2M1(x[m, k] * (1 / (s[m] * sc[m, k / 16]))), 0 where
//                that scale is 0; E2M1 saturates at +-6, E4M3 at 448.
// so x[m, k] ~= s[m] * sc[m, k / 16] * e2m1(code[m, k]).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ig4_gemm.cuh"
#include "ig4_ptx.cuh"

namespace ig4 {

constexpr int NVF4Q_THREADS = 128;  // one warp per row

// Eight fp32 values -> eight E2M1 codes (round to nearest even, saturating),
// element 2i in the low nibble of byte i.
__device__ __forceinline__ uint32_t pack_e2m1x8(const float *v) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return out;
}

// Value of a non-negative E4M3 code (0x00..0x7E): exponent field 0 is
// subnormal, m * 2^-9; otherwise (8 + m) * 2^(e - 10), built as float bits.
__device__ __forceinline__ float e4m3_code_value(uint32_t c) {
  const uint32_t e = c >> 3, m = c & 7;
  return e == 0 ? static_cast<float>(m) * 0.001953125f : __uint_as_float(((e + 120) << 23) | (m << 20));
}

// Byte offset of the scale of (row r, 16-element block b) in the packed
// scale blocks of a [rows][K] operand: 512 bytes per 128 rows x 64 K,
// byte 16 (r % 32) + 4 ((r % 128) / 32) + b % 4.
__device__ __forceinline__ long nvf4_sf_offset(int r, int b, int K) {
  const long blk = static_cast<long>(r >> 7) * (K >> 6) + (b >> 2);
  return blk * 512 + 16 * (r & 31) + 4 * ((r & 127) >> 5) + (b & 3);
}

__device__ __forceinline__ void unpack_bf16x16(uint4 a, uint4 b, float (&f)[16]) {
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// x bf16 [M][K] (K % 64 == 0) -> codes [M][K/2], packed scales, row_scale [M].
__global__ void __launch_bounds__(NVF4Q_THREADS)
    nvf4_quantize_kernel(const __nv_bfloat16 *__restrict__ x, int M, int K,
                         uint8_t *__restrict__ codes, uint8_t *__restrict__ sf,
                         float *__restrict__ row_scale) {
  pdl_wait();
  pdl_trigger();
  const int row = blockIdx.x * (NVF4Q_THREADS / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  const uint4 *xr = reinterpret_cast<const uint4 *>(x + static_cast<long>(row) * K);
  const int nblk = K / 16;
  float amax = 0.0f;
#pragma unroll 4
  for (int b = lane; b < nblk; b += 32) {
    float f[16];
    unpack_bf16x16(__ldg(xr + 2 * b), __ldg(xr + 2 * b + 1), f);
#pragma unroll
    for (int e = 0; e < 16; ++e) amax = fmaxf(amax, fabsf(f[e]));
  }
  amax = warp_max(amax);
  const float s = amax > 0.0f ? amax / 2688.0f : 1.0f;
  const float t = 6.0f * s;
  uint2 *cr = reinterpret_cast<uint2 *>(codes + static_cast<long>(row) * (K / 2));
#pragma unroll 2
  for (int b = lane; b < nblk; b += 32) {
    float f[16];
    unpack_bf16x16(__ldg(xr + 2 * b), __ldg(xr + 2 * b + 1), f);
    float bam = 0.0f;
#pragma unroll
    for (int e = 0; e < 16; ++e) bam = fmaxf(bam, fabsf(f[e]));
    const uint32_t sc = pack_e4m3x2(bam / t, 0.0f) & 0xFFu;
    const float d = s * e4m3_code_value(sc);
    const float inv = d > 0.0f ? 1.0f / d : 0.0f;
#pragma unroll
    for (int e = 0; e < 16; ++e) f[e] = f[e] * inv;
    cr[b] = make_uint2(pack_e2m1x8(f), pack_e2m1x8(f + 8));
    sf[nvf4_sf_offset(row, b, K)] = static_cast<uint8_t>(sc);
  }
  if (lane == 0) row_scale[row] = s;
}

// ------------------------------------------------------ NVFP4 kernel
// C = (A * SFA) (B * SFB)^T on block-scaled FP4 tensor-core MMAs
// (tcgen05.mma kind::mxf4nvf4, block16): A [M][K] and B [N][K] are E2M1 codes,
// two per byte (K contiguous), each row carrying one UE4M3 scale per 16
// K-elements.  Tiles 128 x 128, 256 K-elements (128 bytes per row) per stage:
// TMA brings the A and B code tiles (128-byte swizzle) and a 1D bulk copy
// each 2 KB scale block of A and of B, stored in global memory already in the
// order the tensor cores read them (per 128 rows and 64 K-elements, 512 bytes:
// byte 16 * (r % 32) + 4 * (r / 32) + (k / 16) % 4).  The MMA thread copies a
// stage's scales into TMEM (tcgen05.cp 32x128b.warpx4, a TMEM region per
// stage) and issues four K = 64 MMAs.  The epilogue applies the per-row scale
// of A and the per-column scale of B in fp32 (EpiStore with FP8 = true).
// Two tile widths: 128 (two TMEM accumulators, six stages) and 256 (one
// accumulator, four stages; B brings 2 scale blocks per K chunk): TMEM holds
// the accumulators plus a 16 + 4 * (BN / 128)... scale region per stage.
template <int BN>
struct Nvf4Shape {
  static constexpr int ACC = BN == 128 ? 2 : 1;               // accumulator buffers
  static constexpr int STAGES = BN == 128 ? 6 : 4;
  static constexpr int A_BYTES = GEMM_BM * 128;                // 16 KB of codes
  static constexpr int B_BYTES = BN * 128;
  static constexpr int SFA_BYTES = 2048;                       // 4 blocks of 512 B
  static constexpr int SFB_BYTES = 2048 * (BN / 128);
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
  static constexpr uint32_t SF_COLS = 16 + 16 * (BN / 128);   // TMEM scale columns per stage
  static constexpr uint32_t TMEM_SF = ACC * BN;
  static_assert(TMEM_SF + STAGES * SF_COLS <= 512, "TMEM");
};
constexpr int NVF4_BN = 128;
constexpr uint32_t NVF4_TMEM_COLS = 512;

template <int BN, class Epi>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_nvf4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const uint8_t *__restrict__ sfa, const uint8_t *__restrict__ sfb, int M,
                     int n_tiles_n, int K, int group_m, const Epi epi) {
  using S = Nvf4Shape<BN>;
  constexpr int NVF4_STAGES = S::STAGES;
  constexpr uint32_t IDESC = idesc_nvf4(GEMM_BM, BN);
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = align1024(smem_raw);
  uint8_t *sA = smem;
  uint8_t *sB = sA + NVF4_STAGES * S::A_BYTES;
  uint8_t *sSFA = sB + NVF4_STAGES * S::B_BYTES;
  uint8_t *sSFB = sSFA + NVF4_STAGES * S::SFA_BYTES;
  uint64_t *full = reinterpret_cast<uint64_t *>(sSFB + NVF4_STAGES * S::SFB_BYTES);
  uint64_t *empty = full + NVF4_STAGES;
  uint64_t *tfull = empty + NVF4_STAGES;
  uint64_t *tempty = tfull + 2;
  uint64_t *drain = tempty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m_tiles = (M + GEMM_BM - 1) / GEMM_BM;
  const int n_tiles = m_tiles * n_tiles_n;
  const int kblocks = K / 256;
  const long sf_row_block = static_cast<long>(K / 64) * 512;  // bytes per 128 rows

  if (threadIdx.x == 0) {
    for (int s = 0; s < NVF4_STAGES; ++s) {
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
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, NVF4_TMEM_COLS);
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
      // ---------------- loads: code tiles by TMA, scale blocks by bulk copy
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
          tma_load_2d(sA + s * S::A_BYTES, &tmA, &full[s], kb * 128, mt * GEMM_BM);
          tma_load_2d(sB + s * S::B_BYTES, &tmB, &full[s], kb * 128, nt * BN);
          bulk_load(sSFA + s * S::SFA_BYTES, sfa + mt * sf_row_block + kb * 2048, 2048, &full[s]);
#pragma unroll
          for (int q = 0; q < BN / 128; ++q)
            bulk_load(sSFB + s * S::SFB_BYTES + 2048 * q,
                      sfb + (nt * (BN / 128) + q) * sf_row_block + kb * 2048, 2048, &full[s]);
          ++issued;
          if (++s == NVF4_STAGES) {
            s = 0;
            ph ^= 1;
          }
        }
      }
      if (!ok) {
        for (long i = (issued > NVF4_STAGES ? issued - NVF4_STAGES : 0); i < issued; ++i)
          mbar_wait(&full[i % NVF4_STAGES], static_cast<uint32_t>((i / NVF4_STAGES) & 1), nullptr,
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
        const int buf = local % S::ACC;
        const uint32_t use = static_cast<uint32_t>(local / S::ACC);
        if (!mbar_wait(&tempty[buf], (use & 1) ^ 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * BN;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&full[s], ph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // this stage's scales -> TMEM: A at sf + 4j, B at sf + 16 + (BN / 32) j
          // (per K = 64 step, 4 columns per 128 rows of the operand)
          constexpr uint32_t NB = BN / 128;
          const uint32_t sf = tmem_base + S::TMEM_SF + S::SF_COLS * s;
          const uint32_t sfa_s = smem_u32(sSFA + s * S::SFA_BYTES);
          const uint32_t sfb_s = smem_u32(sSFB + s * S::SFB_BYTES);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            tmem_cp_sf(sf + 4 * j, sdesc_kmajor_none(sfa_s + 512 * j, 128));
#pragma unroll
            for (uint32_t q = 0; q < NB; ++q)
              tmem_cp_sf(sf + 16 + 4 * NB * j + 4 * q, sdesc_kmajor_none(sfb_s + 2048 * q + 512 * j, 128));
          }
          const uint32_t a_base = smem_u32(sA + s * S::A_BYTES);
          const uint32_t b_base = smem_u32(sB + s * S::B_BYTES);
#pragma unroll
          for (int j = 0; j < 4; ++j) {  // K = 64 E2M1 values = 32 bytes per MMA
            const uint64_t ad = sdesc_kmajor_sw128(a_base + 32 * j);
            const uint64_t bd = sdesc_kmajor_sw128(b_base + 32 * j);
            umma_nvf4(d_tmem, ad, bd, IDESC, sf + 4 * j, sf + 16 + 4 * NB * j, (kb | j) != 0);
          }
          umma_commit(&empty[s]);
          if (++s == NVF4_STAGES) {
            s = 0;
            ph ^= 1;
          }
        }
        if (ok) umma_commit(&tfull[buf]);
      }
      umma_commit(drain);
      mbar_wait(drain, 0, nullptr, WAIT_LIMIT_NS / 4);
    }
  } else {
    // ---------------- epilogue warps 0..3
    const int r = warp * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    int local = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++local) {
      const int buf = local % S::ACC;
      const uint32_t use = static_cast<uint32_t>(local / S::ACC);
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
  if (warp == 5) tmem_dealloc(tmem_base, NVF4_TMEM_COLS);
}

// NVFP4 on CTA pairs: a pair tile is 256 rows x 256 columns (tcgen05.mma
// cta_group::2, M = 256): each CTA loads its 128 A rows, half of the B rows,
// its A scale blocks and the scale blocks of all 256 B rows (both CTAs' MMAs
// read the B scales of every column); all loads complete on the leader's
// barrier.  Per stage and CTA: 32 KB of codes + 6 KB of scales per 512 MMA
// clocks at the FP4 rate, the same bytes per clock as the FP8 pair kernel.
// TMEM: two 256-column accumulators that overlap in 96 columns, acc 0 at
// [0, 256) and acc 1 at [160, 416), and two 48-column scale regions at 416
// and 464.  Four copy warps move each k-block's scale blocks into region
// g % 2 (twelve tcgen05.cp of 512 bytes, three per warp: a copy holds its
// issuing thread for ~50 cycles, and copies from different threads run side
// by side, so twelve in one thread would outlast the k-block's 512 cycles of
// FP4 MMAs) and signal the MMA thread through sf_ready (one arrival per copy
// warp); a region is refilled once the MMAs of k-block g - 2 that read it
// have completed (the stage's empty barrier).  The epilogue of a tile drains
// the overlapped columns first and releases them (ovl), so the next tile's
// MMAs start while it converts the rest.
// DUAL_B (SwiGLU gate/up): B rows of the tile's first 128 columns come from
// tmB (gate) and of the last 128 from tmB2 (up), both at rows nt * 128, with
// their scale blocks from tmSFB / tmSFB2 (one 128-row block each); otherwise
// B rows nt * 256 + [0, 256) come from tmB and their two scale blocks from
// tmSFB.
constexpr int NVF4P_STAGES = 5;
constexpr int NVF4P_COPY_WARPS = 4;  // one MMA's scale blocks (three copies) per warp
// Epilogue warps 0-3, TMA 4, MMA 5, copies 6-9.  Registers are allocated per
// group of four warps, so ten warps are charged as twelve: 168 per thread.
constexpr int NVF4P_THREADS = 32 * (6 + NVF4P_COPY_WARPS);
constexpr int NVF4P_A_BYTES = GEMM_BM * 128;
constexpr int NVF4P_BH_BYTES = 128 * 128;
constexpr int NVF4P_SFA_BYTES = 2048;
constexpr int NVF4P_SFB_BYTES = 4096;
constexpr int NVF4P_STAGE_BYTES = NVF4P_A_BYTES + NVF4P_BH_BYTES + NVF4P_SFA_BYTES + NVF4P_SFB_BYTES;
constexpr int NVF4P_SMEM_BYTES = NVF4P_STAGES * NVF4P_STAGE_BYTES + 1024 + 256;
constexpr uint32_t NVF4P_ACC1_COL = 160;
constexpr int NVF4P_OVL = 256 - static_cast<int>(NVF4P_ACC1_COL);  // overlapped columns
constexpr uint32_t NVF4P_SF_COL = 416;                             // two regions of 48
static_assert(NVF4P_ACC1_COL + 256 <= NVF4P_SF_COL && NVF4P_SF_COL + 2 * 48 <= 512, "TMEM");

// SwiGLU epilogue of a dual-B pair tile (EpiSwiGLU layout: gate in
// accumulator columns [0, 128), up in [128, 256)).  The 96 columns shared
// with the other accumulator (acc 0: up columns [160, 256); acc 1: gate
// columns [0, 96)) are read into registers and released first, so the next
// tile's MMAs wait for three TMEM loads rather than for 96 of the 128 output
// columns; then the four 32-column chunks are converted.
template <class Epi>
__device__ __forceinline__ void nvf4_swiglu_epilogue(const Epi &ep, int m0, int n0, uint32_t tacc,
                                                     int r, int acc, uint32_t ovl_leader,
                                                     int lane) {
  float ov[3][32];
  const uint32_t obase = acc ? 0u : 160u;
#pragma unroll
  for (int k = 0; k < 3; ++k) tmem_ld32(tacc + obase + 32 * k, ov[k]);
  tmem_ld_wait();
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive_cluster(ovl_leader);
  const int row = m0 + r;
  const bool valid = row < ep.M;
  const float rs = valid ? __ldg(ep.a_scale + row) : 1.0f;
  const int n = n0 / 2;  // tile index * 128
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    float g[32], up[32];
    if (acc == 0) {  // up of chunks 1..3 preloaded
      tmem_ld32(tacc + 32 * c, g);
      if (c == 0) tmem_ld32(tacc + 128, up);
      tmem_ld_wait();
      if (c > 0) {
#pragma unroll
        for (int i = 0; i < 32; ++i) up[i] = ov[c > 0 ? c - 1 : 0][i];
      }
    } else {  // gate of chunks 0..2 preloaded
      tmem_ld32(tacc + 128 + 32 * c, up);
      if (c == 3) tmem_ld32(tacc + 96, g);
      tmem_ld_wait();
      if (c < 3) {
#pragma unroll
        for (int i = 0; i < 32; ++i) g[i] = ov[c < 3 ? c : 0][i];
      }
    }
    if (!valid) continue;
    apply_scales<true>(g, rs, ep.s_gate + n + 32 * c);
    apply_scales<true>(up, rs, ep.s_up + n + 32 * c);
#pragma unroll
    for (int i = 0; i < 32; ++i) g[i] = silu_f(g[i]) * up[i];
    store32_bf16(ep.u + static_cast<long>(row) * ep.I + n + 32 * c, g);
  }
}

template <bool DUAL_B, class Epi>
__global__ void __launch_bounds__(NVF4P_THREADS, 1)
    gemm_nvf4_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                          const __grid_constant__ CUtensorMap tmB2,
                          const __grid_constant__ CUtensorMap tmSFA,
                          const __grid_constant__ CUtensorMap tmSFB,
                          const __grid_constant__ CUtensorMap tmSFB2, int M, int n_tiles_n, int K,
                          int group_m, const Epi epi) {
  constexpr int BN = 256;
  constexpr uint32_t IDESC = idesc_nvf4(2 * GEMM_BM, BN);
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = align1024(smem_raw);
  uint8_t *sA = smem;
  uint8_t *sB = sA + NVF4P_STAGES * NVF4P_A_BYTES;
  uint8_t *sSFA = sB + NVF4P_STAGES * NVF4P_BH_BYTES;
  uint8_t *sSFB = sSFA + NVF4P_STAGES * NVF4P_SFA_BYTES;
  uint64_t *full = reinterpret_cast<uint64_t *>(sSFB + NVF4P_STAGES * NVF4P_SFB_BYTES);
  uint64_t *empty = full + NVF4P_STAGES;
  uint64_t *tfull = empty + NVF4P_STAGES;  // [2]: accumulator ready
  uint64_t *tempty = tfull + 2;            // [2]: accumulator drained
  uint64_t *ovl = tempty + 2;              // overlapped columns drained
  uint64_t *drain = ovl + 1;
  uint64_t *sf_ready = drain + 1;          // [2]: scale region copied
  uint64_t *cdrain = sf_ready + 2;         // the copy warps' last copies done
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(cdrain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1;
  const int n_pairs = gridDim.x >> 1;
  const int m_tiles = (M + 2 * GEMM_BM - 1) / (2 * GEMM_BM);
  const int n_tiles = m_tiles * n_tiles_n;
  const int kblocks = K / 256;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NVF4P_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * 4);  // one arrival per epilogue warp of the pair
    }
    mbar_init(ovl, 2 * 4);
    mbar_init(drain, 1);
    mbar_init(&sf_ready[0], NVF4P_COPY_WARPS);  // one commit per copy warp
    mbar_init(&sf_ready[1], NVF4P_COPY_WARPS);
    mbar_init(cdrain, NVF4P_COPY_WARPS);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmSFA);
    tma_prefetch_desc(&tmSFB);
    if (DUAL_B) {
      tma_prefetch_desc(&tmB2);
      tma_prefetch_desc(&tmSFB2);
    }
  }
  if (warp == 5) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();
  pdl_trigger();

  if (warp == 4) {
    if (lane == 0) {
      // ---------------- loads (both CTAs), completing on the leader's barrier
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int t = pair; t < n_tiles && ok; t += n_pairs) {
        int mt, nt;
        tile_coords(t, m_tiles, n_tiles_n, group_m, &mt, &nt);
        const int mrow = mt * 2 * GEMM_BM + static_cast<int>(rank) * GEMM_BM;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait_cluster(&empty[s], ph ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * NVF4P_STAGE_BYTES);
          const uint32_t bar = map_shared_to_rank(&full[s], 0);
          tma_load_2d_pair(sA + s * NVF4P_A_BYTES, &tmA, bar, kb * 128, mrow);
          // scale blocks: [128 words of 4 B] x [4 K chunks] x [row blocks]
          tma_load_3d_pair(sSFA + s * NVF4P_SFA_BYTES, &tmSFA, bar, 0, 4 * kb, mrow / 128);
          if constexpr (DUAL_B) {
            tma_load_2d_pair(sB + s * NVF4P_BH_BYTES, rank ? &tmB2 : &tmB, bar, kb * 128, nt * 128);
            tma_load_3d_pair(sSFB + s * NVF4P_SFB_BYTES, &tmSFB, bar, 0, 4 * kb, nt);
            tma_load_3d_pair(sSFB + s * NVF4P_SFB_BYTES + NVF4P_SFB_BYTES / 2, &tmSFB2, bar, 0,
                             4 * kb, nt);
          } else {
            tma_load_2d_pair(sB + s * NVF4P_BH_BYTES, &tmB, bar, kb * 128,
                             nt * BN + static_cast<int>(rank) * (BN / 2));
            tma_load_3d_pair(sSFB + s * NVF4P_SFB_BYTES, &tmSFB, bar, 0, 4 * kb, nt * 2);
          }
          if (++s == NVF4P_STAGES) {
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
      long g = 0;  // k-blocks over the tiles
      for (int t = pair, i = 0; t < n_tiles && ok; t += n_pairs, ++i) {
        const int acc = i & 1;
        // this accumulator's own columns: drained by the epilogue of tile i - 2;
        // the overlapped ones: by the epilogue of tile i - 1
        if (!mbar_wait_cluster(&tempty[acc], static_cast<uint32_t>((i >> 1) & 1) ^ 1, abort_flag))
          break;
        if (i > 0 && !mbar_wait_cluster(ovl, static_cast<uint32_t>((i - 1) & 1), abort_flag)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + (acc ? NVF4P_ACC1_COL : 0);
        for (int kb = 0; kb < kblocks; ++kb, ++g) {
          if (!mbar_wait_cluster(&full[s], ph, abort_flag) ||
              !mbar_wait_cluster(&sf_ready[g & 1], static_cast<uint32_t>((g >> 1) & 1),
                                 abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sf = tmem_base + NVF4P_SF_COL + 48 * static_cast<uint32_t>(g & 1);
          const uint32_t a_base = smem_u32(sA + s * NVF4P_A_BYTES);
          const uint32_t b_base = smem_u32(sB + s * NVF4P_BH_BYTES);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint64_t ad = sdesc_kmajor_sw128(a_base + 32 * j);
            const uint64_t bd = sdesc_kmajor_sw128(b_base + 32 * j);
            umma_nvf4_pair(d, ad, bd, IDESC, sf + 4 * j, sf + 16 + 8 * j, (kb | j) != 0);
          }
          umma_commit_pair_both(&empty[s]);
          if (++s == NVF4P_STAGES) {
            s = 0;
            ph ^= 1;
          }
        }
        if (ok) umma_commit_pair_both(&tfull[acc]);
      }
      umma_commit_pair_both(drain);
      mbar_wait_cluster(drain, 0, nullptr, WAIT_LIMIT_NS / 4);
    }
  } else if (warp >= 6) {
    if (lane == 0 && rank == 0) {
      // ---------------- scale copies (leader CTA): stage data -> TMEM region g % 2,
      // warp 6 + c the blocks of MMA j of the k-block for j % NVF4P_COPY_WARPS == c
      const int j0 = warp - 6;
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      long g = 0;
      for (int t = pair; t < n_tiles && ok; t += n_pairs) {
        for (int kb = 0; kb < kblocks; ++kb, ++g) {
          // the stage has landed; region g % 2 was last read by the MMAs of
          // k-block g - 2, which completed the empty barrier of their stage
          bool ready = mbar_wait_cluster(&full[s], ph, abort_flag);
          if (ready && g >= 2) {
            const long gp = g - 2;
            ready = mbar_wait_cluster(&empty[gp % NVF4P_STAGES],
                                      static_cast<uint32_t>((gp / NVF4P_STAGES) & 1), abort_flag);
          }
          if (!ready) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sf = tmem_base + NVF4P_SF_COL + 48 * static_cast<uint32_t>(g & 1);
          const uint32_t sfa_s = smem_u32(sSFA + s * NVF4P_SFA_BYTES);
          const uint32_t sfb_s = smem_u32(sSFB + s * NVF4P_SFB_BYTES);
#pragma unroll
          for (int j = j0; j < 4; j += NVF4P_COPY_WARPS) {
            tmem_cp_sf_pair(sf + 4 * j, sdesc_kmajor_none(sfa_s + 512 * j, 128));
            tmem_cp_sf_pair(sf + 16 + 8 * j, sdesc_kmajor_none(sfb_s + 512 * j, 128));
            tmem_cp_sf_pair(sf + 16 + 8 * j + 4, sdesc_kmajor_none(sfb_s + 2048 + 512 * j, 128));
          }
          umma_commit_pair_both(&sf_ready[g & 1]);
          if (++s == NVF4P_STAGES) {
            s = 0;
            ph ^= 1;
          }
        }
      }
      // no copy of this thread is in flight when TMEM is freed
      umma_commit_pair_both(cdrain);
      mbar_wait_cluster(cdrain, 0, nullptr, WAIT_LIMIT_NS / 4);
    }
  } else {
    // ---------------- epilogue warps 0..3 (both CTAs, own 128 rows)
    const int r = warp * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t ovl_leader = map_shared_to_rank(ovl, 0);
    constexpr int C = Epi::COLS;  // NVF4P_OVL accumulator columns overlap: the top ones
    constexpr int OV = C - NVF4P_OVL;  // of acc 0's epilogue columns, the bottom ones of acc 1's
    for (int t = pair, i = 0; t < n_tiles; t += n_pairs, ++i) {
      const int acc = i & 1;
      const bool ok =
          mbar_wait_cluster(&tfull[acc], static_cast<uint32_t>((i >> 1) & 1), abort_flag);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      int mt, nt;
      tile_coords(t, m_tiles, n_tiles_n, group_m, &mt, &nt);
      const int m0 = mt * 2 * GEMM_BM + static_cast<int>(rank) * GEMM_BM;
      const uint32_t tacc = tmem_base + (acc ? NVF4P_ACC1_COL : 0) + lane_base;
      if constexpr (DUAL_B) {
        nvf4_swiglu_epilogue(epi, m0, nt * BN, tacc, r, acc, ovl_leader, lane);
      } else {
        epi.part(m0, nt * BN, tacc, r, acc ? 0 : OV, acc ? NVF4P_OVL : C);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(ovl_leader);
        epi.part(m0, nt * BN, tacc, r, acc ? NVF4P_OVL : 0, acc ? C : OV);
      }
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

// Scale factors [rows][K/16] (row-major UE4M3 bytes) -> the tensor cores'
// block order (see gemm_nvf4_kernel); rows padded to a multiple of 128 with
// zero scales.  One thread per output byte.
__global__ void nvf4_pack_scales_kernel(const uint8_t *__restrict__ src, uint8_t *__restrict__ dst,
                                        int rows, int K, long total) {
  const int kc = K / 64;  // 64-element chunks per row
  for (long o = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; o < total;
       o += static_cast<long>(gridDim.x) * blockDim.x) {
    const long blk = o / 512;
    const int w = static_cast<int>(o - blk * 512);
    const long rb = blk / kc;           // 128-row block
    const int c = static_cast<int>(blk - rb * kc);
    const int r = static_cast<int>(rb * 128 + (w >> 4) + 32 * ((w >> 2) & 3));
    const int k16 = c * 4 + (w & 3);
    dst[o] = r < rows ? src[static_cast<long>(r) * (K / 16) + k16] : 0;
  }
}

}  // namespace ig4
