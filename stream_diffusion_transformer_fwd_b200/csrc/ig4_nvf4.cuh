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

}  // namespace ig4
