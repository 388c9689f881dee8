// ig4_mx8.cuh - FP8 activations with 1x32 block scales (MX format) for the
// FP8 path's two activation-side GEMM inputs (the attention output feeding
// the out-projection, u feeding the down-projection): the encoding, the row
// quantiser and the SwiGLU epilogue that writes it.  The block-scaled GEMM
// that consumes it is gemm_pair_kernel's MX8A variant (tcgen05
// kind::mxf8f6f4).
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

}  // namespace ig4
