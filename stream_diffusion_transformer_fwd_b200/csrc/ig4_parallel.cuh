// ig4_parallel.cuh - device code of the multi-GPU layouts of the block
// ("SGLang cookbook: Ideogram 4", section 3, tensor and sequence
// parallelism: TP shards the DiT weights over a degree that divides the 18
// heads; Ulysses SP keeps the weights whole and shards the image tokens).
//
//   tp_reduce_kernel     sum of the tensor-parallel shards' fp32 partial
//                        outputs (rank order, so every rank gets the same
//                        bits), stored in the residual stream's type;
//   exchange_copy_kernel the strided block copies that pack and unpack the
//                        Ulysses exchange buffers (tokens <-> heads).
// Both are memory-bound streaming kernels: 16-byte accesses where the
// layout allows, consecutive threads on consecutive addresses.
#pragma once

#include "ig4_ptx.cuh"

namespace ig4 {

constexpr int TP_MAX_RANKS = 8;

struct TpSources {
  const float *p[TP_MAX_RANKS];
};

// out[i] = sum_r src.p[r][i], r = 0 .. n_src-1, for n8 groups of 8 elements.
template <typename OT>
__global__ void __launch_bounds__(256)
    tp_reduce_kernel(const __grid_constant__ TpSources src, int n_src, OT *__restrict__ out,
                     long n8) {
  pdl_wait();
  pdl_trigger();
  for (long i = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<long>(gridDim.x) * blockDim.x) {
    float a[8];
    {
      const float4 *s = reinterpret_cast<const float4 *>(src.p[0]) + 2 * i;
      const float4 x0 = s[0], x1 = s[1];
      a[0] = x0.x; a[1] = x0.y; a[2] = x0.z; a[3] = x0.w;
      a[4] = x1.x; a[5] = x1.y; a[6] = x1.z; a[7] = x1.w;
    }
    for (int r = 1; r < n_src; ++r) {
      const float4 *s = reinterpret_cast<const float4 *>(src.p[r]) + 2 * i;
      const float4 x0 = s[0], x1 = s[1];
      a[0] += x0.x; a[1] += x0.y; a[2] += x0.z; a[3] += x0.w;
      a[4] += x1.x; a[5] += x1.y; a[6] += x1.z; a[7] += x1.w;
    }
    if constexpr (sizeof(OT) == 4) {
      float4 *d = reinterpret_cast<float4 *>(out) + 2 * i;
      d[0] = make_float4(a[0], a[1], a[2], a[3]);
      d[1] = make_float4(a[4], a[5], a[6], a[7]);
    } else {
      uint4 w;
      w.x = pack_bf16x2(a[0], a[1]);
      w.y = pack_bf16x2(a[2], a[3]);
      w.z = pack_bf16x2(a[4], a[5]);
      w.w = pack_bf16x2(a[6], a[7]);
      reinterpret_cast<uint4 *>(out)[i] = w;
    }
  }
}

// One strided copy of 2-byte elements: for b < n_b, h < n_h, r < rows,
// e < row_elems:  dst[b*d_b + h*d_h + r*d_r + e] = src[b*s_b + h*s_h + r*s_r + e]
// (offsets in elements).  vec: every offset, stride and row length is a
// multiple of 8 elements and both bases are 16-byte aligned, so the copy
// moves 16-byte units.
struct CopyJob {
  const uint16_t *src;
  uint16_t *dst;
  int n_b, n_h, rows, row_elems;
  long long s_b, s_h, s_r, d_b, d_h, d_r;
  int vec;
};

// the largest launch: 3 text jobs + 3 jobs per source rank, at 8 ranks
constexpr int EXCHANGE_MAX_JOBS = 28;

struct CopyJobs {
  CopyJob j[EXCHANGE_MAX_JOBS];
};

// blockIdx.y = job; the job's (b, h, row, unit) space is walked grid-stride
// along x, unit fastest, so a warp reads and writes consecutive addresses.
__global__ void __launch_bounds__(256)
    exchange_copy_kernel(const __grid_constant__ CopyJobs jobs) {
  pdl_wait();
  pdl_trigger();
  const CopyJob &jb = jobs.j[blockIdx.y];
  const int upr = jb.vec ? jb.row_elems / 8 : jb.row_elems;  // units per row
  const long total = static_cast<long>(jb.n_b) * jb.n_h * jb.rows * upr;
  for (long u = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; u < total;
       u += static_cast<long>(gridDim.x) * blockDim.x) {
    const long rowi = u / upr;
    const int e = static_cast<int>(u - rowi * upr);
    const int r = static_cast<int>(rowi % jb.rows);
    const long bh = rowi / jb.rows;
    const int h = static_cast<int>(bh % jb.n_h);
    const int b = static_cast<int>(bh / jb.n_h);
    const long so = b * jb.s_b + h * jb.s_h + r * jb.s_r;
    const long dof = b * jb.d_b + h * jb.d_h + r * jb.d_r;
    if (jb.vec) {
      *reinterpret_cast<uint4 *>(jb.dst + dof + 8 * e) =
          *reinterpret_cast<const uint4 *>(jb.src + so + 8 * e);
    } else {
      jb.dst[dof + e] = jb.src[so + e];
    }
  }
}

}  // namespace ig4
