// ig4_attention.cuh - fused flash-style joint attention, head_dim 256, sm_100a.
//
// One CTA computes o for 128 query rows of one (sample, head), walking the
// keys in tiles of 128:
//   S_j = Q K_j^T     16 tcgen05.mma (M=128, N=128, K=16) with A = Q read from
//                     TMEM and B = K_j from shared memory; fp32 scores in TMEM;
//   softmax           one thread per query row, exp2 domain, in registers;
//   P_j               bf16 into shared memory in the MMA operand layout;
//   O += P_j V_j      8 tcgen05.mma (M=128, N=256, K=16), O (fp32) in TMEM.
// 128-key tiles keep every MMA at N >= 128, the width at which an MMA runs
// at the full tensor rate (N = 64 instructions take ~1.5x their ideal time).
// Q sits in TMEM as the A operand of the scores, so the scores read only K
// from shared memory.
//
// TMEM (512 columns): Q as bf16 pairs [0,128), one S buffer [128,256), O
// [256,512).  S_{j+1} is issued as soon as the softmax has read S_j out of
// TMEM (not when P_j is ready), so the scores of the next tile are computed
// while the exponentials of this one run.
//
// Shared memory: one ring of three 64 KB slots filled by TMA in the order the
// MMAs consume them - Q, K_0, K_1, V_0, K_2, V_1, K_3, V_2, ... - plus one
// 32 KB P buffer.  V arrives transposed ([256, keys], keys contiguous), so
// every operand is K-major with the 128-byte swizzle.
//
// The running maximum used for the exponentials only moves when a row's
// maximum grows by more than 8 (a factor 2^8), so O is rescaled rarely;
// numerator and denominator use the same maximum, so the result is unchanged.
// The softmax computes a tile's exponentials (into packed bf16 registers)
// before it waits for the previous PV product, and only the store of P into
// the single P buffer (and the rare O rescale) waits for it.
//
// Warp roles (192 threads): warps 0-3 softmax + output (warp w owns TMEM
// lanes / query rows 32w..32w+31), warp 4 TMA producer, warp 5 TMEM
// allocation and MMA issue: S_0, S_1, PV_0, S_2, PV_1, ...
//
// Barrier parity: every barrier a role waits on completes at most one phase
// ahead of that wait, so try_wait.parity never mistakes a later phase for the
// awaited one.  Every wait is bounded.
#pragma once

#include "ig4_ptx.cuh"

namespace ig4 {

constexpr int ATT_BM = 128;
constexpr int ATT_BN = 128;   // keys per tile
constexpr int ATT_DH = 256;
constexpr int ATT_THREADS = 192;
constexpr int ATT_SLOTS = 3;
constexpr int ATT_SLOT_BYTES = 65536;                  // Q, K_j (4 chunks [128 x 128 B]) or
                                                       // V_j^T (2 chunks [256 x 128 B])
constexpr int ATT_P_BYTES = ATT_BM * ATT_BN * 2;       // 32 KB: 2 chunks [128 x 128 B]
constexpr int ATT_OFF_P = ATT_SLOTS * ATT_SLOT_BYTES;
constexpr int ATT_OFF_BAR = ATT_OFF_P + ATT_P_BYTES;
constexpr int ATT_SMEM_BYTES = ATT_OFF_BAR + 256 + 1024;
constexpr uint32_t ATT_TMEM_COLS = 512;
constexpr uint32_t ATT_TMEM_Q = 0;
constexpr uint32_t ATT_TMEM_S = 128;
constexpr uint32_t ATT_TMEM_O = 256;
// log2(e) / sqrt(256)
constexpr float ATT_SCALE_LOG2 = 0.09016844005556021f;
constexpr float ATT_RESCALE_THRESHOLD = 8.0f;

// The ring's load / consumption order: item 0 is Q; then K_0, K_1 (if any);
// then, for each tile j, V_j followed by K_{j+2} (if that tile exists).
// kind(): 0 = Q, 1 = K, 2 = V, with the tile index in *tile.
struct AttRing {
  int nkv;
  __device__ __forceinline__ int items() const { return 1 + 2 * nkv; }
  __device__ __forceinline__ int kind(int i, int *tile) const {
    if (i == 0) { *tile = 0; return 0; }
    if (i == 1) { *tile = 0; return 1; }
    if (nkv == 1) { *tile = 0; return 2; }  // items: Q, K_0, V_0
    if (i == 2) { *tile = 1; return 1; }
    // items from 3 on: V_0, K_2, V_1, K_3, ..., V_{nkv-3}, K_{nkv-1}, V_{nkv-2}, V_{nkv-1}
    const int k = i - 3;
    const int pairs = nkv - 2;  // (V_j, K_{j+2}) for j < nkv - 2
    if (k < 2 * pairs) {
      *tile = (k & 1) ? (k >> 1) + 2 : (k >> 1);
      return (k & 1) ? 1 : 2;
    }
    *tile = (nkv - 2) + (k - 2 * pairs);
    return 2;
  }
};

__global__ void __launch_bounds__(ATT_THREADS, 1)
    attention_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, __nv_bfloat16 *__restrict__ o_out,
                     int L, int H) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sP = smem + ATT_OFF_P;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + ATT_OFF_BAR);
  uint64_t *full = bars + 0;     // [ATT_SLOTS]
  uint64_t *empty = bars + 3;    // [ATT_SLOTS]
  uint64_t *s_full = bars + 6;   // S_j in TMEM
  uint64_t *s_free = bars + 7;   // S_j read out of TMEM (one arrival per softmax warp)
  uint64_t *p_full = bars + 8;   // P_j in shared memory (one arrival per softmax warp)
  uint64_t *pv_done = bars + 9;  // PV_j (and every earlier MMA) complete
  uint64_t *q_tmem = bars + 10;  // Q copied into TMEM (one arrival per softmax warp)
  uint64_t *drain = bars + 11;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 12);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int q0 = blockIdx.x * ATT_BM;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int bh = b * H + h;
  const int nkv = (L + ATT_BN - 1) / ATT_BN;
  const AttRing ring{nkv};

  if (threadIdx.x == 0) {
    for (int s = 0; s < ATT_SLOTS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 4);
    mbar_init(p_full, 4);
    mbar_init(pv_done, 1);
    mbar_init(q_tmem, 4);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, ATT_TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      const int n = ring.items();
      int i = 0;
      bool ok = true;
      for (; i < n; ++i) {
        const int slot = i % ATT_SLOTS;
        const uint32_t ph = static_cast<uint32_t>(i / ATT_SLOTS) & 1;
        if (!mbar_wait(&empty[slot], ph ^ 1, abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(&full[slot], ATT_SLOT_BYTES);
        uint8_t *dst = smem + slot * ATT_SLOT_BYTES;
        int t = 0;
        const int kind = ring.kind(i, &t);
        if (kind == 0) {
          for (int c = 0; c < 4; ++c) tma_load_3d(dst + c * 16384, &tmQ, &full[slot], c * 64, q0, bh);
        } else if (kind == 1) {
          for (int c = 0; c < 4; ++c)
            tma_load_3d(dst + c * 16384, &tmK, &full[slot], c * 64, t * ATT_BN, bh);
        } else {
          for (int c = 0; c < 2; ++c)
            tma_load_3d(dst + c * 32768, &tmV, &full[slot], t * ATT_BN + c * 64, 0, bh);
        }
      }
      if (!ok) {
        // let the loads already issued land before the shared memory goes away
        for (int k = (i > ATT_SLOTS ? i - ATT_SLOTS : 0); k < i; ++k)
          mbar_wait(&full[k % ATT_SLOTS], static_cast<uint32_t>(k / ATT_SLOTS) & 1, nullptr,
                    WAIT_LIMIT_NS / 4);
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      constexpr uint32_t IDESC_S = idesc_bf16(ATT_BM, ATT_BN);
      constexpr uint32_t IDESC_PV = idesc_bf16(ATT_BM, ATT_DH);
      const uint32_t p_base = smem_u32(sP);
      int item = 1;  // ring item consumed next (item 0, Q, is read by the softmax warps)
      bool ok = mbar_wait(q_tmem, 0, abort_flag);
      if (ok) mbar_arrive(&empty[0]);  // Q's slot is free once Q is in TMEM
      auto take = [&](uint32_t *base) -> bool {
        const int slot = item % ATT_SLOTS;
        if (!mbar_wait(&full[slot], static_cast<uint32_t>(item / ATT_SLOTS) & 1, abort_flag))
          return false;
        tc_fence_after();
        *base = smem_u32(smem + slot * ATT_SLOT_BYTES);
        return true;
      };
      auto give = [&]() {
        umma_commit(&empty[item % ATT_SLOTS]);
        ++item;
      };
      auto issue_s = [&]() -> bool {  // S_j into the S buffer, K_j from the ring
        uint32_t k_base;
        if (!take(&k_base)) return false;
#pragma unroll
        for (int kk = 0; kk < ATT_DH / 16; ++kk) {
          const uint64_t bd = sdesc_kmajor_sw128(k_base + (kk >> 2) * 16384 + (kk & 3) * 32);
          umma_bf16_ts(tmem + ATT_TMEM_S, tmem + ATT_TMEM_Q + kk * 8, bd, IDESC_S, kk > 0);
        }
        give();
        umma_commit(s_full);
        return true;
      };
      if (ok) ok = issue_s();  // S_0
      for (int j = 0; j < nkv && ok; ++j) {
        // S_{j+1} as soon as S_j has been read out of TMEM
        if (j + 1 < nkv) {
          if (!mbar_wait(s_free, static_cast<uint32_t>(j) & 1, abort_flag)) break;
          if (!(ok = issue_s())) break;
        }
        // PV_j once P_j is in shared memory
        if (!mbar_wait(p_full, static_cast<uint32_t>(j) & 1, abort_flag)) break;
        uint32_t v_base;
        if (!(ok = take(&v_base))) break;
#pragma unroll
        for (int kk = 0; kk < ATT_BN / 16; ++kk) {
          const uint64_t ad = sdesc_kmajor_sw128(p_base + (kk >> 2) * 16384 + (kk & 3) * 32);
          const uint64_t bd = sdesc_kmajor_sw128(v_base + (kk >> 2) * 32768 + (kk & 3) * 32);
          umma_bf16(tmem + ATT_TMEM_O, ad, bd, IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
        }
        give();
        umma_commit(pv_done);
      }
      umma_commit(drain);
      mbar_wait(drain, 0, nullptr, WAIT_LIMIT_NS / 4);
    }
  } else {
    // -------------------------------------------- softmax warps 0..3
    const int r = warp * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    float m_used = -INFINITY;
    float l_sum = 0.0f;
    bool ok = mbar_wait_warp(&full[0], 0, abort_flag);  // Q (ring item 0)
    if (ok) {
      // Q row r: four 64-column chunks of 128 bytes in the 128-byte-swizzled
      // TMA layout -> TMEM columns [ATT_TMEM_Q + 32c, +32), bf16 pairs.
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        const uint8_t *qrow = smem + c * 16384 + r * 128;
        uint32_t w[32];
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          const uint4 v = *reinterpret_cast<const uint4 *>(qrow + ((g ^ (r & 7)) << 4));
          w[4 * g + 0] = v.x;
          w[4 * g + 1] = v.y;
          w[4 * g + 2] = v.z;
          w[4 * g + 3] = v.w;
        }
        tmem_st32_u(tmem + lane_base + ATT_TMEM_Q + c * 32, w);
      }
      tmem_st_wait();
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(q_tmem);

    for (int j = 0; j < nkv && ok; ++j) {
      if (!mbar_wait_warp(s_full, static_cast<uint32_t>(j) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      float t[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float a[32];
        tmem_ld32(tmem + lane_base + ATT_TMEM_S + c * 32, a);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) t[32 * c + i] = a[i];
      }
      // S_j is in registers: the S buffer may take S_{j+1}.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free);

      const int kbase = j * ATT_BN;
      if (kbase + ATT_BN > L) {
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (kbase + i >= L) t[i] = -INFINITY;
      }
      float m16[16];
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const float a0 = fmaxf(t[8 * q + 0], t[8 * q + 1]);
        const float a1 = fmaxf(t[8 * q + 2], t[8 * q + 3]);
        const float a2 = fmaxf(t[8 * q + 4], t[8 * q + 5]);
        const float a3 = fmaxf(t[8 * q + 6], t[8 * q + 7]);
        m16[q] = fmaxf(fmaxf(a0, a1), fmaxf(a2, a3));
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) m16[q] = fmaxf(m16[q], m16[q + 8]);
      const float mx = fmaxf(fmaxf(fmaxf(m16[0], m16[1]), fmaxf(m16[2], m16[3])),
                             fmaxf(fmaxf(m16[4], m16[5]), fmaxf(m16[6], m16[7]))) *
                       ATT_SCALE_LOG2;

      // Running maximum for this tile (moved only when it grows by more than
      // the threshold) and the factor that rescales what came before.
      float m_new = m_used;
      float f = 1.0f;
      bool need = false;
      if (j == 0) {
        m_new = mx;
      } else if (mx > m_used + ATT_RESCALE_THRESHOLD) {
        need = true;
        m_new = mx;
        f = exp2_approx(m_used - mx);
      }
      const bool any_need = __any_sync(0xffffffffu, need);

      // Exponentials into packed bf16 registers first: they need neither
      // PV_{j-1} nor the P buffer, so they overlap the tensor core's work.
      const float neg_m = -m_new;
      uint32_t pk[64];
      float sums[16];
#pragma unroll
      for (int g = 0; g < 16; ++g) {
        float p[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) p[e] = exp2_approx(fmaf(t[8 * g + e], ATT_SCALE_LOG2, neg_m));
        sums[g] = ((p[0] + p[1]) + (p[2] + p[3])) + ((p[4] + p[5]) + (p[6] + p[7]));
        pk[4 * g + 0] = pack_bf16x2(p[0], p[1]);
        pk[4 * g + 1] = pack_bf16x2(p[2], p[3]);
        pk[4 * g + 2] = pack_bf16x2(p[4], p[5]);
        pk[4 * g + 3] = pack_bf16x2(p[6], p[7]);
      }
#pragma unroll
      for (int g = 0; g < 8; ++g) sums[g] += sums[g + 8];
      const float rowsum =
          ((sums[0] + sums[1]) + (sums[2] + sums[3])) + ((sums[4] + sums[5]) + (sums[6] + sums[7]));

      if (j > 0) {
        // PV_{j-1} must be done: it reads the P buffer and writes O.
        if (!mbar_wait_warp(pv_done, static_cast<uint32_t>(j - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (any_need) {
#pragma unroll 1
          for (int c = 0; c < ATT_DH; c += 32) {
            float o[32];
            tmem_ld32(tmem + lane_base + ATT_TMEM_O + c, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= f;
            tmem_st32(tmem + lane_base + ATT_TMEM_O + c, o);
          }
          tmem_st_wait();
        }
      }
      l_sum = l_sum * f + rowsum;
      m_used = m_new;

#pragma unroll
      for (int g = 0; g < 16; ++g) {
        // key chunk g/8 (64 keys), 16-byte piece g%8 of row r, swizzled
        *reinterpret_cast<uint4 *>(sP + (g >> 3) * 16384 + r * 128 + (((g & 7) ^ (r & 7)) << 4)) =
            make_uint4(pk[4 * g + 0], pk[4 * g + 1], pk[4 * g + 2], pk[4 * g + 3]);
      }
      // this thread's P writes -> async proxy; then one arrival per warp
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    const int jl = nkv - 1;
    if (ok && mbar_wait_warp(pv_done, static_cast<uint32_t>(jl) & 1, abort_flag)) {
      tc_fence_after();
      const int lq = q0 + r;
      const bool valid = lq < L;
      const float inv = 1.0f / l_sum;
      __nv_bfloat16 *dst = o_out + (static_cast<long>(b) * L + lq) * (static_cast<long>(H) * ATT_DH) +
                           h * ATT_DH;
#pragma unroll 1
      for (int c = 0; c < ATT_DH; c += 32) {
        float o[32];
        tmem_ld32(tmem + lane_base + ATT_TMEM_O + c, o);
        tmem_ld_wait();
        if (!valid) continue;
        uint4 *d = reinterpret_cast<uint4 *>(dst + c);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 w;
          w.x = pack_bf16x2(o[8 * q + 0] * inv, o[8 * q + 1] * inv);
          w.y = pack_bf16x2(o[8 * q + 2] * inv, o[8 * q + 3] * inv);
          w.z = pack_bf16x2(o[8 * q + 4] * inv, o[8 * q + 5] * inv);
          w.w = pack_bf16x2(o[8 * q + 6] * inv, o[8 * q + 7] * inv);
          d[q] = w;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) tmem_dealloc(tmem, ATT_TMEM_COLS);
}

}  // namespace ig4
