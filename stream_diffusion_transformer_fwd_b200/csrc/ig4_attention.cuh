// ig4_attention.cuh - fused flash-style joint attention, head_dim 256, sm_100a.
//
// One CTA computes o for 128 query rows of one (sample, head):
//   S_j = Q K_j^T (tcgen05, fp32 in TMEM, two 64-column buffers),
//   online softmax in registers (one thread per query row, log2 domain),
//   P_j (bf16) written to shared memory in the MMA operand layout,
//   O += P_j V_j (tcgen05, fp32 in TMEM, 256 columns).
// V arrives transposed ([256, keys], keys contiguous) so that every operand
// is K-major with the 128-byte swizzle.  The running maximum used for the
// exponentials is only moved when a row's maximum grows by more than 2^8
// (in exp2 units), so O in TMEM is rescaled rarely; since the same maximum
// is used for the numerator and the denominator the result is unchanged.
//
// Warp roles (192 threads): warps 0-3 softmax + output, warp 4 TMA loads
// (Q once, K_j and V_j through a 2-stage ring), warp 5 TMEM allocation and
// the MMA issue order S_0, S_1, PV_0, S_2, PV_1, ...
#pragma once

#include "ig4_ptx.cuh"

namespace ig4 {

constexpr int ATT_BM = 128;
constexpr int ATT_BN = 64;
constexpr int ATT_DH = 256;
constexpr int ATT_THREADS = 192;
constexpr int ATT_Q_BYTES = ATT_BM * ATT_DH * 2;      // 64 KB: 4 chunks of [128 x 128 B]
constexpr int ATT_K_BYTES = ATT_BN * ATT_DH * 2;      // 32 KB: 4 chunks of [64 x 128 B]
constexpr int ATT_V_BYTES = ATT_DH * ATT_BN * 2;      // 32 KB: [256 x 128 B]
constexpr int ATT_P_BYTES = ATT_BM * ATT_BN * 2;      // 16 KB: [128 x 128 B]
constexpr int ATT_OFF_K = ATT_Q_BYTES;
constexpr int ATT_OFF_V = ATT_OFF_K + 2 * ATT_K_BYTES;
constexpr int ATT_OFF_P = ATT_OFF_V + 2 * ATT_V_BYTES;
constexpr int ATT_OFF_BAR = ATT_OFF_P + ATT_P_BYTES;
constexpr int ATT_SMEM_BYTES = ATT_OFF_BAR + 256 + 1024;
constexpr uint32_t ATT_TMEM_COLS = 512;
constexpr uint32_t ATT_TMEM_O = 256;
// log2(e) / sqrt(256)
constexpr float ATT_SCALE_LOG2 = 0.09016844005556021f;
constexpr float ATT_RESCALE_THRESHOLD = 8.0f;

__global__ void __launch_bounds__(ATT_THREADS, 1)
    attention_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, __nv_bfloat16 *__restrict__ o_out,
                     int L, int H) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sQ = smem;
  uint8_t *sK = smem + ATT_OFF_K;
  uint8_t *sV = smem + ATT_OFF_V;
  uint8_t *sP = smem + ATT_OFF_P;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + ATT_OFF_BAR);
  uint64_t *q_full = bars + 0;
  uint64_t *k_full = bars + 1;   // [2]
  uint64_t *k_empty = bars + 3;  // [2]
  uint64_t *v_full = bars + 5;   // [2]
  uint64_t *v_empty = bars + 7;  // [2]
  uint64_t *s_full = bars + 9;   // [2]
  uint64_t *p_full = bars + 11;
  uint64_t *pv_done = bars + 12;
  uint64_t *drain = bars + 13;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 14);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int q0 = blockIdx.x * ATT_BM;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int bh = b * H + h;
  const int nkv = (L + ATT_BN - 1) / ATT_BN;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
      mbar_init(&s_full[s], 1);
    }
    mbar_init(p_full, 128);
    mbar_init(pv_done, 1);
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
      long issued_k = 0, issued_v = 0;
      bool ok = true;
      mbar_arrive_expect_tx(q_full, ATT_Q_BYTES);
      for (int c = 0; c < 4; ++c) tma_load_3d(sQ + c * (ATT_BM * 128), &tmQ, q_full, c * 64, q0, bh);
      for (int j = 0; j < nkv && ok; ++j) {
        const int s = j & 1;
        const uint32_t ph = static_cast<uint32_t>(j >> 1) & 1;
        if (!mbar_wait(&k_empty[s], ph ^ 1, abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(&k_full[s], ATT_K_BYTES);
        for (int c = 0; c < 4; ++c)
          tma_load_3d(sK + s * ATT_K_BYTES + c * (ATT_BN * 128), &tmK, &k_full[s], c * 64,
                      j * ATT_BN, bh);
        ++issued_k;
        if (!mbar_wait(&v_empty[s], ph ^ 1, abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(&v_full[s], ATT_V_BYTES);
        tma_load_3d(sV + s * ATT_V_BYTES, &tmV, &v_full[s], j * ATT_BN, 0, bh);
        ++issued_v;
      }
      if (!ok) {
        mbar_wait(q_full, 0, nullptr, WAIT_LIMIT_NS / 4);
        for (long i = (issued_k > 2 ? issued_k - 2 : 0); i < issued_k; ++i)
          mbar_wait(&k_full[i & 1], static_cast<uint32_t>(i >> 1) & 1, nullptr, WAIT_LIMIT_NS / 4);
        for (long i = (issued_v > 2 ? issued_v - 2 : 0); i < issued_v; ++i)
          mbar_wait(&v_full[i & 1], static_cast<uint32_t>(i >> 1) & 1, nullptr, WAIT_LIMIT_NS / 4);
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      constexpr uint32_t IDESC_S = idesc_bf16(ATT_BM, ATT_BN);
      constexpr uint32_t IDESC_PV = idesc_bf16(ATT_BM, ATT_DH);
      const uint32_t q_base = smem_u32(sQ);
      const uint32_t p_base = smem_u32(sP);
      bool ok = mbar_wait(q_full, 0, abort_flag);
      auto issue_s = [&](int j) -> bool {
        const int s = j & 1;
        const uint32_t ph = static_cast<uint32_t>(j >> 1) & 1;
        if (!mbar_wait(&k_full[s], ph, abort_flag)) return false;
        tc_fence_after();
        const uint32_t k_base = smem_u32(sK + s * ATT_K_BYTES);
#pragma unroll
        for (int kk = 0; kk < ATT_DH / 16; ++kk) {
          const uint64_t ad = sdesc_kmajor_sw128(q_base + (kk >> 2) * (ATT_BM * 128) + (kk & 3) * 32);
          const uint64_t bd = sdesc_kmajor_sw128(k_base + (kk >> 2) * (ATT_BN * 128) + (kk & 3) * 32);
          umma_bf16(tmem + s * ATT_BN, ad, bd, IDESC_S, kk > 0);
        }
        umma_commit(&k_empty[s]);
        umma_commit(&s_full[s]);
        return true;
      };
      if (ok) ok = issue_s(0);
      if (ok && nkv > 1) ok = issue_s(1);
      for (int j = 0; j < nkv && ok; ++j) {
        const int s = j & 1;
        const uint32_t ph = static_cast<uint32_t>(j >> 1) & 1;
        if (!mbar_wait(p_full, static_cast<uint32_t>(j) & 1, abort_flag)) break;
        if (!mbar_wait(&v_full[s], ph, abort_flag)) break;
        tc_fence_after();
        const uint32_t v_base = smem_u32(sV + s * ATT_V_BYTES);
#pragma unroll
        for (int kk = 0; kk < ATT_BN / 16; ++kk) {
          const uint64_t ad = sdesc_kmajor_sw128(p_base + kk * 32);
          const uint64_t bd = sdesc_kmajor_sw128(v_base + kk * 32);
          umma_bf16(tmem + ATT_TMEM_O, ad, bd, IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&v_empty[s]);
        umma_commit(pv_done);
        if (j + 2 < nkv) ok = issue_s(j + 2);
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
    bool ok = true;
    uint8_t *prow = sP + r * 128;
    for (int j = 0; j < nkv; ++j) {
      const int s = j & 1;
      const uint32_t ph = static_cast<uint32_t>(j >> 1) & 1;
      if (!mbar_wait_warp(&s_full[s], ph, abort_flag)) { ok = false; break; }
      tc_fence_after();
      float t[64];
      {
        float a[32], c[32];
        tmem_ld32(tmem + lane_base + s * ATT_BN, a);
        tmem_ld32(tmem + lane_base + s * ATT_BN + 32, c);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          t[i] = a[i] * ATT_SCALE_LOG2;
          t[32 + i] = c[i] * ATT_SCALE_LOG2;
        }
      }
      const int kbase = j * ATT_BN;
      if (kbase + ATT_BN > L) {
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (kbase + i >= L) t[i] = -INFINITY;
      }
      float mx = t[0];
#pragma unroll
      for (int i = 1; i < 64; ++i) mx = fmaxf(mx, t[i]);

      if (j > 0) {
        // PV_{j-1} must be done: it reads P (single buffer) and writes O.
        if (!mbar_wait_warp(pv_done, static_cast<uint32_t>(j - 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const bool need = mx > m_used + ATT_RESCALE_THRESHOLD;
        if (__any_sync(0xffffffffu, need)) {
          const float f = need ? exp2_approx(m_used - mx) : 1.0f;
          if (need) m_used = mx;
          l_sum *= f;
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
      } else {
        m_used = mx;
      }

      float rowsum = 0.0f;
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        float p[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          p[e] = exp2_approx(t[8 * g + e] - m_used);
          rowsum += p[e];
        }
        uint4 w;
        w.x = pack_bf16x2(p[0], p[1]);
        w.y = pack_bf16x2(p[2], p[3]);
        w.z = pack_bf16x2(p[4], p[5]);
        w.w = pack_bf16x2(p[6], p[7]);
        *reinterpret_cast<uint4 *>(prow + ((g ^ (r & 7)) << 4)) = w;
      }
      l_sum += rowsum;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    if (ok && mbar_wait_warp(pv_done, static_cast<uint32_t>(nkv - 1) & 1, abort_flag)) {
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
