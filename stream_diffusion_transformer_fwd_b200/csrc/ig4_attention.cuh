// ig4_attention.cuh - fused flash-style joint attention, head_dim 256, sm_100a.
//
// One CTA computes o for 128 query rows of one (sample, head), walking the
// keys in tiles of 128:
//   S_j = Q K_j^T     16 tcgen05.mma (M=128, N=128, K=16), Q and K_j from
//                     shared memory, fp32 scores into TMEM;
//   softmax           one thread per query row, exp2 domain, in registers;
//   P_j               bf16, written into TMEM (tcgen05.st), two buffers;
//   O += P_j V_j      8 tcgen05.mma (M=128, N=256, K=16) with A = P_j read
//                     from TMEM and B = V_j from shared memory; O (fp32) in TMEM.
// 128-key tiles keep every MMA at N >= 128, the width at which an MMA runs at
// the full tensor rate.
//
// TMEM (512 columns): S [0,128), P_0 [128,192), P_1 [192,256) (bf16 pairs),
// O [256,512).  With two P buffers the softmax of tile j never waits for
// PV_{j-1}: it only needs PV_{j-2} (long done) before it overwrites P_{j%2},
// and PV_{j-1} only when it has to rescale O.
//
// Shared memory: Q (64 KB, loaded once) and a ring of five 32 KB slots that
// TMA fills with half tiles in the order the MMAs consume them - K_0, K_1,
// V_0, K_2, V_1, K_3, V_2, ... - each split in two halves (K: head dims
// [0,128) and [128,256); V: keys [0,64) and [64,128)), so a slot is released
// as soon as the MMAs of its half have run.  V arrives transposed ([256,
// keys], keys contiguous), so every shared-memory operand is K-major with the
// 128-byte swizzle.
//
// The running maximum used for the exponentials only moves when a row's
// maximum grows by more than 8 (a factor 2^8), so O is rescaled rarely;
// numerator and denominator use the same maximum, so the result is unchanged.
//
// Warp roles (224 threads): warps 0-3 softmax + output (warp w owns TMEM
// lanes / query rows 32w..32w+31), warp 4 TMA producer, warp 5 TMEM
// allocation and the S MMAs, warp 6 the PV MMAs.  The two MMA threads wait
// on different events (scores read out vs. probabilities written), so one
// keeps the tensor pipe fed while the other waits.
//
// Barrier parity: every barrier a role waits on completes at most one phase
// ahead of that wait, so try_wait.parity never mistakes a later phase for the
// awaited one (this is why P-ready and PV-done exist once per P buffer).
// Every wait is bounded.
#pragma once

#include "ig4_ptx.cuh"

namespace ig4 {

constexpr int ATT_BM = 128;
constexpr int ATT_BN = 128;   // keys per tile
constexpr int ATT_DH = 256;
constexpr int ATT_THREADS = 224;
constexpr int ATT_SLOTS = 5;
constexpr int ATT_SLOT_BYTES = 32768;  // K half: 2 chunks [128 keys x 128 B]; V half: [256 x 128 B]
constexpr int ATT_Q_BYTES = 65536;     // 4 chunks [128 rows x 128 B]
constexpr int ATT_OFF_RING = ATT_Q_BYTES;
constexpr int ATT_OFF_BAR = ATT_OFF_RING + ATT_SLOTS * ATT_SLOT_BYTES;
constexpr int ATT_SMEM_BYTES = ATT_OFF_BAR + 256 + 1024;
constexpr uint32_t ATT_TMEM_COLS = 512;
constexpr uint32_t ATT_TMEM_S = 0;
constexpr uint32_t ATT_TMEM_P = 128;  // + 64 * buffer
constexpr uint32_t ATT_TMEM_O = 256;
// log2(e) / sqrt(256)
constexpr float ATT_SCALE_LOG2 = 0.09016844005556021f;
constexpr float ATT_RESCALE_THRESHOLD = 8.0f;

// The order in which the ring receives whole tiles ("items"): K_0; K_1 (if
// any); then, for each tile j, V_j followed by K_{j+2} (if that tile
// exists).  Each item travels as two 32 KB halves.
struct AttRing {
  int nkv;
  __device__ __forceinline__ int items() const { return 2 * nkv; }
  // kind of item u: 1 = K, 2 = V, with the tile index in *tile
  __device__ __forceinline__ int kind(int u, int *tile) const {
    if (u == 0) { *tile = 0; return 1; }
    if (nkv == 1) { *tile = 0; return 2; }  // items: K_0, V_0
    if (u == 1) { *tile = 1; return 1; }
    // items from 2 on: V_0, K_2, V_1, K_3, ..., V_{nkv-3}, K_{nkv-1}, V_{nkv-2}, V_{nkv-1}
    const int k = u - 2;
    const int pairs = nkv - 2;  // (V_j, K_{j+2}) for j < nkv - 2
    if (k < 2 * pairs) {
      *tile = (k & 1) ? (k >> 1) + 2 : (k >> 1);
      return (k & 1) ? 1 : 2;
    }
    *tile = (nkv - 2) + (k - 2 * pairs);
    return 2;
  }
  // the item that carries K_t, and the one that carries V_t
  __device__ __forceinline__ int item_k(int t) const { return t < 2 ? t : 2 * t - 1; }
  __device__ __forceinline__ int item_v(int t) const { return min(2 * t + 2, 2 * nkv - 1); }
};

__global__ void __launch_bounds__(ATT_THREADS, 1)
    attention_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, __nv_bfloat16 *__restrict__ o_out,
                     int L, int H) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *ring = smem + ATT_OFF_RING;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + ATT_OFF_BAR);
  uint64_t *full = bars + 0;      // [ATT_SLOTS]
  uint64_t *empty = bars + 5;     // [ATT_SLOTS]
  uint64_t *q_full = bars + 10;   // Q landed
  uint64_t *s_full = bars + 11;   // S_j in TMEM
  uint64_t *s_free = bars + 12;   // S_j read out of TMEM (one arrival per softmax warp)
  uint64_t *p_full = bars + 13;   // [2] P_j in TMEM buffer j%2 (one arrival per softmax warp)
  uint64_t *pv_done = bars + 15;  // [2] PV_j complete (buffer j%2)
  uint64_t *drain_s = bars + 17;
  uint64_t *drain_pv = bars + 18;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 20);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int q0 = blockIdx.x * ATT_BM;
  const int h = blockIdx.y;
  const int b = blockIdx.z;
  const int bh = b * H + h;
  const int nkv = (L + ATT_BN - 1) / ATT_BN;
  const AttRing ring_order{nkv};

  if (threadIdx.x == 0) {
    for (int s = 0; s < ATT_SLOTS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(s_full, 1);
    mbar_init(s_free, 4);
    mbar_init(&p_full[0], 4);
    mbar_init(&p_full[1], 4);
    mbar_init(&pv_done[0], 1);
    mbar_init(&pv_done[1], 1);
    mbar_init(drain_s, 1);
    mbar_init(drain_pv, 1);
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
  pdl_wait();
  pdl_trigger();

  if (warp == 4) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      mbar_arrive_expect_tx(q_full, ATT_Q_BYTES);
      for (int c = 0; c < 4; ++c) tma_load_3d(smem + c * 16384, &tmQ, q_full, c * 64, q0, bh);
      const int n = 2 * ring_order.items();  // half items
      int i = 0;
      bool ok = true;
      for (; i < n; ++i) {
        const int slot = i % ATT_SLOTS;
        const uint32_t ph = static_cast<uint32_t>(i / ATT_SLOTS) & 1;
        if (!mbar_wait(&empty[slot], ph ^ 1, abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(&full[slot], ATT_SLOT_BYTES);
        uint8_t *dst = ring + slot * ATT_SLOT_BYTES;
        const int half = i & 1;
        int t = 0;
        if (ring_order.kind(i >> 1, &t) == 1) {
          for (int c = 0; c < 2; ++c)
            tma_load_3d(dst + c * 16384, &tmK, &full[slot], (2 * half + c) * 64, t * ATT_BN, bh);
        } else {
          tma_load_3d(dst, &tmV, &full[slot], t * ATT_BN + half * 64, 0, bh);
        }
      }
      if (!ok) {
        // let the loads already issued land before the shared memory goes away
        mbar_wait(q_full, 0, nullptr, WAIT_LIMIT_NS / 4);
        for (int k = (i > ATT_SLOTS ? i - ATT_SLOTS : 0); k < i; ++k)
          mbar_wait(&full[k % ATT_SLOTS], static_cast<uint32_t>(k / ATT_SLOTS) & 1, nullptr,
                    WAIT_LIMIT_NS / 4);
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      // ------------------------------------------------ S issuer: S_t = Q K_t^T
      constexpr uint32_t IDESC_S = idesc_bf16(ATT_BM, ATT_BN);
      const uint32_t q_base = smem_u32(smem);
      bool ok = mbar_wait(q_full, 0, abort_flag);
      for (int t = 0; t < nkv && ok; ++t) {
        // the S buffer is free once the softmax has read S_{t-1}
        if (t > 0 && !mbar_wait(s_free, static_cast<uint32_t>(t - 1) & 1, abort_flag)) break;
        const int u = ring_order.item_k(t);
        for (int half = 0; half < 2 && ok; ++half) {
          const int i = 2 * u + half;
          const int slot = i % ATT_SLOTS;
          if (!mbar_wait(&full[slot], static_cast<uint32_t>(i / ATT_SLOTS) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t k_base = smem_u32(ring + slot * ATT_SLOT_BYTES);
#pragma unroll
          for (int kq = 0; kq < 8; ++kq) {
            const int kk = half * 8 + kq;  // K step of 16 head dims
            const uint64_t ad = sdesc_kmajor_sw128(q_base + (kk >> 2) * 16384 + (kk & 3) * 32);
            const uint64_t bd = sdesc_kmajor_sw128(k_base + (kq >> 2) * 16384 + (kq & 3) * 32);
            umma_bf16(tmem + ATT_TMEM_S, ad, bd, IDESC_S, kk > 0 ? 1u : 0u);
          }
          umma_commit(&empty[slot]);
        }
        if (ok) umma_commit(s_full);
      }
      umma_commit(drain_s);
      mbar_wait(drain_s, 0, nullptr, WAIT_LIMIT_NS / 4);
    }
  } else if (warp == 6) {
    if (lane == 0) {
      // ------------------------------------------------ PV issuer: O += P_j V_j
      constexpr uint32_t IDESC_PV = idesc_bf16(ATT_BM, ATT_DH);
      bool ok = true;
      for (int j = 0; j < nkv && ok; ++j) {
        const int pb = j & 1;
        if (!mbar_wait(&p_full[pb], static_cast<uint32_t>(j >> 1) & 1, abort_flag)) break;
        tc_fence_after();
        const int u = ring_order.item_v(j);
        for (int half = 0; half < 2 && ok; ++half) {
          const int i = 2 * u + half;
          const int slot = i % ATT_SLOTS;
          if (!mbar_wait(&full[slot], static_cast<uint32_t>(i / ATT_SLOTS) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t v_base = smem_u32(ring + slot * ATT_SLOT_BYTES);
#pragma unroll
          for (int kq = 0; kq < 4; ++kq) {
            const int kk = half * 4 + kq;  // K step of 16 keys
            const uint64_t bd = sdesc_kmajor_sw128(v_base + kq * 32);
            umma_bf16_ts(tmem + ATT_TMEM_O, tmem + ATT_TMEM_P + 64 * pb + kk * 8, bd, IDESC_PV,
                         (j > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&empty[slot]);
        }
        if (ok) umma_commit(&pv_done[pb]);
      }
      umma_commit(drain_pv);
      mbar_wait(drain_pv, 0, nullptr, WAIT_LIMIT_NS / 4);
    }
  } else {
    // -------------------------------------------- softmax warps 0..3
    const int r = warp * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    float m_used = -INFINITY;
    float l_sum = 0.0f;
    bool ok = true;
    const uint64_t scale2 = f2_pack(ATT_SCALE_LOG2, ATT_SCALE_LOG2);

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
      float m4[4] = {t[0], t[1], t[2], t[3]};
#pragma unroll
      for (int i = 4; i < 128; i += 8) {
        m4[0] = fmax3(m4[0], t[i + 0], t[i + 1]);
        m4[1] = fmax3(m4[1], t[i + 2], t[i + 3]);
        m4[2] = fmax3(m4[2], t[i + 4], t[i + 5]);
        m4[3] = fmax3(m4[3], t[i + 6], t[i + 7]);
      }
      const float mx = fmax3(m4[0], m4[1], fmaxf(m4[2], m4[3])) * ATT_SCALE_LOG2;

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

      // p = 2^(s * scale - m), packed to bf16 pairs; row sum in fp32 pairs
      const uint64_t negm2 = f2_pack(-m_new, -m_new);
      uint32_t pk[64];
      uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        const uint64_t x2 = ffma2(f2_pack(t[2 * i], t[2 * i + 1]), scale2, negm2);
        const float p0 = exp2_approx(f2_lo(x2));
        const float p1 = exp2_approx(f2_hi(x2));
        const uint64_t p2 = f2_pack(p0, p1);
        acc[i & 3] = fadd2(acc[i & 3], p2);
        pk[i] = pack_bf16x2(p0, p1);
      }
      const uint64_t s2 = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
      const float rowsum = f2_lo(s2) + f2_hi(s2);

      const int pb = j & 1;
      if (j >= 2) {
        // PV_{j-2} read this P buffer
        if (!mbar_wait_warp(&pv_done[pb], static_cast<uint32_t>((j >> 1) - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
      }
      if (any_need) {
        // PV_{j-1} must be done: it writes O
        if (!mbar_wait_warp(&pv_done[pb ^ 1], static_cast<uint32_t>((j - 1) >> 1) & 1,
                            abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < ATT_DH; c += 32) {
          float o[32];
          tmem_ld32(tmem + lane_base + ATT_TMEM_O + c, o);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= f;
          tmem_st32(tmem + lane_base + ATT_TMEM_O + c, o);
        }
      }
      tc_fence_after();
      {
        uint32_t w[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) w[i] = pk[i];
        tmem_st32_u(tmem + lane_base + ATT_TMEM_P + 64 * pb, w);
#pragma unroll
        for (int i = 0; i < 32; ++i) w[i] = pk[32 + i];
        tmem_st32_u(tmem + lane_base + ATT_TMEM_P + 64 * pb + 32, w);
      }
      tmem_st_wait();
      l_sum = l_sum * f + rowsum;
      m_used = m_new;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[pb]);
    }
    const int jl = nkv - 1;
    if (ok && mbar_wait_warp(&pv_done[jl & 1], static_cast<uint32_t>(jl >> 1) & 1, abort_flag)) {
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
