// ig4_attention.cuh - fused flash-style joint attention, head_dim 256, sm_100a.
//
// Work: for every (sample, head) and every 128-row query tile (an "item"),
// the 128-key tiles of the whole sequence.  A persistent grid of G CTAs (one
// per SM) takes the items round-robin, whole: in round r CTA c takes item
// r G + c, so the CTAs running at the same time share the K and V of a few
// heads through L2.  The rem items of the last, partial round are split
// into k = min(key tiles, G / rem) pieces of consecutive key tiles, piece p
// of tail item j on CTA j k + p, so the last round keeps the SMs busy too.
// A piece stores its unnormalised O (bf16), row maximum m and row sum l into
// a partial slot, and attention_combine_kernel merges the pieces of each tail
// item afterwards, in piece order (deterministic).  With fewer items than
// SMs (or no workspace for partial slots) every CTA takes one whole item.
//
// Per key tile of a segment:
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
// Shared memory: Q (64 KB) and a ring of five 32 KB slots that TMA fills with
// half tiles in the order the MMAs consume them - per segment K_0, K_1, V_0,
// K_2, V_1, K_3, V_2, ... - each split in two halves (K: head dims [0,128)
// and [128,256); V: keys [0,64) and [64,128)), so a slot is released as soon
// as the MMAs of its half have run.  V arrives transposed ([256, keys], keys
// contiguous), so every shared-memory operand is K-major with the 128-byte
// swizzle.  Across segments the pipeline keeps running: the producer loads
// the next segment's Q as soon as the last S MMA of the current one has read
// Q, the next segment's S MMAs run while the softmax warps drain O, and the
// next segment's first PV waits only for that drain.
//
// The running maximum used for the exponentials only moves when a row's
// maximum grows by more than 8 (a factor 2^8), so O is rescaled rarely;
// numerator and denominator use the same maximum, so the result is unchanged.
//
// CTA pairs.  With two or more query tiles the kernel runs on 2-CTA
// clusters (tcgen05.mma.cta_group::2, M = 256): an item is then two query
// tiles of one (sample, head), rank r of the pair holding query tile
// 2 u + r (an odd count leaves rank 1 of the last item a tile past the
// sequence, computed on zero-filled Q and not stored).  Each CTA keeps its
// own 128 query rows, S, P and O in its own TMEM, and loads only HALF of
// every key tile: K of its 64 keys (4 chunks [64 keys x 128 B]) and V^T of
// its 128 head dims (2 chunks [128 dims x 128 B]), 32 KB each, one ring slot
// per K or V item.  The leader issues S_j = Q K_j^T as 16 MMAs of N = 128
// and O += P_j V_j as 8 MMAs of N = 256 with A = P read from both CTAs'
// TMEM.  So per key tile each SM moves 64 KB of K and V instead of 128 KB
// (the single-CTA kernel's L2 traffic starves the ring), and the ring holds
// two and a half tiles instead of one and a quarter.  Both CTAs' loads
// complete on the leader's full barriers (the leader posts the bytes of
// both); the leader's commits arrive on both CTAs' empty / S-ready / PV-done
// barriers; the softmax warps of both CTAs arrive on the leader's S-free,
// P-ready and O-free barriers (8 arrivals).
//
// Warp roles (224 threads): warps 0-3 softmax + output (warp w owns TMEM
// lanes / query rows 32w..32w+31), warp 4 TMA producer, warp 5 TMEM
// allocation and the S MMAs, warp 6 the PV MMAs (the MMA roles only in the
// leader of a pair).  The two MMA threads wait
// on different events (scores read out vs. probabilities written), so one
// keeps the tensor pipe fed while the other waits.
//
// Barrier parity: try_wait.parity only tells the awaited phase from the one
// before it, so every wait must start when the barrier is at most one phase
// ahead of, and not behind, the awaited phase (this is why P-ready and
// PV-done exist once per P buffer).  The ring's full barriers have two
// consumers (K halves for the S issuer, V halves for the PV issuer) and TMA
// loads may land out of order, so one consumer could otherwise start waiting
// for half h while the load of half h - 5 into the same slot (for the other
// consumer) is still in flight, and take the completed phase of half h - 10
// for the one it awaits.  The producer therefore publishes in shared memory
// how many halves it has passed its empty wait for; a consumer waits for
// that count to exceed h before it waits on full: the slot's previous phase
// has then completed.  Phases count tiles (and segments) over the whole
// range.  Every wait is bounded.
#pragma once

#include "ig4_mx8.cuh"
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
// The largest persistent grid (one partial slot per CTA is reserved).
constexpr int ATT_MAX_CTAS = 160;
// A partial slot: unnormalised O bf16 [128][256], then m and l fp32 [128] each.
constexpr long ATT_PART_O_BYTES = static_cast<long>(ATT_BM) * ATT_DH * 2;
constexpr long ATT_PART_BYTES = ATT_PART_O_BYTES + 2L * ATT_BM * 4;

// The order in which the ring receives a segment's whole tiles ("items"):
// K_0; K_1 (if any); then, for each tile j, V_j followed by K_{j+2} (if that
// tile exists).  Tile indices are relative to the segment.  Each item
// travels as two 32 KB halves.
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

// One segment of a CTA's work: key tiles [t0, t0 + n) of item `item`;
// `slot` is the partial slot of a tail piece (-1 for a whole item).
struct AttSeg {
  int item, t0, n, slot;
};

// The persistent grid's schedule (computed the same way by the host).
struct AttSched {
  int n_items, G, nkv;
  int rounds;  // whole rounds: items [0, rounds * G)
  int rem;     // items of the last, partial round
  int k;       // pieces per tail item (1: tail items run whole)
  __device__ __forceinline__ AttSched(int n_items_, int G_, int nkv_)
      : n_items(n_items_), G(G_), nkv(nkv_) {
    rounds = n_items / G;
    rem = n_items - rounds * G;
    k = rem > 0 ? max(1, min(nkv, G / rem)) : 1;
  }
  __device__ __forceinline__ int segments(int c) const { return rounds + (c < rem * k ? 1 : 0); }
  __device__ __forceinline__ AttSeg seg(int c, int s) const {
    if (s < rounds) return AttSeg{s * G + c, 0, nkv, -1};
    const int j = c / k, p = c - j * k;
    const int t0 = p * nkv / k, t1 = (p + 1) * nkv / k;
    return AttSeg{rounds * G + j, t0, t1 - t0, k > 1 ? c : -1};
  }
  // key tiles of the CTA's segments before segment s (every earlier one is whole)
  __device__ __forceinline__ long tiles_before(int s) const {
    return static_cast<long>(min(s, rounds)) * nkv;
  }
};

// Wait (bounded, like mbar_wait) until the producer has passed its empty
// wait for half h of the ring, i.e. *passed > h.
__device__ __forceinline__ bool att_wait_passed(const volatile int *passed, long h,
                                                volatile int *abort_flag) {
  if (*passed > h) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 8; ++i) {
      if (*passed > h) return true;
      __nanosleep(32);  // leave the issue slots to the softmax warp of this SMSP
    }
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > WAIT_LIMIT_NS) {
      atomicOr(&g_device_error, DEVERR_TIMEOUT);
      *abort_flag = 1;
      return false;
    }
  }
}

// Waits and arrivals of the pipeline.  In a pair the hand-offs between the
// CTAs carry no data through ordinary memory (only tensor memory, ordered by
// the tcgen05 fences around them), so they keep the CTA-scope semantics.
template <bool PAIR>
__device__ __forceinline__ bool att_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                         unsigned long long limit_ns = WAIT_LIMIT_NS) {
  return mbar_wait(bar, parity, abort_flag, limit_ns);
}

template <bool PAIR>
__device__ __forceinline__ bool att_wait_warp(uint64_t *bar, uint32_t parity,
                                              volatile int *abort_flag) {
  return __all_sync(0xffffffffu, att_wait<PAIR>(bar, parity, abort_flag));
}

// Commit of the MMAs issued so far to a barrier (in both CTAs of a pair).
template <bool PAIR>
__device__ __forceinline__ void att_commit(uint64_t *bar) {
  if constexpr (PAIR)
    umma_commit_pair_both(bar);
  else
    umma_commit(bar);
}

// 32-byte global store (sm_100 and later; the address 32-byte aligned).  A
// softmax thread writes its own output row, rows H * 512 bytes apart, so a
// warp's store touches 32 lines: 32-byte pieces halve the store instructions
// and write whole sectors.
__device__ __forceinline__ void st_global_v8(void *p, const uint32_t (&w)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(w[0]),
               "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}

// Arrive on a barrier that the leader CTA holds (the CTA itself when single).
template <bool PAIR>
__device__ __forceinline__ void att_arrive_leader(uint64_t *bar) {
  if constexpr (PAIR)
    mbar_arrive_remote(map_shared_to_rank(bar, 0));
  else
    mbar_arrive(bar);
}

template <bool PAIR>
__global__ void __launch_bounds__(ATT_THREADS, 1)
    attention_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, __nv_bfloat16 *__restrict__ o_out,
                     int L, int H, int n_bh, uint8_t *__restrict__ part,
                     uint8_t *__restrict__ o_sf) {
  constexpr int CTAS = PAIR ? 2 : 1;
  constexpr int UPI = PAIR ? 1 : 2;  // ring units (slots) per item
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *ring = smem + ATT_OFF_RING;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + ATT_OFF_BAR);
  uint64_t *full = bars + 0;      // [ATT_SLOTS]
  uint64_t *empty = bars + 5;     // [ATT_SLOTS]
  uint64_t *q_full = bars + 10;   // Q of a segment landed
  uint64_t *s_full = bars + 11;   // S_j in TMEM
  uint64_t *s_free = bars + 12;   // S_j read out of TMEM (one arrival per softmax warp)
  uint64_t *p_full = bars + 13;   // [2] P_j in TMEM buffer j%2 (one arrival per softmax warp)
  uint64_t *pv_done = bars + 15;  // [2] PV_j complete (buffer j%2)
  uint64_t *drain_s = bars + 17;
  uint64_t *drain_pv = bars + 18;
  uint64_t *q_empty = bars + 19;  // the last S MMA of a segment has read Q
  uint64_t *o_free = bars + 20;   // O of a segment drained (one arrival per softmax warp)
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 22);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  volatile int *passed = reinterpret_cast<volatile int *>(tmem_slot + 2);  // ring units past empty

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rank = PAIR ? static_cast<int>(cluster_ctarank()) : 0;
  const bool leader = rank == 0;
  const int nkv = (L + ATT_BN - 1) / ATT_BN;          // key tiles = query tiles
  const int n_units = PAIR ? (nkv + 1) / 2 : nkv;     // items per (sample, head)
  const AttSched sched(n_bh * n_units, static_cast<int>(gridDim.x) / CTAS, nkv);
  const int worker = blockIdx.x / CTAS;
  const int n_seg = sched.segments(worker);

  if (threadIdx.x == 0) {
    for (int s = 0; s < ATT_SLOTS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(s_full, 1);
    mbar_init(s_free, 4 * CTAS);
    mbar_init(&p_full[0], 4 * CTAS);
    mbar_init(&p_full[1], 4 * CTAS);
    mbar_init(&pv_done[0], 1);
    mbar_init(&pv_done[1], 1);
    mbar_init(drain_s, 1);
    mbar_init(drain_pv, 1);
    mbar_init(q_empty, 1);
    mbar_init(o_free, 4 * CTAS);
    *abort_flag = 0;
    *passed = 0;
    fence_mbar_init();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 5) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, ATT_TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, ATT_TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if constexpr (PAIR)
    cluster_sync_all();
  else
    __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();
  pdl_trigger();

  if (warp == 4) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer (each CTA its own part)
      long i = 0;  // ring units issued over the range
      bool ok = true;
      int k = 0;
      int q_issued = -1;  // the last segment whose Q load was issued
      for (; k < n_seg && ok; ++k) {
        const AttSeg sg = sched.seg(worker, k);
        const int bh = sg.item / n_units;
        const int q0 = ((sg.item - bh * n_units) * CTAS + rank) * ATT_BM;
        // Q: free once the last S MMA of the previous segment has run
        if (k > 0 && !att_wait<PAIR>(q_empty, static_cast<uint32_t>(k - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        if (leader) mbar_arrive_expect_tx(q_full, CTAS * ATT_Q_BYTES);
        for (int c = 0; c < 4; ++c) {
          if constexpr (PAIR)
            tma_load_3d_pair(smem + c * 16384, &tmQ, map_shared_to_rank(q_full, 0), c * 64, q0, bh);
          else
            tma_load_3d(smem + c * 16384, &tmQ, q_full, c * 64, q0, bh);
        }
        q_issued = k;
        const AttRing ro{sg.n};
        const int n = UPI * ro.items();  // ring units of this segment
        for (int hi = 0; hi < n; ++hi, ++i) {
          const int slot = static_cast<int>(i % ATT_SLOTS);
          const uint32_t ph = static_cast<uint32_t>(i / ATT_SLOTS) & 1;
          if (!att_wait<PAIR>(&empty[slot], ph ^ 1, abort_flag)) { ok = false; break; }
          if (leader) {
            // unit i - 5 is consumed, so full[slot] has completed its phase
            __threadfence_block();
            *passed = static_cast<int>(i + 1);
            mbar_arrive_expect_tx(&full[slot], CTAS * ATT_SLOT_BYTES);
          }
          uint8_t *dst = ring + slot * ATT_SLOT_BYTES;
          int t = 0;
          const int kind = ro.kind(hi / UPI, &t);
          const int key0 = (sg.t0 + t) * ATT_BN;
          if constexpr (PAIR) {
            // this CTA's half of the pair's tile: keys [64 rank, +64) of K,
            // head dims [128 rank, +128) of V^T
            const uint32_t fb = map_shared_to_rank(&full[slot], 0);
            if (kind == 1) {
              for (int c = 0; c < 4; ++c)
                tma_load_3d_pair(dst + c * 8192, &tmK, fb, c * 64, key0 + 64 * rank, bh);
            } else {
              for (int c = 0; c < 2; ++c)
                tma_load_3d_pair(dst + c * 16384, &tmV, fb, key0 + 64 * c, 128 * rank, bh);
            }
          } else {
            const int half = hi & 1;
            if (kind == 1) {
              for (int c = 0; c < 2; ++c)
                tma_load_3d(dst + c * 16384, &tmK, &full[slot], (2 * half + c) * 64, key0, bh);
            } else {
              tma_load_3d(dst, &tmV, &full[slot], key0 + half * 64, 0, bh);
            }
          }
        }
      }
      if (!ok) {
        // let the loads already issued land before the shared memory goes away
        if constexpr (PAIR) {
          // (a pair's loads complete on the leader's barriers)
          sleep_ns(50000);
        } else {
          if (q_issued >= 0)
            mbar_wait(q_full, static_cast<uint32_t>(q_issued) & 1, nullptr, WAIT_LIMIT_NS / 4);
          for (long j = (i > ATT_SLOTS ? i - ATT_SLOTS : 0); j < i; ++j)
            mbar_wait(&full[j % ATT_SLOTS], static_cast<uint32_t>(j / ATT_SLOTS) & 1, nullptr,
                      WAIT_LIMIT_NS / 4);
        }
      }
    }
  } else if (warp == 5) {
    if (lane == 0 && leader) {
      // ------------------------------------------------ S issuer: S_t = Q K_t^T
      constexpr uint32_t IDESC_S = idesc_bf16(CTAS * ATT_BM, ATT_BN);
      const uint64_t qd = sdesc_kmajor_sw128(smem_u32(smem));
      bool ok = true;
      long gt = 0;  // tiles over the CTA's segments
      for (int k = 0; k < n_seg && ok; ++k) {
        const AttSeg sg = sched.seg(worker, k);
        const AttRing ro{sg.n};
        const long ibase = 2 * UPI * sched.tiles_before(k);  // ring units before this segment
        if (!att_wait<PAIR>(q_full, static_cast<uint32_t>(k) & 1, abort_flag)) break;
        for (int t = 0; t < sg.n && ok; ++t, ++gt) {
          const int it = ro.item_k(t);
          // K_t resident first: its slot checks then stay off the path from the
          // softmax's release of S to the next S MMA (K_t's load waits only on
          // items consumed before it, so this order adds no dependency)
          for (int u = 0; u < UPI && ok; ++u) {
            const long i = ibase + UPI * it + u;
            ok = att_wait_passed(passed, i, abort_flag) &&
                 att_wait<PAIR>(&full[i % ATT_SLOTS], static_cast<uint32_t>(i / ATT_SLOTS) & 1,
                                abort_flag);
          }
          // the S buffer is free once the softmax has read S_{gt-1}
          if (!ok ||
              (gt > 0 && !att_wait<PAIR>(s_free, static_cast<uint32_t>(gt - 1) & 1, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
          for (int u = 0; u < UPI; ++u) {
            const long i = ibase + UPI * it + u;
            const int slot = static_cast<int>(i % ATT_SLOTS);
            // descriptors of the slot's and Q's first chunk; a K step adds its
            // byte offset / 16 to the start-address field (no carry out of it:
            // shared memory addresses stay below 2^18)
            const uint64_t kd = sdesc_kmajor_sw128(smem_u32(ring + slot * ATT_SLOT_BYTES));
            if constexpr (PAIR) {
              // 64 keys x 256 head dims in each CTA: 4 chunks [64 keys x 128 B]
#pragma unroll
              for (int kk = 0; kk < 16; ++kk)
                umma_bf16_pair(tmem + ATT_TMEM_S, qd + ((kk >> 2) * 16384 + (kk & 3) * 32) / 16,
                               kd + ((kk >> 2) * 8192 + (kk & 3) * 32) / 16, IDESC_S,
                               kk > 0 ? 1u : 0u);
            } else {
#pragma unroll
              for (int kq = 0; kq < 8; ++kq) {
                const int kk = u * 8 + kq;  // K step of 16 head dims
                umma_bf16(tmem + ATT_TMEM_S, qd + ((kk >> 2) * 16384 + (kk & 3) * 32) / 16,
                          kd + ((kq >> 2) * 16384 + (kq & 3) * 32) / 16, IDESC_S,
                          kk > 0 ? 1u : 0u);
              }
            }
            att_commit<PAIR>(&empty[slot]);
          }
          if (ok) att_commit<PAIR>(s_full);
        }
        // Q may be replaced once these MMAs have run
        if (ok) att_commit<PAIR>(q_empty);
      }
      att_commit<PAIR>(drain_s);
      att_wait<PAIR>(drain_s, 0, nullptr, WAIT_LIMIT_NS / 4);
    }
  } else if (warp == 6) {
    if (lane == 0 && leader) {
      // ------------------------------------------------ PV issuer: O += P_j V_j
      constexpr uint32_t IDESC_PV = idesc_bf16(CTAS * ATT_BM, ATT_DH);
      bool ok = true;
      long gt = 0;
      for (int k = 0; k < n_seg && ok; ++k) {
        const AttSeg sg = sched.seg(worker, k);
        const AttRing ro{sg.n};
        const long ibase = 2 * UPI * sched.tiles_before(k);
        for (int j = 0; j < sg.n && ok; ++j, ++gt) {
          const int pb = static_cast<int>(gt & 1);
          const int it = ro.item_v(j);
          // V_j resident before waiting for P_j (V_j's load waits only on items
          // consumed before it), so P_j's arrival is followed by the MMAs alone
          for (int u = 0; u < UPI && ok; ++u) {
            const long i = ibase + UPI * it + u;
            ok = att_wait_passed(passed, i, abort_flag) &&
                 att_wait<PAIR>(&full[i % ATT_SLOTS], static_cast<uint32_t>(i / ATT_SLOTS) & 1,
                                abort_flag);
          }
          if (!ok || !att_wait<PAIR>(&p_full[pb], static_cast<uint32_t>(gt >> 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          // the first PV of a segment overwrites O: the previous one's O drained
          if (j == 0 && k > 0 &&
              !att_wait<PAIR>(o_free, static_cast<uint32_t>(k - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          for (int u = 0; u < UPI; ++u) {
            const long i = ibase + UPI * it + u;
            const int slot = static_cast<int>(i % ATT_SLOTS);
            const uint64_t vd = sdesc_kmajor_sw128(smem_u32(ring + slot * ATT_SLOT_BYTES));
            const uint32_t p_col = tmem + ATT_TMEM_P + 64 * pb;
            if constexpr (PAIR) {
              // 128 head dims x 128 keys in each CTA: 2 chunks [128 dims x 128 B]
#pragma unroll
              for (int kk = 0; kk < 8; ++kk)  // K step of 16 keys
                umma_bf16_ts_pair(tmem + ATT_TMEM_O, p_col + kk * 8,
                                  vd + ((kk >> 2) * 16384 + (kk & 3) * 32) / 16, IDESC_PV,
                                  (j > 0 || kk > 0) ? 1u : 0u);
            } else {
#pragma unroll
              for (int kq = 0; kq < 4; ++kq) {
                const int kk = u * 4 + kq;  // K step of 16 keys
                umma_bf16_ts(tmem + ATT_TMEM_O, p_col + kk * 8, vd + (kq * 32) / 16, IDESC_PV,
                             (j > 0 || kk > 0) ? 1u : 0u);
              }
            }
            att_commit<PAIR>(&empty[slot]);
          }
          if (ok) att_commit<PAIR>(&pv_done[pb]);
        }
      }
      att_commit<PAIR>(drain_pv);
      att_wait<PAIR>(drain_pv, 0, nullptr, WAIT_LIMIT_NS / 4);
    }
  } else {
    // -------------------------------------------- softmax warps 0..3 (each CTA its own rows)
    const int r = warp * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const uint64_t scale2 = f2_pack(ATT_SCALE_LOG2, ATT_SCALE_LOG2);
    bool ok = true;
    long gt = 0;
    for (int k = 0; k < n_seg && ok; ++k) {
      const AttSeg sg = sched.seg(worker, k);
      float m_used = -INFINITY;
      float l_sum = 0.0f;
      for (int j = 0; j < sg.n; ++j, ++gt) {
        if (!att_wait_warp<PAIR>(s_full, static_cast<uint32_t>(gt) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // all 128 scores in flight before one wait
        float sc[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tmem + lane_base + ATT_TMEM_S + c * 32, sc[c]);
        tmem_ld_wait();
        float t[128];
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i) t[32 * c + i] = sc[c][i];
        // S_j is in registers: the S buffer may take S_{j+1}.
        tc_fence_before();
        __syncwarp();
        if (lane == 0) att_arrive_leader<PAIR>(s_free);

        const int kbase = (sg.t0 + j) * ATT_BN;
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

        // p = 2^(s * scale - m), packed to bf16 pairs; row sum in fp32 pairs.
        // One pair in eight takes the FMA-pipe exponential, which the MUFU
        // unit (the softmax's bottleneck) does not serve.
        const uint64_t negm2 = f2_pack(-m_new, -m_new);
        uint32_t pk[64];
        uint64_t acc[4] = {0, 0, 0, 0};
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const uint64_t x2 = ffma2(f2_pack(t[2 * i], t[2 * i + 1]), scale2, negm2);
          const uint64_t p2 = (i & 7) == 0
                                  ? exp2_poly2(x2)
                                  : f2_pack(exp2_approx(f2_lo(x2)), exp2_approx(f2_hi(x2)));
          acc[i & 3] = fadd2(acc[i & 3], p2);
          pk[i] = pack_bf16x2(f2_lo(p2), f2_hi(p2));
        }
        const uint64_t s2 = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
        const float rowsum = f2_lo(s2) + f2_hi(s2);

        const int pb = static_cast<int>(gt & 1);
        if (gt >= 2) {
          // PV_{gt-2} read this P buffer
          if (!att_wait_warp<PAIR>(&pv_done[pb], static_cast<uint32_t>((gt >> 1) - 1) & 1,
                                   abort_flag)) {
            ok = false;
            break;
          }
        }
        if (any_need) {
          // PV_{gt-1} (same segment, j > 0) must be done: it writes O
          if (!att_wait_warp<PAIR>(&pv_done[pb ^ 1], static_cast<uint32_t>((gt - 1) >> 1) & 1,
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
        if (lane == 0) att_arrive_leader<PAIR>(&p_full[pb]);
      }
      if (!ok) break;
      // ---- the segment's output: O / l (bf16) or the partial (O, m, l)
      const long gl = gt - 1;
      if (!att_wait_warp<PAIR>(&pv_done[gl & 1], static_cast<uint32_t>(gl >> 1) & 1,
                               abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int bh = sg.item / n_units;
      const int q0 = ((sg.item - bh * n_units) * CTAS + rank) * ATT_BM;
      const int b = bh / H, h = bh - (bh / H) * H;
      const int lq = q0 + r;
      const bool valid = lq < L;
      const float inv = sg.slot < 0 ? 1.0f / l_sum : 1.0f;
      __nv_bfloat16 *dst;
      if (sg.slot < 0) {
        dst = o_out + (static_cast<long>(b) * L + lq) * (static_cast<long>(H) * ATT_DH) +
              h * ATT_DH;
      } else {
        uint8_t *sp = part + static_cast<long>(sg.slot * CTAS + rank) * ATT_PART_BYTES;
        dst = reinterpret_cast<__nv_bfloat16 *>(sp) + static_cast<long>(r) * ATT_DH;
        float *ml = reinterpret_cast<float *>(sp + ATT_PART_O_BYTES);
        ml[r] = m_used;
        ml[ATT_BM + r] = l_sum;
      }
      const bool store = valid || sg.slot >= 0;
      // MX8 output (o_sf != nullptr): E4M3 codes in o_out's bytes, a scale per 32 dims
      const bool mx8 = o_sf != nullptr && sg.slot < 0;
      // every row start and 32-column step is a multiple of 32 bytes from the
      // base, so one test of the base covers all threads' stores
      const bool a32 = ((reinterpret_cast<uintptr_t>(mx8 ? static_cast<void *>(o_out)
                                                          : static_cast<void *>(dst)) &
                         31) == 0);
      // O in two halves of 128 columns: four TMEM loads in flight per wait
#pragma unroll 1
      for (int hc = 0; hc < ATT_DH; hc += 128) {
        float o[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tmem + lane_base + ATT_TMEM_O + hc + 32 * c, o[c]);
        tmem_ld_wait();
        if (!store) continue;
        if (mx8) {
          const long grow = static_cast<long>(b) * L + lq;
          const int HD = H * ATT_DH;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
#pragma unroll
            for (int i = 0; i < 32; ++i) o[c][i] *= inv;
            uint4 q[2];
            const uint8_t sb = mx8_encode32(o[c], q);
            const int col = h * ATT_DH + hc + 32 * c;
            uint4 *d = reinterpret_cast<uint4 *>(reinterpret_cast<uint8_t *>(o_out) + grow * HD + col);
            if (a32) {
              const uint32_t w[8] = {q[0].x, q[0].y, q[0].z, q[0].w, q[1].x, q[1].y, q[1].z, q[1].w};
              st_global_v8(d, w);
            } else {
              d[0] = q[0];
              d[1] = q[1];
            }
            o_sf[mx8_sf_offset(static_cast<int>(grow), col / MX8_BLOCK, HD)] = sb;
          }
          continue;
        }
        if (a32) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              uint32_t w[8];
#pragma unroll
              for (int i = 0; i < 8; ++i)
                w[i] = pack_bf16x2(o[c][16 * q + 2 * i] * inv, o[c][16 * q + 2 * i + 1] * inv);
              st_global_v8(dst + hc + 32 * c + 16 * q, w);
            }
          }
          continue;
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint4 *d = reinterpret_cast<uint4 *>(dst + hc + 32 * c);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 w;
            w.x = pack_bf16x2(o[c][8 * q + 0] * inv, o[c][8 * q + 1] * inv);
            w.y = pack_bf16x2(o[c][8 * q + 2] * inv, o[c][8 * q + 3] * inv);
            w.z = pack_bf16x2(o[c][8 * q + 4] * inv, o[c][8 * q + 5] * inv);
            w.w = pack_bf16x2(o[c][8 * q + 6] * inv, o[c][8 * q + 7] * inv);
            d[q] = w;
          }
        }
      }
      // O is in registers or memory: the next segment's first PV may overwrite it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) att_arrive_leader<PAIR>(o_free);
    }
  }

  __syncwarp();
  tc_fence_before();
  if constexpr (PAIR)
    cluster_sync_all();
  else
    __syncthreads();
  tc_fence_after();
  if (warp == 5) {
    if constexpr (PAIR)
      tmem_dealloc_pair(tmem, ATT_TMEM_COLS);
    else
      tmem_dealloc(tmem, ATT_TMEM_COLS);
  }
}

// Merge of the split tail items: block (j, y) takes rows 8y .. 8y+7 of tail
// item j (128 rows, or 256 for a pair item: rows [128 r, 128 r + 128) come
// from rank r), one warp per row; piece p of the item sits in partial slot
// j k + p (for pairs, 2 (j k + p) + r).  m = max m_p, l = sum l_p 2^(m_p - m),
// o = sum O_p 2^(m_p - m) / l (pieces in order), stored as bf16.  Lane p
// holds m and l of piece p (32 pieces at a time) and passes its weight by
// shuffle; lane i accumulates head dims 8i .. 8i+7.
constexpr int ATT_COMBINE_THREADS = 256;
constexpr int ATT_COMBINE_ROWS = ATT_COMBINE_THREADS / 32;

template <bool PAIR>
__global__ void __launch_bounds__(ATT_COMBINE_THREADS)
    attention_combine_kernel(const uint8_t *__restrict__ part, __nv_bfloat16 *__restrict__ o_out,
                             int L, int H, int n_bh, int G, uint8_t *__restrict__ o_sf) {
  constexpr int CTAS = PAIR ? 2 : 1;
  pdl_wait();
  pdl_trigger();
  const int nkv = (L + ATT_BN - 1) / ATT_BN;
  const int n_units = PAIR ? (nkv + 1) / 2 : nkv;
  const AttSched sched(n_bh * n_units, G, nkv);
  const int j = blockIdx.x;
  const int k = sched.k;
  if (j >= sched.rem || k < 2) return;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rp = blockIdx.y * ATT_COMBINE_ROWS + warp;  // row of the item
  if (rp >= CTAS * ATT_BM) return;
  const int rank = rp / ATT_BM;
  const int r = rp - rank * ATT_BM;
  const int item = sched.rounds * G + j;
  const int bh = item / n_units;
  const int q0 = ((item - bh * n_units) * CTAS + rank) * ATT_BM;
  const int lq = q0 + r;
  if (lq >= L) return;
  const int b = bh / H, h = bh - (bh / H) * H;
  auto slot_of = [&](int p) {
    return part + static_cast<long>((j * k + p) * CTAS + rank) * ATT_PART_BYTES;
  };
  auto ml_of = [&](int p) { return reinterpret_cast<const float *>(slot_of(p) + ATT_PART_O_BYTES); };
  float m = -INFINITY;
  for (int p0 = 0; p0 < k; p0 += 32)
    if (p0 + lane < k) m = fmaxf(m, ml_of(p0 + lane)[r]);
  m = warp_max(m);
  float l = 0.0f, acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int p0 = 0; p0 < k; p0 += 32) {
    float wgt = 0.0f;
    if (p0 + lane < k) {
      const float *ml = ml_of(p0 + lane);
      wgt = exp2f(ml[r] - m);
      l = fmaf(ml[ATT_BM + r], wgt, l);
    }
    const int n = min(32, k - p0);
#pragma unroll 4
    for (int q = 0; q < n; ++q) {
      const float w = __shfl_sync(0xffffffffu, wgt, q);
      const uint4 v = reinterpret_cast<const uint4 *>(slot_of(p0 + q) +
                                                      static_cast<long>(r) * ATT_DH * 2)[lane];
      const uint32_t u4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[2 * e] = fmaf(__uint_as_float(u4[e] << 16), w, acc[2 * e]);
        acc[2 * e + 1] = fmaf(__uint_as_float(u4[e] & 0xFFFF0000u), w, acc[2 * e + 1]);
      }
    }
  }
  const float inv = 1.0f / warp_sum(l);
  if (o_sf != nullptr) {
    // MX8 output: lanes 4j .. 4j + 3 hold a block of 32 head dims
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      acc[i] = bf16_round(acc[i] * inv);  // the bf16 output's value, encoded
      amax = fmaxf(amax, fabsf(acc[i]));
    }
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    const int e = mx8_exponent(amax);
    const float is = mx8_inv_scale(e);
    const long grow = static_cast<long>(b) * L + lq;
    const int HD = H * ATT_DH;
    const int col = h * ATT_DH + 8 * lane;
    uint2 w;
    w.x = static_cast<uint32_t>(pack_e4m3x2(acc[0] * is, acc[1] * is)) |
          (static_cast<uint32_t>(pack_e4m3x2(acc[2] * is, acc[3] * is)) << 16);
    w.y = static_cast<uint32_t>(pack_e4m3x2(acc[4] * is, acc[5] * is)) |
          (static_cast<uint32_t>(pack_e4m3x2(acc[6] * is, acc[7] * is)) << 16);
    *reinterpret_cast<uint2 *>(reinterpret_cast<uint8_t *>(o_out) + grow * HD + col) = w;
    if ((lane & 3) == 0)
      o_sf[mx8_sf_offset(static_cast<int>(grow), col / MX8_BLOCK, HD)] = static_cast<uint8_t>(e + 127);
    return;
  }
  __nv_bfloat16 *dst = o_out + (static_cast<long>(b) * L + lq) * (static_cast<long>(H) * ATT_DH) +
                       h * ATT_DH + 8 * lane;
  *reinterpret_cast<uint4 *>(dst) =
      make_uint4(pack_bf16x2(acc[0] * inv, acc[1] * inv), pack_bf16x2(acc[2] * inv, acc[3] * inv),
                 pack_bf16x2(acc[4] * inv, acc[5] * inv), pack_bf16x2(acc[6] * inv, acc[7] * inv));
}

}  // namespace ig4
