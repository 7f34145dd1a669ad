// attn_tc.cuh -- exact prefill attention over the selected KV blocks on the
// 5th-generation tensor cores (tcgen05 + TMEM).
//
// MiniCPM4 summary page (端设备上的超高效大型语言模型) s2.1.3: each token attends only to
// its most relevant KV blocks; s2.1.2: the 16 query heads of a group share them, so a
// block is fetched once per group.
//
// Work item = (sequence b, kv-head g, query token t).  The item's selected blocks are
// taken in pairs (128 keys); a persistent CTA streams them with TMA (128-byte swizzle, no
// multicast) through two rings of 32 KB slots, one for K pairs (warp 8) and one for V
// pairs (warp 11), so a K slot is free again right after its QK and a V slot right
// after its PV; per pair:
//   warp 9 (one thread) issues  S^T = K_pair . Q^T   (UMMA M128 N16 K128: keys x heads)
//          into one of four TMEM score buffers as soon as the pair has landed;
//   warp 10 (one thread) issues, as soon as P is in shared memory,
//          O^T += V^T . P^T   (UMMA M128 N16 K128: V read through an MN-major
//          descriptor, P K-major) into the TMEM output buffer of the pair's warpgroup.
//          Two issuers keep a PV from waiting behind the next pair's loads;
//   warps 0-7: two softmax warpgroups take alternate pairs (128 threads each, thread =
//          key of the pair), each with its own TMEM output buffer, reference maxima and
//          row sums (a split over the pairs inside the CTA).  A thread reads its key's 16
//          head scores; only when a score exceeds the warpgroup's reference m_h by 2^8
//          (one barrier-OR vote) is the pair maximum reduced across threads and that
//          O^T rescaled in TMEM; p = exp2(s - m_h) goes to shared memory as bf16 and the
//          partial row sums stay in registers.  At the end of the item the two partial
//          states are merged (thread = output column d) and O and the log-sum-exp are
//          written;
//   warp 8 also loads the query tile and compacts the block list of each item.
// In a prefill chunk the cache may end inside the query's own block; key rows past the
// cache end hold arbitrary values, so the V producer loads that one pair onto a barrier of
// its own, zeroes those rows in shared memory and only then marks the pair loaded (their
// P is 0, and 0 x anything stays 0 only when "anything" is finite).
#pragma once
#include "attn.cuh"
#include "common.cuh"
#include "tcgen05.cuh"

namespace infllmv2 {

constexpr int kAtKStages = 4;                      // slots of the K ring
constexpr int kAtVStages = 2;                      // slots of the V ring
constexpr int kAtKHalf = 2 * kKvTileBytes / 2;     // 16 KB: one 64-column half of 128 keys
constexpr int kAtSlotBytes = 2 * kKvTileBytes;     // 32 KB: a pair of K (or V) blocks
constexpr int kAtPBytes = kGroupRows * 128 * 2;    // 4 KB: P (16 heads x 128 keys bf16)
constexpr int kAtSoftWGs = 2;
constexpr int kAtThreads = 32 * (4 * kAtSoftWGs + 4);
constexpr int kAtTmaWarp = 4 * kAtSoftWGs, kAtMmaWarp = kAtTmaWarp + 1, kAtPvWarp = kAtTmaWarp + 2,
              kAtVTmaWarp = kAtTmaWarp + 3;
constexpr int kAtBufs = 4;  // score (TMEM) and probability (shared) buffers in flight
// TMEM columns: scores S[b] at 16 b, outputs O[item parity][wg] at 16 kAtBufs + 16 (2 it + wg);
// the allocation is the next power of two
constexpr uint32_t kAtOCol = 16 * kAtBufs;
constexpr uint32_t kAtTmemCols = kAtOCol + 64 <= 128 ? 128 : (kAtOCol + 64 <= 256 ? 256 : 512);

struct AtSmem {
  uint64_t k_full[kAtKStages], k_empty[kAtKStages], v_full[kAtVStages], v_empty[kAtVStages], q_full[2], q_empty[2];
  uint64_t s_full[kAtBufs], p_full[kAtBufs], pv_done[kAtBufs], mma_done[2];
  uint64_t vtail;   // the V producer's own barrier for the pair that straddles the cache end
  int n_blocks[2];
  int tail_pos[2];  // list position of the block that straddles the cache end (-1: none)
  int list[2][kMaxTopk];
  float red[kAtSoftWGs][4][kGroupRows];
  float mstate[kAtSoftWGs][kGroupRows], lstate[kAtSoftWGs][kGroupRows];
  float lse_out[kGroupRows];
  uint32_t tmem_base;
  volatile int abort;
};

constexpr size_t attn_tc_smem_bytes() {
  return 1024 + static_cast<size_t>(kAtKStages + kAtVStages) * kAtSlotBytes + 2 * kQTileBytes + kAtBufs * kAtPBytes +
         sizeof(AtSmem);
}
static_assert(attn_tc_smem_bytes() <= 227 * 1024, "shared memory of one CTA");

// Zeroes V rows r0 .. 63 of the block whose 64 rows start at `vs` in a pair slot (both
// 64-column halves).  Runs only for the block that straddles a cache end.
__device__ __noinline__ void zero_v_rows(unsigned char* vs, int r0) {
  for (int r = max(r0, 0); r < kBlock; ++r)
    for (int c = 0; c < 8; ++c) {
      *reinterpret_cast<uint4*>(vs + r * 128 + c * 16) = make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4*>(vs + kAtKHalf + r * 128 + c * 16) = make_uint4(0, 0, 0, 0);
    }
}

// Per-lane result of a 32-lane max / sum over 16 values: lane L holds the total for
// value index L >> 1 (lanes 2h and 2h+1 agree).  16 shuffles.
template <bool kMax>
__device__ __forceinline__ float warp_reduce16(const float (&v)[16]) {
  const int lane = threadIdx.x & 31;
  auto op = [](float a, float b) { return kMax ? fmaxf(a, b) : a + b; };
  float a[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const bool up = lane & 16;
    const float send = up ? v[i] : v[i + 8];
    const float keep = up ? v[i + 8] : v[i];
    a[i] = op(keep, __shfl_xor_sync(0xffffffffu, send, 16));
  }
  float b4[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const bool up = lane & 8;
    const float send = up ? a[i] : a[i + 4];
    const float keep = up ? a[i + 4] : a[i];
    b4[i] = op(keep, __shfl_xor_sync(0xffffffffu, send, 8));
  }
  float c2[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const bool up = lane & 4;
    const float send = up ? b4[i] : b4[i + 2];
    const float keep = up ? b4[i + 2] : b4[i];
    c2[i] = op(keep, __shfl_xor_sync(0xffffffffu, send, 4));
  }
  const bool up = lane & 2;
  const float send = up ? c2[0] : c2[1];
  const float keep = up ? c2[1] : c2[0];
  const float d = op(keep, __shfl_xor_sync(0xffffffffu, send, 2));
  return op(d, __shfl_xor_sync(0xffffffffu, d, 1));
}

// Cross-warp (4 warps) max or sum of 16 per-thread values; every thread gets all 16.
template <bool kMax>
__device__ __forceinline__ void wg_reduce16(const float (&v)[16], float (&out)[16], AtSmem& S, int wg) {
  const int wq = (threadIdx.x >> 5) & 3, lane = threadIdx.x & 31;
  const float r = warp_reduce16<kMax>(v);
  if ((lane & 1) == 0) S.red[wg][wq][lane >> 1] = r;
  named_bar_sync(1 + wg, 128);
#pragma unroll
  for (int h = 0; h < kGroupRows; ++h) {
    const float a = S.red[wg][0][h], b = S.red[wg][1][h], c = S.red[wg][2][h], d = S.red[wg][3][h];
    out[h] = kMax ? fmaxf(fmaxf(a, b), fmaxf(c, d)) : (a + b) + (c + d);
  }
  named_bar_sync(1 + wg, 128);  // S.red may be reused afterwards
}

// grid = min(items, SMs) persistent CTAs, block = 384.  Prefill and prefill chunks only
// (p.lens == nullptr).
__global__ void __launch_bounds__(kAtThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = align_smem(smem_raw, 1024);
  unsigned char* kring = base;
  unsigned char* vring = kring + kAtKStages * kAtSlotBytes;
  unsigned char* qtiles = vring + kAtVStages * kAtSlotBytes;
  unsigned char* pbufs = qtiles + 2 * kQTileBytes;
  AtSmem& S = *reinterpret_cast<AtSmem*>(pbufs + kAtBufs * kAtPBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kAtKStages; ++s) {
      mbar_init(&S.k_full[s], 1);
      mbar_init(&S.k_empty[s], 1);
    }
    for (int s = 0; s < kAtVStages; ++s) {
      mbar_init(&S.v_full[s], 1);
      mbar_init(&S.v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&S.q_full[s], 1);
      mbar_init(&S.q_empty[s], 3);  // last QK done + V producer and softmax warps done with the item
    }
    for (int s = 0; s < kAtBufs; ++s) {
      mbar_init(&S.s_full[s], 1);
      mbar_init(&S.p_full[s], 1);
      mbar_init(&S.pv_done[s], 1);
    }
    mbar_init(&S.mma_done[0], 1);
    mbar_init(&S.mma_done[1], 1);
    mbar_init(&S.vtail, 1);
    S.abort = 0;
    fence_mbar_init();
  }
  if (warp == kAtMmaWarp) {
    tmem_alloc(&S.tmem_base, kAtTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;

  if (warp == kAtTmaWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
    }
    uint32_t gpair = 0;
    int it = 0;
    const uint64_t qpol = l2_policy_evict_first();  // queries are read once: K/V keep L2
    // copies issued so far (lane 0), in order: pairs 0 .. k_issued - 1 and query tiles of
    // items 0 .. q_issued - 1 (after an abort nothing more is issued), for the drain
    uint32_t k_issued = 0, q_issued = 0;
    for (long long item = blockIdx.x; item < p.num_items; item += gridDim.x, ++it) {
      const int slot = it & 1, use = it >> 1;
      if (use > 0) mbar_wait(&S.q_empty[slot], (use - 1) & 1, &S.abort);
      const AttnItem a = attn_item(p, item);
      const int cur = a.t >= 0 ? a.t / kBlock : -1;
      const int32_t* row = p.idx + ((a.bg * p.Lq + a.row) * static_cast<long long>(p.topk));
      const int tail_j = (a.kv_len % kBlock) != 0 ? a.kv_len / kBlock : -1;  // straddles the cache end
      int count = 0, tail = -1;
      for (int e0 = 0; e0 < p.topk; e0 += 32) {
        const int e = e0 + lane;
        const int j = (e < p.topk && a.valid) ? __ldcs(row + e) : -1;
        const bool ok = j >= 0 && j <= cur;
        const unsigned msk = __ballot_sync(0xffffffffu, ok);
        const int pos = count + __popc(msk & ((1u << lane) - 1u));
        if (ok) S.list[slot][pos] = j;
        const unsigned tm = __ballot_sync(0xffffffffu, ok && j == tail_j);
        if (tm != 0u) tail = count + __popc(msk & ((1u << (__ffs(tm) - 1)) - 1u));
        count += __popc(msk);
      }
      if (lane == 0) {
        S.n_blocks[slot] = count;
        S.tail_pos[slot] = tail;
      }
      __threadfence_block();
      __syncwarp();
      const int np = (count + 1) / 2;
      if (lane == 0) {
        unsigned char* qs = qtiles + slot * kQTileBytes;
        if (!S.abort) {
          mbar_arrive_expect_tx(&S.q_full[slot], kQTileBytes);
          tma_load_2d_hint(qs, &tm_q, &S.q_full[slot], 0, a.qrow, qpol);
          tma_load_2d_hint(qs + kQTileBytes / 2, &tm_q, &S.q_full[slot], 64, a.qrow, qpol);
          q_issued = static_cast<uint32_t>(it) + 1u;
        }
        const long long kvrow0 = a.bg * p.Lmax;
        for (int i = 0; i < np; ++i, ++gpair) {
          const int st = static_cast<int>(gpair % kAtKStages);
          const uint32_t u = gpair / kAtKStages;
          if (u > 0) mbar_wait(&S.k_empty[st], (u - 1) & 1, &S.abort);
          if (S.abort) continue;
          const int ja = S.list[slot][2 * i];
          const int jb = 2 * i + 1 < count ? S.list[slot][2 * i + 1] : -1;
          const int ra = static_cast<int>(kvrow0 + static_cast<long long>(ja) * kBlock);
          const int rb = jb >= 0 ? static_cast<int>(kvrow0 + static_cast<long long>(jb) * kBlock) : -kBlock;
          unsigned char* sk = kring + st * kAtSlotBytes;
          k_issued = gpair + 1u;
          mbar_arrive_expect_tx(&S.k_full[st], kAtSlotBytes);
          // rows 0-63 of each 128-key half: block a; rows 64-127: block b (zeros when absent)
          tma_load_2d(sk, &tm_k, &S.k_full[st], 0, ra);
          tma_load_2d(sk + kAtKHalf, &tm_k, &S.k_full[st], 64, ra);
          tma_load_2d(sk + kKvTileBytes / 2, &tm_k, &S.k_full[st], 0, rb);
          tma_load_2d(sk + kAtKHalf + kKvTileBytes / 2, &tm_k, &S.k_full[st], 64, rb);
        }
      } else {
        gpair += np;
      }
      gpair = __shfl_sync(0xffffffffu, gpair, 0);
    }
    if (lane == 0 && S.abort) {  // let every copy this warp issued land before the CTA ends
      for (uint32_t st = 0; st < kAtKStages; ++st)
        if (k_issued > st) {  // the last pair issued into stage st
          const uint32_t last = st + kAtKStages * ((k_issued - 1u - st) / kAtKStages);
          mbar_wait_drain(&S.k_full[st], (last / kAtKStages) & 1u);
        }
      for (uint32_t sl = 0; sl < 2; ++sl)
        if (q_issued > sl) {  // the last item whose query tile went to slot sl
          const uint32_t last = sl + 2u * ((q_issued - 1u - sl) / 2u);
          mbar_wait_drain(&S.q_full[sl], (last >> 1) & 1u);
        }
    }
    return;
  }

  if (warp == kAtVTmaWarp) {
    // ------------------------------------------------------------ V producer
    // V pairs are loaded through their own ring, so a V slot is held only until its PV,
    // and K slots recycle right after their QK.
    if (lane == 0) {
      uint32_t gpair = 0, n_tail = 0;
      int it = 0;
      uint32_t v_issued = 0;  // V pairs issued so far, in order (for the drain)
      for (long long item = blockIdx.x; item < p.num_items; item += gridDim.x, ++it) {
        const int slot = it & 1, use = it >> 1;
        mbar_wait(&S.q_full[slot], use & 1, &S.abort);  // the item's block list is ready
        const AttnItem a = attn_item(p, item);
        const int count = S.n_blocks[slot];
        const int tail = S.tail_pos[slot];
        const int np = (count + 1) / 2;
        const long long kvrow0 = a.bg * p.Lmax;
        for (int i = 0; i < np; ++i, ++gpair) {
          const int st = static_cast<int>(gpair % kAtVStages);
          const uint32_t u = gpair / kAtVStages;
          if (u > 0) mbar_wait(&S.v_empty[st], (u - 1) & 1, &S.abort);
          if (S.abort) continue;
          const int ja = S.list[slot][2 * i];
          const int jb = 2 * i + 1 < count ? S.list[slot][2 * i + 1] : -1;
          const int ra = static_cast<int>(kvrow0 + static_cast<long long>(ja) * kBlock);
          const int rb = jb >= 0 ? static_cast<int>(kvrow0 + static_cast<long long>(jb) * kBlock) : -kBlock;
          unsigned char* sv = vring + st * kAtSlotBytes;
          v_issued = gpair + 1u;
          if ((tail >> 1) != i) {  // (tail == -1: no straddling block in the item)
            mbar_arrive_expect_tx(&S.v_full[st], kAtSlotBytes);
            tma_load_2d(sv, &tm_v, &S.v_full[st], 0, ra);
            tma_load_2d(sv + kAtKHalf, &tm_v, &S.v_full[st], 64, ra);
            tma_load_2d(sv + kKvTileBytes / 2, &tm_v, &S.v_full[st], 0, rb);
            tma_load_2d(sv + kAtKHalf + kKvTileBytes / 2, &tm_v, &S.v_full[st], 64, rb);
          } else {
            // the pair with the block that straddles the cache end: load it here, zero the
            // rows past the end, then mark it loaded
            mbar_arrive_expect_tx(&S.vtail, kAtSlotBytes);
            tma_load_2d(sv, &tm_v, &S.vtail, 0, ra);
            tma_load_2d(sv + kAtKHalf, &tm_v, &S.vtail, 64, ra);
            tma_load_2d(sv + kKvTileBytes / 2, &tm_v, &S.vtail, 0, rb);
            tma_load_2d(sv + kAtKHalf + kKvTileBytes / 2, &tm_v, &S.vtail, 64, rb);
            mbar_wait_drain(&S.vtail, n_tail & 1);
            ++n_tail;
            zero_v_rows(sv + (tail & 1) * (kKvTileBytes / 2), a.kv_len - S.list[slot][tail] * kBlock);
            fence_proxy_async_smem();  // the generic writes before the MMA's reads
            mbar_arrive(&S.v_full[st]);
          }
        }
        mbar_arrive(&S.q_empty[slot]);  // done with the item's block list
      }
      if (S.abort)  // let every copy this thread issued land before the CTA ends
        for (int st = 0; st < kAtVStages; ++st)
          if (v_issued > static_cast<uint32_t>(st)) {
            const uint32_t last = st + kAtVStages * ((v_issued - 1u - st) / kAtVStages);
            mbar_wait_drain(&S.v_full[st], (last / kAtVStages) & 1u);
          }
    }
    return;
  }

  if (warp == kAtMmaWarp || warp == kAtPvWarp) {
    // ------------------------------------------------------- MMA issuers (QK / PV)
    const bool is_qk = warp == kAtMmaWarp;
    constexpr uint32_t idesc_qk = idesc_bf16_f32(128, kGroupRows, false, false);
    constexpr uint32_t idesc_pv = idesc_bf16_f32(128, kGroupRows, true, false);
    if (lane == 0) {
      uint32_t gp = 0;
      int it = 0;
      for (long long item = blockIdx.x; item < p.num_items; item += gridDim.x, ++it) {
        const int slot = it & 1, use = it >> 1;
        mbar_wait(&S.q_full[slot], use & 1, &S.abort);
        const int np = (S.n_blocks[slot] + 1) / 2;
        if (is_qk) {
          const uint32_t qa = smem_u32(qtiles + slot * kQTileBytes);
          for (int i = 0; i < np; ++i) {
            const uint32_t pp = gp + i;
            mbar_wait(&S.k_full[pp % kAtKStages], (pp / kAtKStages) & 1, &S.abort);
            if (pp >= kAtBufs) mbar_wait(&S.p_full[pp % kAtBufs], ((pp / kAtBufs) - 1) & 1, &S.abort);  // S read
            tc_fence_after();
            const uint32_t kb = smem_u32(kring + (pp % kAtKStages) * kAtSlotBytes);
            const uint32_t sbuf = tmem + static_cast<uint32_t>(pp % kAtBufs) * 16u;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              umma_bf16(sbuf, desc_k_sw128(kb + (k >> 2) * kAtKHalf + (k & 3) * 32),
                        desc_k_sw128(qa + (k >> 2) * (kQTileBytes / 2) + (k & 3) * 32), idesc_qk,
                        k > 0 ? 1u : 0u);
            }
            umma_commit(&S.s_full[pp % kAtBufs]);
            umma_commit(&S.k_empty[pp % kAtKStages]);
          }
          umma_commit(&S.q_empty[slot]);  // the item's query tile is no longer read
        } else {
          for (int i = 0; i < np; ++i) {
            const uint32_t pp = gp + i;
            mbar_wait(&S.p_full[pp % kAtBufs], (pp / kAtBufs) & 1, &S.abort);
            mbar_wait(&S.v_full[pp % kAtVStages], (pp / kAtVStages) & 1, &S.abort);
            tc_fence_after();
            const uint32_t obuf = tmem + kAtOCol + static_cast<uint32_t>(2 * (it & 1) + (pp & 1)) * 16u;
            const uint32_t vb = smem_u32(vring + (pp % kAtVStages) * kAtSlotBytes);
            const uint32_t pb = smem_u32(pbufs + (pp % kAtBufs) * kAtPBytes);
#pragma unroll
            for (int k = 0; k < 8; ++k) {  // 16 keys per step
              umma_bf16(obuf, desc_mn_sw128(vb + k * 2048, kAtKHalf, 1024),
                        desc_k_sw128(pb + (k >> 2) * (kAtPBytes / 2) + (k & 3) * 32), idesc_pv,
                        (i >= kAtSoftWGs || k > 0) ? 1u : 0u);
            }
            umma_commit(&S.pv_done[pp % kAtBufs]);
            umma_commit(&S.v_empty[pp % kAtVStages]);
          }
        }
        gp += np;
      }
      umma_commit(&S.mma_done[is_qk ? 0 : 1]);
    }
    __syncwarp();
    named_bar_sync(4, 32 * (4 * kAtSoftWGs + 2));  // the softmax warps have read TMEM for the last time
    if (lane == 0) mbar_wait_drain(&S.mma_done[is_qk ? 0 : 1], 0);  // no MMA of this issuer still runs
    __syncwarp();
    named_bar_sync(5, 64);  // both issuers drained
    if (is_qk) {
      tc_fence_after();
      tmem_dealloc(tmem, kAtTmemCols);
    }
    return;
  }

  // ---------------------------------------------------------------- softmax warps
  const int wg = warp >> 2;            // takes the pairs with global index % 2 == wg
  const int tid = threadIdx.x & 127;   // key of the pair, then output column d
  const int bar = 1 + wg;              // this warpgroup's named barrier
  const uint32_t tlane = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
  const float sl2 = p.scale_log2;
  uint32_t gp = 0;
  int it = 0;
  for (long long item = blockIdx.x; item < p.num_items; item += gridDim.x, ++it) {
    const int slot = it & 1, use = it >> 1;
    mbar_wait(&S.q_full[slot], use & 1, &S.abort);
    const AttnItem a = attn_item(p, item);
    const int n = S.n_blocks[slot];
    const int np = (n + 1) / 2;
    const uint32_t obuf = tlane + kAtOCol + static_cast<uint32_t>(2 * (it & 1) + wg) * 16u;
    float m[kGroupRows], l[kGroupRows];
#pragma unroll
    for (int h = 0; h < kGroupRows; ++h) {
      m[h] = -INFINITY;
      l[h] = 0.f;
    }
    int i0 = 0;
    while (i0 < np && ((gp + i0) & 1) != static_cast<uint32_t>(wg)) ++i0;
    for (int i = i0; i < np; i += 2) {
      const uint32_t pp = gp + i;
      mbar_wait(&S.s_full[pp % kAtBufs], (pp / kAtBufs) & 1, &S.abort);
      tc_fence_after();
      uint32_t sv[16];
      tmem_ld16(tlane + static_cast<uint32_t>(pp % kAtBufs) * 16u, sv);
      const int bi = 2 * i + (tid >> 6);
      const int blk = bi < n ? S.list[slot][bi] : -1;
      const int key = blk * kBlock + (tid & 63);
      const bool valid = blk >= 0 && key <= a.t;
      float x[kGroupRows];
      bool viol = false;
#pragma unroll
      for (int h = 0; h < kGroupRows; ++h) {
        x[h] = valid ? __uint_as_float(sv[h]) * sl2 : -INFINITY;
        viol |= x[h] > m[h] + 8.f;
      }
      if (named_bar_or(bar, 128, viol)) {
        // a score rose more than 2^8 above its reference: move the references to the
        // pair maxima and rescale what this warpgroup accumulated so far
        float mx[kGroupRows];
        wg_reduce16<true>(x, mx, S, wg);
        float al[kGroupRows];
#pragma unroll
        for (int h = 0; h < kGroupRows; ++h) {
          const float mn = fmaxf(m[h], mx[h]);
          al[h] = (m[h] == -INFINITY) ? 0.f : ex2(m[h] - mn);
          l[h] *= al[h];
          m[h] = mn;
        }
        if (i >= i0 + 2) {  // this warpgroup has accumulated into its O^T before
          mbar_wait(&S.pv_done[(pp - 2) % kAtBufs], ((pp - 2) / kAtBufs) & 1, &S.abort);  // previous PV
          tc_fence_after();
          uint32_t ov[16];
          tmem_ld16(obuf, ov);
#pragma unroll
          for (int h = 0; h < kGroupRows; ++h) ov[h] = __float_as_uint(__uint_as_float(ov[h]) * al[h]);
          tmem_st16(obuf, ov);
        }
      }
      float pv[kGroupRows];
#pragma unroll
      for (int h = 0; h < kGroupRows; ++h) {
        pv[h] = (m[h] == -INFINITY) ? 0.f : ex2(x[h] - m[h]);
        l[h] += pv[h];
      }
      if (pp >= kAtBufs) mbar_wait(&S.pv_done[pp % kAtBufs], ((pp / kAtBufs) - 1) & 1, &S.abort);  // P free
      {
        unsigned char* pbuf = pbufs + (pp % kAtBufs) * kAtPBytes + (tid >> 6) * (kAtPBytes / 2);
        const int col = tid & 63;
#pragma unroll
        for (int h = 0; h < kGroupRows; ++h) {
          const __nv_bfloat16 v = __float2bfloat16_rn(pv[h]);
          *reinterpret_cast<__nv_bfloat16*>(pbuf + sw128(h, col >> 3) + (col & 7) * 2) = v;
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar_sync(bar, 128);
      if (tid == 0) mbar_arrive(&S.p_full[pp % kAtBufs]);
    }

    // ---- end of item: merge the two warpgroups' partial states (thread = column d)
    float L[kGroupRows];
    wg_reduce16<false>(l, L, S, wg);
    if (tid == 0) {
#pragma unroll
      for (int h = 0; h < kGroupRows; ++h) {
        S.mstate[wg][h] = m[h];
        S.lstate[wg][h] = L[h];
      }
    }
    const bool had = i0 < np;  // this warpgroup accumulated into its O^T
    uint32_t ov[16];
    if (had) {
      const uint32_t last = gp + i0 + 2 * ((np - 1 - i0) / 2);
      mbar_wait(&S.pv_done[last % kAtBufs], (last / kAtBufs) & 1, &S.abort);
      tc_fence_after();
      tmem_ld16(obuf, ov);
    }
    named_bar_sync(3, 32 * 4 * kAtSoftWGs);  // both warpgroups' states are in shared memory
    float M[kGroupRows], Lt[kGroupRows], w0[kGroupRows], w1[kGroupRows];
#pragma unroll
    for (int h = 0; h < kGroupRows; ++h) {
      const float m0 = S.mstate[0][h], m1 = S.mstate[1][h];
      M[h] = fmaxf(m0, m1);
      w0[h] = (m0 == -INFINITY) ? 0.f : ex2(m0 - M[h]);
      w1[h] = (m1 == -INFINITY) ? 0.f : ex2(m1 - M[h]);
      Lt[h] = S.lstate[0][h] * w0[h] + S.lstate[1][h] * w1[h];
    }
    // warpgroup 0 reads warpgroup 1's O^T buffer directly (same TMEM lanes) and merges
    tc_fence_after();
    if (wg == 0) {
      uint32_t ov1[16];
      const uint32_t obuf1 = tlane + kAtOCol + static_cast<uint32_t>(2 * (it & 1) + 1) * 16u;
      const bool had1 = ((gp & 1u) ? 0 : 1) < np;  // first pair of warpgroup 1 in this item
      if (had1) tmem_ld16(obuf1, ov1);
      float of[kGroupRows];
#pragma unroll
      for (int h = 0; h < kGroupRows; ++h) {
        const float a0 = had ? __uint_as_float(ov[h]) * w0[h] : 0.f;
        const float a1 = had1 ? __uint_as_float(ov1[h]) * w1[h] : 0.f;
        of[h] = Lt[h] > 0.f ? (a0 + a1) / Lt[h] : 0.f;
      }
#pragma unroll
      for (int h = 0; h < kGroupRows; ++h)
        if (h < p.G && a.valid)
          st_stream_bf16(p.o + (static_cast<long long>(a.qrow) + h) * kHeadDim + tid, __float2bfloat16_rn(of[h]));
      if (p.lse != nullptr && tid < p.G && a.valid) {
        float lv = -INFINITY;
#pragma unroll
        for (int h = 0; h < kGroupRows; ++h)
          if (h == tid) lv = Lt[h] > 0.f ? (M[h] + lg2(Lt[h])) * 0.6931471805599453f : -INFINITY;
        __stcs(p.lse + (static_cast<long long>(a.b) * p.Hq + a.g * p.G + tid) * p.Lq + a.row, lv);
      }
    }
    tc_fence_before();
    named_bar_sync(3, 32 * 4 * kAtSoftWGs);  // outputs read; states may be overwritten
    if (threadIdx.x == 0) mbar_arrive(&S.q_empty[slot]);
    gp += np;
  }
  named_bar_sync(4, 32 * (4 * kAtSoftWGs + 2));  // TMEM may be freed
}

}  // namespace infllmv2
