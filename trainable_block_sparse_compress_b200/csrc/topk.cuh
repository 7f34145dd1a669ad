// topk.cuh -- deterministic top-k of block scores and ordered emission of the
// selected block list.
//
// Ordering rule (MiniCPM4 summary page s2.1.1: each query token keeps its highest
// scoring blocks): higher score first, lower block index first among equal scores.
// Scores are non-negative fp32 group sums, so their IEEE bit patterns order like the
// values.  A candidate's key is bits(score) + 1 and a non-candidate's key is 0.
// The k-th largest key is found by bisection on the key bits with warp-wide counts; the
// list is then written in ascending block order with forced blocks first-class members
// and ties at the threshold taken from the lowest indices.
#pragma once
#include "common.cuh"

namespace infllmv2 {

struct TopkThreshold {
  uint32_t key;  // threshold key T (0xffffffff when nothing is to be taken)
  int ties;      // how many keys equal to T are taken (0 when T == 0: take all > 0)
};

// One warp.  keys[0..n) in shared memory; `want` keys to take.  Finds the want-th
// largest key T by bisection on its bits, most significant first: T >= c exactly when
// at least `want` keys are >= c.  Each lane holds up to kTopkRegKeys keys in registers
// (n <= 32 * kTopkRegKeys); larger n re-reads shared memory each step.  No atomics.
constexpr int kTopkRegKeys = 64;

__device__ __forceinline__ int warp_count_ge_regs(const uint32_t (&kr)[kTopkRegKeys], uint32_t c) {
  int cnt[4] = {0, 0, 0, 0};  // four independent chains
#pragma unroll
  for (int i = 0; i < kTopkRegKeys; ++i) cnt[i & 3] += kr[i] >= c ? 1 : 0;
  return static_cast<int>(
      __reduce_add_sync(0xffffffffu, static_cast<unsigned>((cnt[0] + cnt[1]) + (cnt[2] + cnt[3]))));
}

__device__ __forceinline__ int warp_count_ge_smem(const uint32_t* keys, int n, uint32_t c) {
  const int lane = threadIdx.x & 31;
  int cnt = 0;
  for (int i = lane; i < n; i += 32) cnt += keys[i] >= c ? 1 : 0;
  return static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(cnt)));
}

__device__ __forceinline__ TopkThreshold warp_radix_threshold(const uint32_t* keys, int n, int want,
                                                              uint32_t* /*unused scratch*/) {
  const int lane = threadIdx.x & 31;
  TopkThreshold r;
  if (want <= 0) {
    r.key = 0xffffffffu;
    r.ties = 0;
    return r;
  }
  uint32_t T = 0;
  if (n <= 32 * kTopkRegKeys) {
    uint32_t kr[kTopkRegKeys];
#pragma unroll
    for (int i = 0; i < kTopkRegKeys; ++i) {
      const int j = lane + 32 * i;
      kr[i] = j < n ? keys[j] : 0u;
    }
    if (warp_count_ge_regs(kr, 1u) <= want) {  // at most `want` candidates: take them all
      r.key = 0;
      r.ties = 0;
      return r;
    }
#pragma unroll 1
    for (int bit = 30; bit >= 0; --bit) {
      const uint32_t c = T | (1u << bit);
      if (warp_count_ge_regs(kr, c) >= want) T = c;
    }
    r.key = T;
    r.ties = want - warp_count_ge_regs(kr, T + 1u);
    return r;
  }
  if (warp_count_ge_smem(keys, n, 1u) <= want) {
    r.key = 0;
    r.ties = 0;
    return r;
  }
#pragma unroll 1
  for (int bit = 30; bit >= 0; --bit) {
    const uint32_t c = T | (1u << bit);
    if (warp_count_ge_smem(keys, n, c) >= want) T = c;
  }
  r.key = T;
  r.ties = want - warp_count_ge_smem(keys, n, T + 1u);
  return r;
}

// One warp: threshold and ordered emission for n <= 32 * kTopkRegKeys keys, with the
// keys held in registers (key j = keys[lane + 32 i] in kr[i]).  The search is narrowed
// first: every lane keeps its 4 largest keys; with r = ceil(want / 32) <= 4, c0 = the
// warp minimum of the lanes' r-th largest keys bounds the threshold from below (each
// lane holds r keys >= c0, so at least 32 r >= want keys are >= c0).  Only the keys
// >= c0 (usually a few hundred) are copied to `cand` (kTopkCand words of this warp's
// shared scratch) and bisected; when the bound does not apply or too many keys pass it,
// the search runs over all keys.  Same result either way: the want-th largest key.
constexpr int kTopkCand = 256;

__device__ __forceinline__ void warp_topk_select(const uint32_t* keys, int n, int want, int cur, int n_init,
                                                 int n_local, int topk, uint32_t* cand, int32_t* out) {
  const int lane = threadIdx.x & 31;
  const unsigned lt = (1u << lane) - 1u;
  uint32_t kr[kTopkRegKeys];
#pragma unroll
  for (int i = 0; i < kTopkRegKeys; ++i) {
    const int j = lane + 32 * i;
    kr[i] = j < n ? keys[j] : 0u;
  }
  TopkThreshold th;
  if (want <= 0) {
    th.key = 0xffffffffu;
    th.ties = 0;
  } else if (warp_count_ge_regs(kr, 1u) <= want) {
    th.key = 0;
    th.ties = 0;
  } else {
    // lower bound c0 from each lane's r-th largest key
    const int r = (want + 31) / 32;
    uint32_t c0 = 0;
    if (r <= 4) {
      uint32_t t0 = 0, t1 = 0, t2 = 0, t3 = 0;  // descending top-4 of this lane
#pragma unroll
      for (int i = 0; i < kTopkRegKeys; ++i) {
        uint32_t x = kr[i], y;
        y = max(x, t0); x = min(x, t0); t0 = y;
        y = max(x, t1); x = min(x, t1); t1 = y;
        y = max(x, t2); x = min(x, t2); t2 = y;
        t3 = max(x, t3);
      }
      const uint32_t cl = r == 1 ? t0 : (r == 2 ? t1 : (r == 3 ? t2 : t3));
      c0 = __reduce_min_sync(0xffffffffu, cl);
    }
    int nc = c0 > 0 ? warp_count_ge_regs(kr, c0) : kTopkCand + 1;
    uint32_t T = 0;
    if (nc <= kTopkCand) {
      int base = 0;
#pragma unroll
      for (int i = 0; i < kTopkRegKeys; ++i) {
        const bool in = kr[i] >= c0;
        const unsigned msk = __ballot_sync(0xffffffffu, in);
        if (in) cand[base + __popc(msk & lt)] = kr[i];
        base += __popc(msk);
      }
      __syncwarp();
      uint32_t cr[kTopkCand / 32];
#pragma unroll
      for (int i = 0; i < kTopkCand / 32; ++i) {
        const int j = lane + 32 * i;
        cr[i] = j < nc ? cand[j] : 0u;
      }
      __syncwarp();
#pragma unroll 1
      for (int bit = 30; bit >= 0; --bit) {
        const uint32_t c = T | (1u << bit);
        bool ok = c <= c0;  // every c <= c0 has >= want keys above it
        if (!ok) {
          int cnt = 0;
#pragma unroll
          for (int i = 0; i < kTopkCand / 32; ++i) cnt += cr[i] >= c ? 1 : 0;
          ok = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(cnt))) >= want;
        }
        if (ok) T = c;
      }
      int above = 0;
#pragma unroll
      for (int i = 0; i < kTopkCand / 32; ++i) above += cr[i] > T ? 1 : 0;
      th.key = T;
      th.ties = want - static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(above)));
    } else {
#pragma unroll 1
      for (int bit = 30; bit >= 0; --bit) {
        const uint32_t c = T | (1u << bit);
        if (warp_count_ge_regs(kr, c) >= want) T = c;
      }
      th.key = T;
      th.ties = want - warp_count_ge_regs(kr, T + 1u);
    }
  }
  // emission in ascending block order, straight from the registers
  int written = 0, ties_seen = 0;
#pragma unroll
  for (int i = 0; i < kTopkRegKeys; ++i) {
    if (32 * i < n) {
      const int j = 32 * i + lane;
      const bool in = j < n;
      const uint32_t k = kr[i];
      const bool forced = in && (j < n_init || j > cur - n_local);
      const bool tie = in && th.key != 0u && k == th.key;
      const unsigned tie_mask = __ballot_sync(0xffffffffu, tie);
      const int tie_rank = ties_seen + __popc(tie_mask & lt);
      bool take;
      if (th.key == 0u)
        take = forced || (in && k > 0u);
      else
        take = forced || (in && k > th.key && th.key != 0xffffffffu) || (tie && tie_rank < th.ties);
      const unsigned take_mask = __ballot_sync(0xffffffffu, take);
      const int pos = written + __popc(take_mask & lt);
      if (take && pos < topk) out[pos] = j;
      written += __popc(take_mask);
      ties_seen += __popc(tie_mask);
    }
  }
  for (int q = written + lane; q < topk; q += 32) out[q] = -1;
}

// One warp writes the selected blocks of one row, ascending, padded with -1.
// Block j in [0, n) is taken when forced, or key > T, or key == T among the first
// `ties` such keys (ascending j).
__device__ __forceinline__ void warp_emit_selection(const uint32_t* keys, int n, TopkThreshold th, int cur,
                                                    int n_init, int n_local, int topk, int32_t* out) {
  const int lane = threadIdx.x & 31;
  const unsigned lt = (1u << lane) - 1u;
  int written = 0, ties_seen = 0;
  for (int b0 = 0; b0 < n; b0 += 32) {
    const int j = b0 + lane;
    const bool in = j < n;
    const uint32_t k = in ? keys[j] : 0u;
    const bool forced = in && (j < n_init || j > cur - n_local);
    const bool tie = in && th.key != 0u && k == th.key;
    const unsigned tie_mask = __ballot_sync(0xffffffffu, tie);
    const int tie_rank = ties_seen + __popc(tie_mask & lt);
    bool take;
    if (th.key == 0u)
      take = forced || (in && k > 0u);
    else
      take = forced || (in && k > th.key && th.key != 0xffffffffu) || (tie && tie_rank < th.ties);
    const unsigned take_mask = __ballot_sync(0xffffffffu, take);
    const int pos = written + __popc(take_mask & lt);
    if (take && pos < topk) out[pos] = j;
    written += __popc(take_mask);
    ties_seen += __popc(tie_mask);
  }
  for (int q = written + lane; q < topk; q += 32) out[q] = -1;
}

}  // namespace infllmv2
