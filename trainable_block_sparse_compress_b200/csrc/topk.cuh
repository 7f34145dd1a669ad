// topk.cuh -- deterministic top-k of block scores and ordered emission of the
// selected block list.
//
// Ordering rule (MiniCPM4 summary page s2.1.1: each query token keeps its highest
// scoring blocks): higher score first, lower block index first among equal scores.
// Scores are non-negative fp32 group sums, so their IEEE bit patterns order like the
// values.  A candidate's key is bits(score) + 1 and a non-candidate's key is 0.
// The k-th largest key is found by a most-significant-digit radix select (4 rounds of
// 8 bits, shared-memory histogram); the list is then written in ascending block order
// with forced blocks first-class members and ties at the threshold taken from the
// lowest indices.
#pragma once
#include "common.cuh"

namespace infllmv2 {

struct TopkThreshold {
  uint32_t key;  // threshold key T (0xffffffff when nothing is to be taken)
  int ties;      // how many keys equal to T are taken (0 when T == 0: take all > 0)
};

// One warp.  keys[0..n) in shared memory; `want` keys to take; hist: 256 words of
// shared scratch owned by this warp.
__device__ __forceinline__ TopkThreshold warp_radix_threshold(const uint32_t* keys, int n, int want,
                                                              uint32_t* hist) {
  const int lane = threadIdx.x & 31;
  TopkThreshold r;
  if (want <= 0) {
    r.key = 0xffffffffu;
    r.ties = 0;
    return r;
  }
  uint32_t prefix = 0, pmask = 0;
  int need = want;
#pragma unroll 1
  for (int shift = 24; shift >= 0; shift -= 8) {
#pragma unroll
    for (int e = 0; e < 8; ++e) hist[lane * 8 + e] = 0;
    __syncwarp();
    for (int i = lane; i < n; i += 32) {
      const uint32_t k = keys[i];
      if ((k & pmask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1u);
    }
    __syncwarp();
    // lane L owns bins 255-8L .. 248-8L (descending)
    uint32_t cnt[8];
    uint32_t tot = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      cnt[e] = hist[255 - 8 * lane - e];
      tot += cnt[e];
    }
    uint32_t incl = tot;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    const uint32_t excl = incl - tot;
    const uint32_t all = __shfl_sync(0xffffffffu, incl, 31);
    if (all < static_cast<uint32_t>(need)) {  // fewer keys than wanted (first round only)
      r.key = 0;
      r.ties = 0;
      __syncwarp();
      return r;
    }
    const bool mine = excl < static_cast<uint32_t>(need) && static_cast<uint32_t>(need) <= incl;
    const unsigned owner_mask = __ballot_sync(0xffffffffu, mine);
    const int owner = __ffs(owner_mask) - 1;
    int digit = 0;
    uint32_t above = 0;
    if (mine) {
      uint32_t c = excl;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        if (c + cnt[e] >= static_cast<uint32_t>(need)) {
          digit = 255 - 8 * lane - e;
          above = c;
          break;
        }
        c += cnt[e];
      }
    }
    digit = __shfl_sync(0xffffffffu, digit, owner);
    above = __shfl_sync(0xffffffffu, above, owner);
    need -= static_cast<int>(above);
    prefix |= static_cast<uint32_t>(digit) << shift;
    pmask |= 255u << shift;
    __syncwarp();
  }
  r.key = prefix;
  r.ties = prefix == 0 ? 0 : need;
  return r;
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
