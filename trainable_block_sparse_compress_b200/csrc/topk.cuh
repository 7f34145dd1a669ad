// topk.cuh -- deterministic top-k of block scores and ordered emission of the
// selected block list.
//
// Ordering rule (MiniCPM4 summary page s2.1.1: each query token keeps its highest
// scoring blocks): higher score first, lower block index first among equal scores.
// A candidate's key is a nonzero uint32 that orders like its score (score_key) and a
// non-candidate's key is 0; all 32 key bits may be in use.
// The k-th largest key T is found either by sorting a prefiltered candidate set
// (warp_topk_select) or by bisection on the key bits with warp-wide counts; the list is
// then written in ascending block order with forced blocks first-class members and
// ties at the threshold taken from the lowest indices.  When every key equal to T is
// taken (the usual case: no duplicate straddles the cut), a block is taken exactly when
// forced or key >= T, and the emission needs no tie ranks.
#pragma once
#include "common.cuh"

namespace infllmv2 {

struct TopkThreshold {
  uint32_t key;   // threshold key T (0xffffffff when nothing is to be taken)
  int ties;       // how many keys equal to T are taken (0 when T == 0: take all > 0)
  bool all_ties;  // every key equal to T is taken
};

// Smallest key taken without a tie rank: every key >= take_from(th) is taken when
// th.all_ties, T == 0 (all candidates) or T == 0xffffffff (none: keys stay below it).
__device__ __forceinline__ bool topk_simple(const TopkThreshold& th) {
  return th.all_ties || th.key == 0u || th.key == 0xffffffffu;
}
__device__ __forceinline__ uint32_t take_from(const TopkThreshold& th) { return th.key == 0u ? 1u : th.key; }

// One warp.  keys[0..n) in shared memory; `want` keys to take.  Finds the want-th
// largest key T by bisection on its 32 bits, most significant first: T >= c exactly when
// at least `want` keys are >= c.  Each lane holds up to kTopkRegKeys keys in registers
// (n <= 32 * kTopkRegKeys); larger n re-reads shared memory each step.  No atomics.
constexpr int kTopkRegKeys = 64;
constexpr int kTopkVoteBatch = 16;  // ballots issued back to back before their stores

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
  r.all_ties = false;
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
    for (int bit = 31; bit >= 0; --bit) {
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
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t c = T | (1u << bit);
    if (warp_count_ge_smem(keys, n, c) >= want) T = c;
  }
  r.key = T;
  r.ties = want - warp_count_ge_smem(keys, n, T + 1u);
  return r;
}

// Descending bitonic sort of 256 keys held 8 per lane (element i = 8 lane + e): 36
// compare-exchange stages, the 21 with stride < 8 inside a lane, the 15 others across
// lanes by shuffles.
__device__ __forceinline__ void warp_bitonic256_desc(uint32_t (&a)[8]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int k = 2; k <= 256; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      if (j >= 8) {
        const int lj = j >> 3;
        const bool keep_max = ((lane & lj) == 0) == (((lane * 8) & k) == 0);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint32_t b = __shfl_xor_sync(0xffffffffu, a[e], lj);
          a[e] = keep_max ? max(a[e], b) : min(a[e], b);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if ((e & j) == 0) {
            const int f = e | j;
            const bool up = (((lane * 8) + e) & k) == 0;
            const uint32_t x = a[e], y = a[f];
            a[e] = up ? max(x, y) : min(x, y);
            a[f] = up ? min(x, y) : max(x, y);
          }
        }
      }
    }
  }
}

// One warp writes the selected blocks of one row, ascending, padded with -1, from keys
// held in registers (key j = kr[i] with j = 32 i + lane, j < n).  Block j is taken when
// forced, or key > T, or key == T among the first `ties` such keys (ascending j).
__device__ __forceinline__ void warp_emit_regs(const uint32_t (&kr)[kTopkRegKeys], int n, const TopkThreshold& th,
                                               int cur, int n_init, int n_local, int topk, int32_t* out) {
  const int lane = threadIdx.x & 31;
  const unsigned lt = (1u << lane) - 1u;
  int written = 0;
  if (topk_simple(th)) {
    // 16 ballots first, then their stores: the votes pipeline instead of alternating
    // with dependent stores
    const uint32_t lo = take_from(th);
#pragma unroll
    for (int g = 0; g < kTopkRegKeys; g += kTopkVoteBatch) {
      if (32 * g < n) {
        unsigned m[kTopkVoteBatch];
#pragma unroll
        for (int u = 0; u < kTopkVoteBatch; ++u) {
          const int j = 32 * (g + u) + lane;
          m[u] = __ballot_sync(0xffffffffu, j < n && (j < n_init || j > cur - n_local || kr[g + u] >= lo));
        }
#pragma unroll
        for (int u = 0; u < kTopkVoteBatch; ++u) {
          const int pos = written + __popc(m[u] & lt);
          if (((m[u] >> lane) & 1u) && pos < topk) out[pos] = 32 * (g + u) + lane;
          written += __popc(m[u]);
        }
      }
    }
  } else {
    int ties_seen = 0;
#pragma unroll
    for (int i = 0; i < kTopkRegKeys; ++i) {
      if (32 * i < n) {
        const int j = 32 * i + lane;
        const bool in = j < n;
        const uint32_t k = kr[i];
        const bool forced = in && (j < n_init || j > cur - n_local);
        const bool tie = in && k == th.key;
        const unsigned tie_mask = __ballot_sync(0xffffffffu, tie);
        const int tie_rank = ties_seen + __popc(tie_mask & lt);
        const bool take = forced || (in && k > th.key) || (tie && tie_rank < th.ties);
        const unsigned take_mask = __ballot_sync(0xffffffffu, take);
        const int pos = written + __popc(take_mask & lt);
        if (take && pos < topk) out[pos] = j;
        written += __popc(take_mask);
        ties_seen += __popc(tie_mask);
      }
    }
  }
  for (int q = written + lane; q < topk; q += 32) out[q] = -1;
}

// One warp: threshold and ordered emission for n <= 32 * kTopkRegKeys keys, with the
// keys held in registers.  The search is narrowed first: every lane keeps its 4 largest
// keys; with r = ceil(want / 32) <= 4, c0 = the warp minimum of the lanes' r-th largest
// keys bounds the threshold from below (each lane holds r keys >= c0, so at least
// 32 r >= want keys are >= c0).  The keys >= c0 (usually a few hundred) are compacted
// into `cand` (kTopkCand words of this warp's shared scratch) and sorted; T is the
// want-th of them.  When the bound does not apply or too many keys pass it, T comes from
// bisection over all keys.  Same result either way: the want-th largest key.
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
  th.all_ties = false;
  if (want <= 0) {
    th.key = 0xffffffffu;
    th.ties = 0;
  } else {
    // per-lane top 4 and candidate count in one pass: four independent insertion chains
    // (keys i % 4), merged at the end
    const int r = (want + 31) / 32;
    uint32_t tt[4][4];
    int cc[4] = {0, 0, 0, 0};
#pragma unroll
    for (int c = 0; c < 4; ++c) tt[c][0] = tt[c][1] = tt[c][2] = tt[c][3] = 0u;
#pragma unroll
    for (int i = 0; i < kTopkRegKeys; ++i) {
      const int c = i & 3;
      uint32_t x = kr[i], y;
      cc[c] += x != 0u ? 1 : 0;
      y = max(x, tt[c][0]); x = min(x, tt[c][0]); tt[c][0] = y;
      y = max(x, tt[c][1]); x = min(x, tt[c][1]); tt[c][1] = y;
      y = max(x, tt[c][2]); x = min(x, tt[c][2]); tt[c][2] = y;
      tt[c][3] = max(x, tt[c][3]);
    }
    // top 4 of two descending 4-lists: the elementwise max of one list and the other
    // reversed is a bitonic sequence holding the 4 largest; two exchange steps sort it
    auto merge4 = [](const uint32_t (&a)[4], const uint32_t (&b)[4], uint32_t (&o)[4]) {
      uint32_t m0 = max(a[0], b[3]), m1 = max(a[1], b[2]), m2 = max(a[2], b[1]), m3 = max(a[3], b[0]);
      uint32_t x = max(m0, m2), y = min(m0, m2);
      m0 = x;
      m2 = y;
      x = max(m1, m3);
      y = min(m1, m3);
      m1 = x;
      m3 = y;
      o[0] = max(m0, m1);
      o[1] = min(m0, m1);
      o[2] = max(m2, m3);
      o[3] = min(m2, m3);
    };
    uint32_t ua[4], ub[4], tf[4];
    merge4(tt[0], tt[1], ua);
    merge4(tt[2], tt[3], ub);
    merge4(ua, ub, tf);
    const uint32_t t0 = tf[0], t1 = tf[1], t2 = tf[2], t3 = tf[3];
    const int c1 = (cc[0] + cc[1]) + (cc[2] + cc[3]);
    const int ncand = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(c1)));
    if (ncand <= want) {  // at most `want` candidates: take them all
      th.key = 0;
      th.ties = 0;
    } else {
      uint32_t c0 = 0;
      if (r <= 4) c0 = __reduce_min_sync(0xffffffffu, r == 1 ? t0 : (r == 2 ? t1 : (r == 3 ? t2 : t3)));
      int nc = kTopkCand + 1;
      if (c0 > 0) {
        int base = 0;
#pragma unroll
        for (int g = 0; g < kTopkRegKeys; g += kTopkVoteBatch) {
          unsigned m[kTopkVoteBatch];
#pragma unroll
          for (int u = 0; u < kTopkVoteBatch; ++u) m[u] = __ballot_sync(0xffffffffu, kr[g + u] >= c0);
#pragma unroll
          for (int u = 0; u < kTopkVoteBatch; ++u) {
            const int pos = base + __popc(m[u] & lt);
            if (((m[u] >> lane) & 1u) && pos < kTopkCand) cand[pos] = kr[g + u];
            base += __popc(m[u]);
          }
        }
        nc = base;
        __syncwarp();
      }
      if (nc <= kTopkCand) {
        uint32_t a[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int idx = 8 * lane + e;
          a[e] = idx < nc ? cand[idx] : 0u;
        }
        __syncwarp();
        warp_bitonic256_desc(a);
        const int wl = (want - 1) >> 3, we = (want - 1) & 7;
        uint32_t v = a[0];
#pragma unroll
        for (int e = 1; e < 8; ++e) v = e == we ? a[e] : v;
        const uint32_t T = __shfl_sync(0xffffffffu, v, wl);
        int above = 0, eq = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          above += a[e] > T ? 1 : 0;
          eq += a[e] == T ? 1 : 0;
        }
        above = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(above)));
        eq = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(eq)));
        th.key = T;
        th.ties = want - above;
        th.all_ties = above + eq == want;
      } else {
        // bisection between the bound c0 <= T and the largest key: the bits above their
        // highest differing bit are T's too
        const uint32_t kmax = __reduce_max_sync(0xffffffffu, t0);
        const int top = (kmax ^ c0) == 0u ? -1 : 31 - __clz(kmax ^ c0);
        uint32_t T = top >= 31 ? 0u : (kmax >> (top + 1)) << (top + 1);
#pragma unroll 1
        for (int bit = top; bit >= 0; --bit) {
          const uint32_t c = T | (1u << bit);
          if (warp_count_ge_regs(kr, c) >= want) T = c;
        }
        th.key = T;
        th.ties = want - warp_count_ge_regs(kr, T + 1u);
      }
    }
  }
  warp_emit_regs(kr, n, th, cur, n_init, n_local, topk, out);
}

// One warp writes the selected blocks of one row, ascending, padded with -1.
// Block j in [0, n) is taken when forced, or key > T, or key == T among the first
// `ties` such keys (ascending j).
__device__ __forceinline__ void warp_emit_selection(const uint32_t* keys, int n, TopkThreshold th, int cur,
                                                    int n_init, int n_local, int topk, int32_t* out) {
  const int lane = threadIdx.x & 31;
  const unsigned lt = (1u << lane) - 1u;
  const bool simple = topk_simple(th);
  const uint32_t lo = take_from(th);
  int written = 0, ties_seen = 0;
  for (int b0 = 0; b0 < n; b0 += 32) {
    const int j = b0 + lane;
    const bool in = j < n;
    const uint32_t k = in ? keys[j] : 0u;
    const bool forced = in && (j < n_init || j > cur - n_local);
    bool take;
    if (simple) {
      take = forced || (in && k >= lo);
    } else {
      const bool tie = in && k == th.key;
      const unsigned tie_mask = __ballot_sync(0xffffffffu, tie);
      const int tie_rank = ties_seen + __popc(tie_mask & lt);
      take = forced || (in && k > th.key) || (tie && tie_rank < th.ties);
      ties_seen += __popc(tie_mask);
    }
    const unsigned take_mask = __ballot_sync(0xffffffffu, take);
    const int pos = written + __popc(take_mask & lt);
    if (take && pos < topk) out[pos] = j;
    written += __popc(take_mask);
  }
  for (int q = written + lane; q < topk; q += 32) out[q] = -1;
}

}  // namespace infllmv2
