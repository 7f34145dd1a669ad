// select_decode.cuh -- block scoring and group-shared top-k for one decode token per
// sequence, one thread-block cluster per (sequence, kv-head).
//
// Same rule as prefill (MiniCPM4 summary page s2.1.1 / s2.1.2) for the query at position
// lens[b]-1, which sees every complete semantic kernel of its sequence.  The kernel axis
// is split over the C CTAs of a cluster; CTA c takes a contiguous chunk of whole
// 64-kernel tiles and streams them from HBM with TMA (128-byte swizzle, no multicast):
//   1. per tile, four warps (16 kernels each) compute the 16 x 64 logits with m16n8k16
//      MMAs and keep an online (max, sum of exp2) per head.  Block j pools kernels
//      4j-1 .. 4j+3, so each aligned quad of kernels 4q .. 4q+3 goes into the block max
//      of block q and its last kernel also into that of block q+1 (shared-memory atomic
//      max on an order-preserving integer image of the float);
//   2. after a cluster barrier each CTA forms lse_h from the C partial states and takes
//      the previous CTA's carry into its first block (both read through distributed
//      shared memory, all loads in parallel), computes S(j) = sum_h exp(m_h(j) - lse_h)
//      (or, with logit-sum scoring, sum_h m_h(j)) for its blocks and stores the keys into
//      CTA 0 (with inside pooling block j pools kernels 4j .. 4j+2 only, and no carry);
//   3. CTA 0 finds the k-th largest key by a 32-way radix search (lane l of every warp
//      counts the keys at or above candidate digit l; once the digit's bucket holds at
//      most 32 keys they are ranked directly) and all its threads write the ascending
//      list (prefix sums place ties and outputs).
// No workspace, one launch; reading Kc once bounds it (HBM).
#pragma once
#include <cooperative_groups.h>

#include "common.cuh"
#include "select_prefill.cuh"
#include "topk.cuh"

namespace infllmv2 {

constexpr int kSdConsumers = 4;
constexpr int kSdWarps = kSdConsumers + 1;  // + the TMA producer warp
constexpr int kSdThreads = 32 * kSdWarps;
constexpr int kSdStages = 4;
constexpr int kSdMaxChunk = 2048;  // kernels per CTA at most
constexpr int kSdMaxQuads = kSdMaxChunk / 4;
constexpr int kSdBStride = kSdMaxQuads + 4;  // per-head block-max rows (quads + 1 carry), padded
constexpr int kSdMaxCluster = 16;
// CTA 0's top-k visits the keys slot-major: thread i takes keys i + kSdThreads s.
constexpr int kSdMaxR = (INFLLMV2_MAX_SEQ_LEN / kBlock + kSdThreads - 1) / kSdThreads;
static_assert(kSdStages * kKcTileBytes >= 4 * (INFLLMV2_MAX_SEQ_LEN / kBlock),
              "the block keys of CTA 0 reuse its tile ring");
static_assert(kSdMaxCluster * kSdMaxChunk >= (INFLLMV2_MAX_SEQ_LEN - kKernel) / kStride + 1,
              "a cluster covers the longest sequence");

struct SelDecodeParams {
  const __nv_bfloat16* q;  // [B, Hq, d]
  const int32_t* lens;     // [B]
  int32_t* idx;            // [B, Hkv, 1, topk]
  int B, Hq, Hkv, G, Lmax, NKmax, topk, n_init, n_local;
  int score_mode, pool_mode;  // kScore*, kPool*
  float scale_log2;
};

struct SdSmem {
  uint64_t full[kSdStages], empty[kSdStages];
  float m[kSdConsumers][kGroupRows], l[kSdConsumers][kGroupRows];
  float cm[kGroupRows], cl[kGroupRows];  // this CTA's (max, sum of exp2) per head
  float pm[kSdMaxCluster][kGroupRows], pl[kSdMaxCluster][kGroupRows];  // every CTA's, gathered
  float lse2[kGroupRows];  // log2-sum-exp2 per head over the whole sequence
  float carry[kGroupRows];  // previous CTA's last kernel, for this CTA's first block
  int cnt[2][kSdWarps][32];
  int wc[kSdMaxR][kSdWarps];          // per (slot, warp) counts of the emission
  int sbase[kSdMaxR];                 // flagged keys in earlier slots
  int total;
  unsigned char tflag[kSdMaxR][kSdThreads];  // take flags when tie ranks are needed
  int nlist;
  uint32_t list[32];
  volatile int abort;
};

constexpr size_t sel_decode_smem_bytes() {
  return 1024 + static_cast<size_t>(kSdStages) * kKcTileBytes + static_cast<size_t>(kGroupRows) * kSdBStride * 4 +
         sizeof(SdSmem);
}

// For each lane l: how many of this warp's keys (thread i takes keys i + kSdThreads s,
// s < R) are >= T | l << shift, where the bits of T below shift + w are zero and l < 2^w
// (lanes l >= 2^w count the keys at or above T + 2^(shift + w), the bucket's upper end).
// `first`: lane 0 counts the keys >= 1 instead (the candidates).  Bit-sliced: one
// ballot per digit bit and slot, then a comparison of the lane's digit l against every
// key's digit on the ballot masks.
__device__ __forceinline__ int warp_count_digits(const uint32_t* keys, int n, int R, uint32_t T, int shift, int w,
                                                 bool first) {
  const int lane = threadIdx.x & 31;
  const bool top = shift + w >= 32;  // the digit holds the key's top bits (a shift by 32 is undefined)
  const uint32_t hT = top ? 0u : T >> (shift + w);
  const uint32_t dmask = (1u << w) - 1u;
  int cnt = 0;
#pragma unroll 2
  for (int s = 0; s < R; ++s) {
    const int j = static_cast<int>(threadIdx.x) + kSdThreads * s;
    const uint32_t k = j < n ? keys[j] : 0u;
    const uint32_t hk = top ? 0u : k >> (shift + w);
    const bool in = hk == hT;
    const uint32_t d = (k >> shift) & dmask;
    const unsigned A = __ballot_sync(0xffffffffu, hk > hT);
    unsigned gt = 0u, eq = __ballot_sync(0xffffffffu, in);
#pragma unroll
    for (int i = 4; i >= 0; --i) {
      if (i < w) {
        const unsigned Bi = __ballot_sync(0xffffffffu, in && ((d >> i) & 1u));
        const unsigned tt = eq & Bi;
        const bool one = (lane >> i) & 1;
        gt = one ? gt : (gt | tt);
        eq = one ? tt : (eq & ~Bi);
      }
    }
    int c = __popc(A) + (lane < (1 << w) ? __popc(gt | eq) : 0);
    if (first) {
      const int cand = __popc(__ballot_sync(0xffffffffu, k != 0u));
      if (lane == 0) c = cand;
    }
    cnt += c;
  }
  return cnt;
}

// k-th largest of the n keys in shared memory by all kSdThreads threads; same result as
// warp_radix_threshold.  Radix search on the 32 key bits in digits of 5 (the last one
// 2): lane l of every warp counts the keys >= T | l << shift (warp_count_digits), the
// counts meet in S.cnt (double-buffered: one barrier per digit) and the largest digit
// with at least `want` keys at or above it is taken.  As soon as the chosen digit's
// bucket holds at most 32 keys, they are gathered and ranked directly.
__device__ __forceinline__ TopkThreshold cta_topk_threshold(const uint32_t* keys, int n, int want, SdSmem& S) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int R = (n + kSdThreads - 1) / kSdThreads;
  TopkThreshold r;
  r.all_ties = false;
  if (want <= 0) {
    r.key = 0xffffffffu;
    r.ties = 0;
    return r;
  }
  int buf = 0;
  auto count_ge = [&](uint32_t T, int shift, int w, bool first) -> int {
    S.cnt[buf][warp][lane] = warp_count_digits(keys, n, R, T, shift, w, first);
    __syncthreads();
    int tot = 0;
#pragma unroll
    for (int ww = 0; ww < kSdWarps; ++ww) tot += S.cnt[buf][ww][lane];
    buf ^= 1;
    return tot;
  };
  // first digit (bits 31..27); lane 0 counts the candidates (keys >= 1): bucket 0 is [1, 2^27)
  int tot = count_ge(0u, 27, 5, true);
  if (__shfl_sync(0xffffffffu, tot, 0) <= want) {  // at most `want` candidates: take them all
    r.key = 0;
    r.ties = 0;
    return r;
  }
  uint32_t T = 0;
  int shift = 27, above = 0, inb = 0;  // bucket [max(T, 1), T + 2^shift): `inb` keys, `above` keys above it
  for (;;) {
    const unsigned ok = __ballot_sync(0xffffffffu, tot >= want);  // lane 0 always qualifies
    const int l = 31 - __clz(ok);
    const int nxt = __shfl_sync(0xffffffffu, tot, min(l + 1, 31));
    if (l < 31) above = nxt;
    inb = __shfl_sync(0xffffffffu, tot, l) - above;
    T |= static_cast<uint32_t>(l) << shift;
    if (inb <= 32 || shift == 0) break;
    const int w = shift >= 7 ? 5 : shift;  // 27, 22, 17, 12, 7, 2 (5 bits each), then bits 1..0
    shift -= w;
    tot = count_ge(T, shift, w, false);
  }
  if (shift == 0) {  // the bucket is the single value T
    r.key = T;
    r.ties = want - above;
    r.all_ties = above + inb == want;
    return r;
  }
  // rank the <= 32 keys of the bucket directly: the answer is the (want - above)-th largest
  const uint32_t lo = max(T, 1u), hi = T + (1u << shift);
  if (threadIdx.x == 0) S.nlist = 0;
  __syncthreads();
  for (int j = threadIdx.x; j < n; j += kSdThreads) {
    const uint32_t k = keys[j];
    if (k >= lo && k < hi) S.list[atomicAdd(&S.nlist, 1)] = k;
  }
  __syncthreads();
  const int nl = S.nlist;  // == inb
  const uint32_t x = lane < nl ? S.list[lane] : 0u;
  int gt = 0, ge = 0;
  for (int i = 0; i < nl; ++i) {
    const uint32_t v = S.list[i];
    gt += v > x ? 1 : 0;
    ge += v >= x ? 1 : 0;
  }
  const int rank = want - above;
  const unsigned hit = __ballot_sync(0xffffffffu, lane < nl && gt < rank && rank <= ge);
  const int src = __ffs(hit) - 1;
  r.key = __shfl_sync(0xffffffffu, x, src);
  r.ties = want - above - __shfl_sync(0xffffffffu, gt, src);
  r.all_ties = above + __shfl_sync(0xffffffffu, ge, src) == want;
  return r;
}

// All kSdThreads threads write the selected blocks of one row, ascending, padded with
// -1: block j in [0, n) is taken when forced, or key > T, or key == T among the first
// `ties` such keys in ascending j (the rule of warp_emit_selection).  Keys are visited
// slot-major (thread i, slot s: key i + kSdThreads s), which is ascending j: one pass
// counts the taken keys per (slot, warp) with ballots, a warp scan turns the slot totals
// into slot bases, and a second pass writes each taken key at its base plus its rank in
// the warp and in the slot.  Tie ranks (only when some keys equal to T stay out) come
// from the same two passes run on the tie flags first.
__device__ __forceinline__ void cta_emit_selection(const uint32_t* keys, int n, TopkThreshold th, int cur,
                                                   int n_init, int n_local, int topk, int32_t* out, SdSmem& S) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned lt = (1u << lane) - 1u;
  const int R = (n + kSdThreads - 1) / kSdThreads;
  const bool simple = topk_simple(th);  // no tie ranks needed: take forced or key >= lo
  const uint32_t lo = take_from(th);
  // per (slot, warp) counts of a flag, then S.sbase[s] = flagged keys in slots < s
  auto slot_counts = [&](auto flag) -> int {
    for (int s = 0; s < R; ++s) {
      const unsigned m = __ballot_sync(0xffffffffu, flag(s));
      if (lane == 0) S.wc[s][warp] = __popc(m);
    }
    __syncthreads();
    int total = 0;
    if (warp == 0) {
      int v = 0;
      if (lane < R)
#pragma unroll
        for (int ww = 0; ww < kSdWarps; ++ww) v += S.wc[lane][ww];
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (lane < R) S.sbase[lane] = incl - v;
      if (lane == 31) S.total = incl;
    }
    __syncthreads();
    total = S.total;
    return total;
  };
  auto rank_of = [&](int s, unsigned m) -> int {  // flagged keys before this thread's key of slot s
    int before = S.sbase[s];
#pragma unroll
    for (int ww = 0; ww < kSdWarps; ++ww) before += ww < warp ? S.wc[s][ww] : 0;
    return before + __popc(m & lt);
  };
  auto key_at = [&](int s, int& j) -> uint32_t {
    j = static_cast<int>(threadIdx.x) + kSdThreads * s;
    return j < n ? keys[j] : 0u;
  };
  auto forced = [&](int j) { return j < n && (j < n_init || j > cur - n_local); };
  if (simple) {
    auto take = [&](int s) {
      int j;
      const uint32_t k = key_at(s, j);
      return j < n && (forced(j) || k >= lo);
    };
    const int total = slot_counts(take);
    for (int s = 0; s < R; ++s) {
      const bool f = take(s);
      const int pos = rank_of(s, __ballot_sync(0xffffffffu, f));
      if (f && pos < topk) out[pos] = static_cast<int>(threadIdx.x) + kSdThreads * s;
    }
    for (int e = total + static_cast<int>(threadIdx.x); e < topk; e += kSdThreads) out[e] = -1;
    __syncthreads();  // S.wc, S.sbase are free again
    return;
  }
  // tie ranks first: S.tie_base[s] + warp part, recomputed per slot below
  auto tie = [&](int s) {
    int j;
    const uint32_t k = key_at(s, j);
    return j < n && k == th.key;
  };
  slot_counts(tie);
  for (int s = 0; s < R; ++s) {  // keep each slot's tie base for this thread's warp
    const bool f = tie(s);
    const int rk = rank_of(s, __ballot_sync(0xffffffffu, f));
    int j;
    const uint32_t k = key_at(s, j);
    S.tflag[s][threadIdx.x] = static_cast<unsigned char>(
        j < n && (forced(j) || k > th.key || (k == th.key && rk < th.ties)) ? 1 : 0);
  }
  __syncthreads();
  auto take = [&](int s) { return S.tflag[s][threadIdx.x] != 0; };
  const int total = slot_counts(take);
  for (int s = 0; s < R; ++s) {
    const bool f = take(s);
    const int pos = rank_of(s, __ballot_sync(0xffffffffu, f));
    if (f && pos < topk) out[pos] = static_cast<int>(threadIdx.x) + kSdThreads * s;
  }
  for (int e = total + static_cast<int>(threadIdx.x); e < topk; e += kSdThreads) out[e] = -1;
  __syncthreads();
}

// grid = C * B * Hkv (cluster r serves item r), cluster = (C, 1, 1), block = 160.
__global__ void __launch_bounds__(kSdThreads)
    select_decode_kernel(const __grid_constant__ CUtensorMap tm_kc, const SelDecodeParams p) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ unsigned char smem_raw[];
  unsigned char* ring = align_smem(smem_raw, 1024);
  uint32_t* bm = reinterpret_cast<uint32_t*>(ring + kSdStages * kKcTileBytes);  // [16][kSdBStride], ord_enc
  SdSmem& S = *reinterpret_cast<SdSmem*>(bm + kGroupRows * kSdBStride);
  uint32_t* keys = reinterpret_cast<uint32_t*>(ring);  // CTA 0 only, once every tile is consumed

  const int C = static_cast<int>(cluster.num_blocks());
  const int c = static_cast<int>(cluster.block_rank());
  const long long bg = blockIdx.x / C;  // clusters are consecutive blocks
  const int b = static_cast<int>(bg / p.Hkv), g = static_cast<int>(bg % p.Hkv);
  allow_dependent_launch();  // the decode attention may set up while this selection runs
  grid_dependency_wait();    // q, Kc and lens may come from the previous kernel
  const int n = min(max(p.lens[b], 0), p.Lmax);
  const int nk = n >= kKernel ? (n - kKernel) / kStride + 1 : 0;
  const int cur = n > 0 ? (n - 1) / kBlock : -1;
  const int chunk = ((nk + C - 1) / C + kKcTile - 1) / kKcTile * kKcTile;  // kernels per CTA
  const int nq = chunk / 4;                                                 // blocks per CTA
  const int k0 = c * chunk;
  const int ntiles = nk > k0 ? (min(chunk, nk - k0) + kKcTile - 1) / kKcTile : 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSdStages; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], kSdConsumers);
    }
    S.abort = 0;
    fence_mbar_init();
  }
  // bm[h][q]: max over this CTA's kernels 4q-1 .. 4q+3 (local numbering); q = nq holds
  // the chunk's last kernel, carried into the next CTA's first block
  for (int e = threadIdx.x; e < kGroupRows * (nq + 1); e += kSdThreads)
    bm[(e / (nq + 1)) * kSdBStride + e % (nq + 1)] = ord_enc(-INFINITY);
  __syncthreads();

  if (warp == kSdConsumers) {
    // ---------------------------------------------------------------- producer
    if (lane == 0 && ntiles > 0) {
      prefetch_tmap(&tm_kc);
      const int row0 = static_cast<int>(bg * p.NKmax) + k0;
      int i = 0;
      for (; i < ntiles; ++i) {
        const int st = i % kSdStages, u = i / kSdStages;
        if (u > 0 && !mbar_wait(&S.empty[st], (u - 1) & 1, &S.abort)) break;
        unsigned char* dst = ring + st * kKcTileBytes;
        mbar_arrive_expect_tx(&S.full[st], kKcTileBytes);
        tma_load_2d(dst, &tm_kc, &S.full[st], 0, row0 + i * kKcTile);
        tma_load_2d(dst + kKcTileBytes / 2, &tm_kc, &S.full[st], 64, row0 + i * kKcTile);
      }
      if (S.abort) {  // let every issued copy land before the ring is reused or released
        for (int j = max(0, i - kSdStages); j < i; ++j) mbar_wait_drain(&S.full[j % kSdStages], (j / kSdStages) & 1);
      }
    }
  } else {
    // ------------------------------------------------------------ consumer warps
    const int q4 = lane & 3, r0 = lane >> 2;
    const int kofs = 16 * warp;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    if (ntiles > 0) {
      uint32_t qa[8][4];
      load_q_frags(p.q + (static_cast<long long>(b) * p.Hq + g * p.G) * kHeadDim, p.G, qa);
      for (int i = 0; i < ntiles; ++i) {
        const int st = i % kSdStages;
        if (!mbar_wait(&S.full[st], (i / kSdStages) & 1, &S.abort)) break;
        const uint32_t tile = smem_u32(ring + st * kKcTileBytes);
        float s[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const int mi = lane >> 3;
          const int row = kofs + (lane & 7) + ((mi >> 1) << 3);
          const int d = 16 * ks + ((mi & 1) << 3);
          uint32_t b0, b1, b2, b3;
          ldsm_x4(tile + (d >> 6) * (kKcTileBytes / 2) + sw128(row, (d & 63) >> 3), b0, b1, b2, b3);
          mma_bf16(s[0], qa[ks], b0, b1);
          mma_bf16(s[1], qa[ks], b2, b3);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.empty[st]);

        const int kb = k0 + i * kKcTile + kofs;  // first kernel of this warp's 16
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const bool ok = kb + 8 * nt + 2 * q4 + e < nk;
            s[nt][e] = ok ? s[nt][e] * p.scale_log2 : -INFINITY;
            s[nt][2 + e] = ok ? s[nt][2 + e] * p.scale_log2 : -INFINITY;
            mx0 = fmaxf(mx0, s[nt][e]);
            mx1 = fmaxf(mx1, s[nt][2 + e]);
          }
        }
        // quad q (lanes q4 = 0, 2 of n-tile nt: quads 2 nt, 2 nt + 1 of the warp's four):
        // its max feeds block q, its last kernel block q + 1 (overlap pooling); with inside
        // pooling only kernels 4q .. 4q+2 feed block q and the last kernel no block
        const bool inside = p.pool_mode == kPoolInside;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const bool drop_last = inside && (q4 & 1);  // this lane's second kernel is 4q+3
          const float pm0 = drop_last ? s[nt][0] : fmaxf(s[nt][0], s[nt][1]);
          const float pm1 = drop_last ? s[nt][2] : fmaxf(s[nt][2], s[nt][3]);
          const float om0 = __shfl_xor_sync(0xffffffffu, pm0, 1), om1 = __shfl_xor_sync(0xffffffffu, pm1, 1);
          const float la0 = __shfl_xor_sync(0xffffffffu, s[nt][1], 1);
          const float la1 = __shfl_xor_sync(0xffffffffu, s[nt][3], 1);
          if ((q4 & 1) == 0) {
            const int qd = (i * kKcTile + kofs + 8 * nt + 4 * (q4 >> 1)) >> 2;
            atomicMax(&bm[r0 * kSdBStride + qd], ord_enc(fmaxf(pm0, om0)));
            atomicMax(&bm[(r0 + 8) * kSdBStride + qd], ord_enc(fmaxf(pm1, om1)));
            if (!inside) {
              atomicMax(&bm[r0 * kSdBStride + qd + 1], ord_enc(la0));
              atomicMax(&bm[(r0 + 8) * kSdBStride + qd + 1], ord_enc(la1));
            }
          }
        }
        // online (max, sum of exp2) per head
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        if (mn0 != -INFINITY) {
          l0 = l0 * ex2(m0 - mn0) + ((ex2(s[0][0] - mn0) + ex2(s[0][1] - mn0)) +
                                     (ex2(s[1][0] - mn0) + ex2(s[1][1] - mn0)));
          m0 = mn0;
        }
        if (mn1 != -INFINITY) {
          l1 = l1 * ex2(m1 - mn1) + ((ex2(s[0][2] - mn1) + ex2(s[0][3] - mn1)) +
                                     (ex2(s[1][2] - mn1) + ex2(s[1][3] - mn1)));
          m1 = mn1;
        }
      }
    }
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    if (q4 == 0) {
      S.m[warp][r0] = m0;
      S.m[warp][r0 + 8] = m1;
      S.l[warp][r0] = l0;
      S.l[warp][r0 + 8] = l1;
    }
  }
  __syncthreads();
  if (threadIdx.x < kGroupRows) {
    const int h = threadIdx.x;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kSdConsumers; ++w) M = fmaxf(M, S.m[w][h]);
    float L = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kSdConsumers; ++w) L += S.l[w][h] * ex2(S.m[w][h] - M);
    }
    S.cm[h] = M;
    S.cl[h] = L;
  }
  cluster.sync();  // every CTA's tiles are consumed and its partial state is final

  // gather every CTA's (max, sum) and the previous CTA's carry, all loads in flight at once
  for (int e = threadIdx.x; e < kGroupRows * C; e += kSdThreads) {
    const int r = e / kGroupRows, h = e % kGroupRows;
    S.pm[r][h] = cluster.map_shared_rank(&S.cm[0], r)[h];
    S.pl[r][h] = cluster.map_shared_rank(&S.cl[0], r)[h];
  }
  if (threadIdx.x >= kSdThreads - kGroupRows) {
    const int h = threadIdx.x - (kSdThreads - kGroupRows);
    S.carry[h] = c > 0 ? ord_dec(cluster.map_shared_rank(bm, c - 1)[h * kSdBStride + nq]) : -INFINITY;
  }
  if (c == 0) {  // zero padding up to a multiple of 4 keys for the vector scan
    for (int j = cur + 1 + threadIdx.x; j < ((cur + 4) & ~3); j += kSdThreads) keys[j] = 0u;
  }
  __syncthreads();
  if (threadIdx.x < kGroupRows) {
    const int h = threadIdx.x;
    float M = -INFINITY;
    for (int r = 0; r < C; ++r) M = fmaxf(M, S.pm[r][h]);
    float L = 0.f;
    if (M != -INFINITY) {
      for (int r = 0; r < C; ++r) L += S.pl[r][h] * ex2(S.pm[r][h] - M);
    }
    S.lse2[h] = L > 0.f ? M + lg2(L) : INFINITY;
  }
  __syncthreads();
  // this CTA's blocks: [c nq, (c + 1) nq); the last CTA also takes the rest up to cur
  {
    uint32_t* keys0 = cluster.map_shared_rank(keys, 0);
    const int jb0 = c * nq;
    const int jb1 = c == C - 1 ? cur + 1 : min(jb0 + nq, cur + 1);
    for (int j = jb0 + threadIdx.x; j < jb1; j += kSdThreads) {
      const int ql = j - jb0;  // <= nq, since cur + 1 <= ceil(nk / 4) + 1 <= C nq + 1
      const bool eligible = block_eligible(j, nk - 1, p.pool_mode);
      const bool forced = j < p.n_init || j > cur - p.n_local;
      uint32_t key = 0u;
      if (eligible && !forced && ql <= nq) {
        float sc = 0.f;
        for (int h = 0; h < p.G; ++h) {
          float mb = ord_dec(bm[h * kSdBStride + ql]);
          if (ql == 0 && p.pool_mode == kPoolOverlap) mb = fmaxf(mb, S.carry[h]);
          sc += p.score_mode == kScoreLogitSum ? mb : ex2(mb - S.lse2[h]);
        }
        key = score_key(sc, p.score_mode);
      }
      keys0[j] = key;
    }
  }
  cluster.sync();  // CTA 0 holds every key; no CTA reads a peer's shared memory after this
  if (c != 0) return;

  int32_t* out = p.idx + bg * p.topk;
  if (cur < 0) {
    for (int e = threadIdx.x; e < p.topk; e += kSdThreads) out[e] = -1;
    return;
  }
  const int want = p.topk - forced_count(cur, p.n_init, p.n_local);
  const TopkThreshold th = cta_topk_threshold(keys, cur + 1, want, S);
  cta_emit_selection(keys, cur + 1, th, cur, p.n_init, p.n_local, p.topk, out, S);
}

}  // namespace infllmv2
