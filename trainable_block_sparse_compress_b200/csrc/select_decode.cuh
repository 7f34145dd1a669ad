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
//      CTA 0 -- in the fused decode step into every CTA of the cluster -- (with inside
//      pooling block j pools kernels 4j .. 4j+2 only, and no carry);
//   3. a CTA that holds every key finds the k-th largest: the candidates' common leading
//      bits come from one AND / OR reduction, the bits below them from shared-memory
//      histograms of 11-bit digits (a suffix scan picks the digit that holds the k-th key;
//      once its bucket holds at most 32 keys they are ranked directly), and all its
//      threads write the ascending list (one scan places ties and outputs).
// The phases are device functions: select_decode_kernel runs them alone, the fused decode
// step (decode_step.cuh) runs them before the attention in the same cluster.
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
constexpr int kSdMaxKeys = INFLLMV2_MAX_SEQ_LEN / kBlock;
constexpr int kSdHistBits = 11;  // digit width of the threshold search
constexpr int kSdHistBins = 1 << kSdHistBits;
constexpr int kSdBinsPerThread = (kSdHistBins + kSdThreads - 1) / kSdThreads;
// The selection scratch of a CTA that selects, in its drained tile ring: block keys and
// the digit histogram
constexpr int kSdKeysOff = 0;
constexpr int kSdHistOff = kSdKeysOff + 4 * kSdMaxKeys;
constexpr int kSdScratchBytes = kSdHistOff + 4 * kSdHistBins;
static_assert(kSdStages * kKcTileBytes >= kSdScratchBytes, "the selection scratch reuses the tile ring");
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
  int kcnt;                    // a selecting CTA: candidates among the keys, and the AND / OR of
  unsigned int kand, kor;      // their keys (every CTA adds its blocks' through DSMEM)
  int wsum[kSdWarps];          // per-warp histogram totals of the digit search
  int dig, dig_above, dig_in;  // the digit found, keys above its bin, keys in it
  int wc[2][kSdWarps];         // per-warp counts of the emission (strict takes, ties)
  int nlist;
  uint32_t list[32];
  volatile int abort;
};

// Tile ring (reused as the selection scratch) and per-head block maxima.
constexpr size_t kSdRegionBytes =
    static_cast<size_t>(kSdStages) * kKcTileBytes + static_cast<size_t>(kGroupRows) * kSdBStride * 4;

constexpr size_t sel_decode_smem_bytes() { return 1024 + kSdRegionBytes + sizeof(SdSmem); }

// One (sequence, kv-head) item of a decode-selection cluster and this CTA's share of it.
struct SdItem {
  int C, c;  // cluster size and rank
  long long bg;
  int b, g;
  int n, nk, cur;  // sequence length (clamped), complete kernels, current block (-1: empty)
  int chunk, nq;   // kernels and blocks per CTA
  int k0, ntiles;  // this CTA's first kernel and Kc tiles
};

// n: the sequence's length, clamped to [0, Lmax] by the caller.
__device__ __forceinline__ SdItem sd_item(const SelDecodeParams& p, int C, int c, long long bg, int n) {
  SdItem it;
  it.C = C;
  it.c = c;
  it.bg = bg;
  it.b = static_cast<int>(bg / p.Hkv);
  it.g = static_cast<int>(bg % p.Hkv);
  it.n = n;
  it.nk = it.n >= kKernel ? (it.n - kKernel) / kStride + 1 : 0;
  it.cur = it.n > 0 ? (it.n - 1) / kBlock : -1;
  it.chunk = ((it.nk + C - 1) / C + kKcTile - 1) / kKcTile * kKcTile;
  it.nq = it.chunk / 4;
  it.k0 = c * it.chunk;
  it.ntiles = it.nk > it.k0 ? (min(it.chunk, it.nk - it.k0) + kKcTile - 1) / kKcTile : 0;
  return it;
}

// k-th largest of the n keys in shared memory (0: not a candidate) by all kSdThreads
// threads; same result as warp_radix_threshold.  The candidates' count and the AND and OR
// of their keys (S.kcnt, S.kand, S.kor) arrive with the keys: the bits above the highest
// bit where the candidates differ are common to all of them.  Below it the threshold is resolved in digits of up to
// kSdHistBits bits: a shared-memory histogram of the digit over the keys of the current
// bucket (keys that agree with the threshold on every bit above the digit), then a
// suffix scan over the bins finds the digit whose bin holds the (want - above)-th
// largest key.  As soon as that bin holds at most 32 keys they are ranked directly.
__device__ __forceinline__ TopkThreshold cta_topk_threshold(const uint32_t* keys, int n, int want, uint32_t* hist,
                                                            SdSmem& S) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  TopkThreshold r;
  r.all_ties = false;
  if (want <= 0) {
    r.key = 0xffffffffu;
    r.ties = 0;
    return r;
  }
  const int cnt = S.kcnt;  // gathered while the keys were stored (sd_block_keys)
  const uint32_t kand = S.kand, kor = S.kor;
  if (cnt <= want) {  // at most `want` candidates: take them all
    r.key = 0;
    r.ties = 0;
    return r;
  }
  if (kand == kor) {  // every candidate has the same key
    r.key = kand;
    r.ties = want;
    return r;
  }
  int top = 31 - __clz(kand ^ kor);  // highest bit in which candidates differ
  uint32_t T = top == 31 ? 0u : (kand >> (top + 1)) << (top + 1);  // the common bits above it
  int above = 0;                      // candidates above the current bucket
  int shift = 0, inb = 0;
  for (int round = 0;; ++round) {
    const int w = min(kSdHistBits, top + 1);
    shift = top + 1 - w;
    const int nb = 1 << w;
    if (round > 0) {  // the first round's bins were zeroed while the keys were stored
      for (int i = tid; i < nb; i += kSdThreads) hist[i] = 0u;
      __syncthreads();
    }
    for (int j = tid; j < n; j += kSdThreads) {
      const uint32_t k = keys[j];
      const bool in = k != 0u && (top == 31 || (k >> (top + 1)) == (T >> (top + 1)));
      if (in) atomicAdd(&hist[(k >> shift) & static_cast<uint32_t>(nb - 1)], 1u);
    }
    __syncthreads();
    // thread i owns bins [i B, i B + B); `higher` counts the keys in the bins of the
    // threads above it, so the bin of the (need)-th largest key is in the thread with
    // higher < need <= higher + own
    const int need = want - above;
    const int b0 = tid * kSdBinsPerThread;
    int hv[kSdBinsPerThread];
    int own = 0;
#pragma unroll
    for (int e = 0; e < kSdBinsPerThread; ++e) {
      hv[e] = b0 + e < nb ? static_cast<int>(hist[b0 + e]) : 0;
      own += hv[e];
    }
    int incl = own;  // this lane's and the higher lanes' bins
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_down_sync(0xffffffffu, incl, o);
      if (lane + o < 32) incl += y;
    }
    if (lane == 0) S.wsum[warp] = incl;
    __syncthreads();
    int higher = incl - own;
#pragma unroll
    for (int ww = 0; ww < kSdWarps; ++ww) higher += ww > warp ? S.wsum[ww] : 0;
    if (higher < need && need <= higher + own) {
      int acc = higher, found = -1, fa = 0, fi = 0;
#pragma unroll
      for (int e = kSdBinsPerThread - 1; e >= 0; --e) {
        if (found < 0 && acc + hv[e] >= need) {
          found = b0 + e;
          fa = acc;
          fi = hv[e];
        }
        acc += hv[e];
      }
      S.dig = found;
      S.dig_above = fa;
      S.dig_in = fi;
    }
    __syncthreads();
    T |= static_cast<uint32_t>(S.dig) << shift;
    above += S.dig_above;
    inb = S.dig_in;
    if (shift == 0 || inb <= 32) break;
    top = shift - 1;
  }
  if (shift == 0) {  // the bucket is the single value T
    r.key = T;
    r.ties = want - above;
    r.all_ties = above + inb == want;
    return r;
  }
  // rank the <= 32 keys of the bucket directly: the answer is the (want - above)-th largest
  const uint32_t lo = max(T, 1u), hi = T + (1u << shift);
  if (tid == 0) S.nlist = 0;
  __syncthreads();
  for (int j = tid; j < n; j += kSdThreads) {
    const uint32_t k = keys[j];
    if (k >= lo && k < hi) S.list[atomicAdd(&S.nlist, 1)] = k;
  }
  __syncthreads();
  const int nl = S.nlist;  // == inb
  const uint32_t x = lane < nl ? S.list[lane] : 0u;
  int gt = 0, ge = 0;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const uint32_t v = __shfl_sync(0xffffffffu, x, i);
    gt += (i < nl && v > x) ? 1 : 0;
    ge += (i < nl && v >= x) ? 1 : 0;
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
// -1, and return how many there are: block j in [0, n) is taken when forced, or key > T,
// or key == T among the first `ties` such keys in ascending j (the rule of
// warp_emit_selection).  Thread i owns the contiguous keys [i R, i R + R), R odd so that a
// warp's strided reads hit 32 different banks: it counts its strict takes (forced or
// above T) and its keys equal to T, one CTA-wide exclusive scan gives every thread the
// counts before its range, and a second pass over the range writes each taken key at
// (strict takes before it) + min(ties before it, ties).
__device__ __forceinline__ int cta_emit_selection(const uint32_t* keys, int n, TopkThreshold th, int cur, int n_init,
                                                  int n_local, int topk, int32_t* out, SdSmem& S) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int R = ((n + kSdThreads - 1) / kSdThreads) | 1;
  const int j0 = min(tid * R, n), j1 = min(j0 + R, n);
  const bool simple = topk_simple(th);  // no tie ranks: take forced or key >= take_from(th)
  const uint32_t lo = simple ? take_from(th) : th.key + 1u;  // strict takes: key >= lo (T < 0xffffffff here)
  const uint32_t tkey = th.key;
  const int ties = simple ? 0 : th.ties;
  auto forced = [&](int j) { return j < n_init || j > cur - n_local; };
  int a = 0, b = 0;
  for (int j = j0; j < j1; ++j) {
    const uint32_t k = keys[j];
    const bool f = forced(j);
    a += (f || k >= lo) ? 1 : 0;
    b += (!simple && !f && k == tkey) ? 1 : 0;
  }
  int ia = a, ib = b;  // inclusive scans over the warp
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int ya = __shfl_up_sync(0xffffffffu, ia, o), yb = __shfl_up_sync(0xffffffffu, ib, o);
    if (lane >= o) {
      ia += ya;
      ib += yb;
    }
  }
  if (lane == 31) {
    S.wc[0][warp] = ia;
    S.wc[1][warp] = ib;
  }
  __syncthreads();
  int sa = ia - a, sb = ib - b, ta = 0, tb = 0;
#pragma unroll
  for (int w = 0; w < kSdWarps; ++w) {
    const int x = S.wc[0][w], y = S.wc[1][w];
    if (w < warp) {
      sa += x;
      sb += y;
    }
    ta += x;
    tb += y;
  }
  const int total = min(ta + min(tb, ties), topk);
  for (int j = j0; j < j1; ++j) {
    const uint32_t k = keys[j];
    const bool f = forced(j);
    const bool st = f || k >= lo;
    const bool ti = !simple && !f && k == tkey;
    const int pos = sa + min(sb, ties);
    if ((st || (ti && sb < ties)) && pos < topk) out[pos] = j;
    sa += st ? 1 : 0;
    sb += ti ? 1 : 0;
  }
  for (int e = total + tid; e < topk; e += kSdThreads) out[e] = -1;
  __syncthreads();  // S.wc is free again; out is complete
  return total;
}

// Phase 1, all threads of the CTA: barrier set-up, then this CTA's Kc tiles streamed and
// scored (online (max, sum of exp2) per head, block maxima in bm), then the CTA's state
// per head in S.cm / S.cl.  Ends after a CTA barrier.
__device__ __forceinline__ void sd_score_chunk(const CUtensorMap* tm_kc, const SelDecodeParams& p, const SdItem& it,
                                               unsigned char* ring, uint32_t* bm, SdSmem& S) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nk = it.nk, nq = it.nq, k0 = it.k0, ntiles = it.ntiles;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kSdStages; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], kSdConsumers);
    }
    S.abort = 0;
    S.kcnt = 0;  // a selecting CTA's are filled by every CTA of the cluster after the next cluster barrier
    S.kand = 0xffffffffu;
    S.kor = 0u;
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
      prefetch_tmap(tm_kc);
      const int row0 = static_cast<int>(it.bg * p.NKmax) + k0;
      int i = 0;
      for (; i < ntiles; ++i) {
        const int st = i % kSdStages, u = i / kSdStages;
        if (u > 0 && !mbar_wait(&S.empty[st], (u - 1) & 1, &S.abort)) break;
        unsigned char* dst = ring + st * kKcTileBytes;
        mbar_arrive_expect_tx(&S.full[st], kKcTileBytes);
        tma_load_2d(dst, tm_kc, &S.full[st], 0, row0 + i * kKcTile);
        tma_load_2d(dst + kKcTileBytes / 2, tm_kc, &S.full[st], 64, row0 + i * kKcTile);
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
      load_q_frags(p.q + (static_cast<long long>(it.b) * p.Hq + it.g * p.G) * kHeadDim, p.G, qa);
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
  __syncthreads();
}

// Phase 2, after a cluster barrier that follows phase 1 in every CTA: the log-sum-exp per
// head from every CTA's state, the previous CTA's carry, and the keys of this CTA's blocks
// stored into CTA 0's key array (kAll: into every CTA's), with their candidate count, AND
// and OR added into the same CTAs' (`scratch` is this CTA's own address of the selection
// scratch); each CTA that will select zeroes the first digit histogram of its threshold
// search.
template <bool kAll>
__device__ __forceinline__ void sd_block_keys(cooperative_groups::cluster_group& cluster, const SelDecodeParams& p,
                                              const SdItem& it, unsigned char* scratch, const uint32_t* bm,
                                              SdSmem& S) {
  uint32_t* keys = reinterpret_cast<uint32_t*>(scratch + kSdKeysOff);
  if (kAll || it.c == 0) {
    uint32_t* hist = reinterpret_cast<uint32_t*>(scratch + kSdHistOff);
    for (int i = threadIdx.x; i < kSdHistBins; i += kSdThreads) hist[i] = 0u;
  }
  const int C = it.C, c = it.c, nq = it.nq, cur = it.cur;
  // gather every CTA's (max, sum) and the previous CTA's carry, all loads in flight at once
  for (int e = threadIdx.x; e < kGroupRows * C; e += kSdThreads) {
    const int r = e / kGroupRows, h = e % kGroupRows;
    S.pm[r][h] = cluster.map_shared_rank(&S.cm[0], r)[h];
    S.pl[r][h] = cluster.map_shared_rank(&S.cl[0], r)[h];
  }
  if (threadIdx.x >= kSdThreads - kGroupRows) {
    const int h = threadIdx.x - (kSdThreads - kGroupRows);
    S.carry[h] = c > 0 ? ord_dec(cluster.map_shared_rank(const_cast<uint32_t*>(bm), c - 1)[h * kSdBStride + nq])
                       : -INFINITY;
  }
  if (kAll || c == 0) {  // zero padding up to a multiple of 4 keys
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
  const int jb0 = c * nq;
  const int jb1 = c == C - 1 ? cur + 1 : min(jb0 + nq, cur + 1);
  int cnt = 0;
  uint32_t kand = 0xffffffffu, kor = 0u;
  for (int j = jb0 + threadIdx.x; j < jb1; j += kSdThreads) {
    const int ql = j - jb0;  // <= nq, since cur + 1 <= ceil(nk / 4) + 1 <= C nq + 1
    const bool eligible = block_eligible(j, it.nk - 1, p.pool_mode);
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
    if (kAll) {
      for (int r = 0; r < C; ++r) cluster.map_shared_rank(keys, r)[j] = key;
    } else {
      cluster.map_shared_rank(keys, 0)[j] = key;
    }
    if (key != 0u) {
      ++cnt;
      kand &= key;
      kor |= key;
    }
  }
  cnt = __reduce_add_sync(0xffffffffu, cnt);
  kand = __reduce_and_sync(0xffffffffu, kand);
  kor = __reduce_or_sync(0xffffffffu, kor);
  if ((threadIdx.x & 31) == 0 && cnt > 0) {
    for (int r = 0; r < (kAll ? C : 1); ++r) {
      atomicAdd(cluster.map_shared_rank(&S.kcnt, r), cnt);
      atomicAnd(cluster.map_shared_rank(&S.kand, r), kand);
      atomicOr(cluster.map_shared_rank(&S.kor, r), kor);
    }
  }
}

// Phase 3, a CTA that holds every key, after a cluster barrier that follows phase 2 in
// every CTA: the top-k of the keys in `scratch` (kSdScratchBytes, the drained tile ring)
// and the ascending list, -1 padded, written to out[0 .. topk) (global or shared memory);
// returns the number of blocks in it.  Ends after a CTA barrier.
__device__ __forceinline__ int sd_select(const SelDecodeParams& p, const SdItem& it, unsigned char* scratch,
                                         int32_t* out, SdSmem& S) {
  const uint32_t* keys = reinterpret_cast<const uint32_t*>(scratch + kSdKeysOff);
  if (it.cur < 0) {
    for (int e = threadIdx.x; e < p.topk; e += kSdThreads) out[e] = -1;
    __syncthreads();
    return 0;
  }
  const int want = p.topk - forced_count(it.cur, p.n_init, p.n_local);
  const TopkThreshold th =
      cta_topk_threshold(keys, it.cur + 1, want, reinterpret_cast<uint32_t*>(scratch + kSdHistOff), S);
  return cta_emit_selection(keys, it.cur + 1, th, it.cur, p.n_init, p.n_local, p.topk, out, S);
}

// grid = C * B * Hkv (cluster r serves item r), cluster = (C, 1, 1), block = 160.
__global__ void __launch_bounds__(kSdThreads)
    select_decode_kernel(const __grid_constant__ CUtensorMap tm_kc, const SelDecodeParams p) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ unsigned char smem_raw[];
  unsigned char* ring = align_smem(smem_raw, 1024);
  uint32_t* bm = reinterpret_cast<uint32_t*>(ring + kSdStages * kKcTileBytes);  // [16][kSdBStride], ord_enc
  SdSmem& S = *reinterpret_cast<SdSmem*>(ring + kSdRegionBytes);

  const int C = static_cast<int>(cluster.num_blocks());
  const int c = static_cast<int>(cluster.block_rank());
  allow_dependent_launch();  // the decode attention may set up while this selection runs
  grid_dependency_wait();    // q, Kc and lens may come from the previous kernel
  const long long bg = blockIdx.x / C;  // clusters are consecutive blocks
  const SdItem it = sd_item(p, C, c, bg, min(max(p.lens[bg / p.Hkv], 0), p.Lmax));
  sd_score_chunk(&tm_kc, p, it, ring, bm, S);
  cluster.sync();  // every CTA's tiles are consumed and its partial state is final
  sd_block_keys<false>(cluster, p, it, ring, bm, S);
  cluster.sync();  // CTA 0 holds every key; no CTA reads a peer's shared memory after this
  if (c != 0) return;
  sd_select(p, it, ring, p.idx + it.bg * p.topk, S);
}

}  // namespace infllmv2
