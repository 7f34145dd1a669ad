// select_decode.cuh -- block scoring and group-shared top-k for one decode token per
// sequence, one thread-block cluster per (sequence, kv-head).
//
// Same rule as prefill (MiniCPM4 summary page s2.1.1 / s2.1.2) for the query at position
// lens[b]-1, which sees every complete semantic kernel of its sequence.  The kernel axis
// is split over the C CTAs of a cluster; CTA c takes a contiguous chunk of whole
// 64-kernel tiles and streams them from HBM with TMA (128-byte swizzle, no multicast):
//   1. per tile, four warps (16 kernels each) compute the 16 x 64 logits with m16n8k16
//      MMAs, keep an online (max, sum of exp2) per head, and store per head the max of
//      every aligned quad of kernels 4q .. 4q+3 and the quad's last kernel;
//   2. after a cluster barrier each CTA forms lse_h from the C partial states (read
//      through distributed shared memory) and, for its share of the blocks, the block
//      maxima m_h(j) = max(quad j, last kernel of quad j-1) -- block j pools kernels
//      4j-1 .. 4j+3 -- and S(j) = sum_h exp(m_h(j) - lse_h); the keys go to CTA 0;
//   3. CTA 0 finds the k-th largest key by a 32-way radix search (lane l of every warp
//      counts the keys at or above candidate digit l) and writes the ascending list.
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
constexpr int kSdMaxChunk = 1024;  // kernels per CTA at most
constexpr int kSdMaxQuads = kSdMaxChunk / 4;
constexpr int kSdQStride = kSdMaxQuads + 4;  // per-head quad arrays, padded against bank conflicts
constexpr int kSdMaxCluster = 16;
static_assert(kSdStages * kKcTileBytes >= 4 * (INFLLMV2_MAX_SEQ_LEN / kBlock),
              "the block keys of CTA 0 reuse its tile ring");
static_assert(kSdMaxCluster * kSdMaxChunk >= (INFLLMV2_MAX_SEQ_LEN - kKernel) / kStride + 1,
              "a cluster covers the longest sequence");

struct SelDecodeParams {
  const __nv_bfloat16* q;  // [B, Hq, d]
  const int32_t* lens;     // [B]
  int32_t* idx;            // [B, Hkv, 1, topk]
  int B, Hq, Hkv, G, Lmax, NKmax, topk, n_init, n_local;
  float scale_log2;
};

struct SdSmem {
  uint64_t full[kSdStages], empty[kSdStages];
  float m[kSdConsumers][kGroupRows], l[kSdConsumers][kGroupRows];
  float cm[kGroupRows], cl[kGroupRows];  // this CTA's (max, sum of exp2) per head
  float lse2[kGroupRows];                // log2-sum-exp2 per head over the whole sequence
  int cnt[2][kSdWarps][32];
  volatile int abort;
};

constexpr size_t sel_decode_smem_bytes() {
  return 1024 + static_cast<size_t>(kSdStages) * kKcTileBytes + 2 * kGroupRows * kSdQStride * 4 + sizeof(SdSmem);
}

// k-th largest of n keys in shared memory (zero-padded to a multiple of 4) by all
// kSdThreads threads: 31 key bits in digits of 5,5,5,5,5,5,1 bits, lane l of each warp
// counting the keys >= T | l << shift over the warp's share; partial counts meet in
// `cnt` (double-buffered: one barrier per digit).  Same result as warp_radix_threshold.
__device__ __forceinline__ TopkThreshold cta_radix_threshold(const uint32_t* keys, int n, int want,
                                                             int (*cnt)[kSdWarps][32]) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  TopkThreshold r;
  if (want <= 0) {
    r.key = 0xffffffffu;
    r.ties = 0;
    return r;
  }
  const uint4* k4 = reinterpret_cast<const uint4*>(keys);
  const int n4 = (n + 3) >> 2;
  int buf = 0;
  auto count_ge = [&](uint32_t c) -> int {
    int a = 0, b = 0;
    for (int i = warp; i < n4; i += kSdWarps) {
      const uint4 v = k4[i];
      a += (v.x >= c ? 1 : 0) + (v.y >= c ? 1 : 0);
      b += (v.z >= c ? 1 : 0) + (v.w >= c ? 1 : 0);
    }
    cnt[buf][warp][lane] = a + b;
    __syncthreads();
    int tot = 0;
#pragma unroll
    for (int w = 0; w < kSdWarps; ++w) tot += cnt[buf][w][lane];
    buf ^= 1;
    return tot;
  };
  // top digit; lane 0 counts the candidates (keys >= 1) instead of testing digit 0
  uint32_t T = 0;
  {
    const int tot = count_ge(lane == 0 ? 1u : static_cast<uint32_t>(lane) << 26);
    if (__shfl_sync(0xffffffffu, tot, 0) <= want) {  // at most `want` candidates: take them all
      r.key = 0;
      r.ties = 0;
      return r;
    }
    const unsigned ok = __ballot_sync(0xffffffffu, lane > 0 && tot >= want);
    if (ok != 0u) T = static_cast<uint32_t>(31 - __clz(ok)) << 26;
  }
#pragma unroll 1
  for (int shift = 21; shift >= 1; shift -= 5) {
    const int tot = count_ge(T | (static_cast<uint32_t>(lane) << shift));
    const unsigned ok = __ballot_sync(0xffffffffu, tot >= want);  // lane 0 tests T itself
    T |= static_cast<uint32_t>(31 - __clz(ok)) << shift;
  }
  {
    const int tot = count_ge(T | (lane == 1 ? 1u : 0u));
    if (__shfl_sync(0xffffffffu, tot, 1) >= want) T |= 1u;
  }
  r.key = T;
  r.ties = want - count_ge(T + 1u);
  return r;
}

// grid = C * B * Hkv (cluster r serves item r), cluster = (C, 1, 1), block = 160.
__global__ void __launch_bounds__(kSdThreads)
    select_decode_kernel(const __grid_constant__ CUtensorMap tm_kc, const SelDecodeParams p) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ unsigned char smem_raw[];
  unsigned char* ring = align_smem(smem_raw, 1024);
  float* qmax = reinterpret_cast<float*>(ring + kSdStages * kKcTileBytes);  // [16][kSdQStride]
  float* qlast = qmax + kGroupRows * kSdQStride;                             // [16][kSdQStride]
  SdSmem& S = *reinterpret_cast<SdSmem*>(qlast + kGroupRows * kSdQStride);
  uint32_t* keys = reinterpret_cast<uint32_t*>(ring);  // CTA 0 only, once every tile is consumed

  const int C = static_cast<int>(cluster.num_blocks());
  const int c = static_cast<int>(cluster.block_rank());
  const long long bg = blockIdx.x / C;  // clusters are consecutive blocks
  const int b = static_cast<int>(bg / p.Hkv), g = static_cast<int>(bg % p.Hkv);
  const int n = min(max(p.lens[b], 0), p.Lmax);
  const int nk = n >= kKernel ? (n - kKernel) / kStride + 1 : 0;
  const int cur = n > 0 ? (n - 1) / kBlock : -1;
  const int chunk = ((nk + C - 1) / C + kKcTile - 1) / kKcTile * kKcTile;  // kernels per CTA
  const int nq = chunk / 4;                                                 // quads per CTA
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
  // quads past this CTA's tiles (and the one after its chunk) hold no visible kernel
  for (int e = threadIdx.x; e < kGroupRows * (nq + 1 - 16 * ntiles); e += kSdThreads) {
    const int h = e / (nq + 1 - 16 * ntiles), qd = 16 * ntiles + e % (nq + 1 - 16 * ntiles);
    qmax[h * kSdQStride + qd] = -INFINITY;
    qlast[h * kSdQStride + qd] = -INFINITY;
  }
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
        // quad maxima and each quad's last kernel (lanes q4 = 0, 2 own quads 2 nt, 2 nt + 1)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const float pm0 = fmaxf(s[nt][0], s[nt][1]), pm1 = fmaxf(s[nt][2], s[nt][3]);
          const float om0 = __shfl_xor_sync(0xffffffffu, pm0, 1), om1 = __shfl_xor_sync(0xffffffffu, pm1, 1);
          const float la0 = __shfl_xor_sync(0xffffffffu, s[nt][1], 1);
          const float la1 = __shfl_xor_sync(0xffffffffu, s[nt][3], 1);
          if ((q4 & 1) == 0) {
            const int qd = (i * kKcTile + kofs + 8 * nt + 4 * (q4 >> 1)) >> 2;
            qmax[r0 * kSdQStride + qd] = fmaxf(pm0, om0);
            qlast[r0 * kSdQStride + qd] = la0;
            qmax[(r0 + 8) * kSdQStride + qd] = fmaxf(pm1, om1);
            qlast[(r0 + 8) * kSdQStride + qd] = la1;
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

  if (threadIdx.x < kGroupRows) {
    const int h = threadIdx.x;
    float M = -INFINITY;
    for (int r = 0; r < C; ++r) M = fmaxf(M, cluster.map_shared_rank(&S.cm[0], r)[h]);
    float L = 0.f;
    if (M != -INFINITY) {
      for (int r = 0; r < C; ++r)
        L += cluster.map_shared_rank(&S.cl[0], r)[h] * ex2(cluster.map_shared_rank(&S.cm[0], r)[h] - M);
    }
    S.lse2[h] = L > 0.f ? M + lg2(L) : INFINITY;
  }
  if (c == 0) {  // zero padding up to a multiple of 4 keys for the vector scan
    for (int j = cur + 1 + threadIdx.x; j < ((cur + 4) & ~3); j += kSdThreads) keys[j] = 0u;
  }
  __syncthreads();
  // this CTA's blocks: quads [c nq, (c + 1) nq); the last CTA also takes the rest up to cur
  {
    uint32_t* keys0 = cluster.map_shared_rank(keys, 0);
    const float* prev_last = c > 0 ? cluster.map_shared_rank(qlast, c - 1) : nullptr;
    const int jb0 = c * nq;
    const int jb1 = c == C - 1 ? cur + 1 : min(jb0 + nq, cur + 1);
    for (int j = jb0 + threadIdx.x; j < jb1; j += kSdThreads) {
      const int ql = j - jb0;  // <= nq, since cur + 1 <= ceil(nk / 4) + 1 <= C nq + 1
      const bool eligible = max(4 * j - 1, 0) < nk;
      const bool forced = j < p.n_init || j > cur - p.n_local;
      uint32_t key = 0u;
      if (eligible && !forced && ql <= nq) {
        float sc = 0.f;
        for (int h = 0; h < p.G; ++h) {
          float mb = qmax[h * kSdQStride + ql];
          if (j > 0) mb = fmaxf(mb, ql > 0 ? qlast[h * kSdQStride + ql - 1] : prev_last[h * kSdQStride + nq - 1]);
          sc += ex2(mb - S.lse2[h]);
        }
        key = __float_as_uint(sc) + 1u;
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
  const TopkThreshold th = cta_radix_threshold(keys, cur + 1, want, S.cnt);
  if (warp == 0) warp_emit_selection(keys, cur + 1, th, cur, p.n_init, p.n_local, p.topk, out);
}

}  // namespace infllmv2
