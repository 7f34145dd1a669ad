// attn_dec.cuh -- sparse attention for one decode token per sequence, split over a
// thread-block cluster and merged through distributed shared memory.
//
// MiniCPM4 summary page (端设备上的超高效大型语言模型) s2.1: InfLLM v2 speeds up decoding
// as well as prefill; s2.1.3: the token attends only to its selected blocks, and the
// query heads of a group share them (s2.1.2), so each block is read once per group.
//
// A decode step has only B x Hkv (sequence, kv-head) items, each reading its selected
// 64-key blocks (32 KB of K and V per block) from HBM.  A cluster of C CTAs serves one
// item: CTA c takes a contiguous share of the compacted block list, streams its blocks
// through a TMA ring (128-byte swizzle, no multicast) and runs the four-warp m16n8k16
// online softmax of the prefill fallback kernel (16 keys of each block per warp).  The
// CTA's partial state -- running max and row sum (base 2) and unnormalised O for the 16
// head rows -- stays in its shared memory.  After a cluster barrier CTA c merges head
// rows [16 c / C, 16 (c + 1) / C) from every peer's state, read through distributed
// shared memory, and writes O and the log-sum-exp.  No workspace, one launch; the
// bound is HBM bandwidth (512 bytes of K and V per attended key and kv-head).
#pragma once
#include <cooperative_groups.h>

#include "attn.cuh"
#include "common.cuh"

namespace infllmv2 {

constexpr int kAdStages = 3;
constexpr int kAdThreads = kAttnThreads;  // 4 consumer warps + 1 producer warp
constexpr int kAdMaxCluster = 16;
constexpr int kAdWarpRows = kGroupRows * kMergeRowFloats;  // floats of one warp's partial O
static_assert((kAttnConsumers + 1) * kAdWarpRows * 4 <= kAdStages * kAttnStageBytes,
              "the merge scratch reuses the drained ring");

struct AdSmem {
  uint64_t full[kAdStages], empty[kAdStages], qbar;
  int n_blocks;
  int list[kMaxTopk];
  float m[kAttnConsumers][kGroupRows], l[kAttnConsumers][kGroupRows];
  float cm[kGroupRows], cl[kGroupRows];  // this CTA's state per head: max (base 2), row sum
  volatile int abort;
};

constexpr size_t attn_dec_smem_bytes() {
  return 1024 + static_cast<size_t>(kAdStages) * kAttnStageBytes + kQTileBytes + sizeof(AdSmem);
}

// Barrier set-up of the attention ring (thread 0; the caller's next CTA barrier publishes it).
__device__ __forceinline__ void ad_init(AdSmem& S) {
  for (int s = 0; s < kAdStages; ++s) {
    mbar_init(&S.full[s], 1);
    mbar_init(&S.empty[s], kAttnConsumers);
  }
  mbar_init(&S.qbar, 1);
  S.abort = 0;
  fence_mbar_init();
}

// This CTA's share of an item, all threads: the group's query tile and the n blocks
// blocks[0 .. n) (shared memory) streamed through the ring, the four consumer warps'
// online softmax, then their states combined in the drained ring into this CTA's state
// (S.cm, S.cl and the unnormalised rows in ad_comb(ring)).  Ends after a CTA barrier.
__device__ __forceinline__ float* ad_comb(unsigned char* ring) {
  return reinterpret_cast<float*>(ring) + kAttnConsumers * kAdWarpRows;
}
__device__ __forceinline__ void ad_partial(const CUtensorMap* tm_q, const CUtensorMap* tm_k, const CUtensorMap* tm_v,
                                           const AttnParams& p, long long bg, int qrow, int t, const int* blocks,
                                           int n, unsigned char* ring, unsigned char* qtile, AdSmem& S) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* part = reinterpret_cast<float*>(ring);  // [4 warps][16][kMergeRowFloats], once the ring drained
  float* comb = ad_comb(ring);                   // [16][kMergeRowFloats]: this CTA's state
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  float o[16][4];
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
  if (warp == kAttnConsumers) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && n > 0) {
      mbar_arrive_expect_tx(&S.qbar, kQTileBytes);
      tma_load_2d(qtile, tm_q, &S.qbar, 0, qrow);
      tma_load_2d(qtile + kQTileBytes / 2, tm_q, &S.qbar, 64, qrow);
      const long long kvrow0 = bg * p.Lmax;
      int i = 0;
      for (; i < n; ++i) {
        const int st = i % kAdStages, u = i / kAdStages;
        if (u > 0 && !mbar_wait(&S.empty[st], (u - 1) & 1, &S.abort)) break;
        const int krow = static_cast<int>(kvrow0 + static_cast<long long>(blocks[i]) * kBlock);
        unsigned char* sk = ring + st * kAttnStageBytes;
        mbar_arrive_expect_tx(&S.full[st], kAttnStageBytes);
        tma_load_2d(sk, tm_k, &S.full[st], 0, krow);
        tma_load_2d(sk + kKvTileBytes / 2, tm_k, &S.full[st], 64, krow);
        tma_load_2d(sk + kKvTileBytes, tm_v, &S.full[st], 0, krow);
        tma_load_2d(sk + kKvTileBytes + kKvTileBytes / 2, tm_v, &S.full[st], 64, krow);
      }
      mbar_wait_drain(&S.qbar, 0);
      if (S.abort) {  // let every issued copy land before the ring is reused
        for (int j = max(0, i - kAdStages); j < i; ++j) mbar_wait_drain(&S.full[j % kAdStages], (j / kAdStages) & 1);
      }
    }
  } else if (n > 0) {
    // --------------------------------------------------------- consumer warps
    uint32_t qa[8][4];
    if (mbar_wait(&S.qbar, 0, &S.abort)) {
      const uint32_t qs = smem_u32(qtile);
      const int mi = lane >> 3;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const int row = (lane & 7) + ((mi & 1) << 3);
        const int d = 16 * ks + ((mi >> 1) << 3);
        ldsm_x4(qs + (d >> 6) * (kQTileBytes / 2) + sw128(row, (d & 63) >> 3), qa[ks][0], qa[ks][1], qa[ks][2],
                qa[ks][3]);
      }
      for (int i = 0; i < n; ++i) {
        const int st = i % kAdStages;
        if (!mbar_wait(&S.full[st], (i / kAdStages) & 1, &S.abort)) break;
        attn_block_update(ring + st * kAttnStageBytes, blocks[i], t, 16 * warp, qa, p.scale_log2, m0, m1, l0, l1,
                          o);
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.empty[st]);
      }
    }
  }
  __syncthreads();  // the ring is drained: it becomes the merge scratch
  if (warp < kAttnConsumers) {
    const int q4 = lane & 3, r0 = lane >> 2;
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    float* mo = part + warp * kAdWarpRows;
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      const int col = 8 * nt + 2 * q4;
      *reinterpret_cast<float2*>(mo + r0 * kMergeRowFloats + col) = make_float2(o[nt][0], o[nt][1]);
      *reinterpret_cast<float2*>(mo + (r0 + 8) * kMergeRowFloats + col) = make_float2(o[nt][2], o[nt][3]);
    }
    if (q4 == 0) {
      S.m[warp][r0] = m0;
      S.m[warp][r0 + 8] = m1;
      S.l[warp][r0] = l0;
      S.l[warp][r0 + 8] = l1;
    }
  }
  __syncthreads();
  // this CTA's state: the four warps combined (warp w: rows 4 w .. 4 w + 3)
  if (warp < kAttnConsumers) {
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
      const int r = 4 * warp + rr;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kAttnConsumers; ++w) M = fmaxf(M, S.m[w][r]);
      float L = 0.f;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < kAttnConsumers; ++w) {
          const float wt = ex2(S.m[w][r] - M);
          L += wt * S.l[w][r];
          const float4 v = *reinterpret_cast<const float4*>(part + w * kAdWarpRows + r * kMergeRowFloats + 4 * lane);
          acc.x += wt * v.x;
          acc.y += wt * v.y;
          acc.z += wt * v.z;
          acc.w += wt * v.w;
        }
      }
      *reinterpret_cast<float4*>(comb + r * kMergeRowFloats + 4 * lane) = acc;
      if (lane == 0) {
        S.cm[r] = M;
        S.cl[r] = L;
      }
    }
  }
  __syncthreads();
}

// Cluster merge, all threads of every CTA (it contains two cluster barriers): CTA crank
// merges head rows [crank 16 / C, (crank + 1) 16 / C) of the C CTAs' states, read through
// distributed shared memory (a warp per row: lane r reads CTA r's max and sum, the
// C partial rows are all in flight before they are summed), and writes O and the lse.
__device__ __forceinline__ void ad_merge(cooperative_groups::cluster_group& cluster, const AttnParams& p, int qrow,
                                         unsigned char* ring, AdSmem& S) {
  const int C = static_cast<int>(cluster.num_blocks());
  const int crank = static_cast<int>(cluster.block_rank());
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* comb = ad_comb(ring);
  cluster.sync();  // every CTA's state is final
  const int h_per = kGroupRows / C;
  for (int hh = warp; hh < h_per; hh += kAdThreads / 32) {
    const int h = crank * h_per + hh;
    const float cmr = lane < C ? cluster.map_shared_rank(&S.cm[0], lane)[h] : -INFINITY;
    const float clr = lane < C ? cluster.map_shared_rank(&S.cl[0], lane)[h] : 0.f;
    float M = cmr;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float wt = (M != -INFINITY && lane < C) ? ex2(cmr - M) : 0.f;
    float L = wt * clr;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int r0 = 0; r0 < kAdMaxCluster; r0 += 8) {
      float4 v[8];
      float w8[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int r = r0 + u;
        w8[u] = __shfl_sync(0xffffffffu, wt, r);
        v[u] = r < C ? *reinterpret_cast<const float4*>(cluster.map_shared_rank(comb, r) + h * kMergeRowFloats +
                                                        4 * lane)
                     : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        acc.x += w8[u] * v[u].x;
        acc.y += w8[u] * v[u].y;
        acc.z += w8[u] * v[u].z;
        acc.w += w8[u] * v[u].w;
      }
    }
    if (h < p.G) {
      const float inv = L > 0.f ? 1.f / L : 0.f;
      uint2 pk;
      pk.x = pack_bf16(acc.x * inv, acc.y * inv);
      pk.y = pack_bf16(acc.z * inv, acc.w * inv);
      *reinterpret_cast<uint2*>(p.o + (static_cast<long long>(qrow) + h) * kHeadDim + 4 * lane) = pk;
      if (p.lse != nullptr && lane == 0)
        p.lse[static_cast<long long>(qrow) + h] = L > 0.f ? (M + lg2(L)) * 0.6931471805599453f : -INFINITY;
    }
  }
  cluster.sync();  // peers' shared memory stays valid until every CTA has read it
}

// grid = C * B * Hkv (cluster r serves item r), cluster = (C, 1, 1), block = 160.  C divides 16.
__global__ void __launch_bounds__(kAdThreads)
    attn_decode_cluster_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                               const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ unsigned char smem_raw[];
  unsigned char* ring = align_smem(smem_raw, 1024);
  unsigned char* qtile = ring + kAdStages * kAttnStageBytes;
  AdSmem& S = *reinterpret_cast<AdSmem*>(qtile + kQTileBytes);

  const int C = static_cast<int>(cluster.num_blocks());
  const int crank = static_cast<int>(cluster.block_rank());
  const long long bg = blockIdx.x / C;  // clusters are consecutive blocks
  const int b = static_cast<int>(bg / p.Hkv), g = static_cast<int>(bg % p.Hkv);
  const int qrow = b * p.Hq + g * p.G;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // prologue that reads no input: it overlaps the end of the selection kernel
  allow_dependent_launch();
  if (threadIdx.x == 0) ad_init(S);
  if (warp == kAttnConsumers && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  grid_dependency_wait();  // block_idx (and q, the caches, lens) are complete from here on
  const int t = min(p.lens[b], p.Lmax) - 1;  // < 0: empty sequence
  const int cur = t >= 0 ? t / kBlock : -1;
  if (warp == kAttnConsumers) {  // compact the item's valid block indices, in list order
    const int32_t* row = p.idx + bg * static_cast<long long>(p.topk);
    int count = 0;
    for (int e0 = 0; e0 < p.topk; e0 += 32) {
      const int e = e0 + lane;
      const int j = e < p.topk ? row[e] : -1;
      const bool ok = j >= 0 && j <= cur;
      const unsigned msk = __ballot_sync(0xffffffffu, ok);
      if (ok) S.list[count + __popc(msk & ((1u << lane) - 1u))] = j;
      count += __popc(msk);
    }
    if (lane == 0) S.n_blocks = count;
  }
  __syncthreads();
  const int n_all = S.n_blocks;
  const int per = (n_all + C - 1) / C;
  const int lo = min(crank * per, n_all);
  const int n = min(lo + per, n_all) - lo;
  ad_partial(&tm_q, &tm_k, &tm_v, p, bg, qrow, t, S.list + lo, n, ring, qtile, S);
  ad_merge(cluster, p, qrow, ring, S);
}

}  // namespace infllmv2
