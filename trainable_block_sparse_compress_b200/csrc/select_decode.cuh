// select_decode.cuh -- block scoring and group-shared top-k for one decode token per
// sequence.
//
// Same rule as prefill (MiniCPM4 summary page s2.1.1 / s2.1.2): the query at position
// lens[b]-1 scores every complete semantic kernel of its sequence.  A decode step has
// only B x Hkv rows, so the kernel axis is split over CTAs:
//   select_decode_score_kernel: CTA (chunk c of 256 kernels, g, b) computes the 16 x 256
//     logits with m16n8k16 MMAs, writes the chunk's per-head (max, sum of exp) and, for
//     the 65 blocks that touch the chunk, the per-head max over the chunk's kernels;
//   select_decode_topk_kernel: CTA (g, b) merges the chunk partials into lse_h and the
//     block maxima, forms S(j) = sum_h exp(m_h(j) - lse_h), and radix-selects the top
//     blocks.
// Reading Kc once (bound by HBM bandwidth) dominates; the partials stay in L2.
#pragma once
#include "common.cuh"
#include "select_prefill.cuh"
#include "topk.cuh"

namespace infllmv2 {

constexpr int kDecChunk = 256;  // kernels per score CTA (4 warps x 64)
constexpr int kDecBlocksPerChunk = kDecChunk / 4 + 1;  // 64 blocks + the next block's straddle
constexpr int kDecScoreThreads = 128;
constexpr int kDecTopkThreads = 256;
constexpr int kLogitStride = kDecChunk + 4;

struct SelDecodeParams {
  const __nv_bfloat16* q;  // [B, Hq, d]
  const int32_t* lens;     // [B]
  int32_t* idx;            // [B, Hkv, 1, topk]
  int B, Hq, Hkv, G, Lmax, NKmax, topk, n_init, n_local;
  int n_chunks;  // ceil(NKmax / 256)
  float scale_log2;
  float2* ws_lse;  // [B*Hkv, n_chunks, 16] (max, sum of exp2(x - max)) per head, base 2
  float* ws_bm;    // [B*Hkv, n_chunks, 65, 16] per-head block max over the chunk's kernels
};

inline size_t sel_decode_ws_bytes(int B, int Hkv, int n_chunks) {
  const size_t rows = static_cast<size_t>(B) * Hkv * n_chunks;
  const size_t a = rows * kGroupRows * sizeof(float2);
  const size_t a_pad = (a + 255) & ~static_cast<size_t>(255);
  return a_pad + rows * kDecBlocksPerChunk * kGroupRows * sizeof(float);
}

inline size_t sel_decode_score_smem_bytes() {
  return 1024 + 4 * static_cast<size_t>(kKcTileBytes) + kGroupRows * kLogitStride * 4 + 2 * 4 * kGroupRows * 4 + 64;
}

__device__ __forceinline__ int decode_len(const int32_t* lens, int b, int Lmax) {
  const int n = lens[b];
  return n < 0 ? 0 : (n > Lmax ? Lmax : n);
}

// grid = (n_chunks, Hkv, B), block = 128.
__global__ void __launch_bounds__(kDecScoreThreads)
    select_decode_score_kernel(const __grid_constant__ CUtensorMap tm_kc, const SelDecodeParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* tiles = align_smem(smem_raw, 1024);
  float* lg = reinterpret_cast<float*>(tiles + 4 * kKcTileBytes);  // [16][kLogitStride]
  float* pm = lg + kGroupRows * kLogitStride;                        // [4][16]
  float* pl = pm + 4 * kGroupRows;                                   // [4][16]
  uint64_t* bar = reinterpret_cast<uint64_t*>(pl + 4 * kGroupRows);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar + 1);

  const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = decode_len(p.lens, b, p.Lmax);
  const int nk = n >= kKernel ? (n - kKernel) / kStride + 1 : 0;
  if (c * kDecChunk >= nk) return;
  const long long bg = static_cast<long long>(b) * p.Hkv + g;

  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(bar, 4 * kKcTileBytes);
    const int row0 = static_cast<int>(bg * p.NKmax) + c * kDecChunk;
    for (int w = 0; w < 4; ++w) {
      tma_load_2d(tiles + w * kKcTileBytes, &tm_kc, bar, 0, row0 + w * kKcTile);
      tma_load_2d(tiles + w * kKcTileBytes + kKcTileBytes / 2, &tm_kc, bar, 64, row0 + w * kKcTile);
    }
  }
  uint32_t qa[8][4];
  load_q_frags(p.q + (static_cast<long long>(b) * p.Hq + g * p.G) * kHeadDim, p.G, qa);
  mbar_wait(bar, 0, abort_flag);

  float s[8][4];
  qk_tile(qa, smem_u32(tiles + warp * kKcTileBytes), s);
  const int q4 = lane & 3, r0 = lane >> 2;
  const int i0 = c * kDecChunk + warp * kKcTile;
  float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int col = 8 * nt + 2 * q4 + e;
      const bool ok = i0 + col < nk;
      const float x0 = ok ? s[nt][e] * p.scale_log2 : -INFINITY;
      const float x1 = ok ? s[nt][2 + e] * p.scale_log2 : -INFINITY;
      s[nt][e] = x0;
      s[nt][2 + e] = x1;
      lg[r0 * kLogitStride + warp * kKcTile + col] = x0;
      lg[(r0 + 8) * kLogitStride + warp * kKcTile + col] = x1;
      mx0 = fmaxf(mx0, x0);
      mx1 = fmaxf(mx1, x1);
    }
  }
  mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
  mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
  mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
  mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
  float a0 = 0.f, a1 = 0.f;
  if (mx0 != -INFINITY) {
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) a0 += ex2(s[nt][0] - mx0) + ex2(s[nt][1] - mx0);
  }
  if (mx1 != -INFINITY) {
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) a1 += ex2(s[nt][2] - mx1) + ex2(s[nt][3] - mx1);
  }
  a0 += __shfl_xor_sync(0xffffffffu, a0, 1);
  a0 += __shfl_xor_sync(0xffffffffu, a0, 2);
  a1 += __shfl_xor_sync(0xffffffffu, a1, 1);
  a1 += __shfl_xor_sync(0xffffffffu, a1, 2);
  if (q4 == 0) {
    pm[warp * kGroupRows + r0] = mx0;
    pm[warp * kGroupRows + r0 + 8] = mx1;
    pl[warp * kGroupRows + r0] = a0;
    pl[warp * kGroupRows + r0 + 8] = a1;
  }
  __syncthreads();
  const long long crow = bg * p.n_chunks + c;
  if (threadIdx.x < kGroupRows) {
    const int h = threadIdx.x;
    float M = -INFINITY;
    for (int w = 0; w < 4; ++w) M = fmaxf(M, pm[w * kGroupRows + h]);
    float L = 0.f;
    if (M != -INFINITY)
      for (int w = 0; w < 4; ++w) L += pl[w * kGroupRows + h] * ex2(pm[w * kGroupRows + h] - M);
    p.ws_lse[crow * kGroupRows + h] = make_float2(M, L);
  }
  // per-head max over this chunk's kernels overlapping each of its 65 blocks
  for (int e = threadIdx.x; e < kDecBlocksPerChunk * kGroupRows; e += kDecScoreThreads) {
    const int r = e / kGroupRows, h = e % kGroupRows;
    const int lo = max(4 * r - 1, 0), hi = min(4 * r + 3, kDecChunk - 1);
    float mb = -INFINITY;
    for (int li = lo; li <= hi; ++li) mb = fmaxf(mb, lg[h * kLogitStride + li]);
    p.ws_bm[crow * (kDecBlocksPerChunk * kGroupRows) + e] = mb;
  }
}

// grid = (Hkv, B), block = 256.  Shared: keys[nblk_cap], lse2[16], hist[256].
__global__ void __launch_bounds__(kDecTopkThreads) select_decode_topk_kernel(const SelDecodeParams p, int nblk_cap) {
  extern __shared__ unsigned char smem_raw[];
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw);
  float* lse2 = reinterpret_cast<float*>(keys + nblk_cap);
  uint32_t* hist = reinterpret_cast<uint32_t*>(lse2 + kGroupRows);

  const int g = blockIdx.x, b = blockIdx.y;
  const long long bg = static_cast<long long>(b) * p.Hkv + g;
  const int n = decode_len(p.lens, b, p.Lmax);
  int32_t* out = p.idx + bg * p.topk;
  if (n <= 0) {
    for (int q = threadIdx.x; q < p.topk; q += kDecTopkThreads) out[q] = -1;
    return;
  }
  const int t = n - 1, cur = t / kBlock;
  const int nk = n >= kKernel ? (n - kKernel) / kStride + 1 : 0;
  const int nch = (nk + kDecChunk - 1) / kDecChunk;
  if (threadIdx.x < kGroupRows) {
    const int h = threadIdx.x;
    float M = -INFINITY;
    for (int c = 0; c < nch; ++c) M = fmaxf(M, p.ws_lse[(bg * p.n_chunks + c) * kGroupRows + h].x);
    float L = 0.f;
    if (M != -INFINITY)
      for (int c = 0; c < nch; ++c) {
        const float2 v = p.ws_lse[(bg * p.n_chunks + c) * kGroupRows + h];
        L += v.y * ex2(v.x - M);
      }
    lse2[h] = L > 0.f ? M + lg2(L) : INFINITY;
  }
  __syncthreads();
  const float* bm = p.ws_bm + bg * p.n_chunks * (kDecBlocksPerChunk * kGroupRows);
  for (int j = threadIdx.x; j <= cur; j += kDecTopkThreads) {
    const bool eligible = max(4 * j - 1, 0) < nk;
    const bool forced = j < p.n_init || j > cur - p.n_local;
    uint32_t key = 0u;
    if (eligible && !forced) {
      const int c = j / (kDecChunk / 4), r = j % (kDecChunk / 4);
      float sc = 0.f;
      for (int h = 0; h < p.G; ++h) {
        float mb = c < nch ? bm[(c * kDecBlocksPerChunk + r) * kGroupRows + h] : -INFINITY;
        if (r == 0 && c > 0) mb = fmaxf(mb, bm[((c - 1) * kDecBlocksPerChunk + kDecChunk / 4) * kGroupRows + h]);
        sc += ex2(mb - lse2[h]);
      }
      key = __float_as_uint(sc) + 1u;
    }
    keys[j] = key;
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    const int want = p.topk - forced_count(cur, p.n_init, p.n_local);
    if (cur + 1 <= 32 * kTopkRegKeys) {
      warp_topk_select(keys, cur + 1, want, cur, p.n_init, p.n_local, p.topk, hist, out);
    } else {
      const TopkThreshold th = warp_radix_threshold(keys, cur + 1, want, hist);
      warp_emit_selection(keys, cur + 1, th, cur, p.n_init, p.n_local, p.topk, out);
    }
  }
}

}  // namespace infllmv2
