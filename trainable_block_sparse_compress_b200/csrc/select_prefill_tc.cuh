// select_prefill_tc.cuh -- block scoring and group-shared top-k for prefill on the
// 5th-generation tensor cores (tcgen05 + TMEM), for GQA groups of 16 heads.
//
// Same rule as select_prefill.cuh (MiniCPM4 summary page s2.1.1 / s2.1.2): per head a
// softmax over the visible semantic kernels, max-pool of the 5 kernels overlapping each
// block, sum over the group's heads, top-k with forced initial/local blocks.
//
// One CTA = 8 consecutive query tokens of one (sequence, kv-head): 8 x 16 heads = the 128
// rows (M) of a UMMA tile.  Warp roles:
//   warp 4  TMA: the 128 x 128 query tile once (3-D map: token, head, dim), then
//           128-kernel tiles of Kc (128 x 128 bf16, 32 KB) through a 3-stage ring, twice;
//   warp 5  allocates 256 TMEM columns and, from one thread, issues for every Kc tile
//           8 UMMAs (M128 N128 K16, bf16 -> fp32) into one of two TMEM accumulators;
//   warps 0-3  epilogue: thread (w, lane) owns TMEM lane 32 w + lane = row
//           (token, head).  Pass A keeps an online log-sum-exp of its row; pass B pools
//           block maxima along its row, forms p = exp(m - lse), sums the 16 heads of a
//           token with a 16-lane transpose-reduce (30 shuffles per 32 blocks) and stores
//           the block keys in shared memory; then each warp radix-selects the top blocks
//           of its two tokens.
#pragma once
#include "common.cuh"
#include "select_prefill.cuh"
#include "tcgen05.cuh"
#include "topk.cuh"

namespace infllmv2 {

constexpr int kTcTokens = 8;
constexpr int kTcN = 128;
constexpr int kTcStages = 3;
constexpr int kTcTileBytes = kTcN * kHeadDim * 2;  // 32 KB
constexpr int kTcQBytes = 128 * kHeadDim * 2;      // 32 KB
constexpr int kTcEpiWarps = 4;
constexpr int kTcThreads = 32 * (kTcEpiWarps + 2);
constexpr uint32_t kTcTmemCols = 2 * kTcN;

struct SelTcSmem {
  uint64_t qbar, full[kTcStages], empty[kTcStages], tfull[2], tempty[2], mma_done;
  uint32_t tmem_base;
  volatile int abort;
};

inline size_t sel_tc_smem_bytes(int nblk_cap) {
  return 1024 + kTcQBytes + static_cast<size_t>(kTcStages) * kTcTileBytes +
         static_cast<size_t>(kTcTokens) * nblk_cap * 4 + kTcEpiWarps * 256 * 4 + sizeof(SelTcSmem);
}

// Sum of v over the 16 lanes sharing lane bits 4+ (one token's heads), scattered: lane
// L (mod 16) returns the totals of entries 2L and 2L+1.
__device__ __forceinline__ float2 reduce_scatter16(const float (&v)[32]) {
  const int lane = threadIdx.x & 31;
  float a[16];
  {
    const bool up = lane & 8;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float send = up ? v[i] : v[i + 16];
      const float keep = up ? v[i + 16] : v[i];
      a[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
  }
  float b8[8];
  {
    const bool up = lane & 4;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float send = up ? a[i] : a[i + 8];
      const float keep = up ? a[i + 8] : a[i];
      b8[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
  }
  float c4[4];
  {
    const bool up = lane & 2;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float send = up ? b8[i] : b8[i + 4];
      const float keep = up ? b8[i + 4] : b8[i];
      c4[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    }
  }
  float d2[2];
  {
    const bool up = lane & 1;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const float send = up ? c4[i] : c4[i + 2];
      const float keep = up ? c4[i + 2] : c4[i];
      d2[i] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
    }
  }
  return make_float2(d2[0], d2[1]);
}

// grid = B * Hkv * ceil(L / 8) (latest tiles first), block = 192.  Requires G == 16.
__global__ void __launch_bounds__(kTcThreads, 1)
    select_prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q3, const __grid_constant__ CUtensorMap tm_kc,
                             const SelPrefillParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = align_smem(smem_raw, 1024);
  unsigned char* qs = base;
  unsigned char* ring = qs + kTcQBytes;
  uint32_t* keys_all = reinterpret_cast<uint32_t*>(ring + kTcStages * kTcTileBytes);
  uint32_t* hist_all = keys_all + kTcTokens * p.nblk_cap;
  SelTcSmem& S = *reinterpret_cast<SelTcSmem*>(hist_all + kTcEpiWarps * 256);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long nbg = static_cast<long long>(p.B) * p.Hkv;
  const int tile = p.tiles_per_bg - 1 - static_cast<int>(blockIdx.x / nbg);
  const long long bg = blockIdx.x % nbg;
  const int b = static_cast<int>(bg / p.Hkv), g = static_cast<int>(bg % p.Hkv);
  const int t0 = tile * kTcTokens;
  const int imax_last = last_visible_kernel(min(t0 + kTcTokens - 1, p.L - 1));
  const int TA = imax_last >= 0 ? imax_last / kTcN + 1 : 0;
  const int TB = imax_last >= 0 ? (imax_last + 1) / kTcN + 1 : 0;
  const int T = TA + TB;

  if (threadIdx.x == 0) {
    mbar_init(&S.qbar, 1);
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&S.tfull[a], 1);
      mbar_init(&S.tempty[a], kTcEpiWarps);
    }
    mbar_init(&S.mma_done, 1);
    S.abort = 0;
    fence_mbar_init();
  }
  if (warp == kTcEpiWarps + 1) {
    tmem_alloc(&S.tmem_base, kTcTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;

  if (warp == kTcEpiWarps) {
    // ---------------------------------------------------------------- TMA warp
    if (lane == 0 && T > 0) {
      prefetch_tmap(&tm_q3);
      prefetch_tmap(&tm_kc);
      mbar_arrive_expect_tx(&S.qbar, kTcQBytes);
      tma_load_3d(qs, &tm_q3, &S.qbar, 0, g * kGroupRows, b * p.L + t0);
      tma_load_3d(qs + kTcQBytes / 2, &tm_q3, &S.qbar, 64, g * kGroupRows, b * p.L + t0);
      const int row0 = static_cast<int>(bg * p.NKmax);
      for (int n = 0; n < T; ++n) {
        const int st = n % kTcStages, u = n / kTcStages;
        if (u > 0) mbar_wait(&S.empty[st], (u - 1) & 1, &S.abort);
        if (S.abort) break;
        const int c = n < TA ? n : n - TA;
        unsigned char* dst = ring + st * kTcTileBytes;
        mbar_arrive_expect_tx(&S.full[st], kTcTileBytes);
        tma_load_2d(dst, &tm_kc, &S.full[st], 0, row0 + c * kTcN);
        tma_load_2d(dst + kTcTileBytes / 2, &tm_kc, &S.full[st], 64, row0 + c * kTcN);
      }
    }
    return;
  }

  if (warp == kTcEpiWarps + 1) {
    // ---------------------------------------------------------------- MMA warp
    if (lane == 0 && T > 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, kTcN, false, false);
      mbar_wait(&S.qbar, 0, &S.abort);
      const uint32_t qa = smem_u32(qs);
      for (int n = 0; n < T; ++n) {
        const int st = n % kTcStages, acc = n & 1, u = n >> 1;
        mbar_wait(&S.full[st], (n / kTcStages) & 1, &S.abort);
        if (u > 0) mbar_wait(&S.tempty[acc], (u - 1) & 1, &S.abort);
        tc_fence_after();
        const uint32_t kb = smem_u32(ring + st * kTcTileBytes);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t off = static_cast<uint32_t>((k >> 2) * (kTcQBytes / 2) + (k & 3) * 32);
          const uint32_t offb = static_cast<uint32_t>((k >> 2) * (kTcTileBytes / 2) + (k & 3) * 32);
          umma_bf16(tmem + static_cast<uint32_t>(acc * kTcN), desc_k_sw128(qa + off), desc_k_sw128(kb + offb),
                    idesc, k > 0 ? 1u : 0u);
        }
        umma_commit(&S.empty[st]);
        umma_commit(&S.tfull[acc]);
      }
      umma_commit(&S.mma_done);
    }
    __syncwarp();
    named_bar_sync(1, 32 * (kTcEpiWarps + 1));  // the epilogue has read TMEM for the last time
    if (lane == 0 && T > 0) mbar_wait_drain(&S.mma_done, 0);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTcTmemCols);
    return;
  }

  // ---------------------------------------------------------------- epilogue warps
  const int w = warp;
  const int tok = (32 * w + lane) >> 4;
  const int t_raw = t0 + tok;
  const bool tok_ok = t_raw < p.L;
  const int t = tok_ok ? t_raw : p.L - 1;
  const int imax = last_visible_kernel(t);
  const int cur = t / kBlock;
  const uint32_t trow = tmem + (static_cast<uint32_t>(32 * w) << 16);
  const float sl2 = p.scale_log2;

  // pass A: log-sum-exp of this row over its visible kernels (base 2)
  float m = -INFINITY, l = 0.f;
  for (int n = 0; n < TA; ++n) {
    const int acc = n & 1;
    mbar_wait(&S.tfull[acc], (n >> 1) & 1, &S.abort);
    tc_fence_after();
#pragma unroll 1
    for (int q = 0; q < kTcN / 32; ++q) {
      uint32_t v[32];
      tmem_ld32(trow + static_cast<uint32_t>(acc * kTcN + 32 * q), v);
      const int i0 = n * kTcN + 32 * q;
      float x[32];
      float cm = -INFINITY;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        x[e] = (i0 + e <= imax) ? __uint_as_float(v[e]) * sl2 : -INFINITY;
        cm = fmaxf(cm, x[e]);
      }
      if (cm != -INFINITY) {
        const float mn = fmaxf(m, cm);
        float s = 0.f;
#pragma unroll
        for (int e = 0; e < 32; ++e) s += ex2(x[e] - mn);
        l = l * ex2(m - mn) + s;
        m = mn;
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.tempty[acc]);
  }
  const float lse = l > 0.f ? m + lg2(l) : INFINITY;

  uint32_t* keys = keys_all + tok * p.nblk_cap;
  for (int j = lane & 15; j <= cur; j += 16) keys[j] = 0u;
  __syncwarp();

  // pass B: block maxima along the row, p = exp(m - lse), group sum over the 16 heads
  float carry = -INFINITY;  // logit of the kernel just before the current tile
  for (int n = TA; n < T; ++n) {
    const int c = n - TA;
    const int acc = n & 1;
    mbar_wait(&S.tfull[acc], (n >> 1) & 1, &S.abort);
    tc_fence_after();
    float pb[32];
#pragma unroll
    for (int q = 0; q < kTcN / 32; ++q) {
      uint32_t v[32];
      tmem_ld32(trow + static_cast<uint32_t>(acc * kTcN + 32 * q), v);
      const int i0 = c * kTcN + 32 * q;
      float x[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) x[e] = (i0 + e <= imax) ? __uint_as_float(v[e]) * sl2 : -INFINITY;
#pragma unroll
      for (int gq = 0; gq < 8; ++gq) {
        float mb = fmaxf(fmaxf(x[4 * gq], x[4 * gq + 1]), fmaxf(x[4 * gq + 2], x[4 * gq + 3]));
        mb = fmaxf(mb, gq == 0 ? carry : x[4 * gq - 1]);
        pb[8 * q + gq] = ex2(mb - lse);
      }
      carry = x[31];
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.tempty[acc]);
    const float2 sum = reduce_scatter16(pb);
    const int j0 = 32 * c + 2 * (lane & 15);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int j = j0 + e;
      if (j <= cur) {
        const bool eligible = max(4 * j - 1, 0) <= imax;
        const bool forced = j < p.n_init || j > cur - p.n_local;
        keys[j] = (eligible && !forced) ? __float_as_uint(e ? sum.y : sum.x) + 1u : 0u;
      }
    }
  }
  tc_fence_before();
  named_bar_sync(1, 32 * (kTcEpiWarps + 1));  // TMEM no longer read: warp 5 may free it
  __syncwarp();

  // top-k of this warp's two tokens
#pragma unroll 1
  for (int tt = 0; tt < 2; ++tt) {
    const int tk = 2 * w + tt;
    const int tr = t0 + tk;
    if (tr >= p.L) break;
    const int cu = tr / kBlock;
    const uint32_t* kt = keys_all + tk * p.nblk_cap;
    const int want = p.topk - forced_count(cu, p.n_init, p.n_local);
    const TopkThreshold th = warp_radix_threshold(kt, cu + 1, want, hist_all + w * 256);
    int32_t* out = p.idx + ((bg * p.L + tr) * static_cast<long long>(p.topk));
    warp_emit_selection(kt, cu + 1, th, cu, p.n_init, p.n_local, p.topk, out);
  }
}

}  // namespace infllmv2
