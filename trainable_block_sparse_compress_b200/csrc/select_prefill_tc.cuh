// select_prefill_tc.cuh -- block scoring and group-shared top-k for prefill on the
// 5th-generation tensor cores (tcgen05 + TMEM), for GQA groups of 16 heads.
//
// Same rule as select_prefill.cuh (MiniCPM4 summary page s2.1.1 / s2.1.2): per head a
// softmax over the visible semantic kernels, max-pool of the 5 kernels overlapping each
// block, sum over the group's heads, top-k with forced initial/local blocks (and the
// same variants: logit-sum scoring without pass A, inside pooling).
//
// One CTA = 128 / G consecutive query rows of one (sequence, kv-head) with the G heads
// of its group each: the 128 rows (M) of a UMMA tile, row = token * G + head.  A chunk's
// rows are the last q_len tokens of a cache of kv_len tokens (a fresh prefill: q_len =
// kv_len = L).  Warp roles (448 threads):
//   warp 12 TMA: the 128 x 128 query tile once (3-D map: token, head, dim), then Kc tiles
//           through a ring of 3 slots (2 when the block keys of long sequences need the
//           room): pass A tiles of 128 kernels, pass B tiles of 144 kernels that start
//           16 kernels early, so each pass-B tile also holds the kernel straddling its
//           first block (4j - 1) and is self-contained;
//   warp 13 allocates TMEM and, from one thread, issues per tile 8 UMMAs (M128 x N128 or
//           N144, K16, bf16 -> fp32) into one of three TMEM accumulators;
//   warps 0-11 three epilogue warpgroups taking every third tile; thread (w, lane) owns TMEM
//           lane 32 (w % 4) + lane = row (token, head).  Pass A keeps an online
//           log-sum-exp per row (the warpgroups' partials are merged once); pass B
//           pools block maxima along the row, forms p = exp(m - lse) and sums the G
//           heads of a token with a G-lane transpose-reduce; block keys go to shared
//           memory; finally warp w selects the top blocks of tokens w, w + 12, ...
#pragma once
#include "common.cuh"
#include "select_prefill.cuh"
#include "tcgen05.cuh"
#include "topk.cuh"

namespace infllmv2 {

constexpr int kTcTokens = 8;           // query rows per CTA at G = 16 (128 / G in general)
constexpr int kTcN = 128;              // kernels per pass-A tile
constexpr int kTcOverlap = 16;         // extra leading kernels of a pass-B tile
constexpr int kTcNB = kTcN + kTcOverlap;  // 144 kernels per pass-B tile
constexpr int kTcStages = 3;
constexpr int kTcHalfBytes = kTcNB * 128;   // one 64-column half of a stage (144 rows x 128 B)
constexpr int kTcStageBytes = 2 * kTcHalfBytes;
constexpr int kTcQBytes = 128 * kHeadDim * 2;  // 32 KB
constexpr int kTcEpiWGs = 3;              // epilogue warpgroups = TMEM accumulators
constexpr int kTcEpiWarps = 4 * kTcEpiWGs;
constexpr int kTcThreads = 32 * (kTcEpiWarps + 2);
constexpr uint32_t kTcTmemCols = 512;
constexpr uint32_t kTcAccStride = 160;
static_assert(kTcAccStride >= kTcNB && (kTcEpiWGs - 1) * kTcAccStride + kTcNB <= kTcTmemCols, "TMEM plan");  // TMEM column offset between accumulators (>= 144)

struct SelTcSmem {
  uint64_t qbar, full[kTcStages], empty[kTcStages], tfull[kTcEpiWGs], tempty[kTcEpiWGs], mma_done;
  float2 part[kTcEpiWGs][128];  // pass-A (max, sum) per warpgroup and row
  uint32_t tmem_base;
  volatile int abort;
};

// Query rows per CTA and warps that run a top-k, for a group of G heads.
inline int sel_tc_tokens(int G) { return 128 / G; }
inline int sel_tc_topk_warps(int G) { return sel_tc_tokens(G) < kTcEpiWarps ? sel_tc_tokens(G) : kTcEpiWarps; }

inline size_t sel_tc_smem_bytes(int nblk_cap, int G, int stages) {
  return 1024 + kTcQBytes + static_cast<size_t>(stages) * kTcStageBytes +
         static_cast<size_t>(sel_tc_tokens(G)) * nblk_cap * 4 + static_cast<size_t>(sel_tc_topk_warps(G)) * 256 * 4 +
         sizeof(SelTcSmem);
}

// Sum of v over the kG lanes that hold one token's heads (lanes sharing lane / kG),
// scattered: lane L returns in v[r], r < 16 / kG, the total of entry (L % kG) * (16 / kG) + r.
// log2(kG) halving steps of one shuffle per kept value (15 shuffles at kG = 16).
template <int kG>
__device__ __forceinline__ void reduce_scatter_group(float (&v)[16]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int m = kG / 2; m >= 1; m >>= 1) {
    const int h = 16 * m / kG;  // values kept after this step
    const bool up = lane & m;
#pragma unroll
    for (int i = 0; i < h; ++i) {
      const float send = up ? v[i] : v[i + h];
      const float keep = up ? v[i + h] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, m);
    }
  }
}

__device__ __forceinline__ float max4(float a, float b, float c, float d) { return fmaxf(fmaxf(a, b), fmaxf(c, d)); }

// grid = B * Hkv * ceil(Lq / (128 / kG)) (latest tiles first), block = 448.  p.G == kG.
template <int kG>
__global__ void __launch_bounds__(kTcThreads, 1)
    select_prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q3, const __grid_constant__ CUtensorMap tm_kca,
                             const __grid_constant__ CUtensorMap tm_kcb, const SelPrefillParams p) {
  constexpr int kTT = 128 / kG;                                     // query rows per CTA
  constexpr int kTopkWarps = kTT < kTcEpiWarps ? kTT : kTcEpiWarps;  // warps that run a top-k
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = align_smem(smem_raw, 1024);
  unsigned char* qs = base;
  unsigned char* ring = qs + kTcQBytes;
  const int NS = p.stages;  // Kc ring slots
  uint32_t* keys_all = reinterpret_cast<uint32_t*>(ring + NS * kTcStageBytes);
  uint32_t* hist_all = keys_all + kTT * p.nblk_cap;
  SelTcSmem& S = *reinterpret_cast<SelTcSmem*>(hist_all + kTopkWarps * 256);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long nbg = static_cast<long long>(p.B) * p.Hkv;
  const int tile = p.tiles_per_bg - 1 - static_cast<int>(blockIdx.x / nbg);
  const long long bg = blockIdx.x % nbg;
  const int b = static_cast<int>(bg / p.Hkv), g = static_cast<int>(bg % p.Hkv);
  const int t0 = tile * kTT;  // first query row of the tile
  const ChunkLens cl = chunk_lens(p.q_lens, p.kv_lens, b, p.Lq, p.Lmax);
  if (t0 >= cl.q_len) return;  // padding rows only (uniform over the CTA, before any set-up)
  const int off = cl.kv_len - cl.q_len;  // position of query row 0
  const int imax_last = last_visible_kernel(off + min(t0 + kTT - 1, cl.q_len - 1));
  // pass A (the per-head lse) only for softmax-sum scoring
  const int TA = (imax_last >= 0 && p.score_mode == kScoreSoftmaxSum) ? imax_last / kTcN + 1 : 0;
  const int TB = imax_last >= 0 ? (imax_last + 1) / kTcN + 1 : 0;
  const int T = TA + TB;

  if (threadIdx.x == 0) {
    mbar_init(&S.qbar, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 1);
    }
    for (int a = 0; a < kTcEpiWGs; ++a) {
      mbar_init(&S.tfull[a], 1);
      mbar_init(&S.tempty[a], 4);  // the four warps of the warpgroup that owns accumulator a
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
      prefetch_tmap(&tm_kca);
      prefetch_tmap(&tm_kcb);
      mbar_arrive_expect_tx(&S.qbar, kTcQBytes);
      tma_load_3d(qs, &tm_q3, &S.qbar, 0, g * kG, b * p.Lq + t0);
      tma_load_3d(qs + kTcQBytes / 2, &tm_q3, &S.qbar, 64, g * kG, b * p.Lq + t0);
      const int row0 = static_cast<int>(bg * p.NKmax);
      int st = 0;        // ring slot of tile n (n % NS, kept incrementally: NS is a runtime value)
      uint32_t ph = 0u;  // parity of (n / NS)
      for (int n = 0; n < T; ++n) {
        if (n >= NS) mbar_wait(&S.empty[st], ph ^ 1u, &S.abort);
        if (S.abort) break;
        unsigned char* dst = ring + st * kTcStageBytes;
        if (n < TA) {
          const int r = row0 + n * kTcN;
          mbar_arrive_expect_tx(&S.full[st], 2 * kTcN * 128);
          tma_load_2d(dst, &tm_kca, &S.full[st], 0, r);
          tma_load_2d(dst + kTcHalfBytes, &tm_kca, &S.full[st], 64, r);
        } else {
          const int r = row0 + (n - TA) * kTcN - kTcOverlap;  // may start before row 0: zero fill
          mbar_arrive_expect_tx(&S.full[st], 2 * kTcNB * 128);
          tma_load_2d(dst, &tm_kcb, &S.full[st], 0, r);
          tma_load_2d(dst + kTcHalfBytes, &tm_kcb, &S.full[st], 64, r);
        }
        if (++st == NS) {
          st = 0;
          ph ^= 1u;
        }
      }
    }
    return;
  }

  if (warp == kTcEpiWarps + 1) {
    // ---------------------------------------------------------------- MMA warp
    if (lane == 0 && T > 0) {
      constexpr uint32_t idesc_a = idesc_bf16_f32(128, kTcN, false, false);
      constexpr uint32_t idesc_b = idesc_bf16_f32(128, kTcNB, false, false);
      mbar_wait(&S.qbar, 0, &S.abort);
      const uint32_t qa = smem_u32(qs);
      int st = 0;        // ring slot of tile n, as in the TMA warp
      uint32_t ph = 0u;
      for (int n = 0; n < T; ++n) {
        const int acc = n % kTcEpiWGs, u = n / kTcEpiWGs;
        mbar_wait(&S.full[st], ph, &S.abort);
        if (u > 0) mbar_wait(&S.tempty[acc], (u - 1) & 1, &S.abort);
        tc_fence_after();
        const uint32_t kb = smem_u32(ring + st * kTcStageBytes);
        const uint32_t idesc = n < TA ? idesc_a : idesc_b;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t off = static_cast<uint32_t>((k >> 2) * (kTcQBytes / 2) + (k & 3) * 32);
          const uint32_t offb = static_cast<uint32_t>((k >> 2) * kTcHalfBytes + (k & 3) * 32);
          umma_bf16(tmem + static_cast<uint32_t>(acc) * kTcAccStride, desc_k_sw128(qa + off),
                    desc_k_sw128(kb + offb), idesc, k > 0 ? 1u : 0u);
        }
        umma_commit(&S.empty[st]);
        umma_commit(&S.tfull[acc]);
        if (++st == NS) {
          st = 0;
          ph ^= 1u;
        }
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
  const int wg = warp >> 2;   // warpgroup: takes tiles n with n % kTcEpiWGs == wg
  const int wq = warp & 3;    // TMEM lane quarter
  const int row = 32 * wq + lane;
  const int tok = row / kG;
  const int t = off + min(t0 + tok, cl.q_len - 1);  // position; rows past q_len compute, write nothing
  const int imax = last_visible_kernel(t);
  const int cur = t / kBlock;
  const uint32_t trow = tmem + (static_cast<uint32_t>(32 * wq) << 16);
  const float sl2 = p.scale_log2;  // > 0: maxima of raw logits scale to maxima of scaled ones

  // pass A: log-sum-exp of this row over its visible kernels (base 2), every third tile
  float m = -INFINITY, l = 0.f;
  for (int n = wg; n < TA; n += kTcEpiWGs) {
    const int acc = n % kTcEpiWGs;
    mbar_wait(&S.tfull[acc], (n / kTcEpiWGs) & 1, &S.abort);
    tc_fence_after();
#pragma unroll 1
    for (int q = 0; q < kTcN / 32; ++q) {
      uint32_t v[32];
      tmem_ld32(trow + static_cast<uint32_t>(acc) * kTcAccStride + static_cast<uint32_t>(32 * q), v);
      const int i0 = n * kTcN + 32 * q;
      float x[32];
      if (i0 + 31 <= imax) {
#pragma unroll
        for (int e = 0; e < 32; ++e) x[e] = __uint_as_float(v[e]);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) x[e] = (i0 + e <= imax) ? __uint_as_float(v[e]) : -INFINITY;
      }
      float c8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) c8[e] = max4(x[e], x[e + 8], x[e + 16], x[e + 24]);
      const float cm = fmaxf(max4(c8[0], c8[1], c8[2], c8[3]), max4(c8[4], c8[5], c8[6], c8[7])) * sl2;
      if (cm != -INFINITY) {
        const float mn = fmaxf(m, cm);
        float s8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
          s8[e] = (ex2(fmaf(x[e], sl2, -mn)) + ex2(fmaf(x[e + 8], sl2, -mn))) +
                  (ex2(fmaf(x[e + 16], sl2, -mn)) + ex2(fmaf(x[e + 24], sl2, -mn)));
        const float s = ((s8[0] + s8[1]) + (s8[2] + s8[3])) + ((s8[4] + s8[5]) + (s8[6] + s8[7]));
        l = l * ex2(m - mn) + s;
        m = mn;
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.tempty[acc]);
  }
  // zero the key rows of tokens warp, warp + 12, ... (blocks 0..cur) while the warpgroups meet
  for (int tw = warp; tw < kTT; tw += kTcEpiWarps) {
    const int tz = off + min(t0 + tw, cl.q_len - 1);
    uint32_t* kz = keys_all + tw * p.nblk_cap;
    for (int j = lane; j <= tz / kBlock; j += 32) kz[j] = 0u;
  }
  S.part[wg][row] = make_float2(m, l);
  named_bar_sync(2, 32 * kTcEpiWarps);
  float lse;
  {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kTcEpiWGs; ++w) M = fmaxf(M, S.part[w][row].x);
    float L = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kTcEpiWGs; ++w) L += S.part[w][row].y * ex2(S.part[w][row].x - M);
    }
    lse = L > 0.f ? M + lg2(L) : INFINITY;
  }

  // pass B: block maxima along the row, p = exp(m - lse) (or m itself for logit-sum
  // scoring), group sum over the G heads
  const bool inside = p.pool_mode == kPoolInside, logit = p.score_mode == kScoreLogitSum;
  uint32_t* keys = keys_all + tok * p.nblk_cap;
  int nb = TA;
  while (nb % kTcEpiWGs != wg) ++nb;
  for (int n = nb; n < T; n += kTcEpiWGs) {
    const int c = n - TA;
    const int acc = n % kTcEpiWGs;
    mbar_wait(&S.tfull[acc], (n / kTcEpiWGs) & 1, &S.abort);
    tc_fence_after();
    const uint32_t tacc = trow + static_cast<uint32_t>(acc) * kTcAccStride;
    // column kTcOverlap-1 holds kernel 128c - 1, the straddle of block 32c
    // (tcgen05.ld is warp-collective: load unconditionally, then mask)
    const int istr = c * kTcN - 1;
    const float cv = __uint_as_float(tmem_ld1(tacc + kTcOverlap - 1));
    float carry = (istr >= 0 && istr <= imax) ? cv : -INFINITY;  // raw logit
#pragma unroll 1
    for (int half = 0; half < 2; ++half) {
      float pb[16];
#pragma unroll
      for (int q2 = 0; q2 < 2; ++q2) {
        uint32_t v[32];
        tmem_ld32(tacc + static_cast<uint32_t>(kTcOverlap + 64 * half + 32 * q2), v);
        const int i0 = c * kTcN + 64 * half + 32 * q2;
        float x[32];
        if (i0 + 31 <= imax) {
#pragma unroll
          for (int e = 0; e < 32; ++e) x[e] = __uint_as_float(v[e]);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) x[e] = (i0 + e <= imax) ? __uint_as_float(v[e]) : -INFINITY;
        }
#pragma unroll
        for (int gq = 0; gq < 8; ++gq) {
          // overlap: kernels 4j-1 (the carry) .. 4j+3; inside: 4j .. 4j+2 (raw logits)
          const float mb = inside ? fmaxf(fmaxf(x[4 * gq], x[4 * gq + 1]), x[4 * gq + 2])
                                  : fmaxf(max4(x[4 * gq], x[4 * gq + 1], x[4 * gq + 2], x[4 * gq + 3]), carry);
          pb[8 * q2 + gq] = logit ? mb : ex2(fmaf(mb, sl2, -lse));  // a logit sum ranks like a scaled one
          carry = x[4 * gq + 3];
        }
      }
      reduce_scatter_group<kG>(pb);
#pragma unroll
      for (int r = 0; r < 16 / kG; ++r) {
        const int j = 32 * c + 16 * half + (lane % kG) * (16 / kG) + r;
        if (j <= cur) {
          const bool eligible = block_eligible(j, imax, p.pool_mode);
          const bool forced = j < p.n_init || j > cur - p.n_local;
          keys[j] = (eligible && !forced) ? score_key(pb[r], p.score_mode) : 0u;
        }
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.tempty[acc]);
  }
  tc_fence_before();
  named_bar_sync(1, 32 * (kTcEpiWarps + 1));  // TMEM no longer read: the MMA warp may free it
  named_bar_sync(2, 32 * kTcEpiWarps);        // all keys written

  // top-k of tokens warp, warp + 12, ...
  if (warp < kTopkWarps) {
    for (int tw = warp; tw < kTT; tw += kTopkWarps) {
      const int tr = t0 + tw;  // query row
      if (tr >= cl.q_len) break;
      const int cu = (off + tr) / kBlock;
      const uint32_t* kt = keys_all + tw * p.nblk_cap;
      const int want = p.topk - forced_count(cu, p.n_init, p.n_local);
      int32_t* out = p.idx + ((bg * p.Lq + tr) * static_cast<long long>(p.topk));
      if (cu + 1 <= 32 * kTopkRegKeys) {
        warp_topk_select(kt, cu + 1, want, cu, p.n_init, p.n_local, p.topk, hist_all + warp * 256, out);
      } else {
        const TopkThreshold th = warp_radix_threshold(kt, cu + 1, want, hist_all + warp * 256);
        warp_emit_selection(kt, cu + 1, th, cu, p.n_init, p.n_local, p.topk, out);
      }
      __syncwarp();
    }
  }
}

}  // namespace infllmv2
