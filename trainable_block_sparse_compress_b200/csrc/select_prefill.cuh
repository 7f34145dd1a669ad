// select_prefill.cuh -- fused block scoring and group-shared top-k for prefill.
//
// MiniCPM4 summary page (端设备上的超高效大型语言模型) s2.1.2: relevance between query
// tokens and KV blocks is scored through semantic kernels, and the heads of a group
// share one set of top blocks; s2.1.1: each token keeps its highest-scoring blocks.
//
// One CTA = 8 consecutive query rows of one (sequence, kv-head); consumer warp w owns
// row t0 + w and its 16 group heads (the MMA rows).  A chunk's rows are the last q_len
// tokens of a cache of kv_len tokens (a fresh prefill: q_len = kv_len = L).  A producer warp streams 64-kernel
// tiles of Kc (64 x 128 bf16, TMA with 128-byte swizzle) through a 4-stage ring twice:
//   pass A: logits x_h(i) = scale q_h . Kc_i, online log-sum-exp per head over the
//           visible kernels;
//   pass B: the logits again; per head the max over the 5 kernels 4j-1..4j+3 that
//           overlap block j, p_h(j) = exp(m_h(j) - lse_h), summed over the 16 heads
//           with warp shuffles, giving the block score S(j) kept in shared memory.
// Variants: logit-sum scoring sums m_h(j) itself and skips pass A; inside pooling takes
// the max over kernels 4j..4j+2 only.
// Finally each warp radix-selects its token's top blocks and writes them ascending.
#pragma once
#include "common.cuh"
#include "topk.cuh"

namespace infllmv2 {

constexpr int kSelWarps = 8;
constexpr int kSelThreads = 32 * (kSelWarps + 1);
constexpr int kSelStages = 4;
constexpr int kKcTile = 64;
constexpr int kKcTileBytes = kKcTile * kHeadDim * 2;

struct SelPrefillParams {
  const __nv_bfloat16* q;  // [B, Lq, Hq, d]
  int32_t* idx;            // [B, Hkv, Lq, topk]
  const int32_t* q_lens;   // [B] queries per sequence (<= Lq), or nullptr (= Lq)
  const int32_t* kv_lens;  // [B] cached tokens per sequence (<= Lmax), or nullptr (= Lmax)
  int B, Lq, Lmax, Hq, Hkv, G, NKmax, topk, n_init, n_local;
  int score_mode, pool_mode;  // kScore*, kPool*
  int nblk_cap;  // score slots per token (>= number of blocks in Lmax tokens, multiple of 32)
  float scale_log2;
  int tiles_per_bg;  // ceil(Lq / query rows per CTA)
  int stages;        // tensor-core kernel: Kc ring slots (2 or 3)
};

struct SelSmem {
  uint64_t full[kSelStages], empty[kSelStages];
  volatile int abort;
};

inline size_t sel_prefill_smem_bytes(int nblk_cap) {
  return 1024 + static_cast<size_t>(kSelStages) * kKcTileBytes + static_cast<size_t>(kSelWarps) * nblk_cap * 4 +
         kSelWarps * 256 * 4 + sizeof(SelSmem);
}

// Number of forced blocks for a query in block cur: 0..n_init-1 and cur-n_local+1..cur.
__device__ __forceinline__ int forced_count(int cur, int n_init, int n_local) {
  const int a = min(n_init, cur + 1);
  const int lo = max(max(cur - n_local + 1, 0), a);
  return a + max(0, cur - lo + 1);
}

// Loads this lane's A fragments of the group's 16 query rows (rows >= G read as 0).
__device__ __forceinline__ void load_q_frags(const __nv_bfloat16* qrow0, int G, uint32_t (&qa)[8][4]) {
  const int lane = threadIdx.x & 31;
  const int r0 = lane >> 2, q4 = lane & 3;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int r = r0 + ((e & 1) << 3);
      const int d = 16 * ks + 2 * q4 + ((e >> 1) << 3);
      qa[ks][e] = r < G ? *reinterpret_cast<const uint32_t*>(qrow0 + static_cast<long long>(r) * kHeadDim + d) : 0u;
    }
  }
}

// s (16 x 64) = Q (16 x 128) * tile^T, tile = 64 rows x 128 in the swizzled layout.
__device__ __forceinline__ void qk_tile(const uint32_t (&qa)[8][4], uint32_t tile, float (&s)[8][4]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
    for (int np = 0; np < 4; ++np) {
      const int mi = lane >> 3;
      const int row = 16 * np + (lane & 7) + ((mi >> 1) << 3);
      const int d = 16 * ks + ((mi & 1) << 3);
      uint32_t b0, b1, b2, b3;
      ldsm_x4(tile + (d >> 6) * (kKcTileBytes / 2) + sw128(row, (d & 63) >> 3), b0, b1, b2, b3);
      mma_bf16(s[2 * np], qa[ks], b0, b1);
      mma_bf16(s[2 * np + 1], qa[ks], b2, b3);
    }
  }
}

// grid = B * Hkv * tiles_per_bg (latest tiles first), block = 288.
__global__ void __launch_bounds__(kSelThreads, 1)
    select_prefill_kernel(const __grid_constant__ CUtensorMap tm_kc, const SelPrefillParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = align_smem(smem_raw, 1024);
  unsigned char* stages = base;
  uint32_t* keys_all = reinterpret_cast<uint32_t*>(stages + kSelStages * kKcTileBytes);
  uint32_t* hist_all = keys_all + kSelWarps * p.nblk_cap;
  SelSmem& S = *reinterpret_cast<SelSmem*>(hist_all + kSelWarps * 256);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long nbg = static_cast<long long>(p.B) * p.Hkv;
  const int tile = p.tiles_per_bg - 1 - static_cast<int>(blockIdx.x / nbg);
  const long long bg = blockIdx.x % nbg;
  const int b = static_cast<int>(bg / p.Hkv), g = static_cast<int>(bg % p.Hkv);
  const int t0 = tile * kSelWarps;  // first query row of the tile
  const ChunkLens cl = chunk_lens(p.q_lens, p.kv_lens, b, p.Lq, p.Lmax);
  if (t0 >= cl.q_len) return;  // padding rows only (uniform over the CTA)
  const int off = cl.kv_len - cl.q_len;  // position of query row 0
  const int imax_last = last_visible_kernel(off + min(t0 + kSelWarps - 1, cl.q_len - 1));
  // pass A (the per-head lse) only for softmax-sum scoring
  const int TA = (imax_last >= 0 && p.score_mode == kScoreSoftmaxSum) ? imax_last / kKcTile + 1 : 0;
  const int TB = imax_last >= 0 ? (imax_last + 1) / kKcTile + 1 : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSelStages; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], kSelWarps);
    }
    S.abort = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kSelWarps) {
    if (lane == 0) {
      prefetch_tmap(&tm_kc);
      const int row0 = static_cast<int>(bg * p.NKmax);
      for (int n = 0; n < TA + TB; ++n) {
        const int st = n % kSelStages, u = n / kSelStages;
        if (u > 0) mbar_wait(&S.empty[st], (u - 1) & 1, &S.abort);
        if (S.abort) break;
        const int c = n < TA ? n : n - TA;
        unsigned char* dst = stages + st * kKcTileBytes;
        mbar_arrive_expect_tx(&S.full[st], kKcTileBytes);
        tma_load_2d(dst, &tm_kc, &S.full[st], 0, row0 + c * kKcTile);
        tma_load_2d(dst + kKcTileBytes / 2, &tm_kc, &S.full[st], 64, row0 + c * kKcTile);
      }
    }
    return;
  }

  // ------------------------------------------------------------ consumer warp
  const int t_raw = t0 + warp;
  const bool tok_ok = t_raw < cl.q_len;
  const int trow = tok_ok ? t_raw : cl.q_len - 1;  // query row (rows past q_len compute, write nothing)
  const int t = off + trow;                        // its position in the sequence
  const int imax = last_visible_kernel(t);
  const int cur = t / kBlock;
  const int q4 = lane & 3, r0 = lane >> 2;
  const bool row0_ok = r0 < p.G, row1_ok = r0 + 8 < p.G;

  uint32_t qa[8][4];
  load_q_frags(p.q + ((static_cast<long long>(b) * p.Lq + trow) * p.Hq + g * p.G) * kHeadDim, p.G, qa);

  // pass A: log-sum-exp over the visible kernels (base 2)
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  float s[8][4];
  for (int n = 0; n < TA; ++n) {
    const int st = n % kSelStages;
    mbar_wait(&S.full[st], (n / kSelStages) & 1, &S.abort);
    qk_tile(qa, smem_u32(stages + st * kKcTileBytes), s);
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.empty[st]);
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const bool ok = n * kKcTile + 8 * nt + 2 * q4 + e <= imax;
        s[nt][e] = ok ? s[nt][e] * p.scale_log2 : -INFINITY;
        s[nt][2 + e] = ok ? s[nt][2 + e] * p.scale_log2 : -INFINITY;
        mx0 = fmaxf(mx0, s[nt][e]);
        mx1 = fmaxf(mx1, s[nt][2 + e]);
      }
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    if (mn0 == -INFINITY && mn1 == -INFINITY) continue;  // nothing visible yet in this tile
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      a0 += ex2(s[nt][0] - mn0) + ex2(s[nt][1] - mn0);
      a1 += ex2(s[nt][2] - mn1) + ex2(s[nt][3] - mn1);
    }
    l0 = l0 * ex2(m0 - mn0) + a0;
    l1 = l1 * ex2(m1 - mn1) + a1;
    m0 = mn0;
    m1 = mn1;
  }
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const float lse0 = l0 > 0.f ? m0 + lg2(l0) : INFINITY;
  const float lse1 = l1 > 0.f ? m1 + lg2(l1) : INFINITY;

  uint32_t* keys = keys_all + warp * p.nblk_cap;
  for (int j = lane; j <= cur; j += 32) keys[j] = 0u;
  __syncwarp();

  // pass B: block scores
  const bool inside = p.pool_mode == kPoolInside, logit = p.score_mode == kScoreLogitSum;
  float carry0 = -INFINITY, carry1 = -INFINITY;
  const int base4 = lane & ~3;
  for (int n = TA; n < TA + TB; ++n) {
    const int c = n - TA;
    const int st = n % kSelStages;
    mbar_wait(&S.full[st], (n / kSelStages) & 1, &S.abort);
    qk_tile(qa, smem_u32(stages + st * kKcTileBytes), s);
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.empty[st]);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const bool ok = c * kKcTile + 8 * nt + 2 * q4 + e <= imax;
        s[nt][e] = ok ? s[nt][e] * p.scale_log2 : -INFINITY;
        s[nt][2 + e] = ok ? s[nt][2 + e] * p.scale_log2 : -INFINITY;
      }
      // group of 4 kernels: cols 0-3 (lanes q4 0,1) or 4-7 (lanes q4 2,3) of this n-tile;
      // with inside pooling the group's last kernel (4j + 3, this lane's second column on
      // odd q4) leaves the block's pool
      const bool drop_last = inside && (q4 & 1);
      float g0 = drop_last ? s[nt][0] : fmaxf(s[nt][0], s[nt][1]);
      float g1 = drop_last ? s[nt][2] : fmaxf(s[nt][2], s[nt][3]);
      g0 = fmaxf(g0, __shfl_xor_sync(0xffffffffu, g0, 1));
      g1 = fmaxf(g1, __shfl_xor_sync(0xffffffffu, g1, 1));
      // the kernel before each group (4j - 1) straddles blocks j-1 and j (overlap pooling)
      const float lastA0 = __shfl_sync(0xffffffffu, s[nt][1], base4 | 1);
      const float lastA1 = __shfl_sync(0xffffffffu, s[nt][3], base4 | 1);
      const float lastB0 = __shfl_sync(0xffffffffu, s[nt][1], base4 | 3);
      const float lastB1 = __shfl_sync(0xffffffffu, s[nt][3], base4 | 3);
      const float mb0 = inside ? g0 : fmaxf(g0, q4 < 2 ? carry0 : lastA0);
      const float mb1 = inside ? g1 : fmaxf(g1, q4 < 2 ? carry1 : lastA1);
      carry0 = lastB0;
      carry1 = lastB1;
      float pr = logit ? ((row0_ok ? mb0 : 0.f) + (row1_ok ? mb1 : 0.f))
                       : ((row0_ok ? ex2(mb0 - lse0) : 0.f) + (row1_ok ? ex2(mb1 - lse1) : 0.f));
      pr += __shfl_xor_sync(0xffffffffu, pr, 4);
      pr += __shfl_xor_sync(0xffffffffu, pr, 8);
      pr += __shfl_xor_sync(0xffffffffu, pr, 16);
      const int j = c * 16 + 2 * nt + (q4 >> 1);
      if ((lane == 0 || lane == 2) && j <= cur) {
        const bool eligible = block_eligible(j, imax, p.pool_mode);
        const bool forced = j < p.n_init || j > cur - p.n_local;
        if (eligible && !forced) keys[j] = score_key(pr, p.score_mode);
      }
    }
  }
  __syncwarp();

  const int want = p.topk - forced_count(cur, p.n_init, p.n_local);
  const TopkThreshold th = warp_radix_threshold(keys, cur + 1, want, hist_all + warp * 256);
  if (tok_ok) {
    int32_t* out = p.idx + ((bg * p.Lq + trow) * static_cast<long long>(p.topk));
    warp_emit_selection(keys, cur + 1, th, cur, p.n_init, p.n_local, p.topk, out);
  }
}

}  // namespace infllmv2
