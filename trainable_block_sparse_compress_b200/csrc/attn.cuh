// attn.cuh -- exact attention over the selected KV blocks on m16n8k16 tensor-core
// MMAs: the split decode path (few sequences), and the work-item mapping, parameters
// and per-block update shared with the other attention kernels.  Prefill and prefill
// chunks run on attn_tc_kernel (attn_tc.cuh) for every group size.
//
// MiniCPM4 summary page (端设备上的超高效大型语言模型) s2.1.3: each token attends only to
// its most relevant KV blocks; s2.1.2: the query heads of one group share those blocks,
// which is what lets a 64-key block be fetched once for the whole group.
//
// Work item = (sequence b, kv-head g, query token t[, split s]).  A persistent CTA
// walks items; its producer warp compacts the item's block list, stages the group's
// 16 query rows and streams every selected K and V block (64 x 128 bf16 each) through
// a ring of shared-memory stages with TMA (128-byte swizzle, no multicast).  Four
// consumer warps read every stage in order, warp w taking keys [16 w, 16 w + 16) of
// each block; each keeps an online softmax for the 16 heads (rows) over its keys and
// accumulates O = P V with m16n8k16 bf16 MMAs (fp32 accumulators).  At the end of an
// item the four partial states are merged in shared memory.
// For decode with very few sequences, an item's blocks are split over several items
// that write partial (O, lse) to the workspace; attn_merge_kernel combines them.
#pragma once
#include "common.cuh"

namespace infllmv2 {

constexpr int kAttnConsumers = 4;
constexpr int kAttnThreads = 32 * (kAttnConsumers + 1);
constexpr int kAttnStages = 5;
constexpr int kKvTileBytes = kBlock * kHeadDim * 2;  // 16 KB: one 64 x 128 bf16 block
constexpr int kAttnStageBytes = 2 * kKvTileBytes;    // K then V
constexpr int kQTileBytes = kGroupRows * kHeadDim * 2;  // 4 KB
constexpr int kMaxTopk = 256;
constexpr int kMergeRowFloats = kHeadDim + 4;

struct AttnParams {
  const int32_t* idx;      // [B, Hkv, Lq, topk]
  const int32_t* lens;     // decode: [B] sequence lengths; prefill / chunk: nullptr
  const int32_t* q_lens;   // chunk: [B] queries per sequence (<= Lq), or nullptr (= Lq)
  const int32_t* kv_lens;  // chunk: [B] cached tokens per sequence (<= Lmax), or nullptr (= Lmax)
  int B, Hq, Hkv, G, Lq, Lmax, topk;
  int n_splits;          // decode: splits per (b, g); prefill: 1
  int blocks_per_split;  // decode: selected blocks per split
  float scale_log2;      // softmax scale * log2(e)
  long long num_items;
  __nv_bfloat16* o;  // prefill: [B, Lq, Hq, d]
  float* lse;        // prefill: [B, Hq, Lq] or nullptr
  float* part_o;     // decode: [B*Hkv, n_splits, 16, d] normalised partial outputs
  float* part_lse;   // decode: [B*Hkv, n_splits, 16] natural-log partial lse
};

// A work item: query row `row` of sequence b (its row in Q, O, lse and the block lists),
// which sits at position t of the sequence; `valid` is false for padding rows of a
// chunk (row >= q_lens[b]), which are skipped and not written.
struct AttnItem {
  int b, g, t, row, split, qrow;
  int kv_len;  // cached tokens of sequence b: key rows at or past it are not the sequence's
  bool valid;
  long long bg;
};

__device__ __forceinline__ AttnItem attn_item(const AttnParams& p, long long item) {
  AttnItem it;
  if (p.lens == nullptr) {
    // prefill: one (sequence, kv-head) after another, so the blocks in use at a time are
    // those of one K/V stream (64 MB at 128K, which L2 holds); latest tokens first
    it.bg = item / p.Lq;
    it.row = p.Lq - 1 - static_cast<int>(item % p.Lq);
    it.split = 0;
  } else {
    it.bg = item / p.n_splits;
    it.split = static_cast<int>(item % p.n_splits);
    it.row = 0;
  }
  it.b = static_cast<int>(it.bg / p.Hkv);
  it.g = static_cast<int>(it.bg % p.Hkv);
  if (p.lens != nullptr) {
    it.t = min(p.lens[it.b], p.Lmax) - 1;  // -1 (no key) when lens[b] <= 0
    it.kv_len = it.t + 1;
    it.valid = true;
    it.qrow = it.b * p.Hq + it.g * p.G;
  } else {
    const ChunkLens c = chunk_lens(p.q_lens, p.kv_lens, it.b, p.Lq, p.Lmax);
    it.kv_len = c.kv_len;
    it.valid = it.row < c.q_len;
    it.t = it.valid ? c.kv_len - c.q_len + it.row : -1;
    it.qrow = (it.b * p.Lq + it.row) * p.Hq + it.g * p.G;
  }
  return it;
}

struct AttnSmem {
  uint64_t full[kAttnStages], empty[kAttnStages], qfull[2], qempty[2];
  int n_blocks[2];
  int list[2][kMaxTopk];
  float m[kAttnConsumers][kGroupRows], l[kAttnConsumers][kGroupRows];
  volatile int abort;
};

constexpr size_t attn_smem_bytes() {
  return 1024 /*alignment slack*/ + static_cast<size_t>(kAttnStages) * kAttnStageBytes + 2 * kQTileBytes +
         static_cast<size_t>(kAttnConsumers) * kGroupRows * kMergeRowFloats * 4 + sizeof(AttnSmem);
}

// One consumer warp's share (keys [kofs, kofs + 16)) of a staged K/V block j (K then V,
// 64 x 128 bf16 each, 128-byte swizzle) for the query rows at position t: S = Q K^T,
// online softmax in base 2 (running max m, row sum l) and O += P V.  Keys past t are
// masked; their V rows are zeroed first so that they contribute exactly 0.
__device__ __forceinline__ void attn_block_update(unsigned char* sk_ptr, int j, int t, int kofs,
                                                  const uint32_t (&qa)[8][4], float scale_log2, float& m0,
                                                  float& m1, float& l0, float& l1, float (&o)[16][4]) {
  const int lane = threadIdx.x & 31;
  const int q4 = lane & 3;
  const uint32_t sk = smem_u32(sk_ptr);
  const uint32_t sv = sk + kKvTileBytes;
  const int valid = t - j * kBlock + 1;  // keys of this block at positions <= t
  const bool partial = valid < kofs + 16;  // some of this warp's 16 keys lie past t
  if (partial) {
    // zero this warp's V rows past t so that masked keys contribute exactly 0
    uint4* vrow = reinterpret_cast<uint4*>(sk_ptr + kKvTileBytes);
    for (int c = max(valid, kofs) * 8 + lane; c < (kofs + 16) * 8; c += 32) {
      const int r = c >> 3, ch = c & 7;
      vrow[r * 8 + ch] = make_uint4(0, 0, 0, 0);
      vrow[(kKvTileBytes / 2) / 16 + r * 8 + ch] = make_uint4(0, 0, 0, 0);
    }
    __syncwarp();
  }

  // S = Q K^T for this warp's 16 keys: 16 x 16
  float s[2][4];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const int mi = lane >> 3;
    const int key = kofs + (lane & 7) + ((mi >> 1) << 3);
    const int d = 16 * ks + ((mi & 1) << 3);
    uint32_t b0, b1, b2, b3;
    ldsm_x4(sk + (d >> 6) * (kKvTileBytes / 2) + sw128(key, (d & 63) >> 3), b0, b1, b2, b3);
    mma_bf16(s[0], qa[ks], b0, b1);
    mma_bf16(s[1], qa[ks], b2, b3);
  }

  // online softmax (base 2)
  float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int col = kofs + 8 * nt + 2 * q4 + e;
      const bool ok = !partial || col < valid;
      s[nt][e] = ok ? s[nt][e] * scale_log2 : -INFINITY;
      s[nt][2 + e] = ok ? s[nt][2 + e] * scale_log2 : -INFINITY;
      mx0 = fmaxf(mx0, s[nt][e]);
      mx1 = fmaxf(mx1, s[nt][2 + e]);
    }
  }
  mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
  mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
  mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
  mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
  const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
  if (mn0 != -INFINITY) {  // all 16 keys of this warp may lie past t
    const float al0 = ex2(m0 - mn0), al1 = ex2(m1 - mn1);
    m0 = mn0;
    m1 = mn1;
    float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      s[nt][0] = ex2(s[nt][0] - mn0);
      s[nt][1] = ex2(s[nt][1] - mn0);
      s[nt][2] = ex2(s[nt][2] - mn1);
      s[nt][3] = ex2(s[nt][3] - mn1);
      rs0 += s[nt][0] + s[nt][1];
      rs1 += s[nt][2] + s[nt][3];
    }
    l0 = l0 * al0 + rs0;
    l1 = l1 * al1 + rs1;
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      o[nt][0] *= al0;
      o[nt][1] *= al0;
      o[nt][2] *= al1;
      o[nt][3] *= al1;
    }

    // O += P V : P (16 x 16) from registers, V rows of this warp via transposed ldmatrix
    uint32_t pa[4];
    pa[0] = pack_bf16(s[0][0], s[0][1]);
    pa[1] = pack_bf16(s[0][2], s[0][3]);
    pa[2] = pack_bf16(s[1][0], s[1][1]);
    pa[3] = pack_bf16(s[1][2], s[1][3]);
#pragma unroll
    for (int dp = 0; dp < 8; ++dp) {
      const int mi = lane >> 3;
      const int key = kofs + (lane & 7) + ((mi & 1) << 3);
      const int d = 16 * dp + ((mi >> 1) << 3);
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(sv + (d >> 6) * (kKvTileBytes / 2) + sw128(key, (d & 63) >> 3), b0, b1, b2, b3);
      mma_bf16(o[2 * dp], pa, b0, b1);
      mma_bf16(o[2 * dp + 1], pa, b2, b3);
    }
  }
  if (partial) fence_proxy_async_smem();
}

__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = align_smem(smem_raw, 1024);
  unsigned char* stages = base;
  unsigned char* qtiles = stages + kAttnStages * kAttnStageBytes;
  float* merge_o = reinterpret_cast<float*>(qtiles + 2 * kQTileBytes);
  AttnSmem& S = *reinterpret_cast<AttnSmem*>(merge_o + kAttnConsumers * kGroupRows * kMergeRowFloats);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kAttnStages; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], kAttnConsumers);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&S.qfull[s], 1);
      mbar_init(&S.qempty[s], kAttnConsumers);
    }
    S.abort = 0;
    fence_mbar_init();
  }
  if (warp == kAttnConsumers && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  __syncthreads();

  if (warp == kAttnConsumers) {
    // ------------------------------------------------------------ producer warp
    long long gblk = 0;
    int it = 0;
    for (long long item = blockIdx.x; item < p.num_items; item += gridDim.x, ++it) {
      const int slot = it & 1, use = it >> 1;
      if (use > 0) mbar_wait(&S.qempty[slot], (use - 1) & 1, &S.abort);
      const AttnItem a = attn_item(p, item);
      const int cur = a.t >= 0 ? a.t / kBlock : -1;
      const int32_t* row = p.idx + ((a.bg * p.Lq + a.row) * static_cast<long long>(p.topk));
      const int lo = a.split * p.blocks_per_split;
      const int hi = p.lens ? lo + p.blocks_per_split : p.topk;
      int count = 0;
      for (int e0 = 0; e0 < p.topk; e0 += 32) {
        const int e = e0 + lane;
        const int j = (e < p.topk && a.valid) ? row[e] : -1;
        const bool ok = j >= 0 && j <= cur;
        const unsigned msk = __ballot_sync(0xffffffffu, ok);
        const int pos = count + __popc(msk & ((1u << lane) - 1u));
        if (ok && pos >= lo && pos < hi) S.list[slot][pos - lo] = j;
        count += __popc(msk);
      }
      const int n = max(0, min(count, hi) - lo);
      if (lane == 0) S.n_blocks[slot] = n;
      __threadfence_block();
      __syncwarp();
      if (lane == 0) {
        unsigned char* qs = qtiles + slot * kQTileBytes;
        mbar_arrive_expect_tx(&S.qfull[slot], kQTileBytes);
        tma_load_2d(qs, &tm_q, &S.qfull[slot], 0, a.qrow);
        tma_load_2d(qs + kQTileBytes / 2, &tm_q, &S.qfull[slot], 64, a.qrow);
        const long long kvrow0 = a.bg * p.Lmax;
        for (int i = 0; i < n; ++i, ++gblk) {
          const int st = static_cast<int>(gblk % kAttnStages);
          const long long u = gblk / kAttnStages;
          if (u > 0) mbar_wait(&S.empty[st], static_cast<uint32_t>((u - 1) & 1), &S.abort);
          if (S.abort) continue;
          const int krow = static_cast<int>(kvrow0 + static_cast<long long>(S.list[slot][i]) * kBlock);
          unsigned char* sk = stages + st * kAttnStageBytes;
          mbar_arrive_expect_tx(&S.full[st], kAttnStageBytes);
          tma_load_2d(sk, &tm_k, &S.full[st], 0, krow);
          tma_load_2d(sk + kKvTileBytes / 2, &tm_k, &S.full[st], 64, krow);
          tma_load_2d(sk + kKvTileBytes, &tm_v, &S.full[st], 0, krow);
          tma_load_2d(sk + kKvTileBytes + kKvTileBytes / 2, &tm_v, &S.full[st], 64, krow);
        }
      } else {
        gblk += n;
      }
      gblk = __shfl_sync(0xffffffffu, gblk, 0);
    }
    return;
  }

  // --------------------------------------------------------------- consumer warps
  const int cw = warp;
  const int q4 = lane & 3, r0 = lane >> 2;
  long long gbase = 0;
  int it = 0;
  for (long long item = blockIdx.x; item < p.num_items; item += gridDim.x, ++it) {
    const int slot = it & 1, use = it >> 1;
    mbar_wait(&S.qfull[slot], use & 1, &S.abort);
    const AttnItem a = attn_item(p, item);
    const int n = S.n_blocks[slot];

    // Q fragments (16 rows x 128) from the swizzled tile
    uint32_t qa[8][4];
    {
      const uint32_t qs = smem_u32(qtiles + slot * kQTileBytes);
      const int mi = lane >> 3;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const int row = (lane & 7) + ((mi & 1) << 3);
        const int d = 16 * ks + ((mi >> 1) << 3);
        ldsm_x4(qs + (d >> 6) * (kQTileBytes / 2) + sw128(row, (d & 63) >> 3), qa[ks][0], qa[ks][1], qa[ks][2],
                qa[ks][3]);
      }
    }

    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    float o[16][4];
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;

    // every consumer warp takes every block, keys [16 cw, 16 cw + 16) of it, so each warp
    // consumes the ring's stages strictly in order
    const int kofs = 16 * cw;
    for (int i = 0; i < n; ++i) {
      const long long gb = gbase + i;
      const int st = static_cast<int>(gb % kAttnStages);
      mbar_wait(&S.full[st], static_cast<uint32_t>((gb / kAttnStages) & 1), &S.abort);
      attn_block_update(stages + st * kAttnStageBytes, S.list[slot][i], a.t, kofs, qa, p.scale_log2, m0, m1, l0,
                        l1, o);
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.empty[st]);
    }
    gbase += n;
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.qempty[slot]);

    // ---- merge the four warps' partial softmax states
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    float* mo = merge_o + cw * kGroupRows * kMergeRowFloats;
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      const int c = 8 * nt + 2 * q4;
      mo[r0 * kMergeRowFloats + c] = o[nt][0];
      mo[r0 * kMergeRowFloats + c + 1] = o[nt][1];
      mo[(r0 + 8) * kMergeRowFloats + c] = o[nt][2];
      mo[(r0 + 8) * kMergeRowFloats + c + 1] = o[nt][3];
    }
    if (q4 == 0) {
      S.m[cw][r0] = m0;
      S.m[cw][r0 + 8] = m1;
      S.l[cw][r0] = l0;
      S.l[cw][r0 + 8] = l1;
    }
    named_bar_sync(1, 32 * kAttnConsumers);
    // warp cw finalises rows 4cw .. 4cw+3; lane covers columns 4 lane .. 4 lane + 3
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
      const int r = 4 * cw + rr;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kAttnConsumers; ++w) M = fmaxf(M, S.m[w][r]);
      float wts[kAttnConsumers], L = 0.f;
#pragma unroll
      for (int w = 0; w < kAttnConsumers; ++w) {
        wts[w] = (M == -INFINITY) ? 0.f : ex2(S.m[w][r] - M);
        L += wts[w] * S.l[w][r];
      }
      const float inv = L > 0.f ? 1.f / L : 0.f;
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int w = 0; w < kAttnConsumers; ++w) {
        const float4 v =
            *reinterpret_cast<const float4*>(merge_o + (w * kGroupRows + r) * kMergeRowFloats + 4 * lane);
        acc[0] += wts[w] * v.x;
        acc[1] += wts[w] * v.y;
        acc[2] += wts[w] * v.z;
        acc[3] += wts[w] * v.w;
      }
      const float lse_nat = L > 0.f ? (M + lg2(L)) * 0.6931471805599453f : -INFINITY;
      if (r < p.G && a.valid) {
        if (p.lens == nullptr) {
          __nv_bfloat16* dst = p.o + (static_cast<long long>(a.qrow) + r) * kHeadDim + 4 * lane;
          uint2 pk;
          pk.x = pack_bf16(acc[0] * inv, acc[1] * inv);
          pk.y = pack_bf16(acc[2] * inv, acc[3] * inv);
          *reinterpret_cast<uint2*>(dst) = pk;
          if (p.lse != nullptr && lane == 0)
            p.lse[(static_cast<long long>(a.b) * p.Hq + a.g * p.G + r) * p.Lq + a.row] = lse_nat;
        } else {
          const long long prow = (a.bg * p.n_splits + a.split) * kGroupRows + r;
          *reinterpret_cast<float4*>(p.part_o + prow * kHeadDim + 4 * lane) =
              make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
          if (lane == 0) p.part_lse[prow] = lse_nat;
        }
      }
    }
    named_bar_sync(1, 32 * kAttnConsumers);
  }
}

// Combines the decode splits: o = sum_s exp(lse_s - lse) o_s, lse = log sum_s exp(lse_s).
// grid = B * Hkv * G (one head row each), block = 128 (one column each; thread s also
// carries split s's weight).
constexpr int kMaxDecodeSplits = 128;

__global__ void __launch_bounds__(128) attn_merge_kernel(const float* __restrict__ part_o,
                                                         const float* __restrict__ part_lse, int n_splits,
                                                         int Hq, int Hkv, int G, __nv_bfloat16* __restrict__ o,
                                                         float* __restrict__ lse) {
  __shared__ float w[kMaxDecodeSplits];
  __shared__ float red_m[4], red_l[4];
  const long long bg = blockIdx.x / G;
  const int r = static_cast<int>(blockIdx.x % G);
  const int b = static_cast<int>(bg / Hkv), g = static_cast<int>(bg % Hkv);
  const int d = threadIdx.x, lane = d & 31, wp = d >> 5;
  const float x = d < n_splits ? part_lse[(bg * n_splits + d) * kGroupRows + r] : -INFINITY;
  float M = x;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  if (lane == 0) red_m[wp] = M;
  __syncthreads();
  M = fmaxf(fmaxf(red_m[0], red_m[1]), fmaxf(red_m[2], red_m[3]));
  const float e = (d < n_splits && M != -INFINITY) ? __expf(x - M) : 0.f;
  if (d < n_splits) w[d] = e;
  float L = e;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
  if (lane == 0) red_l[wp] = L;
  __syncthreads();
  L = (red_l[0] + red_l[1]) + (red_l[2] + red_l[3]);
  float acc = 0.f;
#pragma unroll 4
  for (int s = 0; s < n_splits; ++s) acc += w[s] * part_o[((bg * n_splits + s) * kGroupRows + r) * kHeadDim + d];
  const long long orow = static_cast<long long>(b) * Hq + g * G + r;
  o[orow * kHeadDim + d] = __float2bfloat16_rn(L > 0.f ? acc / L : 0.f);
  if (lse != nullptr && d == 0) lse[orow] = L > 0.f ? M + logf(L) : -INFINITY;
}

}  // namespace infllmv2
