// attn_bwd.cuh -- backward of the sparse attention over fixed selected blocks.
//
// MiniCPM4 summary page (端设备上的超高效大型语言模型) s2.1 and s2.1.3: InfLLM v2 is a
// trainable sparse attention, each token attending only to its selected KV blocks.  The
// top-k block choice is constant almost everywhere, so gradients reach q, k and v through
// the attention over the selected blocks only; the block lists are fixed inputs here.
// With P = softmax(scale q K_J^T) over the keys J of a row's blocks (cut at the row's
// position), D = sum_d dO O (= sum_u P_u dP_u):
//   dP_u = dO . V_u,   dS_u = P_u (dP_u - D),
//   dq   = scale sum_u dS_u K_u,   dK_u += scale dS_u q,   dV_u += P_u dO.
// P is recomputed from the forward's log-sum-exp.
//
// Kernels, in launch order:
//   bwd_delta_kernel   D per (token, q-head): one warp per row;
//   bwd_count_kernel / bwd_scan_kernel / bwd_fill_kernel
//                      the inverse of the block lists: for every (sequence, kv-head,
//                      block) the query rows that selected it, cut into segments of at
//                      most kBwdSeg rows (block 0 is in every row's list);
//   bwd_dq_kernel      token-major like attn_kernel: per (sequence, kv-head, token) the
//                      selected K/V blocks stream through a TMA ring; four warps take 16
//                      keys of each block and accumulate dq (16 heads x 128) with
//                      m16n8k16 MMAs, merged at the end of the item;
//   bwd_dkdv_tc_kernel block-major, on the tcgen05 tensor cores (csrc/attn_bwd_tc.cuh): per
//                      segment the block's K and V stay in shared memory while the segment's
//                      tokens stream their Q and dO rows 8 at a time; dK and dV accumulate in
//                      TMEM and are added to the fp32 workspace (atomics: a block's segments
//                      run on different CTAs, so the summation order of dK / dV may vary
//                      between runs, within fp32 rounding);
//   bwd_cast_kernel    the fp32 dK / dV to bf16.
#pragma once
#include "attn.cuh"
#include "common.cuh"

namespace infllmv2 {

constexpr int kBwdSeg = 128;       // query rows per dK/dV work item at most
constexpr int kBwdConsumers = 4;
constexpr int kBwdThreads = 32 * (kBwdConsumers + 1);
constexpr int kBwdKvStages = 4;    // dq kernel: K+V block stages (32 KB each)
constexpr int kBwdTokBytes = 2 * kQTileBytes;  // dq kernel: a token's Q then dO rows
constexpr int kBwdDqRowFloats = kHeadDim + 4;

struct BwdParams {
  const int32_t* idx;    // [B, Hkv, L, topk]
  const float* lse;      // [B, Hq, L] natural-log normaliser of the forward
  const float* delta;    // [B, Hq, L] sum_d dO O
  const int32_t* cnt;    // [B*Hkv*nblk] rows that selected each block
  const int32_t* off;    // [B*Hkv*nblk] start of each block's row list
  const int32_t* segoff; // [B*Hkv*nblk + 1] first segment of each block; [n] = all segments
  const int32_t* list;   // row lists
  int B, Hq, Hkv, G, L, topk, nblk;
  float scale, scale_log2;
  long long num_items;   // dq kernel: B * Hkv * L
  __nv_bfloat16* dq;     // [B, L, Hq, d]
  float* dk32;           // [B, Hkv, L, d], zeroed before the dkdv kernel
  float* dv32;
};

// D[b, h, t] = sum_d dO[b, t, h, d] * O[b, t, h, d].  One warp per row (b, t, h).
__global__ void __launch_bounds__(256) bwd_delta_kernel(const __nv_bfloat16* __restrict__ d_o,
                                                        const __nv_bfloat16* __restrict__ o, int B, int L, int Hq,
                                                        float* __restrict__ delta) {
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= static_cast<long long>(B) * L * Hq) return;
  const uint2 a = *reinterpret_cast<const uint2*>(d_o + row * kHeadDim + 4 * lane);
  const uint2 c = *reinterpret_cast<const uint2*>(o + row * kHeadDim + 4 * lane);
  const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
  const __nv_bfloat162* c2 = reinterpret_cast<const __nv_bfloat162*>(&c);
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float2 x = __bfloat1622float2(a2[i]), y = __bfloat1622float2(c2[i]);
    s = fmaf(x.x, y.x, fmaf(x.y, y.y, s));
  }
#pragma unroll
  for (int o2 = 16; o2 > 0; o2 >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o2);
  if (lane == 0) {
    const int h = static_cast<int>(row % Hq);
    const long long bt = row / Hq;
    const int t = static_cast<int>(bt % L), b = static_cast<int>(bt / L);
    delta[(static_cast<long long>(b) * Hq + h) * L + t] = s;
  }
}

// cnt[bg * nblk + j] = number of rows t of (b, g) whose list holds block j (entries
// outside [0, t / 64] are ignored; a row lists a block at most once, as the forward
// requires).  One thread per row.
__global__ void __launch_bounds__(256) bwd_count_kernel(const int32_t* __restrict__ idx, int rows, int L, int topk,
                                                        int nblk, int32_t* __restrict__ cnt) {
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= rows) return;
  const int t = r % L;
  const long long bg = r / L;
  const int32_t* e = idx + static_cast<long long>(r) * topk;
  for (int s = 0; s < topk; ++s) {
    const int j = e[s];
    if (j >= 0 && j <= t / kBlock) atomicAdd(&cnt[bg * nblk + j], 1);
  }
}

// Exclusive scans over the n = B * Hkv * nblk counts, in one CTA of 1024 threads:
// off (row lists) and segoff (segments of at most kBwdSeg rows; segoff[n] = total).
__global__ void __launch_bounds__(1024) bwd_scan_kernel(const int32_t* __restrict__ cnt, int n,
                                                        int32_t* __restrict__ off, int32_t* __restrict__ segoff) {
  __shared__ int wsum[2][32];
  __shared__ int carry[2];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) carry[0] = carry[1] = 0;
  __syncthreads();
  for (int base = 0; base < n; base += 1024) {
    const int i = base + tid;
    const int c = i < n ? cnt[i] : 0;
    const int sg = (c + kBwdSeg - 1) / kBwdSeg;
    int a = c, s = sg;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int ya = __shfl_up_sync(0xffffffffu, a, o), ys = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) {
        a += ya;
        s += ys;
      }
    }
    if (lane == 31) {
      wsum[0][warp] = a;
      wsum[1][warp] = s;
    }
    __syncthreads();
    if (warp == 0) {
      int x = wsum[0][lane], y = wsum[1][lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int yx = __shfl_up_sync(0xffffffffu, x, o), yy = __shfl_up_sync(0xffffffffu, y, o);
        if (lane >= o) {
          x += yx;
          y += yy;
        }
      }
      wsum[0][lane] = x;
      wsum[1][lane] = y;
    }
    __syncthreads();
    const int pa = (warp > 0 ? wsum[0][warp - 1] : 0) + a - c + carry[0];
    const int ps = (warp > 0 ? wsum[1][warp - 1] : 0) + s - sg + carry[1];
    if (i < n) {
      off[i] = pa;
      segoff[i] = ps;
    }
    __syncthreads();
    if (tid == 1023) {
      carry[0] = pa + c;
      carry[1] = ps + sg;
    }
    __syncthreads();
  }
  if (tid == 0) segoff[n] = carry[1];
}

// list[off[bg * nblk + j] + k] = t for the k-th row t of (b, g) that selected block j
// (k from an atomic cursor: the order within a block's list may vary between runs).
__global__ void __launch_bounds__(256) bwd_fill_kernel(const int32_t* __restrict__ idx, int rows, int L, int topk,
                                                       int nblk, const int32_t* __restrict__ off,
                                                       int32_t* __restrict__ cursor, int32_t* __restrict__ list) {
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= rows) return;
  const int t = r % L;
  const long long bg = r / L;
  const int32_t* e = idx + static_cast<long long>(r) * topk;
  for (int s = 0; s < topk; ++s) {
    const int j = e[s];
    if (j < 0 || j > t / kBlock) continue;
    const long long e2 = bg * nblk + j;
    list[off[e2] + atomicAdd(&cursor[e2], 1)] = t;
  }
}

// Loads A fragments (16 rows x 128, bf16, 128-byte swizzled tile of 2 x 64-column halves
// of `half_bytes` each) for rows row0 .. row0+15.
__device__ __forceinline__ void load_a_frags(uint32_t tile, int row0, int half_bytes, uint32_t (&fa)[8][4]) {
  const int lane = threadIdx.x & 31, mi = lane >> 3;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const int row = row0 + (lane & 7) + ((mi & 1) << 3);
    const int d = 16 * ks + ((mi >> 1) << 3);
    ldsm_x4(tile + (d >> 6) * half_bytes + sw128(row, (d & 63) >> 3), fa[ks][0], fa[ks][1], fa[ks][2], fa[ks][3]);
  }
}

// acc (16 x 16) = A (16 x 128, fragments) * rows^T, rows = 16 consecutive rows row0 ..
// of a swizzled tile (the B operand read K-major, as K in S = Q K^T).
__device__ __forceinline__ void mma_rows_t(const uint32_t (&fa)[8][4], uint32_t tile, int row0, int half_bytes,
                                           float (&acc)[2][4]) {
  const int lane = threadIdx.x & 31, mi = lane >> 3;
#pragma unroll
  for (int nt = 0; nt < 2; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const int row = row0 + (lane & 7) + ((mi >> 1) << 3);
    const int d = 16 * ks + ((mi & 1) << 3);
    uint32_t b0, b1, b2, b3;
    ldsm_x4(tile + (d >> 6) * half_bytes + sw128(row, (d & 63) >> 3), b0, b1, b2, b3);
    mma_bf16(acc[0], fa[ks], b0, b1);
    mma_bf16(acc[1], fa[ks], b2, b3);
  }
}

// out (16 x 128) += a (16 x 16, fragments) * rows (16 x 128), rows = 16 consecutive rows
// row0 .. of a swizzled tile (the B operand read through transposed ldmatrix, as V in
// O += P V).
__device__ __forceinline__ void mma_acc_rows(const uint32_t (&a)[4], uint32_t tile, int row0, int half_bytes,
                                             float (&out)[16][4]) {
  const int lane = threadIdx.x & 31, mi = lane >> 3;
#pragma unroll
  for (int dp = 0; dp < 8; ++dp) {
    const int row = row0 + (lane & 7) + ((mi & 1) << 3);
    const int d = 16 * dp + ((mi >> 1) << 3);
    uint32_t b0, b1, b2, b3;
    ldsm_x4_t(tile + (d >> 6) * half_bytes + sw128(row, (d & 63) >> 3), b0, b1, b2, b3);
    mma_bf16(out[2 * dp], a, b0, b1);
    mma_bf16(out[2 * dp + 1], a, b2, b3);
  }
}

// accumulator tile (16 x 16 fp32) -> A fragments (bf16)
__device__ __forceinline__ void acc_to_a(const float (&x)[2][4], uint32_t (&a)[4]) {
  a[0] = pack_bf16(x[0][0], x[0][1]);
  a[1] = pack_bf16(x[0][2], x[0][3]);
  a[2] = pack_bf16(x[1][0], x[1][1]);
  a[3] = pack_bf16(x[1][2], x[1][3]);
}

struct BwdDqSmem {
  uint64_t full[kBwdKvStages], empty[kBwdKvStages], qfull[2], qempty[2];
  int n_blocks[2];
  int list[2][kMaxTopk];
  volatile int abort;
};

constexpr size_t bwd_dq_smem_bytes() {
  return 1024 + static_cast<size_t>(kBwdKvStages) * kAttnStageBytes + 2 * kBwdTokBytes +
         static_cast<size_t>(kBwdConsumers) * kGroupRows * kBwdDqRowFloats * 4 + sizeof(BwdDqSmem);
}

// grid = min(items, SMs) persistent CTAs, block = 160.  Item = (b, g, t), latest first.
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const BwdParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = align_smem(smem_raw, 1024);
  unsigned char* stages = base;
  unsigned char* qtiles = stages + kBwdKvStages * kAttnStageBytes;  // per slot: Q then dO
  float* merge = reinterpret_cast<float*>(qtiles + 2 * kBwdTokBytes);
  BwdDqSmem& S = *reinterpret_cast<BwdDqSmem*>(merge + kBwdConsumers * kGroupRows * kBwdDqRowFloats);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kBwdKvStages; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], kBwdConsumers);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&S.qfull[s], 1);
      mbar_init(&S.qempty[s], kBwdConsumers);
    }
    S.abort = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kBwdConsumers) {
    // ------------------------------------------------------------ producer warp
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_do);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
    }
    long long gblk = 0;
    int it = 0;
    for (long long item = blockIdx.x; item < p.num_items; item += gridDim.x, ++it) {
      const int slot = it & 1, use = it >> 1;
      if (use > 0) mbar_wait(&S.qempty[slot], (use - 1) & 1, &S.abort);
      const long long bg = item / p.L;
      const int t = p.L - 1 - static_cast<int>(item % p.L);
      const int b = static_cast<int>(bg / p.Hkv), g = static_cast<int>(bg % p.Hkv);
      const int cur = t / kBlock;
      const int32_t* row = p.idx + (bg * p.L + t) * static_cast<long long>(p.topk);
      int count = 0;
      for (int e0 = 0; e0 < p.topk; e0 += 32) {
        const int e = e0 + lane;
        const int j = e < p.topk ? row[e] : -1;
        const bool ok = j >= 0 && j <= cur;
        const unsigned msk = __ballot_sync(0xffffffffu, ok);
        if (ok) S.list[slot][count + __popc(msk & ((1u << lane) - 1u))] = j;
        count += __popc(msk);
      }
      if (lane == 0) S.n_blocks[slot] = count;
      __threadfence_block();
      __syncwarp();
      if (lane == 0) {
        const int qrow = (b * p.L + t) * p.Hq + g * p.G;
        unsigned char* qs = qtiles + slot * kBwdTokBytes;
        mbar_arrive_expect_tx(&S.qfull[slot], kBwdTokBytes);
        tma_load_2d(qs, &tm_q, &S.qfull[slot], 0, qrow);
        tma_load_2d(qs + kQTileBytes / 2, &tm_q, &S.qfull[slot], 64, qrow);
        tma_load_2d(qs + kQTileBytes, &tm_do, &S.qfull[slot], 0, qrow);
        tma_load_2d(qs + kQTileBytes + kQTileBytes / 2, &tm_do, &S.qfull[slot], 64, qrow);
        const long long kvrow0 = bg * p.L;
        for (int i = 0; i < count; ++i, ++gblk) {
          const int st = static_cast<int>(gblk % kBwdKvStages);
          const long long u = gblk / kBwdKvStages;
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
        gblk += count;
      }
      gblk = __shfl_sync(0xffffffffu, gblk, 0);
    }
    return;
  }

  // --------------------------------------------------------------- consumer warps
  const int q4 = lane & 3, r0 = lane >> 2;
  const int kofs = 16 * warp;
  const float sl2 = p.scale_log2;
  long long gbase = 0;
  int it = 0;
  for (long long item = blockIdx.x; item < p.num_items; item += gridDim.x, ++it) {
    const int slot = it & 1, use = it >> 1;
    mbar_wait(&S.qfull[slot], use & 1, &S.abort);
    const long long bg = item / p.L;
    const int t = p.L - 1 - static_cast<int>(item % p.L);
    const int b = static_cast<int>(bg / p.Hkv), g = static_cast<int>(bg % p.Hkv);
    const int n = S.n_blocks[slot];
    const uint32_t qs = smem_u32(qtiles + slot * kBwdTokBytes);
    uint32_t qa[8][4], da[8][4];
    load_a_frags(qs, 0, kQTileBytes / 2, qa);
    load_a_frags(qs + kQTileBytes, 0, kQTileBytes / 2, da);
    // this lane's rows r0, r0 + 8: base-2 lse (rows past the group: +inf, so P = 0) and D
    float lse2[2], dl[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int h = r0 + 8 * i;
      const long long li = (static_cast<long long>(b) * p.Hq + g * p.G + h) * p.L + t;
      lse2[i] = h < p.G ? p.lse[li] * 1.4426950408889634f : INFINITY;
      dl[i] = h < p.G ? p.delta[li] : 0.f;
    }
    float dq[16][4];
#pragma unroll
    for (int c = 0; c < 16; ++c) dq[c][0] = dq[c][1] = dq[c][2] = dq[c][3] = 0.f;
    for (int i = 0; i < n; ++i) {
      const long long gb = gbase + i;
      const int st = static_cast<int>(gb % kBwdKvStages);
      mbar_wait(&S.full[st], static_cast<uint32_t>((gb / kBwdKvStages) & 1), &S.abort);
      const uint32_t sk = smem_u32(stages + st * kAttnStageBytes);
      const uint32_t sv = sk + kKvTileBytes;
      const int j = S.list[slot][i];
      float s[2][4], dp[2][4];
      mma_rows_t(qa, sk, kofs, kKvTileBytes / 2, s);   // S  = Q K^T   (16 heads x 16 keys)
      mma_rows_t(da, sv, kofs, kKvTileBytes / 2, dp);  // dP = dO V^T
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int key = j * kBlock + kofs + 8 * nt + 2 * q4 + (e & 1);
          const int ri = e >> 1;
          const float pr = key <= t ? ex2(fmaf(s[nt][e], sl2, -lse2[ri])) : 0.f;
          s[nt][e] = pr * (dp[nt][e] - dl[ri]);  // dS
        }
      }
      uint32_t dsa[4];
      acc_to_a(s, dsa);
      mma_acc_rows(dsa, sk, kofs, kKvTileBytes / 2, dq);  // dq += dS K
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.empty[st]);
    }
    gbase += n;
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.qempty[slot]);

    // merge the four warps' partial dq and write rows h < G
    float* mo = merge + warp * kGroupRows * kBwdDqRowFloats;
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const int col = 8 * c + 2 * q4;
      mo[r0 * kBwdDqRowFloats + col] = dq[c][0];
      mo[r0 * kBwdDqRowFloats + col + 1] = dq[c][1];
      mo[(r0 + 8) * kBwdDqRowFloats + col] = dq[c][2];
      mo[(r0 + 8) * kBwdDqRowFloats + col + 1] = dq[c][3];
    }
    named_bar_sync(1, 32 * kBwdConsumers);
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
      const int r = 4 * warp + rr;
      if (r < p.G) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int w = 0; w < kBwdConsumers; ++w) {
          const float4 v = *reinterpret_cast<const float4*>(merge + (w * kGroupRows + r) * kBwdDqRowFloats + 4 * lane);
          acc[0] += v.x;
          acc[1] += v.y;
          acc[2] += v.z;
          acc[3] += v.w;
        }
        __nv_bfloat16* dst = p.dq + ((static_cast<long long>(b) * p.L + t) * p.Hq + g * p.G + r) * kHeadDim + 4 * lane;
        uint2 pk;
        pk.x = pack_bf16(acc[0] * p.scale, acc[1] * p.scale);
        pk.y = pack_bf16(acc[2] * p.scale, acc[3] * p.scale);
        *reinterpret_cast<uint2*>(dst) = pk;
      }
    }
    named_bar_sync(1, 32 * kBwdConsumers);
  }
}

// Segment `item` -> (entry e = bg * nblk + j, segment within the entry's list).
__device__ __forceinline__ int bwd_find_entry(const int32_t* segoff, int n, int item) {
  int lo = 0, hi = n - 1;  // largest e with segoff[e] <= item
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (segoff[mid] <= item) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// dk / dv (bf16) from the fp32 workspace; n4 = elements / 4.
__global__ void __launch_bounds__(256) bwd_cast_kernel(const float4* __restrict__ a, const float4* __restrict__ c,
                                                       long long n4, uint2* __restrict__ da, uint2* __restrict__ dc) {
  for (long long i = blockIdx.x * 256LL + threadIdx.x; i < n4; i += 256LL * gridDim.x) {
    const float4 x = a[i], y = c[i];
    da[i] = make_uint2(pack_bf16(x.x, x.y), pack_bf16(x.z, x.w));
    dc[i] = make_uint2(pack_bf16(y.x, y.y), pack_bf16(y.z, y.w));
  }
}

}  // namespace infllmv2
