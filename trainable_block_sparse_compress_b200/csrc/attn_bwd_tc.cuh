// attn_bwd_tc.cuh -- dK and dV of the sparse attention on the 5th-generation tensor cores
// (tcgen05 + TMEM).
//
// MiniCPM4 summary page (端设备上的超高效大型语言模型) s2.1 and s2.1.3: the sparse attention
// is trained; with the block lists fixed the gradients of one KV block are sums over the
// query rows that selected it.  For block j of (b, g) and those rows (csrc/attn_bwd.cuh
// builds the lists and cuts them into segments of at most kBwdSeg tokens):
//   S = scale' q K_j^T (recomputed), P = exp2(S - lse'), dP = dO V_j^T, dS = P (dP - D),
//   dV_j += P^T dO,   dK_j += scale dS^T q.
// Work item = one segment.  A persistent CTA keeps the block's K and V in shared memory
// and takes the segment's tokens 8 at a time: a 128-row tile of 8 tokens x 16 heads (the
// heads past the group are padding, as are tokens past the segment's end).  Per tile:
//   warp 4 (one thread, TMA): the Q and dO rows of the 8 tokens (16-row boxes gathered
//          into one 128-row, 128-byte-swizzled tile) through a 2-stage ring;
//   warp 5 (one thread) issues S = Q K^T and dP = dO V^T (UMMA M128 N64 K16 x 8 each:
//          rows x keys) into one of two TMEM buffer pairs, and, once the probabilities
//          of the tile are in shared memory, dV^T += dO^T P and dK^T += Q^T dS (M128 N64:
//          dims x keys, the tiles read MN-major) into two TMEM accumulators that live for
//          the whole segment.  S and dP of the next tile are issued before the current
//          tile's dV / dK, so the tensor pipe overlaps the epilogue;
//   warps 0-3, thread = TMEM lane = tile row: P and dS of its row (64 keys; keys past
//          the row's position, padding heads and padding tokens give 0), written as bf16
//          rows of 128 bytes (the MN-major B operands of the dV / dK products) into one of
//          two buffer pairs, so a tile's epilogue runs while the previous tile's dV / dK
//          products read the other pair.
// At the end of a segment the epilogue reads dV^T and dK^T (thread = dimension d, 64
// keys) and adds them to the fp32 workspace (float atomics, coalesced over d: a block's
// segments run on different CTAs).
#pragma once
#include "attn_bwd.cuh"
#include "tcgen05.cuh"

namespace infllmv2 {

constexpr int kBtTok = 8;                          // tokens per 128-row tile
constexpr int kBtHalfBytes = 128 * 128;            // one 64-column half of a 128-row tile: 16 KB
constexpr int kBtTileBytes = 2 * kBtHalfBytes;     // 128 rows x 128 bf16: 32 KB
constexpr int kBtStages = 2;                       // Q + dO tile pairs in flight
constexpr int kBtStageBytes = 2 * kBtTileBytes;    // Q tile, then dO tile: 64 KB
constexpr int kBtPBytes = 128 * 128;               // P or dS: 128 rows x 64 keys bf16 = 16 KB
constexpr int kBtPBufs = 2;                        // P / dS buffer pairs: a tile's epilogue overlaps the
                                                   // previous tile's dV / dK products
constexpr int kBtEpiWarps = 4;
constexpr int kBtTmaWarp = kBtEpiWarps, kBtMmaWarp = kBtEpiWarps + 1;
constexpr int kBtThreads = 32 * (kBtEpiWarps + 2);
constexpr uint32_t kBtTmemCols = 512;
// TMEM columns: S[2] at 0 and 64, dP[2] at 128 and 192, dV^T at 256, dK^T at 320
constexpr uint32_t kBtColS = 0, kBtColDP = 128, kBtColDV = 256, kBtColDK = 320;

struct BtSmem {
  uint64_t kv_full, kv_empty, t_full[kBtStages], t_empty[kBtStages], sdp_full[2], sdp_empty[2];
  uint64_t pds_full[kBtPBufs], pds_empty[kBtPBufs], acc_full, acc_empty, mma_done;
  uint32_t tmem_base;
  volatile int abort;
};

constexpr size_t bwd_dkdv_tc_smem_bytes() {
  return 1024 + static_cast<size_t>(kAttnStageBytes) + static_cast<size_t>(kBtStages) * kBtStageBytes +
         2 * kBtPBufs * static_cast<size_t>(kBtPBytes) + sizeof(BtSmem);
}
static_assert(bwd_dkdv_tc_smem_bytes() <= 227 * 1024, "shared memory of one CTA");

// grid = persistent CTAs over the segments (their total is segoff[n]), block = 192.
__global__ void __launch_bounds__(kBtThreads, 1)
    bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                       const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                       const BwdParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = align_smem(smem_raw, 1024);
  unsigned char* kv = base;                              // K block (16 KB) then V block (16 KB)
  unsigned char* tiles = kv + kAttnStageBytes;           // ring: Q tile then dO tile per stage
  unsigned char* pbuf = tiles + kBtStages * kBtStageBytes;  // P of buffer x at pbuf + 2 x kBtPBytes,
                                                            // dS right after it
  BtSmem& S = *reinterpret_cast<BtSmem*>(pbuf + 2 * kBtPBufs * kBtPBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_entries = p.B * p.Hkv * p.nblk;
  const int total = p.segoff[n_entries];

  if (threadIdx.x == 0) {
    mbar_init(&S.kv_full, 1);
    mbar_init(&S.kv_empty, 1);
    for (int s = 0; s < kBtStages; ++s) {
      mbar_init(&S.t_full[s], 1);
      mbar_init(&S.t_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&S.sdp_full[s], 1);
      mbar_init(&S.sdp_empty[s], kBtEpiWarps);
    }
    for (int s = 0; s < kBtPBufs; ++s) {
      mbar_init(&S.pds_full[s], kBtEpiWarps);
      mbar_init(&S.pds_empty[s], 1);
    }
    mbar_init(&S.acc_full, 1);
    mbar_init(&S.acc_empty, kBtEpiWarps);
    mbar_init(&S.mma_done, 1);
    S.abort = 0;
    fence_mbar_init();
  }
  if (warp == kBtMmaWarp) {
    tmem_alloc(&S.tmem_base, kBtTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;

  if (warp == kBtTmaWarp) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_do);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      uint32_t gt = 0;                        // tiles issued so far (ring position)
      uint32_t kv_issued = 0;                 // items whose K / V were issued
      int it = 0;
      for (int item = blockIdx.x; item < total; item += gridDim.x, ++it) {
        const int e = bwd_find_entry(p.segoff, n_entries, item);
        const int seg = item - p.segoff[e];
        const int bg = e / p.nblk, j = e % p.nblk;
        const int b = bg / p.Hkv, g = bg % p.Hkv;
        const int r0 = seg * kBwdSeg, nrows = min(kBwdSeg, p.cnt[e] - r0);
        const int ntiles = (nrows + kBtTok - 1) / kBtTok;
        if (it > 0) mbar_wait(&S.kv_empty, static_cast<uint32_t>(it - 1) & 1u, &S.abort);
        if (S.abort) break;
        const int krow = bg * p.L + j * kBlock;
        mbar_arrive_expect_tx(&S.kv_full, kAttnStageBytes);
        tma_load_2d(kv, &tm_k, &S.kv_full, 0, krow);
        tma_load_2d(kv + kKvTileBytes / 2, &tm_k, &S.kv_full, 64, krow);
        tma_load_2d(kv + kKvTileBytes, &tm_v, &S.kv_full, 0, krow);
        tma_load_2d(kv + kKvTileBytes + kKvTileBytes / 2, &tm_v, &S.kv_full, 64, krow);
        kv_issued = static_cast<uint32_t>(it) + 1u;
        const int32_t* rows = p.list + p.off[e] + r0;
        for (int ti = 0; ti < ntiles; ++ti, ++gt) {
          // the tile's 8 list entries, loaded together (padding tokens repeat the first row,
          // masked in the epilogue)
          int tok[kBtTok];
#pragma unroll
          for (int u = 0; u < kBtTok; ++u) {
            const int r = ti * kBtTok + u;
            tok[u] = rows[r < nrows ? r : 0];
          }
          const int st = static_cast<int>(gt & 1u);
          if (gt >= kBtStages) mbar_wait(&S.t_empty[st], ((gt >> 1) - 1u) & 1u, &S.abort);
          if (S.abort) break;
          unsigned char* tq = tiles + st * kBtStageBytes;
          mbar_arrive_expect_tx(&S.t_full[st], kBtStageBytes);
#pragma unroll
          for (int u = 0; u < kBtTok; ++u) {
            const int qrow = (b * p.L + tok[u]) * p.Hq + g * p.G;
            tma_load_2d(tq + u * 2048, &tm_q, &S.t_full[st], 0, qrow);
            tma_load_2d(tq + kBtHalfBytes + u * 2048, &tm_q, &S.t_full[st], 64, qrow);
            tma_load_2d(tq + kBtTileBytes + u * 2048, &tm_do, &S.t_full[st], 0, qrow);
            tma_load_2d(tq + kBtTileBytes + kBtHalfBytes + u * 2048, &tm_do, &S.t_full[st], 64, qrow);
          }
        }
        if (S.abort) break;
      }
      if (S.abort) {  // let every copy this thread issued land before the CTA ends
        if (kv_issued > 0) mbar_wait_drain(&S.kv_full, (kv_issued - 1u) & 1u);
        for (uint32_t st = 0; st < kBtStages; ++st)
          if (gt > st) {
            const uint32_t last = st + kBtStages * ((gt - 1u - st) / kBtStages);
            mbar_wait_drain(&S.t_full[st], (last >> 1) & 1u);
          }
      }
    }
    return;
  }

  if (warp == kBtMmaWarp) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_rk = idesc_bf16_f32(128, 64, false, false);  // rows x keys, both K-major
      constexpr uint32_t id_dk = idesc_bf16_f32(128, 64, true, true);    // dims x keys, both MN-major
      const uint32_t kb = smem_u32(kv), vb = kb + kKvTileBytes;
      const uint32_t pb0 = smem_u32(pbuf);
      uint32_t gt = 0;  // tiles whose S / dP were issued
      int it = 0;
      // S = Q K^T and dP = dO V^T of global tile n into buffer pair n & 1 (its Q / dO tile
      // has landed and the epilogue has read the pair's previous contents)
      auto issue_sdp = [&](uint32_t n) {
        const int st = static_cast<int>(n & 1u);
        const uint32_t sb = n & 1u;
        const uint32_t qa = smem_u32(tiles + st * kBtStageBytes), da = qa + kBtTileBytes;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t ao = static_cast<uint32_t>((k >> 2) * kBtHalfBytes + (k & 3) * 32);
          const uint32_t bo = static_cast<uint32_t>((k >> 2) * (kKvTileBytes / 2) + (k & 3) * 32);
          umma_bf16(tmem + kBtColS + 64u * sb, desc_k_sw128(qa + ao), desc_k_sw128(kb + bo), id_rk, k > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t ao = static_cast<uint32_t>((k >> 2) * kBtHalfBytes + (k & 3) * 32);
          const uint32_t bo = static_cast<uint32_t>((k >> 2) * (kKvTileBytes / 2) + (k & 3) * 32);
          umma_bf16(tmem + kBtColDP + 64u * sb, desc_k_sw128(da + ao), desc_k_sw128(vb + bo), id_rk,
                    k > 0 ? 1u : 0u);
        }
        umma_commit(&S.sdp_full[sb]);
      };
      // dV^T += dO^T P and dK^T += Q^T dS of global tile n (first = the segment's first tile)
      auto issue_dvdk = [&](uint32_t n, bool first) {
        const uint32_t x = n % kBtPBufs;
        const uint32_t pb = pb0 + 2u * x * kBtPBytes, db = pb + kBtPBytes;
        const uint32_t qa = smem_u32(tiles + static_cast<int>(n & 1u) * kBtStageBytes), da = qa + kBtTileBytes;
#pragma unroll
        for (int k = 0; k < 8; ++k)  // 16 rows per step
          umma_bf16(tmem + kBtColDV, desc_mn_sw128(da + k * 2048, kBtHalfBytes, 1024),
                    desc_mn_sw128(pb + k * 2048, kBtPBytes, 1024), id_dk, (!first || k > 0) ? 1u : 0u);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          umma_bf16(tmem + kBtColDK, desc_mn_sw128(qa + k * 2048, kBtHalfBytes, 1024),
                    desc_mn_sw128(db + k * 2048, kBtPBytes, 1024), id_dk, (!first || k > 0) ? 1u : 0u);
        umma_commit(&S.pds_empty[x]);                       // P / dS of buffer x may be rewritten
        umma_commit(&S.t_empty[static_cast<int>(n & 1u)]);  // the Q / dO tile is no longer read
      };
      // Within a segment the two kinds of products are issued as soon as their inputs are
      // ready, neither waiting behind the other: a tile's dV / dK never waits for the next
      // tile's Q / dO rows to land (which would chain the gather latency onto every tile).
      // Each barrier is tested only after its previous phase was seen, so a parity test
      // cannot alias.
      for (int item = blockIdx.x; item < total; item += gridDim.x, ++it) {
        const int e = bwd_find_entry(p.segoff, n_entries, item);
        const int seg = item - p.segoff[e];
        const int r0 = seg * kBwdSeg, nrows = min(kBwdSeg, p.cnt[e] - r0);
        const uint32_t ntiles = static_cast<uint32_t>((nrows + kBtTok - 1) / kBtTok);
        if (!mbar_wait(&S.kv_full, static_cast<uint32_t>(it) & 1u, &S.abort)) break;
        tc_fence_after();
        const uint32_t g0 = gt;
        uint32_t ns = 0, nd = 0;  // tiles of the segment whose S / dP, dV / dK were issued
        bool acc_free = it == 0;  // the epilogue has read the previous segment's dV^T / dK^T
        uint32_t idle = 0;
        uint64_t t_idle = 0;
        while (nd < ntiles) {
          bool progress = false;
          if (ns < ntiles) {
            const uint32_t n = g0 + ns, st = n & 1u;
            if (mbar_test(&S.t_full[st], (n >> 1) & 1u) &&
                (n < 2 || mbar_test(&S.sdp_empty[st], ((n >> 1) - 1u) & 1u))) {
              tc_fence_after();
              issue_sdp(n);
              if (++ns == ntiles) umma_commit(&S.kv_empty);  // every read of the block's K / V was issued
              progress = true;
            }
          }
          if (nd < ns) {
            const uint32_t n = g0 + nd;
            if (!acc_free) acc_free = mbar_test(&S.acc_empty, static_cast<uint32_t>(it - 1) & 1u);
            if (acc_free && mbar_test(&S.pds_full[n % kBtPBufs], (n / kBtPBufs) & 1u)) {
              tc_fence_after();
              issue_dvdk(n, nd == 0);
              ++nd;
              progress = true;
            }
          }
          if (progress) {
            idle = 0;
            t_idle = 0;
          } else if (++idle == 64u) {  // bounded: give up like mbar_wait
            idle = 0;
            if (S.abort || (*reinterpret_cast<volatile unsigned int*>(&g_device_error) & kDevErrWaitTimeout) != 0u) {
              S.abort = 1;
              break;
            }
            const uint64_t now = globaltimer_ns();
            if (t_idle == 0) {
              t_idle = now;
            } else if (now - t_idle > kWaitLimitNs) {
              S.abort = 1;
              atomicOr(&g_device_error, kDevErrWaitTimeout);
              break;
            }
          }
        }
        gt = g0 + ns;
        if (S.abort) break;
        umma_commit(&S.acc_full);  // dV^T and dK^T of the segment are complete
      }
      umma_commit(&S.mma_done);
    }
    __syncwarp();
    named_bar_sync(1, 32 * (kBtEpiWarps + 1));  // the epilogue has read TMEM for the last time
    if (lane == 0) mbar_wait_drain(&S.mma_done, 0);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kBtTmemCols);
    return;
  }

  // ---------------------------------------------------------------- epilogue warps
  const int row = threadIdx.x;          // tile row = TMEM lane: token row / 16, head row % 16
  const int u = row >> 4, h = row & 15;
  const uint32_t tl = tmem + (static_cast<uint32_t>(32 * warp) << 16);
  const float sl2 = p.scale_log2;
  uint32_t gt = 0;
  int it = 0;
  for (int item = blockIdx.x; item < total; item += gridDim.x, ++it) {
    const int e = bwd_find_entry(p.segoff, n_entries, item);
    const int seg = item - p.segoff[e];
    const int bg = e / p.nblk, j = e % p.nblk;
    const int b = bg / p.Hkv, g = bg % p.Hkv;
    const int r0 = seg * kBwdSeg, nrows = min(kBwdSeg, p.cnt[e] - r0);
    const int ntiles = (nrows + kBtTok - 1) / kBtTok;
    const int32_t* rows = p.list + p.off[e] + r0;
    // this row's token, lse and D, loaded one tile ahead of their use
    auto load_row = [&](int ti, int& t, float& lse2, float& dl) {
      const int r = ti * kBtTok + u;
      const bool rv = r < nrows && h < p.G;
      t = rows[r < nrows ? r : 0];
      const long long li = (static_cast<long long>(b) * p.Hq + g * p.G + (h < p.G ? h : 0)) * p.L + t;
      lse2 = rv ? p.lse[li] * 1.4426950408889634f : 0.f;
      dl = rv ? p.delta[li] : 0.f;
    };
    int t_n;
    float lse2_n, dl_n;
    load_row(0, t_n, lse2_n, dl_n);
    for (int ti = 0; ti < ntiles; ++ti, ++gt) {
      const uint32_t sb = gt & 1u;
      const bool rv = ti * kBtTok + u < nrows && h < p.G;
      const int t = t_n;
      const float lse2 = lse2_n, dl = dl_n;
      if (ti + 1 < ntiles) load_row(ti + 1, t_n, lse2_n, dl_n);
      const uint32_t x = gt % kBtPBufs;
      unsigned char* pbx = pbuf + 2 * x * kBtPBytes;
      unsigned char* dsx = pbx + kBtPBytes;
      mbar_wait(&S.sdp_full[sb], (gt >> 1) & 1u, &S.abort);
      if (gt >= kBtPBufs)  // dV / dK of the tile that last used buffer x are done
        mbar_wait(&S.pds_empty[x], (gt / kBtPBufs - 1u) & 1u, &S.abort);
      tc_fence_after();
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        uint32_t sv[32], dv[32];
        tmem_ld32(tl + kBtColS + 64u * sb + 32u * half, sv);
        tmem_ld32(tl + kBtColDP + 64u * sb + 32u * half, dv);
        uint32_t pk[16], dk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const int key0 = j * kBlock + 32 * half + c;
          float pr[2], ds[2];
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const bool ok = rv && key0 + q <= t;
            pr[q] = ok ? ex2(fmaf(__uint_as_float(sv[c + q]), sl2, -lse2)) : 0.f;
            ds[q] = pr[q] * (__uint_as_float(dv[c + q]) - dl);
          }
          pk[c >> 1] = pack_bf16(pr[0], pr[1]);
          dk[c >> 1] = pack_bf16(ds[0], ds[1]);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {  // four 16-byte chunks of this row's 32 keys
          const int chunk = 4 * half + q;
          *reinterpret_cast<uint4*>(pbx + sw128(row, chunk)) =
              make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          *reinterpret_cast<uint4*>(dsx + sw128(row, chunk)) =
              make_uint4(dk[4 * q], dk[4 * q + 1], dk[4 * q + 2], dk[4 * q + 3]);
        }
      }
      tc_fence_before();
      fence_proxy_async_smem();  // the generic writes of P and dS before the MMAs read them
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&S.sdp_empty[sb]);
        mbar_arrive(&S.pds_full[x]);
      }
    }
    // the segment's dV^T and dK^T: thread = dimension d, columns = the block's 64 keys
    mbar_wait(&S.acc_full, static_cast<uint32_t>(it) & 1u, &S.abort);
    tc_fence_after();
    const long long kbase = static_cast<long long>(bg) * p.L + j * kBlock;
#pragma unroll 1
    for (int half = 0; half < 2; ++half) {
      uint32_t av[32], ak[32];
      tmem_ld32(tl + kBtColDV + 32u * half, av);
      tmem_ld32(tl + kBtColDK + 32u * half, ak);
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const int key = 32 * half + c;
        if (j * kBlock + key < p.L) {
          atomicAdd(p.dv32 + (kbase + key) * kHeadDim + row, __uint_as_float(av[c]));
          atomicAdd(p.dk32 + (kbase + key) * kHeadDim + row, __uint_as_float(ak[c]) * p.scale);
        }
      }
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.acc_empty);
  }
  tc_fence_before();
  named_bar_sync(1, 32 * (kBtEpiWarps + 1));  // TMEM may be freed
}

}  // namespace infllmv2
