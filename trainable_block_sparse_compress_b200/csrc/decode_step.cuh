// decode_step.cuh -- a whole decode step (block selection, then sparse attention over
// the selected blocks) for one query per sequence, in one launch.
//
// MiniCPM4 summary page (端设备上的超高效大型语言模型) s2.1: InfLLM v2 selects context
// blocks for decoding as well as prefill; s2.1.2 / s2.1.3: the group's heads share the
// selected blocks and attend only to them.
//
// A thread-block cluster per (sequence, kv-head) runs the selection phases of
// select_decode.cuh (Kc streamed and scored by every CTA, every CTA's block keys stored
// into every CTA of the cluster), then each CTA runs the same deterministic top-k over all
// keys in its own shared memory -- so no CTA waits for another's list -- and goes straight
// on to the attention phases of attn_dec.cuh over its contiguous share of that list (it
// streams those K/V blocks, and the partial states are merged across the cluster); CTA 0
// also writes the list to block_idx.  Clusters do not wait for one another,
// so a cluster whose sequence is short streams its K/V while longer sequences are still
// being scored, and nothing round-trips through global memory between the two halves.
// The selection's tile ring and block maxima and the attention's ring share one region of
// shared memory: each half's data is dead before the other half writes it.
// Optionally the step first appends the new token (the cache maintenance of
// append_kv_kernel, same arithmetic): the CTA that scores the sequence's last kernel
// writes the token's key and value rows and the kernel the token completes, before its
// own Kc stream starts; the new length goes to lens_out.
#pragma once
#include <cooperative_groups.h>

#include "append.cuh"
#include "attn_dec.cuh"
#include "select_decode.cuh"

namespace infllmv2 {

constexpr size_t kDsAttnRegion = static_cast<size_t>(kAdStages) * kAttnStageBytes + kQTileBytes;
constexpr size_t kDsRegion = kSdRegionBytes > kDsAttnRegion ? kSdRegionBytes : kDsAttnRegion;

struct DsSmem {
  SdSmem sel;
  AdSmem attn;  // attn.list: the item's list, as every CTA emits it
};

constexpr size_t decode_step_smem_bytes() { return 1024 + kDsRegion + sizeof(DsSmem); }

struct DecodeStepParams {
  SelDecodeParams sel;
  AttnParams attn;
  // the token to append (nullptr: none; lens then counts the query's own token)
  const __nv_bfloat16* k_new;  // [B, Hkv, d]
  const __nv_bfloat16* v_new;  // [B, Hkv, d]
  __nv_bfloat16* k_cache;      // [B, Hkv, Lmax, d]
  __nv_bfloat16* v_cache;
  __nv_bfloat16* kc;           // [B, Hkv, NKmax, d]
  int32_t* lens_out;           // [B]: the new lengths
};

// Appends the token of (b, g) at position pos (< Lmax): key and value rows, and the
// semantic kernel it completes when n = pos + 1 = 32 + 16 i -- kernel i, the mean of key
// rows [16 i, 16 i + 32), fp64 sum rounded once (append_kv_kernel's arithmetic).  Threads
// 0..127, thread = column d; each fences its writes for later bulk-tensor reads.
__device__ __forceinline__ void ds_append(const DecodeStepParams& P, long long bg, int pos) {
  const int d = threadIdx.x;
  if (d >= kHeadDim) return;
  const long long Lmax = P.sel.Lmax;
  const __nv_bfloat16 kv = P.k_new[bg * kHeadDim + d];
  P.k_cache[(bg * Lmax + pos) * kHeadDim + d] = kv;
  P.v_cache[(bg * Lmax + pos) * kHeadDim + d] = P.v_new[bg * kHeadDim + d];
  const int n = pos + 1;
  if (n >= kKernel && (n - kKernel) % kStride == 0) {
    const int ki = (n - kKernel) / kStride;
    const __nv_bfloat16* rows = P.k_cache + (bg * Lmax + static_cast<long long>(kStride) * ki) * kHeadDim + d;
    __nv_bfloat16 r_[kKernel - 1];
#pragma unroll
    for (int r = 0; r < kKernel - 1; ++r) r_[r] = rows[r * kHeadDim];
    double sum = 0.0;
#pragma unroll
    for (int r = 0; r < kKernel - 1; ++r) sum += static_cast<double>(__bfloat162float(r_[r]));
    sum += static_cast<double>(__bfloat162float(kv));  // the new row, from the input
    P.kc[(bg * P.sel.NKmax + ki) * kHeadDim + d] = __double2bfloat16(sum * (1.0 / kKernel));
  }
  fence_proxy_async_global();
}

// grid = C * B * Hkv (cluster r serves item r), cluster = (C, 1, 1), block = 160.  C divides 16.
__global__ void __launch_bounds__(kSdThreads)
    decode_step_kernel(const __grid_constant__ CUtensorMap tm_kc, const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                       const DecodeStepParams P) {
  static_assert(kSdThreads == kAdThreads, "one block shape for both halves");
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ unsigned char smem_raw[];
  unsigned char* region = align_smem(smem_raw, 1024);
  uint32_t* bm = reinterpret_cast<uint32_t*>(region + kSdStages * kKcTileBytes);  // selection: [16][kSdBStride]
  unsigned char* qtile = region + kAdStages * kAttnStageBytes;                      // attention: the query tile
  DsSmem& D = *reinterpret_cast<DsSmem*>(region + kDsRegion);

  const int C = static_cast<int>(cluster.num_blocks());
  const int c = static_cast<int>(cluster.block_rank());
  const long long bg = blockIdx.x / C;  // clusters are consecutive blocks
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int topk = P.sel.topk;

  allow_dependent_launch();
  if (threadIdx.x == 0) ad_init(D.attn);  // published by the first CTA barrier of the selection
  if (warp == kSdConsumers && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  grid_dependency_wait();  // q, the caches, Kc and lens may come from the previous kernel
  const int b = static_cast<int>(bg / P.sel.Hkv);
  const int Lmax = P.sel.Lmax;
  const int raw = P.sel.lens[b];
  const bool append = P.k_new != nullptr && raw >= 0 && raw < Lmax;
  const int n = append ? raw + 1 : min(max(raw, 0), Lmax);
  const SdItem it = sd_item(P.sel, C, c, bg, n);
  if (P.k_new != nullptr) {
    if (append && c == (it.nk > 0 ? (it.nk - 1) / it.chunk : 0)) ds_append(P, bg, raw);
    if (c == 0 && it.g == 0 && threadIdx.x == 0) {
      P.lens_out[b] = append ? n : raw;
      if (!append) atomicOr(&g_device_error, kDevErrCacheFull);  // left untouched, as append_kv does
    }
  }

  // ---- selection: every CTA receives every key and derives the same list
  sd_score_chunk(&tm_kc, P.sel, it, region, bm, D.sel);
  cluster.sync();  // every CTA's tiles are consumed and its partial state is final
  sd_block_keys<true>(cluster, P.sel, it, region, bm, D.sel);
  cluster.sync();  // every CTA holds every key; no CTA touches a peer's memory until the merge
  const int n_all = sd_select(P.sel, it, region, D.attn.list, D.sel);
  if (c == 0) {
    int32_t* out = P.sel.idx + bg * topk;
    for (int e = threadIdx.x; e < topk; e += kSdThreads) out[e] = D.attn.list[e];
  }

  // ---- attention over this CTA's contiguous share of the list
  const int per = (n_all + C - 1) / C;
  const int lo = min(c * per, n_all);
  const int nsh = min(lo + per, n_all) - lo;
  fence_proxy_async_smem();  // the region's generic accesses before the ring's copies
  __syncthreads();
  const int qrow = it.b * P.attn.Hq + it.g * P.attn.G;
  ad_partial(&tm_q, &tm_k, &tm_v, P.attn, bg, qrow, it.n - 1, D.attn.list + lo, nsh, region, qtile, D.attn);
  ad_merge(cluster, P.attn, qrow, region, D.attn);
}

}  // namespace infllmv2
