// infllmv2.cu -- C ABI of the InfLLM v2 block-sparse attention library (sm_100a).
//
// Host side of every entry point declared in include/infllmv2.h: argument checks
// before any launch, TMA tensor-map encoding (driver entry point fetched through the
// runtime, so the library needs no -lcuda), workspace carving and kernel launches on
// the caller's stream.  All device code lives in the included .cuh files.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <utility>

#include "../../include/infllmv2.h"
#include "append.cuh"
#include "attn.cuh"
#include "attn_bwd.cuh"
#include "attn_bwd_tc.cuh"
#include "attn_dec.cuh"
#include "attn_tc.cuh"
#include "common.cuh"
#include "compress.cuh"
#include "decode_step.cuh"
#include "select_decode.cuh"
#include "select_prefill.cuh"
#include "select_prefill_tc.cuh"
#include "topk.cuh"

using namespace infllmv2;

namespace {

constexpr int kVersion = 200;  // 0.2.0

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_params(const infllmv2_params* p) {
  if (p == nullptr) return INFLLMV2_ERR_INVALID_ARG;
  if (p->batch < 1 || p->num_kv_heads < 1 || p->num_q_heads < 1 || p->head_dim < 1) return INFLLMV2_ERR_INVALID_ARG;
  if (p->num_q_heads % p->num_kv_heads != 0) return INFLLMV2_ERR_INVALID_ARG;
  if (p->block_size < 1 || p->kernel_size < 1 || p->kernel_stride < 1) return INFLLMV2_ERR_INVALID_ARG;
  if (p->topk < 1 || p->n_init < 0 || p->n_local < 0) return INFLLMV2_ERR_INVALID_ARG;
  if (static_cast<long long>(p->n_init) + p->n_local > p->topk) return INFLLMV2_ERR_INVALID_ARG;
  if (!(p->softmax_scale <= 0.f || std::isfinite(p->softmax_scale))) return INFLLMV2_ERR_INVALID_ARG;
  if ((p->score_mode != INFLLMV2_SCORE_SOFTMAX_SUM && p->score_mode != INFLLMV2_SCORE_LOGIT_SUM) ||
      (p->pool_mode != INFLLMV2_POOL_OVERLAP && p->pool_mode != INFLLMV2_POOL_INSIDE))
    return INFLLMV2_ERR_INVALID_ARG;
  const int G = p->num_q_heads / p->num_kv_heads;
  if (p->head_dim != kHeadDim || p->block_size != kBlock || p->kernel_size != kKernel ||
      p->kernel_stride != kStride)
    return INFLLMV2_ERR_UNSUPPORTED;
  if (!(G == 1 || G == 2 || G == 4 || G == 8 || G == 16)) return INFLLMV2_ERR_UNSUPPORTED;
  if (p->topk > kMaxTopk) return INFLLMV2_ERR_UNSUPPORTED;
  if (static_cast<long long>(p->batch) * p->num_q_heads > (1LL << 24)) return INFLLMV2_ERR_UNSUPPORTED;
  return INFLLMV2_OK;
}

int check_len(int32_t L) { return (L >= 1 && L <= INFLLMV2_MAX_SEQ_LEN) ? INFLLMV2_OK : INFLLMV2_ERR_INVALID_ARG; }

int64_t num_kernels(int64_t n) { return n >= kKernel ? (n - kKernel) / kStride + 1 : 0; }
int64_t num_blocks(int64_t n) { return (n + kBlock - 1) / kBlock; }
int round32(int64_t x) { return static_cast<int>((x + 31) / 32 * 32); }

float scale_log2(const infllmv2_params* p) {
  const float s = p->softmax_scale > 0.f ? p->softmax_scale : 1.f / std::sqrt(static_cast<float>(p->head_dim));
  return s * 1.4426950408889634f;
}

// ------------------------------------------------------------ tensor maps

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool get_encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode != nullptr;
}

// 2-D view [rows, 128] of a bf16 tensor, box {64 columns, box_rows}, 128-byte swizzle,
// zero fill outside the tensor.
bool make_map(CUtensorMap* m, const void* ptr, uint64_t rows, uint32_t box_rows) {
  if (!get_encoder()) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(kHeadDim) * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D view [tokens, heads, 128] of the prefill queries, box {64 columns, G heads, 128 / G
// tokens}: the 128 (token, head) rows of one selection tile.
bool make_q_map_3d(CUtensorMap* m, const void* q, uint64_t tokens, uint64_t heads, int G) {
  if (!get_encoder()) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(heads),
                        static_cast<cuuint64_t>(tokens)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(kHeadDim) * 2, static_cast<cuuint64_t>(heads * kHeadDim * 2)};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(G), static_cast<cuuint32_t>(128 / G)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

constexpr size_t kMaxSmem = 227 * 1024;

int launch_status() { return cudaGetLastError() == cudaSuccess ? INFLLMV2_OK : INFLLMV2_ERR_CUDA; }

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

int set_smem(const void* fn, size_t bytes) {
  return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes)) ==
                 cudaSuccess
             ? INFLLMV2_OK
             : INFLLMV2_ERR_CUDA;
}

// Launches `kern` on a 1-D grid in clusters of C CTAs.  Sizes above 8 need the
// non-portable opt-in.  With `pdl` the kernel may start while the previous kernel on the
// stream finishes (it must call grid_dependency_wait() before reading any input).  A cluster shape that the device cannot co-schedule is reported
// as unsupported before any launch (checked once per kernel, size and device).
template <typename... Params, typename... Args>
int launch_cluster(void (*kern)(Params...), unsigned grid, int C, int threads, size_t smem, cudaStream_t s,
                   bool pdl, Args&&... args) {
  const void* fn = reinterpret_cast<const void*>(kern);
  int st = set_smem(fn, smem);
  if (st != INFLLMV2_OK) return st;
  if (C > 8 && cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
    return INFLLMV2_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(C);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  {
    static std::mutex mu;
    static std::map<std::tuple<const void*, int, int>, int> fits;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return INFLLMV2_ERR_CUDA;
    std::lock_guard<std::mutex> lock(mu);
    const auto key = std::make_tuple(fn, C, dev);
    auto it = fits.find(key);
    if (it == fits.end()) {
      int active = 0;
      if (cudaOccupancyMaxActiveClusters(&active, kern, &cfg) != cudaSuccess) return INFLLMV2_ERR_CUDA;
      it = fits.emplace(key, active).first;
    }
    if (it->second < 1) return INFLLMV2_ERR_UNSUPPORTED;
  }
  if (cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...) != cudaSuccess) return INFLLMV2_ERR_CUDA;
  return launch_status();
}

// Decode work layout.  Each (sequence, kv-head) item's selected blocks are split over
// CTAs.  Normally a cluster of C CTAs (a power of two up to 16, as large as keeps all
// CTAs resident at two per SM) merges its partials in distributed shared memory.  When
// even 16 CTAs per item leave most SMs idle (fewer items than SMs / 16), the blocks are
// split further, two or more per CTA, and the partials meet in the workspace.
struct DecodePlan {
  int cluster;   // CTAs per cluster (cluster path), 0 for the workspace path
  int n_splits;  // workspace path: splits per item
  int per_split;
};

DecodePlan decode_plan(const infllmv2_params* p) {
  const long long items = static_cast<long long>(p->batch) * p->num_kv_heads;
  const long long target = 2LL * num_sms();
  DecodePlan d{0, 1, p->topk};
  if (items * kAdMaxCluster >= num_sms()) {
    int c = 1;
    while (c < kAdMaxCluster && items * c * 2 <= target) c *= 2;
    d.cluster = c;
    return d;
  }
  int s = static_cast<int>(std::min<long long>((target + items - 1) / items, (p->topk + 1) / 2));
  s = std::max(1, std::min(s, kMaxDecodeSplits));
  d.per_split = (p->topk + s - 1) / s;
  d.n_splits = (p->topk + d.per_split - 1) / d.per_split;
  return d;
}

// Selection cluster size: enough CTAs for the longest sequence's kernels (at most
// kSdMaxChunk per CTA), and as many as keep all CTAs resident at two per SM.
int select_cluster(const infllmv2_params* p, int64_t nk) {
  const long long items = static_cast<long long>(p->batch) * p->num_kv_heads;
  const long long target = 2LL * num_sms();
  int c = 1;
  while (c < kSdMaxCluster && (static_cast<int64_t>(c) * kSdMaxChunk < nk || items * c * 2 <= target)) c *= 2;
  return c;
}

// Clusters of C CTAs of `kern` that the device holds at once (cached per kernel, size,
// shared memory and device).
template <typename... Params>
int max_active_clusters(void (*kern)(Params...), int C, int threads, size_t smem) {
  static std::mutex mu;
  static std::map<std::tuple<const void*, int, size_t, int>, int> cache;
  const void* fn = reinterpret_cast<const void*>(kern);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_tuple(fn, C, smem, dev);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  if (set_smem(fn, smem) != INFLLMV2_OK) return 0;
  if (C > 8 && cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(C));
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(C);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int active = 0;
  if (cudaOccupancyMaxActiveClusters(&active, kern, &cfg) != cudaSuccess) active = 0;
  cache.emplace(key, active);
  return active;
}

// Decode-step cluster size: enough CTAs for the longest sequence's kernels (at most
// kSdMaxChunk per CTA), then doubled while all CTAs stay at two per SM and every item's
// cluster is resident at once (a cluster left for a second wave costs a whole step).
int decode_step_cluster(const infllmv2_params* p, int64_t nk) {
  const long long items = static_cast<long long>(p->batch) * p->num_kv_heads;
  const long long target = 2LL * num_sms();
  int c = 1;
  while (c < kSdMaxCluster && static_cast<int64_t>(c) * kSdMaxChunk < nk) c *= 2;
  while (c < kSdMaxCluster && items * c * 2 <= target &&
         items <= max_active_clusters(decode_step_kernel, 2 * c, kSdThreads, decode_step_smem_bytes()))
    c *= 2;
  return c;
}

// Workspace of the backward pass, in order (each part 256-byte aligned): D [B, Hq, L]
// fp32; cnt, cursor, off [n] and segoff [n + 1] int32 (n = B * Hkv * blocks); the row
// lists [B * Hkv * L * topk] int32; dK and dV accumulators [B, Hkv, L, d] fp32.
struct BwdLayout {
  size_t delta, cnt, cursor, off, segoff, list, dk, dv, total;
  long long n;
};
BwdLayout bwd_layout(const infllmv2_params* p, int32_t L) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  BwdLayout w;
  const size_t B = p->batch, Hq = p->num_q_heads, Hkv = p->num_kv_heads;
  w.n = static_cast<long long>(B * Hkv * num_blocks(L));
  w.delta = 0;
  w.cnt = up(w.delta + B * Hq * L * 4);
  w.cursor = up(w.cnt + w.n * 4);
  w.off = up(w.cursor + w.n * 4);
  w.segoff = up(w.off + w.n * 4);
  w.list = up(w.segoff + (w.n + 1) * 4);
  w.dk = up(w.list + B * Hkv * static_cast<size_t>(L) * p->topk * 4);
  w.dv = up(w.dk + B * Hkv * static_cast<size_t>(L) * kHeadDim * 4);
  w.total = up(w.dv + B * Hkv * static_cast<size_t>(L) * kHeadDim * 4);
  return w;
}

size_t ws_size(const infllmv2_params* p, int op, int32_t L) {
  if (check_params(p) != INFLLMV2_OK || check_len(L) != INFLLMV2_OK) return static_cast<size_t>(-1);
  switch (op) {
    case INFLLMV2_OP_COMPRESS:
    case INFLLMV2_OP_SELECT_PREFILL:
    case INFLLMV2_OP_ATTN_PREFILL:
      return 0;
    case INFLLMV2_OP_SELECT_DECODE:
      return 0;
    case INFLLMV2_OP_ATTN_BACKWARD:
      return bwd_layout(p, L).total;
    case INFLLMV2_OP_ATTN_DECODE: {
      const DecodePlan d = decode_plan(p);
      if (d.cluster > 0) return 0;
      const size_t rows = static_cast<size_t>(p->batch) * p->num_kv_heads * d.n_splits * kGroupRows;
      return rows * kHeadDim * sizeof(float) + rows * sizeof(float);
    }
    default:
      return static_cast<size_t>(-1);
  }
}

// Chunk arguments: Lq and Lmax in [1, INFLLMV2_MAX_SEQ_LEN], Lq <= Lmax, length arrays
// 4-byte aligned (their values are read and clamped on the GPU).
int check_chunk(int32_t Lq, const int32_t* q_lens, const int32_t* kv_lens, int32_t Lmax) {
  if (check_len(Lq) != INFLLMV2_OK || check_len(Lmax) != INFLLMV2_OK || Lq > Lmax) return INFLLMV2_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(q_lens) & 3u) || (reinterpret_cast<uintptr_t>(kv_lens) & 3u))
    return INFLLMV2_ERR_INVALID_ARG;
  return INFLLMV2_OK;
}

// Prefill selection for Lq query rows per sequence against caches of Lmax tokens: a fresh
// prefill (q_lens = kv_lens = NULL, Lq = Lmax = L) or a chunk of the last q_lens[b] of
// kv_lens[b] cached tokens.
int select_prefill(const infllmv2_params* p, const void* q, int32_t Lq, const void* kc, const int32_t* q_lens,
                   const int32_t* kv_lens, int32_t Lmax, int32_t* block_idx, cudaStream_t s) {
  if (q == nullptr || block_idx == nullptr || !aligned16(q) || !aligned16(block_idx)) return INFLLMV2_ERR_INVALID_ARG;
  const int64_t nk = num_kernels(Lmax);
  if (nk > 0 && (kc == nullptr || !aligned16(kc))) return INFLLMV2_ERR_INVALID_ARG;
  if (static_cast<uint64_t>(p->batch) * p->num_kv_heads * static_cast<uint64_t>(nk) > 0x7fffffffULL ||
      static_cast<uint64_t>(p->batch) * Lq > 0x7fffffffULL)
    return INFLLMV2_ERR_UNSUPPORTED;  // TMA coordinates are 32-bit
  const int G = p->num_q_heads / p->num_kv_heads;
  const int nblk_cap = round32(num_blocks(Lmax));
  CUtensorMap tm_kc;
  std::memset(&tm_kc, 0, sizeof tm_kc);
  if (nk > 0) {
    if (!make_map(&tm_kc, kc, static_cast<uint64_t>(p->batch) * p->num_kv_heads * nk, kKcTile))
      return INFLLMV2_ERR_CUDA;
  } else {
    // no complete kernel: every row keeps only its forced blocks; the kernel path runs
    // with an empty score loop (no tile is loaded, so the map is never dereferenced)
    if (!make_map(&tm_kc, q, kKcTile, kKcTile)) return INFLLMV2_ERR_CUDA;
  }
  SelPrefillParams a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.idx = block_idx;
  a.q_lens = q_lens;
  a.kv_lens = kv_lens;
  a.B = p->batch;
  a.Lq = Lq;
  a.Lmax = Lmax;
  a.Hq = p->num_q_heads;
  a.Hkv = p->num_kv_heads;
  a.G = G;
  a.NKmax = static_cast<int>(nk);
  a.topk = p->topk;
  a.n_init = p->n_init;
  a.n_local = p->n_local;
  a.score_mode = p->score_mode;
  a.pool_mode = p->pool_mode;
  a.nblk_cap = nblk_cap;
  a.scale_log2 = scale_log2(p);
  int st;
  // tensor-core path: 128 / G tokens x G heads per 128-row UMMA tile, with a 3-slot Kc
  // ring, or 2 slots when the block keys of long sequences need the room
  a.stages = sel_tc_smem_bytes(nblk_cap, G, 3) <= kMaxSmem ? 3 : 2;
  if (nk > 0 && sel_tc_smem_bytes(nblk_cap, G, a.stages) <= kMaxSmem) {
    const int tt = sel_tc_tokens(G);
    a.tiles_per_bg = (Lq + tt - 1) / tt;
    const long long grid = static_cast<long long>(a.tiles_per_bg) * p->batch * p->num_kv_heads;
    if (grid > 0x7fffffffLL) return INFLLMV2_ERR_UNSUPPORTED;
    CUtensorMap tm_q3, tm_kca, tm_kcb;
    const uint64_t kc_rows = static_cast<uint64_t>(p->batch) * p->num_kv_heads * nk;
    if (!make_q_map_3d(&tm_q3, q, static_cast<uint64_t>(p->batch) * Lq, p->num_q_heads, G) ||
        !make_map(&tm_kca, kc, kc_rows, kTcN) || !make_map(&tm_kcb, kc, kc_rows, kTcNB))
      return INFLLMV2_ERR_CUDA;
    const size_t smem = sel_tc_smem_bytes(nblk_cap, G, a.stages);
    auto run = [&](auto kern) -> int {
      int r = set_smem(reinterpret_cast<const void*>(kern), smem);
      if (r != INFLLMV2_OK) return r;
      kern<<<static_cast<unsigned>(grid), kTcThreads, smem, s>>>(tm_q3, tm_kca, tm_kcb, a);
      return launch_status();
    };
    switch (G) {
      case 16: return run(select_prefill_tc_kernel<16>);
      case 8: return run(select_prefill_tc_kernel<8>);
      case 4: return run(select_prefill_tc_kernel<4>);
      case 2: return run(select_prefill_tc_kernel<2>);
      default: return run(select_prefill_tc_kernel<1>);
    }
  }
  // m16n8k16 path: 8 tokens per CTA, one warp per token
  a.tiles_per_bg = (Lq + kSelWarps - 1) / kSelWarps;
  const long long grid = static_cast<long long>(a.tiles_per_bg) * p->batch * p->num_kv_heads;
  if (grid > 0x7fffffffLL) return INFLLMV2_ERR_UNSUPPORTED;
  const size_t smem = sel_prefill_smem_bytes(nblk_cap);
  if ((st = set_smem(reinterpret_cast<const void*>(select_prefill_kernel), smem)) != INFLLMV2_OK) return st;
  select_prefill_kernel<<<static_cast<unsigned>(grid), kSelThreads, smem, s>>>(tm_kc, a);
  return launch_status();
}

int launch_attn(const infllmv2_params* p, const void* q, uint64_t q_rows, const void* k, const void* v,
                uint64_t kv_rows, AttnParams& a, cudaStream_t s);

// Prefill attention for Lq query rows per sequence against caches of Lmax tokens (a fresh
// prefill or a chunk, as for select_prefill).
int attn_prefill(const infllmv2_params* p, const void* q, int32_t Lq, const void* k, const void* v,
                 const int32_t* q_lens, const int32_t* kv_lens, int32_t Lmax, const int32_t* block_idx, void* o,
                 float* lse, cudaStream_t s) {
  if (!q || !k || !v || !block_idx || !o) return INFLLMV2_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(block_idx) || !aligned16(o))
    return INFLLMV2_ERR_INVALID_ARG;
  if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)) return INFLLMV2_ERR_INVALID_ARG;
  const uint64_t q_rows = static_cast<uint64_t>(p->batch) * Lq * p->num_q_heads;
  const uint64_t kv_rows = static_cast<uint64_t>(p->batch) * p->num_kv_heads * Lmax;
  if (q_rows > 0x7fffffffULL || kv_rows > 0x7fffffffULL) return INFLLMV2_ERR_UNSUPPORTED;  // 32-bit TMA rows
  AttnParams a;
  a.idx = block_idx;
  a.lens = nullptr;
  a.q_lens = q_lens;
  a.kv_lens = kv_lens;
  a.B = p->batch;
  a.Hq = p->num_q_heads;
  a.Hkv = p->num_kv_heads;
  a.G = p->num_q_heads / p->num_kv_heads;
  a.Lq = Lq;
  a.Lmax = Lmax;
  a.topk = p->topk;
  a.n_splits = 1;
  a.blocks_per_split = p->topk;
  a.scale_log2 = scale_log2(p);
  a.num_items = static_cast<long long>(p->batch) * p->num_kv_heads * Lq;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.part_o = nullptr;
  a.part_lse = nullptr;
  {
    // tensor-core path: per item, K/V block pairs against 16 query rows from the group's
    // first head (for G < 16 the rows past the group are other heads' queries: their
    // columns of S, P and O are computed and never written; rows past the end of q are
    // zero-filled by the copy)
    CUtensorMap tq, tk, tv;
    if (!make_map(&tq, q, q_rows, kGroupRows) || !make_map(&tk, k, kv_rows, kBlock) ||
        !make_map(&tv, v, kv_rows, kBlock))
      return INFLLMV2_ERR_CUDA;
    const size_t smem = attn_tc_smem_bytes();
    int st = set_smem(reinterpret_cast<const void*>(attn_tc_kernel), smem);
    if (st != INFLLMV2_OK) return st;
    const long long grid = std::min<long long>(a.num_items, num_sms());
    if (grid <= 0) return INFLLMV2_OK;
    attn_tc_kernel<<<static_cast<unsigned>(grid), kAtThreads, smem, s>>>(tq, tk, tv, a);
    return launch_status();
  }
}

int launch_attn(const infllmv2_params* p, const void* q, uint64_t q_rows, const void* k, const void* v,
                       uint64_t kv_rows, AttnParams& a, cudaStream_t s) {
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, q, q_rows, kGroupRows) || !make_map(&tk, k, kv_rows, kBlock) ||
      !make_map(&tv, v, kv_rows, kBlock))
    return INFLLMV2_ERR_CUDA;
  const size_t smem = attn_smem_bytes();
  int st = set_smem(reinterpret_cast<const void*>(attn_kernel), smem);
  if (st != INFLLMV2_OK) return st;
  const long long grid = std::min<long long>(a.num_items, num_sms());
  if (grid <= 0) return INFLLMV2_OK;
  attn_kernel<<<static_cast<unsigned>(grid), kAttnThreads, smem, s>>>(tq, tk, tv, a);
  return launch_status();
}

}  // namespace

extern "C" {

int64_t infllmv2_num_kernels(const infllmv2_params* p, int64_t n) {
  if (p == nullptr || p->kernel_size < 1 || p->kernel_stride < 1 || n < p->kernel_size) return 0;
  return (n - p->kernel_size) / p->kernel_stride + 1;
}

int infllmv2_check_params(const infllmv2_params* p) { return check_params(p); }

int infllmv2_version(void) { return kVersion; }

const char* infllmv2_status_string(int status) {
  switch (status) {
    case INFLLMV2_OK:
      return "ok";
    case INFLLMV2_ERR_INVALID_ARG:
      return "invalid argument";
    case INFLLMV2_ERR_UNSUPPORTED:
      return "unsupported configuration";
    case INFLLMV2_ERR_WORKSPACE:
      return "workspace missing or too small";
    case INFLLMV2_ERR_CUDA:
      return "CUDA error";
    default:
      return "unknown status";
  }
}

size_t infllmv2_workspace_size(const infllmv2_params* p, int op, int32_t L_or_Lmax) {
  return ws_size(p, op, L_or_Lmax);
}

int infllmv2_device_error(int clear) {
  unsigned int v = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return INFLLMV2_ERR_CUDA;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof v) != cudaSuccess) return INFLLMV2_ERR_CUDA;
  if (clear) {
    unsigned int z = 0;
    if (cudaMemcpyToSymbol(g_device_error, &z, sizeof z) != cudaSuccess) return INFLLMV2_ERR_CUDA;
  }
  return static_cast<int>(v);
}

int infllmv2_compress_keys(const infllmv2_params* p, const void* k, const int32_t* lens, int32_t Lmax, void* kc,
                           infllmv2_stream_t stream) {
  int st = check_params(p);
  if (st != INFLLMV2_OK) return st;
  if ((st = check_len(Lmax)) != INFLLMV2_OK) return st;
  if (k == nullptr || !aligned16(k)) return INFLLMV2_ERR_INVALID_ARG;
  if (lens != nullptr && (reinterpret_cast<uintptr_t>(lens) & 3u)) return INFLLMV2_ERR_INVALID_ARG;
  const int nk = static_cast<int>(num_kernels(Lmax));
  if (nk == 0) return INFLLMV2_OK;  // kc has no rows (and may be NULL)
  if (kc == nullptr || !aligned16(kc)) return INFLLMV2_ERR_INVALID_ARG;
  const long long grid =
      static_cast<long long>(p->batch) * p->num_kv_heads * ((nk + kCompressKPC - 1) / kCompressKPC);
  if (grid > 0x7fffffffLL) return INFLLMV2_ERR_UNSUPPORTED;
  compress_kernel<<<static_cast<unsigned>(grid), kCompressThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(k), lens, Lmax, nk, p->num_kv_heads, static_cast<__nv_bfloat16*>(kc));
  return launch_status();
}

int infllmv2_append_kv(const infllmv2_params* p, const void* k_new, const void* v_new, void* k_cache,
                       void* v_cache, int32_t* lens, int32_t Lmax, void* kc, infllmv2_stream_t stream) {
  int st = check_params(p);
  if (st != INFLLMV2_OK) return st;
  if ((st = check_len(Lmax)) != INFLLMV2_OK) return st;
  if (!k_new || !v_new || !k_cache || !v_cache || !lens) return INFLLMV2_ERR_INVALID_ARG;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache) ||
      (reinterpret_cast<uintptr_t>(lens) & 3u))
    return INFLLMV2_ERR_INVALID_ARG;
  const int64_t nk = num_kernels(Lmax);
  if (nk > 0 && (kc == nullptr || !aligned16(kc))) return INFLLMV2_ERR_INVALID_ARG;
  append_kv_kernel<<<static_cast<unsigned>(p->batch), kHeadDim, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(k_new), static_cast<const __nv_bfloat16*>(v_new),
      static_cast<__nv_bfloat16*>(k_cache), static_cast<__nv_bfloat16*>(v_cache), lens, Lmax,
      static_cast<int>(nk), p->num_kv_heads, static_cast<__nv_bfloat16*>(kc));
  return launch_status();
}

int infllmv2_select_blocks(const infllmv2_params* p, int mode, const void* q, const void* kc,
                           const int32_t* lens, int32_t L, int32_t* block_idx, void* ws, size_t ws_bytes,
                           infllmv2_stream_t stream) {
  int st = check_params(p);
  if (st != INFLLMV2_OK) return st;
  if ((st = check_len(L)) != INFLLMV2_OK) return st;
  if (mode == INFLLMV2_MODE_PREFILL) {
    if (lens != nullptr) return INFLLMV2_ERR_INVALID_ARG;
    return select_prefill(p, q, L, kc, nullptr, nullptr, L, block_idx, reinterpret_cast<cudaStream_t>(stream));
  }
  if (mode != INFLLMV2_MODE_DECODE) return INFLLMV2_ERR_INVALID_ARG;
  (void)ws;  // decode selection needs no workspace
  (void)ws_bytes;
  if (q == nullptr || block_idx == nullptr || !aligned16(q) || !aligned16(block_idx)) return INFLLMV2_ERR_INVALID_ARG;
  if (lens == nullptr || (reinterpret_cast<uintptr_t>(lens) & 3u)) return INFLLMV2_ERR_INVALID_ARG;
  const int64_t nk = num_kernels(L);
  if (nk > 0 && (kc == nullptr || !aligned16(kc))) return INFLLMV2_ERR_INVALID_ARG;
  if (static_cast<uint64_t>(p->batch) * p->num_kv_heads * static_cast<uint64_t>(nk) > 0x7fffffffULL)
    return INFLLMV2_ERR_UNSUPPORTED;  // TMA row coordinates are 32-bit
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int G = p->num_q_heads / p->num_kv_heads;
  CUtensorMap tm_kc;
  std::memset(&tm_kc, 0, sizeof tm_kc);
  // a map over a 1-row dummy extent is never dereferenced when there are no kernels
  if (nk > 0 && !make_map(&tm_kc, kc, static_cast<uint64_t>(p->batch) * p->num_kv_heads * nk, kKcTile))
    return INFLLMV2_ERR_CUDA;
  SelDecodeParams a;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.lens = lens;
  a.idx = block_idx;
  a.B = p->batch;
  a.Hq = p->num_q_heads;
  a.Hkv = p->num_kv_heads;
  a.G = G;
  a.Lmax = L;
  a.NKmax = static_cast<int>(nk);
  a.topk = p->topk;
  a.n_init = p->n_init;
  a.n_local = p->n_local;
  a.score_mode = p->score_mode;
  a.pool_mode = p->pool_mode;
  a.scale_log2 = scale_log2(p);
  if (nk == 0 && !make_map(&tm_kc, q, kKcTile, kKcTile)) return INFLLMV2_ERR_CUDA;  // never read: no tiles
  const int C = select_cluster(p, nk);
  const long long grid = static_cast<long long>(C) * p->batch * p->num_kv_heads;
  if (grid > 0x7fffffffLL) return INFLLMV2_ERR_UNSUPPORTED;
  const size_t smem = sel_decode_smem_bytes();
  return launch_cluster(select_decode_kernel, static_cast<unsigned>(grid), C, kSdThreads, smem, s, true, tm_kc,
                        a);
}

int infllmv2_select_blocks_chunk(const infllmv2_params* p, const void* q, int32_t Lq, const void* kc,
                                 const int32_t* q_lens, const int32_t* kv_lens, int32_t Lmax, int32_t* block_idx,
                                 void* ws, size_t ws_bytes, infllmv2_stream_t stream) {
  (void)ws;  // no workspace needed
  (void)ws_bytes;
  int st = check_params(p);
  if (st != INFLLMV2_OK) return st;
  if ((st = check_chunk(Lq, q_lens, kv_lens, Lmax)) != INFLLMV2_OK) return st;
  return select_prefill(p, q, Lq, kc, q_lens, kv_lens, Lmax, block_idx, reinterpret_cast<cudaStream_t>(stream));
}

int infllmv2_sparse_attn_prefill(const infllmv2_params* p, const void* q, const void* k, const void* v,
                                 const int32_t* block_idx, int32_t L, void* o, float* lse, void* ws,
                                 size_t ws_bytes, infllmv2_stream_t stream) {
  (void)ws;
  (void)ws_bytes;
  int st = check_params(p);
  if (st != INFLLMV2_OK) return st;
  if ((st = check_len(L)) != INFLLMV2_OK) return st;
  return attn_prefill(p, q, L, k, v, nullptr, nullptr, L, block_idx, o, lse, reinterpret_cast<cudaStream_t>(stream));
}

int infllmv2_sparse_attn_chunk(const infllmv2_params* p, const void* q, int32_t Lq, const void* k, const void* v,
                               const int32_t* q_lens, const int32_t* kv_lens, int32_t Lmax,
                               const int32_t* block_idx, void* o, float* lse, void* ws, size_t ws_bytes,
                               infllmv2_stream_t stream) {
  (void)ws;  // no workspace needed
  (void)ws_bytes;
  int st = check_params(p);
  if (st != INFLLMV2_OK) return st;
  if ((st = check_chunk(Lq, q_lens, kv_lens, Lmax)) != INFLLMV2_OK) return st;
  return attn_prefill(p, q, Lq, k, v, q_lens, kv_lens, Lmax, block_idx, o, lse,
                      reinterpret_cast<cudaStream_t>(stream));
}

int infllmv2_sparse_attn_backward(const infllmv2_params* p, const void* q, const void* k, const void* v,
                                  const void* o, const float* lse, const void* d_o, const int32_t* block_idx, int32_t L,
                                  void* dq, void* dk, void* dv, void* ws, size_t ws_bytes, infllmv2_stream_t stream) {
  int st = check_params(p);
  if (st != INFLLMV2_OK) return st;
  if ((st = check_len(L)) != INFLLMV2_OK) return st;
  if (!q || !k || !v || !o || !lse || !d_o || !block_idx || !dq || !dk || !dv) return INFLLMV2_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(d_o) || !aligned16(block_idx) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || (reinterpret_cast<uintptr_t>(lse) & 3u))
    return INFLLMV2_ERR_INVALID_ARG;
  const BwdLayout w = bwd_layout(p, L);
  if (ws == nullptr || ws_bytes < w.total || !aligned16(ws)) return INFLLMV2_ERR_WORKSPACE;
  const long long rows = static_cast<long long>(p->batch) * p->num_kv_heads * L;
  const uint64_t q_rows = static_cast<uint64_t>(p->batch) * L * p->num_q_heads;
  if (rows * p->topk > 0x7fffffffLL || q_rows > 0x7fffffffULL || w.n + 1 > 0x7fffffffLL)
    return INFLLMV2_ERR_UNSUPPORTED;  // 32-bit row lists and TMA rows
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned char* wb = static_cast<unsigned char*>(ws);
  BwdParams a;
  a.idx = block_idx;
  a.lse = lse;
  a.delta = reinterpret_cast<float*>(wb + w.delta);
  a.cnt = reinterpret_cast<int32_t*>(wb + w.cnt);
  a.off = reinterpret_cast<int32_t*>(wb + w.off);
  a.segoff = reinterpret_cast<int32_t*>(wb + w.segoff);
  a.list = reinterpret_cast<int32_t*>(wb + w.list);
  a.B = p->batch;
  a.Hq = p->num_q_heads;
  a.Hkv = p->num_kv_heads;
  a.G = p->num_q_heads / p->num_kv_heads;
  a.L = L;
  a.topk = p->topk;
  a.nblk = static_cast<int>(num_blocks(L));
  a.scale_log2 = scale_log2(p);
  a.scale = a.scale_log2 / 1.4426950408889634f;
  a.num_items = rows;
  a.dq = static_cast<__nv_bfloat16*>(dq);
  a.dk32 = reinterpret_cast<float*>(wb + w.dk);
  a.dv32 = reinterpret_cast<float*>(wb + w.dv);
  CUtensorMap tq, tdo, tk, tv;
  if (!make_map(&tq, q, q_rows, kGroupRows) || !make_map(&tdo, d_o, q_rows, kGroupRows) ||
      !make_map(&tk, k, static_cast<uint64_t>(rows), kBlock) || !make_map(&tv, v, static_cast<uint64_t>(rows), kBlock))
    return INFLLMV2_ERR_CUDA;
  // counters and the fp32 accumulators start at zero
  if (cudaMemsetAsync(wb + w.cnt, 0, w.off - w.cnt, s) != cudaSuccess ||
      cudaMemsetAsync(wb + w.dk, 0, w.total - w.dk, s) != cudaSuccess)
    return INFLLMV2_ERR_CUDA;
  const int n = static_cast<int>(w.n);
  bwd_delta_kernel<<<static_cast<unsigned>((q_rows + 7) / 8), 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(d_o), static_cast<const __nv_bfloat16*>(o), p->batch, L, p->num_q_heads,
      const_cast<float*>(a.delta));
  const unsigned rgrid = static_cast<unsigned>((rows + 255) / 256);
  bwd_count_kernel<<<rgrid, 256, 0, s>>>(block_idx, static_cast<int>(rows), L, p->topk, a.nblk,
                                         const_cast<int32_t*>(a.cnt));
  bwd_scan_kernel<<<1, 1024, 0, s>>>(a.cnt, n, const_cast<int32_t*>(a.off), const_cast<int32_t*>(a.segoff));
  bwd_fill_kernel<<<rgrid, 256, 0, s>>>(block_idx, static_cast<int>(rows), L, p->topk, a.nblk, a.off,
                                        reinterpret_cast<int32_t*>(wb + w.cursor), const_cast<int32_t*>(a.list));
  if ((st = launch_status()) != INFLLMV2_OK) return st;
  const size_t smem_q = bwd_dq_smem_bytes(), smem_kv = bwd_dkdv_tc_smem_bytes();
  if ((st = set_smem(reinterpret_cast<const void*>(bwd_dq_kernel), smem_q)) != INFLLMV2_OK) return st;
  if ((st = set_smem(reinterpret_cast<const void*>(bwd_dkdv_tc_kernel), smem_kv)) != INFLLMV2_OK) return st;
  bwd_dq_kernel<<<static_cast<unsigned>(std::min<long long>(rows, num_sms())), kBwdThreads, smem_q, s>>>(tq, tdo, tk,
                                                                                                        tv, a);
  bwd_dkdv_tc_kernel<<<static_cast<unsigned>(num_sms()), kBtThreads, smem_kv, s>>>(tq, tdo, tk, tv, a);
  const long long n4 = rows * kHeadDim / 4;
  bwd_cast_kernel<<<static_cast<unsigned>(std::min<long long>((n4 + 255) / 256, 8LL * num_sms())), 256, 0, s>>>(
      reinterpret_cast<const float4*>(a.dk32), reinterpret_cast<const float4*>(a.dv32), n4, static_cast<uint2*>(dk),
      static_cast<uint2*>(dv));
  return launch_status();
}

int infllmv2_sparse_attn_decode(const infllmv2_params* p, const void* q, const void* k_cache, const void* v_cache,
                                const int32_t* lens, int32_t Lmax, const int32_t* block_idx, void* o, float* lse,
                                void* ws, size_t ws_bytes, infllmv2_stream_t stream) {
  int st = check_params(p);
  if (st != INFLLMV2_OK) return st;
  if ((st = check_len(Lmax)) != INFLLMV2_OK) return st;
  if (!q || !k_cache || !v_cache || !lens || !block_idx || !o) return INFLLMV2_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(block_idx) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(lens) & 3u))
    return INFLLMV2_ERR_INVALID_ARG;
  if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)) return INFLLMV2_ERR_INVALID_ARG;
  const size_t need = ws_size(p, INFLLMV2_OP_ATTN_DECODE, Lmax);
  if (need > 0 && (ws == nullptr || ws_bytes < need || !aligned16(ws))) return INFLLMV2_ERR_WORKSPACE;
  const uint64_t kv_rows = static_cast<uint64_t>(p->batch) * p->num_kv_heads * Lmax;
  if (kv_rows > 0x7fffffffULL) return INFLLMV2_ERR_UNSUPPORTED;  // TMA row coordinates are 32-bit
  const DecodePlan d = decode_plan(p);
  AttnParams a;
  a.idx = block_idx;
  a.lens = lens;
  a.q_lens = nullptr;
  a.kv_lens = nullptr;
  a.B = p->batch;
  a.Hq = p->num_q_heads;
  a.Hkv = p->num_kv_heads;
  a.G = p->num_q_heads / p->num_kv_heads;
  a.Lq = 1;
  a.Lmax = Lmax;
  a.topk = p->topk;
  a.n_splits = d.n_splits;
  a.blocks_per_split = d.per_split;
  a.scale_log2 = scale_log2(p);
  a.num_items = static_cast<long long>(p->batch) * p->num_kv_heads * d.n_splits;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.part_o = nullptr;
  a.part_lse = nullptr;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const uint64_t q_rows = static_cast<uint64_t>(p->batch) * p->num_q_heads;
  if (d.cluster > 0) {
    CUtensorMap tq, tk, tv;
    if (!make_map(&tq, q, q_rows, kGroupRows) || !make_map(&tk, k_cache, kv_rows, kBlock) ||
        !make_map(&tv, v_cache, kv_rows, kBlock))
      return INFLLMV2_ERR_CUDA;
    const long long grid = static_cast<long long>(d.cluster) * p->batch * p->num_kv_heads;
    if (grid > 0x7fffffffLL) return INFLLMV2_ERR_UNSUPPORTED;
    return launch_cluster(attn_decode_cluster_kernel, static_cast<unsigned>(grid), d.cluster, kAdThreads,
                          attn_dec_smem_bytes(), s, true, tq, tk, tv, a);
  }
  const size_t rows = static_cast<size_t>(p->batch) * p->num_kv_heads * d.n_splits * kGroupRows;
  a.part_o = static_cast<float*>(ws);
  a.part_lse = a.part_o + rows * kHeadDim;
  st = launch_attn(p, q, q_rows, k_cache, v_cache, kv_rows, a, s);
  if (st != INFLLMV2_OK) return st;
  attn_merge_kernel<<<static_cast<unsigned>(static_cast<long long>(p->batch) * p->num_kv_heads * a.G), 128, 0, s>>>(
      a.part_o, a.part_lse, d.n_splits, p->num_q_heads, p->num_kv_heads, a.G, static_cast<__nv_bfloat16*>(o), lse);
  return launch_status();
}

int infllmv2_decode_step(const infllmv2_params* p, const void* q, const void* k_new, const void* v_new, void* k_cache,
                         void* v_cache, void* kc, const int32_t* lens, int32_t* lens_out, int32_t Lmax,
                         int32_t* block_idx, void* o, float* lse, infllmv2_stream_t stream) {
  int st = check_params(p);
  if (st != INFLLMV2_OK) return st;
  if ((st = check_len(Lmax)) != INFLLMV2_OK) return st;
  if (!q || !k_cache || !v_cache || !lens || !block_idx || !o) return INFLLMV2_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(block_idx) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(lens) & 3u))
    return INFLLMV2_ERR_INVALID_ARG;
  if ((k_new == nullptr) != (v_new == nullptr)) return INFLLMV2_ERR_INVALID_ARG;
  if (k_new != nullptr) {  // append: the new rows, and a separate array for the new lengths
    if (!aligned16(k_new) || !aligned16(v_new) || lens_out == nullptr || lens_out == lens ||
        (reinterpret_cast<uintptr_t>(lens_out) & 3u) || kc == nullptr)
      return INFLLMV2_ERR_INVALID_ARG;
  }
  if (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)) return INFLLMV2_ERR_INVALID_ARG;
  const int64_t nk = num_kernels(Lmax);
  if (nk > 0 && (kc == nullptr || !aligned16(kc))) return INFLLMV2_ERR_INVALID_ARG;
  const uint64_t kv_rows = static_cast<uint64_t>(p->batch) * p->num_kv_heads * Lmax;
  if (kv_rows > 0x7fffffffULL ||
      static_cast<uint64_t>(p->batch) * p->num_kv_heads * static_cast<uint64_t>(nk) > 0x7fffffffULL)
    return INFLLMV2_ERR_UNSUPPORTED;  // TMA row coordinates are 32-bit
  const int G = p->num_q_heads / p->num_kv_heads;
  DecodeStepParams P;
  SelDecodeParams& a = P.sel;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.lens = lens;
  a.idx = block_idx;
  a.B = p->batch;
  a.Hq = p->num_q_heads;
  a.Hkv = p->num_kv_heads;
  a.G = G;
  a.Lmax = Lmax;
  a.NKmax = static_cast<int>(nk);
  a.topk = p->topk;
  a.n_init = p->n_init;
  a.n_local = p->n_local;
  a.score_mode = p->score_mode;
  a.pool_mode = p->pool_mode;
  a.scale_log2 = scale_log2(p);
  AttnParams& t = P.attn;
  t.idx = block_idx;
  t.lens = lens;
  t.q_lens = nullptr;
  t.kv_lens = nullptr;
  t.B = p->batch;
  t.Hq = p->num_q_heads;
  t.Hkv = p->num_kv_heads;
  t.G = G;
  t.Lq = 1;
  t.Lmax = Lmax;
  t.topk = p->topk;
  t.n_splits = 1;
  t.blocks_per_split = p->topk;
  t.scale_log2 = a.scale_log2;
  t.num_items = static_cast<long long>(p->batch) * p->num_kv_heads;
  t.o = static_cast<__nv_bfloat16*>(o);
  t.lse = lse;
  t.part_o = nullptr;
  t.part_lse = nullptr;
  P.k_new = static_cast<const __nv_bfloat16*>(k_new);
  P.v_new = static_cast<const __nv_bfloat16*>(v_new);
  P.k_cache = static_cast<__nv_bfloat16*>(k_cache);
  P.v_cache = static_cast<__nv_bfloat16*>(v_cache);
  P.kc = static_cast<__nv_bfloat16*>(kc);
  P.lens_out = lens_out;
  CUtensorMap tm_kc, tq, tk, tv;
  std::memset(&tm_kc, 0, sizeof tm_kc);
  const uint64_t q_rows = static_cast<uint64_t>(p->batch) * p->num_q_heads;
  // with no complete kernel a map over a dummy extent is never dereferenced
  if (!(nk > 0 ? make_map(&tm_kc, kc, static_cast<uint64_t>(p->batch) * p->num_kv_heads * nk, kKcTile)
               : make_map(&tm_kc, q, kKcTile, kKcTile)) ||
      !make_map(&tq, q, q_rows, kGroupRows) || !make_map(&tk, k_cache, kv_rows, kBlock) ||
      !make_map(&tv, v_cache, kv_rows, kBlock))
    return INFLLMV2_ERR_CUDA;
  const int C = decode_step_cluster(p, nk);
  const long long grid = static_cast<long long>(C) * p->batch * p->num_kv_heads;
  if (grid > 0x7fffffffLL) return INFLLMV2_ERR_UNSUPPORTED;
  return launch_cluster(decode_step_kernel, static_cast<unsigned>(grid), C, kSdThreads, decode_step_smem_bytes(),
                        reinterpret_cast<cudaStream_t>(stream), true, tm_kc, tq, tk, tv, P);
}

}  // extern "C"

// ------------------------------------------------ decode attention without allocation
// The split partials of infllmv2_sparse_attn_decode_noalloc live in this file-scope
// device array instead of a caller workspace.  Host code only ever sees the symbol's
// host-side stand-in, so the device address is looked up once per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[INFLLMV2_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return INFLLMV2_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return INFLLMV2_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) return INFLLMV2_ERR_CUDA;
    g_noalloc_ptr[dev] = ptr;
  }
  *out = g_noalloc_ptr[dev];
  return INFLLMV2_OK;
}
}  // namespace

extern "C" int infllmv2_sparse_attn_decode_noalloc(const infllmv2_params* p, const void* q, const void* k_cache,
                                                   const void* v_cache, const int32_t* lens, int32_t Lmax,
                                                   const int32_t* block_idx, void* o, float* lse,
                                                   infllmv2_stream_t stream) {
  const int st = check_params(p);
  if (st != INFLLMV2_OK) return st;
  const size_t need = ws_size(p, INFLLMV2_OP_ATTN_DECODE, Lmax);
  if (need == static_cast<size_t>(-1)) return INFLLMV2_ERR_INVALID_ARG;
  if (need > INFLLMV2_NOALLOC_SCRATCH_BYTES) return INFLLMV2_ERR_WORKSPACE;
  void* scratch = nullptr;
  const int sst = noalloc_scratch(&scratch);
  if (sst != INFLLMV2_OK) return sst;
  return infllmv2_sparse_attn_decode(p, q, k_cache, v_cache, lens, Lmax, block_idx, o, lse, scratch,
                                     INFLLMV2_NOALLOC_SCRATCH_BYTES, stream);
}
