// common.cuh -- device helpers shared by the InfLLM v2 kernels (sm_100a).
//
// PTX wrappers for mbarriers, TMA tile loads (never with cluster multicast),
// ldmatrix and the bf16 m16n8k16 MMA, plus time-bounded mbarrier waits: a wait that
// exceeds its limit sets a device error word and marks the CTA aborted, after which
// every later wait in the CTA -- and, through the sticky error word, in every other CTA
// until the word is cleared -- returns at once, so the kernel runs to its end instead
// of hanging.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace infllmv2 {

constexpr int kHeadDim = 128;
constexpr int kBlock = 64;         // KV block length (tokens)
constexpr int kKernel = 32;        // semantic kernel length
constexpr int kStride = 16;        // semantic kernel stride
constexpr int kGroupRows = 16;     // q-heads per group handled as one MMA row tile
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per wait

// Device error word (one per device), read by infllmv2_device_error().
__device__ unsigned int g_device_error;
constexpr unsigned int kDevErrWaitTimeout = 1u;  // a bounded wait ran out (later waits give up at once)

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// ----------------------------------------------------------------- mbarriers

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t addr, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(addr), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test that the phase with the given parity has completed (valid only
// while the barrier is at most one phase past the one the caller last waited for).
__device__ __forceinline__ bool mbar_test(const uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for the phase with the given parity to complete.  Returns false (and sets
// the device error word and *abort) when the time limit passes or the CTA was
// already aborted; the caller then proceeds without the data.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  const uint32_t addr = smem_u32(bar);
  if (mbar_try_wait(addr, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(addr, parity)) return true;
    if ((it & 63u) == 63u) {
      if (*abort) return false;
      if ((*reinterpret_cast<volatile unsigned int*>(&g_device_error) & kDevErrWaitTimeout) != 0u) {  // another CTA gave up
        *abort = 1;
        return false;
      }
      if (globaltimer_ns() - t0 > kWaitLimitNs) {
        *abort = 1;
        atomicOr(&g_device_error, kDevErrWaitTimeout);
        return false;
      }
    }
  }
}

// Waits like mbar_wait but ignores the CTA abort flag (only the time limit): used for
// the final drains that must complete before TMEM or shared memory is released.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity) {
  const uint32_t addr = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(addr, parity)) return true;
    if ((it & 63u) == 63u && globaltimer_ns() - t0 > kWaitLimitNs) {
      atomicOr(&g_device_error, kDevErrWaitTimeout);
      return false;
    }
  }
}

// ---------------------------------------------------------------------- TMA

// 2-D tiled bulk tensor load global -> shared, completion counted in bytes on `bar`.
// x is the innermost coordinate (elements), y the row.  No multicast.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// L2 policy that evicts first the lines a bulk copy brings in (for data read once, so it
// does not push reused data out of L2).
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// tma_load_2d with an L2 cache policy for the copied lines.
__device__ __forceinline__ void tma_load_2d_hint(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y,
                                                 uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(policy)
      : "memory");
}

// Streaming (evict-first) store of one bf16 value: output written once, not read again.
__device__ __forceinline__ void st_stream_bf16(__nv_bfloat16* p, __nv_bfloat16 v) {
  asm volatile("st.global.cs.b16 [%0], %1;" ::"l"(p), "h"(*reinterpret_cast<unsigned short*>(&v)) : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Orders this thread's generic-proxy shared-memory writes before later async-proxy
// (TMA) accesses of the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// The same for global memory: this thread's generic writes before later bulk-tensor
// (async proxy) reads of them, by this or (after a barrier) another thread.
__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

// Programmatic dependent launch.  grid_dependency_wait() returns once every grid this
// one depends on has completed and its memory writes are visible (at once when there is
// none); nothing may read what an earlier kernel on the stream wrote before it.
// allow_dependent_launch() lets the next kernel on the stream, when launched with
// programmatic stream serialization, start its own prologue early.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void allow_dependent_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Byte offset of 16-byte chunk `chunk` (0..7) of row `row` inside a tile written by
// TMA with 128-byte swizzling (rows of 128 bytes, tile base 1024-byte aligned).
__device__ __forceinline__ uint32_t sw128(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

// ------------------------------------------------------------ warp-level MMA

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D = A * B + D, m16n8k16, bf16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_bf16(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Hardware base-2 exponential and logarithm (PTX ex2.approx / lg2.approx).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Named barrier with an OR reduction of `pred` over the participating threads.
__device__ __forceinline__ bool named_bar_or(int id, int nthreads, bool pred) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(out)
      : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(nthreads)
      : "memory");
  return out != 0;
}

// Rounds a shared-memory pointer up to a multiple of `align` bytes.
__device__ __forceinline__ unsigned char* align_smem(unsigned char* p, uint32_t align) {
  uint32_t a = smem_u32(p);
  uint32_t r = (a + align - 1) & ~(align - 1);
  return p + (r - a);
}

// Order-preserving image of a float in uint32 (a < b exactly when enc(a) < enc(b)), so
// that integer atomicMax computes a float max.  Never 0 for a non-NaN float.
__device__ __forceinline__ uint32_t ord_enc(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float ord_dec(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Block-score variants of the selection (the pages leave the score and the pooling
// open): softmax-sum (sum over heads of exp(block max - lse)) or logit-sum (sum over
// heads of the block max logit, no lse); overlapping kernels 4j-1 .. 4j+3 or the kernels
// inside the block 4j .. 4j+2.
constexpr int kScoreSoftmaxSum = 0, kScoreLogitSum = 1;
constexpr int kPoolOverlap = 0, kPoolInside = 1;

// Top-k key of a candidate block's score: a larger score gives a larger key, and 0 is
// left for non-candidates.  Softmax-sum scores are >= 0: their bit patterns + 1; logit
// sums may be negative: the order-preserving image.
__device__ __forceinline__ uint32_t score_key(float s, int score_mode) {
  return score_mode == kScoreLogitSum ? ord_enc(s) : __float_as_uint(s) + 1u;
}

// Block j has a visible pooled kernel for a query whose last visible kernel is imax.
__device__ __forceinline__ bool block_eligible(int j, int imax, int pool_mode) {
  return (pool_mode == kPoolInside ? 4 * j : max(4 * j - 1, 0)) <= imax;
}

// Semantic-kernel arithmetic for block 64 / kernel 32 / stride 16: kernel i covers
// tokens [16 i, 16 i + 32) and is visible to the query at t iff 16 i + 31 <= t.
// Highest visible kernel index for position t (-1 when none).
__device__ __forceinline__ int last_visible_kernel(int t) {
  return t >= kKernel - 1 ? (t - (kKernel - 1)) / kStride : -1;
}

// Queries and cache of sequence b in a prefill chunk: q_len queries, the last q_len of
// kv_len cached tokens (so query row r sits at position kv_len - q_len + r).  Lengths
// outside [0, Lq] and [0, Lmax] are clamped, and q_len to at most kv_len.
struct ChunkLens {
  int q_len, kv_len;
};
__device__ __forceinline__ ChunkLens chunk_lens(const int32_t* q_lens, const int32_t* kv_lens, int b, int Lq,
                                                int Lmax) {
  ChunkLens c;
  c.kv_len = kv_lens ? min(max(kv_lens[b], 0), Lmax) : Lmax;
  c.q_len = q_lens ? min(max(q_lens[b], 0), Lq) : Lq;
  c.q_len = min(c.q_len, c.kv_len);
  return c;
}

}  // namespace infllmv2
