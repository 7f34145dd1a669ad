// append.cuh -- decode cache maintenance: one new token per sequence and step.
//
// MiniCPM4 summary page (端设备上的超高效大型语言模型) s2.1: InfLLM v2 serves decoding as
// well as prefill; s2.1.2: the semantic kernels summarise the cached keys.  Every decode
// step adds one key row and one value row per (sequence, kv-head).  Kernel i covers key
// rows [16 i, 16 i + 32) and exists once its last row does, so the step whose new length
// is n = 32 + 16 i (i >= 0) completes kernel i.  Its value is the mean of those 32 rows
// with the arithmetic of compress_kernel: an fp64 sum (exact for bf16 inputs) rounded
// once to bf16, so an appended cache holds the same kernels a full compression gives.
// Bound by latency (a few dependent memory round trips): 512 bytes written per (sequence,
// kv-head), plus 8 KB read and 256 bytes written when a kernel completes.
#pragma once
#include "common.cuh"

namespace infllmv2 {

constexpr unsigned int kDevErrCacheFull = 2u;  // an append found lens[b] outside [0, Lmax)

// grid = B, block = 128 (thread = column d).  lens[b] is read once, the new rows of every
// kv-head are written at position lens[b], a completed kernel is emitted, then
// lens[b] += 1.  A sequence whose cache is full (or whose length is negative) is left
// untouched and sets kDevErrCacheFull.
__global__ void __launch_bounds__(kHeadDim)
    append_kv_kernel(const __nv_bfloat16* __restrict__ k_new, const __nv_bfloat16* __restrict__ v_new,
                     __nv_bfloat16* __restrict__ k_cache, __nv_bfloat16* __restrict__ v_cache,
                     int32_t* __restrict__ lens, int Lmax, int NKmax, int Hkv, __nv_bfloat16* __restrict__ kc) {
  const int b = blockIdx.x, d = threadIdx.x;
  const int pos = lens[b];
  if (pos < 0 || pos >= Lmax) {  // same value for every thread: uniform exit
    if (d == 0) atomicOr(&g_device_error, kDevErrCacheFull);
    return;
  }
  const int n = pos + 1;
  const bool completes = n >= kKernel && (n - kKernel) % kStride == 0;
  const int ki = (n - kKernel) / kStride;
  for (int g = 0; g < Hkv; ++g) {
    const size_t bg = static_cast<size_t>(b) * Hkv + g;
    const __nv_bfloat16 kv = k_new[bg * kHeadDim + d];
    k_cache[(bg * Lmax + pos) * kHeadDim + d] = kv;
    v_cache[(bg * Lmax + pos) * kHeadDim + d] = v_new[bg * kHeadDim + d];
    if (completes) {
      // the 31 cached rows are loaded together (one round trip), then summed
      const __nv_bfloat16* rows = k_cache + (bg * Lmax + static_cast<size_t>(kStride) * ki) * kHeadDim + d;
      __nv_bfloat16 r_[kKernel - 1];
#pragma unroll
      for (int r = 0; r < kKernel - 1; ++r) r_[r] = rows[r * kHeadDim];
      double s = 0.0;
#pragma unroll
      for (int r = 0; r < kKernel - 1; ++r) s += static_cast<double>(__bfloat162float(r_[r]));
      s += static_cast<double>(__bfloat162float(kv));  // the new row, from the input
      kc[(bg * NKmax + ki) * kHeadDim + d] = __double2bfloat16(s * (1.0 / kKernel));
    }
  }
  __syncthreads();  // every thread has read lens[b]
  if (d == 0) lens[b] = n;
}

}  // namespace infllmv2
