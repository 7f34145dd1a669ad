// compress.cuh -- semantic-kernel key compression.
//
// MiniCPM4 summary page (端设备上的超高效大型语言模型) s2.1.2: every KV block is
// represented through fine-grained "semantic kernels".  Kernel i of a (sequence,
// kv-head) is the mean of key rows [16 i, 16 i + 32).
//
// A CTA writes kCompressKPC consecutive kernels of one (sequence, kv-head).  It reads the
// kCompressKPC + 1 groups of 16 key rows they span (one group more than it writes, so
// 1/31 of the rows are read twice): thread (slot s, 16-byte column chunk c) sums, for its
// 8 columns, the 16 rows of groups s and s + 16 -- a half-warp reads one 256-byte row per
// load, and each thread keeps its 32 loads in flight -- into shared memory, then thread
// (s, c) emits kernels s and s + 16, kernel i = (R_i + R_{i+1}) / 32.  The whole grid is
// resident at once at the largest sizes (no tail wave).  The group sums are kept in fp64,
// where the sum of 32 bf16 values is exact for any realistic exponent spread, so the
// kernel value is the exact mean rounded once to bf16 (nearest even) -- an fp32 sum can be
// off by many bf16 ulps when the mean nearly cancels.  Bound by HBM bandwidth: 256 bytes
// read per key row, 256 bytes written per kernel.
#pragma once
#include "common.cuh"

namespace infllmv2 {

constexpr int kCompressKPC = 31;                        // kernels written per CTA
constexpr int kCompressGroups = kCompressKPC + 1;       // 16-row groups read per CTA
constexpr int kCompressThreads = 16 * kCompressGroups / 2;  // thread = (slot, 16-byte column chunk)

__device__ __forceinline__ void compress_group_sum(const uint4* rows, double (&acc)[8]) {
  uint4 v[16];
#pragma unroll
  for (int u = 0; u < 16; ++u) v[u] = __ldg(rows + u * 16);
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v[u]);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(h[e]);
      acc[2 * e] += static_cast<double>(f.x);
      acc[2 * e + 1] += static_cast<double>(f.y);
    }
  }
}

// grid = B * Hkv * ceil(NKmax / kCompressKPC) (tiles of one (b, g) consecutive), block = 256.
__global__ void __launch_bounds__(kCompressThreads) compress_kernel(const __nv_bfloat16* __restrict__ k,
                                                                    const int32_t* __restrict__ lens, int Lmax,
                                                                    int NKmax, int Hkv,
                                                                    __nv_bfloat16* __restrict__ kc) {
  __shared__ double gsum[kCompressGroups][16][8];
  const int tiles = (NKmax + kCompressKPC - 1) / kCompressKPC;
  const long long bg = blockIdx.x / tiles;
  const int tile = static_cast<int>(blockIdx.x % tiles);
  const int b = static_cast<int>(bg / Hkv);
  int n = lens ? lens[b] : Lmax;
  n = n < 0 ? 0 : (n > Lmax ? Lmax : n);
  const int nk = n >= kKernel ? (n - kKernel) / kStride + 1 : 0;
  const int i0 = tile * kCompressKPC;
  if (i0 >= nk) return;  // uniform over the CTA
  const int i_end = min(i0 + kCompressKPC, nk);  // kernels i0 .. i_end - 1 need groups i0 .. i_end
  const int sl = threadIdx.x >> 4, ch = threadIdx.x & 15;
  const uint4* base = reinterpret_cast<const uint4*>(k + (bg * Lmax + 16LL * i0) * kHeadDim) + ch;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int gr = sl + 16 * half;
    double acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.0;
    if (i0 + gr <= i_end) compress_group_sum(base + gr * 16 * 16, acc);  // rows < 16 (i_end - 1) + 32 <= n
#pragma unroll
    for (int e = 0; e < 8; ++e) gsum[gr][ch][e] = acc[e];
  }
  __syncthreads();
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int gr = sl + 16 * half;
    const int i = i0 + gr;
    if (gr < kCompressKPC && i < nk) {
      uint4 o;
      uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        __nv_bfloat162 pr;
        pr.x = __double2bfloat16((gsum[gr][ch][2 * e] + gsum[gr + 1][ch][2 * e]) * (1.0 / kKernel));
        pr.y = __double2bfloat16((gsum[gr][ch][2 * e + 1] + gsum[gr + 1][ch][2 * e + 1]) * (1.0 / kKernel));
        ow[e] = *reinterpret_cast<uint32_t*>(&pr);
      }
      reinterpret_cast<uint4*>(kc + (bg * NKmax + i) * kHeadDim)[ch] = o;
    }
  }
}

}  // namespace infllmv2
