// compress.cuh -- semantic-kernel key compression.
//
// MiniCPM4 summary page (端设备上的超高效大型语言模型) s2.1.2: every KV block is
// represented through fine-grained "semantic kernels".  Kernel i of a (sequence,
// kv-head) is the mean of key rows [16 i, 16 i + 32).
//
// Each half-warp streams KPH consecutive kernels: it sums 16-row groups R_r (16 lanes x
// 16-byte loads = one 256-byte key row per step) and emits kernel i = (R_i + R_{i+1}) / 32
// as soon as R_{i+1} is complete, so every key row is read once per half-warp range
// (one extra 16-row group per range).  The group sums are kept in fp64, where the sum
// of 32 bf16 values is exact for any realistic exponent spread, so the kernel value is
// the exact mean rounded once to bf16 (nearest even) -- an fp32 sum can be off by many
// bf16 ulps when the mean nearly cancels.  One DADD per loaded element; the kernel is
// bound by HBM bandwidth: 256 bytes read per key row, 256 bytes written per kernel.
#pragma once
#include "common.cuh"

namespace infllmv2 {

constexpr int kCompressKPH = 16;      // kernels per half-warp
constexpr int kCompressThreads = 128;  // 8 half-warps

__device__ __forceinline__ void add_row(double* acc, uint4 v) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    float2 f = __bfloat1622float2(h[e]);
    acc[2 * e] += static_cast<double>(f.x);
    acc[2 * e + 1] += static_cast<double>(f.y);
  }
}

// Sum of the 16 key rows [16 r, 16 r + 16) for this lane's 8 columns.
__device__ __forceinline__ void group_sum(const uint4* rows, int r, double* acc) {
  uint4 v[16];
#pragma unroll
  for (int u = 0; u < 16; ++u) v[u] = __ldg(rows + static_cast<size_t>(16 * r + u) * 16);
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.0;
#pragma unroll
  for (int u = 0; u < 16; ++u) add_row(acc, v[u]);
}

// grid = (ceil(ceil(NKmax / KPH) / 8), Hkv, B), block = 128.
__global__ void __launch_bounds__(kCompressThreads) compress_kernel(const __nv_bfloat16* __restrict__ k,
                                                                    const int32_t* __restrict__ lens, int Lmax,
                                                                    int NKmax, int Hkv,
                                                                    __nv_bfloat16* __restrict__ kc) {
  const int b = blockIdx.z, g = blockIdx.y;
  const int hw = (blockIdx.x * kCompressThreads + threadIdx.x) >> 4;
  const int lane = threadIdx.x & 15;
  int n = lens ? lens[b] : Lmax;
  n = n < 0 ? 0 : (n > Lmax ? Lmax : n);
  const int nk = n >= kKernel ? (n - kKernel) / kStride + 1 : 0;
  const int i0 = hw * kCompressKPH;
  if (i0 >= nk) return;
  const int i1 = min(i0 + kCompressKPH, nk);
  const size_t bg = static_cast<size_t>(b) * Hkv + g;
  const uint4* rows = reinterpret_cast<const uint4*>(k + bg * Lmax * kHeadDim) + lane;
  uint4* out = reinterpret_cast<uint4*>(kc + bg * NKmax * kHeadDim) + lane;
  double prev[8], cur[8];
  group_sum(rows, i0, prev);
  for (int i = i0; i < i1; ++i) {
    group_sum(rows, i + 1, cur);
    uint4 o;
    uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      __nv_bfloat162 pr;
      pr.x = __double2bfloat16((prev[2 * e] + cur[2 * e]) * (1.0 / kKernel));
      pr.y = __double2bfloat16((prev[2 * e + 1] + cur[2 * e + 1]) * (1.0 / kKernel));
      ow[e] = *reinterpret_cast<uint32_t*>(&pr);
    }
    out[static_cast<size_t>(i) * 16] = o;
#pragma unroll
    for (int e = 0; e < 8; ++e) prev[e] = cur[e];
  }
}

}  // namespace infllmv2
