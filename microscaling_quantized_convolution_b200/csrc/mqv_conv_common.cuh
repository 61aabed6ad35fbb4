// Definitions shared by the convolution kernels and the C ABI: the device
// view of a quantized tensor, pass identifiers, device error bits, the
// K-major 128-byte swizzle, and the deterministic split-K reduction of the
// weight gradient.
#pragma once

#include <cstdint>

#include "mqv_ptx.cuh"

namespace mqv {

enum ConvPass { kFwd = 0, kWgrad = 1, kDgrad = 2 };

// Device error bits set by bounded waits.
constexpr uint32_t kErrWaitEmpty = 1u, kErrWaitFull = 2u, kErrWaitDone = 4u;

struct QView {
  const uint8_t* codes;
  const uint8_t* scales;
  const float* tscale;
  int64_t row_bytes;    // bytes per row of packed codes
  int64_t scale_cols;   // blocks per row of the scale plane (= cols / 4)
};

// Byte offset of (row, k) inside a K-major, 128-byte-swizzled fp16 tile.
__device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t k) {
  return row * 128u + ((((k >> 3) ^ (row & 7u)) << 4) | ((k & 4u) << 1));
}

// G_W = T_g·T_x·sum over splits of the partial tiles, in split order.
__global__ void __launch_bounds__(256)
wgrad_reduce_kernel(const float4* __restrict__ partial, int splits, int64_t n4,
                    const float* __restrict__ ta, const float* __restrict__ tb,
                    float4* __restrict__ out) {
  const float scale = __fmul_rn(*ta, *tb);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  constexpr int kBatch = 8;     // loads in flight per thread; the adds stay in split order
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 acc = __ldg(partial + i);
    int s = 1;
    for (; s + kBatch <= splits; s += kBatch) {
      float4 v[kBatch];
#pragma unroll
      for (int b = 0; b < kBatch; ++b) v[b] = __ldg(partial + (s + b) * n4 + i);
#pragma unroll
      for (int b = 0; b < kBatch; ++b) {
        acc.x += v[b].x;
        acc.y += v[b].y;
        acc.z += v[b].z;
        acc.w += v[b].w;
      }
    }
    for (; s < splits; ++s) {
      const float4 v = __ldg(partial + s * n4 + i);
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    acc.x *= scale;
    acc.y *= scale;
    acc.z *= scale;
    acc.w *= scale;
    out[i] = acc;
  }
}

}  // namespace mqv
