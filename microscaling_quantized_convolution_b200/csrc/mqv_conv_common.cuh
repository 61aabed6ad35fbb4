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
constexpr uint32_t kErrWaitEmpty = 1u, kErrWaitFull = 2u, kErrWaitDone = 4u, kErrWaitSelfTest = 8u;

struct QView {
  const uint8_t* codes;
  const uint8_t* scales;
  const float* tscale;
  int64_t row_bytes;    // bytes per row of packed codes
  int64_t scale_cols;   // entries per row of the scale plane (cols / 4, cols / 16 or cols by `blocks`)
  int32_t blocks;       // scale blocks: 0 4 x 4, 1 1 x 16 along a row, 2 16 x 1 down a column
};

// Scale-plane index of element (row, col) of a view.
__device__ __forceinline__ int64_t scale_index(const QView& v, int64_t row, int64_t col) {
  if (v.blocks == 1) return row * v.scale_cols + (col >> 4);
  if (v.blocks == 2) return (row >> 4) * v.scale_cols + col;
  return (row >> 2) * v.scale_cols + (col >> 2);
}

// Byte offset of (row, k) inside a K-major, 128-byte-swizzled fp16 tile.
__device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t k) {
  return row * 128u + ((((k >> 3) ^ (row & 7u)) << 4) | ((k & 4u) << 1));
}

// G_W = T_g·T_x·sum over splits of the partial tiles.  A block takes 64
// float4 columns; four thread groups each add a contiguous quarter of the
// splits in split order, and the four group sums are added in group order, so
// the result is the same on every run.  Sixteen independent loads per thread
// keep enough bytes in flight to run at memory speed.  The partials are
// scratch: with `discard` set (128-byte aligned lines, checked on the host)
// each 128-byte line, once the block has read it, is dropped from L2 without
// being written back (PTX discard.global.L2), so the partials cost no DRAM
// writes when they never left L2.
constexpr int kReduceCols = 64, kReduceGroups = 4;
__global__ void __launch_bounds__(kReduceCols * kReduceGroups)
wgrad_reduce_kernel(const float4* __restrict__ partial, int splits, int64_t n4,
                    const float* __restrict__ ta, const float* __restrict__ tb,
                    float4* __restrict__ out, int discard) {
  __shared__ float4 part[kReduceGroups][kReduceCols];
  const int col = threadIdx.x % kReduceCols, grp = threadIdx.x / kReduceCols;
  const int64_t i = static_cast<int64_t>(blockIdx.x) * kReduceCols + col;
  const int per = (splits + kReduceGroups - 1) / kReduceGroups;
  const int s0 = grp * per, s1 = min(splits, s0 + per);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (i < n4 && s0 < s1) {
    acc = __ldg(partial + static_cast<int64_t>(s0) * n4 + i);
    int s = s0 + 1;
    constexpr int kBatch = 16;
    for (; s + kBatch <= s1; s += kBatch) {
      float4 v[kBatch];
#pragma unroll
      for (int b = 0; b < kBatch; ++b) v[b] = __ldg(partial + static_cast<int64_t>(s + b) * n4 + i);
#pragma unroll
      for (int b = 0; b < kBatch; ++b) {
        acc.x += v[b].x;
        acc.y += v[b].y;
        acc.z += v[b].z;
        acc.w += v[b].w;
      }
    }
    for (; s < s1; ++s) {
      const float4 v = __ldg(partial + static_cast<int64_t>(s) * n4 + i);
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
  }
  part[grp][col] = acc;
  __syncthreads();
  // every partial of this block's columns has been read and added: drop
  // their lines (one 128-byte line per 8 columns and split)
  if (discard && (col & 7) == 0 && i + 7 < n4) {
    for (int s = s0; s < s1; ++s)
      asm volatile("discard.global.L2 [%0], 128;" ::"l"(partial + static_cast<int64_t>(s) * n4 + i) : "memory");
  }
  if (grp == 0 && i < n4) {
    float4 t = part[0][col];
#pragma unroll
    for (int g = 1; g < kReduceGroups; ++g) {
      const float4 v = part[g][col];
      t.x += v.x;
      t.y += v.y;
      t.z += v.z;
      t.w += v.w;
    }
    const float scale = __fmul_rn(*ta, *tb);
    t.x *= scale;
    t.y *= scale;
    t.z *= scale;
    t.w *= scale;
    out[i] = t;
  }
}

}  // namespace mqv
