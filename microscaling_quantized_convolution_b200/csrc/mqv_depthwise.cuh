// Kernels of the BF16 depthwise layers: one thread per unit of work of
// mqv_depthwise_core.h.  Memory-bound (Kh·Kw multiply-adds per element), so
// no tensor cores: consecutive threads take consecutive groups of four
// batch items, then channels, so a warp's loads and stores are contiguous
// runs of the [H][W][C][N] tensors.
#pragma once

#include <cstdint>

#include "mqv_depthwise_core.h"

namespace mqv {

constexpr int kDwThreads = 256;

__global__ void __launch_bounds__(kDwThreads)
dw_fwd_kernel(const DwGeom g, int64_t total, const uint16_t* __restrict__ w, const uint16_t* __restrict__ x,
              float* __restrict__ y) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kDwThreads + threadIdx.x;
  if (t < total) dw_fwd_thread(g, t, w, x, y);
}

__global__ void __launch_bounds__(kDwThreads)
dw_dgrad_kernel(const DwGeom g, int64_t total, const uint16_t* __restrict__ w, const uint16_t* __restrict__ gy,
                float* __restrict__ gx) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kDwThreads + threadIdx.x;
  if (t < total) dw_dgrad_thread(g, t, w, gy, gx);
}

__global__ void __launch_bounds__(kDwThreads)
dw_wgrad_kernel(const DwGeom g, int64_t total, const uint16_t* __restrict__ gy, const uint16_t* __restrict__ x,
                float* __restrict__ partial) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kDwThreads + threadIdx.x;
  if (t < total) dw_wgrad_thread(g, t, gy, x, partial);
}

__global__ void __launch_bounds__(kDwThreads)
dw_wgrad_reduce_kernel(const DwGeom g, int64_t total, const float* __restrict__ partial, float* __restrict__ gw) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * kDwThreads + threadIdx.x;
  if (t < total) dw_wgrad_reduce_thread(g, t, partial, gw);
}

}  // namespace mqv
