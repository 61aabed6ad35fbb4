// Input gradient of 4-channel stems on CUDA cores (MicroQonv summary,
// onedev.kr/papers/182, section "무엇과 다른가": G_X' = W^T·G_Y, then
// col2im, here gathered directly).
//
// With few input channels the pass is bound by memory, not by tensor work:
// each G_X element takes Cout·(taps reaching it) products.  A YOLO-style
// stem (4 input channels, 16 output channels, 3x3, stride 2) takes 36
// multiply-adds per element, against 4 B written and 0.8 B read.  The
// tensor-core kernel would spend a whole 128-row MMA tile on 4 channels, so
// this kernel computes the gather on CUDA cores:
//   - the CTA dequantizes the weights once into shared memory as fp32
//     ([kh][kw][co][ci]; code·B is exact in fp32);
//   - a thread owns 16 consecutive batch items of one input pixel, for all
//     4 input channels;
//   - for every tap that reaches the pixel it walks the G_Y rows of the
//     output pixel four channels at a time (four 4x4 blocks: one scale word
//     and one wide code load per channel row), dequantized with the
//     tensor-core path's fp16 arithmetic (exact), then multiplies them with
//     the shared weights in fp32 FMAs;
//   - its results, times T_w·T_g, go out as 16-byte stores.
// Consecutive threads take consecutive pixels, so a warp's code loads and
// result stores are runs of neighbouring pixels.  The grid is persistent,
// so the weights are dequantized once per CTA.  No wait on another thread
// block, no barrier other than the one after the weights.
#pragma once

#include <cstdint>

#include "mqv_conv_common.cuh"
#include "mqv_conv_kernels.cuh"

namespace mqv {

constexpr int kNarrowThreads = 256;
constexpr int kNarrowMaxWeightBytes = 48 * 1024;   // Cout x Kh x Kw x 4 fp32 in shared memory

// Value of element (row, col) of a 4x4-block view as fp32 (code·B, exact).
template <int FMT>
__device__ __forceinline__ float narrow_value(const QView& v, int64_t row, int64_t col) {
  const uint8_t* rp = v.codes + row * v.row_bytes;
  uint32_t code;
  if (FMT == 0) {
    code = (__ldg(rp + (col >> 1)) >> ((col & 1) * 4)) & 0xFu;
  } else {
    const uint8_t* q = rp + (col >> 2) * 3;
    const uint32_t w = static_cast<uint32_t>(__ldg(q)) | (static_cast<uint32_t>(__ldg(q + 1)) << 8) |
                       (static_cast<uint32_t>(__ldg(q + 2)) << 16);
    code = (w >> ((col & 3) * 6)) & 0x3Fu;
  }
  const uint32_t s = __ldg(v.scales + (row >> 2) * v.scale_cols + (col >> 2));
  const uint32_t h = hmul2_u32(FMT == 0 ? e2m1x2_to_f16x2(code) : e2m3x2_to_f16x2(code), scale2(s));
  return f16_lo_to_f32(h);
}

// One thread per input pixel and 16 batch items, for all 4 input channels
// (64 accumulators).  Per tap and 4-channel group of G_Y: one scale word
// (the four 4x4 blocks along the 16 items) and, per channel row, the 16
// codes as one 8-byte (FP4) or three 4-byte (FP6) loads.
template <int FMT>
__global__ void __launch_bounds__(kNarrowThreads)
conv_narrow_dgrad_kernel(const V2Args p, const QView w) {
  extern __shared__ float wsm[];
  constexpr int M = 4;                      // input channels (= p.Cin)
  const int Cout = p.Cout, Kw = p.Kw, taps = p.Kh * p.Kw;
  const int K = taps * M;                   // columns of W's view, (kh, kw, ci)
  for (int e = threadIdx.x; e < Cout * K; e += blockDim.x) {
    const int co = e / K, k = e - co * K;
    const int tap = k / M, ci = k - tap * M;
    wsm[(tap * Cout + co) * M + ci] = narrow_value<FMT>(w, co, k);
  }
  __syncthreads();
  const float scale = __fmul_rn(*p.ta, *p.tb);
  const int ng = p.N >> 4;
  const int64_t units = static_cast<int64_t>(p.H) * p.W * ng;
  const int64_t step = static_cast<int64_t>(gridDim.x) * blockDim.x;
  float amax = 0.0f;
  for (int64_t u = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; u < units; u += step) {
    const int g16 = static_cast<int>(u % ng);
    const int64_t pix = u / ng;
    const int wi = static_cast<int>(pix % p.W), hi = static_cast<int>(pix / p.W);
    float acc[M][16];
#pragma unroll
    for (int ci = 0; ci < M; ++ci)
#pragma unroll
      for (int j = 0; j < 16; ++j) acc[ci][j] = 0.0f;
    for (int kh = 0; kh < p.Kh; ++kh) {
      const int th = hi + p.pad - kh;
      if (th < 0 || th % p.stride) continue;
      const int ho = th / p.stride;
      if (ho >= p.Ho) continue;
      for (int kw = 0; kw < Kw; ++kw) {
        const int tw = wi + p.pad - kw;
        if (tw < 0 || tw % p.stride) continue;
        const int wo = tw / p.stride;
        if (wo >= p.Wo) continue;
        const int64_t grow = (static_cast<int64_t>(ho) * p.Wo + wo) * Cout;
        const float* wt = wsm + (kh * Kw + kw) * Cout * M;
        for (int cb = 0; cb < Cout; cb += 4) {
          // scales of the four 4x4 blocks (channels cb..cb+3, items 16·g16 + 4q ..)
          const uint32_t s = __ldg(reinterpret_cast<const uint32_t*>(
              p.b.scales + ((grow + cb) >> 2) * p.b.scale_cols + 4 * g16));
          const uint32_t s0 = scale2(s & 0xFF), s1 = scale2((s >> 8) & 0xFF);
          const uint32_t s2 = scale2((s >> 16) & 0xFF), s3 = scale2(s >> 24);
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const uint8_t* cp = p.b.codes + (grow + cb + r) * p.b.row_bytes;
            uint32_t h[8];
            if (FMT == 0) {
              const uint2 v = __ldg(reinterpret_cast<const uint2*>(cp + 8 * g16));
              uint32_t a[4], b[4];
              dq8_fp4(v.x, s0, s1, a);
              dq8_fp4(v.y, s2, s3, b);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                h[q] = a[q];
                h[4 + q] = b[q];
              }
            } else {
              const uint32_t* q = reinterpret_cast<const uint32_t*>(cp + 12 * g16);
              const uint32_t c0 = __ldg(q), c1 = __ldg(q + 1), c2 = __ldg(q + 2);
              dq4_fp6(c0 & 0xFFFFFF, s0, h[0], h[1]);
              dq4_fp6((c0 >> 24) | ((c1 & 0xFFFF) << 8), s1, h[2], h[3]);
              dq4_fp6((c1 >> 16) | ((c2 & 0xFF) << 16), s2, h[4], h[5]);
              dq4_fp6(c2 >> 8, s3, h[6], h[7]);
            }
            float gv[16];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              gv[2 * q] = f16_lo_to_f32(h[q]);
              gv[2 * q + 1] = f16_hi_to_f32(h[q]);
            }
            const float4 wv = *reinterpret_cast<const float4*>(wt + (cb + r) * M);
            const float wr[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
            for (int ci = 0; ci < M; ++ci)
#pragma unroll
              for (int j = 0; j < 16; ++j) acc[ci][j] = __fmaf_rn(wr[ci], gv[j], acc[ci][j]);
          }
        }
      }
    }
    float* op = p.out + ((static_cast<int64_t>(hi) * p.W + wi) * M) * p.N + 16 * g16;
#pragma unroll
    for (int ci = 0; ci < M; ++ci)
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float4 o = make_float4(acc[ci][4 * q] * scale, acc[ci][4 * q + 1] * scale,
                                     acc[ci][4 * q + 2] * scale, acc[ci][4 * q + 3] * scale);
        if (p.amax_out) amax = epi_absmax(amax, o);
        *reinterpret_cast<float4*>(op + static_cast<int64_t>(ci) * p.N + 4 * q) = o;
      }
  }
  epi_amax_flush(p.amax_out, amax);
}

}  // namespace mqv
