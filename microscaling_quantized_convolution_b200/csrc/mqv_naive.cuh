// Explicit im2col and its adjoint col2im on fp32 tensors, for the baseline the
// method is measured against (MicroQonv summary, onedev.kr/papers/182, section
// "무엇인가": quantizing after the im2col expansion, once per GEMM direction).
// The expanded matrix X' keeps the channel-batch-first order with the
// im2col row index in the channel position:
//   X'[(ho, wo)][(kh, kw, ci)][n] = X[ho·s + kh - p][wo·s + kw - p][ci][n]
// (zero outside), so a 1 x 1 convolution over X' with Kh·Kw·Cin input
// channels is exactly the forward GEMM Y = W·X', and its 2D view is the
// (Ho·Wo·Kh·Kw·Cin) x N view the quantizer takes.
#pragma once

#include <cstdint>

#include "mqv_ptx.cuh"

namespace mqv {

struct Im2colGeom {
  int N, Cin, H, W, Kh, Kw, stride, pad, Ho, Wo;
  FastDiv dn4;      // N / 4
  FastDiv dcin;     // Cin
  FastDiv dk;       // Kh·Kw·Cin
  FastDiv dkw;      // Kw
  FastDiv dwo;      // Wo
  FastDiv dw;       // W
};

constexpr int kNaiveThreads = 256;

// One thread per 4 batch items of X' (a float4): copy or zero.
__global__ void __launch_bounds__(kNaiveThreads)
im2col_kernel(const Im2colGeom g, const float4* __restrict__ x, float4* __restrict__ xc, int64_t n4) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kNaiveThreads;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kNaiveThreads + threadIdx.x; i < n4; i += stride) {
    // i = ((p·K + k)·N/4 + n4)
    const int row = fdiv(static_cast<int>(i), g.dn4);          // p·K + k (below 2^31: checked on the host)
    const int q = static_cast<int>(i - static_cast<int64_t>(row) * (g.N / 4));
    const int p = fdiv(row, g.dk);
    const int k = row - p * (g.Kh * g.Kw * g.Cin);
    const int tap = fdiv(k, g.dcin);
    const int ci = k - tap * g.Cin;
    const int kh = fdiv(tap, g.dkw), kw = tap - kh * g.Kw;
    const int ho = fdiv(p, g.dwo), wo = p - ho * g.Wo;
    const int hi = ho * g.stride + kh - g.pad, wi = wo * g.stride + kw - g.pad;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (hi >= 0 && hi < g.H && wi >= 0 && wi < g.W)
      v = __ldg(x + ((static_cast<int64_t>(hi) * g.W + wi) * g.Cin + ci) * (g.N / 4) + q);
    xc[i] = v;
  }
}

// One thread per float4 of G_X: the sum over the taps that read pixel
// (hi, wi), in (kh, kw) order, of G_X'[(ho, wo)][(kh, kw, ci)][n].
__global__ void __launch_bounds__(kNaiveThreads)
col2im_kernel(const Im2colGeom g, const float4* __restrict__ gc, float4* __restrict__ gx, int64_t n4) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kNaiveThreads;
  const int K = g.Kh * g.Kw * g.Cin;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kNaiveThreads + threadIdx.x; i < n4; i += stride) {
    const int row = fdiv(static_cast<int>(i), g.dn4);          // (hi·W + wi)·Cin + ci
    const int q = static_cast<int>(i - static_cast<int64_t>(row) * (g.N / 4));
    const int pix = fdiv(row, g.dcin);
    const int ci = row - pix * g.Cin;
    const int hi = fdiv(pix, g.dw), wi = pix - hi * g.W;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int kh = 0; kh < g.Kh; ++kh) {
      const int th = hi + g.pad - kh;
      if (th < 0 || th % g.stride) continue;
      const int ho = th / g.stride;
      if (ho >= g.Ho) continue;
      for (int kw = 0; kw < g.Kw; ++kw) {
        const int tw = wi + g.pad - kw;
        if (tw < 0 || tw % g.stride) continue;
        const int wo = tw / g.stride;
        if (wo >= g.Wo) continue;
        const int64_t src = ((static_cast<int64_t>(ho) * g.Wo + wo) * K + (kh * g.Kw + kw) * g.Cin + ci) * (g.N / 4) + q;
        const float4 v = __ldg(gc + src);
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      }
    }
    gx[i] = acc;
  }
}

}  // namespace mqv
