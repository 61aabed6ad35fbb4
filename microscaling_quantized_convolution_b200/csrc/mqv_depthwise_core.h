// Depthwise layers in BF16 (MicroQonv summary, onedev.kr/papers/182,
// section "전제와 한계": the depthwise convolutions stay in BF16, outside
// the quantized path).  One Kh x Kw filter per channel, weights [C][Kh][Kw],
// activations and gradients channel-batch-first [H][W][C][N] like the rest
// of the path; operands are bfloat16 bit patterns, products are summed with
// fp32 FMAs in a fixed order, outputs are fp32.
//
// The per-thread work of the three passes: each function takes the linear
// index of one GPU thread and does all of that thread's loads, arithmetic
// and stores.  The kernels in mqv_depthwise.cuh are one call each; the same
// functions compile for the host too, so their indexing and arithmetic can be
// run over every thread index on a CPU.
#pragma once

#include <cstdint>
#include <cstring>
#include <cmath>

#if defined(__CUDACC__)
#define MQV_DW_HD __host__ __device__ __forceinline__
#else
#define MQV_DW_HD inline
#endif

namespace mqv {

struct DwGeom {
  int64_t N, C, H, W, Kh, Kw, stride, pad, Ho, Wo;
  int64_t parts;        // weight gradient: (ho, wo) ranges per (c, kh, kw)
};

MQV_DW_HD float dw_bf16(uint16_t b) {
#if defined(__CUDA_ARCH__)
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
#else
  const uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return f;
#endif
}

MQV_DW_HD float dw_fma(float a, float b, float c) {
#if defined(__CUDA_ARCH__)
  return __fmaf_rn(a, b, c);
#else
  return std::fmaf(a, b, c);
#endif
}

// Threads of the forward and input-gradient passes: one per four
// consecutive batch items of one (pixel, channel).
MQV_DW_HD int64_t dw_fwd_threads(const DwGeom& g) { return g.Ho * g.Wo * g.C * (g.N / 4); }
MQV_DW_HD int64_t dw_dgrad_threads(const DwGeom& g) { return g.H * g.W * g.C * (g.N / 4); }
// Weight gradient: one thread per (part, c, kh, kw), c fastest.
MQV_DW_HD int64_t dw_wgrad_threads(const DwGeom& g) { return g.parts * g.C * g.Kh * g.Kw; }

// y[ho][wo][c][n0..n0+3] = sum over the taps (kh, kw), in that order, of
// w[c][kh][kw]·x[ho·s + kh - p][wo·s + kw - p][c][n] (taps outside the
// input skipped).
MQV_DW_HD void dw_fwd_thread(const DwGeom& g, int64_t t, const uint16_t* w, const uint16_t* x, float* y) {
  const int64_t n4 = g.N / 4;
  const int64_t n0 = (t % n4) * 4;
  int64_t r = t / n4;
  const int64_t c = r % g.C;
  r /= g.C;
  const int64_t wo = r % g.Wo, ho = r / g.Wo;
  float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  for (int64_t kh = 0; kh < g.Kh; ++kh) {
    const int64_t hi = ho * g.stride + kh - g.pad;
    if (hi < 0 || hi >= g.H) continue;
    for (int64_t kw = 0; kw < g.Kw; ++kw) {
      const int64_t wi = wo * g.stride + kw - g.pad;
      if (wi < 0 || wi >= g.W) continue;
      const float wv = dw_bf16(w[(c * g.Kh + kh) * g.Kw + kw]);
      const uint16_t* xp = x + ((hi * g.W + wi) * g.C + c) * g.N + n0;
      for (int j = 0; j < 4; ++j) acc[j] = dw_fma(wv, dw_bf16(xp[j]), acc[j]);
    }
  }
  float* yp = y + ((ho * g.Wo + wo) * g.C + c) * g.N + n0;
  for (int j = 0; j < 4; ++j) yp[j] = acc[j];
}

// gx[hi][wi][c][n0..n0+3] = sum over the taps (kh, kw), in that order, whose
// output pixel ho = (hi + p - kh) / s, wo = (wi + p - kw) / s exists, of
// w[c][kh][kw]·gy[ho][wo][c][n]: the adjoint of the forward pass, gathered.
MQV_DW_HD void dw_dgrad_thread(const DwGeom& g, int64_t t, const uint16_t* w, const uint16_t* gy, float* gx) {
  const int64_t n4 = g.N / 4;
  const int64_t n0 = (t % n4) * 4;
  int64_t r = t / n4;
  const int64_t c = r % g.C;
  r /= g.C;
  const int64_t wi = r % g.W, hi = r / g.W;
  float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  for (int64_t kh = 0; kh < g.Kh; ++kh) {
    const int64_t th = hi + g.pad - kh;
    if (th < 0 || th % g.stride) continue;
    const int64_t ho = th / g.stride;
    if (ho >= g.Ho) continue;
    for (int64_t kw = 0; kw < g.Kw; ++kw) {
      const int64_t tw = wi + g.pad - kw;
      if (tw < 0 || tw % g.stride) continue;
      const int64_t wo = tw / g.stride;
      if (wo >= g.Wo) continue;
      const float wv = dw_bf16(w[(c * g.Kh + kh) * g.Kw + kw]);
      const uint16_t* gp = gy + ((ho * g.Wo + wo) * g.C + c) * g.N + n0;
      for (int j = 0; j < 4; ++j) acc[j] = dw_fma(wv, dw_bf16(gp[j]), acc[j]);
    }
  }
  float* op = gx + ((hi * g.W + wi) * g.C + c) * g.N + n0;
  for (int j = 0; j < 4; ++j) op[j] = acc[j];
}

// Output pixels [q0, q1) of part `part` of the weight gradient (q = ho·Wo +
// wo): the parts split Ho·Wo as evenly as integers allow.
MQV_DW_HD void dw_part_range(const DwGeom& g, int64_t part, int64_t& q0, int64_t& q1) {
  const int64_t q = g.Ho * g.Wo;
  q0 = part * q / g.parts;
  q1 = (part + 1) * q / g.parts;
}

// partial[part][c][kh][kw] = sum over the part's output pixels q (in
// order) and the batch items n of gy[q][c][n]·x[hi][wi][c][n], four running
// sums (n mod 4) added pairwise at the end, so each running sum has at most
// a quarter of the part's terms.
MQV_DW_HD void dw_wgrad_thread(const DwGeom& g, int64_t t, const uint16_t* gy, const uint16_t* x,
                               float* partial) {
  const int64_t c = t % g.C;
  int64_t r = t / g.C;
  const int64_t kw = r % g.Kw;
  r /= g.Kw;
  const int64_t kh = r % g.Kh, part = r / g.Kh;
  int64_t q0, q1;
  dw_part_range(g, part, q0, q1);
  float a[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  for (int64_t q = q0; q < q1; ++q) {
    const int64_t ho = q / g.Wo, wo = q - ho * g.Wo;
    const int64_t hi = ho * g.stride + kh - g.pad, wi = wo * g.stride + kw - g.pad;
    if (hi < 0 || hi >= g.H || wi < 0 || wi >= g.W) continue;
    const uint16_t* gp = gy + (q * g.C + c) * g.N;
    const uint16_t* xp = x + ((hi * g.W + wi) * g.C + c) * g.N;
    for (int64_t n = 0; n < g.N; n += 4)
      for (int j = 0; j < 4; ++j) a[j] = dw_fma(dw_bf16(gp[n + j]), dw_bf16(xp[n + j]), a[j]);
  }
  partial[((part * g.C + c) * g.Kh + kh) * g.Kw + kw] = (a[0] + a[1]) + (a[2] + a[3]);
}

// gw[c][kh][kw] = the parts' sums added in part order (one thread per entry).
MQV_DW_HD void dw_wgrad_reduce_thread(const DwGeom& g, int64_t t, const float* partial, float* gw) {
  const int64_t per = g.C * g.Kh * g.Kw;
  float s = partial[t];
  for (int64_t p = 1; p < g.parts; ++p) s += partial[p * per + t];
  gw[t] = s;
}

// Parts of the weight gradient: at most about 1024 terms per running sum;
// for small layers up to 16 parts, to spread the (part, c, kh, kw) threads
// over more SMs; never more parts than output pixels.  The reduction then
// adds that many partial sums per weight.
inline int64_t dw_wgrad_parts(int64_t N, int64_t C, int64_t Kh, int64_t Kw, int64_t Ho, int64_t Wo) {
  const int64_t q = Ho * Wo;
  const int64_t by_terms = (q * (N / 4) + 1023) / 1024;
  int64_t by_threads = (148 * 512 + C * Kh * Kw - 1) / (C * Kh * Kw);
  if (by_threads > 16) by_threads = 16;
  int64_t p = by_terms > by_threads ? by_terms : by_threads;
  if (p > q) p = q;
  return p < 1 ? 1 : p;
}

// The geometry of a layer whose descriptor has been checked.
inline DwGeom dw_geom(int64_t N, int64_t C, int64_t H, int64_t W, int64_t Kh, int64_t Kw, int64_t stride,
                      int64_t pad) {
  DwGeom g;
  g.N = N;
  g.C = C;
  g.H = H;
  g.W = W;
  g.Kh = Kh;
  g.Kw = Kw;
  g.stride = stride;
  g.pad = pad;
  g.Ho = (H + 2 * pad - Kh) / stride + 1;
  g.Wo = (W + 2 * pad - Kw) / stride + 1;
  g.parts = dw_wgrad_parts(N, C, Kh, Kw, g.Ho, g.Wo);
  return g;
}

}  // namespace mqv
