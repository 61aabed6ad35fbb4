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

// Four consecutive bfloat16 elements (8-byte aligned: N % 4 == 0 and
// 16-byte aligned tensors) as fp32, one 8-byte load on the GPU; and four
// fp32 results stored together (16-byte aligned).
MQV_DW_HD void dw_load4(const uint16_t* p, float (&v)[4]) {
#if defined(__CUDA_ARCH__)
  const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
  v[0] = __uint_as_float(u.x << 16);
  v[1] = __uint_as_float(u.x & 0xFFFF0000u);
  v[2] = __uint_as_float(u.y << 16);
  v[3] = __uint_as_float(u.y & 0xFFFF0000u);
#else
  for (int j = 0; j < 4; ++j) v[j] = dw_bf16(p[j]);
#endif
}

MQV_DW_HD void dw_store4(float* p, const float (&v)[4]) {
#if defined(__CUDA_ARCH__)
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
#else
  for (int j = 0; j < 4; ++j) p[j] = v[j];
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
  // every tensor has fewer than 2^31 elements (checked on the host), so
  // 32-bit indices suffice
  const int n4 = static_cast<int>(g.N / 4), C = static_cast<int>(g.C), Wo = static_cast<int>(g.Wo);
  const int H = static_cast<int>(g.H), W = static_cast<int>(g.W), N = static_cast<int>(g.N);
  const int Kh = static_cast<int>(g.Kh), Kw = static_cast<int>(g.Kw);
  const int s = static_cast<int>(g.stride), p = static_cast<int>(g.pad);
  int r = static_cast<int>(t);
  const int n0 = (r % n4) * 4;
  r /= n4;
  const int c = r % C;
  r /= C;
  const int wo = r % Wo, ho = r / Wo;
  float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  for (int kh = 0; kh < Kh; ++kh) {
    const int hi = ho * s + kh - p;
    if (hi < 0 || hi >= H) continue;
    for (int kw = 0; kw < Kw; ++kw) {
      const int wi = wo * s + kw - p;
      if (wi < 0 || wi >= W) continue;
      const float wv = dw_bf16(w[(c * Kh + kh) * Kw + kw]);
      float xv[4];
      dw_load4(x + ((hi * W + wi) * C + c) * N + n0, xv);
      for (int j = 0; j < 4; ++j) acc[j] = dw_fma(wv, xv[j], acc[j]);
    }
  }
  dw_store4(y + ((ho * Wo + wo) * C + c) * N + n0, acc);
}

// gx[hi][wi][c][n0..n0+3] = sum over the taps (kh, kw), in that order, whose
// output pixel ho = (hi + p - kh) / s, wo = (wi + p - kw) / s exists, of
// w[c][kh][kw]·gy[ho][wo][c][n]: the adjoint of the forward pass, gathered.
MQV_DW_HD void dw_dgrad_thread(const DwGeom& g, int64_t t, const uint16_t* w, const uint16_t* gy, float* gx) {
  const int n4 = static_cast<int>(g.N / 4), C = static_cast<int>(g.C), W = static_cast<int>(g.W);
  const int Ho = static_cast<int>(g.Ho), Wo = static_cast<int>(g.Wo), N = static_cast<int>(g.N);
  const int Kh = static_cast<int>(g.Kh), Kw = static_cast<int>(g.Kw);
  const int s = static_cast<int>(g.stride), p = static_cast<int>(g.pad);
  int r = static_cast<int>(t);
  const int n0 = (r % n4) * 4;
  r /= n4;
  const int c = r % C;
  r /= C;
  const int wi = r % W, hi = r / W;
  float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  for (int kh = 0; kh < Kh; ++kh) {
    const int th = hi + p - kh;
    if (th < 0 || th % s) continue;
    const int ho = th / s;
    if (ho >= Ho) continue;
    for (int kw = 0; kw < Kw; ++kw) {
      const int tw = wi + p - kw;
      if (tw < 0 || tw % s) continue;
      const int wo = tw / s;
      if (wo >= Wo) continue;
      const float wv = dw_bf16(w[(c * Kh + kh) * Kw + kw]);
      float gv[4];
      dw_load4(gy + ((ho * Wo + wo) * C + c) * N + n0, gv);
      for (int j = 0; j < 4; ++j) acc[j] = dw_fma(wv, gv[j], acc[j]);
    }
  }
  dw_store4(gx + ((hi * W + wi) * C + c) * N + n0, acc);
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
  const int C = static_cast<int>(g.C), H = static_cast<int>(g.H), W = static_cast<int>(g.W);
  const int Wo = static_cast<int>(g.Wo), N = static_cast<int>(g.N);
  const int Kh = static_cast<int>(g.Kh), Kw = static_cast<int>(g.Kw);
  const int s = static_cast<int>(g.stride), p = static_cast<int>(g.pad);
  int r = static_cast<int>(t);
  const int c = r % C;
  r /= C;
  const int kw = r % Kw;
  r /= Kw;
  const int kh = r % Kh, part = r / Kh;
  int64_t q0, q1;
  dw_part_range(g, part, q0, q1);
  float a[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  int ho = static_cast<int>(q0) / Wo, wo = static_cast<int>(q0) - ho * Wo;   // (ho, wo) of q, stepped along
  for (int q = static_cast<int>(q0); q < static_cast<int>(q1); ++q) {
    const int hi = ho * s + kh - p, wi = wo * s + kw - p;
    if (hi >= 0 && hi < H && wi >= 0 && wi < W) {
      const uint16_t* gp = gy + (q * C + c) * N;
      const uint16_t* xp = x + ((hi * W + wi) * C + c) * N;
      for (int n = 0; n < N; n += 4) {
        float gv[4], xv[4];
        dw_load4(gp + n, gv);
        dw_load4(xp + n, xv);
        for (int j = 0; j < 4; ++j) a[j] = dw_fma(gv[j], xv[j], a[j]);
      }
    }
    if (++wo == Wo) {
      wo = 0;
      ++ho;
    }
  }
  partial[((part * C + c) * Kh + kh) * Kw + kw] = (a[0] + a[1]) + (a[2] + a[3]);
}

// gw[c][kh][kw] = the parts' sums added in part order (one thread per entry).
MQV_DW_HD void dw_wgrad_reduce_thread(const DwGeom& g, int64_t t, const float* partial, float* gw) {
  const int64_t per = g.C * g.Kh * g.Kw;
  float s = partial[t];
  for (int64_t p = 1; p < g.parts; ++p) s += partial[p * per + t];
  gw[t] = s;
}

// Parts of the weight gradient: at most about 512 terms per running sum;
// for small layers up to 64 parts, to put about 1024 (part, c, kh, kw)
// threads on each SM; never more parts than output pixels.  The reduction
// then adds that many partial sums per weight.
inline int64_t dw_wgrad_parts(int64_t N, int64_t C, int64_t Kh, int64_t Kw, int64_t Ho, int64_t Wo) {
  const int64_t q = Ho * Wo;
  const int64_t by_terms = (q * (N / 4) + 511) / 512;
  int64_t by_threads = (148 * 1024 + C * Kh * Kw - 1) / (C * Kh * Kw);
  if (by_threads > 64) by_threads = 64;
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
