// Kernels of the BF16 depthwise layers.  Memory-bound (Kh·Kw multiply-adds
// per element), so no tensor cores.
//   - The gathers: one thread per unit of work of mqv_depthwise_core.h;
//     consecutive threads take consecutive groups of four batch items, then
//     channels, so a warp's loads and stores are contiguous runs of the
//     [H][W][C][N] tensors.  They serve the layers the tiles do not take.
//   - The spatial tiles (dw_tile_kernel, dw_wgrad_tile_kernel): a CTA
//     stages the window its output tile reads once in shared memory and
//     computes from there.
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

// Spatial tiles.  A CTA takes TH x TW output pixels of CG channels (all N
// batch items) and stages in shared memory the window of its source tensor
// those pixels read, IH x IW pixels of CG·N bf16 each (zeros outside the
// tensor), with asynchronous 8- or 16-byte copies that zero-fill out of
// range, so every thread has all its copies in flight at once.  Each source
// pixel then comes from memory once per tile instead of once per tap.
//   forward:  source x, window origin (ho0·s - p, wo0·s - p), tap (kh, kw) of
//             output (ho, wo) at window row (ho - ho0)·s + kh;
//   DGRAD:    source G_Y, the adjoint gathered: G_X pixel (hi, wi) takes tap
//             (kh, kw) where hi + p - kh is a multiple of s, from G_Y row
//             (hi + p - kh) / s; window origin r0 = floor((hi0 + p - Kh + 1) / s).
// Taps run in (kh, kw) order, as in dw_fwd_thread and dw_dgrad_thread; a tap
// that lands outside the source reads a staged zero (adds +0·w).  Results go
// out as float4 stores.  S: the stride when it is 1 or 2 (cheap index
// arithmetic), 0 for any other.  ROWS3: 3x3 filters in tiles 8 wide, one
// output row per thread (dw_tile_rows3); otherwise a thread takes one output
// pixel of one (channel, batch quad) lane at a time, taps in runtime loops.
// PIX: the staged pixel's size in bf16 (CG·N) when it is one of 32 .. 512,
// so that the row path's shared-memory offsets are constants; 0 otherwise.
struct DwTile {
  int th, tw, cg;          // output pixels per tile (rows, columns), channels per tile
  int ih, iw;              // staged window, pixels (rows, columns)
  int src_h, src_w;        // extent of the source (x, or G_Y for the input gradient)
  int out_h, out_w;        // extent of the output
  int tiles_w, tiles_h;    // tiles along the output width and height
  int vec16;               // 1: 16-byte copies (C·N and CG·N multiples of 8), else 8-byte
  int rows3;               // 1: the 3x3 row path (tw = 8)
};

__device__ __forceinline__ int dw_floordiv(int a, int b) { return a >= 0 ? a / b : -((-a + b - 1) / b); }

// Stages rows x cols pixels of a [h][w][C][N] source, origin (r0, q0),
// channels c0 .. c0 + pix_elems / N - 1, into shared memory at dst
// ([row][col][pix_elems] bf16) with asynchronous 16- or 8-byte copies; pixels
// outside the source are zero-filled (a copy of 0 source bytes).  The caller
// commits and waits.
__device__ __forceinline__ void dw_stage(uint16_t* dst, const uint16_t* __restrict__ src, int r0, int q0, int rows,
                                         int cols, int src_h, int src_w, int C, int N, int c0, int pix_elems,
                                         int vec16) {
  const int vb = vec16 ? 8 : 4;                   // bf16 per copy
  const int v_per_pix = pix_elems / vb;
  const int ncopy = rows * cols * v_per_pix;
  const uint32_t base = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
  // copy e = (y·cols + x)·v_per_pix + v; each thread steps e by kDwThreads,
  // so (y, x, v) advance by fixed amounts with at most one carry each
  // (every tensor has fewer than 2^31 elements, so 32-bit offsets suffice)
  int pix = threadIdx.x / v_per_pix;
  int v = threadIdx.x - pix * v_per_pix;
  int y = pix / cols, x = pix - y * cols;
  const int dp = kDwThreads / v_per_pix, dv = kDwThreads - dp * v_per_pix;
  const int dy = dp / cols, dx = dp - dy * cols;
  const int pix_stride = C * N;
  for (int e = threadIdx.x; e < ncopy; e += kDwThreads) {
    const int sh = r0 + y, sw = q0 + x;
    const bool in = sh >= 0 && sh < src_h && sw >= 0 && sw < src_w;
    const uint16_t* gp = src + (in ? static_cast<uint32_t>((sh * src_w + sw) * pix_stride + c0 * N + v * vb) : 0u);
    const uint32_t da = base + static_cast<uint32_t>(((y * cols + x) * pix_elems + v * vb) * 2);
    if (vec16)
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(da), "l"(gp), "r"(in ? 16 : 0) : "memory");
    else
      asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;\n" ::"r"(da), "l"(gp), "r"(in ? 8 : 0) : "memory");
    v += dv;
    x += dx;
    y += dy;
    if (v >= v_per_pix) {
      v -= v_per_pix;
      ++x;
    }
    if (x >= cols) {
      x -= cols;
      ++y;
    }
  }
}

// a[e] = fma(w, x[e], a[e]) for e = 0..3, as two packed fp32 FMAs
// (fma.rn.f32x2: each lane one IEEE fp32 FMA, the same result as fmaf).
__device__ __forceinline__ void dw_fma4(float (&a)[4], float w, const float (&x)[4]) {
  asm("{\n\t.reg .b64 p, q, r;\n\t"
      "mov.b64 q, {%4, %4};\n\t"
      "mov.b64 p, {%5, %6};\n\t"
      "mov.b64 r, {%0, %1};\n\t"
      "fma.rn.f32x2 r, p, q, r;\n\t"
      "mov.b64 {%0, %1}, r;\n\t"
      "mov.b64 p, {%7, %8};\n\t"
      "mov.b64 r, {%2, %3};\n\t"
      "fma.rn.f32x2 r, p, q, r;\n\t"
      "mov.b64 {%2, %3}, r;\n\t}"
      : "+f"(a[0]), "+f"(a[1]), "+f"(a[2]), "+f"(a[3])
      : "f"(w), "f"(x[0]), "f"(x[1]), "f"(x[2]), "f"(x[3]));
}

// One staged G_Y row of the stride-2 input gradient into the 8 sums of a
// G_X row.  The tile starts at an even column, so G_X column ox takes tap kw
// when ox + P + kw is even (P = p mod 2), from staged column
// (ox + P + 2 - kw) / 2; the columns are walked right to left so that each
// output sees kw in ascending order.
template <int P, int PIX>
__device__ __forceinline__ void dw_dgrad2_row(const uint16_t* rp, int pix_rt, const float* wk, float (&acc)[8][4]) {
  const int pix_elems = PIX ? PIX : pix_rt;
#pragma unroll
  for (int jj = 0; jj < 6; ++jj) {
    const int j = 5 - jj;
    const uint2 v = *reinterpret_cast<const uint2*>(rp + j * pix_elems);
    const float x[4] = {__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xFFFF0000u),
                        __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xFFFF0000u)};
#pragma unroll
    for (int kw = 0; kw < 3; ++kw) {
      const int o = 2 * j + kw - P - 2;
      if (o < 0 || o >= 8) continue;
      dw_fma4(acc[o], wk[kw], x);
    }
  }
}

// 3x3 filters in tiles 8 pixels wide (the forward pass at stride S, the
// input gradient at stride S): a thread takes one output row of the tile for
// one (channel, batch quad) lane, keeps its nine weights and the row's 8 x 4
// sums in registers, and streams the staged source columns of each kernel
// row once, adding each into every output that reads it.  An output still
// sees its taps in (kh, kw) order: the forward pass walks the columns left
// to right, the input gradient right to left (at stride 1 a correlation
// with the flipped filter; at stride 2 a G_X row takes kernel rows kh with
// oh + p - kh even, from G_Y row (oh + p - kh) / 2).  PIX: the staged
// pixel's bf16 count (channels x batch) when it is one of the common values,
// so that every shared-memory offset is a constant; 0 for any other.
template <bool DGRAD, int S, int PIX>
__device__ __forceinline__ void dw_tile_rows3(const DwTile& t, int N, int p, int r0, int oh0, int ow0,
                                              const float* wsh, const uint16_t* xs, float* out,
                                              int64_t out_pix_stride, int pix_rt) {
  constexpr int TW = 8, NC = 7 * S + 3;
  constexpr int IW = DGRAD ? (S == 1 ? 10 : 6) : NC;   // staged columns (t.iw)
  const int pix_elems = PIX ? PIX : pix_rt;
  const int nq = N >> 2, lanes = t.cg * nq;
  for (int u = threadIdx.x; u < t.th * lanes; u += kDwThreads) {
    const int oy = u / lanes, lane = u - oy * lanes;
    const int c = lane / nq, q = lane - c * nq;
    const int oh = oh0 + oy;
    if (oh >= t.out_h) continue;
    float wr[9];
#pragma unroll
    for (int k = 0; k < 9; ++k) wr[k] = wsh[c * 9 + k];
    float acc[TW][4];
#pragma unroll
    for (int o = 0; o < TW; ++o)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[o][j] = 0.0f;
    const uint16_t* xl = xs + c * N + 4 * q;
    if constexpr (DGRAD && S == 2) {
      for (int kh = 0; kh < 3; ++kh) {
        const int tpos = oh + p - kh;
        if (tpos & 1) continue;
        const uint16_t* rp = xl + ((tpos - 2 * r0) >> 1) * IW * pix_elems;
        if (p & 1)
          dw_dgrad2_row<1, PIX>(rp, pix_elems, wr + 3 * kh, acc);
        else
          dw_dgrad2_row<0, PIX>(rp, pix_elems, wr + 3 * kh, acc);
      }
    } else {
#pragma unroll
    for (int kh = 0; kh < 3; ++kh) {
      const int row = DGRAD ? oy + 2 - kh : oy * S + kh;
      const uint16_t* rp = xl + row * IW * pix_elems;
#pragma unroll
      for (int jj = 0; jj < NC; ++jj) {
        const int j = DGRAD ? NC - 1 - jj : jj;
        const uint2 v = *reinterpret_cast<const uint2*>(rp + j * pix_elems);
        const float x[4] = {__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xFFFF0000u),
                            __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xFFFF0000u)};
#pragma unroll
        for (int kw = 0; kw < 3; ++kw) {
          // the output that reads column j through tap kw
          const int o = DGRAD ? j + kw - 2 : (j - kw) / S;
          if (DGRAD ? (o < 0 || o >= TW) : (j < kw || (j - kw) % S || o >= TW)) continue;
          dw_fma4(acc[o], wr[kh * 3 + kw], x);
        }
      }
    }
    }
    float* orow = out + (static_cast<int64_t>(oh) * t.out_w + ow0) * out_pix_stride + c * N + 4 * q;
#pragma unroll
    for (int o = 0; o < TW; ++o)
      if (ow0 + o < t.out_w)
        *reinterpret_cast<float4*>(orow + o * out_pix_stride) = make_float4(acc[o][0], acc[o][1], acc[o][2], acc[o][3]);
  }
}

template <bool DGRAD, int S, bool ROWS3, int PIX = 0>
__global__ void __launch_bounds__(kDwThreads, 4)
dw_tile_kernel(const DwGeom g, const DwTile t, const uint16_t* __restrict__ w, const uint16_t* __restrict__ src,
               float* __restrict__ out) {
  extern __shared__ __align__(16) unsigned char dw_smem[];
  const int C = static_cast<int>(g.C), N = static_cast<int>(g.N);
  const int Kh = static_cast<int>(g.Kh), Kw = static_cast<int>(g.Kw), p = static_cast<int>(g.pad);
  const int s = S ? S : static_cast<int>(g.stride);
  const int bw = blockIdx.x % t.tiles_w;
  const int r = blockIdx.x / t.tiles_w;
  const int bh = r % t.tiles_h, cgi = r / t.tiles_h;
  const int oh0 = bh * t.th, ow0 = bw * t.tw, c0 = cgi * t.cg;
  const int r0 = DGRAD ? dw_floordiv(oh0 + p - Kh + 1, s) : oh0 * s - p;
  const int q0 = DGRAD ? dw_floordiv(ow0 + p - Kw + 1, s) : ow0 * s - p;
  const int pix_elems = PIX ? PIX : t.cg * N;     // bf16 per staged pixel
  float* wsh = reinterpret_cast<float*>(dw_smem);
  uint16_t* xs = reinterpret_cast<uint16_t*>(dw_smem + ((t.cg * Kh * Kw * 4 + 15) & ~15));
  dw_stage(xs, src, r0, q0, t.ih, t.iw, t.src_h, t.src_w, C, N, c0, pix_elems, t.vec16);
  asm volatile("cp.async.commit_group;\n" ::: "memory");
  for (int e = threadIdx.x; e < t.cg * Kh * Kw; e += kDwThreads) wsh[e] = dw_bf16(w[c0 * Kh * Kw + e]);
  asm volatile("cp.async.wait_all;\n" ::: "memory");
  __syncthreads();
  if constexpr (ROWS3) {
    dw_tile_rows3<DGRAD, S, PIX>(t, N, p, r0, oh0, ow0, wsh, xs, out + static_cast<int64_t>(c0) * N, static_cast<int64_t>(C) * N,
                            pix_elems);
    return;
  }
  const int nq = N >> 2, lanes = t.cg * nq;       // lanes <= kDwThreads (host-checked)
  const int pstep = kDwThreads / lanes;
  if (threadIdx.x >= pstep * lanes) return;
  const int lane = threadIdx.x % lanes, c = lane / nq, q = lane - c * nq;
  const float* wc = wsh + c * Kh * Kw;
  const uint16_t* xl = xs + c * N + 4 * q;
  float* ol = out + static_cast<int64_t>(c0 + c) * N + 4 * q;
  for (int pix = threadIdx.x / lanes; pix < t.th * t.tw; pix += pstep) {
    const int oy = pix / t.tw, ox = pix - oy * t.tw;
    const int oh = oh0 + oy, ow = ow0 + ox;
    if (oh >= t.out_h || ow >= t.out_w) continue;
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    for (int kh = 0; kh < Kh; ++kh) {
      int row;
      if (DGRAD) {
        const int rel = oh + p - kh - r0 * s;     // >= 0 inside the window
        if (S != 1 && rel % s) continue;
        row = rel / s;
      } else {
        row = oy * s + kh;
      }
      for (int kw = 0; kw < Kw; ++kw) {
        int col;
        if (DGRAD) {
          const int rel = ow + p - kw - q0 * s;
          if (S != 1 && rel % s) continue;
          col = rel / s;
        } else {
          col = ox * s + kw;
        }
        const float wv = wc[kh * Kw + kw];
        const uint2 v = *reinterpret_cast<const uint2*>(xl + (row * t.iw + col) * pix_elems);
        acc[0] = __fmaf_rn(wv, __uint_as_float(v.x << 16), acc[0]);
        acc[1] = __fmaf_rn(wv, __uint_as_float(v.x & 0xFFFF0000u), acc[1]);
        acc[2] = __fmaf_rn(wv, __uint_as_float(v.y << 16), acc[2]);
        acc[3] = __fmaf_rn(wv, __uint_as_float(v.y & 0xFFFF0000u), acc[3]);
      }
    }
    *reinterpret_cast<float4*>(ol + (static_cast<int64_t>(oh) * t.out_w + ow) * C * N) =
        make_float4(acc[0], acc[1], acc[2], acc[3]);
  }
}

// Weight gradient of 3x3 filters at stride S in the same tiles: a CTA stages
// the G_Y tile (TH x 8 pixels of CG channels, zeros past the output) and the
// x window it meets, and writes the tile's sums of G_Y·x for its CG x 9
// weights to partial[tile][c][kh][kw] (tile = bh·tiles_w + bw).  A thread
// has a fixed (channel, batch quad) lane and takes the tile's rows
// r, r + 256 / lanes, ...: it keeps the row's 8 x 4 G_Y values and nine sums
// in registers and streams each kernel row's x columns once (each product of
// a G_Y pixel and an x pixel added over the four batch items in order).  The
// CTA then adds the threads' sums of each weight in a fixed order (row group,
// then batch quad), and dw_wgrad_tile_reduce adds the tiles' in order.
template <int S, int PIX = 0>
__global__ void __launch_bounds__(kDwThreads, 4)
dw_wgrad_tile_kernel(const DwGeom g, const DwTile t, const uint16_t* __restrict__ gy,
                     const uint16_t* __restrict__ x, float* __restrict__ partial) {
  extern __shared__ __align__(16) unsigned char dw_smem[];
  constexpr int TW = 8, NC = 7 * S + 3;          // NC = t.iw
  const int C = static_cast<int>(g.C), N = static_cast<int>(g.N), p = static_cast<int>(g.pad);
  const int bw = blockIdx.x % t.tiles_w;
  const int r = blockIdx.x / t.tiles_w;
  const int bh = r % t.tiles_h, cgi = r / t.tiles_h;
  const int oh0 = bh * t.th, ow0 = bw * TW, c0 = cgi * t.cg;
  const int pix_elems = PIX ? PIX : t.cg * N;
  uint16_t* xs = reinterpret_cast<uint16_t*>(dw_smem);
  uint16_t* gs = xs + t.ih * t.iw * pix_elems;
  float* red = reinterpret_cast<float*>(dw_smem + ((t.ih * t.iw + t.th * TW) * pix_elems * 2 + 15) / 16 * 16);
  dw_stage(xs, x, oh0 * S - p, ow0 * S - p, t.ih, t.iw, t.src_h, t.src_w, C, N, c0, pix_elems, t.vec16);
  dw_stage(gs, gy, oh0, ow0, t.th, TW, t.out_h, t.out_w, C, N, c0, pix_elems, t.vec16);
  asm volatile("cp.async.commit_group;\n" ::: "memory");
  asm volatile("cp.async.wait_all;\n" ::: "memory");
  __syncthreads();
  const int nq = N >> 2, lanes = t.cg * nq;       // lanes divides kDwThreads (host-checked)
  const int pstep = kDwThreads / lanes;
  const int lane = threadIdx.x % lanes, c = lane / nq, q = lane - c * nq;
  float acc[9];
#pragma unroll
  for (int k = 0; k < 9; ++k) acc[k] = 0.0f;
  for (int oy = threadIdx.x / lanes; oy < t.th && oh0 + oy < t.out_h; oy += pstep) {
    float gv[TW][4];
    const uint16_t* grow = gs + oy * TW * pix_elems + c * N + 4 * q;
#pragma unroll
    for (int o = 0; o < TW; ++o) {
      const uint2 v = *reinterpret_cast<const uint2*>(grow + o * pix_elems);
      gv[o][0] = __uint_as_float(v.x << 16);
      gv[o][1] = __uint_as_float(v.x & 0xFFFF0000u);
      gv[o][2] = __uint_as_float(v.y << 16);
      gv[o][3] = __uint_as_float(v.y & 0xFFFF0000u);
    }
#pragma unroll
    for (int kh = 0; kh < 3; ++kh) {
      const uint16_t* rp = xs + (oy * S + kh) * NC * pix_elems + c * N + 4 * q;
#pragma unroll
      for (int j = 0; j < NC; ++j) {
        const uint2 v = *reinterpret_cast<const uint2*>(rp + j * pix_elems);
        const float xv[4] = {__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xFFFF0000u),
                             __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xFFFF0000u)};
#pragma unroll
        for (int kw = 0; kw < 3; ++kw) {
          const int o = (j - kw) / S;
          if (j < kw || (j - kw) % S || o >= TW) continue;
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[kh * 3 + kw] = __fmaf_rn(gv[o][e], xv[e], acc[kh * 3 + kw]);
        }
      }
    }
  }
#pragma unroll
  for (int k = 0; k < 9; ++k) red[threadIdx.x * 9 + k] = acc[k];
  __syncthreads();
  const int tile = bh * t.tiles_w + bw;
  for (int e = threadIdx.x; e < t.cg * 9; e += kDwThreads) {
    const int cc = e / 9, k = e - cc * 9;
    float sum = 0.0f;
    for (int rr = 0; rr < pstep; ++rr)
      for (int qq = 0; qq < nq; ++qq) sum += red[(rr * lanes + cc * nq + qq) * 9 + k];
    partial[(static_cast<int64_t>(tile) * C + c0 + cc) * 9 + k] = sum;
  }
}

// gw[i] = the tiles' partial sums of weight i added in tile order: one warp
// per weight, lane l adding tiles l, l + 32, ... in order, then the 32 lane
// sums in a fixed tree.
__global__ void __launch_bounds__(kDwThreads)
dw_wgrad_tile_reduce(int64_t parts, int64_t per, const float* __restrict__ partial, float* __restrict__ gw) {
  const int64_t i = (static_cast<int64_t>(blockIdx.x) * kDwThreads + threadIdx.x) / 32;
  const int l = threadIdx.x & 31;
  if (i >= per) return;                           // whole warps leave together
  float s = 0.0f;
  for (int64_t pt = l; pt < parts; pt += 32) s += partial[pt * per + i];
#pragma unroll
  for (int d = 16; d >= 1; d >>= 1) s += __shfl_down_sync(0xFFFFFFFFu, s, d);
  if (l == 0) gw[i] = s;
}

}  // namespace mqv
