// C ABI of the MicroQonv hot path (declared in include/mqv.h): argument
// validation, launch geometry and error reporting.  Every compute step runs
// in the kernels of mqv_quantize.cuh and mqv_conv_kernels.cuh; this file only checks
// arguments and enqueues launches on the caller's stream.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "mqv.h"
#include "mqv_conv_common.cuh"
#include "mqv_conv_kernels.cuh"
#include "mqv_conv_halo.cuh"
#include "mqv_conv_nvf4.cuh"
#include "mqv_conv_wgk.cuh"
#include "mqv_conv_narrow.cuh"
#include "mqv_depthwise.cuh"
#include "mqv_naive.cuh"
#include "mqv_quantize.cuh"
#include "mqv_replay.cuh"

namespace {

using namespace mqv;

thread_local char g_msg[512] = "";

mqv_status fail(mqv_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return st;
}

mqv_status ok() {
  g_msg[0] = '\0';
  return MQV_OK;
}

mqv_status cuda_fail(cudaError_t e, const char* what) {
  return fail(MQV_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Device word that bounded waits set on timeout (see mqv_ptx.cuh).
__device__ uint32_t g_device_error;

constexpr int kMaxDevices = 64;
uint32_t* g_err_ptr[kMaxDevices] = {};
std::mutex g_err_mu;

mqv_status device_error_word(uint32_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(MQV_ERR_UNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lk(g_err_mu);
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_device_error);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(error word)");
    g_err_ptr[dev] = static_cast<uint32_t*>(p);
  }
  *out = g_err_ptr[dev];
  return MQV_OK;
}

// ------------------------------------------------------------ quantize geometry

constexpr int64_t kMaxAmaxCtas = 148 * 4;
constexpr int64_t kMaxQuantCtas = 148 * 16;

// One partial maximum per amax CTA; every quantize CTA reduces them before it
// can scale anything, so keep them few (at most four CTAs per SM, 128 KB of
// loads in flight per SM: two per SM leave large tensors about 5% short of
// the copy rate) and give every CTA the same number of kAmaxThreads x
// 8-float4 chunks.
int64_t amax_ctas(int64_t rows, int64_t cols) {
  const int64_t n4 = rows * cols / 4;
  const int64_t chunk = kAmaxThreads * 8;
  const int64_t nchunks = n4 > 0 ? (n4 + chunk - 1) / chunk : 1;
  const int64_t passes = (nchunks + kMaxAmaxCtas - 1) / kMaxAmaxCtas;
  return (nchunks + passes - 1) / passes;
}

int64_t quant_ctas(int64_t rows, int64_t cols, int32_t blocks = MQV_BLOCKS_4X4) {
  // one thread per 16 elements; 16 x 1 line blocks take four blocks a thread
  const int64_t nb = rows * cols / (blocks == MQV_BLOCKS_16X1 ? 64 : 16);
  const int64_t per_cta = static_cast<int64_t>(kQuantThreads) * kQuantUnits;
  int64_t g = (nb + per_cta - 1) / per_cta;
  if (g < 1) g = 1;
  return g < kMaxQuantCtas ? g : kMaxQuantCtas;
}

FastDiv make_fastdiv(int64_t d) {
  FastDiv f;
  uint32_t s = 0;
  while ((int64_t(1) << s) < d) ++s;
  const unsigned __int128 num = (static_cast<unsigned __int128>(1) << (32 + s)) + (d - 1);
  f.m = static_cast<uint32_t>(static_cast<uint64_t>(num / static_cast<unsigned __int128>(d)) - (uint64_t(1) << 32));
  f.s = s;
  return f;
}

mqv_status check_view(int64_t rows, int64_t cols) {
  if (rows <= 0 || cols <= 0 || rows % 4 || cols % 4)
    return fail(MQV_ERR_INVALID_ARG, "view %lld x %lld: rows and cols must be positive multiples of 4",
                (long long)rows, (long long)cols);
  if (rows > (int64_t(1) << 34) / cols)     // quantize work units (4 x 4 blocks) stay below 2^30
    return fail(MQV_ERR_UNSUPPORTED, "view %lld x %lld too large", (long long)rows, (long long)cols);
  return MQV_OK;
}

mqv_status check_fmt(int32_t fmt) {
  if (fmt != MQV_NVFP4 && fmt != MQV_NVFP6) return fail(MQV_ERR_INVALID_ARG, "unknown format %d", fmt);
  return MQV_OK;
}

mqv_status check_qtensor(const mqv_qtensor* q, const char* name) {
  if (!q) return fail(MQV_ERR_INVALID_ARG, "%s: null descriptor", name);
  mqv_status st = check_view(q->rows, q->cols);
  if (st) return st;
  if ((st = check_fmt(q->fmt))) return st;
  if (q->blocks != MQV_BLOCKS_4X4 && q->blocks != MQV_BLOCKS_1X16 && q->blocks != MQV_BLOCKS_16X1)
    return fail(MQV_ERR_INVALID_ARG, "%s: unknown block shape %d", name, q->blocks);
  if (q->blocks == MQV_BLOCKS_1X16 && q->cols % 16)
    return fail(MQV_ERR_INVALID_ARG, "%s: 1 x 16 blocks need cols a multiple of 16", name);
  if (q->blocks == MQV_BLOCKS_16X1 && q->rows % 16)
    return fail(MQV_ERR_INVALID_ARG, "%s: 16 x 1 blocks need rows a multiple of 16", name);
  if (!q->codes || !q->scales || !q->tscale) return fail(MQV_ERR_INVALID_ARG, "%s: null pointer", name);
  if (!aligned16(q->codes) || !aligned16(q->scales))
    return fail(MQV_ERR_INVALID_ARG, "%s: codes and scales must be 16-byte aligned", name);
  if (reinterpret_cast<uintptr_t>(q->tscale) & 3u)
    return fail(MQV_ERR_INVALID_ARG, "%s: tscale must be 4-byte aligned", name);
  return MQV_OK;
}

// Round keys of Philox4x32-10 for a 64-bit seed (key = low, high word).
PhiloxKeys philox_keys(uint64_t seed) {
  PhiloxKeys k;
  uint32_t k0 = static_cast<uint32_t>(seed), k1 = static_cast<uint32_t>(seed >> 32);
  for (int r = 0; r < 10; ++r) {
    k.k0[r] = k0;
    k.k1[r] = k1;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return k;
}

QuantArgs make_quant_args(const float* src, int64_t rows, int64_t cols, uint64_t seed, int64_t sr_cols,
                          int64_t sr_col0, const mqv_qtensor* out) {
  QuantArgs qa;
  qa.src = src;
  qa.rows = rows;
  qa.cols = cols;
  qa.codes = static_cast<uint8_t*>(out->codes);
  qa.scales = out->scales;
  qa.tscale = out->tscale;
  qa.keys = philox_keys(seed);
  qa.sr_cols = sr_cols;
  qa.sr_col0 = sr_col0;
  qa.dcb = make_fastdiv(cols / 4);
  qa.blocks = out->blocks;
  return qa;
}

template <int FMT, int RND>
void launch_quantize(const QuantArgs& qa, const float* amax_src, int amax_count, cudaStream_t st) {
  const unsigned g = (unsigned)quant_ctas(qa.rows, qa.cols);
  quantize_kernel<FMT, RND><<<g, kQuantThreads, 0, st>>>(qa, amax_src, amax_count);
}

mqv_status enqueue_quantize(const float* src, int64_t rows, int64_t cols, int32_t fmt,
                            int32_t rounding, uint64_t seed, const float* amax_src,
                            int amax_count, int64_t sr_cols, int64_t sr_col0,
                            const mqv_qtensor* out, cudaStream_t st) {
  const QuantArgs qa = make_quant_args(src, rows, cols, seed, sr_cols, sr_col0, out);
  if (fmt == MQV_NVFP4)
    rounding == MQV_RNE ? launch_quantize<0, 0>(qa, amax_src, amax_count, st)
                        : launch_quantize<0, 1>(qa, amax_src, amax_count, st);
  else
    rounding == MQV_RNE ? launch_quantize<1, 0>(qa, amax_src, amax_count, st)
                        : launch_quantize<1, 1>(qa, amax_src, amax_count, st);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "quantize launch");
  return ok();
}

mqv_status check_quantize_args(const float* src, int64_t rows, int64_t cols, int32_t fmt,
                               int32_t rounding, const mqv_qtensor* out, bool line_blocks = false) {
  mqv_status st = check_view(rows, cols);
  if (st) return st;
  if ((st = check_fmt(fmt))) return st;
  if (rounding != MQV_RNE && rounding != MQV_SR)
    return fail(MQV_ERR_INVALID_ARG, "unknown rounding %d", rounding);
  if (!src || !aligned16(src)) return fail(MQV_ERR_INVALID_ARG, "src must be a 16-byte aligned pointer");
  if ((st = check_qtensor(out, "out"))) return st;
  if (out->rows != rows || out->cols != cols || out->fmt != fmt)
    return fail(MQV_ERR_INVALID_ARG, "out describes a %lld x %lld fmt %d view, expected %lld x %lld fmt %d",
                (long long)out->rows, (long long)out->cols, out->fmt, (long long)rows,
                (long long)cols, fmt);
  if (!line_blocks && out->blocks != MQV_BLOCKS_4X4)
    return fail(MQV_ERR_UNSUPPORTED, "out: this entry point writes 4 x 4 blocks only");
  return MQV_OK;
}

// ------------------------------------------------------------- conv geometry

struct ConvPlan {
  V2Args a;
  bool halo;            // stride-1 fwd/dgrad with the on-chip halo (conv_halo_kernel)
  HaloGeom g;
  bool wgk;             // stride-1 wgrad with the taps of a kernel row sharing operands
  WgkGeom wg;
  bool narrow;          // dgrad of a 4-channel stem on CUDA cores (conv_narrow_dgrad_kernel)
  bool tr;              // generic fwd/dgrad on transposed tiles (M <= 128)
  int bn;               // 128 or 256 columns per tile
  int nu;               // batch items per producer unit: 8, or 4 when N % 8 != 0
  int grid;             // persistent CTAs
  size_t image_bytes;   // fwd/dgrad: dequantized A image (workspace head)
  size_t partial_bytes; // wgrad: split partials (workspace)
  size_t ws_bytes;
};

constexpr int kSMs = 148;

mqv_status check_desc(const mqv_conv_desc* d) {
  if (!d) return fail(MQV_ERR_INVALID_ARG, "null conv descriptor");
  if (d->reserved) return fail(MQV_ERR_INVALID_ARG, "conv descriptor reserved field must be 0");
  if (d->N <= 0 || d->Cin <= 0 || d->Cout <= 0 || d->H <= 0 || d->W <= 0 || d->Kh <= 0 ||
      d->Kw <= 0 || d->stride <= 0 || d->pad < 0)
    return fail(MQV_ERR_INVALID_ARG, "conv shape fields must be positive (pad >= 0)");
  if (d->N % 4 || d->Cin % 4 || d->Cout % 4)
    return fail(MQV_ERR_INVALID_ARG, "N, Cin and Cout must be multiples of 4 (4 x 4 square blocks)");
  if (d->pad >= d->Kh || d->pad >= d->Kw)
    return fail(MQV_ERR_INVALID_ARG, "pad must be smaller than the kernel size");
  mqv_status st = check_fmt(d->fmt);
  if (st) return st;
  const int64_t Ho = (d->H + 2 * d->pad - d->Kh) / d->stride + 1;
  const int64_t Wo = (d->W + 2 * d->pad - d->Kw) / d->stride + 1;
  if (d->H + 2 * d->pad < d->Kh || d->W + 2 * d->pad < d->Kw || Ho <= 0 || Wo <= 0)
    return fail(MQV_ERR_INVALID_ARG, "kernel larger than the padded input");
  const int64_t lim = int64_t(1) << 30;
  if (d->H * d->W > lim || d->Cin > 65536 || d->Cout > 65536 || d->N > 65536 || d->Kh > 64 ||
      d->Kw > 64 || d->H * d->W * d->Cin * d->N > (int64_t(1) << 36) ||
      Ho * Wo * d->Cout * d->N > (int64_t(1) << 36) || Ho * Wo * d->N >= (int64_t(1) << 31) ||
      d->H * d->W * d->N >= (int64_t(1) << 31) || d->Kh * d->Kw * (d->Cin + d->Cout) >= (int64_t(1) << 31))
    return fail(MQV_ERR_UNSUPPORTED, "conv shape exceeds the supported range");
  return MQV_OK;
}

QView make_view(const mqv_qtensor* q) {
  QView v;
  v.codes = static_cast<const uint8_t*>(q->codes);
  v.scales = q->scales;
  v.tscale = q->tscale;
  v.row_bytes = q->fmt == MQV_NVFP4 ? q->cols / 2 : q->cols * 3 / 4;
  v.blocks = q->blocks;
  v.scale_cols = q->blocks == MQV_BLOCKS_1X16 ? q->cols / 16 : q->blocks == MQV_BLOCKS_16X1 ? q->cols : q->cols / 4;
  return v;
}

// Multiplier and shift of mqv::fdiv for divisor d >= 1.

// Geometry of one pass (no pointers needed for sizing).
void plan_conv(const mqv_conv_desc* d, int op, ConvPlan* pl) {
  V2Args& a = pl->a;
  std::memset(&a, 0, sizeof(a));
  a.N = (int)d->N; a.Cin = (int)d->Cin; a.Cout = (int)d->Cout; a.H = (int)d->H; a.W = (int)d->W;
  a.Kh = (int)d->Kh; a.Kw = (int)d->Kw; a.stride = (int)d->stride; a.pad = (int)d->pad;
  a.Ho = (int)((d->H + 2 * d->pad - d->Kh) / d->stride + 1);
  a.Wo = (int)((d->W + 2 * d->pad - d->Kw) / d->stride + 1);
  const int64_t taps = d->Kh * d->Kw;
  if (op == MQV_OP_FWD) {
    a.M = a.Cout; a.Cred = a.Cin;
    a.Ncols = (int64_t)a.Ho * a.Wo * a.N;
    a.Kdim = taps * a.Cin;
  } else if (op == MQV_OP_WGRAD) {
    a.M = a.Cout; a.Cred = a.Cin;
    a.Ncols = taps * a.Cin;
    a.Kdim = (int64_t)a.Ho * a.Wo * a.N;
  } else {
    a.M = a.Cin; a.Cred = a.Cout;
    a.Ncols = (int64_t)a.H * a.W * a.N;
    a.Kdim = taps * a.Cout;
  }
  a.ktiles = (int)((a.Kdim + 63) / 64);
  a.mtiles = (int)((a.M + 127) / 128);
  a.dN = make_fastdiv(a.N);
  a.dWo = make_fastdiv(a.Wo);
  a.dW = make_fastdiv(a.W);
  a.dCred = make_fastdiv(a.Cred);
  a.dKw = make_fastdiv(a.Kw);
  a.dCin = make_fastdiv(a.Cin);
  a.dS = make_fastdiv(a.stride);
  pl->nu = (d->N % 8 == 0) ? 8 : 4;
  // Generic fwd/dgrad with at most 128 output channels: transposed tiles,
  // 128 GEMM columns x the channels rounded up to 16, so the MMA does no
  // work on absent channels and every column's channels are stored by one
  // lane.
  pl->tr = op != MQV_OP_WGRAD && a.M <= 128;
  a.nc = pl->tr ? (a.M + 15) / 16 * 16 : 0;
  // Columns per tile: the option with the smaller (waves x tile width) over
  // one persistent CTA per SM; ties go to the wider tile.
  auto waves = [&](int bn) { return ((a.Ncols + bn - 1) / bn * a.mtiles + kSMs - 1) / kSMs; };
  pl->bn = pl->tr ? 128 : (waves(256) * 256 <= waves(128) * 128 ? 256 : 128);
  a.ntiles = (int)((a.Ncols + pl->bn - 1) / pl->bn);
  a.phases = 1;
  a.ph_tile0[0] = 0;
  a.ph_tile0[1] = a.ntiles;
  a.ph_cols[0] = a.Ncols;
  a.ph_nlive[0] = a.ktiles;
  if (op == MQV_OP_DGRAD && d->stride == 2 && a.ktiles <= kMaxLiveWords * 32 && a.Cred >= 32) {
    // Stride-2 input gradient: group the columns by (hi mod 2, wi mod 2); a
    // K tile is live for a phase when one of its taps (kh, kw) satisfies
    // hi + pad - kh = 0 and wi + pad - kw = 0 (mod 2).  With fewer than 32
    // reduction channels a K tile spans four or more taps, most stay live,
    // and the grouping measured slower (16 channels: 0.52 -> 0.71 ms on the
    // 640 px stem), so it is kept to 32 and more.
    a.phases = kMaxPhases;
    int t0 = 0;
    for (int q = 0; q < kMaxPhases; ++q) {
      const int ph = q >> 1, pw = q & 1;
      const int hp = a.H > ph ? (a.H - ph + 1) / 2 : 0;
      const int wp = a.W > pw ? (a.W - pw + 1) / 2 : 0;
      a.ph_h0[q] = ph;
      a.ph_w0[q] = pw;
      a.ph_wp[q] = wp;
      a.ph_dwp[q] = make_fastdiv(wp > 0 ? wp : 1);
      a.ph_cols[q] = (int64_t)hp * wp * a.N;
      a.ph_tile0[q] = t0;
      t0 += (int)((a.ph_cols[q] + pl->bn - 1) / pl->bn);
      int nlive = 0;
      for (int kt = 0; kt < a.ktiles; ++kt) {
        const int64_t k0 = (int64_t)kt * 64, k1 = std::min<int64_t>(k0 + 63, a.Kdim - 1);
        bool live = false;
        for (int64_t tap = k0 / a.Cred; tap <= k1 / a.Cred && !live; ++tap) {
          const int kh = (int)(tap / a.Kw), kw = (int)(tap % a.Kw);
          live = ((ph + a.pad - kh) & 1) == 0 && ((pw + a.pad - kw) & 1) == 0;
        }
        if (live) {
          a.ph_live[q][kt >> 5] |= 1u << (kt & 31);
          ++nlive;
        }
      }
      a.ph_nlive[q] = nlive;
    }
    a.ph_tile0[kMaxPhases] = t0;
    a.ntiles = t0;
  }
  const int64_t tiles_mn = (int64_t)a.ntiles * a.mtiles;
  int splits = 1;
  if (op == MQV_OP_WGRAD) {
    // split the (ho, wo, n) contraction so that all tiles fit one wave
    int64_t s = tiles_mn >= kSMs ? 1 : kSMs / tiles_mn;
    if (s > a.ktiles) s = a.ktiles;
    if (s < 1) s = 1;
    const int64_t per = (a.ktiles + s - 1) / s;
    splits = (int)((a.ktiles + per - 1) / per);
    a.kt_per_split = (int)per;
  } else {
    a.kt_per_split = a.ktiles;
  }
  a.splits = splits;
  a.tiles = (int)(tiles_mn * splits);
  // Stride-1 fwd/dgrad (NVFP4 or NVFP6) with N | 256, N % 8 == 0, a halo of at most
  // 384 rows and whole 64-channel chunks: the kernel-row halo path.
  pl->halo = op != MQV_OP_WGRAD && d->stride == 1 && d->N % 8 == 0 &&
             256 % d->N == 0 && (d->Kw - 1) * d->N <= 128 && a.Cred % 64 == 0 && d->Kw <= kHaloAStages;
  if (pl->halo) {
    HaloGeom& g = pl->g;
    g.out_h = op == MQV_OP_FWD ? a.Ho : a.H;
    g.out_w = op == MQV_OP_FWD ? a.Wo : a.W;
    g.src_h = op == MQV_OP_FWD ? a.H : a.Ho;
    g.src_w = op == MQV_OP_FWD ? a.W : a.Wo;
    g.cchunks = a.Cred / 64;
    // Tile width: the persistent CTAs run ceil(tiles / SMs) tiles, each
    // stage costing the longer of its MMAs (about BN/2 cycles per 16-deep
    // slice and tap, at least the N = 128 cost) and its producers (about 6
    // cycles per halo row); pick the width with the least total, ties to
    // the wider tile.
    int best_bw = 0;
    int64_t best_cost = 0;
    for (int bw = (int)(256 / d->N); bw >= 1; --bw) {
      const int bn = bw * (int)d->N;
      if (bn % 16) continue;
      const int64_t tiles = (int64_t)a.mtiles * g.out_h * ((g.out_w + bw - 1) / bw);
      const int64_t waves = (tiles + kSMs - 1) / kSMs;
      const int64_t mma = (int64_t)d->Kw * 4 * ((bn > 128 ? bn : 128) / 2);
      const int64_t prod = 6 * (int64_t)(bw + d->Kw - 1) * d->N;
      const int64_t cost = waves * (mma > prod ? mma : prod);
      if (best_bw == 0 || cost < best_cost) {
        best_bw = bw;
        best_cost = cost;
      }
    }
    g.bw = best_bw;
    g.bn = g.bw * (int)d->N;
    g.rows = (int)((g.bw + d->Kw - 1) * d->N);
    g.tpr = (g.out_w + g.bw - 1) / g.bw;
    a.tiles = a.mtiles * g.out_h * g.tpr;
  }
  // Stride-1 weight gradient with N % 16 == 0 and Kw <= 3 whose taps reach
  // at most two 64-element chunks further: the kernel-row path.
  pl->wgk = op == MQV_OP_WGRAD && d->stride == 1 && d->N % 16 == 0 && d->Kw <= kWgkMaxTaps &&
            (48 + (d->Kw - 1) * d->N) / 64 <= 2;
  if (pl->wgk) {
    WgkGeom& w = pl->wg;
    w.chunks = (int)((a.Wo * d->N + 63) / 64);
    w.sx = (int)((48 + (d->Kw - 1) * d->N) / 64);
    w.ctiles = (a.Cin + 127) / 128;
    w.base_tiles = a.mtiles * w.ctiles * a.Kh;
    const int64_t total_q = (int64_t)a.Ho * w.chunks;
    int64_t s = w.base_tiles >= kSMs ? 1 : kSMs / w.base_tiles;
    if (s > total_q) s = total_q;
    const int64_t per = (total_q + s - 1) / s;
    w.q_per_split = (int)per;
    splits = (int)((total_q + per - 1) / per);
    a.splits = splits;
    a.tiles = w.base_tiles * splits;
  }
  a.scale_out = splits == 1;
  // persistent kernels: one CTA per SM at most; the kernel-row weight
  // gradient runs one tile per CTA
  pl->grid = pl->wgk ? a.tiles : (a.tiles < kSMs ? a.tiles : kSMs);
  // Input gradient of a 4-input-channel layer (a stem) with N % 16 == 0:
  // bound by memory (Cout products per element and tap), so it runs on CUDA
  // cores without a weight image (conv_narrow_dgrad_kernel).
  pl->narrow = op == MQV_OP_DGRAD && !pl->halo && d->Cin == 4 && d->N % 16 == 0 &&
               d->Cout * d->Kh * d->Kw * 4 * (int64_t)sizeof(float) <= kNarrowMaxWeightBytes;
  if (pl->narrow) {
    const int64_t units = d->H * d->W * (d->N / 16);
    const int64_t g = (units + kNarrowThreads - 1) / kNarrowThreads;
    pl->grid = (int)(g < 8 * kSMs ? g : 8 * kSMs);
  }
  pl->image_bytes = op == MQV_OP_WGRAD || pl->narrow ? 0 : (size_t)a.mtiles * a.ktiles * kATileBytes;
  pl->partial_bytes = splits > 1 ? (size_t)splits * a.M * a.Ncols * sizeof(float) : 0;
  pl->ws_bytes = pl->image_bytes + pl->partial_bytes;
}

// Opt a kernel into more than 48 KB of dynamic shared memory, once per device.
// `done` must be distinct for every kernel (one static per launcher instance).
template <typename K>
cudaError_t set_smem(K kern, int bytes, bool (&done)[kMaxDevices]) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (!done[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    done[dev] = true;
  }
  return cudaSuccess;
}

template <int PASS, int FMT, int BN, int NU, bool TR, bool PH>
cudaError_t launch_fd_ph(const ConvPlan& pl, cudaStream_t st) {
  // two producer groups where the register budget allows it (transposed
  // tiles with 8-item units)
  constexpr int kGr = TR && NU == 8 ? 2 : 1;
  auto kern = conv_fd_kernel<PASS, FMT, BN, NU, TR, kGr, PH>;
  static bool done[kMaxDevices] = {};
  cudaError_t e = set_smem(kern, V2Smem<BN>::kBytes, done);
  if (e != cudaSuccess) return e;
  kern<<<pl.grid, fd_threads(kGr), V2Smem<BN>::kBytes, st>>>(pl.a);
  return cudaGetLastError();
}

// Stride-2 input gradients run with their columns grouped by phase.
template <int PASS, int FMT, int BN, int NU, bool TR>
cudaError_t launch_fd(const ConvPlan& pl, cudaStream_t st) {
  if (PASS == kDgrad && pl.a.phases > 1) return launch_fd_ph<kDgrad, FMT, BN, NU, TR, true>(pl, st);
  return launch_fd_ph<PASS, FMT, BN, NU, TR, false>(pl, st);
}

template <int FMT, int BN, int NU>
cudaError_t launch_wg(const ConvPlan& pl, cudaStream_t st) {
  auto kern = conv_wg_kernel<FMT, BN, NU>;
  static bool done[kMaxDevices] = {};
  cudaError_t e = set_smem(kern, V2Smem<BN>::kBytes, done);
  if (e != cudaSuccess) return e;
  kern<<<pl.grid, kV2Threads, V2Smem<BN>::kBytes, st>>>(pl.a);
  return cudaGetLastError();
}

template <int PASS, int FMT>
cudaError_t launch_pass(const ConvPlan& pl, cudaStream_t st) {
  if (PASS == kWgrad) {
    if (pl.bn == 256) return pl.nu == 8 ? launch_wg<FMT, 256, 8>(pl, st) : launch_wg<FMT, 256, 4>(pl, st);
    return pl.nu == 8 ? launch_wg<FMT, 128, 8>(pl, st) : launch_wg<FMT, 128, 4>(pl, st);
  }
  constexpr int P = PASS == kWgrad ? kFwd : PASS;
  if (pl.tr) return pl.nu == 8 ? launch_fd<P, FMT, 128, 8, true>(pl, st) : launch_fd<P, FMT, 128, 4, true>(pl, st);
  if (pl.bn == 256)
    return pl.nu == 8 ? launch_fd<P, FMT, 256, 8, false>(pl, st) : launch_fd<P, FMT, 256, 4, false>(pl, st);
  return pl.nu == 8 ? launch_fd<P, FMT, 128, 8, false>(pl, st) : launch_fd<P, FMT, 128, 4, false>(pl, st);
}

// The halo kernel follows its weight-image kernel with programmatic
// dependent launch: its barrier setup, tensor-memory allocation and first
// activation loads overlap the image kernel, and only its weight loader
// waits for the image (pdl_wait_prerequisite).
template <int PASS, int FMT, bool QOUT, bool LINE = false>
cudaError_t launch_halo_q(const ConvPlan& pl, cudaStream_t st) {
  auto kern = conv_halo_kernel<PASS, FMT, QOUT, LINE>;
  static bool done[kMaxDevices] = {};
  cudaError_t e = set_smem(kern, HaloSmem::kBytes, done);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(pl.grid));
  cfg.blockDim = dim3(kHaloThreads);
  cfg.dynamicSmemBytes = HaloSmem::kBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, pl.a, pl.g);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int PASS, int FMT>
cudaError_t launch_halo(const ConvPlan& pl, cudaStream_t st) {
  if (pl.a.b.blocks != MQV_BLOCKS_4X4) return launch_halo_q<PASS, FMT, false, true>(pl, st);
  return pl.a.q_codes ? launch_halo_q<PASS, FMT, true>(pl, st) : launch_halo_q<PASS, FMT, false>(pl, st);
}

template <int FMT, int KW, bool PAIR, bool LINE = false>
cudaError_t launch_wgk(const ConvPlan& pl, cudaStream_t st) {
  auto kern = conv_wgk_kernel<FMT, KW, PAIR, LINE>;
  static bool done[kMaxDevices] = {};
  cudaError_t e = set_smem(kern, WgkSmem::kBytes, done);
  if (e != cudaSuccess) return e;
  kern<<<pl.grid, kWgkThreads, WgkSmem::kBytes, st>>>(pl.a, pl.wg);
  return cudaGetLastError();
}

// Batch 64 puts each tap of a kernel row exactly one X chunk further, so the
// taps share one run of B rows (paired MMAs); other batches use one MMA per tap.
template <int FMT>
cudaError_t launch_wgk_kw(const ConvPlan& pl, cudaStream_t st) {
  const bool pair = pl.a.N == 64;
  if (pl.a.b.blocks != MQV_BLOCKS_4X4) return launch_wgk<FMT, 1, false, true>(pl, st);   // 1 x 1 layers only
  switch (pl.a.Kw) {
    case 1: return launch_wgk<FMT, 1, false>(pl, st);
    case 2: return pair ? launch_wgk<FMT, 2, true>(pl, st) : launch_wgk<FMT, 2, false>(pl, st);
    default: return pair ? launch_wgk<FMT, 3, true>(pl, st) : launch_wgk<FMT, 3, false>(pl, st);
  }
}

template <int PASS>
cudaError_t launch_pass_fmt(int fmt, const ConvPlan& pl, cudaStream_t st) {
  if (PASS != kWgrad && pl.halo)
    return fmt == MQV_NVFP4 ? launch_halo<PASS == kWgrad ? kFwd : PASS, 0>(pl, st)
                            : launch_halo<PASS == kWgrad ? kFwd : PASS, 1>(pl, st);
  if (PASS == kWgrad && pl.wgk) return fmt == MQV_NVFP4 ? launch_wgk_kw<0>(pl, st) : launch_wgk_kw<1>(pl, st);
  return fmt == MQV_NVFP4 ? launch_pass<PASS, 0>(pl, st) : launch_pass<PASS, 1>(pl, st);
}

cudaError_t launch_narrow_dgrad(int fmt, const ConvPlan& pl, const QView& w, cudaStream_t st) {
  const int smem = pl.a.Cout * pl.a.Kh * pl.a.Kw * 4 * (int)sizeof(float);
  if (fmt == MQV_NVFP4) conv_narrow_dgrad_kernel<0><<<pl.grid, kNarrowThreads, smem, st>>>(pl.a, w);
  else conv_narrow_dgrad_kernel<1><<<pl.grid, kNarrowThreads, smem, st>>>(pl.a, w);
  return cudaGetLastError();
}

cudaError_t launch_prep(int op, int fmt, const ConvPlan& pl, const QView& w, uint8_t* image, cudaStream_t st) {
  const V2Args& a = pl.a;
  const int chunks = a.mtiles * 128 * a.ktiles * 8;
  const unsigned g = (unsigned)((chunks + kPrepThreads - 1) / kPrepThreads);
  const FastDiv dkt8 = make_fastdiv((int64_t)a.ktiles * 8), dcout = make_fastdiv(a.Cout);
  const int kd = (int)a.Kdim;
  if (op == MQV_OP_FWD) {
    if (fmt == MQV_NVFP4) prep_image_kernel<0, false><<<g, kPrepThreads, 0, st>>>(w, a.M, kd, a.ktiles, a.mtiles, a.Cin, a.Cout, dkt8, dcout, image);
    else prep_image_kernel<1, false><<<g, kPrepThreads, 0, st>>>(w, a.M, kd, a.ktiles, a.mtiles, a.Cin, a.Cout, dkt8, dcout, image);
  } else {
    if (fmt == MQV_NVFP4) prep_image_kernel<0, true><<<g, kPrepThreads, 0, st>>>(w, a.M, kd, a.ktiles, a.mtiles, a.Cin, a.Cout, dkt8, dcout, image);
    else prep_image_kernel<1, true><<<g, kPrepThreads, 0, st>>>(w, a.M, kd, a.ktiles, a.mtiles, a.Cin, a.Cout, dkt8, dcout, image);
  }
  return cudaGetLastError();
}

// Geometry of the block-scaled forward pass (conv_fwd_nvf4_kernel): halo
// tiles of 128 GEMM columns (128 / N pixels of one output row x N batch
// items) x 128 output channels.
mqv_status plan_blockscaled(const mqv_conv_desc* d, ConvPlan* pl) {
  // N % 64 == 0: a tap shifts the halo rows by N, the scale columns by
  // N / 32, and a scale-factor address in tensor memory must be an even
  // column (an odd one, N = 32, faulted with a misaligned address)
  if (d->fmt != MQV_NVFP4 || d->stride != 1 || d->N % 64 || 128 % d->N || d->Kw > 3 || d->Cin % 64 ||
      (128 / d->N + d->Kw - 1) * d->N > kNvf4MaxRows)
    return fail(MQV_ERR_UNSUPPORTED,
                "block-scaled forward pass: NVFP4, stride 1, N = 64 or 128 with a halo of at most %d rows, "
                "Kw <= 3, Cin a multiple of 64",
                kNvf4MaxRows);
  plan_conv(d, MQV_OP_FWD, pl);
  V2Args& a = pl->a;
  HaloGeom& g = pl->g;
  g.out_h = a.Ho;
  g.out_w = a.Wo;
  g.src_h = a.H;
  g.src_w = a.W;
  g.cchunks = a.Cin / 64;
  g.bw = kNvf4BN / a.N;
  g.bn = kNvf4BN;
  g.rows = (g.bw + a.Kw - 1) * a.N;
  g.tpr = (g.out_w + g.bw - 1) / g.bw;
  a.tiles = a.mtiles * g.out_h * g.tpr;
  pl->grid = a.tiles < kSMs ? a.tiles : kSMs;
  pl->image_bytes = (size_t)a.mtiles * a.ktiles * kNvf4ATile;
  pl->partial_bytes = 0;
  pl->ws_bytes = pl->image_bytes;
  return MQV_OK;
}

mqv_status check_operand(const mqv_qtensor* q, const char* name, int64_t rows, int64_t cols, int32_t fmt) {
  mqv_status st = check_qtensor(q, name);
  if (st) return st;
  if (q->rows != rows || q->cols != cols || q->fmt != fmt)
    return fail(MQV_ERR_INVALID_ARG, "%s: view %lld x %lld fmt %d, expected %lld x %lld fmt %d", name,
                (long long)q->rows, (long long)q->cols, q->fmt, (long long)rows, (long long)cols, fmt);
  return MQV_OK;
}

// Quantized output of a fwd/dgrad pass (see V2Args::q_codes).
struct QuantOut {
  const mqv_qtensor* q;
  const float* t_amax;
  uint64_t seed;
};

mqv_status run_conv(int op, const mqv_conv_desc* d, const mqv_qtensor* qa, const char* na,
                    const mqv_qtensor* qb, const char* nb, float* out, void* ws, size_t ws_bytes,
                    void* stream, int32_t relu = 0, float* amax = nullptr, const QuantOut* qo = nullptr) {
  mqv_status st = check_desc(d);
  if (st) return st;
  const int64_t Ho = (d->H + 2 * d->pad - d->Kh) / d->stride + 1;
  const int64_t Wo = (d->W + 2 * d->pad - d->Kw) / d->stride + 1;
  const int64_t xr = d->H * d->W * d->Cin, wr = d->Cout, wc = d->Kh * d->Kw * d->Cin;
  const int64_t gr = Ho * Wo * d->Cout;
  if (op == MQV_OP_FWD) {
    if ((st = check_operand(qa, na, wr, wc, d->fmt)) || (st = check_operand(qb, nb, xr, d->N, d->fmt))) return st;
  } else if (op == MQV_OP_WGRAD) {
    if ((st = check_operand(qa, na, gr, d->N, d->fmt)) || (st = check_operand(qb, nb, xr, d->N, d->fmt))) return st;
  } else {
    if ((st = check_operand(qa, na, wr, wc, d->fmt)) || (st = check_operand(qb, nb, gr, d->N, d->fmt))) return st;
  }
  if (!qo && (!out || !aligned16(out))) return fail(MQV_ERR_INVALID_ARG, "output must be a 16-byte aligned pointer");
  if (relu != 0 && relu != 1) return fail(MQV_ERR_INVALID_ARG, "relu must be 0 or 1");
  if (amax && (reinterpret_cast<uintptr_t>(amax) & 3u))
    return fail(MQV_ERR_INVALID_ARG, "amax must be a 4-byte aligned pointer");
  ConvPlan pl;
  plan_conv(d, op, &pl);
  if (qa->blocks != MQV_BLOCKS_4X4 || qb->blocks != MQV_BLOCKS_4X4) {
    // the naive scheme's line blocks, on the kernels that run its 1 x 1 GEMMs
    const bool one = d->Kh == 1 && d->Kw == 1 && d->stride == 1 && d->pad == 0;
    const int want_a = op == MQV_OP_DGRAD ? MQV_BLOCKS_16X1 : MQV_BLOCKS_1X16;
    const int want_b = op == MQV_OP_WGRAD ? MQV_BLOCKS_1X16 : MQV_BLOCKS_16X1;
    const bool kern = op == MQV_OP_WGRAD ? pl.wgk : pl.halo;
    if (!one || qa->blocks != want_a || qb->blocks != want_b || !kern || qo)
      return fail(MQV_ERR_UNSUPPORTED,
                  "line blocks: a stride-1 1 x 1 layer of the kernel-row path with %s %s and %s %s, no quantized "
                  "output (got %d and %d)",
                  na, want_a == MQV_BLOCKS_1X16 ? "1 x 16" : "16 x 1", nb, want_b == MQV_BLOCKS_1X16 ? "1 x 16" : "16 x 1",
                  qa->blocks, qb->blocks);
  }
  if (qo) {
    if (!pl.halo)
      return fail(MQV_ERR_UNSUPPORTED, "quantized output: stride-1 layers of the kernel-row path only "
                                       "(N | 256, N %% 8 == 0, reduction channels a multiple of 64)");
    const int64_t rows = op == MQV_OP_FWD ? Ho * Wo * d->Cout : d->H * d->W * d->Cin;
    if ((st = check_operand(qo->q, "quantized output", rows, d->N, d->fmt))) return st;
    if (!qo->t_amax || (reinterpret_cast<uintptr_t>(qo->t_amax) & 3u))
      return fail(MQV_ERR_INVALID_ARG, "t_amax must be a 4-byte aligned device pointer");
    pl.a.q_codes = static_cast<uint8_t*>(qo->q->codes);
    pl.a.q_scales = qo->q->scales;
    pl.a.q_tscale = qo->q->tscale;
    pl.a.q_amax = qo->t_amax;
    pl.a.q_keys = philox_keys(qo->seed);
  }
  if (pl.ws_bytes > 0 && (!ws || ws_bytes < pl.ws_bytes || !aligned16(ws)))
    return fail(MQV_ERR_WORKSPACE, "workspace of %zu bytes (16-byte aligned) required, got %zu",
                pl.ws_bytes, ws ? ws_bytes : (size_t)0);
  uint32_t* err = nullptr;
  if ((st = device_error_word(&err))) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  pl.a.err = err;
  cudaError_t e;
  if (op == MQV_OP_WGRAD) {
    pl.a.a = make_view(qa);
    pl.a.b = make_view(qb);
    pl.a.ta = qa->tscale;
    pl.a.tb = qb->tscale;
    pl.a.out = pl.a.splits > 1 ? reinterpret_cast<float*>(wsb) : out;
    e = launch_pass_fmt<kWgrad>(d->fmt, pl, s);
    if (e != cudaSuccess) return cuda_fail(e, "wgrad launch");
    if (pl.a.splits > 1) {
      const int64_t n4 = (int64_t)pl.a.M * pl.a.Ncols / 4;
      const int64_t g = (n4 + kReduceCols - 1) / kReduceCols;
      // whole 128-byte lines of partials can be dropped from L2 once read
      const int discard = (reinterpret_cast<uintptr_t>(wsb) & 127u) == 0 && n4 % 8 == 0;
      wgrad_reduce_kernel<<<(unsigned)g, kReduceCols * kReduceGroups, 0, s>>>(reinterpret_cast<const float4*>(wsb), pl.a.splits, n4,
                                                       qa->tscale, qb->tscale, reinterpret_cast<float4*>(out),
                                                       discard);
      e = cudaGetLastError();
      if (e != cudaSuccess) return cuda_fail(e, "wgrad reduce launch");
    }
    return ok();
  }
  // fwd / dgrad: qa is W, qb is X (fwd) or G_Y (dgrad)
  if (amax) {
    e = cudaMemsetAsync(amax, 0, sizeof(float), s);
    if (e != cudaSuccess) return cuda_fail(e, "amax clear");
  }
  pl.a.relu = relu;
  pl.a.amax_out = reinterpret_cast<uint32_t*>(amax);
  if (pl.narrow) {
    pl.a.b = make_view(qb);
    pl.a.ta = qa->tscale;
    pl.a.tb = qb->tscale;
    pl.a.out = out;
    e = launch_narrow_dgrad(d->fmt, pl, make_view(qa), s);
    if (e != cudaSuccess) return cuda_fail(e, "narrow dgrad launch");
    return ok();
  }
  e = launch_prep(op, d->fmt, pl, make_view(qa), wsb, s);
  if (e != cudaSuccess) return cuda_fail(e, "operand image launch");
  pl.a.image = wsb;
  pl.a.b = make_view(qb);
  pl.a.ta = qa->tscale;
  pl.a.tb = qb->tscale;
  pl.a.out = out;
  e = op == MQV_OP_FWD ? launch_pass_fmt<kFwd>(d->fmt, pl, s) : launch_pass_fmt<kDgrad>(d->fmt, pl, s);
  if (e != cudaSuccess) return cuda_fail(e, "conv launch");
  return ok();
}

// CTA ranges of every job; pointers are checked only when the plan launches.
static mqv_status plan_quantize_many(const mqv_quantize_job* jobs, int32_t count, QuantJobs* plan,
                                     int* amax_total, int* quant_total, bool check_pointers) {
  if (!jobs || count < 1 || count > kMaxQuantJobs)
    return fail(MQV_ERR_INVALID_ARG, "mqv_quantize_many: 1..%d jobs, got %d", kMaxQuantJobs, count);
  std::memset(plan, 0, sizeof(*plan));
  plan->count = count;
  int a = 0, q = 0;
  for (int i = 0; i < count; ++i) {
    const mqv_quantize_job& j = jobs[i];
    mqv_status st = MQV_OK;
    if (check_pointers) {
      st = check_quantize_args(j.src, j.rows, j.cols, j.fmt, j.rounding, &j.out, true);
      if (!st && (j.out.blocks == MQV_BLOCKS_4X4) != (jobs[0].out.blocks == MQV_BLOCKS_4X4))
        st = fail(MQV_ERR_UNSUPPORTED, "4 x 4 and line blocks mixed in one call");
    } else if (!(st = check_view(j.rows, j.cols)) && !(st = check_fmt(j.fmt)) &&
               j.rounding != MQV_RNE && j.rounding != MQV_SR) {
      st = fail(MQV_ERR_INVALID_ARG, "unknown rounding %d", j.rounding);
    }
    if (st) return fail(st, "job %d: %s", i, std::string(g_msg).c_str());
    QuantJob& qj = plan->job[i];
    qj.qa = make_quant_args(j.src, j.rows, j.cols, j.seed, j.cols, 0, &j.out);
    qj.fmt = j.fmt;
    qj.rounding = j.rounding;
    qj.amax_cta0 = a;
    qj.amax_ctas = (int)amax_ctas(j.rows, j.cols);
    qj.quant_ctas = (int)quant_ctas(j.rows, j.cols, j.out.blocks);
    a += qj.amax_ctas;
  }
  // quantize CTA ranges: stochastic-rounding jobs first (see quantize_many_kernel)
  for (int pass = 0; pass < 2; ++pass)
    for (int i = 0; i < count; ++i)
      if ((plan->job[i].rounding == MQV_SR) == (pass == 0)) {
        plan->job[i].quant_cta0 = q;
        q += plan->job[i].quant_ctas;
      }
  *amax_total = a;
  *quant_total = q;
  return MQV_OK;
}

// The timeout path of the bounded waits, on its own: an mbarrier that
// nothing arrives at (a fresh barrier's phase 0 never completes), waited for
// with mbar_wait_bounded and a caller-given limit.
__global__ void wait_selftest_kernel(uint32_t* err, long long limit) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait_bounded(&bar, 0, err, kErrWaitSelfTest, limit);
}

}  // namespace

extern "C" {

int32_t mqv_version(void) { return 100; }

const char* mqv_last_error(void) { return g_msg; }

mqv_status mqv_qtensor_bytes(int64_t rows, int64_t cols, int32_t fmt, size_t* code_bytes,
                             size_t* scale_bytes) {
  mqv_status st = check_view(rows, cols);
  if (st) return st;
  if ((st = check_fmt(fmt))) return st;
  if (!code_bytes || !scale_bytes) return fail(MQV_ERR_INVALID_ARG, "null output pointer");
  *code_bytes = (size_t)(fmt == MQV_NVFP4 ? rows * cols / 2 : rows * cols * 3 / 4);
  *scale_bytes = (size_t)(rows * cols / 16);
  return ok();
}

mqv_status mqv_quantize_workspace_size(int64_t rows, int64_t cols, size_t* bytes) {
  mqv_status st = check_view(rows, cols);
  if (st) return st;
  if (!bytes) return fail(MQV_ERR_INVALID_ARG, "null output pointer");
  *bytes = (size_t)((amax_ctas(rows, cols) * sizeof(float) + 255) / 256 * 256);
  return ok();
}

mqv_status mqv_amax(const float* src, int64_t rows, int64_t cols, float* amax, void* ws,
                    size_t ws_bytes, void* stream) {
  mqv_status st = check_view(rows, cols);
  if (st) return st;
  if (!src || !aligned16(src)) return fail(MQV_ERR_INVALID_ARG, "src must be a 16-byte aligned pointer");
  if (!amax || (reinterpret_cast<uintptr_t>(amax) & 3u)) return fail(MQV_ERR_INVALID_ARG, "amax must be a 4-byte aligned pointer");
  const int64_t g = amax_ctas(rows, cols);
  if (!ws || ws_bytes < (size_t)g * sizeof(float) || !aligned16(ws))
    return fail(MQV_ERR_WORKSPACE, "workspace of %zu bytes required", (size_t)g * sizeof(float));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* part = static_cast<float*>(ws);
  amax_partial_kernel<<<(unsigned)g, kAmaxThreads, 0, s>>>(reinterpret_cast<const float4*>(src), rows * cols / 4, part);
  amax_finish_kernel<<<1, kAmaxThreads, 0, s>>>(part, (int)g, amax);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "amax launch");
  return ok();
}

mqv_status mqv_quantize_cbf(const float* src, int64_t rows, int64_t cols, int32_t fmt,
                            int32_t rounding, uint64_t seed, const mqv_qtensor* out, void* ws,
                            size_t ws_bytes, void* stream) {
  mqv_status st = check_quantize_args(src, rows, cols, fmt, rounding, out);
  if (st) return st;
  const int64_t g = amax_ctas(rows, cols);
  if (!ws || ws_bytes < (size_t)g * sizeof(float) || !aligned16(ws))
    return fail(MQV_ERR_WORKSPACE, "workspace of %zu bytes required", (size_t)g * sizeof(float));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* part = static_cast<float*>(ws);
  amax_partial_kernel<<<(unsigned)g, kAmaxThreads, 0, s>>>(reinterpret_cast<const float4*>(src), rows * cols / 4, part);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "amax launch");
  return enqueue_quantize(src, rows, cols, fmt, rounding, seed, part, (int)g, cols, 0, out, s);
}

mqv_status mqv_quantize_with_amax(const float* src, int64_t rows, int64_t cols, int32_t fmt,
                                  int32_t rounding, uint64_t seed, const float* amax,
                                  int64_t sr_col0, int64_t sr_cols, const mqv_qtensor* out,
                                  void* stream) {
  mqv_status st = check_quantize_args(src, rows, cols, fmt, rounding, out);
  if (st) return st;
  if (!amax || (reinterpret_cast<uintptr_t>(amax) & 3u)) return fail(MQV_ERR_INVALID_ARG, "amax must be a 4-byte aligned pointer");
  if (sr_cols == 0) sr_cols = cols;
  if (sr_col0 < 0 || sr_col0 % 4 || sr_cols < cols || sr_col0 + cols > sr_cols)
    return fail(MQV_ERR_INVALID_ARG, "columns [%lld, %lld) are not a 4-aligned window of %lld SR columns",
                (long long)sr_col0, (long long)(sr_col0 + cols), (long long)sr_cols);
  return enqueue_quantize(src, rows, cols, fmt, rounding, seed, amax, 1, sr_cols, sr_col0, out,
                          static_cast<cudaStream_t>(stream));
}

mqv_status mqv_quantize_many_workspace_size(const mqv_quantize_job* jobs, int32_t count,
                                            size_t* bytes) {
  if (!bytes) return fail(MQV_ERR_INVALID_ARG, "null output pointer");
  QuantJobs plan;
  int a = 0, q = 0;
  mqv_status st = plan_quantize_many(jobs, count, &plan, &a, &q, false);
  if (st) return st;
  *bytes = (size_t)((a * sizeof(float) + 255) / 256 * 256);
  return ok();
}

mqv_status mqv_quantize_many(const mqv_quantize_job* jobs, int32_t count, void* ws, size_t ws_bytes,
                             void* stream) {
  QuantJobs plan;
  int a = 0, q = 0;
  mqv_status st = plan_quantize_many(jobs, count, &plan, &a, &q, true);
  if (st) return st;
  if (!ws || ws_bytes < (size_t)a * sizeof(float) || !aligned16(ws))
    return fail(MQV_ERR_WORKSPACE, "workspace of %zu bytes required", (size_t)a * sizeof(float));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* part = static_cast<float*>(ws);
  amax_many_kernel<<<a, kAmaxThreads, 0, s>>>(plan, part);
  cudaError_t e;
  if (plan.job[0].qa.blocks == MQV_BLOCKS_4X4) {
    // a programmatic dependent of the max pass: its CTAs become resident as
    // the max pass runs and load their first blocks before they wait for it
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(q));
    cfg.blockDim = dim3(kQuantThreads);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, quantize_many_kernel, plan, static_cast<const float*>(part));
    if (e != cudaSuccess) return cuda_fail(e, "quantize_many launch");
  } else {
    quantize_many_line_kernel<<<q, kQuantThreads, 0, s>>>(plan, part);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "quantize_many launch");
  return ok();
}

mqv_status mqv_dequantize(const mqv_qtensor* q, float* dst, void* stream) {
  mqv_status st = check_qtensor(q, "q");
  if (st) return st;
  if (!dst || !aligned16(dst)) return fail(MQV_ERR_INVALID_ARG, "dst must be a 16-byte aligned pointer");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const unsigned g = (unsigned)quant_ctas(q->rows, q->cols);
  const uint8_t* c = static_cast<const uint8_t*>(q->codes);
  if (q->fmt == MQV_NVFP4)
    dequantize_kernel<0><<<g, kQuantThreads, 0, s>>>(c, q->scales, q->tscale, q->rows, q->cols, q->blocks, dst);
  else
    dequantize_kernel<1><<<g, kQuantThreads, 0, s>>>(c, q->scales, q->tscale, q->rows, q->cols, q->blocks, dst);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "dequantize launch");
  return ok();
}

// ------------------------------------------------------------ replay form

namespace {

mqv_status check_replay_view(int64_t rows, int64_t cols, int32_t fmt) {
  mqv_status st = check_view(rows, cols);
  if (st) return st;
  return check_fmt(fmt);
}

unsigned replay_ctas(int64_t n) {
  const int64_t segs = (n + kReplaySeg - 1) / kReplaySeg;
  const int64_t g = (segs + kReplayWarps - 1) / kReplayWarps;
  return static_cast<unsigned>(g < kMaxQuantCtas ? g : kMaxQuantCtas);
}

}  // namespace

mqv_status mqv_replay_bytes(int64_t rows, int64_t cols, int32_t fmt, size_t* bytes) {
  mqv_status st = check_replay_view(rows, cols, fmt);
  if (st) return st;
  if (!bytes) return fail(MQV_ERR_INVALID_ARG, "null output pointer");
  *bytes = static_cast<size_t>(rows * cols / 8 * (fmt == MQV_NVFP4 ? 3 : 5));
  return ok();
}

mqv_status mqv_replay_pack(const mqv_qtensor* q, void* packed, uint32_t* negatives, void* stream) {
  mqv_status st = check_qtensor(q, "q");
  if (st) return st;
  if (!packed || !aligned16(packed)) return fail(MQV_ERR_INVALID_ARG, "packed must be a 16-byte aligned pointer");
  if (negatives && (reinterpret_cast<uintptr_t>(negatives) & 3u))
    return fail(MQV_ERR_INVALID_ARG, "negatives must be 4-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t n = q->rows * q->cols;
  const uint8_t* c = static_cast<const uint8_t*>(q->codes);
  uint8_t* o = static_cast<uint8_t*>(packed);
  if (q->fmt == MQV_NVFP4)
    replay_pack_kernel<0><<<replay_ctas(n), kReplayThreads, 0, s>>>(c, n, o, negatives);
  else
    replay_pack_kernel<1><<<replay_ctas(n), kReplayThreads, 0, s>>>(c, n, o, negatives);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "replay pack launch");
  return ok();
}

mqv_status mqv_replay_unpack(const void* packed, int64_t rows, int64_t cols, int32_t fmt, void* codes,
                             void* stream) {
  mqv_status st = check_replay_view(rows, cols, fmt);
  if (st) return st;
  if (!packed || !aligned16(packed) || !codes || !aligned16(codes))
    return fail(MQV_ERR_INVALID_ARG, "packed and codes must be 16-byte aligned pointers");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t n = rows * cols;
  const uint8_t* in = static_cast<const uint8_t*>(packed);
  uint8_t* c = static_cast<uint8_t*>(codes);
  if (fmt == MQV_NVFP4)
    replay_unpack_kernel<0><<<replay_ctas(n), kReplayThreads, 0, s>>>(in, n, c);
  else
    replay_unpack_kernel<1><<<replay_ctas(n), kReplayThreads, 0, s>>>(in, n, c);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "replay unpack launch");
  return ok();
}

mqv_status mqv_replay_dequantize(const void* packed, const uint8_t* scales, const float* tscale, int64_t rows,
                                 int64_t cols, int32_t fmt, float* dst, void* stream) {
  mqv_status st = check_replay_view(rows, cols, fmt);
  if (st) return st;
  if (!packed || !aligned16(packed) || !scales || !tscale || !dst || !aligned16(dst))
    return fail(MQV_ERR_INVALID_ARG, "packed and dst must be 16-byte aligned, scales and tscale non-null");
  if (reinterpret_cast<uintptr_t>(tscale) & 3u) return fail(MQV_ERR_INVALID_ARG, "tscale must be 4-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t n = rows * cols;
  const uint8_t* in = static_cast<const uint8_t*>(packed);
  const FastDiv dc4 = make_fastdiv(cols / 4);
  if (fmt == MQV_NVFP4)
    replay_dequantize_kernel<0><<<replay_ctas(n), kReplayThreads, 0, s>>>(in, scales, tscale, cols, dc4, n, dst);
  else
    replay_dequantize_kernel<1><<<replay_ctas(n), kReplayThreads, 0, s>>>(in, scales, tscale, cols, dc4, n, dst);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "replay dequantize launch");
  return ok();
}

mqv_status mqv_conv_workspace_size(const mqv_conv_desc* d, int32_t op, size_t* bytes) {
  mqv_status st = check_desc(d);
  if (st) return st;
  if (op != MQV_OP_FWD && op != MQV_OP_WGRAD && op != MQV_OP_DGRAD && op != MQV_OP_FWD_BLOCKSCALED)
    return fail(MQV_ERR_INVALID_ARG, "unknown op %d", op);
  if (!bytes) return fail(MQV_ERR_INVALID_ARG, "null output pointer");
  ConvPlan pl;
  if (op == MQV_OP_FWD_BLOCKSCALED) {
    if ((st = plan_blockscaled(d, &pl))) return st;
  } else {
    plan_conv(d, op, &pl);
  }
  *bytes = pl.ws_bytes;
  return ok();
}

mqv_status mqv_conv_fwd_blockscaled(const mqv_conv_desc* d, const mqv_qtensor* w, const mqv_qtensor* x, float* y,
                                    void* ws, size_t ws_bytes, void* stream) {
  mqv_status st = check_desc(d);
  if (st) return st;
  ConvPlan pl;
  if ((st = plan_blockscaled(d, &pl))) return st;
  if ((st = check_operand(w, "w", d->Cout, d->Kh * d->Kw * d->Cin, d->fmt)) ||
      (st = check_operand(x, "x", d->H * d->W * d->Cin, d->N, d->fmt)))
    return st;
  if (w->blocks != MQV_BLOCKS_4X4 || x->blocks != MQV_BLOCKS_4X4)
    return fail(MQV_ERR_UNSUPPORTED, "block-scaled forward pass: 4 x 4 blocks only");
  if (!y || !aligned16(y)) return fail(MQV_ERR_INVALID_ARG, "output must be a 16-byte aligned pointer");
  if (!ws || ws_bytes < pl.ws_bytes || !aligned16(ws))
    return fail(MQV_ERR_WORKSPACE, "workspace of %zu bytes (16-byte aligned) required, got %zu", pl.ws_bytes,
                ws ? ws_bytes : (size_t)0);
  uint32_t* err = nullptr;
  if ((st = device_error_word(&err))) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* image = static_cast<uint8_t*>(ws);
  const V2Args& a = pl.a;
  const int chunks = a.mtiles * 128 * a.ktiles * 8;
  prep_nvf4_image_kernel<<<(unsigned)((chunks + kPrepThreads - 1) / kPrepThreads), kPrepThreads, 0, s>>>(
      make_view(w), a.M, a.ktiles, a.mtiles, make_fastdiv((int64_t)a.ktiles * 8), image);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "block-scaled weight image launch");
  pl.a.err = err;
  pl.a.image = image;
  pl.a.b = make_view(x);
  pl.a.ta = w->tscale;
  pl.a.tb = x->tscale;
  pl.a.out = y;
  static bool done[kMaxDevices] = {};
  if ((e = set_smem(conv_fwd_nvf4_kernel, Nvf4Smem::kBytes, done)) != cudaSuccess) return cuda_fail(e, "smem attribute");
  conv_fwd_nvf4_kernel<<<pl.grid, kNvf4Threads, Nvf4Smem::kBytes, s>>>(pl.a, pl.g);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "block-scaled conv launch");
  return ok();
}

mqv_status mqv_conv_fwd(const mqv_conv_desc* d, const mqv_qtensor* w, const mqv_qtensor* x,
                        float* y, void* ws, size_t ws_bytes, void* stream) {
  return run_conv(MQV_OP_FWD, d, w, "w", x, "x", y, ws, ws_bytes, stream);
}

mqv_status mqv_conv_wgrad(const mqv_conv_desc* d, const mqv_qtensor* gy, const mqv_qtensor* x,
                          float* gw, void* ws, size_t ws_bytes, void* stream) {
  return run_conv(MQV_OP_WGRAD, d, gy, "gy", x, "x", gw, ws, ws_bytes, stream);
}

mqv_status mqv_conv_dgrad(const mqv_conv_desc* d, const mqv_qtensor* w, const mqv_qtensor* gy,
                          float* gx, void* ws, size_t ws_bytes, void* stream) {
  return run_conv(MQV_OP_DGRAD, d, w, "w", gy, "gy", gx, ws, ws_bytes, stream);
}

mqv_status mqv_conv_fwd_fused(const mqv_conv_desc* d, const mqv_qtensor* w, const mqv_qtensor* x, float* y,
                              int32_t relu, float* y_amax, void* ws, size_t ws_bytes, void* stream) {
  return run_conv(MQV_OP_FWD, d, w, "w", x, "x", y, ws, ws_bytes, stream, relu, y_amax);
}

mqv_status mqv_conv_dgrad_fused(const mqv_conv_desc* d, const mqv_qtensor* w, const mqv_qtensor* gy, float* gx,
                                float* gx_amax, void* ws, size_t ws_bytes, void* stream) {
  return run_conv(MQV_OP_DGRAD, d, w, "w", gy, "gy", gx, ws, ws_bytes, stream, 0, gx_amax);
}

mqv_status mqv_conv_fwd_quantized(const mqv_conv_desc* d, const mqv_qtensor* w, const mqv_qtensor* x, int32_t relu,
                                  const float* t_amax, const mqv_qtensor* y_q, float* y_amax, void* ws,
                                  size_t ws_bytes, void* stream) {
  const QuantOut qo{y_q, t_amax, 0};
  return run_conv(MQV_OP_FWD, d, w, "w", x, "x", nullptr, ws, ws_bytes, stream, relu, y_amax, &qo);
}

mqv_status mqv_conv_dgrad_quantized(const mqv_conv_desc* d, const mqv_qtensor* w, const mqv_qtensor* gy,
                                    const float* t_amax, uint64_t seed, const mqv_qtensor* gx_q, float* gx_amax,
                                    void* ws, size_t ws_bytes, void* stream) {
  const QuantOut qo{gx_q, t_amax, seed};
  return run_conv(MQV_OP_DGRAD, d, w, "w", gy, "gy", nullptr, ws, ws_bytes, stream, 0, gx_amax, &qo);
}

mqv_status mqv_selftest_wait_timeout(int64_t limit_cycles, void* stream) {
  if (limit_cycles < 1 || limit_cycles > (int64_t(1) << 32))
    return fail(MQV_ERR_INVALID_ARG, "limit_cycles %lld outside 1 .. 2^32", (long long)limit_cycles);
  uint32_t* err = nullptr;
  mqv_status st = device_error_word(&err);
  if (st) return st;
  wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(err, limit_cycles);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
  return ok();
}

mqv_status mqv_device_errors(uint32_t* flags, void* stream) {
  if (!flags) return fail(MQV_ERR_INVALID_ARG, "null output pointer");
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  uint32_t v = 0;
  e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v));
  if (e != cudaSuccess) return cuda_fail(e, "read error word");
  const uint32_t zero = 0;
  e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero));
  if (e != cudaSuccess) return cuda_fail(e, "clear error word");
  *flags = v;
  if (v) return fail(MQV_ERR_TIMEOUT, "device wait timed out (flags 0x%x)", v);
  return ok();
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Weight gradient without any caller-provided workspace.  The split-K
// partial sums live in a fixed device array that belongs to this library, so
// a caller that has no way to allocate device memory can still run the pass.
namespace {

// Largest split-K partial set the built-in scratch holds (32 MiB per GPU; it
// is part of the library's device image and stays resident until exit).  The
// split planner splits only while the tiles fit one wave of one tile per SM,
// and a tile's partial is at most 128 output channels x 3 taps x 128 input
// channels, so partials stay below 148 x 128 x 384 x 4 B = 29.1 MB; the size
// check below guards that bound.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
static __device__ __align__(256) float g_noalloc_wgrad_scratch[kNoAllocScratchBytes / sizeof(float)];

float* g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mu;

// Device address of the scratch array on the current device, looked up once
// per device (host code cannot use the array's name as a device pointer).
mqv_status noalloc_scratch(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(MQV_ERR_UNSUPPORTED, "device index %d", dev);
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_wgrad_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(wgrad scratch)");
    g_noalloc_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return MQV_OK;
}

}  // namespace

namespace {

mqv_status plan_im2col(const mqv_conv_desc* d, Im2colGeom* g, int64_t* xc_n4, int64_t* x_n4) {
  mqv_status st = check_desc(d);
  if (st) return st;
  g->N = (int)d->N; g->Cin = (int)d->Cin; g->H = (int)d->H; g->W = (int)d->W;
  g->Kh = (int)d->Kh; g->Kw = (int)d->Kw; g->stride = (int)d->stride; g->pad = (int)d->pad;
  g->Ho = (int)((d->H + 2 * d->pad - d->Kh) / d->stride + 1);
  g->Wo = (int)((d->W + 2 * d->pad - d->Kw) / d->stride + 1);
  const int64_t K = d->Kh * d->Kw * d->Cin;
  *xc_n4 = (int64_t)g->Ho * g->Wo * K * (d->N / 4);
  *x_n4 = d->H * d->W * d->Cin * (d->N / 4);
  if (*xc_n4 >= (int64_t(1) << 31) || (int64_t)g->Ho * g->Wo * K >= (int64_t(1) << 31))
    return fail(MQV_ERR_UNSUPPORTED, "the expanded matrix exceeds 2^31 float4");
  g->dn4 = make_fastdiv(d->N / 4);
  g->dcin = make_fastdiv(d->Cin);
  g->dk = make_fastdiv(K);
  g->dkw = make_fastdiv(d->Kw);
  g->dwo = make_fastdiv(g->Wo);
  g->dw = make_fastdiv(d->W);
  return MQV_OK;
}

unsigned naive_grid(int64_t n4) {
  int64_t g = (n4 + kNaiveThreads - 1) / kNaiveThreads;
  if (g > kSMs * 16) g = kSMs * 16;
  return (unsigned)(g < 1 ? 1 : g);
}

}  // namespace

extern "C" mqv_status mqv_im2col(const mqv_conv_desc* d, const float* x, float* xc, void* stream) {
  Im2colGeom g;
  int64_t xc_n4 = 0, x_n4 = 0;
  mqv_status st = plan_im2col(d, &g, &xc_n4, &x_n4);
  if (st) return st;
  if (!x || !xc || !aligned16(x) || !aligned16(xc))
    return fail(MQV_ERR_INVALID_ARG, "x and xc must be 16-byte aligned device pointers");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  im2col_kernel<<<naive_grid(xc_n4), kNaiveThreads, 0, s>>>(g, reinterpret_cast<const float4*>(x),
                                                              reinterpret_cast<float4*>(xc), xc_n4);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "im2col launch");
  return ok();
}

extern "C" mqv_status mqv_col2im(const mqv_conv_desc* d, const float* gc, float* gx, void* stream) {
  Im2colGeom g;
  int64_t xc_n4 = 0, x_n4 = 0;
  mqv_status st = plan_im2col(d, &g, &xc_n4, &x_n4);
  if (st) return st;
  if (!gc || !gx || !aligned16(gc) || !aligned16(gx))
    return fail(MQV_ERR_INVALID_ARG, "gc and gx must be 16-byte aligned device pointers");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  col2im_kernel<<<naive_grid(x_n4), kNaiveThreads, 0, s>>>(g, reinterpret_cast<const float4*>(gc),
                                                             reinterpret_cast<float4*>(gx), x_n4);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "col2im launch");
  return ok();
}

extern "C" mqv_status mqv_conv_wgrad_noalloc(const mqv_conv_desc* d, const mqv_qtensor* gy,
                                             const mqv_qtensor* x, float* gw, void* stream) {
  mqv_status st = check_desc(d);
  if (st) return st;
  ConvPlan pl;
  plan_conv(d, MQV_OP_WGRAD, &pl);
  if (pl.ws_bytes > kNoAllocScratchBytes)
    return fail(MQV_ERR_UNSUPPORTED,
                "mqv_conv_wgrad_noalloc: this layer's split partials need %zu bytes, the built-in "
                "scratch holds %zu; call mqv_conv_wgrad with a workspace instead",
                pl.ws_bytes, kNoAllocScratchBytes);
  float* scratch = nullptr;
  if ((st = noalloc_scratch(&scratch))) return st;
  return run_conv(MQV_OP_WGRAD, d, gy, "gy", x, "x", gw, scratch, kNoAllocScratchBytes, stream);
}

// ------------------------------------------------- depthwise layers in BF16

namespace {

// Checks a depthwise descriptor and fills the geometry (every tensor below
// 2^31 elements, so thread indices fit one grid dimension of 2^31 - 1 CTAs).
mqv_status plan_dw(const mqv_dw_desc* d, DwGeom* g) {
  if (!d) return fail(MQV_ERR_INVALID_ARG, "null depthwise descriptor");
  if (d->reserved || d->reserved2)
    return fail(MQV_ERR_INVALID_ARG, "depthwise descriptor: reserved fields must be 0");
  if (d->N <= 0 || d->C <= 0 || d->H <= 0 || d->W <= 0 || d->Kh <= 0 || d->Kw <= 0)
    return fail(MQV_ERR_INVALID_ARG, "depthwise descriptor: sizes must be positive");
  if (d->N % 4) return fail(MQV_ERR_INVALID_ARG, "depthwise descriptor: N = %lld is not a multiple of 4",
                            (long long)d->N);
  if (d->stride < 1 || d->pad < 0 || d->pad >= d->Kh || d->pad >= d->Kw)
    return fail(MQV_ERR_INVALID_ARG, "depthwise descriptor: need stride >= 1 and 0 <= pad < Kh, Kw");
  const int64_t ho = (d->H + 2 * d->pad - d->Kh) / d->stride + 1;
  const int64_t wo = (d->W + 2 * d->pad - d->Kw) / d->stride + 1;
  if (d->H + 2 * d->pad < d->Kh || d->W + 2 * d->pad < d->Kw || ho < 1 || wo < 1)
    return fail(MQV_ERR_INVALID_ARG, "depthwise descriptor: the kernel is larger than the padded input");
  const int64_t lim = int64_t(1) << 31;
  if (d->H * d->W > lim / d->C / d->N || ho * wo > lim / d->C / d->N || d->Kh * d->Kw > lim / d->C)
    return fail(MQV_ERR_UNSUPPORTED, "depthwise layer too large (a tensor of 2^31 elements or more)");
  *g = dw_geom(d->N, d->C, d->H, d->W, d->Kh, d->Kw, d->stride, d->pad);
  return MQV_OK;
}

unsigned dw_grid(int64_t total) { return static_cast<unsigned>((total + kDwThreads - 1) / kDwThreads); }

// Tiles of dw_tile_kernel.  The staged window plus the weights stay within
// 56 KB of shared memory (four CTAs per SM, as the kernel's register bound
// allows); the first tile shape from 8 x 8 down, and the most channels per
// tile (a divisor of C, at most 32), that give at least four CTAs per SM win;
// if none does, the fitting choice with the most CTAs.  3x3 filters at
// stride 1 or 2 take the row path, whose tiles are 8 wide.  N > 1024 (more than 256 batch quads per channel) has no
// tile.
constexpr int kDwTileSmem = 56 * 1024;
constexpr int64_t kDwTileMinCtas = 4 * 148;

void dw_tile_window(const DwGeom& g, bool dgrad, int th, int tw, int* ih, int* iw) {
  const int s = (int)g.stride, Kh = (int)g.Kh, Kw = (int)g.Kw;
  if (dgrad) {
    // G_Y rows r0 .. r0 + (th + Kh + s - 3) / s: see dw_tile_kernel
    *ih = (th + Kh + s - 3) / s + 1;
    *iw = (tw + Kw + s - 3) / s + 1;
  } else {
    *ih = (th - 1) * s + Kh;
    *iw = (tw - 1) * s + Kw;
  }
}

int64_t dw_tile_smem(const DwGeom& g, int ih, int iw, int cg) {
  return ((cg * g.Kh * g.Kw * 4 + 15) & ~int64_t{15}) + (int64_t)ih * iw * cg * g.N * 2;
}

bool plan_dw_tile(const DwGeom& g, bool dgrad, DwTile* t) {
  static const int shapes[][2] = {{8, 8}, {4, 8}, {4, 4}, {2, 4}, {2, 2}, {1, 2}, {1, 1}};
  static const int rows3_shapes[][2] = {{8, 8}, {4, 8}, {2, 8}, {1, 8}};
  t->rows3 = g.Kh == 3 && g.Kw == 3 && g.stride <= 2;
  const int nq = (int)(g.N / 4);
  if (nq > kDwThreads) return false;
  const int out_h = (int)(dgrad ? g.H : g.Ho), out_w = (int)(dgrad ? g.W : g.Wo);
  int64_t best_ctas = 0;
  bool found = false;
  const int nshapes = t->rows3 ? 4 : 7;
  for (int si = 0; si < nshapes; ++si) {
    const int th = t->rows3 ? rows3_shapes[si][0] : shapes[si][0];
    const int tw = t->rows3 ? rows3_shapes[si][1] : shapes[si][1];
    int ih, iw;
    dw_tile_window(g, dgrad, th, tw, &ih, &iw);
    const int64_t tiles = (int64_t)((out_h + th - 1) / th) * ((out_w + tw - 1) / tw);
    for (int c = 32; c >= 1; --c) {
      if (g.C % c || c * nq > kDwThreads || dw_tile_smem(g, ih, iw, c) > kDwTileSmem) continue;
      const int64_t ctas = tiles * (g.C / c);
      if (ctas > best_ctas) {
        best_ctas = ctas;
        found = true;
        t->th = th;
        t->tw = tw;
        t->cg = c;
        t->ih = ih;
        t->iw = iw;
      }
      if (ctas >= kDwTileMinCtas) goto chosen;
    }
  }
  if (!found) return false;
chosen:
  t->src_h = (int)(dgrad ? g.Ho : g.H);
  t->src_w = (int)(dgrad ? g.Wo : g.W);
  t->out_h = out_h;
  t->out_w = out_w;
  t->tiles_w = (out_w + t->tw - 1) / t->tw;
  t->tiles_h = (out_h + t->th - 1) / t->th;
  t->vec16 = (g.C * g.N) % 8 == 0 && ((int64_t)t->cg * g.N) % 8 == 0;
  return (int64_t)t->tiles_w * t->tiles_h * (g.C / t->cg) < (int64_t{1} << 31);
}

// Tiles of dw_wgrad_tile_kernel (3x3 filters, stride 1 or 2): the staged x
// window, G_Y tile and the CTA's 256 x 9 sums within 56 KB; channels per
// tile such that lanes (channels x batch quads) divide 256.  Of the tile
// shapes 8 wide and the channel counts, the one with the most working
// threads (CTAs x the threads that get a row), capped at four full CTAs per
// SM, wins; ties go to the larger tile and the more channels.
int64_t dw_wgrad_tile_smem(const DwGeom& g, int th, int ih, int iw, int cg) {
  return ((int64_t)(ih * iw + th * 8) * cg * g.N * 2 + 15) / 16 * 16 + (int64_t)kDwThreads * 9 * 4;
}

bool plan_dw_wgrad_tile(const DwGeom& g, DwTile* t) {
  if (g.Kh != 3 || g.Kw != 3 || g.stride > 2) return false;
  const int nq = (int)(g.N / 4);
  if (nq > kDwThreads) return false;
  const int s = (int)g.stride;
  int64_t best = 0;
  for (int th : {8, 4, 2, 1}) {
    const int ih = (th - 1) * s + 3, iw = 7 * s + 3;
    const int64_t tiles = (int64_t)((g.Ho + th - 1) / th) * ((g.Wo + 7) / 8);
    for (int c = 32; c >= 1; --c) {
      const int lanes = c * nq;
      if (g.C % c || kDwThreads % lanes || dw_wgrad_tile_smem(g, th, ih, iw, c) > kDwTileSmem) continue;
      const int64_t rows = std::min<int64_t>(kDwThreads / lanes, th);
      const int64_t score = std::min<int64_t>(tiles * (g.C / c) * rows * lanes, kDwTileMinCtas * kDwThreads);
      if (score > best) {
        best = score;
        t->th = th;
        t->tw = 8;
        t->cg = c;
        t->ih = ih;
        t->iw = iw;
      }
    }
  }
  if (best == 0) return false;
  t->src_h = (int)g.H;
  t->src_w = (int)g.W;
  t->out_h = (int)g.Ho;
  t->out_w = (int)g.Wo;
  t->tiles_w = (t->out_w + 7) / 8;
  t->tiles_h = (t->out_h + t->th - 1) / t->th;
  t->vec16 = (g.C * g.N) % 8 == 0 && ((int64_t)t->cg * g.N) % 8 == 0;
  t->rows3 = 1;
  return (int64_t)t->tiles_w * t->tiles_h * (g.C / t->cg) < (int64_t{1} << 31);
}

template <int S, int PIX>
cudaError_t launch_dw_wgrad_tile_p(const DwGeom& g, const DwTile& t, int64_t blocks, size_t smem, const uint16_t* gy,
                                   const uint16_t* x, float* part, cudaStream_t st) {
  static bool done[kMaxDevices] = {};
  cudaError_t e = set_smem(dw_wgrad_tile_kernel<S, PIX>, kDwTileSmem, done);
  if (e != cudaSuccess) return e;
  dw_wgrad_tile_kernel<S, PIX><<<(unsigned)blocks, kDwThreads, smem, st>>>(g, t, gy, x, part);
  return cudaGetLastError();
}

// dw_wgrad_tile_kernel with the staged pixel's size as a constant for the
// common sizes.
template <int S>
cudaError_t launch_dw_wgrad_tile(const DwGeom& g, const DwTile& t, int64_t blocks, size_t smem, const uint16_t* gy,
                                 const uint16_t* x, float* part, cudaStream_t st) {
  switch (t.cg * (int)g.N) {
    case 32: return launch_dw_wgrad_tile_p<S, 32>(g, t, blocks, smem, gy, x, part, st);
    case 64: return launch_dw_wgrad_tile_p<S, 64>(g, t, blocks, smem, gy, x, part, st);
    case 128: return launch_dw_wgrad_tile_p<S, 128>(g, t, blocks, smem, gy, x, part, st);
    case 256: return launch_dw_wgrad_tile_p<S, 256>(g, t, blocks, smem, gy, x, part, st);
    case 512: return launch_dw_wgrad_tile_p<S, 512>(g, t, blocks, smem, gy, x, part, st);
    default: return launch_dw_wgrad_tile_p<S, 0>(g, t, blocks, smem, gy, x, part, st);
  }
}

// Workspace bytes of the weight gradient: the tiles' partial sums, or the
// parts' of the gather kernel.
int64_t dw_wgrad_ws_bytes(const DwGeom& g) {
  DwTile t;
  const int64_t n = plan_dw_wgrad_tile(g, &t) ? (int64_t)t.tiles_w * t.tiles_h * g.C * 9 : dw_wgrad_threads(g);
  return n * (int64_t)sizeof(float);
}

template <bool DGRAD, int S, bool ROWS3, int PIX = 0>
cudaError_t launch_dw_tile_s(const DwGeom& g, const DwTile& t, const uint16_t* w, const uint16_t* src, float* out,
                             cudaStream_t st) {
  auto kern = dw_tile_kernel<DGRAD, S, ROWS3, PIX>;
  static bool done[kMaxDevices] = {};
  cudaError_t e = set_smem(kern, kDwTileSmem, done);
  if (e != cudaSuccess) return e;
  const int64_t blocks = (int64_t)t.tiles_w * t.tiles_h * (g.C / t.cg);
  kern<<<(unsigned)blocks, kDwThreads, (size_t)dw_tile_smem(g, t.ih, t.iw, t.cg), st>>>(g, t, w, src, out);
  return cudaGetLastError();
}

// The row path with the staged pixel's size (channels x batch, bf16) as a
// constant for the common sizes.
template <bool DGRAD, int S>
cudaError_t launch_dw_rows3(const DwGeom& g, const DwTile& t, const uint16_t* w, const uint16_t* src, float* out,
                            cudaStream_t st) {
  switch (t.cg * (int)g.N) {
    case 32: return launch_dw_tile_s<DGRAD, S, true, 32>(g, t, w, src, out, st);
    case 64: return launch_dw_tile_s<DGRAD, S, true, 64>(g, t, w, src, out, st);
    case 128: return launch_dw_tile_s<DGRAD, S, true, 128>(g, t, w, src, out, st);
    case 256: return launch_dw_tile_s<DGRAD, S, true, 256>(g, t, w, src, out, st);
    case 512: return launch_dw_tile_s<DGRAD, S, true, 512>(g, t, w, src, out, st);
    default: return launch_dw_tile_s<DGRAD, S, true, 0>(g, t, w, src, out, st);
  }
}

template <bool DGRAD>
cudaError_t launch_dw_tile(const DwGeom& g, const DwTile& t, const uint16_t* w, const uint16_t* src, float* out,
                           cudaStream_t st) {
  if (t.rows3) {
    if (g.stride == 1) return launch_dw_rows3<DGRAD, 1>(g, t, w, src, out, st);
    if (g.stride == 2) return launch_dw_rows3<DGRAD, 2>(g, t, w, src, out, st);
  }
  if (g.stride == 1) return launch_dw_tile_s<DGRAD, 1, false>(g, t, w, src, out, st);
  if (g.stride == 2) return launch_dw_tile_s<DGRAD, 2, false>(g, t, w, src, out, st);
  return launch_dw_tile_s<DGRAD, 0, false>(g, t, w, src, out, st);
}

}  // namespace

extern "C" mqv_status mqv_dw_wgrad_workspace_size(const mqv_dw_desc* d, size_t* bytes) {
  DwGeom g;
  mqv_status st = plan_dw(d, &g);
  if (st) return st;
  if (!bytes) return fail(MQV_ERR_INVALID_ARG, "null output pointer");
  *bytes = (size_t)((dw_wgrad_ws_bytes(g) + 255) / 256 * 256);
  return ok();
}

extern "C" mqv_status mqv_dw_fwd(const mqv_dw_desc* d, const void* w, const void* x, float* y, void* stream) {
  DwGeom g;
  mqv_status st = plan_dw(d, &g);
  if (st) return st;
  if (!w || !x || !y || !aligned16(w) || !aligned16(x) || !aligned16(y))
    return fail(MQV_ERR_INVALID_ARG, "w, x and y must be 16-byte aligned device pointers");
  cudaError_t e;
  DwTile t;
  if (plan_dw_tile(g, false, &t)) {
    e = launch_dw_tile<false>(g, t, static_cast<const uint16_t*>(w), static_cast<const uint16_t*>(x), y,
                              static_cast<cudaStream_t>(stream));
  } else {
    const int64_t total = dw_fwd_threads(g);
    dw_fwd_kernel<<<dw_grid(total), kDwThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        g, total, static_cast<const uint16_t*>(w), static_cast<const uint16_t*>(x), y);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) return cuda_fail(e, "depthwise fwd launch");
  return ok();
}

extern "C" mqv_status mqv_dw_dgrad(const mqv_dw_desc* d, const void* w, const void* gy, float* gx,
                                   void* stream) {
  DwGeom g;
  mqv_status st = plan_dw(d, &g);
  if (st) return st;
  if (!w || !gy || !gx || !aligned16(w) || !aligned16(gy) || !aligned16(gx))
    return fail(MQV_ERR_INVALID_ARG, "w, gy and gx must be 16-byte aligned device pointers");
  cudaError_t e;
  DwTile t;
  if (plan_dw_tile(g, true, &t)) {
    e = launch_dw_tile<true>(g, t, static_cast<const uint16_t*>(w), static_cast<const uint16_t*>(gy), gx,
                             static_cast<cudaStream_t>(stream));
  } else {
    const int64_t total = dw_dgrad_threads(g);
    dw_dgrad_kernel<<<dw_grid(total), kDwThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        g, total, static_cast<const uint16_t*>(w), static_cast<const uint16_t*>(gy), gx);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) return cuda_fail(e, "depthwise dgrad launch");
  return ok();
}

extern "C" mqv_status mqv_dw_wgrad(const mqv_dw_desc* d, const void* gy, const void* x, float* gw, void* ws,
                                   size_t ws_bytes, void* stream) {
  DwGeom g;
  mqv_status st = plan_dw(d, &g);
  if (st) return st;
  if (!gy || !x || !gw || !aligned16(gy) || !aligned16(x) || !aligned16(gw))
    return fail(MQV_ERR_INVALID_ARG, "gy, x and gw must be 16-byte aligned device pointers");
  const size_t need = (size_t)dw_wgrad_ws_bytes(g);
  if (!ws || ws_bytes < need || !aligned16(ws))
    return fail(MQV_ERR_WORKSPACE, "workspace of %zu bytes required", need);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* part = static_cast<float*>(ws);
  const int64_t nw = g.C * g.Kh * g.Kw;
  cudaError_t e;
  DwTile t;
  if (plan_dw_wgrad_tile(g, &t)) {
    const int64_t blocks = (int64_t)t.tiles_w * t.tiles_h * (g.C / t.cg);
    const size_t smem = (size_t)dw_wgrad_tile_smem(g, t.th, t.ih, t.iw, t.cg);
    const uint16_t* gyp = static_cast<const uint16_t*>(gy);
    const uint16_t* xp = static_cast<const uint16_t*>(x);
    e = g.stride == 1 ? launch_dw_wgrad_tile<1>(g, t, blocks, smem, gyp, xp, part, s)
                      : launch_dw_wgrad_tile<2>(g, t, blocks, smem, gyp, xp, part, s);
    if (e != cudaSuccess) return cuda_fail(e, "depthwise wgrad launch");
    const int64_t parts = (int64_t)t.tiles_w * t.tiles_h;
    dw_wgrad_tile_reduce<<<dw_grid(nw * 32), kDwThreads, 0, s>>>(parts, nw, part, gw);
  } else {
    const int64_t total = dw_wgrad_threads(g);
    dw_wgrad_kernel<<<dw_grid(total), kDwThreads, 0, s>>>(g, total, static_cast<const uint16_t*>(gy),
                                                          static_cast<const uint16_t*>(x), part);
    dw_wgrad_reduce_kernel<<<dw_grid(nw), kDwThreads, 0, s>>>(g, nw, part, gw);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "depthwise wgrad launch");
  return ok();
}
