// Persistent, warp-specialized implicit-GEMM kernels for the three conv
// GEMMs on square-block quantized operands (MicroQonv summary,
// onedev.kr/papers/182, section "무엇과 다른가": Y = W·X', G_W = G_Y·X'^T,
// G_X' = W^T·G_Y; im2col built on chip, section "어떻게 동작하나").
//
// Forward and input-gradient (conv_fd_kernel): D[m][col] = sum_k A[m][k]·B[col][k]
//   m   = output channel of the pass (co for fwd, ci for dgrad), 128 per tile
//   col = (output pixel, n) of the pass, BN per tile
//   k   = (kh, kw, reduced channel)
//   A = W (fwd) or W^T (dgrad): small, dequantized once per call by
//       prep_image_kernel into an fp16 image laid out exactly like the
//       swizzled K-major shared-memory tile, then brought in 16 KB per stage
//       with one plain bulk copy.
//   B = the im2col rows of X (fwd) or the transposed-conv gather of G_Y
//       (dgrad), dequantized on chip by 8 producer warps straight from the
//       channel-batch-first codes into an MN-major tile: for one channel the
//       codes of consecutive batch items are consecutive, which is exactly
//       the MN-major order, so no transpose is needed.
// Weight gradient (conv_wg_kernel): D[co][(kh,kw,ci)] = sum over (ho,wo,n)
//   A = G_Y and B = X', both gathered K-major (their codes run along n, the
//   contraction), split over CTAs along (ho, wo, n).
//
// Roles (one CTA per SM, persistent over tiles):
//   warps 0-3 epilogue (tcgen05.ld from TMEM lane quarter = warp, scale by
//             T_a·T_b, fp32 store), double-buffered accumulators so a tile's
//             epilogue overlaps the next tile's MMAs;
//   warp  4   tensor-memory allocation and the single MMA-issuing thread;
//   warp  5   bulk-copy loader of the A image (fwd/dgrad);
//   warps 6-13 producers (gather + dequantize).
// Every wait is bounded (see mbar_wait_bounded); nothing waits on another
// CTA or GPU.
#pragma once

#include <cstdint>

#include "mqv_conv_common.cuh"
#include "mqv_ptx.cuh"
#include "mqv_quantize.cuh"

namespace mqv {

constexpr int kV2EpiWarps = 4;
constexpr int kV2MmaWarp = 4;
constexpr int kV2LoadWarp = 5;
constexpr int kV2ProdWarp0 = 6;
constexpr int kV2ProdThreads = 256;
constexpr int kV2Threads = (kV2ProdWarp0 + kV2ProdThreads / 32) * 32;   // 448
constexpr int kV2Stages = 4;
constexpr uint32_t kATileBytes = 128 * 64 * 2;                             // 16 KB
constexpr int kMaxPhases = 4;             // stride-2 input gradient: (hi mod 2, wi mod 2)
constexpr int kMaxLiveWords = 8;          // live-K-tile masks cover up to 256 K tiles

struct V2Args {
  const uint8_t* image;   // fwd/dgrad: A image [mtiles][ktiles] x 16 KB
  QView a;                // wgrad: G_Y
  QView b;                // fwd: X, dgrad: G_Y, wgrad: X
  const float* ta;
  const float* tb;
  float* out;
  uint32_t* err;
  int N, Cin, Cout, H, W, Kh, Kw, stride, pad, Ho, Wo;
  int M;                  // GEMM rows (channels)
  int Cred;               // fwd: Cin, dgrad: Cout (channels of the reduction)
  int64_t Ncols;          // GEMM columns
  int64_t Kdim;           // contraction length
  int ktiles;             // K tiles of 64 over the whole contraction
  int kt_per_split;       // wgrad: K tiles per split
  int splits;
  int mtiles, ntiles;
  int tiles;              // mtiles * ntiles * splits
  int scale_out;          // multiply by T_a·T_b (0 for wgrad split partials)
  // Fused producer epilogue (fwd/dgrad only): relu != 0 stores max(v, 0);
  // amax_out != nullptr receives max|stored value| as fp32 bits through
  // atomicMax (non-negative floats order like their bit patterns).
  uint32_t* amax_out;
  int relu;
  // Quantized output (kernel-row halo kernel only): with q_codes set the
  // output is not stored in fp32 but quantized as the next operand of the
  // method, a (pixels·M) x N view in q_codes / q_scales, with the tensor
  // scale T from the device max |x| *q_amax (written to *q_tscale); round to
  // nearest for the forward pass, stochastic rounding (q_keys) for dgrad.
  uint8_t* q_codes;
  uint8_t* q_scales;
  float* q_tscale;
  const float* q_amax;
  PhiloxKeys q_keys;
  // Transposed tiles of the generic fwd/dgrad kernel (TR): the MMA's 128
  // rows are GEMM columns (pixel, n) and its N = nc (M rounded up to 16)
  // columns are the output channels.
  int nc;
  FastDiv dN, dWo, dW, dCred, dKw, dCin, dS;
  // Input gradient with stride 2 on the generic kernel: the GEMM columns are
  // grouped by phase (hi mod 2, wi mod 2) so that the columns of a tile
  // share one phase, and a tile gathers and multiplies only the K tiles that
  // hold a tap of its phase (the other taps never reach its pixels).  With
  // phases = 1 column tile nt covers GEMM columns nt·BN.. of the whole pass.
  int phases;                             // 4, or 1 (no phase grouping)
  int ph_tile0[kMaxPhases + 1];           // first column tile of each phase
  int ph_h0[kMaxPhases], ph_w0[kMaxPhases];
  int ph_wp[kMaxPhases];                  // pixels per row of the phase's grid
  FastDiv ph_dwp[kMaxPhases];
  int64_t ph_cols[kMaxPhases];            // GEMM columns of the phase (phase 0: all when phases = 1)
  int ph_nlive[kMaxPhases];               // live K tiles of the phase
  uint32_t ph_live[kMaxPhases][kMaxLiveWords];
};

// The kernels take the phase grouping as a template flag PH; without it
// (phases = 1) these reduce to the plain column mapping at no cost.
// Phase of column tile nt, and whether K tile kt holds a tap of phase q.
template <bool PH>
__device__ __forceinline__ int phase_of(const V2Args& p, int nt) {
  int q = 0;
  if (PH) {
#pragma unroll
    for (int i = 1; i < kMaxPhases; ++i)
      if (nt >= p.ph_tile0[i]) q = i;
  }
  return q;
}

template <bool PH>
__device__ __forceinline__ bool kt_live(const V2Args& p, int q, int kt) {
  return !PH || ((p.ph_live[q][kt >> 5] >> (kt & 31)) & 1u);
}

// Output pixel and batch item of phase-local GEMM column lcol of phase q;
// false past the phase's columns.
template <bool PH>
__device__ __forceinline__ bool col_pixel(const V2Args& p, int q, int64_t lcol, int& pix, int& n) {
  const bool ok = lcol < (PH ? p.ph_cols[q] : p.Ncols);
  const int c32 = ok ? static_cast<int>(lcol) : 0;     // GEMM columns stay below 2^31
  const int pp = fdiv(c32, p.dN);
  n = c32 - pp * p.N;
  if (!PH) {
    pix = pp;
  } else {
    const int i = fdiv(pp, p.ph_dwp[q]);
    const int j = pp - i * p.ph_wp[q];
    pix = (p.ph_h0[q] + 2 * i) * p.W + p.ph_w0[q] + 2 * j;
  }
  return ok;
}

// Entries of the per-CTA K-tile table of the forward / input-gradient
// producers (16 per K tile): larger contractions decode on the fly.
constexpr int kKtabEntries = 4096;
constexpr uint32_t kKtabInvalid = 0xFFFFFFFFu;

template <int BN>
struct V2Smem {
  static constexpr int kBTile = BN * 128;
  static constexpr int kStage = kATileBytes + kBTile;
  static constexpr int kBarOffset = kV2Stages * kStage;
  static constexpr int kKtabOffset = kBarOffset + 256;
  static constexpr int kLiveOffset = kKtabOffset + kKtabEntries * 4;     // kMaxPhases x 256 K tiles
  static constexpr int kBytes = kLiveOffset + kMaxPhases * 256 + 1024;
};

// MN-major 128B-swizzled fp16 tile of BN rows (MN) x 64 K: atoms of 64 MN x
// 8 K (1 KB); the 8 K-atoms of one MN-atom are consecutive (SBO = 1 KB), the
// MN-atoms 8 KB apart (LBO).
__device__ __forceinline__ uint32_t mn_offset(uint32_t mn, uint32_t k) {
  return (mn >> 6) * 8192u + (k >> 3) * 1024u + (k & 7u) * 128u +
         ((((mn & 63u) >> 3) ^ (k & 7u)) << 4) + (mn & 7u) * 2u;
}

// ---------------------------------------------------------------------------
// Code decoding helpers.  code·scale is exact in fp16: an E2M1 (E2M3) value
// has at most 2 (4) significant bits, an E4M3 scale 4, and every product lies
// between 2^-12 and 3360, inside the fp16 range; the tensor scales are applied
// in the epilogue.

// 8 FP4 codes of one source row (n0..n0+7) times their two block scales
// (n0..n0+3 use s2lo, n0+4..n0+7 use s2hi) -> 4 fp16x2 in n order.
__device__ __forceinline__ void dq8_fp4(uint32_t w, uint32_t s2lo, uint32_t s2hi, uint32_t (&h)[4]) {
  e2m1x8_to_f16x2(w, h);
  h[0] = hmul2_u32(h[0], s2lo);
  h[1] = hmul2_u32(h[1], s2lo);
  h[2] = hmul2_u32(h[2], s2hi);
  h[3] = hmul2_u32(h[3], s2hi);
}

// 4 FP6 codes in the low 24 bits of q -> 2 fp16x2.
__device__ __forceinline__ void dq4_fp6(uint32_t q, uint32_t s2, uint32_t& h01, uint32_t& h23) {
  h01 = hmul2_u32(e2m3x2_to_f16x2((q & 0x3F) | ((q << 2) & 0x3F00)), s2);
  h23 = hmul2_u32(e2m3x2_to_f16x2(((q >> 12) & 0x3F) | ((q >> 10) & 0x3F00)), s2);
}

__device__ __forceinline__ uint32_t scale2(uint32_t s) { return e4m3x2_to_f16x2(s | (s << 8)); }

// Load the codes of `nu` (8 or 4) consecutive columns starting at column c
// of view row `row` (c a multiple of nu).  FP4: nu/2 bytes; FP6: 3·nu/4 bytes.
template <int FMT, int NU>
__device__ __forceinline__ uint32_t load_codes(const QView& v, int64_t row, int64_t c, uint32_t& hi) {
  const uint8_t* p = v.codes + row * v.row_bytes;
  hi = 0;
  if (FMT == 0) {
    if (NU == 8) return __ldg(reinterpret_cast<const uint32_t*>(p + (c >> 1)));
    return __ldg(reinterpret_cast<const unsigned short*>(p + (c >> 1)));
  } else {
    const uint8_t* q = p + ((c * 3) >> 2);
    if (NU == 8) {   // 6 bytes, 2-byte aligned
      const unsigned short* q16 = reinterpret_cast<const unsigned short*>(q);
      const uint32_t a = __ldg(q16), b = __ldg(q16 + 1), d = __ldg(q16 + 2);
      const uint32_t lo = a | (b << 16);          // bytes 0-3
      hi = d;                                      // bytes 4-5
      return lo;
    }
    return static_cast<uint32_t>(__ldg(q)) | (static_cast<uint32_t>(__ldg(q + 1)) << 8) |
           (static_cast<uint32_t>(__ldg(q + 2)) << 16);
  }
}

// Dequantize NU codes of one source row into NU/2 fp16x2 (column order).
template <int FMT, int NU>
__device__ __forceinline__ void dequant_run(uint32_t lo, uint32_t hi, uint32_t s2lo, uint32_t s2hi,
                                            uint32_t (&h)[4]) {
  if (FMT == 0) {
    if (NU == 8) {
      dq8_fp4(lo, s2lo, s2hi, h);
    } else {
      h[0] = hmul2_u32(e2m1x2_to_f16x2(lo & 0xFF), s2lo);
      h[1] = hmul2_u32(e2m1x2_to_f16x2((lo >> 8) & 0xFF), s2lo);
    }
  } else {
    dq4_fp6(lo & 0xFFFFFF, s2lo, h[0], h[1]);
    if (NU == 8) dq4_fp6((lo >> 24) | (hi << 8), s2hi, h[2], h[3]);
  }
}

// ---------------------------------------------------------------------------
// A image: [mtiles][ktiles] tiles, each 128 rows x 64 fp16, K-major, rows of
// 128 B with the 16-byte chunks XOR-swizzled by (row & 7), i.e. byte for byte
// the shared-memory tile the MMA reads.  fwd: A[co][k] = W[co][k];
// dgrad: A[ci][(tap, co)] = W[co][tap·Cin + ci].  Rows/columns past the
// matrix are zero.  One thread per 16-byte chunk.
constexpr int kPrepThreads = 128;

template <int FMT, bool TRANS>
__global__ void __launch_bounds__(kPrepThreads)
prep_image_kernel(QView w, int M, int Kdim, int ktiles, int mtiles, int Cin, int Cout, FastDiv dkt8,
                  FastDiv dcout, uint8_t* __restrict__ image) {
  // the conv kernel after this one may start its own setup now (it waits
  // for this kernel's completion before it reads the image)
  pdl_launch_dependents();
  const int chunks = mtiles * 128 * ktiles * 8;
  const int id = blockIdx.x * kPrepThreads + threadIdx.x;
  if (id >= chunks) return;
  // forward: consecutive threads take consecutive K chunks of one weight row
  // (contiguous codes); transposed: consecutive threads take consecutive rows
  // m = ci of one K chunk, so a warp's code reads walk along a weight row
  int m, k0;
  if (!TRANS) {
    m = fdiv(id, dkt8);
    k0 = (id - m * ktiles * 8) * 8;
  } else {
    const int mrows = mtiles * 128;
    const int kc = id / mrows;
    m = id - kc * mrows;
    k0 = kc * 8;
  }
  uint32_t h[4] = {0u, 0u, 0u, 0u};
  if (m < M) {
    if (!TRANS && w.blocks == 0 && k0 + 8 <= Kdim && (FMT == 0 ? (w.row_bytes & 3) == 0 : (w.row_bytes & 1) == 0)) {
      // eight consecutive codes of one weight row: one word (FP4) or three
      // half-words (FP6) and the two block scales
      uint32_t hi = 0;
      const uint32_t lo = load_codes<FMT, 8>(w, m, k0, hi);
      const uint32_t ss = __ldg(reinterpret_cast<const unsigned short*>(w.scales + (m >> 2) * w.scale_cols + (k0 >> 2)));
      dequant_run<FMT, 8>(lo, hi, scale2(ss & 0xFF), scale2(ss >> 8), h);
    } else {
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        const int k = k0 + e;
        if (k >= Kdim) break;
        int row, col;
        if (!TRANS) {
          row = m;
          col = k;
        } else {
          const int tap = fdiv(k, dcout), co = k - tap * Cout;
          row = co;
          col = tap * Cin + m;
        }
        uint32_t c0, c1;
        const uint8_t* p = w.codes + static_cast<int64_t>(row) * w.row_bytes;
        const int row2 = TRANS ? row + 1 : row;       // second element: next co (dgrad)
        const int col2 = TRANS ? col : col + 1;
        // the pair's two scales (4 x 4 blocks: one block holds both, as
        // row (dgrad) or col (forward) is even)
        const uint32_t s0 = __ldg(w.scales + scale_index(w, row, col));
        const uint32_t s = s0 | ((w.blocks ? __ldg(w.scales + scale_index(w, row2, col2)) : s0) << 8);
        const uint8_t* p2 = w.codes + static_cast<int64_t>(row2) * w.row_bytes;
        if (FMT == 0) {
          c0 = (__ldg(p + (col >> 1)) >> ((col & 1) * 4)) & 0xF;
          c1 = (__ldg(p2 + (col2 >> 1)) >> ((col2 & 1) * 4)) & 0xF;
          h[e >> 1] = hmul2_u32(e2m1x2_to_f16x2(c0 | (c1 << 4)), e4m3x2_to_f16x2(s));
        } else {
          auto code6 = [](const uint8_t* base, int c) -> uint32_t {
            const uint8_t* q = base + (c >> 2) * 3;
            const uint32_t v = static_cast<uint32_t>(__ldg(q)) | (static_cast<uint32_t>(__ldg(q + 1)) << 8) |
                               (static_cast<uint32_t>(__ldg(q + 2)) << 16);
            return (v >> ((c & 3) * 6)) & 0x3F;
          };
          c0 = code6(p, col);
          c1 = code6(p2, col2);
          h[e >> 1] = hmul2_u32(e2m3x2_to_f16x2(c0 | (c1 << 8)), e4m3x2_to_f16x2(s));
        }
      }
    }
  }
  const int mt = m >> 7, r = m & 127, kt = k0 >> 6, kc = (k0 & 63) >> 3;
  uint8_t* dst = image + (static_cast<int64_t>(mt) * ktiles + kt) * kATileBytes + r * 128 + ((kc ^ (r & 7)) << 4);
  *reinterpret_cast<uint4*>(dst) = make_uint4(h[0], h[1], h[2], h[3]);
}

// ---------------------------------------------------------------------------
// Shared control block of the persistent kernels.
struct V2Bars {
  uint64_t full[kV2Stages];
  uint64_t empty[kV2Stages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint32_t tmem;
};

template <int BN>
__device__ __forceinline__ V2Bars* v2_setup(uint8_t* smem, int full_count) {
  V2Bars* bars = reinterpret_cast<V2Bars*>(smem + V2Smem<BN>::kBarOffset);
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kV2Stages; ++s) {
      mbar_init(&bars->full[s], full_count);
      mbar_init(&bars->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&bars->acc_full[a], 1);
      mbar_init(&bars->acc_empty[a], kV2EpiWarps * 32);
    }
    fence_mbar_init();
  }
  if (warp == kV2MmaWarp) {
    tmem_alloc(&bars->tmem, 2 * BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  return bars;
}

template <int BN>
__device__ __forceinline__ void v2_teardown(V2Bars* bars) {
  tc_fence_before();
  __syncthreads();
  if ((threadIdx.x >> 5) == kV2MmaWarp) {
    tc_fence_after();
    tmem_dealloc(bars->tmem, 2 * BN);
  }
}

// Epilogue of one tile: TMEM accumulator buffer `acc` -> fp32 output.
// FD=true: out[(pixel·M + m)·N + n] with col = pixel·N + n;
// FD=false (wgrad): out[(split·M + m)·Ncols + col].
// ReLU that maps -0 and NaN to +0, and the running max of |v|.
__device__ __forceinline__ float4 epi_relu(float4 o) {
  o.x = o.x > 0.f ? o.x : 0.f;
  o.y = o.y > 0.f ? o.y : 0.f;
  o.z = o.z > 0.f ? o.z : 0.f;
  o.w = o.w > 0.f ? o.w : 0.f;
  return o;
}

__device__ __forceinline__ float epi_absmax(float m, float4 o) {
  return fmaxf(m, fmaxf(fmaxf(fabsf(o.x), fabsf(o.y)), fmaxf(fabsf(o.z), fabsf(o.w))));
}

// One atomic per warp: the warp's largest |v| into *amax_out.
__device__ __forceinline__ void epi_amax_flush(uint32_t* amax_out, float m) {
  if (amax_out == nullptr) return;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  if ((threadIdx.x & 31) == 0) atomicMax(amax_out, __float_as_uint(m));
}

// FD: col0 is the tile's first column local to phase q (see col_pixel).
template <int BN, bool FD, bool PH = false>
__device__ __forceinline__ void v2_epilogue(const V2Args& p, V2Bars* bars, int acc, int64_t m0,
                                            int64_t col0, int split, bool has_k, float& amax, int q = 0) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t m = m0 + warp * 32 + lane;
  const float scale = p.scale_out ? __fmul_rn(*p.ta, *p.tb) : 1.0f;
  const uint32_t tbase = bars->tmem + (static_cast<uint32_t>(warp * 32) << 16) + acc * BN;
  // a warp whose 32 accumulator rows all lie past the M channels has nothing to store
  const int cend = m0 + warp * 32 < p.M ? BN : 0;
#pragma unroll 1
  for (int c = 0; c < cend; c += 32) {
    uint32_t r[32];
    tmem_ld_32x32b_x32(tbase + c, r);
    tmem_ld_wait();
    if (m < p.M) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int64_t col = col0 + c + 4 * j;
        if (col >= (FD && PH ? p.ph_cols[q] : p.Ncols)) continue;
        float4 o;
        o.x = has_k ? __uint_as_float(r[4 * j + 0]) * scale : 0.f;
        o.y = has_k ? __uint_as_float(r[4 * j + 1]) * scale : 0.f;
        o.z = has_k ? __uint_as_float(r[4 * j + 2]) * scale : 0.f;
        o.w = has_k ? __uint_as_float(r[4 * j + 3]) * scale : 0.f;
        int64_t idx;
        if (FD) {
          if (p.relu) o = epi_relu(o);
          if (p.amax_out) amax = epi_absmax(amax, o);
          int pix, n;
          col_pixel<PH>(p, q, col, pix, n);
          idx = (static_cast<int64_t>(pix) * p.M + m) * p.N + n;
        } else {
          idx = (static_cast<int64_t>(split) * p.M + m) * p.Ncols + col;
        }
        *reinterpret_cast<float4*>(p.out + idx) = o;
      }
    }
  }
  tc_fence_before();
  mbar_arrive(&bars->acc_empty[acc]);
}

// Epilogue of a transposed tile: TMEM lane = GEMM column (pixel, n), TMEM
// column = output channel.  Each lane stores its column's channels one by
// one; for one channel the 32 lanes of a warp write consecutive batch items,
// so every store of a warp covers runs of N contiguous floats.
template <int BN, bool PH>
__device__ __forceinline__ void v2_epilogue_tr(const V2Args& p, V2Bars* bars, int acc, int64_t col0, int q,
                                               bool has_k, float& amax) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int pix, n;
  const bool ok = col_pixel<PH>(p, q, col0 + warp * 32 + lane, pix, n);
  float* out = p.out + static_cast<int64_t>(pix) * p.M * p.N + n;
  const float scale = __fmul_rn(*p.ta, *p.tb);
  const uint32_t tbase = bars->tmem + (static_cast<uint32_t>(warp * 32) << 16) + acc * BN;
#pragma unroll 1
  for (int c = 0; c < p.nc; c += 16) {
    uint32_t r[16];
    tmem_ld_32x32b_x16(tbase + c, r);
    tmem_ld_wait();
    if (ok) {
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int m = c + j;
        if (m < p.M) {
          float v = has_k ? __uint_as_float(r[j]) * scale : 0.f;
          if (p.relu) v = v > 0.f ? v : 0.f;
          if (p.amax_out) amax = fmaxf(amax, fabsf(v));
          out[static_cast<int64_t>(m) * p.N] = v;
        }
      }
    }
  }
  tc_fence_before();
  mbar_arrive(&bars->acc_empty[acc]);
}

// ---------------------------------------------------------------------------
// Raw codes of one producer unit: 4 view rows (consecutive channels) x NU
// consecutive batch items, plus the one or two E4M3 scales that cover them.
template <int FMT, int NU>
struct UnitRaw {
  uint32_t lo[4];
  uint32_t hi[4];          // FP6 with NU = 8: bytes 4-5 of each run
  uint32_t ss;             // scale byte(s)
  bool ok;
};

template <int FMT, int NU>
__device__ __forceinline__ void load_unit(const QView& v, int64_t row, int n, bool ok, UnitRaw<FMT, NU>& u) {
  u.ok = ok;
  if (!ok) return;
#pragma unroll
  for (int j = 0; j < 4; ++j) u.lo[j] = load_codes<FMT, NU>(v, row + j, n, u.hi[j]);
  const uint8_t* sp = v.scales + (row >> 2) * v.scale_cols + (n >> 2);
  u.ss = NU == 8 ? static_cast<uint32_t>(__ldg(reinterpret_cast<const unsigned short*>(sp))) : __ldg(sp);
}

// Dequantize a unit and store it: MN-major (the unit's NU batch items are
// consecutive MN rows of K column kl + j) or K-major (tile row r0 + j gets
// NU consecutive K values at kl).
template <int FMT, int NU, bool MN_MAJOR>
__device__ __forceinline__ void store_unit(const UnitRaw<FMT, NU>& u, uint32_t tile, uint32_t a, uint32_t kl) {
  const uint32_t s2lo = u.ok ? scale2(u.ss & 0xFF) : 0u;
  const uint32_t s2hi = (u.ok && NU == 8) ? scale2(u.ss >> 8) : 0u;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint32_t h[4] = {0u, 0u, 0u, 0u};
    if (u.ok) dequant_run<FMT, NU>(u.lo[j], u.hi[j], s2lo, s2hi, h);
    const uint32_t off = MN_MAJOR ? mn_offset(a, kl + j) : sw128_offset(a + j, kl);
    if (NU == 8) st_shared_v4(tile + off, h[0], h[1], h[2], h[3]);
    else st_shared_v2(tile + off, h[0], h[1]);
  }
}

// Forward / input-gradient B producer.
//
// K index k = (kh, kw, c) of the reduction decomposes the same way in every
// output tile, so each CTA tabulates it once per (K tile, channel quad):
// entry = (dh + 128) | (dw + 128) << 8 | c << 16 with (dh, dw) = (kh - pad,
// kw - pad) for the forward pass and (pad - kh, pad - kw) for the input
// gradient, or kKtabInvalid past the contraction.
template <int PASS>
__device__ __forceinline__ uint32_t ktab_entry(const V2Args& p, int kt, int kq) {
  const int k = kt * 64 + 4 * kq;
  if (k >= p.Kdim) return kKtabInvalid;
  const int tap = fdiv(k, p.dCred);
  const int c = k - tap * p.Cred;
  const int kh = fdiv(tap, p.dKw), kw = tap - kh * p.Kw;
  const int dh = PASS == kFwd ? kh - p.pad : p.pad - kh;
  const int dw = PASS == kFwd ? kw - p.pad : p.pad - kw;
  return static_cast<uint32_t>(dh + 128) | (static_cast<uint32_t>(dw + 128) << 8) |
         (static_cast<uint32_t>(c) << 16);
}

// Output-tile column of a producer thread: NU batch items of one pixel.
struct TileCol {
  int h, w;       // fwd: ho·s, wo·s;  dgrad: hi, wi
  int n;
  bool ok;
};

// Column `off` of column tile nt (off < BN).
template <int PASS, int BN, bool PH>
__device__ __forceinline__ TileCol tile_col(const V2Args& p, int nt, int off) {
  TileCol c;
  if (PH) {
    const int q = phase_of<PH>(p, nt);
    int pix;
    c.ok = col_pixel<PH>(p, q, static_cast<int64_t>(nt - p.ph_tile0[q]) * BN + off, pix, c.n);
    c.h = fdiv(pix, p.dW);
    c.w = pix - c.h * p.W;
    return c;
  }
  const int64_t col = static_cast<int64_t>(nt) * BN + off;
  c.ok = col < p.Ncols;
  const int c32 = c.ok ? static_cast<int>(col) : 0;
  const int pix = fdiv(c32, p.dN);
  c.n = c32 - pix * p.N;
  const int ph = fdiv(pix, PASS == kFwd ? p.dWo : p.dW);
  const int pw = pix - ph * (PASS == kFwd ? p.Wo : p.W);
  c.h = PASS == kFwd ? ph * p.stride : ph;
  c.w = PASS == kFwd ? pw * p.stride : pw;
  return c;
}

// Unit u of a K tile: column group g = u % G (NU batch items of one output
// pixel), channel quad kq = u / G.  Consecutive lanes take consecutive
// column groups, so the 4-byte code loads of a warp are contiguous and each
// 8-lane phase of a 16-byte shared store lands on 8 different swizzled chunks.
template <int PASS, int FMT, int BN, int NU>
struct FdProducer {
  static constexpr int G = BN / NU;
  static constexpr int UNITS = G * 16;
  static constexpr int PER = UNITS / kV2ProdThreads;
  static_assert(kV2ProdThreads % G == 0 && UNITS % kV2ProdThreads == 0, "producer mapping");
  UnitRaw<FMT, NU> raw[PER];

  __device__ __forceinline__ void load(const V2Args& p, const TileCol& tc, int kt, int t,
                                       const uint32_t* ktab) {
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int kq = t / G + (kV2ProdThreads / G) * i;
      const uint32_t e = ktab ? ktab[kt * 16 + kq] : ktab_entry<PASS>(p, kt, kq);
      bool ok = tc.ok && e != kKtabInvalid;
      const int dh = static_cast<int>(e & 0xFF) - 128, dw = static_cast<int>((e >> 8) & 0xFF) - 128;
      const int c = static_cast<int>(e >> 16);
      int pix = 0;
      if (PASS == kFwd) {
        const int sh = tc.h + dh, sw = tc.w + dw;
        ok = ok && sh >= 0 && sh < p.H && sw >= 0 && sw < p.W;
        pix = sh * p.W + sw;
      } else {
        const int th = tc.h + dh, tw = tc.w + dw;     // = hi + pad - kh, wi + pad - kw
        int sh = th, sw = tw;
        if (p.stride != 1) {
          sh = th >= 0 ? fdiv(th, p.dS) : -1;
          sw = tw >= 0 ? fdiv(tw, p.dS) : -1;
          ok = ok && sh * p.stride == th && sw * p.stride == tw;
        }
        ok = ok && sh >= 0 && sh < p.Ho && sw >= 0 && sw < p.Wo;
        pix = sh * p.Wo + sw;
      }
      load_unit<FMT, NU>(p.b, static_cast<int64_t>(pix) * p.Cred + c, tc.n, ok, raw[i]);
    }
  }

  __device__ __forceinline__ void store(uint32_t tile, int t) const {
    const int g = t % G;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int kq = t / G + (kV2ProdThreads / G) * i;
      store_unit<FMT, NU, true>(raw[i], tile, static_cast<uint32_t>(g * NU), static_cast<uint32_t>(4 * kq));
    }
  }
};

// Producer warps signal a filled stage once per warp: every lane makes its
// shared stores visible to the async proxy, the warp converges, lane 0 arrives.
__device__ __forceinline__ void producer_warp_arrive(uint64_t* bar) {
  fence_proxy_async_smem();
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

// Threads of conv_fd_kernel with GR producer groups.
__host__ __device__ constexpr int fd_threads(int gr) { return kV2ProdWarp0 * 32 + gr * kV2ProdThreads; }

// TR: transposed tiles (M <= 128 output channels as the MMA's N, BN = 128
// GEMM columns as its M); otherwise 128 output channels x BN columns.
// GR producer groups of 8 warps take turns: group g fills the K iterations
// g, g + GR, ... so that GR times as many gathers are in flight (GR = 2
// needs at most 88 registers a thread).
template <int PASS, int FMT, int BN, int NU, bool TR, int GR, bool PH>
__global__ void __launch_bounds__(fd_threads(GR), 1)
conv_fd_kernel(const __grid_constant__ V2Args p) {
  static_assert(!PH || PASS == kDgrad, "phase grouping is for the input gradient");
  static_assert(!TR || BN == 128, "transposed tiles are 128 GEMM columns");
  using L = V2Smem<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  V2Bars* bars = v2_setup<BN>(smem, kV2ProdThreads / 32 + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t sbase = smem_u32(smem);

  if (warp < kV2EpiWarps) {
    int it = 0;
    float amax = 0.f;
    for (int tile = blockIdx.x; tile < p.tiles; tile += gridDim.x, ++it) {
      const int acc = it & 1;
      mbar_wait_bounded(&bars->acc_full[acc], (it >> 1) & 1, p.err, kErrWaitDone);
      tc_fence_after();
      const int mt = tile / p.ntiles, nt = tile - mt * p.ntiles;
      const int q = phase_of<PH>(p, nt);
      const int64_t lcol0 = static_cast<int64_t>(nt - (PH ? p.ph_tile0[q] : 0)) * BN;
      const bool has_k = PH ? p.ph_nlive[q] > 0 : p.ktiles > 0;
      if (TR)
        v2_epilogue_tr<BN, PH>(p, bars, acc, lcol0, q, has_k, amax);
      else
        v2_epilogue<BN, true, PH>(p, bars, acc, static_cast<int64_t>(mt) * 128, lcol0, 0, has_k, amax, q);
    }
    epi_amax_flush(p.amax_out, amax);
  } else if (warp == kV2MmaWarp) {
    if (lane == 0) {
      // TR: the gathered MN-major tile is the A operand, the weight rows B
      const uint32_t idesc = TR ? idesc_f16_f32_amn(128, p.nc) : idesc_f16_f32_bmn(128, BN);
      int it = 0, kit = 0;
      for (int tile = blockIdx.x; tile < p.tiles; tile += gridDim.x, ++it) {
        const int acc = it & 1;
        mbar_wait_bounded(&bars->acc_empty[acc], ((it >> 1) & 1) ^ 1, p.err, kErrWaitEmpty);
        tc_fence_after();
        const uint32_t dt = bars->tmem + acc * BN;
        const int q = phase_of<PH>(p, tile % p.ntiles);
        uint32_t accum = 0;                    // 0 until the tile's first live K tile
        for (int kt = 0; kt < p.ktiles; ++kt) {
          if (!kt_live<PH>(p, q, kt)) continue;
          const int s = kit % kV2Stages;
          mbar_wait_bounded(&bars->full[s], (kit / kV2Stages) & 1, p.err, kErrWaitFull);
          tc_fence_after();
          const uint32_t a_tile = sbase + s * L::kStage;
          const uint64_t wdesc = smem_desc_sw128(a_tile);
          const uint64_t gdesc = smem_desc_sw128_mn(a_tile + kATileBytes, 8192, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            if (TR)
              mma_f16_ss(dt, gdesc + 128 * kk, wdesc + 2 * kk, idesc, (accum | kk) ? 1u : 0u);
            else
              mma_f16_ss(dt, wdesc + 2 * kk, gdesc + 128 * kk, idesc, (accum | kk) ? 1u : 0u);
          }
          accum = 1;
          mma_commit(&bars->empty[s]);
          ++kit;
        }
        mma_commit(&bars->acc_full[acc]);
      }
    }
  } else if (warp == kV2LoadWarp) {
    if (lane == 0) {
      int kit = 0;
      for (int tile = blockIdx.x; tile < p.tiles; tile += gridDim.x) {
        const int mt = tile / p.ntiles;
        const uint8_t* src = p.image + static_cast<int64_t>(mt) * p.ktiles * kATileBytes;
        // TR: only the first nc rows (128 B each) of a weight tile are used
        const uint32_t bytes = TR ? static_cast<uint32_t>(p.nc) * 128u : kATileBytes;
        const int q = phase_of<PH>(p, tile % p.ntiles);
        for (int kt = 0; kt < p.ktiles; ++kt) {
          if (!kt_live<PH>(p, q, kt)) continue;
          const int s = kit % kV2Stages;
          mbar_wait_bounded(&bars->empty[s], ((kit / kV2Stages) & 1) ^ 1, p.err, kErrWaitEmpty);
          mbar_arrive_expect_tx(&bars->full[s], bytes);
          bulk_copy_g2s(sbase + s * L::kStage, src + static_cast<int64_t>(kt) * kATileBytes, bytes,
                        &bars->full[s]);
          ++kit;
        }
      }
    }
  } else {
    // producers: the codes of stage i + kLookahead are requested right after
    // stage i is stored, so each load has kLookahead stages of work (and of
    // waiting for free stages) to arrive in.  The ring of raw registers is
    // indexed at compile time (unrolled by kLookahead).
    const int tg = threadIdx.x - kV2ProdWarp0 * 32;
    const int grp = tg / kV2ProdThreads;      // producer group
    const int t = tg - grp * kV2ProdThreads;
    // the CTA's K iterations: each of its tiles contributes its phase's live K tiles
    int total = p.ktiles * ((p.tiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                            static_cast<int>(gridDim.x));
    if (PH) {
      total = 0;
      for (int tile = blockIdx.x; tile < p.tiles; tile += gridDim.x) total += p.ph_nlive[phase_of<PH>(p, tile % p.ntiles)];
    }
    using Prod = FdProducer<PASS, FMT, BN, NU>;
    constexpr int kLookahead = Prod::PER >= 4 ? 2 : 3;      // keep the ring in registers
    Prod ring[kLookahead];
    // the CTA's K-tile table, built once by the producer warps
    uint32_t* ktab = nullptr;
    // phase grouping: the live K tiles of each phase, in order (built with the table)
    uint8_t* live = smem + L::kLiveOffset;
    if (p.ktiles * 16 <= kKtabEntries) {
      ktab = reinterpret_cast<uint32_t*>(smem + L::kKtabOffset);
      for (int e = tg; e < p.ktiles * 16; e += GR * kV2ProdThreads) ktab[e] = ktab_entry<PASS>(p, e >> 4, e & 15);
    }
    if (PH && tg < kMaxPhases) {
      int i = 0;
      for (int kt = 0; kt < p.ktiles; ++kt)
        if (kt_live<PH>(p, tg, kt)) live[tg * 256 + i++] = static_cast<uint8_t>(kt);
    }
    asm volatile("bar.sync 1, %0;" ::"n"(GR * kV2ProdThreads) : "memory");
    // load cursor: tile ltile, K tile lkt; with phases, lkt is entry li of
    // the phase's live list (tiles whose phase has none are passed over).
    int ltile = blockIdx.x, lkt = 0, li = 0, lq = 0;
    const int toff = (t % Prod::G) * NU;
    auto next_tile = [&]() {
      ltile += gridDim.x;
      if (PH) {
        while (ltile < p.tiles && p.ph_nlive[lq = phase_of<PH>(p, ltile % p.ntiles)] == 0) ltile += gridDim.x;
      }
    };
    if (PH) {
      lq = phase_of<PH>(p, ltile % p.ntiles);
      if (ltile < p.tiles && p.ph_nlive[lq] == 0) next_tile();
      lkt = live[lq * 256];
    }
    TileCol tc = tile_col<PASS, BN, PH>(p, ltile % p.ntiles, toff);
    auto step = [&]() {                        // one K iteration forward
      if (PH) {
        if (++li == p.ph_nlive[lq]) {
          li = 0;
          next_tile();
          tc = tile_col<PASS, BN, PH>(p, ltile % p.ntiles, toff);
        }
        lkt = live[lq * 256 + li];
      } else if (++lkt == p.ktiles) {
        lkt = 0;
        ltile += gridDim.x;
        tc = tile_col<PASS, BN, PH>(p, ltile % p.ntiles, toff);
      }
    };
    for (int g = 0; g < grp; ++g) step();     // this group's first K iteration
    auto load_next = [&](Prod& pr) {
      pr.load(p, tc, lkt, t, ktab);
#pragma unroll
      for (int g = 0; g < GR; ++g) step();
    };
#pragma unroll
    for (int r = 0; r < kLookahead; ++r)
      if (grp + r * GR < total) load_next(ring[r]);
    for (int kit = grp; kit < total;) {
#pragma unroll
      for (int r = 0; r < kLookahead; ++r, kit += GR) {
        if (kit >= total) break;
        const int s = kit % kV2Stages;
        mbar_wait_bounded(&bars->empty[s], ((kit / kV2Stages) & 1) ^ 1, p.err, kErrWaitEmpty);
        ring[r].store(sbase + s * L::kStage + kATileBytes, t);
        producer_warp_arrive(&bars->full[s]);
        if (kit + kLookahead * GR < total) load_next(ring[r]);
      }
    }
  }
  v2_teardown<BN>(bars);
}

// ---------------------------------------------------------------------------
// Weight-gradient producer: the K-major A (G_Y) and B (X') tiles of one K
// tile.  Unit = 4 view rows x NU consecutive batch items of one pixel; lane
// order runs along K first (KG units per tile row), so a warp reads
// contiguous code bytes of each row.
// Contraction position of a producer thread in the weight-gradient pass:
// q = kt·64 + kg·NU = (pixel, n); stepped from one K tile to the next without
// divisions (q grows by 64 per tile).
struct WgPos {
  int ho, wo, n;
  bool ok;
};

__device__ __forceinline__ WgPos wg_pos(const V2Args& p, int q) {
  WgPos w;
  w.ok = q < p.Kdim;
  const int qq = w.ok ? q : 0;
  const int pix = fdiv(qq, p.dN);
  w.n = qq - pix * p.N;
  w.ho = fdiv(pix, p.dWo);
  w.wo = pix - w.ho * p.Wo;
  return w;
}

__device__ __forceinline__ void wg_advance(const V2Args& p, WgPos& w, int q_next) {
  w.ok = q_next < p.Kdim;
  w.n += 64;
  while (w.n >= p.N) {
    w.n -= p.N;
    if (++w.wo == p.Wo) {
      w.wo = 0;
      ++w.ho;
    }
  }
}

// Weight-gradient producer: the K-major A (G_Y) and B (X') tiles of one K
// tile.  Unit = 4 view rows x NU consecutive batch items of one pixel; lane
// order runs along K first (KG units per tile row), so a warp reads
// contiguous code bytes of each row and every unit of a thread has the same
// contraction position.
template <int FMT, int NU, int ROWS>
struct WgOperand {
  static constexpr int KG = 64 / NU;
  static constexpr int UNITS = (ROWS / 4) * KG;
  static constexpr int PER = UNITS / kV2ProdThreads;
  static_assert(UNITS % kV2ProdThreads == 0 && kV2ProdThreads % KG == 0, "producer mapping");
  UnitRaw<FMT, NU> raw[PER];

  template <bool IS_A>
  __device__ __forceinline__ void load(const V2Args& p, const QView& v, int row_base, const WgPos& w, int t) {
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int u = t + kV2ProdThreads * i;
      const int rq = u / KG;
      const int r0 = row_base + 4 * rq;
      bool ok = w.ok;
      int64_t row = 0;
      if (IS_A) {
        ok = ok && r0 < p.M;
        row = static_cast<int64_t>(w.ho * p.Wo + w.wo) * p.Cout + r0;
      } else {
        ok = ok && r0 < p.Ncols;
        const int tap = fdiv(r0, p.dCin), ci = r0 - tap * p.Cin;
        const int kh = fdiv(tap, p.dKw), kw = tap - kh * p.Kw;
        const int hi = w.ho * p.stride + kh - p.pad, wi = w.wo * p.stride + kw - p.pad;
        ok = ok && hi >= 0 && hi < p.H && wi >= 0 && wi < p.W;
        row = (static_cast<int64_t>(hi) * p.W + wi) * p.Cin + ci;
      }
      load_unit<FMT, NU>(v, row, w.n, ok, raw[i]);
    }
  }

  __device__ __forceinline__ void store(uint32_t tile, int t) const {
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int u = t + kV2ProdThreads * i;
      const int kg = u % KG, rq = u / KG;
      store_unit<FMT, NU, false>(raw[i], tile, static_cast<uint32_t>(4 * rq), static_cast<uint32_t>(kg * NU));
    }
  }
};

template <int FMT, int BN, int NU>
struct WgProducer {
  WgOperand<FMT, NU, 128> a;
  WgOperand<FMT, NU, BN> b;
  static constexpr int PER = WgOperand<FMT, NU, 128>::PER + WgOperand<FMT, NU, BN>::PER;
  __device__ __forceinline__ void load(const V2Args& p, int mt, int nt, const WgPos& w, int t) {
    a.template load<true>(p, p.a, mt * 128, w, t);
    b.template load<false>(p, p.b, nt * BN, w, t);
  }
  __device__ __forceinline__ void store(uint32_t a_tile, int t) const {
    a.store(a_tile, t);
    b.store(a_tile + kATileBytes, t);
  }
};

template <int FMT, int BN, int NU>
__global__ void __launch_bounds__(kV2Threads, 1)
conv_wg_kernel(const V2Args p) {
  using L = V2Smem<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  V2Bars* bars = v2_setup<BN>(smem, kV2ProdThreads / 32);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t sbase = smem_u32(smem);

  auto decode = [&](int tile, int& mt, int& nt, int& sp) {
    sp = tile % p.splits;
    const int r = tile / p.splits;
    mt = r / p.ntiles;
    nt = r - mt * p.ntiles;
  };

  if (warp < kV2EpiWarps) {
    int it = 0;
    for (int tile = blockIdx.x; tile < p.tiles; tile += gridDim.x, ++it) {
      const int acc = it & 1;
      int mt, nt, sp;
      decode(tile, mt, nt, sp);
      const int kt0 = sp * p.kt_per_split;
      const bool has_k = min(p.ktiles, kt0 + p.kt_per_split) > kt0;
      mbar_wait_bounded(&bars->acc_full[acc], (it >> 1) & 1, p.err, kErrWaitDone);
      tc_fence_after();
      float unused = 0.f;
      v2_epilogue<BN, false>(p, bars, acc, static_cast<int64_t>(mt) * 128,
                             static_cast<int64_t>(nt) * BN, sp, has_k, unused);
    }
  } else if (warp == kV2MmaWarp) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(128, BN);
      int it = 0, kit = 0;
      for (int tile = blockIdx.x; tile < p.tiles; tile += gridDim.x, ++it) {
        int mt, nt, sp;
        decode(tile, mt, nt, sp);
        const int kt0 = sp * p.kt_per_split, kt1 = min(p.ktiles, kt0 + p.kt_per_split);
        const int acc = it & 1;
        mbar_wait_bounded(&bars->acc_empty[acc], ((it >> 1) & 1) ^ 1, p.err, kErrWaitEmpty);
        tc_fence_after();
        const uint32_t dt = bars->tmem + acc * BN;
        for (int kt = kt0; kt < kt1; ++kt, ++kit) {
          const int s = kit % kV2Stages;
          mbar_wait_bounded(&bars->full[s], (kit / kV2Stages) & 1, p.err, kErrWaitFull);
          tc_fence_after();
          const uint32_t a_tile = sbase + s * L::kStage;
          const uint64_t adesc = smem_desc_sw128(a_tile);
          const uint64_t bdesc = smem_desc_sw128(a_tile + kATileBytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f16_ss(dt, adesc + 2 * kk, bdesc + 2 * kk, idesc, (kt > kt0 || kk > 0) ? 1u : 0u);
          mma_commit(&bars->empty[s]);
        }
        mma_commit(&bars->acc_full[acc]);
      }
    }
  } else if (warp >= kV2ProdWarp0) {
    // producers with a kLookahead-deep load ring, as in conv_fd_kernel; the
    // load cursor walks this CTA's (tile, K tile) sequence, skipping tiles
    // with an empty K range (none with the host's split plan).
    const int t = threadIdx.x - kV2ProdWarp0 * 32;
    int total = 0;
    for (int tl = blockIdx.x; tl < p.tiles; tl += gridDim.x) {
      int m_, n_, s_;
      decode(tl, m_, n_, s_);
      const int k0 = s_ * p.kt_per_split;
      total += max(0, min(p.ktiles, k0 + p.kt_per_split) - k0);
    }
    using Prod = WgProducer<FMT, BN, NU>;
    constexpr int kLookahead = Prod::PER >= 4 ? 2 : 3;      // keep the ring in registers
    Prod ring[kLookahead];
    int ltile = blockIdx.x, lkt = 0, lkt1 = 0, lmt = 0, lnt = 0;
    auto seek = [&]() {                        // first tile at or after ltile with work
      while (ltile < p.tiles) {
        int sp_;
        decode(ltile, lmt, lnt, sp_);
        lkt = sp_ * p.kt_per_split;
        lkt1 = min(p.ktiles, lkt + p.kt_per_split);
        if (lkt < lkt1) return;
        ltile += gridDim.x;
      }
    };
    seek();
    const int kg_off = (t % WgOperand<FMT, NU, 128>::KG) * NU;   // this thread's K offset in a tile
    WgPos wpos = wg_pos(p, lkt * 64 + kg_off);
    auto load_next = [&](Prod& pr) {
      pr.load(p, lmt, lnt, wpos, t);
      if (++lkt == lkt1) {
        ltile += gridDim.x;
        seek();
        wpos = wg_pos(p, lkt * 64 + kg_off);
      } else {
        wg_advance(p, wpos, lkt * 64 + kg_off);
      }
    };
#pragma unroll
    for (int r = 0; r < kLookahead; ++r)
      if (r < total) load_next(ring[r]);
    for (int kit = 0; kit < total;) {
#pragma unroll
      for (int r = 0; r < kLookahead; ++r, ++kit) {
        if (kit >= total) break;
        const int s = kit % kV2Stages;
        mbar_wait_bounded(&bars->empty[s], ((kit / kV2Stages) & 1) ^ 1, p.err, kErrWaitEmpty);
        ring[r].store(sbase + s * L::kStage, t);
        producer_warp_arrive(&bars->full[s]);
        if (kit + kLookahead < total) load_next(ring[r]);
      }
    }
  }
  v2_teardown<BN>(bars);
}

}  // namespace mqv
