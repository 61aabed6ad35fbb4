// Quantize-once kernel pair: a global max|x| reduction, then the per-4x4
// square-block two-level quantizer (MicroQonv summary, onedev.kr/papers/182,
// section "무엇과 다른가": T_scale = max|X| / (max B_sf × max B_ef),
// B_scale = CastE4M3(max|X_i| / (T_scale × max B_ef)),
// X_i^q = Round(X_i / (B_scale × T_scale)); RNE for activations and weights,
// stochastic rounding for gradients; NVFP6 = E2M3 elements, section
// "어떻게 쓰나").  Every scale step is one IEEE fp32 operation in the order
// the formula is written; divisions are correctly rounded (__fdiv_rn).
#pragma once

#include <cstdint>

#include "mqv_ptx.cuh"

namespace mqv {

constexpr int kAmaxThreads = 256;
constexpr int kQuantThreads = 256;

// ---------------------------------------------------------------- Philox
// Philox4x32-10 (Salmon et al., SC'11): ten rounds of two 32x32->64-bit
// multiplies; round r XORs in the key (k0 + r·0x9E3779B9, k1 + r·0xBB67AE85),
// precomputed on the host from the seed so each round is two wide multiplies
// and two three-input XORs.
struct PhiloxKeys {
  uint32_t k0[10], k1[10];
};

__device__ __forceinline__ uint4 philox4x32_10(uint4 c, const PhiloxKeys& k) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint64_t p0 = static_cast<uint64_t>(c.x) * 0xD2511F53u;
    const uint64_t p1 = static_cast<uint64_t>(c.z) * 0xCD9E8D57u;
    c = make_uint4(static_cast<uint32_t>(p1 >> 32) ^ c.y ^ k.k0[r], static_cast<uint32_t>(p1),
                   static_cast<uint32_t>(p0 >> 32) ^ c.w ^ k.k1[r], static_cast<uint32_t>(p0));
  }
  return c;
}

// ------------------------------------------------- element rounding
// Round-to-nearest-even onto the element grid is the hardware conversion
// (cvt.rn.satfinite.e2m1x2 / e2m3x2, see mqv_ptx.cuh).
//
// Stochastic rounding reads the grid as a binary format: with
// E = floor(log2(max(a, 1))) the step on [2^E, 2^(E+1)) (and on [0, 1) for
// E = 0) is 2^(E-1) for E2M1 (0.5, 1, 2) and 2^(E-3) for E2M3 (1/8, 1/4,
// 1/2), and the magnitude code of the grid point at or below a is
// floor(q) + 2E (E2M1) or + 8E (E2M3), q = a / step (a power-of-two
// scaling, exact).  "Round up iff u < frac(q)", u = (w >> 8)·2^-24, gives
// floor(q) + [u < frac(q)] = ceil(q - u): q - u lies in (floor(q) - 1,
// floor(q) + 1) and exceeds floor(q) exactly when u < frac(q); a value on the
// grid (frac(q) = 0) stays.  ceil(q - u) takes two operations rounded toward
// +inf: z = RU(q - u), one FMA of the integer w >> 8 with -2^-24 (rounding
// upward never passes an integer, so ceil(z) = ceil(q - u)), then
// RU(z + 1.5·2^23), whose ulp is 1, so its low mantissa bits are ceil(z)
// for z in (-1, 2^22).  Codes past the largest saturate.
template <int FMT>
__device__ __forceinline__ void round_sr_mag2(float2 a, uint32_t w0, uint32_t w1, uint32_t& m0, uint32_t& m1) {
  constexpr uint32_t kInv = FMT == 0 ? 0x7F800000u : 0x80800000u;    // 1 / step = bits kInv - (127 + E) << 23
  constexpr uint32_t kTop = FMT == 0 ? 7u : 31u;
  const uint32_t e0 = max(__float_as_uint(a.x), 0x3F800000u) & 0x7F800000u;
  const uint32_t e1 = max(__float_as_uint(a.y), 0x3F800000u) & 0x7F800000u;
  const float2 q = __fmul2_rn(a, make_float2(__uint_as_float(kInv - e0), __uint_as_float(kInv - e1)));
  const float2 u = make_float2(__uint2float_rn(w0 >> 8), __uint2float_rn(w1 >> 8));
  const float2 z = __ffma2_ru(u, make_float2(-0x1p-24f, -0x1p-24f), q);
  const float2 t = __fadd2_ru(z, make_float2(12582912.0f, 12582912.0f));      // 1.5·2^23
  // ceil(q - u) + 2E (E2M1: (e >> 22) - 254) or + 8E (E2M3: (e >> 20) - 1016)
  constexpr uint32_t kBase = FMT == 0 ? 0x4B400000u + 254u : 0x4B400000u + 1016u;
  m0 = min(__float_as_uint(t.x) + (FMT == 0 ? e0 >> 22 : e0 >> 20) - kBase, kTop);
  m1 = min(__float_as_uint(t.y) + (FMT == 0 ? e1 >> 22 : e1 >> 20) - kBase, kTop);
}

// Correctly rounded a / d for the elements of a block, which share d, by
// Markstein's method (P. Markstein, "Computation of elementary functions on
// the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990; also
// Muller et al., Handbook of Floating-Point Arithmetic, 2nd ed., 2018,
// sec. 4.9): with y = RN(1/d) and q0 = RN(a·y) within one ulp of a/d, the
// remainder r = a - d·q0 is exact (one FMA) and RN(q0 + r·y) = RN(a/d).
// The theorem needs r to be representable.  For block divisors d >= 2^-64
// (kMarksteinMinDivisor) r is a multiple of at least 2^-140 for every
// quotient >= 2^-30, so the result is exact there; y <= 2^64 stays finite
// and, since d <= FLT_MAX / 6, normal.  Below 2^-30 only whether the
// quotient is zero decides a code (stochastic rounding compares 24-bit u
// against frac(q)): quotients below 1e-30 take the IEEE divide.  Blocks with
// smaller divisors (tensors with max|x| below about 1e-13) divide exactly
// throughout.  Two elements per step with the paired fp32 operations of
// sm_100 (each lane rounds as its scalar counterpart).
constexpr float kMarksteinMinDivisor = 5.42101086242752217e-20f;   // 2^-64

__device__ __forceinline__ float2 div2_shared_divisor(float2 a, float2 nd, float2 y, float2& q0) {
  q0 = __fmul2_rn(a, y);
  const float2 r = __ffma2_rn(nd, q0, a);
  return __ffma2_rn(r, y, q0);
}

__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
  return f16_lo_to_f32(e4m3x2_to_f16x2(code));
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// ------------------------------------------------------------- amax
// Pass 1: CTA `cta` of `nctas` writes max|x| over its grid-stride share of
// the n4 float4 of src to *partial.
__device__ __forceinline__ void amax_partial_body(const float4* __restrict__ src, int64_t n4,
                                                  float* __restrict__ partial, int cta, int nctas) {
  // chunks of kAmaxThreads x 8 float4, eight independent loads per thread
  constexpr int kPer = 8;
  float m = 0.0f;
  const int64_t chunk = static_cast<int64_t>(kAmaxThreads) * kPer;
  for (int64_t base = static_cast<int64_t>(cta) * chunk; base < n4; base += static_cast<int64_t>(nctas) * chunk) {
    float4 v[kPer];
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
      const int64_t i = base + k * kAmaxThreads + threadIdx.x;
      v[k] = i < n4 ? __ldg(src + i) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int k = 0; k < kPer; ++k)
      m = fmaxf(m, fmaxf(fmaxf(fabsf(v[k].x), fabsf(v[k].y)), fmaxf(fabsf(v[k].z), fabsf(v[k].w))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ float warp_max[kAmaxThreads / 32];
  if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    m = threadIdx.x < kAmaxThreads / 32 ? warp_max[threadIdx.x] : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (threadIdx.x == 0) *partial = m;
  }
}

__global__ void __launch_bounds__(kAmaxThreads)
amax_partial_kernel(const float4* __restrict__ src, int64_t n4, float* __restrict__ partial) {
  amax_partial_body(src, n4, partial + blockIdx.x, blockIdx.x, gridDim.x);
}

// Block-wide max over `count` floats (every thread gets the result).
__device__ __forceinline__ float block_max_of(const float* __restrict__ v, int count,
                                              float* red /* >= 32 floats smem */) {
  float m = 0.0f;
#pragma unroll 2
  for (int i = threadIdx.x; i < count; i += blockDim.x) m = fmaxf(m, v[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    m = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (threadIdx.x == 0) red[0] = m;
  }
  __syncthreads();
  const float r = red[0];
  __syncthreads();
  return r;
}

// Pass 1b (only for the split amax entry point): partials -> one float.
__global__ void __launch_bounds__(kAmaxThreads)
amax_finish_kernel(const float* __restrict__ partial, int count, float* __restrict__ amax) {
  __shared__ float red[32];
  const float m = block_max_of(partial, count, red);
  if (threadIdx.x == 0) *amax = m;
}

// ----------------------------------------------------------- quantize
// Each thread quantizes kQuantUnits 4 x 4 blocks (grid-stride, the next
// block's loads issued as soon as a block is done); consecutive threads take
// consecutive column blocks, so each of the 4 rows is read as one coalesced
// run.  `amax_src` holds `amax_count` partial maxima; every CTA reduces them.
// Stochastic rounding numbers element (r, c) as r·sr_cols + sr_col0 + c, so a
// column slice of a wider view (a batch shard) draws the words the whole
// view would (sr_cols = cols, sr_col0 = 0 for an unsharded tensor).
constexpr int kQuantUnits = 1;

// Scale constants of a tensor from its amax (every scale step one IEEE fp32
// operation in the formula's order).
template <int FMT>
struct TensorScale {
  float T, Temax;
  __device__ __forceinline__ explicit TensorScale(float amax) {
    const float emax = FMT == 0 ? 6.0f : 7.5f;
    T = __fdiv_rn(amax, 448.0f * emax);         // 2688 or 3360, exact
    Temax = __fmul_rn(T, emax);
  }
};

// Codes of one 4-element row of a block (element j at bits [j·b, j·b + b),
// b = 4 or 6), given the block divisor d = B·T, y = RN(1/d) (0 for a block
// whose scale is 0) and, for stochastic rounding, the row's Philox words.
template <int FMT, int RND>
__device__ __forceinline__ uint32_t quantize_row4(float4 x, float d, float y, bool exact, uint4 w) {
  const float2 nd = make_float2(-d, -d), y2 = make_float2(y, y);
  constexpr int kB = FMT == 0 ? 4 : 6;
  if (RND == 0) {
    // RNE: the conversion of the signed quotient gives sign bit and
    // magnitude together.  The quotient's sign is copied from x so that
    // zeros keep it (a block whose scale is 0 has y = 0: magnitude 0).
    float v[4];
    if (exact) {
      v[0] = __fdiv_rn(x.x, d); v[1] = __fdiv_rn(x.y, d); v[2] = __fdiv_rn(x.z, d); v[3] = __fdiv_rn(x.w, d);
    } else {
      float2 q0;
      const float2 v01 = div2_shared_divisor(make_float2(x.x, x.y), nd, y2, q0);
      const float2 v23 = div2_shared_divisor(make_float2(x.z, x.w), nd, y2, q0);
      v[0] = copysignf(v01.x, x.x); v[1] = copysignf(v01.y, x.y);
      v[2] = copysignf(v23.x, x.z); v[3] = copysignf(v23.y, x.w);
    }
    if (FMT == 0) return f32x2_to_e2m1x2(v[0], v[1]) | (f32x2_to_e2m1x2(v[2], v[3]) << 8);
    const uint32_t b01 = f32x2_to_e2m3x2(v[0], v[1]), b23 = f32x2_to_e2m3x2(v[2], v[3]);
    return (b01 & 0x3F) | ((b01 >> 2) & 0xFC0) | ((b23 & 0x3F) << 12) | ((b23 & 0x3F00) << 10);
  }
  const float2 a01 = make_float2(fabsf(x.x), fabsf(x.y)), a23 = make_float2(fabsf(x.z), fabsf(x.w));
  float2 v01, v23;
  if (exact) {
    v01 = make_float2(__fdiv_rn(a01.x, d), __fdiv_rn(a01.y, d));
    v23 = make_float2(__fdiv_rn(a23.x, d), __fdiv_rn(a23.y, d));
  } else {
    float2 q01, q23;
    v01 = div2_shared_divisor(a01, nd, y2, q01);
    v23 = div2_shared_divisor(a23, nd, y2, q23);
    if (fminf(fminf(q01.x, q01.y), fminf(q23.x, q23.y)) < 1.0e-30f && d > 0.0f) {
      // a quotient below 1e-30 (or a zero): the IEEE divide where it matters
      if (q01.x < 1.0e-30f && a01.x != 0.0f) v01.x = __fdiv_rn(a01.x, d);
      if (q01.y < 1.0e-30f && a01.y != 0.0f) v01.y = __fdiv_rn(a01.y, d);
      if (q23.x < 1.0e-30f && a23.x != 0.0f) v23.x = __fdiv_rn(a23.x, d);
      if (q23.y < 1.0e-30f && a23.y != 0.0f) v23.y = __fdiv_rn(a23.y, d);
    }
  }
  uint32_t m[4];
  round_sr_mag2<FMT>(v01, w.x, w.y, m[0], m[1]);
  round_sr_mag2<FMT>(v23, w.z, w.w, m[2], m[3]);
  const uint32_t sgn = (__float_as_uint(x.x) >> 31) | ((__float_as_uint(x.y) >> 31) << kB) |
                       ((__float_as_uint(x.z) >> 31) << (2 * kB)) | ((__float_as_uint(x.w) >> 31) << (3 * kB));
  return (m[0] | (m[1] << kB) | (m[2] << (2 * kB)) | (m[3] << (3 * kB))) | (sgn << (kB - 1));
}

// Per-tensor parameters of the quantize pass.
struct QuantArgs {
  const float* src;
  int64_t rows, cols;
  uint8_t* codes;
  uint8_t* scales;
  float* tscale;
  PhiloxKeys keys;
  int64_t sr_cols, sr_col0;
  FastDiv dcb;          // division by the column blocks of a block row (block count < 2^31)
  int32_t blocks;       // 0: 4 x 4 squares; 1: 1 x 16 along a row; 2: 16 x 1 down a column
};

// Block scale of a block with max|x| = bmax: the E4M3 code, the divisor
// d = B·T, y = RN(1/d) (0 where the Markstein quotient does not apply) and
// whether the block divides with the IEEE divide.
template <int FMT>
struct BlockScale {
  uint32_t scode;
  float d, y;
  bool exact;
  __device__ __forceinline__ BlockScale(float bmax, const TensorScale<FMT>& ts) {
    scode = 0;
    d = 0.0f;
    y = 0.0f;
    if (ts.T > 0.0f) {
      scode = f32_to_e4m3_satfinite(__fdiv_rn(bmax, ts.Temax));
      d = __fmul_rn(e4m3_to_f32(scode), ts.T);
      y = d >= kMarksteinMinDivisor ? __frcp_rn(d) : 0.0f;
    }
    exact = d > 0.0f && d < kMarksteinMinDivisor;
  }
};

__device__ __forceinline__ float absmax4(float4 v) {
  return fmaxf(max3f(fabsf(v.x), fabsf(v.y), fabsf(v.z)), fabsf(v.w));
}

// Quantize the 4 x 4 block (br, bc) whose 4 rows are x[r], and store its
// scale and codes.
template <int FMT, int RND>
__device__ __forceinline__ void quantize_block(const float4 (&x)[4], const TensorScale<FMT>& ts, const QuantArgs& qa,
                                               int64_t br, int64_t bc, int64_t cb, int64_t row_bytes) {
  float bmax = max3f(fabsf(x[0].x), fabsf(x[0].y), fabsf(x[0].z));
  bmax = max3f(bmax, fabsf(x[0].w), fabsf(x[1].x));
  bmax = max3f(bmax, fabsf(x[1].y), fabsf(x[1].z));
  float b2 = max3f(fabsf(x[1].w), fabsf(x[2].x), fabsf(x[2].y));
  b2 = max3f(b2, fabsf(x[2].z), fabsf(x[2].w));
  float b3 = max3f(fabsf(x[3].x), fabsf(x[3].y), fabsf(x[3].z));
  bmax = max3f(bmax, b2, fmaxf(b3, fabsf(x[3].w)));
  const BlockScale<FMT> bs(bmax, ts);
  const uint32_t scode = bs.scode;
  const float d = bs.d, y = bs.y;
  const bool exact = bs.exact;
  qa.scales[br * cb + bc] = static_cast<uint8_t>(scode);
  // Philox counter of row r: (element index of its first element) / 4
  uint64_t g = 0, gstep = 0;
  if (RND == 1) {
    g = static_cast<uint64_t>(br * 4 * qa.sr_cols + qa.sr_col0 + bc * 4) >> 2;
    gstep = static_cast<uint64_t>(qa.sr_cols) >> 2;
  }
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    uint4 wd = make_uint4(0u, 0u, 0u, 0u);
    if (RND == 1) {
      wd = philox4x32_10(make_uint4(static_cast<uint32_t>(g), static_cast<uint32_t>(g >> 32), 0u, 0u), qa.keys);
      g += gstep;
    }
    const uint32_t packed = quantize_row4<FMT, RND>(x[r], d, y, exact, wd);
    uint8_t* out = qa.codes + (br * 4 + r) * row_bytes;
    if (FMT == 0) {
      *reinterpret_cast<uint16_t*>(out + bc * 2) = static_cast<uint16_t>(packed);
    } else {
      out += bc * 3;
      out[0] = static_cast<uint8_t>(packed);
      out[1] = static_cast<uint8_t>(packed >> 8);
      out[2] = static_cast<uint8_t>(packed >> 16);
    }
  }
}

__device__ __forceinline__ void load_block(float4 (&x)[4], const float* __restrict__ src, int64_t cols, int64_t br,
                                           int64_t bc) {
  const float* p = src + br * 4 * cols + bc * 4;
#pragma unroll
  for (int r = 0; r < 4; ++r) x[r] = __ldg(reinterpret_cast<const float4*>(p + r * cols));
}

template <int FMT, int RND>
__device__ __forceinline__ void quantize_body(const QuantArgs& qa, const float* __restrict__ amax_src, int amax_count,
                                              int cta, int nctas) {
  const int64_t cols = qa.cols;
  const int64_t cb = cols >> 2;                       // column blocks per block row
  const int nunits = static_cast<int>((qa.rows >> 2) * cb);
  const int64_t row_bytes = FMT == 0 ? (cols >> 1) : (cols * 3) >> 2;
  const int nthr = nctas * kQuantThreads;
  const int w0 = cta * kQuantThreads + static_cast<int>(threadIdx.x);

  // The first blocks' loads do not depend on the tensor scale: issue them
  // before the reduction of the amax partials, so the two latencies overlap.
  float4 x[kQuantUnits][4];
#pragma unroll
  for (int i = 0; i < kQuantUnits; ++i) {
    const int w = w0 + i * nthr;
    if (w < nunits) {
      const int br = fdiv(w, qa.dcb);
      load_block(x[i], qa.src, cols, br, w - static_cast<int64_t>(br) * cb);
    }
  }
  // launched as a programmatic dependent of the max pass (quantize_many),
  // the amax partials are complete only after this wait; otherwise a no-op
  pdl_wait_prerequisite();
  __shared__ float red[32];
  const TensorScale<FMT> ts(block_max_of(amax_src, amax_count, red));
  if (cta == 0 && threadIdx.x == 0) *qa.tscale = ts.T;

  for (int w = w0; w < nunits; w += kQuantUnits * nthr) {
#pragma unroll
    for (int i = 0; i < kQuantUnits; ++i) {
      const int wi = w + i * nthr;
      if (wi < nunits) {
        const int br = fdiv(wi, qa.dcb);
        quantize_block<FMT, RND>(x[i], ts, qa, br, wi - static_cast<int64_t>(br) * cb, cb, row_bytes);
        const int wn = wi + kQuantUnits * nthr;
        if (wn < nunits) {
          const int bn = fdiv(wn, qa.dcb);
          load_block(x[i], qa.src, cols, bn, wn - static_cast<int64_t>(bn) * cb);
        }
      }
    }
  }
}

template <int FMT, int RND>
__global__ void __launch_bounds__(kQuantThreads)
quantize_kernel(const __grid_constant__ QuantArgs qa, const float* __restrict__ amax_src, int amax_count) {
  quantize_body<FMT, RND>(qa, amax_src, amax_count, blockIdx.x, gridDim.x);
}

// ------------------------------------------- 16-element line blocks
// The plain blocks of the scheme MicroQonv is set against (MicroQonv
// summary, section "무엇인가"): 16 consecutive elements along one axis of
// the view.  Every per-element step is the square quantizer's (T, the E4M3
// block scale, the divisor B·T, the division, both roundings and the
// element numbering of stochastic rounding); only the grouping differs.
//   1 x 16: one unit is one block, 16 consecutive columns of a row, scale
//           plane [rows][cols/16];
//   16 x 1: one unit is 16 rows x 4 columns, four blocks side by side (so
//           that each row's 4 codes are one packed store), scale plane
//           [rows/16][cols].

// Codes of 4 consecutive elements of a row that lie in 4 different blocks
// (divisors d.x .. d.w): quantize_row4 with a divisor per element.
template <int FMT, int RND>
__device__ __forceinline__ uint32_t quantize_row4_cols(float4 x, float4 d, float4 y, uint4 w) {
  constexpr int kB = FMT == 0 ? 4 : 6;
  const float xs[4] = {x.x, x.y, x.z, x.w}, ds[4] = {d.x, d.y, d.z, d.w};
  const float2 nd01 = make_float2(-d.x, -d.y), nd23 = make_float2(-d.z, -d.w);
  const float2 y01 = make_float2(y.x, y.y), y23 = make_float2(y.z, y.w);
  float a[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) a[j] = fabsf(xs[j]);
  float2 q01, q23;
  const float2 v01 = div2_shared_divisor(make_float2(a[0], a[1]), nd01, y01, q01);
  const float2 v23 = div2_shared_divisor(make_float2(a[2], a[3]), nd23, y23, q23);
  float v[4] = {v01.x, v01.y, v23.x, v23.y};
  const float q0[4] = {q01.x, q01.y, q23.x, q23.y};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    // the IEEE divide for blocks below the Markstein range, and (stochastic
    // rounding) for quotients below 1e-30, exactly as the square blocks
    const bool exact = ds[j] > 0.0f && ds[j] < kMarksteinMinDivisor;
    const bool tiny = RND == 1 && ds[j] > 0.0f && q0[j] < 1.0e-30f && a[j] != 0.0f;
    if (exact || tiny) v[j] = __fdiv_rn(a[j], ds[j]);
    if (ds[j] == 0.0f) v[j] = 0.0f;
  }
  if (RND == 0) {
#pragma unroll
    for (int j = 0; j < 4; ++j) v[j] = copysignf(v[j], xs[j]);
    if (FMT == 0) return f32x2_to_e2m1x2(v[0], v[1]) | (f32x2_to_e2m1x2(v[2], v[3]) << 8);
    const uint32_t b01 = f32x2_to_e2m3x2(v[0], v[1]), b23 = f32x2_to_e2m3x2(v[2], v[3]);
    return (b01 & 0x3F) | ((b01 >> 2) & 0xFC0) | ((b23 & 0x3F) << 12) | ((b23 & 0x3F00) << 10);
  }
  uint32_t m[4];
  round_sr_mag2<FMT>(make_float2(v[0], v[1]), w.x, w.y, m[0], m[1]);
  round_sr_mag2<FMT>(make_float2(v[2], v[3]), w.z, w.w, m[2], m[3]);
  uint32_t out = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) out |= (m[j] | ((__float_as_uint(xs[j]) >> 31) << (kB - 1))) << (j * kB);
  return out;
}

__device__ __forceinline__ uint4 philox_at(const QuantArgs& qa, uint64_t g) {
  return philox4x32_10(make_uint4(static_cast<uint32_t>(g), static_cast<uint32_t>(g >> 32), 0u, 0u), qa.keys);
}

template <int FMT, int RND>
__device__ __forceinline__ void quantize_unit_1x16(const QuantArgs& qa, const TensorScale<FMT>& ts, int64_t r,
                                                   int64_t c16, int64_t row_bytes) {
  const float* src = qa.src + r * qa.cols + c16 * 16;
  float4 x[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) x[j] = __ldg(reinterpret_cast<const float4*>(src) + j);
  const float bmax = fmaxf(fmaxf(absmax4(x[0]), absmax4(x[1])), fmaxf(absmax4(x[2]), absmax4(x[3])));
  const BlockScale<FMT> bs(bmax, ts);
  qa.scales[r * (qa.cols >> 4) + c16] = static_cast<uint8_t>(bs.scode);
  const uint64_t g = static_cast<uint64_t>(r * qa.sr_cols + qa.sr_col0 + c16 * 16) >> 2;
  uint32_t pk[4];
#pragma unroll
  for (int j = 0; j < 4; ++j)
    pk[j] = quantize_row4<FMT, RND>(x[j], bs.d, bs.y, bs.exact, RND == 1 ? philox_at(qa, g + j) : make_uint4(0, 0, 0, 0));
  uint8_t* out = qa.codes + r * row_bytes;
  if (FMT == 0) {
    *reinterpret_cast<uint2*>(out + c16 * 8) = make_uint2(pk[0] | (pk[1] << 16), pk[2] | (pk[3] << 16));
  } else {
    uint32_t* o = reinterpret_cast<uint32_t*>(out + c16 * 12);
    o[0] = pk[0] | (pk[1] << 24);
    o[1] = (pk[1] >> 8) | (pk[2] << 16);
    o[2] = (pk[2] >> 16) | (pk[3] << 8);
  }
}

template <int FMT, int RND>
__device__ __forceinline__ void quantize_unit_16x1(const QuantArgs& qa, const TensorScale<FMT>& ts, int64_t rb,
                                                   int64_t cq, int64_t row_bytes) {
  const float* src = qa.src + rb * 16 * qa.cols + cq * 4;
  float4 x[16];
#pragma unroll
  for (int r = 0; r < 16; ++r) x[r] = __ldg(reinterpret_cast<const float4*>(src + r * qa.cols));
  float4 m = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
  for (int r = 0; r < 16; ++r) {
    m.x = fmaxf(m.x, fabsf(x[r].x)); m.y = fmaxf(m.y, fabsf(x[r].y));
    m.z = fmaxf(m.z, fabsf(x[r].z)); m.w = fmaxf(m.w, fabsf(x[r].w));
  }
  const BlockScale<FMT> b0(m.x, ts), b1(m.y, ts), b2(m.z, ts), b3(m.w, ts);
  *reinterpret_cast<uint32_t*>(qa.scales + rb * qa.cols + cq * 4) =
      b0.scode | (b1.scode << 8) | (b2.scode << 16) | (b3.scode << 24);
  const float4 d = make_float4(b0.d, b1.d, b2.d, b3.d), y = make_float4(b0.y, b1.y, b2.y, b3.y);
#pragma unroll
  for (int r = 0; r < 16; ++r) {
    const int64_t row = rb * 16 + r;
    uint4 w = make_uint4(0, 0, 0, 0);
    if (RND == 1) w = philox_at(qa, static_cast<uint64_t>(row * qa.sr_cols + qa.sr_col0 + cq * 4) >> 2);
    const uint32_t packed = quantize_row4_cols<FMT, RND>(x[r], d, y, w);
    uint8_t* out = qa.codes + row * row_bytes;
    if (FMT == 0) {
      *reinterpret_cast<uint16_t*>(out + cq * 2) = static_cast<uint16_t>(packed);
    } else {
      out += cq * 3;
      out[0] = static_cast<uint8_t>(packed);
      out[1] = static_cast<uint8_t>(packed >> 8);
      out[2] = static_cast<uint8_t>(packed >> 16);
    }
  }
}

template <int FMT, int RND>
__device__ __forceinline__ void quantize_line_body(const QuantArgs& qa, const float* __restrict__ amax_src,
                                                   int amax_count, int cta, int nctas) {
  __shared__ float red[32];
  const TensorScale<FMT> ts(block_max_of(amax_src, amax_count, red));
  if (cta == 0 && threadIdx.x == 0) *qa.tscale = ts.T;
  const int64_t row_bytes = FMT == 0 ? (qa.cols >> 1) : (qa.cols * 3) >> 2;
  const int64_t per_row = qa.blocks == 1 ? qa.cols >> 4 : qa.cols >> 2;
  const int64_t units = qa.blocks == 1 ? qa.rows * per_row : (qa.rows >> 4) * per_row;
  const int64_t nthr = static_cast<int64_t>(nctas) * kQuantThreads;
  for (int64_t u = static_cast<int64_t>(cta) * kQuantThreads + threadIdx.x; u < units; u += nthr) {
    const int64_t a = u / per_row, b = u - a * per_row;
    if (qa.blocks == 1) quantize_unit_1x16<FMT, RND>(qa, ts, a, b, row_bytes);
    else quantize_unit_16x1<FMT, RND>(qa, ts, a, b, row_bytes);
  }
}

// ------------------------------------------------ several tensors at once
// The quantize-once step of a layer (X, W, G_Y) in two launches instead of
// six: every CTA of a launch serves one tensor ("job"), CTAs are assigned to
// jobs in contiguous ranges.  In the quantize launch the stochastic-rounding
// jobs take the first ranges: their CTAs are bound by arithmetic and start
// first, while the memory-bound round-to-nearest CTAs fill the SMs around
// them.  Results are bit-identical to one amax_partial_kernel +
// quantize_kernel pair per tensor with the same CTA counts.
constexpr int kMaxQuantJobs = 8;

struct QuantJob {
  QuantArgs qa;
  int32_t fmt, rounding;
  int32_t amax_cta0, amax_ctas;     // this job's range of amax CTAs (= its partials)
  int32_t quant_cta0, quant_ctas;   // this job's range of quantize CTAs
};

struct QuantJobs {
  QuantJob job[kMaxQuantJobs];
  int32_t count;
};

__device__ __forceinline__ int job_of(const QuantJobs& jobs, int cta, bool quant) {
  int j = 0;
  for (int i = 0; i < jobs.count; ++i) {
    const int c0 = quant ? jobs.job[i].quant_cta0 : jobs.job[i].amax_cta0;
    const int n = quant ? jobs.job[i].quant_ctas : jobs.job[i].amax_ctas;
    if (cta >= c0 && cta < c0 + n) j = i;
  }
  return j;
}

__global__ void __launch_bounds__(kAmaxThreads)
amax_many_kernel(const __grid_constant__ QuantJobs jobs, float* __restrict__ partial) {
  // the quantizer that follows may start now: it loads its first blocks and
  // then waits for this grid (pdl_wait_prerequisite) before reading `partial`
  pdl_launch_dependents();
  const QuantJob& jb = jobs.job[job_of(jobs, blockIdx.x, false)];
  amax_partial_body(reinterpret_cast<const float4*>(jb.qa.src), jb.qa.rows * jb.qa.cols / 4, partial + blockIdx.x,
                    blockIdx.x - jb.amax_cta0, jb.amax_ctas);
}

__global__ void __launch_bounds__(kQuantThreads)
quantize_many_kernel(const __grid_constant__ QuantJobs jobs, const float* __restrict__ partial) {
  const QuantJob& jb = jobs.job[job_of(jobs, blockIdx.x, true)];
  const int cta = blockIdx.x - jb.quant_cta0;
  const float* amax = partial + jb.amax_cta0;
#define MQV_QUANT_CASE(F, R)                                                                      \
  if (jb.fmt == F && jb.rounding == R) {                                                          \
    quantize_body<F, R>(jb.qa, amax, jb.amax_ctas, cta, jb.quant_ctas);                            \
    return;                                                                                       \
  }
  MQV_QUANT_CASE(0, 0) MQV_QUANT_CASE(0, 1) MQV_QUANT_CASE(1, 0) MQV_QUANT_CASE(1, 1)
#undef MQV_QUANT_CASE
}

// The same for calls whose jobs all use line blocks (a separate kernel, so
// the square quantizer keeps its own register budget).
__global__ void __launch_bounds__(kQuantThreads)
quantize_many_line_kernel(const __grid_constant__ QuantJobs jobs, const float* __restrict__ partial) {
  const QuantJob& jb = jobs.job[job_of(jobs, blockIdx.x, true)];
  const int cta = blockIdx.x - jb.quant_cta0;
  const float* amax = partial + jb.amax_cta0;
#define MQV_QUANT_CASE(F, R)                                                     \
  if (jb.fmt == F && jb.rounding == R) {                                         \
    quantize_line_body<F, R>(jb.qa, amax, jb.amax_ctas, cta, jb.quant_ctas);     \
    return;                                                                      \
  }
  MQV_QUANT_CASE(0, 0) MQV_QUANT_CASE(0, 1) MQV_QUANT_CASE(1, 0) MQV_QUANT_CASE(1, 1)
#undef MQV_QUANT_CASE
}

// ---------------------------------------------------------- dequantize
// dst = (code·B in fp16, exact) · T, one thread per 4 x 4 piece of the
// view; `blocks` as QuantArgs::blocks (each piece lies in one square, in
// 4 line blocks of 1 x 16, one per row, or in 4 of 16 x 1, one per column).
template <int FMT>
__global__ void __launch_bounds__(kQuantThreads)
dequantize_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                  const float* __restrict__ tscale, int64_t rows, int64_t cols, int blocks,
                  float* __restrict__ dst) {
  const float T = *tscale;
  const int64_t cb = cols >> 2;
  const int64_t nblocks = (rows >> 2) * cb;
  const int64_t row_bytes = FMT == 0 ? (cols >> 1) : (cols * 3) >> 2;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kQuantThreads;
  for (int64_t b = static_cast<int64_t>(blockIdx.x) * kQuantThreads + threadIdx.x; b < nblocks;
       b += stride) {
    const int64_t br = b / cb, bc = b - br * cb;
    uint32_t s01 = 0, s23 = 0;
    if (blocks == 0) {
      const uint32_t s = scales[b];
      s01 = s23 = e4m3x2_to_f16x2(s | (s << 8));
    } else if (blocks == 2) {
      const uint32_t s = *reinterpret_cast<const uint32_t*>(scales + (br >> 2) * cols + bc * 4);
      s01 = e4m3x2_to_f16x2(s & 0xFFFF);
      s23 = e4m3x2_to_f16x2(s >> 16);
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      if (blocks == 1) {
        const uint32_t s = scales[(br * 4 + r) * (cols >> 4) + (bc >> 2)];
        s01 = s23 = e4m3x2_to_f16x2(s | (s << 8));
      }
      const uint8_t* in = codes + (br * 4 + r) * row_bytes;
      uint32_t h01, h23;
      if (FMT == 0) {
        const uint32_t q = *reinterpret_cast<const uint16_t*>(in + bc * 2);
        h01 = e2m1x2_to_f16x2(q & 0xFF);
        h23 = e2m1x2_to_f16x2(q >> 8);
      } else {
        in += bc * 3;
        const uint32_t q = in[0] | (in[1] << 8) | (in[2] << 16);
        h01 = e2m3x2_to_f16x2((q & 0x3F) | ((q << 2) & 0x3F00));
        h23 = e2m3x2_to_f16x2(((q >> 12) & 0x3F) | ((q >> 10) & 0x3F00));
      }
      h01 = hmul2_u32(h01, s01);
      h23 = hmul2_u32(h23, s23);
      float4 o;
      o.x = __fmul_rn(f16_lo_to_f32(h01), T);
      o.y = __fmul_rn(f16_hi_to_f32(h01), T);
      o.z = __fmul_rn(f16_lo_to_f32(h23), T);
      o.w = __fmul_rn(f16_hi_to_f32(h23), T);
      *reinterpret_cast<float4*>(dst + (br * 4 + r) * cols + bc * 4) = o;
    }
  }
}

}  // namespace mqv
