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

// ------------------------------------------------- element rounding (a >= 0)
// Round-to-nearest-even onto the element grid is the hardware conversion
// (cvt.rn.satfinite.e2m1x2 / e2m3x2, see mqv_ptx.cuh).  For stochastic
// rounding the grid is read as a binary format: with E = floor(log2(max(a, 1)))
// the step on [2^E, 2^(E+1)) (and on [0, 1) for E = 0) is 2^(E-1) for E2M1
// (0.5, 1, 2) and 2^(E-3) for E2M3 (1/8, 1/4, 1/2), and the magnitude code
// below a is floor(a / step) + 2E (E2M1) or + 8E (E2M3).  q = a / step is a
// power-of-two scaling and frac(q) = q - floor(q) is exact, so "round up
// iff u < frac(q)" is decided exactly.  floor(q) comes from one add rounded
// toward -inf onto 2^23 (the integer lands in the low mantissa bits), which
// keeps the conversion pipe free; codes past the largest saturate.
template <int FMT>
__device__ __forceinline__ uint32_t round_sr_mag(float a, float u) {
  const uint32_t eb = __float_as_uint(fmaxf(a, 1.0f)) & 0x7F800000u;             // (127 + E) << 23
  const float inv = __uint_as_float((FMT == 0 ? 0x7F800000u : 0x80800000u) - eb);  // 1 / step
  const float q = __fmul_rn(a, inv);
  const float t = __fadd_rd(q, 8388608.0f);                                        // 2^23 + floor(q)
  const float f = __fsub_rn(q, __fsub_rn(t, 8388608.0f));
  const uint32_t piece = FMT == 0 ? (eb >> 22) - 254u : (eb >> 20) - 1016u;      // 2E or 8E
  const uint32_t mag = (__float_as_uint(t) - 0x4B000000u) + piece + (u < f ? 1u : 0u);
  return min(mag, FMT == 0 ? 7u : 31u);
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
// throughout.
constexpr float kMarksteinMinDivisor = 5.42101086242752217e-20f;   // 2^-64

__device__ __forceinline__ float div_shared_divisor(float a, float d, float y) {
  const float q0 = __fmul_rn(a, y);
  const float r = __fmaf_rn(-d, q0, a);
  const float q1 = __fmaf_rn(r, y, q0);
  return (q0 >= 1.0e-30f || a == 0.0f) ? q1 : __fdiv_rn(a, d);
}

// Round-to-nearest-even codes need the quotient only where it can reach a
// grid midpoint (>= 1/16), so the tiny-quotient check is dropped; the sign
// is the sign of a in every case (also for y = 0, the zero-scale block,
// where the magnitude comes out 0).
__device__ __forceinline__ float div_shared_divisor_rne(float a, float d, float y) {
  const float q0 = __fmul_rn(a, y);
  const float r = __fmaf_rn(-d, q0, a);
  return copysignf(__fmaf_rn(r, y, q0), a);
}

__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
  return f16_lo_to_f32(e4m3x2_to_f16x2(code));
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
// One thread per QB horizontally adjacent 4 x 4 blocks of the rows x cols
// view (QB = 2 when the view has an even number of column blocks, so each
// thread keeps eight float4 loads in flight and stores 32-bit code words);
// consecutive threads take consecutive column blocks, so each of the 4 rows
// is read as one coalesced run.  `amax_src` holds `amax_count` partial
// maxima; every CTA reduces them.  Stochastic rounding numbers element
// (r, c) as r·sr_cols + sr_col0 + c, so a column slice of a wider view (a
// batch shard) draws the words the whole view would (sr_cols = cols,
// sr_col0 = 0 for an unsharded tensor).
template <int FMT, int RND>
__device__ __forceinline__ uint32_t quantize_row4(const float (&xv)[4], float d, float y, bool exact,
                                                  const float (&u)[4]) {
  if (RND == 0) {
    // RNE: the conversion of the signed quotient gives sign bit and
    // magnitude together (the sign of x, also for a zero quotient; a block
    // whose scale is 0 has y = 0 and gets magnitude 0)
    float v[4];
    if (exact) {
#pragma unroll
      for (int j = 0; j < 4; ++j) v[j] = __fdiv_rn(xv[j], d);
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) v[j] = div_shared_divisor_rne(xv[j], d, y);
    }
    if (FMT == 0) return f32x2_to_e2m1x2(v[0], v[1]) | (f32x2_to_e2m1x2(v[2], v[3]) << 8);
    const uint32_t b01 = f32x2_to_e2m3x2(v[0], v[1]), b23 = f32x2_to_e2m3x2(v[2], v[3]);
    return (b01 & 0x3F) | ((b01 >> 2) & 0xFC0) | ((b23 & 0x3F) << 12) | ((b23 & 0x3F00) << 10);
  }
  uint32_t packed = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float v = d > 0.0f ? (exact ? __fdiv_rn(fabsf(xv[j]), d) : div_shared_divisor(fabsf(xv[j]), d, y)) : 0.0f;
    const uint32_t mag = round_sr_mag<FMT>(v, u[j]);
    const uint32_t sgn = __float_as_uint(xv[j]) >> 31;
    const uint32_t code = FMT == 0 ? (mag | (sgn << 3)) : (mag | (sgn << 5));
    packed |= code << (j * (FMT == 0 ? 4 : 6));
  }
  return packed;
}

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

// Quantize QB horizontally adjacent 4 x 4 blocks (block row br, first column
// block bc0) whose 4 rows are x[q][r], and store their scales and codes.
template <int FMT, int RND, int QB>
__device__ __forceinline__ void quantize_unit(const float4 (&x)[QB][4], const TensorScale<FMT>& ts, int64_t br,
                                              int64_t bc0, int64_t cb, int64_t row_bytes, const PhiloxKeys& keys,
                                              int64_t sr_cols, int64_t sr_col0,
                                              uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
  const float T = ts.T;
  uint32_t scode[QB];
  float d[QB], y[QB];
  bool exact[QB];
#pragma unroll
  for (int q = 0; q < QB; ++q) {
    float bmax = 0.0f;
#pragma unroll
    for (int r = 0; r < 4; ++r)
      bmax = fmaxf(bmax, fmaxf(fmaxf(fabsf(x[q][r].x), fabsf(x[q][r].y)),
                               fmaxf(fabsf(x[q][r].z), fabsf(x[q][r].w))));
    scode[q] = 0;
    d[q] = 0.0f;
    y[q] = 0.0f;
    if (T > 0.0f) {
      scode[q] = f32_to_e4m3_satfinite(__fdiv_rn(bmax, ts.Temax));
      d[q] = __fmul_rn(e4m3_to_f32(scode[q]), T);
      y[q] = d[q] >= kMarksteinMinDivisor ? __frcp_rn(d[q]) : 0.0f;
    }
    exact[q] = d[q] > 0.0f && d[q] < kMarksteinMinDivisor;
  }
  const int64_t b = br * cb + bc0;
  if (QB == 2) *reinterpret_cast<uint16_t*>(scales + b) = static_cast<uint16_t>(scode[0] | (scode[1] << 8));
  else scales[b] = static_cast<uint8_t>(scode[0]);

#pragma unroll
  for (int r = 0; r < 4; ++r) {
    uint32_t packed[QB];
#pragma unroll
    for (int q = 0; q < QB; ++q) {
      const float xv[4] = {x[q][r].x, x[q][r].y, x[q][r].z, x[q][r].w};
      float u[4] = {0.f, 0.f, 0.f, 0.f};
      if (RND == 1) {
        // element index in the (possibly wider) view the SR stream is defined on
        const uint64_t g = static_cast<uint64_t>((br * 4 + r) * sr_cols + sr_col0 + (bc0 + q) * 4) >> 2;
        const uint4 wd = philox4x32_10(make_uint4(static_cast<uint32_t>(g), static_cast<uint32_t>(g >> 32), 0u, 0u), keys);
        const float s24 = 5.9604644775390625e-08f;   // 2^-24
        u[0] = __uint2float_rn(wd.x >> 8) * s24;
        u[1] = __uint2float_rn(wd.y >> 8) * s24;
        u[2] = __uint2float_rn(wd.z >> 8) * s24;
        u[3] = __uint2float_rn(wd.w >> 8) * s24;
      }
      packed[q] = quantize_row4<FMT, RND>(xv, d[q], y[q], exact[q], u);
    }
    uint8_t* out = codes + (br * 4 + r) * row_bytes;
    if (FMT == 0) {
      if (QB == 2) *reinterpret_cast<uint32_t*>(out + bc0 * 2) = packed[0] | (packed[1] << 16);
      else *reinterpret_cast<uint16_t*>(out + bc0 * 2) = static_cast<uint16_t>(packed[0]);
    } else {
      if (QB == 2) {   // 48 bits at a 6-byte (2-aligned) offset
        uint16_t* o16 = reinterpret_cast<uint16_t*>(out + bc0 * 3);
        o16[0] = static_cast<uint16_t>(packed[0]);
        o16[1] = static_cast<uint16_t>((packed[0] >> 16) | (packed[1] << 8));
        o16[2] = static_cast<uint16_t>(packed[1] >> 8);
      } else {
        out += bc0 * 3;
        out[0] = static_cast<uint8_t>(packed[0]);
        out[1] = static_cast<uint8_t>(packed[0] >> 8);
        out[2] = static_cast<uint8_t>(packed[0] >> 16);
      }
    }
  }
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
  FastDiv dcu;          // division by the work units per block row (unit count < 2^31)
};

template <int QB>
__device__ __forceinline__ void load_unit(float4 (&x)[QB][4], const float* __restrict__ src, int64_t cols, int br,
                                          int64_t bc0) {
  const float* p = src + (static_cast<int64_t>(br) * 4) * cols + bc0 * 4;
#pragma unroll
  for (int q = 0; q < QB; ++q)
#pragma unroll
    for (int r = 0; r < 4; ++r) x[q][r] = __ldg(reinterpret_cast<const float4*>(p + r * cols + 4 * q));
}

template <int FMT, int RND, int QB>
__device__ __forceinline__ void quantize_body(const QuantArgs& qa, const float* __restrict__ amax_src, int amax_count,
                                              int cta, int nctas) {
  const int64_t cols = qa.cols;
  const int64_t cb = cols >> 2;                       // column blocks per block row
  const int cu = static_cast<int>(cb / QB);           // work units per block row
  const int nunits = static_cast<int>((qa.rows >> 2) * cu);
  const int64_t row_bytes = FMT == 0 ? (cols >> 1) : (cols * 3) >> 2;
  const int stride = nctas * kQuantThreads;

  // The first unit's loads do not depend on the tensor scale: issue them
  // before the reduction of the amax partials, so the two latencies overlap.
  int w = cta * kQuantThreads + static_cast<int>(threadIdx.x);
  float4 x[QB][4];
  if (w < nunits) {
    const int br = fdiv(w, qa.dcu);
    load_unit<QB>(x, qa.src, cols, br, static_cast<int64_t>(w - br * cu) * QB);
  }
  __shared__ float red[32];
  const TensorScale<FMT> ts(block_max_of(amax_src, amax_count, red));
  if (cta == 0 && threadIdx.x == 0) *qa.tscale = ts.T;

  for (; w < nunits; w += stride) {
    const int br = fdiv(w, qa.dcu);
    const int64_t bc0 = static_cast<int64_t>(w - br * cu) * QB;
    quantize_unit<FMT, RND, QB>(x, ts, br, bc0, cb, row_bytes, qa.keys, qa.sr_cols, qa.sr_col0, qa.codes,
                                qa.scales);
    const int wn = w + stride;
    if (wn < nunits) {
      const int bn = fdiv(wn, qa.dcu);
      load_unit<QB>(x, qa.src, cols, bn, static_cast<int64_t>(wn - bn * cu) * QB);
    }
  }
}

template <int FMT, int RND, int QB>
__global__ void __launch_bounds__(kQuantThreads)
quantize_kernel(const __grid_constant__ QuantArgs qa, const float* __restrict__ amax_src, int amax_count) {
  quantize_body<FMT, RND, QB>(qa, amax_src, amax_count, blockIdx.x, gridDim.x);
}

// ------------------------------------------------ several tensors at once
// The quantize-once step of a layer (X, W, G_Y) in two launches instead of
// six: every CTA of a launch serves one tensor ("job"), CTAs are assigned to
// jobs in contiguous ranges.  Results are bit-identical to one
// amax_partial_kernel + quantize_kernel pair per tensor with the same CTA
// counts.
constexpr int kMaxQuantJobs = 8;

struct QuantJob {
  QuantArgs qa;
  int32_t fmt, rounding, qb;
  int32_t amax_cta0, amax_ctas;     // this job's range of amax CTAs (= its partials)
  int32_t quant_cta0, quant_ctas;   // this job's range of quantize CTAs
};

struct QuantJobs {
  QuantJob job[kMaxQuantJobs];
  int32_t count;
};

__device__ __forceinline__ int job_of(const QuantJobs& jobs, int cta, bool quant) {
  int j = 0;
  for (int i = 1; i < jobs.count; ++i)
    if (cta >= (quant ? jobs.job[i].quant_cta0 : jobs.job[i].amax_cta0)) j = i;
  return j;
}

__global__ void __launch_bounds__(kAmaxThreads)
amax_many_kernel(const __grid_constant__ QuantJobs jobs, float* __restrict__ partial) {
  const QuantJob& jb = jobs.job[job_of(jobs, blockIdx.x, false)];
  amax_partial_body(reinterpret_cast<const float4*>(jb.qa.src), jb.qa.rows * jb.qa.cols / 4, partial + blockIdx.x,
                    blockIdx.x - jb.amax_cta0, jb.amax_ctas);
}

__global__ void __launch_bounds__(kQuantThreads)
quantize_many_kernel(const __grid_constant__ QuantJobs jobs, const float* __restrict__ partial) {
  const QuantJob& jb = jobs.job[job_of(jobs, blockIdx.x, true)];
  const int cta = blockIdx.x - jb.quant_cta0;
  const float* amax = partial + jb.amax_cta0;
#define MQV_QUANT_CASE(F, R, Q)                                                                   \
  if (jb.fmt == F && jb.rounding == R && jb.qb == Q) {                                            \
    quantize_body<F, R, Q>(jb.qa, amax, jb.amax_ctas, cta, jb.quant_ctas);                         \
    return;                                                                                       \
  }
  MQV_QUANT_CASE(0, 0, 1) MQV_QUANT_CASE(0, 1, 1) MQV_QUANT_CASE(1, 0, 1) MQV_QUANT_CASE(1, 1, 1)
#undef MQV_QUANT_CASE
}

// ---------------------------------------------------------- dequantize
// dst = (code·B in fp16, exact) · T, one thread per 4 x 4 block.
template <int FMT>
__global__ void __launch_bounds__(kQuantThreads)
dequantize_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                  const float* __restrict__ tscale, int64_t rows, int64_t cols,
                  float* __restrict__ dst) {
  const float T = *tscale;
  const int64_t cb = cols >> 2;
  const int64_t nblocks = (rows >> 2) * cb;
  const int64_t row_bytes = FMT == 0 ? (cols >> 1) : (cols * 3) >> 2;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kQuantThreads;
  for (int64_t b = static_cast<int64_t>(blockIdx.x) * kQuantThreads + threadIdx.x; b < nblocks;
       b += stride) {
    const int64_t br = b / cb, bc = b - br * cb;
    const uint32_t s = scales[b];
    const uint32_t s2 = e4m3x2_to_f16x2(s | (s << 8));
#pragma unroll
    for (int r = 0; r < 4; ++r) {
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
      h01 = hmul2_u32(h01, s2);
      h23 = hmul2_u32(h23, s2);
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
