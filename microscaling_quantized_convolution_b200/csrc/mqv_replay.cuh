// Latent-replay storage of quantized post-ReLU tensors (MicroQonv summary,
// onedev.kr/papers/182, sections "어떻게 쓰나" and "전제와 한계": an E2M1
// activation needs 3 bits per pixel, and the latent-replay buffer keeps the
// quantized activations).  After ReLU every code has sign bit 0, so only the
// magnitude (m = 3 bits for E2M1, 5 for E2M3) is stored: element i of the
// row-major view at bits [i·m, i·m + m) of a little-endian bit stream.  The
// E4M3 block scales and T stay as they are.
//
// The standard packing of codes is one flat stream too (cols is a multiple
// of 4, so rows never pad), and rows·cols is a multiple of 16.  Each thread
// converts one run of 32 elements (16 for the last one when rows·cols is
// an odd multiple of 16): E2M1 16 -> 12 bytes, E2M3 24 -> 20 bytes, so
// every thread's bytes start on a 4-byte (stored form) or 8-byte (codes)
// boundary and move as 8- and 4-byte words.
#pragma once

#include <cstdint>

#include "mqv_ptx.cuh"

namespace mqv {

constexpr int kReplayThreads = 256;
constexpr int kReplayRun = 32;  // elements per thread

template <int FMT>
struct ReplayFmt {
  static constexpr int kCodeBits = FMT == 0 ? 4 : 6;
  static constexpr int kMagBits = kCodeBits - 1;
  static constexpr uint32_t kMagMask = (1u << kMagBits) - 1;
};

// Bits [pos, pos + len) of a little-endian word array (pos, len constant
// after unrolling; len <= 32 - (pos % 32) or the field spans two words).
template <int N>
__device__ __forceinline__ uint32_t get_bits(const uint32_t (&w)[N], int pos, int len) {
  const int i = pos >> 5, s = pos & 31;
  uint32_t v = w[i] >> s;
  if (s + len > 32) v |= w[i + 1] << (32 - s);
  return v & ((1u << len) - 1);
}

template <int N>
__device__ __forceinline__ void put_bits(uint32_t (&w)[N], int pos, int len, uint32_t v) {
  const int i = pos >> 5, s = pos & 31;
  w[i] |= v << s;
  if (s + len > 32) w[i + 1] |= v >> (32 - s);
}

// BYTES bytes at an 8-byte aligned address, as 8-byte words and a 4-byte tail.
template <int BYTES>
__device__ __forceinline__ void load_words8(const uint8_t* p, uint32_t (&w)[(BYTES + 3) / 4]) {
#pragma unroll
  for (int i = 0; i < BYTES / 8; ++i) {
    const uint2 v = *reinterpret_cast<const uint2*>(p + 8 * i);
    w[2 * i] = v.x;
    w[2 * i + 1] = v.y;
  }
  if (BYTES % 8 == 4) w[BYTES / 4 - 1] = *reinterpret_cast<const uint32_t*>(p + BYTES - 4);
}

template <int BYTES>
__device__ __forceinline__ void store_words8(uint8_t* p, const uint32_t (&w)[(BYTES + 3) / 4]) {
#pragma unroll
  for (int i = 0; i < BYTES / 8; ++i) *reinterpret_cast<uint2*>(p + 8 * i) = make_uint2(w[2 * i], w[2 * i + 1]);
  if (BYTES % 8 == 4) *reinterpret_cast<uint32_t*>(p + BYTES - 4) = w[BYTES / 4 - 1];
}

// BYTES bytes (even) at a 4-byte aligned address, as 4-byte words and a
// 2-byte tail.
template <int BYTES>
__device__ __forceinline__ void load_words4(const uint8_t* p, uint32_t (&w)[(BYTES + 3) / 4]) {
#pragma unroll
  for (int i = 0; i < BYTES / 4; ++i) w[i] = *reinterpret_cast<const uint32_t*>(p + 4 * i);
  if (BYTES % 4 == 2) w[BYTES / 4] = *reinterpret_cast<const uint16_t*>(p + BYTES - 2);
}

template <int BYTES>
__device__ __forceinline__ void store_words4(uint8_t* p, const uint32_t (&w)[(BYTES + 3) / 4]) {
#pragma unroll
  for (int i = 0; i < BYTES / 4; ++i) *reinterpret_cast<uint32_t*>(p + 4 * i) = w[i];
  if (BYTES % 4 == 2) *reinterpret_cast<uint16_t*>(p + BYTES - 2) = static_cast<uint16_t>(w[BYTES / 4]);
}

// Magnitudes of the run of NE elements starting at element e0 of the replay
// form (e0 a multiple of 16).
template <int FMT, int NE>
__device__ __forceinline__ void read_replay_run(const uint8_t* __restrict__ in, int64_t e0, uint32_t (&mag)[NE]) {
  using F = ReplayFmt<FMT>;
  constexpr int kB = NE * F::kMagBits / 8;
  uint32_t w[(kB + 3) / 4];
  load_words4<kB>(in + e0 / 8 * F::kMagBits, w);
#pragma unroll
  for (int j = 0; j < NE; ++j) mag[j] = get_bits(w, j * F::kMagBits, F::kMagBits);
}

// Pack one run: codes -> magnitudes; negative nonzero codes become 0 and
// are counted.
template <int FMT, int NE>
__device__ __forceinline__ unsigned pack_run(const uint8_t* __restrict__ codes, uint8_t* __restrict__ out,
                                             int64_t e0) {
  using F = ReplayFmt<FMT>;
  constexpr int kCB = NE * F::kCodeBits / 8;
  constexpr int kMB = NE * F::kMagBits / 8;
  uint32_t in[(kCB + 3) / 4];
  load_words8<kCB>(codes + e0 / 8 * F::kCodeBits, in);
  uint32_t o[(kMB + 3) / 4];
#pragma unroll
  for (int i = 0; i < (kMB + 3) / 4; ++i) o[i] = 0;
  unsigned neg = 0;
#pragma unroll
  for (int j = 0; j < NE; ++j) {
    const uint32_t c = get_bits(in, j * F::kCodeBits, F::kCodeBits);
    uint32_t m = c & F::kMagMask;
    if ((c >> F::kMagBits) && m) {
      ++neg;
      m = 0;
    }
    put_bits(o, j * F::kMagBits, F::kMagBits, m);
  }
  store_words4<kMB>(out + e0 / 8 * F::kMagBits, o);
  return neg;
}

template <int FMT, int NE>
__device__ __forceinline__ void unpack_run(const uint8_t* __restrict__ in, uint8_t* __restrict__ codes, int64_t e0) {
  using F = ReplayFmt<FMT>;
  constexpr int kCB = NE * F::kCodeBits / 8;
  uint32_t mag[NE];
  read_replay_run<FMT, NE>(in, e0, mag);
  uint32_t o[(kCB + 3) / 4];
#pragma unroll
  for (int i = 0; i < (kCB + 3) / 4; ++i) o[i] = 0;
#pragma unroll
  for (int j = 0; j < NE; ++j) put_bits(o, j * F::kCodeBits, F::kCodeBits, mag[j]);
  store_words8<kCB>(codes + e0 / 8 * F::kCodeBits, o);
}

// n = rows·cols elements; thread t owns elements [32t, 32t + 32) (the last
// one possibly 16).
template <int FMT>
__global__ void __launch_bounds__(kReplayThreads)
replay_pack_kernel(const uint8_t* __restrict__ codes, int64_t n, uint8_t* __restrict__ out,
                   unsigned* __restrict__ negatives) {
  unsigned neg = 0;
  const int64_t runs = (n + kReplayRun - 1) / kReplayRun;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kReplayThreads;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * kReplayThreads + threadIdx.x; t < runs; t += stride) {
    const int64_t e0 = t * kReplayRun;
    neg += e0 + kReplayRun <= n ? pack_run<FMT, kReplayRun>(codes, out, e0) : pack_run<FMT, 16>(codes, out, e0);
  }
  if (negatives != nullptr) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) neg += __shfl_xor_sync(0xffffffffu, neg, off);
    if ((threadIdx.x & 31) == 0 && neg) atomicAdd(negatives, neg);
  }
}

template <int FMT>
__global__ void __launch_bounds__(kReplayThreads)
replay_unpack_kernel(const uint8_t* __restrict__ in, int64_t n, uint8_t* __restrict__ codes) {
  const int64_t runs = (n + kReplayRun - 1) / kReplayRun;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kReplayThreads;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * kReplayThreads + threadIdx.x; t < runs; t += stride) {
    const int64_t e0 = t * kReplayRun;
    if (e0 + kReplayRun <= n)
      unpack_run<FMT, kReplayRun>(in, codes, e0);
    else
      unpack_run<FMT, 16>(in, codes, e0);
  }
}

// code·B in fp16 (exact), times T in fp32: the arithmetic of mqv_dequantize.
template <int FMT>
__device__ __forceinline__ float4 dequant4(const uint32_t* mag, uint32_t s2, float T) {
  uint32_t h01, h23;
  if (FMT == 0) {
    h01 = e2m1x2_to_f16x2(mag[0] | (mag[1] << 4));
    h23 = e2m1x2_to_f16x2(mag[2] | (mag[3] << 4));
  } else {
    h01 = e2m3x2_to_f16x2(mag[0] | (mag[1] << 8));
    h23 = e2m3x2_to_f16x2(mag[2] | (mag[3] << 8));
  }
  h01 = hmul2_u32(h01, s2);
  h23 = hmul2_u32(h23, s2);
  return make_float4(__fmul_rn(f16_lo_to_f32(h01), T), __fmul_rn(f16_hi_to_f32(h01), T),
                     __fmul_rn(f16_lo_to_f32(h23), T), __fmul_rn(f16_hi_to_f32(h23), T));
}

template <int FMT, int NE>
__device__ __forceinline__ void dequant_run(const uint8_t* __restrict__ in, const uint8_t* __restrict__ scales,
                                            float T, int64_t cols, int64_t e0, float* __restrict__ dst) {
  uint32_t mag[NE];
  read_replay_run<FMT, NE>(in, e0, mag);
  int64_t r = e0 / cols, c = e0 - r * cols;
  const int64_t scols = cols >> 2;
#pragma unroll
  for (int k = 0; k < NE / 4; ++k) {
    const uint32_t s = scales[(r >> 2) * scols + (c >> 2)];
    *reinterpret_cast<float4*>(dst + e0 + 4 * k) = dequant4<FMT>(mag + 4 * k, e4m3x2_to_f16x2(s | (s << 8)), T);
    c += 4;
    if (c == cols) {
      c = 0;
      ++r;
    }
  }
}

template <int FMT>
__global__ void __launch_bounds__(kReplayThreads)
replay_dequantize_kernel(const uint8_t* __restrict__ in, const uint8_t* __restrict__ scales,
                         const float* __restrict__ tscale, int64_t cols, int64_t n, float* __restrict__ dst) {
  const float T = *tscale;
  const int64_t runs = (n + kReplayRun - 1) / kReplayRun;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kReplayThreads;
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * kReplayThreads + threadIdx.x; t < runs; t += stride) {
    const int64_t e0 = t * kReplayRun;
    if (e0 + kReplayRun <= n)
      dequant_run<FMT, kReplayRun>(in, scales, T, cols, e0, dst);
    else
      dequant_run<FMT, 16>(in, scales, T, cols, e0, dst);
  }
}

}  // namespace mqv
