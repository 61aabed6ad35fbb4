// Latent-replay storage of quantized post-ReLU tensors (MicroQonv summary,
// onedev.kr/papers/182, sections "어떻게 쓰나" and "전제와 한계": an E2M1
// activation needs 3 bits per pixel, and the latent-replay buffer keeps the
// quantized activations).  After ReLU every code has sign bit 0, so only the
// magnitude (m = 3 bits for E2M1, 5 for E2M3) is stored: element i of the
// row-major view at bits [i·m, i·m + m) of a little-endian bit stream.  The
// E4M3 block scales and T stay as they are.
//
// The standard packing of codes is one flat stream too (cols is a multiple
// of 4, so rows never pad), and rows·cols is a multiple of 16.  A lane
// converts one run of 32 elements (16 for the last one when rows·cols is an
// odd multiple of 16): E2M1 16 -> 12 bytes, E2M3 24 -> 20 bytes, so every
// run starts on a 4-byte boundary in both forms.
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

// ---------------------------------------------------------------------------
// Kernels.  A warp owns segments of kReplaySeg = 1024 consecutive elements
// (32 runs; the last segment of the tensor may be shorter, a multiple of
// 16).  The segment's bytes move between global and shared memory with
// coalesced 16-byte accesses (4-byte ones in a short last segment), and
// each lane converts one run inside shared memory, so every global access
// of a warp is one contiguous range.

constexpr int kReplayWarps = kReplayThreads / 32;
constexpr int kReplaySeg = 32 * kReplayRun;

// Copy `bytes` (a multiple of 2) from a 16-byte aligned global address to
// shared memory (or back): 16-byte pieces while a whole warp's worth fits,
// then 4-byte and 2-byte ones.
__device__ __forceinline__ void warp_copy_in(uint32_t* __restrict__ dst, const uint8_t* __restrict__ src, int bytes,
                                             int lane) {
  const int n16 = bytes >> 4;
  for (int i = lane; i < n16; i += 32)
    reinterpret_cast<uint4*>(dst)[i] = reinterpret_cast<const uint4*>(src)[i];
  const int done = n16 << 4;
  for (int i = done + 4 * lane; i + 4 <= bytes; i += 128) dst[i >> 2] = *reinterpret_cast<const uint32_t*>(src + i);
  if ((bytes & 3) && lane == 0) {
    const int i = bytes & ~3;
    dst[i >> 2] = *reinterpret_cast<const uint16_t*>(src + i);
  }
}

__device__ __forceinline__ void warp_copy_out(uint8_t* __restrict__ dst, const uint32_t* __restrict__ src, int bytes,
                                              int lane) {
  const int n16 = bytes >> 4;
  for (int i = lane; i < n16; i += 32)
    reinterpret_cast<uint4*>(dst)[i] = reinterpret_cast<const uint4*>(src)[i];
  const int done = n16 << 4;
  for (int i = done + 4 * lane; i + 4 <= bytes; i += 128) *reinterpret_cast<uint32_t*>(dst + i) = src[i >> 2];
  if ((bytes & 3) && lane == 0) {
    const int i = bytes & ~3;
    *reinterpret_cast<uint16_t*>(dst + i) = static_cast<uint16_t>(src[i >> 2]);
  }
}

template <int FMT>
struct ReplaySmem {
  using F = ReplayFmt<FMT>;
  static constexpr int kCodeWords = kReplaySeg * F::kCodeBits / 32;  // 128 / 192
  static constexpr int kMagWords = kReplaySeg * F::kMagBits / 32;    // 96 / 160
  // a spare word after the segment (read by the last group's funnel shift),
  // rounded up so that every warp's row starts on a 16-byte boundary
  static constexpr int kMagRow = kMagWords + 4;
};

// Whole-word forms of one conversion.  E2M1: 8 codes of a 32-bit word
// (nibbles) <-> their 8 magnitudes in 24 bits.  E2M3: 4 codes in 24 bits
// <-> 4 magnitudes in 20 bits.  A magnitude field m is nonzero iff
// m + (2^k - 1) carries into the field's sign position; the fields are too
// narrow for that carry to reach the next field.  A negative nonzero code
// gets magnitude 0; *neg counts them.
__device__ __forceinline__ uint32_t pack8_e2m1(uint32_t w, unsigned* neg) {
  const uint32_t mag = w & 0x77777777u;
  const uint32_t ng = w & ((mag + 0x77777777u) & 0x88888888u);
  *neg += __popc(ng);
  uint32_t x = mag & ~((ng >> 3) * 7u);
  x = (x & 0x07070707u) | ((x & 0x70707070u) >> 1);
  x = (x & 0x003F003Fu) | ((x & 0x3F003F00u) >> 2);
  return (x & 0x00000FFFu) | ((x & 0x0FFF0000u) >> 4);
}

__device__ __forceinline__ uint32_t unpack8_e2m1(uint32_t x) {
  x = (x & 0xFFFu) | ((x & 0xFFF000u) << 4);
  x = (x & 0x003F003Fu) | ((x & 0x0FC00FC0u) << 2);
  return (x & 0x07070707u) | ((x & 0x38383838u) << 1);
}

__device__ __forceinline__ uint32_t pack4_e2m3(uint32_t g, unsigned* neg) {
  const uint32_t mag = g & 0x7DF7DFu;
  const uint32_t ng = g & ((mag + 0x7DF7DFu) & 0x820820u);
  *neg += __popc(ng);
  uint32_t x = mag & ~((ng >> 5) * 31u);
  x = (x & 0x01F01Fu) | ((x & 0x7C07C0u) >> 1);
  return (x & 0x3FFu) | ((x & 0x3FF000u) >> 2);
}

__device__ __forceinline__ uint32_t unpack4_e2m3(uint32_t x) {
  x = (x & 0x3FFu) | ((x & 0xFFC00u) << 2);
  return (x & 0x01F01Fu) | ((x & 0x3E03E0u) << 1);
}

// Run j of a segment in shared memory, codes -> magnitudes.
template <int FMT, int NE>
__device__ __forceinline__ unsigned pack_run_smem(const uint32_t* __restrict__ sc, uint32_t* __restrict__ sm, int j) {
  using F = ReplayFmt<FMT>;
  constexpr int kCW = NE * F::kCodeBits / 32, kMW = (NE * F::kMagBits + 31) / 32;
  uint32_t in[kCW], o[kMW];
#pragma unroll
  for (int i = 0; i < kCW; ++i) in[i] = sc[j * (kReplayRun * F::kCodeBits / 32) + i];
#pragma unroll
  for (int i = 0; i < kMW; ++i) o[i] = 0;
  unsigned neg = 0;
  if (FMT == 0) {
#pragma unroll
    for (int k = 0; k < NE / 8; ++k) put_bits(o, 24 * k, 24, pack8_e2m1(in[k], &neg));
  } else {
#pragma unroll
    for (int k = 0; k < NE / 4; ++k) put_bits(o, 20 * k, 20, pack4_e2m3(get_bits(in, 24 * k, 24), &neg));
  }
#pragma unroll
  for (int i = 0; i < kMW; ++i) sm[j * (kReplayRun * F::kMagBits / 32) + i] = o[i];
  return neg;
}

template <int FMT, int NE>
__device__ __forceinline__ void unpack_run_smem(const uint32_t* __restrict__ sm, uint32_t* __restrict__ sc, int j) {
  using F = ReplayFmt<FMT>;
  constexpr int kCW = NE * F::kCodeBits / 32, kMW = (NE * F::kMagBits + 31) / 32;
  uint32_t in[kMW], o[kCW];
#pragma unroll
  for (int i = 0; i < kMW; ++i) in[i] = sm[j * (kReplayRun * F::kMagBits / 32) + i];
  if (FMT == 0) {
#pragma unroll
    for (int k = 0; k < NE / 8; ++k) o[k] = unpack8_e2m1(get_bits(in, 24 * k, 24));
  } else {
#pragma unroll
    for (int i = 0; i < kCW; ++i) o[i] = 0;
#pragma unroll
    for (int k = 0; k < NE / 4; ++k) put_bits(o, 24 * k, 24, unpack4_e2m3(get_bits(in, 20 * k, 20)));
  }
#pragma unroll
  for (int i = 0; i < kCW; ++i) sc[j * (kReplayRun * F::kCodeBits / 32) + i] = o[i];
}

// A whole segment of BYTES bytes held in registers across the warp: lane l
// keeps 16-byte pieces l and l + 32 (those that exist).  The next segment's
// loads are issued before the current one is converted, so they overlap.
template <int BYTES>
struct SegRegs {
  static constexpr int kPieces = BYTES / 16;
  static constexpr int kPer = (kPieces + 31) / 32;
  uint4 r[kPer];

  __device__ __forceinline__ void load(const uint8_t* __restrict__ src, int lane) {
#pragma unroll
    for (int k = 0; k < kPer; ++k)
      if (lane + 32 * k < kPieces) r[k] = reinterpret_cast<const uint4*>(src)[lane + 32 * k];
  }
  __device__ __forceinline__ void to_smem(uint32_t* dst, int lane) const {
#pragma unroll
    for (int k = 0; k < kPer; ++k)
      if (lane + 32 * k < kPieces) reinterpret_cast<uint4*>(dst)[lane + 32 * k] = r[k];
  }
};

// Both conversions share one loop: DIR 0 packs (codes -> magnitudes), DIR 1
// unpacks.  Whole segments go through the register prefetch; the one short
// segment a tensor may end with takes the plain copies.
template <int FMT, int DIR>
__device__ __forceinline__ unsigned replay_convert(const uint8_t* __restrict__ src, int64_t n,
                                                   uint8_t* __restrict__ dst, uint32_t* __restrict__ s_src,
                                                   uint32_t* __restrict__ s_dst) {
  using F = ReplayFmt<FMT>;
  constexpr int kSrcBits = DIR == 0 ? F::kCodeBits : F::kMagBits;
  constexpr int kDstBits = DIR == 0 ? F::kMagBits : F::kCodeBits;
  const int lane = threadIdx.x & 31;
  const int64_t wstride = static_cast<int64_t>(gridDim.x) * kReplayWarps;
  const int64_t first = static_cast<int64_t>(blockIdx.x) * kReplayWarps + (threadIdx.x >> 5);
  const int64_t nfull = n / kReplaySeg;
  unsigned neg = 0;
  auto convert = [&](int ne) {
    if (kReplayRun * lane + kReplayRun <= ne) {
      if (DIR == 0)
        neg += pack_run_smem<FMT, kReplayRun>(s_src, s_dst, lane);
      else
        unpack_run_smem<FMT, kReplayRun>(s_src, s_dst, lane);
    } else if (kReplayRun * lane < ne) {
      if (DIR == 0)
        neg += pack_run_smem<FMT, 16>(s_src, s_dst, lane);
      else
        unpack_run_smem<FMT, 16>(s_src, s_dst, lane);
    }
  };
  SegRegs<kReplaySeg * kSrcBits / 8> regs;
  if (first < nfull) regs.load(src + first * (kReplaySeg / 8 * kSrcBits), lane);
  for (int64_t seg = first; seg < nfull; seg += wstride) {
    regs.to_smem(s_src, lane);
    if (seg + wstride < nfull) regs.load(src + (seg + wstride) * (kReplaySeg / 8 * kSrcBits), lane);
    __syncwarp();
    convert(kReplaySeg);
    __syncwarp();
    warp_copy_out(dst + seg * (kReplaySeg / 8 * kDstBits), s_dst, kReplaySeg / 8 * kDstBits, lane);
    __syncwarp();
  }
  if (nfull * kReplaySeg < n && first == nfull % wstride && nfull >= first) {
    const int64_t e0 = nfull * kReplaySeg;
    const int ne = static_cast<int>(n - e0);
    warp_copy_in(s_src, src + e0 / 8 * kSrcBits, ne * kSrcBits / 8, lane);
    __syncwarp();
    convert(ne);
    __syncwarp();
    warp_copy_out(dst + e0 / 8 * kDstBits, s_dst, ne * kDstBits / 8, lane);
  }
  return neg;
}

template <int FMT>
__global__ void __launch_bounds__(kReplayThreads)
replay_pack_kernel(const uint8_t* __restrict__ codes, int64_t n, uint8_t* __restrict__ out,
                   unsigned* __restrict__ negatives) {
  using S = ReplaySmem<FMT>;
  __shared__ __align__(16) uint32_t s_code[kReplayWarps][S::kCodeWords];
  __shared__ __align__(16) uint32_t s_mag[kReplayWarps][S::kMagRow];
  const int warp = threadIdx.x >> 5;
  unsigned neg = replay_convert<FMT, 0>(codes, n, out, s_code[warp], s_mag[warp]);
  if (negatives != nullptr) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) neg += __shfl_xor_sync(0xffffffffu, neg, off);
    if ((threadIdx.x & 31) == 0 && neg) atomicAdd(negatives, neg);
  }
}

template <int FMT>
__global__ void __launch_bounds__(kReplayThreads)
replay_unpack_kernel(const uint8_t* __restrict__ in, int64_t n, uint8_t* __restrict__ codes) {
  using S = ReplaySmem<FMT>;
  __shared__ __align__(16) uint32_t s_code[kReplayWarps][S::kCodeWords];
  __shared__ __align__(16) uint32_t s_mag[kReplayWarps][S::kMagRow];
  const int warp = threadIdx.x >> 5;
  replay_convert<FMT, 1>(in, n, codes, s_mag[warp], s_code[warp]);
}

// code·B in fp16 (exact), times T in fp32: the arithmetic of mqv_dequantize.
template <int FMT>
__device__ __forceinline__ float4 dequant4(uint32_t m0, uint32_t m1, uint32_t m2, uint32_t m3, uint32_t s2,
                                           float T) {
  uint32_t h01, h23;
  if (FMT == 0) {
    h01 = e2m1x2_to_f16x2(m0 | (m1 << 4));
    h23 = e2m1x2_to_f16x2(m2 | (m3 << 4));
  } else {
    h01 = e2m3x2_to_f16x2(m0 | (m1 << 8));
    h23 = e2m3x2_to_f16x2(m2 | (m3 << 8));
  }
  h01 = hmul2_u32(h01, s2);
  h23 = hmul2_u32(h23, s2);
  return make_float4(__fmul_rn(f16_lo_to_f32(h01), T), __fmul_rn(f16_hi_to_f32(h01), T),
                     __fmul_rn(f16_lo_to_f32(h23), T), __fmul_rn(f16_hi_to_f32(h23), T));
}

// q = floor(u / d) for any 32-bit u (the sum is formed in 64 bits).
__device__ __forceinline__ uint32_t fdiv_u32(uint32_t u, FastDiv f) {
  return static_cast<uint32_t>((static_cast<uint64_t>(__umulhi(u, f.m)) + u) >> f.s);
}

// Values straight from the replay form.  Lane l of a warp handles the groups
// of 4 elements l, l + 32, ... of its segment, so each float4 store of the
// warp writes 512 contiguous bytes.  dcols4: divider by cols/4 (group ->
// row); group indices stay below 2^32 (rows·cols <= 2^34).
template <int FMT>
__global__ void __launch_bounds__(kReplayThreads)
replay_dequantize_kernel(const uint8_t* __restrict__ in, const uint8_t* __restrict__ scales,
                         const float* __restrict__ tscale, int64_t cols, FastDiv dcols4, int64_t n,
                         float* __restrict__ dst) {
  using F = ReplayFmt<FMT>;
  using S = ReplaySmem<FMT>;
  constexpr int kGroupBits = 4 * F::kMagBits;
  __shared__ __align__(16) uint32_t s_mag[kReplayWarps][S::kMagRow];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float T = *tscale;
  const uint32_t cols4 = static_cast<uint32_t>(cols >> 2);
  const int64_t nseg = (n + kReplaySeg - 1) / kReplaySeg;
  const int64_t wstride = static_cast<int64_t>(gridDim.x) * kReplayWarps;
  for (int64_t seg = static_cast<int64_t>(blockIdx.x) * kReplayWarps + warp; seg < nseg; seg += wstride) {
    const int64_t e0 = seg * kReplaySeg;
    const int ne = static_cast<int>(n - e0 < kReplaySeg ? n - e0 : kReplaySeg);
    warp_copy_in(s_mag[warp], in + e0 / 8 * F::kMagBits, ne * F::kMagBits / 8, lane);
    s_mag[warp][S::kMagWords] = 0;
    __syncwarp();
#pragma unroll 4
    for (int g = lane; 4 * g < ne; g += 32) {
      const int bit = g * kGroupBits;
      const uint32_t v = __funnelshift_r(s_mag[warp][bit >> 5], s_mag[warp][(bit >> 5) + 1], bit & 31);
      const uint32_t ga = static_cast<uint32_t>(e0 >> 2) + static_cast<uint32_t>(g);
      const uint32_t row = fdiv_u32(ga, dcols4);
      const uint32_t c4 = ga - row * cols4;
      const uint32_t sc = scales[static_cast<int64_t>(row >> 2) * cols4 + c4];
      constexpr uint32_t kM = F::kMagMask;
      constexpr int kB = F::kMagBits;
      *reinterpret_cast<float4*>(dst + e0 + 4 * g) =
          dequant4<FMT>(v & kM, (v >> kB) & kM, (v >> (2 * kB)) & kM, (v >> (3 * kB)) & kM,
                        e4m3x2_to_f16x2(sc | (sc << 8)), T);
    }
    __syncwarp();
  }
}

}  // namespace mqv
