// Implicit-GEMM kernels for the three convolution GEMMs on square-block
// quantized operands (MicroQonv summary, onedev.kr/papers/182, section
// "무엇과 다른가": Y = W·X', G_W = G_Y·X'^T, G_X' = W^T·G_Y, with the
// im2col rows of X' built on chip, section "어떻게 동작하나").
//
// One kernel template serves all three passes.  A CTA owns a 128 x BN tile
// of D = A·B^T (fp32 accumulators in tensor memory).  Eight producer warps
// gather 4 x 4 quantized blocks straight from the channel-batch-first
// tensors (the sliding-window gather is pure index arithmetic, padding taps
// are zero blocks), dequantize them to fp16 (code·B_scale is exact in
// fp16; the tensor scales are applied once in the epilogue) and store them
// K-major with the 128-byte swizzle.  One elected thread of a ninth warp
// issues tcgen05.mma (M=128, N=BN, K=16) per stage and commits to the
// stage's "empty" barrier.  After the K loop the producer warps read the
// accumulators back with tcgen05.ld, multiply by T_a·T_b and store fp32.
#pragma once

#include <cstdint>

#include "mqv_ptx.cuh"

namespace mqv {

constexpr int kBM = 128;                 // MMA M (rows of A per tile)
constexpr int kBK = 64;                  // K per stage (one 128-byte fp16 row)
constexpr int kProducerWarps = 8;
constexpr int kProducerThreads = kProducerWarps * 32;
constexpr int kConvThreads = kProducerThreads + 32;

enum ConvPass { kFwd = 0, kWgrad = 1, kDgrad = 2 };

// Device error bits set by bounded waits.
constexpr uint32_t kErrWaitEmpty = 1u, kErrWaitFull = 2u, kErrWaitDone = 4u;

struct QView {
  const uint8_t* codes;
  const uint8_t* scales;
  const float* tscale;
  int64_t row_bytes;    // bytes per row of packed codes
  int64_t scale_cols;   // blocks per row of the scale plane (= cols / 4)
};

struct ConvArgs {
  QView a, b;
  float* out;           // Y / G_X / G_W, or the split partials of G_W
  uint32_t* err;
  int N, Cin, Cout, H, W, Kh, Kw, stride, pad, Ho, Wo;
  int M;                // GEMM rows
  int64_t Ncols;        // GEMM columns
  int64_t Kdim;         // contraction length
  int ktiles;           // ceil(Kdim / 64)
  int kt_per_split;     // K tiles per blockIdx.z
  int scale_out;        // 1: multiply by T_a·T_b before storing
};

template <int BN, int STAGES>
struct ConvSmem {
  static constexpr int kATile = kBM * kBK * 2;
  static constexpr int kBTile = BN * kBK * 2;
  static constexpr int kStage = kATile + kBTile;
  static constexpr int kBarOffset = STAGES * kStage;
  static constexpr int kBytes = kBarOffset + 256 + 1024;   // + barriers + alignment slack
};

// Byte offset of (row, k) inside a K-major, 128-byte-swizzled fp16 tile.
__device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t k) {
  return row * 128u + ((((k >> 3) ^ (row & 7u)) << 4) | ((k & 4u) << 1));
}

// ---------------------------------------------------------------------------
// One 4 x 4 quantized block: four source quads (4 codes each, along the
// view's columns) from four consecutive view rows, plus its E4M3 scale.
template <int FMT>
__device__ __forceinline__ void fetch_block(const QView& v, int64_t row0, int64_t col0,
                                            uint32_t (&q)[4], uint32_t& s) {
  const uint8_t* p = v.codes + row0 * v.row_bytes + (FMT == 0 ? (col0 >> 1) : ((col0 * 3) >> 2));
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint8_t* r = p + j * v.row_bytes;
    if (FMT == 0) {
      q[j] = __ldg(reinterpret_cast<const unsigned short*>(r));
    } else {
      q[j] = static_cast<uint32_t>(__ldg(r)) | (static_cast<uint32_t>(__ldg(r + 1)) << 8) |
             (static_cast<uint32_t>(__ldg(r + 2)) << 16);
    }
  }
  s = __ldg(v.scales + (row0 >> 2) * v.scale_cols + (col0 >> 2));
}

// Dequantize the four quads to fp16 pairs: h[j][0] = values 0,1 of quad j,
// h[j][1] = values 2,3 (low half = lower column).
template <int FMT>
__device__ __forceinline__ void dequant_block(const uint32_t (&q)[4], uint32_t s,
                                              uint32_t (&h)[4][2]) {
  const uint32_t s2 = e4m3x2_to_f16x2(s | (s << 8));
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint32_t lo, hi;
    if (FMT == 0) {
      lo = e2m1x2_to_f16x2(q[j] & 0xFF);
      hi = e2m1x2_to_f16x2(q[j] >> 8);
    } else {
      lo = e2m3x2_to_f16x2((q[j] & 0x3F) | ((q[j] << 2) & 0x3F00));
      hi = e2m3x2_to_f16x2(((q[j] >> 12) & 0x3F) | ((q[j] >> 10) & 0x3F00));
    }
    h[j][0] = hmul2_u32(lo, s2);
    h[j][1] = hmul2_u32(hi, s2);
  }
}

// Store a dequantized block into the tile at rows row0..row0+3, k0..k0+3.
// Without transpose, quad j is tile row j (its 4 values run along K).  With
// transpose, quad j is K index j and its 4 values run along the tile rows.
template <bool TRANSPOSE>
__device__ __forceinline__ void store_block(uint32_t tile, uint32_t row0, uint32_t k0,
                                            const uint32_t (&h)[4][2]) {
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    uint32_t x, y;
    if (!TRANSPOSE) {
      x = h[r][0];
      y = h[r][1];
    } else {
      const uint32_t sel = (r & 1) ? 0x7632u : 0x5410u;
      x = __byte_perm(h[0][r >> 1], h[1][r >> 1], sel);
      y = __byte_perm(h[2][r >> 1], h[3][r >> 1], sel);
    }
    st_shared_v2(tile + sw128_offset(row0 + r, k0), x, y);
  }
}

__device__ __forceinline__ void store_zero_block(uint32_t tile, uint32_t row0, uint32_t k0) {
#pragma unroll
  for (int r = 0; r < 4; ++r) st_shared_v2(tile + sw128_offset(row0 + r, k0), 0u, 0u);
}

// ---------------------------------------------------------------------------
// Source coordinates of the blocks of each operand.  Each returns false for
// a block that lies outside the GEMM (ragged tile) or on a padding tap.

// Forward, A = W viewed Cout x (Kh·Kw·Cin): tile rows = co, K = (tap, ci).
__device__ __forceinline__ bool fwd_a(const ConvArgs& p, int64_t co0, int64_t k, int64_t& row0,
                                      int64_t& col0) {
  row0 = co0;
  col0 = k;
  return co0 < p.Cout && k < p.Kdim;
}

// Forward, B = X': tile rows = (ho, wo, n), K = (kh, kw, ci) -> X[hi][wi][ci][n].
__device__ __forceinline__ bool fwd_b(const ConvArgs& p, int64_t q, int64_t k, int64_t& row0,
                                      int64_t& col0) {
  if (q >= p.Ncols || k >= p.Kdim) return false;
  const int64_t pix = q / p.N;
  const int n = static_cast<int>(q - pix * p.N);
  const int ho = static_cast<int>(pix / p.Wo), wo = static_cast<int>(pix - static_cast<int64_t>(ho) * p.Wo);
  const int tap = static_cast<int>(k / p.Cin), ci = static_cast<int>(k - static_cast<int64_t>(tap) * p.Cin);
  const int kh = tap / p.Kw, kw = tap - kh * p.Kw;
  const int hi = ho * p.stride + kh - p.pad, wi = wo * p.stride + kw - p.pad;
  if (hi < 0 || hi >= p.H || wi < 0 || wi >= p.W) return false;
  row0 = (static_cast<int64_t>(hi) * p.W + wi) * p.Cin + ci;
  col0 = n;
  return true;
}

// Weight gradient, A = G_Y as Cout x (Ho·Wo·N): tile rows = co, K = (ho, wo, n).
__device__ __forceinline__ bool wgrad_a(const ConvArgs& p, int64_t co0, int64_t q, int64_t& row0,
                                        int64_t& col0) {
  if (co0 >= p.Cout || q >= p.Kdim) return false;
  const int64_t pix = q / p.N;
  row0 = pix * p.Cout + co0;
  col0 = q - pix * p.N;
  return true;
}

// Weight gradient, B = X' transposed: tile rows = (kh, kw, ci), K = (ho, wo, n).
__device__ __forceinline__ bool wgrad_b(const ConvArgs& p, int64_t kc, int64_t q, int64_t& row0,
                                        int64_t& col0) {
  if (kc >= p.Ncols || q >= p.Kdim) return false;
  const int tap = static_cast<int>(kc / p.Cin), ci = static_cast<int>(kc - static_cast<int64_t>(tap) * p.Cin);
  const int kh = tap / p.Kw, kw = tap - kh * p.Kw;
  const int64_t pix = q / p.N;
  const int n = static_cast<int>(q - pix * p.N);
  const int ho = static_cast<int>(pix / p.Wo), wo = static_cast<int>(pix - static_cast<int64_t>(ho) * p.Wo);
  const int hi = ho * p.stride + kh - p.pad, wi = wo * p.stride + kw - p.pad;
  if (hi < 0 || hi >= p.H || wi < 0 || wi >= p.W) return false;
  row0 = (static_cast<int64_t>(hi) * p.W + wi) * p.Cin + ci;
  col0 = n;
  return true;
}

// Input gradient, A = W^T: tile rows = ci, K = (tap, co) -> W view row co,
// column tap·Cin + ci (the block's quads run along ci: transposed store).
__device__ __forceinline__ bool dgrad_a(const ConvArgs& p, int64_t ci0, int64_t k, int64_t& row0,
                                        int64_t& col0) {
  if (ci0 >= p.Cin || k >= p.Kdim) return false;
  const int tap = static_cast<int>(k / p.Cout), co = static_cast<int>(k - static_cast<int64_t>(tap) * p.Cout);
  row0 = co;
  col0 = static_cast<int64_t>(tap) * p.Cin + ci0;
  return true;
}

// Input gradient, B = G_Y gathered by the transposed-conv map: tile rows =
// (hi, wi, n), K = (kh, kw, co); (ho, wo) = ((hi+pad-kh)/s, (wi+pad-kw)/s)
// when both divide exactly and lie inside the output, else a zero block.
__device__ __forceinline__ bool dgrad_b(const ConvArgs& p, int64_t q, int64_t k, int64_t& row0,
                                        int64_t& col0) {
  if (q >= p.Ncols || k >= p.Kdim) return false;
  const int64_t pix = q / p.N;
  const int n = static_cast<int>(q - pix * p.N);
  const int hi = static_cast<int>(pix / p.W), wi = static_cast<int>(pix - static_cast<int64_t>(hi) * p.W);
  const int tap = static_cast<int>(k / p.Cout), co = static_cast<int>(k - static_cast<int64_t>(tap) * p.Cout);
  const int kh = tap / p.Kw, kw = tap - kh * p.Kw;
  const int th = hi + p.pad - kh, tw = wi + p.pad - kw;
  if (th < 0 || tw < 0) return false;
  const int ho = th / p.stride, wo = tw / p.stride;
  if (ho * p.stride != th || wo * p.stride != tw || ho >= p.Ho || wo >= p.Wo) return false;
  row0 = (static_cast<int64_t>(ho) * p.Wo + wo) * p.Cout + co;
  col0 = n;
  return true;
}

template <int PASS, bool IS_A>
__device__ __forceinline__ bool block_coords(const ConvArgs& p, int64_t tile_row, int64_t k,
                                             int64_t& row0, int64_t& col0) {
  if (PASS == kFwd) return IS_A ? fwd_a(p, tile_row, k, row0, col0) : fwd_b(p, tile_row, k, row0, col0);
  if (PASS == kWgrad) return IS_A ? wgrad_a(p, tile_row, k, row0, col0) : wgrad_b(p, tile_row, k, row0, col0);
  return IS_A ? dgrad_a(p, tile_row, k, row0, col0) : dgrad_b(p, tile_row, k, row0, col0);
}

// Which operands arrive with their block quads along K (no transpose).
template <int PASS, bool IS_A>
struct OperandTraits {
  static constexpr bool kTranspose = (PASS == kFwd && !IS_A) || PASS == kDgrad;
};

// Fill one operand tile (ROWS x 64) for K tile starting at kbase.
// Untransposed operands map consecutive threads to consecutive K quads
// (contiguous bytes of one source row); transposed ones map consecutive
// threads to consecutive tile-row quads (contiguous bytes along the view's
// columns).
template <int PASS, bool IS_A, int FMT, int ROWS>
__device__ __forceinline__ void fill_tile(const ConvArgs& p, const QView& v, uint32_t tile,
                                          int64_t row_base, int64_t kbase, int t) {
  constexpr bool kT = OperandTraits<PASS, IS_A>::kTranspose;
  constexpr int kRowQuads = ROWS / 4;
  constexpr int kBlocks = kRowQuads * (kBK / 4);
  static_assert(kBlocks % kProducerThreads == 0, "tile must split evenly over producers");
#pragma unroll
  for (int i = 0; i < kBlocks / kProducerThreads; ++i) {
    const int id = t + i * kProducerThreads;
    int rq, kq;
    if (kT) {
      rq = id % kRowQuads;
      kq = id / kRowQuads;
    } else {
      kq = id % (kBK / 4);
      rq = id / (kBK / 4);
    }
    int64_t row0, col0;
    const bool ok = block_coords<PASS, IS_A>(p, row_base + 4 * rq, kbase + 4 * kq, row0, col0);
    if (ok) {
      uint32_t q[4], s, h[4][2];
      fetch_block<FMT>(v, row0, col0, q, s);
      dequant_block<FMT>(q, s, h);
      store_block<kT>(tile, 4 * rq, 4 * kq, h);
    } else {
      store_zero_block(tile, 4 * rq, 4 * kq);
    }
  }
}

// ---------------------------------------------------------------------------
template <int PASS, int FMT, int BN, int STAGES>
__global__ void __launch_bounds__(kConvThreads, 1)
conv_gemm_kernel(const ConvArgs p) {
  using L = ConvSmem<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + L::kBarOffset);
  uint64_t* empty_bar = full_bar + STAGES;
  uint64_t* done_bar = empty_bar + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * BN;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * kBM;
  const int kt0 = blockIdx.z * p.kt_per_split;
  const int kt1 = min(p.ktiles, kt0 + p.kt_per_split);
  const int nk = kt1 - kt0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], kProducerThreads);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(done_bar, 1);
    fence_mbar_init();
  }
  if (warp == kProducerWarps) {
    tmem_alloc(tmem_slot, BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t smem_base = smem_u32(smem);

  if (warp < kProducerWarps) {
    // ------------------------------------------------------------ producers
    const int t = threadIdx.x;
    for (int i = 0; i < nk; ++i) {
      const int s = i % STAGES;
      mbar_wait_bounded(&empty_bar[s], ((i / STAGES) & 1) ^ 1, p.err, kErrWaitEmpty);
      const uint32_t a_tile = smem_base + s * L::kStage;
      const uint32_t b_tile = a_tile + L::kATile;
      const int64_t kbase = static_cast<int64_t>(kt0 + i) * kBK;
      fill_tile<PASS, true, FMT, kBM>(p, p.a, a_tile, m0, kbase, t);
      fill_tile<PASS, false, FMT, BN>(p, p.b, b_tile, n0, kbase, t);
      fence_proxy_async_smem();
      mbar_arrive(&full_bar[s]);
    }
    // ------------------------------------------------------------ epilogue
    mbar_wait_bounded(done_bar, 0, p.err, kErrWaitDone);
    tc_fence_after();
    const float scale = p.scale_out ? __fmul_rn(*p.a.tscale, *p.b.tscale) : 1.0f;
    const int quarter = warp & 3;
    const int64_t row = m0 + quarter * 32 + lane;       // GEMM row of this thread
    constexpr int kColsPerWarp = BN / 2;
    const int col_begin = (warp >> 2) * kColsPerWarp;
#pragma unroll 1
    for (int c = 0; c < kColsPerWarp; c += 16) {
      uint32_t r[16];
      tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + col_begin + c, r);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t col = n0 + col_begin + c + 4 * j;
        if (row >= p.M || col >= p.Ncols) continue;
        float4 o;
        o.x = __uint_as_float(r[4 * j + 0]) * scale;
        o.y = __uint_as_float(r[4 * j + 1]) * scale;
        o.z = __uint_as_float(r[4 * j + 2]) * scale;
        o.w = __uint_as_float(r[4 * j + 3]) * scale;
        if (nk == 0) o = make_float4(0.f, 0.f, 0.f, 0.f);
        int64_t idx;
        if (PASS == kWgrad) {
          idx = (static_cast<int64_t>(blockIdx.z) * p.M + row) * p.Ncols + col;
        } else {
          const int64_t pix = col / p.N;
          idx = (pix * p.M + row) * p.N + (col - pix * p.N);
        }
        *reinterpret_cast<float4*>(p.out + idx) = o;
      }
    }
  } else if (lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc = idesc_f16_f32(kBM, BN);
    for (int i = 0; i < nk; ++i) {
      const int s = i % STAGES;
      mbar_wait_bounded(&full_bar[s], (i / STAGES) & 1, p.err, kErrWaitFull);
      tc_fence_after();
      const uint32_t a_tile = smem_base + s * L::kStage;
      const uint64_t adesc = smem_desc_sw128(a_tile);
      const uint64_t bdesc = smem_desc_sw128(a_tile + L::kATile);
#pragma unroll
      for (int kk = 0; kk < kBK / 16; ++kk) {
        // advance 16 fp16 = 32 bytes along K inside the swizzled row
        mma_f16_ss(tmem, adesc + 2 * kk, bdesc + 2 * kk, idesc, (i > 0 || kk > 0) ? 1u : 0u);
      }
      mma_commit(&empty_bar[s]);
    }
    mma_commit(done_bar);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kProducerWarps) {
    tc_fence_after();
    tmem_dealloc(tmem, BN);
  }
}

// G_W = T_g·T_x·sum over splits of the partial tiles, in split order.
__global__ void __launch_bounds__(256)
wgrad_reduce_kernel(const float4* __restrict__ partial, int splits, int64_t n4,
                    const float* __restrict__ ta, const float* __restrict__ tb,
                    float4* __restrict__ out) {
  const float scale = __fmul_rn(*ta, *tb);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 acc = __ldg(partial + i);
    for (int s = 1; s < splits; ++s) {
      const float4 v = __ldg(partial + s * n4 + i);
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    acc.x *= scale;
    acc.y *= scale;
    acc.z *= scale;
    acc.w *= scale;
    out[i] = acc;
  }
}

}  // namespace mqv
