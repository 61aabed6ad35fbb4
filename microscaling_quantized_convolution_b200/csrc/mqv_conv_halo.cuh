// Stride-1 forward and input-gradient convolution with the im2col tile built
// once per kernel row on chip (MicroQonv summary, onedev.kr/papers/182,
// section "어떻게 동작하나": the channel-batch-first layout lets the window
// slide over channel/batch runs read once and reused on chip).
//
// A CTA owns an output tile of BW consecutive pixels of one output row x all
// N batch items (BW·N <= 256 GEMM columns) x 128 output channels; the host
// picks BW to balance the tiles over the SMs.  For
// each kernel row kh and 64-channel chunk of the reduction, the producer
// warps dequantize the BW + Kw - 1 source pixels the window touches (the
// "halo") into one K-major shared tile; the Kw taps of that kernel row are
// then Kw MMA groups on the same tile, each starting kw·N rows further on
// (a descriptor offset: N % 8 == 0 keeps it on the 8-row swizzle atom).  So
// every source pixel is dequantized once per kernel row instead of once per
// tap, and every MMA is 128 x BW·N x 16.
//
// Forward:        source = X,   row  hi = ho + kh - pad,  columns wi = wo0 - pad + q,
//                 tap kw uses halo pixels q = j + kw.
// Input gradient: source = G_Y, row  ho = hi + pad - kh,  columns wo = wi0 + pad - (Kw-1) + q,
//                 tap kw uses halo pixels q = j + (Kw - 1 - kw).
// The weight operand is the fp16 image of prep_image_kernel (tap-major K, so
// the tile of (tap, chunk) is image tile tap·(Cred/64) + chunk), one 16 KB
// bulk copy per tap, the Kw tiles of a stage under one barrier.  Roles,
// bounded waits and the double-buffered accumulators are those of
// conv_fd_kernel.
#pragma once

#include <cstdint>

#include "mqv_conv_common.cuh"
#include "mqv_conv_kernels.cuh"
#include "mqv_ptx.cuh"

namespace mqv {

constexpr int kHaloBN = 256;                  // most GEMM columns per tile (TMEM spacing of the accumulators)
constexpr int kHaloMaxRows = 384;             // halo rows: 256 + (Kw - 1)·N <= 384
constexpr int kHaloBStages = 2;
constexpr int kHaloAStages = 6;
constexpr int kHaloLookahead = 2;                        // stages of codes in flight per producer (block-scaled kernel)
constexpr int kHaloProdWarps = 12;                       // one 8 x 8 unit per thread per stage
constexpr int kHaloProdThreads = kHaloProdWarps * 32;    // 384 = the largest halo
constexpr int kHaloThreads = (kV2ProdWarp0 + kHaloProdWarps) * 32;
constexpr uint32_t kHaloBTile = kHaloMaxRows * 128;   // 48 KB

struct HaloSmem {
  static constexpr int kAOffset = 0;                                  // kHaloAStages weight tiles
  static constexpr int kBOffset = kHaloAStages * kATileBytes;
  static constexpr int kEpiOffset = kBOffset + kHaloBStages * kHaloBTile;   // 32 x 32 fp32 per epilogue warp
  static constexpr int kBarOffset = kEpiOffset + kV2EpiWarps * 4096;
  static constexpr int kBytes = kBarOffset + 512 + 1024;
};

struct HaloBars {
  uint64_t afull[kHaloAStages];
  uint64_t aempty[kHaloAStages];
  uint64_t bfull[kHaloBStages];
  uint64_t bempty[kHaloBStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t last_full;   // the CTA's last tile accumulated (one phase; see the producers' last epilogue)
  uint32_t tmem;
};

// Geometry of the halo pass (filled by the host).
struct HaloGeom {
  int bw;             // output pixels per tile
  int bn;             // GEMM columns per tile, bw·N (a multiple of 16, <= 256)
  int rows;           // halo rows (bw + Kw - 1)·N
  int tpr;            // tiles per output row
  int cchunks;        // 64-channel chunks of the reduction
  int out_h, out_w;   // output pixel grid of the pass
  int src_h, src_w;   // source pixel grid
};

// Raw codes of one halo unit: 8 batch items (rows) x 8 channels (K).
struct HaloUnit {
  uint32_t w[8];      // codes of channel c0 + j for the 8 batch items (NVFP6: bytes 0-3)
  uint32_t wh[8];     // NVFP6: bytes 4-5 of the 6-byte run
  uint32_t s[2];      // scales of channel blocks 0/1 (low byte: batch block 0);
                      // 16 x 1 line blocks: byte j of s[0], s[1] = batch item j, 4 + j
  bool ok;
};

// Transposed dequantize of one unit (halo_dequant_unit, into registers) and
// its store (halo_st_unit): row row0 + r of the tile gets the 8 channels
// (c0..c0+7) of batch item n0 + r at K chunk kg.  Each pair of
// channel words is interleaved nibble-wise first, so one cvt.e2m1x2 per
// byte yields the (channel 2i, channel 2i+1) pair of one batch item.
// LINE: the operand has 16 x 1 line blocks down its (pixel, channel) rows, so
// the unit's 8 channels share one scale per batch item.
template <int FMT, bool LINE>
__device__ __forceinline__ void halo_dequant_unit(const HaloUnit& u, uint32_t (&out)[8][4]) {
  uint32_t sl[8];
  if (LINE) {
#pragma unroll
    for (int r = 0; r < 8; ++r) sl[r] = scale2((u.s[r >> 2] >> (8 * (r & 3))) & 0xFF);
  }
  if (u.ok && FMT == 1) {
    // NVFP6: batch item r of channel c is bits [6r, 6r+6) of the 48-bit run;
    // the two channels of a pair go to the low and high byte of one
    // cvt.e2m3x2 input, giving the (2i, 2i+1) fp16 pair directly.
    const uint32_t sc[2][2] = {{scale2(u.s[0] & 0xFF), scale2(u.s[0] >> 8)},
                               {scale2(u.s[1] & 0xFF), scale2(u.s[1] >> 8)}};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint64_t a = u.w[2 * i] | (static_cast<uint64_t>(u.wh[2 * i]) << 32);
      const uint64_t b = u.w[2 * i + 1] | (static_cast<uint64_t>(u.wh[2 * i + 1]) << 32);
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const uint32_t v = static_cast<uint32_t>((a >> (6 * r)) & 0x3F) |
                           (static_cast<uint32_t>((b >> (6 * r)) & 0x3F) << 8);
        out[r][i] = hmul2_u32(e2m3x2_to_f16x2(v), LINE ? sl[r] : sc[i >> 1][r >> 2]);
      }
    }
  } else if (u.ok) {
    const uint32_t sc[2][2] = {{scale2(u.s[0] & 0xFF), scale2(u.s[0] >> 8)},    // [channel block][batch block]
                               {scale2(u.s[1] & 0xFF), scale2(u.s[1] >> 8)}};
#pragma unroll
    for (int i = 0; i < 4; ++i) {                         // channel pair (2i, 2i+1)
      const uint32_t a = u.w[2 * i], b = u.w[2 * i + 1];
      const uint32_t even = (a & 0x0F0F0F0Fu) | ((b & 0x0F0F0F0Fu) << 4);   // batch items 0,2,4,6
      const uint32_t odd = ((a >> 4) & 0x0F0F0F0Fu) | (b & 0xF0F0F0F0u);    // batch items 1,3,5,7
      uint32_t he[4], ho[4];
      e2m1x8_to_f16x2(even, he);
      e2m1x8_to_f16x2(odd, ho);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t s2 = sc[i >> 1][q >> 1];             // batch items 2q, 2q+1: block q/2
        out[2 * q][i] = hmul2_u32(he[q], LINE ? sl[2 * q] : s2);
        out[2 * q + 1][i] = hmul2_u32(ho[q], LINE ? sl[2 * q + 1] : s2);
      }
    }
  } else {
#pragma unroll
    for (int r = 0; r < 8; ++r) out[r][0] = out[r][1] = out[r][2] = out[r][3] = 0u;
  }
}

__device__ __forceinline__ void halo_st_unit(const uint32_t (&out)[8][4], uint32_t tile, uint32_t row0, uint32_t kg) {
#pragma unroll
  for (int r = 0; r < 8; ++r)
    st_shared_v4(tile + sw128_offset(row0 + r, 8 * kg), out[r][0], out[r][1], out[r][2], out[r][3]);
}

// Producer thread t owns unit t of every stage: K chunk kg = t % 8 (8
// channels), rows 8(t/8)..8(t/8)+7 of the halo.  Lanes of an 8-lane phase
// differ in kg, so their 16-byte stores hit 8 different swizzled chunks.
template <int PASS, int FMT, bool LINE = false>
struct HaloCursor {
  int sc, n0;         // halo pixel column in the source, first batch item
  bool cok;           // unit inside the halo and its column inside the source

  __device__ __forceinline__ void begin_tile(const V2Args& p, const HaloGeom& g, int tile, int t) {
    const int oh = tile / g.tpr;
    const int ow0 = (tile - oh * g.tpr) * g.bw;
    const int base = PASS == kFwd ? ow0 - p.pad : ow0 + p.pad - (p.Kw - 1);
    const int r = 8 * (t >> 3);
    const int q = fdiv(r, p.dN);
    n0 = r - q * p.N;
    sc = base + q;
    cok = t < g.rows && sc >= 0 && sc < g.src_w;
  }

  __device__ __forceinline__ void load(const V2Args& p, const HaloGeom& g, int tile, int kh, int c, int t,
                                       HaloUnit& u) const {
    const int oh = tile / g.tpr;
    const int sr = PASS == kFwd ? oh + kh - p.pad : oh + p.pad - kh;
    u.ok = cok && sr >= 0 && sr < g.src_h;
    if (!u.ok) return;
    const int64_t row0 = (static_cast<int64_t>(sr) * g.src_w + sc) * p.Cred + 64 * c + 8 * (t & 7);
    if (FMT == 0) {
      const uint8_t* cp = p.b.codes + row0 * p.b.row_bytes + (n0 >> 1);
#pragma unroll
      for (int j = 0; j < 8; ++j) u.w[j] = __ldg(reinterpret_cast<const uint32_t*>(cp + j * p.b.row_bytes));
    } else {
      // 6 bytes at a 2-byte aligned offset (n0 is a multiple of 8)
      const uint8_t* cp = p.b.codes + row0 * p.b.row_bytes + ((n0 * 3) >> 2);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const unsigned short* q = reinterpret_cast<const unsigned short*>(cp + j * p.b.row_bytes);
        u.w[j] = static_cast<uint32_t>(__ldg(q)) | (static_cast<uint32_t>(__ldg(q + 1)) << 16);
        u.wh[j] = __ldg(q + 2);
      }
    }
    if (LINE) {
      // rows row0 .. row0 + 7 lie in one 16-row block (row0 % 8 == 0)
      const uint2 sv = __ldg(reinterpret_cast<const uint2*>(p.b.scales + (row0 >> 4) * p.b.scale_cols + n0));
      u.s[0] = sv.x;
      u.s[1] = sv.y;
      return;
    }
    const uint8_t* sp = p.b.scales + (row0 >> 2) * p.b.scale_cols + (n0 >> 2);
    u.s[0] = __ldg(reinterpret_cast<const unsigned short*>(sp));
    u.s[1] = __ldg(reinterpret_cast<const unsigned short*>(sp + p.b.scale_cols));
  }
};

// Epilogue of one tile (accumulator at TMEM column acc_col) for the warp on
// TMEM lane quarter `quarter`: the 32-column chunks first, first + stride,
// ... of the accumulator.  Each lane
// reads one accumulator row from TMEM; a swizzled 32 x 32 transpose in the
// warp's 4 KB of shared memory (wbuf) turns that into stores of 128-byte runs
// of one (pixel, channel) row's batch items.  Columns past bw·N hold no
// output (j >= bw below).
// With p.q_codes set the values are quantized instead of stored: a 4 x 4
// block of the next operand is 4 channel rows x 4 batch items at one pixel,
// held by the lanes q, q + 8, q + 16, q + 24 (rows 4i .. 4i + 3), so two
// shuffles give its max|x|, and each lane quantizes its row of the block
// with the quantizer's own arithmetic (RND 0: round to nearest, 1:
// stochastic with the element's Philox word).
template <int FMT, int RND>
__device__ __forceinline__ void halo_quantize_row(const V2Args& p, float4 o, bool ok, int64_t row, int n,
                                                  const TensorScale<FMT>& ts, int rsub) {
  float bm = ok ? absmax4(o) : 0.0f;
  bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 8));
  bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 16));
  if (!ok) return;
  const BlockScale<FMT> bs(bm, ts);
  uint4 w = make_uint4(0u, 0u, 0u, 0u);
  if (RND == 1) {
    const uint64_t gc = static_cast<uint64_t>(row * p.N + n) >> 2;
    w = philox4x32_10(make_uint4(static_cast<uint32_t>(gc), static_cast<uint32_t>(gc >> 32), 0u, 0u), p.q_keys);
  }
  const uint32_t packed = quantize_row4<FMT, RND>(o, bs.d, bs.y, bs.exact, w);
  if (FMT == 0) {
    *reinterpret_cast<uint16_t*>(p.q_codes + row * (p.N >> 1) + (n >> 1)) = static_cast<uint16_t>(packed);
  } else {
    uint8_t* c = p.q_codes + row * ((p.N * 3) >> 2) + ((n * 3) >> 2);
    c[0] = static_cast<uint8_t>(packed);
    c[1] = static_cast<uint8_t>(packed >> 8);
    c[2] = static_cast<uint8_t>(packed >> 16);
  }
  if (rsub == 0) p.q_scales[(row >> 2) * (p.N >> 2) + (n >> 2)] = static_cast<uint8_t>(bs.scode);
}

template <int FMT, int RND, bool QOUT>
__device__ __forceinline__ void halo_epilogue_tile(const V2Args& p, const HaloGeom& g, uint32_t tmem, int acc_col,
                                                   int tile, int quarter, uint32_t wbuf, int first, int stride,
                                                   float& amax) {
  const int lane = threadIdx.x & 31;
  const int rsub = lane >> 3, q = lane & 7;
  const int mt = tile / (g.out_h * g.tpr);
  const int rest = tile - mt * g.out_h * g.tpr;
  const int oh = rest / g.tpr;
  const int ow0 = (rest - oh * g.tpr) * g.bw;
  if (mt * 128 + quarter * 32 >= p.M) return;   // all 32 rows of this quarter past the M channels
  const float scale = __fmul_rn(*p.ta, *p.tb);
  const uint32_t tbase = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + acc_col;
#pragma unroll 1
  for (int c = 32 * first; c < g.bn; c += 32 * stride) {
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      uint32_t r[16];
      tmem_ld_32x32b_x16(tbase + c + 16 * hf, r);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 4; ++j)
        st_shared_v4(wbuf + lane * 128 + (((4 * hf + j) ^ (lane & 7)) << 4),
                     __float_as_uint(__uint_as_float(r[4 * j + 0]) * scale),
                     __float_as_uint(__uint_as_float(r[4 * j + 1]) * scale),
                     __float_as_uint(__uint_as_float(r[4 * j + 2]) * scale),
                     __float_as_uint(__uint_as_float(r[4 * j + 3]) * scale));
    }
    __syncwarp();
    const int lc = c + 4 * q;
    const int j = fdiv(lc, p.dN);
    const int n = lc - j * p.N;
    const int ow = ow0 + j;
    const bool colok = j < g.bw && ow < g.out_w;
    const int64_t pix = static_cast<int64_t>(oh) * g.out_w + ow;
    if (QOUT) {
      // every lane takes part in the block-max shuffles
      const TensorScale<FMT> ts(*p.q_amax);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int row = 4 * i + rsub;
        const int64_t mrow = static_cast<int64_t>(mt) * 128 + quarter * 32 + row;
        float4 o = ld_shared_v4_f32(wbuf + row * 128 + ((q ^ (row & 7)) << 4));
        const bool ok = colok && mrow < p.M;
        if (p.relu) o = epi_relu(o);
        if (ok && p.amax_out) amax = epi_absmax(amax, o);
        halo_quantize_row<FMT, RND>(p, o, ok, pix * p.M + mrow, n, ts, rsub);
      }
    } else if (colok) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int row = 4 * i + rsub;
        const int64_t mrow = static_cast<int64_t>(mt) * 128 + quarter * 32 + row;
        float4 o = ld_shared_v4_f32(wbuf + row * 128 + ((q ^ (row & 7)) << 4));
        if (mrow < p.M) {
          if (p.relu) o = epi_relu(o);
          if (p.amax_out) amax = epi_absmax(amax, o);
          *reinterpret_cast<float4*>(p.out + (pix * p.M + mrow) * p.N + n) = o;
        }
      }
    }
    __syncwarp();
  }
}

// QOUT: the quantized-output epilogue (V2Args::q_codes), a separate
// instance so that the plain passes keep their code and registers.  LINE:
// the B operand has 16 x 1 line blocks (see halo_dequant_unit).
template <int PASS, int FMT, bool QOUT, bool LINE = false>
__global__ void __launch_bounds__(kHaloThreads, 1)
conv_halo_kernel(const V2Args p, const HaloGeom g) {
  using L = HaloSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  HaloBars* bars = reinterpret_cast<HaloBars*>(smem + L::kBarOffset);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kHaloAStages; ++s) {
      mbar_init(&bars->afull[s], 1);
      mbar_init(&bars->aempty[s], 1);
    }
    for (int s = 0; s < kHaloBStages; ++s) {
      mbar_init(&bars->bfull[s], kHaloProdWarps);
      mbar_init(&bars->bempty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&bars->acc_full[a], 1);
      mbar_init(&bars->acc_empty[a], kV2EpiWarps * 32);
    }
    mbar_init(&bars->last_full, 1);
    fence_mbar_init();
  }
  if (warp == kV2MmaWarp) {
    tmem_alloc(&bars->tmem, 2 * kHaloBN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t sbase = smem_u32(smem);
  const int stages_per_tile = p.Kh * g.cchunks;
  const int na = kHaloAStages / p.Kw;     // weight stages in the ring (Kw <= kHaloAStages)

  if (QOUT && blockIdx.x == 0 && threadIdx.x == 0) *p.q_tscale = TensorScale<FMT>(*p.q_amax).T;
  if (warp < kV2EpiWarps) {
    // epilogue: column lc of the tile = (pixel j, batch item n) -> output
    // pixel (oh, ow0 + j), skipped past the end of the output row.  The
    // CTA's last tile is shared with the producer warps (which are done by
    // then): warp `warp` takes the 32-column chunks 0, 4, 8, ... of it.
    int it = 0;
    float amax = 0.f;
    const uint32_t wbuf = sbase + L::kEpiOffset + warp * 4096;
    for (int tile = blockIdx.x; tile < p.tiles; tile += gridDim.x, ++it) {
      const int acc = it & 1;
      mbar_wait_bounded(&bars->acc_full[acc], (it >> 1) & 1, p.err, kErrWaitDone);
      tc_fence_after();
      const bool last = tile + static_cast<int>(gridDim.x) >= p.tiles;
      halo_epilogue_tile<FMT, PASS == kDgrad, QOUT>(p, g, bars->tmem, acc * kHaloBN, tile, warp & 3, wbuf, 0,
                                                    last ? 4 : 1, amax);
      tc_fence_before();
      mbar_arrive(&bars->acc_empty[acc]);
    }
    epi_amax_flush(p.amax_out, amax);
  } else if (warp == kV2MmaWarp) {
    if (lane == 0) {
      // The issuing thread's own instructions sit on the critical path of
      // every stage, so everything per stage is a counter or an add:
      // descriptors are base + offset in 16-byte units, ring slots and their
      // phases are counters (no division).
      const uint32_t idesc = idesc_f16_f32(128, g.bn);
      const uint64_t adesc0 = smem_desc_sw128(sbase + L::kAOffset);
      const uint64_t bdesc0 = smem_desc_sw128(sbase + L::kBOffset);
      constexpr uint32_t kATileDesc = kATileBytes >> 4;
      constexpr uint32_t kBTileDesc = kHaloBTile >> 4;
      const uint32_t a_stage_desc = static_cast<uint32_t>(p.Kw) * kATileDesc;
      const uint32_t tap_desc = static_cast<uint32_t>(p.N) * 8u;      // N rows of 128 B
      int it = 0, sb = 0, sa = 0;
      uint32_t pb = 0, pa = 0;                                         // ring phases
      for (int tile = blockIdx.x; tile < p.tiles; tile += gridDim.x, ++it) {
        const int acc = it & 1;
        mbar_wait_bounded(&bars->acc_empty[acc], ((it >> 1) & 1) ^ 1, p.err, kErrWaitEmpty);
        tc_fence_after();
        const uint32_t dt = bars->tmem + acc * kHaloBN;
        for (int st = 0; st < stages_per_tile; ++st) {
          mbar_wait_bounded(&bars->bfull[sb], pb, p.err, kErrWaitFull);
          mbar_wait_bounded(&bars->afull[sa], pa, p.err, kErrWaitFull);
          tc_fence_after();
          const uint64_t ad = adesc0 + static_cast<uint32_t>(sa) * a_stage_desc;
          const uint64_t bd = bdesc0 + static_cast<uint32_t>(sb) * kBTileDesc;
          for (int kw = 0; kw < p.Kw; ++kw) {
            const uint32_t shift = PASS == kFwd ? kw : p.Kw - 1 - kw;
            const uint64_t a_k = ad + static_cast<uint32_t>(kw) * kATileDesc;
            const uint64_t b_k = bd + shift * tap_desc;
            const uint32_t acc0 = (st | kw) ? 1u : 0u;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_f16_ss(dt, a_k + 2 * kk, b_k + 2 * kk, idesc, kk ? 1u : acc0);
          }
          mma_commit(&bars->aempty[sa]);
          mma_commit(&bars->bempty[sb]);
          if (++sb == kHaloBStages) {
            sb = 0;
            pb ^= 1u;
          }
          if (++sa == na) {
            sa = 0;
            pa ^= 1u;
          }
        }
        mma_commit(&bars->acc_full[acc]);
        if (tile + static_cast<int>(gridDim.x) >= p.tiles) mma_commit(&bars->last_full);
      }
    }
  } else if (warp == kV2LoadWarp) {
    if (lane == 0) {
      int sa = 0;
      uint32_t pa = 1;                 // first pass: the empty slots count as released
      // the weight image comes from the kernel before this one, which this
      // kernel may overlap (programmatic dependent launch): wait for it
      pdl_wait_prerequisite();
      for (int tile = blockIdx.x; tile < p.tiles; tile += gridDim.x) {
        const int mt = tile / (g.out_h * g.tpr);
        const uint8_t* img = p.image + static_cast<int64_t>(mt) * p.ktiles * kATileBytes;
        for (int kh = 0; kh < p.Kh; ++kh)
          for (int c = 0; c < g.cchunks; ++c) {
            // the Kw weight tiles of the stage, under one barrier
            mbar_wait_bounded(&bars->aempty[sa], pa, p.err, kErrWaitEmpty);
            mbar_arrive_expect_tx(&bars->afull[sa], p.Kw * kATileBytes);
            for (int kw = 0; kw < p.Kw; ++kw) {
              const int kt = (kh * p.Kw + kw) * g.cchunks + c;
              bulk_copy_g2s(sbase + L::kAOffset + (sa * p.Kw + kw) * kATileBytes,
                            img + static_cast<int64_t>(kt) * kATileBytes, kATileBytes, &bars->afull[sa]);
            }
            if (++sa == na) {
              sa = 0;
              pa ^= 1u;
            }
          }
      }
    }
  } else {
    // producers: the next stage's unit is dequantized into registers while
    // the MMAs read the current one, so between a slot's release (bempty)
    // and its refill signal (bfull) a producer only stores; the unit after
    // that is loaded one stage ahead.
    const int t = threadIdx.x - kV2ProdWarp0 * 32;
    const int ntile_cta = (p.tiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                          static_cast<int>(gridDim.x);
    const int total = ntile_cta * stages_per_tile;
    const int spatial = g.out_h * g.tpr;
    HaloCursor<PASS, FMT, LINE> cursor;
    HaloUnit raw;
    uint32_t out[8][4];
    int ltile = blockIdx.x, lkh = 0, lc = 0;
    if (total > 0) cursor.begin_tile(p, g, ltile % spatial, t);
    auto load_next = [&](HaloUnit& u) {
      cursor.load(p, g, ltile % spatial, lkh, lc, t, u);
      if (++lc == g.cchunks) {
        lc = 0;
        if (++lkh == p.Kh) {
          lkh = 0;
          ltile += gridDim.x;
          if (ltile < p.tiles) cursor.begin_tile(p, g, ltile % spatial, t);
        }
      }
    };
    if (total > 0) {
      load_next(raw);
      halo_dequant_unit<FMT, LINE>(raw, out);
      if (total > 1) load_next(raw);
    }
    for (int kit = 0; kit < total; ++kit) {
      const int sb = kit % kHaloBStages;
      mbar_wait_bounded(&bars->bempty[sb], ((kit / kHaloBStages) & 1) ^ 1, p.err, kErrWaitEmpty);
      if (t < g.rows)
        halo_st_unit(out, sbase + L::kBOffset + sb * kHaloBTile, static_cast<uint32_t>(8 * (t >> 3)),
                     static_cast<uint32_t>(t & 7));
      producer_warp_arrive(&bars->bfull[sb]);
      if (kit + 1 < total) {
        halo_dequant_unit<FMT, LINE>(raw, out);
        if (kit + 2 < total) load_next(raw);
      }
    }    // The CTA's last tile: once its accumulator is complete (so the B ring
    // is no longer read), producer warp w takes chunks 1, 2 or 3 (of every 4)
    // on TMEM lane quarter w % 4, staging through 4 KB of the B ring.
    if (ntile_cta > 0) {
      const int lit = ntile_cta - 1;
      const int ltile_last = static_cast<int>(blockIdx.x) + lit * static_cast<int>(gridDim.x);
      const int pw = warp - kV2ProdWarp0;
      float amax = 0.f;
      // The producers can finish their last stage more than one accumulator
      // phase ahead of the MMAs (a 1 x 1 layer has one stage a tile), and a
      // parity wait on acc_full would then alias an earlier phase: the last
      // tile has its own single-phase barrier.
      mbar_wait_bounded(&bars->last_full, 0, p.err, kErrWaitDone);
      tc_fence_after();
      halo_epilogue_tile<FMT, PASS == kDgrad, QOUT>(p, g, bars->tmem, (lit & 1) * kHaloBN, ltile_last, warp & 3,
                                                    sbase + L::kBOffset + pw * 4096, 1 + pw / 4, 4, amax);
      epi_amax_flush(p.amax_out, amax);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kV2MmaWarp) {
    tc_fence_after();
    tmem_dealloc(bars->tmem, 2 * kHaloBN);
  }
}

}  // namespace mqv
