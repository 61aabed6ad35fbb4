// Stride-1 forward pass on the native block-scaled MMA of sm_100a
// (tcgen05.mma kind::mxf4nvf4: E2M1 operands, one UE4M3 scale per 16
// consecutive K elements of a row), kept to compare the two MMA forms the
// method can use (MicroQonv summary, onedev.kr/papers/182, section
// "무엇과 다른가": 4 x 4 square blocks with E4M3 block scales).
//
// A square block has only 4 elements along K in each of its rows, so the
// only exact mapping onto 16-element scale groups pads every 4-element block
// row with 12 zero codes: a 64-channel chunk becomes 16 groups of 16 codes
// (4 codes + 12 zeros, 8 bytes), 128 bytes a row, the same bytes as the
// chunk in fp16; each MMA of K = 64 padded codes covers 16 real channels.
// The codes enter the MMA as they are (no dequantization); the block scales
// go to tensor memory.
//
// Structure: the kernel-row halo pass of conv_halo_kernel (same tiles, roles
// and barriers) with
//   A = the padded weight image (16 KB of codes a tap chunk) plus its scale
//       atoms (2 KB), one bulk copy per tap; the MMA thread moves the scale
//       atoms into tensor memory with tcgen05.cp before the tap's MMAs;
//   B = the halo tile of padded codes, and its scale atoms, both written by
//       the producer warps into shared memory; tcgen05.cp again.
// Scale layout in tensor memory (the 32x128b.warpx4 copy of a 512-byte atom
// holding rows m0 + 32·m1, m0 < 32, m1 < 4, byte m0·16 + m1·4 + group):
// the scales of row r sit in lane r % 32 (of every lane quarter), column
// base + r / 32, one byte per 16-element group, so the taps' row shift of
// kw·N halo rows is a column offset of kw·N / 32 (even for N = 64 and 128:
// a scale-factor address must be an even column).
#pragma once

#include <cstdint>

#include "mqv_conv_common.cuh"
#include "mqv_conv_halo.cuh"
#include "mqv_conv_kernels.cuh"
#include "mqv_ptx.cuh"

namespace mqv {

constexpr int kNvf4BN = 128;                              // GEMM columns per tile
constexpr int kNvf4MaxRows = 256;                         // halo rows
constexpr int kNvf4AStages = 6;                           // weight taps in the A ring
constexpr int kNvf4BStages = 2;
constexpr uint32_t kNvf4ATile = kATileBytes + 2048;       // padded codes + 4 scale atoms
constexpr uint32_t kNvf4BTile = kNvf4MaxRows * 128;       // 32 KB
constexpr uint32_t kNvf4BSf = 4 * 2 * 512;                // 4 k-steps x 2 atoms of 128 halo rows
constexpr int kNvf4ProdWarps = kNvf4MaxRows / 32;         // one 8 x 8 unit per thread: 8 warps
constexpr int kNvf4Threads = (kV2ProdWarp0 + kNvf4ProdWarps) * 32;   // 448
// TMEM columns: accumulators at 0 and 128; the scales of B stage s at
// 256 + 80·s: A (tap kw, k-step ks) at +4·(4·kw + ks), B (k-step ks) at
// +48 + 8·ks.
constexpr int kNvf4SfCol = 256, kNvf4SfStage = 80, kNvf4SfB = 48;

struct Nvf4Smem {
  static constexpr int kAOffset = 0;
  static constexpr int kBOffset = kNvf4AStages * kNvf4ATile;
  static constexpr int kBSfOffset = kBOffset + kNvf4BStages * kNvf4BTile;
  static constexpr int kEpiOffset = kBSfOffset + kNvf4BStages * kNvf4BSf;
  static constexpr int kBarOffset = kEpiOffset + kV2EpiWarps * 4096;
  static constexpr int kBytes = kBarOffset + 512 + 1024;
};

// Instruction descriptor, kind::mxf4nvf4: A and B E2M1 (K-major), UE4M3
// scales, fp32 D, scale ids 0.
__host__ __device__ constexpr uint32_t idesc_nvf4(int M, int N) {
  return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_nvf4_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// 32 rows x 16 bytes of shared memory (one 512-byte scale atom) to 4
// columns of every TMEM lane quarter.
__device__ __forceinline__ void tmem_cp_atom(uint32_t taddr, uint32_t saddr) {
  // no-swizzle matrix descriptor: 8-row x 16-byte core matrices 128 bytes
  // apart along the rows
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>(1) << 16;                         // LBO (one core matrix along K)
  d |= static_cast<uint64_t>(128 >> 4) << 32;                  // SBO = 128 B
  d |= static_cast<uint64_t>(1) << 46;                         // descriptor version
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(d) : "memory");
}

// Byte offset of (halo row h, group byte k1) inside the scale atoms of k-step ks.
__device__ __forceinline__ uint32_t nvf4_sf_offset(uint32_t h, uint32_t ks, uint32_t k1) {
  return (ks * 2 + (h >> 7)) * 512 + (h & 31) * 16 + ((h >> 5) & 3) * 4 + k1;
}

// Padded codes of one producer unit (8 batch items x 8 channels): row r of
// the tile gets, at K chunk kg, group 2kg (channels 0-3 of the unit) and
// group 2kg + 1 (channels 4-7), each 4 codes and 12 zeros; the two scale
// bytes of the row go to the B scale atoms.
__device__ __forceinline__ void nvf4_store_unit(const HaloUnit& u, uint32_t tile, uint32_t sf, uint32_t row0,
                                                uint32_t kg) {
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    uint32_t g0 = 0, g1 = 0, s = 0;
    if (u.ok) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        g0 |= ((u.w[j] >> (4 * r)) & 0xFu) << (4 * j);
        g1 |= ((u.w[4 + j] >> (4 * r)) & 0xFu) << (4 * j);
      }
      // channel block 0 / 1 of the unit, batch block r / 4
      s = ((u.s[0] >> (8 * (r >> 2))) & 0xFFu) | (((u.s[1] >> (8 * (r >> 2))) & 0xFFu) << 8);
    }
    st_shared_v4(tile + sw128_offset(row0 + r, 8 * kg), g0, 0u, g1, 0u);
    asm volatile("st.shared.u16 [%0], %1;" ::"r"(sf + nvf4_sf_offset(row0 + r, kg >> 1, 2 * (kg & 1))),
                 "h"(static_cast<uint16_t>(s))
                 : "memory");
  }
}

// Weight image of the block-scaled form: tile (mt, kt) = 128 rows x 64
// channels of W, K-major and 128-byte swizzled like the fp16 image, each
// 4-element block row padded to 16 codes (8 bytes), then the 4 scale atoms
// of the tile's k-steps (2 KB).  One thread per 8-element chunk of a row.
__global__ void __launch_bounds__(kPrepThreads)
prep_nvf4_image_kernel(QView w, int M, int ktiles, int mtiles, FastDiv dkt8, uint8_t* __restrict__ image) {
  const int chunks = mtiles * 128 * ktiles * 8;
  const int id = blockIdx.x * kPrepThreads + threadIdx.x;
  if (id >= chunks) return;
  const int m = fdiv(id, dkt8);
  const int k0 = (id - m * ktiles * 8) * 8;
  const int mt = m >> 7, r = m & 127, kt = k0 >> 6, kc = (k0 & 63) >> 3;
  uint32_t word = 0, sc = 0;
  if (m < M) {
    word = __ldg(reinterpret_cast<const uint32_t*>(w.codes + static_cast<int64_t>(m) * w.row_bytes + (k0 >> 1)));
    if ((kc & 1) == 0)
      sc = __ldg(reinterpret_cast<const uint32_t*>(w.scales + static_cast<int64_t>(m >> 2) * w.scale_cols + (k0 >> 2)));
  }
  uint8_t* tile = image + (static_cast<int64_t>(mt) * ktiles + kt) * kNvf4ATile;
  *reinterpret_cast<uint4*>(tile + r * 128 + ((kc ^ (r & 7)) << 4)) = make_uint4(word & 0xFFFFu, 0u, word >> 16, 0u);
  if ((kc & 1) == 0)
    *reinterpret_cast<uint32_t*>(tile + kATileBytes + (kc >> 1) * 512 + (r & 31) * 16 + (r >> 5) * 4) = sc;
}

struct Nvf4Bars {
  uint64_t afull[kNvf4AStages];
  uint64_t aempty[kNvf4AStages];
  uint64_t bfull[kNvf4BStages];
  uint64_t bempty[kNvf4BStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t last_full;
  uint32_t tmem;
};

__global__ void __launch_bounds__(kNvf4Threads, 1)
conv_fwd_nvf4_kernel(const V2Args p, const HaloGeom g) {
  using L = Nvf4Smem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Nvf4Bars* bars = reinterpret_cast<Nvf4Bars*>(smem + L::kBarOffset);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kNvf4AStages; ++s) {
      mbar_init(&bars->afull[s], 1);
      mbar_init(&bars->aempty[s], 1);
    }
    for (int s = 0; s < kNvf4BStages; ++s) {
      mbar_init(&bars->bfull[s], kNvf4ProdWarps);
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
    tmem_alloc(&bars->tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t sbase = smem_u32(smem);
  const int stages_per_tile = p.Kh * g.cchunks;

  if (warp < kV2EpiWarps) {
    int it = 0;
    float amax = 0.f;
    const uint32_t wbuf = sbase + L::kEpiOffset + warp * 4096;
    for (int tile = blockIdx.x; tile < p.tiles; tile += gridDim.x, ++it) {
      const int acc = it & 1;
      mbar_wait_bounded(&bars->acc_full[acc], (it >> 1) & 1, p.err, kErrWaitDone);
      tc_fence_after();
      const bool last = tile + static_cast<int>(gridDim.x) >= p.tiles;
      halo_epilogue_tile<0, 0, false>(p, g, bars->tmem, acc * kNvf4BN, tile, warp & 3, wbuf, 0, last ? 3 : 1, amax);
      tc_fence_before();
      mbar_arrive(&bars->acc_empty[acc]);
    }
    epi_amax_flush(p.amax_out, amax);
  } else if (warp == kV2MmaWarp) {
    if (lane == 0) {
      const uint32_t idesc = idesc_nvf4(128, g.bn);
      const uint64_t adesc0 = smem_desc_sw128(sbase + L::kAOffset);
      const uint64_t bdesc0 = smem_desc_sw128(sbase + L::kBOffset);
      constexpr uint32_t kATileDesc = kNvf4ATile >> 4;
      constexpr uint32_t kBTileDesc = kNvf4BTile >> 4;
      const uint32_t tap_desc = static_cast<uint32_t>(p.N) * 8u;      // N rows of 128 B
      const uint32_t tap_sf = static_cast<uint32_t>(p.N) / 32u;       // N rows of scales
      int it = 0, sb = 0, sa = 0;
      uint32_t pb = 0, pa = 0;
      for (int tile = blockIdx.x; tile < p.tiles; tile += gridDim.x, ++it) {
        const int acc = it & 1;
        mbar_wait_bounded(&bars->acc_empty[acc], ((it >> 1) & 1) ^ 1, p.err, kErrWaitEmpty);
        tc_fence_after();
        const uint32_t dt = bars->tmem + acc * kNvf4BN;
        for (int st = 0; st < stages_per_tile; ++st) {
          mbar_wait_bounded(&bars->bfull[sb], pb, p.err, kErrWaitFull);
          tc_fence_after();
          const uint32_t sf = bars->tmem + kNvf4SfCol + static_cast<uint32_t>(sb) * kNvf4SfStage;
          const uint32_t bsf = sbase + L::kBSfOffset + static_cast<uint32_t>(sb) * kNvf4BSf;
          for (int ks = 0; ks < 4; ++ks)
            for (int a = 0; a < 2; ++a) tmem_cp_atom(sf + kNvf4SfB + 8 * ks + 4 * a, bsf + (2 * ks + a) * 512);
          const uint64_t bd = bdesc0 + static_cast<uint32_t>(sb) * kBTileDesc;
          for (int kw = 0; kw < p.Kw; ++kw) {
            mbar_wait_bounded(&bars->afull[sa], pa, p.err, kErrWaitFull);
            tc_fence_after();
            const uint32_t asf = sbase + L::kAOffset + static_cast<uint32_t>(sa) * kNvf4ATile + kATileBytes;
            for (int ks = 0; ks < 4; ++ks) tmem_cp_atom(sf + 4 * (4 * kw + ks), asf + ks * 512);
            const uint64_t a_k = adesc0 + static_cast<uint32_t>(sa) * kATileDesc;
            const uint64_t b_k = bd + static_cast<uint32_t>(kw) * tap_desc;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              mma_nvf4_ss(dt, a_k + 2 * ks, b_k + 2 * ks, idesc, sf + 4 * (4 * kw + ks),
                          sf + kNvf4SfB + 8 * ks + static_cast<uint32_t>(kw) * tap_sf, (st | kw | ks) ? 1u : 0u);
            mma_commit(&bars->aempty[sa]);
            if (++sa == kNvf4AStages) {
              sa = 0;
              pa ^= 1u;
            }
          }
          mma_commit(&bars->bempty[sb]);
          if (++sb == kNvf4BStages) {
            sb = 0;
            pb ^= 1u;
          }
        }
        mma_commit(&bars->acc_full[acc]);
        if (tile + static_cast<int>(gridDim.x) >= p.tiles) mma_commit(&bars->last_full);
      }
    }
  } else if (warp == kV2LoadWarp) {
    if (lane == 0) {
      int sa = 0;
      uint32_t pa = 1;
      for (int tile = blockIdx.x; tile < p.tiles; tile += gridDim.x) {
        const int mt = tile / (g.out_h * g.tpr);
        const uint8_t* img = p.image + static_cast<int64_t>(mt) * p.ktiles * kNvf4ATile;
        for (int kh = 0; kh < p.Kh; ++kh)
          for (int c = 0; c < g.cchunks; ++c)
            for (int kw = 0; kw < p.Kw; ++kw) {
              mbar_wait_bounded(&bars->aempty[sa], pa, p.err, kErrWaitEmpty);
              mbar_arrive_expect_tx(&bars->afull[sa], kNvf4ATile);
              const int kt = (kh * p.Kw + kw) * g.cchunks + c;
              bulk_copy_g2s(sbase + L::kAOffset + sa * kNvf4ATile, img + static_cast<int64_t>(kt) * kNvf4ATile,
                            kNvf4ATile, &bars->afull[sa]);
              if (++sa == kNvf4AStages) {
                sa = 0;
                pa ^= 1u;
              }
            }
      }
    }
  } else {
    // producers: padded codes and scale bytes of the halo, kHaloLookahead
    // stages of codes in flight per thread
    const int t = threadIdx.x - kV2ProdWarp0 * 32;
    const int ntile_cta = (p.tiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                          static_cast<int>(gridDim.x);
    const int total = ntile_cta * stages_per_tile;
    const int spatial = g.out_h * g.tpr;
    HaloCursor<kFwd, 0> cursor;
    HaloUnit ring[kHaloLookahead];
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
#pragma unroll
    for (int r = 0; r < kHaloLookahead; ++r)
      if (r < total) load_next(ring[r]);
    int sb = 0;
    uint32_t pb = 1;
    for (int kit = 0; kit < total;) {
#pragma unroll
      for (int r = 0; r < kHaloLookahead; ++r, ++kit) {
        if (kit >= total) break;
        mbar_wait_bounded(&bars->bempty[sb], pb, p.err, kErrWaitEmpty);
        if (t < g.rows)
          nvf4_store_unit(ring[r], sbase + L::kBOffset + sb * kNvf4BTile, sbase + L::kBSfOffset + sb * kNvf4BSf,
                          static_cast<uint32_t>(8 * (t >> 3)), static_cast<uint32_t>(t & 7));
        producer_warp_arrive(&bars->bfull[sb]);
        if (kit + kHaloLookahead < total) load_next(ring[r]);
        if (++sb == kNvf4BStages) {
          sb = 0;
          pb ^= 1u;
        }
      }
    }
    // the CTA's last tile: producer warp w takes chunks 1 or 2 (of every 3)
    // on TMEM lane quarter w % 4, staging through 4 KB of the B ring
    if (ntile_cta > 0) {
      const int lit = ntile_cta - 1;
      const int ltile_last = static_cast<int>(blockIdx.x) + lit * static_cast<int>(gridDim.x);
      const int pw = warp - kV2ProdWarp0;
      float amax = 0.f;
      mbar_wait_bounded(&bars->last_full, 0, p.err, kErrWaitDone);
      tc_fence_after();
      halo_epilogue_tile<0, 0, false>(p, g, bars->tmem, (lit & 1) * kNvf4BN, ltile_last, warp & 3, sbase + L::kBOffset + pw * 4096,
                         1 + pw / 4, 3, amax);
      epi_amax_flush(p.amax_out, amax);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kV2MmaWarp) {
    tc_fence_after();
    tmem_dealloc(bars->tmem, 512);
  }
}

}  // namespace mqv
