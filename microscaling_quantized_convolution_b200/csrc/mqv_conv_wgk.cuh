// Stride-1 weight gradient with the im2col operand shared by the taps of a
// kernel row (MicroQonv summary, onedev.kr/papers/182, sections
// "무엇과 다른가" (G_W = G_Y·X'^T) and "어떻게 동작하나" (channel/batch runs
// read once and reused on chip)).
//
// A CTA owns G_W[co tile of 128][kh][0..Kw)[ci tile of 128] with one TMEM
// accumulator per tap kw.  The contraction runs over the output rows ho and,
// along each row, over 64-element chunks of its (wo, n) elements.  For tap
// kw the X' elements of output chunk j are X elements (wo + kw - pad, n), the
// same X row shifted by kw·N elements; so the producers dequantize each
// X chunk (128 channels x 64 elements of the row hi = ho + kh - pad) and each
// G_Y chunk once, and the Kw taps are MMA groups whose 16-element K slices
// point at the right X chunk and slice (N % 16 == 0 keeps every slice whole).
//
// Stage t of a row segment [j0, j1) produces G_Y chunk t (t < j1) and X
// chunk t (t < j1 + SX, SX = the furthest X chunk a tap reaches) into ring
// slot t, and for t >= j0 + SX runs output chunk j = t - SX, which reads G_Y
// chunk j and X chunks j..j+SX; slot j is released after that.  Splits of
// the (ho, j) chunk range across CTAs make the partial sums that
// wgrad_reduce_kernel adds in split order.
#pragma once

#include <cstdint>

#include "mqv_conv_common.cuh"
#include "mqv_conv_kernels.cuh"
#include "mqv_ptx.cuh"

namespace mqv {

constexpr int kWgkSlots = 5;            // SX + 1 + producer lookahead, SX <= 2
constexpr int kWgkMaxTaps = 3;

struct WgkGeom {
  int chunks;         // 64-element chunks per output row, ceil(Wo·N / 64)
  int sx;             // X chunks beyond the output chunk a tap reaches
  int ctiles;         // 128-channel tiles of Cin
  int base_tiles;     // mtiles · ctiles · Kh
  int q_per_split;    // (ho, j) chunks per split
};

struct WgkSmem {
  static constexpr int kSlot = 2 * kATileBytes;              // G_Y chunk + X chunk
  static constexpr int kEpiOffset = kWgkSlots * kSlot;       // 32 x 32 fp32 per epilogue warp
  static constexpr int kEpiWarpBytes = 32 * 128;
  static constexpr int kBarOffset = kEpiOffset + kV2EpiWarps * kEpiWarpBytes;
  static constexpr int kBytes = kBarOffset + 256 + 1024;
};

struct WgkBars {
  uint64_t full[kWgkSlots];
  uint64_t empty[kWgkSlots];
  uint64_t done;        // all MMAs of a tile completed (tcgen05.commit)
  uint64_t acc_empty;   // the epilogue has read the accumulators of a tile
  uint32_t tmem;
};

// Tile decode: tile -> (mt, ct, kh, split).
struct WgkTile {
  int mt, ct, kh, sp;
};

__device__ __forceinline__ WgkTile wgk_tile(const V2Args& p, const WgkGeom& g, int tile) {
  WgkTile w;
  w.sp = tile % p.splits;
  int r = tile / p.splits;
  w.kh = r % p.Kh;
  r /= p.Kh;
  w.ct = r % g.ctiles;
  w.mt = r / g.ctiles;
  return w;
}

// Fill one stage: G_Y chunk (rows co, K = 64 (wo, n) elements of output row ho)
// and X chunk (rows ci, K = 64 (wi, n) elements of input row hi, starting
// at wi = -pad).  Unit = 4 rows x 8 batch items of one pixel (K-major,
// natural order: the codes run along n).
template <int FMT>
__device__ __forceinline__ void wgk_fill(const V2Args& p, uint32_t slot, const WgkTile& w, int ho, int t,
                                         bool with_a, int chunk) {
  constexpr int NU = 8;
  constexpr int KG = 64 / NU;
  constexpr int PER = 128 / 4 * KG / kV2ProdThreads;   // units per thread per operand
  const int hi = ho + w.kh - p.pad;
  UnitRaw<FMT, NU> raw[2][PER];
  // all loads of the stage first, then the dequantize + stores
#pragma unroll
  for (int op = 0; op < 2; ++op) {
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int u = t + kV2ProdThreads * i;
      const int kg = u % KG, rq = u / KG;
      const int e = chunk * 64 + kg * NU;           // element of the row: (pixel, n)
      const int pix = fdiv(e, p.dN);
      const int n = e - pix * p.N;
      if (op == 0) {                                 // G_Y[ho][wo = pix][co][n]
        const int co = w.mt * 128 + 4 * rq;
        const bool ok = with_a && co < p.Cout && pix < p.Wo;
        load_unit<FMT, NU>(p.a, (static_cast<int64_t>(ho) * p.Wo + pix) * p.Cout + co, n, ok, raw[0][i]);
      } else {                                       // X[hi][wi = pix - pad][ci][n]
        const int ci = w.ct * 128 + 4 * rq;
        const int wi = pix - p.pad;
        const bool ok = ci < p.Cin && hi >= 0 && hi < p.H && wi >= 0 && wi < p.W;
        load_unit<FMT, NU>(p.b, (static_cast<int64_t>(hi) * p.W + wi) * p.Cin + ci, n, ok, raw[1][i]);
      }
    }
  }
#pragma unroll
  for (int op = 0; op < 2; ++op) {
    if (op == 0 && !with_a) continue;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int u = t + kV2ProdThreads * i;
      const int kg = u % KG, rq = u / KG;
      store_unit<FMT, NU, false>(raw[op][i], slot + op * kATileBytes, static_cast<uint32_t>(4 * rq),
                                 static_cast<uint32_t>(kg * NU));
    }
  }
}

template <int FMT>
__global__ void __launch_bounds__(kV2Threads, 1)
conv_wgk_kernel(const V2Args p, const WgkGeom g) {
  using L = WgkSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  WgkBars* bars = reinterpret_cast<WgkBars*>(smem + L::kBarOffset);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kWgkSlots; ++s) {
      mbar_init(&bars->full[s], kV2ProdThreads / 32);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->done, 1);
    mbar_init(&bars->acc_empty, kV2EpiWarps * 32);
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
  const int total_q = p.Ho * g.chunks;

  // The same (tile, segment, stage) walk in every role: f(tile, w, ho, t, j0, j1)
  // per stage, t running over j0 .. j1 + sx - 1 of each row segment.
  auto walk = [&](auto&& f) {
    for (int tile = blockIdx.x; tile < p.tiles; tile += gridDim.x) {
      const WgkTile w = wgk_tile(p, g, tile);
      const int q0 = w.sp * g.q_per_split;
      const int q1 = min(total_q, q0 + g.q_per_split);
      for (int q = q0; q < q1;) {
        const int ho = q / g.chunks;
        const int j0 = q - ho * g.chunks;
        const int j1 = min(g.chunks, j0 + (q1 - q));
        for (int t = j0; t < j1 + g.sx; ++t) f(tile, w, ho, t, j0, j1);
        q += j1 - j0;
      }
    }
  };

  if (warp >= kV2ProdWarp0) {
    const int t_id = threadIdx.x - kV2ProdWarp0 * 32;
    int kit = 0;
    walk([&](int, const WgkTile& w, int ho, int t, int, int j1) {
      const int s = kit % kWgkSlots;
      mbar_wait_bounded(&bars->empty[s], ((kit / kWgkSlots) & 1) ^ 1, p.err, kErrWaitEmpty);
      wgk_fill<FMT>(p, sbase + s * L::kSlot, w, ho, t_id, t < j1, t);
      producer_warp_arrive(&bars->full[s]);
      ++kit;
    });
  } else if (warp == kV2MmaWarp) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(128, 128);
      int kit = 0, cur_tile = -1, tiles_seen = 0;
      bool started[kWgkMaxTaps] = {false, false, false};
      walk([&](int tile, const WgkTile&, int, int t, int j0, int j1) {
        if (tile != cur_tile) {
          if (cur_tile >= 0) mma_commit(&bars->done);   // previous tile finished: hand over
          if (tiles_seen > 0) {                         // its accumulators must be read first
            mbar_wait_bounded(&bars->acc_empty, (tiles_seen - 1) & 1, p.err, kErrWaitEmpty);
            tc_fence_after();
          }
          ++tiles_seen;
          cur_tile = tile;
          for (int kw = 0; kw < kWgkMaxTaps; ++kw) started[kw] = false;
        }
        const int s = kit % kWgkSlots;
        mbar_wait_bounded(&bars->full[s], (kit / kWgkSlots) & 1, p.err, kErrWaitFull);
        tc_fence_after();
        if (t >= j0 + g.sx) {
          // output chunk j = t - sx: G_Y chunk in slot (kit - sx), X chunks in slots kit - sx .. kit
          const int sj = (kit - g.sx) % kWgkSlots;
          const uint64_t adesc = smem_desc_sw128(sbase + sj * L::kSlot);
          for (int kw = 0; kw < p.Kw; ++kw) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const int o = 16 * kk + kw * p.N;     // element offset from X chunk j
              const int sx = (kit - g.sx + o / 64) % kWgkSlots;
              const uint64_t bdesc = smem_desc_sw128(sbase + sx * L::kSlot + kATileBytes) + 2 * ((o & 63) >> 4);
              mma_f16_ss(bars->tmem + kw * 128, adesc + 2 * kk, bdesc, idesc, started[kw] ? 1u : 0u);
              started[kw] = true;
            }
          }
          mma_commit(&bars->empty[sj]);
        }
        if (t == j1 + g.sx - 1) {
          // end of the segment (always an MMA stage): its last sx slots hold
          // X chunks no later output chunk of this row reads
          for (int k = kit - g.sx + 1; k <= kit; ++k) mma_commit(&bars->empty[k % kWgkSlots]);
        }
        ++kit;
      });
      if (cur_tile >= 0) mma_commit(&bars->done);
    }
  } else if (warp < kV2EpiWarps) {
    int it = 0;
    for (int tile = blockIdx.x; tile < p.tiles; tile += gridDim.x, ++it) {
      const WgkTile w = wgk_tile(p, g, tile);
      mbar_wait_bounded(&bars->done, it & 1, p.err, kErrWaitDone);
      tc_fence_after();
      const float scale = p.scale_out ? __fmul_rn(*p.ta, *p.tb) : 1.0f;
      // Each lane reads one accumulator row (output channel) from TMEM; a
      // swizzled 32 x 32 transpose in shared memory turns that into stores of
      // four whole 128-byte row pieces per warp instruction.
      const uint32_t wbuf = sbase + L::kEpiOffset + warp * L::kEpiWarpBytes;
      const int rsub = lane >> 3, q = lane & 7;
      for (int kw = 0; kw < p.Kw; ++kw) {
        const uint32_t tbase = bars->tmem + (static_cast<uint32_t>(warp * 32) << 16) + kw * 128;
        const int64_t col_base = (static_cast<int64_t>(w.kh) * p.Kw + kw) * p.Cin + w.ct * 128;
#pragma unroll 1
        for (int c = 0; c < 128; c += 32) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tbase + c, r);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            st_shared_v4(wbuf + lane * 128 + ((j ^ (lane & 7)) << 4),
                         __float_as_uint(__uint_as_float(r[4 * j + 0]) * scale),
                         __float_as_uint(__uint_as_float(r[4 * j + 1]) * scale),
                         __float_as_uint(__uint_as_float(r[4 * j + 2]) * scale),
                         __float_as_uint(__uint_as_float(r[4 * j + 3]) * scale));
          }
          __syncwarp();
          const int ci = w.ct * 128 + c + 4 * q;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int row = 4 * i + rsub;
            const float4 o = ld_shared_v4_f32(wbuf + row * 128 + ((q ^ (row & 7)) << 4));
            const int co = w.mt * 128 + warp * 32 + row;
            if (co < p.Cout && ci < p.Cin) {
              const int64_t idx = (static_cast<int64_t>(w.sp) * p.M + co) * p.Ncols + col_base + c + 4 * q;
              *reinterpret_cast<float4*>(p.out + idx) = o;
            }
          }
          __syncwarp();
        }
      }
      tc_fence_before();
      mbar_arrive(&bars->acc_empty);     // the next tile may overwrite the accumulators
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
