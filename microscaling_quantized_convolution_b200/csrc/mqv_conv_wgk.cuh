// Stride-1 weight gradient with the im2col operand shared by the taps of a
// kernel row (MicroQonv summary, onedev.kr/papers/182, sections
// "무엇과 다른가" (G_W = G_Y·X'^T) and "어떻게 동작하나" (channel/batch runs
// read once and reused on chip)).
//
// A CTA owns G_W[co tile of 128][kh][0..Kw)[ci tile of 128] with one TMEM
// accumulator per tap kw.  The contraction runs over the output rows ho and,
// along each row, over 64-element chunks of its (wo, n) elements.  For tap
// kw the X' elements of output chunk j are X elements (wo + kw - pad, n), the
// same X row shifted by kw·N elements; so each X chunk (128 channels x 64
// elements of the row hi = ho + kh - pad) is dequantized once into shared
// memory, and the Kw taps are MMA groups whose 16-element K slices point at
// the right X chunk and slice (N % 16 == 0 keeps every slice whole).
//
// The G_Y chunk (128 output channels x the 64 elements of output chunk j) is
// the MMA's A operand and lives in tensor memory: its producer threads own
// one channel row each, dequantize the row's 64 codes and write them with
// tcgen05.st.  Each MMA then reads only its B tile from shared memory, which
// halves the shared-memory traffic of the 128 x 128 MMAs.
//
// X stage t of a row segment [j0, j1) fills X chunk t for t in
// [j0, j1 + SX), SX = the furthest X chunk a tap reaches; output chunk
// j = t - SX runs at stage t >= j0 + SX and reads X chunks j..j+SX.  The X
// and G_Y rings advance independently.  Splits of the (ho, j) chunk range
// across CTAs make the partial sums that wgrad_reduce_kernel adds in a
// fixed order.
#pragma once

#include <cstdint>

#include "mqv_conv_common.cuh"
#include "mqv_conv_kernels.cuh"
#include "mqv_ptx.cuh"

namespace mqv {

constexpr int kWgkXSlots = 8;           // X chunks in shared memory (a power of two)
constexpr int kWgkXMirrors = 2;         // copies of slots 0 and 1 after the ring (paired taps)
constexpr int kWgkASlots = 4;           // G_Y chunks in tensor memory
constexpr int kWgkMaxTaps = 3;
constexpr int kWgkACol = kWgkMaxTaps * 128;     // first TMEM column of the G_Y ring
// Roles: warps 0-3 produce the even G_Y chunks, warps 8-11 the odd ones
// (each G_Y warp owns its TMEM lane quarter, warp % 4); warps 6, 7 and 12-17
// produce X; warp 4 issues the MMAs; warp 5 has no role.  All 16 producer
// warps then run the epilogue.
constexpr int kWgkWarps = 18;
constexpr int kWgkThreads = kWgkWarps * 32;
constexpr int kWgkXWarps = 8;
constexpr int kWgkGWarps = 8;

__device__ __forceinline__ int wgk_x_index(int warp) {   // X producer number of a warp, or -1
  return warp == 6 ? 0 : warp == 7 ? 1 : (warp >= 12 && warp < 18) ? warp - 10 : -1;
}

struct WgkGeom {
  int chunks;         // 64-element chunks per output row, ceil(Wo·N / 64)
  int sx;             // X chunks beyond the output chunk a tap reaches
  int ctiles;         // 128-channel tiles of Cin
  int base_tiles;     // mtiles · ctiles · Kh
  int q_per_split;    // (ho, j) chunks per split
};

struct WgkSmem {
  static constexpr int kXSlot = kATileBytes;                 // 128 channels x 64 fp16
  static constexpr int kEpiWarpBytes = 32 * 128;                  // epilogue transpose buffer per warp,
                                                                   // inside the X ring once it is idle
  static constexpr int kBarOffset = (kWgkXSlots + kWgkXMirrors) * kXSlot;
  static constexpr int kBytes = kBarOffset + 256 + 1024;
};

// One full and one done barrier per stage of the X ring: the 8 X warps and
// 4 G_Y warps (the chunk's owners, one per lane quarter) arrive on
// full[n % 8] for every stage n (the G_Y warps with the A chunk of an MMA
// stage; warps 0-3 alone, once stage n - 8 is done, otherwise), and the MMA
// thread commits
// done[n % 8] after every stage, so it waits once and commits once a stage.
// X stage n reuses its slot once stage n - 8 + SX (the last that reads the
// previous X chunk in it) is done; G_Y chunk a reuses A slot a % 4 once the
// stage four earlier is done (chunk a - 4 ran no later than that).
struct WgkBars {
  uint64_t full[kWgkXSlots];
  uint64_t done[kWgkXSlots];
  uint64_t tile_done;   // all MMAs of the tile completed (tcgen05.commit)
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

// Walk over the stages of this CTA's tile (one tile per CTA): each row
// segment [j0, j1) of the tile's chunk range yields stages t = j0 .. j1 +
// ext - 1 (ext = SX for the X ring and the MMA, 0 for the G_Y ring).
struct WgkCursor {
  int q, q1, ho, j0, j1, t;
  bool valid;

  __device__ __forceinline__ void begin(const V2Args& p, const WgkGeom& g, const WgkTile& w) {
    q = w.sp * g.q_per_split;
    q1 = min(p.Ho * g.chunks, q + g.q_per_split);
    valid = q < q1;
    ho = q / g.chunks;
    j0 = q - ho * g.chunks;
    j1 = min(g.chunks, j0 + (q1 - q));
    t = j0;
  }
  // after the first segment every segment starts a new output row
  __device__ __forceinline__ void advance(const WgkGeom& g, int ext) {
    if (++t < j1 + ext) return;
    q += j1 - j0;
    valid = q < q1;
    ++ho;
    j0 = 0;
    j1 = min(g.chunks, q1 - q);
    t = 0;
  }
  __device__ __forceinline__ bool mma_stage(const WgkGeom& g) const { return t >= j0 + g.sx; }
};

// X producer: one unit (4 channels x 8 consecutive (pixel, n) elements) per
// thread per stage; 256 units fill a 128-channel x 64-element chunk.
// LINE: both operands carry 1 x 16 line blocks along their batch columns, so
// every row of a unit or piece has one scale for its 8 or 16 elements.
template <int FMT, bool LINE>
__device__ __forceinline__ void wgk_x_load(const V2Args& p, const WgkTile& w, const WgkCursor& c, int tid,
                                           UnitRaw<FMT, 8>& r) {
  const int hi = c.ho + w.kh - p.pad;
  const int kg = tid & 7, rq = tid >> 3;
  const int e = c.t * 64 + kg * 8;              // element (pixel, n) of the padded X row
  const int pix = fdiv(e, p.dN);
  const int n = e - pix * p.N;
  const int ci = w.ct * 128 + 4 * rq;
  const int wi = pix - p.pad;
  const bool ok = ci < p.Cin && hi >= 0 && hi < p.H && wi >= 0 && wi < p.W;
  const int64_t row = (static_cast<int64_t>(hi) * p.W + wi) * p.Cin + ci;
  if (!LINE) {
    load_unit<FMT, 8>(p.b, row, n, ok, r);
    return;
  }
  r.ok = ok;
  if (!ok) return;
  r.ss = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    r.lo[j] = load_codes<FMT, 8>(p.b, row + j, n, r.hi[j]);
    r.ss |= static_cast<uint32_t>(__ldg(p.b.scales + (row + j) * p.b.scale_cols + (n >> 4))) << (8 * j);
  }
}

// Dequantize the unit into registers (wgk_x_dequant), then store it into X
// slot `slot` and, when `mirror` is nonzero, into that second slot as well
// (wgk_x_st).
template <int FMT, bool LINE>
__device__ __forceinline__ void wgk_x_dequant(const UnitRaw<FMT, 8>& un, uint32_t (&h)[4][4]) {
  const uint32_t s2lo = un.ok && !LINE ? scale2(un.ss & 0xFF) : 0u;
  const uint32_t s2hi = un.ok && !LINE ? scale2(un.ss >> 8) : 0u;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    h[j][0] = h[j][1] = h[j][2] = h[j][3] = 0u;
    if (un.ok) {
      const uint32_t sj = LINE ? scale2((un.ss >> (8 * j)) & 0xFF) : 0u;
      dequant_run<FMT, 8>(un.lo[j], un.hi[j], LINE ? sj : s2lo, LINE ? sj : s2hi, h[j]);
    }
  }
}

__device__ __forceinline__ void wgk_x_st(const uint32_t (&h)[4][4], uint32_t slot, uint32_t mirror, int tid) {
  const uint32_t row0 = static_cast<uint32_t>(4 * (tid >> 3)), kl = static_cast<uint32_t>(8 * (tid & 7));
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t off = sw128_offset(row0 + j, kl);
    st_shared_v4(slot + off, h[j][0], h[j][1], h[j][2], h[j][3]);
    if (mirror) st_shared_v4(mirror + off, h[j][0], h[j][1], h[j][2], h[j][3]);
  }
}

// G_Y producer: the 64 codes of one output-channel row of an output chunk,
// as four 16-element pieces, each inside one pixel since N % 16 == 0.
struct WgkGRow {
  uint32_t c[4][3];     // FP4: 8 bytes in c[.][0..1]; FP6: 12 bytes
  uint32_t s[4];        // the four E4M3 block scales of a piece
  uint32_t ok;          // bit per piece
};

template <int FMT, bool LINE>
__device__ __forceinline__ void wgk_g_load_row(const V2Args& p, const WgkTile& w, const WgkCursor& c, int row,
                                               WgkGRow& r) {
  const int co = w.mt * 128 + row;
  r.ok = 0;
#pragma unroll
  for (int pc = 0; pc < 4; ++pc) {
    const int e = c.t * 64 + 16 * pc;
    const int pix = fdiv(e, p.dN);
    const int n = e - pix * p.N;
    if (co < p.Cout && pix < p.Wo) {
      r.ok |= 1u << pc;
      const int64_t vrow = (static_cast<int64_t>(c.ho) * p.Wo + pix) * p.Cout + co;
      const uint8_t* cp = p.a.codes + vrow * p.a.row_bytes;
      if (FMT == 0) {
        const uint2 v = __ldg(reinterpret_cast<const uint2*>(cp + (n >> 1)));
        r.c[pc][0] = v.x;
        r.c[pc][1] = v.y;
      } else {
        const uint32_t* q = reinterpret_cast<const uint32_t*>(cp + ((n * 3) >> 2));
        r.c[pc][0] = __ldg(q);
        r.c[pc][1] = __ldg(q + 1);
        r.c[pc][2] = __ldg(q + 2);
      }
      if (LINE) r.s[pc] = static_cast<uint32_t>(__ldg(p.a.scales + vrow * p.a.scale_cols + (n >> 4))) * 0x01010101u;
      else r.s[pc] = __ldg(reinterpret_cast<const uint32_t*>(p.a.scales + (vrow >> 2) * p.a.scale_cols + (n >> 2)));
    }
  }
}

template <int FMT>
__device__ __forceinline__ void wgk_g_dequant_row(const WgkGRow& r, uint32_t (&h)[32]) {
#pragma unroll
  for (int pc = 0; pc < 4; ++pc) {
    uint32_t* o = h + 8 * pc;
    if (!((r.ok >> pc) & 1u)) {
#pragma unroll
      for (int j = 0; j < 8; ++j) o[j] = 0u;
      continue;
    }
    const uint32_t s = r.s[pc];
    const uint32_t s0 = scale2(s & 0xFF), s1 = scale2((s >> 8) & 0xFF);
    const uint32_t s2 = scale2((s >> 16) & 0xFF), s3 = scale2(s >> 24);
    if (FMT == 0) {
      uint32_t a[4], b[4];
      dq8_fp4(r.c[pc][0], s0, s1, a);
      dq8_fp4(r.c[pc][1], s2, s3, b);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        o[j] = a[j];
        o[4 + j] = b[j];
      }
    } else {
      const uint32_t c0 = r.c[pc][0], c1 = r.c[pc][1], c2 = r.c[pc][2];
      dq4_fp6(c0 & 0xFFFFFF, s0, o[0], o[1]);
      dq4_fp6((c0 >> 24) | ((c1 & 0xFFFF) << 8), s1, o[2], o[3]);
      dq4_fp6((c1 >> 16) | ((c2 & 0xFF) << 16), s2, o[4], o[5]);
      dq4_fp6(c2 >> 8, s3, o[6], o[7]);
    }
  }
}

// Epilogue of the tile, run by all 16 producer warps once the last MMA has
// completed: four warps per TMEM lane quarter (warp % 4), each taking every
// fourth 32-column block of the Kw·128 accumulator columns.  Rows are read
// with tcgen05.ld, transposed through a swizzled 32 x 32 buffer in shared
// memory (the X ring is free by then), and stored as whole 128-byte row
// pieces.
__device__ __forceinline__ void wgk_epilogue(const V2Args& e, const WgkTile& w, WgkBars* bars, uint32_t tmem,
                                             uint32_t wbuf, int quarter, int cpart, int lane) {
  mbar_wait_bounded(&bars->tile_done, 0, e.err, kErrWaitDone);
  tc_fence_after();
  const float scale = e.scale_out ? __fmul_rn(*e.ta, *e.tb) : 1.0f;
  const int rsub = lane >> 3, q = lane & 7;
  const uint32_t tlane = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
#pragma unroll 1
  for (int blk = cpart; blk < 4 * e.Kw; blk += 4) {
    const int kw = blk >> 2, c = (blk & 3) * 32;
    const int64_t col_base = (static_cast<int64_t>(w.kh) * e.Kw + kw) * e.Cin + w.ct * 128;
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {     // 16 columns at a time keeps the register count low
      uint32_t r[16];
      tmem_ld_32x32b_x16(tlane + kw * 128 + c + 16 * hf, r);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        st_shared_v4(wbuf + lane * 128 + (((4 * hf + j) ^ (lane & 7)) << 4),
                     __float_as_uint(__uint_as_float(r[4 * j + 0]) * scale),
                     __float_as_uint(__uint_as_float(r[4 * j + 1]) * scale),
                     __float_as_uint(__uint_as_float(r[4 * j + 2]) * scale),
                     __float_as_uint(__uint_as_float(r[4 * j + 3]) * scale));
      }
    }
    __syncwarp();
    const int ci = w.ct * 128 + c + 4 * q;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int row = 4 * i + rsub;
      const float4 o = ld_shared_v4_f32(wbuf + row * 128 + ((q ^ (row & 7)) << 4));
      const int co = w.mt * 128 + quarter * 32 + row;
      if (co < e.Cout && ci < e.Cin) {
        const int64_t idx = (static_cast<int64_t>(w.sp) * e.M + co) * e.Ncols + col_base + c + 4 * q;
        *reinterpret_cast<float4*>(e.out + idx) = o;
      }
    }
    __syncwarp();
  }
}

template <int FMT, int KW, bool PAIR, bool LINE = false>
__global__ void __launch_bounds__(kWgkThreads, 1)
conv_wgk_kernel(const V2Args p, const WgkGeom g) {
  using L = WgkSmem;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  WgkBars* bars = reinterpret_cast<WgkBars*>(smem + L::kBarOffset);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kWgkXSlots; ++s) {
      mbar_init(&bars->full[s], kWgkXWarps + kWgkGWarps / 2);   // X warps and one G_Y warp per lane quarter
      mbar_init(&bars->done[s], 1);
    }
    mbar_init(&bars->tile_done, 1);
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
  const uint32_t tmem = bars->tmem;

  const WgkTile w = wgk_tile(p, g, blockIdx.x);
  const int xi = wgk_x_index(warp);
  // wait until stage m's MMAs have completed
  auto wait_done = [&](int m) {
    mbar_wait_bounded(&bars->done[m % kWgkXSlots], (m / kWgkXSlots) & 1, p.err, kErrWaitEmpty);
  };
  if (xi >= 0) {
    // X producer: the next stage's unit is dequantized into registers
    // before the slot is free, so the wait is followed only by stores; the
    // unit after that is loaded one stage ahead.
    const int tid = xi * 32 + lane;
    WgkCursor cur, ld;
    cur.begin(p, g, w);
    ld = cur;
    UnitRaw<FMT, 8> raw;
    uint32_t hx[4][4];
    auto load_next = [&]() {
      if (ld.valid) {
        wgk_x_load<FMT, LINE>(p, w, ld, tid, raw);
        ld.advance(g, g.sx);
      }
    };
    load_next();
    if (cur.valid) {
      wgk_x_dequant<FMT, LINE>(raw, hx);
      load_next();
    }
    int n = 0;
    while (cur.valid) {
      const int s = n % kWgkXSlots;
      if (n >= kWgkXSlots) wait_done(n - kWgkXSlots + g.sx);
      const uint32_t mirror = (PAIR && s < kWgkXMirrors) ? sbase + (kWgkXSlots + s) * L::kXSlot : 0u;
      wgk_x_st(hx, sbase + s * L::kXSlot, mirror, tid);
      producer_warp_arrive(&bars->full[s]);
      cur.advance(g, g.sx);
      ++n;
      if (cur.valid) {
        wgk_x_dequant<FMT, LINE>(raw, hx);
        load_next();
      }
    }
  } else if (warp < 4 || (warp >= 8 && warp < 12)) {
    // G_Y producer: thread = output-channel row (this warp's TMEM lane
    // quarter).  Warps 0-3 take the even G_Y chunks, warps 8-11 the odd
    // ones, a whole 64-element row each, so each warp has two stages' time
    // for its loads and its dequantization; the next owned chunk is
    // dequantized while the MMAs run, and the one after it is loaded.
    // Stages with no G_Y chunk are signalled by warps 0-3.  All producer
    // warps run the epilogue afterwards.
    const int quarter = warp & 3, par = warp < 4 ? 0 : 1;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    WgkCursor cur, ld;
    cur.begin(p, g, w);
    ld = cur;
    if (par == 1 && ld.valid) ld.advance(g, 0);
    WgkGRow raw;
    uint32_t h[32];
    auto load_owned = [&]() {          // the chunk at ld, then ld moves two chunks on
      raw.ok = 0;
      if (ld.valid) {
        wgk_g_load_row<FMT, LINE>(p, w, ld, row, raw);
        ld.advance(g, 0);
        if (ld.valid) ld.advance(g, 0);
      }
    };
    load_owned();
    wgk_g_dequant_row<FMT>(raw, h);
    load_owned();
    int n = 0, a = 0;
    while (cur.valid) {
      if (!cur.mma_stage(g)) {           // a stage with no G_Y chunk
        if (par == 0) {
          if (n >= kWgkXSlots) wait_done(n - kWgkXSlots);
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->full[n % kWgkXSlots]);
        }
        cur.advance(g, g.sx);
        ++n;
        continue;
      }
      if ((a & 1) == par) {
        if (n >= kWgkASlots) wait_done(n - kWgkASlots);
        tc_fence_after();
        tmem_st_32x32b_x32(tmem + lane_base + kWgkACol + (a % kWgkASlots) * 32, h);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->full[n % kWgkXSlots]);
        wgk_g_dequant_row<FMT>(raw, h);
        load_owned();
      }
      cur.advance(g, g.sx);
      ++n;
      ++a;
    }
  } else if (warp == kV2MmaWarp) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(128, 128);
      // The B operand of tap kw, K slice kk is X chunk j + o / 64, slice
      // (o % 64) / 16, o = 16·kk + kw·N: a fixed slot delta and descriptor
      // offset per (kw, kk), so each MMA costs a few integer operations.
      uint32_t bdelta[KW][4], boff[KW][4];
#pragma unroll
      for (int kw = 0; kw < KW; ++kw)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint32_t o = 16u * kk + static_cast<uint32_t>(kw * p.N);
          bdelta[kw][kk] = o >> 6;
          boff[kw][kk] = 2u * ((o & 63u) >> 4);
        }
      const uint64_t desc0 = smem_desc_sw128(sbase);
      constexpr uint32_t kSlotDesc = L::kXSlot >> 4;
      int n = 0, a = 0;
      WgkCursor c;
      for (c.begin(p, g, w); c.valid; c.advance(g, g.sx), ++n) {
        const int s = n % kWgkXSlots;
        mbar_wait_bounded(&bars->full[s], (n / kWgkXSlots) & 1, p.err, kErrWaitFull);
        tc_fence_after();
        if (c.mma_stage(g)) {
          // output chunk j = t - sx: G_Y chunk in A slot a % 4, X chunks in X slots n - sx .. n
          const uint32_t a_t = tmem + kWgkACol + (a % kWgkASlots) * 32;
          const uint32_t xbase = static_cast<uint32_t>(n - g.sx);
          const uint32_t first = a == 0 ? 0u : 1u;
          if (PAIR) {
            // N = 64: tap kw reads X chunk j + kw whole, and chunks j..j+KW-1
            // sit in consecutive slots (slots 0 and 1 are mirrored after the
            // ring), so the taps' B operands are one run of KW·128 rows:
            // two N = 192 MMAs for three taps, one N = 256 MMA for two.
            const uint64_t b = desc0 + (xbase & (kWgkXSlots - 1)) * kSlotDesc;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint32_t acc = kk > 0 ? 1u : first;
              if (KW == 3) {
                mma_f16_ts(tmem, a_t + 8 * kk, b + 2 * kk, idesc_f16_f32(128, 192), acc);
                mma_f16_ts(tmem + 192, a_t + 8 * kk, b + (192 * 128 >> 4) + 2 * kk, idesc_f16_f32(128, 192), acc);
              } else {
                mma_f16_ts(tmem, a_t + 8 * kk, b + 2 * kk, idesc_f16_f32(128, 256), acc);
              }
            }
          } else {
#pragma unroll
            for (int kw = 0; kw < KW; ++kw)
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint32_t slot = (xbase + bdelta[kw][kk]) & (kWgkXSlots - 1);
                const uint64_t bdesc = desc0 + (slot * kSlotDesc + boff[kw][kk]);
                mma_f16_ts(tmem + kw * 128, a_t + 8 * kk, bdesc, idesc, kk > 0 ? 1u : first);
              }
          }
          ++a;
        }
        mma_commit(&bars->done[s]);
      }
      mma_commit(&bars->tile_done);
    }
  }
  if (xi >= 0 || warp < 4 || (warp >= 8 && warp < 12)) {
    // column part: G_Y warps 0-3 -> 0, 8-11 -> 1; X warps 6, 7, 12, 13 -> 2; 14-17 -> 3
    const int cpart = warp < 4 ? 0 : warp < 12 && warp >= 8 ? 1 : (warp < 14 ? 2 : 3);
    wgk_epilogue(p, w, bars, tmem, sbase + warp * L::kEpiWarpBytes, warp & 3, cpart, lane);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kV2MmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace mqv
