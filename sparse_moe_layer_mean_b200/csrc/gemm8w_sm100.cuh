// gemm8w_sm100.cuh — the e4m3 block-scaled GEMM with 256 weight columns per
// unit: the FP8 layer's expert GEMMs and projections, and the expert GEMMs of
// the FP4 variant (weights as e2m1 codes, read by the tensor core; see
// Glu4WPolicy).
//
// The arithmetic is gemm8_sm100.cuh's: tokens on M (TMEM lanes), weights on
// N, each 128-deep K block accumulated alone in a TMEM partial and folded by
// eight promotion warps into fp32 registers with one scalar per thread per K
// block (token scale x weight-block scale).  What changes is the width: a
// unit is 128 tokens x 256 weight columns, so one kind::f8f6f4 MMA (M = 128,
// N = 256, K = 32) runs above the instruction's fixed cost instead of at it,
// and each token tile staged in shared memory serves twice the weight
// columns.  A promotion thread then holds 128 accumulators: the producer
// warpgroup gives up registers (setmaxnreg.dec to 56) so that the two
// promotion warpgroups can take 224 each (setmaxnreg.inc); the kernel is
// launched with 384 threads x 168 registers = 64 512, and
// 128 x 56 + 256 x 224 = 64 512.
//
//   warp 0: TMA producer, tokens     warp 2: TMA producer, weights
//   warp 1: TMEM allocator + MMA     warp 3: scale stager
//   warps 4-11: promotion + epilogue; warp w: TMEM lanes 32*(w%4) .. +31
//               (its 32 tokens), columns 128*((w-4)/4) .. +127
//
// Three shared-memory stages (16 KB tokens + 32 KB weights) and two TMEM
// partials of 256 columns are decoupled: the commit after K block g's MMAs
// arrives on empty[g % 3] (the producers reuse the stage) and on done[g % 2]
// (the promotion warps read the partial); the promotion warps' free[g % 2]
// lets the MMA reuse a partial.  All waits are bounded.  No TMA load uses
// multicast.
#pragma once
#include "gemm8_sm100.cuh"
#include "routing.cuh"  // e4m3x2: the activation quantiser's conversion

namespace mrl {

constexpr int kW8Ring = 3;                       // shared-memory stages
constexpr int kW8Parts = 2;                      // TMEM partial buffers
constexpr int kW8N = 256;                        // weight columns per unit
constexpr int kW8Cols = 128;                     // columns per promotion thread
constexpr int kW8BBytes = kW8N * 128;            // weight tile per K block
constexpr int kW8LaunchRegs = 168;               // registers per thread at launch (384 threads)
constexpr int kW8ProducerRegs = 56;              // warpgroup 0 after setmaxnreg.dec
constexpr int kW8PromoRegs = 224;                // warpgroups 1-2 after setmaxnreg.inc
static_assert(128 * kW8ProducerRegs + 256 * kW8PromoRegs == kF8Threads * kW8LaunchRegs,
              "the register split must add up to the launch's registers");

template <class P>
struct Gemm8WSmem {
  static constexpr int kStageBytes = kF8OpBytes + kW8BBytes;
  static constexpr int kRing = kW8Ring * kStageBytes;
  static constexpr int kTabOff = kRing;
  static constexpr int kBarOff = kTabOff + 2 * kF8TabFloats * 4;
  static constexpr int kNumBars = 2 * kW8Ring + 2 * kW8Parts + 4;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kEpiOff = (kMiscOff + 16 + 127) & ~127;
  static constexpr int kAuxOff = (kEpiOff + P::kEpiSmem + 127) & ~127;
  static constexpr int kTotal = kAuxOff + P::kAuxSmem + 1024;
};

template <int N>
__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

// Shared rows of 64 bytes staged for coalesced stores: 16-byte chunk c of row
// r sits at chunk index c ^ ((r >> 1) & 3), so the 128-bit writes of a
// quarter-warp (eight rows) and its reads (two rows' four chunks) both fall
// on distinct bank groups.
__device__ __forceinline__ int row64_chunk(int r, int c) { return r * 4 + (c ^ ((r >> 1) & 3)); }

// acc[OFF + i] += r[i] * s for the 32 values of one TMEM load, as packed
// fp32x2 FMAs (round to nearest per lane: the same values as fmaf).
template <int OFF>
__device__ __forceinline__ void fold32(float (&acc)[kW8Cols], const uint32_t (&r)[32], float2 s) {
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    const float2 v = __ffma2_rn(make_float2(__uint_as_float(r[i]), __uint_as_float(r[i + 1])), s,
                                make_float2(acc[OFF + i], acc[OFF + i + 1]));
    acc[OFF + i] = v.x;
    acc[OFF + i + 1] = v.y;
  }
}

template <class P>
__global__ void __launch_bounds__(kF8Threads, 1) gemm8w_kernel(const __grid_constant__ typename P::Params p) {
  using L = Gemm8WSmem<P>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kBarOff);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMiscOff);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMiscOff + 4);
  volatile int *hold_flag = reinterpret_cast<volatile int *>(smem + L::kMiscOff + 8);
  float *tabs = reinterpret_cast<float *>(smem + L::kTabOff);
  uint8_t *epi_smem = smem + L::kEpiOff;
  uint8_t *aux = smem + L::kAuxOff;

  const uint32_t full0 = smem_u32(bars);             // stage s loaded
  const uint32_t empty0 = full0 + 8 * kW8Ring;       // stage s read by its MMAs
  const uint32_t done0 = empty0 + 8 * kW8Ring;       // partial b written by its MMAs
  const uint32_t free0 = done0 + 8 * kW8Parts;       // partial b read by the promotion warps
  const uint32_t sfull0 = free0 + 8 * kW8Parts;      // scale table b written
  const uint32_t sempty0 = sfull0 + 16;              // scale table b read
  const uint32_t ring = smem_u32(smem);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  uint32_t *status = p.status;

  if (threadIdx.x == 0) {
    const uint2 hdr = call_header(status);
    for (int s = 0; s < kW8Ring; ++s) {
      mbar_init(full0 + 8 * s, 2);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < kW8Parts; ++b) {
      mbar_init(done0 + 8 * b, 1);
      mbar_init(free0 + 8 * b, 8);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(sfull0 + 8 * b, 32);
      mbar_init(sempty0 + 8 * b, 8);
    }
    *abort_flag = hdr.x != DEV_OK;  // an earlier kernel of the call failed: do nothing
    *hold_flag = (hdr.y & HOLD_GEMM_FP8) != 0;
    fence_mbar_init();
  }
  P::stage_aux(p, aux);
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int nunits = P::num_units(p, aux);
  const int kblocks = P::k_blocks(p);
  int issued = -1;  // MMA issuer: last committed K block
  const uint32_t idesc = idesc_f8f6f4(kF8Tile, kW8N, kFmtE4M3, P::kWeightFormat);
  if (*abort_flag) goto done;

  if (warp < 4) {
    // warpgroup 0 (producers, MMA issuer, stager) lends registers to the promotion warpgroups
    setmaxnreg_dec<kW8ProducerRegs>();
    if (warp == 0 || warp == 2) {
      // with the call's loads held (test mask) nothing is issued, so the
      // consumers' bounded waits run out and record DEV_TIMEOUT
      if (lane == 0 && !*hold_flag) {
        const bool isA = warp == 0;
        P::prefetch(p);
        uint32_t g = 0;
        Unit U{};
        if (static_cast<int>(blockIdx.x) < nunits) U = P::unit(p, blockIdx.x, aux);
        for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
          Unit Un = U;
          for (int kb = 0; kb < kblocks; ++kb, ++g) {
            const uint32_t s = g % kW8Ring;
            if (g >= kW8Ring && !mbar_wait(empty0 + 8 * s, ((g / kW8Ring) - 1) & 1, abort_flag, status)) goto done;
            mbar_arrive_expect_tx(full0 + 8 * s, isA ? P::a_bytes(U) : P::kWeightTxBytes);
            const uint32_t st = ring + s * L::kStageBytes;
            if (isA)
              P::load_a(p, U, kb, st, full0 + 8 * s);
            else
              P::load_b(p, U, kb, st + kF8OpBytes, full0 + 8 * s);
            // the next unit's descriptor, while this unit's loads are in flight
            if (kb == 0 && u + static_cast<int>(gridDim.x) < nunits) Un = P::unit(p, u + gridDim.x, aux);
          }
          U = Un;
        }
      }
    } else if (warp == 1) {
      if (lane == 0) {
        uint32_t g = 0;
        for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
          for (int kb = 0; kb < kblocks; ++kb, ++g) {
            const uint32_t s = g % kW8Ring, b = g % kW8Parts;
            if (!mbar_wait(full0 + 8 * s, (g / kW8Ring) & 1, abort_flag, status)) goto done;
            if (g >= kW8Parts && !mbar_wait(free0 + 8 * b, ((g / kW8Parts) - 1) & 1, abort_flag, status)) goto done;
            tc_fence_after();
            const uint32_t a_s = ring + s * L::kStageBytes;
            const uint32_t b_s = a_s + kF8OpBytes;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_f8(tmem_base + b * kW8N, sdesc_sw128(a_s + kk * 32), sdesc_sw128(b_s + kk * 32), idesc, kk != 0);
            umma_commit(empty0 + 8 * s);
            umma_commit(done0 + 8 * b);
            issued = static_cast<int>(g);
          }
        }
      }
    } else if (warp == 3) {
      int ul = 0;
      for (int u = blockIdx.x; u < nunits; u += gridDim.x, ++ul) {
        const Unit U = P::unit(p, u, aux);
        const int b = ul & 1;
        if (ul >= 2 && !__all_sync(0xffffffffu, mbar_wait(sempty0 + 8 * b, ((ul >> 1) - 1) & 1, abort_flag, status)))
          goto done;
        float *tok = tabs + b * kF8TabFloats;
        P::stage_scales(p, U, tok, tok + kF8MaxKB * kF8Tile, tok + kF8TabExtra, lane);
        if (lane == 0) {
          int *d = reinterpret_cast<int *>(tok + kF8TabUnit);
          d[0] = U.g; d[1] = U.m; d[2] = U.n0; d[3] = U.nv; d[4] = U.row0;
        }
        mbar_arrive(sfull0 + 8 * b);
      }
    }
  } else {
    setmaxnreg_inc<kW8PromoRegs>();
    const int pw = warp - kF8PromoWarp0;        // 0..7
    const int q = warp & 3;                     // TMEM lane quarter: tokens 32q..32q+31
    const int h = pw >> 2;                      // column half: 128h .. 128h+127
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    uint32_t g = 0;
    int ul = 0;
    for (int u = blockIdx.x; u < nunits; u += gridDim.x, ++ul) {
      const int tb = ul & 1;
      const float *tok = tabs + tb * kF8TabFloats + q * 32 + lane;
      // weight scales of the thread's columns 0-63 and 64-127 (one weight
      // block for both, or gate then up: P::kGateUp)
      const float *wlo = tabs + tb * kF8TabFloats + kF8MaxKB * kF8Tile + (P::kGateUp ? 0 : h) * kF8MaxKB;
      const float *whi = tabs + tb * kF8TabFloats + kF8MaxKB * kF8Tile + (P::kGateUp ? 1 : h) * kF8MaxKB;
      bool bad = !__all_sync(0xffffffffu, mbar_wait(sfull0 + 8 * tb, (ul >> 1) & 1, abort_flag, status));
      Unit U;
      {
        const int *d = reinterpret_cast<const int *>(tabs + tb * kF8TabFloats + kF8TabUnit);
        U.g = d[0]; U.m = d[1]; U.n0 = d[2]; U.nv = d[3]; U.row0 = d[4]; U.nsub = 1;
      }
      // no token of the unit in this warp's 32 rows: its partials need no
      // promotion, and the epilogue stores nothing for it
      const bool idle = q * 32 >= U.nv;
      float acc[kW8Cols];
#pragma unroll
      for (int i = 0; i < kW8Cols; ++i) acc[i] = 0.f;
      for (int kb = 0; kb < kblocks; ++kb, ++g) {
        const uint32_t b = g % kW8Parts;
        if (!bad) bad = !__all_sync(0xffffffffu, mbar_wait(done0 + 8 * b, (g / kW8Parts) & 1, abort_flag, status));
        if (bad) continue;
        if (idle) {
          __syncwarp();
          if (lane == 0) mbar_arrive(free0 + 8 * b);
          continue;
        }
        const float ts = tok[kb * kF8Tile];
        const float2 slo = make_float2(ts * wlo[kb], ts * wlo[kb]);
        const float2 shi = make_float2(ts * whi[kb], ts * whi[kb]);
        const uint32_t taddr = tmem_base + b * kW8N + lane_off + h * kW8Cols;
        tc_fence_after();
        // four 32-column loads, each in flight while the previous one is
        // folded (two load buffers and the 128 accumulators fit the
        // warpgroup's registers)
        uint32_t ra[32], rb[32];
        tmem_ld32_nowait(taddr, ra);
        tmem_wait_ld32(ra);
        tmem_ld32_nowait(taddr + 32, rb);
        fold32<0>(acc, ra, slo);
        tmem_wait_ld32(rb);
        tmem_ld32_nowait(taddr + 64, ra);
        fold32<32>(acc, rb, slo);
        tmem_wait_ld32(ra);
        tmem_ld32_nowait(taddr + 96, rb);
        fold32<64>(acc, ra, shi);
        tmem_wait_ld32(rb);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(free0 + 8 * b);  // the partial is in registers
        fold32<96>(acc, rb, shi);
      }
      if (bar_red_or(1, kF8PromoThreads, bad || *abort_flag)) goto done;
      P::epilogue_regs(p, U, acc, q, h, lane, epi_smem, tabs + tb * kF8TabFloats + kF8TabExtra);
      __syncwarp();
      if (lane == 0) mbar_arrive(sempty0 + 8 * tb);  // table tb (read by the epilogue too) is free
    }
  }
done:
  if (warp == 1 && lane == 0 && *abort_flag && issued >= 0) {
    // let the MMAs already issued land before the accumulator is freed
    const uint32_t b = static_cast<uint32_t>(issued) % kW8Parts;
    mbar_drain(done0 + 8 * b, (static_cast<uint32_t>(issued) / kW8Parts) & 1);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ------------------------------------------------------- wide policies
// Weight tiles are two 128-row boxes (maps with 128-row boxes).  The weight
// scale of column half h is one fp32 per K block (class h).

// Projection out = bf16(a w^T): unit = (128-token tile m, 256-column tile n0).
struct Dense8WPolicy : Dense8Policy {
  static constexpr uint32_t kWeightFormat = kFmtE4M3;
  static constexpr uint32_t kWeightTxBytes = kW8BBytes;  // bytes the weight loads of a K block complete
  static constexpr bool kGateUp = false;  // the thread's 128 columns share one weight block
  static __device__ __forceinline__ int num_units(const Params &p, const uint8_t *) { return p.m_tiles * p.n_tiles; }
  static __device__ __forceinline__ Unit unit(const Params &p, int u, const uint8_t *) {
    Unit U;
    U.g = 0;
    U.m = u / p.n_tiles;
    U.n0 = (u % p.n_tiles) * kW8N;
    U.row0 = U.m * kF8Tile;
    U.nv = min(kF8Tile, p.M - U.row0);
    U.nsub = 1;
    return U;
  }
  static __device__ __forceinline__ void load_b(const Params &p, const Unit &U, int kb, uint32_t sb, uint32_t bar) {
    tma_load_2d(sb, &p.tb, bar, kb * 128, U.n0);
    tma_load_2d(sb + kF8OpBytes, &p.tb, bar, kb * 128, U.n0 + kF8Tile);  // past N: zero fill, not stored
  }
  static __device__ __forceinline__ void stage_scales(const Params &p, const Unit &U, float *tok, float *w, float *,
                                                      int lane) {
    const int kbs = p.K / 128;
    stage_token_scales(p.as_t, p.M, U.row0, U.nv, kbs, tok, lane);
    const float *ws0 = p.ws + static_cast<size_t>(U.n0 / 128) * kbs;
    stage_weight_scales(ws0, U.n0 + kF8Tile < p.N ? ws0 + kbs : nullptr, kbs, w, lane);
  }
  // bf16 rows staged per warp: [2 outputs][32 tokens][64 bytes] (row64_chunk)
  static constexpr int kEpiSmem = 8 * 2 * 32 * 64;
  // Four passes of 32 columns: the warp's 32 tokens' bf16 values (and, for
  // the down-projection, the residuals of that rounding) go through its
  // shared rows so that each store instruction writes eight tokens' 64
  // contiguous bytes.
  static __device__ __forceinline__ void epilogue_regs(const Params &p, const Unit &U, float (&acc)[kW8Cols], int q,
                                                       int h, int lane, uint8_t *epi, const float *) {
    const int col = U.n0 + h * kW8Cols;
    if (q * 32 >= U.nv || col >= p.N) return;  // the warp holds no token, or its columns lie past N
    uint4 *rows_hi = reinterpret_cast<uint4 *>(epi) + (h * 4 + q) * 2 * 32 * 4;
    uint4 *rows_lo = rows_hi + 32 * 4;
    const bool lo = p.out_lo != nullptr;
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float *v = acc + pass * 32 + 8 * c;
        uint4 w;
        w.x = pack_bf16x2(v[0], v[1]);
        w.y = pack_bf16x2(v[2], v[3]);
        w.z = pack_bf16x2(v[4], v[5]);
        w.w = pack_bf16x2(v[6], v[7]);
        rows_hi[row64_chunk(lane, c)] = w;
        if (lo) {
          // residual v - bf16(v), from the rounded halves just packed
          const uint32_t hw[4] = {w.x, w.y, w.z, w.w};
          uint32_t lw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            lw[e] = pack_bf16x2(v[2 * e] - __uint_as_float(hw[e] << 16),
                                v[2 * e + 1] - __uint_as_float(hw[e] & 0xffff0000u));
          rows_lo[row64_chunk(lane, c)] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
      }
      __syncwarp();
      const int chunk = lane & 3;  // 16-byte quarter of a token's 64 bytes
#pragma unroll
      for (int it = 0; it < 4; ++it) {
        const int i = it * 8 + (lane >> 2);  // token within the warp
        const int t = q * 32 + i;
        if (t < U.nv) {
          const size_t o = static_cast<size_t>(U.row0 + t) * p.ldo + col + pass * 32 + chunk * 8;
          *reinterpret_cast<uint4 *>(p.out + o) = rows_hi[row64_chunk(i, chunk)];
          if (lo) *reinterpret_cast<uint4 *>(p.out_lo + o) = rows_lo[row64_chunk(i, chunk)];
        }
      }
      __syncwarp();
    }
  }
};

// gate/up: unit = (group, 128-wide d_ff slice m, <= 128 dispatched tokens).
// B interleaves gate and up rows in 64-row quarters: slice columns f 0-63 of
// gate, then of up, then f 64-127 of gate, then of up.  So column half h of
// the accumulator holds both factors of h for f = 64h .. 64h+63 (columns
// 0-63 of the half gate, with the gate block's scale; 64-127 up, with the up
// block's), and each promotion warp forms its 64 values of
// h = bf16(SiLU(g) * u) from its own registers.  The slice is exactly one
// 128-wide K block of the down GEMM's input, quantised here: amax over the
// block's bf16 values (the two warps of a token quarter exchange their
// halves' maxima), scale amax / 448 (1 if amax is 0), codes
// e4m3_rn_satfinite(v * (448 / amax)) in fp32, the arithmetic of
// quant_rows_kernel, so no separate pass over h is needed.
struct Glu8WPolicy : Glu8Policy {
  static constexpr uint32_t kWeightFormat = kFmtE4M3;
  static constexpr uint32_t kWeightTxBytes = kW8BBytes;  // bytes the weight loads of a K block complete
  static constexpr bool kGateUp = true;  // columns 0-63 of a thread's half: gate block; 64-127: up block
  static constexpr int kEpiSmem = 8 * 32 * 4 + 8 * 32 * 64;  // block maxima, then the code rows (row64_chunk)
  struct Params {
    CUtensorMap wg, wu, sg, su;  // e4m3 [E*F, L] / [F, L], box 64 x 128
    TokenMaps8 tz;               // quantised dispatched z [(T*k+T), L]
    const float *wg_s, *wu_s, *sg_s, *su_s;  // [E, F/128, L/128] / [F/128, L/128]
    const float *zs_t;                        // [L/128, T*k+T] (transposed)
    GroupTable gt;                            // m_tiles = F / 128
    uint8_t *hq;                              // e4m3 h [(T*k+T), F]
    float *hs_t;                              // its scales [F/128, T*k+T] (transposed)
    int F, L, rows;
    uint32_t *status;
  };
  static __device__ __forceinline__ void prefetch(const Params &p) {
    prefetch_tmap(&p.wg); prefetch_tmap(&p.wu); prefetch_tmap(&p.sg); prefetch_tmap(&p.su);
    prefetch_token_maps8(p.tz);
  }
  static __device__ __forceinline__ void stage_aux(const Params &p, uint8_t *aux) { stage_group_table(p.gt, aux); }
  static __device__ __forceinline__ int num_units(const Params &p, const uint8_t *aux) {
    return grouped_num_units(p.gt, aux);
  }
  static __device__ __forceinline__ int k_blocks(const Params &p) { return p.L / 128; }
  static __device__ __forceinline__ Unit unit(const Params &p, int u, const uint8_t *aux) {
    return grouped_unit(p.gt, aux, u, kF8Tile);
  }
  static __device__ __forceinline__ void load_a(const Params &p, const Unit &U, int kb, uint32_t sa, uint32_t bar) {
    load_token_rows8(p.tz, kb, U.row0, token_rows16(U.nv), sa, bar);
  }
  static __device__ __forceinline__ void load_b(const Params &p, const Unit &U, int kb, uint32_t sb, uint32_t bar) {
    const bool sh = U.g == p.gt.E;
    const CUtensorMap *mg = sh ? &p.sg : &p.wg, *mu = sh ? &p.su : &p.wu;
    const int row = (sh ? 0 : U.g * p.F) + U.m * kF8Tile;
    tma_load_2d(sb, mg, bar, kb * 128, row);
    tma_load_2d(sb + 64 * 128, mu, bar, kb * 128, row);
    tma_load_2d(sb + 128 * 128, mg, bar, kb * 128, row + 64);
    tma_load_2d(sb + 192 * 128, mu, bar, kb * 128, row + 64);
  }
  static __device__ __forceinline__ void stage_scales(const Params &p, const Unit &U, float *tok, float *w, float *,
                                                      int lane) {
    const bool sh = U.g == p.gt.E;
    const int kbs = p.L / 128;
    const size_t blk = (static_cast<size_t>(sh ? 0 : U.g) * (p.F / 128) + U.m) * kbs;
    stage_token_scales(p.zs_t, p.rows, U.row0, U.nv, kbs, tok, lane);
    stage_weight_scales((sh ? p.sg_s : p.wg_s) + blk, (sh ? p.su_s : p.wu_s) + blk, kbs, w, lane);
  }
  // Warp (q, hh): h for its 32 tokens and f = 64hh .. 64hh+63 of the slice;
  // the partner warp (q, 1-hh) holds the other 64 values of each token's
  // block.  Each warp writes its 64 e4m3 codes per token through its own
  // shared rows (one 16-byte store per lane covers a quarter of a token's 64
  // bytes, eight tokens per instruction).
  static __device__ __forceinline__ void epilogue_regs(const Params &p, const Unit &U, float (&acc)[kW8Cols], int q,
                                                       int hh, int lane, uint8_t *epi, const float *) {
    const int pw = hh * 4 + q;
    float *bmax = reinterpret_cast<float *>(epi);  // [8 warps][32]
    // SiLU(g) = g / 2 * (1 + tanh(g / 2)): one special-function instruction
    // per value (exp and reciprocal would take two), with tanh.approx's error
    // (about 2^-11 relative) far below the e4m3 step h is quantised to next
    // (the bf16 rounding of h goes two values per conversion: cvt.rn.bf16x2
    // rounds each half as the scalar conversion does)
    float hv[64];
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 64; i += 2) {
      // packed fp32x2 arithmetic (round to nearest per lane)
      const float2 hg = __fmul2_rn(make_float2(acc[i], acc[i + 1]), make_float2(0.5f, 0.5f));
      float2 th;
      asm("tanh.approx.f32 %0, %1;" : "=f"(th.x) : "f"(hg.x));
      asm("tanh.approx.f32 %0, %1;" : "=f"(th.y) : "f"(hg.y));
      const float2 v = __fmul2_rn(__ffma2_rn(hg, th, hg), make_float2(acc[64 + i], acc[64 + i + 1]));
      const uint32_t b2 = pack_bf16x2(v.x, v.y);
      hv[i] = __uint_as_float(b2 << 16);
      hv[i + 1] = __uint_as_float(b2 & 0xffff0000u);
      amax = fmaxf(amax, fmaxf(fabsf(hv[i]), fabsf(hv[i + 1])));
    }
    // the partner reads this slot before it passes the promotion warps'
    // barrier at the end of the next unit, which comes before the next write
    bmax[pw * 32 + lane] = amax;
    named_bar_sync(3 + q, 64);
    amax = fmaxf(amax, bmax[(pw ^ 4) * 32 + lane]);
    float scale = 1.0f, inv = 0.0f;
    if (amax != 0.0f) {
      scale = amax / 448.0f;
      inv = 448.0f / amax;
    }
    const int t = q * 32 + lane;
    if (hh == 0 && t < U.nv) p.hs_t[static_cast<size_t>(U.m) * p.rows + U.row0 + t] = scale;
    uint4 *rows = reinterpret_cast<uint4 *>(epi + 8 * 32 * 4) + pw * 32 * 4;  // [32 tokens][64 bytes]
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t wd[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = 4 * c + e;  // word i: codes 4i .. 4i+3
        const float2 a = __fmul2_rn(make_float2(hv[4 * i], hv[4 * i + 1]), make_float2(inv, inv));
        const float2 b = __fmul2_rn(make_float2(hv[4 * i + 2], hv[4 * i + 3]), make_float2(inv, inv));
        wd[e] = static_cast<uint32_t>(e4m3x2(a.x, a.y)) | (static_cast<uint32_t>(e4m3x2(b.x, b.y)) << 16);
      }
      rows[row64_chunk(lane, c)] = make_uint4(wd[0], wd[1], wd[2], wd[3]);
    }
    __syncwarp();
    const int chunk = lane & 3;  // 16-byte quarter of a token's 64 bytes
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int i = it * 8 + (lane >> 2);  // token within the warp
      const int tt = q * 32 + i;
      if (tt < U.nv)
        *reinterpret_cast<uint4 *>(p.hq + static_cast<size_t>(U.row0 + tt) * p.F + U.m * kF8Tile + hh * 64 +
                                   chunk * 16) = rows[row64_chunk(i, chunk)];
    }
    __syncwarp();  // the rows are rewritten by the next unit's epilogue
  }
};

// expert down: unit = (group, 256-wide d_lat slice m, <= 128 dispatched
// tokens); column half h = d_lat rows 256m + 128h .. +127 (weight block
// 2m + h).  The stager's slot table is Down8Policy's; the weighted slot
// stores go through the warp's shared rows in four 32-column passes, so each
// store instruction covers four tokens' 128 contiguous bytes.
struct Down8WPolicy : Down8Policy {
  static constexpr uint32_t kWeightFormat = kFmtE4M3;
  static constexpr uint32_t kWeightTxBytes = kW8BBytes;  // bytes the weight loads of a K block complete
  static constexpr bool kGateUp = false;  // the thread's 128 columns share one weight block
  static __device__ __forceinline__ Unit unit(const Params &p, int u, const uint8_t *aux) {
    return grouped_unit(p.gt, aux, u, kF8Tile);
  }
  static __device__ __forceinline__ void load_b(const Params &p, const Unit &U, int kb, uint32_t sb, uint32_t bar) {
    const bool sh = U.g == p.gt.E;
    const int row = (sh ? 0 : U.g * p.L) + U.m * kW8N;
    tma_load_2d(sb, sh ? &p.sd : &p.wd, bar, kb * 128, row);
    tma_load_2d(sb + kF8OpBytes, sh ? &p.sd : &p.wd, bar, kb * 128, row + kF8Tile);
  }
  static __device__ __forceinline__ void stage_scales(const Params &p, const Unit &U, float *tok, float *w,
                                                      float *extra, int lane) {
    const bool sh = U.g == p.gt.E;
    const int kbs = p.F / 128;
    const size_t blk = (static_cast<size_t>(sh ? 0 : U.g) * (p.L / 128) + 2 * U.m) * kbs;
    const float *ws = (sh ? p.sd_s : p.wd_s) + blk;
    stage_token_scales(p.hs_t, p.rows, U.row0, U.nv, kbs, tok, lane);
    stage_weight_scales(ws, ws + kbs, kbs, w, lane);  // blocks 2m and 2m + 1
    stage_slots(p, U, extra, lane);
  }
  static __device__ __forceinline__ void epilogue_regs(const Params &p, const Unit &U, float (&acc)[kW8Cols], int q,
                                                       int h, int lane, uint8_t *epi, const float *extra) {
    const int *slot = reinterpret_cast<const int *>(extra);
    const float *wt = extra + kF8Tile;
    // this warp's rows: [32 tokens][32 floats], 16-byte chunk c of row r at
    // chunk c ^ (r & 7), so the 128-bit writes of a quarter-warp (eight rows)
    // and its 128-bit reads (one row's eight chunks) both spread over all banks
    float4 *wrow = reinterpret_cast<float4 *>(epi) + (h * 4 + q) * 32 * 8;
    const float my_wt = q * 32 + lane < U.nv ? wt[q * 32 + lane] : 0.f;
    const int part = lane & 7;  // 16-byte eighth of a token's 128 bytes
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) {
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const float *a = acc + pass * 32 + 4 * c;
        const float2 lo = __fmul2_rn(make_float2(a[0], a[1]), make_float2(my_wt, my_wt));
        const float2 hi = __fmul2_rn(make_float2(a[2], a[3]), make_float2(my_wt, my_wt));
        wrow[lane * 8 + (c ^ (lane & 7))] = make_float4(lo.x, lo.y, hi.x, hi.y);
      }
      __syncwarp();
#pragma unroll
      for (int it = 0; it < 8; ++it) {
        const int i = it * 4 + (lane >> 3);  // token within the warp
        const int t = q * 32 + i;
        if (t < U.nv)
          *reinterpret_cast<float4 *>(p.slots + static_cast<size_t>(slot[t]) * p.L + U.m * kW8N + h * kW8Cols +
                                      pass * 32 + part * 4) = wrow[i * 8 + (part ^ (i & 7))];
      }
      __syncwarp();
    }
  }
};

// FP4 expert weights: the same units with each weight matrix given as packed
// e2m1 codes (two per byte, the lower K index in the low nibble).  The weight
// maps use the 16U4_ALIGN16B TMA type, which unpacks 16 codes into each 16
// bytes of the shared tile (and completes half a byte per code on the
// barrier), and the MMA reads B as e2m1 (every e2m1 value is an e4m3 value,
// so the partial products equal those of the codes expanded to e4m3);
// scales, promotion and epilogues are the e4m3 policies'.
struct Glu4WPolicy : Glu8WPolicy {
  static constexpr uint32_t kWeightFormat = kFmtE2M1;
  static constexpr uint32_t kWeightTxBytes = kW8BBytes / 2;  // counted as packed codes, half a byte each
};

struct Down4WPolicy : Down8WPolicy {
  static constexpr uint32_t kWeightFormat = kFmtE2M1;
  static constexpr uint32_t kWeightTxBytes = kW8BBytes / 2;
};

}  // namespace mrl
