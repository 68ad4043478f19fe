// gemm8_sm100.cuh — e4m3 x e4m3 tcgen05 GEMM with fp32 block scales (the FP8
// variant of the layer).
//
// Operands carry one fp32 scale per 128-wide K block: the activation (token)
// side per row, the weight side per 128 x 128 block.  Such scales are not
// powers of two, so the tensor core's block-scaled modes cannot apply them:
// each 128-wide K block is accumulated on its own in TMEM (four 32-deep
// kind::f8f6f4 MMAs into one of four partial buffers), and eight promotion
// warps fold it into an fp32 register accumulator,
//     acc[m][n] += partial[m][n] * tok_scale[kb][m] * w_scale[cls(n)][kb],
// before releasing the partial buffer to the MMA issuer.  After the last K
// block the same warps run the policy's epilogue on the registers.
//
// Tokens are on M (TMEM lanes) and weights on N in every FP8 GEMM, and a
// unit's 128 N columns fall in at most two weight blocks (one per column
// half), so the scale a thread applies to its 64 columns is ONE scalar per K
// block: two 4-byte shared loads and an FMUL, then 32 packed fp32x2 FMAs.  (With tokens on
// N every thread would need 64 distinct column scales per K block; as warp-
// wide broadcast loads those cost 8 KB of shared-memory return bandwidth per
// warp per K block and throttled the whole pipeline.)
//
//   warp 0    : TMA producer for A (tokens)   warp 2 : TMA producer for B
//   warp 1    : TMEM allocator + MMA issuer
//   warp 3    : scale stager — writes each unit's token scales and weight
//               scales into one of two shared-memory tables, ahead of use
//   warps 4-11: promotion + epilogue; warp w reads TMEM lanes 32*(w%4)..+31
//               (its 32 tokens), columns 64*((w-4)/4)..+63
//
// Stage j of the 4-deep shared-memory ring and partial buffer j serve global
// K block g with j = g % 4; the commit after block g's MMAs both frees stage j
// for the producers and hands partial j to the promotion warps.  All waits are
// bounded (mbar_wait); the promotion warps agree on an abort once per unit.
// No TMA load uses multicast.
#pragma once
#include "gemm_sm100.cuh"
#include "policies.cuh"

namespace mrl {

constexpr int kF8Threads = 384;
constexpr int kF8Ring = 4;      // stages == TMEM partial buffers
constexpr int kF8Tile = 128;    // tokens (M) and weight columns (N) per unit
constexpr int kF8Half = 64;     // columns per promotion warp
constexpr int kF8MaxKB = 32;    // K blocks of 128 per unit (K <= 4096)
constexpr int kF8PromoWarp0 = 4;
constexpr int kF8PromoThreads = 256;
constexpr int kF8OpBytes = kF8Tile * 128;  // one operand tile per K block

// An e4m3 token tensor [rows, K] with four box heights (16 / 32 / 64 / 128
// rows x 128 B): a unit loads only its dispatched rows, rounded up to 16, so
// a group of a few tokens (decode) moves 2 KB per K block instead of 16 KB.
// The tile's remaining smem rows keep older bytes; an accumulator row depends
// on its own A row only, and rows >= the unit's count are never stored.
struct TokenMaps8 {
  CUtensorMap m16, m32, m64, m128;
};

__device__ __forceinline__ int token_rows16(int nv) { return (nv + 15) & ~15; }

__device__ __forceinline__ void load_token_rows8(const TokenMaps8 &t, int kb, int y0, int n, uint32_t sa,
                                                 uint32_t bar) {
  const int x = kb * 128;
  if (n == kF8Tile) {
    tma_load_2d(sa, &t.m128, bar, x, y0);
    return;
  }
  int r = 0;
  if (r + 64 <= n) { tma_load_2d(sa + r * 128, &t.m64, bar, x, y0 + r); r += 64; }
  if (r + 32 <= n) { tma_load_2d(sa + r * 128, &t.m32, bar, x, y0 + r); r += 32; }
  if (r + 16 <= n) tma_load_2d(sa + r * 128, &t.m16, bar, x, y0 + r);
}

// ------------------------------------------------------------ FP4 weights
// Expert weights given as packed e2m1 codes (two per byte, the lower K index
// in the low nibble) are expanded in shared memory into the e4m3 B tile the
// MMA reads.  The expansion is exact (every e2m1 value is an e4m3 value): a
// table lookup on the integer pipes with byte permutes,
//   magnitude code 0..7 (0, 0.5, 1, 1.5, 2, 3, 4, 6) -> e4m3 byte
//   00 30 38 3C 40 44 48 4C, and the code's sign bit (bit 3) -> bit 7.
// c holds 4 codes in bits 0..15 (code i in nibble i; the permutes read only
// those bits); the result holds their 4 e4m3 bytes (byte i from code i).  The
// second permute uses the selector's bit 3 in its sign-replicating sense: a
// negative code's byte becomes 0xFF (the table bytes 0x80 have their msb
// set), a positive one's 0x80.
__device__ __forceinline__ uint32_t e2m1x4_to_e4m3x4(uint32_t c) {
  uint32_t mag, sgn;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(mag) : "r"(0x3C383000u), "r"(0x4C484440u), "r"(c & 0x7777u));
  asm("prmt.b32 %0, %1, %1, %2;" : "=r"(sgn) : "r"(0x80808080u), "r"(c));
  return mag | (((sgn & 0x7F7F7F7Fu) + 0x01010101u) & 0x80808080u);
}

// 16 packed bytes (32 codes) -> 32 e4m3 bytes in the same element order.
__device__ __forceinline__ void e2m1x32_to_e4m3(uint4 in, uint4 &lo, uint4 &hi) {
  lo = make_uint4(e2m1x4_to_e4m3x4(in.x), e2m1x4_to_e4m3x4(in.x >> 16), e2m1x4_to_e4m3x4(in.y),
                  e2m1x4_to_e4m3x4(in.y >> 16));
  hi = make_uint4(e2m1x4_to_e4m3x4(in.z), e2m1x4_to_e4m3x4(in.z >> 16), e2m1x4_to_e4m3x4(in.w),
                  e2m1x4_to_e4m3x4(in.w >> 16));
}

// One K block of packed weights (128 rows x 64 B, row-major at src) into the
// e4m3 B tile at dst (128 rows x 128 B, 16-byte chunk c of row r at chunk
// position c ^ (r & 7): the SWIZZLE_128B layout TMA would write; dst is
// 1024-byte aligned).  Thread tid of the 256 promotion threads takes 16
// packed bytes: row tid / 4 (+64 in the second pass), quarter tid % 4.
__device__ __forceinline__ void expand_fp4_tile(const uint8_t *src, uint8_t *dst, int tid) {
#pragma unroll
  for (int pass = 0; pass < 2; ++pass) {
    const int r = pass * 64 + (tid >> 2), q = tid & 3;
    const uint4 in = *reinterpret_cast<const uint4 *>(src + r * 64 + q * 16);
    uint4 lo, hi;
    e2m1x32_to_e4m3(in, lo, hi);
    const int sw = r & 7;
    *reinterpret_cast<uint4 *>(dst + r * 128 + (((2 * q) ^ sw) << 4)) = lo;
    *reinterpret_cast<uint4 *>(dst + r * 128 + (((2 * q + 1) ^ sw) << 4)) = hi;
  }
}

// K blocks the promotion warps expand ahead of the one they promote.
constexpr int kF4Ahead = 3;

__device__ __forceinline__ void prefetch_token_maps8(const TokenMaps8 &t) {
  prefetch_tmap(&t.m16);
  prefetch_tmap(&t.m32);
  prefetch_tmap(&t.m64);
  prefetch_tmap(&t.m128);
}

// One scale table: tok[kF8MaxKB][kF8Tile], w[2][kF8MaxKB], the unit's
// descriptor (so the promotion warps need not search the group table), and
// 256 words a policy may fill for its epilogue (the expert-down GEMM: each
// token's slot index and routing weight).
constexpr int kF8TabUnit = kF8MaxKB * kF8Tile + 2 * kF8MaxKB;
constexpr int kF8TabExtra = kF8TabUnit + 8;
constexpr int kF8TabFloats = kF8TabExtra + 2 * kF8Tile;

template <class P>
struct Gemm8Smem {
  static constexpr int kStageBytes = 2 * kF8OpBytes;
  static constexpr int kRing = kF8Ring * kStageBytes;
  static constexpr int kTabOff = kRing;
  static constexpr int kBarOff = kTabOff + 2 * kF8TabFloats * 4;
  static constexpr int kNumBars = 4 * kF8Ring + 4;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kEpiOff = (kMiscOff + 16 + 127) & ~127;
  static constexpr int kAuxOff = (kEpiOff + P::kEpiSmem + 127) & ~127;
  static constexpr int kTotal = kAuxOff + P::kAuxSmem + 1024;
};

// Time-bounded wait that ignores the abort flag: the abort path uses it to let
// the tensor core finish the MMAs already issued before TMEM is freed.
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer() - t0 > kWaitLimitNs) return;
}

template <class P>
__global__ void __launch_bounds__(kF8Threads, 1) gemm8_kernel(const __grid_constant__ typename P::Params p) {
  using L = Gemm8Smem<P>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kBarOff);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMiscOff);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMiscOff + 4);
  volatile int *hold_flag = reinterpret_cast<volatile int *>(smem + L::kMiscOff + 8);
  float *tabs = reinterpret_cast<float *>(smem + L::kTabOff);
  uint8_t *epi_smem = smem + L::kEpiOff;
  uint8_t *aux = smem + L::kAuxOff;

  const uint32_t full0 = smem_u32(bars);
  const uint32_t done0 = full0 + 8 * kF8Ring;   // MMAs of the K block completed
  const uint32_t free0 = done0 + 8 * kF8Ring;   // partial buffer promoted
  const uint32_t ready0 = free0 + 8 * kF8Ring;  // FP4: the stage's B tile expanded
  const uint32_t sfull0 = ready0 + 8 * kF8Ring; // scale table b written
  const uint32_t sempty0 = sfull0 + 16;         // scale table b read
  const uint32_t ring = smem_u32(smem);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  uint32_t *status = p.status;

  if (threadIdx.x == 0) {
    const uint2 hdr = call_header(status);  // loaded first: the barrier set-up hides its latency
    for (int j = 0; j < kF8Ring; ++j) {
      mbar_init(full0 + 8 * j, 2);
      mbar_init(done0 + 8 * j, 1);
      mbar_init(free0 + 8 * j, 8);
      mbar_init(ready0 + 8 * j, kF8PromoThreads / 32);
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
  const uint32_t idesc = idesc_e4m3(kF8Tile, kF8Tile);
  if (*abort_flag) goto done;

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
          const uint32_t j = g & (kF8Ring - 1);
          if (g >= kF8Ring && !mbar_wait(done0 + 8 * j, ((g / kF8Ring) - 1) & 1, abort_flag, status)) goto done;
          mbar_arrive_expect_tx(full0 + 8 * j, isA ? P::a_bytes(U) : P::b_bytes());
          const uint32_t st = ring + j * L::kStageBytes;
          if (isA)
            P::load_a(p, U, kb, st, full0 + 8 * j);
          else  // FP4: the packed tile lands in the A slot's upper half (token tiles <= 64 rows)
            P::load_b(p, U, kb, st + (P::kFp4B ? kF8OpBytes / 2 : kF8OpBytes), full0 + 8 * j);
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
          const uint32_t j = g & (kF8Ring - 1);
          // FP4: the stage is ready once the promotion warps have expanded its B tile
          if (!mbar_wait((P::kFp4B ? ready0 : full0) + 8 * j, (g / kF8Ring) & 1, abort_flag, status)) goto done;
          if (g >= kF8Ring && !mbar_wait(free0 + 8 * j, ((g / kF8Ring) - 1) & 1, abort_flag, status)) goto done;
          tc_fence_after();
          const uint32_t a_s = ring + j * L::kStageBytes;
          const uint32_t b_s = a_s + kF8OpBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_f8(tmem_base + j * kF8Tile, sdesc_sw128(a_s + kk * 32), sdesc_sw128(b_s + kk * 32), idesc, kk != 0);
          umma_commit(done0 + 8 * j);
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
  } else {
    const int pw = warp - kF8PromoWarp0;        // 0..7
    const int q = warp & 3;                     // TMEM lane quarter: tokens 32q..32q+31
    const int h = pw >> 2;                      // column half
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const int cls = P::scale_class(h);
    uint32_t g = 0;
    int ul = 0;
    // FP4: K block c of this CTA's sequence (c < ctot) is expanded while block
    // c - kF4Ahead is promoted; its stage was last read by the MMA of block
    // c - 4, complete once block c - kF4Ahead - 1 <= c - 4 was seen done.
    uint32_t cx = 0;
    const uint32_t ctot =
        static_cast<int>(blockIdx.x) < nunits
            ? static_cast<uint32_t>((nunits - 1 - static_cast<int>(blockIdx.x)) / static_cast<int>(gridDim.x) + 1) *
                  static_cast<uint32_t>(kblocks)
            : 0u;
    auto expand_to = [&](uint32_t lim) -> bool {
      for (; cx < lim && cx < ctot; ++cx) {
        const uint32_t j = cx & (kF8Ring - 1);
        if (!__all_sync(0xffffffffu, mbar_wait(full0 + 8 * j, (cx / kF8Ring) & 1, abort_flag, status))) return false;
        uint8_t *stg = smem + j * L::kStageBytes;
        expand_fp4_tile(stg + kF8OpBytes / 2, stg + kF8OpBytes, pw * 32 + lane);
        fence_proxy_async_shared();
        __syncwarp();
        if (lane == 0) mbar_arrive(ready0 + 8 * j);
      }
      return true;
    };
    bool lost = false;  // FP4: an expansion wait gave up
    if constexpr (P::kFp4B) lost = !expand_to(kF4Ahead);
    for (int u = blockIdx.x; u < nunits; u += gridDim.x, ++ul) {
      const int b = ul & 1;
      const float *tok = tabs + b * kF8TabFloats + q * 32 + lane;
      const float *wsc = tabs + b * kF8TabFloats + kF8MaxKB * kF8Tile + cls * kF8MaxKB;
      bool bad = !__all_sync(0xffffffffu, mbar_wait(sfull0 + 8 * b, (ul >> 1) & 1, abort_flag, status)) || lost;
      Unit U;
      {
        const int *d = reinterpret_cast<const int *>(tabs + b * kF8TabFloats + kF8TabUnit);
        U.g = d[0]; U.m = d[1]; U.n0 = d[2]; U.nv = d[3]; U.row0 = d[4]; U.nsub = 1;
      }
      // no token of the unit in this warp's 32 rows (decode-sized groups):
      // its partials need no promotion, and the epilogue stores nothing for it
      const bool idle = q * 32 >= U.nv;
      float acc[kF8Half];
#pragma unroll
      for (int i = 0; i < kF8Half; ++i) acc[i] = 0.f;
      for (int kb = 0; kb < kblocks; ++kb, ++g) {
        const uint32_t j = g & (kF8Ring - 1);
        if constexpr (P::kFp4B) {
          if (!bad && !expand_to(g + 1 + kF4Ahead)) bad = lost = true;
        }
        if (!bad) bad = !__all_sync(0xffffffffu, mbar_wait(done0 + 8 * j, (g / kF8Ring) & 1, abort_flag, status));
        if (bad) continue;
        if (idle) {
          __syncwarp();
          if (lane == 0) mbar_arrive(free0 + 8 * j);
          continue;
        }
        const float s = tok[kb * kF8Tile] * wsc[kb];
        tc_fence_after();
        float v[kF8Half];
        tmem_ld64_sync(tmem_base + j * kF8Tile + lane_off + h * kF8Half, v);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(free0 + 8 * j);  // the partial is in registers
        // packed fp32x2 FMAs (round to nearest per lane: the same values as fmaf)
        const float2 s2 = make_float2(s, s);
#pragma unroll
        for (int i = 0; i < kF8Half; i += 2) {
          const float2 r = __ffma2_rn(make_float2(v[i], v[i + 1]), s2, make_float2(acc[i], acc[i + 1]));
          acc[i] = r.x;
          acc[i + 1] = r.y;
        }
      }
      if (bar_red_or(1, kF8PromoThreads, bad || *abort_flag)) goto done;
      P::epilogue_regs(p, U, acc, q, h, lane, epi_smem, tabs + b * kF8TabFloats + kF8TabExtra);
      __syncwarp();
      if (lane == 0) mbar_arrive(sempty0 + 8 * b);  // table b (read by the epilogue too) is free
    }
  }
done:
  if (warp == 1 && lane == 0 && *abort_flag && issued >= 0) {
    // let the MMAs already issued land before the accumulator is freed
    const uint32_t j = static_cast<uint32_t>(issued) & (kF8Ring - 1);
    mbar_drain(done0 + 8 * j, (static_cast<uint32_t>(issued) / kF8Ring) & 1);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ------------------------------------------------------------- FP8 policies
// Scale arrays: a weight matrix [out, in] has fp32 scales [out/128, in/128]
// (routed experts: [E, ...]); an activation tensor quantised inside the layer
// has its scales transposed, [K/128, rows], so that a unit's token scales for
// one K block are contiguous.

// Stager helper: tok[kb][r] = act[kb * ld + row0 + r] for r < nv (0 for the
// unit's unused token rows); 16 loads in flight per batch.
__device__ __forceinline__ void stage_token_scales(const float *act, long ld, long row0, int nv, int kbs, float *tok,
                                                   int lane) {
  for (int kb0 = 0; kb0 < kbs; kb0 += 4) {
    float a[4][4];
#pragma unroll
    for (int d = 0; d < 4; ++d)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int r = c * 32 + lane;
        a[d][c] = (kb0 + d < kbs && r < nv) ? __ldg(act + static_cast<long>(kb0 + d) * ld + row0 + r) : 0.f;
      }
#pragma unroll
    for (int d = 0; d < 4; ++d)
      if (kb0 + d < kbs)
#pragma unroll
        for (int c = 0; c < 4; ++c) tok[(kb0 + d) * kF8Tile + c * 32 + lane] = a[d][c];
  }
}

// w[c][kb] = ws_c[kb] for kb < kbs (kbs <= 32: lane kb).
__device__ __forceinline__ void stage_weight_scales(const float *ws0, const float *ws1, int kbs, float *w, int lane) {
  if (lane < kbs) {
    w[lane] = __ldg(ws0 + lane);
    if (ws1) w[kF8MaxKB + lane] = __ldg(ws1 + lane);
  }
}

// Projection out = bf16(a w^T): unit = (128-token tile m, 128-column tile n0);
// the N tile is one weight block.
struct Dense8Policy {
  static constexpr int kEpiSmem = 0;
  static constexpr int kAuxSmem = 0;
  static constexpr bool kFp4B = false;  // weights arrive as e4m3 tiles
  static __device__ __forceinline__ uint32_t b_bytes() { return kF8OpBytes; }
  struct Params {
    CUtensorMap ta;  // a codes [M, K], box 128 x 128
    CUtensorMap tb;  // w codes [N, K], box 128 x 128
    const float *as_t, *ws;  // [K/128, M] (transposed), [N/128, K/128]
    __nv_bfloat16 *out, *out_lo;
    long ldo;
    int M, N, K, m_tiles, n_tiles;
    uint32_t *status;
  };
  static __device__ __forceinline__ void prefetch(const Params &p) {
    prefetch_tmap(&p.ta);
    prefetch_tmap(&p.tb);
  }
  static __device__ __forceinline__ void stage_aux(const Params &, uint8_t *) {}
  static __device__ __forceinline__ int num_units(const Params &p, const uint8_t *) { return p.m_tiles * p.n_tiles; }
  static __device__ __forceinline__ int k_blocks(const Params &p) { return p.K / 128; }
  static __device__ __forceinline__ Unit unit(const Params &p, int u, const uint8_t *) {
    Unit U;
    U.g = 0;
    U.m = u / p.n_tiles;                      // token tile
    U.n0 = (u % p.n_tiles) * kF8Tile;         // weight columns
    U.row0 = U.m * kF8Tile;
    U.nv = min(kF8Tile, p.M - U.row0);        // valid tokens
    U.nsub = 1;
    return U;
  }
  static __device__ __forceinline__ uint32_t a_bytes(const Unit &) { return kF8OpBytes; }
  static __device__ __forceinline__ void load_a(const Params &p, const Unit &U, int kb, uint32_t sa, uint32_t bar) {
    tma_load_2d(sa, &p.ta, bar, kb * 128, U.row0);
  }
  static __device__ __forceinline__ void load_b(const Params &p, const Unit &U, int kb, uint32_t sb, uint32_t bar) {
    tma_load_2d(sb, &p.tb, bar, kb * 128, U.n0);
  }
  static __device__ __forceinline__ int scale_class(int) { return 0; }
  static __device__ __forceinline__ void stage_scales(const Params &p, const Unit &U, float *tok, float *w, float *,
                                                      int lane) {
    const int kbs = p.K / 128;
    stage_token_scales(p.as_t, p.M, U.row0, U.nv, kbs, tok, lane);
    stage_weight_scales(p.ws + static_cast<size_t>(U.n0 / 128) * kbs, nullptr, kbs, w, lane);
  }
  static __device__ __forceinline__ void epilogue_regs(const Params &p, const Unit &U, float (&acc)[kF8Half], int q,
                                                       int h, int lane, uint8_t *, const float *) {
    const int t = q * 32 + lane;
    if (t >= U.nv) return;
    const long row = U.row0 + t;
    const int col = U.n0 + h * kF8Half;
    uint4 *dst = reinterpret_cast<uint4 *>(p.out + row * p.ldo + col);
    uint4 *dlo = p.out_lo ? reinterpret_cast<uint4 *>(p.out_lo + row * p.ldo + col) : nullptr;
#pragma unroll
    for (int i = 0; i < kF8Half / 8; ++i) {
      const float *v = acc + 8 * i;
      uint4 w;
      w.x = pack_bf16x2(v[0], v[1]);
      w.y = pack_bf16x2(v[2], v[3]);
      w.z = pack_bf16x2(v[4], v[5]);
      w.w = pack_bf16x2(v[6], v[7]);
      dst[i] = w;
      if (dlo) {
        float r[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) r[e] = v[e] - __bfloat162float(__float2bfloat16_rn(v[e]));
        uint4 l;
        l.x = pack_bf16x2(r[0], r[1]);
        l.y = pack_bf16x2(r[2], r[3]);
        l.z = pack_bf16x2(r[4], r[5]);
        l.w = pack_bf16x2(r[6], r[7]);
        dlo[i] = l;
      }
    }
  }
};

// gate/up: unit = (group, 64-wide d_ff slice m, <= 128 dispatched tokens);
// B = 64 gate rows then the 64 matching up rows (column half 0 / 1, scale
// class 0 / 1); h = bf16(SiLU(g) * u) (quantised for the down GEMM by a
// separate pass).
struct Glu8Policy {
  static constexpr int kEpiSmem = 8 * 32 * 33 * 4;
  static constexpr int kAuxSmem = kGroupAuxSmem;
  static constexpr bool kFp4B = false;  // weights arrive as e4m3 tiles
  static __device__ __forceinline__ uint32_t b_bytes() { return kF8OpBytes; }
  struct Params {
    CUtensorMap wg, wu, sg, su;  // e4m3 [E*F, L] / [F, L], box 64 x 128
    TokenMaps8 tz;               // quantised dispatched z [(T*k+T), L], boxes 16..128 x 128
    const float *wg_s, *wu_s, *sg_s, *su_s;  // [E, F/128, L/128] / [F/128, L/128]
    const float *zs_t;                        // [L/128, T*k+T] (transposed)
    GroupTable gt;
    __nv_bfloat16 *h;
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
  static __device__ __forceinline__ uint32_t a_bytes(const Unit &U) { return token_rows16(U.nv) * 128; }
  static __device__ __forceinline__ void load_a(const Params &p, const Unit &U, int kb, uint32_t sa, uint32_t bar) {
    load_token_rows8(p.tz, kb, U.row0, token_rows16(U.nv), sa, bar);
  }
  static __device__ __forceinline__ void load_b(const Params &p, const Unit &U, int kb, uint32_t sb, uint32_t bar) {
    const bool sh = U.g == p.gt.E;
    const int row = (sh ? 0 : U.g * p.F) + U.m * 64;
    tma_load_2d(sb, sh ? &p.sg : &p.wg, bar, kb * 128, row);
    tma_load_2d(sb + 64 * 128, sh ? &p.su : &p.wu, bar, kb * 128, row);
  }
  static __device__ __forceinline__ int scale_class(int h) { return h; }
  static __device__ __forceinline__ void stage_scales(const Params &p, const Unit &U, float *tok, float *w, float *,
                                                      int lane) {
    const bool sh = U.g == p.gt.E;
    const int kbs = p.L / 128;
    const size_t blk = (static_cast<size_t>(sh ? 0 : U.g) * (p.F / 128) + (U.m * 64) / 128) * kbs;
    stage_token_scales(p.zs_t, p.rows, U.row0, U.nv, kbs, tok, lane);
    stage_weight_scales((sh ? p.sg_s : p.wg_s) + blk, (sh ? p.su_s : p.wu_s) + blk, kbs, w, lane);
  }
  // Warp (q, 0) holds one token's gate values for f = 64m .. 64m+63, warp
  // (q, 1) the up values; each hands the other half of its row across
  // shared memory (named barrier 3 + q, 64 threads), then warp (q, hh)
  // computes h for f = 64m + 32hh .. +31 of its 32 tokens and writes them
  // through its own shared rows so that each store instruction covers 8
  // tokens' 64 contiguous bytes.
  static __device__ __forceinline__ void epilogue_regs(const Params &p, const Unit &U, float (&acc)[kF8Half], int q,
                                                       int hh, int lane, uint8_t *epi, const float *) {
    float *xb = reinterpret_cast<float *>(epi);  // [8 warps][32][33]
    const int pw = hh * 4 + q;
    float *mine = xb + (pw * 32 + lane) * 33;
    const float *other = xb + ((pw ^ 4) * 32 + lane) * 33;
#pragma unroll
    for (int i = 0; i < 32; ++i) mine[i] = hh == 0 ? acc[32 + i] : acc[i];
    named_bar_sync(3 + q, 64);
    uint32_t packed[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float hv[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int c = 2 * i + e;
        const float gv = hh == 0 ? acc[c] : other[c];
        const float uv = hh == 0 ? other[c] : acc[32 + c];
        hv[e] = __fdividef(gv, 1.0f + __expf(-gv)) * uv;
      }
      packed[i] = pack_bf16x2(hv[0], hv[1]);
    }
    named_bar_sync(3 + q, 64);  // both warps of the pair are done reading the exchange rows
    uint32_t *wrow = reinterpret_cast<uint32_t *>(xb + pw * 32 * 33);  // this warp's rows: [32 tokens][17 words]
#pragma unroll
    for (int i = 0; i < 16; ++i) wrow[lane * 17 + i] = packed[i];
    __syncwarp();
    const int chunk = lane & 3;  // 16-byte quarter of a token's 64 bytes
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int i = it * 8 + (lane >> 2);  // token within the warp
      const int t = q * 32 + i;
      if (t < U.nv) {
        uint4 w;
        w.x = wrow[i * 17 + chunk * 4 + 0];
        w.y = wrow[i * 17 + chunk * 4 + 1];
        w.z = wrow[i * 17 + chunk * 4 + 2];
        w.w = wrow[i * 17 + chunk * 4 + 3];
        *reinterpret_cast<uint4 *>(p.h + static_cast<size_t>(U.row0 + t) * p.F + U.m * 64 + hh * 32 + chunk * 8) = w;
      }
    }
    __syncwarp();  // the rows are rewritten by the next unit's exchange
  }
};

// expert down: unit = (group, 128-wide d_lat slice m, <= 128 dispatched
// tokens).  The stager also looks up each token's slot index and routing
// weight (dispatch permutation, scaled weights) into the table; the epilogue
// scales its 64 columns and writes them through its own shared rows so that
// each store instruction covers four tokens' 128 contiguous bytes.
struct Down8Policy {
  static constexpr int kEpiSmem = 8 * 32 * 33 * 4;
  static constexpr int kAuxSmem = kGroupAuxSmem;
  static constexpr bool kFp4B = false;  // weights arrive as e4m3 tiles
  static __device__ __forceinline__ uint32_t b_bytes() { return kF8OpBytes; }
  struct Params {
    CUtensorMap wd, sd;  // e4m3 [E*L, F] / [L, F], box 128 x 128
    TokenMaps8 th;       // quantised h [(T*k+T), F], boxes 16..128 x 128
    const float *wd_s, *sd_s;  // [E, L/128, F/128] / [L/128, F/128]
    const float *hs_t;         // [F/128, T*k+T] (transposed)
    GroupTable gt;
    const int32_t *perm;
    const float *wscaled;
    float *slots;
    int L, F, k, Tk, rows;
    uint32_t *status;
  };
  static __device__ __forceinline__ void prefetch(const Params &p) {
    prefetch_tmap(&p.wd); prefetch_tmap(&p.sd);
    prefetch_token_maps8(p.th);
  }
  static __device__ __forceinline__ void stage_aux(const Params &p, uint8_t *aux) { stage_group_table(p.gt, aux); }
  static __device__ __forceinline__ int num_units(const Params &p, const uint8_t *aux) {
    return grouped_num_units(p.gt, aux);
  }
  static __device__ __forceinline__ int k_blocks(const Params &p) { return p.F / 128; }
  static __device__ __forceinline__ Unit unit(const Params &p, int u, const uint8_t *aux) {
    return grouped_unit(p.gt, aux, u, kF8Tile);
  }
  static __device__ __forceinline__ uint32_t a_bytes(const Unit &U) { return token_rows16(U.nv) * 128; }
  static __device__ __forceinline__ void load_a(const Params &p, const Unit &U, int kb, uint32_t sa, uint32_t bar) {
    load_token_rows8(p.th, kb, U.row0, token_rows16(U.nv), sa, bar);
  }
  static __device__ __forceinline__ void load_b(const Params &p, const Unit &U, int kb, uint32_t sb, uint32_t bar) {
    const bool sh = U.g == p.gt.E;
    tma_load_2d(sb, sh ? &p.sd : &p.wd, bar, kb * 128, (sh ? 0 : U.g * p.L) + U.m * 128);
  }
  static __device__ __forceinline__ int scale_class(int) { return 0; }
  static __device__ __forceinline__ void stage_scales(const Params &p, const Unit &U, float *tok, float *w,
                                                      float *extra, int lane) {
    const bool sh = U.g == p.gt.E;
    const int kbs = p.F / 128;
    const size_t blk = (static_cast<size_t>(sh ? 0 : U.g) * (p.L / 128) + U.m) * kbs;
    stage_token_scales(p.hs_t, p.rows, U.row0, U.nv, kbs, tok, lane);
    stage_weight_scales((sh ? p.sd_s : p.wd_s) + blk, nullptr, kbs, w, lane);
    stage_slots(p, U, extra, lane);
  }
  // [128] slot row, then [128] weight; the loads go out in two batches (all
  // permutation entries, then all weights) rather than as four dependent pairs
  static __device__ __forceinline__ void stage_slots(const Params &p, const Unit &U, float *extra, int lane) {
    const bool sh = U.g == p.gt.E;
    int *slot = reinterpret_cast<int *>(extra);
    constexpr int C = kF8Tile / 32;
    int flat[C];
#pragma unroll
    for (int c = 0; c < C; ++c) {
      const int n = c * 32 + lane;
      flat[c] = (!sh && n < U.nv) ? __ldg(p.perm + U.row0 + n) : 0;
    }
    float wv[C];
#pragma unroll
    for (int c = 0; c < C; ++c) wv[c] = (!sh && c * 32 + lane < U.nv) ? __ldg(p.wscaled + flat[c]) : 1.0f;
#pragma unroll
    for (int c = 0; c < C; ++c) {
      const int n = c * 32 + lane;
      if (n < U.nv) {
        if (sh) {
          slot[n] = (U.row0 + n - p.Tk) * (p.k + 1) + p.k;
        } else {
          const int tk = flat[c] / p.k;
          slot[n] = tk * (p.k + 1) + (flat[c] - tk * p.k);
        }
        extra[kF8Tile + n] = wv[c];
      }
    }
  }
  static __device__ __forceinline__ void epilogue_regs(const Params &p, const Unit &U, float (&acc)[kF8Half], int q,
                                                       int h, int lane, uint8_t *epi, const float *extra) {
    const int *slot = reinterpret_cast<const int *>(extra);
    const float *wt = extra + kF8Tile;
    float *wrow = reinterpret_cast<float *>(epi) + (h * 4 + q) * 32 * 33;  // this warp's rows: [32 tokens][33]
    const float my_wt = q * 32 + lane < U.nv ? wt[q * 32 + lane] : 0.f;
    const int part = lane & 7;  // 16-byte eighth of a token's 128 bytes
#pragma unroll
    for (int half = 0; half < 2; ++half) {
#pragma unroll
      for (int i = 0; i < 32; ++i) wrow[lane * 33 + i] = acc[half * 32 + i] * my_wt;
      __syncwarp();
#pragma unroll
      for (int it = 0; it < 8; ++it) {
        const int i = it * 4 + (lane >> 3);  // token within the warp
        const int t = q * 32 + i;
        if (t < U.nv) {
          const float *src = wrow + i * 33 + part * 4;
          *reinterpret_cast<float4 *>(p.slots + static_cast<size_t>(slot[t]) * p.L + U.m * 128 + h * kF8Half +
                                      half * 32 + part * 4) = make_float4(src[0], src[1], src[2], src[3]);
        }
      }
      __syncwarp();
    }
  }
};

// FP4 expert weights: Glu8Policy / Down8Policy with each weight matrix given as
// packed e2m1 codes [rows, K / 2] (maps with 64-byte boxes, no swizzle) and
// token tiles of at most 64 rows, so that a K block's packed weight tile
// (8 KB) fits in the upper half of the stage's token slot; the promotion
// warps expand it into the stage's e4m3 B tile (expand_fp4_tile).  Scales,
// promotion and epilogues are the FP8 policies'.
constexpr int kF4TokTile = 64;

struct Glu4Policy : Glu8Policy {
  static constexpr bool kFp4B = true;
  static __device__ __forceinline__ uint32_t b_bytes() { return kF8OpBytes / 2; }
  static __device__ __forceinline__ Unit unit(const Params &p, int u, const uint8_t *aux) {
    return grouped_unit(p.gt, aux, u, kF4TokTile);
  }
  static __device__ __forceinline__ void load_b(const Params &p, const Unit &U, int kb, uint32_t sb, uint32_t bar) {
    const bool sh = U.g == p.gt.E;
    const int row = (sh ? 0 : U.g * p.F) + U.m * 64;
    tma_load_2d(sb, sh ? &p.sg : &p.wg, bar, kb * 64, row);            // 64 gate rows x 64 B
    tma_load_2d(sb + 64 * 64, sh ? &p.su : &p.wu, bar, kb * 64, row);  // then the 64 up rows
  }
};

struct Down4Policy : Down8Policy {
  static constexpr bool kFp4B = true;
  static __device__ __forceinline__ uint32_t b_bytes() { return kF8OpBytes / 2; }
  static __device__ __forceinline__ Unit unit(const Params &p, int u, const uint8_t *aux) {
    return grouped_unit(p.gt, aux, u, kF4TokTile);
  }
  static __device__ __forceinline__ void load_b(const Params &p, const Unit &U, int kb, uint32_t sb, uint32_t bar) {
    const bool sh = U.g == p.gt.E;
    tma_load_2d(sb, sh ? &p.sd : &p.wd, bar, kb * 64, (sh ? 0 : U.g * p.L) + U.m * 128);  // 128 rows x 64 B
  }
};

}  // namespace mrl
