// gemm8_sm100.cuh — e4m3 x e4m3 tcgen05 GEMM with fp32 block scales (the FP8
// variant of the layer).
//
// Operands carry one fp32 scale per 128-wide K block: the activation (token)
// side per row, the weight side per 128 x 128 block.  Such scales are not
// powers of two, so the tensor core's block-scaled modes cannot apply them:
// each 128-wide K block is accumulated on its own in TMEM (four 32-deep
// kind::f8f6f4 MMAs into one of four partial buffers), and the four epilogue
// warps promote it into an fp32 register accumulator,
//     acc[m][n] += partial[m][n] * row_scale(m, kb) * col_scale(n, kb),
// before releasing the partial buffer to the MMA issuer.  After the last K
// block the same warps run the policy's epilogue on the registers.
//
//   warp 0   : TMA producer for A        warp 6 : TMA producer for B
//   warp 1   : TMEM allocator + MMA issuer
//   warps 2-5: promotion + epilogue (TMEM lanes 32*(warp%4) .. +31)
//
// Stage j of the 4-deep shared-memory ring and partial buffer j serve global
// K block g with j = g % 4; the commit after block g's MMAs both frees stage j
// for the producers and hands partial j to the promotion warps.  All waits are
// bounded (mbar_wait).  No TMA load uses multicast.
#pragma once
#include "gemm_sm100.cuh"
#include "policies.cuh"

namespace mrl {

constexpr int kF8Ring = 4;      // stages == TMEM partial buffers
constexpr int kF8MaxN = 128;    // columns per unit (register accumulator size)
constexpr int kF8MaxKB = 32;    // K blocks of 128 per unit (K <= 4096)

template <class P>
struct Gemm8Smem {
  static constexpr int kStageBytes = P::kABytes + P::kBBytesMax;
  static constexpr int kRing = kF8Ring * kStageBytes;
  static constexpr int kBarOff = kRing;
  static constexpr int kNumBars = 3 * kF8Ring;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kColOff = (kMiscOff + 16 + 127) & ~127;
  static constexpr int kEpiOff = kColOff + kF8MaxKB * kF8MaxN * 4;
  static constexpr int kAuxOff = (kEpiOff + P::kEpiSmem + 127) & ~127;
  static constexpr int kTotal = kAuxOff + P::kAuxSmem + 1024;
};

template <class P>
__global__ void __launch_bounds__(kGemmThreads, 1) gemm8_kernel(const __grid_constant__ typename P::Params p) {
  using L = Gemm8Smem<P>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kBarOff);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMiscOff);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMiscOff + 4);
  float *col_scale = reinterpret_cast<float *>(smem + L::kColOff);  // [kb][n]
  uint8_t *epi_smem = smem + L::kEpiOff;
  uint8_t *aux = smem + L::kAuxOff;

  const uint32_t full0 = smem_u32(bars);
  const uint32_t done0 = full0 + 8 * kF8Ring;   // MMAs of the K block completed
  const uint32_t free0 = done0 + 8 * kF8Ring;   // partial buffer promoted
  const uint32_t ring = smem_u32(smem);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  uint32_t *status = p.status;

  if (threadIdx.x == 0) {
    for (int j = 0; j < kF8Ring; ++j) {
      mbar_init(full0 + 8 * j, 2);
      mbar_init(done0 + 8 * j, 1);
      mbar_init(free0 + 8 * j, 4);
    }
    *abort_flag = 0;
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

  if (warp == 0 || warp == 6) {
    if (lane == 0) {
      const bool isA = warp == 0;
      P::prefetch(p);
      uint32_t g = 0;
      for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
        const Unit U = P::unit(p, u, aux);
        const uint32_t bytes = isA ? P::kABytes : P::b_bytes(p, U, 0);
        for (int kb = 0; kb < kblocks; ++kb, ++g) {
          const uint32_t j = g & (kF8Ring - 1);
          if (g >= kF8Ring && !mbar_wait(done0 + 8 * j, ((g / kF8Ring) - 1) & 1, abort_flag, status)) goto done;
          mbar_arrive_expect_tx(full0 + 8 * j, bytes);
          const uint32_t st = ring + j * L::kStageBytes;
          if (isA)
            P::load_a(p, U, 0, kb, st, full0 + 8 * j);
          else
            P::load_b(p, U, 0, kb, st + P::kABytes, full0 + 8 * j);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      uint32_t g = 0;
      for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
        const Unit U = P::unit(p, u, aux);
        const uint32_t idesc = P::idesc(p, U, 0);
        for (int kb = 0; kb < kblocks; ++kb, ++g) {
          const uint32_t j = g & (kF8Ring - 1);
          if (!mbar_wait(full0 + 8 * j, (g / kF8Ring) & 1, abort_flag, status)) goto done;
          if (g >= kF8Ring && !mbar_wait(free0 + 8 * j, ((g / kF8Ring) - 1) & 1, abort_flag, status)) goto done;
          tc_fence_after();
          const uint32_t a_s = ring + j * L::kStageBytes;
          const uint32_t b_s = a_s + P::kABytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_f8(tmem_base + j * kF8MaxN, sdesc_sw128(a_s + kk * 32), sdesc_sw128(b_s + kk * 32), idesc, kk != 0);
          umma_commit(done0 + 8 * j);
        }
      }
    }
  } else {
    const int q = warp & 3;
    const int etid = threadIdx.x - 64;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    uint32_t g = 0;
    for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
      const Unit U = P::unit(p, u, aux);
      named_bar_sync(2, 128);  // the previous unit's readers of col_scale are done
      P::stage_col_scales(p, U, col_scale, etid);
      named_bar_sync(2, 128);
      float acc[kF8MaxN];
#pragma unroll
      for (int i = 0; i < kF8MaxN; ++i) acc[i] = 0.f;
      for (int kb = 0; kb < kblocks; ++kb, ++g) {
        const uint32_t j = g & (kF8Ring - 1);
        const bool ok = mbar_wait(done0 + 8 * j, (g / kF8Ring) & 1, abort_flag, status);
        if (bar_red_or(1, 128, !ok || *abort_flag)) goto done;
        tc_fence_after();
        const float rs = P::row_scale(p, U, kb, q, lane);
        const float *cs = col_scale + kb * kF8MaxN;
#pragma unroll
        for (int c = 0; c < kF8MaxN / 32; ++c) {
          if (c * 32 < U.nv) {
            float v[32];
            tmem_ld32(tmem_base + j * kF8MaxN + lane_off + c * 32, v);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) acc[c * 32 + i] = fmaf(v[i], rs * cs[c * 32 + i], acc[c * 32 + i]);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(free0 + 8 * j);
      }
      P::epilogue_regs(p, U, acc, q, lane, etid, epi_smem);
    }
  }
done:
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ------------------------------------------------------------- FP8 policies
// Scale tables: an activation tensor [rows, K] has fp32 scales [rows, K/128];
// a weight matrix [out, in] has [out/128, in/128] (routed experts: [E, ...]).

// Projection out = bf16(a w^T): tokens on M (TMEM lanes), weights on N.
struct Dense8Policy {
  static constexpr int kABytes = 128 * 128;
  static constexpr int kBBytesMax = kF8MaxN * 128;
  static constexpr int kEpiSmem = 0;
  static constexpr int kAuxSmem = 0;
  struct Params {
    CUtensorMap ta;  // a codes [M, K], box 128 x 128
    CUtensorMap tb;  // w codes [N, K], box 128 x 128
    const float *as, *ws;  // [M, K/128], [N/128, K/128]
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
    U.row0 = 0;
    U.m = u / p.n_tiles;
    U.n0 = (u % p.n_tiles) * kF8MaxN;
    U.nv = min(kF8MaxN, p.N - U.n0);
    U.nsub = 1;
    return U;
  }
  static __device__ __forceinline__ uint32_t b_bytes(const Params &, const Unit &, int) { return kBBytesMax; }
  static __device__ __forceinline__ void load_a(const Params &p, const Unit &U, int, int kb, uint32_t sa,
                                                uint32_t bar) {
    tma_load_2d(sa, &p.ta, bar, kb * 128, U.m * 128);
  }
  static __device__ __forceinline__ void load_b(const Params &p, const Unit &U, int, int kb, uint32_t sb,
                                                uint32_t bar) {
    tma_load_2d(sb, &p.tb, bar, kb * 128, U.n0);
  }
  static __device__ __forceinline__ uint32_t idesc(const Params &, const Unit &U, int) {
    return idesc_e4m3(128, round16(U.nv));
  }
  static __device__ __forceinline__ void stage_col_scales(const Params &p, const Unit &U, float *cs, int etid) {
    const int kbs = p.K / 128;
    for (int i = etid; i < kbs * kF8MaxN; i += 128) {
      const int kb = i / kF8MaxN;
      cs[i] = __ldg(p.ws + static_cast<size_t>(U.n0 / 128) * kbs + kb);
    }
  }
  static __device__ __forceinline__ float row_scale(const Params &p, const Unit &U, int kb, int q, int lane) {
    const int row = U.m * 128 + q * 32 + lane;
    return row < p.M ? __ldg(p.as + static_cast<size_t>(row) * (p.K / 128) + kb) : 0.f;
  }
  static __device__ __forceinline__ void epilogue_regs(const Params &p, const Unit &U, float (&acc)[kF8MaxN], int q,
                                                       int lane, int, uint8_t *) {
    const int row = U.m * 128 + q * 32 + lane;
    if (row >= p.M) return;
#pragma unroll
    for (int c = 0; c < kF8MaxN / 32; ++c) {
      if (c * 32 < U.nv) {
        uint4 *dst = reinterpret_cast<uint4 *>(p.out + row * p.ldo + U.n0 + c * 32);
        uint4 *dlo = p.out_lo ? reinterpret_cast<uint4 *>(p.out_lo + row * p.ldo + U.n0 + c * 32) : nullptr;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float *v = acc + c * 32 + 8 * i;
          uint4 w;
          w.x = pack_bf16x2(v[0], v[1]);
          w.y = pack_bf16x2(v[2], v[3]);
          w.z = pack_bf16x2(v[4], v[5]);
          w.w = pack_bf16x2(v[6], v[7]);
          dst[i] = w;
          if (dlo) {
            float r[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) r[t] = v[t] - __bfloat162float(__float2bfloat16_rn(v[t]));
            uint4 l;
            l.x = pack_bf16x2(r[0], r[1]);
            l.y = pack_bf16x2(r[2], r[3]);
            l.z = pack_bf16x2(r[4], r[5]);
            l.w = pack_bf16x2(r[6], r[7]);
            dlo[i] = l;
          }
        }
      }
    }
  }
};

// B operand for the grouped FP8 GEMMs: the unit's quantised rows as 32-row boxes.
__device__ __forceinline__ void load_rows8(const CUtensorMap *tm, const Unit &U, int kb, uint32_t sb, uint32_t bar) {
  const int nb = (U.nv + 31) >> 5;
  for (int i = 0; i < nb; ++i) tma_load_2d(sb + i * 4096, tm, bar, kb * 128, U.row0 + 32 * i);
}

// gate/up: unit = (group, 64-wide d_ff slice, <= 128 tokens); A = 64 gate rows
// then the 64 matching up rows; h = bf16(SiLU(g) * u) in bf16 (quantised for
// the down GEMM by a separate pass).
struct Glu8Policy {
  static constexpr int kABytes = 128 * 128;
  static constexpr int kBBytesMax = kF8MaxN * 128;
  static constexpr int kEpiSmem = 4 * 32 * 17 * 4;
  static constexpr int kAuxSmem = kGroupAuxSmem;
  struct Params {
    CUtensorMap wg, wu, sg, su;  // e4m3 [E*F, L] / [F, L], box 128 x 64
    CUtensorMap tz;              // quantised dispatched z [(T*k+T), L], box 128 x 32
    const float *wg_s, *wu_s, *sg_s, *su_s;  // [E, F/128, L/128] / [F/128, L/128]
    const float *zs;                          // [(T*k+T), L/128]
    GroupTable gt;
    __nv_bfloat16 *h;
    int F, L;
    uint32_t *status;
  };
  static __device__ __forceinline__ void prefetch(const Params &p) {
    prefetch_tmap(&p.wg); prefetch_tmap(&p.wu); prefetch_tmap(&p.sg); prefetch_tmap(&p.su); prefetch_tmap(&p.tz);
  }
  static __device__ __forceinline__ void stage_aux(const Params &p, uint8_t *aux) { stage_group_table(p.gt, aux); }
  static __device__ __forceinline__ int num_units(const Params &p, const uint8_t *aux) {
    return grouped_num_units(p.gt, aux);
  }
  static __device__ __forceinline__ int k_blocks(const Params &p) { return p.L / 128; }
  static __device__ __forceinline__ Unit unit(const Params &p, int u, const uint8_t *aux) {
    return grouped_unit(p.gt, aux, u, kF8MaxN);
  }
  static __device__ __forceinline__ uint32_t b_bytes(const Params &, const Unit &U, int) {
    return ((U.nv + 31) >> 5) * 4096;
  }
  static __device__ __forceinline__ void load_a(const Params &p, const Unit &U, int, int kb, uint32_t sa,
                                                uint32_t bar) {
    const bool sh = U.g == p.gt.E;
    const int row = (sh ? 0 : U.g * p.F) + U.m * 64;
    tma_load_2d(sa, sh ? &p.sg : &p.wg, bar, kb * 128, row);
    tma_load_2d(sa + 64 * 128, sh ? &p.su : &p.wu, bar, kb * 128, row);
  }
  static __device__ __forceinline__ void load_b(const Params &p, const Unit &U, int, int kb, uint32_t sb,
                                                uint32_t bar) {
    load_rows8(&p.tz, U, kb, sb, bar);
  }
  static __device__ __forceinline__ uint32_t idesc(const Params &, const Unit &U, int) {
    return idesc_e4m3(128, round16(U.nv));
  }
  static __device__ __forceinline__ void stage_col_scales(const Params &p, const Unit &U, float *cs, int etid) {
    const int kbs = p.L / 128;
    for (int i = etid; i < kbs * U.nv; i += 128) {
      const int n = i / kbs, kb = i - n * kbs;
      cs[kb * kF8MaxN + n] = __ldg(p.zs + static_cast<size_t>(U.row0 + n) * kbs + kb);
    }
  }
  static __device__ __forceinline__ float row_scale(const Params &p, const Unit &U, int kb, int q, int) {
    const bool sh = U.g == p.gt.E;
    const int kbs = p.L / 128, fb = (U.m * 64) / 128;
    const float *tab = q < 2 ? (sh ? p.sg_s : p.wg_s) : (sh ? p.su_s : p.wu_s);
    const size_t blk = static_cast<size_t>(sh ? 0 : U.g) * (p.F / 128) + fb;
    return __ldg(tab + blk * kbs + kb);
  }
  // Lanes 0-63 hold gate rows, 64-127 the matching up rows: warp pair (q, q+2)
  // swaps half of each 32-token chunk through shared memory.
  static __device__ __forceinline__ void epilogue_regs(const Params &p, const Unit &U, float (&acc)[kF8MaxN], int q,
                                                       int lane, int, uint8_t *epi) {
    float *xb = reinterpret_cast<float *>(epi);  // [4][32][17]
    const bool is_gate = q < 2;
    const int f = U.m * 64 + (q & 1) * 32 + lane;
    const size_t row0 = static_cast<size_t>(U.row0);
#pragma unroll
    for (int c = 0; c < kF8MaxN / 32; ++c) {
      if (c * 32 < U.nv) {
        const float *v = acc + c * 32;
        float *mine = xb + (q * 32 + lane) * 17;
#pragma unroll
        for (int i = 0; i < 16; ++i) mine[i] = is_gate ? v[16 + i] : v[i];
        named_bar_sync(2, 128);
        const float *other = xb + (((q + 2) & 3) * 32 + lane) * 17;
        const int cbase = c * 32 + (is_gate ? 0 : 16);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float gv = is_gate ? v[i] : other[i];
          const float uv = is_gate ? other[i] : v[16 + i];
          if (cbase + i < U.nv)
            p.h[(row0 + cbase + i) * p.F + f] = __float2bfloat16_rn(__fdividef(gv, 1.0f + __expf(-gv)) * uv);
        }
        named_bar_sync(2, 128);
      }
    }
  }
};

// expert down: unit = (group, 128-wide d_lat slice, <= 128 tokens).
struct Down8Policy {
  static constexpr int kABytes = 128 * 128;
  static constexpr int kBBytesMax = kF8MaxN * 128;
  static constexpr int kEpiSmem = kF8MaxN * 8;
  static constexpr int kAuxSmem = kGroupAuxSmem;
  struct Params {
    CUtensorMap wd, sd;  // e4m3 [E*L, F] / [L, F], box 128 x 128
    CUtensorMap th;      // quantised h [(T*k+T), F], box 128 x 32
    const float *wd_s, *sd_s;  // [E, L/128, F/128] / [L/128, F/128]
    const float *hs;           // [(T*k+T), F/128]
    GroupTable gt;
    const int32_t *perm;
    const float *wscaled;
    float *slots;
    int L, F, k, Tk;
    uint32_t *status;
  };
  static __device__ __forceinline__ void prefetch(const Params &p) {
    prefetch_tmap(&p.wd); prefetch_tmap(&p.sd); prefetch_tmap(&p.th);
  }
  static __device__ __forceinline__ void stage_aux(const Params &p, uint8_t *aux) { stage_group_table(p.gt, aux); }
  static __device__ __forceinline__ int num_units(const Params &p, const uint8_t *aux) {
    return grouped_num_units(p.gt, aux);
  }
  static __device__ __forceinline__ int k_blocks(const Params &p) { return p.F / 128; }
  static __device__ __forceinline__ Unit unit(const Params &p, int u, const uint8_t *aux) {
    return grouped_unit(p.gt, aux, u, kF8MaxN);
  }
  static __device__ __forceinline__ uint32_t b_bytes(const Params &, const Unit &U, int) {
    return ((U.nv + 31) >> 5) * 4096;
  }
  static __device__ __forceinline__ void load_a(const Params &p, const Unit &U, int, int kb, uint32_t sa,
                                                uint32_t bar) {
    const bool sh = U.g == p.gt.E;
    tma_load_2d(sa, sh ? &p.sd : &p.wd, bar, kb * 128, (sh ? 0 : U.g * p.L) + U.m * 128);
  }
  static __device__ __forceinline__ void load_b(const Params &p, const Unit &U, int, int kb, uint32_t sb,
                                                uint32_t bar) {
    load_rows8(&p.th, U, kb, sb, bar);
  }
  static __device__ __forceinline__ uint32_t idesc(const Params &, const Unit &U, int) {
    return idesc_e4m3(128, round16(U.nv));
  }
  static __device__ __forceinline__ void stage_col_scales(const Params &p, const Unit &U, float *cs, int etid) {
    const int kbs = p.F / 128;
    for (int i = etid; i < kbs * U.nv; i += 128) {
      const int n = i / kbs, kb = i - n * kbs;
      cs[kb * kF8MaxN + n] = __ldg(p.hs + static_cast<size_t>(U.row0 + n) * kbs + kb);
    }
  }
  static __device__ __forceinline__ float row_scale(const Params &p, const Unit &U, int kb, int, int) {
    const bool sh = U.g == p.gt.E;
    const int kbs = p.F / 128;
    const size_t blk = static_cast<size_t>(sh ? 0 : U.g) * (p.L / 128) + U.m;
    return __ldg((sh ? p.sd_s : p.wd_s) + blk * kbs + kb);
  }
  static __device__ __forceinline__ void epilogue_regs(const Params &p, const Unit &U, float (&acc)[kF8MaxN], int q,
                                                       int lane, int etid, uint8_t *epi) {
    int *s_slot = reinterpret_cast<int *>(epi);
    float *s_wt = reinterpret_cast<float *>(epi + kF8MaxN * sizeof(int));
    const int l = U.m * 128 + q * 32 + lane;
    const bool sh = U.g == p.gt.E;
    for (int c = etid; c < U.nv; c += 128) {
      const int row = U.row0 + c;
      if (sh) {
        s_slot[c] = (row - p.Tk) * (p.k + 1) + p.k;
        s_wt[c] = 1.0f;
      } else {
        const int flat = __ldg(p.perm + row);
        const int t = flat / p.k;
        s_slot[c] = t * (p.k + 1) + (flat - t * p.k);
        s_wt[c] = __ldg(p.wscaled + flat);
      }
    }
    named_bar_sync(2, 128);
#pragma unroll
    for (int c = 0; c < kF8MaxN; ++c)
      if (c < U.nv) p.slots[static_cast<size_t>(s_slot[c]) * p.L + l] = acc[c] * s_wt[c];
    named_bar_sync(2, 128);
  }
};

}  // namespace mrl
