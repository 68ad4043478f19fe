// gemm2_sm100.cuh — CTA-pair (cta_group::2) persistent tcgen05 GEMM for the
// grouped expert GEMMs.
//
// Two CTAs of a cluster form one M = 256 UMMA: each holds 128 rows of A (its
// own expert-weight rows) and half of the unit's N token rows in its shared
// memory; the even CTA issues tcgen05.mma.cta_group::2 for both, and each CTA
// receives its 128 rows of the accumulator in its own TMEM.  The token tile is
// therefore read from L2 once per pair instead of once per CTA.
//
// Synchronisation (all waits bounded, as in gemm_sm100.cuh):
//  - both CTAs' TMA loads (cta_group::2 form, no multicast) complete on the
//    even CTA's full barriers; the even CTA's two producers set the expected
//    bytes of both halves;
//  - one commit of the even CTA per group of stages, and one per tile, arrive
//    on the release / accumulator-full barriers of both CTAs (tcgen05.commit
//    multicast);
//  - each CTA's epilogue warps arrive on the even CTA's accumulator-empty
//    barrier (count 8) once they have drained their TMEM rows.
#pragma once
#include "gemm_sm100.cuh"
#include "policies.cuh"

namespace mrl {

template <class P>
struct Gemm2Smem {
  static_assert(P::kStages % P::kGroup == 0, "ring depth must be a multiple of the release group");
  static constexpr int kStageBytes = P::kABytes + P::kBBytesMax;
  static constexpr int kRing = P::kStages * kStageBytes;
  static constexpr int kBarOff = kRing;
  static constexpr int kNumBars = P::kStages + P::kStages / P::kGroup + 4;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kEpiOff = (kMiscOff + 16 + 127) & ~127;
  static constexpr int kAuxOff = (kEpiOff + P::kEpiSmem + 127) & ~127;
  static constexpr int kTotal = kAuxOff + P::kAuxSmem + 1024;
};

template <class P>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    gemm2_kernel(const __grid_constant__ typename P::Params p) {
  using L = Gemm2Smem<P>;
  constexpr int S = P::kStages, G = P::kGroup;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kBarOff);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMiscOff);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMiscOff + 4);
  volatile int *entry = reinterpret_cast<volatile int *>(smem + L::kMiscOff + 8);  // [0] skip, [1] hold
  uint8_t *epi_smem = smem + L::kEpiOff;
  uint8_t *aux = smem + L::kAuxOff;

  const uint32_t full0 = smem_u32(bars);   // used in the even CTA only
  const uint32_t empty0 = full0 + 8 * S;   // one per group of G stages, in both CTAs
  const uint32_t accf0 = empty0 + 8 * (S / G);
  const uint32_t acce0 = accf0 + 16;
  const uint32_t ring = smem_u32(smem);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cid = static_cast<int>(cluster_id_x());
  const int ncl = static_cast<int>(nclusters_x());
  uint32_t *status = p.status;

  if (threadIdx.x == 0) {
    // only the even CTA reads the call header; both CTAs act on its reading
    const uint2 hdr = leader ? call_header(status) : make_uint2(0u, 0u);
    for (int s = 0; s < S; ++s) mbar_init(full0 + 8 * s, 2);
    for (int g = 0; g < S / G; ++g) mbar_init(empty0 + 8 * g, 1);
    for (int a = 0; a < 2; ++a) {
      mbar_init(accf0 + 8 * a, 1);
      mbar_init(acce0 + 8 * a, 8);
    }
    *abort_flag = 0;
    entry[0] = hdr.x != DEV_OK;
    entry[1] = (hdr.y & HOLD_GEMM_PAIR) != 0;
    fence_mbar_init();
  }
  P::stage_aux(p, aux);
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // barrier initialisation visible to the peer before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int nunits = P::num_units(p, aux);
  const int kblocks = P::k_blocks(p);
  // the even CTA's entry words, read after the cluster barrier that published them
  const uint32_t entry_l = mapa_shared(smem_u32(const_cast<int *>(entry)), 0);
  if (ld_shared_cluster_u32(entry_l)) goto done;  // an earlier kernel of the call failed

  if (warp == 0 || warp == 6) {
    // loads held (test mask): nothing is issued in either CTA, so the bounded waits run out
    if (lane == 0 && !ld_shared_cluster_u32(entry_l + 4)) {
      const bool isA = warp == 0;
      P::prefetch(p);
      int s = 0;
      uint32_t ph = 0;
      for (int u = cid; u < nunits; u += ncl) {
        const Unit U = P::unit(p, u, aux);
        const uint32_t pair_bytes = isA ? 2u * P::kABytes : P::b_bytes_pair(p, U);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (s % G == 0 && !mbar_wait(empty0 + 8 * (s / G), ph ^ 1, abort_flag, status)) goto done;
          const uint32_t full_local = full0 + 8 * s;
          if (leader) mbar_arrive_expect_tx(full_local, pair_bytes);
          const uint32_t full_cl = mapa_shared(full_local, 0);
          const uint32_t st = ring + s * L::kStageBytes;
          if (isA)
            P::load_a(p, U, kb, st, full_cl, rank);
          else
            P::load_b(p, U, kb, st + P::kABytes, full_cl, rank);
          if (++s == S) { s = 0; ph ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      int s = 0, acc = 0;
      uint32_t ph = 0, aph = 0;
      for (int u = cid; u < nunits; u += ncl) {
        const Unit U = P::unit(p, u, aux);
        if (!mbar_wait(acce0 + 8 * acc, aph ^ 1, abort_flag, status)) goto done;
        tc_fence_after();
        const uint32_t tacc = tmem_base + acc * kAccCols;
        const uint32_t idesc = P::idesc(p, U);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(full0 + 8 * s, ph, abort_flag, status)) goto done;
          tc_fence_after();
          const uint32_t a_s = ring + s * L::kStageBytes;
          const uint32_t b_s = a_s + P::kABytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_f16_pair(tacc, operand_desc<OperandMajor<P>::a_mn, OperandMajor<P>::a_stride, 32>(a_s, kk),
                          operand_desc<OperandMajor<P>::b_mn, OperandMajor<P>::b_stride, 32>(b_s, kk), idesc,
                          (kb | kk) != 0);
          if (s % G == G - 1) umma_commit_pair(empty0 + 8 * (s / G), 0x3);
          if (++s == S) { s = 0; ph ^= 1; }
        }
        umma_commit_pair(accf0 + 8 * acc, 0x3);
        acc ^= 1;
        if (acc == 0) aph ^= 1;
      }
    }
  } else {
    const int q = warp & 3;
    const int etid = threadIdx.x - 64;
    int acc = 0;
    uint32_t aph = 0;
    for (int u = cid; u < nunits; u += ncl) {
      const Unit U = P::unit(p, u, aux);
      const bool ok = mbar_wait(accf0 + 8 * acc, aph, abort_flag, status);
      if (bar_red_or(1, 128, !ok || *abort_flag)) goto done;
      tc_fence_after();
      P::epilogue(p, U, tmem_base + acc * kAccCols + (static_cast<uint32_t>(q * 32) << 16), q, lane, etid, rank,
                  epi_smem);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader)
          mbar_arrive(acce0 + 8 * acc);
        else
          mbar_arrive_remote(mapa_shared(acce0 + 8 * acc, 0));
      }
      acc ^= 1;
      if (acc == 0) aph ^= 1;
    }
  }
done:
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no CTA leaves while its peer may still signal its barriers
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

// --------------------------------------------------------------- policies
__device__ __forceinline__ int round32(int n) { return (n + 31) & ~31; }

// B half of CTA `rank`: rows row0 + rank*N/2 .. + N/2 (N = MMA N, a multiple
// of 32, so N/2 is a multiple of 16), as 64/32/16-row boxes.
__device__ __forceinline__ void load_rows_half(const TokenMaps &t, const Unit &U, int kb, uint32_t sb,
                                               uint32_t bar_cl, uint32_t rank) {
  const int half = round32(U.nv) >> 1;
  load_token_rows<true>(t, kb, U.row0 + static_cast<int>(rank) * half, half, sb, bar_cl);
}

// gate/up over a CTA pair: unit = (group, 128-wide d_ff slice, <= 256 tokens);
// CTA r owns d_ff columns f0 = m*128 + r*64 .. +63: its A tile is 64 gate
// rows (TMEM lanes 0-63) then the 64 matching up rows (lanes 64-127), two
// 64-row TMA boxes per K block (a 64-row box streams at full HBM rate; 16-row
// boxes did not).  In the epilogue, warp pair (q, q+2) swaps half of each
// 32-token chunk through shared memory so each warp owns complete (gate, up)
// pairs for 16 of the chunk's tokens.
struct Glu2Policy {
  static constexpr int kStages = 6;
  static constexpr int kGroup = 2;
  static constexpr int kBN = 256;
  static constexpr int kABytes = 128 * 128;
  static constexpr int kBBytesMax = (kBN / 2) * 128;
  static constexpr int kEpiSmem = 4 * 32 * 17 * 4;
  static constexpr int kAuxSmem = kGroupAuxSmem;
  using Params = GluParams;
  static __device__ __forceinline__ void prefetch(const Params &p) { prefetch_glu(p); }
  static __device__ __forceinline__ void stage_aux(const Params &p, uint8_t *aux) { stage_group_table(p.gt, aux); }
  static __device__ __forceinline__ int num_units(const Params &p, const uint8_t *aux) {
    return grouped_num_units(p.gt, aux);
  }
  static __device__ __forceinline__ int k_blocks(const Params &p) { return p.L / kBK; }
  static __device__ __forceinline__ Unit unit(const Params &p, int u, const uint8_t *aux) {
    return grouped_unit(p.gt, aux, u, kBN);
  }
  static __device__ __forceinline__ uint32_t b_bytes_pair(const Params &, const Unit &U) {
    return round32(U.nv) * 128;
  }
  static __device__ __forceinline__ void load_a(const Params &p, const Unit &U, int kb, uint32_t sa,
                                                uint32_t bar_cl, uint32_t rank) {
    const bool sh = U.g == p.gt.E;
    const int row = (sh ? 0 : U.g * p.F) + U.m * 128 + static_cast<int>(rank) * 64;
    tma_load_2d_pair(sa, sh ? &p.sg : &p.wg, bar_cl, kb * kBK, row);
    tma_load_2d_pair(sa + 64 * 128, sh ? &p.su : &p.wu, bar_cl, kb * kBK, row);
  }
  static __device__ __forceinline__ void load_b(const Params &p, const Unit &U, int kb, uint32_t sb,
                                                uint32_t bar_cl, uint32_t rank) {
    load_rows_half(p.tz, U, kb, sb, bar_cl, rank);
  }
  static __device__ __forceinline__ uint32_t idesc(const Params &, const Unit &U) {
    return idesc_bf16(256, round32(U.nv));
  }
  static __device__ __forceinline__ void epilogue(const Params &p, const Unit &U, uint32_t taddr, int q, int lane,
                                                  int etid, uint32_t rank, uint8_t *epi) {
    float *xb = reinterpret_cast<float *>(epi);  // [4][32][17]
    const bool is_gate = q < 2;
    const int pair = q & 1;
    // h is K-blocked: the CTA's 64 d_ff columns are one plane, so the unit's
    // rows land in one contiguous N x 128 B range of it
    const int plane = U.m * 2 + static_cast<int>(rank);
    const size_t hoff = static_cast<size_t>(plane) * p.rows * 64 + pair * 32 + lane;
    __nv_bfloat16 *hp = p.h + hoff;
    const size_t row0 = static_cast<size_t>(U.row0);
    for (int c0 = 0; c0 < U.nv; c0 += 32) {
      float v[32];
      tmem_ld32(taddr + c0, v);
      tmem_ld_wait();
      float *mine = xb + (q * 32 + lane) * 17;
#pragma unroll
      for (int c = 0; c < 16; ++c) mine[c] = is_gate ? v[16 + c] : v[c];
      named_bar_sync(2, 128);
      const float *other = xb + (((q + 2) & 3) * 32 + lane) * 17;
      const int cbase = c0 + (is_gate ? 0 : 16);
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const float g = is_gate ? v[c] : other[c];
        const float u = is_gate ? other[c] : v[16 + c];
        if (cbase + c < U.nv) {
          const size_t o = (row0 + cbase + c) * 64;
          hp[o] = __float2bfloat16_rn(__fdividef(g, 1.0f + __expf(-g)) * u);
          if (p.gu) p.gu[hoff + o] = pack_bf16x2(g, u);
        }
      }
      named_bar_sync(2, 128);
    }
  }
};

// expert down over a CTA pair: unit = (group, 256-wide d_lat slice, <= 256
// tokens); CTA r owns output rows l = m*256 + r*128 .. +127.
struct Down2Policy {
  static constexpr int kStages = 6;
  static constexpr int kGroup = 2;
  static constexpr int kBN = 256;
  static constexpr int kABytes = 128 * 128;
  static constexpr int kBBytesMax = (kBN / 2) * 128;
  static constexpr int kEpiSmem = DownPolicy::kEpiSmem;
  static constexpr int kAuxSmem = kGroupAuxSmem;
  using Params = DownPolicy::Params;
  static __device__ __forceinline__ void prefetch(const Params &p) { DownPolicy::prefetch(p); }
  static __device__ __forceinline__ void stage_aux(const Params &p, uint8_t *aux) { stage_group_table(p.gt, aux); }
  static __device__ __forceinline__ int num_units(const Params &p, const uint8_t *aux) {
    return grouped_num_units(p.gt, aux);
  }
  static __device__ __forceinline__ int k_blocks(const Params &p) { return p.F / kBK; }
  static __device__ __forceinline__ Unit unit(const Params &p, int u, const uint8_t *aux) {
    return grouped_unit(p.gt, aux, u, kBN);
  }
  static __device__ __forceinline__ uint32_t b_bytes_pair(const Params &, const Unit &U) {
    return round32(U.nv) * 128;
  }
  static __device__ __forceinline__ void load_a(const Params &p, const Unit &U, int kb, uint32_t sa,
                                                uint32_t bar_cl, uint32_t rank) {
    const bool sh = U.g == p.gt.E;
    tma_load_2d_pair(sa, sh ? &p.sd : &p.wd, bar_cl, kb * kBK,
                     (sh ? 0 : U.g * p.L) + U.m * 256 + static_cast<int>(rank) * 128);
  }
  static __device__ __forceinline__ void load_b(const Params &p, const Unit &U, int kb, uint32_t sb,
                                                uint32_t bar_cl, uint32_t rank) {
    load_rows_half(p.th, U, kb, sb, bar_cl, rank);
  }
  static __device__ __forceinline__ uint32_t idesc(const Params &, const Unit &U) {
    return idesc_bf16(256, round32(U.nv));
  }
  static __device__ __forceinline__ void epilogue(const Params &p, const Unit &U, uint32_t taddr, int q, int lane,
                                                  int etid, uint32_t rank, uint8_t *epi) {
    Unit V = U;
    V.m = U.m * 2 + static_cast<int>(rank);  // the CTA's 128-wide d_lat slice
    DownPolicy::EpiState st;
    DownPolicy::epilogue(p, V, 0, taddr, q, lane, etid, st, epi);
  }
};

// Dense bf16 projection over a CTA pair: out[M, N] = bf16(a[M, K] w[N, K]^T)
// (and optionally the residual of that rounding), unit = (256-row M tile,
// 256-column N tile).  CTA r loads A rows m*256 + r*128 (its 128 token rows)
// and the 128 weight rows n0 + r*nv/2 ..; the pair's MMA (M = 256, N = nv)
// leaves CTA r the accumulator of its 128 token rows x all nv columns.  Per
// 64-deep K block a CTA stages 32 KB for 2*128*256*64 FLOPs instead of the
// one-CTA 128 x 256 tile's 48 KB, so a stage crosses from L2 in two thirds
// of the time.  A 128-row weight box is loaded even when nv = 128 (N not a
// multiple of 256): the MMA then reads only its first 64 rows in each CTA.
struct Dense2Policy {
  static constexpr int kStages = 6;
  static constexpr int kGroup = 2;
  static constexpr int kBN = 256;
  static constexpr int kABytes = 128 * 128;
  static constexpr int kBBytesMax = (kBN / 2) * 128;
  static constexpr int kEpiSmem = 0;
  static constexpr int kAuxSmem = 0;
  using Params = DensePolicy::Params;  // m_tiles counts 256-row tiles here
  static __device__ __forceinline__ void prefetch(const Params &p) {
    prefetch_tmap(&p.ta);
    prefetch_tmap(&p.tb);
  }
  static __device__ __forceinline__ void stage_aux(const Params &, uint8_t *) {}
  static __device__ __forceinline__ int num_units(const Params &p, const uint8_t *) { return p.m_tiles * p.n_tiles; }
  static __device__ __forceinline__ int k_blocks(const Params &p) { return p.K / kBK; }
  static __device__ __forceinline__ Unit unit(const Params &p, int u, const uint8_t *) {
    Unit U;
    U.g = 0;
    U.row0 = 0;
    U.m = u / p.n_tiles;
    U.n0 = (u % p.n_tiles) * kBN;
    U.nv = min(kBN, p.N - U.n0);
    U.nsub = 1;
    return U;
  }
  static __device__ __forceinline__ uint32_t b_bytes_pair(const Params &, const Unit &) { return 2u * kBBytesMax; }
  static __device__ __forceinline__ void load_a(const Params &p, const Unit &U, int kb, uint32_t sa, uint32_t bar_cl,
                                                uint32_t rank) {
    tma_load_2d_pair(sa, &p.ta, bar_cl, kb * kBK, U.m * 256 + static_cast<int>(rank) * 128);
  }
  static __device__ __forceinline__ void load_b(const Params &p, const Unit &U, int kb, uint32_t sb, uint32_t bar_cl,
                                                uint32_t rank) {
    tma_load_2d_pair(sb, &p.tb, bar_cl, kb * kBK, U.n0 + static_cast<int>(rank) * (U.nv >> 1));
  }
  static __device__ __forceinline__ uint32_t idesc(const Params &, const Unit &U) { return idesc_bf16(256, U.nv); }
  static __device__ __forceinline__ void epilogue(const Params &p, const Unit &U, uint32_t taddr, int q, int lane, int,
                                                  uint32_t rank, uint8_t *) {
    Unit V = U;
    V.m = U.m * 2 + static_cast<int>(rank);  // the CTA's 128-row M tile
    DensePolicy::EpiState st;
    DensePolicy::epilogue(p, V, 0, taddr, q, lane, 0, st, nullptr);
  }
};

}  // namespace mrl
