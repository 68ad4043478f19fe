// policies.cuh — the layer's GEMMs expressed as policies of gemm_kernel.
//
//  DensePolicyN : out[M,N] = bf16(a[M,K] w[N,K]^T)           (down-/up-projection)
//  RouterPolicy : per token tile, R sigmoid routers x all experts, fused with
//                 the aggregation over routers (mean / sum / max), + bias,
//                 running top-k, renormalisation, alpha
//  GluParams    : parameters of the gate/up GEMM (Glu2Policy, gemm2_sm100.cuh)
//  DownPolicy   : per (expert, 128-wide d_lat slice, token tile):
//                 slot[t, j] = w'_{t,j} * (h W_down^T)          (swap-AB)
#pragma once
#include "gemm_sm100.cuh"
#include "topk.cuh"

namespace mrl {

// Running top-k lists: k <= 16 uses 16-entry lists (fewer registers in the
// router epilogue and the top-k kernels), 16 < k <= 32 the 32-entry ones.
constexpr int kTopKNarrow = 16;
constexpr int kTopKMax = 32;  // the largest k the library accepts

__device__ __forceinline__ int round16(int n) { return (n + 15) & ~15; }

// ---------------------------------------------------------------- dense
// BN output columns per unit: 256 normally; 64 when the token count is small
// (decode) and 256-wide tiles would leave most SMs idle, with a deeper ring of
// the smaller stages.
template <int BN>
struct DensePolicyN {
  static constexpr int kStages = BN >= 256 ? 4 : 8;
  static constexpr int kGroup = 2;
  static constexpr int kBN = BN;
  static constexpr int kABytes = 128 * 128;
  static constexpr int kBBytesMax = kBN * 128;
  static constexpr int kEpiSmem = 0;
  static constexpr int kAuxSmem = 0;
  static constexpr int kUmmaKBytes = 32;
  static constexpr int kASub = 1, kASubBytes = 0;
  struct Params {
    CUtensorMap ta;  // a [M, K], box 64 x 128
    CUtensorMap tb;  // w [N, K], box 64 x BN
    __nv_bfloat16 *out;
    __nv_bfloat16 *out_lo;  // optional: bf16(acc - float(out)), the residual of the rounding
    long ldo;
    int M, N, K, m_tiles, n_tiles;
    uint32_t *status;
  };
  struct EpiState {};
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
  static __device__ __forceinline__ uint32_t b_bytes(const Params &, const Unit &, int) { return kBBytesMax; }
  static __device__ __forceinline__ void load_a(const Params &p, const Unit &U, int, int kb, uint32_t sa,
                                                uint32_t bar) {
    tma_load_2d(sa, &p.ta, bar, kb * kBK, U.m * 128);
  }
  static __device__ __forceinline__ void load_b(const Params &p, const Unit &U, int, int kb, uint32_t sb,
                                                uint32_t bar) {
    tma_load_2d(sb, &p.tb, bar, kb * kBK, U.n0);
  }
  static __device__ __forceinline__ uint32_t idesc(const Params &, const Unit &U, int) {
    return idesc_bf16(128, round16(U.nv));
  }
  static __device__ __forceinline__ void mma(uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
    umma_f16(d, a, b, id, acc);
  }
  static __device__ __forceinline__ void epilogue(const Params &p, const Unit &U, int, uint32_t taddr, int q,
                                                  int lane, int, EpiState &, uint8_t *) {
    const int row = U.m * 128 + q * 32 + lane;
    for (int c0 = 0; c0 < U.nv; c0 += 32) {
      float v[32];
      tmem_ld32(taddr + c0, v);
      tmem_ld_wait();
      if (row < p.M) {
        uint4 *dst = reinterpret_cast<uint4 *>(p.out + row * p.ldo + U.n0 + c0);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint4 w;
          w.x = pack_bf16x2(v[8 * i + 0], v[8 * i + 1]);
          w.y = pack_bf16x2(v[8 * i + 2], v[8 * i + 3]);
          w.z = pack_bf16x2(v[8 * i + 4], v[8 * i + 5]);
          w.w = pack_bf16x2(v[8 * i + 6], v[8 * i + 7]);
          dst[i] = w;
        }
        if (p.out_lo) {
          // residual of the bf16 rounding: hi + lo carries the fp32 accumulator to ~2^-17
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] -= __bfloat162float(__float2bfloat16_rn(v[i]));
          uint4 *dlo = reinterpret_cast<uint4 *>(p.out_lo + row * p.ldo + U.n0 + c0);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint4 w;
            w.x = pack_bf16x2(v[8 * i + 0], v[8 * i + 1]);
            w.y = pack_bf16x2(v[8 * i + 2], v[8 * i + 3]);
            w.z = pack_bf16x2(v[8 * i + 4], v[8 * i + 5]);
            w.w = pack_bf16x2(v[8 * i + 6], v[8 * i + 7]);
            dlo[i] = w;
          }
        }
      }
    }
  }
};
using DensePolicy = DensePolicyN<256>;
using DenseNarrowPolicy = DensePolicyN<64>;

// ---------------------------------------------------------------- router
// B tile = R boxes of `ec` router rows (experts [sub*ec, sub*ec+ec) of router r),
// so accumulator column r*ec + j holds router r's logit for expert sub*ec + j.
// Router GEMM parameters (RouterPolicyK, RouterSplitPolicy).
struct RouterParams {
  CUtensorMap ta;     // z hi [T, L], box 64 x 128
  CUtensorMap ta_lo;  // z lo [T, L], box 64 x 128
  CUtensorMap tb;     // w_router [R*E, L], box 64 x ec
  const float *bias, *alpha;
  int32_t *topk_idx;
  float *topk_w, *wscaled, *scores;
  // parts > 1: the expert chunks are split over `parts` CTAs per token tile;
  // each leaves its best k candidates here for topk_merge_kernel
  float *cand_v, *cand_s;
  int32_t *cand_i;
  int T, L, E, R, ec, k, m_tiles, parts;
  int agg;  // mrlmoe_aggregation: 0 mean, 1 sum, 2 max of the R sigmoid scores
  // K split (RouterSplitPolicy): part[ks][t][r*E + e], fp32 logits of K range ks
  float *part;
  int ksplit;
  uint32_t *status;
};

// The routers read the latent at the down-projection's fp32 precision: z is
// given as bf16 hi + bf16 lo parts, and both halves meet the same router
// weight tile in one accumulator.  KMAX: length of the running top-k list.
template <int KMAX>
struct RouterPolicyK {
  // A stage holds both halves of the fp32 latent's 64-wide K block (z hi and
  // z lo, 128 tokens each) and the router weights once: both MMAs of the
  // block read the same B tile into one accumulator, so the weights cross
  // from L2 once per K block instead of once per half.
  static constexpr int kStages = 3;
  static constexpr int kGroup = 1;
  static constexpr int kASub = 2, kASubBytes = 128 * 128;
  static constexpr int kABytes = kASub * kASubBytes;
  static constexpr int kBBytesMax = 256 * 128;
  static constexpr int kEpiSmem = 0;
  static constexpr int kAuxSmem = 0;
  static constexpr int kUmmaKBytes = 32;
  using Params = RouterParams;
  struct EpiState {
    TopK<KMAX> tk;
  };
  static __device__ __forceinline__ void prefetch(const Params &p) {
    prefetch_tmap(&p.ta);
    prefetch_tmap(&p.ta_lo);
    prefetch_tmap(&p.tb);
  }
  static __device__ __forceinline__ void stage_aux(const Params &, uint8_t *) {}
  static __device__ __forceinline__ int num_units(const Params &p, const uint8_t *) { return p.m_tiles * p.parts; }
  static __device__ __forceinline__ int k_blocks(const Params &p) { return p.L / kBK; }
  static __device__ __forceinline__ Unit unit(const Params &p, int u, const uint8_t *) {
    Unit U;
    U.m = u / p.parts;
    U.g = u - U.m * p.parts;                 // part
    U.row0 = 0;
    U.n0 = 0;
    U.nv = p.R * p.ec;
    U.nsub = p.E / p.ec / p.parts;
    return U;
  }
  static __device__ __forceinline__ uint32_t b_bytes(const Params &p, const Unit &, int) {
    return p.R * p.ec * 128;
  }
  static __device__ __forceinline__ void load_a(const Params &p, const Unit &U, int, int kb, uint32_t sa,
                                                uint32_t bar) {
    tma_load_2d(sa, &p.ta, bar, kb * kBK, U.m * 128);
    tma_load_2d(sa + kASubBytes, &p.ta_lo, bar, kb * kBK, U.m * 128);
  }
  static __device__ __forceinline__ void load_b(const Params &p, const Unit &U, int sub, int kb, uint32_t sb,
                                                uint32_t bar) {
    const int x = kb * kBK;
    const int chunk = U.g * U.nsub + sub;
    for (int r = 0; r < p.R; ++r) tma_load_2d(sb + r * p.ec * 128, &p.tb, bar, x, r * p.E + chunk * p.ec);
  }
  static __device__ __forceinline__ uint32_t idesc(const Params &p, const Unit &, int) {
    return idesc_bf16(128, p.R * p.ec);
  }
  static __device__ __forceinline__ void mma(uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
    umma_f16(d, a, b, id, acc);
  }
  static __device__ __forceinline__ void epilogue(const Params &p, const Unit &U, int sub, uint32_t taddr, int q,
                                                  int lane, int, EpiState &st, uint8_t *) {
    const int t = U.m * 128 + q * 32 + lane;
    const bool valid = t < p.T;
    if (sub == 0) st.tk.init();
    const float invR = 1.0f / static_cast<float>(p.R);
    for (int j0 = 0; j0 < p.ec; j0 += 16) {
      float acc[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) acc[i] = 0.f;
      for (int r = 0; r < p.R; ++r) {
        float v[16];
        tmem_ld16(taddr + r * p.ec + j0, v);
        tmem_ld_wait();
        if (p.agg == 2) {
#pragma unroll
          for (int i = 0; i < 16; ++i) acc[i] = fmaxf(acc[i], sigmoidf_(v[i]));  // sigmoid >= 0
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) acc[i] += sigmoidf_(v[i]);
        }
      }
      const int e0 = (U.g * U.nsub + sub) * p.ec + j0;
      float s16[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        // mean: (sum) / R (R = 2^n makes this an exact scaling); sum and max as accumulated
        s16[i] = p.agg != 0 ? acc[i] : (p.R & (p.R - 1)) == 0 ? acc[i] * invR : acc[i] / static_cast<float>(p.R);
        const float sb = s16[i] + __ldg(p.bias + e0 + i);
        st.tk.offer(sb, e0 + i, s16[i]);
      }
      if (valid && p.scores) {
        float4 *dst = reinterpret_cast<float4 *>(p.scores + static_cast<size_t>(t) * p.E + e0);
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[i] = make_float4(s16[4 * i], s16[4 * i + 1], s16[4 * i + 2], s16[4 * i + 3]);
      }
    }
    if (sub == U.nsub - 1 && valid) {
      if (p.parts == 1) {
        write_selection<KMAX>(st.tk.s, st.tk.i, p.k, p.E, static_cast<size_t>(t), p.alpha, p.topk_idx, p.topk_w,
                              p.wscaled, p.status);
      } else {
        const size_t o = (static_cast<size_t>(t) * p.parts + U.g) * p.k;
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
          if (j < p.k) {
            p.cand_v[o + j] = st.tk.v[j];
            p.cand_s[o + j] = st.tk.s[j];
            p.cand_i[o + j] = st.tk.i[j];
          }
        }
      }
    }
  }
};

using RouterPolicy = RouterPolicyK<kTopKNarrow>;
using RouterPolicyWide = RouterPolicyK<kTopKMax>;

// Router with its K range split over CTAs, for token counts whose token tiles
// times expert chunks would occupy few SMs (decode): unit = (token tile m,
// expert chunk c, K range ks); the epilogue stores the tile's fp32 partial
// logits, router_split_scores_kernel sums the K ranges in order and applies
// the sigmoid and the aggregation, and topk_from_scores_kernel selects.
struct RouterSplitPolicy : RouterPolicy {
  struct EpiState {};
  static __device__ __forceinline__ int num_units(const Params &p, const uint8_t *) {
    return p.m_tiles * (p.E / p.ec) * p.ksplit;
  }
  static __device__ __forceinline__ int k_blocks(const Params &p) { return p.L / kBK / p.ksplit; }
  static __device__ __forceinline__ Unit unit(const Params &p, int u, const uint8_t *) {
    Unit U;
    const int chunks = p.E / p.ec;
    U.n0 = u % p.ksplit;            // K range
    U.g = (u / p.ksplit) % chunks;  // expert chunk
    U.m = u / (p.ksplit * chunks);  // token tile
    U.row0 = 0;
    U.nv = p.R * p.ec;
    U.nsub = 1;
    return U;
  }
  static __device__ __forceinline__ void load_a(const Params &p, const Unit &U, int, int kb, uint32_t sa,
                                                uint32_t bar) {
    const int x = (U.n0 * k_blocks(p) + kb) * kBK;
    tma_load_2d(sa, &p.ta, bar, x, U.m * 128);
    tma_load_2d(sa + kASubBytes, &p.ta_lo, bar, x, U.m * 128);
  }
  static __device__ __forceinline__ void load_b(const Params &p, const Unit &U, int, int kb, uint32_t sb,
                                                uint32_t bar) {
    const int x = (U.n0 * k_blocks(p) + kb) * kBK;
    for (int r = 0; r < p.R; ++r) tma_load_2d(sb + r * p.ec * 128, &p.tb, bar, x, r * p.E + U.g * p.ec);
  }
  // Accumulator column r*ec + i is router r's logit of expert U.g*ec + i.
  static __device__ __forceinline__ void epilogue(const Params &p, const Unit &U, int, uint32_t taddr, int q,
                                                  int lane, int, EpiState &, uint8_t *) {
    const int t = U.m * 128 + q * 32 + lane;
    const bool valid = t < p.T;
    float *row = p.part + (static_cast<size_t>(U.n0) * p.T + t) * (static_cast<size_t>(p.R) * p.E) + U.g * p.ec;
    for (int c0 = 0; c0 < p.R * p.ec; c0 += 16) {
      float v[16];
      tmem_ld16(taddr + c0, v);
      tmem_ld_wait();
      if (valid) {
        const int r = c0 / p.ec, i0 = c0 - r * p.ec;
        float4 *dst = reinterpret_cast<float4 *>(row + static_cast<size_t>(r) * p.E + i0);
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
      }
    }
  }
};

// --------------------------------------------------------- grouped helpers
// Dispatch groups: g < E routed expert g, g == E the shared expert.  Rows of
// group g start at grp_off[g] in the dispatched activation buffers and number
// grp_cnt[g]; unit_off[g] is the exclusive prefix of units per group
// (unit_off[E+1] = total).  The three tables (E+2 ints each) are staged in
// shared memory once per CTA, so mapping a unit to its group costs a short
// binary search in shared memory instead of dependent global loads.
struct GroupTable {
  const int32_t *grp_off, *grp_cnt, *unit_off;
  int E, m_tiles;  // M tiles per group
};

constexpr int kMaxGroups = 1024 + 2;
constexpr int kGroupAuxSmem = 2 * kMaxGroups * 4;

// unit_off and grp_off (E+2 entries each; grp_off[E+1] ends the shared
// group, so a group's row count is grp_off[g+1] - grp_off[g]).
__device__ __forceinline__ void stage_group_table(const GroupTable &gt, uint8_t *aux) {
  int *s = reinterpret_cast<int *>(aux);
  const int n = gt.E + 2;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    s[i] = __ldg(gt.unit_off + i);
    s[kMaxGroups + i] = __ldg(gt.grp_off + i);
  }
}

__device__ __forceinline__ int grouped_num_units(const GroupTable &gt, const uint8_t *aux) {
  return reinterpret_cast<const int *>(aux)[gt.E + 1];
}

__device__ __forceinline__ Unit grouped_unit(const GroupTable &gt, const uint8_t *aux, int u, int BN) {
  const int *uo = reinterpret_cast<const int *>(aux);
  const int *go = uo + kMaxGroups;
  // largest g in [0, E] with unit_off[g] <= u (zero-unit groups share the next offset)
  int lo = 0, hi = gt.E;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (uo[mid] <= u) lo = mid; else hi = mid - 1;
  }
  Unit U;
  U.g = lo;
  const int local = u - uo[lo];
  const int cnt = go[lo + 1] - go[lo];
  const int ntiles = (cnt + BN - 1) / BN;
  U.m = local / ntiles;
  U.n0 = (local - U.m * ntiles) * BN;
  U.nv = min(BN, cnt - U.n0);
  U.nsub = 1;
  U.row0 = go[lo] + U.n0;
  return U;
}

// Token rows y0 .. y0+n-1 (n a multiple of 16) of a K-major token tensor,
// as 64-row boxes, then at most one 32-row and one 16-row box, back to back
// in shared memory (128 B a row; every box is whole 8-row swizzle atoms).
// One TMA copy costs its issuing thread on the order of a hundred cycles,
// so a token tile of 160 rows takes 3 copies instead of 10 16-row ones.
// PAIR: the cta_group::2 form, completing on the even CTA's barrier.
//
// Two layouts of a bf16 token tensor [rows, K]: row-major (plane_rows == 0;
// K block kb of row r at x = 64 kb, y = r), or K-blocked, [K/64][rows][64]
// (plane_rows == rows; the tensor map sees [K/64 * rows, 64] and K block kb
// of row r sits at x = 0, y = kb * rows + r).  In the blocked layout a tile of
// consecutive rows is one contiguous range for every K block, for the TMA
// loads here and for the epilogue that writes it.
struct TokenMaps {
  CUtensorMap m16, m32, m64;  // the same tensor, boxes of 16 / 32 / 64 rows x 128 B
  int plane_rows;             // 0: row-major; else rows per K-block plane
};

template <bool PAIR>
__device__ __forceinline__ void load_token_rows(const TokenMaps &t, int kb, int y0, int n, uint32_t sb, uint32_t bar) {
  const int x = t.plane_rows ? 0 : kb * kBK;
  const int yb = t.plane_rows ? kb * t.plane_rows + y0 : y0;
  auto copy = [&](const CUtensorMap *m, int r) {
    if constexpr (PAIR)
      tma_load_2d_pair(sb + r * 128, m, bar, x, yb + r);
    else
      tma_load_2d(sb + r * 128, m, bar, x, yb + r);
  };
  int r = 0;
  for (; r + 64 <= n; r += 64) copy(&t.m64, r);
  if (r + 32 <= n) { copy(&t.m32, r); r += 32; }
  if (r + 16 <= n) copy(&t.m16, r);
}

__device__ __forceinline__ void prefetch_token_maps(const TokenMaps &t) {
  prefetch_tmap(&t.m16);
  prefetch_tmap(&t.m32);
  prefetch_tmap(&t.m64);
}

// B operand: the unit's dispatched rows, rounded up to a multiple of 32.
__device__ __forceinline__ void load_rows(const TokenMaps &t, const Unit &U, int kb, uint32_t sb, uint32_t bar) {
  load_token_rows<false>(t, kb, U.row0, (U.nv + 31) & ~31, sb, bar);
}

// --------------------------------------------------------------- gate/up
// Parameters of the gate/up GEMM (run on CTA pairs by Glu2Policy in
// gemm2_sm100.cuh): routed and shared gate/up weights, the dispatched latent
// rows, and h.
struct GluParams {
  CUtensorMap wg, wu;  // routed gate/up [E*F, L], box 64 x 64
  CUtensorMap sg, su;  // shared gate/up [F, L], box 64 x 64
  TokenMaps tz;        // dispatched z [(T*k+T), L] row-major, boxes 64 x 16/32/64
  GroupTable gt;
  __nv_bfloat16 *h;    // [F/64][T*k+T][64], K-blocked (see TokenMaps)
  uint32_t *gu;        // training forward: bf16 gate (low half) and up (high half) pre-activations,
                       // one word per element laid out as h (else null)
  int F, L, rows;      // rows = T*k+T
  uint32_t *status;
};

__device__ __forceinline__ void prefetch_glu(const GluParams &p) {
  prefetch_tmap(&p.wg);
  prefetch_tmap(&p.wu);
  prefetch_tmap(&p.sg);
  prefetch_tmap(&p.su);
  prefetch_token_maps(p.tz);
}

// ------------------------------------------------------------------ down
struct DownPolicy {
  static constexpr int kStages = 4;
  static constexpr int kGroup = 2;
  static constexpr int kBN = 256;
  static constexpr int kABytes = 128 * 128;
  static constexpr int kBBytesMax = kBN * 128;
  static constexpr int kEpiSmem = kBN * 8;
  static constexpr int kAuxSmem = kGroupAuxSmem;
  static constexpr int kUmmaKBytes = 32;
  static constexpr int kASub = 1, kASubBytes = 0;
  struct Params {
    CUtensorMap wd;  // routed down [E*L, F], box 64 x 128
    CUtensorMap sd;  // shared down [L, F], box 64 x 128
    TokenMaps th;    // h [F/64][T*k+T][64] K-blocked, boxes 64 x 16/32/64
    GroupTable gt;
    const int32_t *perm;
    const float *wscaled;
    float *slots;    // [T, k+1, L]
    // expert-parallel owner: row r's unweighted output goes to row out_row[r]
    // of `slots` (then [rows, L] fp32) instead of its token's weighted slot
    const int32_t *out_row;
    int L, F, k, Tk;
    uint32_t *status;
  };
  struct EpiState {};
  static __device__ __forceinline__ void prefetch(const Params &p) {
    prefetch_tmap(&p.wd); prefetch_tmap(&p.sd); prefetch_token_maps(p.th);
  }
  static __device__ __forceinline__ void stage_aux(const Params &p, uint8_t *aux) { stage_group_table(p.gt, aux); }
  static __device__ __forceinline__ int num_units(const Params &p, const uint8_t *aux) {
    return grouped_num_units(p.gt, aux);
  }
  static __device__ __forceinline__ int k_blocks(const Params &p) { return p.F / kBK; }
  static __device__ __forceinline__ Unit unit(const Params &p, int u, const uint8_t *aux) {
    return grouped_unit(p.gt, aux, u, kBN);
  }
  static __device__ __forceinline__ uint32_t b_bytes(const Params &, const Unit &U, int) {
    return ((U.nv + 31) >> 5) * 4096;
  }
  static __device__ __forceinline__ void load_a(const Params &p, const Unit &U, int, int kb, uint32_t sa,
                                                uint32_t bar) {
    const bool sh = U.g == p.gt.E;
    tma_load_2d(sa, sh ? &p.sd : &p.wd, bar, kb * kBK, (sh ? 0 : U.g * p.L) + U.m * 128);
  }
  static __device__ __forceinline__ void load_b(const Params &p, const Unit &U, int, int kb, uint32_t sb,
                                                uint32_t bar) {
    load_rows(p.th, U, kb, sb, bar);
  }
  static __device__ __forceinline__ uint32_t idesc(const Params &, const Unit &U, int) {
    return idesc_bf16(128, round16(U.nv));
  }
  static __device__ __forceinline__ void mma(uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
    umma_f16(d, a, b, id, acc);
  }
  // Lane = output dim l; column = token.  The unit's per-column slot row and
  // weight (w', 1 for the shared expert and for the rows of an expert-parallel
  // owner) are first staged in shared memory (one parallel pass over the
  // dispatch record), then for each token column the warp writes 32
  // consecutive fp32 of that token's slot row (128 B, coalesced).
  static __device__ __forceinline__ void epilogue(const Params &p, const Unit &U, int, uint32_t taddr, int q,
                                                  int lane, int etid, EpiState &, uint8_t *epi) {
    int *s_slot = reinterpret_cast<int *>(epi);
    float *s_wt = reinterpret_cast<float *>(epi + kBN * sizeof(int));
    const int l = U.m * 128 + q * 32 + lane;
    const bool sh = U.g == p.gt.E;
    const int row0 = U.row0;
    for (int c = etid; c < U.nv; c += 128) {
      const int row = row0 + c;
      if (p.out_row) {
        s_slot[c] = __ldg(p.out_row + row);
        s_wt[c] = 1.0f;
      } else if (sh) {
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
    for (int c0 = 0; c0 < U.nv; c0 += 32) {
      float v[32];
      tmem_ld32(taddr + c0, v);
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        if (c0 + c < U.nv)
          p.slots[static_cast<size_t>(s_slot[c0 + c]) * p.L + l] = v[c] * s_wt[c0 + c];
      }
    }
    named_bar_sync(2, 128);  // s_slot/s_wt are rewritten by the next unit
  }
};

}  // namespace mrl
