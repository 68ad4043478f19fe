// backward.cuh — the layer's backward pass: gradients of a loss through y
// with respect to x and every learnable tensor, from the activations that
// the training forward keeps in the workspace.
//
// With dy the incoming gradient, the chain (top-k selection and the balancing
// bias carry no gradient; the bf16 rounding points pass it through):
//   dn  = dy W_up                     dW_up = dy^T n                  (dense)
//   c = sum of the slots, r = rms^-1, cn = c r:
//   dc  = r (dn g - cn mean(cn dn g)) dgain = sum_t dn cn           (per token)
//   per dispatch row of expert e (token t, weight w' = w alpha):
//   dh' = dc_t W_d,e                  dw'  = <h, dh'>                (grouped)
//   dh  = w' dh';  dg = dh u SiLU'(g);  du = dh SiLU(g)   (h = SiLU(g) u from the kept bf16 g, u)
//   dz  = dg W_g,e + du W_u,e                                          (grouped)
//   dW_g,e = dg^T z, dW_u,e = du^T z, dW_d,e = (w' dc)^T h            (grouped, K = rows)
//   dalpha_e = sum over e's rows of w dw';  dw = alpha dw'
//   ds_sel = (dw - sum_j w_j dw_j) / sum_j s_j;  router r: dl = dp p (1 - p)
//   dzx = sum of the rows' dz + sum_{j,r} dl W_router[r, e_j]         (per token)
//   dW_router[r, e] = sum over e's rows of dl zx
//   dx  = dzx W_dn                    dW_dn = dzx^T x                  (dense)
// GEMMs whose reduction runs over the stored [out, in] weight's out index, or
// over tokens, read that operand MN-major: the tensor core takes it as is,
// with no transposed copy of any weight or activation.
#pragma once
#include "policies.cuh"
#include "gemm2_sm100.cuh"

namespace mrl {

// ------------------------------------------------------- dense gradients
// out[M, N] = A B over K, fp32 accumulate, written as fp32 or bf16:
//   A K-major [M, K] (one box of 64 K x 128 rows), or MN-major [K, M] (two
//   boxes of 64 M x 64 K rows: x = M index, y = K index);
//   B K-major [N, K] (box 64 K x BN rows), or MN-major [K, N] (BN/64 boxes).
// K beyond the tensors' extent reads the TMA zero fill.
template <bool AMN, bool BMN, bool OUTF32>
struct DenseGradPolicy {
  static constexpr bool kAMN = AMN, kBMN = BMN;
  static constexpr uint32_t kAMNStride = 8192, kBMNStride = 8192;
  static constexpr int kStages = 4;
  static constexpr int kGroup = 2;
  static constexpr int kBN = 256;
  static constexpr int kABytes = 128 * 128;
  static constexpr int kBBytesMax = kBN * 128;
  static constexpr int kEpiSmem = 0;
  static constexpr int kAuxSmem = 0;
  static constexpr int kUmmaKBytes = 32;
  static constexpr int kASub = 1, kASubBytes = 0;
  struct Params {
    CUtensorMap ta, tb;
    void *out;  // fp32 or bf16 [M, ldo]
    long ldo;
    int M, N, K, m_tiles, n_tiles;
    int accumulate;  // fp32 output: add to it instead of overwriting
    uint32_t *status;
  };
  struct EpiState {};
  static __device__ __forceinline__ void prefetch(const Params &p) {
    prefetch_tmap(&p.ta);
    prefetch_tmap(&p.tb);
  }
  static __device__ __forceinline__ void stage_aux(const Params &, uint8_t *) {}
  static __device__ __forceinline__ int num_units(const Params &p, const uint8_t *) { return p.m_tiles * p.n_tiles; }
  static __device__ __forceinline__ int k_blocks(const Params &p) { return (p.K + kBK - 1) / kBK; }
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
  static __device__ __forceinline__ uint32_t b_bytes(const Params &, const Unit &U, int) {
    return BMN ? ((U.nv + 63) / 64) * 8192 : kBBytesMax;
  }
  static __device__ __forceinline__ void load_a(const Params &p, const Unit &U, int, int kb, uint32_t sa,
                                                uint32_t bar) {
    if constexpr (AMN) {
      tma_load_2d(sa, &p.ta, bar, U.m * 128, kb * kBK);
      tma_load_2d(sa + 8192, &p.ta, bar, U.m * 128 + 64, kb * kBK);
    } else {
      tma_load_2d(sa, &p.ta, bar, kb * kBK, U.m * 128);
    }
  }
  static __device__ __forceinline__ void load_b(const Params &p, const Unit &U, int, int kb, uint32_t sb,
                                                uint32_t bar) {
    if constexpr (BMN) {
      for (int i = 0; i * 64 < U.nv; ++i) tma_load_2d(sb + i * 8192, &p.tb, bar, U.n0 + i * 64, kb * kBK);
    } else {
      tma_load_2d(sb, &p.tb, bar, kb * kBK, U.n0);
    }
  }
  static __device__ __forceinline__ uint32_t idesc(const Params &, const Unit &U, int) {
    return idesc_bf16_major(128, round16(U.nv), AMN, BMN);
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
      if (row >= p.M) continue;
      if constexpr (OUTF32) {
        float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(p.out) + row * p.ldo + U.n0 + c0);
        if (p.accumulate) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 o = dst[i];
            v[4 * i] += o.x; v[4 * i + 1] += o.y; v[4 * i + 2] += o.z; v[4 * i + 3] += o.w;
          }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
      } else {
        uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.out) + row * p.ldo + U.n0 + c0);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint4 w;
          w.x = pack_bf16x2(v[8 * i + 0], v[8 * i + 1]);
          w.y = pack_bf16x2(v[8 * i + 2], v[8 * i + 3]);
          w.z = pack_bf16x2(v[8 * i + 4], v[8 * i + 5]);
          w.w = pack_bf16x2(v[8 * i + 6], v[8 * i + 7]);
          dst[i] = w;
        }
      }
    }
  }
};

// Two 64-wide MN-major boxes of an expert weight [rows, inner] at inner
// index x0 (the tile's M index) and row y (its K index).
__device__ __forceinline__ void load_mn_pair(uint32_t sa, const CUtensorMap *m, uint32_t bar, int x0, int y) {
  tma_load_2d(sa, m, bar, x0, y);
  tma_load_2d(sa + 8192, m, bar, x0 + 64, y);
}

// a[c] summed over the warp's 32 lanes, for all 32 c at once: lane i returns
// the sum for c = i (31 shuffles instead of 32 x 5).
__device__ __forceinline__ float transpose_sum32(float (&a)[32], int lane) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < off; ++i) {
      const float send = upper ? a[i] : a[i + off];
      const float keep = upper ? a[i + off] : a[i];
      a[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
  return a[0];
}

// ------------------------------------------ expert dgrad through W_down
// Swap-AB over the dispatch groups: unit = (group, 128-wide d_ff slice m,
// <= 256 dispatch rows); D[f, row] = sum_l W_d[l, f] dc[row, l], so W_d is
// read MN-major straight from its [d_lat, d_ff] storage.  The epilogue
// finishes the GLU backward on the tile and leaves dg, du (K-blocked, as h)
// and the slice's share of dw' = <h, dh'> per row, with h = SiLU(g) u
// recomputed from the bf16 g and u that the training forward kept (one
// 4-byte word per element; the next 32 rows' words load while the current
// ones are used).
struct DhPolicy {
  static constexpr bool kAMN = true, kBMN = false;
  static constexpr uint32_t kAMNStride = 8192, kBMNStride = 0;
  static constexpr int kStages = 4;
  static constexpr int kGroup = 2;
  static constexpr int kBN = 256;
  static constexpr int kABytes = 128 * 128;
  static constexpr int kBBytesMax = kBN * 128;
  static constexpr int kEpiSmem = kBN * 4 + 4 * kBN * 4;  // row weights, per-warp partial sums
  static constexpr int kAuxSmem = kGroupAuxSmem;
  static constexpr int kUmmaKBytes = 32;
  static constexpr int kASub = 1, kASubBytes = 0;
  struct Params {
    CUtensorMap wd;  // routed W_down [E*L, F] as MN-major boxes 64 x 64
    CUtensorMap sd;  // shared W_down [L, F]
    TokenMaps tc;    // dc rows [rows, L] row-major, boxes 64 x 16/32/64
    GroupTable gt;   // M tiles per group: F / 128
    const float *wrow;               // [rows]: w' of each dispatch row (1 for the shared expert's)
    const uint32_t *gu;              // [F/64][rows][64] words: bf16 g (low), u (high)
    __nv_bfloat16 *dgu;              // [2F/64][rows][64]: dg planes, then du planes
    float *dwsp;                     // [F/128][rows]: per-slice share of dw' by dispatch row
    int L, F, rows;
    uint32_t *status;
  };
  struct EpiState {};
  static __device__ __forceinline__ void prefetch(const Params &p) {
    prefetch_tmap(&p.wd); prefetch_tmap(&p.sd); prefetch_token_maps(p.tc);
  }
  static __device__ __forceinline__ void stage_aux(const Params &p, uint8_t *aux) { stage_group_table(p.gt, aux); }
  static __device__ __forceinline__ int num_units(const Params &p, const uint8_t *aux) {
    return grouped_num_units(p.gt, aux);
  }
  static __device__ __forceinline__ int k_blocks(const Params &p) { return p.L / kBK; }
  static __device__ __forceinline__ Unit unit(const Params &p, int u, const uint8_t *aux) {
    return grouped_unit(p.gt, aux, u, kBN);
  }
  static __device__ __forceinline__ uint32_t b_bytes(const Params &, const Unit &U, int) {
    return ((U.nv + 31) >> 5) * 4096;
  }
  static __device__ __forceinline__ void load_a(const Params &p, const Unit &U, int, int kb, uint32_t sa,
                                                uint32_t bar) {
    const bool sh = U.g == p.gt.E;
    load_mn_pair(sa, sh ? &p.sd : &p.wd, bar, U.m * 128, (sh ? 0 : U.g * p.L) + kb * kBK);
  }
  static __device__ __forceinline__ void load_b(const Params &p, const Unit &U, int, int kb, uint32_t sb,
                                                uint32_t bar) {
    load_rows(p.tc, U, kb, sb, bar);
  }
  static __device__ __forceinline__ uint32_t idesc(const Params &, const Unit &U, int) {
    return idesc_bf16_major(128, round16(U.nv), true, false);
  }
  static __device__ __forceinline__ void mma(uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
    umma_f16(d, a, b, id, acc);
  }
  // Lane = f, column = dispatch row.  Per column the warp's 32 lanes hold 32
  // consecutive f of one K-blocked plane (64 contiguous bytes of g, u, h).
  static __device__ __forceinline__ void epilogue(const Params &p, const Unit &U, int, uint32_t taddr, int q,
                                                  int lane, int etid, EpiState &, uint8_t *epi) {
    float *s_ws = reinterpret_cast<float *>(epi);
    float *red = reinterpret_cast<float *>(epi + kBN * 4);  // [4][kBN]
    for (int c = etid; c < U.nv; c += 128) s_ws[c] = __ldg(p.wrow + U.row0 + c);
    named_bar_sync(2, 128);
    const int f = U.m * 128 + q * 32 + lane;
    const size_t plane = static_cast<size_t>(f >> 6);
    const size_t prow = static_cast<size_t>(p.rows) * 64;
    const int within = f & 63;
    const uint32_t *gup = p.gu + plane * prow + within;
    __nv_bfloat16 *dgp = p.dgu + plane * prow + within;
    __nv_bfloat16 *dup = p.dgu + (static_cast<size_t>(p.F >> 6) + plane) * prow + within;
    uint32_t cur[32], nxt[32];
    auto load_chunk = [&](uint32_t (&dst)[32], int c0) {
#pragma unroll
      for (int c = 0; c < 32; ++c)
        dst[c] = c0 + c < U.nv ? __ldg(gup + static_cast<size_t>(U.row0 + c0 + c) * 64) : 0u;
    };
    load_chunk(cur, 0);
    for (int c0 = 0; c0 < U.nv; c0 += 32) {
      float v[32];
      tmem_ld32(taddr + c0, v);
      if (c0 + 32 < U.nv) load_chunk(nxt, c0 + 32);
      tmem_ld_wait();
      float part[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const int col = c0 + c;
        const float g = __uint_as_float(cur[c] << 16);
        const float u = __uint_as_float(cur[c] & 0xFFFF0000u);
        const float sg = __fdividef(1.0f, 1.0f + __expf(-g));
        part[c] = g * sg * u * v[c];
        if (col < U.nv) {  // uniform over the warp
          const size_t o = static_cast<size_t>(U.row0 + col) * 64;
          const float dh = s_ws[col] * v[c];
          dgp[o] = __float2bfloat16_rn(dh * u * sg * (1.0f + g * (1.0f - sg)));
          dup[o] = __float2bfloat16_rn(dh * g * sg);
        }
      }
#pragma unroll
      for (int c = 0; c < 32; ++c) cur[c] = nxt[c];
      const float tot = transpose_sum32(part, lane);  // lane i: column c0 + i summed over the warp's 32 f
      if (c0 + lane < U.nv) red[q * kBN + c0 + lane] = tot;
    }
    named_bar_sync(2, 128);
    for (int c = etid; c < U.nv; c += 128)
      p.dwsp[static_cast<size_t>(U.m) * p.rows + U.row0 + c] =
          (red[c] + red[kBN + c]) + (red[2 * kBN + c] + red[3 * kBN + c]);
    named_bar_sync(2, 128);  // s_ws/red are rewritten by the next unit
  }
};

// ------------------------------------- expert dgrad through W_gate, W_up
// Swap-AB: unit = (group, 128-wide d_lat slice, <= 256 rows); D[l, row] =
// sum_f W_g[f, l] dg[row, f] + W_u[f, l] du[row, f] over K = 2 d_ff (gate
// half, then up half), W_g and W_u read MN-major from their [d_ff, d_lat]
// storage.  The epilogue writes dz of each row into its token's slot
// (t, j), the shared expert's rows into slot k, as the forward's down GEMM
// does for o.
struct DzPolicy {
  static constexpr bool kAMN = true, kBMN = false;
  static constexpr uint32_t kAMNStride = 8192, kBMNStride = 0;
  static constexpr int kStages = 4;
  static constexpr int kGroup = 2;
  static constexpr int kBN = 256;
  static constexpr int kABytes = 128 * 128;
  static constexpr int kBBytesMax = kBN * 128;
  static constexpr int kEpiSmem = kBN * 4;
  static constexpr int kAuxSmem = kGroupAuxSmem;
  static constexpr int kUmmaKBytes = 32;
  static constexpr int kASub = 1, kASubBytes = 0;
  struct Params {
    CUtensorMap wg, wu;  // routed [E*F, L] as MN-major boxes 64 x 64
    CUtensorMap sg, su;  // shared [F, L]
    TokenMaps tgu;       // dgu [2F/64][rows][64] K-blocked
    GroupTable gt;       // M tiles per group: L / 128
    const int32_t *perm;
    float *dzs;          // [T, k+1, L]
    int L, F, k, Tk;
    uint32_t *status;
  };
  struct EpiState {};
  static __device__ __forceinline__ void prefetch(const Params &p) {
    prefetch_tmap(&p.wg); prefetch_tmap(&p.wu); prefetch_tmap(&p.sg); prefetch_tmap(&p.su);
    prefetch_token_maps(p.tgu);
  }
  static __device__ __forceinline__ void stage_aux(const Params &p, uint8_t *aux) { stage_group_table(p.gt, aux); }
  static __device__ __forceinline__ int num_units(const Params &p, const uint8_t *aux) {
    return grouped_num_units(p.gt, aux);
  }
  static __device__ __forceinline__ int k_blocks(const Params &p) { return 2 * p.F / kBK; }
  static __device__ __forceinline__ Unit unit(const Params &p, int u, const uint8_t *aux) {
    return grouped_unit(p.gt, aux, u, kBN);
  }
  static __device__ __forceinline__ uint32_t b_bytes(const Params &, const Unit &U, int) {
    return ((U.nv + 31) >> 5) * 4096;
  }
  static __device__ __forceinline__ void load_a(const Params &p, const Unit &U, int, int kb, uint32_t sa,
                                                uint32_t bar) {
    const bool sh = U.g == p.gt.E;
    const int fb = p.F / kBK;
    const bool up = kb >= fb;
    const CUtensorMap *m = sh ? (up ? &p.su : &p.sg) : (up ? &p.wu : &p.wg);
    load_mn_pair(sa, m, bar, U.m * 128, (sh ? 0 : U.g * p.F) + (kb - (up ? fb : 0)) * kBK);
  }
  static __device__ __forceinline__ void load_b(const Params &p, const Unit &U, int, int kb, uint32_t sb,
                                                uint32_t bar) {
    load_rows(p.tgu, U, kb, sb, bar);
  }
  static __device__ __forceinline__ uint32_t idesc(const Params &, const Unit &U, int) {
    return idesc_bf16_major(128, round16(U.nv), true, false);
  }
  static __device__ __forceinline__ void mma(uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
    umma_f16(d, a, b, id, acc);
  }
  static __device__ __forceinline__ void epilogue(const Params &p, const Unit &U, int, uint32_t taddr, int q,
                                                  int lane, int etid, EpiState &, uint8_t *epi) {
    int *s_slot = reinterpret_cast<int *>(epi);
    const int l = U.m * 128 + q * 32 + lane;
    const bool sh = U.g == p.gt.E;
    for (int c = etid; c < U.nv; c += 128) {
      const int row = U.row0 + c;
      if (sh) {
        s_slot[c] = (row - p.Tk) * (p.k + 1) + p.k;
      } else {
        const int flat = __ldg(p.perm + row);
        const int t = flat / p.k;
        s_slot[c] = t * (p.k + 1) + (flat - t * p.k);
      }
    }
    named_bar_sync(2, 128);
    for (int c0 = 0; c0 < U.nv; c0 += 32) {
      float v[32];
      tmem_ld32(taddr + c0, v);
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < 32; ++c)
        if (c0 + c < U.nv) p.dzs[static_cast<size_t>(s_slot[c0 + c]) * p.L + l] = v[c];
    }
    named_bar_sync(2, 128);
  }
};

// DzPolicy over a CTA pair (gemm2_kernel): unit = (group, 256-wide d_lat
// slice, <= 256 rows); CTA r owns d_lat rows m*256 + r*128 .. +127 (its A
// tile: W_g / W_u MN-major at that offset) and loads half of the unit's dg/du
// rows, so the rows cross from L2 once per pair.
struct Dz2Policy {
  static constexpr bool kAMN = true, kBMN = false;
  static constexpr uint32_t kAMNStride = 8192, kBMNStride = 0;
  static constexpr int kStages = 6;
  static constexpr int kGroup = 2;
  static constexpr int kBN = 256;
  static constexpr int kABytes = 128 * 128;
  static constexpr int kBBytesMax = (kBN / 2) * 128;
  static constexpr int kEpiSmem = DzPolicy::kEpiSmem;
  static constexpr int kAuxSmem = kGroupAuxSmem;
  using Params = DzPolicy::Params;  // gt: M tiles per group = d_lat / 256
  static __device__ __forceinline__ void prefetch(const Params &p) { DzPolicy::prefetch(p); }
  static __device__ __forceinline__ void stage_aux(const Params &p, uint8_t *aux) { stage_group_table(p.gt, aux); }
  static __device__ __forceinline__ int num_units(const Params &p, const uint8_t *aux) {
    return grouped_num_units(p.gt, aux);
  }
  static __device__ __forceinline__ int k_blocks(const Params &p) { return 2 * p.F / kBK; }
  static __device__ __forceinline__ Unit unit(const Params &p, int u, const uint8_t *aux) {
    return grouped_unit(p.gt, aux, u, kBN);
  }
  static __device__ __forceinline__ uint32_t b_bytes_pair(const Params &, const Unit &U) {
    return round32(U.nv) * 128;
  }
  static __device__ __forceinline__ void load_a(const Params &p, const Unit &U, int kb, uint32_t sa,
                                                uint32_t bar_cl, uint32_t rank) {
    const bool sh = U.g == p.gt.E;
    const int fb = p.F / kBK;
    const bool up = kb >= fb;
    const CUtensorMap *m = sh ? (up ? &p.su : &p.sg) : (up ? &p.wu : &p.wg);
    const int x0 = U.m * 256 + static_cast<int>(rank) * 128;
    const int y = (sh ? 0 : U.g * p.F) + (kb - (up ? fb : 0)) * kBK;
    tma_load_2d_pair(sa, m, bar_cl, x0, y);
    tma_load_2d_pair(sa + 8192, m, bar_cl, x0 + 64, y);
  }
  static __device__ __forceinline__ void load_b(const Params &p, const Unit &U, int kb, uint32_t sb,
                                                uint32_t bar_cl, uint32_t rank) {
    load_rows_half(p.tgu, U, kb, sb, bar_cl, rank);
  }
  static __device__ __forceinline__ uint32_t idesc(const Params &, const Unit &U) {
    return idesc_bf16_major(256, round32(U.nv), true, false);
  }
  static __device__ __forceinline__ void epilogue(const Params &p, const Unit &U, uint32_t taddr, int q, int lane,
                                                  int etid, uint32_t rank, uint8_t *epi) {
    Unit V = U;
    V.m = U.m * 2 + static_cast<int>(rank);  // this CTA's 128-row d_lat slice
    DzPolicy::EpiState st;
    DzPolicy::epilogue(p, V, 0, taddr, q, lane, etid, st, epi);
  }
};

// ------------------------------------------------ expert weight gradients
// Unit = (group, matrix, 128 x 256 output tile); the reduction runs over the
// group's dispatch rows (K = rows, ragged), both operands MN-major:
//   dW_g[f, l] = sum_rows dg[row, f] z[row, l]    A: dg planes, B: z rows
//   dW_u[f, l] = sum_rows du[row, f] z[row, l]    A: du planes, B: z rows
//   dW_d[l, f] = sum_rows do[row, l] h[row, f]    A: do rows,   B: h planes
// with do = w' dc.  Rows past the group's end in its last K block belong to
// the next group (or are the TMA zero fill); they are zeroed in shared
// memory before the MMAs.  A group without rows writes zero tiles.  The fp32
// tiles leave through TMA stores: each epilogue warp stages its 32 rows x 32
// columns in a swizzled 4 KB buffer (kStoreBufs per warp, in rotation) and one
// lane issues the bulk store, so the gradient writes go out as whole lines.
struct WgradPolicy {
  static constexpr bool kAMN = true, kBMN = true, kRaggedK = true;
  static constexpr uint32_t kAMNStride = 8192, kBMNStride = 8192;
  static constexpr int kStages = 3;
  static constexpr int kGroup = 1;
  static constexpr int kBN = 256;
  static constexpr int kABytes = 128 * 128;
  static constexpr int kBBytesMax = kBN * 128;
  static constexpr int kStoreBufs = 4;
  static constexpr int kEpiSmem = 4 * kStoreBufs * 4096 + 1024;  // + alignment of the swizzled buffers
  static constexpr int kAuxSmem = kMaxGroups * 4;
  static constexpr int kUmmaKBytes = 32;
  static constexpr int kASub = 1, kASubBytes = 0;
  struct Params {
    CUtensorMap tdgu;  // dgu [2F/64 * rows, 64], boxes 64 x 64
    CUtensorMap tz;    // z rows [rows, L], boxes 64 x 64
    CUtensorMap tdo;   // do rows [rows, L], boxes 64 x 64
    CUtensorMap th;    // h [F/64 * rows, 64], boxes 64 x 64
    // fp32 gradients, boxes of 32 columns x 32 rows, SWIZZLE_128B:
    CUtensorMap og, ou, od;    // routed [E*F, L], [E*F, L], [E*L, F]
    CUtensorMap sog, sou, sod; // shared [F, L], [F, L], [L, F]
    const int32_t *grp_off;  // E + 2 entries
    int E, F, L, rows;
    int accumulate;          // add the tiles to the gradients (TMA reduce-add) instead of storing
    uint32_t *status;
  };
  struct EpiState {
    int n = 0;  // chunks this thread's warp has staged (selects the buffer)
  };
  static __device__ __forceinline__ int tiles_gu(const Params &p) { return (p.F / 128) * ((p.L + kBN - 1) / kBN); }
  static __device__ __forceinline__ int tiles_d(const Params &p) { return (p.L / 128) * ((p.F + kBN - 1) / kBN); }
  static __device__ __forceinline__ void prefetch(const Params &p) {
    prefetch_tmap(&p.tdgu); prefetch_tmap(&p.tz); prefetch_tmap(&p.tdo); prefetch_tmap(&p.th);
    prefetch_tmap(&p.og); prefetch_tmap(&p.ou); prefetch_tmap(&p.od);
  }
  static __device__ __forceinline__ void stage_aux(const Params &p, uint8_t *aux) {
    int *s = reinterpret_cast<int *>(aux);
    for (int i = threadIdx.x; i < p.E + 2; i += blockDim.x) s[i] = __ldg(p.grp_off + i);
  }
  static __device__ __forceinline__ int num_units(const Params &p, const uint8_t *) {
    return (p.E + 1) * (2 * tiles_gu(p) + tiles_d(p));
  }
  static __device__ __forceinline__ int k_blocks(const Params &) { return 0; }  // per unit instead
  // U.g = 3 * group + matrix (0 gate, 1 up, 2 down); U.krows = the group's rows
  static __device__ __forceinline__ Unit unit(const Params &p, int u, const uint8_t *aux) {
    const int *go = reinterpret_cast<const int *>(aux);
    const int tg = tiles_gu(p), per = 2 * tg + tiles_d(p);
    const int g = u / per;
    int r = u - g * per;
    const int which = r < tg ? 0 : (r < 2 * tg ? 1 : 2);
    r -= which * tg;
    const int N = which < 2 ? p.L : p.F;
    const int nt = (N + kBN - 1) / kBN;
    Unit U;
    U.g = 3 * g + which;
    U.m = r / nt;
    U.n0 = (r - U.m * nt) * kBN;
    U.nv = min(kBN, N - U.n0);
    U.row0 = go[g];
    U.krows = go[g + 1] - go[g];
    U.nsub = 1;
    return U;
  }
  static __device__ __forceinline__ int unit_k_blocks(const Params &, const Unit &U) { return (U.krows + kBK - 1) / kBK; }
  static __device__ __forceinline__ int tail_rows(const Params &, const Unit &U) {
    return U.krows - ((U.krows + kBK - 1) / kBK - 1) * kBK;
  }
  // Rows [tail, 64) of every 64-row box of the stage's A and B tiles.
  static __device__ __forceinline__ void zero_tail(const Params &, const Unit &U, uint8_t *a, uint8_t *b, int tail,
                                                   int lane) {
    const int per = (kBK - tail) * 8;  // 16-byte words per box
    const int nb = (U.nv + 63) / 64;
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    for (int box = 0; box < 2 + nb; ++box) {
      uint4 *dst = reinterpret_cast<uint4 *>((box < 2 ? a + box * 8192 : b + (box - 2) * 8192) + tail * 128);
      for (int i = lane; i < per; i += 32) dst[i] = z;
    }
  }
  static __device__ __forceinline__ uint32_t b_bytes(const Params &, const Unit &U, int) {
    return ((U.nv + 63) / 64) * 8192;
  }
  static __device__ __forceinline__ void load_a(const Params &p, const Unit &U, int, int kb, uint32_t sa,
                                                uint32_t bar) {
    const int which = U.g % 3;
    const int y = U.row0 + kb * kBK;
    if (which == 2) {
      load_mn_pair(sa, &p.tdo, bar, U.m * 128, y);
    } else {
      const int plane = (which == 1 ? p.F / 64 : 0) + 2 * U.m;
      tma_load_2d(sa, &p.tdgu, bar, 0, plane * p.rows + y);
      tma_load_2d(sa + 8192, &p.tdgu, bar, 0, (plane + 1) * p.rows + y);
    }
  }
  static __device__ __forceinline__ void load_b(const Params &p, const Unit &U, int, int kb, uint32_t sb,
                                                uint32_t bar) {
    const int which = U.g % 3;
    const int y = U.row0 + kb * kBK;
    for (int i = 0; i * 64 < U.nv; ++i) {
      if (which == 2)
        tma_load_2d(sb + i * 8192, &p.th, bar, 0, (U.n0 / 64 + i) * p.rows + y);
      else
        tma_load_2d(sb + i * 8192, &p.tz, bar, U.n0 + i * 64, y);
    }
  }
  static __device__ __forceinline__ uint32_t idesc(const Params &, const Unit &U, int) {
    return idesc_bf16_major(128, round16(U.nv), true, true);
  }
  static __device__ __forceinline__ void mma(uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
    umma_f16(d, a, b, id, acc);
  }
  // Lane = output row (f for dW_g/dW_u, l for dW_d), columns = the tile's N.
  static __device__ __forceinline__ void epilogue(const Params &p, const Unit &U, int, uint32_t taddr, int q,
                                                  int lane, int, EpiState &st, uint8_t *epi) {
    const int which = U.g % 3, g = U.g / 3;
    const bool sh = g == p.E;
    const CUtensorMap *map = which == 0 ? (sh ? &p.sog : &p.og) : which == 1 ? (sh ? &p.sou : &p.ou)
                                                                               : (sh ? &p.sod : &p.od);
    const int y = (sh ? 0 : g * (which < 2 ? p.F : p.L)) + U.m * 128 + q * 32;
    const uint32_t e0 = smem_u32(epi);
    const uint32_t bufs = ((e0 + 1023u) & ~1023u) + static_cast<uint32_t>(q) * (kStoreBufs * 4096u);
    uint8_t *bufp = epi + (bufs - e0);
    const bool empty = U.krows == 0;
    for (int c0 = 0; c0 < U.nv; c0 += 32) {
      float v[32];
      if (empty) {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.f;
      } else {
        tmem_ld32(taddr + c0, v);
        tmem_ld_wait();
      }
      const int b = st.n & (kStoreBufs - 1);
      if (lane == 0) bulk_wait_read<kStoreBufs - 1>();  // this buffer's previous store has read it
      __syncwarp();
      float4 *row = reinterpret_cast<float4 *>(bufp + b * 4096 + lane * 128);
#pragma unroll
      for (int j = 0; j < 8; ++j)  // 16-byte chunk j of row `lane` sits at chunk j ^ (lane % 8)
        row[j ^ (lane & 7)] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
      fence_proxy_async_shared();
      __syncwarp();
      if (lane == 0) {
        if (p.accumulate)
          tma_reduce_add_2d(map, bufs + b * 4096, U.n0 + c0, y);
        else
          tma_store_2d(map, bufs + b * 4096, U.n0 + c0, y);
        bulk_commit();
      }
      ++st.n;
    }
  }
};

// ------------------------------------------------- per-token kernels
constexpr int kBwdThreads = 256;
constexpr int kBwdMaxV4 = 8192 / 4 / kBwdThreads;  // float4 columns per thread at d_lat <= 8192

__device__ __forceinline__ float block_sum(float v, float *red) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  __syncthreads();  // red is free again
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < kBwdThreads / 32; ++w) tot += red[w];
  return tot;
}

__device__ __forceinline__ uint2 pack_bf16x4(float4 v) {
  return make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
}

// RMSNorm and combine backward, blocks striding over tokens.  Per token:
// c = the slots summed in the forward's order, r = 1/sqrt(mean(c^2) + eps),
// cn = c r, dcn = dn gain, dc = r (dcn - cn mean(cn dcn)); dc goes to every
// dispatch row of the token (dcd: as is; dod: times the row's w'), the
// shared row Tk + t included (weight 1).  gpart[block] = sum over the
// block's tokens of dn cn (the gain's gradient, reduced by gain_reduce_kernel).
// wrow[row] = the row's weight w' (1 for the shared expert's row).
template <int MAXV4>  // float4 columns per thread: d_lat <= 4 * kBwdThreads * MAXV4
__global__ void __launch_bounds__(kBwdThreads) rms_combine_bwd_kernel(
    const float4 *__restrict__ slots, const float4 *__restrict__ dn, const float4 *__restrict__ gain,
    const int32_t *__restrict__ inv, const float *__restrict__ wscaled, int T, int L, int k, float eps,
    __nv_bfloat16 *__restrict__ dcd, __nv_bfloat16 *__restrict__ dod, float *__restrict__ wrow,
    float4 *__restrict__ gpart, const uint32_t *status) {
  __shared__ float red[kBwdThreads / 32];
  if (call_failed(status)) return;
  const int L4 = L >> 2;
  const size_t Tk = static_cast<size_t>(T) * k;
  float4 gacc[MAXV4];
#pragma unroll
  for (int v = 0; v < MAXV4; ++v) gacc[v] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    const float4 *base = slots + static_cast<size_t>(t) * (k + 1) * L4;
    float4 c[MAXV4];
    float ss = 0.f;
#pragma unroll
    for (int v = 0; v < MAXV4; ++v) {
      const int i = threadIdx.x + v * kBwdThreads;
      if (i < L4) {
        float4 a = __ldg(base + i);
#pragma unroll 4
        for (int j = 1; j <= k; ++j) {
          const float4 b = __ldg(base + static_cast<size_t>(j) * L4 + i);
          a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
        }
        c[v] = a;
        ss += a.x * a.x + a.y * a.y + a.z * a.z + a.w * a.w;
      }
    }
    const float r = 1.0f / sqrtf(block_sum(ss, red) / static_cast<float>(L) + eps);
    float4 dcn[MAXV4];
    float dot = 0.f;
#pragma unroll
    for (int v = 0; v < MAXV4; ++v) {
      const int i = threadIdx.x + v * kBwdThreads;
      if (i < L4) {
        const float4 d = __ldg(dn + static_cast<size_t>(t) * L4 + i);
        const float4 g = __ldg(gain + i);
        c[v] = make_float4(c[v].x * r, c[v].y * r, c[v].z * r, c[v].w * r);  // cn
        dcn[v] = make_float4(d.x * g.x, d.y * g.y, d.z * g.z, d.w * g.w);
        dot += c[v].x * dcn[v].x + c[v].y * dcn[v].y + c[v].z * dcn[v].z + c[v].w * dcn[v].w;
        gacc[v].x += d.x * c[v].x; gacc[v].y += d.y * c[v].y;
        gacc[v].z += d.z * c[v].z; gacc[v].w += d.w * c[v].w;
      }
    }
    const float m = block_sum(dot, red) / static_cast<float>(L);
    for (int j = 0; j <= k; ++j) {
      const bool shared = j == k;
      const size_t row = shared ? Tk + t : static_cast<size_t>(__ldg(inv + static_cast<size_t>(t) * k + j));
      const float w = shared ? 1.0f : __ldg(wscaled + static_cast<size_t>(t) * k + j);
      if (threadIdx.x == 0) wrow[row] = w;
      uint2 *d1 = reinterpret_cast<uint2 *>(dcd + row * L);
      uint2 *d2 = reinterpret_cast<uint2 *>(dod + row * L);
#pragma unroll
      for (int v = 0; v < MAXV4; ++v) {
        const int i = threadIdx.x + v * kBwdThreads;
        if (i < L4) {
          const float4 dc = make_float4(r * (dcn[v].x - c[v].x * m), r * (dcn[v].y - c[v].y * m),
                                        r * (dcn[v].z - c[v].z * m), r * (dcn[v].w - c[v].w * m));
          d1[i] = pack_bf16x4(dc);
          d2[i] = pack_bf16x4(make_float4(w * dc.x, w * dc.y, w * dc.z, w * dc.w));
        }
      }
    }
  }
#pragma unroll
  for (int v = 0; v < MAXV4; ++v) {
    const int i = threadIdx.x + v * kBwdThreads;
    if (i < L4) gpart[static_cast<size_t>(blockIdx.x) * L4 + i] = gacc[v];
  }
}

// dgain[l] = sum over blocks b (in order) of gpart[b][l].
__global__ void gain_reduce_kernel(const float *__restrict__ gpart, int nb, int L, float *__restrict__ dgain,
                                   int accumulate, const uint32_t *status) {
  if (call_failed(status)) return;
  const int l = blockIdx.x * blockDim.x + threadIdx.x;
  if (l >= L) return;
  float a = 0.f;
  for (int b = 0; b < nb; ++b) a += __ldg(gpart + static_cast<size_t>(b) * L + l);
  dgain[l] = accumulate ? dgain[l] + a : a;
}

constexpr int kBwdMaxSlices = 64;  // d_ff / 128 at d_ff <= 8192
constexpr int kBwdMaxRouters = 8;

// Router and combine-weight backward plus the reduction of dz, one block per
// token t.  The logits of the k selected experts are recomputed from the
// latent the routers read (zx = z hi + z lo, fp32) as fp32 dot products.
//   dw'_j = sum over d_ff slices of dwsp;  aw_j = w_j dw'_j (for dalpha);
//   dw_j = alpha_{e_j} dw'_j;  ds_j = (dw_j - sum_i w_i dw_i) / sum_i s_i (0 if that sum is 0);
//   dp_{j,r} = ds_j / R (mean), ds_j (sum), ds_j [r = first argmax] (max);
//   dl_{j,r} = dp_{j,r} p_{j,r} (1 - p_{j,r});
//   dzx = sum_{j <= k} dzs[t][j] + sum_{j,r} dl_{j,r} W_router[r, e_j]  (in that order)
// Dynamic shared memory: d_lat floats (zx).
__global__ void __launch_bounds__(kBwdThreads) token_bwd_kernel(
    const float *__restrict__ dwsp, int nsl, int rows, const int32_t *__restrict__ inv,
    const int32_t *__restrict__ topk_idx,
    const float *__restrict__ topk_w, const float *__restrict__ alpha, const __nv_bfloat16 *__restrict__ zhi,
    const __nv_bfloat16 *__restrict__ zlo, const __nv_bfloat16 *__restrict__ wr, const float *__restrict__ dzs,
    int T, int L, int E, int R, int k, int agg, __nv_bfloat16 *__restrict__ dzx, float *__restrict__ dl,
    float *__restrict__ aw, const uint32_t *status) {
  extern __shared__ float zx[];
  __shared__ float part[kTopKMax * kBwdMaxSlices];
  __shared__ float logit[kTopKMax * kBwdMaxRouters];
  __shared__ float coef[kTopKMax * kBwdMaxRouters];
  __shared__ float s_sel[kTopKMax], s_dw[kTopKMax], s_w[kTopKMax], s_tot[2];
  __shared__ int eidx[kTopKMax];
  if (call_failed(status)) return;
  const int t = blockIdx.x;
  const int L8 = L >> 3;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < L8; i += kBwdThreads) {
    const uint4 a = __ldg(reinterpret_cast<const uint4 *>(zhi + static_cast<size_t>(t) * L) + i);
    const uint4 b = __ldg(reinterpret_cast<const uint4 *>(zlo + static_cast<size_t>(t) * L) + i);
    const __nv_bfloat16 *ha = reinterpret_cast<const __nv_bfloat16 *>(&a);
    const __nv_bfloat16 *hb = reinterpret_cast<const __nv_bfloat16 *>(&b);
#pragma unroll
    for (int q = 0; q < 8; ++q) zx[8 * i + q] = __bfloat162float(ha[q]) + __bfloat162float(hb[q]);
  }
  if (threadIdx.x < k) eidx[threadIdx.x] = __ldg(topk_idx + static_cast<size_t>(t) * k + threadIdx.x);
  for (int i = threadIdx.x; i < k * nsl; i += kBwdThreads) {
    const int j = i / nsl, m = i - j * nsl;
    const int row = __ldg(inv + static_cast<size_t>(t) * k + j);
    part[i] = __ldg(dwsp + static_cast<size_t>(m) * rows + row);
  }
  __syncthreads();
  for (int idx = warp; idx < k * R; idx += kBwdThreads / 32) {
    const int j = idx / R, r = idx - j * R;
    const uint4 *row = reinterpret_cast<const uint4 *>(wr + (static_cast<size_t>(r) * E + eidx[j]) * L);
    float a = 0.f;
#pragma unroll 4
    for (int i = lane; i < L8; i += 32) {
      const uint4 v = __ldg(row + i);
      const __nv_bfloat16 *hv = reinterpret_cast<const __nv_bfloat16 *>(&v);
#pragma unroll
      for (int q = 0; q < 8; ++q) a += __bfloat162float(hv[q]) * zx[8 * i + q];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
    if (lane == 0) logit[idx] = a;
  }
  __syncthreads();
  // slot j (thread j): its score s_j, dw'_j, aw_j and dw_j
  if (threadIdx.x < k) {
    const int j = threadIdx.x;
    float sj = 0.f;
    for (int r = 0; r < R; ++r) {
      const float pr = sigmoidf_(logit[j * R + r]);
      sj = agg == 2 ? fmaxf(sj, pr) : sj + pr;
    }
    s_sel[j] = agg == 0 ? sj / static_cast<float>(R) : sj;
    float d = 0.f;
    for (int m = 0; m < nsl; ++m) d += part[j * nsl + m];
    const float wj = __ldg(topk_w + static_cast<size_t>(t) * k + j);
    aw[static_cast<size_t>(t) * k + j] = wj * d;
    s_w[j] = wj;
    s_dw[j] = d * __ldg(alpha + eidx[j]);
  }
  __syncthreads();
  if (threadIdx.x == 0) {  // sums over the slots, in slot order
    float S = 0.f, swdw = 0.f;
    for (int j = 0; j < k; ++j) {
      S += s_sel[j];
      swdw += s_w[j] * s_dw[j];
    }
    s_tot[0] = S;
    s_tot[1] = swdw;
  }
  __syncthreads();
  // (slot j, router r): dl
  if (threadIdx.x < k * R) {
    const int j = threadIdx.x / R, r = threadIdx.x - j * R;
    // selected scores that sum to 0 get the constant weights 1/k: no gradient
    const float ds = s_tot[0] != 0.0f ? (s_dw[j] - s_tot[1]) / s_tot[0] : 0.0f;
    int rmax = 0;
    if (agg == 2)
      for (int q = 1; q < R; ++q)
        if (logit[j * R + q] > logit[j * R + rmax]) rmax = q;
    const float pr = sigmoidf_(logit[j * R + r]);
    const float dp = agg == 0 ? ds / static_cast<float>(R) : (agg == 1 || r == rmax ? ds : 0.f);
    const float d = dp * pr * (1.0f - pr);
    coef[j * R + r] = d;
    dl[(static_cast<size_t>(t) * k + j) * R + r] = d;
  }
  __syncthreads();
  const float *zs = dzs + static_cast<size_t>(t) * (k + 1) * L;
  for (int i = threadIdx.x; i < L8; i += kBwdThreads) {
    float a[8];
    {
      const float4 x0 = __ldg(reinterpret_cast<const float4 *>(zs) + 2 * i);
      const float4 x1 = __ldg(reinterpret_cast<const float4 *>(zs) + 2 * i + 1);
      a[0] = x0.x; a[1] = x0.y; a[2] = x0.z; a[3] = x0.w; a[4] = x1.x; a[5] = x1.y; a[6] = x1.z; a[7] = x1.w;
    }
#pragma unroll 4
    for (int j = 1; j <= k; ++j) {
      const float4 *src = reinterpret_cast<const float4 *>(zs + static_cast<size_t>(j) * L) + 2 * i;
      const float4 x0 = __ldg(src), x1 = __ldg(src + 1);
      a[0] += x0.x; a[1] += x0.y; a[2] += x0.z; a[3] += x0.w; a[4] += x1.x; a[5] += x1.y; a[6] += x1.z; a[7] += x1.w;
    }
#pragma unroll 8
    for (int jr = 0; jr < k * R; ++jr) {
      const int j = jr / R, r = jr - j * R;
      const uint4 v = __ldg(reinterpret_cast<const uint4 *>(wr + (static_cast<size_t>(r) * E + eidx[j]) * L) + i);
      const __nv_bfloat16 *hv = reinterpret_cast<const __nv_bfloat16 *>(&v);
      const float cf = coef[jr];
#pragma unroll
      for (int q = 0; q < 8; ++q) a[q] += cf * __bfloat162float(hv[q]);
    }
    uint4 o;
    o.x = pack_bf16x2(a[0], a[1]);
    o.y = pack_bf16x2(a[2], a[3]);
    o.z = pack_bf16x2(a[4], a[5]);
    o.w = pack_bf16x2(a[6], a[7]);
    reinterpret_cast<uint4 *>(dzx + static_cast<size_t>(t) * L)[i] = o;
  }
}

// Per expert e (one block): dalpha[e] = sum over e's dispatch rows of aw,
// dW_router[r, e, :] = sum over e's rows (ascending, as in the dispatch
// record) of dl[row, r] zx[t(row)].
__global__ void __launch_bounds__(kBwdThreads, 2) expert_param_bwd_kernel(
    const int32_t *__restrict__ grp_off, const int32_t *__restrict__ grp_cnt, const int32_t *__restrict__ perm,
    const float *__restrict__ dl, const float *__restrict__ aw, const __nv_bfloat16 *__restrict__ zhi,
    const __nv_bfloat16 *__restrict__ zlo, int L, int E, int R, int k, float *__restrict__ dwr,
    float *__restrict__ dalpha, int accumulate, const uint32_t *status) {
  __shared__ float red[kBwdThreads / 32];
  if (call_failed(status)) return;
  const int e = blockIdx.x;
  const int r0 = __ldg(grp_off + e), n = __ldg(grp_cnt + e);
  float a = 0.f;
  for (int i = threadIdx.x; i < n; i += kBwdThreads) a += __ldg(aw + __ldg(perm + r0 + i));
  a = block_sum(a, red);
  if (threadIdx.x == 0) dalpha[e] = accumulate ? dalpha[e] + a : a;
  const int L8 = L >> 3;
  for (int c = threadIdx.x; c < L8; c += kBwdThreads) {
    float acc[kBwdMaxRouters][8];
#pragma unroll
    for (int r = 0; r < kBwdMaxRouters; ++r)
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[r][q] = 0.f;
#pragma unroll 4
    for (int i = 0; i < n; ++i) {
      const int flat = __ldg(perm + r0 + i);
      const size_t t = static_cast<size_t>(flat / k);
      const uint4 hv = __ldg(reinterpret_cast<const uint4 *>(zhi + t * L) + c);
      const uint4 lv = __ldg(reinterpret_cast<const uint4 *>(zlo + t * L) + c);
      const __nv_bfloat16 *h8 = reinterpret_cast<const __nv_bfloat16 *>(&hv);
      const __nv_bfloat16 *l8 = reinterpret_cast<const __nv_bfloat16 *>(&lv);
      float z[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) z[q] = __bfloat162float(h8[q]) + __bfloat162float(l8[q]);
#pragma unroll
      for (int r = 0; r < kBwdMaxRouters; ++r) {
        if (r < R) {
          const float d = __ldg(dl + static_cast<size_t>(flat) * R + r);
#pragma unroll
          for (int q = 0; q < 8; ++q) acc[r][q] += d * z[q];
        }
      }
    }
#pragma unroll
    for (int r = 0; r < kBwdMaxRouters; ++r) {
      if (r < R) {
        float4 *dst = reinterpret_cast<float4 *>(dwr + (static_cast<size_t>(r) * E + e) * L + 8 * c);
        if (accumulate) {
          const float4 o0 = dst[0], o1 = dst[1];
          acc[r][0] += o0.x; acc[r][1] += o0.y; acc[r][2] += o0.z; acc[r][3] += o0.w;
          acc[r][4] += o1.x; acc[r][5] += o1.y; acc[r][6] += o1.z; acc[r][7] += o1.w;
        }
        dst[0] = make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
        dst[1] = make_float4(acc[r][4], acc[r][5], acc[r][6], acc[r][7]);
      }
    }
  }
}

}  // namespace mrl
