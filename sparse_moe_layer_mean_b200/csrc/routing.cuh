// routing.cuh — dispatch-record kernels: top-k from given scores, the
// per-chunk expert bitmask histogram, the exclusive scans, the stable
// scatter, the row gather, the fixed-order combine + RMSNorm and the
// balancing-bias step.  No atomics decide any output order.
#pragma once
#include "common.cuh"
#include "topk.cuh"

namespace mrl {

constexpr int kChunk = 32;  // tokens per histogram chunk (one warp, one bit per token)

// ---------------------------------------------------------------------------
// The selection of one token by one warp: lane l has offered experts
// l, l+32, ... (ascending) to its running list; k rounds of a warp arg-max
// (larger biased score, then lower index) emit the selection in rank order,
// and lane 0 writes it with its weights.
template <int KMAX>
__device__ __forceinline__ void warp_select_and_write(TopK<KMAX> &tk, int k, int E, int lane, size_t t,
                                                      const float *__restrict__ alpha, int32_t *__restrict__ topk_idx,
                                                      float *__restrict__ topk_w, float *__restrict__ wscaled,
                                                      uint32_t *status) {
  float sel_s[KMAX];
  int sel_i[KMAX];
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    if (j < k) {
      float bv = tk.v[0], bs = tk.s[0];
      int bi = tk.i[0];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
        const float os = __shfl_xor_sync(0xffffffffu, bs, off);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
        if (ranks_before(ov, oi, bv, bi)) { bv = ov; bs = os; bi = oi; }
      }
      if (tk.i[0] == bi) tk.pop();
      sel_s[j] = bs;
      sel_i[j] = bi;
    }
  }
  if (lane == 0) write_selection<KMAX>(sel_s, sel_i, k, E, t, alpha, topk_idx, topk_w, wscaled, status);
}

// Top-k from caller-given fp32 scores s [T, E]: one warp per token (see
// warp_select_and_write).  sb = s + bias is one fp32 add, as in the CPU
// definition.
template <int KMAX>
__global__ void topk_from_scores_kernel(const float *__restrict__ s, const float *__restrict__ bias,
                                        const float *__restrict__ alpha, int T, int E, int k,
                                        int32_t *__restrict__ topk_idx, float *__restrict__ topk_w,
                                        float *__restrict__ wscaled, uint32_t *status) {
  if (call_failed(status)) return;  // an earlier kernel of the call failed
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= T) return;
  TopK<KMAX> tk;
  tk.init();
  const float *row = s + static_cast<size_t>(warp) * E;
  for (int e = lane; e < E; e += 32) {
    const float sv = __ldg(row + e);
    tk.offer(sv + __ldg(bias + e), e, sv);
  }
  warp_select_and_write<KMAX>(tk, k, E, lane, static_cast<size_t>(warp), alpha, topk_idx, topk_w, wscaled, status);
}

// Scores of the K-split router: part[ks][t][r*E + e] holds router r's logit
// of expert e for token t over the ks-th K range.  One thread per (t, e):
// each logit is the sum of its K ranges in order, then s[t*E + e] = the
// aggregation (over r in order) of the routers' sigmoids, as in the router
// GEMM's epilogue.  topk_from_scores_kernel then selects from s + bias.
__global__ void router_split_scores_kernel(const float *__restrict__ part, int ksplit, int T, int E, int R, int agg,
                                           float *__restrict__ s, const uint32_t *status) {
  if (call_failed(status)) return;  // an earlier kernel of the call failed
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<long long>(T) * E) return;
  const int t = static_cast<int>(i / E), e = static_cast<int>(i - static_cast<long long>(t) * E);
  const size_t RE = static_cast<size_t>(R) * E;
  const size_t plane = static_cast<size_t>(T) * RE;
  const float *l0 = part + static_cast<size_t>(t) * RE + e;
  float acc = 0.f;
  for (int r = 0; r < R; ++r) {
    const float *l = l0 + static_cast<size_t>(r) * E;
    float logit = __ldg(l);
    for (int ks = 1; ks < ksplit; ++ks) logit += __ldg(l + ks * plane);
    const float sg = sigmoidf_(logit);
    acc = agg == 2 ? fmaxf(acc, sg) : acc + sg;  // sigmoid >= 0
  }
  s[i] = agg != 0 ? acc : (R & (R - 1)) == 0 ? acc * (1.0f / static_cast<float>(R)) : acc / static_cast<float>(R);
}

// Merge of the router's partial selections: part p of token t left its best k
// candidates (biased score, score, expert) at [(t * parts + p) * k + j].
// One thread per token keeps the best k of all parts (same ranking rule).
template <int KMAX>
__global__ void topk_merge_kernel(const float *__restrict__ cand_v, const float *__restrict__ cand_s,
                                  const int32_t *__restrict__ cand_i, int T, int E, int parts, int k,
                                  const float *__restrict__ alpha, int32_t *__restrict__ topk_idx,
                                  float *__restrict__ topk_w, float *__restrict__ wscaled,
                                  uint32_t *status) {
  if (call_failed(status)) return;  // an earlier kernel of the call failed
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  TopK<KMAX> tk;
  tk.init();
  const size_t base = static_cast<size_t>(t) * parts * k;
  for (int c = 0; c < parts * k; ++c)
    topk_offer_any<KMAX>(tk, __ldg(cand_v + base + c), __ldg(cand_i + base + c), __ldg(cand_s + base + c));
  write_selection<KMAX>(tk.s, tk.i, k, E, static_cast<size_t>(t), alpha, topk_idx, topk_w, wscaled, status);
}

// ---------------------------------------------------------------------------
// Histogram: for chunk c (tokens 32c .. 32c+31) and expert e, mask[c*E + e]
// has bit i set iff token 32c+i selected e.  One warp per chunk; the warp's
// table lives in shared memory (E <= 1024 words).  An expert index outside
// [0, E) is never used: it records DEV_CHECK, so the kernels after this one
// do nothing.
__global__ void expert_mask_kernel(const int32_t *__restrict__ topk_idx, int T, int E, int k,
                                   uint32_t *__restrict__ mask, int nchunks, uint32_t *status) {
  extern __shared__ uint32_t tab_all[];
  if (call_failed(status)) return;  // an earlier kernel of the call failed
  const int wib = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int c = blockIdx.x * (blockDim.x >> 5) + wib;
  if (c >= nchunks) return;
  uint32_t *tab = tab_all + wib * E;
  for (int e = lane; e < E; e += 32) tab[e] = 0u;
  __syncwarp();
  const int t = c * kChunk + lane;
  bool bad = false;
  if (t < T)
    for (int j = 0; j < k; ++j) {
      const int e = __ldg(topk_idx + static_cast<size_t>(t) * k + j);
      if (static_cast<unsigned>(e) < static_cast<unsigned>(E))
        atomicOr(&tab[e], 1u << lane);
      else
        bad = true;
    }
  if (bad && status) atomicCAS(status, DEV_OK, DEV_CHECK);
  __syncwarp();
  uint32_t *dst = mask + static_cast<size_t>(c) * E;
  for (int e = lane; e < E; e += 32) dst[e] = tab[e];
}

// Column scan: base[c*E + e] = sum over chunks c' < c of popc(mask[c'*E + e]);
// counts[e] = total.  Block (32 x 32): lane = expert of a 32-expert group,
// warp = a contiguous run of chunks.
__global__ void expert_colscan_kernel(const uint32_t *__restrict__ mask, int E, int nchunks,
                                      int32_t *__restrict__ base, int32_t *__restrict__ counts,
                                      const uint32_t *status) {
  __shared__ int tot[32][33];
  if (call_failed(status)) return;  // an earlier kernel of the call failed
  const int lane = threadIdx.x & 31;
  const int w = threadIdx.x >> 5;
  const int e = blockIdx.x * 32 + lane;
  const int cpw = (nchunks + 31) / 32;
  const int c0 = w * cpw, c1 = min(nchunks, c0 + cpw);
  int sum = 0;
  if (e < E)
    for (int c = c0; c < c1; ++c) sum += __popc(__ldg(mask + static_cast<size_t>(c) * E + e));
  tot[w][lane] = sum;
  __syncthreads();
  int run = 0;
  for (int i = 0; i < w; ++i) run += tot[i][lane];
  if (e < E) {
    for (int c = c0; c < c1; ++c) {
      base[static_cast<size_t>(c) * E + e] = run;
      run += __popc(__ldg(mask + static_cast<size_t>(c) * E + e));
    }
    if (w == 31) counts[e] = run;
  }
}

// Block-wide exclusive scan of one int per thread (blockDim.x == 1024).
__device__ __forceinline__ int block_excl_scan(int v, int *warp_tot, int *total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) warp_tot[w] = x;
  __syncthreads();
  if (w == 0) {
    int t = warp_tot[lane];
    int ti = t;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, ti, off);
      if (lane >= off) ti += y;
    }
    warp_tot[lane] = ti - t;  // exclusive prefix of warps
    if (lane == 31) *total = ti;
  }
  __syncthreads();
  const int r = warp_tot[w] + x - v;
  __syncthreads();
  return r;
}

// Offsets and the grouped-GEMM tables.  Group g < E is routed expert g
// (rows offsets[g] .. + counts[g]); group E is the shared expert over all T
// tokens, whose rows start at T*k.  unit_off{1,2}[g] = exclusive prefix of
// m_tiles{1,2} * ceil(cnt_g / BN).  Single block of 1024 threads (E <= 1024).
__global__ void expert_offsets_kernel(const int32_t *__restrict__ counts_in, int T, int E, int k, int BN,
                                      int mt1, int mt2, int32_t *__restrict__ grp_off,
                                      int32_t *__restrict__ grp_cnt, int32_t *__restrict__ unit1,
                                      int32_t *__restrict__ unit2, int32_t *__restrict__ out_counts,
                                      int32_t *__restrict__ out_offsets, const uint32_t *status) {
  __shared__ int wt[32];
  if (call_failed(status)) return;  // an earlier kernel of the call failed
  __shared__ int tot[3];
  const int e = threadIdx.x;
  const int cnt = e < E ? counts_in[e] : 0;
  const int nt = (cnt + BN - 1) / BN;
  const int off = block_excl_scan(cnt, wt, &tot[0]);
  const int u1 = block_excl_scan(nt * mt1, wt, &tot[1]);
  const int u2 = block_excl_scan(nt * mt2, wt, &tot[2]);
  if (e < E) {
    grp_off[e] = off;
    grp_cnt[e] = cnt;
    unit1[e] = u1;
    unit2[e] = u2;
    if (out_counts) out_counts[e] = cnt;
    if (out_offsets) out_offsets[e] = off;
  }
  if (e == 0) {
    const int ntS = (T + BN - 1) / BN;
    grp_off[E] = T * k;
    grp_cnt[E] = T;
    grp_off[E + 1] = T * k + T;
    grp_cnt[E + 1] = 0;
    unit1[E] = tot[1];
    unit2[E] = tot[2];
    unit1[E + 1] = tot[1] + ntS * mt1;
    unit2[E + 1] = tot[2] + ntS * mt2;
    if (out_offsets) out_offsets[E] = tot[0];
  }
}

// Stable scatter: entry (t, j) with expert e goes to row
// offsets[e] + base[c*E + e] + popc(mask[c*E + e] & lanes below t's lane):
// expert-major, ascending tokens within an expert.  An index outside [0, E)
// is skipped and records DEV_CHECK (the mask kernel has already refused it,
// so this kernel only runs on a record it accepted; the check keeps every
// access in bounds on its own).
__global__ void expert_scatter_kernel(const int32_t *__restrict__ topk_idx, const uint32_t *__restrict__ mask,
                                      const int32_t *__restrict__ base, const int32_t *__restrict__ offsets,
                                      int T, int E, int k, int nchunks, int32_t *__restrict__ perm,
                                      int32_t *__restrict__ inv_perm, uint32_t *status) {
  if (call_failed(status)) return;  // an earlier kernel of the call failed
  const int c = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (c >= nchunks) return;
  const int t = c * kChunk + lane;
  if (t >= T) return;
  const uint32_t below = (1u << lane) - 1u;
  for (int j = 0; j < k; ++j) {
    const int flat = t * k + j;
    const int e = __ldg(topk_idx + flat);
    if (static_cast<unsigned>(e) >= static_cast<unsigned>(E)) {
      if (status) atomicCAS(status, DEV_OK, DEV_CHECK);
      continue;
    }
    const size_t ce = static_cast<size_t>(c) * E + e;
    const int row = __ldg(offsets + e) + __ldg(base + ce) + __popc(__ldg(mask + ce) & below);
    perm[row] = flat;
    inv_perm[flat] = row;
  }
}

// Dispatch-row copy: zd[inv[t*k + j]] = zs[t] for j < k.  Warp w takes token
// t = w / nsplit and its destinations j = w % nsplit, + nsplit, ...: it reads
// the token's row, 32 lanes x kCopyU4 uint4 at a time, and writes each chunk
// to those dispatch rows (lane j < k holds the row of (t, j)), so the stores
// of a chunk are in flight behind one round of loads.  nsplit = 1 reads each
// row once; a small batch takes nsplit > 1 to occupy more warps.  A row
// index outside [0, rows) is skipped.
constexpr int kCopyWarps = 8;
constexpr int kCopyU4 = 8;

__global__ void __launch_bounds__(kCopyWarps * 32) copy_dispatch_rows_kernel(
    const uint4 *__restrict__ zs, int T, int row_u4, const int32_t *__restrict__ inv, int k, int nsplit,
    int rows, uint4 *__restrict__ zd, const uint32_t *status) {
  if (call_failed(status)) return;  // an earlier kernel of the call failed
  const int w = blockIdx.x * kCopyWarps + (threadIdx.x >> 5);
  const int t = w / nsplit, part = w - t * nsplit;
  if (t >= T) return;  // whole warps leave together
  const int lane = threadIdx.x & 31;
  const int my_row = lane < k ? __ldg(inv + static_cast<size_t>(t) * k + lane) : -1;
  const uint4 *src = zs + static_cast<size_t>(t) * row_u4;
  for (int c0 = 0; c0 < row_u4; c0 += 32 * kCopyU4) {
    uint4 v[kCopyU4];
#pragma unroll
    for (int j = 0; j < kCopyU4; ++j) {
      const int i = c0 + j * 32 + lane;
      v[j] = i < row_u4 ? __ldg(src + i) : make_uint4(0u, 0u, 0u, 0u);
    }
    for (int d = part; d < k; d += nsplit) {
      const int r = __shfl_sync(0xffffffffu, my_row, d);
      if (r < 0 || r >= rows) continue;  // uniform across the warp
      uint4 *dst = zd + static_cast<size_t>(r) * row_u4;
#pragma unroll
      for (int j = 0; j < kCopyU4; ++j) {
        const int i = c0 + j * 32 + lane;
        if (i < row_u4) dst[i] = v[j];
      }
    }
  }
}

// ---------------------------------------------------------------------------
// FP8 activation quantiser, one warp per row, a half-warp per 128-wide K
// block (16 lanes x 8 bf16: 16-byte loads, 8-byte code stores): amax over the
// block's bf16 values; amax == 0 -> scale 1, codes 0; else scale = amax / 448
// and code = e4m3_rn_satfinite(v * (448 / amax)) (fp32 IEEE ops).
__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));  // first source -> upper byte
  return r;
}

constexpr int kQuantWarps = 8;
constexpr int kQuantBatch = 4;   // warp iterations whose loads are in flight together

// One 128-wide block, quantised by a half-warp: lane hl of the half holds
// elements 8 hl .. 8 hl + 7 in raw and gets their 8 codes; every lane of the
// half gets the block's scale.  (The amax reduction stays within the half.)
__device__ __forceinline__ void quant_block128(uint4 raw, uint2 &codes, float &scale) {
  float v[8];
  const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __low2float(h2[i]);
    v[2 * i + 1] = __high2float(h2[i]);
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
  for (int off = 8; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  float inv = 0.0f;
  scale = 1.0f;
  if (amax != 0.0f) {
    scale = amax / 448.0f;
    inv = 448.0f / amax;
  }
  codes.x = static_cast<uint32_t>(e4m3x2(v[0] * inv, v[1] * inv)) |
            (static_cast<uint32_t>(e4m3x2(v[2] * inv, v[3] * inv)) << 16);
  codes.y = static_cast<uint32_t>(e4m3x2(v[4] * inv, v[5] * inv)) |
            (static_cast<uint32_t>(e4m3x2(v[6] * inv, v[7] * inv)) << 16);
}

// Rows of in [rows, K] to codes q [rows, K] and scales s[r][K/128] (s_ld ==
// 0) or, transposed, s[b * s_ld + r].  A warp's loads are issued kQuantBatch
// iterations (8 blocks) at a time before those blocks are reduced, so a warp
// waits for memory once per 8 blocks while the block keeps few registers
// (and many warps per SM).
__global__ void __launch_bounds__(kQuantWarps * 32) quant_rows_kernel(
    const __nv_bfloat16 *__restrict__ in, long ld_in, int rows, int K, uint8_t *__restrict__ q,
    float *__restrict__ s, long s_ld, const uint32_t *status) {
  if (call_failed(status)) return;  // an earlier kernel of the call failed
  const int kbs = K >> 7;
  const int r = blockIdx.x * kQuantWarps + (threadIdx.x >> 5);
  if (r >= rows) return;  // whole warps leave together
  const int lane = threadIdx.x & 31;
  const int half = lane >> 4, hl = lane & 15;
  const __nv_bfloat16 *row_in = in + static_cast<long>(r) * ld_in;
  uint8_t *row_q = q + static_cast<long>(r) * K;
  for (int it0 = 0; 2 * it0 < kbs; it0 += kQuantBatch) {
    uint4 raw[kQuantBatch];
#pragma unroll
    for (int j = 0; j < kQuantBatch; ++j) {
      const int b = 2 * (it0 + j) + half;
      raw[j] = b < kbs ? __ldg(reinterpret_cast<const uint4 *>(row_in + b * 128 + hl * 8)) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int j = 0; j < kQuantBatch; ++j) {
      if (2 * (it0 + j) >= kbs) break;  // uniform across the warp
      const int b = 2 * (it0 + j) + half;
      uint2 codes;
      float scale;
      quant_block128(raw[j], codes, scale);
      if (b < kbs) {
        *reinterpret_cast<uint2 *>(row_q + b * 128 + hl * 8) = codes;
        if (hl == 0) s[s_ld ? b * s_ld + r : static_cast<long>(r) * kbs + b] = scale;
      }
    }
  }
}

// The FP8 variant's quantised dispatch rows: one warp per token t quantises
// its latent row z[t] once (the arithmetic above, so every copy holds the
// codes and scales that quantising it would give) and writes them to each of
// the token's k dispatch rows inv[t k + j] and to its shared-expert row
// Tk + t; scales transposed, s[b * s_ld + row].  Each latent row is read
// once instead of once per dispatch row.
__global__ void __launch_bounds__(kQuantWarps * 32) quant_dispatch_rows_kernel(
    const __nv_bfloat16 *__restrict__ z, int T, int K, const int32_t *__restrict__ inv, int k, int Tk,
    uint8_t *__restrict__ q, float *__restrict__ s, long s_ld, const uint32_t *status) {
  if (call_failed(status)) return;  // an earlier kernel of the call failed
  const int kbs = K >> 7;
  const int t = blockIdx.x * kQuantWarps + (threadIdx.x >> 5);
  if (t >= T) return;  // whole warps leave together
  const int lane = threadIdx.x & 31;
  const int half = lane >> 4, hl = lane & 15;
  // lane j < k holds the dispatch row of (t, j)
  const int my_row = lane < k ? __ldg(inv + static_cast<size_t>(t) * k + lane) : -1;
  const __nv_bfloat16 *row_in = z + static_cast<size_t>(t) * K;
  for (int it0 = 0; 2 * it0 < kbs; it0 += kQuantBatch) {
    uint4 raw[kQuantBatch];
#pragma unroll
    for (int j = 0; j < kQuantBatch; ++j) {
      const int b = 2 * (it0 + j) + half;
      raw[j] = b < kbs ? __ldg(reinterpret_cast<const uint4 *>(row_in + b * 128 + hl * 8)) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int j = 0; j < kQuantBatch; ++j) {
      if (2 * (it0 + j) >= kbs) break;  // uniform across the warp
      const int b = 2 * (it0 + j) + half;
      uint2 codes;
      float scale;
      quant_block128(raw[j], codes, scale);
      for (int d = 0; d <= k; ++d) {
        const int r = d < k ? __shfl_sync(0xffffffffu, my_row, d) : Tk + t;
        if (b < kbs && r >= 0 && r < Tk + T) {
          *reinterpret_cast<uint2 *>(q + static_cast<size_t>(r) * K + b * 128 + hl * 8) = codes;
          if (hl == 0) s[b * s_ld + r] = scale;
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Combine + RMSNorm, one block (256 threads) per token:
//   c = slot[t,0] + slot[t,1] + ... + slot[t,k-1] + slot[t,k]   (rank order, then shared)
//   n = bf16(c * (1 / sqrt(mean(c^2) + eps)) * gain)
// All sums run in a fixed order, so the result is bitwise reproducible.
constexpr int kCombineThreads = 256;
constexpr int kCombineMaxV4 = 8;  // d_lat <= 8192

// The RMSNorm half of a combine kernel: c[v] holds the thread's float4s of
// token t's combined row (element i = threadIdx.x + v * kCombineThreads);
// sum of squares in a fixed order (per thread, then warp tree, then warps in
// order), n = bf16(c * (1 / sqrt(mean(c^2) + eps)) * gain).
template <int NV>
__device__ __forceinline__ void rmsnorm_row(const float4 (&c)[NV], int L, float eps,
                                            const float4 *__restrict__ gain, __nv_bfloat16 *__restrict__ n_row,
                                            float *red) {
  const int L4 = L >> 2;
  float ss = 0.f;
#pragma unroll
  for (int v = 0; v < NV; ++v) {
    const int i = threadIdx.x + v * kCombineThreads;
    if (i < L4) ss += c[v].x * c[v].x + c[v].y * c[v].y + c[v].z * c[v].z + c[v].w * c[v].w;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < kCombineThreads / 32; ++w) tot += red[w];
  const float inv = 1.0f / sqrtf(tot / static_cast<float>(L) + eps);
  uint2 *dst = reinterpret_cast<uint2 *>(n_row);
#pragma unroll
  for (int v = 0; v < NV; ++v) {
    const int i = threadIdx.x + v * kCombineThreads;
    if (i < L4) {
      const float4 g = __ldg(gain + i);
      uint2 o;
      o.x = pack_bf16x2(c[v].x * inv * g.x, c[v].y * inv * g.y);
      o.y = pack_bf16x2(c[v].z * inv * g.z, c[v].w * inv * g.w);
      dst[i] = o;
    }
  }
}

// NV = float4s per thread (L <= 4 * 256 * NV).  The k + 1 slot loads of a
// thread are issued in batches of kJ per float4 before they are added, so
// several loads are in flight per thread; the adds keep the slot order.
template <int NV>
__global__ void __launch_bounds__(kCombineThreads) combine_rmsnorm_kernel(
    const float4 *__restrict__ slots, int L, int k, float eps, const float4 *__restrict__ gain,
    __nv_bfloat16 *__restrict__ n, const uint32_t *status) {
  constexpr int kJ = NV >= 8 ? 1 : 8 / NV;
  __shared__ float red[kCombineThreads / 32];
  if (call_failed(status)) return;  // an earlier kernel of the call failed
  const int t = blockIdx.x;
  const int L4 = L >> 2;
  const float4 *base = slots + static_cast<size_t>(t) * (k + 1) * L4;
  float4 c[NV];
#pragma unroll
  for (int v = 0; v < NV; ++v) {
    const int i = threadIdx.x + v * kCombineThreads;
    c[v] = i < L4 ? __ldg(base + i) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (int j0 = 1; j0 <= k; j0 += kJ) {
    float4 b[NV][kJ];
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      const int i = threadIdx.x + v * kCombineThreads;
#pragma unroll
      for (int jj = 0; jj < kJ; ++jj)
        b[v][jj] = i < L4 && j0 + jj <= k ? __ldg(base + static_cast<size_t>(j0 + jj) * L4 + i)
                                          : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int v = 0; v < NV; ++v) {
#pragma unroll
      for (int jj = 0; jj < kJ; ++jj) {
        if (j0 + jj <= k) {
          c[v].x += b[v][jj].x; c[v].y += b[v][jj].y; c[v].z += b[v][jj].z; c[v].w += b[v][jj].w;
        }
      }
    }
  }
  rmsnorm_row(c, L, eps, gain, n + static_cast<size_t>(t) * L, red);
}

// bias[e] += gamma * sgn(T*k - E*counts[e]) (exact integer sign; sign(0) = 0).
__global__ void bias_update_kernel(const int32_t *__restrict__ counts, float *__restrict__ bias, int E,
                                   long long Tk, float gamma) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= E) return;
  const long long d = Tk - static_cast<long long>(E) * counts[e];
  const float sgn = d > 0 ? 1.0f : (d < 0 ? -1.0f : 0.0f);
  bias[e] = bias[e] + gamma * sgn;
}

}  // namespace mrl
