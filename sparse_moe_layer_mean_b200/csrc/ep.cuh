// ep.cuh — kernels of the expert-parallel form of the layer: the routed
// experts are spread over n ranks (rank d owns E/n consecutive experts), each
// rank routes its own tokens, ships every dispatched latent row to the owner
// of its expert, and gets the unweighted expert outputs back.  The pages give
// the motivation, not a layout: the experts compute in the 2048-d latent so
// that what crosses between GPUs is latent-wide (blog.derekhsu.net,
// "ERNIE-5.5-Flash-Base", section "多路由潛在 MoE (Multi-Router Latent MoE)").
//
// On the owner, the rows arrive source by source (sources in rank order),
// each source's block expert-major for the owner's experts.  The grouped
// GEMMs want every expert's rows in one run, so the owner first copies them
// expert-major (sources in rank order inside an expert: the order the
// single-GPU layer would have if the sources' tokens were one batch), keeps
// the map back to the arrival position, and the down GEMM's epilogue stores
// each output row at that position.  On the source, the returned rows are in
// its own dispatch order again, and the combine weights them and adds them in
// the single-GPU layer's order.
#pragma once
#include "common.cuh"
#include "routing.cuh"

namespace mrl {

constexpr int kEpMaxRanks = 64;

// Layout of the received rows, one block of 1024 threads (thread = local
// expert e < E_loc <= 1024):
//   cnt[e]            = sum over sources of recv_counts[s * E_loc + e]
//   grp_off/grp_cnt   = the expert-major groups (exclusive scan of cnt); group
//                       E_loc is an empty shared-expert group ending at n_recv
//   unit1/unit2       = units of the two grouped GEMMs (m tiles x token tiles)
//   src[s * E_loc + e] = arrival position of source s's rows of expert e
//   dst[s * E_loc + e] = their expert-major position
// The counts come from other ranks: a negative count, or counts that do not
// add up to n_recv, record DEV_CHECK and leave every table unwritten.
__global__ void __launch_bounds__(1024) ep_layout_kernel(const int32_t *__restrict__ recv_counts, int n_src,
                                                         int E_loc, int n_recv, int BN, int mt1, int mt2,
                                                         int32_t *__restrict__ grp_off, int32_t *__restrict__ grp_cnt,
                                                         int32_t *__restrict__ unit1, int32_t *__restrict__ unit2,
                                                         int32_t *__restrict__ src, int32_t *__restrict__ dst,
                                                         uint32_t *status) {
  __shared__ int wt[32];
  __shared__ int tot[4];
  __shared__ long long s_sum;
  __shared__ int s_bad;
  __shared__ int s_base;  // arrival position of the current source's first row
  if (call_failed(status)) return;
  const int e = threadIdx.x;
  if (e == 0) {
    s_sum = 0;
    s_bad = 0;
  }
  __syncthreads();
  long long cnt = 0;
  if (e < E_loc)
    for (int s = 0; s < n_src; ++s) {
      const int c = __ldg(recv_counts + s * E_loc + e);
      if (c < 0) s_bad = 1;
      cnt += c;
    }
  if (e < E_loc) atomicAdd(reinterpret_cast<unsigned long long *>(&s_sum), static_cast<unsigned long long>(cnt));
  __syncthreads();
  if (s_bad || s_sum != n_recv) {
    if (e == 0 && status) atomicCAS(status, DEV_OK, DEV_CHECK);
    return;
  }
  const int c = static_cast<int>(cnt);
  const int nt = (c + BN - 1) / BN;
  const int off = block_excl_scan(c, wt, &tot[0]);
  const int u1 = block_excl_scan(nt * mt1, wt, &tot[1]);
  const int u2 = block_excl_scan(nt * mt2, wt, &tot[2]);
  if (e < E_loc) {
    grp_off[e] = off;
    grp_cnt[e] = c;
    unit1[e] = u1;
    unit2[e] = u2;
  }
  if (e == 0) {
    grp_off[E_loc] = n_recv;
    grp_cnt[E_loc] = 0;
    grp_off[E_loc + 1] = n_recv;
    grp_cnt[E_loc + 1] = 0;
    unit1[E_loc] = unit1[E_loc + 1] = tot[1];
    unit2[E_loc] = unit2[E_loc + 1] = tot[2];
    s_base = 0;
  }
  __syncthreads();
  int run = off;  // expert-major position of the next source's rows of expert e
  for (int s = 0; s < n_src; ++s) {
    const int cs = e < E_loc ? __ldg(recv_counts + s * E_loc + e) : 0;
    const int pre = block_excl_scan(cs, wt, &tot[3]);
    if (e < E_loc) {
      src[s * E_loc + e] = s_base + pre;
      dst[s * E_loc + e] = run;
    }
    run += cs;
    __syncthreads();
    if (e == 0) s_base += tot[3];
    __syncthreads();
  }
}

// One block per (source, local expert): copies that run of received rows to
// its expert-major position and records, for each expert-major row, the
// arrival position its output goes back to.  Rows of d_lat bf16 (uint4s); a
// thread moves four uint4s per pass, loads first, so four are in flight.
__global__ void ep_gather_kernel(const uint4 *__restrict__ recv, int row_u4, const int32_t *__restrict__ recv_counts,
                                 const int32_t *__restrict__ src, const int32_t *__restrict__ dst,
                                 uint4 *__restrict__ rows, int32_t *__restrict__ out_row, const uint32_t *status) {
  if (call_failed(status)) return;
  const int pe = blockIdx.x;
  const int n = __ldg(recv_counts + pe);
  const int a = __ldg(src + pe), b = __ldg(dst + pe);
  for (int i = threadIdx.x; i < n; i += blockDim.x) out_row[b + i] = a + i;
  const long long total = static_cast<long long>(n) * row_u4;
  const uint4 *from = recv + static_cast<size_t>(a) * row_u4;
  uint4 *to = rows + static_cast<size_t>(b) * row_u4;
  const long long bd = blockDim.x;
  long long i = threadIdx.x;
  for (; i + 3 * bd < total; i += 4 * bd) {
    const uint4 v0 = __ldg(from + i), v1 = __ldg(from + i + bd), v2 = __ldg(from + i + 2 * bd),
                v3 = __ldg(from + i + 3 * bd);
    to[i] = v0;
    to[i + bd] = v1;
    to[i + 2 * bd] = v2;
    to[i + 3 * bd] = v3;
  }
  for (; i < total; i += bd) to[i] = __ldg(from + i);
}

// Combine on the source rank from the returned rows (dispatch order) and the
// shared expert's slot:
//   c = fp32(w'_0 o_0) + fp32(w'_1 o_1) + ... + fp32(w'_{k-1} o_{k-1}) + shared
//   n = bf16(c * (1 / sqrt(mean(c^2) + eps)) * gain)
// with o_j = ret[inv_perm[t*k + j]], in the order and precision of the
// single-GPU combine (whose slots hold fp32(w' o) and the shared output).
// The products are rounded to fp32 before each add (no fused multiply-add),
// as the single-GPU down GEMM stores fp32(w' o) in its slot; the RMSNorm half
// is the single-GPU combine's own (rmsnorm_row).
// NV = float4s per thread; the returned rows' loads are issued in batches
// of kJ per float4 before they are added (in dispatch-slot order), as in
// the single-GPU combine.
template <int NV>
__global__ void __launch_bounds__(kCombineThreads) ep_combine_rmsnorm_kernel(
    const float4 *__restrict__ ret, const int32_t *__restrict__ inv, const float *__restrict__ wscaled,
    const float4 *__restrict__ slots, int L, int k, float eps, const float4 *__restrict__ gain,
    __nv_bfloat16 *__restrict__ n, const uint32_t *status) {
  constexpr int kJ = NV >= 8 ? 1 : 8 / NV;
  __shared__ float red[kCombineThreads / 32];
  __shared__ int s_row[32];
  __shared__ float s_w[32];
  if (call_failed(status)) return;
  const int t = blockIdx.x;
  const int L4 = L >> 2;
  if (threadIdx.x < k) {
    s_row[threadIdx.x] = __ldg(inv + static_cast<size_t>(t) * k + threadIdx.x);
    s_w[threadIdx.x] = __ldg(wscaled + static_cast<size_t>(t) * k + threadIdx.x);
  }
  __syncthreads();
  const float4 *sh = slots + (static_cast<size_t>(t) * (k + 1) + k) * L4;
  const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
  float4 c[NV];
  {
    const float w0 = s_w[0];
    const float4 *r0 = ret + static_cast<size_t>(s_row[0]) * L4;
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      const int i = threadIdx.x + v * kCombineThreads;
      const float4 o0 = i < L4 ? __ldg(r0 + i) : zero;
      c[v] = make_float4(__fmul_rn(o0.x, w0), __fmul_rn(o0.y, w0), __fmul_rn(o0.z, w0), __fmul_rn(o0.w, w0));
    }
  }
  for (int j0 = 1; j0 < k; j0 += kJ) {
    float4 b[NV][kJ];
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      const int i = threadIdx.x + v * kCombineThreads;
#pragma unroll
      for (int jj = 0; jj < kJ; ++jj)
        b[v][jj] = i < L4 && j0 + jj < k ? __ldg(ret + static_cast<size_t>(s_row[j0 + jj]) * L4 + i) : zero;
    }
#pragma unroll
    for (int jj = 0; jj < kJ; ++jj) {
      if (j0 + jj < k) {
        const float wj = s_w[j0 + jj];
#pragma unroll
        for (int v = 0; v < NV; ++v) {
          c[v].x = __fadd_rn(c[v].x, __fmul_rn(b[v][jj].x, wj));
          c[v].y = __fadd_rn(c[v].y, __fmul_rn(b[v][jj].y, wj));
          c[v].z = __fadd_rn(c[v].z, __fmul_rn(b[v][jj].z, wj));
          c[v].w = __fadd_rn(c[v].w, __fmul_rn(b[v][jj].w, wj));
        }
      }
    }
  }
#pragma unroll
  for (int v = 0; v < NV; ++v) {
    const int i = threadIdx.x + v * kCombineThreads;
    const float4 b = i < L4 ? __ldg(sh + i) : zero;
    c[v].x += b.x; c[v].y += b.y; c[v].z += b.z; c[v].w += b.w;
  }
  rmsnorm_row(c, L, eps, gain, n + static_cast<size_t>(t) * L, red);
}

}  // namespace mrl
