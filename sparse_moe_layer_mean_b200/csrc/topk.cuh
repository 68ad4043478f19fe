// topk.cuh — register-resident running top-k with the lower-index tie rule.
#pragma once
#include <math.h>

#include "common.cuh"

namespace mrl {

// Sorted (descending value) list of the best candidates seen so far.
// Candidates must be offered in ascending index order: a candidate equal in
// value to a kept one is placed after it, so ties resolve to the lower index
// under IEEE equality (+0 == -0).  The list holds the best KMAX candidates
// offered so far, so its first k (<= KMAX) entries are the top k.
template <int KMAX>
struct TopK {
  float v[KMAX];  // biased score used for selection
  float s[KMAX];  // unbiased score carried along for the weights
  int i[KMAX];    // expert index
  float thr;

  __device__ __forceinline__ void init() {
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      v[j] = -INFINITY;
      s[j] = 0.f;
      i[j] = 0x7fffffff;
    }
    thr = -INFINITY;
  }

  __device__ __forceinline__ void offer(float cv, int ci, float cs) {
    if (cv > thr) {
      bool take = false;
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        take = take || (cv > v[j]);
        const float tv = v[j], ts = s[j];
        const int ti = i[j];
        v[j] = take ? cv : tv;
        s[j] = take ? cs : ts;
        i[j] = take ? ci : ti;
        cv = take ? tv : cv;
        cs = take ? ts : cs;
        ci = take ? ti : ci;
      }
      // Admission threshold: the KMAX-th best so far.  It is never above the
      // k-th best, so no candidate that belongs in the top k is turned away.
      thr = v[KMAX - 1];
    }
  }

  // Remove the head (used by the warp merge).
  __device__ __forceinline__ void pop() {
#pragma unroll
    for (int j = 0; j < KMAX - 1; ++j) {
      v[j] = v[j + 1]; s[j] = s[j + 1]; i[j] = i[j + 1];
    }
    v[KMAX - 1] = -INFINITY;
    s[KMAX - 1] = 0.f;
    i[KMAX - 1] = 0x7fffffff;
  }
};

// (va, ia) ranks before (vb, ib): larger value, or equal value and lower index.
__device__ __forceinline__ bool ranks_before(float va, int ia, float vb, int ib) {
  return (va > vb) || (va == vb && ia < ib);
}

// Insert a candidate offered in any index order (the merge of partial lists):
// it goes before the first kept entry it ranks before.
template <int KMAX>
__device__ __forceinline__ void topk_offer_any(TopK<KMAX> &tk, float cv, int ci, float cs) {
  if (!ranks_before(cv, ci, tk.v[KMAX - 1], tk.i[KMAX - 1])) return;
  bool take = false;
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    take = take || ranks_before(cv, ci, tk.v[j], tk.i[j]);
    const float tv = tk.v[j], ts = tk.s[j];
    const int ti = tk.i[j];
    tk.v[j] = take ? cv : tv;
    tk.s[j] = take ? cs : ts;
    tk.i[j] = take ? ci : ti;
    cv = take ? tv : cv;
    cs = take ? ts : cs;
    ci = take ? ti : ci;
  }
}

// Final step of routing for one token: w_j = s_j / (s_0 + ... + s_{k-1})
// (fp32, summed in rank order), w'_j = w_j * alpha[e_j].  A zero sum (every
// selected score 0, e.g. sigmoids that underflowed) gives the uniform weights
// 1/k.  A slot whose running list never admitted a candidate (fewer than k
// experts with a biased score that is a number above -inf: NaN scores, or a
// -inf bias on too many experts) is written as expert -1 with weight 0, and
// the call's status word records DEV_CHECK, so the dispatch kernels that
// follow do nothing and no index outside [0, E) is ever used.
template <int KMAX>
__device__ __forceinline__ void write_selection(const float (&sel_s)[KMAX], const int (&sel_i)[KMAX], int k, int E,
                                                size_t t, const float *__restrict__ alpha,
                                                int32_t *__restrict__ topk_idx, float *__restrict__ topk_w,
                                                float *__restrict__ wscaled, uint32_t *status) {
  float den = sel_s[0];
#pragma unroll
  for (int j = 1; j < KMAX; ++j)
    if (j < k) den = den + sel_s[j];
  const float uniform = 1.0f / static_cast<float>(k);
  bool complete = true;
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    if (j < k) {
      const size_t o = t * k + j;
      const int e = sel_i[j];
      if (static_cast<unsigned>(e) < static_cast<unsigned>(E)) {
        const float w = den != 0.0f ? sel_s[j] / den : uniform;
        topk_idx[o] = e;
        topk_w[o] = w;
        wscaled[o] = w * __ldg(alpha + e);
      } else {
        complete = false;
        topk_idx[o] = -1;
        topk_w[o] = 0.0f;
        wscaled[o] = 0.0f;
      }
    }
  }
  if (!complete && status) atomicCAS(status, DEV_OK, DEV_CHECK);
}

}  // namespace mrl
