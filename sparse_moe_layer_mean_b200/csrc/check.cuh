// check.cuh — device checker of a routing record.  It verifies the invariants
// of the dispatch record (each token picks k distinct experts out of the 512
// routed ones: blog.derekhsu.net, "ERNIE-5.5-Flash-Base", section "多路由潛在
// MoE (Multi-Router Latent MoE)"; the entries are then grouped expert-major for
// the grouped GEMMs):
//   - every topk_idx lies in [0, E) and a token's k experts are distinct;
//   - counts >= 0 and offsets are their exclusive scan, ending at T*k;
//   - perm and inv_perm are inverse bijections on [0, T*k);
//   - dispatch row r holds an entry of the expert whose row range holds r, and
//     an expert's rows hold its entries in ascending t*k+j order;
//   - every routing weight is finite.
// A failure sets DEV_CHECK in the status word (if it was clear) and ORs the
// invariant's bit into header word 2.  Every load is range-checked before it
// is used as an index, so a corrupt record is reported, never dereferenced.
#pragma once
#include "common.cuh"

namespace mrl {

enum : uint32_t {
  CHECK_INDEX = 1u << 0,      // an expert index outside [0, E)
  CHECK_DUPLICATE = 1u << 1,  // a token selects one expert twice
  CHECK_OFFSETS = 1u << 2,    // a negative count, or offsets not the exclusive scan of counts
  CHECK_PERM = 1u << 3,       // perm and inv_perm not inverse bijections on [0, T*k)
  CHECK_GROUP = 1u << 4,      // a dispatch row outside the row range of its entry's expert
  CHECK_ORDER = 1u << 5,      // an expert's rows not in ascending t*k+j order
  CHECK_WEIGHT = 1u << 6,     // a routing weight that is not finite
};

constexpr int kCheckThreads = 256;

// Thread i checks entry i and dispatch row i (i < T*k), token i (i < T) and
// expert i (i <= E).  Bits are gathered per warp before the atomics.
__global__ void __launch_bounds__(kCheckThreads) check_routing_kernel(
    const int32_t *__restrict__ idx, const float *__restrict__ w, const int32_t *__restrict__ counts,
    const int32_t *__restrict__ offsets, const int32_t *__restrict__ perm, const int32_t *__restrict__ inv, int T,
    int E, int k, uint32_t *hdr) {
  const long long Tk = static_cast<long long>(T) * k;
  const long long n = Tk > E + 1 ? Tk : E + 1;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  // same trip count for every lane of a warp, so the warp vote below is uniform
  const long long base0 = static_cast<long long>(blockIdx.x) * blockDim.x + (threadIdx.x & ~31u);
  const int lane = threadIdx.x & 31;
  for (long long i0 = base0; i0 < n; i0 += stride) {
    const long long i = i0 + lane;
    uint32_t bad = 0;
    if (i < Tk) {
      const int e = idx[i];
      if (e < 0 || e >= E) bad |= CHECK_INDEX;
      if (w && !isfinite(w[i])) bad |= CHECK_WEIGHT;
      const int r = inv[i];
      if (r < 0 || r >= Tk || perm[r] != i) bad |= CHECK_PERM;
      const int f = perm[i];  // the entry in dispatch row i
      if (f < 0 || f >= Tk || inv[f] != i) {
        bad |= CHECK_PERM;
      } else {
        const int ef = idx[f];
        if (ef >= 0 && ef < E) {
          const long long lo = offsets[ef], hi = lo + static_cast<long long>(counts[ef]);
          if (i < lo || i >= hi) {
            bad |= CHECK_GROUP;
          } else if (i + 1 < hi && i + 1 < Tk) {
            const int f2 = perm[i + 1];
            if (f2 >= 0 && f2 < Tk && idx[f2] == ef && f2 <= f) bad |= CHECK_ORDER;
          }
        }
      }
    }
    if (i < T) {
      const int32_t *row = idx + i * k;
      for (int j = 1; j < k; ++j)
        for (int j2 = 0; j2 < j; ++j2)
          if (row[j] == row[j2]) bad |= CHECK_DUPLICATE;
    }
    if (i < E) {
      const long long c = counts[i];
      if (c < 0 || static_cast<long long>(offsets[i + 1]) - offsets[i] != c) bad |= CHECK_OFFSETS;
    }
    if (i == 0 && (offsets[0] != 0 || offsets[E] != Tk)) bad |= CHECK_OFFSETS;
    // one atomic pair per warp that found something
    bad = __reduce_or_sync(0xffffffffu, bad);
    if (bad && lane == 0) {
      atomicCAS(hdr, DEV_OK, DEV_CHECK);
      atomicOr(hdr + 2, bad);
    }
  }
}

}  // namespace mrl
