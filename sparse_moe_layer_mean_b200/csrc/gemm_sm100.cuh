// gemm_sm100.cuh — persistent, warp-specialised tcgen05 GEMM for sm_100a.
//
// D[128 x N] += A[128 x K] * B[N x K]^T, both operands K-major bf16 staged by
// SWIZZLE_128B TMA tile loads into shared memory; the fp32 accumulator lives
// in tensor memory, double-buffered (2 x 256 columns) so the epilogue of one
// tile overlaps the main loop of the next.  A and B are loaded by producer
// warps of their own into the same ring stages.
//
//   warp 0   : TMA producer for A (one thread)
//   warp 1   : TMEM allocator + UMMA issuer (one thread issues, commits)
//   warps 2-5: epilogue (warp w reads TMEM lanes 32*(w%4) .. +31)
//   warp 6   : TMA producer for B (one thread)
//
// A policy class P describes the problem: how many work units there are, what
// each unit loads per 64-wide K block, the MMA N of each unit, and the
// epilogue.  A unit may hold several sub-tiles that share one epilogue state
// (the router walks its expert chunks that way).  Units are dealt round-robin
// over the persistent CTAs.
//
// Every wait is bounded (see mbar_wait); on a timeout the CTA raises an abort
// flag, every role unwinds, TMEM is freed, and the status word records it.
#pragma once
#include "common.cuh"

namespace mrl {

constexpr int kGemmThreads = 224;
constexpr int kAccCols = 256;   // TMEM columns per accumulator buffer
constexpr int kTmemCols = 512;  // two buffers
constexpr int kBK = 64;         // bf16 elements per K block (128 bytes = one swizzle row)

struct Unit {
  int g;     // group (routed expert e < E, or E for the shared expert); 0 for dense
  int m;     // M tile
  int n0;    // first N column of the unit
  int nv;    // valid N columns in the unit
  int nsub;  // sub-tiles
  int row0;  // grouped GEMMs: first dispatched row of the unit
  int krows; // ragged-K policies: rows of the unit's reduction
};

// Operand major-ness of a policy: P::kAMN / P::kBMN (true = the M or N index
// is contiguous in memory, staged as 64-wide MN blocks of P::kAMNStride /
// P::kBMNStride bytes); policies without them are K-major on both sides.
template <class P, class = void>
struct OperandMajor {
  static constexpr bool a_mn = false, b_mn = false;
  static constexpr uint32_t a_stride = 0, b_stride = 0;
};
template <class P>
struct OperandMajor<P, decltype(void(P::kAMN))> {
  static constexpr bool a_mn = P::kAMN, b_mn = P::kBMN;
  static constexpr uint32_t a_stride = P::kAMNStride, b_stride = P::kBMNStride;
};

// Ragged K (P::kRaggedK): each unit has its own number of K blocks,
// P::unit_k_blocks(p, U) (possibly 0), and only the first
// P::tail_rows(p, U) rows of its last K block belong to it; the MMA warp
// zeroes the rest of that block's tiles in shared memory (P::zero_tail)
// before the MMAs read it.  A unit with no K blocks leaves a zero tile
// (P::epilogue is told through U and writes zeros without reading TMEM).
template <class P, class = void>
struct RaggedK {
  static constexpr bool on = false;
};
template <class P>
struct RaggedK<P, decltype(void(P::kRaggedK))> {
  static constexpr bool on = P::kRaggedK;
};

template <class P>
__device__ __forceinline__ int unit_k_blocks(const typename P::Params &p, const Unit &U, int kblocks) {
  if constexpr (RaggedK<P>::on)
    return P::unit_k_blocks(p, U);
  else
    return kblocks;
}

// Descriptor of the kk-th 16-deep K step of an operand tile at `base`.
template <bool MN, uint32_t STRIDE, int UMMA_K_BYTES>
__device__ __forceinline__ uint64_t operand_desc(uint32_t base, int kk) {
  if constexpr (MN)
    return sdesc_mn_sw128(base + kk * 2048, STRIDE);
  else
    return sdesc_sw128(base + kk * UMMA_K_BYTES);
}

__device__ __forceinline__ bool bar_red_or(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

// Ring: P::kStages stages, each holding one 64-wide K block of A and of B.
// A stage's full barrier completes when both producers' loads have landed
// (arrival count 2 plus the transaction bytes).  Stages are released in
// groups of P::kGroup by a single tcgen05.commit: every commit costs the MMA
// pipe about 100 cycles, so committing once per group instead of once per
// operand per stage keeps the tensor pipe busy.
template <class P>
struct GemmSmem {
  static_assert(P::kStages % P::kGroup == 0, "ring depth must be a multiple of the release group");
  static constexpr int kStageBytes = P::kABytes + P::kBBytesMax;
  static constexpr int kRing = P::kStages * kStageBytes;
  static constexpr int kBarOff = kRing;
  static constexpr int kNumBars = P::kStages + P::kStages / P::kGroup + 4;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kEpiOff = (kMiscOff + 16 + 127) & ~127;
  static constexpr int kAuxOff = (kEpiOff + P::kEpiSmem + 127) & ~127;
  static constexpr int kTotal = kAuxOff + P::kAuxSmem + 1024;  // + alignment slack
};

template <class P>
__global__ void __launch_bounds__(kGemmThreads, 1) gemm_kernel(const __grid_constant__ typename P::Params p) {
  using L = GemmSmem<P>;
  constexpr int S = P::kStages, G = P::kGroup;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kBarOff);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMiscOff);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMiscOff + 4);
  volatile int *hold_flag = reinterpret_cast<volatile int *>(smem + L::kMiscOff + 8);
  uint8_t *epi_smem = smem + L::kEpiOff;
  uint8_t *aux = smem + L::kAuxOff;  // per-launch tables staged once per CTA

  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = full0 + 8 * S;  // one per group of G stages
  const uint32_t accf0 = empty0 + 8 * (S / G);
  const uint32_t acce0 = accf0 + 16;
  const uint32_t ring = smem_u32(smem);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  uint32_t *status = p.status;

  if (threadIdx.x == 0) {
    const uint2 hdr = call_header(status);  // loaded first: the barrier set-up hides its latency
    for (int s = 0; s < S; ++s) mbar_init(full0 + 8 * s, 2);
    for (int g = 0; g < S / G; ++g) mbar_init(empty0 + 8 * g, 1);
    for (int a = 0; a < 2; ++a) {
      mbar_init(accf0 + 8 * a, 1);
      mbar_init(acce0 + 8 * a, 4);
    }
    *abort_flag = hdr.x != DEV_OK;  // an earlier kernel of the call failed: do nothing
    *hold_flag = (hdr.y & HOLD_GEMM) != 0;
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
  if (*abort_flag) goto done;

  if (warp == 0 || warp == 6) {
    // with the call's loads held (test mask) nothing is issued, so the
    // consumers' bounded waits run out and record DEV_TIMEOUT
    if (lane == 0 && !*hold_flag) {
      // producers: warp 0 loads A, warp 6 loads B, into the same stages
      const bool isA = warp == 0;
      P::prefetch(p);
      int s = 0;
      uint32_t ph = 0;
      for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
        const Unit U = P::unit(p, u, aux);
        for (int sub = 0; sub < U.nsub; ++sub) {
          const uint32_t bytes = isA ? P::kABytes : P::b_bytes(p, U, sub);
          const int kbu = unit_k_blocks<P>(p, U, kblocks);
          for (int kb = 0; kb < kbu; ++kb) {
            if (s % G == 0 && !mbar_wait(empty0 + 8 * (s / G), ph ^ 1, abort_flag, status)) goto done;
            mbar_arrive_expect_tx(full0 + 8 * s, bytes);
            const uint32_t st = ring + s * L::kStageBytes;
            if (isA)
              P::load_a(p, U, sub, kb, st, full0 + 8 * s);
            else
              P::load_b(p, U, sub, kb, st + P::kABytes, full0 + 8 * s);
            if (++s == S) { s = 0; ph ^= 1; }
          }
        }
      }
    }
  } else if (warp == 1) {
   if constexpr (RaggedK<P>::on) {
    // the whole warp walks the ring (it zeroes the ragged tails); lane 0 issues
    int s = 0, acc = 0;
    uint32_t ph = 0, aph = 0;
    for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
      const Unit U = P::unit(p, u, aux);
      const int kbu = unit_k_blocks<P>(p, U, kblocks);
      if (!__all_sync(0xffffffffu, mbar_wait(acce0 + 8 * acc, aph ^ 1, abort_flag, status))) goto done;
      tc_fence_after();
      const uint32_t tacc = tmem_base + acc * kAccCols;
      const uint32_t idesc = P::idesc(p, U, 0);
      for (int kb = 0; kb < kbu; ++kb) {
        if (!__all_sync(0xffffffffu, mbar_wait(full0 + 8 * s, ph, abort_flag, status))) goto done;
        tc_fence_after();
        const uint32_t a_s = ring + s * L::kStageBytes;
        const uint32_t b_s = a_s + P::kABytes;
        if (kb == kbu - 1) {
          const int tail = P::tail_rows(p, U);
          if (tail < kBK) {
            P::zero_tail(p, U, smem + (a_s - ring), smem + (b_s - ring), tail, lane);
            fence_proxy_async_shared();  // the zeros are read by the tensor core (async proxy)
          }
          __syncwarp();
        }
        if (lane == 0) {
#pragma unroll
          for (int kk = 0; kk < kBK * 2 / P::kUmmaKBytes; ++kk)
            P::mma(tacc, operand_desc<OperandMajor<P>::a_mn, OperandMajor<P>::a_stride, P::kUmmaKBytes>(a_s, kk),
                   operand_desc<OperandMajor<P>::b_mn, OperandMajor<P>::b_stride, P::kUmmaKBytes>(b_s, kk), idesc,
                   (kb | kk) != 0);
          if (s % G == G - 1) umma_commit(empty0 + 8 * (s / G));
        }
        __syncwarp();
        if (++s == S) { s = 0; ph ^= 1; }
      }
      if (lane == 0) {
        if (kbu > 0)
          umma_commit(accf0 + 8 * acc);
        else
          mbar_arrive(accf0 + 8 * acc);  // nothing to wait for: the epilogue writes a zero tile
      }
      __syncwarp();
      acc ^= 1;
      if (acc == 0) aph ^= 1;
    }
   } else {
    if (lane == 0) {
      int s = 0, acc = 0;
      uint32_t ph = 0, aph = 0;
      for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
        const Unit U = P::unit(p, u, aux);
        for (int sub = 0; sub < U.nsub; ++sub) {
          if (!mbar_wait(acce0 + 8 * acc, aph ^ 1, abort_flag, status)) goto done;
          tc_fence_after();
          const uint32_t tacc = tmem_base + acc * kAccCols;
          const uint32_t idesc = P::idesc(p, U, sub);
          for (int kb = 0; kb < kblocks; ++kb) {
            if (!mbar_wait(full0 + 8 * s, ph, abort_flag, status)) goto done;
            tc_fence_after();
            const uint32_t a_s = ring + s * L::kStageBytes;
            const uint32_t b_s = a_s + P::kABytes;
            // kASub A tiles of the stage (each kASubBytes) share its B tile and the accumulator
#pragma unroll
            for (int as = 0; as < P::kASub; ++as)
#pragma unroll
              for (int kk = 0; kk < kBK * 2 / P::kUmmaKBytes; ++kk)
                P::mma(tacc,
                       operand_desc<OperandMajor<P>::a_mn, OperandMajor<P>::a_stride, P::kUmmaKBytes>(
                           a_s + as * P::kASubBytes, kk),
                       operand_desc<OperandMajor<P>::b_mn, OperandMajor<P>::b_stride, P::kUmmaKBytes>(b_s, kk),
                       idesc, (kb | kk | as) != 0);
            if (s % G == G - 1) umma_commit(empty0 + 8 * (s / G));
            if (++s == S) { s = 0; ph ^= 1; }
          }
          umma_commit(accf0 + 8 * acc);
          acc ^= 1;
          if (acc == 0) aph ^= 1;
        }
      }
    }
   }
  } else {
    // epilogue warps 2..5; TMEM lane quarter = warp % 4
    const int q = warp & 3;
    const int etid = threadIdx.x - 64;
    typename P::EpiState st;
    int acc = 0;
    uint32_t aph = 0;
    for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
      const Unit U = P::unit(p, u, aux);
      for (int sub = 0; sub < U.nsub; ++sub) {
        const bool ok = mbar_wait(accf0 + 8 * acc, aph, abort_flag, status);
        // all four warps take the same decision, so none is left at a named barrier
        if (bar_red_or(1, 128, !ok || *abort_flag)) goto done;
        tc_fence_after();
        P::epilogue(p, U, sub, tmem_base + acc * kAccCols + (static_cast<uint32_t>(q * 32) << 16), q, lane,
                    etid, st, epi_smem);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acce0 + 8 * acc);
        acc ^= 1;
        if (acc == 0) aph ^= 1;
      }
    }
  }
done:
  // bulk tensor stores an epilogue issued finish before the CTA's shared memory goes away
  if (lane == 0) bulk_wait_all();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace mrl
