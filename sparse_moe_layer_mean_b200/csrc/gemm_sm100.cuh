// gemm_sm100.cuh — persistent, warp-specialised tcgen05 GEMM for sm_100a.
//
// D[128 x N] += A[128 x K] * B[N x K]^T, both operands K-major bf16 staged by
// SWIZZLE_128B TMA tile loads into shared memory; the fp32 accumulator lives
// in tensor memory, double-buffered (2 x 256 columns) so the epilogue of one
// tile overlaps the main loop of the next.  A and B have rings of their own
// depths: the grouped expert GEMMs stream A (expert weights) from HBM and
// re-read B (dispatched token rows) from L2, so A gets the deeper ring and
// more HBM bytes stay in flight per SM.
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
};

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

template <class P>
struct GemmSmem {
  static constexpr int kARing = P::kStagesA * P::kABytes;
  static constexpr int kBRing = P::kStagesB * P::kBBytesMax;
  static constexpr int kBarOff = kARing + kBRing;
  static constexpr int kNumBars = 2 * P::kStagesA + 2 * P::kStagesB + 4;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kEpiOff = (kMiscOff + 16 + 127) & ~127;
  static constexpr int kAuxOff = (kEpiOff + P::kEpiSmem + 127) & ~127;
  static constexpr int kTotal = kAuxOff + P::kAuxSmem + 1024;  // + alignment slack
};

template <class P>
__global__ void __launch_bounds__(kGemmThreads, 1) gemm_kernel(const __grid_constant__ typename P::Params p) {
  using L = GemmSmem<P>;
  constexpr int SA = P::kStagesA, SB = P::kStagesB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kBarOff);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMiscOff);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMiscOff + 4);
  uint8_t *epi_smem = smem + L::kEpiOff;
  uint8_t *aux = smem + L::kAuxOff;  // per-launch tables staged once per CTA

  const uint32_t fullA0 = smem_u32(bars);
  const uint32_t emptyA0 = fullA0 + 8 * SA;
  const uint32_t fullB0 = emptyA0 + 8 * SA;
  const uint32_t emptyB0 = fullB0 + 8 * SB;
  const uint32_t accf0 = emptyB0 + 8 * SB;
  const uint32_t acce0 = accf0 + 16;
  const uint32_t ringA = smem_u32(smem);
  const uint32_t ringB = ringA + L::kARing;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  uint32_t *status = p.status;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SA; ++s) {
      mbar_init(fullA0 + 8 * s, 1);
      mbar_init(emptyA0 + 8 * s, 1);
    }
    for (int s = 0; s < SB; ++s) {
      mbar_init(fullB0 + 8 * s, 1);
      mbar_init(emptyB0 + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(accf0 + 8 * a, 1);
      mbar_init(acce0 + 8 * a, 4);
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
      // producers: warp 0 fills the A ring, warp 6 the B ring
      const bool isA = warp == 0;
      const int S = isA ? SA : SB;
      const uint32_t full0 = isA ? fullA0 : fullB0, empty0 = isA ? emptyA0 : emptyB0;
      const uint32_t ring = isA ? ringA : ringB;
      const uint32_t sbytes = isA ? P::kABytes : P::kBBytesMax;
      P::prefetch(p);
      int s = 0;
      uint32_t ph = 0;
      for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
        const Unit U = P::unit(p, u, aux);
        for (int sub = 0; sub < U.nsub; ++sub) {
          const uint32_t bytes = isA ? P::kABytes : P::b_bytes(p, U, sub);
          for (int kb = 0; kb < kblocks; ++kb) {
            if (!mbar_wait(empty0 + 8 * s, ph ^ 1, abort_flag, status)) goto done;
            mbar_arrive_expect_tx(full0 + 8 * s, bytes);
            if (isA)
              P::load_a(p, U, sub, kb, ring + s * sbytes, full0 + 8 * s);
            else
              P::load_b(p, U, sub, kb, ring + s * sbytes, full0 + 8 * s);
            if (++s == S) { s = 0; ph ^= 1; }
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int sa = 0, sb = 0, acc = 0;
      uint32_t pa = 0, pb = 0, aph = 0;
      for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
        const Unit U = P::unit(p, u, aux);
        for (int sub = 0; sub < U.nsub; ++sub) {
          if (!mbar_wait(acce0 + 8 * acc, aph ^ 1, abort_flag, status)) goto done;
          tc_fence_after();
          const uint32_t tacc = tmem_base + acc * kAccCols;
          const uint32_t idesc = P::idesc(p, U, sub);
          for (int kb = 0; kb < kblocks; ++kb) {
            if (!mbar_wait(fullA0 + 8 * sa, pa, abort_flag, status)) goto done;
            if (!mbar_wait(fullB0 + 8 * sb, pb, abort_flag, status)) goto done;
            tc_fence_after();
            const uint32_t a_s = ringA + sa * P::kABytes;
            const uint32_t b_s = ringB + sb * P::kBBytesMax;
#pragma unroll
            for (int kk = 0; kk < kBK * 2 / P::kUmmaKBytes; ++kk)
              P::mma(tacc, sdesc_sw128(a_s + kk * P::kUmmaKBytes), sdesc_sw128(b_s + kk * P::kUmmaKBytes),
                     idesc, (kb | kk) != 0);
            umma_commit(emptyA0 + 8 * sa);
            umma_commit(emptyB0 + 8 * sb);
            if (++sa == SA) { sa = 0; pa ^= 1; }
            if (++sb == SB) { sb = 0; pb ^= 1; }
          }
          umma_commit(accf0 + 8 * acc);
          acc ^= 1;
          if (acc == 0) aph ^= 1;
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
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace mrl
