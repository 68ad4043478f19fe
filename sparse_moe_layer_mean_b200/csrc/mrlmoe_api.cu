// mrlmoe_api.cu — the C ABI: host-side validation, workspace layout, TMA
// descriptor set-up and the launch sequence of the layer on the caller's stream.
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>

#include "mrlmoe.h"
#include "policies.cuh"
#include "gemm2_sm100.cuh"
#include "gemm8_sm100.cuh"
#include "gemm8w_sm100.cuh"
#include "routing.cuh"
#include "check.cuh"
#include "backward.cuh"
#include "ep.cuh"

using namespace mrl;

namespace {

constexpr int kMaxDevices = 64;

// ------------------------------------------------------------ NVTX ranges
// One range per call of an entry point and, inside it, one per stage (the
// stages that the *_timed entry points time with events), so a profiler can
// attribute or filter kernels by stage.  Host-side only: no-ops unless a
// profiling tool is attached, and invisible to a CUDA graph capture.
thread_local bool t_stage_open = false;

void nvtx_stage(const char *name) {
  if (t_stage_open) nvtxRangePop();
  t_stage_open = name != nullptr;
  if (name) nvtxRangePushA(name);
}

struct NvtxCall {
  explicit NvtxCall(const char *name) {
    nvtxRangePushA(name);
    t_stage_open = false;
  }
  ~NvtxCall() {
    nvtx_stage(nullptr);
    nvtxRangePop();
  }
};

constexpr const char *kForwardStages[8] = {"down_proj",   "router_topk", "dispatch",        "gather",
                                           "gate_up_glu", "expert_down", "combine_rmsnorm", "up_proj"};
constexpr const char *kBackwardStages[10] = {"dn", "dw_up", "rms_combine_bwd", "dh_glu_bwd", "dz",
                                             "token_router_bwd", "dw_router_alpha", "expert_wgrad", "dx",
                                             "dw_down"};

// ------------------------------------------------------------ validation
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

mrlmoe_status check_config(const mrlmoe_config *c) {
  if (!c) return MRLMOE_ERR_INVALID_ARG;
  if (c->T < 1 || c->d_model < 128 || c->d_lat < 128 || c->d_ff < 128) return MRLMOE_ERR_INVALID_ARG;
  if (c->d_model % 128 || c->d_lat % 128 || c->d_ff % 128) return MRLMOE_ERR_INVALID_ARG;
  if (c->d_lat > 8192) return MRLMOE_ERR_UNSUPPORTED;
  if (c->n_experts < 16 || c->n_experts > 1024 || c->n_experts % 16) return MRLMOE_ERR_INVALID_ARG;
  if (c->top_k < 1 || c->top_k > c->n_experts || c->top_k > kTopKMax) return MRLMOE_ERR_INVALID_ARG;
  if (c->n_routers < 1 || c->n_routers > 8) return MRLMOE_ERR_INVALID_ARG;
  if (!(c->rms_eps >= 0.f)) return MRLMOE_ERR_INVALID_ARG;
  if (c->dtype != MRLMOE_BF16 && c->dtype != MRLMOE_FP8_E4M3_BLOCK128 && c->dtype != MRLMOE_FP4_E2M1_BLOCK128)
    return MRLMOE_ERR_INVALID_ARG;
  if (c->aggregation != MRLMOE_AGG_MEAN && c->aggregation != MRLMOE_AGG_SUM && c->aggregation != MRLMOE_AGG_MAX)
    return MRLMOE_ERR_INVALID_ARG;
  if (c->hold & ~static_cast<uint32_t>(MRLMOE_HOLD_GEMM | MRLMOE_HOLD_GEMM_PAIR | MRLMOE_HOLD_GEMM_FP8))
    return MRLMOE_ERR_INVALID_ARG;
  // the FP8 GEMMs stage at most kF8MaxKB scales of 128-wide K blocks per unit
  if (c->dtype != MRLMOE_BF16 &&
      (c->d_model > 128 * kF8MaxKB || c->d_lat > 128 * kF8MaxKB || c->d_ff > 128 * kF8MaxKB))
    return MRLMOE_ERR_UNSUPPORTED;
  // dispatched rows are addressed with 32-bit indices
  const long long rows = static_cast<long long>(c->T) * (c->top_k + 1);
  if (rows * 256 >= (1ll << 31)) return MRLMOE_ERR_UNSUPPORTED;
  return MRLMOE_OK;
}

// Router chunk: experts per accumulator so that R * ec <= 256 and ec | E.
// The widest expert chunk that fits one accumulator (R * ec <= 256 columns).
// (Narrower chunks for decode-sized T, to spread the router over more CTAs,
// measured slower: more partial lists to merge and MMAs at the instruction's
// minimum cost.)
int router_ec(int E, int R, int) {
  for (int ec = 256; ec >= 16; ec >>= 1)
    if (ec * R <= 256 && E % ec == 0) return ec;
  return 16;
}

// Router split: the E/ec expert chunks of a token tile are shared by `parts`
// CTAs (a power of two dividing the chunk count) so that m_tiles * parts
// fills the SMs; parts > 1 adds a small merge of the partial selections.
int router_parts(const mrlmoe_config &c, int sms) {
  const int chunks = c.n_experts / router_ec(c.n_experts, c.n_routers, c.T);
  const int m_tiles = (c.T + 127) / 128;
  int parts = 1;
  while (parts * 2 <= chunks && chunks % (parts * 2) == 0 && m_tiles * parts * 2 <= std::max(sms, 1)) parts *= 2;
  return parts;
}

// Router K split for small T: when token tiles x expert chunks would fill at
// most half of a 148-SM GPU, the K range is split (a power of two dividing
// the K blocks) so that about 148 units run at once.  The target is a fixed
// number, not the device's SM count, so the workspace layout depends on the
// config alone.
constexpr int kRouterSplitUnits = 148;
int router_ksplit(const mrlmoe_config &c) {
  const int chunks = c.n_experts / router_ec(c.n_experts, c.n_routers, c.T);
  const int base = ((c.T + 127) / 128) * chunks;
  if (2 * base > kRouterSplitUnits) return 1;
  const int kb = c.d_lat / kBK;
  int ks = 1;
  while (kb % (2 * ks) == 0 && base * 2 * ks <= kRouterSplitUnits) ks *= 2;
  return ks;
}

// ------------------------------------------------------------ workspace
struct Layout {
  size_t status, topk_idx, topk_w, wscaled, counts, offsets, grp_off, grp_cnt, unit1, unit2, perm, inv, mask,
      base, cand_v, cand_s, cand_i, rpart, zbuf, zlo, hbuf, slots, nbuf, xq, xs, zq, zs, hq, hs, nq, ns, total;
  // training forward + backward (bf16): kept pre-activations and the backward's buffers
  size_t gusave, dn, dcd, dod, dgu, dwsp, wrow, dzx, dl, aw, gpart, bgrp_off, bgrp_cnt, bunit1, bunit2;
};

// Blocks of rms_combine_bwd_kernel (a fixed number, so the gain gradient's
// summation order depends on the config alone).
constexpr int kRmsBwdBlocks = 592;
int rms_bwd_blocks(const mrlmoe_config &c) { return std::min(c.T, kRmsBwdBlocks); }

// Training limits beyond check_config: bf16, d_ff <= 8192, and the backward's
// K-blocked dg/du rows ((2 d_ff / 64) planes of T*k + T rows) addressable
// with 32-bit TMA row coordinates (implied by check_config's dispatched-row
// bound once d_ff <= 8192; kept as the stated condition).
bool train_supported(const mrlmoe_config &c) {
  if (c.dtype != MRLMOE_BF16 || c.d_ff > 128 * kBwdMaxSlices) return false;
  const long long rows = static_cast<long long>(c.T) * (c.top_k + 1);
  return (2LL * c.d_ff / 64) * rows < (1LL << 31);
}

Layout layout_of(const mrlmoe_config &c, bool train = false) {
  Layout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += (bytes + 255) & ~size_t(255);
    return o;
  };
  const size_t T = c.T, k = c.top_k, E = c.n_experts, Ld = c.d_lat, F = c.d_ff;
  const size_t Tk = T * k, nch = (T + kChunk - 1) / kChunk;
  L.status = take(256);
  L.topk_idx = take(Tk * 4);
  L.topk_w = take(Tk * 4);
  L.wscaled = take(Tk * 4);
  L.counts = take((E + 2) * 4);
  L.offsets = take((E + 2) * 4);
  L.grp_off = take((E + 2) * 4);
  L.grp_cnt = take((E + 2) * 4);
  L.unit1 = take((E + 2) * 4);
  L.unit2 = take((E + 2) * 4);
  L.perm = take(Tk * 4);
  L.inv = take(Tk * 4);
  L.mask = take(nch * E * 4);
  L.base = take(nch * E * 4);
  const size_t parts = router_parts(c, 1 << 30);  // upper bound over SM counts
  L.cand_v = take(T * parts * k * 4);
  L.cand_s = take(T * parts * k * 4);
  L.cand_i = take(T * parts * k * 4);
  const size_t ks = router_ksplit(c);
  L.rpart = take(ks > 1 ? (ks * T * c.n_routers * E + T * E) * 4 : 0);  // partial logits, then s
  L.zbuf = take((Tk + T) * Ld * 2);
  L.zlo = take(T * Ld * 2);
  L.hbuf = take((Tk + T) * F * 2);
  L.slots = take(T * (k + 1) * Ld * 4);
  L.nbuf = take(T * Ld * 2);
  if (c.dtype != MRLMOE_BF16) {  // e4m3 copies of the GEMM inputs and their 1x128 scales
    const size_t D = c.d_model;
    L.xq = take(T * D);
    L.xs = take(T * (D / 128) * 4);
    L.zq = take((Tk + T) * Ld);
    L.zs = take((Tk + T) * (Ld / 128) * 4);
    L.hq = take((Tk + T) * F);
    L.hs = take((Tk + T) * (F / 128) * 4);
    L.nq = take(T * Ld);
    L.ns = take(T * (Ld / 128) * 4);
  }
  if (train) {
    const size_t rows = Tk + T;
    L.gusave = take(rows * F * 4);
    L.dn = take(T * Ld * 4);
    L.dcd = take(rows * Ld * 2);
    L.dod = take(rows * Ld * 2);
    L.dgu = take(rows * 2 * F * 2);
    L.dwsp = take((F / 128) * rows * 4);
    L.wrow = take(rows * 4);
    L.dzx = take(T * Ld * 2);
    L.dl = take(Tk * c.n_routers * 4);
    L.aw = take(Tk * 4);
    L.gpart = take(static_cast<size_t>(rms_bwd_blocks(c)) * Ld * 4);
    L.bgrp_off = take((E + 2) * 4);
    L.bgrp_cnt = take((E + 2) * 4);
    L.bunit1 = take((E + 2) * 4);
    L.bunit2 = take((E + 2) * 4);
  }
  L.total = off;
  return L;
}

// ------------------------------------------------------------ CUDA helpers
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D map over a row-major [rows, inner] matrix of `esize`-byte elements,
// box = box_rows x (128 / esize) elements (one 128-byte swizzle row).
bool make_map(CUtensorMap *m, const void *base, int esize, uint64_t inner, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {inner * esize};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / esize), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType dt = esize == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  return enc(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 [rows, inner] written by TMA stores: boxes of 32 columns x 32 rows
// (128-byte rows, SWIZZLE_128B).
bool make_map_f32_out(CUtensorMap *m, void *base, uint64_t inner, uint64_t rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {inner * 4};
  const cuuint32_t box[2] = {32, 32};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The three box heights of a bf16 token tensor [rows, inner] (load_token_rows).
bool make_token_maps(TokenMaps *t, const void *base, uint64_t inner, uint64_t rows) {
  t->plane_rows = 0;
  return make_map(&t->m16, base, 2, inner, rows, 16) && make_map(&t->m32, base, 2, inner, rows, 32) &&
         make_map(&t->m64, base, 2, inner, rows, 64);
}

// The same for a K-blocked bf16 token tensor [K/64][rows][64].
bool make_token_maps_blocked(TokenMaps *t, const void *base, uint64_t K, uint64_t rows) {
  if (!make_token_maps(t, base, 64, (K / 64) * rows)) return false;
  t->plane_rows = static_cast<int>(rows);
  return true;
}

// Packed e2m1 weights [rows, inner_bytes]: boxes of 64 bytes (128 codes) x
// box_rows, row-major in shared memory (no swizzle; expand_fp4_tile reads it).
bool make_map_packed(CUtensorMap *m, const void *base, uint64_t inner_bytes, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {inner_bytes, rows};
  const cuuint64_t strides[1] = {inner_bytes};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Packed e2m1 codes [rows, K/2 bytes] read as K 4-bit elements per row and
// unpacked by the TMA into 16-byte chunks of 16 codes (16U4_ALIGN16B; boxes of
// 128 codes x box_rows rows, SWIZZLE_128B: the e4m3 tile's shared layout).
// The type needs a 32-byte-aligned base, K a multiple of 128 and a row stride
// that is a multiple of 32 bytes; the encoder refuses anything else.
bool make_map_e2m1(CUtensorMap *m, const void *base, uint64_t K, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc || (reinterpret_cast<uintptr_t>(base) & 31u)) return false;
  const cuuint64_t dims[2] = {K, rows};
  const cuuint64_t strides[1] = {K / 2};
  const cuuint32_t box[2] = {128, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, const_cast<void *>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The four box heights of an e4m3 token tensor [rows, inner] (load_token_rows8).
bool make_token_maps8(TokenMaps8 *t, const void *base, uint64_t inner, uint64_t rows) {
  return make_map(&t->m16, base, 1, inner, rows, 16) && make_map(&t->m32, base, 1, inner, rows, 32) &&
         make_map(&t->m64, base, 1, inner, rows, 64) && make_map(&t->m128, base, 1, inner, rows, kF8Tile);
}

// The caller's current device, put back when an entry point returns (the
// library switches to the device that owns the call's buffers for its
// launches and leaves the caller's choice as it found it).
struct DeviceRestore {
  int prev = -1;
  ~DeviceRestore() {
    if (prev >= 0) cudaSetDevice(prev);
  }
};

// SM count per device, looked up once per device; concurrent first calls
// from several host threads may each look it up, and store the same value.
std::atomic<int> g_sm_count[kMaxDevices];

// Make the device that owns `p` current for the rest of the call (restored by
// `restore` when the entry point returns); reject host/unknown pointers.
mrlmoe_status bind_device(const void *p, int *sm_count, DeviceRestore *restore) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return MRLMOE_ERR_CUDA;
  }
  if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged) return MRLMOE_ERR_INVALID_ARG;
  if (a.device < 0 || a.device >= kMaxDevices) return MRLMOE_ERR_UNSUPPORTED;
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) return MRLMOE_ERR_CUDA;
  if (cur != a.device) {
    if (cudaSetDevice(a.device) != cudaSuccess) return MRLMOE_ERR_CUDA;
    restore->prev = cur;
  }
  int n = g_sm_count[a.device].load(std::memory_order_relaxed);
  if (!n) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, a.device) != cudaSuccess) return MRLMOE_ERR_CUDA;
    g_sm_count[a.device].store(n, std::memory_order_relaxed);
  }
  *sm_count = n;
  return MRLMOE_OK;
}

// Raise a kernel's dynamic shared-memory limit once per device.  Several host
// threads may race on a device's first launch; each then sets the same
// attribute, which is harmless, and the flag is an atomic.
template <class Kernel>
cudaError_t set_smem_once(std::atomic<bool> (&done)[kMaxDevices], Kernel kern, int bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  if (!done[dev].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    done[dev].store(true, std::memory_order_release);
  }
  return cudaSuccess;
}

template <class P>
cudaError_t launch_gemm(const typename P::Params &p, int grid, cudaStream_t st) {
  static_assert(GemmSmem<P>::kTotal <= 232448, "GEMM shared memory above the 227 KB per-block limit");
  static std::atomic<bool> configured[kMaxDevices];
  cudaError_t e = set_smem_once(configured, gemm_kernel<P>, GemmSmem<P>::kTotal);
  if (e != cudaSuccess) return e;
  gemm_kernel<P><<<grid, kGemmThreads, GemmSmem<P>::kTotal, st>>>(p);
  return cudaGetLastError();
}

template <class P>
cudaError_t launch_gemm_pair(const typename P::Params &p, int grid, cudaStream_t st) {
  static_assert(Gemm2Smem<P>::kTotal <= 232448, "GEMM shared memory above the 227 KB per-block limit");
  static std::atomic<bool> configured[kMaxDevices];
  cudaError_t e = set_smem_once(configured, gemm2_kernel<P>, Gemm2Smem<P>::kTotal);
  if (e != cudaSuccess) return e;
  gemm2_kernel<P><<<grid & ~1, kGemmThreads, Gemm2Smem<P>::kTotal, st>>>(p);
  return cudaGetLastError();
}

// The expert GEMMs run on CTA pairs (M = 256) whenever the slice widths allow:
// gate/up needs d_ff % 128 == 0 (always true), the down GEMM d_lat % 256 == 0.
bool down_uses_pairs(const mrlmoe_config &c) { return c.d_lat % 256 == 0; }
int glu_m_tiles(const mrlmoe_config &c) { return c.d_ff / 128; }
int down_m_tiles(const mrlmoe_config &c) { return down_uses_pairs(c) ? c.d_lat / 256 : c.d_lat / 128; }

#define MRL_TRY(expr)                                  \
  do {                                                 \
    if ((expr) != cudaSuccess) return MRLMOE_ERR_CUDA; \
  } while (0)

// Start of a call: zero the call header (status, hold mask, check bits) and
// store the call's hold mask in the low byte of word 1.  Both are memsets, so
// the call stays capturable in a CUDA graph.
mrlmoe_status init_header(uint32_t *hdr, uint32_t hold, cudaStream_t st) {
  MRL_TRY(cudaMemsetAsync(hdr, 0, 16, st));
  if (hold) MRL_TRY(cudaMemsetAsync(reinterpret_cast<uint8_t *>(hdr) + 4, static_cast<int>(hold & 0xffu), 1, st));
  return MRLMOE_OK;
}

struct Ptrs {
  uint32_t *status;
  int32_t *topk_idx, *counts_e, *offsets_e, *grp_off, *grp_cnt, *unit1, *unit2, *perm, *inv, *base;
  float *topk_w, *wscaled, *scores, *slots, *cand_v, *cand_s, *rpart;
  int32_t *cand_i;
  uint32_t *mask;
  __nv_bfloat16 *zbuf, *zlo, *hbuf, *nbuf;
  uint8_t *xq, *zq, *hq, *nq;  // FP8 variant only
  float *xs, *zs, *hs, *ns;
  int32_t *out_counts, *out_offsets;
};

Ptrs carve(const mrlmoe_config &c, void *ws, const mrlmoe_routing *r) {
  const Layout L = layout_of(c);
  uint8_t *b = static_cast<uint8_t *>(ws);
  Ptrs P{};
  P.status = reinterpret_cast<uint32_t *>(b + L.status);
  P.topk_idx = (r && r->topk_idx) ? r->topk_idx : reinterpret_cast<int32_t *>(b + L.topk_idx);
  P.topk_w = (r && r->topk_w) ? r->topk_w : reinterpret_cast<float *>(b + L.topk_w);
  P.wscaled = reinterpret_cast<float *>(b + L.wscaled);
  P.counts_e = reinterpret_cast<int32_t *>(b + L.counts);
  P.offsets_e = reinterpret_cast<int32_t *>(b + L.offsets);
  P.grp_off = reinterpret_cast<int32_t *>(b + L.grp_off);
  P.grp_cnt = reinterpret_cast<int32_t *>(b + L.grp_cnt);
  P.unit1 = reinterpret_cast<int32_t *>(b + L.unit1);
  P.unit2 = reinterpret_cast<int32_t *>(b + L.unit2);
  P.perm = (r && r->perm) ? r->perm : reinterpret_cast<int32_t *>(b + L.perm);
  P.inv = (r && r->inv_perm) ? r->inv_perm : reinterpret_cast<int32_t *>(b + L.inv);
  P.mask = reinterpret_cast<uint32_t *>(b + L.mask);
  P.base = reinterpret_cast<int32_t *>(b + L.base);
  P.cand_v = reinterpret_cast<float *>(b + L.cand_v);
  P.cand_s = reinterpret_cast<float *>(b + L.cand_s);
  P.cand_i = reinterpret_cast<int32_t *>(b + L.cand_i);
  P.rpart = reinterpret_cast<float *>(b + L.rpart);
  P.zbuf = reinterpret_cast<__nv_bfloat16 *>(b + L.zbuf);
  P.zlo = reinterpret_cast<__nv_bfloat16 *>(b + L.zlo);
  P.hbuf = reinterpret_cast<__nv_bfloat16 *>(b + L.hbuf);
  P.slots = reinterpret_cast<float *>(b + L.slots);
  P.nbuf = reinterpret_cast<__nv_bfloat16 *>(b + L.nbuf);
  if (c.dtype != MRLMOE_BF16) {
    P.xq = b + L.xq; P.zq = b + L.zq; P.hq = b + L.hq; P.nq = b + L.nq;
    P.xs = reinterpret_cast<float *>(b + L.xs);
    P.zs = reinterpret_cast<float *>(b + L.zs);
    P.hs = reinterpret_cast<float *>(b + L.hs);
    P.ns = reinterpret_cast<float *>(b + L.ns);
  }
  P.scores = r ? r->scores : nullptr;
  P.out_counts = r ? r->counts : nullptr;
  P.out_offsets = r ? r->offsets : nullptr;
  return P;
}

constexpr int kExpertBN = 256;  // token tile of the bf16 grouped GEMMs (Glu2Policy/Down2Policy kBN)

// Token tile and M tiles per group of the grouped GEMMs that follow.
struct GroupTiling {
  int bn, mt1, mt2;
};
// The 256-column e4m3 kernels lend registers between warpgroups
// (setmaxnreg), which is only sound when the kernel was built with exactly
// kW8LaunchRegs registers per thread: each instantiation's count is read once
// from its attributes, and one built with another count is never launched
// (the 128-column kernel runs instead).
template <class P>
bool wide8_ready() {
  static const bool ok = [] {
    cudaFuncAttributes a{};
    if (cudaFuncGetAttributes(&a, gemm8w_kernel<P>) != cudaSuccess) {
      (void)cudaGetLastError();
      return false;
    }
    return a.numRegs == kW8LaunchRegs;
  }();
  return ok;
}

// FP8 (not FP4) expert GEMMs on 256-column units: gate/up always, the expert
// down GEMM when d_lat splits into 256-wide slices.
bool fp8_wide_glu(const mrlmoe_config &c) {
  return c.dtype == MRLMOE_FP8_E4M3_BLOCK128 && wide8_ready<Glu8WPolicy>();
}
bool fp8_wide_down(const mrlmoe_config &c) {
  return c.dtype == MRLMOE_FP8_E4M3_BLOCK128 && c.d_lat % kW8N == 0 && wide8_ready<Down8WPolicy>();
}
// FP4 expert weights on the same 256-column units (the tensor core reads the
// e2m1 codes) when d_lat splits into 256-wide slices; else the 128-column
// kernel expands them to e4m3 in shared memory, with 64-token units.
bool fp4_wide(const mrlmoe_config &c) {
  return c.dtype == MRLMOE_FP4_E2M1_BLOCK128 && c.d_lat % kW8N == 0 && wide8_ready<Glu4WPolicy>() &&
         wide8_ready<Down4WPolicy>();
}

GroupTiling group_tiling(const mrlmoe_config &c) {
  if (c.dtype == MRLMOE_FP8_E4M3_BLOCK128)
    return {kF8Tile, c.d_ff / (fp8_wide_glu(c) ? 128 : 64), c.d_lat / (fp8_wide_down(c) ? kW8N : 128)};
  if (c.dtype == MRLMOE_FP4_E2M1_BLOCK128) {
    if (fp4_wide(c)) return {kF8Tile, c.d_ff / 128, c.d_lat / kW8N};
    return {kF4TokTile, c.d_ff / 64, c.d_lat / 128};
  }
  return {kExpertBN, glu_m_tiles(c), down_m_tiles(c)};
}

// counts -> offsets/group tables -> stable scatter (from topk_idx).
mrlmoe_status launch_dispatch(const mrlmoe_config &c, const Ptrs &P, cudaStream_t st) {
  const GroupTiling gtl = group_tiling(c);
  const int T = c.T, E = c.n_experts, k = c.top_k;
  const int nch = (T + kChunk - 1) / kChunk;
  const int wpb = 8;
  expert_mask_kernel<<<(nch + wpb - 1) / wpb, 32 * wpb, wpb * E * sizeof(uint32_t), st>>>(P.topk_idx, T, E, k,
                                                                                         P.mask, nch, P.status);
  MRL_TRY(cudaGetLastError());
  expert_colscan_kernel<<<(E + 31) / 32, 1024, 0, st>>>(P.mask, E, nch, P.base, P.counts_e, P.status);
  MRL_TRY(cudaGetLastError());
  expert_offsets_kernel<<<1, 1024, 0, st>>>(P.counts_e, T, E, k, gtl.bn, gtl.mt1, gtl.mt2, P.grp_off,
                                            P.grp_cnt, P.unit1, P.unit2, P.out_counts, P.out_offsets, P.status);
  MRL_TRY(cudaGetLastError());
  expert_scatter_kernel<<<(nch * 32 + 255) / 256, 256, 0, st>>>(P.topk_idx, P.mask, P.base, P.grp_off, T, E, k,
                                                                 nch, P.perm, P.inv, P.status);
  MRL_TRY(cudaGetLastError());
  return MRLMOE_OK;
}

mrlmoe_status check_weights_bf16(const mrlmoe_weights *w, bool need_all) {
  if (!w || !w->w_router || !w->expert_scale) return MRLMOE_ERR_INVALID_ARG;
  if (need_all) {
    const void *ps[] = {w->w_down, w->w_gate, w->w_up_e, w->w_down_e, w->w_sh_gate,
                        w->w_sh_up, w->w_sh_down, w->rms_gain, w->w_up};
    for (const void *p : ps)
      if (!p || !aligned16(p)) return MRLMOE_ERR_INVALID_ARG;
  }
  if (!aligned16(w->w_router)) return MRLMOE_ERR_INVALID_ARG;
  return MRLMOE_OK;
}

// FP8 / FP4 weights: every code matrix 16-byte aligned; with FP4 experts the
// six expert matrices 32-byte aligned (the 4-bit unpacking TMA type).
mrlmoe_status check_weights_fp8(const mrlmoe_weights *w, bool fp4) {
  if (!w || !w->w_router || !w->expert_scale || !w->rms_gain || !aligned16(w->w_router)) return MRLMOE_ERR_INVALID_ARG;
  const void *codes[] = {w->w_down, w->w_gate, w->w_up_e, w->w_down_e, w->w_sh_gate, w->w_sh_up, w->w_sh_down, w->w_up};
  const float *scales[] = {w->s_down, w->s_gate, w->s_up_e, w->s_down_e, w->s_sh_gate, w->s_sh_up, w->s_sh_down, w->s_up};
  for (const void *p : codes)
    if (!p || !aligned16(p)) return MRLMOE_ERR_INVALID_ARG;
  if (fp4)
    for (const void *p : {w->w_gate, w->w_up_e, w->w_down_e, w->w_sh_gate, w->w_sh_up, w->w_sh_down})
      if (reinterpret_cast<uintptr_t>(p) & 31u) return MRLMOE_ERR_INVALID_ARG;
  for (const float *p : scales)
    if (!p) return MRLMOE_ERR_INVALID_ARG;
  return MRLMOE_OK;
}

// Scales go to sc[rows][K/128], or transposed to sc[K/128][rows] (the layout
// the FP8 GEMMs read) when `transposed`.
cudaError_t launch_quant(const __nv_bfloat16 *in, long ld_in, int rows, int K, uint8_t *q, float *sc,
                         bool transposed, const uint32_t *status, cudaStream_t st) {
  quant_rows_kernel<<<(rows + kQuantWarps - 1) / kQuantWarps, kQuantWarps * 32, 0, st>>>(
      in, ld_in, rows, K, q, sc, transposed ? static_cast<long>(rows) : 0L, status);
  return cudaGetLastError();
}

// Top-k from fp32 scores with the running-list length that k needs.
cudaError_t launch_topk_from_scores(const float *s, const float *bias, const float *alpha, int T, int E, int k,
                                    int32_t *idx, float *w, float *wscaled, uint32_t *status,
                                    cudaStream_t st) {
  const int wpb = 8;
  const int grid = (T + wpb - 1) / wpb;
  if (k <= kTopKNarrow)
    topk_from_scores_kernel<kTopKNarrow><<<grid, 32 * wpb, 0, st>>>(s, bias, alpha, T, E, k, idx, w, wscaled, status);
  else
    topk_from_scores_kernel<kTopKMax><<<grid, 32 * wpb, 0, st>>>(s, bias, alpha, T, E, k, idx, w, wscaled, status);
  return cudaGetLastError();
}

template <class P>
cudaError_t launch_gemm8(const typename P::Params &p, int grid, cudaStream_t st) {
  static_assert(Gemm8Smem<P>::kTotal <= 232448, "GEMM shared memory above the 227 KB per-block limit");
  static std::atomic<bool> configured[kMaxDevices];
  cudaError_t e = set_smem_once(configured, gemm8_kernel<P>, Gemm8Smem<P>::kTotal);
  if (e != cudaSuccess) return e;
  gemm8_kernel<P><<<grid, kF8Threads, Gemm8Smem<P>::kTotal, st>>>(p);
  return cudaGetLastError();
}

template <class P>
cudaError_t launch_gemm8w(const typename P::Params &p, int grid, cudaStream_t st) {
  static_assert(Gemm8WSmem<P>::kTotal <= 232448, "GEMM shared memory above the 227 KB per-block limit");
  static std::atomic<bool> configured[kMaxDevices];
  cudaError_t e = set_smem_once(configured, gemm8w_kernel<P>, Gemm8WSmem<P>::kTotal);
  if (e != cudaSuccess) return e;
  gemm8w_kernel<P><<<grid, kF8Threads, Gemm8WSmem<P>::kTotal, st>>>(p);
  return cudaGetLastError();
}

// FP8 projection out = bf16(q(a) w^T) from e4m3 codes + scales (as_t: the
// activation scales transposed, [K/128, M]).
mrlmoe_status launch_dense8(const uint8_t *aq, const float *as_t, const void *wq, const float *ws, int M, int N, int K,
                            __nv_bfloat16 *out, __nv_bfloat16 *out_lo, const Ptrs &P, int sms, cudaStream_t st) {
  Dense8Policy::Params p{};
  if (!make_map(&p.ta, aq, 1, K, M, 128) || !make_map(&p.tb, wq, 1, K, N, kF8Tile)) return MRLMOE_ERR_CUDA;
  p.as_t = as_t;
  p.ws = ws;
  p.out = out;
  p.out_lo = out_lo;
  p.ldo = N;
  p.M = M; p.N = N; p.K = K;
  p.m_tiles = (M + 127) / 128;
  p.status = P.status;
  // 256-column units when they alone fill the SMs, else 128-column ones
  const int wide_units = p.m_tiles * ((N + kW8N - 1) / kW8N);
  if (wide_units >= sms && wide8_ready<Dense8WPolicy>()) {
    p.n_tiles = (N + kW8N - 1) / kW8N;
    MRL_TRY(launch_gemm8w<Dense8WPolicy>(p, std::min(sms, wide_units), st));
    return MRLMOE_OK;
  }
  p.n_tiles = (N + kF8Tile - 1) / kF8Tile;
  MRL_TRY(launch_gemm8<Dense8Policy>(p, std::min(sms, p.m_tiles * p.n_tiles), st));
  return MRLMOE_OK;
}

// bf16 projection out = bf16(a w^T) (and optionally the residual of that
// rounding): 256-column tiles, or 64-column tiles when the 256-wide grid would
// occupy fewer than half the SMs (decode-sized M).
template <class DP>
mrlmoe_status launch_dense_with(const void *a, const void *w, __nv_bfloat16 *out, __nv_bfloat16 *out_lo, int M, int N,
                                int K, uint32_t *status, int sms, cudaStream_t st) {
  typename DP::Params p{};
  if (!make_map(&p.ta, a, 2, K, M, 128) || !make_map(&p.tb, w, 2, K, N, DP::kBN)) return MRLMOE_ERR_CUDA;
  p.out = out;
  p.out_lo = out_lo;
  p.ldo = N;
  p.M = M; p.N = N; p.K = K;
  p.m_tiles = (M + 127) / 128;
  p.n_tiles = (N + DP::kBN - 1) / DP::kBN;
  p.status = status;
  MRL_TRY(launch_gemm<DP>(p, std::min(sms, p.m_tiles * p.n_tiles), st));
  return MRLMOE_OK;
}

// The same on CTA pairs (M = 256 per unit; Dense2Policy).
mrlmoe_status launch_dense_pair(const void *a, const void *w, __nv_bfloat16 *out, __nv_bfloat16 *out_lo, int M, int N,
                                int K, uint32_t *status, int sms, cudaStream_t st) {
  Dense2Policy::Params p{};
  if (!make_map(&p.ta, a, 2, K, M, 128) || !make_map(&p.tb, w, 2, K, N, Dense2Policy::kBN / 2)) return MRLMOE_ERR_CUDA;
  p.out = out;
  p.out_lo = out_lo;
  p.ldo = N;
  p.M = M; p.N = N; p.K = K;
  p.m_tiles = (M + 255) / 256;
  p.n_tiles = (N + Dense2Policy::kBN - 1) / Dense2Policy::kBN;
  p.status = status;
  MRL_TRY(launch_gemm_pair<Dense2Policy>(p, std::min(sms, 2 * p.m_tiles * p.n_tiles), st));
  return MRLMOE_OK;
}

// bf16 projection: 64-column one-CTA tiles when 256-wide tiles would occupy
// fewer than half the SMs (decode-sized M), else 256 x 256 tiles on CTA pairs.
mrlmoe_status launch_dense_bf16(const void *a, const void *w, __nv_bfloat16 *out, __nv_bfloat16 *out_lo, int M,
                                int N, int K, uint32_t *status, int sms, cudaStream_t st) {
  const int wide_tiles = ((M + 127) / 128) * ((N + DensePolicy::kBN - 1) / DensePolicy::kBN);
  if (2 * wide_tiles < sms && N % DenseNarrowPolicy::kBN == 0)
    return launch_dense_with<DenseNarrowPolicy>(a, w, out, out_lo, M, N, K, status, sms, st);
  return launch_dense_pair(a, w, out, out_lo, M, N, K, status, sms, st);
}

// Routing from x: down-projection into the tail of zbuf, then the fused router.
mrlmoe_status launch_project_and_route(const mrlmoe_config &c, const mrlmoe_weights *w, const float *bias,
                                       const void *x, const Ptrs &P, int sms, cudaStream_t st,
                                       void *const *ev = nullptr) {
  const int T = c.T, D = c.d_model, Ld = c.d_lat, E = c.n_experts, R = c.n_routers, k = c.top_k;
  __nv_bfloat16 *z = P.zbuf + static_cast<size_t>(T) * k * Ld;  // z rows live after the T*k dispatched rows
  if (c.dtype != MRLMOE_BF16) {
    MRL_TRY(launch_quant(static_cast<const __nv_bfloat16 *>(x), D, T, D, P.xq, P.xs, true, P.status, st));
    mrlmoe_status s = launch_dense8(P.xq, P.xs, w->w_down, w->s_down, T, Ld, D, z, P.zlo, P, sms, st);
    if (s != MRLMOE_OK) return s;
  } else {
    mrlmoe_status s = launch_dense_bf16(x, w->w_down, z, P.zlo, T, Ld, D, P.status, sms, st);
    if (s != MRLMOE_OK) return s;
  }
  nvtx_stage(kForwardStages[1]);
  if (ev) MRL_TRY(cudaEventRecord(static_cast<cudaEvent_t>(ev[1]), st));
  {
    RouterParams p{};
    const int ec = router_ec(E, R, T);
    if (!make_map(&p.ta, z, 2, Ld, T, 128) || !make_map(&p.ta_lo, P.zlo, 2, Ld, T, 128) ||
        !make_map(&p.tb, w->w_router, 2, Ld, static_cast<uint64_t>(R) * E, ec))
      return MRLMOE_ERR_CUDA;
    p.bias = bias;
    p.alpha = w->expert_scale;
    p.topk_idx = P.topk_idx;
    p.topk_w = P.topk_w;
    p.wscaled = P.wscaled;
    p.scores = P.scores;
    p.cand_v = P.cand_v;
    p.cand_s = P.cand_s;
    p.cand_i = P.cand_i;
    p.T = T; p.L = Ld; p.E = E; p.R = R; p.ec = ec; p.k = k;
    p.agg = static_cast<int>(c.aggregation);
    p.m_tiles = (T + 127) / 128;
    p.status = P.status;
    const int ks = router_ksplit(c);
    if (ks > 1) {
      // few token tiles: split K over the CTAs, then finish per token
      p.part = P.rpart;
      p.ksplit = ks;
      p.parts = 1;
      MRL_TRY(launch_gemm<RouterSplitPolicy>(p, std::min(sms, p.m_tiles * (E / ec) * ks), st));
      float *s = P.scores ? P.scores : P.rpart + static_cast<size_t>(ks) * T * R * E;
      const long long n = static_cast<long long>(T) * E;
      router_split_scores_kernel<<<static_cast<int>((n + 255) / 256), 256, 0, st>>>(P.rpart, ks, T, E, R, p.agg, s,
                                                                                    P.status);
      MRL_TRY(cudaGetLastError());
      MRL_TRY(launch_topk_from_scores(s, bias, w->expert_scale, T, E, k, P.topk_idx, P.topk_w, P.wscaled, P.status,
                                      st));
      return MRLMOE_OK;
    }
    p.parts = router_parts(c, sms);
    const int grid = std::min(sms, p.m_tiles * p.parts);
    if (k <= kTopKNarrow)
      MRL_TRY(launch_gemm<RouterPolicy>(p, grid, st));
    else
      MRL_TRY(launch_gemm<RouterPolicyWide>(p, grid, st));
    if (p.parts > 1) {
      if (k <= kTopKNarrow)
        topk_merge_kernel<kTopKNarrow><<<(T + 127) / 128, 128, 0, st>>>(
            P.cand_v, P.cand_s, P.cand_i, T, E, p.parts, k, w->expert_scale, P.topk_idx, P.topk_w, P.wscaled,
            P.status);
      else
        topk_merge_kernel<kTopKMax><<<(T + 127) / 128, 128, 0, st>>>(
            P.cand_v, P.cand_s, P.cand_i, T, E, p.parts, k, w->expert_scale, P.topk_idx, P.topk_w, P.wscaled,
            P.status);
      MRL_TRY(cudaGetLastError());
    }
  }
  return MRLMOE_OK;
}

// FP8 variant after the dispatch record: quantised gather of the dispatched
// latent rows, gate/up, quantised h, expert down, combine + RMSNorm,
// quantised n, up-projection.  Stage events 4..7 as in the bf16 sequence.
// Combine + RMSNorm of the T tokens' slots into nbuf, instantiated for the
// float4s each of the 256 threads holds (d_lat <= 1024 / 2048 / 4096 / 8192).
cudaError_t launch_combine(const Ptrs &P, int T, int Ld, int k, float eps, const void *gain, cudaStream_t st) {
  const float4 *slots = reinterpret_cast<const float4 *>(P.slots);
  const float4 *g = reinterpret_cast<const float4 *>(gain);
  const int L4 = Ld / 4;
  if (L4 <= kCombineThreads)
    combine_rmsnorm_kernel<1><<<T, kCombineThreads, 0, st>>>(slots, Ld, k, eps, g, P.nbuf, P.status);
  else if (L4 <= 2 * kCombineThreads)
    combine_rmsnorm_kernel<2><<<T, kCombineThreads, 0, st>>>(slots, Ld, k, eps, g, P.nbuf, P.status);
  else if (L4 <= 4 * kCombineThreads)
    combine_rmsnorm_kernel<4><<<T, kCombineThreads, 0, st>>>(slots, Ld, k, eps, g, P.nbuf, P.status);
  else
    combine_rmsnorm_kernel<kCombineMaxV4><<<T, kCombineThreads, 0, st>>>(slots, Ld, k, eps, g, P.nbuf, P.status);
  return cudaGetLastError();
}

// The T*k dispatched bf16 latent rows, in dispatch order, into dst from z
// (rows [T*k, T*k + T) of zbuf).  One warp per token while the batch gives
// at least 16 warps per SM; a smaller batch splits each token's k
// destinations over up to k warps.
cudaError_t launch_copy_dispatch_rows(const Ptrs &P, int T, int Ld, int k, void *dst, int sms, cudaStream_t st) {
  const int Tk = T * k;
  const int nsplit = std::min(k, std::max(1, (16 * sms + T - 1) / T));
  const long long warps = static_cast<long long>(T) * nsplit;
  copy_dispatch_rows_kernel<<<static_cast<unsigned>((warps + kCopyWarps - 1) / kCopyWarps), kCopyWarps * 32, 0, st>>>(
      reinterpret_cast<const uint4 *>(P.zbuf + static_cast<size_t>(Tk) * Ld), T, Ld * 2 / 16, P.inv, k, nsplit, Tk,
      static_cast<uint4 *>(dst), P.status);
  return cudaGetLastError();
}

mrlmoe_status forward_experts_fp8(const mrlmoe_config &c, const mrlmoe_weights *w, const Ptrs &P, int sms,
                                  cudaStream_t st, void *const *ev, void *y_out = nullptr);

mrlmoe_status forward_impl(const mrlmoe_config *cfg, const mrlmoe_weights *w, const float *bias, const void *x,
                           void *y, mrlmoe_routing *route_out, void *workspace, size_t ws_bytes, void *stream,
                           void *const *ev, bool train = false) {
  mrlmoe_status s = check_config(cfg);
  if (s != MRLMOE_OK) return s;
  if (train && !train_supported(*cfg)) return MRLMOE_ERR_UNSUPPORTED;
  if (!bias || !x || !y || !aligned16(x) || !aligned16(y)) return MRLMOE_ERR_INVALID_ARG;
  const bool fp8 = cfg->dtype != MRLMOE_BF16;  // e4m3 projections and activations (FP8 and FP4 variants)
  if ((s = fp8 ? check_weights_fp8(w, cfg->dtype == MRLMOE_FP4_E2M1_BLOCK128) : check_weights_bf16(w, true)) !=
      MRLMOE_OK)
    return s;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return MRLMOE_ERR_WORKSPACE;
  if (ws_bytes < layout_of(*cfg, train).total) return MRLMOE_ERR_WORKSPACE;
  int sms = 0;
  DeviceRestore restore;
  if ((s = bind_device(workspace, &sms, &restore)) != MRLMOE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the training forward keeps the routing record in the workspace (the
  // backward reads it there) and copies it to route_out afterwards
  Ptrs P = carve(*cfg, workspace, train ? nullptr : route_out);
  if (train && route_out) {
    P.scores = route_out->scores;
    P.out_counts = route_out->counts;
    P.out_offsets = route_out->offsets;
  }
  const int T = cfg->T, D = cfg->d_model, Ld = cfg->d_lat, F = cfg->d_ff, E = cfg->n_experts, k = cfg->top_k;
  const Layout LT = layout_of(*cfg, train);
  const int Tk = T * k;
  if ((s = init_header(P.status, cfg->hold, st)) != MRLMOE_OK) return s;
  NvtxCall nvtx_call(train ? "mrlmoe_forward_train" : "mrlmoe_forward");
  auto mark = [&](int i) -> bool {
    nvtx_stage(i < 8 ? kForwardStages[i] : nullptr);
    return !ev || cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), st) == cudaSuccess;
  };

  if (!mark(0)) return MRLMOE_ERR_CUDA;
  if ((s = launch_project_and_route(*cfg, w, bias, x, P, sms, st, ev)) != MRLMOE_OK) return s;
  if (!mark(2)) return MRLMOE_ERR_CUDA;
  if ((s = launch_dispatch(*cfg, P, st)) != MRLMOE_OK) return s;
  if (train && route_out) {
    const size_t n = static_cast<size_t>(T) * k * 4;
    if (route_out->topk_idx) MRL_TRY(cudaMemcpyAsync(route_out->topk_idx, P.topk_idx, n, cudaMemcpyDeviceToDevice, st));
    if (route_out->topk_w) MRL_TRY(cudaMemcpyAsync(route_out->topk_w, P.topk_w, n, cudaMemcpyDeviceToDevice, st));
    if (route_out->perm) MRL_TRY(cudaMemcpyAsync(route_out->perm, P.perm, n, cudaMemcpyDeviceToDevice, st));
    if (route_out->inv_perm) MRL_TRY(cudaMemcpyAsync(route_out->inv_perm, P.inv, n, cudaMemcpyDeviceToDevice, st));
  }
  if (!mark(3)) return MRLMOE_ERR_CUDA;
  if (fp8) {
    if ((s = forward_experts_fp8(*cfg, w, P, sms, st, ev, y)) != MRLMOE_OK) return s;
    if (!mark(8)) return MRLMOE_ERR_CUDA;
    return MRLMOE_OK;
  }

  // gather the dispatched latent rows (rows [0, T*k) of zbuf) from z (rows [T*k, T*k+T))
  MRL_TRY(launch_copy_dispatch_rows(P, T, Ld, k, P.zbuf, sms, st));
  if (!mark(4)) return MRLMOE_ERR_CUDA;
  GroupTable gt1{P.grp_off, P.grp_cnt, P.unit1, E, glu_m_tiles(*cfg)};
  GroupTable gt2{P.grp_off, P.grp_cnt, P.unit2, E, down_m_tiles(*cfg)};
  {
    GluParams p{};
    if (!make_map(&p.wg, w->w_gate, 2, Ld, static_cast<uint64_t>(E) * F, 64) ||
        !make_map(&p.wu, w->w_up_e, 2, Ld, static_cast<uint64_t>(E) * F, 64) ||
        !make_map(&p.sg, w->w_sh_gate, 2, Ld, F, 64) || !make_map(&p.su, w->w_sh_up, 2, Ld, F, 64) ||
        !make_token_maps(&p.tz, P.zbuf, Ld, static_cast<uint64_t>(Tk) + T))
      return MRLMOE_ERR_CUDA;
    p.gt = gt1;
    p.h = P.hbuf;
    if (train) p.gu = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(workspace) + LT.gusave);
    p.F = F; p.L = Ld; p.rows = Tk + T;
    p.status = P.status;
    MRL_TRY(launch_gemm_pair<Glu2Policy>(p, sms, st));
  }
  if (!mark(5)) return MRLMOE_ERR_CUDA;
  {
    DownPolicy::Params p{};
    if (!make_map(&p.wd, w->w_down_e, 2, F, static_cast<uint64_t>(E) * Ld, 128) ||
        !make_map(&p.sd, w->w_sh_down, 2, F, Ld, 128) ||
        !make_token_maps_blocked(&p.th, P.hbuf, F, static_cast<uint64_t>(Tk) + T))
      return MRLMOE_ERR_CUDA;
    p.gt = gt2;
    p.perm = P.perm;
    p.wscaled = P.wscaled;
    p.slots = P.slots;
    p.L = Ld; p.F = F; p.k = k; p.Tk = Tk;
    p.status = P.status;
    if (down_uses_pairs(*cfg))
      MRL_TRY(launch_gemm_pair<Down2Policy>(p, sms, st));
    else
      MRL_TRY(launch_gemm<DownPolicy>(p, sms, st));
  }
  if (!mark(6)) return MRLMOE_ERR_CUDA;
  MRL_TRY(launch_combine(P, T, Ld, k, cfg->rms_eps, w->rms_gain, st));
  if (!mark(7)) return MRLMOE_ERR_CUDA;
  {
    mrlmoe_status s = launch_dense_bf16(P.nbuf, w->w_up, static_cast<__nv_bfloat16 *>(y), nullptr, T, D, Ld,
                                        P.status, sms, st);
    if (s != MRLMOE_OK) return s;
  }
  if (!mark(8)) return MRLMOE_ERR_CUDA;
  return MRLMOE_OK;
}

mrlmoe_status forward_experts_fp8(const mrlmoe_config &c, const mrlmoe_weights *w, const Ptrs &P, int sms,
                                  cudaStream_t st, void *const *ev, void *y_out) {
  const int T = c.T, D = c.d_model, Ld = c.d_lat, F = c.d_ff, E = c.n_experts, k = c.top_k;
  const int Tk = T * k;
  auto mark = [&](int i) -> bool {
    nvtx_stage(i < 8 ? kForwardStages[i] : nullptr);
    return !ev || cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), st) == cudaSuccess;
  };
  // quantised dispatched latent rows (rows < T*k) and the shared expert's rows
  // (all T tokens): each token's latent row quantised once, written to its rows
  quant_dispatch_rows_kernel<<<(T + kQuantWarps - 1) / kQuantWarps, kQuantWarps * 32, 0, st>>>(
      P.zbuf + static_cast<size_t>(Tk) * Ld, T, Ld, P.inv, k, Tk, P.zq, P.zs, static_cast<long>(Tk) + T, P.status);
  MRL_TRY(cudaGetLastError());
  if (!mark(4)) return MRLMOE_ERR_CUDA;
  const GroupTiling gtl = group_tiling(c);
  const bool fp4 = c.dtype == MRLMOE_FP4_E2M1_BLOCK128;  // expert matrices as packed e2m1 codes
  // an expert weight map: e4m3 [rows, K] with 128-byte boxes, or packed e2m1 [rows, K/2] with 64-byte boxes
  auto wmap = [&](CUtensorMap *m, const void *base, uint64_t K, uint64_t rows, uint32_t box_rows) {
    return fp4 ? make_map_packed(m, base, K / 2, rows, box_rows) : make_map(m, base, 1, K, rows, box_rows);
  };
  const bool wide4 = fp4_wide(c);
  if (fp8_wide_glu(c) || wide4) {
    // 128 gate + 128 up rows per unit (64-row quarters); h is quantised in the epilogue
    Glu8WPolicy::Params p{};
    auto wmapw = [&](CUtensorMap *m, const void *base, uint64_t rows) {
      return wide4 ? make_map_e2m1(m, base, Ld, rows, 64) : make_map(m, base, 1, Ld, rows, 64);
    };
    const uint64_t EF = static_cast<uint64_t>(E) * F;
    if (!wmapw(&p.wg, w->w_gate, EF) || !wmapw(&p.wu, w->w_up_e, EF) || !wmapw(&p.sg, w->w_sh_gate, F) ||
        !wmapw(&p.su, w->w_sh_up, F) ||
        !make_token_maps8(&p.tz, P.zq, Ld, static_cast<uint64_t>(Tk) + T))
      return MRLMOE_ERR_CUDA;
    p.wg_s = w->s_gate; p.wu_s = w->s_up_e; p.sg_s = w->s_sh_gate; p.su_s = w->s_sh_up;
    p.zs_t = P.zs;
    p.rows = Tk + T;
    p.gt = GroupTable{P.grp_off, P.grp_cnt, P.unit1, E, gtl.mt1};
    p.hq = P.hq;
    p.hs_t = P.hs;
    p.F = F; p.L = Ld;
    p.status = P.status;
    if (wide4)
      MRL_TRY(launch_gemm8w<Glu4WPolicy>(p, sms, st));
    else
      MRL_TRY(launch_gemm8w<Glu8WPolicy>(p, sms, st));
  } else {
    Glu8Policy::Params p{};
    if (!wmap(&p.wg, w->w_gate, Ld, static_cast<uint64_t>(E) * F, 64) ||
        !wmap(&p.wu, w->w_up_e, Ld, static_cast<uint64_t>(E) * F, 64) ||
        !wmap(&p.sg, w->w_sh_gate, Ld, F, 64) || !wmap(&p.su, w->w_sh_up, Ld, F, 64) ||
        !make_token_maps8(&p.tz, P.zq, Ld, static_cast<uint64_t>(Tk) + T))
      return MRLMOE_ERR_CUDA;
    p.wg_s = w->s_gate; p.wu_s = w->s_up_e; p.sg_s = w->s_sh_gate; p.su_s = w->s_sh_up;
    p.zs_t = P.zs;
    p.rows = Tk + T;
    p.gt = GroupTable{P.grp_off, P.grp_cnt, P.unit1, E, gtl.mt1};
    p.h = P.hbuf;
    p.F = F; p.L = Ld;
    p.status = P.status;
    if (fp4)
      MRL_TRY(launch_gemm8<Glu4Policy>(p, sms, st));
    else
      MRL_TRY(launch_gemm8<Glu8Policy>(p, sms, st));
    MRL_TRY(launch_quant(P.hbuf, F, Tk + T, F, P.hq, P.hs, true, P.status, st));
  }
  if (!mark(5)) return MRLMOE_ERR_CUDA;
  {
    Down8Policy::Params p{};
    if (wide4 ? !make_map_e2m1(&p.wd, w->w_down_e, F, static_cast<uint64_t>(E) * Ld, 128) ||
                    !make_map_e2m1(&p.sd, w->w_sh_down, F, Ld, 128)
              : !wmap(&p.wd, w->w_down_e, F, static_cast<uint64_t>(E) * Ld, 128) ||
                    !wmap(&p.sd, w->w_sh_down, F, Ld, 128))
      return MRLMOE_ERR_CUDA;
    if (!make_token_maps8(&p.th, P.hq, F, static_cast<uint64_t>(Tk) + T)) return MRLMOE_ERR_CUDA;
    p.wd_s = w->s_down_e; p.sd_s = w->s_sh_down;
    p.hs_t = P.hs;
    p.rows = Tk + T;
    p.gt = GroupTable{P.grp_off, P.grp_cnt, P.unit2, E, gtl.mt2};
    p.perm = P.perm;
    p.wscaled = P.wscaled;
    p.slots = P.slots;
    p.L = Ld; p.F = F; p.k = k; p.Tk = Tk;
    p.status = P.status;
    if (wide4)
      MRL_TRY(launch_gemm8w<Down4WPolicy>(p, sms, st));
    else if (fp4)
      MRL_TRY(launch_gemm8<Down4Policy>(p, sms, st));
    else if (fp8_wide_down(c))
      MRL_TRY(launch_gemm8w<Down8WPolicy>(p, sms, st));
    else
      MRL_TRY(launch_gemm8<Down8Policy>(p, sms, st));
  }
  if (!mark(6)) return MRLMOE_ERR_CUDA;
  MRL_TRY(launch_combine(P, T, Ld, k, c.rms_eps, w->rms_gain, st));
  MRL_TRY(launch_quant(P.nbuf, Ld, T, Ld, P.nq, P.ns, true, P.status, st));
  if (!mark(7)) return MRLMOE_ERR_CUDA;
  return launch_dense8(P.nq, P.ns, w->w_up, w->s_up, T, D, Ld, static_cast<__nv_bfloat16 *>(y_out), nullptr, P, sms,
                       st);
}

// ------------------------------------------------------------ backward
template <class DP>
mrlmoe_status launch_dense_grad(const CUtensorMap &ta, const CUtensorMap &tb, void *out, int M, int N, int K,
                                uint32_t *status, int sms, cudaStream_t st, int accumulate = 0) {
  typename DP::Params p{};
  p.accumulate = accumulate;
  p.ta = ta;
  p.tb = tb;
  p.out = out;
  p.ldo = N;
  p.M = M; p.N = N; p.K = K;
  p.m_tiles = (M + 127) / 128;
  p.n_tiles = (N + DP::kBN - 1) / DP::kBN;
  p.status = status;
  MRL_TRY(launch_gemm<DP>(p, std::min(sms, p.m_tiles * p.n_tiles), st));
  return MRLMOE_OK;
}

mrlmoe_status backward_impl(const mrlmoe_config *cfg, const mrlmoe_weights *w, const void *x, const void *dy,
                            const mrlmoe_grads *g, void *workspace, size_t ws_bytes, void *stream,
                            void *const *ev = nullptr) {
  mrlmoe_status s = check_config(cfg);
  if (s != MRLMOE_OK) return s;
  if (!train_supported(*cfg)) return MRLMOE_ERR_UNSUPPORTED;
  if (!x || !dy || !g || !aligned16(x) || !aligned16(dy)) return MRLMOE_ERR_INVALID_ARG;
  if ((s = check_weights_bf16(w, true)) != MRLMOE_OK) return s;
  {
    const void *outs[] = {g->dx, g->d_w_down, g->d_w_router, g->d_w_gate, g->d_w_up_e, g->d_w_down_e,
                          g->d_w_sh_gate, g->d_w_sh_up, g->d_w_sh_down, g->d_rms_gain, g->d_w_up, g->d_expert_scale};
    for (const void *o : outs)
      if (!o || !aligned16(o)) return MRLMOE_ERR_INVALID_ARG;
  }
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return MRLMOE_ERR_WORKSPACE;
  const Layout LT = layout_of(*cfg, true);
  if (ws_bytes < LT.total) return MRLMOE_ERR_WORKSPACE;
  int sms = 0;
  DeviceRestore restore;
  if ((s = bind_device(workspace, &sms, &restore)) != MRLMOE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Ptrs P = carve(*cfg, workspace, nullptr);
  uint8_t *b = static_cast<uint8_t *>(workspace);
  const int T = cfg->T, D = cfg->d_model, Ld = cfg->d_lat, F = cfg->d_ff, E = cfg->n_experts, k = cfg->top_k;
  const int R = cfg->n_routers, Tk = T * k, rows = Tk + T;
  const int acc = g->accumulate != 0;  // weight gradients: add instead of overwrite
  auto bf = [&](size_t off) { return reinterpret_cast<__nv_bfloat16 *>(b + off); };
  auto f32 = [&](size_t off) { return reinterpret_cast<float *>(b + off); };
  auto i32 = [&](size_t off) { return reinterpret_cast<int32_t *>(b + off); };
  const uint32_t *gusave = reinterpret_cast<const uint32_t *>(b + LT.gusave);
  __nv_bfloat16 *dcd = bf(LT.dcd), *dod = bf(LT.dod);
  __nv_bfloat16 *dgu = bf(LT.dgu), *dzx = bf(LT.dzx);
  float *dn = f32(LT.dn), *dwsp = f32(LT.dwsp), *wrow = f32(LT.wrow), *dl = f32(LT.dl), *aw = f32(LT.aw), *gpart = f32(LT.gpart);
  const __nv_bfloat16 *zhi = P.zbuf + static_cast<size_t>(Tk) * Ld;
  NvtxCall nvtx_call("mrlmoe_backward");
  auto mark = [&](int i) -> bool {
    nvtx_stage(i < 10 ? kBackwardStages[i] : nullptr);
    return !ev || cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), st) == cudaSuccess;
  };
  // the call continues the forward's status word; only this call's hold mask is set
  MRL_TRY(cudaMemsetAsync(reinterpret_cast<uint8_t *>(P.status) + 4, static_cast<int>(cfg->hold & 0xffu), 1, st));
  if (!mark(0)) return MRLMOE_ERR_CUDA;

  // dn = dy W_up (W_up [D, Ld] MN-major); dW_up = dy^T n (both MN-major, K = T)
  {
    CUtensorMap ta, tb;
    if (!make_map(&ta, dy, 2, D, T, 128) || !make_map(&tb, w->w_up, 2, Ld, D, 64)) return MRLMOE_ERR_CUDA;
    if ((s = launch_dense_grad<DenseGradPolicy<false, true, true>>(ta, tb, dn, T, Ld, D, P.status, sms, st)) !=
        MRLMOE_OK)
      return s;
    if (!mark(1)) return MRLMOE_ERR_CUDA;
    if (!make_map(&ta, dy, 2, D, T, 64) || !make_map(&tb, P.nbuf, 2, Ld, T, 64)) return MRLMOE_ERR_CUDA;
    if ((s = launch_dense_grad<DenseGradPolicy<true, true, true>>(ta, tb, g->d_w_up, D, Ld, T, P.status, sms, st,
                                                                    acc)) != MRLMOE_OK)
      return s;
  }
  if (!mark(2)) return MRLMOE_ERR_CUDA;
  // RMSNorm + combine backward: dc rows (plain and weighted) per dispatch row
  const int nb = rms_bwd_blocks(*cfg);
  {
    auto kern = Ld <= 4 * kBwdThreads * 2 ? rms_combine_bwd_kernel<2>
              : Ld <= 4 * kBwdThreads * 4 ? rms_combine_bwd_kernel<4> : rms_combine_bwd_kernel<kBwdMaxV4>;
    kern<<<nb, kBwdThreads, 0, st>>>(reinterpret_cast<const float4 *>(P.slots), reinterpret_cast<const float4 *>(dn),
                                     reinterpret_cast<const float4 *>(w->rms_gain), P.inv, P.wscaled, T, Ld, k,
                                     cfg->rms_eps, dcd, dod, wrow, reinterpret_cast<float4 *>(gpart), P.status);
  }
  MRL_TRY(cudaGetLastError());
  gain_reduce_kernel<<<(Ld + 255) / 256, 256, 0, st>>>(gpart, nb, Ld, g->d_rms_gain, acc, P.status);
  MRL_TRY(cudaGetLastError());
  if (!mark(3)) return MRLMOE_ERR_CUDA;
  // unit tables of the two grouped dgrad GEMMs (token tiles of 256; d_ff / 128 and d_lat / 128 M tiles)
  int32_t *bgo = i32(LT.bgrp_off), *bgc = i32(LT.bgrp_cnt), *bu1 = i32(LT.bunit1), *bu2 = i32(LT.bunit2);
  const bool dz_pairs = Ld % 256 == 0;  // the dz GEMM on CTA pairs (256-wide d_lat slices)
  expert_offsets_kernel<<<1, 1024, 0, st>>>(P.counts_e, T, E, k, DhPolicy::kBN, F / 128,
                                            dz_pairs ? Ld / 256 : Ld / 128, bgo, bgc, bu1, bu2, nullptr, nullptr,
                                            P.status);
  MRL_TRY(cudaGetLastError());
  {
    DhPolicy::Params p{};
    if (!make_map(&p.wd, w->w_down_e, 2, F, static_cast<uint64_t>(E) * Ld, 64) ||
        !make_map(&p.sd, w->w_sh_down, 2, F, Ld, 64) || !make_token_maps(&p.tc, dcd, Ld, rows))
      return MRLMOE_ERR_CUDA;
    p.gt = GroupTable{bgo, bgc, bu1, E, F / 128};
    p.wrow = wrow;
    p.gu = gusave;
    p.dgu = dgu;
    p.dwsp = dwsp;
    p.L = Ld; p.F = F; p.rows = rows;
    p.status = P.status;
    MRL_TRY(launch_gemm<DhPolicy>(p, sms, st));
  }
  if (!mark(4)) return MRLMOE_ERR_CUDA;
  {
    DzPolicy::Params p{};
    if (!make_map(&p.wg, w->w_gate, 2, Ld, static_cast<uint64_t>(E) * F, 64) ||
        !make_map(&p.wu, w->w_up_e, 2, Ld, static_cast<uint64_t>(E) * F, 64) ||
        !make_map(&p.sg, w->w_sh_gate, 2, Ld, F, 64) || !make_map(&p.su, w->w_sh_up, 2, Ld, F, 64) ||
        !make_token_maps_blocked(&p.tgu, dgu, 2 * F, rows))
      return MRLMOE_ERR_CUDA;
    p.gt = GroupTable{bgo, bgc, bu2, E, dz_pairs ? Ld / 256 : Ld / 128};
    p.perm = P.perm;
    p.dzs = P.slots;  // the forward's slots were consumed by rms_combine_bwd_kernel
    p.L = Ld; p.F = F; p.k = k; p.Tk = Tk;
    p.status = P.status;
    if (dz_pairs)
      MRL_TRY(launch_gemm_pair<Dz2Policy>(p, sms, st));
    else
      MRL_TRY(launch_gemm<DzPolicy>(p, sms, st));
  }
  if (!mark(5)) return MRLMOE_ERR_CUDA;
  // routers, combine weights, alpha; dz reduced per token
  token_bwd_kernel<<<T, kBwdThreads, Ld * sizeof(float), st>>>(
      dwsp, F / 128, rows, P.inv, P.topk_idx, P.topk_w, w->expert_scale, zhi, P.zlo,
      static_cast<const __nv_bfloat16 *>(w->w_router), P.slots, T, Ld, E, R, k, static_cast<int>(cfg->aggregation),
      dzx, dl, aw, P.status);
  MRL_TRY(cudaGetLastError());
  if (!mark(6)) return MRLMOE_ERR_CUDA;
  expert_param_bwd_kernel<<<E, kBwdThreads, 0, st>>>(P.grp_off, P.grp_cnt, P.perm, dl, aw, zhi, P.zlo, Ld, E, R, k,
                                                     g->d_w_router, g->d_expert_scale, acc, P.status);
  MRL_TRY(cudaGetLastError());
  if (!mark(7)) return MRLMOE_ERR_CUDA;
  // expert weight gradients (K = each group's rows)
  {
    WgradPolicy::Params p{};
    if (!make_map(&p.tdgu, dgu, 2, 64, static_cast<uint64_t>(2 * F / 64) * rows, 64) ||
        !make_map(&p.tz, P.zbuf, 2, Ld, rows, 64) || !make_map(&p.tdo, dod, 2, Ld, rows, 64) ||
        !make_map(&p.th, P.hbuf, 2, 64, static_cast<uint64_t>(F / 64) * rows, 64))
      return MRLMOE_ERR_CUDA;
    const uint64_t EF = static_cast<uint64_t>(E) * F, EL = static_cast<uint64_t>(E) * Ld;
    if (!make_map_f32_out(&p.og, g->d_w_gate, Ld, EF) || !make_map_f32_out(&p.ou, g->d_w_up_e, Ld, EF) ||
        !make_map_f32_out(&p.od, g->d_w_down_e, F, EL) || !make_map_f32_out(&p.sog, g->d_w_sh_gate, Ld, F) ||
        !make_map_f32_out(&p.sou, g->d_w_sh_up, Ld, F) || !make_map_f32_out(&p.sod, g->d_w_sh_down, F, Ld))
      return MRLMOE_ERR_CUDA;
    p.grp_off = P.grp_off;
    p.accumulate = acc;
    p.E = E; p.F = F; p.L = Ld; p.rows = rows;
    p.status = P.status;
    MRL_TRY(launch_gemm<WgradPolicy>(p, sms, st));
  }
  if (!mark(8)) return MRLMOE_ERR_CUDA;
  // dx = dzx W_dn (W_dn [Ld, D] MN-major); dW_dn = dzx^T x (K = T)
  {
    CUtensorMap ta, tb;
    if (!make_map(&ta, dzx, 2, Ld, T, 128) || !make_map(&tb, w->w_down, 2, D, Ld, 64)) return MRLMOE_ERR_CUDA;
    if ((s = launch_dense_grad<DenseGradPolicy<false, true, false>>(ta, tb, g->dx, T, D, Ld, P.status, sms, st)) !=
        MRLMOE_OK)
      return s;
    if (!mark(9)) return MRLMOE_ERR_CUDA;
    if (!make_map(&ta, dzx, 2, Ld, T, 64) || !make_map(&tb, x, 2, D, T, 64)) return MRLMOE_ERR_CUDA;
    if ((s = launch_dense_grad<DenseGradPolicy<true, true, true>>(ta, tb, g->d_w_down, Ld, D, T, P.status, sms,
                                                                    st, acc)) != MRLMOE_OK)
      return s;
  }
  if (!mark(10)) return MRLMOE_ERR_CUDA;
  return MRLMOE_OK;
}

// ------------------------------------------------ static-scratch routing
// Scratch for mrlmoe_route_scores_static: one array per device that loads
// the library.  Host code never dereferences this symbol; it asks the runtime
// for the device address once per device (static_scratch()).
static __device__ __align__(256) uint8_t g_route_scratch[MRLMOE_STATIC_SCRATCH_BYTES];

struct StaticRouteLayout {
  size_t status, wscaled, counts, grp_off, grp_cnt, unit1, unit2, mask, base, total;
};

StaticRouteLayout static_route_layout(const mrlmoe_config &c) {
  StaticRouteLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += (bytes + 255) & ~size_t(255);
    return o;
  };
  const size_t T = c.T, k = c.top_k, E = c.n_experts, nch = (T + kChunk - 1) / kChunk;
  L.status = take(256);
  L.wscaled = take(T * k * 4);
  L.counts = take((E + 2) * 4);
  L.grp_off = take((E + 2) * 4);
  L.grp_cnt = take((E + 2) * 4);
  L.unit1 = take((E + 2) * 4);
  L.unit2 = take((E + 2) * 4);
  L.mask = take(nch * E * 4);
  L.base = take(nch * E * 4);
  L.total = off;
  return L;
}

// Device address of g_route_scratch on the current device (looked up once per
// device, with that device current).  nullptr if the lookup failed.
uint8_t *static_scratch(int dev) {
  static std::mutex mu;
  static uint8_t *addr[kMaxDevices] = {nullptr};
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    addr[dev] = static_cast<uint8_t *>(p);
  }
  return addr[dev];
}

// ------------------------------------------------ expert parallelism
// The region after the single-GPU workspace that the expert-parallel phases
// add: fixed-size tables first (so the combine finds them whatever the owner
// received), then the received rows, expert-major, and their h.
struct EpLayout {
  size_t ep_off, ep_cnt, ep_u1, ep_u2, src, dst, zero, c_off, c_cnt, c_u1, c_u2, fixed_end, out_row, rows, h, total;
};

bool ep_supported(const mrlmoe_config &c, int n) {
  return c.dtype == MRLMOE_BF16 && n >= 1 && n <= kEpMaxRanks && c.n_experts % n == 0;
}

// Rows one owner can receive when every rank routes at most cfg.T tokens:
// a token sends a rank at most min(k, E/n) rows.
size_t ep_rows_max(const mrlmoe_config &c, int n) {
  return static_cast<size_t>(n) * c.T * std::min(c.top_k, c.n_experts / n);
}

EpLayout ep_layout_of(const mrlmoe_config &c, int n, size_t rows) {
  EpLayout L{};
  size_t off = layout_of(c).total;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += (bytes + 255) & ~size_t(255);
    return o;
  };
  const size_t E = c.n_experts, El = c.n_experts / std::max(n, 1);
  L.ep_off = take((El + 2) * 4);
  L.ep_cnt = take((El + 2) * 4);
  L.ep_u1 = take((El + 2) * 4);
  L.ep_u2 = take((El + 2) * 4);
  L.src = take(E * 4);
  L.dst = take(E * 4);
  L.zero = take((E + 2) * 4);
  L.c_off = take((E + 2) * 4);
  L.c_cnt = take((E + 2) * 4);
  L.c_u1 = take((E + 2) * 4);
  L.c_u2 = take((E + 2) * 4);
  L.fixed_end = off;
  L.out_row = take(rows * 4);
  L.rows = take(rows * c.d_lat * 2);
  L.h = take(rows * c.d_ff * 2);
  L.total = off;
  return L;
}

}  // namespace

extern "C" {

size_t mrlmoe_workspace_size(const mrlmoe_config *cfg) {
  if (check_config(cfg) != MRLMOE_OK) return 0;
  return layout_of(*cfg).total;
}

const char *mrlmoe_status_string(mrlmoe_status s) {
  switch (s) {
    case MRLMOE_OK: return "ok";
    case MRLMOE_ERR_INVALID_ARG: return "invalid argument";
    case MRLMOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case MRLMOE_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case MRLMOE_ERR_CUDA: return "CUDA runtime error";
    case MRLMOE_ERR_TIMEOUT: return "device wait timed out";
    case MRLMOE_ERR_CHECK: return "device consistency check failed";
    case MRLMOE_ERR_SCRATCH_LIMIT: return "problem exceeds the static scratch of mrlmoe_route_scores_static";
  }
  return "unknown status";
}

mrlmoe_status mrlmoe_route(const mrlmoe_config *cfg, const mrlmoe_weights *w, const float *bias, const void *x,
                           int scores_in, mrlmoe_routing *out, void *workspace, size_t ws_bytes, void *stream) {
  mrlmoe_status s = check_config(cfg);
  if (s != MRLMOE_OK) return s;
  if (!out || !bias || !w || !w->expert_scale) return MRLMOE_ERR_INVALID_ARG;
  if (scores_in) {
    if (!out->scores) return MRLMOE_ERR_INVALID_ARG;
  } else {
    if (!x || !aligned16(x)) return MRLMOE_ERR_INVALID_ARG;
    if ((s = check_weights_bf16(w, false)) != MRLMOE_OK) return s;
    if (!w->w_down || !aligned16(w->w_down)) return MRLMOE_ERR_INVALID_ARG;
    if (cfg->dtype != MRLMOE_BF16 && !w->s_down) return MRLMOE_ERR_INVALID_ARG;
  }
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return MRLMOE_ERR_WORKSPACE;
  if (ws_bytes < layout_of(*cfg).total) return MRLMOE_ERR_WORKSPACE;
  int sms = 0;
  DeviceRestore restore;
  if ((s = bind_device(workspace, &sms, &restore)) != MRLMOE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Ptrs P = carve(*cfg, workspace, out);
  if ((s = init_header(P.status, cfg->hold, st)) != MRLMOE_OK) return s;
  NvtxCall nvtx_call("mrlmoe_route");
  if (scores_in) {
    MRL_TRY(launch_topk_from_scores(out->scores, bias, w->expert_scale, cfg->T, cfg->n_experts, cfg->top_k,
                                    P.topk_idx, P.topk_w, P.wscaled, P.status, st));
  } else {
    if ((s = launch_project_and_route(*cfg, w, bias, x, P, sms, st)) != MRLMOE_OK) return s;
  }
  return launch_dispatch(*cfg, P, st);
}

mrlmoe_status mrlmoe_forward(const mrlmoe_config *cfg, const mrlmoe_weights *w, const float *bias, const void *x,
                             void *y, mrlmoe_routing *route_out, void *workspace, size_t ws_bytes, void *stream) {
  return forward_impl(cfg, w, bias, x, y, route_out, workspace, ws_bytes, stream, nullptr);
}

mrlmoe_status mrlmoe_forward_timed(const mrlmoe_config *cfg, const mrlmoe_weights *w, const float *bias,
                                   const void *x, void *y, mrlmoe_routing *route_out, void *workspace,
                                   size_t ws_bytes, void *stream, void *const *events, int n_events) {
  if (!events || n_events != MRLMOE_NUM_STAGE_EVENTS) return MRLMOE_ERR_INVALID_ARG;
  for (int i = 0; i < n_events; ++i)
    if (!events[i]) return MRLMOE_ERR_INVALID_ARG;
  return forward_impl(cfg, w, bias, x, y, route_out, workspace, ws_bytes, stream, events);
}

size_t mrlmoe_train_workspace_size(const mrlmoe_config *cfg) {
  if (check_config(cfg) != MRLMOE_OK || !train_supported(*cfg)) return 0;
  return layout_of(*cfg, true).total;
}

mrlmoe_status mrlmoe_forward_train(const mrlmoe_config *cfg, const mrlmoe_weights *w, const float *bias,
                                   const void *x, void *y, mrlmoe_routing *route_out, void *workspace,
                                   size_t ws_bytes, void *stream) {
  return forward_impl(cfg, w, bias, x, y, route_out, workspace, ws_bytes, stream, nullptr, true);
}

mrlmoe_status mrlmoe_backward(const mrlmoe_config *cfg, const mrlmoe_weights *w, const void *x, const void *dy,
                              const mrlmoe_grads *grads, void *workspace, size_t ws_bytes, void *stream) {
  return backward_impl(cfg, w, x, dy, grads, workspace, ws_bytes, stream);
}

mrlmoe_status mrlmoe_backward_timed(const mrlmoe_config *cfg, const mrlmoe_weights *w, const void *x,
                                    const void *dy, const mrlmoe_grads *grads, void *workspace, size_t ws_bytes,
                                    void *stream, void *const *events, int n_events) {
  if (!events || n_events != MRLMOE_NUM_BACKWARD_EVENTS) return MRLMOE_ERR_INVALID_ARG;
  for (int i = 0; i < n_events; ++i)
    if (!events[i]) return MRLMOE_ERR_INVALID_ARG;
  return backward_impl(cfg, w, x, dy, grads, workspace, ws_bytes, stream, events);
}

mrlmoe_status mrlmoe_bias_update(const mrlmoe_config *cfg, const int32_t *counts, float *bias, float gamma,
                                 void *stream) {
  mrlmoe_status s = check_config(cfg);
  if (s != MRLMOE_OK) return s;
  if (!counts || !bias) return MRLMOE_ERR_INVALID_ARG;
  int sms = 0;
  DeviceRestore restore;
  if ((s = bind_device(bias, &sms, &restore)) != MRLMOE_OK) return s;
  const int E = cfg->n_experts;
  bias_update_kernel<<<(E + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      counts, bias, E, static_cast<long long>(cfg->T) * cfg->top_k, gamma);
  MRL_TRY(cudaGetLastError());
  return MRLMOE_OK;
}

mrlmoe_status mrlmoe_linear(const void *a, const void *w, void *out, int M, int N, int K, void *stream) {
  if (!a || !w || !out || M < 1 || N < 128 || K < 128 || N % 128 || K % 128) return MRLMOE_ERR_INVALID_ARG;
  if (!aligned16(a) || !aligned16(w) || !aligned16(out)) return MRLMOE_ERR_INVALID_ARG;
  int sms = 0;
  DeviceRestore restore;
  mrlmoe_status s = bind_device(w, &sms, &restore);
  if (s != MRLMOE_OK) return s;
  return launch_dense_bf16(a, w, static_cast<__nv_bfloat16 *>(out), nullptr, M, N, K, nullptr, sms,
                           static_cast<cudaStream_t>(stream));
}

mrlmoe_status mrlmoe_route_scores_static(const mrlmoe_config *cfg, const float *bias, const float *expert_scale,
                                         mrlmoe_routing *out, void *stream) {
  mrlmoe_status s = check_config(cfg);
  if (s != MRLMOE_OK) return s;
  if (!bias || !expert_scale || !out || !out->scores || !out->topk_idx || !out->topk_w || !out->counts ||
      !out->offsets || !out->perm || !out->inv_perm)
    return MRLMOE_ERR_INVALID_ARG;
  const StaticRouteLayout SL = static_route_layout(*cfg);
  if (SL.total > MRLMOE_STATIC_SCRATCH_BYTES) return MRLMOE_ERR_SCRATCH_LIMIT;
  int sms = 0;
  DeviceRestore restore;
  if ((s = bind_device(out->scores, &sms, &restore)) != MRLMOE_OK) return s;
  int dev = 0;
  MRL_TRY(cudaGetDevice(&dev));
  uint8_t *b = static_scratch(dev);
  if (!b) return MRLMOE_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Ptrs P{};
  P.status = reinterpret_cast<uint32_t *>(b + SL.status);
  P.topk_idx = out->topk_idx;
  P.topk_w = out->topk_w;
  P.wscaled = reinterpret_cast<float *>(b + SL.wscaled);
  P.counts_e = reinterpret_cast<int32_t *>(b + SL.counts);
  P.grp_off = reinterpret_cast<int32_t *>(b + SL.grp_off);
  P.grp_cnt = reinterpret_cast<int32_t *>(b + SL.grp_cnt);
  P.unit1 = reinterpret_cast<int32_t *>(b + SL.unit1);
  P.unit2 = reinterpret_cast<int32_t *>(b + SL.unit2);
  P.perm = out->perm;
  P.inv = out->inv_perm;
  P.mask = reinterpret_cast<uint32_t *>(b + SL.mask);
  P.base = reinterpret_cast<int32_t *>(b + SL.base);
  P.out_counts = out->counts;
  P.out_offsets = out->offsets;
  // the array keeps the previous call's contents: the header must start at
  // zero; every other region is fully rewritten below before it is read
  if ((s = init_header(P.status, 0, st)) != MRLMOE_OK) return s;
  MRL_TRY(launch_topk_from_scores(out->scores, bias, expert_scale, cfg->T, cfg->n_experts, cfg->top_k, P.topk_idx,
                                  P.topk_w, P.wscaled, P.status, st));
  return launch_dispatch(*cfg, P, st);
}

mrlmoe_status mrlmoe_quantize_e4m3(const void *in, int rows, int K, void *q, float *scale, void *stream) {
  if (!in || !q || !scale || rows < 1 || K < 128 || K % 128) return MRLMOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(in) & 15u) || (reinterpret_cast<uintptr_t>(q) & 7u) ||
      (reinterpret_cast<uintptr_t>(scale) & 3u))
    return MRLMOE_ERR_INVALID_ARG;
  int sms = 0;
  DeviceRestore restore;
  mrlmoe_status s = bind_device(in, &sms, &restore);
  if (s != MRLMOE_OK) return s;
  MRL_TRY(launch_quant(static_cast<const __nv_bfloat16 *>(in), K, rows, K, static_cast<uint8_t *>(q), scale, false,
                       nullptr, static_cast<cudaStream_t>(stream)));
  return MRLMOE_OK;
}

mrlmoe_status mrlmoe_get_device_status(const void *workspace, void *stream) {
  uint32_t bits = 0;
  return mrlmoe_get_device_detail(workspace, &bits, stream);
}

mrlmoe_status mrlmoe_get_device_detail(const void *workspace, uint32_t *check_bits, void *stream) {
  if (!workspace) return MRLMOE_ERR_WORKSPACE;
  if (!check_bits) return MRLMOE_ERR_INVALID_ARG;
  uint32_t h[3] = {0, 0, 0};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  MRL_TRY(cudaStreamSynchronize(st));
  MRL_TRY(cudaMemcpy(h, workspace, sizeof(h), cudaMemcpyDeviceToHost));
  *check_bits = h[2];
  if (h[0] == DEV_TIMEOUT) return MRLMOE_ERR_TIMEOUT;
  if (h[0] == DEV_CHECK) return MRLMOE_ERR_CHECK;
  return h[0] == 0 ? MRLMOE_OK : MRLMOE_ERR_CHECK;
}

mrlmoe_status mrlmoe_check_routing(const mrlmoe_config *cfg, const mrlmoe_routing *r, void *workspace,
                                   size_t ws_bytes, int clear, void *stream) {
  mrlmoe_status s = check_config(cfg);
  if (s != MRLMOE_OK) return s;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return MRLMOE_ERR_WORKSPACE;
  const bool whole = r && r->topk_idx && r->counts && r->offsets && r->perm && r->inv_perm;
  const bool full = ws_bytes >= layout_of(*cfg).total;
  if (ws_bytes < 256 || (!whole && !full)) return MRLMOE_ERR_WORKSPACE;
  int sms = 0;
  DeviceRestore restore;
  if ((s = bind_device(workspace, &sms, &restore)) != MRLMOE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t *hdr = static_cast<uint32_t *>(workspace);
  // r's arrays where given, else the workspace copies that route/forward keep
  // (counts and offsets from the group table, whose entry E is T*k)
  Ptrs P{};
  if (full) P = carve(*cfg, workspace, r);
  const int32_t *idx = (r && r->topk_idx) ? r->topk_idx : P.topk_idx;
  const int32_t *perm = (r && r->perm) ? r->perm : P.perm;
  const int32_t *inv = (r && r->inv_perm) ? r->inv_perm : P.inv;
  const int32_t *counts = (r && r->counts) ? r->counts : P.grp_cnt;
  const int32_t *offsets = (r && r->offsets) ? r->offsets : P.grp_off;
  const float *w = (r && r->topk_w) ? r->topk_w : P.topk_w;  // NULL: weights unchecked
  if (clear) MRL_TRY(cudaMemsetAsync(hdr, 0, 16, st));
  const long long Tk = static_cast<long long>(cfg->T) * cfg->top_k;
  const long long n = std::max<long long>(Tk, cfg->n_experts + 1);
  const long long blocks = std::min<long long>((n + kCheckThreads - 1) / kCheckThreads, 8ll * sms);
  check_routing_kernel<<<static_cast<int>(blocks), kCheckThreads, 0, st>>>(idx, w, counts, offsets, perm, inv,
                                                                          cfg->T, cfg->n_experts, cfg->top_k, hdr);
  MRL_TRY(cudaGetLastError());
  return MRLMOE_OK;
}

size_t mrlmoe_ep_workspace_size(const mrlmoe_config *cfg, int n_ranks) {
  if (check_config(cfg) != MRLMOE_OK || !ep_supported(*cfg, n_ranks)) return 0;
  return ep_layout_of(*cfg, n_ranks, ep_rows_max(*cfg, n_ranks)).total;
}

mrlmoe_status mrlmoe_ep_dispatch(const mrlmoe_config *cfg, const mrlmoe_weights *w, const float *bias, const void *x,
                                 int n_ranks, mrlmoe_routing *out, void *send_rows, void *workspace, size_t ws_bytes,
                                 void *stream) {
  mrlmoe_status s = check_config(cfg);
  if (s != MRLMOE_OK) return s;
  if (!ep_supported(*cfg, n_ranks)) return cfg->dtype != MRLMOE_BF16 ? MRLMOE_ERR_UNSUPPORTED : MRLMOE_ERR_INVALID_ARG;
  if (!bias || !x || !aligned16(x) || !send_rows || !aligned16(send_rows)) return MRLMOE_ERR_INVALID_ARG;
  if (!out || !out->counts || !out->offsets) return MRLMOE_ERR_INVALID_ARG;
  if ((s = check_weights_bf16(w, false)) != MRLMOE_OK) return s;
  if (!w->w_down || !aligned16(w->w_down)) return MRLMOE_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return MRLMOE_ERR_WORKSPACE;
  if (ws_bytes < layout_of(*cfg).total) return MRLMOE_ERR_WORKSPACE;
  int sms = 0;
  DeviceRestore restore;
  if ((s = bind_device(workspace, &sms, &restore)) != MRLMOE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the record stays in the workspace (the combine reads it there) and is copied out
  Ptrs P = carve(*cfg, workspace, nullptr);
  P.scores = out->scores;
  P.out_counts = out->counts;
  P.out_offsets = out->offsets;
  const int T = cfg->T, Ld = cfg->d_lat, k = cfg->top_k, Tk = T * k;
  if ((s = init_header(P.status, cfg->hold, st)) != MRLMOE_OK) return s;
  NvtxCall nvtx_call("mrlmoe_ep_dispatch");
  nvtx_stage(kForwardStages[0]);
  if ((s = launch_project_and_route(*cfg, w, bias, x, P, sms, st)) != MRLMOE_OK) return s;
  nvtx_stage(kForwardStages[2]);
  if ((s = launch_dispatch(*cfg, P, st)) != MRLMOE_OK) return s;
  nvtx_stage(kForwardStages[3]);
  MRL_TRY(launch_copy_dispatch_rows(P, T, Ld, k, send_rows, sms, st));
  const size_t n = static_cast<size_t>(Tk) * 4;
  if (out->topk_idx) MRL_TRY(cudaMemcpyAsync(out->topk_idx, P.topk_idx, n, cudaMemcpyDeviceToDevice, st));
  if (out->topk_w) MRL_TRY(cudaMemcpyAsync(out->topk_w, P.topk_w, n, cudaMemcpyDeviceToDevice, st));
  if (out->perm) MRL_TRY(cudaMemcpyAsync(out->perm, P.perm, n, cudaMemcpyDeviceToDevice, st));
  if (out->inv_perm) MRL_TRY(cudaMemcpyAsync(out->inv_perm, P.inv, n, cudaMemcpyDeviceToDevice, st));
  return MRLMOE_OK;
}

mrlmoe_status mrlmoe_ep_experts(const mrlmoe_config *cfg, const mrlmoe_weights *w_local, int n_ranks,
                                const void *recv_rows, const int32_t *recv_counts, int n_recv, float *out_rows,
                                void *workspace, size_t ws_bytes, void *stream) {
  mrlmoe_status s = check_config(cfg);
  if (s != MRLMOE_OK) return s;
  if (!ep_supported(*cfg, n_ranks)) return cfg->dtype != MRLMOE_BF16 ? MRLMOE_ERR_UNSUPPORTED : MRLMOE_ERR_INVALID_ARG;
  if (n_recv < 0 || !recv_counts || !w_local) return MRLMOE_ERR_INVALID_ARG;
  if (n_recv > 0 && (!recv_rows || !aligned16(recv_rows) || !out_rows || !aligned16(out_rows)))
    return MRLMOE_ERR_INVALID_ARG;
  {
    const void *ps[] = {w_local->w_gate, w_local->w_up_e, w_local->w_down_e};
    for (const void *p : ps)
      if (!p || !aligned16(p)) return MRLMOE_ERR_INVALID_ARG;
  }
  if (static_cast<long long>(n_recv) * 256 >= (1ll << 31)) return MRLMOE_ERR_UNSUPPORTED;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return MRLMOE_ERR_WORKSPACE;
  const EpLayout EL = ep_layout_of(*cfg, n_ranks, static_cast<size_t>(n_recv));
  if (ws_bytes < EL.total) return MRLMOE_ERR_WORKSPACE;
  if (n_recv == 0) return MRLMOE_OK;  // nothing arrived: no work
  int sms = 0;
  DeviceRestore restore;
  if ((s = bind_device(workspace, &sms, &restore)) != MRLMOE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t *b = static_cast<uint8_t *>(workspace);
  uint32_t *status = reinterpret_cast<uint32_t *>(b + layout_of(*cfg).status);  // continues the rank's status word
  auto i32 = [&](size_t off) { return reinterpret_cast<int32_t *>(b + off); };
  const int El = cfg->n_experts / n_ranks, Ld = cfg->d_lat, F = cfg->d_ff;
  __nv_bfloat16 *rows = reinterpret_cast<__nv_bfloat16 *>(b + EL.rows);
  __nv_bfloat16 *h = reinterpret_cast<__nv_bfloat16 *>(b + EL.h);
  NvtxCall nvtx_call("mrlmoe_ep_experts");
  nvtx_stage(kForwardStages[3]);
  ep_layout_kernel<<<1, 1024, 0, st>>>(recv_counts, n_ranks, El, n_recv, kExpertBN, glu_m_tiles(*cfg),
                                       down_m_tiles(*cfg), i32(EL.ep_off), i32(EL.ep_cnt), i32(EL.ep_u1),
                                       i32(EL.ep_u2), i32(EL.src), i32(EL.dst), status);
  MRL_TRY(cudaGetLastError());
  ep_gather_kernel<<<n_ranks * El, 256, 0, st>>>(static_cast<const uint4 *>(recv_rows), Ld * 2 / 16, recv_counts,
                                                 i32(EL.src), i32(EL.dst), reinterpret_cast<uint4 *>(rows),
                                                 i32(EL.out_row), status);
  MRL_TRY(cudaGetLastError());
  nvtx_stage(kForwardStages[4]);
  {
    GluParams p{};
    const uint64_t EF = static_cast<uint64_t>(El) * F;
    // no shared-expert rows here: its maps are never used and stand in as the routed ones
    if (!make_map(&p.wg, w_local->w_gate, 2, Ld, EF, 64) || !make_map(&p.wu, w_local->w_up_e, 2, Ld, EF, 64) ||
        !make_map(&p.sg, w_local->w_gate, 2, Ld, EF, 64) || !make_map(&p.su, w_local->w_up_e, 2, Ld, EF, 64) ||
        !make_token_maps(&p.tz, rows, Ld, static_cast<uint64_t>(n_recv)))
      return MRLMOE_ERR_CUDA;
    p.gt = GroupTable{i32(EL.ep_off), i32(EL.ep_cnt), i32(EL.ep_u1), El, glu_m_tiles(*cfg)};
    p.h = h;
    p.F = F; p.L = Ld; p.rows = n_recv;
    p.status = status;
    MRL_TRY(launch_gemm_pair<Glu2Policy>(p, sms, st));
  }
  nvtx_stage(kForwardStages[5]);
  {
    DownPolicy::Params p{};
    const uint64_t EL_rows = static_cast<uint64_t>(El) * Ld;
    if (!make_map(&p.wd, w_local->w_down_e, 2, F, EL_rows, 128) ||
        !make_map(&p.sd, w_local->w_down_e, 2, F, EL_rows, 128) ||
        !make_token_maps_blocked(&p.th, h, F, static_cast<uint64_t>(n_recv)))
      return MRLMOE_ERR_CUDA;
    p.gt = GroupTable{i32(EL.ep_off), i32(EL.ep_cnt), i32(EL.ep_u2), El, down_m_tiles(*cfg)};
    p.out_row = i32(EL.out_row);
    p.slots = out_rows;
    p.L = Ld; p.F = F; p.k = cfg->top_k; p.Tk = 0;
    p.status = status;
    if (down_uses_pairs(*cfg))
      MRL_TRY(launch_gemm_pair<Down2Policy>(p, sms, st));
    else
      MRL_TRY(launch_gemm<DownPolicy>(p, sms, st));
  }
  return MRLMOE_OK;
}

mrlmoe_status mrlmoe_ep_combine(const mrlmoe_config *cfg, const mrlmoe_weights *w, const float *ret_rows, void *y,
                                void *workspace, size_t ws_bytes, void *stream) {
  mrlmoe_status s = check_config(cfg);
  if (s != MRLMOE_OK) return s;
  if (cfg->dtype != MRLMOE_BF16) return MRLMOE_ERR_UNSUPPORTED;
  if (!w || !w->expert_scale || !ret_rows || !aligned16(ret_rows) || !y || !aligned16(y)) return MRLMOE_ERR_INVALID_ARG;
  {
    const void *ps[] = {w->w_sh_gate, w->w_sh_up, w->w_sh_down, w->rms_gain, w->w_up};
    for (const void *p : ps)
      if (!p || !aligned16(p)) return MRLMOE_ERR_INVALID_ARG;
  }
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return MRLMOE_ERR_WORKSPACE;
  const EpLayout EL = ep_layout_of(*cfg, 1, 0);
  if (ws_bytes < EL.fixed_end) return MRLMOE_ERR_WORKSPACE;
  int sms = 0;
  DeviceRestore restore;
  if ((s = bind_device(workspace, &sms, &restore)) != MRLMOE_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Ptrs P = carve(*cfg, workspace, nullptr);  // the dispatch's record; its status word continues
  uint8_t *b = static_cast<uint8_t *>(workspace);
  auto i32 = [&](size_t off) { return reinterpret_cast<int32_t *>(b + off); };
  const int T = cfg->T, D = cfg->d_model, Ld = cfg->d_lat, F = cfg->d_ff, E = cfg->n_experts, k = cfg->top_k;
  const int Tk = T * k;
  NvtxCall nvtx_call("mrlmoe_ep_combine");
  nvtx_stage(kForwardStages[4]);
  // group tables with the shared expert alone (every routed count 0)
  MRL_TRY(cudaMemsetAsync(b + EL.zero, 0, (E + 2) * 4, st));
  expert_offsets_kernel<<<1, 1024, 0, st>>>(i32(EL.zero), T, E, k, kExpertBN, glu_m_tiles(*cfg), down_m_tiles(*cfg),
                                            i32(EL.c_off), i32(EL.c_cnt), i32(EL.c_u1), i32(EL.c_u2), nullptr,
                                            nullptr, P.status);
  MRL_TRY(cudaGetLastError());
  {
    GluParams p{};
    if (!make_map(&p.wg, w->w_sh_gate, 2, Ld, F, 64) || !make_map(&p.wu, w->w_sh_up, 2, Ld, F, 64) ||
        !make_map(&p.sg, w->w_sh_gate, 2, Ld, F, 64) || !make_map(&p.su, w->w_sh_up, 2, Ld, F, 64) ||
        !make_token_maps(&p.tz, P.zbuf, Ld, static_cast<uint64_t>(Tk) + T))
      return MRLMOE_ERR_CUDA;
    p.gt = GroupTable{i32(EL.c_off), i32(EL.c_cnt), i32(EL.c_u1), E, glu_m_tiles(*cfg)};
    p.h = P.hbuf;
    p.F = F; p.L = Ld; p.rows = Tk + T;
    p.status = P.status;
    MRL_TRY(launch_gemm_pair<Glu2Policy>(p, sms, st));
  }
  nvtx_stage(kForwardStages[5]);
  {
    DownPolicy::Params p{};
    if (!make_map(&p.wd, w->w_sh_down, 2, F, Ld, 128) || !make_map(&p.sd, w->w_sh_down, 2, F, Ld, 128) ||
        !make_token_maps_blocked(&p.th, P.hbuf, F, static_cast<uint64_t>(Tk) + T))
      return MRLMOE_ERR_CUDA;
    p.gt = GroupTable{i32(EL.c_off), i32(EL.c_cnt), i32(EL.c_u2), E, down_m_tiles(*cfg)};
    p.perm = P.perm;
    p.wscaled = P.wscaled;
    p.slots = P.slots;
    p.L = Ld; p.F = F; p.k = k; p.Tk = Tk;
    p.status = P.status;
    if (down_uses_pairs(*cfg))
      MRL_TRY(launch_gemm_pair<Down2Policy>(p, sms, st));
    else
      MRL_TRY(launch_gemm<DownPolicy>(p, sms, st));
  }
  nvtx_stage(kForwardStages[6]);
  {
    const float4 *ret = reinterpret_cast<const float4 *>(ret_rows);
    const float4 *slots = reinterpret_cast<const float4 *>(P.slots);
    const float4 *g = reinterpret_cast<const float4 *>(w->rms_gain);
    const float eps = cfg->rms_eps;
    const int L4 = Ld / 4;
    if (L4 <= kCombineThreads)
      ep_combine_rmsnorm_kernel<1><<<T, kCombineThreads, 0, st>>>(ret, P.inv, P.wscaled, slots, Ld, k, eps, g,
                                                                  P.nbuf, P.status);
    else if (L4 <= 2 * kCombineThreads)
      ep_combine_rmsnorm_kernel<2><<<T, kCombineThreads, 0, st>>>(ret, P.inv, P.wscaled, slots, Ld, k, eps, g,
                                                                  P.nbuf, P.status);
    else if (L4 <= 4 * kCombineThreads)
      ep_combine_rmsnorm_kernel<4><<<T, kCombineThreads, 0, st>>>(ret, P.inv, P.wscaled, slots, Ld, k, eps, g,
                                                                  P.nbuf, P.status);
    else
      ep_combine_rmsnorm_kernel<kCombineMaxV4><<<T, kCombineThreads, 0, st>>>(ret, P.inv, P.wscaled, slots, Ld, k,
                                                                              eps, g, P.nbuf, P.status);
    MRL_TRY(cudaGetLastError());
  }
  nvtx_stage(kForwardStages[7]);
  return launch_dense_bf16(P.nbuf, w->w_up, static_cast<__nv_bfloat16 *>(y), nullptr, T, D, Ld, P.status, sms, st);
}

}  // extern "C"
