/*
 * mrlmoe.h — C ABI of the Multi-Router Latent MoE layer (sm_100a): the forward
 * pass, its balancing-bias update, and the backward pass for training.
 *
 * The layer (ERNIE 5.5 Flash release pages: blog.derekhsu.net "ERNIE-5.5-Flash-Base"
 * translation, section "多路由潛在 MoE (Multi-Router Latent MoE)"; aitest123.com
 * "ERNIE-5.5-Flash-Base开源", section "模型结构"; lininn.cn "2800 亿参数的模型，每次只叫醒
 * 140 亿", section "路由器，不止一个"):
 *
 *   z   = x W_down^T                        tokens projected d_model -> d_lat (4096 -> 2048)
 *   s   = mean_r sigmoid(z W_router[r]^T)   R sigmoid routers on the latent, aggregated
 *   sel = top-k of (s + bias)               aux-loss-free balancing bias: selection only
 *   w   = s_sel / sum(s_sel);  w' = w * alpha[e]   renormalised, per-expert learnable scalar
 *   o_e = (SiLU(z W_gate,e^T) * (z W_up,e^T)) W_down,e^T     latent experts, d_ff = 2048
 *   c   = sum_j w'_j o_{e_j} + o_shared     one always-on shared expert (weight 1)
 *   y   = RMSNorm(c; gain, eps) W_up^T      shared up-projection d_lat -> d_model
 *   bias[e] += gamma * sign(T*k/E - count[e])          balancing-bias update
 *
 * The mean aggregation, R, the renormalisation, the lower-index tie rule and
 * the bias-update rule are this library's readings of pages that fix none of
 * them.  The printed activation name "SiTU-GLU" is read as SiLU-GLU.
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller; matrices are
 *    row-major and weights are stored [out, in] (the reduction dim contiguous).
 *  - bf16 = IEEE bfloat16 (2 bytes); e4m3 = OCP FP8 E4M3 (1 byte).
 *  - `stream` is a cudaStream_t (0 = legacy default stream).  Calls only
 *    enqueue work on it; none synchronises except mrlmoe_get_device_status.
 *  - Argument problems found on the host return a non-zero status before
 *    anything is enqueued.  Faults found on the device (a bounded wait that
 *    gave up, a failed check) are written to a status word inside the
 *    workspace; read it with mrlmoe_get_device_status.  No kernel traps.
 *    Once a kernel of a call has failed, the call's later kernels do nothing,
 *    so no kernel reads a record that a failed kernel left unwritten.
 *  - The library allocates no device memory: all scratch lives in the
 *    caller's workspace of mrlmoe_workspace_size() bytes (256-byte aligned).
 *  - The library keeps no state between calls; two calls that share a
 *    workspace must be ordered on one stream.
 */
#ifndef MRLMOE_H_
#define MRLMOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MRLMOE_OK = 0,
  MRLMOE_ERR_INVALID_ARG = 1,   /* null pointer, bad size, bad dims            */
  MRLMOE_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. dtype)      */
  MRLMOE_ERR_WORKSPACE = 3,     /* workspace missing, too small or misaligned  */
  MRLMOE_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed         */
  MRLMOE_ERR_TIMEOUT = 5,       /* device: a bounded wait gave up              */
  MRLMOE_ERR_CHECK = 6,         /* device: a consistency check failed          */
  MRLMOE_ERR_SCRATCH_LIMIT = 7  /* problem larger than the built-in scratch of
                                   mrlmoe_route_scores_static                    */
} mrlmoe_status;

typedef enum {
  MRLMOE_BF16 = 0,              /* bf16 weights and activations, fp32 accumulate */
  MRLMOE_FP8_E4M3_BLOCK128 = 1, /* e4m3 weights with fp32 scales per 128x128 block,
                                   activations quantised e4m3 per 1x128 block;
                                   the routers stay bf16, y is bf16               */
  MRLMOE_FP4_E2M1_BLOCK128 = 2  /* as MRLMOE_FP8_E4M3_BLOCK128, but the six expert
                                   matrices (routed gate/up/down, shared gate/up/
                                   down) hold e2m1 codes (OCP MX FP4), two per
                                   byte along K (lower index in the low nibble):
                                   [.., out, in/2] bytes, 32-byte aligned (the
                                   tensor core reads the codes through the 4-bit
                                   unpacking TMA type, which needs it), with the
                                   same fp32 128x128 block scales s_*; the
                                   projections stay e4m3.  Reading of "the
                                   release ships FP4 weights"                 */
} mrlmoe_dtype;

/* How the R sigmoid router scores of a (token, expert) are aggregated into
 * the score s used for selection and weights.  The pages say the routers'
 * scores are aggregated without fixing the rule (aitest123, "模型结构";
 * derekhsu, "多路由潛在 MoE"); MEAN is the layer's reading, SUM and MAX are
 * the alternatives for sensitivity studies.                                   */
typedef enum {
  MRLMOE_AGG_MEAN = 0,          /* s = (sum_r sigmoid(l_r)) / R  (default)       */
  MRLMOE_AGG_SUM = 1,           /* s = sum_r sigmoid(l_r)                        */
  MRLMOE_AGG_MAX = 2            /* s = max_r sigmoid(l_r)                        */
} mrlmoe_aggregation;

/* Layer shape.  Limits checked on the host:
 *   T >= 1; d_model, d_lat, d_ff multiples of 128; 1 <= n_routers <= 8;
 *   16 <= n_experts <= 1024 with n_experts a multiple of 16;
 *   1 <= top_k <= min(n_experts, 32); rms_eps >= 0; aggregation one of
 *   mrlmoe_aggregation.  d_lat <= 8192, and in
 *   FP8 mode d_model, d_lat, d_ff <= 4096; beyond those the status is
 *   MRLMOE_ERR_UNSUPPORTED, otherwise MRLMOE_ERR_INVALID_ARG.                 */
typedef struct {
  int T;            /* tokens in this call                                       */
  int d_model;      /* hidden size (4096 at full width)                          */
  int d_lat;        /* latent size (2048)                                        */
  int n_experts;    /* routed experts E (512)                                    */
  int top_k;        /* experts selected per token k (10)                         */
  int d_ff;         /* expert intermediate size F (2048)                         */
  int n_routers;    /* sigmoid routers R (4)                                     */
  float rms_eps;    /* RMSNorm epsilon (1e-6)                                    */
  mrlmoe_dtype dtype;
  mrlmoe_aggregation aggregation;  /* router score aggregation (0 = mean)      */
  uint32_t hold;    /* 0 in normal use.  Test hook for the bounded waits: an OR
                       of mrlmoe_hold bits; the GEMM kernels of those families
                       issue no tile loads in this call, so their waits run out
                       (after about 2 s) and the call ends with
                       MRLMOE_ERR_TIMEOUT in the status word.  Other bits:
                       MRLMOE_ERR_INVALID_ARG.                                 */
} mrlmoe_config;

/* GEMM families for mrlmoe_config.hold.                                       */
typedef enum {
  MRLMOE_HOLD_GEMM = 1,         /* one-CTA bf16 GEMMs: projections, routers, expert down */
  MRLMOE_HOLD_GEMM_PAIR = 2,    /* CTA-pair bf16 grouped GEMMs: gate/up (and wide down)  */
  MRLMOE_HOLD_GEMM_FP8 = 4      /* the FP8 variant's GEMMs                               */
} mrlmoe_hold;

/* Weights: device pointers, caller-owned.  Element type is bf16 in BF16 mode;
 * in FP8 mode every matrix except w_router is e4m3 and carries a scale array
 * s_* of fp32 [ceil(out/128), ceil(in/128)] per matrix (per expert for the
 * routed experts: [E, ...]).                                                   */
typedef struct {
  const void *w_down;      /* [d_lat, d_model]                                    */
  const void *w_router;    /* [R, E, d_lat]   always bf16                         */
  const void *w_gate;      /* [E, d_ff, d_lat]  routed experts, gate projection    */
  const void *w_up_e;      /* [E, d_ff, d_lat]  routed experts, up projection      */
  const void *w_down_e;    /* [E, d_lat, d_ff]  routed experts, down projection    */
  const void *w_sh_gate;   /* [d_ff, d_lat]     shared expert                      */
  const void *w_sh_up;     /* [d_ff, d_lat]                                        */
  const void *w_sh_down;   /* [d_lat, d_ff]                                        */
  const float *rms_gain;   /* [d_lat] fp32                                         */
  const void *w_up;        /* [d_model, d_lat]  shared up-projection               */
  const float *expert_scale; /* alpha [E] fp32                                     */
  const float *s_down, *s_gate, *s_up_e, *s_down_e,
              *s_sh_gate, *s_sh_up, *s_sh_down, *s_up;   /* FP8 only, else NULL   */
} mrlmoe_weights;

/* Routing record.  Every pointer is optional (NULL = keep it in the workspace
 * only).  Sizes: topk_idx, topk_w, perm, inv_perm: T*k; counts: E;
 * offsets: E+1; scores: T*E.
 *   topk_idx[t*k+j] expert of rank j for token t (descending biased score,
 *                   ties to the lower index);
 *   topk_w[t*k+j]   normalised weight BEFORE alpha (sums to 1 per token; if
 *                   the k selected scores sum to exactly 0, every weight is
 *                   the uniform fp32(1/k));
 *   counts[e]       (token, slot) pairs routed to e; offsets = exclusive scan;
 *   perm[row]       t*k+j of dispatch row `row` (expert-major, tokens ascending);
 *   inv_perm[t*k+j] its dispatch row;
 *   scores[t*E+e]   fp32 aggregated router score s (output of mrlmoe_route /
 *                   mrlmoe_forward when non-NULL; INPUT when scores_in = 1).  */
typedef struct {
  int32_t *topk_idx;
  float   *topk_w;
  int32_t *counts;
  int32_t *offsets;
  int32_t *perm;
  int32_t *inv_perm;
  float   *scores;
} mrlmoe_routing;

/* Bytes of device workspace that mrlmoe_route / mrlmoe_forward need for cfg
 * (0 if cfg is invalid).  Dominant terms: the dispatched latent rows and
 * expert activations, (T*k + T) * (d_lat + d_ff) * 2 bytes, and the
 * per-slot expert outputs T * (k+1) * d_lat * 4 bytes.                       */
size_t mrlmoe_workspace_size(const mrlmoe_config *cfg);

/* Routing only (projection, routers, aggregation, bias, top-k, weights,
 * dispatch record).  x: [T, d_model] bf16, unused (may be NULL) when
 * scores_in != 0, in which case out->scores must hold the fp32 scores s
 * [T, E] to route from (this mode is bit-exact against a CPU definition).
 * bias: [E] fp32.  out: the routing record to fill (non-NULL struct).
 *
 * Precondition on the values (every routing entry point, and the routers of
 * mrlmoe_forward): scores, x and bias are finite, or at least every token has
 * k experts whose biased score s + bias is a number above -inf (NaN scores
 * and -inf biases are never selected).  A token without k such experts gets
 * expert -1 and weight 0 in its empty slots; the device status becomes
 * MRLMOE_ERR_CHECK, the call's later kernels do nothing (the dispatch record
 * and y are left unwritten), and no index outside [0, E) is ever used.       */
mrlmoe_status mrlmoe_route(const mrlmoe_config *cfg, const mrlmoe_weights *w,
                           const float *bias, const void *x, int scores_in,
                           mrlmoe_routing *out, void *workspace, size_t ws_bytes,
                           void *stream);

/* The full layer forward: y [T, d_model] bf16 from x [T, d_model] bf16.
 * route_out may be NULL; otherwise its non-NULL fields receive the routing
 * record of this call (scores, if non-NULL, are an output here).              */
mrlmoe_status mrlmoe_forward(const mrlmoe_config *cfg, const mrlmoe_weights *w,
                             const float *bias, const void *x, void *y,
                             mrlmoe_routing *route_out, void *workspace,
                             size_t ws_bytes, void *stream);

/* Same as mrlmoe_forward, and records caller-created CUDA events
 * (cudaEvent_t, cast to void*) on `stream` at the stage boundaries, so a
 * caller can time each kernel of the layer without a profiler:
 *   events[0] before the down-projection      events[5] after the gate/up GEMM
 *   events[1] after the down-projection       events[6] after the down GEMM
 *   events[2] after the router + top-k        events[7] after combine + RMSNorm
 *   events[3] after the dispatch record       events[8] after the up-projection
 *   events[4] after the row gather
 * n_events must be MRLMOE_NUM_STAGE_EVENTS.                                  */
#define MRLMOE_NUM_STAGE_EVENTS 9
mrlmoe_status mrlmoe_forward_timed(const mrlmoe_config *cfg, const mrlmoe_weights *w,
                                   const float *bias, const void *x, void *y,
                                   mrlmoe_routing *route_out, void *workspace,
                                   size_t ws_bytes, void *stream,
                                   void *const *events, int n_events);

/* Balancing-bias step, in place: bias[e] += gamma * sgn(T*k - E*counts[e])
 * (sign taken exactly in 64-bit integers, sign(0) = 0; one fp32 add).
 * counts: [E] int32 from a routing record of cfg->T tokens.                  */
mrlmoe_status mrlmoe_bias_update(const mrlmoe_config *cfg, const int32_t *counts,
                                 float *bias, float gamma, void *stream);

/* One bf16 projection, out[M, N] = bf16(a[M, K] w[N, K]^T) with fp32
 * accumulation: the layer's down-projection and shared up-projection steps
 * on their own.  M >= 1; N, K multiples of 128.  No workspace.               */
mrlmoe_status mrlmoe_linear(const void *a, const void *w, void *out,
                            int M, int N, int K, void *stream);

/* Routing from caller-given fp32 scores WITHOUT a workspace (no counterpart
 * in the method's description: an entry point for callers that cannot
 * allocate device memory, e.g. code running inside a framework that owns
 * every allocation, or a graph of pre-planned buffers).  Same results as mrlmoe_route with
 * scores_in = 1: out->scores holds s [T, E]; out->topk_idx, topk_w, counts,
 * offsets, perm and inv_perm must all be non-NULL and receive the record.
 * Its scratch (per-chunk expert masks and prefixes, scaled weights, group
 * tables) lives in one static device array of MRLMOE_STATIC_SCRATCH_BYTES
 * that every GPU which loads this library holds until process exit; the
 * library allocates nothing.  Problems whose scratch would not fit (about
 * T * (8*E/32 + 4*k) bytes) are rejected with MRLMOE_ERR_SCRATCH_LIMIT before
 * anything is enqueued.  The first call on a device looks up the array's
 * device address (cudaGetSymbolAddress); make that first call before any
 * stream capture.  All calls share the one array, so calls that overlap on
 * the GPU (different streams, or graphs replayed concurrently) race: order
 * them on one stream.  Its device status word lives in the static array and
 * cannot be read directly: scores that break the routing precondition above
 * leave expert -1 in topk_idx and the rest of the record unwritten, which
 * mrlmoe_check_routing (with a 256-byte status workspace) reports as
 * MRLMOE_ERR_CHECK.                                                          */
#define MRLMOE_STATIC_SCRATCH_BYTES (2u * 1024u * 1024u)
mrlmoe_status mrlmoe_route_scores_static(const mrlmoe_config *cfg, const float *bias,
                                         const float *expert_scale, mrlmoe_routing *out,
                                         void *stream);

/* FP8 activation quantiser of the FP8 variant: for each row r and 128-wide
 * block b of in [rows, K] bf16 (K a multiple of 128), amax = max |v|;
 * scale[r*K/128 + b] = amax / 448 (1 if amax == 0) and
 * q[r*K + b*128 + i] = e4m3(v_i * 448 / amax) rounded to nearest even with
 * saturation (0 if amax == 0).  q: [rows, K] e4m3 bytes; scale: fp32.
 * Device pointers, caller-owned; in 16-byte, q 8-byte and scale 4-byte
 * aligned, else MRLMOE_ERR_INVALID_ARG (as for rows < 1 or a bad K).
 * The variant's reading of "activations quantised e4m3 per 1x128 block".    */
mrlmoe_status mrlmoe_quantize_e4m3(const void *in, int rows, int K, void *q, float *scale,
                                   void *stream);

/* ------------------------------------------------------------ training
 * Backward pass of the layer (bf16 mode only).  The pages train the model
 * with this layer and motivate the several routers by how they learn
 * (derekhsu, "多路由潛在 MoE"), but give no gradient formulas; the library's
 * readings: the top-k selection and the balancing bias carry no gradient;
 * the selected experts' scores get it through the renormalised weights
 * w = s_sel / sum(s_sel); the bf16 rounding points of the forward pass it
 * through unchanged; alpha and the RMSNorm gain are learnable; with MAX
 * aggregation the router attaining the maximum (the lowest index on ties)
 * takes the gradient.
 *
 * Gradients: device pointers, caller-owned, all required.  Weight gradients
 * are fp32 with the shapes of mrlmoe_weights; accumulate = 0 overwrites
 * them, accumulate != 0 adds this call's gradients to their contents (one
 * fp32 add per element, e.g. for micro-batches).  dx is bf16 [T, d_model]
 * and always overwritten.                                                     */
typedef struct {
  void  *dx;              /* [T, d_model] bf16                                  */
  float *d_w_down;        /* [d_lat, d_model]                                   */
  float *d_w_router;      /* [R, E, d_lat]                                      */
  float *d_w_gate;        /* [E, d_ff, d_lat]                                   */
  float *d_w_up_e;        /* [E, d_ff, d_lat]                                   */
  float *d_w_down_e;      /* [E, d_lat, d_ff]                                   */
  float *d_w_sh_gate;     /* [d_ff, d_lat]                                      */
  float *d_w_sh_up;       /* [d_ff, d_lat]                                      */
  float *d_w_sh_down;     /* [d_lat, d_ff]                                      */
  float *d_rms_gain;      /* [d_lat]                                            */
  float *d_w_up;          /* [d_model, d_lat]                                   */
  float *d_expert_scale;  /* [E]                                                */
  int    accumulate;      /* 0: write the weight gradients; else add to them   */
} mrlmoe_grads;

/* Workspace bytes for mrlmoe_forward_train + mrlmoe_backward (0 if cfg is
 * invalid, not bf16, or d_ff > 8192).  Beyond mrlmoe_workspace_size: the kept gate/up
 * pre-activations (T*k + T) * d_ff * 4 bytes and the backward's buffers,
 * about (T*k + T) * (2 * d_lat + 2 * d_ff) * 2 bytes more.                    */
size_t mrlmoe_train_workspace_size(const mrlmoe_config *cfg);

/* mrlmoe_forward that also keeps, in `workspace`, what mrlmoe_backward reads
 * (the forward's own scratch plus the bf16 gate and up pre-activations).
 * ws_bytes >= mrlmoe_train_workspace_size(cfg).  bf16 mode only
 * (MRLMOE_ERR_UNSUPPORTED otherwise), d_ff <= 8192.                           */
mrlmoe_status mrlmoe_forward_train(const mrlmoe_config *cfg, const mrlmoe_weights *w,
                                   const float *bias, const void *x, void *y,
                                   mrlmoe_routing *route_out, void *workspace,
                                   size_t ws_bytes, void *stream);

/* Gradients of a loss L with respect to x and every learnable tensor, given
 * dy = dL/dy [T, d_model] bf16, for the mrlmoe_forward_train call that last
 * used `workspace` on `stream` with the same cfg, w and x.  Nothing is
 * re-validated against that call: a different cfg, w or x gives wrong
 * gradients.  The call continues the forward's status word (it does not
 * clear it): if the forward failed, every backward kernel does nothing and
 * the status stays the forward's.  cfg->hold applies to the backward's GEMMs
 * (MRLMOE_HOLD_GEMM).  Enqueues about 14 kernels; allocates nothing.          */
mrlmoe_status mrlmoe_backward(const mrlmoe_config *cfg, const mrlmoe_weights *w,
                              const void *x, const void *dy, const mrlmoe_grads *grads,
                              void *workspace, size_t ws_bytes, void *stream);

/* Same as mrlmoe_backward, and records caller-created CUDA events on `stream`
 * at its stage boundaries (as mrlmoe_forward_timed does):
 *   events[0]  before the first kernel     events[6]  after the router/token backward
 *   events[1]  after dn = dy W_up          events[7]  after dW_router and dalpha
 *   events[2]  after dW_up                 events[8]  after the expert weight gradients
 *   events[3]  after RMSNorm/combine bwd   events[9]  after dx
 *   events[4]  after dh (W_down dgrad)     events[10] after dW_down
 *   events[5]  after dz (W_gate/W_up dgrad)
 * n_events must be MRLMOE_NUM_BACKWARD_EVENTS.                               */
#define MRLMOE_NUM_BACKWARD_EVENTS 11
mrlmoe_status mrlmoe_backward_timed(const mrlmoe_config *cfg, const mrlmoe_weights *w,
                                    const void *x, const void *dy, const mrlmoe_grads *grads,
                                    void *workspace, size_t ws_bytes, void *stream,
                                    void *const *events, int n_events);

/* ------------------------------------------------- expert parallelism
 * The layer with its routed experts spread over n_ranks ranks.  The pages
 * motivate the latent design by this layout: the experts compute in the
 * 2048-d latent, so the rows that travel to another GPU's experts are latent
 * wide (blog.derekhsu.net "ERNIE-5.5-Flash-Base", section "多路由潛在 MoE";
 * aitest123.com, section "模型结构").  They give no layout; the library's:
 * rank d owns the E/n_ranks consecutive routed experts [d E/n, (d+1) E/n);
 * the projections, routers, shared expert and RMSNorm are replicated; every
 * rank routes its own tokens.  The library computes each phase on one rank;
 * the two exchanges are the caller's (an NCCL all-to-all, or copies):
 *
 *   1. mrlmoe_ep_dispatch: this rank's tokens routed, their dispatched latent
 *      rows gathered expert-major into send_rows.  The rows for rank d are
 *      the contiguous slice offsets[d E/n] .. offsets[(d+1) E/n], and
 *      counts[d E/n .. (d+1) E/n) says how many belong to each of its experts.
 *   2. exchange: rank s sends rank d that slice and those counts.
 *   3. mrlmoe_ep_experts: on the owner, the received rows (sources in rank
 *      order, each source's rows expert-major) through its experts; row r's
 *      UNWEIGHTED output, fp32, goes to out_rows[r] (arrival order).
 *   4. exchange back: each source gets the outputs of the rows it sent, in the
 *      order it sent them, i.e. in its own dispatch order.
 *   5. mrlmoe_ep_combine: on the source, each returned row times its weight
 *      w' = w * alpha, the shared expert, the fixed-order combine, RMSNorm and
 *      the up-projection.  The additions are the single-GPU layer's, in its
 *      order and precision, so y equals mrlmoe_forward's y for the same tokens
 *      whenever the expert GEMMs reproduce each row's products.
 * bf16 mode only (else MRLMOE_ERR_UNSUPPORTED); E divisible by n_ranks,
 * 1 <= n_ranks <= 64 (else MRLMOE_ERR_INVALID_ARG).  All three calls of a rank
 * take the same cfg (cfg->T = this rank's tokens) and the same workspace, in
 * this order on one stream; mrlmoe_ep_dispatch clears the workspace's status
 * word and the other two continue it (read it with mrlmoe_get_device_status).
 * The returned rows are fp32: rounding them to bf16 on the wire would add a
 * rounding of every expert output that the single-GPU layer does not have.  */

/* Workspace bytes for the three calls on one rank, whose owner receives rows
 * from n_ranks ranks of at most cfg->T tokens each (0 if cfg or n_ranks is
 * invalid).  Beyond mrlmoe_workspace_size: the received rows expert-major and
 * their h, n_ranks * T * min(k, E/n_ranks) * (d_lat + d_ff) * 2 bytes.        */
size_t mrlmoe_ep_workspace_size(const mrlmoe_config *cfg, int n_ranks);

/* Phase 1.  x [T, d_model] bf16; bias [E]; w: w_down, w_router, expert_scale
 * (the expert matrices are not read).  out->counts [E] and out->offsets [E+1]
 * are required (the caller derives the split sizes from them); its other
 * fields are optional copies of the record.  send_rows: [T*k, d_lat] bf16,
 * 16-byte aligned, caller-owned.                                              */
mrlmoe_status mrlmoe_ep_dispatch(const mrlmoe_config *cfg, const mrlmoe_weights *w,
                                 const float *bias, const void *x, int n_ranks,
                                 mrlmoe_routing *out, void *send_rows, void *workspace,
                                 size_t ws_bytes, void *stream);

/* Phase 3, on the owner of experts [rank E/n, (rank+1) E/n).  w_local:
 * w_gate, w_up_e [E/n, d_ff, d_lat] and w_down_e [E/n, d_lat, d_ff] of the
 * owner's experts only (other fields unused).  recv_rows [n_recv, d_lat]
 * bf16; recv_counts: DEVICE int32 [n_ranks, E/n], rows of source s for local
 * expert e; n_recv = their sum (the device checks it and the counts' signs:
 * a mismatch is MRLMOE_ERR_CHECK in the status word, nothing is read through
 * the bad counts).  out_rows [n_recv, d_lat] fp32.  n_recv = 0 enqueues
 * nothing.  ws_bytes must cover n_recv rows (MRLMOE_ERR_WORKSPACE).           */
mrlmoe_status mrlmoe_ep_experts(const mrlmoe_config *cfg, const mrlmoe_weights *w_local,
                                int n_ranks, const void *recv_rows, const int32_t *recv_counts,
                                int n_recv, float *out_rows, void *workspace, size_t ws_bytes,
                                void *stream);

/* Phase 5.  ret_rows [T*k, d_lat] fp32 in this rank's dispatch order; w:
 * the shared expert, rms_gain, w_up and expert_scale; y [T, d_model] bf16.  */
mrlmoe_status mrlmoe_ep_combine(const mrlmoe_config *cfg, const mrlmoe_weights *w,
                                const float *ret_rows, void *y, void *workspace,
                                size_t ws_bytes, void *stream);

/* Synchronises `stream`, then returns the device status word of `workspace`
 * written by the last call that used it (MRLMOE_OK if none failed).          */
mrlmoe_status mrlmoe_get_device_status(const void *workspace, void *stream);

/* Invariants of a routing record that mrlmoe_check_routing verifies; each
 * failed one sets its bit (mrlmoe_get_device_detail).                         */
typedef enum {
  MRLMOE_CHECK_INDEX = 1,       /* an expert index outside [0, E)                   */
  MRLMOE_CHECK_DUPLICATE = 2,   /* a token selects one expert twice                 */
  MRLMOE_CHECK_OFFSETS = 4,     /* a negative count, or offsets not the exclusive
                                   scan of counts ending at T*k                     */
  MRLMOE_CHECK_PERM = 8,        /* perm, inv_perm not inverse bijections of [0,T*k) */
  MRLMOE_CHECK_GROUP = 16,      /* a dispatch row outside its expert's row range    */
  MRLMOE_CHECK_ORDER = 32,      /* an expert's rows not in ascending t*k+j order    */
  MRLMOE_CHECK_WEIGHT = 64      /* a routing weight that is not finite              */
} mrlmoe_check_bits;

/* Device check of the routing record of cfg->T tokens: the invariants above,
 * every index range-checked before use, so a corrupt record is reported and
 * never dereferenced out of bounds.  r's non-NULL fields name the record (as
 * filled by mrlmoe_route / mrlmoe_forward); NULL fields are read from the
 * workspace copy that those calls keep.  If any of topk_idx, counts, offsets,
 * perm, inv_perm is NULL, ws_bytes must be at least mrlmoe_workspace_size(cfg),
 * else 256 (the status header).  The weights are checked from r->topk_w, or
 * from the workspace copy when the workspace is full-sized, else skipped.  clear != 0
 * zeroes the workspace's status header first; clear == 0 keeps the status of
 * the call it follows on `stream`.  A failure sets MRLMOE_ERR_CHECK (if the
 * status was clear) and the failed invariants' bits; read them with
 * mrlmoe_get_device_detail.  Enqueues one kernel.                            */
mrlmoe_status mrlmoe_check_routing(const mrlmoe_config *cfg, const mrlmoe_routing *r,
                                   void *workspace, size_t ws_bytes, int clear,
                                   void *stream);

/* As mrlmoe_get_device_status; also stores the OR of the mrlmoe_check_bits
 * that failed since the header was last cleared in *check_bits (non-NULL).   */
mrlmoe_status mrlmoe_get_device_detail(const void *workspace, uint32_t *check_bits,
                                       void *stream);

/* Static, human-readable name of a status code.                              */
const char *mrlmoe_status_string(mrlmoe_status s);

#ifdef __cplusplus
}
#endif
#endif /* MRLMOE_H_ */
