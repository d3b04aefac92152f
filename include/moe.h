/*
 * moe.h -- C ABI of the B200 (sm_100a) routed Mixture-of-Experts FFN layer.
 *
 * The layer is the MoE block of Gemma-4-26B-A4B: hidden H = 2816 in bf16, E = 128
 * experts, top-k = 8 softmax routing, expert intermediate I = 704, GEGLU with the tanh
 * form of GELU (cann-recipes-infer "Gemma-4-26B-A4B 模型优化报告" §1 模型概况 and §5 阶段3
 * 融合算子 "MoE Router npu_moe_gating_top_k_softmax"; Gemma-4-26B-A4B-NVFP4 Ascend
 * verification report §2.1 模型架构参数).  The shapes are runtime arguments; the limits
 * each call accepts are listed below.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Pointers marked (device) are CUDA device pointers OWNED BY THE CALLER; the library
 *    never frees them and allocates nothing on the call path.  They must be 16-byte
 *    aligned.  Arrays are dense and row-major in the layout stated at each argument.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).  All
 *    work is enqueued asynchronously on it; a call returns before the GPU finishes.
 *  - Argument errors are detected on the host before anything is launched and return
 *    MOE_ERR_INVALID_ARG (null required pointer, negative size, k < 1, k > E,
 *    misaligned pointer) or MOE_ERR_UNSUPPORTED (a shape outside the limits below).
 *    T == 0 returns MOE_OK and launches nothing.
 *  - A launch failure returns MOE_ERR_CUDA.  Device-side faults detected by the kernels
 *    themselves (a bounded wait that ran out, an out-of-range index read from memory)
 *    set a per-device error word; moe_sync_status() synchronises the stream, reads and
 *    clears it, and returns MOE_ERR_TIMEOUT / MOE_ERR_CUDA.
 *  - Inputs must be finite.  Calls on distinct workspaces may run concurrently.
 *
 * Shape limits (MOE_ERR_UNSUPPORTED otherwise):
 *    1 <= T <= 1048576;  64 <= H <= 16384, H % 64 == 0;  64 <= I <= 8192, I % 64 == 0;
 *    4 <= E <= 256, E % 4 == 0;  1 <= k <= min(8, E).
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_ABI_VERSION 6

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,
  MOE_ERR_UNSUPPORTED = 2,
  MOE_ERR_NO_WORKSPACE = 3,
  MOE_ERR_CUDA = 4,
  MOE_ERR_TIMEOUT = 5
} moe_status_t;

enum {
  /* Return the raw softmax probabilities of the k selected experts instead of
   * renormalising them to sum to one (renormalisation is the default).  Implies the
   * fp64 router path (the denominator needs every logit to fp64 accuracy). */
  MOE_FLAG_NO_RENORM = 1u << 0,
  /* Router path.  By default batches of T >= 256 screen the logits on the tensor cores
   * and recompute in fp64 only the experts that can still reach the top-k; smaller
   * batches compute every logit in fp64.  Both give the same ids.  These flags force one
   * path (testing and diagnosis); setting both is MOE_ERR_INVALID_ARG.  The screen needs
   * E % 8 == 0 (16-byte rows of W_router for its TMA loads): the default takes the fp64
   * path otherwise, and forcing the screen is then MOE_ERR_UNSUPPORTED. */
  MOE_FLAG_ROUTER_FP64 = 1u << 1,
  MOE_FLAG_ROUTER_SCREEN = 1u << 2,
  /* Record a CUDA event at every stage boundary of the call; moe_last_stage_times()
   * then reports the per-stage device times of the most recent such call. */
  MOE_FLAG_PROFILE_STAGES = 1u << 3,
  /* Expert-GEMM tile family (moe_forward).  Decode tiles (weights as the 128-row MMA
   * operand, at most 16 tokens as the other; T <= 16 only) or prefill tiles (128 sorted
   * rows x 256 columns, the default).  Setting both, or decode tiles for T > 16, is
   * MOE_ERR_INVALID_ARG. */
  MOE_FLAG_DECODE_TILES = 1u << 4,
  MOE_FLAG_PREFILL_TILES = 1u << 5,
  /* Prefill tiles run GEMM-1 (+GEGLU) and GEMM-2 as one persistent launch that hands its
   * work out dynamically: CTAs take whole (row tile, column block) units of GEMM-1, then of
   * GEMM-2, from a shared counter, and a GEMM-2 unit starts as soon as the GEMM-1 tiles it
   * reads are stored.  Every output tile is summed over its full K in one accumulator.
   * MOE_FLAG_FUSED_FFN forces one launch with a static stream-K schedule, and
   * MOE_FLAG_UNFUSED_FFN two launches with that schedule; these two give the same bytes, but
   * stream-K splits the sums of some tiles across CTAs, so their bytes can differ from the
   * default's in the last bit of a few elements.  Setting both is MOE_ERR_INVALID_ARG. */
  MOE_FLAG_UNFUSED_FFN = 1u << 6,
  MOE_FLAG_FUSED_FFN = 1u << 7,
  /* Tiles of the default (dynamically scheduled) expert FFN for batches of more than 64
   * tokens: CTA pairs -- a 2-CTA cluster computes 256 sorted rows x 256 columns with one
   * tcgen05.mma.cta_group::2, each CTA loading its own 128 rows and half of the weight
   * columns -- or single CTAs with 128-row tiles.  moe_ffn_kernel_name() tells which one a
   * batch gets by default.  Both give the same bytes (every output element is the same fp32
   * sum over K in the same order).  Setting both, or either with
   * MOE_FLAG_FUSED_FFN / MOE_FLAG_UNFUSED_FFN / MOE_FLAG_DECODE_TILES, is MOE_ERR_INVALID_ARG;
   * at 64 tokens or fewer both are ignored (the A tiles then hold at most 64 rows). */
  MOE_FLAG_FFN_PAIRS = 1u << 8,
  MOE_FLAG_FFN_SINGLE = 1u << 9,
  /* How the default expert FFN gets GEMM-1's A rows (the routed tokens' x rows, in expert
   * order) for batches of more than 64 tokens: copied first into an expert-sorted buffer by
   * one more kernel and then loaded by TMA tiles (ROWS_COPY), or gathered from x inside the
   * FFN kernel through the permutation (ROWS_GATHER).  Both give the same bytes.  The default
   * is moe_ffn_kernel_name()'s choice; setting both, or either with a static or decode tile
   * family, is MOE_ERR_INVALID_ARG; at 64 tokens or fewer both are ignored. */
  MOE_FLAG_FFN_ROWS_COPY = 1u << 10,
  MOE_FLAG_FFN_ROWS_GATHER = 1u << 11
};

/* Optional caller-owned device outputs of moe_forward (any member may be NULL). */
typedef struct {
  int32_t *expert_counts;  /* [E]    pairs routed to each expert ("split sizes")     */
  int32_t *expert_offsets; /* [E+1]  exclusive scan of expert_counts                  */
  int32_t *perm;           /* [T*k]  expert-sorted position -> pair index t*k+j       */
  int32_t *topk_ids;       /* [T*k]  as moe_route                                     */
  float *topk_weights;     /* [T*k]  as moe_route                                     */
  uint32_t *router_stats;  /* [5]    {candidates recomputed, tokens that needed the exact
                            *         sequential recomputation, largest screen error /
                            *         (|x_t| |w_e|) seen (float bits), path: 0 = fp64
                            *         logits, 1 = tensor-core screen, tokens whose fp32
                            *         pair-sum recheck was too close to call and were
                            *         recomputed in fp64 (screen path)}                 */
} moe_aux_t;

/* ABI version of the loaded library (MOE_ABI_VERSION at build time). */
int moe_abi_version(void);

/* Human-readable name of a status code (static storage, never NULL). */
const char *moe_status_string(moe_status_t s);

/* Bytes of device workspace moe_route / moe_forward need for these sizes (0 when the
 * shape is unsupported).  The workspace is caller-owned, 256-byte aligned device memory;
 * its contents need no initialisation and are scratch between calls. */
size_t moe_route_workspace_size(int T, int H, int E, int k, unsigned flags);
size_t moe_workspace_size(int T, int H, int E, int I, int k, unsigned flags);

/*
 * moe_route -- the router: logits, softmax, top-k, renormalisation
 * (optimisation report §5, "MoE Router npu_moe_gating_top_k_softmax"; top-8 of 128, §1).
 *
 *   logits   L[t,e] = sum_h x[t,h] * w_router[h,e] + router_bias[e]
 *   ids      the k experts with the largest L[t,:], slot 0 largest, equal logits ordered
 *            by the lower expert id.  The ranking is decided on values that agree with
 *            a double-precision ascending-order sum of the exact bf16 products, so it is
 *            reproducible bit for bit.
 *   weights  p = softmax over all E logits; w_j = p[id_j] / sum_i p[id_i]
 *            (or p[id_j] with MOE_FLAG_NO_RENORM).
 *
 *   x            (device) bf16 [T, H]
 *   w_router     (device) bf16 [H, E]   (E contiguous)
 *   router_bias  (device) fp32 [E], or NULL for no bias
 *   topk_ids     (device) int32 [T, k]  output
 *   topk_weights (device) fp32  [T, k]  output
 *   workspace    (device) >= moe_route_workspace_size(T,H,E,k,flags) bytes, else
 *                MOE_ERR_NO_WORKSPACE
 */
moe_status_t moe_route(const void *x, const void *w_router, const float *router_bias, int T,
                       int H, int E, int k, unsigned flags, int32_t *topk_ids,
                       float *topk_weights, void *workspace, size_t workspace_bytes,
                       void *stream);

/*
 * moe_forward -- the whole routed FFN layer: route, dispatch, expert FFNs, combine.
 *
 *   route     as moe_route
 *   dispatch  counts[e], offsets = exclusive scan, and a stable permutation that groups the
 *             (token, slot) pairs expert by expert in ascending token order (the per-expert
 *             "split sizes" of the double_routing dispatch, optimisation report §6.1)
 *   expert e  h = gelu_tanh(x W_gate[e]) * (x W_up[e]);  o = h W_down[e]
 *             (GEGLU, intermediate 704, §1; gelu_pytorch_tanh, verification report §2.1;
 *             computed as a grouped matmul, the role of SwiftGMM in "MoE推理「王炸」组合：
 *             昇腾×盘古让推理性能狂飙6-8倍", Group 4)
 *   combine   y[t] = sum_j w[t,j] * o_{t,j}
 *   Precision: bf16 operands, fp32 accumulation; h, o and y are rounded to bf16.
 *
 *   x, w_router, router_bias  as moe_route
 *   w_gate, w_up  (device) bf16 [E, H, I]  (I contiguous)
 *   w_down        (device) bf16 [E, I, H]  (H contiguous)
 *   y             (device) bf16 [T, H]  output (may not alias x)
 *   aux           NULL, or optional extra outputs (see moe_aux_t)
 *   workspace     (device) >= moe_workspace_size(T,H,E,I,k,flags) bytes
 */
moe_status_t moe_forward(const void *x, const void *w_router, const float *router_bias,
                         const void *w_gate, const void *w_up, const void *w_down, int T, int H,
                         int E, int I, int k, unsigned flags, void *y, const moe_aux_t *aux,
                         void *workspace, size_t workspace_bytes, void *stream);

/*
 * moe_dense_ffn -- the dense MLP that runs beside the MoE in every layer ("每层同时有 Dense
 * MLP 和 MoE", gate/up/down, intermediate 2112, GELU: cann-recipes-infer "Gemma-4-26B-A4B
 * 模型优化报告", §1 模型概况), in the experts' GEGLU form:
 *
 *   y = (gelu_tanh(x W_gate) * (x W_up)) W_down
 *   Precision: bf16 operands, fp32 accumulation; h and y are rounded to bf16.
 *
 *   x       (device) bf16 [T, H]
 *   w_gate, w_up  (device) bf16 [H, I]  (I contiguous)
 *   w_down  (device) bf16 [I, H]  (H contiguous)
 *   y       (device) bf16 [T, H]  output (may not alias x)
 *   workspace (device) >= moe_dense_workspace_size(T, H, I) bytes, else MOE_ERR_NO_WORKSPACE
 *   Shapes as moe_forward (H, I multiples of 64); T == 0 launches nothing.  One kernel
 *   launch (the expert FFN kernel with every row in one "expert"); y rows are written in
 *   token order, so no combine is needed.
 */
size_t moe_dense_workspace_size(int T, int H, int I);
moe_status_t moe_dense_ffn(const void *x, const void *w_gate, const void *w_up,
                           const void *w_down, int T, int H, int I, void *y, void *workspace,
                           size_t workspace_bytes, void *stream);

/*
 * The steps of moe_forward as separate calls.  An expert-parallel layer (experts split over
 * ranks, cann-recipes-infer "Gemma-4-26B-A4B 模型优化报告" §3 部署 EP8 with 16 experts per
 * rank, and §6.1 方案: the double_routing AllToAll that sends each rank the rows of its
 * experts by the per-expert "split sizes", and the local-expert AllReduce of decode) strings
 * them together around its exchanges; moe_forward runs the same kernels in one call.
 * Arguments are (device) caller-owned memory as above; T == 0 (or no rows) launches nothing.
 */

/* Dispatch (step a3 alone): from topk_ids [T, k] (int32, ids in [0, E)) write
 *   counts [E]    pairs routed to each expert ("split sizes"),
 *   offsets [E+1] their exclusive scan,
 *   perm [T*k]    expert-sorted position -> pair index t*k + j (stable: expert by expert,
 *                 ascending pair index within an expert),
 *   inv [T*k]     pair index -> expert-sorted position.
 * Limits: 1 <= E <= 256, 1 <= k <= min(8, E), T <= 1048576.  An id outside [0, E) is skipped
 * and reported by moe_sync_status() as MOE_ERR_CUDA.  Workspace: moe_dispatch_workspace_size
 * bytes (0 = unsupported shape). */
size_t moe_dispatch_workspace_size(int T, int E, int k);
moe_status_t moe_dispatch(const int32_t *topk_ids, int T, int E, int k, int32_t *counts,
                          int32_t *offsets, int32_t *perm, int32_t *inv, void *workspace,
                          size_t workspace_bytes, void *stream);

/* Row gather: xp[r, :] = x[perm[r] / k, :] for r < n_rows.  x bf16 [T, H], xp bf16
 * [n_rows, H], perm int32 [n_rows] of pair indices below T*k (a slice of moe_dispatch's perm
 * selects the rows of a range of experts).  H % 8 == 0.  A pair index out of range leaves
 * its row unwritten and is reported by moe_sync_status() as MOE_ERR_CUDA. */
moe_status_t moe_gather_rows(const void *x, const int32_t *perm, int n_rows, int T, int H, int k,
                             void *xp, void *stream);

/* Grouped expert FFN over row segments (steps a4 + a5 alone): rows are N consecutive bf16
 * rows xs [N, H] cut into n_seg segments, segment i holding seg_rows[i] rows of expert
 * seg_expert[i] (both int32 [n_seg], device), back to back from row 0; for every row r of
 * a segment of expert e
 *     out[r, :] = (gelu_tanh(xs[r] W_gate[e]) * (xs[r] W_up[e])) W_down[e]
 * with W_gate, W_up bf16 [E, H, I] and W_down bf16 [E, I, H] (the E experts this caller
 * holds), out bf16 [N, H] (may not alias xs).  Precision as moe_forward.  Segments may be
 * empty; an expert id outside [0, E), a negative count, or counts adding up to more than N
 * are reported by moe_sync_status() as MOE_ERR_CUDA and nothing is computed.
 * Limits: N <= 8388608, 1 <= n_seg <= 1024, shapes as moe_forward.  Workspace:
 * moe_expert_ffn_workspace_size bytes (0 = unsupported shape). */
size_t moe_expert_ffn_workspace_size(int N, int H, int E, int I, int n_seg);
moe_status_t moe_expert_ffn(const void *xs, int N, const int32_t *seg_rows,
                            const int32_t *seg_expert, int n_seg, const void *w_gate,
                            const void *w_up, const void *w_down, int H, int E, int I, void *out,
                            void *workspace, size_t workspace_bytes, void *stream);

/* Combine (step a6 alone): y[t, :] = sum_{j ascending} topk_weights[t, j] * o[inv[t, j], :]
 * over the slots whose expert-sorted row inv[t, j] lies in [row_lo, row_hi) (the others add
 * nothing), summed in fp32 and rounded once to bf16 -- or, with MOE_COMBINE_F32, written as
 * fp32 (a partial sum for a cross-rank reduction).  o bf16 [T*k, H] in expert-sorted row
 * order (only rows in the range are read), inv int32 [T*k], topk_weights fp32 [T*k],
 * y [T, H].  0 <= row_lo <= row_hi <= T*k; H % 8 == 0; k <= 8. */
enum { MOE_COMBINE_F32 = 1u << 0 };
moe_status_t moe_combine(const void *o, const int32_t *inv, const float *topk_weights, int T,
                         int k, int H, int row_lo, int row_hi, unsigned flags, void *y,
                         void *stream);

/*
 * NVFP4 experts.  The Gemma-4-26B-A4B-NVFP4 checkpoint keeps weights AND activations in
 * "4-bit float, group_size=16" (Gemma-4-26B-A4B-NVFP4 Ascend verification report, §2.3 量化配置
 * (NVFP4)).  The format (its published definition): E2M1 elements (magnitudes 0, 0.5, 1, 1.5,
 * 2, 3, 4, 6), one E4M3 scale per 16 consecutive elements along the reduction axis K, one fp32
 * scale per tensor; value = e2m1 * e4m3 * tensor_scale.  Quantisation of a group v[16], each
 * step one IEEE fp32 operation rounding to nearest even: amax = max |v|; s = (amax / 6) / ts;
 * s8 = E4M3(s) (saturating at 448); S = e4m3(s8) * ts; code_i = E2M1(v_i / S) (saturating
 * at 6, sign kept), or 0 when S == 0.  A weight tensor's ts = amax / (6 * 448).
 *
 * Layout of one projection with reduction depth K and N outputs (a Linear layer's weight,
 * K contiguous): codes uint8 [E][N][K/2] (byte b of a row holds element 2b in its low nibble,
 * 2b+1 in its high nibble); ts fp32 [E]; scales (E4M3 bytes) in a BLOCKED layout, the one the
 * tensor cores read: E * ceil(N/128) * (K/64) blocks of 512 bytes, ordered [e][n/128][g/4]
 * for row n and group g (= k/16); inside a block the scale of (n, g) is byte
 *     16 * (n % 32) + 4 * ((n % 128) / 32) + (g % 4),
 * and rows N .. ceil(N/128)*128 - 1 hold scale 0.  The layer's projections: gate and up with
 * K = H, N = I; down with K = I, N = H.
 */
typedef struct {
  const uint8_t *gate_codes, *gate_scales; /* [E][I][H/2], blocked (N = I, K = H) */
  const float *gate_ts;                    /* [E]                                 */
  const uint8_t *up_codes, *up_scales;     /* [E][I][H/2], blocked (N = I, K = H) */
  const float *up_ts;                      /* [E]                                 */
  const uint8_t *down_codes, *down_scales; /* [E][H][I/2], blocked (N = H, K = I) */
  const float *down_ts;                    /* [E]                                 */
} moe_nvfp4_weights_t;

/* Quantise bf16 weights w [E][K][N] (N contiguous: the layout moe_forward takes, e.g. W_gate
 * with K = H, N = I) into the layout above: codes [E][N][K/2], blocked scales
 * (E * ceil(N/128) * K/64 * 512 bytes, 16-byte aligned), ts [E].  K % 64 == 0, K <= 16384.
 * Workspace: moe_nvfp4_quantize_workspace_size(E) bytes. */
size_t moe_nvfp4_quantize_workspace_size(int E);
moe_status_t moe_nvfp4_quantize_weights(const void *w, int E, int K, int N, uint8_t *codes,
                                        uint8_t *scales, float *ts, void *workspace,
                                        size_t workspace_bytes, void *stream);

/* The activation quantiser as a call of its own: x bf16 [rows][K] with tensor scale ts ->
 * codes [rows][K/2], scales [rows][K/16] (the decisions moe_forward_nvfp4 takes on x). */
moe_status_t moe_nvfp4_quantize_rows(const void *x, int rows, int K, float ts, uint8_t *codes,
                                     uint8_t *scales, void *stream);

/*
 * moe_forward_nvfp4 -- the routed layer with NVFP4 expert weights and activations, for
 * batches of 1 <= T <= 16 tokens (decode).  Router, dispatch and combine as moe_forward
 * (bf16 router, same ids and weights); expert e on a routed row:
 *     xq = NVFP4(x row, act_scale_x);  g = xq Wg[e];  u = xq Wu[e];  h = gelu_tanh(g) * u;
 *     hq = NVFP4(h, act_scale_h) (groups of 16 consecutive features);  o = hq Wd[e]
 * with the dequantised weights; products exact, sums in fp32, h quantised from fp32, o and y
 * rounded to bf16.  act_scale_x / act_scale_h: the fixed activation tensor scales (> 0).
 * flags: MOE_FLAG_NO_RENORM, MOE_FLAG_ROUTER_FP64 / _SCREEN, MOE_FLAG_PROFILE_STAGES only.
 * The expert FFN runs on the tensor cores (block-scaled NVFP4 MMAs, scales from the blocked
 * layout).  Limits: shapes as moe_forward, T <= 16.  Codes and scales 16-byte aligned.
 * Workspace: moe_nvfp4_workspace_size bytes.
 */
size_t moe_nvfp4_workspace_size(int T, int H, int E, int I, int k, unsigned flags);
moe_status_t moe_forward_nvfp4(const void *x, const void *w_router, const float *router_bias,
                               const moe_nvfp4_weights_t *w, int T, int H, int E, int I, int k,
                               unsigned flags, float act_scale_x, float act_scale_h, void *y,
                               const moe_aux_t *aux, void *workspace, size_t workspace_bytes,
                               void *stream);

/*
 * moe_route_static -- moe_route for callers that cannot allocate device memory.
 *
 * The pages have no counterpart of this call; it exists for the library's users.  Some
 * callers have no way to provide the workspace moe_route needs: code that runs while a
 * stream is being captured into a CUDA graph (cudaMalloc is not allowed there and would
 * synchronise the device), plugin hosts that hand a kernel only its inputs and outputs,
 * and runtimes with a fixed memory budget that forbid allocations after start-up.  This
 * entry point takes the same inputs and outputs as moe_route (all caller-owned device
 * memory) and allocates nothing: its scratch is a 4 MiB array compiled into the library,
 * which every GPU that loads the library holds until the process exits.
 *
 *   Same arguments, results and ranking guarantee as moe_route, always on the fp64 logits
 *   path.  MOE_FLAG_ROUTER_SCREEN and MOE_FLAG_PROFILE_STAGES are MOE_ERR_INVALID_ARG.
 *   The scratch a call needs is moe_route_workspace_size(T, H, E, k, MOE_FLAG_ROUTER_FP64);
 *   above 4 MiB the call returns MOE_ERR_NO_WORKSPACE and launches nothing (at the Gemma-4
 *   shape, H = 2816, E = 128, k = 8, batches of T = 1..64, 128 and 256 tokens fit).
 *   The first call on a device looks up the array's device address (cudaGetSymbolAddress
 *   with that device current); make that first call before any stream capture.
 *   All calls on a device share the one array and it keeps the last call's contents (the
 *   counters that must start at zero are cleared by every call): calls whose GPU work
 *   overlaps -- on different streams, or from several host threads -- race on it and must
 *   be serialised by the caller.
 */
moe_status_t moe_route_static(const void *x, const void *w_router, const float *router_bias,
                              int T, int H, int E, int k, unsigned flags, int32_t *topk_ids,
                              float *topk_weights, void *stream);

/* Name of the expert-FFN kernel moe_forward launches for a batch of T tokens with these
 * flags (static storage; "" for an invalid combination). */
const char *moe_ffn_kernel_name(int T, unsigned flags);

/* Synchronise `stream`, then read and clear this device's error word.
 * MOE_OK, MOE_ERR_TIMEOUT (a bounded device wait ran out), or MOE_ERR_CUDA (a CUDA error,
 * or an out-of-range index seen by a kernel). */
moe_status_t moe_sync_status(void *stream);

/* The CUDA error behind the most recent MOE_ERR_CUDA returned to this host thread: its
 * cudaError_t value (0 if none has occurred; -1 when a TMA tensor map could not be encoded),
 * and its name (static string, "" for 0).  Reading it does not clear it. */
int moe_last_cuda_error(void);
const char *moe_cuda_error_name(int code);

/* Number of kernels the most recent moe_route / moe_route_static / moe_forward call on this
 * host thread launched (memsets not counted).  A CUDA graph captured from a call replays
 * the same kernels. */
int moe_last_kernel_count(void);

/* Stage timing of the most recent call made with MOE_FLAG_PROFILE_STAGES on this host
 * thread's current device.  Synchronises on that call's last event.  Writes up to n
 * per-stage times in milliseconds to ms (host) and returns the number of stages, or -1
 * when no profiled call has been made.  moe_stage_name(i) names stage i: "router",
 * "dispatch", "expert_ffn" (GEMM-1 + GEGLU and GEMM-2, one or two kernels), "combine". */
int moe_last_stage_times(float *ms, int n);
const char *moe_stage_name(int i);

/* Testing aid for the failure path: set the wall-clock limit (ns) of every bounded wait
 * in later launches on the current device (0 restores the default of 2 s), and launch a
 * kernel that waits on a barrier nothing will ever complete, so that its bounded wait
 * runs out and raises MOE_ERR_TIMEOUT in moe_sync_status().  No other state is touched. */
moe_status_t moe_debug_set_wait_limit_ns(unsigned long long ns);
moe_status_t moe_debug_unsatisfied_wait(void *stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
