/*
 * fused_moe.h -- C ABI of a fused Mixture-of-Experts layer for NVIDIA B200 (sm_100a).
 *
 * The layer.  A fused MoE merges token routing, data shuffling and the expert-network
 * computations into one batched GPU operation instead of separate sequential loops
 * (readmex.ai story "AWS details fused MoE kernel optimizations on SageMaker, up to 10%
 * throughput gain", opening section; agentic-affairs.com, "Swap-AB targets matrix
 * execution on Hopper").  For T tokens x[T,H], E experts and top_k = k:
 *
 *   route:    logits = x . router_w^T (fp32), the k largest per token, weights =
 *             softmax over all E renormalised over the k chosen experts
 *   permute:  rows (t, j) grouped by expert (stable), activations gathered in that
 *             order and, for FP8, quantised to e4m3 with a per-tensor scale
 *   experts:  per expert e, h = SiLU(A_e . W1_e^T) * (A_e . W3_e^T), y = h . W2_e^T,
 *             fp32 accumulation; FP8 weights carry one fp32 scale per expert and
 *             tensor ("tensor-quantized" FP8: readmex.ai opening section;
 *             agentic-affairs.com, "Triton improves the FP8 execution path"); h is
 *             re-quantised per tensor before the second contraction; each row is
 *             multiplied by its routing weight
 *   combine:  out[t] = bf16( sum over j < k of y[row of (t, j)] ), in slot order
 *
 * Readings where the pages are silent: router logits are summed in fp32 in a fixed
 * order (chunks of 8 columns, chunk c on lane c mod 32, ascending, then an xor
 * butterfly 16,8,4,2,1), so expert choice is exactly reproducible; top-k ties go to
 * the lower expert index; activation scales are amax/448 (dynamic, the default) or a
 * static value; rows 0..I-1 of w13 are W1 (gate) and rows I..2I-1 are W3 (up).
 *
 * Conventions for every call.
 *  - Pointers named "device" are CUDA device pointers, 16-byte aligned; the caller
 *    owns all memory.  The library never allocates or frees memory and never
 *    synchronises the stream, except in the calls documented as synchronous.
 *  - Layouts are row-major and contiguous.  bf16 values are passed as raw 16-bit
 *    patterns, e4m3 values as bytes (OCP e4m3fn: bias 7, max 448, no infinities).
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Work is enqueued
 *    asynchronously on it; results are valid once the stream reaches that point.
 *  - Argument checks run before any CUDA call and return synchronously:
 *      FMOE_ERR_INVALID_ARG  null dims / pointer, T < 0, H, I < 1, E < 1 or > 256,
 *                            top_k < 1 or > E, unknown wdtype / variant / routing
 *                            mode, routing parameters outside their ranges (n_shared
 *                            outside 0..8 included), FP8 without weight scales
 *      FMOE_ERR_UNSUPPORTED  H % 256 != 0, I % 128 != 0, H > 16384, a device pointer
 *                            not 16-byte aligned, sizes whose element counts exceed
 *                            2^31
 *      FMOE_ERR_WORKSPACE    ws_bytes < fused_moe_workspace_size(dims), or ws not
 *                            256-byte aligned
 *    T == 0 returns FMOE_OK after the dims checks and launches nothing.
 *    FMOE_ERR_CUDA reports a failed launch (cudaGetLastError after the launch).
 *  - Device-side problems (a bounded wait that ran out: FMOE_ERR_TIMEOUT; an expert
 *    id outside [0, E) in topk_ids: FMOE_ERR_DEVICE_BOUNDS) are recorded in a sticky
 *    status word inside the workspace and read with fused_moe_get_device_status.
 *  - The steps share state through the workspace: permute stores the activation
 *    scale it used there and experts reads it back, so use one workspace (sized for
 *    the same dims) for the steps of one call sequence.  Calls that use the same
 *    workspace must not overlap on the GPU.
 */
#ifndef FUSED_MOE_H_
#define FUSED_MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FUSED_MOE_ABI_VERSION 4

#if defined(__GNUC__)
#define FMOE_API __attribute__((visibility("default")))
#else
#define FMOE_API
#endif

typedef enum {
  FMOE_OK = 0,
  FMOE_ERR_INVALID_ARG = 1,
  FMOE_ERR_UNSUPPORTED = 2,
  FMOE_ERR_WORKSPACE = 3,
  FMOE_ERR_CUDA = 4,
  FMOE_ERR_TIMEOUT = 5,
  FMOE_ERR_DEVICE_BOUNDS = 6
} fmoe_status;

/* Storage format of the activations entering the contractions and of the weights. */
typedef enum {
  FMOE_BF16 = 0,     /* bf16 weights, no quantisation; h rounded to bf16 */
  FMOE_FP8_E4M3 = 1  /* e4m3 weights with per-expert fp32 scales; e4m3 activations */
} fmoe_wdtype;

/* Tile shape of the grouped GEMMs.  AUTO picks SWAP_AB when an expert receives at
 * most 64 rows on average (T*k/E <= 64), NORMAL for 65..128 rows and NORMAL_PAIR above.
 * SWAP_AB puts 128 weight rows in the MMA's M slot and the expert's tokens in N
 * (decode); NORMAL puts 128 tokens in M and 256 weight rows in N (prefill); NORMAL_PAIR
 * runs the NORMAL tiles on pairs of CTAs (clusters of two on one TPC) that share one
 * MMA over 256 tokens x 256 weight rows, each CTA staging half of the weight rows.
 * NORMAL and NORMAL_PAIR give identical results; SWAP_AB agrees with them up to fp32
 * summation order. */
typedef enum {
  FMOE_VARIANT_AUTO = 0,
  FMOE_VARIANT_SWAP_AB = 1,
  FMOE_VARIANT_NORMAL = 2,
  FMOE_VARIANT_NORMAL_PAIR = 3
} fmoe_variant;

/* How tokens choose experts.
 *  FMOE_ROUTE_SOFTMAX: the k largest logits; weights = softmax over all E experts
 *    renormalised over the k chosen.
 *  FMOE_ROUTE_SIGMOID_GROUPED: the group-limited router of DeepSeek-V3 (the pages name
 *    the model but not its router; this follows its published design):
 *    s = fp32(sigmoid(logit)) (evaluated in fp64, rounded once), sb = s + bias[e] (fp32);
 *    the E experts form n_group groups of E/n_group consecutive experts, a group scores
 *    the sum of its two largest sb, the topk_group best groups are kept (ties to the
 *    lower group), then the k largest sb inside them (ties to the lower expert);
 *    weights = s / (sum of the chosen s) * routed_scaling. */
typedef enum { FMOE_ROUTE_SOFTMAX = 0, FMOE_ROUTE_SIGMOID_GROUPED = 1 } fmoe_route_mode;

/* Shared experts (either mode; DeepSeek-V3's always-active experts): n_shared = S > 0
 * appends experts E..E+S-1, which every token uses with weight exactly 1 (outside the
 * renormalisation and outside routed_scaling).  They take slots k..k+S-1 of each token,
 * after its k routed slots, so with K = k + S:
 *   w13 [E+S, 2I, H], w2 [E+S, H, I] and the FP8 weight scales [E+S] hold the routed
 *   experts first and the shared ones after them; router_w and bias stay [E];
 *   topk_ids / topk_w are [T, K]; counts [E+S]; offsets [E+S+1]; sorted_rows,
 *   inv_perm [T*K]; a_perm, y_perm [T*K, H]; the combine sums the K slots in order.
 * Shared rows take part in the per-tensor scale of h like every other row. */
typedef struct {
  int32_t mode;           /* fmoe_route_mode */
  int32_t n_group;        /* SIGMOID_GROUPED: 1..32 groups, E % n_group == 0, E/n_group >= 2 */
  int32_t topk_group;     /* SIGMOID_GROUPED: 1..n_group, topk_group * E/n_group >= top_k */
  float routed_scaling;   /* SIGMOID_GROUPED: > 0, multiplies the renormalised weights */
  const float* bias;      /* SIGMOID_GROUPED: [E] device fp32 selection bias, or NULL */
  int32_t n_shared;       /* 0..8 shared experts (any mode) */
} fmoe_routing;

typedef struct {
  int32_t T;        /* tokens */
  int32_t H;        /* hidden size */
  int32_t I;        /* expert intermediate size */
  int32_t E;        /* experts */
  int32_t top_k;    /* experts per token */
  int32_t wdtype;   /* fmoe_wdtype */
  int32_t variant;  /* fmoe_variant */
  const fmoe_routing* routing; /* host pointer, read during the call; NULL = softmax,
                                  no shared experts */
} fmoe_dims;

typedef struct {
  const float* w13_scale; /* [E] device: scale of each expert's w13 (FP8 only) */
  const float* w2_scale;  /* [E] device: scale of each expert's w2 (FP8 only) */
  float a1_scale;         /* > 0: static activation scale; <= 0: amax(|x|)/448 */
  float a2_scale;         /* > 0: static scale of h; <= 0: amax(|h|)/448 */
} fmoe_scales;

typedef void* fmoe_stream; /* a cudaStream_t */

/* ABI version of the loaded library (FUSED_MOE_ABI_VERSION). */
FMOE_API int32_t fused_moe_abi_version(void);

/* Human-readable name of a status code (static string). */
FMOE_API const char* fused_moe_status_string(fmoe_status status);

/* Bytes of device workspace the calls below need for these dims; 0 if the dims are
 * invalid.  Host-only, makes no CUDA call. */
FMOE_API size_t fused_moe_workspace_size(const fmoe_dims* dims);

/* Zero the workspace header (status word and routing counters).  Call once on a new
 * workspace before its first use; the calls below leave the counters at zero.
 * Asynchronous on `stream`. */
FMOE_API fmoe_status fused_moe_workspace_init(void* ws, size_t ws_bytes, fmoe_stream stream);

/* Step 1, routing.
 *   x         [T, H]  bf16, device
 *   router_w  [E, H]  bf16, device
 *   topk_ids  [T, k]  int32 out, device: chosen experts, by descending logit
 *   topk_w    [T, k]  fp32 out, device: renormalised softmax weights
 * Also records max |x| partials in ws for the FP8 activation scale. */
FMOE_API fmoe_status fused_moe_route(const fmoe_dims* dims, const void* x, const void* router_w,
                            int32_t* topk_ids, float* topk_w, void* ws, size_t ws_bytes,
                            fmoe_stream stream);

/* Step 2, data shuffling.
 *   topk_ids    [T*k]   int32, device (from route)
 *   x           [T, H]  bf16, device
 *   scales      may be NULL (dynamic activation scale); only a1_scale is read
 *   counts      [E]     int32 out: rows per expert
 *   offsets     [E+1]   int32 out: exclusive prefix sum of counts
 *   sorted_rows [T*k]   int32 out: flattened indices t*k+j grouped by expert,
 *                       ascending within an expert
 *   inv_perm    [T*k]   int32 out: inverse of sorted_rows
 *   a_perm      [T*k, H] out: x[sorted_rows[p] / k], as e4m3 bytes (FP8: multiplied by
 *                       448/amax(|x|) in fp32, round to nearest even, saturating) or bf16
 * Needs the ws that route wrote (the max |x| partials); stores the activation scale
 * in ws for experts. */
FMOE_API fmoe_status fused_moe_permute(const fmoe_dims* dims, const int32_t* topk_ids, const void* x,
                              const fmoe_scales* scales, int32_t* counts, int32_t* offsets,
                              int32_t* sorted_rows, int32_t* inv_perm, void* a_perm, void* ws,
                              size_t ws_bytes, fmoe_stream stream);

/* Step 3, the expert networks on the permuted rows.
 *   a_perm      [T*k, H] e4m3 or bf16, device (from permute)
 *   offsets     [E+1], sorted_rows [T*k]: from permute
 *   topk_w      [T*k] fp32 routing weights in (t, j) order (from route)
 *   w13         [E, 2I, H] e4m3 bytes or bf16: rows 0..I-1 = W1 (gate), I..2I-1 = W3 (up)
 *   w2          [E, H, I]  e4m3 bytes or bf16
 *   scales      FP8: w13_scale, w2_scale required; a2_scale read
 *   y_perm      [T*k, H] fp32 out: row p = topk_w of its (t, j) times the expert MLP
 *               output of a_perm[p]
 * Uses the activation scale permute stored in ws. */
FMOE_API fmoe_status fused_moe_experts(const fmoe_dims* dims, const void* a_perm, const int32_t* offsets,
                              const int32_t* sorted_rows, const float* topk_w, const void* w13,
                              const void* w2, const fmoe_scales* scales, float* y_perm, void* ws,
                              size_t ws_bytes, fmoe_stream stream);

/* Step 4, back to token order.
 *   y_perm   [T*k, H] fp32, device;  inv_perm [T*k] int32, device
 *   out      [T, H] bf16 out: out[t] = bf16(sum over j of y_perm[inv_perm[t*k+j]]),
 *            fp32 adds in j order, round to nearest even
 * Needs no workspace. */
FMOE_API fmoe_status fused_moe_combine(const fmoe_dims* dims, const float* y_perm, const int32_t* inv_perm,
                              void* out, fmoe_stream stream);

/* The whole layer in one call: route, permute, experts, combine with every
 * intermediate kept in ws.  x [T, H] bf16, router_w [E, H] bf16, w13, w2 as above,
 * out [T, H] bf16; all device pointers.  No host synchronisation happens between
 * the steps. */
FMOE_API fmoe_status fused_moe(const fmoe_dims* dims, const void* x, const void* router_w, const void* w13,
                      const void* w2, const fmoe_scales* scales, void* out, void* ws,
                      size_t ws_bytes, fmoe_stream stream);

/* fused_moe with x and out in HOST memory (pinned memory gives asynchronous copies):
 * copies x to ws, runs the layer, copies out back and synchronises `stream` before
 * returning.  Weights and scales stay device pointers. */
FMOE_API fmoe_status fused_moe_host_io(const fmoe_dims* dims, const void* x_host, const void* router_w,
                              const void* w13, const void* w2, const fmoe_scales* scales,
                              void* out_host, void* ws, size_t ws_bytes, fmoe_stream stream);

/* ---------------------------------------------------------------------------------
 * Tensor parallelism over the intermediate dimension (N shards).
 *
 * The pages measure their serving result at 8-way tensor parallelism (agentic-affairs.com,
 * third change; modelsatwork.news, "The three changes", recompilation) and note that on
 * multi-GPU setups every GPU waits when one of them stalls (codebridge-ai.com blog
 * "AWS MoE kernel: WGMMA, Triton, TTFT", section 3).  The layer splits over the expert
 * intermediate features: shard r of N holds, for every expert, features
 * [r*I/N, (r+1)*I/N) -- those rows of W1 and of W3, and those columns of W2 -- so
 *   w13_r [E, 2*I/N, H]: rows 0..I/N-1 = W1 rows r*I/N.., rows I/N.. = W3 rows r*I/N..
 *   w2_r  [E, H, I/N]:   W2[:, :, r*I/N : (r+1)*I/N]
 * with the unsharded per-expert FP8 scales (the bytes are slices of the same tensors).
 * Routing and the activation quantisation are computed identically on every shard.  Each
 * shard's h is a slice of the unsharded h, and the per-tensor scale of h needs the max
 * over all of it, so a shard's call is split around one cross-shard exchange:
 *   1. fused_moe_tp_begin    route, permute, first contraction; writes this shard's
 *                            max |h| to amax_h (one fp32 device word)
 *   2. the caller reduces amax_h with MAX over the shards (e.g. NCCL all-reduce)
 *   3. fused_moe_tp_end      quantises h with the shards' max, second contraction and
 *                            combine into this shard's fp32 partial output [T, H]
 *   4. the caller reduces the partial outputs with SUM over the shards
 *   5. fused_moe_tp_finish   out = bf16(sum), round to nearest even
 * The result is the unsharded layer's up to fp32 summation order: the e4m3 codes of h
 * are the unsharded ones.  dims.I is the shard's I/N (a multiple of 128); the workspace
 * is sized by fused_moe_workspace_size(dims) and carries state from step 1 to step 3, so
 * use the same ws for both.  With one shard the five steps equal fused_moe.
 * T == 0 launches nothing (amax_h is not written).  The same checks and status codes as
 * fused_moe apply, and amax_h must be non-null and 4-byte aligned. */
FMOE_API fmoe_status fused_moe_tp_begin(const fmoe_dims* dims, const void* x, const void* router_w,
                                        const void* w13, const fmoe_scales* scales, float* amax_h,
                                        void* ws, size_t ws_bytes, fmoe_stream stream);

/* Step 3.  amax_h: device word holding the max of every shard's step-1 value (ignored in
 * the bf16 format and when scales->a2_scale > 0); out_partial [T, H] fp32 device out:
 * this shard's sum over the K slots of each token, before any rounding to bf16. */
FMOE_API fmoe_status fused_moe_tp_end(const fmoe_dims* dims, const void* w2, const fmoe_scales* scales,
                                      const float* amax_h, float* out_partial, void* ws,
                                      size_t ws_bytes, fmoe_stream stream);

/* Step 5.  out_sum [n] fp32, out [n] bf16 (device, 16-byte aligned); n a multiple of 8
 * (T*H always is).  Asynchronous on `stream`. */
FMOE_API fmoe_status fused_moe_tp_finish(int64_t n, const float* out_sum, void* out,
                                         fmoe_stream stream);

/* Number of kernels one fused_moe call launches for these dims: router, gemm1,
 * finalize1 (SWAP_AB only), quant_h (FP8 only), gemm2 and combine, plus permute and
 * gather unless the router runs them (T*k <= 2048; the gather only when
 * T*k*H*2 <= 128 KB).  0 for T == 0, -1 for invalid dims.  Host-only. */
FMOE_API int32_t fused_moe_launches_per_call(const fmoe_dims* dims);

/* Measurement: runs fused_moe once with a CUDA event recorded on `stream` before the
 * first and after every kernel launch, waits for the stream, and writes the device
 * time of launch i to ms_host[i] (milliseconds) and a static name of the kernel to
 * names_host[i] (may be NULL), for at most `cap` launches; *n_host = launches
 * written.  Synchronous.  Creates its CUDA events on first use. */
FMOE_API fmoe_status fused_moe_profile(const fmoe_dims* dims, const void* x, const void* router_w,
                                       const void* w13, const void* w2, const fmoe_scales* scales,
                                       void* out, void* ws, size_t ws_bytes, fmoe_stream stream,
                                       float* ms_host, const char** names_host, int32_t cap,
                                       int32_t* n_host);

/* ---------------------------------------------------------------------------------
 * Fused inverse rotary embedding + per-head FP8 quantisation.
 *
 * The pages' second kernel: a fused rotary-embedding plus FP8-quantisation kernel
 * (`_fused_inv_rope_fp8_quant_per_head`) that Triton recompiled for every new token
 * count (codebridge-ai.com blog "AWS MoE kernel: WGMMA, Triton, TTFT", section "3. Kill
 * JIT recompilation"; agentic-affairs.com, third change).  The pages give no formula;
 * this is the plainest reading of the name.  Token t of x was rotated by the angles of
 * its position pos[t]; the call undoes that and quantises every head:
 *   pairs (a, b) of the first rot_dim coordinates of a head, (i, i + rot_dim/2) for
 *   style 0 (half split) or (2i, 2i+1) for style 1 (interleaved), i < rot_dim/2:
 *     y_a =  x_a * cos(pos, i) + x_b * sin(pos, i)
 *     y_b = -(x_a * sin(pos, i)) + x_b * cos(pos, i)
 *   each product and each sum rounded to fp32 separately (no fused multiply-add);
 *   coordinates rot_dim..head_dim-1 pass through (y = x);
 *   scales[t, h] = max|y| / 448 over the head (1 for an all-zero head) and
 *   q = e4m3(y * (448 / max|y|)), the product in fp32, round to nearest even,
 *   saturating to +-448.
 */
typedef struct {
  int32_t T;         /* tokens (0: nothing to do) */
  int32_t n_heads;   /* >= 1 */
  int32_t head_dim;  /* 64, 128 or 256 */
  int32_t rot_dim;   /* rotated coordinates per head: 2*head_dim/32 <= rot_dim <= head_dim;
                        style 0: a power of two; style 1: a multiple of 2*head_dim/32 */
  int32_t style;     /* 0: pairs (i, i + rot_dim/2); 1: pairs (2i, 2i+1) */
  int32_t max_pos;   /* rows of the rotary table, >= 1 */
} fmoe_rope_dims;

/* x         [T, n_heads, head_dim] bf16, device
 * positions [T] int32, device: row of cos_sin for each token; a position outside
 *           [0, max_pos) is treated as 0 and reported as FMOE_ERR_DEVICE_BOUNDS in
 *           *device_status (if not NULL)
 * cos_sin   [max_pos, rot_dim] fp32, device: the rot_dim/2 cosines, then the rot_dim/2
 *           sines of each position's angles
 * q         [T, n_heads, head_dim] e4m3 bytes out, device
 * scales    [T, n_heads] fp32 out, device
 * device_status  int32 device word or NULL; first error kept (set it to 0 beforehand)
 * All device pointers 16-byte aligned.  Asynchronous on `stream`; no workspace.
 * Errors: FMOE_ERR_INVALID_ARG (null pointer, sizes outside the ranges above),
 * FMOE_ERR_UNSUPPORTED (alignment, element counts >= 2^31), FMOE_ERR_CUDA. */
FMOE_API fmoe_status fused_inv_rope_fp8_quant_per_head(const fmoe_rope_dims* dims, const void* x,
                                                       const int32_t* positions, const float* cos_sin,
                                                       void* q, float* scales, int32_t* device_status,
                                                       fmoe_stream stream);

/* Size of the library-owned workspace used by fused_moe_static_workspace: 64 MiB. */
#define FUSED_MOE_STATIC_WS_BYTES ((size_t)64 << 20)

/* fused_moe for callers that cannot allocate device memory.  The pages have no
 * counterpart to this call; it exists for callers such as a plugin inside a serving
 * process whose framework owns the GPU's memory pool and gives the plugin no
 * allocator, or code that must not call cudaMalloc/cudaFree because they can
 * synchronise the device.  It takes the same inputs and output as fused_moe but no
 * workspace: the workspace is a file-scope device array of FUSED_MOE_STATIC_WS_BYTES
 * that the library owns, and every GPU that loads the library holds it until the
 * process exits.  It allocates nothing.
 *   - Every argument check of fused_moe runs first, with its status codes, then dims
 *     whose fused_moe_workspace_size exceeds FUSED_MOE_STATIC_WS_BYTES are rejected with
 *     FMOE_ERR_WORKSPACE (use fused_moe with your own workspace); no CUDA call happens
 *     before these checks.
 *   - Every call looks up the array's device address in the current context (a host-side
 *     lookup that enqueues nothing); the first call in a context loads the library's
 *     module there, so make it before any stream capture.
 *   - All calls share the one array and it keeps the last call's contents; each call
 *     first clears what fused_moe_workspace_init clears (the status word and the
 *     router's tile counters).  Calls that overlap on the GPU race on the array: the
 *     caller must serialise them.
 *   - device_status (device pointer to one int32, 4-byte aligned, may be NULL)
 *     receives this call's device status word (FMOE_OK, FMOE_ERR_TIMEOUT or
 *     FMOE_ERR_DEVICE_BOUNDS) when the stream reaches the end of the call. */
FMOE_API fmoe_status fused_moe_static_workspace(const fmoe_dims* dims, const void* x,
                                                const void* router_w, const void* w13,
                                                const void* w2, const fmoe_scales* scales,
                                                void* out, int32_t* device_status,
                                                fmoe_stream stream);

/* Test of the device-side failure path: launches one warp that waits on an mbarrier
 * nothing ever arrives at, with the same bounded wait every kernel of the library
 * uses, limited to budget_ns (at most 10 s).  The wait gives up, records
 * FMOE_ERR_TIMEOUT in the workspace status word and the kernel returns normally, so
 * the CUDA context stays usable.  Asynchronous on `stream`. */
FMOE_API fmoe_status fused_moe_selftest_wait(void* ws, size_t ws_bytes, uint64_t budget_ns,
                                             fmoe_stream stream);

/* Synchronous: waits for `stream`, then returns the sticky device status recorded in
 * ws (FMOE_OK, FMOE_ERR_TIMEOUT or FMOE_ERR_DEVICE_BOUNDS), or FMOE_ERR_CUDA if the
 * wait or copy failed. */
FMOE_API fmoe_status fused_moe_get_device_status(const void* ws, fmoe_stream stream);

/* Synchronous: copies the scalars of the last call in ws to host memory:
 *   f[0..5] = amax|x|, s1, 448/amax|x| (or 1/s1), amax|h|, s2, inverse of s2
 *   i[0..2] = expert row chunks, split-K of the first and of the second contraction
 * Either pointer may be NULL. */
FMOE_API fmoe_status fused_moe_debug_scalars(const void* ws, float* f6_host, int32_t* i3_host,
                                    fmoe_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* FUSED_MOE_H_ */
