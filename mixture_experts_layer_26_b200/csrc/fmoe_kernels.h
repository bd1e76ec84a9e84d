// Internal launcher interface between the C ABI (capi.cu) and the kernel files.
// Every launcher enqueues work on `stream` and returns cudaGetLastError().
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fmoe_common.cuh"
#include "fused_moe.h"

namespace fmoe {

// Raise a kernel's dynamic shared memory limit once per device (one bit mask per kernel).
template <auto Kernel>
inline cudaError_t set_max_dynamic_smem(int bytes) {
  static unsigned configured = 0;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  const unsigned bit = 1u << (dev & 31);
  if (configured & bit) return cudaSuccess;
  err = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (err == cudaSuccess)
    configured |= bit;
  else
    (void)cudaGetLastError();  // reported here; must not surface at a later launch check
  return err;
}

// Launch with programmatic stream serialisation (see griddep_wait in fmoe_common.cuh).
// FMOE_DISABLE_PDL=1 in the environment launches plainly instead (a debugging aid).
bool pdl_enabled();

template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                            cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
  return e != cudaSuccess ? e : cudaGetLastError();
}

// ----------------------------------------------------------------------------- permute
// How the grouped GEMMs are planned from the per-expert offsets.
struct PlanParams {
  Chunk* chunks;           // [max_chunks]
  int chunk_rows, max_chunks;
  int swap_ab;
  int units1_per_chunk;    // output tiles of the first contraction per chunk
  int units2_per_chunk;
  int kblocks1, kblocks2;  // K blocks of each contraction
  int s1max, s2max;        // largest split-K factors the workspace holds
  int num_sms;
  int32_t* ready;          // [max_chunks] per-chunk counters zeroed with the plan, or null
};

struct PermuteArgs {
  const int32_t* topk_ids;  // [R]
  int32_t* counts;          // [E]
  int32_t* offsets;         // [E + 1]
  int32_t* sorted_rows;     // [R]
  int32_t* inv_perm;        // [R]
  const float* amax_part;   // router partials
  WsHeader* hdr;
  int R, E, k;
  int fp8;                  // compute the activation scale (FP8 format)
  float a1_static;          // > 0: static scale
  int with_plan;            // also write the GEMM plan (one-call path)
  PlanParams plan;
};
cudaError_t launch_permute(const PermuteArgs& a, cudaStream_t s);

struct GatherArgs {
  const uint16_t* x;          // [T, H] bf16
  const int32_t* sorted_rows; // [R]
  const int32_t* inv_perm;    // [R]: permuted row of each (token, slot)
  void* a_perm;               // [R, H] e4m3 bytes or bf16
  const WsHeader* hdr;        // inv1
  int32_t* status;
  int R, H, k;
  int fp8;
};
cudaError_t launch_gather(const GatherArgs& a, cudaStream_t s);

// ----------------------------------------------------------------------------- router
struct RouterArgs {
  const uint16_t* x;       // [T, H] bf16 bits
  const uint16_t* wr;      // [E, H] bf16 bits
  int32_t* topk_ids;       // [T, k]
  float* topk_w;           // [T, k]
  float* amax_part;        // [token tiles] per-tile max |x|
  float* logits_g;         // [T, E] logits when the experts are split over CTAs
  int32_t* tile_counters;  // [kRouterMaxTiles] zero between calls (self-resetting)
  WsHeader* hdr;
  int T, H, E, k;          // E routed experts, k routed slots per token
  int n_shared;            // shared experts E..E+n_shared-1: slots k.., weight 1
  int num_sms;
  int experts_per_cta;     // set by the launcher
  // routing mode (fmoe_route_mode) and the grouped-sigmoid parameters
  int mode, n_group, topk_group;
  float routed_scaling;
  const float* bias;       // [E] or null
  // one-call path, small batches: the CTA that finishes the last token tile also runs
  // the permutation (+ plan) and, if fuse_gather, the gather
  int fuse_permute, fuse_gather;
  int32_t* route_done;     // tiles finished so far (zero between calls)
  PermuteArgs perm;
  GatherArgs gather;
};
// Token tiles that may split their experts over several CTAs (counters in the header area).
constexpr int kRouterMaxTiles = 4096;
cudaError_t launch_router(const RouterArgs& a, cudaStream_t s);

// Tiled router for large T*E (router.cu): TMA tensor maps of x [T, H] and router_w [E, H],
// bf16 without swizzle, boxes of 256 columns x router_tile_tokens(E) token rows and
// x router_tile_experts(E) expert rows.
struct alignas(64) RouterMaps {
  CUtensorMap x;
  CUtensorMap wr;
};
int router_tile_tokens(int E);
int router_tile_experts(int E);
// Whether (T, E) has enough token x expert tiles for the tiled router to fill the GPU.
bool router_use_tiled(int T, int E, int num_sms);
cudaError_t launch_router_tiled(const RouterArgs& a, const RouterMaps& m, cudaStream_t s);
int router_tokens_per_cta(int T, int H, int E, int num_sms);
int router_experts_per_warp(int E);

// ----------------------------------------------------------------------------- experts
struct PlanArgs {
  const int32_t* offsets;  // [E + 1]
  WsHeader* hdr;
  int R, E;
  PlanParams plan;
};
cudaError_t launch_plan(const PlanArgs& a, cudaStream_t s);

struct GemmArgs {
  CUtensorMap map_w;       // weights [E * rows_per_expert, K], box {BK, 128} (swap-AB
                           // first contraction: box {BK, 16})
  CUtensorMap map_x;       // activations [R, K], box {BK, 16 (swap) or 128 (normal)}
  const Chunk* chunks;
  const WsHeader* hdr;
  int32_t* status;
  float* out;              // swap: partials [S][R][Nout]; normal: h [R, I] or y [R, H]
  uint16_t* out_bf16;      // first contraction, bf16 format: h rounded to bf16
  float* h_out;            // swap-AB first contraction, FP8: h [R, I] fp32
  const float* w_scale;    // [E] per-expert weight scale (FP8) or null
  const float* topk_w;     // [R] flattened routing weights (normal, second contraction)
  const int32_t* sorted_rows;
  float* amax_part;        // normal, first contraction: per-CTA max |h|
  WsHeader* hdr_w;         // amax_h_count (normal, first contraction)
  int R, K, Nout, I, H;
  int rows_per_expert;     // weight rows per expert in map_w (2I or H)
  int chunk_rows;
  int nstages;             // shared-memory pipeline depth (gemm_stages)
  int prefetch_w;          // 1: the chunk list was written at least two launches earlier,
                           // so weight tiles may be loaded before griddepcontrol.wait
  uint64_t wait_budget_ns;
  // CTA-pair second contraction, FP8: quantise h inside the kernel (launch_gemm_pair with
  // fuse_quant = 1) instead of a separate quant_h pass -- see gemm_pair.cu
  int fuse_quant;
  const float* q_h;        // [R, I] fp32 h
  uint8_t* q_hq;           // [R, I] e4m3 out: the activations map_x reads
  int32_t* q_ready;        // [max_chunks] CTAs that finished their share of each chunk (zero
                           // at launch: the plan zeroes them)
  float q_a2_static;       // > 0: static scale of h
};
// gemm = 1 (w13, gate/up) or 2 (w2); fp8 selects kind::f8f6f4 vs kind::f16.
cudaError_t launch_gemm(const GemmArgs& a, bool fp8, bool swap_ab, int gemm, int num_sms,
                        cudaStream_t s);
int gemm_stages(bool swap_ab, int chunk_rows);
// The normal variant on CTA pairs (chunks of up to 256 rows); same arguments and outputs
// as launch_gemm(..., swap_ab = false, ...).
cudaError_t launch_gemm_pair(const GemmArgs& a, bool fp8, int gemm, int num_sms, cudaStream_t s);

struct Finalize1Args {
  const float* part;        // [S][R][2I]
  const int32_t* offsets;   // [E + 1]
  const float* w13_scale;   // [E] or null
  float* h;                 // [R, I] fp32 (FP8) -- or null
  uint16_t* hq_bf16;        // [R, I] bf16 (bf16 format) -- or null
  float* amax_part;
  WsHeader* hdr;
  int R, I, E;
  int fp8;
};
cudaError_t launch_finalize1(const Finalize1Args& a, int num_sms, cudaStream_t s);

struct QuantHArgs {
  const float* h;           // [R, I] fp32, or
  const uint16_t* h_bf16;   // [R, I] bf16 (when non-null)
  uint8_t* hq;              // [R, I] e4m3
  const float* amax_part;
  const float* amax_in;     // non-null: max |h| taken from this device word (tensor
                            // parallelism: the max over every shard) instead of amax_part
  WsHeader* hdr;
  int R, I;
  float a2_static;
};
cudaError_t launch_quant_h(const QuantHArgs& a, int num_sms, cudaStream_t s);

// Tensor parallelism: reduce this shard's per-CTA max |h| partials into one device word
// (0 in the bf16 format, which has no second quantisation).
struct AmaxReduceArgs {
  const float* amax_part;
  const WsHeader* hdr;      // amax_h_count
  float* amax_out;
  int fp8;
};
cudaError_t launch_amax_reduce(const AmaxReduceArgs& a, cudaStream_t s);

// Tensor parallelism: out = bf16(sum) of the shards' summed fp32 partial outputs, round to
// nearest even; n a multiple of 8.
cudaError_t launch_to_bf16(const float* in, uint16_t* out, size_t n, int num_sms, cudaStream_t s);

struct Finalize2Args {
  const float* part;        // [S][R][H]
  const int32_t* offsets;
  const float* w2_scale;
  const float* topk_w;      // [R] flattened
  const int32_t* sorted_rows;
  const WsHeader* hdr;
  int32_t* status;
  float* y;                 // [R, H]
  int R, H, E;
  int fp8;
};
cudaError_t launch_finalize2(const Finalize2Args& a, int num_sms, cudaStream_t s);

// finalize2 and combine in one pass (one-call swap-AB path): out[t] = bf16(sum over j of
// (sum over s of part[s][p_j]) * s2 * w2_scale[e_j] * topk_w[t*k+j]), p_j = inv_perm[t*k+j].
struct CombinePartialsArgs {
  const float* part;        // [S][R][H]
  const int32_t* inv_perm;  // [R]
  const int32_t* topk_ids;  // [R]
  const float* topk_w;      // [R]
  const float* w2_scale;    // [E] or null
  const WsHeader* hdr;
  uint16_t* out;            // [T, H] bf16, or
  float* out_f32;           // [T, H] fp32 sums before rounding (when non-null)
  int T, H, k, E;
  int fp8;
};
cudaError_t launch_combine_partials(const CombinePartialsArgs& a, int num_sms, cudaStream_t s);

// A wait on an mbarrier nothing arrives at, bounded by budget_ns (records ST_TIMEOUT).
cudaError_t launch_wait_selftest(WsHeader* hdr, uint64_t budget_ns, cudaStream_t s);

struct CombineArgs {
  const float* y;           // [R, H]
  const int32_t* inv_perm;  // [R]
  uint16_t* out;            // [T, H] bf16, or
  float* out_f32;           // [T, H] fp32 sums before rounding (when non-null)
  int T, H, k;
};
cudaError_t launch_combine(const CombineArgs& a, int num_sms, cudaStream_t s);

// ----------------------------------------------------------------------------- host checks
// The argument checks fused_moe runs before any CUDA call (capi.cu): dims, then for
// T > 0 the tensor pointers (non-null, 16-byte aligned) and the FP8 weight scales.
fmoe_status check_layer_args(const fmoe_dims* dims, const void* x, const void* router_w,
                             const void* w13, const void* w2, const fmoe_scales* scales,
                             const void* out);

// ----------------------------------------------------------------------------- inverse RoPE
struct RopeArgs {
  const uint16_t* x;        // [T, n_heads, head_dim] bf16
  const int32_t* positions; // [T]
  const float* cos_sin;     // [max_pos, rot_dim]: rot_dim/2 cosines, then sines
  uint8_t* q;               // [T, n_heads, head_dim] e4m3
  float* scales;            // [T, n_heads]
  int32_t* status;          // device status word (FMOE_ERR_DEVICE_BOUNDS), or null
  int T, n_heads, head_dim, rot_dim, style, max_pos;
};
// head_dim in {64, 128, 256}; rot_dim checked by the caller (see fused_moe.h).
cudaError_t launch_inv_rope_fp8(const RopeArgs& a, int num_sms, cudaStream_t s);

}  // namespace fmoe
