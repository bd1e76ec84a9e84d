// Data shuffling: group the routed (token, slot) rows by expert, quantise the
// activations while gathering them, and plan the grouped-GEMM work on the device.
//
// A fused MoE merges token routing, data shuffling and the expert networks into one
// GPU operation (readmex.ai story "AWS details fused MoE kernel optimizations on
// SageMaker", opening section).  The shuffle is the irregular, data-dependent part
// (explore.n1n.ai "Mixture-of-Experts Kernel Engineering on Amazon SageMaker AI",
// "The Core Bottlenecks of MoE Inference on H200 GPUs": irregular memory access and
// dynamic per-expert batch sizes), so it is done here without any host round trip.
//
// permute_kernel (one CTA): per-expert histogram, exclusive scan into offsets, and a
//   stable rank: row p of expert e lists the flattened indices t*k+j routed to e in
//   ascending order (sorted_rows), inv_perm is its inverse.  It also turns the
//   router's per-CTA max |x| into the per-tensor activation scale s1 = amax/448 and its
//   inverse 448/amax (each one fp32 division; amax == 0 gives 1; a static scale s
//   gives s and 1/s).
// gather_kernel: A[p] = x[sorted_rows[p] / k], read with 16-byte loads and, for the
//   FP8 format, multiplied by the inverse scale in fp32 and rounded to e4m3
//   (round to nearest even, saturating at +-448); token-major (each x row read once and
//   stored to its k rows p = inv_perm[t*k + j]).
// plan_kernel (one warp): splits every expert's rows into chunks of at most
//   chunk_rows rows and picks split-K factors for the swap-AB contractions.
#include "permute_body.cuh"

namespace fmoe {

namespace {

constexpr int kPermThreads = 1024;
constexpr int kGatherThreads = 256;

__global__ void __launch_bounds__(kPermThreads) permute_kernel(PermuteArgs a) {
  constexpr int kWarps = kPermThreads / 32;
  __shared__ int cnt[kMaxAllExperts];
  __shared__ int base[kMaxAllExperts + 1];
  __shared__ int wc[kWarps * kMaxAllExperts];
  griddep_wait();
  griddep_launch_dependents();
  permute_body<kWarps>(a, wc, cnt, base);
}

__global__ void __launch_bounds__(kGatherThreads) gather_kernel(GatherArgs a) {
  griddep_wait();
  griddep_launch_dependents();
  const int gwarp = (blockIdx.x * kGatherThreads + threadIdx.x) >> 5;
  const int nwarps = (gridDim.x * kGatherThreads) >> 5;
  gather_rows(a, gwarp, nwarps);
}

__global__ void plan_kernel(PlanArgs a) {
  griddep_wait();
  griddep_launch_dependents();
  build_plan(a.offsets, a.E, a.R, a.plan, a.hdr);
}

}  // namespace

cudaError_t launch_permute(const PermuteArgs& a, cudaStream_t s) {
  return launch_k(permute_kernel, dim3(1), dim3(kPermThreads), 0, s, a);
}

cudaError_t launch_gather(const GatherArgs& a, cudaStream_t s) {
  const int warps_per_block = kGatherThreads / 32;
  const int steps = a.fp8 ? a.H / 16 : a.H / 8;
  const long items = static_cast<long>(a.R / a.k) * ((steps + 32 * kGatherU - 1) / (32 * kGatherU));
  int grid = static_cast<int>((items + warps_per_block - 1) / warps_per_block);
  grid = grid < 1 ? 1 : grid;
  return launch_k(gather_kernel, dim3(grid), dim3(kGatherThreads), 0, s, a);
}

cudaError_t launch_plan(const PlanArgs& a, cudaStream_t s) {
  return launch_k(plan_kernel, dim3(1), dim3(32), 0, s, a);
}

}  // namespace fmoe
