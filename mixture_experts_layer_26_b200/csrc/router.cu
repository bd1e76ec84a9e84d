// Router: logits -> top-k -> renormalised softmax weights, plus per-CTA max |x|.
//
// Token routing is the first of the three steps a fused MoE merges into one GPU
// operation (readmex.ai story "AWS details fused MoE kernel optimizations on
// SageMaker", opening section); expert selection stays on the device instead of in
// host control flow (explore.n1n.ai "Mixture-of-Experts Kernel Engineering on Amazon
// SageMaker AI", section "2. Triton Backend Routing for FP8 Quantization").
//
// Logits are summed in fp32 in one fixed order so that the expert choice is exactly
// reproducible: the H products are split into chunks of 8 consecutive columns, chunk c
// belongs to lane c mod 32, each lane accumulates its chunks in ascending order (the 8
// elements of a chunk in ascending order), then the 32 lane partials are combined by an
// xor butterfly with offsets 16, 8, 4, 2, 1.  bf16 x bf16 products are exact in fp32,
// so FMA and multiply-then-add agree and only this order matters.  The reduction runs
// on CUDA cores: a tensor-core dot product would not follow a fixed fp32 order.
//
// One CTA (8 warps) handles TB tokens.  Their x rows are staged in shared memory with
// 16-byte loads; each warp takes groups of EG experts and streams the router rows from
// L2, so each x chunk read from shared memory feeds 8*EG FMAs.  Top-k is then one warp
// per token: k rounds of a shuffle argmax over (logit desc, expert index asc).
#include <float.h>

#include "fmoe_kernels.h"

namespace fmoe {

namespace {

constexpr int kRouterThreads = 256;

__device__ __forceinline__ void fma8_bf16(float& acc, const uint4& xa, const uint4& wa) {
  const uint32_t xs[4] = {xa.x, xa.y, xa.z, xa.w};
  const uint32_t ws[4] = {wa.x, wa.y, wa.z, wa.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    // element 2i sits in the low half, element 2i+1 in the high half
    const float x0 = __uint_as_float(xs[i] << 16), x1 = __uint_as_float(xs[i] & 0xFFFF0000u);
    const float w0 = __uint_as_float(ws[i] << 16), w1 = __uint_as_float(ws[i] & 0xFFFF0000u);
    acc = __fmaf_rn(x0, w0, acc);
    acc = __fmaf_rn(x1, w1, acc);
  }
}

__device__ __forceinline__ bool better(float av, int ae, float bv, int be) {
  return av > bv || (av == bv && ae < be);
}

template <int TB, int EG>
__global__ void __launch_bounds__(kRouterThreads) router_kernel(RouterArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem);                    // [TB][H]
  float* logits = reinterpret_cast<float*>(smem + TB * a.H * 2);       // [TB][E]
  __shared__ float red[kRouterThreads / 32];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * TB;
  const int H = a.H, E = a.E;
  const int vec_per_row = H / 8;  // 16-byte vectors per row

  griddep_wait();
  griddep_launch_dependents();

  // ---- stage x rows (zero for tokens past T) and their max |x|
  float amax = 0.f;
  for (int i = threadIdx.x; i < TB * vec_per_row; i += kRouterThreads) {
    const int t = i / vec_per_row, v = i % vec_per_row;
    uint4 val = make_uint4(0, 0, 0, 0);
    if (t0 + t < a.T)
      val = __ldg(reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(t0 + t) * H) + v);
    reinterpret_cast<uint4*>(xs + t * H)[v] = val;
    const uint32_t w4[4] = {val.x, val.y, val.z, val.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      amax = fmaxf(amax, fabsf(__uint_as_float(w4[j] << 16)));
      amax = fmaxf(amax, fabsf(__uint_as_float(w4[j] & 0xFFFF0000u)));
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if (lane == 0) red[warp] = amax;
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = 0.f;
    for (int w = 0; w < kRouterThreads / 32; ++w) m = fmaxf(m, red[w]);
    a.amax_part[blockIdx.x] = m;
    if (blockIdx.x == 0) a.hdr->router_ctas = gridDim.x;
  }

  // ---- logits in the canonical order
  const int steps = H / 256;  // chunks per lane
  for (int eb = warp * EG; eb < E; eb += (kRouterThreads / 32) * EG) {
    float acc[TB][EG];
#pragma unroll
    for (int t = 0; t < TB; ++t)
#pragma unroll
      for (int g = 0; g < EG; ++g) acc[t][g] = 0.f;
    for (int s = 0; s < steps; ++s) {
      const int chunk = lane + 32 * s;
      uint4 wv[EG];
#pragma unroll
      for (int g = 0; g < EG; ++g) {
        const int e = min(eb + g, E - 1);
        wv[g] = __ldg(reinterpret_cast<const uint4*>(a.wr + static_cast<size_t>(e) * H) + chunk);
      }
#pragma unroll
      for (int t = 0; t < TB; ++t) {
        const uint4 xv = reinterpret_cast<const uint4*>(xs + t * H)[chunk];
#pragma unroll
        for (int g = 0; g < EG; ++g) fma8_bf16(acc[t][g], xv, wv[g]);
      }
    }
#pragma unroll
    for (int t = 0; t < TB; ++t)
#pragma unroll
      for (int g = 0; g < EG; ++g) {
        float p = acc[t][g];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) p = p + __shfl_xor_sync(0xffffffffu, p, off);
        if (lane == 0 && eb + g < E) logits[t * E + eb + g] = p;
      }
  }
  __syncthreads();

  // ---- top-k, one warp per token
  for (int t = warp; t < TB; t += kRouterThreads / 32) {
    const int tok = t0 + t;
    if (tok >= a.T) break;
    constexpr int kPer = kMaxExperts / 32;
    float v[kPer];
    bool taken[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int e = lane + 32 * j;
      float l = e < E ? logits[t * E + e] : -INFINITY;
      if (l != l) l = -INFINITY;  // NaN logits are unsupported; keep the selection well defined
      v[j] = l;
      taken[j] = e >= E;
    }
    float top0 = 0.f, wsum = 0.f;
    float* wout = a.topk_w + static_cast<size_t>(tok) * a.k;
    int32_t* iout = a.topk_ids + static_cast<size_t>(tok) * a.k;
    for (int r = 0; r < a.k; ++r) {
      float bv = -INFINITY;
      int be = 0x7fffffff;
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const int e = lane + 32 * j;
        if (!taken[j] && better(v[j], e, bv, be)) { bv = v[j]; be = e; }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
        const int oe = __shfl_xor_sync(0xffffffffu, be, off);
        if (better(ov, oe, bv, be)) { bv = ov; be = oe; }
      }
#pragma unroll
      for (int j = 0; j < kPer; ++j)
        if (lane + 32 * j == be) taken[j] = true;
      if (r == 0) top0 = bv;
      const float ex = expf(bv - top0);  // exp(l_j - l_max) of the j-th choice
      wsum += ex;                         // summed in choice order
      if (lane == 0) { iout[r] = be; wout[r] = ex; }
    }
    if (lane == 0)
      for (int r = 0; r < a.k; ++r) wout[r] = wout[r] / wsum;
  }
}

template <int TB, int EG>
cudaError_t launch_tb(const RouterArgs& a, cudaStream_t s) {
  const size_t smem = static_cast<size_t>(TB) * a.H * 2 + static_cast<size_t>(TB) * a.E * 4;
  cudaError_t err = set_max_dynamic_smem<router_kernel<TB, EG>>(160 * 1024);
  if (err != cudaSuccess) return err;
  const int grid = (a.T + TB - 1) / TB;
  return launch_k(router_kernel<TB, EG>, dim3(grid), dim3(kRouterThreads), smem, s, a);
}

template <int TB>
cudaError_t launch_eg(const RouterArgs& a, cudaStream_t s) {
  if (a.E >= 128) return launch_tb<TB, 4>(a, s);
  if (a.E >= 16) return launch_tb<TB, 2>(a, s);
  return launch_tb<TB, 1>(a, s);
}

}  // namespace

int router_tokens_per_cta(int T, int H, int E, int num_sms) {
  (void)H;
  (void)E;
  if (T >= 8 * num_sms) return 4;
  if (T >= 2 * num_sms) return 2;
  return 1;
}

cudaError_t launch_router(const RouterArgs& a, cudaStream_t s) {
  switch (router_tokens_per_cta(a.T, a.H, a.E, a.num_sms)) {
    case 4: return launch_eg<4>(a, s);
    case 2: return launch_eg<2>(a, s);
    default: return launch_eg<1>(a, s);
  }
}

}  // namespace fmoe
