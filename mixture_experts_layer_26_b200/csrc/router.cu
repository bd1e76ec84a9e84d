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
// per token: k rounds of a warp argmax over (logit desc, expert index asc), each two
// redux.sync reductions; lane r keeps the weight of choice r, so the k weights are
// normalised by k lanes at once.  Shared experts, when present, fill the token's last slots
// with weight 1.
#include <float.h>

#include "permute_body.cuh"

namespace fmoe {

namespace {

constexpr int kRouterThreads = 256;

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  // element 2i sits in the low half of word i, element 2i+1 in the high half
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ bool better(float av, int ae, float bv, int be) {
  return av > bv || (av == bv && ae < be);
}

// Warp-wide best candidate: the largest v, ties to the smallest e -- the pair a pairwise
// reduction with better() keeps -- in two warp reductions (redux.sync) instead of five
// shuffle rounds.  Scores map to unsigned keys that order like the floats (-0 counted as
// +0, as float comparison does; NaN never occurs here).  Every lane gets the result.
__device__ __forceinline__ void warp_best(float& v, int& e) {
  uint32_t b = __float_as_uint(v);
  if (b == 0x80000000u) b = 0u;
  const uint32_t key = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  const uint32_t kmax = __reduce_max_sync(0xffffffffu, key);
  const uint32_t emin =
      __reduce_min_sync(0xffffffffu, key == kmax ? static_cast<uint32_t>(e) : 0xffffffffu);
  v = __uint_as_float((kmax & 0x80000000u) ? (kmax & 0x7fffffffu) : ~kmax);
  e = static_cast<int>(emin);
}

// Affinity of the grouped router: sigmoid evaluated in fp64, rounded once to fp32.
__device__ __forceinline__ float sigmoid_f64(float l) {
  return static_cast<float>(1.0 / (1.0 + exp(-static_cast<double>(l))));
}

// After the logits: the hand-off of a split token tile to its last CTA, top-k and the
// routing weights (one warp per token), and -- one-call path, small batches -- the
// permutation, plan and gather by the CTA that finishes the last token tile.  `logits`
// is [TB][E] (and [TB][E] of grouped selection scores after it) in shared memory; when
// the experts are split over CTAs the tile's logits are in a.logits_g.  The dynamic
// shared memory from `smem` on is reused by the permutation.
template <int TB, int NTHR = kRouterThreads>
__device__ void router_tail(const RouterArgs& a, uint8_t* smem, float* logits, int tile,
                            bool split) {
  __shared__ int is_last;
  __shared__ int is_final;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = tile * TB;
  const int E = a.E;
  if (split) {
    // The last of the gridDim.y CTAs of this token tile to finish picks the top-k
    // (counter reset for the next call by that CTA).  The barrier orders every thread's
    // logits before thread 0's gpu-scope fence, whose release covers them (cumulativity).
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence();
      const int prev = atomicAdd(&a.tile_counters[tile], 1);
      is_last = prev == static_cast<int>(gridDim.y) - 1;
      if (is_last) {
        a.tile_counters[tile] = 0;
        __threadfence();
      }
    }
    __syncthreads();
    if (!is_last) return;
    for (int i = threadIdx.x; i < TB * E; i += NTHR) {
      const int t = i / E, e = i % E;
      logits[i] = (t0 + t < a.T) ? __ldcg(a.logits_g + static_cast<size_t>(t0 + t) * E + e) : 0.f;
    }
  }
  __syncthreads();

  // ---- top-k, one warp per token
  const bool grouped = a.mode == 1;
  float* sbs = logits + TB * E;  // grouped: selection scores [TB][E]
  for (int t = warp; t < TB; t += NTHR / 32) {
    const int tok = t0 + t;
    if (tok >= a.T) break;
    constexpr int kPer = kMaxExperts / 32;
    float v[kPer], aff[kPer];  // selection scores; grouped: the unbiased affinities
    bool taken[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int e = lane + 32 * j;
      float l = -INFINITY;
      aff[j] = 0.f;
      if (e < E) {
        l = logits[t * E + e];
        if (grouped) {
          aff[j] = sigmoid_f64(l);
          l = aff[j] + (a.bias != nullptr ? a.bias[e] : 0.f);
          sbs[t * E + e] = l;
        }
      }
      if (l != l) l = -INFINITY;  // NaN scores are unsupported; keep the selection well defined
      v[j] = l;
      taken[j] = e >= E;
    }
    if (grouped) {
      // group score: the sum of the group's two largest selection scores
      __syncwarp();
      const int G = a.n_group, eg = E / a.n_group;
      float gs = -INFINITY;
      if (lane < G) {
        float m1 = -INFINITY, m2 = -INFINITY;
        for (int i = 0; i < eg; ++i) {
          const float x = sbs[t * E + lane * eg + i];
          if (x > m1) {
            m2 = m1;
            m1 = x;
          } else if (x > m2) {
            m2 = x;
          }
        }
        gs = m1 + m2;
      }
      // keep the topk_group best groups (ties to the lower group)
      uint32_t keep = 0;
      bool gtaken = lane >= G;
      for (int r = 0; r < a.topk_group; ++r) {
        float bv = gtaken ? -INFINITY : gs;
        int be = gtaken ? 0x7fffffff : lane;
        warp_best(bv, be);
        keep |= 1u << be;
        if (lane == be) gtaken = true;
      }
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const int e = lane + 32 * j;
        if (e < E && !((keep >> (e / eg)) & 1u)) v[j] = -INFINITY;
      }
    }
    float top0 = 0.f, wsum = 0.f;
    const int K = a.k + a.n_shared;  // slots per token: k routed, then the shared experts
    float* wout = a.topk_w + static_cast<size_t>(tok) * K;
    int32_t* iout = a.topk_ids + static_cast<size_t>(tok) * K;
    float my_ex = 0.f;  // lane r < 32 keeps the weight and expert of choice r
    int my_e = 0;
    for (int r = 0; r < a.k; ++r) {
      float bv = -INFINITY;
      int be = 0x7fffffff;
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const int e = lane + 32 * j;
        if (!taken[j] && better(v[j], e, bv, be)) { bv = v[j]; be = e; }
      }
      warp_best(bv, be);
      float mine = 0.f;
#pragma unroll
      for (int j = 0; j < kPer; ++j)
        if (lane + 32 * j == be) {
          taken[j] = true;
          mine = aff[j];
        }
      float ex;
      if (grouped) {
        ex = __shfl_sync(0xffffffffu, mine, be & 31);  // the unbiased affinity of the choice
      } else {
        if (r == 0) top0 = bv;
        ex = expf(bv - top0);  // exp(l_j - l_max) of the j-th choice
      }
      wsum += ex;  // summed in choice order
      if (r < 32) {
        if (lane == r) {
          my_ex = ex;
          my_e = be;
        }
      } else if (lane == 0) {
        iout[r] = be;
        wout[r] = ex;
      }
    }
    // the k weights normalised lane-parallel (choices past 32 went through memory)
    const float scale = grouped ? a.routed_scaling : 1.f;
    if (lane < a.k) {
      iout[lane] = my_e;
      wout[lane] = grouped ? my_ex / wsum * scale : my_ex / wsum;
    }
    __syncwarp();
    for (int r = 32 + lane; r < a.k; r += 32) wout[r] = grouped ? wout[r] / wsum * scale : wout[r] / wsum;
    // shared experts: every token, weight exactly 1, after the routed slots
    for (int r = lane; r < a.n_shared; r += 32) {
      iout[a.k + r] = a.E + r;
      wout[a.k + r] = 1.f;
    }
  }

  if (a.fuse_permute) {
    // The CTA that finishes the last token tile groups the rows by expert (and plans
    // the GEMMs, and for small batches gathers the activations) for the whole batch.
    __syncthreads();  // this CTA's top-k results (and max |x|), published by thread 0's fence
    if (threadIdx.x == 0) {
      __threadfence();
      const int prev = atomicAdd(a.route_done, 1);
      is_final = prev == static_cast<int>(gridDim.x) - 1;  // one top-k CTA per tile
      if (is_final) {
        *a.route_done = 0;
        __threadfence();
      }
    }
    __syncthreads();
    if (!is_final) return;
    // reuse: wc[8*Ea], cnt[Ea], base[Ea+1] over all Ea experts (shared ones included)
    const int Ea = a.perm.E;
    int* ps = reinterpret_cast<int*>(smem);
    __shared__ float inv1_s;  // the activation scale, handed from the permutation to the gather
    permute_body<NTHR / 32>(a.perm, ps, ps + (NTHR / 32) * Ea, ps + (NTHR / 32 + 1) * Ea,
                            static_cast<int>(gridDim.x), &inv1_s);
    if (a.fuse_gather) {
      __syncthreads();
      gather_rows(a.gather, warp, NTHR / 32, &inv1_s);
    }
  }
}

template <int TB, int EG>
__global__ void __launch_bounds__(kRouterThreads, 2) router_kernel(RouterArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem);                    // [TB][H]
  float* logits = reinterpret_cast<float*>(smem + TB * a.H * 2);       // [TB][E]
  __shared__ float red[kRouterThreads / 32];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x, group = blockIdx.y;
  const int t0 = tile * TB;
  const int H = a.H, E = a.E;
  const int vec_per_row = H / 8;  // 16-byte vectors per row
  const bool split = gridDim.y > 1;

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
  if (threadIdx.x == 0 && group == 0) {
    float m = 0.f;
    for (int w = 0; w < kRouterThreads / 32; ++w) m = fmaxf(m, red[w]);
    a.amax_part[tile] = m;
    if (tile == 0) a.hdr->router_ctas = gridDim.x;
  }

  // ---- logits of this CTA's experts, in the canonical order
  const int steps = H / 256;  // chunks per lane
  const int e_begin = group * a.experts_per_cta;
  const int e_end = min(E, e_begin + a.experts_per_cta);
  // chunk steps whose router rows are loaded together: more when a warp owns fewer
  // experts, so that every warp keeps about eight 16-byte loads in flight
  constexpr int U = EG >= 4 ? 2 : 8 / EG;
  // Accumulators acc[t][g] are updated in pairs with one paired FMA (each component
  // rounds exactly like a scalar fmaf), element by element in ascending order, so
  // every logit keeps the canonical summation order.
  constexpr int NACC = TB * EG;
  constexpr bool kPairG = (EG % 2 == 0);  // pairs (t, g), (t, g+1); else (t, g), (t+1, g)
  for (int eb = e_begin + warp * EG; eb < e_end; eb += (kRouterThreads / 32) * EG) {
    float acc[TB][EG];
#pragma unroll
    for (int t = 0; t < TB; ++t)
#pragma unroll
      for (int g = 0; g < EG; ++g) acc[t][g] = 0.f;
    for (int s0 = 0; s0 < steps; s0 += U) {
      uint4 wv[U][EG];
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int g = 0; g < EG; ++g) {
          const int e = min(eb + g, e_end - 1);
          const int chunk = lane + 32 * min(s0 + u, steps - 1);
          wv[u][g] = __ldg(reinterpret_cast<const uint4*>(a.wr + static_cast<size_t>(e) * H) + chunk);
        }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (s0 + u < steps) {
          const int chunk = lane + 32 * (s0 + u);
          float wf[EG][8], xf[TB][8];
#pragma unroll
          for (int g = 0; g < EG; ++g) unpack8(wv[u][g], wf[g]);
#pragma unroll
          for (int t = 0; t < TB; ++t) unpack8(reinterpret_cast<const uint4*>(xs + t * H)[chunk], xf[t]);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            if constexpr (NACC % 2 == 0) {
#pragma unroll
              for (int m = 0; m < NACC; m += 2) {
                const int ta = m / EG, ga = m % EG;
                const int tb = kPairG ? ta : ta + 1, gb = kPairG ? ga + 1 : ga;
                const float2 r = __ffma2_rn(make_float2(xf[ta][i], xf[tb][i]),
                                            make_float2(wf[ga][i], wf[gb][i]),
                                            make_float2(acc[ta][ga], acc[tb][gb]));
                acc[ta][ga] = r.x;
                acc[tb][gb] = r.y;
              }
            } else {
              acc[0][0] = __fmaf_rn(xf[0][i], wf[0][i], acc[0][0]);
            }
          }
        }
      }
    }
#pragma unroll
    for (int t = 0; t < TB; ++t)
#pragma unroll
      for (int g = 0; g < EG; ++g) {
        float p = acc[t][g];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) p = p + __shfl_xor_sync(0xffffffffu, p, off);
        if (lane == 0 && eb + g < e_end) {
          if (split) {
            if (t0 + t < a.T) a.logits_g[static_cast<size_t>(t0 + t) * E + eb + g] = p;
          } else {
            logits[t * E + eb + g] = p;
          }
        }
      }
  }

  router_tail<TB>(a, smem, logits, tile, split);
}

// ------------------------------------------------------------------------------------
// Tiled router for large T*E
//
// One CTA computes the logits of TBC tokens x ECC experts.  Their x rows and router rows
// stream through shared memory in slices of 256 columns, loaded by TMA into a ring of
// kRtStages stages (one elected thread issues two tensor copies per slice), so no warp
// waits on L2 latency.  A slice holds exactly one 8-column chunk per lane and row: lane l
// reads chunk l of every row it needs, and over the slices in ascending order it adds the
// chunks l, l+32, l+64, ... of each row, element by element -- the canonical order.
// Warp w owns TBW tokens x 8 experts of the tile, one fp32 accumulator per pair and lane,
// updated with paired FMAs (each half rounds like a scalar FMA; bf16 products are exact).
// The 32 lane partials of a logit are combined by the xor butterfly 16, 8, 4, 2, 1 for 32
// logits at once by recursive halving: at each step a lane keeps the half of its logits
// whose index bit equals its lane bit and adds the partner lane's partial of the same
// logit -- the same two operands the plain butterfly adds (fp32 addition commutes) -- so
// logit j ends in lane j holding exactly the plain butterfly's value, after 31 shuffles
// instead of 160.  Max |x| (CTAs of expert group 0) is taken on the bf16 bit patterns,
// which order like the magnitudes once the sign is cleared.  The tail (expert groups
// handed to the token tile's last CTA, top-k, weights, fused permutation) is router_tail.
// ------------------------------------------------------------------------------------
constexpr int kRtStages = 8;
constexpr int kRtSlice = 256;                 // columns per slice
constexpr int kRtRowBytes = kRtSlice * 2;     // bf16
constexpr uint64_t kRtBudgetNs = 2000000000ull;
constexpr int kRtLogitsOff = 32 * 1024;       // logits after the permutation scratch
constexpr int kRtTokensPerWarp32 = 4;         // tokens per warp of the 16 x 32 tile (8, with
                                              // half the warps, measured 8-12% slower)

template <int N>
__device__ __forceinline__ void halve(float (&v)[32], int lane) {
  constexpr int off = N / 2;
  const bool upper = (lane & off) != 0;
#pragma unroll
  for (int i = 0; i < off; ++i) {
    const float send = upper ? v[i] : v[i + off];
    const float keep = upper ? v[i + off] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
  }
}

__device__ __forceinline__ float lo_bf16(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi_bf16(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t word_of(const uint4& v, int i) {
  return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

template <int TBC, int ECC>
constexpr size_t rt_stage_bytes() { return static_cast<size_t>(TBC + ECC) * kRtRowBytes; }

// Warps of the tiled router: (ECC / 8) expert groups x as many token groups as give each
// warp TBW tokens, i.e. 8 * TBW accumulators per lane.
template <int TBC, int ECC, int TBW>
constexpr int rt_warps() { return (ECC / 8) * (TBC / TBW); }

template <int TBC, int ECC, int TBW>
__global__ void __launch_bounds__(rt_warps<TBC, ECC, TBW>() * 32, 1)
    router_tiled_kernel(const __grid_constant__ RouterArgs a, const __grid_constant__ RouterMaps m) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full[kRtStages];
  __shared__ __align__(8) uint64_t empty[kRtStages];
  __shared__ int abort_flag;
  __shared__ uint32_t amax_bits;
  constexpr int NW = rt_warps<TBC, ECC, TBW>();
  constexpr int NTHR = NW * 32;
  constexpr int NG = ECC / 8;        // groups of 8 experts in the tile
  static_assert(TBW % 4 == 0 && NG * (TBC / TBW) == NW, "warp tiling");
  constexpr uint32_t kStageBytes = static_cast<uint32_t>(rt_stage_bytes<TBC, ECC>());

  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x, group = blockIdx.y;
  const int t0 = tile * TBC, e0 = group * ECC;
  const int tg = warp / NG, eg = warp % NG;
  const bool split = gridDim.y > 1;
  const int nslices = a.H / kRtSlice;
  int32_t* status = &a.hdr->status;

  if (threadIdx.x == 0) {
    for (int st = 0; st < kRtStages; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], NW);
    }
    abort_flag = 0;
    amax_bits = 0;
    fence_barrier_init();
    tma_prefetch_desc(&m.x);
    tma_prefetch_desc(&m.wr);
  }
  __syncthreads();
  griddep_wait();
  griddep_launch_dependents();

  const uint64_t pol = policy_evict_last();  // x rows and router rows are re-read by other CTAs
  auto issue = [&](int sl) {
    const int st = sl % kRtStages;
    uint8_t* dst = smem + st * kStageBytes;
    mbar_arrive_expect_tx(&full[st], kStageBytes);
    tma_load_2d(dst, &m.x, &full[st], sl * kRtSlice, t0, pol);
    tma_load_2d(dst + TBC * kRtRowBytes, &m.wr, &full[st], sl * kRtSlice, e0, pol);
  };
  int issued = 0;  // slices whose copies thread 0 started
  if (threadIdx.x == 0) {
    for (; issued < kRtStages && issued < nslices; ++issued) issue(issued);
  }

  float acc[TBW][8];
#pragma unroll
  for (int t = 0; t < TBW; ++t)
#pragma unroll
    for (int g = 0; g < 8; ++g) acc[t][g] = 0.f;
  const bool do_amax = group == 0 && eg == 0;
  uint32_t xmax = 0;  // two bf16 magnitudes, as bit patterns
  bool ok = true;
  for (int sl = 0; sl < nslices; ++sl) {
    const int st = sl % kRtStages;
    if (ok) ok = mbar_wait(&full[st], static_cast<uint32_t>((sl / kRtStages) & 1), &abort_flag, status,
                           kRtBudgetNs);
    if (ok) {
      const uint8_t* xs = smem + st * kStageBytes + (tg * TBW) * kRtRowBytes;
      const uint8_t* ws = smem + st * kStageBytes + (TBC + eg * 8) * kRtRowBytes;
      uint4 xv[TBW], wv[8];
#pragma unroll
      for (int t = 0; t < TBW; ++t) xv[t] = reinterpret_cast<const uint4*>(xs + t * kRtRowBytes)[lane];
#pragma unroll
      for (int g = 0; g < 8; ++g) wv[g] = reinterpret_cast<const uint4*>(ws + g * kRtRowBytes)[lane];
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);  // this warp has read the stage
      if (do_amax) {
#pragma unroll
        for (int t = 0; t < TBW; ++t)
#pragma unroll
          for (int q = 0; q < 4; ++q) xmax = __vmaxu2(xmax, word_of(xv[t], q) & 0x7FFF7FFFu);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float xf[TBW], wf[8];
#pragma unroll
        for (int t = 0; t < TBW; ++t) {
          const uint32_t w = word_of(xv[t], i >> 1);
          xf[t] = (i & 1) ? hi_bf16(w) : lo_bf16(w);
        }
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          const uint32_t w = word_of(wv[g], i >> 1);
          wf[g] = (i & 1) ? hi_bf16(w) : lo_bf16(w);
        }
#pragma unroll
        for (int t = 0; t < TBW; ++t)
#pragma unroll
          for (int g = 0; g < 8; g += 2) {
            const float2 r = __ffma2_rn(make_float2(xf[t], xf[t]), make_float2(wf[g], wf[g + 1]),
                                        make_float2(acc[t][g], acc[t][g + 1]));
            acc[t][g] = r.x;
            acc[t][g + 1] = r.y;
          }
      }
    }
    // refill: slice `issued` goes into the stage slice issued - kRtStages used, once every
    // warp has read that slice
    if (threadIdx.x == 0 && ok && issued < nslices && issued <= sl + kRtStages) {
      const int old = issued - kRtStages;
      if (mbar_wait(&empty[old % kRtStages], static_cast<uint32_t>((old / kRtStages) & 1), &abort_flag,
                    status, kRtBudgetNs))
        issue(issued++);
      else
        ok = false;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && abort_flag) {
    // aborted: let the copies in flight land before the CTA exits
    int dummy = 0;
    for (int sl = issued > kRtStages ? issued - kRtStages : 0; sl < issued; ++sl)
      mbar_wait(&full[sl % kRtStages], static_cast<uint32_t>((sl / kRtStages) & 1), &dummy, status,
                kRtBudgetNs);
  }
  __syncthreads();
  if (abort_flag) return;

  // ---- max |x| of this token tile (expert group 0)
  if (do_amax) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) xmax = __vmaxu2(xmax, __shfl_xor_sync(0xffffffffu, xmax, off));
    if (lane == 0) atomicMax(&amax_bits, max(xmax & 0xFFFFu, xmax >> 16));
  }

  // ---- butterfly over lanes for the warp's 32 logits, into smem or the split buffer
  float* logits = reinterpret_cast<float*>(smem + kRtLogitsOff);  // [TBC][E] (+ scores)
  const int e_end = min(a.E, e0 + ECC);
#pragma unroll
  for (int pass = 0; pass < TBW / 4; ++pass) {  // 32 logits (4 tokens x 8 experts) per pass
    float v[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = acc[4 * pass + j / 8][j % 8];
    halve<32>(v, lane);
    halve<16>(v, lane);
    halve<8>(v, lane);
    halve<4>(v, lane);
    halve<2>(v, lane);
    const int tl = tg * TBW + 4 * pass + lane / 8;  // token within the tile
    const int e = e0 + eg * 8 + (lane & 7);
    if (e < e_end) {
      if (split) {
        if (t0 + tl < a.T) a.logits_g[static_cast<size_t>(t0 + tl) * a.E + e] = v[0];
      } else {
        logits[tl * a.E + e] = v[0];
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && group == 0) {
    a.amax_part[tile] = __uint_as_float(amax_bits << 16);
    if (tile == 0) a.hdr->router_ctas = gridDim.x;
  }
  router_tail<TBC, NTHR>(a, smem, logits, tile, split);
}

template <int TBC, int ECC, int TBW>
cudaError_t launch_tiled(const RouterArgs& a0, const RouterMaps& m, cudaStream_t s) {
  RouterArgs a = a0;
  constexpr int NTHR = rt_warps<TBC, ECC, TBW>() * 32;
  constexpr size_t ring = kRtStages * rt_stage_bytes<TBC, ECC>();
  const size_t need = kRtLogitsOff + static_cast<size_t>(TBC) * a.E * 4 * 2;
  if (a.fuse_permute) {  // permute_body's scratch sits below the logits
    const size_t perm = static_cast<size_t>(NTHR / 32 + 2) * a.perm.E * 4 + 4;
    if (perm > kRtLogitsOff) return cudaErrorInvalidValue;  // cannot happen: E_all <= 264
  }
  const size_t smem = 1024 + (ring > need ? ring : need);
  cudaError_t err = set_max_dynamic_smem<router_tiled_kernel<TBC, ECC, TBW>>(static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  const int tiles = (a.T + TBC - 1) / TBC;
  const int groups = (a.E + ECC - 1) / ECC;
  a.experts_per_cta = groups == 1 ? a.E : ECC;
  return launch_k(router_tiled_kernel<TBC, ECC, TBW>, dim3(tiles, groups), dim3(NTHR), smem, s, a, m);
}

template <int TB, int EG>
cudaError_t launch_tb(RouterArgs a, cudaStream_t s) {
  size_t smem = static_cast<size_t>(TB) * a.H * 2 + static_cast<size_t>(TB) * a.E * 4 * (a.mode == 1 ? 2 : 1);
  if (a.fuse_permute) {  // permute_body's wc, cnt, base over all experts (shared included)
    const size_t need = static_cast<size_t>(kRouterThreads / 32 + 2) * a.perm.E * 4 + 4;
    smem = smem > need ? smem : need;
  }
  cudaError_t err = set_max_dynamic_smem<router_kernel<TB, EG>>(160 * 1024);
  if (err != cudaSuccess) return err;
  // favour shared memory over L1 so that two CTAs fit per SM
  cudaFuncSetAttribute(router_kernel<TB, EG>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  const int tiles = (a.T + TB - 1) / TB;
  const int per_cta = (kRouterThreads / 32) * EG;
  int groups = (a.E + per_cta - 1) / per_cta;
  if (tiles > kRouterMaxTiles) groups = 1;  // no tile counters for that many tiles
  a.experts_per_cta = groups == 1 ? a.E : per_cta;
  return launch_k(router_kernel<TB, EG>, dim3(tiles, groups), dim3(kRouterThreads), smem, s, a);
}

template <int TB>
cudaError_t launch_eg(const RouterArgs& a, cudaStream_t s) {
  const int eg = router_experts_per_warp(a.E);
  if (eg == 4) return launch_tb<TB, 4>(a, s);
  if (eg == 2) return launch_tb<TB, 2>(a, s);
  return launch_tb<TB, 1>(a, s);
}

}  // namespace

int router_experts_per_warp(int E) { return E >= 128 ? 4 : (E >= 16 ? 2 : 1); }

// Tokens per CTA: the largest of 4, 2, 1 that still gives at least two CTAs per SM
// (counting the expert groups), else 1.
int router_tokens_per_cta(int T, int H, int E, int num_sms) {
  (void)H;
  const int per_cta = (kRouterThreads / 32) * router_experts_per_warp(E);
  const int groups = (E + per_cta - 1) / per_cta;
  for (int tb : {4, 2}) {
    const long ctas = static_cast<long>((T + tb - 1) / tb) * groups;
    if (ctas >= 2L * num_sms) return tb;
  }
  return 1;
}

int router_tile_tokens(int E) { return E <= 8 ? 32 : 16; }
int router_tile_experts(int E) { return E <= 8 ? 8 : 32; }

bool router_use_tiled(int T, int E, int num_sms) {
  const long tiles = static_cast<long>((T + router_tile_tokens(E) - 1) / router_tile_tokens(E));
  const long groups = (E + router_tile_experts(E) - 1) / router_tile_experts(E);
  return tiles * groups * 3 >= 2L * num_sms && tiles <= kRouterMaxTiles;
}

cudaError_t launch_router_tiled(const RouterArgs& a, const RouterMaps& m, cudaStream_t s) {
  if (a.E <= 8) return launch_tiled<32, 8, 4>(a, m, s);
  return launch_tiled<16, 32, kRtTokensPerWarp32>(a, m, s);
}

cudaError_t launch_router(const RouterArgs& a, cudaStream_t s) {
  switch (router_tokens_per_cta(a.T, a.H, a.E, a.num_sms)) {
    case 4: return launch_eg<4>(a, s);
    case 2: return launch_eg<2>(a, s);
    default: return launch_eg<1>(a, s);
  }
}

}  // namespace fmoe
