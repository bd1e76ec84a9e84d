// Normal-variant grouped GEMMs on CTA pairs (tcgen05.mma with cta_group::2).
//
// The prefill tile of the one-CTA kernel (gemm.cu) is 128 token rows x 256 weight rows:
// every K step stages 16 KB of token rows and 32 KB of weight rows in shared memory for
// 128 x 256 x 128 bytes of MMA work, and the ring holds four such stages.  Here two CTAs
// of a cluster (one TPC) share an M = 256 MMA: each CTA stages its own 128 token rows and
// one half of the 256 weight rows, and the tensor cores of both SMs read both halves of
// B.  A CTA then moves 32 KB per K step for the same work per SM, and seven stages fit.
// The contraction, the tile order and the epilogue arithmetic are those of the one-CTA
// normal variant ("grouped GEMM over the experts' token chunks, scaling and SiLU(g)*u
// fused into the epilogue": agentic-affairs.com, "Triton improves the FP8 execution
// path"), so both produce identical results.
//
// Roles in each CTA of a pair (192 threads):
//   warp 0    TMA producer: this CTA's token rows and weight half; the copies complete on
//             the leader CTA's `full` barrier, which the leader arms for both CTAs' bytes
//   warp 1    allocates 512 TMEM columns for the pair; in the leader, one elected thread
//             issues the pair's MMAs and commits stage release and accumulator-ready to
//             the barriers of both CTAs
//   warps 2-5 epilogue of this CTA's 128 rows from its own TMEM; every warp reports the
//             accumulator drained on the leader's `tmem_empty` barrier
// Work units (up to 256 rows of one expert x one output tile) are spread over the pairs.
// No TMA load uses multicast: each CTA loads its own tiles.  Every wait is bounded; after
// a timeout the pair reconciles the copies either CTA issued, waits (bounded) for them
// and for the MMAs in flight, frees its TMEM and returns.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "fmoe_kernels.h"

namespace fmoe {

namespace {

// ------------------------------------------------------------------------------------
// PTX wrappers for CTA pairs (a cluster of two CTAs sharing one tcgen05 MMA)
// ------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Address of the same shared-memory offset in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t smem_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
  return r;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Arrive once on an mbarrier given by its shared::cluster address (any CTA of the
// cluster), releasing this thread's earlier accesses at cluster scope.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// mbar_wait for a barrier that threads of the other CTA of the pair arrive on
// (acquire at cluster scope); same budget and abort behaviour.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity,
                                                  volatile int* abort_flag, int32_t* status,
                                                  uint64_t budget_ns) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > budget_ns) {
      *abort_flag = 1;
      record_status(status, ST_TIMEOUT);
      return false;
    }
  }
}

// Stand in for `bytes` of copies that will never be issued (completes them on `bar`).
__device__ __forceinline__ void mbar_complete_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.complete_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ int ld_shared_cluster_s32(uint32_t cluster_addr) {
  int v;
  asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(cluster_addr) : "memory");
  return v;
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// Tiled 2-D load into this CTA's shared memory whose completion is counted on the
// pair's leader mbarrier (`leader_bar`: a shared::cluster address).  No multicast.
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, uint32_t leader_bar,
                                                 int x, int y, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(leader_bar), "r"(x), "r"(y), "l"(policy)
      : "memory");
}

// D (M = 256 across the pair) (+)= A * B^T, issued by the leader CTA only.
template <bool kFp8>
__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
  if constexpr (kFp8) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
  }
}

// Arrive on the mbarrier at `bar`'s offset in every CTA of cta_mask once the pair's
// previously issued tcgen05 operations are complete.
__device__ __forceinline__ void tc_commit_pair_mc(uint64_t* bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"(cta_mask)
      : "memory");
}

// ------------------------------------------------------------------------------------
// in-kernel quantisation of h (second contraction, FP8)
// ------------------------------------------------------------------------------------
__device__ __forceinline__ int ld_acquire_gpu(const int32_t* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void red_release_gpu_add(int32_t* p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Generic-proxy global writes before, async-proxy (TMA) reads after.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ void quant_warps_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ uint32_t e4m3x4_q(float a, float b, float c, float d) {
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return lo | (hi << 16);
}

// The per-tensor scale of h from the first contraction's per-CTA max |h| partials (one
// warp; every warp that calls it gets the same values): s2 = amax/448 and 448/amax, each one
// fp32 division, 1 for amax = 0, or a static scale s and 1/s -- the quant_h pass's rule.
__device__ __forceinline__ void h_scales(const GemmArgs& a, float& amax, float& s2, float& inv2) {
  const int lane = threadIdx.x & 31;
  const int n = a.hdr->amax_h_count;
  float m = 0.f;
  for (int i = lane; i < n; i += 32) m = fmaxf(m, a.amax_part[i]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  amax = m;
  s2 = 1.f;
  inv2 = 1.f;
  if (a.q_a2_static > 0.f) {
    s2 = a.q_a2_static;
    inv2 = 1.0f / a.q_a2_static;
  } else if (m > 0.f) {
    s2 = m / 448.0f;
    inv2 = 448.0f / m;
  }
}

// ------------------------------------------------------------------------------------
// the kernel
// ------------------------------------------------------------------------------------
constexpr int kThreads = 192;       // producer, MMA, 4 epilogue warps
constexpr int kQuantThreads = 320;  // + 4 warps quantising h (second contraction, FP8)
constexpr int kTile = 128 * 128;        // bytes of a 128-row x 128-byte operand tile
constexpr int kStageBytes = 2 * kTile;  // per CTA and K step: 128 token rows + 128 weight rows
constexpr int kStages = 7;
constexpr int kAccStages = 2;
constexpr int kAccCols = 256;
constexpr int kTmemCols = 512;
constexpr size_t kDynSmem = 1024 + static_cast<size_t>(kStages) * kStageBytes;
constexpr uint16_t kBothCtas = 0x3;

struct PairCtl {
  uint64_t full[kStages];          // leader: both CTAs' copies of a stage landed
  uint64_t empty[kStages];         // each CTA: the pair's MMAs finished reading a stage
  uint64_t tmem_full[kAccStages];  // each CTA: accumulator ready
  uint64_t tmem_empty[kAccStages]; // leader: all eight epilogue warps drained it
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int amax_bits;
  int n_chunks;
  int issued;  // stage fills this CTA's producer issued
};

struct PairUnit {
  int e, row0, nrows, tile, nch, chunk;
};

__device__ __forceinline__ uint64_t policy_evict_normal() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Unit u -> (expert chunk, output tile).  The units of expert e occupy
// [cb_e * tiles, (cb_e + nch_e) * tiles); inside an expert the chunk varies fastest, so
// pairs running at the same time share weight tiles through L2.
__device__ __forceinline__ PairUnit decode_pair_unit(long u, const Chunk* chunks, int tiles) {
  const int q = static_cast<int>(u / tiles);
  const Chunk cq = chunks[q];
  const long local = u - static_cast<long>(cq.cb) * tiles;
  const int ci = cq.cb + static_cast<int>(local % cq.nch);
  const Chunk cc = chunks[ci];
  PairUnit t;
  t.chunk = ci;
  t.tile = static_cast<int>(local / cq.nch);
  t.e = cc.e;
  t.row0 = cc.row0;
  t.nrows = cc.nrows;
  t.nch = cc.nch;
  return t;
}

template <bool kFp8, int kGemm, bool kQuant>
__global__ void __launch_bounds__(kQuant ? kQuantThreads : kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ GemmArgs a) {
  static_assert(!kQuant || (kFp8 && kGemm == 2), "h is quantised in the FP8 second contraction");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ PairCtl ctl;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  constexpr int kBK = kFp8 ? 128 : 64;  // K elements per stage (128 bytes per row)
  const int KB = a.K / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ctl.full[s], 1);
      mbar_init(&ctl.empty[s], 1);
    }
    for (int i = 0; i < kAccStages; ++i) {
      mbar_init(&ctl.tmem_full[i], 1);
      mbar_init(&ctl.tmem_empty[i], 8);
    }
    mbar_init(&ctl.drain, 1);
    ctl.abort_flag = 0;
    ctl.amax_bits = 0;
    ctl.issued = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&a.map_w);
    tma_prefetch_desc(&a.map_x);
  }
  if (warp == 1) {
    tmem_alloc_pair(&ctl.tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  // As in the one-CTA kernel: weight tiles are prefetched before waiting on the previous
  // kernel when the work list was written at least two kernels earlier (a.prefetch_w).
  const bool prefetch = a.prefetch_w != 0;
  if (!prefetch) griddep_wait();
  if (threadIdx.x == 0) ctl.n_chunks = a.hdr->n_chunks;
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers initialised, the pair's TMEM allocated
  tc_fence_after();
  if (!prefetch) {
    if (threadIdx.x == 0) griddep_launch_dependents();
  }

  const uint32_t tmem_base = ctl.tmem_base;
  const int tiles = kGemm == 1 ? a.I / 128 : a.H / 256;
  const long total = static_cast<long>(ctl.n_chunks) * tiles;
  const long pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  volatile int* abort_flag = &ctl.abort_flag;
  const uint64_t budget = a.wait_budget_ns;

  if (warp == 0) {
    // ------------------------------------------------------------- TMA producer
    if (elect_one()) {
      // a weight tile is read once per chunk of its expert: streamed when the expert has
      // one chunk, kept at normal priority for the pairs that run its other chunks
      const uint64_t pol_w_once = policy_evict_first();
      const uint64_t pol_w_shared = policy_evict_normal();
      const uint64_t pol_x = policy_evict_last();  // token rows: re-read by every tile
      int stage = 0, issued = 0;
      uint32_t phase = 0;
      bool ok = true;
      auto leader_full = [&](int st) { return map_to_rank(smem_u32(&ctl.full[st]), 0); };
      auto arm = [&](int st) {
        if (leader) mbar_arrive_expect_tx(&ctl.full[st], 2 * kStageBytes);
      };
      // this CTA's half of the weight rows: gate (rank 0) or up (rank 1) rows of the
      // tile's 128 features, or rows 128*rank.. of the tile's 256 output features
      auto load_w = [&](int st, const PairUnit& t, int kb) {
        const int wrow = t.e * a.rows_per_expert +
                         (kGemm == 1 ? t.tile * 128 + static_cast<int>(rank) * a.I
                                     : t.tile * 256 + static_cast<int>(rank) * 128);
        tma_load_2d_pair(smem + st * kStageBytes + kTile, &a.map_w, leader_full(st), kb * kBK, wrow,
                         t.nch > 1 ? pol_w_shared : pol_w_once);
      };
      // kQuant: the token rows of a chunk are e4m3 codes the quantiser warps of every CTA
      // write; wait (bounded) until all CTAs have counted the chunk done.  A wait that runs
      // out raises the abort flag; the load is still issued so that both CTAs of the pair
      // issue the same fills and the teardown below stays exact.
      int ready_upto = 0;
      auto wait_ready = [&](int c) {
        if constexpr (kQuant) {
          if (c < ready_upto || *abort_flag) return;
          const uint64_t t0 = globaltimer_ns();
          while (ld_acquire_gpu(a.q_ready + c) < static_cast<int>(gridDim.x)) {
            if (*abort_flag) return;
            if (globaltimer_ns() - t0 > budget) {
              *abort_flag = 1;
              record_status(a.status, ST_TIMEOUT);
              return;
            }
            __nanosleep(100);
          }
          ready_upto = c + 1;
          fence_proxy_async_global();
        }
      };
      auto load_x = [&](int st, const PairUnit& t, int kb) {
        wait_ready(t.chunk);
        tma_load_2d_pair(smem + st * kStageBytes, &a.map_x, leader_full(st), kb * kBK,
                         t.row0 + 128 * static_cast<int>(rank), pol_x);
      };
      auto bump = [&]() {
        ++issued;
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
      };

      long u = pair;
      int kb = 0;
      PairUnit t{};
      if (u < total) t = decode_pair_unit(u, a.chunks, tiles);
      auto next = [&]() {
        if (++kb == KB) {
          kb = 0;
          u += npairs;
          if (u < total) t = decode_pair_unit(u, a.chunks, tiles);
        }
      };
      if (prefetch) {
        // weights of the first stages (fresh stages: nothing to wait for)
        const long u_first = u;
        const PairUnit t_first = t;
        int npre = 0;
        while (u < total && npre < kStages) {
          arm(stage);
          load_w(stage, t, kb);
          bump();
          ++npre;
          next();
        }
        griddep_wait();
        griddep_launch_dependents();
        // their token rows, now that they are written
        long u2 = u_first;
        int kb2 = 0;
        PairUnit t2 = t_first;
        for (int i = 0; i < npre; ++i) {
          load_x(i, t2, kb2);
          if (++kb2 == KB) {
            kb2 = 0;
            u2 += npairs;
            if (u2 < total) t2 = decode_pair_unit(u2, a.chunks, tiles);
          }
        }
      }
      while (u < total) {
        if (!mbar_wait(&ctl.empty[stage], phase ^ 1u, abort_flag, a.status, budget)) {
          ok = false;
          break;
        }
        arm(stage);
        load_w(stage, t, kb);
        load_x(stage, t, kb);
        bump();
        next();
      }
      // tail: the MMAs' last stage releases have reached this CTA
      for (int i = 0; ok && i < kStages; ++i) {
        if (!mbar_wait(&ctl.empty[stage], phase ^ 1u, abort_flag, a.status, budget)) ok = false;
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      ctl.issued = issued;
    } else if (prefetch) {
      griddep_wait();
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer (leader)
    if (leader && elect_one()) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      const uint32_t idesc = make_idesc(kFp8, 256, 256);
      for (long u = pair; u < total && ok; u += npairs) {
        if (!mbar_wait_cluster(&ctl.tmem_empty[acc], acc_phase ^ 1u, abort_flag, a.status, budget)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(acc * kAccCols);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(&ctl.full[stage], phase, abort_flag, a.status, budget)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * kStageBytes);
          const uint64_t ad = sw128_kmajor_desc(sa);
          const uint64_t bd = sw128_kmajor_desc(sa + kTile);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc_mma_pair<kFp8>(d, ad + 2u * k, bd + 2u * k, idesc, (kb > 0 || k > 0) ? 1u : 0u);
          tc_commit_pair_mc(&ctl.empty[stage], kBothCtas);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair_mc(&ctl.tmem_full[acc], kBothCtas);
        if (++acc == kAccStages) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      // tail: every epilogue warp of both CTAs has drained the last accumulators
      for (int i = 0; ok && i < kAccStages; ++i) {
        if (!mbar_wait_cluster(&ctl.tmem_empty[acc], acc_phase ^ 1u, abort_flag, a.status, budget))
          ok = false;
        if (++acc == kAccStages) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (!ok) {
        // aborted: wait for the MMAs already issued (they read both CTAs' shared memory)
        tc_commit_pair_mc(&ctl.drain, 0x1);
        int dummy = 0;
        mbar_wait(&ctl.drain, 0, &dummy, a.status, budget);
      }
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------- epilogue
    if (prefetch) griddep_wait();  // scales and routing weights of this call
    float s2_local = 1.f;
    if constexpr (kQuant) {
      float amax_unused, inv_unused;
      h_scales(a, amax_unused, s2_local, inv_unused);
    }
    const int q = warp & 3;                   // TMEM lane quarter this warp may access
    const int r = static_cast<int>(rank) * 128 + q * 32 + lane;  // row within the unit
    int acc = 0;
    uint32_t acc_phase = 0;
    float amax = 0.f;
    for (long u = pair; u < total; u += npairs) {
      const PairUnit t = decode_pair_unit(u, a.chunks, tiles);
      const bool ready = mbar_wait(&ctl.tmem_full[acc], acc_phase, abort_flag, a.status, budget);
      __syncwarp();
      if (!__all_sync(0xffffffffu, ready)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + static_cast<uint32_t>(acc * kAccCols) +
                          (static_cast<uint32_t>(q * 32) << 16);
      const bool valid = r < t.nrows;
      if constexpr (kGemm == 1) {
        // lane = token row0 + r; columns 0..127 gate, 128..255 up of features tile*128..
        const float sc = kFp8 ? a.hdr->s1 * a.w_scale[t.e] : 1.f;
        const size_t o = static_cast<size_t>(t.row0 + r) * a.I + t.tile * 128;
        for (int c0 = 0; c0 < 128; c0 += 16) {
          float g[16], up[16], h[16];
          tmem_ld16(tb + c0, g);
          tmem_ld16(tb + 128 + c0, up);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) h[i] = silu_f(g[i] * sc) * (up[i] * sc);
          if (valid) {
            if constexpr (kFp8) {
              // fp32 h is read once, by the re-quantisation pass: streaming stores
              float4* dst = reinterpret_cast<float4*>(a.out + o + c0);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                __stcs(dst + i, make_float4(h[4 * i], h[4 * i + 1], h[4 * i + 2], h[4 * i + 3]));
                amax = fmaxf(amax, fmaxf(fmaxf(fabsf(h[4 * i]), fabsf(h[4 * i + 1])),
                                         fmaxf(fabsf(h[4 * i + 2]), fabsf(h[4 * i + 3]))));
              }
            } else {
              uint32_t pk[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const __nv_bfloat162 b2 = __floats2bfloat162_rn(h[2 * i], h[2 * i + 1]);
                pk[i] = *reinterpret_cast<const uint32_t*>(&b2);
              }
              uint4* dst = reinterpret_cast<uint4*>(a.out_bf16 + o + c0);
              dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
              dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            }
          }
        }
      } else {
        // lane = token row0 + r; columns = output features tile*256 ..
        const float sc = kFp8 ? (kQuant ? s2_local : a.hdr->s2) * a.w_scale[t.e] : 1.f;
        const int src_row = valid ? a.sorted_rows[t.row0 + r] : 0;
        const bool in_range = src_row >= 0 && src_row < a.R;
        if (valid && !in_range) record_status(a.status, ST_BOUNDS);
        const float wr = (valid && in_range) ? a.topk_w[src_row] : 0.f;
        float4* dst =
            reinterpret_cast<float4*>(a.out + static_cast<size_t>(t.row0 + r) * a.H + t.tile * 256);
        for (int c0 = 0; c0 < 256; c0 += 16) {
          float v[16];
          tmem_ld16(tb + c0, v);
          tmem_ld_wait();
          if (valid) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[c0 / 4 + i] = make_float4(v[4 * i] * sc * wr, v[4 * i + 1] * sc * wr,
                                            v[4 * i + 2] * sc * wr, v[4 * i + 3] * sc * wr);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(map_to_rank(smem_u32(&ctl.tmem_empty[acc]), 0));
      if (++acc == kAccStages) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if constexpr (kGemm == 1 && kFp8) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      if (lane == 0) atomicMax(&ctl.amax_bits, __float_as_int(amax));
    }
  } else {
    // ------------------------------------------------------------- quantisation of h
    // Every CTA quantises an equal share of every chunk, chunks in the order of the chunk
    // list (the order the units need them), and counts the chunk done; the producers of all
    // CTAs load a chunk's token rows once every CTA has counted it.
    if constexpr (kQuant) {
      griddep_wait();  // h and the max |h| partials of the first contraction are complete
      float amax2, s2, inv2;
      h_scales(a, amax2, s2, inv2);
      WsHeader* hw = a.hdr_w;
      if (blockIdx.x == 0 && threadIdx.x == 6 * 32) {  // recorded for the debug scalars
        hw->amax_h = amax2;
        hw->s2 = s2;
        hw->inv2 = inv2;
      }
      const int qt = threadIdx.x - 6 * 32;  // 0..127
      const int nc = ctl.n_chunks;
      const size_t G = gridDim.x;
      for (int c = 0; c < nc; ++c) {
        const Chunk ch = a.chunks[c];
        const size_t base = static_cast<size_t>(ch.row0) * a.I;  // elements
        const size_t n16 = static_cast<size_t>(ch.nrows) * (a.I / 16);
        const size_t per = (n16 + G - 1) / G;
        const size_t v0 = min(n16, blockIdx.x * per), v1 = min(n16, v0 + per);
        const float4* src = reinterpret_cast<const float4*>(a.q_h + base);
        uint4* dst = reinterpret_cast<uint4*>(a.q_hq + base);
        // kQU vectors of 16 values per thread in flight (256 bytes), so that 128 threads
        // per SM keep enough loads outstanding to stream h near HBM speed
        constexpr int kQU = 4;
        for (size_t v = v0 + qt; v < v1; v += 128 * kQU) {
          float4 f[kQU][4];
#pragma unroll
          for (int u = 0; u < kQU; ++u) {
            const size_t w = v + 128 * u;
            if (w < v1) {
#pragma unroll
              for (int j = 0; j < 4; ++j) f[u][j] = __ldcs(src + 4 * w + j);
            }
          }
#pragma unroll
          for (int u = 0; u < kQU; ++u) {
            const size_t w = v + 128 * u;
            if (w < v1) {
              uint4 q;
              q.x = e4m3x4_q(f[u][0].x * inv2, f[u][0].y * inv2, f[u][0].z * inv2, f[u][0].w * inv2);
              q.y = e4m3x4_q(f[u][1].x * inv2, f[u][1].y * inv2, f[u][1].z * inv2, f[u][1].w * inv2);
              q.z = e4m3x4_q(f[u][2].x * inv2, f[u][2].y * inv2, f[u][2].z * inv2, f[u][2].w * inv2);
              q.w = e4m3x4_q(f[u][3].x * inv2, f[u][3].y * inv2, f[u][3].z * inv2, f[u][3].w * inv2);
              dst[w] = q;
            }
          }
        }
        fence_proxy_async_global();  // these codes are read by TMA (the async proxy)
        quant_warps_sync();
        if (qt == 0) red_release_gpu_add(a.q_ready + c, 1);
      }
    }
  }

  __syncthreads();
  if constexpr (kGemm == 1 && kFp8) {
    if (threadIdx.x == 0) {
      a.amax_part[blockIdx.x] = __int_as_float(ctl.amax_bits);
      if (blockIdx.x == 0) a.hdr_w->amax_h_count = gridDim.x;
    }
  }
  tc_fence_before();
  cluster_sync_all();  // neither CTA issues copies or MMAs any more
  if (leader && threadIdx.x == 0) {
    const int peer_abort = ld_shared_cluster_s32(map_to_rank(smem_u32(&ctl.abort_flag), 1));
    if (ctl.abort_flag || peer_abort) {
      // Fill j of stage j % kStages completes on the leader's barrier once the leader has
      // armed it and both CTAs' bytes have landed.  The two producers stop at most one
      // ring apart; close the fills only one of them issued, then wait for every fill.
      const int nl = ctl.issued;
      const int np = ld_shared_cluster_s32(map_to_rank(smem_u32(&ctl.issued), 1));
      const int lo = min(nl, np), hi = max(nl, np);
      for (int j = lo; j < hi; ++j) {
        uint64_t* bar = &ctl.full[j % kStages];
        if (nl > np)
          mbar_complete_tx(bar, kStageBytes);  // the peer's half was never issued
        else
          mbar_arrive_expect_tx(bar, kStageBytes);  // the leader never armed this fill
      }
      int dummy = 0;
      for (int j = max(0, hi - kStages); j < hi; ++j)
        mbar_wait(&ctl.full[j % kStages], static_cast<uint32_t>((j / kStages) & 1), &dummy, a.status,
                  budget);
    }
  }
  cluster_sync_all();  // every copy into either CTA has landed
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, kTmemCols);
}

// Pairs that can be resident at once (cached per device and kernel).
template <auto Kernel>
int resident_pairs(const cudaLaunchConfig_t& cfg, int num_sms) {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return num_sms / 2;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, Kernel, &cfg) != cudaSuccess || n <= 0) {
      (void)cudaGetLastError();
      n = num_sms / 2;
    }
    cache[dev] = n < num_sms / 2 ? n : num_sms / 2;
  }
  return cache[dev];
}

template <bool kFp8, int kGemm, bool kQuant = false>
cudaError_t launch_pair(const GemmArgs& a, int num_sms, cudaStream_t s) {
  constexpr auto kernel = gemm_pair_kernel<kFp8, kGemm, kQuant>;
  cudaError_t err = set_max_dynamic_smem<gemm_pair_kernel<kFp8, kGemm, kQuant>>(static_cast<int>(kDynSmem));
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg{};
  cfg.blockDim = dim3(kQuant ? kQuantThreads : kThreads);
  cfg.dynamicSmemBytes = kDynSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3(2);
  const int pairs = resident_pairs<gemm_pair_kernel<kFp8, kGemm, kQuant>>(cfg, num_sms);
  cfg.gridDim = dim3(2 * pairs);
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  err = cudaLaunchKernelEx(&cfg, kernel, a);
  return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_pair(const GemmArgs& a, bool fp8, int gemm, int num_sms, cudaStream_t s) {
  if (fp8 && gemm == 2 && a.fuse_quant) return launch_pair<true, 2, true>(a, num_sms, s);
  if (fp8) return gemm == 1 ? launch_pair<true, 1>(a, num_sms, s) : launch_pair<true, 2>(a, num_sms, s);
  return gemm == 1 ? launch_pair<false, 1>(a, num_sms, s) : launch_pair<false, 2>(a, num_sms, s);
}

}  // namespace fmoe
