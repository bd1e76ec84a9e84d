// Shared device helpers and workspace layout for the fused MoE library (sm_100a).
//
// Inline-PTX wrappers for mbarriers, TMA tensor loads and the 5th-generation tensor
// core instructions (tcgen05: TMEM allocation, MMA with shared-memory descriptors,
// commit, TMEM loads).  Every wait on an mbarrier is bounded by a %globaltimer budget;
// on expiry the waiting thread records FMOE_ERR_TIMEOUT in the workspace status word,
// raises the CTA's abort flag and returns false, so that no kernel can spin forever.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace fmoe {

// Device status codes (same numbers as fmoe_status in include/fused_moe.h).
enum : int32_t { ST_OK = 0, ST_TIMEOUT = 5, ST_BOUNDS = 6 };

constexpr int kMaxExperts = 256;                          // routed experts
constexpr int kMaxShared = 8;                             // shared experts
constexpr int kMaxAllExperts = kMaxExperts + kMaxShared;  // rows of the expert tensors
constexpr int kExpertsPerLane = (kMaxAllExperts + 31) / 32;  // one warp covers them all
constexpr int kE4M3Max = 448;
constexpr int kAmaxSlots = 4096;  // capacity of the per-CTA max |h| partials

// Header at the start of the workspace.  Written by device kernels, read by later
// kernels of the same call (stream order) and by the host through the status API.
struct alignas(256) WsHeader {
  int32_t status;        // first device-side error, sticky until cleared
  int32_t n_chunks;      // expert row chunks scheduled for the grouped GEMMs
  int32_t split1;        // split-K factor of the first contraction (swap-AB only)
  int32_t split2;        // split-K factor of the second contraction (swap-AB only)
  int32_t amax_h_count;  // number of valid entries in amax_h_part
  int32_t router_ctas;   // number of valid entries in amax_x_part
  int32_t route_done;    // router tiles finished (fused permutation); zero between calls
  int32_t pad0[9];
  float amax_x, s1, inv1;  // activation amax and the scale / inverse scale used for Aq
  float amax_h, s2, inv2;  // intermediate amax and the scale / inverse scale used for hq
  float pad1[10];
};

// One chunk of consecutive permuted rows that belong to a single expert.
struct alignas(32) Chunk {
  int32_t e;      // expert
  int32_t row0;   // first permuted row
  int32_t nrows;  // rows in this chunk (<= chunk_rows)
  int32_t cb;     // index of the first chunk of this expert
  int32_t nch;    // number of chunks of this expert
  int32_t pad[3];
};

// ------------------------------------------------------------------------------------
// small utilities
// ------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void record_status(int32_t* status, int32_t code) {
  atomicCAS(status, 0, code);
}

__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }

__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "elect.sync _|p, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(pred));
  return pred != 0;
}

// ------------------------------------------------------------------------------------
// programmatic dependent launch
//
// Every kernel of the library is launched with programmatic stream serialisation, so
// it may start while its predecessor in the stream is still running.  Each kernel
// calls griddep_wait() before its first global-memory access that depends on earlier
// work in the stream, and calls griddep_launch_dependents() only after that wait.
// Hence when a kernel starts, the kernel two places before it has completed.
// ------------------------------------------------------------------------------------
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------------------------------
// mbarrier
// ------------------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait until the phase with the given parity of `bar` has completed.  Gives up when
// the CTA's abort flag is raised or when `budget_ns` has passed; in the latter case
// it records ST_TIMEOUT and raises the abort flag.  Returns true on completion.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          int32_t* status, uint64_t budget_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > budget_ns) {
      *abort_flag = 1;
      record_status(status, ST_TIMEOUT);
      return false;
    }
  }
}

// ------------------------------------------------------------------------------------
// TMA (bulk tensor copies global -> shared, completion counted on an mbarrier)
// ------------------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Tiled 2-D load of the box at element coordinates (x = inner / K, y = row).
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x,
                                            int y, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// ------------------------------------------------------------------------------------
// tcgen05: tensor memory and MMA
// ------------------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Arrive once on `bar` when every tcgen05 operation issued so far by this thread is done.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, one instruction (M=128, N per idesc,
// K = 32 bytes of each operand row).
template <bool kFp8>
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
  if constexpr (kFp8) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
  }
}

// 32 lanes x 32 bits, 16 consecutive columns per thread (thread i <- TMEM lane base+i).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor for a K-major operand tile stored as rows of 128
// bytes with the 128-byte swizzle (the layout a TMA load with SWIZZLE_128B writes):
// start address, leading byte offset 16 (unused for this layout), stride byte offset
// 1024 (distance between groups of 8 rows), descriptor version 1, layout SWIZZLE_128B.
// The tile base must be 1024-byte aligned; successive K steps of 32 bytes advance the
// start address field by 2.
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(1u) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

// Instruction descriptor: fp32 accumulator, A and B K-major, e4m3 (kind::f8f6f4) or
// bf16 (kind::f16) inputs, shape M x N.
__host__ __device__ constexpr uint32_t make_idesc(bool fp8, int M, int N) {
  return (1u << 4) | ((fp8 ? 0u : 1u) << 7) | ((fp8 ? 0u : 1u) << 10) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// SiLU(g) = g / (1 + e^-g) with the hardware exponential and fast division.  Every kernel
// that applies the activation uses this one function, so the GEMM variants stay bit-identical
// to each other; against the oracle's fp64 SiLU the difference is a few fp32 ulps, far inside
// the layer tolerances.  (The correctly rounded expf and IEEE division made the first
// contraction's epilogue the limit of the prefill GEMM: 837 us vs 743-765 us at T=4096.)
// For g below about -88, e^-g overflows to infinity and the quotient is 0, the limit.
__device__ __forceinline__ float silu_f(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

}  // namespace fmoe
