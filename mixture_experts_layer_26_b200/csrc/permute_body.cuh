// Device code shared by the permute / gather / plan kernels (permute.cu) and by the
// router's final CTA, which runs them itself on the one-call path for small batches
// (router.cu).  Included by both translation units.
#pragma once

#include <cuda_fp8.h>

#include "fmoe_kernels.h"

namespace fmoe {
namespace {

// Split-K factor for `units` output tiles of `kblocks` K blocks on `sms` persistent
// CTAs: the smallest factor whose last wave is at least 90% full, else the best one.
__device__ int choose_split(int units, int kblocks, int smax, int sms) {
  if (units <= 0) return 1;
  const int cap = max(1, min(smax, kblocks / 2));
  int best = 1;
  float best_eff = -1.f;
  for (int s = 1; s <= cap; ++s) {
    // 32-bit arithmetic (units * 16 stays far below 2^31): a 64-bit division is a long
    // serial call on the one thread that plans
    const int u = units * s;
    const int waves = (u + sms - 1) / sms;
    const float eff = static_cast<float>(u) / static_cast<float>(waves * sms);
    if (eff >= 0.9f) return s;
    if (eff > best_eff + 1e-6f) { best_eff = eff; best = s; }
  }
  return best;
}

// One warp: split every expert's rows [offsets[e], offsets[e+1]) into chunks of at most
// chunk_rows rows, write the chunk list and the split-K factors.  `offsets` may live in
// shared or global memory; malformed offsets are reported and treated as empty.
__device__ void build_plan(const int* offsets, int E, int R, const PlanParams& p, WsHeader* hdr) {
  const int lane = threadIdx.x & 31;
  const int CH = p.chunk_rows;
  int n[kExpertsPerLane], nch[kExpertsPerLane], s = 0;
#pragma unroll
  for (int j = 0; j < kExpertsPerLane; ++j) {
    const int e = lane * kExpertsPerLane + j;
    n[j] = 0;
    if (e < E) {
      const int lo = offsets[e], hi = offsets[e + 1];
      if (lo < 0 || hi < lo || hi > R) record_status(&hdr->status, ST_BOUNDS);
      else n[j] = hi - lo;
    }
    nch[j] = (n[j] + CH - 1) / CH;
    s += nch[j];
  }
  int incl = s;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += t;
  }
  const int total = __shfl_sync(0xffffffffu, incl, 31);
  int cb = incl - s;
#pragma unroll
  for (int j = 0; j < kExpertsPerLane; ++j) {
    const int e = lane * kExpertsPerLane + j;
    for (int c = 0; c < nch[j]; ++c) {
      const int idx = cb + c;
      if (idx >= p.max_chunks) {
        record_status(&hdr->status, ST_BOUNDS);
        break;
      }
      Chunk ch;
      ch.e = e;
      ch.row0 = offsets[e] + c * CH;
      ch.nrows = min(CH, n[j] - c * CH);
      ch.cb = cb;
      ch.nch = nch[j];
      ch.pad[0] = ch.pad[1] = ch.pad[2] = 0;
      p.chunks[idx] = ch;
    }
    cb += nch[j];
  }
  if (p.ready != nullptr)  // counters of the second contraction's in-kernel quantisation
    for (int i = lane; i < p.max_chunks; i += 32) p.ready[i] = 0;
  if (lane == 0) {
    const int nc = min(total, p.max_chunks);
    hdr->n_chunks = nc;
    if (p.swap_ab) {
      hdr->split1 = choose_split(nc * p.units1_per_chunk, p.kblocks1, p.s1max, p.num_sms);
      hdr->split2 = choose_split(nc * p.units2_per_chunk, p.kblocks2, p.s2max, p.num_sms);
    } else {
      hdr->split1 = 1;
      hdr->split2 = 1;
    }
  }
}


__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return lo | (hi << 16);
}

// 8 bf16 (one uint4) times inv -> 8 e4m3 bytes (uint2)
__device__ __forceinline__ uint2 quant8(const uint4& v, float inv) {
  const float f0 = __uint_as_float(v.x << 16) * inv, f1 = __uint_as_float(v.x & 0xFFFF0000u) * inv;
  const float f2 = __uint_as_float(v.y << 16) * inv, f3 = __uint_as_float(v.y & 0xFFFF0000u) * inv;
  const float f4 = __uint_as_float(v.z << 16) * inv, f5 = __uint_as_float(v.z & 0xFFFF0000u) * inv;
  const float f6 = __uint_as_float(v.w << 16) * inv, f7 = __uint_as_float(v.w & 0xFFFF0000u) * inv;
  return make_uint2(e4m3x4(f0, f1, f2, f3), e4m3x4(f4, f5, f6, f7));
}

// Stable grouping in one CTA: warp w owns the contiguous segment of routed rows
// [w*seg, (w+1)*seg).  Pass 1 counts each warp's rows per expert, the counts give the
// offsets and each (expert, warp) start position, and pass 2 walks every segment again
// in ascending order, so rows of one expert keep their flattened order (t*k+j).
// Runs on a whole CTA of kWarps warps.  wc: kWarps*E ints, cnt: E, base: E+1 (shared).
// Reads ids and amax partials through L2 (__ldcg): when fused into the router they were
// written by other CTAs of the same grid.  n_parts > 0: the number of max |x| partials (the
// router's grid, when fused into it) instead of the header's count; inv_s (shared, or null)
// also receives the inverse activation scale, for a gather in the same CTA.
template <int kWarps>
__device__ void permute_body(const PermuteArgs& a, int* wc_flat, int* cnt, int* base,
                             int n_parts = 0, float* inv_s = nullptr) {
  constexpr int kPermThreads = kWarps * 32;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = a.E, R = a.R;
  const int seg = (R + kWarps - 1) / kWarps;
  const int lo = min(R, warp * seg), hi = min(R, lo + seg);

  auto wc = [&](int w, int e) -> int& { return wc_flat[w * E + e]; };
  for (int i = tid; i < kWarps * E; i += kPermThreads) wc_flat[i] = 0;
  __syncthreads();

  // The ids of a warp's segment are read kBatch*32 at a time (kBatch loads in flight
  // per lane), then handled 32 at a time in ascending order.
  constexpr int kBatch = 8;
  auto load_batch = [&](int i0, int (&ev)[kBatch]) {
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int i = i0 + 32 * j + lane;
      int e = i < hi ? __ldcg(a.topk_ids + i) : E;
      if (i < hi && (e < 0 || e >= E)) {
        record_status(&a.hdr->status, ST_BOUNDS);
        e = E + 1;  // invalid: matches only other invalid lanes, never placed
      }
      ev[j] = e;
    }
  };

  // pass 1: rows per (warp, expert); a segment of one batch keeps its ids for pass 2
  const bool one_batch = hi - lo <= 32 * kBatch;
  int ev_kept[kBatch];
  for (int i0 = lo; i0 < hi; i0 += 32 * kBatch) {
    int ev[kBatch];
    load_batch(i0, ev);
    if (one_batch) {
#pragma unroll
      for (int j = 0; j < kBatch; ++j) ev_kept[j] = ev[j];
    }
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      if (i0 + 32 * j >= hi) break;  // warp-uniform
      const int e = ev[j];
      const unsigned peers = __match_any_sync(0xffffffffu, e);
      if (e < E && lane == __ffs(peers) - 1) wc(warp, e) += __popc(peers);
      __syncwarp();
    }
  }
  __syncthreads();
  for (int e = tid; e < E; e += kPermThreads) {
    int c = 0;
    for (int w = 0; w < kWarps; ++w) c += wc(w, e);
    cnt[e] = c;
  }
  __syncthreads();

  // exclusive scan of the counts: lane l owns experts l*kExpertsPerLane ..
  if (warp == 0) {
    int v[kExpertsPerLane], s = 0;
#pragma unroll
    for (int j = 0; j < kExpertsPerLane; ++j) {
      const int e = lane * kExpertsPerLane + j;
      v[j] = e < E ? cnt[e] : 0;
      s += v[j];
    }
    int incl = s;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += t;
    }
    int run = incl - s;
#pragma unroll
    for (int j = 0; j < kExpertsPerLane; ++j) {
      const int e = lane * kExpertsPerLane + j;
      if (e < E) {
        a.counts[e] = v[j];
        a.offsets[e] = run;
        base[e] = run;
      }
      run += v[j];
    }
    if (lane == 31) {
      a.offsets[E] = incl;
      base[E] = incl;
    }
  }
  if (warp == 1) {
    // activation scale from the router's per-tile maxima (one warp, strided)
    float amax = 0.f;
    const int n = n_parts > 0 ? n_parts : __ldcg(&a.hdr->router_ctas);
    for (int i0 = lane; i0 < n; i0 += 32 * 8) {  // eight loads in flight per lane
      float v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = i0 + 32 * j < n ? __ldcg(a.amax_part + i0 + 32 * j) : 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) amax = fmaxf(amax, v[j]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    float s1 = 1.f, inv1 = 1.f;
    if (a.fp8) {
      if (a.a1_static > 0.f) {
        s1 = a.a1_static;
        inv1 = 1.0f / a.a1_static;
      } else if (amax > 0.f) {
        s1 = amax / 448.0f;
        inv1 = 448.0f / amax;
      }
    }
    if (lane == 0) {
      a.hdr->amax_x = amax;
      a.hdr->s1 = s1;
      a.hdr->inv1 = inv1;
      if (inv_s != nullptr) *inv_s = inv1;
    }
  }
  __syncthreads();
  if (a.with_plan && warp == 0) build_plan(base, E, R, a.plan, a.hdr);
  // first position of each (warp, expert)
  for (int e = tid; e < E; e += kPermThreads) {
    int run = base[e];
    for (int w = 0; w < kWarps; ++w) {
      const int v = wc(w, e);
      wc(w, e) = run;
      run += v;
    }
  }
  __syncthreads();

  // pass 2: place every row, in ascending order within each warp's segment
  for (int i0 = lo; i0 < hi; i0 += 32 * kBatch) {
    int ev[kBatch];
    if (one_batch) {
#pragma unroll
      for (int j = 0; j < kBatch; ++j) ev[j] = ev_kept[j];
    } else {
      load_batch(i0, ev);
    }
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      if (i0 + 32 * j >= hi) break;  // warp-uniform
      const int i = i0 + 32 * j + lane;
      const int e = ev[j];
      const unsigned peers = __match_any_sync(0xffffffffu, e);
      const int rank = __popc(peers & ((1u << lane) - 1u));
      if (e < E) {
        const int pos = wc(warp, e) + rank;
        a.sorted_rows[pos] = i;
        a.inv_perm[i] = pos;
      }
      __syncwarp();
      if (e < E && lane == __ffs(peers) - 1) wc(warp, e) += __popc(peers);
      __syncwarp();
    }
  }
}

// The permuted activations A[p] = x[sorted_rows[p] / k], read with 16-byte loads; FP8:
// times 448/amax in fp32, rounded to e4m3 (nearest even, saturating).
// Token-major gather: a warp takes one (token, segment of up to 32*kGatherU 16-byte steps)
// item, reads that part of the token's x row once, quantises it once (FP8), and stores it to
// each of the token's k permuted rows p = inv_perm[t*k + j] (lane j holds slot j's row when
// k <= 32).  Every permuted row gets exactly the bytes a row-major gather would write; x is
// read once instead of k times.
constexpr int kGatherU = 4;  // 16-byte steps per lane and item

__device__ __forceinline__ int gather_items(const GatherArgs& a) {
  const int steps = a.fp8 ? a.H / 16 : a.H / 8;  // FP8: 16 elements; bf16: 8 per step
  return (a.R / a.k) * ((steps + 32 * kGatherU - 1) / (32 * kGatherU));
}

__device__ void gather_rows(const GatherArgs& a, int gwarp, int nwarps, const float* inv_s = nullptr) {
  const int lane = threadIdx.x & 31;
  const float inv = a.fp8 ? (inv_s != nullptr ? *inv_s : a.hdr->inv1) : 1.f;
  const int k = a.k;
  const int steps = a.fp8 ? a.H / 16 : a.H / 8;
  const int nseg = (steps + 32 * kGatherU - 1) / (32 * kGatherU);
  const int items = gather_items(a);
  for (int it = gwarp; it < items; it += nwarps) {
    const int t = it / nseg, s0 = (it % nseg) * 32 * kGatherU;
    auto row_of = [&](int j) {  // permuted row of slot j, -1 if out of range (reported)
      int p = a.inv_perm[static_cast<size_t>(t) * k + j];
      if (p < 0 || p >= a.R) {
        record_status(a.status, ST_BOUNDS);
        p = -1;
      }
      return p;
    };
    const int pl = lane < k ? row_of(lane) : -1;
    const uint4* src = reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(t) * a.H);
    uint4 v[kGatherU];
    if (a.fp8) {
      uint4 x0[kGatherU], x1[kGatherU];
#pragma unroll
      for (int u = 0; u < kGatherU; ++u) {
        const int st = s0 + lane + 32 * u;
        if (st < steps) {
          x0[u] = __ldg(src + 2 * st);
          x1[u] = __ldg(src + 2 * st + 1);
        }
      }
#pragma unroll
      for (int u = 0; u < kGatherU; ++u) {
        if (s0 + lane + 32 * u < steps) {
          const uint2 q0 = quant8(x0[u], inv), q1 = quant8(x1[u], inv);
          v[u] = make_uint4(q0.x, q0.y, q1.x, q1.y);
        }
      }
    } else {
#pragma unroll
      for (int u = 0; u < kGatherU; ++u) {
        const int st = s0 + lane + 32 * u;
        if (st < steps) v[u] = __ldg(src + st);
      }
    }
    const size_t row_bytes = static_cast<size_t>(a.H) * (a.fp8 ? 1 : 2);
    for (int j = 0; j < k; ++j) {
      const int p = j < 32 ? __shfl_sync(0xffffffffu, pl, j) : row_of(j);  // warp-uniform
      if (p < 0) continue;
      uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(a.a_perm) + static_cast<size_t>(p) * row_bytes);
#pragma unroll
      for (int u = 0; u < kGatherU; ++u) {
        const int st = s0 + lane + 32 * u;
        if (st < steps) dst[st] = v[u];
      }
    }
  }
}

}  // namespace
}  // namespace fmoe
