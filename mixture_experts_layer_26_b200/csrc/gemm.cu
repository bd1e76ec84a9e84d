// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// Both contractions of the expert MLP run here, for every expert the router selected,
// as one persistent launch each:
//   first:  [g | u] = A_e . W13_e^T            (K = H, 2I output features)
//   second: Y       = hq_e . W2_e^T            (K = I, H output features)
// with e4m3 operands (tcgen05.mma kind::f8f6f4) or bf16 operands (kind::f16) and fp32
// accumulation in tensor memory.
//
// Swap-AB.  On Hopper the warpgroup MMA fixes the row dimension M of the A operand at
// 64, so a decode step with a handful of tokens per expert leaves most of the tensor
// core idle; moving the large expert dimension into the A slot fills it (readmex.ai
// story "AWS details fused MoE kernel optimizations on SageMaker", section "Swap-AB for
// WGMMA utilization"; codebridge-ai.com blog, "1. Matrix swap: lie down for WGMMA").
// tcgen05.mma has the same asymmetry (M is 64 or 128 per CTA, N is any multiple of 16
// up to 256), so the decode variant keeps it: A = 128 weight rows, B = the expert's
// token rows (N = rows rounded up to 16), and the weights stream through TMA as the A
// operand.  Decode is bound by that weight stream, so the variant also splits K when
// there are too few output tiles to fill every SM (device-chosen split factor) and
// writes fp32 partials that a small element-wise kernel finishes.
// The normal variant (prefill: many tokens per expert) puts 128 token rows in M and
// 256 weight rows in N; the first contraction loads 128 gate rows and the matching 128
// up rows into one B tile, so the epilogue applies the scales and SiLU(g)*u directly
// from TMEM ("scaling, matrix multiplication and expert aggregation in one pass":
// agentic-affairs.com, "Triton improves the FP8 execution path").
//
// Kernel structure (one CTA per SM, 192 threads):
//   warp 0    TMA producer: one elected thread fills a ring of shared-memory stages
//   warp 1    MMA issuer: allocates 512 TMEM columns, one elected thread issues 4 MMAs
//             per stage and commits stage release / accumulator-ready to mbarriers
//   warps 2-5 epilogue: tcgen05.ld of the accumulator (warp w reads TMEM lanes
//             32*(w%4)..+31), scale / activation, stores to global memory
// Two accumulator buffers of 256 columns let the epilogue of one tile overlap the MMAs
// of the next.  Work units are read from a device-side chunk list written by the plan
// kernel, so no host synchronisation sits between routing and the expert GEMMs.
// Every mbarrier wait is bounded; on expiry the kernel records a timeout, waits
// (bounded) for its own TMA copies and MMAs, frees its TMEM and returns.
#include <cuda_bf16.h>

#include "fmoe_kernels.h"

namespace fmoe {

namespace {

constexpr int kThreads = 192;
constexpr int kMaxStages = 12;
constexpr int kTileA = 128 * 128;       // bytes of a 128-row x 128-byte operand tile
constexpr int kSwapBoxRows = 16;        // token rows per TMA box in the swap-AB variant
// Accumulator buffers in the 512 TMEM columns: the normal variant's 256-column tiles
// take two; the swap-AB variant's tiles are at most 64 columns (chunk_rows <= 64), so it
// keeps eight, letting the epilogue (stores, split-K hand-off) lag up to seven tiles; its
// wide form (chunk_rows <= 128, for batches whose heavy experts would otherwise stream the
// same weight tiles once per 64-row chunk) keeps four of 128 columns.
constexpr int kMaxAccStages = 8;
template <bool kSwap, bool kWide = false> struct AccLayout {
  static constexpr int kStages = kSwap ? (kWide ? 4 : 8) : 2;
  static constexpr int kCols = kSwap ? (kWide ? 128 : 64) : 256;
};
constexpr int kTmemCols = 512;
constexpr int kSmemBudget = 220 * 1024;

struct SmemCtl {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  uint64_t tmem_full[kMaxAccStages];
  uint64_t tmem_empty[kMaxAccStages];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int amax_bits;
  int n_chunks;
  int split;
};

struct Unit {
  int e, c, row0, nrows, tile, s, kb0, kb1;
};

// Unit u -> (expert, chunk rows, output tile, split, K-block range).  The units of
// expert e occupy [cb_e * per_chunk, (cb_e + nch_e) * per_chunk); inside an expert
// the split index varies fastest, then the chunk, then the output tile, so that
// concurrently running CTAs share weight tiles through L2 when an expert has several
// chunks.
__device__ __forceinline__ Unit decode_unit(long u, const Chunk* chunks, int per_chunk, int S,
                                            int KB) {
  const int q = static_cast<int>(u / per_chunk);
  const Chunk cq = chunks[q];
  const long local = u - static_cast<long>(cq.cb) * per_chunk;
  Unit t;
  t.s = static_cast<int>(local % S);
  const long l2 = local / S;
  const int c = cq.cb + static_cast<int>(l2 % cq.nch);
  t.tile = static_cast<int>(l2 / cq.nch);
  const Chunk cc = chunks[c];
  t.c = c;
  t.e = cc.e;
  t.row0 = cc.row0;
  t.nrows = cc.nrows;
  t.kb0 = t.s * KB / S;
  t.kb1 = (t.s + 1) * KB / S;
  return t;
}

template <bool kFp8, bool kSwap, int kGemm, bool kWide>
__global__ void __launch_bounds__(kThreads, 1) gemm_kernel(const __grid_constant__ GemmArgs a) {
  using Acc = AccLayout<kSwap, kWide>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ SmemCtl ctl;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  const int stage_bytes = kTileA + (kSwap ? a.chunk_rows * 128 : 2 * kTileA);
  const int nst = a.nstages;
  constexpr int kBK = kFp8 ? 128 : 64;  // K elements per stage (128 bytes per row)
  const int KB = a.K / kBK;

  // Set-up that reads nothing produced earlier in the stream: barriers, TMEM, descriptors.
  if (threadIdx.x == 0) {
    for (int s = 0; s < nst; ++s) {
      mbar_init(&ctl.full[s], 1);
      mbar_init(&ctl.empty[s], 1);
    }
    for (int i = 0; i < Acc::kStages; ++i) {
      mbar_init(&ctl.tmem_full[i], 1);
      mbar_init(&ctl.tmem_empty[i], 4);
    }
    mbar_init(&ctl.drain, 1);
    ctl.abort_flag = 0;
    ctl.amax_bits = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&a.map_w);
    tma_prefetch_desc(&a.map_x);
  }
  if (warp == 1) {
    tmem_alloc(&ctl.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  // When the work list was written by the kernel right before this one it waits here.
  // When it was written at least two kernels earlier (a.prefetch_w: always for the second
  // contraction, and for the first one when the gather runs as its own launch), that
  // kernel has completed by the time this grid starts (every kernel triggers its
  // dependents only after its own wait), so the weight tiles are prefetched before
  // waiting for the activations.
  const bool prefetch = a.prefetch_w != 0;
  if (!prefetch) griddep_wait();
  if (threadIdx.x == 0) {
    ctl.n_chunks = a.hdr->n_chunks;
    ctl.split = kSwap ? (kGemm == 1 ? a.hdr->split1 : a.hdr->split2) : 1;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (!prefetch) {
    if (threadIdx.x == 0) griddep_launch_dependents();
  }

  const uint32_t tmem_base = ctl.tmem_base;
  const int S = ctl.split > 0 ? ctl.split : 1;
  const int tiles = kSwap ? a.Nout / 128 : (kGemm == 1 ? a.I / 128 : a.H / 256);
  const int per_chunk = tiles * S;
  const long total = static_cast<long>(ctl.n_chunks) * per_chunk;
  volatile int* abort_flag = &ctl.abort_flag;
  const uint64_t budget = a.wait_budget_ns;

  if (warp == 0) {
    // ------------------------------------------------------------- TMA producer
    if (elect_one()) {
      const uint64_t pol_w = policy_evict_first();  // weights: streamed once
      const uint64_t pol_x = policy_evict_last();   // activations: re-read by every tile
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_parity = 0;
      bool ok = true;

      struct Cursor {
        long u;
        int kb;
        bool have;
        Unit t;
      };
      auto cursor_start = [&](Cursor& c) {
        c.u = blockIdx.x;
        c.have = c.u < total;
        if (c.have) {
          c.t = decode_unit(c.u, a.chunks, per_chunk, S, KB);
          c.kb = c.t.kb0;
        }
      };
      auto cursor_next = [&](Cursor& c) {
        if (++c.kb >= c.t.kb1) {
          c.u += gridDim.x;
          c.have = c.u < total;
          if (c.have) {
            c.t = decode_unit(c.u, a.chunks, per_chunk, S, KB);
            c.kb = c.t.kb0;
          }
        }
      };
      auto nbox_of = [&](const Unit& t) { return kSwap ? (t.nrows + kSwapBoxRows - 1) / kSwapBoxRows : 1; };
      auto tx_bytes = [&](const Unit& t) -> uint32_t {
        return kSwap ? kTileA + nbox_of(t) * kSwapBoxRows * 128 : 3 * kTileA;
      };
      // weight tile(s) of one stage
      auto load_w = [&](int st, const Unit& t, int kb) {
        uint8_t* sa = smem + st * stage_bytes;
        const int kx = kb * kBK;
        if (kSwap && kGemm == 1) {
          // 128 rows as four 32-row quarters: quarter q = 16 gate rows of features
          // tile*64 + 16q .. +15, then the 16 matching up rows, so one warp's TMEM lanes
          // hold both halves of its features
          const int row = t.e * a.rows_per_expert + t.tile * 64;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            tma_load_2d(sa + (32 * q) * 128, &a.map_w, &ctl.full[st], kx, row + 16 * q, pol_w);
            tma_load_2d(sa + (32 * q + 16) * 128, &a.map_w, &ctl.full[st], kx, row + a.I + 16 * q,
                        pol_w);
          }
        } else if (kSwap) {
          tma_load_2d(sa, &a.map_w, &ctl.full[st], kx, t.e * a.rows_per_expert + t.tile * 128, pol_w);
        } else {
          uint8_t* sb = sa + kTileA;
          const int wrow = t.e * a.rows_per_expert + (kGemm == 1 ? t.tile * 128 : t.tile * 256);
          tma_load_2d(sb, &a.map_w, &ctl.full[st], kx, wrow, pol_w);
          tma_load_2d(sb + kTileA, &a.map_w, &ctl.full[st], kx, kGemm == 1 ? wrow + a.I : wrow + 128,
                      pol_w);
        }
      };
      // activation tile(s) of one stage
      auto load_x = [&](int st, const Unit& t, int kb) {
        uint8_t* sa = smem + st * stage_bytes;
        const int kx = kb * kBK;
        if (kSwap) {
          uint8_t* sb = sa + kTileA;
          for (int b = 0; b < nbox_of(t); ++b)
            tma_load_2d(sb + b * kSwapBoxRows * 128, &a.map_x, &ctl.full[st], kx,
                        t.row0 + b * kSwapBoxRows, pol_x);
        } else {
          tma_load_2d(sa, &a.map_x, &ctl.full[st], kx, t.row0, pol_x);
        }
      };
      auto bump = [&]() {
        issued_mask |= 1u << stage;
        issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == nst) {
          stage = 0;
          phase ^= 1u;
        }
      };

      Cursor cur;
      cursor_start(cur);
      if (prefetch) {
        // weights of the first stages (fresh stages: nothing to wait for)
        Cursor first = cur;
        int npre = 0;
        while (cur.have && npre < nst) {
          mbar_arrive_expect_tx(&ctl.full[stage], tx_bytes(cur.t));
          load_w(stage, cur.t, cur.kb);
          bump();
          ++npre;
          cursor_next(cur);
        }
        griddep_wait();
        griddep_launch_dependents();
        for (int i = 0; i < npre; ++i) {  // their activations, now that they are written
          load_x(i, first.t, first.kb);
          cursor_next(first);
        }
      }
      while (cur.have) {
        if (!mbar_wait(&ctl.empty[stage], phase ^ 1u, abort_flag, a.status, budget)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&ctl.full[stage], tx_bytes(cur.t));
        load_w(stage, cur.t, cur.kb);
        load_x(stage, cur.t, cur.kb);
        bump();
        cursor_next(cur);
      }
      if (!ok) {
        // aborted: let every copy this thread issued land before the CTA exits
        for (int s = 0; s < nst; ++s)
          if (issued_mask & (1u << s)) {
            int dummy = 0;
            mbar_wait(&ctl.full[s], (issued_parity >> s) & 1u, &dummy, a.status, budget);
          }
      }
    } else if (prefetch) {
      // lanes that do not produce still order their later reads after the wait
      griddep_wait();
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (elect_one()) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (long u = blockIdx.x; u < total && ok; u += gridDim.x) {
        const Unit t = decode_unit(u, a.chunks, per_chunk, S, KB);
        const int n_mma = kSwap ? ((t.nrows + 15) / 16) * 16 : 256;
        const uint32_t idesc = make_idesc(kFp8, 128, n_mma);
        if (!mbar_wait(&ctl.tmem_empty[acc], acc_phase ^ 1u, abort_flag, a.status, budget)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(acc * Acc::kCols);
        for (int kb = t.kb0; kb < t.kb1; ++kb) {
          if (!mbar_wait(&ctl.full[stage], phase, abort_flag, a.status, budget)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * stage_bytes);
          const uint64_t ad = sw128_kmajor_desc(sa);
          const uint64_t bd = sw128_kmajor_desc(sa + kTileA);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc_mma<kFp8>(d, ad + 2u * k, bd + 2u * k, idesc, (kb > t.kb0 || k > 0) ? 1u : 0u);
          tc_commit(&ctl.empty[stage]);
          if (++stage == nst) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(&ctl.tmem_full[acc]);
        if (++acc == Acc::kStages) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (!ok) {
        // aborted: wait for the MMAs already issued before TMEM is released
        tc_commit(&ctl.drain);
        int dummy = 0;
        mbar_wait(&ctl.drain, 0, &dummy, a.status, budget);
      }
    }
  } else {
    // ------------------------------------------------------------- epilogue
    if (prefetch) griddep_wait();  // scales and routing weights of this call
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int r = q * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    float amax = 0.f;
    for (long u = blockIdx.x; u < total; u += gridDim.x) {
      const Unit t = decode_unit(u, a.chunks, per_chunk, S, KB);
      const bool ready = mbar_wait(&ctl.tmem_full[acc], acc_phase, abort_flag, a.status, budget);
      __syncwarp();
      if (!__all_sync(0xffffffffu, ready)) break;
      tc_fence_after();
      const uint32_t tb =
          tmem_base + static_cast<uint32_t>(acc * Acc::kCols) + (static_cast<uint32_t>(q * 32) << 16);
      if constexpr (kSwap && kGemm == 1) {
        // lane r of quarter q: gate (r%32 < 16) or up (r%32 >= 16) of feature
        // tile*64 + 16q + r%16; column c = token row0 + c
        const int ncols = ((t.nrows + 15) / 16) * 16;
        const int f = t.tile * 64 + q * 16 + (lane & 15);
        if (S == 1) {
          // whole K in this tile: apply the scale and SiLU(g)*u here
          const float sc = kFp8 ? a.hdr->s1 * a.w_scale[t.e] : 1.f;
          for (int c0 = 0; c0 < ncols; c0 += 16) {
            float v[16];
            tmem_ld16(tb + c0, v);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float up = __shfl_xor_sync(0xffffffffu, v[i], 16);
              if (lane < 16 && c0 + i < t.nrows) {
                const float h = silu_f(v[i] * sc) * (up * sc);
                const size_t o = static_cast<size_t>(t.row0 + c0 + i) * a.I + f;
                if constexpr (kFp8) {
                  a.h_out[o] = h;
                  amax = fmaxf(amax, fabsf(h));
                } else {
                  a.out_bf16[o] = __bfloat16_as_ushort(__float2bfloat16_rn(h));
                }
              }
            }
          }
        } else {
          // split-K: write this split's fp32 partial; finalize1 sums the splits in order
          const int feat = (lane & 16) ? a.I + f : f;
          const size_t plane = static_cast<size_t>(a.R) * a.Nout;
          float* dst = a.out + static_cast<size_t>(t.s) * plane + static_cast<size_t>(t.row0) * a.Nout + feat;
          for (int c0 = 0; c0 < ncols; c0 += 16) {
            float v[16];
            tmem_ld16(tb + c0, v);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i)
              if (c0 + i < t.nrows) dst[static_cast<size_t>(c0 + i) * a.Nout] = v[i];
          }
        }
      } else if constexpr (kSwap) {
        // lane r = output feature tile*128 + r, column c = token row0 + c
        const int ncols = ((t.nrows + 15) / 16) * 16;
        float* dst = a.out + (static_cast<size_t>(t.s) * a.R + t.row0) * a.Nout + t.tile * 128 + r;
        for (int c0 = 0; c0 < ncols; c0 += 16) {
          float v[16];
          tmem_ld16(tb + c0, v);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (c0 + i < t.nrows) dst[static_cast<size_t>(c0 + i) * a.Nout] = v[i];
        }
      } else if constexpr (kGemm == 1) {
        // lane r = token row0 + r; columns 0..127 gate, 128..255 up of features tile*128..
        const bool valid = r < t.nrows;
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
              // fp32 h for the per-tensor re-quantisation (quant_h); storing it rounded
              // to bf16 would double-round a few percent of the e4m3 codes
              float4* dst = reinterpret_cast<float4*>(a.out + o + c0);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                dst[i] = make_float4(h[4 * i], h[4 * i + 1], h[4 * i + 2], h[4 * i + 3]);
                amax = fmaxf(amax, fmaxf(fmaxf(fabsf(h[4 * i]), fabsf(h[4 * i + 1])),
                                         fmaxf(fabsf(h[4 * i + 2]), fabsf(h[4 * i + 3]))));
              }
            } else {
              // bf16 format: h rounded to bf16 is the second contraction's input
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
        // lane r = token row0 + r; columns = output features tile*256 ..
        const bool valid = r < t.nrows;
        const float sc = kFp8 ? a.hdr->s2 * a.w_scale[t.e] : 1.f;
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
      if (lane == 0) mbar_arrive(&ctl.tmem_empty[acc]);
      if (++acc == Acc::kStages) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if constexpr (kGemm == 1 && kFp8) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
      if (lane == 0) atomicMax(&ctl.amax_bits, __float_as_int(amax));
    }
  }

  __syncthreads();
  // per-CTA max |h| when this kernel produced h (normal variant, or swap-AB unsplit)
  if constexpr (kGemm == 1 && kFp8) {
    if (threadIdx.x == 0 && (!kSwap || S == 1)) {
      a.amax_part[blockIdx.x] = __int_as_float(ctl.amax_bits);
      if (blockIdx.x == 0) a.hdr_w->amax_h_count = gridDim.x;
    }
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

template <bool kFp8, bool kSwap, int kGemm, bool kWide = false>
cudaError_t launch_one(const GemmArgs& a, int num_sms, cudaStream_t s) {
  if (kSwap && !kWide && a.chunk_rows > 64) return launch_one<kFp8, kSwap, kGemm, true>(a, num_sms, s);
  if (a.chunk_rows > AccLayout<kSwap, kWide>::kCols) return cudaErrorInvalidValue;
  const int stage_bytes = kTileA + (kSwap ? a.chunk_rows * 128 : 2 * kTileA);
  const size_t smem = 1024 + static_cast<size_t>(a.nstages) * stage_bytes;
  cudaError_t err = set_max_dynamic_smem<gemm_kernel<kFp8, kSwap, kGemm, kWide>>(kSmemBudget + 1024);
  if (err != cudaSuccess) return err;
  return launch_k(gemm_kernel<kFp8, kSwap, kGemm, kWide>, dim3(num_sms), dim3(kThreads), smem, s, a);
}

}  // namespace

int gemm_stages(bool swap_ab, int chunk_rows) {
  const int stage_bytes = kTileA + (swap_ab ? chunk_rows * 128 : 2 * kTileA);
  int n = kSmemBudget / stage_bytes;
  if (n > kMaxStages) n = kMaxStages;
  return n;
}

cudaError_t launch_gemm(const GemmArgs& a, bool fp8, bool swap_ab, int gemm, int num_sms,
                        cudaStream_t s) {
  if (fp8) {
    if (swap_ab) return gemm == 1 ? launch_one<true, true, 1>(a, num_sms, s)
                                  : launch_one<true, true, 2>(a, num_sms, s);
    return gemm == 1 ? launch_one<true, false, 1>(a, num_sms, s)
                     : launch_one<true, false, 2>(a, num_sms, s);
  }
  if (swap_ab) return gemm == 1 ? launch_one<false, true, 1>(a, num_sms, s)
                                : launch_one<false, true, 2>(a, num_sms, s);
  return gemm == 1 ? launch_one<false, false, 1>(a, num_sms, s)
                   : launch_one<false, false, 2>(a, num_sms, s);
}

}  // namespace fmoe
