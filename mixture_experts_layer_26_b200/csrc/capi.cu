// Host side of the C ABI declared in include/fused_moe.h: argument checks, workspace
// layout, TMA descriptors and the launch sequence of each step.  Nothing here
// allocates device memory or synchronises, except the calls the header documents as
// synchronous.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "fmoe_kernels.h"
#include "fused_moe.h"

using namespace fmoe;

namespace {

constexpr size_t kAlign = 256;
constexpr size_t kPartialBudget = size_t(64) << 20;  // bytes of split-K partials per GEMM
constexpr int kMaxSplit = 16;
constexpr uint64_t kWaitBudgetNs = 2000000000ull;  // bounded mbarrier waits: 2 s

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct Layout {
  bool fp8 = false, swap = false, pair = false;
  int R = 0, chunk_rows = 0, max_chunks = 0, s1max = 0, s2max = 0;
  size_t hdr = 0, counters = 0, amax_x = 0, amax_h = 0, chunks = 0, logits = 0, ready = 0;
  size_t ids = 0, tw = 0, counts = 0, offsets = 0, rows = 0, inv = 0;
  size_t x_in = 0, out_dev = 0, a_perm = 0, p1 = 0, h = 0, hq = 0, p2 = 0, y = 0;
  size_t total = 0;
};

// Shared experts: S = n_shared; every token has K = top_k + S slots and the expert
// tensors hold E + S experts.
inline int shared_of(const fmoe_dims& d) { return d.routing != nullptr ? d.routing->n_shared : 0; }
inline int slots_of(const fmoe_dims& d) { return d.top_k + shared_of(d); }
inline int experts_all(const fmoe_dims& d) { return d.E + shared_of(d); }

fmoe_status check_dims(const fmoe_dims* d) {
  if (d == nullptr) return FMOE_ERR_INVALID_ARG;
  if (d->T < 0 || d->H < 1 || d->I < 1 || d->E < 1 || d->E > kMaxExperts || d->top_k < 1 ||
      d->top_k > d->E)
    return FMOE_ERR_INVALID_ARG;
  if (d->wdtype != FMOE_BF16 && d->wdtype != FMOE_FP8_E4M3) return FMOE_ERR_INVALID_ARG;
  if (d->variant < FMOE_VARIANT_AUTO || d->variant > FMOE_VARIANT_NORMAL_PAIR)
    return FMOE_ERR_INVALID_ARG;
  if (d->routing != nullptr) {
    const fmoe_routing& r = *d->routing;
    if (r.mode != FMOE_ROUTE_SOFTMAX && r.mode != FMOE_ROUTE_SIGMOID_GROUPED)
      return FMOE_ERR_INVALID_ARG;
    if (r.n_shared < 0 || r.n_shared > kMaxShared) return FMOE_ERR_INVALID_ARG;
    if (r.mode == FMOE_ROUTE_SIGMOID_GROUPED) {
      if (r.n_group < 1 || r.n_group > 32 || d->E % r.n_group != 0 || d->E / r.n_group < 2)
        return FMOE_ERR_INVALID_ARG;
      if (r.topk_group < 1 || r.topk_group > r.n_group ||
          static_cast<int64_t>(r.topk_group) * (d->E / r.n_group) < d->top_k)
        return FMOE_ERR_INVALID_ARG;
      if (!(r.routed_scaling > 0.f) || r.routed_scaling > 1e30f) return FMOE_ERR_INVALID_ARG;
      if (r.bias != nullptr && (reinterpret_cast<uintptr_t>(r.bias) & 3u) != 0)
        return FMOE_ERR_UNSUPPORTED;
    }
  }
  if (d->H % 256 != 0 || d->I % 128 != 0 || d->H > 16384) return FMOE_ERR_UNSUPPORTED;
  const int64_t R = static_cast<int64_t>(d->T) * slots_of(*d);
  const int64_t lim = int64_t(1) << 31;
  if (R * std::max<int64_t>(d->H, 2 * int64_t(d->I)) >= lim) return FMOE_ERR_UNSUPPORTED;
  const int64_t ea = experts_all(*d);
  if (ea * 2 * d->I >= lim || ea * d->H >= lim) return FMOE_ERR_UNSUPPORTED;
  return FMOE_OK;
}

int swap_chunk_cap(const fmoe_dims& d) {
  const bool concentrated =
      d.routing != nullptr && (d.routing->n_shared > 0 || d.routing->mode == FMOE_ROUTE_SIGMOID_GROUPED);
  return concentrated ? 128 : 64;
}

Layout make_layout(const fmoe_dims& d) {
  Layout L;
  L.fp8 = d.wdtype == FMOE_FP8_E4M3;
  const int T = d.T, H = d.H, I = d.I, E = experts_all(d);
  const int R = T * slots_of(d);
  L.R = R;
  int variant = d.variant;
  if (variant == FMOE_VARIANT_AUTO) {
    const int avg = (R + E - 1) / E;
    variant = avg <= 64 ? FMOE_VARIANT_SWAP_AB : avg <= 128 ? FMOE_VARIANT_NORMAL : FMOE_VARIANT_NORMAL_PAIR;
  }
  L.swap = variant == FMOE_VARIANT_SWAP_AB;
  L.pair = variant == FMOE_VARIANT_NORMAL_PAIR;
  // an expert receives at most T rows (one per token).  Swap-AB chunks hold up to 64 rows,
  // or 128 when some experts are known to receive many more than the average: every token
  // uses a shared expert, and grouped routing concentrates the batch on a few groups
  L.chunk_rows = L.swap ? std::min(swap_chunk_cap(d), static_cast<int>(align_up(std::max(T, 1), 16)))
                        : (L.pair ? 256 : 128);
  L.max_chunks = R / L.chunk_rows + std::min(E, R) + 1;
  const size_t es = L.fp8 ? 1 : 2;
  const size_t p1_plane = static_cast<size_t>(R) * 2 * I * 4;
  const size_t p2_plane = static_cast<size_t>(R) * H * 4;
  if (L.swap) {
    L.s1max = static_cast<int>(std::clamp<size_t>(kPartialBudget / std::max<size_t>(p1_plane, 1), 1, kMaxSplit));
    L.s2max = static_cast<int>(std::clamp<size_t>(kPartialBudget / std::max<size_t>(p2_plane, 1), 1, kMaxSplit));
  }
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, kAlign);
    return o;
  };
  L.hdr = take(sizeof(WsHeader));
  L.counters = take(static_cast<size_t>(kRouterMaxTiles) * 4);  // zeroed with the header
  L.amax_x = take(static_cast<size_t>(std::max(T, 1)) * 4);
  L.logits = take(static_cast<size_t>(T) * E * 4);
  L.amax_h = take(static_cast<size_t>(kAmaxSlots) * 4);
  L.chunks = take(static_cast<size_t>(L.max_chunks) * sizeof(Chunk));
  L.ready = take(static_cast<size_t>(L.max_chunks) * 4);
  L.ids = take(static_cast<size_t>(R) * 4);
  L.tw = take(static_cast<size_t>(R) * 4);
  L.counts = take(static_cast<size_t>(E) * 4);
  L.offsets = take(static_cast<size_t>(E + 1) * 4);
  L.rows = take(static_cast<size_t>(R) * 4);
  L.inv = take(static_cast<size_t>(R) * 4);
  L.x_in = take(static_cast<size_t>(T) * H * 2);
  L.out_dev = take(static_cast<size_t>(T) * H * 2);
  L.a_perm = take(static_cast<size_t>(R) * H * es);
  L.p1 = take(L.swap ? L.s1max * p1_plane : 0);
  L.h = take(L.fp8 ? static_cast<size_t>(R) * I * 4 : 0);
  L.hq = take(static_cast<size_t>(R) * I * es);
  L.p2 = take(L.swap ? L.s2max * p2_plane : 0);
  L.y = take(static_cast<size_t>(R) * H * 4);
  L.total = off;
  return L;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

fmoe_status check_ws(const Layout& L, const void* ws, size_t ws_bytes) {
  if (ws == nullptr) return FMOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ws) & (kAlign - 1)) != 0) return FMOE_ERR_WORKSPACE;
  if (ws_bytes < L.total) return FMOE_ERR_WORKSPACE;
  return FMOE_OK;
}

// Every pointer non-null and 16-byte aligned.
template <typename... P>
fmoe_status check_ptrs(P... ptrs) {
  const void* list[] = {static_cast<const void*>(ptrs)...};
  for (const void* p : list) {
    if (p == nullptr) return FMOE_ERR_INVALID_ARG;
    if (!aligned16(p)) return FMOE_ERR_UNSUPPORTED;
  }
  return FMOE_OK;
}

fmoe_status check_fp8_scales(const fmoe_dims& d, const fmoe_scales* sc) {
  if (d.wdtype != FMOE_FP8_E4M3) return FMOE_OK;
  if (sc == nullptr || sc->w13_scale == nullptr || sc->w2_scale == nullptr)
    return FMOE_ERR_INVALID_ARG;
  return FMOE_OK;
}

int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

PFN_cuTensorMapEncodeTiled_v12000 tma_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D K-major operand [rows, inner] with 128-byte rows per box and the 128-byte swizzle.
bool encode_map(CUtensorMap* m, const void* base, bool fp8, uint64_t inner, uint64_t rows,
                uint32_t box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = tma_encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {inner * (fp8 ? 1 : 2)};
  const cuuint32_t box[2] = {fp8 ? 128u : 64u, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r =
      fn(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
         const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D bf16 rows [rows, inner] without swizzle, boxes of 256 columns x box_rows rows (the
// tiled router's x and router_w slices); rows past the end read as zeros.
bool encode_rows_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                     uint32_t box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = tma_encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {inner * 2};
  const cuuint32_t box[2] = {256u, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

inline fmoe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? FMOE_OK : FMOE_ERR_CUDA; }

#define FMOE_TRY(expr)                   \
  do {                                   \
    const fmoe_status _s = (expr);       \
    if (_s != FMOE_OK) return _s;        \
  } while (0)

}  // namespace

namespace fmoe {
bool pdl_enabled() {
  static const bool on = [] {
    const char* v = std::getenv("FMOE_DISABLE_PDL");
    return !(v != nullptr && v[0] == '1');
  }();
  return on;
}
}  // namespace fmoe

namespace {

// Measurement hook: when active (fused_moe_profile only), every kernel launch of the
// call sequence is followed by an event record on the launching stream.
struct StageRecorder {
  static constexpr int kCap = 32;
  bool active = false;
  int n = 0;
  cudaEvent_t ev[kCap + 1] = {};
  const char* names[kCap] = {};
};
thread_local StageRecorder g_rec;

inline cudaError_t mark(const char* name, cudaStream_t s) {
  if (!g_rec.active) return cudaSuccess;
  if (g_rec.n >= StageRecorder::kCap) return cudaSuccess;
  g_rec.names[g_rec.n] = name;
  return cudaEventRecord(g_rec.ev[++g_rec.n], s);
}

// launch `expr` (a launcher returning cudaError_t), then mark it
#define FMOE_LAUNCH(name, expr, stream)                      \
  do {                                                       \
    FMOE_TRY(cuda_status(expr));                             \
    FMOE_TRY(cuda_status(mark(name, stream)));               \
  } while (0)

// NVTX range over the host-side enqueue of one step (route, permute, experts, combine), so
// that a timeline profiler shows which launches belong to which stage.  NVTX is header-only
// and costs a few tens of nanoseconds when no tool is attached.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};


// ------------------------------------------------------------------ step bodies

PlanParams plan_params(const fmoe_dims& d, const Layout& L, char* W) {
  const int bk = L.fp8 ? 128 : 64;
  PlanParams p{};
  p.chunks = reinterpret_cast<Chunk*>(W + L.chunks);
  p.chunk_rows = L.chunk_rows;
  p.max_chunks = L.max_chunks;
  p.swap_ab = L.swap ? 1 : 0;
  p.units1_per_chunk = L.swap ? 2 * d.I / 128 : d.I / 128;
  p.units2_per_chunk = L.swap ? d.H / 128 : d.H / 256;
  p.kblocks1 = d.H / bk;
  p.kblocks2 = d.I / bk;
  p.s1max = std::max(L.s1max, 1);
  p.s2max = std::max(L.s2max, 1);
  p.num_sms = num_sms();
  p.ready = reinterpret_cast<int32_t*>(W + L.ready);
  return p;
}

// The CTA-pair FP8 second contraction quantises h itself (no quant_h launch) unless the
// max |h| comes from outside the call (a tensor-parallel shard).
bool fuse_quant_h(const Layout& L, const float* amax_in) { return L.pair && L.fp8 && amax_in == nullptr; }

// Small batches whose routed rows fit one CTA's permutation: the router's final CTA
// also runs permute (+ plan) and, when the gathered rows are at most 128 KB, the gather.
bool fuse_route_permute(const Layout& L) { return L.R <= 2048; }
bool fuse_route_gather(const fmoe_dims& d, const Layout& L) {
  return fuse_route_permute(L) && static_cast<size_t>(L.R) * d.H * 2 <= (size_t(128) << 10);
}

PermuteArgs permute_args(const fmoe_dims& d, const Layout& L, const int32_t* ids,
                         const fmoe_scales* sc, int32_t* counts, int32_t* offsets, int32_t* rows,
                         int32_t* inv, char* W, bool with_plan);
GatherArgs gather_args(const fmoe_dims& d, const Layout& L, const void* x, const int32_t* rows,
                       const int32_t* inv, void* a_perm, char* W);

fmoe_status route_impl(const fmoe_dims& d, const Layout& L, const void* x, const void* rw,
                       int32_t* ids, float* tw, char* W, cudaStream_t s,
                       const PermuteArgs* fused_perm = nullptr, const GatherArgs* fused_gather = nullptr) {
  const NvtxRange range("fused_moe.route");
  RouterArgs a{};
  a.x = static_cast<const uint16_t*>(x);
  a.wr = static_cast<const uint16_t*>(rw);
  a.topk_ids = ids;
  a.topk_w = tw;
  a.amax_part = reinterpret_cast<float*>(W + L.amax_x);
  a.logits_g = reinterpret_cast<float*>(W + L.logits);
  a.tile_counters = reinterpret_cast<int32_t*>(W + L.counters);
  a.hdr = reinterpret_cast<WsHeader*>(W + L.hdr);
  a.T = d.T;
  a.H = d.H;
  a.E = d.E;
  a.k = d.top_k;
  a.n_shared = shared_of(d);
  a.num_sms = num_sms();
  a.mode = FMOE_ROUTE_SOFTMAX;
  a.routed_scaling = 1.f;
  if (d.routing != nullptr && d.routing->mode == FMOE_ROUTE_SIGMOID_GROUPED) {
    a.mode = FMOE_ROUTE_SIGMOID_GROUPED;
    a.n_group = d.routing->n_group;
    a.topk_group = d.routing->topk_group;
    a.routed_scaling = d.routing->routed_scaling;
    a.bias = d.routing->bias;
  }
  a.route_done = &reinterpret_cast<WsHeader*>(W + L.hdr)->route_done;
  if (fused_perm != nullptr) {
    a.fuse_permute = 1;
    a.perm = *fused_perm;
    if (fused_gather != nullptr) {
      a.fuse_gather = 1;
      a.gather = *fused_gather;
    }
  }
  const char* name = fused_perm == nullptr ? "router"
                                            : (fused_gather == nullptr ? "router_permute"
                                                                       : "router_permute_gather");
  if (router_use_tiled(d.T, d.E, a.num_sms)) {
    RouterMaps m;
    if (!encode_rows_map(&m.x, x, static_cast<uint64_t>(d.H), static_cast<uint64_t>(d.T),
                         static_cast<uint32_t>(router_tile_tokens(d.E))) ||
        !encode_rows_map(&m.wr, rw, static_cast<uint64_t>(d.H), static_cast<uint64_t>(d.E),
                         static_cast<uint32_t>(router_tile_experts(d.E))))
      return FMOE_ERR_CUDA;
    FMOE_LAUNCH(name, launch_router_tiled(a, m, s), s);
  } else {
    FMOE_LAUNCH(name, launch_router(a, s), s);
  }
  return FMOE_OK;
}

PermuteArgs permute_args(const fmoe_dims& d, const Layout& L, const int32_t* ids,
                         const fmoe_scales* sc, int32_t* counts, int32_t* offsets, int32_t* rows,
                         int32_t* inv, char* W, bool with_plan) {
  PermuteArgs p{};
  p.topk_ids = ids;
  p.counts = counts;
  p.offsets = offsets;
  p.sorted_rows = rows;
  p.inv_perm = inv;
  p.amax_part = reinterpret_cast<const float*>(W + L.amax_x);
  p.hdr = reinterpret_cast<WsHeader*>(W + L.hdr);
  p.R = L.R;
  p.E = experts_all(d);
  p.k = slots_of(d);
  p.fp8 = L.fp8 ? 1 : 0;
  p.a1_static = sc != nullptr ? sc->a1_scale : 0.f;
  p.with_plan = with_plan ? 1 : 0;
  p.plan = plan_params(d, L, W);
  return p;
}

GatherArgs gather_args(const fmoe_dims& d, const Layout& L, const void* x, const int32_t* rows,
                       const int32_t* inv, void* a_perm, char* W) {
  WsHeader* hdr = reinterpret_cast<WsHeader*>(W + L.hdr);
  GatherArgs g{};
  g.x = static_cast<const uint16_t*>(x);
  g.sorted_rows = rows;
  g.inv_perm = inv;
  g.a_perm = a_perm;
  g.hdr = hdr;
  g.status = &hdr->status;
  g.R = L.R;
  g.H = d.H;
  g.k = slots_of(d);
  g.fp8 = L.fp8 ? 1 : 0;
  return g;
}

fmoe_status permute_impl(const fmoe_dims& d, const Layout& L, const int32_t* ids, const void* x,
                         const fmoe_scales* sc, int32_t* counts, int32_t* offsets, int32_t* rows,
                         int32_t* inv, void* a_perm, char* W, cudaStream_t s, bool with_plan) {
  const NvtxRange range("fused_moe.permute");
  const PermuteArgs p = permute_args(d, L, ids, sc, counts, offsets, rows, inv, W, with_plan);
  FMOE_LAUNCH(with_plan ? "permute_plan" : "permute", launch_permute(p, s), s);
  const GatherArgs g = gather_args(d, L, x, rows, inv, a_perm, W);
  FMOE_LAUNCH("gather_quant", launch_gather(g, s), s);
  return FMOE_OK;
}

// The grouped-GEMM arguments both contractions share.
GemmArgs gemm_base(const Layout& L, const int32_t* rows, const float* tw, char* W,
                   const fmoe_dims& d) {
  WsHeader* hdr = reinterpret_cast<WsHeader*>(W + L.hdr);
  GemmArgs g{};
  g.chunks = reinterpret_cast<Chunk*>(W + L.chunks);
  g.hdr = hdr;
  g.hdr_w = hdr;
  g.status = &hdr->status;
  g.topk_w = tw;
  g.sorted_rows = rows;
  g.amax_part = reinterpret_cast<float*>(W + L.amax_h);
  g.R = L.R;
  g.I = d.I;
  g.H = d.H;
  g.chunk_rows = L.chunk_rows;
  g.nstages = gemm_stages(L.swap, L.chunk_rows);
  g.wait_budget_ns = kWaitBudgetNs;
  return g;
}

// Step a3: plan (unless the permutation launch wrote it), the first contraction with
// SiLU(g)*u, and (swap-AB) the split-K finish of h with its max partials.
fmoe_status experts_first(const fmoe_dims& d, const Layout& L, const void* a_perm,
                          const int32_t* offsets, const int32_t* rows, const float* tw,
                          const void* w13, const fmoe_scales* sc, char* W, cudaStream_t s,
                          bool plan_done, bool plan_two_back) {
  const NvtxRange range("fused_moe.experts.first");
  const int sms = num_sms();
  const bool fp8 = L.fp8, swap = L.swap;
  const int H = d.H, I = d.I, E = experts_all(d), R = L.R;
  WsHeader* hdr = reinterpret_cast<WsHeader*>(W + L.hdr);
  float* amax_h = reinterpret_cast<float*>(W + L.amax_h);
  float* hbuf = reinterpret_cast<float*>(W + L.h);
  void* hq = W + L.hq;

  if (!plan_done) {
    PlanArgs pa{};
    pa.offsets = offsets;
    pa.hdr = hdr;
    pa.R = R;
    pa.E = E;
    pa.plan = plan_params(d, L, W);
    FMOE_LAUNCH("plan", launch_plan(pa, s), s);
  }

  const uint32_t xbox = swap ? 16u : 128u;
  GemmArgs g = gemm_base(L, rows, tw, W, d);
  if (!encode_map(&g.map_w, w13, fp8, static_cast<uint64_t>(H), static_cast<uint64_t>(E) * 2 * I,
                  swap ? 16u : 128u) ||
      !encode_map(&g.map_x, a_perm, fp8, static_cast<uint64_t>(H), static_cast<uint64_t>(R), xbox))
    return FMOE_ERR_CUDA;
  g.out = swap ? reinterpret_cast<float*>(W + L.p1) : (fp8 ? hbuf : nullptr);
  g.out_bf16 = fp8 ? nullptr : static_cast<uint16_t*>(hq);
  g.h_out = fp8 ? hbuf : nullptr;
  g.w_scale = fp8 ? sc->w13_scale : nullptr;
  g.K = H;
  g.Nout = 2 * I;
  g.rows_per_expert = 2 * I;
  // the first contraction may prefetch weights when its plan came two launches back (the
  // gather ran in between)
  g.prefetch_w = plan_two_back ? 1 : 0;
  if (L.pair)
    FMOE_LAUNCH("gemm1_pair", launch_gemm_pair(g, fp8, 1, sms, s), s);
  else
    FMOE_LAUNCH(swap ? "gemm1_swapab" : "gemm1_normal", launch_gemm(g, fp8, swap, 1, sms, s), s);

  if (swap) {
    // split-K > 1: finish h from the partials (returns at once when the plan chose split 1)
    Finalize1Args f{};
    f.part = reinterpret_cast<const float*>(W + L.p1);
    f.offsets = offsets;
    f.w13_scale = fp8 ? sc->w13_scale : nullptr;
    f.h = fp8 ? hbuf : nullptr;
    f.hq_bf16 = fp8 ? nullptr : static_cast<uint16_t*>(hq);
    f.amax_part = amax_h;
    f.hdr = hdr;
    f.R = R;
    f.I = I;
    f.E = E;
    f.fp8 = fp8 ? 1 : 0;
    FMOE_LAUNCH("finalize1", launch_finalize1(f, sms, s), s);
  }
  return FMOE_OK;
}

// Step a4 (and, swap-AB, the finish of the output): FP8 re-quantisation of h (its max
// from this call's partials, or from amax_in), the second contraction, then either the
// combined output (fused_out bf16 or out_f32 fp32 sums, swap-AB: split-K partials
// finished and combined in one pass) or y (finalize2 for swap-AB; the normal variants'
// GEMM writes y itself and the caller combines).
fmoe_status experts_second(const fmoe_dims& d, const Layout& L, const int32_t* offsets,
                           const int32_t* rows, const float* tw, const void* w2,
                           const fmoe_scales* sc, float* y, char* W, cudaStream_t s,
                           void* fused_out, float* out_f32, const int32_t* ids,
                           const int32_t* inv, const float* amax_in) {
  const NvtxRange range("fused_moe.experts.second");
  const int sms = num_sms();
  const bool fp8 = L.fp8, swap = L.swap;
  const int H = d.H, I = d.I, E = experts_all(d), R = L.R;
  WsHeader* hdr = reinterpret_cast<WsHeader*>(W + L.hdr);
  float* amax_h = reinterpret_cast<float*>(W + L.amax_h);
  float* hbuf = reinterpret_cast<float*>(W + L.h);
  void* hq = W + L.hq;

  const bool fq = fuse_quant_h(L, amax_in);
  if (fp8 && !fq) {
    QuantHArgs q{};
    q.h = hbuf;
    q.h_bf16 = nullptr;
    q.hq = static_cast<uint8_t*>(hq);
    q.amax_part = amax_h;
    q.amax_in = amax_in;
    q.hdr = hdr;
    q.R = R;
    q.I = I;
    q.a2_static = sc != nullptr ? sc->a2_scale : 0.f;
    FMOE_LAUNCH("quant_h", launch_quant_h(q, sms, s), s);
  }

  const uint32_t xbox = swap ? 16u : 128u;
  GemmArgs g2 = gemm_base(L, rows, tw, W, d);
  if (!encode_map(&g2.map_w, w2, fp8, static_cast<uint64_t>(I), static_cast<uint64_t>(E) * H, 128) ||
      !encode_map(&g2.map_x, hq, fp8, static_cast<uint64_t>(I), static_cast<uint64_t>(R), xbox))
    return FMOE_ERR_CUDA;
  g2.out = swap ? reinterpret_cast<float*>(W + L.p2) : y;
  g2.out_bf16 = nullptr;
  g2.h_out = nullptr;
  g2.w_scale = fp8 ? sc->w2_scale : nullptr;
  g2.K = I;
  g2.Nout = H;
  g2.rows_per_expert = H;
  g2.prefetch_w = 1;  // the chunk list was written at least two launches back (gemm1 between)
  if (fq) {
    g2.fuse_quant = 1;
    g2.q_h = hbuf;
    g2.q_hq = static_cast<uint8_t*>(hq);
    g2.q_ready = reinterpret_cast<int32_t*>(W + L.ready);
    g2.q_a2_static = sc != nullptr ? sc->a2_scale : 0.f;
  }
  if (L.pair)
    FMOE_LAUNCH("gemm2_pair", launch_gemm_pair(g2, fp8, 2, sms, s), s);
  else
    FMOE_LAUNCH(swap ? "gemm2_swapab" : "gemm2_normal", launch_gemm(g2, fp8, swap, 2, sms, s), s);

  if (swap && (fused_out != nullptr || out_f32 != nullptr)) {
    CombinePartialsArgs c{};
    c.part = reinterpret_cast<const float*>(W + L.p2);
    c.inv_perm = inv;
    c.topk_ids = ids;
    c.topk_w = tw;
    c.w2_scale = fp8 ? sc->w2_scale : nullptr;
    c.hdr = hdr;
    c.out = static_cast<uint16_t*>(fused_out);
    c.out_f32 = out_f32;
    c.T = d.T;
    c.H = H;
    c.k = slots_of(d);
    c.E = E;
    c.fp8 = fp8 ? 1 : 0;
    FMOE_LAUNCH("combine_partials", launch_combine_partials(c, sms, s), s);
  } else if (swap) {
    Finalize2Args f{};
    f.part = reinterpret_cast<const float*>(W + L.p2);
    f.offsets = offsets;
    f.w2_scale = fp8 ? sc->w2_scale : nullptr;
    f.topk_w = tw;
    f.sorted_rows = rows;
    f.hdr = hdr;
    f.status = &hdr->status;
    f.y = y;
    f.R = R;
    f.H = H;
    f.E = E;
    f.fp8 = fp8 ? 1 : 0;
    FMOE_LAUNCH("finalize2", launch_finalize2(f, sms, s), s);
  }
  return FMOE_OK;
}

// Steps a3-a4.  plan_done: the permute launch already wrote the GEMM plan.  fused_out
// (one-call path): in the swap-AB variant finish the second contraction's partials
// straight into the combined output (needs ids and inv) instead of writing y.
fmoe_status experts_impl(const fmoe_dims& d, const Layout& L, const void* a_perm,
                         const int32_t* offsets, const int32_t* rows, const float* tw,
                         const void* w13, const void* w2, const fmoe_scales* sc, float* y,
                         char* W, cudaStream_t s, bool plan_done = false,
                         void* fused_out = nullptr, const int32_t* ids = nullptr,
                         const int32_t* inv = nullptr, bool plan_two_back = false) {
  FMOE_TRY(experts_first(d, L, a_perm, offsets, rows, tw, w13, sc, W, s, plan_done, plan_two_back));
  return experts_second(d, L, offsets, rows, tw, w2, sc, y, W, s, fused_out, nullptr, ids, inv,
                        nullptr);
}

fmoe_status combine_impl(const fmoe_dims& d, const float* y, const int32_t* inv, void* out,
                         cudaStream_t s, float* out_f32 = nullptr) {
  const NvtxRange range("fused_moe.combine");
  CombineArgs c{};
  c.y = y;
  c.inv_perm = inv;
  c.out = static_cast<uint16_t*>(out);
  c.out_f32 = out_f32;
  c.T = d.T;
  c.H = d.H;
  c.k = slots_of(d);
  FMOE_LAUNCH("combine", launch_combine(c, num_sms(), s), s);
  return FMOE_OK;
}

// Workspace views of the one-call path's routing buffers and y.
struct OneCall {
  int32_t *ids, *counts, *offsets, *rows, *inv;
  float *tw, *y;
  OneCall(const Layout& L, char* W)
      : ids(reinterpret_cast<int32_t*>(W + L.ids)),
        counts(reinterpret_cast<int32_t*>(W + L.counts)),
        offsets(reinterpret_cast<int32_t*>(W + L.offsets)),
        rows(reinterpret_cast<int32_t*>(W + L.rows)),
        inv(reinterpret_cast<int32_t*>(W + L.inv)),
        tw(reinterpret_cast<float*>(W + L.tw)),
        y(reinterpret_cast<float*>(W + L.y)) {}
};

// Steps a1-a2 of the one-call path, then a3 (the first contraction).
fmoe_status first_half(const fmoe_dims& d, const Layout& L, const OneCall& b, const void* x,
                       const void* rw, const void* w13, const fmoe_scales* sc, char* W,
                       cudaStream_t s) {
  bool plan_two_back = true;  // the plan-writing launch is followed by the gather launch
  if (fuse_route_permute(L)) {
    const PermuteArgs p = permute_args(d, L, b.ids, sc, b.counts, b.offsets, b.rows, b.inv, W, true);
    const GatherArgs g = gather_args(d, L, x, b.rows, b.inv, W + L.a_perm, W);
    const bool fg = fuse_route_gather(d, L);
    FMOE_TRY(route_impl(d, L, x, rw, b.ids, b.tw, W, s, &p, fg ? &g : nullptr));
    if (!fg) FMOE_LAUNCH("gather_quant", launch_gather(g, s), s);
    plan_two_back = !fg;
  } else {
    FMOE_TRY(route_impl(d, L, x, rw, b.ids, b.tw, W, s));
    FMOE_TRY(permute_impl(d, L, b.ids, x, sc, b.counts, b.offsets, b.rows, b.inv, W + L.a_perm, W,
                          s, /*with_plan=*/true));
  }
  return experts_first(d, L, W + L.a_perm, b.offsets, b.rows, b.tw, w13, sc, W, s,
                       /*plan_done=*/true, plan_two_back);
}

// Step a4 and a5 of the one-call path: bf16 `out`, or (a tensor-parallel shard) the fp32
// sums `out_f32` with the max |h| taken from amax_in.
fmoe_status second_half(const fmoe_dims& d, const Layout& L, const OneCall& b, const void* w2,
                        const fmoe_scales* sc, void* out, float* out_f32, const float* amax_in,
                        char* W, cudaStream_t s) {
  FMOE_TRY(experts_second(d, L, b.offsets, b.rows, b.tw, w2, sc, b.y, W, s, out, out_f32, b.ids,
                          b.inv, amax_in));
  if (L.swap) return FMOE_OK;  // combined by combine_partials
  return combine_impl(d, b.y, b.inv, out, s, out_f32);
}

fmoe_status fused_impl(const fmoe_dims& d, const Layout& L, const void* x, const void* rw,
                       const void* w13, const void* w2, const fmoe_scales* sc, void* out, char* W,
                       cudaStream_t s) {
  const OneCall b(L, W);
  FMOE_TRY(first_half(d, L, b, x, rw, w13, sc, W, s));
  return second_half(d, L, b, w2, sc, out, nullptr, nullptr, W, s);
}

}  // namespace

namespace fmoe {
// The argument checks of the one-call layer, in the order fused_moe runs them: dims,
// then (T > 0) the tensor pointers and the FP8 weight scales.  No CUDA call.
fmoe_status check_layer_args(const fmoe_dims* dims, const void* x, const void* router_w,
                             const void* w13, const void* w2, const fmoe_scales* scales,
                             const void* out) {
  FMOE_TRY(check_dims(dims));
  if (dims->T == 0) return FMOE_OK;
  FMOE_TRY(check_ptrs(x, router_w, w13, w2, out));
  FMOE_TRY(check_fp8_scales(*dims, scales));
  if (dims->wdtype == FMOE_FP8_E4M3) FMOE_TRY(check_ptrs(scales->w13_scale, scales->w2_scale));
  return FMOE_OK;
}
}  // namespace fmoe

// ------------------------------------------------------------------ public API

extern "C" {

int32_t fused_moe_abi_version(void) { return FUSED_MOE_ABI_VERSION; }

const char* fused_moe_status_string(fmoe_status st) {
  switch (st) {
    case FMOE_OK: return "FMOE_OK";
    case FMOE_ERR_INVALID_ARG: return "FMOE_ERR_INVALID_ARG";
    case FMOE_ERR_UNSUPPORTED: return "FMOE_ERR_UNSUPPORTED";
    case FMOE_ERR_WORKSPACE: return "FMOE_ERR_WORKSPACE";
    case FMOE_ERR_CUDA: return "FMOE_ERR_CUDA";
    case FMOE_ERR_TIMEOUT: return "FMOE_ERR_TIMEOUT";
    case FMOE_ERR_DEVICE_BOUNDS: return "FMOE_ERR_DEVICE_BOUNDS";
  }
  return "FMOE_ERR_UNKNOWN";
}

size_t fused_moe_workspace_size(const fmoe_dims* dims) {
  if (check_dims(dims) != FMOE_OK) return 0;
  return make_layout(*dims).total;
}

fmoe_status fused_moe_workspace_init(void* ws, size_t ws_bytes, fmoe_stream stream) {
  if (ws == nullptr) return FMOE_ERR_INVALID_ARG;
  const size_t head = sizeof(WsHeader) + static_cast<size_t>(kRouterMaxTiles) * 4;
  if (ws_bytes < head) return FMOE_ERR_WORKSPACE;
  return cuda_status(cudaMemsetAsync(ws, 0, head, static_cast<cudaStream_t>(stream)));
}

fmoe_status fused_moe_route(const fmoe_dims* dims, const void* x, const void* router_w,
                            int32_t* topk_ids, float* topk_w, void* ws, size_t ws_bytes,
                            fmoe_stream stream) {
  FMOE_TRY(check_dims(dims));
  if (dims->T == 0) return FMOE_OK;
  FMOE_TRY(check_ptrs(x, router_w, topk_ids, topk_w));
  const Layout L = make_layout(*dims);
  FMOE_TRY(check_ws(L, ws, ws_bytes));
  return route_impl(*dims, L, x, router_w, topk_ids, topk_w, static_cast<char*>(ws),
                    static_cast<cudaStream_t>(stream));
}

fmoe_status fused_moe_permute(const fmoe_dims* dims, const int32_t* topk_ids, const void* x,
                              const fmoe_scales* scales, int32_t* counts, int32_t* offsets,
                              int32_t* sorted_rows, int32_t* inv_perm, void* a_perm, void* ws,
                              size_t ws_bytes, fmoe_stream stream) {
  FMOE_TRY(check_dims(dims));
  if (dims->T == 0) return FMOE_OK;
  FMOE_TRY(check_ptrs(topk_ids, x, counts, offsets, sorted_rows, inv_perm, a_perm));
  const Layout L = make_layout(*dims);
  FMOE_TRY(check_ws(L, ws, ws_bytes));
  return permute_impl(*dims, L, topk_ids, x, scales, counts, offsets, sorted_rows, inv_perm,
                      a_perm, static_cast<char*>(ws), static_cast<cudaStream_t>(stream),
                      /*with_plan=*/false);
}

fmoe_status fused_moe_experts(const fmoe_dims* dims, const void* a_perm, const int32_t* offsets,
                              const int32_t* sorted_rows, const float* topk_w, const void* w13,
                              const void* w2, const fmoe_scales* scales, float* y_perm, void* ws,
                              size_t ws_bytes, fmoe_stream stream) {
  FMOE_TRY(check_dims(dims));
  if (dims->T == 0) return FMOE_OK;
  FMOE_TRY(check_ptrs(a_perm, offsets, sorted_rows, topk_w, w13, w2, y_perm));
  FMOE_TRY(check_fp8_scales(*dims, scales));
  if (dims->wdtype == FMOE_FP8_E4M3) FMOE_TRY(check_ptrs(scales->w13_scale, scales->w2_scale));
  const Layout L = make_layout(*dims);
  FMOE_TRY(check_ws(L, ws, ws_bytes));
  return experts_impl(*dims, L, a_perm, offsets, sorted_rows, topk_w, w13, w2, scales, y_perm,
                      static_cast<char*>(ws), static_cast<cudaStream_t>(stream));
}

fmoe_status fused_moe_combine(const fmoe_dims* dims, const float* y_perm, const int32_t* inv_perm,
                              void* out, fmoe_stream stream) {
  FMOE_TRY(check_dims(dims));
  if (dims->T == 0) return FMOE_OK;
  FMOE_TRY(check_ptrs(y_perm, inv_perm, out));
  return combine_impl(*dims, y_perm, inv_perm, out, static_cast<cudaStream_t>(stream));
}

fmoe_status fused_moe(const fmoe_dims* dims, const void* x, const void* router_w, const void* w13,
                      const void* w2, const fmoe_scales* scales, void* out, void* ws,
                      size_t ws_bytes, fmoe_stream stream) {
  FMOE_TRY(fmoe::check_layer_args(dims, x, router_w, w13, w2, scales, out));
  if (dims->T == 0) return FMOE_OK;
  const Layout L = make_layout(*dims);
  FMOE_TRY(check_ws(L, ws, ws_bytes));
  return fused_impl(*dims, L, x, router_w, w13, w2, scales, out, static_cast<char*>(ws),
                    static_cast<cudaStream_t>(stream));
}

fmoe_status fused_moe_tp_begin(const fmoe_dims* dims, const void* x, const void* router_w,
                               const void* w13, const fmoe_scales* scales, float* amax_h,
                               void* ws, size_t ws_bytes, fmoe_stream stream) {
  FMOE_TRY(check_dims(dims));
  if (dims->T == 0) return FMOE_OK;
  FMOE_TRY(check_ptrs(x, router_w, w13));
  if (amax_h == nullptr) return FMOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(amax_h) & 3u) != 0) return FMOE_ERR_UNSUPPORTED;
  FMOE_TRY(check_fp8_scales(*dims, scales));
  if (dims->wdtype == FMOE_FP8_E4M3) FMOE_TRY(check_ptrs(scales->w13_scale, scales->w2_scale));
  const Layout L = make_layout(*dims);
  FMOE_TRY(check_ws(L, ws, ws_bytes));
  char* W = static_cast<char*>(ws);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const OneCall b(L, W);
  FMOE_TRY(first_half(*dims, L, b, x, router_w, w13, scales, W, s));
  AmaxReduceArgs r{};
  r.amax_part = reinterpret_cast<const float*>(W + L.amax_h);
  r.hdr = reinterpret_cast<const WsHeader*>(W + L.hdr);
  r.amax_out = amax_h;
  r.fp8 = L.fp8 ? 1 : 0;
  FMOE_LAUNCH("amax_reduce", launch_amax_reduce(r, s), s);
  return FMOE_OK;
}

fmoe_status fused_moe_tp_end(const fmoe_dims* dims, const void* w2, const fmoe_scales* scales,
                             const float* amax_h, float* out_partial, void* ws, size_t ws_bytes,
                             fmoe_stream stream) {
  FMOE_TRY(check_dims(dims));
  if (dims->T == 0) return FMOE_OK;
  FMOE_TRY(check_ptrs(w2, out_partial));
  if (amax_h == nullptr) return FMOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(amax_h) & 3u) != 0) return FMOE_ERR_UNSUPPORTED;
  FMOE_TRY(check_fp8_scales(*dims, scales));
  if (dims->wdtype == FMOE_FP8_E4M3) FMOE_TRY(check_ptrs(scales->w13_scale, scales->w2_scale));
  const Layout L = make_layout(*dims);
  FMOE_TRY(check_ws(L, ws, ws_bytes));
  char* W = static_cast<char*>(ws);
  const OneCall b(L, W);
  return second_half(*dims, L, b, w2, scales, nullptr, out_partial, amax_h, W,
                     static_cast<cudaStream_t>(stream));
}

fmoe_status fused_moe_tp_finish(int64_t n, const float* out_sum, void* out, fmoe_stream stream) {
  if (n < 0) return FMOE_ERR_INVALID_ARG;
  if (n == 0) return FMOE_OK;
  FMOE_TRY(check_ptrs(out_sum, out));
  if (n % 8 != 0 || n >= (int64_t(1) << 40)) return FMOE_ERR_UNSUPPORTED;
  return cuda_status(launch_to_bf16(out_sum, static_cast<uint16_t*>(out), static_cast<size_t>(n),
                                    num_sms(), static_cast<cudaStream_t>(stream)));
}

fmoe_status fused_moe_host_io(const fmoe_dims* dims, const void* x_host, const void* router_w,
                              const void* w13, const void* w2, const fmoe_scales* scales,
                              void* out_host, void* ws, size_t ws_bytes, fmoe_stream stream) {
  FMOE_TRY(check_dims(dims));
  if (dims->T == 0) return FMOE_OK;
  if (x_host == nullptr || out_host == nullptr) return FMOE_ERR_INVALID_ARG;
  FMOE_TRY(check_ptrs(router_w, w13, w2));
  FMOE_TRY(check_fp8_scales(*dims, scales));
  if (dims->wdtype == FMOE_FP8_E4M3) FMOE_TRY(check_ptrs(scales->w13_scale, scales->w2_scale));
  const Layout L = make_layout(*dims);
  FMOE_TRY(check_ws(L, ws, ws_bytes));
  char* W = static_cast<char*>(ws);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t xbytes = static_cast<size_t>(dims->T) * dims->H * 2;
  FMOE_TRY(cuda_status(cudaMemcpyAsync(W + L.x_in, x_host, xbytes, cudaMemcpyHostToDevice, s)));
  FMOE_TRY(fused_impl(*dims, L, W + L.x_in, router_w, w13, w2, scales, W + L.out_dev, W, s));
  FMOE_TRY(cuda_status(cudaMemcpyAsync(out_host, W + L.out_dev, xbytes, cudaMemcpyDeviceToHost, s)));
  return cuda_status(cudaStreamSynchronize(s));
}

int32_t fused_moe_launches_per_call(const fmoe_dims* dims) {
  if (check_dims(dims) != FMOE_OK) return -1;
  if (dims->T == 0) return 0;
  const Layout L = make_layout(*dims);
  // router [+ permute (+plan) [+ gather]], gemm1, [finalize1], [quant_h], gemm2, combine;
  // the CTA-pair FP8 second contraction quantises h itself
  int n = 4 + (L.fp8 && !fuse_quant_h(L, nullptr) ? 1 : 0) + (L.swap ? 1 : 0);
  if (!fuse_route_permute(L)) n += 2;        // permute, gather
  else if (!fuse_route_gather(*dims, L)) n += 1;  // gather
  return n;
}

fmoe_status fused_moe_profile(const fmoe_dims* dims, const void* x, const void* router_w,
                              const void* w13, const void* w2, const fmoe_scales* scales, void* out,
                              void* ws, size_t ws_bytes, fmoe_stream stream, float* ms_host,
                              const char** names_host, int32_t cap, int32_t* n_host) {
  FMOE_TRY(check_dims(dims));
  if (n_host == nullptr || ms_host == nullptr || cap < 1) return FMOE_ERR_INVALID_ARG;
  *n_host = 0;
  if (dims->T == 0) return FMOE_OK;
  FMOE_TRY(check_ptrs(x, router_w, w13, w2, out));
  FMOE_TRY(check_fp8_scales(*dims, scales));
  if (dims->wdtype == FMOE_FP8_E4M3) FMOE_TRY(check_ptrs(scales->w13_scale, scales->w2_scale));
  const Layout L = make_layout(*dims);
  FMOE_TRY(check_ws(L, ws, ws_bytes));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  static thread_local bool created = false;
  if (!created) {
    for (auto& e : g_rec.ev)
      if (cudaEventCreate(&e) != cudaSuccess) return FMOE_ERR_CUDA;
    created = true;
  }
  g_rec.n = 0;
  g_rec.active = true;
  fmoe_status st = cuda_status(cudaEventRecord(g_rec.ev[0], s));
  if (st == FMOE_OK)
    st = fused_impl(*dims, L, x, router_w, w13, w2, scales, out, static_cast<char*>(ws), s);
  g_rec.active = false;
  FMOE_TRY(st);
  FMOE_TRY(cuda_status(cudaStreamSynchronize(s)));
  const int n = std::min<int>(g_rec.n, cap);
  for (int i = 0; i < n; ++i) {
    float ms = 0.f;
    FMOE_TRY(cuda_status(cudaEventElapsedTime(&ms, g_rec.ev[i], g_rec.ev[i + 1])));
    ms_host[i] = ms;
    if (names_host != nullptr) names_host[i] = g_rec.names[i];
  }
  *n_host = n;
  return FMOE_OK;
}

fmoe_status fused_moe_selftest_wait(void* ws, size_t ws_bytes, uint64_t budget_ns,
                                    fmoe_stream stream) {
  if (ws == nullptr) return FMOE_ERR_INVALID_ARG;
  if (ws_bytes < sizeof(WsHeader)) return FMOE_ERR_WORKSPACE;
  if (budget_ns > 10000000000ull) return FMOE_ERR_INVALID_ARG;  // at most 10 s
  return cuda_status(launch_wait_selftest(static_cast<WsHeader*>(ws), budget_ns,
                                          static_cast<cudaStream_t>(stream)));
}

fmoe_status fused_moe_get_device_status(const void* ws, fmoe_stream stream) {
  if (ws == nullptr) return FMOE_ERR_INVALID_ARG;
  int32_t st = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&st, ws, sizeof(st), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return FMOE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return FMOE_ERR_CUDA;
  return static_cast<fmoe_status>(st);
}

fmoe_status fused_moe_debug_scalars(const void* ws, float* f6, int32_t* i3, fmoe_stream stream) {
  if (ws == nullptr) return FMOE_ERR_INVALID_ARG;
  WsHeader h;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&h, ws, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess) return FMOE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return FMOE_ERR_CUDA;
  if (f6 != nullptr) {
    f6[0] = h.amax_x;
    f6[1] = h.s1;
    f6[2] = h.inv1;
    f6[3] = h.amax_h;
    f6[4] = h.s2;
    f6[5] = h.inv2;
  }
  if (i3 != nullptr) {
    i3[0] = h.n_chunks;
    i3[1] = h.split1;
    i3[2] = h.split2;
  }
  return FMOE_OK;
}

fmoe_status fused_inv_rope_fp8_quant_per_head(const fmoe_rope_dims* d, const void* x,
                                              const int32_t* positions, const float* cos_sin,
                                              void* q, float* scales, int32_t* device_status,
                                              fmoe_stream stream) {
  if (d == nullptr) return FMOE_ERR_INVALID_ARG;
  if (d->T < 0 || d->n_heads < 1 || d->max_pos < 1 || (d->style != 0 && d->style != 1))
    return FMOE_ERR_INVALID_ARG;
  if (d->head_dim != 64 && d->head_dim != 128 && d->head_dim != 256) return FMOE_ERR_INVALID_ARG;
  const int epl = d->head_dim / 32, r = d->rot_dim;
  if (r < 2 * epl || r > d->head_dim) return FMOE_ERR_INVALID_ARG;
  if (d->style == 0 ? (r & (r - 1)) != 0 : r % (2 * epl) != 0) return FMOE_ERR_INVALID_ARG;
  const int64_t lim = int64_t(1) << 31;
  if (static_cast<int64_t>(d->T) * d->n_heads * d->head_dim >= lim ||
      static_cast<int64_t>(d->max_pos) * r >= lim)
    return FMOE_ERR_UNSUPPORTED;
  if (d->T == 0) return FMOE_OK;
  FMOE_TRY(check_ptrs(x, positions, cos_sin, q, scales));
  if (device_status != nullptr && (reinterpret_cast<uintptr_t>(device_status) & 3u) != 0)
    return FMOE_ERR_UNSUPPORTED;
  RopeArgs a{};
  a.x = static_cast<const uint16_t*>(x);
  a.positions = positions;
  a.cos_sin = cos_sin;
  a.q = static_cast<uint8_t*>(q);
  a.scales = scales;
  a.status = device_status;
  a.T = d->T;
  a.n_heads = d->n_heads;
  a.head_dim = d->head_dim;
  a.rot_dim = r;
  a.style = d->style;
  a.max_pos = d->max_pos;
  return cuda_status(launch_inv_rope_fp8(a, num_sms(), static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
