// Fused inverse rotary embedding + per-head FP8 quantisation.
//
// The second kernel the pages optimise: a fused rotary-embedding plus FP8-quantisation
// kernel that Triton recompiled for every new token count (codebridge-ai.com blog "AWS
// MoE kernel: WGMMA, Triton, TTFT", section "3. Kill JIT recompilation";
// agentic-affairs.com, third change).  This one is compiled ahead of time for every
// shape, so the recompilation the pages fix cannot arise.
//
// For token t (position pos[t]) and head h of x [T, n_heads, head_dim] (bf16):
//   pairs (a, b) of the first rot_dim coordinates, (i, i + rot_dim/2) (style 0) or
//   (2i, 2i+1) (style 1), are rotated by -theta(pos, i):
//     y_a = x_a*cos + x_b*sin,  y_b = -(x_a*sin) + x_b*cos
//   each product and each sum rounded to fp32 separately (no fused multiply-add), in
//   that order; coordinates past rot_dim pass through;
//   scale[t, h] = amax|y| / 448 (1 if the head is zero), q = e4m3(y * (448/amax)),
//   round to nearest even, saturating.
//
// HBM-bound: 2 bytes read and 1 byte written per element plus 4 bytes of scale per
// head; the rotary table (max_pos x rot_dim fp32) is gathered through L2.  One warp
// handles units of up to four heads of one token, lane l owning the EPL = head_dim/32
// consecutive coordinates [EPL*l, EPL*l + EPL) of each head: one vector load and one
// packed store per head and lane, with the next unit's loads in flight meanwhile.  The
// half-split partner of a coordinate lives rot_dim/(2*EPL) lanes away (a lane xor for
// power-of-two rot_dim); interleaved partners are in the same lane.  A unit's scales are
// computed one head per lane (two IEEE divisions per head, issued once per unit) and
// broadcast by shuffles.  The grid is the number of blocks that fit on the GPU at once
// (a persistent grid-stride loop).
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "fmoe_kernels.h"

namespace fmoe {

namespace {

constexpr int kRopeThreads = 256;

template <int EPL> struct Vec;
template <> struct Vec<2> { using X = uint32_t; using F = float2; using Q = uint16_t; };
template <> struct Vec<4> { using X = uint2; using F = float4; using Q = uint32_t; };
template <> struct Vec<8> { using X = uint4; using F = float4; using Q = uint2; };

template <int EPL>
__device__ __forceinline__ void unpack_bf16(const typename Vec<EPL>::X& v, float (&f)[EPL]) {
  const uint32_t* w = reinterpret_cast<const uint32_t*>(&v);
#pragma unroll
  for (int i = 0; i < EPL / 2; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// n consecutive fp32 values of a table row (n = 1, 2, 4 or 8; 4-byte aligned at least
// n*4 bytes when n <= 4, 16 bytes when n == 8).
template <int N>
__device__ __forceinline__ void load_row(const float* p, float (&v)[N]) {
  if constexpr (N == 1) {
    v[0] = __ldg(p);
  } else if constexpr (N == 2) {
    const float2 a = __ldg(reinterpret_cast<const float2*>(p));
    v[0] = a.x; v[1] = a.y;
  } else if constexpr (N == 4) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  } else {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}

// Heads a warp takes per unit: 4, so that the registers of a unit in flight and of the
// next one stay small enough for three 256-thread blocks per SM (two for head_dim 256).
template <int EPL> constexpr int heads_per_step() { return 4; }

// fadd(fmul(x, c), fmul(o, s)) for two coordinates, each product and each sum rounded
// separately (__fmul_rn / __fadd_rn are never contracted into a fused multiply-add).  The
// paired fp32 instructions were tried here and changed the last bit of some results, so
// the scalar forms stay.
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  return make_float2(__fmul_rn(a.x, b.x), __fmul_rn(a.y, b.y));
}
__device__ __forceinline__ float2 rot2(float2 x, float2 c, float2 o, float2 s) {
  return make_float2(__fadd_rn(__fmul_rn(x.x, c.x), __fmul_rn(o.x, s.x)),
                     __fadd_rn(__fmul_rn(x.y, c.y), __fmul_rn(o.y, s.y)));
}

template <int EPL, int kStyle, bool kFull>
__device__ __forceinline__ void rope_unit(const typename Vec<EPL>::X (&xv)[heads_per_step<EPL>()],
                                          int nh, const float* cc, const float* sn, bool rotated,
                                          int partner_xor, int lane, uint8_t* qdst, int hd,
                                          float* sdst) {
  constexpr int HPS = heads_per_step<EPL>();
  constexpr int NW = EPL / 2;  // 32-bit words (bf16 pairs) per lane
  float y[HPS][EPL];
  float m[HPS];
#pragma unroll
  for (int k = 0; k < HPS; ++k) {
    m[k] = 0.f;
    if (k >= nh) continue;  // warp-uniform
    float x[EPL];
    unpack_bf16<EPL>(xv[k], x);
    if constexpr (kStyle == 0) {
      // the partner's coordinates, moved as packed bf16 pairs (one shuffle per word)
      const uint32_t* wv = reinterpret_cast<const uint32_t*>(&xv[k]);
      float o[EPL];
#pragma unroll
      for (int i = 0; i < NW; ++i) {
        const uint32_t ow = __shfl_xor_sync(0xffffffffu, wv[i], partner_xor);
        o[2 * i] = __uint_as_float(ow << 16);
        o[2 * i + 1] = __uint_as_float(ow & 0xFFFF0000u);
      }
#pragma unroll
      for (int e = 0; e < EPL; e += 2) {
        const float2 r = rot2(make_float2(x[e], x[e + 1]), make_float2(cc[e], cc[e + 1]),
                              make_float2(o[e], o[e + 1]), make_float2(sn[e], sn[e + 1]));
        y[k][e] = (kFull || rotated) ? r.x : x[e];
        y[k][e + 1] = (kFull || rotated) ? r.y : x[e + 1];
      }
    } else {
#pragma unroll
      for (int e = 0; e < EPL; e += 2) {
        const float c = cc[e / 2], s = sn[e / 2];
        const float2 r = rot2(make_float2(x[e], x[e + 1]), make_float2(c, c),
                              make_float2(x[e + 1], x[e]), make_float2(s, -s));
        y[k][e] = (kFull || rotated) ? r.x : x[e];
        y[k][e + 1] = (kFull || rotated) ? r.y : x[e + 1];
      }
    }
    float mx = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) mx = fmaxf(mx, fabsf(y[k][e]));
    m[k] = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(mx)));
  }
  float ml = 0.f;  // head `lane`'s max |y|
#pragma unroll
  for (int k = 0; k < HPS; ++k) ml = lane == k ? m[k] : ml;
  const float inv_l = ml > 0.f ? 448.0f / ml : 1.f;
  if (lane < nh) __stcs(sdst + lane, ml > 0.f ? ml / 448.0f : 1.f);
#pragma unroll
  for (int k = 0; k < HPS; ++k) {
    if (k >= nh) break;  // warp-uniform
    const float inv = __shfl_sync(0xffffffffu, inv_l, k);
    typename Vec<EPL>::Q qv;
    uint16_t* q16 = reinterpret_cast<uint16_t*>(&qv);
#pragma unroll
    for (int e = 0; e < EPL; e += 2) {
      const float2 p = mul2(make_float2(y[k][e], y[k][e + 1]), make_float2(inv, inv));
      q16[e / 2] = static_cast<uint16_t>(__nv_cvt_float2_to_fp8x2(p, __NV_SATFINITE, __NV_E4M3));
    }
    __stcs(reinterpret_cast<typename Vec<EPL>::Q*>(qdst + k * hd), qv);
  }
}

// Lane geometry shared by both kernels.
template <int EPL, int kStyle>
struct RopeLane {
  int j0, half, i0, partner_xor;
  bool rotated, is_a;
  __device__ RopeLane(const RopeArgs& a, int lane) {
    const int rot = a.rot_dim;
    half = rot / 2;
    j0 = lane * EPL;                 // first coordinate of this lane
    rotated = j0 < rot;              // EPL divides rot: a lane is all in or all out
    is_a = kStyle == 0 ? j0 < half : true;
    // style 0: pair index of coordinate j0 (its partner's too); style 1: j0 / 2
    i0 = kStyle == 0 ? (is_a ? j0 : j0 - half) : j0 / 2;
    partner_xor = kStyle == 0 ? half / EPL : 0;
  }
};

// ------------------------------------------------------------------------------------
// The kernel: each warp keeps the next unit's x rows and table entries in registers
// while it works on the current one.
// ------------------------------------------------------------------------------------
template <int EPL, int kStyle, bool kFull>
__global__ void __launch_bounds__(kRopeThreads, EPL == 8 ? 2 : 3) inv_rope_fp8_kernel(const RopeArgs a) {
  griddep_wait();
  griddep_launch_dependents();
  constexpr int HPS = heads_per_step<EPL>();
  constexpr int NC = kStyle == 0 ? EPL : EPL / 2;  // table entries a lane needs
  using XV = typename Vec<EPL>::X;
  const int lane = threadIdx.x & 31;
  const int gwarp = (blockIdx.x * kRopeThreads + threadIdx.x) >> 5;
  const int nwarps = (gridDim.x * kRopeThreads) >> 5;
  const int hd = 32 * EPL, rot = a.rot_dim;
  const RopeLane<EPL, kStyle> L(a, lane);
  const int hgroups = (a.n_heads + HPS - 1) / HPS;
  const int units = a.T * hgroups;  // < 2^31: T * n_heads * head_dim is checked on the host

  // Software pipeline over this warp's units u, u + nwarps, ...: the position of unit
  // u + 2*nwarps and the x rows and table entries of unit u + nwarps are in flight while
  // unit u is rotated, quantised and stored.  Unit u is (token u / hgroups, head group
  // u % hgroups); the three units in flight carry their indices forward by nwarps.
  struct Unit {
    int t, hg;
  };
  const int dq = nwarps / hgroups, dr = nwarps % hgroups;
  auto advance = [&](Unit w) {
    w.t += dq;
    w.hg += dr;
    if (w.hg >= hgroups) {
      w.hg -= hgroups;
      ++w.t;
    }
    return w;
  };
  auto pos_of = [&](Unit w) -> int {
    if (w.t >= a.T) return 0;
    int p = __ldg(a.positions + w.t);
    if (p < 0 || p >= a.max_pos) {
      if (lane == 0 && w.hg == 0 && a.status != nullptr) record_status(a.status, ST_BOUNDS);
      p = 0;
    }
    return p;
  };
  auto load_x = [&](Unit w, XV (&xv)[HPS]) {
    if (w.t >= a.T) return;
    const int h0 = w.hg * HPS;
    const XV* src = reinterpret_cast<const XV*>(
        a.x + (static_cast<size_t>(w.t) * a.n_heads + h0) * hd + L.j0);
#pragma unroll
    for (int k = 0; k < HPS; ++k)
      if (h0 + k < a.n_heads) xv[k] = __ldcs(src + k * 32);  // streamed once
  };
  // the sines come pre-negated for the b coordinates of a half-split pair, so that every
  // rotated coordinate is fadd(fmul(x, cos), fmul(partner, sin')): for b that is
  // -(x_a*sin) + x_b*cos exactly (IEEE addition commutes and negation is exact)
  auto load_table = [&](Unit w, int p, float (&cs)[NC], float (&sn)[NC]) {
    if (w.t >= a.T || !(kFull || L.rotated)) return;
    const float* row = a.cos_sin + static_cast<size_t>(p) * rot;
    load_row<NC>(row + L.i0, cs);
    load_row<NC>(row + L.half + L.i0, sn);
    if (kStyle == 0 && !L.is_a) {
#pragma unroll
      for (int i = 0; i < NC; ++i) sn[i] = -sn[i];
    }
  };

  if (gwarp >= units) return;
  Unit uc{gwarp / hgroups, gwarp % hgroups};
  Unit un = advance(uc), ua = advance(un);
  XV xc[HPS], xn[HPS];
  float cc[NC], sc_[NC], cn[NC], sn_[NC];
  for (int i = 0; i < NC; ++i) cc[i] = sc_[i] = cn[i] = sn_[i] = 0.f;
  int p_next = pos_of(un);
  load_x(uc, xc);
  load_table(uc, pos_of(uc), cc, sc_);
  while (uc.t < a.T) {
    // next unit's x and table (its position is already here), the one after's position
    load_x(un, xn);
    load_table(un, p_next, cn, sn_);
    const int p_after = pos_of(ua);
    const int h0 = uc.hg * HPS;
    const size_t head0 = static_cast<size_t>(uc.t) * a.n_heads + h0;
    rope_unit<EPL, kStyle, kFull>(xc, min(HPS, a.n_heads - h0), cc, sc_, L.rotated,
                                  L.partner_xor, lane, a.q + head0 * hd + L.j0, hd, a.scales + head0);
#pragma unroll
    for (int k = 0; k < HPS; ++k) xc[k] = xn[k];
#pragma unroll
    for (int i = 0; i < NC; ++i) {
      cc[i] = cn[i];
      sc_[i] = sn_[i];
    }
    p_next = p_after;
    uc = un;
    un = ua;
    ua = advance(ua);
  }
}

template <int EPL, int kStyle, bool kFull>
cudaError_t launch_rope(const RopeArgs& a, int num_sms, cudaStream_t s) {
  constexpr int HPS = heads_per_step<EPL>();
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  const long units = static_cast<long>(a.T) * ((a.n_heads + HPS - 1) / HPS);  // < 2^31
  const long warps_per_block = kRopeThreads / 32;
  long grid = (units + warps_per_block - 1) / warps_per_block;
  static int resident[64] = {0};  // blocks per SM, per device
  if (resident[dev] == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, inv_rope_fp8_kernel<EPL, kStyle, kFull>,
                                                      kRopeThreads, 0) != cudaSuccess || n < 1) {
      (void)cudaGetLastError();
      n = 1;
    }
    resident[dev] = n;
  }
  const long cap = static_cast<long>(num_sms) * resident[dev];
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  return launch_k(inv_rope_fp8_kernel<EPL, kStyle, kFull>, dim3(static_cast<unsigned>(grid)),
                  dim3(kRopeThreads), 0, s, a);
}

template <int EPL, int kStyle>
cudaError_t launch_rope_rot(const RopeArgs& a, int num_sms, cudaStream_t s) {
  // every coordinate rotated (the usual full rotary): no pass-through selects
  if (a.rot_dim == a.head_dim) return launch_rope<EPL, kStyle, true>(a, num_sms, s);
  return launch_rope<EPL, kStyle, false>(a, num_sms, s);
}

}  // namespace

cudaError_t launch_inv_rope_fp8(const RopeArgs& a, int num_sms, cudaStream_t s) {
  const int epl = a.head_dim / 32;
  if (a.style == 0) {
    if (epl == 2) return launch_rope_rot<2, 0>(a, num_sms, s);
    if (epl == 4) return launch_rope_rot<4, 0>(a, num_sms, s);
    return launch_rope_rot<8, 0>(a, num_sms, s);
  }
  if (epl == 2) return launch_rope_rot<2, 1>(a, num_sms, s);
  if (epl == 4) return launch_rope_rot<4, 1>(a, num_sms, s);
  return launch_rope_rot<8, 1>(a, num_sms, s);
}

}  // namespace fmoe
