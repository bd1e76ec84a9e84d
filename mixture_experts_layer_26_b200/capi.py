"""ctypes binding of libfused_moe.so (include/fused_moe.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  torch supplies device memory (tensor.data_ptr()) and streams.  Importing
this module fails loudly when the library has not been built; there is no fallback.

Low-level functions keep the C names (fused_moe_route, fused_moe_permute,
fused_moe_experts, fused_moe_combine, fused_moe, fused_moe_host_io, ...) and take
torch tensors; `FusedMoE` wraps a workspace for repeated one-call use.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_float, c_int32, c_size_t, c_void_p
from typing import Optional

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfused_moe.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m mixture_experts_layer_26_b200.build` "
        "(the fused MoE layer has no CPU or Python fallback)")

_lib = ctypes.CDLL(LIB_PATH)

FMOE_OK, FMOE_ERR_INVALID_ARG, FMOE_ERR_UNSUPPORTED, FMOE_ERR_WORKSPACE = 0, 1, 2, 3
FMOE_ERR_CUDA, FMOE_ERR_TIMEOUT, FMOE_ERR_DEVICE_BOUNDS = 4, 5, 6
FMOE_BF16, FMOE_FP8_E4M3 = 0, 1
VARIANTS = {"auto": 0, "swap_ab": 1, "normal": 2, "normal_pair": 3}

EXPORTED = (
    "fused_moe_abi_version", "fused_moe_status_string", "fused_moe_workspace_size",
    "fused_moe_workspace_init", "fused_moe_route", "fused_moe_permute", "fused_moe_experts",
    "fused_moe_combine", "fused_moe", "fused_moe_host_io", "fused_moe_get_device_status",
    "fused_moe_debug_scalars", "fused_moe_launches_per_call", "fused_moe_profile",
    "fused_moe_static_workspace", "fused_moe_selftest_wait",
    "fused_inv_rope_fp8_quant_per_head", "fused_moe_tp_begin", "fused_moe_tp_end",
    "fused_moe_tp_finish",
)
STATIC_WS_BYTES = 64 << 20  # FUSED_MOE_STATIC_WS_BYTES


FMOE_ROUTE_SOFTMAX, FMOE_ROUTE_SIGMOID_GROUPED = 0, 1


class FmoeRouting(ctypes.Structure):
    _fields_ = [("mode", c_int32), ("n_group", c_int32), ("topk_group", c_int32),
                ("routed_scaling", c_float), ("bias", c_void_p), ("n_shared", c_int32)]


class FmoeDims(ctypes.Structure):
    _fields_ = [("T", c_int32), ("H", c_int32), ("I", c_int32), ("E", c_int32),
                ("top_k", c_int32), ("wdtype", c_int32), ("variant", c_int32),
                ("routing", POINTER(FmoeRouting))]


class FmoeRopeDims(ctypes.Structure):
    _fields_ = [("T", c_int32), ("n_heads", c_int32), ("head_dim", c_int32),
                ("rot_dim", c_int32), ("style", c_int32), ("max_pos", c_int32)]


class FmoeScales(ctypes.Structure):
    _fields_ = [("w13_scale", c_void_p), ("w2_scale", c_void_p),
                ("a1_scale", c_float), ("a2_scale", c_float)]


def _sig(name, restype, *argtypes):
    f = getattr(_lib, name)
    f.restype = restype
    f.argtypes = list(argtypes)
    return f


_DP = POINTER(FmoeDims)
_SP = POINTER(FmoeScales)
_abi = _sig("fused_moe_abi_version", c_int32)
_status_string = _sig("fused_moe_status_string", c_char_p, c_int32)
_ws_size = _sig("fused_moe_workspace_size", c_size_t, _DP)
_ws_init = _sig("fused_moe_workspace_init", c_int32, c_void_p, c_size_t, c_void_p)
_route = _sig("fused_moe_route", c_int32, _DP, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
              c_size_t, c_void_p)
_permute = _sig("fused_moe_permute", c_int32, _DP, c_void_p, c_void_p, _SP, c_void_p, c_void_p,
                c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p)
_experts = _sig("fused_moe_experts", c_int32, _DP, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                c_void_p, _SP, c_void_p, c_void_p, c_size_t, c_void_p)
_combine = _sig("fused_moe_combine", c_int32, _DP, c_void_p, c_void_p, c_void_p, c_void_p)
_fused = _sig("fused_moe", c_int32, _DP, c_void_p, c_void_p, c_void_p, c_void_p, _SP, c_void_p,
              c_void_p, c_size_t, c_void_p)
_host_io = _sig("fused_moe_host_io", c_int32, _DP, c_void_p, c_void_p, c_void_p, c_void_p, _SP,
                c_void_p, c_void_p, c_size_t, c_void_p)
_dev_status = _sig("fused_moe_get_device_status", c_int32, c_void_p, c_void_p)
_dbg = _sig("fused_moe_debug_scalars", c_int32, c_void_p, POINTER(c_float), POINTER(c_int32),
            c_void_p)
_launches = _sig("fused_moe_launches_per_call", c_int32, _DP)
_selftest_wait = _sig("fused_moe_selftest_wait", c_int32, c_void_p, c_size_t, ctypes.c_uint64,
                      c_void_p)
_static_ws = _sig("fused_moe_static_workspace", c_int32, _DP, c_void_p, c_void_p, c_void_p, c_void_p,
                  _SP, c_void_p, c_void_p, c_void_p)
_inv_rope = _sig("fused_inv_rope_fp8_quant_per_head", c_int32, POINTER(FmoeRopeDims), c_void_p,
                 c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p)
_profile = _sig("fused_moe_profile", c_int32, _DP, c_void_p, c_void_p, c_void_p, c_void_p, _SP,
                c_void_p, c_void_p, c_size_t, c_void_p, POINTER(c_float), POINTER(c_char_p),
                c_int32, POINTER(c_int32))


_tp_begin = _sig("fused_moe_tp_begin", c_int32, _DP, c_void_p, c_void_p, c_void_p, _SP, c_void_p,
                 c_void_p, c_size_t, c_void_p)
_tp_end = _sig("fused_moe_tp_end", c_int32, _DP, c_void_p, _SP, c_void_p, c_void_p, c_void_p,
               c_size_t, c_void_p)
_tp_finish = _sig("fused_moe_tp_finish", c_int32, ctypes.c_int64, c_void_p, c_void_p, c_void_p)


class FusedMoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_string(status)} ({status})")
        self.status = status


def abi_version() -> int:
    return int(_abi())


def status_string(status: int) -> str:
    return _status_string(int(status)).decode()


def _check(st: int, where: str) -> int:
    if st != FMOE_OK:
        raise FusedMoEError(st, where)
    return st


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def make_routing(n_group: int, topk_group: int, routed_scaling: float = 1.0,
                 bias: Optional[torch.Tensor] = None, n_shared: int = 0) -> FmoeRouting:
    """Group-limited sigmoid routing (DeepSeek-V3 style); bias: [E] fp32 device tensor;
    n_shared shared experts stored after the E routed ones."""
    r = FmoeRouting(FMOE_ROUTE_SIGMOID_GROUPED, n_group, topk_group, float(routed_scaling),
                    _ptr(bias), int(n_shared))
    r._bias_ref = bias  # keep the tensor alive with the descriptor
    return r


def make_softmax_routing(n_shared: int = 0) -> FmoeRouting:
    """Softmax top-k routing with n_shared shared experts after the E routed ones."""
    return FmoeRouting(FMOE_ROUTE_SOFTMAX, 0, 0, 1.0, None, int(n_shared))


def make_dims(T: int, H: int, I: int, E: int, top_k: int, fp8: bool, variant: str = "auto",
              routing: Optional[FmoeRouting] = None) -> FmoeDims:
    d = FmoeDims(T, H, I, E, top_k, FMOE_FP8_E4M3 if fp8 else FMOE_BF16, VARIANTS[variant],
                 ctypes.pointer(routing) if routing is not None else None)
    d._routing_ref = routing  # the C struct holds a raw pointer to it
    return d


def dims_of(x: torch.Tensor, router_w: torch.Tensor, w13: torch.Tensor, top_k: int,
            variant: str = "auto", routing: Optional[FmoeRouting] = None) -> FmoeDims:
    """Dims from x [T,H], router_w [E,H] and w13 [E+S,2I,H] (uint8 = e4m3 bytes, bfloat16 =
    bf16), where S = routing.n_shared shared experts follow the E routed ones."""
    T, H = x.shape
    E, H1 = router_w.shape
    EA, twoI, H2 = w13.shape
    n_shared = routing.n_shared if routing is not None else 0
    if H1 != H or H2 != H or twoI % 2 != 0:
        raise ValueError(f"shapes do not match: x {tuple(x.shape)}, router_w "
                         f"{tuple(router_w.shape)}, w13 {tuple(w13.shape)}")
    if EA != E + n_shared:
        raise ValueError(f"w13 holds {EA} experts, expected E + n_shared = {E + n_shared}")
    return make_dims(T, H, twoI // 2, E, top_k, w13.dtype == torch.uint8, variant, routing)


def make_scales(w13_scale=None, w2_scale=None, a1_scale: float = 0.0, a2_scale: float = 0.0) -> FmoeScales:
    return FmoeScales(_ptr(w13_scale), _ptr(w2_scale), float(a1_scale), float(a2_scale))


def workspace_size(dims: FmoeDims) -> int:
    return int(_ws_size(ctypes.byref(dims)))


def alloc_workspace(dims: FmoeDims, device="cuda") -> torch.Tensor:
    """A workspace tensor (uint8, 256-byte aligned by the caching allocator), initialised."""
    n = workspace_size(dims)
    if n == 0:
        raise FusedMoEError(FMOE_ERR_INVALID_ARG, "workspace_size")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    _check(_ws_init(ws.data_ptr(), n, _stream(None)), "fused_moe_workspace_init")
    return ws


def fused_moe_workspace_init(ws: torch.Tensor, stream=None) -> int:
    return _check(_ws_init(ws.data_ptr(), ws.numel(), _stream(stream)), "fused_moe_workspace_init")


def fused_moe_route(dims, x, router_w, topk_ids, topk_w, ws, stream=None, check=True) -> int:
    st = _route(ctypes.byref(dims), _ptr(x), _ptr(router_w), _ptr(topk_ids), _ptr(topk_w),
                _ptr(ws), ws.numel() if ws is not None else 0, _stream(stream))
    return _check(st, "fused_moe_route") if check else st


def fused_moe_permute(dims, topk_ids, x, scales, counts, offsets, sorted_rows, inv_perm, a_perm,
                      ws, stream=None, check=True) -> int:
    sp = ctypes.byref(scales) if scales is not None else None
    st = _permute(ctypes.byref(dims), _ptr(topk_ids), _ptr(x), sp, _ptr(counts), _ptr(offsets),
                  _ptr(sorted_rows), _ptr(inv_perm), _ptr(a_perm), _ptr(ws),
                  ws.numel() if ws is not None else 0, _stream(stream))
    return _check(st, "fused_moe_permute") if check else st


def fused_moe_experts(dims, a_perm, offsets, sorted_rows, topk_w, w13, w2, scales, y_perm, ws,
                      stream=None, check=True) -> int:
    sp = ctypes.byref(scales) if scales is not None else None
    st = _experts(ctypes.byref(dims), _ptr(a_perm), _ptr(offsets), _ptr(sorted_rows), _ptr(topk_w),
                  _ptr(w13), _ptr(w2), sp, _ptr(y_perm), _ptr(ws),
                  ws.numel() if ws is not None else 0, _stream(stream))
    return _check(st, "fused_moe_experts") if check else st


def fused_moe_combine(dims, y_perm, inv_perm, out, stream=None, check=True) -> int:
    st = _combine(ctypes.byref(dims), _ptr(y_perm), _ptr(inv_perm), _ptr(out), _stream(stream))
    return _check(st, "fused_moe_combine") if check else st


def fused_moe(dims, x, router_w, w13, w2, scales, out, ws, stream=None, check=True) -> int:
    sp = ctypes.byref(scales) if scales is not None else None
    st = _fused(ctypes.byref(dims), _ptr(x), _ptr(router_w), _ptr(w13), _ptr(w2), sp, _ptr(out),
                _ptr(ws), ws.numel() if ws is not None else 0, _stream(stream))
    return _check(st, "fused_moe") if check else st


def fused_moe_host_io(dims, x_host, router_w, w13, w2, scales, out_host, ws, stream=None,
                      check=True) -> int:
    sp = ctypes.byref(scales) if scales is not None else None
    st = _host_io(ctypes.byref(dims), _ptr(x_host), _ptr(router_w), _ptr(w13), _ptr(w2), sp,
                  _ptr(out_host), _ptr(ws), ws.numel() if ws is not None else 0, _stream(stream))
    return _check(st, "fused_moe_host_io") if check else st


def fused_moe_tp_begin(dims, x, router_w, w13, scales, amax_h, ws, stream=None, check=True) -> int:
    """Tensor-parallel shard, step 1: route, permute and the first contraction on this
    shard's w13; writes the shard's max |h| into amax_h (one fp32 device word)."""
    sp = ctypes.byref(scales) if scales is not None else None
    st = _tp_begin(ctypes.byref(dims), _ptr(x), _ptr(router_w), _ptr(w13), sp, _ptr(amax_h),
                   _ptr(ws), ws.numel() if ws is not None else 0, _stream(stream))
    return _check(st, "fused_moe_tp_begin") if check else st


def fused_moe_tp_end(dims, w2, scales, amax_h, out_partial, ws, stream=None, check=True) -> int:
    """Tensor-parallel shard, step 3: with amax_h holding the max over all shards, the
    second contraction and combine into this shard's fp32 partial output [T, H]."""
    sp = ctypes.byref(scales) if scales is not None else None
    st = _tp_end(ctypes.byref(dims), _ptr(w2), sp, _ptr(amax_h), _ptr(out_partial), _ptr(ws),
                 ws.numel() if ws is not None else 0, _stream(stream))
    return _check(st, "fused_moe_tp_end") if check else st


def fused_moe_tp_finish(out_sum, out, stream=None, check=True) -> int:
    """Tensor-parallel step 5: out (bf16) = round(out_sum (fp32)), element by element."""
    n = out_sum.numel() if out_sum is not None else 0
    st = _tp_finish(n, _ptr(out_sum), _ptr(out), _stream(stream))
    return _check(st, "fused_moe_tp_finish") if check else st


def fused_moe_get_device_status(ws, stream=None) -> int:
    return int(_dev_status(_ptr(ws), _stream(stream)))


def fused_moe_debug_scalars(ws, stream=None):
    """({amax_x, s1, inv1, amax_h, s2, inv2}, {n_chunks, split1, split2})."""
    f = (c_float * 6)()
    i = (c_int32 * 3)()
    _check(_dbg(_ptr(ws), f, i, _stream(stream)), "fused_moe_debug_scalars")
    names_f = ("amax_x", "s1", "inv1", "amax_h", "s2", "inv2")
    names_i = ("n_chunks", "split1", "split2")
    return dict(zip(names_f, list(f))), dict(zip(names_i, list(i)))


def fused_moe_static_workspace(dims, x, router_w, w13, w2, scales, out, device_status=None,
                               stream=None, check=True) -> int:
    """fused_moe without a caller workspace (library-owned 64 MiB device array)."""
    sp = ctypes.byref(scales) if scales is not None else None
    st = _static_ws(ctypes.byref(dims), _ptr(x), _ptr(router_w), _ptr(w13), _ptr(w2), sp,
                    _ptr(out), _ptr(device_status), _stream(stream))
    return _check(st, "fused_moe_static_workspace") if check else st


def fused_moe_selftest_wait(ws, budget_ns: int, stream=None, check=True) -> int:
    """A bounded wait that must run out (records FMOE_ERR_TIMEOUT in ws)."""
    st = _selftest_wait(_ptr(ws), ws.numel(), int(budget_ns), _stream(stream))
    return _check(st, "fused_moe_selftest_wait") if check else st


def fused_moe_launches_per_call(dims) -> int:
    return int(_launches(ctypes.byref(dims)))


def fused_moe_profile(dims, x, router_w, w13, w2, scales, out, ws, stream=None):
    """One fused_moe call with an event after every launch: [(kernel name, ms), ...]."""
    cap = 32
    ms = (c_float * cap)()
    names = (c_char_p * cap)()
    n = c_int32(0)
    sp = ctypes.byref(scales) if scales is not None else None
    _check(_profile(ctypes.byref(dims), _ptr(x), _ptr(router_w), _ptr(w13), _ptr(w2), sp,
                    _ptr(out), _ptr(ws), ws.numel(), _stream(stream), ms, names, cap,
                    ctypes.byref(n)), "fused_moe_profile")
    return [(names[i].decode(), float(ms[i])) for i in range(n.value)]


class FusedMoE:
    """The whole layer on device tensors, with its own workspace.

    x [T,H] bf16, router_w [E,H] bf16, w13 [E+S,2I,H] and w2 [E+S,H,I] as uint8 e4m3
    bytes (with w13_scale, w2_scale [E+S] fp32) or bf16, where S = w13.shape[0] - E
    shared experts follow the E routed ones.  routing: a descriptor from make_routing
    or make_softmax_routing (default: softmax with the S shared experts).
    Returns out [T,H] bf16."""

    def __init__(self, router_w, w13, w2, top_k, w13_scale=None, w2_scale=None,
                 a1_scale=0.0, a2_scale=0.0, variant="auto", routing=None):
        self.router_w, self.w13, self.w2 = router_w, w13, w2
        self.top_k, self.variant = top_k, variant
        self.w13_scale, self.w2_scale = w13_scale, w2_scale
        self.scales = make_scales(w13_scale, w2_scale, a1_scale, a2_scale)
        n_shared = w13.shape[0] - router_w.shape[0]
        if routing is None and n_shared > 0:
            routing = make_softmax_routing(n_shared)
        if n_shared != (routing.n_shared if routing is not None else 0):
            raise ValueError("w13 holds E + n_shared experts: n_shared must match the routing")
        self.routing = routing
        self._ws = {}

    def workspace(self, T: int) -> torch.Tensor:
        if T not in self._ws:
            self._ws[T] = alloc_workspace(self.dims(T), self.w13.device)
        return self._ws[T]

    def dims(self, T: int) -> FmoeDims:
        return make_dims(T, self.w13.shape[2], self.w13.shape[1] // 2, self.router_w.shape[0],
                         self.top_k, self.w13.dtype == torch.uint8, self.variant,
                         routing=self.routing)

    def __call__(self, x: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None):
        T = x.shape[0]
        if out is None:
            out = torch.empty(T, x.shape[1], dtype=torch.bfloat16, device=x.device)
        fused_moe(self.dims(T), x, self.router_w, self.w13, self.w2, self.scales, out,
                  self.workspace(T), stream)
        return out


def make_rope_dims(T: int, n_heads: int, head_dim: int, rot_dim: int, style: int = 0,
                   max_pos: int = 32768) -> FmoeRopeDims:
    return FmoeRopeDims(T, n_heads, head_dim, rot_dim, style, max_pos)


def fused_inv_rope_fp8_quant_per_head(dims: FmoeRopeDims, x, positions, cos_sin, q, scales,
                                      device_status=None, stream=None, check=True) -> int:
    """x [T,n_heads,head_dim] bf16, positions [T] int32, cos_sin [max_pos,rot_dim] fp32 ->
    q [T,n_heads,head_dim] uint8 (e4m3 codes), scales [T,n_heads] fp32 (device tensors)."""
    st = _inv_rope(ctypes.byref(dims), _ptr(x), _ptr(positions), _ptr(cos_sin), _ptr(q),
                   _ptr(scales), _ptr(device_status), _stream(stream))
    return _check(st, "fused_inv_rope_fp8_quant_per_head") if check else st


def moe(x: torch.Tensor, router_w: torch.Tensor, w13: torch.Tensor, w2: torch.Tensor, top_k: int,
        w13_scale=None, w2_scale=None, out: Optional[torch.Tensor] = None,
        routing: Optional[FmoeRouting] = None, a1_scale: float = 0.0, a2_scale: float = 0.0,
        variant: str = "auto", ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """The whole layer on device tensors in one call: dims from the shapes, a workspace
    allocated when none is given, out [T,H] bf16 allocated when none is given."""
    for name, t in (("x", x), ("router_w", router_w), ("w13", w13), ("w2", w2)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if x.dtype != torch.bfloat16 or router_w.dtype != torch.bfloat16:
        raise ValueError("x and router_w must be bfloat16")
    if w2.dtype != w13.dtype or w13.dtype not in (torch.uint8, torch.bfloat16):
        raise ValueError("w13 and w2 must both be uint8 (e4m3 bytes) or both bfloat16")
    dims = dims_of(x, router_w, w13, top_k, variant, routing)
    if ws is None:
        ws = alloc_workspace(dims, x.device)
    if out is None:
        out = torch.empty(x.shape[0], x.shape[1], dtype=torch.bfloat16, device=x.device)
    fused_moe(dims, x, router_w, w13, w2, make_scales(w13_scale, w2_scale, a1_scale, a2_scale),
              out, ws, stream)
    return out
