"""Host-only checks of the C ABI: the library loads, exports every symbol the header
declares, sizes workspaces, and rejects bad arguments with the documented status
codes before making any CUDA call (these tests run on machines without a GPU)."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fused_moe.h")

capi = pytest.importorskip("mixture_experts_layer_26_b200.capi",
                           reason="libfused_moe.so not built")


def header_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"FMOE_API\s+[\w\s\*]+?\b(fused_\w*)\s*\(", text)))


def test_header_symbols_are_exported():
    syms = header_symbols()
    assert len(syms) == 20
    assert set(syms) == set(capi.EXPORTED)
    lib = ctypes.CDLL(capi.LIB_PATH)
    for s in syms:
        assert hasattr(lib, s), s


def test_abi_version_and_strings():
    assert capi.abi_version() == 4
    for code, name in [(0, "FMOE_OK"), (1, "FMOE_ERR_INVALID_ARG"), (2, "FMOE_ERR_UNSUPPORTED"),
                       (3, "FMOE_ERR_WORKSPACE"), (4, "FMOE_ERR_CUDA"), (5, "FMOE_ERR_TIMEOUT"),
                       (6, "FMOE_ERR_DEVICE_BOUNDS")]:
        assert capi.status_string(code) == name


def dims(T=4, H=256, I=512, E=8, k=2, fp8=True, variant="auto"):
    return capi.make_dims(T, H, I, E, k, fp8, variant)


def test_workspace_size_valid_and_invalid():
    assert capi.workspace_size(dims()) > 0
    assert capi.workspace_size(dims(k=9)) == 0          # k > E
    assert capi.workspace_size(dims(H=128)) == 0        # H % 256
    assert capi.workspace_size(dims(I=100)) == 0        # I % 128
    assert capi.workspace_size(dims(E=257, k=2)) == 0   # E > 256
    assert capi.workspace_size(dims(T=-1)) == 0
    # bigger problems need more workspace; the normal variant needs no split partials
    assert capi.workspace_size(dims(T=64)) > capi.workspace_size(dims(T=4))
    big_sw = capi.workspace_size(dims(T=64, H=4096, I=14336, variant="swap_ab"))
    big_nm = capi.workspace_size(dims(T=64, H=4096, I=14336, variant="normal"))
    assert big_sw > big_nm
    # full-size workloads fit comfortably in HBM
    assert capi.workspace_size(dims(T=4096, H=4096, I=14336)) < (2 << 30)
    assert capi.workspace_size(dims(T=256, H=7168, I=2048, E=256, k=8)) < (1 << 30)


FAKE = 1 << 20   # 16-byte aligned fake device addresses; never dereferenced


class _T:
    """Stands in for a tensor: data_ptr() and numel() only."""

    def __init__(self, ptr, n=0):
        self.p, self.n = ptr, n

    def data_ptr(self):
        return self.p

    def numel(self):
        return self.n


def call_fused(d, x=FAKE, rw=FAKE, w13=FAKE, w2=FAKE, out=FAKE, ws=FAKE * 16, ws_bytes=None,
               scales=True):
    sc = capi.FmoeScales(FAKE, FAKE, 0.0, 0.0) if scales else None
    if ws_bytes is None:
        ws_bytes = capi.workspace_size(d) - 1           # always too small: no launch happens
    return capi.fused_moe(d, _T(x), _T(rw), _T(w13), _T(w2), sc, _T(out), _T(ws, ws_bytes),
                          stream=0, check=False)


def test_validation_codes_without_cuda():
    assert call_fused(dims(k=9)) == capi.FMOE_ERR_INVALID_ARG
    assert call_fused(dims(k=0)) == capi.FMOE_ERR_INVALID_ARG
    assert call_fused(dims(E=300)) == capi.FMOE_ERR_INVALID_ARG
    assert call_fused(dims(T=-3)) == capi.FMOE_ERR_INVALID_ARG
    assert call_fused(dims(H=384)) == capi.FMOE_ERR_UNSUPPORTED
    assert call_fused(dims(I=64)) == capi.FMOE_ERR_UNSUPPORTED
    assert call_fused(dims(H=16384 + 256)) == capi.FMOE_ERR_UNSUPPORTED
    bad_variant = dims()
    bad_variant.variant = 7
    assert call_fused(bad_variant) == capi.FMOE_ERR_INVALID_ARG
    bad_fmt = dims()
    bad_fmt.wdtype = 3
    assert call_fused(bad_fmt) == capi.FMOE_ERR_INVALID_ARG
    assert call_fused(dims(), x=0) == capi.FMOE_ERR_INVALID_ARG
    assert call_fused(dims(), out=0) == capi.FMOE_ERR_INVALID_ARG
    assert call_fused(dims(), x=FAKE + 8) == capi.FMOE_ERR_UNSUPPORTED      # not 16-byte aligned
    assert call_fused(dims(), scales=False) == capi.FMOE_ERR_INVALID_ARG   # FP8 needs scales
    assert call_fused(dims()) == capi.FMOE_ERR_WORKSPACE                   # one byte short
    assert call_fused(dims(), ws=FAKE * 16 + 128,
                      ws_bytes=1 << 40) == capi.FMOE_ERR_WORKSPACE          # ws not 256-aligned
    assert call_fused(dims(), ws=0, ws_bytes=1 << 40) == capi.FMOE_ERR_INVALID_ARG
    # bf16 weights need no scales; still stops at the workspace check
    assert call_fused(dims(fp8=False), scales=False) == capi.FMOE_ERR_WORKSPACE


def test_launch_counts():
    # small batch: router (+ permute, plan, gather), gemm1, finalize1 (swap-AB),
    # quant_h (FP8), gemm2, combine
    assert capi.fused_moe_launches_per_call(dims(T=4, variant="swap_ab")) == 6
    assert capi.fused_moe_launches_per_call(dims(T=4, variant="normal")) == 5
    assert capi.fused_moe_launches_per_call(dims(T=4, fp8=False, variant="swap_ab")) == 5
    assert capi.fused_moe_launches_per_call(dims(T=0)) == 0
    assert capi.fused_moe_launches_per_call(dims(k=9)) == -1
    # gathered rows above 128 KB: the gather is its own launch
    assert capi.fused_moe_launches_per_call(dims(T=256, E=8, k=2)) == 7
    # more than 2048 routed rows: permute and gather are their own launches (AUTO picks the
    # CTA pairs here, whose FP8 second contraction quantises h itself)
    assert capi.fused_moe_launches_per_call(dims(T=2048, E=8, k=2)) == 6
    assert capi.fused_moe_launches_per_call(dims(T=2048, E=8, k=2, variant="normal")) == 7
    # the CTA-pair kernels launch once per contraction like the one-CTA ones, and the FP8
    # second contraction quantises h itself (no quant_h launch)
    assert capi.fused_moe_launches_per_call(dims(T=4, variant="normal_pair")) == 4
    assert capi.fused_moe_launches_per_call(dims(T=2048, E=8, k=2, variant="normal_pair")) == 6
    assert capi.fused_moe_launches_per_call(dims(T=4, fp8=False, variant="normal_pair")) == 4


def test_shared_expert_validation_and_workspace():
    # n_shared outside 0..8 is rejected; shared experts add K = k + S slots per token
    for bad in (-1, 9):
        d = dims()
        r = capi.make_softmax_routing(bad)
        d = capi.make_dims(4, 256, 512, 8, 2, True, routing=r)
        assert call_fused(d) == capi.FMOE_ERR_INVALID_ARG
    base = capi.workspace_size(dims(T=64, H=4096, I=1024))
    r = capi.make_softmax_routing(1)
    with_shared = capi.workspace_size(capi.make_dims(64, 4096, 1024, 8, 2, True, routing=r))
    assert with_shared > base
    # same launch sequence with or without shared experts
    assert capi.fused_moe_launches_per_call(capi.make_dims(4, 256, 512, 8, 2, True, "swap_ab",
                                                           routing=r)) == 6
    # E + S may exceed 256 (DeepSeek-V3: 256 routed + 1 shared)
    g = capi.make_routing(8, 4, 2.5, None, n_shared=1)
    assert capi.workspace_size(capi.make_dims(16, 7168, 2048, 256, 8, True, routing=g)) > 0


def test_variant_choice_and_pair_workspace():
    # AUTO: <= 64 rows per expert on average -> swap-AB; 65..128 -> normal; above -> pairs.
    # Pair chunks hold 256 rows, so the workspace never grows over the one-CTA normal one,
    # and a forced variant outside AUTO's choice is still accepted.
    ws = capi.workspace_size
    assert ws(dims(T=4096, H=4096, I=1024, variant="normal_pair")) <= \
        ws(dims(T=4096, H=4096, I=1024, variant="normal"))
    for v in ("auto", "swap_ab", "normal", "normal_pair"):
        assert ws(dims(T=300, variant=v)) > 0
    bad = dims()
    bad.variant = 4
    assert call_fused(bad) == capi.FMOE_ERR_INVALID_ARG


def test_zero_tokens_is_a_noop():
    # T == 0 returns OK after the dims checks, even with null buffers, and launches nothing
    d = dims(T=0)
    assert capi.fused_moe(d, _T(0), _T(0), _T(0), _T(0), None, _T(0), _T(0, 0), stream=0,
                          check=False) == capi.FMOE_OK
    assert capi.fused_moe_route(d, _T(0), _T(0), _T(0), _T(0), _T(0, 0), stream=0,
                                check=False) == capi.FMOE_OK
    assert capi.fused_moe_combine(d, _T(0), _T(0), _T(0), stream=0, check=False) == capi.FMOE_OK


def test_step_validation():
    d = dims()
    small = _T(FAKE * 16, 10)
    assert capi.fused_moe_route(d, _T(FAKE), _T(0), _T(FAKE), _T(FAKE), small, stream=0,
                                check=False) == capi.FMOE_ERR_INVALID_ARG
    assert capi.fused_moe_route(d, _T(FAKE), _T(FAKE), _T(FAKE), _T(FAKE), small, stream=0,
                                check=False) == capi.FMOE_ERR_WORKSPACE
    assert capi.fused_moe_permute(d, _T(FAKE), _T(FAKE), None, _T(FAKE), _T(FAKE), _T(FAKE),
                                  _T(FAKE + 4), _T(FAKE), small, stream=0,
                                  check=False) == capi.FMOE_ERR_UNSUPPORTED
    assert capi.fused_moe_experts(d, _T(FAKE), _T(FAKE), _T(FAKE), _T(FAKE), _T(FAKE), _T(FAKE),
                                  None, _T(FAKE), small, stream=0,
                                  check=False) == capi.FMOE_ERR_INVALID_ARG    # FP8, no scales
    assert capi.fused_moe_combine(d, _T(FAKE), _T(0), _T(FAKE), stream=0,
                                  check=False) == capi.FMOE_ERR_INVALID_ARG


def test_routing_descriptor_validation():
    def grouped(n_group, topk_group, scaling=2.5, bias=None, k=8, E=64):
        r = capi.FmoeRouting(capi.FMOE_ROUTE_SIGMOID_GROUPED, n_group, topk_group, scaling, bias)
        return call_fused(capi.make_dims(4, 256, 512, E, k, True, routing=r))
    assert grouped(8, 4) == capi.FMOE_ERR_WORKSPACE          # valid: stops at the ws check
    assert grouped(8, 1) == capi.FMOE_ERR_WORKSPACE          # 1 group of 8 experts, k = 8: valid
    assert grouped(16, 1, k=8) == capi.FMOE_ERR_INVALID_ARG  # 1 group of 4 experts < k
    assert grouped(7, 2) == capi.FMOE_ERR_INVALID_ARG        # E % n_group != 0
    assert grouped(64, 8, k=2) == capi.FMOE_ERR_INVALID_ARG  # groups of 1 expert
    assert grouped(8, 9) == capi.FMOE_ERR_INVALID_ARG        # topk_group > n_group
    assert grouped(8, 4, scaling=0.0) == capi.FMOE_ERR_INVALID_ARG
    assert grouped(8, 4, bias=FAKE + 2) == capi.FMOE_ERR_UNSUPPORTED   # misaligned bias
    bad = capi.FmoeRouting(7, 1, 1, 1.0, None)
    assert call_fused(capi.make_dims(4, 256, 512, 8, 2, True, routing=bad)) == capi.FMOE_ERR_INVALID_ARG
    softmax = capi.FmoeRouting(capi.FMOE_ROUTE_SOFTMAX, 0, 0, 0.0, None)
    assert call_fused(capi.make_dims(4, 256, 512, 8, 2, True, routing=softmax)) == capi.FMOE_ERR_WORKSPACE


def test_inv_rope_validation_makes_no_cuda_call():
    # every rejection happens before any launch (fake pointers are never dereferenced)
    def call(**kw):
        args = dict(T=8, n_heads=4, head_dim=128, rot_dim=128, style=0, max_pos=64)
        args.update(kw)
        d = capi.make_rope_dims(**args)
        return capi.fused_inv_rope_fp8_quant_per_head(d, _T(FAKE), _T(FAKE), _T(FAKE), _T(FAKE),
                                                      _T(FAKE), None, stream=0, check=False)
    inv = capi.FMOE_ERR_INVALID_ARG
    assert call(head_dim=96) == inv                  # 64, 128 or 256 only
    assert call(rot_dim=4) == inv                    # at least 2 * head_dim / 32
    assert call(rot_dim=256) == inv                  # at most head_dim
    assert call(rot_dim=96) == inv                   # style 0: a power of two
    assert call(style=1, rot_dim=100) == inv         # style 1: a multiple of 2 * head_dim / 32
    assert call(style=2) == inv
    assert call(n_heads=0) == inv
    assert call(max_pos=0) == inv
    assert call(T=-1) == inv
    assert call(T=0) == capi.FMOE_OK                 # nothing to do, nothing launched
    d = capi.make_rope_dims(8, 4, 128, 128)
    assert capi.fused_inv_rope_fp8_quant_per_head(d, None, _T(FAKE), _T(FAKE), _T(FAKE), _T(FAKE),
                                                  None, stream=0, check=False) == inv
    assert capi.fused_inv_rope_fp8_quant_per_head(d, _T(FAKE + 8), _T(FAKE), _T(FAKE), _T(FAKE),
                                                  _T(FAKE), None, stream=0,
                                                  check=False) == capi.FMOE_ERR_UNSUPPORTED


def test_dims_from_tensor_shapes():
    import torch
    x = torch.empty(5, 256, dtype=torch.bfloat16)
    wr = torch.empty(8, 256, dtype=torch.bfloat16)
    w13 = torch.empty(9, 1024, 256, dtype=torch.uint8)      # 8 routed + 1 shared, I = 512
    r = capi.make_softmax_routing(1)
    d = capi.dims_of(x, wr, w13, 2, routing=r)
    assert (d.T, d.H, d.I, d.E, d.top_k, d.wdtype) == (5, 256, 512, 8, 2, capi.FMOE_FP8_E4M3)
    with pytest.raises(ValueError):
        capi.dims_of(x, wr, w13, 2)                          # a shared expert without routing
    with pytest.raises(ValueError):
        capi.dims_of(x, torch.empty(8, 128, dtype=torch.bfloat16), w13, 2, routing=r)


def test_tensor_level_call_rejects_bad_tensors_before_any_cuda_call():
    import torch
    x = torch.empty(5, 256, dtype=torch.bfloat16)      # CPU tensors: rejected up front
    wr = torch.empty(8, 256, dtype=torch.bfloat16)
    w13 = torch.empty(8, 1024, 256, dtype=torch.uint8)
    w2 = torch.empty(8, 256, 512, dtype=torch.uint8)
    with pytest.raises(ValueError):
        capi.moe(x, wr, w13, w2, 2)


def test_host_properties_over_many_dims():
    """Host-only properties over a grid of dims: the workspace holds at least the routed
    rows' buffers, the launch count follows the documented rule, invalid dims report
    size 0.  (The size is not monotone in T: the swap-AB variant also holds split-K
    partials, capped at 64 MB per contraction, which the normal variants do not.)"""
    import itertools
    rules = 0
    for (H, I), (E, k), fp8, variant, ns in itertools.product(
            [(256, 128), (4096, 1024), (7168, 2048)], [(8, 2), (64, 6), (256, 8)],
            [True, False], ["auto", "swap_ab", "normal", "normal_pair"], [0, 1]):
        r = capi.make_softmax_routing(ns) if ns else None
        for T in (1, 7, 64, 300, 2048):
            d = capi.make_dims(T, H, I, E, k, fp8, variant, routing=r)
            R = T * (k + ns)
            # at least the permuted activations, y and hq of every routed row
            es = 1 if fp8 else 2
            assert capi.workspace_size(d) >= R * H * (es + 4) + R * I * es
            # variant the library resolves for AUTO: <= 64 rows per expert on average ->
            # swap-AB, else the normal tiles (one CTA or pairs)
            avg = (R + E + ns - 1) // (E + ns)
            swap = variant == "swap_ab" or (variant == "auto" and avg <= 64)
            pair = variant == "normal_pair" or (variant == "auto" and avg > 128)
            # quant_h runs as its own launch in the FP8 format, except that the CTA-pair
            # second contraction quantises h itself
            n = 4 + (1 if fp8 and not pair else 0) + (1 if swap else 0)
            if R > 2048:
                n += 2
            elif R * H * 2 > 128 * 1024:
                n += 1
            assert capi.fused_moe_launches_per_call(d) == n, (T, H, I, E, k, fp8, variant, ns)
            rules += 1
    assert rules == 3 * 3 * 2 * 4 * 2 * 5
    for bad in (dict(E=257), dict(k=0), dict(H=300), dict(I=100)):
        kw = dict(T=4, H=256, I=128, E=8, k=2)
        kw.update(bad)
        assert capi.workspace_size(capi.make_dims(kw["T"], kw["H"], kw["I"], kw["E"], kw["k"], True)) == 0


def call_static(d, x=FAKE, rw=FAKE, w13=FAKE, w2=FAKE, out=FAKE, status=None, scales=True):
    sc = capi.FmoeScales(FAKE, FAKE, 0.0, 0.0) if scales else None
    return capi.fused_moe_static_workspace(d, _T(x), _T(rw), _T(w13), _T(w2), sc, _T(out),
                                           None if status is None else _T(status), stream=0,
                                           check=False)


def test_static_workspace_checks_arguments_before_any_cuda_call():
    """fused_moe_static_workspace returns fused_moe's own status codes for bad arguments,
    and the size limit, before any CUDA call: on a machine without a GPU every one of
    these returns its code instead of FMOE_ERR_CUDA."""
    assert call_static(dims(), x=0) == capi.FMOE_ERR_INVALID_ARG
    assert call_static(dims(), out=0) == capi.FMOE_ERR_INVALID_ARG
    assert call_static(dims(), w2=FAKE + 8) == capi.FMOE_ERR_UNSUPPORTED   # misaligned
    assert call_static(dims(), scales=False) == capi.FMOE_ERR_INVALID_ARG  # FP8 needs scales
    assert call_static(dims(k=9)) == capi.FMOE_ERR_INVALID_ARG
    assert call_static(dims(H=384)) == capi.FMOE_ERR_UNSUPPORTED           # H % 256 != 0
    assert call_static(dims(), status=FAKE + 2) == capi.FMOE_ERR_UNSUPPORTED
    # dims whose workspace exceeds the 64 MiB array (Mixtral-like FP8 decode at T = 64)
    big = dims(T=64, H=4096, I=14336)
    assert capi.workspace_size(big) > capi.STATIC_WS_BYTES
    assert call_static(big) == capi.FMOE_ERR_WORKSPACE
    assert call_static(dims(T=0)) == capi.FMOE_OK  # no tokens: nothing to do


@pytest.mark.skipif(capi is not None and __import__("torch").cuda.is_available(),
                    reason="checks the no-GPU behaviour")
def test_static_workspace_valid_arguments_reach_cuda():
    # valid arguments pass every check and only then meet the missing GPU
    assert call_static(dims()) == capi.FMOE_ERR_CUDA
