#!/usr/bin/env python3
"""Benchmark of the fused MoE layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload prefill_fp8] [--T 4096]

A step is one call of the whole layer (route -> permute/quantise -> both expert
contractions -> combine) through the C ABI on one batch of T tokens.  The default
workload is the largest single-GPU configuration: the FP8 prefill batch of T=4096 tokens
on Mixtral-like shapes (H=4096, I=14336, E=8, top_k=2), bound by the FP8 tensor pipe.
Inputs are seeded synthetic tensors resident in HBM; the expert weights (1.41 GB)
exceed the 126 MB L2, so no L2 flush is needed between steps.  W untimed warm-up steps,
then exactly K steps timed with CUDA events on the launching stream between a barrier +
synchronize on both sides; the time is the max over ranks.  For N > 1 every rank runs an
independent replica of the layer (the single-GPU layer has no exchange step) and `value`
is the tokens of all ranks divided by that time.

Rank 0 prints one JSON line.  Besides the contract keys it reports the roofline of
the dominant kernel (timed live per launch with CUDA events through
fused_moe_profile) against the burst peak of its bound (the FP8 tensor peak is measured
in the same run with the library GEMM, torch._scaled_mm on e4m3 operands), the oracle
timed on the host cores on a bounded sample (cpu_baseline, all cores and one core), an
end-to-end number through fused_moe_host_io with pinned host buffers, and the SM clocks
sampled with nvidia-smi from the timed region on.  With the default workload the line
also carries `decode`: the HBM-bound decode regime (Mixtral-like T=64, DeepSeek-V3-like
T=256), each measured the same way with its own roofline and end-to-end number.

--impl reference times the CPU oracle (the reference arm) on the same workload:
each step runs the oracle's expert networks for one (touched expert, block of
intermediate features) slice over all of that expert's rows; one cycle over the slices
plus routing and combine is one full layer pass.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from mixture_experts_layer_26_b200 import inputs as minp  # noqa: E402

METRIC = "fused-MoE tokens/s; achieved HBM GB/s (decode) / FP8 TFLOPS (prefill) vs peak"
DEFAULT_WORKLOAD = "prefill_fp8"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 2 ** 20
# sources whose hash an ncu summary of a GEMM kernel records (pair kernels: gemm_pair.cu)
GEMM_SOURCES = ("mixture_experts_layer_26_b200/csrc/gemm.cu",
                "mixture_experts_layer_26_b200/csrc/fmoe_common.cuh")
PAIR_GEMM_SOURCES = ("mixture_experts_layer_26_b200/csrc/gemm_pair.cu",
                     "mixture_experts_layer_26_b200/csrc/fmoe_common.cuh")


# --------------------------------------------------------------------------- helpers

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def gemm_source_hash(kernel: str = "") -> str:
    h = hashlib.sha256()
    srcs = ROPE_SOURCES if "rope" in kernel else (PAIR_GEMM_SOURCES if "pair" in kernel
                                                   else GEMM_SOURCES)
    for rel in srcs:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload_tag: str):
    """DRAM bytes per launch of `kernel` from a committed ncu summary, if it was taken
    on the current kernel source (profiles/*.md lines 'traffic_bytes_per_launch' and
    'source_hash'); else None."""
    pdir = os.path.join(ROOT, "profiles")
    if not os.path.isdir(pdir):
        return None
    # the workload tag must be whole: "..._T1" must not match a summary of "..._T16"
    tag = re.compile(re.escape(workload_tag) + r"(?=[._])")
    for name in sorted(os.listdir(pdir)):
        if not (name.startswith(kernel) and tag.search(name) and name.endswith(".md")):
            continue
        text = open(os.path.join(pdir, name)).read()
        t = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
        hsh = re.search(r"source_hash:\s*([0-9a-f]+)", text)
        if t and hsh and hsh.group(1) == gemm_source_hash(kernel):
            return float(t.group(1))
    return None


class ClockSampler:
    """nvidia-smi samples (200 ms) of the GPU with the given PCI bus id."""

    FIELDS = ("pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, props):
        # nvidia-smi prints the bus id as DDDDDDDD:BB:DD.F
        self.bus_id = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9 or not self._match(parts[0]):
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}

    def _match(self, bus: str) -> bool:
        return bus.lower()[-7:] == self.bus_id[-7:]


def blas_threads() -> int:
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max([i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"] or [1])
    except Exception:
        return 1


def np_inputs(inp: minp.MoEInputs):
    fp8 = inp.shape.wdtype == "fp8"
    wb = (lambda t: t.numpy()) if fp8 else minp.bf16_bits
    return dict(x_bits=minp.bf16_bits(inp.x), wr_bits=minp.bf16_bits(inp.router_w),
                w13=wb(inp.w13), w2=wb(inp.w2),
                w13_scale=None if inp.w13_scale is None else inp.w13_scale.numpy(),
                w2_scale=None if inp.w2_scale is None else inp.w2_scale.numpy(), fp8=fp8)


def oracle_grouped(inp: minp.MoEInputs):
    """The oracle's grouped-routing arguments for these inputs (None: softmax)."""
    s = inp.shape
    if s.grouped is None:
        return None
    return dict(n_group=s.grouped[0], topk_group=s.grouped[1], routed_scaling=s.grouped[2],
                bias=inp.router_bias.numpy())


def routing_desc(inp: minp.MoEInputs, device):
    """The C-ABI routing descriptor of these inputs (None: softmax, no shared experts)."""
    from mixture_experts_layer_26_b200 import capi
    s = inp.shape
    if s.grouped is not None:
        return capi.make_routing(*s.grouped, inp.router_bias.to(device), n_shared=s.n_shared)
    if s.n_shared:
        return capi.make_softmax_routing(s.n_shared)
    return None


def reduce_max(dist, v: float, device) -> float:
    """Max of a per-rank scalar over all ranks (identity without a process group)."""
    if dist is None:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def tokens_per_second(world: int, T: int, steps: int, ms_max: float) -> float:
    """Whole-job throughput: every rank processes T tokens per step."""
    return world * T * steps / (ms_max / 1e3)


# --------------------------------------------------------------------------- CPU oracle timing

class OracleSlices:
    """Bounded steps of the oracle.  A step runs the oracle's expert networks for one
    touched expert over all of its rows, restricted to a block of F intermediate features
    (the gate/up rows and the w2 columns of those features: the same computation on a
    narrower expert); F is chosen so that a step costs a few tens of milliseconds.  The
    layer is all (expert, feature block) slices plus routing, permutation and combine,
    which are timed once."""

    WORK_PER_STEP = 384e6  # weight elements decoded + row x weight products, per step

    def __init__(self, inp):
        from oracle import fused_moe_oracle as O
        self.O, self.inp, self.d = O, inp, np_inputs(inp)
        s = inp.shape
        t0 = time.perf_counter()
        d = self.d
        grouped = oracle_grouped(inp)
        if grouped is None:
            ids, w, _ = O.router(d["x_bits"], d["wr_bits"], s.top_k)
        else:
            ids, w, _, _ = O.router_grouped(d["x_bits"], d["wr_bits"], s.top_k, **grouped)
        ids, w = O.append_shared(ids, w, s.E, s.n_shared)
        K = s.top_k + s.n_shared
        counts, offsets, rows, inv = O.permute(ids, s.E_all)
        a_perm, s1, _, _ = O.permute_quant(d["x_bits"], rows, K, d["fp8"])
        self.prep = (ids, w, counts, offsets, rows, inv, a_perm, s1)
        self.fixed_s = time.perf_counter() - t0
        self.touched = [e for e in range(s.E_all) if counts[e] > 0]
        # feature blocks: (expert, f0, f1), F a multiple of 64 dividing into I
        self.slices = []
        for e in self.touched:
            n = int(counts[e])
            F = int(self.WORK_PER_STEP / (3.0 * s.H * (n + 64)))
            F = max(64, min(s.I, F // 64 * 64))
            self.slices += [(e, f0, min(s.I, f0 + F)) for f0 in range(0, s.I, F)]
        self.i = 0

    def step(self):
        s, d, O = self.inp.shape, self.d, self.O
        ids, w, counts, offsets, rows, inv, a_perm, s1 = self.prep
        e, f0, f1 = self.slices[self.i % len(self.slices)]
        self.i += 1
        r0, r1 = offsets[e], offsets[e + 1]
        offs = np.zeros(2, dtype=offsets.dtype)
        offs[1] = r1 - r0
        w13 = d["w13"][e:e + 1]
        w13 = np.concatenate([w13[:, f0:f1], w13[:, s.I + f0:s.I + f1]], axis=1)
        w2 = d["w2"][e:e + 1, :, f0:f1]
        sc13 = None if d["w13_scale"] is None else d["w13_scale"][e:e + 1]
        sc2 = None if d["w2_scale"] is None else d["w2_scale"][e:e + 1]
        return e, O.experts(a_perm[r0:r1], offs, rows[r0:r1], w, w13, w2, s.H, f1 - f0, 1,
                            d["fp8"], s1, sc13, sc2)[0]

    def combine_seconds(self):
        s = self.inp.shape
        y = np.zeros((s.R, s.H))
        t0 = time.perf_counter()
        self.O.combine(y, self.prep[5], s.T, s.top_k + s.n_shared)
        return time.perf_counter() - t0


def run_reference(args, rank):
    if rank != 0:
        return 0
    s = minp.shape(args.workload, args.T)
    inp = minp.make_inputs(s, seed=0)
    sl = OracleSlices(inp)
    warm = min(args.warmup, 2)  # the oracle has no caches to warm beyond BLAS thread start-up
    for _ in range(warm):
        sl.step()
    sl.i = 0
    t0 = time.perf_counter()
    for _ in range(args.steps):
        sl.step()
    dt = time.perf_counter() - t0
    cycles = args.steps / len(sl.slices)  # layers' worth of expert work timed
    total = dt + cycles * (sl.fixed_s + sl.combine_seconds())
    value = s.T * cycles / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp64 (oracle; e4m3 codes decoded exactly)",
        "data": "synthetic", "config": workload_config(s), "variant": "oracle",
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(),
                         "kind": "oracle", "cores_available": len(os.sched_getaffinity(0)),
                         "sample": f"{args.steps} steps, each the expert networks of one "
                                   f"(touched expert, block of intermediate features) slice, "
                                   f"{len(sl.slices)} slices per layer over "
                                   f"{len(sl.touched)} touched experts and all T={s.T} tokens; "
                                   "routing/permutation/combine added once per layer; "
                                   f"{warm} of the {args.warmup} warm-up steps executed"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# --------------------------------------------------------------------------- GPU arm

# Decode workloads measured beside the default (prefill) workload in the same run, so one
# line covers both regimes of the metric: HBM-bound decode and tensor-bound prefill.
EXTRA_WORKLOADS = (("mixtral_fp8_decode", 64), ("dsv3_fp8_decode", 256))


def workload_config(s):
    weights = 3 * s.H * s.I * s.E_all * (1 if s.wdtype == "fp8" else 2)
    routing = "softmax top-k" if s.grouped is None else \
        (f"grouped sigmoid: {s.grouped[0]} groups, {s.grouped[1]} kept, "
         f"routed scaling {s.grouped[2]}, selection bias")
    shared = f" + {s.n_shared} shared" if s.n_shared else ""
    return {"workload": f"{s.name}: H={s.H} I={s.I} E={s.E}{shared} top_k={s.top_k} T={s.T} "
                        f"({s.wdtype} weights)",
            "T": s.T, "H": s.H, "I": s.I, "E": s.E, "top_k": s.top_k, "n_shared": s.n_shared,
            "routing": routing,
            "l2": f"inputs larger than L2: expert weights {weights / 1e9:.2f} GB vs "
                  f"{L2_BYTES / 2 ** 20:.0f} MB L2, no flush",
            "parallelism": "replicas (one independent layer per GPU)"}


class Layer:
    """Device tensors, descriptors and workspace of one workload."""

    def __init__(self, s, dev, variant="auto", weights_on_device=False):
        from mixture_experts_layer_26_b200 import capi
        self.s, self.dev = s, dev
        self.fp8 = s.wdtype == "fp8"
        if weights_on_device:
            # measurement only: the same distributions and per-expert quantisation drawn
            # by the device's generator (the CPU draw of 11 GB takes about a minute)
            x, wr = minp.make_activations(s, seed=0)
            w13, w2, s13, s2 = minp.make_weights(s, seed=0, device=dev)
            bias = minp.make_router_bias(s, seed=0)
            self.inp = minp.MoEInputs(s, x, wr, w13, w2, s13, s2, bias)
            self.weights_drawn = "on the device (torch CUDA generator, seed 0)"
        else:
            self.inp = minp.make_inputs(s, seed=0)
            self.weights_drawn = "on the host (torch CPU generator, seed 0)"
        inp = self.inp
        self.x = inp.x.to(dev)
        self.wr = inp.router_w.to(dev)
        self.w13, self.w2 = inp.w13.to(dev), inp.w2.to(dev)
        self.s13 = inp.w13_scale.to(dev) if self.fp8 else None
        self.s2 = inp.w2_scale.to(dev) if self.fp8 else None
        self.routing = routing_desc(inp, dev)
        self.dims = capi.make_dims(s.T, s.H, s.I, s.E, s.top_k, self.fp8, variant,
                                   routing=self.routing)
        self.ws = capi.alloc_workspace(self.dims, dev)
        self.sc = capi.make_scales(self.s13, self.s2)
        self.out = torch.empty(s.T, s.H, dtype=torch.bfloat16, device=dev)

    def call(self, stream):
        from mixture_experts_layer_26_b200 import capi
        capi.fused_moe(self.dims, self.x, self.wr, self.w13, self.w2, self.sc, self.out,
                       self.ws, stream)

    def release(self):
        for name in ("x", "wr", "w13", "w2", "s13", "s2", "ws", "out"):
            setattr(self, name, None)
        if self.inp is not None and self.inp.w13.is_cuda:
            self.inp = None


def measure_layer(L: Layer, args, dist, rank, world, dev, sample_clocks=True):
    """Warm-up, exactly K timed steps (CUDA events on the launching stream, max over
    ranks), then per-call events, a CUDA-graph replay, per-kernel events and the end-to-end
    host-buffer call.  Returns the measured numbers (rank 0 reads them)."""
    from mixture_experts_layer_26_b200 import capi
    s = L.s
    stream = torch.cuda.current_stream(dev)

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(args.warmup):
        L.call(stream)
    torch.cuda.synchronize()
    assert capi.fused_moe_get_device_status(L.ws, stream) == capi.FMOE_OK

    # ---- timed region: exactly K steps.  The clock sampler runs from here through the
    # per-call and per-kernel loops of the same workload (short timed regions would
    # otherwise see one or two samples).
    barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(torch.cuda.get_device_properties(dev)) \
        if (rank == 0 and sample_clocks) else None
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        L.call(stream)
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = reduce_max(dist, ev0.elapsed_time(ev1), dev)
    status = capi.fused_moe_get_device_status(L.ws, stream)
    assert status == capi.FMOE_OK, capi.status_string(status)

    # ---- per-call distribution (events around every call) and a CUDA-graph replay of the
    # same call; both after the timed region, neither feeds `value`
    n_calls = max(5, min(args.steps, 200))
    call_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n_calls)]
    for c0, c1 in call_ev:
        c0.record(stream)
        L.call(stream)
        c1.record(stream)
    torch.cuda.synchronize()
    per_call = sorted(c0.elapsed_time(c1) for c0, c1 in call_ev)
    graph_ms = None
    try:
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            L.call(side)  # warm-up on the side stream
        stream.wait_stream(side)
        with torch.cuda.graph(g, stream=side):
            L.call(side)
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        r0.record(stream)
        for _ in range(n_calls):
            g.replay()
        r1.record(stream)
        torch.cuda.synchronize()
        graph_ms = r0.elapsed_time(r1) / n_calls
        del g
    except RuntimeError as exc:  # capture unsupported in this environment: report, go on
        print(f"graph replay skipped: {exc}", file=sys.stderr)
    assert capi.fused_moe_get_device_status(L.ws, stream) == capi.FMOE_OK

    # ---- per-kernel times (events after every launch), same inputs, after the timed region
    nprof = max(5, min(args.steps, 200))
    per = {}
    for _ in range(nprof):
        for name, t in capi.fused_moe_profile(L.dims, L.x, L.wr, L.w13, L.w2, L.sc, L.out,
                                              L.ws, stream):
            per.setdefault(name, []).append(t)
    kern_ms = {k: statistics.mean(v) for k, v in per.items()}
    clocks = sampler.stop() if sampler is not None else None
    _, plan = capi.fused_moe_debug_scalars(L.ws, stream)

    # ---- end to end through the host-buffer entry point
    x_host = L.inp.x.clone().pin_memory()
    out_host = torch.empty(s.T, s.H, dtype=torch.bfloat16).pin_memory()
    n_e2e = max(3, min(args.steps, 500))
    for _ in range(3):
        capi.fused_moe_host_io(L.dims, x_host, L.wr, L.w13, L.w2, L.sc, out_host, L.ws, stream)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n_e2e):
        capi.fused_moe_host_io(L.dims, x_host, L.wr, L.w13, L.w2, L.sc, out_host, L.ws, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = reduce_max(dist, e0.elapsed_time(e1), dev)

    # ---- experts the batch touched, from the GPU routing + permutation steps
    R = s.R
    ids_d = torch.empty(R, dtype=torch.int32, device=dev)
    tw_d = torch.empty(R, dtype=torch.float32, device=dev)
    counts_d = torch.empty(s.E_all, dtype=torch.int32, device=dev)
    offs_d = torch.empty(s.E_all + 1, dtype=torch.int32, device=dev)
    rows_d = torch.empty(R, dtype=torch.int32, device=dev)
    inv_d = torch.empty(R, dtype=torch.int32, device=dev)
    aperm_d = torch.empty(R, s.H, dtype=torch.uint8 if L.fp8 else torch.bfloat16, device=dev)
    capi.fused_moe_route(L.dims, L.x, L.wr, ids_d, tw_d, L.ws, stream)
    capi.fused_moe_permute(L.dims, ids_d, L.x, L.sc, counts_d, offs_d, rows_d, inv_d, aperm_d,
                           L.ws, stream)
    touched = int((counts_d > 0).sum().item())
    max_rows = int(counts_d.max().item())
    return dict(ms=ms, ms_step=ms / args.steps, value=tokens_per_second(world, s.T, args.steps, ms),
                per_call=per_call, n_calls=n_calls, graph_ms=graph_ms, kern_ms=kern_ms,
                plan=plan, clocks=clocks, e2e_value=tokens_per_second(world, s.T, n_e2e, e2e_ms),
                touched=touched, max_rows=max_rows,
                launches=capi.fused_moe_launches_per_call(L.dims) * args.steps)


def fp8_peak_probe(dev, burst_iters=10, sustained_s=4.0, n=8192):
    """The FP8 dense tensor peak of this GPU, measured with the library GEMM:
    torch._scaled_mm on e4m3 operands (n x n x n, unit scales, bf16 out).  Burst: the best
    of `burst_iters` individually timed calls after warm-up.  Sustained: back-to-back calls
    for about `sustained_s` seconds (the power cap settles in).  Returns TFLOP/s figures."""
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    a = torch.randn(n, n, device=dev, generator=g).to(torch.float8_e4m3fn)
    b = torch.randn(n, n, device=dev, generator=g).to(torch.float8_e4m3fn).t()  # column-major
    one = torch.ones((), device=dev, dtype=torch.float32)
    flops = 2.0 * n * n * n

    def mm():
        return torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)

    for _ in range(5):
        mm()
    torch.cuda.synchronize()
    best = float("inf")
    for _ in range(burst_iters):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        mm()
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    # sustained: batches of 50 calls until the time is spent
    total_ms, calls = 0.0, 0
    t_end = time.perf_counter() + sustained_s
    while time.perf_counter() < t_end:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(50):
            mm()
        e1.record()
        torch.cuda.synchronize()
        total_ms += e0.elapsed_time(e1)
        calls += 50
    del a, b
    return {"burst_tflops": round(flops / (best / 1e3) / 1e12, 1),
            "sustained_tflops": round(flops * calls / (total_ms / 1e3) / 1e12, 1),
            "how": f"torch._scaled_mm e4m3 {n}x{n}x{n}, unit per-tensor scales, bf16 out; "
                   f"burst = best of {burst_iters} timed calls, sustained = {calls} "
                   f"back-to-back calls over {total_ms / 1e3:.1f} s"}


def tensor_peak(fp8: bool, peaks, peak_kind, probe):
    """(TFLOP/s, description) of the burst tensor peak for a contraction timed per launch."""
    if fp8 and "fp8_tflops" in peaks:
        return float(peaks["fp8_tflops"]), f"{peak_kind}: MEASURED_PEAKS.json fp8_tflops (burst)"
    if fp8 and probe is not None:
        return probe["burst_tflops"], "measured in this run: FP8 burst (" + probe["how"] + ")"
    if fp8:
        return 2.0 * peaks["bf16_tflops"], (f"{peak_kind}: 2 x bf16_tflops (burst), the nominal "
                                            "dense FP8/bf16 ratio 4.5/2.25 (no FP8 probe)")
    return float(peaks["bf16_tflops"]), f"{peak_kind}: bf16_tflops (burst)"


def roofline_of(s, m, peaks, peak_kind, probe, args_workload):
    """Roofline of the dominant kernel plus the step's HBM and tensor figures."""
    kern_ms = m["kern_ms"]
    esz = 1 if s.wdtype == "fp8" else 2
    fp8 = s.wdtype == "fp8"
    dom = max(kern_ms, key=kern_ms.get)
    names = "".join(kern_ms)
    variant = "swap_ab" if "swapab" in names else ("normal_pair" if "pair" in names else "normal")
    touched = m["touched"]
    gemm1_bytes = touched * 2 * s.H * s.I * esz          # weights of the touched experts
    gemm2_bytes = touched * s.H * s.I * esz
    gemm1_flops = 4.0 * s.R * s.H * s.I                  # gate and up: 2 x (2 R H I)
    gemm2_flops = 2.0 * s.R * s.H * s.I
    kind = dom.split("_")[0]
    roof = None
    traffic = profiled_traffic(dom, f"{args_workload}_T{s.T}")
    if variant == "swap_ab" and kind in ("gemm1", "gemm2"):
        dom_bytes = gemm1_bytes if kind == "gemm1" else gemm2_bytes
        ach = dom_bytes / (kern_ms[dom] / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(ach / peaks["hbm_gbs"], 4), "traffic": traffic,
                "kernel": dom, "kernel_us": round(1e3 * kern_ms[dom], 2),
                "algorithmic_bytes": dom_bytes,
                "peak_kind": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs, copy stream)"
                             if peak_kind == "measured" else
                             "fallback 6650 GB/s (no MEASURED_PEAKS.json)"}
    elif kind in ("gemm1", "gemm2"):
        dom_flops = gemm1_flops if kind == "gemm1" else gemm2_flops
        # a contraction timed per launch (events around it): the burst peak of its dtype
        peak, how = tensor_peak(fp8, peaks, peak_kind, probe)
        ach = dom_flops / (kern_ms[dom] / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": round(ach, 1), "peak": round(peak, 1),
                "unit": "TFLOP/s", "frac": round(ach / peak, 4), "traffic": traffic,
                "kernel": dom, "kernel_us": round(1e3 * kern_ms[dom], 2),
                "algorithmic_flops": dom_flops, "peak_kind": how}
    step_weight_bytes = gemm1_bytes + gemm2_bytes
    step_flops = gemm1_flops + gemm2_flops
    ms_step = m["ms_step"]
    step_hbm = {"weight_bytes": step_weight_bytes,
                "achieved_gbs": round(step_weight_bytes / (ms_step / 1e3) / 1e9, 1),
                "frac": round(step_weight_bytes / (ms_step / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
                "touched_experts": touched, "max_rows_per_expert": m["max_rows"]}
    ach_t = step_flops / (ms_step / 1e3) / 1e12
    peak_t, how_t = tensor_peak(fp8, peaks, peak_kind, probe)
    step_tensor = {"flops": step_flops, "achieved_tflops": round(ach_t, 1),
                   "frac": round(ach_t / peak_t, 4), "peak_tflops": round(peak_t, 1),
                   "peak_kind": how_t}
    return variant, roof, step_hbm, step_tensor


def cpu_baseline_sample(inp, budget_s: float):
    """The oracle as it stands on a bounded sample of the workload, on all host cores the
    process may use and on one core: the routing, permutation and combine once, then
    (touched expert, feature block) slices of the expert networks for about `budget_s`
    seconds per setting, extrapolated to the whole layer (all slices)."""
    import threadpoolctl
    cores = len(os.sched_getaffinity(0))
    res = {}
    for label, limit in (("all", cores), ("one", 1)):
        with threadpoolctl.threadpool_limits(limit, user_api="blas"):
            sl = OracleSlices(inp)
            sl.step()  # BLAS thread start-up
            sl.i = 0
            n, t0 = 0, time.perf_counter()
            while (time.perf_counter() - t0 < budget_s or n == 0) and n < len(sl.slices):
                sl.step()
                n += 1
            dt = time.perf_counter() - t0
            layer_s = sl.fixed_s + sl.combine_seconds() + dt / n * len(sl.slices)
            res[label] = (inp.shape.T / layer_s, n, len(sl.slices), layer_s, blas_threads())
    v, n, total, layer_s, threads = res["all"]
    v1, n1, _, layer_s1, _ = res["one"]
    return {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "cores_available": cores, "value_1core": v1,
            "sample": f"routing, permutation and combine of the T={inp.shape.T} batch once, then "
                      f"{n} of the {total} (touched expert, feature block) slices of the expert "
                      f"networks timed on {threads} BLAS threads ({n1} on 1 core), extrapolated "
                      f"to all slices: one layer = {layer_s:.1f} s ({layer_s1:.1f} s on 1 core)"}


def run_ours(args, rank, world, local_rank):
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    s = minp.shape(args.workload, args.T)
    L = Layer(s, dev, args.variant, weights_on_device=s.E_all * s.H * s.I > 2 ** 31)
    m = measure_layer(L, args, dist, rank, world, dev)

    # decode regimes beside the default prefill workload, measured the same way
    extras = []
    if args.workload == DEFAULT_WORKLOAD and args.T in (None, minp.shape(DEFAULT_WORKLOAD).T) \
            and not args.no_extras:
        L.release()
        torch.cuda.empty_cache()
        for wl, T in EXTRA_WORKLOADS:
            se = minp.shape(wl, T)
            Le = Layer(se, dev, "auto", weights_on_device=se.E_all * se.H * se.I > 2 ** 31)
            me = measure_layer(Le, args, dist, rank, world, dev)
            extras.append((se, Le.weights_drawn, me))
            Le.release()
            torch.cuda.empty_cache()

    # the FP8 tensor peak of this GPU (after the timed regions, so that they do not run on
    # a GPU the probe has just heated)
    probe = fp8_peak_probe(dev) if (rank == 0 and not args.no_peak_probe) else None

    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks, peak_kind = load_peaks()
    variant, roof, step_hbm, step_tensor = roofline_of(s, m, peaks, peak_kind, probe,
                                                       args.workload)
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        inp = L.inp
        if inp.w13.is_cuda:  # weights drawn on the device: the oracle reads host copies
            inp = minp.MoEInputs(s, inp.x, inp.router_w, inp.w13.cpu(), inp.w2.cpu(), inp.w13_scale,
                                 inp.w2_scale, inp.router_bias)
        cpu = cpu_baseline_sample(inp, args.cpu_budget)
    fp8 = s.wdtype == "fp8"
    line = {
        "metric": METRIC, "value": round(m["value"], 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(m["ms_step"], 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp8_e4m3 (fp32 accumulate)" if fp8 else "bf16 (fp32 accumulate)",
        "data": "synthetic (seeded; N(0,1) x, N(0,1/sqrt(fan_in)) weights, per-expert e4m3 scales)",
        "config": workload_config(s),
        "variant": variant,
        "roofline": roof,
        "step_hbm": step_hbm,
        "step_tensor": step_tensor,
        "kernels_us": {k: round(1e3 * v, 2) for k, v in m["kern_ms"].items()},
        "plan": m["plan"],
        "cpu_baseline": cpu,
        "e2e": {"value": round(m["e2e_value"], 1), "unit": "tokens/s",
                "h2d_bytes_per_step": s.T * s.H * 2, "d2h_bytes_per_step": s.T * s.H * 2,
                "api": "fused_moe_host_io (pinned host x and out)"},
        "gpu_launches": m["launches"],
        "clocks": m["clocks"],
        "per_call_ms": {"calls": m["n_calls"], "median": round(statistics.median(m["per_call"]), 5),
                        "p95": round(m["per_call"][min(m["n_calls"] - 1, int(0.95 * m["n_calls"]))], 5),
                        "note": "events around each call, after the timed region"},
        "graph_replay_ms_per_call": None if m["graph_ms"] is None else round(m["graph_ms"], 5),
        "fp8_peak_probe": probe,
        "hbm_peak": {"gbs": peaks["hbm_gbs"], "kind": peak_kind},
    }
    if extras:
        line["decode"] = []
        for se, drawn, me in extras:
            v_e, roof_e, hbm_e, ten_e = roofline_of(se, me, peaks, peak_kind, probe, se.name)
            line["decode"].append({
                "config": workload_config(se), "weights_drawn": drawn, "variant": v_e,
                "value": round(me["value"], 1), "unit": "tokens/s", "steps": args.steps,
                "ms_per_step": round(me["ms_step"], 5), "roofline": roof_e, "step_hbm": hbm_e,
                "step_tensor": ten_e,
                "kernels_us": {k: round(1e3 * v, 2) for k, v in me["kern_ms"].items()},
                "e2e": {"value": round(me["e2e_value"], 1), "unit": "tokens/s",
                        "h2d_bytes_per_step": se.T * se.H * 2,
                        "d2h_bytes_per_step": se.T * se.H * 2,
                        "api": "fused_moe_host_io (pinned host x and out)"},
                "gpu_launches": me["launches"], "clocks": me["clocks"],
                "per_call_ms": {"median": round(statistics.median(me["per_call"]), 5)},
                "graph_replay_ms_per_call": None if me["graph_ms"] is None else round(me["graph_ms"], 5),
            })
    print(json.dumps(line))
    return 0


def run_route_only(args, rank, world, local_rank):
    """`--step route`: the routing step alone (fused_moe_route: the router kernel and its
    tail) on the workload's x and router_w, back to back; no expert weights are allocated,
    so the run is small enough for a detailed profile of the router.  Prints one line with
    the mean time per call."""
    from mixture_experts_layer_26_b200 import capi
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    s = minp.shape(args.workload, args.T)
    x, wr = minp.make_activations(s, seed=0)
    bias = minp.make_router_bias(s, seed=0)
    routing = None
    if s.grouped is not None:
        routing = capi.make_routing(*s.grouped, bias.to(dev), n_shared=s.n_shared)
    elif s.n_shared:
        routing = capi.make_softmax_routing(s.n_shared)
    dims = capi.make_dims(s.T, s.H, s.I, s.E, s.top_k, s.wdtype == "fp8", routing=routing)
    ws = capi.alloc_workspace(dims, dev)
    ids = torch.empty(s.R, dtype=torch.int32, device=dev)
    tw = torch.empty(s.R, dtype=torch.float32, device=dev)
    xd, wd = x.to(dev), wr.to(dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        capi.fused_moe_route(dims, xd, wd, ids, tw, ws, stream)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        capi.fused_moe_route(dims, xd, wd, ids, tw, ws, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    assert capi.fused_moe_get_device_status(ws, stream) == capi.FMOE_OK
    us = 1e3 * e0.elapsed_time(e1) / args.steps
    if rank == 0:
        print(json.dumps({"step": "route", "workload": workload_config(s)["workload"],
                          "us_per_call": round(us, 2), "calls": args.steps,
                          "fmas": s.T * s.E * s.H, "tokens_per_s": round(s.T / (us / 1e6), 1)}))
    return 0


def run_tp_ours(args, rank, world, local_rank):
    """Tensor parallelism over the intermediate features: rank r of N holds shard r of
    every expert and the N ranks compute ONE batch together (strong scaling).  A step is
    one layer call: begin (route, permute, first contraction), all-reduce MAX of max |h|,
    end (second contraction, fp32 partial output), all-reduce SUM of the partial outputs,
    finish (bf16).  With N = 1 the collectives are skipped (a group of one)."""
    from mixture_experts_layer_26_b200 import capi, tp
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    s = minp.shape(args.workload, args.T)
    fp8 = s.wdtype == "fp8"
    inp = minp.make_inputs(s, seed=0)
    w13_r, w2_r = tp.shard_weights(inp.w13, inp.w2, rank, world)
    x = inp.x.to(dev)
    ident = (lambda t: t) if dist is None else None
    layer = tp.TensorParallelMoE(inp.router_w.to(dev), w13_r.to(dev), w2_r.to(dev), s.top_k,
                                 inp.w13_scale.to(dev) if fp8 else None,
                                 inp.w2_scale.to(dev) if fp8 else None,
                                 routing=routing_desc(inp, dev), variant=args.variant,
                                 reduce_max=ident, reduce_sum=ident)
    out = torch.empty(s.T, s.H, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(args.warmup):
        layer(x, out, stream)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(torch.cuda.get_device_properties(dev)) if rank == 0 else None
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        layer(x, out, stream)
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clocks = sampler.stop() if sampler is not None else None
    ms = reduce_max(dist, ev0.elapsed_time(ev1), dev)
    ws = next(iter(layer._bufs.values()))[0]
    assert capi.fused_moe_get_device_status(ws, stream) == capi.FMOE_OK
    # end to end: x from pinned host memory, out back to pinned host memory, every step
    x_host = inp.x.clone().pin_memory()
    out_host = torch.empty(s.T, s.H, dtype=torch.bfloat16).pin_memory()
    n_e2e = max(3, min(args.steps, 200))
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(n_e2e):
        x.copy_(x_host, non_blocking=True)
        layer(x, out, stream)
        out_host.copy_(out, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = reduce_max(dist, e0.elapsed_time(e1), dev)
    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return 0
    ms_step = ms / args.steps
    cfg = workload_config(s)
    cfg["parallelism"] = f"tensor parallel over the intermediate features: {world} shard(s) " \
                         f"of I/{world} = {s.I // world}, NCCL all-reduce of max|h| and of the " \
                         "fp32 partial output"
    line = {
        "metric": METRIC, "value": round(s.T * args.steps / (ms / 1e3), 1), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None,
        "dtype": "fp8_e4m3 (fp32 accumulate)" if fp8 else "bf16 (fp32 accumulate)",
        "data": "synthetic (seeded; N(0,1) x, N(0,1/sqrt(fan_in)) weights, per-expert e4m3 scales)",
        "config": cfg, "variant": f"tp{world}",
        "e2e": {"value": round(s.T * n_e2e / (e2e_ms / 1e3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": s.T * s.H * 2, "d2h_bytes_per_step": s.T * s.H * 2,
                "api": "TensorParallelMoE with pinned host copies of x and out"},
        # the one-call kernels plus amax_reduce and the bf16 finish, per step
        "gpu_launches": (capi.fused_moe_launches_per_call(layer.dims(s.T)) + 2) * args.steps,
        "clocks": clocks, "cpu_baseline": None,
    }
    print(json.dumps(line))
    return 0


# --------------------------------------------------------------------------- inverse RoPE

ROPE_METRIC = ("inverse-RoPE + per-head FP8 quantisation tokens/s; achieved HBM GB/s vs peak")
ROPE_SOURCES = ("mixture_experts_layer_26_b200/csrc/inv_rope_fp8.cu",
                "mixture_experts_layer_26_b200/csrc/fmoe_common.cuh")


def rope_bytes(s) -> int:
    """Algorithmic bytes of one launch: x read (bf16), codes written, scales written,
    positions read, and the rotary table rows the tokens gather (rot_dim fp32 each)."""
    el = s.T * s.n_heads * s.head_dim
    return el * 2 + el + s.T * s.n_heads * 4 + s.T * 4 + s.T * s.rot_dim * 4


def rope_config(s):
    x_bytes = s.T * s.n_heads * s.head_dim * 2
    big = x_bytes > L2_BYTES
    return {"workload": f"{s.name}: T={s.T} heads={s.n_heads} head_dim={s.head_dim} "
                        f"rot_dim={s.rot_dim} style={'half-split' if s.style == 0 else 'interleaved'}",
            "T": s.T, "n_heads": s.n_heads, "head_dim": s.head_dim, "rot_dim": s.rot_dim,
            "style": s.style, "max_pos": s.max_pos,
            "l2": (f"inputs larger than L2 ({x_bytes / 2 ** 20:.0f} MB x), no flush" if big else
                   f"L2 flushed before every timed launch ({x_bytes / 2 ** 20:.0f} MB x < "
                   f"{L2_BYTES / 2 ** 20:.0f} MB L2)"),
            "parallelism": "replicas (one independent kernel per GPU)"}


def rope_oracle_seconds(inp, tokens):
    """The oracle on the first `tokens` tokens of the batch: seconds."""
    from oracle import inv_rope_fp8_oracle as RO
    s = inp.shape
    xb = inp.x[:tokens].contiguous().view(torch.int16).numpy().view(np.uint16)
    t0 = time.perf_counter()
    RO.inv_rope_fp8_quant(xb, inp.positions[:tokens].numpy(), inp.cos_sin.numpy(), s.rot_dim,
                          s.style)
    return time.perf_counter() - t0


def run_rope_ours(args, rank, world, local_rank):
    from mixture_experts_layer_26_b200 import capi
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    s = minp.rope_shape(args.workload, args.T)
    inp = minp.make_rope_inputs(s, seed=0)
    x, pos, cs = inp.x.to(dev), inp.positions.to(dev), inp.cos_sin.to(dev)
    q = torch.empty(s.T, s.n_heads, s.head_dim, dtype=torch.uint8, device=dev)
    sc = torch.empty(s.T, s.n_heads, dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    d = capi.make_rope_dims(s.T, s.n_heads, s.head_dim, s.rot_dim, s.style, s.max_pos)
    stream = torch.cuda.current_stream(dev)
    flush = s.T * s.n_heads * s.head_dim * 2 <= L2_BYTES
    scratch = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=dev) if flush else None

    def barrier():
        if dist is not None:
            dist.barrier()

    def launch():
        capi.fused_inv_rope_fp8_quant_per_head(d, x, pos, cs, q, sc, status, stream)

    for _ in range(args.warmup):
        launch()
    torch.cuda.synchronize()
    assert int(status.item()) == capi.FMOE_OK

    # ---- timed region: exactly K launches; with small inputs the L2 is flushed before
    # each launch and only the launches are timed (events around each one)
    barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(torch.cuda.get_device_properties(dev)) if rank == 0 else None
    if flush:
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        for e0, e1 in evs:
            scratch.fill_(1)
            e0.record(stream)
            launch()
            e1.record(stream)
        torch.cuda.synchronize()
        ms = sum(e0.elapsed_time(e1) for e0, e1 in evs)
    else:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            launch()
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
    barrier()
    clocks = sampler.stop() if sampler is not None else None
    ms = reduce_max(dist, ms, dev)
    assert int(status.item()) == capi.FMOE_OK
    ms_launch = ms / args.steps
    value = tokens_per_second(world, s.T, args.steps, ms)

    # ---- end to end: x and positions from pinned host memory, codes and scales back
    x_h, pos_h = inp.x.clone().pin_memory(), inp.positions.clone().pin_memory()
    q_h = torch.empty(q.shape, dtype=torch.uint8).pin_memory()
    sc_h = torch.empty(sc.shape, dtype=torch.float32).pin_memory()
    n_e2e = max(3, min(args.steps, 200))

    def e2e_step():
        x.copy_(x_h, non_blocking=True)
        pos.copy_(pos_h, non_blocking=True)
        launch()
        q_h.copy_(q, non_blocking=True)
        sc_h.copy_(sc, non_blocking=True)

    for _ in range(3):
        e2e_step()
    barrier()
    torch.cuda.synchronize()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for _ in range(n_e2e):
        e2e_step()
    a1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = reduce_max(dist, a0.elapsed_time(a1), dev)
    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks, peak_kind = load_peaks()
    nbytes = rope_bytes(s)
    ach = nbytes / (ms_launch / 1e3) / 1e9
    kname = "inv_rope_fp8"
    roof = {"bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(ach / peaks["hbm_gbs"], 4),
            "traffic": profiled_traffic(kname, f"{args.workload}_T{s.T}"),
            "kernel": kname, "kernel_us": round(1e3 * ms_launch, 2), "algorithmic_bytes": nbytes,
            "peak_kind": (f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs, copy stream)"
                          if peak_kind == "measured" else
                          "fallback 6650 GB/s (no MEASURED_PEAKS.json)")}
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        n = min(s.T, 2048)
        secs = rope_oracle_seconds(inp, n)
        cpu = {"value": n / secs, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"the oracle on the first {n} of the {s.T} tokens ({secs:.2f} s)"}
    el = s.T * s.n_heads * s.head_dim
    line = {
        "metric": ROPE_METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_launch, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16 in, fp32 rotation, e4m3 + fp32 per-head scales out",
        "data": "synthetic (seeded; N(0,1) x, uniform positions, rotary table of base 10000)",
        "config": rope_config(s), "roofline": roof, "cpu_baseline": cpu,
        "e2e": {"value": round(tokens_per_second(world, s.T, n_e2e, e2e_ms), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": el * 2 + s.T * 4,
                "d2h_bytes_per_step": el + s.T * s.n_heads * 4,
                "api": "fused_inv_rope_fp8_quant_per_head with pinned host copies"},
        "gpu_launches": args.steps, "clocks": clocks,
    }
    print(json.dumps(line))
    return 0


def run_rope_reference(args, rank):
    if rank != 0:
        return 0
    s = minp.rope_shape(args.workload, args.T)
    inp = minp.make_rope_inputs(s, seed=0)
    n = min(s.T, 1024)  # each step: the oracle on a bounded slice of the batch
    for _ in range(min(args.warmup, 2)):
        rope_oracle_seconds(inp, n)
    total = sum(rope_oracle_seconds(inp, n) for _ in range(args.steps))
    value = n * args.steps / total
    line = {
        "impl": "reference", "metric": ROPE_METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp32 (oracle)", "data": "synthetic",
        "config": rope_config(s),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(),
                         "kind": "oracle", "sample": f"{args.steps} steps of {n} tokens each"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=sorted(minp.WORKLOADS) + sorted(minp.ROPE_WORKLOADS))
    ap.add_argument("--T", type=int, default=None,
                    help="tokens (default: the workload's largest; 4096 for the default workload)")
    ap.add_argument("--variant", default="auto", choices=["auto", "swap_ab", "normal", "normal_pair"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--step", choices=["layer", "route"], default="layer",
                    help="route: time the routing step alone (no expert weights allocated)")
    ap.add_argument("--tp", action="store_true",
                    help="tensor parallelism: the ranks share one layer, each holding I/N")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the decode workloads measured beside the default one")
    ap.add_argument("--no-peak-probe", action="store_true",
                    help="skip the FP8 tensor-peak probe (torch._scaled_mm)")
    ap.add_argument("--cpu-budget", type=float, default=8.0,
                    help="seconds of oracle expert work per core setting in cpu_baseline")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.workload in minp.ROPE_WORKLOADS:
        if args.impl == "reference":
            return run_rope_reference(args, rank)
        return run_rope_ours(args, rank, world, local_rank)
    if args.impl == "reference":
        return run_reference(args, rank)
    if args.step == "route":
        return run_route_only(args, rank, world, local_rank)
    if args.tp:
        return run_tp_ours(args, rank, world, local_rank)
    return run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    sys.exit(main())
