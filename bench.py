"""Throughput of the MoE feed-forward layer on B200: one JSON line on stdout.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload r1_decode] [--impl reference]

A step is one ``moe_layer_forward`` (router GEMM, route, permute, tile plan,
grouped SwiGLU FFN for routed + shared experts, combine) over one batch of T
tokens with the weights resident in HBM.  ``value`` is tokens/s over all
ranks (replicas: the layer does not shard on this path, so each rank runs its
own copy), timed with CUDA events between a barrier + synchronize on both
sides, max over ranks.  ``e2e`` is the same metric through the public call with
the activations copied in from pinned host memory and the output copied back
every step, the copies on their own streams so that they overlap the
neighbouring steps' layer calls (as a serving loop would run them).  The per-stage times come from ``moe_layer_forward_staged`` events
recorded inside the timed steps; ``roofline`` is the dominant kernel's
algorithmic bytes (or flops) per launch over its average in-place duration.

``--impl reference`` times the fp64 CPU oracle (the reference arm of this
build) on a bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s at 1 B200; % of HBM (decode) / tensor (prefill) roofline"
DEFAULT_WORKLOAD = "r1_decode"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tokens", type=int, default=None,
                    help="profiling case: the workload with this many tokens T (with --experts)")
    ap.add_argument("--experts", type=int, default=None,
                    help="profiling case: the workload with only this many routed experts "
                         "(drawn without the stored recipe; not a bench line)")
    ap.add_argument("--stages-only", action="store_true",
                    help="time moe_route, moe_permute and moe_combine alone at the workload's "
                         "sizes on random inputs (no expert weights; profiling case, not a "
                         "bench line)")
    ap.add_argument("--fp8-peak", action="store_true",
                    help="measure the dense e4m3 GEMM peak (cuBLASLt) on cuda:0, print it, exit")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


PEAKS_DATA = os.path.join(ROOT, "profiles", "peaks.json")


def _peaks_data():
    """Figures measured on this machine beyond MEASURED_PEAKS.json: the dense e4m3 GEMM peak
    (``bench.py --fp8-peak``) and per-launch DRAM traffic from ncu captures."""
    try:
        with open(PEAKS_DATA) as f:
            return json.load(f)
    except (OSError, ValueError):
        return {}


def load_fp8_peak():
    """Sustained dense e4m3 GEMM throughput measured on this machine's B200s, else None."""
    v = _peaks_data().get("fp8", {}).get("fp8_tflops_sustained")
    return None if v is None else float(v)


def measure_fp8_peak(dev, n=8192, seconds=4.0):
    """cuBLASLt e4m3 x e4m3 -> bf16 GEMM (torch._scaled_mm) n^3: best of 10 (burst) and a
    back-to-back loop of `seconds` (sustained), 2 n^3 flops each."""
    import torch
    a = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn)
    b = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn)
    one = torch.ones((), device=dev)

    def mm():
        return torch._scaled_mm(a, b.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16)

    for _ in range(3):
        mm()
    torch.cuda.synchronize(dev)
    best = float("inf")
    for _ in range(10):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        mm()
        e1.record()
        e1.synchronize()
        best = min(best, e0.elapsed_time(e1))
    iters = max(1, int(seconds * 1e3 / best))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(iters):
        mm()
    e1.record()
    e1.synchronize()
    flops = 2.0 * n ** 3
    return {"fp8_tflops": flops / (best * 1e-3) / 1e12,
            "fp8_tflops_sustained": flops / (e0.elapsed_time(e1) / iters * 1e-3) / 1e12,
            "n": n, "iters": iters, "how": "torch._scaled_mm e4m3 x e4m3 -> bf16, unit scales"}


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count() or 1


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML, else nvidia-smi)
# ---------------------------------------------------------------------------

class ClockSampler:
    REASONS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index: int):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._dev = device_index
        self._thread = None

    def _run(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self._dev)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            get_r = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            while not self._stop.is_set():
                self.samples.append(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                r = get_r(h)
                for name, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
                time.sleep(0.02)
            pynvml.nvmlShutdown()
        except Exception as e:  # NVML missing: one nvidia-smi reading instead
            self.samples.append(None)
            self.error = repr(e)

    def __enter__(self):
        self._thread = threading.Thread(target=self._run, daemon=True)
        self._thread.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        self._thread.join(timeout=5)

    def summary(self):
        vals = [s for s in self.samples if s]
        return {"sm_mhz": statistics.median(vals) if vals else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(vals)}


# ---------------------------------------------------------------------------
# algorithmic work
# ---------------------------------------------------------------------------

def _e4m3(dtype):
    """e4m3 storage, with power-of-two ("e4m3") or any fp32 ("e4m3_fs") block scales."""
    return dtype in ("e4m3", "e4m3_fs")


def work_model(spec, offsets):
    """Algorithmic bytes / flops of the layer and of its two expert GEMM launches.

    Decode units: the weight bytes of every expert that received at least one
    row (plus the shared experts and the router) -- a dense pass over all
    experts is not the measure.  Prefill units: 2 * rows * 3 * d * I flops over
    the routed and shared rows plus the router's 2 * T * d * E.
    """
    T, d, E, k, I, S = spec.T, spec.d_model, spec.E, spec.top_k, spec.d_ff, spec.n_shared
    # weight bytes per element: MXFP4 = half a byte + one E8M0 byte per 32 elements
    wb = {"e4m3": 1.0, "e4m3_fs": 1.0, "e2m1": 0.5 + 1.0 / 32}.get(spec.weight, 2.0)
    ab = 1 if _e4m3(spec.act) else 2
    sizes = np.diff(offsets)
    touched = int((sizes > 0).sum())
    R = T * k
    rows = R + S * T
    ffn1_bytes = (touched + S) * 2 * I * d * wb + rows * d * ab + rows * I * 2
    ffn2_bytes = (touched + S) * d * I * wb + rows * I * 2 + rows * d * 2
    layer_weight_bytes = (touched + S) * 3 * I * d * wb + E * d * 2
    ffn1_flops = 2.0 * rows * 2 * I * d
    ffn2_flops = 2.0 * rows * I * d
    layer_flops = 2.0 * rows * 3 * I * d + 2.0 * T * d * E
    # per-expert operands of the two GEMMs: each expert (group of n > 0 rows) is bound by
    # its own flops or by its own bytes (weights once, its rows in, h out and in, y out)
    n_all = np.concatenate([sizes[sizes > 0], np.full(S, T)]).astype(np.float64)
    group_flops = 2.0 * n_all * 3 * I * d
    group_bytes = 3.0 * I * d * wb + n_all * (d * ab + 2 * I * 2 + d * 2)
    return dict(touched=touched, ffn1_bytes=ffn1_bytes, ffn2_bytes=ffn2_bytes,
                layer_weight_bytes=layer_weight_bytes, ffn1_flops=ffn1_flops,
                ffn2_flops=ffn2_flops, layer_flops=layer_flops,
                group_flops=group_flops, group_bytes=group_bytes)


def small_stage_bytes(spec):
    """Algorithmic HBM bytes of the bandwidth-bound stages around the expert GEMMs (reads +
    writes each stage must make at least once)."""
    T, d, E, k, S = spec.T, spec.d_model, spec.E, spec.top_k, spec.n_shared
    ab = 1 if _e4m3(spec.act) else 2
    xs = 4 * (d // 128) if _e4m3(spec.act) else 0          # per-row activation scales
    ob = 4 if spec.out == "f32" else 2
    R = T * k
    return {
        "router_gemm": T * d * 2 + E * d * 2 + T * E * 4,
        "route": T * E * 4 + (E * 4 if spec.score == "sigmoid_bias" else 0) + R * 8,
        "permute": R * 4 + T * (d * ab + xs) + R * (d * ab + xs) + R * 8 + (E + 1) * 4,
        "combine": (R + S * T) * d * 2 + R * 8 + T * d * ob,
    }


def per_expert_bound_ms(wm, tflops, gbs):
    """Sum over experts of max(flops / tensor peak, bytes / HBM peak) for the two expert
    GEMMs: the time they take when every expert runs at its own roofline and experts do
    not overlap one another's HBM and tensor phases."""
    t = np.maximum(wm["group_flops"] / (tflops * 1e12), wm["group_bytes"] / (gbs * 1e9))
    return float(t.sum() * 1e3)


def bound_of(name):
    return "tensor" if name in ("r1_prefill", "r1_prefill_fp8") else "hbm"


def read_traffic(kernel_key):
    """Per-launch DRAM bytes of an ncu capture, if it was taken on the current kernel
    source (else None)."""
    import hashlib
    ent = _peaks_data().get("traffic", {}).get(kernel_key)
    if not ent:
        return None
    src = os.path.join(ROOT, "sparse_expert_moe_b200", "csrc", "grouped_gemm.cu")
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    if ent.get("grouped_gemm_sha256_prefix") != sha:
        return None
    return float(ent["dram_bytes_per_launch"])


# ---------------------------------------------------------------------------
# replicas: one layer copy per rank, timed together
# ---------------------------------------------------------------------------

def max_over_ranks_dist(v, world, device):
    """Max of a per-rank value over all ranks (the slowest replica sets the time)."""
    if world == 1:
        return float(v)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(tokens_per_rank, world, ms_total_max, steps):
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return tokens_per_rank * world * steps / (ms_total_max * 1e-3)


# ---------------------------------------------------------------------------
# the reference arm: the fp64 oracle on the host
# ---------------------------------------------------------------------------

def light_workload(name, seed=0):
    """Activations, router and bias of a named workload (no expert weights)."""
    from sparse_expert_moe_b200 import inputs
    import oracle
    spec = inputs.SPECS[name]
    rec = inputs.load_recipe(name)
    bias = rec.get("sel_bias")
    if bias is None and name in inputs.BIAS_SOURCE:
        bias = inputs.load_recipe(inputs.BIAS_SOURCE[name]).get("sel_bias")
    if bias is None:
        b = inputs.draw_sel_bias(spec, seed)
        bias = None if b is None else b.numpy()
    x32 = inputs._draw_x_fp32(spec, seed, rec.get("redraw"))
    x, xs = inputs.encode_act(spec, x32)
    return {"spec": spec, "x": x, "x_scale": xs, "wr": inputs.draw_router(spec, seed),
            "bias": None if bias is None else np.asarray(bias, np.float64)}


def _act_values(light, rows):
    import oracle
    import torch
    x = light["x"][rows]
    if light["x_scale"] is not None:
        return oracle.dequantize_blocks(x.view(torch.uint8).numpy(),
                                        light["x_scale"][rows].numpy(), 1, 128)
    return x.double().numpy()


def _weight_values(w, s):
    import oracle
    import torch
    if s is None:
        return w.double().numpy()
    if s.dtype == torch.uint8:           # MXFP4: packed E2M1 codes + E8M0 scale atoms
        from sparse_expert_moe_b200 import inputs
        return oracle.dequantize_mxfp4(w.numpy(), inputs.scale_rows(s.numpy()).numpy())
    return oracle.dequantize_blocks(w.view(torch.uint8).numpy(), s.numpy(), 128, 128)


def needed_experts(light, rows):
    import oracle
    spec = light["spec"]
    L = oracle.router_logits(_act_values(light, rows), light["wr"].double().numpy())
    idx, _ = oracle.route(L, spec.score, spec.top_k, light["bias"])
    return sorted({int(e) for e in np.unique(idx)})


def stored_experts(spec, seed, routed, host_weights=None):
    """Storage-typed (bf16 / e4m3 + scales) tensors of the listed routed experts and the
    shared experts: taken from resident host copies or drawn."""
    from sparse_expert_moe_b200 import inputs
    out = {}
    for kind, ids in (("r", routed), ("s", range(spec.n_shared))):
        for e in ids:
            if host_weights is not None:
                pre = "ws" if kind == "s" else "w"
                get = lambda n: None if host_weights.get(n) is None else host_weights[n][e]
                out[(kind, e)] = (get(pre + "13"), get(pre + "13_s"), get(pre + "2"), get(pre + "2_s"))
            else:
                out[(kind, e)] = inputs.draw_expert(spec, seed, e, kind == "s")
    return out


def time_oracle(light, rows, stored):
    """One oracle run on `rows`, timed as it stands: routing, decoding the inputs to fp64
    (activations and every expert it touches) and the fp64 arithmetic."""
    import oracle
    spec = light["spec"]

    def expert(kind, e):
        w13, s13, w2, s2 = stored[(kind, e)]
        return _weight_values(w13, s13), _weight_values(w2, s2)

    t0 = time.perf_counter()
    xv = _act_values(light, rows)
    expert_x = None
    if spec.act == "bf16" and spec.weight in ("e4m3", "e2m1"):   # quantised in the permutation
        codes, sc = oracle.quantize_e4m3_blocks(xv)
        expert_x = oracle.dequantize_blocks(codes, sc, 1, 128)
    oracle.layer_forward(xv, light["wr"].double().numpy(), spec.score, spec.top_k,
                         lambda e: expert("r", e), spec.E,
                         [(lambda s=s: expert("s", s)) for s in range(spec.n_shared)],
                         sel_bias=light["bias"], expert_x=expert_x)
    return time.perf_counter() - t0


def cpu_baseline(name, host_weights=None, budget_s=25.0):
    """The oracle as it stands on a bounded sample of the workload's tokens (rank 0 only):
    the first n tokens, n the largest power of two (<= T) whose run stays in the budget."""
    light = light_workload(name)
    spec = light["spec"]
    n = 1
    rows = np.arange(n)
    stored = stored_experts(spec, 0, needed_experts(light, rows), host_weights)
    dt = time_oracle(light, rows, stored)
    while n * 2 <= spec.T:
        n2 = n * 2
        rows2 = np.arange(n2)
        routed = needed_experts(light, rows2)
        # cost grows with the experts touched (their fp64 decoding dominates)
        if dt * (len(routed) + spec.n_shared) / max(len(stored), 1) * 1.2 > budget_s:
            break
        stored = stored_experts(spec, 0, routed, host_weights)
        n, rows = n2, rows2
        dt = time_oracle(light, rows, stored)
    return {"value": n / dt, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"first {n} tokens of {name}: fp64 NumPy oracle incl. decoding "
                      f"{len(stored)} experts to fp64; {dt:.2f} s"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    light = light_workload(args.workload)
    spec = light["spec"]
    rows = np.arange(1)
    # inputs drawn outside the timing; each step = the oracle on one token of the workload
    stored = stored_experts(spec, 0, needed_experts(light, rows))
    for _ in range(args.warmup):
        time_oracle(light, rows, stored)
    t = [time_oracle(light, rows, stored) for _ in range(args.steps)]
    total = sum(t)
    value = len(rows) * args.steps / total
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "sample_tokens_per_step": len(rows)},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(),
                             "kind": "oracle",
                             "sample": f"token 0 of {args.workload} per step: fp64 NumPy oracle "
                                       f"incl. decoding its {len(stored)} experts to fp64"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def time_e2e(layer, wl, y, idx, gw, stream, K, dev, barrier, max_over_ranks):
    """ms per step of K layer calls through ``moe_layer_forward`` with every step's input
    copied up from pinned host memory and its output copied back, the copies on their own
    streams so that step i's copy in and step i-1's copy out overlap step i-1's and step
    i+1's compute (two device input and output buffers; events order every buffer's
    reuse).  The timed region spans all K copies in, K layer calls and K copies out."""
    import torch
    fp8 = wl.x.dtype == torch.float8_e4m3fn
    x_host = (wl.x.view(torch.uint8) if fp8 else wl.x).pin_memory()
    xs_host = None if wl.x_scale is None else wl.x_scale.pin_memory()
    nb = 2
    x_dev = [torch.empty_like(x_host, device=dev) for _ in range(nb)]
    xs_dev = [None if xs_host is None else torch.empty_like(xs_host, device=dev) for _ in range(nb)]
    y_dev = [torch.empty_like(y) for _ in range(nb)]
    y_host = [torch.empty(y.shape, dtype=y.dtype).pin_memory() for _ in range(nb)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    ev_in, ev_comp, ev_out = [ev() for _ in range(nb)], [ev() for _ in range(nb)], [ev() for _ in range(nb)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    barrier()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    for i in range(K):
        j = i % nb
        if i >= nb:
            s_in.wait_event(ev_comp[j])          # step i - 2 has read x_dev[j]
        with torch.cuda.stream(s_in):
            x_dev[j].copy_(x_host, non_blocking=True)
            if xs_host is not None:
                xs_dev[j].copy_(xs_host, non_blocking=True)
        ev_in[j].record(s_in)
        stream.wait_event(ev_in[j])
        if i >= nb:
            stream.wait_event(ev_out[j])         # step i - 2's output has left y_dev[j]
        xj = x_dev[j].view(torch.float8_e4m3fn) if fp8 else x_dev[j]
        layer.forward(xj, xs_dev[j], y_dev[j], idx, gw, stream)
        ev_comp[j].record(stream)
        s_out.wait_event(ev_comp[j])
        with torch.cuda.stream(s_out):
            y_host[j].copy_(y_dev[j], non_blocking=True)
        ev_out[j].record(s_out)
    for j in range(nb):
        stream.wait_event(ev_out[j])
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    ms = max_over_ranks(e0.elapsed_time(e1)) / K
    h2d = x_host.numel() * x_host.element_size() + (0 if xs_host is None else xs_host.numel() * 4)
    d2h = y_host[0].numel() * y_host[0].element_size()
    return ms, h2d, d2h


def time_staged(moe, layer, weights, x, xs, y, idx, gw, K, stream, dev, barrier, max_over_ranks):
    """K ``moe_layer_forward_staged`` calls between a barrier + synchronize on both sides:
    (max over ranks of the total ms, mean ms per stage from the in-place events)."""
    import torch
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(8)] for _ in range(K)]
    for row in evs:
        for e in row:
            e.record(stream)   # create the events before they are handed to the library
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    barrier()
    torch.cuda.synchronize(dev)
    start.record(stream)
    for i in range(K):
        moe.moe_layer_forward_staged(layer.cfg, weights, x, xs, y, idx, gw, layer.ws, evs[i], stream)
    end.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    ms_total = max_over_ranks(start.elapsed_time(end))
    stage_ms = {s: 0.0 for s in moe.STAGES}
    for row in evs:
        for j, s in enumerate(moe.STAGES):
            stage_ms[s] += row[j].elapsed_time(row[j + 1]) / K
    return ms_total, stage_ms


def decode_uniform(moe, inputs, layer, wl, y, idx, gw, K, W, stream, dev, barrier, max_over_ranks,
                   peaks):
    """The uniformly routed R1 decode batch (no selection bias: about 252 of 256 experts
    touched, the full weight traffic of a decode step) on the same resident weights, timed
    like the main line; reported beside it."""
    import torch
    wu = inputs.load_workload("r1_decode_uniform", reuse=wl)
    xu = wu.x.to(dev)
    t = layer.tensors
    weights = moe.make_weights(t["wr"], None, t["w13"], t["w2"], t["ws13"], t["ws2"])
    for _ in range(W):
        moe.moe_layer_forward(layer.cfg, weights, xu, None, y, idx, gw, layer.ws, stream)
    torch.cuda.synchronize(dev)
    ms_total, stage_ms = time_staged(moe, layer, weights, xu, None, y, idx, gw, K, stream, dev,
                                     barrier, max_over_ranks)
    ms = ms_total / K
    spec = wu.spec
    sizes = np.bincount(idx.cpu().numpy().ravel(), minlength=spec.E)
    wm = work_model(spec, np.concatenate([[0], np.cumsum(sizes)]))
    hbm = peaks["hbm_gbs"]
    gbs = lambda b, t: b / (t * 1e-3) / 1e9
    return {"workload": "r1_decode_uniform", "ms_per_step": ms, "value": spec.T / (ms * 1e-3),
            "unit": "tokens/s", "touched_experts": wm["touched"],
            "weight_bytes_touched": wm["layer_weight_bytes"],
            "hbm_frac_layer": gbs(wm["layer_weight_bytes"], ms) / hbm,
            "ffn1": {"ms": stage_ms["ffn1"], "gbs": gbs(wm["ffn1_bytes"], stage_ms["ffn1"]),
                     "frac": gbs(wm["ffn1_bytes"], stage_ms["ffn1"]) / hbm},
            "ffn2": {"ms": stage_ms["ffn2"], "gbs": gbs(wm["ffn2_bytes"], stage_ms["ffn2"]),
                     "frac": gbs(wm["ffn2_bytes"], stage_ms["ffn2"]) / hbm},
            "stages_ms": stage_ms}


def time_graph(moe, layer, x, xs, y, idx, gw, K, W, stream, dev, barrier, max_over_ranks):
    """K replays of the layer recorded once as a CUDA graph (moe_layer_graph_*), device time
    between a barrier + synchronize on both sides: ms per step (max over ranks)."""
    import torch
    g = moe.LayerGraph(layer.cfg, layer.weights, x, xs, y, idx, gw, layer.ws)
    for _ in range(W):
        g.launch(stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    barrier()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(K):
        g.launch(stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    g.close()
    return max_over_ranks(e0.elapsed_time(e1)) / K


def launches_per_step(spec):
    """Kernels one ``moe_layer_forward`` launches: router GEMM, route, permute (count, then
    rank for T > 256, then the row copy -- none when the first GEMM gathers e4m3 rows on
    wide tiles, T > 128), plan, FFN1, FFN2, combine; the f32 family adds its bf16
    conversions, e4m3 activations their scale preparation (and, on decode-sized tiles with
    power-of-two scales, the permuted rows' scale gather), e4m3 weights with power-of-two
    scales their UE8M0 conversion."""
    wide = spec.T > 128
    e4m3_tok = _e4m3(spec.act) or spec.weight in ("e4m3", "e2m1")
    gather = e4m3_tok and wide and spec.weight != "e4m3_fs"
    quant = spec.act == "bf16" and spec.weight in ("e4m3", "e2m1")
    n = 1 + 1 + 1 + (1 if spec.T > 256 else 0) + (0 if gather and not quant else 1) + 1 + 2 + 1
    if spec.act == "f32":
        n += 4 + (2 if spec.n_shared else 0)
    if _e4m3(spec.act):
        n += 1                                  # activation scale preparation
        if spec.act == "e4m3" and not gather:
            n += 1                              # permuted rows' UE8M0 scale factors
    if spec.weight == "e4m3":
        n += 2 + (2 if spec.n_shared else 0)    # weight block scales -> UE8M0
    return n


def run_ours(args):
    import torch
    import torch.distributed as dist
    from sparse_expert_moe_b200 import inputs, moe

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(v):
        return max_over_ranks_dist(v, world, dev)

    name = args.workload
    if args.experts:
        from dataclasses import replace
        spec = replace(inputs.SPECS[name], E=args.experts)
        if args.tokens:
            spec = replace(spec, T=args.tokens)
        wl = inputs.make_workload(spec, 0)
    else:
        wl = inputs.load_workload(name)
    spec = wl.spec
    layer = moe.DeviceLayer.from_workload(wl, dev)
    x = wl.x.to(dev)
    xs = None if wl.x_scale is None else wl.x_scale.to(dev)
    y = layer.output(dev)
    idx = torch.empty((spec.T, spec.top_k), dtype=torch.int32, device=dev)
    gw = torch.empty((spec.T, spec.top_k), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    # warm-up (untimed)
    for _ in range(args.warmup):
        layer.forward(x, xs, y, idx, gw)
    torch.cuda.synchronize(dev)
    if moe.moe_read_device_status(layer.ws) != 0:
        raise SystemExit("device status set during warm-up")

    # timed steps: stage events recorded in place
    K = args.steps
    with ClockSampler(local) as clocks:
        ms_total, stage_ms = time_staged(moe, layer, layer.weights, x, xs, y, idx, gw, K, stream,
                                         dev, barrier, max_over_ranks)
    ms_step = ms_total / K
    status = moe.moe_read_device_status(layer.ws)

    # end to end through the public call, pipelined as a serving loop runs it
    e2e_ms, h2d, d2h = time_e2e(layer, wl, y, idx, gw, stream, K, dev, barrier, max_over_ranks)
    graph_ms = None
    if spec.T <= 256:      # decode-sized batches: the layer's launches as one graph
        graph_ms = time_graph(moe, layer, x, xs, y, idx, gw, K, args.warmup, stream, dev, barrier,
                              max_over_ranks)
    idx_np = idx.cpu().numpy()
    peaks, peak_src = load_peaks()
    uniform = None
    if name == "r1_decode" and not args.experts:
        uniform = decode_uniform(moe, inputs, layer, wl, y, idx, gw, K, args.warmup, stream, dev,
                                 barrier, max_over_ranks, peaks)

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return

    sizes = np.bincount(idx_np.ravel(), minlength=spec.E)
    off = np.concatenate([[0], np.cumsum(sizes)])
    wm = work_model(spec, off)
    bound = bound_of(name)
    if bound == "hbm":
        dom = "ffn1"
        achieved = wm["ffn1_bytes"] / (stage_ms["ffn1"] * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        unit = "GB/s"
        units_note = f"{wm['touched']} touched routed experts + {spec.n_shared} shared: W13 bytes, " \
                     "token rows read once, h written once"
    else:
        dom = "ffn1"
        achieved = wm["ffn1_flops"] / (stage_ms["ffn1"] * 1e-3) / 1e12
        peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
        if _e4m3(spec.weight):
            fp8 = load_fp8_peak()
            if fp8 is not None:
                peak, peak_src = fp8, "measured e4m3 sustained (profiles/peaks.json)"
            else:
                peak *= 2.0   # nominal fp8 : bf16 ratio of the dense tensor-core peaks
                peak_src += " bf16 x 2 (nominal fp8 ratio)"
        unit = "TFLOP/s"
        units_note = "2 * (T*k + S*T) * 2I * d"
    tensor_peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    if _e4m3(spec.weight):
        tensor_peak = load_fp8_peak() or 2.0 * tensor_peak
    ffn_bound_ms = per_expert_bound_ms(wm, tensor_peak, peaks["hbm_gbs"])
    tokens = spec.T * world
    value = replica_throughput(spec.T, world, ms_total, K)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": {"e4m3": "e4m3", "e4m3_fs": "e4m3 (fp32 block scales)",
                  "e2m1": "e2m1 x e4m3"}.get(spec.weight, "bf16"),
        "data": "synthetic",
        "config": {"workload": name if not args.experts else
                   f"{name} with E={spec.E}, T={spec.T} (profiling case)",
                   "T": spec.T, "d_model": spec.d_model, "E": spec.E,
                   "top_k": spec.top_k, "d_ff": spec.d_ff, "n_shared": spec.n_shared,
                   "score": spec.score, "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2: each step streams "
                         f"{wm['layer_weight_bytes'] / 1e9:.1f} GB of expert weights"},
        "roofline": {"bound": bound,
                     "kernel": f"{dom} (" + ("grouped_gemm_fs_kernel<11>" if spec.weight == "e4m3_fs" else
                                             f"grouped_gemm_kernel<{ {'e4m3': 3, 'e2m1': 7}.get(spec.weight, 1)}>") + ")",
                     "achieved": achieved, "peak": peak, "peak_source": peak_src, "unit": unit,
                     "frac": achieved / peak, "traffic": read_traffic(f"ffn1_{name}"),
                     "units": units_note},
        "layer": {"weight_bytes_touched": wm["layer_weight_bytes"],
                  "hbm_frac_layer": wm["layer_weight_bytes"] / (ms_step * 1e-3) / 1e9 / peaks["hbm_gbs"],
                  "tflops_layer": wm["layer_flops"] / (ms_step * 1e-3) / 1e12,
                  "touched_experts": wm["touched"],
                  "ffn_per_expert_bound_ms": ffn_bound_ms,
                  "ffn_frac_of_per_expert_bound": ffn_bound_ms / (stage_ms["ffn1"] + stage_ms["ffn2"])},
        "stages_ms": stage_ms,
        "stages_hbm": {n: {"bytes": int(v), "gbs": v / (stage_ms[n] * 1e-3) / 1e9,
                           "frac": v / (stage_ms[n] * 1e-3) / 1e9 / peaks["hbm_gbs"]}
                       for n, v in small_stage_bytes(spec).items()},
        "e2e": {"value": tokens / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "how": "pinned host copies in and out every step on two copy streams, overlapping "
                       "the neighbouring steps' moe_layer_forward calls",
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": launches_per_step(spec) * K,
        "clocks": clocks.summary(),
        "device_status": status,
    }
    if uniform is not None:
        line["decode_uniform"] = uniform
    if graph_ms is not None:
        line["graph"] = {"ms_per_step": graph_ms, "value": spec.T * world / (graph_ms * 1e-3),
                         "unit": "tokens/s",
                         "how": "moe_layer_graph_launch: the layer recorded once as a CUDA graph"}
    if not args.no_cpu_baseline and world == 1:
        host = {n: getattr(wl, n) for n in ("w13", "w2", "ws13", "ws2", "w13_s", "w2_s", "ws13_s",
                                            "ws2_s")}
        line["cpu_baseline"] = cpu_baseline(name, host)
    elif world > 1:
        line["cpu_baseline"] = None
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def run_stages(args):
    """moe_route, moe_permute and moe_combine alone at the sizes of a workload, on random
    inputs of its shapes and dtypes (the bandwidth-bound stages around the expert GEMMs),
    each timed over K calls with CUDA events, an L2 flush (a 256 MB write) before every
    call; GB/s against the algorithmic bytes of ``small_stage_bytes``."""
    import torch
    from sparse_expert_moe_b200 import inputs, moe
    spec = inputs.SPECS[args.workload]
    if args.tokens:
        from dataclasses import replace
        spec = replace(spec, T=args.tokens)
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    T, d, E, k, S = spec.T, spec.d_model, spec.E, spec.top_k, spec.n_shared
    R = T * k
    g = torch.Generator(device=dev).manual_seed(0)
    cfg = moe.config_from_spec(spec)
    logits = torch.randn((T, E), generator=g, device=dev)
    bias = None if spec.score != "sigmoid_bias" else 0.1 * torch.rand(E, generator=g, device=dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    gw = torch.empty((T, k), dtype=torch.float32, device=dev)
    fp8 = _e4m3(spec.act)
    x = torch.randn((T, d), generator=g, device=dev).to(torch.bfloat16)
    xs = xps = None
    if fp8:
        x = x.to(torch.float8_e4m3fn).view(torch.uint8)
        xs = torch.ones((T, d // 128), device=dev)
        xps = torch.empty((R, d // 128), device=dev)
    x_perm = torch.empty((R, d), dtype=x.dtype, device=dev)
    perm_token = torch.empty(R, dtype=torch.int32, device=dev)
    inv_perm = torch.empty((T, k), dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    ws = torch.zeros(moe.moe_workspace_size(cfg), dtype=torch.uint8, device=dev)
    y_perm = torch.randn((R, d), generator=g, device=dev).to(torch.bfloat16)
    y_sh = torch.randn((S, T, d), generator=g, device=dev).to(torch.bfloat16) if S else None
    y = torch.empty((T, d), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    calls = {
        "route": lambda: moe.moe_route(cfg, logits, bias, idx, gw),
        "permute": lambda: moe.moe_permute(cfg, idx, x, xs, x_perm, xps, perm_token, inv_perm,
                                           offsets, ws),
        "combine": lambda: moe.moe_combine(cfg, y_perm, inv_perm, gw, y_sh, y),
    }
    nbytes = small_stage_bytes(spec)
    out = {}
    for name, fn in calls.items():
        for _ in range(args.warmup):
            fn()
        ms = []
        for _ in range(args.steps):
            flush.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            e1.synchronize()
            ms.append(e0.elapsed_time(e1))
        t = statistics.median(ms)
        gbs = nbytes[name] / (t * 1e-3) / 1e9
        out[name] = {"ms": t, "bytes": nbytes[name], "gbs": gbs, "frac": gbs / load_peaks()[0]["hbm_gbs"]}
    status = moe.moe_read_device_status(ws)
    print(json.dumps({"workload": args.workload, "T": T, "stages": out, "device_status": status,
                      "how": "median of --steps calls, L2 flushed before each"}), flush=True)


def main():
    args = parse()
    if args.stages_only:
        run_stages(args)
        return
    if args.fp8_peak:
        print(json.dumps(measure_fp8_peak("cuda:0")), flush=True)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
