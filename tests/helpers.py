"""Test-side helpers: margin filtering with the oracle, oracle evaluation of workloads,
and the error metric.  Uses the oracle (allowed in tests); never the CUDA path."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from sparse_expert_moe_b200 import inputs


def max_rel_err(y, ref) -> float:
    """||y - ref||_inf / ||ref||_inf over the whole output."""
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.abs(y - ref).max() / max(np.abs(ref).max(), 1e-30))


def topk_gaps(keys, k):
    """Smallest gap between consecutive keys among each row's k+1 largest (selection and
    slot order both decided by more than the margin)."""
    m = min(k + 1, keys.shape[1])
    if m < 2:
        return np.full(keys.shape[0], np.inf)
    s = -np.sort(-keys, axis=1)
    return (s[:, : m - 1] - s[:, 1:m]).min(axis=1)


def margin_logits(T, E, k, score, bias, margin=1e-3, seed=0, stream=0):
    """U(-3, 3) fp32 logits whose rows are redrawn until the top k+1 keys are >= margin apart
    (``inputs.draw_logits`` with those redraws; only the failing rows are redrawn and
    re-checked each round)."""
    b64 = None if bias is None else np.asarray(bias, np.float64)
    L = inputs.draw_logits(T, E, seed, stream=stream)
    attempts = np.zeros(T, np.int64)
    bad = np.arange(T)
    while bad.size:
        keys = oracle.selection_keys(L[bad].astype(np.float64), score, b64)
        bad = bad[topk_gaps(keys, k) < margin]
        for t in bad:
            attempts[t] += 1
            L[t] = inputs.draw_logit_row(T, E, seed, int(t), int(attempts[t]), stream=stream)
    return L


def act_values(wl) -> np.ndarray:
    if inputs.is_e4m3(wl.spec.act):
        return oracle.dequantize_blocks(wl.x.view(torch.uint8).numpy(), wl.x_scale.numpy(), 1, 128)
    return wl.x.double().numpy()


def margin_workload(spec, seed=0, threads=None):
    """A custom workload whose activation rows are redrawn until routing has the spec's margin."""
    wr = inputs.draw_router(spec, seed).double().numpy()
    b = inputs.draw_sel_bias(spec, seed)
    b64 = None if b is None else b.double().numpy()
    attempts = {}
    while True:
        x32 = inputs._draw_x_fp32(spec, seed, sorted(attempts.items()))
        x, xs = inputs.encode_act(spec, x32)
        xv = x.double().numpy() if not inputs.is_e4m3(spec.act) else oracle.dequantize_blocks(
            x.view(torch.uint8).numpy(), xs.numpy(), 1, 128)
        keys = oracle.selection_keys(oracle.router_logits(xv, wr), spec.score, b64)
        bad = np.nonzero(topk_gaps(keys, spec.top_k) < spec.margin)[0]
        if bad.size == 0:
            break
        for t in bad:
            attempts[int(t)] = attempts.get(int(t), 0) + 1
    return inputs.make_workload(spec, seed, redraw=sorted(attempts.items()), threads=threads)


_E4M3_TABLE = None


def dequant_fast(codes, scales, br, bc):
    """oracle.dequantize_blocks by table lookup: the oracle's decoding of all 256 e4m3 codes,
    indexed by the codes, times each block's scale (broadcast, no repeated scale array).
    Equal to oracle.dequantize_blocks bit for bit (tests/test_oracle_pins.py checks it);
    used where whole expert weight sets are decoded, to keep the oracle runs short."""
    global _E4M3_TABLE
    if _E4M3_TABLE is None:
        _E4M3_TABLE = oracle.decode_e4m3(np.arange(256, dtype=np.uint8))
    c = np.asarray(codes, np.uint8)
    R, C = c.shape
    v = _E4M3_TABLE[c].reshape(R // br, br, C // bc, bc)
    v *= np.asarray(scales, np.float64)[:, None, :, None]
    return v.reshape(R, C)


_FP4_TABLE = None


def dequant_mxfp4_fast(packed, scale_codes):
    """oracle.dequantize_mxfp4 by table lookup: the oracle's decoding of both nibbles of
    all 256 bytes, indexed by the packed bytes, times each 32-element run's decoded E8M0
    scale (broadcast).  Equal to the oracle bit for bit (tests/test_oracle_pins.py)."""
    global _FP4_TABLE
    if _FP4_TABLE is None:
        _FP4_TABLE = oracle.decode_e2m1(oracle.unpack_fp4(np.arange(256, dtype=np.uint8)[:, None]))
    p = np.asarray(packed, np.uint8)
    R, half = p.shape
    v = _FP4_TABLE[p].reshape(R, 2 * half // 32, 32)
    v *= oracle.decode_e8m0(scale_codes)[:, :, None]
    return v.reshape(R, 2 * half)


def _w_values(w, s, shape_blocks):
    if s is None:
        return w.double().numpy()
    if s.dtype == torch.uint8:          # MXFP4: packed E2M1 + E8M0 scale atoms
        return dequant_mxfp4_fast(w.numpy(), inputs.scale_rows(s.numpy()).numpy())
    return dequant_fast(w.view(torch.uint8).numpy(), s.numpy(), 128, 128)


def oracle_routing(wl):
    """The oracle's router, top-k and permutation over every token of workload wl."""
    spec = wl.spec
    logits = oracle.router_logits(act_values(wl), wl.wr.double().numpy())
    bias = None if wl.sel_bias is None else wl.sel_bias.double().numpy()
    idx, gates = oracle.route(logits, spec.score, spec.top_k, bias)
    offsets, perm_token, inv_perm = oracle.permute(idx, spec.E)
    return dict(idx=idx, gates=gates, offsets=offsets, perm_token=perm_token, inv_perm=inv_perm)


def tile_edge_tokens(routing, T, n_shared, unit):
    """Tokens holding the first and the last row of every `unit`-row piece of every routed
    group (the GEMM tiles' token ranges: every group's first and last chunk among them),
    and of the shared experts' T rows."""
    off, pt = routing["offsets"], routing["perm_token"]
    rows = []
    for e in range(len(off) - 1):
        lo, hi = int(off[e]), int(off[e + 1])
        for s in range(lo, hi, unit):
            rows += [s, min(s + unit, hi) - 1]
    toks = set(pt[np.asarray(rows, np.int64)].tolist()) if rows else set()
    if n_shared:
        for s in range(0, T, unit):
            toks.update((s, min(s + unit, T) - 1))
    return np.array(sorted(toks), np.int64)


def oracle_layer(wl, rows=None, return_routing=False):
    """The oracle on workload wl, optionally on a subset of token rows."""
    xv = act_values(wl)
    if rows is not None:
        xv = xv[np.asarray(rows)]
    spec = wl.spec

    def expert(e):
        return (_w_values(wl.w13[e], None if wl.w13_s is None else wl.w13_s[e], None),
                _w_values(wl.w2[e], None if wl.w2_s is None else wl.w2_s[e], None))

    shared = []
    for s in range(spec.n_shared):
        shared.append((lambda s=s: (
            _w_values(wl.ws13[s], None if wl.ws13_s is None else wl.ws13_s[s], None),
            _w_values(wl.ws2[s], None if wl.ws2_s is None else wl.ws2_s[s], None))))
    bias = None if wl.sel_bias is None else wl.sel_bias.double().numpy()
    expert_x = None
    if spec.act == "bf16" and spec.weight in ("e4m3", "e2m1"):
        # bf16 activations into e4m3 / FP4 experts: the experts take x quantised to e4m3
        expert_x = quantised_values(xv)
    return oracle.layer_forward(xv, wl.wr.double().numpy(), spec.score, spec.top_k, expert, spec.E,
                                shared, sel_bias=bias, return_routing=return_routing,
                                expert_x=expert_x)


def quantised_values(x):
    """The values of the oracle's e4m3 block quantisation of x (1 x 128 blocks)."""
    codes, sc = oracle.quantize_e4m3_blocks(x)
    return dequant_fast(codes, sc, 1, 128)
