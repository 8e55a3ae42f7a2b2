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
    """U(-3, 3) fp32 logits whose rows are redrawn until the top k+1 keys are >= margin apart."""
    redraw = {}
    while True:
        L = inputs.draw_logits(T, E, seed, redraw=sorted(redraw.items()), stream=stream)
        keys = oracle.selection_keys(L.astype(np.float64), score,
                                     None if bias is None else np.asarray(bias, np.float64))
        bad = np.nonzero(topk_gaps(keys, k) < margin)[0]
        if bad.size == 0:
            return L
        for t in bad:
            redraw[int(t)] = redraw.get(int(t), 0) + 1


def act_values(wl) -> np.ndarray:
    if wl.spec.act == "e4m3":
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
        xv = x.double().numpy() if spec.act != "e4m3" else oracle.dequantize_blocks(
            x.view(torch.uint8).numpy(), xs.numpy(), 1, 128)
        keys = oracle.selection_keys(oracle.router_logits(xv, wr), spec.score, b64)
        bad = np.nonzero(topk_gaps(keys, spec.top_k) < spec.margin)[0]
        if bad.size == 0:
            break
        for t in bad:
            attempts[int(t)] = attempts.get(int(t), 0) + 1
    return inputs.make_workload(spec, seed, redraw=sorted(attempts.items()), threads=threads)


def _w_values(w, s, shape_blocks):
    if s is None:
        return w.double().numpy()
    return oracle.dequantize_blocks(w.view(torch.uint8).numpy(), s.numpy(), 128, 128)


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
    return oracle.layer_forward(xv, wl.wr.double().numpy(), spec.score, spec.top_k, expert, spec.E,
                                shared, sel_bias=bias, return_routing=return_routing)
