"""Write the stored input recipes of the named workloads (seed 0).

A recipe holds what the input generator cannot derive without the layer's
arithmetic:

* ``redraw``: activation rows that were redrawn (row, attempt) until, for
  every token, consecutive fp64 selection keys among its k+1 largest differ
  by at least ``margin``, so that the selection and the slot order are both
  well defined under fp32 accumulation;
* ``sel_bias`` (Zipf workloads): the per-expert selection bias fitted so that
  the realised expert loads follow the target loads of Zipf(1.1) sampling
  (Gumbel-top-k, k distinct experts per token); see ``fit_bias``;
* ``realised_loads``: the expert loads the recipe's inputs produce.

It calls only the oracle and the input generator's raw draws.  Run from the
repository root:  python tests/golden/make_recipes.py [name ...]
"""
from __future__ import annotations

import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from sparse_expert_moe_b200 import inputs  # noqa: E402

FIT_STEPS = 60
FIT_ETA = 0.5


def _values(spec, x32):
    """Real values the layer sees for fp32 activation draws x32 (after storage encoding)."""
    x, xs = inputs.encode_act(spec, x32)
    if inputs.is_e4m3(spec.act):
        import torch
        return oracle.dequantize_blocks(x.view(torch.uint8).numpy(), xs.numpy(), 1, 128)
    return x.double().numpy()


def _keys(spec, xv, wr, bias):
    logits = oracle.router_logits(xv, wr)
    return oracle.selection_keys(logits, spec.score, bias)


def _gaps(spec, keys):
    """Smallest gap between consecutive keys among each token's k+1 largest: the selection
    and the slot order are then both decided by more than ``margin``."""
    s = -np.sort(-keys, axis=1)
    m = min(spec.top_k + 1, spec.E)
    if m < 2:
        return np.full(keys.shape[0], np.inf)
    return (s[:, : m - 1] - s[:, 1:m]).min(axis=1)


def fit_bias(spec, xv, wr, target):
    """Per-expert selection bias whose realised loads match ``target``.

    Coordinate reading of the selection rule: with the other experts' keys
    fixed, expert e is selected by token t exactly when
    s(t, e) + b_e > thr(t, e), thr being the k-th largest key among the other
    experts.  So the b_e that gives e exactly target_e tokens lies between the
    target_e-th and (target_e+1)-th smallest value of thr(t, e) - s(t, e).
    Damped Jacobi sweeps of that update; the best sweep (least total load
    error) is kept.
    """
    logits = oracle.router_logits(xv, wr)
    s = oracle.selection_keys(logits, spec.score, None)
    T, E = s.shape
    k = spec.top_k
    b = np.zeros(E)
    best, best_err = b.copy(), None
    for _ in range(FIT_STEPS):
        keys = s + b[None, :]
        srt = -np.sort(-keys, axis=1)
        kth, k1th = srt[:, k - 1], srt[:, k]
        sel = keys >= kth[:, None]
        thr = np.where(sel, k1th[:, None], kth[:, None])
        v = np.sort(thr - s, axis=0)                       # [T, E] ascending per expert
        tgt = np.clip(target, 1, T - 1)
        lo = v[tgt - 1, np.arange(E)]
        hi = v[tgt, np.arange(E)]
        b_new = 0.5 * (lo + hi)
        loads = sel.sum(axis=0)
        err = int(np.abs(loads - target).sum())
        if best_err is None or err < best_err:
            best, best_err = b.copy(), err
        b = b + FIT_ETA * (b_new - b)
    return best.astype(np.float32)


def make(name: str, seed: int = 0) -> dict:
    spec = inputs.SPECS[name]
    wr = inputs.draw_router(spec, seed).double().numpy()
    x32 = inputs._draw_x_fp32(spec, seed, None)
    rec = {"config": name, "seed": seed, "margin": spec.margin,
           "generator": "sparse_expert_moe_b200/inputs.py",
           "script": "tests/golden/make_recipes.py"}
    if spec.loads == "zipf" and name not in inputs.BIAS_SOURCE:
        target = inputs.zipf_assignment(spec, seed)
        bias = fit_bias(spec, _values(spec, x32), wr, target)
        rec["zipf_target_loads"] = target.tolist()
        rec["sel_bias"] = bias.tolist()
    elif name in inputs.BIAS_SOURCE:
        bias = np.asarray(inputs.load_recipe(inputs.BIAS_SOURCE[name])["sel_bias"], np.float32)
    else:
        b = inputs.draw_sel_bias(spec, seed)
        bias = None if b is None else b.numpy()
    bias64 = None if bias is None else bias.astype(np.float64)

    attempts = np.zeros(spec.T, np.int64)
    xv = _values(spec, x32)
    bad = np.nonzero(_gaps(spec, _keys(spec, xv, wr, bias64)) < spec.margin)[0]
    while bad.size:
        for t in bad:
            attempts[t] += 1
            x32[t] = inputs.redraw_row(spec, seed, int(t), int(attempts[t]))
        # encode whole matrices: a storage whose block scales carry per-matrix factors
        # ("e4m3_fs") does not encode a subset of rows the same way
        xv_bad = _values(spec, x32)[bad]
        gaps = _gaps(spec, _keys(spec, xv_bad, wr, bias64))
        bad = bad[gaps < spec.margin]
    rec["redraw"] = [[int(t), int(a)] for t, a in enumerate(attempts) if a]
    xv = _values(spec, x32)
    idx = oracle.select_topk(_keys(spec, xv, wr, bias64), spec.top_k)
    loads = np.bincount(idx.ravel(), minlength=spec.E)
    rec["realised_loads"] = loads.tolist()
    rec["load_summary"] = {"max": int(loads.max()), "median": float(np.median(loads)),
                           "min": int(loads.min()), "empty": int((loads == 0).sum())}
    return rec


def main(names):
    os.makedirs(inputs.RECIPE_DIR, exist_ok=True)
    for name in names:
        rec = make(name)
        with open(os.path.join(inputs.RECIPE_DIR, f"{name}.json"), "w") as f:
            json.dump(rec, f, indent=1)
        print(name, "redrawn rows:", len(rec["redraw"]), "loads:", rec["load_summary"])


if __name__ == "__main__":
    main(sys.argv[1:] or ["tiny", "r1_decode", "r1_prefill", "kimi", "r1_prefill_fp8"])
