"""The oracle's pins catch plausible mistakes: each case below plants one bug in the
oracle (on the CPU, for the duration of the case) and runs every pin of
``test_oracle_pins.py``; at least one pin must fail.  Without a planted bug every pin
passes."""
import contextlib
import importlib.util
import os

import numpy as np
import pytest

import oracle
import oracle.moe_oracle as om

_PINS_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "test_oracle_pins.py")


def _pins():
    spec = importlib.util.spec_from_file_location("oracle_pins_for_mutations", _PINS_PATH)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    calls = []
    for name in sorted(dir(mod)):
        fn = getattr(mod, name)
        if not (name.startswith("test_") and callable(fn)):
            continue
        marks = [m for m in getattr(fn, "pytestmark", []) if m.name == "parametrize"]
        if not marks:
            calls.append((name, fn, ()))
            continue
        argnames, argvalues = marks[0].args[0], marks[0].args[1]
        multi = "," in argnames
        for v in argvalues:
            calls.append((name, fn, tuple(v) if multi else (v,)))
    return calls


def _failing_pins():
    failed = []
    for name, fn, args in _pins():
        try:
            with np.errstate(all="ignore"):
                fn(*args)
        except Exception:             # an assertion or any error the bug provokes
            failed.append(name)
    return failed


@contextlib.contextmanager
def _planted(name, replacement):
    """Replace oracle function `name` in the module (internal calls) and the package
    (the pins' calls)."""
    saved = getattr(om, name)
    setattr(om, name, replacement)
    setattr(oracle, name, replacement)
    try:
        yield
    finally:
        setattr(om, name, saved)
        setattr(oracle, name, saved)


# ---- the planted bugs: each a plausible slip in one step ---------------------------

def _topk_ties_to_higher_index(keys, k):
    keys = np.asarray(keys, np.float64)
    E = keys.shape[1]
    order = np.argsort(-keys[:, ::-1], axis=1, kind="stable")
    return (E - 1 - order)[:, :k].astype(np.int64)


def _topk_slots_ascending(keys, k):
    keys = np.asarray(keys, np.float64)
    return np.argsort(-keys, axis=1, kind="stable")[:, :k][:, ::-1].astype(np.int64)


def _gates_full_softmax_not_renormalised(logits, idx, score):
    L = np.asarray(logits, np.float64)
    if score == om.SOFTMAX:
        e = np.exp(L - L.max(axis=1, keepdims=True))
        return np.take_along_axis(e / e.sum(axis=1, keepdims=True), idx, axis=1)
    return _REAL["gate_weights"](logits, idx, score)


def _gates_sigmoid_not_renormalised(logits, idx, score):
    if score == om.SIGMOID_BIAS:
        return om.sigmoid(np.take_along_axis(np.asarray(logits, np.float64), idx, axis=1))
    return _REAL["gate_weights"](logits, idx, score)


def _route_gates_from_biased_keys(logits, score, k, sel_bias=None):
    keys = om.selection_keys(logits, score, sel_bias)
    idx = om.select_topk(keys, k)
    if score == om.SIGMOID_BIAS:
        s = np.take_along_axis(keys, idx, axis=1)
        return idx, s / s.sum(axis=1, keepdims=True)
    return idx, om.gate_weights(logits, idx, score)


def _keys_without_bias(logits, score, sel_bias=None):
    return _REAL["selection_keys"](logits, score, None)


def _silu_wrong_sign(z):
    z = np.asarray(z, np.float64)
    return z / (1.0 + np.exp(z))


def _swiglu_gate_and_up_swapped(X, w13, w2):
    X, w13, w2 = (np.asarray(a, np.float64) for a in (X, w13, w2))
    inter = w13.shape[0] // 2
    return (om.silu(X @ w13[inter:].T) * (X @ w13[:inter].T)) @ w2.T


def _combine_without_shared(y_perm, inv_perm, gates, y_shared=None):
    return _REAL["combine"](y_perm, inv_perm, gates, None)


def _combine_by_slot_not_inv_perm(y_perm, inv_perm, gates, y_shared=None):
    T, k = inv_perm.shape
    rows = np.arange(T * k).reshape(T, k)
    return _REAL["combine"](y_perm, rows, gates, y_shared)


def _permute_descending_tokens(idx, n_experts):
    idx = np.asarray(idx, np.int64)
    T, k = idx.shape
    counts = np.bincount(idx.ravel(), minlength=n_experts)
    offsets = np.zeros(n_experts + 1, np.int64)
    offsets[1:] = np.cumsum(counts)
    cursor = offsets[1:].copy()
    perm_token = np.empty(T * k, np.int64)
    inv_perm = np.empty((T, k), np.int64)
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            cursor[e] -= 1
            perm_token[cursor[e]] = t
            inv_perm[t, j] = cursor[e]
    return offsets, perm_token, inv_perm


def _e4m3_exponent_bias_8(codes):
    return _REAL["decode_e4m3"](codes) / 2.0


def _dequant_scales_transposed(q_codes, scales, block_rows, block_cols):
    s = np.asarray(scales, np.float64)
    return _REAL["dequantize_blocks"](q_codes, s.T if s.shape[0] == s.shape[1] else s[::-1],
                                      block_rows, block_cols)


def _e2m1_exponent_bias_0(codes):
    return _REAL["decode_e2m1"](codes) * 2.0


def _fp4_nibbles_swapped(packed):
    out = _REAL["unpack_fp4"](packed)
    return out.reshape(out.shape[:-1] + (-1, 2))[..., ::-1].reshape(out.shape)


def _e8m0_bias_128(codes):
    return _REAL["decode_e8m0"](codes) / 2.0


def _quantise_ties_away_from_zero(x, block=128):
    codes, sc = _REAL["quantize_e4m3_blocks"](x, block)
    q = np.abs(np.asarray(x, np.float64) / np.repeat(sc, block, axis=1))
    vals = om.decode_e4m3(np.arange(0x7F, dtype=np.uint8))
    c = codes & 0x7F
    tie = (c < 0x7E) & (q == (vals[np.minimum(c, 0x7D)] + vals[np.minimum(c, 0x7D) + 1]) / 2)
    return np.where(tie, codes + 1, codes).astype(np.uint8), sc


def _quantise_scale_half(x, block=128):
    codes, sc = _REAL["quantize_e4m3_blocks"](np.asarray(x) * 2.0, block)
    return codes, sc / 2.0


def _router_logits_without_transpose(x, wr):
    x, wr = np.asarray(x, np.float64), np.asarray(wr, np.float64)
    return x @ wr.reshape(wr.shape[1], wr.shape[0])


_REAL = {n: getattr(om, n) for n in ("gate_weights", "selection_keys", "combine", "decode_e4m3",
                                      "dequantize_blocks", "decode_e2m1", "unpack_fp4",
                                      "decode_e8m0", "quantize_e4m3_blocks")}

MUTATIONS = [
    ("select_topk", _topk_ties_to_higher_index),
    ("select_topk", _topk_slots_ascending),
    ("gate_weights", _gates_full_softmax_not_renormalised),
    ("gate_weights", _gates_sigmoid_not_renormalised),
    ("route", _route_gates_from_biased_keys),
    ("selection_keys", _keys_without_bias),
    ("silu", _silu_wrong_sign),
    ("swiglu_expert", _swiglu_gate_and_up_swapped),
    ("combine", _combine_without_shared),
    ("combine", _combine_by_slot_not_inv_perm),
    ("permute", _permute_descending_tokens),
    ("decode_e4m3", _e4m3_exponent_bias_8),
    ("dequantize_blocks", _dequant_scales_transposed),
    ("router_logits", _router_logits_without_transpose),
    ("decode_e2m1", _e2m1_exponent_bias_0),
    ("unpack_fp4", _fp4_nibbles_swapped),
    ("decode_e8m0", _e8m0_bias_128),
    ("quantize_e4m3_blocks", _quantise_ties_away_from_zero),
    ("quantize_e4m3_blocks", _quantise_scale_half),
]


def test_every_pin_passes_without_a_planted_bug():
    assert _failing_pins() == []


@pytest.mark.parametrize("name,bug", MUTATIONS, ids=[b.__name__.lstrip("_") for _, b in MUTATIONS])
def test_planted_bug_is_caught(name, bug):
    with _planted(name, bug):
        failed = _failing_pins()
    assert failed, f"no pin catches {bug.__name__} in {name}"
