"""fp64 CPU oracle for the Mixture-of-Experts feed-forward layer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may use it.  It shares no code with
the CUDA library (no kernels, headers, helpers or constant tables); the two
meet only in the seeded input generators, which hold none of the layer's
arithmetic.

What it computes is the layer the pages state as the ``moe_ffn`` pseudocode
in "Decoding Trillion-Parameter MoE LLMs: Sparse Architecture and Agentic
Intelligence", section "Routing: Top-K Experts Plus a Shared Expert":

    logits = gate(x)
    weights, idx = topk_softmax(logits, k)
    out = sum_k weights[:, k] * expert_{idx[:, k]}(x) + sum_s shared_s(x)

written out step by step, in fp64, with no rounding between the steps and no
blocking, fusion or reordering beyond what that definition states.  Library
primitives (a matrix product, a stable sort, ``bincount``/``cumsum``) serve as
single steps.  Readings of points the pages leave open:

* Sigmoid scoring with a per-expert selection bias is the "auxiliary-loss-free
  bias routing" that "Chapter 7: Serving Mega MoE at scale" (roadmap item
  "Architectural Foundations of Trillion-Parameter Sparse MoE Models") names
  without a formula.  Reading: score s = sigmoid(l); the bias is added for
  selection only; gates are the unbiased scores of the selected experts
  renormalised to sum to one.  No group-limited pre-selection, scale 1.0.
* ``topk_softmax``: the k largest logits are selected (softmax is monotone)
  and the softmax is taken over the selected logits, which equals the full
  softmax renormalised over the selection.
* Ties: slots are ordered by key descending, equal keys by lower expert index.
* Expert network: SwiGLU, h = silu(x W1^T) * (x W3^T), y = h W2^T with
  silu(z) = z / (1 + exp(-z)); W13 stacks the gate block W1 over the up block
  W3; no biases ("GC-MoE: Overlapping Expert-Parallel Token Dispatch with
  FP8/FP4 Grouped GEMM via CUDA Green Contexts", key change on fused SwiGLU).
* Dispatch on one GPU is a permutation of token rows into per-expert
  contiguous groups, expert-major, ascending token order inside a group.
* FP8 inputs are e4m3 codes times power-of-two block scales; the oracle
  decodes the codes from the OCP OFP8 E4M3 definition and multiplies the scale
  in, exactly, in fp64.
* FP4 ("FP8/FP4 Grouped GEMM" in the GC-MoE title names the precision, not the
  format).  Reading: the OCP Microscaling (MX) MXFP4 format -- E2M1 elements,
  two per byte (the even element in the low nibble), one E8M0 scale per 32
  consecutive elements along K.  The oracle decodes both from their
  definitions and multiplies, exactly, in fp64.

Every function is pinned by ``tests/test_oracle_pins.py`` (closed forms,
brute force over expert subsets, library special cases, invariants and the
hand-derived fixtures in ``tests/golden/``).
"""
from __future__ import annotations

import numpy as np

SOFTMAX = "softmax"
SIGMOID_BIAS = "sigmoid_bias"


# ---------------------------------------------------------------------------
# Input decoding
# ---------------------------------------------------------------------------

def decode_e4m3(codes) -> np.ndarray:
    """Decode OCP OFP8 E4M3 byte codes to fp64.

    Format (OCP 8-bit Floating Point Specification, E4M3): 1 sign bit,
    4 exponent bits with bias 7, 3 mantissa bits; exponent field 0 encodes
    subnormals m/8 * 2^-6; S.1111.111 is NaN; there are no infinities, so the
    largest finite magnitude is 1.75 * 2^8 = 448.
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    exp = (c >> 3) & 0xF
    man = (c & 0x7).astype(np.float64)
    normal = (1.0 + man / 8.0) * np.exp2(exp.astype(np.float64) - 7.0)
    sub = (man / 8.0) * np.exp2(-6.0)
    val = np.where(exp == 0, sub, normal)
    val = np.where((exp == 0xF) & ((c & 0x7) == 0x7), np.nan, val)
    return sign * val


def dequantize_blocks(q_codes, scales, block_rows: int, block_cols: int) -> np.ndarray:
    """Block-scaled FP8 to fp64: value[r, c] = e4m3(q[r, c]) * scales[r // br, c // bc].

    Activations use 1x128 blocks (one scale per token per 128 channels),
    weights 128x128 blocks.  The pages say only "block-scaled"; the block
    shapes are the workload's.
    """
    v = decode_e4m3(q_codes)
    s = np.asarray(scales, dtype=np.float64)
    s = np.repeat(np.repeat(s, block_rows, axis=0), block_cols, axis=1)
    return v * s[: v.shape[0], : v.shape[1]]


def decode_e2m1(codes) -> np.ndarray:
    """Decode 4-bit FP4 E2M1 codes (the low 4 bits of each value) to fp64.

    Format (OCP Microscaling Formats (MX) v1.0, element type FP4 E2M1): 1 sign
    bit, 2 exponent bits with bias 1, 1 mantissa bit; exponent field 0 encodes
    the subnormals m/2 * 2^0; no infinities or NaN, so the largest magnitude is
    1.5 * 2^2 = 6.
    """
    c = np.asarray(codes).astype(np.int64) & 0xF
    sign = np.where(c & 0x8, -1.0, 1.0)
    exp = (c >> 1) & 0x3
    man = (c & 0x1).astype(np.float64)
    normal = (1.0 + man / 2.0) * np.exp2(exp.astype(np.float64) - 1.0)
    sub = man / 2.0
    return sign * np.where(exp == 0, sub, normal)


def unpack_fp4(packed) -> np.ndarray:
    """[R, C/2] bytes of packed FP4 codes -> [R, C] codes: byte j holds element 2j in its
    low nibble and element 2j+1 in its high nibble."""
    b = np.asarray(packed, np.uint8)
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), np.uint8)
    out[..., 0::2] = b & 0xF
    out[..., 1::2] = b >> 4
    return out


def decode_e8m0(codes) -> np.ndarray:
    """Decode E8M0 scale codes to fp64 (OCP MX v1.0, scale type E8M0): 8 exponent bits,
    bias 127, no sign and no mantissa, value 2^(code - 127); code 0xFF is NaN."""
    c = np.asarray(codes, np.uint8).astype(np.float64)
    return np.where(c == 255.0, np.nan, np.exp2(c - 127.0))


def dequantize_mxfp4(packed, scale_codes, block: int = 32) -> np.ndarray:
    """MXFP4 to fp64: value[r, c] = e2m1(code[r, c]) * e8m0(scale[r, c // block])."""
    v = decode_e2m1(unpack_fp4(packed))
    s = decode_e8m0(scale_codes)
    return v * np.repeat(s, block, axis=-1)[..., : v.shape[-1]]


def quantize_e4m3_blocks(x, block: int = 128):
    """Quantise rows to e4m3 with one power-of-two scale per `block` consecutive values of a
    row (the activation quantisation of the FP8 path; GC-MoE key change on fused
    requantisation).  Reading: the scale of a block is 2^e for the smallest integer e with
    amax <= 448 * 2^e (448 = the largest e4m3 magnitude; e = 0 for an all-zero block;
    e kept within the E8M0 range [-127, 127]); each value x / 2^e (exact: a power-of-two
    division) goes to the nearest e4m3 value, ties to the even code, with its sign (a
    negative value that rounds to zero gives negative zero).

    Returns (codes uint8 [R, C], scales fp64 [R, C / block])."""
    x = np.asarray(x, np.float64)
    R, C = x.shape
    amax = np.abs(x).reshape(R, C // block, block).max(axis=2)
    m, e = np.frexp(amax / 448.0)                   # amax / 448 = m * 2^e, m in [0.5, 1)
    e = np.where(m == 0.5, e - 1, e)                 # exact powers of two
    e = np.where(amax > 0, e, 0)
    e = np.clip(e, -127, 127)
    scales = np.exp2(e.astype(np.float64))
    q = x / np.repeat(scales, block, axis=1)
    # the non-negative finite e4m3 values in code order 0x00 .. 0x7E (increasing)
    values = decode_e4m3(np.arange(0x7F, dtype=np.uint8))
    a = np.abs(q)
    hi = np.clip(np.searchsorted(values, a, side="left"), 0, 0x7E)   # values[hi] >= a
    lo = np.clip(hi - 1, 0, 0x7E)
    d_lo, d_hi = a - values[lo], values[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    code = np.where(np.signbit(q), code | 0x80, code).astype(np.uint8)
    return code, scales


# ---------------------------------------------------------------------------
# Router: gate(x), scores, top-k, gates
# ---------------------------------------------------------------------------

def router_logits(x, wr) -> np.ndarray:
    """logits[t, e] = sum_i x[t, i] * Wr[e, i]  (the ``gate(x)`` step)."""
    return np.asarray(x, np.float64) @ np.asarray(wr, np.float64).T


def sigmoid(z) -> np.ndarray:
    z = np.asarray(z, np.float64)
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-z))


def selection_keys(logits, score: str, sel_bias=None) -> np.ndarray:
    """Key each expert is ranked by.

    softmax: the logit itself (softmax is monotone).
    sigmoid_bias: sigmoid(logit) + bias[e]; the bias steers selection only.
    """
    logits = np.asarray(logits, np.float64)
    if score == SOFTMAX:
        return logits.copy()
    if score == SIGMOID_BIAS:
        keys = sigmoid(logits)
        if sel_bias is not None:
            keys = keys + np.asarray(sel_bias, np.float64)[None, :]
        return keys
    raise ValueError(f"unknown score function {score!r}")


def select_topk(keys, k: int) -> np.ndarray:
    """Indices of the k largest keys per row, key descending, ties to the lower index.

    A stable sort of -key keeps equal keys in ascending expert order.
    """
    keys = np.asarray(keys, np.float64)
    order = np.argsort(-keys, axis=1, kind="stable")
    return order[:, :k].astype(np.int64)


def gate_weights(logits, idx, score: str) -> np.ndarray:
    """Renormalised gate weight of each selected expert.

    softmax: exp(l_j - max) / sum over the selected j.
    sigmoid_bias: sigmoid(l_j) / sum over the selected j (bias not included).
    """
    sel = np.take_along_axis(np.asarray(logits, np.float64), idx, axis=1)
    if score == SOFTMAX:
        e = np.exp(sel - sel.max(axis=1, keepdims=True))
        return e / e.sum(axis=1, keepdims=True)
    if score == SIGMOID_BIAS:
        s = sigmoid(sel)
        return s / s.sum(axis=1, keepdims=True)
    raise ValueError(f"unknown score function {score!r}")


def route(logits, score: str, k: int, sel_bias=None):
    """The ``topk_softmax`` step, generalised to both score functions.

    Returns (idx [T, k] int64, gates [T, k] fp64).
    """
    idx = select_topk(selection_keys(logits, score, sel_bias), k)
    return idx, gate_weights(logits, idx, score)


# ---------------------------------------------------------------------------
# Dispatch on one device: permutation into per-expert groups
# ---------------------------------------------------------------------------

def permute(idx, n_experts: int):
    """Group the T*k (token, slot) pairs by expert.

    Returns
      offsets    [E+1]  exclusive prefix of per-expert counts,
      perm_token [T*k]  token of each permuted row (expert-major, ascending token),
      inv_perm   [T, k] permuted row that holds (token t, slot j).
    """
    idx = np.asarray(idx, np.int64)
    T, k = idx.shape
    counts = np.bincount(idx.ravel(), minlength=n_experts)
    offsets = np.zeros(n_experts + 1, np.int64)
    offsets[1:] = np.cumsum(counts)
    cursor = offsets[:-1].copy()
    perm_token = np.empty(T * k, np.int64)
    inv_perm = np.empty((T, k), np.int64)
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            r = cursor[e]
            perm_token[r] = t
            inv_perm[t, j] = r
            cursor[e] += 1
    return offsets, perm_token, inv_perm


# ---------------------------------------------------------------------------
# Expert network
# ---------------------------------------------------------------------------

def silu(z) -> np.ndarray:
    z = np.asarray(z, np.float64)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def swiglu_expert(X, w13, w2) -> np.ndarray:
    """One expert on the rows X [n, d]: silu(X W1^T) * (X W3^T) then W2.

    w13 [2I, d] holds W1 (rows 0..I-1) over W3 (rows I..2I-1); w2 [d, I].
    """
    X = np.asarray(X, np.float64)
    w13 = np.asarray(w13, np.float64)
    w2 = np.asarray(w2, np.float64)
    inter = w13.shape[0] // 2
    gate = X @ w13[:inter].T
    up = X @ w13[inter:].T
    return (silu(gate) * up) @ w2.T


# ---------------------------------------------------------------------------
# Combine and the whole layer
# ---------------------------------------------------------------------------

def combine(y_perm, inv_perm, gates, y_shared=None) -> np.ndarray:
    """y[t] = sum_j gates[t, j] * y_perm[inv_perm[t, j]] (+ shared outputs), slot order."""
    y_perm = np.asarray(y_perm, np.float64)
    T, k = inv_perm.shape
    out = np.zeros((T, y_perm.shape[1]), np.float64)
    for j in range(k):
        out += gates[:, j : j + 1] * y_perm[inv_perm[:, j]]
    if y_shared is not None:
        for ys in y_shared:
            out += np.asarray(ys, np.float64)
    return out


def layer_forward(x, wr, score: str, k: int, expert_weights, n_experts: int,
                  shared_weights=(), sel_bias=None, return_routing: bool = False,
                  expert_x=None):
    """The whole layer, step by step.

    x               [T, d] activation values (already decoded to real numbers)
    expert_x        [T, d] the values the experts (routed and shared) take instead of x,
                    e.g. x quantised for FP8 expert weights; the router always takes x
    wr              [E, d] router weights
    expert_weights  callable e -> (w13 [2I, d], w2 [d, I]); called once per
                    expert that has at least one row, so only one expert's
                    weights need to be held in fp64 at a time
    shared_weights  sequence of callables () -> (w13, w2), or of tuples
    """
    x = np.asarray(x, np.float64)
    logits = router_logits(x, wr)
    idx, gates = route(logits, score, k, sel_bias)
    offsets, perm_token, inv_perm = permute(idx, n_experts)
    if expert_x is not None:
        x = np.asarray(expert_x, np.float64)
    x_perm = x[perm_token]
    d = x.shape[1]
    y_perm = np.zeros((x_perm.shape[0], d), np.float64)
    for e in range(n_experts):
        lo, hi = offsets[e], offsets[e + 1]
        if hi == lo:
            continue
        w13, w2 = expert_weights(e)
        y_perm[lo:hi] = swiglu_expert(x_perm[lo:hi], w13, w2)
    shared_out = []
    for sw in shared_weights:
        w13, w2 = sw() if callable(sw) else sw
        shared_out.append(swiglu_expert(x, w13, w2))
    y = combine(y_perm, inv_perm, gates, shared_out)
    if return_routing:
        return y, dict(logits=logits, idx=idx, gates=gates, offsets=offsets,
                       perm_token=perm_token, inv_perm=inv_perm)
    return y
