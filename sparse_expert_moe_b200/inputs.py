"""Seeded synthetic inputs for the MoE layer.

This module is shared by the oracle tests, the GPU parity tests, ``bench.py``
and ``smoke()``.  It holds none of the layer's arithmetic: it only draws
random numbers, encodes the drawn values in the storage types the layer
consumes (bf16 round-to-nearest-even, e4m3 with power-of-two block scales),
and applies a stored per-workload recipe (rows to redraw so that routing has a
score margin -- consecutive keys among each token's k+1 largest differ by at
least the margin -- and for the Zipf workloads a fitted selection bias).  Recipes are
JSON files under ``tests/golden/recipes/``, written by
``tests/golden/make_recipes.py``, which computes them with the oracle only.

Every tensor is drawn from its own numpy ``Generator(PCG64)`` stream keyed by
(seed, family, tensor, index), so one expert's weights can be redrawn alone
and the result does not depend on the number of threads used.

Workloads (shapes from the pages: DeepSeek R1 in the InferenceX v2 claim
record IX2-0397, section "WideEP" -- 256 routed experts, 1 shared, 8 per
token; "Decoding Trillion-Parameter MoE LLMs", section "Expert Granularity:
More, Smaller Experts" -- 384 experts, top-8 plus one shared expert):

  tiny            T=64   d=128  E=8   k=2 I=256  S=0 softmax       fp32
  r1_decode       T=128  d=7168 E=256 k=8 I=2048 S=1 sigmoid+bias  bf16
  r1_decode_uniform  r1_decode's activations with no selection bias: uniform routing,
                  about 252 of the 256 experts touched per batch
  r1_prefill      T=8192 d=7168 E=256 k=8 I=2048 S=1 sigmoid+bias  bf16, Zipf(1.1) loads
  kimi            T=4096 d=7168 E=384 k=8 I=2048 S=1 sigmoid+bias  bf16
  r1_prefill_fp8  r1_prefill with e4m3 activations (1x128 scales) and e4m3
                  weights (128x128 scales), bf16 output
  r1_decode_fp8   r1_decode with e4m3 activations and e4m3 weights
  r1_decode_fp4   r1_decode with e4m3 activations and MXFP4 weights (E2M1 codes, one E8M0
                  scale per 32 elements along K)
  r1_decode_fp4q  r1_decode (bf16 activations) with MXFP4 weights: the activations are
                  quantised to e4m3 in the permutation
  r1_decode_fp8s  r1_decode_fp8 with block scales that are not powers of two (each scale
                  multiplied by a seeded factor in [1, 2))
"""
from __future__ import annotations

import json
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace
from typing import Optional

import numpy as np
import torch

RECIPE_DIR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                          "tests", "golden", "recipes")

# stream ids
_X, _WR, _BIAS, _W13, _W2, _WS13, _WS2, _XRE, _LOGITS, _ZIPF, _FS = range(1, 12)
_FAMILY = {"tiny": 1, "r1": 2, "kimi": 3, "custom": 9}

W_STD = 0.02
E4M3_MAX = 448.0


@dataclass(frozen=True)
class Spec:
    name: str
    T: int
    d_model: int
    E: int
    top_k: int
    d_ff: int
    n_shared: int
    score: str            # "softmax" | "sigmoid_bias"
    act: str              # "f32" | "bf16" | "e4m3"
    weight: str           # "f32" | "bf16" | "e4m3"
    out: str              # "f32" | "bf16"
    family: str           # weight-draw family: workloads of one family share weights
    x_stream: int         # activation-draw stream
    loads: str = "uniform"            # "uniform" | "zipf"
    bias_range: Optional[float] = None  # sel bias ~ U(-r, r) when drawn
    margin: float = 1e-3
    zipf_s: float = 1.1


SPECS = {
    "tiny": Spec("tiny", 64, 128, 8, 2, 256, 0, "softmax", "f32", "f32", "f32",
                 family="tiny", x_stream=1, margin=1e-2),
    "r1_decode": Spec("r1_decode", 128, 7168, 256, 8, 2048, 1, "sigmoid_bias", "bf16", "bf16",
                      "bf16", family="r1", x_stream=2, bias_range=0.1),
    "r1_decode_uniform": Spec("r1_decode_uniform", 128, 7168, 256, 8, 2048, 1, "sigmoid_bias",
                              "bf16", "bf16", "bf16", family="r1", x_stream=2),
    "r1_prefill": Spec("r1_prefill", 8192, 7168, 256, 8, 2048, 1, "sigmoid_bias", "bf16", "bf16",
                       "bf16", family="r1", x_stream=3, loads="zipf"),
    "kimi": Spec("kimi", 4096, 7168, 384, 8, 2048, 1, "sigmoid_bias", "bf16", "bf16", "bf16",
                 family="kimi", x_stream=4),
    "r1_decode_fp8": Spec("r1_decode_fp8", 128, 7168, 256, 8, 2048, 1, "sigmoid_bias", "e4m3",
                          "e4m3", "bf16", family="r1", x_stream=2, bias_range=0.1),
    "r1_decode_fp4": Spec("r1_decode_fp4", 128, 7168, 256, 8, 2048, 1, "sigmoid_bias", "e4m3",
                          "e2m1", "bf16", family="r1", x_stream=2, bias_range=0.1),
    "r1_decode_fp4q": Spec("r1_decode_fp4q", 128, 7168, 256, 8, 2048, 1, "sigmoid_bias", "bf16",
                           "e2m1", "bf16", family="r1", x_stream=2, bias_range=0.1),
    "r1_decode_fp8s": Spec("r1_decode_fp8s", 128, 7168, 256, 8, 2048, 1, "sigmoid_bias", "e4m3_fs",
                           "e4m3_fs", "bf16", family="r1", x_stream=2, bias_range=0.1),
    "r1_prefill_fp8": Spec("r1_prefill_fp8", 8192, 7168, 256, 8, 2048, 1, "sigmoid_bias", "e4m3",
                           "e4m3", "bf16", family="r1", x_stream=3, loads="zipf"),
}

# the Zipf workload whose fitted selection bias the FP8 variant reuses
BIAS_SOURCE = {"r1_prefill_fp8": "r1_prefill"}


def custom_spec(T, d_model, E, top_k, d_ff, n_shared=0, score="sigmoid_bias", act="bf16",
                weight="bf16", out="bf16", bias_range=0.1, x_stream=7, margin=1e-3):
    """A small workload for parity tests (own weight family, no stored recipe)."""
    return Spec(f"custom_T{T}_d{d_model}_E{E}_k{top_k}_I{d_ff}_S{n_shared}", T, d_model, E, top_k,
                d_ff, n_shared, score, act, weight, out, family="custom", x_stream=x_stream,
                bias_range=bias_range if score == "sigmoid_bias" else None, margin=margin)


def _rng(seed, *key):
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), *map(int, key)])))


# ---------------------------------------------------------------------------
# storage encodings of drawn values
# ---------------------------------------------------------------------------

def to_bf16(a: np.ndarray) -> torch.Tensor:
    """fp32 draw -> bf16 tensor (round to nearest even)."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def _pow2_scale(amax: np.ndarray) -> np.ndarray:
    """Smallest power of two s with amax / s <= 448 (1.0 for an all-zero block)."""
    v = np.asarray(amax, np.float64) / E4M3_MAX
    m, e = np.frexp(v)                  # v = m * 2^e, m in [0.5, 1)
    e = np.where(m == 0.5, e - 1, e)    # exact powers of two
    s = np.ldexp(1.0, e.astype(np.int64))
    return np.where(v > 0, s, 1.0).astype(np.float32)


def to_e4m3_blocks(a: np.ndarray, br: int, bc: int):
    """fp32 draw [R, C] -> (e4m3 codes as torch.float8_e4m3fn [R, C], fp32 scales [R/br, C/bc])."""
    R, C = a.shape
    blocks = np.abs(a).reshape(R // br, br, C // bc, bc).max(axis=(1, 3))
    s = _pow2_scale(blocks)
    full = np.repeat(np.repeat(s, br, axis=0), bc, axis=1)
    q = torch.from_numpy(np.ascontiguousarray(a / full, dtype=np.float32)).to(torch.float8_e4m3fn)
    return q, torch.from_numpy(s)


E2M1_MAX = 6.0


def to_mxfp4(a: np.ndarray, block: int = 32):
    """fp32 draw [R, C] -> MXFP4: (packed E2M1 codes as uint8 [R, C/2], the even element in
    the low nibble; E8M0 scale codes as uint8 [R, C/block]).

    Each 1 x block run along C shares the smallest power-of-two scale s with amax / s <= 6
    (E2M1's largest magnitude; 1.0 for an all-zero block); the elements a / s are rounded
    to the nearest E2M1 value, ties to even (ml_dtypes' float4_e2m1fn conversion)."""
    import ml_dtypes
    R, C = a.shape
    amax = np.abs(a).reshape(R, C // block, block).max(axis=2)
    v = np.asarray(amax, np.float64) / E2M1_MAX
    m, e = np.frexp(v)
    e = np.where(m == 0.5, e - 1, e)                    # exact powers of two
    e = np.where(v > 0, e, 0)
    q = (np.asarray(a, np.float32) / np.repeat(np.ldexp(1.0, e), block, axis=1).astype(np.float32))
    codes = q.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return torch.from_numpy(packed), torch.from_numpy((e + 127).astype(np.uint8))


def scale_atoms(codes):
    """E8M0 codes [R, K/32] -> the ABI's scale atoms [R/128, K/128, 512]: row r, run q of an
    atom at byte (r % 32) * 16 + (r / 32) * 4 + q (a pure reordering of the bytes)."""
    c = np.asarray(codes, np.uint8)
    R, Q = c.shape
    a = c.reshape(R // 128, 4, 32, Q // 4, 4)           # [rb, r / 32, r % 32, kb, q]
    return torch.from_numpy(np.ascontiguousarray(a.transpose(0, 3, 2, 1, 4)).reshape(R // 128, Q // 4, 512))


def scale_rows(atoms):
    """The inverse of scale_atoms: [R/128, K/128, 512] -> [R, K/32]."""
    a = np.asarray(atoms, np.uint8)
    RB, KB, _ = a.shape
    b = a.reshape(RB, KB, 32, 4, 4).transpose(0, 3, 2, 1, 4)   # [rb, r / 32, r % 32, kb, q]
    return torch.from_numpy(np.ascontiguousarray(b).reshape(RB * 128, KB * 4))


# ---------------------------------------------------------------------------
# draws
# ---------------------------------------------------------------------------

def _draw_x_fp32(spec: Spec, seed: int, redraw) -> np.ndarray:
    x = _rng(seed, _FAMILY[spec.family], _X, spec.x_stream).standard_normal(
        (spec.T, spec.d_model), dtype=np.float32)
    for t, attempt in (redraw or []):
        x[t] = redraw_row(spec, seed, t, attempt)
    return x


def redraw_row(spec: Spec, seed: int, t: int, attempt: int) -> np.ndarray:
    """Replacement draw number ``attempt`` (>= 1) for activation row t."""
    return _rng(seed, _FAMILY[spec.family], _XRE, spec.x_stream, t, attempt).standard_normal(
        spec.d_model, dtype=np.float32)


def is_e4m3(dtype: str) -> bool:
    """e4m3 storage: power-of-two block scales ("e4m3") or any fp32 block scales ("e4m3_fs")."""
    return dtype in ("e4m3", "e4m3_fs")


def _fs_mantissas(shape, *key):
    """Block-scale multipliers in [1, 2) for the "e4m3_fs" storage: the stored values are the
    e4m3 codes times (power-of-two scale x multiplier), so no block scale is a power of two."""
    return _rng(0, _FS, *key).uniform(1.0, 2.0, shape).astype(np.float32)


def encode_act(spec: Spec, x32: np.ndarray):
    if spec.act == "f32":
        return torch.from_numpy(np.ascontiguousarray(x32)), None
    if spec.act == "bf16":
        return to_bf16(x32), None
    if spec.act == "e4m3":
        return to_e4m3_blocks(x32, 1, 128)
    if spec.act == "e4m3_fs":
        q, s = to_e4m3_blocks(x32, 1, 128)
        m = _fs_mantissas(s.shape, _FAMILY[spec.family], spec.x_stream, spec.T, spec.d_model)
        return q, torch.from_numpy(s.numpy() * m)
    raise ValueError(spec.act)


def _encode_weight(spec: Spec, w32: np.ndarray, key=()):
    if spec.weight == "f32":
        return torch.from_numpy(np.ascontiguousarray(w32)), None
    if spec.weight == "bf16":
        return to_bf16(w32), None
    if spec.weight == "e4m3":
        return to_e4m3_blocks(w32, 128, 128)
    if spec.weight == "e2m1":
        q, s = to_mxfp4(w32)
        return q, scale_atoms(s.numpy())
    if spec.weight == "e4m3_fs":
        q, s = to_e4m3_blocks(w32, 128, 128)
        return q, torch.from_numpy(s.numpy() * _fs_mantissas(s.shape, _FAMILY[spec.family], *key))
    raise ValueError(spec.weight)


def draw_expert(spec: Spec, seed: int, e: int, shared: bool = False):
    """(w13, w13_scale, w2, w2_scale) of routed expert e or shared expert e."""
    fam = _FAMILY[spec.family]
    I, d = spec.d_ff, spec.d_model
    r13 = _rng(seed, fam, _WS13 if shared else _W13, e)
    w13 = r13.standard_normal((2 * I, d), dtype=np.float32)
    w13 *= np.float32(W_STD)
    r2 = _rng(seed, fam, _WS2 if shared else _W2, e)
    w2 = r2.standard_normal((d, I), dtype=np.float32)
    w2 *= np.float32(W_STD)
    q13, s13 = _encode_weight(spec, w13, (int(shared), e, 13))
    q2, s2 = _encode_weight(spec, w2, (int(shared), e, 2))
    return q13, s13, q2, s2


def draw_router(spec: Spec, seed: int):
    wr = _rng(seed, _FAMILY[spec.family], _WR, 0).standard_normal((spec.E, spec.d_model),
                                                                  dtype=np.float32)
    wr *= np.float32(W_STD)
    if spec.weight == "f32":
        return torch.from_numpy(wr)
    return to_bf16(wr)   # router weights are bf16 for the bf16 and e4m3 workloads


def draw_sel_bias(spec: Spec, seed: int):
    if spec.bias_range is None:
        return None
    r = spec.bias_range
    b = _rng(seed, _FAMILY[spec.family], _BIAS, spec.x_stream).uniform(-r, r, spec.E)
    return torch.from_numpy(b.astype(np.float32))


def zipf_assignment(spec: Spec, seed: int) -> np.ndarray:
    """Target expert loads: k distinct experts per token drawn by Gumbel-top-k from Zipf(s) weights.

    Rank r (1-based) has weight r^-s; ranks map to expert ids by a seeded permutation.
    Returns the per-expert target counts [E].
    """
    g = _rng(seed, _FAMILY[spec.family], _ZIPF, spec.x_stream)
    ranks = np.arange(1, spec.E + 1, dtype=np.float64)
    logw = -spec.zipf_s * np.log(ranks)
    expert_of_rank = g.permutation(spec.E)
    gumbel = g.gumbel(size=(spec.T, spec.E))
    pick = np.argsort(-(logw[None, :] + gumbel), axis=1, kind="stable")[:, : spec.top_k]
    counts = np.bincount(expert_of_rank[pick].ravel(), minlength=spec.E)
    return counts


def draw_logits(T: int, E: int, seed: int, lo=-3.0, hi=3.0, redraw=None, stream=0):
    """fp32 router logits U(lo, hi) supplied directly to the routing kernels."""
    L = _rng(seed, _FAMILY["custom"], _LOGITS, stream, T, E).uniform(lo, hi, (T, E)).astype(np.float32)
    for t, attempt in (redraw or []):
        L[t] = draw_logit_row(T, E, seed, t, attempt, lo, hi, stream)
    return L


def draw_logit_row(T: int, E: int, seed: int, t: int, attempt: int, lo=-3.0, hi=3.0, stream=0):
    """Replacement draw number ``attempt`` (>= 1) for row t of ``draw_logits``."""
    return _rng(seed, _FAMILY["custom"], _LOGITS, stream, T, E, t, attempt).uniform(
        lo, hi, E).astype(np.float32)


# ---------------------------------------------------------------------------
# whole workloads
# ---------------------------------------------------------------------------

@dataclass
class Workload:
    spec: Spec
    seed: int
    x: torch.Tensor                       # [T, d] f32 | bf16 | float8_e4m3fn
    x_scale: Optional[torch.Tensor]       # [T, d/128] fp32 (e4m3 only)
    wr: torch.Tensor                      # [E, d]
    sel_bias: Optional[torch.Tensor]      # [E] fp32
    w13: torch.Tensor                     # [E, 2I, d]
    w13_s: Optional[torch.Tensor]         # [E, 2I/128, d/128]
    w2: torch.Tensor                      # [E, d, I]
    w2_s: Optional[torch.Tensor]          # [E, d/128, I/128]
    ws13: Optional[torch.Tensor]          # [S, 2I, d]
    ws13_s: Optional[torch.Tensor]
    ws2: Optional[torch.Tensor]           # [S, d, I]
    ws2_s: Optional[torch.Tensor]
    recipe: dict = field(default_factory=dict)


def _stack_experts(spec, seed, n, shared, threads):
    I, d = spec.d_ff, spec.d_model
    if spec.weight == "e2m1":          # packed codes [rows, K/2] + E8M0 scale atoms
        w13 = torch.empty((n, 2 * I, d // 2), dtype=torch.uint8)
        w2 = torch.empty((n, d, I // 2), dtype=torch.uint8)
        s13 = torch.empty((n, 2 * I // 128, d // 128, 512), dtype=torch.uint8)
        s2 = torch.empty((n, d // 128, I // 128, 512), dtype=torch.uint8)
        scaled = True
    else:
        wdt = {"f32": torch.float32, "bf16": torch.bfloat16, "e4m3": torch.float8_e4m3fn,
               "e4m3_fs": torch.float8_e4m3fn}[spec.weight]
        w13 = torch.empty((n, 2 * I, d), dtype=wdt)
        w2 = torch.empty((n, d, I), dtype=wdt)
        scaled = is_e4m3(spec.weight)
        s13 = torch.empty((n, 2 * I // 128, d // 128), dtype=torch.float32) if scaled else None
        s2 = torch.empty((n, d // 128, I // 128), dtype=torch.float32) if scaled else None

    def one(e):
        q13, a13, q2, a2 = draw_expert(spec, seed, e, shared)
        w13[e].copy_(q13)
        w2[e].copy_(q2)
        if scaled:
            s13[e].copy_(a13)
            s2[e].copy_(a2)

    if n:
        with ThreadPoolExecutor(max(1, min(threads, n))) as ex:
            list(ex.map(one, range(n)))
    return w13, s13, w2, s2


def load_recipe(name: str) -> dict:
    path = os.path.join(RECIPE_DIR, f"{name}.json")
    with open(path) as f:
        return json.load(f)


def make_workload(spec: Spec, seed: int = 0, redraw=None, sel_bias=None, threads=None,
                  recipe=None) -> Workload:
    """Draw every input of one layer call."""
    threads = threads or os.cpu_count() or 1
    x32 = _draw_x_fp32(spec, seed, redraw)
    x, x_scale = encode_act(spec, x32)
    del x32
    wr = draw_router(spec, seed)
    if sel_bias is None:
        sel_bias = draw_sel_bias(spec, seed)
    elif not isinstance(sel_bias, torch.Tensor):
        sel_bias = torch.tensor(np.asarray(sel_bias, np.float32))
    w13, w13_s, w2, w2_s = _stack_experts(spec, seed, spec.E, False, threads)
    if spec.n_shared:
        ws13, ws13_s, ws2, ws2_s = _stack_experts(spec, seed, spec.n_shared, True, threads)
    else:
        ws13 = ws13_s = ws2 = ws2_s = None
    return Workload(spec, seed, x, x_scale, wr, sel_bias, w13, w13_s, w2, w2_s,
                    ws13, ws13_s, ws2, ws2_s, recipe or {})


def _same_weights(a: Spec, b: Spec) -> bool:
    return (a.family, a.weight, a.E, a.d_model, a.d_ff, a.n_shared) == \
        (b.family, b.weight, b.E, b.d_model, b.d_ff, b.n_shared)


def load_workload(name: str, seed: int = 0, threads=None, T: Optional[int] = None,
                  reuse: Optional[Workload] = None) -> Workload:
    """A named workload with its stored recipe applied (seed 0 recipes are committed).

    ``T`` may shrink the token count (rows 0..T-1 of the same draw).  ``reuse``: a
    workload of the same weight family and seed whose expert tensors are taken as they
    are (expert draws depend only on family, seed, index and storage type).
    """
    spec = SPECS[name]
    recipe = load_recipe(name) if seed == 0 else {}
    bias = recipe.get("sel_bias")
    if bias is None and name in BIAS_SOURCE and seed == 0:
        bias = load_recipe(BIAS_SOURCE[name]).get("sel_bias")
    if reuse is not None and reuse.seed == seed and _same_weights(reuse.spec, spec):
        x, x_scale = encode_act(spec, _draw_x_fp32(spec, seed, recipe.get("redraw")))
        if bias is None:
            sb = draw_sel_bias(spec, seed)
        else:
            sb = torch.tensor(np.asarray(bias, np.float32))
        w = Workload(spec, seed, x, x_scale, draw_router(spec, seed), sb, reuse.w13, reuse.w13_s,
                     reuse.w2, reuse.w2_s, reuse.ws13, reuse.ws13_s, reuse.ws2, reuse.ws2_s, recipe)
    else:
        w = make_workload(spec, seed, redraw=recipe.get("redraw"), sel_bias=bias, threads=threads,
                          recipe=recipe)
    if T is not None and T != spec.T:
        w.spec = replace(spec, T=T)
        w.x = w.x[:T].contiguous()
        if w.x_scale is not None:
            w.x_scale = w.x_scale[:T].contiguous()
    return w
