"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each test fixes one step of the layer stated by the ``moe_ffn`` pseudocode in
"Decoding Trillion-Parameter MoE LLMs: Sparse Architecture and Agentic
Intelligence", section "Routing: Top-K Experts Plus a Shared Expert":
closed forms derived by hand, brute force over all expert subsets, special
cases that reduce to library routines (scipy softmax/expit, torch silu,
torch's float8 decoder), and invariants of the permutation.
"""
import itertools
import math

import numpy as np
import pytest
import scipy.special
import torch
import torch.nn.functional as F

import oracle
from sparse_expert_moe_b200 import inputs

LN3 = math.log(3.0)


# ---------------------------------------------------------------------------
# hand-derived closed forms
# ---------------------------------------------------------------------------

def _hand_layer():
    """d=2, E=3, I=1, one shared expert; every number below is derived by hand.

    x = (1, 0).  Expert weights: W1 row (gate), W3 row (up), W2 column.
      expert 0: g = ln3 -> silu = ln3 * 3/4; u = 1;  W2 = (1, 0)^T -> y0 = (3/4 ln3, 0)
      expert 1: g = -ln3 -> silu = -ln3 * 1/4; u = 2; W2 = (0, 1)^T -> y1 = (0, -1/2 ln3)
      expert 2: g = 0 -> silu = 0                                   -> y2 = (0, 0)
      shared:   g = ln3, u = -1, W2 = (1, 1)^T                       -> ys = (-3/4 ln3, -3/4 ln3)
    """
    x = np.array([[1.0, 0.0]])
    w13 = {0: np.array([[LN3, 0.0], [1.0, 0.0]]),
           1: np.array([[-LN3, 0.0], [2.0, 0.0]]),
           2: np.array([[0.0, 0.0], [5.0, 0.0]])}
    w2 = {0: np.array([[1.0], [0.0]]), 1: np.array([[0.0], [1.0]]), 2: np.array([[3.0], [3.0]])}
    shared = (np.array([[LN3, 0.0], [-1.0, 0.0]]), np.array([[1.0], [1.0]]))
    return x, w13, w2, shared


def test_hand_softmax_layer():
    # router rows give logits (ln2, 0, -1): top-2 = experts 0, 1 with softmax gates 2/3, 1/3
    x, w13, w2, shared = _hand_layer()
    wr = np.array([[math.log(2.0), 0.0], [0.0, 0.0], [-1.0, 0.0]])
    y, r = oracle.layer_forward(x, wr, oracle.SOFTMAX, 2, lambda e: (w13[e], w2[e]), 3,
                                [shared], return_routing=True)
    assert r["idx"].tolist() == [[0, 1]]
    np.testing.assert_allclose(r["gates"], [[2 / 3, 1 / 3]], rtol=1e-14)
    # y = 2/3 y0 + 1/3 y1 + ys = (1/2 ln3 - 3/4 ln3, -1/6 ln3 - 3/4 ln3)
    np.testing.assert_allclose(y, [[-0.25 * LN3, -(11.0 / 12.0) * LN3]], rtol=1e-13)


def test_hand_sigmoid_bias_layer():
    # logits (0, ln3, -ln3): sigmoid scores (1/2, 3/4, 1/4).  Bias (0, 0, 0.6) gives keys
    # (0.5, 0.75, 0.85): the bias moves expert 2 to the front, but the gates come from the
    # unbiased scores: 1/4 / (1/4 + 3/4) = 1/4 and 3/4.
    x, w13, w2, shared = _hand_layer()
    wr = np.array([[0.0, 0.0], [LN3, 0.0], [-LN3, 0.0]])
    bias = np.array([0.0, 0.0, 0.6])
    y, r = oracle.layer_forward(x, wr, oracle.SIGMOID_BIAS, 2, lambda e: (w13[e], w2[e]), 3,
                                [shared], sel_bias=bias, return_routing=True)
    assert r["idx"].tolist() == [[2, 1]]
    np.testing.assert_allclose(r["gates"], [[0.25, 0.75]], rtol=1e-14)
    # y = 1/4 * y2 + 3/4 * y1 + ys = (-3/4 ln3, -3/8 ln3 - 3/4 ln3)
    np.testing.assert_allclose(y, [[-0.75 * LN3, -(9.0 / 8.0) * LN3]], rtol=1e-13)
    # without the bias, selection follows the scores: experts 1 then 0, gates 3/5, 2/5
    _, r0 = oracle.layer_forward(x, wr, oracle.SIGMOID_BIAS, 2, lambda e: (w13[e], w2[e]), 3,
                                 [shared], return_routing=True)
    assert r0["idx"].tolist() == [[1, 0]]
    np.testing.assert_allclose(r0["gates"], [[0.6, 0.4]], rtol=1e-14)


def test_silu_closed_forms():
    np.testing.assert_allclose(oracle.silu([LN3, -LN3, 0.0]), [0.75 * LN3, -0.25 * LN3, 0.0],
                               rtol=1e-15, atol=0)
    # large arguments: silu(z) -> z for z >> 0 and -> 0 for z << 0, without NaN
    big = oracle.silu([800.0, -800.0])
    assert big[0] == 800.0 and big[1] == 0.0


# ---------------------------------------------------------------------------
# library special cases
# ---------------------------------------------------------------------------

def test_e4m3_decode_matches_torch_for_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.decode_e4m3(codes)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(lib)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], lib[~nan])
    assert ours[0x7E] == 448.0 and ours[0x38] == 1.0
    assert ours[0x08] == 2.0 ** -6 and ours[0x01] == 2.0 ** -9 and ours[0x80] == 0.0


def test_block_dequant_round_trip():
    rng = np.random.default_rng(3)
    # rows with very different magnitudes so that a mis-indexed scale shows
    a = (rng.standard_normal((256, 384)) * np.exp2(rng.integers(-8, 8, (256, 1)))).astype(np.float32)
    for br, bc in ((1, 128), (128, 128)):
        q, s = inputs.to_e4m3_blocks(a, br, bc)
        back = oracle.dequantize_blocks(q.view(torch.uint8).numpy(), s.numpy(), br, bc)
        # e4m3 keeps 3 mantissa bits: relative error <= 2^-4 for normal values; block-relative
        # error for values near the bottom of a block
        blk = np.repeat(np.repeat(s.numpy().astype(np.float64), br, 0), bc, 1)
        err = np.abs(back - a)
        assert np.all(err <= np.maximum(np.abs(a) * 2.0 ** -4, blk * 2.0 ** -9) * 1.0000001)


def test_e2m1_decode_matches_ml_dtypes_for_all_codes():
    import ml_dtypes
    codes = np.arange(16, dtype=np.uint8)
    lib = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    assert np.array_equal(oracle.decode_e2m1(codes), lib)
    assert oracle.decode_e2m1(np.uint8(0x7)) == 6.0 and oracle.decode_e2m1(np.uint8(0x1)) == 0.5
    # only the low nibble is a code
    assert np.array_equal(oracle.decode_e2m1(codes | 0xF0), lib)


def test_e8m0_decode_matches_ml_dtypes_for_all_codes():
    import ml_dtypes
    codes = np.arange(256, dtype=np.uint8)
    lib = codes.view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    ours = oracle.decode_e8m0(codes)
    assert np.array_equal(np.isnan(ours), np.isnan(lib))
    ok = ~np.isnan(lib)
    assert np.array_equal(ours[ok], lib[ok])
    assert oracle.decode_e8m0(np.uint8(127)) == 1.0


def test_fp4_packing_order():
    """Byte j of a packed row holds element 2j in its low nibble: 0x72 is (1.0, 6.0)."""
    packed = np.array([[0x72, 0x0B]], np.uint8)
    assert np.array_equal(oracle.unpack_fp4(packed), [[2, 7, 11, 0]])
    vals = oracle.dequantize_mxfp4(np.tile(packed, (1, 8)), np.array([[128]], np.uint8))
    assert np.array_equal(vals[0, :4], [2.0, 12.0, -3.0, 0.0])


def test_mxfp4_round_trip():
    rng = np.random.default_rng(4)
    # rows and 32-element blocks of very different magnitudes so a misplaced scale shows
    a = (rng.standard_normal((64, 256)) * np.exp2(rng.integers(-6, 6, (64, 8))).repeat(32, 1)
         ).astype(np.float32)
    a[3, 32:64] = 0.0
    packed, sc = inputs.to_mxfp4(a)
    back = oracle.dequantize_mxfp4(packed.numpy(), sc.numpy())
    s = np.exp2(sc.numpy().astype(np.float64) - 127.0).repeat(32, 1)
    # nearest of E2M1's values (steps of 0.5 below 2, 1 below 4, 2 below 6, relative to s):
    # at most half a step away
    assert np.all(np.abs(back - a) <= np.maximum(np.abs(a) * 2.0 ** -2, s * 2.0 ** -2) * 1.0000001)
    assert np.all(np.abs(a) <= 6.0 * s)
    assert np.all(back[3, 32:64] == 0.0)


def test_table_mxfp4_helper_equals_oracle():
    from helpers import dequant_mxfp4_fast
    rng = np.random.default_rng(6)
    packed = rng.integers(0, 256, (64, 128)).astype(np.uint8)
    packed[0, :] = np.arange(128) * 2
    packed[1, :] = np.arange(128) * 2 + 1
    sc = rng.integers(100, 150, (64, 8)).astype(np.uint8)
    assert np.array_equal(dequant_mxfp4_fast(packed, sc), oracle.dequantize_mxfp4(packed, sc))


def test_e4m3_block_quantisation_matches_torch():
    """Codes: torch's float8_e4m3fn conversion (round to nearest even) of x / 2^e; scales: the
    smallest power of two that brings the block's amax to 448 or below."""
    rng = np.random.default_rng(8)
    x = (rng.standard_normal((64, 512)) * np.exp2(rng.integers(-20, 20, (64, 4))).repeat(128, 1))
    x = inputs.to_bf16(x.astype(np.float32)).double().numpy()     # bf16 values, as the layer gets
    x[0, :128] = 0.0
    x[1, :128] = 0.0
    x[1, 5] = -448.0 * 2.0 ** 3                                   # amax exactly 448 * 2^3
    x[2, 128:256] = -1e-30                                        # rounds to negative zero
    x[2, 128] = 1.0
    codes, sc = oracle.quantize_e4m3_blocks(x)
    e = np.log2(sc)
    assert np.array_equal(e, np.round(e))
    amax = np.abs(x).reshape(64, 4, 128).max(axis=2)
    assert np.all(amax <= 448.0 * sc) and np.all((amax > 224.0 * sc) | (amax == 0))
    assert sc[0, 0] == 1.0 and np.all(codes[0, :128] == 0)
    assert sc[1, 0] == 8.0 and codes[1, 5] == 0xFE
    assert np.all(codes[2, 129:256] == 0x80)
    lib = torch.from_numpy(x / np.repeat(sc, 128, axis=1)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codes, lib)
    # and the stored-input encoder of the generator agrees on power-of-two scaled data
    q, s = inputs.to_e4m3_blocks(x.astype(np.float32), 1, 128)
    assert np.array_equal(q.view(torch.uint8).numpy(), codes) and np.array_equal(s.numpy(), sc)


def test_table_dequant_helper_equals_oracle():
    """The tests' table-driven block dequantisation (used on whole expert weight sets) gives
    oracle.dequantize_blocks's values bit for bit, every code and block shape included."""
    from helpers import dequant_fast
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 256, (256, 384)).astype(np.uint8)
    codes[0, :256] = np.arange(256)
    for br, bc in ((1, 128), (128, 128)):
        s = np.exp2(rng.integers(-10, 10, (256 // br, 384 // bc))).astype(np.float32)
        a = dequant_fast(codes, s, br, bc)
        b = oracle.dequantize_blocks(codes, s, br, bc)
        assert np.array_equal(np.isnan(a), np.isnan(b))
        assert np.array_equal(a[~np.isnan(a)], b[~np.isnan(b)])


def test_block_dequant_takes_any_scale():
    """A block scale that is not a power of two multiplies each decoded code as it is."""
    codes = np.full((2, 256), 0x38, np.uint8)           # e4m3 1.0
    codes[1, 128] = 0xC0                                # e4m3 -2.0
    s = np.array([[0.3, 1.7], [5.0, 0.1]])
    v = oracle.dequantize_blocks(codes, s, 1, 128)
    assert v[0, 0] == 0.3 and v[0, 200] == 1.7 and v[1, 5] == 5.0 and v[1, 128] == -0.2


def test_softmax_k_equals_E_is_full_softmax():
    rng = np.random.default_rng(0)
    L = rng.uniform(-3, 3, (32, 7))
    idx, g = oracle.route(L, oracle.SOFTMAX, 7)
    full = scipy.special.softmax(L, axis=1)
    np.testing.assert_allclose(g, np.take_along_axis(full, idx, axis=1), rtol=1e-13)


def test_softmax_topk_equals_renormalised_full_softmax():
    rng = np.random.default_rng(1)
    L = rng.uniform(-3, 3, (32, 9))
    idx, g = oracle.route(L, oracle.SOFTMAX, 3)
    full = np.take_along_axis(scipy.special.softmax(L, axis=1), idx, axis=1)
    np.testing.assert_allclose(g, full / full.sum(axis=1, keepdims=True), rtol=1e-13)
    # invariant to a per-token shift of all logits
    _, g2 = oracle.route(L + 5.0, oracle.SOFTMAX, 3)
    np.testing.assert_allclose(g, g2, rtol=1e-12)


def test_sigmoid_gates_match_expit():
    rng = np.random.default_rng(2)
    L = rng.uniform(-3, 3, (16, 12))
    b = rng.uniform(-0.1, 0.1, 12)
    idx, g = oracle.route(L, oracle.SIGMOID_BIAS, 4, b)
    s = scipy.special.expit(np.take_along_axis(L, idx, axis=1))
    np.testing.assert_allclose(g, s / s.sum(axis=1, keepdims=True), rtol=1e-13)
    np.testing.assert_allclose(oracle.selection_keys(L, oracle.SIGMOID_BIAS, b),
                               scipy.special.expit(L) + b, rtol=1e-14)


def test_single_expert_gate_is_one():
    L = np.random.default_rng(4).uniform(-3, 3, (10, 1))
    for score in (oracle.SOFTMAX, oracle.SIGMOID_BIAS):
        idx, g = oracle.route(L, score, 1)
        assert np.all(idx == 0) and np.all(g == 1.0)


def test_router_logits_one_hot_rows():
    rng = np.random.default_rng(5)
    wr = rng.standard_normal((6, 4))
    np.testing.assert_array_equal(oracle.router_logits(np.eye(4), wr), wr.T)


def test_swiglu_expert_matches_torch():
    rng = np.random.default_rng(6)
    X = rng.standard_normal((5, 16))
    w13 = rng.standard_normal((2 * 8, 16)) * 0.3
    w2 = rng.standard_normal((16, 8)) * 0.3
    Xt, w13t, w2t = map(torch.from_numpy, (X, w13, w2))
    ref = (F.silu(Xt @ w13t[:8].T) * (Xt @ w13t[8:].T)) @ w2t.T
    np.testing.assert_allclose(oracle.swiglu_expert(X, w13, w2), ref.numpy(), rtol=1e-12, atol=1e-14)


def test_E1_k1_is_dense_swiglu():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((9, 16))
    wr = rng.standard_normal((1, 16))
    w13 = rng.standard_normal((2 * 12, 16)) * 0.2
    w2 = rng.standard_normal((16, 12)) * 0.2
    xt = torch.from_numpy(x)
    dense = (F.silu(xt @ torch.from_numpy(w13[:12]).T) * (xt @ torch.from_numpy(w13[12:]).T)) \
        @ torch.from_numpy(w2).T
    for score in (oracle.SOFTMAX, oracle.SIGMOID_BIAS):
        y = oracle.layer_forward(x, wr, score, 1, lambda e: (w13, w2), 1)
        np.testing.assert_allclose(y, dense.numpy(), rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------------------
# brute force over expert subsets
# ---------------------------------------------------------------------------

def _brute_topk(keys_row, k):
    """Lexicographically smallest k-subset S with every key in S >= every key outside S,
    then ordered by (key descending, index ascending) with Python's tuple sort."""
    E = len(keys_row)
    for S in itertools.combinations(range(E), k):      # lexicographic order
        rest = [j for j in range(E) if j not in S]
        if all(keys_row[i] >= keys_row[j] for i in S for j in rest):
            return [i for _, i in sorted((-keys_row[i], i) for i in S)]
    raise AssertionError("no top-k subset")


@pytest.mark.parametrize("E,k", [(8, 2), (6, 3), (5, 5), (7, 1)])
def test_topk_brute_force(E, k):
    rng = np.random.default_rng(E * 10 + k)
    for trial in range(60):
        if trial % 3 == 0:
            keys = rng.integers(0, 3, E).astype(np.float64)   # many exact ties
        else:
            keys = rng.uniform(-1, 1, E)
        got = oracle.select_topk(keys[None, :], k)[0].tolist()
        assert got == _brute_topk(keys.tolist(), k), keys


def test_topk_max_sum_brute_force():
    # with distinct keys the selected subset is the unique subset of maximal key sum
    rng = np.random.default_rng(11)
    for _ in range(40):
        keys = rng.permutation(10).astype(np.float64)        # distinct integers: exact sums
        best = max(itertools.combinations(range(10), 3), key=lambda S: sum(keys[list(S)]))
        assert sorted(oracle.select_topk(keys[None], 3)[0].tolist()) == list(best)


def test_all_equal_keys_select_lowest_experts():
    for score in (oracle.SOFTMAX, oracle.SIGMOID_BIAS):
        idx, g = oracle.route(np.zeros((3, 9)), score, 4)
        assert idx.tolist() == [[0, 1, 2, 3]] * 3
        np.testing.assert_allclose(g, 0.25)


def test_layer_brute_force_dense_gate_matrix():
    """The permute -> grouped experts -> combine path equals evaluating every expert on
    every token and weighting by a dense [T, E] gate matrix (zeros off the selection)."""
    rng = np.random.default_rng(12)
    T, d, E, k, I = 13, 16, 6, 3, 8
    x = rng.standard_normal((T, d))
    wr = rng.standard_normal((E, d)) * 0.5
    w13 = [rng.standard_normal((2 * I, d)) * 0.3 for _ in range(E)]
    w2 = [rng.standard_normal((d, I)) * 0.3 for _ in range(E)]
    sh = [(rng.standard_normal((2 * I, d)) * 0.3, rng.standard_normal((d, I)) * 0.3) for _ in range(2)]
    b = rng.uniform(-0.1, 0.1, E)
    for score in (oracle.SOFTMAX, oracle.SIGMOID_BIAS):
        y = oracle.layer_forward(x, wr, score, k, lambda e: (w13[e], w2[e]), E, sh, sel_bias=b)
        L = x @ wr.T
        keys = L if score == oracle.SOFTMAX else scipy.special.expit(L) + b
        G = np.zeros((T, E))
        for t in range(T):
            S = _brute_topk(keys[t].tolist(), k)
            if score == oracle.SOFTMAX:
                w = scipy.special.softmax(L[t, S])
            else:
                s = scipy.special.expit(L[t, S])
                w = s / s.sum()
            G[t, S] = w
        ref = np.zeros((T, d))
        for e in range(E):
            xt = torch.from_numpy(x)
            ye = (F.silu(xt @ torch.from_numpy(w13[e][:I]).T) * (xt @ torch.from_numpy(w13[e][I:]).T)) \
                @ torch.from_numpy(w2[e]).T
            ref += G[:, e : e + 1] * ye.numpy()
        for a, c in sh:
            xt = torch.from_numpy(x)
            ref += ((F.silu(xt @ torch.from_numpy(a[:I]).T) * (xt @ torch.from_numpy(a[I:]).T))
                    @ torch.from_numpy(c).T).numpy()
        np.testing.assert_allclose(y, ref, rtol=1e-11, atol=1e-13)


def test_zero_routed_down_projection_leaves_shared_only_and_linearity():
    rng = np.random.default_rng(13)
    T, d, E, k, I = 11, 16, 5, 2, 8
    x = rng.standard_normal((T, d))
    wr = rng.standard_normal((E, d))
    w13 = [rng.standard_normal((2 * I, d)) * 0.3 for _ in range(E)]
    w2 = [rng.standard_normal((d, I)) * 0.3 for _ in range(E)]
    sh = (rng.standard_normal((2 * I, d)) * 0.3, rng.standard_normal((d, I)) * 0.3)
    shared_only = oracle.swiglu_expert(x, *sh)
    y0 = oracle.layer_forward(x, wr, oracle.SOFTMAX, k, lambda e: (w13[e], 0 * w2[e]), E, [sh])
    np.testing.assert_allclose(y0, shared_only, rtol=1e-13)
    y1 = oracle.layer_forward(x, wr, oracle.SOFTMAX, k, lambda e: (w13[e], w2[e]), E, [sh])
    y2 = oracle.layer_forward(x, wr, oracle.SOFTMAX, k, lambda e: (w13[e], 2 * w2[e]), E, [sh])
    np.testing.assert_allclose(y2 - shared_only, 2 * (y1 - shared_only), rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------------------
# permutation invariants
# ---------------------------------------------------------------------------

def _check_permutation(idx, E, offsets, perm_token, inv_perm):
    T, k = idx.shape
    assert offsets[0] == 0 and offsets[-1] == T * k
    assert np.all(np.diff(offsets) >= 0)
    assert np.array_equal(np.diff(offsets), np.bincount(idx.ravel(), minlength=E))
    assert sorted(inv_perm.ravel().tolist()) == list(range(T * k))       # bijection
    for t in range(T):
        for j in range(k):
            r = inv_perm[t, j]
            assert perm_token[r] == t
            e = np.searchsorted(offsets, r, side="right") - 1
            assert e == idx[t, j]
    for e in range(E):
        grp = perm_token[offsets[e]:offsets[e + 1]]
        assert np.all(np.diff(grp) > 0)                                   # ascending tokens
    assert np.array_equal(np.bincount(perm_token, minlength=T), np.full(T, k))  # k groups each


@pytest.mark.parametrize("T,E,k", [(1, 8, 2), (63, 8, 2), (64, 256, 8), (200, 384, 8), (37, 5, 5)])
def test_permutation_invariants(T, E, k):
    rng = np.random.default_rng(T + E + k)
    L = rng.uniform(-3, 3, (T, E))
    idx, _ = oracle.route(L, oracle.SIGMOID_BIAS, k, rng.uniform(-0.1, 0.1, E))
    _check_permutation(idx, E, *oracle.permute(idx, E))


def test_forced_empty_experts():
    # bias -2 puts sigmoid + bias below -1 < every other key: those experts never get rows
    rng = np.random.default_rng(14)
    T, E, k = 50, 32, 8
    L = rng.uniform(-3, 3, (T, E))
    b = rng.uniform(-0.1, 0.1, E)
    empty = rng.choice(E, 16, replace=False)
    b[empty] = -2.0
    idx, _ = oracle.route(L, oracle.SIGMOID_BIAS, k, b)
    offsets, perm_token, inv_perm = oracle.permute(idx, E)
    assert np.all(np.diff(offsets)[empty] == 0)
    _check_permutation(idx, E, offsets, perm_token, inv_perm)


def test_combine_slot_order_and_gathers():
    # one token, rows in a known permuted position: combine must read inv_perm, not slot index
    y_perm = np.array([[1.0, 0.0], [0.0, 10.0], [100.0, 0.0]])
    inv = np.array([[2, 0]])
    g = np.array([[0.25, 0.75]])
    out = oracle.combine(y_perm, inv, g, [np.array([[0.5, 0.5]])])
    np.testing.assert_array_equal(out, [[25.0 + 0.75 + 0.5, 0.5]])
