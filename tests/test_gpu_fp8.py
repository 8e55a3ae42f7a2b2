"""The FP8 block-scaled path (e4m3 activations with 1x128 scales, e4m3 weights with
128x128 scales, h requantised to e4m3 in the first GEMM's epilogue) against the fp64
oracle on the decoded input values.  Bar: max relative error 6e-2."""
import numpy as np
import pytest
import torch

import oracle
from sparse_expert_moe_b200 import inputs, moe

from helpers import (dequant_fast, dequant_mxfp4_fast, margin_workload, max_rel_err, oracle_layer,
                     oracle_routing, tile_edge_tokens)

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL_FP8 = 6e-2


def _e4m3(a, br, bc):
    return inputs.to_e4m3_blocks(np.asarray(a, np.float32), br, bc)


def _dq(q, s, br, bc):
    return oracle.dequantize_blocks(q.view(torch.uint8).numpy(), s.numpy(), br, bc)


@pytest.mark.parametrize("sizes,d,I", [
    ([5, 0, 1, 130, 16, 17, 0, 112], 256, 256),
    ([300], 128, 384),
    ([1, 2, 3], 512, 128),
])
def test_grouped_ffn_fp8_vs_oracle(sizes, d, I):
    rng = np.random.default_rng(sum(sizes) + d)
    G, n_rows = len(sizes), sum(sizes)
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    a, a_s = _e4m3(rng.standard_normal((n_rows, d)) * np.exp2(rng.integers(-3, 3, (n_rows, 1))), 1, 128)
    w13 = [_e4m3(rng.standard_normal((2 * I, d)) * 0.05 * 2.0 ** rng.integers(-2, 3), 128, 128)
           for _ in range(G)]
    w2 = [_e4m3(rng.standard_normal((d, I)) * 0.05 * 2.0 ** rng.integers(-2, 3), 128, 128)
          for _ in range(G)]
    W13 = torch.stack([q for q, _ in w13]).to(DEV)
    S13 = torch.stack([s for _, s in w13]).to(DEV)
    W2 = torch.stack([q for q, _ in w2]).to(DEV)
    S2 = torch.stack([s for _, s in w2]).to(DEV)
    cfg = moe.make_config(n_rows, d, G, 1, I, 0, act="e4m3", weight="e4m3")
    ws = torch.zeros(moe.moe_workspace_size(cfg), dtype=torch.uint8, device=DEV)
    y = torch.full((n_rows, d), float("nan"), dtype=torch.bfloat16, device=DEV)
    moe.moe_grouped_ffn(cfg, G, torch.from_numpy(offsets).to(DEV), n_rows, a.to(DEV), a_s.to(DEV),
                        W13, S13, W2, S2, y, ws)
    assert moe.moe_read_device_status(ws) == 0
    av = _dq(a, a_s, 1, 128)
    ref = np.zeros((n_rows, d))
    for g in range(G):
        lo, hi = offsets[g], offsets[g + 1]
        if hi > lo:
            ref[lo:hi] = oracle.swiglu_expert(av[lo:hi], _dq(*w13[g], 128, 128), _dq(*w2[g], 128, 128))
    got = y.float().cpu().numpy()
    assert np.isfinite(got).all()
    assert max_rel_err(got, ref) < TOL_FP8


@pytest.mark.slow
def test_grouped_ffn_fp8_r1_shape_every_row():
    """FP8 at the DeepSeek-R1 expert shape (d = 7168, I = 2048: 56 K blocks of 128 in the
    first GEMM, 16 in the second): a 7300-row group (33 chunks of 224 rows; the first GEMM
    takes them as 112-row halves, the last chunk's second half holding 20 rows), one of 257
    rows (224 + 33), one of 1 row and an empty one.  Every output row is compared with the
    oracle on the decoded inputs."""
    sizes, d, I = [7300, 257, 1, 0], 7168, 2048
    rng = np.random.default_rng(72)
    G, n_rows = len(sizes), sum(sizes)
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    a, a_s = _e4m3(rng.standard_normal((n_rows, d), dtype=np.float32), 1, 128)
    w13 = [_e4m3(rng.standard_normal((2 * I, d), dtype=np.float32) * np.float32(0.02), 128, 128)
           for _ in range(G)]
    w2 = [_e4m3(rng.standard_normal((d, I), dtype=np.float32) * np.float32(0.02), 128, 128)
          for _ in range(G)]
    cfg = moe.make_config(n_rows, d, G, 1, I, 0, act="e4m3", weight="e4m3")
    ws = torch.zeros(moe.moe_workspace_size(cfg), dtype=torch.uint8, device=DEV)
    y = torch.full((n_rows, d), float("nan"), dtype=torch.bfloat16, device=DEV)
    moe.moe_grouped_ffn(cfg, G, torch.from_numpy(offsets).to(DEV), n_rows,
                        a.view(torch.uint8).to(DEV), a_s.to(DEV),
                        torch.stack([q for q, _ in w13]).to(DEV), torch.stack([s for _, s in w13]).to(DEV),
                        torch.stack([q for q, _ in w2]).to(DEV), torch.stack([s for _, s in w2]).to(DEV),
                        y, ws)
    assert moe.moe_read_device_status(ws) == 0
    got = y.float().cpu().numpy()
    assert np.isfinite(got).all()
    av = dequant_fast(a.view(torch.uint8).numpy(), a_s.numpy(), 1, 128)
    for g in range(G):
        lo, hi = offsets[g], offsets[g + 1]
        if hi == lo:
            continue
        ref = oracle.swiglu_expert(av[lo:hi], dequant_fast(w13[g][0].view(torch.uint8).numpy(),
                                                           w13[g][1].numpy(), 128, 128),
                                   dequant_fast(w2[g][0].view(torch.uint8).numpy(),
                                                w2[g][1].numpy(), 128, 128))
        assert max_rel_err(got[lo:hi], ref) < TOL_FP8, g
        # per row: h is requantised to e4m3 (3 mantissa bits), so single rows scatter more
        # than the whole output; twice the bar still exposes a wrong tile or chunk
        row = np.abs(got[lo:hi] - ref).max(axis=1) / np.abs(ref).max(axis=1)
        assert row.max() < 2 * TOL_FP8, g


def _mxfp4(rows, cols, rng, std=0.05):
    """MXFP4 weights whose 32-element runs differ in magnitude by up to 2^6, so that every
    run needs its own E8M0 scale (a scale applied to the wrong run shows in the output)."""
    w = rng.standard_normal((rows, cols)) * std * np.exp2(rng.integers(-3, 4, (rows, cols // 32))).repeat(32, 1)
    return inputs.to_mxfp4(w.astype(np.float32))


@pytest.mark.parametrize("sizes,d,I", [
    ([5, 0, 1, 130, 16, 17, 0, 112], 256, 256),     # 112 / 224-row tiles, ragged, empty
    ([300], 128, 384),
    ([1, 2, 3], 512, 128),                           # decode-sized: 32-token tiles
    ([3, 0, 17, 32, 33], 1024, 256),
])
def test_grouped_ffn_fp4_weights_vs_oracle(sizes, d, I):
    """FP4 (MXFP4) expert weights with e4m3 token rows; h requantised to e4m3."""
    rng = np.random.default_rng(sum(sizes) + d + 1)
    G, n_rows = len(sizes), sum(sizes)
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    a, a_s = _e4m3(rng.standard_normal((n_rows, d)) * np.exp2(rng.integers(-3, 3, (n_rows, 1))), 1, 128)
    w13 = [_mxfp4(2 * I, d, rng) for _ in range(G)]
    w2 = [_mxfp4(d, I, rng) for _ in range(G)]
    atoms = lambda ws: torch.stack([inputs.scale_atoms(s.numpy()) for _, s in ws]).to(DEV)
    cfg = moe.make_config(n_rows, d, G, 1, I, 0, act="e4m3", weight="e2m1")
    ws = torch.zeros(moe.moe_workspace_size(cfg), dtype=torch.uint8, device=DEV)
    y = torch.full((n_rows, d), float("nan"), dtype=torch.bfloat16, device=DEV)
    moe.moe_grouped_ffn(cfg, G, torch.from_numpy(offsets).to(DEV), n_rows, a.view(torch.uint8).to(DEV),
                        a_s.to(DEV), torch.stack([q for q, _ in w13]).to(DEV), atoms(w13),
                        torch.stack([q for q, _ in w2]).to(DEV), atoms(w2), y, ws)
    assert moe.moe_read_device_status(ws) == 0
    av = _dq(a, a_s, 1, 128)
    ref = np.zeros((n_rows, d))
    for g in range(G):
        lo, hi = offsets[g], offsets[g + 1]
        if hi > lo:
            ref[lo:hi] = oracle.swiglu_expert(av[lo:hi], oracle.dequantize_mxfp4(*[t.numpy() for t in w13[g]]),
                                              oracle.dequantize_mxfp4(*[t.numpy() for t in w2[g]]))
    got = y.float().cpu().numpy()
    assert np.isfinite(got).all()
    assert max_rel_err(got, ref) < TOL_FP8


@pytest.mark.parametrize("T,E,k,d", [(300, 32, 4, 256), (64, 8, 2, 128), (1000, 256, 8, 7168)])
@pytest.mark.parametrize("weight", ["e4m3", "e2m1"])
def test_permute_quantises_bf16_rows_for_low_precision_experts(T, E, k, d, weight):
    """bf16 activations with e4m3 / FP4 expert weights: moe_permute quantises the rows to e4m3
    in the copy -- codes and power-of-two scales equal to the oracle's quantisation, bit for
    bit, placed by the oracle's permutation."""
    rng = np.random.default_rng(T + d)
    idx, _ = oracle.route(rng.uniform(-3, 3, (T, E)), "softmax", k)
    x32 = rng.standard_normal((T, d)) * np.exp2(rng.integers(-12, 12, (T, d // 128))).repeat(128, 1)
    x32[0, :128] = 0.0                                   # an all-zero block
    x = inputs.to_bf16(x32.astype(np.float32))
    cfg = moe.make_config(T, d, E, k, 128, 0, act="bf16", weight=weight)
    ws = torch.zeros(moe.moe_workspace_size(cfg), dtype=torch.uint8, device=DEV)
    R = T * k
    x_perm = torch.zeros((R, d), dtype=torch.uint8, device=DEV)
    x_perm_s = torch.zeros((R, d // 128), dtype=torch.float32, device=DEV)
    perm_token = torch.empty(R, dtype=torch.int32, device=DEV)
    inv_perm = torch.empty((T, k), dtype=torch.int32, device=DEV)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    moe.moe_permute(cfg, torch.from_numpy(idx.astype(np.int32)).to(DEV), x.to(DEV), None, x_perm,
                    x_perm_s, perm_token, inv_perm, offsets, ws)
    assert moe.moe_read_device_status(ws) == 0
    ro, rp, ri = oracle.permute(idx, E)
    codes, sc = oracle.quantize_e4m3_blocks(x.double().numpy())
    assert np.array_equal(offsets.cpu().numpy(), ro)
    assert np.array_equal(perm_token.cpu().numpy(), rp)
    assert np.array_equal(inv_perm.cpu().numpy(), ri)
    assert np.array_equal(x_perm.cpu().numpy(), codes[rp])
    assert np.array_equal(x_perm_s.cpu().numpy().astype(np.float64), sc[rp])


def test_quantising_permute_drops_out_of_range_pairs():
    """Pairs with an expert index outside [0, E) are dropped by the quantising permutation as
    by the plain one (inv_perm -1, not counted) and reported in the device status."""
    T, E, k, d = 40, 8, 2, 256
    idx = np.tile(np.array([0, 1]), (T, 1))
    idx[5, 1] = 8
    idx[9, 0] = -1
    x = inputs.to_bf16(np.random.default_rng(3).standard_normal((T, d)).astype(np.float32))
    cfg = moe.make_config(T, d, E, k, 128, 0, act="bf16", weight="e4m3")
    ws = torch.zeros(moe.moe_workspace_size(cfg), dtype=torch.uint8, device=DEV)
    R = T * k
    x_perm = torch.zeros((R, d), dtype=torch.uint8, device=DEV)
    x_perm_s = torch.zeros((R, d // 128), dtype=torch.float32, device=DEV)
    perm_token = torch.empty(R, dtype=torch.int32, device=DEV)
    inv_perm = torch.empty((T, k), dtype=torch.int32, device=DEV)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    moe.moe_permute(cfg, torch.from_numpy(idx.astype(np.int32)).to(DEV), x.to(DEV), None, x_perm,
                    x_perm_s, perm_token, inv_perm, offsets, ws)
    assert moe.moe_read_device_status(ws) == 5
    ip = inv_perm.cpu().numpy()
    assert ip[5, 1] == -1 and ip[9, 0] == -1 and offsets.cpu().numpy()[-1] == R - 2
    codes, sc = oracle.quantize_e4m3_blocks(x.double().numpy())
    pt = perm_token.cpu().numpy()[: R - 2]
    assert np.array_equal(x_perm.cpu().numpy()[: R - 2], codes[pt])
    assert np.array_equal(x_perm_s.cpu().numpy()[: R - 2].astype(np.float64), sc[pt])


def _e4m3_any_scale(a, br, bc, rng):
    """e4m3 codes with block scales that are not powers of two: the power-of-two scales of
    the encoding times factors in [1, 2) (the stored values are codes x these scales)."""
    q, s = inputs.to_e4m3_blocks(np.asarray(a, np.float32), br, bc)
    return q, torch.from_numpy(s.numpy() * rng.uniform(1.0, 2.0, s.shape).astype(np.float32))


@pytest.mark.parametrize("sizes,d,I", [
    ([5, 0, 1, 130, 16, 17, 0, 112], 256, 256),
    ([300], 128, 384),
    ([1, 2, 3], 512, 128),
    ([33, 0, 64, 7], 1024, 256),
])
def test_grouped_ffn_fp32_block_scales_vs_oracle(sizes, d, I):
    """e4m3 rows and weights whose block scales are arbitrary fp32 values (MOE_E4M3_FP32_SCALE):
    every 128-K block rescaled in fp32; h requantised to e4m3 as on the power-of-two path."""
    rng = np.random.default_rng(sum(sizes) + d + 7)
    G, n_rows = len(sizes), sum(sizes)
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    a, a_s = _e4m3_any_scale(rng.standard_normal((n_rows, d)) * np.exp2(rng.integers(-3, 3, (n_rows, 1))),
                             1, 128, rng)
    w13 = [_e4m3_any_scale(rng.standard_normal((2 * I, d)) * 0.05 * 2.0 ** rng.integers(-2, 3), 128, 128, rng)
           for _ in range(G)]
    w2 = [_e4m3_any_scale(rng.standard_normal((d, I)) * 0.05 * 2.0 ** rng.integers(-2, 3), 128, 128, rng)
          for _ in range(G)]
    assert not np.all(np.log2(a_s.numpy()) == np.round(np.log2(a_s.numpy())))
    cfg = moe.make_config(n_rows, d, G, 1, I, 0, act="e4m3_fs", weight="e4m3_fs")
    ws = torch.zeros(moe.moe_workspace_size(cfg), dtype=torch.uint8, device=DEV)
    y = torch.full((n_rows, d), float("nan"), dtype=torch.bfloat16, device=DEV)
    moe.moe_grouped_ffn(cfg, G, torch.from_numpy(offsets).to(DEV), n_rows, a.view(torch.uint8).to(DEV),
                        a_s.to(DEV), torch.stack([q for q, _ in w13]).view(torch.uint8).to(DEV),
                        torch.stack([s for _, s in w13]).to(DEV),
                        torch.stack([q for q, _ in w2]).view(torch.uint8).to(DEV),
                        torch.stack([s for _, s in w2]).to(DEV), y, ws)
    assert moe.moe_read_device_status(ws) == 0
    av = _dq(a, a_s, 1, 128)
    ref = np.zeros((n_rows, d))
    for g in range(G):
        lo, hi = offsets[g], offsets[g + 1]
        if hi > lo:
            ref[lo:hi] = oracle.swiglu_expert(av[lo:hi], _dq(*w13[g], 128, 128), _dq(*w2[g], 128, 128))
    got = y.float().cpu().numpy()
    assert np.isfinite(got).all()
    assert max_rel_err(got, ref) < TOL_FP8


@pytest.mark.parametrize("T,d,E,k,I,S", [(70, 256, 16, 4, 256, 1), (300, 384, 8, 2, 128, 2),
                                         (1, 128, 4, 1, 128, 1)])
def test_layer_fp32_block_scales(T, d, E, k, I, S):
    spec = inputs.custom_spec(T, d, E, k, I, S, act="e4m3_fs", weight="e4m3_fs")
    wl = margin_workload(spec, seed=T + 11)
    assert not np.all(np.log2(wl.w13_s.numpy()) == np.round(np.log2(wl.w13_s.numpy())))
    _check_fp8_layer(wl)


def test_permute_fp8_rows_and_scales():
    T, E, k, d = 300, 32, 4, 256
    rng = np.random.default_rng(9)
    idx, _ = oracle.route(rng.uniform(-3, 3, (T, E)), "softmax", k)
    x, xs = _e4m3(rng.standard_normal((T, d)), 1, 128)
    cfg = moe.make_config(T, d, E, k, 128, 0, act="e4m3", weight="e4m3")
    ws = torch.zeros(moe.moe_workspace_size(cfg), dtype=torch.uint8, device=DEV)
    R = T * k
    x_perm = torch.zeros((R, d), dtype=torch.uint8, device=DEV)
    x_perm_s = torch.zeros((R, d // 128), dtype=torch.float32, device=DEV)
    perm_token = torch.empty(R, dtype=torch.int32, device=DEV)
    inv_perm = torch.empty((T, k), dtype=torch.int32, device=DEV)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    moe.moe_permute(cfg, torch.from_numpy(idx.astype(np.int32)).to(DEV), x.view(torch.uint8).to(DEV),
                    xs.to(DEV), x_perm, x_perm_s, perm_token, inv_perm, offsets, ws)
    ro, rp, ri = oracle.permute(idx, E)
    assert np.array_equal(offsets.cpu().numpy(), ro)
    assert np.array_equal(perm_token.cpu().numpy(), rp)
    assert np.array_equal(inv_perm.cpu().numpy(), ri)
    tp = torch.from_numpy(rp)
    assert torch.equal(x_perm.cpu(), x.view(torch.uint8)[tp])
    assert torch.equal(x_perm_s.cpu(), xs[tp])


def _check_fp8_layer(wl, rows=None, routing=None):
    layer = moe.DeviceLayer.from_workload(wl, DEV)
    idx = torch.empty((layer.cfg.T, layer.cfg.top_k), dtype=torch.int32, device=DEV)
    gw = torch.empty((layer.cfg.T, layer.cfg.top_k), dtype=torch.float32, device=DEV)
    xs = None if wl.x_scale is None else wl.x_scale.to(DEV)
    y = layer.forward(wl.x.to(DEV), xs, topk_idx=idx, topk_w=gw)
    torch.cuda.synchronize()
    assert moe.moe_read_device_status(layer.ws) == 0
    got, idx, gw = y.float().cpu().numpy(), idx.cpu().numpy(), gw.cpu().numpy()
    del layer
    if routing is not None:
        assert np.array_equal(idx, routing["idx"])
        np.testing.assert_allclose(gw, routing["gates"], rtol=1e-5, atol=1e-6)
    ref, r = oracle_layer(wl, rows=rows, return_routing=True)
    if rows is not None:
        got, idx, gw = got[rows], idx[rows], gw[rows]
    assert np.array_equal(idx, r["idx"])
    np.testing.assert_allclose(gw, r["gates"], rtol=1e-5, atol=1e-6)
    err = max_rel_err(got, ref)
    assert err < TOL_FP8, err


@pytest.mark.parametrize("T,d,E,k,I,S", [(70, 256, 16, 4, 256, 1), (300, 384, 8, 2, 128, 2),
                                         (1, 128, 4, 1, 128, 1),
                                         (129, 512, 8, 4, 256, 1)])   # smallest wide-tile batch
@pytest.mark.parametrize("weight", ["e4m3", "e2m1"])
def test_layer_fp8_custom(T, d, E, k, I, S, weight):
    spec = inputs.custom_spec(T, d, E, k, I, S, act="e4m3", weight=weight)
    _check_fp8_layer(margin_workload(spec, seed=T + 1))


@pytest.mark.parametrize("T,d,E,k,I,S", [(70, 256, 16, 4, 256, 1), (300, 384, 8, 2, 128, 2),
                                         (1, 128, 4, 1, 128, 1)])
@pytest.mark.parametrize("weight", ["e4m3", "e2m1"])
def test_layer_bf16_activations_low_precision_experts(T, d, E, k, I, S, weight):
    """bf16 activations, e4m3 / FP4 experts: the router takes x as given, the experts take x
    quantised to e4m3 in the permutation (the oracle applies its own quantisation)."""
    spec = inputs.custom_spec(T, d, E, k, I, S, act="bf16", weight=weight)
    wl = margin_workload(spec, seed=T + 3)
    layer = moe.DeviceLayer.from_workload(wl, DEV)
    idx = torch.empty((T, k), dtype=torch.int32, device=DEV)
    gw = torch.empty((T, k), dtype=torch.float32, device=DEV)
    y = layer.forward(wl.x.to(DEV), None, topk_idx=idx, topk_w=gw)
    torch.cuda.synchronize()
    assert moe.moe_read_device_status(layer.ws) == 0
    ref, r = oracle_layer(wl, return_routing=True)
    assert np.array_equal(idx.cpu().numpy(), r["idx"])
    np.testing.assert_allclose(gw.cpu().numpy(), r["gates"], rtol=1e-5, atol=1e-6)
    assert max_rel_err(y.float().cpu().numpy(), ref) < TOL_FP8


@pytest.mark.slow
@pytest.mark.parametrize("name", ["r1_decode_fp8", "r1_decode_fp4", "r1_decode_fp4q",
                                  "r1_decode_fp8s"])
def test_layer_r1_decode_low_precision_full(name):
    """The DeepSeek-R1 decode layer with e4m3 activations and e4m3 or MXFP4 weights, every
    token checked."""
    wl = inputs.load_workload(name)
    _check_fp8_layer(wl, routing=oracle_routing(wl))


@pytest.mark.parametrize("which,value", [("w13_s", 0.75), ("w2_s", 0.0), ("ws2_s", -0.5),
                                         ("x_scale", 3.0), ("x_scale", float("inf"))])
def test_layer_fp8_scale_outside_ue8m0_sets_device_status(which, value):
    """A block scale the tensor cores' UE8M0 factors cannot hold exactly (not a positive
    normal power of two) is reported through the device status, not silently rounded."""
    spec = inputs.custom_spec(40, 256, 8, 2, 256, 1, act="e4m3", weight="e4m3")
    wl = margin_workload(spec, seed=5)
    layer = moe.DeviceLayer.from_workload(wl, DEV)
    x, xs = wl.x.to(DEV), wl.x_scale.to(DEV).clone()
    moe.moe_reset_device_status(layer.ws)
    layer.forward(x, xs)
    torch.cuda.synchronize()
    assert moe.moe_read_device_status(layer.ws) == 0
    if which == "x_scale":
        xs[3, 1] = value
        weights = layer.weights
    else:
        t = {k: v for k, v in layer.tensors.items()}
        t[which] = t[which].clone()
        t[which].view(-1)[-1] = value
        weights = moe.make_weights(t["wr"], t["sel_bias"], t["w13"], t["w2"], t["ws13"], t["ws2"],
                                   t["w13_s"], t["w2_s"], t["ws13_s"], t["ws2_s"])
    y = layer.output(DEV)
    moe.moe_layer_forward(layer.cfg, weights, x, xs, y, None, None, layer.ws)
    assert moe.moe_read_device_status(layer.ws) == 7
    moe.moe_reset_device_status(layer.ws)
    layer.forward(x, wl.x_scale.to(DEV))
    assert moe.moe_read_device_status(layer.ws) == 0


@pytest.mark.slow
def test_layer_fp8_full_size_sampled():
    """The full-size FP8 prefill layer: routing of every token; outputs of the tokens holding
    the first and the last row of every 112-row token tile of every expert group."""
    wl = inputs.load_workload("r1_prefill_fp8")
    routing = oracle_routing(wl)
    rows = tile_edge_tokens(routing, wl.spec.T, wl.spec.n_shared, 112)
    assert rows.size >= 256
    _check_fp8_layer(wl, rows=rows, routing=routing)
