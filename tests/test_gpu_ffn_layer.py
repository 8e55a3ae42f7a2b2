"""moe_grouped_ffn, moe_combine and moe_layer_forward on the GPU against the oracle.

Metric: max relative error ||y - ref||_inf / ||ref||_inf, bar 2e-2 for bf16 (the
layer's stated tolerance); the oracle is fp64 on the exact input values."""
import numpy as np
import pytest
import torch

import oracle
from sparse_expert_moe_b200 import inputs, moe

from helpers import margin_workload, max_rel_err, oracle_layer, oracle_routing, tile_edge_tokens

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL_BF16 = 2e-2


def _bf16(a):
    return inputs.to_bf16(np.asarray(a, np.float32))


# ---------------------------------------------------------------------------
# grouped FFN alone
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("sizes,d,I", [
    ([5, 0, 1, 130, 16, 17, 0, 128], 256, 256),     # ragged: empty, 1 row, > one 128-row chunk
    ([300], 128, 384),                               # one group, three chunks, ragged tail
    ([1, 1, 1, 1], 512, 128),
    ([3, 0, 17, 32, 33], 1024, 256),                # decode-sized: 32-row chunks, 512-row weight tiles
    # heavy groups over many 256-row chunks with ragged last chunks, then light groups
    ([4000, 3000, 2600, 300, 5, 0, 70], 256, 2048),
])
def test_grouped_ffn_vs_oracle(sizes, d, I):
    rng = np.random.default_rng(sum(sizes) + d + I)
    G = len(sizes)
    n_rows = sum(sizes)
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    a = _bf16(rng.standard_normal((n_rows, d)))
    w13 = _bf16(rng.standard_normal((G, 2 * I, d)) * 0.05)
    w2 = _bf16(rng.standard_normal((G, d, I)) * 0.05)
    cfg = moe.make_config(n_rows, d, G, 1, I, 0)
    ws = torch.zeros(moe.moe_workspace_size(cfg), dtype=torch.uint8, device=DEV)
    y = torch.full((n_rows, d), float("nan"), dtype=torch.bfloat16, device=DEV)
    moe.moe_grouped_ffn(cfg, G, torch.from_numpy(offsets).to(DEV), n_rows, a.to(DEV), None,
                        w13.to(DEV), None, w2.to(DEV), None, y, ws)
    assert moe.moe_read_device_status(ws) == 0
    ref = np.zeros((n_rows, d))
    for g in range(G):
        lo, hi = offsets[g], offsets[g + 1]
        if hi > lo:
            ref[lo:hi] = oracle.swiglu_expert(a[lo:hi].double().numpy(), w13[g].double().numpy(),
                                              w2[g].double().numpy())
    got = y.float().cpu().numpy()
    assert np.isfinite(got).all()
    assert max_rel_err(got, ref) < TOL_BF16


def row_rel_err(y, ref):
    """Per row: ||y_r - ref_r||_inf / ||ref_r||_inf."""
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    return np.abs(y - ref).max(axis=1) / np.maximum(np.abs(ref).max(axis=1), 1e-30)


@pytest.mark.slow
def test_grouped_ffn_r1_shape_every_row():
    """The DeepSeek-R1 expert shape (d = 7168, I = 2048: 112 K blocks in the first GEMM, 32 in
    the second) on groups that take every path of the tile scheduler: a Zipf-head group of
    7300 rows (29 chunks of 256 rows, a ragged last chunk whose second half holds 4 rows),
    one of 257 rows (a full chunk and a 1-row chunk), one of 1 row and an empty one.  Every
    output row is compared with the oracle."""
    sizes, d, I = [7300, 257, 1, 0], 7168, 2048
    rng = np.random.default_rng(71)
    G, n_rows = len(sizes), sum(sizes)
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    a = _bf16(rng.standard_normal((n_rows, d), dtype=np.float32))
    w13 = _bf16(rng.standard_normal((G, 2 * I, d), dtype=np.float32) * np.float32(0.02))
    w2 = _bf16(rng.standard_normal((G, d, I), dtype=np.float32) * np.float32(0.02))
    cfg = moe.make_config(n_rows, d, G, 1, I, 0)
    ws = torch.zeros(moe.moe_workspace_size(cfg), dtype=torch.uint8, device=DEV)
    y = torch.full((n_rows, d), float("nan"), dtype=torch.bfloat16, device=DEV)
    moe.moe_grouped_ffn(cfg, G, torch.from_numpy(offsets).to(DEV), n_rows, a.to(DEV), None,
                        w13.to(DEV), None, w2.to(DEV), None, y, ws)
    assert moe.moe_read_device_status(ws) == 0
    got = y.float().cpu().numpy()
    assert np.isfinite(got).all()
    for g in range(G):
        lo, hi = offsets[g], offsets[g + 1]
        if hi == lo:
            continue
        ref = oracle.swiglu_expert(a[lo:hi].double().numpy(), w13[g].double().numpy(),
                                   w2[g].double().numpy())
        assert max_rel_err(got[lo:hi], ref) < TOL_BF16, g
        assert row_rel_err(got[lo:hi], ref).max() < TOL_BF16, g


def test_grouped_ffn_all_groups_empty():
    """Rows allocated but every group empty: the planner yields no tiles, the persistent
    kernels exit at once, nothing is written and no status is set."""
    d, I, G, n_rows = 256, 128, 5, 32
    cfg = moe.make_config(n_rows, d, G, 1, I, 0)
    ws = torch.zeros(moe.moe_workspace_size(cfg), dtype=torch.uint8, device=DEV)
    a = torch.randn((n_rows, d), device=DEV).to(torch.bfloat16)
    w13 = torch.zeros((G, 2 * I, d), dtype=torch.bfloat16, device=DEV)
    w2 = torch.zeros((G, d, I), dtype=torch.bfloat16, device=DEV)
    y = torch.full((n_rows, d), 7.0, dtype=torch.bfloat16, device=DEV)
    offsets = torch.zeros(G + 1, dtype=torch.int32, device=DEV)
    moe.moe_grouped_ffn(cfg, G, offsets, n_rows, a, None, w13, None, w2, None, y, ws)
    assert moe.moe_read_device_status(ws) == 0
    assert bool((y == 7.0).all())


def test_layer_empty_batch_leaves_output_untouched():
    spec = inputs.custom_spec(8, 256, 8, 2, 128, 1)
    wl = margin_workload(spec, seed=8)
    layer = moe.DeviceLayer.from_workload(wl, DEV, T=0)
    y = torch.full((1, 256), 3.0, dtype=torch.bfloat16, device=DEV)
    moe.moe_layer_forward(layer.cfg, layer.weights, wl.x.to(DEV), None, y, None, None, layer.ws)
    torch.cuda.synchronize()
    assert moe.moe_read_device_status(layer.ws) == 0
    assert bool((y == 3.0).all())


def test_grouped_ffn_bad_offsets_set_device_status():
    d, I, G = 128, 128, 3
    cfg = moe.make_config(8, d, G, 1, I, 0)
    ws = torch.zeros(moe.moe_workspace_size(cfg), dtype=torch.uint8, device=DEV)
    offsets = torch.tensor([0, 5, 3, 8], dtype=torch.int32, device=DEV)     # decreasing
    a = torch.zeros((8, d), dtype=torch.bfloat16, device=DEV)
    w13 = torch.zeros((G, 2 * I, d), dtype=torch.bfloat16, device=DEV)
    w2 = torch.zeros((G, d, I), dtype=torch.bfloat16, device=DEV)
    y = torch.zeros((8, d), dtype=torch.bfloat16, device=DEV)
    moe.moe_grouped_ffn(cfg, G, offsets, 8, a, None, w13, None, w2, None, y, ws)
    assert moe.moe_read_device_status(ws) == 5


# ---------------------------------------------------------------------------
# combine alone
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("T,k,d,S", [(1, 2, 128, 0), (77, 8, 7168, 1), (64, 16, 256, 1),
                                     (50, 4, 512, 3)])
def test_combine_vs_oracle(T, k, d, S):
    """S shared experts' outputs stacked [S, T, d] are all added."""
    rng = np.random.default_rng(T * k)
    R = T * k
    y_perm = _bf16(rng.standard_normal((R, d)))
    inv = rng.permutation(R).reshape(T, k).astype(np.int32)
    w = rng.uniform(0, 1, (T, k)).astype(np.float32)
    ys = _bf16(rng.standard_normal((S, T, d))) if S else None
    cfg = moe.make_config(T, d, 16, k, 128, S)
    y = torch.empty((T, d), dtype=torch.bfloat16, device=DEV)
    moe.moe_combine(cfg, y_perm.to(DEV), torch.from_numpy(inv).to(DEV), torch.from_numpy(w).to(DEV),
                    None if ys is None else ys.to(DEV), y)
    ref = oracle.combine(y_perm.double().numpy(), inv, w.astype(np.float64),
                         None if ys is None else list(ys.double().numpy()))
    got = y.float().cpu().numpy()
    # one bf16 rounding of an fp32 sum
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-5 * np.abs(ref).max())


# ---------------------------------------------------------------------------
# the whole layer
# ---------------------------------------------------------------------------

def _run_layer(wl, T=None):
    layer = moe.DeviceLayer.from_workload(wl, DEV, T=T)
    x = wl.x.to(DEV)
    xs = None if wl.x_scale is None else wl.x_scale.to(DEV)
    idx = torch.empty((layer.cfg.T, layer.cfg.top_k), dtype=torch.int32, device=DEV)
    gw = torch.empty((layer.cfg.T, layer.cfg.top_k), dtype=torch.float32, device=DEV)
    y = layer.forward(x, xs, topk_idx=idx, topk_w=gw)
    torch.cuda.synchronize()
    assert moe.moe_read_device_status(layer.ws) == 0
    return layer, y.float().cpu().numpy(), idx.cpu().numpy(), gw.cpu().numpy()


def _check_layer(wl, rows=None):
    """The layer against the oracle: routing of every token bit-exact (indices) and within
    1e-5 (gates); outputs of every token, or of the sampled `rows`, within the bar."""
    layer, y, idx, gw = _run_layer(wl)
    if rows is not None:
        full = oracle_routing(wl)
        assert np.array_equal(idx, full["idx"])
        np.testing.assert_allclose(gw, full["gates"], rtol=1e-5, atol=1e-6)
    ref, r = oracle_layer(wl, rows=rows, return_routing=True)
    if rows is not None:
        y, idx, gw = y[rows], idx[rows], gw[rows]
    assert np.array_equal(idx, r["idx"])
    if wl.spec.act == "f32":
        # f32 inputs are rounded to bf16 on entry: each product x_i * w_i moves by up to
        # 2^-8 relative, so a logit by up to sum |x_i w_i| 2^-8 (~6e-3 at d = 128) and a
        # gate by up to a quarter of the difference of two such errors
        np.testing.assert_allclose(gw, r["gates"], rtol=0, atol=3e-3)
    else:
        np.testing.assert_allclose(gw, r["gates"], rtol=1e-5, atol=1e-6)
    err = max_rel_err(y, ref)
    assert err < TOL_BF16, err
    return layer, err


def test_layer_tiny_config():
    wl = inputs.load_workload("tiny")
    _check_layer(wl)


@pytest.mark.parametrize("T,d,E,k,I,S,score", [
    (1, 128, 8, 2, 128, 1, "sigmoid_bias"),
    (63, 256, 16, 4, 256, 1, "softmax"),
    (200, 384, 32, 8, 256, 2, "sigmoid_bias"),
    (130, 128, 1, 1, 128, 0, "softmax"),          # E = 1, k = 1: a dense SwiGLU FFN
    (520, 256, 4, 2, 128, 1, "sigmoid_bias"),     # heavy groups: several 128-row chunks each
    (96, 1024, 16, 4, 256, 1, "sigmoid_bias"),    # decode-sized, two 512-row FFN2 weight tiles
    (129, 256, 8, 4, 128, 1, "softmax"),          # smallest batch on wide (256-row) chunks
])
def test_layer_custom(T, d, E, k, I, S, score):
    spec = inputs.custom_spec(T, d, E, k, I, S, score=score)
    _check_layer(margin_workload(spec, seed=T))


@pytest.mark.parametrize("act", ["bf16", "e4m3"])
def test_layer_graph_replays_match_eager(act):
    """The layer recorded as a CUDA graph gives moe_layer_forward's results bit for bit, and
    a replay after new activations are written into x computes on the new values."""
    spec = inputs.custom_spec(96, 512, 16, 4, 256, 1, act=act, weight=act)
    wl = margin_workload(spec, seed=12)
    layer = moe.DeviceLayer.from_workload(wl, DEV)
    x = (wl.x.view(torch.uint8) if act == "e4m3" else wl.x).to(DEV)
    xv = x.view(torch.float8_e4m3fn) if act == "e4m3" else x
    xs = None if wl.x_scale is None else wl.x_scale.to(DEV)
    T, k = spec.T, spec.top_k
    y_g, y_e = layer.output(DEV), layer.output(DEV)
    idx_g = torch.empty((T, k), dtype=torch.int32, device=DEV)
    gw_g = torch.empty((T, k), dtype=torch.float32, device=DEV)
    graph = moe.LayerGraph(layer.cfg, layer.weights, xv, xs, y_g, idx_g, gw_g, layer.ws)
    other = x.flip(0).clone()
    for step in range(2):
        if step == 1:
            x.copy_(other)                 # new activations, same buffer
        graph.launch()
        torch.cuda.synchronize()
        g = (y_g.clone(), idx_g.clone(), gw_g.clone())
        idx_e = torch.empty_like(idx_g)
        gw_e = torch.empty_like(gw_g)
        layer.forward(xv, xs, y_e, idx_e, gw_e)
        torch.cuda.synchronize()
        assert torch.equal(g[0], y_e) and torch.equal(g[1], idx_e) and torch.equal(g[2], gw_e)
    assert moe.moe_read_device_status(layer.ws) == 0
    graph.close()


def test_layer_is_deterministic():
    spec = inputs.custom_spec(300, 256, 16, 4, 256, 1)
    wl = margin_workload(spec, seed=4)
    layer = moe.DeviceLayer.from_workload(wl, DEV)
    x = wl.x.to(DEV)
    a = layer.forward(x).clone()
    b = layer.forward(x).clone()
    assert torch.equal(a, b)


_FULL = {}


def _full_workload(name):
    """Full-size workloads share their expert draws within a weight family."""
    prev = _FULL.get(inputs.SPECS[name].family)
    wl = inputs.load_workload(name, reuse=prev)
    _FULL.clear()
    _FULL[wl.spec.family] = wl
    return wl


@pytest.mark.slow
@pytest.mark.parametrize("name", ["r1_decode", "r1_decode_uniform"])
def test_layer_r1_decode_full(name):
    """The DeepSeek-R1-shaped decode layer, every token checked: with the stated selection
    bias (143 experts touched) and uniformly routed (252 experts touched)."""
    wl = _full_workload(name)
    _check_layer(wl)


@pytest.mark.slow
@pytest.mark.parametrize("name", ["r1_prefill", "kimi"])
def test_layer_full_size_sampled(name):
    """Full-size prefill-shaped layers in the launch configuration the bench times.  The
    routing of every token is compared; the oracle evaluates the outputs of the tokens that
    hold the first and the last row of every 128-row token tile of every expert group
    (every group's first and last chunk among them) -- the layer is per-token, so these
    are exact comparisons of those tokens."""
    wl = _full_workload(name)
    rows = tile_edge_tokens(oracle_routing(wl), wl.spec.T, wl.spec.n_shared, 128)
    assert rows.size >= 256
    _check_layer(wl, rows=rows)
