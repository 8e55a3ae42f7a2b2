"""The seeded input generator and the stored recipes (CPU only)."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from sparse_expert_moe_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_page_shapes_match_workloads():
    with open(os.path.join(GOLDEN, "page_shapes.json")) as f:
        pages = json.load(f)
    r1 = pages["deepseek_r1"]
    for name in ("r1_decode", "r1_prefill", "r1_prefill_fp8"):
        s = inputs.SPECS[name]
        assert (s.E, s.n_shared, s.top_k) == (r1["routed_experts"], r1["shared_experts"],
                                              r1["experts_per_token"])
    t = pages["trillion_param_design"]
    s = inputs.SPECS["kimi"]
    assert (s.E, s.n_shared, s.top_k) == (t["routed_experts"], t["shared_experts"],
                                          t["experts_per_token"])


def test_draws_are_deterministic_and_per_expert():
    spec = inputs.custom_spec(T=5, d_model=128, E=3, top_k=2, d_ff=128, n_shared=1)
    a = inputs.make_workload(spec, seed=1, threads=1)
    b = inputs.make_workload(spec, seed=1, threads=3)
    for name in ("x", "wr", "sel_bias", "w13", "w2", "ws13", "ws2"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name
    q13, _, q2, _ = inputs.draw_expert(spec, 1, 2)
    assert torch.equal(q13, a.w13[2]) and torch.equal(q2, a.w2[2])
    c = inputs.make_workload(spec, seed=2, threads=1)
    assert not torch.equal(a.w13, c.w13)


def test_e4m3_scales_are_powers_of_two_and_in_range():
    spec = inputs.custom_spec(T=4, d_model=256, E=2, top_k=1, d_ff=128, act="e4m3", weight="e4m3")
    w = inputs.make_workload(spec, seed=0, threads=1)
    for s in (w.x_scale, w.w13_s, w.w2_s):
        m, _ = np.frexp(s.numpy())
        assert np.all(m == 0.5)
    for q in (w.x, w.w13, w.w2):
        v = oracle.decode_e4m3(q.view(torch.uint8).numpy())
        assert np.all(np.isfinite(v)) and np.abs(v).max() <= 448.0


def _routing_of(w):
    spec = w.spec
    if inputs.is_e4m3(spec.act):
        xv = oracle.dequantize_blocks(w.x.view(torch.uint8).numpy(), w.x_scale.numpy(), 1, 128)
    else:
        xv = w.x.double().numpy()
    L = oracle.router_logits(xv, w.wr.double().numpy())
    b = None if w.sel_bias is None else w.sel_bias.double().numpy()
    keys = oracle.selection_keys(L, spec.score, b)
    return keys, oracle.select_topk(keys, spec.top_k)


@pytest.mark.parametrize("name", ["tiny", "r1_decode"])
def test_recipe_margin_and_loads(name):
    spec = inputs.SPECS[name]
    rec = inputs.load_recipe(name)
    x32 = inputs._draw_x_fp32(spec, 0, rec["redraw"])
    x, xs = inputs.encode_act(spec, x32)
    wr = inputs.draw_router(spec, 0)
    b = inputs.draw_sel_bias(spec, 0)
    w = inputs.Workload(spec, 0, x, xs, wr, b, *([None] * 8))
    keys, idx = _routing_of(w)
    srt = -np.sort(-keys, axis=1)
    m = min(spec.top_k + 1, spec.E)
    assert np.all((srt[:, : m - 1] - srt[:, 1:m]).min(axis=1) >= spec.margin)
    assert np.bincount(idx.ravel(), minlength=spec.E).tolist() == rec["realised_loads"]


def test_zipf_recipe_summary():
    rec = inputs.load_recipe("r1_prefill")
    loads = np.asarray(rec["realised_loads"])
    target = np.asarray(rec["zipf_target_loads"])
    spec = inputs.SPECS["r1_prefill"]
    assert loads.sum() == spec.T * spec.top_k == target.sum()
    assert loads.max() <= spec.T
    # heavy-tailed like the target: same heaviest expert, similar spread
    assert np.argmax(loads) == np.argmax(target)
    assert loads.max() > 50 * np.median(loads)
    assert np.corrcoef(np.log(loads + 1), np.log(target + 1))[0, 1] > 0.99
    fp8 = inputs.load_recipe("r1_prefill_fp8")
    assert fp8["margin"] == spec.margin and "sel_bias" not in fp8


def test_reuse_gives_identical_expert_tensors():
    spec = inputs.custom_spec(T=4, d_model=128, E=2, top_k=1, d_ff=128, n_shared=1)
    a = inputs.make_workload(spec, seed=5, threads=1)
    for e in range(2):
        q13, _, q2, _ = inputs.draw_expert(spec, 5, e)
        assert torch.equal(q13, a.w13[e]) and torch.equal(q2, a.w2[e])
    q13, _, q2, _ = inputs.draw_expert(spec, 5, 0, shared=True)
    assert torch.equal(q13, a.ws13[0]) and torch.equal(q2, a.ws2[0])


def test_fp4_scale_atoms_layout_and_inverse():
    """The ABI's FP4 scale atoms: row r, 32-element run q of a 128 x 128 block at byte
    (r % 32) * 16 + (r / 32) * 4 + q of its 512-byte atom; scale_rows undoes it."""
    rng = np.random.default_rng(0)
    codes = rng.integers(0, 255, (256, 12)).astype(np.uint8)   # 2 row blocks x 3 K blocks
    at = inputs.scale_atoms(codes).numpy()
    assert at.shape == (2, 3, 512)
    for rb, kb, r, q in [(0, 0, 0, 0), (1, 2, 127, 3), (0, 1, 37, 2), (1, 0, 96, 1)]:
        assert at[rb, kb, (r % 32) * 16 + (r // 32) * 4 + q] == codes[rb * 128 + r, kb * 4 + q]
    assert np.array_equal(inputs.scale_rows(at).numpy(), codes)
