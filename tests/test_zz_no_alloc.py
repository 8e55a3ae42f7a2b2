"""moe_permute_noalloc -- the permutation for callers that cannot allocate device
memory for a workspace -- through the C ABI.

Its results must equal the oracle's permutation (the dispatch step of the moe_ffn
pseudocode: expert-major groups, ascending token inside a group) and moe_permute's,
bit for bit, for every activation dtype the layer takes: bf16, f32, and e4m3 rows
with their fp32 1x128 scales.  Every output buffer carries one guard row of sentinel
bytes after its end, which must come back untouched.  The shapes run two calls in a
row: the library's internal scratch array keeps the previous call's contents, so the
second call shows the entry point clears what it must.  This file runs last (it sorts
after every other test file)."""
import numpy as np
import pytest
import torch

import oracle
from sparse_expert_moe_b200 import inputs, moe

pytestmark = pytest.mark.gpu
DEV = "cuda"
SENTINEL = 0xA5


def _guarded(rows, cols, dtype):
    """A [rows + 1, cols] buffer of sentinel bytes; the caller gets rows 0..rows-1."""
    buf = torch.full(((rows + 1) * cols * torch.empty((), dtype=dtype).element_size(),), SENTINEL,
                     dtype=torch.uint8, device=DEV)
    return buf, buf.view(dtype).view(rows + 1, cols)


def _inputs(T, E, k, d, act, seed):
    rng = np.random.default_rng(seed)
    idx, _ = oracle.route(rng.uniform(-3, 3, (T, E)), "softmax", k)
    x32 = rng.standard_normal((T, d)).astype(np.float32)
    xs = None
    if act == "bf16":
        x = inputs.to_bf16(x32)
    elif act == "f32":
        x = torch.from_numpy(x32)
    else:
        x, xs = inputs.to_e4m3_blocks(x32 * np.exp2(rng.integers(-4, 4, (T, 1))), 1, 128)
        x = x.view(torch.uint8)
    return idx, x, xs


def _run(T, E, k, d, act, idx, x, xs, use_ws):
    """One permutation through the C ABI; returns the outputs with their guard rows."""
    R = T * k
    dt = {"bf16": torch.bfloat16, "f32": torch.float32, "e4m3": torch.uint8}[act]
    cfg = moe.make_config(T, d, E, k, 128, 0, score="softmax", act=act, weight=act,
                          out="f32" if act == "f32" else "bf16")
    raw = {}
    raw["x_perm"], x_perm = _guarded(R, d, dt)
    raw["perm_token"], perm_token = _guarded(R, 1, torch.int32)
    raw["inv_perm"], inv_perm = _guarded(R, 1, torch.int32)
    raw["offsets"], offsets = _guarded(E + 1, 1, torch.int32)
    x_perm_s = None
    if act == "e4m3":
        raw["x_perm_s"], x_perm_s = _guarded(R, d // 128, torch.float32)
    idx_d = torch.from_numpy(idx.astype(np.int32)).to(DEV)
    x_d = x.to(DEV)
    xs_d = None if xs is None else xs.to(DEV)
    if use_ws:
        ws = torch.zeros(moe.moe_workspace_size(cfg), dtype=torch.uint8, device=DEV)
        moe.moe_permute(cfg, idx_d, x_d, xs_d, x_perm, x_perm_s, perm_token, inv_perm, offsets, ws)
    else:
        moe.moe_permute_noalloc(cfg, idx_d, x_d, xs_d, x_perm, x_perm_s, perm_token, inv_perm,
                                offsets)
    torch.cuda.synchronize()
    return {n: b.cpu() for n, b in raw.items()}


def _views(out, T, E, k, d, act):
    """The outputs proper (guard rows stripped) and the guard rows."""
    R = T * k
    dt = {"bf16": torch.bfloat16, "f32": torch.float32, "e4m3": torch.uint8}[act]
    esz = torch.empty((), dtype=dt).element_size()
    body = {"x_perm": out["x_perm"][: R * d * esz].view(dt).view(R, d),
            "perm_token": out["perm_token"][: R * 4].view(torch.int32),
            "inv_perm": out["inv_perm"][: R * 4].view(torch.int32).view(T, k),
            "offsets": out["offsets"][: (E + 1) * 4].view(torch.int32)}
    guard = {"x_perm": out["x_perm"][R * d * esz:], "perm_token": out["perm_token"][R * 4:],
             "inv_perm": out["inv_perm"][R * 4:], "offsets": out["offsets"][(E + 1) * 4:]}
    if act == "e4m3":
        body["x_perm_s"] = out["x_perm_s"][: R * (d // 128) * 4].view(torch.float32).view(R, d // 128)
        guard["x_perm_s"] = out["x_perm_s"][R * (d // 128) * 4:]
    return body, guard


SHAPES = [
    # (T, E, k, d, act, seed): each dtype twice in a row on different shapes
    (300, 32, 4, 256, "e4m3", 1), (77, 8, 2, 384, "e4m3", 2),
    (1000, 256, 8, 256, "bf16", 3), (77, 8, 2, 128, "bf16", 4),
    (257, 16, 3, 128, "f32", 5), (40, 64, 8, 256, "f32", 6),
]


@pytest.mark.parametrize("act", ["e4m3", "bf16", "f32"])
def test_noalloc_matches_oracle_and_workspace_permute_twice(act):
    for T, E, k, d, a, seed in [s for s in SHAPES if s[4] == act]:
        idx, x, xs = _inputs(T, E, k, d, act, seed)
        ro, rp, ri = oracle.permute(idx, E)
        got, guard = _views(_run(T, E, k, d, act, idx, x, xs, use_ws=False), T, E, k, d, act)
        for name, g in guard.items():
            assert bool((g == SENTINEL).all()), f"{act} T={T}: write past the end of {name}"
        assert np.array_equal(got["offsets"].numpy(), ro)
        assert np.array_equal(got["perm_token"].numpy(), rp)
        assert np.array_equal(got["inv_perm"].numpy(), ri)
        tp = torch.from_numpy(rp)
        assert torch.equal(got["x_perm"], x[tp])
        if act == "e4m3":
            assert torch.equal(got["x_perm_s"], xs[tp])
        ref, _ = _views(_run(T, E, k, d, act, idx, x, xs, use_ws=True), T, E, k, d, act)
        for name in ref:
            assert torch.equal(got[name], ref[name]), name


def test_noalloc_e4m3_requires_scales():
    cfg = moe.make_config(16, 128, 8, 2, 128, 0, act="e4m3", weight="e4m3")
    with pytest.raises(moe.MoeError) as e:
        moe.moe_permute_noalloc(cfg, 16, 16, None, 16, None, 16, 16, 16)
    assert e.value.code == 1


def test_noalloc_rejects_shapes_beyond_its_scratch():
    cfg = moe.make_config(65536 + 256, 128, 1024, 2, 128, 0)
    with pytest.raises(moe.MoeError) as e:
        moe.moe_permute_noalloc(cfg, 16, 16, None, 16, None, 16, 16, 16)
    assert e.value.code == 2
