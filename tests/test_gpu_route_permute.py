"""moe_route and moe_permute on the GPU against the oracle: bit-exact indices,
permutation and offsets on fp32 logits supplied as input; gates within 1e-6."""
import numpy as np
import pytest
import torch

import oracle
from sparse_expert_moe_b200 import inputs, moe

from helpers import margin_logits

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _route_gpu(cfg, L, bias):
    T, E, k = cfg.T, cfg.E, cfg.top_k
    Ld = torch.from_numpy(L).to(DEV)
    bd = None if bias is None else torch.from_numpy(np.asarray(bias, np.float32)).to(DEV)
    idx = torch.full((T, k), -7, dtype=torch.int32, device=DEV)
    w = torch.full((T, k), -7.0, dtype=torch.float32, device=DEV)
    moe.moe_route(cfg, Ld, bd, idx, w)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), w.cpu().numpy()


CASES = [(T, E, k, score) for (E, k) in [(8, 2), (256, 8), (384, 8), (1024, 16), (33, 5)]
         for T in (1, 63, 64, 128) for score in ("softmax", "sigmoid_bias")]


@pytest.mark.parametrize("T,E,k,score", CASES)
def test_route_bit_exact(T, E, k, score):
    bias = None
    if score == "sigmoid_bias":
        bias = inputs._rng(0, 9, 99, E).uniform(-0.1, 0.1, E).astype(np.float32)
    L = margin_logits(T, E, k, score, bias, seed=T * 7 + E)
    cfg = moe.make_config(T, 128, E, k, 128, 0, score=score)
    idx, w = _route_gpu(cfg, L, bias)
    ridx, rw = oracle.route(L.astype(np.float64), score, k,
                            None if bias is None else bias.astype(np.float64))
    assert np.array_equal(idx, ridx)
    np.testing.assert_allclose(w, rw, rtol=1e-6, atol=1e-7)


@pytest.mark.parametrize("score", ["softmax", "sigmoid_bias"])
def test_route_large_T(score):
    T, E, k = 8192, 256, 8
    bias = inputs._rng(0, 9, 98, E).uniform(-0.1, 0.1, E).astype(np.float32) if score != "softmax" else None
    L = margin_logits(T, E, k, score, bias, seed=5)
    idx, w = _route_gpu(moe.make_config(T, 128, E, k, 128, 0, score=score), L, bias)
    ridx, rw = oracle.route(L.astype(np.float64), score, k,
                            None if bias is None else bias.astype(np.float64))
    assert np.array_equal(idx, ridx)
    np.testing.assert_allclose(w, rw, rtol=1e-6, atol=1e-7)


@pytest.mark.parametrize("score", ["softmax", "sigmoid_bias"])
def test_route_exact_ties_pick_lowest_experts(score):
    T, E, k = 70, 256, 8
    L = np.zeros((T, E), np.float32)
    L[1] = 0.5                       # a whole row of equal non-zero logits
    idx, w = _route_gpu(moe.make_config(T, 128, E, k, 128, 0, score=score), L, None)
    assert np.array_equal(idx, np.tile(np.arange(k, dtype=np.int32), (T, 1)))
    np.testing.assert_allclose(w, 1.0 / k, rtol=1e-6)


def test_route_forced_empty_experts():
    T, E, k = 300, 64, 8
    rng = np.random.default_rng(1)
    bias = rng.uniform(-0.1, 0.1, E).astype(np.float32)
    empty = rng.choice(E, 16, replace=False)
    bias[empty] = -2.0
    L = margin_logits(T, E, k, "sigmoid_bias", bias, seed=11)
    idx, _ = _route_gpu(moe.make_config(T, 128, E, k, 128, 0), L, bias)
    assert not np.isin(idx, empty).any()
    ridx, _ = oracle.route(L.astype(np.float64), "sigmoid_bias", k, bias.astype(np.float64))
    assert np.array_equal(idx, ridx)


# ---------------------------------------------------------------------------
# permute
# ---------------------------------------------------------------------------

def _permute_gpu(cfg, idx, x):
    T, E, k, d = cfg.T, cfg.E, cfg.top_k, cfg.d_model
    R = T * k
    ws = torch.zeros(moe.moe_workspace_size(cfg), dtype=torch.uint8, device=DEV)
    idx_d = torch.from_numpy(np.ascontiguousarray(idx, np.int32)).to(DEV)
    x_d = x.to(DEV)
    x_perm = torch.zeros((max(R, 1), d), dtype=x.dtype, device=DEV)
    perm_token = torch.full((max(R, 1),), -5, dtype=torch.int32, device=DEV)
    inv_perm = torch.full((T, k), -5, dtype=torch.int32, device=DEV)
    offsets = torch.full((E + 1,), -5, dtype=torch.int32, device=DEV)
    moe.moe_permute(cfg, idx_d, x_d, None, x_perm, None, perm_token, inv_perm, offsets, ws)
    status = moe.moe_read_device_status(ws)
    return (x_perm.cpu(), perm_token.cpu().numpy()[:R], inv_perm.cpu().numpy(),
            offsets.cpu().numpy(), status, ws)


@pytest.mark.parametrize("T,E,k", [(1, 8, 2), (63, 8, 2), (64, 256, 8), (128, 256, 8),
                                   (257, 384, 8), (1000, 1024, 16), (8192, 256, 8)])
def test_permute_bit_exact(T, E, k):
    rng = np.random.default_rng(T + E)
    L = rng.uniform(-3, 3, (T, E))
    idx, _ = oracle.route(L, "softmax", k)
    d = 256
    x = inputs.to_bf16(rng.standard_normal((T, d)).astype(np.float32))
    cfg = moe.make_config(T, d, E, k, 128, 0)
    x_perm, perm_token, inv_perm, offsets, status, _ = _permute_gpu(cfg, idx, x)
    ro, rp, ri = oracle.permute(idx, E)
    assert status == 0
    assert np.array_equal(offsets, ro)
    assert np.array_equal(perm_token, rp)
    assert np.array_equal(inv_perm, ri)
    assert torch.equal(x_perm[: T * k], x[torch.from_numpy(rp)])


def test_permute_skewed_and_empty_groups():
    # every token picks experts 0..k-1 except a few: most groups empty, one group of T rows
    T, E, k = 700, 64, 4
    idx = np.tile(np.arange(k), (T, 1))
    idx[::7] = [10, 20, 30, 63]
    x = inputs.to_bf16(np.random.default_rng(2).standard_normal((T, 128)).astype(np.float32))
    cfg = moe.make_config(T, 128, E, k, 128, 0)
    x_perm, perm_token, inv_perm, offsets, status, _ = _permute_gpu(cfg, idx, x)
    ro, rp, ri = oracle.permute(idx, E)
    assert status == 0 and np.array_equal(offsets, ro) and np.array_equal(perm_token, rp)
    assert np.array_equal(inv_perm, ri)
    assert torch.equal(x_perm, x[torch.from_numpy(rp)])


def test_permute_f32_rows_and_repeat_calls():
    T, E, k = 300, 16, 3
    rng = np.random.default_rng(3)
    idx, _ = oracle.route(rng.uniform(-3, 3, (T, E)), "softmax", k)
    x = torch.from_numpy(rng.standard_normal((T, 128)).astype(np.float32))
    cfg = moe.make_config(T, 128, E, k, 128, 0, score="softmax", act="f32", weight="f32", out="f32")
    ws = None
    for _ in range(2):   # the workspace ticket must be left ready for the next call
        x_perm, perm_token, inv_perm, offsets, status, ws = _permute_gpu(cfg, idx, x)
        ro, rp, ri = oracle.permute(idx, E)
        assert status == 0 and np.array_equal(offsets, ro) and np.array_equal(inv_perm, ri)
        assert torch.equal(x_perm, x[torch.from_numpy(rp)])


def test_permute_out_of_range_index_sets_device_status():
    T, E, k = 40, 8, 2
    idx = np.tile(np.array([0, 1]), (T, 1))
    idx[5, 1] = 8            # outside [0, E)
    idx[9, 0] = -1
    x = inputs.to_bf16(np.zeros((T, 128), np.float32))
    cfg = moe.make_config(T, 128, E, k, 128, 0)
    _, perm_token, inv_perm, offsets, status, ws = _permute_gpu(cfg, idx, x)
    assert status == 5       # MOE_ERR_DEVICE_INDEX, no trap
    assert offsets[-1] == T * k - 2
    assert inv_perm[5, 1] == -1 and inv_perm[9, 0] == -1
    moe.moe_reset_device_status(ws)
    assert moe.moe_read_device_status(ws) == 0


def test_bounded_wait_times_out_and_context_survives():
    """A wait that nothing completes ends after its budget with MOE_ERR_TIMEOUT in the
    status word (no trap, no hang), and the device keeps working afterwards."""
    ws = torch.zeros(4096, dtype=torch.uint8, device=DEV)
    moe.moe_selftest_bounded_wait(ws, 2_000_000)          # ~1 ms of SM clock
    assert moe.moe_read_device_status(ws) == 6             # MOE_ERR_TIMEOUT
    moe.moe_reset_device_status(ws)
    assert moe.moe_read_device_status(ws) == 0
    T, E, k = 16, 8, 2
    L = margin_logits(T, E, k, "softmax", None, seed=3)
    idx, _ = _route_gpu(moe.make_config(T, 128, E, k, 128, 0, score="softmax"), L, None)
    ridx, _ = oracle.route(L.astype(np.float64), "softmax", k)
    assert np.array_equal(idx, ridx)
