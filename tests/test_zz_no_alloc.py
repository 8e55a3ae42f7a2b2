"""moe_permute_noalloc -- the permutation for callers that cannot allocate device
memory for a workspace -- against moe_permute, through the C ABI.

Two calls in a row on different shapes: the library's internal scratch array keeps
the previous call's contents, so the second call shows the entry point clears what
it must.  The permutation is integer work, so the bar is bit-exact.  This file runs
last (it sorts after every other test file)."""
import numpy as np
import pytest
import torch

import oracle
from sparse_expert_moe_b200 import moe

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _both(T, E, k, d, seed):
    rng = np.random.default_rng(seed)
    idx, _ = oracle.route(rng.uniform(-3, 3, (T, E)), "softmax", k)
    idx_d = torch.from_numpy(idx.astype(np.int32)).to(DEV)
    x = torch.randn((T, d), generator=torch.Generator().manual_seed(seed)).to(torch.bfloat16).to(DEV)
    cfg = moe.make_config(T, d, E, k, 128, 0)
    outs = []
    for use_ws in (True, False):
        x_perm = torch.zeros((T * k, d), dtype=torch.bfloat16, device=DEV)
        perm_token = torch.full((T * k,), -9, dtype=torch.int32, device=DEV)
        inv_perm = torch.full((T, k), -9, dtype=torch.int32, device=DEV)
        offsets = torch.full((E + 1,), -9, dtype=torch.int32, device=DEV)
        if use_ws:
            ws = torch.zeros(moe.moe_workspace_size(cfg), dtype=torch.uint8, device=DEV)
            moe.moe_permute(cfg, idx_d, x, None, x_perm, None, perm_token, inv_perm, offsets, ws)
        else:
            moe.moe_permute_noalloc(cfg, idx_d, x, None, x_perm, None, perm_token, inv_perm, offsets)
        torch.cuda.synchronize()
        outs.append((x_perm.cpu(), perm_token.cpu(), inv_perm.cpu(), offsets.cpu()))
    return outs


def test_noalloc_matches_workspace_permute_twice():
    for T, E, k, d, seed in [(1000, 256, 8, 256, 1), (77, 8, 2, 128, 2)]:
        ref, got = _both(T, E, k, d, seed)
        for a, b in zip(ref, got):
            assert torch.equal(a, b)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    cfg = moe.make_config(65536 + 256, 128, 1024, 2, 128, 0)
    with pytest.raises(moe.MoeError) as e:
        moe.moe_permute_noalloc(cfg, 16, 16, None, 16, None, 16, 16, 16)
    assert e.value.code == 2
