"""bench.py's work model: the algorithmic units the roofline fractions divide by."""
import numpy as np
import pytest

import bench
from sparse_expert_moe_b200 import inputs


def _spec(**kw):
    return inputs.custom_spec(kw.pop("T", 64), kw.pop("d", 256), kw.pop("E", 4), kw.pop("k", 2),
                              kw.pop("I", 128), kw.pop("S", 1), **kw)


def test_units_count_touched_experts_and_rows():
    spec = _spec()
    sizes = np.array([100, 0, 28, 0])                 # T k = 128 rows over 2 touched experts
    wm = bench.work_model(spec, np.concatenate([[0], np.cumsum(sizes)]))
    T, d, I = 64, 256, 128
    rows = 128 + T
    assert wm["touched"] == 2
    assert wm["ffn1_flops"] == 2.0 * rows * 2 * I * d
    assert wm["ffn2_flops"] == 2.0 * rows * I * d
    assert wm["layer_weight_bytes"] == 3 * 3 * I * d * 2 + 4 * d * 2   # 2 touched + 1 shared, + router
    assert sorted(wm["group_flops"] / (6.0 * I * d)) == [28, 64, 100]


def test_per_expert_bound_reduces_to_each_side():
    spec = _spec()
    sizes = np.array([100, 0, 28, 0])
    wm = bench.work_model(spec, np.concatenate([[0], np.cumsum(sizes)]))
    # infinite HBM: the bound is the flops alone; infinite tensor rate: the bytes alone
    assert bench.per_expert_bound_ms(wm, 1.0, 1e30) == pytest.approx(wm["group_flops"].sum() / 1e12 * 1e3)
    assert bench.per_expert_bound_ms(wm, 1e30, 1.0) == pytest.approx(wm["group_bytes"].sum() / 1e9 * 1e3)
    # a bound never below either total divided by its own peak
    b = bench.per_expert_bound_ms(wm, 1.0, 1.0)
    assert b >= max(wm["group_flops"].sum() / 1e12, wm["group_bytes"].sum() / 1e9) * 1e3


def test_small_stage_bytes_prefill_shape():
    """R1 prefill: the permutation reads x once and writes T k rows; the combine reads the
    T k routed rows and T shared rows and writes T rows (d = 7168, bf16)."""
    spec = inputs.SPECS["r1_prefill"]
    b = bench.small_stage_bytes(spec)
    T, d, k = 8192, 7168, 8
    assert b["permute"] == pytest.approx(T * d * 2 * (1 + k), rel=1e-3)
    assert b["combine"] == pytest.approx((T * k + T) * d * 2 + T * d * 2, rel=1e-3)
    assert b["route"] == pytest.approx(T * 256 * 4, rel=0.1)


def test_launch_count_per_layer_call():
    """Kernels per moe_layer_forward: 8 for the bf16 decode layer (one-chunk permutation),
    9 with the three-kernel permutation, + the FP8 scale preparation (act prep, 2 + 2
    weight-scale conversions, scale gather), + the f32 family's bf16 conversions."""
    assert bench.launches_per_step(inputs.SPECS["r1_decode"]) == 8
    assert bench.launches_per_step(inputs.SPECS["r1_prefill"]) == 9
    assert bench.launches_per_step(inputs.SPECS["kimi"]) == 9
    assert bench.launches_per_step(inputs.SPECS["r1_prefill_fp8"]) == 13   # rows gathered by FFN1
    assert bench.launches_per_step(inputs.SPECS["r1_decode_fp8"]) == 14
    assert bench.launches_per_step(inputs.SPECS["r1_decode_fp4q"]) == 8
    assert bench.launches_per_step(inputs.SPECS["tiny"]) == 12
