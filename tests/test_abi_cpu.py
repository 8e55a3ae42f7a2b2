"""The C ABI library on a machine without a GPU: it loads, exports every entry point the
header declares, and its host-side checks answer without touching the device."""
import ctypes
import os

import pytest

from sparse_expert_moe_b200 import moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(moe.LIB_PATH):
        from sparse_expert_moe_b200 import build
        build.build()
    return moe.load_library()


def test_exports_every_declared_symbol(lib):
    names = moe.declared_symbols()
    assert set(names) >= {"moe_workspace_size", "moe_route", "moe_permute", "moe_grouped_ffn",
                          "moe_combine", "moe_layer_forward", "moe_read_device_status",
                          "moe_reset_device_status", "moe_status_string"}
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    assert moe.moe_status_string(0) == "ok"
    assert "workspace" in moe.moe_status_string(3)
    assert "power of two" in moe.moe_status_string(7)
    assert moe.moe_status_string(99) == "unknown status"


def test_workspace_size_host_only(lib):
    cfg = moe.make_config(128, 7168, 256, 8, 2048, 1)
    n = moe.moe_workspace_size(cfg)
    # at least x_perm, h and y rows: T*k*d*2 + (T*k + T)*(I + d)*2
    assert n >= 128 * 8 * 7168 * 2 + (128 * 9) * (2048 + 7168) * 2
    tiny = moe.make_config(64, 128, 8, 2, 256, 0, score="softmax", act="f32", weight="f32", out="f32")
    assert moe.moe_workspace_size(tiny) > 0


def test_low_precision_workspaces_host_only(lib):
    """Every accepted low-precision family sizes its workspace without a GPU, decode- and
    prefill-sized (the fp32-scale family keeps x_perm and its fp32 scales at every width)."""
    for T in (128, 8192):
        for act, weight in (("e4m3", "e4m3"), ("e4m3", "e2m1"), ("bf16", "e4m3"), ("bf16", "e2m1"),
                            ("e4m3_fs", "e4m3_fs")):
            cfg = moe.make_config(T, 7168, 256, 8, 2048, 1, act=act, weight=weight)
            n = moe.moe_workspace_size(cfg)
            # at least h (e4m3) and the bf16 expert outputs: (T*k + T) * (I + 2 d)
            assert n >= T * 9 * (2048 + 2 * 7168), (T, act, weight)
            if act == "e4m3_fs":
                # plus x_perm (e4m3) and its fp32 1x128 scales
                assert n >= T * 9 * (2048 + 2 * 7168) + T * 8 * 7168 * (1 + 4 / 128)


@pytest.mark.parametrize("kw,code", [
    (dict(top_k=9, E=8), 2),                    # k > E
    (dict(top_k=17, E=64), 2),                  # k > 16
    (dict(E=1025), 2),                          # E > 1024
    (dict(d_model=100), 2),                     # d % 128
    (dict(d_ff=200), 2),                        # I % 128
    (dict(T=-1), 1),                            # negative size
    (dict(act="e4m3", weight="bf16"), 2),       # mixed dtype family
    (dict(act="e4m3_fs", weight="e4m3"), 2),    # fp32-scale rows need fp32-scale weights
    (dict(act="e4m3", weight="e4m3_fs"), 2),    # ... and the converse
    (dict(act="bf16", weight="e4m3_fs"), 2),    # no quantising permutation to fp32 scales
    (dict(act="e2m1", weight="e2m1"), 2),       # FP4 is a weight format only
])
def test_config_rejections(lib, kw, code):
    base = dict(T=16, d_model=256, E=8, top_k=2, d_ff=256, n_shared=1)
    base.update({k: v for k, v in kw.items() if k in base})
    extra = {k: v for k, v in kw.items() if k not in base}
    cfg = moe.make_config(**base, **extra)
    out = ctypes.c_size_t(0)
    assert lib.moe_workspace_size(ctypes.byref(cfg), ctypes.byref(out)) == code


def test_null_pointers_rejected_before_launch(lib):
    cfg = moe.make_config(16, 256, 8, 2, 256, 0)
    # null logits / outputs: INVALID_ARG, no CUDA call made
    assert lib.moe_route(ctypes.byref(cfg), None, None, None, None, None) == 1
    assert lib.moe_combine(ctypes.byref(cfg), None, None, None, None, None, None) == 1
    w = moe.MoeWeights()
    assert lib.moe_layer_forward(ctypes.byref(cfg), ctypes.byref(w), None, None, None, None, None,
                                 None, 0, None) == 1
    assert lib.moe_grouped_ffn(ctypes.byref(cfg), 0, None, 0, None, None, None, None, None, None,
                               None, None, 0, None) == 1


def test_layer_graph_argument_checks(lib):
    """moe_layer_graph_create checks its arguments before recording anything; destroying a
    null handle is a no-op and launching one is rejected."""
    cfg = moe.make_config(16, 256, 8, 2, 256, 0)
    fake = 256
    w = moe.MoeWeights(fake, 0, fake, fake, 0, 0, 0, 0, 0, 0)
    h = ctypes.c_void_p(0)
    assert lib.moe_layer_graph_create(ctypes.byref(cfg), ctypes.byref(w), fake, None, fake, None,
                                      None, fake, 1024, None) == 1          # no handle pointer
    assert lib.moe_layer_graph_create(ctypes.byref(cfg), ctypes.byref(w), fake, None, fake, None,
                                      None, fake, 1024, ctypes.byref(h)) == 3  # workspace
    assert lib.moe_layer_graph_create(ctypes.byref(cfg), None, fake, None, fake, None, None, fake,
                                      1 << 30, ctypes.byref(h)) == 1
    assert h.value is None
    assert lib.moe_layer_graph_destroy(None) == 0
    assert lib.moe_layer_graph_launch(None, None) == 1


def test_noalloc_rejects_the_quantising_permutation(lib):
    """bf16 rows for e4m3 / FP4 experts are quantised by moe_permute only."""
    fake = 256
    for weight in ("e4m3", "e2m1"):
        cfg = moe.make_config(16, 256, 8, 2, 256, 0, act="bf16", weight=weight)
        assert lib.moe_permute_noalloc(ctypes.byref(cfg), fake, fake, None, fake, fake, fake, fake,
                                       fake, None) == 2


def test_workspace_too_small_rejected(lib):
    cfg = moe.make_config(16, 256, 8, 2, 256, 0)
    fake = 256  # a non-null, 16-byte-aligned address; never dereferenced on this path
    w = moe.MoeWeights(fake, 0, fake, fake, 0, 0, 0, 0, 0, 0)
    assert lib.moe_layer_forward(ctypes.byref(cfg), ctypes.byref(w), fake, None, fake, None, None,
                                 fake, 1024, None) == 3


def test_empty_batch_is_a_no_op(lib):
    """T = 0: the calls succeed without launching anything (no device needed here), and
    the workspace of an empty batch has a size (its header)."""
    cfg = moe.make_config(0, 256, 8, 2, 256, 1)
    assert moe.moe_workspace_size(cfg) >= 256
    fake = 256
    w = moe.MoeWeights(fake, 0, fake, fake, 0, 0, fake, fake, 0, 0)
    assert lib.moe_layer_forward(ctypes.byref(cfg), ctypes.byref(w), None, None, None, None, None,
                                 fake, 1 << 20, None) == 0
    assert lib.moe_route(ctypes.byref(cfg), None, None, None, None, None) == 0
    assert lib.moe_combine(ctypes.byref(cfg), None, None, None, None, None, None) == 0
