"""Python binding of the C ABI in ``include/moe.h`` (argument marshalling only).

Every function keeps the C name and argument order; tensors are passed as
device pointers (``tensor.data_ptr()``), ``None`` as NULL, and the stream
defaults to PyTorch's current stream.  All arithmetic happens in the CUDA
library ``libmoe_b200.so``; if it is missing the import fails loudly -- there
is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import re
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "moe.h")

MOE_OK = 0
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE",
                4: "MOE_ERR_CUDA", 5: "MOE_ERR_DEVICE_INDEX", 6: "MOE_ERR_TIMEOUT",
                7: "MOE_ERR_DEVICE_VALUE"}
SCORE = {"softmax": 0, "sigmoid_bias": 1}
DTYPE = {"f32": 0, "bf16": 1, "e4m3": 2, "e2m1": 3, "e4m3_fs": 4}


class MoeError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned {STATUS_NAMES.get(code, code)}")
        self.code = code


class MoeConfig(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d_model", ctypes.c_int32), ("E", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("d_ff", ctypes.c_int32), ("n_shared", ctypes.c_int32),
                ("d_ff_shared", ctypes.c_int32), ("score", ctypes.c_int), ("act", ctypes.c_int),
                ("weight", ctypes.c_int), ("out", ctypes.c_int)]


class MoeWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("wr", "sel_bias", "w13", "w2", "w13_s", "w2_s",
                                                "ws13", "ws2", "ws13_s", "ws2_s")]


_lib: Optional[ctypes.CDLL] = None


def load_library() -> ctypes.CDLL:
    """Load libmoe_b200.so (built by ``python -m sparse_expert_moe_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m sparse_expert_moe_b200.build` (no CPU fallback exists)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    cfgp = ctypes.POINTER(MoeConfig)
    sigs = {
        "moe_workspace_size": [cfgp, ctypes.POINTER(SZ)],
        "moe_route": [cfgp, P, P, P, P, P],
        "moe_permute": [cfgp, P, P, P, P, P, P, P, P, P, SZ, P],
        "moe_permute_noalloc": [cfgp, P, P, P, P, P, P, P, P, P],
        "moe_grouped_ffn": [cfgp, I32, P, I32, P, P, P, P, P, P, P, P, SZ, P],
        "moe_combine": [cfgp, P, P, P, P, P, P],
        "moe_layer_forward": [cfgp, ctypes.POINTER(MoeWeights), P, P, P, P, P, P, SZ, P],
        "moe_layer_forward_staged": [cfgp, ctypes.POINTER(MoeWeights), P, P, P, P, P, P, SZ, P,
                                     ctypes.POINTER(ctypes.c_void_p)],
        "moe_read_device_status": [P, P, ctypes.POINTER(ctypes.c_int)],
        "moe_reset_device_status": [P, P],
        "moe_selftest_bounded_wait": [P, ctypes.c_longlong, P],
        "moe_layer_graph_create": [cfgp, ctypes.POINTER(MoeWeights), P, P, P, P, P, P, SZ,
                                   ctypes.POINTER(ctypes.c_void_p)],
        "moe_layer_graph_launch": [P, P],
        "moe_layer_graph_destroy": [P],
    }
    for name, argtypes in sigs.items():
        fn = getattr(lib, name)
        fn.argtypes = argtypes
        fn.restype = ctypes.c_int
    lib.moe_status_string.argtypes = [ctypes.c_int]
    lib.moe_status_string.restype = ctypes.c_char_p
    _lib = lib
    return lib


def declared_symbols():
    """Names of the entry points include/moe.h declares."""
    with open(HEADER) as f:
        text = f.read()
    return re.findall(r"^MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text, flags=re.M)


# ---------------------------------------------------------------------------
# marshalling helpers
# ---------------------------------------------------------------------------

def _p(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(name: str, code: int):
    if code != MOE_OK:
        raise MoeError(name, code)


def make_config(T, d_model, E, top_k, d_ff, n_shared=0, score="sigmoid_bias", act="bf16",
                weight="bf16", out="bf16") -> MoeConfig:
    return MoeConfig(T, d_model, E, top_k, d_ff, n_shared, d_ff if n_shared else 0, SCORE[score],
                     DTYPE[act], DTYPE[weight], DTYPE[out])


def config_from_spec(spec, T: Optional[int] = None) -> MoeConfig:
    return make_config(spec.T if T is None else T, spec.d_model, spec.E, spec.top_k, spec.d_ff,
                       spec.n_shared, spec.score, spec.act, spec.weight, spec.out)


# ---------------------------------------------------------------------------
# the C entry points
# ---------------------------------------------------------------------------

def moe_workspace_size(cfg: MoeConfig) -> int:
    n = ctypes.c_size_t(0)
    _check("moe_workspace_size", load_library().moe_workspace_size(ctypes.byref(cfg), ctypes.byref(n)))
    return n.value


def moe_route(cfg, logits, sel_bias, topk_idx, topk_w, stream=None):
    _check("moe_route", load_library().moe_route(ctypes.byref(cfg), _p(logits), _p(sel_bias),
                                                 _p(topk_idx), _p(topk_w), _stream(stream)))


def moe_permute(cfg, topk_idx, x, x_scale, x_perm, x_perm_scale, perm_token, inv_perm,
                group_offsets, ws, stream=None):
    _check("moe_permute", load_library().moe_permute(
        ctypes.byref(cfg), _p(topk_idx), _p(x), _p(x_scale), _p(x_perm), _p(x_perm_scale),
        _p(perm_token), _p(inv_perm), _p(group_offsets), _p(ws), ws.numel() * ws.element_size(),
        _stream(stream)))


def moe_permute_noalloc(cfg, topk_idx, x, x_scale, x_perm, x_perm_scale, perm_token, inv_perm,
                        group_offsets, stream=None):
    """moe_permute without a workspace (scratch inside the library; see include/moe.h)."""
    _check("moe_permute_noalloc", load_library().moe_permute_noalloc(
        ctypes.byref(cfg), _p(topk_idx), _p(x), _p(x_scale), _p(x_perm), _p(x_perm_scale),
        _p(perm_token), _p(inv_perm), _p(group_offsets), _stream(stream)))


def moe_grouped_ffn(cfg, n_groups, group_offsets, n_rows, a, a_scale, w13, w13_s, w2, w2_s, y, ws,
                    stream=None):
    _check("moe_grouped_ffn", load_library().moe_grouped_ffn(
        ctypes.byref(cfg), n_groups, _p(group_offsets), n_rows, _p(a), _p(a_scale), _p(w13),
        _p(w13_s), _p(w2), _p(w2_s), _p(y), _p(ws), ws.numel() * ws.element_size(),
        _stream(stream)))


def moe_combine(cfg, y_perm, inv_perm, topk_w, y_shared, y, stream=None):
    _check("moe_combine", load_library().moe_combine(
        ctypes.byref(cfg), _p(y_perm), _p(inv_perm), _p(topk_w), _p(y_shared), _p(y),
        _stream(stream)))


def make_weights(wr, sel_bias, w13, w2, ws13=None, ws2=None, w13_s=None, w2_s=None, ws13_s=None,
                 ws2_s=None) -> MoeWeights:
    return MoeWeights(_p(wr), _p(sel_bias), _p(w13), _p(w2), _p(w13_s), _p(w2_s), _p(ws13), _p(ws2),
                      _p(ws13_s), _p(ws2_s))


def moe_layer_forward(cfg, weights: MoeWeights, x, x_scale, y, topk_idx_out, topk_w_out, ws,
                      stream=None):
    _check("moe_layer_forward", load_library().moe_layer_forward(
        ctypes.byref(cfg), ctypes.byref(weights), _p(x), _p(x_scale), _p(y), _p(topk_idx_out),
        _p(topk_w_out), _p(ws), ws.numel() * ws.element_size(), _stream(stream)))


STAGES = ("router_gemm", "route", "permute", "plan", "ffn1", "ffn2", "combine")


def moe_layer_forward_staged(cfg, weights: MoeWeights, x, x_scale, y, topk_idx_out, topk_w_out, ws,
                             events, stream=None):
    """``events``: 8 recorded-once ``torch.cuda.Event(enable_timing=True)`` objects."""
    handles = (ctypes.c_void_p * 8)(*[ev.cuda_event for ev in events])
    _check("moe_layer_forward_staged", load_library().moe_layer_forward_staged(
        ctypes.byref(cfg), ctypes.byref(weights), _p(x), _p(x_scale), _p(y), _p(topk_idx_out),
        _p(topk_w_out), _p(ws), ws.numel() * ws.element_size(), _stream(stream), handles))


class LayerGraph:
    """moe_layer_graph_create / _launch / _destroy: the layer recorded once for fixed
    tensors (x, y, routing outputs, workspace) and replayed with one graph launch."""

    def __init__(self, cfg, weights: MoeWeights, x, x_scale, y, topk_idx_out, topk_w_out, ws):
        h = ctypes.c_void_p(0)
        _check("moe_layer_graph_create", load_library().moe_layer_graph_create(
            ctypes.byref(cfg), ctypes.byref(weights), _p(x), _p(x_scale), _p(y), _p(topk_idx_out),
            _p(topk_w_out), _p(ws), ws.numel() * ws.element_size(), ctypes.byref(h)))
        self._h = h
        self._keep = (cfg, weights, x, x_scale, y, topk_idx_out, topk_w_out, ws)

    def launch(self, stream=None):
        _check("moe_layer_graph_launch", load_library().moe_layer_graph_launch(self._h, _stream(stream)))

    def close(self):
        if self._h:
            _check("moe_layer_graph_destroy", load_library().moe_layer_graph_destroy(self._h))
            self._h = ctypes.c_void_p(0)

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def moe_read_device_status(ws, stream=None) -> int:
    v = ctypes.c_int(0)
    _check("moe_read_device_status",
           load_library().moe_read_device_status(_p(ws), _stream(stream), ctypes.byref(v)))
    return v.value


def moe_reset_device_status(ws, stream=None):
    _check("moe_reset_device_status", load_library().moe_reset_device_status(_p(ws), _stream(stream)))


def moe_selftest_bounded_wait(ws, budget_cycles, stream=None):
    _check("moe_selftest_bounded_wait",
           load_library().moe_selftest_bounded_wait(_p(ws), int(budget_cycles), _stream(stream)))


def moe_status_string(code: int) -> str:
    return load_library().moe_status_string(code).decode()


# ---------------------------------------------------------------------------
# a resident layer: weights and workspace on the device
# ---------------------------------------------------------------------------

_TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16, "e4m3": torch.float8_e4m3fn,
                "e4m3_fs": torch.float8_e4m3fn}


@dataclass
class DeviceLayer:
    """One layer's weights and workspace held in device memory."""
    cfg: MoeConfig
    tensors: dict
    weights: MoeWeights
    ws: torch.Tensor

    @classmethod
    def from_workload(cls, wl, device="cuda", T: Optional[int] = None):
        spec = wl.spec
        cfg = config_from_spec(spec, T)
        names = ("wr", "sel_bias", "w13", "w2", "w13_s", "w2_s", "ws13", "ws2", "ws13_s", "ws2_s")
        ten = {}
        for n in names:
            t = getattr(wl, n)
            ten[n] = None if t is None else t.to(device, non_blocking=False)
        weights = make_weights(ten["wr"], ten["sel_bias"], ten["w13"], ten["w2"], ten["ws13"],
                               ten["ws2"], ten["w13_s"], ten["w2_s"], ten["ws13_s"], ten["ws2_s"])
        ws = torch.zeros(moe_workspace_size(cfg), dtype=torch.uint8, device=device)
        return cls(cfg, ten, weights, ws)

    def output(self, device="cuda"):
        dt = torch.float32 if self.cfg.out == DTYPE["f32"] else torch.bfloat16
        return torch.empty((self.cfg.T, self.cfg.d_model), dtype=dt, device=device)

    def forward(self, x, x_scale=None, y=None, topk_idx=None, topk_w=None, stream=None):
        if y is None:
            y = self.output(x.device)
        moe_layer_forward(self.cfg, self.weights, x, x_scale, y, topk_idx, topk_w, self.ws, stream)
        return y
