"""Thin Python binding of libmoe_b200.so (the C ABI in include/moe.h).

Argument marshalling only: each function checks dtypes, devices and
contiguity of torch tensors and passes their device pointers, sizes and the
current CUDA stream to the C entry point of the same name. Every step of the
layer runs in the library's CUDA kernels; there is no Python or CPU fallback,
and loading fails loudly when the shared library is missing.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

_lib = None

MOE_OK = 0
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_INVALID_ARG", 2: "MOE_UNSUPPORTED_SHAPE",
                3: "MOE_WORKSPACE_TOO_SMALL", 4: "MOE_CUDA_ERROR", 5: "MOE_DEVICE_TIMEOUT",
                6: "MOE_BAD_EXPERT_ID", 7: "MOE_BAD_SCHEDULE"}
DEV_BAD_EXPERT_ID = 0x1
DEV_TIMEOUT = 0x2
DEV_BAD_SCHEDULE = 0x4
N_STAGE_EVENTS = 7
STAGES = ("route", "schedule", "dispatch", "ffn_gemm1", "ffn_gemm2", "combine")
N_BWD_EVENTS = 8
BWD_STAGES = ("reverse_combine", "dgrad_h", "dgrad_x", "reverse_dispatch", "router_bwd",
              "wgrad_w2", "wgrad_w13")


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")
        self.status = status


class Shape(ctypes.Structure):
    _fields_ = [("P", ctypes.c_int32), ("N", ctypes.c_int32), ("E", ctypes.c_int32),
                ("k", ctypes.c_int32), ("H", ctypes.c_int32), ("I", ctypes.c_int32),
                ("pad", ctypes.c_int32)]

    def __repr__(self):
        return "Shape(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


def shape(P: int, N: int, E: int, k: int, H: int = 0, I: int = 0, pad: int = 256) -> Shape:
    return Shape(P, N, E, k, H, I, pad)


_vp = ctypes.c_void_p
_SIGS = {
    "moe_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "moe_status_from_device_flags": ([ctypes.c_int32], ctypes.c_int),
    "moe_rows_max": ([ctypes.POINTER(Shape)], ctypes.c_int64),
    "moe_schedule_workspace_bytes": ([ctypes.POINTER(Shape)], ctypes.c_size_t),
    "moe_layer_workspace_bytes": ([ctypes.POINTER(Shape)], ctypes.c_size_t),
    "moe_layer_host_workspace_bytes": ([ctypes.POINTER(Shape)], ctypes.c_size_t),
    "moe_route_topk": ([_vp, _vp, _vp, ctypes.POINTER(Shape), _vp], ctypes.c_int),
    "moe_schedule": ([_vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp, ctypes.POINTER(Shape),
                      _vp], ctypes.c_int),
    "moe_dispatch": ([_vp, _vp, _vp, _vp, _vp, ctypes.POINTER(Shape), _vp], ctypes.c_int),
    "moe_expert_ffn": ([_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(Shape), _vp],
                       ctypes.c_int),
    "moe_expert_ffn_gather": ([_vp] * 10 + [ctypes.POINTER(Shape), _vp], ctypes.c_int),
    "moe_combine": ([_vp, _vp, _vp, _vp, _vp, ctypes.POINTER(Shape), _vp], ctypes.c_int),
    "moe_layer_forward": ([_vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_int32, _vp, ctypes.c_size_t, _vp,
                           ctypes.POINTER(Shape), _vp, ctypes.POINTER(_vp)], ctypes.c_int),
    "moe_layer_forward_host": ([_vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_int32, _vp,
                                ctypes.c_size_t, _vp, ctypes.POINTER(Shape), _vp], ctypes.c_int),
    "moe_layer_forward_host_async": ([_vp] * 6 + [ctypes.c_int32, _vp, ctypes.c_size_t, _vp,
                                      ctypes.POINTER(Shape), _vp, _vp], ctypes.c_int),
    "moe_schedule_static_ws": ([_vp, _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(Shape), _vp],
                               ctypes.c_int),
    "moe_train_workspace_bytes": ([ctypes.POINTER(Shape)], ctypes.c_size_t),
    "moe_expert_ffn_train": ([_vp] * 10 + [ctypes.POINTER(Shape), _vp], ctypes.c_int),
    "moe_layer_forward_train": ([_vp] * 7 + [ctypes.c_size_t, _vp, ctypes.POINTER(Shape), _vp,
                                              ctypes.POINTER(_vp)], ctypes.c_int),
    "moe_reverse_combine": ([_vp] * 8 + [ctypes.POINTER(Shape), _vp], ctypes.c_int),
    "moe_expert_ffn_dgrad": ([_vp] * 14 + [ctypes.POINTER(Shape), _vp], ctypes.c_int),
    "moe_reverse_dispatch": ([_vp] * 4 + [ctypes.POINTER(Shape), _vp], ctypes.c_int),
    "moe_router_backward": ([_vp] * 6 + [ctypes.POINTER(Shape), _vp], ctypes.c_int),
    "moe_expert_ffn_wgrad": ([_vp] * 10 + [ctypes.POINTER(Shape), _vp], ctypes.c_int),
    "moe_layer_backward": ([_vp] * 10 + [ctypes.c_size_t, _vp, ctypes.POINTER(Shape), _vp,
                                         ctypes.POINTER(_vp)], ctypes.c_int),
    "moe_mx_quantize_rows": ([_vp, ctypes.c_int64, ctypes.c_int32, _vp, _vp, _vp], ctypes.c_int),
    "moe_dispatch_mxfp8": ([_vp] * 6 + [ctypes.POINTER(Shape), _vp], ctypes.c_int),
    "moe_dispatch_mxfp8_tiled": ([_vp] * 6 + [ctypes.POINTER(Shape), _vp], ctypes.c_int),
    "moe_mx_quantize_weights": ([_vp, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, _vp, _vp, _vp],
                                ctypes.c_int),
    "moe_expert_ffn_mxfp8": ([_vp] * 14 + [ctypes.POINTER(Shape), _vp], ctypes.c_int),
    "moe_layer_forward_mxfp8": ([_vp] * 13 + [ctypes.c_size_t, _vp, ctypes.POINTER(Shape), _vp,
                                              ctypes.POINTER(_vp)], ctypes.c_int),
    "moe_layer_mxfp8_workspace_bytes": ([ctypes.POINTER(Shape)], ctypes.c_size_t),
    "moe_launch_count": ([], ctypes.c_int64),
    "moe_selftest_bounded_wait": ([_vp, ctypes.c_int64, _vp], ctypes.c_int),
    "moe_selftest_schedule_barrier": ([_vp] * 6 + [ctypes.c_size_t, _vp, ctypes.POINTER(Shape),
                                                   ctypes.c_int64, _vp], ctypes.c_int),
}


def load():
    """Load the shared library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -c 'import __graft_entry__ as g; g.build()'`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def exported_symbols():
    return sorted(_SIGS)


# ---------------------------------------------------------------- marshalling
def _ptr(t: torch.Tensor | None, dtype: torch.dtype, name: str, device=True):
    if t is None:
        return None
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if device and not t.is_cuda:
        raise TypeError(f"{name}: expected a CUDA tensor")
    if not device and t.is_cuda:
        raise TypeError(f"{name}: expected a host tensor")
    if not t.is_contiguous():
        raise TypeError(f"{name}: must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(status: int, where: str):
    if status != MOE_OK:
        raise MoeError(status, where)


def status_string(status: int) -> str:
    return load().moe_status_string(status).decode()


def status_from_device_flags(flags: int) -> int:
    return load().moe_status_from_device_flags(int(flags))


def rows_max(sh: Shape) -> int:
    return int(load().moe_rows_max(ctypes.byref(sh)))


def schedule_workspace_bytes(sh: Shape) -> int:
    return int(load().moe_schedule_workspace_bytes(ctypes.byref(sh)))


def layer_workspace_bytes(sh: Shape) -> int:
    return int(load().moe_layer_workspace_bytes(ctypes.byref(sh)))


def layer_host_workspace_bytes(sh: Shape) -> int:
    return int(load().moe_layer_host_workspace_bytes(ctypes.byref(sh)))


def layer_mxfp8_workspace_bytes(sh: Shape) -> int:
    return int(load().moe_layer_mxfp8_workspace_bytes(ctypes.byref(sh)))


def train_workspace_bytes(sh: Shape) -> int:
    return int(load().moe_train_workspace_bytes(ctypes.byref(sh)))


def launch_count() -> int:
    return int(load().moe_launch_count())


# ---------------------------------------------------------------- entry points
def moe_route_topk(logits, ids, gates, sh: Shape, stream=None):
    _check(load().moe_route_topk(_ptr(logits, torch.float32, "logits"),
                                 _ptr(ids, torch.int32, "ids"), _ptr(gates, torch.float32, "gates"),
                                 ctypes.byref(sh), _stream(stream)), "moe_route_topk")


def moe_schedule(ids, phi, offsets, counts, route_row, ws, dev_status, sh: Shape, stream=None):
    _check(load().moe_schedule(_ptr(ids, torch.int32, "ids"), _ptr(phi, torch.int32, "phi"),
                               _ptr(offsets, torch.int32, "offsets"),
                               _ptr(counts, torch.int32, "counts"),
                               _ptr(route_row, torch.int32, "route_row"),
                               _ptr(ws, torch.uint8, "ws"), ws.numel(),
                               _ptr(dev_status, torch.int32, "dev_status"), ctypes.byref(sh),
                               _stream(stream)), "moe_schedule")


def moe_schedule_static_ws(ids, phi, offsets, counts, route_row, dev_status, sh: Shape,
                           stream=None):
    """moe_schedule with the library's fixed 4 MiB device scratch instead of a
    caller-provided workspace (for callers that cannot allocate one)."""
    _check(load().moe_schedule_static_ws(_ptr(ids, torch.int32, "ids"),
                                         _ptr(phi, torch.int32, "phi"),
                                         _ptr(offsets, torch.int32, "offsets"),
                                         _ptr(counts, torch.int32, "counts"),
                                         _ptr(route_row, torch.int32, "route_row"),
                                         _ptr(dev_status, torch.int32, "dev_status"),
                                         ctypes.byref(sh), _stream(stream)),
           "moe_schedule_static_ws")


def moe_dispatch(x, phi, offsets, xg, dev_status, sh: Shape, stream=None):
    _check(load().moe_dispatch(_ptr(x, torch.bfloat16, "x"), _ptr(phi, torch.int32, "phi"),
                               _ptr(offsets, torch.int32, "offsets"),
                               _ptr(xg, torch.bfloat16, "xg"),
                               _ptr(dev_status, torch.int32, "dev_status"), ctypes.byref(sh),
                               _stream(stream)), "moe_dispatch")


def moe_expert_ffn(xg, W1, W3, W2, offsets, counts, h, y, dev_status, sh: Shape, stream=None):
    _check(load().moe_expert_ffn(_ptr(xg, torch.bfloat16, "xg"), _ptr(W1, torch.bfloat16, "W1"),
                                 _ptr(W3, torch.bfloat16, "W3"), _ptr(W2, torch.bfloat16, "W2"),
                                 _ptr(offsets, torch.int32, "offsets"),
                                 _ptr(counts, torch.int32, "counts"),
                                 _ptr(h, torch.bfloat16, "h"), _ptr(y, torch.float32, "y"),
                                 _ptr(dev_status, torch.int32, "dev_status"), ctypes.byref(sh),
                                 _stream(stream)), "moe_expert_ffn")


def moe_expert_ffn_gather(x, phi, W1, W3, W2, offsets, counts, h, y, dev_status, sh: Shape,
                          stream=None):
    _check(load().moe_expert_ffn_gather(_ptr(x, torch.bfloat16, "x"), _ptr(phi, torch.int32, "phi"),
                                        _ptr(W1, torch.bfloat16, "W1"),
                                        _ptr(W3, torch.bfloat16, "W3"),
                                        _ptr(W2, torch.bfloat16, "W2"),
                                        _ptr(offsets, torch.int32, "offsets"),
                                        _ptr(counts, torch.int32, "counts"),
                                        _ptr(h, torch.bfloat16, "h"), _ptr(y, torch.float32, "y"),
                                        _ptr(dev_status, torch.int32, "dev_status"),
                                        ctypes.byref(sh), _stream(stream)), "moe_expert_ffn_gather")


def moe_combine(y, route_row, gates, out, dev_status, sh: Shape, stream=None):
    _check(load().moe_combine(_ptr(y, torch.float32, "y"),
                              _ptr(route_row, torch.int32, "route_row"),
                              _ptr(gates, torch.float32, "gates"), _ptr(out, torch.bfloat16, "out"),
                              _ptr(dev_status, torch.int32, "dev_status"), ctypes.byref(sh),
                              _stream(stream)), "moe_combine")


def _events(events, n=N_STAGE_EVENTS):
    if events is None:
        return None
    if len(events) != n:
        raise ValueError(f"need {n} events")
    arr = (ctypes.c_void_p * n)()
    for i, e in enumerate(events):
        arr[i] = e.cuda_event if hasattr(e, "cuda_event") else int(e)
    return ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p))


def moe_layer_forward(logits, x, W1, W3, W2, out, ws, dev_status, sh: Shape, minibatch_tokens=0,
                      stream=None, stage_events=None):
    _check(load().moe_layer_forward(_ptr(logits, torch.float32, "logits"),
                                    _ptr(x, torch.bfloat16, "x"), _ptr(W1, torch.bfloat16, "W1"),
                                    _ptr(W3, torch.bfloat16, "W3"), _ptr(W2, torch.bfloat16, "W2"),
                                    _ptr(out, torch.bfloat16, "out"), int(minibatch_tokens),
                                    _ptr(ws, torch.uint8, "ws"), ws.numel(),
                                    _ptr(dev_status, torch.int32, "dev_status"),
                                    ctypes.byref(sh), _stream(stream), _events(stage_events)),
           "moe_layer_forward")


def moe_layer_forward_host(logits_host, x_host, W1, W3, W2, out_host, ws, dev_status, sh: Shape,
                           minibatch_tokens=0, stream=None):
    _check(load().moe_layer_forward_host(
        _ptr(logits_host, torch.float32, "logits_host", device=False),
        _ptr(x_host, torch.bfloat16, "x_host", device=False), _ptr(W1, torch.bfloat16, "W1"),
        _ptr(W3, torch.bfloat16, "W3"), _ptr(W2, torch.bfloat16, "W2"),
        _ptr(out_host, torch.bfloat16, "out_host", device=False), int(minibatch_tokens),
        _ptr(ws, torch.uint8, "ws"), ws.numel(), _ptr(dev_status, torch.int32, "dev_status"),
        ctypes.byref(sh), _stream(stream)), "moe_layer_forward_host")


# ---------------------------------------------------------------- backward
def moe_expert_ffn_train(xg, W1, W3, W2, offsets, counts, h, ab, y, dev_status, sh: Shape,
                         stream=None):
    _check(load().moe_expert_ffn_train(_ptr(xg, torch.bfloat16, "xg"), _ptr(W1, torch.bfloat16, "W1"),
                                       _ptr(W3, torch.bfloat16, "W3"), _ptr(W2, torch.bfloat16, "W2"),
                                       _ptr(offsets, torch.int32, "offsets"),
                                       _ptr(counts, torch.int32, "counts"),
                                       _ptr(h, torch.bfloat16, "h"), _ptr(ab, torch.bfloat16, "ab"),
                                       _ptr(y, torch.float32, "y"),
                                       _ptr(dev_status, torch.int32, "dev_status"),
                                       ctypes.byref(sh), _stream(stream)), "moe_expert_ffn_train")


def moe_layer_forward_train(logits, x, W1, W3, W2, out, ws, dev_status, sh: Shape, stream=None,
                            stage_events=None):
    _check(load().moe_layer_forward_train(_ptr(logits, torch.float32, "logits"),
                                          _ptr(x, torch.bfloat16, "x"),
                                          _ptr(W1, torch.bfloat16, "W1"),
                                          _ptr(W3, torch.bfloat16, "W3"),
                                          _ptr(W2, torch.bfloat16, "W2"),
                                          _ptr(out, torch.bfloat16, "out"),
                                          _ptr(ws, torch.uint8, "ws"), ws.numel(),
                                          _ptr(dev_status, torch.int32, "dev_status"),
                                          ctypes.byref(sh), _stream(stream),
                                          _events(stage_events)), "moe_layer_forward_train")


def moe_reverse_combine(dout, phi, offsets, route_row, gates, dys, gate_row, dev_status, sh: Shape,
                        stream=None):
    _check(load().moe_reverse_combine(_ptr(dout, torch.bfloat16, "dout"),
                                      _ptr(phi, torch.int32, "phi"),
                                      _ptr(offsets, torch.int32, "offsets"),
                                      _ptr(route_row, torch.int32, "route_row"),
                                      _ptr(gates, torch.float32, "gates"),
                                      _ptr(dys, torch.bfloat16, "dys"),
                                      _ptr(gate_row, torch.float32, "gate_row"),
                                      _ptr(dev_status, torch.int32, "dev_status"),
                                      ctypes.byref(sh), _stream(stream)), "moe_reverse_combine")


def moe_expert_ffn_dgrad(dys, gate_row, ab, h, W1, W3, W2, offsets, counts, dab, hg, dgate_part,
                         dxg, dev_status, sh: Shape, stream=None):
    _check(load().moe_expert_ffn_dgrad(_ptr(dys, torch.bfloat16, "dys"),
                                       _ptr(gate_row, torch.float32, "gate_row"),
                                       _ptr(ab, torch.bfloat16, "ab"), _ptr(h, torch.bfloat16, "h"),
                                       _ptr(W1, torch.bfloat16, "W1"), _ptr(W3, torch.bfloat16, "W3"),
                                       _ptr(W2, torch.bfloat16, "W2"),
                                       _ptr(offsets, torch.int32, "offsets"),
                                       _ptr(counts, torch.int32, "counts"),
                                       _ptr(dab, torch.bfloat16, "dab"),
                                       _ptr(hg, torch.bfloat16, "hg"),
                                       _ptr(dgate_part, torch.float32, "dgate_part"),
                                       _ptr(dxg, torch.float32, "dxg"),
                                       _ptr(dev_status, torch.int32, "dev_status"),
                                       ctypes.byref(sh), _stream(stream)), "moe_expert_ffn_dgrad")


def moe_reverse_dispatch(dxg, route_row, dx, dev_status, sh: Shape, stream=None):
    _check(load().moe_reverse_dispatch(_ptr(dxg, torch.float32, "dxg"),
                                       _ptr(route_row, torch.int32, "route_row"),
                                       _ptr(dx, torch.bfloat16, "dx"),
                                       _ptr(dev_status, torch.int32, "dev_status"),
                                       ctypes.byref(sh), _stream(stream)), "moe_reverse_dispatch")


def moe_router_backward(dgate_part, route_row, ids, gates, dlogits, dev_status, sh: Shape,
                        stream=None):
    _check(load().moe_router_backward(_ptr(dgate_part, torch.float32, "dgate_part"),
                                      _ptr(route_row, torch.int32, "route_row"),
                                      _ptr(ids, torch.int32, "ids"),
                                      _ptr(gates, torch.float32, "gates"),
                                      _ptr(dlogits, torch.float32, "dlogits"),
                                      _ptr(dev_status, torch.int32, "dev_status"),
                                      ctypes.byref(sh), _stream(stream)), "moe_router_backward")


def moe_expert_ffn_wgrad(xg, dys, dab, hg, offsets, counts, dW1, dW3, dW2, dev_status, sh: Shape,
                         stream=None):
    _check(load().moe_expert_ffn_wgrad(_ptr(xg, torch.bfloat16, "xg"),
                                       _ptr(dys, torch.bfloat16, "dys"),
                                       _ptr(dab, torch.bfloat16, "dab"),
                                       _ptr(hg, torch.bfloat16, "hg"),
                                       _ptr(offsets, torch.int32, "offsets"),
                                       _ptr(counts, torch.int32, "counts"),
                                       _ptr(dW1, torch.float32, "dW1"),
                                       _ptr(dW3, torch.float32, "dW3"),
                                       _ptr(dW2, torch.float32, "dW2"),
                                       _ptr(dev_status, torch.int32, "dev_status"),
                                       ctypes.byref(sh), _stream(stream)), "moe_expert_ffn_wgrad")


def moe_layer_backward(dout, W1, W3, W2, dx, dlogits, dW1, dW3, dW2, ws, dev_status, sh: Shape,
                       stream=None, stage_events=None):
    _check(load().moe_layer_backward(_ptr(dout, torch.bfloat16, "dout"),
                                     _ptr(W1, torch.bfloat16, "W1"), _ptr(W3, torch.bfloat16, "W3"),
                                     _ptr(W2, torch.bfloat16, "W2"), _ptr(dx, torch.bfloat16, "dx"),
                                     _ptr(dlogits, torch.float32, "dlogits"),
                                     _ptr(dW1, torch.float32, "dW1"),
                                     _ptr(dW3, torch.float32, "dW3"),
                                     _ptr(dW2, torch.float32, "dW2"),
                                     _ptr(ws, torch.uint8, "ws"), ws.numel(),
                                     _ptr(dev_status, torch.int32, "dev_status"),
                                     ctypes.byref(sh), _stream(stream),
                                     _events(stage_events, N_BWD_EVENTS)), "moe_layer_backward")


def moe_layer_forward_host_async(logits_host, x_host, W1, W3, W2, out_host, ws, dev_status,
                                 sh: Shape, out_ready, minibatch_tokens=0, stream=None):
    """out_ready: a torch.cuda.Event (recorded once before first use, so that it
    exists) or a raw cudaEvent_t; it completes when out_host holds the output."""
    ev = out_ready.cuda_event if hasattr(out_ready, "cuda_event") else int(out_ready)
    if not ev:
        raise ValueError("out_ready: the event has not been created (record it once first)")
    _check(load().moe_layer_forward_host_async(
        _ptr(logits_host, torch.float32, "logits_host", device=False),
        _ptr(x_host, torch.bfloat16, "x_host", device=False), _ptr(W1, torch.bfloat16, "W1"),
        _ptr(W3, torch.bfloat16, "W3"), _ptr(W2, torch.bfloat16, "W2"),
        _ptr(out_host, torch.bfloat16, "out_host", device=False), int(minibatch_tokens),
        _ptr(ws, torch.uint8, "ws"), ws.numel(), _ptr(dev_status, torch.int32, "dev_status"),
        ctypes.byref(sh), _stream(stream), ctypes.c_void_p(ev)), "moe_layer_forward_host_async")


# ---------------------------------------------------------------- MXFP8
def moe_mx_quantize_rows(src, q, scale, stream=None):
    """src bf16 [n, K] -> q uint8 [n, K] E4M3 codes, scale uint8 [n, K/32] E8M0 codes."""
    n, K = src.shape
    _check(load().moe_mx_quantize_rows(_ptr(src, torch.bfloat16, "src"), n, K,
                                       _ptr(q, torch.uint8, "q"), _ptr(scale, torch.uint8, "scale"),
                                       _stream(stream)), "moe_mx_quantize_rows")


def moe_dispatch_mxfp8(x, phi, offsets, xq, xs, dev_status, sh: Shape, stream=None):
    _check(load().moe_dispatch_mxfp8(_ptr(x, torch.bfloat16, "x"), _ptr(phi, torch.int32, "phi"),
                                     _ptr(offsets, torch.int32, "offsets"),
                                     _ptr(xq, torch.uint8, "xq"), _ptr(xs, torch.uint8, "xs"),
                                     _ptr(dev_status, torch.int32, "dev_status"), ctypes.byref(sh),
                                     _stream(stream)), "moe_dispatch_mxfp8")


def moe_dispatch_mxfp8_tiled(x, phi, offsets, xq, xs, dev_status, sh: Shape, stream=None):
    """moe_dispatch_mxfp8 with xs in the tiled scale layout of include/moe.h."""
    _check(load().moe_dispatch_mxfp8_tiled(
        _ptr(x, torch.bfloat16, "x"), _ptr(phi, torch.int32, "phi"),
        _ptr(offsets, torch.int32, "offsets"), _ptr(xq, torch.uint8, "xq"),
        _ptr(xs, torch.uint8, "xs"), _ptr(dev_status, torch.int32, "dev_status"),
        ctypes.byref(sh), _stream(stream)), "moe_dispatch_mxfp8_tiled")


def moe_mx_quantize_weights(W, q, scale, stream=None):
    """W bf16 [E, K, N] -> q uint8 [E, N, K] (transposed E4M3 codes), scale uint8
    [E*N*K/32] (E8M0 codes of the blocks of 32 along K, tiled layout)."""
    E, K, N = W.shape
    _check(load().moe_mx_quantize_weights(_ptr(W, torch.bfloat16, "W"), E, K, N,
                                          _ptr(q, torch.uint8, "q"),
                                          _ptr(scale, torch.uint8, "scale"), _stream(stream)),
           "moe_mx_quantize_weights")


def moe_expert_ffn_mxfp8(xq, xs, W1q, W1s, W3q, W3s, W2q, W2s, offsets, counts, hq, hs, y,
                         dev_status, sh: Shape, stream=None):
    u8 = torch.uint8
    _check(load().moe_expert_ffn_mxfp8(
        _ptr(xq, u8, "xq"), _ptr(xs, u8, "xs"), _ptr(W1q, u8, "W1q"), _ptr(W1s, u8, "W1s"),
        _ptr(W3q, u8, "W3q"), _ptr(W3s, u8, "W3s"), _ptr(W2q, u8, "W2q"), _ptr(W2s, u8, "W2s"),
        _ptr(offsets, torch.int32, "offsets"), _ptr(counts, torch.int32, "counts"),
        _ptr(hq, u8, "hq"), _ptr(hs, u8, "hs"), _ptr(y, torch.float32, "y"),
        _ptr(dev_status, torch.int32, "dev_status"), ctypes.byref(sh), _stream(stream)),
        "moe_expert_ffn_mxfp8")


def moe_layer_forward_mxfp8(logits, x, W1q, W1s, W3q, W3s, W2q, W2s, out, ws, dev_status,
                            sh: Shape, stream=None, stage_events=None, shared=None):
    """shared: None, or the bf16 shared expert's (Ws1 [H, I], Ws3 [H, I], Ws2 [I, H])."""
    u8, bf = torch.uint8, torch.bfloat16
    Ws = shared if shared is not None else (None, None, None)
    _check(load().moe_layer_forward_mxfp8(
        _ptr(logits, torch.float32, "logits"), _ptr(x, bf, "x"),
        _ptr(W1q, u8, "W1q"), _ptr(W1s, u8, "W1s"), _ptr(W3q, u8, "W3q"), _ptr(W3s, u8, "W3s"),
        _ptr(W2q, u8, "W2q"), _ptr(W2s, u8, "W2s"), _ptr(Ws[0], bf, "Ws1"), _ptr(Ws[1], bf, "Ws3"),
        _ptr(Ws[2], bf, "Ws2"), _ptr(out, bf, "out"),
        _ptr(ws, u8, "ws"), ws.numel(), _ptr(dev_status, torch.int32, "dev_status"),
        ctypes.byref(sh), _stream(stream), _events(stage_events)), "moe_layer_forward_mxfp8")


def moe_selftest_bounded_wait(dev_status, timeout_ns: int, stream=None):
    _check(load().moe_selftest_bounded_wait(_ptr(dev_status, torch.int32, "dev_status"),
                                            int(timeout_ns), _stream(stream)),
           "moe_selftest_bounded_wait")


def moe_selftest_schedule_barrier(ids, phi, offsets, counts, route_row, ws, dev_status, sh: Shape,
                                  timeout_ns: int, stream=None):
    _check(load().moe_selftest_schedule_barrier(
        _ptr(ids, torch.int32, "ids"), _ptr(phi, torch.int32, "phi"),
        _ptr(offsets, torch.int32, "offsets"), _ptr(counts, torch.int32, "counts"),
        _ptr(route_row, torch.int32, "route_row"), _ptr(ws, torch.uint8, "ws"), ws.numel(),
        _ptr(dev_status, torch.int32, "dev_status"), ctypes.byref(sh), int(timeout_ns),
        _stream(stream)), "moe_selftest_schedule_barrier")


# ---------------------------------------------------------------- buffers
def alloc_schedule_outputs(sh: Shape, device="cuda"):
    """Device buffers of moe_schedule: phi, offsets, counts, route_row, ws, dev_status."""
    rm = rows_max(sh)
    return dict(
        phi=torch.empty((max(rm, 1), 2), dtype=torch.int32, device=device),
        offsets=torch.empty(sh.E + 1, dtype=torch.int32, device=device),
        counts=torch.empty((sh.E, sh.P), dtype=torch.int32, device=device),
        route_row=torch.empty((sh.P, sh.N, sh.k), dtype=torch.int32, device=device),
        ws=torch.empty(max(schedule_workspace_bytes(sh), 16), dtype=torch.uint8, device=device),
        dev_status=torch.zeros(1, dtype=torch.int32, device=device),
    )
