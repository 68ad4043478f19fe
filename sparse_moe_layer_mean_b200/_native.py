"""ctypes binding of libmrlmoe.so (include/mrlmoe.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  Functions carry the C ABI's names and take torch tensors (device
memory) or raw integers; a non-zero status raises MrlmoeError.  There is no
fallback: if the library is missing, loading fails loudly.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_float, c_int, c_size_t, c_uint32, c_void_p
from typing import Dict, Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmrlmoe.so")

MRLMOE_BF16 = 0
MRLMOE_FP8_E4M3_BLOCK128 = 1
MRLMOE_FP4_E2M1_BLOCK128 = 2

STATUS = {0: "MRLMOE_OK", 1: "MRLMOE_ERR_INVALID_ARG", 2: "MRLMOE_ERR_UNSUPPORTED",
          3: "MRLMOE_ERR_WORKSPACE", 4: "MRLMOE_ERR_CUDA", 5: "MRLMOE_ERR_TIMEOUT",
          6: "MRLMOE_ERR_CHECK", 7: "MRLMOE_ERR_SCRATCH_LIMIT"}

EXPORTED = ("mrlmoe_workspace_size", "mrlmoe_route", "mrlmoe_forward", "mrlmoe_forward_timed",
            "mrlmoe_bias_update", "mrlmoe_linear", "mrlmoe_get_device_status",
            "mrlmoe_status_string", "mrlmoe_route_scores_static", "mrlmoe_quantize_e4m3",
            "mrlmoe_check_routing", "mrlmoe_get_device_detail", "mrlmoe_train_workspace_size",
            "mrlmoe_forward_train", "mrlmoe_backward", "mrlmoe_backward_timed",
            "mrlmoe_ep_workspace_size", "mrlmoe_ep_dispatch", "mrlmoe_ep_experts", "mrlmoe_ep_combine")
STATIC_SCRATCH_BYTES = 2 * 1024 * 1024
NUM_STAGE_EVENTS = 9
NUM_BACKWARD_EVENTS = 11
BACKWARD_STAGES = ("dn", "dw_up", "rms_combine_bwd", "dh_glu_bwd", "dz", "token_router_bwd",
                   "dw_router_alpha", "expert_wgrad", "dx", "dw_down")
STAGES = ("down_proj", "router_topk", "dispatch", "gather", "gate_up_glu", "expert_down",
          "combine_rmsnorm", "up_proj")


class MrlmoeError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)} ({status_string(code)})")


class Config(ctypes.Structure):
    _fields_ = [("T", c_int), ("d_model", c_int), ("d_lat", c_int), ("n_experts", c_int),
                ("top_k", c_int), ("d_ff", c_int), ("n_routers", c_int), ("rms_eps", c_float),
                ("dtype", c_int), ("aggregation", c_int), ("hold", c_uint32)]


# mrlmoe_hold: GEMM families whose tile loads a call may hold (test hook)
HOLD = {"gemm": 1, "gemm_pair": 2, "gemm_fp8": 4}

# mrlmoe_check_bits: invariants of a routing record
CHECK_BITS = {"index": 1, "duplicate": 2, "offsets": 4, "perm": 8, "group": 16, "order": 32, "weight": 64}


WEIGHT_FIELDS = ("w_down", "w_router", "w_gate", "w_up_e", "w_down_e", "w_sh_gate", "w_sh_up",
                 "w_sh_down", "rms_gain", "w_up", "expert_scale", "s_down", "s_gate", "s_up_e",
                 "s_down_e", "s_sh_gate", "s_sh_up", "s_sh_down", "s_up")


class Weights(ctypes.Structure):
    _fields_ = [(n, c_void_p) for n in WEIGHT_FIELDS]


ROUTING_FIELDS = ("topk_idx", "topk_w", "counts", "offsets", "perm", "inv_perm", "scores")


class Routing(ctypes.Structure):
    _fields_ = [(n, c_void_p) for n in ROUTING_FIELDS]


GRAD_FIELDS = ("dx", "d_w_down", "d_w_router", "d_w_gate", "d_w_up_e", "d_w_down_e", "d_w_sh_gate",
               "d_w_sh_up", "d_w_sh_down", "d_rms_gain", "d_w_up", "d_expert_scale")


class Grads(ctypes.Structure):
    _fields_ = [(n, c_void_p) for n in GRAD_FIELDS] + [("accumulate", c_int)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libmrlmoe.so (raises OSError when it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise OSError(f"{LIB_PATH} not found: build it with "
                          "`python -m sparse_moe_layer_mean_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        L.mrlmoe_workspace_size.argtypes = [POINTER(Config)]
        L.mrlmoe_workspace_size.restype = c_size_t
        L.mrlmoe_route.argtypes = [POINTER(Config), POINTER(Weights), c_void_p, c_void_p, c_int,
                                   POINTER(Routing), c_void_p, c_size_t, c_void_p]
        L.mrlmoe_route.restype = c_int
        L.mrlmoe_forward.argtypes = [POINTER(Config), POINTER(Weights), c_void_p, c_void_p, c_void_p,
                                     POINTER(Routing), c_void_p, c_size_t, c_void_p]
        L.mrlmoe_forward.restype = c_int
        L.mrlmoe_forward_timed.argtypes = [POINTER(Config), POINTER(Weights), c_void_p, c_void_p,
                                           c_void_p, POINTER(Routing), c_void_p, c_size_t, c_void_p,
                                           POINTER(c_void_p), c_int]
        L.mrlmoe_forward_timed.restype = c_int
        L.mrlmoe_bias_update.argtypes = [POINTER(Config), c_void_p, c_void_p, c_float, c_void_p]
        L.mrlmoe_bias_update.restype = c_int
        L.mrlmoe_linear.argtypes = [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_void_p]
        L.mrlmoe_linear.restype = c_int
        L.mrlmoe_route_scores_static.argtypes = [POINTER(Config), c_void_p, c_void_p, POINTER(Routing),
                                                 c_void_p]
        L.mrlmoe_route_scores_static.restype = c_int
        L.mrlmoe_quantize_e4m3.argtypes = [c_void_p, c_int, c_int, c_void_p, c_void_p, c_void_p]
        L.mrlmoe_quantize_e4m3.restype = c_int
        L.mrlmoe_get_device_status.argtypes = [c_void_p, c_void_p]
        L.mrlmoe_get_device_status.restype = c_int
        L.mrlmoe_get_device_detail.argtypes = [c_void_p, POINTER(c_uint32), c_void_p]
        L.mrlmoe_get_device_detail.restype = c_int
        L.mrlmoe_check_routing.argtypes = [POINTER(Config), POINTER(Routing), c_void_p, c_size_t, c_int,
                                           c_void_p]
        L.mrlmoe_check_routing.restype = c_int
        L.mrlmoe_train_workspace_size.argtypes = [POINTER(Config)]
        L.mrlmoe_train_workspace_size.restype = c_size_t
        L.mrlmoe_forward_train.argtypes = [POINTER(Config), POINTER(Weights), c_void_p, c_void_p, c_void_p,
                                           POINTER(Routing), c_void_p, c_size_t, c_void_p]
        L.mrlmoe_forward_train.restype = c_int
        L.mrlmoe_backward.argtypes = [POINTER(Config), POINTER(Weights), c_void_p, c_void_p, POINTER(Grads),
                                      c_void_p, c_size_t, c_void_p]
        L.mrlmoe_backward.restype = c_int
        L.mrlmoe_backward_timed.argtypes = [POINTER(Config), POINTER(Weights), c_void_p, c_void_p, POINTER(Grads),
                                            c_void_p, c_size_t, c_void_p, c_void_p, c_int]
        L.mrlmoe_backward_timed.restype = c_int
        L.mrlmoe_ep_workspace_size.argtypes = [POINTER(Config), c_int]
        L.mrlmoe_ep_workspace_size.restype = c_size_t
        L.mrlmoe_ep_dispatch.argtypes = [POINTER(Config), POINTER(Weights), c_void_p, c_void_p, c_int,
                                         POINTER(Routing), c_void_p, c_void_p, c_size_t, c_void_p]
        L.mrlmoe_ep_dispatch.restype = c_int
        L.mrlmoe_ep_experts.argtypes = [POINTER(Config), POINTER(Weights), c_int, c_void_p, c_void_p, c_int,
                                        c_void_p, c_void_p, c_size_t, c_void_p]
        L.mrlmoe_ep_experts.restype = c_int
        L.mrlmoe_ep_combine.argtypes = [POINTER(Config), POINTER(Weights), c_void_p, c_void_p, c_void_p, c_size_t,
                                        c_void_p]
        L.mrlmoe_ep_combine.restype = c_int
        L.mrlmoe_status_string.argtypes = [c_int]
        L.mrlmoe_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


# ----------------------------------------------------------------- marshalling
def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream_ptr(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


AGGREGATIONS = {"mean": 0, "sum": 1, "max": 2}   # mrlmoe_aggregation


def make_config(shape, T: Optional[int] = None, fp8: Optional[bool] = None, hold: int = 0) -> Config:
    """Config from a workloads.LayerShape-like object (duck-typed; a missing
    `aggregation` attribute means the mean).  ``hold``: mrlmoe_config.hold
    (0 in normal use; an OR of HOLD values makes those GEMMs' waits run out)."""
    f8 = shape.fp8 if fp8 is None else fp8
    f4 = bool(getattr(shape, "fp4", False))
    return Config(shape.T if T is None else T, shape.d_model, shape.d_lat, shape.n_experts,
                  shape.top_k, shape.d_ff, shape.n_routers, float(shape.rms_eps),
                  MRLMOE_FP4_E2M1_BLOCK128 if f4 else MRLMOE_FP8_E4M3_BLOCK128 if f8 else MRLMOE_BF16,
                  AGGREGATIONS[getattr(shape, "aggregation", "mean")], int(hold))


def make_weights(w: Dict[str, object]) -> Weights:
    return Weights(*[_ptr(w.get(n)) for n in WEIGHT_FIELDS])


def make_routing(r: Optional[Dict[str, object]]) -> Optional[Routing]:
    if r is None:
        return None
    return Routing(*[_ptr(r.get(n)) for n in ROUTING_FIELDS])


def _check(code: int, where: str):
    if code != 0:
        raise MrlmoeError(code, where)


# ---------------------------------------------------------- the C ABI by name
def status_string(code: int) -> str:
    return lib().mrlmoe_status_string(int(code)).decode()


def mrlmoe_workspace_size(cfg: Config) -> int:
    return int(lib().mrlmoe_workspace_size(ctypes.byref(cfg)))


def mrlmoe_route(cfg: Config, weights: Weights, bias, x, scores_in: bool, routing: Routing,
                 workspace, ws_bytes: int, stream=None) -> None:
    _check(lib().mrlmoe_route(ctypes.byref(cfg), ctypes.byref(weights), _ptr(bias), _ptr(x),
                              int(bool(scores_in)), ctypes.byref(routing), _ptr(workspace),
                              int(ws_bytes), _stream_ptr(stream)), "mrlmoe_route")


def mrlmoe_forward(cfg: Config, weights: Weights, bias, x, y, routing: Optional[Routing],
                   workspace, ws_bytes: int, stream=None) -> None:
    rp = ctypes.byref(routing) if routing is not None else None
    _check(lib().mrlmoe_forward(ctypes.byref(cfg), ctypes.byref(weights), _ptr(bias), _ptr(x),
                                _ptr(y), rp, _ptr(workspace), int(ws_bytes), _stream_ptr(stream)),
           "mrlmoe_forward")


def mrlmoe_forward_timed(cfg: Config, weights: Weights, bias, x, y, routing: Optional[Routing],
                         workspace, ws_bytes: int, events, stream=None) -> None:
    """``events``: NUM_STAGE_EVENTS torch.cuda.Event objects (created with
    enable_timing=True), recorded at the layer's stage boundaries."""
    arr = (c_void_p * NUM_STAGE_EVENTS)()
    for i, e in enumerate(events):
        arr[i] = e.cuda_event if hasattr(e, "cuda_event") else int(e)
    rp = ctypes.byref(routing) if routing is not None else None
    _check(lib().mrlmoe_forward_timed(ctypes.byref(cfg), ctypes.byref(weights), _ptr(bias), _ptr(x),
                                      _ptr(y), rp, _ptr(workspace), int(ws_bytes),
                                      _stream_ptr(stream), arr, len(events)),
           "mrlmoe_forward_timed")


def make_grads(g: Dict[str, object], accumulate: bool = False) -> Grads:
    return Grads(*[_ptr(g.get(n)) for n in GRAD_FIELDS], int(bool(accumulate)))


def mrlmoe_train_workspace_size(cfg: Config) -> int:
    return int(lib().mrlmoe_train_workspace_size(ctypes.byref(cfg)))


def mrlmoe_forward_train(cfg: Config, weights: Weights, bias, x, y, routing: Optional[Routing],
                         workspace, ws_bytes: int, stream=None) -> None:
    rp = ctypes.byref(routing) if routing is not None else None
    _check(lib().mrlmoe_forward_train(ctypes.byref(cfg), ctypes.byref(weights), _ptr(bias), _ptr(x),
                                      _ptr(y), rp, _ptr(workspace), int(ws_bytes), _stream_ptr(stream)),
           "mrlmoe_forward_train")


def mrlmoe_backward(cfg: Config, weights: Weights, x, dy, grads: Grads, workspace, ws_bytes: int,
                    stream=None) -> None:
    _check(lib().mrlmoe_backward(ctypes.byref(cfg), ctypes.byref(weights), _ptr(x), _ptr(dy),
                                 ctypes.byref(grads), _ptr(workspace), int(ws_bytes), _stream_ptr(stream)),
           "mrlmoe_backward")


def mrlmoe_backward_timed(cfg: Config, weights: Weights, x, dy, grads: Grads, workspace, ws_bytes: int,
                          events, stream=None) -> None:
    """``events``: NUM_BACKWARD_EVENTS timing events, recorded at the
    backward's stage boundaries (BACKWARD_STAGES lie between them)."""
    arr = (c_void_p * NUM_BACKWARD_EVENTS)()
    for i, e in enumerate(events):
        arr[i] = e.cuda_event if hasattr(e, "cuda_event") else int(e)
    _check(lib().mrlmoe_backward_timed(ctypes.byref(cfg), ctypes.byref(weights), _ptr(x), _ptr(dy),
                                       ctypes.byref(grads), _ptr(workspace), int(ws_bytes), _stream_ptr(stream),
                                       arr, len(events)),
           "mrlmoe_backward_timed")


def mrlmoe_bias_update(cfg: Config, counts, bias, gamma: float, stream=None) -> None:
    _check(lib().mrlmoe_bias_update(ctypes.byref(cfg), _ptr(counts), _ptr(bias), float(gamma),
                                    _stream_ptr(stream)), "mrlmoe_bias_update")


def mrlmoe_linear(a, w, out, M: int, N: int, K: int, stream=None) -> None:
    _check(lib().mrlmoe_linear(_ptr(a), _ptr(w), _ptr(out), int(M), int(N), int(K),
                               _stream_ptr(stream)), "mrlmoe_linear")


def mrlmoe_route_scores_static(cfg: Config, bias, expert_scale, routing: Routing, stream=None) -> None:
    """Routing from given scores with the library's static scratch (no workspace)."""
    _check(lib().mrlmoe_route_scores_static(ctypes.byref(cfg), _ptr(bias), _ptr(expert_scale),
                                            ctypes.byref(routing), _stream_ptr(stream)),
           "mrlmoe_route_scores_static")


def mrlmoe_quantize_e4m3(x, rows: int, K: int, q, scale, stream=None) -> None:
    _check(lib().mrlmoe_quantize_e4m3(_ptr(x), int(rows), int(K), _ptr(q), _ptr(scale), _stream_ptr(stream)),
           "mrlmoe_quantize_e4m3")


def mrlmoe_get_device_status(workspace, stream=None) -> int:
    return int(lib().mrlmoe_get_device_status(_ptr(workspace), _stream_ptr(stream)))


def mrlmoe_get_device_detail(workspace, stream=None):
    """(status, check_bits): the status word and the failed routing invariants."""
    bits = c_uint32(0)
    st = int(lib().mrlmoe_get_device_detail(_ptr(workspace), ctypes.byref(bits), _stream_ptr(stream)))
    return st, int(bits.value)


def mrlmoe_check_routing(cfg: Config, routing: Optional[Routing], workspace, ws_bytes: int, clear: bool,
                         stream=None) -> None:
    """Enqueue the device check of a routing record (read the verdict with
    mrlmoe_get_device_detail)."""
    rp = ctypes.byref(routing) if routing is not None else None
    _check(lib().mrlmoe_check_routing(ctypes.byref(cfg), rp, _ptr(workspace), int(ws_bytes), int(bool(clear)),
                                      _stream_ptr(stream)), "mrlmoe_check_routing")


# ------------------------------------------------------ expert parallelism
def mrlmoe_ep_workspace_size(cfg: Config, n_ranks: int) -> int:
    return int(lib().mrlmoe_ep_workspace_size(ctypes.byref(cfg), int(n_ranks)))


def mrlmoe_ep_dispatch(cfg: Config, weights: Weights, bias, x, n_ranks: int, routing: Routing, send_rows,
                       workspace, ws_bytes: int, stream=None) -> None:
    _check(lib().mrlmoe_ep_dispatch(ctypes.byref(cfg), ctypes.byref(weights), _ptr(bias), _ptr(x), int(n_ranks),
                                    ctypes.byref(routing), _ptr(send_rows), _ptr(workspace), int(ws_bytes),
                                    _stream_ptr(stream)), "mrlmoe_ep_dispatch")


def mrlmoe_ep_experts(cfg: Config, w_local: Weights, n_ranks: int, recv_rows, recv_counts, n_recv: int, out_rows,
                      workspace, ws_bytes: int, stream=None) -> None:
    _check(lib().mrlmoe_ep_experts(ctypes.byref(cfg), ctypes.byref(w_local), int(n_ranks), _ptr(recv_rows),
                                   _ptr(recv_counts), int(n_recv), _ptr(out_rows), _ptr(workspace), int(ws_bytes),
                                   _stream_ptr(stream)), "mrlmoe_ep_experts")


def mrlmoe_ep_combine(cfg: Config, weights: Weights, ret_rows, y, workspace, ws_bytes: int, stream=None) -> None:
    _check(lib().mrlmoe_ep_combine(ctypes.byref(cfg), ctypes.byref(weights), _ptr(ret_rows), _ptr(y),
                                   _ptr(workspace), int(ws_bytes), _stream_ptr(stream)), "mrlmoe_ep_combine")
