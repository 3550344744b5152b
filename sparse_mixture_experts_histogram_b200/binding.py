"""Python binding of the C ABI in ``include/moe.h`` (ctypes).

Argument marshalling only: every function has the same name and argument
order as its C counterpart, takes torch tensors (or raw device addresses as
ints) and turns a non-zero status into ``MoEError``.  All work runs in the
CUDA library ``libmoe_b200.so``; there is no other implementation to fall
back to, so a missing library is an error.
"""
from __future__ import annotations

import ctypes
import os
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmoe_b200.so")

MOE_OK = 0
STATUS_NAMES = {
    0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE",
    4: "MOE_ERR_CUDA", 5: "MOE_ERR_DEVICE", 6: "MOE_ERR_TIMEOUT",
}
DEVERR_BITS = {0x1: "TIMEOUT_TMA", 0x2: "TIMEOUT_MMA", 0x4: "TIMEOUT_EPI", 0x8: "OFFSETS",
               0x10: "INDEX", 0x20: "LAYOUT", 0x40: "EP_COUNTS"}
#: Bytes of an inter-process memory handle (MOE_IPC_HANDLE_BYTES).
IPC_HANDLE_BYTES = 64

#: Every symbol the C header declares (checked against ``include/moe.h`` by the tests).
ABI_FUNCTIONS = ("moe_workspace_size", "moe_workspace_size_ex", "moe_route", "moe_permute",
                 "moe_expert_ffn", "moe_combine", "moe_forward", "moe_forward_ex",
                 "moe_forward_traced", "moe_get_device_error", "moe_status_string",
                 "moe_expert_ffn_static", "moe_expert_ffn_static_bytes",
                 "moe_expert_ffn_static_error", "moe_forward_variant", "moe_route_variant",
                 "moe_forward_fp8", "moe_forward_fp8_traced", "moe_ep_recv_rows",
                 "moe_ep_workspace_size", "moe_ep_ffn_splits", "moe_ep_output_bf16",
                 "moe_ep_dispatch",
                 "moe_ep_expert_ffn", "moe_ep_combine", "moe_ipc_get_handle",
                 "moe_ipc_open_handle", "moe_ipc_close", "moe_selftest_wait_timeout")
TRACE_EVENTS = 6
#: What each of moe_forward_traced's events marks (event i = start of stage i).
TRACE_STAGES = ("route", "scatter", "expert_ffn", "shared_ffn", "combine")


#: Gate-weight rules and expert activations of ``moe_variant`` (include/moe.h).
WEIGHTS_SOFTMAX_TOPK, WEIGHTS_SOFTMAX_ALL, WEIGHTS_SIGMOID, WEIGHTS_ENTROPY = 0, 1, 2, 3
ACT_SILU, ACT_SIGMOID = 0, 1


class MoEVariant(ctypes.Structure):
    """``moe_variant``: gate-weight rule, expert activation, capacity factor."""
    _fields_ = [("weights", ctypes.c_int), ("activation", ctypes.c_int),
                ("capacity_factor", ctypes.c_double)]


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


_lib = None
_lock = threading.Lock()

_I, _P, _SZ = ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t


def load_library(path: str | None = None) -> ctypes.CDLL:
    """Load ``libmoe_b200.so`` (built in-tree by ``build.py``)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise RuntimeError(
                f"{p} is missing: build it with `python -m sparse_mixture_experts_histogram_b200"
                ".build` (the layer has no implementation other than this CUDA library)")
        lib = ctypes.CDLL(p)
        sig = {
            "moe_workspace_size": (_SZ, [_I] * 5),
            "moe_workspace_size_ex": (_SZ, [_I] * 6),
            "moe_route": (_I, [_I] * 4 + [_P] * 6 + [_P, _SZ, _P]),
            "moe_permute": (_I, [_I] * 4 + [_P] * 6 + [_SZ, _P]),
            "moe_expert_ffn": (_I, [_I] * 4 + [_P] * 7 + [_SZ, _P]),
            "moe_combine": (_I, [_I] * 3 + [_P] * 5 + [_P]),
            "moe_forward": (_I, [_I] * 5 + [_P] * 7 + [_SZ, _P]),
            "moe_forward_ex": (_I, [_I] * 5 + [_P] * 6 + [_I] + [_P] * 5 + [_SZ, _P]),
            "moe_forward_traced": (_I, [_I] * 5 + [_P] * 6 + [_I] + [_P] * 5 + [_SZ, _P, _P, _I]),
            "moe_forward_variant": (_I, [_I] * 5 + [_P] * 6 + [_I] + [_P] * 3 + [_P, _P, _P, _SZ,
                                                                               _P]),
            "moe_route_variant": (_I, [_I] * 4 + [_P] * 3 + [_I] + [_P] * 4 + [_SZ, _P]),
            "moe_forward_fp8": (_I, [_I] * 5 + [_P] * 11 + [_SZ, _P]),
            "moe_forward_fp8_traced": (_I, [_I] * 5 + [_P] * 11 + [_SZ, _P, _P, _I]),
            "moe_get_device_error": (_I, [_P, _P, _P]),
            "moe_expert_ffn_static": (_I, [_I] * 4 + [_P] * 6 + [_P]),
            "moe_expert_ffn_static_bytes": (_SZ, [_I] * 3),
            "moe_expert_ffn_static_error": (_I, [_P, _P]),
            "moe_status_string": (ctypes.c_char_p, [_I]),
            "moe_ep_recv_rows": (_I, [_I] * 4),
            "moe_ep_workspace_size": (_SZ, [_I] * 6),
            "moe_ep_ffn_splits": (_I, [_I] * 4),
            "moe_ep_dispatch": (_I, [_I] * 6 + [_P] * 4 + [_I] + [_P] * 3 + [_SZ, _P]),
            "moe_ep_output_bf16": (_I, [_I] * 4),
            "moe_ep_expert_ffn": (_I, [_I] * 9 + [_P] * 7 + [_SZ, _P]),
            "moe_ep_combine": (_I, [_I] * 8 + [_P] * 6 + [_P]),
            "moe_ipc_get_handle": (_I, [_P, _P, _P]),
            "moe_ipc_open_handle": (_I, [_P, _P]),
            "moe_ipc_close": (_I, [_P]),
            "moe_selftest_wait_timeout": (_I, [_P, _SZ, _P]),
        }
        for name, (res, args) in sig.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _lib = lib
        return lib


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str) -> None:
    if status != MOE_OK:
        raise MoEError(status, where)


def status_string(status: int) -> str:
    try:
        return load_library().moe_status_string(status).decode()
    except RuntimeError:
        return STATUS_NAMES.get(status, f"status {status}")


moe_status_string = status_string


def moe_workspace_size(T, d, E, d_ff, k) -> int:
    return int(load_library().moe_workspace_size(T, d, E, d_ff, k))


def moe_workspace_size_ex(T, d, E, d_ff, k, d_ff_shared) -> int:
    return int(load_library().moe_workspace_size_ex(T, d, E, d_ff, k, d_ff_shared))


def _ws_bytes(ws) -> int:
    if isinstance(ws, int):
        raise TypeError("pass the workspace as a tensor so its size is known")
    return ws.numel() * ws.element_size()


def moe_route(T, d, E, k, x, Wg, router_bias, idx, w, counts, ws, stream=None):
    _check(load_library().moe_route(T, d, E, k, _ptr(x), _ptr(Wg), _ptr(router_bias), _ptr(idx),
                                    _ptr(w), _ptr(counts), _ptr(ws), _ws_bytes(ws),
                                    _stream(stream)), "moe_route")


def moe_permute(T, d, E, k, x, idx, offsets, row_of_slot, x_perm, ws, stream=None):
    _check(load_library().moe_permute(T, d, E, k, _ptr(x), _ptr(idx), _ptr(offsets),
                                      _ptr(row_of_slot), _ptr(x_perm), _ptr(ws), _ws_bytes(ws),
                                      _stream(stream)), "moe_permute")


def moe_expert_ffn(S, d, E, d_ff, x_perm, offsets, W1, W3, W2, y_perm, ws, stream=None):
    _check(load_library().moe_expert_ffn(S, d, E, d_ff, _ptr(x_perm), _ptr(offsets), _ptr(W1),
                                         _ptr(W3), _ptr(W2), _ptr(y_perm), _ptr(ws),
                                         _ws_bytes(ws), _stream(stream)), "moe_expert_ffn")


def moe_expert_ffn_static(S, d, E, d_ff, x_perm, offsets, W1, W3, W2, y_perm, stream=None):
    """moe_expert_ffn without a workspace argument, for callers that cannot
    allocate device memory: the intermediate lives in a fixed 32 MiB array
    inside the library (see include/moe.h for its limit and sharing rules;
    moe_expert_ffn_static_bytes gives a call's need)."""
    _check(load_library().moe_expert_ffn_static(S, d, E, d_ff, _ptr(x_perm), _ptr(offsets),
                                                _ptr(W1), _ptr(W3), _ptr(W2), _ptr(y_perm),
                                                _stream(stream)), "moe_expert_ffn_static")


def moe_expert_ffn_static_bytes(S, E, d_ff) -> int:
    """Bytes of the fixed array a moe_expert_ffn_static call needs (0: unsupported)."""
    return int(load_library().moe_expert_ffn_static_bytes(S, E, d_ff))


def moe_expert_ffn_static_error(stream=None) -> tuple[int, int]:
    """(status, error word) the last moe_expert_ffn_static call on the current
    device left in the fixed array."""
    code = ctypes.c_uint32(0)
    st = load_library().moe_expert_ffn_static_error(ctypes.byref(code), _stream(stream))
    return int(st), int(code.value)


def moe_combine(T, d, k, y_perm, row_of_slot, w, shared_y, out, stream=None):
    _check(load_library().moe_combine(T, d, k, _ptr(y_perm), _ptr(row_of_slot), _ptr(w),
                                      _ptr(shared_y), _ptr(out), _stream(stream)), "moe_combine")


def moe_forward(T, d, E, d_ff, k, x, Wg, W1, W3, W2, out, ws, stream=None):
    _check(load_library().moe_forward(T, d, E, d_ff, k, _ptr(x), _ptr(Wg), _ptr(W1), _ptr(W3),
                                      _ptr(W2), _ptr(out), _ptr(ws), _ws_bytes(ws),
                                      _stream(stream)), "moe_forward")


def moe_forward_ex(T, d, E, d_ff, k, x, Wg, router_bias, W1, W3, W2, d_ff_shared, Ws1, Ws3, Ws2,
                   out, ws, stream=None):
    _check(load_library().moe_forward_ex(T, d, E, d_ff, k, _ptr(x), _ptr(Wg), _ptr(router_bias),
                                         _ptr(W1), _ptr(W3), _ptr(W2), d_ff_shared, _ptr(Ws1),
                                         _ptr(Ws3), _ptr(Ws2), _ptr(out), _ptr(ws),
                                         _ws_bytes(ws), _stream(stream)), "moe_forward_ex")


def moe_forward_variant(T, d, E, d_ff, k, x, Wg, router_bias, W1, W3, W2, d_ff_shared, Ws1, Ws3,
                        Ws2, variant, out, ws, stream=None):
    """``variant``: a MoEVariant, a (weights, activation, capacity_factor)
    tuple, or None for the method."""
    if variant is not None and not isinstance(variant, MoEVariant):
        variant = MoEVariant(*variant)
    vp = None if variant is None else ctypes.cast(ctypes.pointer(variant), ctypes.c_void_p)
    _check(load_library().moe_forward_variant(T, d, E, d_ff, k, _ptr(x), _ptr(Wg),
                                              _ptr(router_bias), _ptr(W1), _ptr(W3), _ptr(W2),
                                              d_ff_shared, _ptr(Ws1), _ptr(Ws3), _ptr(Ws2), vp,
                                              _ptr(out), _ptr(ws), _ws_bytes(ws),
                                              _stream(stream)), "moe_forward_variant")


def moe_route_variant(T, d, E, k, x, Wg, router_bias, weights, idx, w, counts, ws, stream=None):
    _check(load_library().moe_route_variant(T, d, E, k, _ptr(x), _ptr(Wg), _ptr(router_bias),
                                            int(weights), _ptr(idx), _ptr(w), _ptr(counts),
                                            _ptr(ws), _ws_bytes(ws), _stream(stream)),
           "moe_route_variant")


def moe_forward_fp8(T, d, E, d_ff, k, x, Wg, router_bias, W1q, s1, W3q, s3, W2q, s2, out, ws,
                    stream=None):
    """FP8 experts: W*q uint8 e4m3 codes, s* fp32 row scales (include/moe.h)."""
    _check(load_library().moe_forward_fp8(T, d, E, d_ff, k, _ptr(x), _ptr(Wg), _ptr(router_bias),
                                          _ptr(W1q), _ptr(s1), _ptr(W3q), _ptr(s3), _ptr(W2q),
                                          _ptr(s2), _ptr(out), _ptr(ws), _ws_bytes(ws),
                                          _stream(stream)), "moe_forward_fp8")


def moe_forward_fp8_traced(T, d, E, d_ff, k, x, Wg, router_bias, W1q, s1, W3q, s3, W2q, s2, out,
                           ws, events, stream=None):
    if len(events) != TRACE_EVENTS:
        raise ValueError(f"need {TRACE_EVENTS} events")
    arr = (ctypes.c_void_p * TRACE_EVENTS)(
        *[e if isinstance(e, int) else e.cuda_event for e in events])
    _check(load_library().moe_forward_fp8_traced(T, d, E, d_ff, k, _ptr(x), _ptr(Wg),
                                                 _ptr(router_bias), _ptr(W1q), _ptr(s1),
                                                 _ptr(W3q), _ptr(s3), _ptr(W2q), _ptr(s2),
                                                 _ptr(out), _ptr(ws), _ws_bytes(ws),
                                                 _stream(stream), arr, TRACE_EVENTS),
           "moe_forward_fp8_traced")


def moe_forward_traced(T, d, E, d_ff, k, x, Wg, router_bias, W1, W3, W2, d_ff_shared, Ws1, Ws3,
                       Ws2, out, ws, events, stream=None):
    """``events``: TRACE_EVENTS torch.cuda.Event(enable_timing=True) objects
    (or raw cudaEvent_t handles as ints)."""
    if len(events) != TRACE_EVENTS:
        raise ValueError(f"need {TRACE_EVENTS} events")
    arr = (ctypes.c_void_p * TRACE_EVENTS)(
        *[e if isinstance(e, int) else e.cuda_event for e in events])
    _check(load_library().moe_forward_traced(T, d, E, d_ff, k, _ptr(x), _ptr(Wg),
                                             _ptr(router_bias), _ptr(W1), _ptr(W3), _ptr(W2),
                                             d_ff_shared, _ptr(Ws1), _ptr(Ws3), _ptr(Ws2),
                                             _ptr(out), _ptr(ws), _ws_bytes(ws),
                                             _stream(stream), arr, TRACE_EVENTS),
           "moe_forward_traced")


def moe_get_device_error(ws, stream=None) -> tuple[int, int]:
    """(status, error word) of the last call that used workspace ``ws``."""
    code = ctypes.c_uint32(0)
    st = load_library().moe_get_device_error(_ptr(ws), ctypes.byref(code), _stream(stream))
    return int(st), int(code.value)


# ------------------------------------------------------- expert parallelism

def _ptr_array(ptrs):
    return (ctypes.c_void_p * len(ptrs))(*[_ptr(p) for p in ptrs])


def moe_ep_recv_rows(T_max, E, k, R) -> int:
    return int(load_library().moe_ep_recv_rows(T_max, E, k, R))


def moe_ep_workspace_size(T_max, d, E, d_ff, k, R) -> int:
    return int(load_library().moe_ep_workspace_size(T_max, d, E, d_ff, k, R))


def moe_ep_ffn_splits(rows_hint, d, E_local, d_ff) -> int:
    return int(load_library().moe_ep_ffn_splits(rows_hint, d, E_local, d_ff))


def moe_ep_dispatch(T, d, E, k, R, rank, x, idx, counts_all, recv_x, recv_rows, pos_of_slot,
                    recv_offsets, ws, stream=None):
    """``recv_x``: the R ranks' receive buffers (tensors or device addresses
    as this GPU sees them), in rank order."""
    if len(recv_x) != R:
        raise ValueError(f"need {R} receive buffers")
    _check(load_library().moe_ep_dispatch(T, d, E, k, R, rank, _ptr(x), _ptr(idx),
                                          _ptr(counts_all), _ptr_array(recv_x), recv_rows,
                                          _ptr(pos_of_slot), _ptr(recv_offsets), _ptr(ws),
                                          _ws_bytes(ws), _stream(stream)), "moe_ep_dispatch")


def moe_ep_output_bf16(rows_hint, d, E_local, d_ff) -> int:
    return int(load_library().moe_ep_output_bf16(rows_hint, d, E_local, d_ff))


def moe_ep_expert_ffn(T_max, d, E, d_ff, k, R, rows_hint, ksplit, y_bf16, recv_x, recv_offsets,
                      W1, W3, W2, recv_y, ws, stream=None):
    _check(load_library().moe_ep_expert_ffn(T_max, d, E, d_ff, k, R, rows_hint, ksplit,
                                            int(y_bf16), _ptr(recv_x), _ptr(recv_offsets),
                                            _ptr(W1), _ptr(W3), _ptr(W2), _ptr(recv_y), _ptr(ws),
                                            _ws_bytes(ws), _stream(stream)), "moe_ep_expert_ffn")


def moe_ep_combine(T, d, E, k, R, recv_rows, ksplit, y_bf16, idx, pos_of_slot, w, recv_y,
                   shared_y, out, stream=None):
    """``recv_y``: the R ranks' output buffers, in rank order."""
    if len(recv_y) != R:
        raise ValueError(f"need {R} output buffers")
    _check(load_library().moe_ep_combine(T, d, E, k, R, recv_rows, ksplit, int(y_bf16),
                                         _ptr(idx), _ptr(pos_of_slot), _ptr(w),
                                         _ptr_array(recv_y), _ptr(shared_y), _ptr(out),
                                         _stream(stream)), "moe_ep_combine")


def moe_ipc_get_handle(dev_ptr) -> tuple[bytes, int]:
    """(handle bytes, offset of dev_ptr in its allocation)."""
    h = ctypes.create_string_buffer(IPC_HANDLE_BYTES)
    off = ctypes.c_size_t(0)
    _check(load_library().moe_ipc_get_handle(_ptr(dev_ptr), h, ctypes.byref(off)),
           "moe_ipc_get_handle")
    return h.raw, int(off.value)


def moe_ipc_open_handle(handle: bytes) -> int:
    """Base address of another process's allocation, mapped here."""
    if len(handle) != IPC_HANDLE_BYTES:
        raise ValueError(f"an IPC handle has {IPC_HANDLE_BYTES} bytes")
    h = ctypes.create_string_buffer(bytes(handle), IPC_HANDLE_BYTES)
    base = ctypes.c_void_p(0)
    _check(load_library().moe_ipc_open_handle(h, ctypes.byref(base)), "moe_ipc_open_handle")
    return int(base.value)


def moe_ipc_close(base: int) -> None:
    _check(load_library().moe_ipc_close(base), "moe_ipc_close")


def moe_selftest_wait_timeout(ws, stream=None):
    """Runs a bounded wait that nothing completes (about 2 s); read the
    result with moe_get_device_error(ws)."""
    _check(load_library().moe_selftest_wait_timeout(_ptr(ws), _ws_bytes(ws), _stream(stream)),
           "moe_selftest_wait_timeout")
