"""ctypes front end of the fp64 C oracle (``moe_oracle.c``).

TEST INFRASTRUCTURE ONLY -- see ``moe_oracle.c`` for what is computed and
which passages of the pages each step follows.  Inputs are numpy ``uint16``
arrays holding raw bf16 bits (the exact bits the GPU library receives);
outputs are float64 / int32 numpy arrays.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")
_lib = None

_P = ctypes.c_void_p
_I = ctypes.c_int


def build(force: bool = False) -> str:
    """Compile ``moe_oracle.c`` with gcc (OpenMP across tokens, no fast-math,
    no FMA contraction) into ``libmoe_oracle.so`` next to it."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(
            ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
             "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"],
            check=True,
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        # MOE_ORACLE_LIB points the tests' mutation check at a deliberately
        # broken copy of the oracle; normally the library is built from source.
        path = os.environ.get("MOE_ORACLE_LIB") or build()
        lib = ctypes.CDLL(path)
        lib.oracle_num_threads.restype = _I
        lib.oracle_route.restype = _I
        lib.oracle_route.argtypes = [_I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P]
        lib.oracle_route_v.restype = _I
        lib.oracle_route_v.argtypes = [_I, _I, _I, _I, _P, _P, _P, _I, _P, _P, _P, _P, _P]
        lib.oracle_forward_v.restype = _I
        lib.oracle_forward_v.argtypes = [_I, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P,
                                         _I, _P, _P, _P, _P, _I, _I, ctypes.c_longlong, _P, _P]
        lib.oracle_forward.restype = _I
        lib.oracle_forward.argtypes = [_I, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P,
                                       _I, _P, _P, _P, _P, _P]
        lib.oracle_e4m3_to_double.restype = ctypes.c_double
        lib.oracle_e4m3_to_double.argtypes = [_I]
        lib.oracle_forward_fp8.restype = _I
        lib.oracle_forward_fp8.argtypes = [_I, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P,
                                           _P, _P, _P, _P, _P]
        lib.oracle_swiglu.restype = _I
        lib.oracle_swiglu.argtypes = [_I, _I, _I, _P, _P, _P, _P, _P]
        lib.oracle_ep_plan.restype = _I
        lib.oracle_ep_plan.argtypes = [_I, _I, _I, _P, _P, _P, _P]
        _lib = lib
    return _lib


def _bits(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("oracle inputs are raw bf16 bits (numpy uint16)")
    return a


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_P)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


#: Gate-weight rules: the method's softmax over the k selected logits, the
#: softmax over all E logits without renormalisation ("Mixtral 8x7B模型架构解析"
#: Router.forward), the sigmoid of each selected logit ("万亿 MoE" forward
#: listing), and the entropy-controlled k of "Mixtral 8x7B模型架构解析"
#: (entropy_aware_routing: weights softmax(l / 0.1) over all experts, k kept
#: when its entropy exceeds 0.8 nats, k - 1 otherwise; unused slots hold
#: expert -1 and weight 0).
W_SOFTMAX_TOPK, W_SOFTMAX_ALL, W_SIGMOID, W_ENTROPY = 0, 1, 2, 3
#: The listing's temperature and entropy threshold.
ENTROPY_TAU, ENTROPY_THRESHOLD = 0.1, 0.8
#: Expert activations: SwiGLU silu(W1 x) * W3 x, and the "万亿 MoE" listing's
#: sigmoid gate sigmoid(W1 x) * W3 x.
ACT_SILU, ACT_SIGMOID = 0, 1


def capacity_limit(capacity_factor: float, T: int, k: int, E: int) -> int:
    """Per-expert capacity for a capacity factor: floor(cf * T * k / E), the
    factor times the mean number of (token, slot) pairs per expert (computed
    in double precision in exactly this order)."""
    return int(math.floor(float(capacity_factor) * float(T * k) / float(E)))


def route(x, Wg, k: int, bias=None, w_mode: int = W_SOFTMAX_TOPK):
    """Router of every token.  Returns dict with ``idx`` [T,k] int32, ``w``
    [T,k] f64, ``gap`` [T] f64 (k-th minus (k+1)-th logit, inf if k == E),
    ``logits`` [T,E] f64 and ``counts`` [E] int64.  ``w_mode`` picks the
    gate-weight rule (the selected set does not depend on it, except that
    W_ENTROPY may leave the last slot unused: expert -1, weight 0)."""
    x, Wg = _bits(x), _bits(Wg)
    T, d = x.shape
    E = Wg.shape[0]
    assert Wg.shape[1] == d
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float64)
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    gap = np.empty((T,), np.float64)
    logits = np.empty((T, E), np.float64)
    counts = np.empty((E,), np.int64)
    rc = _load().oracle_route_v(T, d, E, k, _ptr(x), _ptr(Wg), _ptr(b), int(w_mode), _ptr(idx),
                                _ptr(w), _ptr(gap), _ptr(logits), _ptr(counts))
    if rc != 0:
        raise ValueError("oracle_route rejected its arguments")
    return {"idx": idx, "w": w, "gap": gap, "logits": logits, "counts": counts}


def forward(x, Wg, W1, W3, W2, k: int, bias=None, tokens=None, shared=None, forced=None,
            w_mode: int = W_SOFTMAX_TOPK, act_mode: int = ACT_SILU, capacity=None,
            route_all=None):
    """Layer output (f64) for ``tokens`` (default: all).  ``shared`` is an
    optional (Ws1, Ws3, Ws2) triple of the always-on expert; ``forced`` an
    optional [n,k] int array of experts to use instead of the token's top-k.
    Variants: ``w_mode`` / ``act_mode`` (see the constants above);
    ``capacity`` (int, per-expert limit, None = dropless) keeps each expert's
    first ``capacity`` (token, slot) pairs in token order, ranked by the
    routing ``route_all`` [T,k] (default: the oracle's own)."""
    x, Wg, W1, W3, W2 = (_bits(a) for a in (x, Wg, W1, W3, W2))
    T, d = x.shape
    E, dff = W1.shape[0], W1.shape[1]
    assert Wg.shape == (E, d) and W1.shape == (E, dff, d) and W3.shape == (E, dff, d)
    assert W2.shape == (E, d, dff)
    tok = None
    if tokens is not None:
        tok = np.ascontiguousarray(tokens, dtype=np.int32)
        n = tok.shape[0]
    else:
        n = T
    dffs, Ws1, Ws3, Ws2 = 0, None, None, None
    if shared is not None:
        Ws1, Ws3, Ws2 = (_bits(a) for a in shared)
        dffs = Ws1.shape[0]
        assert Ws1.shape == (dffs, d) and Ws3.shape == (dffs, d) and Ws2.shape == (d, dffs)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float64)
    f = None if forced is None else np.ascontiguousarray(forced, dtype=np.int32)
    if f is not None:
        assert f.shape == (n, k)
    ra = None if route_all is None else np.ascontiguousarray(route_all, dtype=np.int32)
    if ra is not None:
        assert ra.shape == (T, k)
    cap = -1 if capacity is None else int(capacity)
    assert capacity is None or cap >= 0
    out = np.empty((n, d), np.float64)
    rc = _load().oracle_forward_v(n, _ptr(tok), T, d, E, dff, k, _ptr(x), _ptr(Wg), _ptr(b),
                                  _ptr(W1), _ptr(W3), _ptr(W2), dffs, _ptr(Ws1), _ptr(Ws3),
                                  _ptr(Ws2), _ptr(f), int(w_mode), int(act_mode), cap, _ptr(ra),
                                  _ptr(out))
    if rc != 0:
        raise ValueError("oracle_forward rejected its arguments")
    return out


def swiglu(x, W1, W3, W2):
    """One SwiGLU expert applied to every row of x (f64 result)."""
    x, W1, W3, W2 = (_bits(a) for a in (x, W1, W3, W2))
    n, d = x.shape
    dff = W1.shape[0]
    assert W1.shape == (dff, d) and W3.shape == (dff, d) and W2.shape == (d, dff)
    out = np.empty((n, d), np.float64)
    rc = _load().oracle_swiglu(n, d, dff, _ptr(x), _ptr(W1), _ptr(W3), _ptr(W2), _ptr(out))
    if rc != 0:
        raise ValueError("oracle_swiglu rejected its arguments")
    return out


def e4m3_to_double(code: int) -> float:
    """Value of one e4m3 code (OCP E4M3, no infinities)."""
    return float(_load().oracle_e4m3_to_double(int(code)))


def forward_fp8(x, Wg, q1, s1, q3, s3, q2, s2, k: int, bias=None, tokens=None, forced=None):
    """Layer output (f64) with FP8 experts: q1/q3 [E,dff,d] and q2 [E,d,dff]
    e4m3 codes (numpy uint8), s1/s3 [E,dff] and s2 [E,d] row scales; the
    router reads bf16 x and Wg as in ``forward``."""
    x, Wg = _bits(x), _bits(Wg)
    q1, q3, q2 = (np.ascontiguousarray(a, dtype=np.uint8) for a in (q1, q3, q2))
    s1, s3, s2 = (np.ascontiguousarray(a, dtype=np.float64) for a in (s1, s3, s2))
    T, d = x.shape
    E, dff = q1.shape[0], q1.shape[1]
    assert q1.shape == (E, dff, d) and q3.shape == (E, dff, d) and q2.shape == (E, d, dff)
    assert s1.shape == (E, dff) and s3.shape == (E, dff) and s2.shape == (E, d)
    assert Wg.shape == (E, d)
    tok = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int32)
    n = T if tok is None else tok.shape[0]
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float64)
    f = None if forced is None else np.ascontiguousarray(forced, dtype=np.int32)
    out = np.empty((n, d), np.float64)
    rc = _load().oracle_forward_fp8(n, _ptr(tok), T, d, E, dff, k, _ptr(x), _ptr(Wg), _ptr(b),
                                    _ptr(q1), _ptr(s1), _ptr(q3), _ptr(s3), _ptr(q2), _ptr(s2),
                                    _ptr(f), _ptr(out))
    if rc != 0:
        raise ValueError("oracle_forward_fp8 rejected its arguments")
    return out



def ep_plan(idx_per_rank, E: int, R: int):
    """Receive layout of the layer split over R ranks by experts (see
    ``oracle_ep_plan`` in moe_oracle.c for the order).  ``idx_per_rank[r]``:
    rank r's [T_r, k] expert indices.  Returns ``(pos, offsets)``: pos[r]
    [T_r, k] int32, the receive row of each pair in the owner of its expert;
    offsets[q] [E/R + 1] int32, owner q's segment starts."""
    assert R >= 1 and E % R == 0 and len(idx_per_rank) == R
    arrs = [np.ascontiguousarray(i, dtype=np.int32) for i in idx_per_rank]
    k = arrs[0].shape[1]
    assert all(a.ndim == 2 and a.shape[1] == k for a in arrs)
    T_of = np.array([a.shape[0] for a in arrs], np.int32)
    idx_all = np.ascontiguousarray(np.concatenate([a.ravel() for a in arrs]), dtype=np.int32)
    pos_all = np.empty_like(idx_all)
    offsets = np.empty((R, E // R + 1), np.int32)
    rc = _load().oracle_ep_plan(R, E, k, _ptr(T_of), _ptr(idx_all), _ptr(pos_all),
                                _ptr(offsets))
    if rc != 0:
        raise ValueError("oracle_ep_plan rejected its arguments")
    pos, start = [], 0
    for a in arrs:
        pos.append(pos_all[start:start + a.size].reshape(a.shape))
        start += a.size
    return pos, [offsets[q] for q in range(R)]
