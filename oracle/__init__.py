"""ctypes binding of the fp64 C oracle (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product path never does.

``build()`` compiles ``oracle.c`` with gcc (OpenMP over jets, no fast-math,
no fp contraction, so the compensated sums stay exact). The functions below
take a ``synth.JetBatch`` and return float64 numpy arrays.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

H = 8
D = 16


def build(force: bool = False) -> str:
    """Compile the oracle shared library if it is missing or stale."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
               "-ffp-contract=off", "-o", _LIB_PATH + ".tmp", _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB_PATH + ".tmp", _LIB_PATH)
    return _LIB_PATH


class _Params(C.Structure):
    _fields_ = [(n, C.POINTER(C.c_float)) for n in (
        "a0", "c0", "W1", "b1", "a1", "c1", "W2", "b2", "a2", "c2",
        "W3", "b3", "a3", "c3", "W4", "b4")]


class _Jets(C.Structure):
    _fields_ = [("E", C.POINTER(C.c_float)), ("px", C.POINTER(C.c_float)),
                ("py", C.POINTER(C.c_float)), ("pz", C.POINTER(C.c_float)),
                ("mask", C.POINTER(C.c_uint8)), ("ptr", C.POINTER(C.c_int32)),
                ("N", C.c_int32), ("P", C.c_int32)]


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = C.CDLL(_LIB_PATH)
            dp = C.POINTER(C.c_double)
            u16 = C.POINTER(C.c_uint16)
            L.orc_pair_features.argtypes = [dp, dp, dp]
            L.orc_gelu.argtypes = [C.c_double]
            L.orc_gelu.restype = C.c_double
            L.orc_mlp_row.argtypes = [dp, C.POINTER(_Params), dp]
            L.orc_features.argtypes = [C.POINTER(_Jets), dp]
            L.orc_pair_bias.argtypes = [C.POINTER(_Jets), C.POINTER(_Params), dp]
            L.orc_attention.argtypes = [C.POINTER(_Jets), dp, u16, u16, u16, C.c_int, dp]
            L.orc_forward.argtypes = [C.POINTER(_Jets), C.POINTER(_Params), u16, u16, u16, C.c_int, dp]
            i8 = C.POINTER(C.c_int8)
            L.orc_quantize_act.argtypes = [dp, C.c_int, i8, dp, C.POINTER(C.c_int)]
            L.orc_quantize_weights.argtypes = [dp, C.c_int, C.c_int, i8, dp]
            L.orc_int8_linear.argtypes = [dp, C.c_int, dp, dp, C.c_int, dp]
            L.orc_mlp_row_i8.argtypes = [dp, C.POINTER(_Params), dp]
            L.orc_pair_bias_i8.argtypes = [C.POINTER(_Jets), C.POINTER(_Params), dp]
            L.orc_forward_i8.argtypes = [C.POINTER(_Jets), C.POINTER(_Params), u16, u16, u16, C.c_int, dp]
            L.orc_set_threads.argtypes = [C.c_int]
            L.orc_get_threads.restype = C.c_int
            _lib = L
        return _lib


def _ptr(a, ctype):
    return a.ctypes.data_as(C.POINTER(ctype)) if a is not None else None


def _params(p):
    arrs = {k: np.ascontiguousarray(v, dtype=np.float32) for k, v in p.items()}
    st = _Params(**{name: _ptr(arrs[name], C.c_float) for name, _t in _Params._fields_})
    return st, arrs          # keep the arrays alive with the struct


def _jets(b):
    arrs = dict(E=np.ascontiguousarray(b.E, np.float32), px=np.ascontiguousarray(b.px, np.float32),
                py=np.ascontiguousarray(b.py, np.float32), pz=np.ascontiguousarray(b.pz, np.float32),
                mask=None if b.mask is None else np.ascontiguousarray(b.mask, np.uint8),
                ptr=None if b.ptr is None else np.ascontiguousarray(b.ptr, np.int32))
    st = _Jets(_ptr(arrs["E"], C.c_float), _ptr(arrs["px"], C.c_float), _ptr(arrs["py"], C.c_float),
               _ptr(arrs["pz"], C.c_float), _ptr(arrs["mask"], C.c_uint8), _ptr(arrs["ptr"], C.c_int32),
               int(b.N), int(b.P))
    return st, arrs


def set_threads(n: int) -> None:
    lib().orc_set_threads(int(n))


def threads() -> int:
    return int(lib().orc_get_threads())


def pair_features(a, b) -> np.ndarray:
    """Features (ln kT, ln z, ln dR, ln m^2) of two (E, px, py, pz) vectors."""
    a = np.ascontiguousarray(a, np.float64)
    b = np.ascontiguousarray(b, np.float64)
    out = np.zeros(4)
    lib().orc_pair_features(_ptr(a, C.c_double), _ptr(b, C.c_double), _ptr(out, C.c_double))
    return out


def gelu(x: float) -> float:
    return float(lib().orc_gelu(float(x)))


def mlp_row(f, params) -> np.ndarray:
    f = np.ascontiguousarray(f, np.float64)
    st, _keep = _params(params)
    out = np.zeros(8)
    lib().orc_mlp_row(_ptr(f, C.c_double), C.byref(st), _ptr(out, C.c_double))
    return out


def quantize_act(x):
    """Zero-point int8 quantisation of one input row: (codes int8, s, z)."""
    x = np.ascontiguousarray(x, np.float64)
    q = np.zeros(x.shape[0], np.int8)
    s = C.c_double()
    z = C.c_int()
    lib().orc_quantize_act(_ptr(x, C.c_double), int(x.shape[0]), _ptr(q, C.c_int8), C.byref(s), C.byref(z))
    return q, s.value, z.value


def quantize_weights(W):
    """Per-row symmetric int8 weight codes of W [rows, cols]: (codes, alpha)."""
    W = np.ascontiguousarray(W, np.float64)
    T = np.zeros(W.shape, np.int8)
    alpha = np.zeros(W.shape[0])
    lib().orc_quantize_weights(_ptr(W, C.c_double), int(W.shape[0]), int(W.shape[1]), _ptr(T, C.c_int8),
                               _ptr(alpha, C.c_double))
    return T, alpha


def int8_linear(x, W, b) -> np.ndarray:
    """y = W x + b with x and W quantised to int8 (the int8 variant's layer)."""
    x = np.ascontiguousarray(x, np.float64)
    W = np.ascontiguousarray(W, np.float64)
    b = np.ascontiguousarray(b, np.float64)
    y = np.zeros(W.shape[0])
    lib().orc_int8_linear(_ptr(x, C.c_double), int(x.shape[0]), _ptr(W, C.c_double), _ptr(b, C.c_double),
                          int(W.shape[0]), _ptr(y, C.c_double))
    return y


def mlp_row_i8(f, params) -> np.ndarray:
    f = np.ascontiguousarray(f, np.float64)
    st, _keep = _params(params)
    out = np.zeros(8)
    lib().orc_mlp_row_i8(_ptr(f, C.c_double), C.byref(st), _ptr(out, C.c_double))
    return out


def pair_bias_i8(b, params=None) -> np.ndarray:
    """U [N, 8, P, P] float64 of the MLP with int8 hidden-layer inputs."""
    js, _k = _jets(b)
    ps, _kp = _params(params if params is not None else b.params)
    out = np.zeros((b.N, H, b.P, b.P))
    if lib().orc_pair_bias_i8(C.byref(js), C.byref(ps), _ptr(out, C.c_double)) != 0:
        raise ValueError("oracle: invalid jet description")
    return out


def forward_i8(b, params=None) -> np.ndarray:
    """The block with the int8 MLP variant; output in the layout of q."""
    js, _k = _jets(b)
    ps, _kp = _params(params if params is not None else b.params)
    q = np.ascontiguousarray(b.q, np.uint16)
    k = np.ascontiguousarray(b.k, np.uint16)
    v = np.ascontiguousarray(b.v, np.uint16)
    out = np.zeros(q.shape)
    if lib().orc_forward_i8(C.byref(js), C.byref(ps), _ptr(q, C.c_uint16), _ptr(k, C.c_uint16),
                            _ptr(v, C.c_uint16), D, _ptr(out, C.c_double)) != 0:
        raise ValueError("oracle: invalid jet description")
    return out


def features(b) -> np.ndarray:
    """feat [N, P, P, 4] float64."""
    js, _k = _jets(b)
    out = np.zeros((b.N, b.P, b.P, 4))
    if lib().orc_features(C.byref(js), _ptr(out, C.c_double)) != 0:
        raise ValueError("oracle: invalid jet description")
    return out


def pair_bias(b, params=None) -> np.ndarray:
    """U [N, 8, P, P] float64."""
    js, _k = _jets(b)
    ps, _kp = _params(params if params is not None else b.params)
    out = np.zeros((b.N, H, b.P, b.P))
    if lib().orc_pair_bias(C.byref(js), C.byref(ps), _ptr(out, C.c_double)) != 0:
        raise ValueError("oracle: invalid jet description")
    return out


def attention(b, U, q=None, k=None, v=None) -> np.ndarray:
    """Attention output (layout of q) float64 for a given padded bias U."""
    js, _k = _jets(b)
    q = np.ascontiguousarray(b.q if q is None else q, np.uint16)
    k = np.ascontiguousarray(b.k if k is None else k, np.uint16)
    v = np.ascontiguousarray(b.v if v is None else v, np.uint16)
    U = np.ascontiguousarray(U, np.float64)
    out = np.zeros(q.shape)
    if lib().orc_attention(C.byref(js), _ptr(U, C.c_double), _ptr(q, C.c_uint16), _ptr(k, C.c_uint16),
                           _ptr(v, C.c_uint16), D, _ptr(out, C.c_double)) != 0:
        raise ValueError("oracle: invalid jet description")
    return out


def forward(b, params=None) -> np.ndarray:
    """The whole block (features -> MLP -> attention); output in the layout of q."""
    js, _k = _jets(b)
    ps, _kp = _params(params if params is not None else b.params)
    q = np.ascontiguousarray(b.q, np.uint16)
    k = np.ascontiguousarray(b.k, np.uint16)
    v = np.ascontiguousarray(b.v, np.uint16)
    out = np.zeros(q.shape)
    if lib().orc_forward(C.byref(js), C.byref(ps), _ptr(q, C.c_uint16), _ptr(k, C.c_uint16),
                         _ptr(v, C.c_uint16), D, _ptr(out, C.c_double)) != 0:
        raise ValueError("oracle: invalid jet description")
    return out


def _bf16_bits_to_f64(bits) -> np.ndarray:
    """Exact widening of raw bf16 bit patterns."""
    b = np.ascontiguousarray(bits, np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def block_forward(b, bi, params=None) -> np.ndarray:
    """Multi-head attention with the pair bias and the projections either side
    of it, in fp64 (the attention of page 1 "Fusion 3" inside a ParT block of
    embedding 128 = 8 heads x 16): for each jet's valid particles X,
    q, k, v = X Wqkv^T + bqkv split into 8 heads of 16, o_h = softmax(q_h k_h^T
    / sqrt(16) + U_h) v_h over the jet's valid keys, y = concat_h(o_h) Wo^T +
    bo. Rows of masked slots are 0. `bi` is a ``synth.BlockInputs``; the
    result is float64 [rows, 128] in the layout of bi.x."""
    U = pair_bias(b, params)
    x = _bf16_bits_to_f64(bi.x)
    Wqkv = _bf16_bits_to_f64(bi.Wqkv)
    Wo = _bf16_bits_to_f64(bi.Wo)
    bqkv = np.asarray(bi.bqkv, np.float64)
    bo = np.asarray(bi.bo, np.float64)
    y = np.zeros_like(x)
    for n in range(b.N):
        if b.layout == "padded":
            slots = np.flatnonzero(b.mask[n * b.P:(n + 1) * b.P])
            rows = n * b.P + slots
            local = slots
        else:
            rows = np.arange(int(b.ptr[n]), int(b.ptr[n + 1]))
            local = np.arange(len(rows))
        m = len(rows)
        if m == 0:
            continue
        qkv = x[rows] @ Wqkv.T + bqkv
        o = np.zeros((m, H * D))
        for h in range(H):
            q = qkv[:, h * D:(h + 1) * D]
            k = qkv[:, H * D + h * D:H * D + (h + 1) * D]
            v = qkv[:, 2 * H * D + h * D:2 * H * D + (h + 1) * D]
            s = q @ k.T / np.sqrt(D) + U[n, h][np.ix_(local, local)]
            s = s - s.max(axis=1, keepdims=True)
            p = np.exp(s)
            o[:, h * D:(h + 1) * D] = (p / p.sum(axis=1, keepdims=True)) @ v
        y[rows] = o @ Wo.T + bo
    return y
