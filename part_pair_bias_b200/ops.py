"""Thin Python binding of the C-ABI library ``libpairbias.so``.

Argument marshalling only: every step of the path runs in the library's CUDA
kernels. PyTorch provides device memory and streams. The library is loaded
on first use and its absence is an error -- there is no fallback.

Entry points mirror ``include/pairbias.h``: ``pairfeat_compute``,
``pairbias_mlp_forward``, ``pair_attention_forward``,
``pair_attention_forward_noalloc``, ``pair_block_forward``,
``pair_attention_backward``, the int8 variants ``pairbias_mlp_forward_i8``
and ``pair_attention_forward_i8``, ``get_device_status`` and the host
helpers ``fold_affine``, ``unfold_grad`` and ``quantize_mlp_i8``.
"""
from __future__ import annotations

import ctypes as C
import os
import threading
from dataclasses import dataclass
from typing import Dict, Optional

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpairbias.so")

PB_OK, PB_EINVAL, PB_EUNSUPPORTED, PB_ECUDA, PB_EDEVICE = range(5)
PB_BF16, PB_F32 = 0, 1
PB_DEV_TIMEOUT, PB_DEV_BADPTR = 1, 2
PB_STATIC_SCRATCH_BYTES = 32 << 20
H, D = 8, 16

# offsets of the folded parameters in the flat buffer (PB_OFF_* in the header)
FOLDED_OFFSETS = dict(W1=(0, (64, 4)), b1=(256, (64,)), W2=(320, (64, 64)), b2=(4416, (64,)),
                      W3=(4480, (64, 64)), b3=(8576, (64,)), W4=(8640, (8, 64)), b4=(9152, (8,)))
FOLDED_FLOATS = 9160
# offsets of the unfolded parameters' gradients (PB_UOFF_* in the header)
UNFOLDED_OFFSETS = dict(a0=(0, (4,)), c0=(4, (4,)), W1=(8, (64, 4)), b1=(264, (64,)), a1=(328, (64,)),
                        c1=(392, (64,)), W2=(456, (64, 64)), b2=(4552, (64,)), a2=(4616, (64,)),
                        c2=(4680, (64,)), W3=(4744, (64, 64)), b3=(8840, (64,)), a3=(8904, (64,)),
                        c3=(8968, (64,)), W4=(9032, (8, 64)), b4=(9544, (8,)))
UNFOLDED_FLOATS = 9552
# offsets of pb_quantize_mlp_i8's outputs (PB_I8_* in the header)
I8_CODES, I8_ALPHAS = 8704, 136
I8_CODE_OFFSETS = dict(T2=(0, (64, 64)), T3=(4096, (64, 64)), T4=(8192, (8, 64)))
I8_ALPHA_OFFSETS = dict(a2=(0, 64), a3=(64, 64), a4=(128, 8))


class PairBiasError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"pairbias status {status}: {msg}")
        self.status = status


class _Jets(C.Structure):
    _fields_ = [("E", C.c_void_p), ("px", C.c_void_p), ("py", C.c_void_p), ("pz", C.c_void_p),
                ("mask", C.c_void_p), ("ptr", C.c_void_p), ("N", C.c_int32), ("P", C.c_int32),
                ("tokens", C.c_int64)]


class _Mlp(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("W1", "b1", "W2", "b2", "W3", "b3", "W4", "b4")]


class _Proj(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("Wqkv", "bqkv", "Wo", "bo")]


class _MlpI8(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("W1", "b1", "T2", "T3", "T4", "a2", "a3", "a4", "b2", "b3", "b4")]


class _MlpUnfolded(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("a0", "c0", "W1", "b1", "a1", "c1", "W2", "b2", "a2", "c2",
                                          "W3", "b3", "a3", "c3", "W4", "b4")]


DEBUG_LIB_PATH = os.path.join(_HERE, "libpairbias_debug.so")
PB_DEV_BOUNDS = 4

_lock = threading.Lock()
_lib = None


def lib():
    """Load libpairbias.so (built by ``__graft_entry__.build()``); fail loudly if absent."""
    global _lib
    with _lock:
        if _lib is None:
            _lib = load(LIB_PATH)
        return _lib


def use_library(path: str):
    """Route every call of this module to the library at `path` (e.g. the
    bounds-checking build); returns the previous one for restoring."""
    global _lib
    with _lock:
        prev = _lib
        _lib = load(path)
        return prev


def restore_library(prev) -> None:
    global _lib
    with _lock:
        _lib = prev


def load(path: str):
    """Open one build of the library and declare its signatures."""
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with __graft_entry__.build()")
    L = C.CDLL(path)
    vp = C.c_void_p
    L.pairfeat_compute.argtypes = [C.POINTER(_Jets), vp, vp]
    L.pairbias_mlp_forward.argtypes = [C.POINTER(_Jets), C.POINTER(_Mlp), vp, C.c_int, vp]
    L.pair_attention_forward.argtypes = [C.POINTER(_Jets), C.POINTER(_Mlp), vp, C.c_int, C.c_int,
                                         vp, vp, vp, vp, vp, C.c_size_t, vp]
    L.pair_attention_forward_noalloc.argtypes = [C.POINTER(_Jets), C.POINTER(_Mlp), C.c_int, C.c_int,
                                                 vp, vp, vp, vp, vp]
    L.pair_block_forward.argtypes = [C.POINTER(_Jets), C.POINTER(_Mlp), C.POINTER(_Proj), C.c_int, C.c_int,
                                     C.c_int, vp, vp, vp, C.c_size_t, vp]
    L.pb_block_workspace_bytes.argtypes = [C.POINTER(_Jets)]
    L.pb_block_workspace_bytes.restype = C.c_size_t
    L.pb_workspace_bytes.argtypes = [C.POINTER(_Jets)]
    L.pb_workspace_bytes.restype = C.c_size_t
    L.pb_get_device_status.argtypes = [vp, C.POINTER(C.c_uint32)]
    L.pb_fold_affine.argtypes = [C.POINTER(_MlpUnfolded), C.POINTER(C.c_float)]
    L.pb_last_error.restype = C.c_char_p
    L.pb_version.restype = C.c_char_p
    L.pb_selftest_wait_timeouts.argtypes = [vp]
    L.pair_attention_backward.argtypes = [C.POINTER(_Jets), C.POINTER(_Mlp), C.c_int, C.c_int, vp, vp, vp, vp,
                                          vp, vp, vp, C.POINTER(_Mlp), vp, C.c_size_t, vp]
    L.pb_backward_workspace_bytes.argtypes = [C.POINTER(_Jets)]
    L.pb_backward_workspace_bytes.restype = C.c_size_t
    L.pb_unfold_grad.argtypes = [C.POINTER(_MlpUnfolded), C.POINTER(C.c_float), C.POINTER(C.c_float)]
    L.pb_quantize_mlp_i8.argtypes = [C.POINTER(C.c_float), C.POINTER(C.c_int8), C.POINTER(C.c_float)]
    L.pairbias_mlp_forward_i8.argtypes = [C.POINTER(_Jets), C.POINTER(_MlpI8), vp, C.c_int, vp]
    L.pair_attention_forward_i8.argtypes = [C.POINTER(_Jets), C.POINTER(_MlpI8), C.c_int, C.c_int, vp, vp, vp, vp,
                                            vp]
    for f in (L.pairfeat_compute, L.pairbias_mlp_forward, L.pair_attention_forward, L.pb_selftest_wait_timeouts,
              L.pair_attention_forward_noalloc, L.pair_block_forward, L.pb_get_device_status,
              L.pb_fold_affine, L.pair_attention_backward, L.pb_unfold_grad, L.pb_quantize_mlp_i8,
              L.pairbias_mlp_forward_i8, L.pair_attention_forward_i8):
        f.restype = C.c_int
    return L


def _check(st: int) -> None:
    if st != PB_OK:
        raise PairBiasError(st, lib().pb_last_error().decode())


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream) -> int:
    """cudaStream_t of `stream`, or of torch's current stream on the current device."""
    if stream is None:
        if _raw_stream is not None:
            return int(_raw_stream(torch.cuda.current_device()))
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _dp(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else int(t.data_ptr())


@dataclass
class Jets:
    """Device tensors of one jet batch (see pb_jets in the header)."""

    E: torch.Tensor
    px: torch.Tensor
    py: torch.Tensor
    pz: torch.Tensor
    mask: Optional[torch.Tensor]
    ptr: Optional[torch.Tensor]
    N: int
    P: int

    @property
    def tokens(self) -> int:
        return int(self.E.numel())

    def struct(self) -> _Jets:
        return _Jets(_dp(self.E), _dp(self.px), _dp(self.py), _dp(self.pz), _dp(self.mask), _dp(self.ptr),
                     int(self.N), int(self.P), self.tokens if self.ptr is not None else 0)


@dataclass
class FoldedMLP:
    """Folded MLP parameters in one flat fp32 device buffer (PB_OFF_* layout)."""

    flat: torch.Tensor

    def struct(self) -> _Mlp:
        base = self.flat.data_ptr()
        return _Mlp(**{k: base + 4 * off for k, (off, _s) in FOLDED_OFFSETS.items()})


def unfold_grad(params: Dict[str, np.ndarray], folded_grad: np.ndarray) -> Dict[str, np.ndarray]:
    """Gradients of the unfolded parameters from those of the folded ones
    (host, C library): a dict keyed like ``params``."""
    arrs = {k: np.ascontiguousarray(v, np.float32) for k, v in params.items()}
    st = _MlpUnfolded(**{n: arrs[n].ctypes.data for n, _t in _MlpUnfolded._fields_})
    g = np.ascontiguousarray(folded_grad, np.float32)
    assert g.size == FOLDED_FLOATS
    out = np.zeros(UNFOLDED_FLOATS, np.float32)
    fp = C.POINTER(C.c_float)
    _check(lib().pb_unfold_grad(C.byref(st), g.ctypes.data_as(fp), out.ctypes.data_as(fp)))
    return {k: out[off:off + int(np.prod(shape))].reshape(shape) for k, (off, shape) in UNFOLDED_OFFSETS.items()}


def fold_affine(params: Dict[str, np.ndarray]) -> np.ndarray:
    """Fold the batch-norm affines of an unfolded MLP (host, C library)."""
    arrs = {k: np.ascontiguousarray(v, np.float32) for k, v in params.items()}
    st = _MlpUnfolded(**{n: arrs[n].ctypes.data for n, _t in _MlpUnfolded._fields_})
    out = np.zeros(FOLDED_FLOATS, np.float32)
    _check(lib().pb_fold_affine(C.byref(st), out.ctypes.data_as(C.POINTER(C.c_float))))
    return out


def folded_mlp(params: Dict[str, np.ndarray], device="cuda") -> FoldedMLP:
    return FoldedMLP(torch.from_numpy(fold_affine(params)).to(device))


@dataclass
class MlpI8:
    """The int8 MLP (see pb_mlp_i8 in the header): the folded fp32 buffer
    (for W1, b1 and the biases) plus the int8 weight codes and row scales of
    layers 2..4, all on the device."""

    flat: torch.Tensor
    codes: torch.Tensor
    alpha: torch.Tensor

    def struct(self) -> _MlpI8:
        f, c, a = self.flat.data_ptr(), self.codes.data_ptr(), self.alpha.data_ptr()
        return _MlpI8(W1=f + 4 * FOLDED_OFFSETS["W1"][0], b1=f + 4 * FOLDED_OFFSETS["b1"][0],
                      T2=c + I8_CODE_OFFSETS["T2"][0], T3=c + I8_CODE_OFFSETS["T3"][0],
                      T4=c + I8_CODE_OFFSETS["T4"][0], a2=a + 4 * I8_ALPHA_OFFSETS["a2"][0],
                      a3=a + 4 * I8_ALPHA_OFFSETS["a3"][0], a4=a + 4 * I8_ALPHA_OFFSETS["a4"][0],
                      b2=f + 4 * FOLDED_OFFSETS["b2"][0], b3=f + 4 * FOLDED_OFFSETS["b3"][0],
                      b4=f + 4 * FOLDED_OFFSETS["b4"][0])


def quantize_mlp_i8(folded: np.ndarray):
    """int8 codes (PB_I8_CODES) and row scales (PB_I8_ALPHAS) of the folded
    layers 2..4 (host, C library)."""
    f = np.ascontiguousarray(folded, np.float32)
    assert f.size == FOLDED_FLOATS
    codes = np.zeros(I8_CODES, np.int8)
    alpha = np.zeros(I8_ALPHAS, np.float32)
    _check(lib().pb_quantize_mlp_i8(f.ctypes.data_as(C.POINTER(C.c_float)), codes.ctypes.data_as(C.POINTER(C.c_int8)),
                                    alpha.ctypes.data_as(C.POINTER(C.c_float))))
    return codes, alpha


def mlp_i8(params: Dict[str, np.ndarray], device="cuda") -> MlpI8:
    folded = fold_affine(params)
    codes, alpha = quantize_mlp_i8(folded)
    to = lambda a: torch.from_numpy(a).to(device)  # noqa: E731
    return MlpI8(to(folded), to(codes), to(alpha))


def pairbias_mlp_forward_i8(jets: Jets, mlp: MlpI8, U: torch.Tensor, stream=None) -> None:
    """U (bfloat16 or float32 [N, 8, P, P]) with the int8 MLP."""
    assert U.is_contiguous() and U.dtype in (torch.bfloat16, torch.float32)
    js, ms = jets.struct(), mlp.struct()
    dtype = PB_F32 if U.dtype == torch.float32 else PB_BF16
    _check(lib().pairbias_mlp_forward_i8(C.byref(js), C.byref(ms), U.data_ptr(), dtype, _stream(stream)))


def pair_attention_forward_i8(jets: Jets, mlp: MlpI8, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                              out: torch.Tensor, stream=None) -> None:
    """The fused path with the int8 MLP; bf16 q/k/v/out."""
    for t in (q, k, v, out):
        assert t.dtype == torch.bfloat16 and t.is_contiguous()
    js, ms = jets.struct(), mlp.struct()
    _check(lib().pair_attention_forward_i8(C.byref(js), C.byref(ms), H, D, q.data_ptr(), k.data_ptr(),
                                           v.data_ptr(), out.data_ptr(), _stream(stream)))


def jets_to_device(b, device="cuda") -> Jets:
    """Momenta, mask / ptr of a ``synth.JetBatch`` as device tensors."""
    t = lambda a, dt: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(device=device, dtype=dt)
    return Jets(t(b.E, torch.float32), t(b.px, torch.float32), t(b.py, torch.float32), t(b.pz, torch.float32),
                t(b.mask, torch.uint8), t(b.ptr, torch.int32), int(b.N), int(b.P))


def bf16_to_device(bits: np.ndarray, device="cuda") -> torch.Tensor:
    """Raw bf16 bit patterns (uint16) -> a torch.bfloat16 device tensor."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def pairfeat_compute(jets: Jets, feat: torch.Tensor, stream=None) -> None:
    """feat: float32 [N, P, P, 4] on the device."""
    assert feat.dtype == torch.float32 and feat.is_contiguous()
    js = jets.struct()
    _check(lib().pairfeat_compute(C.byref(js), feat.data_ptr(), _stream(stream)))


def pairbias_mlp_forward(jets: Jets, mlp: FoldedMLP, U: torch.Tensor, stream=None) -> None:
    """U: bfloat16 or float32 [N, 8, P, P] on the device."""
    assert U.is_contiguous() and U.dtype in (torch.bfloat16, torch.float32)
    js, ms = jets.struct(), mlp.struct()
    dtype = PB_F32 if U.dtype == torch.float32 else PB_BF16
    _check(lib().pairbias_mlp_forward(C.byref(js), C.byref(ms), U.data_ptr(), dtype, _stream(stream)))


def workspace_bytes(jets: Jets) -> int:
    """Bytes of the optional workspace of the fused path (0 if it does not apply)."""
    js = jets.struct()
    return int(lib().pb_workspace_bytes(C.byref(js)))


def workspace_for(jets: Jets, device="cuda") -> Optional[torch.Tensor]:
    """A zero-filled workspace tensor for the fused path, or None."""
    n = workspace_bytes(jets)
    return torch.zeros(n, dtype=torch.uint8, device=device) if n else None


def pair_attention_forward(jets: Jets, mlp: Optional[FoldedMLP], U: Optional[torch.Tensor], q: torch.Tensor,
                           k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
                           workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    """Fused (mlp given) or bias-reading (U given, bf16) attention; bf16 q/k/v/out.
    An optional uint8 workspace (``workspace_for``) selects the fused path
    that balances the MLP tiles of all jets over all SMs."""
    for t in (q, k, v, out):
        assert t.dtype == torch.bfloat16 and t.is_contiguous()
    if U is not None:
        assert U.dtype == torch.bfloat16 and U.is_contiguous()
    js = jets.struct()
    ms = mlp.struct() if mlp is not None else None
    ws_ptr = _dp(workspace)
    ws_len = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().pair_attention_forward(C.byref(js), C.byref(ms) if ms is not None else None,
                                        _dp(U), H, D, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                        out.data_ptr(), ws_ptr, ws_len, _stream(stream)))


def pair_attention_forward_noalloc(jets: Jets, mlp: FoldedMLP, q: torch.Tensor, k: torch.Tensor,
                                   v: torch.Tensor, out: torch.Tensor, stream=None) -> None:
    """The fused path on the library's static per-device scratch (no
    allocation anywhere); calls on one device must not overlap."""
    for t in (q, k, v, out):
        assert t.dtype == torch.bfloat16 and t.is_contiguous()
    js, ms = jets.struct(), mlp.struct()
    _check(lib().pair_attention_forward_noalloc(C.byref(js), C.byref(ms), H, D, q.data_ptr(), k.data_ptr(),
                                                v.data_ptr(), out.data_ptr(), _stream(stream)))


@dataclass
class Proj:
    """Projection weights of the attention block (see pb_proj in the header):
    bf16 Wqkv [384, 128] and Wo [128, 128], fp32 bqkv [384] and bo [128]."""

    Wqkv: torch.Tensor
    bqkv: torch.Tensor
    Wo: torch.Tensor
    bo: torch.Tensor

    def struct(self) -> _Proj:
        return _Proj(_dp(self.Wqkv), _dp(self.bqkv), _dp(self.Wo), _dp(self.bo))


def proj_to_device(bi, device="cuda") -> Proj:
    """The weights of a ``synth.BlockInputs`` as device tensors."""
    f = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(device)
    return Proj(bf16_to_device(bi.Wqkv, device), f(bi.bqkv), bf16_to_device(bi.Wo, device), f(bi.bo))


def block_workspace_bytes(jets: Jets) -> int:
    js = jets.struct()
    return int(lib().pb_block_workspace_bytes(C.byref(js)))


def pair_block_forward(jets: Jets, mlp: FoldedMLP, proj: Proj, x: torch.Tensor, y: torch.Tensor,
                       workspace: torch.Tensor, stream=None) -> None:
    """y = multi-head attention of x with the pair bias and its in/out
    projections; x, y bf16 [rows, 128]; workspace uint8 of
    ``block_workspace_bytes(jets)`` bytes."""
    for t in (x, y):
        assert t.dtype == torch.bfloat16 and t.is_contiguous()
    js, ms, ps = jets.struct(), mlp.struct(), proj.struct()
    _check(lib().pair_block_forward(C.byref(js), C.byref(ms), C.byref(ps), H, D, H * D, x.data_ptr(), y.data_ptr(),
                                    workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                    _stream(stream)))


class MlpGrad:
    """Gradients of the folded MLP parameters in one flat fp32 device buffer
    (PB_OFF_* layout, the layout of ``FoldedMLP.flat``)."""

    def __init__(self, device="cuda"):
        self.flat = torch.empty(FOLDED_FLOATS, dtype=torch.float32, device=device)

    def struct(self) -> _Mlp:
        base = self.flat.data_ptr()
        return _Mlp(**{k: base + 4 * off for k, (off, _s) in FOLDED_OFFSETS.items()})

    def as_dict(self) -> Dict[str, np.ndarray]:
        f = self.flat.cpu().numpy()
        return {k: f[off:off + int(np.prod(shape))].reshape(shape) for k, (off, shape) in FOLDED_OFFSETS.items()}


def backward_workspace_bytes(jets: Jets) -> int:
    js = jets.struct()
    return int(lib().pb_backward_workspace_bytes(C.byref(js)))


def pair_attention_backward(jets: Jets, mlp: FoldedMLP, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                            dout: torch.Tensor, dq: torch.Tensor, dk: torch.Tensor, dv: torch.Tensor,
                            dmlp: MlpGrad, workspace: torch.Tensor, stream=None) -> None:
    """Gradients of the fused forward for the upstream gradient `dout`: dq,
    dk, dv (bf16, layout of q) and the folded MLP's parameter gradients into
    `dmlp`; workspace uint8 of ``backward_workspace_bytes(jets)`` bytes."""
    for t in (q, k, v, dout, dq, dk, dv):
        assert t.dtype == torch.bfloat16 and t.is_contiguous()
    js, ms, gs = jets.struct(), mlp.struct(), dmlp.struct()
    _check(lib().pair_attention_backward(C.byref(js), C.byref(ms), H, D, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                         dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), C.byref(gs),
                                         _dp(workspace), 0 if workspace is None else workspace.numel(),
                                         _stream(stream)))


def selftest_wait_timeouts(stream=None) -> None:
    """Run the bounded-wait diagnostic (sets PB_DEV_TIMEOUT after ~4 s)."""
    _check(lib().pb_selftest_wait_timeouts(_stream(stream)))


def get_device_status(stream=None) -> int:
    """Synchronise the stream; return (and clear) the device status bits."""
    bits = C.c_uint32(0)
    st = lib().pb_get_device_status(_stream(stream), C.byref(bits))
    if st not in (PB_OK, PB_EDEVICE):
        _check(st)
    return int(bits.value)


def version() -> str:
    return lib().pb_version().decode()
