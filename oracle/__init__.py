"""ctypes binding of the plain CPU oracle (liboracle.so).

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference arm are the only callers.  The product
package never imports this module.

Arrays are numpy: storage ``"f32"`` -> float32, ``"f16"`` -> float16,
``"bf16"`` -> uint16 holding bfloat16 bit patterns, ``"f64"`` -> float64.
Results and gradients come back as float64.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os

import numpy as np

from . import build as _build

DTYPES = {"f32": 0, "f16": 1, "bf16": 2, "f64": 3}
NUMPY_STORAGE = {"f32": np.float32, "f16": np.float16, "bf16": np.uint16, "f64": np.float64}


class _Problem(ctypes.Structure):
    _fields_ = [
        ("N", ctypes.c_int), ("H", ctypes.c_int), ("W", ctypes.c_int),
        ("G", ctypes.c_int), ("Cg", ctypes.c_int),
        ("kh", ctypes.c_int), ("kw", ctypes.c_int),
        ("sh", ctypes.c_int), ("sw", ctypes.c_int),
        ("ph", ctypes.c_int), ("pw", ctypes.c_int),
        ("dh", ctypes.c_int), ("dw", ctypes.c_int),
        ("offset_scale", ctypes.c_double),
        ("remove_center", ctypes.c_int),
        ("P", ctypes.c_int),
        ("dtype", ctypes.c_int),
        ("location_fp32", ctypes.c_int),
        ("softmax", ctypes.c_int),
    ]


@dataclasses.dataclass
class Problem:
    """Geometry of one DCNv4 core call, as the oracle sees it."""

    N: int
    H: int
    W: int
    G: int
    Cg: int
    kh: int = 3
    kw: int = 3
    sh: int = 1
    sw: int = 1
    ph: int = 1
    pw: int = 1
    dh: int = 1
    dw: int = 1
    offset_scale: float = 1.0
    remove_center: int = 0
    P: int | None = None          # None: the smallest multiple of 8 >= G*3K
    dtype: str = "f64"
    location_fp32: bool = False
    softmax: bool = False         # DCNv3 variant: the masks are logits, softmax over k

    @property
    def K(self) -> int:
        return self.kh * self.kw - (1 if self.remove_center else 0)

    @property
    def C(self) -> int:
        return self.G * self.Cg

    @property
    def row(self) -> int:
        if self.P is not None:
            return self.P
        return -(-self.G * 3 * self.K // 8) * 8

    def c_struct(self) -> _Problem:
        return _Problem(
            self.N, self.H, self.W, self.G, self.Cg, self.kh, self.kw, self.sh, self.sw,
            self.ph, self.pw, self.dh, self.dw, float(self.offset_scale),
            1 if self.remove_center else 0, self.row, DTYPES[self.dtype],
            1 if self.location_fp32 else 0, 1 if self.softmax else 0,
        )


class _AttnProblem(ctypes.Structure):
    _fields_ = [
        ("N", ctypes.c_int), ("H", ctypes.c_int), ("W", ctypes.c_int),
        ("G", ctypes.c_int), ("Cg", ctypes.c_int),
        ("Nq", ctypes.c_int), ("K", ctypes.c_int),
        ("offset_scale", ctypes.c_double),
        ("P", ctypes.c_int),
        ("dtype", ctypes.c_int),
        ("location_fp32", ctypes.c_int),
    ]


@dataclasses.dataclass
class AttnProblem:
    """Geometry of one single-scale deformable attention call, as the oracle sees it."""

    N: int
    H: int
    W: int
    G: int
    Cg: int
    Nq: int
    K: int
    offset_scale: float = 1.0
    P: int | None = None          # None: the smallest multiple of 8 >= G*3K
    dtype: str = "f64"
    location_fp32: bool = False

    @property
    def C(self) -> int:
        return self.G * self.Cg

    @property
    def row(self) -> int:
        return self.P if self.P is not None else -(-self.G * 3 * self.K // 8) * 8

    def c_struct(self) -> _AttnProblem:
        return _AttnProblem(self.N, self.H, self.W, self.G, self.Cg, self.Nq, self.K, float(self.offset_scale),
                            self.row, DTYPES[self.dtype], 1 if self.location_fp32 else 0)


_lib = None


def lib() -> ctypes.CDLL:
    """Load liboracle.so, compiling it first when it is missing or stale."""
    global _lib
    if _lib is None:
        # DCN4_ORACLE_LIB lets the mutation tests load a deliberately broken copy.
        path = os.environ.get("DCN4_ORACLE_LIB") or _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.POINTER(_Problem)
        vp, dp = ctypes.c_void_p, ctypes.POINTER(ctypes.c_double)
        L.ref_output_dims.argtypes = [P, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]
        L.ref_output_dims.restype = ctypes.c_int
        L.ref_num_points.argtypes = [P]
        L.ref_num_points.restype = ctypes.c_int
        L.ref_forward.argtypes = [P, vp, vp, dp, ctypes.c_int]
        L.ref_forward.restype = ctypes.c_int
        L.ref_backward.argtypes = [P, vp, vp, vp, dp, dp, ctypes.c_int]
        L.ref_backward.restype = ctypes.c_int
        L.ref_decode.argtypes = [ctypes.c_int, vp, dp, ctypes.c_int64]
        L.ref_decode.restype = None
        L.ref_encode.argtypes = [ctypes.c_int, dp, vp, ctypes.c_int64]
        L.ref_encode.restype = None
        L.ref_linear.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, vp, vp, vp]
        L.ref_linear.restype = ctypes.c_int
        L.ref_linear_backward.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, vp, vp,
                                          dp, dp, dp, ctypes.c_int]
        L.ref_linear_backward.restype = ctypes.c_int
        AP = ctypes.POINTER(_AttnProblem)
        L.ref_attn_forward.argtypes = [AP, vp, vp, vp, dp, ctypes.c_int]
        L.ref_attn_forward.restype = ctypes.c_int
        L.ref_attn_backward.argtypes = [AP, vp, vp, vp, vp, dp, dp, ctypes.c_int]
        L.ref_attn_backward.restype = ctypes.c_int
        _lib = L
    return _lib


def output_dims(prob: Problem) -> tuple[int, int]:
    ho, wo = ctypes.c_int(), ctypes.c_int()
    st = prob.c_struct()
    if lib().ref_output_dims(ctypes.byref(st), ctypes.byref(ho), ctypes.byref(wo)) != 0:
        raise ValueError(f"malformed problem {prob}")
    return ho.value, wo.value


def _check(arr: np.ndarray, prob: Problem, shape: tuple, name: str) -> np.ndarray:
    want = NUMPY_STORAGE[prob.dtype]
    if arr.dtype != want:
        raise TypeError(f"{name}: storage {prob.dtype} wants {np.dtype(want)}, got {arr.dtype}")
    if tuple(arr.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {arr.shape}, expected {shape}")
    return np.ascontiguousarray(arr)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _dptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def forward(prob: Problem, value: np.ndarray, offset_mask: np.ndarray, nthreads: int = 1) -> np.ndarray:
    """y[N,Ho,Wo,C] in float64."""
    Ho, Wo = output_dims(prob)
    value = _check(value, prob, (prob.N, prob.H, prob.W, prob.C), "value")
    offset_mask = _check(offset_mask, prob, (prob.N, Ho, Wo, prob.row), "offset_mask")
    out = np.empty((prob.N, Ho, Wo, prob.C), dtype=np.float64)
    st = prob.c_struct()
    if lib().ref_forward(ctypes.byref(st), _ptr(value), _ptr(offset_mask), _dptr(out), int(nthreads)) != 0:
        raise ValueError(f"oracle forward rejected {prob}")
    return out


def backward(prob: Problem, value: np.ndarray, offset_mask: np.ndarray, grad_out: np.ndarray,
             nthreads: int = 1) -> tuple[np.ndarray, np.ndarray]:
    """(grad_value[N,H,W,C], grad_offset_mask[N,Ho,Wo,P]) in float64."""
    Ho, Wo = output_dims(prob)
    value = _check(value, prob, (prob.N, prob.H, prob.W, prob.C), "value")
    offset_mask = _check(offset_mask, prob, (prob.N, Ho, Wo, prob.row), "offset_mask")
    grad_out = _check(grad_out, prob, (prob.N, Ho, Wo, prob.C), "grad_out")
    gv = np.empty((prob.N, prob.H, prob.W, prob.C), dtype=np.float64)
    gom = np.empty((prob.N, Ho, Wo, prob.row), dtype=np.float64)
    st = prob.c_struct()
    rc = lib().ref_backward(ctypes.byref(st), _ptr(value), _ptr(offset_mask), _ptr(grad_out),
                            _dptr(gv), _dptr(gom), int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle backward rejected {prob}")
    return gv, gom


def decode(dtype: str, arr: np.ndarray) -> np.ndarray:
    """Exact float64 value of every stored element."""
    arr = np.ascontiguousarray(arr)
    if arr.dtype != NUMPY_STORAGE[dtype]:
        raise TypeError(f"decode {dtype}: got {arr.dtype}")
    out = np.empty(arr.shape, dtype=np.float64)
    lib().ref_decode(DTYPES[dtype], _ptr(arr), _dptr(out), arr.size)
    return out


def encode(dtype: str, values: np.ndarray) -> np.ndarray:
    """values (float64) stored in `dtype`, rounded to nearest, ties to even."""
    v = np.ascontiguousarray(values, dtype=np.float64)
    out = np.empty(v.shape, dtype=NUMPY_STORAGE[dtype])
    lib().ref_encode(DTYPES[dtype], _dptr(v), _ptr(out), v.size)
    return out


def linear(dtype: str, x: np.ndarray, weight: np.ndarray, bias: np.ndarray | None = None) -> np.ndarray:
    """The merged offset/mask linear layer: round_dtype(x @ weight.T + bias) with x
    [..., Cin], weight [Cout, Cin], bias [Cout] (or None), all stored in `dtype`;
    returns [..., Cout] stored in `dtype`."""
    want = NUMPY_STORAGE[dtype]
    x = np.ascontiguousarray(x)
    weight = np.ascontiguousarray(weight)
    for name, a in (("x", x), ("weight", weight)) + ((("bias", bias),) if bias is not None else ()):
        if a.dtype != want:
            raise TypeError(f"{name}: storage {dtype} wants {np.dtype(want)}, got {a.dtype}")
    Cout, Cin = weight.shape
    if x.shape[-1] != Cin or (bias is not None and tuple(bias.shape) != (Cout,)):
        raise ValueError("linear: shape mismatch")
    M = int(np.prod(x.shape[:-1]))
    out = np.empty(x.shape[:-1] + (Cout,), dtype=want)
    b = _ptr(np.ascontiguousarray(bias)) if bias is not None else None
    if lib().ref_linear(M, Cin, Cout, DTYPES[dtype], _ptr(x), _ptr(weight), b, _ptr(out)) != 0:
        raise ValueError("oracle linear rejected its arguments")
    return out


def linear_backward(dtype: str, x: np.ndarray, weight: np.ndarray, grad: np.ndarray, nthreads: int = 1,
                    want_x: bool = True, want_weight: bool = True):
    """Gradients of the merged offset/mask linear layer for the upstream gradient
    `grad` [..., Cout] of its output (x [..., Cin], weight [Cout, Cin], all stored in
    `dtype`): (grad_x [..., Cin], grad_weight [Cout, Cin], grad_bias [Cout]) in
    float64, unrounded; grad_x (want_x=False) or grad_weight and grad_bias
    (want_weight=False) come back as None when not wanted."""
    want = NUMPY_STORAGE[dtype]
    x, weight, grad = (np.ascontiguousarray(a) for a in (x, weight, grad))
    for name, a in (("x", x), ("weight", weight), ("grad", grad)):
        if a.dtype != want:
            raise TypeError(f"{name}: storage {dtype} wants {np.dtype(want)}, got {a.dtype}")
    Cout, Cin = weight.shape
    if x.shape[-1] != Cin or grad.shape != x.shape[:-1] + (Cout,):
        raise ValueError("linear_backward: shape mismatch")
    M = int(np.prod(x.shape[:-1]))
    gx = np.empty(x.shape, dtype=np.float64)
    gw = np.empty((Cout, Cin), dtype=np.float64)
    gb = np.empty((Cout,), dtype=np.float64)
    if lib().ref_linear_backward(M, Cin, Cout, DTYPES[dtype], _ptr(x), _ptr(weight), _ptr(grad),
                                 _dptr(gx) if want_x else None, _dptr(gw) if want_weight else None,
                                 _dptr(gb) if want_weight else None, int(nthreads)) != 0:
        raise ValueError("oracle linear_backward rejected its arguments")
    return (gx if want_x else None), (gw if want_weight else None), (gb if want_weight else None)


def _attn_check(prob: AttnProblem, value, ref_points, offset_logits):
    value = _check(value, prob, (prob.N, prob.H, prob.W, prob.C), "value")
    offset_logits = _check(offset_logits, prob, (prob.N, prob.Nq, prob.row), "offset_logits")
    ref_points = np.ascontiguousarray(ref_points)
    if ref_points.dtype != np.float32 or tuple(ref_points.shape) != (prob.N, prob.Nq, 2):
        raise ValueError(f"ref_points must be float32 [{prob.N}, {prob.Nq}, 2]")
    return value, ref_points, offset_logits


def attn_forward(prob: AttnProblem, value, ref_points, offset_logits, nthreads: int = 1) -> np.ndarray:
    """Single-scale deformable attention: out[N,Nq,G*Cg] in float64."""
    value, ref_points, offset_logits = _attn_check(prob, value, ref_points, offset_logits)
    out = np.empty((prob.N, prob.Nq, prob.C), dtype=np.float64)
    st = prob.c_struct()
    if lib().ref_attn_forward(ctypes.byref(st), _ptr(value), _ptr(ref_points), _ptr(offset_logits), _dptr(out),
                              int(nthreads)) != 0:
        raise ValueError(f"oracle attention forward rejected {prob}")
    return out


def attn_backward(prob: AttnProblem, value, ref_points, offset_logits, grad_out, nthreads: int = 1):
    """(grad_value[N,H,W,C], grad_offset_logits[N,Nq,P]) in float64."""
    value, ref_points, offset_logits = _attn_check(prob, value, ref_points, offset_logits)
    grad_out = _check(grad_out, prob, (prob.N, prob.Nq, prob.C), "grad_out")
    gv = np.empty((prob.N, prob.H, prob.W, prob.C), dtype=np.float64)
    gol = np.empty((prob.N, prob.Nq, prob.row), dtype=np.float64)
    st = prob.c_struct()
    if lib().ref_attn_backward(ctypes.byref(st), _ptr(value), _ptr(ref_points), _ptr(offset_logits),
                               _ptr(grad_out), _dptr(gv), _dptr(gol), int(nthreads)) != 0:
        raise ValueError(f"oracle attention backward rejected {prob}")
    return gv, gol


def host_threads() -> int:
    """Host cores this process may run on (what nthreads=-1 callers should use)."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1
