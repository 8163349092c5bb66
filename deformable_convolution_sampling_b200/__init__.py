"""Python binding of libdcn4, the sm_100a DCNv4 core spatial aggregation.

The C ABI (include/dcn4.h) is exposed under the same names -- ``dcn4_forward``,
``dcn4_backward``, ``dcn4_output_dims`` ... -- taking a :class:`dcn4_params`
and raw device pointers.  They only marshal arguments: every step of the
operator runs in the library's CUDA kernels.  There is no CPU fallback; if the
library is not built, importing this package fails.

``forward`` / ``backward`` are conveniences over the same calls for torch
tensors (torch provides device memory and streams only).
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdcn4.so")

DCN4_F32, DCN4_F16, DCN4_BF16 = 0, 1, 2
STATUS = {
    0: "DCN4_OK", -1: "DCN4_ERR_NULL", -2: "DCN4_ERR_BAD_SHAPE", -3: "DCN4_ERR_BAD_P",
    -4: "DCN4_ERR_MISALIGNED", -5: "DCN4_ERR_UNSUPPORTED", -6: "DCN4_ERR_WORKSPACE",
    -7: "DCN4_ERR_LAUNCH", -8: "DCN4_ERR_DTYPE",
}
DTYPE_NAMES = {"f32": DCN4_F32, "f16": DCN4_F16, "bf16": DCN4_BF16}


class Dcn4Error(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"{STATUS.get(status, status)}: {detail}")
        self.status = status


class dcn4_params(ctypes.Structure):
    """Mirror of the C struct dcn4_params."""

    _fields_ = [
        ("N", ctypes.c_int), ("H", ctypes.c_int), ("W", ctypes.c_int),
        ("G", ctypes.c_int), ("Cg", ctypes.c_int),
        ("kh", ctypes.c_int), ("kw", ctypes.c_int),
        ("sh", ctypes.c_int), ("sw", ctypes.c_int),
        ("ph", ctypes.c_int), ("pw", ctypes.c_int),
        ("dh", ctypes.c_int), ("dw", ctypes.c_int),
        ("offset_scale", ctypes.c_float),
        ("remove_center", ctypes.c_int),
        ("P", ctypes.c_int),
        ("dtype", ctypes.c_int),
        ("softmax", ctypes.c_int),
    ]


class dcn4_attn_params(ctypes.Structure):
    """Mirror of dcn4_attn_params in include/dcn4.h (field order matters)."""

    _fields_ = [
        ("N", ctypes.c_int), ("H", ctypes.c_int), ("W", ctypes.c_int),
        ("G", ctypes.c_int), ("Cg", ctypes.c_int),
        ("Nq", ctypes.c_int), ("K", ctypes.c_int),
        ("offset_scale", ctypes.c_float),
        ("P", ctypes.c_int),
        ("dtype", ctypes.c_int),
    ]


def make_attn_params(*, N, H, W, G, Cg, Nq, K, offset_scale=1.0, P=None, dtype="f16") -> dcn4_attn_params:
    """dcn4_attn_params for a single-scale deformable attention call; P defaults to G*3K rounded up to 8."""
    if isinstance(dtype, str):
        dtype = DTYPE_NAMES[dtype]
    if P is None:
        P = -(-G * 3 * K // 8) * 8
    return dcn4_attn_params(N, H, W, G, Cg, Nq, K, float(offset_scale), P, dtype)


def make_params(*, N, H, W, G, Cg, kh=3, kw=3, sh=1, sw=1, ph=1, pw=1, dh=1, dw=1,
                offset_scale=1.0, remove_center=0, P=None, dtype="f32", softmax=0) -> dcn4_params:
    """Build a dcn4_params; P defaults to the smallest valid padded row.  softmax=1
    normalises the K masks of each (pixel, group) with a softmax (the DCNv3 form)."""
    if isinstance(dtype, str):
        dtype = DTYPE_NAMES[dtype]
    if P is None:
        P = dcn4_padded_offset_dim(G, kh * kw - (1 if remove_center else 0))
    return dcn4_params(N, H, W, G, Cg, kh, kw, sh, sw, ph, pw, dh, dw, float(offset_scale),
                       1 if remove_center else 0, P, dtype, 1 if softmax else 0)


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is not built; run `python deformable_convolution_sampling_b200/build.py` "
            "(there is no CPU fallback)")
    L = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER(dcn4_params)
    AP = ctypes.POINTER(dcn4_attn_params)
    vp, ip = ctypes.c_void_p, ctypes.POINTER(ctypes.c_int)
    sig = {
        "dcn4_version": ([], ctypes.c_int),
        "dcn4_num_points": ([P], ctypes.c_int),
        "dcn4_padded_offset_dim": ([ctypes.c_int, ctypes.c_int], ctypes.c_int),
        "dcn4_output_dims": ([P, ip, ip], ctypes.c_int),
        "dcn4_check_params": ([P], ctypes.c_int),
        "dcn4_forward": ([P, vp, vp, vp, vp], ctypes.c_int),
        "dcn4_forward_linear": ([P, ctypes.c_int, vp, vp, vp, vp, vp, vp, vp], ctypes.c_int),
        "dcn4_backward_workspace_size": ([P], ctypes.c_size_t),
        "dcn4_backward": ([P, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp], ctypes.c_int),
        "dcn4_status_string": ([ctypes.c_int], ctypes.c_char_p),
        "dcn4_last_error": ([], ctypes.c_char_p),
        "dcn4_backward_offset_mask": ([P, vp, vp, vp, vp, vp, ctypes.c_size_t, vp], ctypes.c_int),
        "dcn4_backward_value": ([P, vp, vp, vp, vp, ctypes.c_size_t, vp], ctypes.c_int),
        "dcn4_backward_noalloc": ([P, vp, vp, vp, vp, vp, vp], ctypes.c_int),
        "dcn4_backward_noalloc_capacity": ([], ctypes.c_size_t),
        "dcn4_noalloc_last_error": ([], ctypes.c_char_p),
        "dcn4_backward_diagnostics": ([P, vp, ctypes.c_size_t, ip, vp], ctypes.c_int),
        "dcn4_backward_linear_workspace_size": ([P, ctypes.c_int], ctypes.c_size_t),
        "dcn4_backward_linear": ([P, ctypes.c_int] + [vp] * 11 + [ctypes.c_size_t, vp], ctypes.c_int),
        "dcn4_forward_proj": ([P, ctypes.c_int, vp, vp, vp, vp, vp, vp, vp], ctypes.c_int),
        "dcn4_forward_tc_status": ([ctypes.c_int], ctypes.c_int),
        "dcn4_backward_proj_workspace_size": ([P, ctypes.c_int], ctypes.c_size_t),
        "dcn4_backward_proj": ([P, ctypes.c_int] + [vp] * 10 + [ctypes.c_size_t, vp], ctypes.c_int),
        "dcn4_attn_check_params": ([AP], ctypes.c_int),
        "dcn4_attn_forward": ([AP, vp, vp, vp, vp, vp], ctypes.c_int),
        "dcn4_attn_backward_workspace_size": ([AP], ctypes.c_size_t),
        "dcn4_attn_backward": ([AP, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp], ctypes.c_int),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    return L


lib = _load()


# ---------------------------------------------------------------------------
# Same-name wrappers of the C ABI (pointers are ints or None; stream is a
# cudaStream_t handle as an int, 0 / None for the legacy default stream).
# ---------------------------------------------------------------------------

def dcn4_version() -> int:
    return lib.dcn4_version()


def dcn4_num_points(p: dcn4_params) -> int:
    return lib.dcn4_num_points(ctypes.byref(p))


def dcn4_padded_offset_dim(G: int, K: int) -> int:
    return lib.dcn4_padded_offset_dim(G, K)


def dcn4_output_dims(p: dcn4_params) -> tuple[int, int, int]:
    ho, wo = ctypes.c_int(), ctypes.c_int()
    st = lib.dcn4_output_dims(ctypes.byref(p), ctypes.byref(ho), ctypes.byref(wo))
    return st, ho.value, wo.value


def dcn4_check_params(p: dcn4_params) -> int:
    return lib.dcn4_check_params(ctypes.byref(p))


def dcn4_forward(p: dcn4_params, value, offset_mask, out, stream=None) -> int:
    return lib.dcn4_forward(ctypes.byref(p), value, offset_mask, out, stream)


def dcn4_forward_linear(p: dcn4_params, Cx: int, value, x, weight, bias, out, offset_mask_out=None,
                        stream=None) -> int:
    return lib.dcn4_forward_linear(ctypes.byref(p), int(Cx), value, x, weight, bias, out, offset_mask_out, stream)


def dcn4_forward_proj(p: dcn4_params, Cout: int, value, offset_mask, weight, bias, out, core_out=None,
                      stream=None) -> int:
    return lib.dcn4_forward_proj(ctypes.byref(p), int(Cout), value, offset_mask, weight, bias, out, core_out, stream)


def dcn4_forward_tc_status(reset: bool = False) -> int:
    return lib.dcn4_forward_tc_status(1 if reset else 0)


def dcn4_backward_proj_workspace_size(p: dcn4_params, Cout: int) -> int:
    return lib.dcn4_backward_proj_workspace_size(ctypes.byref(p), int(Cout))


def dcn4_backward_proj(p: dcn4_params, Cout: int, value, offset_mask, core_out, weight, grad_out, grad_value,
                       grad_offset_mask, grad_weight, grad_bias, workspace, workspace_bytes: int, stream=None) -> int:
    return lib.dcn4_backward_proj(ctypes.byref(p), int(Cout), value, offset_mask, core_out, weight, grad_out,
                                  grad_value, grad_offset_mask, grad_weight, grad_bias, workspace, workspace_bytes,
                                  stream)


def dcn4_backward_workspace_size(p: dcn4_params) -> int:
    return lib.dcn4_backward_workspace_size(ctypes.byref(p))


def dcn4_backward(p: dcn4_params, value, offset_mask, grad_out, grad_value, grad_offset_mask,
                  workspace, workspace_bytes: int, stream=None) -> int:
    return lib.dcn4_backward(ctypes.byref(p), value, offset_mask, grad_out, grad_value,
                             grad_offset_mask, workspace, workspace_bytes, stream)


def dcn4_backward_offset_mask(p: dcn4_params, value, offset_mask, grad_out, grad_offset_mask, workspace,
                              workspace_bytes: int, stream=None) -> int:
    return lib.dcn4_backward_offset_mask(ctypes.byref(p), value, offset_mask, grad_out, grad_offset_mask,
                                         workspace, workspace_bytes, stream)


def dcn4_backward_value(p: dcn4_params, offset_mask, grad_out, grad_value, workspace, workspace_bytes: int,
                        stream=None) -> int:
    return lib.dcn4_backward_value(ctypes.byref(p), offset_mask, grad_out, grad_value, workspace,
                                   workspace_bytes, stream)


def dcn4_backward_diagnostics(p: dcn4_params, workspace, workspace_bytes: int, stream=None):
    """(status, [corrupt bucket tiles, rescanned tiles, direct-path tiles]) of the last
    backward run on `workspace`; waits for `stream`."""
    counts = (ctypes.c_int * 3)()
    st = lib.dcn4_backward_diagnostics(ctypes.byref(p), workspace, workspace_bytes, counts, stream)
    return st, list(counts)


def dcn4_backward_linear_workspace_size(p: dcn4_params, Cx: int) -> int:
    return lib.dcn4_backward_linear_workspace_size(ctypes.byref(p), int(Cx))


def dcn4_backward_linear(p: dcn4_params, Cx: int, value, offset_mask, x, weight, grad_out, grad_value,
                         grad_offset_mask, grad_x, grad_weight, grad_bias, workspace, workspace_bytes: int,
                         stream=None) -> int:
    return lib.dcn4_backward_linear(ctypes.byref(p), int(Cx), value, offset_mask, x, weight, grad_out, grad_value,
                                    grad_offset_mask, grad_x, grad_weight, grad_bias, workspace, workspace_bytes,
                                    stream)


def dcn4_attn_check_params(p: dcn4_attn_params) -> int:
    return lib.dcn4_attn_check_params(ctypes.byref(p))


def dcn4_attn_forward(p: dcn4_attn_params, value, ref_points, offset_logits, out, stream=None) -> int:
    return lib.dcn4_attn_forward(ctypes.byref(p), value, ref_points, offset_logits, out, stream)


def dcn4_attn_backward_workspace_size(p: dcn4_attn_params) -> int:
    return lib.dcn4_attn_backward_workspace_size(ctypes.byref(p))


def dcn4_attn_backward(p: dcn4_attn_params, value, ref_points, offset_logits, grad_out, grad_value,
                       grad_offset_logits, workspace, workspace_bytes: int, stream=None) -> int:
    return lib.dcn4_attn_backward(ctypes.byref(p), value, ref_points, offset_logits, grad_out, grad_value,
                                  grad_offset_logits, workspace, workspace_bytes, stream)


def dcn4_backward_noalloc(p: dcn4_params, value, offset_mask, grad_out, grad_value, grad_offset_mask,
                          stream=None) -> int:
    """dcn4_backward with the library's built-in scratch area instead of a workspace
    (for callers that cannot provide device memory when they call)."""
    return lib.dcn4_backward_noalloc(ctypes.byref(p), value, offset_mask, grad_out, grad_value,
                                     grad_offset_mask, stream)


def dcn4_backward_noalloc_capacity() -> int:
    return lib.dcn4_backward_noalloc_capacity()


def dcn4_noalloc_last_error() -> str:
    return lib.dcn4_noalloc_last_error().decode()


def dcn4_status_string(status: int) -> str:
    return lib.dcn4_status_string(status).decode()


def dcn4_last_error() -> str:
    return lib.dcn4_last_error().decode()


def check(status: int) -> None:
    """Raise Dcn4Error for a negative status."""
    if status != 0:
        raise Dcn4Error(status, dcn4_last_error())


# ---------------------------------------------------------------------------
# torch conveniences (device memory and the current stream come from torch)
# ---------------------------------------------------------------------------

def _torch_dtype(code: int):
    import torch
    return {DCN4_F32: torch.float32, DCN4_F16: torch.float16, DCN4_BF16: torch.bfloat16}[code]


def _stream_handle(device):
    import torch
    return torch.cuda.current_stream(device).cuda_stream


def forward(p: dcn4_params, value, offset_mask, out=None):
    """y[N,Ho,Wo,C] for CUDA tensors value[N,H,W,C] and offset_mask[N,Ho,Wo,P]."""
    import torch
    st, Ho, Wo = dcn4_output_dims(p)
    check(st)
    if out is None:
        out = torch.empty((p.N, Ho, Wo, p.G * p.Cg), dtype=_torch_dtype(p.dtype), device=value.device)
    check(dcn4_forward(p, value.data_ptr(), offset_mask.data_ptr(), out.data_ptr(),
                       _stream_handle(value.device)))
    return out


def forward_linear(p: dcn4_params, value, x, weight, bias=None, out=None, offset_mask_out=None):
    """y[N,Ho,Wo,C] with the offset_mask formed in the kernel as x @ weight.T + bias
    (x [N,Ho,Wo,Cx], weight [P,Cx], bias [P] or None); offset_mask_out, when given
    ([N,Ho,Wo,P]), receives that offset_mask.  CUDA tensors, fp16 or bf16."""
    import torch
    st, Ho, Wo = dcn4_output_dims(p)
    check(st)
    if out is None:
        out = torch.empty((p.N, Ho, Wo, p.G * p.Cg), dtype=_torch_dtype(p.dtype), device=value.device)
    check(dcn4_forward_linear(p, x.shape[-1], value.data_ptr(), x.data_ptr(), weight.data_ptr(),
                              bias.data_ptr() if bias is not None else None, out.data_ptr(),
                              offset_mask_out.data_ptr() if offset_mask_out is not None else None,
                              _stream_handle(value.device)))
    return out


def backward(p: dcn4_params, value, offset_mask, grad_out, grad_value=None, grad_offset_mask=None,
             workspace=None):
    """(grad_value[N,H,W,C], grad_offset_mask[N,Ho,Wo,P]) for CUDA tensors.  `workspace`
    (a uint8 CUDA tensor of dcn4_backward_workspace_size bytes) is allocated when not
    given; pass one to read the call's fallback counters with backward_diagnostics."""
    import torch
    st, Ho, Wo = dcn4_output_dims(p)
    check(st)
    dt = _torch_dtype(p.dtype)
    if grad_value is None:
        grad_value = torch.empty_like(value, dtype=dt)
    if grad_offset_mask is None:
        grad_offset_mask = torch.empty((p.N, Ho, Wo, p.P), dtype=dt, device=value.device)
    need = dcn4_backward_workspace_size(p)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=value.device)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    check(dcn4_backward(p, value.data_ptr(), offset_mask.data_ptr(), grad_out.data_ptr(),
                        grad_value.data_ptr(), grad_offset_mask.data_ptr(), ws_ptr, ws_bytes,
                        _stream_handle(value.device)))
    return grad_value, grad_offset_mask


def backward_linear(p: dcn4_params, value, offset_mask, x, weight, grad_out, with_bias: bool = True,
                    want_x: bool = True, want_weight: bool = True, workspace=None):
    """Backward of forward_linear for CUDA tensors (offset_mask: the one the forward
    formed): (grad_value, grad_offset_mask, grad_x or None, grad_weight or None,
    grad_bias or None), all computed in libdcn4."""
    import torch
    st, Ho, Wo = dcn4_output_dims(p)
    check(st)
    dt = _torch_dtype(p.dtype)
    dev = value.device
    Cx = x.shape[-1]
    gv = torch.empty_like(value, dtype=dt)
    gom = torch.empty((p.N, Ho, Wo, p.P), dtype=dt, device=dev)
    gx = torch.empty_like(x) if want_x else None
    gw = torch.empty_like(weight) if want_weight else None
    gb = torch.empty((p.P,), dtype=dt, device=dev) if with_bias else None
    need = dcn4_backward_linear_workspace_size(p, Cx)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)

    def ptr(t):
        return t.data_ptr() if t is not None else None

    check(dcn4_backward_linear(p, Cx, value.data_ptr(), offset_mask.data_ptr(), x.data_ptr(), weight.data_ptr(),
                               grad_out.data_ptr(), gv.data_ptr(), gom.data_ptr(), ptr(gx), ptr(gw), ptr(gb),
                               workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                               _stream_handle(dev)))
    return gv, gom, gx, gw, gb


def forward_proj(p: dcn4_params, value, offset_mask, weight, bias=None, out=None, core_out=None):
    """y[N,Ho,Wo,Cout] = (aggregation of value at offset_mask) @ weight.T + bias, the
    projection formed inside the forward kernel (weight [Cout,C], bias [Cout] or None);
    core_out, when given ([N,Ho,Wo,C]), receives the aggregation's own output.  CUDA
    tensors, fp16 or bf16."""
    import torch
    st, Ho, Wo = dcn4_output_dims(p)
    check(st)
    Cout = weight.shape[0]
    if out is None:
        out = torch.empty((p.N, Ho, Wo, Cout), dtype=_torch_dtype(p.dtype), device=value.device)
    check(dcn4_forward_proj(p, Cout, value.data_ptr(), offset_mask.data_ptr(), weight.data_ptr(),
                            bias.data_ptr() if bias is not None else None, out.data_ptr(),
                            core_out.data_ptr() if core_out is not None else None, _stream_handle(value.device)))
    return out


def backward_proj(p: dcn4_params, value, offset_mask, core_out, weight, grad_out, with_bias: bool = True,
                  want_weight: bool = True, workspace=None):
    """Backward of forward_proj for CUDA tensors (core_out: the aggregation output the
    forward saved): (grad_value, grad_offset_mask, grad_weight or None, grad_bias or
    None), all computed in libdcn4."""
    import torch
    st, Ho, Wo = dcn4_output_dims(p)
    check(st)
    dt = _torch_dtype(p.dtype)
    dev = value.device
    Cout = weight.shape[0]
    gv = torch.empty_like(value, dtype=dt)
    gom = torch.empty((p.N, Ho, Wo, p.P), dtype=dt, device=dev)
    gw = torch.empty_like(weight) if want_weight else None
    gb = torch.empty((Cout,), dtype=dt, device=dev) if with_bias else None
    need = dcn4_backward_proj_workspace_size(p, Cout)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)

    def ptr(t):
        return t.data_ptr() if t is not None else None

    check(dcn4_backward_proj(p, Cout, value.data_ptr(), offset_mask.data_ptr(), ptr(core_out), weight.data_ptr(),
                             grad_out.data_ptr(), gv.data_ptr(), gom.data_ptr(), ptr(gw), ptr(gb),
                             workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                             _stream_handle(dev)))
    return gv, gom, gw, gb


def attn_forward(p: dcn4_attn_params, value, ref_points, offset_logits, out=None):
    """y[N,Nq,C] of single-scale deformable attention for CUDA tensors value [N,H,W,C],
    ref_points [N,Nq,2] (float32) and offset_logits [N,Nq,P]."""
    import torch
    if out is None:
        out = torch.empty((p.N, p.Nq, p.G * p.Cg), dtype=_torch_dtype(p.dtype), device=value.device)
    check(dcn4_attn_forward(p, value.data_ptr(), ref_points.data_ptr(), offset_logits.data_ptr(), out.data_ptr(),
                            _stream_handle(value.device)))
    return out


def attn_backward(p: dcn4_attn_params, value, ref_points, offset_logits, grad_out):
    """(grad_value[N,H,W,C], grad_offset_logits[N,Nq,P]) for CUDA tensors."""
    import torch
    dt = _torch_dtype(p.dtype)
    gv = torch.empty((p.N, p.H, p.W, p.G * p.Cg), dtype=dt, device=value.device)
    gol = torch.empty((p.N, p.Nq, p.P), dtype=dt, device=value.device)
    need = dcn4_attn_backward_workspace_size(p)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device=value.device)
    check(dcn4_attn_backward(p, value.data_ptr(), ref_points.data_ptr(), offset_logits.data_ptr(),
                             grad_out.data_ptr(), gv.data_ptr(), gol.data_ptr(), ws.data_ptr(), need,
                             _stream_handle(value.device)))
    return gv, gol


def backward_diagnostics(p: dcn4_params, workspace) -> dict:
    """Fallback counters of the last backward on `workspace` (a uint8 CUDA tensor)."""
    st, c = dcn4_backward_diagnostics(p, workspace.data_ptr(), workspace.numel(), _stream_handle(workspace.device))
    check(st)
    return {"corrupt_bucket_tiles": c[0], "rescanned_tiles": c[1], "direct_tiles": c[2]}


# ---------------------------------------------------------------------------
# torch.autograd wrapper (argument marshalling only: both passes run in libdcn4)
# ---------------------------------------------------------------------------

_TORCH_CODES = None


def _dtype_code(t) -> int:
    import torch
    global _TORCH_CODES
    if _TORCH_CODES is None:
        _TORCH_CODES = {torch.float32: DCN4_F32, torch.float16: DCN4_F16, torch.bfloat16: DCN4_BF16}
    if t.dtype not in _TORCH_CODES:
        raise ValueError(f"dtype {t.dtype} is not float32, float16 or bfloat16")
    return _TORCH_CODES[t.dtype]


def _pair(v):
    return (v, v) if isinstance(v, int) else tuple(v)


def params_for_tensors(value, offset_mask, *, group: int, kernel=3, stride=1, pad=1, dilation=1,
                       offset_scale: float = 1.0, remove_center: bool = False,
                       softmax: bool = False) -> dcn4_params:
    """dcn4_params for NHWC value [N,H,W,C] and offset_mask [N,Ho,Wo,P]; checks shapes,
    dtypes, devices and contiguity on the host (ValueError) before anything is launched."""
    if value.dim() != 4 or offset_mask.dim() != 4:
        raise ValueError("value must be [N,H,W,C] and offset_mask [N,Ho,Wo,P]")
    if value.dtype != offset_mask.dtype:
        raise ValueError("value and offset_mask must have the same dtype")
    if not (value.is_contiguous() and offset_mask.is_contiguous()):
        raise ValueError("value and offset_mask must be contiguous (channels last)")
    N, H, W, C = value.shape
    if group < 1 or C % group != 0:
        raise ValueError(f"C={C} is not a multiple of group={group}")
    if not (value.is_cuda and offset_mask.is_cuda):
        raise ValueError("value and offset_mask must be CUDA tensors")
    if value.device != offset_mask.device:
        raise ValueError("value and offset_mask must be on the same device")
    (kh, kw), (sh, sw), (ph, pw), (dh, dw) = _pair(kernel), _pair(stride), _pair(pad), _pair(dilation)
    p = make_params(N=N, H=H, W=W, G=group, Cg=C // group, kh=kh, kw=kw, sh=sh, sw=sw, ph=ph, pw=pw, dh=dh,
                    dw=dw, offset_scale=float(offset_scale), remove_center=int(bool(remove_center)),
                    P=offset_mask.shape[-1], dtype={DCN4_F32: "f32", DCN4_F16: "f16", DCN4_BF16: "bf16"}[_dtype_code(value)],
                    softmax=int(bool(softmax)))
    st, Ho, Wo = dcn4_output_dims(p)
    check(st)
    if tuple(offset_mask.shape[:3]) != (N, Ho, Wo):
        raise ValueError(f"offset_mask must be [N={N}, Ho={Ho}, Wo={Wo}, P], got {tuple(offset_mask.shape)}")
    check(dcn4_check_params(p))
    return p


def _autograd_function():
    import torch

    class DCNv4Core(torch.autograd.Function):
        """The DCNv4 core aggregation as a torch.autograd.Function: forward and backward
        are dcn4_forward and dcn4_backward on the tensors' device and current stream."""

        @staticmethod
        def forward(ctx, value, offset_mask, p):
            ctx.save_for_backward(value, offset_mask)
            ctx.p = p
            return forward(p, value, offset_mask)

        @staticmethod
        def backward(ctx, grad_out):
            value, offset_mask = ctx.saved_tensors
            grad_value, grad_offset_mask = backward(ctx.p, value, offset_mask, grad_out.contiguous())
            return grad_value, grad_offset_mask, None

    return DCNv4Core


_DCNV4_CORE = None
_DCNV4_CORE_LINEAR = None
_DCNV4_CORE_PROJ = None


def _autograd_function_proj():
    import torch

    class DCNv4CoreProj(torch.autograd.Function):
        """The aggregation with the output projection fused behind it as a
        torch.autograd.Function.  Forward: dcn4_forward_proj, keeping the core output.
        Backward: dcn4_backward_proj (the projection's gradients in libdcn4's
        tensor-core kernels, then dcn4_backward with grad_core = grad_out W)."""

        @staticmethod
        def forward(ctx, value, offset_mask, weight, bias, p):
            st, Ho, Wo = dcn4_output_dims(p)
            check(st)
            core = torch.empty((p.N, Ho, Wo, p.G * p.Cg), dtype=value.dtype, device=value.device)
            y = forward_proj(p, value, offset_mask, weight, bias, core_out=core)
            ctx.save_for_backward(value, offset_mask, weight, core)
            ctx.p = p
            ctx.has_bias = bias is not None
            return y

        @staticmethod
        def backward(ctx, grad_out):
            value, offset_mask, weight, core = ctx.saved_tensors
            grad_value, grad_om, grad_w, grad_b = backward_proj(
                ctx.p, value, offset_mask, core, weight, grad_out.contiguous(), with_bias=ctx.has_bias,
                want_weight=ctx.needs_input_grad[2])
            return grad_value, grad_om, grad_w, grad_b, None

    return DCNv4CoreProj


def _autograd_function_linear():
    import torch

    class DCNv4CoreLinear(torch.autograd.Function):
        """The offset/mask linear layer fused into the aggregation as a
        torch.autograd.Function.  Forward: dcn4_forward_linear, keeping the
        offset_mask it formed.  Backward: dcn4_backward_linear, i.e. dcn4_backward on
        that offset_mask, then the linear layer's gradients (grad_x = g W,
        grad_W = g^T x, grad_b = sum g, with g = grad_offset_mask as [M, P]) in
        libdcn4's tensor-core kernels."""

        @staticmethod
        def forward(ctx, value, x, weight, bias, p):
            st, Ho, Wo = dcn4_output_dims(p)
            check(st)
            om = torch.empty((p.N, Ho, Wo, p.P), dtype=value.dtype, device=value.device)
            y = forward_linear(p, value, x, weight, bias, offset_mask_out=om)
            ctx.save_for_backward(value, x, weight, om)
            ctx.p = p
            ctx.has_bias = bias is not None
            return y

        @staticmethod
        def backward(ctx, grad_out):
            value, x, weight, om = ctx.saved_tensors
            grad_value, _, grad_x, grad_w, grad_b = backward_linear(
                ctx.p, value, om, x, weight, grad_out.contiguous(), with_bias=ctx.has_bias,
                want_x=ctx.needs_input_grad[1], want_weight=ctx.needs_input_grad[2])
            return grad_value, grad_x, grad_w, grad_b, None

    return DCNv4CoreLinear


def dcnv4_core(value, offset_mask, *, group: int, kernel=3, stride=1, pad=1, dilation=1,
               offset_scale: float = 1.0, remove_center: bool = False, softmax: bool = False):
    """y = DCNv4 core aggregation of value [N,H,W,C] at the offsets and masks of
    offset_mask [N,Ho,Wo,P], differentiable in both (torch.autograd).  softmax=True
    takes the masks as logits normalised over the K points (the DCNv3 form)."""
    global _DCNV4_CORE
    p = params_for_tensors(value, offset_mask, group=group, kernel=kernel, stride=stride, pad=pad,
                           dilation=dilation, offset_scale=offset_scale, remove_center=remove_center,
                           softmax=softmax)
    if _DCNV4_CORE is None:
        _DCNV4_CORE = _autograd_function()
    return _DCNV4_CORE.apply(value, offset_mask, p)


def dcnv4_core_linear(value, x, weight, bias=None, *, group: int, kernel=3, stride=1, pad=1, dilation=1,
                      offset_scale: float = 1.0, remove_center: bool = False, softmax: bool = False):
    """y = DCNv4 core aggregation of value [N,H,W,C] at offset_mask = x @ weight.T + bias,
    formed inside the forward kernel (x [N,Ho,Wo,Cx], weight [P,Cx], bias [P] or None;
    fp16/bf16), differentiable in value, x, weight and bias (torch.autograd)."""
    global _DCNV4_CORE_LINEAR
    if weight.dim() != 2 or x.dim() != 4 or x.shape[-1] != weight.shape[1]:
        raise ValueError("x must be [N,Ho,Wo,Cx] and weight [P,Cx]")
    if bias is not None and tuple(bias.shape) != (weight.shape[0],):
        raise ValueError("bias must be [P]")
    for name, t in (("x", x), ("weight", weight)) + ((("bias", bias),) if bias is not None else ()):
        if t.dtype != value.dtype or not t.is_contiguous() or t.device != value.device:
            raise ValueError(f"{name} must be contiguous, on value's device and of value's dtype")
    # the shape checks of the operator itself, on an offset_mask-shaped view of the producer
    N = value.shape[0]
    p = params_for_tensors(value, _OffsetMaskShape(x.shape[:3], weight.shape[0], value), group=group, kernel=kernel,
                           stride=stride, pad=pad, dilation=dilation, offset_scale=offset_scale,
                           remove_center=remove_center, softmax=softmax)
    if x.shape[0] != N:
        raise ValueError("x and value must have the same batch")
    if _DCNV4_CORE_LINEAR is None:
        _DCNV4_CORE_LINEAR = _autograd_function_linear()
    return _DCNV4_CORE_LINEAR.apply(value, x, weight, bias, p)


def dcnv4_core_proj(value, offset_mask, weight, bias=None, *, group: int, kernel=3, stride=1, pad=1, dilation=1,
                    offset_scale: float = 1.0, remove_center: bool = False, softmax: bool = False):
    """y = (DCNv4 core aggregation of value [N,H,W,C] at offset_mask [N,Ho,Wo,P]) @ weight.T
    + bias, the output projection (weight [Cout,C], bias [Cout] or None; fp16/bf16)
    formed inside the forward kernel; differentiable in value, offset_mask, weight and
    bias (torch.autograd)."""
    global _DCNV4_CORE_PROJ
    if weight.dim() != 2 or weight.shape[1] != value.shape[-1]:
        raise ValueError("weight must be [Cout, C]")
    if bias is not None and tuple(bias.shape) != (weight.shape[0],):
        raise ValueError("bias must be [Cout]")
    for name, t in (("weight", weight),) + ((("bias", bias),) if bias is not None else ()):
        if t.dtype != value.dtype or not t.is_contiguous() or t.device != value.device:
            raise ValueError(f"{name} must be contiguous, on value's device and of value's dtype")
    p = params_for_tensors(value, offset_mask, group=group, kernel=kernel, stride=stride, pad=pad,
                           dilation=dilation, offset_scale=offset_scale, remove_center=remove_center,
                           softmax=softmax)
    if _DCNV4_CORE_PROJ is None:
        _DCNV4_CORE_PROJ = _autograd_function_proj()
    return _DCNV4_CORE_PROJ.apply(value, offset_mask, weight, bias, p)


class _OffsetMaskShape:
    """Stands in for an offset_mask tensor [N,Ho,Wo,P] in params_for_tensors' checks."""

    def __init__(self, lead, P, like):
        self.shape = tuple(lead) + (int(P),)
        self.dtype = like.dtype
        self.is_cuda = like.is_cuda
        self.device = like.device

    def dim(self):
        return 4

    def is_contiguous(self):
        return True
