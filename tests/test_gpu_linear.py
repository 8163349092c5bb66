"""Parity of dcn4_forward_linear (the merged offset/mask linear layer fused in
front of the aggregation) with the oracle, on a B200, through the C ABI.

The oracle forms offset_mask = round(x W^T + b) in double and rounds once to
the storage format; the kernel accumulates in fp32 on the tensor cores and
rounds once.  An entry may then differ by one unit in the last place where the
exact value lies next to a rounding boundary, plus the fp32 accumulation error
where the sum cancels to far below its terms (|error| <= (Cx+1) 2^-23 sum|x w|,
the standard bound for Cx+1 additions with a unit roundoff of 2^-23, which
also covers a tensor core that truncates).  The checks:
  * the offset_mask the kernel used (offset_mask_out) is within that bound of
    the oracle's everywhere, and equal almost everywhere;
  * y matches the oracle's aggregation of the oracle's offset_mask (normwise);
  * y is bit-identical to dcn4_forward on the kernel's own offset_mask (the
    same sampler on the same rows).
"""
import dataclasses

import numpy as np
import pytest

import dcn4_inputs as gen
import oracle
from _parity import FWD_TOL, gpu_forward, normwise, oracle_forward, params_for, take, to_device, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _ulp(v: np.ndarray, dtype: str) -> np.ndarray:
    """Unit in the last place of the storage format at |v|."""
    frac, emin = {"f16": (10, -14), "bf16": (7, -126)}[dtype]
    e = np.floor(np.log2(np.maximum(np.abs(v), 2.0 ** emin)))
    return 2.0 ** (e - frac)


def _run(w, Cx, *, bias=True, sample=None, seed=None):
    import torch
    import deformable_convolution_sampling_b200 as dcn
    inp = gen.make_inputs(w, with_grad=False, seed=seed)
    lin = gen.make_linear_inputs(w, Cx, bias=bias, seed=seed)
    p = params_for(w)
    v = to_device(inp["value"], w.dtype)
    x = to_device(lin["x"], w.dtype)
    wt = to_device(lin["weight"], w.dtype)
    b = to_device(lin["bias"], w.dtype) if bias else None
    om_out = torch.full((w.N, w.Ho, w.Wo, w.P), float("nan"), dtype=v.dtype, device="cuda")
    y = dcn.forward_linear(p, v, x, wt, b, offset_mask_out=om_out)
    y_plain = dcn.forward(p, v, om_out)
    y_only = dcn.forward_linear(p, v, x, wt, b)  # without storing the offset_mask
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), y_plain.view(torch.int16)), "fused sampler differs from dcn4_forward"
    assert torch.equal(y.view(torch.int16), y_only.view(torch.int16))

    idx = slice(None) if sample is None else sample
    x_s = np.ascontiguousarray(lin["x"][idx])
    om_ref = oracle.linear(w.dtype, x_s, lin["weight"], lin["bias"])
    got = to_f64(om_out)[idx]
    ref = gen.storage_to_f64(om_ref, w.dtype)
    diff = np.abs(got - ref)
    mag = np.abs(gen.storage_to_f64(x_s, w.dtype)) @ np.abs(gen.storage_to_f64(lin["weight"], w.dtype)).T
    if bias:
        mag = mag + np.abs(gen.storage_to_f64(lin["bias"], w.dtype))
    bound = _ulp(ref, w.dtype) + (Cx + 1) * 2.0 ** -23 * mag
    worst = np.unravel_index(np.argmax(diff / bound), diff.shape)
    assert np.all(diff <= bound), f"offset_mask entry {worst}: got {got[worst]}, oracle {ref[worst]}"
    assert np.mean(diff > 0) < 0.05, f"{np.mean(diff > 0):.3f} of the entries differ"

    sub = {"value": np.ascontiguousarray(inp["value"][idx]), "offset_mask": om_ref}
    ry = oracle_forward(w, sub)
    e = normwise(to_f64(y)[idx], ry)
    assert e <= FWD_TOL[w.dtype], f"{w.name} forward {e:.3e}"
    return e


@pytest.mark.parametrize("name", ["stage1_f16", "stage3_bf16", "highres_f16", "train_bf16_k8"])
def test_workloads(name):
    """The measured workloads at full size, Cx = C (the module's linear layer reads the
    block's input); the oracle checks sampled images."""
    w = gen.WORKLOADS[name]
    _run(w, w.C, sample=None if w.N <= 2 else [0, w.N // 2, w.N - 1])


VARIANTS = [
    dict(name="no_bias_f16", bias=False, Cx=64, N=2, H=12, W=10, G=4, Cg=16, Ho=12, Wo=10, K=9, P=112, dtype="f16"),
    dict(name="cx16_bf16", Cx=16, N=2, H=9, W=9, G=2, Cg=16, Ho=9, Wo=9, K=9, P=56, dtype="bf16"),
    dict(name="cx32_ne_c_f16", Cx=32, N=2, H=8, W=11, G=4, Cg=16, Ho=8, Wo=11, K=9, P=112, dtype="f16"),
    dict(name="ragged_s2_d2_rc_f16", Cx=48, N=3, H=7, W=5, G=3, Cg=8, Ho=3, Wo=3, K=8, P=72, dtype="f16",
         sh=2, sw=2, ph=1, pw=2, dh=2, dw=2, remove_center=1, offset_scale=0.7),
    dict(name="k5x5_bf16", Cx=32, N=2, H=9, W=11, G=2, Cg=16, Ho=9, Wo=11, K=25, P=152, dtype="bf16", kh=5, kw=5,
         ph=2, pw=2),
    dict(name="g32_f16", Cx=64, N=2, H=7, W=7, G=32, Cg=8, Ho=7, Wo=7, K=9, P=864, dtype="f16"),
    dict(name="wide_P_bf16", Cx=64, N=2, H=6, W=6, G=2, Cg=16, Ho=6, Wo=6, K=9, P=120, dtype="bf16"),
    dict(name="softmax_f16", Cx=64, N=2, H=10, W=12, G=4, Cg=16, Ho=10, Wo=12, K=9, P=112, dtype="f16", softmax=1),
    dict(name="one_pixel_bf16", Cx=16, N=1, H=1, W=1, G=4, Cg=8, Ho=1, Wo=1, K=9, P=112, dtype="bf16"),
    dict(name="cx128_f16", Cx=128, N=2, H=9, W=10, G=2, Cg=32, Ho=9, Wo=10, K=9, P=56, dtype="f16"),
    dict(name="cx80_bf16", Cx=80, N=2, H=9, W=10, G=2, Cg=16, Ho=9, Wo=10, K=9, P=56, dtype="bf16"),
]


@pytest.mark.parametrize("spec", VARIANTS, ids=[v["name"] for v in VARIANTS])
def test_variants(spec):
    spec = dict(spec)
    Cx, bias = spec.pop("Cx"), spec.pop("bias", True)
    w = gen.custom(**spec)
    _run(w, Cx, bias=bias)


def test_identity_weight_reproduces_offset_mask():
    """x = the offset_mask itself and weight = identity: the fused forward equals
    dcn4_forward on that offset_mask bit for bit (every product is exact)."""
    import torch
    import deformable_convolution_sampling_b200 as dcn
    w = gen.custom(name="ident", N=2, H=9, W=10, G=4, Cg=16, Ho=9, Wo=10, K=9, P=112, dtype="f16")
    inp = gen.make_inputs(w, with_grad=False, tail_fill=0.0)
    p = params_for(w)
    v = to_device(inp["value"], w.dtype)
    om = to_device(inp["offset_mask"], w.dtype)
    eye = torch.eye(w.P, dtype=v.dtype, device="cuda")
    y = dcn.forward_linear(p, v, om, eye)
    torch.cuda.synchronize()
    assert torch.equal(y, dcn.forward(p, v, om))


def test_empty_batch_is_a_noop():
    import torch
    import deformable_convolution_sampling_b200 as dcn
    p = dcn.make_params(N=0, H=8, W=8, G=4, Cg=16, dtype="f16")
    assert dcn.dcn4_forward_linear(p, 64, None, None, None, None, None, None, None) == 0
