"""Parity of the softmax-over-K option (the DCNv3 form of the modulation
scalars) with the CPU oracle, on a B200, through the C ABI.

With softmax set, the K mask entries of every (pixel, group) are logits and
the weights are their softmax; grad_offset_mask then holds the logit
gradients.  The cases cover the two grid paths of the kernels (3x3 unrolled,
generic kernel sizes), the bucket, rescan and direct-scan paths of the
grad_value pass, logits far apart (the largest is subtracted before exp), and
the torch.autograd wrapper.
"""
import dataclasses

import numpy as np
import pytest

import dcn4_inputs as gen
from _parity import BWD_TOL, FWD_TOL, gpu_backward, gpu_forward, normwise, oracle_backward, oracle_forward, take, \
    to_device, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _softmax(w, **kw):
    return dataclasses.replace(w, softmax=1, name=w.name + "_softmax", **kw)


def _check(w, inp, sample=None, logits_scale=None):
    """Normwise errors of y, grad_value, the offset gradients and the logit gradients.
    logits_scale: measure the logit gradients' error against this magnitude instead of
    their own largest value (for cases where they all vanish)."""
    y = to_f64(gpu_forward(w, inp))
    gv, gom = (to_f64(t) for t in gpu_backward(w, inp))
    assert np.all(np.isfinite(y)) and np.all(np.isfinite(gv)) and np.all(np.isfinite(gom))
    body = w.G * 3 * w.K
    assert np.all(gom[..., body:] == 0.0)
    sub = inp if sample is None else take(inp, sample)
    if sample is not None:
        y, gv, gom = y[sample], gv[sample], gom[sample]
    ry = oracle_forward(w, sub)
    rgv, rgom = oracle_backward(w, sub)
    e_y = normwise(y, ry)
    e_v = normwise(gv, rgv)
    lead = gom.shape[:-1] + (w.G, 3 * w.K)
    offs, roffs = gom[..., :body].reshape(lead), rgom[..., :body].reshape(lead)
    e_off = normwise(offs[..., :2 * w.K], roffs[..., :2 * w.K])
    if logits_scale is None:
        e_m = normwise(offs[..., 2 * w.K:], roffs[..., 2 * w.K:])
    else:
        e_m = float(np.max(np.abs(offs[..., 2 * w.K:] - roffs[..., 2 * w.K:]))) / logits_scale
    assert e_y <= FWD_TOL[w.dtype], f"{w.name} forward {e_y:.3e}"
    assert e_v <= BWD_TOL[w.dtype], f"{w.name} grad_value {e_v:.3e}"
    assert e_off <= BWD_TOL[w.dtype], f"{w.name} grad offsets {e_off:.3e}"
    assert e_m <= BWD_TOL[w.dtype], f"{w.name} grad logits {e_m:.3e}"
    return e_y, e_v, e_off, e_m, offs


def test_tiny_f32_tight():
    w = _softmax(gen.WORKLOADS["tiny_f32"])
    e_y, e_v, e_off, e_m, offs = _check(w, gen.make_inputs(w))
    assert e_y < 1e-6 and e_v < 1e-6 and e_off < 1e-5 and e_m < 1e-5
    # the logit gradients of a (pixel, group) sum to zero (shift invariance)
    gm = offs[..., 2 * w.K:]
    assert np.max(np.abs(gm.sum(-1))) < 1e-5 * np.max(np.abs(gm)) * w.K


@pytest.mark.parametrize("name", ["stage1_f16", "stage3_bf16", "highres_f16", "train_bf16_k8"])
def test_workloads(name):
    """The measured workloads at full size with softmax; the oracle checks sampled images."""
    w = _softmax(gen.WORKLOADS[name])
    inp = gen.make_inputs(w)
    _check(w, inp, sample=None if w.N <= 2 else [0, w.N // 2, w.N - 1])


VARIANTS = [
    dict(name="ragged_f16_s2_d2_rc", N=3, H=7, W=5, G=3, Cg=8, Ho=3, Wo=3, K=8, P=72, dtype="f16", sh=2, sw=2,
         ph=1, pw=2, dh=2, dw=2, remove_center=1, offset_scale=0.7),
    dict(name="k5x5_bf16", N=2, H=9, W=11, G=2, Cg=16, Ho=9, Wo=11, K=25, P=152, dtype="bf16", kh=5, kw=5,
         ph=2, pw=2),
    dict(name="k1x3_f32", N=2, H=6, W=7, G=2, Cg=4, Ho=6, Wo=7, K=3, P=24, dtype="f32", kh=1, kw=3, ph=0, pw=1),
    dict(name="k3x5_f16_pad0", N=2, H=10, W=12, G=4, Cg=32, Ho=8, Wo=8, K=15, P=184, dtype="f16", kh=3, kw=5,
         ph=0, pw=0),
    dict(name="cg32_f32_nslice4", N=2, H=8, W=9, G=3, Cg=32, Ho=8, Wo=9, K=9, P=88, dtype="f32"),
    dict(name="g32_f16", N=2, H=7, W=7, G=32, Cg=8, Ho=7, Wo=7, K=9, P=864, dtype="f16"),
    dict(name="one_pixel_f16", N=1, H=1, W=1, G=4, Cg=8, Ho=1, Wo=1, K=9, P=112, dtype="f16"),
    dict(name="far_offsets_f16", N=2, H=6, W=8, G=2, Cg=8, Ho=6, Wo=8, K=9, P=56, dtype="f16",
         offset=("uniform", -40.0, 40.0)),
    dict(name="single_point_f32", N=2, H=5, W=6, G=2, Cg=4, Ho=5, Wo=6, K=1, P=8, dtype="f32", kh=1, kw=1,
         ph=0, pw=0),
]


@pytest.mark.parametrize("spec", VARIANTS, ids=[v["name"] for v in VARIANTS])
def test_variants(spec):
    w = gen.custom(softmax=1, mask=("normal", 0.0, 2.0), **spec)
    _check(w, gen.make_inputs(w))


def test_single_point_weight_is_one():
    """K = 1: the softmax weight is exactly 1 whatever the logit, and the logit gradient is 0."""
    w = gen.custom(name="k1", N=2, H=5, W=6, G=2, Cg=4, Ho=5, Wo=6, K=1, P=8, dtype="f32", kh=1, kw=1, ph=0,
                   pw=0, softmax=1, mask=("normal", 0.0, 30.0))
    inp = gen.make_inputs(w)
    plain = dataclasses.replace(w, softmax=0)
    ones = {k: v.copy() for k, v in inp.items()}
    ones["offset_mask"][..., 2:6:3] = 1.0
    assert np.array_equal(to_f64(gpu_forward(w, inp)), to_f64(gpu_forward(plain, ones)))
    _, gom = gpu_backward(w, inp)
    assert np.all(to_f64(gom)[..., 2:6:3] == 0.0)


@pytest.mark.parametrize("dtype", ["f32", "f16"])
def test_logits_far_apart(dtype):
    """One logit per (pixel, group) 90 above the rest: without subtracting the largest
    logit, exp overflows fp32; with it the weight is one-hot to within exp(-90).  The
    logit gradients then all vanish (below 1e-30): their error is measured against the
    size of the weight gradients <gy, S_k>, which the plain operator's mask gradients give."""
    w = gen.custom(name="dominant", N=2, H=12, W=10, G=2, Cg=8, Ho=12, Wo=10, K=9, P=56, dtype=dtype, softmax=1)
    inp = gen.make_inputs(w)
    rng = np.random.default_rng(11)
    body = inp["offset_mask"][..., : w.G * 27].reshape(w.N, w.Ho, w.Wo, w.G, 27)
    j = rng.integers(0, 9, size=body.shape[:-1])
    logits = np.where(np.eye(9)[j] > 0, 90.0, rng.normal(0.0, 1.0, size=body.shape[:-1] + (9,)))
    body[..., 18:] = gen.to_storage(logits, dtype).reshape(body[..., 18:].shape)
    inp["offset_mask"][..., : w.G * 27] = body.reshape(w.N, w.Ho, w.Wo, w.G * 27)
    _, plain_gom = oracle_backward(dataclasses.replace(w, softmax=0), inp)
    gw_scale = float(np.max(np.abs(plain_gom[..., : w.G * 27].reshape(-1, w.G, 27)[..., 18:])))
    _check(w, inp, logits_scale=gw_scale)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_clustered_samples_direct_path(dtype):
    """Every sample of image 0 in one cell: grad_value takes the direct scan, which
    forms each softmax weight from the logits itself."""
    w = gen.custom(name="cluster", N=2, H=48, W=40, G=4, Cg=16 if dtype == "bf16" else 8, Ho=48, Wo=40, K=9,
                   P=112, dtype=dtype, softmax=1)
    inp = gen.make_inputs(w)
    ho = np.arange(w.Ho)[:, None, None]
    wo = np.arange(w.Wo)[None, :, None]
    cells = [(ih, iw) for iw in range(3) for ih in range(3)]
    ah = ho - 1 + np.array([c[0] for c in cells])[None, None, :]
    aw = wo - 1 + np.array([c[1] for c in cells])[None, None, :]
    body = inp["offset_mask"][0, ..., : w.G * 27].reshape(w.Ho, w.Wo, w.G, 27)
    for g in range(w.G):
        body[..., g, 0:18:2] = gen.to_storage((17 - 0.25 - aw).astype(np.float64), dtype)
        body[..., g, 1:18:2] = gen.to_storage((20 + 0.25 - ah).astype(np.float64), dtype)
    inp["offset_mask"][0, ..., : w.G * 27] = body.reshape(w.Ho, w.Wo, w.G * 27)
    _check(w, inp)


def test_samples_beyond_the_filing_window():
    """Vertical offsets of up to 60 rows on 16-group tiles: overflowed tiles rescan the
    offsets and re-form the softmax weights from the logits."""
    w = gen.custom(name="window", N=2, H=128, W=14, G=16, Cg=16, Ho=128, Wo=14, K=9, P=432, dtype="bf16",
                   offset=("normal", 0.0, 1.0), softmax=1)
    inp = gen.make_inputs(w)
    rng = np.random.default_rng(7)
    body = inp["offset_mask"][..., : w.G * 27].reshape(w.N, w.Ho, w.Wo, w.G, 27)
    body[..., 1:18:2] = gen.to_storage(rng.uniform(-60.0, 60.0, size=body[..., 1:18:2].shape), w.dtype)
    inp["offset_mask"][..., : w.G * 27] = body.reshape(w.N, w.Ho, w.Wo, w.G * 27)
    _check(w, inp)


def test_softmax_flag_changes_the_result():
    """The same buffers with and without softmax give different outputs (the flag reaches the kernels)."""
    w = gen.custom(name="flag", N=1, H=8, W=8, G=2, Cg=8, Ho=8, Wo=8, K=9, P=56, dtype="f32", softmax=1)
    inp = gen.make_inputs(w)
    a = to_f64(gpu_forward(w, inp))
    b = to_f64(gpu_forward(dataclasses.replace(w, softmax=0), inp))
    assert normwise(a, b) > 1e-2


def test_autograd_softmax():
    """dcnv4_core(softmax=True) under torch.autograd against the oracle."""
    import torch
    import deformable_convolution_sampling_b200 as dcn
    w = _softmax(gen.WORKLOADS["tiny_f32"])
    inp = gen.make_inputs(w)
    v = to_device(inp["value"], w.dtype).requires_grad_(True)
    om = to_device(inp["offset_mask"], w.dtype).requires_grad_(True)
    y = dcn.dcnv4_core(v, om, group=w.G, softmax=True)
    y.backward(to_device(inp["grad_out"], w.dtype))
    torch.cuda.synchronize()
    ry = oracle_forward(w, inp)
    rgv, rgom = oracle_backward(w, inp)
    body = w.G * 3 * w.K
    assert normwise(to_f64(y), ry) < 1e-6
    assert normwise(to_f64(v.grad), rgv) < 1e-6
    assert normwise(to_f64(om.grad)[..., :body], rgom[..., :body]) < 1e-5
