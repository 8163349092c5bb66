"""Parity of the CUDA path (through the C ABI) with the CPU oracle, on a B200.

Every workload of the measured configuration table is compared with the
oracle element by element on the same seeded, storage-rounded inputs (whole
batches where the oracle finishes in seconds, whole sampled images otherwise:
images are independent, so an image's outputs depend on that image only).
The oracle forms sampling locations with the same fp32 fused multiply-add as
the kernels, so both sides pick the same bilinear cell.
"""
import math

import numpy as np
import pytest

import dcn4_inputs as gen
from _parity import (BWD_TOL, FWD_TOL, gpu_backward, gpu_forward, normwise, oracle_backward,
                     oracle_forward, params_for, take, to_device, to_f64)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _check_forward(w, inp, sample=None):
    y = to_f64(gpu_forward(w, inp))
    assert np.all(np.isfinite(y))
    if sample is None:
        ref = oracle_forward(w, inp)
        got = y
    else:
        ref = oracle_forward(w, take(inp, sample))
        got = y[sample]
    err = normwise(got, ref)
    assert err <= FWD_TOL[w.dtype], f"{w.name} forward normwise error {err:.3e}"
    return err


def _check_backward(w, inp, sample=None):
    gv, gom = gpu_backward(w, inp)
    gv, gom = to_f64(gv), to_f64(gom)
    body = w.G * 3 * w.K
    assert np.all(gom[..., body:] == 0.0), "padding tail of grad_offset_mask must be 0"
    sub = inp if sample is None else take(inp, sample)
    rgv, rgom = oracle_backward(w, sub)
    if sample is not None:
        gv, gom = gv[sample], gom[sample]
    e_v = normwise(gv, rgv)
    e_om = normwise(gom[..., :body], rgom[..., :body])
    assert e_v <= BWD_TOL[w.dtype], f"{w.name} grad_value normwise error {e_v:.3e}"
    assert e_om <= BWD_TOL[w.dtype], f"{w.name} grad_offset_mask normwise error {e_om:.3e}"
    # offsets and masks separately (different magnitudes)
    offs = gom[..., :body].reshape(gom.shape[:-1] + (w.G, 3 * w.K))
    roffs = rgom[..., :body].reshape(rgom.shape[:-1] + (w.G, 3 * w.K))
    e_off = normwise(offs[..., :2 * w.K], roffs[..., :2 * w.K])
    e_m = normwise(offs[..., 2 * w.K:], roffs[..., 2 * w.K:])
    assert e_off <= BWD_TOL[w.dtype] and e_m <= BWD_TOL[w.dtype], (e_off, e_m)
    return e_v, e_om


# ---------------------------------------------------------------------------
# The measured workloads, at full size
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("name", gen.WORKLOAD_ORDER)
def test_forward_workload(name):
    w = gen.WORKLOADS[name]
    inp = gen.make_inputs(w, with_grad=False)
    _check_forward(w, inp)


@pytest.mark.parametrize("name", gen.WORKLOAD_ORDER)
def test_backward_workload(name):
    w = gen.WORKLOADS[name]
    inp = gen.make_inputs(w)
    sample = None if w.N <= 2 else [0, w.N // 2, w.N - 1]
    if name == "train_bf16_k8" or name == "tiny_f32":
        sample = None                    # the workloads with a backward pass: whole batch
    _check_backward(w, inp, sample)


def test_fp32_tolerance_is_tight_on_tiny():
    w = gen.WORKLOADS["tiny_f32"]
    inp = gen.make_inputs(w)
    assert _check_forward(w, inp) < 1e-6
    e_v, e_om = _check_backward(w, inp)
    assert e_v < 1e-6 and e_om < 1e-5


# ---------------------------------------------------------------------------
# Geometry, dtype and layout variants (ragged tiles, generic kernel sizes,
# one and several threads per group, tiny and large G)
# ---------------------------------------------------------------------------

VARIANTS = [
    dict(name="ragged_f16_s2_d2_rc", N=3, H=7, W=5, G=3, Cg=8, Ho=3, Wo=3, K=8, P=72, dtype="f16", sh=2, sw=2,
         ph=1, pw=2, dh=2, dw=2, remove_center=1, offset_scale=0.7),
    dict(name="k5x5_bf16", N=2, H=9, W=11, G=2, Cg=16, Ho=9, Wo=11, K=25, P=152, dtype="bf16", kh=5, kw=5,
         ph=2, pw=2),
    dict(name="k1x3_f32", N=2, H=6, W=7, G=2, Cg=4, Ho=6, Wo=7, K=3, P=24, dtype="f32", kh=1, kw=3, ph=0, pw=1),
    dict(name="k3x5_f16_pad0", N=2, H=10, W=12, G=4, Cg=32, Ho=8, Wo=8, K=15, P=184, dtype="f16", kh=3, kw=5,
         ph=0, pw=0),
    dict(name="cg64_f16_nslice4", N=2, H=9, W=10, G=2, Cg=64, Ho=9, Wo=10, K=9, P=56, dtype="f16"),
    dict(name="cg32_f32_nslice4", N=2, H=8, W=9, G=3, Cg=32, Ho=8, Wo=9, K=9, P=88, dtype="f32"),
    dict(name="g1_bf16", N=3, H=5, W=6, G=1, Cg=16, Ho=5, Wo=6, K=9, P=32, dtype="bf16"),
    dict(name="g32_f16", N=2, H=7, W=7, G=32, Cg=8, Ho=7, Wo=7, K=9, P=864, dtype="f16"),
    dict(name="wide_P_f32", N=2, H=6, W=6, G=2, Cg=8, Ho=6, Wo=6, K=9, P=120, dtype="f32"),
    dict(name="one_pixel_f16", N=1, H=1, W=1, G=4, Cg=8, Ho=1, Wo=1, K=9, P=112, dtype="f16"),
    dict(name="far_offsets_f16", N=2, H=6, W=8, G=2, Cg=8, Ho=6, Wo=8, K=9, P=56, dtype="f16",
         offset=("uniform", -40.0, 40.0)),
]


@pytest.mark.parametrize("spec", VARIANTS, ids=[v["name"] for v in VARIANTS])
def test_variant_forward_backward(spec):
    w = gen.custom(**spec)
    inp = gen.make_inputs(w)
    _check_forward(w, inp)
    _check_backward(w, inp)


def test_integer_offsets_exact_cells():
    w = gen.custom(name="int", N=2, H=8, W=8, G=2, Cg=8, Ho=8, Wo=8, K=9, P=56, dtype="f32")
    inp = gen.make_inputs(w)
    om = inp["offset_mask"]
    body = om[..., :54].reshape(2, 8, 8, 2, 27)
    body[..., :18] = np.round(body[..., :18] * 2.0)        # integers in [-6, 6]
    om[..., :54] = body.reshape(2, 8, 8, 54)
    assert _check_forward(w, inp) < 1e-6
    _check_backward(w, inp)


def test_all_samples_off_image_give_zero():
    import torch
    w = gen.custom(name="off", N=2, H=6, W=6, G=2, Cg=8, Ho=6, Wo=6, K=9, P=56, dtype="f16")
    inp = gen.make_inputs(w)
    body = inp["offset_mask"][..., :54].reshape(2, 6, 6, 2, 27)
    body[..., :18] = np.float16(1000.0)
    inp["offset_mask"][..., :54] = body.reshape(2, 6, 6, 54)
    y = gpu_forward(w, inp)
    assert torch.count_nonzero(y).item() == 0
    gv, gom = gpu_backward(w, inp)
    assert torch.count_nonzero(gv).item() == 0 and torch.count_nonzero(gom).item() == 0


def test_empty_batch_is_a_noop():
    import torch
    import deformable_convolution_sampling_b200 as dcn
    p = dcn.make_params(N=0, H=5, W=5, G=2, Cg=8, dtype="f16")
    out = torch.full((4,), 7.0, device="cuda", dtype=torch.float16)
    assert dcn.dcn4_forward(p, None, None, out.data_ptr(), None) == 0
    assert dcn.dcn4_backward(p, None, None, None, None, None, None, 0, None) == 0
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)


def test_forward_is_deterministic_and_stream_ordered():
    import torch
    import deformable_convolution_sampling_b200 as dcn
    w = gen.WORKLOADS["stage3_bf16"]
    inp = gen.make_inputs(w, with_grad=False)
    p = params_for(w)
    v, om = to_device(inp["value"], w.dtype), to_device(inp["offset_mask"], w.dtype)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        a = dcn.forward(p, v, om)
        b = dcn.forward(p, v, om)
    s.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_more_than_2_pow_31_elements():
    """64-bit addressing: a batch whose tensors hold > 2^31 elements (tiled copies of 4 images)."""
    import torch
    import deformable_convolution_sampling_b200 as dcn
    w = gen.WORKLOADS["stage1_f16"]
    base = gen.custom(**{**w.__dict__, "N": 4, "name": "big_base"})
    inp = gen.make_inputs(base)
    reps = math.ceil((2 ** 31 + 1) / (w.H * w.W * w.C) / 4)
    Nb = 4 * reps
    assert Nb * w.H * w.W * w.C > 2 ** 31
    p = dcn.make_params(dtype=w.dtype, **{**w.geometry(), "N": Nb})
    v = to_device(inp["value"], w.dtype).repeat(reps, 1, 1, 1)
    om = to_device(inp["offset_mask"], w.dtype).repeat(reps, 1, 1, 1)
    gy = to_device(inp["grad_out"], w.dtype).repeat(reps, 1, 1, 1)
    y = dcn.forward(p, v, om)
    last = to_f64(y[Nb - 4:])
    ref = oracle_forward(base, inp)
    assert normwise(last, ref) <= FWD_TOL[w.dtype]
    del y
    gv, gom = dcn.backward(p, v, om, gy)
    rgv, rgom = oracle_backward(base, inp)
    assert normwise(to_f64(gv[Nb - 4:]), rgv) <= BWD_TOL[w.dtype]
    assert normwise(to_f64(gom[Nb - 4:]), rgom) <= BWD_TOL[w.dtype]
    del v, om, gy, gv, gom
    torch.cuda.empty_cache()


@pytest.mark.parametrize("dtype", ["f16", "f32"])
def test_16_byte_aligned_pointers(dtype):
    """Pointers that are 16- but not 32-byte aligned take the 16-byte access path."""
    import torch
    import deformable_convolution_sampling_b200 as dcn
    w = gen.custom(name="align", N=2, H=9, W=7, G=4, Cg=16 if dtype == "f16" else 8, Ho=9, Wo=7, K=9, P=112,
                   dtype=dtype)
    inp = gen.make_inputs(w)
    p = params_for(w)
    eb = 2 if dtype == "f16" else 4
    shift = 16 // eb                                   # 16 bytes, in elements

    def shifted(a):
        t = to_device(a.reshape(-1), dtype)
        buf = torch.empty(t.numel() + 2 * shift, dtype=t.dtype, device="cuda")
        buf[shift:shift + t.numel()] = t
        return buf[shift:shift + t.numel()].view(a.shape)

    v, om, gy = shifted(inp["value"]), shifted(inp["offset_mask"]), shifted(inp["grad_out"])
    assert v.data_ptr() % 32 == 16
    out = torch.empty(v.numel() + 2 * shift, dtype=v.dtype, device="cuda")[shift:shift + v.numel()].view(v.shape)
    y = dcn.forward(p, v, om, out=out)
    ref = oracle_forward(w, inp)
    assert normwise(to_f64(y), ref) <= FWD_TOL[dtype]
    gv = torch.empty(v.numel() + 2 * shift, dtype=v.dtype, device="cuda")[shift:shift + v.numel()].view(v.shape)
    gv, gom = dcn.backward(p, v, om, gy, grad_value=gv)
    rgv, rgom = oracle_backward(w, inp)
    assert normwise(to_f64(gv), rgv) <= BWD_TOL[dtype]
    assert normwise(to_f64(gom), rgom) <= BWD_TOL[dtype]


def _anchors(w):
    """Grid anchors (row, col) of every (pixel, point) in k order (columns outer, rows inner)."""
    cells = [(ih, iw) for iw in range(w.kw) for ih in range(w.kh)
             if not (w.remove_center and ih == w.kh // 2 and iw == w.kw // 2)]
    ho = np.arange(w.Ho)[:, None, None]
    wo = np.arange(w.Wo)[None, :, None]
    ah = ho * w.sh - w.ph + np.array([c[0] for c in cells])[None, None, :] * w.dh
    aw = wo * w.sw - w.pw + np.array([c[1] for c in cells])[None, None, :] * w.dw
    return np.broadcast_to(ah, (w.Ho, w.Wo, len(cells))), np.broadcast_to(aw, (w.Ho, w.Wo, len(cells)))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_samples_clustered_on_one_cell(dtype):
    """Every sample of image 0 lands in the same cell: the per-tile sort overflows
    and grad_value takes the direct-scan path; image 1 keeps ordinary offsets."""
    w = gen.custom(name="cluster", N=2, H=48, W=40, G=4, Cg=16 if dtype == "bf16" else 8, Ho=48, Wo=40, K=9,
                   P=112, dtype=dtype)
    inp = gen.make_inputs(w)
    ah, aw = _anchors(w)
    frac = 0.25
    dy = (20 + frac - ah).astype(np.float64)     # s = 1: location = anchor + offset = (20.25, 17.75)
    dx = (17 - frac - aw).astype(np.float64)
    body = inp["offset_mask"][0, ..., : w.G * 27].reshape(w.Ho, w.Wo, w.G, 27)
    for g in range(w.G):
        body[..., g, 0:18:2] = gen.to_storage(dx, dtype)
        body[..., g, 1:18:2] = gen.to_storage(dy, dtype)
    inp["offset_mask"][0, ..., : w.G * 27] = body.reshape(w.Ho, w.Wo, w.G * 27)
    _check_forward(w, inp)
    _check_backward(w, inp)
    diag = _diagnostics(w, inp)
    assert diag["corrupt_bucket_tiles"] == 0 and diag["direct_tiles"] > 0, diag


def _diagnostics(w, inp):
    """Fallback counters of one backward through the C ABI on these inputs."""
    import torch
    import deformable_convolution_sampling_b200 as dcn
    p = params_for(w)
    ws = torch.empty(dcn.dcn4_backward_workspace_size(p), dtype=torch.uint8, device="cuda")
    dcn.backward(p, *(to_device(inp[k], w.dtype) for k in ("value", "offset_mask", "grad_out")), workspace=ws)
    return dcn.backward_diagnostics(p, ws)


def test_images_with_different_reach():
    """Per-image reach: one image with tiny offsets, one with offsets spanning the image."""
    w = gen.custom(name="reach", N=3, H=24, W=33, G=4, Cg=16, Ho=24, Wo=33, K=9, P=112, dtype="f16",
                   offset=("normal", 0.0, 0.2))
    inp = gen.make_inputs(w)
    big = gen.make_inputs(gen.custom(**{**w.__dict__, "offset": ("uniform", -30.0, 30.0)}), seed=9)
    inp["offset_mask"][1] = big["offset_mask"][1]
    zero = inp["offset_mask"][2, ..., : w.G * 27].reshape(w.Ho, w.Wo, w.G, 27)
    zero[..., :18] = 0                               # integer anchors exactly
    inp["offset_mask"][2, ..., : w.G * 27] = zero.reshape(w.Ho, w.Wo, w.G * 27)
    _check_forward(w, inp)
    _check_backward(w, inp)


def test_backward_stages_equal_backward():
    """dcn4_backward_offset_mask then dcn4_backward_value == dcn4_backward."""
    import torch
    import deformable_convolution_sampling_b200 as dcn
    w = gen.WORKLOADS["train_bf16_k8"]
    inp = gen.make_inputs(gen.custom(**{**w.__dict__, "N": 4, "name": "stages"}))
    p = dcn.make_params(dtype=w.dtype, **{**w.geometry(), "N": 4})
    v, om, gy = (to_device(inp[k], w.dtype) for k in ("value", "offset_mask", "grad_out"))
    gv_ref, gom_ref = dcn.backward(p, v, om, gy)
    nbytes = dcn.dcn4_backward_workspace_size(p)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    gv, gom = torch.empty_like(gv_ref), torch.empty_like(gom_ref)
    s = torch.cuda.current_stream().cuda_stream
    dcn.check(dcn.dcn4_backward_offset_mask(p, v.data_ptr(), om.data_ptr(), gy.data_ptr(), gom.data_ptr(),
                                            ws.data_ptr(), nbytes, s))
    dcn.check(dcn.dcn4_backward_value(p, om.data_ptr(), gy.data_ptr(), gv.data_ptr(), ws.data_ptr(), nbytes, s))
    torch.cuda.synchronize()
    assert torch.equal(gom.view(torch.int16), gom_ref.view(torch.int16))
    # grad_value sums the samples of a cell in the order the shared-memory sort placed
    # them, which may differ between calls: one bfloat16 ulp apart at most, plus fp32
    # summation noise where the sum cancels to almost nothing.
    a, b = to_f64(gv), to_f64(gv_ref)
    assert np.all(np.abs(a - b) <= 2.0 ** -7 * np.maximum(np.abs(a), np.abs(b)) + 2.0 ** -20 * np.abs(b).max())


def test_backward_value_twice_on_one_workspace():
    """The grad_value stage only reads the workspace: calling it twice after one
    grad_offset_mask stage gives the same gradient (up to the summation order
    within a cell)."""
    import torch
    import deformable_convolution_sampling_b200 as dcn
    w = gen.WORKLOADS["stage1_f16"]
    w = gen.custom(**{**w.__dict__, "N": 4, "name": "twice"})
    inp = gen.make_inputs(w)
    p = dcn.make_params(dtype=w.dtype, **w.geometry())
    v, om, gy = (to_device(inp[k], w.dtype) for k in ("value", "offset_mask", "grad_out"))
    nbytes = dcn.dcn4_backward_workspace_size(p)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    gom = torch.empty_like(om)
    s = torch.cuda.current_stream().cuda_stream
    dcn.check(dcn.dcn4_backward_offset_mask(p, v.data_ptr(), om.data_ptr(), gy.data_ptr(), gom.data_ptr(),
                                            ws.data_ptr(), nbytes, s))
    out = []
    for _ in range(2):
        gv = torch.full_like(v, float("nan"))
        dcn.check(dcn.dcn4_backward_value(p, om.data_ptr(), gy.data_ptr(), gv.data_ptr(), ws.data_ptr(), nbytes, s))
        out.append(gv)
    torch.cuda.synchronize()
    a, b = to_f64(out[0]), to_f64(out[1])
    assert np.all(np.isfinite(a)) and np.all(np.isfinite(b))
    assert np.all(np.abs(a - b) <= 2.0 ** -10 * np.maximum(np.abs(a), np.abs(b)) + 2.0 ** -20 * np.abs(b).max())


def test_samples_beyond_the_filing_window():
    """Third-stage-like tiles (16 groups: three rows per grad_value tile, a filing
    window of 16 x 4 tiles) with vertical offsets of up to 60 rows: samples land
    outside the window of tiles a grad_offset_mask CTA files into, those tiles are
    marked overflowed, and grad_value rescans their offsets."""
    w = gen.custom(name="window", N=2, H=128, W=14, G=16, Cg=16, Ho=128, Wo=14, K=9, P=432, dtype="bf16",
                   offset=("normal", 0.0, 1.0))
    inp = gen.make_inputs(w)
    rng = np.random.default_rng(7)
    body = inp["offset_mask"][..., : w.G * 27].reshape(w.N, w.Ho, w.Wo, w.G, 27)
    dy = rng.uniform(-60.0, 60.0, size=body[..., 1:18:2].shape)
    body[..., 1:18:2] = gen.to_storage(dy, w.dtype)
    inp["offset_mask"][..., : w.G * 27] = body.reshape(w.N, w.Ho, w.Wo, w.G * 27)
    _check_forward(w, inp)
    _check_backward(w, inp)
    diag = _diagnostics(w, inp)
    assert diag["corrupt_bucket_tiles"] == 0 and diag["rescanned_tiles"] > 0, diag


def test_copies_of_samples_filed_outside_the_window():
    """32 groups of 8 channels on a 14 x 14 map: grad_value tiles of two rows, so the filing
    window of the bottom grad_offset_mask CTAs leaves out the top tile rows.  With offsets
    N(0, 4^2) some of their samples land in a cell on the border of an excluded tile and the
    next one down: the excluded tile rescans, and the tile below (inside every CTA's window)
    must rescan too, since it does not get the sample's copy.  Both against the oracle."""
    w = gen.custom(name="window_copies", N=4, H=14, W=14, G=32, Cg=8, Ho=14, Wo=14, K=9, P=864, dtype="bf16",
                   offset=("normal", 0.0, 4.0))
    inp = gen.make_inputs(w)
    _check_backward(w, inp)
    diag = _diagnostics(w, inp)
    assert diag["corrupt_bucket_tiles"] == 0 and diag["rescanned_tiles"] > 0, diag


@pytest.mark.parametrize("name", gen.WORKLOAD_ORDER)
def test_no_fallback_tiles_on_the_workloads(name):
    """On every measured workload no grad_value tile finds its filed records
    inconsistent (the counter of tiles sent to the direct path by a failed bucket
    check stays 0)."""
    w = gen.WORKLOADS[name]
    if w.N > 8:
        w = gen.custom(**{**w.__dict__, "N": 8, "name": name + "_8"})
    inp = gen.make_inputs(w)
    diag = _diagnostics(w, inp)
    assert diag["corrupt_bucket_tiles"] == 0, diag


# ---------------------------------------------------------------------------
# Larger grids at a feature-map size: the generic kernels, a filing window
# shaped by the grad_value tile height, and filing in chunks of points
# ---------------------------------------------------------------------------

LARGE_GRIDS = [
    dict(name="k5x5_f16", k=5, dtype="f16", remove_center=0, softmax=0),
    dict(name="k7x7_bf16_rc", k=7, dtype="bf16", remove_center=1, softmax=0),
    dict(name="k5x5_bf16_softmax", k=5, dtype="bf16", remove_center=0, softmax=1),
    dict(name="k5x5_f32", k=5, dtype="f32", remove_center=0, softmax=0),
]


@pytest.mark.parametrize("spec", LARGE_GRIDS, ids=[s["name"] for s in LARGE_GRIDS])
def test_large_grid_forward_backward(spec):
    k = spec["k"]
    K = k * k - spec["remove_center"]
    P = -(-4 * 3 * K // 8) * 8
    w = gen.custom(name=spec["name"], N=2, H=40, W=48, G=4, Cg=16, Ho=40, Wo=48, K=K, P=P, dtype=spec["dtype"],
                   kh=k, kw=k, ph=k // 2, pw=k // 2, remove_center=spec["remove_center"], softmax=spec["softmax"])
    inp = gen.make_inputs(w)
    _check_forward(w, inp)
    _check_backward(w, inp)



def test_worked_example_2x2_exact():
    """The hand-derived worked example (tests/golden) in fp32 through the C ABI: every
    value is dyadic, so the kernels must reproduce it exactly."""
    import torch
    import _golden
    import deformable_convolution_sampling_b200 as dcn
    ex = _golden.load()
    p = dcn.make_params(dtype="f32", **_golden.GEOMETRY)
    t = {k: torch.from_numpy(ex[k].astype(np.float32)).cuda() for k in ("value", "offset_mask", "grad_out")}
    y = dcn.forward(p, t["value"], t["offset_mask"])
    gv, gom = dcn.backward(p, t["value"], t["offset_mask"], t["grad_out"])
    torch.cuda.synchronize()
    assert np.array_equal(to_f64(y), ex["y"])
    assert np.array_equal(to_f64(gom), ex["grad_offset_mask"])
    assert np.array_equal(to_f64(gv), ex["grad_value"])


def test_location_rounded_once_on_the_gpu():
    """The kernels form s*dy + anchor with one fp32 rounding (fmaf): on the case where
    two roundings would move the sample to the next cell row, grad_offset and
    grad_value match the hand-derived values of the single rounding exactly
    (1x1 grid on a 4 x 1 image; the same constants as the oracle pin)."""
    import torch
    import deformable_convolution_sampling_b200 as dcn
    s, dy = 10066330 * 2.0 ** -25, -13981013 * 2.0 ** -21
    lh = 1.0 - 2.0 ** -24
    p = dcn.make_params(N=1, H=4, W=1, G=1, Cg=4, kh=1, kw=1, ph=0, pw=0, offset_scale=s, dtype="f32", P=8)
    value = torch.tensor([1.0, 2.0, 10.0, 0.0], dtype=torch.float32).repeat_interleave(4).view(1, 4, 1, 4).cuda()
    om = torch.zeros((1, 4, 1, 8), dtype=torch.float32)
    om[..., 2] = 1.0
    om[0, 3, 0, 1] = dy
    om = om.cuda()
    gy = torch.zeros((1, 4, 1, 4), dtype=torch.float32)
    gy[0, 3, 0, 0] = 1.0                               # <gy, v> = channel 0 of v
    gy = gy.cuda()
    y = dcn.forward(p, value, om)
    gv, gom = dcn.backward(p, value, om, gy)
    torch.cuda.synchronize()
    assert np.all(to_f64(y)[0, 3, 0] == np.float32((1.0 - lh) + lh * 2.0))
    g = to_f64(gom)[0, 3, 0]
    assert g[1] == np.float32(s * 1.0) and g[0] == np.float32(s * -(1.0 + lh))
    assert np.array_equal(to_f64(gv)[0, :, 0, 0], np.float32([1.0 - lh, lh, 0.0, 0.0]).astype(np.float64))
