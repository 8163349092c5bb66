"""Pins of the CPU oracle against things other than itself (CPU only).

The pages print no worked numeric example, so the oracle is pinned by:
  * library routines that compute special cases of the operator on the host
    (grouped conv2d, grid_sample, torchvision's deform_conv2d);
  * exact special cases (integer offsets are plain gathers, far-off-image
    samples are zero, remove_center is a zero centre mask, offset_scale only
    scales the offsets);
  * identities the mathematics fixes (linearity in value and mask, the
    adjoint identity for grad_value, <grad_mask, m> = <grad_out, y>);
  * central finite differences for grad_offset / grad_mask.

The operator is the DCNv3 aggregation of the CSDN summary of "Efficient
Deformable ConvNets" (section 1.2 equation) without the softmax (section 2.1),
sampled bilinearly (section 2.2), with offset_scale / remove_center from the
DCNv4 module signature on the mhpn.cn architecture page.
"""
import math

import dataclasses

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import dcn4_inputs as gen
import oracle

torch.set_default_dtype(torch.float64)


def rand_problem_inputs(prob: oracle.Problem, seed: int, offset=("uniform", -2.0, 2.0),
                        mask=("normal", 0.0, 1.0)):
    Ho, Wo = oracle.output_dims(prob)
    w = gen.custom(N=prob.N, H=prob.H, W=prob.W, G=prob.G, Cg=prob.Cg, Ho=Ho, Wo=Wo, K=prob.K,
                   P=prob.row, dtype=prob.dtype, offset=offset, mask=mask)
    return gen.make_inputs(w, seed=seed), Ho, Wo


def split_om(om: np.ndarray, G: int, K: int):
    """offset_mask rows -> (dx [..,G,K], dy [..,G,K], m [..,G,K]) as float64 views of storage."""
    body = om[..., : G * 3 * K].reshape(om.shape[:-1] + (G, 3 * K))
    pairs = body[..., : 2 * K].reshape(om.shape[:-1] + (G, K, 2))
    return pairs[..., 0], pairs[..., 1], body[..., 2 * K:]


def cells(kh, kw, remove_center):
    """Grid cells (ih, iw) in k order: columns outer, rows inner, centre optionally dropped."""
    out = []
    for iw in range(kw):
        for ih in range(kh):
            if remove_center and ih == kh // 2 and iw == kw // 2:
                continue
            out.append((ih, iw))
    return out


def rel_err(a, b):
    scale = max(np.max(np.abs(b)), 1e-300)
    return np.max(np.abs(a - b)) / scale


GEOMS = [
    dict(kh=3, kw=3, sh=1, sw=1, ph=1, pw=1, dh=1, dw=1),
    dict(kh=3, kw=3, sh=2, sw=1, ph=0, pw=2, dh=1, dw=2),
    dict(kh=3, kw=5, sh=1, sw=2, ph=2, pw=1, dh=2, dw=1),
    dict(kh=1, kw=3, sh=1, sw=1, ph=0, pw=1, dh=1, dw=1),
]


# ---------------------------------------------------------------------------
# Decoders
# ---------------------------------------------------------------------------

def test_decode_f16_all_patterns():
    bits = np.arange(1 << 16, dtype=np.uint16)
    got = oracle.decode("f16", bits.view(np.float16))
    want = bits.view(np.float16).astype(np.float64)
    np.testing.assert_array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    np.testing.assert_array_equal(got[ok], want[ok])


def test_decode_bf16_all_patterns():
    bits = np.arange(1 << 16, dtype=np.uint16)
    got = oracle.decode("bf16", bits)
    want = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    np.testing.assert_array_equal(got[ok], want[ok])


# ---------------------------------------------------------------------------
# Geometry: zero offsets + per-(g,k) constant mask == grouped convolution
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("geom", GEOMS)
@pytest.mark.parametrize("remove_center", [0, 1])
def test_zero_offsets_equal_grouped_conv(geom, remove_center):
    if remove_center and (geom["kh"] % 2 == 0 or geom["kw"] % 2 == 0):
        pytest.skip("remove_center needs odd kernels")
    prob = oracle.Problem(N=2, H=7, W=9, G=3, Cg=2, remove_center=remove_center, dtype="f64", **geom)
    inp, Ho, Wo = rand_problem_inputs(prob, seed=11)
    K = prob.K
    rng = np.random.default_rng(3)
    wk = rng.normal(size=(prob.G, K))                 # one weight per (group, grid point)
    om = inp["offset_mask"]
    dx, dy, m = split_om(om, prob.G, K)
    dx[...] = 0.0
    dy[...] = 0.0
    m[...] = wk                                        # broadcast over pixels
    y = oracle.forward(prob, inp["value"], om)

    # depthwise conv2d weight [C, 1, kh, kw]: channel c of group g gets wk[g, k(ih, iw)]
    weight = np.zeros((prob.C, 1, prob.kh, prob.kw))
    for k, (ih, iw) in enumerate(cells(prob.kh, prob.kw, remove_center)):
        for g in range(prob.G):
            weight[g * prob.Cg:(g + 1) * prob.Cg, 0, ih, iw] = wk[g, k]
    x = torch.from_numpy(inp["value"]).permute(0, 3, 1, 2)
    ref = F.conv2d(x, torch.from_numpy(weight), stride=(prob.sh, prob.sw), padding=(prob.ph, prob.pw),
                   dilation=(prob.dh, prob.dw), groups=prob.C).permute(0, 2, 3, 1).numpy()
    assert ref.shape == y.shape
    assert rel_err(y, ref) < 1e-13


def test_output_dims_match_conv2d():
    for geom in GEOMS:
        for H, W in [(5, 6), (8, 8), (13, 4)]:
            prob = oracle.Problem(N=1, H=H, W=W, G=1, Cg=1, dtype="f64", **geom)
            x = torch.zeros(1, 1, H, W)
            try:
                ref = F.conv2d(x, torch.zeros(1, 1, prob.kh, prob.kw), stride=(prob.sh, prob.sw),
                               padding=(prob.ph, prob.pw), dilation=(prob.dh, prob.dw)).shape[2:]
            except RuntimeError:
                continue
            assert oracle.output_dims(prob) == tuple(ref)


# ---------------------------------------------------------------------------
# Integer offsets: exact shifted gathers
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("geom", GEOMS[:3])
def test_integer_offsets_exact_gather(geom):
    prob = oracle.Problem(N=2, H=6, W=7, G=2, Cg=3, dtype="f32", **geom)
    inp, Ho, Wo = rand_problem_inputs(prob, seed=5)
    K = prob.K
    om = inp["offset_mask"]
    dx, dy, m = split_om(om, prob.G, K)
    rng = np.random.default_rng(9)
    dx[...] = rng.integers(-3, 4, size=dx.shape).astype(np.float32)
    dy[...] = rng.integers(-3, 4, size=dy.shape).astype(np.float32)
    y = oracle.forward(prob, inp["value"], om)

    x = inp["value"].astype(np.float64)
    want = np.zeros_like(y)
    for n in range(prob.N):
        for ho in range(Ho):
            for wo in range(Wo):
                for g in range(prob.G):
                    for k, (ih, iw) in enumerate(cells(prob.kh, prob.kw, 0)):
                        yy = ho * prob.sh - prob.ph + ih * prob.dh + int(dy[n, ho, wo, g, k])
                        xx = wo * prob.sw - prob.pw + iw * prob.dw + int(dx[n, ho, wo, g, k])
                        if 0 <= yy < prob.H and 0 <= xx < prob.W:
                            sl = slice(g * prob.Cg, (g + 1) * prob.Cg)
                            want[n, ho, wo, sl] += float(m[n, ho, wo, g, k]) * x[n, yy, xx, sl]
    np.testing.assert_array_equal(y, want)


# ---------------------------------------------------------------------------
# Bilinear sampling + zero padding == grid_sample(align_corners=True, zeros)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("offset", [("uniform", -2.0, 2.0), ("uniform", -6.0, 6.0)])
def test_single_point_matches_grid_sample(offset):
    prob = oracle.Problem(N=2, H=6, W=8, G=2, Cg=3, dtype="f64", offset_scale=0.75)
    inp, Ho, Wo = rand_problem_inputs(prob, seed=21, offset=offset)
    K = prob.K
    om0 = inp["offset_mask"]
    for k, (ih, iw) in enumerate(cells(3, 3, 0)):
        om = om0.copy()
        dx, dy, m = split_om(om, prob.G, K)
        m[...] = 0.0
        m[..., k] = 1.0
        y = oracle.forward(prob, inp["value"], om)
        ho = np.arange(Ho)[:, None]
        wo = np.arange(Wo)[None, :]
        for g in range(prob.G):
            h = (ho * prob.sh - prob.ph + ih * prob.dh) + prob.offset_scale * dy[..., g, k]
            w = (wo * prob.sw - prob.pw + iw * prob.dw) + prob.offset_scale * dx[..., g, k]
            grid = np.stack([2.0 * w / (prob.W - 1) - 1.0, 2.0 * h / (prob.H - 1) - 1.0], axis=-1)
            x = torch.from_numpy(inp["value"][..., g * prob.Cg:(g + 1) * prob.Cg]).permute(0, 3, 1, 2)
            ref = F.grid_sample(x, torch.from_numpy(grid), mode="bilinear", padding_mode="zeros",
                                align_corners=True).permute(0, 2, 3, 1).numpy()
            got = y[..., g * prob.Cg:(g + 1) * prob.Cg]
            assert rel_err(got, ref) < 1e-12


# ---------------------------------------------------------------------------
# Whole operator == torchvision.ops.deform_conv2d with a depthwise all-ones weight
# ---------------------------------------------------------------------------

def _torchvision():
    tv = pytest.importorskip("torchvision")
    return tv.ops.deform_conv2d


def test_torchvision_offset_layout_probe():
    """torchvision's offset channels per kernel position are (row shift, column shift), row-major."""
    deform_conv2d = _torchvision()
    H = W = 5
    ramp_h = torch.arange(H, dtype=torch.float64)[:, None].expand(H, W).reshape(1, 1, H, W)
    ramp_w = torch.arange(W, dtype=torch.float64)[None, :].expand(H, W).reshape(1, 1, H, W)
    weight = torch.zeros(1, 1, 3, 3)
    weight[0, 0, 0, 1] = 1.0                         # kernel position (i=0, j=1) -> index 1
    off = torch.zeros(1, 18, H, W)
    off[0, 2 * 1] = 0.5                              # first channel of position 1
    a = deform_conv2d(ramp_h, off, weight, padding=1)
    b = deform_conv2d(ramp_h, torch.zeros_like(off), weight, padding=1)
    assert torch.allclose((a - b)[0, 0, 2, 2], torch.tensor(0.5))   # moved along rows
    c = deform_conv2d(ramp_w, off, weight, padding=1)
    d = deform_conv2d(ramp_w, torch.zeros_like(off), weight, padding=1)
    assert torch.allclose((c - d)[0, 0, 2, 2], torch.tensor(0.0))


@pytest.mark.parametrize("geom", GEOMS)
@pytest.mark.parametrize("remove_center,scale", [(0, 1.0), (1, 0.5), (0, 1.7)])
def test_matches_torchvision_deform_conv2d(geom, remove_center, scale):
    deform_conv2d = _torchvision()
    if remove_center and (geom["kh"] % 2 == 0 or geom["kw"] % 2 == 0):
        pytest.skip("remove_center needs odd kernels")
    prob = oracle.Problem(N=2, H=9, W=7, G=3, Cg=2, dtype="f64", offset_scale=scale,
                          remove_center=remove_center, **geom)
    inp, Ho, Wo = rand_problem_inputs(prob, seed=31, offset=("normal", 0.0, 2.0))
    y = oracle.forward(prob, inp["value"], inp["offset_mask"])
    dx, dy, m = split_om(inp["offset_mask"], prob.G, prob.K)
    kh, kw = prob.kh, prob.kw
    off_tv = np.zeros((prob.N, prob.G, kh * kw, 2, Ho, Wo))
    mask_tv = np.zeros((prob.N, prob.G, kh * kw, Ho, Wo))
    for k, (ih, iw) in enumerate(cells(kh, kw, remove_center)):
        j = ih * kw + iw
        off_tv[:, :, j, 0] = np.moveaxis(scale * dy[..., k], 3, 1)
        off_tv[:, :, j, 1] = np.moveaxis(scale * dx[..., k], 3, 1)
        mask_tv[:, :, j] = np.moveaxis(m[..., k], 3, 1)
    x = torch.from_numpy(inp["value"]).permute(0, 3, 1, 2).contiguous()
    ref = deform_conv2d(x, torch.from_numpy(off_tv.reshape(prob.N, -1, Ho, Wo)),
                        torch.ones(prob.C, 1, kh, kw), stride=(prob.sh, prob.sw),
                        padding=(prob.ph, prob.pw), dilation=(prob.dh, prob.dw),
                        mask=torch.from_numpy(mask_tv.reshape(prob.N, -1, Ho, Wo)))
    ref = ref.permute(0, 2, 3, 1).numpy()
    assert rel_err(y, ref) < 1e-12


# ---------------------------------------------------------------------------
# Structural identities and special cases
# ---------------------------------------------------------------------------

def _tiny(dtype="f64", **kw):
    base = dict(N=2, H=6, W=5, G=2, Cg=3, dtype=dtype)
    base.update(kw)
    return oracle.Problem(**base)


def test_linear_in_value_and_mask():
    prob = _tiny()
    a, Ho, Wo = rand_problem_inputs(prob, seed=1)
    b, _, _ = rand_problem_inputs(prob, seed=2)
    y1 = oracle.forward(prob, a["value"], a["offset_mask"])
    y2 = oracle.forward(prob, b["value"], a["offset_mask"])
    y12 = oracle.forward(prob, 2.5 * a["value"] - 0.75 * b["value"], a["offset_mask"])
    assert rel_err(y12, 2.5 * y1 - 0.75 * y2) < 1e-13
    om2 = a["offset_mask"].copy()
    _, _, m2 = split_om(om2, prob.G, prob.K)
    _, _, m1 = split_om(b["offset_mask"], prob.G, prob.K)
    om_sum = a["offset_mask"].copy()
    _, _, ms = split_om(om_sum, prob.G, prob.K)
    ms[...] = 3.0 * m2 + m1
    om_b = a["offset_mask"].copy()
    _, _, mb = split_om(om_b, prob.G, prob.K)
    mb[...] = m1
    ya = oracle.forward(prob, a["value"], a["offset_mask"])
    yb = oracle.forward(prob, a["value"], om_b)
    ys = oracle.forward(prob, a["value"], om_sum)
    assert rel_err(ys, 3.0 * ya + yb) < 1e-13


def test_remove_center_is_zero_centre_mask():
    p8 = _tiny(remove_center=1)
    p9 = _tiny(remove_center=0)
    inp, Ho, Wo = rand_problem_inputs(p8, seed=4)
    dx8, dy8, m8 = split_om(inp["offset_mask"], p8.G, 8)
    om9 = np.full(inp["offset_mask"].shape[:-1] + (p9.row,), np.nan)
    dx9, dy9, m9 = split_om(om9, p9.G, 9)
    order9 = cells(3, 3, 0)
    order8 = cells(3, 3, 1)
    for k8, c in enumerate(order8):
        k9 = order9.index(c)
        dx9[..., k9], dy9[..., k9], m9[..., k9] = dx8[..., k8], dy8[..., k8], m8[..., k8]
    kc = order9.index((1, 1))
    dx9[..., kc], dy9[..., kc], m9[..., kc] = 0.3, -0.2, 0.0
    y8 = oracle.forward(p8, inp["value"], inp["offset_mask"])
    y9 = oracle.forward(p9, inp["value"], om9)
    np.testing.assert_array_equal(y8, y9)


def test_offset_scale_scales_offsets_only():
    p_half = _tiny(offset_scale=0.5)
    p_one = _tiny(offset_scale=1.0)
    inp, Ho, Wo = rand_problem_inputs(p_half, seed=6, offset=("normal", 0.0, 2.0))
    om_scaled = inp["offset_mask"].copy()
    dx, dy, _ = split_om(om_scaled, p_half.G, p_half.K)
    dx *= 0.5
    dy *= 0.5
    np.testing.assert_array_equal(oracle.forward(p_half, inp["value"], inp["offset_mask"]),
                                  oracle.forward(p_one, inp["value"], om_scaled))
    p_odd = _tiny(offset_scale=0.3)
    om_odd = inp["offset_mask"].copy()
    dx, dy, _ = split_om(om_odd, p_odd.G, p_odd.K)
    dx *= 0.3
    dy *= 0.3
    assert rel_err(oracle.forward(p_odd, inp["value"], inp["offset_mask"]),
                   oracle.forward(p_one, inp["value"], om_odd)) < 1e-13


def test_far_off_image_is_zero():
    prob = _tiny()
    inp, Ho, Wo = rand_problem_inputs(prob, seed=8)
    gy = inp["grad_out"]
    for far in (1e3, -1e3, 7.0, -2.0 - 1e-9 - 8.0):
        om = inp["offset_mask"].copy()
        dx, dy, _ = split_om(om, prob.G, prob.K)
        dy[...] = far
        y = oracle.forward(prob, inp["value"], om)
        assert np.all(y == 0.0)
        gv, gom = oracle.backward(prob, inp["value"], om, gy)
        assert np.all(gv == 0.0) and np.all(gom == 0.0)


def test_padding_tail_ignored_and_zeroed():
    prob = _tiny(P=48)                                 # G*3K = 54 -> force a bigger row
    prob = _tiny(P=64)
    inp, Ho, Wo = rand_problem_inputs(prob, seed=12)
    om_nan = inp["offset_mask"]
    assert np.all(np.isnan(om_nan[..., prob.G * 3 * prob.K:]))
    om_zero = om_nan.copy()
    om_zero[..., prob.G * 3 * prob.K:] = 0.0
    y_nan = oracle.forward(prob, inp["value"], om_nan)
    assert np.all(np.isfinite(y_nan))
    np.testing.assert_array_equal(y_nan, oracle.forward(prob, inp["value"], om_zero))
    gv, gom = oracle.backward(prob, inp["value"], om_nan, inp["grad_out"])
    assert np.all(gom[..., prob.G * 3 * prob.K:] == 0.0)
    assert np.all(np.isfinite(gv)) and np.all(np.isfinite(gom))


def test_storage_types_agree_on_representable_inputs():
    """The same numbers stored as f16 / bf16 / f32 / f64 give the same result."""
    p64 = _tiny()
    inp, Ho, Wo = rand_problem_inputs(p64, seed=13)
    v = gen.bf16_bits_to_f64(gen.f64_to_bf16_bits(inp["value"]))          # bf16-representable
    om = inp["offset_mask"].copy()
    om = np.where(np.isnan(om), 0.0, om)
    om = np.round(om * 64.0) / 64.0                                           # exact in all 4 types
    y64 = oracle.forward(p64, v, om)
    for dt in ("f32", "f16", "bf16"):
        p = _tiny(dtype=dt)
        y = oracle.forward(p, gen.to_storage(v, dt), gen.to_storage(om, dt))
        np.testing.assert_array_equal(y, y64)


def test_location_fp32_mode():
    prob = _tiny(dtype="f32", offset_scale=0.7)
    inp, Ho, Wo = rand_problem_inputs(prob, seed=14)
    y64 = oracle.forward(prob, inp["value"], inp["offset_mask"])
    prob32 = _tiny(dtype="f32", offset_scale=0.7, location_fp32=True)
    y32 = oracle.forward(prob32, inp["value"], inp["offset_mask"])
    assert 0.0 < rel_err(y32, y64) < 1e-6
    # integer offsets with a power-of-two scale: locations exact in both modes
    om = inp["offset_mask"].copy()
    dx, dy, _ = split_om(om, prob.G, prob.K)
    dx[...] = np.round(dx)
    dy[...] = np.round(dy)
    pa = _tiny(dtype="f32", offset_scale=0.5)
    pb = _tiny(dtype="f32", offset_scale=0.5, location_fp32=True)
    np.testing.assert_array_equal(oracle.forward(pa, inp["value"], om), oracle.forward(pb, inp["value"], om))


# One location where a single rounding of s*dy + base and two roundings
# (the product rounded to fp32 first, then the sum) pick different cells.
# fp32 constants, checked below: s = fl(0.3) = 10066330 * 2^-25 and
# dy = -13981013 * 2^-21 (= -6.6666665077...); their exact product is
# -2.0000000317891... .  With base 3 the exact sum 0.99999996821... lies
# closer to 1 - 2^-24 than to 1, so fmaf gives h = 1 - 2^-24 (cell row 0,
# lh = 1 - 2^-24); fl(s*dy) = -2 exactly, and -2 + 3 = 1 puts h on row 1.
FUSED_S = 10066330 * 2.0 ** -25
FUSED_DY = -13981013 * 2.0 ** -21


def _fused_location_case():
    """1x1 grid on a 4 x 1 image, one group of one channel; output pixel 3 (anchor
    row 3) samples at 3 + s*dy, every other pixel at its own anchor.  value rows
    1, 2, 10, 0; grad_out 1 at pixel 3 only; masks 1."""
    prob = oracle.Problem(N=1, H=4, W=1, G=1, Cg=1, kh=1, kw=1, ph=0, pw=0, offset_scale=FUSED_S,
                          dtype="f32", P=8, location_fp32=True)
    value = np.array([1.0, 2.0, 10.0, 0.0], dtype=np.float32).reshape(1, 4, 1, 1)
    om = np.zeros((1, 4, 1, 8), dtype=np.float32)
    om[..., 2] = 1.0                                   # the mask of every pixel
    om[0, 3, 0, 1] = FUSED_DY                          # dy of pixel 3
    gy = np.zeros((1, 4, 1, 1), dtype=np.float32)
    gy[0, 3] = 1.0
    return prob, value, om, gy


def test_location_is_one_fused_rounding():
    """The fp32 location mode rounds s*dy + base once (fmaf), as the kernels do."""
    assert np.float32(0.3) == np.float32(FUSED_S) and float(np.float32(FUSED_S)) == FUSED_S
    assert float(np.float32(FUSED_DY)) == FUSED_DY
    exact = FUSED_S * FUSED_DY + 3.0                   # exact in float64 (24 x 24 bits)
    assert 1.0 - 2.0 ** -24 < exact < 1.0 - 2.0 ** -25  # rounds down to 1 - 2^-24 in fp32
    assert float(np.float32(FUSED_S * FUSED_DY)) == -2.0
    prob, value, om, gy = _fused_location_case()
    lh = 1.0 - 2.0 ** -24                              # h = 1 - 2^-24: cell rows 0 and 1
    y = oracle.forward(prob, value, om)
    assert y[0, 3, 0, 0] == (1.0 - lh) * 1.0 + lh * 2.0
    assert y[0, 0, 0, 0] == 1.0 and y[0, 1, 0, 0] == 2.0 and y[0, 2, 0, 0] == 10.0
    gv, gom = oracle.backward(prob, value, om, gy)
    # d/d dy = s * m * <gy, dS/dh>, dS/dh = v[row 1] - v[row 0] on this cell (lw = 0)
    assert gom[0, 3, 0, 1] == FUSED_S * (2.0 - 1.0)
    # d/d dx: dS/dw = (1 - lh)(0 - v[row 0]) + lh (0 - v[row 1]) (the right corners are off the image)
    assert gom[0, 3, 0, 0] == FUSED_S * -(1.0 + lh)
    assert gom[0, 3, 0, 2] == (1.0 - lh) * 1.0 + lh * 2.0
    np.testing.assert_array_equal(gv[0, :, 0, 0], [1.0 - lh, lh, 0.0, 0.0])


def test_threads_do_not_change_results():
    prob = _tiny(N=3)
    inp, Ho, Wo = rand_problem_inputs(prob, seed=15)
    y1 = oracle.forward(prob, inp["value"], inp["offset_mask"], nthreads=1)
    y4 = oracle.forward(prob, inp["value"], inp["offset_mask"], nthreads=4)
    np.testing.assert_array_equal(y1, y4)
    g1 = oracle.backward(prob, inp["value"], inp["offset_mask"], inp["grad_out"], nthreads=1)
    g3 = oracle.backward(prob, inp["value"], inp["offset_mask"], inp["grad_out"], nthreads=3)
    for a, b in zip(g1, g3):
        np.testing.assert_array_equal(a, b)


# ---------------------------------------------------------------------------
# Backward
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("geom", GEOMS[:3])
def test_grad_value_is_adjoint(geom):
    prob = oracle.Problem(N=2, H=7, W=6, G=2, Cg=3, dtype="f64", offset_scale=0.8, **geom)
    inp, Ho, Wo = rand_problem_inputs(prob, seed=17, offset=("normal", 0.0, 2.0))
    rng = np.random.default_rng(0)
    v2 = rng.normal(size=inp["value"].shape)
    gy = inp["grad_out"]
    gv, _ = oracle.backward(prob, inp["value"], inp["offset_mask"], gy)
    lhs = np.sum(gy * oracle.forward(prob, v2, inp["offset_mask"]))
    rhs = np.sum(gv * v2)
    assert abs(lhs - rhs) <= 1e-12 * (np.sum(np.abs(gy)) * np.max(np.abs(v2)))
    # grad_value does not depend on value (the operator is linear in value)
    gv2, _ = oracle.backward(prob, v2, inp["offset_mask"], gy)
    np.testing.assert_array_equal(gv, gv2)


def test_grad_mask_identities():
    prob = _tiny(remove_center=1, offset_scale=0.5)
    inp, Ho, Wo = rand_problem_inputs(prob, seed=19)
    gy = inp["grad_out"]
    om = inp["offset_mask"]
    y = oracle.forward(prob, inp["value"], om)
    _, gom = oracle.backward(prob, inp["value"], om, gy)
    _, _, m = split_om(om, prob.G, prob.K)
    _, _, gm = split_om(gom, prob.G, prob.K)
    assert abs(np.sum(gm * m) - np.sum(gy * y)) < 1e-12 * np.sum(np.abs(gy * y))
    # elementwise: gm[k] = sum_c gy * S_k with S_k from a one-hot mask
    C = prob.C
    for k in range(prob.K):
        om_k = om.copy()
        _, _, mk = split_om(om_k, prob.G, prob.K)
        mk[...] = 0.0
        mk[..., k] = 1.0
        S = oracle.forward(prob, inp["value"], om_k).reshape(prob.N, Ho, Wo, prob.G, prob.Cg)
        want = np.sum(gy.reshape(prob.N, Ho, Wo, prob.G, prob.Cg) * S, axis=-1)
        assert rel_err(gm[..., k], want) < 1e-13
    assert C == prob.G * prob.Cg


@pytest.mark.parametrize("scale,remove_center", [(1.0, 0), (0.5, 1), (1.3, 0)])
def test_grad_offset_mask_finite_differences(scale, remove_center):
    prob = oracle.Problem(N=1, H=8, W=8, G=2, Cg=4, dtype="f64", offset_scale=scale,
                          remove_center=remove_center)
    inp, Ho, Wo = rand_problem_inputs(prob, seed=23)
    om = inp["offset_mask"].copy()
    om[..., prob.G * 3 * prob.K:] = 0.0
    dx, dy, _ = split_om(om, prob.G, prob.K)
    # keep every location >= 1e-3 away from an integer (a cell boundary)
    for d in (dx, dy):
        frac = np.mod(scale * d, 1.0)
        bad = (frac < 1e-3) | (frac > 1 - 1e-3)
        d[bad] += 0.01
    gy = inp["grad_out"]
    _, gom = oracle.backward(prob, inp["value"], om, gy)
    eps = 1e-6
    G, K, Cg = prob.G, prob.K, prob.Cg
    body = G * 3 * K
    for e in range(3 * K):
        plus, minus = om.copy(), om.copy()
        idx = np.arange(G) * 3 * K + e
        plus[..., idx] += eps
        minus[..., idx] -= eps
        yp = oracle.forward(prob, inp["value"], plus).reshape(1, Ho, Wo, G, Cg)
        ym = oracle.forward(prob, inp["value"], minus).reshape(1, Ho, Wo, G, Cg)
        fd = np.sum(gy.reshape(1, Ho, Wo, G, Cg) * (yp - ym), axis=-1) / (2 * eps)
        got = gom[..., idx]
        scale_ref = max(np.max(np.abs(gom[..., :body])), 1e-12)
        assert np.max(np.abs(got - fd)) / scale_ref < 1e-6, f"entry {e}"


def test_grad_offset_zero_offsets_at_border_uses_floor_cell():
    """At an integer location the derivative is the one of the cell floor() picks."""
    prob = oracle.Problem(N=1, H=4, W=4, G=1, Cg=1, dtype="f64")
    value = np.arange(16, dtype=np.float64).reshape(1, 4, 4, 1) + 1.0
    Ho, Wo = oracle.output_dims(prob)
    om = np.zeros((1, Ho, Wo, prob.row))
    _, _, m = split_om(om, 1, 9)
    m[...] = 1.0
    gy = np.zeros((1, Ho, Wo, 1))
    gy[0, 0, 0, 0] = 1.0
    _, gom = oracle.backward(prob, value, om, gy)
    dxg, dyg, _ = split_om(gom, 1, 9)
    # k = 0 is cell (ih=0, iw=0): location (-1, -1); floor cell rows {-1, 0}, cols {-1, 0}
    # dS/dh = (1-lw)(v10 - v00) + lw(v11 - v01) with lw = 0 -> v[0,-1] - v[-1,-1] = 0 (col -1 is outside)
    assert dyg[0, 0, 0, 0, 0] == 0.0 and dxg[0, 0, 0, 0, 0] == 0.0
    # k = 1 is cell (ih=1, iw=0): location (0, -1): dS/dw = (1-lh)(v01 - v00) = v[0,0] - 0 = 1
    assert dxg[0, 0, 0, 0, 1] == 1.0
    # dS/dh = (1-lw)(v10 - v00) = v[1,-1] - v[0,-1] = 0 (column -1 is outside)
    assert dyg[0, 0, 0, 0, 1] == 0.0
    # k = 4 is the centre (1, 1): location (0, 0): dS/dh = v[1,0]-v[0,0] = 4, dS/dw = v[0,1]-v[0,0] = 1
    assert dyg[0, 0, 0, 0, 4] == 4.0 and dxg[0, 0, 0, 0, 4] == 1.0
    assert math.isfinite(float(np.sum(gom)))


# ---------------------------------------------------------------------------
# Softmax variant (DCNv3 normalisation of the K masks of each (pixel, group))
# ---------------------------------------------------------------------------

def _softmax_problem(**kw):
    return oracle.Problem(**{**dict(N=2, H=7, W=9, G=2, Cg=3, dtype="f64"), **kw})


def _set_logits(om, prob, fn):
    """Replace the masks of every (pixel, group) by fn(shape) (in place)."""
    _, _, m = split_om(om, prob.G, prob.K)
    m[...] = fn(m.shape)
    return om


def test_softmax_shift_invariance():
    """Adding one constant to the K logits of a (pixel, group) changes nothing."""
    prob = _softmax_problem(softmax=True)
    inp, Ho, Wo = rand_problem_inputs(prob, seed=41)
    om = inp["offset_mask"].copy()
    y0 = oracle.forward(prob, inp["value"], om)
    _, _, m = split_om(om, prob.G, prob.K)
    m += np.random.default_rng(5).uniform(-30, 30, size=m.shape[:-1] + (1,))
    y1 = oracle.forward(prob, inp["value"], om)
    assert rel_err(y1, y0) < 1e-12


def test_softmax_equal_logits_average_the_points():
    """Equal logits weigh every point 1/K: the plain operator with mask 1/K."""
    prob = _softmax_problem(softmax=True, remove_center=1)
    inp, Ho, Wo = rand_problem_inputs(prob, seed=42)
    om_sm = _set_logits(inp["offset_mask"].copy(), prob,
                        lambda sh: np.repeat(np.random.default_rng(6).normal(size=sh[:-1] + (1,)), sh[-1], -1))
    om_plain = _set_logits(inp["offset_mask"].copy(), prob, lambda sh: np.full(sh, 1.0 / prob.K))
    y_sm = oracle.forward(prob, inp["value"], om_sm)
    y_plain = oracle.forward(dataclasses.replace(prob, softmax=False), inp["value"], om_plain)
    assert rel_err(y_sm, y_plain) < 1e-13


def test_softmax_dominant_logit_selects_its_point():
    """Logits +800 at point j and -800 elsewhere weigh point j by exactly 1 (this
    also needs the largest logit subtracted before exp, or exp overflows)."""
    prob = _softmax_problem(softmax=True)
    inp, Ho, Wo = rand_problem_inputs(prob, seed=43)
    rng = np.random.default_rng(7)
    j = rng.integers(0, prob.K, size=(prob.N, Ho, Wo, prob.G))
    onehot = np.eye(prob.K)[j]
    om_sm = _set_logits(inp["offset_mask"].copy(), prob, lambda sh: 1600.0 * onehot - 800.0)
    om_plain = _set_logits(inp["offset_mask"].copy(), prob, lambda sh: onehot)
    y_sm = oracle.forward(prob, inp["value"], om_sm)
    y_plain = oracle.forward(dataclasses.replace(prob, softmax=False), inp["value"], om_plain)
    assert np.all(np.isfinite(y_sm))
    assert rel_err(y_sm, y_plain) < 1e-15


def test_softmax_logit_gradients_sum_to_zero():
    """The softmax is invariant to a common shift, so the logit gradients of each
    (pixel, group) sum to zero, while the samples' own gradients do not."""
    prob = _softmax_problem(softmax=True)
    inp, Ho, Wo = rand_problem_inputs(prob, seed=44)
    _, gom = oracle.backward(prob, inp["value"], inp["offset_mask"], inp["grad_out"])
    _, _, gm = split_om(gom, prob.G, prob.K)
    scale = np.max(np.abs(gm))
    assert scale > 1e-3
    assert np.max(np.abs(gm.sum(-1))) < 1e-12 * scale * prob.K


@pytest.mark.parametrize("remove_center", [0, 1])
def test_softmax_backward_finite_differences(remove_center):
    """Offsets and logits: central differences of the softmax forward."""
    prob = oracle.Problem(N=1, H=8, W=8, G=2, Cg=4, dtype="f64", softmax=True, remove_center=remove_center,
                          offset_scale=0.7)
    inp, Ho, Wo = rand_problem_inputs(prob, seed=45)
    om = inp["offset_mask"].copy()
    om[..., prob.G * 3 * prob.K:] = 0.0
    dx, dy, _ = split_om(om, prob.G, prob.K)
    for d in (dx, dy):
        frac = np.mod(prob.offset_scale * d, 1.0)
        bad = (frac < 1e-3) | (frac > 1 - 1e-3)
        d[bad] += 0.01
    gy = inp["grad_out"]
    _, gom = oracle.backward(prob, inp["value"], om, gy)
    eps = 1e-6
    G, K, Cg = prob.G, prob.K, prob.Cg
    body = G * 3 * K
    scale_ref = max(np.max(np.abs(gom[..., :body])), 1e-12)
    for e in range(3 * K):
        plus, minus = om.copy(), om.copy()
        idx = np.arange(G) * 3 * K + e
        plus[..., idx] += eps
        minus[..., idx] -= eps
        yp = oracle.forward(prob, inp["value"], plus).reshape(1, Ho, Wo, G, Cg)
        ym = oracle.forward(prob, inp["value"], minus).reshape(1, Ho, Wo, G, Cg)
        fd = np.sum(gy.reshape(1, Ho, Wo, G, Cg) * (yp - ym), axis=-1) / (2 * eps)
        assert np.max(np.abs(gom[..., idx] - fd)) / scale_ref < 1e-6, f"entry {e}"


def test_softmax_grad_value_is_adjoint():
    """y is linear in value for fixed offsets and logits: <gy, y(v)> = <grad_value, v>."""
    prob = _softmax_problem(softmax=True)
    inp, Ho, Wo = rand_problem_inputs(prob, seed=46)
    y = oracle.forward(prob, inp["value"], inp["offset_mask"])
    gv, _ = oracle.backward(prob, inp["value"], inp["offset_mask"], inp["grad_out"])
    lhs = float(np.sum(inp["grad_out"] * y))
    rhs = float(np.sum(gv * inp["value"]))
    assert abs(lhs - rhs) <= 1e-12 * max(abs(lhs), 1.0)


# ---------------------------------------------------------------------------
# Rounding to storage and the merged offset/mask linear layer
# ---------------------------------------------------------------------------

def _lattice(fmt):
    """Every finite non-negative value of the 16-bit format with its bit pattern, ascending
    (decoded by numpy's own bit views, independent of the oracle's decoders)."""
    bits = np.arange(0, 0x8000, dtype=np.uint16)
    if fmt == "f16":
        vals = bits.view(np.float16).astype(np.float64)
    else:
        vals = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    keep = np.isfinite(vals)
    return vals[keep], bits[keep]


def _nearest_even(fmt, v):
    """Brute force: the nearest lattice value of |v| (ties: even pattern), with v's sign;
    beyond the largest finite value by half a unit or more: infinity."""
    vals, bits = _lattice(fmt)
    a = np.abs(v)
    i = np.clip(np.searchsorted(vals, a), 1, len(vals) - 1)
    lo, hi = vals[i - 1], vals[i]
    pick_hi = (a - lo > hi - a) | ((a - lo == hi - a) & (bits[i] % 2 == 0))
    out = np.where(pick_hi, bits[i], bits[i - 1]).astype(np.uint16)
    top = vals[-1]
    half_ulp = (vals[-1] - vals[-2]) / 2
    inf = np.uint16(0x7c00 if fmt == "f16" else 0x7f80)
    out = np.where(a >= top + half_ulp, inf, np.where(a > top, bits[-1], out))
    return (out | np.where(np.signbit(v), 0x8000, 0).astype(np.uint16)).astype(np.uint16)


@pytest.mark.parametrize("fmt", ["f16", "bf16"])
def test_encode_round_trips_every_finite_pattern(fmt):
    vals, bits = _lattice(fmt)
    for sign in (0, 0x8000):
        got = oracle.encode(fmt, vals if sign == 0 else -vals).view(np.uint16)
        want = bits | np.uint16(sign)
        same = got == want
        # -0.0 encodes as 0x8000, +0.0 as 0
        assert np.all(same), np.flatnonzero(~same)[:5]


@pytest.mark.parametrize("fmt", ["f16", "bf16"])
def test_encode_is_nearest_ties_to_even(fmt):
    """Midpoints between neighbouring values (exact ties), points just either side of
    them, random values over the whole range, subnormals and the overflow threshold."""
    vals, _ = _lattice(fmt)
    mids = (vals[:-1] + vals[1:]) / 2
    rng = np.random.default_rng(3)
    span = np.log2(vals[-1])
    v = np.concatenate([mids, np.nextafter(mids, 0), np.nextafter(mids, np.inf),
                        rng.uniform(-1, 1, 20000) * 2.0 ** rng.uniform(-30 if fmt == "f16" else -140, span, 20000),
                        [vals[-1] * 1.0001, vals[-1] + (vals[-1] - vals[-2]) / 2, 1e300, -1e300]])
    got = oracle.encode(fmt, v).view(np.uint16)
    assert np.array_equal(got, _nearest_even(fmt, v))
    if fmt == "f16":  # numpy's float64 -> float16 cast rounds the same way
        with np.errstate(over="ignore"):
            assert np.array_equal(got, v.astype(np.float16).view(np.uint16))


def test_encode_nan_and_f32():
    out = oracle.encode("f16", np.array([np.nan])).view(np.uint16)
    assert (out[0] & 0x7c00) == 0x7c00 and (out[0] & 0x3ff) != 0
    v = np.random.default_rng(4).normal(size=1000) * 1e3
    assert np.array_equal(oracle.encode("f32", v), v.astype(np.float32))


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("with_bias", [True, False])
def test_linear_is_the_rounded_affine_map(dtype, with_bias):
    """x @ W.T + b in float64 (numpy's matmul), rounded once to the storage format."""
    rng = np.random.default_rng(5)
    M, Cin, Cout = 37, 48, 40
    x = gen.to_storage(rng.normal(size=(M, Cin)), dtype)
    w = gen.to_storage(rng.normal(size=(Cout, Cin)) / 8, dtype)
    b = gen.to_storage(rng.normal(size=Cout), dtype) if with_bias else None
    got = oracle.linear(dtype, x, w, b)
    exact = gen.storage_to_f64(x, dtype) @ gen.storage_to_f64(w, dtype).T + (gen.storage_to_f64(b, dtype) if with_bias else 0.0)
    if dtype == "f32":
        assert np.array_equal(got, exact.astype(np.float32))
    else:
        assert np.array_equal(got.view(np.uint16), _nearest_even(dtype, exact))
    # an identity weight copies x, a zero weight gives the bias
    eye = gen.to_storage(np.eye(Cin), dtype)
    assert np.array_equal(gen.storage_to_f64(oracle.linear(dtype, x, eye), dtype), gen.storage_to_f64(x, dtype))
    if with_bias:
        zero = gen.to_storage(np.zeros((Cout, Cin)), dtype)
        assert np.array_equal(gen.storage_to_f64(oracle.linear(dtype, x, zero, b), dtype),
                              np.broadcast_to(gen.storage_to_f64(b, dtype), (M, Cout)))


def test_linear_shapes_and_rows():
    """Leading dimensions are flattened rows; row m of the output depends on row m of x only."""
    rng = np.random.default_rng(6)
    x = gen.to_storage(rng.normal(size=(2, 3, 5, 16)), "f16")
    w = gen.to_storage(rng.normal(size=(24, 16)), "f16")
    out = oracle.linear("f16", x, w)
    assert out.shape == (2, 3, 5, 24)
    assert np.array_equal(out[1, 2, 4], oracle.linear("f16", x[1, 2, 4][None], w)[0])
    with pytest.raises(ValueError):
        oracle.linear("f16", x, w[:, :8])



@pytest.mark.parametrize("dtype", ["f64", "f16", "bf16"])
def test_linear_backward_is_the_derivative_of_the_forward(dtype):
    """Every entry of grad_x, grad_weight and grad_bias equals the central difference
    of L = <g, linear(x, W, b)> in that coordinate, L evaluated with the forward
    oracle.  The layer is affine, so a unit step gives the derivative exactly; with
    small integers every forward output (and L) is exact even in 16-bit storage."""
    rng = np.random.default_rng(11)
    M, Cin, Cout = 5, 4, 6
    xs = rng.integers(-2, 3, size=(M, Cin)).astype(np.float64)
    ws = rng.integers(-2, 3, size=(Cout, Cin)).astype(np.float64)
    bs = rng.integers(-3, 4, size=Cout).astype(np.float64)
    gs = rng.integers(-3, 4, size=(M, Cout)).astype(np.float64)
    st = lambda a: gen.to_storage(a, dtype) if dtype != "f64" else a.copy()
    dec = lambda a: gen.storage_to_f64(a, dtype) if dtype != "f64" else a

    def loss(x, w, b):
        return float(np.sum(gs * dec(oracle.linear(dtype, st(x), st(w), st(b)))))

    gx, gw, gb = oracle.linear_backward(dtype, st(xs), st(ws), st(gs))
    for arr, grad, which in ((xs, gx, 0), (ws, gw, 1), (bs, gb, 2)):
        for idx in np.ndindex(arr.shape):
            args = [xs, ws, bs]
            up, dn = arr.copy(), arr.copy()
            up[idx] += 1.0
            dn[idx] -= 1.0
            args_up, args_dn = list(args), list(args)
            args_up[which], args_dn[which] = up, dn
            assert grad[idx] == (loss(*args_up) - loss(*args_dn)) / 2.0, (which, idx)


def test_linear_backward_rows_and_shapes():
    """Leading dimensions are rows; grad_x's row m depends on g's row m only; grad_weight
    and grad_bias are sums of per-row contributions (so they add over a split of the rows)."""
    rng = np.random.default_rng(12)
    x = gen.to_storage(rng.normal(size=(2, 3, 16)), "bf16")
    w = gen.to_storage(rng.normal(size=(8, 16)), "bf16")
    g = gen.to_storage(rng.normal(size=(2, 3, 8)), "bf16")
    gx, gw, gb = oracle.linear_backward("bf16", x, w, g)
    assert gx.shape == (2, 3, 16) and gw.shape == (8, 16) and gb.shape == (8,)
    gx1, gw1, gb1 = oracle.linear_backward("bf16", x[1, 2][None], w, g[1, 2][None])
    assert np.array_equal(gx[1, 2], gx1[0])
    gxa, gwa, gba = oracle.linear_backward("bf16", x[0], w, g[0])
    gxb, gwb, gbb = oracle.linear_backward("bf16", x[1], w, g[1])
    assert np.allclose(gw, gwa + gwb, rtol=1e-14, atol=1e-12) and np.allclose(gb, gba + gbb, rtol=1e-14, atol=1e-12)
    with pytest.raises(ValueError):
        oracle.linear_backward("bf16", x, w, g[..., :4])


# ---------------------------------------------------------------------------
# The hand-derived worked example (tests/golden/bilinear_2x2_worked.txt)
# ---------------------------------------------------------------------------

def test_worked_example_2x2():
    """Fractional offsets, an out-of-image corner and a sample that touches no pixel,
    worked out by hand from the definition: forward, grad_offset_mask and grad_value."""
    import _golden
    ex = _golden.load()
    prob = oracle.Problem(dtype="f64", **_golden.GEOMETRY)
    y = oracle.forward(prob, ex["value"], ex["offset_mask"])
    gv, gom = oracle.backward(prob, ex["value"], ex["offset_mask"], ex["grad_out"])
    assert np.array_equal(y, ex["y"])
    assert np.array_equal(gom, ex["grad_offset_mask"])
    assert np.array_equal(gv, ex["grad_value"])


# ---------------------------------------------------------------------------
# Deformable attention, single scale (CSDN summary section 1.1: each query
# attends to a selected number of sampling points whose positions and weights
# are dynamic; the weights normalised with a softmax over the points as in the
# section 1.2 DCNv3 equation)
# ---------------------------------------------------------------------------

def _attn_problem(w, **kw):
    return oracle.AttnProblem(dtype=w.dtype, **{**w.geometry(), **kw})


def _dyadic(x, bits=10):
    return np.round(np.asarray(x) * 2.0 ** bits) / 2.0 ** bits


def test_attn_on_the_grid_is_the_dcnv3_aggregation():
    """Queries at the pixel centres of a 3x3, stride-1, pad-1 grid whose offsets are the
    grid cells p_k plus DCN offsets reproduce the DCNv3 form of the aggregation (softmax
    over the K = 9 points) bit for bit, forward and backward: the same sampling
    locations, weights and sums.  (The DCN oracle is pinned independently above.)"""
    N, H, W, G, Cg, K = 2, 6, 7, 2, 3, 9
    rng = np.random.default_rng(31)
    value = rng.standard_normal((N, H, W, G * Cg)).astype(np.float32)
    dxy = _dyadic(rng.normal(0.0, 1.5, (N, H, W, G, K, 2))).astype(np.float32)
    logits = _dyadic(rng.normal(0.0, 1.0, (N, H, W, G, K))).astype(np.float32)
    gy = rng.standard_normal((N, H, W, G * Cg)).astype(np.float32)
    P = -(-G * 3 * K // 8) * 8
    om = gen.assemble_offset_mask(dxy, logits, P, "f32", tail_fill=0.0)
    dcn = oracle.Problem(N=N, H=H, W=W, G=G, Cg=Cg, dtype="f32", softmax=True, P=P)
    y_dcn = oracle.forward(dcn, value, om)
    gv_dcn, gom_dcn = oracle.backward(dcn, value, om, gy)
    # the same samples as queries: reference = output pixel centre (x, y), offset = p_k + dp
    grid = np.array([(iw - 1, ih - 1) for (ih, iw) in cells(3, 3, False)], dtype=np.float32)  # (x, y) per k
    off_attn = (dxy + grid[None, None, None, None, :, :]).astype(np.float32)
    assert np.array_equal(off_attn.astype(np.float64), dxy.astype(np.float64) + grid)  # exact in fp32
    ys, xs = np.divmod(np.arange(H * W), W)
    ref = np.broadcast_to(np.stack([xs, ys], -1).astype(np.float32), (N, H * W, 2)).copy()
    ol = gen.assemble_offset_mask(off_attn.reshape(N, H * W, G, K, 2), logits.reshape(N, H * W, G, K), P, "f32",
                                  tail_fill=0.0)
    attn = oracle.AttnProblem(N=N, H=H, W=W, G=G, Cg=Cg, Nq=H * W, K=K, P=P, dtype="f32")
    y = oracle.attn_forward(attn, value, ref, ol)
    gv, gol = oracle.attn_backward(attn, value, ref, ol, gy.reshape(N, H * W, G * Cg))
    np.testing.assert_array_equal(y.reshape(y_dcn.shape), y_dcn)
    np.testing.assert_array_equal(gv, gv_dcn)
    np.testing.assert_array_equal(gol.reshape(gom_dcn.shape), gom_dcn)


def test_attn_single_point_is_grid_sample():
    """K = 1: the weight is 1 and the output is the bilinear sample of the zero-padded map
    at reference + offset, which torch's grid_sample computes (align_corners=True)."""
    w = gen.attn_custom(N=2, H=9, W=11, G=3, Cg=4, Nq=40, K=1, P=16, dtype="f64", ref=("uniform", 2.0),
                        offset=("normal", 0.0, 3.0))
    inp = gen.make_attn_inputs(w, tail_fill=0.0)
    y = oracle.attn_forward(_attn_problem(w), inp["value"], inp["ref_points"], inp["offset_logits"])
    off = inp["offset_logits"][..., :9].reshape(2, 40, 3, 3)[..., :2]            # (dx, dy) per group
    loc = inp["ref_points"][:, :, None, :].astype(np.float64) + off               # (x, y)
    for g in range(3):
        img = torch.from_numpy(inp["value"][..., g * 4:(g + 1) * 4]).permute(0, 3, 1, 2)
        gx = 2.0 * loc[..., g, 0] / (w.W - 1) - 1.0
        gyy = 2.0 * loc[..., g, 1] / (w.H - 1) - 1.0
        grid = torch.from_numpy(np.stack([gx, gyy], -1)[:, :, None, :])
        ref = F.grid_sample(img, grid, mode="bilinear", padding_mode="zeros", align_corners=True)
        np.testing.assert_allclose(y[..., g * 4:(g + 1) * 4], ref[..., 0].permute(0, 2, 1).numpy(), rtol=0,
                                   atol=1e-12)


def test_attn_weights_are_a_softmax():
    """Equal logits average the K samples; one logit far above the rest selects its
    point; adding a constant to a query's logits changes nothing."""
    w = gen.attn_custom(N=1, H=8, W=8, G=2, Cg=3, Nq=12, K=4, P=24, dtype="f64", ref=("uniform", 1.0))
    inp = gen.make_attn_inputs(w, tail_fill=0.0)
    prob = _attn_problem(w)
    ol = inp["offset_logits"].copy()
    body = ol[..., :24].reshape(1, 12, 2, 12)
    body[..., 8:] = 0.3
    y_eq = oracle.attn_forward(prob, inp["value"], inp["ref_points"], ol)
    singles = []
    for k in range(4):
        one = ol.copy()
        b1 = one[..., :24].reshape(1, 12, 2, 12)
        b1[..., 8:] = -800.0
        b1[..., 8 + k] = 0.0
        singles.append(oracle.attn_forward(prob, inp["value"], inp["ref_points"], one))
    np.testing.assert_allclose(y_eq, sum(singles) / 4.0, rtol=1e-13, atol=1e-14)
    shifted = inp["offset_logits"].copy()
    shifted[..., :24].reshape(1, 12, 2, 12)[..., 8:] += 17.5
    np.testing.assert_allclose(oracle.attn_forward(prob, inp["value"], inp["ref_points"], shifted),
                               oracle.attn_forward(prob, inp["value"], inp["ref_points"], inp["offset_logits"]),
                               rtol=1e-12, atol=1e-14)


def test_attn_gradients():
    """grad_value by the adjoint identity <gy, y(v)> = <grad_value, v> (y is linear in
    value); offset and logit gradients by central differences; logit gradients of a
    (query, group) sum to 0; the padding tail is 0."""
    w = gen.attn_custom(N=2, H=6, W=7, G=2, Cg=3, Nq=10, K=3, P=24, dtype="f64", ref=("uniform", 0.5),
                        offset=("uniform", -1.7, 1.7))
    inp = gen.make_attn_inputs(w, tail_fill=0.0)
    prob = _attn_problem(w)
    v, ref, ol, gy = inp["value"], inp["ref_points"], inp["offset_logits"], inp["grad_out"]
    y = oracle.attn_forward(prob, v, ref, ol)
    gv, gol = oracle.attn_backward(prob, v, ref, ol, gy)
    assert np.isclose(np.sum(gy * y), np.sum(gv * v), rtol=1e-12)
    assert np.all(gol[..., 18:] == 0.0)
    np.testing.assert_allclose(gol[..., :18].reshape(2, 10, 2, 9)[..., 6:].sum(-1), 0.0, atol=1e-12)
    eps = 1e-6
    rng = np.random.default_rng(5)
    for _ in range(40):
        n, q, e = rng.integers(2), rng.integers(10), rng.integers(18)
        a, b = ol.copy(), ol.copy()
        a[n, q, e] += eps
        b[n, q, e] -= eps
        fd = (np.sum(gy * oracle.attn_forward(prob, v, ref, a)) - np.sum(gy * oracle.attn_forward(prob, v, ref, b))) / (2 * eps)
        assert abs(fd - gol[n, q, e]) <= 1e-6 * max(1.0, abs(fd)), (n, q, e, fd, gol[n, q, e])


def test_attn_far_offsets_touch_nothing():
    w = gen.attn_custom(N=1, H=5, W=6, G=2, Cg=4, Nq=8, K=3, P=24, dtype="f64", ref=("uniform", 0.0),
                        offset=("uniform", 50.0, 60.0))
    inp = gen.make_attn_inputs(w, tail_fill=0.0)
    prob = _attn_problem(w)
    assert np.all(oracle.attn_forward(prob, inp["value"], inp["ref_points"], inp["offset_logits"]) == 0.0)
    gv, gol = oracle.attn_backward(prob, inp["value"], inp["ref_points"], inp["offset_logits"], inp["grad_out"])
    assert np.all(gv == 0.0) and np.all(gol == 0.0)
