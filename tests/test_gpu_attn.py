"""Single-scale deformable attention through the C ABI against the CPU oracle, on a B200.

Tolerances are the operator's (normwise max|gpu - ref| / max|ref|): forward
1e-5 (fp32) and 2e-2 (16-bit); backward 1e-4 (fp32) and 3e-2 (16-bit), the
backward's grad_value being summed with fp32 atomics in no fixed order.  The
oracle forms the sampling location with the same fp32 fma as the kernels.
"""
import numpy as np
import pytest

import dcn4_inputs as gen
import oracle
from _parity import BWD_TOL, FWD_TOL, normwise, to_device, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _params(w):
    import deformable_convolution_sampling_b200 as dcn
    return dcn.make_attn_params(dtype=w.dtype, **w.geometry())


def _problem(w, n):
    return oracle.AttnProblem(dtype=w.dtype, location_fp32=True, **{**w.geometry(), "N": n})


def _ref_tensor(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _run(w, inp, backward=True):
    import deformable_convolution_sampling_b200 as dcn
    p = _params(w)
    v, ol = to_device(inp["value"], w.dtype), to_device(inp["offset_logits"], w.dtype)
    ref = _ref_tensor(inp["ref_points"])
    y = dcn.attn_forward(p, v, ref, ol)
    if not backward:
        return to_f64(y), None, None
    gv, gol = dcn.attn_backward(p, v, ref, ol, to_device(inp["grad_out"], w.dtype))
    return to_f64(y), to_f64(gv), to_f64(gol)


def _check(w, inp, sample=None, backward=True):
    y, gv, gol = _run(w, inp, backward)
    sub = inp if sample is None else {k: np.ascontiguousarray(a[sample]) for k, a in inp.items()}
    n = sub["value"].shape[0]
    prob = _problem(w, n)
    ry = oracle.attn_forward(prob, sub["value"], sub["ref_points"], sub["offset_logits"],
                             nthreads=oracle.host_threads())
    if sample is not None:
        y = y[sample]
    e_y = normwise(y, ry)
    assert e_y <= FWD_TOL[w.dtype], f"{w.name} forward {e_y:.3e}"
    if not backward:
        return e_y, None
    rgv, rgol = oracle.attn_backward(prob, sub["value"], sub["ref_points"], sub["offset_logits"], sub["grad_out"],
                                     nthreads=oracle.host_threads())
    if sample is not None:
        gv, gol = gv[sample], gol[sample]
    body = w.G * 3 * w.K
    assert np.all(gol[..., body:] == 0.0), "padding tail of grad_offset_logits must be 0"
    e_v = normwise(gv, rgv)
    parts = gol[..., :body].reshape(gol.shape[:-1] + (w.G, 3 * w.K))
    rparts = rgol[..., :body].reshape(rgol.shape[:-1] + (w.G, 3 * w.K))
    e_off = normwise(parts[..., :2 * w.K], rparts[..., :2 * w.K])
    e_l = normwise(parts[..., 2 * w.K:], rparts[..., 2 * w.K:])
    for name, e in (("grad_value", e_v), ("grad_offset", e_off), ("grad_logit", e_l)):
        assert e <= BWD_TOL[w.dtype], f"{w.name} {name} {e:.3e}"
    return e_y, max(e_v, e_off, e_l)


@pytest.mark.parametrize("name", gen.ATTN_WORKLOAD_ORDER)
def test_attn_workload(name):
    w = gen.ATTN_WORKLOADS[name]
    inp = gen.make_attn_inputs(w)
    sample = None if w.N <= 2 else [0, w.N // 2, w.N - 1]
    _check(w, inp, sample)


def test_attn_fp32_is_tight():
    w = gen.ATTN_WORKLOADS["attn_tiny_f32"]
    e_y, e_b = _check(w, gen.make_attn_inputs(w))
    assert e_y < 1e-6 and e_b < 1e-5


ATTN_VARIANTS = [
    dict(name="one_point_f16", N=2, H=9, W=11, G=3, Cg=8, Nq=40, K=1, P=16, dtype="f16", ref=("uniform", 2.0)),
    dict(name="many_points_bf16", N=2, H=12, W=10, G=2, Cg=16, Nq=50, K=16, P=96, dtype="bf16", ref=("uniform", 1.0)),
    dict(name="one_head_wide_f16", N=2, H=10, W=10, G=1, Cg=64, Nq=100, K=4, P=16, dtype="f16"),
    dict(name="wide_f32", N=2, H=7, W=9, G=2, Cg=32, Nq=20, K=3, P=24, dtype="f32", ref=("uniform", 1.5)),
    dict(name="far_f16", N=2, H=6, W=8, G=2, Cg=8, Nq=30, K=4, P=24, dtype="f16", ref=("uniform", 3.0),
         offset=("uniform", -20.0, 20.0)),
    dict(name="scaled_bf16", N=3, H=8, W=13, G=4, Cg=8, Nq=17, K=5, P=64, dtype="bf16", offset_scale=0.37,
         ref=("uniform", 0.5)),
]


@pytest.mark.parametrize("spec", ATTN_VARIANTS, ids=[v["name"] for v in ATTN_VARIANTS])
def test_attn_variants(spec):
    w = gen.attn_custom(**spec)
    _check(w, gen.make_attn_inputs(w))


def test_attn_no_queries_gives_zero_grad_value():
    import torch
    import deformable_convolution_sampling_b200 as dcn
    p = dcn.make_attn_params(N=2, H=6, W=6, G=2, Cg=8, Nq=0, K=4, dtype="f16")
    v = torch.randn(2, 6, 6, 16, device="cuda").half()
    empty = torch.empty(0, device="cuda")
    gv, gol = dcn.attn_backward(p, v, empty, empty.half(), empty.half())
    torch.cuda.synchronize()
    assert torch.count_nonzero(gv).item() == 0 and gol.numel() == 0


def test_attn_encoder_queries_match_the_aggregation():
    """Pixel-centre queries whose offsets are the 3x3 grid plus DCN offsets sample exactly
    what the softmax form of dcn4_forward samples: the two kernels agree to fp32
    summation order on the same data."""
    import torch
    import deformable_convolution_sampling_b200 as dcn
    N, H, W, G, Cg, K = 2, 12, 14, 4, 16, 9
    w = gen.custom(name="grid", N=N, H=H, W=W, G=G, Cg=Cg, Ho=H, Wo=W, K=K, P=112, dtype="f32", softmax=1)
    inp = gen.make_inputs(w, tail_fill=0.0, with_grad=False)
    p = dcn.make_params(dtype="f32", **w.geometry())
    v = torch.from_numpy(inp["value"]).cuda()
    om = inp["offset_mask"]
    y_dcn = to_f64(dcn.forward(p, v, torch.from_numpy(om).cuda()))
    body = om[..., :G * 3 * K].reshape(N, H, W, G, 3 * K).copy()
    cells = [(ih, iw) for iw in range(3) for ih in range(3)]
    for k, (ih, iw) in enumerate(cells):
        body[..., 2 * k] += np.float32(iw - 1)
        body[..., 2 * k + 1] += np.float32(ih - 1)
    ol = np.zeros((N, H * W, 112), dtype=np.float32)
    ol[..., :G * 3 * K] = body.reshape(N, H * W, G * 3 * K)
    ys, xs = np.divmod(np.arange(H * W), W)
    ref = np.broadcast_to(np.stack([xs, ys], -1).astype(np.float32), (N, H * W, 2)).copy()
    pa = dcn.make_attn_params(N=N, H=H, W=W, G=G, Cg=Cg, Nq=H * W, K=K, P=112, dtype="f32")
    y = to_f64(dcn.attn_forward(pa, v, _ref_tensor(ref), torch.from_numpy(ol).cuda()))
    assert normwise(y.reshape(y_dcn.shape), y_dcn) < 1e-6
