"""Parity of dcn4_backward_linear (the backward of the aggregation with its
merged offset/mask linear layer) with the oracle, on a B200, through the C ABI.

The entry point runs dcn4_backward on the offset_mask the fused forward formed,
then the linear layer's gradients from the grad_offset_mask g it produced:
grad_x = g W, grad_W = g^T x, grad_b = column sums of g, each accumulated in
fp32 and rounded once to the storage format.  The checks:
  * grad_offset_mask is bit-identical to dcn4_backward's on the same inputs (the
    same kernels), grad_value matches the oracle (normwise, the operator's
    backward tolerance);
  * the linear step alone: the oracle's exact gradients from the kernel's own g
    (so the aggregation's rounding is not counted twice).  Each entry lies
    within ulp(ref) + (n+1) 2^-23 sum|terms| of the exact value (one rounding
    to storage plus the standard bound for an fp32 sum of n products), and
    normwise within one unit in the last place of the storage format;
  * the whole chain against the oracle's chain in float64 (grad_offset_mask
    from the oracle's backward, never rounded, through the oracle's linear
    backward): normwise within the operator's backward tolerance.
"""
import numpy as np
import pytest

import dcn4_inputs as gen
import oracle
from _parity import BWD_TOL, normwise, params_for, to_device, to_f64

pytestmark = pytest.mark.gpu

# one unit in the last place of the storage format, relative to the largest entry
ULP_REL = {"f16": 2.0 ** -10, "bf16": 2.0 ** -7}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _ulp(v: np.ndarray, dtype: str) -> np.ndarray:
    frac, emin = {"f16": (10, -14), "bf16": (7, -126)}[dtype]
    e = np.floor(np.log2(np.maximum(np.abs(v), 2.0 ** emin)))
    return 2.0 ** (e - frac)


def _within(got, ref, mag, n, dtype, what):
    bound = _ulp(ref, dtype) + (n + 1) * 2.0 ** -23 * mag
    diff = np.abs(got - ref)
    worst = np.unravel_index(np.argmax(diff / bound), diff.shape)
    assert np.all(diff <= bound), f"{what} entry {worst}: got {got[worst]}, exact {ref[worst]}"
    e = normwise(got, ref)
    assert e <= ULP_REL[dtype], f"{what} normwise {e:.3e}"


def _run(w, Cx, *, bias=True, sample=None, want_x=True, want_weight=True):
    import torch
    import deformable_convolution_sampling_b200 as dcn
    inp = gen.make_inputs(w, tail_fill=0.0)
    lin = gen.make_linear_inputs(w, Cx, bias=bias)
    p = params_for(w)
    v, gy = to_device(inp["value"], w.dtype), to_device(inp["grad_out"], w.dtype)
    x, wt = to_device(lin["x"], w.dtype), to_device(lin["weight"], w.dtype)
    b = to_device(lin["bias"], w.dtype) if bias else None
    om = torch.empty((w.N, w.Ho, w.Wo, w.P), dtype=v.dtype, device="cuda")
    dcn.forward_linear(p, v, x, wt, b, offset_mask_out=om)
    need = dcn.dcn4_backward_linear_workspace_size(p, Cx)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    gv, gom, gx, gw, gb = dcn.backward_linear(p, v, om, x, wt, gy, with_bias=bias, want_x=want_x,
                                              want_weight=want_weight, workspace=ws)
    _, gom_plain = dcn.backward(p, v, om, gy)
    torch.cuda.synchronize()
    # the linear kernels' status word (after dcn4_backward's part and the fp32 accumulators): no wait gave up
    off = (dcn.dcn4_backward_workspace_size(p) + 255) // 256 * 256 + 4 * (w.P * Cx + w.P)
    assert int(ws[off:off + 4].view(torch.int32).item()) == 0, "a bounded wait in the linear kernels gave up"
    assert torch.equal(gom.view(torch.int16), gom_plain.view(torch.int16)), "grad_offset_mask differs from dcn4_backward"
    assert (gx is None) != want_x and (gw is None) != want_weight and (gb is None) != bias

    # the linear step on the kernel's own g
    g_st = gom.cpu().view(torch.int16).numpy().view(np.uint16 if w.dtype == "bf16" else np.float16)
    idx = slice(None) if sample is None else sample
    xw = gen.storage_to_f64(lin["weight"], w.dtype)
    if want_x:
        rx, _, _ = oracle.linear_backward(w.dtype, np.ascontiguousarray(lin["x"][idx]), lin["weight"],
                                          np.ascontiguousarray(g_st[idx]), nthreads=oracle.host_threads(),
                                          want_weight=False)
        g64 = gen.storage_to_f64(np.ascontiguousarray(g_st[idx]), w.dtype)
        _within(to_f64(gx)[idx], rx, np.abs(g64) @ np.abs(xw), w.P, w.dtype, "grad_x")
    if want_weight or bias:
        _, rw, rb = oracle.linear_backward(w.dtype, lin["x"], lin["weight"], g_st, nthreads=oracle.host_threads(),
                                           want_x=False)
        g64 = gen.storage_to_f64(g_st, w.dtype).reshape(-1, w.P)
        M = g64.shape[0]
        if want_weight:
            x64 = gen.storage_to_f64(lin["x"], w.dtype).reshape(-1, Cx)
            _within(to_f64(gw), rw, np.abs(g64).T @ np.abs(x64), M, w.dtype, "grad_weight")
        if bias:
            _within(to_f64(gb), rb, np.abs(g64).sum(0), M, w.dtype, "grad_bias")

    # the whole chain against the oracle's, in float64 throughout, on the sampled images
    sub = {k: np.ascontiguousarray(inp[k][idx]) for k in ("value", "grad_out")}
    om_st = om.cpu().view(torch.int16).numpy().view(np.uint16 if w.dtype == "bf16" else np.float16)
    sub["offset_mask"] = np.ascontiguousarray(om_st[idx])
    n = sub["value"].shape[0]
    prob = oracle.Problem(dtype=w.dtype, location_fp32=True, **{**w.geometry(), "N": n})
    rgv, rgom = oracle.backward(prob, sub["value"], sub["offset_mask"], sub["grad_out"],
                                nthreads=oracle.host_threads())
    e_v = normwise(to_f64(gv)[idx], rgv)
    assert e_v <= BWD_TOL[w.dtype], f"{w.name} grad_value {e_v:.3e}"
    if want_x:
        xs = gen.storage_to_f64(np.ascontiguousarray(lin["x"][idx]), w.dtype)
        cx, _, _ = oracle.linear_backward("f64", xs, xw, rgom, want_weight=False)
        e_x = normwise(to_f64(gx)[idx], cx)
        assert e_x <= BWD_TOL[w.dtype], f"{w.name} chained grad_x {e_x:.3e}"
    if want_weight and sample is None:
        x64 = gen.storage_to_f64(lin["x"], w.dtype)
        _, cw, cb = oracle.linear_backward("f64", x64, xw, rgom, want_x=False)
        e_w = normwise(to_f64(gw), cw)
        assert e_w <= BWD_TOL[w.dtype], f"{w.name} chained grad_weight {e_w:.3e}"
        if bias:
            e_b = normwise(to_f64(gb), cb)
            assert e_b <= BWD_TOL[w.dtype], f"{w.name} chained grad_bias {e_b:.3e}"


@pytest.mark.parametrize("name", ["stage1_f16", "stage3_bf16", "highres_f16", "train_bf16_k8"])
def test_workloads(name):
    """The measured workloads at full size with Cx = C: grad_weight and grad_bias over
    every row, grad_x and the chain on sampled images."""
    w = gen.WORKLOADS[name]
    _run(w, w.C, sample=None if w.N <= 2 else [0, w.N // 2, w.N - 1])


VARIANTS = [
    dict(name="no_bias_f16", bias=False, Cx=64, N=2, H=12, W=10, G=4, Cg=16, Ho=12, Wo=10, K=9, P=112, dtype="f16"),
    dict(name="cx16_bf16", Cx=16, N=2, H=9, W=9, G=2, Cg=16, Ho=9, Wo=9, K=9, P=56, dtype="bf16"),
    dict(name="cx48_ragged_rc_f16", Cx=48, N=3, H=7, W=5, G=3, Cg=8, Ho=3, Wo=3, K=8, P=72, dtype="f16",
         sh=2, sw=2, ph=1, pw=2, dh=2, dw=2, remove_center=1, offset_scale=0.7),
    dict(name="g32_f16", Cx=64, N=2, H=7, W=7, G=32, Cg=8, Ho=7, Wo=7, K=9, P=864, dtype="f16"),
    dict(name="softmax_bf16", Cx=64, N=2, H=10, W=12, G=4, Cg=16, Ho=10, Wo=12, K=9, P=112, dtype="bf16", softmax=1),
    dict(name="one_pixel_bf16", Cx=16, N=1, H=1, W=1, G=4, Cg=8, Ho=1, Wo=1, K=9, P=112, dtype="bf16"),
    dict(name="cx208_f16", Cx=208, N=2, H=9, W=10, G=2, Cg=32, Ho=9, Wo=10, K=9, P=56, dtype="f16"),
    dict(name="rows_not_tiles_bf16", Cx=80, N=3, H=13, W=11, G=2, Cg=16, Ho=13, Wo=11, K=9, P=64, dtype="bf16"),
]


@pytest.mark.parametrize("spec", VARIANTS, ids=[v["name"] for v in VARIANTS])
def test_variants(spec):
    spec = dict(spec)
    Cx, bias = spec.pop("Cx"), spec.pop("bias", True)
    _run(gen.custom(**spec), Cx, bias=bias)


@pytest.mark.parametrize("want_x,want_weight", [(False, True), (True, False), (False, False)])
def test_gradients_not_wanted_are_skipped(want_x, want_weight):
    w = gen.custom(name="partial", N=2, H=9, W=8, G=4, Cg=16, Ho=9, Wo=8, K=9, P=112, dtype="f16")
    _run(w, 32, want_x=want_x, want_weight=want_weight)


def test_empty_batch_zeroes_weight_and_bias_gradients():
    import torch
    import deformable_convolution_sampling_b200 as dcn
    p = dcn.make_params(N=0, H=8, W=8, G=4, Cg=16, dtype="bf16")
    Cx = 32
    gw = torch.full((p.P, Cx), 7.0, dtype=torch.bfloat16, device="cuda")
    gb = torch.full((p.P,), 7.0, dtype=torch.bfloat16, device="cuda")
    need = dcn.dcn4_backward_linear_workspace_size(p, Cx)
    ws = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
    st = dcn.dcn4_backward_linear(p, Cx, None, None, None, None, None, None, None, None, gw.data_ptr(),
                                  gb.data_ptr(), ws.data_ptr(), need, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert st == 0 and torch.count_nonzero(gw).item() == 0 and torch.count_nonzero(gb).item() == 0


def test_autograd_linear_uses_the_library_backward():
    """dcnv4_core_linear's gradients equal dcn4_backward_linear's bit for bit."""
    import torch
    import deformable_convolution_sampling_b200 as dcn
    w = gen.custom(name="ag", N=2, H=10, W=9, G=4, Cg=16, Ho=10, Wo=9, K=9, P=112, dtype="bf16")
    inp = gen.make_inputs(w, tail_fill=0.0)
    lin = gen.make_linear_inputs(w, 64)
    v = to_device(inp["value"], w.dtype).requires_grad_()
    x = to_device(lin["x"], w.dtype).requires_grad_()
    wt = to_device(lin["weight"], w.dtype).requires_grad_()
    b = to_device(lin["bias"], w.dtype).requires_grad_()
    gy = to_device(inp["grad_out"], w.dtype)
    y = dcn.dcnv4_core_linear(v, x, wt, b, group=w.G)
    y.backward(gy)
    p = params_for(w)
    om = torch.empty((w.N, w.Ho, w.Wo, w.P), dtype=v.dtype, device="cuda")
    dcn.forward_linear(p, v.detach(), x.detach(), wt.detach(), b.detach(), offset_mask_out=om)
    _, _, gx, gw, gb = dcn.backward_linear(p, v.detach(), om, x.detach(), wt.detach(), gy)
    torch.cuda.synchronize()
    assert torch.equal(x.grad.view(torch.int16), gx.view(torch.int16))
    # grad_weight and grad_bias sum fp32 partials with atomics: equal up to their order
    assert normwise(to_f64(wt.grad), to_f64(gw)) <= ULP_REL[w.dtype]
    assert normwise(to_f64(b.grad), to_f64(gb)) <= ULP_REL[w.dtype]
