"""Parity of dcn4_forward_proj / dcn4_backward_proj (the output projection fused
behind the aggregation) with the oracle, on a B200, through the C ABI.

Forward.  The kernel rounds the aggregation's sums to the storage format (as the
unfused pair would store its core output), multiplies that tile by W on the
tensor cores with fp32 accumulation, adds the bias in fp32 and rounds once.
The checks:
  * core_out is bit-identical to dcn4_forward (the same sampler), and y does not
    depend on whether core_out is stored;
  * y against the oracle's linear layer applied to the kernel's own core
    output: each entry within one unit in the last place plus the fp32
    accumulation bound (C+1) 2^-23 sum|core w|, and equal almost everywhere;
  * y against the oracle's chain (its aggregation, rounded to storage, then its
    linear layer), normwise within the operator's forward tolerance.
Backward.  grad_core = grad_y W (rounded to storage), grad_W = grad_y^T core,
grad_b = column sums of grad_y, then dcn4_backward with grad_core.  The checks:
  * grad_core (read from the workspace), grad_W and grad_b against the oracle's
    exact gradients from the same operands, entrywise as above and normwise
    within one unit in the last place;
  * grad_offset_mask bit-identical to dcn4_backward on that grad_core and
    grad_value within one unit in the last place of it (its per-cell sums follow
    the order in which samples were filed), both within the backward tolerance
    of the oracle's backward on the oracle's own grad_core.
"""
import numpy as np
import pytest

import dcn4_inputs as gen
import oracle
from _parity import BWD_TOL, FWD_TOL, normwise, oracle_forward, params_for, to_device, to_f64

pytestmark = pytest.mark.gpu

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


def _within(got, ref, mag, n, dtype, what, *, mostly_equal=False):
    bound = _ulp(ref, dtype) + (n + 1) * 2.0 ** -23 * mag
    diff = np.abs(got - ref)
    worst = np.unravel_index(np.argmax(diff / bound), diff.shape)
    assert np.all(diff <= bound), f"{what} entry {worst}: got {got[worst]}, exact {ref[worst]}"
    assert normwise(got, ref) <= ULP_REL[dtype], f"{what} normwise {normwise(got, ref):.3e}"
    if mostly_equal:
        assert np.mean(diff > 0) < 0.05, f"{what}: {np.mean(diff > 0):.3f} of the entries differ"


def _storage(t, dtype):
    import torch
    return t.cpu().view(torch.int16).numpy().view(np.uint16 if dtype == "bf16" else np.float16)


def _run(w, Cout, *, bias=True, sample=None, want_weight=True):
    import torch
    import deformable_convolution_sampling_b200 as dcn
    inp = gen.make_inputs(w, with_grad=False, tail_fill=0.0)
    pj = gen.make_proj_inputs(w, Cout, bias=bias)
    p = params_for(w)  # also checks the output grid the tensors are sized for
    v, om = to_device(inp["value"], w.dtype), to_device(inp["offset_mask"], w.dtype)
    wt = to_device(pj["weight"], w.dtype)
    b = to_device(pj["bias"], w.dtype) if bias else None
    gy = to_device(pj["grad_out"], w.dtype)
    dcn.dcn4_forward_tc_status(reset=True)

    # ---- forward
    core = torch.full((w.N, w.Ho, w.Wo, w.C), float("nan"), dtype=v.dtype, device="cuda")
    y = dcn.forward_proj(p, v, om, wt, b, core_out=core)
    y_only = dcn.forward_proj(p, v, om, wt, b)
    core_plain = dcn.forward(p, v, om)
    torch.cuda.synchronize()
    assert dcn.dcn4_forward_tc_status() == 0, "a bounded wait of the projection gave up"
    assert torch.equal(core.view(torch.int16), core_plain.view(torch.int16)), "core_out differs from dcn4_forward"
    assert torch.equal(y.view(torch.int16), y_only.view(torch.int16))

    idx = slice(None) if sample is None else sample
    core_st = _storage(core, w.dtype)
    w64 = gen.storage_to_f64(pj["weight"], w.dtype)
    c64 = gen.storage_to_f64(np.ascontiguousarray(core_st[idx]), w.dtype)
    ref = gen.storage_to_f64(oracle.linear(w.dtype, np.ascontiguousarray(core_st[idx]), pj["weight"], pj["bias"]),
                             w.dtype)
    mag = np.abs(c64) @ np.abs(w64).T
    if bias:
        mag = mag + np.abs(gen.storage_to_f64(pj["bias"], w.dtype))
    got = to_f64(y)[idx]
    _within(got, ref, mag, w.C, w.dtype, "y", mostly_equal=True)
    rcore = oracle_forward(w, {k: np.ascontiguousarray(inp[k][idx]) for k in ("value", "offset_mask")})
    ry = gen.storage_to_f64(oracle.linear(w.dtype, oracle.encode(w.dtype, rcore), pj["weight"], pj["bias"]), w.dtype)
    e = normwise(got, ry)
    assert e <= FWD_TOL[w.dtype], f"{w.name} chained y {e:.3e}"

    # ---- backward
    need = dcn.dcn4_backward_proj_workspace_size(p, Cout)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    gv, gom, gw, gb = dcn.backward_proj(p, v, om, core, wt, gy, with_bias=bias, want_weight=want_weight,
                                        workspace=ws)
    torch.cuda.synchronize()
    assert (gw is None) != want_weight and (gb is None) != bias
    M = w.N * w.Ho * w.Wo
    core_ws = (dcn.dcn4_backward_workspace_size(p) + 255) // 256 * 256
    gcore_bytes = (M * w.C * 2 + 255) // 256 * 256
    status = core_ws + gcore_bytes + 4 * (Cout * w.C + Cout)
    assert int(ws[status:status + 4].view(torch.int32).item()) == 0, "a bounded wait in the linear kernels gave up"
    gcore = ws[core_ws:core_ws + M * w.C * 2].view(v.dtype).view(w.N, w.Ho, w.Wo, w.C).clone()
    gv_plain, gom_plain = dcn.backward(p, v, om, gcore)
    torch.cuda.synchronize()
    # grad_value sums each cell's samples in the order they were filed (atomic slots), so two
    # calls agree up to that order: within one unit in the last place
    e_rep = normwise(to_f64(gv), to_f64(gv_plain))
    assert e_rep <= ULP_REL[w.dtype], f"grad_value differs from dcn4_backward's by {e_rep:.3e}"
    assert torch.equal(gom.view(torch.int16), gom_plain.view(torch.int16)), "grad_offset_mask differs"

    gy_st = pj["grad_out"]
    rx, _, _ = oracle.linear_backward(w.dtype, np.ascontiguousarray(core_st[idx]), pj["weight"],
                                      np.ascontiguousarray(gy_st[idx]), nthreads=oracle.host_threads(),
                                      want_weight=False)
    g64 = gen.storage_to_f64(np.ascontiguousarray(gy_st[idx]), w.dtype)
    _within(to_f64(gcore)[idx], rx, np.abs(g64) @ np.abs(w64), Cout, w.dtype, "grad_core")
    if want_weight or bias:
        _, rw, rb = oracle.linear_backward(w.dtype, core_st, pj["weight"], gy_st, nthreads=oracle.host_threads(),
                                           want_x=False)
        gall = gen.storage_to_f64(gy_st, w.dtype).reshape(-1, Cout)
        if want_weight:
            call = gen.storage_to_f64(core_st, w.dtype).reshape(-1, w.C)
            _within(to_f64(gw), rw, np.abs(gall).T @ np.abs(call), M, w.dtype, "grad_weight")
        if bias:
            _within(to_f64(gb), rb, np.abs(gall).sum(0), M, w.dtype, "grad_bias")

    # the aggregation's backward against the oracle's on the oracle's own grad_core
    sub = {k: np.ascontiguousarray(inp[k][idx]) for k in ("value", "offset_mask")}
    n = sub["value"].shape[0]
    prob = oracle.Problem(dtype=w.dtype, location_fp32=True, **{**w.geometry(), "N": n})
    rgv, rgom = oracle.backward(prob, sub["value"], sub["offset_mask"], oracle.encode(w.dtype, rx),
                                nthreads=oracle.host_threads())
    e_v = normwise(to_f64(gv)[idx], rgv)
    e_om = normwise(to_f64(gom)[idx][..., :w.G * 3 * w.K], rgom[..., :w.G * 3 * w.K])
    assert e_v <= BWD_TOL[w.dtype], f"{w.name} grad_value {e_v:.3e}"
    assert e_om <= BWD_TOL[w.dtype], f"{w.name} grad_offset_mask {e_om:.3e}"


@pytest.mark.parametrize("name,Cout", [("stage1_f16", 64), ("highres_f16", 64), ("train_bf16_k8", 64),
                                       ("stage3_bf16", 128)])
def test_workloads(name, Cout):
    """The measured workloads at full size (C -> C where the kernel forms it; the
    third-stage shape's 256 channels -> 128, the most one tile forms); the oracle
    checks sampled images, grad_weight and grad_bias over every row."""
    w = gen.WORKLOADS[name]
    _run(w, Cout, sample=None if w.N <= 2 else [0, w.N // 2, w.N - 1])


VARIANTS = [
    dict(name="no_bias_ragged_f16", bias=False, Cout=64, N=2, H=12, W=10, G=4, Cg=16, Ho=12, Wo=10, K=9, P=112,
         dtype="f16"),
    dict(name="cout128_bf16", Cout=128, N=2, H=9, W=11, G=4, Cg=16, Ho=9, Wo=11, K=9, P=112, dtype="bf16"),
    dict(name="cout16_f16", Cout=16, N=2, H=8, W=8, G=4, Cg=16, Ho=8, Wo=8, K=9, P=112, dtype="f16"),
    dict(name="c64_g2_f16", Cout=48, N=2, H=10, W=9, G=2, Cg=32, Ho=10, Wo=9, K=9, P=56, dtype="f16"),
    dict(name="c128_g4_32px_f16", Cout=64, N=2, H=9, W=10, G=4, Cg=32, Ho=9, Wo=10, K=9, P=112, dtype="f16"),
    dict(name="c128_g8_32px_bf16", Cout=96, N=2, H=9, W=10, G=8, Cg=16, Ho=9, Wo=10, K=9, P=216, dtype="bf16"),
    dict(name="c256_g16_16px_bf16", Cout=128, N=2, H=9, W=9, G=16, Cg=16, Ho=9, Wo=9, K=9, P=432, dtype="bf16"),
    dict(name="ragged_s2_d2_rc_f16", Cout=64, N=3, H=11, W=9, G=4, Cg=16, Ho=5, Wo=5, K=8, P=96, dtype="f16",
         sh=2, sw=2, ph=1, pw=2, dh=2, dw=2, remove_center=1, offset_scale=0.7),
    dict(name="softmax_f16", Cout=64, N=2, H=10, W=12, G=4, Cg=16, Ho=10, Wo=12, K=9, P=112, dtype="f16", softmax=1),
    dict(name="k5x5_bf16", Cout=64, N=2, H=9, W=11, G=4, Cg=16, Ho=9, Wo=11, K=25, P=304, dtype="bf16", kh=5, kw=5,
         ph=2, pw=2),
    dict(name="one_pixel_bf16", Cout=32, N=1, H=1, W=1, G=4, Cg=16, Ho=1, Wo=1, K=9, P=112, dtype="bf16"),
]


@pytest.mark.parametrize("spec", VARIANTS, ids=[v["name"] for v in VARIANTS])
def test_variants(spec):
    spec = dict(spec)
    Cout, bias = spec.pop("Cout"), spec.pop("bias", True)
    _run(gen.custom(**spec), Cout, bias=bias)


def test_without_weight_gradient():
    w = gen.custom(name="no_gw", N=2, H=9, W=10, G=4, Cg=16, Ho=9, Wo=10, K=9, P=112, dtype="bf16")
    _run(w, 64, want_weight=False)


def test_identity_weight_reproduces_the_core():
    """weight = identity, no bias: y equals dcn4_forward bit for bit (each output is
    one exact product)."""
    import torch
    import deformable_convolution_sampling_b200 as dcn
    w = gen.custom(name="ident", N=2, H=9, W=10, G=4, Cg=16, Ho=9, Wo=10, K=9, P=112, dtype="f16")
    inp = gen.make_inputs(w, with_grad=False, tail_fill=0.0)
    p = params_for(w)
    v, om = to_device(inp["value"], w.dtype), to_device(inp["offset_mask"], w.dtype)
    eye = torch.eye(w.C, dtype=v.dtype, device="cuda")
    y = dcn.forward_proj(p, v, om, eye)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), dcn.forward(p, v, om).view(torch.int16))


def test_unsupported_shapes_are_refused():
    """Shapes the kernel does not form come back as DCN4_ERR_UNSUPPORTED before any
    launch, with a message; the valid neighbour of each runs."""
    import torch
    import deformable_convolution_sampling_b200 as dcn
    w = gen.custom(name="c32", N=1, H=8, W=8, G=2, Cg=16, Ho=8, Wo=8, K=9, P=56, dtype="f16")  # C = 32
    inp = gen.make_inputs(w, with_grad=False, tail_fill=0.0)
    p = params_for(w)
    v, om = to_device(inp["value"], w.dtype), to_device(inp["offset_mask"], w.dtype)
    wt = torch.zeros((64, 32), dtype=v.dtype, device="cuda")
    out = torch.empty((1, 8, 8, 64), dtype=v.dtype, device="cuda")
    assert dcn.dcn4_forward_proj(p, 64, v.data_ptr(), om.data_ptr(), wt.data_ptr(), None, out.data_ptr()) == -5
    assert "multiple of 64" in dcn.dcn4_last_error()


def test_empty_batch():
    """N = 0: the forward is a no-op; the backward writes zero weight and bias gradients."""
    import torch
    import deformable_convolution_sampling_b200 as dcn
    p = dcn.make_params(N=0, H=8, W=8, G=4, Cg=16, dtype="bf16")
    assert dcn.dcn4_forward_proj(p, 64, None, None, None, None, None) == 0
    gw = torch.full((64, 64), 7.0, dtype=torch.bfloat16, device="cuda")
    gb = torch.full((64,), 7.0, dtype=torch.bfloat16, device="cuda")
    need = dcn.dcn4_backward_proj_workspace_size(p, 64)
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device="cuda")
    assert dcn.dcn4_backward_proj(p, 64, None, None, None, None, None, None, None, gw.data_ptr(), gb.data_ptr(),
                                  ws.data_ptr(), ws.numel()) == 0
    torch.cuda.synchronize()
    assert not gw.any() and not gb.any()


def test_autograd():
    """dcnv4_core_proj through torch.autograd: gradients of value, offset_mask, weight
    and bias are those of backward_proj (grad_value up to the order of each cell's
    sums, grad_weight and grad_bias up to the last bit of their fp32 atomic sums)."""
    import torch
    import deformable_convolution_sampling_b200 as dcn
    w = gen.custom(name="ag", N=2, H=10, W=9, G=4, Cg=16, Ho=10, Wo=9, K=9, P=112, dtype="f16")
    inp = gen.make_inputs(w, with_grad=False, tail_fill=0.0)
    pj = gen.make_proj_inputs(w, 64)
    v = to_device(inp["value"], w.dtype).requires_grad_()
    om = to_device(inp["offset_mask"], w.dtype).requires_grad_()
    wt = to_device(pj["weight"], w.dtype).requires_grad_()
    b = to_device(pj["bias"], w.dtype).requires_grad_()
    gy = to_device(pj["grad_out"], w.dtype)
    y = dcn.dcnv4_core_proj(v, om, wt, b, group=w.G)
    y.backward(gy)
    p = params_for(w)
    core = dcn.forward(p, v.detach(), om.detach())
    gv, gom, gw, gb = dcn.backward_proj(p, v.detach(), om.detach(), core, wt.detach(), gy)
    torch.cuda.synchronize()
    assert torch.equal(y.detach(), dcn.forward_proj(p, v.detach(), om.detach(), wt.detach(), b.detach()))
    assert torch.equal(om.grad, gom)
    assert normwise(to_f64(v.grad), to_f64(gv)) <= ULP_REL[w.dtype]  # up to the order of each cell's sums
    assert torch.allclose(wt.grad.float(), gw.float(), rtol=2 ** -9, atol=0)
    assert torch.allclose(b.grad.float(), gb.float(), rtol=2 ** -9, atol=0)
