"""The torch.autograd wrapper against the oracle: y and both gradients of
y.backward(grad_out) equal the oracle's within the parity tolerances."""
import numpy as np
import pytest

import dcn4_inputs as gen
from _parity import BWD_TOL, FWD_TOL, normwise, oracle_backward, oracle_forward, to_device, to_f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["tiny_f32", "train_bf16_k8"])
def test_autograd_matches_oracle(name):
    import torch
    import deformable_convolution_sampling_b200 as dcn
    w = gen.WORKLOADS[name]
    if w.N > 2:
        w = gen.custom(**{**w.__dict__, "N": 2, "name": name + "_n2"})
    inp = gen.make_inputs(w)
    v = to_device(inp["value"], w.dtype).requires_grad_(True)
    om = to_device(inp["offset_mask"], w.dtype).requires_grad_(True)
    gy = to_device(inp["grad_out"], w.dtype)
    y = dcn.dcnv4_core(v, om, group=w.G, kernel=(w.kh, w.kw), stride=(w.sh, w.sw), pad=(w.ph, w.pw),
                       dilation=(w.dh, w.dw), offset_scale=w.offset_scale, remove_center=bool(w.remove_center))
    y.backward(gy)
    torch.cuda.synchronize()
    assert normwise(to_f64(y.detach()), oracle_forward(w, inp)) <= FWD_TOL[w.dtype]
    ref_gv, ref_gom = oracle_backward(w, inp)
    assert normwise(to_f64(v.grad), ref_gv) <= BWD_TOL[w.dtype]
    body = w.G * 3 * w.K
    assert normwise(to_f64(om.grad)[..., :body], ref_gom[..., :body]) <= BWD_TOL[w.dtype]
    assert np.all(to_f64(om.grad)[..., body:] == 0)     # the padding tail's gradient is 0


@pytest.mark.parametrize("dtype,bias", [("f16", True), ("bf16", False)])
def test_autograd_linear_matches_oracle(dtype, bias):
    """dcnv4_core_linear: y and the gradients of value, x, W and b against the oracle's
    chain: offset_mask = linear(x, W, b), y = aggregation, then the aggregation's
    backward and the linear layer's gradients in float64."""
    import torch
    import deformable_convolution_sampling_b200 as dcn
    import oracle
    from _parity import BWD_TOL, FWD_TOL, normwise, oracle_backward, oracle_forward, to_device, to_f64
    w = gen.custom(name="lin_autograd", N=2, H=12, W=10, G=4, Cg=16, Ho=12, Wo=10, K=9, P=112, dtype=dtype)
    inp = gen.make_inputs(w)
    lin = gen.make_linear_inputs(w, w.C, bias=bias)
    v = to_device(inp["value"], dtype).requires_grad_(True)
    x = to_device(lin["x"], dtype).requires_grad_(True)
    wt = to_device(lin["weight"], dtype).requires_grad_(True)
    b = to_device(lin["bias"], dtype).requires_grad_(True) if bias else None
    y = dcn.dcnv4_core_linear(v, x, wt, b, group=w.G)
    y.backward(to_device(inp["grad_out"], dtype))
    torch.cuda.synchronize()

    om_ref = oracle.linear(dtype, lin["x"], lin["weight"], lin["bias"])
    sub = {"value": inp["value"], "offset_mask": om_ref, "grad_out": inp["grad_out"]}
    ry = oracle_forward(w, sub)
    rgv, rgom = oracle_backward(w, sub)
    g = rgom.reshape(-1, w.P)
    xf = gen.storage_to_f64(lin["x"], dtype).reshape(-1, w.C)
    wf = gen.storage_to_f64(lin["weight"], dtype)
    assert normwise(to_f64(y), ry) <= FWD_TOL[dtype]
    assert normwise(to_f64(v.grad), rgv) <= BWD_TOL[dtype]
    assert normwise(to_f64(x.grad).reshape(-1, w.C), g @ wf) <= BWD_TOL[dtype]
    assert normwise(to_f64(wt.grad), g.T @ xf) <= BWD_TOL[dtype]
    if bias:
        assert normwise(to_f64(b.grad), g.sum(0)) <= BWD_TOL[dtype]
