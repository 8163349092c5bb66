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
