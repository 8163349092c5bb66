"""dcn4_backward_noalloc: the backward for callers that cannot provide device
memory when they call (for example a plugin inside a host runtime that owns
all device buffers and offers no allocator).  Its gradients must match the
CPU oracle within the backward tolerance, call after call on the same built-in
area, and it must refuse problems whose scratch does not fit that area.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import dataclasses

import numpy as np
import pytest

import dcn4_inputs as gen
from _parity import BWD_TOL, normwise, oracle_backward, params_for, to_device, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


# The training-step shape at 16 images and the tiny case.
@pytest.mark.parametrize("name", ["train_bf16_k8", "tiny_f32"])
def test_noalloc_matches_the_oracle_twice(cuda, name):
    torch = cuda
    import deformable_convolution_sampling_b200 as dcn
    w = gen.WORKLOADS[name]
    if name == "train_bf16_k8":
        w = dataclasses.replace(w, N=16)
    inp = gen.make_inputs(w)
    p = params_for(w)
    v, om, gy = (to_device(inp[k], w.dtype) for k in ("value", "offset_mask", "grad_out"))
    assert dcn.dcn4_backward_workspace_size(p) <= dcn.dcn4_backward_noalloc_capacity()
    rgv, rgom = oracle_backward(w, inp)
    body = w.G * 3 * w.K
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):                                  # the area keeps the last call's contents
        gv = torch.full_like(v, float("nan"))
        gom = torch.full_like(om, float("nan"))
        st = dcn.dcn4_backward_noalloc(p, v.data_ptr(), om.data_ptr(), gy.data_ptr(), gv.data_ptr(),
                                       gom.data_ptr(), stream)
        assert st == 0, dcn.dcn4_noalloc_last_error() or dcn.dcn4_last_error()
        torch.cuda.synchronize()
        a, g = to_f64(gv), to_f64(gom)
        assert np.all(np.isfinite(a)) and np.all(np.isfinite(g))
        assert normwise(a, rgv) <= BWD_TOL[w.dtype]
        assert normwise(g[..., :body], rgom[..., :body]) <= BWD_TOL[w.dtype]
        assert np.all(g[..., body:] == 0.0)


def test_noalloc_rejects_problems_beyond_its_area(cuda):
    """The size check comes first; the tensors are NULL, so even a regressed check
    would stop at the pointer check and launch nothing."""
    import deformable_convolution_sampling_b200 as dcn
    p = dcn.make_params(N=4096, H=224, W=224, G=4, Cg=16, dtype="f16")
    assert dcn.dcn4_backward_workspace_size(p) > dcn.dcn4_backward_noalloc_capacity()
    st = dcn.dcn4_backward_noalloc(p, None, None, None, None, None, None)
    assert st == -6
    assert "scratch" in dcn.dcn4_noalloc_last_error()
