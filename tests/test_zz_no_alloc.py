"""dcn4_backward_noalloc: the backward for callers that cannot provide device
memory when they call (for example a plugin inside a host runtime that owns
all device buffers and offers no allocator).  It must give the same gradients
as dcn4_backward with a caller workspace, call after call, and refuse problems
whose scratch does not fit its built-in area.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import dataclasses

import numpy as np
import pytest

import dcn4_inputs as gen
from _parity import BWD_TOL, normwise, params_for, to_device, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch


# The training-step shape at 16 images (its scratch fits the built-in area) and the tiny case.
@pytest.mark.parametrize("name", ["train_bf16_k8", "tiny_f32"])
def test_noalloc_matches_workspace_backward_twice(cuda, name):
    torch = cuda
    import deformable_convolution_sampling_b200 as dcn
    w = gen.WORKLOADS[name]
    if name == "train_bf16_k8":
        w = dataclasses.replace(w, N=16)
    inp = gen.make_inputs(w)
    p = params_for(w)
    v, om, gy = (to_device(inp[k], w.dtype) for k in ("value", "offset_mask", "grad_out"))
    assert dcn.dcn4_backward_workspace_size(p) <= dcn.dcn4_backward_noalloc_capacity()
    ref_gv, ref_gom = dcn.backward(p, v, om, gy)
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):                                  # the area keeps the last call's contents
        gv = torch.full_like(ref_gv, float("nan"))
        gom = torch.full_like(ref_gom, float("nan"))
        st = dcn.dcn4_backward_noalloc(p, v.data_ptr(), om.data_ptr(), gy.data_ptr(), gv.data_ptr(),
                                       gom.data_ptr(), stream)
        assert st == 0, dcn.dcn4_noalloc_last_error() or dcn.dcn4_last_error()
        torch.cuda.synchronize()
        a, b = to_f64(gv), to_f64(ref_gv)
        assert np.all(np.isfinite(a))
        assert normwise(a, b) <= BWD_TOL[w.dtype]
        assert normwise(to_f64(gom), to_f64(ref_gom)) <= BWD_TOL[w.dtype]


def test_noalloc_rejects_problems_beyond_its_area(cuda):
    import deformable_convolution_sampling_b200 as dcn
    p = dcn.make_params(N=512, H=112, W=112, G=4, Cg=16, dtype="f16")
    assert dcn.dcn4_backward_workspace_size(p) > dcn.dcn4_backward_noalloc_capacity()
    st = dcn.dcn4_backward_noalloc(p, 256, 512, 768, 1024, 1280, None)
    assert st == -6
    assert "scratch" in dcn.dcn4_noalloc_last_error()
