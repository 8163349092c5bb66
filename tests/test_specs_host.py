"""Every workload spec of the GPU tests states output sizes, a point count and a row
length P that agree with the library's own geometry (dcn4_output_dims,
dcn4_num_points, dcn4_padded_offset_dim).  The tests size their tensors from the
spec while the kernels read and write the sizes the library computes, so a spec
that disagrees would hand a kernel tensors of the wrong size.  Host only."""
import importlib
import os
import sys

import pytest

import dcn4_inputs as gen

dcn = pytest.importorskip("deformable_convolution_sampling_b200")
sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

SPEC_LISTS = {
    "test_gpu_parity": ["VARIANTS"],
    "test_gpu_softmax": ["VARIANTS"],
    "test_gpu_linear": ["VARIANTS"],
    "test_gpu_linear_backward": ["VARIANTS"],
    "test_gpu_proj": ["VARIANTS"],
}
EXTRA_KEYS = ("Cx", "Cout", "bias")  # the test's own arguments, not geometry


def _specs():
    out = []
    for mod, names in SPEC_LISTS.items():
        m = importlib.import_module(mod)
        for n in names:
            for spec in getattr(m, n):
                out.append(pytest.param(spec, id=f"{mod}.{spec['name']}"))
    return out


@pytest.mark.parametrize("spec", _specs())
def test_variant_spec_matches_the_library(spec):
    w = gen.custom(**{k: v for k, v in spec.items() if k not in EXTRA_KEYS})
    p = dcn.make_params(dtype=w.dtype, **w.geometry())
    st, Ho, Wo = dcn.dcn4_output_dims(p)
    assert st == 0 and (Ho, Wo) == (w.Ho, w.Wo), f"{spec['name']}: library {Ho}x{Wo}, spec {w.Ho}x{w.Wo}"
    assert dcn.dcn4_num_points(p) == w.K
    assert w.P >= dcn.dcn4_padded_offset_dim(w.G, w.K) and w.P % 8 == 0


@pytest.mark.parametrize("name", sorted(gen.WORKLOADS))
def test_workload_matches_the_library(name):
    w = gen.WORKLOADS[name]
    p = dcn.make_params(dtype=w.dtype, **w.geometry())
    st, Ho, Wo = dcn.dcn4_output_dims(p)
    assert st == 0 and (Ho, Wo) == (w.Ho, w.Wo)
    assert dcn.dcn4_num_points(p) == w.K and w.P >= dcn.dcn4_padded_offset_dim(w.G, w.K)


@pytest.mark.parametrize("spec", [s for s in importlib.import_module("test_gpu_proj").VARIANTS],
                         ids=[s["name"] for s in importlib.import_module("test_gpu_proj").VARIANTS])
def test_projection_takes_every_test_shape(spec):
    """The fused projection forms every shape its GPU tests use (16-, 32- or 64-pixel full
    tiles on small and ragged maps too): with N = 0 the call runs its host checks and
    returns before any launch."""
    w = gen.custom(**{k: v for k, v in spec.items() if k not in EXTRA_KEYS})
    p = dcn.make_params(dtype=w.dtype, **{**w.geometry(), "N": 0})
    assert dcn.dcn4_forward_proj(p, spec["Cout"], None, None, None, None, None) == 0, dcn.dcn4_last_error()


@pytest.mark.parametrize("name,Cout", [("stage1_f16", 64), ("highres_f16", 64), ("train_bf16_k8", 64),
                                       ("stage3_bf16", 128)])
def test_projection_takes_the_workloads(name, Cout):
    w = gen.WORKLOADS[name]
    p = dcn.make_params(dtype=w.dtype, **{**w.geometry(), "N": 0})
    assert dcn.dcn4_forward_proj(p, Cout, None, None, None, None, None) == 0, dcn.dcn4_last_error()
    # one tile forms at most 128 outputs: the third-stage shape's own width is refused
    if w.C > 128:
        assert dcn.dcn4_forward_proj(p, w.C, None, None, None, None, None) == -5
