"""Host-side checks of the torch.autograd wrapper: every argument error is a
ValueError raised before anything reaches a GPU."""
import pytest

torch = pytest.importorskip("torch")
dcn = pytest.importorskip("deformable_convolution_sampling_b200")


def _t(*shape, dtype=torch.float32):
    return torch.zeros(*shape, dtype=dtype)


@pytest.mark.parametrize("value,om,kw,msg", [
    (_t(1, 8, 8), _t(1, 8, 8, 56), dict(group=2), "N,H,W,C"),
    (_t(1, 8, 8, 16), _t(1, 8, 8, 56, dtype=torch.float16), dict(group=2), "same dtype"),
    (_t(1, 8, 8, 16).transpose(1, 2), _t(1, 8, 8, 56), dict(group=2), "contiguous"),
    (_t(1, 8, 8, 16), _t(1, 8, 8, 56), dict(group=3), "multiple of group"),
    (_t(1, 8, 8, 16), _t(1, 8, 8, 56), dict(group=2), "CUDA tensors"),
])
def test_argument_errors(value, om, kw, msg):
    with pytest.raises(ValueError, match=msg):
        dcn.dcnv4_core(value, om, **kw)


def test_float64_is_refused():
    with pytest.raises(ValueError):
        dcn._dtype_code(_t(1, dtype=torch.float64))


@pytest.mark.parametrize("x,w,b,msg", [
    (_t(1, 8, 8, 64, dtype=torch.float16), _t(56, 64, 1, dtype=torch.float16), None, "weight"),
    (_t(1, 8, 8, 32, dtype=torch.float16), _t(56, 64, dtype=torch.float16), None, "weight"),
    (_t(1, 8, 8, 64, dtype=torch.float16), _t(56, 64, dtype=torch.float16), _t(55, dtype=torch.float16), "bias"),
    (_t(1, 8, 8, 64), _t(56, 64, dtype=torch.float16), None, "dtype"),
    (_t(1, 8, 8, 64, dtype=torch.float16), _t(56, 64, dtype=torch.float16), None, "CUDA tensors"),
])
def test_linear_argument_errors(x, w, b, msg):
    value = _t(1, 8, 8, 16, dtype=torch.float16)
    with pytest.raises(ValueError, match=msg):
        dcn.dcnv4_core_linear(value, x, w, b, group=2)


@pytest.mark.parametrize("w,b,msg", [
    (_t(64, 16, 1, dtype=torch.float16), None, "weight"),
    (_t(64, 32, dtype=torch.float16), None, "weight"),
    (_t(64, 16, dtype=torch.float16), _t(63, dtype=torch.float16), "bias"),
    (_t(64, 16), None, "dtype"),
    (_t(64, 16, dtype=torch.float16).t().contiguous().t(), None, "contiguous"),
    (_t(64, 16, dtype=torch.float16), None, "CUDA tensors"),
])
def test_proj_argument_errors(w, b, msg):
    value = _t(1, 8, 8, 16, dtype=torch.float16)
    om = _t(1, 8, 8, 56, dtype=torch.float16)
    with pytest.raises(ValueError, match=msg):
        dcn.dcnv4_core_proj(value, om, w, b, group=2)
