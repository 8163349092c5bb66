"""Helpers shared by the GPU parity tests: move seeded inputs to the device,
run the CUDA path through the C ABI and the oracle on the same buffers, and
measure the error the way the tolerances are stated."""
from __future__ import annotations

import numpy as np

import dcn4_inputs as gen
import oracle

# Tolerances of the operator's specification, normwise: max|gpu - ref| / max|ref|.
FWD_TOL = {"f32": 1e-5, "f16": 2e-2, "bf16": 2e-2}
BWD_TOL = {"f32": 1e-4, "f16": 3e-2, "bf16": 3e-2}


def to_device(a: np.ndarray, dtype: str):
    import torch
    a = np.ascontiguousarray(a)
    if dtype == "bf16":
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(a)
    return t.cuda()


def to_f64(t) -> np.ndarray:
    import torch
    return t.detach().to(torch.float64).cpu().numpy()


def params_for(w: gen.Workload, dtype: str | None = None):
    """The workload's dcn4_params, after checking that the library's output grid is the
    one the workload's tensors are sized for."""
    import deformable_convolution_sampling_b200 as dcn
    p = dcn.make_params(dtype=dtype or w.dtype, **w.geometry())
    st, Ho, Wo = dcn.dcn4_output_dims(p)
    assert st == 0 and (Ho, Wo) == (w.Ho, w.Wo), f"{w.name}: the library's output is {Ho}x{Wo}, not {w.Ho}x{w.Wo}"
    return p


def problem_for(w: gen.Workload, n: int | None = None, dtype: str | None = None) -> oracle.Problem:
    geo = w.geometry()
    if n is not None:
        geo["N"] = n
    return oracle.Problem(dtype=dtype or w.dtype, location_fp32=True, **geo)


def gpu_forward(w: gen.Workload, inp: dict):
    import deformable_convolution_sampling_b200 as dcn
    p = params_for(w)
    return dcn.forward(p, to_device(inp["value"], w.dtype), to_device(inp["offset_mask"], w.dtype))


def gpu_backward(w: gen.Workload, inp: dict):
    """The backward through the C ABI; also checks that no grad_value tile found its
    filed sample records inconsistent (the kernel's fallback counter stays 0)."""
    import torch
    import deformable_convolution_sampling_b200 as dcn
    p = params_for(w)
    ws = torch.empty(max(dcn.dcn4_backward_workspace_size(p), 16), dtype=torch.uint8, device="cuda")
    out = dcn.backward(p, to_device(inp["value"], w.dtype), to_device(inp["offset_mask"], w.dtype),
                       to_device(inp["grad_out"], w.dtype), workspace=ws)
    if p.N > 0:
        diag = dcn.backward_diagnostics(p, ws)
        assert diag["corrupt_bucket_tiles"] == 0, diag
    return out


def take(inp: dict, idx) -> dict:
    return {k: np.ascontiguousarray(v[idx]) for k, v in inp.items()}


def oracle_forward(w: gen.Workload, inp: dict) -> np.ndarray:
    return oracle.forward(problem_for(w, n=inp["value"].shape[0]), inp["value"], inp["offset_mask"],
                          nthreads=oracle.host_threads())


def oracle_backward(w: gen.Workload, inp: dict):
    return oracle.backward(problem_for(w, n=inp["value"].shape[0]), inp["value"], inp["offset_mask"],
                           inp["grad_out"], nthreads=oracle.host_threads())


def normwise(got: np.ndarray, ref: np.ndarray) -> float:
    scale = float(np.max(np.abs(ref))) if ref.size else 0.0
    err = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    if scale == 0.0:
        return err
    return err / scale
