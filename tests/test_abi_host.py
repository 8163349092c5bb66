"""The C-ABI library loads, exports every declared symbol, and validates
calls on the host before touching a GPU (CPU only: no kernel is launched)."""
import ctypes
import os
import re
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dcn4.h")


@pytest.fixture(scope="module")
def dcn():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "dcn4_build", os.path.join(ROOT, "deformable_convolution_sampling_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    import deformable_convolution_sampling_b200 as d
    return d


def run_without_gpu(code: str):
    """Runs `code` (with `dcn`, the binding, imported) in a child process whose
    CUDA runtime sees no device, so that no address it passes can reach a GPU."""
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    prelude = "import sys; sys.path.insert(0, %r)\nimport deformable_convolution_sampling_b200 as dcn\n" % ROOT
    r = subprocess.run([sys.executable, "-c", prelude + code], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dcn4_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("dcn4_forward", "dcn4_backward", "dcn4_backward_workspace_size", "dcn4_output_dims",
                     "dcn4_padded_offset_dim", "dcn4_status_string", "dcn4_last_error", "dcn4_check_params"):
        assert required in names


def test_every_declared_symbol_is_exported(dcn):
    raw = ctypes.CDLL(dcn.LIB_PATH)
    for name in declared_functions():
        assert hasattr(raw, name), f"{name} declared in dcn4.h but not exported"
    out = subprocess.run(["nm", "-D", "--defined-only", dcn.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (dcn4_\w+)", out))
    assert exported == set(declared_functions()), exported ^ set(declared_functions())


def test_params_mirror_matches_the_header(dcn):
    """The binding's ctypes dcn4_params has the header's fields, in order, all 4 bytes."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    body = re.search(r"typedef struct \{(.*?)\} dcn4_params;", text, flags=re.S).group(1)
    fields = []
    for decl in body.split(";"):
        decl = decl.strip()
        if decl:
            ctype, names = decl.split(None, 1)
            assert ctype in ("int", "float"), decl
            fields += [n.strip() for n in names.split(",")]
    assert [f[0] for f in dcn.dcn4_params._fields_] == fields
    assert ctypes.sizeof(dcn.dcn4_params) == 4 * len(fields)
    assert dcn.dcn4_version() == 160


def test_attn_params_mirror_matches_the_header(dcn):
    """The binding's ctypes dcn4_attn_params has the header's fields, in order, all 4 bytes."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    body = re.search(r"typedef struct \{([^}]*)\} dcn4_attn_params;", text, flags=re.S).group(1)
    fields = []
    for decl in body.split(";"):
        decl = decl.strip()
        if decl:
            ctype, names = decl.split(None, 1)
            assert ctype in ("int", "float"), decl
            fields += [n.strip() for n in names.split(",")]
    assert [f[0] for f in dcn.dcn4_attn_params._fields_] == fields
    assert ctypes.sizeof(dcn.dcn4_attn_params) == 4 * len(fields)


@pytest.mark.parametrize("field,value,status", [
    ("dtype", 5, -8), ("N", -1, -2), ("H", 0, -2), ("G", 0, -2), ("Cg", 0, -2), ("Nq", -1, -2), ("K", 0, -2),
    ("P", 16, -3), ("P", 50, -3), ("Cg", 4, -5), ("Cg", 24, -5), ("K", 2000, -5), ("H", 1 << 24, -5),
])
def test_attn_invalid_params_are_rejected_before_launch(dcn, field, value, status):
    p = dcn.make_attn_params(N=2, H=8, W=8, G=2, Cg=8, Nq=10, K=4, dtype="f16")
    setattr(p, field, value)
    assert dcn.dcn4_attn_check_params(p) == status
    assert dcn.dcn4_attn_forward(p, None, None, None, None, None) == status
    assert dcn.dcn4_attn_backward(p, None, None, None, None, None, None, None, 0, None) == status


def test_attn_workspace_and_null_pointers():
    """Workspace size (an fp32 grad_value accumulator for 16-bit I/O, none for fp32) and
    the NULL / misaligned / missing-workspace refusals (made-up addresses: checked in a
    child process that sees no GPU)."""
    run_without_gpu("""
p = dcn.make_attn_params(N=2, H=8, W=8, G=2, Cg=8, Nq=10, K=4, dtype="f16")
assert dcn.dcn4_attn_check_params(p) == 0
assert dcn.dcn4_attn_backward_workspace_size(p) == 2 * 8 * 8 * 16 * 4
assert dcn.dcn4_attn_backward_workspace_size(dcn.make_attn_params(N=2, H=8, W=8, G=2, Cg=8, Nq=10, K=4, dtype="f32")) == 0
assert dcn.dcn4_attn_forward(p, None, 32, 48, 64, None) == -1
assert dcn.dcn4_attn_forward(p, 16, 36, 48, 64, None) == -4
assert dcn.dcn4_attn_backward(p, 16, 32, 48, 64, 80, 96, None, 0, None) == -6
assert dcn.dcn4_attn_backward(p, 16, 32, 48, 64, 80, 96, 112, 100, None) == -6
assert dcn.dcn4_attn_backward(p, 16, 32, 48, 64, None, 96, 112, 1 << 20, None) == -1
empty = dcn.make_attn_params(N=0, H=8, W=8, G=2, Cg=8, Nq=10, K=4, dtype="f16")
assert dcn.dcn4_attn_forward(empty, None, None, None, None, None) == 0
""")


def test_library_does_not_link_the_oracle(dcn):
    out = subprocess.run(["ldd", dcn.LIB_PATH], capture_output=True, text=True).stdout
    assert "oracle" not in out
    syms = subprocess.run(["nm", "-D", dcn.LIB_PATH], capture_output=True, text=True).stdout
    assert "ref_forward" not in syms and "ref_backward" not in syms


def test_padded_offset_dim_and_points(dcn):
    assert dcn.dcn4_padded_offset_dim(2, 9) == 56
    assert dcn.dcn4_padded_offset_dim(4, 9) == 112
    assert dcn.dcn4_padded_offset_dim(16, 9) == 432
    assert dcn.dcn4_padded_offset_dim(4, 8) == 96
    assert dcn.dcn4_padded_offset_dim(0, 9) < 0
    p = dcn.make_params(N=1, H=8, W=8, G=2, Cg=8, remove_center=1, dtype="f32")
    assert dcn.dcn4_num_points(p) == 8


def test_output_dims_agree_with_the_oracle(dcn):
    import oracle
    for (kh, kw, sh, sw, ph, pw, dh, dw) in [(3, 3, 1, 1, 1, 1, 1, 1), (3, 5, 2, 1, 0, 2, 2, 1),
                                             (1, 3, 3, 2, 0, 0, 1, 3), (5, 5, 2, 2, 2, 2, 1, 1)]:
        for H, W in [(7, 9), (16, 5), (33, 33)]:
            geo = dict(N=1, H=H, W=W, G=2, Cg=8, kh=kh, kw=kw, sh=sh, sw=sw, ph=ph, pw=pw, dh=dh, dw=dw)
            try:
                want = oracle.output_dims(oracle.Problem(dtype="f32", **geo))
            except ValueError:
                want = None
            st, ho, wo = dcn.dcn4_output_dims(dcn.make_params(dtype="f16", **geo))
            if want is None:
                assert st == -2
            else:
                assert st == 0 and (ho, wo) == want


def test_workspace_size(dcn):
    """Per image a reach word, per output pixel a cell box; then per sample a 2-byte cell code
    (fp32), or (16-bit dtypes) a record counter per grad_value tile and each tile's bucket of
    12-byte records; each array starts on a 256-byte boundary."""
    def up(x):
        return (x + 255) // 256 * 256
    p = dcn.make_params(N=64, H=56, W=56, G=4, Cg=16, dtype="f16")
    # grad_value tiles of 8 x 31 pixels: 7 x 2 per image; bucket room for 1.0625x the expected
    # records (K per cell and group, (8+1) x (31+1) cells, 4 groups) + 512
    tiles = 64 * 7 * 2
    expect = 4 * 9 * 32 * 9
    cap = expect + expect // 16 + 512
    header = up((4 + 64 + tiles) * 4)          # counters, reach words, bucket counters
    assert dcn.dcn4_backward_workspace_size(p) == (header + up(64 * 56 * 56 * 4)
                                                   + up(tiles * cap * 4) + tiles * cap * 8)
    p = dcn.make_params(N=100, H=8, W=8, G=2, Cg=8, dtype="f32", remove_center=1)
    assert dcn.dcn4_backward_workspace_size(p) == up((4 + 100) * 4) + up(100 * 64 * 4) + up(100 * 64 * 2 * 8 * 2)
    p.Cg = 6
    assert dcn.dcn4_backward_workspace_size(p) == 0


@pytest.mark.parametrize("field,value,status", [
    ("dtype", 7, -8), ("N", -1, -2), ("H", 0, -2), ("G", 0, -2), ("Cg", 0, -2), ("kh", 0, -2),
    ("sh", 0, -2), ("ph", -1, -2), ("dh", 0, -2), ("remove_center", 2, -2), ("softmax", 2, -2), ("softmax", -1, -2), ("P", 50, -3),
    ("P", 60, -3), ("Cg", 4, -5), ("Cg", 24, -5), ("Cg", 48, -5), ("H", 1 << 24, -5),
])
def test_invalid_params_are_rejected_before_launch(dcn, field, value, status):
    p = dcn.make_params(N=2, H=8, W=8, G=2, Cg=8, dtype="f16")
    setattr(p, field, value)
    assert dcn.dcn4_check_params(p) == status
    # NULL tensors: the parameter check must answer first (a regression would
    # return DCN4_ERR_NULL instead, still without a launch)
    assert dcn.dcn4_forward(p, None, None, None, None) == status
    assert dcn.dcn4_last_error() != ""


def test_forward_linear_checks_before_launch():
    """dcn4_forward_linear validates on the host.  The checks need non-NULL
    (made-up, never dereferenced) addresses, so they run in a child process that
    sees no GPU: should a check ever regress, the launch fails with "no device"
    instead of reaching a GPU with those addresses."""
    run_without_gpu("""
p = dcn.make_params(N=2, H=8, W=8, G=4, Cg=16, dtype="f16")
ok = dict(value=16, x=32, weight=48, bias=None, out=64, om=None)

def call(params, Cx, **kw):
    a = {**ok, **kw}
    return dcn.dcn4_forward_linear(params, Cx, a["value"], a["x"], a["weight"], a["bias"], a["out"], a["om"],
                                   None)
p32 = dcn.make_params(N=2, H=8, W=8, G=4, Cg=16, dtype="f32")
assert call(p32, 64) == -5                      # fp32: no fused producer
assert call(p, 24) == -2 and call(p, 0) == -2   # Cx not a multiple of 16
assert call(p, 1 << 14) == -5                   # x tiles too large for shared memory
assert call(p, 64, x=None) == -1
assert call(p, 64, bias=40) == -4 and call(p, 64, om=72) == -4 and call(p, 64, x=36) == -4
bad = dcn.make_params(N=2, H=8, W=8, G=4, Cg=16, dtype="f16")
bad.P = 100
assert call(bad, 64) == -3
assert dcn.dcn4_last_error() != ""
""")


def test_backward_linear_checks_before_launch():
    """dcn4_backward_linear validates on the host before its first launch (made-up
    addresses: checked in a child process that sees no GPU)."""
    run_without_gpu("""
p = dcn.make_params(N=2, H=8, W=8, G=4, Cg=16, dtype="bf16")
need = dcn.dcn4_backward_linear_workspace_size(p, 64)
assert need >= dcn.dcn4_backward_workspace_size(p) + 4 * (p.P * 64 + p.P)
assert need % 256 == 0 and dcn.dcn4_backward_linear_workspace_size(p, 0) == 0
ok = dict(value=16, om=32, x=48, w=64, gy=80, gv=96, gom=112, gx=128, gw=144, gb=160, ws=4096, nb=need)

def call(params, Cx, **kw):
    a = {**ok, **kw}
    return dcn.dcn4_backward_linear(params, Cx, a["value"], a["om"], a["x"], a["w"], a["gy"], a["gv"], a["gom"],
                                    a["gx"], a["gw"], a["gb"], a["ws"], a["nb"], None)
p32 = dcn.make_params(N=2, H=8, W=8, G=4, Cg=16, dtype="f32")
assert call(p32, 64, nb=1 << 24) == -5              # fp32: no linear producer
assert call(p, 24) == -2 and call(p, 0) == -2       # Cx not a multiple of 16
assert call(p, 64, nb=need - 1) == -6 and call(p, 64, ws=None) == -6
assert call(p, 64, ws=4100) == -4                   # misaligned workspace
assert call(p, 64, gw=148) == -4 and call(p, 64, x=52) == -4 and call(p, 64, gb=161) == -4
assert call(p, 64, gom=None) == -1
assert call(p, 64, w=None) == -1 and call(p, 64, x=None) == -1
assert call(p, 64, value=None) == -1 and call(p, 64, gv=None) == -1
bad = dcn.make_params(N=2, H=8, W=8, G=4, Cg=16, dtype="bf16")
bad.P = 100
assert call(bad, 64) == -3
# the tensor-map row coordinates are 32-bit: N*Ho*Wo must stay below 2^31
big = dcn.make_params(N=2048, H=1024, W=1024, G=4, Cg=16, dtype="bf16")
assert call(big, 64, nb=1 << 62) == -5 and "2^31" in dcn.dcn4_last_error()
assert dcn.dcn4_last_error() != ""
""")


def test_forward_proj_checks_before_launch():
    """dcn4_forward_proj validates on the host (made-up addresses: checked in a child
    process that sees no GPU)."""
    run_without_gpu("""
p = dcn.make_params(N=2, H=8, W=8, G=4, Cg=16, dtype="f16")
ok = dict(value=16, om=32, w=48, b=None, out=64, core=None)

def call(params, Cout, **kw):
    a = {**ok, **kw}
    return dcn.dcn4_forward_proj(params, Cout, a["value"], a["om"], a["w"], a["b"], a["out"], a["core"], None)
p32 = dcn.make_params(N=2, H=8, W=8, G=4, Cg=16, dtype="f32")
assert call(p32, 64) == -5                                           # fp32: no fused projection
assert call(p, 24) == -2 and call(p, 0) == -2 and call(p, 8) == -2   # Cout not a multiple of 16
assert call(p, 144) == -5 and "128" in dcn.dcn4_last_error()         # more outputs than one tile forms
c32 = dcn.make_params(N=2, H=8, W=8, G=2, Cg=16, dtype="f16")
assert call(c32, 64) == -5 and "multiple of 64" in dcn.dcn4_last_error()
c512 = dcn.make_params(N=2, H=8, W=8, G=32, Cg=16, dtype="f16")
assert call(c512, 64) == -5
assert call(p, 64, w=None) == -1 and call(p, 64, om=None) == -1 and call(p, 64, out=None) == -1
assert call(p, 64, b=40) == -4 and call(p, 64, core=72) == -4 and call(p, 64, w=52) == -4
bad = dcn.make_params(N=2, H=8, W=8, G=4, Cg=16, dtype="f16")
bad.P = 100
assert call(bad, 64) == -3
assert dcn.dcn4_last_error() != ""
""")


def test_backward_proj_checks_before_launch():
    """dcn4_backward_proj validates on the host before its first launch (made-up
    addresses: checked in a child process that sees no GPU)."""
    run_without_gpu("""
p = dcn.make_params(N=2, H=8, W=8, G=4, Cg=16, dtype="bf16")
need = dcn.dcn4_backward_proj_workspace_size(p, 64)
assert need >= dcn.dcn4_backward_workspace_size(p) + 2 * 8 * 8 * 64 * 2 + 4 * (64 * 64 + 64)
assert need % 256 == 0 and dcn.dcn4_backward_proj_workspace_size(p, 0) == 0
ok = dict(value=16, om=32, core=48, w=64, gy=80, gv=96, gom=112, gw=144, gb=160, ws=4096, nb=need)

def call(params, Cout, **kw):
    a = {**ok, **kw}
    return dcn.dcn4_backward_proj(params, Cout, a["value"], a["om"], a["core"], a["w"], a["gy"], a["gv"], a["gom"],
                                  a["gw"], a["gb"], a["ws"], a["nb"], None)
p32 = dcn.make_params(N=2, H=8, W=8, G=4, Cg=16, dtype="f32")
assert call(p32, 64, nb=1 << 24) == -5              # fp32: no projection
assert call(p, 24) == -2 and call(p, 0) == -2       # Cout not a multiple of 16
c8 = dcn.make_params(N=2, H=8, W=8, G=1, Cg=8, dtype="bf16", P=32)
assert call(c8, 64, nb=1 << 24) == -2               # C not a multiple of 16
assert call(p, 64, nb=need - 1) == -6 and call(p, 64, ws=None) == -6
assert call(p, 64, ws=4100) == -4                   # misaligned workspace
assert call(p, 64, gw=148) == -4 and call(p, 64, core=52) == -4 and call(p, 64, gb=161) == -4
assert call(p, 64, gom=None) == -1 and call(p, 64, gv=None) == -1
assert call(p, 64, w=None) == -1 and call(p, 64, gy=None) == -1
assert call(p, 64, value=None) == -1 and call(p, 64, om=None) == -1
assert call(p, 64, value=20) == -4 and call(p, 64, gv=100) == -4
assert call(p, 64, core=None) == -1 and "core_out" in dcn.dcn4_last_error()
bad = dcn.make_params(N=2, H=8, W=8, G=4, Cg=16, dtype="bf16")
bad.P = 100
assert call(bad, 64) == -3
big = dcn.make_params(N=2048, H=1024, W=1024, G=4, Cg=16, dtype="bf16")
assert call(big, 64, nb=1 << 62) == -5 and "2^31" in dcn.dcn4_last_error()
""")


def test_remove_center_needs_odd_kernel(dcn):
    p = dcn.make_params(N=1, H=8, W=8, G=2, Cg=8, kh=2, kw=3, ph=0, dtype="f16", P=48)
    p.remove_center = 1
    assert dcn.dcn4_check_params(p) == -2


def test_null_and_misaligned_pointers():
    """NULL, misaligned and missing-workspace arguments are refused on the host
    (made-up addresses: checked in a child process that sees no GPU)."""
    run_without_gpu("""
p = dcn.make_params(N=1, H=8, W=8, G=2, Cg=8, dtype="f16")
assert dcn.dcn4_forward(p, None, 16, 32, None) == -1
assert dcn.dcn4_forward(p, 16, 18, 32, None) == -4
assert dcn.dcn4_backward(p, 16, 32, 48, 64, None, 96, 1 << 20, None) == -1
assert dcn.dcn4_backward(p, 16, 32, 48, 64, 80, 97, 1 << 20, None) == -4
assert dcn.dcn4_backward(p, 16, 32, 48, 64, 80, None, 0, None) == -6
assert dcn.dcn4_backward(p, 16, 32, 48, 64, 80, 96, 100, None) == -6
assert dcn.lib.dcn4_forward(None, None, None, None, None) == -1
""")


def test_diagnostics_checks_before_reading():
    """dcn4_backward_diagnostics validates its arguments on the host (NULL counts,
    missing or small workspace) before any copy; made-up addresses only in a child
    process that sees no GPU."""
    run_without_gpu("""
import ctypes
p = dcn.make_params(N=2, H=8, W=8, G=2, Cg=8, dtype="f16")
st, c = dcn.dcn4_backward_diagnostics(p, None, 0)
assert st == -6 and c == [0, 0, 0], (st, c)
st, c = dcn.dcn4_backward_diagnostics(p, 256, 100)
assert st == -6, st
st, c = dcn.dcn4_backward_diagnostics(p, 264, 1 << 24)
assert st == -4, st
assert dcn.lib.dcn4_backward_diagnostics(ctypes.byref(p), None, 0, None, None) == -1
bad = dcn.make_params(N=2, H=8, W=8, G=2, Cg=8, dtype="f16")
bad.P = 50
st, c = dcn.dcn4_backward_diagnostics(bad, None, 0)
assert st == -3, st
""")


def test_child_process_sees_no_gpu():
    """The isolation the checks above rely on: with CUDA_VISIBLE_DEVICES empty the
    library's CUDA runtime finds no device (the no-allocation entry point's device
    look-up fails; every pointer argument is NULL)."""
    run_without_gpu("""
p = dcn.make_params(N=1, H=8, W=8, G=2, Cg=8, dtype="f16")
st = dcn.dcn4_backward_noalloc(p, None, None, None, None, None, None)
assert st == -7, st                               # DCN4_ERR_LAUNCH: no usable device
assert "device" in dcn.dcn4_noalloc_last_error()
""")


def test_status_strings(dcn):
    for code, name in dcn.STATUS.items():
        assert dcn.dcn4_status_string(code) == name


def test_missing_library_fails_loudly(tmp_path):
    pkg = tmp_path / "deformable_convolution_sampling_b200"
    pkg.mkdir()
    shutil.copy(os.path.join(ROOT, "deformable_convolution_sampling_b200", "__init__.py"), pkg)
    r = subprocess.run([sys.executable, "-c", "import deformable_convolution_sampling_b200"], cwd=tmp_path,
                       capture_output=True, text=True)
    assert r.returncode != 0 and "ImportError" in r.stderr and "no CPU fallback" in r.stderr


def _code_only(path: str) -> str:
    """Source text without // and /* */ comments."""
    text = open(path).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.sub(r"//[^\n]*", "", text)


def test_backward_path_allocates_nothing():
    """dcn4_backward_noalloc promises no device allocation: no source on the
    backward's call path (the entry point, the C ABI, the backward kernels and
    their shared helpers) names an allocating or freeing CUDA call."""
    csrc = os.path.join(ROOT, "deformable_convolution_sampling_b200", "csrc")
    pattern = re.compile(r"\b(cudaMalloc\w*|cudaFree\w*|cuMemAlloc\w*|cuMemFree\w*|cudaHostAlloc|cudaMemPool\w*)\b")
    for name in ("dcn4_noalloc.cu", "dcn4_api.cu", "dcn4_backward.cu", "dcn4_common.cuh"):
        found = pattern.findall(_code_only(os.path.join(csrc, name)))
        assert not found, f"{name} calls {sorted(set(found))}"
