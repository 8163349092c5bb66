"""Seeded synthetic inputs for the DCNv4 core operator.

This module is the only code the CPU oracle and the CUDA path have in common:
it draws numbers and lays them out, and holds none of the operator's
arithmetic.

Random numbers come from a counter-based generator: SplitMix64 (Steele, Lea &
Flood, "Fast splittable pseudorandom number generators", OOPSLA 2014) applied
to ``seed * K1 + (stream << 40 | index + 1) * golden``, so every element is a
pure function of (seed, stream, index) and any slice can be regenerated
without the rest.  Uniforms take the top 53 bits; normals use the Box-Muller
transform.  Values are drawn in float64 and rounded once to the storage type
(round to nearest, ties to even):

    "f32"  -> numpy float32
    "f16"  -> numpy float16
    "bf16" -> numpy uint16 holding bfloat16 bit patterns
    "f64"  -> numpy float64

Workloads.  ``WORKLOADS`` lists the five shapes this library is measured and
parity-tested on: a tiny fp32 case, the first- and third-stage backbone
feature maps of a 224x224 hierarchical backbone, a high-resolution
dense-prediction map and a remove_center training step.  Distribution
parameters are (mean, standard deviation) for normals and (low, high) for
uniforms.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_SEED_MUL = np.uint64(0xD1342543DE82EF95)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

STREAM_VALUE, STREAM_OFFSET, STREAM_MASK, STREAM_GRAD = 1, 2, 3, 4
STREAM_X, STREAM_WEIGHT, STREAM_BIAS = 5, 6, 7
STREAM_REF = 8
STREAM_PROJ_WEIGHT, STREAM_PROJ_BIAS, STREAM_PROJ_GRAD = 9, 10, 11


def _splitmix64(z: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        return z ^ (z >> np.uint64(31))


def _bits(seed: int, stream: int, start: int, n: int) -> np.ndarray:
    ctr = np.arange(start, start + n, dtype=np.uint64) + np.uint64(1)
    ctr = ctr | (np.uint64(stream) << np.uint64(40))
    with np.errstate(over="ignore"):
        z = np.uint64(seed) * _SEED_MUL + ctr * _GOLDEN
    return _splitmix64(z)


def uniform01(seed: int, stream: int, n: int, start: int = 0) -> np.ndarray:
    """n doubles in (0, 1]: (top 53 bits + 1) * 2^-53."""
    b = _bits(seed, stream, start, n) >> np.uint64(11)
    return (b.astype(np.float64) + 1.0) * (2.0 ** -53)


def uniform(seed: int, stream: int, n: int, low: float, high: float) -> np.ndarray:
    return low + (high - low) * uniform01(seed, stream, n)


def normal(seed: int, stream: int, n: int, mean: float, std: float) -> np.ndarray:
    """Box-Muller on two sub-streams (2*stream, 2*stream+1)."""
    u1 = uniform01(seed, 2 * stream, n)
    u2 = uniform01(seed, 2 * stream + 1, n)
    z = np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)
    return mean + std * z


def draw(dist: tuple, seed: int, stream: int, n: int) -> np.ndarray:
    kind, a, b = dist
    if kind == "normal":
        return normal(seed, stream, n, a, b)
    if kind == "uniform":
        return uniform(seed, stream, n, a, b)
    raise ValueError(f"unknown distribution {dist}")


# ---------------------------------------------------------------------------
# Storage rounding
# ---------------------------------------------------------------------------

def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float64 to bfloat16 (8 significant bits, nearest-even) -> uint16 bits."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                          # x = m * 2^e, 0.5 <= |m| < 1
    r = np.ldexp(np.rint(m * 256.0) / 256.0, e)  # np.rint: ties to even
    tiny = np.abs(x) < 2.0 ** -126               # bfloat16 subnormal range: round the fp32 bits
    f = r.astype(np.float32)
    bits = (f.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    if np.any(tiny):
        t = x[tiny].astype(np.float32).view(np.uint32)
        lsb = (t >> np.uint32(16)) & np.uint32(1)
        t = (t + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
        bits[tiny] = t.astype(np.uint16)
    nan = np.isnan(x)
    if np.any(nan):
        bits[nan] = np.uint16(0x7FC0)
    return bits


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def to_storage(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f64":
        return np.asarray(x, dtype=np.float64)
    if dtype == "f32":
        return np.asarray(x, dtype=np.float64).astype(np.float32)
    if dtype == "f16":
        return np.asarray(x, dtype=np.float64).astype(np.float16)
    if dtype == "bf16":
        return f64_to_bf16_bits(x)
    raise ValueError(dtype)


def storage_to_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return bf16_bits_to_f64(a)
    return np.asarray(a).astype(np.float64)


# ---------------------------------------------------------------------------
# Workloads
# ---------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    N: int
    H: int
    W: int
    G: int
    Cg: int
    Ho: int
    Wo: int
    K: int
    P: int
    dtype: str
    value: tuple
    offset: tuple
    mask: tuple
    grad_out: tuple = ("normal", 0.0, 1.0)
    kh: int = 3
    kw: int = 3
    sh: int = 1
    sw: int = 1
    ph: int = 1
    pw: int = 1
    dh: int = 1
    dw: int = 1
    offset_scale: float = 1.0
    remove_center: int = 0
    softmax: int = 0          # masks are logits normalised over the K points
    seed: int = 0
    passes: str = "fwd"
    note: str = ""

    @property
    def C(self) -> int:
        return self.G * self.Cg

    def geometry(self) -> dict:
        """Keyword arguments shared by the oracle's Problem and the library's params."""
        return dict(N=self.N, H=self.H, W=self.W, G=self.G, Cg=self.Cg, kh=self.kh, kw=self.kw,
                    sh=self.sh, sw=self.sw, ph=self.ph, pw=self.pw, dh=self.dh, dw=self.dw,
                    offset_scale=self.offset_scale, remove_center=self.remove_center, P=self.P,
                    softmax=self.softmax)

    def describe(self) -> str:
        rc = (" remove_center" if self.remove_center else "") + (" softmax" if self.softmax else "")
        return (f"N{self.N} H{self.H} W{self.W} C{self.C} G{self.G} (C'={self.Cg}) "
                f"{self.kh}x{self.kw} s{self.sh} p{self.ph} d{self.dh} K{self.K} P{self.P} "
                f"offset_scale {self.offset_scale}{rc} {self.dtype}")


WORKLOADS: dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("tiny_f32", N=1, H=8, W=8, G=2, Cg=8, Ho=8, Wo=8, K=9, P=56, dtype="f32",
                 value=("normal", 0.0, 1.0), offset=("uniform", -2.0, 2.0), mask=("normal", 0.0, 1.0),
                 passes="fwd+bwd", note="tiny fp32 forward+backward"),
        Workload("stage1_f16", N=64, H=56, W=56, G=4, Cg=16, Ho=56, Wo=56, K=9, P=112, dtype="f16",
                 value=("normal", 0.0, 1.0), offset=("normal", 0.0, 1.5), mask=("normal", 0.0, 0.5),
                 note="first-stage backbone feature map, fp16"),
        Workload("stage3_bf16", N=64, H=14, W=14, G=16, Cg=16, Ho=14, Wo=14, K=9, P=432, dtype="bf16",
                 value=("normal", 0.0, 1.0), offset=("normal", 0.0, 1.5), mask=("normal", 0.0, 0.5),
                 note="third-stage backbone feature map, bf16"),
        Workload("highres_f16", N=2, H=200, W=304, G=4, Cg=16, Ho=200, Wo=304, K=9, P=112, dtype="f16",
                 value=("normal", 0.0, 1.0), offset=("uniform", -8.0, 8.0), mask=("normal", 0.0, 1.0),
                 note="high-resolution dense-prediction map, fp16"),
        Workload("train_bf16_k8", N=64, H=56, W=56, G=4, Cg=16, Ho=56, Wo=56, K=8, P=96, dtype="bf16",
                 value=("normal", 0.0, 1.0), offset=("normal", 0.0, 2.0), mask=("normal", 0.0, 0.5),
                 offset_scale=0.5, remove_center=1, passes="fwd+bwd",
                 note="training step with remove_center, bf16"),
    ]
}

WORKLOAD_ORDER = ["tiny_f32", "stage1_f16", "stage3_bf16", "highres_f16", "train_bf16_k8"]


def _fill_value(dtype: str, fill: float) -> np.ndarray:
    return to_storage(np.array([fill], dtype=np.float64), dtype)[0]


def assemble_offset_mask(offsets: np.ndarray, masks: np.ndarray, P: int, dtype: str,
                         tail_fill: float = math.nan) -> np.ndarray:
    """Lay out [..., G, K, 2] offsets (dx, dy) and [..., G, K] masks into P-wide rows.

    Group g owns entries [g*3K, (g+1)*3K): its K (dx, dy) pairs, then its K
    masks; entries [G*3K, P) are the padding tail, filled with ``tail_fill``.
    Both inputs must already be in storage form.
    """
    lead = offsets.shape[:-3]
    G, K = offsets.shape[-3], offsets.shape[-2]
    if masks.shape != lead + (G, K):
        raise ValueError("offsets / masks shape mismatch")
    if P < G * 3 * K:
        raise ValueError("P too small")
    om = np.empty(lead + (P,), dtype=offsets.dtype)
    body = om[..., : G * 3 * K].reshape(lead + (G, 3 * K))
    body[..., : 2 * K] = offsets.reshape(lead + (G, 2 * K))
    body[..., 2 * K:] = masks
    om[..., G * 3 * K:] = _fill_value(dtype, tail_fill)
    return om


def make_inputs(w: Workload, *, seed: int | None = None, tail_fill: float = math.nan,
                with_grad: bool = True, dtype: str | None = None) -> dict:
    """value [N,H,W,C], offset_mask [N,Ho,Wo,P] and (optionally) grad_out [N,Ho,Wo,C]."""
    seed = w.seed if seed is None else seed
    dtype = w.dtype if dtype is None else dtype
    nval = w.N * w.H * w.W * w.C
    nsamp = w.N * w.Ho * w.Wo * w.G * w.K
    value = to_storage(draw(w.value, seed, STREAM_VALUE, nval), dtype).reshape(w.N, w.H, w.W, w.C)
    offs = to_storage(draw(w.offset, seed, STREAM_OFFSET, 2 * nsamp), dtype)
    offs = offs.reshape(w.N, w.Ho, w.Wo, w.G, w.K, 2)
    masks = to_storage(draw(w.mask, seed, STREAM_MASK, nsamp), dtype).reshape(w.N, w.Ho, w.Wo, w.G, w.K)
    out = {"value": value, "offset_mask": assemble_offset_mask(offs, masks, w.P, dtype, tail_fill)}
    if with_grad:
        ng = w.N * w.Ho * w.Wo * w.C
        out["grad_out"] = to_storage(draw(w.grad_out, seed, STREAM_GRAD, ng), dtype).reshape(
            w.N, w.Ho, w.Wo, w.C)
    return out


def make_linear_inputs(w: Workload, Cx: int, *, seed: int | None = None, bias: bool = True,
                       dtype: str | None = None) -> dict:
    """Inputs of the merged offset/mask linear layer in front of the aggregation:
    x [N,Ho,Wo,Cx] ~ N(0,1), weight [P,Cx] and bias [P] (or None), in storage form.
    Weight rows are drawn N(0, s^2 / Cx) so that each produced entry has about the
    spread of the workload's own offsets (offset rows) or masks (mask rows and the
    padding rows); bias ~ N(0, 0.1^2)."""
    seed = w.seed if seed is None else seed
    dtype = w.dtype if dtype is None else dtype
    x = to_storage(draw(("normal", 0.0, 1.0), seed, STREAM_X, w.N * w.Ho * w.Wo * Cx), dtype)
    row_sd = np.full(w.P, float(w.mask[2]) if w.mask[0] == "normal" else 0.5)
    off_sd = float(w.offset[2]) if w.offset[0] == "normal" else (w.offset[2] - w.offset[1]) / 12 ** 0.5
    for g in range(w.G):
        row_sd[g * 3 * w.K: g * 3 * w.K + 2 * w.K] = off_sd
    z = draw(("normal", 0.0, 1.0), seed, STREAM_WEIGHT, w.P * Cx).reshape(w.P, Cx)
    weight = to_storage(z * (row_sd[:, None] / np.sqrt(Cx)), dtype)
    out = {"x": x.reshape(w.N, w.Ho, w.Wo, Cx), "weight": weight, "bias": None}
    if bias:
        out["bias"] = to_storage(draw(("normal", 0.0, 0.1), seed, STREAM_BIAS, w.P), dtype)
    return out


def make_proj_inputs(w: Workload, Cout: int, *, seed: int | None = None, bias: bool = True,
                     with_grad: bool = True, dtype: str | None = None) -> dict:
    """The output projection behind the aggregation, in storage form: weight
    [Cout, C] ~ N(0, 1 / C) (so each output has about the spread of one core
    channel), bias [Cout] ~ N(0, 0.1^2) (or None) and, with_grad, the upstream
    gradient of its output grad_out [N, Ho, Wo, Cout] drawn like the workload's own."""
    seed = w.seed if seed is None else seed
    dtype = w.dtype if dtype is None else dtype
    z = draw(("normal", 0.0, 1.0), seed, STREAM_PROJ_WEIGHT, Cout * w.C).reshape(Cout, w.C)
    out = {"weight": to_storage(z / np.sqrt(w.C), dtype), "bias": None}
    if bias:
        out["bias"] = to_storage(draw(("normal", 0.0, 0.1), seed, STREAM_PROJ_BIAS, Cout), dtype)
    if with_grad:
        ng = w.N * w.Ho * w.Wo * Cout
        out["grad_out"] = to_storage(draw(w.grad_out, seed, STREAM_PROJ_GRAD, ng), dtype).reshape(
            w.N, w.Ho, w.Wo, Cout)
    return out


def custom(name: str = "custom", **kw) -> Workload:
    """A Workload for ad-hoc test shapes; Ho, Wo, K and P must be given explicitly."""
    base = dict(value=("normal", 0.0, 1.0), offset=("normal", 0.0, 1.5), mask=("normal", 0.0, 0.5))
    base.update(kw)
    return Workload(name=name, **base)


# ---------------------------------------------------------------------------
# Deformable attention (single scale): value [N,H,W,G*Cg], reference points
# ref [N,Nq,2] (fp32, (x, y) in pixel coordinates), offset_logits [N,Nq,P]
# (per group K (dx, dy) pairs, then K logits), grad_out [N,Nq,G*Cg].
# ---------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class AttnWorkload:
    name: str
    N: int
    H: int
    W: int
    G: int
    Cg: int
    Nq: int
    K: int
    P: int
    dtype: str
    offset_scale: float = 1.0
    # "pixels": one query per pixel, reference at its centre (Nq = H*W, row-major);
    # ("uniform", margin): reference points uniform over [-margin, W-1+margin] x [-margin, H-1+margin]
    ref: object = "pixels"
    value: tuple = ("normal", 0.0, 1.0)
    offset: tuple = ("normal", 0.0, 2.0)
    logit: tuple = ("normal", 0.0, 1.0)
    grad_out: tuple = ("normal", 0.0, 1.0)
    seed: int = 0

    @property
    def C(self) -> int:
        return self.G * self.Cg

    def geometry(self) -> dict:
        return dict(N=self.N, H=self.H, W=self.W, G=self.G, Cg=self.Cg, Nq=self.Nq, K=self.K, P=self.P,
                    offset_scale=self.offset_scale)

    def describe(self) -> str:
        ref = "pixel-centre queries" if self.ref == "pixels" else f"{self.Nq} queries at random reference points"
        return (f"N{self.N} H{self.H} W{self.W} C{self.C} G{self.G} (C'={self.Cg}) Nq{self.Nq} K{self.K} "
                f"P{self.P} offset_scale {self.offset_scale} {self.dtype}, {ref}")


ATTN_WORKLOADS: dict[str, AttnWorkload] = {
    w.name: w
    for w in [
        AttnWorkload("attn_tiny_f32", N=1, H=8, W=8, G=2, Cg=8, Nq=32, K=4, P=24, dtype="f32",
                     ref=("uniform", 1.0), offset=("uniform", -2.0, 2.0)),
        # encoder-style self-attention on one 64x64 map: every pixel queries K=4 points per head
        AttnWorkload("attn_enc_f16", N=8, H=64, W=64, G=8, Cg=32, Nq=64 * 64, K=4, P=96, dtype="f16"),
        # decoder-style: 300 object queries per image at random reference points
        AttnWorkload("attn_dec_bf16", N=8, H=64, W=64, G=8, Cg=32, Nq=300, K=4, P=96, dtype="bf16",
                     ref=("uniform", 0.0), offset=("normal", 0.0, 4.0)),
    ]
}
ATTN_WORKLOAD_ORDER = ["attn_tiny_f32", "attn_enc_f16", "attn_dec_bf16"]


def attn_custom(name: str = "attn_custom", **kw) -> AttnWorkload:
    return AttnWorkload(name=name, **kw)


def make_attn_inputs(w: AttnWorkload, *, seed: int | None = None, tail_fill: float = math.nan,
                     with_grad: bool = True) -> dict:
    """value, ref_points (float32), offset_logits and (optionally) grad_out, in storage form."""
    seed = w.seed if seed is None else seed
    value = to_storage(draw(w.value, seed, STREAM_VALUE, w.N * w.H * w.W * w.C), w.dtype).reshape(
        w.N, w.H, w.W, w.C)
    if w.ref == "pixels":
        if w.Nq != w.H * w.W:
            raise ValueError("pixel-centre queries need Nq = H*W")
        ys, xs = np.divmod(np.arange(w.Nq), w.W)
        ref = np.broadcast_to(np.stack([xs, ys], axis=-1).astype(np.float32), (w.N, w.Nq, 2)).copy()
    else:
        kind, margin = w.ref
        u = uniform01(seed, STREAM_REF, w.N * w.Nq * 2).reshape(w.N, w.Nq, 2)
        span = np.array([w.W - 1 + 2 * margin, w.H - 1 + 2 * margin])
        ref = (-margin + u * span).astype(np.float32)
    ns = w.N * w.Nq * w.G * w.K
    offs = to_storage(draw(w.offset, seed, STREAM_OFFSET, 2 * ns), w.dtype).reshape(w.N, w.Nq, w.G, w.K, 2)
    logits = to_storage(draw(w.logit, seed, STREAM_MASK, ns), w.dtype).reshape(w.N, w.Nq, w.G, w.K)
    out = {"value": value, "ref_points": ref,
           "offset_logits": assemble_offset_mask(offs, logits, w.P, w.dtype, tail_fill)}
    if with_grad:
        out["grad_out"] = to_storage(draw(w.grad_out, seed, STREAM_GRAD, w.N * w.Nq * w.C), w.dtype).reshape(
            w.N, w.Nq, w.C)
    return out
