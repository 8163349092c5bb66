"""Seeded input generator: determinism, slicing, rounding (CPU only)."""
import numpy as np
import torch

import dcn4_inputs as gen


def test_counter_based_slices():
    a = gen.uniform01(7, 3, 1000)
    b = gen.uniform01(7, 3, 400, start=600)
    np.testing.assert_array_equal(a[600:], b)
    assert np.all((a > 0) & (a <= 1))
    assert not np.array_equal(a, gen.uniform01(8, 3, 1000))
    assert not np.array_equal(a, gen.uniform01(7, 4, 1000))


def test_distribution_moments():
    z = gen.normal(0, 1, 200_000, 0.5, 2.0)
    assert abs(z.mean() - 0.5) < 0.03 and abs(z.std() - 2.0) < 0.03
    u = gen.uniform(0, 2, 200_000, -8.0, 8.0)
    assert u.min() >= -8.0 and u.max() <= 8.0 and abs(u.mean()) < 0.05


def test_f16_rounding_matches_torch_on_fp32_values():
    # torch rounds float64 -> float16 through float32; on float32 inputs both are one rounding
    x = gen.normal(1, 1, 50_000, 0.0, 3.0).astype(np.float32).astype(np.float64)
    want = torch.from_numpy(x).to(torch.float16).numpy()
    np.testing.assert_array_equal(gen.to_storage(x, "f16").view(np.uint16), want.view(np.uint16))


def test_f16_direct_rounding_is_nearest():
    x = gen.normal(4, 1, 20_000, 0.0, 3.0)
    bits = gen.to_storage(x, "f16").view(np.uint16)
    r = bits.view(np.float16).astype(np.float64)
    up = (bits + np.uint16(1)).view(np.float16).astype(np.float64)
    dn = (bits - np.uint16(1)).view(np.float16).astype(np.float64)
    err = np.abs(r - x)
    assert np.all(err <= np.abs(up - x)) and np.all(err <= np.abs(dn - x))


def test_bf16_rounding_matches_torch_on_fp32_values():
    x = gen.normal(2, 1, 50_000, 0.0, 3.0).astype(np.float32).astype(np.float64)
    want = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(gen.to_storage(x, "bf16"), want)
    back = gen.bf16_bits_to_f64(gen.to_storage(x, "bf16"))
    assert np.max(np.abs(back - x) / np.maximum(np.abs(x), 1e-30)) <= 2.0 ** -8


def test_bf16_direct_rounding_is_nearest():
    x = gen.normal(3, 1, 20_000, 0.0, 1.0)
    bits = gen.f64_to_bf16_bits(x)
    r = gen.bf16_bits_to_f64(bits)
    up = gen.bf16_bits_to_f64(bits + np.uint16(1))
    dn = gen.bf16_bits_to_f64(bits - np.uint16(1))
    err = np.abs(r - x)
    assert np.all(err <= np.abs(up - x)) and np.all(err <= np.abs(dn - x))


def test_workload_layout():
    w = gen.WORKLOADS["tiny_f32"]
    inp = gen.make_inputs(w)
    assert inp["value"].shape == (1, 8, 8, 16) and inp["value"].dtype == np.float32
    om = inp["offset_mask"]
    assert om.shape == (1, 8, 8, 56)
    assert np.all(np.isnan(om[..., 54:])) and np.all(np.isfinite(om[..., :54]))
    body = om[..., :54].reshape(1, 8, 8, 2, 27)
    offs = body[..., :18]
    assert offs.min() >= -2.0 and offs.max() <= 2.0
    again = gen.make_inputs(w)
    for k in inp:
        np.testing.assert_array_equal(inp[k], again[k])
    zero_tail = gen.make_inputs(w, tail_fill=0.0)["offset_mask"]
    assert np.all(zero_tail[..., 54:] == 0.0)


def test_workload_table_consistent():
    for w in gen.WORKLOADS.values():
        assert w.K == w.kh * w.kw - w.remove_center
        assert w.P % 8 == 0 and w.P >= w.G * 3 * w.K and w.P - w.G * 3 * w.K < 8
        assert w.Ho == (w.H + 2 * w.ph - (w.dh * (w.kh - 1) + 1)) // w.sh + 1
        assert w.Wo == (w.W + 2 * w.pw - (w.dw * (w.kw - 1) + 1)) // w.sw + 1


def test_linear_inputs_are_seeded_and_shaped():
    """make_linear_inputs: same seed, same bits; shapes [N,Ho,Wo,Cx], [P,Cx], [P]; the
    produced offsets and masks have about the workload's own spread."""
    import numpy as np
    w = gen.custom(**{**gen.WORKLOADS["stage1_f16"].__dict__, "N": 2, "name": "lin"})
    a = gen.make_linear_inputs(w, 64)
    b = gen.make_linear_inputs(w, 64)
    assert all(np.array_equal(a[k], b[k]) for k in ("x", "weight", "bias"))
    assert a["x"].shape == (2, 56, 56, 64) and a["weight"].shape == (112, 64) and a["bias"].shape == (112,)
    assert gen.make_linear_inputs(w, 64, bias=False)["bias"] is None
    c = gen.make_linear_inputs(w, 64, seed=1)
    assert not np.array_equal(a["x"], c["x"])
    om = gen.storage_to_f64(a["x"], "f16").reshape(-1, 64) @ gen.storage_to_f64(a["weight"], "f16").T
    offs = np.concatenate([om[:, g * 27:g * 27 + 18] for g in range(4)], axis=1)
    masks = np.concatenate([om[:, g * 27 + 18:g * 27 + 27] for g in range(4)], axis=1)
    assert abs(offs.std() - 1.5) < 0.1 and abs(masks.std() - 0.5) < 0.05
