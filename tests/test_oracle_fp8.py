"""Pins of the FP8 (e4m3) oracle: the format's defining values, rounding ties
to even, saturation, agreement with torch's float8_e4m3fn cast on in-range
values, and per-tensor scaling."""

import numpy as np
import torch

from oracle import fp8


def test_decode_defining_values():
    vals = fp8.e4m3_decode(np.array([0x00, 0x01, 0x07, 0x08, 0x38, 0x3C, 0x7E, 0x80, 0xBE, 0xFE]))
    np.testing.assert_array_equal(vals, [0.0, 2.0 ** -9, 7 * 2.0 ** -9, 2.0 ** -6, 1.0, 1.5, 448.0, -0.0, -1.75,
                                         -448.0])
    assert np.isnan(fp8.e4m3_decode(np.array([0x7F, 0xFF]))).all()


def test_every_finite_code_round_trips():
    codes = np.array([c for c in range(256) if c & 0x7F != 0x7F], dtype=np.uint8)
    np.testing.assert_array_equal(fp8.e4m3_encode(fp8.e4m3_decode(codes)), codes)


def test_ties_go_to_the_even_mantissa_and_large_values_saturate():
    # 1.0625 lies halfway between 1.0 (mantissa 0) and 1.125 (mantissa 1): 1.0
    # 1.1875 lies halfway between 1.125 (mantissa 1) and 1.25 (mantissa 2): 1.25
    # 2^-10 lies halfway between 0 and 2^-9 (code 1): 0
    got = fp8.e4m3_encode(np.array([1.0625, 1.1875, 2.0 ** -10, 2.0 ** -10 * 1.001, 460.0, 1e6, -1e6]))
    np.testing.assert_array_equal(got, [0x38, 0x3A, 0x00, 0x01, 0x7E, 0x7E, 0xFE])


def test_encode_matches_torch_cast_in_range():
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.standard_normal(200000) * 60, rng.standard_normal(20000) * 1e-3,
                        rng.uniform(-448, 448, 20000)]).astype(np.float32)
    x = x[np.abs(x) <= 448]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(fp8.e4m3_encode(x.astype(np.float64)), ref)


def test_per_tensor_scaling_maps_amax_to_448():
    rng = np.random.default_rng(6)
    x = (rng.standard_normal(4096) * 0.02).astype(np.float32)
    q, s = fp8.quantize(x)
    i = int(np.argmax(np.abs(x)))
    assert q[i] & 0x7F == 0x7E
    assert s == np.float32(np.max(np.abs(x))) / np.float32(448.0)
    err = np.abs(fp8.e4m3_decode(q) * s - x) / np.max(np.abs(x))
    assert err.max() <= 2.0 ** -4 + 1e-6            # half an ulp at the top binade, relative to amax


def test_gemm_closed_form():
    """Identity codes (1.0) with scale 2 times B: C = 2 sb decode(B)."""
    qa = fp8.e4m3_encode(np.eye(8))
    qb = fp8.e4m3_encode(np.arange(-12, 12, dtype=np.float64).reshape(3, 8) / 4)
    np.testing.assert_array_equal(fp8.gemm(qa, 2.0, qb, 0.5), fp8.e4m3_decode(qb).T * 1.0)
