"""Pins of the oracle's number formats (CPU only).

The E4M3 and bf16 routines are checked against torch's own casts (library
routines written independently of the oracle) and against the code points of
the OCP FP8 specification (tests/golden/e4m3_points.txt).
"""
import os

import numpy as np
import pytest
import torch

from oracle import numerics as nm

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _torch_e4m3_decode(codes):
    t = torch.tensor(codes, dtype=torch.uint8).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def test_e4m3_decode_matches_torch_on_all_256_codes():
    codes = np.arange(256, dtype=np.uint8)
    ours = nm.e4m3_to_f64(codes)
    ref = _torch_e4m3_decode(codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    assert np.array_equal(np.signbit(ours[~nan]), np.signbit(ref[~nan]))
    assert set(np.flatnonzero(nan)) == {0x7F, 0xFF}


def test_e4m3_code_points_from_spec():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "e4m3_points.txt"))
            if l.strip() and not l.startswith("#")]
    for code_s, val_s in rows:
        code = int(code_s, 16)
        val = float(val_s)
        got = nm.e4m3_to_f64(np.uint8(code))
        assert got == val and np.signbit(got) == np.signbit(val), (code_s, got, val)
        assert nm.e4m3_from_f32(np.float32(val)) == code


def test_e4m3_extremes():
    finite = nm.E4M3_TABLE[np.isfinite(nm.E4M3_TABLE)]
    assert finite.max() == 448.0 and finite.min() == -448.0
    pos = finite[finite > 0]
    assert pos.min() == 2.0 ** -9          # subnormal step
    sub = pos[pos < 2.0 ** -6]
    assert np.allclose(np.diff(np.sort(sub)), 2.0 ** -9)


def _torch_e4m3_encode(x):
    return torch.tensor(x, dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(1)
    vals = [rng.standard_normal(20000) * s for s in (1e-3, 1e-2, 0.1, 1, 10, 100)]
    pos = nm.E4M3_TABLE[:0x7F]
    mids = (pos[1:] + pos[:-1]) / 2                    # exact ties (fp32-representable)
    f32 = np.float32
    ties = np.concatenate([mids, -mids])
    near = np.concatenate([np.nextafter(mids.astype(f32), f32(0)),
                           np.nextafter(mids.astype(f32), f32(1000))])
    x = np.concatenate(vals + [ties, near, pos, -pos, [0.0, -0.0, 447.9, 448.0, -448.0, 1e-30, -1e-30]])
    x = x.astype(np.float32)
    x = x[np.abs(x) <= 448]
    assert np.array_equal(nm.e4m3_from_f32(x), _torch_e4m3_encode(x))


def test_e4m3_ties_go_to_even():
    # 1.0 (0x38) and 1.125 (0x39): midpoint 1.0625 -> even code 0x38
    assert nm.e4m3_from_f32(np.float32(1.0625)) == 0x38
    # 1.125 (0x39) and 1.25 (0x3A): midpoint 1.1875 -> 0x3A
    assert nm.e4m3_from_f32(np.float32(1.1875)) == 0x3A
    # half of the smallest subnormal rounds to zero (even), just above rounds up
    assert nm.e4m3_from_f32(np.float32(2.0 ** -10)) == 0x00
    assert nm.e4m3_from_f32(np.nextafter(np.float32(2.0 ** -10), np.float32(1))) == 0x01


def test_e4m3_saturates_and_never_emits_nan():
    x = np.array([448.0, 449.0, 463.9, 464.0, 480.0, 1e6, 3e38, -500.0, -3e38], np.float32)
    c = nm.e4m3_from_f32(x)
    assert list(c) == [0x7E] * 7 + [0xFE] * 2
    rng = np.random.default_rng(2)
    y = (rng.standard_normal(100000) * 1000).astype(np.float32)
    codes = nm.e4m3_from_f32(y)
    assert not np.any((codes == 0x7F) | (codes == 0xFF))


def test_e4m3_round_trip_all_finite_codes():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    vals = nm.e4m3_to_f64(codes).astype(np.float32)
    assert np.array_equal(nm.e4m3_from_f32(vals), codes)


def test_bf16_decode_matches_torch_on_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = nm.bf16_to_f64(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


def test_quantise_uses_fp32_quotient_and_counts_saturation():
    x = torch.tensor([1.0, -2.5, 300.0, 0.0], dtype=torch.bfloat16)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    codes, sat = nm.quantise_e4m3(bits, np.float32(0.5))
    # quotients 2, -5, 600 (clipped), 0
    assert list(codes) == [0x40, 0xCA, 0x7E, 0x00]
    assert sat == 1


def test_calibration_scale():
    assert nm.calibration_scale(448.0) == np.float32(1.0)
    assert nm.calibration_scale(0.0) == np.float32(np.float32(2.0 ** -126) / np.float32(448))
    s = nm.calibration_scale(3.0)
    assert s == np.float32(np.float32(3.0) / np.float32(448.0))
