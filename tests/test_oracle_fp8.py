"""Pins of the oracle's FP8 E4M3 codec and per-row quantiser.

Independent references: torch's float8_e4m3fn conversion (a library routine) and
values fixed by the OCP E4M3 format definition itself.
"""

import numpy as np
import pytest
import torch

from oracle import E4M3_MAX, e4m3_decode, e4m3_encode, e4m3_value_table, quantize_rows


def _torch_decode_all():
    return torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_decode_table_matches_torch_for_all_256_codes():
    ours = e4m3_value_table()
    ref = _torch_decode_all()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok], ref[ok])
    assert np.isnan(ours).sum() == 2          # S.1111.111 only


@pytest.mark.parametrize("code,value", [
    (0x00, 0.0), (0x80, -0.0), (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9), (0x08, 2.0 ** -6),
    (0x38, 1.0), (0x39, 1.125), (0x7E, 448.0), (0xFE, -448.0), (0x77, 240.0),
])
def test_format_definition_landmarks(code, value):
    v = e4m3_decode(np.array([code], dtype=np.uint8))[0]
    assert v == value and np.signbit(v) == np.signbit(value)


def test_encode_decode_roundtrip_all_finite_codes():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    assert np.array_equal(e4m3_encode(e4m3_decode(codes)), codes)


def test_encode_matches_torch_on_sweep_and_midpoints():
    rng = np.random.default_rng(7)
    x = np.concatenate([
        rng.standard_normal(100000).astype(np.float32) * np.float32(50.0),
        rng.uniform(-2.0 ** -5, 2.0 ** -5, 20000).astype(np.float32),      # subnormal range
    ])
    # every midpoint between adjacent positive finite values (ties -> even code)
    vals = np.sort(np.unique(e4m3_value_table()[:0x7F]))
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9))])
    x = x[np.abs(x) < 464].astype(np.float32)
    ours = e4m3_encode(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_satfinite_and_signed_zero():
    x = np.array([448.0, 449.0, 463.9, 464.0, 500.0, 1e30, -1e30, -448.5, -0.0, -1e-12, 1e-12],
                 dtype=np.float64)
    got = e4m3_encode(x)
    assert list(got) == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE, 0x80, 0x80, 0x00]


def test_quantize_rows_scale_and_error_bound():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((64, 512)).astype(np.float32)
    x[5] = 0.0
    codes, scale = quantize_rows(x)
    assert scale.dtype == np.float32
    absmax = np.abs(x).max(axis=1)
    expect = np.where(absmax > 0, absmax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    assert np.array_equal(scale, expect)
    assert np.all(codes[5] == 0)
    # the absmax element lands on the largest code, +-448
    for r in range(64):
        if r == 5:
            continue
        j = np.argmax(np.abs(x[r]))
        assert codes[r, j] & 0x7F == 0x7E
    deq = e4m3_decode(codes) * scale[:, None].astype(np.float64)
    err = np.abs(deq - x.astype(np.float64))
    # half an ulp of a 3-bit mantissa (2^-4 relative) or half a subnormal step
    bound = np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10 * scale[:, None]) * (1 + 1e-6)
    assert np.all(err <= bound)
    assert E4M3_MAX == 448.0


def test_bf16_bits_decode_matches_torch():
    from oracle import bf16_bits_to_f64
    x = torch.randn(50000, dtype=torch.float32) * 100
    b = x.to(torch.bfloat16)
    bits = b.view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bf16_bits_to_f64(bits), b.to(torch.float64).numpy())
