"""Pins for the oracle's element codecs against library decoders and the formats' own rules."""

import numpy as np
import pytest
import torch

from oracle import codecs


def _same(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    both_nan = np.isnan(a) & np.isnan(b)
    eq = (a == b) & (np.signbit(a) == np.signbit(b))
    return bool(np.all(both_nan | eq))


def test_f16_every_code_matches_numpy():
    codes = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ref = codes.view(np.float16).astype(np.float64)
    assert _same(codecs.decode_f16(codes), ref)


def test_bf16_every_code_matches_torch():
    codes = np.arange(1 << 16, dtype=np.int64).astype(np.uint16)
    ref = torch.from_numpy(codes.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert _same(codecs.decode_bf16(codes), ref)


def test_e4m3_every_code_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert _same(codecs.decode_e4m3(codes), ref)


def test_e4m3_format_landmarks():
    d = codecs.decode_e4m3(np.array([0x00, 0x01, 0x07, 0x08, 0x38, 0x7E, 0x7F, 0x80, 0xFE, 0xFF], dtype=np.uint8))
    assert d[0] == 0.0 and d[1] == 2.0 ** -9 and d[2] == 7 * 2.0 ** -9
    assert d[3] == 2.0 ** -6 and d[4] == 1.0 and d[5] == 448.0
    assert np.isnan(d[6]) and np.signbit(d[7]) and d[8] == -448.0 and np.isnan(d[9])


def test_e4m3_encode_round_trips_every_finite_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = codecs.decode_e4m3(codes)
    assert np.array_equal(codecs.encode_e4m3(vals), codes)


def test_e4m3_encode_ties_go_to_even():
    # midpoint of every adjacent pair of positive finite codes
    pos = np.arange(0, 0x7E, dtype=np.uint8)
    lo = codecs.decode_e4m3(pos)
    hi = codecs.decode_e4m3(pos + 1)
    mid = (lo + hi) / 2.0
    got = codecs.encode_e4m3(mid).astype(np.int64)
    want = np.where(pos % 2 == 0, pos, pos + 1)
    assert np.array_equal(got, want)
    assert np.array_equal(codecs.encode_e4m3(-mid).astype(np.int64), want | 0x80)
    # just off the midpoint rounds to the nearer code
    assert np.array_equal(codecs.encode_e4m3(np.nextafter(mid, 0)).astype(np.int64), pos)
    assert np.array_equal(codecs.encode_e4m3(np.nextafter(mid, np.inf)).astype(np.int64), pos + 1)


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(7)
    x = np.concatenate([rng.normal(0, 1, 20000) * s for s in (1e-3, 0.1, 1, 30, 200)]).astype(np.float32)
    x = x[np.abs(x) <= 448]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codecs.encode_e4m3(x.astype(np.float64)), ref)


def test_e4m3_encode_saturates():
    x = np.array([448.0, 449.0, 463.99, 464.0, 470.0, 480.0, 1e6, np.inf, 3e38], dtype=np.float64)
    assert np.all(codecs.encode_e4m3(x) == 0x7E)
    assert np.all(codecs.encode_e4m3(-x) == 0xFE)
    assert np.isnan(codecs.decode_e4m3(codecs.encode_e4m3(np.array([np.nan])))[0])
    assert codecs.encode_e4m3(np.array([-0.0]))[0] == 0x80
    assert codecs.encode_e4m3(np.array([2.0 ** -11]))[0] == 0x00      # below half the smallest subnormal
    assert codecs.encode_e4m3(np.array([3 * 2.0 ** -11]))[0] == 0x01   # above it


def test_f32_div_is_correctly_rounded():
    rng = np.random.default_rng(3)
    x = rng.normal(0, 3, 10000).astype(np.float32)
    s = np.float32(0.013671875 * 1.37)
    want = (x.astype(np.float64) / np.float64(s)).astype(np.float32)  # f64 quotient of f32s rounds once correctly
    assert np.array_equal(codecs.f32_div(x, s), want)
