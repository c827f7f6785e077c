"""Pins for the oracle's E4M3 encoder/decoder (CPU only).

The oracle's encoder is pinned against (a) the OCP FP8 specification values
in tests/golden/e4m3_spec_values.json, (b) an exhaustive round trip of every
finite code, (c) a brute-force nearest-value search written here (a different
algorithm: enumerate all finite values, no binade arithmetic), and (d)
PyTorch's independent float8_e4m3fn cast.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_spec_values.json")

FINITE = [c for c in range(256) if (c & 0x7F) != 0x7F]


def all_finite_values():
    codes = np.array(FINITE, np.uint8)
    return codes, oracle.e4m3_decode(codes)


def test_spec_values():
    spec = json.load(open(GOLDEN))
    for code_hex, value in spec["values"].items():
        code = int(code_hex, 16)
        want = float.fromhex(value) if isinstance(value, str) else float(value)
        got = oracle.e4m3_decode(np.array([code], np.uint8))[0]
        assert got == want, code_hex
    for code_hex in spec["nan"]:
        assert np.isnan(oracle.e4m3_decode(np.array([int(code_hex, 16)], np.uint8))[0])


def test_decode_matches_torch():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.e4m3_decode(codes.numpy())
    fin = ~np.isnan(ref)
    assert np.array_equal(np.isnan(got), ~fin)
    assert np.array_equal(got[fin], ref[fin])


def test_roundtrip_all_finite_codes():
    codes, vals = all_finite_values()
    assert len(codes) == 254
    back = oracle.e4m3_encode(vals.astype(np.float32))
    assert np.array_equal(back, codes)


def brute_force_encode(y: float, vals: np.ndarray, codes: np.ndarray) -> int:
    """Nearest finite E4M3 value, ties to the even code; |y| >= 448 -> +-448."""
    if abs(y) >= 448.0:
        return 0x7E | (0x80 if np.signbit(y) else 0)
    same_sign = (np.signbit(vals) == np.signbit(y))
    v, c = vals[same_sign], codes[same_sign]
    d = np.abs(v - float(y))
    best = np.flatnonzero(d == d.min())
    if len(best) > 1:
        even = [b for b in best if (c[b] & 1) == 0]
        assert len(even) == 1
        return int(c[even[0]])
    return int(c[best[0]])


def test_encode_matches_brute_force():
    codes, vals = all_finite_values()
    rng = np.random.default_rng(1)
    y = np.concatenate([
        rng.standard_normal(3000) * 100,
        np.exp(rng.uniform(np.log(1e-4), np.log(460), 3000)) * rng.choice([-1, 1], 3000),
        rng.uniform(-2e-3, 2e-3, 1000),
    ]).astype(np.float32)
    got = oracle.e4m3_encode(y)
    want = np.array([brute_force_encode(float(v), vals, codes) for v in y], np.uint8)
    assert np.array_equal(got, want)


def midpoints():
    """All midpoints between adjacent positive finite values (exact in fp32)."""
    _, vals = all_finite_values()
    pos = np.unique(vals[vals >= 0])
    return pos, (pos[:-1] + pos[1:]) / 2


def test_midpoints_round_to_even():
    codes, vals = all_finite_values()
    pos, mids = midpoints()
    y = np.concatenate([mids, -mids]).astype(np.float32)
    assert np.array_equal(y.astype(np.float64), np.concatenate([mids, -mids]))  # exact
    got = oracle.e4m3_encode(y)
    assert np.all((got & 1) == 0), "ties must go to the even code"
    # and each tie lands on one of its two neighbours
    dec = np.abs(oracle.e4m3_decode(got))
    lo = np.concatenate([pos[:-1], pos[:-1]])
    hi = np.concatenate([pos[1:], pos[1:]])
    assert np.all((dec == lo) | (dec == hi))
    # one fp32 ulp either side of a midpoint rounds to the nearer neighbour
    up = np.nextafter(mids.astype(np.float32), np.float32(np.inf))
    dn = np.nextafter(mids.astype(np.float32), np.float32(0))
    assert np.array_equal(oracle.e4m3_decode(oracle.e4m3_encode(up)), pos[1:])
    assert np.array_equal(oracle.e4m3_decode(oracle.e4m3_encode(dn)), pos[:-1])


def test_matches_torch_cast_random():
    rng = np.random.default_rng(2)
    y = np.concatenate([
        rng.standard_normal(200000) * 50,
        np.exp(rng.uniform(np.log(1e-6), np.log(463), 200000)) * rng.choice([-1, 1], 200000),
    ]).astype(np.float32)
    y = y[np.abs(y) < 464]  # torch maps |y| >= 464 (beyond the tie) to NaN
    ref = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.e4m3_encode(y)
    assert np.array_equal(got, ref)


def test_saturation_and_zero():
    y = np.array([448.0, 449.0, 463.9, 464.0, 500.0, 1e30, -1e30, -449.0], np.float32)
    got = oracle.e4m3_encode(y)
    assert list(got) == [0x7E] * 6 + [0xFE, 0xFE]
    z = oracle.e4m3_encode(np.array([0.0, -0.0, 2.0 ** -11, -(2.0 ** -11)], np.float32))
    assert list(z) == [0x00, 0x80, 0x00, 0x80]
    # 2^-10 is the midpoint between 0 and the smallest subnormal: ties to even (0)
    assert oracle.e4m3_encode(np.array([2.0 ** -10], np.float32))[0] == 0x00


def test_near_boundary_matches_brute_force():
    _, mids = midpoints()
    rng = np.random.default_rng(3)
    base = rng.choice(mids, 4000)
    rel = rng.choice([0.0, 3e-7, -9e-7, 1.2e-6, -2e-6, 1e-4, 0.01], 4000)
    y = (base * (1 + rel)).astype(np.float32)
    y = np.concatenate([y, rng.standard_normal(4000).astype(np.float32) * 30])
    got = oracle.e4m3_near_boundary(y)
    a = np.abs(y.astype(np.float64))
    want = (np.abs(a[:, None] / mids[None, :] - 1.0) <= 1e-6).any(axis=1)
    assert np.array_equal(got.astype(bool), want)
    assert got[: len(base)][rel == 0.0].all()


@pytest.mark.parametrize("amax_code", [0x7E, 0xFE])
def test_quantize_row_amax_lands_on_max_code(amax_code):
    rng = np.random.default_rng(4)
    x = rng.standard_normal((16, 128)).astype(np.float32)
    sign = -1.0 if amax_code & 0x80 else 1.0
    x[:, 5] = sign * (np.abs(x).max(axis=1) + 1.0)
    codes, scales, _ = oracle.quantize_rows(x)
    assert np.all(codes[:, 5] == amax_code)
    amax = np.abs(x).max(axis=1)
    assert np.array_equal(scales, (amax / np.float32(448.0)).astype(np.float32))
