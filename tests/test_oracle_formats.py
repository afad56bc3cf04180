"""Pins for the oracle's codecs: library routines (ml_dtypes, torch), the published format
tables, and brute force over every code and every rounding midpoint."""
import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import formats as F

ALL8 = np.arange(256, dtype=np.uint8)


def test_e4m3_decode_matches_ml_dtypes_all_codes():
    ours = F.e4m3_decode(ALL8)
    lib = ALL8.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    assert np.array_equal(np.isnan(ours), np.isnan(lib))
    ok = ~np.isnan(lib)
    assert np.array_equal(ours[ok], lib[ok])
    # the two NaN codes of E4M3FN and the published extremes
    assert np.isnan(ours[0x7F]) and np.isnan(ours[0xFF])
    assert ours[0x7E] == 448.0 and ours[0xFE] == -448.0
    assert ours[0x01] == 2.0 ** -9 and ours[0x08] == 2.0 ** -6


def test_e4m3_decode_matches_torch():
    t = torch.from_numpy(ALL8.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = F.e4m3_decode(ALL8)
    ok = ~np.isnan(t)
    assert np.array_equal(ours[ok], t[ok])


def test_e4m3_encode_roundtrip_every_code():
    vals = F.e4m3_decode(ALL8)
    ok = ~np.isnan(vals)
    assert np.array_equal(F.e4m3_encode(vals[ok].astype(np.float32)), ALL8[ok])


def _midpoints_and_neighbours():
    pos = np.sort(F.e4m3_decode(np.arange(0x7F, dtype=np.uint8)))
    mids = (pos[:-1] + pos[1:]) / 2
    pts = [pos, mids]
    m32 = mids.astype(np.float32)
    pts.append(np.nextafter(m32, np.float32(0)))
    pts.append(np.nextafter(m32, np.float32(np.inf)))
    x = np.concatenate([np.asarray(p, dtype=np.float32) for p in pts])
    x = np.concatenate([x, -x, np.float32([449, 463.99, 464, 464.01, 480, 1e6, 3e38])])
    return x.astype(np.float32)


def test_e4m3_encode_bruteforce_midpoints():
    x = _midpoints_and_neighbours()
    assert np.array_equal(F.e4m3_encode(x), F.e4m3_encode_bruteforce(x))


def test_e4m3_encode_random_bruteforce():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(3000) * np.exp2(rng.integers(-14, 10, 3000))).astype(np.float32)
    assert np.array_equal(F.e4m3_encode(x), F.e4m3_encode_bruteforce(x))


def test_e4m3_encode_matches_ml_dtypes_in_range():
    rng = np.random.default_rng(2)
    x = (rng.uniform(-447.9, 447.9, 200000) * np.exp2(rng.integers(-20, 1, 200000)))
    x = x.astype(np.float32)
    lib = x.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    ours = F.e4m3_encode(x)
    # ml_dtypes may drop the sign of values that round to zero; compare magnitudes there
    zero = (lib & 0x7F) == 0
    assert np.array_equal(ours[~zero], lib[~zero])
    assert np.all((ours[zero] & 0x7F) == 0)


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(3)
    x = torch.from_numpy((rng.standard_normal(100000) * 50).astype(np.float32))
    x = x.clamp(-447, 447)
    lib = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = F.e4m3_encode(x.numpy())
    nz = (lib & 0x7F) != 0
    assert np.array_equal(ours[nz], lib[nz])


def test_e4m3_saturation_and_signed_zero():
    x = np.float32([448, 449, 464, 480, 1e30, -448, -500, 0.0, -0.0, -1e-9, 1e-9])
    c = F.e4m3_encode(x)
    assert list(c[:7]) == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE]
    assert list(c[7:]) == [0x00, 0x80, 0x80, 0x00]


def test_e8m0_decode_matches_ml_dtypes():
    ours = F.e8m0_decode(ALL8)
    lib = ALL8.view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    assert np.isnan(ours[255]) and np.isnan(lib[255])
    assert np.array_equal(ours[:255], lib[:255])


def test_e2m1_decode_matches_ml_dtypes():
    codes = np.arange(16, dtype=np.uint8)
    lib = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    assert np.array_equal(F.e2m1_decode(codes), lib)


def test_e2m1_rne_ties_textbook():
    x = np.float32([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.5, 100.0, -0.25, -5.0])
    vals = F.e2m1_decode(F.e2m1_encode_rne(x))
    assert list(vals) == [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, 6.0, 6.0, -0.0, -4.0]
    assert np.signbit(vals[9])


def test_e2m1_rne_bruteforce_dense():
    grid = F.E2M1_VALUES
    mids = (grid[:-1] + grid[1:]) / 2
    x = np.concatenate([grid, mids, np.linspace(0, 7, 2001)]).astype(np.float32)
    x = np.concatenate([x, np.nextafter(x, np.float32(0)), np.nextafter(x, np.float32(9)), -x])
    assert np.array_equal(F.e2m1_encode_rne(x), F.e2m1_encode_bruteforce(x))


def test_e2m1_rne_matches_ml_dtypes_in_range():
    rng = np.random.default_rng(4)
    x = rng.uniform(-6, 6, 100000).astype(np.float32)
    lib = x.astype(ml_dtypes.float4_e2m1fn).astype(np.float64)
    ours = F.e2m1_decode(F.e2m1_encode_rne(x))
    assert np.array_equal(np.abs(ours), np.abs(lib))


def test_pack_unpack_e2m1():
    rng = np.random.default_rng(5)
    c = rng.integers(0, 16, (7, 32)).astype(np.uint8)
    p = F.pack_e2m1(c)
    assert p.shape == (7, 16)
    assert np.array_equal(p[:, 0] & 0xF, c[:, 0]) and np.array_equal(p[:, 0] >> 4, c[:, 1])
    assert np.array_equal(F.unpack_e2m1(p), c)


def test_bf16_conversions_match_torch():
    rng = np.random.default_rng(6)
    x = (rng.standard_normal(50000) * np.exp2(rng.integers(-130, 120, 50000))).astype(np.float32)
    t = torch.from_numpy(x).to(torch.bfloat16)
    bits = t.view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(F.f32_to_bf16_bits(x), bits)
    assert np.array_equal(F.bf16_bits_to_f32(bits), t.to(torch.float32).numpy())


# ----------------------------------------------------------------------------- E5M2
def test_e5m2_decode_matches_ml_dtypes_and_torch_all_codes():
    ours = F.e5m2_decode(ALL8)
    lib = ALL8.view(ml_dtypes.float8_e5m2).astype(np.float64)
    tor = torch.from_numpy(ALL8.copy()).view(torch.float8_e5m2).to(torch.float64).numpy()
    for ref in (lib, tor):
        assert np.array_equal(np.isnan(ours), np.isnan(ref))
        ok = ~np.isnan(ref)
        assert np.array_equal(ours[ok], ref[ok])
    # published extremes: largest finite 57344, infinity at 0x7C, smallest subnormal 2^-16
    assert ours[0x7B] == 57344.0 and ours[0x7C] == np.inf and ours[0xFC] == -np.inf
    assert ours[0x01] == 2.0 ** -16 and ours[0x04] == 2.0 ** -14


def _e5m2_midpoints_and_neighbours():
    pos = np.sort(F.e5m2_decode(np.arange(0x7C, dtype=np.uint8)))
    mids = (pos[:-1] + pos[1:]) / 2
    m32 = mids.astype(np.float32)
    x = np.concatenate([pos.astype(np.float32), m32, np.nextafter(m32, np.float32(0)),
                        np.nextafter(m32, np.float32(np.inf))])
    x = np.concatenate([x, -x, np.float32([57345, 61439.9, 61440, 61440.1, 65536, 1e9, 3e38])])
    return x.astype(np.float32)


def test_e5m2_encode_roundtrip_every_finite_code():
    vals = F.e5m2_decode(ALL8)
    ok = np.isfinite(vals)
    assert np.array_equal(F.e5m2_encode(vals[ok].astype(np.float32)), ALL8[ok])


def test_e5m2_encode_bruteforce_midpoints_and_saturation():
    x = _e5m2_midpoints_and_neighbours()
    got = F.e5m2_encode(x)
    assert np.array_equal(got, F.e5m2_encode_bruteforce(x))
    assert np.all((got & 0x7F) <= 0x7B)            # satfinite: never infinity or NaN


def test_e5m2_encode_matches_torch_in_range():
    rng = np.random.default_rng(7)
    x = (rng.standard_normal(20000) * np.exp2(rng.integers(-20, 14, 20000))).astype(np.float32)
    x = x[np.abs(x) < 57344]
    t = torch.from_numpy(x).to(torch.float8_e5m2).view(torch.uint8).numpy()
    assert np.array_equal(F.e5m2_encode(x), t)
