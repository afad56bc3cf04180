"""Pins of the CPU oracle against CUDA's own outputs, on the GPU:
  * the oracle's Philox4x32-10 equals cuRAND's curand_Philox4x32_10 on 2^20 random
    (counter, key) pairs;
  * the oracle's E4M3 encoder equals the hardware cvt.rn.satfinite.e4m3x2.f32 on every BF16
    value in range, on all rounding midpoints (and their FP32 neighbours) and on 4M random
    FP32 bit patterns;
  * the oracle's E2M1 round-to-nearest-even encoder equals cvt.rn.satfinite.e2m1x2.f32."""
import ctypes
import os

import numpy as np
import pytest
import torch

from oracle import formats as F
from oracle import philox

PINS = os.path.join(os.path.dirname(os.path.abspath(__file__)), "cuda", "libpins.so")


@pytest.fixture(scope="module")
def pins():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    if not os.path.exists(PINS):
        pytest.fail("tests/cuda/libpins.so missing: run __graft_entry__.build()")
    L = ctypes.CDLL(PINS)
    for f in ("pins_curand_philox", "pins_cvt_e4m3", "pins_cvt_e5m2", "pins_cvt_e2m1"):
        getattr(L, f).restype = ctypes.c_int
    return L


def _s():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


@pytest.mark.gpu
def test_philox_matches_curand(pins):
    n = 1 << 20
    rng = np.random.default_rng(2024)
    ctr = rng.integers(0, 2 ** 32, (n, 4), dtype=np.uint64).astype(np.uint32)
    ctr[:16] = 0
    ctr[16:32] = 0xFFFFFFFF
    key = rng.integers(0, 2 ** 32, (n, 2), dtype=np.uint64).astype(np.uint32)
    key[:8] = 0
    dc = torch.from_numpy(ctr.view(np.int32)).cuda()
    dk = torch.from_numpy(key.view(np.int32)).cuda()
    out = torch.empty((n, 4), dtype=torch.int32, device="cuda")
    assert pins.pins_curand_philox(ctypes.c_void_p(dc.data_ptr()), ctypes.c_void_p(dk.data_ptr()),
                                   ctypes.c_void_p(out.data_ptr()), n, _s()) == 0
    got = out.cpu().numpy().view(np.uint32)
    want = philox.philox4x32_10(ctr, key)
    assert np.array_equal(got, want)


def _cvt(pins, fn, x):
    dx = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()
    out = torch.empty(dx.numel(), dtype=torch.uint8, device="cuda")
    assert getattr(pins, fn)(ctypes.c_void_p(dx.data_ptr()), ctypes.c_void_p(out.data_ptr()), dx.numel(), _s()) == 0
    return out.cpu().numpy()


def _e4m3_sweep_inputs():
    bf = np.arange(1 << 16, dtype=np.uint16)
    x_bf = F.bf16_bits_to_f32(bf)
    x_bf = x_bf[np.isfinite(x_bf) & (np.abs(x_bf) <= 600)]
    pos = np.sort(F.e4m3_decode(np.arange(0x7F, dtype=np.uint8))).astype(np.float32)
    mids = ((pos[:-1].astype(np.float64) + pos[1:]) / 2).astype(np.float32)
    around = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e9))])
    rng = np.random.default_rng(7)
    bits = rng.integers(0, 1 << 32, 1 << 22, dtype=np.uint64).astype(np.uint32)
    x_rand = bits.view(np.float32)
    x_rand = x_rand[np.isfinite(x_rand) & (np.abs(x_rand) <= 1000)]
    x = np.concatenate([x_bf, around, -around, x_rand, np.float32([0.0, -0.0, 448, 464, 480, 1e30, -1e30])])
    return x.astype(np.float32)


@pytest.mark.gpu
def test_e4m3_cvt_matches_oracle(pins):
    x = _e4m3_sweep_inputs()
    got = _cvt(pins, "pins_cvt_e4m3", x)
    want = F.e4m3_encode(x)
    bad = np.flatnonzero(got != want)
    assert bad.size == 0, f"{bad.size} mismatches, e.g. x={x[bad[:5]]} hw={got[bad[:5]]} oracle={want[bad[:5]]}"


@pytest.mark.gpu
def test_e2m1_cvt_matches_oracle(pins):
    grid = F.E2M1_VALUES
    mids = (grid[:-1] + grid[1:]) / 2
    base = np.concatenate([grid, mids, np.linspace(0, 8, 100001)]).astype(np.float32)
    x = np.concatenate([base, np.nextafter(base, np.float32(0)), np.nextafter(base, np.float32(9))])
    x = np.concatenate([x, -x]).astype(np.float32)
    got = _cvt(pins, "pins_cvt_e2m1", x)
    want = F.e2m1_encode_rne(x)
    # compare magnitudes and signs separately so a -0 convention difference is visible
    bad = np.flatnonzero(got != want)
    assert bad.size == 0, f"{bad.size} mismatches, e.g. x={x[bad[:5]]} hw={got[bad[:5]]} oracle={want[bad[:5]]}"


@pytest.mark.gpu
def test_e5m2_cvt_matches_oracle(pins):
    """The oracle's E5M2 encoder equals cvt.rn.satfinite.e5m2x2.f32 on every BF16 value in
    range, every rounding midpoint and its neighbours, random FP32 bit patterns and the
    saturation region."""
    bf = np.arange(1 << 16, dtype=np.uint16)
    x_bf = F.bf16_bits_to_f32(bf)
    x_bf = x_bf[np.isfinite(x_bf)]
    pos = np.sort(F.e5m2_decode(np.arange(0x7C, dtype=np.uint8))).astype(np.float32)
    mids = ((pos[:-1].astype(np.float64) + pos[1:]) / 2).astype(np.float32)
    around = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(1e30))])
    rng = np.random.default_rng(8)
    bits = rng.integers(0, 1 << 32, 1 << 22, dtype=np.uint64).astype(np.uint32)
    x_rand = bits.view(np.float32)
    x_rand = x_rand[np.isfinite(x_rand)]
    x = np.concatenate([x_bf, around, -around, x_rand, np.float32([0.0, -0.0, 57344, 61440, 1e30, -1e30])])
    got = _cvt(pins, "pins_cvt_e5m2", x)
    want = F.e5m2_encode(x)
    bad = np.flatnonzero(got != want)
    assert bad.size == 0, f"{bad.size} mismatches, e.g. x={x[bad[:5]]} hw={got[bad[:5]]} oracle={want[bad[:5]]}"
