"""Number formats written out from their bit definitions (oracle; test infrastructure only).

The pages fix E4M3 as the one FP8 format for every tensor ("Can you explain the role of
FP8 precision in DeepSeek-V3 training", section "Unified E4M3 format"), 4-bit values for
NVFP4 ("NVIDIA developed a method to train neural networks in 4-bit precision", section
"How it works") and power-of-two block scales for MXFP8 ("Accelerating FP8 training
performance with the NVIDIA NeMo framework").  They give no bit layouts; those come from
the public format definitions:

* E4M3 ("E4M3FN", OCP 8-bit floating point spec): 1 sign, 4 exponent (bias 7), 3 mantissa
  bits; no infinities; exponent 15 with mantissa 7 is NaN; largest finite value
  1.75 * 2^8 = 448; smallest subnormal 2^-9.
* E5M2 (OCP 8-bit floating point spec), the gradient format of the delayed-scaling recipe's
  comparison variant: 1 sign, 5 exponent (bias 15), 2 mantissa bits; exponent 31 holds
  infinity (mantissa 0) and NaN; largest finite value 1.75 * 2^15 = 57344; smallest
  subnormal 2^-16.
* E8M0 (OCP MX spec v1.0): unsigned 8-bit exponent, value 2^(c - 127); code 255 is NaN.
* E2M1 (OCP MX spec v1.0): 1 sign, 2 exponent (bias 1), 1 mantissa bit; values
  {0, 0.5, 1, 1.5, 2, 3, 4, 6}; no NaN or infinity.
* BF16: the upper 16 bits of an IEEE binary32.

Encoders round to nearest, ties to even, and saturate to the largest finite value
(the "satfinite" reading: a magnitude at or above the format maximum after rounding
maps to the maximum).  The sign of zero is kept.
"""
import numpy as np

E4M3_MAX = 448.0
E5M2_MAX = 57344.0
E2M1_MAX = 6.0
FLT_MAX = np.float32(np.finfo(np.float32).max)


# ----------------------------------------------------------------------------- BF16
def bf16_bits_to_f32(bits):
    """BF16 bit patterns (uint16 / int16 array) -> float32, exactly."""
    b = np.asarray(bits).view(np.uint16).astype(np.uint32)
    return (b << np.uint32(16)).view(np.float32)


def f32_to_bf16_bits(x):
    """float32 -> BF16 bit pattern, round to nearest even (finite inputs)."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return r.astype(np.uint16)


# ----------------------------------------------------------------------------- E4M3
def e4m3_decode(codes):
    """E4M3 codes (uint8) -> float64 values; NaN for 0x7F / 0xFF."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    s = (c >> 7) & 1
    e = (c >> 3) & 0xF
    m = c & 7
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return np.where(s == 1, -mag, mag)


def _exponent_floor(a):
    """floor(log2(a)) for a > 0 (float64), exact via frexp; 0 -> a very small number."""
    _, ex = np.frexp(a)
    return np.where(a > 0, ex - 1, -1000).astype(np.int64)


def e4m3_encode(y):
    """float32 -> E4M3 code, round to nearest even, saturating at +-448.

    On the grid of exponent E (E >= -6; the subnormal range shares the 2^-9 quantum of
    E = -6) a magnitude a is a multiple q of 2^(E-3) with q in [8, 16); code = 8*(E+7) +
    (q - 8).  q is a / 2^(E-3) rounded half to even, and a carry to q = 16 lands on the
    next exponent's first code, so one formula covers every binade.  NaN -> 0x7F.
    """
    y = np.asarray(y, dtype=np.float32)
    a = np.abs(y.astype(np.float64))
    E = np.maximum(_exponent_floor(a), -6)
    q = np.rint(a / np.exp2(E - 3.0))             # exact scaling, ties to even
    code = 8 * (E + 7) + (q.astype(np.int64) - 8)
    code = np.clip(code, 0, 0x7E)                 # satfinite: never the NaN code
    code = np.where(np.isnan(y), 0x7F, code | (np.signbit(y).astype(np.int64) << 7))
    return code.astype(np.uint8)


def e4m3_encode_bruteforce(y):
    """Reference encoder for small arrays: nearest finite E4M3 value, tie -> even code."""
    y = np.asarray(y, dtype=np.float32).ravel()
    pos = np.arange(0, 0x7F, dtype=np.uint8)      # 0x00..0x7E, all finite non-negative
    vals = e4m3_decode(pos)
    out = np.empty(y.shape, dtype=np.uint8)
    for i, v in enumerate(y.astype(np.float64)):
        a = abs(v)
        if a >= E4M3_MAX:
            c = 0x7E
        else:
            d = np.abs(vals - a)
            best = np.flatnonzero(d == d.min())
            c = int(best[0]) if len(best) == 1 else int([b for b in best if b % 2 == 0][0])
        out[i] = c | (0x80 if np.signbit(v) else 0)
    return out


# ----------------------------------------------------------------------------- E5M2
def e5m2_decode(codes):
    """E5M2 codes (uint8) -> float64 values; +-inf for exponent 31 / mantissa 0, NaN for the
    other exponent-31 codes."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    s = (c >> 7) & 1
    e = (c >> 2) & 0x1F
    m = c & 3
    mag = np.where(e == 0, (m / 4.0) * 2.0 ** -14, (1.0 + m / 4.0) * np.exp2(e - 15.0))
    mag = np.where(e == 31, np.where(m == 0, np.inf, np.nan), mag)
    return np.where(s == 1, -mag, mag)


def e5m2_encode(y):
    """float32 -> E5M2 code, round to nearest even, saturating at +-57344.

    As for E4M3 with 2 mantissa bits: on the grid of exponent E (E >= -14; subnormals share
    the 2^-16 quantum of E = -14) a magnitude is q * 2^(E-2) with q in [4, 8); code =
    4*(E+15) + (q - 4); a carry to q = 8 lands on the next exponent's first code.  The
    largest finite code is 0x7B; NaN -> 0x7F.
    """
    y = np.asarray(y, dtype=np.float32)
    a = np.abs(y.astype(np.float64))
    E = np.maximum(_exponent_floor(a), -14)
    q = np.rint(a / np.exp2(E - 2.0))             # exact scaling, ties to even
    code = 4 * (E + 15) + (q.astype(np.int64) - 4)
    code = np.clip(code, 0, 0x7B)                 # satfinite: never infinity or NaN
    code = np.where(np.isnan(y), 0x7F, code | (np.signbit(y).astype(np.int64) << 7))
    return code.astype(np.uint8)


def e5m2_encode_bruteforce(y):
    """Reference encoder for small arrays: nearest finite E5M2 value, tie -> even code."""
    y = np.asarray(y, dtype=np.float32).ravel()
    pos = np.arange(0, 0x7C, dtype=np.uint8)      # 0x00..0x7B, all finite non-negative
    vals = e5m2_decode(pos)
    out = np.empty(y.shape, dtype=np.uint8)
    for i, v in enumerate(y.astype(np.float64)):
        a = abs(v)
        if a >= E5M2_MAX:
            c = 0x7B
        else:
            d = np.abs(vals - a)
            best = np.flatnonzero(d == d.min())
            c = int(best[0]) if len(best) == 1 else int([b for b in best if b % 2 == 0][0])
        out[i] = c | (0x80 if np.signbit(v) else 0)
    return out


# ----------------------------------------------------------------------------- E8M0
def e8m0_decode(codes):
    """E8M0 codes -> float64 2^(c-127); code 255 is NaN."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.float64)
    return np.where(c == 255, np.nan, np.exp2(c - 127.0))


# ----------------------------------------------------------------------------- E2M1
E2M1_VALUES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e2m1_decode(codes):
    """E2M1 4-bit codes (low nibble of a uint8) -> float64.

    code = 8*s + 2*e + m; e = 0 is the subnormal 0.5*m, else 2^(e-1) * (1 + m/2).
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64) & 0xF
    s = c >> 3
    e = (c >> 1) & 3
    m = c & 1
    mag = np.where(e == 0, 0.5 * m, np.exp2(e - 1.0) * (1.0 + m / 2.0))
    return np.where(s == 1, -mag, mag)


def e2m1_encode_rne(y):
    """float32 -> E2M1 code, round to nearest even, saturating at +-6.

    For magnitude a in binade E (E >= 0; below 1 the quantum 0.5 of E = 0 is shared)
    the quantum is 2^(E-1) and code = 2*E + round_half_even(a / 2^(E-1)).
    """
    y = np.asarray(y, dtype=np.float32)
    a = np.abs(y.astype(np.float64))
    E = np.maximum(_exponent_floor(a), 0)
    q = np.rint(a / np.exp2(E - 1.0)).astype(np.int64)
    code = np.minimum(2 * E + q, 7)
    return (code | (np.signbit(y).astype(np.int64) << 3)).astype(np.uint8)


def e2m1_encode_bruteforce(y):
    """Reference: nearest of the 8 magnitudes, tie -> even code, saturate at 6."""
    y = np.asarray(y, dtype=np.float32).ravel()
    out = np.empty(y.shape, dtype=np.uint8)
    for i, v in enumerate(y.astype(np.float64)):
        a = min(abs(v), E2M1_MAX)
        d = np.abs(E2M1_VALUES - a)
        best = np.flatnonzero(d == d.min())
        c = int(best[0]) if len(best) == 1 else int([b for b in best if b % 2 == 0][0])
        out[i] = c | (8 if np.signbit(v) else 0)
    return out


def e2m1_grid_neighbours(a):
    """For magnitudes 0 <= a < 6: the adjacent E2M1 magnitudes lo <= a < hi (float64)."""
    a = np.asarray(a, dtype=np.float64)
    idx = np.searchsorted(E2M1_VALUES, a, side="right") - 1
    idx = np.clip(idx, 0, 6)
    return E2M1_VALUES[idx], E2M1_VALUES[idx + 1], idx


def pack_e2m1(codes):
    """(..., 2n) 4-bit codes -> (..., n) bytes; the even index goes to the low nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] & 0xF) | ((c[..., 1::2] & 0xF) << 4)


def unpack_e2m1(packed):
    """(..., n) bytes -> (..., 2n) 4-bit codes (low nibble first)."""
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out
