"""Writes tests/golden/oracle_small.json: a small BF16 input with edge cases and what the
oracle's quantizers make of it.  Calls only oracle/ (test infrastructure).  The file is a
regression fixture for the oracle itself: a later change to the oracle's arithmetic that
changes these bytes must name, in its commit message, the page passage or reading behind it.

Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from oracle import formats as F  # noqa: E402
from oracle import quant as Q  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_small.json")


def small_input():
    """16 x 128 BF16 bit patterns: a spread of magnitudes and signs, an all-zero row, a row
    with one value near the BF16 maximum, a row of subnormals and a row of signed zeros."""
    k = np.arange(16 * 128, dtype=np.int64).reshape(16, 128)
    mag = np.exp2(((k * 7) % 23) - 12.0) * (1.0 + (k % 7) / 8.0)
    sign = np.where((k * 5) % 3 == 0, -1.0, 1.0)
    x = (sign * mag).astype(np.float32)
    x[0] = 0.0
    x[1, 17] = np.float32(3.0e38)
    x[2] = np.float32(1.0e-40) * (1 + np.arange(128, dtype=np.float32) % 5)
    x[3] = np.where(np.arange(128) % 2 == 0, np.float32(0.0), np.float32(-0.0))
    return F.f32_to_bf16_bits(x)


def nvfp4_input():
    """The same input without its near-maximum value (row 1 holds 96.0 there instead).  NVFP4
    scales every 16-block against the tensor amax, so with 3e38 in the tensor every other
    block scale would round to zero; here most blocks get a non-zero E4M3 scale and the
    stochastic-rounding and transform entries make real decisions."""
    x = small_input().copy()
    x[1, 17] = F.f32_to_bf16_bits(np.array([96.0], np.float32))[0]
    return x


def hexes(a, width):
    """One hex string per row (each element `width` hex digits)."""
    a = np.atleast_2d(np.asarray(a))
    return ["".join(format(int(v), f"0{width}x") for v in row) for row in a]


def f32hex(v):
    return hexes(np.asarray(v, dtype=np.float32).reshape(1, -1).view(np.uint32), 8)


def build():
    x = small_input()
    q1, s1 = Q.quantize_1x128_rowwise(x)
    qm, em = Q.quantize_mx_rowwise(x)
    qt, st = Q.quantize_tensor(x)
    x4 = nvfp4_input()
    n_q, n_s, n_g = Q.quantize_nvfp4_rowwise(x4)
    r_q, r_s, r_g = Q.quantize_nvfp4_rowwise(x4, rht=True, rht_seed=5, sr=True, sr_seed=6)
    c_q, c_s, c_g = Q.quantize_nvfp4_colwise(x4, rht=True, rht_seed=5, sr=True, sr_seed=6)
    w_row, w_sr, w_col, w_sc, w_g = Q.quantize_nvfp4_2d(x4)
    return {
        "source": "tests/golden/make_golden.py (oracle/ only)",
        "shape": [16, 128],
        "x_bf16": hexes(x, 4),
        "x_nvfp4_bf16": hexes(x4, 4),
        "1x128_rowwise": {"cite": "Can you explain the role of FP8 precision in DeepSeek-V3 training, "
                                  "Fine-grained quantization / Online quantization",
                          "q": hexes(q1, 2), "s": f32hex(s1)},
        "mx32_rowwise": {"cite": "Accelerating FP8 training performance with the NVIDIA NeMo framework "
                                 "(MXFP8, blocks of 32)",
                         "q": hexes(qm, 2), "e8m0": hexes(em, 2)},
        "per_tensor": {"cite": "Accelerating FP8 training performance with the NVIDIA NeMo framework "
                               "(per-tensor scaling)",
                       "q": hexes(qt, 2), "s": f32hex([st])},
        "nvfp4_rowwise_rne": {"cite": "NVIDIA developed a method to train neural networks in 4-bit precision, "
                                      "How it works",
                              "q": hexes(n_q, 2), "sf": hexes(n_s, 2), "g": f32hex([n_g])},
        "nvfp4_rowwise_rht5_sr6": {"q": hexes(r_q, 2), "sf": hexes(r_s, 2), "g": f32hex([r_g])},
        "nvfp4_colwise_rht5_sr6": {"q": hexes(c_q, 2), "sf": hexes(c_s, 2), "g": f32hex([c_g])},
        "nvfp4_16x16": {"q_row": hexes(w_row, 2), "sf_row": hexes(w_sr, 2), "q_col": hexes(w_col, 2),
                        "sf_col": hexes(w_sc, 2), "g": f32hex([w_g])},
    }


if __name__ == "__main__":
    with open(OUT, "w") as f:
        json.dump(build(), f, indent=1)
        f.write("\n")
    print(OUT)
