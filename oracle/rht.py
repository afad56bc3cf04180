"""16x16 random Hadamard transform (oracle; test infrastructure only).

"NVIDIA developed a method to train neural networks in 4-bit precision", section
"How it works": gradient inputs go through 16x16 random Hadamard transforms before the
4-bit cast.  The page fixes only the size.  Reading taken here (parity unpinned beyond
the spec for the sign derivation; the transform itself is pinned to the Sylvester
Hadamard matrix and to orthogonality by the tests):

* one sign vector d (16 entries of +-1) per tensor: bit i of word 0 of
  Philox4x32-10(counter = (0, 0, 0, 0x52485431), key = rht_seed) is 1 -> d_i = -1;
* for every group of 16 consecutive elements along the quantized dimension:
  v_i = d_i * x_i, then the four in-place butterfly stages h = 1, 2, 4, 8 of the fast
  Walsh-Hadamard transform, each pair (i, i + h) with (i & h) == 0 becoming
  (v_i + v_{i+h}, v_i - v_{i+h}) in FP32, then y_i = v_i * 0.25.

So y = x Q with Q = D H16 / 4, an orthogonal matrix (H16 H16^T = 16 I); applying the
same Q along K to both operands of a GEMM leaves the product unchanged.  Every output
is one fixed FP32 expression of its inputs, so the result is bit-reproducible.
"""
import numpy as np

from .philox import philox4x32_10, seed_to_key

RHT_COUNTER = np.array([0, 0, 0, 0x52485431], dtype=np.uint32)


def rht_signs(rht_seed):
    """The 16 signs (float32 +-1) derived from rht_seed."""
    word = int(philox4x32_10(RHT_COUNTER, seed_to_key(rht_seed))[0])
    bits = np.array([(word >> i) & 1 for i in range(16)])
    return np.where(bits == 1, -1.0, 1.0).astype(np.float32)


def fwht16_stages(v):
    """Butterflies h = 1, 2, 4, 8 on the last axis (length 16), FP32.

    For stage h the 16 positions split into 16 / (2h) blocks of [i .. i+h) (bit h clear)
    followed by [i+h .. i+2h) (bit h set); each pair becomes (a + b, a - b)."""
    v = np.array(v, dtype=np.float32, copy=True)
    lead = v.shape[:-1]
    for h in (1, 2, 4, 8):
        w = v.reshape(lead + (16 // (2 * h), 2, h))
        a = w[..., 0, :].copy()
        b = w[..., 1, :].copy()
        w[..., 0, :] = a + b          # float32 + float32 -> float32 (round to nearest even)
        w[..., 1, :] = a - b
        v = w.reshape(lead + (16,))
    return v


def rht16_lastdim(x, signs):
    """Apply the transform to every 16-element group along the last axis of x (float32)."""
    x = np.asarray(x, dtype=np.float32)
    assert x.shape[-1] % 16 == 0
    g = x.reshape(x.shape[:-1] + (x.shape[-1] // 16, 16))
    v = fwht16_stages(g * signs)     # sign flips are exact
    return (v * np.float32(0.25)).reshape(x.shape)
