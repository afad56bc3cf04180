"""Philox4x32-10 counter-based generator (oracle; test infrastructure only).

The NVFP4 page ("NVIDIA developed a method to train neural networks in 4-bit precision",
section "How it works") uses stochastic rounding and a *random* Hadamard transform but
names no generator.  Both draw their random bits from Philox4x32-10 as published by
Salmon, Moraes, Dror and Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3" (SC'11):

* state: a 128-bit counter (c0, c1, c2, c3) and a 64-bit key (k0, k1), 32-bit words;
* one round: (hi0, lo0) = 0xD2511F53 * c0, (hi1, lo1) = 0xCD9E8D57 * c2 (full 64-bit
  products), then (c0, c1, c2, c3) <- (hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0);
* between rounds the key is bumped by the Weyl constants (0x9E3779B9, 0xBB67AE85);
* ten rounds; the output is the final counter block.
"""
import numpy as np

_M0 = np.uint64(0xD2511F53)
_M1 = np.uint64(0xCD9E8D57)
_W0 = np.uint64(0x9E3779B9)
_W1 = np.uint64(0xBB67AE85)
_MASK = np.uint64(0xFFFFFFFF)
_S32 = np.uint64(32)


def philox4x32_10(counter, key):
    """counter: (..., 4) uint32; key: (..., 2) uint32 (broadcast) -> (..., 4) uint32."""
    ctr = np.asarray(counter, dtype=np.uint32).astype(np.uint64)
    k = np.asarray(key, dtype=np.uint32).astype(np.uint64)
    c0, c1, c2, c3 = (ctr[..., i] for i in range(4))
    k0 = np.broadcast_to(k[..., 0], c0.shape).copy()
    k1 = np.broadcast_to(k[..., 1], c0.shape).copy()
    for rnd in range(10):
        if rnd > 0:
            k0 = (k0 + _W0) & _MASK
            k1 = (k1 + _W1) & _MASK
        p0 = _M0 * c0
        p1 = _M1 * c2
        hi0, lo0 = p0 >> _S32, p0 & _MASK
        hi1, lo1 = p1 >> _S32, p1 & _MASK
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return np.stack([c0, c1, c2, c3], axis=-1).astype(np.uint32)


def seed_to_key(seed):
    """64-bit seed -> Philox key words (low 32 bits, high 32 bits)."""
    s = int(seed) & 0xFFFFFFFFFFFFFFFF
    return np.array([s & 0xFFFFFFFF, s >> 32], dtype=np.uint32)
