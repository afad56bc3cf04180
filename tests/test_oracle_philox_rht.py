"""Pins for Philox (the generator's published known-answer vectors, statistics here;
bit-exact against cuRAND in the GPU tests) and for the random Hadamard transform (Sylvester
Hadamard matrix from SciPy, orthogonality)."""
import os

import numpy as np
import scipy.linalg

from oracle import philox, rht

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_philox_known_answer_vectors():
    """tests/golden/philox4x32_10_kat.txt: counter, key -> output words published with the
    generator's reference implementation."""
    rows = [line.split() for line in open(os.path.join(GOLDEN, "philox4x32_10_kat.txt"))
            if line.strip() and not line.startswith("#")]
    assert len(rows) == 3
    for r in rows:
        w = [int(x, 16) for x in r]
        out = philox.philox4x32_10(np.array([w[0:4]], dtype=np.uint32), np.array(w[4:6], dtype=np.uint32))
        assert [int(x) for x in np.asarray(out).ravel()] == w[6:10]


def test_philox_deterministic_and_key_sensitive():
    ctr = np.array([[i, 0, 0, 0] for i in range(8)], dtype=np.uint32)
    a = philox.philox4x32_10(ctr, philox.seed_to_key(7))
    b = philox.philox4x32_10(ctr, philox.seed_to_key(7))
    c = philox.philox4x32_10(ctr, philox.seed_to_key(8))
    assert a.dtype == np.uint32 and a.shape == (8, 4)
    assert np.array_equal(a, b)
    assert not np.any(a == c)


def test_philox_bits_balanced_and_uniform():
    n = 1 << 16
    ctr = np.stack([np.arange(n, dtype=np.uint32), np.zeros(n, np.uint32),
                    np.zeros(n, np.uint32), np.full(n, 3, np.uint32)], axis=-1)
    out = philox.philox4x32_10(ctr, philox.seed_to_key(0x1234_5678_9ABC)).ravel()
    bits = ((out[:, None] >> np.arange(32, dtype=np.uint32)) & 1).mean(axis=0)
    assert np.all(np.abs(bits - 0.5) < 0.01)
    hist = np.bincount(out >> np.uint32(28), minlength=16)
    expect = out.size / 16
    chi2 = float(((hist - expect) ** 2 / expect).sum())
    assert chi2 < 45.0          # 15 dof, p ~ 1e-4


def test_philox_single_counter_bit_avalanche():
    base = np.zeros((1, 4), np.uint32)
    flip = base.copy()
    flip[0, 0] = 1
    k = philox.seed_to_key(99)
    x = philox.philox4x32_10(base, k) ^ philox.philox4x32_10(flip, k)
    pop = sum(bin(int(w)).count("1") for w in x.ravel())
    assert 40 < pop < 88        # about half of 128 bits change


def test_fwht_is_sylvester_hadamard():
    H = rht.fwht16_stages(np.eye(16, dtype=np.float32)).astype(np.float64)
    # row i of the output is H applied to e_i; Sylvester H16 is symmetric
    assert np.array_equal(H, scipy.linalg.hadamard(16).astype(np.float64))
    assert np.array_equal(H @ H.T, 16 * np.eye(16))


def test_rht_signs_are_pm1_and_seeded():
    s5 = rht.rht_signs(5)
    assert set(np.unique(s5)) <= {-1.0, 1.0} and s5.shape == (16,)
    assert np.array_equal(s5, rht.rht_signs(5))
    assert not np.array_equal(s5, rht.rht_signs(6)) or not np.array_equal(s5, rht.rht_signs(7))


def test_rht_matrix_is_orthogonal():
    s = rht.rht_signs(5)
    Q = rht.rht16_lastdim(np.eye(16, dtype=np.float32), s).astype(np.float64)
    expect = np.diag(s.astype(np.float64)) @ scipy.linalg.hadamard(16) / 4.0
    assert np.array_equal(Q, expect)
    assert np.array_equal(Q @ Q.T, np.eye(16))


def test_rht_small_integers_equal_fp64_product():
    rng = np.random.default_rng(11)
    s = rht.rht_signs(123)
    x = rng.integers(-64, 64, (9, 48)).astype(np.float32)
    y = rht.rht16_lastdim(x, s).astype(np.float64)
    Q = np.diag(s.astype(np.float64)) @ scipy.linalg.hadamard(16) / 4.0
    expect = np.concatenate([x[:, 16 * g:16 * g + 16].astype(np.float64) @ Q
                             for g in range(3)], axis=1)
    assert np.array_equal(y, expect)


def test_rht_preserves_products():
    rng = np.random.default_rng(12)
    s = rht.rht_signs(5)
    A = rng.integers(-8, 8, (6, 64)).astype(np.float32)
    B = rng.integers(-8, 8, (5, 64)).astype(np.float32)
    AQ = rht.rht16_lastdim(A, s).astype(np.float64)
    BQ = rht.rht16_lastdim(B, s).astype(np.float64)
    assert np.array_equal(AQ @ BQ.T, A.astype(np.float64) @ B.astype(np.float64).T)
