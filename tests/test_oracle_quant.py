"""Pins for the oracle's quantizers: the scaled-amax invariant (each tile's amax encodes to
exactly 448), exact round trips on inputs whose scales are powers of two (which fixes the
scale formula, its stored form and its layout), brute-force encoders, brute-force MX
exponent minimality, and the statistics of stochastic rounding."""
import numpy as np
import pytest

import workloads
from oracle import formats as F
from oracle import quant as Q
from oracle import rht as RHT


def exact_matrix(R, C, tr, tc, rng, top=448.0, grid="e4m3", jrange=(-12, 12)):
    """Values on the element grid times a power of two per (tr x tc) tile, with one element
    of each tile at +-top * 2^j: quantization of such a matrix is exact."""
    if grid == "e4m3":
        mags = F.e4m3_decode(rng.integers(0, 0x7F, (R, C)).astype(np.uint8))
    else:
        mags = F.E2M1_VALUES[rng.integers(0, 8, (R, C))]
    sign = np.where(rng.random((R, C)) < 0.5, -1.0, 1.0)
    x = mags * sign
    js = rng.integers(jrange[0], jrange[1], (-(-R // tr), -(-C // tc)))
    for i in range(js.shape[0]):
        for j in range(js.shape[1]):
            blk = x[i * tr:(i + 1) * tr, j * tc:(j + 1) * tc]
            blk[0, 0] = top * (1 if rng.random() < 0.5 else -1)
            blk *= 2.0 ** js[i, j]
    return x.astype(np.float32), js


def test_1x128_exact_roundtrip_pins_scale_and_layout():
    rng = np.random.default_rng(0)
    x, js = exact_matrix(24, 384, 1, 128, rng)
    q, s = Q.quantize_1x128_rowwise(x)
    assert s.shape == (3, 24)
    assert np.array_equal(s, np.exp2(js.T).astype(np.float32))
    deq = F.e4m3_decode(q) * np.repeat(s.T.astype(np.float64), 128, axis=1)
    assert np.array_equal(deq, x.astype(np.float64))


def test_1x128_amax_maps_to_448_on_real_inputs():
    x = Q.as_f32(workloads.bf16_bits(workloads.tiny()["A"]))
    q, s = Q.quantize_1x128_rowwise(x)
    t = np.abs(x).reshape(256, 4, 128)
    amax = t.max(-1, keepdims=True)
    hit = (t == amax) & (amax > 0)
    assert np.all((q.reshape(256, 4, 128)[hit] & 0x7F) == 0x7E)
    # stored decode scale times 448 recovers amax to FP32 rounding
    rel = np.abs(s.T.astype(np.float64) * 448.0 / amax[..., 0] - 1.0)
    assert rel.max() < 2.0 ** -22


def test_1x128_codes_match_bruteforce_encoder():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal((3, 256)) * np.exp2(rng.integers(-10, 10, (3, 1)))).astype(np.float32)
    q, _ = Q.quantize_1x128_rowwise(x)
    t = x.reshape(3, 2, 128)
    sf = (np.float32(448.0) / np.abs(t).max(-1)).astype(np.float32)
    y = (t * sf[..., None]).astype(np.float32).reshape(3, 256)
    assert np.array_equal(q, F.e4m3_encode_bruteforce(y).reshape(3, 256))


def test_1x128_zero_tile_and_colwise_transpose():
    rng = np.random.default_rng(2)
    x, js = exact_matrix(256, 256, 128, 1, rng)
    x[:128, 5] = 0.0
    qc, sc = Q.quantize_1x128_colwise(x)
    assert qc.shape == (256, 256) and sc.shape == (2, 256)
    assert sc[0, 5] == 1.0 and np.all(qc[5, :128] == 0)
    keep = np.ones(256, bool)
    keep[5] = False
    expect = np.exp2(js).astype(np.float32)
    assert np.array_equal(sc[:, keep], expect[:, keep])
    deq = F.e4m3_decode(qc) * np.repeat(sc.T.astype(np.float64), 128, axis=1)
    assert np.array_equal(deq, x.T.astype(np.float64))


def test_scale_overflow_clamps_to_flt_max():
    x = np.zeros((1, 128), np.float32)
    x[0, 0] = np.float32(1e-40)         # a subnormal amax: 448 / amax overflows FP32
    q, s = Q.quantize_1x128_rowwise(x)
    assert np.isfinite(s[0, 0]) and s[0, 0] == np.float32(1.0) / F.FLT_MAX


def test_128x128_exact_and_transposed_layout():
    rng = np.random.default_rng(3)
    w, js = exact_matrix(256, 384, 128, 128, rng)
    q, qt, s = Q.quantize_128x128(w)
    assert s.shape == (3, 2) and np.array_equal(qt, q.T)
    assert np.array_equal(s, np.exp2(js.T).astype(np.float32))
    scale = np.exp2(np.repeat(np.repeat(js, 128, 0), 128, 1).astype(np.float64))
    assert np.array_equal(F.e4m3_decode(q) * scale, w.astype(np.float64))


def test_128x128_amax_maps_to_448():
    w = Q.as_f32(workloads.bf16_bits(workloads.tiny()["B"]))
    q, _, _ = Q.quantize_128x128(w)
    for i in range(4):
        for j in range(2):
            blk = np.abs(w[128 * i:128 * i + 128, 128 * j:128 * j + 128])
            hit = blk == blk.max()
            assert np.all((q[128 * i:128 * i + 128, 128 * j:128 * j + 128][hit] & 0x7F) == 0x7E)


def test_per_tensor_exact_and_amax():
    rng = np.random.default_rng(4)
    x = F.e4m3_decode(rng.integers(0, 0x7E, (64, 96)).astype(np.uint8)) * 2.0 ** -5
    x[7, 9] = -448 * 2.0 ** -5
    q, s = Q.quantize_tensor(x.astype(np.float32))
    assert s == np.float32(2.0 ** -5) and q[7, 9] == 0xFE
    assert np.array_equal(F.e4m3_decode(q) * float(s), x)


# ----------------------------------------------------------------------------- MX
def _mx_bruteforce(amax):
    out = []
    for a in np.asarray(amax, np.float32).astype(np.float64).ravel():
        if a == 0:
            out.append(-127)
            continue
        for e in range(-127, 128):
            if a <= 448.0 * 2.0 ** e:
                out.append(e)
                break
        else:
            out.append(127)
    return np.array(out)


def test_mx_exponent_is_minimal_bruteforce():
    rng = np.random.default_rng(5)
    a = [0.0, 448.0, 448.0 * 2 ** -3, np.nextafter(np.float32(448.0), np.float32(1e9)),
         np.float32(1e-40), np.float32(3e-45), np.float32(3.3e38), 1.0, 1.75, 1.7500001, 224.0]
    a = np.concatenate([np.float32(a), (rng.random(3000) * np.exp2(rng.integers(-140, 120, 3000)))
                        .astype(np.float32)])
    assert np.array_equal(Q.mx_exponent(a), _mx_bruteforce(a))


def test_mx_no_saturation_and_exact_roundtrip():
    rng = np.random.default_rng(6)
    x, js = exact_matrix(16, 256, 1, 32, rng)
    q, e = Q.quantize_mx_rowwise(x)
    assert np.array_equal(e.astype(np.int64) - 127, js)
    deq = F.e4m3_decode(q) * np.repeat(F.e8m0_decode(e), 32, axis=1)
    assert np.array_equal(deq, x.astype(np.float64))
    # random inputs: the scaled amax lies in (224, 448] and nothing exceeds 448
    xr = Q.as_f32(workloads.bf16_bits(workloads.tiny()["A"]))
    q, e = Q.quantize_mx_rowwise(xr)
    amax = np.abs(xr).reshape(256, 16, 32).max(-1)
    scaled = amax.astype(np.float64) / F.e8m0_decode(e)
    assert np.all((scaled > 224) & (scaled <= 448))
    assert np.all(np.abs(xr).reshape(256, 16, 32) / F.e8m0_decode(e)[..., None] <= 448)


def test_mx_colwise_is_transposed():
    x = Q.as_f32(workloads.bf16_bits(workloads.tiny()["B"]))
    qc, ec = Q.quantize_mx_colwise(x)
    assert qc.shape == (256, 512) and ec.shape == (256, 16)
    qr, er = Q.quantize_mx_rowwise(np.ascontiguousarray(x.T))
    assert np.array_equal(qc, qr) and np.array_equal(ec, er)


# ----------------------------------------------------------------------------- NVFP4
def test_nvfp4_exact_grid_roundtrip():
    rng = np.random.default_rng(7)
    x, js = exact_matrix(8, 128, 1, 16, rng, top=6.0, grid="e2m1", jrange=(-5, 5))
    q, sf, g = Q.quantize_nvfp4_rowwise(x)
    deq = _deq_nvfp4(q, sf, g)
    assert np.allclose(deq, x.astype(np.float64), rtol=2.0 ** -23, atol=0)
    jmax = js.max()
    assert np.array_equal(F.e4m3_decode(sf), 448.0 * np.exp2(js - jmax))


def _deq_nvfp4(q, sf, g):
    codes = F.unpack_e2m1(q)
    return F.e2m1_decode(codes) * np.repeat(F.e4m3_decode(sf), 16, axis=1) * float(g)


def test_nvfp4_scale_invariants_and_rne_bruteforce():
    d = workloads.nvfp4(M=64, H=64, F=256, which=("dY",))
    x = Q.as_f32(workloads.bf16_bits(d["dY"]))
    q, sf, g = Q.quantize_nvfp4_rowwise(x)
    dec = F.e4m3_decode(sf)
    assert np.all(dec <= 448) and np.all(sf < 0x80)
    # rebuild y from the stored scales and compare codes with the brute-force encoder
    S_g = np.float32(np.float32(2688.0) / np.float32(np.abs(x).max()))
    assert np.float32(np.float32(1.0) / S_g) == g
    enc = np.where(sf == 0, 0, (S_g / dec.astype(np.float32))).astype(np.float32)
    y = (x.reshape(64, 16, 16) * enc[..., None]).astype(np.float32).reshape(64, 256)
    assert np.all(np.abs(y) <= 6.0 / (1 - 2.0 ** -4))
    assert np.array_equal(F.unpack_e2m1(q), F.e2m1_encode_bruteforce(y).reshape(64, 256))


def test_nvfp4_sr_is_unbiased_and_picks_neighbours():
    n_blocks = 65536
    v, w = np.float32(1.0), np.float32(0.3)
    x = np.full((n_blocks, 16), w, np.float32)
    x[:, 0] = v
    x = x.reshape(1024, 1024)
    q, sf, g = Q.quantize_nvfp4_rowwise(x, sr=True, sr_seed=6)
    deq = _deq_nvfp4(q, sf, g).reshape(n_blocks, 16)[:, 1:].ravel()
    scale = float(F.e4m3_decode(sf[0, 0])) * float(g)
    y = float(np.float32(w * np.float32(np.float32(np.float32(2688.0) / v)
                                        / np.float32(F.e4m3_decode(sf[0, 0])))))
    lo, hi, _ = F.e2m1_grid_neighbours(np.array([y]))
    vals = np.unique(deq / scale)
    assert set(np.round(vals, 6)) <= {round(float(lo[0]), 6), round(float(hi[0]), 6)}
    p = (y - lo[0]) / (hi[0] - lo[0])
    sigma = np.sqrt(p * (1 - p)) * (hi[0] - lo[0])
    mean = (deq / scale).mean()
    assert abs(mean - y) < 4 * sigma / np.sqrt(deq.size)
    assert deq.size > 900_000
    # a different seed changes the draws, the same seed reproduces them
    q2, _, _ = Q.quantize_nvfp4_rowwise(x, sr=True, sr_seed=6)
    q3, _, _ = Q.quantize_nvfp4_rowwise(x, sr=True, sr_seed=7)
    assert np.array_equal(q, q2) and not np.array_equal(q, q3)


def _sr_pattern(R, C):
    """R x C values whose NVFP4 quantization leaves one fair coin per element: each 16-group
    holds one anchor 6.0 (the block and tensor amax, so S_g = 448, the block scale is 448 and
    the encode scale is exactly 1) and fifteen 1.25s, which sit halfway between the E2M1
    values 1.0 (code 2) and 1.5 (code 3).  With p = 1/2 the reading's rule rounds up iff the
    element's 32-bit Philox word is below 2^31."""
    x = np.full((R, C), 1.25, np.float32)
    x[:, 0::16] = 6.0
    return x


def _up(q_packed):
    """Rounding decisions (True = up to 1.5) of a quantized _sr_pattern, as a code matrix."""
    codes = F.unpack_e2m1(q_packed)
    fair = codes != 7
    assert set(np.unique(codes[fair])) <= {2, 3}
    return codes == 3


def _corr(a, b):
    a = a.astype(np.float64) - a.mean()
    b = b.astype(np.float64) - b.mean()
    return float((a * b).sum() / np.sqrt((a * a).sum() * (b * b).sum()))


def test_nvfp4_sr_words_are_independent_within_and_across_philox_blocks():
    """Reading: element idx of an output takes word (idx & 3) of the Philox call at counter
    idx >> 2.  Over ~10^6 fair coins the decisions of the four elements sharing one call,
    and of the same element slot in neighbouring calls, must be uncorrelated (|r| < 4/sqrt(n)):
    a word mapping that reuses one word for several elements (e.g. always word 0, or word
    (idx >> 2) & 3) makes them identical."""
    R, C = 1024, 1088
    x = _sr_pattern(R, C)
    for name, (q, _, _) in (("rowwise", Q.quantize_nvfp4_rowwise(x, sr=True, sr_seed=6)),
                            ("colwise", Q.quantize_nvfp4_colwise(np.ascontiguousarray(x.T), sr=True, sr_seed=6))):
        d = _up(q).reshape(-1, 16)[:, 4:].reshape(-1, 3, 4)    # Philox blocks 1..3 of each group
        n = d.shape[0]
        assert 3 * 4 * n >= 1_000_000 - 200_000 and abs(d.mean() - 0.5) < 4 * 0.5 / np.sqrt(d.size)
        bound = 4.0 / np.sqrt(n)
        for blk in range(3):
            for i in range(4):
                for j in range(i + 1, 4):
                    r = _corr(d[:, blk, i], d[:, blk, j])
                    assert abs(r) < bound, (name, "same call", blk, i, j, r)
        for blk in range(2):
            for i in range(4):
                r = _corr(d[:, blk, i], d[:, blk + 1, i])
                assert abs(r) < bound, (name, "neighbouring calls", blk, i, r)


def test_nvfp4_sr_rowwise_and_colwise_outputs_draw_from_different_streams():
    """The two outputs of one tensor use tags 0 and 1: at the same output index their fair
    coins must be uncorrelated (one stream for both would make them identical)."""
    x = _sr_pattern(1024, 1024)
    q_row, _, _ = Q.quantize_nvfp4_rowwise(x, sr=True, sr_seed=11)
    q_col, _, _ = Q.quantize_nvfp4_colwise(np.ascontiguousarray(x.T), sr=True, sr_seed=11)
    a, b = _up(q_row).ravel(), _up(q_col).ravel()
    keep = (np.arange(a.size) % 16) != 0
    assert abs(_corr(a[keep], b[keep])) < 4.0 / np.sqrt(keep.sum())


def test_nvfp4_sr_decisions_match_brute_force_over_output_indices():
    """Brute force on a small non-square input: every fair coin of the rowwise output (R x C,
    tag 0) and of the colwise output (C x R, transposed, tag 1) is recomputed element by
    element from one scalar call of the generator (pinned by its published known-answer
    vectors) at counter (idx >> 2, 0, 0, tag), word idx & 3, idx the element's position in
    that output.  A colwise output indexed by the input position, a wrong word or a wrong
    counter split fails here."""
    from oracle.philox import philox4x32_10, seed_to_key
    R, C = 48, 32
    x = _sr_pattern(R, C)                       # rowwise coins along rows
    xc = np.ascontiguousarray(_sr_pattern(C, R).T)   # R x C; colwise coins along columns
    key = seed_to_key(0x1234_5678_9ABC)
    cases = ((Q.quantize_nvfp4_rowwise(x, sr=True, sr_seed=0x1234_5678_9ABC)[0], 0, (R, C)),
             (Q.quantize_nvfp4_colwise(xc, sr=True, sr_seed=0x1234_5678_9ABC)[0], 1, (C, R)))
    for q, tag, (orows, ocols) in cases:
        up = _up(q)
        assert up.shape == (orows, ocols)
        for r in range(orows):
            for c in range(ocols):
                if c % 16 == 0:
                    continue
                idx = r * ocols + c
                w = philox4x32_10(np.array([idx >> 2, 0, 0, tag], np.uint32), key)[idx & 3]
                assert bool(up[r, c]) == (int(w) < (1 << 31)), (tag, r, c)


def test_nvfp4_rht_roundtrip_close_and_orthogonal_gemm():
    rng = np.random.default_rng(8)
    A = rng.standard_normal((32, 256)).astype(np.float32)
    B = rng.standard_normal((24, 256)).astype(np.float32)
    qa, sa, ga = Q.quantize_nvfp4_rowwise(A, rht=True, rht_seed=5)
    qb, sb, gb = Q.quantize_nvfp4_rowwise(B, rht=True, rht_seed=5)
    C_rht = _deq_nvfp4(qa, sa, ga) @ _deq_nvfp4(qb, sb, gb).T
    qa0, sa0, ga0 = Q.quantize_nvfp4_rowwise(A)
    qb0, sb0, gb0 = Q.quantize_nvfp4_rowwise(B)
    C_plain = _deq_nvfp4(qa0, sa0, ga0) @ _deq_nvfp4(qb0, sb0, gb0).T
    C = A.astype(np.float64) @ B.astype(np.float64).T
    scale = np.sqrt(256.0)
    assert np.abs(C_rht - C).max() < 0.25 * scale * 4
    assert np.abs(C_plain - C).max() < 0.25 * scale * 4
    # undoing the transform on the dequantized operand recovers A approximately
    s = RHT.rht_signs(5)
    Qm = np.diag(s.astype(np.float64)) @ __import__("scipy").linalg.hadamard(16) / 4.0
    Ad = _deq_nvfp4(qa, sa, ga).reshape(32, 16, 16) @ Qm.T
    assert np.abs(Ad.reshape(32, 256) - A).max() < 1.0


def test_nvfp4_colwise_uses_tag_one():
    x = np.full((32, 16), 0.3, np.float32)
    x[0] = 1.0
    qc, sc, gc = Q.quantize_nvfp4_colwise(x, sr=True, sr_seed=9)
    qr, sr_, gr = Q.quantize_nvfp4_rowwise(np.ascontiguousarray(x.T), sr=True, sr_seed=9, tag=1)
    assert np.array_equal(qc, qr) and np.array_equal(sc, sr_)
    qr0, _, _ = Q.quantize_nvfp4_rowwise(np.ascontiguousarray(x.T), sr=True, sr_seed=9, tag=0)
    assert not np.array_equal(qc, qr0)


def test_sf_tiled_layout_is_a_permutation():
    rng = np.random.default_rng(10)
    for R, S in [(128, 4), (200, 7), (300, 33), (5, 1)]:
        sf = rng.integers(1, 255, (R, S)).astype(np.uint8)
        flat = Q.sf_to_tiled(sf)
        assert flat.size == Q.sf_tiled_size(R, S)
        assert np.array_equal(Q.sf_from_tiled(flat, R, S), sf)
        assert np.count_nonzero(flat) == R * S
        rr, cc = np.meshgrid(np.arange(R), np.arange(S), indexing="ij")
        assert len(np.unique(Q.sf_tiled_offset(rr, cc, S))) == R * S


# ----------------------------------------------------------------------------- delayed
def test_delayed_with_own_amax_in_history_equals_current_scaling():
    """History holding exactly this tensor's amax: delayed scaling reduces to current
    (per-tensor) scaling, codes and decode scale identical."""
    x = Q.as_f32(workloads.bf16_bits(workloads.tiny()["A"]))
    q, s = Q.quantize_tensor(x)
    amax = np.float32(np.max(np.abs(x)))
    qd, sd, a = Q.quantize_tensor_delayed(x, np.float32([0.0, amax, amax / 3]))
    assert np.array_equal(qd, q) and sd == s and a == amax


def test_delayed_scale_from_history_max_and_saturation():
    """The scale comes from the largest historical amax (a power of two here, so it is exact);
    values beyond the history's range saturate; the returned amax is the tensor's own."""
    rng = np.random.default_rng(11)
    x = (rng.standard_normal((64, 96)) * 4.0).astype(np.float32)
    x[3, 5] = 100.0                              # beyond the historical range
    hist = np.float32([2.0, 7.0, 8.0, 0.0])      # max 8 -> sf = 448 / 8 = 56
    q, s, a = Q.quantize_tensor_delayed(x, hist)
    assert s == np.float32(1.0 / 56.0) and a == np.float32(100.0)
    assert q[3, 5] == 0x7E                        # saturated at +448
    assert np.array_equal(q, F.e4m3_encode_bruteforce((x * np.float32(56.0)).ravel()).reshape(x.shape))


def test_delayed_e5m2_and_empty_history():
    x = np.float32([[1.0, -2.0, 3.0, 0.5]])
    q, s, a = Q.quantize_tensor_delayed(x, np.float32([0.0, 0.0]), fmt="e5m2")   # no history -> sf 1
    assert s == np.float32(1.0) and a == np.float32(3.0)
    assert np.array_equal(F.e5m2_decode(q).astype(np.float32), x)
    q, s, _ = Q.quantize_tensor_delayed(x, np.float32([3584.0]), fmt="e5m2")      # sf = 57344 / 3584 = 16
    assert s == np.float32(1.0 / 16.0)
    assert np.array_equal(F.e5m2_decode(q) * float(s), x.astype(np.float64))
    q, s, _ = Q.quantize_tensor_delayed(x, np.float32([4.0]), fmt="e5m2")         # sf = 14336, not exact
    assert s == np.float32(np.float32(1.0) / np.float32(14336.0))
    assert np.array_equal(q, F.e5m2_encode_bruteforce(x.ravel() * np.float32(14336.0)).reshape(x.shape))


# ------------------------------------------------------------ NVFP4 16x16 weight blocks
def test_nvfp4_2d_exact_grid_roundtrip():
    """Each 16x16 block on the E2M1 grid times 2^j, with one element at +-6 * 2^j: every code
    is exact, the block scale decodes to 448 * 2^(j - jmax) and both layouts round-trip."""
    rng = np.random.default_rng(17)
    x, js = exact_matrix(48, 64, 16, 16, rng, top=6.0, grid="e2m1", jrange=(-5, 5))
    q_row, sf_row, q_col, sf_col, g = Q.quantize_nvfp4_2d(x)
    assert np.allclose(_deq_nvfp4(q_row, sf_row, g), x.astype(np.float64), rtol=2.0 ** -23, atol=0)
    assert np.allclose(_deq_nvfp4(q_col, sf_col, g), x.T.astype(np.float64), rtol=2.0 ** -23, atol=0)
    want = 448.0 * np.exp2(js - js.max())                    # (R/16, C/16)
    assert np.array_equal(F.e4m3_decode(sf_row), np.repeat(want, 16, axis=0))
    assert np.array_equal(F.e4m3_decode(sf_col), np.repeat(want.T, 16, axis=0))


def test_nvfp4_2d_reduces_to_1d_when_block_rows_or_columns_repeat():
    """If the 16 rows of every block band are equal, a 16x16 block's amax is each row
    group's amax and the rowwise output is the 1x16 quantizer's; likewise for columns."""
    rng = np.random.default_rng(18)
    base = (rng.standard_normal((4, 96)) * 0.02).astype(np.float32)
    base[1, 5] = 0.9                                          # an outlier block
    rows_rep = np.repeat(base, 16, axis=0)                    # (64, 96)
    q_row, sf_row, _, _, g = Q.quantize_nvfp4_2d(rows_rep)
    q1, sf1, g1 = Q.quantize_nvfp4_rowwise(rows_rep)
    assert np.array_equal(q_row, q1) and np.array_equal(sf_row, sf1) and g == g1
    cols_rep = np.ascontiguousarray(rows_rep.T)               # (96, 64): columns repeat
    _, _, q_col, sf_col, g = Q.quantize_nvfp4_2d(cols_rep)
    q2, sf2, g2 = Q.quantize_nvfp4_colwise(cols_rep)
    assert np.array_equal(q_col, q2) and np.array_equal(sf_col, sf2) and g == g2


def test_nvfp4_2d_bruteforce_and_layout_consistency():
    """Per block: amax over 256 values by a plain loop, the scale by the brute-force E4M3
    encoder, each code by the brute-force E2M1 encoder; both layouts hold the same codes
    and dequantize to one matrix."""
    d = workloads.nvfp4(M=64, H=32, F=48, which=("W",))
    x = Q.as_f32(workloads.bf16_bits(d["W"]))                 # (32, 48) weights
    x[3, 7] = np.float32(0.75)
    q_row, sf_row, q_col, sf_col, g = Q.quantize_nvfp4_2d(x)
    S_g = np.float32(np.float32(2688.0) / np.float32(np.abs(x).max()))
    assert g == np.float32(np.float32(1.0) / S_g)
    codes = np.zeros(x.shape, np.uint8)
    for bi in range(2):
        for bj in range(3):
            blk = x[16 * bi:16 * bi + 16, 16 * bj:16 * bj + 16]
            m = max(abs(float(v)) for v in blk.ravel())
            sb = int(F.e4m3_encode_bruteforce(np.float32(np.float32(np.float32(m) / np.float32(6.0)) * S_g))[0])
            assert np.all(sf_row[16 * bi:16 * bi + 16, bj] == sb) and np.all(sf_col[16 * bj:16 * bj + 16, bi] == sb)
            enc = np.float32(0.0) if sb == 0 else np.float32(S_g / np.float32(F.e4m3_decode(np.uint8(sb))))
            codes[16 * bi:16 * bi + 16, 16 * bj:16 * bj + 16] = F.e2m1_encode_bruteforce(
                (blk * enc).astype(np.float32)).reshape(16, 16)
    assert np.array_equal(F.unpack_e2m1(q_row), codes)
    assert np.array_equal(F.unpack_e2m1(q_col), codes.T)
    assert np.array_equal(_deq_nvfp4(q_row, sf_row, g), _deq_nvfp4(q_col, sf_col, g).T)


def test_nvfp4_2d_sub_rectangle_with_global_amax():
    """A 16-aligned sub-rectangle quantized with the whole tensor's amax equals the matching
    slice of the whole tensor's result (what the sampled full-size checks rely on)."""
    rng = np.random.default_rng(19)
    x = (rng.standard_normal((64, 80)) * 0.02).astype(np.float32)
    x[50, 3] = np.float32(-1.5)
    q_row, sf_row, q_col, sf_col, g = Q.quantize_nvfp4_2d(x)
    G = np.abs(x).max()
    a_row, a_sfr, a_col, a_sfc, ga = Q.quantize_nvfp4_2d(x[16:48, 32:80], amax=G)
    assert ga == g
    assert np.array_equal(a_row, q_row[16:48, 16:40]) and np.array_equal(a_sfr, sf_row[16:48, 2:5])
    assert np.array_equal(a_col, q_col[32:80, 8:24]) and np.array_equal(a_sfc, sf_col[32:80, 1:3])
