"""Pins for the GEMM oracle: on operands whose quantization is exact the reference equals
the FP64 product of the raw inputs (fixes operand orientation and every scale mode),
exact rational arithmetic on a tiny case, the acceptance bound itself, and the pages'
qualitative claim that fine-grained scaling beats per-tensor scaling."""
from fractions import Fraction

import numpy as np

import workloads
from oracle import formats as F
from oracle import gemm as G
from oracle import quant as Q
from tests.test_oracle_quant import exact_matrix


def test_blockwise_fprop_dgrad_wgrad_exact_cases():
    rng = np.random.default_rng(0)
    M, K, N = 96, 384, 256
    X, _ = exact_matrix(M, K, 1, 128, rng)                  # activations, 1x128 tiles
    W, _ = exact_matrix(K, N, 128, 128, rng)                # weights K x N, 128x128 blocks
    qx, sx = Q.quantize_1x128_rowwise(X)
    qw, qwt, sw = Q.quantize_128x128(W)
    ref = X.astype(np.float64) @ W.astype(np.float64)
    # FPROP: C = X . W  with B = W^T (N x K)
    C, T = G.reference(G.dequant_a_1x128(qx, sx), G.dequant_b_blockwise(qwt, sw, G.FPROP))
    assert np.array_equal(C, ref)
    # DGRAD: dX = dY . W^T ; B = W (rows are W's K, columns W's N)
    dY, _ = exact_matrix(M, N, 1, 128, rng)
    qd, sd = Q.quantize_1x128_rowwise(dY)
    C, _ = G.reference(G.dequant_a_1x128(qd, sd), G.dequant_b_blockwise(qw, sw, G.DGRAD))
    assert np.array_equal(C, dY.astype(np.float64) @ W.astype(np.float64).T)
    # WGRAD: dW = X^T . dY, both operands 1x128 along tokens (colwise, transposed)
    Xt, _ = exact_matrix(256, 128, 128, 1, rng)              # tokens x features
    dYt, _ = exact_matrix(256, 64, 128, 1, rng)
    qa, sa = Q.quantize_1x128_colwise(Xt)
    qb, sb = Q.quantize_1x128_colwise(dYt)
    C, _ = G.reference(G.dequant_a_1x128(qa, sa), G.dequant_b_blockwise(qb, sb, G.WGRAD))
    assert np.array_equal(C, Xt.astype(np.float64).T @ dYt.astype(np.float64))


def test_mx_and_per_tensor_exact_cases():
    rng = np.random.default_rng(1)
    A, _ = exact_matrix(40, 192, 1, 32, rng)
    W, _ = exact_matrix(192, 72, 32, 1, rng)
    qa, ea = Q.quantize_mx_rowwise(A)
    qb, eb = Q.quantize_mx_colwise(W)
    C, _ = G.reference(G.dequant_mx(qa, ea), G.dequant_mx(qb, eb))
    assert np.array_equal(C, A.astype(np.float64) @ W.astype(np.float64))
    At = (F.e4m3_decode(rng.integers(0, 0x7E, (8, 64)).astype(np.uint8)) * 4).astype(np.float32)
    At[0, 0] = 448 * 4
    qt, st = Q.quantize_tensor(At)
    C, _ = G.reference(G.dequant_tensor(qt, st), G.dequant_tensor(qt, st))
    assert np.array_equal(C, At.astype(np.float64) @ At.astype(np.float64).T)


def test_nvfp4_exact_case():
    rng = np.random.default_rng(2)
    A, _ = exact_matrix(16, 64, 1, 16, rng, top=6.0, grid="e2m1", jrange=(-3, 3))
    B, _ = exact_matrix(12, 64, 1, 16, rng, top=6.0, grid="e2m1", jrange=(-3, 3))
    qa, sa, ga = Q.quantize_nvfp4_rowwise(A)
    qb, sb, gb = Q.quantize_nvfp4_rowwise(B)
    C, T = G.reference(G.dequant_nvfp4(qa, sa, ga), G.dequant_nvfp4(qb, sb, gb))
    ref = A.astype(np.float64) @ B.astype(np.float64).T
    assert np.all(np.abs(C - ref) <= 2.0 ** -22 * T)


def test_tiny_gemm_against_exact_rationals():
    d = workloads.tiny()
    A = Q.as_f32(workloads.bf16_bits(d["A"]))[:4, :256]
    W = Q.as_f32(workloads.bf16_bits(d["B"]))[:256, :128]
    qa, sa = Q.quantize_1x128_rowwise(A)
    qw, qwt, sw = Q.quantize_128x128(W)
    C, T = G.reference(G.dequant_a_1x128(qa, sa), G.dequant_b_blockwise(qwt, sw, G.FPROP))
    dec = {c: Fraction(float(v)) for c, v in enumerate(F.e4m3_decode(np.arange(256, dtype=np.uint8)))
           if not np.isnan(v)}
    for m in range(4):
        for n in (0, 77, 127):
            acc = Fraction(0)
            for k in range(256):
                a = dec[int(qa[m, k])] * Fraction(float(sa[k // 128, m]))
                b = dec[int(qwt[n, k])] * Fraction(float(sw[n // 128, k // 128]))
                acc += a * b
            assert abs(Fraction(C[m, n]) - acc) <= Fraction(2.0 ** -40) * Fraction(float(T[m, n]))


def test_tolerance_bound_accepts_bf16_rounding_and_rejects_2_pow_minus_6():
    rng = np.random.default_rng(3)
    C = rng.standard_normal((64, 64)) * 10
    T = np.abs(C) * 3
    bf16 = F.bf16_bits_to_f32(F.f32_to_bf16_bits(C.astype(np.float32))).astype(np.float64)
    assert np.all(G.tolerance_violation(bf16, C, T) <= 0)
    bad = C * (1 + 2.0 ** -5)
    assert np.any(G.tolerance_violation(bad, C, np.zeros_like(T)) > 0)


def test_sample_tiles_distinct_and_in_range():
    t = G.sample_tiles(8192, 14336, 64, seed=2)
    assert len(set(t)) == 64
    assert all(0 <= m < 8192 and 0 <= n < 14336 and m % 128 == 0 and n % 128 == 0 for m, n in t)
    counts, offs = workloads.moe_routing(seed=workloads.tensor_seed(4, 0))
    gt = G.sample_group_tiles(offs.numpy(), 2048, 64, seed=4)
    assert len(gt) == 64
    assert {g for g, *_ in gt} >= {g for g in range(32) if counts[g] > 0} or len(gt) == 64
    bt = G.sample_band_tiles(16384, 53248, 8, 8, seed=6)
    assert len(set(bt)) == 64
    assert len({m for m, _ in bt}) == 8 and len({n for _, n in bt}) == 8
    assert all(0 <= m < 16384 and 0 <= n < 53248 and m % 128 == 0 and n % 128 == 0 for m, n in bt)


def test_fine_grained_beats_per_tensor_on_wide_range():
    """NeMo page: finer scaling (blockwise, MXFP8) is more accurate than per-tensor.  The
    effect needs a dynamic range wider than E4M3's (~2^-9..448), so token magnitudes are
    spread over 2^-10..2^10 on top of the 0.1% x50 outliers."""
    d = workloads.llama8b(M=256, K=1024, N=384)
    rng = np.random.default_rng(5)
    X = Q.as_f32(workloads.bf16_bits(d["X"])) * np.exp2(rng.integers(-10, 11, (256, 1)))
    X = X.astype(np.float32)
    W = Q.as_f32(workloads.bf16_bits(d["W"]))
    ref = X.astype(np.float64) @ W.astype(np.float64)

    def err(c):
        # per-row relative error, averaged: every token counts, whatever its magnitude
        return float(np.mean(np.linalg.norm(c - ref, axis=1) / np.linalg.norm(ref, axis=1)))

    qx, sx = Q.quantize_1x128_rowwise(X)
    _, qwt, sw = Q.quantize_128x128(W)
    e_blk = err(G.reference(G.dequant_a_1x128(qx, sx),
                            G.dequant_b_blockwise(qwt, sw, G.FPROP))[0])
    qa, ea = Q.quantize_mx_rowwise(X)
    qb, eb = Q.quantize_mx_colwise(W)
    e_mx = err(G.reference(G.dequant_mx(qa, ea), G.dequant_mx(qb, eb))[0])
    qta, sta = Q.quantize_tensor(X)
    qtb, stb = Q.quantize_tensor(np.ascontiguousarray(W.T))
    e_pt = err(G.reference(G.dequant_tensor(qta, sta), G.dequant_tensor(qtb, stb))[0])
    assert 2 * e_blk < e_pt and 2 * e_mx < e_pt
